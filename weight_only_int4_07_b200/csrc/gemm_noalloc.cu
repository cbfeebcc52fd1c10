// gemm_noalloc.cu -- w4a16_gemm_noalloc: the plain-layout split-K GEMV for callers that cannot
// allocate device memory.
//
// w4a16_gemm asks its caller for a workspace (the split-K partial sums). Some callers have no
// way to provide one: a plugin inside a host application that owns every device allocation and
// forbids allocations outside its own pool, or a latency-critical loop that must never call
// cudaMalloc (which can block and synchronise the whole device). This entry point serves them:
// the partial sums live in one static device array of this library, g_noalloc_scratch, which the
// CUDA driver reserves on every GPU that loads the library and keeps until the process exits.
//
// Nothing here calls cudaMalloc, cudaFree or any allocating routine. The array's name is only a
// host-side stand-in in host code; its device address is looked up by cudaGetSymbolAddress, with
// the caller's device current, on every call, and passed to the kernels.
#include "common.cuh"

namespace w4a16 {
namespace {

// Capacity of the shared scratch: the split-K partial sums of one call, splits x min(M, 16) x N
// FP32 values, must fit.
constexpr size_t kNoallocScratchBytes = size_t(8) << 20;  // 8 MiB

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

// Device address of g_noalloc_scratch on the current device. Looked up on every call (a cheap
// runtime query): a cached address would go stale if the device's primary context were
// destroyed and created again (cudaDeviceReset), since the module, and the array with it, is
// then loaded anew and may land elsewhere.
int scratch_on_current_device(void** addr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return W4A16_ECUDA;
    *addr = p;
    return W4A16_OK;
}

bool aligned(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace w4a16

using namespace w4a16;

extern "C" W4A16_API int w4a16_gemm_noalloc(const void* A, int a_dtype, int M, int K,
                                            const int32_t* codes, const void* scales,
                                            const int32_t* zeros, int N, int group, int sym,
                                            void* C, void* stream) {
    if (K <= 0 || N <= 0 || M < 1 || K % 8 != 0 || N % 8 != 0) return W4A16_EINVAL;
    if (group != 32 && group != 64 && group != 128) return W4A16_EUNSUPPORTED;
    if (K % group != 0) return W4A16_EINVAL;
    if (a_dtype != W4A16_F16 && a_dtype != W4A16_BF16) return W4A16_EINVAL;
    if (sym != 0 && sym != 1) return W4A16_EINVAL;
    if (!A || !codes || !scales || !C) return W4A16_EINVAL;
    if (sym ? zeros != nullptr : zeros == nullptr) return W4A16_EINVAL;
    if (!aligned(A) || !aligned(codes) || !aligned(scales) || !aligned(C) || (zeros && !aligned(zeros)))
        return W4A16_EALIGN;

    const GemvPlan plan = plan_gemv_plain(M, N, K, group);
    if (plan.ws_bytes > kNoallocScratchBytes) return W4A16_EWORKSPACE;  // beyond the static scratch

    void* scratch = nullptr;
    int st = scratch_on_current_device(&scratch);
    if (st != W4A16_OK) return st;

    // Every partial sum the reduce kernel reads is written first by the GEMV kernel of the same
    // call, so nothing in the scratch has to start at zero.
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t elt = 2;
    for (int m0 = 0; m0 < M; m0 += plan.mt) {
        const int mc = (M - m0) < plan.mt ? (M - m0) : plan.mt;
        st = launch_gemv_plain(static_cast<const char*>(A) + (size_t)m0 * K * elt, a_dtype, mc, K, codes,
                               scales, zeros, N, group, sym, static_cast<char*>(C) + (size_t)m0 * N * elt,
                               scratch, plan, s);
        if (st != W4A16_OK) return st;
    }
    return W4A16_OK;
}
