// api.cu -- the C ABI of include/w4a16.h: host-side argument checks, the M-based dispatch and
// the launches. Nothing here allocates device memory or synchronises the device.
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "tiled_layout.cuh"

using namespace w4a16;

namespace {

bool valid_group(int group) { return group == 32 || group == 64 || group == 128; }

int check_shape(int K, int N, int group) {
    if (K <= 0 || N <= 0) return W4A16_EINVAL;
    if (K % 8 != 0 || N % 8 != 0) return W4A16_EINVAL;
    if (!valid_group(group)) return W4A16_EUNSUPPORTED;
    if (K % group != 0) return W4A16_EINVAL;
    return W4A16_OK;
}

// W4A16_FORCE_KERNEL=gemv|tc, read once.
int forced_kernel() {
    static int forced = -1;
    static std::once_flag once;
    std::call_once(once, [] {
        forced = W4A16_KERNEL_AUTO;
        const char* e = getenv("W4A16_FORCE_KERNEL");
        if (e && strcmp(e, "gemv") == 0) forced = W4A16_KERNEL_GEMV;
        if (e && strcmp(e, "tc") == 0) forced = W4A16_KERNEL_TC;
    });
    return forced;
}

}  // namespace

// The limit of every bounded device wait, read by each launch (w4a16_set_wait_limit_ns).
static std::atomic<uint64_t> g_wait_limit_ns{2000000000ull};

uint64_t w4a16::wait_limit_ns() { return g_wait_limit_ns.load(std::memory_order_relaxed); }

namespace {

bool log_enabled() {
    static bool on = false;
    static std::once_flag once;
    std::call_once(once, [] {
        const char* e = getenv("W4A16_LOG");
        on = e && e[0] == '1';
    });
    return on;
}

const char* kernel_name(int k) {
    switch (k) {
        case W4A16_KERNEL_GEMV: return "gemv";
        case W4A16_KERNEL_TC: return "tc";
        default: return "auto";
    }
}

// The dispatch proper (tiled layout), without the environment override. For small M the layer is
// bound by the weight stream and the stream-K decode GEMV serves it (over K slices when the M rows
// of A do not fit in its shared memory at once); above, the tensor-core GEMM. Measured on the
// (8192, 28672), (28672, 8192) and (4096, 28672) layers (bf16, g128): for M <= 8 the decode kernel
// beats the tensor-core GEMM (1.2-1.6x) whether K is held whole or in slices; for M = 9..16 (two
// 8-row MMA tiles) it wins only when K is held whole, and is 1.7-2.2x slower when K needs slices.
int dispatch(int M, int N, int K, int group) {
    if (M > 16) return W4A16_KERNEL_TC;
    if (M <= 8) return W4A16_KERNEL_GEMV;
    int n_sm = gemv_stream_sm_count();
    if (n_sm <= 0) n_sm = 148;
    const GemvStreamPlan q = plan_gemv_stream(M, N, K, group, 0, n_sm);
    return q.ok && q.slices == 1 ? W4A16_KERNEL_GEMV : W4A16_KERNEL_TC;
}

}  // namespace

extern "C" {

W4A16_API int w4a16_version(void) { return 200; }

W4A16_API uint64_t w4a16_set_wait_limit_ns(uint64_t ns) {
    const uint64_t v = ns == 0 ? 2000000000ull : ns;
    return g_wait_limit_ns.exchange(v, std::memory_order_relaxed);
}

W4A16_API const char* w4a16_status_str(int status) {
    switch (status) {
        case W4A16_OK: return "W4A16_OK";
        case W4A16_EINVAL: return "W4A16_EINVAL";
        case W4A16_EALIGN: return "W4A16_EALIGN";
        case W4A16_EUNSUPPORTED: return "W4A16_EUNSUPPORTED";
        case W4A16_ENONFINITE: return "W4A16_ENONFINITE";
        case W4A16_EWORKSPACE: return "W4A16_EWORKSPACE";
        case W4A16_ECUDA: return "W4A16_ECUDA";
        case W4A16_ETIMEOUT: return "W4A16_ETIMEOUT";
        default: return "W4A16_UNKNOWN";
    }
}

W4A16_API int w4a16_quantize(const void* W, int K, int N, int group, int sym, int32_t* codes,
                             void* scales, int32_t* zeros, int* dev_status, void* stream) {
    int st = check_shape(K, N, group);
    if (st != W4A16_OK) return st;
    if (sym != 0 && sym != 1) return W4A16_EINVAL;
    if (!W || !codes || !scales) return W4A16_EINVAL;
    if (sym ? zeros != nullptr : zeros == nullptr) return W4A16_EINVAL;
    if (!aligned16(W) || !aligned16(codes) || !aligned16(scales) || (zeros && !aligned16(zeros)))
        return W4A16_EALIGN;
    return launch_quantize(W, K, N, group, sym, codes, scales, zeros, dev_status,
                           static_cast<cudaStream_t>(stream));
}

W4A16_API int w4a16_dequantize(const int32_t* codes, const void* scales, const int32_t* zeros, int K, int N,
                               int group, int sym, int out_dtype, void* W, void* stream) {
    int st = check_shape(K, N, group);
    if (st != W4A16_OK) return st;
    if (sym != 0 && sym != 1) return W4A16_EINVAL;
    if (out_dtype != W4A16_F16 && out_dtype != W4A16_BF16) return W4A16_EINVAL;
    if (!codes || !scales || !W) return W4A16_EINVAL;
    if (sym ? zeros != nullptr : zeros == nullptr) return W4A16_EINVAL;
    if (!aligned16(codes) || !aligned16(scales) || !aligned16(W) || (zeros && !aligned16(zeros)))
        return W4A16_EALIGN;
    return launch_dequantize(codes, scales, zeros, K, N, group, sym, out_dtype, W,
                             static_cast<cudaStream_t>(stream));
}

W4A16_API size_t w4a16_gptq_workspace_bytes(int K, int N) {
    if (K <= 0 || N <= 0) return 0;
    return gptq_workspace_bytes(K, N);
}

W4A16_API int w4a16_gptq_quantize(const void* W, const void* X, int x_dtype, int S, int K, int N, int group,
                                  int sym, double damp, int32_t* codes, void* scales, int32_t* zeros,
                                  void* workspace, size_t ws_bytes, int* dev_status, void* stream) {
    int st = check_shape(K, N, group);
    if (st != W4A16_OK) return st;
    if (sym != 0 && sym != 1) return W4A16_EINVAL;
    if (x_dtype != W4A16_F16 && x_dtype != W4A16_BF16) return W4A16_EINVAL;
    if (S < 1 || !(damp >= 0.0) || !(damp < 1e30)) return W4A16_EINVAL;
    if (!W || !X || !codes || !scales || !workspace) return W4A16_EINVAL;
    if (sym ? zeros != nullptr : zeros == nullptr) return W4A16_EINVAL;
    if (!aligned16(W) || !aligned16(X) || !aligned16(codes) || !aligned16(scales) || !aligned16(workspace) ||
        (zeros && !aligned16(zeros)))
        return W4A16_EALIGN;
    if (ws_bytes < gptq_workspace_bytes(K, N)) return W4A16_EWORKSPACE;
    return launch_gptq(W, X, x_dtype, S, K, N, group, sym, damp, codes, scales, zeros, workspace, dev_status,
                       static_cast<cudaStream_t>(stream));
}

W4A16_API size_t w4a16_awq_workspace_bytes(int K, int N, int S) {
    if (K <= 0 || N <= 0 || S <= 0) return 0;
    return awq_workspace_bytes(K, N, S);
}

W4A16_API int w4a16_awq_quantize(const void* W, const void* X, int x_dtype, int S, int K, int N, int group,
                                 int sym, int32_t* codes, void* scales, int32_t* zeros, void* s_in,
                                 void* workspace, size_t ws_bytes, int* dev_status, void* stream) {
    int st = check_shape(K, N, group);
    if (st != W4A16_OK) return st;
    if (sym != 0 && sym != 1) return W4A16_EINVAL;
    if (x_dtype != W4A16_F16 && x_dtype != W4A16_BF16) return W4A16_EINVAL;
    if (S < 1) return W4A16_EINVAL;
    if (!W || !X || !codes || !scales || !s_in || !workspace) return W4A16_EINVAL;
    if (sym ? zeros != nullptr : zeros == nullptr) return W4A16_EINVAL;
    if (!aligned16(W) || !aligned16(X) || !aligned16(codes) || !aligned16(scales) || !aligned16(s_in) ||
        !aligned16(workspace) || (zeros && !aligned16(zeros)))
        return W4A16_EALIGN;
    if (ws_bytes < awq_workspace_bytes(K, N, S)) return W4A16_EWORKSPACE;
    return launch_awq(W, X, x_dtype, S, K, N, group, sym, codes, scales, zeros, s_in, workspace, dev_status,
                      static_cast<cudaStream_t>(stream));
}

W4A16_API int w4a16_fp8_quantize_weights(const void* W, int K, int N, uint8_t* Wq, float* w_scales, void* stream) {
    if (K <= 0 || N <= 0 || K % 128 != 0 || N % 128 != 0) return K > 0 && N > 0 ? W4A16_EUNSUPPORTED : W4A16_EINVAL;
    if (!W || !Wq || !w_scales) return W4A16_EINVAL;
    if (!aligned16(W) || !aligned16(Wq) || !aligned16(w_scales)) return W4A16_EALIGN;
    return launch_fp8_quantize_weights(W, K, N, Wq, w_scales, static_cast<cudaStream_t>(stream));
}

W4A16_API int w4a16_fp8_quantize_acts(const void* A, int a_dtype, int M, int K, uint8_t* Aq, float* a_scales,
                                      void* stream) {
    if (M < 1 || K <= 0) return W4A16_EINVAL;
    if (K % 128 != 0) return W4A16_EUNSUPPORTED;
    if (a_dtype != W4A16_F16 && a_dtype != W4A16_BF16) return W4A16_EINVAL;
    if (!A || !Aq || !a_scales) return W4A16_EINVAL;
    if (!aligned16(A) || !aligned16(Aq) || !aligned16(a_scales)) return W4A16_EALIGN;
    return launch_fp8_quantize_acts(A, a_dtype, M, K, Aq, a_scales, static_cast<cudaStream_t>(stream));
}

W4A16_API int w4a16_fp8_gemm(const uint8_t* Aq, const float* a_scales, int M, int K, const uint8_t* Wq,
                             const float* w_scales, int N, void* C, int c_dtype, int* dev_status, void* stream) {
    if (M < 1 || K <= 0 || N <= 0) return W4A16_EINVAL;
    if (K % 128 != 0 || N % 128 != 0) return W4A16_EUNSUPPORTED;
    if (c_dtype != W4A16_F16 && c_dtype != W4A16_BF16) return W4A16_EINVAL;
    if (!Aq || !a_scales || !Wq || !w_scales || !C) return W4A16_EINVAL;
    if (!aligned16(Aq) || !aligned16(Wq) || !aligned16(C) || !aligned16(a_scales) || !aligned16(w_scales))
        return W4A16_EALIGN;
    return launch_fp8_gemm(Aq, a_scales, M, K, Wq, w_scales, N, C, c_dtype, dev_status,
                           static_cast<cudaStream_t>(stream));
}

W4A16_API size_t w4a16_repack_bytes(int K, int N, int group, int sym) {
    if (check_shape(K, N, group) != W4A16_OK || (sym != 0 && sym != 1)) return 0;
    if (N % kTileN != 0 || K % kTileK != 0) return 0;
    return tiled_layout(K, N, group, sym).total;
}

W4A16_API int w4a16_repack(const int32_t* codes, const void* scales, const int32_t* zeros, int K,
                           int N, int group, int sym, void* tiled, void* stream) {
    int st = check_shape(K, N, group);
    if (st != W4A16_OK) return st;
    if (sym != 0 && sym != 1) return W4A16_EINVAL;
    if (N % kTileN != 0 || K % kTileK != 0) return W4A16_EUNSUPPORTED;
    if (!codes || !scales || !tiled) return W4A16_EINVAL;
    if (sym ? zeros != nullptr : zeros == nullptr) return W4A16_EINVAL;
    if (!aligned16(codes) || !aligned16(scales) || !aligned16(tiled) || (zeros && !aligned16(zeros)))
        return W4A16_EALIGN;
    return launch_repack(codes, scales, zeros, K, N, group, sym, tiled,
                         static_cast<cudaStream_t>(stream));
}

W4A16_API int w4a16_select_kernel(int M, int N, int K, int group) {
    const int f = forced_kernel();
    if (f != W4A16_KERNEL_AUTO) return f;
    return dispatch(M, N, K, group);
}

W4A16_API size_t w4a16_workspace_bytes(int M, int N, int K, int group) {
    if (M < 1 || check_shape(K, N, group) != W4A16_OK) return 0;
    // the largest need over every kernel a call may run, so a forced kernel also fits; the tile
    // counters of the stream-K kernel come first and are always reserved
    const GemvPlan p = plan_gemv_plain(M, N, K, group);
    int n_sm = gemv_stream_sm_count();
    if (n_sm <= 0) n_sm = 148;
    const GemvStreamPlan q = plan_gemv_stream(M, N, K, group, 0, n_sm);   // asymmetric: the larger plan
    size_t rest = q.ok && q.partial_bytes > p.ws_bytes ? q.partial_bytes : p.ws_bytes;
    const TcPlan t = plan_gemm_tc(M, N, K, group, 0, n_sm);
    if (t.ok && t.partial_bytes > rest) rest = t.partial_bytes;
    return kGemvStreamCounterBytes + rest;
}

W4A16_API int w4a16_gemm(const void* A, int a_dtype, int M, int K, const void* wq, int layout,
                         const void* scales, const int32_t* zeros, int N, int group, int sym,
                         void* C, void* workspace, size_t ws_bytes, int kernel, int* dev_status,
                         void* stream) {
    int st = check_shape(K, N, group);
    if (st != W4A16_OK) return st;
    if (M < 1) return W4A16_EINVAL;
    if (a_dtype != W4A16_F16 && a_dtype != W4A16_BF16) return W4A16_EINVAL;
    if (layout != W4A16_LAYOUT_PLAIN && layout != W4A16_LAYOUT_TILED) return W4A16_EINVAL;
    if (sym != 0 && sym != 1) return W4A16_EINVAL;
    if (kernel != W4A16_KERNEL_AUTO && kernel != W4A16_KERNEL_GEMV && kernel != W4A16_KERNEL_TC)
        return W4A16_EINVAL;
    if (!A || !wq || !C) return W4A16_EINVAL;
    if (layout == W4A16_LAYOUT_PLAIN) {
        if (!scales) return W4A16_EINVAL;
        if (sym ? zeros != nullptr : zeros == nullptr) return W4A16_EINVAL;
        if (!aligned16(scales) || (zeros && !aligned16(zeros))) return W4A16_EALIGN;
    } else if (N % kTileN != 0 || K % kTileK != 0) {
        return W4A16_EUNSUPPORTED;
    }
    if (!aligned16(A) || !aligned16(wq) || !aligned16(C)) return W4A16_EALIGN;
    const size_t need = w4a16_workspace_bytes(M, N, K, group);
    if (ws_bytes < need || (need > 0 && !workspace)) return W4A16_EWORKSPACE;
    if (workspace && !aligned16(workspace)) return W4A16_EALIGN;
    // partial sums of the split-K kernels live after the stream-K tile counters
    void* scratch = static_cast<char*>(workspace) + kGemvStreamCounterBytes;

    int chosen = kernel == W4A16_KERNEL_AUTO ? w4a16_select_kernel(M, N, K, group) : kernel;
    // the plain layout has only the CUDA-core kernel
    if (kernel == W4A16_KERNEL_AUTO && layout == W4A16_LAYOUT_PLAIN) chosen = W4A16_KERNEL_GEMV;
    if (log_enabled())
        fprintf(stderr, "[w4a16] gemm M=%d N=%d K=%d g=%d sym=%d layout=%d -> %s\n", M, N, K, group,
                sym, layout, kernel_name(chosen));
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    if (chosen == W4A16_KERNEL_GEMV && layout == W4A16_LAYOUT_PLAIN) {
        const GemvPlan p = plan_gemv_plain(M, N, K, group);
        const size_t elt = 2;
        for (int m0 = 0; m0 < M; m0 += p.mt) {
            const int mc = (M - m0) < p.mt ? (M - m0) : p.mt;
            st = launch_gemv_plain(static_cast<const char*>(A) + (size_t)m0 * K * elt, a_dtype, mc, K,
                                   static_cast<const int32_t*>(wq), scales, zeros, N, group, sym,
                                   static_cast<char*>(C) + (size_t)m0 * N * elt, scratch, p, s);
            if (st != W4A16_OK) return st;
        }
        return W4A16_OK;
    }
    if (chosen == W4A16_KERNEL_GEMV && layout == W4A16_LAYOUT_TILED) {
        st = launch_gemv_stream(A, a_dtype, M, K, wq, N, group, sym, C, workspace, dev_status, s);
        // M > 16, or M rows of A too long for shared memory: the tensor-core kernel
        if (st == W4A16_EUNSUPPORTED && kernel == W4A16_KERNEL_AUTO)
            return launch_gemm_tc(A, a_dtype, M, K, wq, N, group, sym, C, workspace, dev_status, s);
        return st;
    }
    if (chosen == W4A16_KERNEL_TC && layout == W4A16_LAYOUT_TILED) {
        return launch_gemm_tc(A, a_dtype, M, K, wq, N, group, sym, C, workspace, dev_status, s);
    }
    return W4A16_EUNSUPPORTED;
}

}  // extern "C"
