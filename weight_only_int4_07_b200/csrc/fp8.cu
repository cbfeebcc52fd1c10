// fp8.cu -- the W8A8 comparison path: FP8 (E4M3) weights and activations into a tcgen05
// kind::f8f6f4 GEMM.
//
// "INT8 vs INT4 Quantization, in depth", section "Two regimes: waiting for memory, waiting for
// math" and its worked example: an 8-bit path reads twice the weight bytes of W4A16 but runs the
// multiply at twice the 16-bit tensor rate, so W4A16 wins while the layer waits for memory and
// the 8-bit path once it waits for math; this path is what the crossover is measured against.
// Readings (the pages fix neither format nor scaling): E4M3 codes, one FP32 scale per output
// channel (weights) and per row (activations), s = fp32(amax / 448) (1 when amax = 0), codes =
// E4M3 round-to-nearest-even of x / s computed in FP64, saturated to +-448;
// y[m, n] = (sum_k qa[m, k] qw[n, k]) s_a[m] s_w[n] with FP32 accumulation.
//
// GEMM mapping (as the W4A16 tensor-core kernel, without the dequant warps): D[n, m] =
// sum_k Wq[n, k] Aq[m, k] with the weight tile (128 output channels x 128 K bytes) as operand A
// and the activation tile (BN rows x 128 K bytes) as operand B, both loaded by TMA with the
// 128-byte swizzle; four MMAs of K = 32 per stage; D (FP32) in tensor memory.
// Warps: 0 issues the TMA loads, 1 owns tensor memory and issues the MMAs, 2..5 read D back,
// apply both scales and store C. Every mbarrier wait is bounded (2 s): on expiry the kernel
// records W4A16_ETIMEOUT and every role drains and returns, freeing its tensor memory.
#include <cuda_fp8.h>
#include <cudaTypedefs.h>

#include <mutex>
#include <type_traits>

#include "common.cuh"
#include "sm100_ptx.cuh"

namespace w4a16 {

bool make_u8_map(CUtensorMap* map, const void* base, int rows, int K, int box_rows);

namespace {

using namespace sm100;

constexpr uint64_t kFp8Spin = 2000000000ull;
constexpr int kFp8Threads = 192;

__device__ __forceinline__ double f16_bits_to_f64(uint16_t h) {
    return (double)__half2float(__ushort_as_half(h));
}

template <typename T>
__device__ __forceinline__ double act_to_f64(uint16_t bits) {
    if constexpr (std::is_same<T, __half>::value) return (double)__half2float(__ushort_as_half(bits));
    return (double)__uint_as_float((uint32_t)bits << 16);
}

__device__ __forceinline__ uint8_t e4m3_rn(double x) {
    return (uint8_t)__nv_cvt_double_to_fp8(x, __NV_SATFINITE, __NV_E4M3);
}

__device__ __forceinline__ float scale_from_amax(double amax) {
    const float s = (float)(amax / 448.0);
    return s == 0.0f ? 1.0f : s;
}

// s_w[n] from the column maximum of W [K, N] (one thread per column).
__global__ void __launch_bounds__(256) fp8_wscale_kernel(const uint16_t* __restrict__ W, int K, int N,
                                                         float* __restrict__ sw) {
    const int n = blockIdx.x * 256 + threadIdx.x;
    if (n >= N) return;
    double amax = 0.0;
    for (int k = 0; k < K; ++k) amax = fmax(amax, fabs(f16_bits_to_f64(W[(size_t)k * N + n])));
    sw[n] = scale_from_amax(amax);
}

// Wq[n, k] = e4m3(W[k, n] / s_w[n]): 32 x 32 tiles through shared memory (reads along n, writes
// along k).
__global__ void __launch_bounds__(256) fp8_wquant_kernel(const uint16_t* __restrict__ W, const float* __restrict__ sw,
                                                         int K, int N, uint8_t* __restrict__ Wq) {
    __shared__ uint8_t t[32][33];
    const int k0 = blockIdx.y * 32, n0 = blockIdx.x * 32;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
    for (int r = ty; r < 32; r += 8) {
        const int k = k0 + r, n = n0 + tx;
        t[r][tx] = e4m3_rn(f16_bits_to_f64(W[(size_t)k * N + n]) / (double)sw[n]);
    }
    cta_sync();
    for (int r = ty; r < 32; r += 8) Wq[(size_t)(n0 + r) * K + k0 + tx] = t[tx][r];
}

// One CTA per activation row: s_a[m] from the row maximum, then Aq[m, k] = e4m3(A[m, k] / s_a[m]).
template <typename T>
__global__ void __launch_bounds__(256) fp8_aquant_kernel(const uint16_t* __restrict__ A, int K, uint8_t* __restrict__ Aq,
                                                         float* __restrict__ sa) {
    __shared__ double red[256];
    const int m = blockIdx.x;
    const uint16_t* row = A + (size_t)m * K;
    double amax = 0.0;
    for (int k = threadIdx.x; k < K; k += 256) amax = fmax(amax, fabs(act_to_f64<T>(row[k])));
    red[threadIdx.x] = amax;
    cta_sync();
    for (int w = 128; w > 0; w >>= 1) {
        if (threadIdx.x < w) red[threadIdx.x] = fmax(red[threadIdx.x], red[threadIdx.x + w]);
        cta_sync();
    }
    const float s = scale_from_amax(red[0]);
    if (threadIdx.x == 0) sa[m] = s;
    for (int k = threadIdx.x; k < K; k += 256) Aq[(size_t)m * K + k] = e4m3_rn(act_to_f64<T>(row[k]) / (double)s);
}

template <int BN>
struct Fp8Cfg {
    static constexpr int kA = 128 * 128;   // weight tile: 128 channels x 128 K bytes
    static constexpr int kB = BN * 128;    // activation tile
    static constexpr int kStage = kA + kB;
    static constexpr int kBudget = 227 * 1024 - 1024 - 256;
    static constexpr int kStagesRaw = kBudget / kStage;
    static constexpr int kStages = kStagesRaw > 8 ? 8 : kStagesRaw;
    static constexpr int kTmemCols = BN < 32 ? 32 : BN;
    static constexpr int kSmem = kStages * kStage + 1024 + 256;
    static_assert(kStages >= 2, "pipeline needs two stages");
};

template <int BN, typename T>
__global__ void __launch_bounds__(kFp8Threads, 1)
fp8_gemm_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmA,
                const float* __restrict__ sw, const float* __restrict__ sa, int M, int K, int N, T* __restrict__ C,
                int* dev_status) {
    using Cfg = Fp8Cfg<BN>;
    constexpr int NS = Cfg::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + NS * Cfg::kStage);
    uint64_t* empty = full + NS;
    uint64_t* accfull = empty + NS;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accfull + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * 128, m0 = blockIdx.y * BN;
    const int kstages = K / 128;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accfull, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, Cfg::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    cta_sync();
    tc_fence_after();
    const uint32_t tmem_d = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            prefetch_tensormap(&tmW);
            prefetch_tensormap(&tmA);
            int issued = 0;
            for (int it = 0; it < kstages; ++it) {
                const int s = it % NS;
                const uint32_t r = (uint32_t)(it / NS);
                if (!mbar_wait(&empty[s], (r & 1u) ^ 1u, abort_flag, dev_status, kFp8Spin)) break;
                uint8_t* st = smem + s * Cfg::kStage;
                mbar_arrive_expect_tx(&full[s], (uint32_t)Cfg::kStage);
                tma_2d_g2s(st, &tmW, it * 128, n0, &full[s]);
                tma_2d_g2s(st + Cfg::kA, &tmA, it * 128, m0, &full[s]);
                ++issued;
            }
            for (int it = (issued > NS ? issued - NS : 0); it < issued; ++it)
                mbar_wait(&full[it % NS], (uint32_t)(it / NS) & 1u, abort_flag, dev_status, kFp8Spin);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_f16(BN, false);   // E4M3 = format 0 for A and B
            for (int it = 0; it < kstages; ++it) {
                const int s = it % NS;
                if (!mbar_wait(&full[s], (uint32_t)(it / NS) & 1u, abort_flag, dev_status, kFp8Spin)) break;
                tc_fence_after();
                const uint32_t a_base = smem_u32(smem + s * Cfg::kStage);
                mma4_f8_ss_commit(tmem_d, smem_desc_sw128(a_base), smem_desc_sw128(a_base + Cfg::kA), idesc,
                                  it > 0 ? 1u : 0u, &empty[s]);
            }
            mma_commit(accfull);
        }
    } else {
        const int q = warp & 3;              // tensor-memory lane quarter of this warp
        const int n = 32 * q + lane;         // output channel within the tile
        if (mbar_wait(accfull, 0, abort_flag, dev_status, kFp8Spin) && !*abort_flag) {
            tc_fence_after();
            const float swn = sw[n0 + n];
            const uint32_t lane_base = tmem_d + ((uint32_t)(32 * q) << 16);
            constexpr int kChunks = BN / 16 > 0 ? BN / 16 : 1;
#pragma unroll 1
            for (int c = 0; c < kChunks; ++c) {
                uint32_t v[16];
                tmem_ld16(lane_base + c * 16, v);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int m = m0 + c * 16 + i;
                    if (m < M) C[(size_t)m * N + n0 + n] = Act<T>::from_f32(__uint_as_float(v[i]) * swn * sa[m]);
                }
            }
        }
    }

    tc_fence_before();
    cta_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_d, Cfg::kTmemCols);
    }
}

template <int BN, typename T>
int launch_fp8_typed(const uint8_t* Aq, const float* sa, int M, int K, const uint8_t* Wq, const float* sw, int N,
                     void* C, int* dev_status, cudaStream_t stream) {
    using Cfg = Fp8Cfg<BN>;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(fp8_gemm_kernel<BN, T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        Cfg::kSmem);
    });
    if (attr_err != cudaSuccess) return W4A16_ECUDA;
    CUtensorMap mw, ma;
    if (!make_u8_map(&mw, Wq, N, K, 128) || !make_u8_map(&ma, Aq, M, K, BN)) return W4A16_ECUDA;
    dim3 grid(N / 128, (M + BN - 1) / BN);
    fp8_gemm_kernel<BN, T><<<grid, kFp8Threads, Cfg::kSmem, stream>>>(mw, ma, sw, sa, M, K, N, static_cast<T*>(C),
                                                                     dev_status);
    return launch_status();
}

template <typename T>
int launch_fp8_bn(const uint8_t* Aq, const float* sa, int M, int K, const uint8_t* Wq, const float* sw, int N,
                  void* C, int* dev_status, cudaStream_t stream) {
    if (M <= 16) return launch_fp8_typed<16, T>(Aq, sa, M, K, Wq, sw, N, C, dev_status, stream);
    if (M <= 32) return launch_fp8_typed<32, T>(Aq, sa, M, K, Wq, sw, N, C, dev_status, stream);
    if (M <= 64) return launch_fp8_typed<64, T>(Aq, sa, M, K, Wq, sw, N, C, dev_status, stream);
    if (M <= 128) return launch_fp8_typed<128, T>(Aq, sa, M, K, Wq, sw, N, C, dev_status, stream);
    return launch_fp8_typed<256, T>(Aq, sa, M, K, Wq, sw, N, C, dev_status, stream);
}

}  // namespace

int launch_fp8_quantize_weights(const void* W, int K, int N, uint8_t* Wq, float* sw, cudaStream_t stream) {
    const uint16_t* Wb = static_cast<const uint16_t*>(W);
    fp8_wscale_kernel<<<(N + 255) / 256, 256, 0, stream>>>(Wb, K, N, sw);
    fp8_wquant_kernel<<<dim3(N / 32, K / 32), 256, 0, stream>>>(Wb, sw, K, N, Wq);
    return launch_status();
}

int launch_fp8_quantize_acts(const void* A, int a_dtype, int M, int K, uint8_t* Aq, float* sa, cudaStream_t stream) {
    const uint16_t* Ab = static_cast<const uint16_t*>(A);
    if (a_dtype == W4A16_BF16)
        fp8_aquant_kernel<__nv_bfloat16><<<M, 256, 0, stream>>>(Ab, K, Aq, sa);
    else
        fp8_aquant_kernel<__half><<<M, 256, 0, stream>>>(Ab, K, Aq, sa);
    return launch_status();
}

int launch_fp8_gemm(const uint8_t* Aq, const float* sa, int M, int K, const uint8_t* Wq, const float* sw, int N,
                    void* C, int c_dtype, int* dev_status, cudaStream_t stream) {
    if (c_dtype == W4A16_BF16)
        return launch_fp8_bn<__nv_bfloat16>(Aq, sa, M, K, Wq, sw, N, C, dev_status, stream);
    return launch_fp8_bn<__half>(Aq, sa, M, K, Wq, sw, N, C, dev_status, stream);
}

}  // namespace w4a16
