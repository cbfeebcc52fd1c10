// gemm_skinny.cu -- split-K tcgen05 W4A16 kernel for decode-sized M (1..16) on the tiled layout.
//
// C[m, n] = sum_g s[g, n] * sum_{k in g} A[m, k] * (u[k, n] - z[g, n]), FP32 accumulation.
// "4.3 Weight-only INT4", section 4: read, unpack, dequantize and multiply in one pipeline so each
// weight byte crosses HBM once; "INT8 vs INT4 Quantization, in depth", "Two regimes": at small
// batch the layer waits for memory, so the kernel is built to stream the codes at HBM rate.
//
// Why tensor cores at M = 1: at the measured 6.5 TB/s a B200 SM must consume about 45 weights per
// clock. An exact FP32-accumulating dot on CUDA cores costs about 2.5 issue slots per weight
// (unpack, convert, subtract, multiply-add); here a weight costs about 1.4 (one shift+mask pair
// and one packed subtract per two weights) and the products and sums run on the tensor core.
// The integer weights (u - z) are exact in fp16/bf16 and the scale is applied per group in FP32,
// so no weight is ever rounded.
//
// Per CTA: 128 output channels x a K range (split-K over a thread-block cluster of S CTAs), in
// stages of 128 K (two 4 KiB code tiles).
//   warp 0      producer: per stage, two TMA loads of the activation tile (16 rows x 64 K each,
//               128-byte swizzle, rows past M read as zero), one bulk copy of the 8 KiB of codes and
//               bulk copies of the stage's zero-points.
//   warp 1      allocates 256 TMEM columns; one thread issues, per stage and in one instruction
//               sequence, the eight tcgen05.mma (M = 128 channels, N = 16 rows of A, K = 16,
//               operand A read from TMEM) into one accumulator per group, and two commits. (An
//               issuing thread stalls for hundreds of cycles between separately issued sequences,
//               which would cap the kernel well below the HBM rate at this small N.)
//   warps 2..9  dequant: two warps per 32 channels, one per 64-K tile of the stage. A thread first
//               drains its TMEM slot's accumulators from the slot's previous use (tcgen05.ld, then
//               s[g, n] * D added into FP32 registers), then turns its 64 codes into exact 16-bit
//               integers (u - z) -- a half2/bf162 "magic" OR plus one packed subtract per pair --
//               and writes them into the slot's A region with tcgen05.st.
// At the end the two warps of a channel group add their sums, and the S CTAs of the cluster add
// their partial sums through distributed shared memory in rank order and store C.
// TMEM: NSLOT slots of (64 A columns + 16 columns per group of the stage); 256 columns allocated.
// At least 77 KiB of shared memory per CTA keeps at most two CTAs on an SM, so tcgen05.alloc never
// waits (a wait could deadlock the CTAs of a cluster).
// Every mbarrier wait is bounded (2 s); on expiry W4A16_ETIMEOUT is recorded and all roles drain.
#include <cudaTypedefs.h>

#include <mutex>
#include <type_traits>

#include "common.cuh"
#include "sm100_ptx.cuh"
#include "tiled_layout.cuh"

namespace w4a16 {

// defined in gemm_tc.cu
bool make_act_map(CUtensorMap* map, const void* A, int M, int K, int box_rows, bool bf16);

namespace {

using namespace sm100;

constexpr int kSkThreads = 320;       // 10 warps
constexpr int kSkDeqWarps = 8;
constexpr int kSkNS = 6;              // shared-memory stages of 128 K
constexpr int kSkActs = 4096;         // two 16 x 64 activation boxes (each 1024-aligned)
constexpr int kSkCodes = 8192;        // two code tiles
constexpr int kSkStage = kSkActs + kSkCodes + 1024;  // + zeros (<= 256 B), keeps 1024 alignment
constexpr int kSkRed = 2 * 16 * 128 * 4;
constexpr int kSkSmem = 1024 + kSkNS * kSkStage + kSkRed + 512;
constexpr int kSkTmemCols = 256;
constexpr uint64_t kSkSpin = 2000000000ull;
// 228 KiB of shared memory per SM, 1 KiB reserved per CTA: three CTAs of this size cannot fit
static_assert(3 * (kSkSmem + 1024) > 228 * 1024, "shared memory bounds the CTAs per SM (TMEM budget)");

template <int GROUP>
struct SkCfg {
    static constexpr int kG = 128 / GROUP;                 // groups per stage: 1, 2 or 4
    static constexpr int kSlot = 64 + 16 * kG;             // TMEM columns per slot
    static constexpr int kNSlot = GROUP == 128 ? 3 : 2;    // TMEM slots
    static constexpr int kGPerHalf = kG >= 2 ? kG / 2 : 1; // groups drained by one dequant warp
    static_assert(kNSlot * kSlot <= kSkTmemCols, "TMEM slots exceed the allocation");
};

template <typename T>
struct Sub;

template <>
struct Sub<__half> {
    static constexpr uint32_t kMagic = 0x64006400u;  // 1024 + u
    __half2 zz;
    __device__ __forceinline__ void set(int z) { zz = __half2half2(__ushort_as_half((unsigned short)(0x6400 + z))); }
    __device__ __forceinline__ uint32_t pair(uint32_t x) const {
        __half2 h = *reinterpret_cast<__half2*>(&x);
        __half2 r = __hsub2(h, zz);
        return *reinterpret_cast<uint32_t*>(&r);
    }
};

template <>
struct Sub<__nv_bfloat16> {
    static constexpr uint32_t kMagic = 0x43004300u;  // 128 + u
    __nv_bfloat162 zz;
    __device__ __forceinline__ void set(int z) {
        zz = __bfloat162bfloat162(__ushort_as_bfloat16((unsigned short)(0x4300 + z)));
    }
    __device__ __forceinline__ uint32_t pair(uint32_t x) const {
        __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&x);
        __nv_bfloat162 r = __hsub2(h, zz);
        return *reinterpret_cast<uint32_t*>(&r);
    }
};

// The stage's eight MMAs (K = 8 x 16 = 128) with operand A in TMEM and B in shared memory (two
// 64-K boxes), then the commits of the shared-memory stage and of the TMEM slot. The first MMA of
// each group overwrites its accumulator (predicate f), the others accumulate (predicate t).
// d0..d3: accumulators of the stage's groups (group of MMA kk = kk / (8 / G)).
#define W4A16_MMA8(P0, P1, P2, P3, P4, P5, P6, P7, D0, D1, D2, D3, D4, D5, D6, D7)                          \
    "{\n\t.reg .pred f, t;\n\t"                                                                               \
    "setp.ne.b32 f, %4, %4;\n\t"                                                                              \
    "setp.eq.b32 t, %4, %4;\n\t"                                                                              \
    "tcgen05.mma.cta_group::1.kind::f16 [" D0 "], [%7], %15, %4, " P0 ";\n\t"                                \
    "tcgen05.mma.cta_group::1.kind::f16 [" D1 "], [%8], %16, %4, " P1 ";\n\t"                                \
    "tcgen05.mma.cta_group::1.kind::f16 [" D2 "], [%9], %17, %4, " P2 ";\n\t"                                \
    "tcgen05.mma.cta_group::1.kind::f16 [" D3 "], [%10], %18, %4, " P3 ";\n\t"                               \
    "tcgen05.mma.cta_group::1.kind::f16 [" D4 "], [%11], %19, %4, " P4 ";\n\t"                               \
    "tcgen05.mma.cta_group::1.kind::f16 [" D5 "], [%12], %20, %4, " P5 ";\n\t"                               \
    "tcgen05.mma.cta_group::1.kind::f16 [" D6 "], [%13], %21, %4, " P6 ";\n\t"                               \
    "tcgen05.mma.cta_group::1.kind::f16 [" D7 "], [%14], %22, %4, " P7 ";\n\t"                               \
    "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%5];\n\t"                        \
    "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%6];\n\t}"

template <int GROUP>
__device__ __forceinline__ void mma8_stage(uint32_t a, uint32_t d, uint64_t b0, uint64_t b1, uint32_t idesc,
                                           uint64_t* bar_smem, uint64_t* bar_slot) {
    const uint32_t d0 = d, d1 = d + 16, d2 = d + 32, d3 = d + 48;
#define W4A16_MMA8_OPERANDS                                                                                 \
    "r"(d0), "r"(d1), "r"(d2), "r"(d3), "r"(idesc), "r"(smem_u32(bar_smem)), "r"(smem_u32(bar_slot)),    \
        "r"(a), "r"(a + 8), "r"(a + 16), "r"(a + 24), "r"(a + 32), "r"(a + 40), "r"(a + 48), "r"(a + 56),  \
        "l"(b0), "l"(b0 + 2), "l"(b0 + 4), "l"(b0 + 6), "l"(b1), "l"(b1 + 2), "l"(b1 + 4), "l"(b1 + 6)
    if constexpr (GROUP == 128) {
        asm volatile(W4A16_MMA8("f", "t", "t", "t", "t", "t", "t", "t", "%0", "%0", "%0", "%0", "%0", "%0", "%0", "%0")
                     ::W4A16_MMA8_OPERANDS : "memory");
    } else if constexpr (GROUP == 64) {
        asm volatile(W4A16_MMA8("f", "t", "t", "t", "f", "t", "t", "t", "%0", "%0", "%0", "%0", "%1", "%1", "%1", "%1")
                     ::W4A16_MMA8_OPERANDS : "memory");
    } else {
        asm volatile(W4A16_MMA8("f", "t", "f", "t", "f", "t", "f", "t", "%0", "%0", "%1", "%1", "%2", "%2", "%3", "%3")
                     ::W4A16_MMA8_OPERANDS : "memory");
    }
#undef W4A16_MMA8_OPERANDS
}

template <typename T, int GROUP>
__global__ void __launch_bounds__(kSkThreads, 2)
skinny_kernel(const __grid_constant__ CUtensorMap tmA, const uint8_t* __restrict__ tiled, int M, int K, int N,
              int sym, uint32_t scales_off, uint32_t zeros_off, int splits, T* __restrict__ C, int* dev_status) {
    using Cfg = SkCfg<GROUP>;
    constexpr int G = Cfg::kG;
    constexpr int NSLOT = Cfg::kNSlot;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* red = reinterpret_cast<float*>(smem + kSkNS * kSkStage);       // [2][16][128]
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kSkNS * kSkStage + kSkRed);
    uint64_t* empty = full + kSkNS;
    uint64_t* afull = empty + kSkNS;
    uint64_t* sdone = afull + NSLOT;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sdone + NSLOT);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nt = blockIdx.x;
    const int n0 = nt * 128;
    const int split = blockIdx.y;
    const int units = K / 128;
    const int st0 = (int)(((long long)split * units) / splits);          // first global stage
    const int nst = (int)(((long long)(split + 1) * units) / splits) - st0;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kSkNS; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < NSLOT; ++i) {
            mbar_init(&afull[i], 32 * kSkDeqWarps);
            mbar_init(&sdone[i], 1);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kSkTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    float acc[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) acc[j] = 0.0f;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0 && nst > 0) {
            prefetch_tensormap(&tmA);
            const uint32_t zbytes = sym ? 0u : 64u * G;
            const uint8_t* zsrc0 = tiled + zeros_off + (size_t)(n0 / 8) * 4;
            const uint8_t* csrc = tiled + ((size_t)nt * (K / 64) + 2 * (size_t)st0) * 4096;
            int issued = 0;
            for (int it = 0; it < nst; ++it) {
                const int s = it % kSkNS;
                if (!mbar_wait(&empty[s], ((uint32_t)(it / kSkNS) & 1u) ^ 1u, abort_flag, dev_status, kSkSpin)) break;
                uint8_t* st = smem + s * kSkStage;
                const int gs = st0 + it;
                mbar_arrive_expect_tx(&full[s], (uint32_t)(kSkActs + kSkCodes) + zbytes);
                tma_2d_g2s(st, &tmA, gs * 128, 0, &full[s]);
                tma_2d_g2s(st + 2048, &tmA, gs * 128 + 64, 0, &full[s]);
                bulk_g2s(st + kSkActs, csrc + (size_t)it * 8192, 8192, &full[s]);
                if (!sym) {
#pragma unroll
                    for (int g = 0; g < G; ++g)
                        bulk_g2s(st + kSkActs + kSkCodes + 64 * g, zsrc0 + (size_t)(gs * G + g) * (N / 8) * 4, 64,
                                 &full[s]);
                }
                ++issued;
            }
            for (int it = (issued > kSkNS ? issued - kSkNS : 0); it < issued; ++it)
                mbar_wait(&full[it % kSkNS], (uint32_t)(it / kSkNS) & 1u, abort_flag, dev_status, kSkSpin);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && nst > 0) {
            constexpr uint32_t idesc = idesc_f16(16, !std::is_same<T, __half>::value);
            const uint32_t smem_base = smem_u32(smem);
            for (int it = 0; it < nst; ++it) {
                const int s = it % kSkNS, j = it % NSLOT;
                // the dequant threads arrive only after they saw the stage's copies land
                if (!mbar_wait(&afull[j], (uint32_t)(it / NSLOT) & 1u, abort_flag, dev_status, kSkSpin)) break;
                tc_fence_after();
                const uint32_t sb = smem_base + s * kSkStage;
                const uint32_t slot = tmem + (uint32_t)(j * Cfg::kSlot);
                mma8_stage<GROUP>(slot, slot + 64, smem_desc_sw128(sb), smem_desc_sw128(sb + 2048), idesc, &empty[s],
                                  &sdone[j]);
            }
        }
    } else {
        // ------------------------------------------------------------ dequant + accumulator drain
        const int dw = warp - 2;             // 0..7
        const int q = warp & 3;              // TMEM lane quarter of this warp
        const int h = dw >> 2;               // 64-K tile of the stage this warp dequantizes
        const int n = 32 * q + lane;
        const uint32_t lane_off = (uint32_t)(32 * q) << 16;
        const __half* srow = reinterpret_cast<const __half*>(tiled + scales_off) + n0 + n;
        // groups of the stage this warp drains: G = 1 -> tile 0's warps take group 0;
        // G = 2 -> group h; G = 4 -> groups 2h, 2h + 1
        const bool drains = (G > 1) || (h == 0);
        const int gbase = G >= 2 ? h * Cfg::kGPerHalf : 0;
        // Scales of the stages whose accumulators are still to be drained: one register pair per
        // TMEM slot, loaded when the slot is filled and read NSLOT stages later when it is drained.
        // The loop is unrolled by NSLOT so that the slot index, and with it the register, is a
        // compile-time constant: a loaded register is never moved while its load is in flight.
        // (kept as raw fp16 bits: converting at load time would wait for the load)
        unsigned short sreg[NSLOT][2];
#pragma unroll
        for (int i = 0; i < NSLOT; ++i) sreg[i][0] = sreg[i][1] = 0;
        Sub<T> sub;
        bool ok = true;
        const unsigned short* srow_bits = reinterpret_cast<const unsigned short*>(srow);
        auto step = [&](const int it, const int j, unsigned short (&sr)[2]) {
            const bool fill = it < nst;
            const int s = it % kSkNS;
            // this slot's previous stage has completed: its accumulators can be read
            if (!mbar_wait(&sdone[j], ((uint32_t)(it / NSLOT) & 1u) ^ 1u, abort_flag, dev_status, kSkSpin)) {
                ok = false;
                return;
            }
            tc_fence_after();
            const uint32_t slot = tmem + (uint32_t)(j * Cfg::kSlot) + lane_off;
            uint32_t d0[16], d1[16];
            const bool drain = it >= NSLOT && drains;
            if (drain) {
                tmem_ld16(slot + 64 + 16 * gbase, d0);
                if (Cfg::kGPerHalf == 2) tmem_ld16(slot + 64 + 16 * (gbase + 1), d1);
            }
            const unsigned short s_old0 = sr[0], s_old1 = sr[1];
            if (fill && drains) {
                // scales of stage `it`, drained NSLOT stages later
                const size_t g = (size_t)(st0 + it) * G + gbase;
                sr[0] = srow_bits[g * N];
                if (Cfg::kGPerHalf == 2) sr[1] = srow_bits[(g + 1) * N];
            }
            if (fill) {
                if (!mbar_wait(&full[s], (uint32_t)(it / kSkNS) & 1u, abort_flag, dev_status, kSkSpin)) {
                    ok = false;
                    return;
                }
                const uint8_t* st = smem + s * kSkStage;
                const uint4* ct = reinterpret_cast<const uint4*>(st + kSkActs + 4096 * h);
                const uint4 wlo = ct[n];
                const uint4 whi = ct[128 + n];
                const uint32_t words[8] = {wlo.x, wlo.y, wlo.z, wlo.w, whi.x, whi.y, whi.z, whi.w};
                const uint32_t* zs = reinterpret_cast<const uint32_t*>(st + kSkActs + kSkCodes);
                uint32_t v[32];
#pragma unroll
                for (int jl = 0; jl < 8; ++jl) {
                    if (jl == 0 || (GROUP == 32 && jl == 4)) {
                        // group of these K inside the stage: (64 h + 8 jl) / GROUP
                        const int lg = (64 * h + 8 * jl) / GROUP;
                        const int z = sym ? 8 : (int)((zs[16 * lg + n / 8] >> (4 * (n % 8))) & 0xFu);
                        sub.set(z);
                    }
                    const uint32_t w = words[jl];
                    v[4 * jl + 0] = sub.pair((w & 0x000F000Fu) | Sub<T>::kMagic);
                    v[4 * jl + 1] = sub.pair(((w >> 4) & 0x000F000Fu) | Sub<T>::kMagic);
                    v[4 * jl + 2] = sub.pair(((w >> 8) & 0x000F000Fu) | Sub<T>::kMagic);
                    v[4 * jl + 3] = sub.pair(((w >> 12) & 0x000F000Fu) | Sub<T>::kMagic);
                }
                tmem_st32(slot + 32 * h, v);
            }
            if (drain) {
                tmem_ld_wait();
#pragma unroll
                const float sv0 = __half2float(__ushort_as_half(s_old0));
                for (int m = 0; m < 16; ++m) acc[m] = fmaf(sv0, __uint_as_float(d0[m]), acc[m]);
                if (Cfg::kGPerHalf == 2) {
                    const float sv1 = __half2float(__ushort_as_half(s_old1));
#pragma unroll
                    for (int m = 0; m < 16; ++m) acc[m] = fmaf(sv1, __uint_as_float(d1[m]), acc[m]);
                }
            }
            if (fill) {
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&afull[j]);
            }
        };
        for (int base = 0; base < nst + NSLOT && ok; base += NSLOT) {
#pragma unroll
            for (int j = 0; j < NSLOT; ++j)
                if (base + j < nst + NSLOT && ok) step(base + j, j, sreg[j]);
        }
        // the two warps of a channel quarter add their sums (named barrier over the dequant warps)
#pragma unroll
        for (int m = 0; m < 16; ++m) red[(h * 16 + m) * 128 + n] = acc[m];
        asm volatile("bar.sync 1, %0;" ::"r"(32 * kSkDeqWarps) : "memory");
        if (h == 0) {
#pragma unroll
            for (int m = 0; m < 16; ++m) acc[m] += red[(16 + m) * 128 + n];
            if (splits == 1) {
#pragma unroll
                for (int m = 0; m < 16; ++m)
                    if (m < M) C[(size_t)m * N + n0 + n] = Act<T>::from_f32(acc[m]);
            } else {
#pragma unroll
                for (int m = 0; m < 16; ++m) red[m * 128 + n] = acc[m];
            }
        }
    }

    if (splits > 1) {
        // split-K: the S CTAs of the cluster add their partial sums in rank order
        cluster_sync();
        if (warp >= 2 && warp < 6) {
            const int e = threadIdx.x - 64;
            const int rank = (int)cluster_ctarank();
            const int cnt = (128 - rank + splits - 1) / splits;  // channels rank, rank + S, ...
            for (int i = e; i < M * cnt; i += 128) {
                const int m = i / cnt;
                const int c = rank + splits * (i - m * cnt);
                float sum = 0.0f;
                for (int p = 0; p < splits; ++p) sum += ld_cluster_f32(cluster_map(red + m * 128 + c, (uint32_t)p));
                C[(size_t)m * N + n0 + c] = Act<T>::from_f32(sum);
            }
        }
        cluster_sync();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kSkTmemCols);
    }
}

template <typename T, int GROUP>
int launch_skinny_typed(const void* A, int M, int K, const void* tiled, int N, int sym, void* C, int splits,
                        int* dev_status, cudaStream_t stream) {
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(skinny_kernel<T, GROUP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        kSkSmem);
    });
    if (attr_err != cudaSuccess) return W4A16_ECUDA;
    CUtensorMap map;
    if (!make_act_map(&map, A, M, K, 16, !std::is_same<T, __half>::value)) return W4A16_ECUDA;
    const TiledOffsets off = tiled_offsets(K, N, GROUP, sym);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(N / 128, splits, 1);
    cfg.blockDim = dim3(kSkThreads, 1, 1);
    cfg.dynamicSmemBytes = kSkSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = splits;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, skinny_kernel<T, GROUP>, map, static_cast<const uint8_t*>(tiled), M, K,
                                       N, sym, (uint32_t)off.scales, (uint32_t)off.zeros, splits, static_cast<T*>(C),
                                       dev_status);
    return e == cudaSuccess ? W4A16_OK : W4A16_ECUDA;
}

template <typename T>
int launch_skinny_group(const void* A, int M, int K, const void* tiled, int N, int group, int sym, void* C,
                        int splits, int* dev_status, cudaStream_t stream) {
    switch (group) {
        case 32: return launch_skinny_typed<T, 32>(A, M, K, tiled, N, sym, C, splits, dev_status, stream);
        case 64: return launch_skinny_typed<T, 64>(A, M, K, tiled, N, sym, C, splits, dev_status, stream);
        case 128: return launch_skinny_typed<T, 128>(A, M, K, tiled, N, sym, C, splits, dev_status, stream);
        default: return W4A16_EUNSUPPORTED;
    }
}

}  // namespace

// K splits of the skinny kernel: the 128-channel tiles times the splits should fill the 296
// resident CTA slots of a 148-SM B200 (two per SM) about once; at most 8 (a portable cluster),
// at most one per 128-K stage.
int skinny_splits(int N, int K, int group) {
    (void)group;
    const int tiles = N / 128;
    const int units = K / 128;
    int s = (2 * 148 + tiles / 2) / tiles;
    if (s > 8) s = 8;
    if (s > units) s = units;
    return s < 1 ? 1 : s;
}

int launch_gemm_skinny(const void* A, int a_dtype, int M, int K, const void* tiled, int N, int group, int sym,
                       void* C, int* dev_status, cudaStream_t stream) {
    if (M > 16 || K % 128 != 0) return W4A16_EUNSUPPORTED;
    const int splits = skinny_splits(N, K, group);
    if (a_dtype == W4A16_BF16)
        return launch_skinny_group<__nv_bfloat16>(A, M, K, tiled, N, group, sym, C, splits, dev_status, stream);
    return launch_skinny_group<__half>(A, M, K, tiled, N, group, sym, C, splits, dev_status, stream);
}

}  // namespace w4a16
