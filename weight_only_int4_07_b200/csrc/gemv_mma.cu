// gemv_mma.cu -- split-K decode GEMV / skinny GEMM (M <= 16) on the tiled layout, with the
// multiply-accumulate on the warp-level tensor-core MMA (mma.sync m16n8k16, FP32 accumulators).
//
// C[m, n] = sum_k A[m, k] * (u[k, n] - z[g, n]) * s[g, n], FP32 accumulation.
// "4.3 Weight-only INT4", section 4 (read, unpack, dequantize and multiply in one pass so each
// weight byte crosses HBM once); "INT8 vs INT4 Quantization, in depth", "Two regimes" (at small
// batch the layer waits for memory).
//
// Why this engine. At the measured 6.5 TB/s a B200 SM has to take in about 45 weights per clock,
// i.e. under 2.8 issue slots per weight. Measured on this part: a CUDA-core loop (unpack, exact
// subtract, mixed-precision FMA into FP32) executes about 4.6 warp-lane instructions per weight,
// and tcgen05.mma at its smallest N (16) is bound by its per-instruction issue cost. The
// warp-level MMA takes the dequantized pairs straight from registers: per 8 weights a lane spends
// 3 shifts + 4 mask-ORs (nibble pairs -> 16-bit (1024 + u) / (128 + u)) + 4 packed subtracts
// (exact u - z), and one MMA covers 256 weights of a warp -- about 1.6 slots per weight.
//
// Mapping. A CTA of 8 warps owns one 128-channel column of 4 KiB tiles and a K range of whole
// 128-K steps; warp w owns channels 16 w .. 16 w + 15 (the MMA's 16 rows). Per 128-K step, lane
// (g = lane / 4, t = lane % 4) loads 16 bytes -- 32 consecutive K of 32-K block t -- for channel
// 16 w + g and for 16 w + g + 8, and feeds them to eight MMAs. The MMA's K order is a permutation
// of the step's 128 K (the same for both operands): for MMA s, lane t's columns (2t, 2t+1) and
// (2t+8, 2t+9) are K = 32 t + 8 (s/2) + 4 (s%2) + {0,1} and + {2,3}. Activations of the CTA's
// K range sit in shared memory; lane (g', t') reads rows 8 b + g' of n8-tile b.
// Scaling: with group 128 a step is one group: the MMAs see exact integers (u - z) and the FP32
// fragment is scaled by s[g, n] after the step (no weight is rounded). With smaller groups a
// step spans several groups, so the weights are scaled before the MMA, (u - z) * s rounded once
// to the 16-bit type (fp16: exact subtract then one multiply; bf16: s split into a bf16 high
// part and an exact remainder, then one fused multiply-add).
// Split-K partial sums of the S CTAs of a thread-block cluster are added through distributed
// shared memory in rank order. No workspace, one launch.
#include <mutex>
#include <type_traits>

#include "common.cuh"
#include "sm100_ptx.cuh"
#include "tiled_layout.cuh"

namespace w4a16 {
namespace {

using namespace sm100;

constexpr int kGmThreads = 256;
constexpr int kGmActBytes = 96 * 1024;   // activation budget in shared memory

template <typename T>
struct Frag;

template <>
struct Frag<__half> {
    static constexpr uint32_t kMagic = 0x64006400u;  // 1024 + u
    static __device__ __forceinline__ uint32_t zz(int z) { return (uint32_t)(0x6400 + z) * 0x00010001u; }
    static __device__ __forceinline__ uint32_t sub(uint32_t x, uint32_t zz2) {
        uint32_t r;
        asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(zz2));
        return r;
    }
    // scaled pair: (x - zz) * s, one rounding
    struct Scale {
        uint32_t s2;
        __device__ __forceinline__ void set(float s) {
            __half2 h = __float2half2_rn(s);
            s2 = *reinterpret_cast<uint32_t*>(&h);
        }
        __device__ __forceinline__ uint32_t apply(uint32_t d) const {
            uint32_t r;
            asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(d), "r"(s2));
            return r;
        }
    };
    static __device__ __forceinline__ void mma(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
            "{%0, %1, %2, %3};"
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    }
};

template <>
struct Frag<__nv_bfloat16> {
    static constexpr uint32_t kMagic = 0x43004300u;  // 128 + u
    static __device__ __forceinline__ uint32_t zz(int z) { return (uint32_t)(0x4300 + z) * 0x00010001u; }
    static __device__ __forceinline__ uint32_t sub(uint32_t x, uint32_t zz2) {
        uint32_t r;
        asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(zz2));
        return r;
    }
    // scaled pair: d * s rounded once, s = s_hi (bf16 truncation) + s_lo (exact in bf16)
    struct Scale {
        uint32_t hi2, lo2;
        __device__ __forceinline__ void set(float s) {
            const uint32_t sb = __float_as_uint(s) & 0xFFFF0000u;
            const float lo = s - __uint_as_float(sb);
            hi2 = (sb >> 16) * 0x00010001u;
            __nv_bfloat162 l = __float2bfloat162_rn(lo);
            lo2 = *reinterpret_cast<uint32_t*>(&l);
        }
        __device__ __forceinline__ uint32_t apply(uint32_t d) const {
            uint32_t t, r;
            asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(t) : "r"(d), "r"(lo2));
            asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(d), "r"(hi2), "r"(t));
            return r;
        }
    };
    static __device__ __forceinline__ void mma(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
            "{%0, %1, %2, %3};"
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    }
};

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// NB: n8 tiles of A rows (1 for M <= 8, 2 for M <= 16).
template <int NB, typename T, int GROUP>
__global__ void __launch_bounds__(kGmThreads)
gemv_mma_kernel(const T* __restrict__ A, int M, int K, int N, const uint8_t* __restrict__ tiled, int sym,
                uint32_t scales_off, uint32_t zeros_off, int splits, uint32_t act_bytes, T* __restrict__ C) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    constexpr int MT = 8 * NB;
    constexpr bool kPostScale = (GROUP == 128);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int nt = blockIdx.x;
    const int n0 = nt * 128;
    const int split = blockIdx.y;
    const int steps = K / 128;
    const int sp0 = (int)(((long long)split * steps) / splits);
    const int sp1 = (int)(((long long)(split + 1) * steps) / splits);
    const int kspan = 128 * (sp1 - sp0);

    // activations of the CTA's K range, [M][kspan] 16-bit (lanes of rows >= M use zeros)
    T* acts = reinterpret_cast<T*>(smem_raw);
    float* red = reinterpret_cast<float*>(smem_raw + act_bytes);   // [MT][128]
    {
        const int vec_per_row = kspan / 8;
        for (int v = threadIdx.x; v < M * vec_per_row; v += kGmThreads) {
            const int m = v / vec_per_row, c = v - m * vec_per_row;
            *reinterpret_cast<uint4*>(acts + (size_t)m * kspan + 8 * c) =
                *reinterpret_cast<const uint4*>(A + (size_t)m * K + 128 * sp0 + 8 * c);
        }
    }
    __syncthreads();

    const int ch0 = 16 * warp + g;            // this lane's rows: channels ch0 and ch0 + 8 of the tile
    const int ktiles = K / 64;
    // 16-byte vector of channel ch, 32-K block t of step sp: tile 2 sp + t/2, half t%2
    const uint8_t* vbase = tiled + ((size_t)nt * ktiles) * 4096 + ((size_t)((t & 1) * 128 + ch0)) * 16 +
                           (size_t)(t >> 1) * 4096;
    const unsigned short* sbits = reinterpret_cast<const unsigned short*>(tiled + scales_off) + n0 + ch0;
    const uint32_t* zw = reinterpret_cast<const uint32_t*>(tiled + zeros_off);
    const int zsh0 = 4 * ((n0 + ch0) % 8), zsh1 = 4 * ((n0 + ch0 + 8) % 8);
    const int zc0 = (n0 + ch0) / 8, zc1 = (n0 + ch0 + 8) / 8;

    float tot[NB][4];
#pragma unroll
    for (int b = 0; b < NB; ++b) tot[b][0] = tot[b][1] = tot[b][2] = tot[b][3] = 0.0f;

    // software pipeline: the next step's 32 bytes of codes, zero-points and scale bits are in flight
    // while this step computes (kept as raw bits: converting at load time would wait for the load)
    auto grp_of = [&](int sp) { return (sp * 128 + 32 * t) / GROUP; };
    uint4 wcur0 = make_uint4(0, 0, 0, 0), wcur1 = wcur0;
    uint32_t zcur0 = 0, zcur1 = 0;
    unsigned short scur0 = 0, scur1 = 0;
    auto load_step = [&](int sp, uint4& w0, uint4& w1, uint32_t& zr0, uint32_t& zr1, unsigned short& sr0,
                         unsigned short& sr1) {
        w0 = ldg_stream(vbase + (size_t)(2 * sp) * 4096);
        w1 = ldg_stream(vbase + (size_t)(2 * sp) * 4096 + 8 * 16);
        const int grp = grp_of(sp);
        if (!sym) {
            const uint32_t* zr = zw + (size_t)grp * (N / 8);
            zr0 = __ldg(zr + zc0);
            zr1 = __ldg(zr + zc1);
        }
        sr0 = __ldg(sbits + (size_t)grp * N);
        sr1 = __ldg(sbits + (size_t)grp * N + 8);
    };
    if (sp0 < sp1) load_step(sp0, wcur0, wcur1, zcur0, zcur1, scur0, scur1);
    for (int sp = sp0; sp < sp1; ++sp) {
        uint4 wn0 = wcur0, wn1 = wcur1;
        uint32_t zn0 = zcur0, zn1 = zcur1;
        unsigned short sn0 = scur0, sn1 = scur1;
        if (sp + 1 < sp1) load_step(sp + 1, wn0, wn1, zn0, zn1, sn0, sn1);
        const int z0 = sym ? 8 : (int)((zcur0 >> zsh0) & 0xFu);
        const int z1 = sym ? 8 : (int)((zcur1 >> zsh1) & 0xFu);
        const float s0 = __half2float(__ushort_as_half(scur0));
        const float s1 = __half2float(__ushort_as_half(scur1));
        const uint32_t zz0 = Frag<T>::zz(z0), zz1 = Frag<T>::zz(z1);
        typename Frag<T>::Scale sc0, sc1;
        if (!kPostScale) {
            sc0.set(s0);
            sc1.set(s1);
        }
        // activation fragments: lane (g', t') of n8-tile b holds row 8 b + g', K 32 t' .. 32 t' + 31
        uint32_t bfr[NB][16];
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            const int row = 8 * b + g;
            const bool live = row < M;
            // rows >= M are not in shared memory: read row 0 (in range) and use zeros
            const uint4* ap =
                reinterpret_cast<const uint4*>(acts + (size_t)(live ? row : 0) * kspan + 128 * (sp - sp0) + 32 * t);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint4 v = ap[q];
                if (!live) v = make_uint4(0, 0, 0, 0);
                bfr[b][4 * q + 0] = v.x;
                bfr[b][4 * q + 1] = v.y;
                bfr[b][4 * q + 2] = v.z;
                bfr[b][4 * q + 3] = v.w;
            }
        }
        float acc[NB][4];
#pragma unroll
        for (int b = 0; b < NB; ++b) acc[b][0] = acc[b][1] = acc[b][2] = acc[b][3] = 0.0f;
        const uint32_t wr0[4] = {wcur0.x, wcur0.y, wcur0.z, wcur0.w};   // channel ch0
        const uint32_t wr1[4] = {wcur1.x, wcur1.y, wcur1.z, wcur1.w};   // channel ch0 + 8
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            // the four K pairs of word j of both rows
            uint32_t p0[4], p1[4];
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                p0[p] = Frag<T>::sub(((wr0[j] >> (4 * p)) & 0x000F000Fu) | Frag<T>::kMagic, zz0);
                p1[p] = Frag<T>::sub(((wr1[j] >> (4 * p)) & 0x000F000Fu) | Frag<T>::kMagic, zz1);
                if (!kPostScale) {
                    p0[p] = sc0.apply(p0[p]);
                    p1[p] = sc1.apply(p1[p]);
                }
            }
            // MMA s = 2 j + h uses pairs 2h (columns 2t, 2t+1) and 2h + 1 (columns 2t+8, 2t+9)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int r = 4 * j + 2 * hh;   // activation pair index inside the lane's 32 K
#pragma unroll
                for (int b = 0; b < NB; ++b) {
                    if (kPostScale)
                        Frag<T>::mma(acc[b], p0[2 * hh], p1[2 * hh], p0[2 * hh + 1], p1[2 * hh + 1], bfr[b][r],
                                     bfr[b][r + 1]);
                    else
                        Frag<T>::mma(tot[b], p0[2 * hh], p1[2 * hh], p0[2 * hh + 1], p1[2 * hh + 1], bfr[b][r],
                                     bfr[b][r + 1]);
                }
            }
        }
        if (kPostScale) {
            // fragment rows: c0, c1 -> channel ch0; c2, c3 -> channel ch0 + 8
#pragma unroll
            for (int b = 0; b < NB; ++b) {
                tot[b][0] = fmaf(s0, acc[b][0], tot[b][0]);
                tot[b][1] = fmaf(s0, acc[b][1], tot[b][1]);
                tot[b][2] = fmaf(s1, acc[b][2], tot[b][2]);
                tot[b][3] = fmaf(s1, acc[b][3], tot[b][3]);
            }
        }
        wcur0 = wn0;
        wcur1 = wn1;
        zcur0 = zn0;
        zcur1 = zn1;
        scur0 = sn0;
        scur1 = sn1;
    }

    // fragment (row ch0 / ch0 + 8, columns 2t, 2t + 1 of n8-tile b) -> rows m = 8 b + 2 t (+1)
    if (splits == 1) {
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            const int m = 8 * b + 2 * t;
            if (m < M) {
                C[(size_t)m * N + n0 + ch0] = Act<T>::from_f32(tot[b][0]);
                C[(size_t)m * N + n0 + ch0 + 8] = Act<T>::from_f32(tot[b][2]);
            }
            if (m + 1 < M) {
                C[(size_t)(m + 1) * N + n0 + ch0] = Act<T>::from_f32(tot[b][1]);
                C[(size_t)(m + 1) * N + n0 + ch0 + 8] = Act<T>::from_f32(tot[b][3]);
            }
        }
        return;
    }
#pragma unroll
    for (int b = 0; b < NB; ++b) {
        const int m = 8 * b + 2 * t;
        red[m * 128 + ch0] = tot[b][0];
        red[m * 128 + ch0 + 8] = tot[b][2];
        red[(m + 1) * 128 + ch0] = tot[b][1];
        red[(m + 1) * 128 + ch0 + 8] = tot[b][3];
    }
    // the S CTAs of the cluster add their partial sums in rank order
    cluster_sync();
    const int rank = (int)cluster_ctarank();
    const int cnt = (128 - rank + splits - 1) / splits;  // channels rank, rank + S, ...
    for (int e = threadIdx.x; e < M * cnt; e += kGmThreads) {
        const int m = e / cnt;
        const int chn = rank + splits * (e - m * cnt);
        float sum = 0.0f;
        for (int p = 0; p < splits; ++p) sum += ld_cluster_f32(cluster_map(red + m * 128 + chn, (uint32_t)p));
        C[(size_t)m * N + n0 + chn] = Act<T>::from_f32(sum);
    }
    cluster_sync();
}

template <int NB, typename T, int GROUP>
int launch_typed(const void* A, int M, int K, const void* tiled, int N, int sym, void* C, int splits,
                 uint32_t act_bytes, cudaStream_t stream) {
    const size_t smem = act_bytes + 8 * NB * 128 * sizeof(float);
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(gemv_mma_kernel<NB, T, GROUP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)(kGmActBytes + 8 * NB * 128 * sizeof(float)));
        if (attr_err == cudaSuccess)
            attr_err = cudaFuncSetAttribute(gemv_mma_kernel<NB, T, GROUP>,
                                            cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    });
    if (attr_err != cudaSuccess) return W4A16_ECUDA;
    const TiledOffsets off = tiled_offsets(K, N, GROUP, sym);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(N / 128, splits, 1);
    cfg.blockDim = dim3(kGmThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = splits;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, gemv_mma_kernel<NB, T, GROUP>, static_cast<const T*>(A), M, K, N,
                                       static_cast<const uint8_t*>(tiled), sym, (uint32_t)off.scales,
                                       (uint32_t)off.zeros, splits, act_bytes, static_cast<T*>(C));
    return e == cudaSuccess ? W4A16_OK : W4A16_ECUDA;
}

template <int NB, typename T>
int launch_group(const void* A, int M, int K, const void* tiled, int N, int group, int sym, void* C, int splits,
                 uint32_t act_bytes, cudaStream_t stream) {
    switch (group) {
        case 32: return launch_typed<NB, T, 32>(A, M, K, tiled, N, sym, C, splits, act_bytes, stream);
        case 64: return launch_typed<NB, T, 64>(A, M, K, tiled, N, sym, C, splits, act_bytes, stream);
        case 128: return launch_typed<NB, T, 128>(A, M, K, tiled, N, sym, C, splits, act_bytes, stream);
        default: return W4A16_EUNSUPPORTED;
    }
}

}  // namespace

// K splits (cluster size, at most 16): the 128-channel tiles times the splits should fill about
// four 256-thread CTAs per SM of a 148-SM B200 once, with the CTA's activations inside the
// shared-memory budget; at most one split per 128-K step.
int gemv_mma_splits(int M, int N, int K) {
    const int tiles = N / 128;
    const int steps = K / 128;
    int s = (4 * 148 + tiles / 2) / tiles;
    if (s > 16) s = 16;
    while (s < 16 && (size_t)M * (size_t)(128 * ((steps + s - 1) / s)) * 2 > (size_t)kGmActBytes) ++s;
    if (s > steps) s = steps;
    return s < 1 ? 1 : s;
}

int launch_gemv_mma(const void* A, int a_dtype, int M, int K, const void* tiled, int N, int group, int sym,
                    void* C, cudaStream_t stream) {
    if (M > 16 || K % 128 != 0) return W4A16_EUNSUPPORTED;
    const int splits = gemv_mma_splits(M, N, K);
    const int steps = K / 128;
    const size_t act_bytes = (size_t)M * 128 * ((steps + splits - 1) / splits) * 2;
    if (act_bytes > (size_t)kGmActBytes) return W4A16_EUNSUPPORTED;
    const uint32_t ab = (uint32_t)act_bytes;
    if (a_dtype == W4A16_BF16) {
        if (M <= 8) return launch_group<1, __nv_bfloat16>(A, M, K, tiled, N, group, sym, C, splits, ab, stream);
        return launch_group<2, __nv_bfloat16>(A, M, K, tiled, N, group, sym, C, splits, ab, stream);
    }
    if (M <= 8) return launch_group<1, __half>(A, M, K, tiled, N, group, sym, C, splits, ab, stream);
    return launch_group<2, __half>(A, M, K, tiled, N, group, sym, C, splits, ab, stream);
}

}  // namespace w4a16
