// gemv_tiled.cu -- split-K CUDA-core GEMV for decode (M = 1, 2) on the tiled layout.
//
// C[m, n] = sum_g s[g, n] * sum_{k in g} A[m, k] * (u[k, n] - z[g, n]), FP32 accumulation.
// "4.3 Weight-only INT4", section 4 (read, unpack, dequantize and multiply in one pass, each weight
// byte crossing HBM once); "INT8 vs INT4 Quantization, in depth", "Two regimes" (at batch 1 the
// layer waits for memory: it is a GEMV, so it runs on the CUDA cores, not reshaped into a GEMM).
//
// Per weight the CUDA cores spend: an eighth of a 16-byte load, (3 shifts + 4 mask-ORs) / 8 to
// turn nibble pairs into 16-bit (1024 + u) or (128 + u) values, half a packed subtract for the
// exact integer (u - z), and one mixed-precision FMA (16-bit x 16-bit + FP32 accumulator), i.e.
// about 2.4 issue slots -- close to but under the ~2.8 slots per weight a B200 SM has at the
// HBM rate. The scale is applied once per group in FP32. No weight is ever rounded.
//
// Work split: a CTA of 256 threads owns one 128-channel column of 4 KiB tiles and a K range of
// whole groups; thread i reads bytes [16 i, 16 i + 16) of every tile (a linear 4 KiB read): the
// 32 K of half h = i / 128 for channel n = i % 128. Four tiles are in flight per thread. The
// activations of the CTA's K range sit in shared memory (read by broadcast). The two halves of a
// channel are added in shared memory, and the S CTAs of a thread-block cluster (split-K) add their
// partial sums through distributed shared memory in rank order. No workspace, one launch.
#include <mutex>
#include <type_traits>

#include "common.cuh"
#include "sm100_ptx.cuh"
#include "tiled_layout.cuh"

namespace w4a16 {
namespace {

using namespace sm100;

constexpr int kGvThreads = 256;
constexpr int kGvUnroll = 4;              // tiles in flight per thread
constexpr int kGvActBytes = 64 * 1024;    // activation budget in shared memory

template <typename T>
struct Mix;

// fp16: weights (1024 + u) - (1024 + z) exact; fma.rn.f32.f16 multiplies two fp16 exactly into FP32.
template <>
struct Mix<__half> {
    static constexpr uint32_t kMagic = 0x64006400u;
    static __device__ __forceinline__ uint32_t zz(int z) { return (uint32_t)(0x6400 + z) * 0x00010001u; }
    static __device__ __forceinline__ uint32_t sub(uint32_t x, uint32_t zz2) {
        uint32_t r;
        asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(zz2));
        return r;
    }
    // acc += a.lo * w.lo + a.hi * w.hi (two mixed-precision FMAs, in this order)
    static __device__ __forceinline__ void fma2(float& acc, uint32_t a2, uint32_t w2) {
        asm("{\n\t.reg .b16 al, ah, wl, wh;\n\t"
            "mov.b32 {al, ah}, %1;\n\t"
            "mov.b32 {wl, wh}, %2;\n\t"
            "fma.rn.f32.f16 %0, al, wl, %0;\n\t"
            "fma.rn.f32.f16 %0, ah, wh, %0;\n\t}"
            : "+f"(acc)
            : "r"(a2), "r"(w2));
    }
};

// bf16: weights (128 + u) - (128 + z) exact; fma.rn.f32.bf16 multiplies two bf16 exactly into FP32.
template <>
struct Mix<__nv_bfloat16> {
    static constexpr uint32_t kMagic = 0x43004300u;
    static __device__ __forceinline__ uint32_t zz(int z) { return (uint32_t)(0x4300 + z) * 0x00010001u; }
    static __device__ __forceinline__ uint32_t sub(uint32_t x, uint32_t zz2) {
        uint32_t r;
        asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(zz2));
        return r;
    }
    static __device__ __forceinline__ void fma2(float& acc, uint32_t a2, uint32_t w2) {
        asm("{\n\t.reg .b16 al, ah, wl, wh;\n\t"
            "mov.b32 {al, ah}, %1;\n\t"
            "mov.b32 {wl, wh}, %2;\n\t"
            "fma.rn.f32.bf16 %0, al, wl, %0;\n\t"
            "fma.rn.f32.bf16 %0, ah, wh, %0;\n\t}"
            : "+f"(acc)
            : "r"(a2), "r"(w2));
    }
};

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

template <int MT, typename T, int GROUP>
__global__ void __launch_bounds__(kGvThreads)
gemv_tiled_kernel(const T* __restrict__ A, int M, int K, int N, const uint8_t* __restrict__ tiled, int sym,
                  uint32_t scales_off, uint32_t zeros_off, int splits, uint32_t act_bytes, T* __restrict__ C) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    constexpr int kUnitTiles = GROUP >= 64 ? GROUP / 64 : 1;   // tiles per whole-group unit
    const int i = threadIdx.x;
    const int h = i >> 7;
    const int n = i & 127;
    const int nt = blockIdx.x;
    const int n0 = nt * 128;
    const int split = blockIdx.y;
    const int ktiles = K / 64;
    const int units = ktiles / kUnitTiles;
    const int c0 = (int)(((long long)split * units) / splits) * kUnitTiles;
    const int c1 = (int)(((long long)(split + 1) * units) / splits) * kUnitTiles;
    const int kspan = 64 * (c1 - c0);

    // activations of the CTA's K range, [MT][kspan] 16-bit, rows >= M zero
    T* acts = reinterpret_cast<T*>(smem_raw);
    float* red = reinterpret_cast<float*>(smem_raw + act_bytes);     // [2][MT][128]
    {
        const int vec_per_row = kspan / 8;   // 16-byte vectors
        for (int v = i; v < MT * vec_per_row; v += kGvThreads) {
            const int m = v / vec_per_row, c = v - m * vec_per_row;
            uint4 val = make_uint4(0, 0, 0, 0);
            if (m < M) val = *reinterpret_cast<const uint4*>(A + (size_t)m * K + 64 * c0 + 8 * c);
            *reinterpret_cast<uint4*>(acts + (size_t)m * kspan + 8 * c) = val;
        }
    }
    __syncthreads();

    const uint8_t* tbase = tiled + ((size_t)nt * ktiles) * 4096 + 16 * i;
    const unsigned short* sbits = reinterpret_cast<const unsigned short*>(tiled + scales_off) + n0 + n;
    const uint32_t* zw = reinterpret_cast<const uint32_t*>(tiled + zeros_off) + (n0 + n) / 8;
    const int zshift = 4 * ((n0 + n) % 8);

    float y[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) y[m] = 0.0f;

    // group of tile c for this thread's half: g128 -> c / 2, g64 -> c, g32 -> 2 c + h
    auto group_of = [&](int c) { return GROUP == 128 ? c / 2 : (GROUP == 64 ? c : 2 * c + h); };

    for (int cb = c0; cb < c1; cb += kGvUnroll) {
        uint4 w[kGvUnroll];
        unsigned short sraw[kGvUnroll];
        uint32_t zraw[kGvUnroll];
#pragma unroll
        for (int u = 0; u < kGvUnroll; ++u) {
            const int c = cb + u;
            if (c < c1) {
                w[u] = ldg_stream(tbase + (size_t)c * 4096);
                const int g = group_of(c);
                sraw[u] = __ldg(sbits + (size_t)g * N);
                zraw[u] = sym ? 0u : __ldg(zw + (size_t)g * (N / 8));
            }
        }
#pragma unroll
        for (int u = 0; u < kGvUnroll; ++u) {
            const int c = cb + u;
            if (c >= c1) break;
            const int z = sym ? 8 : (int)((zraw[u] >> zshift) & 0xFu);
            const uint32_t zz2 = Mix<T>::zz(z);
            const uint32_t words[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
            const T* arow = acts + 64 * (c - c0) + 32 * h;
            float acc[MT][2];
#pragma unroll
            for (int m = 0; m < MT; ++m) acc[m][0] = acc[m][1] = 0.0f;
#pragma unroll
            for (int jl = 0; jl < 4; ++jl) {
                const uint32_t wd = words[jl];
                uint32_t d[4];
                d[0] = Mix<T>::sub((wd & 0x000F000Fu) | Mix<T>::kMagic, zz2);
                d[1] = Mix<T>::sub(((wd >> 4) & 0x000F000Fu) | Mix<T>::kMagic, zz2);
                d[2] = Mix<T>::sub(((wd >> 8) & 0x000F000Fu) | Mix<T>::kMagic, zz2);
                d[3] = Mix<T>::sub(((wd >> 12) & 0x000F000Fu) | Mix<T>::kMagic, zz2);
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    const uint4 a = *reinterpret_cast<const uint4*>(arow + (size_t)m * kspan + 8 * jl);
                    Mix<T>::fma2(acc[m][0], a.x, d[0]);
                    Mix<T>::fma2(acc[m][1], a.y, d[1]);
                    Mix<T>::fma2(acc[m][0], a.z, d[2]);
                    Mix<T>::fma2(acc[m][1], a.w, d[3]);
                }
            }
            const float s = __half2float(__ushort_as_half(sraw[u]));
#pragma unroll
            for (int m = 0; m < MT; ++m) y[m] = fmaf(s, acc[m][0] + acc[m][1], y[m]);
        }
    }

    // the two halves of a channel
#pragma unroll
    for (int m = 0; m < MT; ++m) red[(h * MT + m) * 128 + n] = y[m];
    __syncthreads();
    if (h == 0) {
#pragma unroll
        for (int m = 0; m < MT; ++m) y[m] += red[(MT + m) * 128 + n];
        if (splits == 1) {
#pragma unroll
            for (int m = 0; m < MT; ++m)
                if (m < M) C[(size_t)m * N + n0 + n] = Act<T>::from_f32(y[m]);
        } else {
#pragma unroll
            for (int m = 0; m < MT; ++m) red[m * 128 + n] = y[m];
        }
    }
    if (splits > 1) {
        // the S CTAs of the cluster add their partial sums in rank order
        cluster_sync();
        const int rank = (int)cluster_ctarank();
        const int cnt = (128 - rank + splits - 1) / splits;  // channels rank, rank + S, ...
        for (int e = i; e < M * cnt; e += kGvThreads) {
            const int m = e / cnt;
            const int ch = rank + splits * (e - m * cnt);
            float sum = 0.0f;
            for (int p = 0; p < splits; ++p) sum += ld_cluster_f32(cluster_map(red + m * 128 + ch, (uint32_t)p));
            C[(size_t)m * N + n0 + ch] = Act<T>::from_f32(sum);
        }
        cluster_sync();
    }
}

template <int MT, typename T, int GROUP>
int launch_typed(const void* A, int M, int K, const void* tiled, int N, int sym, void* C, int splits,
                 uint32_t act_bytes, cudaStream_t stream) {
    const size_t smem = act_bytes + 2 * MT * 128 * sizeof(float);
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(gemv_tiled_kernel<MT, T, GROUP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)(kGvActBytes + 2 * MT * 128 * sizeof(float)));
        if (attr_err == cudaSuccess)
            attr_err = cudaFuncSetAttribute(gemv_tiled_kernel<MT, T, GROUP>,
                                            cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    });
    if (attr_err != cudaSuccess) return W4A16_ECUDA;
    const TiledOffsets off = tiled_offsets(K, N, GROUP, sym);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(N / 128, splits, 1);
    cfg.blockDim = dim3(kGvThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = splits;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, gemv_tiled_kernel<MT, T, GROUP>, static_cast<const T*>(A), M, K, N,
                                       static_cast<const uint8_t*>(tiled), sym, (uint32_t)off.scales,
                                       (uint32_t)off.zeros, splits, act_bytes, static_cast<T*>(C));
    return e == cudaSuccess ? W4A16_OK : W4A16_ECUDA;
}

template <int MT, typename T>
int launch_group(const void* A, int M, int K, const void* tiled, int N, int group, int sym, void* C, int splits,
                 uint32_t act_bytes, cudaStream_t stream) {
    switch (group) {
        case 32: return launch_typed<MT, T, 32>(A, M, K, tiled, N, sym, C, splits, act_bytes, stream);
        case 64: return launch_typed<MT, T, 64>(A, M, K, tiled, N, sym, C, splits, act_bytes, stream);
        case 128: return launch_typed<MT, T, 128>(A, M, K, tiled, N, sym, C, splits, act_bytes, stream);
        default: return W4A16_EUNSUPPORTED;
    }
}

}  // namespace

// K splits (cluster size, at most 16): the 128-channel tiles times the splits should fill the 592
// resident 256-thread CTA slots of a 148-SM B200 (four per SM) about once, while the CTA's
// activations fit the shared-memory budget and every split keeps whole groups.
int gemv_tiled_splits(int M, int N, int K, int group) {
    const int tiles = N / 128;
    const int unit = group >= 64 ? group / 64 : 1;
    const int units = (K / 64) / unit;
    const int mt = M <= 1 ? 1 : 2;
    int s = (4 * 148 + tiles / 2) / tiles;
    if (s > 16) s = 16;
    // the activations of one split must fit: mt * (K / s + a unit) * 2 bytes
    while (s < 16 && (size_t)mt * (size_t)(K / s + 64 * unit) * 2 > (size_t)kGvActBytes) ++s;
    if (s > units) s = units;
    return s < 1 ? 1 : s;
}

int launch_gemv_tiled(const void* A, int a_dtype, int M, int K, const void* tiled, int N, int group, int sym,
                      void* C, cudaStream_t stream) {
    if (M > 2) return W4A16_EUNSUPPORTED;
    const int splits = gemv_tiled_splits(M, N, K, group);
    const int unit = group >= 64 ? group / 64 : 1;
    const int units = (K / 64) / unit;
    const int max_span = 64 * unit * ((units + splits - 1) / splits);
    const size_t act_bytes = (size_t)(M <= 1 ? 1 : 2) * max_span * 2;
    if (act_bytes > (size_t)kGvActBytes) return W4A16_EUNSUPPORTED;
    const uint32_t ab = (uint32_t)act_bytes;
    if (a_dtype == W4A16_BF16) {
        if (M <= 1) return launch_group<1, __nv_bfloat16>(A, M, K, tiled, N, group, sym, C, splits, ab, stream);
        return launch_group<2, __nv_bfloat16>(A, M, K, tiled, N, group, sym, C, splits, ab, stream);
    }
    if (M <= 1) return launch_group<1, __half>(A, M, K, tiled, N, group, sym, C, splits, ab, stream);
    return launch_group<2, __half>(A, M, K, tiled, N, group, sym, C, splits, ab, stream);
}

}  // namespace w4a16
