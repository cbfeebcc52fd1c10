// awq.cu -- the AWQ activation-aware encoder: FP16 weights + 16-bit calibration inputs -> the
// plain packed W4A16 format of S W plus the input factors s (fp16, one per input channel), to be
// folded into whatever produces the layer's input (X S^-1).
//
// "4.3 Weight-only INT4", section 3 "AWQ: find channels to protect from activations":
//   3.1  a weight's importance follows the activation it multiplies: salient input channels are
//        found from the activation distribution;
//   3.2  Y = (X S^-1)(S W), Y_hat = (X S^-1) D(Q(S W)); the factors are searched on calibration
//        data and paired with clipping to control the total error.
// Readings (the page leaves the grids open; the plainest ones, as in the FP64 oracle):
//   a_j = mean_s |x_sj|; candidates s_j(alpha) = fp16(max(a_j, 2^-14)^alpha), alpha = i / 20,
//   i = 0..19, scored by ||X W - (X S^-1) D(Q(S W))||_F^2 (FP64), the first minimum wins; then per
//   group and output channel the RTN range of s w is shrunk by r = 1 - i / 20, i = 0..10, scored
//   by delta^T (X_g^T X_g) delta with delta = w - D(Q(s w)) / s, the first minimum wins.
//
// Pipeline (FP64, one stream, no host synchronisation):
//   stats     a_j                                     one thread per channel, fixed order
//   alphas    alpha_i = i / 20 on the device
//   per alpha scale (s_j), delta (W - S^-1 D(Q(S W))), then ||X Delta||^2 as per-tile partial
//             sums of a tiled FP64 GEMM and a fixed-order sum
//   pick      the first alpha with the smallest error; s for it (also written out as fp16)
//   hessian   X^T X (its diagonal g x g blocks are read)
//   clip      one warp per (group, 32 output channels): every ratio scored, the best one's
//             codes, scale and zero written
#include <type_traits>

#include "common.cuh"

namespace w4a16 {

namespace {

constexpr int kAwqAlphas = 20;
constexpr int kAwqClips = 11;
constexpr int kErrTile = 64;     // ||X Delta||^2: output tile (calibration rows x channels)
constexpr int kErrK = 16;

__device__ __forceinline__ uint16_t f64_to_f16_bits_rn(double x) {
    uint16_t h;
    asm("cvt.rn.f16.f64 %0, %1;" : "=h"(h) : "d"(x));
    return h;
}

__device__ __forceinline__ double f16_bits_to_f64(uint16_t h) {
    return (double)__half2float(__ushort_as_half(h));
}

template <typename T>
__device__ __forceinline__ double act_to_f64(uint16_t bits) {
    if constexpr (std::is_same<T, __half>::value) return (double)__half2float(__ushort_as_half(bits));
    return (double)__uint_as_float((uint32_t)bits << 16);
}

// RTN of one value with a group's (clipped) parameters: the group's scale and zero from its
// range (lo, hi) or amax shrunk by r, then the code and the dequantized value (q - z) s.
struct Rtn {
    uint16_t sbits;
    double s;
    int z;
    bool degen;
    __device__ __forceinline__ void set(double lo, double hi, double amax, double r, bool sym) {
        sbits = sym ? f64_to_f16_bits_rn(r * amax / 7.0) : f64_to_f16_bits_rn((r * hi - r * lo) / 15.0);
        s = f16_bits_to_f64(sbits);
        degen = s == 0.0;
        z = 0;
        if (degen) {
            sbits = 0x3C00;
            s = 1.0;
        } else if (!sym) {
            double zr = rint(-(r * lo) / s);
            z = (int)(zr < 0.0 ? 0.0 : (zr > 15.0 ? 15.0 : zr));
        }
    }
    __device__ __forceinline__ int code(double v, bool sym) const {
        if (sym) {
            double t = rint(v / s);
            t = t < -8.0 ? -8.0 : (t > 7.0 ? 7.0 : t);
            return degen ? 0 : (int)t;
        }
        double t = rint(v / s) + z;
        t = t < 0.0 ? 0.0 : (t > 15.0 ? 15.0 : t);
        return degen ? z : (int)t;
    }
    __device__ __forceinline__ double deq(int q, bool sym) const { return sym ? q * s : (q - z) * s; }
};

template <typename T>
__global__ void __launch_bounds__(256) awq_stats_kernel(const uint16_t* __restrict__ X, int S, int K,
                                                        double* __restrict__ a) {
    const int j = blockIdx.x * 256 + threadIdx.x;
    if (j >= K) return;
    double acc = 0.0;
    for (int s = 0; s < S; ++s) acc += fabs(act_to_f64<T>(X[(size_t)s * K + j]));
    a[j] = acc / S;
}

__global__ void awq_alphas_kernel(double* __restrict__ alphas) {
    if (threadIdx.x < kAwqAlphas) alphas[threadIdx.x] = threadIdx.x / 20.0;
}

// s_j = fp16(max(a_j, 2^-14) ^ alpha); alpha read from the device (alphas[*idx] when idx is
// given, else alphas[i]).
__global__ void __launch_bounds__(256) awq_scale_kernel(const double* __restrict__ a, int K, const double* alphas, int i,
                                                        const int* idx, double* __restrict__ s,
                                                        uint16_t* __restrict__ s_bits) {
    const int j = blockIdx.x * 256 + threadIdx.x;
    if (j >= K) return;
    const double alpha = alphas[idx ? *idx : i];
    const uint16_t b = f64_to_f16_bits_rn(pow(fmax(a[j], 0x1p-14), alpha));
    s[j] = f16_bits_to_f64(b);
    if (s_bits) s_bits[j] = b;
}

// Delta[k, n] = w_kn - D(Q(s w))_kn / s_k for r = 1 (no clipping): one thread per (group, n).
__global__ void __launch_bounds__(256) awq_delta_kernel(const uint16_t* __restrict__ W, const double* __restrict__ s,
                                                        int K, int N, int group, int sym, double* __restrict__ Delta) {
    const int n = blockIdx.x * 256 + threadIdx.x;
    const int g = blockIdx.y;
    if (n >= N) return;
    const int k0 = g * group;
    double lo = 0.0, hi = 0.0, amax = 0.0;
    for (int k = k0; k < k0 + group; ++k) {
        const double v = f16_bits_to_f64(W[(size_t)k * N + n]) * s[k];
        lo = v < lo ? v : lo;
        hi = v > hi ? v : hi;
        amax = fabs(v) > amax ? fabs(v) : amax;
    }
    Rtn q;
    q.set(lo, hi, amax, 1.0, sym != 0);
    for (int k = k0; k < k0 + group; ++k) {
        const double w = f16_bits_to_f64(W[(size_t)k * N + n]);
        const double v = w * s[k];
        Delta[(size_t)k * N + n] = w - q.deq(q.code(v, sym != 0), sym != 0) / s[k];
    }
}

// Partial sums of ||X Delta||^2: a 64 x 64 tile of X Delta per CTA (256 threads, 4 x 4 each),
// k in chunks of 16 in increasing order; each CTA writes the sum of squares of its tile to
// part[tile] (a fixed place, so the total is summed in a fixed order afterwards).
template <typename T>
__global__ void __launch_bounds__(256)
awq_err_kernel(const uint16_t* __restrict__ X, const double* __restrict__ Delta, int S, int K, int N,
               double* __restrict__ part) {
    __shared__ double xt[kErrK][kErrTile + 1];   // xt[k][s - s0]
    __shared__ double dt[kErrK][kErrTile + 1];   // dt[k][n - n0]
    __shared__ double red[256];
    const int s0 = blockIdx.y * kErrTile, n0 = blockIdx.x * kErrTile;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    double acc[4][4] = {};
    for (int k0 = 0; k0 < K; k0 += kErrK) {
        for (int e = threadIdx.x; e < kErrK * kErrTile; e += 256) {
            const int c = e % kErrTile, kk = e / kErrTile;
            const int sx = e / kErrK, kx = e % kErrK;   // X tile read along k (rows of X)
            xt[kx][sx] = (s0 + sx < S && k0 + kx < K) ? act_to_f64<T>(X[(size_t)(s0 + sx) * K + k0 + kx]) : 0.0;
            dt[kk][c] = (k0 + kk < K && n0 + c < N) ? Delta[(size_t)(k0 + kk) * N + n0 + c] : 0.0;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < kErrK; ++kk) {
            double xa[4], db[4];
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                xa[x] = xt[kk][ty + 16 * x];
                db[x] = dt[kk][tx + 16 * x];
            }
#pragma unroll
            for (int x = 0; x < 4; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) acc[x][y] = fma(xa[x], db[y], acc[x][y]);
        }
        __syncthreads();
    }
    double sq = 0.0;
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) sq = fma(acc[x][y], acc[x][y], sq);   // rows / columns outside are 0
    red[threadIdx.x] = sq;
    __syncthreads();
    for (int w = 128; w > 0; w >>= 1) {
        if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) part[blockIdx.y * gridDim.x + blockIdx.x] = red[0];
}

// errs[i] = sum of the partial sums, in index order (one CTA).
__global__ void __launch_bounds__(256) awq_sum_kernel(const double* __restrict__ part, int n, double* __restrict__ out) {
    __shared__ double red[256];
    double s = 0.0;
    for (int i = threadIdx.x; i < n; i += 256) s += part[i];
    red[threadIdx.x] = s;
    __syncthreads();
    for (int w = 128; w > 0; w >>= 1) {
        if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) *out = red[0];
}

// The first alpha with the smallest error.
__global__ void awq_pick_kernel(const double* __restrict__ errs, int* __restrict__ idx) {
    if (threadIdx.x != 0) return;
    int best = 0;
    for (int i = 1; i < kAwqAlphas; ++i)
        if (errs[i] < errs[best]) best = i;
    *idx = best;
}

// Clip search and output: one warp per (group g = blockIdx.y, channels 32 blockIdx.x + lane).
// delta for a ratio sits in shared memory [group][32]; the group's block of H = 2 X^T X is read
// from global memory (every lane reads the same entry). The factor 2 does not move the minimum.
__global__ void __launch_bounds__(32)
awq_clip_kernel(const uint16_t* __restrict__ W, const double* __restrict__ s, const double* __restrict__ H, int K,
                int N, int group, int sym, int32_t* __restrict__ codes, uint16_t* __restrict__ scales,
                int32_t* __restrict__ zeros) {
    __shared__ double d[128][32];
    const int lane = threadIdx.x;
    const int n = blockIdx.x * 32 + lane;
    const bool active = n < N;
    const int g = blockIdx.y, k0 = g * group;
    const bool sy = sym != 0;
    double lo = 0.0, hi = 0.0, amax = 0.0;
    for (int k = k0; k < k0 + group; ++k) {
        const double v = active ? f16_bits_to_f64(W[(size_t)k * N + n]) * s[k] : 0.0;
        lo = v < lo ? v : lo;
        hi = v > hi ? v : hi;
        amax = fabs(v) > amax ? fabs(v) : amax;
    }
    double best_err = 0.0;
    int best = 0;
    for (int ci = 0; ci < kAwqClips; ++ci) {
        const double r = 1.0 - ci / 20.0;
        Rtn q;
        q.set(lo, hi, amax, r, sy);
        for (int a = 0; a < group; ++a) {
            const int k = k0 + a;
            const double w = active ? f16_bits_to_f64(W[(size_t)k * N + n]) : 0.0;
            d[a][lane] = w - q.deq(q.code(w * s[k], sy), sy) / s[k];
        }
        double err = 0.0;
        for (int a = 0; a < group; ++a) {
            const double* h = H + (size_t)(k0 + a) * K + k0;
            double t = 0.0;
            for (int b = 0; b < group; ++b) t = fma(h[b], d[b][lane], t);
            err = fma(d[a][lane], t, err);
        }
        if (ci == 0 || err < best_err) {
            best_err = err;
            best = ci;
        }
    }
    Rtn q;
    q.set(lo, hi, amax, 1.0 - best / 20.0, sy);
    if (active) scales[(size_t)g * N + n] = q.sbits;
    for (int j = k0 / 8; j < (k0 + group) / 8; ++j) {
        uint32_t word = 0;
        for (int i = 0; i < 8; ++i) {
            const int k = 8 * j + i;
            const double w = active ? f16_bits_to_f64(W[(size_t)k * N + n]) : 0.0;
            word |= ((uint32_t)q.code(w * s[k], sy) & 0xFu) << (4 * i);
        }
        if (active) codes[(size_t)j * N + n] = (int32_t)word;
    }
    if (!sy) {
        uint32_t zw = (uint32_t)q.z << (4 * (n & 7));
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) zw |= __shfl_xor_sync(0xffffffffu, zw, o);
        if (active && (n & 7) == 0) zeros[(size_t)g * (N / 8) + n / 8] = (int32_t)zw;
    }
}

struct AwqWs {
    double *a, *s, *alphas, *errs, *part, *Delta, *H;
    int* idx;
    size_t nparts;
};

AwqWs awq_carve(void* workspace, int K, int N, int S) {
    AwqWs w;
    double* p = static_cast<double*>(workspace);
    w.a = p;
    w.s = w.a + K;
    w.alphas = w.s + K;
    w.errs = w.alphas + 32;
    w.nparts = (size_t)((N + kErrTile - 1) / kErrTile) * ((S + kErrTile - 1) / kErrTile);
    w.part = w.errs + 32;
    w.Delta = w.part + ((w.nparts + 1) & ~(size_t)1);
    w.H = w.Delta + (size_t)K * N;
    w.idx = reinterpret_cast<int*>(w.H + (size_t)K * K);
    return w;
}

}  // namespace

size_t awq_workspace_bytes(int K, int N, int S) {
    const size_t nparts = (size_t)((N + kErrTile - 1) / kErrTile) * ((S + kErrTile - 1) / kErrTile);
    return sizeof(double) * (2 * (size_t)K + 64 + ((nparts + 1) & ~(size_t)1) + (size_t)K * N + (size_t)K * K) + 256;
}

int launch_awq(const void* W, const void* X, int x_dtype, int S, int K, int N, int group, int sym, int32_t* codes,
               void* scales, int32_t* zeros, void* s_in, void* workspace, int* dev_status, cudaStream_t stream) {
    (void)dev_status;
    const AwqWs w = awq_carve(workspace, K, N, S);
    const uint16_t* Wb = static_cast<const uint16_t*>(W);
    const uint16_t* Xb = static_cast<const uint16_t*>(X);
    const bool bf = x_dtype == W4A16_BF16;
    const unsigned kb = (unsigned)((K + 255) / 256);
    if (bf)
        awq_stats_kernel<__nv_bfloat16><<<kb, 256, 0, stream>>>(Xb, S, K, w.a);
    else
        awq_stats_kernel<__half><<<kb, 256, 0, stream>>>(Xb, S, K, w.a);
    awq_alphas_kernel<<<1, 32, 0, stream>>>(w.alphas);
    const dim3 dg((N + 255) / 256, K / group);
    const dim3 eg((N + kErrTile - 1) / kErrTile, (S + kErrTile - 1) / kErrTile);
    for (int i = 0; i < kAwqAlphas; ++i) {
        awq_scale_kernel<<<kb, 256, 0, stream>>>(w.a, K, w.alphas, i, nullptr, w.s, nullptr);
        awq_delta_kernel<<<dg, 256, 0, stream>>>(Wb, w.s, K, N, group, sym, w.Delta);
        if (bf)
            awq_err_kernel<__nv_bfloat16><<<eg, 256, 0, stream>>>(Xb, w.Delta, S, K, N, w.part);
        else
            awq_err_kernel<__half><<<eg, 256, 0, stream>>>(Xb, w.Delta, S, K, N, w.part);
        awq_sum_kernel<<<1, 256, 0, stream>>>(w.part, (int)w.nparts, w.errs + i);
    }
    awq_pick_kernel<<<1, 32, 0, stream>>>(w.errs, w.idx);
    awq_scale_kernel<<<kb, 256, 0, stream>>>(w.a, K, w.alphas, 0, w.idx, w.s, static_cast<uint16_t*>(s_in));
    launch_hessian(X, x_dtype, S, K, w.H, stream);
    const dim3 cg((N + 31) / 32, K / group);
    awq_clip_kernel<<<cg, 32, 0, stream>>>(Wb, w.s, w.H, K, N, group, sym, codes, static_cast<uint16_t*>(scales),
                                            zeros);
    return launch_status();
}

}  // namespace w4a16
