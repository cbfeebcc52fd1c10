// gptq.cu -- the GPTQ calibrated encoder: FP16 weights + 16-bit calibration inputs -> the plain
// packed W4A16 format (the same codes / scales / zeros as w4a16_quantize produces).
//
// "4.3 Weight-only INT4", section 2 "GPTQ: quantize and compensate as you go":
//   2.1  objective ||X W - X W_hat||^2, curvature H = 2 X^T X over the input channels;
//   2.2  input channels are fixed one at a time; after channel i is set to its dequantized value,
//        the channels F still free move by -(w_i - w_hat_i) / [H_F^-1]_ii [H_F^-1]_{:,i};
//        damping is added to H, and the work is organised with a Cholesky factorisation and
//        block updates.
//
// The Cholesky form used here. Let U be the upper-triangular factor of the damped inverse,
// (H + lambda I)^-1 = U^T U. Then [H_F^-1]_{:,i} / [H_F^-1]_ii restricted to F is row i of U
// divided by U_ii, and [H_F^-1]_ii = U_ii^2, at every step (removing channel i from F leaves the
// factor U[i+1:, i+1:] of the remaining inverse). So step i is
//     e_i = (w_i - w_hat_i) / U_ii,   w_j -= e_i U_ij  for j > i.
// U is obtained without forming an inverse of H: H + lambda I = V V^T with V upper triangular
// (a Cholesky factorisation run from the last channel down), and U = V^-1.
//
// Pipeline (all FP64, one stream):
//   hessian   H = 2 X^T X                     one thread per 4 entries, fixed summation order
//   damp      H += damp * mean(diag H) * I    one block
//   rchol     V (in place of H), column j = K-1 .. 0: one launch for V_jj, one for the column
//   trinv     U = V^-1, one block per column (back substitution)
//   widen     W (fp16) -> FP64 working copy
//   block b   channels b0 .. b0+127: one thread per output channel quantizes the block's channels
//             in order, compensating inside the block at once and recording e_i; then
//   trailing  W[b0+128:, :] -= U[block, b0+128:]^T E[block, :]  (FP64 tiled GEMM)
// The group parameters (RTN: FP16 scale rounded once from the FP64 quotient, optional INT4 zero)
// are taken from a group's compensated weights when its first channel comes up, as the FP64
// oracle does.
#include <type_traits>

#include "common.cuh"

namespace w4a16 {

namespace {

constexpr int kGptqBlock = 128;     // channels per block update
constexpr int kGptqThreads = 32;    // output channels per CTA (one warp) of the block kernel
constexpr int kTrailTile = 64;      // trailing GEMM output tile (rows x columns)
constexpr int kTrailK = 16;         // trailing GEMM k-chunk

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

// H[i, j] = 2 sum_s X[s, i] X[s, j]. A 32 x 32 tile per CTA (32 x 8 threads, 4 rows each),
// X staged through shared memory 32 samples at a time; every entry sums s in increasing order.
template <typename T>
__global__ void __launch_bounds__(256) hessian_kernel(const uint16_t* __restrict__ X, int S, int K,
                                                      double* __restrict__ H) {
    __shared__ double xi[32][33], xj[32][33];
    const int i0 = blockIdx.y * 32, j0 = blockIdx.x * 32;
    const int tx = threadIdx.x, ty = threadIdx.y;
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
    for (int s0 = 0; s0 < S; s0 += 32) {
        for (int r = ty; r < 32; r += 8) {
            const int s = s0 + r;
            xi[r][tx] = (s < S && i0 + tx < K) ? act_to_f64<T>(X[(size_t)s * K + i0 + tx]) : 0.0;
            xj[r][tx] = (s < S && j0 + tx < K) ? act_to_f64<T>(X[(size_t)s * K + j0 + tx]) : 0.0;
        }
        __syncthreads();
        for (int r = 0; r < 32; ++r)
#pragma unroll
            for (int a = 0; a < 4; ++a) acc[a] = fma(xi[r][ty + 8 * a], xj[r][tx], acc[a]);
        __syncthreads();
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        const int i = i0 + ty + 8 * a, j = j0 + tx;
        if (i < K && j < K) H[(size_t)i * K + j] = 2.0 * acc[a];
    }
}

// H += damp * mean(diag H) * I (one CTA; the mean is summed in a fixed order).
__global__ void __launch_bounds__(256) damp_kernel(double* __restrict__ H, int K, double damp) {
    __shared__ double part[256];
    double s = 0.0;
    for (int i = threadIdx.x; i < K; i += 256) s += H[(size_t)i * K + i];
    part[threadIdx.x] = s;
    __syncthreads();
    for (int w = 128; w > 0; w >>= 1) {
        if (threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
        __syncthreads();
    }
    const double add = damp * (part[0] / K);
    for (int i = threadIdx.x; i < K; i += 256) H[(size_t)i * K + i] += add;
}

// Warp dot product of a[lo..hi) and b[lo..hi), summed lane-strided then by a fixed tree.
__device__ __forceinline__ double warp_dot(const double* a, const double* b, int lo, int hi, int lane) {
    double s = 0.0;
    for (int k = lo + lane; k < hi; k += 32) s = fma(a[k], b[k], s);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    return s;
}

// Reverse Cholesky, column j (run for j = K-1 down to 0): H = V V^T with V upper triangular,
// V_jj = sqrt(H_jj - sum_{k>j} V_jk^2); V_ij = (H_ij - sum_{k>j} V_ik V_jk) / V_jj for i < j.
// V overwrites the upper triangle of H in place (H_ij is read only by the step that writes V_ij).
__global__ void rchol_diag_kernel(double* __restrict__ V, int K, int j, int* dev_status) {
    const int lane = threadIdx.x;
    const double* row = V + (size_t)j * K;
    const double d = V[(size_t)j * K + j] - warp_dot(row, row, j + 1, K, lane);
    if (lane == 0) {
        if (!(d > 0.0)) {
            report_status(dev_status, W4A16_ENONFINITE);   // H + damping is not positive definite
            V[(size_t)j * K + j] = __longlong_as_double(0x7FF8000000000000ll);
        } else {
            V[(size_t)j * K + j] = sqrt(d);
        }
    }
}

__global__ void __launch_bounds__(256) rchol_col_kernel(double* __restrict__ V, int K, int j) {
    const int lane = threadIdx.x & 31;
    const int i = blockIdx.x * 8 + (threadIdx.x >> 5);   // one warp per row i < j
    if (i >= j) return;
    const double* rj = V + (size_t)j * K;
    const double* ri = V + (size_t)i * K;
    const double dot = warp_dot(ri, rj, j + 1, K, lane);
    if (lane == 0) V[(size_t)i * K + j] = (ri[j] - dot) / rj[j];
}

// U = V^-1 (both upper triangular), one CTA (one warp) per column j: U_jj = 1 / V_jj and, for
// i = j-1 down to 0, U_ij = -(sum_{k=i+1..j} V_ik U_kj) / V_ii, with column j kept in shared
// memory. The lower triangle of U is written as zero.
__global__ void __launch_bounds__(32) trinv_kernel(const double* __restrict__ V, int K, double* __restrict__ U) {
    extern __shared__ double u[];   // [K]
    const int j = blockIdx.x, lane = threadIdx.x;
    for (int k = lane; k < K; k += 32) u[k] = 0.0;
    __syncwarp();
    if (lane == 0) u[j] = 1.0 / V[(size_t)j * K + j];
    __syncwarp();
    for (int i = j - 1; i >= 0; --i) {
        const double* vi = V + (size_t)i * K;
        const double dot = warp_dot(vi, u, i + 1, j + 1, lane);
        if (lane == 0) u[i] = -dot / vi[i];
        __syncwarp();
    }
    for (int k = lane; k < K; k += 32) U[(size_t)k * K + j] = u[k];
}

// fp16 W -> FP64 working copy; a non-finite weight is reported (its group's codes are then
// unspecified).
__global__ void __launch_bounds__(256) widen_kernel(const uint16_t* __restrict__ W, size_t n, double* __restrict__ Wd,
                                                    int* dev_status) {
    for (size_t i = (size_t)blockIdx.x * 256 + threadIdx.x; i < n; i += (size_t)gridDim.x * 256) {
        const double w = f16_bits_to_f64(W[i]);
        if (!isfinite(w)) report_status(dev_status, W4A16_ENONFINITE);
        Wd[i] = w;
    }
}

// One block of channels [b0, b0 + nb): thread = output channel n. Its nb weights sit in shared
// memory (column n of the block); channel i is quantized with its group's parameters, the rest
// of the block is compensated at once, and e_i goes to E for the trailing update.
template <bool SYM>
__global__ void __launch_bounds__(kGptqThreads)
gptq_block_kernel(double* __restrict__ Wd, const double* __restrict__ U, int K, int N, int b0, int nb, int group,
                  double* __restrict__ E, int32_t* __restrict__ codes, uint16_t* __restrict__ scales,
                  int32_t* __restrict__ zeros) {
    __shared__ double w[kGptqBlock][kGptqThreads];
    const int tid = threadIdx.x;
    const int n = blockIdx.x * kGptqThreads + tid;
    const bool active = n < N;
    for (int r = 0; r < nb; ++r) w[r][tid] = active ? Wd[(size_t)(b0 + r) * N + n] : 0.0;
    // (each thread touches only its own column of w: no barrier is needed)
    double s = 1.0;
    int z = 0;
    bool degen = false;
    uint32_t word = 0;
    for (int r = 0; r < nb; ++r) {
        const int i = b0 + r;
        if (i % group == 0) {
            double lo = 0.0, hi = 0.0, amax = 0.0;
            for (int c = r; c < r + group; ++c) {
                const double v = w[c][tid];
                lo = v < lo ? v : lo;
                hi = v > hi ? v : hi;
                amax = fabs(v) > amax ? fabs(v) : amax;
            }
            uint16_t sb = SYM ? f64_to_f16_bits_rn(amax / 7.0) : f64_to_f16_bits_rn((hi - lo) / 15.0);
            s = f16_bits_to_f64(sb);
            degen = s == 0.0;
            z = 0;
            if (degen) {
                sb = 0x3C00;
                s = 1.0;
            } else if (!SYM) {
                double zr = rint(-lo / s);
                zr = zr < 0.0 ? 0.0 : (zr > 15.0 ? 15.0 : zr);
                z = (int)zr;
            }
            const int g = i / group;
            if (active) scales[(size_t)g * N + n] = sb;
            if (!SYM) {
                // zeros word (g, n / 8): the eight channels of a word are eight consecutive lanes
                uint32_t zw = (uint32_t)z << (4 * (n & 7));
#pragma unroll
                for (int o = 1; o < 8; o <<= 1) zw |= __shfl_xor_sync(0xffffffffu, zw, o);
                if (active && (n & 7) == 0) zeros[(size_t)g * (N / 8) + n / 8] = (int32_t)zw;
            }
        }
        const double v = w[r][tid];
        int q;
        double what;
        if (SYM) {
            double t = rint(v / s);
            t = t < -8.0 ? -8.0 : (t > 7.0 ? 7.0 : t);
            q = degen ? 0 : (int)t;
            what = q * s;
        } else {
            double t = rint(v / s) + z;
            t = t < 0.0 ? 0.0 : (t > 15.0 ? 15.0 : t);
            q = degen ? z : (int)t;
            what = (q - z) * s;
        }
        word |= ((uint32_t)q & 0xFu) << (4 * (i & 7));
        if ((i & 7) == 7) {
            if (active) codes[(size_t)(i / 8) * N + n] = (int32_t)word;
            word = 0;
        }
        const double* urow = U + (size_t)i * K + b0;
        const double e = (v - what) / urow[r];
        for (int c = r + 1; c < nb; ++c) w[c][tid] = fma(-e, __ldg(urow + c), w[c][tid]);
        if (active) E[(size_t)r * N + n] = e;
    }
}

// Wd[j, n] -= sum_{r < nb} U[b0 + r, j] E[r, n] for j >= b1 = b0 + nb: a 64 x 64 output tile per
// CTA (256 threads, 4 x 4 each), r in chunks of 16 through shared memory, in increasing order.
__global__ void __launch_bounds__(256)
trailing_kernel(double* __restrict__ Wd, const double* __restrict__ U, const double* __restrict__ E, int K, int N,
                int b0, int nb) {
    __shared__ double ut[kTrailK][kTrailTile + 1];   // ut[r][j - j0] = U[b0 + r, j]
    __shared__ double et[kTrailK][kTrailTile + 1];   // et[r][n - n0] = E[r, n]
    const int b1 = b0 + nb;
    const int j0 = b1 + blockIdx.y * kTrailTile, n0 = blockIdx.x * kTrailTile;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    double acc[4][4] = {};
    for (int r0 = 0; r0 < nb; r0 += kTrailK) {
        for (int e = threadIdx.x; e < kTrailK * kTrailTile; e += 256) {
            const int r = e / kTrailTile, c = e % kTrailTile;
            ut[r][c] = (r0 + r < nb && j0 + c < K) ? U[(size_t)(b0 + r0 + r) * K + j0 + c] : 0.0;
            et[r][c] = (r0 + r < nb && n0 + c < N) ? E[(size_t)(r0 + r) * N + n0 + c] : 0.0;
        }
        __syncthreads();
#pragma unroll
        for (int r = 0; r < kTrailK; ++r) {
            double a[4], b[4];
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                a[x] = ut[r][ty + 16 * x];
                b[x] = et[r][tx + 16 * x];
            }
#pragma unroll
            for (int x = 0; x < 4; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) acc[x][y] = fma(a[x], b[y], acc[x][y]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) {
            const int j = j0 + ty + 16 * x, n = n0 + tx + 16 * y;
            if (j < K && n < N) Wd[(size_t)j * N + n] -= acc[x][y];
        }
}

}  // namespace

void launch_hessian(const void* X, int x_dtype, int S, int K, double* H, cudaStream_t stream) {
    const dim3 hg((K + 31) / 32, (K + 31) / 32);
    const uint16_t* Xb = static_cast<const uint16_t*>(X);
    if (x_dtype == W4A16_BF16)
        hessian_kernel<__nv_bfloat16><<<hg, dim3(32, 8), 0, stream>>>(Xb, S, K, H);
    else
        hessian_kernel<__half><<<hg, dim3(32, 8), 0, stream>>>(Xb, S, K, H);
}

size_t gptq_workspace_bytes(int K, int N) {
    const size_t kk = (size_t)K * K * sizeof(double);
    return 2 * kk + (size_t)K * N * sizeof(double) + (size_t)kGptqBlock * N * sizeof(double) + 256;
}

int launch_gptq(const void* W, const void* X, int x_dtype, int S, int K, int N, int group, int sym, double damp,
                int32_t* codes, void* scales, int32_t* zeros, void* workspace, int* dev_status,
                cudaStream_t stream) {
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const size_t kk = (size_t)K * K;
    double* H = reinterpret_cast<double*>(ws);          // H, then V in place
    double* U = H + kk;
    double* Wd = U + kk;
    double* E = Wd + (size_t)K * N;

    launch_hessian(X, x_dtype, S, K, H, stream);
    damp_kernel<<<1, 256, 0, stream>>>(H, K, damp);
    for (int j = K - 1; j >= 0; --j) {
        rchol_diag_kernel<<<1, 32, 0, stream>>>(H, K, j, dev_status);
        if (j > 0) rchol_col_kernel<<<(j + 7) / 8, 256, 0, stream>>>(H, K, j);
    }
    const size_t tri_smem = (size_t)K * sizeof(double);
    if (tri_smem > 48 * 1024 &&
        cudaFuncSetAttribute(trinv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tri_smem) != cudaSuccess)
        return W4A16_ECUDA;
    trinv_kernel<<<K, 32, tri_smem, stream>>>(H, K, U);
    const size_t wn = (size_t)K * N;
    widen_kernel<<<(unsigned)((wn + 255) / 256 < 4096 ? (wn + 255) / 256 : 4096), 256, 0, stream>>>(
        static_cast<const uint16_t*>(W), wn, Wd, dev_status);
    uint16_t* sc = static_cast<uint16_t*>(scales);
    for (int b0 = 0; b0 < K; b0 += kGptqBlock) {
        const int nb = K - b0 < kGptqBlock ? K - b0 : kGptqBlock;
        const unsigned nblk = (unsigned)((N + kGptqThreads - 1) / kGptqThreads);
        if (sym)
            gptq_block_kernel<true><<<nblk, kGptqThreads, 0, stream>>>(Wd, U, K, N, b0, nb, group, E, codes, sc, zeros);
        else
            gptq_block_kernel<false><<<nblk, kGptqThreads, 0, stream>>>(Wd, U, K, N, b0, nb, group, E, codes, sc, zeros);
        if (b0 + nb < K) {
            const dim3 tg((N + kTrailTile - 1) / kTrailTile, (K - b0 - nb + kTrailTile - 1) / kTrailTile);
            trailing_kernel<<<tg, 256, 0, stream>>>(Wd, U, E, K, N, b0, nb);
        }
    }
    return launch_status();
}

}  // namespace w4a16
