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
//   factor    U = V^-1 by recursive halving of the channel range (V's panels kept transposed in
//             H's lower triangle), down to 64-channel blocks factored and inverted by one CTA;
//             every other step is a tiled FP64 product of 64 x 64 output tiles
//   widen     W (fp16) -> FP64 working copy
//   block b   channels b0 .. b0+127, 32 output channels per CTA: the block's channels are
//             quantized in order, compensating inside the block at once and recording e_i; then
//   trailing  W[b0+128:, :] -= U[block, b0+128:]^T E[block, :]  (FP64 tiled GEMM)
// The group parameters (RTN: FP16 scale rounded once from the FP64 quotient, optional INT4 zero)
// are taken from a group's compensated weights when its first channel comes up, as the FP64
// oracle does.
#include <type_traits>

#include "common.cuh"

namespace w4a16 {

namespace {

constexpr int kGptqBlock = 128;     // channels per block update
constexpr int kGptqWarps = 8;       // warps of the block kernel (each owns every 8th row)
constexpr int kGptqThreads = 32 * kGptqWarps;   // block kernel: 32 output channels per CTA
constexpr int kTrailTile = 64;      // trailing GEMM output tile (rows x columns)
constexpr int kTrailK = 16;         // trailing GEMM k-chunk
constexpr int kCholBlock = 64;      // leaf block and tile size of the recursive factorisation
constexpr int kCP = kCholBlock + 1; // padded shared-memory row pitch (doubles)
constexpr int kCholK = 16;          // k-chunk of the tiled products

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

// 8-byte asynchronous global -> shared copy; ok == false writes zero and reads nothing.
__device__ __forceinline__ void async_copy8(double* dst, const double* src, bool ok) {
    const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(d), "l"(src), "r"(ok ? 8 : 0) : "memory");
}
__device__ __forceinline__ void async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

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

// ---- Recursive reverse Cholesky and triangular inverse -----------------------------------------
// factor(lo, hi) turns H'[lo:hi, lo:hi] (the damped H with the updates of the channels after hi
// subtracted) into U[lo:hi, lo:hi], the inverse of its reverse Cholesky factor. With
// A = [lo, mid), C = [mid, hi) and V the factor, [[V_A, V_B], [0, V_C]] [[V_A, V_B], [0, V_C]]^T
// = H' gives V_C = rchol(H'_C), V_B = H'_AC V_C^-T, V_A = rchol(H'_A - V_B V_B^T), and the inverse
// of a block upper-triangular matrix gives U_AC = -U_A V_B U_C. So:
//   factor(C); panel V_B = H'_AC U_C^T; syrk H'_A -= V_B V_B^T; factor(A);
//   tmul T = V_B U_C; uleft U_AC = -U_A T
// down to blocks of 64 channels, which one CTA factors and inverts in shared memory. Storage, in
// the K x K matrix Hm that holds H: its upper triangle holds H' (updated in place by syrk), V_B^T
// goes to the lower triangle (rows C, columns A; H's lower triangle is never read), and T goes to
// the upper triangle at A x C once panel has consumed H'_AC. V itself is never needed whole. U is
// written on and above its diagonal only. In every step the region written is disjoint from the
// regions read.

// One block D = [d0, d0 + nb), nb <= 64: right-looking reverse Cholesky of H'_DD in shared memory
// (for j = nb-1 .. 0: v_jj = sqrt(a_jj), a_ij /= v_jj for i < j, then a_ik -= a_ij a_kj for
// i <= k < j), then back substitution per column for U_DD = V_DD^-1.
__global__ void __launch_bounds__(256) chol_diag_kernel(const double* __restrict__ Hm, double* __restrict__ U,
                                                        int K, int d0, int nb, int* dev_status) {
    extern __shared__ double sm[];
    double* a = sm;                          // a[r * kCP + c]
    double* w = sm + kCholBlock * kCP;       // w[r * kCP + c] = U_DD
    const int tid = threadIdx.x;
    for (int e = tid; e < nb * nb; e += 256) {
        const int r = e / nb, c = e % nb;
        a[r * kCP + c] = r <= c ? Hm[(size_t)(d0 + r) * K + d0 + c] : 0.0;
    }
    __syncthreads();
    for (int j = nb - 1; j >= 0; --j) {
        const double d = a[j * kCP + j];
        const double vjj = d > 0.0 ? sqrt(d) : __longlong_as_double(0x7FF8000000000000ll);
        for (int i = tid; i < j; i += 256) a[i * kCP + j] /= vjj;
        __syncthreads();
        if (tid == 0) {
            if (!(d > 0.0)) report_status(dev_status, W4A16_ENONFINITE);   // H + damping is not positive definite
            a[j * kCP + j] = vjj;
        }
        for (int e = tid; e < j * j; e += 256) {
            const int i = e / j, k = e % j;
            if (i <= k) a[i * kCP + k] = fma(-a[i * kCP + j], a[k * kCP + j], a[i * kCP + k]);
        }
        __syncthreads();
    }
    // thread c owns column c: u_cc = 1 / v_cc, u_ic = -(sum_{k=i+1..c} v_ik u_kc) / v_ii
    for (int c = tid; c < nb; c += 256) {
        w[c * kCP + c] = 1.0 / a[c * kCP + c];
        for (int i = c - 1; i >= 0; --i) {
            double s = 0.0;
            for (int k = i + 1; k <= c; ++k) s = fma(a[i * kCP + k], w[k * kCP + c], s);
            w[i * kCP + c] = -s / a[i * kCP + i];
        }
    }
    __syncthreads();
    for (int e = tid; e < nb * nb; e += 256) {
        const int r = e / nb, c = e % nb;
        if (r <= c) U[(size_t)(d0 + r) * K + d0 + c] = w[r * kCP + c];
    }
}

enum CholOp { kOpPanel, kOpSyrk, kOpTmul, kOpUleft };

// One 64 x 64 output tile of a factor() product: out[i, j] = sum_k L(i, k) R(k, j), k increasing.
//   op      rows i   cols j   k range               L(i, k)              R(k, j)          result
//   panel   C        A        [i, hi)               U[i, k]  (k >= i)    Hm[j, k]         Hm[i, j] = out
//   syrk    A        A, i<=j  [mid, hi)             Hm[k, i]             Hm[k, j]         Hm[i, j] -= out
//   tmul    A        C        [mid, min(tile, hi))  Hm[k, i]             U[k, j] (k <= j) Hm[i, j] = out
//   uleft   A        C        [i, mid)              U[i, k]  (k >= i)    Hm[k, j]         U[i, j] = -out
// Operands are staged in chunks of 16 k, transposed to [k][row], with the load mapping following
// each operand's contiguous index, and the next chunk copied (cp.async, two buffers) while this
// one is multiplied; masked and out-of-range entries read as zero.
template <int OP>
__global__ void __launch_bounds__(256, 4) chol_tile_kernel(double* __restrict__ Hm, double* __restrict__ U, int K,
                                                        int lo, int mid, int hi) {
    __shared__ double lt[2][kCholK * kCP], rt[2][kCholK * kCP];
    int i0, j0, iend, jend, klo, khi;
    if (OP == kOpSyrk) {
        const int x = blockIdx.x;
        int J = (int)((sqrt(8.0 * x + 1.0) - 1.0) * 0.5);
        while ((J + 1) * (J + 2) / 2 <= x) ++J;
        while (J * (J + 1) / 2 > x) --J;
        i0 = lo + (x - J * (J + 1) / 2) * kCholBlock;
        j0 = lo + J * kCholBlock;
        iend = jend = mid;
        klo = mid;
        khi = hi;
    } else if (OP == kOpPanel) {
        i0 = mid + blockIdx.y * kCholBlock;
        j0 = lo + blockIdx.x * kCholBlock;
        iend = hi;
        jend = mid;
        klo = i0;
        khi = hi;
    } else {
        i0 = lo + blockIdx.y * kCholBlock;
        j0 = mid + blockIdx.x * kCholBlock;
        iend = mid;
        jend = hi;
        klo = OP == kOpTmul ? mid : i0;
        khi = OP == kOpTmul ? (j0 + kCholBlock < hi ? j0 + kCholBlock : hi) : mid;
    }
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    // Element e of a chunk is split as (row, kk) along the operand's contiguous index: L is
    // contiguous in k (U[i, k]) for panel / uleft and in i (Hm[k, i]) otherwise; R is contiguous in
    // k (Hm[j, k]) for panel and in j otherwise.
    constexpr bool kLRowK = OP == kOpPanel || OP == kOpUleft;
    constexpr bool kRRowK = OP == kOpPanel;
    const double* R = OP == kOpTmul ? U : Hm;
    auto issue = [&](int k0, int buf) {
        double* lb = lt[buf];
        double* rb = rt[buf];
        for (int e = threadIdx.x; e < kCholK * kCholBlock; e += 256) {
            int r = kLRowK ? e / kCholK : e % kCholBlock, kk = kLRowK ? e % kCholK : e / kCholBlock;
            int i = i0 + r, k = k0 + kk;
            if (kLRowK) {
                const bool ok = i < iend && k < khi && k >= i;
                async_copy8(lb + kk * kCP + r, ok ? U + (size_t)i * K + k : U, ok);
            } else {
                const bool ok = i < iend && k < khi;
                async_copy8(lb + kk * kCP + r, ok ? Hm + (size_t)k * K + i : Hm, ok);
            }
            r = kRRowK ? e / kCholK : e % kCholBlock;
            kk = kRRowK ? e % kCholK : e / kCholBlock;
            const int j = j0 + r;
            k = k0 + kk;
            if (kRRowK) {
                const bool ok = j < jend && k < khi;
                async_copy8(rb + kk * kCP + r, ok ? Hm + (size_t)j * K + k : Hm, ok);
            } else {
                const bool ok = j < jend && k < khi && (OP != kOpTmul || k <= j);
                async_copy8(rb + kk * kCP + r, ok ? R + (size_t)k * K + j : R, ok);
            }
        }
        async_commit();
    };
    double acc[4][4] = {};
    issue(klo, 0);
    for (int k0 = klo, buf = 0; k0 < khi; k0 += kCholK, buf ^= 1) {
        if (k0 + kCholK < khi) {   // the next chunk's copies overlap this chunk's FMAs
            issue(k0 + kCholK, buf ^ 1);
            async_wait<1>();
        } else {
            async_wait<0>();
        }
        __syncthreads();
        const double* lb = lt[buf];
        const double* rb = rt[buf];
#pragma unroll
        for (int kk = 0; kk < kCholK; ++kk) {
            double x4[4], y4[4];
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                x4[x] = lb[kk * kCP + ty + 16 * x];
                y4[x] = rb[kk * kCP + tx + 16 * x];
            }
#pragma unroll
            for (int x = 0; x < 4; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) acc[x][y] = fma(x4[x], y4[y], acc[x][y]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) {
            const int i = i0 + ty + 16 * x, j = j0 + tx + 16 * y;
            if (i >= iend || j >= jend) continue;
            if (OP == kOpPanel || OP == kOpTmul) Hm[(size_t)i * K + j] = acc[x][y];
            else if (OP == kOpSyrk) { if (i <= j) Hm[(size_t)i * K + j] -= acc[x][y]; }
            else U[(size_t)i * K + j] = -acc[x][y];
        }
}

// Host recursion of factor(lo, hi); the split puts half of the 64-channel blocks (rounded down)
// in A, so every boundary but hi = K is a multiple of 64.
void chol_factor(double* Hm, double* U, int K, int lo, int hi, size_t diag_smem, int* dev_status,
                 cudaStream_t stream) {
    if (hi - lo <= kCholBlock) {
        chol_diag_kernel<<<1, 256, diag_smem, stream>>>(Hm, U, K, lo, hi - lo, dev_status);
        return;
    }
    const int nblk = (hi - lo + kCholBlock - 1) / kCholBlock;
    const int mid = lo + kCholBlock * (nblk / 2);
    const unsigned ta = (unsigned)((mid - lo) / kCholBlock), tc = (unsigned)((hi - mid + kCholBlock - 1) / kCholBlock);
    chol_factor(Hm, U, K, mid, hi, diag_smem, dev_status, stream);
    chol_tile_kernel<kOpPanel><<<dim3(ta, tc), 256, 0, stream>>>(Hm, U, K, lo, mid, hi);
    chol_tile_kernel<kOpSyrk><<<ta * (ta + 1) / 2, 256, 0, stream>>>(Hm, U, K, lo, mid, hi);
    chol_factor(Hm, U, K, lo, mid, diag_smem, dev_status, stream);
    chol_tile_kernel<kOpTmul><<<dim3(tc, ta), 256, 0, stream>>>(Hm, U, K, lo, mid, hi);
    chol_tile_kernel<kOpUleft><<<dim3(tc, ta), 256, 0, stream>>>(Hm, U, K, lo, mid, hi);
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

// One block of channels [b0, b0 + nb) for 32 output channels (lane = channel n): the block's
// weights sit in shared memory, and warp v owns the block rows r with r % 8 == v. Row r is
// quantized by its owner with its group's parameters, e_r goes to shared memory (and to E for the
// trailing update), and after a barrier every warp applies w_c -= e_r U_rc to its own rows c > r.
// Each weight thus receives its updates in increasing r, as in the sequential statement. A
// group's parameters come from its compensated weights when its first row comes up: each warp
// reduces min / max / max|w| over its rows of the group, and every warp combines the eight
// partial results (exact operations, so all warps hold the same parameters). The block's triangle
// of U is staged in shared memory first.
template <bool SYM>
__global__ void __launch_bounds__(kGptqThreads)
gptq_block_kernel(double* __restrict__ Wd, const double* __restrict__ U, int K, int N, int b0, int nb, int group,
                  double* __restrict__ E, int32_t* __restrict__ codes, uint16_t* __restrict__ scales,
                  int32_t* __restrict__ zeros) {
    __shared__ double w[kGptqBlock][32];
    __shared__ double es[2][32];
    __shared__ double red[3][kGptqWarps][32];
    __shared__ uint8_t qs[kGptqBlock][32];
    extern __shared__ double ut[];   // U's block triangle: row r, columns r .. nb-1, at tri_off(r)
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int n = blockIdx.x * 32 + lane;
    const bool active = n < N;
    auto tri_off = [nb](int r) { return r * nb - r * (r - 1) / 2; };
    for (int r = warp; r < nb; r += kGptqWarps) {
        w[r][lane] = active ? Wd[(size_t)(b0 + r) * N + n] : 0.0;
        for (int c = r + lane; c < nb; c += 32) ut[tri_off(r) + c - r] = U[(size_t)(b0 + r) * K + b0 + c];
    }
    __syncthreads();
    double s = 1.0;
    int z = 0;
    bool degen = false;
    for (int r = 0; r < nb; ++r) {
        const int i = b0 + r;
        if (i % group == 0) {
            __syncthreads();   // the updates of the rows before r are in place
            double lo = 0.0, hi = 0.0, amax = 0.0;
            for (int c = r + ((warp - r) & (kGptqWarps - 1)); c < r + group; c += kGptqWarps) {
                const double v = w[c][lane];
                lo = v < lo ? v : lo;
                hi = v > hi ? v : hi;
                amax = fabs(v) > amax ? fabs(v) : amax;
            }
            red[0][warp][lane] = lo;
            red[1][warp][lane] = hi;
            red[2][warp][lane] = amax;
            __syncthreads();
#pragma unroll
            for (int v = 0; v < kGptqWarps; ++v) {
                lo = red[0][v][lane] < lo ? red[0][v][lane] : lo;
                hi = red[1][v][lane] > hi ? red[1][v][lane] : hi;
                amax = red[2][v][lane] > amax ? red[2][v][lane] : amax;
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
            if (warp == 0) {
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
            __syncthreads();   // red[] is free again before the next group
        }
        const double* urow = ut + tri_off(r) - r;   // urow[c] = U[i, b0 + c] for c >= r
        if ((r & (kGptqWarps - 1)) == warp) {
            const double v = w[r][lane];
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
            qs[r][lane] = (uint8_t)(q & 0xF);
            const double e = (v - what) / urow[r];
            es[r & 1][lane] = e;
            if (active) E[(size_t)r * N + n] = e;
        }
        __syncthreads();
        const double e = es[r & 1][lane];
        for (int c = r + 1 + ((warp - r - 1) & (kGptqWarps - 1)); c < nb; c += kGptqWarps)
            w[c][lane] = fma(-e, urow[c], w[c][lane]);
    }
    __syncthreads();
    // codes word (b0 / 8 + t, n): the eight rows of a word, first row in the low nibble
    for (int x = threadIdx.x; x < (nb / 8) * 32; x += kGptqThreads) {
        const int t = x >> 5, l = x & 31, nn = blockIdx.x * 32 + l;
        uint32_t word = 0;
#pragma unroll
        for (int b = 0; b < 8; ++b) word |= (uint32_t)qs[8 * t + b][l] << (4 * b);
        if (nn < N) codes[(size_t)(b0 / 8 + t) * N + nn] = (int32_t)word;
    }
}

// Wd[j, n] -= sum_{r < nb} U[b0 + r, j] E[r, n] for j >= b1 = b0 + nb: a 64 x 64 output tile per
// CTA (256 threads, 4 x 4 each), r in chunks of 16 through shared memory (cp.async, two buffers),
// in increasing order.
__global__ void __launch_bounds__(256, 4)
trailing_kernel(double* __restrict__ Wd, const double* __restrict__ U, const double* __restrict__ E, int K, int N,
                int b0, int nb) {
    __shared__ double ut[2][kTrailK][kTrailTile + 1];   // ut[.][r][j - j0] = U[b0 + r, j]
    __shared__ double et[2][kTrailK][kTrailTile + 1];   // et[.][r][n - n0] = E[r, n]
    const int b1 = b0 + nb;
    const int j0 = b1 + blockIdx.y * kTrailTile, n0 = blockIdx.x * kTrailTile;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    auto issue = [&](int r0, int buf) {
        for (int e = threadIdx.x; e < kTrailK * kTrailTile; e += 256) {
            const int r = e / kTrailTile, c = e % kTrailTile;
            const bool uok = r0 + r < nb && j0 + c < K, eok = r0 + r < nb && n0 + c < N;
            async_copy8(&ut[buf][r][c], uok ? U + (size_t)(b0 + r0 + r) * K + j0 + c : U, uok);
            async_copy8(&et[buf][r][c], eok ? E + (size_t)(r0 + r) * N + n0 + c : E, eok);
        }
        async_commit();
    };
    double acc[4][4] = {};
    issue(0, 0);
    for (int r0 = 0, buf = 0; r0 < nb; r0 += kTrailK, buf ^= 1) {
        if (r0 + kTrailK < nb) {   // the next chunk's copies overlap this chunk's FMAs
            issue(r0 + kTrailK, buf ^ 1);
            async_wait<1>();
        } else {
            async_wait<0>();
        }
        __syncthreads();
#pragma unroll
        for (int r = 0; r < kTrailK; ++r) {
            double a[4], b[4];
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                a[x] = ut[buf][r][ty + 16 * x];
                b[x] = et[buf][r][tx + 16 * x];
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
    double* H = reinterpret_cast<double*>(ws);          // H, then H' / V's panels / T (see factor)
    double* U = H + kk;
    double* Wd = U + kk;
    double* E = Wd + (size_t)K * N;

    launch_hessian(X, x_dtype, S, K, H, stream);
    damp_kernel<<<1, 256, 0, stream>>>(H, K, damp);
    const size_t diag_smem = 2 * kCholBlock * kCP * sizeof(double);
    if (cudaFuncSetAttribute(chol_diag_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)diag_smem) !=
        cudaSuccess)
        return W4A16_ECUDA;
    chol_factor(H, U, K, 0, K, diag_smem, dev_status, stream);
    const size_t wn = (size_t)K * N;
    widen_kernel<<<(unsigned)((wn + 255) / 256 < 4096 ? (wn + 255) / 256 : 4096), 256, 0, stream>>>(
        static_cast<const uint16_t*>(W), wn, Wd, dev_status);
    uint16_t* sc = static_cast<uint16_t*>(scales);
    const size_t tri_smem = (size_t)kGptqBlock * (kGptqBlock + 1) / 2 * sizeof(double);
    if (cudaFuncSetAttribute(gptq_block_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tri_smem) !=
            cudaSuccess ||
        cudaFuncSetAttribute(gptq_block_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tri_smem) !=
            cudaSuccess)
        return W4A16_ECUDA;
    for (int b0 = 0; b0 < K; b0 += kGptqBlock) {
        const int nb = K - b0 < kGptqBlock ? K - b0 : kGptqBlock;
        const unsigned nblk = (unsigned)((N + 31) / 32);
        if (sym)
            gptq_block_kernel<true><<<nblk, kGptqThreads, tri_smem, stream>>>(Wd, U, K, N, b0, nb, group, E, codes, sc, zeros);
        else
            gptq_block_kernel<false><<<nblk, kGptqThreads, tri_smem, stream>>>(Wd, U, K, N, b0, nb, group, E, codes, sc, zeros);
        if (b0 + nb < K) {
            const dim3 tg((N + kTrailTile - 1) / kTrailTile, (K - b0 - nb + kTrailTile - 1) / kTrailTile);
            trailing_kernel<<<tg, 256, 0, stream>>>(Wd, U, E, K, N, b0, nb);
        }
    }
    return launch_status();
}

}  // namespace w4a16
