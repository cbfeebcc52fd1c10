// gemv_plain.cu -- split-K CUDA-core GEMV / skinny GEMM that reads the plain packed layout.
//
// C[m, n] = sum_k A[m, k] * (q[k, n] - z[k/g, n]) * s[k/g, n], FP32 accumulation.
// "4.3 Weight-only INT4", section 1 (dequantize on chip, multiply with 16-bit activations) and
// section 4 (read, unpack, dequantize and multiply in one pass: every weight byte crosses HBM
// once). The per-group factorisation sum_g s_g * sum_{k in g} a_k (q_k - z_g) applies the scale
// once per group instead of once per weight; (q - z) is an exact small integer.
//
// Work split: a thread owns four consecutive output channels (one 16-byte load of the plain
// codes row covers them) for every row m of A and the K range of its split. blockIdx.y is the K
// split; each split writes FP32 partial sums to the workspace [splits, M, N]; a second kernel
// adds the splits in a fixed order (deterministic) and converts to the output type.
#include "common.cuh"

namespace w4a16 {

namespace {

constexpr int kThreads = 128;          // one thread = 4 columns -> 512 columns per block
constexpr int kSmemBytes = 48 * 1024;  // activations of one split, as FP32

template <int MT, typename T, bool SYM>
__global__ void __launch_bounds__(kThreads)
gemv_plain_kernel(const T* __restrict__ A, int M, int K, const int4* __restrict__ codes,
                  const __half* __restrict__ scales, const uint32_t* __restrict__ zeros, int N,
                  int group, float* __restrict__ partial, int rows_per_split) {
    extern __shared__ float a_s[];  // [MT][8 * rows_per_split]
    const int rows = K / 8;
    const int j0 = blockIdx.y * rows_per_split;
    const int j1 = min(rows, j0 + rows_per_split);
    const int kspan = 8 * (j1 - j0);
    const int kstride = 8 * rows_per_split;

    for (int idx = threadIdx.x; idx < MT * kspan; idx += kThreads) {
        const int m = idx / kspan, kk = idx - m * kspan;
        a_s[m * kstride + kk] = m < M ? Act<T>::to_f32(A[(size_t)m * K + 8 * j0 + kk]) : 0.0f;
    }
    __syncthreads();

    const int c4 = blockIdx.x * kThreads + threadIdx.x;  // index of a 4-column group
    if (4 * c4 >= N) return;
    const int n0 = 4 * c4;

    float acc[MT][4];
    float accg[MT][4];
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[m][c] = accg[m][c] = 0.0f;

    int gcur = -1;
    float s[4] = {0.f, 0.f, 0.f, 0.f};
    int z[4] = {0, 0, 0, 0};
    const int rows_per_group = group / 8;

    for (int j = j0; j < j1; ++j) {
        const int g = j / rows_per_group;
        if (g != gcur) {
            if (gcur >= 0) {
#pragma unroll
                for (int m = 0; m < MT; ++m)
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        acc[m][c] = fmaf(s[c], accg[m][c], acc[m][c]);
                        accg[m][c] = 0.0f;
                    }
            }
            gcur = g;
#pragma unroll
            for (int c = 0; c < 4; ++c) s[c] = __half2float(scales[(size_t)g * N + n0 + c]);
            if (!SYM) {
                const uint32_t zw = zeros[(size_t)g * (N / 8) + n0 / 8];
#pragma unroll
                for (int c = 0; c < 4; ++c) z[c] = nibble_u(zw, (n0 % 8) + c);
            }
        }
        const int4 w4 = codes[(size_t)j * (N / 4) + c4];
        const uint32_t wc[4] = {(uint32_t)w4.x, (uint32_t)w4.y, (uint32_t)w4.z, (uint32_t)w4.w};
        const float* a_row = a_s + 8 * (j - j0);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                float v;
                if (SYM) {
                    v = (float)((int32_t)(wc[c] << (28 - 4 * i)) >> 28);  // sign-extended nibble
                } else {
                    v = (float)(nibble_u(wc[c], i) - z[c]);
                }
#pragma unroll
                for (int m = 0; m < MT; ++m) accg[m][c] = fmaf(a_row[m * kstride + i], v, accg[m][c]);
            }
        }
    }
    if (gcur >= 0) {
#pragma unroll
        for (int m = 0; m < MT; ++m)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[m][c] = fmaf(s[c], accg[m][c], acc[m][c]);
    }
    float* out = partial + (size_t)blockIdx.y * M * N;
#pragma unroll
    for (int m = 0; m < MT; ++m)
        if (m < M)
            *reinterpret_cast<float4*>(out + (size_t)m * N + n0) =
                make_float4(acc[m][0], acc[m][1], acc[m][2], acc[m][3]);
}

// C[m, n] = out_type(sum over splits, in split order).
template <typename T>
__global__ void splitk_reduce_kernel(const float* __restrict__ partial, int splits, int M, int N,
                                     T* __restrict__ C) {
    const size_t i4 = (size_t)blockIdx.x * blockDim.x + threadIdx.x;  // 4-element group
    const size_t total4 = (size_t)M * N / 4;
    if (i4 >= total4) return;
    float4 acc = reinterpret_cast<const float4*>(partial)[i4];
    for (int sp = 1; sp < splits; ++sp) {
        const float4 p = reinterpret_cast<const float4*>(partial + (size_t)sp * M * N)[i4];
        acc.x += p.x;
        acc.y += p.y;
        acc.z += p.z;
        acc.w += p.w;
    }
    T* c = C + 4 * i4;
    c[0] = Act<T>::from_f32(acc.x);
    c[1] = Act<T>::from_f32(acc.y);
    c[2] = Act<T>::from_f32(acc.z);
    c[3] = Act<T>::from_f32(acc.w);
}

template <int MT, typename T>
int launch_typed(const void* A, int M, int K, const int32_t* codes, const void* scales,
                 const int32_t* zeros, int N, int group, int sym, void* C, float* ws,
                 const GemvPlan& p, cudaStream_t stream) {
    dim3 grid((N / 4 + kThreads - 1) / kThreads, p.splits);
    const size_t smem = (size_t)MT * 8 * p.rows_per_split * sizeof(float);
    if (sym)
        gemv_plain_kernel<MT, T, true><<<grid, kThreads, smem, stream>>>(
            static_cast<const T*>(A), M, K, reinterpret_cast<const int4*>(codes),
            static_cast<const __half*>(scales), nullptr, N, group, ws, p.rows_per_split);
    else
        gemv_plain_kernel<MT, T, false><<<grid, kThreads, smem, stream>>>(
            static_cast<const T*>(A), M, K, reinterpret_cast<const int4*>(codes),
            static_cast<const __half*>(scales), reinterpret_cast<const uint32_t*>(zeros), N, group,
            ws, p.rows_per_split);
    if (cudaGetLastError() != cudaSuccess) return W4A16_ECUDA;
    const size_t total4 = (size_t)M * N / 4;
    const int rthreads = 256;
    splitk_reduce_kernel<T><<<(unsigned)((total4 + rthreads - 1) / rthreads), rthreads, 0, stream>>>(
        ws, p.splits, M, N, static_cast<T*>(C));
    return launch_status();
}

template <typename T>
int launch_by_mt(const void* A, int M, int K, const int32_t* codes, const void* scales,
                 const int32_t* zeros, int N, int group, int sym, void* C, float* ws,
                 const GemvPlan& p, cudaStream_t stream) {
    switch (p.mt) {
        case 1: return launch_typed<1, T>(A, M, K, codes, scales, zeros, N, group, sym, C, ws, p, stream);
        case 2: return launch_typed<2, T>(A, M, K, codes, scales, zeros, N, group, sym, C, ws, p, stream);
        case 4: return launch_typed<4, T>(A, M, K, codes, scales, zeros, N, group, sym, C, ws, p, stream);
        case 8: return launch_typed<8, T>(A, M, K, codes, scales, zeros, N, group, sym, C, ws, p, stream);
        case 16: return launch_typed<16, T>(A, M, K, codes, scales, zeros, N, group, sym, C, ws, p, stream);
        default: return W4A16_EUNSUPPORTED;
    }
}

}  // namespace

// Rows of A handled per launch (template width) for M rows: the next power of two, at most 16.
static int gemv_mt(int M) {
    int mt = 1;
    while (mt < M && mt < 16) mt *= 2;
    return mt;
}

GemvPlan plan_gemv_plain(int M, int N, int K, int group) {
    GemvPlan p;
    p.mt = gemv_mt(M);
    const int rows = K / 8;
    const int rows_per_group = group / 8;
    const int blocks_x = (N / 4 + kThreads - 1) / kThreads;
    // aim for about four blocks per SM (148 SMs when no device answers, as on a build host)
    int n_sm = gemv_stream_sm_count();
    if (n_sm <= 0) n_sm = 148;
    const int target_blocks = 4 * n_sm;
    int splits = (target_blocks + blocks_x - 1) / blocks_x;
    splits = splits < 1 ? 1 : splits;
    int rps = (rows + splits - 1) / splits;
    rps = ((rps + rows_per_group - 1) / rows_per_group) * rows_per_group;  // whole groups
    const int rps_max = kSmemBytes / (p.mt * 8 * (int)sizeof(float));
    const int rps_cap = (rps_max / rows_per_group) * rows_per_group;
    if (rps > rps_cap) rps = rps_cap;
    if (rps < rows_per_group) rps = rows_per_group;
    p.rows_per_split = rps;
    p.splits = (rows + rps - 1) / rps;
    const int m_launch = M < p.mt ? M : p.mt;
    p.ws_bytes = (size_t)p.splits * m_launch * N * sizeof(float);
    return p;
}

int launch_gemv_plain(const void* A, int a_dtype, int M, int K, const int32_t* codes,
                      const void* scales, const int32_t* zeros, int N, int group, int sym, void* C,
                      void* workspace, const GemvPlan& plan, cudaStream_t stream) {
    float* ws = static_cast<float*>(workspace);
    if (a_dtype == W4A16_BF16)
        return launch_by_mt<__nv_bfloat16>(A, M, K, codes, scales, zeros, N, group, sym, C, ws, plan, stream);
    return launch_by_mt<__half>(A, M, K, codes, scales, zeros, N, group, sym, C, ws, plan, stream);
}

}  // namespace w4a16
