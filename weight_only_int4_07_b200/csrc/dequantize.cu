// dequantize.cu -- the packed W4A16 weight expanded to a 16-bit matrix, for the naive path that
// the fused kernels are measured against.
//
// "4.3 Weight-only INT4", section 4: the straightforward implementation dequantizes the whole INT4
// matrix to FP16 in memory and then calls a standard GEMM, so the weights cross HBM three times
// (the 4-bit read, the 16-bit write and the 16-bit read by the GEMM) instead of once. "INT4 and
// Low-Bit Inference", section 5 "The kernel is half the story": the format saves memory but only
// a fused kernel turns it into speed.
//
// w[k, n] = (q[k, n] - z[g, n]) * s[g, n], g = k / group: q - z is a small integer and s an fp16
// value, so the product is exact in FP32 and rounded once to the output type (fp16 or bf16).
// Symmetric codes are two's complement nibbles (-8..7) with no zero-point.
#include "common.cuh"

namespace w4a16 {

namespace {

constexpr int kDeqThreads = 256;

template <typename T>
struct Pack2;
template <>
struct Pack2<__half> {
    static __device__ __forceinline__ uint32_t rn(float a, float b) {
        __half2 h = __floats2half2_rn(a, b);
        return *reinterpret_cast<uint32_t*>(&h);
    }
};
template <>
struct Pack2<__nv_bfloat16> {
    static __device__ __forceinline__ uint32_t rn(float a, float b) {
        __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
        return *reinterpret_cast<uint32_t*>(&h);
    }
};

// One thread per 8 rows x 8 columns: packed row j, columns 8c .. 8c+7. It reads 8 code words
// (32 B), the 8 fp16 scales of its group (16 B) and one zeros word, and writes each of its 8 rows
// as one 16-byte store; consecutive threads take consecutive column blocks, so a warp reads 1 KB
// of codes and writes 512 contiguous bytes per row.
template <typename T, bool SYM>
__global__ void __launch_bounds__(kDeqThreads)
dequantize_kernel(const int32_t* __restrict__ codes, const uint16_t* __restrict__ scales,
                  const int32_t* __restrict__ zeros, int K, int N, int group, T* __restrict__ W) {
    const int nb = N / 8;
    const size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (size_t)(K / 8) * nb) return;
    const int j = (int)(idx / nb);
    const int c = (int)(idx - (size_t)j * nb);
    const int g = (8 * j) / group;
    const uint4* cw = reinterpret_cast<const uint4*>(codes + (size_t)j * N + 8 * c);
    const uint4 w0 = __ldg(cw), w1 = __ldg(cw + 1);
    const uint32_t w[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
    const uint4 sv = __ldg(reinterpret_cast<const uint4*>(scales + (size_t)g * N + 8 * c));
    const uint32_t sw[4] = {sv.x, sv.y, sv.z, sv.w};
    float s[8];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        s[2 * t] = __half2float(__ushort_as_half((uint16_t)(sw[t] & 0xFFFFu)));
        s[2 * t + 1] = __half2float(__ushort_as_half((uint16_t)(sw[t] >> 16)));
    }
    const uint32_t zw = SYM ? 0u : (uint32_t)__ldg(zeros + (size_t)g * nb + c);
#pragma unroll
    for (int i = 0; i < 8; ++i) {          // row 8j + i
        uint32_t o[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            float v[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int col = 2 * t + e;
                const int u = (int)((w[col] >> (4 * i)) & 0xFu);
                const int z = (int)((zw >> (4 * col)) & 0xFu);
                const int q = SYM ? (u ^ 8) - 8 : u - z;   // sign-extended nibble, or code minus zero
                v[e] = (float)q * s[col];                  // exact: |q| < 16, s has 11 bits
            }
            o[t] = Pack2<T>::rn(v[0], v[1]);
        }
        *reinterpret_cast<uint4*>(W + (size_t)(8 * j + i) * N + 8 * c) = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

}  // namespace

int launch_dequantize(const int32_t* codes, const void* scales, const int32_t* zeros, int K, int N, int group,
                      int sym, int out_dtype, void* W, cudaStream_t stream) {
    const size_t items = (size_t)(K / 8) * (N / 8);
    const unsigned blocks = (unsigned)((items + kDeqThreads - 1) / kDeqThreads);
    const uint16_t* s = static_cast<const uint16_t*>(scales);
    if (out_dtype == W4A16_BF16) {
        if (sym)
            dequantize_kernel<__nv_bfloat16, true><<<blocks, kDeqThreads, 0, stream>>>(
                codes, s, zeros, K, N, group, static_cast<__nv_bfloat16*>(W));
        else
            dequantize_kernel<__nv_bfloat16, false><<<blocks, kDeqThreads, 0, stream>>>(
                codes, s, zeros, K, N, group, static_cast<__nv_bfloat16*>(W));
    } else {
        if (sym)
            dequantize_kernel<__half, true><<<blocks, kDeqThreads, 0, stream>>>(codes, s, zeros, K, N, group,
                                                                                static_cast<__half*>(W));
        else
            dequantize_kernel<__half, false><<<blocks, kDeqThreads, 0, stream>>>(codes, s, zeros, K, N, group,
                                                                                 static_cast<__half*>(W));
    }
    return launch_status();
}

}  // namespace w4a16
