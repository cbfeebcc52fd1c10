// quantize.cu -- round-to-nearest group quantization of an FP16 weight matrix into the packed
// W4A16 format.
//
// "INT4 LLMs: What 4-Bit Quantization Means and When to Use It", sections "What INT4 means in an
// LLM" (16 signed levels -8..7, two codes per byte) and "Why mapping to 16 values still works"
// (one grid per group; symmetric grid centred on zero, affine grid with an offset).
// "4.3 Weight-only INT4", section 1 (eight codes per 32-bit word, FP16 scale per group,
// zero-point for asymmetric schemes).
//
// Arithmetic (FP64 throughout, so that the codes are reproducible bit for bit):
//   sym : s = fp16(amax / 7),                       q = clamp(rne(w / s), -8, 7)
//   asym: s = fp16((hi - lo) / 15), lo = min(0, min w), hi = max(0, max w),
//         z = clamp(rne(-lo / s), 0, 15),           q = clamp(rne(w / s) + z, 0, 15)
// hi - lo of two fp16 values is exact in FP64; the FP64 quotient is one IEEE rounding and the
// conversion to fp16 (cvt.rn.f16.f64) a second one that cannot meet a tie the first one made:
// the quotient of a multiple of 2^-24 by 15 is either exact or at least 2^-45 (relative) away
// from every fp16 midpoint. A group whose scale rounds to zero stores s = 1, z = 0, q = z.
#include "common.cuh"

namespace w4a16 {

namespace {

__device__ __forceinline__ uint16_t f64_to_f16_bits_rn(double x) {
    uint16_t h;
    asm("cvt.rn.f16.f64 %0, %1;" : "=h"(h) : "d"(x));
    return h;
}

__device__ __forceinline__ double f16_bits_to_f64(uint16_t h) {
    return (double)__half2float(__ushort_as_half(h));
}

constexpr int kQuantThreads = 256;

// One thread per (group g = blockIdx.y, column n). Consecutive threads own consecutive columns,
// so every read of a row of W and every write of a row of codes is coalesced.
template <bool SYM>
__global__ void __launch_bounds__(kQuantThreads)
quantize_kernel(const uint16_t* __restrict__ W, int N, int group, int32_t* __restrict__ codes,
                uint16_t* __restrict__ scales, int32_t* __restrict__ zeros, int* dev_status) {
    const int n = blockIdx.x * kQuantThreads + threadIdx.x;
    const int g = blockIdx.y;
    const bool active = n < N;
    const size_t k0 = (size_t)g * group;

    double lo = 0.0, hi = 0.0, amax = 0.0;
    bool finite = true;
    if (active) {
        for (int i = 0; i < group; ++i) {
            const double w = f16_bits_to_f64(W[(k0 + i) * N + n]);
            finite = finite && isfinite(w);
            lo = w < lo ? w : lo;
            hi = w > hi ? w : hi;
            amax = fabs(w) > amax ? fabs(w) : amax;
        }
    }

    uint16_t sbits = SYM ? f64_to_f16_bits_rn(amax / 7.0) : f64_to_f16_bits_rn((hi - lo) / 15.0);
    double s = f16_bits_to_f64(sbits);
    int z = 0;
    const bool degenerate = (s == 0.0);
    if (degenerate) {
        sbits = 0x3C00;  // 1.0
        s = 1.0;
    } else if (!SYM) {
        double zr = rint(-lo / s);
        zr = zr < 0.0 ? 0.0 : (zr > 15.0 ? 15.0 : zr);
        z = (int)zr;
    }
    if (active && !finite) {
        report_status(dev_status, W4A16_ENONFINITE);
        sbits = 0;
        z = 0;
    }

    if (active) {
        scales[(size_t)g * N + n] = sbits;
        for (int j = 0; j < group / 8; ++j) {
            uint32_t word = 0;
            if (finite && !degenerate) {
                for (int i = 0; i < 8; ++i) {
                    const double w = f16_bits_to_f64(W[(k0 + 8 * j + i) * N + n]);
                    double r = rint(w / s);
                    int q;
                    if (SYM) {
                        r = r < -8.0 ? -8.0 : (r > 7.0 ? 7.0 : r);
                        q = (int)r;
                    } else {
                        r += (double)z;
                        r = r < 0.0 ? 0.0 : (r > 15.0 ? 15.0 : r);
                        q = (int)r;
                    }
                    word |= ((uint32_t)q & 0xFu) << (4 * i);
                }
            } else if (!SYM) {
                word = 0;  // q = z = 0
            }
            codes[(k0 / 8 + j) * N + n] = (int32_t)word;
        }
    }

    if (!SYM) {
        // gather the zeros of eight consecutive columns (eight consecutive lanes) into one word
        const int lane = threadIdx.x & 31;
        const int base = lane & ~7;
        uint32_t word = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int zi = __shfl_sync(0xffffffffu, z, base + i);
            word |= ((uint32_t)zi & 0xFu) << (4 * i);
        }
        if (active && (lane & 7) == 0) zeros[(size_t)g * (N / 8) + n / 8] = (int32_t)word;
    }
}

}  // namespace

int launch_quantize(const void* W, int K, int N, int group, int sym, int32_t* codes, void* scales,
                    int32_t* zeros, int* dev_status, cudaStream_t stream) {
    dim3 grid((N + kQuantThreads - 1) / kQuantThreads, K / group);
    if (sym)
        quantize_kernel<true><<<grid, kQuantThreads, 0, stream>>>(
            static_cast<const uint16_t*>(W), N, group, codes, static_cast<uint16_t*>(scales), nullptr,
            dev_status);
    else
        quantize_kernel<false><<<grid, kQuantThreads, 0, stream>>>(
            static_cast<const uint16_t*>(W), N, group, codes, static_cast<uint16_t*>(scales), zeros,
            dev_status);
    return launch_status();
}

}  // namespace w4a16
