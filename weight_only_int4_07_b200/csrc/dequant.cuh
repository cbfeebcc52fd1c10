// dequant.cuh -- 16-bit operands from the tiled layout's packed words (sm_100a).
//
// A tiled word holds eight 4-bit codes of consecutive K with its nibbles re-ordered: slot p
// (bits 4p..4p+3) holds element 2p and slot p + 4 element 2p + 1, so nibble p of each 16-bit half
// is the pair (2p, 2p + 1). One mask-OR with a float "magic" exponent turns a pair into two
// 16-bit values ("4.3 Weight-only INT4", section 1: codes dequantized on chip to FP16/BF16):
//   fp16: 0x6400 | u = 1024 + u, and for the nibble one position up 0x6400 | (u << 4) =
//         1024 + 16 u (no shift needed);
//   bf16: 0x4300 | u = 128 + u.
// The zero point is subtracted exactly in 16 bits: (1024 + u) - (1024 + z), (1024 + 16 u) / 16 -
// (64 + z), (128 + u) - (128 + z). A scale s (an fp16 value) multiplies (u - z) with one
// rounding: fp16 directly; bf16 as s = s_hi + s_lo with s_hi the bf16 truncation of s and s_lo
// (at most 3 significant bits) exact in bf16, d s_lo exact, fma(d, s_hi, d s_lo) rounded once.
// A third fp16 form needs no magic and no subtraction: the mask alone leaves u (or 16 u) in the
// low mantissa bits of an fp16 whose exponent field is zero, the subnormal u 2^-24 (16 u 2^-24),
// which the warp-level MMA multiplies exactly; the zero point then comes off the FP32 sums.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace w4a16 {

__device__ __forceinline__ uint32_t mulhi(uint32_t a, uint32_t b) {   // a >> k for b = 2^(32-k)
    uint32_t r;
    asm("mul.hi.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

__device__ __forceinline__ uint32_t andor(uint32_t a, uint32_t b, uint32_t c) {   // (a & b) | c
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
    return r;
}

// Masks and shift multipliers, passed at run time so that the compiler keeps them in registers:
// one lop3 per operand register, shifts on the multiply pipe.
struct GsMasks {
    uint32_t lo, hi, magic, m4, m8, m12;
};

template <typename T>
struct GsOps;

template <>
struct GsOps<__half> {
    // operands: r0 = elements (0,1), r2 = (4,5) as 1024 + u; r1 = (2,3), r3 = (6,7) as 1024 + 16 u
    static __device__ __forceinline__ void unpack(uint32_t w, const GsMasks& k, uint32_t (&r)[4]) {
        const uint32_t h = mulhi(w, k.m8);
        r[0] = andor(w, k.lo, k.magic);
        r[1] = andor(w, k.hi, k.magic);
        r[2] = andor(h, k.lo, k.magic);
        r[3] = andor(h, k.hi, k.magic);
    }
    static __device__ __forceinline__ uint32_t zz_a(uint32_t z) { return (0x6400u + z) * 0x00010001u; }
    static __device__ __forceinline__ uint32_t zz_b(uint32_t z) { return (0xD400u + (z << 4)) * 0x00010001u; }
    static __device__ __forceinline__ uint32_t sub_a(uint32_t x, uint32_t zz) {   // (1024+u) - (1024+z)
        uint32_t r;
        asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(zz));
        return r;
    }
    static __device__ __forceinline__ uint32_t sub_b(uint32_t x, uint32_t zz) {   // x / 16 - (64 + z)
        uint32_t r;
        asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(x), "r"(0x2C002C00u), "r"(zz));
        return r;
    }
    struct Scale {   // d * s, one rounding (s is an fp16 value)
        uint32_t s2;
        __device__ __forceinline__ void set(uint16_t bits) { s2 = (uint32_t)bits * 0x00010001u; }
        __device__ __forceinline__ uint32_t apply(uint32_t d) const {
            uint32_t r;
            asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(d), "r"(s2));
            return r;
        }
    };
    static __device__ __forceinline__ void mma(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
        asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
            "{%0, %1, %2, %3};"
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    }
    // the first MMA of a chain: C = 0
    static __device__ __forceinline__ void mma_z(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                                 uint32_t b0, uint32_t b1) {
        asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
            "{%10, %10, %10, %10};"
            : "=f"(c[0]), "=f"(c[1]), "=f"(c[2]), "=f"(c[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));
    }
};

template <>
struct GsOps<__nv_bfloat16> {
    // operands: all four registers as 128 + u (elements (0,1), (2,3), (4,5), (6,7))
    static __device__ __forceinline__ void unpack(uint32_t w, const GsMasks& k, uint32_t (&r)[4]) {
        r[0] = andor(w, k.lo, k.magic);
        r[1] = andor(mulhi(w, k.m4), k.lo, k.magic);
        r[2] = andor(mulhi(w, k.m8), k.lo, k.magic);
        r[3] = andor(mulhi(w, k.m12), k.lo, k.magic);
    }
    static __device__ __forceinline__ uint32_t zz_a(uint32_t z) { return (0x4300u + z) * 0x00010001u; }
    static __device__ __forceinline__ uint32_t zz_b(uint32_t z) { return zz_a(z); }
    static __device__ __forceinline__ uint32_t sub_a(uint32_t x, uint32_t zz) {   // (128+u) - (128+z)
        uint32_t r;
        asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(zz));
        return r;
    }
    static __device__ __forceinline__ uint32_t sub_b(uint32_t x, uint32_t zz) { return sub_a(x, zz); }
    struct Scale {   // d * s rounded once: s = s_hi (bf16 truncation of s) + s_lo (exact in bf16)
        uint32_t hi2, lo2;
        __device__ __forceinline__ void set(uint16_t bits) {
            const float s = __half2float(__ushort_as_half(bits));
            const uint32_t sb = __float_as_uint(s) & 0xFFFF0000u;
            hi2 = (sb >> 16) * 0x00010001u;
            __nv_bfloat162 l = __float2bfloat162_rn(s - __uint_as_float(sb));
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
        asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
            "{%0, %1, %2, %3};"
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    }
};

template <typename X>
struct OpsTag {
    using type = X;
};

}  // namespace w4a16
