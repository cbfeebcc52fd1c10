/*
 * w4a16_oracle.c -- plain, slow, FP64 CPU oracle of the W4A16 weight-only INT4 linear layer.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may call, link or load this file:
 * only the test-suite, the smoke check and the benchmark's CPU-baseline leg use it. It shares
 * no code, header, table or constant generator with the CUDA library.
 *
 * What it computes, and the passages it follows:
 *   - 16-bit float <-> double conversion, written from the IEEE-754 binary16 / bfloat16
 *     definitions (round to nearest, ties to even).
 *   - Round-to-nearest group quantization, symmetric and asymmetric:
 *       "INT4 LLMs: What 4-Bit Quantization Means and When to Use It", section
 *       "What INT4 means in an LLM" (signed codes -8..7, two per byte) and
 *       "Why mapping to 16 values still works" (group-wise scales; symmetric grid centred on
 *       zero vs. affine grid with an offset);
 *       "4.3 Weight-only INT4", section 1 "W4A16 storage and compute" (eight 4-bit codes per
 *       32-bit word, one FP16 scale per group, a zero-point for asymmetric schemes).
 *     The pages give no formula for the rounding quantizer. The reading taken here:
 *       symmetric : s = fp16(amax / 7),            q = clamp(rne(w / s), -8, 7), no zero;
 *       asymmetric: lo = min(0, min w), hi = max(0, max w),
 *                   s = fp16((hi - lo) / 15),      z = clamp(rne(-lo / s), 0, 15),
 *                   q = clamp(rne(w / s) + z, 0, 15);
 *       15 = 16 levels - 1 (the INT4 vs INT8 tick gap of "4.3 Weight-only INT4", introduction,
 *       is 255/15 = 17). A group whose scale rounds to zero stores s = 1, z = 0, q = z.
 *       Every division is an IEEE FP64 division, every rounding to an integer is ties-to-even.
 *   - Packing (layout of "INT4 and Low-Bit Inference", section "Under the hood -- the packed
 *     layout": qweight (K/8, N) int32, scales (K/g, N) fp16, qzeros (K/g, N/8) int32):
 *       codes word (j, n) bits [4i, 4i+4) hold q[8j+i, n] & 0xF;
 *       zeros word (g, j) bits [4i, 4i+4) hold z[g, 8j+i].
 *     The nibble order (least significant nibble first) is this oracle's reading.
 *   - Dequantization w = (q - z) * s ("4.3 Weight-only INT4", section 3.2: D dequantizes with
 *     the scale and the zero-point), exact in FP64.
 *   - The linear layer y[m, n] = sum_k a[m, k] * w[k, n] in FP64, and sum_k |a[m,k] * w[k,n]|,
 *     the quantity the acceptance bound is stated against.
 *
 * No blocking, fusion or reordering beyond the definitions above. OpenMP only splits
 * independent output columns across threads; each column is summed in k order.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define W4O_OK 0
#define W4O_EINVAL (-1)
#define W4O_ENONFINITE (-4)

#define W4O_F16 0
#define W4O_BF16 1

/* ---------------------------------------------------------------------------------------------
 * 16-bit floating point formats, from the IEEE-754 definition of a binary format with
 * `mbits` stored significand bits and an exponent field of `ebits` bits.
 *   binary16: mbits = 10, ebits = 5 (bias 15)      bfloat16: mbits = 7, ebits = 8 (bias 127)
 * ------------------------------------------------------------------------------------------- */
static double fmt_decode(uint16_t bits, int mbits, int ebits) {
    const int bias = (1 << (ebits - 1)) - 1;
    const uint32_t emax_field = (1u << ebits) - 1u;
    const int sign = (bits >> (mbits + ebits)) & 1;
    const uint32_t e = (bits >> mbits) & emax_field;
    const uint32_t m = bits & ((1u << mbits) - 1u);
    double v;
    if (e == 0) {
        v = ldexp((double)m, 1 - bias - mbits);          /* subnormal: m * 2^(emin - mbits) */
    } else if (e == emax_field) {
        v = (m == 0) ? INFINITY : NAN;
    } else {
        v = ldexp((double)((1u << mbits) | m), (int)e - bias - mbits);
    }
    return sign ? -v : v;
}

static uint16_t fmt_encode(double x, int mbits, int ebits) {
    const int bias = (1 << (ebits - 1)) - 1;
    const uint32_t emax_field = (1u << ebits) - 1u;
    const int emin = 1 - bias;                         /* exponent of the smallest normal */
    const uint16_t sign = signbit(x) ? (uint16_t)(1u << (mbits + ebits)) : 0;
    if (isnan(x)) return (uint16_t)((emax_field << mbits) | (1u << (mbits - 1)));  /* quiet NaN */
    double a = fabs(x);
    if (isinf(a)) return sign | (uint16_t)(emax_field << mbits);
    if (a == 0.0) return sign;
    int e2;
    frexp(a, &e2);                                     /* a in [2^(e2-1), 2^e2) */
    int E = e2 - 1;
    if (E < emin) E = emin;                            /* subnormal range shares emin's quantum */
    const double quantum = ldexp(1.0, E - mbits);
    const double r = nearbyint(a / quantum);           /* exact scaling, one ties-to-even rounding */
    const double v = r * quantum;                      /* the rounded magnitude, exact in FP64 */
    if (v == 0.0) return sign;                         /* underflow to a signed zero */
    /* encode the exactly representable magnitude v */
    int ev2;
    frexp(v, &ev2);
    const int Ev = ev2 - 1;
    if (Ev > bias) return sign | (uint16_t)(emax_field << mbits);   /* overflow -> infinity */
    if (Ev < emin) {
        return sign | (uint16_t)(uint32_t)(v / ldexp(1.0, emin - mbits));   /* subnormal */
    }
    const uint32_t sig = (uint32_t)(v / ldexp(1.0, Ev - mbits));           /* 2^mbits .. 2^(mbits+1)-1 */
    return sign | (uint16_t)(((uint32_t)(Ev + bias) << mbits) | (sig - (1u << mbits)));
}

double w4o_half_to_double(uint16_t h) { return fmt_decode(h, 10, 5); }
uint16_t w4o_double_to_half(double x) { return fmt_encode(x, 10, 5); }
double w4o_bf16_to_double(uint16_t b) { return fmt_decode(b, 7, 8); }
uint16_t w4o_double_to_bf16(double x) { return fmt_encode(x, 7, 8); }

static double act_to_double(uint16_t bits, int dtype) {
    return dtype == W4O_BF16 ? w4o_bf16_to_double(bits) : w4o_half_to_double(bits);
}

/* Batch conversions (used by tests for the exhaustive checks). */
void w4o_decode16(const uint16_t* in, long n, int dtype, double* out) {
    for (long i = 0; i < n; ++i) out[i] = act_to_double(in[i], dtype);
}
void w4o_encode16(const double* in, long n, int dtype, uint16_t* out) {
    for (long i = 0; i < n; ++i)
        out[i] = dtype == W4O_BF16 ? w4o_double_to_bf16(in[i]) : w4o_double_to_half(in[i]);
}

/* ---------------------------------------------------------------------------------------------
 * Storage sizes of the packed format ("INT4 and Low-Bit Inference", section "Under the hood --
 * the packed layout"; "4.3 Weight-only INT4", section 1).
 * out[0] = codes bytes, out[1] = scale bytes, out[2] = zero bytes (0 when symmetric).
 * ------------------------------------------------------------------------------------------- */
void w4o_sizes(long K, long N, long group, int sym, long* out) {
    out[0] = (K / 8) * N * 4;
    out[1] = (K / group) * N * 2;
    out[2] = sym ? 0 : (K / group) * (N / 8) * 4;
}

static int valid_shape(long K, long N, long group) {
    return K > 0 && N > 0 && group > 0 && K % group == 0 && K % 8 == 0 && N % 8 == 0 &&
           group % 8 == 0;
}

/* ---------------------------------------------------------------------------------------------
 * Round-to-nearest group quantization (reading stated in the file header).
 * W: fp16 bits, row-major [K, N]. codes: int32 [K/8, N]. scales: fp16 bits [K/g, N].
 * zeros: int32 [K/g, N/8], unused (may be NULL) when sym != 0.
 * Returns W4O_OK, W4O_EINVAL, or W4O_ENONFINITE (a group held Inf/NaN; its outputs are zeroed).
 * ------------------------------------------------------------------------------------------- */
int w4o_quantize(const uint16_t* W, long K, long N, long group, int sym, int32_t* codes,
                 uint16_t* scales, int32_t* zeros, int nthreads) {
    if (!valid_shape(K, N, group) || !W || !codes || !scales || (!sym && !zeros)) return W4O_EINVAL;
    const long G = K / group;
    int status = W4O_OK;
    /* per-element codes and per-group zeros, packed after the column loop */
    int* q = (int*)malloc(sizeof(int) * (size_t)K * (size_t)N);
    int* z = (int*)malloc(sizeof(int) * (size_t)G * (size_t)N);
    if (!q || !z) { free(q); free(z); return W4O_EINVAL; }
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(static) reduction(min : status)
#endif
    for (long n = 0; n < N; ++n) {
        for (long g = 0; g < G; ++g) {
            const long k0 = g * group;
            double lo = 0.0, hi = 0.0, amax = 0.0;
            int finite = 1;
            for (long k = k0; k < k0 + group; ++k) {
                const double w = w4o_half_to_double(W[k * N + n]);
                if (!isfinite(w)) { finite = 0; break; }
                if (w < lo) lo = w;
                if (w > hi) hi = w;
                if (fabs(w) > amax) amax = fabs(w);
            }
            if (!finite) {
                status = W4O_ENONFINITE;
                scales[g * N + n] = 0;
                z[g * N + n] = 0;
                for (long k = k0; k < k0 + group; ++k) q[k * N + n] = 0;
                continue;
            }
            uint16_t sbits = sym ? w4o_double_to_half(amax / 7.0) : w4o_double_to_half((hi - lo) / 15.0);
            double s = w4o_half_to_double(sbits);
            int zp = 0;
            if (s == 0.0) {
                /* degenerate group: s = 1, z = 0, every code equals the zero-point */
                sbits = 0x3C00;
                scales[g * N + n] = sbits;
                z[g * N + n] = 0;
                for (long k = k0; k < k0 + group; ++k) q[k * N + n] = 0;
                continue;
            }
            if (!sym) {
                double zr = nearbyint(-lo / s);
                if (zr < 0.0) zr = 0.0;
                if (zr > 15.0) zr = 15.0;
                zp = (int)zr;
            }
            scales[g * N + n] = sbits;
            z[g * N + n] = zp;
            for (long k = k0; k < k0 + group; ++k) {
                const double w = w4o_half_to_double(W[k * N + n]);
                double r = nearbyint(w / s);
                if (sym) {
                    if (r < -8.0) r = -8.0;
                    if (r > 7.0) r = 7.0;
                } else {
                    r += (double)zp;
                    if (r < 0.0) r = 0.0;
                    if (r > 15.0) r = 15.0;
                }
                q[k * N + n] = (int)r;
            }
        }
    }
    /* pack: eight codes along K per word, eight zeros along N per word */
    for (long j = 0; j < K / 8; ++j)
        for (long n = 0; n < N; ++n) {
            uint32_t word = 0;
            for (int i = 0; i < 8; ++i) word |= ((uint32_t)q[(8 * j + i) * N + n] & 0xFu) << (4 * i);
            codes[j * N + n] = (int32_t)word;
        }
    if (!sym)
        for (long g = 0; g < G; ++g)
            for (long j = 0; j < N / 8; ++j) {
                uint32_t word = 0;
                for (int i = 0; i < 8; ++i) word |= ((uint32_t)z[g * N + 8 * j + i] & 0xFu) << (4 * i);
                zeros[g * (N / 8) + j] = (int32_t)word;
            }
    free(q);
    free(z);
    return status;
}

/* ---------------------------------------------------------------------------------------------
 * Unpacking. q: int [K, N] (sym: -8..7 by two's complement of the nibble; asym: 0..15).
 * z: int [K/g, N] (0..15).
 * ------------------------------------------------------------------------------------------- */
static int nibble(uint32_t word, int i) { return (int)((word >> (4 * i)) & 0xFu); }

static int code_at(const int32_t* codes, long N, int sym, long k, long n) {
    const int v = nibble((uint32_t)codes[(k / 8) * N + n], (int)(k % 8));
    return sym ? (v >= 8 ? v - 16 : v) : v;
}

static int zero_at(const int32_t* zeros, long N, int sym, long g, long n) {
    if (sym) return 0;
    return nibble((uint32_t)zeros[g * (N / 8) + n / 8], (int)(n % 8));
}

void w4o_unpack_codes(const int32_t* codes, long K, long N, int sym, int* q) {
    for (long k = 0; k < K; ++k)
        for (long n = 0; n < N; ++n) q[k * N + n] = code_at(codes, N, sym, k, n);
}

void w4o_unpack_zeros(const int32_t* zeros, long G, long N, int* z) {
    for (long g = 0; g < G; ++g)
        for (long n = 0; n < N; ++n) z[g * N + n] = zero_at(zeros, N, 0, g, n);
}

/* Dequantized weight w[k, n] = (q - z) * s, exact in FP64. */
static double dequant_at(const int32_t* codes, const uint16_t* scales, const int32_t* zeros,
                         long N, long group, int sym, long k, long n) {
    const long g = k / group;
    const int q = code_at(codes, N, sym, k, n);
    const int z = zero_at(zeros, N, sym, g, n);
    return (double)(q - z) * w4o_half_to_double(scales[g * N + n]);
}

void w4o_dequant(const int32_t* codes, const uint16_t* scales, const int32_t* zeros, long K,
                 long N, long group, int sym, double* What) {
    for (long k = 0; k < K; ++k)
        for (long n = 0; n < N; ++n)
            What[k * N + n] = dequant_at(codes, scales, zeros, N, group, sym, k, n);
}

/* ---------------------------------------------------------------------------------------------
 * The linear layer on packed weights, for a list of output columns.
 * A: 16-bit bits [M, K] (dtype W4O_F16 or W4O_BF16). cols: ncols column indices (NULL = all N).
 * Y, Yabs: double [M, ncols], column c of the output is column cols[c] of the layer.
 *   Y[m, c]    = sum_k a[m, k] * w[k, cols[c]]
 *   Yabs[m, c] = sum_k |a[m, k] * w[k, cols[c]]|
 * ------------------------------------------------------------------------------------------- */
int w4o_linear(const uint16_t* A, int a_dtype, long M, long K, const int32_t* codes,
               const uint16_t* scales, const int32_t* zeros, long N, long group, int sym,
               const long* cols, long ncols, double* Y, double* Yabs, int nthreads) {
    if (!valid_shape(K, N, group) || M < 1 || !A || !codes || !scales || (!sym && !zeros))
        return W4O_EINVAL;
    if (!cols) ncols = N;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (long c = 0; c < ncols; ++c) {
        const long n = cols ? cols[c] : c;
        double* w = (double*)malloc(sizeof(double) * (size_t)K);
        for (long k = 0; k < K; ++k) w[k] = dequant_at(codes, scales, zeros, N, group, sym, k, n);
        for (long m = 0; m < M; ++m) {
            double acc = 0.0, accabs = 0.0;
            for (long k = 0; k < K; ++k) {
                const double p = act_to_double(A[m * K + k], a_dtype) * w[k];
                acc += p;
                accabs += fabs(p);
            }
            Y[m * ncols + c] = acc;
            Yabs[m * ncols + c] = accabs;
        }
        free(w);
    }
    return W4O_OK;
}

/* Plain FP64 matmul of 16-bit activations by an FP64 weight matrix: Y = A . What. */
void w4o_matmul(const uint16_t* A, int a_dtype, long M, long K, const double* What, long N,
                double* Y) {
    for (long m = 0; m < M; ++m)
        for (long n = 0; n < N; ++n) {
            double acc = 0.0;
            for (long k = 0; k < K; ++k) acc += act_to_double(A[m * K + k], a_dtype) * What[k * N + n];
            Y[m * N + n] = acc;
        }
}

int w4o_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ---------------------------------------------------------------------------------------------
 * The tiled weight buffer of the library's repack entry point, restated from its definition.
 * The pages ask for weights permuted once at load into a layout that suits the kernel
 * ("INT4 and Low-Bit Inference", section 5 "The kernel is half the story"; "4.3 Weight-only
 * INT4", section 4) and leave its form open; this is the library's.
 *
 * Unit (t, c) = output channels [128 t, 128 t + 128) x input channels [128 c, 128 c + 128); its
 * record has index t * (K/128) + c and R = 8192 + G * 256 + (asym ? G * 64 : 0) bytes, where
 * G = 128 / group groups of K fall in a unit. Inside a record:
 *   codes, bytes [0, 8192): block h (h = 0..3, input channels 128 c + 32 h .. + 31) at 2048 h;
 *     in it, channel n (n = 0..127 within the tile) owns the 16 bytes at slot (n XOR 2 h); word
 *     w (w = 0..3) of those 16 bytes is plain packed row j = 16 c + 4 h + w of channel 128 t + n,
 *     its codes re-ordered: nibble slot p (p = 0..3) holds the code of element 2p and slot p + 4
 *     that of element 2p + 1 (element e = input channel 8 j + e); symmetric codes are stored
 *     offset-binary, q + 8 (zero-point 8);
 *   scales, from byte 8192: group gg (gg = 0..G-1, plain group row c * G + gg) at 8192 + 256 gg,
 *     channel n at + 2 n (fp16 bits), except that a (group, channel) whose codes all equal its
 *     zero point (0 for the symmetric scheme) stores scale 0 (its dequantized weights are 0
 *     with either scale);
 *   zeros (asymmetric only), from byte 8192 + 256 G: group gg at + 64 gg, the 16 plain words of
 *     the tile's channels (word n / 8 holds channel n at nibble n mod 8).
 * Records follow each other with no padding.
 * ------------------------------------------------------------------------------------------- */
void w4o_tiled_offsets(long K, long N, long group, int sym, long* out) {
    const long G = 128 / group;
    const long record = 8192 + G * 256 + (sym ? 0 : G * 64);
    out[0] = record;                 /* bytes per unit record */
    out[1] = 8192;                   /* codes bytes per record */
    out[2] = 8192;                   /* scales offset in a record */
    out[3] = G * 256;                /* scales bytes per record */
    out[4] = 8192 + G * 256;         /* zeros offset in a record */
    out[5] = sym ? 0 : G * 64;       /* zeros bytes per record */
    out[6] = (N / 128) * (K / 128) * record;   /* whole buffer */
}

int w4o_repack(const int32_t* codes, const uint16_t* scales, const int32_t* zeros, long K, long N,
               long group, int sym, uint8_t* out) {
    if (!valid_shape(K, N, group) || N % 128 != 0 || K % 128 != 0) return W4O_EINVAL;
    long off[7];
    w4o_tiled_offsets(K, N, group, sym, off);
    const long R = off[0], G = 128 / group, units = K / 128;
    memset(out, 0, (size_t)off[6]);
    for (long t = 0; t < N / 128; ++t)
        for (long c = 0; c < units; ++c) {
            uint8_t* rec = out + (t * units + c) * R;
            for (long h = 0; h < 4; ++h)
                for (long nl = 0; nl < 128; ++nl)
                    for (long w = 0; w < 4; ++w) {
                        const long j = 16 * c + 4 * h + w, n = 128 * t + nl;
                        const uint32_t word = (uint32_t)codes[j * N + n];
                        uint32_t enc = 0;
                        for (int e = 0; e < 8; ++e) {
                            uint32_t u = (word >> (4 * e)) & 0xFu;     /* element e */
                            if (sym) u = (u + 8u) & 0xFu;              /* q + 8 for q in -8..7 */
                            const int slot = (e % 2 == 0) ? e / 2 : 4 + e / 2;
                            enc |= u << (4 * slot);
                        }
                        memcpy(rec + 2048 * h + 16 * (nl ^ (2 * h)) + 4 * w, &enc, 4);
                    }
            for (long gg = 0; gg < G; ++gg) {
                const long gi = c * G + gg;
                for (long nl = 0; nl < 128; ++nl) {
                    const long n = 128 * t + nl;
                    const uint32_t zp = sym ? 0u : ((uint32_t)zeros[gi * (N / 8) + n / 8] >> (4 * (n % 8))) & 0xFu;
                    int all_zero_point = 1;
                    for (long k = gi * group; k < (gi + 1) * group; ++k)
                        if ((((uint32_t)codes[(k / 8) * N + n] >> (4 * (k % 8))) & 0xFu) != zp) all_zero_point = 0;
                    const uint16_t sv = all_zero_point ? (uint16_t)0 : scales[gi * N + n];
                    memcpy(rec + off[2] + 256 * gg + 2 * nl, &sv, 2);
                }
                if (!sym)
                    for (long wd = 0; wd < 16; ++wd)
                        memcpy(rec + off[4] + 64 * gg + 4 * wd, &zeros[gi * (N / 8) + 16 * t + wd], 4);
            }
        }
    return W4O_OK;
}
