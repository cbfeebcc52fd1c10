// gemv_stream.cu -- persistent stream-K decode GEMV / skinny GEMM (M <= 16) on the tiled layout.
//
// C[m, n] = sum_k A[m, k] * (u[k, n] - z[g, n]) * s[g, n], FP32 accumulation.
// "4.3 Weight-only INT4", section 4 (read, unpack, dequantize and multiply in one pipeline so each
// weight byte crosses HBM once, with data movement overlapped with compute); "INT8 vs INT4
// Quantization, in depth", "Two regimes" (at small batch the layer waits for memory).
//
// Work split. The weights are a sequence of units, one unit = one 128-channel tile x one 128-K
// step (8 KiB of codes), ordered tile-major. One CTA per SM takes a contiguous range of
// floor(U / P) or ceil(U / P) units, so every SM streams the same number of bytes whatever the
// shape. A tile whose units all belong to one CTA is written straight to C; a tile cut between
// CTAs is finished by the last of them to arrive (a counter per tile in the workspace), which
// adds the FP32 partial sums of all of them in CTA order, so the result does not depend on timing.
//
// Bytes in flight. Warp 16 (one thread) keeps `ns` (8..16) stages of bulk copies in flight: per
// unit the four 2 KiB half-tiles of codes (to shared-memory offsets 2048 + 32 bytes apart, which
// makes the consumers' 16-byte reads bank-conflict free) and the unit's scales and zero-points.
// Sixteen consumer warps in two groups take the units alternately (group = unit parity).
//
// Math (warp-level tensor-core MMA, m16n8k16, FP32 accumulators). Warp w of a group owns channels
// 16 w .. 16 w + 15 of the tile; lane (g = lane / 4, t = lane % 4) reads the 32 K of half-tile t
// for channels 16 w + g and 16 w + g + 8 and batch rows 8 b + g of A. Nibble pairs become 16-bit
// operands by one mask-OR with a magic exponent: fp16 0x6400 | u = 1024 + u, and for the nibble
// one position up 0x6400 | (u << 4) = 1024 + 16 u; bf16 0x4300 | u = 128 + u (its 7-bit mantissa
// has no room for the shifted form). Two MMA chains per unit: chain A takes the 1024 + u operands,
// chain B the 1024 + 16 u ones (bf16: both chains 128 + u).
// Group size 128 (one group per unit): the chains run on the raw operands. The same chains with
// every code at its zero reference (u = 0; offset-binary 8 for symmetric codes) give R_A and R_B;
// these depend only on A, are computed once per CTA and unit into shared memory, and
//   sum_k a_k (u_k - z) = (acc_A - R_A f_A) + (acc_B - R_B f_B) / 16,
// f_A = (1024 + z) / (1024 + z_ref), f_B = (1024 + 16 z) / (1024 + 16 z_ref), both exact in FP32.
// A group whose codes all equal the reference has acc = R bit for bit (the same MMAs on the same
// operands), so an all-zero group contributes exactly zero. The FP32 sum is scaled by s[g, n].
// Smaller groups (several per unit): each operand is dequantized before the MMA, (u - z) exact in
// the 16-bit type, then times s rounded once (bf16: s = s_hi + s_lo, both exact in bf16).
//
// Every mbarrier wait is bounded (2 s); on expiry the kernel records W4A16_ETIMEOUT and skips
// its remaining work, still passing every CTA barrier and tile counter.
#include <mutex>

#include "common.cuh"
#include "sm100_ptx.cuh"
#include "tiled_layout.cuh"

namespace w4a16 {
namespace {

using namespace sm100;

constexpr int kGsGroupWarps = 8;                         // warps per consumer group (128 channels)
constexpr int kGsConsumers = 2 * kGsGroupWarps;          // two groups: even and odd units
constexpr int kGsThreads = 32 * (kGsConsumers + 1);      // + one producer warp
constexpr int kGsHalf = 2048 + 32;                       // skewed half-tile stride in a stage
constexpr int kGsScalesOff = 4 * kGsHalf;                // up to 4 groups x 256 B
constexpr int kGsZerosOff = kGsScalesOff + 4 * 256;      // up to 4 groups x 64 B
constexpr int kGsStage = kGsZerosOff + 4 * 64;           // 9600 bytes
constexpr int kGsMinStages = 6, kGsMaxStages = 16;
constexpr int kGsSmemMax = 227 * 1024;
constexpr uint64_t kGsSpin = 2000000000ull;

static_assert(kGsStage % 128 == 0, "stage size");

// 16-bit operand handling per activation type.
template <typename T>
struct GsOps;

template <>
struct GsOps<__half> {
    static constexpr uint32_t kMagic = 0x64006400u;
    static constexpr float kInvB = 1.0f / 16.0f;           // chain B carries 16 u
    static __device__ __forceinline__ uint32_t ref_a(int zr) { return (uint32_t)(0x6400 + zr) * 0x00010001u; }
    static __device__ __forceinline__ uint32_t ref_b(int zr) { return (uint32_t)(0x6400 + 16 * zr) * 0x00010001u; }
    static __device__ __forceinline__ float fa(int z) { return fmaf((float)z, 1.0f / 1024.0f, 1.0f); }
    static __device__ __forceinline__ float fb(int z) { return fmaf((float)z, 1.0f / 64.0f, 1.0f); }
    // nibble pairs of one word: r0 (elements 0,1) and r2 (4,5) for chain A, r1 (2,3) and r3 (6,7) for B
    static __device__ __forceinline__ void unpack(uint32_t w, uint32_t (&r)[4]) {
        const uint32_t h = w >> 8;
        r[0] = (w & 0x000F000Fu) | kMagic;
        r[1] = (w & 0x00F000F0u) | kMagic;
        r[2] = (h & 0x000F000Fu) | kMagic;
        r[3] = (h & 0x00F000F0u) | kMagic;
    }
    // exact (u - z) for chain A / chain B operands
    static __device__ __forceinline__ uint32_t zz_a(int z) { return (uint32_t)(0x6400 + z) * 0x00010001u; }
    static __device__ __forceinline__ uint32_t zz_b(int z) {  // -(64 + z), packed
        __half2 h = __floats2half2_rn(-(64.0f + (float)z), -(64.0f + (float)z));
        return *reinterpret_cast<uint32_t*>(&h);
    }
    static __device__ __forceinline__ uint32_t sub_a(uint32_t x, uint32_t zz) {
        uint32_t r;
        asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(zz));
        return r;
    }
    static __device__ __forceinline__ uint32_t sub_b(uint32_t x, uint32_t zz) {  // x / 16 - (64 + z)
        uint32_t r;
        asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(x), "r"(0x2C002C00u), "r"(zz));
        return r;
    }
    struct Scale {
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
};

template <>
struct GsOps<__nv_bfloat16> {
    static constexpr uint32_t kMagic = 0x43004300u;
    static constexpr float kInvB = 1.0f;
    static __device__ __forceinline__ uint32_t ref_a(int zr) { return (uint32_t)(0x4300 + zr) * 0x00010001u; }
    static __device__ __forceinline__ uint32_t ref_b(int zr) { return ref_a(zr); }
    static __device__ __forceinline__ float fa(int z) { return fmaf((float)z, 1.0f / 128.0f, 1.0f); }
    static __device__ __forceinline__ float fb(int z) { return fa(z); }
    static __device__ __forceinline__ void unpack(uint32_t w, uint32_t (&r)[4]) {
        r[0] = (w & 0x000F000Fu) | kMagic;
        r[1] = ((w >> 4) & 0x000F000Fu) | kMagic;
        r[2] = ((w >> 8) & 0x000F000Fu) | kMagic;
        r[3] = ((w >> 12) & 0x000F000Fu) | kMagic;
    }
    static __device__ __forceinline__ uint32_t zz_a(int z) { return (uint32_t)(0x4300 + z) * 0x00010001u; }
    static __device__ __forceinline__ uint32_t zz_b(int z) { return zz_a(z); }
    static __device__ __forceinline__ uint32_t sub_a(uint32_t x, uint32_t zz) {
        uint32_t r;
        asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(zz));
        return r;
    }
    static __device__ __forceinline__ uint32_t sub_b(uint32_t x, uint32_t zz) { return sub_a(x, zz); }
    struct Scale {  // d * s rounded once: s = s_hi (bf16 truncation of s) + s_lo (exact in bf16)
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

__device__ __forceinline__ void named_bar(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dependents_launch() { asm volatile("griddepcontrol.launch_dependents;" :::); }

// First unit of CTA c when U units are cut into P contiguous ranges.
__device__ __forceinline__ long long unit_begin(int c, long long U, int P) { return ((long long)c * U) / P; }
// The CTA whose range holds unit u.
__device__ __forceinline__ int unit_owner(long long u, long long U, int P) {
    return (int)(((u + 1) * P - 1) / U);
}

// Byte offset of A[m, k] (k a multiple of 8) in the shared activation copy: rows of 2K + 32 bytes,
// each 128-K unit 256 bytes, and inside it the 16-byte chunk q of 32-K block t stored at
// position (q + t / 2) mod 4 (conflict-free 16-byte reads by the MMA lanes).
__device__ __forceinline__ uint32_t act_offset(int m, int k, uint32_t row_bytes) {
    const int kk = k & 127, t = kk >> 5, q = (kk >> 3) & 3;
    return (uint32_t)m * row_bytes + (uint32_t)(k >> 7) * 256u + (uint32_t)t * 64u +
           (uint32_t)((q + (t >> 1)) & 3) * 16u;
}

struct GsParams {
    const void* A;
    const uint8_t* tiled;
    void* C;
    int* counters;      // one int per tile, zero between calls
    float* partials;    // [P][2][M][128]
    int* dev_status;
    unsigned long long scales_off, zeros_off;
    int M, K, N, sym, ns, P;
    uint32_t row_bytes;   // 2 K + 32
    uint32_t act_bytes, ref_bytes, red_bytes;
};

template <int NB, typename T, int GROUP>
__global__ void __launch_bounds__(kGsThreads, 1) gemv_stream_kernel(const GsParams p) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    using Ops = GsOps<T>;
    constexpr int MT = 8 * NB;
    constexpr bool kRef = (GROUP == 128);
    constexpr int G = GROUP >= 128 ? 1 : 128 / GROUP;   // groups per unit
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int M = p.M, K = p.K, N = p.N, ns = p.ns, P = p.P;
    const int steps = K / 128;
    const int tiles = N / 128;
    const long long U = (long long)tiles * steps;
    const int cta = blockIdx.x;
    const long long u0 = unit_begin(cta, U, P), u1 = unit_begin(cta + 1, U, P);

    uint8_t* acts = smem_raw;                                               // [M][2K + 32] rotated
    float* refs = reinterpret_cast<float*>(smem_raw + p.act_bytes);         // [steps][2][MT]
    float* red = reinterpret_cast<float*>(smem_raw + p.act_bytes + p.ref_bytes);       // [MT][128]
    uint8_t* stages = smem_raw + p.act_bytes + p.ref_bytes + p.red_bytes;  // ns x kGsStage
    uint64_t* full = reinterpret_cast<uint64_t*>(stages + (size_t)ns * kGsStage);
    uint64_t* empty = full + ns;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + ns);
    volatile int* last_flag = abort_flag + 1;

    if (threadIdx.x == 0) {
        for (int i = 0; i < ns; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kGsGroupWarps);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    grid_dependents_launch();

    if (warp == kGsConsumers) {
        // ------------------------------------------------------------------------ producer
        if (lane == 0) {
            const int ktiles = K / 64;
            const uint32_t bytes = 8192u + (uint32_t)G * (256u + (p.sym ? 0u : 64u));
            int s = 0;
            uint32_t ph = 0;
            long long issued = 0;
            int tile = (int)(u0 / steps), sp = (int)(u0 - (long long)tile * steps);
            for (long long u = u0; u < u1; ++u) {
                if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, p.dev_status, kGsSpin)) break;
                uint8_t* st = stages + (size_t)s * kGsStage;
                mbar_arrive_expect_tx(&full[s], bytes);
                const uint8_t* src = p.tiled + ((size_t)tile * ktiles + 2 * (size_t)sp) * 4096;
#pragma unroll
                for (int b = 0; b < 4; ++b) bulk_g2s(st + b * kGsHalf, src + b * 2048, 2048, &full[s]);
#pragma unroll
                for (int gg = 0; gg < G; ++gg) {
                    const size_t gi = (size_t)sp * G + gg;
                    bulk_g2s(st + kGsScalesOff + 256 * gg, p.tiled + p.scales_off + (gi * N + (size_t)tile * 128) * 2,
                             256, &full[s]);
                    if (!p.sym)
                        bulk_g2s(st + kGsZerosOff + 64 * gg,
                                 p.tiled + p.zeros_off + (gi * (N / 8) + (size_t)tile * 16) * 4, 64, &full[s]);
                }
                ++issued;
                if (++s == ns) { s = 0; ph ^= 1u; }
                if (++sp == steps) { sp = 0; ++tile; }
            }
            // copies still in flight land before the CTA exits (only a cut-short run has any)
            const long long first = issued > ns ? issued - ns : 0;
            for (long long i = first; i < issued; ++i)
                mbar_wait(&full[i % ns], (uint32_t)((i / ns) & 1), abort_flag, p.dev_status, kGsSpin);
        }
        return;
    }

    // ---------------------------------------------------------------------------- consumers
    const int grp = warp / kGsGroupWarps;           // 0: even units, 1: odd units
    const int wg = warp % kGsGroupWarps;            // channel block of the warp
    const int ctid = threadIdx.x;                   // 0 .. 511
    const int g = lane >> 2, t = lane & 3;
    const int ch0 = 16 * wg + g, ch1 = ch0 + 8;
    const int zr = p.sym ? 8 : 0;
    const T* A = static_cast<const T*>(p.A);

    // A may be the output of the previous kernel in the stream
    grid_dependency_wait();
    {
        const int vpr = K / 8;
        for (int m = 0; m < M; ++m)
            for (int c = ctid; c < vpr; c += 32 * kGsConsumers)
                *reinterpret_cast<uint4*>(acts + act_offset(m, 8 * c, p.row_bytes)) =
                    *reinterpret_cast<const uint4*>(A + (size_t)m * K + 8 * c);
    }
    named_bar(1, 32 * kGsConsumers);

    // activation fragments of one unit: lane holds row 8 b + g, K 32 t .. 32 t + 31 of the unit
    auto load_b = [&](int sp, uint32_t (&bfr)[NB][16]) {
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            const int row = 8 * b + g;
            if (row < M) {
                const uint8_t* base = acts + (uint32_t)row * p.row_bytes + (uint32_t)sp * 256u + (uint32_t)t * 64u;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint4 v = *reinterpret_cast<const uint4*>(base + ((q + (t >> 1)) & 3) * 16);
                    bfr[b][4 * q + 0] = v.x;
                    bfr[b][4 * q + 1] = v.y;
                    bfr[b][4 * q + 2] = v.z;
                    bfr[b][4 * q + 3] = v.w;
                }
            } else {
#pragma unroll
                for (int r = 0; r < 16; ++r) bfr[b][r] = 0u;
            }
        }
    };

    if constexpr (kRef) {
        // R_A, R_B of every unit this CTA touches: the chains below with all codes at the reference
        const long long span = u1 - u0;
        const int nref = span >= steps ? steps : (int)span;
        const int sp_first = (int)(u0 % steps);
        const uint32_t ca = Ops::ref_a(zr), cb = Ops::ref_b(zr);
        for (int i = warp; i < nref; i += kGsConsumers) {
            int sp = sp_first + i;
            if (sp >= steps) sp -= steps;
            uint32_t bfr[NB][16];
            load_b(sp, bfr);
#pragma unroll
            for (int b = 0; b < NB; ++b) {
                float ra[4] = {0.f, 0.f, 0.f, 0.f}, rb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    Ops::mma(ra, ca, ca, ca, ca, bfr[b][4 * j + 0], bfr[b][4 * j + 2]);
                    Ops::mma(rb, cb, cb, cb, cb, bfr[b][4 * j + 1], bfr[b][4 * j + 3]);
                }
                if (g == 0) {  // row 0 of the MMA; columns 2t, 2t + 1 = batch rows 8 b + 2t (+1)
                    float* r = refs + (size_t)sp * 2 * MT;
                    r[8 * b + 2 * t] = ra[0];
                    r[8 * b + 2 * t + 1] = ra[1];
                    r[MT + 8 * b + 2 * t] = rb[0];
                    r[MT + 8 * b + 2 * t + 1] = rb[1];
                }
            }
        }
        named_bar(1, 32 * kGsConsumers);
    }

    const int lgi = GROUP >= 128 ? 0 : (32 * t) / GROUP;   // group of this lane's 32 K inside a unit
    const int zsh0 = 4 * (ch0 & 7), zsh1 = 4 * (ch1 & 7);
    bool aborted = false;
    int s = grp;                 // stage of this group's next unit (ns is even)
    uint32_t ph = 0;
    long long u = u0;
    while (u < u1) {
        const int tile = (int)(u / steps);
        const long long seg_end = ((long long)tile + 1) * steps < u1 ? ((long long)tile + 1) * steps : u1;
        float tot[NB][4], tot2[NB][4];
#pragma unroll
        for (int b = 0; b < NB; ++b)
#pragma unroll
            for (int e = 0; e < 4; ++e) tot[b][e] = tot2[b][e] = 0.0f;

        for (long long uu = u + (((u - u0) & 1) != grp ? 1 : 0); uu < seg_end; uu += 2) {
            if (!aborted && !mbar_wait(&full[s], ph, abort_flag, p.dev_status, kGsSpin)) aborted = true;
            if (!aborted) {
                const int sp = (int)(uu - (long long)tile * steps);
                const uint8_t* st = stages + (size_t)s * kGsStage;
                const uint4 w0 = *reinterpret_cast<const uint4*>(st + t * kGsHalf + ch0 * 16);
                const uint4 w1 = *reinterpret_cast<const uint4*>(st + t * kGsHalf + ch1 * 16);
                const uint16_t* sc = reinterpret_cast<const uint16_t*>(st + kGsScalesOff + 256 * lgi);
                const uint16_t sb0 = sc[ch0], sb1 = sc[ch1];
                int z0 = zr, z1 = zr;
                if (!p.sym) {
                    const uint32_t* zw = reinterpret_cast<const uint32_t*>(st + kGsZerosOff + 64 * lgi);
                    z0 = (int)((zw[ch0 >> 3] >> zsh0) & 0xFu);
                    z1 = (int)((zw[ch1 >> 3] >> zsh1) & 0xFu);
                }
                uint32_t bfr[NB][16];
                load_b(sp, bfr);
                float2 ra[NB], rb[NB];
                if constexpr (kRef) {
#pragma unroll
                    for (int b = 0; b < NB; ++b) {
                        const float* r = refs + (size_t)sp * 2 * MT;
                        ra[b] = *reinterpret_cast<const float2*>(r + 8 * b + 2 * t);
                        rb[b] = *reinterpret_cast<const float2*>(r + MT + 8 * b + 2 * t);
                    }
                }
                // the stage is in registers: let the producer refill it
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);

                const uint32_t wr0[4] = {w0.x, w0.y, w0.z, w0.w};
                const uint32_t wr1[4] = {w1.x, w1.y, w1.z, w1.w};
                if constexpr (kRef) {
                    float acc_a[NB][4], acc_b[NB][4];
#pragma unroll
                    for (int b = 0; b < NB; ++b)
#pragma unroll
                        for (int e = 0; e < 4; ++e) acc_a[b][e] = acc_b[b][e] = 0.0f;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        uint32_t q0[4], q1[4];
                        Ops::unpack(wr0[j], q0);
                        Ops::unpack(wr1[j], q1);
#pragma unroll
                        for (int b = 0; b < NB; ++b) {
                            Ops::mma(acc_a[b], q0[0], q1[0], q0[2], q1[2], bfr[b][4 * j + 0], bfr[b][4 * j + 2]);
                            Ops::mma(acc_b[b], q0[1], q1[1], q0[3], q1[3], bfr[b][4 * j + 1], bfr[b][4 * j + 3]);
                        }
                    }
                    const float s0 = __half2float(__ushort_as_half(sb0));
                    const float s1 = __half2float(__ushort_as_half(sb1));
                    const float fa0 = p.sym ? 1.0f : Ops::fa(z0), fa1 = p.sym ? 1.0f : Ops::fa(z1);
                    const float fb0 = p.sym ? 1.0f : Ops::fb(z0), fb1 = p.sym ? 1.0f : Ops::fb(z1);
#pragma unroll
                    for (int b = 0; b < NB; ++b) {
                        // elements: 0, 1 -> channel ch0, batch rows 2t, 2t+1; 2, 3 -> channel ch1
                        const float d0 = fmaf(fmaf(-rb[b].x, fb0, acc_b[b][0]), Ops::kInvB, fmaf(-ra[b].x, fa0, acc_a[b][0]));
                        const float d1 = fmaf(fmaf(-rb[b].y, fb0, acc_b[b][1]), Ops::kInvB, fmaf(-ra[b].y, fa0, acc_a[b][1]));
                        const float d2 = fmaf(fmaf(-rb[b].x, fb1, acc_b[b][2]), Ops::kInvB, fmaf(-ra[b].x, fa1, acc_a[b][2]));
                        const float d3 = fmaf(fmaf(-rb[b].y, fb1, acc_b[b][3]), Ops::kInvB, fmaf(-ra[b].y, fa1, acc_a[b][3]));
                        tot[b][0] = fmaf(s0, d0, tot[b][0]);
                        tot[b][1] = fmaf(s0, d1, tot[b][1]);
                        tot[b][2] = fmaf(s1, d2, tot[b][2]);
                        tot[b][3] = fmaf(s1, d3, tot[b][3]);
                    }
                } else {
                    const uint32_t za0 = Ops::zz_a(z0), za1 = Ops::zz_a(z1);
                    const uint32_t zb0 = Ops::zz_b(z0), zb1 = Ops::zz_b(z1);
                    typename Ops::Scale sc0, sc1;
                    sc0.set(sb0);
                    sc1.set(sb1);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        uint32_t q0[4], q1[4];
                        Ops::unpack(wr0[j], q0);
                        Ops::unpack(wr1[j], q1);
                        q0[0] = sc0.apply(Ops::sub_a(q0[0], za0));
                        q0[2] = sc0.apply(Ops::sub_a(q0[2], za0));
                        q0[1] = sc0.apply(Ops::sub_b(q0[1], zb0));
                        q0[3] = sc0.apply(Ops::sub_b(q0[3], zb0));
                        q1[0] = sc1.apply(Ops::sub_a(q1[0], za1));
                        q1[2] = sc1.apply(Ops::sub_a(q1[2], za1));
                        q1[1] = sc1.apply(Ops::sub_b(q1[1], zb1));
                        q1[3] = sc1.apply(Ops::sub_b(q1[3], zb1));
#pragma unroll
                        for (int b = 0; b < NB; ++b) {
                            Ops::mma(tot[b], q0[0], q1[0], q0[2], q1[2], bfr[b][4 * j + 0], bfr[b][4 * j + 2]);
                            Ops::mma(tot2[b], q0[1], q1[1], q0[3], q1[3], bfr[b][4 * j + 1], bfr[b][4 * j + 3]);
                        }
                    }
                }
            }
            s += 2;
            if (s >= ns) { s -= ns; ph ^= 1u; }
        }

        // ---------------------------------------------------------------- segment output
        if constexpr (!kRef) {
#pragma unroll
            for (int b = 0; b < NB; ++b)
#pragma unroll
                for (int e = 0; e < 4; ++e) tot[b][e] += tot2[b][e];
        }
        // group 1 hands its sums to group 0 through shared memory
        if (grp == 1) {
#pragma unroll
            for (int b = 0; b < NB; ++b) {
                const int m = 8 * b + 2 * t;
                red[m * 128 + ch0] = tot[b][0];
                red[(m + 1) * 128 + ch0] = tot[b][1];
                red[m * 128 + ch1] = tot[b][2];
                red[(m + 1) * 128 + ch1] = tot[b][3];
            }
        }
        named_bar(1, 32 * kGsConsumers);
        if (grp == 0) {
#pragma unroll
            for (int b = 0; b < NB; ++b) {
                const int m = 8 * b + 2 * t;
                tot[b][0] += red[m * 128 + ch0];
                tot[b][1] += red[(m + 1) * 128 + ch0];
                tot[b][2] += red[m * 128 + ch1];
                tot[b][3] += red[(m + 1) * 128 + ch1];
            }
        }
        named_bar(1, 32 * kGsConsumers);
        if (grp == 0) {
            T* C = static_cast<T*>(p.C);
            const size_t n0 = (size_t)tile * 128;
            const int c_first = unit_owner((long long)tile * steps, U, P);
            const int c_last = unit_owner((long long)tile * steps + steps - 1, U, P);
            if (c_first == c_last) {
#pragma unroll
                for (int b = 0; b < NB; ++b) {
                    const int m = 8 * b + 2 * t;
                    if (m < M) {
                        C[(size_t)m * N + n0 + ch0] = Act<T>::from_f32(tot[b][0]);
                        C[(size_t)m * N + n0 + ch1] = Act<T>::from_f32(tot[b][2]);
                    }
                    if (m + 1 < M) {
                        C[(size_t)(m + 1) * N + n0 + ch0] = Act<T>::from_f32(tot[b][1]);
                        C[(size_t)(m + 1) * N + n0 + ch1] = Act<T>::from_f32(tot[b][3]);
                    }
                }
            } else {
                // partial sums of this CTA for the tile: slot 0 if it is the CTA's first tile
                const int slot = (tile == (int)(u0 / steps)) ? 0 : 1;
                float* part = p.partials + ((size_t)cta * 2 + slot) * (size_t)M * 128;
#pragma unroll
                for (int b = 0; b < NB; ++b) {
                    const int m = 8 * b + 2 * t;
                    if (m < M) {
                        part[(size_t)m * 128 + ch0] = tot[b][0];
                        part[(size_t)m * 128 + ch1] = tot[b][2];
                    }
                    if (m + 1 < M) {
                        part[(size_t)(m + 1) * 128 + ch0] = tot[b][1];
                        part[(size_t)(m + 1) * 128 + ch1] = tot[b][3];
                    }
                }
                __threadfence();
                named_bar(2, 32 * kGsGroupWarps);
                if (ctid == 0) {
                    const int old = atomicAdd(&p.counters[tile], 1);
                    *last_flag = (old == c_last - c_first) ? 1 : 0;
                }
                named_bar(2, 32 * kGsGroupWarps);
                if (*last_flag) {
                    // the last CTA of the tile adds every CTA's partial sums in CTA order
                    __threadfence();
                    for (int e = ctid; e < M * 128; e += 32 * kGsGroupWarps) {
                        float sum = 0.0f;
                        for (int c = c_first; c <= c_last; ++c) {
                            const int sl = (tile == (int)(unit_begin(c, U, P) / steps)) ? 0 : 1;
                            sum += __ldcg(p.partials + ((size_t)c * 2 + sl) * (size_t)M * 128 + e);
                        }
                        C[(size_t)(e >> 7) * N + n0 + (e & 127)] = Act<T>::from_f32(sum);
                    }
                    if (ctid == 0) p.counters[tile] = 0;
                }
                named_bar(2, 32 * kGsGroupWarps);
            }
        }
        u = seg_end;
    }
}

template <int NB, typename T, int GROUP>
int launch_typed(const GsParams& prm, size_t smem, cudaStream_t stream) {
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(gemv_stream_kernel<NB, T, GROUP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        kGsSmemMax);
    });
    if (attr_err != cudaSuccess) return W4A16_ECUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(prm.P, 1, 1);
    cfg.blockDim = dim3(kGsThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, gemv_stream_kernel<NB, T, GROUP>, prm);
    return e == cudaSuccess ? W4A16_OK : W4A16_ECUDA;
}

template <int NB, typename T>
int launch_group(const GsParams& prm, int group, size_t smem, cudaStream_t stream) {
    switch (group) {
        case 32: return launch_typed<NB, T, 32>(prm, smem, stream);
        case 64: return launch_typed<NB, T, 64>(prm, smem, stream);
        case 128: return launch_typed<NB, T, 128>(prm, smem, stream);
        default: return W4A16_EUNSUPPORTED;
    }
}

int sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (dev < 0 || dev >= 64) return 0;
    if (cached[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
        cached[dev] = n;
    }
    return cached[dev];
}

}  // namespace

GemvStreamPlan plan_gemv_stream(int M, int N, int K, int group, int n_sm) {
    GemvStreamPlan pl = {};
    if (M < 1 || M > 16 || K % 128 != 0 || N % 128 != 0 || K < 128 || N < 128) return pl;
    if (group != 32 && group != 64 && group != 128) return pl;
    if (N / 128 > kGemvStreamMaxTiles) return pl;
    const int nb = M <= 8 ? 1 : 2;
    const size_t row_bytes = 2 * (size_t)K + 32;
    pl.act_bytes = ((size_t)M * row_bytes + 127) & ~(size_t)127;
    pl.ref_bytes = group == 128 ? (((size_t)(K / 128) * 2 * 8 * nb * 4 + 127) & ~(size_t)127) : 0;
    pl.red_bytes = (size_t)8 * nb * 128 * 4;
    const size_t fixed = pl.act_bytes + pl.ref_bytes + pl.red_bytes + 2 * kGsMaxStages * 8 + 16;
    if (fixed >= (size_t)kGsSmemMax) return pl;
    size_t ns = ((size_t)kGsSmemMax - fixed) / (kGsStage + 16);
    if (ns > kGsMaxStages) ns = kGsMaxStages;
    ns &= ~(size_t)1;
    if (ns < kGsMinStages) return pl;
    pl.ns = (int)ns;
    pl.smem = pl.act_bytes + pl.ref_bytes + pl.red_bytes + ns * kGsStage + 2 * ns * 8 + 16;
    const long long units = (long long)(N / 128) * (K / 128);
    pl.ctas = n_sm > 0 ? (int)(units < n_sm ? units : n_sm) : 0;
    pl.partial_bytes = (size_t)(n_sm > 0 ? n_sm : 0) * 2 * M * 128 * 4;
    pl.ok = pl.ctas > 0;
    return pl;
}

int gemv_stream_sm_count() { return sm_count(); }

int launch_gemv_stream(const void* A, int a_dtype, int M, int K, const void* tiled, int N, int group, int sym,
                       void* C, void* workspace, int* dev_status, cudaStream_t stream) {
    const GemvStreamPlan pl = plan_gemv_stream(M, N, K, group, sm_count());
    if (!pl.ok) return W4A16_EUNSUPPORTED;
    if (!workspace) return W4A16_EWORKSPACE;
    const TiledOffsets off = tiled_offsets(K, N, group, sym);
    GsParams prm = {};
    prm.A = A;
    prm.tiled = static_cast<const uint8_t*>(tiled);
    prm.C = C;
    prm.counters = static_cast<int*>(workspace);
    prm.partials = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kGemvStreamCounterBytes);
    prm.dev_status = dev_status;
    prm.scales_off = off.scales;
    prm.zeros_off = off.zeros;
    prm.M = M;
    prm.K = K;
    prm.N = N;
    prm.sym = sym;
    prm.ns = pl.ns;
    prm.P = pl.ctas;
    prm.row_bytes = (uint32_t)(2 * (size_t)K + 32);
    prm.act_bytes = (uint32_t)pl.act_bytes;
    prm.ref_bytes = (uint32_t)pl.ref_bytes;
    prm.red_bytes = (uint32_t)pl.red_bytes;
    if (a_dtype == W4A16_BF16) {
        if (M <= 8) return launch_group<1, __nv_bfloat16>(prm, group, pl.smem, stream);
        return launch_group<2, __nv_bfloat16>(prm, group, pl.smem, stream);
    }
    if (M <= 8) return launch_group<1, __half>(prm, group, pl.smem, stream);
    return launch_group<2, __half>(prm, group, pl.smem, stream);
}

}  // namespace w4a16
