// gemv_stream.cu -- persistent stream-K decode GEMV / skinny GEMM (M <= 16) on the tiled layout.
//
// C[m, n] = sum_k A[m, k] * (u[k, n] - z[g, n]) * s[g, n], FP32 accumulation.
// "4.3 Weight-only INT4", section 4 (read, unpack, dequantize and multiply in one pipeline so each
// weight byte crosses HBM once, with data movement overlapped with compute); "INT8 vs INT4
// Quantization, in depth", "Two regimes" (at small batch the layer waits for memory).
//
// Work split. The weights are the tiled buffer's unit records (128 channels x 128 K, codes then
// scales then zeros), ordered tile-major, so a contiguous range of units is one contiguous range
// of bytes. One CTA per SM takes floor(U / P) or ceil(U / P) consecutive units. A tile whose units
// all belong to one CTA is written straight to C. A tile cut between CTAs cf < ... < cl is the
// last tile of cf's range and the first of every later one: each later CTA publishes its FP32
// sums to the workspace and counts them (release, no wait) as soon as it has them; cf's epilogue
// warp, while cf's compute warps are still on the tile, waits for the count (acquire, bounded),
// adds the later CTAs' sums in CTA order and resets the counter; cf's own sums plus that total
// go to C. The result does not depend on timing.
//
// Pipeline. Stages of up to 4 records (34 KiB at group 128) are filled by one bulk copy each.
// Sixteen compute warps in four groups: group q takes unit q of every stage, warp w of a group
// owns channels 32 w .. 32 w + 31 of the unit; leaving a stage, each warp arrives on the slot's
// `empty` barrier. Two service warps: a producer warp refills a slot with the stage ns positions
// later once all sixteen have left it, and an epilogue warp adds the four groups' sums of each
// tile (handed over through shared memory and an mbarrier) and writes C or runs the cut-tile
// protocol. No compute warp waits for another: they wait only for their data.
//
// Math (warp-level tensor-core MMA, m16n8k16, FP32 accumulators), per warp and unit: lane
// (g = lane / 4, t = lane % 4) reads the 16 bytes of block t (32 K) of channels 32 w + g + 8 r,
// r = 0..3 (block t keeps channel n at slot n ^ 2t: the four lanes t of a channel hit different
// banks), and the unit's activations of batch rows 8 b + g.
//   Group 128, fp16 arithmetic: one AND per operand leaves a code pair in the low mantissa bits of
//   two fp16 subnormals, u 2^-24 (or 16 u 2^-24 for the upper nibble, kept in a second chain and
//   scaled by 1/16 in FP32), which the MMA multiplies exactly; the zero point comes off the unit's
//   FP32 sum as z * sum_k a_k (per-unit activation sums, formed while the activations are
//   staged), and the scale multiplies it once. bf16 activations take this path too: each CTA
//   scales every row by a power of two 2^-k (from the largest exponent among the row's staged
//   values) and converts it to fp16 exactly, then multiplies its own sums by 2^k; when some row's
//   values span more binades than fp16 holds, the CTA keeps bf16 and the next form.
//   Other cases: one mask-OR with a magic exponent (fp16 0x6400 | u = 1024 + u, 0x6400 | (u << 4)
//   = 1024 + 16 u; bf16 0x4300 | u = 128 + u) and an exact 16-bit subtraction of the zero point;
//   group 128 scales the unit's FP32 sum once; groups 64 and 32 (a lane's 32 K may span several
//   groups) scale each operand first, (u - z) * s rounded once to the 16-bit type (bf16: s = s_hi
//   + s_lo, both exact in bf16), and the MMAs accumulate the whole tile segment.
// Staging. Only the units of K that the CTA's range touches are staged. The producer issues the
// first GS_PREFETCH stages before the activations are read and the rest of the ring after: a full
// ring of weight copies issued by every SM at once is several microseconds of HBM traffic, and
// the activation loads would queue behind it.
// Every wait is bounded (the limit of w4a16_set_wait_limit_ns, 2 s by default); on expiry the
// kernel records W4A16_ETIMEOUT, stops issuing copies, still passes every barrier and tile
// counter, and lets the copies in flight land before it exits.
#include <mutex>
#include <type_traits>

#include "common.cuh"
#include "dequant.cuh"
#include "sm100_ptx.cuh"
#include "tiled_layout.cuh"

#ifndef GS_PREFETCH
#define GS_PREFETCH 2
#endif

namespace w4a16 {
namespace {

using namespace sm100;

// Four groups of 4 warps per CTA (each group takes one unit of a stage), one CTA per SM. (Two
// groups and two CTAs per SM, which let the next launch's CTAs start on an SM before the previous
// launch has left it, measured 12% slower on the Llama-3-70B-shaped stack.)
constexpr int kGsGroups = 4, kGsGroupWarps = 4, kGsWarps = kGsGroups * kGsGroupWarps;   // compute warps
constexpr int kGsCtasPerSm = 1;
// two service warps after the compute warps: one issues the weight copies, one sums the tiles
constexpr int kGsWarpProducer = kGsWarps, kGsWarpEpilogue = kGsWarps + 1, kGsAllWarps = kGsWarps + 2;
constexpr int kGsThreads = 32 * kGsAllWarps;
constexpr int kGsUnitsPerStage = kGsGroups;
static_assert(kGsGroups >= 2 && kGsGroups <= 4, "two to four groups");
constexpr int kGsMinStages = 3, kGsMaxStages = 16;
constexpr int kGsSmemMax = (228 * 1024) / kGsCtasPerSm - 1024;   // per CTA; 1 KiB reserved each
constexpr uint64_t kGsSpin = 2000000000ull;
constexpr int kGsZrowBytes = 512;   // the zero activation block, then per-row exponent bounds

__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dependents_launch() { asm volatile("griddepcontrol.launch_dependents;" :::); }

// First unit of CTA c when U units are cut into P contiguous ranges, and the CTA holding unit u.
__device__ __forceinline__ long long unit_begin(int c, long long U, int P) { return ((long long)c * U) / P; }
__device__ __forceinline__ int unit_owner(long long u, long long U, int P) { return (int)(((u + 1) * P - 1) / U); }

// Warp-uniform bounded wait: the common case (phase already complete) costs one try and a vote.
__device__ __forceinline__ bool wait_uniform(uint64_t* bar, uint32_t parity, volatile int* abort, int* dev_status,
                                             uint64_t limit_ns) {
    if (__all_sync(0xffffffffu, mbar_test_wait(bar, parity))) return true;
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, dev_status, limit_ns));
}

struct GsParams {
    const void* A;
    const uint8_t* tiled;
    void* C;
    int* counters;      // one int per tile, zero between calls
    float* partials;    // [P][M][128]: sums a CTA publishes for the tile that opens its range
    int* dev_status;
    int M, K, N, sym, ns, P;
    uint32_t record, scales_off, zeros_off;
    uint32_t stage_bytes, row_bytes, act_bytes, red_bytes, sa_bytes;
    GsMasks km;
    GsMasks km_native;   // bf16 masks, for bf16 rows kept in bf16 at group 128
    // K slices: K is the width of one slice, A points at the first column of slice 0, rows lda
    // elements apart; slice sl covers the K-steps c0 + sl K/128 .. of every tile of a
    // ktot-step weight and is served by CTAs sl P .. sl P + P - 1 of the grid (slices x P CTAs);
    // with out_f32 set the FP32 sums of slice sl go to out_f32 + sl M N ([M][N]) instead of C
    int lda, c0, ktot, slices;
    float* out_f32;
    uint64_t wait_ns;   // limit of every bounded wait (the drain after a timeout keeps kGsSpin)
};

// NB: n8 tiles of activation rows (1: M <= 8, 2: M <= 16). ODD: rows 2t + 1 of an n8 tile exist.
// SL: the launch serves several K slices (a separate instance, so that the single-slice one keeps
// no slice arithmetic).
template <int NB, typename T, int GROUP, bool ODD, bool SL>
__global__ void __launch_bounds__(kGsThreads, kGsCtasPerSm) gemv_stream_kernel(const GsParams p) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    constexpr bool kPost = (GROUP == 128);   // one group per unit: scale the unit's sum
    // bf16 activations at group 128 run the fp16 arithmetic (fewer instructions per weight)
    // whenever that is exact: each row is scaled by a power of two 2^-k that puts its largest
    // value in [2^14, 2^15) and converted to fp16. A bf16 value whose exponent is at most 31 below
    // the row's largest lands on an fp16 normal or on the fp16 subnormal grid with all 8 of its
    // significant bits, so the conversion is exact; the MMAs then form the same products
    // a * (u - z) as bf16 operands would, and the sums are multiplied back by 2^k when C is
    // written. When some row holds a nonzero value further below its maximum, every CTA keeps
    // the bf16 values and the bf16 arithmetic. Each CTA decides from the part of A it stages and
    // takes its own sums back to the scale of A before they leave it, so CTAs need not agree.
    constexpr bool kConv = kPost && std::is_same<T, __nv_bfloat16>::value;
    using MathT = typename std::conditional<kConv, __half, T>::type;
    using Ops = GsOps<MathT>;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int M = p.M, K = p.K, N = p.N, ns = p.ns, P = p.P;
    const int steps = K / 128;
    const long long U = (long long)(N / 128) * steps;
    // K slices fused into one launch: CTAs [sl P, sl P + P) serve slice sl, i.e. columns
    // sl K .. sl K + K - 1 of A and weight steps c0 + sl K/128 .., with their own tile counters and
    // partial sums, and FP32 sums to out_f32 + sl M N (a single slice: sl = 0)
    const int sl = SL ? (int)blockIdx.x / P : 0;
    const int cta = (int)blockIdx.x - sl * P;
    const int kc0 = p.c0 + sl * steps;
    int* const counters = p.counters + sl * (N / 128);
    float* const partials = p.partials + (size_t)sl * P * M * 128;
    float* const out_f32 = p.out_f32 ? p.out_f32 + (size_t)sl * M * N : nullptr;
    const long long u0 = unit_begin(cta, U, P), u1 = unit_begin(cta + 1, U, P);
    const int nunits = (int)(u1 - u0);
    const uint32_t R = p.record, stage_bytes = p.stage_bytes, RS = p.row_bytes;

    uint8_t* acts = smem_raw;                                             // [M][RS]
    float* red = reinterpret_cast<float*>(smem_raw + p.act_bytes);        // [2][groups][M][128]
    float* sa = reinterpret_cast<float*>(smem_raw + p.act_bytes + p.red_bytes);   // [K/128][Me] unit sums
    uint8_t* zrow = smem_raw + p.act_bytes + p.red_bytes + p.sa_bytes;    // 320 zero bytes
    int* rowexp = reinterpret_cast<int*>(zrow + 320);                     // [16] largest exponent per row
    int* rowmin = reinterpret_cast<int*>(zrow + 384);                     // [16] smallest nonzero one
    uint8_t* stages = zrow + kGsZrowBytes;                                // ns x stage_bytes
    uint64_t* full = reinterpret_cast<uint64_t*>(stages + (size_t)ns * stage_bytes);   // [ns] stage landed
    uint64_t* empty = full + ns;        // [ns] the 16 compute warps left the slot's stage
    uint64_t* tfull = empty + ns;       // [2] the groups' sums of a tile are in `red`
    uint64_t* tempty = tfull + 2;       // [2] the epilogue warp has read them
    int* flags = reinterpret_cast<int*>(tempty + 2);
    volatile int* abort_flag = flags;
    int* issued = flags + 2;            // [ns] copies issued into each slot

    if (threadIdx.x == 0) {
        for (int i = 0; i < ns; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kGsWarps);
            issued[i] = 0;
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tfull[i], kGsWarps);
            mbar_init(&tempty[i], 1);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    for (int i = threadIdx.x; i < 96; i += kGsThreads) reinterpret_cast<uint32_t*>(zrow)[i] = 0u;
    if (threadIdx.x < 2) reinterpret_cast<uint32_t*>(zrow + 448)[threadIdx.x] = 0u;   // two zero sums
    if (threadIdx.x < 16) rowmin[threadIdx.x] = 255;
    cta_sync();
    grid_dependents_launch();

    // stage st = records u0 + 4 st .. (up to 4), one bulk copy into slot st % ns
    const int nst = (nunits + kGsUnitsPerStage - 1) / kGsUnitsPerStage;
    auto issue = [&](int st) {
        const int s = st % ns;
        const int n = nunits - st * kGsUnitsPerStage < kGsUnitsPerStage ? nunits - st * kGsUnitsPerStage
                                                                        : kGsUnitsPerStage;
        const uint32_t bytes = (uint32_t)n * R;
        mbar_arrive_expect_tx(&full[s], bytes);
        const long long ua = u0 + (long long)st * kGsUnitsPerStage;
        uint8_t* dst = stages + (size_t)s * stage_bytes;
        if (p.ktot == steps) {
            bulk_g2s(dst, p.tiled + (size_t)ua * R, bytes, &full[s]);
        } else {
            // a K slice: units of one tile are contiguous; a stage may run into the next tile
            const long long t = ua / steps;
            const int cc = (int)(ua - t * steps);
            const int n1 = steps - cc < n ? steps - cc : n;
            bulk_g2s(dst, p.tiled + ((size_t)t * p.ktot + kc0 + cc) * R, (uint32_t)n1 * R, &full[s]);
            if (n1 < n)
                bulk_g2s(dst + (size_t)n1 * R, p.tiled + ((size_t)(t + 1) * p.ktot + kc0) * R, (uint32_t)(n - n1) * R,
                         &full[s]);
        }
        ++issued[s];
    };
    const bool producer = warp == kGsWarpProducer && lane == 0;
    const int npre = min(min(nst, ns), GS_PREFETCH);
    if (producer)
        for (int st = 0; st < npre; ++st) issue(st);

    const int grp = warp / kGsGroupWarps, wg = warp % kGsGroupWarps;
    const int g = lane >> 2, t = lane & 3;
    const int ch0 = 32 * wg + g;     // this lane's channels: ch0 + 8 r, r = 0..3
    const T* A = static_cast<const T*>(p.A) + (size_t)sl * K;

    bool wide = false;   // kConv: some row keeps bf16 values and the bf16 arithmetic

    // The units of K this CTA's range touches: all of them when the range holds a whole tile, else
    // a run of nneed units from sp0, wrapping at the end of the tile. Only their activations are
    // staged, scanned and summed (a CTA of the 28672-input down projection touches 43% of K).
    const int sp0 = (int)(u0 % steps);
    const int nneed = nunits < steps ? nunits : steps;
    const int nchunk = 16 * nneed;   // 8-element chunks of A

    // A may be the output of the previous kernel in the stream
    grid_dependency_wait();

    // Staging: activations: 32-K block t of unit sp at sp * 320 + 80 t (the 16-byte padding makes
    // the lanes' 16-byte reads conflict free); pairs in each 16-byte chunk stored (p0, p2, p1, p3)
    // so that each MMA's two B registers are adjacent; each CTA starts at a different chunk. Chunk
    // c0 of the pass (c0 = thread + i * threads) is chunk q = c0 + rot (mod nchunk) of the needed
    // run; since threads, rot and nchunk are multiples of 16, the 16 lanes of a half warp hold the
    // 16 chunks of one unit, whose sum (group 128 on the fp16 arithmetic: z sum_k a_k comes off the
    // FP32 sums) is then a half-warp reduction in a fixed order, kept times 2^-24 (the subnormal
    // codes' scale).
    constexpr bool kSub = kPost && std::is_same<MathT, __half>::value;
    const int Me = (M + 1) & ~1;
    const int rot = (cta * 64) % nchunk;
    auto chunk_of = [&](int c0, int& sp) {
        int q = c0 + rot;
        if (q >= nchunk) q -= nchunk;
        sp = sp0 + (q >> 4);
        if (sp >= steps) sp -= steps;
        return 16 * sp + (q & 15);
    };
    auto chunk_off = [&](int m, int c) {
        return (uint32_t)m * RS + (uint32_t)(c >> 4) * 320u + (uint32_t)((c >> 2) & 3) * 80u + (uint32_t)(c & 3) * 16u;
    };
    // sum of the unit over the half warp (a pass's bound on c0 is the same for all 16 lanes of a
    // half, not always for the other half: hence the half's own mask); lane 0 of the half writes it
    const uint32_t half_mask = 0xFFFFu << (lane & 16);
    auto unit_sum = [&](float v, int m, int sp) {
        v += __shfl_xor_sync(half_mask, v, 8);
        v += __shfl_xor_sync(half_mask, v, 4);
        v += __shfl_xor_sync(half_mask, v, 2);
        v += __shfl_xor_sync(half_mask, v, 1);
        if ((lane & 15) == 0) sa[sp * Me + m] = v * 5.9604644775390625e-08f;   // 2^-24
    };
    auto half8_sum = [](const uint4& v) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        float s8 = 0.0f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __half2 h = *reinterpret_cast<const __half2*>(&w[i]);
            s8 += __low2float(h) + __high2float(h);
        }
        return s8;
    };
    for (int m = 0; m < M; ++m) {
        uint32_t emax = 0, emin = 255;   // largest, smallest nonzero biased exponent of row m
        for (int c0 = threadIdx.x; c0 < nchunk; c0 += 4 * kGsThreads) {
            uint4 vv[4];
            int cc[4], sps[4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (c0 + j * kGsThreads < nchunk) {
                    cc[j] = chunk_of(c0 + j * kGsThreads, sps[j]);
                    vv[j] = *reinterpret_cast<const uint4*>(A + (size_t)m * p.lda + 8 * cc[j]);
                }
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (c0 + j * kGsThreads < nchunk) {
                    *reinterpret_cast<uint4*>(acts + chunk_off(m, cc[j])) = make_uint4(vv[j].x, vv[j].z, vv[j].y, vv[j].w);
                    if constexpr (kConv) {
                        const uint32_t x[4] = {vv[j].x, vv[j].y, vv[j].z, vv[j].w};
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const uint32_t e0 = (x[q] >> 7) & 0xFFu, e1 = (x[q] >> 23) & 0xFFu;
                            emax = max(emax, max(e0, e1));
                            if (x[q] & 0x7FFFu) emin = min(emin, e0);
                            if (x[q] & 0x7FFF0000u) emin = min(emin, e1);
                        }
                    } else if constexpr (kSub) {
                        unit_sum(half8_sum(vv[j]), m, sps[j]);
                    }
                }
        }
        if constexpr (kConv) {
            emax = __reduce_max_sync(0xffffffffu, emax);
            emin = __reduce_min_sync(0xffffffffu, emin);
            if (lane == 0) {
                atomicMax(&rowexp[m], (int)emax);
                atomicMin(&rowmin[m], (int)emin);
            }
        }
    }
    if constexpr (kConv) {
        // second pass, in shared memory: bf16 -> 2^-k * a in fp16, unless some row is too wide, and
        // the unit sums of the converted values
        cta_sync();
        for (int m = 0; m < M; ++m) wide = wide || rowexp[m] - rowmin[m] > 31;
        for (int m = 0; m < M && !wide; ++m) {
            const int k = min(max(rowexp[m] - 141, -100), 114);
            const float down = __int_as_float((127 - k) << 23);
            for (int c0 = threadIdx.x; c0 < nchunk; c0 += kGsThreads) {
                int sp;
                const int c = chunk_of(c0, sp);
                uint4* q = reinterpret_cast<uint4*>(acts + chunk_off(m, c));
                uint4 v = *q;
                uint32_t* w = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    __half2 h = __floats2half2_rn(__uint_as_float(w[i] << 16) * down,
                                                  __uint_as_float(w[i] & 0xFFFF0000u) * down);
                    w[i] = *reinterpret_cast<uint32_t*>(&h);
                }
                *q = v;
                unit_sum(half8_sum(v), m, sp);
            }
        }
    }
    if constexpr (kSub)
        if (M & 1)
            for (int q = threadIdx.x; q < nneed; q += kGsThreads) {
                int sp = sp0 + q;
                if (sp >= steps) sp -= steps;
                sa[sp * Me + M] = 0.0f;
            }
    cta_sync();

    // activation fragments: lane holds row 8 b + g (rows at or past M read a zero block)
    const uint8_t* abase[NB];
    uint32_t astride[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b) {
        const bool real = 8 * b + g < M;
        abase[b] = real ? acts + (uint32_t)(8 * b + g) * RS + (uint32_t)t * 80u : zrow + (uint32_t)t * 80u;
        astride[b] = real ? 320u : 0u;
    }

    // unit sums of the two batch columns 8 b + 2 t, + 1 this lane's MMA results hold
    const float* sbase[NB];
    uint32_t sstride[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b) {
        const bool real = 8 * b + 2 * t < M;
        sbase[b] = real ? sa + 8 * b + 2 * t : reinterpret_cast<const float*>(zrow + 448);
        sstride[b] = real ? (uint32_t)Me : 0u;
    }

    const GsMasks km = p.km;
    const int lg = kPost ? 0 : (32 * t) / GROUP;                                  // group of block t
    const uint32_t coff = (uint32_t)t * 2048u + (uint32_t)(ch0 ^ (2 * t)) * 16u;   // channel ch0 + 8 r: + 128 r
    const uint32_t soff = p.scales_off + 256u * (uint32_t)lg + 2u * (uint32_t)ch0; // + 16 r
    const uint32_t zoff = p.zeros_off + 64u * (uint32_t)lg + 16u * (uint32_t)wg;   // words of ch0 + 8 r
    const int zsh = 4 * g;
    const uint32_t rec_off = (uint32_t)grp * R;
    const int sym = p.sym;

    float tot[2][NB][4];
    auto zero_tot = [&]() {
#pragma unroll
        for (int rt = 0; rt < 2; ++rt)
#pragma unroll
            for (int b = 0; b < NB; ++b) tot[rt][b][0] = tot[rt][b][1] = tot[rt][b][2] = tot[rt][b][3] = 0.0f;
    };
    zero_tot();
    int tile = (int)(u0 / steps);
    int seg_lo = 0, sp_lo = (int)(u0 - (long long)tile * steps);
    int seg_hi = (steps - sp_lo) < nunits ? (steps - sp_lo) : nunits;

    // End of a tile segment (compute warps): each group writes its FP32 sums of the tile's 128
    // channels to one of two shared buffers (by tile parity) and arrives on its `full` barrier; the
    // epilogue warp adds the four groups' sums and writes C (or this CTA's partial sums when the
    // tile is cut between CTAs) and frees the buffer. A group waits only before it reuses a buffer
    // two tiles later, which the epilogue warp has normally long released; no compute warp waits
    // for another.
    int n_tile = 0;
    auto tile_end = [&]() {
        const int bsel = n_tile & 1;
        const uint32_t use = (uint32_t)(n_tile >> 1) & 1u;
        (void)wait_uniform(&tempty[bsel], use ^ 1u, abort_flag, p.dev_status, p.wait_ns);
        float* rb = red + ((size_t)bsel * kGsGroups + grp) * M * 128;
#pragma unroll
        for (int rt = 0; rt < 2; ++rt)
#pragma unroll
            for (int b = 0; b < NB; ++b)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int m = 8 * b + 2 * t + (e & 1), ch = ch0 + 16 * rt + 8 * (e >> 1);
                    if (m < M) rb[m * 128 + ch] = tot[rt][b][e];
                }
        __syncwarp();
        if (lane == 0) mbar_arrive(&tfull[bsel]);
        ++n_tile;
        zero_tot();
        ++tile;
        sp_lo = 0;
        seg_lo = seg_hi;
        seg_hi = seg_lo + steps < nunits ? seg_lo + steps : nunits;
    };

    // the MMAs of one unit, with the operand arithmetic of O (fp16 or bf16)
    auto unit_math = [&](auto tag, const GsMasks& kx, const uint4 (&cw)[4], const uint16_t (&sb)[4],
                         const uint4& zw, const uint4 (&v)[NB][4]) {
        using O = typename decltype(tag)::type;
        const uint32_t zws[4] = {zw.x, zw.y, zw.z, zw.w};
#pragma unroll
        for (int rt = 0; rt < 2; ++rt) {
            // MMA rows g / g + 8: channels ch0 + 16 rt / ch0 + 16 rt + 8
            const uint4 c0 = cw[2 * rt], c1 = cw[2 * rt + 1];
            const uint32_t w0[4] = {c0.x, c0.y, c0.z, c0.w}, w1[4] = {c1.x, c1.y, c1.z, c1.w};
            const uint32_t z0 = (zws[2 * rt] >> zsh) & 0xFu, z1 = (zws[2 * rt + 1] >> zsh) & 0xFu;
            const uint32_t za0 = O::zz_a(z0), za1 = O::zz_a(z1), zb0 = O::zz_b(z0), zb1 = O::zz_b(z1);
            typename O::Scale sc0, sc1;
            if constexpr (!kPost) {
                sc0.set(sb[2 * rt]);
                sc1.set(sb[2 * rt + 1]);
            }
            float acc[NB][4];
#pragma unroll
            for (int b = 0; b < NB; ++b) acc[b][0] = acc[b][1] = acc[b][2] = acc[b][3] = 0.0f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                uint32_t q0[4], q1[4];
                O::unpack(w0[i], kx, q0);
                O::unpack(w1[i], kx, q1);
                q0[0] = O::sub_a(q0[0], za0);
                q0[2] = O::sub_a(q0[2], za0);
                q0[1] = O::sub_b(q0[1], zb0);
                q0[3] = O::sub_b(q0[3], zb0);
                q1[0] = O::sub_a(q1[0], za1);
                q1[2] = O::sub_a(q1[2], za1);
                q1[1] = O::sub_b(q1[1], zb1);
                q1[3] = O::sub_b(q1[3], zb1);
                if constexpr (!kPost) {
#pragma unroll
                    for (int x = 0; x < 4; ++x) {
                        q0[x] = sc0.apply(q0[x]);
                        q1[x] = sc1.apply(q1[x]);
                    }
                }
#pragma unroll
                for (int b = 0; b < NB; ++b) {
                    float (&d)[4] = kPost ? acc[b] : tot[rt][b];
                    O::mma(d, q0[0], q1[0], q0[2], q1[2], v[b][i].x, v[b][i].y);
                    O::mma(d, q0[1], q1[1], q0[3], q1[3], v[b][i].z, v[b][i].w);
                }
            }
            if constexpr (kPost) {
                const float s0 = __half2float(__ushort_as_half(sb[2 * rt]));
                const float s1 = __half2float(__ushort_as_half(sb[2 * rt + 1]));
#pragma unroll
                for (int b = 0; b < NB; ++b) {
                    tot[rt][b][0] = fmaf(s0, acc[b][0], tot[rt][b][0]);
                    tot[rt][b][2] = fmaf(s1, acc[b][2], tot[rt][b][2]);
                    if (ODD) {
                        tot[rt][b][1] = fmaf(s0, acc[b][1], tot[rt][b][1]);
                        tot[rt][b][3] = fmaf(s1, acc[b][3], tot[rt][b][3]);
                    }
                }
            }
        }
    };

    // Group 128 on the fp16 arithmetic: each operand register is one AND of a packed word, which
    // leaves the codes as fp16 subnormals u 2^-24 (pairs (0, 1), (4, 5) of the word) and 16 u 2^-24
    // (pairs (2, 3), (6, 7)), multiplied exactly by the MMA and summed in two chains (lo, hi) per
    // row tile; no magic exponent and no zero-point arithmetic per weight. Per unit and channel
    // the zero point then comes off the FP32 sum, lo + hi / 16 - z sum_k a_k 2^-24, and the scale
    // (times 2^24) multiplies the result. A group whose codes all equal its zero point has scale
    // 0 in the tiled layout, so it adds exactly nothing.
    auto unit_math_sub = [&](const uint4 (&cw)[4], const uint16_t (&sb)[4], const uint4& zw, const uint4 (&v)[NB][4],
                             int sp) {
        using O = GsOps<__half>;
        const uint32_t zws[4] = {zw.x, zw.y, zw.z, zw.w};
        float2 su[NB];
#pragma unroll
        for (int b = 0; b < NB; ++b) su[b] = *reinterpret_cast<const float2*>(sbase[b] + (uint32_t)sp * sstride[b]);
#pragma unroll
        for (int rt = 0; rt < 2; ++rt) {
            // MMA rows g / g + 8: channels ch0 + 16 rt / ch0 + 16 rt + 8
            const uint4 c0 = cw[2 * rt], c1 = cw[2 * rt + 1];
            const uint32_t w0[4] = {c0.x, c0.y, c0.z, c0.w}, w1[4] = {c1.x, c1.y, c1.z, c1.w};
            float alo[NB][4], ahi[NB][4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint32_t h0 = mulhi(w0[i], km.m8), h1 = mulhi(w1[i], km.m8);
                const uint32_t a0 = w0[i] & 0x000F000Fu, a1 = w1[i] & 0x000F000Fu;
                const uint32_t a2 = h0 & 0x000F000Fu, a3 = h1 & 0x000F000Fu;
                const uint32_t b0 = w0[i] & 0x00F000F0u, b1 = w1[i] & 0x00F000F0u;
                const uint32_t b2 = h0 & 0x00F000F0u, b3 = h1 & 0x00F000F0u;
#pragma unroll
                for (int b = 0; b < NB; ++b) {
                    if (i == 0) {
                        O::mma_z(alo[b], a0, a1, a2, a3, v[b][i].x, v[b][i].y);
                        O::mma_z(ahi[b], b0, b1, b2, b3, v[b][i].z, v[b][i].w);
                    } else {
                        O::mma(alo[b], a0, a1, a2, a3, v[b][i].x, v[b][i].y);
                        O::mma(ahi[b], b0, b1, b2, b3, v[b][i].z, v[b][i].w);
                    }
                }
            }
            const float z0 = (float)((zws[2 * rt] >> zsh) & 0xFu), z1 = (float)((zws[2 * rt + 1] >> zsh) & 0xFu);
            const float s0 = __half2float(__ushort_as_half(sb[2 * rt])) * 16777216.0f;
            const float s1 = __half2float(__ushort_as_half(sb[2 * rt + 1])) * 16777216.0f;
#pragma unroll
            for (int b = 0; b < NB; ++b) {
                tot[rt][b][0] = fmaf(s0, fmaf(-z0, su[b].x, fmaf(ahi[b][0], 0.0625f, alo[b][0])), tot[rt][b][0]);
                tot[rt][b][2] = fmaf(s1, fmaf(-z1, su[b].x, fmaf(ahi[b][2], 0.0625f, alo[b][2])), tot[rt][b][2]);
                if (ODD) {
                    tot[rt][b][1] = fmaf(s0, fmaf(-z0, su[b].y, fmaf(ahi[b][1], 0.0625f, alo[b][1])), tot[rt][b][1]);
                    tot[rt][b][3] = fmaf(s1, fmaf(-z1, su[b].y, fmaf(ahi[b][3], 0.0625f, alo[b][3])), tot[rt][b][3]);
                }
            }
        }
    };

    if (warp == kGsWarpProducer) {
        // ------------------------------------------------------------ producer (lane 0)
        // refills slot s with stage st once the 16 compute warps have left stage st - ns
        if (lane == 0) {
            for (int st = npre; st < nst && st < ns; ++st) issue(st);
            for (int st = ns; st < nst; ++st) {
                if (!mbar_wait(&empty[st % ns], (uint32_t)((st / ns) - 1) & 1u, abort_flag, p.dev_status, p.wait_ns))
                    break;
                issue(st);
            }
        }
    } else if (warp == kGsWarpEpilogue) {
        // ------------------------------------------------------------ epilogue warp
        // per tile segment of this CTA's range: the four groups' sums (in group order), then C, or
        // the cut-tile protocol; lane l handles channels l + 32 j
        T* C = static_cast<T*>(p.C);
        int etile = (int)(u0 / steps);
        int elo = 0;
        int ehi = (steps - (int)(u0 - (long long)etile * steps)) < nunits ? (steps - (int)(u0 - (long long)etile * steps))
                                                                            : nunits;
        for (int et = 0; elo < nunits; ++et) {
            const int bsel = et & 1;
            const size_t n0 = (size_t)etile * 128;
            const int cf = unit_owner((long long)etile * steps, U, P);
            const int cl = unit_owner((long long)etile * steps + steps - 1, U, P);
            // The tile is cut between CTAs cf .. cl and this is cf: the tile is the last of this
            // range, and the later CTAs hold it at the start of theirs. Before this CTA's own sums
            // are in, wait until they have all published theirs and add them up, in CTA order, into
            // the other shared buffer (free: no tile follows), so that reaching them from L2 is off
            // the path once the compute warps finish.
            const bool gather = cf != cl && cta == cf;
            float* pre = red + (size_t)(bsel ^ 1) * kGsGroups * M * 128;
            if (gather) {
                if (lane == 0) {
                    const uint64_t t0 = globaltimer_ns();
                    for (;;) {
                        int n;
                        asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(n) : "l"(counters + etile)
                                     : "memory");
                        if (n >= cl - cf) break;
                        if (*abort_flag || globaltimer_ns() - t0 > p.wait_ns) {
                            *abort_flag = 1;
                            report_status(p.dev_status, W4A16_ETIMEOUT);
                            break;
                        }
                    }
                    counters[etile] = 0;
                }
                __syncwarp();
                for (int m = 0; m < M; ++m) {
                    float y[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                    // the loads of four CTAs in flight together
                    for (int c0 = cf + 1; c0 <= cl; c0 += 4) {
                        float ld[4][4];
#pragma unroll
                        for (int q = 0; q < 4; ++q)
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                ld[q][j] = c0 + q <= cl ? __ldcg(partials + ((size_t)(c0 + q) * M + m) * 128 + lane + 32 * j)
                                                        : 0.0f;
#pragma unroll
                        for (int q = 0; q < 4; ++q)
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                if (c0 + q <= cl) y[j] += ld[q][j];
                    }
#pragma unroll
                    for (int j = 0; j < 4; ++j) pre[m * 128 + lane + 32 * j] = y[j];
                }
            }
            (void)wait_uniform(&tfull[bsel], (uint32_t)(et >> 1) & 1u, abort_flag, p.dev_status, p.wait_ns);
            const float* rb = red + (size_t)bsel * kGsGroups * M * 128;
            if (cf == cl || cta == cf) {
                for (int m = 0; m < M; ++m) {
                    float up = 1.0f;
                    if constexpr (kConv)   // undo the row's 2^-k
                        if (!wide) up = __int_as_float((127 + min(max(rowexp[m] - 141, -100), 114)) << 23);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int ch = lane + 32 * j;
                        // this CTA's sums, back in the scale of A, then the later CTAs' (a lane
                        // reads back only what it wrote)
                        float o = (rb[(0 * M + m) * 128 + ch] + rb[(1 * M + m) * 128 + ch] + rb[(2 * M + m) * 128 + ch] +
                                   rb[(3 * M + m) * 128 + ch]) * up;
                        if (gather) o += pre[m * 128 + ch];
                        if (out_f32)
                            out_f32[(size_t)m * N + n0 + ch] = o;
                        else
                            C[(size_t)m * N + n0 + ch] = Act<T>::from_f32(o);
                    }
                }
            } else {
                // a later CTA of a cut tile (the tile opens its range): publish this CTA's sums and
                // count them, without waiting
                float* part = partials + (size_t)cta * M * 128;
                for (int m = 0; m < M; ++m) {
                    float up = 1.0f;
                    if constexpr (kConv)   // undo the row's 2^-k (this CTA's)
                        if (!wide) up = __int_as_float((127 + min(max(rowexp[m] - 141, -100), 114)) << 23);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int ch = lane + 32 * j;
                        part[m * 128 + ch] = (rb[(0 * M + m) * 128 + ch] + rb[(1 * M + m) * 128 + ch] +
                                              rb[(2 * M + m) * 128 + ch] + rb[(3 * M + m) * 128 + ch]) * up;
                    }
                }
                __threadfence();
                __syncwarp();
                if (lane == 0)
                    asm volatile("red.release.gpu.global.add.s32 [%0], 1;" ::"l"(counters + etile) : "memory");
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[bsel]);
            ++etile;
            elo = ehi;
            ehi = elo + steps < nunits ? elo + steps : nunits;
        }
    } else {
        // ------------------------------------------------------------ compute warps
        // Group grp takes unit 4 st + grp of stage st. The loop runs over the tile segments of the
        // range, each ended by tile_end outside the unit loop (which keeps its registers to
        // itself); the units of consecutive segments are consecutive stages. A group with no unit
        // in the last stage neither waits for it nor leaves it: no copy refills the last stage.
        bool aborted = false;
        int s_idx = -1;
        uint32_t ph = 0;
        for (;;) {
            for (int li = seg_lo + ((grp - seg_lo) & 3); li < seg_hi; li += kGsUnitsPerStage) {
                if (++s_idx == ns) {
                    s_idx = 0;
                    ph ^= 1u;
                }
                if (!aborted && !wait_uniform(&full[s_idx], ph, abort_flag, p.dev_status, p.wait_ns)) aborted = true;
                if (!aborted) {
                    const int sp = sp_lo + (li - seg_lo);
                    const uint8_t* rec = stages + (uint32_t)s_idx * stage_bytes + rec_off;
                    uint4 cw[4];
#pragma unroll
                    for (int r = 0; r < 4; ++r) cw[r] = *reinterpret_cast<const uint4*>(rec + coff + 128 * r);
                    uint16_t sb[4];
#pragma unroll
                    for (int r = 0; r < 4; ++r) sb[r] = *reinterpret_cast<const uint16_t*>(rec + soff + 16 * r);
                    uint4 zw = make_uint4(0x88888888u, 0x88888888u, 0x88888888u, 0x88888888u);   // symmetric: z = 8
                    if (!sym) zw = *reinterpret_cast<const uint4*>(rec + zoff);
                    uint4 v[NB][4];
#pragma unroll
                    for (int b = 0; b < NB; ++b) {
                        const uint8_t* a = abase[b] + (uint32_t)sp * astride[b];
#pragma unroll
                        for (int i = 0; i < 4; ++i) v[b][i] = *reinterpret_cast<const uint4*>(a + 16 * i);
                    }
                    if constexpr (kConv) {
                        if (wide) unit_math(OpsTag<GsOps<__nv_bfloat16>>{}, p.km_native, cw, sb, zw, v);
                        else unit_math_sub(cw, sb, zw, v, sp);
                    } else if constexpr (kSub) {
                        unit_math_sub(cw, sb, zw, v, sp);
                    } else {
                        unit_math(OpsTag<Ops>{}, km, cw, sb, zw, v);
                    }
                }
                // leave the stage: this warp's reads of the slot were consumed by its MMAs (after
                // giving up, no more: the slot may still have a copy in flight, not to be reissued)
                __syncwarp();
                if (lane == 0 && !aborted) mbar_arrive(&empty[s_idx]);
            }
            tile_end();
            if (seg_lo >= nunits) break;
        }
    }

    // after a timeout: let every copy still in flight land before the CTA exits (a wait that does
    // not give up on the raised abort flag, still bounded in time); only the producer issues copies
    cta_sync();
    if (producer && *abort_flag) {
        volatile int keep_waiting = 0;
        for (int s = 0; s < ns; ++s)
            if (issued[s] > 0) mbar_wait(&full[s], (uint32_t)(issued[s] - 1) & 1u, &keep_waiting, nullptr, kGsSpin);
    }
}

template <int NB, typename T, int GROUP, bool ODD, bool SL>
int launch_typed(const GsParams& prm, size_t smem, cudaStream_t stream) {
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(gemv_stream_kernel<NB, T, GROUP, ODD, SL>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, kGsSmemMax);
    });
    if (attr_err != cudaSuccess) return W4A16_ECUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(prm.P * prm.slices, 1, 1);
    cfg.blockDim = dim3(kGsThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, gemv_stream_kernel<NB, T, GROUP, ODD, SL>, prm);
    return e == cudaSuccess ? W4A16_OK : W4A16_ECUDA;
}

template <int NB, typename T, bool ODD, bool SL>
int launch_group(const GsParams& prm, int group, size_t smem, cudaStream_t stream) {
    switch (group) {
        case 32: return launch_typed<NB, T, 32, ODD, SL>(prm, smem, stream);
        case 64: return launch_typed<NB, T, 64, ODD, SL>(prm, smem, stream);
        case 128: return launch_typed<NB, T, 128, ODD, SL>(prm, smem, stream);
        default: return W4A16_EUNSUPPORTED;
    }
}

template <int NB, typename T, bool ODD>
int launch_sliced(const GsParams& prm, int group, size_t smem, cudaStream_t stream) {
    return prm.slices > 1 ? launch_group<NB, T, ODD, true>(prm, group, smem, stream)
                          : launch_group<NB, T, ODD, false>(prm, group, smem, stream);
}

template <typename T>
int launch_rows(const GsParams& prm, int group, size_t smem, cudaStream_t stream) {
    if (prm.M > 8) return launch_sliced<2, T, true>(prm, group, smem, stream);
    if (prm.M > 1) return launch_sliced<1, T, true>(prm, group, smem, stream);
    return launch_sliced<1, T, false>(prm, group, smem, stream);
}

// C = sum over the S slices of the FP32 partial outputs, in slice order.
template <typename T>
__global__ void __launch_bounds__(256) gs_slice_reduce_kernel(const float* __restrict__ parts, int S, size_t MN,
                                                              T* __restrict__ C) {
    for (size_t i = (size_t)blockIdx.x * 256 + threadIdx.x; i < MN; i += (size_t)gridDim.x * 256) {
        float y = 0.0f;
        for (int k = 0; k < S; ++k) y += parts[(size_t)k * MN + i];
        C[i] = Act<T>::from_f32(y);
    }
}

int sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (cached[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
        cached[dev] = n;
    }
    return cached[dev];
}

}  // namespace

namespace {

// The layout of one launch over a K slice of Ks input channels.
GemvStreamPlan plan_slice(int M, int N, int Ks, int group, int sym, int n_sm) {
    GemvStreamPlan pl = {};
    const TiledLayout L = tiled_layout(Ks, N, group, sym);   // the record size does not depend on K
    const size_t units = (size_t)(Ks / 128);
    pl.row_bytes = 320 * units + ((units & 1) ? 0 : 64);          // 80-byte blocks; rows 64 mod 128 apart
    pl.act_bytes = ((size_t)M * pl.row_bytes + 127) & ~(size_t)127;
    pl.red_bytes = (size_t)2 * kGsGroups * M * 128 * 4;
    pl.sa_bytes = (((size_t)units * ((M + 1) & ~1) * 4) + 127) & ~(size_t)127;   // unit sums (group 128)
    pl.stage_bytes = ((size_t)kGsUnitsPerStage * L.record + 127) & ~(size_t)127;
    const size_t flags = ((size_t)2 * kGsMaxStages * 8 + 32 + 8 + 4 * kGsMaxStages + 127) & ~(size_t)127;
    const size_t fixed = pl.act_bytes + pl.red_bytes + pl.sa_bytes + kGsZrowBytes + flags;
    if (fixed >= (size_t)kGsSmemMax) return pl;
    size_t ns = ((size_t)kGsSmemMax - fixed) / pl.stage_bytes;
    if (ns > kGsMaxStages) ns = kGsMaxStages;
    if (ns < kGsMinStages) return pl;
    pl.ns = (int)ns;
    pl.smem = fixed + ns * pl.stage_bytes;
    const long long total_units = (long long)(N / 128) * (Ks / 128);
    const long long slots = (long long)kGsCtasPerSm * n_sm;
    pl.ctas = n_sm > 0 ? (int)(total_units < slots ? total_units : slots) : 0;
    pl.ok = pl.ctas > 0;
    return pl;
}

}  // namespace

// The whole K at once when the M rows of A fit in shared memory beside three stages; otherwise K
// is cut into S equal slices (S a power of two dividing K / 128), each served by its own group of
// n_sm / S CTAs of the same launch, whose FP32 outputs a last kernel adds in slice order.
GemvStreamPlan plan_gemv_stream(int M, int N, int K, int group, int sym, int n_sm) {
    GemvStreamPlan pl = {};
    if (M < 1 || M > 16 || K % 128 != 0 || N % 128 != 0 || K < 128 || N < 128) return pl;
    if (group != 32 && group != 64 && group != 128) return pl;
    if (N / 128 > kGemvStreamMaxTiles) return pl;
    for (int S = 1; S <= 64 && (K / 128) % S == 0; S *= 2) {
        if ((long long)(N / 128) * S > kGemvStreamMaxTiles) break;   // tile counters of every slice
        pl = plan_slice(M, N, K / S, group, sym, S > 1 ? n_sm / S : n_sm);
        if (pl.ok) {
            pl.slices = S;
            pl.partial_bytes = (size_t)2 * kGsCtasPerSm * (n_sm > 0 ? n_sm : 0) * M * 128 * 4 +
                               (S > 1 ? (size_t)S * M * N * 4 : 0);
            return pl;
        }
    }
    return GemvStreamPlan{};
}

int gemv_stream_sm_count() { return sm_count(); }

int launch_gemv_stream(const void* A, int a_dtype, int M, int K, const void* tiled, int N, int group, int sym,
                       void* C, void* workspace, int* dev_status, cudaStream_t stream) {
    const GemvStreamPlan pl = plan_gemv_stream(M, N, K, group, sym, sm_count());
    if (!pl.ok) return W4A16_EUNSUPPORTED;
    if (!workspace) return W4A16_EWORKSPACE;
    const int S = pl.slices;
    const int Ks = K / S;
    const TiledLayout L = tiled_layout(K, N, group, sym);
    GsParams prm = {};
    prm.tiled = static_cast<const uint8_t*>(tiled);
    prm.C = C;
    prm.counters = static_cast<int*>(workspace);
    prm.partials = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kGemvStreamCounterBytes);
    float* slice_out = prm.partials + (size_t)2 * kGsCtasPerSm * sm_count() * M * 128;
    prm.dev_status = dev_status;
    prm.M = M;
    prm.K = Ks;
    prm.N = N;
    prm.sym = sym;
    prm.ns = pl.ns;
    prm.P = pl.ctas;
    prm.record = L.record;
    prm.scales_off = L.scales;
    prm.zeros_off = L.zeros;
    prm.stage_bytes = (uint32_t)pl.stage_bytes;
    prm.row_bytes = (uint32_t)pl.row_bytes;
    prm.act_bytes = (uint32_t)pl.act_bytes;
    prm.red_bytes = (uint32_t)pl.red_bytes;
    prm.sa_bytes = (uint32_t)pl.sa_bytes;
    prm.lda = K;
    prm.ktot = K / 128;
    prm.wait_ns = wait_limit_ns();
    const bool bf16 = a_dtype == W4A16_BF16;
    const bool bf16_math = bf16 && group != 128;   // bf16 at group 128 runs the fp16 arithmetic
    prm.km.lo = 0x000F000Fu;
    prm.km.hi = bf16_math ? 0x000F000Fu : 0x00F000F0u;
    prm.km.magic = bf16_math ? 0x43004300u : 0x64006400u;
    prm.km.m4 = 1u << 28;
    prm.km.m8 = 1u << 24;
    prm.km.m12 = 1u << 20;
    prm.km_native = prm.km;
    prm.km_native.hi = 0x000F000Fu;
    prm.km_native.magic = 0x43004300u;
    prm.A = A;
    prm.c0 = 0;
    prm.slices = S;
    prm.out_f32 = S > 1 ? slice_out : nullptr;
    const int st = bf16 ? launch_rows<__nv_bfloat16>(prm, group, pl.smem, stream)
                        : launch_rows<__half>(prm, group, pl.smem, stream);
    if (st != W4A16_OK) return st;
    if (S > 1) {
        const size_t MN = (size_t)M * N;
        const unsigned blocks = (unsigned)((MN + 255) / 256 < 2048 ? (MN + 255) / 256 : 2048);
        if (bf16)
            gs_slice_reduce_kernel<__nv_bfloat16><<<blocks, 256, 0, stream>>>(slice_out, S, MN,
                                                                              static_cast<__nv_bfloat16*>(C));
        else
            gs_slice_reduce_kernel<__half><<<blocks, 256, 0, stream>>>(slice_out, S, MN, static_cast<__half*>(C));
        return launch_status();
    }
    return W4A16_OK;
}

}  // namespace w4a16
