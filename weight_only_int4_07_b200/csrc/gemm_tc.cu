// gemm_tc.cu -- persistent stream-K tcgen05 tensor-core W4A16 GEMM for sm_100a (the larger-M path).
//
// C[M, N] = A[M, K] . dequant(W)[K, N], FP32 accumulation in tensor memory.
// "4.3 Weight-only INT4", section 4: read, unpack, dequantize and multiply in one pipeline, each
// weight byte crossing HBM once, data movement overlapped with on-chip compute; section 1: codes
// dequantized on chip to FP16/BF16, multiply inputs stay 16-bit. "INT8 vs INT4 Quantization, in
// depth", "Two regimes": for tens of rows the layer still waits for memory, so every SM streams
// weights; for hundreds it waits for the tensor cores.
//
// Mapping. The MMA computes D[n, m] = sum_k W^T[n, k] A^T[k, m] (swap-AB): the dequantized weight
// tile (128 output channels x 64 K) is operand A (M_mma = 128), the activation tile (BN rows of
// A x 64 K, 128-byte swizzle, loaded by TMA) is operand B (N_mma = BN), D (128 x BN, FP32) lives
// in tensor memory, lane = output channel, column = row of A.
//
// Work split (stream-K). A tile is 128 output channels x one block of BN rows of A, the whole K;
// tiles are ordered channel-major (the row blocks of one channel tile are neighbours, so their
// weights are read from HBM once and from L2 after). The U = tiles x K/128 unit steps (one unit
// record of the tiled buffer each) are cut into P contiguous ranges, one per SM, so every SM
// streams the same number of weight bytes whatever the shape. A tile cut between CTAs cf < ... <
// cl is the last of cf's range and the first of every later one: each later CTA publishes its
// FP32 sums to the workspace and counts them (release, no wait); cf, after its own last unit,
// waits for the count (acquire, bounded), adds the sums in CTA order, writes C and resets the
// counter. The result does not depend on timing.
//
// Warp roles (768 threads):
//   warp 0      : weight loader -- one bulk copy per two unit records (codes, scales and zeros
//                 of 2 x 128 K, contiguous in the tiled buffer) into a ring of record slots.
//   warp 1      : activation loader -- per 128-K step (one unit), two TMA boxes of BN rows x
//                 64 K into the step's slot of a ring (4-7 slots: the tiles come from L2, and a
//                 slot stays busy until its MMAs complete); owns the tensor memory.
//   warps 2, 3  : MMA issuers (two below BN = 128, one at 128) -- lane 0 of warp 2 + j takes the
//                 units j, j + 2, .. of the range:
//                 the eight tcgen05.mma (K = 16 each) of a step, operand A (the weights) from
//                 tensor memory and B (the activations) from shared memory, into issuer j's own
//                 accumulator of the tile, and one commit that frees the step's activation and
//                 weight tiles together; after a tile's last step a commit to the tile's barrier
//                 (one arrival per issuer). The epilogue adds the accumulators.
//   warps 4..7  : epilogue -- tcgen05.ld of the accumulator (warp w reads lanes 32 (w % 4) ..),
//                 then C (or the published partial sums of a cut tile); two accumulators, so one
//                 tile's epilogue runs under the next tile's MMAs.
//   warps 8..23 : dequantize -- thread (n, b) turns the 32 codes of channel n in 32-K block b
//                 of a unit into 16-bit weights (u - z) s (one rounding) and stores them with
//                 tcgen05.st into a ring of weight tiles in tensor memory (lane n = channel n, 64
//                 columns of K pairs per 128-K step); warp w writes the lanes 32 (w % 4) .. its
//                 channels occupy.
// Unit-scaled mode (BN = 16, group 128, where one group spans a unit): the dequant warps store
// u - z only (exact in 16 bits), each unit's MMAs go to a fresh accumulator (two per issuer), and
// the epilogue warps add s times the unit's sums into registers as each unit completes, saving the
// dequant warps the scale multiply (two instructions per register with bf16).
// Tensor memory (512 columns): two tiles in flight (one at BN = 256), each with one accumulator per
// issuer (BN columns), then the weight tiles of the step ring (64 columns per step). A has at
// most 256 rows per tile (one MMA of N = 256 per K step); more rows of A are more tiles (row
// blocks), whose weights are dequantized again but read from L2.
// Record slots are freed by the dequant warps, activation and weight-tile slots by the MMA
// commits, so the weight stream runs several units ahead of the tensor cores, and the shared
// memory holds only copies in flight (weight records and activation tiles).
// Every wait on an mbarrier or a tile counter is bounded; on expiry the kernel records
// W4A16_ETIMEOUT in dev_status, every role stops, the loaders wait for their copies in flight,
// the MMA thread waits for its last MMAs, and the CTA frees its tensor memory and returns.
#include <cudaTypedefs.h>

#include <mutex>
#include <type_traits>

#include "common.cuh"
#include "dequant.cuh"
#include "sm100_ptx.cuh"
#include "tiled_layout.cuh"

namespace w4a16 {

namespace {

using namespace sm100;

constexpr int kTcThreads = 768;
constexpr int kTcWarpLoadW = 0, kTcWarpLoadA = 1, kTcWarpMma = 2, kTcWarpEpi = 4, kTcWarpDeq = 8;
constexpr int kTcDeqWarps = 16;
// unit records per record slot (one bulk copy): two, one at BN = 256 (whose activation tiles take
// most of the shared memory)
__host__ __device__ constexpr int tc_units_per_load(int bn) { return bn >= 256 ? 1 : 2; }
constexpr int kTcSmemMax = 227 * 1024;
constexpr int kTcMaxRing = 16;
constexpr int kTcTmemCols = 512;
constexpr int kTcStepCols = 64;        // tensor-memory columns of one 128-K weight tile (K pairs)

// MMA threads: two below BN = 128 (issuer j takes the units j, j + 2, .. of the range; at small N
// one thread's issue rate, not the tensor pipe, sets the time), one from BN = 128. Tensor memory:
// two tiles in flight below BN = 256 (one tile's epilogue runs under the next tile's MMAs), one
// at 256, each with one accumulator per issuer (BN columns, at least 32), then the step ring's
// weight tiles: as many as fit, at most 8; at BN = 256 three (the shared memory holds three
// activation tiles of 64 KiB).
__host__ __device__ constexpr int tc_issuers(int bn) { return bn >= 128 ? 1 : 2; }
__host__ __device__ constexpr int tc_acc_bufs(int bn) { return bn >= 256 ? 1 : 2; }
__host__ __device__ constexpr int tc_acc_cols(int bn) { return bn < 32 ? 32 : bn; }
__host__ __device__ constexpr int tc_steps(int bn) {
    return bn >= 256 ? 3
                     : ((kTcTmemCols - 2 * tc_issuers(bn) * tc_acc_cols(bn)) / kTcStepCols > 8
                            ? 8
                            : (kTcTmemCols - 2 * tc_issuers(bn) * tc_acc_cols(bn)) / kTcStepCols);
}
constexpr uint64_t kTcDrainNs = 2000000000ull;

struct TcParams {
    const uint8_t* tiled;
    void* C;
    int* counters;      // one int per tile, zero between calls
    float* partials;    // [P][BN][128]: sums a CTA publishes for the tile that opens its range
    int* dev_status;
    int M, K, N, sym, group;
    uint32_t record, scales_off, zeros_off, slot_w;
    int P, mblocks, nr;
    uint32_t off_w, off_bar;   // shared-memory offsets; the activation tiles start at 0
    uint64_t wait_ns;
    GsMasks km;
};

__device__ __forceinline__ long long tc_unit_begin(int c, long long U, int P) { return ((long long)c * U) / P; }
__device__ __forceinline__ int tc_unit_owner(long long u, long long U, int P) {
    return (int)(((u + 1) * P - 1) / U);
}

__device__ __forceinline__ void tc_named_bar(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Warp-uniform bounded wait.
__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity, volatile int* abort, int* dev_status,
                                        uint64_t ns) {
    if (__all_sync(0xffffffffu, mbar_test_wait(bar, parity))) return true;
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, dev_status, ns));
}

// US (unit-scaled, run at BN = 16 with group 128): every unit's MMAs go to an accumulator of
// their own, the dequant warps store the exact integers u - z, and the epilogue warps add s times
// each unit's sums into registers (the unit's scale s of channel n read from its record).
// Otherwise the dequant warps store (u - z) s and the MMAs accumulate a whole tile segment.
template <int BN, typename T, bool US>
__global__ void __launch_bounds__(kTcThreads, 1)
tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const TcParams p) {
    static_assert(!US || BN <= 32, "unit-scaled accumulation keeps BN sums per thread in registers");
    using Ops = GsOps<T>;
    constexpr int kCols = tc_acc_cols(BN);       // tensor-memory columns of one accumulator
    constexpr int kIss = tc_issuers(BN);         // MMA threads
    constexpr int kBufs = tc_acc_bufs(BN);       // tiles in flight
    constexpr int kUPL = tc_units_per_load(BN);  // unit records per record slot
    constexpr int NS = tc_steps(BN);             // steps in flight (activation + weight tiles)
    constexpr uint32_t kSlotA = (uint32_t)BN * 256u;   // 128 K of BN rows: two 64-K TMA boxes
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned base, kept a shared-memory pointer (no integer round trip)
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int nr = p.nr;
    uint8_t* ring_a = smem;
    uint8_t* ring_w = smem + p.off_w;
    uint64_t* full_r = reinterpret_cast<uint64_t*>(smem + p.off_bar);
    uint64_t* empty_r = full_r + nr;
    uint64_t* full_a = empty_r + nr;     // [NS] the step's activation tile landed
    uint64_t* full_d = full_a + NS;      // [NS] the step's weight tile is in tensor memory
    uint64_t* free_s = full_d + NS;      // [NS] the step's MMAs completed: both tiles free
    constexpr int kAccBars = US ? 2 * kIss : 2;   // per tile buffer, or per accumulator (US)
    uint64_t* accfull = free_s + NS;              // [kAccBars]
    uint64_t* accempty = accfull + kAccBars;      // [kAccBars]
    uint64_t* lastmma = accempty + kAccBars;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(lastmma + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int UT = p.K / 128;                              // unit steps per tile
    const long long tiles = (long long)(p.N / 128) * p.mblocks;
    const long long U = tiles * UT;
    const int cta = blockIdx.x, P = p.P;
    const long long u0 = tc_unit_begin(cta, U, P), u1 = tc_unit_begin(cta + 1, U, P);
    const uint32_t R = p.record;
    const uint64_t wait_ns = p.wait_ns;

    if (threadIdx.x == 0) {
        for (int i = 0; i < nr; ++i) {
            mbar_init(&full_r[i], 1);
            mbar_init(&empty_r[i], kTcDeqWarps);
        }
        for (int i = 0; i < NS; ++i) {
            mbar_init(&full_a[i], 1);
            mbar_init(&full_d[i], kTcDeqWarps);
            mbar_init(&free_s[i], 1);
        }
        for (int i = 0; i < kAccBars; ++i) {
            mbar_init(&accfull[i], US ? 1 : kIss);
            mbar_init(&accempty[i], 4);
        }
        mbar_init(lastmma, kIss);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kTcWarpLoadA) {
        tmem_alloc(tmem_slot, kTcTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    cta_sync();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tmem_w = tmem + (uint32_t)(kBufs * kIss * kCols);   // the step ring's weight tiles

    if (warp == kTcWarpLoadW) {
        // ------------------------------------------------------------ weight records
        if (lane == 0) {
            int rs = 0, issued[kTcMaxRing];
            uint32_t rph = 0;
            for (int i = 0; i < nr; ++i) issued[i] = 0;
            // unit i = tile tau (channel tile nt, row block mb), step ku (kept by increments)
            const long long tau0 = u0 / UT;
            int ku = (int)(u0 - tau0 * UT), mb = (int)(tau0 % p.mblocks);
            long long nt = tau0 / p.mblocks;
            for (long long i = u0; i < u1;) {
                const int n = UT - ku < kUPL ? (u1 - i < UT - ku ? (int)(u1 - i) : UT - ku)
                                              : (u1 - i < kUPL ? (int)(u1 - i) : kUPL);
                if (!mbar_wait(&empty_r[rs], rph ^ 1u, abort_flag, p.dev_status, wait_ns)) break;
                const long long rec = nt * UT + ku;
                mbar_arrive_expect_tx(&full_r[rs], (uint32_t)n * R);
                bulk_g2s(ring_w + (size_t)rs * p.slot_w, p.tiled + (size_t)rec * R, (uint32_t)n * R, &full_r[rs]);
                ++issued[rs];
                i += n;
                if ((ku += n) == UT) {
                    ku = 0;
                    if (++mb == p.mblocks) {
                        mb = 0;
                        ++nt;
                    }
                }
                if (++rs == nr) {
                    rs = 0;
                    rph ^= 1u;
                }
            }
            // every copy issued lands before the CTA may exit
            volatile int keep = 0;
            for (int s = 0; s < nr; ++s)
                if (issued[s] > 0) mbar_wait(&full_r[s], (uint32_t)(issued[s] - 1) & 1u, &keep, nullptr, kTcDrainNs);
        }
    } else if (warp == kTcWarpLoadA) {
        // ------------------------------------------------------------ activation tiles
        if (lane == 0) {
            prefetch_tensormap(&tmA);
            int issued[8];
            for (int i = 0; i < NS; ++i) issued[i] = 0;
            int s = 0;
            uint32_t ph = 0;
            // unit i = tile tau, step ku; row block mb = tau mod mblocks (kept by increments)
            long long tau0 = u0 / UT;
            int ku = (int)(u0 - tau0 * UT), mb = (int)(tau0 % p.mblocks);
            for (long long i = u0; i < u1; ++i) {
                if (i > u0 && ++ku == UT) {
                    ku = 0;
                    if (++mb == p.mblocks) mb = 0;
                }
                if (!mbar_wait(&free_s[s], ph ^ 1u, abort_flag, p.dev_status, wait_ns)) break;
                mbar_arrive_expect_tx(&full_a[s], kSlotA);
                uint8_t* dst = ring_a + (size_t)s * kSlotA;
                tma_2d_g2s(dst, &tmA, ku * 128, mb * BN, &full_a[s]);
                tma_2d_g2s(dst + kSlotA / 2, &tmA, ku * 128 + 64, mb * BN, &full_a[s]);
                ++issued[s];
                if (++s == NS) {
                    s = 0;
                    ph ^= 1u;
                }
            }
            volatile int keep = 0;
            for (int q = 0; q < NS; ++q)
                if (issued[q] > 0) mbar_wait(&full_a[q], (uint32_t)(issued[q] - 1) & 1u, &keep, nullptr, kTcDrainNs);
        }
    } else if (warp >= kTcWarpMma && warp < kTcWarpMma + kIss) {
        // ------------------------------------------------------------ MMA issuers
        // Issuer j (lane 0 of warp kTcWarpMma + j) takes the units j, j + kIss, .. of the range into
        // its own accumulator of the tile; the epilogue adds them. (One thread issuing all the
        // MMAs measured about 1.1k cycles per unit at N = 16, the tensor pipe mostly idle.)
        if (lane == 0) {
            const int j = warp - kTcWarpMma;
            constexpr uint32_t idesc = idesc_f16(BN, std::is_same<T, __nv_bfloat16>::value);
            int s = 0, use[2] = {0, 0}, ab = 0;
            uint32_t ph = 0;
            bool ok = true;
            if constexpr (US) {
                // each own unit into accumulator ab * kIss + j (two per issuer, alternating)
                for (long long i = u0; i < u1; ++i) {
                    if (kIss == 1 || (int)((i - u0) & 1) == j) {
                        const int slot = ab * kIss + j;
                        if (!mbar_wait(&accempty[slot], ((uint32_t)use[ab] & 1u) ^ 1u, abort_flag, p.dev_status,
                                       wait_ns) ||
                            !mbar_wait(&full_d[s], ph, abort_flag, p.dev_status, wait_ns) ||
                            !mbar_wait(&full_a[s], ph, abort_flag, p.dev_status, wait_ns))
                            break;
                        tc_fence_after();
                        const uint32_t d_tmem = tmem + (uint32_t)(slot * kCols);
                        const uint32_t a_tm = tmem_w + (uint32_t)(s * kTcStepCols);
                        const uint32_t b_sm = smem_u32(ring_a + (size_t)s * kSlotA);
                        mma4_f16_ts(d_tmem, a_tm, smem_desc_sw128(b_sm), idesc, 0u);
                        mma4_f16_ts(d_tmem, a_tm + 32u, smem_desc_sw128(b_sm + kSlotA / 2), idesc, 1u);
                        mma_commit(&free_s[s]);
                        mma_commit(&accfull[slot]);
                        ++use[ab];
                        ab ^= 1;
                    }
                    if (++s == NS) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                ok = false;   // (the tile loop below is not run)
            }
            for (long long i = u0; i < u1 && ok;) {
                const long long tau = i / UT;
                const long long seg_end = u1 < (tau + 1) * UT ? u1 : (tau + 1) * UT;
                if (!mbar_wait(&accempty[ab], ((uint32_t)use[ab] & 1u) ^ 1u, abort_flag, p.dev_status, wait_ns)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)((ab * kIss + j) * kCols);
                bool first = true;
                for (; i < seg_end; ++i) {
                    if (kIss == 1 || (int)((i - u0) & 1) == j) {
                        if (!mbar_wait(&full_d[s], ph, abort_flag, p.dev_status, wait_ns) ||
                            !mbar_wait(&full_a[s], ph, abort_flag, p.dev_status, wait_ns)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        // the unit's eight K-steps of 16: weights from tensor memory, activations
                        // from the two 64-K boxes of the step's tile; one commit frees both tiles
                        const uint32_t a_tm = tmem_w + (uint32_t)(s * kTcStepCols);
                        const uint32_t b_sm = smem_u32(ring_a + (size_t)s * kSlotA);
                        mma4_f16_ts(d_tmem, a_tm, smem_desc_sw128(b_sm), idesc, first ? 0u : 1u);
                        mma4_f16_ts(d_tmem, a_tm + 32u, smem_desc_sw128(b_sm + kSlotA / 2), idesc, 1u);
                        mma_commit(&free_s[s]);
                        first = false;
                    }
                    if (++s == NS) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
                // (with no unit of this tile, the commit arrives at once)
                mma_commit(&accfull[ab]);
                ++use[ab];
                if (kBufs == 2) ab ^= 1;
            }
            // the CTA exits only after the last MMAs of every issuer completed
            mma_commit(lastmma);
            volatile int keep = 0;
            mbar_wait(lastmma, 0, &keep, nullptr, kTcDrainNs);
        }
    } else if (warp >= kTcWarpEpi && warp < kTcWarpEpi + 4) {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;                   // tensor-memory lane quarter
        const int n = 32 * q + lane;              // channel within the tile
        const bool leader = warp == kTcWarpEpi && lane == 0;
        T* C = static_cast<T*>(p.C);
        int use[2] = {0, 0}, ab = 0;
        bool ok = true;
        if constexpr (US) {
            // per unit: s times the unit's sums into run[] (row m0 + r of channel n); per tile
            // segment: run[] to C, or to the published sums of a cut tile
            float run[BN];
#pragma unroll
            for (int r = 0; r < BN; ++r) run[r] = 0.0f;
            int abj[2] = {0, 0}, uses[2 * kIss];
#pragma unroll
            for (int k = 0; k < 2 * kIss; ++k) uses[k] = 0;
            const uint16_t* scl = reinterpret_cast<const uint16_t*>(p.tiled + p.scales_off) + n;
            for (long long i = u0; i < u1;) {
                const long long tau = i / UT;
                const long long seg_end = u1 < (tau + 1) * UT ? u1 : (tau + 1) * UT;
                const int nt = (int)(tau / p.mblocks), mb = (int)(tau % p.mblocks);
                const size_t n0 = (size_t)nt * 128;
                const int m0 = mb * BN;
                const int cf = tc_unit_owner(tau * UT, U, P), cl = tc_unit_owner(tau * UT + UT - 1, U, P);
                for (; i < seg_end; ++i) {
                    const int j = kIss == 1 ? 0 : (int)((i - u0) & 1);
                    const int slot = abj[j] * kIss + j;
                    // the unit's record is nt K/128 + its K-step; its scale of channel n (group 128)
                    const long long rec = (long long)nt * UT + (i - tau * UT);
                    const uint16_t sb = __ldg(scl + (size_t)rec * (R / 2));
                    ok = ok && tc_wait(&accfull[slot], (uint32_t)uses[slot] & 1u, abort_flag, p.dev_status, wait_ns);
                    tc_fence_after();
                    if (ok) {
                        const float sf = __half2float(__ushort_as_half(sb));
                        const uint32_t lb = tmem + (uint32_t)(slot * kCols) + ((uint32_t)(32 * q) << 16);
#pragma unroll
                        for (int c = 0; c < BN / 16; ++c) {
                            uint32_t v[16];
                            tmem_ld16(lb + (uint32_t)(c * 16), v);
                            tmem_ld_wait();
#pragma unroll
                            for (int jj = 0; jj < 16; ++jj) run[c * 16 + jj] = fmaf(sf, __uint_as_float(v[jj]), run[c * 16 + jj]);
                        }
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&accempty[slot]);
                    ++uses[slot];
                    abj[j] ^= 1;
                }
                if (cf == cl || cta == cf) {
                    if (cf != cl) {
                        if (leader) {
                            const uint64_t t0 = globaltimer_ns();
                            for (;;) {
                                int c;
                                asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(c) : "l"(p.counters + tau)
                                             : "memory");
                                if (c >= cl - cf) break;
                                if (*abort_flag || globaltimer_ns() - t0 > wait_ns) {
                                    *abort_flag = 1;
                                    report_status(p.dev_status, W4A16_ETIMEOUT);
                                    break;
                                }
                            }
                            p.counters[tau] = 0;
                        }
                        tc_named_bar(1, 128);
                    }
                    if (ok && !*abort_flag) {
#pragma unroll
                        for (int c = 0; c < BN / 16; ++c) {
                            float y[16];
#pragma unroll
                            for (int jj = 0; jj < 16; ++jj) y[jj] = run[c * 16 + jj];
#pragma unroll 1
                            for (int cc = cf + 1; cc <= cl; ++cc) {
                                const float* part = p.partials + ((size_t)cc * BN + c * 16) * 128 + n;
                                float pv[16];
#pragma unroll
                                for (int jj = 0; jj < 16; ++jj)
                                    pv[jj] = m0 + c * 16 + jj < p.M ? __ldcg(part + jj * 128) : 0.0f;
#pragma unroll
                                for (int jj = 0; jj < 16; ++jj) y[jj] += pv[jj];
                            }
#pragma unroll
                            for (int jj = 0; jj < 16; ++jj) {
                                const int m = m0 + c * 16 + jj;
                                if (m < p.M) C[(size_t)m * p.N + n0 + n] = Act<T>::from_f32(y[jj]);
                            }
                        }
                    }
                } else {
                    if (ok && !*abort_flag) {
                        float* part = p.partials + (size_t)cta * BN * 128;
#pragma unroll
                        for (int r = 0; r < BN; ++r)
                            if (m0 + r < p.M) __stcg(part + (size_t)r * 128 + n, run[r]);
                    }
                    __threadfence();
                    tc_named_bar(1, 128);
                    if (leader) asm volatile("red.release.gpu.global.add.s32 [%0], 1;" ::"l"(p.counters + tau) : "memory");
                }
#pragma unroll
                for (int r = 0; r < BN; ++r) run[r] = 0.0f;
            }
            ok = false;   // (the tile loop below is not run)
        }
        for (long long i = u0; i < u1 && (!US || ok);) {
            const long long tau = i / UT;
            const long long seg_end = u1 < (tau + 1) * UT ? u1 : (tau + 1) * UT;
            // the issuers that hold units of this tile segment (issuer j: units j, j + 2, ..)
            const long long seg_lo = i;
            const bool has0 = kIss == 1 || seg_end - seg_lo >= 2 || ((seg_lo - u0) & 1) == 0;
            const bool has1 = kIss == 2 && (seg_end - seg_lo >= 2 || ((seg_lo - u0) & 1) == 1);
            ok = ok && tc_wait(&accfull[ab], (uint32_t)use[ab] & 1u, abort_flag, p.dev_status, wait_ns);
            tc_fence_after();
            const int nt = (int)(tau / p.mblocks), mb = (int)(tau % p.mblocks);
            const size_t n0 = (size_t)nt * 128;
            const int m0 = mb * BN;
            const int cf = tc_unit_owner(tau * UT, U, P), cl = tc_unit_owner(tau * UT + UT - 1, U, P);
            i = seg_end;
            const uint32_t lane_base = tmem + (uint32_t)(ab * kIss * kCols) + ((uint32_t)(32 * q) << 16);
            // the tile's FP32 sums, 16 columns from c: the issuers' accumulators added
            auto acc16 = [&](int c, float (&y)[16]) {
                uint32_t v[16];
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) y[jj] = 0.0f;
                if (has0) {
                    tmem_ld16(lane_base + (uint32_t)(c * 16), v);
                    tmem_ld_wait();
#pragma unroll
                    for (int jj = 0; jj < 16; ++jj) y[jj] = __uint_as_float(v[jj]);
                }
                if (has1) {
                    tmem_ld16(lane_base + (uint32_t)(kCols + c * 16), v);
                    tmem_ld_wait();
#pragma unroll
                    for (int jj = 0; jj < 16; ++jj) y[jj] += __uint_as_float(v[jj]);
                }
            };
            if (cf == cl || cta == cf) {
                if (cf != cl) {
                    // the tile is cut between CTAs cf .. cl and this is cf: wait until every later
                    // CTA of the tile has published its sums (the tile opens their ranges)
                    if (leader) {
                        const uint64_t t0 = globaltimer_ns();
                        for (;;) {
                            int c;
                            asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(c) : "l"(p.counters + tau)
                                         : "memory");
                            if (c >= cl - cf) break;
                            if (*abort_flag || globaltimer_ns() - t0 > wait_ns) {
                                *abort_flag = 1;
                                report_status(p.dev_status, W4A16_ETIMEOUT);
                                break;
                            }
                        }
                        p.counters[tau] = 0;
                    }
                    tc_named_bar(1, 128);
                }
                if (ok && !*abort_flag) {
#pragma unroll 1
                    for (int c = 0; c < BN / 16; ++c) {
                        float y[16];
                        acc16(c, y);
                        // the other CTAs' sums, in CTA order; the 16 loads of one CTA in flight together
#pragma unroll 1
                        for (int cc = cf + 1; cc <= cl; ++cc) {
                            const float* part = p.partials + ((size_t)cc * BN + c * 16) * 128 + n;
                            float pv[16];
#pragma unroll
                            for (int j = 0; j < 16; ++j) pv[j] = m0 + c * 16 + j < p.M ? __ldcg(part + j * 128) : 0.0f;
#pragma unroll
                            for (int j = 0; j < 16; ++j) y[j] += pv[j];
                        }
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const int m = m0 + c * 16 + j;
                            if (m < p.M) C[(size_t)m * p.N + n0 + n] = Act<T>::from_f32(y[j]);
                        }
                    }
                }
            } else {
                // a later CTA of a cut tile (the tile opens its range): publish the sums and count
                // them, without waiting
                if (ok && !*abort_flag) {
                    float* part = p.partials + (size_t)cta * BN * 128;
#pragma unroll 1
                    for (int c = 0; c < BN / 16; ++c) {
                        float y[16];
                        acc16(c, y);
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const int mr = c * 16 + j;
                            if (m0 + mr < p.M) __stcg(part + (size_t)mr * 128 + n, y[j]);
                        }
                    }
                }
                __threadfence();
                tc_named_bar(1, 128);
                if (leader) asm volatile("red.release.gpu.global.add.s32 [%0], 1;" ::"l"(p.counters + tau) : "memory");
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&accempty[ab]);
            ++use[ab];
            if (kBufs == 2) ab ^= 1;
        }
    } else if (warp >= kTcWarpDeq) {
        // ------------------------------------------------------------ dequantize
        const int dt = threadIdx.x - 32 * kTcWarpDeq;
        const int n = dt & 127, blk = dt >> 7;   // channel, and the unit's 32-K block (0..3)
        const int sym = p.sym;
        const GsMasks km = p.km;
        const int lg = (32 * blk) / p.group;     // the block's group within the unit
        const uint32_t coff = 2048u * (uint32_t)blk + 16u * (uint32_t)(n ^ (2 * blk));
        const uint32_t soff = p.scales_off + 256u * (uint32_t)lg + 2u * (uint32_t)n;
        const uint32_t zoff = p.zeros_off + 64u * (uint32_t)lg + 4u * (uint32_t)(n >> 3);
        const int zsh = 4 * (n & 7);
        // this warp's lanes of tensor memory (its 32 channels), columns [16 blk, 16 blk + 16) of the
        // step's tile
        const uint32_t d_lane = tmem_w + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)(16 * blk);
        int rs = 0, s = 0;
        uint32_t rph = 0, ph = 0;
        bool ok = true;
        long long tend = (u0 / UT + 1) * UT;   // end of the current tile's units
        for (long long i = u0; i < u1 && ok;) {
            const long long seg_end = u1 < tend ? u1 : tend;
            const int nu = (int)(seg_end - i < kUPL ? seg_end - i : kUPL);
            i += nu;
            if (i == tend) tend += UT;
            if (!tc_wait(&full_r[rs], rph, abort_flag, p.dev_status, wait_ns)) {
                ok = false;
                break;
            }
            for (int uu = 0; uu < nu; ++uu) {
                const uint8_t* rec = ring_w + (size_t)rs * p.slot_w + (size_t)uu * R;
                const uint4 cw = *reinterpret_cast<const uint4*>(rec + coff);
                const uint16_t sb = US ? (uint16_t)0 : *reinterpret_cast<const uint16_t*>(rec + soff);
                const uint32_t zv = sym ? 8u : (*reinterpret_cast<const uint32_t*>(rec + zoff) >> zsh) & 0xFu;
                if (!tc_wait(&free_s[s], ph ^ 1u, abort_flag, p.dev_status, wait_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();   // the MMAs that read this tile completed before the stores
                const uint32_t za = Ops::zz_a(zv), zb = Ops::zz_b(zv);
                typename Ops::Scale sc;
                if constexpr (!US) sc.set(sb);
                const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
                uint32_t out[16];   // column c: K pair (2 c, 2 c + 1) of the block
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    uint32_t r[4];
                    Ops::unpack(words[w], km, r);
                    if constexpr (US) {   // u - z, exact; the scale multiplies the unit's sums
                        out[4 * w + 0] = Ops::sub_a(r[0], za);
                        out[4 * w + 1] = Ops::sub_b(r[1], zb);
                        out[4 * w + 2] = Ops::sub_a(r[2], za);
                        out[4 * w + 3] = Ops::sub_b(r[3], zb);
                    } else {
                        out[4 * w + 0] = sc.apply(Ops::sub_a(r[0], za));
                        out[4 * w + 1] = sc.apply(Ops::sub_b(r[1], zb));
                        out[4 * w + 2] = sc.apply(Ops::sub_a(r[2], za));
                        out[4 * w + 3] = sc.apply(Ops::sub_b(r[3], zb));
                    }
                }
                tmem_st16(d_lane + (uint32_t)(s * kTcStepCols), out);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&full_d[s]);
                if (++s == NS) {
                    s = 0;
                    ph ^= 1u;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty_r[rs]);
            if (++rs == nr) {
                rs = 0;
                rph ^= 1u;
            }
        }
    }

    tc_fence_before();
    cta_sync();
    if (warp == kTcWarpLoadA) {
        tc_fence_after();
        tmem_dealloc(tmem, kTcTmemCols);
    }
}

}  // namespace

// ------------------------------------------------------------------------------ host side
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* q = nullptr;
        cudaDriverEntryPointQueryResult r;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &q, cudaEnableDefault, &r) == cudaSuccess &&
            r == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(q);
    });
    return fn;
}

// Activations A [M, K] (16-bit, row-major) as a 2-D tensor map: box 64 (K) x box_rows,
// 128-byte swizzle; rows past M read as zero.
bool make_act_map(CUtensorMap* map, const void* A, int M, int K, int box_rows, bool bf16) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
    cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                    const_cast<void*>(A), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// An 8-bit matrix [rows, K] (row-major, K bytes per row) as a 2-D tensor map: box 128 (K) x
// box_rows, 128-byte swizzle; rows past the end read as zero.
bool make_u8_map(CUtensorMap* map, const void* base, int rows, int K, int box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)K};
    cuuint32_t box[2] = {128, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int tc_block_rows(int M) {
    if (M <= 16) return 16;
    if (M <= 32) return 32;
    if (M <= 64) return 64;
    if (M <= 128) return 128;
    return 256;   // more rows: blocks of 256 (one accumulator of 256 columns in TMEM, one MMA of
                  // N = 256 per K step, each weight unit dequantized once per 256 rows)
}

TcPlan plan_gemm_tc(int M, int N, int K, int group, int sym, int n_sm) {
    TcPlan pl = {};
    if (M < 1 || K % 128 != 0 || N % 128 != 0 || K < 128 || N < 128 || n_sm <= 0) return pl;
    const TiledLayout L = tiled_layout(K, N, group, sym);
    pl.bn = tc_block_rows(M);
    pl.mblocks = (M + pl.bn - 1) / pl.bn;
    const long long tiles = (long long)(N / 128) * pl.mblocks;
    if (tiles > kGemvStreamMaxTiles) return pl;
    const long long units = tiles * (K / 128);
    pl.ctas = (int)(units < n_sm ? units : n_sm);
    pl.slot_w = (uint32_t)((tc_units_per_load(pl.bn) * L.record + 127) & ~127u);
    pl.nd = tc_steps(pl.bn);   // steps in flight: activation tiles in shared memory, weights in TMEM
    pl.na = pl.nd;
    const uint32_t slot_a = (uint32_t)pl.bn * 256u;
    const size_t bars = 1024;   // barriers, tensor-memory slot, abort flag
    const size_t avail = (size_t)kTcSmemMax - 1024 /* alignment */ - bars;
    if ((size_t)pl.na * slot_a + 2 * (size_t)pl.slot_w > avail) return TcPlan{};
    size_t nr = (avail - (size_t)pl.na * slot_a) / pl.slot_w;
    if (nr > kTcMaxRing) nr = kTcMaxRing;
    pl.nr = (int)nr;
    pl.off_a = 0;
    pl.off_w = (uint32_t)pl.na * slot_a;
    pl.off_bar = pl.off_w + (uint32_t)pl.nr * pl.slot_w;
    pl.off_bar = (pl.off_bar + 127u) & ~127u;
    pl.smem = 1024 + pl.off_bar + bars;
    pl.partial_bytes = (size_t)pl.ctas * pl.bn * 128 * sizeof(float);
    pl.ok = pl.smem <= (size_t)kTcSmemMax;
    return pl;
}

namespace {

template <int BN, typename T, bool US>
int launch_tc_typed(const CUtensorMap& map, const TcParams& prm, size_t smem, cudaStream_t stream) {
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(tc_gemm_kernel<BN, T, US>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        kTcSmemMax);
    });
    if (attr_err != cudaSuccess) return W4A16_ECUDA;
    tc_gemm_kernel<BN, T, US><<<prm.P, kTcThreads, smem, stream>>>(map, prm);
    return launch_status();
}

template <typename T>
int launch_tc_bn(int bn, const CUtensorMap& map, const TcParams& prm, size_t smem, cudaStream_t stream) {
    switch (bn) {
        // unit-scaled accumulation where one group spans a unit, at BN = 16 (measured on the
        // (8192, 28672) layer: 71.2 -> 67.8 us at M = 16; at BN = 32 it was slower, 74.4 -> 76.6)
        case 16: return prm.group == 128 ? launch_tc_typed<16, T, true>(map, prm, smem, stream)
                                         : launch_tc_typed<16, T, false>(map, prm, smem, stream);
        case 32: return launch_tc_typed<32, T, false>(map, prm, smem, stream);
        case 64: return launch_tc_typed<64, T, false>(map, prm, smem, stream);
        case 128: return launch_tc_typed<128, T, false>(map, prm, smem, stream);
        case 256: return launch_tc_typed<256, T, false>(map, prm, smem, stream);
        default: return W4A16_EUNSUPPORTED;
    }
}

}  // namespace

int launch_gemm_tc(const void* A, int a_dtype, int M, int K, const void* tiled, int N, int group, int sym,
                   void* C, void* workspace, int* dev_status, cudaStream_t stream) {
    const TcPlan pl = plan_gemm_tc(M, N, K, group, sym, gemv_stream_sm_count());
    if (!pl.ok) return W4A16_EUNSUPPORTED;
    if (!workspace) return W4A16_EWORKSPACE;
    const bool bf16 = a_dtype == W4A16_BF16;
    CUtensorMap map;
    if (!make_act_map(&map, A, M, K, pl.bn, bf16)) return W4A16_ECUDA;
    const TiledLayout L = tiled_layout(K, N, group, sym);
    TcParams prm = {};
    prm.tiled = static_cast<const uint8_t*>(tiled);
    prm.C = C;
    prm.counters = static_cast<int*>(workspace);
    prm.partials = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kGemvStreamCounterBytes);
    prm.dev_status = dev_status;
    prm.M = M;
    prm.K = K;
    prm.N = N;
    prm.sym = sym;
    prm.group = group;
    prm.record = L.record;
    prm.scales_off = L.scales;
    prm.zeros_off = L.zeros;
    prm.slot_w = pl.slot_w;
    prm.P = pl.ctas;
    prm.mblocks = pl.mblocks;
    prm.nr = pl.nr;
    prm.off_w = pl.off_w;
    prm.off_bar = pl.off_bar;
    prm.wait_ns = wait_limit_ns();
    prm.km.lo = 0x000F000Fu;
    prm.km.hi = bf16 ? 0x000F000Fu : 0x00F000F0u;
    prm.km.magic = bf16 ? 0x43004300u : 0x64006400u;
    prm.km.m4 = 1u << 28;
    prm.km.m8 = 1u << 24;
    prm.km.m12 = 1u << 20;
    if (bf16) return launch_tc_bn<__nv_bfloat16>(pl.bn, map, prm, pl.smem, stream);
    return launch_tc_bn<__half>(pl.bn, map, prm, pl.smem, stream);
}

}  // namespace w4a16
