// gemm_tc.cu -- tcgen05 tensor-core W4A16 GEMM for sm_100a (the larger-M path).
//
// C[M, N] = A[M, K] . dequant(W)[K, N], FP32 accumulation in tensor memory.
// "4.3 Weight-only INT4", section 4: read, unpack, dequantize and multiply in one pipeline, each
// weight byte crossing HBM once, data movement overlapped with on-chip compute; section 1: codes
// dequantized on chip to FP16/BF16, multiply inputs stay 16-bit.
//
// Mapping. The MMA computes D[n, m] = sum_k W^T[n, k] A^T[k, m] (swap-AB): the dequantized weight
// tile (128 output channels x 64 K) is operand A (M_mma = 128), the activation tile
// (BN rows of A x 64 K) is operand B (N_mma = BN), D (128 x BN, FP32) lives in tensor memory,
// lane = output channel, column = row of A. One CTA computes one 128-channel x BN-row tile over
// the whole K range.
//
// Warp roles (192 threads):
//   warp 0      : one thread issues, per 64-K stage, a TMA tile load of the activations
//                 (128-byte swizzle), a bulk copy of the stage's 4 KiB of codes (half of a unit
//                 record of the tiled buffer), and bulk copies of the stage's scales and zeros
//                 from the same record.
//   warp 1      : allocates tensor memory; one thread issues the four tcgen05.mma of a stage
//                 and commits them to the stage's "empty" barrier.
//   warps 2..5  : dequantize -- one thread per output channel turns its 64 codes of the stage
//                 into 16-bit weights w = (u - z) * s (one rounding) and writes them into the
//                 stage's A tile in the 128-byte-swizzled K-major layout; after the last stage
//                 they read D back (tcgen05.ld) and store C.
// Every wait on an mbarrier is bounded; on expiry the kernel records W4A16_ETIMEOUT in
// dev_status and every role drains and returns, freeing its tensor memory.
#include <cudaTypedefs.h>

#include <mutex>
#include <type_traits>

#include "common.cuh"
#include "sm100_ptx.cuh"
#include "tiled_layout.cuh"

namespace w4a16 {

namespace {

using namespace sm100;

constexpr int kThreadsTC = 320;  // producer, MMA, 8 dequant/epilogue warps
constexpr uint64_t kSpin = 2000000000ull;  // a wait gives up after 2 s (nanoseconds)

template <int BN>
struct TcCfg {
    static constexpr int kA = 128 * 128;           // dequantized weight tile: 128 rows x 128 B
    static constexpr int kB = BN * 128;            // activation tile: BN rows x 128 B
    static constexpr int kCodes = 4096;            // one tiled code tile
    static constexpr int kScales = 2 * 256;        // up to two groups (group 32) x 128 fp16
    static constexpr int kZeros = 2 * 64;          // up to two groups x 16 words
    static constexpr int kStage = ((kA + kB + kCodes + kScales + kZeros + 1023) / 1024) * 1024;
    static constexpr int kBudget = 227 * 1024 - 1024 - 256;  // alignment slack and barriers
    static constexpr int kStagesRaw = kBudget / kStage;
    static constexpr int kStages = kStagesRaw > 8 ? 8 : kStagesRaw;
    static constexpr int kTmemCols = BN < 32 ? 32 : BN;
    static constexpr int kSmem = kStages * kStage + 1024 + 256;
    static_assert(kStages >= 2, "pipeline needs two stages");
};

template <typename T>
struct Deq;

// fp16: (1024 + u) - (1024 + z) is exact, one rounding in the product with s.
template <>
struct Deq<__half> {
    static constexpr uint32_t kMagic = 0x64006400u;
    __half2 zz, s2;
    __device__ __forceinline__ void set(float s, int z) {
        zz = __half2half2(__ushort_as_half((unsigned short)(0x6400 + z)));
        s2 = __float2half2_rn(s);  // s is an fp16 value: exact
    }
    __device__ __forceinline__ uint32_t pair(uint32_t x) const {
        __half2 h = *reinterpret_cast<__half2*>(&x);
        __half2 r = __hmul2(__hsub2(h, zz), s2);
        return *reinterpret_cast<uint32_t*>(&r);
    }
};

// bf16: d = (128 + u) - (128 + z) is exact; s = s_hi + s_lo with s_hi = s truncated to bf16 and
// s_lo (at most 3 significant bits) exact in bf16; d * s_lo is exact, and
// fma(d, s_hi, d * s_lo) rounds d * s once.
template <>
struct Deq<__nv_bfloat16> {
    static constexpr uint32_t kMagic = 0x43004300u;
    __nv_bfloat162 zz, shi, slo;
    __device__ __forceinline__ void set(float s, int z) {
        zz = __bfloat162bfloat162(__ushort_as_bfloat16((unsigned short)(0x4300 + z)));
        const uint32_t sb = __float_as_uint(s) & 0xFFFF0000u;
        const float hi = __uint_as_float(sb);
        const float lo = s - hi;  // exact
        shi = __bfloat162bfloat162(__ushort_as_bfloat16((unsigned short)(sb >> 16)));
        slo = __float2bfloat162_rn(lo);  // exact
    }
    __device__ __forceinline__ uint32_t pair(uint32_t x) const {
        __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&x);
        __nv_bfloat162 d = __hsub2(h, zz);
        __nv_bfloat162 t = __hmul2(d, slo);
        __nv_bfloat162 r = __hfma2(d, shi, t);
        return *reinterpret_cast<uint32_t*>(&r);
    }
};

template <int BN, typename T>
__global__ void __launch_bounds__(kThreadsTC, 1)
tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const uint8_t* __restrict__ tiled, int M, int K,
               int N, int group, int sym, const TiledLayout L, T* __restrict__ C, int* dev_status) {
    using Cfg = TcCfg<BN>;
    constexpr int NS = Cfg::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + NS * Cfg::kStage);
    uint64_t* afull = full + NS;
    uint64_t* empty = afull + NS;
    uint64_t* accfull = empty + NS;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accfull + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nt = blockIdx.x;
    const int n0 = nt * 128;
    const int m0 = blockIdx.y * BN;
    const int kstages = K / 64;
    const int groups_per_stage = group >= 64 ? 1 : 64 / group;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&afull[s], 256);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accfull, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, Cfg::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_d = *tmem_slot;

    if (warp == 0) {
        // ---------------------------------------------------------------- producer
        if (lane == 0) {
            prefetch_tensormap(&tmA);
            const uint32_t stage_bytes = (uint32_t)Cfg::kB + (uint32_t)Cfg::kCodes +
                                         (uint32_t)groups_per_stage * (256u + (sym ? 0u : 64u));
            int issued = 0;
            for (int it = 0; it < kstages; ++it) {
                const int s = it % NS;
                const uint32_t r = (uint32_t)(it / NS);
                if (!mbar_wait(&empty[s], (r & 1u) ^ 1u, abort_flag, dev_status, kSpin)) break;
                uint8_t* st = smem + s * Cfg::kStage;
                mbar_arrive_expect_tx(&full[s], stage_bytes);
                tma_2d_g2s(st + Cfg::kA, &tmA, it * 64, m0, &full[s]);
                // unit record (nt, it / 2): blocks 2 (it % 2), 2 (it % 2) + 1 of its codes, and
                // the record's groups that fall in this stage (contiguous in the record)
                const uint8_t* rec = tiled + ((size_t)nt * (K / 128) + it / 2) * L.record;
                bulk_g2s(st + Cfg::kA + Cfg::kB, rec + (it & 1) * 4096, 4096, &full[s]);
                const int lg0 = (it * 64) / group - (it / 2) * L.groups;
                bulk_g2s(st + Cfg::kA + Cfg::kB + Cfg::kCodes, rec + L.scales + lg0 * 256, groups_per_stage * 256,
                         &full[s]);
                if (!sym)
                    bulk_g2s(st + Cfg::kA + Cfg::kB + Cfg::kCodes + Cfg::kScales, rec + L.zeros + lg0 * 64,
                             groups_per_stage * 64, &full[s]);
                ++issued;
            }
            // drain: every copy issued has landed before the block may exit
            for (int it = (issued > NS ? issued - NS : 0); it < issued; ++it) {
                const int s = it % NS;
                mbar_wait(&full[s], (uint32_t)(it / NS) & 1u, abort_flag, dev_status, kSpin);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_f16(BN, sizeof(T) == 2 && !std::is_same<T, __half>::value);
            int done = 0;
            for (int it = 0; it < kstages; ++it) {
                const int s = it % NS;
                const uint32_t r = (uint32_t)(it / NS);
                if (!mbar_wait(&full[s], r & 1u, abort_flag, dev_status, kSpin)) break;
                if (!mbar_wait(&afull[s], r & 1u, abort_flag, dev_status, kSpin)) break;
                tc_fence_after();
                const uint32_t a_base = smem_u32(smem + s * Cfg::kStage);
                const uint32_t b_base = a_base + Cfg::kA;
                // the stage's four K-steps of 16 and the commit that frees the stage
                mma4_f16_ss_commit(tmem_d, smem_desc_sw128(a_base), smem_desc_sw128(b_base), idesc,
                                   it > 0 ? 1u : 0u, &empty[s]);
                ++done;
            }
            mma_commit(accfull);  // also completes when nothing was issued
            (void)done;
        }
    } else {
        // ---------------------------------------------------------------- dequant + epilogue
        // two warps per TMEM lane quarter: warp half hf dequantizes rows 4 hf .. 4 hf + 3 of the
        // stage's code tile (K 32 hf .. 32 hf + 31) and stores columns [BN/2 hf, BN/2 (hf + 1)) of C
        const int q = warp & 3;           // tensor-memory lane quarter this warp may access
        const int hf = (warp - 2) >> 2;   // 0 for warps 2..5, 1 for warps 6..9
        const int n = 32 * q + lane;      // output channel within the tile = TMEM lane
        Deq<T> dq;
        bool ok = true;
        for (int it = 0; it < kstages && ok; ++it) {
            const int s = it % NS;
            const uint32_t r = (uint32_t)(it / NS);
            ok = mbar_wait(&empty[s], (r & 1u) ^ 1u, abort_flag, dev_status, kSpin) &&
                 mbar_wait(&full[s], r & 1u, abort_flag, dev_status, kSpin);
            if (!ok) break;
            uint8_t* st = smem + s * Cfg::kStage;
            const uint4* ctile = reinterpret_cast<const uint4*>(st + Cfg::kA + Cfg::kB);
            const __half* ssm = reinterpret_cast<const __half*>(st + Cfg::kA + Cfg::kB + Cfg::kCodes);
            const uint32_t* zsm = reinterpret_cast<const uint32_t*>(st + Cfg::kA + Cfg::kB + Cfg::kCodes + Cfg::kScales);
            uint8_t* atile = st;
            // rows 4 hf .. 4 hf + 3 of the stage: block h = 2 (it % 2) + hf of the unit record,
            // channel n in slot n ^ 2h
            const uint4 w4 = ctile[128 * hf + (n ^ (2 * (2 * (it & 1) + hf)))];
            const uint32_t words[4] = {w4.x, w4.y, w4.z, w4.w};
            // group of this half inside the stage (group 32: one group per half)
            const int lg = groups_per_stage > 1 ? hf : 0;
            const float sv = __half2float(ssm[lg * 128 + n]);
            const int zv = sym ? 8 : (int)((zsm[lg * 16 + n / 8] >> (4 * (n % 8))) & 0xFu);
            dq.set(sv, zv);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int jl = 4 * hf + i;
                const uint32_t w = words[i];
                uint4 out;
                out.x = dq.pair((w & 0x000F000Fu) | Deq<T>::kMagic);
                out.y = dq.pair(((w >> 4) & 0x000F000Fu) | Deq<T>::kMagic);
                out.z = dq.pair(((w >> 8) & 0x000F000Fu) | Deq<T>::kMagic);
                out.w = dq.pair(((w >> 12) & 0x000F000Fu) | Deq<T>::kMagic);
                const int row = n;
                const uint32_t off = (uint32_t)((row >> 3) * 1024 + (row & 7) * 128 + ((jl ^ (row & 7)) << 4));
                *reinterpret_cast<uint4*>(atile + off) = out;
            }
            fence_proxy_async_smem();
            mbar_arrive(&afull[s]);
        }
        // epilogue: D (lane n, columns 0..BN-1) -> C[m0 + m, n0 + n]; this warp stores half the columns
        if (mbar_wait(accfull, 0, abort_flag, dev_status, kSpin) && ok && !*abort_flag) {
            tc_fence_after();
            const uint32_t lane_base = tmem_d + ((uint32_t)(32 * q) << 16);
            constexpr int kChunks = BN / 16;
            const int c0 = kChunks > 1 ? hf * (kChunks / 2) : 0;
            const int c1 = kChunks > 1 ? c0 + kChunks / 2 : (hf == 0 ? 1 : 0);
#pragma unroll 1
            for (int c = c0; c < c1; ++c) {
                uint32_t v[16];
                tmem_ld16(lane_base + c * 16, v);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int m = m0 + c * 16 + i;
                    if (m < M) C[(size_t)m * N + n0 + n] = Act<T>::from_f32(__uint_as_float(v[i]));
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_d, Cfg::kTmemCols);
    }
}

}  // namespace

// ------------------------------------------------------------------------------ host side
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// Activations A [M, K] (16-bit, row-major) as a 2-D tensor map: box 64 (K) x BN (rows),
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

namespace {

template <int BN, typename T>
int launch_tc_typed(const void* A, int M, int K, const void* tiled, int N, int group, int sym, void* C,
                    int* dev_status, cudaStream_t stream) {
    using Cfg = TcCfg<BN>;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(tc_gemm_kernel<BN, T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        Cfg::kSmem);
    });
    if (attr_err != cudaSuccess) return W4A16_ECUDA;
    CUtensorMap map;
    if (!make_act_map(&map, A, M, K, BN, !std::is_same<T, __half>::value)) return W4A16_ECUDA;
    const TiledLayout L = tiled_layout(K, N, group, sym);
    dim3 grid(N / 128, (M + BN - 1) / BN);
    tc_gemm_kernel<BN, T><<<grid, kThreadsTC, Cfg::kSmem, stream>>>(
        map, static_cast<const uint8_t*>(tiled), M, K, N, group, sym, L, static_cast<T*>(C), dev_status);
    return launch_status();
}

template <typename T>
int launch_tc_bn(const void* A, int M, int K, const void* tiled, int N, int group, int sym, void* C,
                 int* dev_status, cudaStream_t stream) {
    if (M <= 16) return launch_tc_typed<16, T>(A, M, K, tiled, N, group, sym, C, dev_status, stream);
    if (M <= 32) return launch_tc_typed<32, T>(A, M, K, tiled, N, group, sym, C, dev_status, stream);
    if (M <= 64) return launch_tc_typed<64, T>(A, M, K, tiled, N, group, sym, C, dev_status, stream);
    if (M <= 128) return launch_tc_typed<128, T>(A, M, K, tiled, N, group, sym, C, dev_status, stream);
    return launch_tc_typed<256, T>(A, M, K, tiled, N, group, sym, C, dev_status, stream);
}

}  // namespace

int launch_gemm_tc(const void* A, int a_dtype, int M, int K, const void* tiled, int N, int group, int sym,
                   void* C, int* dev_status, cudaStream_t stream) {
    if (a_dtype == W4A16_BF16)
        return launch_tc_bn<__nv_bfloat16>(A, M, K, tiled, N, group, sym, C, dev_status, stream);
    return launch_tc_bn<__half>(A, M, K, tiled, N, group, sym, C, dev_status, stream);
}

}  // namespace w4a16
