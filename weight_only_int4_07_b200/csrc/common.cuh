// common.cuh -- shared device/host helpers of the W4A16 CUDA library (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "w4a16.h"

namespace w4a16 {

// 16-bit activation types and their conversions to/from FP32.
template <typename T>
struct Act;

template <>
struct Act<__half> {
    static __device__ __forceinline__ float to_f32(__half x) { return __half2float(x); }
    static __device__ __forceinline__ __half from_f32(float x) { return __float2half_rn(x); }
};

template <>
struct Act<__nv_bfloat16> {
    static __device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
    static __device__ __forceinline__ __nv_bfloat16 from_f32(float x) { return __float2bfloat16_rn(x); }
};

// First device-side error wins; the caller zeroes the status word.
__device__ __forceinline__ void report_status(int* dev_status, int code) {
    if (dev_status) atomicCAS(dev_status, 0, code);
}

// Nibble i of a packed word as an unsigned code 0..15.
__device__ __forceinline__ int nibble_u(uint32_t w, int i) { return (int)((w >> (4 * i)) & 0xFu); }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline int launch_status() {
    return cudaGetLastError() == cudaSuccess ? W4A16_OK : W4A16_ECUDA;
}

// ---------------------------------------------------------------------------------------------
// Kernel entry points implemented in the .cu files (host-side launchers).
// ---------------------------------------------------------------------------------------------
int launch_quantize(const void* W, int K, int N, int group, int sym, int32_t* codes, void* scales,
                    int32_t* zeros, int* dev_status, cudaStream_t stream);

// H = 2 X^T X in FP64 for 16-bit X [S, K] (the curvature of the layer-output error).
void launch_hessian(const void* X, int x_dtype, int S, int K, double* H, cudaStream_t stream);
size_t gptq_workspace_bytes(int K, int N);
size_t awq_workspace_bytes(int K, int N, int S);
int launch_fp8_quantize_weights(const void* W, int K, int N, uint8_t* Wq, float* sw, cudaStream_t stream);
int launch_fp8_quantize_acts(const void* A, int a_dtype, int M, int K, uint8_t* Aq, float* sa, cudaStream_t stream);
int launch_fp8_gemm(const uint8_t* Aq, const float* sa, int M, int K, const uint8_t* Wq, const float* sw, int N,
                    void* C, int c_dtype, int* dev_status, cudaStream_t stream);
int launch_awq(const void* W, const void* X, int x_dtype, int S, int K, int N, int group, int sym, int32_t* codes,
               void* scales, int32_t* zeros, void* s_in, void* workspace, int* dev_status, cudaStream_t stream);
int launch_gptq(const void* W, const void* X, int x_dtype, int S, int K, int N, int group, int sym, double damp,
                int32_t* codes, void* scales, int32_t* zeros, void* workspace, int* dev_status,
                cudaStream_t stream);

int launch_dequantize(const int32_t* codes, const void* scales, const int32_t* zeros, int K, int N, int group,
                      int sym, int out_dtype, void* W, cudaStream_t stream);

int launch_repack(const int32_t* codes, const void* scales, const int32_t* zeros, int K, int N,
                  int group, int sym, void* tiled, cudaStream_t stream);

// Split-K GEMV plan: how the K dimension is cut and how much workspace that needs.
struct GemvPlan {
    int mt;              // rows of A per launch (template width), >= rows handled
    int splits;          // K splits (grid.y)
    int rows_per_split;  // packed rows (8 k each) per split
    size_t ws_bytes;     // workspace for the partial sums of one launch
};
GemvPlan plan_gemv_plain(int M, int N, int K, int group);

int launch_gemv_plain(const void* A, int a_dtype, int M, int K, const int32_t* codes,
                      const void* scales, const int32_t* zeros, int N, int group, int sym, void* C,
                      void* workspace, const GemvPlan& plan, cudaStream_t stream);


// Persistent stream-K decode kernel. Its workspace starts with one int counter per 128-channel
// tile (kGemvStreamCounterBytes, zero between calls; each call leaves them zero), followed by
// the FP32 partial sums of tiles cut between CTAs.
constexpr size_t kGemvStreamCounterBytes = 64 * 1024;
constexpr int kGemvStreamMaxTiles = (int)(kGemvStreamCounterBytes / 4);
struct GemvStreamPlan {
    bool ok;
    int ns;               // pipeline stages
    int ctas;             // persistent CTAs of each slice (one per SM in all)
    size_t row_bytes, act_bytes, red_bytes, sa_bytes, stage_bytes, smem;
    size_t partial_bytes; // workspace after the counters (cut-tile sums, then the slices' outputs)
    int slices;           // equal K slices, each served by its own CTAs (1: the whole K at once)
};
GemvStreamPlan plan_gemv_stream(int M, int N, int K, int group, int sym, int n_sm);
int gemv_stream_sm_count();
int launch_gemv_stream(const void* A, int a_dtype, int M, int K, const void* tiled, int N, int group, int sym,
                       void* C, void* workspace, int* dev_status, cudaStream_t stream);

// Persistent stream-K tensor-core GEMM. Its workspace is the same tile counters (one int per tile
// of 128 channels x BN rows), followed by the FP32 sums of tiles cut between CTAs ([P][BN][128]).
struct TcPlan {
    bool ok;
    int bn;               // rows of A per tile (the MMA's N)
    int mblocks;          // tiles of BN rows
    int ctas;             // persistent CTAs of each slice (one per SM in all)
    int nr, na, nd;       // ring depths: record slots, activation tiles, weight tiles
    uint32_t slot_w, off_a, off_w, off_bar;
    size_t smem;
    size_t partial_bytes; // workspace after the counters
};
TcPlan plan_gemm_tc(int M, int N, int K, int group, int sym, int n_sm);
int launch_gemm_tc(const void* A, int a_dtype, int M, int K, const void* tiled, int N, int group, int sym,
                   void* C, void* workspace, int* dev_status, cudaStream_t stream);

// Limit of every bounded wait on the device, in nanoseconds (2 s unless w4a16_set_wait_limit_ns
// changed it); each launch reads it once.
uint64_t wait_limit_ns();

}  // namespace w4a16
