// repack.cu -- one-time permutation of the plain packed weight into the tiled layout of unit
// records (tiled_layout.cuh).
//
// "INT4 and Low-Bit Inference", section 5 "The kernel is half the story": weights are permuted
// once at load so that unpacking is branch-free and coalesced. "4.3 Weight-only INT4", section 4:
// weights pre-reordered into a layout that suits runtime reads. Nothing is rounded: a bijection
// of the code bits, plus copies of the scales and zeros into the records of their units (with
// scale 0 for a group whose codes all equal its zero point, which dequantizes to the same zeros).
#include "common.cuh"
#include "tiled_layout.cuh"

namespace w4a16 {

namespace {

__global__ void repack_codes_kernel(const int32_t* __restrict__ codes, int K, int N, int sym, uint32_t record,
                                    uint8_t* __restrict__ tiled) {
    // one thread per plain word, in plain order: coalesced reads
    const size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const size_t total = (size_t)(K / 8) * N;
    if (idx >= total) return;
    const int j = (int)(idx / N);
    const int n = (int)(idx - (size_t)j * N);
    *reinterpret_cast<uint32_t*>(tiled + tiled_word_byte(j, n, K, record)) =
        tiled_encode_word((uint32_t)codes[idx], sym);
}

// One thread per (group row, channel): the scale, and for the first channel of each 8 the zeros
// word, into the record of the unit that holds the group. A (group, channel) whose codes all
// equal its zero point (0 for the symmetric scheme: the degenerate group) stores scale 0: its
// dequantized weights are 0 with either scale, and the decode kernel's zero-point correction is
// then exactly zero there.
__global__ void repack_meta_kernel(const int32_t* __restrict__ codes, const uint16_t* __restrict__ scales,
                                   const int32_t* __restrict__ zeros, int K, int N, int group, TiledLayout L,
                                   uint8_t* __restrict__ tiled) {
    const size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const size_t total = (size_t)(K / group) * N;
    if (idx >= total) return;   // writes nothing, so nothing to make visible
    const int gi = (int)(idx / N);
    const int n = (int)(idx - (size_t)gi * N);
    const int c = gi / L.groups, gg = gi % L.groups;
    const int t = n / kTileN, nl = n % kTileN;
    uint8_t* rec = tiled + ((size_t)t * (K / kTileK) + c) * L.record;
    const uint32_t zp = zeros ? ((uint32_t)zeros[(size_t)gi * (N / 8) + n / 8] >> (4 * (n % 8))) & 0xFu : 0u;
    const uint32_t zrep = zp * 0x11111111u;
    bool all_zero_point = true;
    for (int jj = 0; jj < group / 8; ++jj)
        all_zero_point = all_zero_point && (uint32_t)codes[((size_t)gi * (group / 8) + jj) * N + n] == zrep;
    *reinterpret_cast<uint16_t*>(rec + L.scales + 256 * gg + 2 * nl) = all_zero_point ? (uint16_t)0 : scales[idx];
    if (zeros && (nl & 7) == 0)
        *reinterpret_cast<int32_t*>(rec + L.zeros + 64 * gg + 4 * (nl / 8)) = zeros[(size_t)gi * (N / 8) + n / 8];
    // the decode kernel may start on the next launch before this grid has completed (programmatic
    // dependent launch) and begins streaming weight records before it waits for this grid: every
    // thread's stores are made visible device-wide before the thread exits
    __threadfence();
}

}  // namespace

int launch_repack(const int32_t* codes, const void* scales, const int32_t* zeros, int K, int N,
                  int group, int sym, void* tiled, cudaStream_t stream) {
    const TiledLayout L = tiled_layout(K, N, group, sym);
    const int threads = 256;
    const size_t words = (size_t)(K / 8) * N;
    repack_codes_kernel<<<(unsigned)((words + threads - 1) / threads), threads, 0, stream>>>(
        codes, K, N, sym, L.record, static_cast<uint8_t*>(tiled));
    if (cudaGetLastError() != cudaSuccess) return W4A16_ECUDA;
    const size_t meta = (size_t)(K / group) * N;
    repack_meta_kernel<<<(unsigned)((meta + threads - 1) / threads), threads, 0, stream>>>(
        codes, static_cast<const uint16_t*>(scales), sym ? nullptr : zeros, K, N, group, L,
        static_cast<uint8_t*>(tiled));
    return launch_status();
}

}  // namespace w4a16
