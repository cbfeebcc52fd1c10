// tiled_layout.cuh -- index map and region offsets of the tiled weight buffer (w4a16_repack).
#pragma once

#include <stddef.h>
#include <stdint.h>

namespace w4a16 {

constexpr int kTileN = 128;        // output channels per tile
constexpr int kTileK = 64;         // input channels per tile (8 packed rows)
constexpr int kTileWords = 1024;   // 128 x 8 int32 words = 4 KiB

// Word offset of plain word (j, n) inside the tiled codes region.
__host__ __device__ __forceinline__ size_t tiled_word_offset(int j, int n, int K) {
    const int t = n / kTileN, c = j / 8, jl = j % 8, nl = n % kTileN;
    const size_t tile = (size_t)t * (K / kTileK) + c;
    return tile * kTileWords + (size_t)((jl / 4) * 512 + nl * 4 + (jl % 4));
}

// Re-encoding of one plain word (nibble i = element i) for the tiled layout: slot p <- element
// 2p, slot p + 4 <- element 2p + 1; symmetric codes become offset-binary (two's complement
// nibble XOR 8 = q + 8).
__host__ __device__ __forceinline__ uint32_t tiled_encode_word(uint32_t w, int sym) {
    if (sym) w ^= 0x88888888u;
    uint32_t t = 0;
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        t |= ((w >> (8 * p)) & 0xFu) << (4 * p);             // element 2p
        t |= ((w >> (8 * p + 4)) & 0xFu) << (16 + 4 * p);    // element 2p + 1
    }
    return t;
}

struct TiledOffsets {
    size_t codes, codes_bytes;
    size_t scales, scales_bytes;
    size_t zeros, zeros_bytes;
    size_t total;
};

__host__ __device__ __forceinline__ size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

__host__ __device__ __forceinline__ TiledOffsets tiled_offsets(int K, int N, int group, int sym) {
    TiledOffsets o;
    o.codes = 0;
    o.codes_bytes = (size_t)K * N / 2;
    o.scales = align256(o.codes_bytes);
    o.scales_bytes = (size_t)(K / group) * N * 2;
    o.zeros = align256(o.scales + o.scales_bytes);
    o.zeros_bytes = sym ? 0 : (size_t)(K / group) * (N / 8) * 4;
    o.total = align256(o.zeros + o.zeros_bytes);
    return o;
}

}  // namespace w4a16
