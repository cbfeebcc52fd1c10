// tiled_layout.cuh -- the tiled weight buffer of w4a16_repack: one contiguous record per unit of
// 128 output channels x 128 input channels.
//
// "INT4 and Low-Bit Inference", section 5 "The kernel is half the story": weights are permuted once
// at load so that unpacking is branch-free and the reads are coalesced; "4.3 Weight-only INT4",
// section 4: a pre-reordered layout that suits runtime reads. The form is the library's own:
//   unit (t, c) = channels [128 t, 128 t + 128) x input channels [128 c, 128 c + 128), record index
//   t * (K / 128) + c, R = 8192 + G * 256 + (asym ? G * 64 : 0) bytes, G = 128 / group;
//   codes  [0, 8192): block h = 0..3 (input channels 128 c + 32 h ..) at 2048 h; channel n owns the
//          16 bytes at slot (n ^ 2h) of its block; word w of them is packed row 16 c + 4 h + w,
//          nibbles re-ordered (slot p <- element 2p, slot p + 4 <- element 2p + 1), symmetric
//          codes offset-binary (q + 8);
//   scales [8192, + G * 256): group gg of the unit at 256 gg, channel n at + 2 n;
//   zeros  (asymmetric) [8192 + G * 256, + G * 64): group gg at 64 gg, the tile's 16 plain words.
// A CTA that streams consecutive units reads one contiguous range (one bulk copy per stage); the
// XOR slot makes the 16-byte reads of an MMA fragment (lanes g, t reading block t, channel g)
// bank-conflict free.
#pragma once

#include <stddef.h>
#include <stdint.h>

namespace w4a16 {

constexpr int kTileN = 128;   // output channels per unit
constexpr int kTileK = 128;   // input channels per unit (16 packed rows)

struct TiledLayout {
    uint32_t record;   // bytes per unit record
    uint32_t scales;   // scales offset inside a record
    uint32_t zeros;    // zeros offset inside a record
    int groups;        // groups of K per unit
    size_t total;      // whole buffer
};

__host__ __device__ __forceinline__ TiledLayout tiled_layout(int K, int N, int group, int sym) {
    TiledLayout l;
    l.groups = 128 / group;
    l.scales = 8192u;
    l.zeros = 8192u + 256u * (uint32_t)l.groups;
    l.record = l.zeros + (sym ? 0u : 64u * (uint32_t)l.groups);
    l.total = (size_t)(N / kTileN) * (size_t)(K / kTileK) * l.record;
    return l;
}

// Byte offset of plain word (j, n) (packed row j, channel n) in the tiled buffer.
__host__ __device__ __forceinline__ size_t tiled_word_byte(int j, int n, int K, uint32_t record) {
    const int t = n / kTileN, nl = n % kTileN, c = j / 16, h = (j % 16) / 4, w = j % 4;
    const size_t rec = (size_t)t * (K / kTileK) + c;
    return rec * record + (size_t)(2048 * h + 16 * (nl ^ (2 * h)) + 4 * w);
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

}  // namespace w4a16
