// repack.cu -- one-time permutation of the plain packed codes into the tiled layout.
//
// "INT4 and Low-Bit Inference", section 5 "The kernel is half the story": weights are permuted
// once at load so that unpacking is branch-free and coalesced. "4.3 Weight-only INT4", section 4:
// weights pre-reordered into a layout that suits runtime reads.
//
// Tile (t, c): output channels [128 t, 128 t + 128), packed rows j in [8 c, 8 c + 8)
// (input channels [64 c, 64 c + 64)); tile index t * (K / 64) + c; 1024 words per tile.
// Word (j, n) of the plain layout goes to word offset, inside its tile,
//     ((j % 8) / 4) * 512 + (n % 128) * 4 + (j % 4)
// so a 16-byte vector holds four consecutive packed rows of one output channel and 32
// consecutive channels read 512 contiguous bytes. Inside each word the eight codes are
// re-ordered (tiled_encode_word): nibble slot p holds element 2p and slot p + 4 holds element
// 2p + 1 (p = 0..3), so that one mask of the word yields two adjacent K elements in the two
// 16-bit halves of a register. Symmetric codes are stored offset-binary (q + 8, zero-point 8).
// Scales and zeros are copied unchanged after the codes, each region starting on a 256-byte
// boundary. Nothing is rounded: a bijection of bits.
#include "common.cuh"
#include "tiled_layout.cuh"

namespace w4a16 {

namespace {

__global__ void repack_codes_kernel(const int32_t* __restrict__ codes, int K, int N, int sym,
                                    int32_t* __restrict__ tiled) {
    // one thread per plain word, in plain order: coalesced reads, 16-byte-grouped writes
    const size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const size_t total = (size_t)(K / 8) * N;
    if (idx >= total) return;
    const int j = (int)(idx / N);
    const int n = (int)(idx - (size_t)j * N);
    tiled[tiled_word_offset(j, n, K)] = (int32_t)tiled_encode_word((uint32_t)codes[idx], sym);
}

}  // namespace

int launch_repack(const int32_t* codes, const void* scales, const int32_t* zeros, int K, int N,
                  int group, int sym, void* tiled, cudaStream_t stream) {
    const TiledOffsets off = tiled_offsets(K, N, group, sym);
    const size_t total = (size_t)(K / 8) * N;
    const int threads = 256;
    repack_codes_kernel<<<(unsigned)((total + threads - 1) / threads), threads, 0, stream>>>(
        codes, K, N, sym, static_cast<int32_t*>(tiled));
    if (cudaGetLastError() != cudaSuccess) return W4A16_ECUDA;
    char* base = static_cast<char*>(tiled);
    if (cudaMemcpyAsync(base + off.scales, scales, off.scales_bytes, cudaMemcpyDeviceToDevice,
                        stream) != cudaSuccess)
        return W4A16_ECUDA;
    if (!sym && cudaMemcpyAsync(base + off.zeros, zeros, off.zeros_bytes, cudaMemcpyDeviceToDevice,
                                stream) != cudaSuccess)
        return W4A16_ECUDA;
    return W4A16_OK;
}

}  // namespace w4a16
