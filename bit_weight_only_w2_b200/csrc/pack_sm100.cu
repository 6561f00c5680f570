// Packing of weight codes into the library's uint32 layout, and the inverse.
//
// Codes are packed along K into uint32 words (Bonsai-Image-Demo PR #20, GemLite int2 layout
// note; image-studio backend.md, "uint32 packed weights + scales"). The order inside the words
// is this library's own (cpw = 32 / bits codes per word):
//   * offset i of a word occupies bits [pos, pos + bits), pos = (i % 2) * 16 + (i / 2) * bits,
//     so offsets 2p and 2p + 1 (pair p) sit in the two 16-bit halves of the word;
//   * 2- and 4-bit rows are taken in blocks of four words (4 * cpw columns). In word q of a
//     block, pair p holds columns 8p + 2q and 8p + 2q + 1 of the block: exactly the codes lane
//     q of an mma.sync m16n8k16 B fragment needs for 2 (4-bit) or 4 (ternary) 16-wide K
//     steps, in order, so the small-M kernel loads one word per lane instead of a whole row;
//   * binary words, and the words after the last whole block of a 2- or 4-bit row, keep the
//     plain order: word j, offset i holds column cpw * j + i.
// Stored fields: binary +1 -> 1, -1 -> 0; ternary t -> t + 1; uint4 q -> q.
//
// One thread builds one word from its cpw codes (byte pairs gathered at a stride of 8 in block
// order, 16-byte loads in plain order). Invalid codes are counted in a device word (field
// written as 0); the host reads the count after the stream has drained.
#include <cuda_runtime.h>

#include <cstdint>

#include "lowbit_internal.h"

namespace lowbit {

__device__ unsigned long long g_pack_bad = 0;

namespace {

template <int BITS>
__device__ __forceinline__ uint32_t field_of(int c, bool& bad) {
    if (BITS == 1) {
        bad |= (c != 1 && c != -1);
        return c == 1 ? 1u : 0u;
    } else if (BITS == 2) {
        const bool ok = (c >= -1 && c <= 1);
        bad |= !ok;
        return ok ? static_cast<uint32_t>(c + 1) : 0u;
    } else {
        const bool ok = (c >= 0 && c <= 15);
        bad |= !ok;
        return ok ? static_cast<uint32_t>(c) : 0u;
    }
}

// Where word wi's codes start in the row-major code array, and whether they are in block order
// (pairs at columns start + 8p, p = 0 .. CPW/2 - 1) or plain order (columns start .. start+CPW-1).
// Rows hold wpr = K / CPW words.
template <int BITS>
__device__ __forceinline__ int64_t word_codes(int64_t wi, int64_t wpr, bool& block) {
    constexpr int CPW = 32 / BITS;
    const int64_t row = wi / wpr, j = wi - row * wpr;
    block = BITS != 1 && j < wpr / 4 * 4;
    const int64_t col = block ? (j / 4) * (4 * CPW) + 2 * (j % 4) : j * CPW;
    return row * wpr * CPW + col;
}

template <int BITS>
__global__ void pack_kernel(const int8_t* __restrict__ codes, int64_t total_words, int64_t wpr,
                            uint32_t* __restrict__ packed) {
    constexpr int CPW = 32 / BITS;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    unsigned long long bad_count = 0;
    for (int64_t wi = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; wi < total_words; wi += stride) {
        bool block;
        const int8_t* src = codes + word_codes<BITS>(wi, wpr, block);
        int8_t c[CPW];
        if (block) {
#pragma unroll
            for (int p = 0; p < CPW / 2; ++p)
                *reinterpret_cast<int16_t*>(c + 2 * p) = *reinterpret_cast<const int16_t*>(src + 8 * p);
        } else if (CPW >= 16) {
#pragma unroll
            for (int q = 0; q < CPW / 16; ++q) {
                const int4 v = reinterpret_cast<const int4*>(src)[q];
                *reinterpret_cast<int4*>(c + 16 * q) = v;
            }
        } else {
            *reinterpret_cast<int2*>(c) = *reinterpret_cast<const int2*>(src);
        }
        uint32_t w = 0;
        bool bad = false;
#pragma unroll
        for (int i = 0; i < CPW; ++i) {
            const int pos = (i % 2) * 16 + (i / 2) * BITS;
            w |= field_of<BITS>(c[i], bad) << pos;
        }
        packed[wi] = w;
        bad_count += bad ? 1 : 0;
    }
    if (bad_count) atomicAdd(&g_pack_bad, bad_count);
}

template <int BITS>
__global__ void unpack_kernel(const uint32_t* __restrict__ packed, int64_t total_words, int64_t wpr,
                              int8_t* __restrict__ codes) {
    constexpr int CPW = 32 / BITS;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    unsigned long long bad_count = 0;
    for (int64_t wi = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; wi < total_words; wi += stride) {
        const uint32_t w = packed[wi];
        int8_t c[CPW];
#pragma unroll
        for (int i = 0; i < CPW; ++i) {
            const int pos = (i % 2) * 16 + (i / 2) * BITS;
            const uint32_t f = (w >> pos) & ((1u << BITS) - 1u);
            if (BITS == 1) {
                c[i] = f ? 1 : -1;
            } else if (BITS == 2) {
                if (f == 3u) {
                    ++bad_count;
                    c[i] = 0;
                } else {
                    c[i] = static_cast<int8_t>(static_cast<int>(f) - 1);
                }
            } else {
                c[i] = static_cast<int8_t>(f);
            }
        }
        bool block;
        int8_t* dst = codes + word_codes<BITS>(wi, wpr, block);
        if (block) {
#pragma unroll
            for (int p = 0; p < CPW / 2; ++p)
                *reinterpret_cast<int16_t*>(dst + 8 * p) = *reinterpret_cast<const int16_t*>(c + 2 * p);
        } else if (CPW >= 16) {
#pragma unroll
            for (int q = 0; q < CPW / 16; ++q)
                reinterpret_cast<int4*>(dst)[q] = *reinterpret_cast<const int4*>(c + 16 * q);
        } else {
            *reinterpret_cast<int2*>(dst) = *reinterpret_cast<const int2*>(c);
        }
    }
    if (bad_count) atomicAdd(&g_pack_bad, bad_count);
}

int grid_for(int64_t words) {
    int64_t blocks = (words + 255) / 256;
    if (blocks > 148 * 16) blocks = 148 * 16;
    return static_cast<int>(blocks < 1 ? 1 : blocks);
}

lowbit_status finish(cudaStream_t stream, unsigned long long* bad) {
    if (cudaGetLastError() != cudaSuccess) return LOWBIT_ERR_CUDA;
    unsigned long long* dbad = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&dbad), g_pack_bad) != cudaSuccess) return LOWBIT_ERR_CUDA;
    if (cudaMemcpyAsync(bad, dbad, sizeof(*bad), cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return LOWBIT_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return LOWBIT_ERR_CUDA;
    return LOWBIT_OK;
}

lowbit_status reset_counter(cudaStream_t stream) {
    unsigned long long* dbad = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&dbad), g_pack_bad) != cudaSuccess) return LOWBIT_ERR_CUDA;
    if (cudaMemsetAsync(dbad, 0, sizeof(*dbad), stream) != cudaSuccess) return LOWBIT_ERR_CUDA;
    return LOWBIT_OK;
}

}  // namespace

lowbit_status pack_launch(const int8_t* codes, int64_t N, int64_t K, int bits, uint32_t* packed,
                          cudaStream_t stream, unsigned long long* bad) {
    *bad = 0;
    const int64_t words = N * K * bits / 32;
    if (words == 0) return LOWBIT_OK;
    lowbit_status st = reset_counter(stream);
    if (st != LOWBIT_OK) return st;
    const int grid = grid_for(words);
    const int64_t wpr = K * bits / 32;
    if (bits == 1) pack_kernel<1><<<grid, 256, 0, stream>>>(codes, words, wpr, packed);
    else if (bits == 2) pack_kernel<2><<<grid, 256, 0, stream>>>(codes, words, wpr, packed);
    else pack_kernel<4><<<grid, 256, 0, stream>>>(codes, words, wpr, packed);
    return finish(stream, bad);
}

lowbit_status unpack_launch(const uint32_t* packed, int64_t N, int64_t K, int bits, int8_t* codes,
                            cudaStream_t stream, unsigned long long* bad) {
    *bad = 0;
    const int64_t words = N * K * bits / 32;
    if (words == 0) return LOWBIT_OK;
    lowbit_status st = reset_counter(stream);
    if (st != LOWBIT_OK) return st;
    const int grid = grid_for(words);
    const int64_t wpr = K * bits / 32;
    if (bits == 1) unpack_kernel<1><<<grid, 256, 0, stream>>>(packed, words, wpr, codes);
    else if (bits == 2) unpack_kernel<2><<<grid, 256, 0, stream>>>(packed, words, wpr, codes);
    else unpack_kernel<4><<<grid, 256, 0, stream>>>(packed, words, wpr, codes);
    return finish(stream, bad);
}

}  // namespace lowbit
