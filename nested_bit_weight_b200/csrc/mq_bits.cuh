// Bit-plane rearrangements shared by the kernels of libmq (device only).
//
// Input: the r plane words of one 32-column word (P[p] bit j = bit (7 - p)
// of the code of column j; planes p >= r are passed as 0).
#pragma once

#include <stdint.h>

namespace mq {

// Pair stage: two planes (a more significant) -> 2-bit fields.
//   odd  word: bits (2i+1, 2i) = (a, b) of column 2i + 1
//   even word: bits (2i+1, 2i) = (a, b) of column 2i
__device__ __forceinline__ uint32_t pair_odd(uint32_t a, uint32_t b) {
    return (a & 0xAAAAAAAAu) | ((b >> 1) & 0x55555555u);
}
__device__ __forceinline__ uint32_t pair_even(uint32_t a, uint32_t b) {
    return ((a << 1) & 0xAAAAAAAAu) | (b & 0x55555555u);
}

// Quad stage: two pair words of one column class c (0 even, 1 odd) -> nibbles.
//   lo: nibble f = column 4f + c,   hi: nibble f = column 4f + 2 + c
__device__ __forceinline__ uint32_t quad_lo(uint32_t x, uint32_t y) {
    return ((x << 2) & 0xCCCCCCCCu) | (y & 0x33333333u);
}
__device__ __forceinline__ uint32_t quad_hi(uint32_t x, uint32_t y) {
    return (x & 0xCCCCCCCCu) | ((y >> 2) & 0x33333333u);
}

// Nibble words of planes [4h, 4h + 4): N[d] nibble f = column 4f + d, most
// significant plane in the nibble's top bit.
template <int R>
__device__ __forceinline__ void nibble_words(const uint32_t (&P)[8], int h, uint32_t (&N)[4]) {
    const uint32_t p0 = (4 * h < R) ? P[4 * h] : 0u;
    const uint32_t p1 = (4 * h + 1 < R) ? P[4 * h + 1] : 0u;
    const uint32_t p2 = (4 * h + 2 < R) ? P[4 * h + 2] : 0u;
    const uint32_t p3 = (4 * h + 3 < R) ? P[4 * h + 3] : 0u;
    const uint32_t x0 = pair_even(p0, p1), x1 = pair_odd(p0, p1);
    const uint32_t y0 = pair_even(p2, p3), y1 = pair_odd(p2, p3);
    N[0] = quad_lo(x0, y0);
    N[1] = quad_lo(x1, y1);
    N[2] = quad_hi(x0, y0);
    N[3] = quad_hi(x1, y1);
}

// Byte words: byte b of B[e] = q_r << (8 - r) of column 8b + e.
template <int R>
__device__ __forceinline__ void byte_words(const uint32_t (&P)[8], uint32_t (&B)[8]) {
    uint32_t hi[4], lo[4] = {0u, 0u, 0u, 0u};
    nibble_words<R>(P, 0, hi);
    if constexpr (R > 4) nibble_words<R>(P, 1, lo);
#pragma unroll
    for (int d = 0; d < 4; ++d) {
        B[d] = ((hi[d] << 4) & 0xF0F0F0F0u) | (lo[d] & 0x0F0F0F0Fu);
        B[4 + d] = (hi[d] & 0xF0F0F0F0u) | ((lo[d] >> 4) & 0x0F0F0F0Fu);
    }
}

}  // namespace mq
