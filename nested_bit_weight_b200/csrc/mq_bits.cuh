// Bit-plane rearrangements shared by the kernels of libmq (integer only, so
// that host checks can run them as well).
//
// Input: the r plane words of one 32-column word (P[p] bit j = bit (7 - p)
// of the code of column j; planes p >= r are passed as 0).
#pragma once

#include <stdint.h>

namespace mq {

// Pair stage: two planes (a more significant) -> 2-bit fields.
//   odd  word: bits (2i+1, 2i) = (a, b) of column 2i + 1
//   even word: bits (2i+1, 2i) = (a, b) of column 2i
__host__ __device__ __forceinline__ uint32_t pair_odd(uint32_t a, uint32_t b) {
    return (a & 0xAAAAAAAAu) | ((b >> 1) & 0x55555555u);
}
__host__ __device__ __forceinline__ uint32_t pair_even(uint32_t a, uint32_t b) {
    return ((a << 1) & 0xAAAAAAAAu) | (b & 0x55555555u);
}

// Quad stage: two pair words of one column class c (0 even, 1 odd) -> nibbles.
//   lo: nibble f = column 4f + c,   hi: nibble f = column 4f + 2 + c
__host__ __device__ __forceinline__ uint32_t quad_lo(uint32_t x, uint32_t y) {
    return ((x << 2) & 0xCCCCCCCCu) | (y & 0x33333333u);
}
__host__ __device__ __forceinline__ uint32_t quad_hi(uint32_t x, uint32_t y) {
    return (x & 0xCCCCCCCCu) | ((y >> 2) & 0x33333333u);
}

// Nibble words of planes [4h, 4h + 4): N[d] nibble f = column 4f + d, most
// significant plane in the nibble's top bit.
template <int R>
__host__ __device__ __forceinline__ void nibble_words(const uint32_t (&P)[8], int h, uint32_t (&N)[4]) {
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
__host__ __device__ __forceinline__ void byte_words(const uint32_t (&P)[8], uint32_t (&B)[8]) {
    uint32_t hi[4], lo[4] = {0u, 0u, 0u, 0u};
    nibble_words<R>(P, 0, hi);
    if constexpr (R > 4) nibble_words<R>(P, 1, lo);
#pragma unroll
    for (int d = 0; d < 4; ++d) {
        B[d] = ((hi[d] << 4) & 0xF0F0F0F0u) | (lo[d] & 0x0F0F0F0Fu);
        B[4 + d] = (hi[d] & 0xF0F0F0F0u) | ((lo[d] >> 4) & 0x0F0F0F0Fu);
    }
}

// Bytes b of E0 and E1 (two adjacent columns) as the low and high byte.
__host__ __device__ __forceinline__ uint32_t byte_pair(uint32_t E0, uint32_t E1, int b) {
    return ((E0 >> (8 * b)) & 0xFFu) | (((E1 >> (8 * b)) & 0xFFu) << 8);
}

// bf16 bit patterns of 256 + e0 (low half) and 256 + e1 (high half) for the
// bytes e0, e1 of t, both even (q_r << (8 - r) with r <= 7): bf16 0x4380 is
// 256 with a unit of 2 in its 7-bit mantissa, so e / 2 is the mantissa.
__host__ __device__ __forceinline__ uint32_t bf16_pair_256(uint32_t t) {
    return ((t >> 1) & 0x7Fu) | (((t >> 9) & 0x7Fu) << 16) | 0x43804380u;
}

// Byte permute: byte i of the result is byte (sel >> 4i) & 7 of the 8 bytes
// {a (bytes 0..3), b (bytes 4..7)} (PRMT, default mode; the host computes
// the same from the definition).
__host__ __device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
#ifdef __CUDA_ARCH__
    return __byte_perm(a, b, sel);
#else
    const uint64_t ab = (uint64_t)a | ((uint64_t)b << 32);
    uint32_t r = 0;
    for (int i = 0; i < 4; ++i) r |= (uint32_t)((ab >> (8 * ((sel >> (4 * i)) & 7u))) & 0xFFu) << (8 * i);
    return r;
#endif
}

// As byte_words with every byte halved (r <= 7): byte b of B[e] =
// q_r << (7 - r) of column 8b + e, at most 7 bits.
template <int R>
__host__ __device__ __forceinline__ void half_byte_words(const uint32_t (&P)[8], uint32_t (&B)[8]) {
    uint32_t hi[4], lo[4] = {0u, 0u, 0u, 0u};
    nibble_words<R>(P, 0, hi);
    if constexpr (R > 4) nibble_words<R>(P, 1, lo);
#pragma unroll
    for (int d = 0; d < 4; ++d) {
        B[d] = ((hi[d] << 3) & 0x78787878u) | ((lo[d] >> 1) & 0x07070707u);
        B[4 + d] = ((hi[d] >> 1) & 0x78787878u) | ((lo[d] >> 5) & 0x07070707u);
    }
}

// bf16 bit patterns of 256 + 2 h0 (low half) and 256 + 2 h1 (high half) for
// the halved bytes h0 = byte b of H0, h1 = byte b of H1 (adjacent columns):
// bf16 0x4380 is 256 with a unit of 2 in its 7-bit mantissa.
__host__ __device__ __forceinline__ uint32_t bf16_pair_from_halves(uint32_t H0, uint32_t H1, int b) {
    const uint32_t t = prmt(H0, H1, (uint32_t)b * 0x11u | ((uint32_t)(b + 4) * 0x1100u));
    return (t & 0x007F007Fu) | 0x43804380u;
}

}  // namespace mq
