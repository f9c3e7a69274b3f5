// kq_decode.cuh -- exact fp32 decode of 8 consecutive weights of a block.
//
// A "unit" is weights [8u, 8u+8) of one block.  Each decoder follows the
// codec's definition as IEEE fp32 operations: every product is exact (at
// most 21 significant bits), so the single rounding is the final
// subtraction and the result is unique.  The fused form fmaf(a, q, -b)
// with a = d*sc and b = dmin*m (both exact) rounds once, like a*q - b.
//
// Codec sources:
//  * Q8_0: ds4_metal.m, MSL `struct block_q8_0 { half d; int8_t qs[32]; }`.
//  * TQ1_G128: ternel_packed_model.py -- trit decode tables
//    (`_trit_table_source`, `_direct_trit_table_source`: digit i of byte p is
//    (p / 3^i) % 3, weight (digit - 1) * scale, illegal bytes -> 0) and
//    `_GET_ROWS_SOURCE` (weight j: slot j/5, digit j%5; tail slot 25 holds
//    weights 125..127).  Byte order in the 28-byte block: 25 full code bytes,
//    the tail byte, then the raw little-endian fp16 scale.
//  * Q4_K / Q2_K / Q5_K / Q6_K: the GGUF block layouts (named but not printed
//    on the pages: mlx-native quantized_matmul_id_ggml.rs type table).
#pragma once

#include "kq_common.cuh"

namespace kq {

__device__ __forceinline__ uint32_t ld_u32(const uint8_t *p) {
    return *reinterpret_cast<const uint32_t *>(p);
}
__device__ __forceinline__ uint32_t ld_u16(const uint8_t *p) {
    return *reinterpret_cast<const uint16_t *>(p);
}
__device__ __forceinline__ uint32_t byte_of(uint32_t w, int i) { return (w >> (8 * i)) & 0xFFu; }

// Q4_K 6-bit scale and min of sub-block j (0..7) from the 12 packed bytes,
// given as three little-endian words s0 = bytes 0..3, s1 = 4..7, s2 = 8..11.
__device__ __forceinline__ void q4k_scale_min(uint32_t s0, uint32_t s1, uint32_t s2, int j,
                                              uint32_t &sc, uint32_t &m) {
    if (j < 4) {
        sc = byte_of(s0, j) & 63u;
        m = byte_of(s1, j) & 63u;
    } else {
        const int i = j - 4;
        const uint32_t lo = byte_of(s2, i);        // byte j+4
        sc = (lo & 15u) | ((byte_of(s0, i) >> 6) << 4);
        m = (lo >> 4) | ((byte_of(s1, i) >> 6) << 4);
    }
}

template <int TYPE> struct Unit;

template <> struct Unit<KQ_Q8_0> {
    static constexpr int PER_BLOCK = 4;
    __device__ static void decode(const uint8_t *b, int u, float w[8]) {
        const float d = half_bits_to_float(ld_u16(b));
        const uint8_t *q = b + 2 + 8 * u;   // 2-byte aligned
        #pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t v = ld_u16(q + 2 * i);
            w[2 * i] = d * (float)(int8_t)(v & 0xFF);
            w[2 * i + 1] = d * (float)(int8_t)(v >> 8);
        }
    }
};

template <> struct Unit<KQ_Q4_K> {
    static constexpr int PER_BLOCK = 32;
    __device__ static void decode(const uint8_t *b, int u, float w[8]) {
        const int c = u >> 3, hi = (u >> 2) & 1, l0 = (u & 3) * 8;
        const uint32_t dd = ld_u32(b);
        const float d = half_bits_to_float(dd), dmin = half_bits_to_float(dd >> 16);
        uint32_t sc, m;
        q4k_scale_min(ld_u32(b + 4), ld_u32(b + 8), ld_u32(b + 12), 2 * c + hi, sc, m);
        const float a = d * (float)sc, bm = dmin * (float)m;
        const uint2 q = *reinterpret_cast<const uint2 *>(b + 16 + 32 * c + l0);
        const int sh = hi ? 4 : 0;
        #pragma unroll
        for (int i = 0; i < 4; ++i) {
            w[i] = fmaf(a, (float)((q.x >> (8 * i + sh)) & 15u), -bm);
            w[4 + i] = fmaf(a, (float)((q.y >> (8 * i + sh)) & 15u), -bm);
        }
    }
};

template <> struct Unit<KQ_Q2_K> {
    static constexpr int PER_BLOCK = 32;
    __device__ static void decode(const uint8_t *b, int u, float w[8]) {
        const int h = u >> 4, j = (u >> 2) & 3, l0 = (u & 3) * 8;
        const uint32_t dd = ld_u32(b + 80);
        const float d = half_bits_to_float(dd), dmin = half_bits_to_float(dd >> 16);
        const uint32_t s = b[8 * h + 2 * j + (l0 >> 4)];
        const float a = d * (float)(s & 15u), bm = dmin * (float)(s >> 4);
        const uint32_t q0 = ld_u32(b + 16 + 32 * h + l0), q1 = ld_u32(b + 16 + 32 * h + l0 + 4);
        #pragma unroll
        for (int i = 0; i < 4; ++i) {
            w[i] = fmaf(a, (float)((q0 >> (8 * i + 2 * j)) & 3u), -bm);
            w[4 + i] = fmaf(a, (float)((q1 >> (8 * i + 2 * j)) & 3u), -bm);
        }
    }
};

// Q5_K (GGUF layout): Q4_K's header and 6-bit scale/min packing, then 32
// high-bit bytes at 16 and 128 nibble bytes at 48.  Unit u: chunk c = u/8,
// nibble half hi = (u/4)&1, positions l0..l0+7 (l0 = 8*(u&3)) of the chunk;
// the fifth bit of position l is bit 2c+hi of high-bit byte l.
template <> struct Unit<KQ_Q5_K> {
    static constexpr int PER_BLOCK = 32;
    __device__ static void decode(const uint8_t *b, int u, float w[8]) {
        const int c = u >> 3, hi = (u >> 2) & 1, l0 = (u & 3) * 8;
        const uint32_t dd = ld_u32(b);
        const float d = half_bits_to_float(dd), dmin = half_bits_to_float(dd >> 16);
        uint32_t sc, m;
        q4k_scale_min(ld_u32(b + 4), ld_u32(b + 8), ld_u32(b + 12), 2 * c + hi, sc, m);
        const float a = d * (float)sc, bm = dmin * (float)m;
        const uint2 q = *reinterpret_cast<const uint2 *>(b + 48 + 32 * c + l0);
        const uint2 h = *reinterpret_cast<const uint2 *>(b + 16 + l0);
        const int sh = hi ? 4 : 0, hb = 2 * c + hi;
        #pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t q0 = ((q.x >> (8 * i + sh)) & 15u) | (((h.x >> (8 * i + hb)) & 1u) << 4);
            const uint32_t q1 = ((q.y >> (8 * i + sh)) & 15u) | (((h.y >> (8 * i + hb)) & 1u) << 4);
            w[i] = fmaf(a, (float)q0, -bm);
            w[4 + i] = fmaf(a, (float)q1, -bm);
        }
    }
};

// Q6_K (GGUF layout): ql[128] low bits, qh[64] high bits, int8 scales[16],
// fp16 d at 208.  Unit u covers weights 8u..8u+7 of half h = u/16, quarter
// r = (u/4)&3, positions l0..l0+7 (l0 = 8*(u&3)); quarters 0/1 take the low
// nibbles of ql[64h + l] / ql[64h + 32 + l], quarters 2/3 the high nibbles,
// with bits 2r, 2r+1 of qh[32h + l] on top; minus 32.  w = (d*sc)*q: the
// first product is exact, the second rounds once.
template <> struct Unit<KQ_Q6_K> {
    static constexpr int PER_BLOCK = 32;
    __device__ static void decode(const uint8_t *b, int u, float w[8]) {
        const int h = u >> 4, r = (u >> 2) & 3, l0 = (u & 3) * 8;
        const float d = half_bits_to_float(ld_u16(b + 208));
        const int sidx = 8 * h + (32 * r + l0) / 16;
        const float ds = d * (float)(int8_t)b[192 + sidx];
        const uint8_t *lq = b + 64 * h + ((r & 1) ? 32 : 0) + l0;
        const uint8_t *hq = b + 128 + 32 * h + l0;
        const int sh = (r & 2) ? 4 : 0;
        #pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int q = (int)(((uint32_t)lq[i] >> sh) & 15u) | (int)((((uint32_t)hq[i] >> (2 * r)) & 3u) << 4);
            w[i] = ds * (float)(q - 32);
        }
    }
};

// Base-3 digit `i` of a TQ1 code byte; an illegal byte reads as digit 1
// (weight 0) at every position.
__device__ __forceinline__ int tq1_digit(uint32_t code, int i, uint32_t max_legal) {
    if (code > max_legal) return 1;
    const uint32_t p3 = (i == 0) ? 1u : (i == 1) ? 3u : (i == 2) ? 9u : (i == 3) ? 27u : 81u;
    return (int)((code / p3) % 3u);
}

template <> struct Unit<KQ_TQ1_G128> {
    static constexpr int PER_BLOCK = 16;
    __device__ static void decode(const uint8_t *b, int u, float w[8]) {
        const float scale = half_bits_to_float(ld_u16(b + 26));
        #pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int j = 8 * u + i;
            int t;
            if (j < 125) t = tq1_digit(b[j / 5], j % 5, 242u);
            else t = tq1_digit(b[25], j - 125, 26u);
            w[i] = (float)(t - 1) * scale;
        }
    }
};

}  // namespace kq
