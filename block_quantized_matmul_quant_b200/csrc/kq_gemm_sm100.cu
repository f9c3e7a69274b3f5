// kq_gemm_sm100.cu -- tensor-core product for many activation rows (prefill).
//
// Y[m][n] = sum_k X[m][k] * dequant(W)[n][k]: the qmm case of mlx-kquant
// `quantized_matmul` (the pages' Metal form stages a 64 x 32 weight tile in
// threadgroup memory and reuses it across routed rows, mlx-native
// `kernel_mul_mm_id_*`; Ternary Bonsai `tq1_gemm` decodes into 8 x 8
// simdgroup fragments).  Here it is written for sm_100a:
//
//  * Persistent kernel, one CTA per SM, static round-robin over output tiles
//    of 128 weight rows (the MMA's M) x BN tokens (the MMA's N, a multiple of
//    16 <= 192 picked by the host to balance waves over the SMs).
//  * The decoded weights never touch shared memory: decoder threads turn raw
//    super-block bytes into bf16 in registers and write them straight into
//    tensor memory (tcgen05.st), where the MMA reads its A operand
//    (tcgen05.mma with A in TMEM, B = activations in shared memory).  Shared
//    memory only carries the activation tiles and the raw bytes, so the
//    tensor core's operand reads do not compete with decoder stores.
//  * Warp roles:  warp 0  TMA producer of bf16 activation tiles (64 K x BN,
//                         128-byte swizzle) into a shared-memory ring;
//                 warp 6  TMA producer of raw weight units (128 rows x one
//                         Q4_K super-block, 144 bytes, one Q5_K super-block,
//                         176 bytes, eight Q8_0 blocks, 272 bytes, four Q2_K
//                         super-blocks, 336 bytes, or four TQ1_G128 blocks,
//                         112 bytes) into their own ring;
//                 warp 1  MMA issuer -- one thread issues tcgen05.mma
//                         (kind::f16, bf16 x bf16 -> fp32 in TMEM) and
//                         tcgen05.commit's to the stage / accumulator barriers;
//                 warps 2-5  epilogue -- tcgen05.ld from TMEM, convert, store;
//                 warps 7..  decoders, in groups of four warps (one per TMEM
//                         lane quadrant, so lane = weight row; two groups
//                         for Q4_K, four for TQ1_G128): group j
//                         decodes the stages s with s % groups == j, 64 K
//                         positions of its 32 rows per warp.  Q4_K: exact
//                         fp32 (d*sc*q - dmin*m, one rounding) -> bf16 (round
//                         to nearest even); Q5_K (five-bit q), Q8_0 (d * q)
//                         and Q2_K (d*sc*q - dmin*m) likewise.
//                         TQ1_G128 (Ternary Bonsai
//                         `tq1_gemm`, the prefill form of the ternary
//                         product): base-3 digits by integer arithmetic, two
//                         bytes' digits a 32-bit word, then (t - 1) * bf16(scale)
//                         -- the round-to-nearest-even bf16 of the weight.
//  * TMEM (512 columns): accumulators at columns 0 and 256 (BN each, so the
//    epilogue of tile i overlaps the main loop of tile i+1); the stage ring's
//    A slots (32 columns = 128 rows x 64 bf16) fill the gaps after them.
//  * Every mbarrier wait is bounded (kq_ptx.cuh): on timeout the kernel sets
//    the device error word and the waiting role stops; TMEM is released by
//    the allocating warp after a block barrier that every thread reaches.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "kq_decode.cuh"
#include "kq_ptx.cuh"
#include "kq_tc.cuh"
#include "kq_launch.h"

namespace kq {

namespace {

constexpr int BM = 128;            // weight rows per tile (MMA M)
constexpr int BK = 64;             // K per swizzle atom (128 bytes of bf16); a stage holds CPS atoms
// Raw weights move in units of one TMA box row, the fewest whole blocks
// whose bytes are a multiple of 16 (so K must be a multiple of the unit's
// K): a Q4_K super-block (144 bytes, 256 K), a Q5_K super-block (176, 256),
// eight Q8_0 blocks (272, 256), four Q2_K super-blocks (336, 1024) or four
// TQ1_G128 blocks (112, 512).  ELEM: bytes per tensor-map element -- 2 for
// the units above 256 bytes, since a box row holds at most 256 elements.
template <int FMT> struct RawUnit;
template <> struct RawUnit<KQ_Q4_K> { static constexpr int BYTES = 144, K = 256, ELEM = 1; };
template <> struct RawUnit<KQ_Q5_K> { static constexpr int BYTES = 176, K = 256, ELEM = 1; };
template <> struct RawUnit<KQ_Q8_0> { static constexpr int BYTES = 272, K = 256, ELEM = 2; };
template <> struct RawUnit<KQ_Q2_K> { static constexpr int BYTES = 336, K = 1024, ELEM = 2; };
template <> struct RawUnit<KQ_TQ1_G128> { static constexpr int BYTES = 112, K = 512, ELEM = 1; };
constexpr int raw_unit_bytes(int type) {
    return type == KQ_TQ1_G128 ? 112 : type == KQ_Q8_0 ? 272 : type == KQ_Q2_K ? 336 : type == KQ_Q5_K ? 176 : 144;
}
constexpr int raw_unit_k(int type) { return type == KQ_TQ1_G128 ? 512 : type == KQ_Q2_K ? 1024 : 256; }
constexpr int raw_stage_bytes(int type) { return BM * raw_unit_bytes(type); }
constexpr int RAW_WARP = 6;  // raw weight producer
constexpr int DEC_WARP0 = 7;
// Decoder warps per format: eight (two groups) for the K-quants and Q8_0,
// sixteen (four groups) for TQ1_G128, whose integer digit decode bounds the
// narrow tiles.  Measured on B200 (µs): Q4_K 512x11008x4096 65.9 with eight
// against 67.7 with sixteen, 16 rows 25.8 against 26.3; TQ1 512x5120x17408
// 135.9 against 140.0 but 16 rows 108.0 against 101.0.
template <int FMT> constexpr int dec_warps() { return FMT == KQ_TQ1_G128 ? 16 : 8; }
template <int FMT> constexpr int num_threads() { return (DEC_WARP0 + dec_warps<FMT>()) * 32; }
constexpr int EPI_WARP0 = 2;
constexpr int MAX_RAW_STAGES = 8;
constexpr int MAX_A_STAGES = 8;   // TMEM A slots
constexpr int MAX_B_STAGES = 32;  // activation tiles in shared memory
constexpr int MAX_BN = 192;
constexpr int SMEM_BUDGET = 227 * 1024;
// Epilogue staging: each epilogue warp owns two buffers of one 16-token x
// 32-row output chunk, written to global memory by TMA stores.
constexpr int EPI_CHUNK_M = 16, EPI_CHUNK_N = 32;
constexpr int EPI_STAGE_BYTES = 2 * 4 * EPI_CHUNK_M * EPI_CHUNK_N * 4;  // 2 buffers x 4 warps, f32 size

struct GemmParams {
    int n, k, m;
    int bn, m_tiles, n_tiles, tiles;
    int a_stages;  // decoded-weight ring: A slots in TMEM
    int b_stages;  // activation ring: tiles in shared memory (deeper: their loads come from L2)
    int raw_stages;  // raw weight ring (each slot: 128 rows x one raw unit)
    int a_col0;    // first TMEM column after an accumulator (BN rounded up to 32)
    int b_stage_bytes;
    void *y;
    unsigned int *err;
    int y_tma;     // dense output through TMA stores (tmap_y) instead of per-element stores
    // expert-indexed mode: token tiles come from the device-side grouping
    const int32_t *perm;      // pair indices t * top_k + s, grouped by expert
    const int32_t *offsets;   // [E + 1] segment starts in perm
    const int2 *id_tiles;     // (expert, first position in perm) per token tile
    const int32_t *id_n_tiles;
    int top_k;
    int n_pairs, n_experts;   // entries of perm; experts of the stack
    // expert-indexed GLU, second pass: y = act(this product) * y, y holding
    // the up projection written by the first pass (glu: 0 plain store, 1
    // combine; act: KQ_ACT_*)
    int glu, act;
};

__device__ __forceinline__ float load_out(const float *p) { return *p; }
__device__ __forceinline__ float load_out(const __nv_bfloat16 *p) { return __bfloat162float(*p); }

// One output tile: weight rows n0.. of expert e times BN activation rows.
// Dense: activation rows m0..m0+rows-1.  Expert-indexed: the activation rows
// of pairs perm[m0 .. m0+rows-1].
struct Tile {
    int n0, e, m0, rows;
};

template <bool ID>
__device__ __forceinline__ Tile tile_at(const GemmParams &p, int u) {
    Tile t;
    if constexpr (ID) {
        int2 tt = p.id_tiles[u / p.n_tiles];
        // KQ_DEBUG: a tile outside the grouping becomes an empty tile of
        // expert 0 at position 0 (its loads stay in bounds, nothing is stored)
        const bool ok = KQ_DCHECK(tt.x >= 0 && tt.x < p.n_experts && tt.y >= 0 && tt.y < p.n_pairs &&
                                      p.offsets[tt.x + 1] <= p.n_pairs, p.err);
        if (!ok) tt = make_int2(0, 0);
        t.n0 = (u % p.n_tiles) * BM;
        t.e = tt.x;
        t.m0 = tt.y;
        t.rows = ok ? min(p.bn, p.offsets[tt.x + 1] - tt.y) : 0;
    } else {
        t.n0 = (u / p.m_tiles) * BM;
        t.e = 0;
        t.m0 = (u % p.m_tiles) * p.bn;
        t.rows = min(p.bn, p.m - t.m0);
    }
    return t;
}

// TMEM accumulators: two (columns 0 and 256; the epilogue of one tile
// overlaps the next tile's main loop) or, as a build option, one (more A
// slots; measured slower).
#ifndef KQ_GEMM_ACC_BUFS
#define KQ_GEMM_ACC_BUFS 2
#endif
constexpr int ACC_BUFS = KQ_GEMM_ACC_BUFS;
static_assert(ACC_BUFS == 1 || ACC_BUFS == 2, "one or two accumulators");

// TMEM column of stage slot s, 32 columns per 64 K of the stage (CPS of
// them).  Two accumulators: slots alternate between the gap after the first
// (a_col0..255) and the gap after the second (256 + a_col0..511).  One
// accumulator: slots follow it.
template <int CPS>
__device__ __forceinline__ uint32_t a_slot_col(uint32_t s, int a_col0) {
    return ACC_BUFS == 2 ? ((s & 1u) << 8) + (uint32_t)a_col0 + (s >> 1) * (32u * CPS)
                         : (uint32_t)a_col0 + s * (32u * CPS);
}

__device__ __forceinline__ float half_f(uint32_t bits) { return half_bits_to_float(bits); }

// Byte i of w as an exact float (2^23 exponent trick).
__device__ __forceinline__ float byte_float(uint32_t w, int i) {
    return __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7440u | (uint32_t)i)) - 8388608.0f;
}

// Four quant bytes (one nibble each, already masked: q or 16*q) -> two bf16x2
// words of w = scale * nibble + bias with one fp32 rounding, then RNE to bf16.
__device__ __forceinline__ void decode4(uint32_t nib, float2 scale, float2 bias, uint32_t &o0,
                                        uint32_t &o1) {
    const float2 magic = make_float2(-8388608.0f, -8388608.0f), one = make_float2(1.f, 1.f);
    float2 f0 = make_float2(__uint_as_float(__byte_perm(nib, 0x4B000000u, 0x7440u)),
                            __uint_as_float(__byte_perm(nib, 0x4B000000u, 0x7441u)));
    float2 f1 = make_float2(__uint_as_float(__byte_perm(nib, 0x4B000000u, 0x7442u)),
                            __uint_as_float(__byte_perm(nib, 0x4B000000u, 0x7443u)));
    f0 = ffma2(f0, one, magic);  // exact: the nibble value
    f1 = ffma2(f1, one, magic);
    f0 = ffma2(f0, scale, bias);  // exact products, one rounding each
    f1 = ffma2(f1, scale, bias);
    const __nv_bfloat162 b0 = __floats2bfloat162_rn(f0.x, f0.y);
    const __nv_bfloat162 b1 = __floats2bfloat162_rn(f1.x, f1.y);
    o0 = *reinterpret_cast<const uint32_t *>(&b0);
    o1 = *reinterpret_cast<const uint32_t *>(&b1);
}

// Base-3 digits of a TQ1 code byte b (0..242), two to a 32-bit word in
// 16-bit lanes, the order of the weights: lo = (d1 << 16) | d0,
// mid = (d3 << 16) | d2, hi = d4.  Division by 3 of both lanes at once is a
// multiply by 171 and a shift by 9 (exact for 0..255; a lane's product stays
// below 2^16, so the lanes do not mix).
__device__ __forceinline__ void tq1_digits(uint32_t b, uint32_t &lo, uint32_t &mid, uint32_t &hi) {
    const uint32_t x0 = b | (((b * 171u) >> 9) << 16);          // (b, b/3)
    const uint32_t q0 = ((x0 * 171u) >> 9) & 0x007F007Fu;       // (b/3, b/9)
    lo = x0 - 3u * q0;                                           // (d0, d1)
    const uint32_t x1 = ((q0 * 171u) >> 9) & 0x007F007Fu;       // (b/9, b/27)
    const uint32_t q1 = ((x1 * 171u) >> 9) & 0x007F007Fu;       // (b/27, b/81)
    mid = x1 - 3u * q1;                                          // (d2, d3)
    hi = q1 >> 16;                                               // b/81 = d4
}

// Two digits (16-bit lanes, 0..2) -> bf16x2 of (d - 1) * s: the lanes as
// bf16 are 128 + d, and 128 + d - 129 and the product with +-1 or 0 are exact.
__device__ __forceinline__ uint32_t tq1_word(uint32_t dd, __nv_bfloat162 s2) {
    const uint32_t v = dd | 0x43004300u, c = 0x43014301u;   // bf16x2 (128 + d), (129, 129)
    const __nv_bfloat162 t = __hmul2(__hsub2(*reinterpret_cast<const __nv_bfloat162 *>(&v),
                                             *reinterpret_cast<const __nv_bfloat162 *>(&c)),
                                     s2);
    return *reinterpret_cast<const uint32_t *>(&t);
}

// Weights 64 H .. 64 H + 63 of the TQ1_G128 block at `blk` (4-byte aligned)
// as 32 bf16x2 words of bf16(scale) * (t - 1), word j holding weights
// 64 H + 2 j and + 1.  Weight i of a block is digit i % 5 of byte i / 5 (the
// tail byte 25 holds weights 125..127); a full byte above 242 or a tail
// byte above 26 is not a code and decodes to zeros (as byte 121, all digits
// 1).  The block's position in the raw unit is a runtime offset, so the
// decoders hold two copies of this code (one per half), not one per chunk
// position: fewer instructions to fetch.
template <int H>
__device__ __forceinline__ void tq1_decode64(const uint8_t *blk, uint32_t out[32]) {
    // block words: half 0 needs bytes 0..12 (words 0..3) and the scale (word
    // 6), half 1 bytes 12..27 (words 3..6)
    const uint32_t *bw = reinterpret_cast<const uint32_t *>(blk);
    uint32_t wv[7];
    #pragma unroll
    for (int q = 0; q < 7; ++q)
        if ((H == 0 && (q <= 3 || q == 6)) || (H == 1 && q >= 3)) wv[q] = bw[q];
    const __nv_bfloat16 sb = __float2bfloat16_rn(half_bits_to_float(wv[6] >> 16));   // bytes 26..27
    const __nv_bfloat162 s2 = __halves2bfloat162(sb, sb);
    // digit words of block bytes J0 .. J0 + 13 (13 used by half 0)
    constexpr int J0 = H == 0 ? 0 : 12;
    uint32_t dg[14][3];
    #pragma unroll
    for (int jj = 0; jj < 14; ++jj) {
        const int j = J0 + jj;
        if (j > 25 || (H == 0 && j > 12)) continue;
        uint32_t b = (wv[j / 4] >> (8 * (j % 4))) & 0xFFu;
        b = b > (j == 25 ? 26u : 242u) ? 121u : b;
        tq1_digits(b, dg[jj][0], dg[jj][1], dg[jj][2]);
    }
    #pragma unroll
    for (int w = 0; w < 32; ++w) {
        const int i0 = 64 * H + 2 * w, i1 = i0 + 1;
        const int j0 = i0 / 5 - J0, d0 = i0 % 5, j1 = i1 / 5 - J0, d1 = i1 % 5;
        // lane of digit d in its byte's words: word d / 2, 16-bit half d % 2
        const uint32_t a = dg[j0][d0 >> 1], c = dg[j1][d1 >> 1];
        uint32_t dd;
        if (j0 == j1 && (d0 & 1) == 0) dd = a;                           // (d0, d0 + 1) of one word
        else dd = __byte_perm(a, c, ((d0 & 1) ? 0x32u : 0x10u) | ((d1 & 1) ? 0x7600u : 0x5400u));
        out[w] = tq1_word(dd, s2);
    }
}

// 64-K chunk cc (0..7) of a row's raw TQ1 unit: half cc % 2 of block cc / 2.
__device__ __forceinline__ void tq1_decode_chunk(const uint8_t *row, int cc, uint32_t out[32]);

// 64-K chunk cc (0..3) of a row's raw Q8_0 unit (eight 34-byte blocks: fp16
// d, then 32 int8 q; weight d * q): blocks 2 cc and 2 cc + 1, bytes
// 68 cc .. 68 cc + 67 of the row (4-byte aligned), as 32 bf16x2 words of the
// round-to-nearest-even bf16 of d * q.  The second block's codes are
// word-aligned; the first block's sit two bytes in and are realigned with
// funnel shifts.  Each code goes in as the byte q + 128 (xor 0x80) and
// comes out as d * (q + 128) - 128 d in one fused rounding (decode4).
__device__ __forceinline__ void q8_0_decode_chunk(const uint8_t *row, int cc, uint32_t out[32]) {
    const uint32_t *w = reinterpret_cast<const uint32_t *>(row + 68 * cc);
    uint32_t v[17];
    #pragma unroll
    for (int i = 0; i < 17; ++i) v[i] = w[i];
    const float d0 = half_f(v[0] & 0xFFFFu), d1 = half_f(v[8] >> 16);
    const float2 s0 = make_float2(d0, d0), b0 = make_float2(-128.0f * d0, -128.0f * d0);
    const float2 s1 = make_float2(d1, d1), b1 = make_float2(-128.0f * d1, -128.0f * d1);
    #pragma unroll
    for (int j = 0; j < 8; ++j) {
        const uint32_t qa = __funnelshift_r(v[j], v[j + 1], 16);   // block 2 cc: codes 4 j .. 4 j + 3
        decode4(qa ^ 0x80808080u, s0, b0, out[2 * j], out[2 * j + 1]);
        decode4(v[9 + j] ^ 0x80808080u, s1, b1, out[16 + 2 * j], out[17 + 2 * j]);
    }
}

// 64-K chunk cc (0..15) of a row's raw Q2_K unit (four 84-byte super-blocks:
// scale/min bytes at 0 (low nibble scale, high nibble min, one per 16
// weights), 2-bit codes at 16 (bit pair j of byte 32 h + l is weight
// 128 h + 32 j + l), fp16 d and dmin at 80; weight d*sc*q - dmin*m): chunk
// c4 = cc % 4 of super-block cc / 4 is weights 128 h + 32 j + l with
// h = c4 / 2, j = 2 (c4 % 2) + jj (jj = 0, 1), l = 0..31, as 32 bf16x2 words
// of the round-to-nearest-even bf16 of the exact weight (decode4: one fused
// rounding of q * (d*sc) - dmin*m, both products exact).
__device__ __forceinline__ void q2_k_decode_chunk(const uint8_t *row, int cc, uint32_t out[32]) {
    const uint32_t *bw = reinterpret_cast<const uint32_t *>(row + 84 * (cc >> 2));   // 4-byte aligned
    const int c4 = cc & 3, h = c4 >> 1, j0 = 2 * (c4 & 1);
    const uint32_t dd = bw[20];
    const float d = half_f(dd & 0xFFFFu), dmin = half_f(dd >> 16);
    const uint32_t sw = bw[2 * h + (c4 & 1)];   // scale/min bytes of sub-blocks 8 h + 2 j0 .. + 3
    uint32_t q[8];
    #pragma unroll
    for (int i = 0; i < 8; ++i) q[i] = bw[4 + 8 * h + i];
    #pragma unroll
    for (int jj = 0; jj < 2; ++jj) {
        const int shift = 2 * (j0 + jj);
        #pragma unroll
        for (int hf = 0; hf < 2; ++hf) {   // positions l < 16, l >= 16: one scale each
            const uint32_t sb = (sw >> (8 * (2 * jj + hf))) & 0xFFu;
            const float a = d * (float)(sb & 15u), bm = dmin * (float)(sb >> 4);
            const float2 sc = make_float2(a, a), bi = make_float2(-bm, -bm);
            #pragma unroll
            for (int qi = 0; qi < 4; ++qi) {
                const int i = 4 * hf + qi;   // positions 4 i .. 4 i + 3
                decode4((q[i] >> shift) & 0x03030303u, sc, bi, out[16 * jj + 2 * i], out[16 * jj + 2 * i + 1]);
            }
        }
    }
}

// 64-K chunk cc (0..7) of a row's raw TQ1 unit: half cc % 2 of block cc / 2.
__device__ __forceinline__ void tq1_decode_chunk(const uint8_t *row, int cc, uint32_t out[32]) {
    const uint8_t *blk = row + 28 * (cc >> 1);
    if (cc & 1) tq1_decode64<1>(blk, out);
    else tq1_decode64<0>(blk, out);
}

// CPS: 64-K swizzle atoms per pipeline stage (1, or 2 for narrow token tiles,
// which halves the per-K barrier traffic of the single MMA thread).  FMT: the
// weight format (KQ_Q4_K or KQ_TQ1_G128; TQ1 dense only).
template <typename YT, bool ID, int CPS, int FMT>
__device__ __forceinline__ void gemm_body(const CUtensorMap &tmap_x, const CUtensorMap &tmap_w,
                                          const CUtensorMap &tmap_y, const GemmParams &p) {
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte alignment for the swizzled tiles
    uint8_t *smem = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);
    const int SA = p.a_stages, SB = p.b_stages, SR = p.raw_stages;
    uint8_t *b_ring = smem;                                    // SB x bn*128
    constexpr int UNIT_BYTES = RawUnit<FMT>::BYTES, UNIT_K = RawUnit<FMT>::K;
    constexpr int RAW_STAGE_BYTES = BM * UNIT_BYTES;
    uint8_t *raw_ring = b_ring + SB * p.b_stage_bytes;         // SR x 18 or 14 KB
    uint8_t *epi_stage = raw_ring + SR * RAW_STAGE_BYTES;      // EPI_STAGE_BYTES
    uint64_t *bars = reinterpret_cast<uint64_t *>(epi_stage + EPI_STAGE_BYTES);
    uint64_t *full_a = bars;                 // [SA] one decoder group (4 warps) -> MMA
    uint64_t *empty_a = full_a + SA;         // [SA] MMA -> decoders
    uint64_t *full_b = empty_a + SA;         // [SB] TMA bytes -> MMA
    uint64_t *empty_b = full_b + SB;         // [SB] MMA -> TMA
    uint64_t *raw_full = empty_b + SB;       // [RAW] TMA -> decoders
    uint64_t *raw_empty = raw_full + SR;     // [RAW] decoders -> TMA
    uint64_t *acc_full = raw_empty + SR;     // [2] MMA -> epilogue
    uint64_t *acc_empty = acc_full + 2;           // [2] epilogue -> MMA
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_empty + 2);
    int *s_rows = reinterpret_cast<int *>(bars + 128);  // expert-indexed: activation row per tile row
    if ((uint32_t)(reinterpret_cast<uint8_t *>(s_rows + MAX_BN) - smem_raw) > dynamic_smem_size()) {
        if (threadIdx.x == 0) atomicOr(p.err, ERR_BOUNDS);   // the host planned another layout: no work
        return;
    }

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int SPS = UNIT_K / (BK * CPS);   // stages per raw unit
    constexpr int DEC_WARPS_T = dec_warps<FMT>(), DEC_GROUPS_T = DEC_WARPS_T / 4;
    static_assert(DEC_GROUPS_T == 2 || DEC_GROUPS_T == 4, "decoder warps come in 2 or 4 groups of 4");
    const int nk = p.k / (BK * CPS);       // stages per tile

    if (threadIdx.x == 0) {
        for (int s = 0; s < SA; ++s) {
            mbar_init(&full_a[s], 4);
            mbar_init(&empty_a[s], 1);
        }
        for (int s = 0; s < SB; ++s) {
            mbar_init(&full_b[s], 1);
            mbar_init(&empty_b[s], 1);
        }
        for (int r = 0; r < SR; ++r) {
            mbar_init(&raw_full[r], 1);
            mbar_init(&raw_empty[r], DEC_WARPS_T);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], 4);
        }
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(tmem_slot, 512);
    if (warp == 0 && lane == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_x)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_w)) : "memory");
        if (p.y_tma)
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_y)) : "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    griddep_wait();
    // Work units: dense tiles, or (token tile, weight tile) pairs whose token
    // tiles the grouping step wrote on the device.
    const int units = ID ? *p.id_n_tiles * p.n_tiles : p.tiles;

    if (warp == RAW_WARP) {
        // ---------------- raw weight producer ----------------
        // Runs ahead of the decoders by the whole raw ring, independently of
        // the activation ring (narrow token tiles stream fresh weights).
        if (lane == 0) {
            uint32_t rslot = 0, rphase = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
                const Tile t = tile_at<ID>(p, u);
                for (int sb = 0; sb < p.k / UNIT_K; ++sb) {
                    ok = mbar_wait(&raw_empty[rslot], rphase ^ 1, p.err);
                    if (!ok) break;
                    mbar_arrive_expect_tx(&raw_full[rslot], RAW_STAGE_BYTES);
                    tma_load_3d(raw_ring + rslot * RAW_STAGE_BYTES, &tmap_w, sb * (UNIT_BYTES / RawUnit<FMT>::ELEM),
                                t.n0, t.e, &raw_full[rslot]);
                    if (++rslot == (uint32_t)SR) { rslot = 0; rphase ^= 1; }
                }
            }
        }
    } else if (warp == 0) {
        // ---------------- activation producer ----------------
        // Ring positions advance incrementally (no division in the issue
        // loop: this single thread must keep pace with the tensor core).
        // Expert-indexed tiles first gather their activation row numbers
        // (the whole warp, into s_rows; rows past the segment repeat its
        // first row and their outputs are dropped), then load the tile four
        // rows per gather.
        uint32_t slot = 0, phase = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
            const Tile t = tile_at<ID>(p, u);
            if constexpr (ID) {
                __syncwarp();  // lane 0 has issued every load of the previous tile
                for (int i = lane; i < p.bn; i += 32) {
                    int pr = p.perm[t.m0 + (i < t.rows ? i : 0)];
                    if (!KQ_DCHECK(pr >= 0 && pr < p.n_pairs, p.err)) pr = 0;
                    s_rows[i] = pr / p.top_k;
                }
                __syncwarp();
            }
            if (lane == 0) {
                for (int ks = 0; ks < nk; ++ks) {
                    ok = mbar_wait(&empty_b[slot], phase ^ 1, p.err);
                    if (!ok) break;
                    mbar_arrive_expect_tx(&full_b[slot], p.b_stage_bytes);
                    #pragma unroll
                    for (int c = 0; c < CPS; ++c) {   // one 64-K atom (bn rows x 128 B) each
                        uint8_t *dst = b_ring + slot * p.b_stage_bytes + c * p.bn * 128;
                        const int kx = (ks * CPS + c) * BK;
                        if constexpr (ID) {
                            for (int i = 0; i < p.bn; i += 4)
                                tma_gather4(dst + i * 128, &tmap_x, kx, s_rows[i], s_rows[i + 1], s_rows[i + 2],
                                            s_rows[i + 3], &full_b[slot]);
                        } else {
                            tma_load_2d(dst, &tmap_x, kx, t.m0, &full_b[slot]);
                        }
                    }
                    if (++slot == (uint32_t)SB) { slot = 0; phase ^= 1; }
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        // Per stage: wait for the activation tile's bytes and for the four
        // warps that decoded the weights, four MMAs of K = 16 (A: 8 TMEM
        // columns apart, B: 32 bytes apart in the swizzle atom), and one
        // commit per ring that frees the slots when the MMAs are done.
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(BM, p.bn);
            const uint64_t b_desc0 = sw128_desc(smem_addr(b_ring));
            const uint32_t b_step = (uint32_t)p.b_stage_bytes >> 4;
            uint32_t sa = 0, pa = 0, sb = 0, pb = 0;
            uint64_t bd = b_desc0;
            int tl = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++tl) {
                const int acc = tl % ACC_BUFS;
                ok = mbar_wait(&acc_empty[acc], ((tl / ACC_BUFS) & 1) ^ 1, p.err);
                if (!ok) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * 256);
                for (int ks = 0; ks < nk; ++ks) {
                    ok = mbar_wait(&full_b[sb], pb, p.err) && mbar_wait(&full_a[sa], pa, p.err);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t at = tmem_base + a_slot_col<CPS>(sa, p.a_col0);
                    #pragma unroll
                    for (int c = 0; c < CPS; ++c) {
                        const uint64_t bc = bd + (uint64_t)(c * ((p.bn * 128) >> 4));
                        mma_bf16_ts(d_tmem, at + 32 * c, bc, idesc, (ks > 0 || c > 0) ? 1u : 0u);
                        mma_bf16_ts(d_tmem, at + 32 * c + 8, bc + 2, idesc, 1u);
                        mma_bf16_ts(d_tmem, at + 32 * c + 16, bc + 4, idesc, 1u);
                        mma_bf16_ts(d_tmem, at + 32 * c + 24, bc + 6, idesc, 1u);
                    }
                    mma_commit(&empty_b[sb]);  // frees both slots once these MMAs finish
                    mma_commit(&empty_a[sa]);
                    if (++sb == (uint32_t)SB) {
                        sb = 0;
                        pb ^= 1;
                        bd = b_desc0;
                    } else {
                        bd += b_step;
                    }
                    if (++sa == (uint32_t)SA) { sa = 0; pa ^= 1; }
                }
                if (ok) mma_commit(&acc_full[acc]);
            }
        }
    } else if (warp < EPI_WARP0 + 4) {
        // ---------------- epilogue ----------------
        // Warp q drains TMEM lanes 32q..32q+31 (weight rows n0+32q..) 16
        // tokens at a time.  Dense outputs go through shared memory: the
        // chunk is written as [16 tokens][32 rows] and one TMA store moves it
        // (two buffers per warp, so converting the next chunk overlaps the
        // store of this one).  Expert-indexed outputs scatter rows and are
        // stored element by element.
        const int q = warp & 3;  // TMEM lane quadrant this warp may access
        YT *y = static_cast<YT *>(p.y);
        YT *stage = reinterpret_cast<YT *>(epi_stage) + (size_t)(warp - EPI_WARP0) * 2 * EPI_CHUNK_M * EPI_CHUNK_N;
        int sbuf = 0;
        int tl = 0;
        for (int u = blockIdx.x; u < units; u += gridDim.x, ++tl) {
            const int acc = tl % ACC_BUFS;
            const Tile t = tile_at<ID>(p, u);
            // warp-uniform outcome: the TMEM loads below are .sync.aligned
            if (!warp_wait(&acc_full[acc], (tl / ACC_BUFS) & 1, p.err)) break;
            tc_fence_after();
            const int n = t.n0 + 32 * q + lane;
            const uint32_t t_row = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(acc * 256);
            for (int c0 = 0; c0 < p.bn; c0 += 16) {
                uint32_t r[16];
                tmem_ld16(t_row + (uint32_t)c0, r);
                if (!ID && p.y_tma) {
                    if (c0 >= t.rows) continue;   // tokens past the end: nothing to store
                    if (lane == 0) bulk_wait_read_le1();   // this buffer's previous store has read it
                    __syncwarp();
                    YT *buf = stage + sbuf * EPI_CHUNK_M * EPI_CHUNK_N;
                    #pragma unroll
                    for (int j = 0; j < 16; ++j) store_out(buf + j * EPI_CHUNK_N + lane, __uint_as_float(r[j]));
                    fence_proxy_async_smem();
                    __syncwarp();
                    // the map clips rows past n and tokens past m
                    if (lane == 0 && t.n0 + 32 * q < p.n) tma_store_2d(&tmap_y, buf, t.n0 + 32 * q, t.m0 + c0);
                    sbuf ^= 1;
                } else if (n < p.n) {
                    #pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        if (c0 + j < t.rows) {
                            // output row: the activation row, or the (token, slot) pair
                            const int64_t m = ID ? (int64_t)__ldg(p.perm + t.m0 + c0 + j) : (int64_t)(t.m0 + c0 + j);
                            if (!ID || KQ_DCHECK(m >= 0 && m < p.n_pairs, p.err)) {
                                YT *dst = y + m * p.n + n;
                                const float v = __uint_as_float(r[j]);
                                if (ID && p.glu) store_out(dst, glu_activation(v, p.act) * load_out(dst));
                                else store_out(dst, v);
                            }
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[acc]);
        }
        if (lane == 0) bulk_wait_all();   // stores have read shared memory before the CTA exits
    } else {
        // ---------------- decoders ----------------
        // Group grp (four consecutive warps, one per TMEM lane quadrant)
        // decodes stage g when g % DEC_GROUPS_T == grp.  Lane l of a warp in
        // quadrant q owns weight row r = 32 q + l: per stage it reads the
        // row's 32 quant bytes of chunk cc = g % 4 (low nibbles: K positions
        // 0..31 of the stage = sub-block 2cc, high nibbles: K 32..63 =
        // sub-block 2cc+1) and writes 32 TMEM columns of its lane, column j
        // holding the bf16 pair at K positions 2j, 2j+1.
        const int grp = (warp - DEC_WARP0) >> 2;
        const int quad = warp & 3;
        const int r = 32 * quad + lane;
        const uint32_t t_lane = tmem_base + ((uint32_t)(32 * quad) << 16);
        uint32_t slot = 0, phase = 0, rs = 0, rph = 0;
        uint32_t g = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
            for (int sb = 0; sb < p.k / UNIT_K && ok; ++sb) {
                ok = warp_wait(&raw_full[rs], rph, p.err);
                if (!ok) break;
                const uint8_t *blk = raw_ring + rs * RAW_STAGE_BYTES + r * UNIT_BYTES;
                // Q4_K / Q5_K super-block header (fp16 d, dmin, packed 6-bit
                // scales and mins; unused by the other formats)
                const uint4 hd = (FMT == KQ_Q4_K || FMT == KQ_Q5_K) ? *reinterpret_cast<const uint4 *>(blk)
                                                                     : make_uint4(0u, 0u, 0u, 0u);
                const float d = half_f(hd.x), dmin = half_f(hd.x >> 16);
                // packed 6-bit scales / mins of sub-blocks 0..3 and 4..7
                const uint32_t sc_lo = hd.y & 0x3F3F3F3Fu, m_lo = hd.z & 0x3F3F3F3Fu;
                const uint32_t sc_hi = (hd.w & 0x0F0F0F0Fu) | ((hd.y >> 2) & 0x30303030u);
                const uint32_t m_hi = ((hd.w >> 4) & 0x0F0F0F0Fu) | ((hd.z >> 2) & 0x30303030u);
                // A rolled loop: the chunk position stays a runtime value and
                // the decode code is not copied per stage.  Instruction fetch
                // was the top stall of the unrolled TQ1 decoders (eight
                // chunk-specific copies); rolled, the TQ1 prefill went from
                // 167.9 to 136.3 us and the Q4_K one from 68.5 to 65.7 us.
                #pragma unroll 1
                for (int st = 0; st < SPS; ++st) {
                    if ((int)(g & (DEC_GROUPS_T - 1)) == grp) {
                        // warp-uniform outcome: the TMEM stores below are .sync.aligned
                        ok = warp_wait(&empty_a[slot], phase ^ 1, p.err);
                        if (!ok) break;
                        tc_fence_after();
                      #pragma unroll
                      for (int c = 0; c < CPS; ++c) {
                        const int cc = st * CPS + c;   // 64-K chunk of the raw unit
                        uint32_t out[32];
                        if constexpr (FMT == KQ_TQ1_G128) {
                            tq1_decode_chunk(blk, cc, out);
                        } else if constexpr (FMT == KQ_Q8_0) {
                            q8_0_decode_chunk(blk, cc, out);
                        } else if constexpr (FMT == KQ_Q2_K) {
                            q2_k_decode_chunk(blk, cc, out);
                        } else if constexpr (FMT == KQ_Q5_K) {
                            // chunk cc: low nibbles (sub-block 2cc) and high
                            // nibbles (2cc+1) of qs bytes 32cc.. at 48, each
                            // with its fifth bit, bit 2cc (+1) of qh byte l at 16
                            const uint32_t scw = cc < 2 ? sc_lo : sc_hi, mw = cc < 2 ? m_lo : m_hi;
                            const int b0 = (2 * cc) & 3;
                            const float ds_lo = d * byte_float(scw, b0), dm_lo = dmin * byte_float(mw, b0);
                            const float ds_hi = d * byte_float(scw, b0 + 1), dm_hi = dmin * byte_float(mw, b0 + 1);
                            const float2 sl = make_float2(ds_lo, ds_lo), bl = make_float2(-dm_lo, -dm_lo);
                            const float2 sh = make_float2(ds_hi, ds_hi), bh = make_float2(-dm_hi, -dm_hi);
                            const uint4 v0 = *reinterpret_cast<const uint4 *>(blk + 48 + 32 * cc);
                            const uint4 v1 = *reinterpret_cast<const uint4 *>(blk + 64 + 32 * cc);
                            const uint4 h0 = *reinterpret_cast<const uint4 *>(blk + 16);
                            const uint4 h1 = *reinterpret_cast<const uint4 *>(blk + 32);
                            const uint32_t qw[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
                            const uint32_t hw[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
                            #pragma unroll
                            for (int wd = 0; wd < 8; ++wd) {
                                const uint32_t lo = (qw[wd] & 0x0F0F0F0Fu) | (((hw[wd] >> (2 * cc)) & 0x01010101u) << 4);
                                const uint32_t hi =
                                    ((qw[wd] >> 4) & 0x0F0F0F0Fu) | (((hw[wd] >> (2 * cc + 1)) & 0x01010101u) << 4);
                                decode4(lo, sl, bl, out[2 * wd], out[2 * wd + 1]);
                                decode4(hi, sh, bh, out[16 + 2 * wd], out[17 + 2 * wd]);
                            }
                        } else {
                            const uint32_t scw = cc < 2 ? sc_lo : sc_hi, mw = cc < 2 ? m_lo : m_hi;
                            const int b0 = (2 * cc) & 3;
                            // exact products: d*sc (17 bits), dmin*m (17 bits); high
                            // nibbles arrive as 16*q, so their scale is divided by 16
                            const float ds_lo = d * byte_float(scw, b0), dm_lo = dmin * byte_float(mw, b0);
                            const float ds_hi = d * byte_float(scw, b0 + 1) * 0.0625f;
                            const float dm_hi = dmin * byte_float(mw, b0 + 1);
                            const float2 sl = make_float2(ds_lo, ds_lo), bl = make_float2(-dm_lo, -dm_lo);
                            const float2 sh = make_float2(ds_hi, ds_hi), bh = make_float2(-dm_hi, -dm_hi);
                            const uint4 v0 = *reinterpret_cast<const uint4 *>(blk + 16 + 32 * cc);
                            const uint4 v1 = *reinterpret_cast<const uint4 *>(blk + 32 + 32 * cc);
                            const uint32_t qw[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
                            #pragma unroll
                            for (int wd = 0; wd < 8; ++wd) {
                                decode4(qw[wd] & 0x0F0F0F0Fu, sl, bl, out[2 * wd], out[2 * wd + 1]);
                                decode4(qw[wd] & 0xF0F0F0F0u, sh, bh, out[16 + 2 * wd], out[17 + 2 * wd]);
                            }
                        }
                        tmem_st32(t_lane + a_slot_col<CPS>(slot, p.a_col0) + 32 * c, out);
                      }
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&full_a[slot]);
                    }
                    ++g;
                    if (++slot == (uint32_t)SA) { slot = 0; phase ^= 1; }
                }
                if (!ok) break;
                __syncwarp();
                if (lane == 0) mbar_arrive(&raw_empty[rs]);
                if (++rs == (uint32_t)SR) { rs = 0; rph ^= 1; }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    griddep_launch_dependents();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

template <typename YT, bool ID, int CPS>
__global__ void __launch_bounds__(num_threads<KQ_Q4_K>(), 1)
    gemm_q4k_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                    const __grid_constant__ CUtensorMap tmap_y, const GemmParams p) {
    gemm_body<YT, ID, CPS, KQ_Q4_K>(tmap_x, tmap_w, tmap_y, p);
}

template <typename YT, bool ID, int CPS>
__global__ void __launch_bounds__(num_threads<KQ_TQ1_G128>(), 1)
    gemm_tq1_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                    const __grid_constant__ CUtensorMap tmap_y, const GemmParams p) {
    gemm_body<YT, ID, CPS, KQ_TQ1_G128>(tmap_x, tmap_w, tmap_y, p);
}

template <typename YT, bool ID, int CPS>
__global__ void __launch_bounds__(num_threads<KQ_Q8_0>(), 1)
    gemm_q8_0_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                     const __grid_constant__ CUtensorMap tmap_y, const GemmParams p) {
    gemm_body<YT, ID, CPS, KQ_Q8_0>(tmap_x, tmap_w, tmap_y, p);
}

template <typename YT, bool ID, int CPS>
__global__ void __launch_bounds__(num_threads<KQ_Q2_K>(), 1)
    gemm_q2_k_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                     const __grid_constant__ CUtensorMap tmap_y, const GemmParams p) {
    gemm_body<YT, ID, CPS, KQ_Q2_K>(tmap_x, tmap_w, tmap_y, p);
}

template <typename YT, bool ID, int CPS>
__global__ void __launch_bounds__(num_threads<KQ_Q5_K>(), 1)
    gemm_q5_k_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                     const __grid_constant__ CUtensorMap tmap_y, const GemmParams p) {
    gemm_body<YT, ID, CPS, KQ_Q5_K>(tmap_x, tmap_w, tmap_y, p);
}

// ---------------------------------------------------------------- host side
// Choose BN (tokens per tile).  A stage of a tile costs about the larger of
// its MMAs (4 x BN/2 cycles for 128 x BN x 64) and the decode of its 128 x 64
// weights, which does not shrink with BN (about 400 cycles, measured): the
// cost of a shape is rounds of tiles over the SMs x that per-stage cost, so
// extra token tiles (each one decodes its weight tile again) must buy fewer
// rounds.  Ties go to the narrower tile.
int pick_bn(int m, int n_tiles, int sms) {
#ifdef KQ_GEMM_FORCE_BN
    return KQ_GEMM_FORCE_BN;
#endif
    constexpr double DECODE_CYCLES_PER_STAGE = 400.0, MMA_FIXED = 48.0;
    static const int cands[] = {192, 176, 160, 128, 112, 96, 80, 64, 48, 32, 16};
    int best = cands[0];
    double best_cost = 1e30;
    for (int bn : cands) {
        if (bn > 16 && bn >= 2 * m + 16) continue;  // far wider than the problem
        const int mt = (m + bn - 1) / bn;
        const long tiles = (long)mt * n_tiles;
        const long rounds = (tiles + sms - 1) / sms;
        const double stage = 2.0 * bn + MMA_FIXED > DECODE_CYCLES_PER_STAGE ? 2.0 * bn + MMA_FIXED
                                                                           : DECODE_CYCLES_PER_STAGE;
        const double cost = (double)rounds * stage;
        if (cost <= best_cost) {
            best_cost = cost;
            best = bn;
        }
    }
    return best;
}

// First TMEM column after an accumulator of bn columns (32-column aligned).
int a_col0_for(int bn) { return (bn + 31) / 32 * 32; }

// Ring depths: the A slots (32 TMEM columns each) that fit in the two gaps
// after the accumulators, and as many activation tiles as shared memory
// holds next to the raw ring (barriers and the row list take 2.25 KB).
int a_stages_for(int bn, int cps) {
    const int st = ACC_BUFS == 2 ? 2 * ((256 - a_col0_for(bn)) / (32 * cps)) : (512 - a_col0_for(bn)) / (32 * cps);
    return st < MAX_A_STAGES ? st : MAX_A_STAGES;
}
// Shared memory: activation ring first (up to ten stages next to KQ_GEMM_MIN_RAW raw
// slots), then as many raw slots as the rest holds (up to eight: narrow
// token tiles stream fresh weights, whose HBM latency needs depth).
constexpr int SMEM_RINGS = SMEM_BUDGET - 1024 - 2560 - EPI_STAGE_BYTES;  // less alignment, barriers, rows, epilogue
#ifndef KQ_GEMM_MIN_RAW
#define KQ_GEMM_MIN_RAW 2
#endif
int b_stages_for(int b_stage_bytes, int raw_bytes) {
    const int st = (SMEM_RINGS - KQ_GEMM_MIN_RAW * raw_bytes) / b_stage_bytes;
    return st < MAX_B_STAGES ? st : MAX_B_STAGES;
}
int raw_stages_for(int b_stage_bytes, int b_stages, int raw_bytes) {
    const int st = (SMEM_RINGS - b_stages * b_stage_bytes) / raw_bytes;
    return st < MAX_RAW_STAGES ? st : MAX_RAW_STAGES;
}

}  // namespace

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// Activations [rows, k] bf16: 64-column boxes of box_rows rows, 128-byte swizzle.
bool encode_x_map(CUtensorMap *m, const void *x, int64_t rows, int64_t k, int box_rows) {
    cuuint64_t dims[2] = {(cuuint64_t)k, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)k * 2};
    cuuint32_t box[2] = {BK, (cuuint32_t)box_rows};
    cuuint32_t es[2] = {1, 1};
    return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(x), dims, strides, box,
                       es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Raw rows of one or more experts: (row bytes, rows, experts), one raw unit
// column (a Q4_K super-block, or four TQ1_G128 blocks) of BM rows per box.
bool encode_w_map(CUtensorMap *m, const void *w, int64_t n, int64_t k, int64_t n_experts,
                  int64_t expert_stride, int type) {
    const int ub = raw_unit_bytes(type), uk = raw_unit_k(type);
    const int el = (type == KQ_Q8_0 || type == KQ_Q2_K) ? 2 : 1;   // bytes per element of the map
    if (k % uk) return false;
    const int64_t rb = (k / uk) * ub;
    cuuint64_t dims[3] = {(cuuint64_t)(rb / el), (cuuint64_t)n, (cuuint64_t)n_experts};
    cuuint64_t strides[2] = {(cuuint64_t)rb, (cuuint64_t)expert_stride};
    cuuint32_t box[3] = {(cuuint32_t)(ub / el), BM, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return encode_fn()(m, el == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 3,
                       const_cast<void *>(w), dims, strides, box, es,
                       CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool gemm_supported(int type, int64_t n, int64_t k, int x_dtype, int y_dtype, bool expert_indexed) {
    if (x_dtype != KQ_BF16) return false;
    if (y_dtype != KQ_F32 && y_dtype != KQ_BF16) return false;
    if (k > (1 << 24) || n < 1 || n > (1 << 30)) return false;
    if (type == KQ_Q4_K) {
        if (k % 256) return false;
    } else if (type == KQ_TQ1_G128 && !expert_indexed) {
        if (k % 512) return false;   // the row pitch and box rows must be multiples of 16 bytes
    } else if (type == KQ_Q8_0) {
        if (k % 256) return false;   // likewise: eight 34-byte blocks are 272 bytes
    } else if (type == KQ_Q2_K) {
        if (k % 1024) return false;   // and four 84-byte super-blocks are 336 bytes
    } else if (type == KQ_Q5_K) {
        if (k % 256) return false;
    } else {
        return false;
    }
    return encode_fn() != nullptr;
}

namespace {

// Dense output [m, n] of 2- or 4-byte elements: boxes of 32 rows (n) x 16
// tokens (m) for the epilogue's stores.  false if the row pitch is not a
// multiple of 16 bytes (the epilogue then stores element by element).
bool encode_y_map(CUtensorMap *mp, void *y, int64_t m, int64_t n, int ydt) {
    const int es = ydt == KQ_F32 ? 4 : 2;
    if ((n * es) % 16) return false;
    cuuint64_t dims[2] = {(cuuint64_t)n, (cuuint64_t)m};
    cuuint64_t strides[1] = {(cuuint64_t)(n * es)};
    cuuint32_t box[2] = {EPI_CHUNK_N, EPI_CHUNK_M};
    cuuint32_t estr[2] = {1, 1};
    return encode_fn()(mp, ydt == KQ_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                       y, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                       CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 64-K atoms per stage: two for narrow token tiles (their MMAs are short, so
// the single MMA thread's per-stage waits and commits dominate), else one.
int cps_for(int bn) { return bn <= 64 ? 2 : 1; }

bool fill_ring(GemmParams *p, int cps, int type) {
    const int rbytes = raw_stage_bytes(type);
    p->b_stage_bytes = p->bn * 128 * cps;
    p->a_stages = a_stages_for(p->bn, cps);
    p->b_stages = b_stages_for(p->b_stage_bytes, rbytes);
    p->raw_stages = raw_stages_for(p->b_stage_bytes, p->b_stages, rbytes);
    p->a_col0 = a_col0_for(p->bn);
    return p->bn <= MAX_BN && p->bn % 16 == 0 && p->a_stages >= 2 && p->b_stages >= 2 && p->raw_stages >= 2;
}

template <typename YT, bool ID, int CPS, int FMT = KQ_Q4_K>
cudaError_t launch_kernel(const CUtensorMap &tx, const CUtensorMap &tw, const CUtensorMap &ty,
                          const GemmParams &p, int grid, cudaStream_t s) {
    // alignment slack, activation ring, raw ring, epilogue staging, barriers
    // (384 B) and the expert-indexed row list (768 B)
    const size_t smem = 1024 + (size_t)p.b_stages * p.b_stage_bytes +
                        (size_t)p.raw_stages * raw_stage_bytes(FMT) + EPI_STAGE_BYTES + 2560;
    void (*kern)(CUtensorMap, CUtensorMap, CUtensorMap, GemmParams);
    if constexpr (FMT == KQ_TQ1_G128) kern = gemm_tq1_kernel<YT, ID, CPS>;
    else if constexpr (FMT == KQ_Q8_0) kern = gemm_q8_0_kernel<YT, ID, CPS>;
    else if constexpr (FMT == KQ_Q2_K) kern = gemm_q2_k_kernel<YT, ID, CPS>;
    else if constexpr (FMT == KQ_Q5_K) kern = gemm_q5_k_kernel<YT, ID, CPS>;
    else kern = gemm_q4k_kernel<YT, ID, CPS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(num_threads<FMT>());
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, tx, tw, ty, p);
}

}  // namespace

cudaError_t launch_gemm(int type, const void *w, int64_t n, int64_t k, const void *x, int64_t m,
                        void *y, int ydt, cudaStream_t s) {
    if (!encode_fn() || m < 1 || m > (1 << 30)) return cudaErrorNotSupported;
    if (type != KQ_Q4_K && type != KQ_TQ1_G128 && type != KQ_Q8_0 && type != KQ_Q2_K && type != KQ_Q5_K)
        return cudaErrorNotSupported;
    const int sms = sm_count();
    GemmParams p = {};
    p.n = (int)n; p.k = (int)k; p.m = (int)m;
    p.n_tiles = (int)((n + BM - 1) / BM);
    p.bn = pick_bn((int)m, p.n_tiles, sms);
    p.m_tiles = (int)((m + p.bn - 1) / p.bn);
    p.tiles = p.n_tiles * p.m_tiles;
    const int cps = cps_for(p.bn);
    if (!fill_ring(&p, cps, type)) return cudaErrorNotSupported;
    p.y = y;
    p.err = error_word();
    CUtensorMap tx, tw, ty;
    const int64_t row_bytes = (k / raw_unit_k(type)) * raw_unit_bytes(type);
    if (!encode_x_map(&tx, x, m, k, p.bn) || !encode_w_map(&tw, w, n, k, 1, n * row_bytes, type))
        return cudaErrorInvalidValue;
    p.y_tma = encode_y_map(&ty, y, m, n, ydt) ? 1 : 0;
    if (!p.y_tma) ty = tx;   // unused
    const int grid = p.tiles < sms ? p.tiles : sms;
    if (type == KQ_TQ1_G128) {
        if (cps == 2)
            return ydt == KQ_F32 ? launch_kernel<float, false, 2, KQ_TQ1_G128>(tx, tw, ty, p, grid, s)
                                 : launch_kernel<__nv_bfloat16, false, 2, KQ_TQ1_G128>(tx, tw, ty, p, grid, s);
        return ydt == KQ_F32 ? launch_kernel<float, false, 1, KQ_TQ1_G128>(tx, tw, ty, p, grid, s)
                             : launch_kernel<__nv_bfloat16, false, 1, KQ_TQ1_G128>(tx, tw, ty, p, grid, s);
    }
    if (type == KQ_Q8_0) {
        if (cps == 2)
            return ydt == KQ_F32 ? launch_kernel<float, false, 2, KQ_Q8_0>(tx, tw, ty, p, grid, s)
                                 : launch_kernel<__nv_bfloat16, false, 2, KQ_Q8_0>(tx, tw, ty, p, grid, s);
        return ydt == KQ_F32 ? launch_kernel<float, false, 1, KQ_Q8_0>(tx, tw, ty, p, grid, s)
                             : launch_kernel<__nv_bfloat16, false, 1, KQ_Q8_0>(tx, tw, ty, p, grid, s);
    }
    if (type == KQ_Q2_K) {
        if (cps == 2)
            return ydt == KQ_F32 ? launch_kernel<float, false, 2, KQ_Q2_K>(tx, tw, ty, p, grid, s)
                                 : launch_kernel<__nv_bfloat16, false, 2, KQ_Q2_K>(tx, tw, ty, p, grid, s);
        return ydt == KQ_F32 ? launch_kernel<float, false, 1, KQ_Q2_K>(tx, tw, ty, p, grid, s)
                             : launch_kernel<__nv_bfloat16, false, 1, KQ_Q2_K>(tx, tw, ty, p, grid, s);
    }
    if (type == KQ_Q5_K) {
        if (cps == 2)
            return ydt == KQ_F32 ? launch_kernel<float, false, 2, KQ_Q5_K>(tx, tw, ty, p, grid, s)
                                 : launch_kernel<__nv_bfloat16, false, 2, KQ_Q5_K>(tx, tw, ty, p, grid, s);
        return ydt == KQ_F32 ? launch_kernel<float, false, 1, KQ_Q5_K>(tx, tw, ty, p, grid, s)
                             : launch_kernel<__nv_bfloat16, false, 1, KQ_Q5_K>(tx, tw, ty, p, grid, s);
    }
    if (cps == 2)
        return ydt == KQ_F32 ? launch_kernel<float, false, 2>(tx, tw, ty, p, grid, s)
                             : launch_kernel<__nv_bfloat16, false, 2>(tx, tw, ty, p, grid, s);
    return ydt == KQ_F32 ? launch_kernel<float, false, 1>(tx, tw, ty, p, grid, s)
                         : launch_kernel<__nv_bfloat16, false, 1>(tx, tw, ty, p, grid, s);
}

int gemm_id_bn(int64_t n_tokens, int64_t top_k, int64_t n_experts) {
    // about 1.5x the mean number of pairs per expert, in steps of 16
    const int64_t pairs = n_tokens * top_k;
    int64_t bn = (3 * pairs / (2 * n_experts) + 15) / 16 * 16;
    if (bn < 16) bn = 16;
    if (bn > 176) bn = 176;
    return (int)bn;
}

namespace {

template <int FMT>
cudaError_t launch_id_fmt(const CUtensorMap &tx, const CUtensorMap &tw, const GemmParams &p, int grid, int cps,
                          int ydt, cudaStream_t s) {
    if (cps == 2)
        return ydt == KQ_F32 ? launch_kernel<float, true, 2, FMT>(tx, tw, tx, p, grid, s)
                             : launch_kernel<__nv_bfloat16, true, 2, FMT>(tx, tw, tx, p, grid, s);
    return ydt == KQ_F32 ? launch_kernel<float, true, 1, FMT>(tx, tw, tx, p, grid, s)
                         : launch_kernel<__nv_bfloat16, true, 1, FMT>(tx, tw, tx, p, grid, s);
}

}  // namespace

cudaError_t launch_gemm_id(const IdArgs &a, int bn, cudaStream_t s, bool glu_combine) {
    if (!encode_fn()) return cudaErrorNotSupported;
    const int sms = sm_count();
    GemmParams p = {};
    p.n = (int)a.n; p.k = (int)a.k; p.m = (int)a.n_tokens;
    p.n_tiles = (int)((a.n + BM - 1) / BM);
    p.bn = bn;
    if (a.type != KQ_Q4_K && a.type != KQ_Q8_0 && a.type != KQ_Q2_K && a.type != KQ_Q5_K)
        return cudaErrorNotSupported;
    const int cps = cps_for(bn);
    if (!fill_ring(&p, cps, a.type)) return cudaErrorNotSupported;
    p.y = a.y;
    p.err = error_word();
    p.perm = a.perm;
    p.offsets = a.offsets;
    p.id_tiles = reinterpret_cast<const int2 *>(a.tiles);
    p.id_n_tiles = a.n_tiles;
    p.top_k = a.x_div();
    p.n_pairs = (int)(a.n_tokens * a.top_k);
    p.n_experts = (int)a.n_experts;
    p.glu = glu_combine ? 1 : 0;
    p.act = a.act;
    CUtensorMap tx, tw;
    if (!encode_x_map(&tx, a.x, a.x_rows(), a.k, 1) ||
        !encode_w_map(&tw, a.w, a.n, a.k, a.n_experts, a.expert_stride, (int)a.type))
        return cudaErrorInvalidValue;
    // persistent grid: the number of token tiles is only known on the device
    const int64_t max_units = (a.n_tokens * a.top_k / bn + a.n_experts) * p.n_tiles;
    const int grid = (int)(max_units < sms ? max_units : sms);
    switch (a.type) {
    case KQ_Q8_0: return launch_id_fmt<KQ_Q8_0>(tx, tw, p, grid, cps, a.y_dtype, s);
    case KQ_Q2_K: return launch_id_fmt<KQ_Q2_K>(tx, tw, p, grid, cps, a.y_dtype, s);
    case KQ_Q5_K: return launch_id_fmt<KQ_Q5_K>(tx, tw, p, grid, cps, a.y_dtype, s);
    default: return launch_id_fmt<KQ_Q4_K>(tx, tw, p, grid, cps, a.y_dtype, s);
    }
}

}  // namespace kq
