// kq_moe_mma.cu -- expert-indexed Q4_K product for few routed pairs per
// expert, on the tensor cores (bf16 activations).
//
// The product of mlx-native `quantized_matmul_id_ggml` / mlx-kquant
// `gather_qmm` (y[t][s] = x[t] @ dequant(W_e)^T, e = ids[t][s]) when every
// expert has only a handful of routed pairs, the decode step of a
// mixture-of-experts layer.  There the weights dominate the bytes, each
// expert's rows are read once, and the work is to decode them fast enough
// to keep up with HBM.  A Q4_K weight is d*sc_j*q - dmin*m_j with q a 4-bit
// code and (sc_j, m_j) the scale and min of its 32-weight sub-block j, so
//
//   sum_k w_k x_k = d*sc_j * sum_k q_k x_k - dmin*m_j * sum_k x_k   (per sub-block)
//
// and the codes alone can go through the tensor core, the scales being
// applied once per (row, sub-block, token) afterwards:
//
//  * Decoder threads (lane = TMEM lane = weight row) write the codes of one
//    256-weight super-block as bf16 (128 + q: the nibble ORed into the
//    mantissa of 128.0, exact) straight into tensor memory; no scale
//    arithmetic per weight.
//  * The MMA (tcgen05 kind::f16, M = 128 rows, N = 16 pairs, A from TMEM, B
//    = the pairs' activations in shared memory) runs each 32-weight
//    sub-block into an accumulator of its own: D_j = sum (128 + q) x.
//  * Epilogue threads (lane = row again) read the eight accumulators and add
//    d*sc_j * D_j - (128*d*sc_j + dmin*m_j) * S_j to the row's outputs, S_j
//    the activations' sum over the sub-block (computed once per token tile).
//
// Work units are (token tile of one expert's pairs, 128-row tile); a CTA
// per SM takes a contiguous range of units, so consecutive units share a
// token tile, whose activations stay in shared memory (16 MMA rows x K,
// 128-byte swizzle) until the tile changes.  The epilogue warps fill the
// tile with plain loads and compute its exact sub-block sums in the same
// pass: bf16 activations as they are (16 tokens a tile), fp32 ones as a
// bf16 high row and a bf16 low row per token (8 tokens a tile; the MMA sums
// both, so the product keeps fp32 accuracy).  Raw super-blocks stream
// through a ring by TMA (several super-blocks of the tile's 128 rows per
// slot).  Warp roles: 0 raw producer, 1 MMA issuer (and TMEM owner), 2 pair
// list, 4..7 epilogue (warp 4+q reads TMEM lanes 32q..), 8..15 decoders
// (two per lane quadrant, half a super-block each).  TMEM: accumulators at
// columns 0 and 128 (8 sub-blocks x 16 columns, two stages in flight), A
// slots at 256 and 384 (256 codes of 128 rows each).  Fused GLU: each unit
// runs the gate stack's stages, then the up stack's, into two sets of row
// sums.  Dense mode: one matrix, activation rows in tiles, no grouping.
// What bounds it (measured): a tcgen05.mma of M = 128, K = 16 costs a fixed
// ~83 cycles whatever N is, so 16 of them per super-block set the pace.
// Every wait is bounded (kq_ptx.cuh); activations that are not finite make
// the epilogue compute that token tile exactly in fp32 instead.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "kq_decode.cuh"
#include "kq_ptx.cuh"
#include "kq_tc.cuh"
#include "kq_launch.h"

namespace kq {

namespace {

constexpr int MM_BM = 128;                        // weight rows per unit (MMA M)
constexpr int MM_BN = 16;                         // pairs per token tile (MMA N)
constexpr int MM_SB = 144;                        // Q4_K super-block bytes
constexpr int MM_RAW_BYTES = MM_BM * MM_SB;       // one raw stage: 128 rows x one super-block
constexpr int MM_THREADS = 512;
constexpr int MM_RAW_WARP = 0, MM_MMA_WARP = 1, MM_X_WARP = 2, MM_EPI_WARP0 = 4, MM_DEC_WARP0 = 8;
constexpr int MM_MAX_K = 4096;
constexpr int MM_SMEM_LIMIT = 232448;             // dynamic shared memory of one CTA
constexpr uint32_t MM_ACC_COL = 0, MM_A_COL = 256;  // TMEM columns: accumulators, A slots

struct MoeMmaParams {
    int n, k, nk;                 // weight rows, K, super-blocks per row
    int n_row_tiles;              // ceil(n / 128)
    int raw_slots;                // ring slots, each spb super-blocks of the unit's 128 rows
    int spb;
    int x_div;                    // pair p reads activation row p / x_div
    int n_pairs, n_experts;
    const int32_t *perm, *offsets;
    const int2 *tiles;            // (expert, first position in perm) per token tile
    const int32_t *n_tiles;
    void *y;
    unsigned int *err;
    int glu, act;                 // fused GLU: each unit runs the gate stack, then the up stack
    int dense_m;                  // > 0: no grouping, activation rows 0..dense_m-1 of one matrix
    const void *x;                // activations [rows][k], bf16 or (x32) fp32
    int x32;                      // fp32 activations: two MMA rows per token (bf16 high and low parts)
    int tpt;                      // tokens per tile: 16, or 8 (fp32 activations, or the int8 form)
};

// Shared-memory layout, bytes from the 1024-aligned base.
struct MmLayout {
    int x, raw, s, sx, pairs, bars, total;
};
__host__ __device__ inline MmLayout mm_layout(int k, int raw_slots, int spb, bool i8) {
    MmLayout l;
    int off = 0;
    l.x = off;     off += (i8 ? 16 : 32) * k;               // 16 rows x K (bf16: 64-K atoms; int8: 128-K atoms; 2 KB each)
    l.raw = off;   off += raw_slots * spb * MM_RAW_BYTES;
    l.s = off;     off += 2 * (k / 32) * MM_BN * 4;         // two tiles' sub-block sums [K/32][16]
    l.sx = off;    off += i8 ? 2 * (k / 32) * MM_BN * 4 : 0;   // int8 form: the codes' scales [K/32][16]
    l.pairs = off; off += 4 * MM_BN * 4 + 2 * 4 + 2 * 4;    // pair ids and x rows [2][16] each, counts [2], flags [2]
    off = (off + 7) / 8 * 8;
    l.bars = off;  off += (2 * raw_slots + 9) * 8 + 8;      // barriers and the TMEM address
    l.total = off + 1024;                                   // alignment slack
    return l;
}

// Four codes (bytes 0..3 of v, each < 16) -> two bf16x2 words of 128 + q.
__device__ __forceinline__ void codes4(uint32_t v, uint32_t &w01, uint32_t &w23) {
    w01 = __byte_perm(v, 0x43434343u, 0x4140);
    w23 = __byte_perm(v, 0x43434343u, 0x4342);
}

__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

// Byte i of w as an exact float.
__device__ __forceinline__ float mm_byte_f(uint32_t w, int i) {
    return __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7440u | (uint32_t)i)) - 8388608.0f;
}

// Activation (row t, column k) of the swizzled tile: 64-column atoms of 16
// rows x 128 bytes; 16-byte chunk c of row t sits at chunk c ^ (t & 7) (the
// layout the MMA's 128-byte-swizzle descriptor reads).
__device__ __forceinline__ uint8_t *x_tile_w(uint8_t *xt, int t, int k) {
    return xt + (k >> 6) * 2048 + t * 128 + ((((k & 63) >> 3) ^ (t & 7)) << 4);
}
// The int8 form of the tile: 128-column atoms (one byte an element).
__device__ __forceinline__ uint8_t *x_tile_w8(uint8_t *xt, int t, int k) {
    return xt + (k >> 7) * 2048 + t * 128 + ((((k & 127) >> 4) ^ (t & 7)) << 4);
}

// D (TMEM, s32) += A (TMEM, u8) * B (shared memory, s8), K = 32.
__device__ __forceinline__ void mma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Instruction descriptor, kind::i8: u8 A, s8 B (K-major), s32 D.
__host__ __device__ constexpr uint32_t idesc_u8s8(int m, int n) {
    return (2u << 4) | (0u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

}  // namespace

// I8: the int8 form -- 4-bit codes as u8 and 14-bit activation codes as
// two s8 rows per token (high = c >> 7, low = c & 127, so c = 128 high +
// low), one K = 32 MMA per sub-block instead of two K = 16 ones.
template <typename YT, bool I8>
__global__ void __launch_bounds__(MM_THREADS, 1)
    moe_mma_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_w2,
                   const MoeMmaParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);
    const MmLayout lay = mm_layout(p.k, p.raw_slots, p.spb, I8);
    const int R = p.raw_slots, SPB = p.spb;
    const int slot_bytes = SPB * MM_RAW_BYTES;
    uint8_t *x_tile = smem + lay.x;
    uint8_t *raw = smem + lay.raw;
    float *s_sum = reinterpret_cast<float *>(smem + lay.s);          // [2][K/32][16]
    float *s_xsc = reinterpret_cast<float *>(smem + lay.sx);         // [2][K/32][16] (int8 form)
    int *s_pair = reinterpret_cast<int *>(smem + lay.pairs);         // [2][16] output row (pair) per token
    int *s_xrow = s_pair + 2 * MM_BN;                                // [2][16] activation row per token
    int *s_ntok = s_xrow + 2 * MM_BN;                                // [2]
    int *s_nf = s_ntok + 2;                                          // [2] non-finite activations
    uint64_t *raw_full = reinterpret_cast<uint64_t *>(smem + lay.bars);
    uint64_t *raw_empty = raw_full + R;
    uint64_t *a_full = raw_empty + R;      // [2] decoders -> MMA: codes in the A slot
    uint64_t *mma_done = a_full + 2;       // [2] MMA -> epilogue and decoders: accumulators ready, A slot free
    uint64_t *acc_empty = mma_done + 2;    // [2] epilogue -> MMA: the accumulators are read
    uint64_t *x_full = acc_empty + 2;      // epilogue warps -> MMA, themselves: tile and sums written
    uint64_t *x_empty = x_full + 1;        // MMA and epilogue -> loader: done with the tile
    uint64_t *x_meta = x_empty + 1;        // loader -> epilogue warps: the tile's pair list
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(x_meta + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if ((uint32_t)(smem - smem_raw) + (uint32_t)lay.total - 1024u > dynamic_smem_size()) {
        if (threadIdx.x == 0) atomicOr(p.err, ERR_BOUNDS);   // the host planned another layout: no work
        return;
    }
    if (threadIdx.x == 0) {
        for (int r = 0; r < R; ++r) {
            mbar_init(&raw_full[r], 1);
            mbar_init(&raw_empty[r], 12);   // 8 decode warps, 4 epilogue warps
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&a_full[b], 8);
            mbar_init(&mma_done[b], 1);
            mbar_init(&acc_empty[b], 4);
        }
        mbar_init(x_full, 4);               // the 4 epilogue warps
        mbar_init(x_empty, 5);              // the MMA commit and the 4 epilogue warps
        mbar_init(x_meta, 1);
        fence_mbar_init();
    }
    if (warp == MM_MMA_WARP) tmem_alloc(tmem_slot, 512);
    if (warp == MM_RAW_WARP && lane == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_w)) : "memory");
        if (p.glu) asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_w2)) : "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    griddep_wait();   // the grouping and the tile list come from the preceding kernels

    const int nrt = p.n_row_tiles, nk = p.nk;
    const int ns = p.glu ? 2 * nk : nk;   // stages per unit (GLU: gate stages, then up stages)
    const int tpt = p.tpt;
    const int n_tok_tiles = p.dense_m > 0 ? (p.dense_m + tpt - 1) / tpt : *p.n_tiles;
    const int total = n_tok_tiles * nrt;
    const int u0 = (int)((int64_t)total * blockIdx.x / gridDim.x);
    const int u1 = (int)((int64_t)total * (blockIdx.x + 1) / gridDim.x);
    // Token tile -> (expert, first position in perm, pairs); KQ_DEBUG: a tile
    // outside the grouping becomes an empty tile of expert 0.
    auto tile_info = [&](int tile, int &e, int &m0, int &rows) {
        if (p.dense_m > 0) {
            e = 0;
            m0 = tile * tpt;
            rows = min(tpt, p.dense_m - m0);
            return;
        }
        const int2 tt = p.tiles[tile];
        const bool ok = KQ_DCHECK(tt.x >= 0 && tt.x < p.n_experts && tt.y >= 0 && tt.y < p.n_pairs &&
                                      p.offsets[tt.x + 1] <= p.n_pairs, p.err);
        e = ok ? tt.x : 0;
        m0 = ok ? tt.y : 0;
        rows = ok ? min(tpt, p.offsets[tt.x + 1] - tt.y) : 0;
    };

    if (warp == MM_RAW_WARP) {
        // ---------------- raw super-block producer ----------------
        if (lane == 0) {
            uint32_t g = 0;
            bool ok = true;
            for (int u = u0; u < u1 && ok; ++u) {
                int e, m0, rows;
                tile_info(u / nrt, e, m0, rows);
                const int n0 = (u % nrt) * MM_BM;
                // one ring slot per spb super-blocks of a matrix (the GLU's
                // gate and up stacks fill separate slots)
                for (int mat = 0; mat < ns / nk && ok; ++mat) {
                    for (int sb0 = 0; sb0 < nk; sb0 += SPB, ++g) {
                        const uint32_t slot = g % (uint32_t)R, ph = (g / (uint32_t)R) & 1u;
                        ok = mbar_wait(&raw_empty[slot], ph ^ 1u, p.err);
                        if (!ok) break;
                        mbar_arrive_expect_tx(&raw_full[slot], (uint32_t)slot_bytes);
                        tma_load_4d(raw + slot * slot_bytes, mat == 0 ? &tmap_w : &tmap_w2, 0, sb0, n0, e,
                                    &raw_full[slot]);
                    }
                }
            }
        }
    } else if (warp == MM_X_WARP) {
        // ---------------- pair list ----------------
        // When the token tile changes: wait until the previous tile's MMAs
        // and epilogues are done with the tile, then publish its pair ids
        // and activation rows for the epilogue warps, which load the tile.
        if (lane == 0) {
            int xt = 0, prev = -1;
            bool ok = true;
            for (int u = u0; u < u1 && ok; ++u) {
                const int tile = u / nrt;
                if (tile == prev) continue;
                prev = tile;
                if (xt > 0) {
                    ok = mbar_wait(x_empty, (uint32_t)(xt - 1) & 1u, p.err);
                    if (!ok) break;
                }
                int e, m0, rows;
                tile_info(tile, e, m0, rows);
                const int buf = xt & 1;
                for (int i = 0; i < tpt; ++i) {
                    int pr = -1;
                    if (i < rows) {
                        pr = p.dense_m > 0 ? m0 + i : p.perm[m0 + i];
                        if (!KQ_DCHECK(pr >= 0 && pr < p.n_pairs, p.err)) pr = -1;
                    }
                    s_pair[buf * MM_BN + i] = pr;
                    s_xrow[buf * MM_BN + i] = pr >= 0 ? pr / p.x_div : -1;
                }
                s_ntok[buf] = rows;
                s_nf[buf] = 0;
                mbar_arrive(x_meta);
                ++xt;
            }
        }
    } else if (warp == MM_MMA_WARP) {
        // ---------------- MMA issuer ----------------
        // Per stage (one super-block): eight sub-blocks, each two MMAs of
        // K = 16 into its own 16-column accumulator; one commit frees the A
        // slot and publishes the accumulators.
        if (lane == 0) {
            const uint32_t idesc = I8 ? idesc_u8s8(MM_BM, MM_BN) : idesc_bf16(MM_BM, MM_BN);
            const uint64_t xdesc0 = sw128_desc(smem_addr(x_tile));
            uint32_t g = 0;
            int xt = 0, prev = -1;
            bool ok = true;
            for (int u = u0; u < u1 && ok; ++u) {
                const int tile = u / nrt;
                if (tile != prev) {
                    if (xt > 0) mma_commit(x_empty);   // once the previous tile's MMAs are done
                    ok = mbar_wait(x_full, (uint32_t)xt & 1u, p.err);
                    if (!ok) break;
                    prev = tile;
                    ++xt;
                }
                for (int s = 0; s < ns; ++s, ++g) {
                    const uint32_t b = g & 1u;
                    ok = mbar_wait(&acc_empty[b], ((g >> 1) & 1u) ^ 1u, p.err) &&
                         mbar_wait(&a_full[b], (g >> 1) & 1u, p.err);
                    if (!ok) break;
                    tc_fence_after();
                    #pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int kidx = 256 * (s % nk) + 32 * j;     // first K of the sub-block
                        const uint32_t d = tmem_base + MM_ACC_COL + b * 128u + 16u * j;
                        if constexpr (I8) {
                            // one K = 32 MMA: 8 TMEM columns of codes, 32 bytes of the 128-K atom
                            const uint64_t bd = xdesc0 + (uint64_t)((kidx >> 7) * (2048 >> 4) + ((kidx & 127) >> 4));
                            mma_i8_ts(d, tmem_base + MM_A_COL + b * 128u + 8u * j, bd, idesc, 0u);
                        } else {
                            const uint64_t bd = xdesc0 + (uint64_t)((kidx >> 6) * (2048 >> 4) + ((kidx & 63) >> 3));
                            const uint32_t a = tmem_base + MM_A_COL + b * 128u + 16u * j;
                            mma_bf16_ts(d, a, bd, idesc, 0u);
                            mma_bf16_ts(d, a + 8, bd + 2, idesc, 1u);
                        }
                    }
                    mma_commit(&mma_done[b]);
                }
            }
        }
    } else if (warp >= MM_EPI_WARP0 && warp < MM_EPI_WARP0 + 4) {
        // ---------------- epilogue warps ----------------
        // Lane l of warp 4+q owns weight row 32q + l of the unit (TMEM lane
        // 32q + l).  Per token tile: the activations into the swizzled tile
        // (bf16 as they are; fp32 as a bf16 high row and a bf16 low row per
        // token) and their exact sub-block sums S (thread i of the 128 takes
        // (token, sub-block) items i, i + 128, ...).  Per stage: the
        // row's scales from the raw slot, applied to the eight sub-block
        // accumulators once the stage's MMAs are done; then the accumulator
        // and the raw slot are released.
        const int q = warp & 3, r = 32 * q + lane, ti = threadIdx.x - 32 * MM_EPI_WARP0;
        const uint32_t t_lane = tmem_base + ((uint32_t)(32 * q) << 16);
        const int nsub = p.k / 32;
        YT *y = static_cast<YT *>(p.y);
        uint32_t g = 0, L = 0;   // stages and raw ring slots consumed
        int xt = 0, prev = -1, buf = 0, ntok = 0;
        bool nf = false;
        bool ok = true;
        float acc[MM_BN];     // the row's outputs (GLU: the up projection)
        float accg[MM_BN];    // GLU: the gate projection
        float a[8], c[8];     // the stage's d*sc_j and 128*d*sc_j + dmin*m_j
        float dm[8];          // and dmin*m_j
        auto apply = [&](float (&A)[MM_BN], uint32_t b, int sp) {
            const float *sb = s_sum + (buf * nsub + 8 * (sp % nk)) * MM_BN;
            if constexpr (I8) {
                // columns 2t and 2t+1: token t's high and low code rows (int32)
                const float *xs = s_xsc + (buf * nsub + 8 * (sp % nk)) * MM_BN;
                #pragma unroll
                for (int tg = 0; tg < MM_BN / 4; ++tg) {
                    if (2 * tg >= ntok) break;   // warp-uniform
                    uint32_t dv[32];
                    tmem_ld4x8(t_lane + MM_ACC_COL + b * 128u + 4u * tg, dv);
                    #pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const float2 sv = *reinterpret_cast<const float2 *>(sb + j * MM_BN + 2 * tg);
                        const float2 xv = *reinterpret_cast<const float2 *>(xs + j * MM_BN + 2 * tg);
                        const float d0 = (float)(128 * (int)dv[4 * j + 0] + (int)dv[4 * j + 1]);   // exact
                        const float d1 = (float)(128 * (int)dv[4 * j + 2] + (int)dv[4 * j + 3]);
                        A[2 * tg + 0] = fmaf(a[j] * xv.x, d0, fmaf(-dm[j], sv.x, A[2 * tg + 0]));
                        A[2 * tg + 1] = fmaf(a[j] * xv.y, d1, fmaf(-dm[j], sv.y, A[2 * tg + 1]));
                    }
                }
                return;
            }
            if (p.x32) {
                // columns 2t and 2t+1: token t's high and low parts
                #pragma unroll
                for (int tg = 0; tg < MM_BN / 4; ++tg) {
                    if (2 * tg >= ntok) break;   // warp-uniform
                    uint32_t dv[32];
                    tmem_ld4x8(t_lane + MM_ACC_COL + b * 128u + 4u * tg, dv);
                    #pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const float2 sv = *reinterpret_cast<const float2 *>(sb + j * MM_BN + 2 * tg);
                        const float d0 = __uint_as_float(dv[4 * j + 0]) + __uint_as_float(dv[4 * j + 1]);
                        const float d1 = __uint_as_float(dv[4 * j + 2]) + __uint_as_float(dv[4 * j + 3]);
                        A[2 * tg + 0] = fmaf(a[j], d0, fmaf(-c[j], sv.x, A[2 * tg + 0]));
                        A[2 * tg + 1] = fmaf(a[j], d1, fmaf(-c[j], sv.y, A[2 * tg + 1]));
                    }
                }
                return;
            }
            #pragma unroll
            for (int tg = 0; tg < MM_BN / 4; ++tg) {
                if (4 * tg >= ntok) break;   // warp-uniform
                uint32_t dv[32];
                tmem_ld4x8(t_lane + MM_ACC_COL + b * 128u + 4u * tg, dv);
                #pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float4 sv = *reinterpret_cast<const float4 *>(sb + j * MM_BN + 4 * tg);
                    A[4 * tg + 0] = fmaf(a[j], __uint_as_float(dv[4 * j + 0]), fmaf(-c[j], sv.x, A[4 * tg + 0]));
                    A[4 * tg + 1] = fmaf(a[j], __uint_as_float(dv[4 * j + 1]), fmaf(-c[j], sv.y, A[4 * tg + 1]));
                    A[4 * tg + 2] = fmaf(a[j], __uint_as_float(dv[4 * j + 2]), fmaf(-c[j], sv.z, A[4 * tg + 2]));
                    A[4 * tg + 3] = fmaf(a[j], __uint_as_float(dv[4 * j + 3]), fmaf(-c[j], sv.w, A[4 * tg + 3]));
                }
            }
        };
        // Exact fp32 (non-finite activations): each decoded weight of the
        // stage times the activation itself, so infinities and NaNs combine
        // as IEEE arithmetic does.
        auto exact = [&](float (&A)[MM_BN], const uint8_t *blk, const float *dm, int sp) {
            #pragma unroll 1
            for (int t = 0; t < MM_BN; ++t) {
                if (t >= ntok) break;
                float v = 0.f;
                #pragma unroll 1
                for (int kk = 0; kk < 256; ++kk) {
                    const int j = kk >> 5, cc = kk >> 6, l = kk & 31;
                    const uint32_t byte = blk[16 + 32 * cc + l];
                    const float qv = (float)((j & 1) ? (byte >> 4) : (byte & 15u));
                    const int64_t k = 256 * (sp % nk) + kk;
                    const int xr = s_xrow[buf * MM_BN + t];
                    const int64_t xi = (int64_t)(xr < 0 ? 0 : xr) * p.k + k;
                    const float xv = p.x32 ? static_cast<const float *>(p.x)[xi]
                                           : __bfloat162float(static_cast<const __nv_bfloat16 *>(p.x)[xi]);
                    v = fmaf(fmaf(a[j], qv, -dm[j]), xv, v);
                }
                #pragma unroll
                for (int tt = 0; tt < MM_BN; ++tt)
                    if (tt == t) A[tt] += v;
            }
        };
        for (int u = u0; u < u1 && ok; ++u) {
            const int tile = u / nrt;
            if (tile != prev) {
                if (xt > 0) {   // done with the previous tile's activations and pair ids
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(x_empty);
                }
                ok = __all_sync(0xffffffffu, mbar_wait(x_meta, (uint32_t)xt & 1u, p.err));
                if (!ok) break;
                buf = xt & 1;
                ntok = s_ntok[buf];
                float *sb = s_sum + buf * nsub * MM_BN;
                bool bad = false;
                for (int v = ti; v < ntok * nsub; v += 128) {
                    const int t = v / nsub, jg = v - t * nsub;
                    const int xr = s_xrow[buf * MM_BN + t];   // -1 only for a pair a KQ_DEBUG check dropped
                    const int64_t xi = (int64_t)(xr < 0 ? 0 : xr) * p.k + 32 * jg;
                    float xf[32];
                    if (p.x32) {
                        const float4 *src = reinterpret_cast<const float4 *>(static_cast<const float *>(p.x) + xi);
                        #pragma unroll
                        for (int c4 = 0; c4 < 8; ++c4) {
                            const float4 f = src[c4];
                            xf[4 * c4] = f.x; xf[4 * c4 + 1] = f.y; xf[4 * c4 + 2] = f.z; xf[4 * c4 + 3] = f.w;
                        }
                    } else {
                        const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(p.x) + xi);
                        #pragma unroll
                        for (int cq = 0; cq < 4; ++cq) {
                            const uint4 w = src[cq];
                            xf[8 * cq] = bf16_lo(w.x); xf[8 * cq + 1] = bf16_hi(w.x);
                            xf[8 * cq + 2] = bf16_lo(w.y); xf[8 * cq + 3] = bf16_hi(w.y);
                            xf[8 * cq + 4] = bf16_lo(w.z); xf[8 * cq + 5] = bf16_hi(w.z);
                            xf[8 * cq + 6] = bf16_lo(w.w); xf[8 * cq + 7] = bf16_hi(w.w);
                            if (!I8) *reinterpret_cast<uint4 *>(x_tile_w(x_tile, t, 32 * jg + 8 * cq)) = w;
                        }
                    }
                    if constexpr (I8) {
                        // 14-bit codes c = x / 2^(e-13), e = floor(log2 max |x|): rows 2t
                        // (c >> 7) and 2t+1 (c & 127) of the int8 tile
                        float amax = 0.f;
                        #pragma unroll
                        for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(xf[i]));
                        int e = (int)((__float_as_uint(amax) >> 23) & 0xFF) - 127;
                        e = min(max(e, -100), 100);
                        const float inv = __uint_as_float((uint32_t)(13 - e + 127) << 23);
                        s_xsc[(buf * nsub + jg) * MM_BN + t] = __uint_as_float((uint32_t)(e - 13 + 127) << 23);
                        uint32_t hw[8], lw[8];
                        #pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            uint32_t h = 0, l = 0;
                            #pragma unroll
                            for (int bb = 0; bb < 4; ++bb) {
                                const int cv = min(__float2int_rn(xf[4 * i + bb] * inv), 16383);
                                h |= (uint32_t)((cv >> 7) & 0xFF) << (8 * bb);
                                l |= (uint32_t)(cv & 127) << (8 * bb);
                            }
                            hw[i] = h;
                            lw[i] = l;
                        }
                        #pragma unroll
                        for (int c16 = 0; c16 < 2; ++c16) {
                            *reinterpret_cast<uint4 *>(x_tile_w8(x_tile, 2 * t, 32 * jg + 16 * c16)) =
                                make_uint4(hw[4 * c16], hw[4 * c16 + 1], hw[4 * c16 + 2], hw[4 * c16 + 3]);
                            *reinterpret_cast<uint4 *>(x_tile_w8(x_tile, 2 * t + 1, 32 * jg + 16 * c16)) =
                                make_uint4(lw[4 * c16], lw[4 * c16 + 1], lw[4 * c16 + 2], lw[4 * c16 + 3]);
                        }
                    } else if (p.x32) {
                        // rows 2t (bf16 high part) and 2t+1 (bf16 low part)
                        #pragma unroll
                        for (int cq = 0; cq < 4; ++cq) {
                            uint32_t hw[4], lw[4];
                            #pragma unroll
                            for (int h = 0; h < 4; ++h) {
                                const float x0 = xf[8 * cq + 2 * h], x1 = xf[8 * cq + 2 * h + 1];
                                const __nv_bfloat162 hi = __floats2bfloat162_rn(x0, x1);
                                const __nv_bfloat162 lo = __floats2bfloat162_rn(x0 - __low2float(hi), x1 - __high2float(hi));
                                hw[h] = *reinterpret_cast<const uint32_t *>(&hi);
                                lw[h] = *reinterpret_cast<const uint32_t *>(&lo);
                            }
                            *reinterpret_cast<uint4 *>(x_tile_w(x_tile, 2 * t, 32 * jg + 8 * cq)) =
                                make_uint4(hw[0], hw[1], hw[2], hw[3]);
                            *reinterpret_cast<uint4 *>(x_tile_w(x_tile, 2 * t + 1, 32 * jg + 8 * cq)) =
                                make_uint4(lw[0], lw[1], lw[2], lw[3]);
                        }
                    }
                    float sum = 0.f;
                    #pragma unroll
                    for (int i = 0; i < 32; i += 4) sum += (xf[i] + xf[i + 1]) + (xf[i + 2] + xf[i + 3]);
                    sb[jg * MM_BN + t] = sum;
                    bad |= !(fabsf(sum) <= 3.402823466e38f);   // an infinity or NaN in the sub-block
                }
                if (__any_sync(0xffffffffu, bad) && lane == 0) s_nf[buf] = 1;
                fence_proxy_async_smem();   // the tile's generic writes before the MMA reads them
                __syncwarp();
                if (lane == 0) mbar_arrive(x_full);
                ok = __all_sync(0xffffffffu, mbar_wait(x_full, (uint32_t)xt & 1u, p.err));
                if (!ok) break;
                nf = s_nf[buf] != 0;
                prev = tile;
                ++xt;
            }
            const int row = (u % nrt) * MM_BM + r;
            #pragma unroll
            for (int t = 0; t < MM_BN; ++t) acc[t] = accg[t] = 0.f;
            for (int s = 0; s < ns && ok; ++s, ++g) {
                const uint32_t rs = L % (uint32_t)R, rph = (L / (uint32_t)R) & 1u, b = g & 1u;
                const int sb = s % nk;
                const bool slot_end = (sb % SPB) == SPB - 1 || sb == nk - 1;
                ok = __all_sync(0xffffffffu, mbar_wait(&raw_full[rs], rph, p.err) &&
                                                 mbar_wait(&mma_done[b], (g >> 1) & 1u, p.err));
                if (!ok) break;
                tc_fence_after();
                const uint8_t *blk = raw + rs * slot_bytes + (r * SPB + sb % SPB) * MM_SB;
                const uint4 hd = *reinterpret_cast<const uint4 *>(blk);
                const float d = half_bits_to_float(hd.x), dmin = half_bits_to_float(hd.x >> 16);
                const uint32_t sc_lo = hd.y & 0x3F3F3F3Fu, m_lo = hd.z & 0x3F3F3F3Fu;
                const uint32_t sc_hi = (hd.w & 0x0F0F0F0Fu) | ((hd.y >> 2) & 0x30303030u);
                const uint32_t m_hi = ((hd.w >> 4) & 0x0F0F0F0Fu) | ((hd.z >> 2) & 0x30303030u);
                #pragma unroll
                for (int j = 0; j < 8; ++j) {
                    a[j] = d * mm_byte_f(j < 4 ? sc_lo : sc_hi, j & 3);      // exact
                    dm[j] = dmin * mm_byte_f(j < 4 ? m_lo : m_hi, j & 3);    // exact
                    c[j] = fmaf(128.0f, a[j], dm[j]);
                }
                // every stage adds into acc; the GLU form's gate sums move to
                // accg when its up pass starts (one copy of each accumulate
                // path in the code, not one per target)
                if (p.glu && s == nk) {
                    #pragma unroll
                    for (int t = 0; t < MM_BN; ++t) {
                        accg[t] = acc[t];
                        acc[t] = 0.f;
                    }
                }
                if (nf) exact(acc, blk, dm, s);
                else apply(acc, b, s);
                tc_fence_before();
                fence_proxy_async_smem();   // generic reads of the raw slot before TMA refills it
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&acc_empty[b]);
                    if (slot_end) mbar_arrive(&raw_empty[rs]);
                }
                if (slot_end) ++L;
            }
            if (!ok) break;
            if (row < p.n) {
                if (p.glu) {
                    #pragma unroll
                    for (int t = 0; t < MM_BN; ++t)
                        if (t < ntok) acc[t] *= glu_activation(accg[t], p.act);
                }
                // (a select of both forms per token measured several thousand
                // cycles slower at each unit's end)
                #pragma unroll
                for (int t = 0; t < MM_BN; ++t) {
                    if (t >= ntok) break;
                    const int pr = s_pair[buf * MM_BN + t];
                    if (pr >= 0) store_out(y + (int64_t)pr * p.n + row, acc[t]);
                }
            }
        }
    } else if (warp >= MM_DEC_WARP0) {
        // ---------------- decode warps ----------------
        // Two warps per TMEM lane quadrant: warp 8 + 4h + q writes the codes
        // of chunks 2h and 2h+1 (128 weights) of row 32q + lane's
        // super-block into the stage's A slot, once the MMAs that read the
        // slot two stages ago are done.
        const int q = warp & 3, r = 32 * q + lane, half = (warp - MM_DEC_WARP0) >> 2;
        const uint32_t t_lane = tmem_base + ((uint32_t)(32 * q) << 16);
        uint32_t g = 0, L = 0;   // stages and raw ring slots consumed
        bool ok = true;
        for (int u = u0; u < u1 && ok; ++u) {
            for (int s = 0; s < ns; ++s, ++g) {
                const uint32_t rs = L % (uint32_t)R, rph = (L / (uint32_t)R) & 1u, b = g & 1u;
                const int sb = s % nk;
                const bool slot_end = (sb % SPB) == SPB - 1 || sb == nk - 1;
                ok = __all_sync(0xffffffffu, mbar_wait(&raw_full[rs], rph, p.err) &&
                                                 (g < 2 || mbar_wait(&mma_done[b], ((g - 2) >> 1) & 1u, p.err)));
                if (!ok) break;
                tc_fence_after();
                const uint8_t *blk = raw + rs * slot_bytes + (r * SPB + sb % SPB) * MM_SB;
                if constexpr (I8) {
                    // u8 codes, four a column: chunk cc's low nibbles (sub-block
                    // 2cc) then its high nibbles (2cc+1), 16 columns a chunk
                    uint32_t out[32];
                    #pragma unroll
                    for (int c2 = 0; c2 < 2; ++c2) {
                        const int cc = 2 * half + c2;
                        const uint4 v0 = *reinterpret_cast<const uint4 *>(blk + 16 + 32 * cc);
                        const uint4 v1 = *reinterpret_cast<const uint4 *>(blk + 32 + 32 * cc);
                        const uint32_t qw[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
                        #pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            out[16 * c2 + i] = qw[i] & 0x0F0F0F0Fu;
                            out[16 * c2 + 8 + i] = (qw[i] >> 4) & 0x0F0F0F0Fu;
                        }
                    }
                    tmem_st32(t_lane + MM_A_COL + b * 128u + 32u * half, out);
                } else {
                    #pragma unroll
                    for (int c2 = 0; c2 < 2; ++c2) {
                        const int cc = 2 * half + c2;
                        const uint4 v0 = *reinterpret_cast<const uint4 *>(blk + 16 + 32 * cc);
                        const uint4 v1 = *reinterpret_cast<const uint4 *>(blk + 32 + 32 * cc);
                        const uint32_t qw[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
                        uint32_t out[32];
                        #pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            codes4(qw[i] & 0x0F0F0F0Fu, out[2 * i], out[2 * i + 1]);
                            codes4((qw[i] >> 4) & 0x0F0F0F0Fu, out[16 + 2 * i], out[17 + 2 * i]);
                        }
                        tmem_st32(t_lane + MM_A_COL + b * 128u + 32u * cc, out);
                    }
                }
                tc_fence_before();
                fence_proxy_async_smem();   // generic reads of the raw slot before TMA refills it
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&a_full[b]);
                    if (slot_end) mbar_arrive(&raw_empty[rs]);
                }
                if (slot_end) ++L;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    griddep_launch_dependents();
    if (warp == MM_MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

namespace {

// Raw ring: slots of spb super-blocks (the longest contiguous run of each
// row that still leaves two slots next to the activation tile and the
// sums; 4, 2 or 1), as many slots as fit, at most four.
bool mm_ring(int64_t k, bool i8, int *slots, int *spb) {
    for (int b = 4; b >= 1; b >>= 1) {
        if (b > 1 && b > k / 256) continue;
        int r = 4;
        while (r >= 2 && mm_layout((int)k, r, b, i8).total > MM_SMEM_LIMIT) --r;
        if (r >= 2) {
            *slots = r;
            *spb = b;
            return true;
        }
    }
    return false;
}

// Raw Q4_K rows as (bytes of a super-block, super-blocks, rows, experts):
// a box of spb super-blocks of 128 rows reads spb * 144 contiguous bytes a row.
bool encode_w_map4(CUtensorMap *m, const void *w, int64_t n, int64_t k, int64_t n_experts, int64_t expert_stride,
                   int spb) {
    const int64_t nk = k / 256;
    cuuint64_t dims[4] = {(cuuint64_t)MM_SB, (cuuint64_t)nk, (cuuint64_t)n, (cuuint64_t)n_experts};
    cuuint64_t strides[3] = {(cuuint64_t)MM_SB, (cuuint64_t)(nk * MM_SB), (cuuint64_t)expert_stride};
    cuuint32_t box[4] = {MM_SB, (cuuint32_t)spb, MM_BM, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void *>(w), dims, strides, box, es,
                       CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool moe_mma_supported(int type, int64_t n, int64_t k, int x_dtype, int y_dtype) {
    if (type != KQ_Q4_K || (x_dtype != KQ_BF16 && x_dtype != KQ_F32)) return false;
    if (y_dtype != KQ_F32 && y_dtype != KQ_BF16) return false;
    if (k % 256 || k > MM_MAX_K || n < 1 || n > (1 << 30)) return false;
    int slots, spb;
    return mm_ring(k, false, &slots, &spb) && mm_ring(k, true, &slots, &spb) && encode_fn() != nullptr;
}

// Tokens per tile: 16 bf16 activation rows, or 8 (fp32 rows, or the int8
// form): two MMA rows each.
int moe_mma_bn(int x_dtype, bool i8) { return x_dtype == KQ_F32 || i8 ? MM_BN / 2 : MM_BN; }

namespace {

cudaError_t launch_mm(MoeMmaParams p, const CUtensorMap &tw, const CUtensorMap &tw2, int x_dtype, int y_dtype,
                      bool i8, cudaStream_t s) {
    p.nk = p.k / 256;
    p.n_row_tiles = (p.n + MM_BM - 1) / MM_BM;
    p.x32 = x_dtype == KQ_F32 ? 1 : 0;
    p.tpt = moe_mma_bn(x_dtype, i8);
    p.err = error_word();
    const int smem = mm_layout(p.k, p.raw_slots, p.spb, i8).total;
    auto kern = y_dtype == KQ_F32 ? (i8 ? moe_mma_kernel<float, true> : moe_mma_kernel<float, false>)
                                  : (i8 ? moe_mma_kernel<__nv_bfloat16, true> : moe_mma_kernel<__nv_bfloat16, false>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)sm_count());
    cfg.blockDim = dim3(MM_THREADS);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, tw, tw2, p);
}

}  // namespace

cudaError_t launch_moe_mma(const IdArgs &a, cudaStream_t s) {
    if (!moe_mma_supported(a.type, a.n, a.k, a.x_dtype, a.y_dtype)) return cudaErrorNotSupported;
    MoeMmaParams p = {};
    p.n = (int)a.n;
    p.k = (int)a.k;
    p.x_div = a.x_div();
    p.n_pairs = (int)(a.n_tokens * a.top_k);
    p.n_experts = (int)a.n_experts;
    p.perm = a.perm;
    p.offsets = a.offsets;
    p.tiles = reinterpret_cast<const int2 *>(a.tiles);
    p.n_tiles = a.n_tiles;
    p.y = a.y;
    p.x = a.x;
    p.glu = a.w2 != nullptr;
    p.act = a.act;
    mm_ring(a.k, a.tc_i8, &p.raw_slots, &p.spb);
    CUtensorMap tw, tw2;
    if (!encode_w_map4(&tw, a.w, a.n, a.k, a.n_experts, a.expert_stride, p.spb) ||
        !encode_w_map4(&tw2, p.glu ? a.w2 : a.w, a.n, a.k, a.n_experts, a.expert_stride, p.spb))
        return cudaErrorInvalidValue;
    return launch_mm(p, tw, tw2, a.x_dtype, a.y_dtype, a.tc_i8, s);
}

cudaError_t launch_gemv_tc(const void *w, int64_t n, int64_t k, const void *x, int x_dtype, int64_t m, void *y,
                           int y_dtype, bool i8, cudaStream_t s) {
    if (!moe_mma_supported(KQ_Q4_K, n, k, x_dtype, y_dtype) || m < 1 || m > INT32_MAX / 2)
        return cudaErrorNotSupported;
    MoeMmaParams p = {};
    p.n = (int)n;
    p.k = (int)k;
    p.x_div = 1;
    p.n_pairs = (int)m;
    p.n_experts = 1;
    p.dense_m = (int)m;
    p.y = y;
    p.x = x;
    mm_ring(k, i8, &p.raw_slots, &p.spb);
    CUtensorMap tw;
    if (!encode_w_map4(&tw, w, n, k, 1, n * (k / 256) * MM_SB, p.spb)) return cudaErrorInvalidValue;
    return launch_mm(p, tw, tw, x_dtype, y_dtype, i8, s);
}

}  // namespace kq
