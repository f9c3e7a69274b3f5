// kq_moe_gemv.cu -- expert-indexed product with few (token, slot) pairs per
// expert (the decode-time mixture-of-experts matmul): Q4_K weights.
//
// y[t][s][n] = sum_k dequant(w[ids[t][s]])[n][k] * x[t][k]: mlx-native 0.21.0
// quantized_matmul_id_ggml.rs (the mv_id route: every routed pair of an
// expert shares one pass over that expert's rows), after the device-side
// grouping of kq_moe.cu (per-expert counts, offsets, ascending pair list).
// Fused GLU mode (mlx-kquant `moe_glu_gather_kq`): a tile carries each
// output row's gate and up weights as a group's two rows, both products
// share the activations in registers, and the finishing step writes
// act(gate) * up.
//
// B200 design
//  * Work items: (expert, round, tile).  A round is up to four of the
//    expert's pairs; a tile is G*R consecutive weight rows (G row groups of R
//    rows).  Only experts somebody chose have items; the items are split in
//    contiguous ranges over the CTAs (one CTA per SM), so each CTA streams
//    its share of the hit experts' rows once per round.
//  * A producer warp bulk-copies tiles into a ring of shared-memory slots.
//  * K is split over the lanes of a row group: lane j owns 32-weight
//    sub-block j of every row, so its four tokens' activation codes (16-bit
//    fixed point per sub-block, exact fp32 sub-block sums beside them) stay
//    in registers for the whole round.  Per row the lane reads 32 quant
//    bytes and the block header, masks its nibble half, and runs 16 dp2a
//    per token; per sub-block the exact identity
//        sum_i (d*sc*q_i - dmin*m) x_i = d*sc*s * sum_i q_i xq_i - dmin*m * sum_i x_i
//    gives the product.
//  * After R rows a lane holds R x 4 partial sums; a transposed butterfly
//    adds them over the warp (each level halves the values a lane keeps),
//    lanes write the warp's sums next to the tile and the producer adds the
//    group's warps and writes y -- every sum in a fixed order.
//  * Calls whose staged activations hold an infinity or a NaN compute those
//    rounds exactly in fp32 (decoded weights times x), so non-finite values
//    propagate as in the IEEE product.
//  * Every wait is bounded (kq_ptx.cuh).
#include "kq_decode.cuh"
#include "kq_ptx.cuh"
#include "kq_launch.h"

namespace kq {

namespace {

constexpr int MG_CWARPS = 12;                       // consumer warps
constexpr int MG_THREADS = (MG_CWARPS + 1) * 32;    // + the producer warp
constexpr int MG_PRODUCER = MG_CWARPS;
constexpr int MG_TB = 4;                            // pairs a round
constexpr int MG_R = 2;                             // rows a group takes per tile
constexpr int MG_XSTRIDE = 40;                      // staged codes per sub-block (int16; 80 B: bank-spread)
constexpr int MG_SMEM_MAX = 232448;
constexpr int MG_PART = MG_R * MG_TB;               // partial sums a warp leaves per tile
static_assert(MG_PART == 8 || MG_PART == 16 || MG_PART == 32, "butterfly over a power of two");
constexpr int MG_SHIFT = MG_PART == 8 ? 2 : MG_PART == 16 ? 1 : 0;   // 32 = MG_PART << MG_SHIFT

struct MoeGemvParams {
    const uint8_t *w;
    const uint8_t *w2;         // fused GLU: the up stack (w is the gate stack)
    int glu, act;              // fused GLU mode; activation (KQ_ACT_*)
    int64_t expert_stride;
    int n, k, nb, nsub;        // rows per expert, K, super-blocks and sub-blocks per row
    int n_experts, top_k;
    const void *x;
    void *y;
    const int32_t *counts, *offsets, *perm;
    int n_pairs;                    // entries of perm; pair ids are below it
    int wg, groups;            // warps per row group, row groups
    int tile_rows, tiles;      // output rows per tile, tiles per expert
    int slots, slot_bytes, part_off;
    unsigned int *err;
};

__device__ __forceinline__ int dp2a_lo(int a, uint32_t b, int c) {
    int d;
    asm("dp2a.lo.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
__device__ __forceinline__ int dp2a_hi(int a, uint32_t b, int c) {
    int d;
    asm("dp2a.hi.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
__device__ __forceinline__ float byte_f(uint32_t w, int i) {   // byte i of w, exactly
    return __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7440u | (uint32_t)i)) - 8388608.0f;
}

// Shared-memory offsets (bytes from the dynamic base).
struct MgLayout {
    int cum, bars, xq, xs, slots, total;
};
__host__ __device__ inline MgLayout mg_layout(int n_experts, int nsub, int slots, int slot_bytes) {
    MgLayout l{};
    int off = 0;
    l.cum = off;   off += ((n_experts + 1) * 4 + 15) / 16 * 16;
    l.bars = off;  off += (2 * slots + 2) * 8;
    off = (off + 15) / 16 * 16;
    l.xq = off;    off += MG_TB * nsub * MG_XSTRIDE * 2;
    l.xs = off;    off += MG_TB * nsub * 8;
    off = (off + 127) / 128 * 128;
    l.slots = off; off += slots * slot_bytes;
    l.total = off;
    return l;
}

template <typename XT>
__device__ __forceinline__ float load_xf(const XT *p);
template <> __device__ __forceinline__ float load_xf(const float *p) { return *p; }
template <> __device__ __forceinline__ float load_xf(const __nv_bfloat16 *p) { return __bfloat162float(*p); }

template <typename XT, typename YT>
__global__ void __launch_bounds__(MG_THREADS, 1) moe_gemv_kernel(const MoeGemvParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int S = p.slots;
    const MgLayout lay = mg_layout(p.n_experts, p.nsub, S, p.slot_bytes);
    int *cum = reinterpret_cast<int *>(smem + lay.cum);            // first item of each expert
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + lay.bars);
    uint64_t *empty = full + S;
    uint64_t *stg = empty + S;                                     // staging done (consumer warps)
    int *s_nonfinite = reinterpret_cast<int *>(stg + 1);
    int16_t *xq = reinterpret_cast<int16_t *>(smem + lay.xq);       // [TB][nsub][MG_XSTRIDE]
    float2 *xs = reinterpret_cast<float2 *>(smem + lay.xs);        // [TB][nsub]: (scale, exact sum)
    const int64_t row_bytes = (int64_t)p.nb * 144;
    const int E = p.n_experts;
    if ((uint32_t)lay.total > dynamic_smem_size()) {   // the host planned another layout: no work
        if (tid == 0) atomicOr(p.err, ERR_BOUNDS);
        return;
    }
    // A pair id of the grouping at position idx of perm (checked in KQ_DEBUG
    // builds: a bad position or id reads pair 0's activations instead).
    auto pair_at = [&](int idx) -> int {
        int v = 0;
        if (KQ_DCHECK(idx >= 0 && idx < p.n_pairs, p.err)) v = p.perm[idx];
        return KQ_DCHECK(v >= 0 && v < p.n_pairs, p.err) ? v : 0;
    };

    // ---- items: expert e has ceil(count / 4) rounds of p.tiles tiles
    if (warp == 0) {
        int carry = 0;
        for (int base = 0; base < E; base += 32) {
            const int e = base + lane;
            const int c = e < E ? (p.counts[e] + MG_TB - 1) / MG_TB * p.tiles : 0;
            int incl = c;
            #pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += t;
            }
            if (e < E) cum[e] = carry + incl - c;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) cum[E] = carry;
    }
    if (tid == 32) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], MG_CWARPS);
        }
        mbar_init(stg, MG_CWARPS);
        *s_nonfinite = -1;
        fence_mbar_init();
    }
    __syncthreads();
    const int total = cum[E];
    const int i0 = (int)((int64_t)total * blockIdx.x / gridDim.x);
    const int i1 = (int)((int64_t)total * (blockIdx.x + 1) / gridDim.x);

    // item i -> (expert, round, tile), walking forward from a known expert
    auto locate = [&](int i, int &e, int &round, int &tile) {
        while (e + 1 < E && cum[e + 1] <= i) ++e;
        const int rel = i - cum[e];
        round = rel / p.tiles;
        tile = rel - round * p.tiles;
    };

    if (warp == MG_PRODUCER) {
        // ---------------- producer: copies tiles in, finishes them
        int e_iss = 0, e_fin = 0;
        auto issue = [&](int i) {
            int r, t;
            locate(i, e_iss, r, t);
            const int s = (i - i0) % S;
            const int row0 = t * p.tile_rows;
            const int rows = min(p.tile_rows, p.n - row0);
            const uint32_t bytes = (uint32_t)(rows * row_bytes);
            const int64_t src = (int64_t)e_iss * p.expert_stride + (int64_t)row0 * row_bytes;
            uint8_t *dst = smem + lay.slots + s * p.slot_bytes;
            mbar_arrive_expect_tx(&full[s], p.glu ? 2 * bytes : bytes);
            bulk_g2s(dst, p.w + src, bytes, &full[s]);
            // fused GLU: the up rows follow the gate rows, p.groups rows on
            if (p.glu) bulk_g2s(dst + p.groups * row_bytes, p.w2 + src, bytes, &full[s]);
        };
        if (lane == 0)
            for (int i = i0; i < min(i1, i0 + S); ++i) issue(i);
        YT *y = static_cast<YT *>(p.y);
        // the round's pair ids, read once per round: lane t holds pair t
        int f_e = -1, f_round = -1, nt = 0, my_pair = 0;
        for (int i = i0; i < i1; ++i) {
            const int s = (i - i0) % S;
            int round, tile;
            locate(i, e_fin, round, tile);
            if (e_fin != f_e || round != f_round) {   // loads overlap the wait below
                f_e = e_fin;
                f_round = round;
                nt = min(MG_TB, p.counts[e_fin] - MG_TB * round);
                // a pair id that fails a KQ_DEBUG check becomes -1: no store
                const int idx = p.offsets[e_fin] + MG_TB * round + lane;
                my_pair = -1;
                if (lane < nt && KQ_DCHECK(idx >= 0 && idx < p.n_pairs, p.err)) {
                    my_pair = p.perm[idx];
                    if (!KQ_DCHECK(my_pair >= 0 && my_pair < p.n_pairs, p.err)) my_pair = -1;
                }
            }
            if (!__all_sync(0xffffffffu, mbar_wait_poll(&empty[s], (uint32_t)((i - i0) / S) & 1u, p.err))) break;
            const float *part = reinterpret_cast<const float *>(smem + lay.slots + s * p.slot_bytes + p.part_off);
            if (p.glu) {
                // output (group g, token t): act(gate sum) * up sum, each the
                // sum of the group's warps
                const int outs = p.groups * MG_TB;
                for (int o0 = 0; o0 < outs; o0 += 32) {
                    const int o = o0 + lane;
                    const int g = o / MG_TB, t = o - g * MG_TB;
                    const int pr = __shfl_sync(0xffffffffu, my_pair, t);
                    const int row = tile * p.tile_rows + g;
                    if (o < outs && t < nt && row < p.n && pr >= 0) {
                        float gs = 0.f, us = 0.f;
                        for (int w = 0; w < p.wg; ++w) {
                            gs += part[(g * p.wg + w) * MG_PART + t];
                            us += part[(g * p.wg + w) * MG_PART + MG_TB + t];
                        }
                        store_out(y + (int64_t)pr * p.n + row, glu_activation(gs, p.act) * us);
                    }
                }
            } else {
                // output (group g, row r, token t): sum of the group's warps
                const int outs = p.groups * MG_PART;
                for (int o0 = 0; o0 < outs; o0 += 32) {
                    const int o = o0 + lane;
                    const int g = o / MG_PART, v = o - g * MG_PART, r = v / MG_TB, t = v - r * MG_TB;
                    const int pr = __shfl_sync(0xffffffffu, my_pair, t & (MG_TB - 1));
                    const int row = tile * p.tile_rows + g * MG_R + r;
                    if (o < outs && t < nt && row < p.n && pr >= 0) {
                        float acc = 0.f;
                        for (int w = 0; w < p.wg; ++w) acc += part[(g * p.wg + w) * MG_PART + v];
                        store_out(y + (int64_t)pr * p.n + row, acc);
                    }
                }
            }
            __syncwarp();
            if (lane == 0 && i + S < i1) {
                fence_proxy_async_smem();   // generic reads of the slot before the async refill
                issue(i + S);
            }
        }
        return;
    }

    // ---------------- consumers
    const int g = warp / p.wg;                       // row group
    const int j = (warp - g * p.wg) * 32 + lane;     // sub-block this lane owns
    const bool in_group = g < p.groups;
    const bool active = in_group && j < p.nsub;
    const int sb = j >> 3, sj = j & 7;               // super-block, sub-block inside it
    const int qoff = sb * 144 + 16 + 32 * (sj >> 1); // its 32 quant bytes
    const uint32_t nmask = (sj & 1) ? 0xF0F0F0F0u : 0x0F0F0F0Fu;   // high nibbles arrive as 16*q
    const float nscale = (sj & 1) ? 0.0625f : 1.0f;
    const XT *x = static_cast<const XT *>(p.x);
    int e_cur = 0, e_key = -1, r_key = -1, stage_no = 0;
    uint32_t X[MG_TB][16];
    float sxv[MG_TB], sumv[MG_TB];
    int nt = 0;
    bool nonfinite = false;
    for (int i = i0; i < i1; ++i) {
        int round, tile;
        locate(i, e_cur, round, tile);
        if (e_cur != e_key || round != r_key) {
            // ---- stage the round's activations: item (t, sub-block) of up
            // to four pairs; every consumer warp takes part.  Two bounded
            // barriers of the consumer warps: the first lets every warp
            // finish reading the previous staging into its registers before
            // anything is overwritten, the second publishes the new one.
            e_key = e_cur;
            r_key = round;
            const int cnt = p.counts[e_cur];
            nt = min(MG_TB, cnt - MG_TB * round);
            const int pbase = p.offsets[e_cur] + MG_TB * round;
            __syncwarp();
            if (lane == 0) mbar_arrive(stg);
            if (!__all_sync(0xffffffffu, mbar_wait_poll(stg, (uint32_t)stage_no & 1u, p.err))) break;
            ++stage_no;
            for (int it = tid; it < nt * p.nsub; it += MG_CWARPS * 32) {
                const int t = it / p.nsub, sjj = it - t * p.nsub;
                const int tok = pair_at(pbase + t) / p.top_k;
                const XT *src = x + (int64_t)tok * p.k + 32 * sjj;
                float v[32];
                if (sizeof(XT) == 2) {
                    const uint4 *s4 = reinterpret_cast<const uint4 *>(src);
                    #pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const uint4 a = s4[c];
                        v[8 * c] = bf16lo(a.x); v[8 * c + 1] = bf16hi(a.x);
                        v[8 * c + 2] = bf16lo(a.y); v[8 * c + 3] = bf16hi(a.y);
                        v[8 * c + 4] = bf16lo(a.z); v[8 * c + 5] = bf16hi(a.z);
                        v[8 * c + 6] = bf16lo(a.w); v[8 * c + 7] = bf16hi(a.w);
                    }
                } else {
                    const float4 *s4 = reinterpret_cast<const float4 *>(src);
                    #pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const float4 a = s4[c];
                        v[4 * c] = a.x; v[4 * c + 1] = a.y; v[4 * c + 2] = a.z; v[4 * c + 3] = a.w;
                    }
                }
                uint32_t m = 0;
                float sum = 0.f;
                #pragma unroll
                for (int q = 0; q < 32; ++q) {
                    m = max(m, __float_as_uint(v[q]) & 0x7FFFFFFFu);   // NaN and inf above all finite
                    sum += v[q];
                }
                const int ex = (int)(m >> 23);
                if (ex >= 0xFF) *s_nonfinite = stage_no;   // inf or NaN in this staging
                const int e = max(ex - 127, -100);
                const float inv = __uint_as_float((uint32_t)(13 - e + 127) << 23);   // 2^(13-e): |code| <= 2^14
                const float magic = 12582912.0f;   // 1.5 * 2^23: the sum's low 16 bits are the rounded code
                uint4 *dst = reinterpret_cast<uint4 *>(xq + (t * p.nsub + sjj) * MG_XSTRIDE);
                #pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t wv[4];
                    #pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        const uint32_t lo = __float_as_uint(fmaf(v[8 * c + 2 * h], inv, magic));
                        const uint32_t hi = __float_as_uint(fmaf(v[8 * c + 2 * h + 1], inv, magic));
                        wv[h] = __byte_perm(lo, hi, 0x5410);
                    }
                    dst[c] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
                }
                xs[t * p.nsub + sjj] = make_float2(__uint_as_float((uint32_t)(e - 13 + 127) << 23), sum);
            }
            // every consumer warp has staged its items (bounded barrier)
            __syncwarp();
            if (lane == 0) mbar_arrive(stg);
            if (!__all_sync(0xffffffffu, mbar_wait_poll(stg, (uint32_t)stage_no & 1u, p.err))) break;
            nonfinite = *s_nonfinite == stage_no;
            ++stage_no;
            // every lane reassigns its activation registers (zeros where it
            // has no sub-block or the round has fewer pairs), so the previous
            // round's values are dead during the staging above
            #pragma unroll
            for (int t = 0; t < MG_TB; ++t) {
                const bool ld = active && t < nt;
                const uint4 *src = reinterpret_cast<const uint4 *>(xq + (t * p.nsub + (ld ? j : 0)) * MG_XSTRIDE);
                #pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint4 a = ld ? src[c] : make_uint4(0u, 0u, 0u, 0u);
                    X[t][4 * c] = a.x; X[t][4 * c + 1] = a.y; X[t][4 * c + 2] = a.z; X[t][4 * c + 3] = a.w;
                }
                const float2 v = ld ? xs[t * p.nsub + j] : make_float2(0.f, 0.f);
                sxv[t] = v.x;
                sumv[t] = v.y;
            }
        }
        const int s = (i - i0) % S;
        if (!__all_sync(0xffffffffu, mbar_wait_poll(&full[s], (uint32_t)((i - i0) / S) & 1u, p.err))) break;
        const uint8_t *slot = smem + lay.slots + s * p.slot_bytes;
        float acc[MG_R][MG_TB];
        #pragma unroll
        for (int r = 0; r < MG_R; ++r)
            #pragma unroll
            for (int t = 0; t < MG_TB; ++t) acc[r][t] = 0.f;
        if (active) {
            #pragma unroll
            for (int r = 0; r < MG_R; ++r) {
                // plain: rows g*R + r of the tile; fused GLU: row g, gate (r = 0)
                // and up (r = 1) weights
                const int row = tile * p.tile_rows + (p.glu ? g : g * MG_R + r);
                if (row >= p.n) break;
                const uint8_t *rp = slot + (int64_t)(p.glu ? r * p.groups + g : g * MG_R + r) * row_bytes;
                const uint4 hd = *reinterpret_cast<const uint4 *>(rp + sb * 144);
                const float d = half_bits_to_float(hd.x), dmin = half_bits_to_float(hd.x >> 16);
                // 6-bit scale and min of sub-block sj (GGUF Q4_K packing)
                const uint32_t scw = sj < 4 ? (hd.y & 0x3F3F3F3Fu) : ((hd.w & 0x0F0F0F0Fu) | ((hd.y >> 2) & 0x30303030u));
                const uint32_t mw = sj < 4 ? (hd.z & 0x3F3F3F3Fu) : (((hd.w >> 4) & 0x0F0F0F0Fu) | ((hd.z >> 2) & 0x30303030u));
                const float a = d * byte_f(scw, sj & 3) * nscale;
                const float dm = dmin * byte_f(mw, sj & 3);
                if (nonfinite) {
                    // exact fp32: decoded weights times the activations
                    const float ae = d * byte_f(scw, sj & 3);
                    #pragma unroll
                    for (int t = 0; t < MG_TB; ++t) {
                        if (t < nt) {
                            const int tok = pair_at(p.offsets[e_cur] + MG_TB * round + t) / p.top_k;
                            const XT *xt = x + (int64_t)tok * p.k + 32 * j;
                            float v = 0.f;
                            for (int l = 0; l < 32; ++l) {
                                const uint32_t byte = rp[qoff + l];
                                const float q = (float)((sj & 1) ? (byte >> 4) : (byte & 15));
                                v = fmaf(fmaf(ae, q, -dm), load_xf(xt + l), v);
                            }
                            acc[r][t] = v;
                        }
                    }
                    continue;
                }
                const uint4 q0 = *reinterpret_cast<const uint4 *>(rp + qoff);
                const uint4 q1 = *reinterpret_cast<const uint4 *>(rp + qoff + 16);
                const uint32_t qw[8] = {q0.x & nmask, q0.y & nmask, q0.z & nmask, q0.w & nmask,
                                        q1.x & nmask, q1.y & nmask, q1.z & nmask, q1.w & nmask};
                #pragma unroll
                for (int t = 0; t < MG_TB; ++t) {
                    if (t < nt) {
                        int s0 = 0, s1 = 0;
                        #pragma unroll
                        for (int w = 0; w < 8; ++w) {
                            s0 = dp2a_lo((int)X[t][2 * w], qw[w], s0);
                            s1 = dp2a_hi((int)X[t][2 * w + 1], qw[w], s1);
                        }
                        acc[r][t] = fmaf(a * sxv[t], (float)(s0 + s1), -dm * sumv[t]);
                    }
                }
            }
        }
        // transposed butterfly: MG_PART values per lane; each level gives
        // away half of a lane's values and adds the partner's, the last
        // levels add whole sums -> lane l holds value (l >> MG_SHIFT) of the
        // warp's sums (lanes differing in the low MG_SHIFT bits alike)
        float v[MG_PART];
        #pragma unroll
        for (int q = 0; q < MG_PART; ++q) v[q] = acc[q / MG_TB][q % MG_TB];
        #pragma unroll
        for (int h = MG_PART / 2, bit = 16; h >= 1; h >>= 1, bit >>= 1) {
            const bool up = (lane & bit) != 0;
            #pragma unroll
            for (int q = 0; q < h; ++q) {
                const float keep = up ? v[q + h] : v[q];
                const float send = up ? v[q] : v[q + h];
                v[q] = keep + __shfl_xor_sync(0xffffffffu, send, bit);
            }
        }
        #pragma unroll
        for (int bit = (1 << MG_SHIFT) / 2; bit >= 1; bit >>= 1) v[0] += __shfl_xor_sync(0xffffffffu, v[0], bit);
        if (in_group && (lane & ((1 << MG_SHIFT) - 1)) == 0) {
            float *part = reinterpret_cast<float *>(smem + lay.slots + s * p.slot_bytes + p.part_off);
            part[warp * MG_PART + (lane >> MG_SHIFT)] = v[0];
        }
        __syncwarp();   // the warp's reads of the slot and partial writes are done
        if (lane == 0) mbar_arrive(&empty[s]);
    }
}

bool plan_moe_gemv(int64_t n, int64_t k, int64_t n_experts, bool glu, MoeGemvParams *p) {
    if (k % 256 || k > 32 * 32 * MG_CWARPS || n < 1 || n > INT32_MAX / 2 || n_experts < 1) return false;
    const int nb = (int)(k / 256), nsub = (int)(k / 32);
    const int wg = (nsub + 31) / 32;
    const int groups = MG_CWARPS / wg;
    if (groups < 1) return false;
    static_assert(MG_R == 2, "the fused GLU takes a group's two rows as gate and up");
    const int tile_rows = glu ? groups : groups * MG_R;   // output rows per tile
    const int64_t row_bytes = (int64_t)nb * 144;
    const int part_off = (int)(groups * MG_R * row_bytes);   // weight rows per slot
    const int slot_bytes = (int)((part_off + MG_CWARPS * MG_PART * 4 + 127) / 128 * 128);
    int slots = 8;
    for (; slots >= 2; --slots)
        if (mg_layout((int)n_experts, nsub, slots, slot_bytes).total <= MG_SMEM_MAX) break;
    if (slots < 2) return false;
    p->n = (int)n; p->k = (int)k; p->nb = nb; p->nsub = nsub; p->n_experts = (int)n_experts;
    p->wg = wg; p->groups = groups; p->tile_rows = tile_rows;
    p->tiles = (int)((n + tile_rows - 1) / tile_rows);
    p->slots = slots; p->slot_bytes = slot_bytes; p->part_off = part_off;
    return true;
}

template <typename XT, typename YT>
cudaError_t launch_mg(const MoeGemvParams &p, cudaStream_t s) {
    auto kern = moe_gemv_kernel<XT, YT>;
    const int smem = mg_layout(p.n_experts, p.nsub, p.slots, p.slot_bytes).total;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kern<<<sm_count(), MG_THREADS, smem, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

bool moe_gemv_supported(int type, int64_t n, int64_t k, int64_t n_experts) {
    MoeGemvParams p;
    return type == KQ_Q4_K && plan_moe_gemv(n, k, n_experts, false, &p);
}

cudaError_t launch_moe_gemv(const IdArgs &a, cudaStream_t s) {
    MoeGemvParams p = {};
    const bool glu = a.w2 != nullptr;
    if (a.type != KQ_Q4_K || !plan_moe_gemv(a.n, a.k, a.n_experts, glu, &p)) return cudaErrorNotSupported;
    p.w = static_cast<const uint8_t *>(a.w);
    p.w2 = static_cast<const uint8_t *>(a.w2);
    p.glu = glu ? 1 : 0;
    p.act = a.act;
    p.expert_stride = a.expert_stride;
    p.top_k = a.x_div();
    p.x = a.x;
    p.y = a.y;
    p.counts = a.counts;
    p.offsets = a.offsets;
    p.perm = a.perm;
    p.n_pairs = (int)(a.n_tokens * a.top_k);
    p.err = error_word();
    if (a.x_dtype == KQ_F32)
        return a.y_dtype == KQ_F32 ? launch_mg<float, float>(p, s) : launch_mg<float, __nv_bfloat16>(p, s);
    return a.y_dtype == KQ_F32 ? launch_mg<__nv_bfloat16, float>(p, s)
                               : launch_mg<__nv_bfloat16, __nv_bfloat16>(p, s);
}

}  // namespace kq
