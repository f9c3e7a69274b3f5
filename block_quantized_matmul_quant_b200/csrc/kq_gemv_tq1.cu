// kq_gemv_tq1.cu -- bandwidth-bound product for TQ1_G128 weights (decode).
//
// y[t][n] = sum_k dequant(w)[n][k] * x[t][k] for few activation rows, with
// w in the ternary 28-byte / 128-weight block of Ternary Bonsai (weight j of
// a block: base-3 digit j % 5 of code byte j / 5 for j < 125, digit j - 125
// of the tail byte 25; value (digit - 1) * fp16 scale at bytes 26..27;
// code bytes above 242 (full) or 26 (tail) decode to zero).  This is the
// ternary GEMV the pages run on Metal (ternel `tq1_gemv`, `_trit_table_source`
// / `_direct_trit_table_source`), written here for sm_100a.
//
// Two kernels.
//
// gemv_tq1_split_kernel (row bytes a multiple of 16, at most 144 blocks a
// row): the K dimension is split over the lanes of the CTA -- lane (g, b)
// owns block b of every row of row group g -- so each lane's activations
// live in registers for the whole kernel and the shared-memory traffic per
// code byte is one 32-bit table load.
//  * Digit algebra.  With f_i = floor(p / 3^i) the digits of a legal byte p
//    are t_i = f_i - 3 f_{i+1} (f_5 = 0), so
//        sum_i t_i x_i = sum_i f_i y_i,   y_0 = x_0,  y_i = x_i - 3 x_{i-1}.
//    A 256-entry table gives (f1, f2, f3, f4) as four bytes; f0 is the code
//    byte itself.  Per byte: one prmt forms the table address straight from
//    the weight word, one shared load, two dp2a (y1 f1 + y2 f2, y3 f3 + y4 f4);
//    the f0 terms take one dp2a per two bytes on the raw weight words.  With
//    the weights' mean removed through sum_j x_j, the block's product is
//    scale * s_x * (sum_bytes sum_i f_i y_i - sum_j xq_j), all in int32.
//  * Activations: 13-bit fixed point per 128-wide block (x ~= s_x * xq,
//    s_x = 2^(e-12), e = floor(log2 max|x|), |xq| <= 8191, error <= 2^-13 of
//    the block maximum), so every y fits int16.
//  * The table is replicated 32 times (copy = lane) at a 256-byte stride:
//    address = table | p << 8 | lane << 2 is a single prmt of the weight
//    word with a per-lane constant, and the lanes' loads never share a bank.
//    A second table (the other 128 bytes of each row) serves the tail byte.
//  * Illegal bytes map to an entry with bit 7 set; the lane ORs its entries
//    and recomputes a flagged block exactly in fp32 (decoding each digit).
//    Non-finite activations take the same exact path for the whole call, so
//    infinities and NaNs propagate as in the IEEE product.
//  * A producer warp bulk-copies batches of G consecutive rows (one per row
//    group) into a ring of shared-memory slots, as far ahead as the ring
//    allows; consumers write one fp32 partial per (row, block) next to the
//    rows, and the producer adds a batch's partials in a fixed order, writes
//    y and refills the slot.
//
// gemv_tq1_kernel (the other shapes): a warp takes two rows at a time and
// lane l takes blocks l, l + 32, ...; activations are staged in shared
// memory as one 16-byte record per code byte and a replicated byte -> five
// trits table feeds dp2a.  Bound by the shared-memory instruction queue.
#include <atomic>

#include "kq_ptx.cuh"
#include "kq_launch.h"

namespace kq {

namespace {

constexpr int TQ_BB = 28;            // bytes per block
constexpr int TQ_QK = 128;           // weights per block

__device__ __forceinline__ int dp2a_lo_ss(int a, int b, int c) {
    int d;
    asm("dp2a.lo.s32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
__device__ __forceinline__ int dp2a_hi_ss(int a, int b, int c) {
    int d;
    asm("dp2a.hi.s32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
// 16-bit signed pairs of a times unsigned bytes 0,1 (lo) or 2,3 (hi) of b.
__device__ __forceinline__ int dp2a_lo_su(int a, uint32_t b, int c) {
    int d;
    asm("dp2a.lo.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
__device__ __forceinline__ int dp2a_hi_su(int a, uint32_t b, int c) {
    int d;
    asm("dp2a.hi.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ float load_x(const float *x, int64_t i) { return x[i]; }
__device__ __forceinline__ float load_x(const __nv_bfloat16 *x, int64_t i) {
    return __bfloat162float(x[i]);
}

__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

// ============================================================ split kernel

constexpr int T1_CONSUMERS = 544;                  // consumer threads at most (17 warps)
constexpr int T1_THREADS = T1_CONSUMERS + 32;      // + the producer warp
constexpr int T1_PRODUCER_WARP = T1_CONSUMERS / 32;
constexpr int T1_TABLE_BYTES = 65536;              // 256 rows of 256 bytes
constexpr int T1_MAX_NB = 144;                     // staging rounds of S2 (registers)
constexpr int T1_ZSTRIDE = 68;                     // staged code words per block (16-byte aligned, bank-spread)
constexpr int T1_SMEM_MAX = 232448;                // opt-in dynamic shared memory per CTA

struct Tq1SplitParams {
    const uint8_t *w;
    int n, nb;
    const void *x;
    void *y;
    int groups;         // row groups G: lanes g*nb .. g*nb+nb-1 form group g
    int rows_per_cta;
    int slots;          // ring slots, each G rows + their partials
    int slot_bytes;
    int row_bytes;
    int smem_bytes;     // dynamic shared memory of the launch
    int indep;          // independent call: never wait for the preceding kernel
    unsigned int *err;
};

// Table entry of code byte p: bytes (f1, f2, f3, f4) of a legal byte, or
// bit 7 alone for a byte above `max_legal`.
__host__ __device__ constexpr uint32_t prefix_entry(uint32_t p, uint32_t max_legal) {
    return p > max_legal ? 0x80u : (p / 3u) | ((p / 9u) << 8) | ((p / 27u) << 16) | ((p / 81u) << 24);
}

// The shared-memory table image: row p (256 bytes) holds 32 copies of the
// main entry of byte p, then 32 copies of its tail entry.  Kept in global
// memory and bulk-copied into every CTA, so no thread spends time on it.
struct PrefixTable {
    uint32_t w[T1_TABLE_BYTES / 4];
};
constexpr PrefixTable make_prefix_table() {
    PrefixTable t{};
    for (int i = 0; i < T1_TABLE_BYTES / 4; ++i)
        t.w[i] = prefix_entry((uint32_t)i >> 6, (i & 32) ? 26u : 242u);
    return t;
}
__device__ __align__(128) const PrefixTable g_prefix_table = make_prefix_table();

// Shared-memory layout of the split kernel, the same on host and device.
// The tables take the 64 KB-aligned window that the prmt addressing needs;
// scratch (per-block activation sums and exponents, flags, barriers), the
// staged codes and the ring slots fill the space before it (A) and after
// it (B), in that order of preference.
// Scratch: per block (activation-code sum, scale bits) pairs, four flag
// words, the slots' shared addresses, then the barriers.
__host__ __device__ constexpr int t1_bar_offset(int nb, int S) { return (8 * nb + 16 + 4 * S + 7) / 8 * 8; }
__host__ __device__ constexpr int t1_scratch_bytes(int nb, int S) {
    return (t1_bar_offset(nb, S) + 8 * (2 * S + 2) + 15) & ~15;
}
struct T1Layout {
    uint32_t tab, scratch, codes, slot_a0, slot_b0;
    int slots_a;
    uint32_t end;   // one past the last byte used
};
__host__ __device__ inline T1Layout t1_layout(uint32_t base, int nb, int S, int slot_bytes) {
    T1Layout l{};
    l.tab = (base + 65535u) & ~65535u;
    uint32_t a = base, b = l.tab + T1_TABLE_BYTES;
    const uint32_t sb = (uint32_t)t1_scratch_bytes(nb, S), cb = (uint32_t)(nb * T1_ZSTRIDE * 4);
    if (l.tab - a >= sb) { l.scratch = a; a += sb; } else { l.scratch = b; b += sb; }
    if (l.tab - a >= cb) { l.codes = a; a += cb; } else { l.codes = b; b += cb; }
    l.slots_a = (int)((l.tab - a) / (uint32_t)slot_bytes);
    if (l.slots_a > S) l.slots_a = S;
    l.slot_a0 = a;
    l.slot_b0 = b;
    l.end = b + (uint32_t)(S - l.slots_a) * (uint32_t)slot_bytes;
    if (l.end < l.tab + T1_TABLE_BYTES) l.end = l.tab + T1_TABLE_BYTES;
    return l;
}

// Exact fp32 product of one block with 128 activations (each weight decoded
// from its digits, illegal bytes as zero), for flagged blocks and calls with
// non-finite activations.
template <typename XT>
__device__ float block_exact(const uint8_t *blk, const XT *xb) {
    const float scale = half_bits_to_float((uint32_t)blk[26] | ((uint32_t)blk[27] << 8));
    float acc = 0.f;
    for (int j = 0; j < 26; ++j) {
        const uint32_t p = blk[j];
        const int nd = j < 25 ? 5 : 3;
        const bool legal = p <= (j < 25 ? 242u : 26u);
        uint32_t r = p;
        for (int d = 0; d < nd; ++d) {
            const int t = legal ? (int)(r % 3u) : 1;
            r /= 3u;
            acc = fmaf((float)(t - 1) * scale, load_x(xb, (j < 25 ? 5 * j : 125) + d), acc);
        }
    }
    return acc;
}

// 18 warps: a scheduler's 16384-register partition takes five of them, so a
// thread holds at most 96 registers (the 64 activation words, a product in
// flight and a few spilled loop values; 14 warps with 128 registers and no
// spills measured slower).
template <typename XT, typename YT>
__global__ void __launch_bounds__(T1_THREADS, 1) gemv_tq1_split_kernel(const Tq1SplitParams p) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int G = p.groups, nb = p.nb;
    const int row_begin = blockIdx.x * p.rows_per_cta;
    const int row_end = min(p.n, row_begin + p.rows_per_cta);
    if (row_begin >= row_end) return;
    const int n_batches = (row_end - row_begin + G - 1) / G;
    const int S = p.slots;

    const uint32_t base = smem_addr(smem);
    const T1Layout lay = t1_layout(base, nb, S, p.slot_bytes);
    if (lay.end - base > dynamic_smem_size()) {   // the host planned another layout: no work
        if (tid == 0) atomicOr(p.err, ERR_BOUNDS);
        return;
    }
    // Pointers into shared memory are formed as smem + offset, so that the
    // compiler keeps them in the shared state space; only the table lookups
    // use raw shared addresses.
    auto sp = [&](uint32_t a) -> uint8_t * { return smem + (a - base); };
    auto slot_addr = [&](int s) -> uint32_t {
        return s < lay.slots_a ? lay.slot_a0 + (uint32_t)s * p.slot_bytes
                               : lay.slot_b0 + (uint32_t)(s - lay.slots_a) * p.slot_bytes;
    };
    int2 *s_bs = reinterpret_cast<int2 *>(sp(lay.scratch));   // [nb]: (sum of codes, 2^(e-12) bits)
    int *s_flags = reinterpret_cast<int *>(s_bs + nb);         // [0] non-finite activations
    uint32_t *s_slot = reinterpret_cast<uint32_t *>(s_flags + 4);   // [S]: slot shared addresses
    uint64_t *full = reinterpret_cast<uint64_t *>(sp(lay.scratch) + t1_bar_offset(nb, S));
    uint64_t *empty = full + S;
    uint64_t *tbar = empty + S;      // the table copy
    uint64_t *pbar = tbar + 1;       // consumer warps: a pair of batches' partials written
    const int consumer_warps = (G * nb + 31) / 32;   // warps holding block lanes
    const int64_t row_bytes = p.row_bytes;

    auto issue = [&](int i) {   // batch i: rows row_begin + i*G .. (contiguous, 16-byte aligned)
        const int s = i % S;
        const int r0 = row_begin + i * G;
        const int rows = min(G, row_end - r0);
        const uint32_t bytes = (uint32_t)(rows * row_bytes);
        mbar_arrive_expect_tx(&full[s], bytes);
        bulk_g2s(sp(slot_addr(s)), p.w + (int64_t)r0 * row_bytes, bytes, &full[s]);
    };

    griddep_launch_dependents();
    if (warp == T1_PRODUCER_WARP && lane == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], consumer_warps);
        }
        mbar_init(tbar, 1);
        mbar_init(pbar, consumer_warps);
        fence_mbar_init();
        mbar_arrive_expect_tx(tbar, T1_TABLE_BYTES);
        bulk_g2s(sp(lay.tab), &g_prefix_table, T1_TABLE_BYTES, tbar);
    }
    if (tid < 4) s_flags[tid] = 0;
    for (int i = tid; i < S; i += blockDim.x) s_slot[i] = slot_addr(i);
    if (!p.indep) griddep_wait();
    __syncthreads();

    // ---- activations: thread (b, c) of four per block takes positions
    // 32c .. 32c+31 of block b: the block's largest |x| (an integer max over
    // the absolute bit patterns, so infinities and NaNs come out above every
    // finite value), 13-bit codes rounded to nearest even by the float-add
    // trick, their sum, and the codes as int16 into the staging area.
    const XT *x = static_cast<const XT *>(p.x);
    uint32_t *zst = reinterpret_cast<uint32_t *>(sp(lay.codes));   // [nb][T1_ZSTRIDE] words
    // every lane runs every round (the shuffles take the whole warp)
    for (int r0 = 0; r0 < 4 * nb; r0 += blockDim.x) {
        const int item = r0 + tid;
        const bool in = item < 4 * nb;   // groups of four lanes are wholly in or out
        const int b = in ? item >> 2 : 0, c = item & 3;
        float v[32];
        uint32_t m = 0;   // largest |x| as an fp32 bit pattern
        if (!in) {
            #pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = 0.f;
        } else if (sizeof(XT) == 2) {
            const uint4 *src = reinterpret_cast<const uint4 *>(x + (int64_t)b * TQ_QK + 32 * c);
            uint4 a[4];
            #pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = src[i];
            uint32_t mm = 0;
            #pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint32_t wds[4] = {a[i].x, a[i].y, a[i].z, a[i].w};
                #pragma unroll
                for (int k = 0; k < 4; ++k) {
                    mm = __vmaxu2(mm, wds[k] & 0x7FFF7FFFu);
                    v[8 * i + 2 * k] = bf16lo(wds[k]);
                    v[8 * i + 2 * k + 1] = bf16hi(wds[k]);
                }
            }
            m = max(mm & 0xFFFFu, mm >> 16) << 16;
        } else {
            const float4 *src = reinterpret_cast<const float4 *>(x + (int64_t)b * TQ_QK + 32 * c);
            float4 a[8];
            #pragma unroll
            for (int i = 0; i < 8; ++i) a[i] = src[i];
            #pragma unroll
            for (int i = 0; i < 8; ++i) {
                v[4 * i] = a[i].x; v[4 * i + 1] = a[i].y; v[4 * i + 2] = a[i].z; v[4 * i + 3] = a[i].w;
            }
            #pragma unroll
            for (int i = 0; i < 32; ++i) m = max(m, __float_as_uint(v[i]) & 0x7FFFFFFFu);
        }
        #pragma unroll
        for (int o = 2; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
        const int ex = (int)(m >> 23);
        const int e = max(ex - 127, -100);
        if (in && ex >= 0xFF) s_flags[0] = 1;   // inf or NaN somewhere in x
        // x * 2^(12-e) + 1.5 * 2^23: the low 16 bits of the sum's pattern
        // are the code (|code| <= 8192 < 2^22), rounded to nearest even
        const float inv = __uint_as_float((uint32_t)(12 - e + 127) << 23);
        const float magic = 12582912.0f;
        uint32_t pk[16];
        int sum = 0;
        #pragma unroll
        for (int i = 0; i < 16; ++i) {
            const uint32_t lo = __float_as_uint(fmaf(v[2 * i], inv, magic));
            const uint32_t hi = __float_as_uint(fmaf(v[2 * i + 1], inv, magic));
            pk[i] = __vmins2(__byte_perm(lo, hi, 0x5410), 0x1FFF1FFFu);   // codes <= 8191
            sum = dp2a_lo_ss((int)pk[i], 0x0101, sum);
        }
        #pragma unroll
        for (int o = 2; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (in) {
            if (c == 0) s_bs[b] = make_int2(sum, (int)((uint32_t)(e - 12 + 127) << 23));   // 2^(e-12)
            uint4 *zb = reinterpret_cast<uint4 *>(zst + b * T1_ZSTRIDE) + 4 * c;
            #pragma unroll
            for (int i = 0; i < 4; ++i) zb[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
        }
    }
    // The ring's first copies go out only now, after the activations were
    // read: issued earlier (before the wait for the preceding kernel, or
    // before the activation loads), their 15 MB across the CTAs delayed the
    // activation loads by more than they gained (measured 14.1 -> 13.6 us
    // for independent calls, 14.8 -> 13.6 for ordered ones).
    if (warp == T1_PRODUCER_WARP && lane == 0)
        for (int i = 0; i < min(S, n_batches); ++i) issue(i);
    __syncthreads();

    // ---- step 2: item (b, j) turns the five codes of code byte j of block
    // b into its activation words -- word j: y1 | y2, word 26 + j: y3 | y4,
    // half j of words 51..63: y0 (y0 = x0, y_i = x_i - 3 x_{i-1}) -- in
    // place over the block's codes: every code is read before any word is
    // written.
    {
        constexpr int S2_ROUNDS = (26 * T1_MAX_NB + T1_THREADS - 1) / T1_THREADS;
        const int16_t *zst16 = reinterpret_cast<const int16_t *>(zst);
        uint32_t y12[S2_ROUNDS], y34[S2_ROUNDS], y0[S2_ROUNDS];
        #pragma unroll
        for (int r = 0; r < S2_ROUNDS; ++r) {
            const int item = tid + r * T1_THREADS;
            if (item < 26 * nb) {
                const int b = item / 26, j = item - 26 * b;
                const int16_t *zq = zst16 + 2 * b * T1_ZSTRIDE + (j < 25 ? 5 * j : 125);
                const int q0 = zq[0], q1 = zq[1], q2 = zq[2];
                const int q3 = j < 25 ? zq[3] : 0, q4 = j < 25 ? zq[4] : 0;
                y12[r] = __byte_perm((uint32_t)(q1 - 3 * q0), (uint32_t)(q2 - 3 * q1), 0x5410);
                y34[r] = __byte_perm((uint32_t)(q3 - 3 * q2), (uint32_t)(q4 - 3 * q3), 0x5410);
                y0[r] = (uint32_t)q0;
            }
        }
        __syncthreads();
        #pragma unroll
        for (int r = 0; r < S2_ROUNDS; ++r) {
            const int item = tid + r * T1_THREADS;
            if (item < 26 * nb) {
                const int b = item / 26, j = item - 26 * b;
                uint32_t *zw = zst + b * T1_ZSTRIDE;
                zw[j] = y12[r];
                if (j < 25) zw[26 + j] = y34[r];
                reinterpret_cast<uint16_t *>(zw + 51)[j] = (uint16_t)y0[r];
            }
        }
    }
    __syncthreads();

    // The last pair of batches (the consumers' last iteration) is added up by
    // the consumer warps after their loop; the producer adds the ones before.
    const int i_last = (n_batches - 1) & ~1;
    YT *y = static_cast<YT *>(p.y);
    // rows of batch i: lpr lanes add the nb partials of a row (four
    // independent sums in a fixed order), then a butterfly over the lpr lanes
    auto reduce_rows = [&](int i, int r_begin, int r_step, int lpr) {
        const int s = i % S;
        const float *part = reinterpret_cast<const float *>(sp(s_slot[s] + (uint32_t)(G * row_bytes)));
        const int r0 = row_begin + i * G;
        const int rows_per_pass = 32 / lpr;
        for (int g0 = r_begin; g0 < G; g0 += r_step * rows_per_pass) {
            const int gi = g0 + (lane / lpr) * r_step, sub = lane % lpr;
            float v = 0.f;
            if (gi < G) {
                const float *pr = part + gi * nb;
                float v0 = 0.f, v1 = 0.f, v2 = 0.f, v3 = 0.f;
                int bb = sub;
                for (; bb + 3 * lpr < nb; bb += 4 * lpr) {
                    v0 += pr[bb];
                    v1 += pr[bb + lpr];
                    v2 += pr[bb + 2 * lpr];
                    v3 += pr[bb + 3 * lpr];
                }
                for (; bb < nb; bb += lpr) v0 += pr[bb];
                v = (v0 + v1) + (v2 + v3);
            }
            for (int o = lpr / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (gi < G && sub == 0 && r0 + gi < row_end) store_out(y + r0 + gi, v);
        }
    };

    if (warp == T1_PRODUCER_WARP) {
        // ---------------- producer: reduce finished batches, refill slots
        const int lpr_raw = 32 / min(G, 32);
        int lpr = 1;
        while (lpr * 2 <= lpr_raw) lpr *= 2;              // lanes per row (power of two)
        for (int i = 0; i < i_last; ++i) {
            const int s = i % S;
            if (!__all_sync(0xffffffffu, mbar_wait_poll(&empty[s], (uint32_t)(i / S) & 1u, p.err))) break;
            reduce_rows(i, 0, 1, lpr);
            if (i + S < n_batches) {
                __syncwarp();
                if (lane == 0) {
                    fence_proxy_async_smem();   // generic reads of the slot before the async refill
                    issue(i + S);
                }
            }
        }
    } else if (warp < consumer_warps) {
        // ---------------- consumers (warps holding block lanes; the lanes
        // without a block, at the top of the last such warp, take part in
        // the waits, barriers and the reduction)
        const int g = tid / nb, b = tid - g * nb;
        const bool active = g < G;
        // the lane's block's 64 activation words (16-byte loads at a 272-byte
        // block stride: the eight lanes of a load phase hit distinct banks)
        const int bb = active ? b : 0;
        uint32_t Y[64];
        {
            const uint4 *zb = reinterpret_cast<const uint4 *>(zst + bb * T1_ZSTRIDE);
            #pragma unroll
            for (int c = 0; c < 16; ++c) {
                const uint4 v = zb[c];
                Y[4 * c] = v.x; Y[4 * c + 1] = v.y; Y[4 * c + 2] = v.z; Y[4 * c + 3] = v.w;
            }
        }
        const bool nonfinite = s_flags[0] != 0;   // CTA-uniform
        // the table must have landed before the first lookup
        if (!__all_sync(0xffffffffu, mbar_wait(tbar, 0, p.err))) goto done;
        {
            const uint32_t cb_main = (uint32_t)(lane << 2) | ((lay.tab >> 16) << 16);
            const uint32_t off = (uint32_t)(g * row_bytes + bb * TQ_BB);
            const uint32_t poff = (uint32_t)(G * row_bytes) + 4u * (uint32_t)(g * nb + bb);
            // one (row, block) product: integer sum of f_i y_i over the block's
            // code bytes minus the sum of its activation codes, times the
            // block's weight scale and activation scale; the exact fp32
            // product when the block holds an illegal byte
            auto block_dot = [&](uint32_t blk) -> float {
                uint32_t wv[7];
                #pragma unroll
                for (int q = 0; q < 7; ++q) wv[q] = lds_u32(blk + 4 * q);
                const int2 bs = s_bs[bb];
                int acc[4] = {-bs.x, 0, 0, 0};   // four independent dp2a chains
                uint32_t flag = 0;
                #pragma unroll
                for (int j = 0; j < 26; ++j) {
                    const uint32_t cb = j < 25 ? cb_main : (cb_main | 0x80u);   // tail table: bytes 128..255
                    const uint32_t addr = __byte_perm(wv[j >> 2], cb, 0x7604u | ((uint32_t)(j & 3) << 4));
                    const uint32_t e = lds_u32(addr);
                    flag |= e;
                    int &a = acc[j & 3];
                    a = dp2a_lo_su((int)Y[j], e, a);
                    if (j < 25) a = dp2a_hi_su((int)Y[26 + j], e, a);
                }
                #pragma unroll
                for (int q = 0; q < 7; ++q) {   // f0 terms: the code bytes themselves
                    acc[q & 3] = dp2a_lo_su((int)Y[51 + 2 * q], wv[q], acc[q & 3]);
                    if (q < 6) acc[(q + 2) & 3] = dp2a_hi_su((int)Y[52 + 2 * q], wv[q], acc[(q + 2) & 3]);
                }
                if (flag & 0x80u) return block_exact(sp(blk), static_cast<const XT *>(p.x) + (int64_t)bb * TQ_QK);
                const float scale = half_bits_to_float(wv[6] >> 16);
                return (float)((acc[0] + acc[1]) + (acc[2] + acc[3])) * (scale * __int_as_float(bs.y));
            };
            // two batches (two slots) per iteration
            for (int i = 0; i < n_batches; i += 2) {
                const bool two = i + 1 < n_batches;
                const int s0 = i % S, s1 = (i + 1) % S;
                const uint32_t par0 = (uint32_t)(i / S) & 1u, par1 = (uint32_t)((i + 1) / S) & 1u;
                // one outcome per warp, so every lane leaves the loop together
                bool ok = mbar_wait_poll(&full[s0], par0, p.err);
                if (two) ok = ok && mbar_wait_poll(&full[s1], par1, p.err);
                if (!__all_sync(0xffffffffu, ok)) break;
                const int row0 = row_begin + i * G + g;
                if (active) {
                    // nonfinite: exact fp32 products (IEEE infinities and NaNs)
                    const XT *xb = static_cast<const XT *>(p.x) + (int64_t)bb * TQ_QK;
                    if (row0 < row_end) {
                        const uint32_t sa = s_slot[s0];
                        *reinterpret_cast<float *>(sp(sa + poff)) = nonfinite ? block_exact(sp(sa + off), xb) : block_dot(sa + off);
                    }
                    if (two && row0 + G < row_end) {
                        const uint32_t sa = s_slot[s1];
                        *reinterpret_cast<float *>(sp(sa + poff)) = nonfinite ? block_exact(sp(sa + off), xb) : block_dot(sa + off);
                    }
                }
                __syncwarp();   // the warp's reads of the slots and partial writes are done
                if (lane == 0) {
                    mbar_arrive(&empty[s0]);
                    if (two) mbar_arrive(&empty[s1]);
                }
            }
        }
        // the last pair: once every consumer warp has written its partials
        // (a barrier on an mbarrier, so the wait is bounded), warp w adds up
        // rows w, w + consumer_warps, ... of the pair
        __syncwarp();
        if (lane == 0) mbar_arrive(pbar);
        if (__all_sync(0xffffffffu, mbar_wait_poll(pbar, 0, p.err))) {
            reduce_rows(i_last, warp, consumer_warps, 1);
            if (i_last + 1 < n_batches) reduce_rows(i_last + 1, warp, consumer_warps, 1);
        }
    done:;
    }
    if (p.indep) griddep_wait();   // complete after the work before it (stream order)
}

// ============================================================ table kernel

constexpr int TQ_REC = 27;           // 16-byte activation records per block (26 used, odd stride)
constexpr int TQ_WARPS = 16;
constexpr int TQ_COPIES = 16;
constexpr int TQ_TABLE_BYTES = 256 * TQ_COPIES * 8;
constexpr int TQ_SMEM_LIMIT = 220 * 1024;

struct Tq1Params {
    const uint8_t *w;
    int n, k, nb;
    const void *x;
    void *y;
    int rows_per_cta;
    int early;   // weights constant: prefetch before griddepcontrol.wait
    int indep;   // independent call: never wait for the preceding kernel
};

// The five digits of a legal code byte, minus one, as signed bytes.
__device__ __forceinline__ uint2 trit_entry(uint32_t p) {
    if (p > 242u) return make_uint2(0u, 0u);
    uint32_t b[5];
    #pragma unroll
    for (int i = 0; i < 5; ++i) {
        b[i] = (uint32_t)((int)(p % 3u) - 1) & 0xFFu;
        p /= 3u;
    }
    return make_uint2(b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24), b[4]);
}

template <int TB, typename XT, typename YT>
__global__ void __launch_bounds__(32 * TQ_WARPS, 1) gemv_tq1_kernel(const Tq1Params p) {
    extern __shared__ __align__(16) uint8_t smem[];
    uint2 *table = reinterpret_cast<uint2 *>(smem);                              // [256][16]
    uint4 *xrec = reinterpret_cast<uint4 *>(smem + TQ_TABLE_BYTES);              // [TB][nb][27]
    float *xs = reinterpret_cast<float *>(smem + TQ_TABLE_BYTES + (size_t)TB * p.nb * TQ_REC * 16);  // [TB][nb]

    __shared__ int s_nonfinite;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int row_begin = blockIdx.x * p.rows_per_cta;
    const int row_end = min(p.n, row_begin + p.rows_per_cta);
    if (row_begin >= row_end) return;
    const int64_t row_bytes = (int64_t)p.nb * TQ_BB;
    if (threadIdx.x == 0) s_nonfinite = 0;

    griddep_launch_dependents();
    auto prefetch_rows = [&]() {
        if (threadIdx.x == 0) {
            // [start, end) rounded inwards to 16 bytes (w is 16-byte aligned)
            const uint64_t base = reinterpret_cast<uint64_t>(p.w);
            uint64_t a = base + (uint64_t)row_begin * row_bytes, e = base + (uint64_t)row_end * row_bytes;
            a &= ~(uint64_t)15;
            e &= ~(uint64_t)15;
            for (uint64_t off = a; off < e; off += 32768)
                prefetch_l2(reinterpret_cast<const void *>(off), (uint32_t)(e - off < 32768 ? e - off : 32768));
        }
    };
    if (p.early) prefetch_rows();

    // trit table: thread t fills entry t's copies, copy (c + t) % 16 at
    // step c, so a half-warp's stores fall in distinct banks
    for (int e = threadIdx.x; e < 256; e += blockDim.x) {
        const uint2 v = trit_entry((uint32_t)e);
        for (int c = 0; c < TQ_COPIES; ++c) table[e * TQ_COPIES + ((c + e) & (TQ_COPIES - 1))] = v;
    }
    // zero the activation records (their pad halves stay zero)
    {
        const int nrec = TB * p.nb * TQ_REC;
        for (int i = threadIdx.x; i < nrec; i += blockDim.x) xrec[i] = make_uint4(0u, 0u, 0u, 0u);
    }
    if (!p.indep) griddep_wait();
    if (!p.early) prefetch_rows();
    __syncthreads();

    // ---- stage activations: one warp per (token, block), 4 values per lane
    {
        const XT *x = static_cast<const XT *>(p.x);
        const int items = TB * p.nb;
        for (int it = warp; it < items; it += TQ_WARPS) {
            const int t = it / p.nb, b = it % p.nb;
            const int64_t base = (int64_t)t * p.k + (int64_t)b * TQ_QK + 4 * lane;
            float v[4];
            #pragma unroll
            for (int i = 0; i < 4; ++i) v[i] = load_x(x, base + i);
            float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
            const bool bad = !(fabsf(v[0]) < __int_as_float(0x7f800000)) || !(fabsf(v[1]) < __int_as_float(0x7f800000)) ||
                             !(fabsf(v[2]) < __int_as_float(0x7f800000)) || !(fabsf(v[3]) < __int_as_float(0x7f800000));
            if (bad) s_nonfinite = 1;   // inf or NaN: the call runs the exact fp32 path
            #pragma unroll
            for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
            int ex = (int)((__float_as_uint(amax) >> 23) & 0xFF) - 127;   // floor(log2 amax)
            ex = max(ex, -100);
            const float inv_s = __uint_as_float((uint32_t)(13 - ex + 127) << 23);  // 2^(13-ex)
            if (lane == 0) xs[it] = __uint_as_float((uint32_t)(ex - 13 + 127) << 23);
            uint16_t *rec = reinterpret_cast<uint16_t *>(xrec + (size_t)it * TQ_REC);
            #pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int pos = 4 * lane + i;               // position in the block
                const int j = pos < 125 ? pos / 5 : 25;     // code byte
                const int d = pos < 125 ? pos % 5 : pos - 125;  // digit
                rec[j * 8 + d] = (uint16_t)(int16_t)__float2int_rn(v[i] * inv_s);
            }
        }
    }
    __syncthreads();

    if (s_nonfinite) {
        // Non-finite activations: every (row, block) product in fp32 from the
        // decoded weights, so infinities and NaNs propagate as in the IEEE
        // product; lane l takes blocks l, l + 32, ...
        const XT *x = static_cast<const XT *>(p.x);
        YT *y = static_cast<YT *>(p.y);
        for (int r = row_begin + warp; r < row_end; r += TQ_WARPS) {
            for (int t = 0; t < TB; ++t) {
                float v = 0.f;
                for (int b = lane; b < p.nb; b += 32)
                    v += block_exact(p.w + (int64_t)r * row_bytes + (int64_t)b * TQ_BB,
                                     x + (int64_t)t * p.k + (int64_t)b * TQ_QK);
                #pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                if (lane == 0) store_out(y + (int64_t)t * p.n + r, v);
            }
        }
        if (p.indep) griddep_wait();
        return;
    }

    // ---- rows: warp w takes rows w, w + TQ_WARPS, ... two at a time (one
    // activation record load serves both); lane l takes blocks l, l + 32, ...
    const uint2 *tab = table + (lane & (TQ_COPIES - 1));
    const int steps_per_row = (p.nb + 31) / 32;
    const int my_rows = warp < row_end - row_begin ? (row_end - row_begin - warp + TQ_WARPS - 1) / TQ_WARPS : 0;
    const int npairs = (my_rows + 1) / 2;
    const int nsteps = npairs * steps_per_row;
    auto load_step = [&](int s, uint32_t wv[2][7]) {
        const int pr = s / steps_per_row;
        const int b = (s % steps_per_row) * 32 + lane;
        #pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int i = 2 * pr + h;
            if (s < nsteps && i < my_rows && b < p.nb) {
                const int r = row_begin + warp + i * TQ_WARPS;
                const uint32_t *src =
                    reinterpret_cast<const uint32_t *>(p.w + (int64_t)r * row_bytes + (int64_t)b * TQ_BB);
                #pragma unroll
                for (int j = 0; j < 7; ++j) wv[h][j] = __ldg(src + j);
            } else {
                #pragma unroll
                for (int j = 0; j < 7; ++j) wv[h][j] = 0u;
            }
        }
    };
    YT *y = static_cast<YT *>(p.y);
    uint32_t cur[2][7], nxt[2][7];
    load_step(0, cur);
    float acc[2][TB];
    #pragma unroll
    for (int h = 0; h < 2; ++h)
        #pragma unroll
        for (int t = 0; t < TB; ++t) acc[h][t] = 0.f;
    for (int s = 0; s < nsteps; ++s) {
        load_step(s + 1, nxt);
        const int b = (s % steps_per_row) * 32 + lane;
        const int bb = b < p.nb ? b : 0;
        int ia[2][TB][2];
        #pragma unroll
        for (int h = 0; h < 2; ++h)
            #pragma unroll
            for (int t = 0; t < TB; ++t) ia[h][t][0] = ia[h][t][1] = 0;
        #pragma unroll
        for (int j = 0; j < 26; ++j) {
            uint2 tv[2];
            #pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t code = __byte_perm(cur[h][j >> 2], 0u, 0x4440u | (uint32_t)(j & 3));
                if (j == 25 && code > 26u) code = 255u;
                tv[h] = tab[code * TQ_COPIES];
            }
            #pragma unroll
            for (int t = 0; t < TB; ++t) {
                const uint4 xv = xrec[((size_t)t * p.nb + bb) * TQ_REC + j];
                #pragma unroll
                for (int h = 0; h < 2; ++h) {
                    int a = dp2a_lo_ss((int)xv.x, (int)tv[h].x, ia[h][t][j & 1]);
                    a = dp2a_hi_ss((int)xv.y, (int)tv[h].x, a);
                    ia[h][t][j & 1] = dp2a_lo_ss((int)xv.z, (int)tv[h].y, a);
                }
            }
        }
        #pragma unroll
        for (int h = 0; h < 2; ++h) {
            const float scale = half_bits_to_float(cur[h][6] >> 16);
            #pragma unroll
            for (int t = 0; t < TB; ++t)
                acc[h][t] = fmaf((float)(ia[h][t][0] + ia[h][t][1]), scale * xs[t * p.nb + bb], acc[h][t]);
        }
        if ((s + 1) % steps_per_row == 0) {
            const int pr = s / steps_per_row;
            #pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int i = 2 * pr + h;
                #pragma unroll
                for (int t = 0; t < TB; ++t) {
                    float v = acc[h][t];
                    #pragma unroll
                    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                    if (lane == 0 && i < my_rows) store_out(y + (int64_t)t * p.n + row_begin + warp + i * TQ_WARPS, v);
                    acc[h][t] = 0.f;
                }
            }
        }
        #pragma unroll
        for (int h = 0; h < 2; ++h)
            #pragma unroll
            for (int j = 0; j < 7; ++j) cur[h][j] = nxt[h][j];
    }
    if (p.indep) griddep_wait();   // complete after the work before it (stream order)
}

size_t tq1_smem_bytes(int tb, int nb) {
    return (size_t)TQ_TABLE_BYTES + (size_t)tb * nb * TQ_REC * 16 + (size_t)tb * nb * 4;
}

template <int TB, typename XT, typename YT>
cudaError_t launch_tq1_t(const Tq1Params &p, cudaStream_t s) {
    auto kern = gemv_tq1_kernel<TB, XT, YT>;
    const size_t smem = tq1_smem_bytes(TB, p.nb);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((p.n + p.rows_per_cta - 1) / p.rows_per_cta));
    cfg.blockDim = dim3(32 * TQ_WARPS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, p);
}

template <int TB>
cudaError_t launch_tq1_tb(const Tq1Params &p, int xdt, int ydt, cudaStream_t s) {
    if (xdt == KQ_F32)
        return ydt == KQ_F32 ? launch_tq1_t<TB, float, float>(p, s) : launch_tq1_t<TB, float, __nv_bfloat16>(p, s);
    return ydt == KQ_F32 ? launch_tq1_t<TB, __nv_bfloat16, float>(p, s)
                         : launch_tq1_t<TB, __nv_bfloat16, __nv_bfloat16>(p, s);
}

}  // namespace

namespace {

// Shared address of the first byte of a kernel's dynamic shared memory: the
// CTA's reserved system bytes come first (the split kernel declares no
// static shared memory).
int dynamic_smem_base() {
    static std::atomic<int> cache[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    int v = cache[dev].load(std::memory_order_relaxed);
    if (v == 0) {
        int r = 0;
        if (cudaDeviceGetAttribute(&r, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess) r = 1024;
        v = r + 1;   // stored off by one so that 0 means unknown
        cache[dev].store(v, std::memory_order_relaxed);
    }
    return v - 1;
}

bool plan_tq1_split(int64_t n, int64_t k, int sms, Tq1SplitParams *p) {
    if (k % TQ_QK || n < 1 || n > INT32_MAX / 2) return false;
    const int nb = (int)(k / TQ_QK);
    if (nb % 4 || nb > T1_MAX_NB) return false;   // rows must be 16-byte multiples for the bulk copies
    const int G = T1_CONSUMERS / nb;
    const int row_bytes = nb * TQ_BB;
    int64_t ctas = (n + G - 1) / G;
    if (ctas > sms) ctas = sms;
    const int rows_per_cta = (int)((n + ctas - 1) / ctas);
    const int n_batches = (rows_per_cta + G - 1) / G;
    const int slot_bytes = (G * row_bytes + G * nb * 4 + 15) / 16 * 16;
    const uint32_t base = (uint32_t)dynamic_smem_base();
    int S = n_batches < 32 ? n_batches : 32;
    for (; S >= 1; --S)
        if (t1_layout(base, nb, S, slot_bytes).end - base <= (uint32_t)T1_SMEM_MAX) break;
    // consumers take two batches per iteration: two batches must be in
    // flight together, in distinct slots
    if (S < 1 || (n_batches >= 2 && S < 2)) return false;
    p->n = (int)n; p->nb = nb; p->groups = G; p->rows_per_cta = rows_per_cta;
    p->slots = S; p->slot_bytes = slot_bytes; p->row_bytes = row_bytes;
    p->smem_bytes = (int)(t1_layout(base, nb, S, slot_bytes).end - base);
    return true;
}

template <typename XT, typename YT>
cudaError_t launch_split_t(const Tq1SplitParams &p, cudaStream_t s) {
    auto kern = gemv_tq1_split_kernel<XT, YT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, p.smem_bytes);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((p.n + p.rows_per_cta - 1) / p.rows_per_cta));
    cfg.blockDim = dim3(T1_THREADS);
    cfg.dynamicSmemBytes = (size_t)p.smem_bytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, p);
}

}  // namespace

bool gemv_tq1_supported(int64_t n, int64_t k) {
    if (k % TQ_QK || k > (1 << 22) || n < 1 || n > INT32_MAX / 2) return false;
    return tq1_smem_bytes(1, (int)(k / TQ_QK)) <= (size_t)TQ_SMEM_LIMIT;
}

// Rows whose byte length is a multiple of 16 (K a multiple of 512, up to
// 24576) run the split kernel, one launch per activation row (the weights
// of later rows come from L2 when they fit there).  Other shapes run the
// table kernel, two activation rows per launch.
cudaError_t launch_gemv_tq1(const void *w, int64_t n, int64_t k, const void *x, int xdt, int64_t m,
                            void *y, int ydt, GemvOrder order, cudaStream_t s) {
    if (!gemv_tq1_supported(n, k)) return cudaErrorNotSupported;
    const size_t xs = (xdt == KQ_F32 ? 4 : 2), ys = (ydt == KQ_F32 ? 4 : 2);
    const int sms = sm_count();
    Tq1SplitParams sp = {};
    if (plan_tq1_split(n, k, sms, &sp)) {
        sp.w = static_cast<const uint8_t *>(w);
        sp.indep = order == GemvOrder::kIndependent ? 1 : 0;
        sp.err = error_word();
        for (int64_t m0 = 0; m0 < m; ++m0) {
            sp.x = static_cast<const char *>(x) + (size_t)m0 * (size_t)k * xs;
            sp.y = static_cast<char *>(y) + (size_t)m0 * (size_t)n * ys;
            cudaError_t e;
            if (xdt == KQ_F32)
                e = ydt == KQ_F32 ? launch_split_t<float, float>(sp, s) : launch_split_t<float, __nv_bfloat16>(sp, s);
            else
                e = ydt == KQ_F32 ? launch_split_t<__nv_bfloat16, float>(sp, s)
                                  : launch_split_t<__nv_bfloat16, __nv_bfloat16>(sp, s);
            if (e != cudaSuccess) return e;
        }
        return cudaSuccess;
    }
    const int nb = (int)(k / TQ_QK);
    const int tb_max = tq1_smem_bytes(2, nb) <= (size_t)TQ_SMEM_LIMIT ? 2 : 1;
    for (int64_t m0 = 0; m0 < m; m0 += tb_max) {
        const int tb = (int)(m - m0 < tb_max ? m - m0 : tb_max);
        Tq1Params p = {};
        p.w = static_cast<const uint8_t *>(w);
        p.n = (int)n; p.k = (int)k; p.nb = nb;
        p.x = static_cast<const char *>(x) + (size_t)m0 * (size_t)k * xs;
        p.y = static_cast<char *>(y) + (size_t)m0 * (size_t)n * ys;
        p.rows_per_cta = (int)((n + sms - 1) / sms);
        p.early = order != GemvOrder::kStream ? 1 : 0;
        p.indep = order == GemvOrder::kIndependent ? 1 : 0;
        cudaError_t e = tb == 2 ? launch_tq1_tb<2>(p, xdt, ydt, s) : launch_tq1_tb<1>(p, xdt, ydt, s);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace kq
