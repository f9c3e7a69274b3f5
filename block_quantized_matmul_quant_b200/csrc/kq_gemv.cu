// kq_gemv.cu -- bandwidth-bound product for few activation rows (decode).
//
// y[t][n] = sum_k dequant(w)[n][k] * x[t][k] for t < m <= 8: the qmv case of
// mlx-kquant `quantized_matmul` (the pages' Metal forms are ds4's
// `kernel_mul_mv_q8_0_f32`; the expert-indexed form lives in kq_moe_gemv.cu).
//
// B200 design
//  * A CTA owns a contiguous range of weight rows; warp w of the CTA owns
//    rows w, w + W, w + 2W, ... of that range and streams them through a
//    private ring of shared-memory row slots with cp.async.bulk copies (one
//    per row, completion counted on one mbarrier per slot).  Each warp starts
//    on its first row as soon as that row has landed; the ring keeps the
//    next rows in flight without registers.
//  * Two CTA shapes.  A call ordered after the preceding kernel: one CTA per
//    SM, 16 warps (its latency is what counts).  A call declared independent
//    of earlier work: a third of an SM per CTA (4 warps) on half as many
//    CTAs as SMs, so three calls stream side by side on every SM.
//  * Activations are staged once per CTA as 16-bit fixed point per 32-wide
//    sub-block: x ~= s * xq with s = 2^(e-13), e = floor(log2) of the
//    sub-block's largest |x| (|xq| < 2^14, error <= 2^-14 of that maximum,
//    exact for bf16 inputs whose exponent is within 6 of the maximum's), plus
//    the fp32 sum of the sub-block.  The mlx-kquant pages ship int8
//    activation kernels for the same reason (arm64 NEON int8 GEMV); 16 bits
//    keep the error near 1e-5, far inside the 2e-3 / 1e-2 bars.
//  * Q4_K weights stay integer: the low nibbles of a quant word are `v &
//    0x0F0F0F0F`, the high nibbles (times 16) `v & 0xF0F0F0F0`; dp2a
//    multiplies two 16-bit activations by two 8-bit quants and accumulates
//    in int32.  Per sub-block j the exact identity
//        sum_i (d*sc_j*q_i - dmin*m_j) x_i = d*sc_j*s_j*sum_i q_i xq_i - dmin*m_j*sum_i x_i
//    turns the integer sums into the product; every 32-weight sum fits int32.
//  * Programmatic dependent launch: activations are read after
//    griddepcontrol.wait.  When the caller declares the weights constant the
//    row copies are issued before it, overlapping the previous kernel; an
//    independent call never waits before its work and waits once at its end,
//    so that it completes after the work before it.
#include "kq_decode.cuh"
#include "kq_ptx.cuh"
#include "kq_launch.h"

namespace kq {

namespace {

// Two CTA sizes.  A call ordered after the preceding kernel gets a whole
// SM (16 warps, up to 200 KB of row slots): its latency is what counts.
// Independent calls get a fraction of an SM (KQ_GEMV_SHARE_BLOCKS CTAs fit
// on one: KQ_GEMV_SHARE_WARPS warps, at most 128 registers a thread, an
// equal share of shared memory), so the next calls' CTAs are resident
// beside this one and stream their weights while this one computes.
#ifndef KQ_GEMV_XREG
#define KQ_GEMV_XREG 1
#endif
#ifndef KQ_GEMV_SHARE_WARPS
#define KQ_GEMV_SHARE_WARPS 4
#endif
#ifndef KQ_GEMV_SHARE_BLOCKS
#define KQ_GEMV_SHARE_BLOCKS 3
#endif
constexpr int GEMV_SMEM_LIMIT = 200 * 1024;
constexpr int GEMV_MAX_WARPS = 16;
constexpr int GEMV_HALF_MAX_WARPS = KQ_GEMV_SHARE_WARPS;
constexpr int GEMV_HALF_BLOCKS = KQ_GEMV_SHARE_BLOCKS;
// An SM has 228 KB of shared memory and reserves 1 KB per resident CTA;
// leave 256 B for the kernel's static arrays.
constexpr int GEMV_HALF_SMEM_LIMIT = 233472 / GEMV_HALF_BLOCKS - 1024 - 256;
constexpr int GEMV_MAX_SLOTS = 4;
// Slots a warp of a shared-SM CTA keeps in flight (more, measured, is slower:
// fewer CTAs fit side by side).
#ifndef KQ_GEMV_SHARE_SLOTS
#define KQ_GEMV_SHARE_SLOTS 4
#endif
constexpr int GEMV_HALF_MAX_SLOTS = KQ_GEMV_SHARE_SLOTS;
// Independent calls spread over (SMs / KQ_GEMV_SHARE_GRID_DIV) CTAs.
#ifndef KQ_GEMV_SHARE_GRID_DIV
#define KQ_GEMV_SHARE_GRID_DIV 2
#endif

struct GemvParams {
    const uint8_t *w;
    int n, k, m;
    const void *x;
    void *y;
    int nb;           // Q4_K blocks per row
    int units;        // lane work units per row (C chunks of 64 weights each)
    int units_pad;    // units rounded up to a multiple of 8 (staging layout)
    int rows_per_cta, warps, slots, row_bytes;
    int xq_bytes;     // staged int16 activations
    int xs_bytes;     // per-sub-block scales (and as many bytes again of sums)
    int early;        // issue weight copies before griddepcontrol.wait
    int indep;        // independent call: no griddepcontrol.wait at all
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

// Byte i (0..3) of w as an exact float.
[[maybe_unused]] __device__ __forceinline__ float byte_f(uint32_t w, int i) {
    return __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7440u | (uint32_t)i)) - 8388608.0f;
}

__device__ __forceinline__ int comp(const int4 &v, int i) {
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}
__device__ __forceinline__ uint32_t ucomp(const uint4 &v, int i) {
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// 8 consecutive activations (16- or 32-byte aligned) as fp32.
__device__ __forceinline__ void load_x8v(const float *p, float v[8]) {
    const float4 a = reinterpret_cast<const float4 *>(p)[0], b = reinterpret_cast<const float4 *>(p)[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void load_x8v(const __nv_bfloat16 *p, float v[8]) {
    const uint4 a = *reinterpret_cast<const uint4 *>(p);
    v[0] = bf16lo(a.x); v[1] = bf16hi(a.x); v[2] = bf16lo(a.y); v[3] = bf16hi(a.y);
    v[4] = bf16lo(a.z); v[5] = bf16hi(a.z); v[6] = bf16lo(a.w); v[7] = bf16hi(a.w);
}

// Stage TB activation rows for a CTA: slot t holds activation row tok[t]
// (zeros where tok[t] < 0).
//   codes  int16, layout [t][j16][unit ^ (j16 & 7)] of 16-byte groups (8
//          consecutive positions); units padded to a multiple of 8 so the XOR
//          swizzle stays in range.  Readers (lane = unit, fixed j16) and
//          writers (lanes = consecutive j16) are both free of bank conflicts.
//   scales s (power of two) and sums of x, one per 32-wide sub-block, layout
//          [t][unit][2C] so a lane reads its unit's 2C values as one vector.
// x ~= s * code with s = 2^(e-13), e = floor(log2 max|x|) over the sub-block,
// so |code| < 2^14 and the rounding error is <= 2^-14 of the sub-block max.
// A thread owns 8 consecutive positions; the four threads of a sub-block are
// adjacent lanes.  All loads of up to XIT rounds are issued before use.
template <int C, int TB, typename XT, typename F>
__device__ __forceinline__ void stage_activations(const GemvParams &p, const int *tok, int4 *xq,
                                                  float *xsc, float *xsum, int *nonfinite,
                                                  F &&after_first_loads) {
    constexpr int XIT = 4;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nthr = blockDim.x;
    const int per_row = p.k / 8, nitems = TB * per_row;
    const int nrounds = (nitems + nthr - 1) / nthr;
    const XT *x = static_cast<const XT *>(p.x);
    for (int r0 = 0; r0 < nrounds; r0 += XIT) {
        float v[XIT][8];
        #pragma unroll
        for (int it = 0; it < XIT; ++it) {
            const int idx = (r0 + it) * nthr + (int)threadIdx.x;
            const int t = idx / per_row, pos = (idx % per_row) * 8;
            if (r0 + it < nrounds && idx < nitems && tok[t] >= 0) {
                load_x8v(x + (int64_t)tok[t] * p.k + pos, v[it]);
            } else {
                #pragma unroll
                for (int e = 0; e < 8; ++e) v[it][e] = 0.f;
            }
        }
        if (r0 == 0) after_first_loads();
        #pragma unroll
        for (int it = 0; it < XIT; ++it) {
            if (r0 + it >= nrounds || (r0 + it) * nthr + warp * 32 >= nitems) break;  // warp-uniform
            const int idx = (r0 + it) * nthr + (int)threadIdx.x;
            float amax = 0.f, sum = 0.f;
            bool nf = false;   // an infinity or NaN: the call takes the exact path
            #pragma unroll
            for (int e = 0; e < 8; ++e) {
                amax = fmaxf(amax, fabsf(v[it][e]));
                sum += v[it][e];
                nf |= !(fabsf(v[it][e]) <= 3.402823466e38f);
            }
            #pragma unroll
            for (int o = 1; o < 4; o <<= 1) {
                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
                sum += __shfl_xor_sync(0xffffffffu, sum, o);
            }
            if (__any_sync(0xffffffffu, nf) && lane == 0) *nonfinite = 1;
            if (idx >= nitems) continue;
            int e = (int)((__float_as_uint(amax) >> 23) & 0xFF) - 127;  // floor(log2 amax)
            e = max(e, -100);
            const float inv_s = __uint_as_float((uint32_t)(13 - e + 127) << 23);  // 2^(13-e)
            const float sc = __uint_as_float((uint32_t)(e - 13 + 127) << 23);     // 2^(e-13)
            int q[8];
            #pragma unroll
            for (int k = 0; k < 8; ++k) q[k] = __float2int_rn(v[it][k] * inv_s);
            const int t = idx / per_row, pos = (idx % per_row) * 8;
            const int u = pos / (64 * C), within = pos % (64 * C), j16 = within / 8;
            int4 packed;
            packed.x = (int)__byte_perm((uint32_t)q[0], (uint32_t)q[1], 0x5410);
            packed.y = (int)__byte_perm((uint32_t)q[2], (uint32_t)q[3], 0x5410);
            packed.z = (int)__byte_perm((uint32_t)q[4], (uint32_t)q[5], 0x5410);
            packed.w = (int)__byte_perm((uint32_t)q[6], (uint32_t)q[7], 0x5410);
            xq[((int64_t)t * 8 * C + j16) * p.units_pad + (u ^ (j16 & 7))] = packed;
            if ((lane & 3) == 0) {
                const int si = (t * p.units + u) * 2 * C + within / 32;
                xsc[si] = sc;
                xsum[si] = sum;
            }
        }
    }
}

template <int C> struct Vec;
template <> struct Vec<1> {
    float v[2];
    __device__ __forceinline__ void load(const float *p) {
        const float2 a = *reinterpret_cast<const float2 *>(p);
        v[0] = a.x; v[1] = a.y;
    }
};
template <> struct Vec<2> {
    float v[4];
    __device__ __forceinline__ void load(const float *p) {
        const float4 a = *reinterpret_cast<const float4 *>(p);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    }
};
template <> struct Vec<4> {
    float v[8];
    __device__ __forceinline__ void load(const float *p) {
        const float4 a = reinterpret_cast<const float4 *>(p)[0], b = reinterpret_cast<const float4 *>(p)[1];
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
};

// One pass of a CTA over weight rows [row_begin, row_end) of `w` with TB
// activation slots: slot t multiplies activation row tok[t] (none if < 0) and
// writes output row yrow[t].  XREG: the lane's activation codes live in
// registers (one slot, at most 32 units of at most 2 chunks, K <= 4096).
// `pass` counts earlier passes of this CTA over the same row range: the ring's
// barriers are initialised in pass 0 only and their phases run on across
// passes (a live mbarrier is never initialised again).  Returns false if a
// wait gave up (the device error word is set).
template <int C, int TB, int R, bool XREG, typename XT, typename YT>
__device__ __forceinline__ bool gemv_pass(const GemvParams &p, const uint8_t *w, int row_begin,
                                          int row_end, const int *tok, const int64_t *yrow,
                                          uint8_t *smem, int *nonfinite, int pass) {
    int4 *xq = reinterpret_cast<int4 *>(smem);
    float *xsc = reinterpret_cast<float *>(smem + p.xq_bytes);
    float *xsum = reinterpret_cast<float *>(smem + p.xq_bytes + p.xs_bytes);
    uint8_t *ring = smem + p.xq_bytes + 2 * p.xs_bytes;
    uint64_t *full = reinterpret_cast<uint64_t *>(ring + (size_t)p.warps * p.slots * p.row_bytes);

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int my_rows = warp < row_end - row_begin ? (row_end - row_begin - warp + p.warps - 1) / p.warps : 0;
    uint8_t *my_ring = ring + (size_t)warp * p.slots * p.row_bytes;
    uint64_t *my_full = full + warp * p.slots;
    const int64_t row_bytes = p.row_bytes;
    // Fills of this warp's ring before this pass (every pass has my_rows rows).
    const int base = pass * my_rows;

    if (pass == 0) {
        if (lane == 0) {
            for (int s = 0; s < p.slots; ++s) mbar_init(&my_full[s], 1);
            fence_mbar_init();
        }
        __syncwarp();
    }
    auto issue = [&](int i) {
        const int slot = (base + i) % p.slots;
        const int64_t r = row_begin + warp + (int64_t)i * p.warps;
        mbar_arrive_expect_tx(&my_full[slot], (uint32_t)row_bytes);
        bulk_g2s(my_ring + slot * row_bytes, w + r * row_bytes, (uint32_t)row_bytes, &my_full[slot]);
    };
    // Let the next kernel on the stream be scheduled now: it only prefetches
    // constant weights before its own griddepcontrol.wait, which waits for
    // this grid to complete.
    griddep_launch_dependents();
    // Constant weights: before waiting for the preceding kernel, copy this
    // warp's first rows straight into its slots and start the CTA's other
    // rows towards L2.  (A CTA fits beside the preceding kernel's CTA, so
    // this runs while that kernel is still computing.)
    const int first = min(p.slots, my_rows);
    auto prefetch_rest = [&]() {  // rows beyond the ring's first fill, towards L2
        if (threadIdx.x == 0 && (row_end - row_begin) > p.slots * p.warps) {
            const int64_t bytes = (int64_t)(row_end - row_begin) * row_bytes;
            const uint8_t *src = w + (int64_t)row_begin * row_bytes;
            for (int64_t off = 0; off < bytes; off += 32768)
                prefetch_l2(src + off, (uint32_t)(bytes - off < 32768 ? bytes - off : 32768));
        }
    };
    // An ordered call with constant weights issues its row copies before
    // waiting for the preceding kernel (early mode makes one pass).
    const bool copies_first = p.early && !p.indep;
    if (copies_first) {
        if (lane == 0)
            for (int i = 0; i < first; ++i) issue(i);
        prefetch_rest();
    }
    if (!p.indep) griddep_wait();
    // Otherwise the activation loads go out first (they gate every row; an
    // independent call's are ready at once) and the row copies follow right
    // behind them.  An independent call asks L2 for nothing more: its ring
    // keeps enough bytes in flight (an L2 prefetch of its rows, before or
    // after staging, measured slower).
    stage_activations<C, TB, XT>(p, tok, xq, xsc, xsum, nonfinite, [&]() {
        if (!copies_first && lane == 0) {
            fence_proxy_async_smem();  // generic reads of the slots in an earlier pass
            for (int i = 0; i < first; ++i) issue(i);
        }
    });
    __syncthreads();
    // Non-finite activations (block-uniform): every weight is decoded to fp32
    // and multiplied by the activation itself, so that infinities and NaNs
    // combine with the weights' signs and zeros as IEEE arithmetic does (the
    // 16-bit codes cannot hold them).  The ring is consumed as usual.
    if (*nonfinite) {
        const XT *x = static_cast<const XT *>(p.x);
        YT *y = static_cast<YT *>(p.y);
        for (int i = 0; i < my_rows; ++i) {
            const int ii = base + i, slot = ii % p.slots;
            const uint32_t par = (uint32_t)(ii / p.slots) & 1u;
            if (!__all_sync(0xffffffffu, mbar_wait(&my_full[slot], par, p.err))) return false;
            const uint8_t *rp = my_ring + slot * row_bytes;
            float acc[TB];
            #pragma unroll
            for (int t = 0; t < TB; ++t) acc[t] = 0.f;
            for (int u8 = lane; u8 < p.nb * Unit<KQ_Q4_K>::PER_BLOCK; u8 += 32) {   // weights 8 u8 ..
                const int b = u8 / Unit<KQ_Q4_K>::PER_BLOCK;
                float wv[8];
                Unit<KQ_Q4_K>::decode(rp + b * 144, u8 - b * Unit<KQ_Q4_K>::PER_BLOCK, wv);
                #pragma unroll
                for (int t = 0; t < TB; ++t) {
                    if (tok[t] < 0) continue;
                    float xv[8];
                    load_x8v(x + (int64_t)tok[t] * p.k + 8 * u8, xv);
                    #pragma unroll
                    for (int j = 0; j < 8; ++j) acc[t] = fmaf(wv[j], xv[j], acc[t]);
                }
            }
            #pragma unroll
            for (int t = 0; t < TB; ++t) {
                #pragma unroll
                for (int o = 16; o > 0; o >>= 1) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], o);
            }
            const int64_t row = row_begin + warp + (int64_t)i * p.warps;
            #pragma unroll
            for (int t = 0; t < TB; ++t)
                if (lane == 0 && tok[t] >= 0) store_out(y + yrow[t] * p.n + row, acc[t]);
            __syncwarp();
            if (lane == 0 && i + p.slots < my_rows) {
                fence_proxy_async_smem();
                issue(i + p.slots);
            }
        }
        return true;
    }

    // Lane constants: which chunks of a block this lane's units cover, which
    // form of the packed scale bytes they use, and which byte of that word.
    constexpr int UPB = 4 / C;  // units per block
    const int c0 = (lane % UPB) * C;
    const bool hi_form = (2 * c0) >= 4;
    uint32_t sel[2 * C];
    #pragma unroll
    for (int jj = 0; jj < 2 * C; ++jj) sel[jj] = 0x7440u | (uint32_t)((2 * c0 + jj) & 3);

    int4 xr[XREG ? 8 * C : 1];
    Vec<C> sxr, ssr;
    if constexpr (XREG) {
        const int u = lane < p.units ? lane : 0;
        #pragma unroll
        for (int j16 = 0; j16 < 8 * C; ++j16) xr[j16] = xq[j16 * p.units_pad + (u ^ (j16 & 7))];
        sxr.load(xsc + u * 2 * C);
        ssr.load(xsum + u * 2 * C);
    }

    YT *y = static_cast<YT *>(p.y);
    for (int i = 0; i < my_rows; i += R) {
        const int nr = min(R, my_rows - i);  // rows in this step (warp-uniform)
        const uint8_t *rowp[R];
        #pragma unroll
        for (int r = 0; r < R; ++r) {
            const int ii = base + i + min(r, nr - 1);
            const int slot = ii % p.slots;
            if (r < nr) {
                // a landed row costs one non-blocking poll (measured faster than
                // going straight to the suspending wait); one outcome per warp
                const uint32_t par = (uint32_t)(ii / p.slots) & 1u;
                if (!__all_sync(0xffffffffu, mbar_test_wait(&my_full[slot], par) || mbar_wait(&my_full[slot], par, p.err)))
                    return false;
            }
            rowp[r] = my_ring + slot * row_bytes;
        }
        float acc[R][TB];
        #pragma unroll
        for (int r = 0; r < R; ++r)
            #pragma unroll
            for (int t = 0; t < TB; ++t) acc[r][t] = 0.f;
        for (int u = lane; u < p.units; u += 32) {
            const int blk_off = (u / UPB) * 144;
            int ia[R][TB][2 * C];
            #pragma unroll
            for (int r = 0; r < R; ++r)
                #pragma unroll
                for (int t = 0; t < TB; ++t)
                    #pragma unroll
                    for (int j = 0; j < 2 * C; ++j) ia[r][t][j] = 0;
            #pragma unroll
            for (int c = 0; c < C; ++c) {
                const int cc = c0 + c;
                uint4 q0[R], q1[R];
                #pragma unroll
                for (int r = 0; r < R; ++r) {
                    q0[r] = *reinterpret_cast<const uint4 *>(rowp[r] + blk_off + 16 + 32 * cc);
                    q1[r] = *reinterpret_cast<const uint4 *>(rowp[r] + blk_off + 32 + 32 * cc);
                }
                #pragma unroll
                for (int g = 0; g < 4; ++g) {  // quant words 2g, 2g+1 of this chunk
                    int4 xl[TB], xh[TB];
                    #pragma unroll
                    for (int t = 0; t < TB; ++t) {
                        if constexpr (XREG) {
                            xl[t] = xr[8 * c + g];
                            xh[t] = xr[8 * c + 4 + g];
                        } else {
                            const int base = t * 8 * C + 8 * c + g;
                            xl[t] = xq[base * p.units_pad + (u ^ g)];
                            xh[t] = xq[(base + 4) * p.units_pad + (u ^ (g + 4))];
                        }
                    }
                    #pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) {
                        const int ww = 2 * g + h2;
                        #pragma unroll
                        for (int r = 0; r < R; ++r) {
                            const uint32_t v = ww < 4 ? ucomp(q0[r], ww) : ucomp(q1[r], ww - 4);
                            const uint32_t lo = v & 0x0F0F0F0Fu, hi = v & 0xF0F0F0F0u;
                            #pragma unroll
                            for (int t = 0; t < TB; ++t) {
                                int a = ia[r][t][2 * c], bb = ia[r][t][2 * c + 1];
                                a = dp2a_lo(comp(xl[t], 2 * h2), lo, a);
                                a = dp2a_hi(comp(xl[t], 2 * h2 + 1), lo, a);
                                bb = dp2a_lo(comp(xh[t], 2 * h2), hi, bb);
                                bb = dp2a_hi(comp(xh[t], 2 * h2 + 1), hi, bb);
                                ia[r][t][2 * c] = a;
                                ia[r][t][2 * c + 1] = bb;
                            }
                        }
                    }
                }
            }
            Vec<C> sx[TB], ss[TB];
            #pragma unroll
            for (int t = 0; t < TB; ++t) {
                if constexpr (XREG) {
                    sx[t] = sxr;
                    ss[t] = ssr;
                } else {
                    sx[t].load(xsc + (t * p.units + u) * 2 * C);
                    ss[t].load(xsum + (t * p.units + u) * 2 * C);
                }
            }
            #pragma unroll
            for (int r = 0; r < R; ++r) {
                const uint4 h = *reinterpret_cast<const uint4 *>(rowp[r] + blk_off);
                const float d = half_bits_to_float(h.x), dmin = half_bits_to_float(h.x >> 16);
                // packed 6-bit scale and min bytes of sub-blocks 0..3 (lo) / 4..7 (hi)
                uint32_t scw_lo = h.y & 0x3F3F3F3Fu, mw_lo = h.z & 0x3F3F3F3Fu;
                uint32_t scw_hi = (h.w & 0x0F0F0F0Fu) | ((h.y >> 2) & 0x30303030u);
                uint32_t mw_hi = ((h.w >> 4) & 0x0F0F0F0Fu) | ((h.z >> 2) & 0x30303030u);
                #pragma unroll
                for (int jj = 0; jj < 2 * C; ++jj) {
                    // C == 4 covers both forms; otherwise the lane uses one.
                    const bool hf = (C == 4) ? (jj >= 4) : hi_form;
                    const uint32_t scw = hf ? scw_hi : scw_lo, mw = hf ? mw_hi : mw_lo;
                    const float scf = __uint_as_float(__byte_perm(scw, 0x4B000000u, sel[jj])) - 8388608.0f;
                    const float mf = __uint_as_float(__byte_perm(mw, 0x4B000000u, sel[jj])) - 8388608.0f;
                    const float a = d * scf * ((jj & 1) ? 0.0625f : 1.0f);
                    const float bm = dmin * mf;
                    #pragma unroll
                    for (int t = 0; t < TB; ++t) {
                        float v = acc[r][t];
                        v = fmaf(a * sx[t].v[jj], (float)ia[r][t][jj], v);
                        v = fmaf(-bm, ss[t].v[jj], v);
                        acc[r][t] = v;
                    }
                }
            }
        }
        #pragma unroll
        for (int r = 0; r < R; ++r)
            #pragma unroll
            for (int t = 0; t < TB; ++t) {
                float v = acc[r][t];
                #pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                acc[r][t] = v;
            }
        #pragma unroll
        for (int r = 0; r < R; ++r) {
            if (r < nr) {
                const int64_t row = row_begin + warp + (int64_t)(i + r) * p.warps;
                if (lane < TB && tok[lane] >= 0) {
                    float v = acc[r][0];
                    #pragma unroll
                    for (int t = 1; t < TB; ++t)
                        if (lane == t) v = acc[r][t];
                    store_out(y + yrow[lane] * p.n + row, v);
                }
            }
        }
        __syncwarp();
        if (lane == 0) {
            fence_proxy_async_smem();  // generic reads of the slots before async refills
            for (int r = 0; r < nr; ++r)
                if (i + r + p.slots < my_rows) issue(i + r + p.slots);
        }
    }
    return true;
}

template <int C, int TB, int R, bool XREG, int MINB, typename XT, typename YT>
__global__ void __launch_bounds__(MINB == 1 ? 32 * GEMV_MAX_WARPS : 32 * GEMV_HALF_MAX_WARPS, MINB)
    gemv_q4k_kernel(const GemvParams p) {
    static_assert(MINB == 1 || MINB == GEMV_HALF_BLOCKS, "whole-SM or shared-SM build");
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ int s_tok[TB];
    __shared__ int64_t s_yrow[TB];
    __shared__ int s_nonfinite;
    const int row_begin = blockIdx.x * p.rows_per_cta;
    const int row_end = min(p.n, row_begin + p.rows_per_cta);
    if (row_begin >= row_end) return;
    if (threadIdx.x < TB) {
        s_tok[threadIdx.x] = (int)threadIdx.x < p.m ? (int)threadIdx.x : -1;
        s_yrow[threadIdx.x] = threadIdx.x;
    }
    if (threadIdx.x == 0) s_nonfinite = 0;
    __syncthreads();
    gemv_pass<C, TB, R, XREG, XT, YT>(p, p.w, row_begin, row_end, s_tok, s_yrow, smem, &s_nonfinite, 0);
    // An independent call still completes after the work before it, so that
    // stream order holds for whatever follows.
    if (p.indep) griddep_wait();
}

int chunks_per_unit(int nb) { return nb >= 32 ? 4 : nb >= 16 ? 2 : 1; }
int tb_for(int64_t m) { return m <= 1 ? 1 : m <= 2 ? 2 : m <= 4 ? 4 : 8; }
#ifndef KQ_GEMV_ROWS_PER_STEP_1
#define KQ_GEMV_ROWS_PER_STEP_1 2   // weight rows per step with one activation row
#endif
int rows_per_step(int tb) { return tb == 1 ? KQ_GEMV_ROWS_PER_STEP_1 : tb <= 2 ? 2 : 1; }

bool plan_gemv(int type, int64_t n, int64_t k, int64_t m, int num_sms, int max_warps,
               int smem_limit, int max_slots, GemvParams *p) {
    if (type != KQ_Q4_K) return false;
    if (m < 1 || m > 8 || n < 1 || n > INT32_MAX / 2 || k > (1 << 20)) return false;
    const int tb = tb_for(m), R = rows_per_step(tb);
    const int nb = (int)(k / 256);
    const int C = chunks_per_unit(nb);
    const int units = nb * 4 / C, units_pad = (units + 7) / 8 * 8;
    const int64_t row_bytes = (int64_t)nb * 144;
    const int rows_per_cta = (int)((n + num_sms - 1) / num_sms);
    const size_t xq_bytes = (size_t)tb * 8 * C * units_pad * 16;
    const size_t xs_bytes = (size_t)tb * units * 2 * C * 4;
    const size_t fixed = xq_bytes + 2 * xs_bytes;
    if (fixed + 1024 >= (size_t)smem_limit) return false;
    int warps = rows_per_cta < max_warps ? rows_per_cta : max_warps;
    for (; warps >= 1; --warps) {
        const int rows_per_warp = (rows_per_cta + warps - 1) / warps;
        const int want = rows_per_warp < max_slots ? rows_per_warp : max_slots;
        const int min_slots = rows_per_warp < R ? rows_per_warp : R;
        int slots = want;
        while (slots > min_slots && fixed + (size_t)warps * slots * (row_bytes + 8) > (size_t)smem_limit)
            --slots;
        if (fixed + (size_t)warps * slots * (row_bytes + 8) <= (size_t)smem_limit) {
            p->nb = nb; p->units = units; p->units_pad = units_pad; p->rows_per_cta = rows_per_cta;
            p->warps = warps; p->slots = slots; p->row_bytes = (int)row_bytes;
            p->xq_bytes = (int)xq_bytes; p->xs_bytes = (int)xs_bytes;
            p->n = (int)n; p->k = (int)k; p->m = (int)m;
            return true;
        }
    }
    return false;
}

template <int C, int TB, bool XREG, typename XT, typename YT>
cudaError_t launch_q4k(GemvParams p, GemvOrder order, cudaStream_t s) {
    // half-SM build when the plan fits it (independent calls)
    constexpr int R = TB == 1 ? KQ_GEMV_ROWS_PER_STEP_1 : TB <= 2 ? 2 : 1;
    auto kern = p.warps <= GEMV_HALF_MAX_WARPS && order == GemvOrder::kIndependent
                    ? gemv_q4k_kernel<C, TB, R, XREG, GEMV_HALF_BLOCKS, XT, YT>
                    : gemv_q4k_kernel<C, TB, R, XREG, 1, XT, YT>;
    const size_t smem = (size_t)p.xq_bytes + 2 * (size_t)p.xs_bytes +
                        (size_t)p.warps * p.slots * ((size_t)p.row_bytes + 8);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    // the whole shared-memory carveout, so that the shared-SM CTAs fit side by side
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((p.n + p.rows_per_cta - 1) / p.rows_per_cta));
    cfg.blockDim = dim3(32 * p.warps);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    // Programmatic overlap with the preceding kernel is always allowed: the
    // kernel reads nothing produced by earlier work before griddepcontrol.wait,
    // except the weights when the caller declared them constant, and waits
    // not at all when the caller declared the call independent.
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    p.early = order != GemvOrder::kStream ? 1 : 0;
    p.indep = order == GemvOrder::kIndependent ? 1 : 0;
    p.err = error_word();
    return cudaLaunchKernelEx(&cfg, kern, p);
}

template <int C, typename XT, typename YT>
cudaError_t dispatch_tb(GemvParams p, int tb, GemvOrder order, cudaStream_t s) {
    switch (tb) {
    case 1:
        // Activation codes in registers, except for an ordered call with
        // constant weights: its rows have landed by the time the activations
        // are staged, and reading the codes from shared memory per row
        // shortens that critical path (measured 5.05 -> 4.68 us per call at
        // 4096 x 4096; the other orderings are faster with registers).
        if (KQ_GEMV_XREG && C <= 2 && p.units <= 32 && order != GemvOrder::kConstWeights)
            return launch_q4k<C, 1, (KQ_GEMV_XREG && C <= 2), XT, YT>(p, order, s);
        return launch_q4k<C, 1, false, XT, YT>(p, order, s);
    case 2: return launch_q4k<C, 2, false, XT, YT>(p, order, s);
    case 4: return launch_q4k<C, 4, false, XT, YT>(p, order, s);
    default: return launch_q4k<C, 8, false, XT, YT>(p, order, s);
    }
}

template <typename XT, typename YT>
cudaError_t dispatch_c(GemvParams p, int tb, GemvOrder order, cudaStream_t s) {
    switch (chunks_per_unit(p.nb)) {
    case 4: return dispatch_tb<4, XT, YT>(p, tb, order, s);
    case 2: return dispatch_tb<2, XT, YT>(p, tb, order, s);
    default: return dispatch_tb<1, XT, YT>(p, tb, order, s);
    }
}

}  // namespace

bool gemv_supported(int type, int64_t n, int64_t k, int x_dtype, int64_t m) {
    (void)x_dtype;
    if (type == KQ_TQ1_G128) return m >= 1 && gemv_tq1_supported(n, k);
    GemvParams p;
    return m >= 1 && plan_gemv(type, n, k, m < 8 ? m : 8, sm_count(), GEMV_MAX_WARPS, GEMV_SMEM_LIMIT,
                               GEMV_MAX_SLOTS, &p);
}

// More than eight activation rows run as consecutive launches of up to eight
// rows each (the weights are streamed once per launch).
cudaError_t launch_gemv(int type, const void *w, int64_t n, int64_t k, const void *x, int xdt,
                        int64_t m, void *y, int ydt, GemvOrder order, cudaStream_t s) {
    if (type == KQ_TQ1_G128) return launch_gemv_tq1(w, n, k, x, xdt, m, y, ydt, order, s);
    const bool half = order == GemvOrder::kIndependent;
    const size_t xs = (xdt == KQ_F32 ? 4 : 2), ys = (ydt == KQ_F32 ? 4 : 2);
    for (int64_t m0 = 0; m0 < m; m0 += 8) {
        const int64_t mc = m - m0 < 8 ? m - m0 : 8;
        GemvParams p = {};
        const int tb = tb_for(mc);
        // independent calls take the half-SM plan when it fits, else a whole SM
        if (!(half && plan_gemv(type, n, k, mc, sm_count() / KQ_GEMV_SHARE_GRID_DIV, GEMV_HALF_MAX_WARPS,
                                GEMV_HALF_SMEM_LIMIT, GEMV_HALF_MAX_SLOTS, &p)) &&
            !plan_gemv(type, n, k, mc, sm_count(), GEMV_MAX_WARPS, GEMV_SMEM_LIMIT, GEMV_MAX_SLOTS, &p))
            return cudaErrorNotSupported;
        p.w = static_cast<const uint8_t *>(w);
        p.x = static_cast<const char *>(x) + (size_t)m0 * (size_t)k * xs;
        p.y = static_cast<char *>(y) + (size_t)m0 * (size_t)n * ys;
        cudaError_t e;
        if (xdt == KQ_F32) {
            e = ydt == KQ_F32 ? dispatch_c<float, float>(p, tb, order, s)
                              : dispatch_c<float, __nv_bfloat16>(p, tb, order, s);
        } else {
            e = ydt == KQ_F32 ? dispatch_c<__nv_bfloat16, float>(p, tb, order, s)
                              : dispatch_c<__nv_bfloat16, __nv_bfloat16>(p, tb, order, s);
        }
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace kq
