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
//    16 <= 256 picked by the host to balance waves over the SMs).
//  * Warp roles:  warp 0  TMA producer -- bf16 activation tiles (64 K x BN,
//                         128-byte swizzle) and raw Q4_K super-blocks
//                         (128 rows x 144 bytes) into shared-memory rings;
//                 warp 1  MMA issuer -- one thread issues tcgen05.mma
//                         (kind::f16, bf16 x bf16 -> fp32 in TMEM) and
//                         tcgen05.commit's to the stage / accumulator barriers;
//                 warps 2-5  epilogue -- tcgen05.ld from TMEM, convert, store;
//                 warps 6-13 decoders -- raw super-block bytes -> exact fp32
//                         weights (d*sc*q - dmin*m, one rounding) -> bf16
//                         (round to nearest even) written in the canonical
//                         K-major 128-byte-swizzled layout the MMA reads.
//  * Two TMEM accumulators (2 x BN columns) let the epilogue of tile i
//    overlap the main loop of tile i+1.
//  * Every mbarrier wait is bounded (kq_ptx.cuh): on timeout the kernel sets
//    the device error word and the waiting role stops; TMEM is released by
//    the allocating warp after a block barrier that every thread reaches.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "kq_decode.cuh"
#include "kq_ptx.cuh"
#include "kq_launch.h"

namespace kq {

namespace {

constexpr int BM = 128;            // weight rows per tile (MMA M)
constexpr int BK = 64;             // K per stage (one 128-byte swizzle atom of bf16)
constexpr int SB_BYTES = 144;      // Q4_K super-block
constexpr int RAW_STAGE_BYTES = BM * SB_BYTES;   // 18432
constexpr int A_STAGE_BYTES = BM * BK * 2;       // 16384
#ifndef KQ_GEMM_DEC_WARPS
#define KQ_GEMM_DEC_WARPS 16
#endif
constexpr int DEC_WARP0 = 6, DEC_WARPS = KQ_GEMM_DEC_WARPS;  // 8 or 16
constexpr int NUM_THREADS = (DEC_WARP0 + DEC_WARPS) * 32;
constexpr int EPI_WARP0 = 2;
constexpr int RAW_STAGES = 2;
constexpr int SMEM_BUDGET = 227 * 1024;

struct GemmParams {
    int n, k, m;
    int bn, m_tiles, n_tiles, tiles;
    int stages;  // depth of the shared stage ring (decoded weights + activations)
    int b_stage_bytes;
    void *y;
    unsigned int *err;
};

// ---- tcgen05 / TMA wrappers ----
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y,
                                            uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(dst_smem)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_addr(bar))
        : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t r[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (SBO), leading offset 16 bytes, sm_100 descriptor version 1.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)1 << 16;               // LBO = 16 B
    d |= (uint64_t)(1024 >> 4) << 32;     // SBO = 1024 B
    d |= (uint64_t)1 << 46;               // version
    d |= (uint64_t)2 << 61;               // SWIZZLE_128B
    return d;
}

// Instruction descriptor, kind::f16: bf16 A and B (K-major), fp32 D.
__host__ __device__ constexpr uint32_t idesc_bf16(int m, int n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) |
           ((uint32_t)(m >> 4) << 24);
}

__device__ __forceinline__ float half_f(uint32_t bits) { return half_bits_to_float(bits); }

// Byte i of w as an exact float (2^23 exponent trick).
__device__ __forceinline__ float byte_float(uint32_t w, int i) {
    return __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7440u | (uint32_t)i)) - 8388608.0f;
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}

template <typename YT>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_q4k_kernel(const __grid_constant__ CUtensorMap tmap_x,
                    const __grid_constant__ CUtensorMap tmap_w, const GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte alignment for the swizzled tiles
    uint8_t *smem = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);
    const int S = p.stages;
    uint8_t *a_ring = smem;                                    // S x 16 KB
    uint8_t *b_ring = a_ring + S * A_STAGE_BYTES;              // S x bn*128
    uint8_t *raw_ring = b_ring + S * p.b_stage_bytes;          // RAW_STAGES x 18 KB
    uint64_t *bars = reinterpret_cast<uint64_t *>(raw_ring + RAW_STAGES * RAW_STAGE_BYTES);
    uint64_t *full = bars;                   // [S]  TMA bytes + decoder warps -> MMA
    uint64_t *empty = full + S;              // [S]  MMA -> TMA, decoders
    uint64_t *raw_full = empty + S;          // [RAW] TMA -> decoders
    uint64_t *raw_empty = raw_full + RAW_STAGES;  // [RAW] decoders -> TMA
    uint64_t *acc_full = raw_empty + RAW_STAGES;  // [2] MMA -> epilogue
    uint64_t *acc_empty = acc_full + 2;           // [2] epilogue -> MMA
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_empty + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nk = p.k / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1 + DEC_WARPS);
            mbar_init(&empty[s], 1);
        }
        for (int r = 0; r < RAW_STAGES; ++r) {
            mbar_init(&raw_full[r], 1);
            mbar_init(&raw_empty[r], DEC_WARPS);
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
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    griddep_wait();

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        // Ring positions advance incrementally (no division in the issue
        // loop: this single thread must keep pace with the tensor core).
        if (lane == 0) {
            uint32_t slot = 0, phase = 0, rslot = 0, rphase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < p.tiles && ok; tile += gridDim.x) {
                const int n0 = (tile / p.m_tiles) * BM, m0 = (tile % p.m_tiles) * p.bn;
                for (int ks = 0; ks < nk; ++ks) {
                    if ((ks & 3) == 0) {  // raw super-block for this and the next 3 stages
                        ok = mbar_wait(&raw_empty[rslot], rphase ^ 1, p.err);
                        if (!ok) break;
                        mbar_arrive_expect_tx(&raw_full[rslot], RAW_STAGE_BYTES);
                        tma_load_2d(raw_ring + rslot * RAW_STAGE_BYTES, &tmap_w, (ks >> 2) * SB_BYTES, n0,
                                    &raw_full[rslot]);
                        if (++rslot == RAW_STAGES) { rslot = 0; rphase ^= 1; }
                    }
                    ok = mbar_wait(&empty[slot], phase ^ 1, p.err);
                    if (!ok) break;
                    mbar_arrive_expect_tx(&full[slot], p.b_stage_bytes);
                    tma_load_2d(b_ring + slot * p.b_stage_bytes, &tmap_x, ks * BK, m0, &full[slot]);
                    if (++slot == (uint32_t)S) { slot = 0; phase ^= 1; }
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        // One wait per stage (the stage's barrier collects the activation
        // tile's bytes and the eight decoder warps), four MMAs whose
        // descriptors only advance their start address, one commit that
        // frees the stage when the MMAs are done.
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(BM, p.bn);
            const uint64_t a_desc0 = sw128_desc(smem_addr(a_ring));
            const uint64_t b_desc0 = sw128_desc(smem_addr(b_ring));
            const uint32_t a_step = A_STAGE_BYTES >> 4, b_step = (uint32_t)p.b_stage_bytes >> 4;
            uint32_t slot = 0, phase = 0;
            uint64_t ad = a_desc0, bd = b_desc0;
            int tl = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < p.tiles && ok; tile += gridDim.x, ++tl) {
                const int acc = tl & 1;
                ok = mbar_wait(&acc_empty[acc], ((tl >> 1) & 1) ^ 1, p.err);
                if (!ok) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * 256);
                for (int ks = 0; ks < nk; ++ks) {
                    ok = mbar_wait(&full[slot], phase, p.err);
                    if (!ok) break;
                    mma_bf16(d_tmem, ad, bd, idesc, ks > 0 ? 1u : 0u);
                    mma_bf16(d_tmem, ad + 2, bd + 2, idesc, 1u);
                    mma_bf16(d_tmem, ad + 4, bd + 4, idesc, 1u);
                    mma_bf16(d_tmem, ad + 6, bd + 6, idesc, 1u);
                    mma_commit(&empty[slot]);  // frees the stage once these MMAs finish
                    if (++slot == (uint32_t)S) {
                        slot = 0;
                        phase ^= 1;
                        ad = a_desc0;
                        bd = b_desc0;
                    } else {
                        ad += a_step;
                        bd += b_step;
                    }
                }
                if (ok) mma_commit(&acc_full[acc]);
            }
        }
    } else if (warp < EPI_WARP0 + 4) {
        // ---------------- epilogue ----------------
        const int q = warp & 3;  // TMEM lane quadrant this warp may access
        YT *y = static_cast<YT *>(p.y);
        int tl = 0;
        for (int tile = blockIdx.x; tile < p.tiles; tile += gridDim.x, ++tl) {
            const int acc = tl & 1;
            const int n0 = (tile / p.m_tiles) * BM, m0 = (tile % p.m_tiles) * p.bn;
            if (!mbar_wait(&acc_full[acc], (tl >> 1) & 1, p.err)) break;
            tc_fence_after();
            const int n = n0 + 32 * q + lane;
            const uint32_t t_row = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(acc * 256);
            for (int c0 = 0; c0 < p.bn; c0 += 16) {
                uint32_t r[16];
                tmem_ld16(t_row + (uint32_t)c0, r);
                if (n < p.n) {
                    #pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int m = m0 + c0 + j;
                        if (m < p.m) store_out(y + (int64_t)m * p.n + n, __uint_as_float(r[j]));
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[acc]);
        }
    } else {
        // ---------------- decoders ----------------
        // DEC_WARPS * 32 threads share the 128 rows x 32 quant bytes of a
        // stage: QB = 32 * 128 / threads bytes each (16 or 8).  Eight
        // consecutive lanes take eight consecutive rows and the same byte
        // range, so the raw reads (rows 144 bytes apart) and the swizzled
        // 16-byte stores hit distinct bank groups.  A thread decodes both
        // nibbles of its bytes: low nibbles are K positions QB*part + 0.. of
        // the stage (sub-block 2cc), high nibbles K positions 32 + QB*part
        // + 0.. (sub-block 2cc+1).
        constexpr int PARTS = DEC_WARPS / 4;      // byte ranges per row: 2 or 4
        constexpr int QB = 32 / PARTS;            // quant bytes per thread: 16 or 8
        constexpr int NW = QB / 4;                // quant words per thread
        const int t = threadIdx.x - DEC_WARP0 * 32;
        const int r = 8 * (t / (8 * PARTS)) + (t & 7);   // weight row in the tile
        const int part = (t >> 3) % PARTS;               // which QB bytes
        const float2 magic = make_float2(-8388608.0f, -8388608.0f), one = make_float2(1.f, 1.f);
        uint32_t g = 0, rsb = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < p.tiles && ok; tile += gridDim.x) {
            for (int ks = 0; ks < nk && ok; ks += 4) {
                const int rs = rsb % RAW_STAGES;
                ok = mbar_wait(&raw_full[rs], (rsb / RAW_STAGES) & 1, p.err);
                if (!ok) break;
                const uint8_t *blk = raw_ring + rs * RAW_STAGE_BYTES + r * SB_BYTES;
                const uint4 hd = *reinterpret_cast<const uint4 *>(blk);
                const float d = half_f(hd.x), dmin = half_f(hd.x >> 16);
                // packed 6-bit scales / mins of sub-blocks 0..3 and 4..7
                const uint32_t sc_lo = hd.y & 0x3F3F3F3Fu, m_lo = hd.z & 0x3F3F3F3Fu;
                const uint32_t sc_hi = (hd.w & 0x0F0F0F0Fu) | ((hd.y >> 2) & 0x30303030u);
                const uint32_t m_hi = ((hd.w >> 4) & 0x0F0F0F0Fu) | ((hd.z >> 2) & 0x30303030u);
                #pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    const int s = g % S;
                    ok = mbar_wait(&empty[s], ((g / S) & 1) ^ 1, p.err);
                    if (!ok) break;
                    const uint32_t scw = cc < 2 ? sc_lo : sc_hi, mw = cc < 2 ? m_lo : m_hi;
                    const int b0 = (2 * cc) & 3;
                    // exact products: d*sc (17 bits), dmin*m (17 bits); high
                    // nibbles arrive as 16*q, so their scale is divided by 16
                    const float ds_lo = d * byte_float(scw, b0), dm_lo = dmin * byte_float(mw, b0);
                    const float ds_hi = d * byte_float(scw, b0 + 1) * 0.0625f;
                    const float dm_hi = dmin * byte_float(mw, b0 + 1);
                    const float2 dsl = make_float2(ds_lo, ds_lo), dml = make_float2(-dm_lo, -dm_lo);
                    const float2 dsh = make_float2(ds_hi, ds_hi), dmh = make_float2(-dm_hi, -dm_hi);
                    uint32_t qw[NW];
                    if constexpr (NW == 4) {
                        const uint4 v = *reinterpret_cast<const uint4 *>(blk + 16 + 32 * cc + QB * part);
                        qw[0] = v.x; qw[1] = v.y; qw[2] = v.z; qw[3] = v.w;
                    } else {
                        const uint2 v = *reinterpret_cast<const uint2 *>(blk + 16 + 32 * cc + QB * part);
                        qw[0] = v.x; qw[1] = v.y;
                    }
                    uint32_t lo_out[2 * NW], hi_out[2 * NW];
                    #pragma unroll
                    for (int wd = 0; wd < NW; ++wd) {
                        const uint32_t lo = qw[wd] & 0x0F0F0F0Fu, hi = qw[wd] & 0xF0F0F0F0u;
                        #pragma unroll
                        for (int pr = 0; pr < 2; ++pr) {
                            // bytes 2pr, 2pr+1 -> 2^23 + q (exact), minus 2^23 -> q
                            float2 fl = make_float2(
                                __uint_as_float(__byte_perm(lo, 0x4B000000u, 0x7440u + 2 * pr)),
                                __uint_as_float(__byte_perm(lo, 0x4B000000u, 0x7441u + 2 * pr)));
                            float2 fh = make_float2(
                                __uint_as_float(__byte_perm(hi, 0x4B000000u, 0x7440u + 2 * pr)),
                                __uint_as_float(__byte_perm(hi, 0x4B000000u, 0x7441u + 2 * pr)));
                            fl = ffma2(fl, one, magic);
                            fh = ffma2(fh, one, magic);
                            const float2 wl = ffma2(fl, dsl, dml);  // one rounding each
                            const float2 wh = ffma2(fh, dsh, dmh);
                            const __nv_bfloat162 bl = __floats2bfloat162_rn(wl.x, wl.y);
                            const __nv_bfloat162 bh = __floats2bfloat162_rn(wh.x, wh.y);
                            lo_out[2 * wd + pr] = *reinterpret_cast<const uint32_t *>(&bl);
                            hi_out[2 * wd + pr] = *reinterpret_cast<const uint32_t *>(&bh);
                        }
                    }
                    const uint32_t arow = smem_addr(a_ring + s * A_STAGE_BYTES + r * 128);
                    #pragma unroll
                    for (int j = 0; j < NW / 2; ++j) {  // 16-byte chunks: QB/8 low, QB/8 high
                        const int c_lo = (QB / 8) * part + j, c_hi = 4 + (QB / 8) * part + j;
                        st_shared_v4(arow + ((c_lo ^ (r & 7)) << 4), lo_out[4 * j], lo_out[4 * j + 1],
                                     lo_out[4 * j + 2], lo_out[4 * j + 3]);
                        st_shared_v4(arow + ((c_hi ^ (r & 7)) << 4), hi_out[4 * j], hi_out[4 * j + 1],
                                     hi_out[4 * j + 2], hi_out[4 * j + 3]);
                    }
                    fence_proxy_async_smem();  // make the generic writes visible to the MMA
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&full[s]);
                    ++g;
                }
                if (!ok) break;
                __syncwarp();
                if (lane == 0) mbar_arrive(&raw_empty[rs]);
                ++rsb;
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

// ---------------------------------------------------------------- host side
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

int num_sms() {
    static int cached[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    if (!cached[dev]) {
        int v = 0;
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
        cached[dev] = v > 0 ? v : 148;
    }
    return cached[dev];
}

// Choose BN (tokens per tile) minimising rounds * BN over the SMs, with a
// small charge per extra token tile (each one re-decodes the weight tile).
int pick_bn(int m, int n_tiles, int sms) {
#ifdef KQ_GEMM_FORCE_BN
    return KQ_GEMM_FORCE_BN;
#endif
    static const int cands[] = {256, 224, 192, 176, 160, 128, 112, 96, 80, 64, 48, 32, 16};
    int best = 256;
    double best_cost = 1e30;
    for (int bn : cands) {
        if (bn > 16 && bn >= 2 * m + 16) continue;  // far wider than the problem
        const int mt = (m + bn - 1) / bn;
        const long tiles = (long)mt * n_tiles;
        const long rounds = (tiles + sms - 1) / sms;
        const double cost = (double)rounds * (bn + 24);  // 24 ~ per-tile fixed cost in token units
        if (cost < best_cost) {
            best_cost = cost;
            best = bn;
        }
    }
    return best;
}

// Depth of the stage ring: as many (decoded A + activation B) stages as
// shared memory holds next to the raw super-block ring, at most six.
int stages_for(int bn) {
    const int per = A_STAGE_BYTES + bn * 128;
    const int st = (SMEM_BUDGET - 2048 - RAW_STAGES * RAW_STAGE_BYTES) / per;
    return st > 6 ? 6 : st;
}

}  // namespace

bool gemm_supported(int type, int64_t n, int64_t k, int x_dtype, int y_dtype) {
    if (type != KQ_Q4_K || x_dtype != KQ_BF16) return false;
    if (y_dtype != KQ_F32 && y_dtype != KQ_BF16) return false;
    if (k % 256 || k > (1 << 24) || n < 1 || n > (1 << 30)) return false;
    return encode_fn() != nullptr;
}

cudaError_t launch_gemm(int type, const void *w, int64_t n, int64_t k, const void *x, int64_t m,
                        void *y, int ydt, cudaStream_t s) {
    (void)type;
    auto enc = encode_fn();
    if (!enc || m < 1 || m > (1 << 30)) return cudaErrorNotSupported;
    const int sms = num_sms();
    GemmParams p;
    p.n = (int)n; p.k = (int)k; p.m = (int)m;
    p.n_tiles = (int)((n + BM - 1) / BM);
    p.bn = pick_bn((int)m, p.n_tiles, sms);
    p.m_tiles = (int)((m + p.bn - 1) / p.bn);
    p.tiles = p.n_tiles * p.m_tiles;
    p.stages = stages_for(p.bn);
    p.b_stage_bytes = p.bn * 128;
    p.y = y;
    p.err = error_word();

    CUtensorMap tx, tw;
    {
        cuuint64_t dims[2] = {(cuuint64_t)k, (cuuint64_t)m};
        cuuint64_t strides[1] = {(cuuint64_t)k * 2};
        cuuint32_t box[2] = {BK, (cuuint32_t)p.bn};
        cuuint32_t es[2] = {1, 1};
        if (enc(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(x), dims, strides, box,
                es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {
        const int64_t rb = (k / 256) * SB_BYTES;
        cuuint64_t dims[2] = {(cuuint64_t)rb, (cuuint64_t)n};
        cuuint64_t strides[1] = {(cuuint64_t)rb};
        cuuint32_t box[2] = {SB_BYTES, BM};
        cuuint32_t es[2] = {1, 1};
        if (enc(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(w), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    const size_t smem = 1024 + (size_t)p.stages * (A_STAGE_BYTES + p.b_stage_bytes) +
                        RAW_STAGES * RAW_STAGE_BYTES + 256;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(p.tiles < sms ? p.tiles : sms));
    cfg.blockDim = dim3(NUM_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (ydt == KQ_F32) {
        cudaError_t e = cudaFuncSetAttribute(gemm_q4k_kernel<float>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        return cudaLaunchKernelEx(&cfg, gemm_q4k_kernel<float>, tx, tw, p);
    }
    cudaError_t e = cudaFuncSetAttribute(gemm_q4k_kernel<__nv_bfloat16>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return cudaLaunchKernelEx(&cfg, gemm_q4k_kernel<__nv_bfloat16>, tx, tw, p);
}

}  // namespace kq
