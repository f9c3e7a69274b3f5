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
// Per block the product is scale * sum_j (digit_j - 1) * x_j, an integer-
// weighted sum, so it runs on integer dot products:
//  * Activations are staged once per CTA as 16-bit fixed point per 128-wide
//    block (x ~= s * xq, s a power of two from the block's largest |x|,
//    |xq| < 2^14), laid out per code byte: byte j of block b gets one
//    16-byte record (xq[5j], xq[5j+1] | xq[5j+2], xq[5j+3] | xq[5j+4], 0 | 0)
//    so a lane reads the five activations of a byte with one 128-bit load.
//  * A 256-entry table in shared memory maps a code byte to its five digits
//    minus one as signed bytes (d0-1 .. d3-1 | d4-1, 0, 0, 0); illegal bytes
//    map to zeros.  A 64-bit load is served per half-warp, so the table is
//    replicated 16 times (lane l reads copy l % 16) and the lookups of
//    arbitrary bytes never share a bank.
//  * dp2a multiplies two 16-bit activations by two signed trits and
//    accumulates in int32 (|sum| < 2^21 per block: exact), then one fp32
//    multiply by s * scale per block.
//  * A warp takes two weight rows at a time, so one activation-record load
//    serves both (the shared-memory instruction queue is the limit: per code
//    byte one record load and one table load per row before).
//  * Weights are read straight from global memory, one block (28 bytes) per
//    lane and row, with the next blocks' words loaded before the current
//    ones are used; each CTA first asks L2 to prefetch its whole row range,
//    so the weights are on chip when the lanes reach them.  The lanes'
//    shared-memory loads, not the weight stream, bound the kernel (about a
//    sixth of the copy bandwidth).
#include "kq_ptx.cuh"
#include "kq_launch.h"

namespace kq {

namespace {

constexpr int TQ_BB = 28;            // bytes per block
constexpr int TQ_QK = 128;           // weights per block
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

__device__ __forceinline__ float load_x(const float *x, int64_t i) { return x[i]; }
__device__ __forceinline__ float load_x(const __nv_bfloat16 *x, int64_t i) {
    return __bfloat162float(x[i]);
}

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

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int row_begin = blockIdx.x * p.rows_per_cta;
    const int row_end = min(p.n, row_begin + p.rows_per_cta);
    if (row_begin >= row_end) return;
    const int64_t row_bytes = (int64_t)p.nb * TQ_BB;

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

bool gemv_tq1_supported(int64_t n, int64_t k) {
    if (k % TQ_QK || k > (1 << 22) || n < 1 || n > INT32_MAX / 2) return false;
    return tq1_smem_bytes(1, (int)(k / TQ_QK)) <= (size_t)TQ_SMEM_LIMIT;
}

// Up to two activation rows per launch (their staged records must fit next
// to the table); more rows run as consecutive launches.
cudaError_t launch_gemv_tq1(const void *w, int64_t n, int64_t k, const void *x, int xdt, int64_t m,
                            void *y, int ydt, GemvOrder order, cudaStream_t s) {
    if (!gemv_tq1_supported(n, k)) return cudaErrorNotSupported;
    const int nb = (int)(k / TQ_QK);
    const int tb_max = tq1_smem_bytes(2, nb) <= (size_t)TQ_SMEM_LIMIT ? 2 : 1;
    const size_t xs = (xdt == KQ_F32 ? 4 : 2), ys = (ydt == KQ_F32 ? 4 : 2);
    const int sms = sm_count();
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
