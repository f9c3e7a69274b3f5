// kq_simple.cu -- decode-to-fp32 kernels: dequantize, the row gather, the
// plain CUDA-core product (any codec, any m, fp32 or bf16 x) and the TQ1
// legality scan.
//
// These kernels decode each weight exactly (kq_decode.cuh) and accumulate in
// fp32.  The plain product is the general-purpose path; the shape-specialised
// kernels (kq_gemv.cu, kq_gemm_sm100.cu) serve the measured workloads.
#include "kq_decode.cuh"
#include "kq_ptx.cuh"
#include "kq_launch.h"

namespace kq {

// ---------------------------------------------------------------- dequantize
// One thread per 8-weight unit; output rows are contiguous [rows, K].
template <int TYPE, typename OT>
__global__ void __launch_bounds__(256) dequant_kernel(const uint8_t *__restrict__ w, int64_t rows,
                                                      int64_t k, OT *__restrict__ out) {
    using G = Geom<TYPE>;
    using U = Unit<TYPE>;
    const int64_t nb = k / G::QK;
    const int64_t row_bytes = nb * G::BB;
    const int64_t units = rows * nb * U::PER_BLOCK;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < units;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int u = (int)(i % U::PER_BLOCK);
        const int64_t blk = i / U::PER_BLOCK;
        const int64_t r = blk / nb, bi = blk % nb;
        float v[8];
        U::decode(w + r * row_bytes + bi * G::BB, u, v);
        OT *o = out + r * k + bi * G::QK + 8 * u;
        if constexpr (sizeof(OT) == 4) {
            reinterpret_cast<float4 *>(o)[0] = make_float4(v[0], v[1], v[2], v[3]);
            reinterpret_cast<float4 *>(o)[1] = make_float4(v[4], v[5], v[6], v[7]);
        } else {
            OT t[8];
            #pragma unroll
            for (int j = 0; j < 8; ++j) store_out(&t[j], v[j]);
            *reinterpret_cast<uint4 *>(o) = *reinterpret_cast<const uint4 *>(t);
        }
    }
}

// ---------------------------------------------------------------- plain product
// One warp per (weight row, group of up to 4 activation rows).  Lanes stride
// over the row's 8-weight units (UNROLL units' loads in flight at a time;
// each lane's sums keep their order, so the result does not depend on it);
// a warp shuffle reduces the partial sums.
template <int TYPE, int UNROLL, typename XT, typename YT>
__device__ __forceinline__ void simple_matmul_rows(const uint8_t *__restrict__ w, int64_t n, int64_t k,
                                                   const XT *__restrict__ x, int64_t m, YT *__restrict__ y) {
    using G = Geom<TYPE>;
    using U = Unit<TYPE>;
    constexpr int TB = 4;
    const int lane = threadIdx.x & 31;
    const int64_t warp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int64_t mgroups = (m + TB - 1) / TB;
    if (warp >= n * mgroups) return;
    const int64_t row = warp % n, mg = warp / n;
    const int64_t nb = k / G::QK;
    const uint8_t *wr = w + row * nb * G::BB;
    float acc[TB] = {0.f, 0.f, 0.f, 0.f};
    const int64_t units = nb * U::PER_BLOCK;
    #pragma unroll UNROLL
    for (int64_t i = lane; i < units; i += 32) {
        const int64_t bi = i / U::PER_BLOCK;
        const int u = (int)(i % U::PER_BLOCK);
        float wv[8];
        U::decode(wr + bi * G::BB, u, wv);
        const int64_t col = bi * G::QK + 8 * u;
        #pragma unroll
        for (int t = 0; t < TB; ++t) {
            const int64_t xm = mg * TB + t;
            if (xm < m) {
                float xv[8];
                load_x8(x + xm * k + col, xv);
                #pragma unroll
                for (int j = 0; j < 8; ++j) acc[t] = fmaf(wv[j], xv[j], acc[t]);
            }
        }
    }
    #pragma unroll
    for (int t = 0; t < TB; ++t) {
        float v = acc[t];
        #pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        const int64_t xm = mg * TB + t;
        if (lane == 0 && xm < m) store_out(y + xm * n + row, v);
    }
}

// Launched as a programmatic dependent: it lets the next kernel launch at
// once and waits for the preceding one before touching memory, or, for an
// independent call (`indep`), only before it completes (stream order of
// completion), so that consecutive independent calls overlap.  An ordered
// Q8_0 call with one activation row keeps four units' loads in flight per
// lane (4096 x 4096: 18.7 -> 15.8 us); independent calls, which overlap one
// another, calls with more rows and the other codecs keep one (four
// measured 9.5 -> 12.5 us for independent calls, 68.2 -> 82.8 us for 16
// rows, and for Q2_K's one row 22.9 -> 23.4 us).
template <int TYPE, int UNROLL, typename XT, typename YT>
__global__ void __launch_bounds__(256) simple_matmul_kernel(
    const uint8_t *__restrict__ w, int64_t n, int64_t k, const XT *__restrict__ x, int64_t m,
    YT *__restrict__ y, int indep) {
    griddep_launch_dependents();
    if (!indep) griddep_wait();
    simple_matmul_rows<TYPE, UNROLL>(w, n, k, x, m, y);
    if (indep) griddep_wait();
}

// ---------------------------------------------------------------- row gather
// One thread per 8-weight unit of an output row: out[t] = decode of row
// ids[t]; an id outside [0, rows) gives a zero row and flags the error word.
template <int TYPE, typename OT>
__global__ void __launch_bounds__(256) get_rows_kernel(const uint8_t *__restrict__ w, int64_t rows, int64_t k,
                                                       const int32_t *__restrict__ ids, int64_t n_ids,
                                                       OT *__restrict__ out, unsigned int *err) {
    using G = Geom<TYPE>;
    using U = Unit<TYPE>;
    const int64_t nb = k / G::QK;
    const int64_t per_row = nb * U::PER_BLOCK;
    const int64_t units = n_ids * per_row;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < units;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = i / per_row, r = i - t * per_row;
        const int64_t bi = r / U::PER_BLOCK;
        const int u = (int)(r - bi * U::PER_BLOCK);
        const int32_t id = __ldg(ids + t);
        float v[8];
        if (id < 0 || (int64_t)id >= rows) {
            #pragma unroll
            for (int j = 0; j < 8; ++j) v[j] = 0.f;
            if (r == 0) atomicOr(err, ERR_BAD_ID);
        } else {
            U::decode(w + (int64_t)id * nb * G::BB + bi * G::BB, u, v);
        }
        OT *o = out + t * k + bi * G::QK + 8 * u;
        if constexpr (sizeof(OT) == 4) {
            reinterpret_cast<float4 *>(o)[0] = make_float4(v[0], v[1], v[2], v[3]);
            reinterpret_cast<float4 *>(o)[1] = make_float4(v[4], v[5], v[6], v[7]);
        } else {
            OT tt[8];
            #pragma unroll
            for (int j = 0; j < 8; ++j) store_out(&tt[j], v[j]);
            *reinterpret_cast<uint4 *>(o) = *reinterpret_cast<const uint4 *>(tt);
        }
    }
}

// ---------------------------------------------------------------- TQ1 scan
__global__ void tq1_scan_kernel(const uint8_t *__restrict__ w, int64_t blocks,
                                unsigned long long *first_bad) {
    for (int64_t b = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; b < blocks;
         b += (int64_t)gridDim.x * blockDim.x) {
        const uint8_t *p = w + b * 28;
        bool bad = p[25] > 26;
        #pragma unroll
        for (int i = 0; i < 25; ++i) bad |= p[i] > 242;
        if (bad) atomicMin(first_bad, (unsigned long long)b);
    }
}

// ---------------------------------------------------------------- launchers
static int grid_for(int64_t work, int threads) {
    int64_t g = (work + threads - 1) / threads;
    const int64_t cap = 148LL * 16;
    if (g > cap) g = cap;
    if (g < 1) g = 1;
    return (int)g;
}

template <int TYPE>
static cudaError_t dequant_t(const void *w, int64_t rows, int64_t k, void *out, int dt,
                             cudaStream_t s) {
    const int64_t units = rows * (k / Geom<TYPE>::QK) * Unit<TYPE>::PER_BLOCK;
    const int g = grid_for(units, 256);
    const uint8_t *wp = static_cast<const uint8_t *>(w);
    if (dt == KQ_F32)
        dequant_kernel<TYPE, float><<<g, 256, 0, s>>>(wp, rows, k, static_cast<float *>(out));
    else if (dt == KQ_BF16)
        dequant_kernel<TYPE, __nv_bfloat16><<<g, 256, 0, s>>>(wp, rows, k,
                                                              static_cast<__nv_bfloat16 *>(out));
    else
        dequant_kernel<TYPE, __half><<<g, 256, 0, s>>>(wp, rows, k, static_cast<__half *>(out));
    return cudaGetLastError();
}

cudaError_t launch_dequant(int type, const void *w, int64_t rows, int64_t k, void *out, int dt,
                           cudaStream_t s) {
    switch (type) {
    case KQ_Q8_0: return dequant_t<KQ_Q8_0>(w, rows, k, out, dt, s);
    case KQ_Q4_K: return dequant_t<KQ_Q4_K>(w, rows, k, out, dt, s);
    case KQ_Q2_K: return dequant_t<KQ_Q2_K>(w, rows, k, out, dt, s);
    case KQ_Q5_K: return dequant_t<KQ_Q5_K>(w, rows, k, out, dt, s);
    case KQ_Q6_K: return dequant_t<KQ_Q6_K>(w, rows, k, out, dt, s);
    case KQ_TQ1_G128: return dequant_t<KQ_TQ1_G128>(w, rows, k, out, dt, s);
    default: return cudaErrorInvalidValue;
    }
}

template <int TYPE, typename XT, typename YT>
static cudaError_t simple_t(const void *w, int64_t n, int64_t k, const void *x, int64_t m, void *y,
                            bool indep, cudaStream_t s) {
    const int64_t warps = n * ((m + 3) / 4);
    const int64_t blocks = (warps + 7) / 8;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)blocks);
    cfg.blockDim = dim3(256);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    auto kern = (TYPE == KQ_Q8_0 && !indep && m == 1) ? simple_matmul_kernel<TYPE, 4, XT, YT>
                                                      : simple_matmul_kernel<TYPE, 1, XT, YT>;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<const uint8_t *>(w), n, k, static_cast<const XT *>(x), m,
                              static_cast<YT *>(y), indep ? 1 : 0);
}

template <int TYPE>
static cudaError_t simple_xy(const void *w, int64_t n, int64_t k, const void *x, int xdt, int64_t m,
                             void *y, int ydt, bool indep, cudaStream_t s) {
    if (xdt == KQ_F32) {
        if (ydt == KQ_F32) return simple_t<TYPE, float, float>(w, n, k, x, m, y, indep, s);
        return simple_t<TYPE, float, __nv_bfloat16>(w, n, k, x, m, y, indep, s);
    }
    if (ydt == KQ_F32) return simple_t<TYPE, __nv_bfloat16, float>(w, n, k, x, m, y, indep, s);
    return simple_t<TYPE, __nv_bfloat16, __nv_bfloat16>(w, n, k, x, m, y, indep, s);
}

cudaError_t launch_simple_matmul(int type, const void *w, int64_t n, int64_t k, const void *x,
                                 int xdt, int64_t m, void *y, int ydt, cudaStream_t s, bool independent) {
    const bool ind = independent;
    switch (type) {
    case KQ_Q8_0: return simple_xy<KQ_Q8_0>(w, n, k, x, xdt, m, y, ydt, ind, s);
    case KQ_Q4_K: return simple_xy<KQ_Q4_K>(w, n, k, x, xdt, m, y, ydt, ind, s);
    case KQ_Q2_K: return simple_xy<KQ_Q2_K>(w, n, k, x, xdt, m, y, ydt, ind, s);
    case KQ_Q5_K: return simple_xy<KQ_Q5_K>(w, n, k, x, xdt, m, y, ydt, ind, s);
    case KQ_Q6_K: return simple_xy<KQ_Q6_K>(w, n, k, x, xdt, m, y, ydt, ind, s);
    case KQ_TQ1_G128: return simple_xy<KQ_TQ1_G128>(w, n, k, x, xdt, m, y, ydt, ind, s);
    default: return cudaErrorInvalidValue;
    }
}

template <int TYPE>
static cudaError_t get_rows_t(const void *w, int64_t rows, int64_t k, const int32_t *ids, int64_t n_ids,
                              void *out, int dt, cudaStream_t s) {
    const int64_t units = n_ids * (k / Geom<TYPE>::QK) * Unit<TYPE>::PER_BLOCK;
    const int g = grid_for(units, 256);
    const uint8_t *wp = static_cast<const uint8_t *>(w);
    unsigned int *err = error_word();
    if (dt == KQ_F32)
        get_rows_kernel<TYPE, float><<<g, 256, 0, s>>>(wp, rows, k, ids, n_ids, static_cast<float *>(out), err);
    else if (dt == KQ_BF16)
        get_rows_kernel<TYPE, __nv_bfloat16><<<g, 256, 0, s>>>(wp, rows, k, ids, n_ids,
                                                               static_cast<__nv_bfloat16 *>(out), err);
    else
        get_rows_kernel<TYPE, __half><<<g, 256, 0, s>>>(wp, rows, k, ids, n_ids, static_cast<__half *>(out), err);
    return cudaGetLastError();
}

cudaError_t launch_get_rows(int type, const void *w, int64_t rows, int64_t k, const int32_t *ids,
                            int64_t n_ids, void *out, int dt, cudaStream_t s) {
    switch (type) {
    case KQ_Q8_0: return get_rows_t<KQ_Q8_0>(w, rows, k, ids, n_ids, out, dt, s);
    case KQ_Q4_K: return get_rows_t<KQ_Q4_K>(w, rows, k, ids, n_ids, out, dt, s);
    case KQ_Q2_K: return get_rows_t<KQ_Q2_K>(w, rows, k, ids, n_ids, out, dt, s);
    case KQ_Q5_K: return get_rows_t<KQ_Q5_K>(w, rows, k, ids, n_ids, out, dt, s);
    case KQ_Q6_K: return get_rows_t<KQ_Q6_K>(w, rows, k, ids, n_ids, out, dt, s);
    case KQ_TQ1_G128: return get_rows_t<KQ_TQ1_G128>(w, rows, k, ids, n_ids, out, dt, s);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_tq1_scan(const void *w, int64_t blocks, unsigned long long *first_bad,
                            cudaStream_t s) {
    tq1_scan_kernel<<<grid_for(blocks, 256), 256, 0, s>>>(static_cast<const uint8_t *>(w), blocks,
                                                          first_bad);
    return cudaGetLastError();
}

}  // namespace kq
