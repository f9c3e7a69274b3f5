// kq_moe.cu -- expert grouping and the plain expert-indexed product.
//
// Grouping (mlx-kquant `expert_tile_map`, mlx-native map0 schedule): the
// (token, slot) pairs are grouped by expert id on the device -- per-expert
// counts, their exclusive prefix sum, and the pair indices of each expert in
// ascending order (a stable sort).  No host synchronisation: ids may come
// from earlier GPU work.  Invalid ids (outside [0, E)) write a NaN output
// row and set the sticky device error word (mlx-native
// `quantized_matmul_id_ggml`: invalid routing metadata reads no expert
// weights and writes a non-finite poison sentinel).
#include "kq_decode.cuh"
#include "kq_ptx.cuh"
#include "kq_launch.h"

namespace kq {

constexpr int GROUP_THREADS = 1024;

// One CTA.  Warp w owns experts w, w + 32, ...; it scans the ids in order,
// so each expert's pair list comes out ascending.  With bn > 0 it also
// writes the tensor-core kernels' token tiles: each expert's segment in
// tiles of at most bn pairs, (expert, first position in perm) each, and
// their number.  Launched as a programmatic dependent of the preceding
// kernel: nothing is read or written before that kernel has completed.
__global__ void __launch_bounds__(GROUP_THREADS) moe_group_kernel(
    const int32_t *__restrict__ ids, int n_pairs, int n_experts, int32_t *__restrict__ counts,
    int32_t *__restrict__ offsets, int32_t *__restrict__ perm, void *y, int y_dtype, int64_t n,
    int bn, int2 *__restrict__ tiles, int32_t *__restrict__ n_tiles, int max_tiles, unsigned int *err) {
    extern __shared__ int s_off[];  // n_experts + 1, then (bn > 0) the first tile of each expert
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    __shared__ int s_bad;
    griddep_wait();
    if (threadIdx.x == 0) s_bad = 0;
    __syncthreads();
    // validation (+ poison rows)
    for (int p = threadIdx.x; p < n_pairs; p += blockDim.x) {
        const int e = ids[p];
        if (e < 0 || e >= n_experts) {
            s_bad = 1;
            if (y != nullptr) {
                if (y_dtype == KQ_F32) {
                    float *yr = static_cast<float *>(y) + (int64_t)p * n;
                    for (int64_t j = 0; j < n; ++j) yr[j] = __int_as_float(0x7fc00000);
                } else {
                    __nv_bfloat16 *yr = static_cast<__nv_bfloat16 *>(y) + (int64_t)p * n;
                    for (int64_t j = 0; j < n; ++j) yr[j] = __ushort_as_bfloat16((unsigned short)0x7fc0);
                }
            }
        }
    }
    // pass 1: counts
    for (int e = warp; e < n_experts; e += nwarps) {
        int cnt = 0;
        for (int base = 0; base < n_pairs; base += 32) {
            const int p = base + lane;
            const bool hit = p < n_pairs && ids[p] == e;
            cnt += __popc(__ballot_sync(0xffffffffu, hit));
        }
        if (lane == 0) s_off[e] = cnt;
    }
    __syncthreads();
    // exclusive scan by warp 0, 32 experts at a time
    if (warp == 0) {
        int carry = 0;
        for (int base = 0; base < n_experts; base += 32) {
            const int e = base + lane;
            const int c = e < n_experts ? s_off[e] : 0;
            int incl = c;
            #pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += t;
            }
            if (e < n_experts) {
                counts[e] = c;
                s_off[e] = carry + incl - c;
            }
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) s_off[n_experts] = carry;
    }
    __syncthreads();
    for (int e = threadIdx.x; e <= n_experts; e += blockDim.x) offsets[e] = s_off[e];
    // pass 2: stable scatter
    const unsigned lt = (1u << lane) - 1u;
    for (int e = warp; e < n_experts; e += nwarps) {
        int pos = s_off[e];
        for (int base = 0; base < n_pairs; base += 32) {
            const int p = base + lane;
            const bool hit = p < n_pairs && ids[p] == e;
            const unsigned mask = __ballot_sync(0xffffffffu, hit);
            if (hit && KQ_DCHECK(pos + __popc(mask & lt) < n_pairs, err)) perm[pos + __popc(mask & lt)] = p;
            pos += __popc(mask);
        }
    }
    for (int p = s_off[n_experts] + threadIdx.x; p < n_pairs; p += blockDim.x) perm[p] = -1;
    if (threadIdx.x == 0 && s_bad) atomicOr(err, ERR_BAD_ID);
    if (bn > 0) {
        int *s_first = s_off + n_experts + 1;
        if (warp == 0) {
            int carry = 0;
            for (int base = 0; base < n_experts; base += 32) {
                const int e = base + lane;
                const int c = e < n_experts ? (s_off[e + 1] - s_off[e] + bn - 1) / bn : 0;
                int incl = c;
                #pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int t = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += t;
                }
                if (e < n_experts) s_first[e] = carry + incl - c;
                carry += __shfl_sync(0xffffffffu, incl, 31);
            }
            if (lane == 0) *n_tiles = KQ_DCHECK(carry <= max_tiles, err) ? carry : max_tiles;
        }
        __syncthreads();
        for (int e = threadIdx.x; e < n_experts; e += blockDim.x) {
            const int p0 = s_off[e], p1 = s_off[e + 1];
            int i = s_first[e];
            for (int q = p0; q < p1; q += bn, ++i)
                if (KQ_DCHECK(i < max_tiles, err)) tiles[i] = make_int2(e, q);
        }
    }
    griddep_launch_dependents();
}

cudaError_t launch_moe_group(const int32_t *ids, int64_t n_pairs, int64_t n_experts,
                             int32_t *counts, int32_t *offsets, int32_t *perm, void *y,
                             int y_dtype, int64_t n, cudaStream_t s, int bn, int32_t *tiles,
                             int32_t *n_tiles, int64_t max_tiles) {
    const size_t smem = sizeof(int) * (size_t)(n_experts + 1) * (bn > 0 ? 2 : 1);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(moe_group_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1);
    cfg.blockDim = dim3(GROUP_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, moe_group_kernel, ids, (int)n_pairs, (int)n_experts, counts, offsets, perm,
                              y, y_dtype, n, bn, reinterpret_cast<int2 *>(tiles), n_tiles, (int)max_tiles,
                              error_word());
}

// Token tiles for the tensor-core expert product: expert e's segment
// [offsets[e], offsets[e+1]) of the grouped pair list splits into
// ceil(count / bn) tiles.  One CTA; warp 0 scans the per-expert tile counts
// 32 experts at a time, then every thread writes the tiles of its experts.
constexpr int TILE_THREADS = 256;

__global__ void __launch_bounds__(TILE_THREADS) moe_tiles_kernel(const int32_t *__restrict__ offsets,
                                                                 int n_experts, int bn,
                                                                 int2 *__restrict__ tiles,
                                                                 int32_t *__restrict__ n_tiles,
                                                                 int max_tiles, unsigned int *err) {
    extern __shared__ int s_first[];  // n_experts: first tile index of each expert
    const int lane = threadIdx.x & 31;
    if (threadIdx.x < 32) {
        int carry = 0;
        for (int base = 0; base < n_experts; base += 32) {
            const int e = base + lane;
            const int c = e < n_experts ? (offsets[e + 1] - offsets[e] + bn - 1) / bn : 0;
            int incl = c;
            #pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += t;
            }
            if (e < n_experts) s_first[e] = carry + incl - c;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) *n_tiles = KQ_DCHECK(carry <= max_tiles, err) ? carry : max_tiles;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < n_experts; e += blockDim.x) {
        const int p0 = offsets[e], p1 = offsets[e + 1];
        int i = s_first[e];
        for (int q = p0; q < p1; q += bn, ++i)
            if (KQ_DCHECK(i < max_tiles, err)) tiles[i] = make_int2(e, q);
    }
}

cudaError_t launch_moe_tiles(const int32_t *offsets, int64_t n_experts, int bn, int32_t *tiles,
                             int32_t *n_tiles, int64_t max_tiles, cudaStream_t s) {
    const size_t smem = sizeof(int) * (size_t)n_experts;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(moe_tiles_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
    }
    moe_tiles_kernel<<<1, TILE_THREADS, smem, s>>>(offsets, (int)n_experts, bn,
                                                   reinterpret_cast<int2 *>(tiles), n_tiles,
                                                   (int)max_tiles, error_word());
    return cudaGetLastError();
}

// ---------------------------------------------------------------- plain grouped product
// Grid (ceil(n / 8), n_experts): warp = one weight row of expert e; it walks
// the pairs routed to e four at a time.
template <int TYPE, typename XT, typename YT>
__global__ void __launch_bounds__(256) simple_id_kernel(
    const uint8_t *__restrict__ w, int64_t n, int64_t k, int64_t expert_stride,
    const XT *__restrict__ x, int top_k, const int32_t *__restrict__ counts,
    const int32_t *__restrict__ offsets, const int32_t *__restrict__ perm, YT *__restrict__ y, int n_pairs,
    unsigned int *err) {
    using G = Geom<TYPE>;
    using U = Unit<TYPE>;
    constexpr int TB = 4;
    const int e = blockIdx.y;
    const int cnt = counts[e];
    if (cnt == 0) return;
    const int lane = threadIdx.x & 31;
    const int64_t row = blockIdx.x * 8LL + (threadIdx.x >> 5);
    if (row >= n) return;
    const int64_t nb = k / G::QK;
    const uint8_t *wr = w + e * expert_stride + row * nb * G::BB;
    if (!KQ_DCHECK(offsets[e] >= 0 && offsets[e] + cnt <= n_pairs, err)) return;
    const int32_t *plist = perm + offsets[e];
    const int64_t units = nb * U::PER_BLOCK;
    for (int c0 = 0; c0 < cnt; c0 += TB) {
        int pr[TB];
        #pragma unroll
        for (int t = 0; t < TB; ++t) {
            pr[t] = (c0 + t < cnt) ? plist[c0 + t] : -1;
            if (pr[t] >= 0 && !KQ_DCHECK(pr[t] < n_pairs, err)) pr[t] = -1;
        }
        float acc[TB] = {0.f, 0.f, 0.f, 0.f};
        for (int64_t i = lane; i < units; i += 32) {
            const int64_t bi = i / U::PER_BLOCK;
            const int u = (int)(i % U::PER_BLOCK);
            float wv[8];
            U::decode(wr + bi * G::BB, u, wv);
            const int64_t col = bi * G::QK + 8 * u;
            #pragma unroll
            for (int t = 0; t < TB; ++t) {
                if (pr[t] >= 0) {
                    float xv[8];
                    load_x8(x + (int64_t)(pr[t] / top_k) * k + col, xv);
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
            if (lane == 0 && pr[t] >= 0) store_out(y + (int64_t)pr[t] * n + row, v);
        }
    }
}

// Plain fused GLU: the same walk with a gate and an up row per warp;
// y = act(gate) * up (mlx-kquant `moe_glu_gather_kq`).
template <int TYPE, typename XT, typename YT>
__global__ void __launch_bounds__(256) simple_glu_kernel(
    const uint8_t *__restrict__ wg, const uint8_t *__restrict__ wu, int64_t n, int64_t k,
    int64_t expert_stride, const XT *__restrict__ x, int top_k, const int32_t *__restrict__ counts,
    const int32_t *__restrict__ offsets, const int32_t *__restrict__ perm, YT *__restrict__ y, int act,
    int n_pairs, unsigned int *err) {
    using G = Geom<TYPE>;
    using U = Unit<TYPE>;
    constexpr int TB = 4;
    const int e = blockIdx.y;
    const int cnt = counts[e];
    if (cnt == 0) return;
    const int lane = threadIdx.x & 31;
    const int64_t row = blockIdx.x * 8LL + (threadIdx.x >> 5);
    if (row >= n) return;
    const int64_t nb = k / G::QK;
    const int64_t off = e * expert_stride + row * nb * G::BB;
    if (!KQ_DCHECK(offsets[e] >= 0 && offsets[e] + cnt <= n_pairs, err)) return;
    const int32_t *plist = perm + offsets[e];
    const int64_t units = nb * U::PER_BLOCK;
    for (int c0 = 0; c0 < cnt; c0 += TB) {
        int pr[TB];
        #pragma unroll
        for (int t = 0; t < TB; ++t) {
            pr[t] = (c0 + t < cnt) ? plist[c0 + t] : -1;
            if (pr[t] >= 0 && !KQ_DCHECK(pr[t] < n_pairs, err)) pr[t] = -1;
        }
        float ag[TB] = {0.f, 0.f, 0.f, 0.f}, au[TB] = {0.f, 0.f, 0.f, 0.f};
        for (int64_t i = lane; i < units; i += 32) {
            const int64_t bi = i / U::PER_BLOCK;
            const int u = (int)(i % U::PER_BLOCK);
            float vg[8], vu[8];
            U::decode(wg + off + bi * G::BB, u, vg);
            U::decode(wu + off + bi * G::BB, u, vu);
            const int64_t col = bi * G::QK + 8 * u;
            #pragma unroll
            for (int t = 0; t < TB; ++t) {
                if (pr[t] >= 0) {
                    float xv[8];
                    load_x8(x + (int64_t)(pr[t] / top_k) * k + col, xv);
                    #pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        ag[t] = fmaf(vg[j], xv[j], ag[t]);
                        au[t] = fmaf(vu[j], xv[j], au[t]);
                    }
                }
            }
        }
        #pragma unroll
        for (int t = 0; t < TB; ++t) {
            float g = ag[t], uu = au[t];
            #pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                g += __shfl_xor_sync(0xffffffffu, g, o);
                uu += __shfl_xor_sync(0xffffffffu, uu, o);
            }
            if (lane == 0 && pr[t] >= 0) store_out(y + (int64_t)pr[t] * n + row, glu_activation(g, act) * uu);
        }
    }
}

// ---------------------------------------------------------------- routing mix
// mlx-kquant `gather_qmv_mix_kq`: the slots' products are summed in fp32,
// each weighted by its routing score.  Grid (column chunks, tokens); a
// thread owns VW adjacent columns of one token and reads the token's top_k
// pair rows in slot order, so the sum is the same on every run.
constexpr int MIX_THREADS = 256;

template <int VW, typename YT>
__global__ void __launch_bounds__(MIX_THREADS) moe_mix_kernel(
    const float *__restrict__ pair_out, const int32_t *__restrict__ ids,
    const float *__restrict__ scores, int n_tokens, int top_k, int n_experts, int64_t n,
    YT *__restrict__ y) {
    const int64_t j0 = ((int64_t)blockIdx.x * MIX_THREADS + threadIdx.x) * VW;
    if (j0 >= n) return;
    for (int t = blockIdx.y; t < n_tokens; t += gridDim.y) {
        float acc[VW];
        #pragma unroll
        for (int v = 0; v < VW; ++v) acc[v] = 0.f;
        bool bad = false;
        for (int sl = 0; sl < top_k; ++sl) {
            const int64_t pr = (int64_t)t * top_k + sl;
            const int e = ids[pr];
            bad |= e < 0 || e >= n_experts;
            const float sc = scores[pr];
            const float *row = pair_out + pr * n + j0;
            float q[VW];
            if constexpr (VW == 4) {
                const float4 f = *reinterpret_cast<const float4 *>(row);
                q[0] = f.x; q[1] = f.y; q[2] = f.z; q[3] = f.w;
            } else {
                q[0] = row[0];
            }
            #pragma unroll
            for (int v = 0; v < VW; ++v) acc[v] = fmaf(sc, q[v], acc[v]);
        }
        YT *yr = y + (int64_t)t * n + j0;
        #pragma unroll
        for (int v = 0; v < VW; ++v) store_out(yr + v, bad ? __int_as_float(0x7fc00000) : acc[v]);
    }
}

template <typename YT>
static cudaError_t moe_mix_t(const float *pair_out, const int32_t *ids, const float *scores,
                             int64_t n_tokens, int64_t top_k, int64_t n_experts, int64_t n, YT *y,
                             cudaStream_t s) {
    const int vw = n % 4 == 0 ? 4 : 1;
    const int64_t chunks = (n / vw + MIX_THREADS - 1) / MIX_THREADS;
    if (chunks > INT32_MAX) return cudaErrorInvalidValue;
    dim3 grid((unsigned)chunks, (unsigned)(n_tokens < 65535 ? n_tokens : 65535));
    if (vw == 4)
        moe_mix_kernel<4, YT><<<grid, MIX_THREADS, 0, s>>>(pair_out, ids, scores, (int)n_tokens,
                                                          (int)top_k, (int)n_experts, n, y);
    else
        moe_mix_kernel<1, YT><<<grid, MIX_THREADS, 0, s>>>(pair_out, ids, scores, (int)n_tokens,
                                                          (int)top_k, (int)n_experts, n, y);
    return cudaGetLastError();
}

cudaError_t launch_moe_mix(const float *pair_out, const int32_t *ids, const float *scores,
                           int64_t n_tokens, int64_t top_k, int64_t n_experts, int64_t n, void *y,
                           int y_dtype, cudaStream_t s) {
    if (y_dtype == KQ_F32)
        return moe_mix_t(pair_out, ids, scores, n_tokens, top_k, n_experts, n, static_cast<float *>(y), s);
    if (y_dtype == KQ_BF16)
        return moe_mix_t(pair_out, ids, scores, n_tokens, top_k, n_experts, n,
                         static_cast<__nv_bfloat16 *>(y), s);
    return cudaErrorInvalidValue;
}

template <int TYPE, typename XT, typename YT>
static cudaError_t simple_glu_t(const IdArgs &a, cudaStream_t s) {
    dim3 grid((unsigned)((a.n + 7) / 8), (unsigned)a.n_experts);
    simple_glu_kernel<TYPE, XT, YT><<<grid, 256, 0, s>>>(
        static_cast<const uint8_t *>(a.w), static_cast<const uint8_t *>(a.w2), a.n, a.k, a.expert_stride,
        static_cast<const XT *>(a.x), a.x_div(), a.counts, a.offsets, a.perm, static_cast<YT *>(a.y), a.act,
        (int)(a.n_tokens * a.top_k), error_word());
    return cudaGetLastError();
}

template <int TYPE>
static cudaError_t simple_glu_xy(const IdArgs &a, cudaStream_t s) {
    if (a.x_dtype == KQ_F32) {
        if (a.y_dtype == KQ_F32) return simple_glu_t<TYPE, float, float>(a, s);
        return simple_glu_t<TYPE, float, __nv_bfloat16>(a, s);
    }
    if (a.y_dtype == KQ_F32) return simple_glu_t<TYPE, __nv_bfloat16, float>(a, s);
    return simple_glu_t<TYPE, __nv_bfloat16, __nv_bfloat16>(a, s);
}

cudaError_t launch_simple_glu(const IdArgs &a, cudaStream_t s) {
    switch (a.type) {
    case KQ_Q8_0: return simple_glu_xy<KQ_Q8_0>(a, s);
    case KQ_Q4_K: return simple_glu_xy<KQ_Q4_K>(a, s);
    case KQ_Q2_K: return simple_glu_xy<KQ_Q2_K>(a, s);
    case KQ_Q5_K: return simple_glu_xy<KQ_Q5_K>(a, s);
    case KQ_Q6_K: return simple_glu_xy<KQ_Q6_K>(a, s);
    case KQ_TQ1_G128: return simple_glu_xy<KQ_TQ1_G128>(a, s);
    default: return cudaErrorInvalidValue;
    }
}

template <int TYPE, typename XT, typename YT>
static cudaError_t simple_id_t(const IdArgs &a, cudaStream_t s) {
    dim3 grid((unsigned)((a.n + 7) / 8), (unsigned)a.n_experts);
    simple_id_kernel<TYPE, XT, YT><<<grid, 256, 0, s>>>(
        static_cast<const uint8_t *>(a.w), a.n, a.k, a.expert_stride,
        static_cast<const XT *>(a.x), a.x_div(), a.counts, a.offsets, a.perm,
        static_cast<YT *>(a.y), (int)(a.n_tokens * a.top_k), error_word());
    return cudaGetLastError();
}

template <int TYPE>
static cudaError_t simple_id_xy(const IdArgs &a, cudaStream_t s) {
    if (a.x_dtype == KQ_F32) {
        if (a.y_dtype == KQ_F32) return simple_id_t<TYPE, float, float>(a, s);
        return simple_id_t<TYPE, float, __nv_bfloat16>(a, s);
    }
    if (a.y_dtype == KQ_F32) return simple_id_t<TYPE, __nv_bfloat16, float>(a, s);
    return simple_id_t<TYPE, __nv_bfloat16, __nv_bfloat16>(a, s);
}

cudaError_t launch_simple_id(const IdArgs &a, cudaStream_t s) {
    switch (a.type) {
    case KQ_Q8_0: return simple_id_xy<KQ_Q8_0>(a, s);
    case KQ_Q4_K: return simple_id_xy<KQ_Q4_K>(a, s);
    case KQ_Q2_K: return simple_id_xy<KQ_Q2_K>(a, s);
    case KQ_Q5_K: return simple_id_xy<KQ_Q5_K>(a, s);
    case KQ_Q6_K: return simple_id_xy<KQ_Q6_K>(a, s);
    case KQ_TQ1_G128: return simple_id_xy<KQ_TQ1_G128>(a, s);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace kq
