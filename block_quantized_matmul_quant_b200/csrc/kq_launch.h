// kq_launch.h -- internal launcher declarations (host side).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace kq {

struct IdArgs {
    int type;
    const void *w;
    int64_t n_experts, n, k, expert_stride;
    const void *x;
    int x_dtype;
    int64_t n_tokens, top_k;
    void *y;
    int y_dtype;
    const int32_t *counts, *offsets, *perm;  // grouping (device)
    const int32_t *tiles;                    // tensor-core tile list (device)
    const int32_t *n_tiles;                  // its length (device)
    const void *w2 = nullptr;                // fused GLU: up stack (w: gate stack)
    int act = 0;                             // fused GLU activation (KQ_ACT_*)
    bool x_slotted = false;                  // x holds one row per pair [n_tokens * top_k, k]
    bool tc_i8 = false;                      // few-pairs kernel: the int8 form
    // Pair index p = t * top_k + s reads x row p / x_div().
    int x_div() const { return x_slotted ? 1 : (int)top_k; }
    int64_t x_rows() const { return x_slotted ? n_tokens * top_k : n_tokens; }
};

cudaError_t launch_dequant(int type, const void *w, int64_t rows, int64_t k, void *out, int dt,
                           cudaStream_t s);
// The plain product; `independent`: the call may overlap the preceding
// kernel (KQ_FLAG_INDEPENDENT), else it runs after it.
cudaError_t launch_simple_matmul(int type, const void *w, int64_t n, int64_t k, const void *x,
                                 int xdt, int64_t m, void *y, int ydt, cudaStream_t s, bool independent = false);
cudaError_t launch_tq1_scan(const void *w, int64_t blocks, unsigned long long *first_bad,
                            cudaStream_t s);
cudaError_t launch_get_rows(int type, const void *w, int64_t rows, int64_t k, const int32_t *ids,
                            int64_t n_ids, void *out, int dt, cudaStream_t s);
// Grouping of the (token, slot) pairs by expert; with bn > 0 also the token
// tiles of at most bn pairs (as launch_moe_tiles).  Programmatic dependent
// launch: it waits for the preceding kernel before touching memory.
cudaError_t launch_moe_group(const int32_t *ids, int64_t n_pairs, int64_t n_experts,
                             int32_t *counts, int32_t *offsets, int32_t *perm, void *y,
                             int y_dtype, int64_t n, cudaStream_t s, int bn = 0, int32_t *tiles = nullptr,
                             int32_t *n_tiles = nullptr, int64_t max_tiles = 0);
cudaError_t launch_simple_id(const IdArgs &a, cudaStream_t s);
// Plain fused GLU over the grouping (any codec): y = act(x W_gate^T) * (x W_up^T).
cudaError_t launch_simple_glu(const IdArgs &a, cudaStream_t s);
// Routing mix: y[t] = sum over s of scores[t][s] * pair_out[t * top_k + s]
// (fp32 rows of n), slots in order; a token with an id outside [0, E) gets a
// NaN row.
cudaError_t launch_moe_mix(const float *pair_out, const int32_t *ids, const float *scores,
                           int64_t n_tokens, int64_t top_k, int64_t n_experts, int64_t n, void *y,
                           int y_dtype, cudaStream_t s);
// Token tiles of at most bn pairs per expert segment, (expert, first
// position in perm) each, and their number -- from the grouping's offsets;
// the tile list holds max_tiles entries.
cudaError_t launch_moe_tiles(const int32_t *offsets, int64_t n_experts, int bn, int32_t *tiles,
                             int32_t *n_tiles, int64_t max_tiles, cudaStream_t s);

// Bandwidth kernels (kq_gemv.cu).  Return cudaErrorNotSupported when the
// shape is outside what the kernel serves.
bool gemv_supported(int type, int64_t n, int64_t k, int x_dtype, int64_t m);
// How a bandwidth-kernel call is ordered against earlier work on its stream:
//   kStream        read everything after the preceding kernel completes;
//   kConstWeights  weights are never written by earlier work: stream them
//                  before the preceding kernel completes (PDL), x after;
//   kIndependent   nothing earlier touches w, x or y: never wait, and use a
//                  half-SM CTA so consecutive calls run side by side.
enum class GemvOrder { kStream, kConstWeights, kIndependent };
cudaError_t launch_gemv(int type, const void *w, int64_t n, int64_t k, const void *x, int xdt,
                        int64_t m, void *y, int ydt, GemvOrder order, cudaStream_t s);
// TQ1_G128 bandwidth kernel (kq_gemv_tq1.cu); launch_gemv routes to it.
bool gemv_tq1_supported(int64_t n, int64_t k);
cudaError_t launch_gemv_tq1(const void *w, int64_t n, int64_t k, const void *x, int xdt, int64_t m,
                            void *y, int ydt, GemvOrder order, cudaStream_t s);
// Expert-indexed bandwidth kernel (kq_moe_gemv.cu): Q4_K, few pairs per
// expert; runs after launch_moe_group on the same stream.
bool moe_gemv_supported(int type, int64_t n, int64_t k, int64_t n_experts);
cudaError_t launch_moe_gemv(const IdArgs &a, cudaStream_t s);

// Tensor-core kernels (kq_gemm_sm100.cu): Q4_K dense and expert-indexed,
// Q8_0 and Q5_K dense (K % 256 == 0), Q2_K dense (K % 1024 == 0), TQ1_G128
// dense (K % 512 == 0).
bool gemm_supported(int type, int64_t n, int64_t k, int x_dtype, int y_dtype, bool expert_indexed = false);
cudaError_t launch_gemm(int type, const void *w, int64_t n, int64_t k, const void *x, int64_t m,
                        void *y, int ydt, cudaStream_t s);
// Expert-indexed form over the grouping's token tiles (a.tiles / a.n_tiles,
// written by launch_moe_tiles with the same bn).
int gemm_id_bn(int64_t n_tokens, int64_t top_k, int64_t n_experts);
// glu_combine: the GLU's second pass, y = act(this product) * y (a.act).
cudaError_t launch_gemm_id(const IdArgs &a, int bn, cudaStream_t s, bool glu_combine = false);
// Expert-indexed tensor-core kernel for few pairs per expert
// (kq_moe_mma.cu), over token tiles of moe_mma_bn(x_dtype) pairs.
bool moe_mma_supported(int type, int64_t n, int64_t k, int x_dtype, int y_dtype);
int moe_mma_bn(int x_dtype, bool i8);
cudaError_t launch_moe_mma(const IdArgs &a, cudaStream_t s);   // a.w2 set: fused GLU
// The same kernel on one matrix and m activation rows (tiles of
// moe_mma_bn(x_dtype) rows).
cudaError_t launch_gemv_tc(const void *w, int64_t n, int64_t k, const void *x, int x_dtype, int64_t m, void *y,
                           int y_dtype, bool i8, cudaStream_t s);

}  // namespace kq
