/*
 * kq.h -- C ABI of libkq: matrix products against block-quantized
 *         (GGUF-style) weights on NVIDIA B200 (sm_100a).
 *
 * The library decodes the weight blocks on the fly inside its CUDA kernels.
 * Codecs: Q8_0, Q2_K, Q4_K, Q5_K, Q6_K (GGML block formats) and TQ1_G128
 * (28-byte, 128-weight ternary blocks).
 *
 * Conventions shared by every call
 * --------------------------------
 *  * Pointers named `w`, `x`, `y`, `out`, `ids`, `workspace` are DEVICE
 *    pointers (memory of the current CUDA device, allocated by the caller).
 *    Pointers named `first_bad_block` are HOST pointers.  The caller owns all
 *    memory; no call allocates device memory.
 *  * `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls
 *    enqueue work on it and return without synchronizing, except where a
 *    call says it synchronizes.
 *  * Weights are row-major: row n of a [N, K] weight is (K / QK) consecutive
 *    wire blocks, kq_row_bytes(type, K) bytes, rows packed back to back
 *    (the mlx-kquant `quantized_matmul` layout, w laid out [N, K] with the
 *    byte-packed last dimension).  Activations x are row-major [M, K],
 *    outputs y row-major [M, N]; all contiguous.
 *  * Alignment: w, x, y, out, ids and workspace must be 16-byte aligned.
 *  * Return value: KQ_OK (0) or a negative KQ_ERR_* code.  Every argument is
 *    validated on the host before anything is enqueued, so an argument error
 *    means no work was launched (no partial output).  KQ_ERR_CUDA (a failed
 *    launch) from a call made of several kernels (kq_matmul_id: grouping,
 *    then the product; the bandwidth kernel: one launch per eight activation
 *    rows) may follow the launch of its earlier kernels; the output is then
 *    unspecified.
 *  * Floating-point dtypes: KQ_F32, KQ_BF16 (and KQ_F16 for kq_dequantize's
 *    output).  Accumulation is always fp32.
 */
#ifndef KQ_H
#define KQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KQ_API __attribute__((visibility("default")))
#else
#define KQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---- codecs (GGML type numbers where GGML has one) ---- */
#define KQ_Q8_0     8     /* 34 B / 32 w:  fp16 d, int8 q[32]; w = d*q            */
#define KQ_Q2_K     10    /* 84 B / 256 w: scales[16], qs[64], fp16 d, fp16 dmin   */
#define KQ_Q4_K     12    /* 144 B / 256 w: fp16 d, fp16 dmin, scales[12], qs[128] */
#define KQ_Q5_K     13    /* 176 B / 256 w: fp16 d, fp16 dmin, scales[12], qh[32], qs[128] */
#define KQ_Q6_K     14    /* 210 B / 256 w: ql[128], qh[64], int8 scales[16], fp16 d */
#define KQ_TQ1_G128 1001  /* 28 B / 128 w: 25 full trit bytes, tail byte, fp16 scale */

/* ---- dtypes ---- */
#define KQ_F32  0
#define KQ_BF16 1
#define KQ_F16  2

/* ---- status codes ---- */
#define KQ_OK                   0
#define KQ_ERR_ARG             -1   /* null pointer, zero/negative dim, top_k not in 1..E */
#define KQ_ERR_TYPE            -2   /* unknown codec                                  */
#define KQ_ERR_SHAPE           -3   /* K not a multiple of the block size, bad stride  */
#define KQ_ERR_DTYPE           -4   /* unsupported dtype for this argument             */
#define KQ_ERR_ALIGN           -5   /* pointer not 16-byte aligned                     */
#define KQ_ERR_OVERFLOW        -6   /* a byte or element count overflows int64 / int32 */
#define KQ_ERR_WORKSPACE       -7   /* workspace null or smaller than required         */
#define KQ_ERR_CUDA            -8   /* a CUDA runtime call failed                      */
#define KQ_ERR_DEVICE          -9   /* device-side error word was set (bad expert/row id) */
#define KQ_ERR_DEVICE_TIMEOUT  -10  /* a bounded device-side wait gave up              */
#define KQ_ERR_UNSUPPORTED     -11  /* current device is not sm_100 / path unavailable */
#define KQ_ERR_DEVICE_BOUNDS   -12  /* a KQ_DEBUG build's device bounds check failed  */

/* ---- matmul paths (kq_matmul_ex / kq_matmul_id_ex) ---- */
#define KQ_PATH_AUTO     0  /* dispatch by shape (the default of kq_matmul)          */
#define KQ_PATH_SIMPLE   1  /* plain CUDA-core kernel, any codec/shape               */
#define KQ_PATH_GEMV     2  /* bandwidth kernel: weights decoded in registers         */
/* TMA + tcgen05 tensor-core kernel: bf16 x only; Q4_K (K % 256 == 0), or,
 * dense only, Q8_0 and Q5_K with K % 256 == 0, Q2_K with K % 1024 == 0 and
 * TQ1_G128 with K % 512 == 0 (Ternary Bonsai `tq1_gemm`). */
#define KQ_PATH_GEMM     3
/* Tensor-core kernel for few activation rows / pairs per expert: 4-bit codes
 * through the MMA, one accumulator per 32-weight sub-block, the scales
 * applied after it (Q4_K, K <= 4096; tiles of 16 bf16 activation rows, or 8
 * fp32 rows each split into a bf16 high and low part). */
#define KQ_PATH_GEMV_TC  4
/* Flag OR-ed into `path`: the caller guarantees that no work enqueued earlier
 * on the stream writes the weight bytes (they are constant, as model weights
 * are).  The kernel may then start streaming weights before the preceding
 * kernel has finished (programmatic dependent launch); x is still read only
 * after the preceding work completes. */
#define KQ_FLAG_CONST_WEIGHTS 0x100
/* Flag OR-ed into `path`: the call is independent of everything enqueued
 * before it on the stream -- no earlier work writes w or x, or reads or
 * writes y (e.g. separate projections of one activation, or a batch of
 * weight matrices).  The kernel then never waits for the preceding kernel:
 * consecutive independent calls stream their weights concurrently.  Implies
 * KQ_FLAG_CONST_WEIGHTS.  Honoured by the bandwidth kernels and the plain
 * kernel (KQ_PATH_SIMPLE); the tensor-core paths keep stream order. */
#define KQ_FLAG_INDEPENDENT 0x200

/* Weights per block and bytes per block of a codec; 0 for an unknown codec. */
KQ_API int kq_block_weights(int type);
KQ_API int kq_block_bytes(int type);
/* Bytes of one weight row of length k; -1 if k is not a multiple of the
 * block size or the codec is unknown. */
KQ_API int64_t kq_row_bytes(int type, int64_t k);

/*
 * kq_dequantize -- decode weights to floats.
 * Defines: mlx-kquant bindings.cpp `dequantize(w, scales, kquant_type, dtype)`
 * (wire bytes -> float array; the K-quant scales live inside w).
 *   w       [rows, kq_row_bytes(type, k)] u8 wire blocks (device)
 *   out     [rows, k] of out_dtype (KQ_F32, KQ_BF16 or KQ_F16) (device)
 * The fp32 result is bit-exact: each weight is the codec definition's IEEE
 * fp32 operation sequence (products exact, one rounding at the final
 * subtraction).  bf16/f16 outputs are that fp32 value rounded to nearest even.
 * TQ1_G128 bytes above the legal maximum (242 full, 26 tail) decode to zero.
 */
KQ_API int kq_dequantize(int type, const void *w, int64_t rows, int64_t k,
                  void *out, int out_dtype, void *stream);

/*
 * kq_matmul -- y = x @ dequant(w)^T.
 * Defines: mlx-kquant bindings.cpp `quantized_matmul(x, w, scales,
 * kquant_type, transpose=True)`: `x @ dequant(w)` with w laid out [N, K].
 *   w  [n, kq_row_bytes(type, k)] u8 (device)
 *   x  [m, k] of x_dtype (KQ_F32 or KQ_BF16) (device)
 *   y  [m, n] of y_dtype (KQ_F32 or KQ_BF16) (device), fully overwritten
 *   y[i][j] = sum_k dequant(w)[j][k] * x[i][k], fp32 accumulation.
 * Small m runs the bandwidth-bound kernel that decodes weights in
 * registers; large m with bf16 x (Q4_K and Q5_K from 5 rows, Q8_0 with
 * K % 256 == 0 from 3 rows, Q2_K with K % 1024 == 0 from 2 rows, TQ1_G128
 * with K % 512 == 0 from 8 rows) runs the tensor-core kernel, which rounds
 * decoded weights to bf16 before the bf16 x bf16 -> fp32 MMA (for TQ1:
 * (t - 1) times the bf16 rounding of the block scale, the same value).
 */
KQ_API int kq_matmul(int type, const void *w, int64_t n, int64_t k,
              const void *x, int x_dtype, int64_t m,
              void *y, int y_dtype, void *stream);

/* kq_matmul with an explicit path (KQ_PATH_*); KQ_ERR_UNSUPPORTED if the
 * path cannot serve these arguments (e.g. KQ_PATH_GEMM with fp32 x). */
KQ_API int kq_matmul_ex(int type, const void *w, int64_t n, int64_t k,
                 const void *x, int x_dtype, int64_t m,
                 void *y, int y_dtype, int path, void *stream);

/*
 * kq_matmul_id -- expert-indexed (mixture-of-experts) product.
 * Defines: mlx-native 0.21.0 quantized_matmul_id_ggml.rs (module doc and
 * `quantized_matmul_id_ggml`): for every token t and slot s,
 *   e = ids[t][s];  y[t][s][j] = sum_k dequant(w_e)[j][k] * x[t][k].
 * Same operation as mlx-kquant `gather_qmm` with rhs_indices = ids.
 *   w    expert stack; expert e's [n, kq_row_bytes(type, k)] rows start at
 *        w + e * expert_stride bytes (expert_stride >= n * row bytes, a
 *        multiple of 16 for Q4_K and Q5_K, of 4 for Q2_K, of 2 for the
 *        others) (device)
 *   x    [n_tokens, k] of x_dtype (KQ_F32 or KQ_BF16) (device)
 *   ids  [n_tokens, top_k] int32 (device; may be produced by earlier work
 *        on the same stream -- the host never reads it)
 *   y    [n_tokens, top_k, n] of y_dtype (KQ_F32 or KQ_BF16) (device)
 *   workspace  device scratch of at least
 *        kq_matmul_id_workspace_bytes(n_tokens, top_k, n_experts) bytes,
 *        owned by the caller; its contents are overwritten.  Calls that
 *        share one workspace must be ordered on the GPU (one stream).
 * Duplicate ids within a token are legal.  An id outside [0, n_experts)
 * reads no weights, writes NaN to its whole output row and sets the
 * device error word (see kq_device_status); the other rows are exact.
 * Tokens routed to one expert are grouped before the decode, so each hit
 * expert's weights are streamed once per group of tokens; the result of a
 * (t, s) row does not depend on the other tokens' ids.
 * Paths: Q4_K with bf16 x runs the few-pairs tensor-core kernel or, past
 * 32 routed pairs per expert, the grouped tensor-core GEMM (weights rounded
 * to bf16, like kq_matmul's GEMM); Q4_K with fp32 x the grouped mat-vec up
 * to one pair per expert (exact fp32 weights), else the few-pairs kernel;
 * Q8_0 and Q5_K (K % 256 == 0) and Q2_K (K % 1024 == 0) with bf16 x the
 * grouped tensor-core GEMM (expert_stride a multiple of 16 bytes); other
 * codecs and shapes the plain grouped kernel.
 */
KQ_API size_t kq_matmul_id_workspace_bytes(int64_t n_tokens, int64_t top_k, int64_t n_experts);
KQ_API int kq_matmul_id(int type, const void *w, int64_t n_experts, int64_t n, int64_t k,
                 int64_t expert_stride, const void *x, int x_dtype, int64_t n_tokens,
                 const int32_t *ids, int64_t top_k, void *y, int y_dtype,
                 void *workspace, size_t workspace_bytes, void *stream);
/* kq_matmul_id with an explicit path: KQ_PATH_SIMPLE, KQ_PATH_GEMV (grouped
 * mat-vec), KQ_PATH_GEMM (grouped tensor-core GEMM, bf16 x only) or
 * KQ_PATH_GEMV_TC (tensor-core kernel for few pairs per expert). */
KQ_API int kq_matmul_id_ex(int type, const void *w, int64_t n_experts, int64_t n, int64_t k,
                    int64_t expert_stride, const void *x, int x_dtype, int64_t n_tokens,
                    const int32_t *ids, int64_t top_k, void *y, int y_dtype,
                    void *workspace, size_t workspace_bytes, int path, void *stream);

/*
 * kq_matmul_id_noalloc -- kq_matmul_id for callers that cannot allocate
 * device memory.  (The pages have no counterpart of this call.)
 * Some callers are handed only their input and output buffers and have no
 * device allocator of their own -- a plugin running inside another
 * framework's execution plan, or a host language that cannot call
 * cudaMalloc -- so they cannot provide kq_matmul_id's workspace.  This call
 * takes the same arguments minus the workspace and computes the same result
 * with the same kernels, using a scratch array built into the library:
 *   * The array holds 256 KiB; a request whose
 *     kq_matmul_id_workspace_bytes(n_tokens, top_k, n_experts) exceeds it is
 *     rejected with KQ_ERR_WORKSPACE before any work is enqueued.
 *   * Every GPU that loads the library keeps the array until the process
 *     exits.  Each call looks up the array's device address in the current
 *     device's context (cudaGetSymbolAddress), so the address stays valid
 *     after that context is destroyed and created again.  The first call on
 *     a device is its set-up: it loads the library's device code there (lazy
 *     module loading), so make that first call before any stream capture.
 *   * Every call shares the one array: calls that overlap on the GPU (on
 *     different streams, or from different host threads) race and give
 *     wrong results.  Order them on one stream.  The array keeps the last
 *     call's contents; nothing in it needs to start at zero.
 *   * Nothing is allocated: no cudaMalloc, cudaFree or allocating library call.
 */
KQ_API int kq_matmul_id_noalloc(int type, const void *w, int64_t n_experts, int64_t n, int64_t k,
                                int64_t expert_stride, const void *x, int x_dtype, int64_t n_tokens,
                                const int32_t *ids, int64_t top_k, void *y, int y_dtype,
                                void *stream);

/* ---- fused GLU activations (kq_matmul_id_glu) ---- */
#define KQ_ACT_SILU       0   /* g / (1 + exp(-g))                                   */
#define KQ_ACT_GELU_TANH  1   /* 0.5 g (1 + tanh(sqrt(2/pi) (g + 0.044715 g^3)))      */

/*
 * kq_matmul_id_glu -- fused mixture-of-experts GLU: gate and up expert
 * products share the grouping and each activation load, and the epilogue
 * writes act(gate) * up.
 * Defines: mlx-kquant bindings.cpp `moe_glu_gather_kq(x, gate_w, up_w,
 * kquant_type, indices, act)`: for every token t and slot s, e = ids[t][s],
 *   y[t][s][j] = act(sum_k dequant(w_gate_e)[j][k] x[t][k]) *
 *                sum_k dequant(w_up_e)[j][k] x[t][k].
 *   w_gate, w_up  two expert stacks of the same shape and expert_stride, laid
 *                 out as kq_matmul_id's w (device)
 *   act           KQ_ACT_SILU or KQ_ACT_GELU_TANH
 * Other arguments, the workspace (kq_matmul_id_workspace_bytes), invalid
 * ids (NaN rows, device error word) and errors as kq_matmul_id.  Q4_K with
 * fp32 x up to one routed pair per expert runs the grouped bandwidth kernel
 * (a tile holding each output row's gate and up weights), otherwise the
 * few-pairs tensor-core kernel (a gate pass and an up pass per unit over
 * the same activation tile).  Q8_0 and Q5_K (K % 256 == 0) and Q2_K
 * (K % 1024 == 0) with bf16 x run the grouped tensor-core GEMM twice over
 * one grouping: the up projection into y, then the gate projection, whose
 * epilogue writes act(gate) * y (a bf16 y holds the up projection rounded
 * to bf16 in between).  Other codecs and shapes: the plain grouped kernel.
 */
KQ_API int kq_matmul_id_glu(int type, const void *w_gate, const void *w_up, int64_t n_experts,
                            int64_t n, int64_t k, int64_t expert_stride, const void *x, int x_dtype,
                            int64_t n_tokens, const int32_t *ids, int64_t top_k, void *y,
                            int y_dtype, int act, void *workspace, size_t workspace_bytes,
                            void *stream);

/*
 * kq_matmul_id_mix -- mixture-of-experts down projection with the routing
 * mix folded in.
 * Defines: mlx-kquant bindings.cpp `gather_qmv_mix_kq(x, w, shexp_w,
 * kquant_type, indices, scores)` (every slot's product accumulated in f32,
 * weighted by its score, in place of a gather followed by a weighted sum),
 * with the slotted input of mlx-native's `quantized_matmul_id_ggml_pooled_
 * slotted` (one activation row per routed slot).  For every token t:
 *   y[t][j] = sum over s = 0 .. top_k-1 of
 *             scores[t][s] * sum_k dequant(w_{ids[t][s]})[j][k] x[t][s][k].
 *   x        [n_tokens, top_k, k] f32 or bf16 (device), e.g. the output of
 *            kq_matmul_id_glu for the same ids
 *   ids      [n_tokens, top_k] int32 (device)
 *   scores   [n_tokens, top_k] f32 (device)
 *   y        [n_tokens, n] f32 or bf16 (device)
 *   w, n_experts, n, k, expert_stride  as kq_matmul_id
 *   workspace  device scratch of at least
 *        kq_matmul_id_mix_workspace_bytes(n_tokens, top_k, n_experts, n) bytes:
 *        kq_matmul_id's sections at the same offsets, then the fp32
 *        per-pair products [n_tokens * top_k, n].
 *   path     KQ_PATH_AUTO / SIMPLE / GEMV / GEMM as kq_matmul_id_ex,
 *            optionally OR KQ_FLAG_REUSE_GROUPING.
 * The slots are summed in order in fp32, so equal inputs give equal bits.
 * A shared expert of the routed experts' shape is one more slot: store it in
 * the stack as one more expert and give each token a slot with its id and
 * weight.  A token with any id outside [0, n_experts) gets a NaN row and the
 * device error word is set (KQ_ERR_DEVICE from kq_device_status).
 * KQ_FLAG_REUSE_GROUPING skips the grouping step and uses the one the
 * workspace already holds.  Use it only when an earlier kq_matmul_id,
 * kq_matmul_id_ex, kq_matmul_id_glu or kq_matmul_id_mix call on the same
 * stream grouped these same ids (same n_tokens, top_k, n_experts) into this
 * workspace and nothing has written the workspace's first
 * kq_matmul_id_workspace_bytes(n_tokens, top_k, n_experts) bytes since: a
 * stale grouping makes the kernels read and write outside the buffers.
 * Errors as kq_matmul_id; scores null gives KQ_ERR_ARG.
 */
#define KQ_FLAG_REUSE_GROUPING 0x400
KQ_API size_t kq_matmul_id_mix_workspace_bytes(int64_t n_tokens, int64_t top_k, int64_t n_experts,
                                               int64_t n);
KQ_API int kq_matmul_id_mix(int type, const void *w, int64_t n_experts, int64_t n, int64_t k,
                            int64_t expert_stride, const void *x, int x_dtype, int64_t n_tokens,
                            const int32_t *ids, const float *scores, int64_t top_k, void *y,
                            int y_dtype, void *workspace, size_t workspace_bytes, int path,
                            void *stream);

/*
 * kq_moe_group -- the grouping step of kq_matmul_id, exposed for testing.
 * Defines: mlx-kquant bindings.cpp `expert_tile_map` and mlx-native's map0
 * schedule (per-expert routed counts and routed-token lists, built on the
 * device without a host sync).
 *   ids      [n_tokens * top_k] int32 (device)
 *   counts   [n_experts] int32 out: pairs routed to each expert (device)
 *   offsets  [n_experts + 1] int32 out: exclusive prefix sum of counts (device)
 *   perm     [n_tokens * top_k] int32 out: pair indices p = t*top_k + s
 *            grouped by expert, ascending p inside each expert (a stable
 *            sort by expert id); pairs with an invalid id are left out and
 *            the tail perm[offsets[n_experts] ..] is set to -1 (device)
 * ids must be 16-byte aligned (KQ_ERR_ALIGN otherwise), counts, offsets and
 * perm 4-byte aligned.  Sets the device error word if any id is outside
 * [0, n_experts).
 */
KQ_API int kq_moe_group(const int32_t *ids, int64_t n_pairs, int64_t n_experts,
                 int32_t *counts, int32_t *offsets, int32_t *perm, void *stream);

/*
 * kq_get_rows -- decode selected weight rows (an embedding lookup).
 * Defines: Ternary Bonsai ternel_packed_model.py `_GET_ROWS_SOURCE` /
 * `tq1_get_rows`: decode exactly the requested rows of a packed table, with
 * no intermediate row buffer; a row id outside the table reads as an
 * all-zero row.
 *   w     [rows, kq_row_bytes(type, k)] u8 wire blocks (device)
 *   ids   [n_ids] int32 row ids (device; may come from earlier work)
 *   out   [n_ids, k] of out_dtype (KQ_F32, KQ_BF16 or KQ_F16) (device)
 * Row t of out is the fp32 decode of row ids[t] (bit-exact, as
 * kq_dequantize), rounded to nearest even for bf16/f16.  An id outside
 * [0, rows) writes zeros to its row and sets the device error word
 * (kq_device_status returns KQ_ERR_DEVICE).  All codecs.
 */
KQ_API int kq_get_rows(int type, const void *w, int64_t rows, int64_t k, const int32_t *ids,
                       int64_t n_ids, void *out, int out_dtype, void *stream);

/*
 * kq_validate -- scan TQ1_G128 weights for bytes above the legal maximum
 * (ternel_packed_model.py: MAX_FULL_CODE_BYTE = 242, MAX_TAIL_CODE_BYTE = 26).
 * SYNCHRONIZES `stream`.  *first_bad_block (host) receives the row-major index
 * of the first block holding an illegal byte, or -1.  Other codecs have no
 * illegal byte patterns and report -1.
 */
KQ_API int kq_validate(int type, const void *w, int64_t rows, int64_t k,
                int64_t *first_bad_block, void *stream);

/*
 * kq_device_status -- SYNCHRONIZES `stream`, then returns and clears the
 * current device's sticky error word: KQ_OK, KQ_ERR_DEVICE (an expert id was
 * out of range in some call since the last check), KQ_ERR_DEVICE_TIMEOUT (a
 * kernel gave up a bounded wait and left its outputs incomplete) or, from
 * the KQ_DEBUG build only, KQ_ERR_DEVICE_BOUNDS (a device bounds check found
 * an index out of range and skipped the access).  When more than one is set
 * it reports the timeout before the bounds check and that before the ids.
 */
KQ_API int kq_device_status(void *stream);

/* Static description of a status code. */
KQ_API const char *kq_status_string(int status);

#ifdef __cplusplus
}
#endif
#endif /* KQ_H */
