// kq_api.cu -- the C ABI (include/kq.h): argument validation, dispatch and
// the device status word.  All validation happens before any launch.
#include <atomic>
#include <mutex>
#include <string.h>

#include "kq_common.cuh"
#include "kq_launch.h"

namespace kq {

__device__ unsigned long long g_scan_first_bad;
__device__ unsigned int g_error_word = 0;

// Per-device host caches below are atomics: calls may come from several
// host threads, and each thread that finds an entry empty stores the same
// value.
static int current_device() {
    int dev = 0;
    cudaGetDevice(&dev);
    return dev >= 0 && dev < 64 ? dev : 0;
}

// Device address of this device's error word (cached per device ordinal).
unsigned int *error_word() {
    static std::atomic<unsigned int *> cache[64];
    const int dev = current_device();
    unsigned int *w = cache[dev].load(std::memory_order_relaxed);
    if (w == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_error_word) == cudaSuccess) {
            w = static_cast<unsigned int *>(p);
            cache[dev].store(w, std::memory_order_relaxed);
        }
    }
    return w;
}

int sm_count() {
    static std::atomic<int> cache[64];
    const int dev = current_device();
    int v = cache[dev].load(std::memory_order_relaxed);
    if (v == 0) {
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
        cache[dev].store(v, std::memory_order_relaxed);
    }
    return v;
}

static int block_weights(int type) {
    switch (type) {
    case KQ_Q8_0: return Geom<KQ_Q8_0>::QK;
    case KQ_Q2_K: return Geom<KQ_Q2_K>::QK;
    case KQ_Q4_K: return Geom<KQ_Q4_K>::QK;
    case KQ_Q5_K: return Geom<KQ_Q5_K>::QK;
    case KQ_Q6_K: return Geom<KQ_Q6_K>::QK;
    case KQ_TQ1_G128: return Geom<KQ_TQ1_G128>::QK;
    default: return 0;
    }
}
static int block_bytes(int type) {
    switch (type) {
    case KQ_Q8_0: return Geom<KQ_Q8_0>::BB;
    case KQ_Q2_K: return Geom<KQ_Q2_K>::BB;
    case KQ_Q4_K: return Geom<KQ_Q4_K>::BB;
    case KQ_Q5_K: return Geom<KQ_Q5_K>::BB;
    case KQ_Q6_K: return Geom<KQ_Q6_K>::BB;
    case KQ_TQ1_G128: return Geom<KQ_TQ1_G128>::BB;
    default: return 0;
    }
}

// Alignment an expert stride must keep for the codec's loads: 16 bytes for
// Q4_K and Q5_K (bulk copies, tensor maps and 8-byte loads of the block),
// 4 for Q2_K's word loads, 2 for the codecs read as bytes and half words.
static int64_t stride_align(int type) {
    switch (type) {
    case KQ_Q4_K: case KQ_Q5_K: return 16;
    case KQ_Q2_K: return 4;
    default: return 2;
    }
}

static bool mul_ok(int64_t a, int64_t b, int64_t *r) { return !__builtin_mul_overflow(a, b, r); }
static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Current device must be sm_100 (B200); cached per device ordinal.
static int check_device() {
    static std::atomic<int> cache[64];  // 0 unknown, 1 ok, -1 not sm_100
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return KQ_ERR_CUDA;
    if (dev < 0 || dev >= 64) return KQ_ERR_UNSUPPORTED;
    int c = cache[dev].load(std::memory_order_relaxed);
    if (c == 0) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
            return KQ_ERR_CUDA;
        c = (major == 10 && minor == 0) ? 1 : -1;
        cache[dev].store(c, std::memory_order_relaxed);
    }
    return c == 1 ? KQ_OK : KQ_ERR_UNSUPPORTED;
}

static int to_status(cudaError_t e) { return e == cudaSuccess ? KQ_OK : KQ_ERR_CUDA; }

// Shared checks of a weight matrix [n, k] of `type`.
static int check_weights(int type, const void *w, int64_t n, int64_t k, int64_t *row_bytes) {
    const int qk = block_weights(type);
    if (qk == 0) return KQ_ERR_TYPE;
    if (w == nullptr) return KQ_ERR_ARG;
    if (n <= 0 || k <= 0) return KQ_ERR_ARG;
    if (k % qk) return KQ_ERR_SHAPE;
    if (!aligned16(w)) return KQ_ERR_ALIGN;
    int64_t rb = (k / qk) * block_bytes(type), total;
    if (!mul_ok(rb, n, &total)) return KQ_ERR_OVERFLOW;
    *row_bytes = rb;
    return KQ_OK;
}

static int check_act(const void *p, int dtype, int64_t rows, int64_t cols, bool allow_f16) {
    if (p == nullptr) return KQ_ERR_ARG;
    if (dtype != KQ_F32 && dtype != KQ_BF16 && !(allow_f16 && dtype == KQ_F16)) return KQ_ERR_DTYPE;
    if (!aligned16(p)) return KQ_ERR_ALIGN;
    int64_t e, b;
    if (!mul_ok(rows, cols, &e) || !mul_ok(e, 4, &b)) return KQ_ERR_OVERFLOW;
    return KQ_OK;
}

// Workspace layout of kq_matmul_id (256-byte aligned sections).
struct IdWorkspace {
    size_t counts, offsets, perm, tiles, n_tiles, total;
};
static size_t up256(size_t v) { return (v + 255) & ~size_t(255); }
// Entries of the tensor-core tile list: tiles of at least 8 pairs (the
// few-pairs kernel with fp32 activations; 16 and more otherwise), one ragged
// tile per expert at most.
static int64_t id_max_tiles(int64_t pairs, int64_t n_experts) { return pairs / 8 + n_experts + 1; }
// The routing-mix call adds one section after the grouping: the fp32
// per-pair products [pairs, n].
static bool mix_workspace_bytes(const struct IdWorkspace &l, int64_t pairs, int64_t n, size_t *total) {
    int64_t e, b;
    if (n <= 0 || !mul_ok(pairs, n, &e) || !mul_ok(e, 4, &b) || b > INT64_MAX - 512) return false;
    *total = l.total + up256((size_t)b);
    return true;
}
static bool id_workspace_layout(int64_t n_tokens, int64_t top_k, int64_t n_experts, IdWorkspace *l) {
    int64_t pairs;
    if (n_tokens <= 0 || top_k <= 0 || n_experts <= 0) return false;
    if (!mul_ok(n_tokens, top_k, &pairs) || pairs > INT32_MAX) return false;
    size_t off = 0;
    l->counts = off;  off += up256(4 * (size_t)n_experts);
    l->offsets = off; off += up256(4 * (size_t)(n_experts + 1));
    l->perm = off;    off += up256(4 * (size_t)pairs);
    l->tiles = off;   off += up256(8 * (size_t)id_max_tiles(pairs, n_experts));
    l->n_tiles = off; off += 256;
    l->total = off;
    return true;
}

// Activation rows from which the tensor-core kernel serves bf16 inputs.
// Measured on B200 (Q4_K 11008 x 4096, us per call, bandwidth vs tensor-core
// kernel): 4 rows 20.3 vs 26.9, 8 rows 34.4 vs 26.9; the bandwidth kernel
// takes 5..8 rows in one pass of eight, so five rows already cost 34.
constexpr int64_t GEMM_MIN_M = 5;
// Expert-indexed dispatch by mean (token, slot) pairs per expert, from the
// sweep on B200 (64 experts of 1408 x 2048, top-6, bf16; us per call,
// bandwidth kernel / few-pairs tensor-core kernel / GEMM): 8 tokens 48.9 /
// 41.7 / 51.8, 32 tokens 98.6 / 65.5 / 82.0, 128 tokens 265.4 / 93.3 /
// 112.1, 256 tokens 494.2 / 144.7 / 151.9, 512 tokens 943.4 / 243.4 /
// 227.9.  With bf16 activations the few-pairs kernel up to 32 pairs per
// expert, the GEMM beyond; with fp32 ones (no GEMM, tiles of 8 in the
// few-pairs kernel) the bandwidth kernel up to one pair per expert and the
// few-pairs kernel beyond.
constexpr int64_t ID_GEMV_MAX_PAIRS_PER_EXPERT = 1;
constexpr int64_t ID_TC_MAX_PAIRS_PER_EXPERT = 32;
// The few-pairs kernel's int8 form (one K = 32 MMA per sub-block, 8 pairs a
// tile) measured faster only at the smallest routings (8 tokens: 40.1 vs
// 41.7 us; 32 tokens: 69.4 vs 65.5; 64 tokens: 89.8 vs 72.1).
constexpr int64_t ID_TC_I8_MAX_PAIRS_PER_EXPERT = 1;
// The TQ1 bandwidth kernel takes two activation rows per pass over the
// weights; beyond this many rows the tensor-core kernel (K % 512 == 0, bf16
// activations) or else the plain kernel is used.
constexpr int64_t TQ1_GEMV_MAX_M = 8;
// Activation rows from which the tensor-core kernel serves TQ1 products.
// Measured on B200 (TQ1_G128 5120 x 17408, bf16, us per call, bandwidth vs
// tensor-core kernel): 6 rows 84.5 vs 101.1, 8 rows 112.4 vs 101.2, 12 rows
// 168.3 vs 101.2 (the tensor-core kernel has only 40 weight-row tiles here,
// so its time stays flat up to 128 rows; 512 rows 136.3).
constexpr int64_t TQ1_GEMM_MIN_M = 8;
// Activation rows from which the tensor-core kernel serves Q8_0 products
// (bf16 activations, K % 256 == 0); below it the plain kernel.  Measured on
// B200 (Q8_0 4096 x 4096, us per call, plain vs tensor-core kernel): 1 row
// 18.7 vs 24.6, 4 rows 31.4 vs 24.9, 16 rows 68.2 vs 24.9, 512 rows 1825 vs
// 34.8.
constexpr int64_t Q8_0_GEMM_MIN_M = 3;
// Likewise for Q2_K (K % 1024 == 0): 1 row 22.9 vs 25.2, 2 rows 26.1 vs
// 25.2, 16 rows 75.4 vs 25.2, 512 rows 2076 vs 35.2.
constexpr int64_t Q2_K_GEMM_MIN_M = 2;

}  // namespace kq

using namespace kq;

extern "C" {

int kq_block_weights(int type) { return block_weights(type); }
int kq_block_bytes(int type) { return block_bytes(type); }
int64_t kq_row_bytes(int type, int64_t k) {
    const int qk = block_weights(type);
    if (qk == 0 || k < 0 || k % qk) return -1;
    return (k / qk) * block_bytes(type);
}

int kq_dequantize(int type, const void *w, int64_t rows, int64_t k, void *out, int out_dtype,
                  void *stream) {
    int64_t rb;
    int st = check_weights(type, w, rows, k, &rb);
    if (st) return st;
    if ((st = check_act(out, out_dtype, rows, k, true))) return st;
    if ((st = check_device())) return st;
    return to_status(launch_dequant(type, w, rows, k, out, out_dtype, (cudaStream_t)stream));
}

int kq_matmul_ex(int type, const void *w, int64_t n, int64_t k, const void *x, int x_dtype,
                 int64_t m, void *y, int y_dtype, int path, void *stream) {
    int64_t rb;
    int st = check_weights(type, w, n, k, &rb);
    if (st) return st;
    if (m <= 0) return KQ_ERR_ARG;
    if ((st = check_act(x, x_dtype, m, k, false))) return st;
    if ((st = check_act(y, y_dtype, m, n, false))) return st;
    const bool indep = (path & KQ_FLAG_INDEPENDENT) != 0;
    const bool const_w = indep || (path & KQ_FLAG_CONST_WEIGHTS) != 0;
    path &= ~(KQ_FLAG_CONST_WEIGHTS | KQ_FLAG_INDEPENDENT);
    if (path < KQ_PATH_AUTO || path > KQ_PATH_GEMV_TC) return KQ_ERR_ARG;
    if ((st = check_device())) return st;
    cudaStream_t s = (cudaStream_t)stream;
    const bool can_tc = moe_mma_supported(type, n, k, x_dtype, y_dtype);
    const bool can_gemm = gemm_supported(type, n, k, x_dtype, y_dtype);
    const bool can_gemv = gemv_supported(type, n, k, x_dtype, m);
    if (path == KQ_PATH_AUTO) {
        if (can_gemm && m >= (type == KQ_TQ1_G128 ? TQ1_GEMM_MIN_M
                              : type == KQ_Q8_0   ? Q8_0_GEMM_MIN_M
                              : type == KQ_Q2_K   ? Q2_K_GEMM_MIN_M
                                                  : GEMM_MIN_M))
            path = KQ_PATH_GEMM;
        // fp32 activations past one pass of the bandwidth kernel: the
        // few-rows tensor-core kernel reads the weights once per 8 rows of a
        // tile instead of once per 8-row launch
        else if (can_tc && x_dtype == KQ_F32 && m > 8) path = KQ_PATH_GEMV_TC;
        else if (can_gemv && (type != KQ_TQ1_G128 || m <= TQ1_GEMV_MAX_M)) path = KQ_PATH_GEMV;
        else path = KQ_PATH_SIMPLE;
    }
    switch (path) {
    case KQ_PATH_GEMV_TC:
        if (!can_tc) return KQ_ERR_UNSUPPORTED;
        return to_status(launch_gemv_tc(w, n, k, x, x_dtype, m, y, y_dtype, m <= 4, s));
    case KQ_PATH_GEMM:
        if (!can_gemm) return KQ_ERR_UNSUPPORTED;
        return to_status(launch_gemm(type, w, n, k, x, m, y, y_dtype, s));
    case KQ_PATH_GEMV:
        if (!can_gemv) return KQ_ERR_UNSUPPORTED;
        return to_status(launch_gemv(type, w, n, k, x, x_dtype, m, y, y_dtype,
                                     indep ? GemvOrder::kIndependent
                                           : const_w ? GemvOrder::kConstWeights : GemvOrder::kStream,
                                     s));
    default:
        return to_status(launch_simple_matmul(type, w, n, k, x, x_dtype, m, y, y_dtype, s, indep));
    }
}

int kq_matmul(int type, const void *w, int64_t n, int64_t k, const void *x, int x_dtype, int64_t m,
              void *y, int y_dtype, void *stream) {
    return kq_matmul_ex(type, w, n, k, x, x_dtype, m, y, y_dtype, KQ_PATH_AUTO, stream);
}

size_t kq_matmul_id_workspace_bytes(int64_t n_tokens, int64_t top_k, int64_t n_experts) {
    IdWorkspace l;
    if (!id_workspace_layout(n_tokens, top_k, n_experts, &l)) return 0;
    return l.total;
}

size_t kq_matmul_id_mix_workspace_bytes(int64_t n_tokens, int64_t top_k, int64_t n_experts, int64_t n) {
    IdWorkspace l;
    size_t total;
    if (!id_workspace_layout(n_tokens, top_k, n_experts, &l)) return 0;
    if (!mix_workspace_bytes(l, n_tokens * top_k, n, &total)) return 0;
    return total;
}

}  // extern "C"

namespace kq {
// Host validation shared by the expert-indexed calls; fills the kernel
// arguments (workspace sections included).  Nothing is launched.  With
// `slotted` (the routing-mix call) x has one row per pair, y one row per
// token, and the per-pair products go to an fp32 section of the workspace
// after the grouping's sections.
static int id_setup(int type, const void *w, int64_t n_experts, int64_t n, int64_t k,
                    int64_t expert_stride, const void *x, int x_dtype, int64_t n_tokens,
                    const int32_t *ids, int64_t top_k, void *y, int y_dtype, void *workspace,
                    size_t workspace_bytes, IdArgs *a, int64_t *pairs_out, bool slotted = false) {
    int64_t rb;
    int st = check_weights(type, w, n, k, &rb);
    if (st) return st;
    if (n_experts <= 0 || n_experts > 65535 || n_tokens <= 0) return KQ_ERR_ARG;
    if (top_k <= 0 || top_k > n_experts) return KQ_ERR_ARG;
    int64_t per_expert, last, pairs, ypairs;
    if (!mul_ok(n, rb, &per_expert)) return KQ_ERR_OVERFLOW;
    if (expert_stride < per_expert || expert_stride % stride_align(type)) return KQ_ERR_SHAPE;
    if (!mul_ok(n_experts - 1, expert_stride, &last) ||
        __builtin_add_overflow(last, per_expert, &last))
        return KQ_ERR_OVERFLOW;
    if (!mul_ok(n_tokens, top_k, &pairs) || pairs > INT32_MAX) return KQ_ERR_OVERFLOW;
    if (!mul_ok(pairs, n, &ypairs)) return KQ_ERR_OVERFLOW;
    if ((st = check_act(x, x_dtype, slotted ? pairs : n_tokens, k, false))) return st;
    if ((st = check_act(y, y_dtype, slotted ? n_tokens : pairs, n, false))) return st;
    if (ids == nullptr) return KQ_ERR_ARG;
    if (!aligned16(ids)) return KQ_ERR_ALIGN;
    IdWorkspace l;
    if (!id_workspace_layout(n_tokens, top_k, n_experts, &l)) return KQ_ERR_OVERFLOW;
    size_t need = l.total;
    if (slotted && !mix_workspace_bytes(l, pairs, n, &need)) return KQ_ERR_OVERFLOW;
    if (workspace == nullptr || workspace_bytes < need) return KQ_ERR_WORKSPACE;
    if (!aligned16(workspace)) return KQ_ERR_ALIGN;
    char *ws = static_cast<char *>(workspace);
    a->type = type; a->w = w; a->n_experts = n_experts; a->n = n; a->k = k;
    a->expert_stride = expert_stride; a->x = x; a->x_dtype = x_dtype; a->n_tokens = n_tokens;
    a->top_k = top_k; a->y = y; a->y_dtype = y_dtype;
    a->counts = reinterpret_cast<int32_t *>(ws + l.counts);
    a->offsets = reinterpret_cast<int32_t *>(ws + l.offsets);
    a->perm = reinterpret_cast<int32_t *>(ws + l.perm);
    a->tiles = reinterpret_cast<int32_t *>(ws + l.tiles);
    a->n_tiles = reinterpret_cast<int32_t *>(ws + l.n_tiles);
    if (slotted) {
        a->x_slotted = true;
        a->y = ws + l.total;
        a->y_dtype = KQ_F32;
    }
    *pairs_out = pairs;
    return KQ_OK;
}
}  // namespace kq

// The expert product's kernel for these arguments (KQ_PATH_AUTO resolved),
// or a negative status; *bn: the token-tile width its tile list needs (0:
// none).
static int id_path(IdArgs &a, int path, int64_t pairs, int *bn) {
    const bool can_gemv = moe_gemv_supported(a.type, a.n, a.k, a.n_experts);
    // (the weights' tensor map needs an expert stride of whole 16-byte units)
    const bool can_gemm = gemm_supported(a.type, a.n, a.k, a.x_dtype, a.y_dtype, true) && a.expert_stride % 16 == 0;
    const bool can_tc = moe_mma_supported(a.type, a.n, a.k, a.x_dtype, a.y_dtype);
    if (path == KQ_PATH_AUTO) {
        const bool f32x = a.x_dtype == KQ_F32;
        if (can_gemv && ((f32x && pairs <= ID_GEMV_MAX_PAIRS_PER_EXPERT * a.n_experts) || !(can_tc || can_gemm)))
            path = KQ_PATH_GEMV;
        else if (can_tc && (pairs <= ID_TC_MAX_PAIRS_PER_EXPERT * a.n_experts || !can_gemm)) path = KQ_PATH_GEMV_TC;
        else if (can_gemm) path = KQ_PATH_GEMM;
        else path = can_gemv ? KQ_PATH_GEMV : KQ_PATH_SIMPLE;
    }
    if (path == KQ_PATH_GEMM && !can_gemm) return KQ_ERR_UNSUPPORTED;
    if (path == KQ_PATH_GEMV && !can_gemv) return KQ_ERR_UNSUPPORTED;
    if (path == KQ_PATH_GEMV_TC && !can_tc) return KQ_ERR_UNSUPPORTED;
    // the few-pairs kernel's int8 form (8 pairs a tile) while the pairs of
    // an expert fit one such tile on average
    a.tc_i8 = path == KQ_PATH_GEMV_TC && pairs <= ID_TC_I8_MAX_PAIRS_PER_EXPERT * a.n_experts;
    *bn = path == KQ_PATH_GEMM ? gemm_id_bn(a.n_tokens, a.top_k, a.n_experts)
        : path == KQ_PATH_GEMV_TC ? moe_mma_bn(a.x_dtype, a.tc_i8) : 0;
    return path;
}

// The grouping (and the tile list when bn > 0) into the workspace; y (or
// nullptr) takes the NaN rows of invalid ids.
static cudaError_t id_group(const IdArgs &a, const int32_t *ids, int64_t pairs, void *y, int y_dtype, int bn,
                            cudaStream_t s) {
    return launch_moe_group(ids, pairs, a.n_experts, const_cast<int32_t *>(a.counts), const_cast<int32_t *>(a.offsets),
                            const_cast<int32_t *>(a.perm), y, y_dtype, a.n, s, bn, const_cast<int32_t *>(a.tiles),
                            const_cast<int32_t *>(a.n_tiles), id_max_tiles(pairs, a.n_experts));
}

// The expert product over a grouping (and tile list) already in the
// workspace (a.y: its output, a.y_dtype).
static int id_product(const IdArgs &a, int path, int bn, cudaStream_t s) {
    cudaError_t e;
    if (path == KQ_PATH_GEMM) e = launch_gemm_id(a, bn, s);
    else if (path == KQ_PATH_GEMV_TC) e = launch_moe_mma(a, s);
    else if (path == KQ_PATH_GEMV) e = launch_moe_gemv(a, s);
    else e = launch_simple_id(a, s);
    return to_status(e);
}

extern "C" {

int kq_matmul_id_ex(int type, const void *w, int64_t n_experts, int64_t n, int64_t k,
                    int64_t expert_stride, const void *x, int x_dtype, int64_t n_tokens,
                    const int32_t *ids, int64_t top_k, void *y, int y_dtype, void *workspace,
                    size_t workspace_bytes, int path, void *stream) {
    IdArgs a;
    int64_t pairs;
    int st = id_setup(type, w, n_experts, n, k, expert_stride, x, x_dtype, n_tokens, ids, top_k, y,
                      y_dtype, workspace, workspace_bytes, &a, &pairs);
    if (st) return st;
    if (path < KQ_PATH_AUTO || path > KQ_PATH_GEMV_TC) return KQ_ERR_ARG;
    if ((st = check_device())) return st;
    int bn = 0;
    if ((path = id_path(a, path, pairs, &bn)) < 0) return path;
    cudaStream_t s = (cudaStream_t)stream;
    if (id_group(a, ids, pairs, y, y_dtype, bn, s) != cudaSuccess) return KQ_ERR_CUDA;
    return id_product(a, path, bn, s);
}

int kq_matmul_id_glu(int type, const void *w_gate, const void *w_up, int64_t n_experts, int64_t n,
                     int64_t k, int64_t expert_stride, const void *x, int x_dtype, int64_t n_tokens,
                     const int32_t *ids, int64_t top_k, void *y, int y_dtype, int act, void *workspace,
                     size_t workspace_bytes, void *stream) {
    IdArgs a;
    int64_t pairs, rb_unused;
    int st = id_setup(type, w_gate, n_experts, n, k, expert_stride, x, x_dtype, n_tokens, ids, top_k,
                      y, y_dtype, workspace, workspace_bytes, &a, &pairs);
    if (st) return st;
    if ((st = check_weights(type, w_up, n, k, &rb_unused))) return st;
    if (act != KQ_ACT_SILU && act != KQ_ACT_GELU_TANH) return KQ_ERR_ARG;
    if ((st = check_device())) return st;
    a.w2 = w_up;
    a.act = act;
    cudaStream_t s = (cudaStream_t)stream;
    // Q4_K: the few-pairs tensor-core kernel (a gate pass and an up pass per
    // unit), except fp32 activations up to one pair per expert (the
    // bandwidth kernel).  Q8_0, Q2_K and Q5_K with bf16 activations: the
    // grouped tensor-core GEMM twice over one grouping -- the up projection
    // into y, then the gate projection, whose epilogue writes
    // act(gate) * y.  Other codecs and shapes: the plain kernel.
    const bool few = x_dtype == KQ_F32 && pairs <= ID_GEMV_MAX_PAIRS_PER_EXPERT * n_experts;
    const bool tc = moe_mma_supported(type, n, k, x_dtype, y_dtype) && !(few && moe_gemv_supported(type, n, k, n_experts));
    const bool gemm = !tc && type != KQ_Q4_K && gemm_supported(type, n, k, x_dtype, y_dtype, true) &&
                      expert_stride % 16 == 0;
    a.tc_i8 = tc && pairs <= ID_TC_I8_MAX_PAIRS_PER_EXPERT * n_experts;
    const int bn = tc ? moe_mma_bn(x_dtype, a.tc_i8) : gemm ? gemm_id_bn(n_tokens, top_k, n_experts) : 0;
    if (id_group(a, ids, pairs, y, y_dtype, bn, s) != cudaSuccess) return KQ_ERR_CUDA;
    if (tc) return to_status(launch_moe_mma(a, s));
    if (gemm) {
        IdArgs up = a;
        up.w = w_up;
        const cudaError_t e = launch_gemm_id(up, bn, s, false);
        if (e != cudaSuccess) return to_status(e);
        return to_status(launch_gemm_id(a, bn, s, true));
    }
    if (moe_gemv_supported(type, n, k, n_experts)) return to_status(launch_moe_gemv(a, s));
    return to_status(launch_simple_glu(a, s));
}

int kq_matmul_id_mix(int type, const void *w, int64_t n_experts, int64_t n, int64_t k,
                     int64_t expert_stride, const void *x, int x_dtype, int64_t n_tokens,
                     const int32_t *ids, const float *scores, int64_t top_k, void *y, int y_dtype,
                     void *workspace, size_t workspace_bytes, int path, void *stream) {
    IdArgs a;
    int64_t pairs;
    int st = id_setup(type, w, n_experts, n, k, expert_stride, x, x_dtype, n_tokens, ids, top_k, y,
                      y_dtype, workspace, workspace_bytes, &a, &pairs, true);
    if (st) return st;
    if (scores == nullptr) return KQ_ERR_ARG;
    if (!aligned16(scores)) return KQ_ERR_ALIGN;
    const bool reuse = (path & KQ_FLAG_REUSE_GROUPING) != 0;
    path &= ~KQ_FLAG_REUSE_GROUPING;
    if (path < KQ_PATH_AUTO || path > KQ_PATH_GEMV_TC) return KQ_ERR_ARG;
    if ((st = check_device())) return st;
    int bn = 0;
    if ((path = id_path(a, path, pairs, &bn)) < 0) return path;
    cudaStream_t s = (cudaStream_t)stream;
    if (!reuse) {
        if (id_group(a, ids, pairs, nullptr, KQ_F32, bn, s) != cudaSuccess) return KQ_ERR_CUDA;
    } else if (bn > 0 &&
               launch_moe_tiles(a.offsets, n_experts, bn, const_cast<int32_t *>(a.tiles),
                                const_cast<int32_t *>(a.n_tiles), id_max_tiles(pairs, n_experts), s) != cudaSuccess) {
        return KQ_ERR_CUDA;   // a reused grouping gets the tile list this product needs
    }
    if ((st = id_product(a, path, bn, s))) return st;
    return to_status(launch_moe_mix(static_cast<const float *>(a.y), ids, scores, n_tokens, top_k,
                                    n_experts, n, y, y_dtype, s));
}

int kq_matmul_id(int type, const void *w, int64_t n_experts, int64_t n, int64_t k,
                 int64_t expert_stride, const void *x, int x_dtype, int64_t n_tokens,
                 const int32_t *ids, int64_t top_k, void *y, int y_dtype, void *workspace,
                 size_t workspace_bytes, void *stream) {
    return kq_matmul_id_ex(type, w, n_experts, n, k, expert_stride, x, x_dtype, n_tokens, ids,
                           top_k, y, y_dtype, workspace, workspace_bytes, KQ_PATH_AUTO, stream);
}

int kq_moe_group(const int32_t *ids, int64_t n_pairs, int64_t n_experts, int32_t *counts,
                 int32_t *offsets, int32_t *perm, void *stream) {
    if (!ids || !counts || !offsets || !perm) return KQ_ERR_ARG;
    if (n_pairs <= 0 || n_pairs > INT32_MAX || n_experts <= 0 || n_experts > 65535)
        return KQ_ERR_ARG;
    auto aligned4 = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; };
    if (!aligned16(ids) || !aligned4(counts) || !aligned4(offsets) || !aligned4(perm))
        return KQ_ERR_ALIGN;
    int st = check_device();
    if (st) return st;
    return to_status(launch_moe_group(ids, n_pairs, n_experts, counts, offsets, perm, nullptr,
                                      KQ_F32, 0, (cudaStream_t)stream));
}

int kq_get_rows(int type, const void *w, int64_t rows, int64_t k, const int32_t *ids, int64_t n_ids,
                void *out, int out_dtype, void *stream) {
    int64_t rb;
    int st = check_weights(type, w, rows, k, &rb);
    if (st) return st;
    if (ids == nullptr || n_ids <= 0) return KQ_ERR_ARG;
    if (rows > INT32_MAX) return KQ_ERR_OVERFLOW;
    if (!aligned16(ids)) return KQ_ERR_ALIGN;
    if ((st = check_act(out, out_dtype, n_ids, k, true))) return st;
    if ((st = check_device())) return st;
    return to_status(launch_get_rows(type, w, rows, k, ids, n_ids, out, out_dtype, (cudaStream_t)stream));
}

int kq_validate(int type, const void *w, int64_t rows, int64_t k, int64_t *first_bad_block,
                void *stream) {
    int64_t rb;
    int st = check_weights(type, w, rows, k, &rb);
    if (st) return st;
    if (first_bad_block == nullptr) return KQ_ERR_ARG;
    *first_bad_block = -1;
    if (type != KQ_TQ1_G128) return KQ_OK;
    if ((st = check_device())) return st;
    static std::mutex mu;  // the scan result lives in one device word
    std::lock_guard<std::mutex> g(mu);
    cudaStream_t s = (cudaStream_t)stream;
    const unsigned long long none = ~0ull;
    unsigned long long got = none;
    if (cudaMemcpyToSymbolAsync(g_scan_first_bad, &none, sizeof(none), 0,
                                cudaMemcpyHostToDevice, s) != cudaSuccess)
        return KQ_ERR_CUDA;
    unsigned long long *dev_word = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void **>(&dev_word), g_scan_first_bad) != cudaSuccess)
        return KQ_ERR_CUDA;
    if (launch_tq1_scan(w, rows * (k / 128), dev_word, s) != cudaSuccess) return KQ_ERR_CUDA;
    if (cudaMemcpyFromSymbolAsync(&got, g_scan_first_bad, sizeof(got), 0, cudaMemcpyDeviceToHost,
                                  s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return KQ_ERR_CUDA;
    *first_bad_block = (got == none) ? -1 : (int64_t)got;
    return KQ_OK;
}

int kq_device_status(void *stream) {
    int st = check_device();
    if (st) return st;
    cudaStream_t s = (cudaStream_t)stream;
    unsigned int word = 0, zero = 0;
    if (cudaStreamSynchronize(s) != cudaSuccess) return KQ_ERR_CUDA;
    if (cudaMemcpyFromSymbolAsync(&word, g_error_word, sizeof(word), 0, cudaMemcpyDeviceToHost, s) !=
            cudaSuccess ||
        cudaMemcpyToSymbolAsync(g_error_word, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, s) !=
            cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return KQ_ERR_CUDA;
    if (word & ERR_TIMEOUT) return KQ_ERR_DEVICE_TIMEOUT;
    if (word & ERR_BOUNDS) return KQ_ERR_DEVICE_BOUNDS;
    if (word & ERR_BAD_ID) return KQ_ERR_DEVICE;
    return KQ_OK;
}

const char *kq_status_string(int status) {
    switch (status) {
    case KQ_OK: return "ok";
    case KQ_ERR_ARG: return "invalid argument (null pointer, non-positive dimension or top_k)";
    case KQ_ERR_TYPE: return "unknown codec";
    case KQ_ERR_SHAPE: return "K is not a multiple of the block size, or bad stride";
    case KQ_ERR_DTYPE: return "unsupported dtype";
    case KQ_ERR_ALIGN: return "pointer is not 16-byte aligned";
    case KQ_ERR_OVERFLOW: return "size overflow";
    case KQ_ERR_WORKSPACE: return "workspace missing or too small";
    case KQ_ERR_CUDA: return "CUDA runtime error";
    case KQ_ERR_DEVICE: return "device reported an out-of-range expert or row id";
    case KQ_ERR_DEVICE_TIMEOUT: return "a bounded device wait timed out";
    case KQ_ERR_UNSUPPORTED: return "unsupported device or path for these arguments";
    case KQ_ERR_DEVICE_BOUNDS: return "a device bounds check (debug build) found an index out of range";
    default: return "unknown status";
    }
}

}  // extern "C"
