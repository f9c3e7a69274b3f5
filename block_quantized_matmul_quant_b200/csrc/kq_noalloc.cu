// kq_noalloc.cu -- kq_matmul_id_noalloc: the expert-indexed product for
// callers that cannot allocate device memory.
//
// kq_matmul_id needs a caller-owned scratch buffer for its expert grouping
// (per-expert counts, offsets and the grouped pair list).  Some callers are
// handed only their input and output buffers and have no device allocator
// of their own: a plugin running inside another framework's execution plan,
// or a host language that cannot call cudaMalloc.  This entry point serves
// them from a scratch array compiled into the library instead.
//
// The array is a file-scope __device__ object of KQ_NOALLOC_SCRATCH_BYTES
// bytes: every GPU that loads the library holds it until the process exits.
// In host code the array's name is only a host-side stand-in, so its device
// address is looked up with cudaGetSymbolAddress on every call, with the
// calling device current, and passed on as the workspace of the ordinary
// kq_matmul_id path.  Looking it up each time (a table lookup in the CUDA
// runtime, no allocation) keeps the address right for the context that is
// current now: an address cached from an earlier context (one destroyed by
// cudaDeviceReset and created again) could point at memory the module no
// longer owns.  The first call on a device is the set-up: it loads the
// library's device code on that device (lazy module loading) and so should
// come before any stream capture.  Nothing here allocates.
#include "kq_common.cuh"

namespace {

constexpr size_t KQ_NOALLOC_SCRATCH_BYTES = 256 * 1024;

static __device__ __align__(256) unsigned char g_noalloc_scratch[KQ_NOALLOC_SCRATCH_BYTES];

// Device address of the scratch array in the current device's context.
int scratch_for_current_device(void **out) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return KQ_ERR_CUDA;
    *out = p;
    return KQ_OK;
}

}  // namespace

extern "C" int kq_matmul_id_noalloc(int type, const void *w, int64_t n_experts, int64_t n,
                                    int64_t k, int64_t expert_stride, const void *x, int x_dtype,
                                    int64_t n_tokens, const int32_t *ids, int64_t top_k, void *y,
                                    int y_dtype, void *stream) {
    const size_t need = kq_matmul_id_workspace_bytes(n_tokens, top_k, n_experts);
    if (need == 0) return KQ_ERR_ARG;
    if (need > KQ_NOALLOC_SCRATCH_BYTES) return KQ_ERR_WORKSPACE;  // beyond the built-in scratch
    void *scratch = nullptr;
    const int st = scratch_for_current_device(&scratch);
    if (st != KQ_OK) return st;
    // The grouping step rewrites every scratch word that the product later
    // reads (counts, offsets, the full pair list), so nothing is cleared.
    return kq_matmul_id(type, w, n_experts, n, k, expert_stride, x, x_dtype, n_tokens, ids, top_k, y,
                        y_dtype, scratch, KQ_NOALLOC_SCRATCH_BYTES, stream);
}
