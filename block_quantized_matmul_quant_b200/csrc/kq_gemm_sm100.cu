// kq_gemm_sm100.cu -- tensor-core product for many activation rows (prefill).
#include "kq_launch.h"

namespace kq {

bool gemm_supported(int, int64_t, int64_t, int, int) { return false; }
cudaError_t launch_gemm(int, const void *, int64_t, int64_t, const void *, int64_t, void *, int,
                        cudaStream_t) {
    return cudaErrorNotSupported;
}

}  // namespace kq
