// kq_debug.cu -- entry points that only the KQ_DEBUG build exports
// (include/kq_debug.h).  The release library compiles this file to nothing.
#ifdef KQ_DEBUG
#include "kq_ptx.cuh"

namespace kq {

// One warp.  An mbarrier that expects two arrivals gets one, so its first
// phase never completes.  Lane 0 waits on it with the library's own bounded
// wait (mode 0: the suspending try_wait loop; mode 1: the test-and-sleep
// loop), which gives up after its KQ_SPIN_LIMIT rounds and sets ERR_TIMEOUT
// in the error word.  Nothing else is in flight: no copy, no TMEM.
__global__ void debug_wait_timeout_kernel(int mode, unsigned int *err) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 2);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        mbar_arrive(&bar);
        if (mode == 0)
            mbar_wait(&bar, 0, err);
        else
            mbar_wait_poll(&bar, 0, err);
    }
}

}  // namespace kq

extern "C" KQ_API int kq_debug_wait_timeout(int mode, void *stream) {
    if (mode != 0 && mode != 1) return KQ_ERR_ARG;
    int dev = 0, major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
        return KQ_ERR_CUDA;
    if (major != 10) return KQ_ERR_UNSUPPORTED;
    kq::debug_wait_timeout_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(mode, kq::error_word());
    return cudaGetLastError() == cudaSuccess ? KQ_OK : KQ_ERR_CUDA;
}

extern "C" KQ_API int kq_debug_spin_limit(void) { return (int)KQ_SPIN_LIMIT; }
#endif
