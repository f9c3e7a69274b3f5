// kq_common.cuh -- shared device/host definitions of the CUDA library.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "../../include/kq.h"

namespace kq {

// Codec geometry: weights and bytes per wire block.
template <int TYPE> struct Geom;
template <> struct Geom<KQ_Q8_0>     { static constexpr int QK = 32;  static constexpr int BB = 34; };
template <> struct Geom<KQ_Q2_K>     { static constexpr int QK = 256; static constexpr int BB = 84; };
template <> struct Geom<KQ_Q4_K>     { static constexpr int QK = 256; static constexpr int BB = 144; };
template <> struct Geom<KQ_Q5_K>     { static constexpr int QK = 256; static constexpr int BB = 176; };
template <> struct Geom<KQ_Q6_K>     { static constexpr int QK = 256; static constexpr int BB = 210; };
template <> struct Geom<KQ_TQ1_G128> { static constexpr int QK = 128; static constexpr int BB = 28; };

// Sticky per-device error word (bit 0: bad expert id, bit 1: wait timeout,
// bit 2: a KQ_DEBUG build's bounds check failed).
// It lives in kq_api.cu; kernels receive its device address as a parameter
// (error_word() on the host), since each translation unit is compiled
// without relocatable device code.
unsigned int *error_word();
// Streaming multiprocessors of the current device (cached per device).
int sm_count();
constexpr unsigned ERR_BAD_ID = 1u;
constexpr unsigned ERR_TIMEOUT = 2u;
constexpr unsigned ERR_BOUNDS = 4u;

// Device bounds checks of the KQ_DEBUG build.  KQ_DCHECK(cond, err) checks
// an index that comes from data (a grouping entry, a tile list, a shared-
// memory layout) before it is used: when cond is false it sets ERR_BOUNDS in
// the error word and yields false, and the caller skips or clamps the
// access instead of touching memory outside its buffer.  In the release
// build it is the constant true and cond is not evaluated.
#ifdef KQ_DEBUG
constexpr bool kDebug = true;
#else
constexpr bool kDebug = false;
#endif
__device__ __forceinline__ bool dcheck_record(bool ok, unsigned int *err) {
    if (!ok) atomicOr(err, ERR_BOUNDS);
    return ok;
}
#define KQ_DCHECK(cond, err) (!::kq::kDebug || ::kq::dcheck_record((cond), (err)))

// Bytes of dynamic shared memory this launch was given.
__device__ __forceinline__ uint32_t dynamic_smem_size() {
    uint32_t v;
    asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(v));
    return v;
}

// GLU activation (KQ_ACT_*, mlx-kquant `moe_glu_gather_kq`): SiLU
// g / (1 + e^-g), or the tanh form of GELU 0.5 g (1 + tanh(sqrt(2/pi) (g +
// 0.044715 g^3))).
__device__ __forceinline__ float glu_activation(float g, int act) {
    if (act == KQ_ACT_GELU_TANH)
        return 0.5f * g * (1.0f + tanhf(0.7978845608028654f * fmaf(0.044715f * g, g * g, g)));
    return g / (1.0f + expf(-g));
}

__device__ __forceinline__ float half_bits_to_float(uint32_t bits16) {
    return __half2float(__ushort_as_half((unsigned short)(bits16 & 0xFFFFu)));
}

// bf16 pair (packed in one 32-bit word) -> two fp32 values (exact).
__device__ __forceinline__ float bf16lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

template <typename T> struct XLoad;

__device__ __forceinline__ void store_out(float *p, float v) { *p = v; }
__device__ __forceinline__ void store_out(__nv_bfloat16 *p, float v) { *p = __float2bfloat16_rn(v); }
__device__ __forceinline__ void store_out(__half *p, float v) { *p = __float2half_rn(v); }

// Load 8 consecutive activations (16-byte aligned group) as fp32.
__device__ __forceinline__ void load_x8(const float *x, float v[8]) {
    float4 a = __ldg(reinterpret_cast<const float4 *>(x));
    float4 b = __ldg(reinterpret_cast<const float4 *>(x) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void load_x8(const __nv_bfloat16 *x, float v[8]) {
    uint4 a = __ldg(reinterpret_cast<const uint4 *>(x));
    v[0] = bf16lo(a.x); v[1] = bf16hi(a.x); v[2] = bf16lo(a.y); v[3] = bf16hi(a.y);
    v[4] = bf16lo(a.z); v[5] = bf16hi(a.z); v[6] = bf16lo(a.w); v[7] = bf16hi(a.w);
}

}  // namespace kq
