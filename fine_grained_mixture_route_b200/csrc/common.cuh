// Shared device helpers of the sm_100a MoE kernels: element conversion, the workspace error
// word, and the host-side launch context every kernel file uses.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

// Error bits recorded in the workspace error word (see moe_check_device_error).
constexpr uint32_t ERR_EXPERT_RANGE = 1u;
constexpr uint32_t ERR_PIPE_TIMEOUT = 2u;
constexpr uint32_t ERR_INDEX_RANGE = 4u;

__device__ __forceinline__ void flag_error(uint32_t* err, uint32_t bits) {
    if (err) atomicOr(err, bits);
}

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// silu(a) = a * sigmoid(a)
__device__ __forceinline__ float silu_f32(float a) { return a / (1.0f + expf(-a)); }

__host__ __device__ constexpr inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Block-scaled FP8 (MOE_FMT_MXFP8): the exponent e of a run of 32 values from the fp32 bits of
// its maximum magnitude amax >= 0: the smallest integer with amax <= 448 * 2^e, 0 for amax == 0,
// within [-127, 127].  amax in [2^e0, 2^(e0+1)) and 448 * 2^(e0-8) = 1.75 * 2^e0, so e = e0 - 8
// when the mantissa field is at most 0.75 (0x600000), else e0 - 7.
__device__ __forceinline__ int mx_exponent(float amax) {
    const uint32_t b = __float_as_uint(amax);
    if (b == 0u) return 0;
    const int eb = (int)(b >> 23);
    if (eb == 0) return -127;                              // below 2^-126: clamped
    const int e = eb - 127 - 8 + ((b & 0x7FFFFFu) > 0x600000u ? 1 : 0);
    return e < -127 ? -127 : (e > 127 ? 127 : e);
}

}  // namespace moe
