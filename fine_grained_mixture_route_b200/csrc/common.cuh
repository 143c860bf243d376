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

}  // namespace moe
