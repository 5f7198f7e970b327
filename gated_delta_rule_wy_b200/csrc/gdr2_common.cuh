// gdr2_common.cuh -- device helpers shared by the GDR-2 kernels.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gdr2 {

// Lower bound applied to log_alpha on the device: exp(-64) = 1.6e-28 is a
// reset to fp32 precision, and a finite floor keeps differences of
// cumulative decays finite.
constexpr float kLogAlphaFloor = -64.0f;

// Gate layouts (the gates argument of the gated entry points): a set bit means the gate
// is one value per token-head ([..., T, H]) instead of a vector over its channels.
enum : int {
    kGateScalarB = 1,
    kGateScalarW = 2,
};

// Bits of the device status word (one per device, read by gdr2_sync_status).
enum : unsigned {
    kStatusTimeout = 1u,      // a kernel gave up a bounded wait
    kStatusBadSeqlens = 2u,   // cu_seqlens was not a nondecreasing run from 0 to T (no work done)
};

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

__device__ __forceinline__ float clamp_log_alpha(float la) { return fmaxf(la, kLogAlphaFloor); }

}  // namespace gdr2
