// Shared device helpers of the CUDA path (type conversion, gate functions,
// warp scans).  Nothing here is shared with the CPU oracle.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace mlstm {

typedef __nv_bfloat16 bf16;

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(bf16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ bf16 from_f32<bf16>(float x) { return __float2bfloat16_rn(x); }

// Chunk states on the bf16 path are kept as two bf16 planes, hi = bf16(C) and
// lo = bf16(C - hi), so hi + lo carries about 16 mantissa bits: the tensor-core
// forward reads hi alone, the backward reads both.  The fp32 path keeps one
// fp32 plane.  `plane` is the element count of one plane.
template <typename TS> struct StatePlanes;
template <> struct StatePlanes<float> {
  static __device__ __forceinline__ void store(float* base, size_t, size_t i, float x, bool) {
    base[i] = x;
  }
  static __device__ __forceinline__ float load(const float* base, size_t, size_t i, bool = true) {
    return base[i];
  }
};
template <> struct StatePlanes<bf16> {
  static __device__ __forceinline__ void store(bf16* base, size_t plane, size_t i, float x, bool lo) {
    const bf16 hi = __float2bfloat16_rn(x);
    base[i] = hi;
    if (lo) base[plane + i] = __float2bfloat16_rn(x - __bfloat162float(hi));
  }
  static __device__ __forceinline__ float load(const bf16* base, size_t plane, size_t i, bool lo = true) {
    return __bfloat162float(base[i]) + (lo ? __bfloat162float(base[plane + i]) : 0.f);
  }
};

// log sigmoid(x) = min(x, 0) - log(1 + exp(-|x|)); no overflow for any x.
__device__ __forceinline__ float log_sigmoid(float x) {
  return fminf(x, 0.f) - log1pf(expf(-fabsf(x)));
}

// sigmoid(-x) = exp(logsigmoid(-x)), the derivative of logsigmoid at x.
__device__ __forceinline__ float dlog_sigmoid(float x) { return expf(log_sigmoid(-x)); }

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ double warp_sum(double x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

// Inclusive prefix sum across the lanes of a warp.
__device__ __forceinline__ float warp_incl_sum(float x) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    float y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  return x;
}

// Inclusive prefix sum across the lanes of a warp, in fp64.
__device__ __forceinline__ double warp_incl_sum(double x) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    double y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  return x;
}

// Inclusive prefix max across the lanes of a warp.
__device__ __forceinline__ float warp_incl_max(float x) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    float y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x = fmaxf(x, y);
  }
  return x;
}

// Inclusive suffix sum across the lanes of a warp (lane i gets sum of lanes >= i).
__device__ __forceinline__ float warp_incl_suffix_sum(float x) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    float y = __shfl_down_sync(0xffffffffu, x, o);
    if (lane + o < 32) x += y;
  }
  return x;
}

}  // namespace mlstm
