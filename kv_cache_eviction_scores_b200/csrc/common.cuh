// common.cuh -- small device helpers shared by the CUDA-core kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math_constants.h>
#include <stdint.h>

namespace dropkv {

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

// Programmatic dependent launch.  A kernel launched with the programmatic
// stream-serialization attribute may begin while its predecessor in the
// stream is still running: pdl_wait() returns once the predecessor grid has
// completed and its memory writes are visible (at once when there is no such
// predecessor).  pdl_trigger() lets the successor grid begin launching early;
// the successor still waits in its own pdl_wait() for this grid to finish.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Warp reductions over all 32 lanes.
__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_min(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fminf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Block reductions for blockDim.x == NT (a multiple of 32).  `red` needs
// NT/32 floats.  Every thread returns the result.  Contains __syncthreads.
template <int NT>
__device__ __forceinline__ float block_max(float x, float* red) {
  x = warp_max(x);
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0) red[wid] = x;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int i = 1; i < NT / 32; ++i) r = fmaxf(r, red[i]);
  return r;
}
template <int NT>
__device__ __forceinline__ float block_sum(float x, float* red) {
  x = warp_sum(x);
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0) red[wid] = x;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int i = 1; i < NT / 32; ++i) r += red[i];
  return r;
}

}  // namespace dropkv
