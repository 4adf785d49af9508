// Shared device utilities: the device error word, element-type traits and small reductions.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "../../include/mla.h"

namespace mla {

// The one piece of state the library keeps: the first error a kernel saw since the host last
// read it (mla_get_device_error). 0 = none.
__device__ int g_device_error = 0;

__device__ __forceinline__ void record_error(int code) {
  atomicCAS(&g_device_error, 0, code);
}

// ------------------------------------------------------------------------- element traits

template <typename T> struct Elem;
template <> struct Elem<float> {
  __device__ __forceinline__ static float load(const float* p) { return *p; }
  __device__ __forceinline__ static float to_f(float v) { return v; }
  __device__ __forceinline__ static float from_f(float v) { return v; }
};
template <> struct Elem<__nv_bfloat16> {
  __device__ __forceinline__ static float load(const __nv_bfloat16* p) {
    return __bfloat162float(*p);
  }
  __device__ __forceinline__ static float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
  __device__ __forceinline__ static __nv_bfloat16 from_f(float v) {
    return __float2bfloat16_rn(v);
  }
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Sum over the whole block (blockDim.x a multiple of 32, <= 1024). `red` holds >= 32 floats.
__device__ __forceinline__ float block_sum(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  const int nw = (blockDim.x + 31) >> 5;
  float t = (threadIdx.x < nw) ? red[threadIdx.x] : 0.0f;
  if (warp == 0) t = warp_sum(t);
  if (threadIdx.x == 0) red[0] = t;
  __syncthreads();
  const float r = red[0];
  __syncthreads();
  return r;
}

__device__ __forceinline__ float block_max(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_max(v);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  const int nw = (blockDim.x + 31) >> 5;
  float t = (threadIdx.x < nw) ? red[threadIdx.x] : -INFINITY;
  if (warp == 0) t = warp_max(t);
  if (threadIdx.x == 0) red[0] = t;
  __syncthreads();
  const float r = red[0];
  __syncthreads();
  return r;
}

// RoPE of one pair (x, y) = (v[2i], v[2i+1]) at position pos: turn by pos * theta^(-2i/d).
// The angle is formed in double precision and reduced to [-pi, pi] there, so that positions
// up to 2^17 keep full fp32 accuracy; the rotation itself is done in fp32.
__device__ __forceinline__ void rope_pair(float x, float y, int pair, int d, int pos,
                                          float theta, float* ox, float* oy) {
  const double two_pi = 6.283185307179586476925286766559;
  const double inv_freq = exp2(-(2.0 * pair / static_cast<double>(d)) * log2(static_cast<double>(theta)));
  const double ang = static_cast<double>(pos) * inv_freq;
  const float r = static_cast<float>(ang - two_pi * rint(ang / two_pi));
  float s, c;
  sincosf(r, &s, &c);
  *ox = x * c - y * s;
  *oy = x * s + y * c;
}

}  // namespace mla
