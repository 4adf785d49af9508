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

// Position of unit (b, mt) (sequence b, 128-row query tile mt) in the split-KV planner's unit
// stream, which lists every sequence's tile 0, then every sequence's tile 1, ... (B sequences).
__host__ __device__ __forceinline__ int unit_stream_pos(int b, int mt, int B) {
  return mt * B + b;
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

// Which cached keys a query may attend to. Query token t of a sequence of length L with Tq new
// tokens sits at position p = L - Tq + t and sees the keys j with lo <= j <= hi:
//   causal          j <= p (a query sees itself and earlier tokens),
//   sliding window  j > p - window when window > 0 (only the last `window` tokens are kept),
//   key range       kv_begin[b] <= j < kv_end[b] when given (the share of a sequence's keys that
//                   one GPU holds when a long context is split over several GPUs).
// lo > hi means the query sees no key here.
struct KeyRange {
  const int32_t* kv_begin;   // [B] or null (= 0)
  const int32_t* kv_end;     // [B] or null (= L)
  int window;                // 0 = unlimited
};

__device__ __forceinline__ void visible_keys(const KeyRange& kr, int b, int L, int Tq, int t,
                                             int* lo, int* hi) {
  const int p = L - Tq + t;
  int l = 0, h = p;
  if (kr.window > 0) l = max(l, p - kr.window + 1);
  if (kr.kv_begin != nullptr) l = max(l, kr.kv_begin[b]);
  if (kr.kv_end != nullptr) h = min(h, kr.kv_end[b] - 1);
  *lo = l;
  *hi = h;
}

constexpr int MLA_MAX_ROPE_PAIRS = 64;   // d_rope <= 128

// Per rotary pair i, f_i = theta^(-2i/d_rope) / pi split into two floats (f_hi + f_lo carries
// f_i to ~48 bits), formed on the host in double precision and passed to the kernels by value.
struct RopeFreqs {
  float f_hi[MLA_MAX_ROPE_PAIRS];
  float f_lo[MLA_MAX_ROPE_PAIRS];
};

// RoPE of one pair (x, y) = (v[2i], v[2i+1]) at position pos: turn by pos * theta^(-2i/d).
// In units of pi the angle is t = pos * f_i. pos is split into a = pos with its low 12 bits
// cleared and b = its low 12 bits (both exact in fp32); each product with f_hi is formed exactly
// as a rounded value plus its fma residual, the rounded parts are reduced modulo 2 (exact: they
// are within 1 of an even integer, or are even integers themselves), and sinpi/cospi take the
// small remainder. Everything stays in fp32 (fp64 is slow on the device), and for positions up
// to 2^30 the angle keeps an absolute error of about 1e-6 rad.
__device__ __forceinline__ void rope_sincos(float f_hi, float f_lo, int pos, float* s, float* c) {
  const float a = static_cast<float>(pos & ~0xFFF), b = static_cast<float>(pos & 0xFFF);
  const float p1 = a * f_hi, e1 = fmaf(a, f_hi, -p1);
  const float p2 = b * f_hi, e2 = fmaf(b, f_hi, -p2);
  const float r1 = p1 - 2.0f * rintf(0.5f * p1);
  const float r2 = p2 - 2.0f * rintf(0.5f * p2);
  const float t = (r1 + r2) + ((e1 + e2) + fmaf(a, f_lo, b * f_lo));
  sincospif(t, s, c);
}
// The turn itself, (x, y) -> (x cos - y sin, x sin + y cos), with explicit fused rounding so
// that every caller rounds alike.
__device__ __forceinline__ void rope_turn(float x, float y, float s, float c, float* ox, float* oy) {
  *ox = fmaf(x, c, -(y * s));
  *oy = fmaf(x, s, y * c);
}
__device__ __forceinline__ void rope_pair(float x, float y, float f_hi, float f_lo, int pos,
                                          float* ox, float* oy) {
  float s, c;
  rope_sincos(f_hi, f_lo, pos, &s, &c);
  rope_turn(x, y, s, c, ox, oy);
}

}  // namespace mla
