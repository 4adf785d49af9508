// The quantised latent cache: every token's row [c_KV | k_R] stored as FP8 E4M3 codes with one
// float32 scale per token (row value = code * scale), the per-token latent quantisation of
// 「Multi-Head Latent Attention（MLA）原理与工程实践全解析」.
//
// Page layout (page_size tokens, row = d_c + d_rope codes per token):
//   bytes [0, page_size*row)                    the codes, token after token
//   bytes [page_size*row, page_size*(row + 4))  the float32 scales, one per token
// so a page is page_size * (row + 4) bytes (37,120 at DeepSeek-V2 shape against 73,728 for a
// bf16 page), and one pool allocation holds both.
//
// Quantising a row v (float32 values): scale = max_i |v_i| / 448 (one correctly rounded
// division; 0 for a row of zeros), code_i = E4M3(v_i / scale) (one correctly rounded division,
// then the conversion instruction's round-to-nearest-even onto the E4M3 grid, saturating at
// ±448). A zero row keeps its zeros' signs and scale 0.
#pragma once

#include <cuda_fp8.h>

#include "common.cuh"
#include "ptx.cuh"

namespace mla {

constexpr float E4M3_MAX_F = 448.0f;

__host__ __device__ __forceinline__ int64_t fp8_page_bytes(int page_size, int row) {
  return static_cast<int64_t>(page_size) * (row + 4);
}

// Code row and scale slot of (sequence b, position p) in a quantised paged cache; false (and
// nothing resolved) when the sequence index, the position or the page id is out of range.
__device__ __forceinline__ bool fp8_cache_slot(uint8_t* cache, const int32_t* block_table, int b,
                                               int p, int batch, int max_pages, int num_pages,
                                               int page_size, int row, uint8_t** codes,
                                               float** scale) {
  if (b < 0 || b >= batch || p < 0 || p / page_size >= max_pages) return false;
  const int page = block_table[static_cast<int64_t>(b) * max_pages + p / page_size];
  if (page < 0 || page >= num_pages) return false;
  uint8_t* base = cache + static_cast<int64_t>(page) * fp8_page_bytes(page_size, row);
  const int slot = p % page_size;
  *codes = base + static_cast<int64_t>(slot) * row;
  *scale = reinterpret_cast<float*>(base + static_cast<int64_t>(page_size) * row) + slot;
  return true;
}

__device__ __forceinline__ float e4m3_row_scale(float amax) {
  return __fdiv_rn(amax, E4M3_MAX_F);
}
// Codes of two row values v0, v1 under `scale` (from e4m3_row_scale); v0 in the low byte.
__device__ __forceinline__ uint16_t e4m3_encode2(float v0, float v1, float scale) {
  if (scale > 0.0f) {
    v0 = __fdiv_rn(v0, scale);
    v1 = __fdiv_rn(v1, scale);
  }
  return static_cast<uint16_t>(
      __nv_cvt_float2_to_fp8x2(make_float2(v0, v1), __NV_SATFINITE, __NV_E4M3));
}
// Quantise n_tok float32 rows [n_tok][row] into their cache slots: one block per token (even
// row, blockDim a multiple of 32). Out-of-range tokens are skipped and flagged DEVICE_OOB.
__global__ void __launch_bounds__(256)
quantize_rows_kernel(const float* __restrict__ rows, int n_tok, int row,
                     const int32_t* __restrict__ seq_idx, const int32_t* __restrict__ pos,
                     const int32_t* __restrict__ block_table, int batch, int max_pages,
                     uint8_t* __restrict__ cache, int num_pages, int page_size) {
  __shared__ float red[32];
  const int i = blockIdx.x;
  if (i >= n_tok) return;
  const float* v = rows + static_cast<int64_t>(i) * row;
  float amax = 0.0f;
  for (int f = threadIdx.x; f < row; f += blockDim.x) amax = fmaxf(amax, fabsf(v[f]));
  amax = block_max(amax, red);
  uint8_t* codes = nullptr;
  float* scale_slot = nullptr;
  if (!fp8_cache_slot(cache, block_table, seq_idx[i], pos[i], batch, max_pages, num_pages,
                      page_size, row, &codes, &scale_slot)) {
    if (threadIdx.x == 0) record_error(MLA_ERR_DEVICE_OOB);
    return;
  }
  const float scale = e4m3_row_scale(amax);
  for (int f = 2 * threadIdx.x; f < row; f += 2 * blockDim.x)
    *reinterpret_cast<uint16_t*>(codes + f) = e4m3_encode2(v[f], v[f + 1], scale);
  if (threadIdx.x == 0) *scale_slot = scale;
}

// The tensor-core append's finish step for a quantised cache: as append_finish_cluster_kernel
// (RMSNorm on c_KV, RoPE on k_R, one cluster of FIN_CLUSTER CTAs per token, each a slice of the
// features), then the row maximum combined over the cluster through distributed shared memory
// (a maximum is exact in any order), the scale, and each CTA's codes; rank 0 writes the scale.
template <int CLUSTER>
__global__ void __launch_bounds__(128)
append_finish_cluster_fp8_kernel(const float* __restrict__ kv, int n_splits, int n_tok,
                                 const __nv_bfloat16* __restrict__ kv_gain,
                                 const int32_t* __restrict__ seq_idx,
                                 const int32_t* __restrict__ pos,
                                 const int32_t* __restrict__ block_table, int batch,
                                 int max_pages, uint8_t* __restrict__ cache, int num_pages,
                                 int page_size, int d_c, int d_r, float eps,
                                 const __grid_constant__ RopeFreqs rf) {
  __shared__ float red[32];
  __shared__ float ss_part, amax_part;
  extern __shared__ float slice_s[];   // this CTA's feature values
  const int i = blockIdx.x / CLUSTER;
  const uint32_t rank = cluster_ctarank();
  const int row = d_c + d_r;
  const int per = (((row + CLUSTER - 1) / CLUSTER) + 1) & ~1;   // even slice width
  const int f0 = static_cast<int>(rank) * per, f1 = min(row, f0 + per);
  const int b = seq_idx[i], p = pos[i];
  uint8_t* codes = nullptr;
  float* scale_slot = nullptr;
  const bool ok = fp8_cache_slot(cache, block_table, b, p, batch, max_pages, num_pages,
                                 page_size, row, &codes, &scale_slot);
  pdl_wait();   // the split-K partials of the GEMM just before are complete from here on
  const int64_t stride = static_cast<int64_t>(n_tok) * row;
  float ss = 0.0f;
  for (int f = f0 + threadIdx.x; f < f1; f += blockDim.x) {
    const float* src = kv + static_cast<int64_t>(i) * row + f;
    float v = 0.0f;
    for (int s0 = 0; s0 < n_splits; s0 += 16) {   // 16 partials in flight, summed in order
      float part[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) part[j] = (s0 + j < n_splits) ? src[(s0 + j) * stride] : 0.0f;
#pragma unroll
      for (int j = 0; j < 16; ++j) v += part[j];
    }
    slice_s[f - f0] = v;
    if (f < d_c) ss = fmaf(v, v, ss);
  }
  ss = block_sum(ss, red);   // also orders the slice_s writes before the reads below
  if (threadIdx.x == 0) ss_part = ss;
  cluster_sync_all();
  float total = 0.0f;
  for (uint32_t r = 0; r < CLUSTER; ++r)
    total += ld_shared_cluster_f32(map_to_rank(smem_addr(&ss_part), r));
  // the row's final values, in place: normalised c_KV, rotated k_R (pairs never straddle a
  // slice: d_c, f0 and per are even)
  const float rstd = 1.0f / sqrtf(total / static_cast<float>(d_c) + eps);
  for (int f = f0 + threadIdx.x; f < min(f1, d_c); f += blockDim.x)
    slice_s[f - f0] = slice_s[f - f0] * rstd * __bfloat162float(kv_gain[f]);
  const int r0 = max(f0, d_c);
  for (int f = r0 + 2 * static_cast<int>(threadIdx.x); f < f1; f += 2 * blockDim.x) {
    const int pr = (f - d_c) / 2;
    float ox, oy;
    rope_pair(slice_s[f - f0], slice_s[f + 1 - f0], rf.f_hi[pr], rf.f_lo[pr], p, &ox, &oy);
    slice_s[f - f0] = ox;
    slice_s[f + 1 - f0] = oy;
  }
  __syncthreads();
  float amax = 0.0f;
  for (int f = f0 + threadIdx.x; f < f1; f += blockDim.x) amax = fmaxf(amax, fabsf(slice_s[f - f0]));
  amax = block_max(amax, red);
  if (threadIdx.x == 0) amax_part = amax;
  cluster_sync_all();
  float row_max = 0.0f;
  for (uint32_t r = 0; r < CLUSTER; ++r)
    row_max = fmaxf(row_max, ld_shared_cluster_f32(map_to_rank(smem_addr(&amax_part), r)));
  cluster_sync_all();   // no CTA leaves while another may still read its ss_part / amax_part
  if (!ok) {
    if (threadIdx.x == 0 && rank == 0) record_error(MLA_ERR_DEVICE_OOB);
    return;
  }
  const float scale = e4m3_row_scale(row_max);
  for (int f = f0 + 2 * static_cast<int>(threadIdx.x); f < f1; f += 2 * blockDim.x)
    *reinterpret_cast<uint16_t*>(codes + f) = e4m3_encode2(slice_s[f - f0], slice_s[f + 1 - f0], scale);
  if (threadIdx.x == 0 && rank == 0) *scale_slot = scale;
}

}  // namespace mla
