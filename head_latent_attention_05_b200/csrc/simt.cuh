// CUDA-core kernels (fp32 arithmetic, any shape, fp32 or bf16 storage).
//
// They implement the fp32 decode path (q absorption, attention, value projection) and the
// reference prefill path, plus the append step for shapes the tensor-core path does not take
// and the bit-exact weight split. Each block works on one row (a token, or one (token, head)
// query) and is written for clarity and coalesced loads rather than peak throughput.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace mla {

// --------------------------------------------------------------- a0: absorbed weight packs
// w_uk_t[h][c][n] = wkv_b[h*(dn+dv)+n][c];  w_uv[h][v][c] = wkv_b[h*(dn+dv)+dn+v][c].
template <typename T>
__global__ void absorb_kernel(const T* __restrict__ wkv_b, T* __restrict__ w_uk_t,
                              T* __restrict__ w_uv, int H, int d_c, int d_nope, int d_v) {
  const int64_t per_head = static_cast<int64_t>(d_nope + d_v) * d_c;
  const int64_t total = per_head * H;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int h = static_cast<int>(i / per_head);
    const int64_t rem = i - h * per_head;
    if (rem < static_cast<int64_t>(d_c) * d_nope) {
      // output index inside w_uk_t[h]: (c, n), n fastest
      const int c = static_cast<int>(rem / d_nope), n = static_cast<int>(rem % d_nope);
      w_uk_t[static_cast<int64_t>(h) * d_c * d_nope + rem] =
          wkv_b[(static_cast<int64_t>(h) * (d_nope + d_v) + n) * d_c + c];
    } else {
      const int64_t r2 = rem - static_cast<int64_t>(d_c) * d_nope;  // (v, c), c fastest
      const int v = static_cast<int>(r2 / d_c), c = static_cast<int>(r2 % d_c);
      w_uv[static_cast<int64_t>(h) * d_v * d_c + r2] =
          wkv_b[(static_cast<int64_t>(h) * (d_nope + d_v) + d_nope + v) * d_c + c];
    }
  }
}

// ------------------------------------------------------------------------ a1: append (SIMT)
// kv[n][f] = sum_k x[n][k] * w[f][k] in fp32. One warp per output feature, 8 warps per block.
template <typename T>
__global__ void __launch_bounds__(256)
linear_rows_kernel(const T* __restrict__ x, const T* __restrict__ w, float* __restrict__ out,
                   int n_tok, int F, int K) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int f = blockIdx.x * 8 + warp;
  const int n = blockIdx.y;
  if (f >= F || n >= n_tok) return;
  const T* xr = x + static_cast<int64_t>(n) * K;
  const T* wr = w + static_cast<int64_t>(f) * K;
  float acc = 0.0f;
  for (int k = lane; k < K; k += 32) acc = fmaf(Elem<T>::to_f(xr[k]), Elem<T>::to_f(wr[k]), acc);
  acc = warp_sum(acc);
  if (lane == 0) out[static_cast<int64_t>(n) * F + f] = acc;
}

// Resolve the cache row of (sequence b, position p). Returns nullptr (and records the error)
// when the sequence index, the position or the page id is out of range.
template <typename T>
__device__ __forceinline__ T* cache_row(T* cache, const int32_t* block_table, int b, int p,
                                        int batch, int max_pages, int num_pages,
                                        int page_size, int row) {
  if (b < 0 || b >= batch || p < 0 || p / page_size >= max_pages) return nullptr;
  const int page = block_table[static_cast<int64_t>(b) * max_pages + p / page_size];
  if (page < 0 || page >= num_pages) return nullptr;
  return cache + (static_cast<int64_t>(page) * page_size + p % page_size) * row;
}

// Per token: RMSNorm over c_KV, RoPE on k_R at the token's position, one rounding to the
// cache type, scatter to its page slot. kv holds n_splits partial sums [n_splits][n_tok][row],
// added in a fixed order. One thread per feature (blockDim >= row), so the partial sums of a
// row are read in parallel.
template <typename T>
__global__ void __launch_bounds__(1024)
append_finish_kernel(const float* __restrict__ kv, int n_splits, int n_tok,
                     const T* __restrict__ kv_gain, const int32_t* __restrict__ seq_idx,
                     const int32_t* __restrict__ pos, const int32_t* __restrict__ block_table,
                     int batch, int max_pages, T* __restrict__ cache, int num_pages,
                     int page_size, int d_c, int d_r, float eps,
                     const __grid_constant__ RopeFreqs rf) {
  __shared__ float red[32];
  extern __shared__ float row_s[];  // [d_c + d_r]
  pdl_wait();   // the split-K partials of the GEMM just before are complete from here on
  const int i = blockIdx.x;
  const int row = d_c + d_r;
  const int b = seq_idx[i], p = pos[i];
  T* dst = cache_row(cache, block_table, b, p, batch, max_pages, num_pages, page_size, row);
  if (dst == nullptr) {
    if (threadIdx.x == 0) record_error(MLA_ERR_DEVICE_OOB);
    return;
  }
  float ss = 0.0f;
  for (int f = threadIdx.x; f < row; f += blockDim.x) {
    const float* src = kv + static_cast<int64_t>(i) * row + f;
    const int64_t stride = static_cast<int64_t>(n_tok) * row;
    float v = 0.0f;
    // 16 partials in flight per round, summed in split order
    for (int s0 = 0; s0 < n_splits; s0 += 16) {
      float part[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) part[j] = (s0 + j < n_splits) ? src[(s0 + j) * stride] : 0.0f;
#pragma unroll
      for (int j = 0; j < 16; ++j) v += part[j];
    }
    row_s[f] = v;
    if (f < d_c) ss = fmaf(v, v, ss);
  }
  ss = block_sum(ss, red);  // also orders the row_s writes before the reads below
  const float rstd = 1.0f / sqrtf(ss / static_cast<float>(d_c) + eps);
  for (int f = threadIdx.x; f < d_c; f += blockDim.x)
    dst[f] = Elem<T>::from_f(row_s[f] * rstd * Elem<T>::to_f(kv_gain[f]));
  for (int pr = threadIdx.x; pr < d_r / 2; pr += blockDim.x) {
    float ox, oy;
    rope_pair(row_s[d_c + 2 * pr], row_s[d_c + 2 * pr + 1], rf.f_hi[pr], rf.f_lo[pr], p, &ox, &oy);
    dst[d_c + 2 * pr] = Elem<T>::from_f(ox);
    dst[d_c + 2 * pr + 1] = Elem<T>::from_f(oy);
  }
}

// Cluster form of the same step, for the tensor-core append: the FIN_CLUSTER CTAs of a cluster
// share one token (grid.x = FIN_CLUSTER * n_tok), each owning a contiguous, even-sized slice of
// the row's features, so that the split-K partials are read by that many SMs at once (one SM
// alone is limited by its outstanding misses, not by bandwidth). The RMSNorm's sum of squares
// is combined over the cluster through distributed shared memory, in rank order, so the result
// does not depend on timing. Every thread reaches both cluster barriers, whatever happens.
constexpr int FIN_CLUSTER = 8;
constexpr int FIN_THREADS = 128;

template <typename T>
__global__ void __launch_bounds__(FIN_THREADS)
append_finish_cluster_kernel(const float* __restrict__ kv, int n_splits, int n_tok,
                             const T* __restrict__ kv_gain, const int32_t* __restrict__ seq_idx,
                             const int32_t* __restrict__ pos,
                             const int32_t* __restrict__ block_table, int batch, int max_pages,
                             T* __restrict__ cache, int num_pages, int page_size, int d_c,
                             int d_r, float eps, const __grid_constant__ RopeFreqs rf) {
  __shared__ float red[32];
  __shared__ float ss_part;
  extern __shared__ float slice_s[];   // this CTA's feature values
  const int i = blockIdx.x / FIN_CLUSTER;
  const uint32_t rank = cluster_ctarank();
  const int row = d_c + d_r;
  const int per = (((row + FIN_CLUSTER - 1) / FIN_CLUSTER) + 1) & ~1;   // even slice width
  const int f0 = static_cast<int>(rank) * per, f1 = min(row, f0 + per);
  // the destination comes from inputs of the call (complete before its first kernel ran):
  // look it up while the GEMM still runs
  const int b = seq_idx[i], p = pos[i];
  T* dst = cache_row(cache, block_table, b, p, batch, max_pages, num_pages, page_size, row);
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
  for (uint32_t r = 0; r < FIN_CLUSTER; ++r)
    total += ld_shared_cluster_f32(map_to_rank(smem_addr(&ss_part), r));
  cluster_sync_all();   // no CTA leaves while another may still read its ss_part
  if (dst == nullptr) {
    if (threadIdx.x == 0 && rank == 0) record_error(MLA_ERR_DEVICE_OOB);
    return;
  }
  const float rstd = 1.0f / sqrtf(total / static_cast<float>(d_c) + eps);
  for (int f = f0 + threadIdx.x; f < min(f1, d_c); f += blockDim.x)
    dst[f] = Elem<T>::from_f(slice_s[f - f0] * rstd * Elem<T>::to_f(kv_gain[f]));
  // rotary pairs (d_c + 2q, d_c + 2q + 1) never straddle a slice: d_c, f0 and per are even
  const int r0 = max(f0, d_c);
  for (int f = r0 + 2 * static_cast<int>(threadIdx.x); f < f1; f += 2 * blockDim.x) {
    const int pr = (f - d_c) / 2;
    float ox, oy;
    rope_pair(slice_s[f - f0], slice_s[f + 1 - f0], rf.f_hi[pr], rf.f_lo[pr], p, &ox, &oy);
    dst[f] = Elem<T>::from_f(ox);
    dst[f + 1] = Elem<T>::from_f(oy);
  }
}

// ------------------------------------------------------- q path and output projection
// The q path's normalisation (the module's q_norm after wq_a): per token n,
//   out[n][f] = v[f] / sqrt(mean(v^2) + eps) * gain[f],  v[f] = sum_s partial[s][n][f]
// with the split-K partials added in split order. One block per token.
template <typename T>
__global__ void __launch_bounds__(256)
rms_rows_kernel(const float* __restrict__ partial, int n_splits, int n_tok, int F,
                const T* __restrict__ gain, float eps, T* __restrict__ out) {
  __shared__ float red[32];
  extern __shared__ float row_s[];   // [F]
  pdl_wait();   // the partials of the GEMM just before are complete from here on
  const int n = blockIdx.x;
  const int64_t stride = static_cast<int64_t>(n_tok) * F;
  float ss = 0.0f;
  for (int f = threadIdx.x; f < F; f += blockDim.x) {
    const float* src = partial + static_cast<int64_t>(n) * F + f;
    float v = 0.0f;
    for (int s = 0; s < n_splits; ++s) v += src[s * stride];
    row_s[f] = v;
    ss = fmaf(v, v, ss);
  }
  ss = block_sum(ss, red);   // also orders the row_s writes before the reads below
  const float rstd = 1.0f / sqrtf(ss / static_cast<float>(F) + eps);
  for (int f = threadIdx.x; f < F; f += blockDim.x)
    out[static_cast<int64_t>(n) * F + f] = Elem<T>::from_f(row_s[f] * rstd * Elem<T>::to_f(gain[f]));
}

// out[i] = sum_s partial[s][i] in split order, rounded to T (the output projection's split-K
// sum). Grid-stride over the n_tok * F outputs.
template <typename T>
__global__ void __launch_bounds__(256)
sum_splits_kernel(const float* __restrict__ partial, int n_splits, int64_t count,
                  T* __restrict__ out) {
  pdl_wait();
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < count;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float v = 0.0f;
    for (int s = 0; s < n_splits; ++s) v += partial[s * count + i];
    out[i] = Elem<T>::from_f(v);
  }
}

// Rows of fp32 values rounded to T (the SIMT q path's up-projection output).
template <typename T>
__global__ void __launch_bounds__(256)
round_rows_kernel(const float* __restrict__ in, int64_t count, T* __restrict__ out) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < count;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    out[i] = Elem<T>::from_f(in[i]);
}

// ---------------------------------------------------- decode on CUDA cores (fp32 arithmetic)
// Query rows are r = (b*Tq + t)*H + h. The length of sequence b must lie in [Tq, max_pos].
__device__ __forceinline__ bool length_ok(int L, int Tq, int max_pos) {
  return L >= Tq && L <= max_pos;
}

// qhat[r] = [ q_nope·W_UK[h] (d_c) | RoPE(q_rope, L_b - Tq + t) (d_r) ] in fp32.
template <typename T>
__global__ void __launch_bounds__(256)
qabs_simt_kernel(const T* __restrict__ q, const T* __restrict__ w_uk_t,
                 const int32_t* __restrict__ seq_lens, float* __restrict__ qhat, int H, int Tq,
                 int d_c, int d_r, int d_nope, int max_pos,
                 const __grid_constant__ RopeFreqs rf) {
  extern __shared__ float qs[];  // [d_nope + d_r]
  const int r = blockIdx.x;
  const int h = r % H, t = (r / H) % Tq, b = r / (H * Tq);
  const int L = seq_lens[b];
  const bool ok = length_ok(L, Tq, max_pos);
  const T* qr = q + static_cast<int64_t>(r) * (d_nope + d_r);
  float* out = qhat + static_cast<int64_t>(r) * (d_c + d_r);
  for (int i = threadIdx.x; i < d_nope + d_r; i += blockDim.x) qs[i] = Elem<T>::to_f(qr[i]);
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const T* wh = w_uk_t + static_cast<int64_t>(h) * d_c * d_nope;
  for (int c = warp; c < d_c; c += nw) {
    float acc = 0.0f;
    for (int n = lane; n < d_nope; n += 32)
      acc = fmaf(qs[n], Elem<T>::to_f(wh[static_cast<int64_t>(c) * d_nope + n]), acc);
    acc = warp_sum(acc);
    if (lane == 0) out[c] = ok ? acc : 0.0f;
  }
  const int p = L - Tq + t;
  for (int pr = threadIdx.x; pr < d_r / 2; pr += blockDim.x) {
    float ox = 0.0f, oy = 0.0f;
    if (ok) rope_pair(qs[d_nope + 2 * pr], qs[d_nope + 2 * pr + 1], rf.f_hi[pr], rf.f_lo[pr], p, &ox, &oy);
    out[d_c + 2 * pr] = ox;
    out[d_c + 2 * pr + 1] = oy;
  }
}

// One block per query row: online softmax over chunks of 256 keys.
//   s_j = scale * qhat · cache_row_j  (all d_c + d_r dims),  j in the row's visible_keys range
//   o_lat = sum_j softmax(s)_j * cache_row_j[:d_c]
// lse_out (optional): natural-log log-sum-exp of the row's scores, -inf if it sees no key.
template <typename T>
__global__ void __launch_bounds__(256)
attn_simt_kernel(const float* __restrict__ qhat, const T* __restrict__ cache,
                 const int32_t* __restrict__ block_table, const int32_t* __restrict__ seq_lens,
                 float* __restrict__ o_lat, int H, int Tq, int d_c, int d_r, int max_pages,
                 int num_pages, int page_size, float scale, KeyRange keys,
                 float* __restrict__ lse_out) {
  constexpr int CH = 256;
  __shared__ float red[32];
  __shared__ float p_s[CH];
  __shared__ const T* rows_s[CH];
  extern __shared__ float dyn[];  // qs [d_c + d_r] | acc [d_c]
  const int row = d_c + d_r;
  float* qs = dyn;
  float* acc = dyn + row;
  const int r = blockIdx.x;
  const int t = (r / H) % Tq, b = r / (H * Tq);
  const int L = seq_lens[b];
  float* out = o_lat + static_cast<int64_t>(r) * d_c;
  if (!length_ok(L, Tq, max_pages * page_size)) {
    for (int c = threadIdx.x; c < d_c; c += blockDim.x) out[c] = 0.0f;
    if (threadIdx.x == 0 && lse_out != nullptr) lse_out[r] = -INFINITY;
    if (threadIdx.x == 0 && (r % H) == 0 && t == 0) record_error(MLA_ERR_DEVICE_BAD_LENGTH);
    return;
  }
  int k_lo, k_hi;
  visible_keys(keys, b, L, Tq, t, &k_lo, &k_hi);
  for (int i = threadIdx.x; i < row; i += blockDim.x) qs[i] = qhat[static_cast<int64_t>(r) * row + i];
  for (int c = threadIdx.x; c < d_c; c += blockDim.x) acc[c] = 0.0f;
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  float m = -INFINITY, l = 0.0f;
  bool oob = false;
  for (int j0 = k_lo; j0 <= k_hi; j0 += CH) {
    const int cnt = min(CH, k_hi - j0 + 1);
    for (int jj = threadIdx.x; jj < cnt; jj += blockDim.x) {
      const int j = j0 + jj;
      const int page = block_table[static_cast<int64_t>(b) * max_pages + j / page_size];
      const bool bad = page < 0 || page >= num_pages;
      oob |= bad;
      rows_s[jj] = bad ? nullptr : cache + (static_cast<int64_t>(page) * page_size + j % page_size) * row;
    }
    __syncthreads();
    for (int jj = warp; jj < cnt; jj += nw) {
      const T* cr = rows_s[jj];
      float s = 0.0f;
      if (cr != nullptr)
        for (int i = lane; i < row; i += 32) s = fmaf(qs[i], Elem<T>::to_f(cr[i]), s);
      s = warp_sum(s);
      if (lane == 0) p_s[jj] = (cr != nullptr) ? s * scale : -INFINITY;
    }
    __syncthreads();
    float cm = -INFINITY;
    for (int jj = threadIdx.x; jj < cnt; jj += blockDim.x) cm = fmaxf(cm, p_s[jj]);
    cm = block_max(cm, red);
    const float m_new = fmaxf(m, cm);
    const float base = (m_new == -INFINITY) ? 0.0f : m_new;
    const float factor = (m == -INFINITY) ? 0.0f : expf(m - base);
    float ps = 0.0f;
    for (int jj = threadIdx.x; jj < cnt; jj += blockDim.x) {
      const float e = expf(p_s[jj] - base);
      p_s[jj] = e;
      ps += e;
    }
    ps = block_sum(ps, red);  // also publishes p_s
    l = l * factor + ps;
    m = m_new;
    for (int c = threadIdx.x; c < d_c; c += blockDim.x) {
      float a = acc[c] * factor;
      for (int jj = 0; jj < cnt; ++jj) {
        const T* cr = rows_s[jj];
        if (cr != nullptr) a = fmaf(p_s[jj], Elem<T>::to_f(cr[c]), a);
      }
      acc[c] = a;
    }
    __syncthreads();
  }
  if (oob) record_error(MLA_ERR_DEVICE_OOB);
  const float inv = (l > 0.0f) ? 1.0f / l : 0.0f;
  for (int c = threadIdx.x; c < d_c; c += blockDim.x) out[c] = acc[c] * inv;
  if (threadIdx.x == 0 && lse_out != nullptr) lse_out[r] = (l > 0.0f) ? m + logf(l) : -INFINITY;
}

// Merge of n_parts partial decodes over disjoint key ranges (rows r, natural-log lse):
//   o_lat[r][:] = sum_k e^(lse_k - m) O_k[r][:] / sum_k e^(lse_k - m), in part order.
// One block per row; zeros when no part saw a key.
template <typename T>
__global__ void __launch_bounds__(256)
combine_simt_kernel(const T* __restrict__ o_parts, const float* __restrict__ lse_parts,
                    int n_parts, int rows, int d_c, float* __restrict__ o_lat) {
  const int r = blockIdx.x;
  float m = -INFINITY;
  for (int k = 0; k < n_parts; ++k) m = fmaxf(m, lse_parts[static_cast<int64_t>(k) * rows + r]);
  float den = 0.0f;
  if (m > -INFINITY)
    for (int k = 0; k < n_parts; ++k) den += expf(lse_parts[static_cast<int64_t>(k) * rows + r] - m);
  const float inv = den > 0.0f ? 1.0f / den : 0.0f;
  for (int c = threadIdx.x; c < d_c; c += blockDim.x) {
    float a = 0.0f;
    if (m > -INFINITY)
      for (int k = 0; k < n_parts; ++k) {
        const int64_t i = static_cast<int64_t>(k) * rows + r;
        a = fmaf(expf(lse_parts[i] - m), Elem<T>::to_f(o_parts[i * d_c + c]), a);
      }
    o_lat[static_cast<int64_t>(r) * d_c + c] = a * inv;
  }
}

// out[r][v] = sum_c o_lat[r][c] * w_uv[h][v][c]. One warp per output column v.
template <typename T>
__global__ void __launch_bounds__(256)
outproj_simt_kernel(const float* __restrict__ o_lat, const T* __restrict__ w_uv,
                    T* __restrict__ out, int H, int d_c, int d_v) {
  extern __shared__ float os[];  // [d_c]
  const int r = blockIdx.x, h = r % H;
  for (int c = threadIdx.x; c < d_c; c += blockDim.x) os[c] = o_lat[static_cast<int64_t>(r) * d_c + c];
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const T* wh = w_uv + static_cast<int64_t>(h) * d_v * d_c;
  for (int v = warp; v < d_v; v += nw) {
    float a = 0.0f;
    for (int c = lane; c < d_c; c += 32) a = fmaf(os[c], Elem<T>::to_f(wh[static_cast<int64_t>(v) * d_c + c]), a);
    a = warp_sum(a);
    if (lane == 0) out[static_cast<int64_t>(r) * d_v + v] = Elem<T>::from_f(a);
  }
}

}  // namespace mla
