// Split-KV merge fused with the value up-projection (bf16, tcgen05):
//   o_lat[n][h][:] = sum_s 2^(lse_s - m) * O_s / sum_s 2^(lse_s - m)      (over the segments s
//                                                                       of the row's unit)
//   out[n][h][m]   = sum_c W_UV[h][m][c] * o_lat[n][h][c]                 (m < d_v, c < 512)
// One CTA per (128-row m-tile of d_v, BN tokens, head h). The W_UV[h] tile is the A operand
// (all 8 K-chunks of 64, 128 KB, loaded by TMA at once: the kernel is HBM-bound on W_UV and
// these loads are issued before the kernel waits for the attention kernel, so they overlap its
// tail). The merged latent rows never go to global memory: the 8 warps merge them straight into
// the K-major, 128-byte-swizzled B operand in shared memory, then warp 1 issues the MMAs.
#pragma once

#include "common.cuh"
#include "ptx.cuh"
#include "tc_decode.cuh"

namespace mla {

// Two sources of partials. Segment mode (n_parts == 0): the attention kernel's per-segment O / l
// [segments][128][512] with base-2 lse [segments][128], a row's segments listed by unit_seg.
// Parts mode (n_parts > 0): n_parts full sets of rows [n_parts][n_q * H][512] with natural-log
// lse [n_parts][n_q * H] (the partial decodes of several GPUs over disjoint key ranges,
// gathered), merged in part order.
struct VprojParams {
  const __nv_bfloat16* o_part;  // partial O / l (bf16), see above
  const float* lse;             // their log-sum-exp, see above
  const int32_t* unit_seg;      // [U + 1] first segment of each unit by stream position
                                //   (unit_stream_pos; segment mode)
  __nv_bfloat16* out;           // [n_q][H][d_v]
  int H, Tq, n_mt, n_q, d_v;
  int n_parts;                  // 0: segment mode
};

constexpr int VP_THREADS = 256;
constexpr int VP_KCHUNKS = ATT_DC / 64;              // 8
constexpr int VP_A_CHUNK = 128 * 64 * 2;             // 16 KB

template <int BN>
__host__ __device__ constexpr int vproj_smem_bytes() {
  return VP_KCHUNKS * VP_A_CHUNK + VP_KCHUNKS * BN * 128 + 1024;
}

template <int BN>
__global__ void __launch_bounds__(VP_THREADS, 1)
vproj_merge_kernel(const __grid_constant__ CUtensorMap map_wuv, VprojParams p) {
  constexpr uint32_t IDESC = idesc_bf16(128, BN, false, false);
  constexpr uint32_t TMEM_COLS = BN < 32 ? 32 : BN;
  constexpr int B_CHUNK = BN * 128;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* a_buf = smem;                                   // chunk c at c * 16 KB
  uint8_t* b_buf = smem + VP_KCHUNKS * VP_A_CHUNK;         // chunk c at c * BN * 128
  __shared__ uint64_t full_bar[VP_KCHUNKS], done_bar;
  __shared__ uint32_t tmem_base_s;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * 128;
  const int n0 = blockIdx.y * BN;
  const int h = blockIdx.z;

  if (threadIdx.x == 0) {
    for (int c = 0; c < VP_KCHUNKS; ++c) mbar_init(&full_bar[c], 1);
    mbar_init(&done_bar, 1);
    fence_mbar_init();
    tma_prefetch_desc(&map_wuv);
    // W_UV is an input of the call, complete before its first kernel ran: load it now
    for (int c = 0; c < VP_KCHUNKS; ++c) {
      mbar_arrive_expect_tx(&full_bar[c], VP_A_CHUNK);
      tma_load_3d(a_buf + c * VP_A_CHUNK, &map_wuv, &full_bar[c], c * 64, m0, h);
    }
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_s, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = tmem_base_s;
  // ---- merge. 16 threads per B row, 16 rows per pass; thread k of a row owns the 16-byte
  // groups q = k + 16 i (i = 0..3) of the row's 512 bf16 dims, i.e. 16-byte piece k%8 of
  // K-chunk 2i + k/8.
  constexpr int RP = 16, TPR = VP_THREADS / RP, PASSES = BN / RP;
  const int rr_l = threadIdx.x / TPR, k = threadIdx.x % TPR;
  // each row's partials: cnt of them, the first at row base of the partial arrays, then every
  // `stride` rows. The segment lists were written two kernels back (by the planner): read them
  // before waiting.
  const int64_t stride = p.n_parts > 0 ? static_cast<int64_t>(p.n_q) * p.H : 128;
  const float lse_scale = p.n_parts > 0 ? 1.4426950408889634f : 1.0f;   // to base 2
  int64_t base[PASSES];
  int cnt[PASSES];
#pragma unroll
  for (int ps = 0; ps < PASSES; ++ps) {
    const int n = n0 + ps * RP + rr_l;
    base[ps] = 0;
    cnt[ps] = 0;
    if (n < p.n_q) {
      if (p.n_parts > 0) {
        base[ps] = static_cast<int64_t>(n) * p.H + h;
        cnt[ps] = p.n_parts;
      } else {
        const int b = n / p.Tq, t = n % p.Tq;
        const int r = t * p.H + h;
        const int u = unit_stream_pos(b, r / 128, p.n_q / p.Tq);
        const int s0 = p.unit_seg[u];
        base[ps] = static_cast<int64_t>(s0) * 128 + r % 128;
        cnt[ps] = p.unit_seg[u + 1] - s0;
      }
    }
  }
  pdl_wait();   // the attention partials are complete and visible from here on
  pdl_trigger();
  // thread k of a row holds the lse of the row's segment k (rows rarely have more than TPR
  // segments; later ones are read where needed), every pass's load in flight at once; the
  // other threads of the row take it by shuffle, so each pass waits for one round of partial
  // loads only
  float lse_k[PASSES];
#pragma unroll
  for (int ps = 0; ps < PASSES; ++ps)
    lse_k[ps] = k < cnt[ps] ? p.lse[base[ps] + k * stride] * lse_scale : -INFINITY;
#pragma unroll
  for (int ps = 0; ps < PASSES; ++ps) {
    const int rr = ps * RP + rr_l;
    const int s1 = cnt[ps];
    const int64_t rb = base[ps];
    auto lse_of = [&](int s) { return p.lse[rb + s * stride] * lse_scale; };
    float mx = lse_k[ps];
    for (int s = k + TPR; s < s1; s += TPR) mx = fmaxf(mx, lse_of(s));
#pragma unroll
    for (int o = TPR / 2; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const bool any = mx > -INFINITY;
    float den = 0.0f;
    float acc[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) acc[e] = 0.0f;
    if (any) {
      if (k < s1) den = exp2f(lse_k[ps] - mx);
      for (int s = k + TPR; s < s1; s += TPR) den += exp2f(lse_of(s) - mx);
    }
    // four partials' loads in flight at a time; the sum runs in partial order. The trip count
    // is the larger of the warp's two rows (the shuffles need every lane).
    const int s1w = __reduce_max_sync(0xffffffffu, s1);
    for (int sb = 0; sb < s1w; sb += 4) {
      float w[4];
      uint4 v[4][4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int s = sb + j;
        float ls = __shfl_sync(0xffffffffu, lse_k[ps], s & (TPR - 1), TPR);
        w[j] = 0.0f;
        if (any && s < s1) {
          if (s >= TPR) ls = lse_of(s);
          w[j] = exp2f(ls - mx);
          const uint4* src = reinterpret_cast<const uint4*>(p.o_part + (rb + s * stride) * ATT_DC);
#pragma unroll
          for (int i = 0; i < 4; ++i) v[j][i] = src[k + TPR * i];
        }
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (!any || sb + j >= s1) break;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t u[4] = {v[j][i].x, v[j][i].y, v[j][i].z, v[j][i].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u[e]));
            acc[8 * i + 2 * e] = fmaf(w[j], f.x, acc[8 * i + 2 * e]);
            acc[8 * i + 2 * e + 1] = fmaf(w[j], f.y, acc[8 * i + 2 * e + 1]);
          }
        }
      }
    }
#pragma unroll
    for (int o = TPR / 2; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    const float inv = den > 0.0f ? 1.0f / den : 0.0f;
    // group q = k + 16 i: K-chunk 2i + k/8, 16-byte piece k%8 of row rr (swizzled)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint8_t* dst = b_buf + (2 * i + (k >> 3)) * B_CHUNK + rr * 128 + (((k & 7) ^ (rr & 7)) << 4);
      *reinterpret_cast<uint4*>(dst) = make_uint4(
          pack_bf16x2(acc[8 * i + 0] * inv, acc[8 * i + 1] * inv),
          pack_bf16x2(acc[8 * i + 2] * inv, acc[8 * i + 3] * inv),
          pack_bf16x2(acc[8 * i + 4] * inv, acc[8 * i + 5] * inv),
          pack_bf16x2(acc[8 * i + 6] * inv, acc[8 * i + 7] * inv));
    }
  }
  fence_proxy_async_smem();
  __syncthreads();

  // ---- MMA: D[128 x BN] = W_UV tile · o_latᵀ, K = 512
  if (warp == 1) {   // the whole warp runs the loop, one elected lane issues
    const uint64_t a0 = smem_desc_sw128(smem_addr(a_buf), 16, 1024);
    const uint64_t b0 = smem_desc_sw128(smem_addr(b_buf), 16, 1024);
    for (int c = 0; c < VP_KCHUNKS; ++c) {
      bool ok = true;
      if (lane == 0) ok = mbar_wait(&full_bar[c], 0);
      if (__shfl_sync(0xffffffffu, ok ? 1 : 0, 0) == 0) {
        if (lane == 0) record_error(MLA_ERR_DEVICE_TIMEOUT);
        break;
      }
      (void)mbar_try_wait(&full_bar[c], 0);
      tc_fence_after_sync();
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16_ss_elect(tmem, a0 + static_cast<uint64_t>((c * VP_A_CHUNK + kk * 32) >> 4),
                          b0 + static_cast<uint64_t>((c * B_CHUNK + kk * 32) >> 4), IDESC,
                          (c > 0 || kk > 0) ? 1u : 0u);
    }
    mma_commit_elect(&done_bar);
  }
  __syncwarp();

  // ---- epilogue: warps 0..3 (thread = row m0 + threadIdx.x of the d_v tile) stage D as
  // [token][128] bf16 in the B operand buffer (its MMAs are done), then all threads store each
  // (token, head) row's 128 outputs in 16-byte pieces (one 2-byte store per thread and token
  // measured far slower)
  bool ready = true;
  if (warp < 4) {
    ready = false;
    if (lane == 0) ready = mbar_wait(&done_bar, 0);
    ready = __shfl_sync(0xffffffffu, ready ? 1 : 0, 0) != 0;
    if (ready) (void)mbar_try_wait(&done_bar, 0);
    else if (lane == 0) record_error(MLA_ERR_DEVICE_TIMEOUT);
  }
  ready = __syncthreads_and(ready ? 1 : 0) != 0;   // block-uniform: the stores below sync
  tc_fence_after_sync();
  if (ready) {
    __nv_bfloat16* stage = reinterpret_cast<__nv_bfloat16*>(b_buf);
    if (warp < 4) {
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 16) {
        uint32_t v[16];
        tmem_ld16(tmem_at(tmem, warp * 32, c0), v);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j)
          stage[(c0 + j) * 128 + threadIdx.x] = __float2bfloat16_rn(__uint_as_float(v[j]));
      }
    }
    __syncthreads();
    const int m_rows = min(128, p.d_v - m0);
    for (int i = threadIdx.x; i < BN * 16; i += VP_THREADS) {
      const int nl = i >> 4, mv = (i & 15) * 8;
      const int n = n0 + nl;
      if (n >= p.n_q || mv >= m_rows) continue;
      __nv_bfloat16* dst = p.out + (static_cast<int64_t>(n) * p.H + h) * p.d_v + m0 + mv;
      const __nv_bfloat16* src = stage + nl * 128 + mv;
      if (mv + 8 <= m_rows && (reinterpret_cast<uintptr_t>(dst) & 15u) == 0) {
        *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
      } else {
        for (int e = 0; e < 8 && mv + e < m_rows; ++e) dst[e] = src[e];
      }
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// Merge of the attention kernel's per-segment partials into one partial per query row, for a
// decode over a key range whose result another GPU's partials will be combined with:
//   o_out[row][:] = sum_s 2^(lse_s - m) O_s / sum_s 2^(lse_s - m),   lse_out[row] = (m +
//   log2(sum_s 2^(lse_s - m))) * ln 2  (natural log), -inf and zeros when the row saw no key.
// Rows are row = n * H + h (n = b * Tq + t); 64 threads per row, 8 dims each, 4 rows a block.
__global__ void __launch_bounds__(256)
merge_partials_kernel(const __nv_bfloat16* __restrict__ o_seg, const float* __restrict__ lse_seg,
                      const int32_t* __restrict__ unit_seg, int rows, int R,
                      __nv_bfloat16* __restrict__ o_out, float* __restrict__ lse_out) {
  pdl_wait();
  const int row = blockIdx.x * 4 + static_cast<int>(threadIdx.x >> 6);
  const int k = threadIdx.x & 63;
  if (row >= rows) return;
  const int b = row / R, r_in = row % R;
  const int u = unit_stream_pos(b, r_in / 128, rows / R), rl = r_in % 128;
  const int s0 = unit_seg[u], s1 = unit_seg[u + 1];
  float mx = -INFINITY;
  for (int s = s0; s < s1; ++s) mx = fmaxf(mx, lse_seg[static_cast<int64_t>(s) * 128 + rl]);
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  float den = 0.0f;
  if (mx > -INFINITY) {
    for (int s = s0; s < s1; ++s) {
      const float w = exp2f(lse_seg[static_cast<int64_t>(s) * 128 + rl] - mx);
      den += w;
      const uint4 v = reinterpret_cast<const uint4*>(
          o_seg + (static_cast<int64_t>(s) * 128 + rl) * ATT_DC)[k];
      const uint32_t q[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&q[e]));
        acc[2 * e] = fmaf(w, f.x, acc[2 * e]);
        acc[2 * e + 1] = fmaf(w, f.y, acc[2 * e + 1]);
      }
    }
  }
  const float inv = den > 0.0f ? 1.0f / den : 0.0f;
  reinterpret_cast<uint4*>(o_out + static_cast<int64_t>(row) * ATT_DC)[k] = make_uint4(
      pack_bf16x2(acc[0] * inv, acc[1] * inv), pack_bf16x2(acc[2] * inv, acc[3] * inv),
      pack_bf16x2(acc[4] * inv, acc[5] * inv), pack_bf16x2(acc[6] * inv, acc[7] * inv));
  if (k == 0)
    lse_out[row] = den > 0.0f ? (mx + log2f(den)) * 0.6931471805599453f : -INFINITY;
}

}  // namespace mla
