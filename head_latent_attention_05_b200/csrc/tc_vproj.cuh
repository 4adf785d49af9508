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

struct VprojParams {
  const __nv_bfloat16* o_part;  // [segments][128][512] per-segment O / l (bf16)
  const float* lse;           // [segments][128] base-2 log-sum-exp of each partial
  const int32_t* unit_seg;    // [U + 1] first segment of each unit
  __nv_bfloat16* out;         // [n_q][H][d_v]
  int H, Tq, n_mt, n_q, d_v;
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
  // the segment lists were written two kernels back (by the planner): read them before waiting
  int seg0[PASSES], seg1[PASSES], rowl[PASSES];
#pragma unroll
  for (int ps = 0; ps < PASSES; ++ps) {
    const int n = n0 + ps * RP + rr_l;
    seg0[ps] = seg1[ps] = rowl[ps] = 0;
    if (n < p.n_q) {
      const int b = n / p.Tq, t = n % p.Tq;
      const int r = t * p.H + h;
      const int u = b * p.n_mt + r / 128;
      seg0[ps] = p.unit_seg[u];
      seg1[ps] = p.unit_seg[u + 1];
      rowl[ps] = r % 128;
    }
  }
  pdl_wait();   // the attention partials are complete and visible from here on
  pdl_trigger();
#pragma unroll
  for (int ps = 0; ps < PASSES; ++ps) {
    const int rr = ps * RP + rr_l;
    const int s0 = seg0[ps], s1 = seg1[ps], rl = rowl[ps];
    float mx = -INFINITY;
    for (int s = s0 + k; s < s1; s += TPR) mx = fmaxf(mx, p.lse[static_cast<int64_t>(s) * 128 + rl]);
#pragma unroll
    for (int o = TPR / 2; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float den = 0.0f;
    float acc[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) acc[e] = 0.0f;
    if (mx > -INFINITY) {
      for (int s = s0 + k; s < s1; s += TPR) den += exp2f(p.lse[static_cast<int64_t>(s) * 128 + rl] - mx);
      // four segments' loads in flight at a time; the sum runs in segment order
      for (int sb = s0; sb < s1; sb += 4) {
        float w[4];
        uint4 v[4][4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int s = sb + j;
          w[j] = 0.0f;
          if (s < s1) {
            w[j] = exp2f(p.lse[static_cast<int64_t>(s) * 128 + rl] - mx);
            const uint4* src = reinterpret_cast<const uint4*>(
                p.o_part + (static_cast<int64_t>(s) * 128 + rl) * ATT_DC);
#pragma unroll
            for (int i = 0; i < 4; ++i) v[j][i] = src[k + TPR * i];
          }
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (sb + j >= s1) break;
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

  // ---- epilogue: warps 0..3, thread = row m0 + threadIdx.x of the d_v tile
  if (warp < 4) {
    bool ready = false;
    if (lane == 0) ready = mbar_wait(&done_bar, 0);
    ready = __shfl_sync(0xffffffffu, ready ? 1 : 0, 0) != 0;
    if (ready) (void)mbar_try_wait(&done_bar, 0);
    else if (lane == 0) record_error(MLA_ERR_DEVICE_TIMEOUT);
    tc_fence_after_sync();
    const int m = m0 + threadIdx.x;
    if (ready) {
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 16) {
        uint32_t v[16];
        tmem_ld16(tmem_at(tmem, warp * 32, c0), v);
        tmem_ld_wait();
        if (m < p.d_v) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int n = n0 + c0 + j;
            if (n < p.n_q)
              p.out[(static_cast<int64_t>(n) * p.H + h) * p.d_v + m] =
                  __float2bfloat16_rn(__uint_as_float(v[j]));
          }
        }
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

}  // namespace mla
