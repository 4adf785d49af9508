// tcgen05 GEMM for the projections around the attention step:
//   D[m][n] = sum_k A[z][m][k] * B[n][z'][k]        (fp32 accumulate in TMEM)
// A is a weight matrix (K-major, M up to thousands of rows), B holds the activations of the
// N = batch*Tq query tokens (K-major, N small). The weights sit on the 128-row M side of the
// MMA so that a decode batch of a few tokens still fills the tensor core; each token is one
// column of D. This is HBM-bound work (every weight byte is read once per call), so the kernel
// is a TMA -> shared-memory ring -> tcgen05.mma pipeline whose ring is deep enough (8 stages
// of 16 KB weights for small N) that one CTA per SM keeps ~128 KB of loads in flight. A CTA
// may own several consecutive 128-row m-tiles (one TMEM accumulator each) so that a short-K
// product such as the per-head query absorption (K = 128) still streams many tiles per CTA.
//
// Roles in a 128-thread CTA: warp 0 / lane 0 issues TMA loads, warp 1 allocates TMEM and issues
// the MMAs (the whole warp runs the loop, one elected lane issues), warps 2-3 run the epilogue
// functor's side job (Epi::side); afterwards all four warps read D out of TMEM (warp w owns TMEM lanes
// 32w..32w+31 = rows m0+32w..) and hand each value to the epilogue functor. Extra blocks at the
// end of grid.z (GemmShape::aux_blocks) skip the GEMM and run the functor's aux() job instead.
#pragma once

#include "common.cuh"
#include "ptx.cuh"
#include "tc_decode.cuh"

namespace mla {

struct GemmShape {
  int M;             // rows of A (per batch index)
  int N;             // valid activation rows
  int k_chunks;      // total K / 64
  int chunks_per_split;
  int k_splits;      // grid.z = Z * k_splits + aux_blocks
  int b_uses_z;      // B's middle TMA coordinate is z (per-head activations) or 0
  int m_per_cta;     // consecutive 128-row m-tiles per CTA (grid.x = ceil(m_tiles / m_per_cta))
  int aux_blocks;    // trailing blocks of grid.z that run Epi::aux() instead
};

constexpr int GEMM_BK = 64;        // one 128-byte swizzle row of bf16

template <int BN>
__host__ __device__ constexpr int gemm_stages() {
  return BN <= 32 ? 8 : (BN == 64 ? 6 : (BN == 128 ? 5 : 4));
}

template <int BN, class Epi>
__host__ __device__ constexpr int gemm_smem_bytes() {
  return gemm_stages<BN>() * (128 * GEMM_BK * 2 + BN * GEMM_BK * 2) + Epi::side_bytes(BN) + 1024;
}

// TMEM columns for m_per_cta accumulators of BN columns: a power of two, at least 32.
__host__ __device__ constexpr uint32_t gemm_tmem_cols(int BN, int m_per_cta) {
  uint32_t n = 32;
  while (n < static_cast<uint32_t>(BN * m_per_cta)) n <<= 1;
  return n;
}

template <int BN, class Epi>
__global__ void __launch_bounds__(128)
gemm_tc_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
               GemmShape shp, const __grid_constant__ Epi epi) {
  constexpr int STAGES = gemm_stages<BN>();
  constexpr int A_BYTES = 128 * GEMM_BK * 2;
  constexpr int B_BYTES = BN * GEMM_BK * 2;
  constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  constexpr uint32_t IDESC = idesc_bf16(128, BN, false, false);

  if (static_cast<int>(blockIdx.z) >= static_cast<int>(gridDim.z) - shp.aux_blocks) {
    // the aux slice of grid.z exists for every (x, y); its job runs once
    if (blockIdx.x == 0 && blockIdx.y == 0) epi.aux();
    return;
  }

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  __shared__ uint64_t full_bar[STAGES], empty_bar[STAGES], done_bar, side_bar;
  __shared__ uint32_t tmem_base_s;
  uint8_t* side_smem = smem + STAGES * STAGE_BYTES;   // Epi::side_bytes(BN), 1024-aligned

  const int warp = threadIdx.x >> 5;
  const int mt0 = blockIdx.x * shp.m_per_cta;
  const int n_mt_total = (shp.M + 127) / 128;
  const int n_mt = min(shp.m_per_cta, n_mt_total - mt0);   // m-tiles of this CTA
  const int n0 = blockIdx.y * BN;
  const int z = blockIdx.z / shp.k_splits;
  const int split = blockIdx.z % shp.k_splits;
  const int kc0 = split * shp.chunks_per_split;
  const int kc1 = min(shp.k_chunks, kc0 + shp.chunks_per_split);
  const int nk = kc1 - kc0;
  const int n_iter = n_mt * nk;                // (m-tile, k-chunk) pairs, m-tile outer
  const uint32_t tmem_cols = gemm_tmem_cols(BN, shp.m_per_cta);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(&done_bar, 1);
    mbar_init(&side_bar, 1);
    fence_mbar_init();
    tma_prefetch_desc(&mapA);
    tma_prefetch_desc(&mapB);
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_s, tmem_cols);
    tmem_relinquish();
  }
  // the side job's own small loads go out before anything else of this CTA
  typename Epi::SideState side_state{};
  if (warp >= 2) side_state = epi.side_begin(static_cast<int>(threadIdx.x) - 64,
                                             static_cast<int>(blockDim.x) - 64, n0);
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = tmem_base_s;
  pdl_wait();
  pdl_trigger();

  if (threadIdx.x == 0) {
    // ---- TMA producer (the side job's box first, so that it lands ahead of the weights)
    epi.side_issue(&mapB, side_smem, &side_bar, z, n0);
    for (int i = 0; i < n_iter; ++i) {
      const int s = i % STAGES;
      if (i >= STAGES && !mbar_wait(&empty_bar[s], ((i / STAGES) - 1) & 1)) {
        record_error(MLA_ERR_DEVICE_TIMEOUT);
        break;
      }
      uint8_t* sa = smem + s * STAGE_BYTES;
      mbar_arrive_expect_tx(&full_bar[s], STAGE_BYTES);
      const int mt = i / nk, k = (kc0 + i % nk) * GEMM_BK;
      tma_load_3d(sa, &mapA, &full_bar[s], k, (mt0 + mt) * 128, z);
      tma_load_3d(sa + A_BYTES, &mapB, &full_bar[s], k, shp.b_uses_z ? z : 0, n0);
    }
  } else if (warp >= 2) {
    // ---- warps 2-3: the epilogue functor's side work, while the loads and MMAs run
    epi.side(z, split, static_cast<int>(threadIdx.x) - 64, static_cast<int>(blockDim.x) - 64, n0,
             side_state, side_smem, &side_bar);
  } else if (warp == 1) {
    // ---- MMA issuer: the whole warp runs the loop, one elected lane issues
    const int lane = threadIdx.x & 31;
    for (int i = 0; i < n_iter; ++i) {
      const int s = i % STAGES;
      bool ok = true;
      if (lane == 0) ok = mbar_wait(&full_bar[s], (i / STAGES) & 1);
      if (__shfl_sync(0xffffffffu, ok ? 1 : 0, 0) == 0) {
        if (lane == 0) record_error(MLA_ERR_DEVICE_TIMEOUT);
        break;
      }
      (void)mbar_try_wait(&full_bar[s], (i / STAGES) & 1);
      tc_fence_after_sync();
      const int mt = i / nk, kc = i % nk;
      const uint32_t sa = smem_addr(smem + s * STAGE_BYTES);
      const uint64_t a0 = smem_desc_sw128(sa, 16, 1024);
      const uint64_t b0 = smem_desc_sw128(sa + A_BYTES, 16, 1024);
#pragma unroll
      for (int kk = 0; kk < GEMM_BK / 16; ++kk) {   // +32 bytes per K-step of 16
        mma_bf16_ss_elect(tmem + mt * BN, a0 + static_cast<uint64_t>(kk * 2),
                          b0 + static_cast<uint64_t>(kk * 2), IDESC, (kc > 0 || kk > 0) ? 1u : 0u);
      }
      mma_commit_elect(&empty_bar[s]);
    }
    mma_commit_elect(&done_bar);
  }
  __syncwarp();

  // ---- epilogue: all 128 threads, thread = row (mt0 + mt)*128 + threadIdx.x
  bool ready = false;
  if ((threadIdx.x & 31) == 0) ready = mbar_wait(&done_bar, 0);
  ready = __shfl_sync(0xffffffffu, ready ? 1 : 0, 0) != 0;
  if (ready) (void)mbar_try_wait(&done_bar, 0);
  else if ((threadIdx.x & 31) == 0) record_error(MLA_ERR_DEVICE_TIMEOUT);
  tc_fence_after_sync();
  if (ready && nk > 0) {
#pragma unroll 1
    for (int mt = 0; mt < n_mt; ++mt) {
      const int m = (mt0 + mt) * 128 + threadIdx.x;
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 16) {
        uint32_t v[16];
        tmem_ld16(tmem_at(tmem, warp * 32, mt * BN + c0), v);
        tmem_ld_wait();
        if (m < shp.M) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int n = n0 + c0 + j;
            if (n < shp.N) epi(z, split, m, n, __uint_as_float(v[j]));
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
    tmem_dealloc(tmem, tmem_cols);
  }
}

// ------------------------------------------------------------------------------ epilogues

// Append down-projection with split-K: partial[split][n][m] (fp32), summed later in order.
struct EpiSplitK {
  float* partial;
  int n_tok, F;
  struct SideState {};
  __host__ __device__ static constexpr int side_bytes(int) { return 0; }
  __device__ void aux() const {}
  __device__ SideState side_begin(int, int, int) const { return {}; }
  __device__ void side_issue(const CUtensorMap*, uint8_t*, uint64_t*, int, int) const {}
  __device__ void side(int, int, int, int, int, const SideState&, const uint8_t*, uint64_t*) const {}
  __device__ void operator()(int, int split, int m, int n, float v) const {
    partial[(static_cast<int64_t>(split) * n_tok + n) * F + m] = v;
  }
};

// Plain store: out[n][m] = v rounded to bf16, rows of `ld` elements (the q path's up-projection
// wq_b, whose M side is the n_heads * (d_nope + d_rope) query features of each token).
struct EpiStoreBf16 {
  __nv_bfloat16* out;
  int ld;
  struct SideState {};
  __host__ __device__ static constexpr int side_bytes(int) { return 0; }
  __device__ void aux() const {}
  __device__ SideState side_begin(int, int, int) const { return {}; }
  __device__ void side_issue(const CUtensorMap*, uint8_t*, uint64_t*, int, int) const {}
  __device__ void side(int, int, int, int, int, const SideState&, const uint8_t*, uint64_t*) const {}
  __device__ void operator()(int, int, int m, int n, float v) const {
    out[static_cast<int64_t>(n) * ld + m] = __float2bfloat16_rn(v);
  }
};

// Absorbed query: qhat[(n*H + h)][m] = q_lat (bf16), m < d_c. Warps 2-3 of the n-tile-0 CTA of
// head h also write the rotated rope part qhat[..][d_c + i] while the MMAs run, and the one aux
// block runs the split-KV planner of the attention kernel that follows.
struct EpiQhat {
  __nv_bfloat16* qhat;
  const __nv_bfloat16* q;        // [B*Tq][H][d_nope + d_r]
  const int32_t* seq_lens;       // [B]
  int H, Tq, d_c, d_r, d_nope, n_rows, max_pos;
  int box_rows;                  // tokens per CTA (the GEMM's BN)
  PlanParams plan;
  RopeFreqs rope;
  __device__ void aux() const { attn_plan_block(plan); }
  // RoPE(q_rope) of head h for this CTA's BN tokens, written to qhat[..][d_c:] by warps 2-3 of
  // the m-tile-0 CTA while the MMAs run. The producer brings the BN x 64 q_rope box in with the
  // B tensor map (128-byte swizzle) ahead of the weight stream; each side thread owns one token
  // (the token's length is read at the start, before the stream begins) and a share of its
  // rotary pairs.
  struct SideState {
    int len;   // seq_lens of the first token this thread handles
  };
  __host__ __device__ static constexpr int side_bytes(int bn) { return bn * 128; }
  __device__ bool rope_cta() const { return blockIdx.x == 0; }
  __device__ SideState side_begin(int tid, int nt, int n0) const {
    SideState st{-1};
    const int t1 = box_rows < nt ? box_rows : nt;
    const int n = n0 + tid % t1;
    if (rope_cta() && n < n_rows) st.len = seq_lens[n / Tq];
    return st;
  }
  __device__ void side_issue(const CUtensorMap* map_q, uint8_t* side_smem, uint64_t* bar, int h,
                             int n0) const {
    if (!rope_cta()) return;
    mbar_arrive_expect_tx(bar, static_cast<uint32_t>(side_box_rows() * 128));
    tma_load_3d(side_smem, map_q, bar, d_nope, h, n0);
  }
  __device__ int side_box_rows() const { return box_rows; }
  __device__ void side(int h, int, int tid, int nt, int n0, const SideState& st,
                       const uint8_t* side_smem, uint64_t* bar) const {
    if (!rope_cta()) return;
    const int lane = tid & 31;
    bool ok = true;
    if (lane == 0) ok = mbar_wait(bar, 0);
    if (__shfl_sync(0xffffffffu, ok ? 1 : 0, 0) == 0) {
      if (lane == 0) record_error(MLA_ERR_DEVICE_TIMEOUT);
      return;
    }
    (void)mbar_try_wait(bar, 0);
    const int row = d_c + d_r;
    const int half = d_r / 2;                    // 32 pairs, one 128-byte smem row per token
    const int t1 = box_rows < nt ? box_rows : nt;   // token columns handled at once
    const int groups = nt / t1;                  // pair groups per token
    const int pg = tid / t1;
    for (int nl = tid % t1, first = 1; nl < box_rows; nl += t1, first = 0) {
      const int n = n0 + nl;
      if (n >= n_rows) break;
      const int L = first ? st.len : seq_lens[n / Tq];
      const bool ok_len = L >= Tq && L <= max_pos;
      const int ps = L - Tq + n % Tq;
      for (int r = pg; r < half; r += groups) {
        // element 2r of row nl in the swizzled box: 16-byte chunk (2r/8) ^ (nl % 8)
        const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(
            side_smem + nl * 128 + ((((2 * r) >> 3) ^ (nl & 7)) << 4) + ((2 * r) & 7) * 2);
        float ox = 0.0f, oy = 0.0f;
        if (ok_len)
          rope_pair(__low2float(v), __high2float(v), rope.f_hi[r], rope.f_lo[r], ps, &ox, &oy);
        *reinterpret_cast<__nv_bfloat162*>(qhat + (static_cast<int64_t>(n) * H + h) * row + d_c +
                                           2 * r) = __floats2bfloat162_rn(ox, oy);
      }
    }
  }
  __device__ void operator()(int h, int, int m, int n, float v) const {
    qhat[(static_cast<int64_t>(n) * H + h) * (d_c + d_r) + m] = __float2bfloat16_rn(v);
  }
};

}  // namespace mla
