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
// functor's side job (Epi::side); afterwards all four warps read D out of TMEM (warp w owns TMEM
// lanes 32w..32w+31 = rows m0+32w..), convert each value to the functor's output type and stage
// the m-tile in shared memory (the drained load ring) as [token][128 m], so that each token's
// 128 outputs, contiguous in every output layout used here, leave in 16-byte stores: scattered
// 2-byte stores (one per thread and token) measured ~85 cycles a warp instruction on B200 and
// made the epilogue most of the kernel. Extra blocks at the end of grid.z
// (GemmShape::aux_blocks) skip the GEMM and run the functor's aux() job instead.
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
    // the aux slice of grid.z exists for every (x, y); each of its jobs runs once
    if (blockIdx.x == 0 && blockIdx.y == 0)
      epi.aux(static_cast<int>(blockIdx.z) - (static_cast<int>(gridDim.z) - shp.aux_blocks));
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
  // block-uniform (every thread has left its role): the staging loop below syncs the block
  ready = __syncthreads_and(ready ? 1 : 0) != 0;
  tc_fence_after_sync();
  if (ready && nk > 0) {
    using Out = typename Epi::Out;
    constexpr int TILE = BN * 128;                              // staged outputs per m-tile
    constexpr int GROUP = (STAGES * STAGE_BYTES) / (TILE * static_cast<int>(sizeof(Out)));
    static_assert(GROUP >= 1, "staging tile exceeds the ring");
    constexpr int VEC = 16 / static_cast<int>(sizeof(Out));   // outputs per 16-byte store
    constexpr int ROW_VECS = 128 / VEC;
    Out* stage = reinterpret_cast<Out*>(smem);   // [m-tile][BN][128]; loads and MMAs are done
    // as many m-tiles as the ring holds are staged, then all their rows leave at once
#pragma unroll 1
    for (int g0 = 0; g0 < n_mt; g0 += GROUP) {
      const int g1 = min(n_mt, g0 + GROUP);
#pragma unroll 1
      for (int mt = g0; mt < g1; ++mt) {
        Out* tile = stage + (mt - g0) * TILE;
        if constexpr (BN % 64 == 0) {   // 64 columns per wait
#pragma unroll 1
          for (int c0 = 0; c0 < BN; c0 += 64) {
            uint32_t v0[32], v1[32];
            tmem_ld32(tmem_at(tmem, warp * 32, mt * BN + c0), v0);
            tmem_ld32(tmem_at(tmem, warp * 32, mt * BN + c0 + 32), v1);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              tile[(c0 + j) * 128 + threadIdx.x] = Epi::cvt(__uint_as_float(v0[j]));
              tile[(c0 + 32 + j) * 128 + threadIdx.x] = Epi::cvt(__uint_as_float(v1[j]));
            }
          }
        } else {
#pragma unroll 1
          for (int c0 = 0; c0 < BN; c0 += 16) {
            uint32_t v[16];
            tmem_ld16(tmem_at(tmem, warp * 32, mt * BN + c0), v);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 16; ++j) tile[(c0 + j) * 128 + threadIdx.x] = Epi::cvt(__uint_as_float(v[j]));
          }
        }
      }
      __syncthreads();
      const int items = (g1 - g0) * BN * ROW_VECS;
      for (int i = threadIdx.x; i < items; i += blockDim.x) {
        const int t = i / (BN * ROW_VECS), rem = i % (BN * ROW_VECS);
        const int nl = rem / ROW_VECS, mv = (rem % ROW_VECS) * VEC;
        const int n = n0 + nl;
        const int m_base = (mt0 + g0 + t) * 128;
        const int m_rows = min(128, shp.M - m_base);
        if (n >= shp.N || mv >= m_rows) continue;
        Out* dst = epi.row(z, split, n) + m_base + mv;
        const Out* src = stage + t * TILE + nl * 128 + mv;
        if (mv + VEC <= m_rows && (reinterpret_cast<uintptr_t>(dst) & 15u) == 0) {
          *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
        } else {
          for (int e = 0; e < VEC && mv + e < m_rows; ++e) dst[e] = src[e];
        }
      }
      __syncthreads();   // the next group reuses the staging area
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

// Output interface of every functor: Out (the stored type), cvt (fp32 accumulator -> Out) and
// row(z, split, n), the address of output (m = 0, n); a row's m outputs are contiguous.

// Append down-projection with split-K: partial[split][n][m] (fp32), summed later in order.
struct EpiSplitK {
  float* partial;
  int n_tok, F;
  using Out = float;
  __device__ static float cvt(float v) { return v; }
  __device__ float* row(int, int split, int n) const {
    return partial + (static_cast<int64_t>(split) * n_tok + n) * F;
  }
  struct SideState {};
  __host__ __device__ static constexpr int side_bytes(int) { return 0; }
  __device__ void aux(int) const {}
  __device__ SideState side_begin(int, int, int) const { return {}; }
  __device__ void side_issue(const CUtensorMap*, uint8_t*, uint64_t*, int, int) const {}
  __device__ void side(int, int, int, int, int, const SideState&, const uint8_t*, uint64_t*) const {}
};

// Plain store: out[n][m] = v rounded to bf16, rows of `ld` elements (the q path's up-projection
// wq_b, whose M side is the n_heads * (d_nope + d_rope) query features of each token).
struct EpiStoreBf16 {
  __nv_bfloat16* out;
  int ld;
  using Out = __nv_bfloat16;
  __device__ static __nv_bfloat16 cvt(float v) { return __float2bfloat16_rn(v); }
  __device__ __nv_bfloat16* row(int, int, int n) const { return out + static_cast<int64_t>(n) * ld; }
  struct SideState {};
  __host__ __device__ static constexpr int side_bytes(int) { return 0; }
  __device__ void aux(int) const {}
  __device__ SideState side_begin(int, int, int) const { return {}; }
  __device__ void side_issue(const CUtensorMap*, uint8_t*, uint64_t*, int, int) const {}
  __device__ void side(int, int, int, int, int, const SideState&, const uint8_t*, uint64_t*) const {}
};

// Absorbed query: qhat[(n*H + h)][m] = q_lat (bf16), m < d_c. Aux block 0 runs the split-KV
// planner of the attention kernel that follows; aux blocks 1..rope_blocks write the rotated rope
// part qhat[..][d_c:] (rope_rows) while the head CTAs stream W_UK.
struct EpiQhat {
  __nv_bfloat16* qhat;
  const __nv_bfloat16* q;        // [B*Tq][H][d_nope + d_r]
  const int32_t* seq_lens;       // [B]
  int H, Tq, d_c, d_r, d_nope, n_rows, max_pos;
  int rope_blocks;               // aux blocks that rotate q_rope (after the planner's one)
  PlanParams plan;
  RopeFreqs rope;
  using Out = __nv_bfloat16;
  __device__ static __nv_bfloat16 cvt(float v) { return __float2bfloat16_rn(v); }
  __device__ __nv_bfloat16* row(int h, int, int n) const {
    return qhat + (static_cast<int64_t>(n) * H + h) * (d_c + d_r);
  }
  struct SideState {};
  __host__ __device__ static constexpr int side_bytes(int) { return 0; }
  __device__ SideState side_begin(int, int, int) const { return {}; }
  __device__ void side_issue(const CUtensorMap*, uint8_t*, uint64_t*, int, int) const {}
  __device__ void side(int, int, int, int, int, const SideState&, const uint8_t*, uint64_t*) const {}
  __device__ void aux(int i) const {
    if (i == 0) attn_plan_block(plan);
    else rope_rows(i - 1);
  }
  // RoPE(q_rope) of every (token, head). The angle depends on the token's position and the pair
  // only, so one thread per (token, pair) computes it once and turns that pair for all H heads;
  // a warp covers 32 pairs of one token, i.e. 128 contiguous bytes of a (token, head) row per
  // load and store.
  __device__ void rope_rows(int blk) const {
    const int half = d_r / 2;
    const int qrow = d_nope + d_r, orow = d_c + d_r;   // elements per (token, head) row
    const int64_t total = static_cast<int64_t>(n_rows) * half;
    const int64_t step = static_cast<int64_t>(rope_blocks) * blockDim.x;
    for (int64_t idx = static_cast<int64_t>(blk) * blockDim.x + threadIdx.x; idx < total;
         idx += step) {
      const int n = static_cast<int>(idx / half), r = static_cast<int>(idx % half);
      const int L = seq_lens[n / Tq];
      const bool ok = L >= Tq && L <= max_pos;
      float sn = 0.0f, cs = 0.0f;
      if (ok) rope_sincos(rope.f_hi[r], rope.f_lo[r], L - Tq + n % Tq, &sn, &cs);
      const __nv_bfloat162* src = reinterpret_cast<const __nv_bfloat162*>(
          q + static_cast<int64_t>(n) * H * qrow + d_nope) + r;
      __nv_bfloat162* dst = reinterpret_cast<__nv_bfloat162*>(
          qhat + static_cast<int64_t>(n) * H * orow + d_c) + r;
      // 64 heads' loads in flight at a time (the rows come from HBM: latency, not bandwidth)
      constexpr int HB = 64;
      for (int h0 = 0; h0 < H; h0 += HB) {
        __nv_bfloat162 v[HB];
#pragma unroll
        for (int j = 0; j < HB; ++j)
          v[j] = h0 + j < H ? src[static_cast<int64_t>(h0 + j) * (qrow / 2)]
                            : __floats2bfloat162_rn(0.0f, 0.0f);
#pragma unroll
        for (int j = 0; j < HB; ++j) {
          if (h0 + j >= H) break;
          const float2 f = __bfloat1622float2(v[j]);
          float ox = 0.0f, oy = 0.0f;
          if (ok) rope_turn(f.x, f.y, sn, cs, &ox, &oy);
          dst[static_cast<int64_t>(h0 + j) * (orow / 2)] = __floats2bfloat162_rn(ox, oy);
        }
      }
    }
  }
};

}  // namespace mla
