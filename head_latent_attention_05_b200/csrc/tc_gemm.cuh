// tcgen05 GEMM for the projections around the attention step:
//   D[m][n] = sum_k A[z][m][k] * B[n][z'][k]        (fp32 accumulate in TMEM)
// A is a weight matrix (K-major, M up to thousands of rows), B holds the activations of the
// N = batch*Tq query tokens (K-major, N small). The weights sit on the 128-row M side of the
// MMA so that a decode batch of a few tokens still fills the tensor core; each token is one
// column of D. This is HBM-bound work (every weight byte is read once per call), so the kernel
// is a plain TMA -> smem ring -> tcgen05.mma pipeline with one 128 x BN tile per CTA and as
// many CTAs as (m-tiles x n-tiles x batch index x K-splits).
//
// Roles in a 128-thread CTA: warp 0 / lane 0 issues TMA loads, warp 1 allocates TMEM and its
// lane 0 issues the MMAs; afterwards all four warps read D out of TMEM (warp w owns TMEM lanes
// 32w..32w+31 = rows m0+32w..) and hand each value to the epilogue functor.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace mla {

struct GemmShape {
  int M;             // rows of A (per batch index)
  int N;             // valid activation rows
  int k_chunks;      // total K / 64
  int chunks_per_split;
  int k_splits;      // grid.z = Z * k_splits
  int b_uses_z;      // B's middle TMA coordinate is z (per-head activations) or 0
};

constexpr int GEMM_BK = 64;        // one 128-byte swizzle row of bf16
constexpr int GEMM_STAGES = 4;

template <int BN>
constexpr int gemm_smem_bytes() {
  return GEMM_STAGES * (128 * GEMM_BK * 2 + BN * GEMM_BK * 2) + 1024;
}

template <int BN, class Epi>
__global__ void __launch_bounds__(128)
gemm_tc_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
               GemmShape shp, Epi epi) {
  constexpr int A_BYTES = 128 * GEMM_BK * 2;
  constexpr int B_BYTES = BN * GEMM_BK * 2;
  constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  constexpr uint32_t TMEM_COLS = BN < 32 ? 32 : BN;
  constexpr uint32_t IDESC = idesc_bf16(128, BN, false, false);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  __shared__ uint64_t full_bar[GEMM_STAGES], empty_bar[GEMM_STAGES], done_bar;
  __shared__ uint32_t tmem_base_s;

  const int warp = threadIdx.x >> 5;
  const int m0 = blockIdx.x * 128;
  const int n0 = blockIdx.y * BN;
  const int z = blockIdx.z / shp.k_splits;
  const int split = blockIdx.z % shp.k_splits;
  const int kc0 = split * shp.chunks_per_split;
  const int kc1 = min(shp.k_chunks, kc0 + shp.chunks_per_split);
  const int nk = kc1 - kc0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < GEMM_STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(&done_bar, 1);
    fence_mbar_init();
    tma_prefetch_desc(&mapA);
    tma_prefetch_desc(&mapB);
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_s, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = tmem_base_s;

  if (threadIdx.x == 0) {
    // ---- TMA producer
    for (int i = 0; i < nk; ++i) {
      const int s = i % GEMM_STAGES;
      if (i >= GEMM_STAGES && !mbar_wait(&empty_bar[s], ((i / GEMM_STAGES) - 1) & 1)) {
        record_error(MLA_ERR_DEVICE_TIMEOUT);
        break;
      }
      uint8_t* sa = smem + s * STAGE_BYTES;
      mbar_arrive_expect_tx(&full_bar[s], STAGE_BYTES);
      const int k = (kc0 + i) * GEMM_BK;
      tma_load_3d(sa, &mapA, &full_bar[s], k, m0, z);
      tma_load_3d(sa + A_BYTES, &mapB, &full_bar[s], k, shp.b_uses_z ? z : 0, n0);
    }
  } else if (threadIdx.x == 32) {
    // ---- MMA issuer
    bool ok = true;
    for (int i = 0; i < nk; ++i) {
      const int s = i % GEMM_STAGES;
      if (!mbar_wait(&full_bar[s], (i / GEMM_STAGES) & 1)) {
        record_error(MLA_ERR_DEVICE_TIMEOUT);
        ok = false;
        break;
      }
      tc_fence_after_sync();
      const uint32_t sa = smem_addr(smem + s * STAGE_BYTES);
      const uint64_t a0 = smem_desc_sw128(sa, 16, 1024);
      const uint64_t b0 = smem_desc_sw128(sa + A_BYTES, 16, 1024);
#pragma unroll
      for (int kk = 0; kk < GEMM_BK / 16; ++kk) {   // +32 bytes per K-step of 16
        mma_bf16_ss(tmem, a0 + static_cast<uint64_t>(kk * 2), b0 + static_cast<uint64_t>(kk * 2), IDESC,
                    (i > 0 || kk > 0) ? 1u : 0u);
      }
      mma_commit(&empty_bar[s]);
    }
    (void)ok;
    mma_commit(&done_bar);
  }
  __syncwarp();

  // ---- epilogue: all 128 threads, thread = row m0 + threadIdx.x
  epi.prologue(z, split);
  bool ready = false;
  if ((threadIdx.x & 31) == 0) ready = mbar_wait(&done_bar, 0);
  ready = __shfl_sync(0xffffffffu, ready ? 1 : 0, 0) != 0;
  if (ready) (void)mbar_try_wait(&done_bar, 0);
  else if ((threadIdx.x & 31) == 0) record_error(MLA_ERR_DEVICE_TIMEOUT);
  tc_fence_after_sync();
  const int m = m0 + threadIdx.x;
  if (ready && nk > 0) {
#pragma unroll 1
    for (int c0 = 0; c0 < BN; c0 += 16) {
      uint32_t v[16];
      tmem_ld16(tmem_at(tmem, warp * 32, c0), v);
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
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ------------------------------------------------------------------------------ epilogues

// Append down-projection with split-K: partial[split][n][m] (fp32), summed later in order.
struct EpiSplitK {
  float* partial;
  int n_tok, F;
  __device__ void prologue(int, int) const {}
  __device__ void operator()(int, int split, int m, int n, float v) const {
    partial[(static_cast<int64_t>(split) * n_tok + n) * F + m] = v;
  }
};

// Absorbed query: qhat[(n*H + h)][m] = q_lat (bf16), m < d_c. The CTAs of m-tile 0 also write
// the rotated rope part qhat[..][d_c + i] while their MMAs run.
struct EpiQhat {
  __nv_bfloat16* qhat;
  const __nv_bfloat16* q;        // [B*Tq][H][d_nope + d_r]
  const int32_t* seq_lens;       // [B]
  int H, Tq, d_c, d_r, d_nope, n_rows, max_pos;
  float theta;
  __device__ void prologue(int h, int) const {
    if (blockIdx.x != 0 || blockIdx.y != 0) return;
    const int row = d_c + d_r;
    const int half = d_r / 2;
    for (int i = threadIdx.x; i < n_rows * half; i += blockDim.x) {
      const int n = i / half, pr = i % half;
      const int b = n / Tq, t = n % Tq;
      const int L = seq_lens[b];
      const __nv_bfloat16* qr = q + (static_cast<int64_t>(n) * H + h) * (d_nope + d_r) + d_nope;
      float ox = 0.0f, oy = 0.0f;
      if (L >= Tq && L <= max_pos)
        rope_pair(__bfloat162float(qr[2 * pr]), __bfloat162float(qr[2 * pr + 1]), pr, d_r,
                  L - Tq + t, theta, &ox, &oy);
      __nv_bfloat16* dst = qhat + (static_cast<int64_t>(n) * H + h) * row + d_c + 2 * pr;
      dst[0] = __float2bfloat16_rn(ox);
      dst[1] = __float2bfloat16_rn(oy);
    }
  }
  __device__ void operator()(int h, int, int m, int n, float v) const {
    qhat[(static_cast<int64_t>(n) * H + h) * (d_c + d_r) + m] = __float2bfloat16_rn(v);
  }
};

// Value up-projection: out[(n*H + h)][m] (bf16), m < d_v.
struct EpiOut {
  __nv_bfloat16* out;
  int H, d_v;
  __device__ void prologue(int, int) const {}
  __device__ void operator()(int h, int, int m, int n, float v) const {
    out[(static_cast<int64_t>(n) * H + h) * d_v + m] = __float2bfloat16_rn(v);
  }
};

}  // namespace mla
