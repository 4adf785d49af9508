// Absorbed-MLA decode attention on tcgen05 (bf16 cache, d_c = 512, d_r = 64, 64-token pages).
//
// Work split. For sequence b the R = Tq*H query rows (row r = t*H + h) form ceil(R/128)
// "units" of 128 rows; every unit attends over the sequence's pages (tiles of 64 tokens). A
// planning kernel cuts the concatenated tile list of all units into P equal ranges, one per
// pair of CTAs, so long and short sequences spread evenly over the GPU (split-KV). Each
// range piece inside one unit is a "segment"; it produces a partial result (O / l, lse) that
// the combine kernel merges by log-sum-exp.
//
// One pair of CTAs per range. Both CTAs run the same token tiles: each computes the full
// score tile S = Q̂·Cᵀ (K = 576) and the same softmax, and accumulates its own half of the
// latent output O[:, half*256 : half*256+256] += P·C[:, half]. Splitting d_c this way keeps
// the fp32 accumulator within TMEM (256 columns per CTA) without any cross-CTA exchange.
//
// Per CTA: TMEM columns [0,256) O half, [256,320) S, [320,512) Q̂[:, 0:384] as bf16 pairs (the
// A operand of the first 24 K-steps of S). Shared memory: 2 stages x 9 chunks of
// [64 tokens x 64 dims] (the whole 576-wide page, 128-byte swizzle, one TMA box per chunk),
// Q̂[:, 384:576] (3 chunks of [128 x 64]) and P [128 x 64] bf16.
//
// Warp roles (192 threads): warp 0 TMA producer, warp 1 TMEM owner + MMA issuer, warps 2..5
// softmax / rescale / epilogue (warp w owns TMEM lanes 32*(w%4).., i.e. query rows).
// Online softmax in base 2 with a lazy rescale: the running maximum only moves (and O is
// rescaled) when a new score exceeds it by more than 2^8, which keeps every P <= 256.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace mla {

constexpr int ATT_DC = 512;
constexpr int ATT_DR = 64;
constexpr int ATT_ROW = ATT_DC + ATT_DR;          // 576
constexpr int ATT_PAGE = 64;
constexpr int ATT_CHUNK_BYTES = ATT_PAGE * 128;   // [64 rows x 64 bf16]
constexpr int ATT_CHUNKS = ATT_ROW / 64;          // 9
constexpr int ATT_TILE_BYTES = ATT_CHUNKS * ATT_CHUNK_BYTES;
constexpr int ATT_STAGES = 2;
constexpr int ATT_QT_ELEMS = 384;                 // Q̂ columns kept in TMEM
constexpr int ATT_QS_CHUNKS = (ATT_ROW - ATT_QT_ELEMS) / 64;   // 3 chunks of Q̂ in smem
constexpr int ATT_QS_CHUNK_BYTES = 128 * 128;     // [128 rows x 64 bf16]
constexpr int ATT_P_BYTES = 128 * 128;            // P [128 x 64] bf16
constexpr int ATT_THREADS = 192;
constexpr int ATT_SMEM_BYTES =
    ATT_STAGES * ATT_TILE_BYTES + ATT_QS_CHUNKS * ATT_QS_CHUNK_BYTES + ATT_P_BYTES + 1024;
constexpr uint32_t TM_O = 0, TM_S = 256, TM_Q = 320;
constexpr float ATT_RESCALE_THRESHOLD = 8.0f;     // log2 units

struct AttnSeg {
  int32_t unit;        // b * n_mt + mt
  int32_t tile_begin;  // first 64-token page of the segment
  int32_t tile_end;    // one past the last
  int32_t pair;        // CTA pair that runs it
};

struct AttnParams {
  const int32_t* block_table;
  const int32_t* seq_lens;
  const AttnSeg* segs;
  const int32_t* pair_seg;   // [P + 1]: pair p runs segments [pair_seg[p], pair_seg[p+1])
  const __nv_bfloat16* qhat; // [B*R][576]
  float* o_part;             // [max_segs][128][512]
  float* lse;                // [max_segs][128]   (base-2 log-sum-exp of the scaled scores)
  int max_pages, num_pages;
  int H, Tq, R, n_mt;
  float scale_log2;          // softmax_scale * log2(e)
};

// ------------------------------------------------------------------------ planning kernel

struct PlanParams {
  const int32_t* seq_lens;
  int B, Tq, n_mt, max_pos, P, max_segs;
  int32_t* unit_tiles;   // [U] scratch: first global tile of each unit
  int32_t* unit_seg;     // [U + 1]
  int32_t* pair_seg;     // [P + 1]
  AttnSeg* segs;         // [max_segs]
};

__device__ __forceinline__ int64_t pair_start(int p, int64_t T, int P) {
  return (static_cast<int64_t>(p) * T) / P;
}
// Largest p in [0, P) with pair_start(p) <= x (x in [0, T)).
__device__ __forceinline__ int pair_of(int64_t x, int64_t T, int P) {
  int p = static_cast<int>((x * P) / T);
  while (p + 1 < P && pair_start(p + 1, T, P) <= x) ++p;
  while (p > 0 && pair_start(p, T, P) > x) --p;
  return p;
}

// Block-wide exclusive scan of one int per thread (blockDim.x == 1024); returns the total.
__device__ __forceinline__ int block_exclusive_scan(int v, int* excl, int* warp_tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = warp_tot[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    warp_tot[lane] = w;  // inclusive
  }
  __syncthreads();
  const int before = (warp > 0 ? warp_tot[warp - 1] : 0);
  *excl = before + x - v;
  const int total = warp_tot[31];
  __syncthreads();
  return total;
}

__global__ void __launch_bounds__(1024) attn_plan_kernel(PlanParams pp) {
  __shared__ int warp_tot[32];
  __shared__ int carry_s;
  const int U = pp.B * pp.n_mt;
  // pass 1: tiles per unit -> global tile offsets
  if (threadIdx.x == 0) carry_s = 0;
  __syncthreads();
  for (int u0 = 0; u0 < U; u0 += 1024) {
    const int u = u0 + threadIdx.x;
    int n = 0;
    if (u < U) {
      const int b = u / pp.n_mt;
      const int L = pp.seq_lens[b];
      if (L >= pp.Tq && L <= pp.max_pos) {
        n = (L + ATT_PAGE - 1) / ATT_PAGE;
      } else if (u % pp.n_mt == 0) {
        record_error(MLA_ERR_DEVICE_BAD_LENGTH);
      }
    }
    int excl;
    const int tot = block_exclusive_scan(n, &excl, warp_tot);
    if (u < U) pp.unit_tiles[u] = carry_s + excl;
    __syncthreads();
    if (threadIdx.x == 0) carry_s += tot;
    __syncthreads();
  }
  const int64_t T = carry_s;
  __syncthreads();
  // pass 2: segments per unit (one per pair its tile range touches)
  if (threadIdx.x == 0) carry_s = 0;
  __syncthreads();
  for (int u0 = 0; u0 < U; u0 += 1024) {
    const int u = u0 + threadIdx.x;
    int nseg = 0, t0 = 0, t1 = 0;
    if (u < U) {
      t0 = pp.unit_tiles[u];
      t1 = (u + 1 < U) ? pp.unit_tiles[u + 1] : static_cast<int>(T);
      if (t1 > t0) nseg = pair_of(t1 - 1, T, pp.P) - pair_of(t0, T, pp.P) + 1;
    }
    int excl;
    const int tot = block_exclusive_scan(nseg, &excl, warp_tot);
    if (u < U) {
      const int s0 = carry_s + excl;
      pp.unit_seg[u] = s0;
      if (nseg > 0) {
        const int p0 = pair_of(t0, T, pp.P);
        for (int i = 0; i < nseg; ++i) {
          const int p = p0 + i;
          const int64_t a = max(static_cast<int64_t>(t0), pair_start(p, T, pp.P));
          const int64_t e = min(static_cast<int64_t>(t1), pair_start(p + 1, T, pp.P));
          AttnSeg sg;
          sg.unit = u;
          sg.tile_begin = static_cast<int32_t>(a - t0);
          sg.tile_end = static_cast<int32_t>(e - t0);
          sg.pair = p;
          if (s0 + i < pp.max_segs) pp.segs[s0 + i] = sg;
        }
      }
    }
    __syncthreads();
    if (threadIdx.x == 0) carry_s += tot;
    __syncthreads();
  }
  const int S = carry_s;
  if (threadIdx.x == 0) pp.unit_seg[U] = S;
  __syncthreads();
  // pass 3: first segment of every pair (segments are ordered by pair)
  for (int p = threadIdx.x; p <= pp.P; p += blockDim.x) {
    // binary search: first segment whose pair >= p
    int lo = 0, hi = S;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (pp.segs[mid].pair < p) lo = mid + 1; else hi = mid;
    }
    pp.pair_seg[p] = (p == pp.P) ? S : lo;
  }
}

// ------------------------------------------------------------------------ attention kernel

struct AttnShared {
  uint64_t tile_full[ATT_STAGES];
  uint64_t tile_empty[ATT_STAGES];
  uint64_t q_full, q_free, s_full, s_free, p_full, pv_done, o_free, drain;
  uint32_t tmem_base;
  volatile int abort_flag;
};

__device__ __forceinline__ bool att_wait(AttnShared& sh, uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (sh.abort_flag) return false;
    if (global_timer_ns() - t0 > MLA_WAIT_TIMEOUT_NS) {
      sh.abort_flag = 1;
      record_error(MLA_ERR_DEVICE_TIMEOUT);
      return false;
    }
  }
}

// Warp-uniform wait for the softmax warps (their TMEM loads/stores are warp-collective): lane 0
// waits, the verdict is broadcast, then every lane acquires the completed phase itself.
__device__ __forceinline__ bool att_warp_wait(AttnShared& sh, uint64_t* bar, uint32_t parity) {
  bool ok = false;
  if ((threadIdx.x & 31) == 0) ok = att_wait(sh, bar, parity);
  ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
  if (ok) (void)mbar_try_wait(bar, parity);
  return ok;
}

__global__ void __launch_bounds__(ATT_THREADS, 1)
mla_decode_attn_kernel(const __grid_constant__ CUtensorMap map_cache,
                       const __grid_constant__ CUtensorMap map_qhat, AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* stage_buf = smem;
  uint8_t* qs_buf = smem + ATT_STAGES * ATT_TILE_BYTES;
  uint8_t* p_buf = qs_buf + ATT_QS_CHUNKS * ATT_QS_CHUNK_BYTES;
  __shared__ AttnShared sh;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = blockIdx.x >> 1, half = blockIdx.x & 1;
  const int seg_begin = p.pair_seg[pair], seg_end = p.pair_seg[pair + 1];

  if (threadIdx.x == 0) {
    for (int s = 0; s < ATT_STAGES; ++s) {
      mbar_init(&sh.tile_full[s], 1);
      mbar_init(&sh.tile_empty[s], 1);
    }
    mbar_init(&sh.q_full, 1 + 4);
    mbar_init(&sh.q_free, 1);
    mbar_init(&sh.s_full, 1);
    mbar_init(&sh.s_free, 4);
    mbar_init(&sh.p_full, 4);
    mbar_init(&sh.pv_done, 1);
    mbar_init(&sh.o_free, 4);
    mbar_init(&sh.drain, 1);
    sh.abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&map_cache);
    tma_prefetch_desc(&map_qhat);
  }
  if (warp == 1) {
    tmem_alloc(&sh.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = sh.tmem_base;

  if (seg_begin < seg_end) {
    if (warp == 0) {
      if (lane == 0) {
        // =========================================================== TMA producer
        int g = 0;
        for (int k = 0, s_i = seg_begin; s_i < seg_end; ++k, ++s_i) {
          const AttnSeg sg = p.segs[s_i];
          const int b = sg.unit / p.n_mt, mt = sg.unit % p.n_mt;
          if (k >= 1 && !att_wait(sh, &sh.q_free, (k - 1) & 1)) break;
          mbar_arrive_expect_tx(&sh.q_full, ATT_QS_CHUNKS * ATT_QS_CHUNK_BYTES);
          const int qrow = b * p.R + mt * 128;
          for (int c = 0; c < ATT_QS_CHUNKS; ++c)
            tma_load_2d(qs_buf + c * ATT_QS_CHUNK_BYTES, &map_qhat, &sh.q_full,
                        ATT_QT_ELEMS + 64 * c, qrow);
          bool ok = true;
          for (int tile = sg.tile_begin; tile < sg.tile_end; ++tile, ++g) {
            const int st = g % ATT_STAGES;
            if (g >= ATT_STAGES && !att_wait(sh, &sh.tile_empty[st], ((g / ATT_STAGES) - 1) & 1)) {
              ok = false;
              break;
            }
            int page = p.block_table[static_cast<int64_t>(b) * p.max_pages + tile];
            if (page < 0 || page >= p.num_pages) {
              record_error(MLA_ERR_DEVICE_OOB);
              page = 0;
            }
            uint8_t* dst = stage_buf + st * ATT_TILE_BYTES;
            mbar_arrive_expect_tx(&sh.tile_full[st], ATT_TILE_BYTES);
            for (int c = 0; c < ATT_CHUNKS; ++c)
              tma_load_2d(dst + c * ATT_CHUNK_BYTES, &map_cache, &sh.tile_full[st], 64 * c,
                          page * ATT_PAGE);
          }
          if (!ok) break;
        }
        // drain: the last loads must land before the CTA can exit (bounded, abort or not)
        for (int j = max(0, g - ATT_STAGES); j < g; ++j)
          (void)mbar_wait(&sh.tile_full[j % ATT_STAGES], (j / ATT_STAGES) & 1);
      }
    } else if (warp == 1) {
      if (lane == 0) {
        // =========================================================== MMA issuer
        constexpr uint32_t IDESC_QK = idesc_bf16(128, 64, false, false);
        constexpr uint32_t IDESC_PV = idesc_bf16(128, 256, false, true);
        const uint32_t stage0 = smem_addr(stage_buf);
        const uint32_t qs0 = smem_addr(qs_buf);
        const uint32_t pb0 = smem_addr(p_buf);
        int g = 0;            // tile counter over the CTA's segments
        int pend_g = -1;      // tile whose PV is still to be issued
        int pend_k = 0;       // its segment counter
        bool pend_first = false;
        bool ok = true;
        auto issue_pv = [&](int gg, int kk_seg, bool first_of_seg) -> bool {
          if (first_of_seg && kk_seg >= 1 && !att_wait(sh, &sh.o_free, (kk_seg - 1) & 1))
            return false;
          if (!att_wait(sh, &sh.p_full, gg & 1)) return false;
          tc_fence_after_sync();
          const uint32_t st = stage0 + (gg % ATT_STAGES) * ATT_TILE_BYTES +
                              half * 4 * ATT_CHUNK_BYTES;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {   // 16 tokens per K-step
            mma_bf16_ss(tmem + TM_O, smem_desc_sw128(pb0 + kk * 32, 16, 1024),
                        smem_desc_sw128(st + kk * 2048, ATT_CHUNK_BYTES, 1024), IDESC_PV,
                        (first_of_seg && kk == 0) ? 0u : 1u);
          }
          mma_commit(&sh.tile_empty[gg % ATT_STAGES]);
          mma_commit(&sh.pv_done);
          return true;
        };
        for (int k = 0, s_i = seg_begin; ok && s_i < seg_end; ++k, ++s_i) {
          const AttnSeg sg = p.segs[s_i];
          if (!att_wait(sh, &sh.q_full, k & 1)) { ok = false; break; }
          for (int tile = sg.tile_begin; tile < sg.tile_end; ++tile, ++g) {
            if (g >= 1 && !att_wait(sh, &sh.s_free, (g - 1) & 1)) { ok = false; break; }
            if (!att_wait(sh, &sh.tile_full[g % ATT_STAGES], (g / ATT_STAGES) & 1)) { ok = false; break; }
            tc_fence_after_sync();
            const uint32_t st = stage0 + (g % ATT_STAGES) * ATT_TILE_BYTES;
            // S = Q̂ · Cᵀ over 36 K-steps of 16: Q̂[:, 0:384] from TMEM, Q̂[:, 384:576] from smem
#pragma unroll 4
            for (int ks = 0; ks < ATT_ROW / 16; ++ks) {
              const uint64_t bdesc =
                  smem_desc_sw128(st + (ks >> 2) * ATT_CHUNK_BYTES + (ks & 3) * 32, 16, 1024);
              if (ks < ATT_QT_ELEMS / 16) {
                mma_bf16_ts(tmem + TM_S, tmem + TM_Q + ks * 8, bdesc, IDESC_QK, ks > 0 ? 1u : 0u);
              } else {
                const int qk = ks - ATT_QT_ELEMS / 16;
                mma_bf16_ss(tmem + TM_S,
                            smem_desc_sw128(qs0 + (qk >> 2) * ATT_QS_CHUNK_BYTES + (qk & 3) * 32, 16, 1024),
                            bdesc, IDESC_QK, 1u);
              }
            }
            mma_commit(&sh.s_full);
            if (tile + 1 == sg.tile_end) mma_commit(&sh.q_free);
            if (pend_g >= 0 && !issue_pv(pend_g, pend_k, pend_first)) { ok = false; break; }
            pend_g = g;
            pend_k = k;
            pend_first = (tile == sg.tile_begin);
          }
        }
        if (ok && pend_g >= 0) issue_pv(pend_g, pend_k, pend_first);
        // drain: every MMA issued above completes before TMEM is released
        mma_commit(&sh.drain);
        (void)mbar_wait(&sh.drain, 0);
      }
    } else {
      // ============================================================ softmax warps
      const int quarter = warp & 3;
      const int r_local = quarter * 32 + lane;
      const uint32_t t_lane = static_cast<uint32_t>(quarter * 32) << 16;
      int g = 0;
      bool ok = true;
      // Q̂[:, 0:384] of a unit into TMEM (row r_local), zeros for rows past the unit.
      auto load_q_tmem = [&](const AttnSeg& sg) {
        const int b = sg.unit / p.n_mt, mt = sg.unit % p.n_mt;
        const int r_in = mt * 128 + r_local;
        const bool valid = r_in < p.R;
        const uint4* src = reinterpret_cast<const uint4*>(
            p.qhat + (static_cast<int64_t>(b) * p.R + r_in) * ATT_ROW);
#pragma unroll 1
        for (int c = 0; c < ATT_QT_ELEMS / 64; ++c) {
          uint32_t v[32];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            uint4 x = valid ? src[c * 8 + j] : make_uint4(0, 0, 0, 0);
            v[4 * j + 0] = x.x; v[4 * j + 1] = x.y; v[4 * j + 2] = x.z; v[4 * j + 3] = x.w;
          }
          tmem_st32(tmem + t_lane + TM_Q + c * 32, v);
        }
        tmem_st_wait();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.q_full);
      };
      if (true) load_q_tmem(p.segs[seg_begin]);
      for (int k = 0, s_i = seg_begin; ok && s_i < seg_end; ++k, ++s_i) {
        const AttnSeg sg = p.segs[s_i];
        const int b = sg.unit / p.n_mt, mt = sg.unit % p.n_mt;
        const int L = p.seq_lens[b];
        const int r_in = mt * 128 + r_local;
        const bool row_valid = r_in < p.R;
        const int t = row_valid ? r_in / p.H : 0;
        const int limit = L - p.Tq + t;     // last key this row may see
        float m_ref = -INFINITY, l_sum = 0.0f;
        for (int tile = sg.tile_begin; tile < sg.tile_end; ++tile, ++g) {
          if (!att_warp_wait(sh, &sh.s_full, g & 1)) { ok = false; break; }
          tc_fence_after_sync();
          uint32_t sr[64];
          {
            uint32_t (&a)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[0]);
            uint32_t (&c)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[32]);
            tmem_ld32(tmem + t_lane + TM_S, a);
            tmem_ld32(tmem + t_lane + TM_S + 32, c);
          }
          tmem_ld_wait();
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sh.s_free);
          // masked, base-2 scaled scores and their maximum
          const int j0 = tile * ATT_PAGE;
          const int jmax = row_valid ? min(limit, L - 1) : -1;   // inclusive
          float mt_max = -INFINITY;
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            const float s = (j0 + c <= jmax) ? __uint_as_float(sr[c]) * p.scale_log2 : -INFINITY;
            sr[c] = __float_as_uint(s);
            mt_max = fmaxf(mt_max, s);
          }
          float factor = 1.0f;
          bool rescale = false;
          if (mt_max > -INFINITY) {
            if (m_ref == -INFINITY) {
              m_ref = mt_max;
            } else if (mt_max > m_ref + ATT_RESCALE_THRESHOLD) {
              factor = exp2f(m_ref - mt_max);
              m_ref = mt_max;
              rescale = true;
            }
          }
          // previous PV must be done before P is overwritten or O is rescaled
          if (g >= 1 && !att_warp_wait(sh, &sh.pv_done, (g - 1) & 1)) { ok = false; break; }
          tc_fence_after_sync();
          if (__any_sync(0xffffffffu, rescale) && tile > sg.tile_begin) {
#pragma unroll 1
            for (int c0 = 0; c0 < 256; c0 += 32) {
              uint32_t o[32];
              tmem_ld32(tmem + t_lane + TM_O + c0, o);
              tmem_ld_wait();
#pragma unroll
              for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * factor);
              tmem_st32(tmem + t_lane + TM_O + c0, o);
            }
            tmem_st_wait();
          }
          l_sum *= factor;
          // P = 2^(s - m_ref) -> bf16, row r_local of the swizzled K-major P tile
          const float mref_use = (m_ref == -INFINITY) ? 0.0f : m_ref;
          float psum = 0.0f;
          uint8_t* prow = p_buf + r_local * 128;
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float x0 = exp2f(__uint_as_float(sr[ch * 8 + 2 * e]) - mref_use);
              const float x1 = exp2f(__uint_as_float(sr[ch * 8 + 2 * e + 1]) - mref_use);
              psum += x0 + x1;
              w[e] = pack_bf16x2(x0, x1);
            }
            *reinterpret_cast<uint4*>(prow + ((ch ^ (r_local & 7)) * 16)) =
                make_uint4(w[0], w[1], w[2], w[3]);
          }
          l_sum += psum;
          // rows past the sequence end must be zero in the value chunks (P is 0 there, but
          // stale cache contents could be non-finite)
          const int valid_tok = L - j0;
          if (valid_tok < ATT_PAGE) {
            if (!att_warp_wait(sh, &sh.tile_full[g % ATT_STAGES], (g / ATT_STAGES) & 1)) { ok = false; break; }
            uint8_t* vbase = stage_buf + (g % ATT_STAGES) * ATT_TILE_BYTES + half * 4 * ATT_CHUNK_BYTES;
            const int nrows = ATT_PAGE - valid_tok;
            for (int i = r_local; i < 4 * nrows * 8; i += 128) {
              const int chunk = i / (nrows * 8);
              const int rem = i % (nrows * 8);
              const int row = valid_tok + rem / 8, piece = rem % 8;
              *reinterpret_cast<uint4*>(vbase + chunk * ATT_CHUNK_BYTES + row * 128 + piece * 16) =
                  make_uint4(0, 0, 0, 0);
            }
          }
          fence_proxy_async_smem();
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sh.p_full);
        }
        if (!ok) break;
        const int seg_last_g = g - 1;
        // next segment's Q̂ goes into TMEM now: its QK may start before this epilogue ends
        if (s_i + 1 < seg_end) {
          if (!att_warp_wait(sh, &sh.q_free, k & 1)) { ok = false; break; }
          tc_fence_after_sync();
          load_q_tmem(p.segs[s_i + 1]);
        }
        // segment epilogue: O / l and the log-sum-exp
        if (!att_warp_wait(sh, &sh.pv_done, seg_last_g & 1)) { ok = false; break; }
        tc_fence_after_sync();
        const float inv_l = (l_sum > 0.0f) ? 1.0f / l_sum : 0.0f;
        float* dst = p.o_part + (static_cast<int64_t>(s_i) * 128 + r_local) * ATT_DC + half * 256;
#pragma unroll 1
        for (int c0 = 0; c0 < 256; c0 += 32) {
          uint32_t o[32];
          tmem_ld32(tmem + t_lane + TM_O + c0, o);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; j += 4)
            *reinterpret_cast<float4*>(dst + c0 + j) =
                make_float4(__uint_as_float(o[j]) * inv_l, __uint_as_float(o[j + 1]) * inv_l,
                            __uint_as_float(o[j + 2]) * inv_l, __uint_as_float(o[j + 3]) * inv_l);
        }
        if (half == 0)
          p.lse[static_cast<int64_t>(s_i) * 128 + r_local] =
              (l_sum > 0.0f) ? m_ref + log2f(l_sum) : -INFINITY;
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.o_free);
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------------ split-KV combine
// One warp per query row g = b*R + r: merge the row's partials (one per segment of its unit)
// by their base-2 log-sum-exp and store o_lat in bf16 (the B operand of the value projection).
__global__ void __launch_bounds__(256)
attn_combine_kernel(const float* __restrict__ o_part, const float* __restrict__ lse,
                    const int32_t* __restrict__ unit_seg, __nv_bfloat16* __restrict__ o_lat,
                    int n_rows, int R, int n_mt) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gr = blockIdx.x * 8 + warp;
  if (gr >= n_rows) return;
  const int b = gr / R, r = gr % R;
  const int u = b * n_mt + r / 128, rl = r % 128;
  const int s0 = unit_seg[u], s1 = unit_seg[u + 1];
  float mx = -INFINITY;
  for (int s = s0; s < s1; ++s) mx = fmaxf(mx, lse[static_cast<int64_t>(s) * 128 + rl]);
  float4 acc[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  float den = 0.0f;
  if (mx > -INFINITY) {
    for (int s = s0; s < s1; ++s) {
      const float w = exp2f(lse[static_cast<int64_t>(s) * 128 + rl] - mx);
      den += w;
      const float4* src = reinterpret_cast<const float4*>(o_part + (static_cast<int64_t>(s) * 128 + rl) * ATT_DC);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 v = src[lane + 32 * i];
        acc[i].x = fmaf(w, v.x, acc[i].x);
        acc[i].y = fmaf(w, v.y, acc[i].y);
        acc[i].z = fmaf(w, v.z, acc[i].z);
        acc[i].w = fmaf(w, v.w, acc[i].w);
      }
    }
  }
  const float inv = den > 0.0f ? 1.0f / den : 0.0f;
  uint2* dst = reinterpret_cast<uint2*>(o_lat + static_cast<int64_t>(gr) * ATT_DC);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    dst[lane + 32 * i] = make_uint2(pack_bf16x2(acc[i].x * inv, acc[i].y * inv),
                                    pack_bf16x2(acc[i].z * inv, acc[i].w * inv));
  }
}

}  // namespace mla
