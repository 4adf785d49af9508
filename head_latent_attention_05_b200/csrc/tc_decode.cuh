// Absorbed-MLA decode attention on tcgen05 (bf16 cache, d_c = 512, d_r = 64, 64-token pages).
//
// Work split. For sequence b the R = Tq*H query rows (row r = t*H + h) form ceil(R/128)
// "units" of 128 rows; every unit attends over the sequence's pages (tiles of 64 tokens). A
// planner (one extra block of the query-absorption GEMM) cuts the concatenated tile list of
// all units into P equal ranges, one per pair of CTAs, so long and short sequences spread
// evenly over the GPU (split-KV). Each range piece inside one unit is a "segment"; it produces
// a partial result (O / l, lse) that the value-projection kernel merges by log-sum-exp.
//
// One pair of CTAs per range. Both CTAs run the same token tiles: each computes the full
// score tile S = Q̂·Cᵀ (K = 576, heads on the MMA M side) and the same softmax, and accumulates
// its own half of the latent output O[:, half*256 : half*256+256] += P·C[:, half]. Splitting
// d_c keeps the fp32 accumulator within TMEM (256 columns per CTA). The pair shares nothing:
// exchanging partial scores through distributed shared memory instead of recomputing them
// measured slower on B200 (DSMEM moves ~8 bytes/clock per SM).
//
// Per CTA: TMEM columns [0,256) O half, [256,320) and [320,384) two score buffers S (tile g
// uses buffer g%2), [384,512) Q̂[:, 0:256] as bf16 pairs (the A operand of the first 16 K-steps
// of S). The softmax writes P (bf16) over the first 32 columns of its tile's S buffer, and P·C
// reads it from there (A from TMEM), so a score buffer is free again once P·C of its tile is
// done: the score MMAs of tile g+1 run while the softmax of tile g works, and the tensor pipe
// does not wait for it. Shared memory: 2 stages x 9 chunks of [64 tokens x 64 dims] (the whole
// 576-wide page, 128-byte swizzle, one TMA box per chunk), Q̂[:, 256:576] (5 chunks of
// [128 x 64]) and the barriers and row maxima (227 KB in all, no alignment slack: the dynamic
// shared memory starts 1024-byte aligned, which the kernel checks).
//
// Shared memory bandwidth, not the tensor pipe, sets the pace on B200: an A-from-smem N = 64
// K-step reads 6 KB and takes 48 cycles (128 B/clock), an A-from-TMEM one reads 2 KB and
// takes the MMA's own 32. Per tile a CTA moves ~256 KB through shared memory (72 KB of TMA
// writes, 152 KB of score operands, 32 KB of P·C operands), ~2000 cycles.
//
// Each stage is released in two parts: the 5 chunks only the score MMA reads (the other half's
// c_KV and k_R) as soon as S is computed, the 4 chunks of this CTA's c_KV half after P·C. The
// score MMA consumes the early chunks first, so the late chunks' load latency hides behind it.
//
// Warp roles (320 threads): warp 0 TMA producer, warp 1 issues every MMA (S of a tile, then
// P·C of the tile before; it stays converged and issues through elect.sync; a single issuer
// keeps the summation order, and the result, deterministic). A second issuing warp for P·C
// measured ~200 ns per tcgen05 instruction on B200 against ~36 ns in the score warp. Warps
// 2..5 and 6..9 run the softmax, rescale and epilogue: warp w owns TMEM lanes 32*(w%4)..
// (query rows), and the two warps of a lane quarter split each row's 64 scores (columns 0..31
// and 32..63), agreeing on the row maximum through shared memory once per tile.
// Online softmax in base 2 with a lazy rescale: the running maximum only moves (and O is
// rescaled) when a new score exceeds it by more than 2^8, which keeps every P <= 256.
#pragma once

#include <climits>
#include <type_traits>

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
constexpr int ATT_QT_ELEMS = 256;                 // Q̂ columns kept in TMEM
constexpr int ATT_QT_CHUNKS = ATT_QT_ELEMS / 64;  // 4
constexpr int ATT_QS_CHUNKS = (ATT_ROW - ATT_QT_ELEMS) / 64;   // 5 chunks of Q̂ in smem
constexpr int ATT_QS_CHUNK_BYTES = 128 * 128;     // [128 rows x 64 bf16]
constexpr int ATT_THREADS = 320;
constexpr int ATT_SM_WARPS = 8;                   // softmax warps: 2 per TMEM lane quarter
constexpr uint32_t TM_O = 0, TM_S = 256, TM_Q = 384;   // score buffer b at TM_S + 64*b
constexpr float ATT_RESCALE_THRESHOLD = 8.0f;     // log2 units

struct AttnSeg {
  int32_t unit;        // b * n_mt + mt
  int32_t tile_begin;  // first 64-token page of the segment (page index within the sequence)
  int32_t tile_end;    // one past the last
  int32_t pair;        // CTA pair that runs it
};

struct AttnParams {
  const int32_t* block_table;
  const int32_t* seq_lens;
  const AttnSeg* segs;
  const int32_t* pair_seg;   // [P + 1]: pair p runs segments [pair_seg[p], pair_seg[p+1])
  const __nv_bfloat16* qhat; // [B*R][576]
  __nv_bfloat16* o_part;     // [max_segs][128][512] per-segment O / l, rounded to bf16
  float* lse;                // [max_segs][128]   (base-2 log-sum-exp of the scaled scores)
  int max_pages, num_pages;
  int H, Tq, R, n_mt;
  float scale_log2;          // softmax_scale * log2(e)
  KeyRange keys;             // keys each query row may see (causal, window, key range)
  const uint8_t* cache8;     // fp8 kernel only: the quantised cache (its pages' scales),
  const uint8_t* qcodes;     //   the split query rows [B*R][1152] (qsplit_rows_kernel)
  const float* qalpha;       //   and their scales [B*R]
};

// ------------------------------------------------------------------------ split-KV planner

struct PlanParams {
  const int32_t* seq_lens;
  int B, Tq, H, n_mt, max_pos, P, max_segs;
  KeyRange keys;
  int32_t* unit_first;   // [U] scratch: first page of each unit's key range (by stream position)
  int32_t* unit_tiles;   // [U] scratch: first virtual tile of each unit (by stream position)
  int32_t* unit_seg;     // [U + 1] first segment of each unit (by stream position)
  int32_t* pair_seg;     // [P + 1]
  AttnSeg* segs;         // [max_segs]
};

constexpr int ATT_MAX_PAIRS = 1024;   // CTA pairs of the attention grid (one per two SMs)
constexpr int ATT_SEG_COST_TILES = 5;  // planner's price of one more segment, in tiles

// Start of pair p's tile range, p*T/P; the planner tabulates it once per call.
__device__ __forceinline__ int64_t pair_start(int p, int64_t T, int P) {
  return (static_cast<int64_t>(p) * T) / P;
}
// Largest p in [0, P) with ps[p] <= x (x in [0, T)), by bisection over the table ps.
__device__ __forceinline__ int pair_of(int64_t x, const int* ps, int P) {
  int lo = 0, hi = P - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (ps[mid] <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Block-wide exclusive scan of one int per thread (blockDim.x a multiple of 32, at most 1024);
// returns the total.
__device__ __forceinline__ int block_exclusive_scan(int v, int* excl, int* warp_tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int n_warps = static_cast<int>(blockDim.x >> 5);
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < n_warps ? warp_tot[lane] : 0;
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
  const int total = warp_tot[n_warps - 1];
  __syncthreads();
  return total;
}

// The planner, run by one whole block of any size (a multiple of 32): it rides along as an
// extra block of the query-absorption GEMM, which runs just before the attention kernel.
//
// Pages of a unit. A unit's rows are query tokens t0..t1 of one sequence (all heads of each);
// the unit covers the pages from the one holding the first key its first token sees to the one
// holding the last key its last token sees (visible_keys: causal, window, key range), so a
// prefill's early tokens and a windowed decode skip the pages none of their rows can see.
//
// Order. Units are laid out in the stream query-tile major: position i = mt * B + b holds
// unit (b, mt) (unit_stream_pos). The units of one sequence cover nearly the same pages, so
// cutting this stream into equal ranges gives the pairs of every query tile the same relative
// position in their part: pair j of tile 0 and pair j of tile 1 stream the same pages at the
// same time, and the second read of each page comes from L2 instead of HBM. Everything the
// planner writes per unit (unit_first, unit_tiles, unit_seg) is indexed by stream position;
// a segment's `unit` field holds the unit itself, b * n_mt + mt.
//
// Balance. A CTA pair pays a fixed price each time it moves on to another unit (the finished
// segment's epilogue and the next unit's Q̂ load lie on its critical path; measured at about
// five tiles' worth on B200). So the tile list is cut in a virtual stream in which every unit
// is followed by a gap of ATT_SEG_COST_TILES tiles: unit u occupies [vs_u, vs_u + n_u) with
// vs_u = (tiles of units before u) + ATT_SEG_COST_TILES * u, and pair p takes the virtual range
// [p*V/P, (p+1)*V/P). A pair whose range crosses into another unit then gets correspondingly
// fewer tiles, and every pair carries about the same cost.
__device__ __noinline__ void attn_plan_block(const PlanParams& pp) {
  __shared__ int warp_tot[32];
  __shared__ int carry_s;
  __shared__ int ps[ATT_MAX_PAIRS + 1];          // virtual start of pair p's range, p = 0..P
  __shared__ int first_seg[ATT_MAX_PAIRS + 1];   // lowest segment index of each pair
  constexpr int C = ATT_SEG_COST_TILES;
  const int U = pp.B * pp.n_mt;
  const int nt = static_cast<int>(blockDim.x);
  // pass 1: tiles per unit -> virtual unit starts (u: stream position)
  if (threadIdx.x == 0) carry_s = 0;
  __syncthreads();
  for (int u0 = 0; u0 < U; u0 += nt) {
    const int u = u0 + threadIdx.x;
    int n = 0;
    if (u < U) {
      const int b = u % pp.B, mt = u / pp.B;
      const int L = pp.seq_lens[b];
      int first = 0;
      if (L >= pp.Tq && L <= pp.max_pos) {
        const int t0 = (mt * 128) / pp.H;
        const int t1 = min(pp.Tq - 1, (mt * 128 + 127) / pp.H);
        int lo0, hi0, lo1, hi1;
        visible_keys(pp.keys, b, L, pp.Tq, t0, &lo0, &hi0);
        visible_keys(pp.keys, b, L, pp.Tq, t1, &lo1, &hi1);
        if (hi1 >= lo0) {
          first = lo0 / ATT_PAGE;
          n = hi1 / ATT_PAGE + 1 - first;
        }
      } else if (mt == 0) {
        record_error(MLA_ERR_DEVICE_BAD_LENGTH);
      }
      pp.unit_first[u] = first;
    }
    int excl;
    const int tot = block_exclusive_scan(n, &excl, warp_tot);
    if (u < U) pp.unit_tiles[u] = carry_s + excl + C * u;
    __syncthreads();
    if (threadIdx.x == 0) carry_s += tot;
    __syncthreads();
  }
  const int V = carry_s + C * U;   // virtual length: all tiles and one gap per unit
  for (int p = threadIdx.x; p <= pp.P; p += nt) {
    ps[p] = static_cast<int>(pair_start(p, V, pp.P));
    first_seg[p] = INT_MAX;
  }
  __syncthreads();
  // pass 2: segments per unit: one per pair whose range meets the unit's virtual range
  if (threadIdx.x == 0) carry_s = 0;
  __syncthreads();
  for (int u0 = 0; u0 < U; u0 += nt) {
    const int u = u0 + threadIdx.x;
    int nseg = 0, v0 = 0, v1 = 0, p0 = 0, p1 = -1;
    if (u < U) {
      v0 = pp.unit_tiles[u];
      v1 = ((u + 1 < U) ? pp.unit_tiles[u + 1] : V) - C;   // end of this unit's tiles
      if (v1 > v0) {
        p0 = pair_of(v0, ps, pp.P);
        p1 = pair_of(v1 - 1, ps, pp.P);
        for (int p = p0; p <= p1; ++p) nseg += min(v1, ps[p + 1]) > max(v0, ps[p]) ? 1 : 0;
      }
    }
    int excl;
    const int tot = block_exclusive_scan(nseg, &excl, warp_tot);
    if (u < U) {
      const int s0 = carry_s + excl;
      pp.unit_seg[u] = s0;
      int i = 0;
      for (int p = p0; p <= p1; ++p) {
        const int a = max(v0, ps[p]);
        const int e = min(v1, ps[p + 1]);
        if (e <= a) continue;
        AttnSeg sg;
        sg.unit = (u % pp.B) * pp.n_mt + u / pp.B;
        sg.tile_begin = pp.unit_first[u] + (a - v0);
        sg.tile_end = pp.unit_first[u] + (e - v0);
        sg.pair = p;
        if (s0 + i < pp.max_segs) pp.segs[s0 + i] = sg;
        atomicMin(&first_seg[p], s0 + i);
        ++i;
      }
    }
    __syncthreads();
    if (threadIdx.x == 0) carry_s += tot;
    __syncthreads();
  }
  const int S = carry_s;
  if (threadIdx.x == 0) pp.unit_seg[U] = S;
  // pass 3: segments are ordered by pair; a pair without segments starts where the next pair
  // that has some starts, and pair_seg[P] = S closes the list
  for (int p = threadIdx.x; p <= pp.P; p += nt) {
    int q = p;
    while (q < pp.P && first_seg[q] == INT_MAX) ++q;
    pp.pair_seg[p] = (q < pp.P) ? first_seg[q] : S;
  }
}

// ------------------------------------------------------------------------ attention kernel

struct AttnShared {
  uint64_t full_qk[ATT_STAGES], full_own[ATT_STAGES];    // stage chunks landed (TMA)
  uint64_t empty_qk[ATT_STAGES], empty_own[ATT_STAGES];  // stage chunks free again (MMA commit)
  uint64_t s_full[2], p_full[2], pv_done[2];             // per score buffer (tile parity)
  uint64_t q_full;                 // the softmax warps wrote a unit's Q̂[:, 0:256] into TMEM
  uint64_t qs_full;                // the unit's Q̂[:, 256:576] landed in shared memory (TMA)
  uint64_t q_free, o_free, drain;
  uint64_t pair_bar[4];            // the two softmax warps of a lane quarter meet here
  // [tile parity][column half][row] partial row maxima; a segment's partial row sums reuse
  // the slot of the parity after its last tile
  float row_max[2][2][128];
  uint32_t tmem_base;
  volatile int abort_flag;
};

constexpr int ATT_SMEM_BYTES = ATT_STAGES * ATT_TILE_BYTES + ATT_QS_CHUNKS * ATT_QS_CHUNK_BYTES +
                               static_cast<int>(sizeof(AttnShared));
static_assert(ATT_SMEM_BYTES <= 227 * 1024, "attention kernel exceeds the shared memory of a CTA");

template <class SH>
__device__ __forceinline__ bool att_wait(SH& sh, uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (sh.abort_flag) return false;
    if (global_timer_ns() - t0 > MLA_PIPE_WAIT_NS) {
      sh.abort_flag = 1;
      record_error(MLA_ERR_DEVICE_TIMEOUT);
      return false;
    }
  }
}

// Warp-uniform wait for the softmax warps (their TMEM loads/stores are warp-collective): lane 0
// waits, the verdict is broadcast, then every lane acquires the completed phase itself.
template <class SH>
__device__ __forceinline__ bool att_warp_wait(SH& sh, uint64_t* bar, uint32_t parity) {
  bool ok = false;
  if ((threadIdx.x & 31) == 0) ok = att_wait(sh, bar, parity);
  ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
  if (ok) (void)mbar_try_wait(bar, parity);
  return ok;
}

// Walks the tiles of a CTA's segments in order: (segment index, tile within the unit).
struct TileCursor {
  const AttnSeg* segs;
  int s_i, s_end, tile, k;   // k: segment counter (0-based) within the CTA
  AttnSeg sg;
  __device__ void init(const AttnSeg* sg_ptr, int begin, int end) {
    segs = sg_ptr; s_i = begin; s_end = end; k = 0;
    if (s_i < s_end) { sg = segs[s_i]; tile = sg.tile_begin; }
  }
  __device__ bool valid() const { return s_i < s_end; }
  __device__ bool first_of_seg() const { return tile == sg.tile_begin; }
  __device__ bool last_of_seg() const { return tile + 1 == sg.tile_end; }
  __device__ void next() {
    if (++tile >= sg.tile_end) {
      ++s_i; ++k;
      if (s_i < s_end) { sg = segs[s_i]; tile = sg.tile_begin; }
    }
  }
};

// The score MMA consumes a tile's chunks in two parts: first the 5 chunks only it needs (the
// other half's 4 c_KV chunks, then k_R = chunk 8), then this CTA's own 4 c_KV chunks.

// Score K-steps over a run of consecutive chunks c .. c+n-1 of a tile into the score buffer at
// TMEM column d_s. In the A-from-TMEM form (chunks 0..3: Q̂[:, 0:256] sits in TMEM) and the
// A-from-smem form (chunks 4..8, Q̂[:, 256:576]). Each run is a short loop whose descriptors
// only step by constants: the issuing warp shares the instruction cache with the producer, P·C
// and softmax code (a fully unrolled tile costs more overall), and per-chunk index arithmetic
// or branching measured ~20 cycles per MMA.
__device__ __forceinline__ void att_qk_ts(uint32_t tmem, uint32_t d_s, uint64_t b_stage, int c,
                                          int n, bool first) {
  constexpr uint32_t IDESC_QK = idesc_bf16(128, 64, false, false);
  uint64_t b0 = b_stage + static_cast<uint64_t>((c * ATT_CHUNK_BYTES) >> 4);
  uint32_t a0 = tmem + TM_Q + c * 32;
#pragma unroll 1
  for (int i = 0; i < n; ++i, b0 += ATT_CHUNK_BYTES >> 4, a0 += 32)
    mma_bf16_ts_x4_elect(tmem + d_s, a0, b0, IDESC_QK, (first && i == 0) ? 0u : 1u);
}
__device__ __forceinline__ void att_qk_ss(uint32_t tmem, uint32_t d_s, uint64_t b_stage,
                                          uint64_t qs_desc, int c, int n, bool first) {
  constexpr uint32_t IDESC_QK = idesc_bf16(128, 64, false, false);
  uint64_t b0 = b_stage + static_cast<uint64_t>((c * ATT_CHUNK_BYTES) >> 4);
  uint64_t a0 =
      qs_desc + static_cast<uint64_t>(((c - ATT_QT_CHUNKS) * ATT_QS_CHUNK_BYTES) >> 4);
#pragma unroll 1
  for (int i = 0; i < n; ++i, b0 += ATT_CHUNK_BYTES >> 4, a0 += ATT_QS_CHUNK_BYTES >> 4)
    mma_bf16_ss_x4_elect(tmem + d_s, a0, b0, IDESC_QK, (first && i == 0) ? 0u : 1u);
}
// The score-only chunks of a tile: half 0 reads chunks 4..7 | 8, half 1 chunks 0..3 | 8; the
// tile's first K-step overwrites S.
__device__ __forceinline__ void att_qk_score_only(uint32_t tmem, uint32_t d_s, uint64_t b_stage,
                                                  uint64_t qs_desc, int half) {
  if (half == 0) {
    att_qk_ss(tmem, d_s, b_stage, qs_desc, 4, 5, true);
  } else {
    att_qk_ts(tmem, d_s, b_stage, 0, 4, true);
    att_qk_ss(tmem, d_s, b_stage, qs_desc, 8, 1, false);
  }
}
// This CTA's own chunks: half 0 chunks 0..3, half 1 chunks 4..7.
__device__ __forceinline__ void att_qk_own(uint32_t tmem, uint32_t d_s, uint64_t b_stage,
                                           uint64_t qs_desc, int half) {
  if (half == 0) att_qk_ts(tmem, d_s, b_stage, 0, 4, false);
  else att_qk_ss(tmem, d_s, b_stage, qs_desc, 4, 4, false);
}

__global__ void __launch_bounds__(ATT_THREADS, 1)
mla_decode_attn_kernel(const __grid_constant__ CUtensorMap map_cache,
                       const __grid_constant__ CUtensorMap map_cache4,
                       const __grid_constant__ CUtensorMap map_qhat, AttnParams p) {
  // no static shared memory: the dynamic buffer starts at the CTA's (1024-byte aligned) shared
  // window, which the 128-byte swizzle of the TMA boxes and MMA descriptors needs
  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_addr(smem) & 1023u) != 0) {   // uniform over the CTA: nothing has started yet
    if (threadIdx.x == 0) record_error(MLA_ERR_UNSUPPORTED);
    return;
  }
  uint8_t* stage_buf = smem;   // chunk c of stage s at stage_buf + s*TILE + c*CHUNK
  uint8_t* qs_buf = smem + ATT_STAGES * ATT_TILE_BYTES;
  AttnShared& sh =
      *reinterpret_cast<AttnShared*>(qs_buf + ATT_QS_CHUNKS * ATT_QS_CHUNK_BYTES);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = blockIdx.x >> 1, half = blockIdx.x & 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < ATT_STAGES; ++s) {
      mbar_init(&sh.full_qk[s], 1);
      mbar_init(&sh.full_own[s], 1);
      mbar_init(&sh.empty_qk[s], 1);
      mbar_init(&sh.empty_own[s], 1);   // committed after the stage's P·C
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sh.s_full[b], 1);
      mbar_init(&sh.p_full[b], ATT_SM_WARPS);
      mbar_init(&sh.pv_done[b], 1);
    }
    mbar_init(&sh.q_full, ATT_SM_WARPS);
    mbar_init(&sh.qs_full, 1);
    mbar_init(&sh.q_free, 1);
    mbar_init(&sh.o_free, ATT_SM_WARPS);
    mbar_init(&sh.drain, 1);
    for (int q = 0; q < 4; ++q) mbar_init(&sh.pair_bar[q], 2);
    sh.abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&map_cache);
    tma_prefetch_desc(&map_cache4);
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
  pdl_wait();   // the plan and Q̂ of the previous kernel are complete and visible from here on
  pdl_trigger();
  const int seg_begin = p.pair_seg[pair], seg_end = p.pair_seg[pair + 1];

  if (seg_begin < seg_end) {
    if (warp == 0) {
      if (lane == 0) {
        // =========================================================== TMA producer
        // Two cursors: the score-only chunks run one tile ahead of this CTA's own chunks,
        // because their slots free up earlier (after S instead of after P·C).
        auto page_of = [&](const TileCursor& c) {
          const int b = c.sg.unit / p.n_mt;
          int page = p.block_table[static_cast<int64_t>(b) * p.max_pages + c.tile];
          if (page < 0 || page >= p.num_pages) {
            record_error(MLA_ERR_DEVICE_OOB);
            page = 0;
          }
          return page;
        };
        // A page's chunks c..c+3 come in one box of the 3-D view [chunk][token][64 dims] (TMA
        // instructions are slow to issue, so fewer, larger boxes), the rope chunk 8 in its own.
        auto load_chunks = [&](const TileCursor& c, int g, bool own, uint64_t* bar) {
          const int page = page_of(c);
          uint8_t* st = stage_buf + (g % ATT_STAGES) * ATT_TILE_BYTES;
          const int c0 = own ? 4 * half : 4 * (1 - half);
          mbar_arrive_expect_tx(bar, (own ? 4 : 5) * ATT_CHUNK_BYTES);
          tma_load_3d(st + c0 * ATT_CHUNK_BYTES, &map_cache4, bar, 0, page * ATT_PAGE, c0);
          if (!own)
            tma_load_2d(st + 8 * ATT_CHUNK_BYTES, &map_cache, bar, 64 * 8, page * ATT_PAGE);
        };
        int n_qloads = 0;   // Q̂ loads issued: the last one is drained before the CTA leaves
        auto load_q_smem = [&](const AttnSeg& sg) {   // Q̂[:, 256:576] of a unit
          const int b = sg.unit / p.n_mt, mt = sg.unit % p.n_mt;
          mbar_arrive_expect_tx(&sh.qs_full, ATT_QS_CHUNKS * ATT_QS_CHUNK_BYTES);
          for (int c = 0; c < ATT_QS_CHUNKS; ++c)
            tma_load_2d(qs_buf + c * ATT_QS_CHUNK_BYTES, &map_qhat, &sh.qs_full,
                        ATT_QT_ELEMS + 64 * c, b * p.R + mt * 128);
          ++n_qloads;
        };
        // Step for tile g: its own chunks, then (new segment at g+1) the next Q̂, then the
        // score-only chunks of tile g+1. Own chunks of g wait for P·C of g-2; score-only chunks
        // of g+1 wait for S of g-1, which completes earlier, so neither load delays the other.
        // (No L2 prefetch of pages ahead of these loads: the TMA engine that would issue it is
        // the one these loads wait on, and on B200 it measured no faster with it.)
        TileCursor cq, co;   // score-only cursor (one tile ahead), own-chunk cursor
        cq.init(p.segs, seg_begin, seg_end);
        co.init(p.segs, seg_begin, seg_end);
        // Q̂ rows of this pair's later segments into L2 now, so that switching units later
        // reads them from L2 rather than HBM
        if (half == 0) {
          for (int s_i = seg_begin + 1; s_i < seg_end; ++s_i) {
            const AttnSeg sg = p.segs[s_i];
            const int b = sg.unit / p.n_mt, mt = sg.unit % p.n_mt;
            const int rows = min(128, p.R - mt * 128);
            prefetch_l2_bulk(p.qhat + (static_cast<int64_t>(b) * p.R + mt * 128) * ATT_ROW,
                             static_cast<uint32_t>(rows * ATT_ROW * 2));
          }
        }
        int gq = 0, go = 0;
        bool ok = true;
        load_q_smem(cq.sg);
        load_chunks(cq, gq, false, &sh.full_qk[0]);
        cq.next();
        ++gq;
        while (ok && co.valid()) {
          int st = go % ATT_STAGES;
          if (go >= ATT_STAGES && !att_wait(sh, &sh.empty_own[st], ((go / ATT_STAGES) - 1) & 1)) {
            ok = false;
            break;
          }
          load_chunks(co, go, true, &sh.full_own[st]);
          const bool seg_ends = co.last_of_seg();
          const int k_done = co.k;
          co.next();
          ++go;
          if (!cq.valid()) continue;
          if (seg_ends) {   // Q̂ smem of the next segment: the last S of this one must be done
            if (!att_wait(sh, &sh.q_free, k_done & 1)) { ok = false; break; }
            load_q_smem(cq.sg);
          }
          st = gq % ATT_STAGES;
          if (gq >= ATT_STAGES && !att_wait(sh, &sh.empty_qk[st], ((gq / ATT_STAGES) - 1) & 1)) {
            ok = false;
            break;
          }
          load_chunks(cq, gq, false, &sh.full_qk[st]);
          cq.next();
          ++gq;
        }
        // drain: the last loads must land before the CTA can exit (bounded, abort or not); a
        // Q̂ load is issued only after the score MMAs consumed the one before, so only the last
        // can still be in flight, and likewise for each stage's two rings
        if (n_qloads > 0) (void)mbar_wait(&sh.qs_full, (n_qloads - 1) & 1);
        for (int j = max(0, gq - ATT_STAGES); j < gq; ++j)
          (void)mbar_wait(&sh.full_qk[j % ATT_STAGES], (j / ATT_STAGES) & 1);
        for (int j = max(0, go - ATT_STAGES); j < go; ++j)
          (void)mbar_wait(&sh.full_own[j % ATT_STAGES], (j / ATT_STAGES) & 1);
      }
    } else if (warp == 1) {
      {
        // ======================================== MMA issuer: S of tile g, then P·C of g-1
        // (the whole warp runs this loop; one elected lane issues each MMA and commit). One
        // warp issues both streams in this order: S(g) needs only P·C(g-2) done (its score
        // buffer), and the softmax of g-1 overlaps S(g); P·C(g-1) follows as soon as P(g-1)
        // is in TMEM. (Issuing P·C(g-1) between the two parts of S(g) measured no faster: the
        // tensor pipe runs its queue in order.)
        constexpr uint32_t IDESC_PV = idesc_bf16(128, 256, false, true);
        const uint32_t stage0 = smem_addr(stage_buf);
        const uint64_t qs_desc = smem_desc_sw128(smem_addr(qs_buf), 16, 1024);
        // O_half += P · C[:, own half] for tile gv: P (bf16 pairs) from the tile's score buffer
        // in TMEM, chunks 4*half .. 4*half+3 of its stage read MN-major (N = 256); the first
        // tile of a segment (k-th of this CTA) overwrites O once the last epilogue has read it
        auto issue_pv = [&](int gv, bool first_v, int kv) -> bool {
          const int st = gv % ATT_STAGES, sb = gv & 1;
          if (first_v && kv >= 1 && !att_warp_wait(sh, &sh.o_free, (kv - 1) & 1)) return false;
          if (!att_warp_wait(sh, &sh.p_full[sb], (gv >> 1) & 1)) return false;
          tc_fence_after_sync();
          const uint64_t b0 = smem_desc_sw128(
              stage0 + st * ATT_TILE_BYTES + half * 4 * ATT_CHUNK_BYTES, ATT_CHUNK_BYTES, 1024);
          const uint32_t a_p = tmem + TM_S + 64 * sb;
          // 4 K-steps of 16 tokens (8 TMEM columns of P, 16 rows of the chunks)
          mma_bf16_ts_mn_x4_elect(tmem + TM_O, a_p, b0, IDESC_PV, first_v ? 0u : 1u);
          // (tracks every earlier MMA of this thread: the stage's own chunks are free after it)
          mma_commit_elect(&sh.empty_own[st]);
          mma_commit_elect(&sh.pv_done[sb]);
          return true;
        };
        TileCursor cur;
        cur.init(p.segs, seg_begin, seg_end);
        bool ok = true, prev_first = false;
        int g = 0, prev_k = 0;
        for (; cur.valid(); ++g, cur.next()) {
          const int st = g % ATT_STAGES, sb = g & 1;
          const uint32_t d_s = TM_S + 64 * sb;
          if (cur.first_of_seg() && (!att_warp_wait(sh, &sh.q_full, cur.k & 1) ||
                                     !att_warp_wait(sh, &sh.qs_full, cur.k & 1))) {
            ok = false;
            break;
          }
          // score buffer sb held P of tile g-2: free once P·C of that tile is done
          if (g >= 2 && !att_warp_wait(sh, &sh.pv_done[sb], ((g >> 1) - 1) & 1)) { ok = false; break; }
          const uint64_t b_stage = smem_desc_sw128(stage0 + st * ATT_TILE_BYTES, 16, 1024);
          // S over the score-only chunks first, then this CTA's own chunks
          if (!att_warp_wait(sh, &sh.full_qk[st], (g / ATT_STAGES) & 1)) { ok = false; break; }
          tc_fence_after_sync();
          att_qk_score_only(tmem, d_s, b_stage, qs_desc, half);
          mma_commit_elect(&sh.empty_qk[st]);   // arrives once these MMAs have read their chunks
          if (!att_warp_wait(sh, &sh.full_own[st], (g / ATT_STAGES) & 1)) { ok = false; break; }
          tc_fence_after_sync();
          att_qk_own(tmem, d_s, b_stage, qs_desc, half);
          mma_commit_elect(&sh.s_full[sb]);
          if (cur.last_of_seg()) mma_commit_elect(&sh.q_free);
          if (g >= 1 && !issue_pv(g - 1, prev_first, prev_k)) { ok = false; break; }
          prev_first = cur.first_of_seg();
          prev_k = cur.k;
        }
        if (ok && g >= 1) (void)issue_pv(g - 1, prev_first, prev_k);
        // drain: every MMA issued above completes before TMEM is released
        mma_commit_elect(&sh.drain);
        if (lane == 0) (void)mbar_wait(&sh.drain, 0);
        __syncwarp();
      }
    } else {
      // ============================================================ softmax warps
      // Warps 2..5 take score columns 0..31, warps 6..9 columns 32..63 of the same rows (each
      // group covers the four TMEM lane quarters, warp w reading lanes 32*(w%4)..).
      const int hc = warp >= 6 ? 1 : 0;   // column half of the score tile
      const int quarter = warp & 3;
      const int r_local = quarter * 32 + lane;
      const int t_idx = hc * 128 + r_local;   // 0..255 among the softmax threads
      const uint32_t t_lane = static_cast<uint32_t>(quarter * 32) << 16;
      int g = 0, xc = 0;   // tile counter, partner-exchange counter
      bool ok = true;
      // both warps of this lane quarter have published their partial: a bounded meeting
      auto meet = [&]() -> bool {
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.pair_bar[quarter]);
        const bool r = att_warp_wait(sh, &sh.pair_bar[quarter], xc & 1);
        ++xc;
        return r;
      };
      // Q̂[:, 0:256] of a unit into TMEM (row r_local), zeros for rows past the unit; each warp
      // of the pair writes 2 of the 4 column groups.
      auto load_q_tmem = [&](const AttnSeg& sg) {
        const int b = sg.unit / p.n_mt, mt = sg.unit % p.n_mt;
        const int r_in = mt * 128 + r_local;
        const bool valid = r_in < p.R;
        const uint4* src = reinterpret_cast<const uint4*>(
            p.qhat + (static_cast<int64_t>(b) * p.R + r_in) * ATT_ROW);
        uint32_t v[32];
#pragma unroll 1
        for (int c = hc * (ATT_QT_CHUNKS / 2); c < (hc + 1) * (ATT_QT_CHUNKS / 2); ++c) {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint4 x = valid ? src[c * 8 + j] : make_uint4(0, 0, 0, 0);
            v[4 * j + 0] = x.x; v[4 * j + 1] = x.y; v[4 * j + 2] = x.z; v[4 * j + 3] = x.w;
          }
          tmem_st32(tmem + t_lane + TM_Q + c * 32, v);
        }
        tmem_st_wait();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.q_full);
      };
      load_q_tmem(p.segs[seg_begin]);
      for (int k = 0, s_i = seg_begin; ok && s_i < seg_end; ++k, ++s_i) {
        const AttnSeg sg = p.segs[s_i];
        const int b = sg.unit / p.n_mt, mt = sg.unit % p.n_mt;
        const int L = p.seq_lens[b];
        const int r_in = mt * 128 + r_local;
        const bool row_valid = r_in < p.R;
        // keys this row sees (lo > hi: none), and the union over the unit's rows
        int lo_row = 1, hi_row = 0, lo_u, hi_u, unused;
        if (row_valid) visible_keys(p.keys, b, L, p.Tq, r_in / p.H, &lo_row, &hi_row);
        visible_keys(p.keys, b, L, p.Tq, (mt * 128) / p.H, &lo_u, &unused);
        visible_keys(p.keys, b, L, p.Tq, min(p.Tq - 1, (mt * 128 + 127) / p.H), &unused, &hi_u);
        float m_ref = -INFINITY, l_part = 0.0f;
        for (int tile = sg.tile_begin; tile < sg.tile_end; ++tile, ++g) {
          const int sb = g & 1;
          const uint32_t s_col = TM_S + 64 * sb;
          if (!att_warp_wait(sh, &sh.s_full[sb], (g >> 1) & 1)) { ok = false; break; }
          tc_fence_after_sync();
          uint32_t sr[32];
          tmem_ld32(tmem + t_lane + s_col + hc * 32, sr);
          tmem_ld_wait();
          tc_fence_before_sync();   // the partner's P store into these columns follows the meeting
          // this thread's visible columns: c_lo .. c_hi of its 32 (none if c_lo > c_hi)
          const int j0 = tile * ATT_PAGE + hc * 32;
          const int c_lo = max(0, lo_row - j0), c_hi = min(31, hi_row - j0);
          const bool all_vis = c_lo == 0 && c_hi == 31;
          float mx0 = -INFINITY, mx1 = -INFINITY;
          if (all_vis) {
#pragma unroll
            for (int c = 0; c < 32; c += 4) {
              mx0 = fmax3(mx0, __uint_as_float(sr[c]), __uint_as_float(sr[c + 1]));
              mx1 = fmax3(mx1, __uint_as_float(sr[c + 2]), __uint_as_float(sr[c + 3]));
            }
          } else {
#pragma unroll
            for (int c = 0; c < 32; c += 2) {
              mx0 = fmaxf(mx0, (c >= c_lo && c <= c_hi) ? __uint_as_float(sr[c]) : -INFINITY);
              mx1 = fmaxf(mx1, (c + 1 >= c_lo && c + 1 <= c_hi) ? __uint_as_float(sr[c + 1])
                                                                 : -INFINITY);
            }
          }
          // agree on the row maximum with the partner warp (same rows, other 32 columns); after
          // this meeting both warps hold their S columns in registers, so P may overwrite S
          sh.row_max[g & 1][hc][r_local] = fmaxf(mx0, mx1);
          if (!meet()) { ok = false; break; }
          tc_fence_after_sync();
          const float raw_max = fmaxf(sh.row_max[g & 1][0][r_local], sh.row_max[g & 1][1][r_local]);
          const float mt_max = raw_max > -INFINITY ? raw_max * p.scale_log2 : -INFINITY;
          float factor = 1.0f;
          bool rescale = false;
          if (mt_max > -INFINITY) {
            if (m_ref == -INFINITY) {
              m_ref = mt_max;
            } else if (mt_max > m_ref + ATT_RESCALE_THRESHOLD) {
              factor = fast_exp2(m_ref - mt_max);
              m_ref = mt_max;
              rescale = true;
            }
          }
          // P·C of the previous tile must be done before O is rescaled
          if (g >= 1 && !att_warp_wait(sh, &sh.pv_done[(g - 1) & 1], ((g - 1) >> 1) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          if (__any_sync(0xffffffffu, rescale) && tile > sg.tile_begin) {
#pragma unroll 1
            for (int c0 = hc * 128; c0 < hc * 128 + 128; c0 += 32) {
              uint32_t o[32];
              tmem_ld32(tmem + t_lane + TM_O + c0, o);
              tmem_ld_wait();
#pragma unroll
              for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * factor);
              tmem_st32(tmem + t_lane + TM_O + c0, o);
            }
            tmem_st_wait();
          }
          l_part *= factor;
          // P = 2^(scale*s - m_ref) -> bf16 (0 for hidden columns): this thread's 32 keys of row
          // r_local as 16 bf16 pairs over TMEM columns hc*16.. of the tile's score buffer (key
          // j of the tile in column j/2, the even key in the low half), the A operand of P·C
          // (pairs of columns in f32x2 arithmetic: the even and odd columns' exponent arguments
          // and partial sums, each lane rounded as its scalar form would be)
          const float neg_m = (m_ref == -INFINITY) ? 0.0f : -m_ref;
          const float sc = p.scale_log2;
          const uint64_t sc2 = f2_pack(sc, sc), nm2 = f2_pack(neg_m, neg_m);
          uint64_t ps2 = f2_pack(0.0f, 0.0f);
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int c = 2 * e;
            float x0, x1;
            f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), sc2, nm2),
                      x0, x1);
            x0 = fast_exp2(x0);
            x1 = fast_exp2(x1);
            if (!all_vis) {
              x0 = (c >= c_lo && c <= c_hi) ? x0 : 0.0f;
              x1 = (c + 1 >= c_lo && c + 1 <= c_hi) ? x1 : 0.0f;
            }
            ps2 = f2_add(ps2, f2_pack(x0, x1));
            w[e] = pack_bf16x2(x0, x1);
          }
          tmem_st16(tmem + t_lane + s_col + hc * 16, w);
          float ps0, ps1;
          f2_unpack(ps2, ps0, ps1);
          l_part += ps0 + ps1;
          // rows outside the keys any row of the unit sees must be zero in the value chunks
          // (P is 0 there, but stale slots past the sequence end, or slots outside a key range,
          // could hold non-finite values); S is done, so they have landed. Kept: [z_lo, z_keep).
          const int z_lo = min(ATT_PAGE, max(0, lo_u - tile * ATT_PAGE));
          const int z_keep = max(z_lo, min(ATT_PAGE, hi_u + 1 - tile * ATT_PAGE));
          const int nz = z_lo + (ATT_PAGE - z_keep);
          if (nz > 0) {
            uint8_t* vbase = stage_buf + (g % ATT_STAGES) * ATT_TILE_BYTES + half * 4 * ATT_CHUNK_BYTES;
            for (int i = t_idx; i < 4 * nz * 8; i += 256) {
              const int chunk = i / (nz * 8);
              const int rem = i % (nz * 8);
              const int ri = rem / 8, piece = rem % 8;
              const int row = ri < z_lo ? ri : z_keep + (ri - z_lo);
              *reinterpret_cast<uint4*>(vbase + chunk * ATT_CHUNK_BYTES + row * 128 + piece * 16) =
                  make_uint4(0, 0, 0, 0);
            }
          }
          tmem_st_wait();
          fence_proxy_async_smem();
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sh.p_full[sb]);
        }
        if (!ok) break;
        const int seg_last_g = g - 1;
        // next segment's Q̂ goes into TMEM now: its QK may start before this epilogue ends
        if (s_i + 1 < seg_end) {
          if (!att_warp_wait(sh, &sh.q_free, k & 1)) { ok = false; break; }
          tc_fence_after_sync();
          load_q_tmem(p.segs[s_i + 1]);
        }
        // segment epilogue: O / l (this thread's 128 of the CTA's 256 columns) and the lse. The
        // partial sums go through the row-maximum slot of the other tile parity: the partner
        // read its last maxima (tile seg_last_g - 1) before the meeting of tile seg_last_g,
        // which this warp has passed; a second meeting after the sums are read keeps the next
        // tile's maxima out of the slot until both warps hold l_sum.
        float (*row_sum)[128] = sh.row_max[(seg_last_g + 1) & 1];
        row_sum[hc][r_local] = l_part;
        if (!meet()) { ok = false; break; }
        const float l_sum = row_sum[0][r_local] + row_sum[1][r_local];
        if (!meet()) { ok = false; break; }
        if (!att_warp_wait(sh, &sh.pv_done[seg_last_g & 1], (seg_last_g >> 1) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const float inv_l = (l_sum > 0.0f) ? 1.0f / l_sum : 0.0f;
        __nv_bfloat16* dst =
            p.o_part + (static_cast<int64_t>(s_i) * 128 + r_local) * ATT_DC + half * 256;
        // the merge reads these partials right after this kernel: keep them in L2 while the
        // cache stream of the other CTAs passes through it
        const uint64_t keep = l2_policy_evict_last();
#pragma unroll 1
        for (int c0 = hc * 128; c0 < hc * 128 + 128; c0 += 32) {
          uint32_t o[32];
          tmem_ld32(tmem + t_lane + TM_O + c0, o);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; j += 8)
            st_global_u4_hint(dst + c0 + j,
                              pack_bf16x2(__uint_as_float(o[j]) * inv_l, __uint_as_float(o[j + 1]) * inv_l),
                              pack_bf16x2(__uint_as_float(o[j + 2]) * inv_l, __uint_as_float(o[j + 3]) * inv_l),
                              pack_bf16x2(__uint_as_float(o[j + 4]) * inv_l, __uint_as_float(o[j + 5]) * inv_l),
                              pack_bf16x2(__uint_as_float(o[j + 6]) * inv_l, __uint_as_float(o[j + 7]) * inv_l),
                              keep);
        }
        if (half == 0 && hc == 0)
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

}  // namespace mla
