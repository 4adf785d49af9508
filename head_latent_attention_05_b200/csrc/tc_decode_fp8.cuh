// Absorbed-MLA decode attention over a quantised latent cache (FP8 E4M3 codes, one float32
// scale per token; layout in fp8_cache.cuh), on tcgen05. Same work split, planner, TMEM map,
// pipeline and outputs as mla_decode_attn_kernel (tc_decode.cuh); what changes is how a page
// meets the tensor cores.
//
// Scores. A row of the cache means C_j = sc_j * K_j (codes K_j, scale sc_j), so
//     s_rj = scale * Q̂_r · C_j = scale * sc_j * (Q̂_r · K_j).
// The codes go to the tensor cores as they are (kind::f8f6f4, E4M3 x E4M3, fp32 accumulate),
// which needs Q̂ in E4M3 too. One E4M3 value keeps 4 significant bits, so each query row is
// split, with its own scale a_r = max|Q̂_r| / 448, into a high and a low part,
//     Q̂_r / a_r = hi_r + lo_r + (error of about 2^-8 relative),   hi = E4M3(Q̂_r / a_r),
//                                                                lo = E4M3(Q̂_r / a_r - hi),
// and both parts multiply the same codes: D_rj = (hi_r + lo_r) · K_j, two MMAs per K-step into
// one accumulator. The softmax then works with s_rj = D_rj * sc_j * (a_r * scale). The split is
// its own small kernel (qsplit_rows_kernel), run between the query absorption and this kernel,
// which lays every row out as the attention kernel loads it (F8_QROW_BYTES below). This costs
// the same tensor time as the bf16 kernel's score (twice the MMAs at twice the rate) and keeps
// its precision (bf16 also keeps about 8 bits), while each page is half the bytes.
//
// Values. O_r = Σ_j P_rj C_j[:d_c] = Σ_j (P_rj sc_j) K_j[:d_c]: the scale joins P before P is
// rounded to bf16, and the codes of this CTA's c_KV half are converted to bf16 in shared memory
// (exactly: every E4M3 value is a bf16 value), so P·C runs as in the bf16 kernel. The softmax
// warps convert each tile right after agreeing on its row maxima, where they would otherwise
// wait for the previous tile's P·C; rows outside the keys the unit sees are written as zeros.
//
// Shared memory: 2 stages x [4 code chunks of 64 tokens x 128 codes (128-byte swizzle) | k_R
// codes 64 x 64 (64-byte swizzle)] = 36 KB each, 2 converted buffers of 4 x [64 x 64] bf16 (32 KB
// each), the query parts for features 256..575 (5 chunks of 128 rows x 128 bytes: hi 256..383,
// hi 384..511, lo 256..383, lo 384..511, and [hi 512..575 | lo 512..575]), the page scales and
// the barriers. TMEM: [0,256) O half, [256,384) two score buffers, [384,448) hi and [448,512) lo
// of the query's features 0..255 (four codes per column).
//
// Warp roles (320 threads): 0 TMA producer, 1 MMA issuer, 2..9 softmax (they also place each
// unit's query features 0..255 in TMEM and convert the value codes).
#pragma once

#include "fp8_cache.cuh"
#include "tc_decode.cuh"

namespace mla {

constexpr int F8_PAGE_CODES = ATT_PAGE * ATT_ROW;                 // 36,864
constexpr int F8_PAGE_BYTES = F8_PAGE_CODES + 4 * ATT_PAGE;      // + 64 float32 scales
constexpr int F8_CHUNK_BYTES = ATT_PAGE * 128;                   // [64 tokens x 128 codes]
constexpr int F8_ROPE_BYTES = ATT_PAGE * ATT_DR;                 // [64 tokens x 64 codes]
constexpr int F8_STAGE_BYTES = 4 * F8_CHUNK_BYTES + F8_ROPE_BYTES;
constexpr int F8_CV_BYTES = 4 * ATT_CHUNK_BYTES;                 // own c_KV half in bf16
constexpr int F8_QS_CHUNKS = 5;
constexpr int F8_QS_CHUNK_BYTES = 128 * 128;
constexpr int F8_THREADS = 320;
constexpr uint32_t TM_QHI = TM_Q, TM_QLO = TM_Q + 64;

struct AttnSharedF8 {
  float scales[ATT_STAGES][ATT_PAGE];   // the stage's token scales (bulk-copy target)
  uint64_t full_qk[ATT_STAGES], full_own[ATT_STAGES];
  uint64_t empty_qk[ATT_STAGES], empty_own[ATT_STAGES];
  uint64_t s_full[2], p_full[2], pv_done[2];
  uint64_t q_full;                     // the softmax warps placed a unit's query in TMEM
  uint64_t qs_full;                    // the unit's query chunks landed in shared memory (TMA)
  uint64_t q_free, o_free, drain;
  uint64_t pair_bar[4];
  float row_max[2][2][128];
  uint32_t tmem_base;
  volatile int abort_flag;
};

constexpr int F8_SMEM_BYTES = ATT_STAGES * (F8_STAGE_BYTES + F8_CV_BYTES) +
                              F8_QS_CHUNKS * F8_QS_CHUNK_BYTES +
                              static_cast<int>(sizeof(AttnSharedF8));
static_assert(F8_SMEM_BYTES <= 227 * 1024, "fp8 attention kernel exceeds the shared memory of a CTA");

__device__ __forceinline__ uint16_t e4m3x2_raw(float a, float b) {
  return static_cast<uint16_t>(
      __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3));
}
// Value of an E4M3 code (low byte of c) in float32, exactly, without the conversion pipe: the
// code's exponent and mantissa bits placed in a float32's exponent and mantissa fields make a
// float32 equal to the value times 2^-120 (subnormal codes become float32 denormals, which
// keep every bit), and the multiplication by 2^120 is exact.
__device__ __forceinline__ float e4m3_value_f32(uint32_t c) {
  return __uint_as_float(((c & 0x80u) << 24) | ((c & 0x7Fu) << 20)) * 0x1p120f;
}
// Four E4M3 codes (one 32-bit word, first code in the lowest byte) as two bf16 pairs, exactly,
// in the same way: each code's bits placed in a bf16 lane give the value times 2^-120 (a bf16
// denormal for a subnormal code), and one bf16x2 multiplication by 2^120 restores it.
__device__ __forceinline__ void e4m3x4_to_bf16x4(uint32_t x, uint32_t& lo, uint32_t& hi) {
  const __nv_bfloat162 k = __halves2bfloat162(__ushort_as_bfloat16(0x7B80), __ushort_as_bfloat16(0x7B80));
  const uint32_t t0 = __byte_perm(x, 0u, 0x1404);   // lanes: code 0 << 8, code 1 << 8
  const uint32_t t1 = __byte_perm(x, 0u, 0x3424);   // lanes: code 2 << 8, code 3 << 8
  const uint32_t v0 = (t0 & 0x80008000u) | ((t0 >> 4) & 0x07F007F0u);
  const uint32_t v1 = (t1 & 0x80008000u) | ((t1 >> 4) & 0x07F007F0u);
  const __nv_bfloat162 r0 = __hmul2(*reinterpret_cast<const __nv_bfloat162*>(&v0), k);
  const __nv_bfloat162 r1 = __hmul2(*reinterpret_cast<const __nv_bfloat162*>(&v1), k);
  lo = *reinterpret_cast<const uint32_t*>(&r0);
  hi = *reinterpret_cast<const uint32_t*>(&r1);
}
// Eight bf16 query values times inv -> their high and low E4M3 parts (two 32-bit words each,
// the first feature in the lowest byte).
__device__ __forceinline__ void f8_split8(const uint4& x, float inv, uint32_t& h0, uint32_t& h1,
                                          uint32_t& l0, uint32_t& l1) {
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
  uint32_t hc[4], lc[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float a = __uint_as_float(w[i] << 16) * inv;
    const float b = __uint_as_float(w[i] & 0xFFFF0000u) * inv;
    const uint16_t hh = e4m3x2_raw(a, b);
    const float ha = e4m3_value_f32(hh), hb = e4m3_value_f32(static_cast<uint32_t>(hh) >> 8);
    hc[i] = hh;
    lc[i] = e4m3x2_raw(a - ha, b - hb);   // exact differences (ha, hb are a, b rounded)
  }
  h0 = hc[0] | (hc[1] << 16);
  h1 = hc[2] | (hc[3] << 16);
  l0 = lc[0] | (lc[1] << 16);
  l1 = lc[2] | (lc[3] << 16);
}
__device__ __forceinline__ float absmax_bf16x8(const uint4& x) {
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < 4; ++i)
    m = fmax3(m, fabsf(__uint_as_float(w[i] << 16)), fabsf(__uint_as_float(w[i] & 0xFFFF0000u)));
  return m;
}

// A split query row, 1152 bytes: [hi 0..255 | lo 0..255 | hi 256..511 | lo 256..511 |
// hi 512..575, lo 512..575] (feature indices; one code per feature). The first 512 bytes go to
// TMEM, the other 640 are the five [128 rows x 128 B] shared-memory chunks of the kernel, each
// one TMA box.
constexpr int F8_QROW_BYTES = 2 * ATT_ROW;
__device__ __forceinline__ int qsplit_hi_pos(int f) {
  return f < 256 ? f : (f < 512 ? 512 + (f - 256) : 1024 + (f - 512));
}
__device__ __forceinline__ int qsplit_lo_pos(int f) {
  return f < 256 ? 256 + f : (f < 512 ? 768 + (f - 256) : 1088 + (f - 512));
}

// Split n_rows bf16 query rows [n_rows][576] into their high and low E4M3 parts under the row's
// scale a = max|row| / 448 (0 for a zero row): codes [n_rows][1152] in the layout above and
// a [n_rows]. One warp per row, 8 rows per 256-thread block; lane l takes 8-feature groups l,
// l + 32 and l + 64 (< 72).
__global__ void __launch_bounds__(256)
qsplit_rows_kernel(const __nv_bfloat16* __restrict__ qhat, int n_rows, uint8_t* __restrict__ codes,
                   float* __restrict__ alpha) {
  pdl_wait();   // the query absorption just before wrote qhat
  pdl_trigger();
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= n_rows) return;
  const uint4* src = reinterpret_cast<const uint4*>(qhat + static_cast<int64_t>(row) * ATT_ROW);
  uint4 x[3];
  float am = 0.0f;
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    const int gi = lane + 32 * k;
    x[k] = gi < ATT_ROW / 8 ? src[gi] : make_uint4(0, 0, 0, 0);
    am = fmaxf(am, absmax_bf16x8(x[k]));
  }
  am = warp_max(am);
  const float inv = am > 0.0f ? __fdiv_rn(E4M3_MAX_F, am) : 0.0f;
  uint8_t* dst = codes + static_cast<int64_t>(row) * F8_QROW_BYTES;
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    const int gi = lane + 32 * k;
    if (gi >= ATT_ROW / 8) break;
    uint2 h, l;
    f8_split8(x[k], inv, h.x, h.y, l.x, l.y);
    *reinterpret_cast<uint2*>(dst + qsplit_hi_pos(8 * gi)) = h;
    *reinterpret_cast<uint2*>(dst + qsplit_lo_pos(8 * gi)) = l;
  }
  if (lane == 0) alpha[row] = __fdiv_rn(am, E4M3_MAX_F);
}

// This CTA's c_KV half of a page, codes -> bf16 (exactly) in the K-major 128-byte-swizzled
// chunks P·C reads ([64 tokens x 64 features] each), rows outside [z_lo, z_keep) written as
// zeros: 1024 16-byte code units (source chunk j = i / 512, token row r, 16 features u), thread
// tid of nthreads taking units tid, tid + nthreads, ...
__device__ __forceinline__ void f8_convert_own(const uint8_t* src, uint8_t* dst, int tid,
                                               int nthreads, int z_lo, int z_keep) {
#pragma unroll 2
  for (int i = tid; i < 1024; i += nthreads) {
    const int j = i >> 9, r = (i >> 3) & 63, u = i & 7;
    const int sw = r & 7;
    uint4 lo4 = make_uint4(0, 0, 0, 0), hi4 = make_uint4(0, 0, 0, 0);
    if (r >= z_lo && r < z_keep) {
      const uint4 x = *reinterpret_cast<const uint4*>(src + j * F8_CHUNK_BYTES + r * 128 + ((u ^ sw) << 4));
      e4m3x4_to_bf16x4(x.x, lo4.x, lo4.y);
      e4m3x4_to_bf16x4(x.y, lo4.z, lo4.w);
      e4m3x4_to_bf16x4(x.z, hi4.x, hi4.y);
      e4m3x4_to_bf16x4(x.w, hi4.z, hi4.w);
    }
    // features 16u .. 16u+15 of source chunk j: bf16 chunk 2j + u/4, 16-byte units 2(u%4) and
    // 2(u%4) + 1 of row r
    uint8_t* d = dst + (2 * j + (u >> 2)) * ATT_CHUNK_BYTES + r * 128;
    const int w0 = 2 * (u & 3);
    *reinterpret_cast<uint4*>(d + ((w0 ^ sw) << 4)) = lo4;
    *reinterpret_cast<uint4*>(d + (((w0 + 1) ^ sw) << 4)) = hi4;
  }
}

// Score K-steps of one 128-code chunk c of a page into the score buffer at TMEM column d_s:
// the hi and the lo part of the query each meet the chunk's four K = 32 steps. Chunks 0, 1
// take A from TMEM, chunks 2, 3 from shared memory (query chunks c-2 (hi) and c (lo)).
__device__ __forceinline__ void f8_qk_chunk(uint32_t tmem, uint32_t d_s, uint64_t b_stage,
                                            uint64_t qs_desc, int c, bool first) {
  constexpr uint32_t IDESC = idesc_e4m3(128, 64);
  const uint64_t b0 = b_stage + static_cast<uint64_t>((c * F8_CHUNK_BYTES) >> 4);
  if (c < 2) {
    mma_f8_ts_x4_elect(tmem + d_s, tmem + TM_QHI + 32 * c, b0, IDESC, first ? 0u : 1u);
    mma_f8_ts_x4_elect(tmem + d_s, tmem + TM_QLO + 32 * c, b0, IDESC, 1u);
  } else {
    const uint64_t a_hi = qs_desc + static_cast<uint64_t>(((c - 2) * F8_QS_CHUNK_BYTES) >> 4);
    const uint64_t a_lo = qs_desc + static_cast<uint64_t>((c * F8_QS_CHUNK_BYTES) >> 4);
    mma_f8_ss_x4_elect(tmem + d_s, a_hi, b0, IDESC, first ? 0u : 1u);
    mma_f8_ss_x4_elect(tmem + d_s, a_lo, b0, IDESC, 1u);
  }
}
// The k_R codes (64 wide, 64-byte swizzle) against query chunk 4 = [hi | lo] of features
// 512..575: never the first K-step of a tile.
__device__ __forceinline__ void f8_qk_rope(uint32_t tmem, uint32_t d_s, uint32_t rope_saddr,
                                           uint64_t qs_desc) {
  constexpr uint32_t IDESC = idesc_e4m3(128, 64);
  mma_f8_ss_pair_elect(tmem + d_s, qs_desc + static_cast<uint64_t>((4 * F8_QS_CHUNK_BYTES) >> 4),
                       smem_desc_sw64(rope_saddr, 512), IDESC);
}

__global__ void __launch_bounds__(F8_THREADS, 1)
mla_decode_attn_fp8_kernel(const __grid_constant__ CUtensorMap map_c8,
                           const __grid_constant__ CUtensorMap map_r8,
                           const __grid_constant__ CUtensorMap map_q8, AttnParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_addr(smem) & 1023u) != 0) {
    if (threadIdx.x == 0) record_error(MLA_ERR_UNSUPPORTED);
    return;
  }
  uint8_t* stage_buf = smem;                                     // stage s: + s*F8_STAGE_BYTES
  uint8_t* cv_buf = smem + ATT_STAGES * F8_STAGE_BYTES;          // stage s: + s*F8_CV_BYTES
  uint8_t* qs_buf = cv_buf + ATT_STAGES * F8_CV_BYTES;
  AttnSharedF8& sh =
      *reinterpret_cast<AttnSharedF8*>(qs_buf + F8_QS_CHUNKS * F8_QS_CHUNK_BYTES);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = blockIdx.x >> 1, half = blockIdx.x & 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < ATT_STAGES; ++s) {
      mbar_init(&sh.full_qk[s], 1);
      mbar_init(&sh.full_own[s], 1);
      mbar_init(&sh.empty_qk[s], 1);
      // the stage's codes and scales are free once the score MMAs are done and the softmax
      // warps have read the scales and converted the value codes: P·C reads the converted copy
      mbar_init(&sh.empty_own[s], 1 + ATT_SM_WARPS);
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
    tma_prefetch_desc(&map_c8);
    tma_prefetch_desc(&map_r8);
    tma_prefetch_desc(&map_q8);
  }
  if (warp == 1) {
    tmem_alloc(&sh.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = sh.tmem_base;
  pdl_wait();
  pdl_trigger();
  const int seg_begin = p.pair_seg[pair], seg_end = p.pair_seg[pair + 1];

  if (seg_begin < seg_end) {
    if (warp == 0) {
      if (lane == 0) {
        // =========================================================== TMA producer
        auto page_of = [&](const TileCursor& c) {
          const int b = c.sg.unit / p.n_mt;
          int page = p.block_table[static_cast<int64_t>(b) * p.max_pages + c.tile];
          if (page < 0 || page >= p.num_pages) {
            record_error(MLA_ERR_DEVICE_OOB);
            page = 0;
          }
          return page;
        };
        // own: this CTA's two c_KV code chunks and the page's scales; score-only: the other
        // two c_KV chunks and the k_R codes
        auto load_chunks = [&](const TileCursor& c, int g, bool own, uint64_t* bar) {
          const int page = page_of(c);
          const int s = g % ATT_STAGES;
          uint8_t* st = stage_buf + s * F8_STAGE_BYTES;
          const int c0 = own ? 2 * half : 2 * (1 - half);
          if (own) {
            mbar_arrive_expect_tx(bar, 2 * F8_CHUNK_BYTES + 4 * ATT_PAGE);
            tma_load_4d(st + c0 * F8_CHUNK_BYTES, &map_c8, bar, 0, 0, c0, page);
            bulk_load_g2s(sh.scales[s], p.cache8 + static_cast<int64_t>(page) * F8_PAGE_BYTES + F8_PAGE_CODES,
                          4 * ATT_PAGE, bar);
          } else {
            mbar_arrive_expect_tx(bar, 2 * F8_CHUNK_BYTES + F8_ROPE_BYTES);
            tma_load_4d(st + c0 * F8_CHUNK_BYTES, &map_c8, bar, 0, 0, c0, page);
            tma_load_3d(st + 4 * F8_CHUNK_BYTES, &map_r8, bar, 0, 0, page);
          }
        };
        int n_qloads = 0;   // query loads issued: the last one is drained before the CTA leaves
        auto load_q_smem = [&](const AttnSeg& sg) {   // query bytes 512..1151 of a unit's rows
          const int b = sg.unit / p.n_mt, mt = sg.unit % p.n_mt;
          mbar_arrive_expect_tx(&sh.qs_full, F8_QS_CHUNKS * F8_QS_CHUNK_BYTES);
          for (int c = 0; c < F8_QS_CHUNKS; ++c)
            tma_load_2d(qs_buf + c * F8_QS_CHUNK_BYTES, &map_q8, &sh.qs_full, 512 + 128 * c,
                        b * p.R + mt * 128);
          ++n_qloads;
        };
        TileCursor cq, co;   // score-only cursor (one tile ahead), own-chunk cursor
        cq.init(p.segs, seg_begin, seg_end);
        co.init(p.segs, seg_begin, seg_end);
        if (half == 0) {   // later segments' query rows into L2
          for (int s_i = seg_begin + 1; s_i < seg_end; ++s_i) {
            const AttnSeg sg = p.segs[s_i];
            const int b = sg.unit / p.n_mt, mt = sg.unit % p.n_mt;
            const int rows = min(128, p.R - mt * 128);
            prefetch_l2_bulk(p.qcodes + (static_cast<int64_t>(b) * p.R + mt * 128) * F8_QROW_BYTES,
                             static_cast<uint32_t>(rows * F8_QROW_BYTES));
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
          if (seg_ends) {   // the next unit's query chunks: the last S of this one must be done
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
        // drain: the last query load and the last loads of each ring must land before the CTA
        // can exit
        if (n_qloads > 0) (void)mbar_wait(&sh.qs_full, (n_qloads - 1) & 1);
        for (int j = max(0, gq - ATT_STAGES); j < gq; ++j)
          (void)mbar_wait(&sh.full_qk[j % ATT_STAGES], (j / ATT_STAGES) & 1);
        for (int j = max(0, go - ATT_STAGES); j < go; ++j)
          (void)mbar_wait(&sh.full_own[j % ATT_STAGES], (j / ATT_STAGES) & 1);
      }
    } else if (warp == 1) {
      // ======================================== MMA issuer: S of tile g, then P·C of g-1
      constexpr uint32_t IDESC_PV = idesc_bf16(128, 256, false, true);
      const uint32_t stage0 = smem_addr(stage_buf), cv0 = smem_addr(cv_buf);
      const uint64_t qs_desc = smem_desc_sw128(smem_addr(qs_buf), 16, 1024);
      auto issue_pv = [&](int gv, bool first_v, int kv) -> bool {
        const int st = gv % ATT_STAGES, sb = gv & 1;
        if (first_v && kv >= 1 && !att_warp_wait(sh, &sh.o_free, (kv - 1) & 1)) return false;
        if (!att_warp_wait(sh, &sh.p_full[sb], (gv >> 1) & 1)) return false;
        tc_fence_after_sync();
        const uint64_t b0 = smem_desc_sw128(cv0 + st * F8_CV_BYTES, ATT_CHUNK_BYTES, 1024);
        mma_bf16_ts_mn_x4_elect(tmem + TM_O, tmem + TM_S + 64 * sb, b0, IDESC_PV, first_v ? 0u : 1u);
        mma_commit_elect(&sh.pv_done[sb]);   // the score buffer and the converted half are free
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
        if (g >= 2 && !att_warp_wait(sh, &sh.pv_done[sb], ((g >> 1) - 1) & 1)) { ok = false; break; }
        const uint32_t st_addr = stage0 + st * F8_STAGE_BYTES;
        const uint64_t b_stage = smem_desc_sw128(st_addr, 16, 1024);
        if (!att_warp_wait(sh, &sh.full_qk[st], (g / ATT_STAGES) & 1)) { ok = false; break; }
        tc_fence_after_sync();
        // score-only chunks (the other half's c_KV codes, then k_R), then this CTA's own
        const int other = 2 * (1 - half), own = 2 * half;
        f8_qk_chunk(tmem, d_s, b_stage, qs_desc, other, true);
        f8_qk_chunk(tmem, d_s, b_stage, qs_desc, other + 1, false);
        f8_qk_rope(tmem, d_s, st_addr + 4 * F8_CHUNK_BYTES, qs_desc);
        mma_commit_elect(&sh.empty_qk[st]);
        if (!att_warp_wait(sh, &sh.full_own[st], (g / ATT_STAGES) & 1)) { ok = false; break; }
        tc_fence_after_sync();
        f8_qk_chunk(tmem, d_s, b_stage, qs_desc, own, false);
        f8_qk_chunk(tmem, d_s, b_stage, qs_desc, own + 1, false);
        mma_commit_elect(&sh.s_full[sb]);
        mma_commit_elect(&sh.empty_own[st]);   // the score MMAs are done with the codes
        if (cur.last_of_seg()) mma_commit_elect(&sh.q_free);
        if (g >= 1 && !issue_pv(g - 1, prev_first, prev_k)) { ok = false; break; }
        prev_first = cur.first_of_seg();
        prev_k = cur.k;
      }
      if (ok && g >= 1) (void)issue_pv(g - 1, prev_first, prev_k);
      mma_commit_elect(&sh.drain);
      if (lane == 0) (void)mbar_wait(&sh.drain, 0);
      __syncwarp();
    } else {
      // ============================================================ softmax warps
      const int hc = warp >= 6 ? 1 : 0;
      const int quarter = warp & 3;
      const int r_local = quarter * 32 + lane;
      const uint32_t t_lane = static_cast<uint32_t>(quarter * 32) << 16;
      int g = 0, xc = 0;
      bool ok = true;
      auto meet = [&]() -> bool {
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.pair_bar[quarter]);
        const bool r = att_warp_wait(sh, &sh.pair_bar[quarter], xc & 1);
        ++xc;
        return r;
      };
      // A unit's split query features 0..255 into TMEM (row r_local; zeros past the unit):
      // the warps of column half 0 write the hi codes, those of half 1 the lo codes. Returns
      // false on abort; *rowf = a_r * softmax_scale * log2(e).
      auto load_q = [&](const AttnSeg& sg, float* rowf) -> bool {
        const int b = sg.unit / p.n_mt, mt = sg.unit % p.n_mt;
        const int r_in = mt * 128 + r_local;
        const bool valid = r_in < p.R;
        const int64_t grow = static_cast<int64_t>(b) * p.R + (valid ? r_in : 0);
        const uint4* src = reinterpret_cast<const uint4*>(p.qcodes + grow * F8_QROW_BYTES + 256 * hc);
        *rowf = valid ? p.qalpha[grow] * p.scale_log2 : 0.0f;
        uint32_t v[32];
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint4 x = valid ? src[8 * c + j] : make_uint4(0, 0, 0, 0);
            v[4 * j + 0] = x.x; v[4 * j + 1] = x.y; v[4 * j + 2] = x.z; v[4 * j + 3] = x.w;
          }
          tmem_st32(tmem + t_lane + (hc ? TM_QLO : TM_QHI) + 32 * c, v);
        }
        tmem_st_wait();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.q_full);
        return true;
      };
      float rowf_next = 0.0f;
      ok = load_q(p.segs[seg_begin], &rowf_next);
      for (int k = 0, s_i = seg_begin; ok && s_i < seg_end; ++k, ++s_i) {
        const AttnSeg sg = p.segs[s_i];
        const float rowf = rowf_next;
        const int b = sg.unit / p.n_mt, mt = sg.unit % p.n_mt;
        const int L = p.seq_lens[b];
        const int r_in = mt * 128 + r_local;
        const bool row_valid = r_in < p.R;
        int lo_row = 1, hi_row = 0, lo_u, hi_u, unused;
        if (row_valid) visible_keys(p.keys, b, L, p.Tq, r_in / p.H, &lo_row, &hi_row);
        visible_keys(p.keys, b, L, p.Tq, (mt * 128) / p.H, &lo_u, &unused);
        visible_keys(p.keys, b, L, p.Tq, min(p.Tq - 1, (mt * 128 + 127) / p.H), &unused, &hi_u);
        float m_ref = -INFINITY, l_part = 0.0f;
        for (int tile = sg.tile_begin; tile < sg.tile_end; ++tile, ++g) {
          const int sb = g & 1, st = g % ATT_STAGES;
          const uint32_t s_col = TM_S + 64 * sb;
          if (!att_warp_wait(sh, &sh.s_full[sb], (g >> 1) & 1)) { ok = false; break; }
          // the page's scales came with the own chunks, which S has consumed
          if (!att_warp_wait(sh, &sh.full_own[st], (g / ATT_STAGES) & 1)) { ok = false; break; }
          tc_fence_after_sync();
          uint32_t sr[32];
          tmem_ld32(tmem + t_lane + s_col + hc * 32, sr);
          float scl[32];
#pragma unroll
          for (int c = 0; c < 32; c += 4) {
            const float4 v = *reinterpret_cast<const float4*>(&sh.scales[st][hc * 32 + c]);
            scl[c] = v.x; scl[c + 1] = v.y; scl[c + 2] = v.z; scl[c + 3] = v.w;
          }
          tmem_ld_wait();
          tc_fence_before_sync();
          float xs[32];   // D_rj * sc_j
#pragma unroll
          for (int c = 0; c < 32; ++c) xs[c] = __uint_as_float(sr[c]) * scl[c];
          const int j0 = tile * ATT_PAGE + hc * 32;
          const int c_lo = max(0, lo_row - j0), c_hi = min(31, hi_row - j0);
          const bool all_vis = c_lo == 0 && c_hi == 31;
          float mx0 = -INFINITY, mx1 = -INFINITY;
          if (all_vis) {
#pragma unroll
            for (int c = 0; c < 32; c += 4) {
              mx0 = fmax3(mx0, xs[c], xs[c + 1]);
              mx1 = fmax3(mx1, xs[c + 2], xs[c + 3]);
            }
          } else {
#pragma unroll
            for (int c = 0; c < 32; c += 2) {
              mx0 = fmaxf(mx0, (c >= c_lo && c <= c_hi) ? xs[c] : -INFINITY);
              mx1 = fmaxf(mx1, (c + 1 >= c_lo && c + 1 <= c_hi) ? xs[c + 1] : -INFINITY);
            }
          }
          sh.row_max[g & 1][hc][r_local] = fmaxf(mx0, mx1);
          if (!meet()) { ok = false; break; }
          tc_fence_after_sync();
          const float raw_max = fmaxf(sh.row_max[g & 1][0][r_local], sh.row_max[g & 1][1][r_local]);
          const float mt_max = raw_max > -INFINITY ? raw_max * rowf : -INFINITY;
          // this tile's c_KV half as bf16 for P·C (its codes have landed: S has read them; P·C
          // of tile g-2, the last reader of this converted buffer, finished before S(g) began),
          // done here, where the warps would otherwise wait for P·C of the previous tile; the
          // stage may then take the codes of tile g+2 while P·C of tile g is still to come
          {
            const int z_lo = min(ATT_PAGE, max(0, lo_u - tile * ATT_PAGE));
            const int z_keep = max(z_lo, min(ATT_PAGE, hi_u + 1 - tile * ATT_PAGE));
            f8_convert_own(stage_buf + st * F8_STAGE_BYTES + 2 * half * F8_CHUNK_BYTES,
                           cv_buf + st * F8_CV_BYTES, hc * 128 + r_local, 256, z_lo, z_keep);
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.empty_own[st]);   // done with the codes and scales
          }
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
          // P = 2^(rowf*x - m_ref); the sum takes P, the value MMA takes P * sc_j (0 where the
          // key is hidden, whatever the slot's scale holds)
          const float neg_m = (m_ref == -INFINITY) ? 0.0f : -m_ref;
          const uint64_t rf2 = f2_pack(rowf, rowf), nm2 = f2_pack(neg_m, neg_m);
          uint64_t ps2 = f2_pack(0.0f, 0.0f);
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int c = 2 * e;
            float x0, x1;
            f2_unpack(f2_fma(f2_pack(xs[c], xs[c + 1]), rf2, nm2), x0, x1);
            x0 = fast_exp2(x0);
            x1 = fast_exp2(x1);
            float y0 = x0 * scl[c], y1 = x1 * scl[c + 1];
            if (!all_vis) {
              const bool v0 = c >= c_lo && c <= c_hi, v1 = c + 1 >= c_lo && c + 1 <= c_hi;
              x0 = v0 ? x0 : 0.0f;
              x1 = v1 ? x1 : 0.0f;
              y0 = v0 ? y0 : 0.0f;
              y1 = v1 ? y1 : 0.0f;
            }
            ps2 = f2_add(ps2, f2_pack(x0, x1));
            w[e] = pack_bf16x2(y0, y1);
          }
          tmem_st16(tmem + t_lane + s_col + hc * 16, w);
          float ps0, ps1;
          f2_unpack(ps2, ps0, ps1);
          l_part += ps0 + ps1;
          tmem_st_wait();
          fence_proxy_async_smem();   // the converted half is read by P·C (async proxy)
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sh.p_full[sb]);
        }
        if (!ok) break;
        const int seg_last_g = g - 1;
        if (s_i + 1 < seg_end) {
          if (!att_warp_wait(sh, &sh.q_free, k & 1)) { ok = false; break; }
          tc_fence_after_sync();
          if (!load_q(p.segs[s_i + 1], &rowf_next)) { ok = false; break; }
        }
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
