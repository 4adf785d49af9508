// libmla.so: the C ABI declared in include/mla.h.
//
// Host side of every entry point: validate the arguments (nothing is launched on error), carve
// the caller's workspace, encode TMA descriptors and enqueue the kernels on the caller's
// stream. No device memory is ever allocated here.
#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <unordered_map>

#include "../../include/mla.h"
#include "common.cuh"
#include "ptx.cuh"
#include "simt.cuh"
#include "tc_decode.cuh"
#include "tc_decode_fp8.cuh"
#include "fp8_cache.cuh"
#include "tc_gemm.cuh"
#include "tc_vproj.cuh"

using namespace mla;

namespace {

// ------------------------------------------------------------------------------ helpers

constexpr size_t kAlign = 256;
size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

struct Carve {
  uint8_t* base;
  size_t off = 0;
  explicit Carve(void* b) : base(static_cast<uint8_t*>(b)) {}
  template <typename T>
  T* take(size_t count) {
    T* p = reinterpret_cast<T*>(base == nullptr ? nullptr : base + off);
    off += align_up(count * sizeof(T));
    return p;
  }
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// An NVTX range named after the entry point around each call (host side: it brackets the
// validation and the launches, which profilers then group under the call's name; without a
// profiler attached it costs a few nanoseconds).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

int elem_bytes(const mla_config* c) { return c->dtype == MLA_DTYPE_F32 ? 4 : 2; }
bool fp8_cache(const mla_config* c) { return c->kv_format == MLA_KV_FP8_E4M3; }

mla_status check_config(const mla_config* c) {
  if (c == nullptr) return MLA_ERR_INVALID_ARG;
  if (c->n_heads < 1 || c->d_model < 1 || c->d_c < 1 || c->d_rope < 2 || (c->d_rope & 1) ||
      c->d_nope < 1 || c->d_v < 1 || c->page_size < 1)
    return MLA_ERR_INVALID_ARG;
  if (c->dtype != MLA_DTYPE_F32 && c->dtype != MLA_DTYPE_BF16) return MLA_ERR_INVALID_ARG;
  if (!(c->softmax_scale > 0.0f) || !std::isfinite(c->softmax_scale)) return MLA_ERR_INVALID_ARG;
  if (!(c->rms_eps >= 0.0f) || !(c->rope_theta > 0.0f)) return MLA_ERR_INVALID_ARG;
  if (c->window < 0) return MLA_ERR_INVALID_ARG;
  if (c->kv_format != MLA_KV_PLAIN && c->kv_format != MLA_KV_FP8_E4M3) return MLA_ERR_INVALID_ARG;
  // every row must stay 16-byte aligned for vector loads and TMA (a quantised row: its codes)
  const int64_t row_bytes = static_cast<int64_t>(c->d_c + c->d_rope) * (fp8_cache(c) ? 1 : elem_bytes(c));
  if (row_bytes % 16 != 0) return MLA_ERR_UNSUPPORTED;
  if (fp8_cache(c) && c->dtype != MLA_DTYPE_BF16) return MLA_ERR_UNSUPPORTED;
  if (c->d_rope > 2 * MLA_MAX_ROPE_PAIRS) return MLA_ERR_UNSUPPORTED;
  return MLA_OK;
}

// theta^(-2i/d_rope) / pi per rotary pair, in double precision on the host, split hi + lo.
RopeFreqs rope_freqs(const mla_config* c) {
  RopeFreqs f{};
  const double pi = 3.141592653589793238462643383279502884;
  for (int i = 0; i < c->d_rope / 2 && i < MLA_MAX_ROPE_PAIRS; ++i) {
    const double v = std::pow(static_cast<double>(c->rope_theta),
                              -2.0 * static_cast<double>(i) / static_cast<double>(c->d_rope)) / pi;
    f.f_hi[i] = static_cast<float>(v);
    f.f_lo[i] = static_cast<float>(v - static_cast<double>(f.f_hi[i]));
  }
  return f;
}

// The bf16 decode path: tcgen05 kernels written for DeepSeek-V2 latent shapes.
bool tc_decode_shape(const mla_config* c) {
  return c->dtype == MLA_DTYPE_BF16 && c->d_c == ATT_DC && c->d_rope == ATT_DR &&
         c->page_size == ATT_PAGE && c->d_nope % 64 == 0;
}

int device_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

mla_status last_launch_status() {
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

// Launch with programmatic stream serialization: the kernel may start while the previous
// kernel of the stream finishes, and calls pdl_wait() before it reads that kernel's output.
// Used only for the second and later kernels of one call, whose predecessor is the library's
// own kernel (which triggers only after its own wait).
// cluster_x > 1 also launches the grid as clusters of cluster_x CTAs along x.
template <typename... KArgs, typename... Args>
mla_status launch_pdl_clustered(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                cudaStream_t st, unsigned cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.numAttrs = 1;
  if (cluster_x > 1) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster_x;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
  }
  cfg.attrs = attr;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) == cudaSuccess
             ? MLA_OK
             : MLA_ERR_CUDA;
}
template <typename... KArgs, typename... Args>
mla_status launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                      cudaStream_t st, Args&&... args) {
  return launch_pdl_clustered(kernel, grid, block, smem, st, 1u, std::forward<Args>(args)...);
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link-time libcuda).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Encoded maps are cached: a map is a pure function of (base, rank, dims, strides, box, element
// type, swizzle), so a hit is always exact, and decode steps that reuse their buffers skip the
// driver call.
struct MapKey {
  uint64_t v[16];
  bool operator==(const MapKey& o) const {
    for (int i = 0; i < 16; ++i)
      if (v[i] != o.v[i]) return false;
    return true;
  }
};
struct MapKeyHash {
  size_t operator()(const MapKey& k) const {
    uint64_t h = 1469598103934665603ull;
    for (int i = 0; i < 16; ++i) h = (h ^ k.v[i]) * 1099511628211ull;
    return static_cast<size_t>(h);
  }
};
constexpr size_t kMapCacheMax = 4096;

bool encode_map(CUtensorMap* m, const void* base, int rank, const uint64_t* dims,
                const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapDataType dt,
                CUtensorMapSwizzle sw) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t d[4], s[3];
  cuuint32_t bx[4], es[4] = {1, 1, 1, 1};
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
  }
  for (int i = 0; i + 1 < rank; ++i) s[i] = strides_bytes[i];
  return enc(m, dt, rank, const_cast<void*>(base), d, s, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tiled tensor map (rank <= 4). dims[0] is the contiguous dimension; strides are the byte
// strides of dims 1.. . The default is bf16 with 128-byte swizzle (box[0] = 64 elements, one
// swizzle row).
bool make_map(CUtensorMap* m, const void* base, int rank, const uint64_t* dims,
              const uint64_t* strides_bytes, const uint32_t* box,
              CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
              CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B) {
  static std::mutex mu;
  static std::unordered_map<MapKey, CUtensorMap, MapKeyHash> cache;
  if (rank < 1 || rank > 4) return false;
  MapKey k{};
  k.v[0] = reinterpret_cast<uint64_t>(base);
  k.v[1] = static_cast<uint64_t>(rank);
  for (int i = 0; i < rank; ++i) {
    k.v[2 + i] = dims[i];
    k.v[6 + i] = box[i];
  }
  for (int i = 0; i + 1 < rank; ++i) k.v[10 + i] = strides_bytes[i];
  k.v[13] = static_cast<uint64_t>(dt);
  k.v[14] = static_cast<uint64_t>(sw);
  {
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(k);
    if (it != cache.end()) {
      *m = it->second;
      return true;
    }
  }
  if (!encode_map(m, base, rank, dims, strides_bytes, box, dt, sw)) return false;
  std::lock_guard<std::mutex> lock(mu);
  if (cache.size() >= kMapCacheMax) cache.clear();
  cache.emplace(k, *m);
  return true;
}

// Raise a kernel's dynamic shared-memory limit, once per (kernel, device): later calls, which
// may be inside a CUDA-graph capture, then make no CUDA runtime call here at all.
template <typename K>
bool allow_smem(K kernel, int bytes) {
  if (bytes <= 48 * 1024) return true;
  static std::mutex mu;
  static std::unordered_map<const void*, uint64_t> done;  // kernel -> bitmask of devices
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64) return false;
  const void* key = reinterpret_cast<const void*>(kernel);
  std::lock_guard<std::mutex> lock(mu);
  uint64_t& mask = done[key];
  if (mask & (1ull << dev)) return true;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
      cudaSuccess)
    return false;
  mask |= 1ull << dev;
  return true;
}

// Record a profiling event: as an event-record node of the graph while the stream is being
// captured, as a plain record otherwise.
void record_mark(cudaEvent_t ev, cudaStream_t st) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaStreamIsCapturing(st, &cs);
  if (cs == cudaStreamCaptureStatusActive)
    cudaEventRecordWithFlags(ev, st, cudaEventRecordExternal);
  else
    cudaEventRecord(ev, st);
}

// ------------------------------------------------------------------ tcgen05 GEMM launcher

int pick_bn(int n) {
  if (n <= 16) return 16;
  if (n <= 32) return 32;
  if (n <= 64) return 64;
  if (n <= 128) return 128;
  return 256;
}

template <int BN, class Epi>
mla_status launch_gemm_bn(const CUtensorMap& A, const CUtensorMap& B, const GemmShape& shp,
                          int m_tiles, int Z, const Epi& epi, cudaStream_t st) {
  auto kern = gemm_tc_kernel<BN, Epi>;
  constexpr int smem = gemm_smem_bytes<BN, Epi>();
  if (shp.m_per_cta < 1 || gemm_tmem_cols(BN, shp.m_per_cta) > 512) return MLA_ERR_UNSUPPORTED;
  if (!allow_smem(kern, smem)) return MLA_ERR_CUDA;
  const dim3 grid((m_tiles + shp.m_per_cta - 1) / shp.m_per_cta, (shp.N + BN - 1) / BN,
                  Z * shp.k_splits + shp.aux_blocks);
  kern<<<grid, 128, smem, st>>>(A, B, shp, epi);
  return last_launch_status();
}

// bn: the activation tile (16..256; pick_bn(N) unless a caller caps it).
template <class Epi>
mla_status launch_gemm(const CUtensorMap& A, const CUtensorMap& B, const GemmShape& shp,
                       int m_tiles, int Z, const Epi& epi, cudaStream_t st, int bn) {
  switch (bn) {
    case 16: return launch_gemm_bn<16>(A, B, shp, m_tiles, Z, epi, st);
    case 32: return launch_gemm_bn<32>(A, B, shp, m_tiles, Z, epi, st);
    case 64: return launch_gemm_bn<64>(A, B, shp, m_tiles, Z, epi, st);
    case 128: return launch_gemm_bn<128>(A, B, shp, m_tiles, Z, epi, st);
    default: return launch_gemm_bn<256>(A, B, shp, m_tiles, Z, epi, st);
  }
}

// Split-K plan of the append down-projection (identical in the size query and the call).
struct AppendPlan {
  int m_tiles, k_chunks, chunks_per_split, k_splits;
};
AppendPlan append_plan(const mla_config* c, int n_tok) {
  AppendPlan p{};
  const int row = c->d_c + c->d_rope;
  p.m_tiles = (row + 127) / 128;
  p.k_chunks = c->d_model / 64;
  const int n_tiles = (n_tok + 255) / 256;
  const int sms = device_sm_count() > 0 ? device_sm_count() : 148;
  // K-splits for about half the SMs (m_tiles x splits ~ SMs / 2): each CTA streams twice the
  // weights and the finish kernel sums half as many partials; measured faster overall on B200
  // than one CTA per SM
  int splits = (sms + 2 * p.m_tiles * n_tiles - 1) / (2 * p.m_tiles * n_tiles);
  splits = splits < 1 ? 1 : (splits > p.k_chunks ? p.k_chunks : splits);
  p.chunks_per_split = (p.k_chunks + splits - 1) / splits;
  p.k_splits = (p.k_chunks + p.chunks_per_split - 1) / p.chunks_per_split;
  return p;
}

// One thread per cache-row feature (a multiple of 32, at most 1024).
int finish_threads(int row) {
  const int t = (row + 31) / 32 * 32;
  return t > 1024 ? 1024 : t;
}

bool tc_append_shape(const mla_config* c) {
  return c->dtype == MLA_DTYPE_BF16 && c->d_model % 64 == 0;
}

// ------------------------------------------------------------------ decode workspace layout

struct DecodeLayout {
  int P, n_mt, R, U, max_segs;
  int32_t *unit_first, *unit_tiles, *unit_seg, *pair_seg;
  AttnSeg* segs;
  __nv_bfloat16* qhat;
  __nv_bfloat16* o_part;
  float* lse;
  uint8_t* qcodes;   // quantised cache only: the split query rows and their scales
  float* qalpha;
  size_t bytes;
};

// Number of CTA pairs of the attention kernel: one CTA per SM (its shared memory and TMEM fill
// an SM), two CTAs per pair.
int attn_pairs() {
  const int sms = device_sm_count();
  const int pairs = (sms >= 2 ? sms : 2) / 2;
  return pairs < ATT_MAX_PAIRS ? pairs : ATT_MAX_PAIRS;
}

DecodeLayout decode_layout_tc(const mla_config* c, int B, int Tq, void* ws) {
  DecodeLayout L{};
  L.P = attn_pairs();
  L.R = Tq * c->n_heads;
  L.n_mt = (L.R + 127) / 128;
  L.U = B * L.n_mt;
  L.max_segs = L.U + L.P;
  Carve cv(ws);
  L.unit_first = cv.take<int32_t>(L.U);
  L.unit_tiles = cv.take<int32_t>(L.U);
  L.unit_seg = cv.take<int32_t>(L.U + 1);
  L.pair_seg = cv.take<int32_t>(L.P + 1);
  L.segs = cv.take<AttnSeg>(L.max_segs);
  L.qhat = cv.take<__nv_bfloat16>(static_cast<size_t>(B) * L.R * ATT_ROW);
  L.o_part = cv.take<__nv_bfloat16>(static_cast<size_t>(L.max_segs) * 128 * ATT_DC);
  L.lse = cv.take<float>(static_cast<size_t>(L.max_segs) * 128);
  if (fp8_cache(c)) {
    L.qcodes = cv.take<uint8_t>(static_cast<size_t>(B) * L.R * F8_QROW_BYTES);
    L.qalpha = cv.take<float>(static_cast<size_t>(B) * L.R);
  }
  L.bytes = cv.off;
  return L;
}

struct SimtLayout {
  float *qhat, *o_lat, *kv;
  int32_t *seq_idx, *pos;
  size_t bytes;
};

SimtLayout simt_layout(const mla_config* c, int64_t rows, int64_t n_append_tok, void* ws) {
  SimtLayout L{};
  Carve cv(ws);
  L.kv = cv.take<float>(static_cast<size_t>(n_append_tok) * (c->d_c + c->d_rope));
  L.seq_idx = cv.take<int32_t>(static_cast<size_t>(n_append_tok));
  L.pos = cv.take<int32_t>(static_cast<size_t>(n_append_tok));
  L.qhat = cv.take<float>(static_cast<size_t>(rows) * (c->d_c + c->d_rope));
  L.o_lat = cv.take<float>(static_cast<size_t>(rows) * c->d_c);
  L.bytes = cv.off;
  return L;
}

// -------------------------------------------------------------------- SIMT decode (any T)

// keys: which keys each row sees; with o_lat_out given the latent output (O / l) goes there
// with its log-sum-exp in lse_out, and the value projection is skipped.
template <typename T>
mla_status simt_decode(const mla_config* c, const void* q, int B, int Tq, const void* cache,
                       int num_pages, const int32_t* block_table, int max_pages,
                       const int32_t* seq_lens, const void* w_uk_t, const void* w_uv,
                       const SimtLayout& L, void* out, cudaStream_t st,
                       void* const* events = nullptr, KeyRange keys = KeyRange{nullptr, nullptr, 0},
                       float* o_lat_out = nullptr, float* lse_out = nullptr) {
  auto mark = [&](int i) {
    if (events != nullptr && events[i] != nullptr)
      record_mark(static_cast<cudaEvent_t>(events[i]), st);
  };
  const int rows = B * Tq * c->n_heads;
  const int row = c->d_c + c->d_rope;
  const int max_pos = max_pages * c->page_size;
  if (keys.window == 0) keys.window = c->window;
  qabs_simt_kernel<T><<<rows, 256, (c->d_nope + c->d_rope) * sizeof(float), st>>>(
      static_cast<const T*>(q), static_cast<const T*>(w_uk_t), seq_lens, L.qhat, c->n_heads,
      Tq, c->d_c, c->d_rope, c->d_nope, max_pos, rope_freqs(c));
  const int attn_smem = (row + c->d_c) * static_cast<int>(sizeof(float));
  if (!allow_smem(attn_simt_kernel<T>, attn_smem)) return MLA_ERR_CUDA;
  mark(1);
  attn_simt_kernel<T><<<rows, 256, attn_smem, st>>>(
      L.qhat, static_cast<const T*>(cache), block_table, seq_lens,
      o_lat_out != nullptr ? o_lat_out : L.o_lat, c->n_heads, Tq, c->d_c, c->d_rope, max_pages,
      num_pages, c->page_size, c->softmax_scale, keys, lse_out);
  mark(2);
  if (o_lat_out != nullptr) return last_launch_status();
  outproj_simt_kernel<T><<<rows, 256, c->d_c * sizeof(float), st>>>(
      L.o_lat, static_cast<const T*>(w_uv), static_cast<T*>(out), c->n_heads, c->d_c, c->d_v);
  return last_launch_status();
}

template <typename T>
mla_status simt_append(const mla_config* c, const void* x, int n_tok, const void* w_dkv,
                       const void* kv_gain, const int32_t* seq_idx, const int32_t* pos,
                       const int32_t* block_table, int batch, int max_pages, void* cache,
                       int num_pages, float* kv, cudaStream_t st) {
  const int row = c->d_c + c->d_rope;
  const dim3 g1((row + 7) / 8, n_tok);
  linear_rows_kernel<T><<<g1, 256, 0, st>>>(static_cast<const T*>(x),
                                            static_cast<const T*>(w_dkv), kv, n_tok, row,
                                            c->d_model);
  append_finish_kernel<T><<<n_tok, finish_threads(row), row * sizeof(float), st>>>(
      kv, 1, n_tok, static_cast<const T*>(kv_gain), seq_idx, pos, block_table, batch,
      max_pages, static_cast<T*>(cache), num_pages, c->page_size, c->d_c, c->d_rope,
      c->rms_eps, rope_freqs(c));
  return last_launch_status();
}

__global__ void prefill_positions_kernel(const int32_t* __restrict__ seq_lens, int t_new,
                                         int n_tok, int32_t* __restrict__ seq_idx,
                                         int32_t* __restrict__ pos) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n_tok) return;
  const int b = i / t_new, t = i % t_new;
  seq_idx[i] = b;
  pos[i] = seq_lens[b] - t_new + t;  // out-of-range values are caught by the append kernel
}

// ------------------------------------------------------- q path and output projection plans

// Split-K plan of a weight-streaming GEMM with m_tiles x n_tiles output tiles and k_chunks
// 64-wide K chunks: enough K-splits that the grid covers about `ctas` CTAs (one per SM when
// ctas is the SM count), every split non-empty.
struct SplitPlan {
  int k_chunks, chunks_per_split, k_splits;
};
SplitPlan split_plan(int m_tiles, int n_tiles, int k_chunks, int ctas, bool round_up) {
  SplitPlan p{};
  p.k_chunks = k_chunks;
  const int tiles = m_tiles * n_tiles;
  int splits = round_up ? (ctas + tiles - 1) / tiles : ctas / tiles;
  splits = splits < 1 ? 1 : (splits > k_chunks ? k_chunks : splits);
  p.chunks_per_split = (k_chunks + splits - 1) / splits;
  p.k_splits = (k_chunks + p.chunks_per_split - 1) / p.chunks_per_split;
  return p;
}

int sm_count_or_default() {
  const int n = device_sm_count();
  return n > 0 ? n : 148;
}

bool tc_query_shape(const mla_config* c, int q_lora) {
  return c->dtype == MLA_DTYPE_BF16 && c->d_model % 64 == 0 && q_lora % 64 == 0;
}
bool tc_output_shape(const mla_config* c) {
  return c->dtype == MLA_DTYPE_BF16 && (c->n_heads * c->d_v) % 64 == 0;
}

struct QueryPlan {
  SplitPlan a;      // wq_a: M = q_lora, K = d_model
  int bn, n_tiles, m_tiles_a, m_tiles_b, m_per_cta_b;
};
QueryPlan query_plan(const mla_config* c, int q_lora, int n_tok) {
  QueryPlan p{};
  p.bn = pick_bn(n_tok);
  p.n_tiles = (n_tok + p.bn - 1) / p.bn;
  p.m_tiles_a = (q_lora + 127) / 128;
  p.a = split_plan(p.m_tiles_a, p.n_tiles, c->d_model / 64, sm_count_or_default(), true);
  const int M_b = c->n_heads * (c->d_nope + c->d_rope);
  p.m_tiles_b = (M_b + 127) / 128;
  // wq_b: consecutive m-tiles per CTA so that one wave of CTAs covers the weight
  int per = (p.m_tiles_b * p.n_tiles + sm_count_or_default() - 1) / sm_count_or_default();
  while (per > 1 && p.bn * per > 512) --per;   // the accumulators must fit TMEM
  p.m_per_cta_b = per < 1 ? 1 : per;
  return p;
}

struct QueryLayout {
  float* partial;   // [splits][n_tok][q_lora] (tensor-core path) or [n_tok][q_lora] (SIMT)
  void* qa;         // [n_tok][q_lora] in cfg->dtype
  float* q32;       // [n_tok][M_b] fp32 (SIMT path only)
  size_t bytes;
};
QueryLayout query_layout(const mla_config* c, int q_lora, int n_tok, void* ws) {
  QueryLayout L{};
  Carve cv(ws);
  const size_t M_b = static_cast<size_t>(c->n_heads) * (c->d_nope + c->d_rope);
  if (tc_query_shape(c, q_lora)) {
    const QueryPlan p = query_plan(c, q_lora, n_tok);
    L.partial = cv.take<float>(static_cast<size_t>(p.a.k_splits) * n_tok * q_lora);
    L.qa = cv.take<__nv_bfloat16>(static_cast<size_t>(n_tok) * q_lora);
  } else {
    L.partial = cv.take<float>(static_cast<size_t>(n_tok) * q_lora);
    L.qa = cv.take<float>(static_cast<size_t>(n_tok) * q_lora);   // room for either dtype
    L.q32 = cv.take<float>(static_cast<size_t>(n_tok) * M_b);
  }
  L.bytes = cv.off;
  return L;
}

struct OutputPlan {
  SplitPlan s;
  int bn, n_tiles, m_tiles;
};
OutputPlan output_plan(const mla_config* c, int n_tok) {
  OutputPlan p{};
  p.bn = pick_bn(n_tok);
  p.n_tiles = (n_tok + p.bn - 1) / p.bn;
  p.m_tiles = (c->d_model + 127) / 128;
  // as many K-splits as keep the grid within one wave of CTAs
  p.s = split_plan(p.m_tiles, p.n_tiles, c->n_heads * c->d_v / 64, sm_count_or_default(), false);
  return p;
}
size_t output_ws_bytes(const mla_config* c, int n_tok) {
  const size_t per = static_cast<size_t>(n_tok) * c->d_model;
  if (tc_output_shape(c)) return align_up(static_cast<size_t>(output_plan(c, n_tok).s.k_splits) * per * sizeof(float));
  return align_up(per * sizeof(float));
}

// Launch a bf16 tensor-core GEMM D = W · Xᵀ: W [M, K] weights (K contiguous), X [N, K]
// activations, epilogue epi; m_per_cta consecutive m-tiles per CTA, K split as in sp.
template <class Epi>
mla_status weight_gemm(const void* w, int M, int K, const void* x, int N, const SplitPlan& sp,
                       int m_per_cta, int bn, const Epi& epi, cudaStream_t st) {
  CUtensorMap mA, mB;
  const uint64_t da[3] = {static_cast<uint64_t>(K), static_cast<uint64_t>(M), 1};
  const uint64_t sa[2] = {static_cast<uint64_t>(K) * 2, static_cast<uint64_t>(K) * 2 * M};
  const uint32_t ba[3] = {64, 128, 1};
  const uint64_t db[3] = {static_cast<uint64_t>(K), 1, static_cast<uint64_t>(N)};
  const uint64_t sb[2] = {static_cast<uint64_t>(K) * 2, static_cast<uint64_t>(K) * 2};
  const uint32_t bb[3] = {64, 1, static_cast<uint32_t>(bn)};
  if (!make_map(&mA, w, 3, da, sa, ba) || !make_map(&mB, x, 3, db, sb, bb)) return MLA_ERR_CUDA;
  GemmShape shp{M, N, sp.k_chunks, sp.chunks_per_split, sp.k_splits, 0, m_per_cta, 0};
  return launch_gemm(mA, mB, shp, (M + 127) / 128, 1, epi, st, bn);
}

// The split merge fused with the value projection (vproj_merge_kernel) over the rows of p;
// pdl: launched with programmatic dependent launch (it follows the library's own kernel).
mla_status launch_vproj(const mla_config* cfg, const void* w_uv, const VprojParams& vp,
                        cudaStream_t st, bool pdl) {
  CUtensorMap mA;
  const int H = cfg->n_heads;
  const uint64_t da[3] = {ATT_DC, static_cast<uint64_t>(cfg->d_v), static_cast<uint64_t>(H)};
  const uint64_t sa[2] = {ATT_DC * 2, static_cast<uint64_t>(ATT_DC) * 2 * cfg->d_v};
  const uint32_t ba[3] = {64, 128, 1};
  if (!make_map(&mA, w_uv, 3, da, sa, ba)) return MLA_ERR_CUDA;
  const int n_q = vp.n_q;
  const int bn = pick_bn(n_q) > 64 ? 64 : pick_bn(n_q);
  const dim3 grid((cfg->d_v + 127) / 128, (n_q + bn - 1) / bn, H);
  auto go = [&](auto kern, int smem) -> mla_status {
    if (!allow_smem(kern, smem)) return MLA_ERR_CUDA;
    if (pdl) return launch_pdl(kern, grid, dim3(VP_THREADS), smem, st, mA, vp);
    kern<<<grid, VP_THREADS, smem, st>>>(mA, vp);
    return last_launch_status();
  };
  switch (bn) {
    case 16: return go(vproj_merge_kernel<16>, vproj_smem_bytes<16>());
    case 32: return go(vproj_merge_kernel<32>, vproj_smem_bytes<32>());
    default: return go(vproj_merge_kernel<64>, vproj_smem_bytes<64>());
  }
}

}  // namespace

// ====================================================================== exported functions

extern "C" {

const char* mla_status_string(mla_status s) {
  switch (s) {
    case MLA_OK: return "MLA_OK";
    case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG";
    case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED";
    case MLA_ERR_WORKSPACE_TOO_SMALL: return "MLA_ERR_WORKSPACE_TOO_SMALL";
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA";
    case MLA_ERR_DEVICE_TIMEOUT: return "MLA_ERR_DEVICE_TIMEOUT";
    case MLA_ERR_DEVICE_OOB: return "MLA_ERR_DEVICE_OOB";
    case MLA_ERR_DEVICE_BAD_LENGTH: return "MLA_ERR_DEVICE_BAD_LENGTH";
  }
  return "MLA_ERR_UNKNOWN";
}

mla_status mla_absorb_weights(const mla_config* cfg, const void* wkv_b, void* w_uk_t,
                              void* w_uv, void* stream) {
  NvtxRange nvtx_range("mla_absorb_weights");
  const mla_status cs = check_config(cfg);
  if (cs != MLA_OK) return cs;
  if (wkv_b == nullptr || w_uk_t == nullptr || w_uv == nullptr) return MLA_ERR_INVALID_ARG;
  if (!aligned16(wkv_b) || !aligned16(w_uk_t) || !aligned16(w_uv)) return MLA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t total = static_cast<int64_t>(cfg->n_heads) * (cfg->d_nope + cfg->d_v) * cfg->d_c;
  const int blocks = static_cast<int>((total + 255) / 256 < 65535 * 8 ? (total + 255) / 256 : 65535 * 8);
  if (cfg->dtype == MLA_DTYPE_F32)
    absorb_kernel<float><<<blocks, 256, 0, st>>>(static_cast<const float*>(wkv_b),
                                                 static_cast<float*>(w_uk_t),
                                                 static_cast<float*>(w_uv), cfg->n_heads,
                                                 cfg->d_c, cfg->d_nope, cfg->d_v);
  else
    absorb_kernel<__nv_bfloat16><<<blocks, 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(wkv_b), static_cast<__nv_bfloat16*>(w_uk_t),
        static_cast<__nv_bfloat16*>(w_uv), cfg->n_heads, cfg->d_c, cfg->d_nope, cfg->d_v);
  return last_launch_status();
}

size_t mla_append_workspace_size(const mla_config* cfg, int32_t n_tok) {
  if (check_config(cfg) != MLA_OK || n_tok < 1) return 0;
  const size_t row = static_cast<size_t>(cfg->d_c + cfg->d_rope);
  if (cfg->dtype == MLA_DTYPE_BF16) {
    if (!tc_append_shape(cfg)) return 0;
    const AppendPlan p = append_plan(cfg, n_tok);
    return align_up(static_cast<size_t>(p.k_splits) * n_tok * row * sizeof(float));
  }
  return align_up(static_cast<size_t>(n_tok) * row * sizeof(float));
}

mla_status mla_append_latent(const mla_config* cfg, const void* x, int32_t n_tok,
                             const void* w_dkv, const void* kv_gain, const int32_t* seq_idx,
                             const int32_t* pos, const int32_t* block_table, int32_t batch,
                             int32_t max_pages, void* cache, int32_t num_pages, void* workspace,
                             size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("mla_append_latent");
  const mla_status cs = check_config(cfg);
  if (cs != MLA_OK) return cs;
  if (n_tok < 1 || batch < 1 || max_pages < 1 || num_pages < 1) return MLA_ERR_INVALID_ARG;
  const void* ptrs[] = {x, w_dkv, kv_gain, seq_idx, pos, block_table, cache, workspace};
  for (const void* p : ptrs)
    if (p == nullptr || !aligned16(p)) return MLA_ERR_INVALID_ARG;
  if (cfg->dtype == MLA_DTYPE_BF16 && !tc_append_shape(cfg)) return MLA_ERR_UNSUPPORTED;
  if (ws_bytes < mla_append_workspace_size(cfg, n_tok)) return MLA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int row = cfg->d_c + cfg->d_rope;
  if (cfg->dtype == MLA_DTYPE_F32)
    return simt_append<float>(cfg, x, n_tok, w_dkv, kv_gain, seq_idx, pos, block_table, batch,
                              max_pages, cache, num_pages, static_cast<float*>(workspace), st);

  // bf16: tcgen05 split-K GEMM kv = x · w_dkvᵀ, then norm / RoPE / scatter per token
  const AppendPlan ap = append_plan(cfg, n_tok);
  CUtensorMap mA, mB;
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(cfg->d_model), static_cast<uint64_t>(row), 1};
    const uint64_t strides[2] = {static_cast<uint64_t>(cfg->d_model) * 2,
                                 static_cast<uint64_t>(cfg->d_model) * 2 * row};
    const uint32_t box[3] = {64, 128, 1};
    if (!make_map(&mA, w_dkv, 3, dims, strides, box)) return MLA_ERR_CUDA;
  }
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(cfg->d_model), 1, static_cast<uint64_t>(n_tok)};
    const uint64_t strides[2] = {static_cast<uint64_t>(cfg->d_model) * 2,
                                 static_cast<uint64_t>(cfg->d_model) * 2};
    const uint32_t box[3] = {64, 1, static_cast<uint32_t>(pick_bn(n_tok))};
    if (!make_map(&mB, x, 3, dims, strides, box)) return MLA_ERR_CUDA;
  }
  float* partial = static_cast<float*>(workspace);
  GemmShape shp{row, n_tok, ap.k_chunks, ap.chunks_per_split, ap.k_splits, 0, 1, 0};
  EpiSplitK epi{partial, n_tok, row};
  mla_status s = launch_gemm(mA, mB, shp, ap.m_tiles, 1, epi, st, pick_bn(n_tok));
  if (s != MLA_OK) return s;
  // the finish runs as clusters of FIN_CLUSTER CTAs per token (see append_finish_cluster_kernel)
  const int per = (((row + FIN_CLUSTER - 1) / FIN_CLUSTER) + 1) & ~1;
  if (fp8_cache(cfg))
    return launch_pdl_clustered(append_finish_cluster_fp8_kernel<FIN_CLUSTER>,
                                dim3(static_cast<unsigned>(n_tok) * FIN_CLUSTER), dim3(FIN_THREADS),
                                per * sizeof(float), st, FIN_CLUSTER,
                                static_cast<const float*>(partial), ap.k_splits, n_tok,
                                static_cast<const __nv_bfloat16*>(kv_gain), seq_idx, pos,
                                block_table, batch, max_pages, static_cast<uint8_t*>(cache),
                                num_pages, cfg->page_size, cfg->d_c, cfg->d_rope, cfg->rms_eps,
                                rope_freqs(cfg));
  return launch_pdl_clustered(append_finish_cluster_kernel<__nv_bfloat16>,
                              dim3(static_cast<unsigned>(n_tok) * FIN_CLUSTER), dim3(FIN_THREADS),
                              per * sizeof(float), st, FIN_CLUSTER,
                              static_cast<const float*>(partial), ap.k_splits, n_tok,
                              static_cast<const __nv_bfloat16*>(kv_gain), seq_idx, pos,
                              block_table, batch, max_pages, static_cast<__nv_bfloat16*>(cache),
                              num_pages, cfg->page_size, cfg->d_c, cfg->d_rope, cfg->rms_eps,
                              rope_freqs(cfg));
}

mla_status mla_quantize_latent(const mla_config* cfg, const float* rows, int32_t n_tok,
                               const int32_t* seq_idx, const int32_t* pos,
                               const int32_t* block_table, int32_t batch, int32_t max_pages,
                               void* cache, int32_t num_pages, void* stream) {
  NvtxRange nvtx_range("mla_quantize_latent");
  const mla_status cs = check_config(cfg);
  if (cs != MLA_OK) return cs;
  if (!fp8_cache(cfg)) return MLA_ERR_INVALID_ARG;
  if (n_tok < 1 || batch < 1 || max_pages < 1 || num_pages < 1) return MLA_ERR_INVALID_ARG;
  const void* ptrs[] = {rows, seq_idx, pos, block_table, cache};
  for (const void* p : ptrs)
    if (p == nullptr || !aligned16(p)) return MLA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  quantize_rows_kernel<<<n_tok, 128, 0, st>>>(rows, n_tok, cfg->d_c + cfg->d_rope, seq_idx, pos,
                                              block_table, batch, max_pages,
                                              static_cast<uint8_t*>(cache), num_pages,
                                              cfg->page_size);
  return last_launch_status();
}

size_t mla_decode_workspace_size(const mla_config* cfg, int32_t batch, int32_t tq) {
  if (check_config(cfg) != MLA_OK || batch < 1 || tq < 1) return 0;
  if (cfg->dtype == MLA_DTYPE_BF16) {
    if (!tc_decode_shape(cfg)) return 0;
    return decode_layout_tc(cfg, batch, tq, nullptr).bytes;
  }
  return simt_layout(cfg, static_cast<int64_t>(batch) * tq * cfg->n_heads, 0, nullptr).bytes;
}

// mla_decode and its variants. kv_begin / kv_end (optional) restrict the keys read; with
// part_out given the result is the merged latent output O / l of each row (and lse_out its
// natural-log log-sum-exp) instead of the projected output, and w_uv / out are not used.
static mla_status decode_impl(const mla_config* cfg, const void* q, int32_t batch, int32_t tq,
                              const void* cache, int32_t num_pages, const int32_t* block_table,
                              int32_t max_pages, const int32_t* seq_lens, const void* w_uk_t,
                              const void* w_uv, void* workspace, size_t ws_bytes, void* out,
                              void* stream, void* const* events,
                              const int32_t* kv_begin = nullptr, const int32_t* kv_end = nullptr,
                              void* part_out = nullptr, float* lse_out = nullptr) {
  const mla_status cs = check_config(cfg);
  if (cs != MLA_OK) return cs;
  if (batch < 1 || tq < 1 || num_pages < 1 || max_pages < 1) return MLA_ERR_INVALID_ARG;
  const bool partial = part_out != nullptr;
  const void* ptrs[] = {q, cache, block_table, seq_lens, w_uk_t, workspace,
                        partial ? part_out : out, partial ? static_cast<void*>(lse_out) : w_uv};
  for (const void* p : ptrs)
    if (p == nullptr || !aligned16(p)) return MLA_ERR_INVALID_ARG;
  if ((kv_begin == nullptr) != (kv_end == nullptr)) return MLA_ERR_INVALID_ARG;
  const KeyRange keys{kv_begin, kv_end, cfg->window};
  if (static_cast<int64_t>(max_pages) * cfg->page_size > (1 << 30)) return MLA_ERR_INVALID_ARG;
  if (cfg->dtype == MLA_DTYPE_BF16 && !tc_decode_shape(cfg)) return MLA_ERR_UNSUPPORTED;
  if (ws_bytes < mla_decode_workspace_size(cfg, batch, tq)) return MLA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // events[i] (if given): [0] before the query absorption (which also plans the split-KV
  // work), [1] before the attention kernel, [2] before the merge + value projection, [3] after.
  auto mark = [&](int i) {
    if (events != nullptr && events[i] != nullptr)
      record_mark(static_cast<cudaEvent_t>(events[i]), st);
  };

  if (cfg->dtype == MLA_DTYPE_F32) {
    const SimtLayout L = simt_layout(cfg, static_cast<int64_t>(batch) * tq * cfg->n_heads, 0, workspace);
    mark(0);
    const mla_status s = simt_decode<float>(cfg, q, batch, tq, cache, num_pages, block_table,
                                            max_pages, seq_lens, w_uk_t, w_uv, L, out, st,
                                            events, keys, static_cast<float*>(part_out), lse_out);
    mark(3);
    return s;
  }

  const DecodeLayout L = decode_layout_tc(cfg, batch, tq, workspace);
  const int H = cfg->n_heads;
  const int n_q = batch * tq;                 // query tokens
  const int max_pos = max_pages * ATT_PAGE;
  const int qrow = cfg->d_nope + cfg->d_rope;

  // (1) Q̂ = [q_nope · W_UK | RoPE(q_rope)], one CTA per head and token tile (all 4 m-tiles of
  //     d_c); one extra block plans the split-KV work list. Launched normally: the call's
  //     inputs may come from the kernel just before it.
  mark(0);
  {
    CUtensorMap mA, mB;
    const uint64_t da[3] = {static_cast<uint64_t>(cfg->d_nope), ATT_DC, static_cast<uint64_t>(H)};
    const uint64_t sa[2] = {static_cast<uint64_t>(cfg->d_nope) * 2,
                            static_cast<uint64_t>(cfg->d_nope) * 2 * ATT_DC};
    const uint32_t ba[3] = {64, 128, 1};
    const uint64_t db[3] = {static_cast<uint64_t>(qrow), static_cast<uint64_t>(H),
                            static_cast<uint64_t>(n_q)};
    const uint64_t sb[2] = {static_cast<uint64_t>(qrow) * 2, static_cast<uint64_t>(qrow) * 2 * H};
    // at most 128 tokens per CTA: 4 accumulators of bn columns fill TMEM's 512
    const int bn = pick_bn(n_q) > 128 ? 128 : pick_bn(n_q);
    const uint32_t bb[3] = {64, 1, static_cast<uint32_t>(bn)};
    if (!make_map(&mA, w_uk_t, 3, da, sa, ba) || !make_map(&mB, q, 3, db, sb, bb))
      return MLA_ERR_CUDA;
    const int m_per_cta = ATT_DC / 128;
    // q_rope turns: one thread per (token, rotary pair), at most 16 blocks (the SMs the H head
    // CTAs leave free)
    const int rope_items = n_q * (ATT_DR / 2);
    const int rope_blocks = std::min(16, (rope_items + 127) / 128);
    GemmShape shp{ATT_DC, n_q, cfg->d_nope / 64, cfg->d_nope / 64, 1, 1, m_per_cta,
                  1 + rope_blocks};
    PlanParams pp{seq_lens, batch, tq, H, L.n_mt, max_pos, L.P, L.max_segs, keys,
                  L.unit_first, L.unit_tiles, L.unit_seg, L.pair_seg, L.segs};
    EpiQhat epi{L.qhat, static_cast<const __nv_bfloat16*>(q), seq_lens, H, tq, ATT_DC, ATT_DR,
                cfg->d_nope, n_q, max_pos, rope_blocks, pp, rope_freqs(cfg)};
    const mla_status s = launch_gemm(mA, mB, shp, ATT_DC / 128, H, epi, st, bn);
    if (s != MLA_OK) return s;
  }

  // (2) fused latent attention, one partial per segment
  if (fp8_cache(cfg)) {
    // codes as [page][chunk of 128][token][128 codes] (two chunks per box) and the k_R codes as
    // [page][token][64 codes] starting 512 bytes into the page; the scales follow the codes
    CUtensorMap mc8, mr8;
    const uint64_t dc[4] = {128, ATT_PAGE, ATT_DC / 128, static_cast<uint64_t>(num_pages)};
    const uint64_t sc[3] = {ATT_ROW, 128, F8_PAGE_BYTES};
    const uint32_t bc[4] = {128, ATT_PAGE, 2, 1};
    const uint64_t dr[3] = {ATT_DR, ATT_PAGE, static_cast<uint64_t>(num_pages)};
    const uint64_t sr[2] = {ATT_ROW, F8_PAGE_BYTES};
    const uint32_t br[3] = {ATT_DR, ATT_PAGE, 1};
    // the split query rows: [row][1152 bytes], five 128-byte chunks per box row
    CUtensorMap mq8;
    const uint64_t dq[2] = {F8_QROW_BYTES, static_cast<uint64_t>(batch) * L.R};
    const uint64_t sq[1] = {F8_QROW_BYTES};
    const uint32_t bq[2] = {128, 128};
    const uint8_t* c8 = static_cast<const uint8_t*>(cache);
    if (!make_map(&mc8, c8, 4, dc, sc, bc, CU_TENSOR_MAP_DATA_TYPE_UINT8, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mr8, c8 + ATT_DC, 3, dr, sr, br, CU_TENSOR_MAP_DATA_TYPE_UINT8,
                  CU_TENSOR_MAP_SWIZZLE_64B) ||
        !make_map(&mq8, L.qcodes, 2, dq, sq, bq, CU_TENSOR_MAP_DATA_TYPE_UINT8,
                  CU_TENSOR_MAP_SWIZZLE_128B))
      return MLA_ERR_CUDA;
    // Q̂ rows -> their high and low E4M3 parts and row scales
    const int n_rows = batch * L.R;
    mla_status s = launch_pdl(qsplit_rows_kernel, dim3((n_rows + 7) / 8), dim3(256), 0, st,
                              static_cast<const __nv_bfloat16*>(L.qhat), n_rows, L.qcodes, L.qalpha);
    if (s != MLA_OK) return s;
    AttnParams ap{block_table, seq_lens, L.segs, L.pair_seg, L.qhat, L.o_part, L.lse,
                  max_pages, num_pages, H, tq, L.R, L.n_mt,
                  cfg->softmax_scale * 1.4426950408889634f, keys, c8, L.qcodes, L.qalpha};
    if (!allow_smem(mla_decode_attn_fp8_kernel, F8_SMEM_BYTES)) return MLA_ERR_CUDA;
    mark(1);
    s = launch_pdl(mla_decode_attn_fp8_kernel, dim3(2 * L.P), dim3(F8_THREADS), F8_SMEM_BYTES, st,
                   mc8, mr8, mq8, ap);
    if (s != MLA_OK) return s;
  } else {
    CUtensorMap mc, mc4, mq;
    const uint64_t dc[2] = {ATT_ROW, static_cast<uint64_t>(num_pages) * ATT_PAGE};
    const uint64_t sc[1] = {ATT_ROW * 2};
    const uint32_t bc[2] = {64, ATT_PAGE};
    // the same cache as [chunk of 64 dims][token][64 dims], 4 chunks of one page per box
    const uint64_t dc4[3] = {64, static_cast<uint64_t>(num_pages) * ATT_PAGE, ATT_ROW / 64};
    const uint64_t sc4[2] = {ATT_ROW * 2, 128};
    const uint32_t bc4[3] = {64, ATT_PAGE, 4};
    const uint64_t dq[2] = {ATT_ROW, static_cast<uint64_t>(batch) * L.R};
    const uint32_t bq[2] = {64, 128};
    if (!make_map(&mc, cache, 2, dc, sc, bc) || !make_map(&mc4, cache, 3, dc4, sc4, bc4) ||
        !make_map(&mq, L.qhat, 2, dq, sc, bq))
      return MLA_ERR_CUDA;
    AttnParams ap{block_table, seq_lens, L.segs, L.pair_seg, L.qhat, L.o_part, L.lse,
                  max_pages, num_pages, H, tq, L.R, L.n_mt,
                  cfg->softmax_scale * 1.4426950408889634f, keys, nullptr, nullptr, nullptr};
    if (!allow_smem(mla_decode_attn_kernel, ATT_SMEM_BYTES)) return MLA_ERR_CUDA;
    mark(1);
    const mla_status s = launch_pdl(mla_decode_attn_kernel, dim3(2 * L.P), dim3(ATT_THREADS),
                                    ATT_SMEM_BYTES, st, mc, mc4, mq, ap);
    if (s != MLA_OK) return s;
  }

  // (3a) partial decode: merge each row's segments into one partial and its lse
  if (partial) {
    mark(2);
    const int rows = batch * L.R;
    const mla_status s = launch_pdl(merge_partials_kernel, dim3((rows + 3) / 4), dim3(256), 0, st,
                                    static_cast<const __nv_bfloat16*>(L.o_part),
                                    static_cast<const float*>(L.lse),
                                    static_cast<const int32_t*>(L.unit_seg), rows, L.R,
                                    static_cast<__nv_bfloat16*>(part_out), lse_out);
    mark(3);
    return s;
  }
  // (3) merge the split partials and project: out = o_lat · W_UVᵀ per head
  VprojParams vp{L.o_part, L.lse, L.unit_seg, static_cast<__nv_bfloat16*>(out), H, tq, L.n_mt,
                 n_q, cfg->d_v, 0};
  mark(2);
  const mla_status s = launch_vproj(cfg, w_uv, vp, st, true);
  mark(3);
  return s;
}

mla_status mla_decode(const mla_config* cfg, const void* q, int32_t batch, int32_t tq,
                      const void* cache, int32_t num_pages, const int32_t* block_table,
                      int32_t max_pages, const int32_t* seq_lens, const void* w_uk_t,
                      const void* w_uv, void* workspace, size_t ws_bytes, void* out,
                      void* stream) {
  NvtxRange nvtx_range("mla_decode");
  return decode_impl(cfg, q, batch, tq, cache, num_pages, block_table, max_pages, seq_lens,
                     w_uk_t, w_uv, workspace, ws_bytes, out, stream, nullptr);
}

mla_status mla_decode_profiled(const mla_config* cfg, const void* q, int32_t batch, int32_t tq,
                               const void* cache, int32_t num_pages, const int32_t* block_table,
                               int32_t max_pages, const int32_t* seq_lens, const void* w_uk_t,
                               const void* w_uv, void* workspace, size_t ws_bytes, void* out,
                               void* stream, void* const* events) {
  NvtxRange nvtx_range("mla_decode_profiled");
  if (events == nullptr) return MLA_ERR_INVALID_ARG;
  return decode_impl(cfg, q, batch, tq, cache, num_pages, block_table, max_pages, seq_lens,
                     w_uk_t, w_uv, workspace, ws_bytes, out, stream, events);
}

size_t mla_query_workspace_size(const mla_config* cfg, int32_t q_lora, int32_t n_tok) {
  if (check_config(cfg) != MLA_OK || q_lora < 1 || n_tok < 1) return 0;
  return query_layout(cfg, q_lora, n_tok, nullptr).bytes;
}

mla_status mla_query(const mla_config* cfg, int32_t q_lora, const void* x, int32_t n_tok,
                     const void* w_qa, const void* q_gain, const void* w_qb, void* workspace,
                     size_t ws_bytes, void* q_out, void* stream) {
  NvtxRange nvtx_range("mla_query");
  const mla_status cs = check_config(cfg);
  if (cs != MLA_OK) return cs;
  if (q_lora < 1 || n_tok < 1 || n_tok > 65535) return MLA_ERR_INVALID_ARG;
  const void* ptrs[] = {x, w_qa, q_gain, w_qb, workspace, q_out};
  for (const void* p : ptrs)
    if (p == nullptr || !aligned16(p)) return MLA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(q_lora) * elem_bytes(cfg) % 16 != 0 ||
      static_cast<int64_t>(cfg->d_model) * elem_bytes(cfg) % 16 != 0)
    return MLA_ERR_UNSUPPORTED;
  if (ws_bytes < mla_query_workspace_size(cfg, q_lora, n_tok)) return MLA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const QueryLayout L = query_layout(cfg, q_lora, n_tok, workspace);
  const int M_b = cfg->n_heads * (cfg->d_nope + cfg->d_rope);
  const size_t rms_smem = static_cast<size_t>(q_lora) * sizeof(float);
  if (rms_smem > 200 * 1024) return MLA_ERR_UNSUPPORTED;
  if (tc_query_shape(cfg, q_lora)) {
    // (1) q_a partial sums = x · w_qaᵀ, split over K; (2) sum + q_norm -> bf16 q_a;
    // (3) q = q_a · w_qbᵀ -> bf16
    const QueryPlan p = query_plan(cfg, q_lora, n_tok);
    mla_status s = weight_gemm(w_qa, q_lora, cfg->d_model, x, n_tok, p.a, 1, p.bn,
                               EpiSplitK{L.partial, n_tok, q_lora}, st);
    if (s != MLA_OK) return s;
    if (!allow_smem(rms_rows_kernel<__nv_bfloat16>, static_cast<int>(rms_smem))) return MLA_ERR_CUDA;
    s = launch_pdl(rms_rows_kernel<__nv_bfloat16>, dim3(n_tok), dim3(256), rms_smem, st,
                   static_cast<const float*>(L.partial), p.a.k_splits, static_cast<int>(n_tok),
                   static_cast<int>(q_lora), static_cast<const __nv_bfloat16*>(q_gain),
                   cfg->rms_eps, static_cast<__nv_bfloat16*>(L.qa));
    if (s != MLA_OK) return s;
    const SplitPlan sb = split_plan(1, 1, q_lora / 64, 1, false);   // whole K per CTA
    return weight_gemm(w_qb, M_b, q_lora, L.qa, n_tok, sb, p.m_per_cta_b, p.bn,
                       EpiStoreBf16{static_cast<__nv_bfloat16*>(q_out), M_b}, st);
  }
  // CUDA cores: fp32 sums, the same roundings
  auto run = [&](auto tag) -> mla_status {
    using T = decltype(tag);
    linear_rows_kernel<T><<<dim3((q_lora + 7) / 8, n_tok), 256, 0, st>>>(
        static_cast<const T*>(x), static_cast<const T*>(w_qa), L.partial, n_tok, q_lora,
        cfg->d_model);
    if (!allow_smem(rms_rows_kernel<T>, static_cast<int>(rms_smem))) return MLA_ERR_CUDA;
    rms_rows_kernel<T><<<n_tok, 256, rms_smem, st>>>(L.partial, 1, n_tok, q_lora,
                                                      static_cast<const T*>(q_gain),
                                                      cfg->rms_eps, static_cast<T*>(L.qa));
    linear_rows_kernel<T><<<dim3((M_b + 7) / 8, n_tok), 256, 0, st>>>(
        static_cast<const T*>(L.qa), static_cast<const T*>(w_qb), L.q32, n_tok, M_b, q_lora);
    const int64_t count = static_cast<int64_t>(n_tok) * M_b;
    round_rows_kernel<T><<<static_cast<int>((count + 255) / 256 < 4096 ? (count + 255) / 256 : 4096),
                           256, 0, st>>>(L.q32, count, static_cast<T*>(q_out));
    return last_launch_status();
  };
  return cfg->dtype == MLA_DTYPE_F32 ? run(float{}) : run(__nv_bfloat16{});
}

size_t mla_output_workspace_size(const mla_config* cfg, int32_t n_tok) {
  if (check_config(cfg) != MLA_OK || n_tok < 1) return 0;
  return output_ws_bytes(cfg, n_tok);
}

mla_status mla_output(const mla_config* cfg, const void* attn, int32_t n_tok, const void* w_o,
                      void* workspace, size_t ws_bytes, void* y, void* stream) {
  NvtxRange nvtx_range("mla_output");
  const mla_status cs = check_config(cfg);
  if (cs != MLA_OK) return cs;
  if (n_tok < 1 || n_tok > 65535) return MLA_ERR_INVALID_ARG;
  const void* ptrs[] = {attn, w_o, workspace, y};
  for (const void* p : ptrs)
    if (p == nullptr || !aligned16(p)) return MLA_ERR_INVALID_ARG;
  const int K = cfg->n_heads * cfg->d_v;
  if (static_cast<int64_t>(K) * elem_bytes(cfg) % 16 != 0) return MLA_ERR_UNSUPPORTED;
  if (ws_bytes < mla_output_workspace_size(cfg, n_tok)) return MLA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* partial = static_cast<float*>(workspace);
  const int64_t count = static_cast<int64_t>(n_tok) * cfg->d_model;
  const int sum_blocks = static_cast<int>((count + 255) / 256 < 4096 ? (count + 255) / 256 : 4096);
  if (tc_output_shape(cfg)) {
    const OutputPlan p = output_plan(cfg, n_tok);
    const mla_status s = weight_gemm(w_o, cfg->d_model, K, attn, n_tok, p.s, 1, p.bn,
                                     EpiSplitK{partial, n_tok, cfg->d_model}, st);
    if (s != MLA_OK) return s;
    return launch_pdl(sum_splits_kernel<__nv_bfloat16>, dim3(sum_blocks), dim3(256), 0, st,
                      static_cast<const float*>(partial), p.s.k_splits, count,
                      static_cast<__nv_bfloat16*>(y));
  }
  auto run = [&](auto tag) -> mla_status {
    using T = decltype(tag);
    linear_rows_kernel<T><<<dim3((cfg->d_model + 7) / 8, n_tok), 256, 0, st>>>(
        static_cast<const T*>(attn), static_cast<const T*>(w_o), partial, n_tok, cfg->d_model, K);
    sum_splits_kernel<T><<<sum_blocks, 256, 0, st>>>(partial, 1, count, static_cast<T*>(y));
    return last_launch_status();
  };
  return cfg->dtype == MLA_DTYPE_F32 ? run(float{}) : run(__nv_bfloat16{});
}

mla_status mla_decode_partial(const mla_config* cfg, const void* q, int32_t batch, int32_t tq,
                              const void* cache, int32_t num_pages, const int32_t* block_table,
                              int32_t max_pages, const int32_t* seq_lens,
                              const int32_t* kv_begin, const int32_t* kv_end, const void* w_uk_t,
                              void* workspace, size_t ws_bytes, void* o_part, float* lse,
                              void* stream) {
  NvtxRange nvtx_range("mla_decode_partial");
  if (kv_begin == nullptr || kv_end == nullptr || o_part == nullptr || lse == nullptr)
    return MLA_ERR_INVALID_ARG;
  if (!aligned16(kv_begin) || !aligned16(kv_end)) return MLA_ERR_INVALID_ARG;
  return decode_impl(cfg, q, batch, tq, cache, num_pages, block_table, max_pages, seq_lens,
                     w_uk_t, nullptr, workspace, ws_bytes, nullptr, stream, nullptr, kv_begin,
                     kv_end, o_part, lse);
}

size_t mla_combine_workspace_size(const mla_config* cfg, int32_t batch, int32_t tq) {
  if (check_config(cfg) != MLA_OK || batch < 1 || tq < 1) return 0;
  if (tc_decode_shape(cfg)) return 0;
  return align_up(static_cast<size_t>(batch) * tq * cfg->n_heads * cfg->d_c * sizeof(float));
}

mla_status mla_combine(const mla_config* cfg, int32_t n_parts, int32_t batch, int32_t tq,
                       const void* o_parts, const float* lse_parts, const void* w_uv,
                       void* workspace, size_t ws_bytes, void* out, void* stream) {
  NvtxRange nvtx_range("mla_combine");
  const mla_status cs = check_config(cfg);
  if (cs != MLA_OK) return cs;
  if (n_parts < 1 || batch < 1 || tq < 1) return MLA_ERR_INVALID_ARG;
  const void* ptrs[] = {o_parts, lse_parts, w_uv, out};
  for (const void* p : ptrs)
    if (p == nullptr || !aligned16(p)) return MLA_ERR_INVALID_ARG;
  const size_t need = mla_combine_workspace_size(cfg, batch, tq);
  if (ws_bytes < need) return MLA_ERR_WORKSPACE_TOO_SMALL;
  if (need > 0 && (workspace == nullptr || !aligned16(workspace))) return MLA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int n_q = batch * tq;
  const int rows = n_q * cfg->n_heads;
  if (tc_decode_shape(cfg)) {
    // the fused merge + value projection, reading the gathered parts in part order
    VprojParams vp{static_cast<const __nv_bfloat16*>(o_parts), lse_parts, nullptr,
                   static_cast<__nv_bfloat16*>(out), cfg->n_heads, tq, 1, n_q, cfg->d_v, n_parts};
    return launch_vproj(cfg, w_uv, vp, st, false);
  }
  auto run = [&](auto tag) -> mla_status {
    using T = decltype(tag);
    float* o_lat = static_cast<float*>(workspace);
    combine_simt_kernel<T><<<rows, 256, 0, st>>>(static_cast<const T*>(o_parts), lse_parts,
                                                 n_parts, rows, cfg->d_c, o_lat);
    outproj_simt_kernel<T><<<rows, 256, cfg->d_c * sizeof(float), st>>>(
        o_lat, static_cast<const T*>(w_uv), static_cast<T*>(out), cfg->n_heads, cfg->d_c,
        cfg->d_v);
    return last_launch_status();
  };
  return cfg->dtype == MLA_DTYPE_F32 ? run(float{}) : run(__nv_bfloat16{});
}

// The tensor-core prefill: positions, the tcgen05 append, then decode with tq = t_new.
static bool tc_prefill_shape(const mla_config* c) {
  return tc_decode_shape(c) && tc_append_shape(c);
}

struct PrefillLayout {
  int32_t *seq_idx, *pos;
  void *app_ws, *dec_ws;
  size_t app_bytes, dec_bytes, bytes;
};
static PrefillLayout prefill_layout(const mla_config* c, int batch, int t_new, void* ws) {
  PrefillLayout L{};
  Carve cv(ws);
  const size_t n = static_cast<size_t>(batch) * t_new;
  L.seq_idx = cv.take<int32_t>(n);
  L.pos = cv.take<int32_t>(n);
  L.app_bytes = mla_append_workspace_size(c, static_cast<int32_t>(n));
  L.app_ws = cv.take<uint8_t>(L.app_bytes);
  L.dec_bytes = mla_decode_workspace_size(c, batch, t_new);
  L.dec_ws = cv.take<uint8_t>(L.dec_bytes);
  L.bytes = cv.off;
  return L;
}

size_t mla_prefill_workspace_size(const mla_config* cfg, int32_t batch, int32_t t_new) {
  if (check_config(cfg) != MLA_OK || batch < 1 || t_new < 1) return 0;
  if (!tc_prefill_shape(cfg)) return mla_prefill_ref_workspace_size(cfg, batch, t_new);
  const PrefillLayout L = prefill_layout(cfg, batch, t_new, nullptr);
  return (L.app_bytes == 0 || L.dec_bytes == 0) ? 0 : L.bytes;
}

mla_status mla_prefill(const mla_config* cfg, const void* x, const void* q, int32_t batch,
                       int32_t t_new, const void* w_dkv, const void* kv_gain, const void* w_uk_t,
                       const void* w_uv, const int32_t* seq_lens, const int32_t* block_table,
                       int32_t max_pages, void* cache, int32_t num_pages, void* workspace,
                       size_t ws_bytes, void* out, void* stream) {
  NvtxRange nvtx_range("mla_prefill");
  const mla_status cs = check_config(cfg);
  if (cs != MLA_OK) return cs;
  if (!tc_prefill_shape(cfg) && fp8_cache(cfg)) return MLA_ERR_UNSUPPORTED;
  if (!tc_prefill_shape(cfg))
    return mla_prefill_ref(cfg, x, q, batch, t_new, w_dkv, kv_gain, w_uk_t, w_uv, seq_lens,
                           block_table, max_pages, cache, num_pages, workspace, ws_bytes, out,
                           stream);
  if (batch < 1 || t_new < 1 || max_pages < 1 || num_pages < 1) return MLA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(batch) * t_new > 65535) return MLA_ERR_INVALID_ARG;
  const void* ptrs[] = {x, q, w_dkv, kv_gain, w_uk_t, w_uv, seq_lens, block_table, cache,
                        workspace, out};
  for (const void* p : ptrs)
    if (p == nullptr || !aligned16(p)) return MLA_ERR_INVALID_ARG;
  const size_t need = mla_prefill_workspace_size(cfg, batch, t_new);
  if (need == 0) return MLA_ERR_INVALID_ARG;
  if (ws_bytes < need) return MLA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int n = batch * t_new;
  const PrefillLayout L = prefill_layout(cfg, batch, t_new, workspace);
  prefill_positions_kernel<<<(n + 255) / 256, 256, 0, st>>>(seq_lens, t_new, n, L.seq_idx, L.pos);
  mla_status s = last_launch_status();
  if (s != MLA_OK) return s;
  s = mla_append_latent(cfg, x, n, w_dkv, kv_gain, L.seq_idx, L.pos, block_table, batch,
                        max_pages, cache, num_pages, L.app_ws, L.app_bytes, stream);
  if (s != MLA_OK) return s;
  return decode_impl(cfg, q, batch, t_new, cache, num_pages, block_table, max_pages, seq_lens,
                     w_uk_t, w_uv, L.dec_ws, L.dec_bytes, out, stream, nullptr);
}

size_t mla_prefill_ref_workspace_size(const mla_config* cfg, int32_t batch, int32_t t_new) {
  if (check_config(cfg) != MLA_OK || batch < 1 || t_new < 1) return 0;
  const int64_t n = static_cast<int64_t>(batch) * t_new;
  return simt_layout(cfg, n * cfg->n_heads, n, nullptr).bytes;
}

mla_status mla_prefill_ref(const mla_config* cfg, const void* x, const void* q, int32_t batch,
                           int32_t t_new, const void* w_dkv, const void* kv_gain,
                           const void* w_uk_t, const void* w_uv, const int32_t* seq_lens,
                           const int32_t* block_table, int32_t max_pages, void* cache,
                           int32_t num_pages, void* workspace, size_t ws_bytes, void* out,
                           void* stream) {
  NvtxRange nvtx_range("mla_prefill_ref");
  const mla_status cs = check_config(cfg);
  if (cs != MLA_OK) return cs;
  if (fp8_cache(cfg)) return MLA_ERR_UNSUPPORTED;
  if (batch < 1 || t_new < 1 || max_pages < 1 || num_pages < 1) return MLA_ERR_INVALID_ARG;
  const void* ptrs[] = {x, q, w_dkv, kv_gain, w_uk_t, w_uv, seq_lens, block_table, cache,
                        workspace, out};
  for (const void* p : ptrs)
    if (p == nullptr || !aligned16(p)) return MLA_ERR_INVALID_ARG;
  if (ws_bytes < mla_prefill_ref_workspace_size(cfg, batch, t_new))
    return MLA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int n = batch * t_new;
  const SimtLayout L = simt_layout(cfg, static_cast<int64_t>(n) * cfg->n_heads, n, workspace);
  prefill_positions_kernel<<<(n + 255) / 256, 256, 0, st>>>(seq_lens, t_new, n, L.seq_idx, L.pos);
  mla_status s;
  if (cfg->dtype == MLA_DTYPE_F32) {
    s = simt_append<float>(cfg, x, n, w_dkv, kv_gain, L.seq_idx, L.pos, block_table, batch,
                           max_pages, cache, num_pages, L.kv, st);
    if (s != MLA_OK) return s;
    return simt_decode<float>(cfg, q, batch, t_new, cache, num_pages, block_table, max_pages,
                              seq_lens, w_uk_t, w_uv, L, out, st);
  }
  s = simt_append<__nv_bfloat16>(cfg, x, n, w_dkv, kv_gain, L.seq_idx, L.pos, block_table,
                                 batch, max_pages, cache, num_pages, L.kv, st);
  if (s != MLA_OK) return s;
  return simt_decode<__nv_bfloat16>(cfg, q, batch, t_new, cache, num_pages, block_table,
                                    max_pages, seq_lens, w_uk_t, w_uv, L, out, st);
}

// ---------------------------------------------------------------- allocation-free decode
// Scratch for mla_decode_noalloc: a file-scope device array, present on every GPU that loads
// this library until the process exits. Host code must not pass the symbol itself to a
// kernel (on the host it is only a stand-in); its device address is looked up once per
// device with cudaGetSymbolAddress and cached.
static __device__ __align__(256) unsigned char g_noalloc_scratch[MLA_DECODE_NOALLOC_MAX_SCRATCH];

static mla_status noalloc_scratch_ptr(void** out) {
  static std::mutex mu;
  static void* ptrs[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MLA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (ptrs[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return MLA_ERR_CUDA;
    ptrs[dev] = p;
  }
  *out = ptrs[dev];
  return MLA_OK;
}

mla_status mla_decode_noalloc(const mla_config* cfg, const void* q, int32_t batch, int32_t tq,
                              const void* cache, int32_t num_pages, const int32_t* block_table,
                              int32_t max_pages, const int32_t* seq_lens, const void* w_uk_t,
                              const void* w_uv, void* out, void* stream) {
  const mla_status cs = check_config(cfg);
  if (cs != MLA_OK) return cs;
  if (batch < 1 || tq < 1) return MLA_ERR_INVALID_ARG;
  const size_t need = mla_decode_workspace_size(cfg, batch, tq);
  if (need == 0) return cfg->dtype == MLA_DTYPE_BF16 ? MLA_ERR_UNSUPPORTED : MLA_ERR_INVALID_ARG;
  if (need > MLA_DECODE_NOALLOC_MAX_SCRATCH) return MLA_ERR_WORKSPACE_TOO_SMALL;
  void* scratch = nullptr;
  const mla_status ps = noalloc_scratch_ptr(&scratch);
  if (ps != MLA_OK) return ps;
  return decode_impl(cfg, q, batch, tq, cache, num_pages, block_table, max_pages, seq_lens,
                     w_uk_t, w_uv, scratch, MLA_DECODE_NOALLOC_MAX_SCRATCH, out, stream, nullptr);
}

mla_status mla_get_device_error(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MLA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int)) != cudaSuccess) return MLA_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)) != cudaSuccess) return MLA_ERR_CUDA;
  }
  return static_cast<mla_status>(v);
}

}  // extern "C"
