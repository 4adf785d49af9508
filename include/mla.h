/*
 * mla.h — C ABI of libmla.so: Multi-head Latent Attention (MLA) decode over a paged latent
 * KV cache on NVIDIA B200 (sm_100a).
 *
 * What is computed. Each cached token stores one row [c_KV (d_c) | k_R (d_rope)] shared by all
 * heads (「论文复现工坊 No.4 从零复现 DeepSeek-V2/V3 多头潜在注意力 MLA」 §1: the cache holds
 * (d_c + d_R) elements per token). Decoding uses the absorbed form (same page, §4; and
 * 「淺析DeepSeek多頭潛在注意力機制（MLA）」, section "MLA的數學原理"): per head h
 *     q_lat = q_nope · W_UK[h]                       (d_nope -> d_c)
 *     s_j   = (q_lat · c_j + RoPE(q_rope, p) · k_R,j) · softmax_scale
 *     P     = softmax_j(s),   o_lat = Σ_j P_j c_j,   out = o_lat · W_UV[h]ᵀ   (d_c -> d_v)
 * which equals the page's expanded module (§2 of the first page) up to rounding.
 *
 * Conventions for every call:
 *   - Tensors are dense, row-major, and live in device memory unless stated otherwise. The
 *     element type of every floating-point tensor is cfg->dtype (fp32 or bf16), except a
 *     quantised cache (mla_kv_format below). Index tensors are int32.
 *   - The caller owns every buffer. The library never allocates or frees device memory and
 *     keeps no state between calls other than one device-side error word (see
 *     mla_get_device_error), the scratch array of mla_decode_noalloc, and a host-side cache of
 *     encoded TMA descriptors (each a pure function of a tensor's address, shape and strides,
 *     so a reused buffer skips re-encoding).
 *   - Device pointers must be 16-byte aligned.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream). Calls are asynchronous;
 *     they enqueue kernels on `stream` and return. Arguments are validated on the host first:
 *     on any error the call returns a non-zero mla_status and enqueues nothing.
 *   - Errors that only the device can see (a page id outside the pool, a sequence length out
 *     of range, a stalled pipeline) are recorded in the device error word, and the next
 *     mla_get_device_error call reports the first such error. No memory outside the given
 *     buffers is touched. A bad page id or length zero-fills the affected outputs; after a
 *     stalled pipeline (a bounded wait that ran out, MLA_ERR_DEVICE_TIMEOUT) the kernel drains
 *     its copies and MMAs and leaves, and the call's outputs are undefined.
 *   - Calls that share a workspace or a cache must not overlap on the GPU (use one stream).
 *   - Every call except mla_decode_noalloc opens an NVTX range named after it on the host
 *     thread (visible to Nsight tools; a no-op without one).
 *   - Within a call, kernels after the first are launched with programmatic dependent launch
 *     and let the next kernel of the stream start early. A caller's own kernel enqueued right
 *     after a call with programmatic stream serialization must therefore wait
 *     (griddepcontrol.wait / cudaGridDependencySynchronize) before reading the call's
 *     outputs; kernels launched the ordinary way are unaffected. The first kernel of every
 *     call is launched the ordinary way, so the call sees all earlier work on the stream.
 */
#ifndef MLA_H_
#define MLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = 1,          /* null/unaligned pointer, bad size, inconsistent config  */
  MLA_ERR_UNSUPPORTED = 2,          /* valid config this build has no kernel for             */
  MLA_ERR_WORKSPACE_TOO_SMALL = 3,  /* ws_bytes below the matching *_workspace_size()         */
  MLA_ERR_CUDA = 4,                 /* a CUDA runtime/driver call failed                      */
  MLA_ERR_DEVICE_TIMEOUT = 5,       /* a kernel's bounded wait ran out (pipeline stalled)     */
  MLA_ERR_DEVICE_OOB = 6,           /* a block-table entry or sequence index out of range     */
  MLA_ERR_DEVICE_BAD_LENGTH = 7     /* seq_len < number of query tokens, or beyond the table  */
} mla_status;

typedef enum { MLA_DTYPE_F32 = 0, MLA_DTYPE_BF16 = 1 } mla_dtype;

/*
 * How the latent cache stores a row (mla_config.kv_format).
 * MLA_KV_PLAIN: rows of d_c + d_rope values in cfg->dtype; a page is
 *   [page_size][d_c + d_rope] elements.
 * MLA_KV_FP8_E4M3: the per-token quantised latent of
 *   「Multi-Head Latent Attention（MLA）原理与工程实践全解析」 (one scale per token's whole latent
 *   row). Each row is d_c + d_rope FP8 E4M3 codes (OCP E4M3: bias 7, largest finite 448, 0x7F /
 *   0xFF are NaN) plus one float32 scale, and means code * scale. A page is
 *   page_size * (d_c + d_rope + 4) bytes: the page_size rows of codes, token after token, then
 *   the page_size scales. Quantising a row v (float32): scale = max|v| / 448, code_i =
 *   E4M3(v_i / scale) (each a correctly rounded float32 division, then round to nearest, ties
 *   to even, saturating at ±448); a row of zeros gets scale 0. It halves the cache's bytes; the
 *   model's other tensors stay in cfg->dtype, which must be bf16. Decode, prefill and partial
 *   decode run it on the tcgen05 path (its DeepSeek-V2 latent shapes); mla_prefill_ref and the
 *   fp32 path do not take it (MLA_ERR_UNSUPPORTED).
 */
typedef enum { MLA_KV_PLAIN = 0, MLA_KV_FP8_E4M3 = 1 } mla_kv_format;

/*
 * Model dimensions, named as in the page's module (「从零复现 DeepSeek-V2/V3 多头潜在注意力 MLA」
 * §2): n_heads, dim (d_model), kv_lora_rank (d_c), qk_rope_head_dim (d_rope),
 * qk_nope_head_dim (d_nope), v_head_dim (d_v). softmax_scale is normally
 * 1/sqrt(d_nope + d_rope) (the module's self.scale). rms_eps is the kv_norm epsilon.
 * rope_theta is the RoPE base: pair i of a d_rope-wide vector at position p turns by
 * p * rope_theta^(-2i/d_rope) (「淺析DeepSeek多頭潛在注意力機制（MLA）」, "MLA與ROPE的融合";
 * pairs are adjacent elements (2i, 2i+1)). page_size is the number of tokens per cache page.
 * window limits attention to the most recent keys: with window > 0 a query at position p sees
 * the keys p - window + 1 .. p only (the sliding-window "Streaming-MLA" variant, which keeps the
 * last 1024 latents, in 「Multi-Head Latent Attention（MLA）原理与工程实践全解析」 §7); 0 means
 * every earlier key (plain causal attention). The window applies to every decode and prefill
 * entry point; appends are unaffected.
 * kv_format selects the cache's row format (mla_kv_format above).
 * Every entry point rejects d_rope > 128 with MLA_ERR_UNSUPPORTED, window < 0 and an unknown
 * kv_format with MLA_ERR_INVALID_ARG.
 */
typedef struct {
  int32_t n_heads;
  int32_t d_model;
  int32_t d_c;
  int32_t d_rope;
  int32_t d_nope;
  int32_t d_v;
  int32_t page_size;
  int32_t dtype; /* mla_dtype */
  float softmax_scale;
  float rms_eps;
  float rope_theta;
  int32_t window;    /* 0 = unlimited */
  int32_t kv_format; /* mla_kv_format; 0 = rows in cfg->dtype */
} mla_config;

/* Human-readable name of a status code (static string). */
const char* mla_status_string(mla_status status);

/*
 * Split the key/value up-projection into the two absorbed weight packs.
 * Source: the module's wkv_b (「从零复现 DeepSeek-V2/V3 多头潜在注意力 MLA」 §2), whose output is
 * viewed as (n_heads, d_nope + d_v) and split into the no-rope key part and the value part.
 *   wkv_b  [n_heads*(d_nope+d_v), d_c]   input
 *   w_uk_t [n_heads, d_c, d_nope]        output: w_uk_t[h][c][n] = wkv_b[h*(d_nope+d_v)+n][c]
 *                                        (W_UK[h] transposed, so q_lat = q_nope · W_UK[h])
 *   w_uv   [n_heads, d_v, d_c]           output: w_uv[h][v][c] = wkv_b[h*(d_nope+d_v)+d_nope+v][c]
 * A pure re-indexing copy: bit-exact. Buffers must not overlap.
 */
mla_status mla_absorb_weights(const mla_config* cfg, const void* wkv_b, void* w_uk_t,
                              void* w_uv, void* stream);

/* Bytes of workspace mla_append_latent needs for n_tok tokens (0 if the arguments are invalid). */
size_t mla_append_workspace_size(const mla_config* cfg, int32_t n_tok);

/*
 * Append n_tok tokens to the paged latent cache (the KV half of the page's module, §2 of
 * 「从零复现 DeepSeek-V2/V3 多头潜在注意力 MLA」: wkv_a, split, kv_norm; plus RoPE on k_R from
 * 「淺析DeepSeek多頭潛在注意力機制（MLA）」, "MLA與ROPE的融合"). For token i:
 *     kv   = x[i] · w_dkvᵀ                                   (d_c + d_rope outputs)
 *     c    = kv[:d_c] / sqrt(mean(kv[:d_c]^2) + rms_eps) * kv_gain
 *     k_R  = RoPE(kv[d_c:], pos[i])
 *     cache[block_table[seq_idx[i]][pos[i] / page_size]][pos[i] % page_size] = [c | k_R]
 * rounded once to cfg->dtype (with kv_format MLA_KV_FP8_E4M3: quantised from the float32 row,
 * codes and scale; bf16 and d_model a multiple of 64 only). fp32 accumulation.
 *   x           [n_tok, d_model]
 *   w_dkv       [d_c + d_rope, d_model]     (wkv_a weight; rows [0,d_c) give c_KV)
 *   kv_gain     [d_c]                       (kv_norm weight)
 *   seq_idx     [n_tok] int32, in [0, batch)
 *   pos         [n_tok] int32, 0-based position in its sequence, < max_pages*page_size
 *   block_table [batch, max_pages] int32    page ids in [0, num_pages)
 *   cache       [num_pages, page_size, d_c + d_rope]   updated in place, only the addressed rows
 *               (quantised: pages of page_size * (d_c + d_rope + 4) bytes, see mla_kv_format)
 *   workspace   >= mla_append_workspace_size(cfg, n_tok) bytes, 256-byte aligned
 * Tokens whose sequence, position or page is out of range are skipped and flagged
 * MLA_ERR_DEVICE_OOB. Two tokens addressing the same row race (caller's responsibility).
 */
mla_status mla_append_latent(const mla_config* cfg, const void* x, int32_t n_tok,
                             const void* w_dkv, const void* kv_gain, const int32_t* seq_idx,
                             const int32_t* pos, const int32_t* block_table, int32_t batch,
                             int32_t max_pages, void* cache, int32_t num_pages, void* workspace,
                             size_t ws_bytes, void* stream);

/*
 * Write n_tok given rows into a quantised cache (kv_format MLA_KV_FP8_E4M3): row i is quantised
 * as described at mla_kv_format and stored at position pos[i] of sequence seq_idx[i]. For
 * filling such a cache from rows computed elsewhere (a bf16 cache being converted, rows from
 * another model run); mla_append_latent computes and quantises new rows itself.
 *   rows        [n_tok, d_c + d_rope] float32
 *   seq_idx, pos, block_table, batch, max_pages, num_pages: as in mla_append_latent
 *   cache       [num_pages] pages of page_size * (d_c + d_rope + 4) bytes, updated in place
 * Tokens whose sequence, position or page is out of range are skipped and flagged
 * MLA_ERR_DEVICE_OOB. Any kv_format other than MLA_KV_FP8_E4M3 is MLA_ERR_INVALID_ARG.
 */
mla_status mla_quantize_latent(const mla_config* cfg, const float* rows, int32_t n_tok,
                               const int32_t* seq_idx, const int32_t* pos,
                               const int32_t* block_table, int32_t batch, int32_t max_pages,
                               void* cache, int32_t num_pages, void* stream);

/* Bytes of workspace mla_decode needs for (batch, tq) on the current device (0 if invalid). */
size_t mla_decode_workspace_size(const mla_config* cfg, int32_t batch, int32_t tq);

/*
 * Batched, variable-length decode attention over the paged latent cache (absorbed form, see the
 * top of this file), with split-KV: long sequences are cut into chunks of whole pages that run
 * in parallel and are merged by their log-sum-exp.
 * The cache must already hold the tq new tokens of each sequence (append first): sequence b
 * has seq_lens[b] tokens and its query t sits at position seq_lens[b] - tq + t; it attends to
 * tokens 0 .. seq_lens[b] - tq + t (causal among the new tokens; a query sees itself —
 * 「淺析DeepSeek多頭潛在注意力機制（MLA）」: the new token attends to all N+1 keys).
 *   q           [batch, tq, n_heads, d_nope + d_rope]  un-rotated queries ([q_nope | q_rope])
 *   cache       [num_pages, page_size, d_c + d_rope] (quantised: see mla_kv_format)
 *   block_table [batch, max_pages] int32
 *   seq_lens    [batch] int32 (device), each in [tq, max_pages*page_size]
 *   w_uk_t      [n_heads, d_c, d_nope], w_uv [n_heads, d_v, d_c]   (from mla_absorb_weights)
 *   workspace   >= mla_decode_workspace_size(cfg, batch, tq) bytes, 256-byte aligned
 *   out         [batch, tq, n_heads, d_v]
 * bf16 runs on the tcgen05 tensor-core path and needs d_c = 512, d_rope = 64, page_size = 64
 * and d_nope a multiple of 64 (DeepSeek-V2 latent shapes); fp32 runs on CUDA cores for any
 * shape. A quantised cache (kv_format MLA_KV_FP8_E4M3) runs on the tcgen05 path at the same
 * shapes: the attention multiplies the E4M3 codes on the tensor cores (the query split into
 * two E4M3 parts under a per-row scale, about 8 significant bits kept) and applies the
 * per-token scales in the softmax; the result matches the same attention over the dequantised
 * rows within the bf16 parity bound.
 * A sequence whose length is out of range gets zero output and MLA_ERR_DEVICE_BAD_LENGTH.
 */
mla_status mla_decode(const mla_config* cfg, const void* q, int32_t batch, int32_t tq,
                      const void* cache, int32_t num_pages, const int32_t* block_table,
                      int32_t max_pages, const int32_t* seq_lens, const void* w_uk_t,
                      const void* w_uv, void* workspace, size_t ws_bytes, void* out,
                      void* stream);

/*
 * mla_decode with per-kernel timing: identical arguments and results, plus `events`, an array
 * of 4 cudaEvent_t created by the caller, recorded on `stream` at the kernel boundaries of the
 * bf16 path: events[0] before the query absorption (whose extra block also plans the split-KV
 * work), events[1] before the latent attention kernel, events[2] before the fused split merge
 * + value projection, events[3] after it; cudaEventElapsedTime(events[1], events[2]) is the
 * attention kernel's device time. The event records sit between the kernels, so kernels that
 * otherwise overlap their start with the previous kernel's end (programmatic dependent launch)
 * run back to back here. While `stream` is being captured the events are recorded with
 * cudaEventRecordExternal, so they become event-record nodes of the graph. The fp32 path marks
 * the same three stages (absorption, attention, projection). NULL entries are skipped.
 */
mla_status mla_decode_profiled(const mla_config* cfg, const void* q, int32_t batch, int32_t tq,
                               const void* cache, int32_t num_pages, const int32_t* block_table,
                               int32_t max_pages, const int32_t* seq_lens, const void* w_uk_t,
                               const void* w_uv, void* workspace, size_t ws_bytes, void* out,
                               void* stream, void* const* events);

/* Bytes of workspace mla_query needs for n_tok tokens (0 if the arguments are invalid). */
size_t mla_query_workspace_size(const mla_config* cfg, int32_t q_lora, int32_t n_tok);

/*
 * The query path of the module (「从零复现 DeepSeek-V2/V3 多头潜在注意力 MLA」 §2: wq_a, q_norm,
 * wq_b), producing the un-rotated per-head queries that mla_decode takes:
 *     q_a = x · w_qaᵀ                                              (q_lora outputs, fp32 sums)
 *     q_a = q_a / sqrt(mean(q_a^2) + rms_eps) * q_gain, rounded once to cfg->dtype
 *     q   = q_a · w_qbᵀ, viewed as [n_heads][d_nope + d_rope], rounded to cfg->dtype
 *   x       [n_tok, d_model]
 *   w_qa    [q_lora, d_model]                      (wq_a weight)
 *   q_gain  [q_lora]                               (q_norm weight)
 *   w_qb    [n_heads * (d_nope + d_rope), q_lora]  (wq_b weight; per head [q_nope | q_rope])
 *   workspace >= mla_query_workspace_size(cfg, q_lora, n_tok) bytes, 256-byte aligned
 *   q_out   [n_tok, n_heads, d_nope + d_rope]
 * bf16 with d_model and q_lora multiples of 64 runs two tcgen05 weight-streaming GEMMs (the
 * first split over K) around a normalisation kernel; other shapes and fp32 run on CUDA cores.
 * The pre-absorbed form (W_UK folded into wq_b) is not offered: at DeepSeek-V2 shape its weight
 * is five times the bytes of wq_b's no-rope part plus W_UK, and decode streams every byte.
 */
mla_status mla_query(const mla_config* cfg, int32_t q_lora, const void* x, int32_t n_tok,
                     const void* w_qa, const void* q_gain, const void* w_qb, void* workspace,
                     size_t ws_bytes, void* q_out, void* stream);

/* Bytes of workspace mla_output needs for n_tok tokens (0 if the arguments are invalid). */
size_t mla_output_workspace_size(const mla_config* cfg, int32_t n_tok);

/*
 * The module's output projection wo (「从零复现 DeepSeek-V2/V3 多头潜在注意力 MLA」 §2): the
 * heads' outputs laid side by side, head after head, times woᵀ:
 *     y[n][m] = sum_{h, v} w_o[m][h * d_v + v] * attn[n][h][v]     (fp32 sums, one rounding)
 *   attn    [n_tok, n_heads, d_v]          (mla_decode's out)
 *   w_o     [d_model, n_heads * d_v]       (wo weight)
 *   workspace >= mla_output_workspace_size(cfg, n_tok) bytes, 256-byte aligned
 *   y       [n_tok, d_model]
 * bf16 with n_heads * d_v a multiple of 64 runs a split-K tcgen05 GEMM whose partial sums are
 * added in split order; other shapes and fp32 run on CUDA cores. The variant with W_UV folded
 * into wo is not offered: its weight (d_model x n_heads*d_c) is four times wo's at V2 shape.
 */
mla_status mla_output(const mla_config* cfg, const void* attn, int32_t n_tok, const void* w_o,
                      void* workspace, size_t ws_bytes, void* y, void* stream);

/*
 * Decode over a share of each sequence's keys, for a long context whose cache is split over
 * several GPUs (each holds whole pages of a key range): the same attention as mla_decode, but
 * only keys kv_begin[b] <= j < kv_end[b] are read (with the causal rule and cfg->window), and
 * the result is the partial latent output and its log-sum-exp instead of the projected output:
 *     o_part[row][:] = sum_j softmax_j o_j  over the visible keys of the range (O / l),
 *     lse[row]       = ln sum_j exp(s_j)    (natural log of the scaled scores; -inf and a zero
 *                                            row when the range holds no key the row sees)
 * with row = (b * tq + t) * n_heads + h. Partials of disjoint ranges that cover every key are
 * merged by mla_combine into exactly mla_decode's result (up to rounding): the split-KV merge of
 * this library, moved across GPUs. Pages outside [kv_begin, kv_end) are never read, so their
 * block-table entries may be anything. The ranges should start on page boundaries (a page whose
 * keys straddle two ranges is read by both GPUs).
 *   kv_begin, kv_end  [batch] int32 (device), 0 <= kv_begin[b], kv_end[b] <= seq_lens[b]
 *   o_part  [batch * tq * n_heads, d_c] in cfg->dtype;  lse [batch * tq * n_heads] float
 *   other arguments and the workspace as in mla_decode (mla_decode_workspace_size)
 * w_uv is not needed. Shapes and dtypes as mla_decode.
 */
mla_status mla_decode_partial(const mla_config* cfg, const void* q, int32_t batch, int32_t tq,
                              const void* cache, int32_t num_pages, const int32_t* block_table,
                              int32_t max_pages, const int32_t* seq_lens,
                              const int32_t* kv_begin, const int32_t* kv_end, const void* w_uk_t,
                              void* workspace, size_t ws_bytes, void* o_part, float* lse,
                              void* stream);

/* Bytes of workspace mla_combine needs (0 if the arguments are invalid). */
size_t mla_combine_workspace_size(const mla_config* cfg, int32_t batch, int32_t tq);

/*
 * Merge n_parts partial results of mla_decode_partial (one per key range, typically gathered
 * from the GPUs that hold the ranges) and project:
 *     o_lat[row] = sum_k e^(lse_k - m) o_part_k[row] / sum_k e^(lse_k - m),  m = max_k lse_k
 *     out[b][t][h][:] = o_lat[row] · W_UV[h]ᵀ
 * The parts are added in index order, so every GPU that runs this on the same gathered parts
 * gets the same bits. A row that no part saw any key of gets zeros.
 *   o_parts [n_parts, batch * tq * n_heads, d_c] in cfg->dtype
 *   lse_parts [n_parts, batch * tq * n_heads] float
 *   w_uv [n_heads, d_v, d_c];  out [batch, tq, n_heads, d_v]
 *   workspace >= mla_combine_workspace_size(cfg, batch, tq) bytes (may be 0)
 */
mla_status mla_combine(const mla_config* cfg, int32_t n_parts, int32_t batch, int32_t tq,
                       const void* o_parts, const float* lse_parts, const void* w_uv,
                       void* workspace, size_t ws_bytes, void* out, void* stream);

/* Bytes of workspace mla_prefill needs (0 if the arguments are invalid). */
size_t mla_prefill_workspace_size(const mla_config* cfg, int32_t batch, int32_t t_new);

/*
 * Prefill on the tensor cores: append t_new tokens per sequence (as mla_append_latent) and
 * return the attention outputs of all of them, each new token seeing the keys up to its own
 * position (the prompt pass of 「淺析DeepSeek多頭潛在注意力機制（MLA）」, "大模型的整體推理過程",
 * done token-causal, in the absorbed form). Same arguments and results as mla_prefill_ref. For
 * bf16 at DeepSeek-V2 latent shapes (those mla_decode runs on tcgen05) the append is the
 * tcgen05 down-projection and the attention is mla_decode's latent attention kernel with
 * tq = t_new, each 128-row unit of query rows reading only the pages its tokens can see; other
 * shapes run mla_prefill_ref's CUDA-core path.
 */
mla_status mla_prefill(const mla_config* cfg, const void* x, const void* q, int32_t batch,
                       int32_t t_new, const void* w_dkv, const void* kv_gain, const void* w_uk_t,
                       const void* w_uv, const int32_t* seq_lens, const int32_t* block_table,
                       int32_t max_pages, void* cache, int32_t num_pages, void* workspace,
                       size_t ws_bytes, void* out, void* stream);

/* Bytes of workspace mla_prefill_ref needs (0 if the arguments are invalid). */
size_t mla_prefill_ref_workspace_size(const mla_config* cfg, int32_t batch, int32_t t_new);

/*
 * Reference prefill: append t_new tokens per sequence and return their attention outputs, on
 * CUDA cores with fp32 arithmetic, for any shape and either dtype (the correctness path; the
 * prompt pass of 「淺析DeepSeek多頭潛在注意力機制（MLA）」, "大模型的整體推理過程", done token-causal).
 * Sequence b ends up with seq_lens[b] tokens; its new tokens take positions
 * seq_lens[b] - t_new .. seq_lens[b] - 1 (earlier positions must already be in the cache).
 *   x    [batch, t_new, d_model]                    hidden states of the new tokens
 *   q    [batch, t_new, n_heads, d_nope + d_rope]   their un-rotated queries
 *   w_dkv, kv_gain, block_table, cache: as in mla_append_latent
 *   w_uk_t, w_uv, seq_lens: as in mla_decode (each seq_lens[b] >= t_new)
 *   out  [batch, t_new, n_heads, d_v]
 */
mla_status mla_prefill_ref(const mla_config* cfg, const void* x, const void* q, int32_t batch,
                           int32_t t_new, const void* w_dkv, const void* kv_gain,
                           const void* w_uk_t, const void* w_uv, const int32_t* seq_lens,
                           const int32_t* block_table, int32_t max_pages, void* cache,
                           int32_t num_pages, void* workspace, size_t ws_bytes, void* out,
                           void* stream);

/*
 * Allocation-free decode, for callers that cannot allocate device memory themselves: code
 * running where cudaMalloc is unavailable or forbidden (inside a memory-pool-managed serving
 * runtime that owns all device memory, or a host callback), or that must not grow its
 * footprint per call. The paper has no counterpart: this is a deployment convenience.
 * Same arguments and results as mla_decode, minus the workspace: the scratch it needs lives in
 * a fixed device array of MLA_DECODE_NOALLOC_MAX_SCRATCH bytes inside this library, which
 * every GPU that loads the library holds until the process exits.
 *   - A call whose scratch need (mla_decode_workspace_size) exceeds that maximum returns
 *     MLA_ERR_WORKSPACE_TOO_SMALL and launches nothing. On a 148-SM B200, 32 MiB covers a
 *     DeepSeek-V2-shaped batch of up to 85 sequences with one query token each over a bf16
 *     cache, 55 over a quantised one (the scratch holds Q̂ for every query row, with a
 *     quantised cache also its split E4M3 form, and one bf16 partial per split, whose count
 *     grows with the SM count).
 *   - It never calls cudaMalloc, cudaFree or any allocating routine.
 *   - The first call on a device looks up the array's device address (cudaGetSymbolAddress)
 *     and caches it; make that first call before any stream capture on that device.
 *   - Every call on a device shares the one array, and no part of it needs to start zeroed
 *     (each call writes all scratch it reads). Calls that overlap on the GPU (different
 *     streams, or concurrent host threads) race on it: serialise them.
 */
#define MLA_DECODE_NOALLOC_MAX_SCRATCH (32u << 20)
mla_status mla_decode_noalloc(const mla_config* cfg, const void* q, int32_t batch, int32_t tq,
                              const void* cache, int32_t num_pages, const int32_t* block_table,
                              int32_t max_pages, const int32_t* seq_lens, const void* w_uk_t,
                              const void* w_uv, void* out, void* stream);

/*
 * Synchronise `stream`, then return (and clear) the first error a kernel of this library
 * recorded on the current device since the previous call: MLA_OK if none. Returns
 * MLA_ERR_CUDA if the synchronisation itself fails.
 */
mla_status mla_get_device_error(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MLA_H_ */
