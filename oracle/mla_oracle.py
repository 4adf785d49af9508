"""Plain fp64 CPU oracle for Multi-head Latent Attention decode.

TEST INFRASTRUCTURE ONLY. Only the test suite, the smoke check and the benchmark's CPU-baseline
leg may import this module. The CUDA library never calls it, and it shares no code, constants
or helpers with the CUDA path.

It follows the un-absorbed (expanded) form of the module printed on the page
「论文复现工坊 No.4 从零复现 DeepSeek-V2/V3 多头潜在注意力 MLA」, §2 (PyTorch module): every head
gets its own key [c_KV·W_UKᵀ | k_R] and value c_KV·W_UVᵀ, then plain softmax attention. The
rotary step that the page's code leaves out is filled in from 「淺析DeepSeek多頭潛在注意力機制
（MLA）」, section "MLA與ROPE的融合". The absorbed form (section "MLA的數學原理" of the same page,
and §4 of the first page) is kept separately, only to check that the two forms agree.

Readings where the pages are silent (each is also listed in the design notes):
  * RoPE rotates adjacent pairs (2i, 2i+1) with angle pos·θ_i, θ_i = theta^(-2i/d_r);
  * positions are 0-based; query t of Tq new tokens sits at position L - Tq + t;
  * the new tokens are appended before attending, so a query sees itself;
  * RMSNorm is x / sqrt(mean(x^2) + eps) * gain, applied to c_KV only (not to k_R);
  * decode_expanded stops before the output projection wo; output_projection applies it and
    decode_layer chains the whole layer (q path, append, attention, wo).
All arithmetic is float64; bf16 inputs are promoted exactly.
"""

from __future__ import annotations

import numpy as np


def f64(a) -> np.ndarray:
    """Exact promotion of a torch tensor / array (any float dtype) to a float64 ndarray."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            return a.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(a, dtype=np.float64)


def rms_norm(v: np.ndarray, gain: np.ndarray, eps: float) -> np.ndarray:
    """RMSNorm over the last axis.

    The page 「从零复现 DeepSeek-V2/V3 多头潜在注意力 MLA」 §2 applies nn.RMSNorm to the d_c part
    of the down-projection (kv_norm) and §4 says the norm after W_DKV is required.
    """
    v = f64(v)
    ms = np.mean(v * v, axis=-1, keepdims=True)
    return v / np.sqrt(ms + eps) * f64(gain)


def rope_frequencies(d_r: int, theta: float) -> np.ndarray:
    """θ_i = theta^(-2i/d_r), i = 0 .. d_r/2 - 1.

    「淺析DeepSeek多頭潛在注意力機制（MLA）」, "MLA與ROPE的融合": θ_i = 10000^(-2i/d) with i from 0
    to d/2 - 1; for the decoupled key the rotated width d is d_r.
    """
    i = np.arange(d_r // 2, dtype=np.float64)
    return np.power(float(theta), -2.0 * i / d_r)


def rope(v: np.ndarray, pos, theta: float) -> np.ndarray:
    """Apply the block-diagonal rotation R_pos to the last axis of v.

    Each 2x2 block turns the pair (v[2i], v[2i+1]) by the angle pos·θ_i
    (「淺析DeepSeek多頭潛在注意力機制（MLA）」, "MLA與ROPE的融合": R_m is block diagonal and
    R_m R_nᵀ = R_{m-n}). pos broadcasts against v[..., 0].
    """
    v = f64(v)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * rope_frequencies(v.shape[-1], theta)
    c, s = np.cos(ang), np.sin(ang)
    x, y = v[..., 0::2], v[..., 1::2]
    out = np.empty_like(v)
    out[..., 0::2] = x * c - y * s
    out[..., 1::2] = x * s + y * c
    return out


def latent_rows(x, w_dkv, kv_gain, pos, d_c: int, eps: float, theta: float) -> np.ndarray:
    """Cache rows [c_KV | k_R] of tokens x at positions pos (the append step).

    「从零复现 DeepSeek-V2/V3 多头潜在注意力 MLA」 §2: one down-projection wkv_a gives d_c + d_r
    outputs, split into the latent (then kv_norm) and the rotary key; §1 says only c_KV and k_R
    are cached. k_R is computed from the hidden state, not from c_KV, and is rotated with the
    token's own position (「淺析DeepSeek多頭潛在注意力機制（MLA）」, "MLA與ROPE的融合").
    """
    kv = f64(x) @ f64(w_dkv).T
    c = rms_norm(kv[..., :d_c], kv_gain, eps)
    kr = rope(kv[..., d_c:], pos, theta)
    return np.concatenate([c, kr], axis=-1)


def split_wkv_b(wkv_b, H: int, d_nope: int, d_v: int):
    """W_UK [H, d_nope, d_c] and W_UV [H, d_v, d_c] from wkv_b [H*(d_nope+d_v), d_c].

    The page's module views wkv_b's output as (heads, d_nope + d_v) and splits it into the
    no-rope key part and the value part (「从零复现 DeepSeek-V2/V3 多头潜在注意力 MLA」 §2).
    """
    w = f64(wkv_b).reshape(H, d_nope + d_v, -1)
    return w[:, :d_nope, :], w[:, d_nope:, :]


def query_from_x(x, w_qa, q_gain, w_qb, H: int, d_nope: int, d_r: int, eps: float) -> np.ndarray:
    """Un-rotated per-head queries [.., H, d_nope + d_r] from hidden states (q low-rank path).

    「从零复现 DeepSeek-V2/V3 多头潜在注意力 MLA」 §2: q = wq_b(q_norm(wq_a(x))), viewed per head.
    """
    qa = rms_norm(f64(x) @ f64(w_qa).T, q_gain, eps)
    q = qa @ f64(w_qb).T
    return q.reshape(q.shape[:-1] + (H, d_nope + d_r))


def _softmax(s: np.ndarray) -> np.ndarray:
    e = np.exp(s - s.max(axis=-1, keepdims=True))
    return e / e.sum(axis=-1, keepdims=True)


def _visible(L: int, Tq: int, window: int) -> np.ndarray:
    """mask[t, j]: key j is visible to query token t (position p = L - Tq + t).

    Causal rule (「淺析DeepSeek多頭潛在注意力機制（MLA）」: the new token attends to all earlier
    tokens and itself) and, for window > 0, the sliding window of the Streaming-MLA variant
    (「Multi-Head Latent Attention（MLA）原理与工程实践全解析」 §7 keeps only the latents of the most
    recent 1024 tokens): read here as key j visible iff p - window < j <= p.
    """
    pos = L - Tq + np.arange(Tq)
    j = np.arange(L)[None, :]
    vis = j <= pos[:, None]
    if window > 0:
        vis &= j > pos[:, None] - window
    return vis


def decode_expanded(q, rows, W_UK, W_UV, scale: float, theta: float, heads=None,
                    return_probs: bool = False, window: int = 0):
    """Attention output of the Tq newest tokens of one sequence, un-absorbed form.

    q     [Tq, H, d_nope + d_r]  un-rotated queries of the new tokens
    rows  [L, d_c + d_r]          cache rows of the whole sequence, new tokens included
    W_UK  [H, d_nope, d_c], W_UV [H, d_v, d_c]
    Returns out [Tq, len(heads), d_v] (and the probabilities [Tq, len(heads), L] if asked).

    Per head (「从零复现 DeepSeek-V2/V3 多头潜在注意力 MLA」 §2): K = [c·W_UKᵀ | k_R broadcast to
    every head], V = c·W_UVᵀ, q_full = [q_nope | RoPE(q_rope)], scores = q_full·Kᵀ·scale with
    scale = 1/sqrt(d_nope + d_r), softmax, then probs·V. Query t sits at position L - Tq + t
    and sees keys 0 .. L - Tq + t (causal rule and the 1×(N+1) decode step in
    「淺析DeepSeek多頭潛在注意力機制（MLA）」); with window > 0 only the last `window` of them
    (_visible).
    """
    q, rows = f64(q), f64(rows)
    W_UK, W_UV = f64(W_UK), f64(W_UV)
    Tq, H = q.shape[0], q.shape[1]
    L = rows.shape[0]
    d_nope, d_c = W_UK.shape[1], W_UK.shape[2]
    heads = list(range(H)) if heads is None else list(heads)
    c, kr = rows[:, :d_c], rows[:, d_c:]
    pos = L - Tq + np.arange(Tq)
    out = np.zeros((Tq, len(heads), W_UV.shape[1]))
    probs = np.zeros((Tq, len(heads), L))
    for j, h in enumerate(heads):
        K = np.concatenate([c @ W_UK[h].T, kr], axis=1)          # [L, d_nope + d_r]
        V = c @ W_UV[h].T                                         # [L, d_v]
        qf = np.concatenate([q[:, h, :d_nope], rope(q[:, h, d_nope:], pos, theta)], axis=1)
        s = (qf @ K.T) * scale                                    # [Tq, L]
        s[~_visible(L, Tq, window)] = -np.inf
        P = _softmax(s)
        out[:, j] = P @ V
        probs[:, j] = P
    return (out, probs) if return_probs else out


def decode_absorbed(q, rows, W_UK, W_UV, scale: float, theta: float, heads=None, window: int = 0):
    """Same result as decode_expanded, in the absorbed (latent-space) form.

    q_lat = q_nope·W_UK, score_j = (q_lat·c_j + RoPE(q_rope)·k_R,j)·scale, o_lat = P·c,
    out = o_lat·W_UVᵀ (「从零复现 DeepSeek-V2/V3 多头潜在注意力 MLA」 §4 and
    「淺析DeepSeek多頭潛在注意力機制（MLA）」, "MLA的數學原理"). Used only to check that the
    two forms agree.
    """
    q, rows = f64(q), f64(rows)
    W_UK, W_UV = f64(W_UK), f64(W_UV)
    Tq, H = q.shape[0], q.shape[1]
    L = rows.shape[0]
    d_nope, d_c = W_UK.shape[1], W_UK.shape[2]
    heads = list(range(H)) if heads is None else list(heads)
    c, kr = rows[:, :d_c], rows[:, d_c:]
    pos = L - Tq + np.arange(Tq)
    out = np.zeros((Tq, len(heads), W_UV.shape[1]))
    for j, h in enumerate(heads):
        q_lat = q[:, h, :d_nope] @ W_UK[h]                        # [Tq, d_c]
        q_r = rope(q[:, h, d_nope:], pos, theta)
        s = (q_lat @ c.T + q_r @ kr.T) * scale
        s[~_visible(L, Tq, window)] = -np.inf
        o_lat = _softmax(s) @ c
        out[:, j] = o_lat @ W_UV[h].T
    return out


def latent_partial(q, rows, W_UK, scale: float, theta: float, kv_begin: int, kv_end: int,
                   heads=None, window: int = 0):
    """Attention of the Tq newest tokens of one sequence over the keys kv_begin <= j < kv_end
    only, in latent space: returns o [Tq, len(heads), d_c] = sum_j P_j c_j with P the softmax over
    those keys (O / l), and lse [Tq, len(heads)] = ln sum_j exp(s_j) (-inf, and o = 0, when the
    range holds no key the query sees).

    The pages are silent on splitting one sequence's keys: this is the plain reading of split
    attention, the softmax restricted to a subset of keys plus the log of its normaliser, which
    merge_partials turns back into the whole softmax. Scores as in decode_absorbed.
    """
    q, rows = f64(q), f64(rows)
    W_UK = f64(W_UK)
    Tq, H = q.shape[0], q.shape[1]
    L = rows.shape[0]
    d_nope, d_c = W_UK.shape[1], W_UK.shape[2]
    heads = list(range(H)) if heads is None else list(heads)
    c, kr = rows[:, :d_c], rows[:, d_c:]
    pos = L - Tq + np.arange(Tq)
    vis = _visible(L, Tq, window)
    idx = np.arange(L)
    vis &= (idx >= kv_begin)[None, :] & (idx < kv_end)[None, :]
    o = np.zeros((Tq, len(heads), d_c))
    lse = np.full((Tq, len(heads)), -np.inf)
    for jh, h in enumerate(heads):
        q_lat = q[:, h, :d_nope] @ W_UK[h]
        q_r = rope(q[:, h, d_nope:], pos, theta)
        s = (q_lat @ c.T + q_r @ kr.T) * scale
        for t in range(Tq):
            st = s[t, vis[t]]
            if st.size == 0:
                continue
            m = st.max()
            e = np.exp(st - m)
            o[t, jh] = (e / e.sum()) @ c[vis[t]]
            lse[t, jh] = m + np.log(e.sum())
    return o, lse


def merge_partials(o_parts, lse_parts):
    """Merge partial results over disjoint key ranges: sum_k e^(lse_k - M) o_k / sum_k
    e^(lse_k - M), M = max_k lse_k (zeros where every lse is -inf). o_parts [K, ..., d],
    lse_parts [K, ...]. Because e^(lse_k) is the normaliser of part k, this is the softmax over
    the union of the ranges applied to the same values."""
    o_parts, lse_parts = f64(o_parts), f64(lse_parts)
    M = lse_parts.max(axis=0)
    Ms = np.where(np.isfinite(M), M, 0.0)
    w = np.where(np.isfinite(lse_parts), np.exp(lse_parts - Ms[None]), 0.0)
    den = w.sum(axis=0)
    num = (w[..., None] * o_parts).sum(axis=0)
    return np.where(den[..., None] > 0, num / np.where(den > 0, den, 1.0)[..., None], 0.0)


def module_attention(x, w_dkv, kv_gain, wkv_b, w_qa, q_gain, w_qb, H, d_c, d_r, d_nope, d_v,
                     eps, theta):
    """Whole-sequence (prefill) attention output [L, H, d_v] of the page's module, before wo.

    Every step of 「从零复现 DeepSeek-V2/V3 多头潜在注意力 MLA」 §2 for one sequence x [L, d_model]:
    q path, joint KV down-projection with kv_norm, decoupled RoPE, expanded keys and values,
    causal softmax attention.
    """
    x = f64(x)
    L = x.shape[0]
    q = query_from_x(x, w_qa, q_gain, w_qb, H, d_nope, d_r, eps)
    rows = latent_rows(x, w_dkv, kv_gain, np.arange(L), d_c, eps, theta)
    W_UK, W_UV = split_wkv_b(wkv_b, H, d_nope, d_v)
    return decode_expanded(q, rows, W_UK, W_UV, 1.0 / np.sqrt(d_nope + d_r), theta)


def output_projection(out, w_o) -> np.ndarray:
    """The module's output projection wo applied to per-head attention outputs.

    「从零复现 DeepSeek-V2/V3 多头潜在注意力 MLA」 §2: the heads' outputs are laid side by side,
    head after head, into one vector of heads * d_v values per token, and wo, a bias-free linear
    map from heads * d_v to the model width, brings them back to d_model.
    out [..., H, d_v], w_o [d_model, H * d_v]; returns [..., d_model].
    """
    out = f64(out)
    flat = out.reshape(out.shape[:-2] + (out.shape[-2] * out.shape[-1],))
    return flat @ f64(w_o).T


def decode_layer(x_new, rows_hist, w_dkv, kv_gain, wkv_b, w_qa, q_gain, w_qb, w_o, H: int,
                 d_c: int, d_r: int, d_nope: int, d_v: int, eps: float, theta: float):
    """One decode step of the whole attention layer for one sequence, expanded form.

    x_new [Tq, d_model] are the hidden states of the Tq new tokens; rows_hist [L - Tq, d_c+d_r]
    the cache rows already stored for the sequence. Steps, in the order of the page's module
    (「从零复现 DeepSeek-V2/V3 多头潜在注意力 MLA」 §2): the q path wq_a -> q_norm -> wq_b; the
    new tokens' latent rows appended at positions L - Tq .. L - 1; attention of the new tokens
    over all L rows (each sees itself and earlier tokens); the output projection wo.
    Returns y [Tq, d_model].
    """
    x_new = f64(x_new)
    Tq = x_new.shape[0]
    L = rows_hist.shape[0] + Tq
    q = query_from_x(x_new, w_qa, q_gain, w_qb, H, d_nope, d_r, eps)
    new_rows = latent_rows(x_new, w_dkv, kv_gain, np.arange(L - Tq, L), d_c, eps, theta)
    rows = np.concatenate([f64(rows_hist), new_rows], axis=0)
    W_UK, W_UV = split_wkv_b(wkv_b, H, d_nope, d_v)
    out = decode_expanded(q, rows, W_UK, W_UV, 1.0 / np.sqrt(d_nope + d_r), theta)
    return output_projection(out, w_o)


def gather_rows(cache, block_table_row, L: int, page_size: int = 64) -> np.ndarray:
    """The L logical cache rows of one sequence, read through its block-table row."""
    idx = np.arange(L)
    pages = np.asarray(block_table_row, dtype=np.int64)[idx // page_size]
    slots = idx % page_size
    if isinstance(cache, np.ndarray):
        return f64(cache[pages, slots])
    import torch
    return f64(cache[torch.from_numpy(pages), torch.from_numpy(slots)])


# --- KV cache size arithmetic -------------------------------------------------------------

def mla_cache_elems_per_token(d_c: int, d_r: int) -> int:
    """Latent cache elements per token per layer: d_c + d_r (one row shared by every head).

    「从零复现 DeepSeek-V2/V3 多头潜在注意力 MLA」 §1 (cache per token = (d_c + d_R) × bytes).
    """
    return d_c + d_r


def mha_cache_elems_per_token(n_heads: int, d_h: int) -> int:
    """Standard MHA cache elements per token per layer: 2·n_heads·d_h (keys and values)."""
    return 2 * n_heads * d_h


def gqa_cache_elems_per_token(n_groups: int, d_h: int) -> int:
    """GQA with n_groups key/value groups: 2·n_groups·d_h."""
    return 2 * n_groups * d_h


# --- quantised latent cache (8-bit codes with one scale per token) --------------------------
#
# 「Multi-Head Latent Attention（MLA）原理与工程实践全解析」 (context only) quantises the latent
# per token: one scale for a token's whole latent row. Read here as: every cache row
# [c_KV | k_R] is stored as FP8 E4M3 codes (1 sign, 4 exponent bits with bias 7, 3 mantissa bits;
# no infinities, 0x7F/0xFF are NaN; largest finite value 448) plus one float32 scale
#     scale = max_i |v_i| / 448,   code_i = E4M3(v_i / scale)   (round to nearest, ties to
# even, saturating at ±448), and the stored row means code_i * scale. A row of zeros gets scale 0.
# The rounding to E4M3 decides an integer code, so these steps are done in float32, as the
# device does them (row values arrive as float32): the max is exact, each division is one
# correctly rounded float32 division, then one rounding onto the E4M3 grid.

E4M3_MAX = 448.0


def e4m3_value(code) -> np.ndarray:
    """Real value of FP8 E4M3 codes (uint8 array), float64; NaN for 0x7F and 0xFF.

    From the format's definition: exponent field e and mantissa m give (1 + m/8)·2^(e-7) for
    e >= 1 and m/8·2^(-6) for e = 0 (subnormal); e = 15, m = 7 is NaN (the format keeps the
    rest of the top binade for finite values, up to 1.75·2^8 = 448).
    """
    c = np.asarray(code, dtype=np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 7).astype(np.float64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7))
    out = sign * mag
    return np.where((c & 0x7F) == 0x7F, np.nan, out)


_E4M3_GRID = e4m3_value(np.arange(127))   # the non-negative finite values, increasing with code


def e4m3_encode(x) -> np.ndarray:
    """Nearest FP8 E4M3 code of each value of x (float64 view of float32 inputs): round to
    nearest, ties to the even code (even mantissa), magnitudes at or above 448 saturate to
    ±448, the sign of zero and of values that round to zero is kept (IEEE rounding)."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    hi = np.clip(np.searchsorted(_E4M3_GRID, a, side="left"), 1, 126)   # grid[hi-1] < a <= grid[hi]
    lo = hi - 1
    d_lo = a - _E4M3_GRID[lo]
    d_hi = _E4M3_GRID[hi] - a
    pick = np.where(d_lo < d_hi, lo, np.where(d_hi < d_lo, hi, np.where(lo % 2 == 0, lo, hi)))
    pick = np.where(a >= E4M3_MAX, 126, pick)
    pick = np.where(a == 0.0, 0, pick)
    neg = np.signbit(x)
    return (pick | np.where(neg, 0x80, 0)).astype(np.uint8)


def quantize_rows_e4m3(rows):
    """Per-token quantisation of cache rows: rows [n, d] (float32 values) ->
    (codes uint8 [n, d], scales float32 [n]). Every step in float32, as the device does it."""
    r = np.asarray(rows, dtype=np.float32)
    amax = np.max(np.abs(r), axis=-1)
    scale = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    safe = np.where(scale > 0, scale, np.float32(1.0)).astype(np.float32)
    q = (r / safe[..., None]).astype(np.float32)                          # one rounding each
    codes = e4m3_encode(q.astype(np.float64))
    return codes, scale


def dequantize_rows_e4m3(codes, scales) -> np.ndarray:
    """The row values a quantised cache stores: code value × the token's scale, float64."""
    return e4m3_value(codes) * f64(scales)[..., None]


def gather_rows_fp8(codes, scales, block_table_row, L: int, page_size: int = 64) -> np.ndarray:
    """The L dequantised rows of one sequence of a quantised paged cache, read through its
    block-table row: codes [num_pages, page_size, d], scales [num_pages, page_size]."""
    idx = np.arange(L)
    pages = np.asarray(block_table_row, dtype=np.int64)[idx // page_size]
    slots = idx % page_size
    c = np.asarray(codes)[pages, slots]
    s = np.asarray(scales)[pages, slots]
    return dequantize_rows_e4m3(c, s)
