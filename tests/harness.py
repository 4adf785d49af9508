"""Shared helpers for the GPU parity tests: put a workload on the device, run the library,
and build the oracle's reference from the same generator inputs (never from GPU output)."""

from __future__ import annotations

import dataclasses

import numpy as np
import torch

import head_latent_attention_05_b200 as mla
import workloads as W
from oracle import mla_oracle as O


def tol_bound(ref: np.ndarray, dtype: str) -> float:
    """Parity bound: fp32 max|err| <= 1e-4 max|ref|; bf16 max|err| <= 1e-2 max|ref| + 1e-3."""
    m = float(np.max(np.abs(ref))) if ref.size else 0.0
    return 1e-4 * m if dtype == "f32" else 1e-2 * m + 1e-3


def assert_parity(got, ref, dtype: str, what: str = ""):
    got = O.f64(got)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = float(np.max(np.abs(got - ref))) if ref.size else 0.0
    bound = tol_bound(ref, dtype)
    assert err <= bound, f"{what}: max|err| {err:.3e} > bound {bound:.3e}"
    return err, bound


def config_of(w: W.Workload) -> mla.MlaConfig:
    return mla.make_config(w.H, w.d_model, w.d_c, w.d_r, w.d_nope, w.d_v, W.PAGE_SIZE, w.dtype,
                           w.scale, w.rms_eps, w.rope_theta, kv_format=w.kv)


def fp8_views(w: W.Workload, cache: torch.Tensor):
    """(codes [pages, 64, row] uint8, scales [pages, 64] float32) views of a quantised pool."""
    n = W.PAGE_SIZE * w.row
    return (cache[:, :n].view(cache.shape[0], W.PAGE_SIZE, w.row),
            cache[:, n:].view(torch.float32))


@dataclasses.dataclass
class Case:
    w: W.Workload
    cfg: mla.MlaConfig
    lens: torch.Tensor          # host int32 [B]
    pt: W.PageTable
    weights: W.Weights          # host
    cache_host: torch.Tensor    # history contents before the append (host)
    x_new: torch.Tensor
    seq_idx: torch.Tensor
    pos: torch.Tensor
    q: torch.Tensor
    # device copies
    d: dict


def make_case(w: W.Workload, lens: torch.Tensor | None = None, tail_fill=None,
              device="cuda", window: int = 0) -> Case:
    lens = W.seq_lens(w) if lens is None else lens.to(torch.int32)
    pt = W.page_table(w, lens)
    weights = W.weights(w)
    if w.kv == "fp8":
        cache = W.cache_pool_fp8(w, pt.num_pages)
        if tail_fill is not None:   # stale slots: NaN codes and NaN scales
            codes, scales = fp8_views(w, cache)
            for page, slot in W.tail_slots(lens, pt):
                codes[page, slot:] = 0x7F
                scales[page, slot:] = float("nan")
    else:
        cache = W.cache_pool(w, pt.num_pages)
        if tail_fill is not None:
            for page, slot in W.tail_slots(lens, pt):
                cache[page, slot:] = tail_fill
    x_new, seq_idx, pos, q = W.new_token_inputs(w, lens)
    cfg = config_of(w)
    cfg.window = window
    d = dict(
        cache=cache.to(device), block_table=pt.block_table.to(device),
        seq_lens=lens.to(device), x_new=x_new.to(device), seq_idx=seq_idx.to(device),
        pos=pos.to(device), q=q.contiguous().to(device), w_dkv=weights.w_dkv.to(device),
        kv_gain=weights.kv_gain.to(device), wkv_b=weights.wkv_b.to(device),
    )
    dt = w.torch_dtype
    d["w_uk_t"] = torch.empty((w.H, w.d_c, w.d_nope), dtype=dt, device=device)
    d["w_uv"] = torch.empty((w.H, w.d_v, w.d_c), dtype=dt, device=device)
    mla.mla_absorb_weights(cfg, d["wkv_b"], d["w_uk_t"], d["w_uv"])
    return Case(w, cfg, lens, pt, weights, cache, x_new, seq_idx, pos, q, d)


def run_append(c: Case):
    ws = mla.workspace(mla.mla_append_workspace_size(c.cfg, c.x_new.shape[0]))
    mla.mla_append_latent(c.cfg, c.d["x_new"], c.d["w_dkv"], c.d["kv_gain"], c.d["seq_idx"],
                          c.d["pos"], c.d["block_table"], c.d["cache"], ws)


def run_decode(c: Case) -> torch.Tensor:
    w = c.w
    out = torch.empty((w.B, w.Tq, w.H, w.d_v), dtype=w.torch_dtype, device="cuda")
    ws = mla.workspace(mla.mla_decode_workspace_size(c.cfg, w.B, w.Tq))
    mla.mla_decode(c.cfg, c.d["q"], c.d["cache"], c.d["block_table"], c.d["seq_lens"],
                   c.d["w_uk_t"], c.d["w_uv"], ws, out)
    return out


def oracle_new_rows(c: Case) -> np.ndarray:
    """fp64 cache rows of the appended tokens, from the oracle's own append."""
    w = c.w
    return O.latent_rows(c.x_new, c.weights.w_dkv, c.weights.kv_gain, c.pos.numpy(), w.d_c,
                         w.rms_eps, w.rope_theta)


def oracle_rows_of(c: Case, b: int, new_rows: np.ndarray) -> np.ndarray:
    """All L_b rows of sequence b as the oracle sees them: generator history, then its own new
    rows for the last Tq positions."""
    w = c.w
    L = int(c.lens[b])
    mine = new_rows[b * w.Tq:(b + 1) * w.Tq]
    if w.kv == "fp8":
        codes, scales = fp8_views(w, c.cache_host)
        rows = O.gather_rows_fp8(codes.numpy(), scales.numpy(), c.pt.block_table[b].numpy(), L,
                                 W.PAGE_SIZE)
        qc, qs = O.quantize_rows_e4m3(mine.astype(np.float32))   # the oracle's own stored rows
        rows[L - w.Tq:] = O.dequantize_rows_e4m3(qc, qs)
        return rows
    rows = O.gather_rows(c.cache_host, c.pt.block_table[b].numpy(), L, W.PAGE_SIZE)
    rows[L - w.Tq:] = mine
    return rows


def oracle_out(c: Case, b: int, heads, new_rows: np.ndarray) -> np.ndarray:
    """Oracle output [Tq, len(heads), d_v] for sequence b (expanded form, the case's window)."""
    w = c.w
    W_UK, W_UV = O.split_wkv_b(c.weights.wkv_b, w.H, w.d_nope, w.d_v)
    rows = oracle_rows_of(c, b, new_rows)
    return O.decode_expanded(c.q[b], rows, W_UK, W_UV, w.scale, w.rope_theta, heads=heads,
                             window=int(c.cfg.window))


def plant_score_staircase(c: Case, b: int, h: int, t: int = 0, base: float = 8.0,
                          step: float = 7.0, period: int = 4, slot: int = 10) -> list:
    """Overwrite one history row per 64-token page of sequence b so that, for head h and query
    token t, the planted rows score base + step * (page % period) (natural-log units, after the
    softmax scale) and dominate their page. Consecutive pages then raise the running maximum by
    `step` > 8 ln 2, which is what makes the attention kernel move its reference maximum and
    rescale its accumulator inside a segment. The planted row is c = (s / scale) q_lat / |q_lat|^2
    with k_R = 0 (q_lat = q_nope W_UK[h], from the same inputs the oracle gets), rounded to the
    cache dtype; host and device caches are updated alike. Returns the planted positions."""
    w = c.w
    L = int(c.lens[b])
    W_UK, _ = O.split_wkv_b(c.weights.wkv_b, w.H, w.d_nope, w.d_v)
    q_lat = O.f64(c.q[b, t, h, :w.d_nope]) @ W_UK[h]
    planted = []
    for page_i in range((L - w.Tq) // W.PAGE_SIZE + 1):
        j = page_i * W.PAGE_SIZE + slot
        if j >= L - w.Tq:
            break
        s = base + step * (page_i % period)
        row = np.zeros(w.row)
        row[:w.d_c] = (s / w.scale) * q_lat / float(q_lat @ q_lat)
        page = int(c.pt.block_table[b, page_i])
        if w.kv == "fp8":
            qc, qs = O.quantize_rows_e4m3(row[None].astype(np.float32))
            for cache in (c.cache_host, c.d["cache"]):
                codes, scales = fp8_views(w, cache)
                codes[page, slot] = torch.from_numpy(qc[0]).to(cache.device)
                scales[page, slot] = float(qs[0])
        else:
            val = torch.from_numpy(row).to(w.torch_dtype)
            c.cache_host[page, slot] = val
            c.d["cache"][page, slot] = val.to(c.d["cache"].device)
        planted.append(j)
    return planted


def oracle_scores(c: Case, b: int, h: int, t: int, rows: np.ndarray) -> np.ndarray:
    """Scaled scores of head h, query token t of sequence b against every row (fp64, from the
    oracle's own pieces), used to check properties of a test's inputs."""
    w = c.w
    W_UK, _ = O.split_wkv_b(c.weights.wkv_b, w.H, w.d_nope, w.d_v)
    L = rows.shape[0]
    q = O.f64(c.q[b, t, h])
    qf = np.concatenate([q[:w.d_nope], O.rope(q[w.d_nope:], L - w.Tq + t, w.rope_theta)])
    K = np.concatenate([rows[:, :w.d_c] @ W_UK[h].T, rows[:, w.d_c:]], axis=1)
    return (K @ qf) * w.scale
