"""Sliding-window decode and split-KV decode (key ranges merged across GPUs), on the GPU
through the C ABI, against the fp64 oracle.

Window: a query at position p sees keys p - window < j <= p (the Streaming-MLA variant of
「Multi-Head Latent Attention（MLA）原理与工程实践全解析」 §7). Pages wholly before the window must
never be read: their block-table entries are made invalid, and the slots before the window in
the first visible page hold NaN.
Split-KV: every sequence's pages are dealt out over emulated ranks (split_kv.kv_ranges); each
range runs mla_decode_partial on this GPU one after the other (nothing waits on another range),
and mla_combine merges the stacked partials. Pages outside a range get invalid block-table
entries for that range's call. Tolerances: fp32 1e-4 max|ref|; bf16 1e-2 max|ref| + 1e-3.
"""

import numpy as np
import pytest
import torch

import harness as Hs
import head_latent_attention_05_b200 as mla
import workloads as W
from head_latent_attention_05_b200.split_kv import kv_ranges
from oracle import mla_oracle as O

pytestmark = pytest.mark.gpu

TINY = W.WORKLOADS["tiny_f32_b1_h4_ctx128"]
V2 = W.WORKLOADS["v2_bf16_b16_ctx4096"]
H32 = W.WORKLOADS["h32_bf16_b32_ctx512to8192_shuffled"]
LONG = W.WORKLOADS["v2_bf16_b4_ctx131072_tq2"]


@pytest.fixture(autouse=True)
def _no_device_error():
    mla.mla_get_device_error()
    yield
    assert mla.mla_get_device_error() == 0


def _lens(*ls):
    return torch.tensor(ls, dtype=torch.int32)


def _check(c, out, heads=None, bs=None):
    new_rows = Hs.oracle_new_rows(c)
    for b in (range(c.w.B) if bs is None else bs):
        hs = list(range(c.w.H)) if heads is None else heads
        Hs.assert_parity(out[b][:, hs], Hs.oracle_out(c, b, hs, new_rows), c.w.dtype,
                         f"b={b} L={int(c.lens[b])} window={int(c.cfg.window)}")


# ------------------------------------------------------------------------------ window

@pytest.mark.parametrize("window", [1, 64, 100, 1024])
def test_window_decode_parity_v2(window):
    c = Hs.make_case(W.small_variant(V2, B=4, pages="shuffled"), _lens(5000, 64, 1500, 3000),
                     window=window)
    Hs.run_append(c)
    _check(c, Hs.run_decode(c).float().cpu(), heads=[0, 63, 127])


def test_window_never_reads_pages_before_it():
    """Pages wholly before the window have invalid block-table entries and the slots before the
    window in the first visible page hold NaN: no device error, output as the oracle's."""
    window = 200
    lens = _lens(3000, 900, 250)
    c = Hs.make_case(W.small_variant(V2, B=3), lens, window=window)
    Hs.run_append(c)
    for b, L in enumerate(lens.tolist()):
        lo = max(0, L - window)                    # first key the (single) query sees
        for pg in range(lo // 64):
            c.d["block_table"][b, pg] = c.pt.num_pages + 7
        page = int(c.pt.block_table[b, lo // 64])
        if lo % 64:
            c.d["cache"][page, :lo % 64] = float("nan")
    out = Hs.run_decode(c).float().cpu()
    assert torch.isfinite(out).all()
    _check(c, out, heads=[0, 77, 127])


def test_window_two_causal_queries():
    c = Hs.make_case(W.small_variant(LONG, B=2), _lens(3000, 700), window=100)
    Hs.run_append(c)
    _check(c, Hs.run_decode(c).float().cpu(), heads=[0, 5, 127])


def test_window_fp32_cuda_cores():
    c = Hs.make_case(W.small_variant(TINY, B=2), _lens(128, 40), window=17)
    Hs.run_append(c)
    _check(c, Hs.run_decode(c).cpu())


# ---------------------------------------------------------------------------- split-KV

def _split_decode(c, world, bogus_outside=True):
    """Run every emulated rank's mla_decode_partial in turn, then mla_combine. Returns the
    combined output and the per-rank (o_part, lse)."""
    w = c.w
    rows = w.B * w.Tq * w.H
    ranges = kv_ranges(c.lens.tolist(), world)
    o_parts = torch.empty((world, rows, w.d_c), dtype=w.torch_dtype, device="cuda")
    lse = torch.empty((world, rows), dtype=torch.float32, device="cuda")
    ws = mla.workspace(mla.mla_decode_workspace_size(c.cfg, w.B, w.Tq))
    for r in range(world):
        bt = c.d["block_table"].clone()
        if bogus_outside:   # this rank holds only the pages of its ranges
            for b, (a, e) in enumerate(ranges[r]):
                for pg in range(bt.shape[1]):
                    if not (a // 64 <= pg < (e + 63) // 64):
                        bt[b, pg] = c.pt.num_pages + 3
        kb = torch.tensor([a for a, _ in ranges[r]], dtype=torch.int32, device="cuda")
        ke = torch.tensor([e for _, e in ranges[r]], dtype=torch.int32, device="cuda")
        mla.mla_decode_partial(c.cfg, c.d["q"], c.d["cache"], bt, c.d["seq_lens"], kb, ke,
                               c.d["w_uk_t"], ws, o_parts[r], lse[r])
    out = torch.empty((w.B, w.Tq, w.H, w.d_v), dtype=w.torch_dtype, device="cuda")
    n = mla.mla_combine_workspace_size(c.cfg, w.B, w.Tq)
    mla.mla_combine(c.cfg, o_parts, lse, c.d["w_uv"], mla.workspace(n) if n else None, out)
    return out, o_parts, lse, ranges


@pytest.mark.parametrize("w,lens,world", [
    (W.small_variant(V2, B=3, pages="shuffled"), _lens(6000, 700, 129), 2),
    (W.small_variant(V2, B=3), _lens(6000, 700, 129), 3),
    (W.small_variant(H32, B=4), _lens(3000, 64, 1, 999), 4),
    (W.small_variant(LONG, B=2), _lens(4000, 130), 2),
    (W.small_variant(TINY, B=2), _lens(128, 70), 2),
], ids=["v2_w2", "v2_w3", "h32_w4", "tq2_w2", "tiny_f32_w2"])
def test_split_kv_partials_combine_to_the_decode(w, lens, world):
    c = Hs.make_case(w, lens)
    Hs.run_append(c)
    out, o_parts, lse, ranges = _split_decode(c, world)
    out = out.float().cpu()
    heads = list(range(w.H)) if w.H <= 8 else [0, w.H // 2, w.H - 1]
    _check(c, out, heads=heads)
    # and the whole-sequence decode on one GPU agrees within the same bound
    ref = Hs.run_decode(c).float().cpu()
    for b in range(w.B):
        Hs.assert_parity(out[b], ref[b].numpy().astype(np.float64), w.dtype, f"vs decode b={b}")


def test_split_kv_partials_match_the_oracle_partials():
    """One rank's o_part / lse against oracle.latent_partial over the same key range."""
    w = W.small_variant(V2, B=2)
    c = Hs.make_case(w, _lens(3000, 300))
    Hs.run_append(c)
    _, o_parts, lse, ranges = _split_decode(c, 2)
    new_rows = Hs.oracle_new_rows(c)
    W_UK, _ = O.split_wkv_b(c.weights.wkv_b, w.H, w.d_nope, w.d_v)
    heads = [0, 64, 127]
    for r in range(2):
        for b in range(w.B):
            a, e = ranges[r][b]
            rows = Hs.oracle_rows_of(c, b, new_rows)
            o_ref, l_ref = O.latent_partial(c.q[b], rows, W_UK, w.scale, w.rope_theta, a, e,
                                            heads=heads)
            got_o = o_parts[r].float().cpu().view(w.B, w.Tq, w.H, w.d_c)[b][:, heads]
            got_l = lse[r].cpu().view(w.B, w.Tq, w.H)[b][:, heads].double().numpy()
            if a == e:
                assert np.all(got_l == -np.inf) and torch.count_nonzero(got_o) == 0
                continue
            Hs.assert_parity(got_o, o_ref, "bf16", f"o_part rank {r} b={b}")
            assert np.max(np.abs(got_l - l_ref)) <= 1e-2 * np.max(np.abs(l_ref)) + 1e-3


def test_split_kv_with_window():
    c = Hs.make_case(W.small_variant(V2, B=2), _lens(5000, 1000), window=700)
    Hs.run_append(c)
    out, _, _, _ = _split_decode(c, 3)
    _check(c, out.float().cpu(), heads=[0, 127])
