"""GPU parity of the CUDA path (through the C ABI) against the fp64 oracle.

Tolerances: fp32 workloads max|err| <= 1e-4 max|ref|; bf16-cache workloads
max|err| <= 1e-2 max|ref| + 1e-3. Placement, paging and indexing are checked bit-exactly.
"""

import numpy as np
import pytest
import torch

import head_latent_attention_05_b200 as mla
import workloads as W
from oracle import mla_oracle as O
import harness as Hs

pytestmark = pytest.mark.gpu

TINY = W.WORKLOADS["tiny_f32_b1_h4_ctx128"]
V2 = W.WORKLOADS["v2_bf16_b16_ctx4096"]
H32 = W.WORKLOADS["h32_bf16_b32_ctx512to8192_shuffled"]
MIX = W.WORKLOADS["v2_bf16_b64_ctx1kto32k_mix"]
LONG = W.WORKLOADS["v2_bf16_b4_ctx131072_tq2"]


@pytest.fixture(autouse=True)
def _no_device_error():
    mla.mla_get_device_error()
    yield
    assert mla.mla_get_device_error() == 0


def _lens(*ls):
    return torch.tensor(ls, dtype=torch.int32)


# ------------------------------------------------------------------------------- absorb

@pytest.mark.parametrize("w", [TINY, W.small_variant(V2, H=16)], ids=lambda w: w.dtype)
def test_absorb_weights_bit_exact(w):
    c = Hs.make_case(W.small_variant(w, B=1, lens=("fixed", 64)))
    blk = c.weights.wkv_b.view(w.H, w.d_nope + w.d_v, w.d_c)
    assert torch.equal(c.d["w_uk_t"].cpu(), blk[:, :w.d_nope, :].transpose(1, 2).contiguous())
    assert torch.equal(c.d["w_uv"].cpu(), blk[:, w.d_nope:, :].contiguous())


# ------------------------------------------------------------------------------- append

@pytest.mark.parametrize("w,lens", [
    (TINY, _lens(128)),
    (W.small_variant(H32, B=4), _lens(70, 64, 1, 513)),
    (W.small_variant(V2, B=3, pages="shuffled"), _lens(5, 200, 64)),
    (W.small_variant(LONG, B=2), _lens(2, 131)),
], ids=["tiny_f32", "h32_bf16", "v2_bf16", "tq2_bf16"])
def test_append_placement_bit_exact_and_values(w, lens):
    c = Hs.make_case(w, lens)
    before = c.d["cache"].clone()
    Hs.run_append(c)
    torch.cuda.synchronize()
    after = c.d["cache"]
    written = torch.zeros(after.shape[:2], dtype=torch.bool)
    for i in range(c.x_new.shape[0]):
        b, p = int(c.seq_idx[i]), int(c.pos[i])
        written[int(c.pt.block_table[b, p // W.PAGE_SIZE]), p % W.PAGE_SIZE] = True
    # every other cell keeps its exact previous bits
    keep = ~written.to(after.device)
    assert torch.equal(after[keep].view(torch.int16 if w.dtype == "bf16" else torch.int32),
                       before[keep].view(torch.int16 if w.dtype == "bf16" else torch.int32))
    ref = Hs.oracle_new_rows(c)
    got = np.stack([O.f64(after[int(c.pt.block_table[int(c.seq_idx[i]), int(c.pos[i]) // 64]),
                                int(c.pos[i]) % 64].cpu()) for i in range(c.x_new.shape[0])])
    Hs.assert_parity(got, ref, w.dtype, "appended rows")


# ------------------------------------------------------------------------------- decode

def _decode_and_check(c, heads=None, bs=None):
    Hs.run_append(c)
    out = Hs.run_decode(c).float().cpu()
    new_rows = Hs.oracle_new_rows(c)
    bs = range(c.w.B) if bs is None else bs
    for b in bs:
        hs = list(range(c.w.H)) if heads is None else heads
        ref = Hs.oracle_out(c, b, hs, new_rows)
        Hs.assert_parity(out[b][:, hs], ref, c.w.dtype, f"b={b} L={int(c.lens[b])}")
    return out


def test_tiny_f32_whole_sequence_through_append():
    """All 128 tokens appended from x on the GPU; the oracle builds its rows from the same x."""
    w = TINY
    lens = W.seq_lens(w)
    c = Hs.make_case(w, lens)
    x = W.full_sequence_x(w, lens)[0]                         # [128, d_model]
    L = int(lens[0])
    d = c.d
    d["x_new"] = x.to("cuda")
    d["seq_idx"] = torch.zeros(L, dtype=torch.int32, device="cuda")
    d["pos"] = torch.arange(L, dtype=torch.int32, device="cuda")
    ws = mla.workspace(mla.mla_append_workspace_size(c.cfg, L))
    mla.mla_append_latent(c.cfg, d["x_new"], d["w_dkv"], d["kv_gain"], d["seq_idx"], d["pos"],
                          d["block_table"], d["cache"], ws)
    out = Hs.run_decode(c).cpu()
    rows = O.latent_rows(x, c.weights.w_dkv, c.weights.kv_gain, np.arange(L), w.d_c, w.rms_eps,
                         w.rope_theta)
    W_UK, W_UV = O.split_wkv_b(c.weights.wkv_b, w.H, w.d_nope, w.d_v)
    ref = O.decode_expanded(c.q[0], rows, W_UK, W_UV, w.scale, w.rope_theta)
    Hs.assert_parity(out[0], ref, "f32", "tiny")


@pytest.mark.parametrize("w,lens", [
    (TINY, _lens(128)),
    (W.small_variant(TINY, B=3), _lens(1, 65, 300)),
    (W.small_variant(V2, B=3), _lens(1, 130, 700)),
    (W.small_variant(H32, B=5), _lens(70, 512, 64, 1100, 3)),
    (W.small_variant(MIX, B=4), _lens(1024, 1500, 65, 2049)),
    (W.small_variant(LONG, B=3), _lens(2, 65, 777)),
], ids=["tiny", "tiny_b3", "v2_b3", "h32_b5", "mix_b4", "tq2_b3"])
def test_decode_parity_all_heads(w, lens):
    _decode_and_check(Hs.make_case(w, lens))


@pytest.mark.parametrize("L", [1, 2, 63, 64, 65, 127, 128, 129, 191, 4097])
def test_decode_edge_lengths_v2(L):
    w = W.small_variant(V2, B=1)
    _decode_and_check(Hs.make_case(w, _lens(L)), heads=[0, 1, 63, 64, 127])


@pytest.mark.parametrize("L", [2, 3, 64, 65, 66, 128, 129])
def test_decode_edge_lengths_two_queries(L):
    w = W.small_variant(LONG, B=1)
    _decode_and_check(Hs.make_case(w, _lens(L)), heads=[0, 5, 127])


def test_decode_nonfinite_stale_tail_is_ignored():
    """Unwritten slots of a sequence's last page hold NaN; the output must not see them."""
    w = W.small_variant(V2, B=3)
    _decode_and_check(Hs.make_case(w, _lens(65, 100, 191), tail_fill=float("nan")),
                      heads=[0, 77, 127])


def test_decode_long_sequence_alone_and_in_batch():
    """A long sequence alone is split over every CTA pair; inside a batch of short ones it gets
    few splits. Both match the oracle, and a repeated call is bit-identical."""
    alone = Hs.make_case(W.small_variant(V2, B=1), _lens(6000))
    out1 = _decode_and_check(alone, heads=[0, 127])
    out2 = Hs.run_decode(alone).float().cpu()
    assert torch.equal(out1, out2)
    mixed = Hs.make_case(W.small_variant(V2, B=6), _lens(6000, 64, 65, 1, 300, 129))
    _decode_and_check(mixed, heads=[0, 64, 127])


def test_decode_more_sequences_than_cta_pairs():
    """160 short sequences: more units than CTA pairs, so pairs run several units each and
    the planner's multi-segment ranges, empty-unit edges and pair starts are all exercised."""
    g = torch.Generator().manual_seed(11)
    lens = torch.randint(1, 300, (160,), generator=g, dtype=torch.int32)
    lens[::37] = 1
    c = Hs.make_case(W.small_variant(V2, B=160), lens)
    _decode_and_check(c, heads=[0, 127], bs=list(range(0, 160, 9)) + [159])


def test_decode_profiled_matches_decode_and_records_events():
    """mla_decode_profiled computes exactly what mla_decode computes and records its four
    events in order."""
    w = W.small_variant(V2, B=3)
    c = Hs.make_case(w, _lens(4097, 65, 300))
    Hs.run_append(c)
    ref = Hs.run_decode(c)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    for e in ev:
        e.record()
    out = torch.empty_like(ref)
    ws = mla.workspace(mla.mla_decode_workspace_size(c.cfg, w.B, w.Tq))
    mla.mla_decode_profiled(c.cfg, c.d["q"], c.d["cache"], c.d["block_table"], c.d["seq_lens"],
                            c.d["w_uk_t"], c.d["w_uv"], ws, out, ev)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    gaps = [ev[i].elapsed_time(ev[i + 1]) for i in range(3)]
    assert all(t >= 0.0 for t in gaps) and gaps[1] > 0.0   # the attention kernel takes time


@pytest.mark.parametrize("name", ["v2_bf16_b16_ctx4096", "h32_bf16_b32_ctx512to8192_shuffled",
                                  "v2_bf16_b64_ctx1kto32k_mix", "v2_bf16_b4_ctx131072_tq2"])
def test_decode_full_size_sampled(name):
    """Full-size workloads in the launch configuration the benchmark times: every sequence,
    heads {0, H/2, H-1} plus two seeded heads per sequence, against the oracle."""
    w = W.WORKLOADS[name]
    c = Hs.make_case(w)
    Hs.run_append(c)
    out = Hs.run_decode(c).float().cpu()
    assert torch.isfinite(out).all()
    new_rows = Hs.oracle_new_rows(c)
    rng = np.random.default_rng(123)
    for b in range(w.B):
        hs = sorted(set([0, w.H // 2, w.H - 1] + [int(v) for v in rng.integers(0, w.H, 2)]))
        ref = Hs.oracle_out(c, b, hs, new_rows)
        Hs.assert_parity(out[b][:, hs], ref, w.dtype, f"{name} b={b} L={int(c.lens[b])}")


# ------------------------------------------------------------------------------ prefill

@pytest.mark.parametrize("w,lens,t_new", [
    (TINY, _lens(128), 128),
    (W.small_variant(TINY, B=2), _lens(40, 9), 9),
    (W.small_variant(H32, B=2), _lens(100, 70), 7),
], ids=["tiny_prompt", "tiny_b2", "h32_b2"])
def test_prefill_ref_parity(w, lens, t_new):
    w = W.small_variant(w, Tq=t_new)
    c = Hs.make_case(w, lens)
    out = torch.empty((w.B, t_new, w.H, w.d_v), dtype=w.torch_dtype, device="cuda")
    x = c.d["x_new"].view(w.B, t_new, w.d_model)
    ws = mla.workspace(mla.mla_prefill_ref_workspace_size(c.cfg, w.B, t_new))
    mla.mla_prefill_ref(c.cfg, x, c.d["q"], c.d["w_dkv"], c.d["kv_gain"], c.d["w_uk_t"],
                        c.d["w_uv"], c.d["seq_lens"], c.d["block_table"], c.d["cache"], ws, out)
    out = out.float().cpu()
    new_rows = Hs.oracle_new_rows(c)
    for b in range(w.B):
        ref = Hs.oracle_out(c, b, list(range(w.H)), new_rows)
        Hs.assert_parity(out[b], ref, w.dtype, f"prefill b={b}")


# ------------------------------------------------------------------------- device errors

def test_device_error_bad_page_is_reported_not_faulted():
    w = W.small_variant(V2, B=2)
    c = Hs.make_case(w, _lens(100, 100))
    c.d["block_table"][1, 1] = c.pt.num_pages + 5           # out of the pool
    out = Hs.run_decode(c)
    assert mla.mla_get_device_error() == 6
    assert torch.isfinite(out[0].float()).all()


def test_device_error_bad_length_zero_output():
    w = W.small_variant(V2, B=2)
    c = Hs.make_case(w, _lens(100, 100))
    c.d["seq_lens"][1] = 10_000_000                          # beyond the block table
    out = Hs.run_decode(c).float()
    assert mla.mla_get_device_error() == 7
    assert torch.count_nonzero(out[1]) == 0
    c.d["seq_lens"][1] = 0                                   # shorter than Tq
    out = Hs.run_decode(c).float()
    assert mla.mla_get_device_error() == 7
    assert torch.count_nonzero(out[1]) == 0


def test_append_bad_position_is_skipped_and_reported():
    w = W.small_variant(V2, B=2)
    c = Hs.make_case(w, _lens(100, 100))
    before = c.d["cache"].clone()
    c.d["pos"][1] = 64 * c.pt.max_pages + 3                  # past the block table
    Hs.run_append(c)
    assert mla.mla_get_device_error() == 6
    # only sequence 0's row changed
    changed = (c.d["cache"].view(torch.int16) != before.view(torch.int16)).any(-1)
    p0 = int(c.pos[0])
    assert int(changed.sum()) == 1
    assert bool(changed[int(c.pt.block_table[0, p0 // 64]), p0 % 64])
