"""GPU parity of the quantised latent cache (FP8 E4M3 codes, one float32 scale per token)
through the C ABI, against the fp64 oracle.

* The quantiser's integer decisions (codes and scales) are bit-exact against the oracle's
  float32 quantiser on the same float32 rows (mla_quantize_latent), including exact ties,
  saturation, zero rows and signed zeros; every byte it does not address keeps its value.
* The quantised append writes exactly the addressed slots; its rows dequantise to the oracle's
  rows within the E4M3 rounding bound.
* Decode, prefill and partial decode over a quantised cache match the oracle run on the
  dequantised rows (the oracle quantises its own new rows) within the bf16 parity bound,
  including edge lengths, two query tokens, NaN-filled stale slots, the rescale path, a window,
  full size and a cache of subnormal codes only.
"""

import numpy as np
import pytest
import torch

import head_latent_attention_05_b200 as mla
import workloads as W
from oracle import mla_oracle as O
import harness as Hs

pytestmark = pytest.mark.gpu

V2 = W.small_variant(W.WORKLOADS["v2_bf16_b16_ctx4096"], kv="fp8")
MIX = W.EXTRA_WORKLOADS["v2_fp8_b64_ctx1kto32k_mix"]
LONG = W.small_variant(W.WORKLOADS["v2_bf16_b4_ctx131072_tq2"], kv="fp8")
H32 = W.small_variant(W.WORKLOADS["h32_bf16_b32_ctx512to8192_shuffled"], kv="fp8")


@pytest.fixture(autouse=True)
def _no_device_error():
    mla.mla_get_device_error()
    yield
    assert mla.mla_get_device_error() == 0


def _lens(*ls):
    return torch.tensor(ls, dtype=torch.int32)


def _decode_and_check(c, heads=None, bs=None):
    Hs.run_append(c)
    out = Hs.run_decode(c).float().cpu()
    new_rows = Hs.oracle_new_rows(c)
    for b in (range(c.w.B) if bs is None else bs):
        hs = list(range(c.w.H)) if heads is None else heads
        ref = Hs.oracle_out(c, b, hs, new_rows)
        Hs.assert_parity(out[b][:, hs], ref, "bf16", f"fp8 b={b} L={int(c.lens[b])}")
    return out


# ----------------------------------------------------------------------------- quantiser

def _quantize_rows_input(row):
    rng = np.random.default_rng(9)
    rows = [rng.standard_normal(row) * 2.0 ** float(e) for e in (-30, -8, 0, 3, 17)]
    ties = np.zeros(row)          # max 448 -> scale exactly 1: codes are E4M3 of the values
    ties[0] = 448.0
    grid = O.e4m3_value(np.arange(1, 127))
    mids = (grid[:-1] + grid[1:]) / 2
    ties[1:1 + mids.size] = mids
    ties[1 + mids.size:1 + 2 * mids.size] = -mids[: row - 1 - mids.size][: mids.size]
    rows.append(ties)
    zero = np.zeros(row)
    zero[::3] = -0.0
    rows.append(zero)
    spiky = rng.standard_normal(row) * 1e-3
    spiky[5] = 1e4
    rows.append(spiky)
    return np.stack(rows).astype(np.float32)


def test_quantize_latent_bit_exact_against_oracle():
    w = W.small_variant(V2, B=3, pages="shuffled")
    cfg = Hs.config_of(w)
    lens = _lens(130, 64, 300)
    pt = W.page_table(w, lens)
    rows = _quantize_rows_input(w.row)
    n = rows.shape[0]
    seq_idx = torch.tensor([i % 3 for i in range(n)], dtype=torch.int32)
    pos = torch.tensor([(37 * i + 5) % int(lens[i % 3]) for i in range(n)], dtype=torch.int32)
    cache = torch.full((pt.num_pages, w.fp8_page_bytes), 0xAB, dtype=torch.uint8, device="cuda")
    before = cache.clone()
    mla.mla_quantize_latent(cfg, torch.from_numpy(rows).cuda(), seq_idx.cuda(), pos.cuda(),
                            pt.block_table.cuda(), cache)
    torch.cuda.synchronize()
    codes_ref, scales_ref = O.quantize_rows_e4m3(rows)
    codes, scales = Hs.fp8_views(w, cache)
    touched = torch.zeros_like(cache, dtype=torch.bool)
    for i in range(n):
        b, p = int(seq_idx[i]), int(pos[i])
        page, slot = int(pt.block_table[b, p // 64]), p % 64
        assert np.array_equal(codes[page, slot].cpu().numpy(), codes_ref[i]), f"codes of row {i}"
        got_s = scales[page, slot].cpu().numpy()
        assert got_s.tobytes() == np.float32(scales_ref[i]).tobytes(), f"scale of row {i}"
        touched[page, slot * w.row:(slot + 1) * w.row] = True
        off = 64 * w.row + 4 * slot
        touched[page, off:off + 4] = True
    assert torch.equal(cache[~touched], before[~touched])


def test_quantize_latent_rejects_a_plain_cache_config():
    w = W.small_variant(V2, kv="plain")
    cfg = Hs.config_of(w)
    z = torch.zeros(16, dtype=torch.int32, device="cuda")
    with pytest.raises(mla.MlaError) as e:
        mla.mla_quantize_latent(cfg, torch.zeros((1, w.row), device="cuda"), z[:1], z[:1],
                                z.view(1, 16), torch.zeros((1, 64 * w.row * 2), dtype=torch.uint8,
                                                          device="cuda"))
    assert e.value.code == 1


# ------------------------------------------------------------------------------- append

@pytest.mark.parametrize("w,lens", [
    (W.small_variant(V2, B=3, pages="shuffled"), _lens(5, 200, 64)),
    (W.small_variant(H32, B=4), _lens(70, 64, 1, 513)),
    (W.small_variant(LONG, B=2), _lens(2, 131)),
], ids=["v2", "h32", "tq2"])
def test_fp8_append_placement_bit_exact_and_values(w, lens):
    c = Hs.make_case(w, lens)
    before = c.d["cache"].clone()
    Hs.run_append(c)
    torch.cuda.synchronize()
    after = c.d["cache"]
    touched = torch.zeros_like(after, dtype=torch.bool)
    slots = []
    for i in range(c.x_new.shape[0]):
        b, p = int(c.seq_idx[i]), int(c.pos[i])
        page, slot = int(c.pt.block_table[b, p // 64]), p % 64
        slots.append((page, slot))
        touched[page, slot * w.row:(slot + 1) * w.row] = True
        off = 64 * w.row + 4 * slot
        touched[page, off:off + 4] = True
    assert torch.equal(after[~touched], before[~touched])
    codes, scales = Hs.fp8_views(w, after.cpu())
    ref = Hs.oracle_new_rows(c)
    for i, (page, slot) in enumerate(slots):
        cd = codes[page, slot].numpy()
        sc = float(scales[page, slot])
        amax = float(np.max(np.abs(ref[i])))
        assert abs(sc - amax / 448.0) <= 1e-4 * amax / 448.0, f"scale of token {i}"
        assert np.max(cd & 0x7F) == 0x7E          # the row maximum is coded as ±448
        deq = O.dequantize_rows_e4m3(cd[None], np.float32(sc)[None])[0]
        bound = 2.0 ** -4 * np.abs(ref[i]) + 2.0 ** -10 * sc + 1e-5 * amax
        assert np.all(np.abs(deq - ref[i]) <= bound), f"dequantised row of token {i}"


# ------------------------------------------------------------------------------- decode

@pytest.mark.parametrize("w,lens", [
    (W.small_variant(V2, B=3), _lens(1, 130, 700)),
    (W.small_variant(H32, B=5), _lens(70, 512, 64, 1100, 3)),
    (W.small_variant(MIX, B=4), _lens(1024, 1500, 65, 2049)),
    (W.small_variant(LONG, B=3), _lens(2, 65, 777)),
], ids=["v2_b3", "h32_b5", "mix_b4", "tq2_b3"])
def test_fp8_decode_parity_all_heads(w, lens):
    _decode_and_check(Hs.make_case(w, lens))


@pytest.mark.parametrize("L", [1, 2, 63, 64, 65, 128, 129, 4097])
def test_fp8_decode_edge_lengths(L):
    _decode_and_check(Hs.make_case(W.small_variant(V2, B=1), _lens(L)), heads=[0, 1, 63, 64, 127])


@pytest.mark.parametrize("L", [2, 3, 65, 129])
def test_fp8_decode_edge_lengths_two_queries(L):
    _decode_and_check(Hs.make_case(W.small_variant(LONG, B=1), _lens(L)), heads=[0, 5, 127])


def test_fp8_decode_nonfinite_stale_tail_is_ignored():
    """Unwritten slots hold NaN codes and NaN scales; the output must not see them."""
    c = Hs.make_case(W.small_variant(V2, B=3), _lens(65, 100, 191), tail_fill=float("nan"))
    _decode_and_check(c, heads=[0, 77, 127])


def test_fp8_decode_long_sequence_split_over_every_pair_and_repeatable():
    c = Hs.make_case(W.small_variant(V2, B=1), _lens(6000))
    out1 = _decode_and_check(c, heads=[0, 127])
    out2 = Hs.run_decode(c).float().cpu()
    assert torch.equal(out1, out2)
    mixed = Hs.make_case(W.small_variant(V2, B=6), _lens(6000, 64, 65, 1, 300, 129))
    _decode_and_check(mixed, heads=[0, 64, 127])


def test_fp8_decode_rescale_path():
    """Planted rows raise the running maximum by more than 8 (log2 units) page after page, so
    the kernel rescales its accumulator inside a segment."""
    c = Hs.make_case(W.small_variant(V2, B=1), _lens(2000))
    planted = Hs.plant_score_staircase(c, b=0, h=3)
    rows = Hs.oracle_rows_of(c, 0, Hs.oracle_new_rows(c))
    s = Hs.oracle_scores(c, 0, 3, 0, rows)
    first = s[:64].max()
    assert s[planted].max() - first > 8 * np.log(2.0)
    _decode_and_check(c, heads=[0, 3, 127])


def test_fp8_decode_window():
    c = Hs.make_case(W.small_variant(V2, B=3), _lens(3000, 700, 64), window=1024)
    _decode_and_check(c, heads=[0, 64, 127])


@pytest.mark.parametrize("name", ["v2_fp8_b64_ctx1kto32k_mix"])
def test_fp8_decode_full_size_sampled(name):
    """The benchmark's quantised workload at full size: every sequence, heads {0, H/2, H-1}
    plus two seeded heads per sequence."""
    w = W.EXTRA_WORKLOADS[name]
    c = Hs.make_case(w)
    Hs.run_append(c)
    out = Hs.run_decode(c).float().cpu()
    assert torch.isfinite(out).all()
    new_rows = Hs.oracle_new_rows(c)
    rng = np.random.default_rng(123)
    for b in range(w.B):
        hs = sorted(set([0, w.H // 2, w.H - 1] + [int(v) for v in rng.integers(0, w.H, 2)]))
        ref = Hs.oracle_out(c, b, hs, new_rows)
        Hs.assert_parity(out[b][:, hs], ref, "bf16", f"{name} b={b} L={int(c.lens[b])}")


# ------------------------------------------------------------------ prefill and partials

def test_fp8_prefill_parity():
    w = W.small_variant(V2, B=2, Tq=40)
    c = Hs.make_case(w, _lens(300, 40))
    out = torch.empty((w.B, w.Tq, w.H, w.d_v), dtype=torch.bfloat16, device="cuda")
    x = c.d["x_new"].view(w.B, w.Tq, w.d_model)
    ws = mla.workspace(mla.mla_prefill_workspace_size(c.cfg, w.B, w.Tq))
    mla.mla_prefill(c.cfg, x, c.d["q"], c.d["w_dkv"], c.d["kv_gain"], c.d["w_uk_t"], c.d["w_uv"],
                    c.d["seq_lens"], c.d["block_table"], c.d["cache"], ws, out)
    out = out.float().cpu()
    new_rows = Hs.oracle_new_rows(c)
    for b in range(w.B):
        ref = Hs.oracle_out(c, b, [0, 9, 127], new_rows)
        Hs.assert_parity(out[b][:, [0, 9, 127]], ref, "bf16", f"fp8 prefill b={b}")


def test_fp8_prefill_ref_is_unsupported():
    w = W.small_variant(V2, B=1, Tq=1)
    c = Hs.make_case(w, _lens(64))
    out = torch.empty((1, 1, w.H, w.d_v), dtype=torch.bfloat16, device="cuda")
    ws = mla.workspace(1 << 20)
    with pytest.raises(mla.MlaError) as e:
        mla.mla_prefill_ref(c.cfg, c.d["x_new"].view(1, 1, -1), c.d["q"], c.d["w_dkv"],
                            c.d["kv_gain"], c.d["w_uk_t"], c.d["w_uv"], c.d["seq_lens"],
                            c.d["block_table"], c.d["cache"], ws, out)
    assert e.value.code == 2


def test_fp8_partials_merge_to_decode():
    """Two key ranges decoded separately over the quantised cache and merged by mla_combine
    give mla_decode's result (within rounding), and each partial matches the oracle's."""
    w = W.small_variant(V2, B=2)
    c = Hs.make_case(w, _lens(1000, 130))
    Hs.run_append(c)
    full = Hs.run_decode(c).float().cpu()
    cut = torch.tensor([512, 64], dtype=torch.int32)
    ranges = [(torch.zeros(2, dtype=torch.int32), cut), (cut, c.lens.clone())]
    rows_n = w.B * w.Tq * w.H
    parts, lses = [], []
    for kb, ke in ranges:
        o = torch.empty((rows_n, w.d_c), dtype=torch.bfloat16, device="cuda")
        lse = torch.empty(rows_n, dtype=torch.float32, device="cuda")
        ws = mla.workspace(mla.mla_decode_workspace_size(c.cfg, w.B, w.Tq))
        mla.mla_decode_partial(c.cfg, c.d["q"], c.d["cache"], c.d["block_table"], c.d["seq_lens"],
                               kb.cuda(), ke.cuda(), c.d["w_uk_t"], ws, o, lse)
        parts.append(o)
        lses.append(lse)
    out = torch.empty_like(full, dtype=torch.bfloat16, device="cuda")
    mla.mla_combine(c.cfg, torch.stack(parts), torch.stack(lses), c.d["w_uv"], None, out)
    new_rows = Hs.oracle_new_rows(c)
    W_UK, _ = O.split_wkv_b(c.weights.wkv_b, w.H, w.d_nope, w.d_v)
    for b in range(w.B):
        rows = Hs.oracle_rows_of(c, b, new_rows)
        o_ref, _ = O.latent_partial(c.q[b], rows, W_UK, w.scale, w.rope_theta, 0, int(cut[b]),
                                    heads=[0, 127])
        got = parts[0].float().cpu().view(w.B, w.Tq, w.H, w.d_c)[b][:, [0, 127]]
        Hs.assert_parity(got, o_ref, "bf16", f"fp8 partial b={b}")
        ref = Hs.oracle_out(c, b, [0, 64, 127], new_rows)
        Hs.assert_parity(out.float().cpu()[b][:, [0, 64, 127]], ref, "bf16", f"fp8 merged b={b}")


def test_fp8_subnormal_codes_keep_their_values():
    """History rows made only of subnormal codes (±m·2^-9, m = 1..7): decoding just those keys
    (a key range that leaves out the appended token) must see their exact values, in the score
    and in the value product; a conversion that flushed them would return zeros."""
    w = W.small_variant(V2, B=2)
    c = Hs.make_case(w, _lens(300, 129))
    g = torch.Generator().manual_seed(5)
    shape = (c.pt.num_pages, W.PAGE_SIZE, w.row)
    sub = torch.randint(1, 8, shape, generator=g, dtype=torch.uint8)
    sub |= torch.randint(0, 2, shape, generator=g, dtype=torch.uint8) << 7
    for cache in (c.cache_host, c.d["cache"]):
        codes, scales = Hs.fp8_views(w, cache)
        codes.copy_(sub.to(cache.device))
        scales.fill_(64.0)   # row values m/8: far above the parity bound's absolute term
    Hs.run_append(c)
    rows_n = w.B * w.Tq * w.H
    o = torch.empty((rows_n, w.d_c), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(rows_n, dtype=torch.float32, device="cuda")
    ws = mla.workspace(mla.mla_decode_workspace_size(c.cfg, w.B, w.Tq))
    kb = torch.zeros(w.B, dtype=torch.int32)
    ke = c.lens - 1
    mla.mla_decode_partial(c.cfg, c.d["q"], c.d["cache"], c.d["block_table"], c.d["seq_lens"],
                           kb.cuda(), ke.cuda(), c.d["w_uk_t"], ws, o, lse)
    got = o.float().cpu().view(w.B, w.Tq, w.H, w.d_c)
    new_rows = Hs.oracle_new_rows(c)
    W_UK, _ = O.split_wkv_b(c.weights.wkv_b, w.H, w.d_nope, w.d_v)
    for b in range(w.B):
        rows = Hs.oracle_rows_of(c, b, new_rows)
        o_ref, _ = O.latent_partial(c.q[b], rows, W_UK, w.scale, w.rope_theta, 0, int(ke[b]),
                                    heads=[0, 64, 127])
        assert np.max(np.abs(o_ref)) > 0
        Hs.assert_parity(got[b][:, [0, 64, 127]], o_ref, "bf16", f"subnormal codes b={b}")
