"""The allocation-free decode entry point, through the C ABI, against mla_decode.

mla_decode_noalloc serves callers that cannot allocate device memory themselves (a serving
runtime that owns the whole device memory pool, code that runs where cudaMalloc is not
allowed): its scratch is a fixed device array inside the library instead of a caller-given
workspace. The array is shared by every call and keeps the previous call's contents, so the
check runs two calls in a row (with a different-sized call in between) and compares each with
mla_decode on the same inputs. Both run the same deterministic kernels on the same plan, so the
outputs must be bit-identical; the first call is also compared with the fp64 oracle within the
bf16 parity bound the other tests use. This file is collected last so that a run stopping at
the first failure has already run everything else.
"""

import pytest
import torch

import harness as Hs
import head_latent_attention_05_b200 as mla
import workloads as W

pytestmark = pytest.mark.gpu

V2 = W.WORKLOADS["v2_bf16_b16_ctx4096"]


def _noalloc(c):
    w = c.w
    out = torch.full((w.B, w.Tq, w.H, w.d_v), float("nan"), dtype=w.torch_dtype, device="cuda")
    mla.mla_decode_noalloc(c.cfg, c.d["q"], c.d["cache"], c.d["block_table"], c.d["seq_lens"],
                           c.d["w_uk_t"], c.d["w_uv"], out)
    assert mla.mla_get_device_error() == 0
    return out.float().cpu()


def test_noalloc_decode_matches_decode_on_consecutive_calls():
    mla.mla_get_device_error()
    big = Hs.make_case(W.small_variant(V2, B=4), torch.tensor([4096, 130, 1, 777], dtype=torch.int32))
    small = Hs.make_case(W.small_variant(V2, B=2, seed=7), torch.tensor([65, 300], dtype=torch.int32))
    Hs.run_append(big)
    Hs.run_append(small)
    ref_big = Hs.run_decode(big).float().cpu()
    ref_small = Hs.run_decode(small).float().cpu()
    new_rows = Hs.oracle_new_rows(big)
    for i in range(2):
        got_big = _noalloc(big)
        assert torch.equal(got_big, ref_big), "noalloc differs from mla_decode (4 sequences)"
        got_small = _noalloc(small)
        assert torch.equal(got_small, ref_small), "noalloc differs from mla_decode (2 sequences)"
        if i == 0:
            for b in range(big.w.B):
                heads = [0, 63, 127]
                Hs.assert_parity(got_big[b][:, heads], Hs.oracle_out(big, b, heads, new_rows),
                                 "bf16", f"noalloc vs oracle b={b}")


def test_noalloc_rejects_a_batch_beyond_its_scratch():
    cfg = Hs.config_of(V2)
    big = 64   # the smallest power-of-two batch whose scratch exceeds the built-in array
    while mla.mla_decode_workspace_size(cfg, big, 1) <= mla.MLA_DECODE_NOALLOC_MAX_SCRATCH:
        big *= 2
    c = Hs.make_case(W.small_variant(V2, B=2), torch.tensor([64, 64], dtype=torch.int32))
    q = torch.zeros((big, 1, V2.H, V2.d_nope + V2.d_r), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((big, 1, V2.H, V2.d_v), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(mla.MlaError) as e:
        mla.mla_decode_noalloc(cfg, q, c.d["cache"], c.d["block_table"], c.d["seq_lens"],
                               c.d["w_uk_t"], c.d["w_uv"], out)
    assert e.value.code == 3   # MLA_ERR_WORKSPACE_TOO_SMALL, nothing launched


def test_noalloc_decode_over_a_quantised_cache():
    """The same built-in scratch serves a decode over an FP8 E4M3 cache (it then also holds the
    split query rows): bit-identical to mla_decode on two calls in a row."""
    mla.mla_get_device_error()
    w = W.small_variant(V2, B=3, kv="fp8")
    c = Hs.make_case(w, torch.tensor([1500, 64, 321], dtype=torch.int32))
    Hs.run_append(c)
    ref = Hs.run_decode(c).float().cpu()
    for _ in range(2):
        assert torch.equal(_noalloc(c), ref), "noalloc differs from mla_decode (quantised cache)"
