"""Tensor-core prefill (mla_prefill) on the GPU through the C ABI, against the fp64 oracle and
against the CUDA-core reference prefill (mla_prefill_ref).

Every new token sees the keys up to its own position (causal among the new tokens), with an
optional sliding window. Tolerances: bf16 max|err| <= 1e-2 max|ref| + 1e-3.
"""

import numpy as np
import pytest
import torch

import harness as Hs
import head_latent_attention_05_b200 as mla
import workloads as W

pytestmark = pytest.mark.gpu

V2 = W.WORKLOADS["v2_bf16_b16_ctx4096"]
H32 = W.WORKLOADS["h32_bf16_b32_ctx512to8192_shuffled"]
TINY = W.WORKLOADS["tiny_f32_b1_h4_ctx128"]


@pytest.fixture(autouse=True)
def _no_device_error():
    mla.mla_get_device_error()
    yield
    assert mla.mla_get_device_error() == 0


def _lens(*ls):
    return torch.tensor(ls, dtype=torch.int32)


def _prefill(c, fn, ws_fn):
    w = c.w
    out = torch.empty((w.B, w.Tq, w.H, w.d_v), dtype=w.torch_dtype, device="cuda")
    x = c.d["x_new"].view(w.B, w.Tq, w.d_model)
    ws = mla.workspace(ws_fn(c.cfg, w.B, w.Tq))
    fn(c.cfg, x, c.d["q"], c.d["w_dkv"], c.d["kv_gain"], c.d["w_uk_t"], c.d["w_uv"],
       c.d["seq_lens"], c.d["block_table"], c.d["cache"], ws, out)
    return out


@pytest.mark.parametrize("w,lens,t_new,window", [
    (V2, _lens(700, 200), 128, 0),
    (V2, _lens(256, 300), 256, 0),           # whole prompts, and one with a prefix
    (V2, _lens(1000, 130), 65, 300),         # with a sliding window
    (H32, _lens(900, 77, 40), 37, 0),        # 32 heads: four tokens per 128-row unit
], ids=["v2_t128", "v2_prompt256", "v2_window", "h32_t37"])
def test_prefill_tensor_core_parity(w, lens, t_new, window):
    w = W.small_variant(w, B=len(lens), Tq=t_new)
    c = Hs.make_case(w, lens, window=window)
    cache0 = c.d["cache"].clone()
    out = _prefill(c, mla.mla_prefill, mla.mla_prefill_workspace_size).float().cpu()
    new_rows = Hs.oracle_new_rows(c)
    heads = [0, w.H // 2, w.H - 1]
    for b in range(w.B):
        Hs.assert_parity(out[b][:, heads], Hs.oracle_out(c, b, heads, new_rows), w.dtype,
                         f"prefill b={b}")
    # the CUDA-core reference prefill on the same inputs agrees within the same bound
    c.d["cache"].copy_(cache0)
    ref = _prefill(c, mla.mla_prefill_ref, mla.mla_prefill_ref_workspace_size).float().cpu()
    for b in range(w.B):
        Hs.assert_parity(out[b], ref[b].numpy().astype(np.float64), w.dtype, f"vs ref b={b}")


def test_prefill_fp32_takes_the_cuda_core_path():
    w = W.small_variant(TINY, B=2, Tq=9)
    c = Hs.make_case(w, _lens(40, 9))
    out = _prefill(c, mla.mla_prefill, mla.mla_prefill_workspace_size).cpu()
    new_rows = Hs.oracle_new_rows(c)
    for b in range(2):
        Hs.assert_parity(out[b], Hs.oracle_out(c, b, list(range(w.H)), new_rows), "f32",
                         f"b={b}")
