"""The whole decode layer on the GPU through the C ABI, against the fp64 oracle.

mla_query (wq_a -> q_norm -> wq_b), mla_append_latent, mla_decode and mla_output (wo), chained
as the page's module runs them (「论文复现工坊 No.4 从零复现 DeepSeek-V2/V3 多头潜在注意力 MLA」 §2),
against oracle.query_from_x, oracle.output_projection and oracle.decode_layer on the same seeded
inputs. Tolerances: fp32 max|err| <= 1e-4 max|ref|; bf16 max|err| <= 1e-2 max|ref| + 1e-3.
"""

import numpy as np
import pytest
import torch

import harness as Hs
import head_latent_attention_05_b200 as mla
import workloads as W
from oracle import mla_oracle as O

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


def _query(c, x):
    w = c.w
    d = c.d
    for k, v in (("w_qa", c.weights.w_qa), ("q_gain", c.weights.q_gain), ("w_qb", c.weights.w_qb)):
        if k not in d:
            d[k] = v.to("cuda")
    q = torch.empty((x.shape[0], w.H, w.d_nope + w.d_r), dtype=w.torch_dtype, device="cuda")
    ws = mla.workspace(mla.mla_query_workspace_size(c.cfg, w.q_lora, x.shape[0]))
    mla.mla_query(c.cfg, x, d["w_qa"], d["q_gain"], d["w_qb"], ws, q)
    return q


def _output(c, attn, w_o):
    w = c.w
    y = torch.empty((attn.shape[0], w.d_model), dtype=w.torch_dtype, device="cuda")
    ws = mla.workspace(mla.mla_output_workspace_size(c.cfg, attn.shape[0]))
    mla.mla_output(c.cfg, attn.contiguous(), w_o, ws, y)
    return y


CASES = [
    (TINY, _lens(128)),
    (W.small_variant(V2, B=3), _lens(1, 130, 700)),
    (W.small_variant(H32, B=5), _lens(70, 512, 64, 1100, 3)),
    (W.small_variant(MIX, B=4), _lens(1024, 1500, 65, 2049)),
    (W.small_variant(LONG, B=2), _lens(2, 777)),
]
IDS = ["tiny_f32", "v2_b3", "h32_b5", "mix_b4", "tq2_b2"]


@pytest.mark.parametrize("w,lens", CASES, ids=IDS)
def test_query_path_parity(w, lens):
    c = Hs.make_case(w, lens)
    got = _query(c, c.d["x_new"]).float().cpu()
    ref = O.query_from_x(c.x_new, c.weights.w_qa, c.weights.q_gain, c.weights.w_qb, w.H,
                         w.d_nope, w.d_r, w.rms_eps)
    Hs.assert_parity(got, ref, w.dtype, "q path")


@pytest.mark.parametrize("w,n_tok", [(TINY, 3), (V2, 1), (V2, 16), (H32, 37), (MIX, 64),
                                     (V2, 300)], ids=["tiny", "v2_1", "v2_16", "h32_37",
                                                      "mix_64", "v2_300"])
def test_output_projection_parity(w, n_tok):
    w_o = W.output_weight(w)
    attn = W.randn((n_tok, w.H, w.d_v), 77, 1, 1.0, w.torch_dtype)
    cfg = Hs.config_of(w)
    y = torch.empty((n_tok, w.d_model), dtype=w.torch_dtype, device="cuda")
    ws = mla.workspace(mla.mla_output_workspace_size(cfg, n_tok))
    mla.mla_output(cfg, attn.to("cuda"), w_o.to("cuda"), ws, y)
    Hs.assert_parity(y.float().cpu(), O.output_projection(attn, w_o), w.dtype, "wo")


@pytest.mark.parametrize("w,lens", CASES, ids=IDS)
def test_decode_layer_parity(w, lens):
    """x of the new tokens -> q path, append, decode, wo; against oracle.decode_layer."""
    c = Hs.make_case(w, lens)
    q = _query(c, c.d["x_new"])
    c.d["q"] = q.view(w.B, w.Tq, w.H, w.d_nope + w.d_r).contiguous()
    Hs.run_append(c)
    attn = Hs.run_decode(c)
    w_o = W.output_weight(w)
    y = _output(c, attn.view(w.B * w.Tq, w.H, w.d_v), w_o.to("cuda")).float().cpu()
    for b in range(w.B):
        L = int(c.lens[b])
        hist = O.gather_rows(c.cache_host, c.pt.block_table[b].numpy(), L - w.Tq, W.PAGE_SIZE)
        x_b = c.x_new[b * w.Tq:(b + 1) * w.Tq]
        ref = O.decode_layer(x_b, hist, c.weights.w_dkv, c.weights.kv_gain, c.weights.wkv_b,
                             c.weights.w_qa, c.weights.q_gain, c.weights.w_qb, w_o, w.H, w.d_c,
                             w.d_r, w.d_nope, w.d_v, w.rms_eps, w.rope_theta)
        Hs.assert_parity(y[b * w.Tq:(b + 1) * w.Tq], ref, w.dtype, f"layer b={b} L={L}")


def test_decode_layer_full_size_v2_sampled():
    """Batch 16 x 4096 at DeepSeek-V2 shape, the whole layer; three sequences checked."""
    w = V2
    c = Hs.make_case(w)
    q = _query(c, c.d["x_new"])
    c.d["q"] = q.view(w.B, w.Tq, w.H, w.d_nope + w.d_r).contiguous()
    Hs.run_append(c)
    attn = Hs.run_decode(c)
    w_o = W.output_weight(w)
    y = _output(c, attn.view(w.B, w.H, w.d_v), w_o.to("cuda")).float().cpu()
    for b in (0, 7, 15):
        hist = O.gather_rows(c.cache_host, c.pt.block_table[b].numpy(), int(c.lens[b]) - 1)
        ref = O.decode_layer(c.x_new[b:b + 1], hist, c.weights.w_dkv, c.weights.kv_gain,
                             c.weights.wkv_b, c.weights.w_qa, c.weights.q_gain, c.weights.w_qb,
                             w_o, w.H, w.d_c, w.d_r, w.d_nope, w.d_v, w.rms_eps, w.rope_theta)
        Hs.assert_parity(y[b:b + 1], ref, w.dtype, f"layer b={b}")
