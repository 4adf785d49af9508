"""Pins for the fp64 oracle: checks against things other than the oracle itself.

* brute force: scalar nested loops over the page's module on tiny sizes, with RoPE written as
  complex multiplication;
* a library routine: torch fp64 (F.linear, F.rms_norm, complex RoPE via torch.polar and
  F.scaled_dot_product_attention with its default 1/sqrt(E) scale) on materialised keys/values;
* the absorption identity (expanded == absorbed);
* closed forms and invariants (one token, zero query, constant cache, RoPE properties,
  softmax sums, causality);
* the cache-size numbers printed on the pages (tests/golden/cache_sizes.json).
"""

import cmath
import json
import math
import os
import random

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import mla_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_module(rng, d_model, H, d_c, d_r, d_nope, d_v, q_lora):
    n = rng.standard_normal
    return dict(
        w_dkv=n((d_c + d_r, d_model)) / math.sqrt(d_model),
        kv_gain=1.0 + 0.1 * n(d_c),
        wkv_b=n((H * (d_nope + d_v), d_c)) / math.sqrt(d_c),
        w_qa=n((q_lora, d_model)) / math.sqrt(d_model),
        q_gain=1.0 + 0.1 * n(q_lora),
        w_qb=n((H * (d_nope + d_r), q_lora)) / math.sqrt(q_lora),
    )


# ----------------------------------------------------------------------------- brute force

def _brute_module(x, W, H, d_c, d_r, d_nope, d_v, eps, theta):
    """Scalar loops over the module of the page's §2 (lists of floats, cmath for RoPE)."""
    L, d_model = len(x), len(x[0])

    def linear(vec, w):  # w is [out][in]
        return [sum(w[o][i] * vec[i] for i in range(len(vec))) for o in range(len(w))]

    def rmsn(vec, g):
        ms = sum(v * v for v in vec) / len(vec)
        return [vec[i] / math.sqrt(ms + eps) * g[i] for i in range(len(vec))]

    def rot(vec, p):  # treat (v0 + i v1), (v2 + i v3), ... as complex numbers
        out = []
        d = len(vec)
        for i in range(d // 2):
            z = complex(vec[2 * i], vec[2 * i + 1]) * cmath.exp(1j * p * theta ** (-2.0 * i / d))
            out += [z.real, z.imag]
        return out

    w_dkv, wkv_b = W["w_dkv"].tolist(), W["wkv_b"].tolist()
    w_qa, w_qb = W["w_qa"].tolist(), W["w_qb"].tolist()
    kv_gain, q_gain = W["kv_gain"].tolist(), W["q_gain"].tolist()
    keys, vals, queries = [], [], []
    for t in range(L):
        kv = linear(x[t], w_dkv)
        c = rmsn(kv[:d_c], kv_gain)
        kr = rot(kv[d_c:], t)
        up = linear(c, wkv_b)  # [H * (d_nope + d_v)]
        qv = linear(rmsn(linear(x[t], w_qa), q_gain), w_qb)
        kh, vh, qh = [], [], []
        for h in range(H):
            blk = up[h * (d_nope + d_v):(h + 1) * (d_nope + d_v)]
            kh.append(blk[:d_nope] + kr)
            vh.append(blk[d_nope:])
            qb = qv[h * (d_nope + d_r):(h + 1) * (d_nope + d_r)]
            qh.append(qb[:d_nope] + rot(qb[d_nope:], t))
        keys.append(kh), vals.append(vh), queries.append(qh)
    scale = 1.0 / math.sqrt(d_nope + d_r)
    out = [[[0.0] * d_v for _ in range(H)] for _ in range(L)]
    for t in range(L):
        for h in range(H):
            s = [scale * sum(a * b for a, b in zip(queries[t][h], keys[j][h])) for j in range(t + 1)]
            m = max(s)
            e = [math.exp(v - m) for v in s]
            z = sum(e)
            for j in range(t + 1):
                for k in range(d_v):
                    out[t][h][k] += e[j] / z * vals[j][h][k]
    return np.array(out)


def test_brute_force_tiny_module():
    rng = np.random.default_rng(1)
    dims = dict(H=2, d_c=6, d_r=4, d_nope=3, d_v=2)
    d_model, q_lora, L, eps, theta = 7, 5, 6, 1e-6, 10000.0
    W = _rand_module(rng, d_model, q_lora=q_lora, **dims)
    x = rng.standard_normal((L, d_model))
    ref = _brute_module(x.tolist(), W, eps=eps, theta=theta, **dims)
    got = O.module_attention(x, W["w_dkv"], W["kv_gain"], W["wkv_b"], W["w_qa"], W["q_gain"],
                             W["w_qb"], eps=eps, theta=theta, **dims)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-13)


def test_brute_force_decode_two_new_tokens():
    """decode_expanded for the 2 newest tokens equals the brute-force prefill's last 2 rows."""
    rng = np.random.default_rng(2)
    dims = dict(H=3, d_c=8, d_r=4, d_nope=4, d_v=3)
    d_model, q_lora, L, eps, theta = 6, 4, 7, 1e-6, 500.0
    W = _rand_module(rng, d_model, q_lora=q_lora, **dims)
    x = rng.standard_normal((L, d_model))
    ref = _brute_module(x.tolist(), W, eps=eps, theta=theta, **dims)
    rows = O.latent_rows(x, W["w_dkv"], W["kv_gain"], np.arange(L), dims["d_c"], eps, theta)
    q = O.query_from_x(x[-2:], W["w_qa"], W["q_gain"], W["w_qb"], dims["H"], dims["d_nope"],
                       dims["d_r"], eps)
    W_UK, W_UV = O.split_wkv_b(W["wkv_b"], dims["H"], dims["d_nope"], dims["d_v"])
    got = O.decode_expanded(q, rows, W_UK, W_UV, 1 / math.sqrt(dims["d_nope"] + dims["d_r"]), theta)
    np.testing.assert_allclose(got, ref[-2:], rtol=1e-12, atol=1e-13)


# -------------------------------------------------------------------------- library routine

def _torch_module(x, W, H, d_c, d_r, d_nope, d_v, eps, theta):
    """The page's module with torch fp64 library calls: F.linear, F.rms_norm, complex RoPE
    (freqs_cis = polar(1, pos·θ)), materialised K/V, and SDPA with its default scale."""
    t = lambda a: torch.as_tensor(a, dtype=torch.float64)
    x = t(x)
    L = x.shape[0]
    freqs = 1.0 / theta ** (torch.arange(0, d_r, 2, dtype=torch.float64) / d_r)
    cis = torch.polar(torch.ones(L, d_r // 2, dtype=torch.float64),
                      torch.outer(torch.arange(L, dtype=torch.float64), freqs))

    def apply_rope(v):  # v [L, ..., d_r]
        vc = torch.view_as_complex(v.reshape(*v.shape[:-1], d_r // 2, 2).contiguous())
        shape = (L,) + (1,) * (vc.dim() - 2) + (d_r // 2,)
        return torch.view_as_real(vc * cis.reshape(shape)).flatten(-2)

    qa = F.rms_norm(F.linear(x, t(W["w_qa"])), (t(W["q_gain"]).numel(),), t(W["q_gain"]), eps)
    q = F.linear(qa, t(W["w_qb"])).view(L, H, d_nope + d_r)
    q_nope, q_rope = torch.split(q, [d_nope, d_r], dim=-1)
    kv = F.linear(x, t(W["w_dkv"]))
    c, k_rope = torch.split(kv, [d_c, d_r], dim=-1)
    c = F.rms_norm(c, (d_c,), t(W["kv_gain"]), eps)
    up = F.linear(c, t(W["wkv_b"])).view(L, H, d_nope + d_v)
    k_nope, v = torch.split(up, [d_nope, d_v], dim=-1)
    q_full = torch.cat([q_nope, apply_rope(q_rope)], -1).transpose(0, 1)          # [H, L, E]
    k_full = torch.cat([k_nope, apply_rope(k_rope)[:, None, :].expand(L, H, d_r)], -1).transpose(0, 1)
    o = F.scaled_dot_product_attention(q_full, k_full, v.transpose(0, 1), is_causal=True)
    return o.transpose(0, 1).numpy()                                              # [L, H, d_v]


@pytest.mark.parametrize("dims", [
    dict(H=4, d_c=64, d_r=16, d_nope=32, d_v=32, d_model=128, q_lora=48, L=40),
    dict(H=3, d_c=24, d_r=8, d_nope=16, d_v=12, d_model=20, q_lora=10, L=70),
])
def test_module_matches_torch_sdpa(dims):
    dims = dict(dims)
    L, d_model, q_lora = dims.pop("L"), dims.pop("d_model"), dims.pop("q_lora")
    rng = np.random.default_rng(3)
    W = _rand_module(rng, d_model, q_lora=q_lora, **dims)
    x = rng.standard_normal((L, d_model))
    ref = _torch_module(x, W, eps=1e-6, theta=10000.0, **dims)
    got = O.module_attention(x, W["w_dkv"], W["kv_gain"], W["wkv_b"], W["w_qa"], W["q_gain"],
                             W["w_qb"], eps=1e-6, theta=10000.0, **dims)
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-12)


def test_rms_norm_matches_torch():
    rng = np.random.default_rng(4)
    v, g = rng.standard_normal((5, 33)), rng.standard_normal(33)
    ref = F.rms_norm(torch.tensor(v), (33,), torch.tensor(g), 1e-6).numpy()
    np.testing.assert_allclose(O.rms_norm(v, g, 1e-6), ref, rtol=1e-13)


# ----------------------------------------------------------------------- absorption identity

@pytest.mark.parametrize("Tq", [1, 2, 3])
def test_absorbed_equals_expanded(Tq):
    rng = np.random.default_rng(5 + Tq)
    H, d_c, d_r, d_nope, d_v, L = 5, 48, 16, 24, 20, 97
    q = rng.standard_normal((Tq, H, d_nope + d_r))
    rows = rng.standard_normal((L, d_c + d_r))
    W_UK = rng.standard_normal((H, d_nope, d_c)) / math.sqrt(d_c)
    W_UV = rng.standard_normal((H, d_v, d_c)) / math.sqrt(d_c)
    a = O.decode_expanded(q, rows, W_UK, W_UV, 0.2, 10000.0)
    b = O.decode_absorbed(q, rows, W_UK, W_UV, 0.2, 10000.0)
    assert np.max(np.abs(a - b)) <= 1e-12 * np.max(np.abs(a))


# ------------------------------------------------------------------------------ closed forms

def _rand_decode(rng, H=3, d_c=16, d_r=8, d_nope=8, d_v=6, L=20, Tq=1):
    return (rng.standard_normal((Tq, H, d_nope + d_r)), rng.standard_normal((L, d_c + d_r)),
            rng.standard_normal((H, d_nope, d_c)), rng.standard_normal((H, d_v, d_c)))


def test_single_token_returns_its_value():
    rng = np.random.default_rng(6)
    q, rows, W_UK, W_UV = _rand_decode(rng, L=1)
    out = O.decode_expanded(q, rows, W_UK, W_UV, 0.3, 10000.0)
    expect = np.einsum("d,hvd->hv", rows[0, :16], W_UV)
    np.testing.assert_allclose(out[0], expect, rtol=1e-13, atol=1e-13)


def test_zero_query_gives_mean_value():
    rng = np.random.default_rng(7)
    q, rows, W_UK, W_UV = _rand_decode(rng, L=33, Tq=2)
    q[:] = 0.0
    out = O.decode_expanded(q, rows, W_UK, W_UV, 0.3, 10000.0)
    for t, p in enumerate([31, 32]):  # query t sees keys 0..p
        expect = np.einsum("d,hvd->hv", rows[:p + 1, :16].mean(0), W_UV)
        np.testing.assert_allclose(out[t], expect, rtol=1e-12, atol=1e-13)


def test_constant_cache_returns_that_value():
    rng = np.random.default_rng(8)
    q, rows, W_UK, W_UV = _rand_decode(rng, L=50)
    rows[:] = rows[0]
    # k_R rows are identical, so scores are equal for every key and P is uniform
    out = O.decode_expanded(q, rows, W_UK, W_UV, 0.3, 10000.0)
    np.testing.assert_allclose(out[0], np.einsum("d,hvd->hv", rows[0, :16], W_UV), rtol=1e-12)


def test_softmax_rows_sum_to_one_and_are_causal():
    rng = np.random.default_rng(9)
    q, rows, W_UK, W_UV = _rand_decode(rng, L=40, Tq=3)
    _, P = O.decode_expanded(q, rows, W_UK, W_UV, 0.3, 10000.0, return_probs=True)
    np.testing.assert_allclose(P.sum(-1), 1.0, rtol=1e-14)
    for t in range(3):
        assert np.all(P[t, :, 38 + t:] == 0.0)
        assert np.all(P[t, :, :38 + t] > 0.0)


def test_future_rows_do_not_change_earlier_queries():
    rng = np.random.default_rng(10)
    q, rows, W_UK, W_UV = _rand_decode(rng, L=30, Tq=2)
    a = O.decode_expanded(q, rows, W_UK, W_UV, 0.3, 10000.0)
    rows2 = rows.copy()
    rows2[29] += 5.0  # only the last query (position 29) may see it
    b = O.decode_expanded(q, rows2, W_UK, W_UV, 0.3, 10000.0)
    np.testing.assert_array_equal(a[0], b[0])
    assert np.max(np.abs(a[1] - b[1])) > 1e-3


def test_rope_identity_norm_and_relative_position():
    rng = np.random.default_rng(11)
    a, b = rng.standard_normal(64), rng.standard_normal(64)
    np.testing.assert_array_equal(O.rope(a, 0, 10000.0), a)
    for p in [1, 77, 4095, 131071]:
        np.testing.assert_allclose(np.linalg.norm(O.rope(a, p, 10000.0)), np.linalg.norm(a),
                                   rtol=1e-13)
    for m, n in [(5, 3), (1000, 17), (131071, 65536)]:
        lhs = O.rope(a, m, 10000.0) @ O.rope(b, n, 10000.0)
        rhs = O.rope(a, m - n, 10000.0) @ b
        assert abs(lhs - rhs) <= 1e-9 * (np.linalg.norm(a) * np.linalg.norm(b))


def test_rope_first_pair_turns_by_position():
    """θ_0 = 1: the first pair turns by exactly `pos` radians; the last pair by pos·θ^(-(d-2)/d)."""
    d, p = 16, 3
    v = np.zeros(d)
    v[0] = 1.0
    r = O.rope(v, p, 10000.0)
    np.testing.assert_allclose(r[:2], [math.cos(p), math.sin(p)], rtol=1e-15)
    v = np.zeros(d)
    v[d - 2] = 1.0
    r = O.rope(v, p, 10000.0)
    ang = p * 10000.0 ** (-(d - 2) / d)
    np.testing.assert_allclose(r[d - 2:], [math.cos(ang), math.sin(ang)], rtol=1e-14)


def test_rms_norm_unit_rms():
    rng = np.random.default_rng(12)
    v = rng.standard_normal((7, 512)) * 3.0
    y = O.rms_norm(v, np.ones(512), 0.0)
    np.testing.assert_allclose(np.sqrt((y * y).mean(-1)), 1.0, rtol=1e-14)


def test_gather_rows_follows_block_table():
    cache = np.arange(5 * 4 * 2, dtype=np.float64).reshape(5, 4, 2)
    rows = O.gather_rows(cache, [3, 0, 4], 10, page_size=4)
    expect = np.concatenate([cache[3], cache[0], cache[4][:2]])
    np.testing.assert_array_equal(rows, expect)


# ------------------------------------------------------------------------ printed numbers

def _close(a, b, tol):
    return abs(a - b) <= tol * abs(b)


def test_cache_sizes_page1_table():
    g = json.load(open(os.path.join(GOLDEN, "cache_sizes.json")))["page1_table"]
    mha = O.mha_cache_elems_per_token(g["n_heads"], g["d_h"])
    gqa = O.gqa_cache_elems_per_token(8, g["d_h"])
    mla = O.mla_cache_elems_per_token(512, 64)
    assert (mha, gqa, mla) == (g["mha_elems"], g["gqa8_elems"], g["mla_elems"])
    mib = lambda e: e * g["bytes_per_elem"] * g["context"] / 2 ** 20
    assert (mib(mha), mib(gqa)) == (g["mha_MiB"], g["gqa8_MiB"])
    assert round(mib(mla)) == g["mla_MiB"]
    assert round(mha / gqa, 2) == g["gqa8_ratio"]
    assert round(mha / mla, 2) == g["mla_ratio"]
    assert round(100 * (1 - mla / mha), 1) == g["mla_saving_percent"]


def test_cache_sizes_page4_v2():
    g = json.load(open(os.path.join(GOLDEN, "cache_sizes.json")))["page4_v2"]
    tol = g["rel_tol"]
    mha = O.mha_cache_elems_per_token(g["n_heads"], g["d_h"])
    mla = O.mla_cache_elems_per_token(g["d_c"], g["d_r"])
    assert mha == g["mha_elems_per_layer"] and mla == g["mla_elems_per_layer"]
    assert g["d_c"] == 4 * g["d_h"] and g["d_r"] == g["d_h"] // 2
    per_tok = mha * g["layers"]
    assert _close(per_tok, g["mha_elems_all_layers_approx"], tol)
    assert _close(per_tok * g["bytes_per_elem"], g["mha_bytes_per_token_approx"], tol)
    assert _close(per_tok * g["bytes_per_elem"] * g["context"], g["mha_bytes_32k_approx"], tol)
    assert round(mha / mla) == g["mla_ratio_approx"]
    assert _close(mla * g["layers"] * g["bytes_per_elem"] * g["context"],
                  g["mla_bytes_32k_approx"], tol)
    assert round(O.mha_cache_elems_per_token(64, g["d_h"]) / mla, 1) == g["ratio_at_64_heads"]


def test_cache_sizes_page4_gqa():
    g = json.load(open(os.path.join(GOLDEN, "cache_sizes.json")))
    v2, q = g["page4_v2"], g["page4_gqa"]
    e = O.gqa_cache_elems_per_token(v2["n_heads"] // q["r"], v2["d_h"])
    assert e == q["elems_per_layer_approx"]
    assert round(e / O.mla_cache_elems_per_token(512, 64)) == q["times_mla_approx"]
    gib = e * v2["layers"] * v2["bytes_per_elem"] * v2["context"] / 2 ** 30
    assert _close(gib, q["GiB_32k_approx"], q["rel_tol"])


# --------------------------------------------------------------- output projection and layer

def _brute_wo(out, w_o):
    """Scalar loops: y[t][m] = sum over heads h and value dims k of w_o[m][h*d_v + k] out[t][h][k]."""
    L, H, d_v = len(out), len(out[0]), len(out[0][0])
    return np.array([[sum(w_o[m][h * d_v + k] * out[t][h][k] for h in range(H) for k in range(d_v))
                      for m in range(len(w_o))] for t in range(L)])


def test_output_projection_brute_force():
    rng = np.random.default_rng(20)
    dims = dict(H=3, d_c=6, d_r=4, d_nope=3, d_v=2)
    d_model, q_lora, L, eps, theta = 5, 4, 6, 1e-6, 10000.0
    W = _rand_module(rng, d_model, q_lora=q_lora, **dims)
    w_o = rng.standard_normal((d_model, dims["H"] * dims["d_v"]))
    x = rng.standard_normal((L, d_model))
    attn = _brute_module(x.tolist(), W, eps=eps, theta=theta, **dims)
    ref = _brute_wo(attn.tolist(), w_o.tolist())
    got = O.output_projection(O.module_attention(x, W["w_dkv"], W["kv_gain"], W["wkv_b"],
                                                 W["w_qa"], W["q_gain"], W["w_qb"], eps=eps,
                                                 theta=theta, **dims), w_o)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-13)


def test_output_projection_flattens_head_after_head():
    """Identity wo returns the heads laid side by side; a one-hot row picks (head 1, dim 0)."""
    rng = np.random.default_rng(21)
    out = rng.standard_normal((2, 3, 4))                      # [Tq, H, d_v]
    np.testing.assert_array_equal(O.output_projection(out, np.eye(12)), out.reshape(2, 12))
    w_o = np.zeros((1, 12))
    w_o[0, 1 * 4 + 0] = 1.0
    np.testing.assert_array_equal(O.output_projection(out, w_o)[:, 0], out[:, 1, 0])


def test_output_projection_matches_torch_linear_on_the_module():
    rng = np.random.default_rng(22)
    dims = dict(H=4, d_c=32, d_r=8, d_nope=16, d_v=12)
    d_model, q_lora, L = 24, 16, 30
    W = _rand_module(rng, d_model, q_lora=q_lora, **dims)
    w_o = rng.standard_normal((d_model, dims["H"] * dims["d_v"])) / math.sqrt(48)
    x = rng.standard_normal((L, d_model))
    o = torch.as_tensor(_torch_module(x, W, eps=1e-6, theta=10000.0, **dims))
    ref = F.linear(o.reshape(L, -1), torch.as_tensor(w_o)).numpy()
    got = O.output_projection(O.module_attention(x, W["w_dkv"], W["kv_gain"], W["wkv_b"],
                                                 W["w_qa"], W["q_gain"], W["w_qb"], eps=1e-6,
                                                 theta=10000.0, **dims), w_o)
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("Tq", [1, 3])
def test_decode_layer_equals_brute_force_prefill_tail(Tq):
    """The whole decode layer for the Tq newest tokens (q path, append at their positions,
    attention, wo) equals the last Tq rows of the brute-force module over the whole sequence."""
    rng = np.random.default_rng(23 + Tq)
    dims = dict(H=2, d_c=6, d_r=4, d_nope=3, d_v=2)
    d_model, q_lora, L, eps, theta = 5, 4, 7, 1e-6, 300.0
    W = _rand_module(rng, d_model, q_lora=q_lora, **dims)
    w_o = rng.standard_normal((d_model, dims["H"] * dims["d_v"]))
    x = rng.standard_normal((L, d_model))
    ref = _brute_wo(_brute_module(x.tolist(), W, eps=eps, theta=theta, **dims).tolist(),
                    w_o.tolist())[-Tq:]
    hist = O.latent_rows(x[:L - Tq], W["w_dkv"], W["kv_gain"], np.arange(L - Tq), dims["d_c"],
                         eps, theta)
    got = O.decode_layer(x[L - Tq:], hist, W["w_dkv"], W["kv_gain"], W["wkv_b"], W["w_qa"],
                         W["q_gain"], W["w_qb"], w_o, eps=eps, theta=theta, **dims)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-13)


def test_query_path_brute_force():
    """q = wq_b(q_norm(wq_a(x))) per head, by scalar loops, against query_from_x."""
    rng = np.random.default_rng(25)
    H, d_nope, d_r, d_model, q_lora, eps = 2, 3, 4, 6, 5, 1e-6
    W = _rand_module(rng, d_model, H=H, d_c=4, d_r=d_r, d_nope=d_nope, d_v=2, q_lora=q_lora)
    x = rng.standard_normal(d_model)
    qa = [sum(W["w_qa"][o, i] * x[i] for i in range(d_model)) for o in range(q_lora)]
    ms = sum(v * v for v in qa) / q_lora
    qn = [qa[i] / math.sqrt(ms + eps) * W["q_gain"][i] for i in range(q_lora)]
    q = [sum(W["w_qb"][o, i] * qn[i] for i in range(q_lora)) for o in range(H * (d_nope + d_r))]
    got = O.query_from_x(x, W["w_qa"], W["q_gain"], W["w_qb"], H, d_nope, d_r, eps)
    np.testing.assert_allclose(got, np.array(q).reshape(H, d_nope + d_r), rtol=1e-12, atol=1e-13)


# ------------------------------------------------------------ sliding window and key ranges

def test_window_special_cases():
    """window >= L is plain causal attention; window = 1 returns each query's own value."""
    rng = np.random.default_rng(30)
    q, rows, W_UK, W_UV = _rand_decode(rng, L=40, Tq=3)
    full = O.decode_expanded(q, rows, W_UK, W_UV, 0.3, 10000.0)
    np.testing.assert_array_equal(O.decode_expanded(q, rows, W_UK, W_UV, 0.3, 10000.0,
                                                    window=40), full)
    own = O.decode_expanded(q, rows, W_UK, W_UV, 0.3, 10000.0, window=1)
    for t in range(3):
        expect = np.einsum("d,hvd->hv", rows[37 + t, :16], W_UV)
        np.testing.assert_allclose(own[t], expect, rtol=1e-13, atol=1e-13)


def test_window_equals_truncated_history():
    """With window W, the output equals plain attention over the last W rows only, with the
    query's position (and RoPE angle) unchanged: brute force by cutting the history. RoPE depends
    only on relative positions, so the cut is rotated back to position 0 and the query too."""
    rng = np.random.default_rng(31)
    q, rows, W_UK, W_UV = _rand_decode(rng, L=50, Tq=1)
    W = 13
    got = O.decode_expanded(q, rows, W_UK, W_UV, 0.3, 10000.0, window=W)
    # keep the last W rows; re-rotate their k_R by -(50 - W) and the query's q_rope by the same
    tail = rows[50 - W:].copy()
    tail[:, 16:] = O.rope(tail[:, 16:], -(50 - W), 10000.0)
    ref = O.decode_expanded(q, tail, W_UK, W_UV, 0.3, 10000.0)
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("window", [0, 7])
def test_absorbed_equals_expanded_with_window(window):
    rng = np.random.default_rng(32)
    q, rows, W_UK, W_UV = _rand_decode(rng, L=30, Tq=2)
    a = O.decode_expanded(q, rows, W_UK, W_UV, 0.3, 10000.0, window=window)
    b = O.decode_absorbed(q, rows, W_UK, W_UV, 0.3, 10000.0, window=window)
    assert np.max(np.abs(a - b)) <= 1e-12 * np.max(np.abs(a))


@pytest.mark.parametrize("cuts,window", [([0, 64, 100], 0), ([0, 1, 2, 100], 0),
                                         ([0, 50, 100], 30), ([0, 99, 100], 0)])
def test_partials_merge_to_the_whole_softmax(cuts, window):
    """Splitting the keys at any cut points and merging the partials reproduces the absorbed
    form's latent output over all keys (then W_UV gives decode_expanded's output)."""
    rng = np.random.default_rng(33)
    q, rows, W_UK, W_UV = _rand_decode(rng, L=100, Tq=2)
    parts = [O.latent_partial(q, rows, W_UK, 0.3, 10000.0, a, b, window=window)
             for a, b in zip(cuts[:-1], cuts[1:])]
    o = O.merge_partials(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
    out = np.einsum("thd,hvd->thv", o, W_UV)
    ref = O.decode_expanded(q, rows, W_UK, W_UV, 0.3, 10000.0, window=window)
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-12)


def test_partial_of_an_empty_range_is_minus_infinity_and_ignored():
    rng = np.random.default_rng(34)
    q, rows, W_UK, W_UV = _rand_decode(rng, L=20, Tq=1)
    o, lse = O.latent_partial(q, rows, W_UK, 0.3, 10000.0, 20, 20)
    assert np.all(lse == -np.inf) and np.all(o == 0.0)
    o2, lse2 = O.latent_partial(q, rows, W_UK, 0.3, 10000.0, 0, 20)
    m = O.merge_partials(np.stack([o, o2]), np.stack([lse, lse2]))
    np.testing.assert_array_equal(m, o2)


def test_partial_lse_is_the_log_normaliser():
    """Brute force: lse = ln sum_j exp(s_j) over the range, s_j from the expanded form's keys."""
    rng = np.random.default_rng(35)
    q, rows, W_UK, W_UV = _rand_decode(rng, L=12, Tq=1)
    _, lse = O.latent_partial(q, rows, W_UK, 0.3, 10000.0, 3, 9, heads=[1])
    K = np.concatenate([rows[:, :16] @ W_UK[1].T, rows[:, 16:]], axis=1)
    qf = np.concatenate([q[0, 1, :8], O.rope(q[0, 1, 8:], 11, 10000.0)])
    s = [0.3 * sum(qf[i] * K[j, i] for i in range(16)) for j in range(3, 9)]
    assert abs(lse[0, 0] - math.log(sum(math.exp(v) for v in s))) <= 1e-12 * abs(lse[0, 0])
