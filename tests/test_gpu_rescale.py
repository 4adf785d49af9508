"""Parity of the latent attention's online softmax when the running maximum moves.

The attention kernel keeps a reference maximum per query row and only moves it (rescaling the
accumulated output and row sum) when a page's scores exceed it by more than 2^8 in base 2. With
N(0,1) inputs the scores never rise that far after a segment's first page, so these tests plant
one row per page whose score for one head climbs by 7 (natural units, above 8 ln 2 = 5.55)
from page to page in a sawtooth of period 4. Each test first checks, from the oracle's own
scores, that most page boundaries of that head rise by more than 8 ln 2 (so every segment of
two pages or more that starts on a rising page takes the rescale path), then compares the GPU
output with the oracle on the planted heads and a few others, within the bf16 bound
max|err| <= 1e-2 max|ref| + 1e-3.
"""

import math

import numpy as np
import pytest
import torch

import harness as Hs
import head_latent_attention_05_b200 as mla
import workloads as W

pytestmark = pytest.mark.gpu

V2 = W.WORKLOADS["v2_bf16_b16_ctx4096"]
LONG = W.WORKLOADS["v2_bf16_b4_ctx131072_tq2"]
RISE = 8.0 * math.log(2.0)


@pytest.fixture(autouse=True)
def _no_device_error():
    mla.mla_get_device_error()
    yield
    assert mla.mla_get_device_error() == 0


def _lens(*ls):
    return torch.tensor(ls, dtype=torch.int32)


def _check_rises(c, b, h, t, new_rows):
    rows = Hs.oracle_rows_of(c, b, new_rows)
    s = Hs.oracle_scores(c, b, h, t, rows)
    L = rows.shape[0]
    n_pages = (L + W.PAGE_SIZE - 1) // W.PAGE_SIZE
    tile_max = np.array([s[p * W.PAGE_SIZE:min(L, (p + 1) * W.PAGE_SIZE)].max()
                         for p in range(n_pages)])
    rises = np.diff(tile_max) > RISE
    assert rises.mean() >= 0.6, f"only {rises.mean():.2f} of page boundaries rise by 8 ln 2"
    return rises


def _run(c, plants, extra_heads):
    """plants: list of (b, h, t). Appends, decodes, and checks every planted (b, h, t) plus
    extra heads of each planted sequence against the oracle."""
    Hs.run_append(c)
    out = Hs.run_decode(c).float().cpu()
    new_rows = Hs.oracle_new_rows(c)
    for b, h, t in plants:
        _check_rises(c, b, h, t, new_rows)
        heads = sorted(set([h] + list(extra_heads)))
        ref = Hs.oracle_out(c, b, heads, new_rows)
        Hs.assert_parity(out[b][:, heads], ref, c.w.dtype, f"b={b} planted head {h}")
    assert torch.isfinite(out).all()


def test_rescale_one_long_sequence_split_over_every_pair():
    """40,000 tokens alone: ~8.5 pages per CTA pair, so every pair runs multi-page segments."""
    c = Hs.make_case(W.small_variant(V2, B=1), _lens(40000))
    Hs.plant_score_staircase(c, 0, 5)
    _run(c, [(0, 5, 0)], [0, 64, 127])


def test_rescale_mixed_batch():
    """Long and short sequences together, a different planted head in each long one."""
    c = Hs.make_case(W.small_variant(V2, B=6, pages="shuffled"),
                     _lens(20000, 64, 9000, 300, 15000, 4100))
    plants = [(0, 0, 0), (2, 77, 0), (4, 127, 0), (5, 31, 0)]
    for b, h, t in plants:
        Hs.plant_score_staircase(c, b, h, t)
    _run(c, plants, [64])


def test_rescale_two_causal_query_tokens():
    """Tq = 2: the planted rows climb for query token 0 of head 9; token 1 sees them too."""
    c = Hs.make_case(W.small_variant(LONG, B=2), _lens(30000, 12000))
    Hs.plant_score_staircase(c, 0, 9, t=0)
    Hs.plant_score_staircase(c, 1, 100, t=0, base=9.0)
    _run(c, [(0, 9, 0), (1, 100, 0)], [0, 127])
