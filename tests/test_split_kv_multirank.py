"""The split-KV exchange of head_latent_attention_05_b200.split_kv with two gloo ranks on CPU.

Each rank takes its page-aligned key range of every sequence (kv_ranges), computes its partial
latent outputs and log-sum-exps with the oracle (standing in for mla_decode_partial, which needs
a GPU), and the ranks exchange them with gather_parts. Merging the gathered parts (oracle
merge_partials) and projecting must reproduce the whole decode, and the ranges must cover every
key exactly once.
"""

import math
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from head_latent_attention_05_b200.split_kv import gather_parts, kv_ranges
from oracle import mla_oracle as O

H, D_C, D_R, D_NOPE, D_V, TQ = 3, 16, 8, 8, 6, 2
LENS = [130, 64, 1 + TQ, 700]


def _inputs():
    rng = np.random.default_rng(40)
    q = rng.standard_normal((len(LENS), TQ, H, D_NOPE + D_R))
    rows = [rng.standard_normal((L, D_C + D_R)) for L in LENS]
    W_UK = rng.standard_normal((H, D_NOPE, D_C)) / math.sqrt(D_C)
    W_UV = rng.standard_normal((H, D_V, D_C)) / math.sqrt(D_C)
    return q, rows, W_UK, W_UV


def test_ranges_cover_every_key_once_on_page_boundaries():
    for world in (1, 2, 3, 8):
        rng = kv_ranges(LENS, world)
        for b, L in enumerate(LENS):
            cov = np.zeros(L, dtype=int)
            for r in range(world):
                a, e = rng[r][b]
                assert a % 64 == 0 and (e % 64 == 0 or e == L) and 0 <= a <= e <= L
                cov[a:e] += 1
            assert np.all(cov == 1)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, rows, W_UK, W_UV = _inputs()
        rng = kv_ranges(LENS, world)[rank]
        o_rows, l_rows = [], []
        for b in range(len(LENS)):
            o, lse = O.latent_partial(q[b], rows[b], W_UK, 0.25, 10000.0, rng[b][0], rng[b][1])
            o_rows.append(o.reshape(TQ * H, D_C))
            l_rows.append(lse.reshape(TQ * H))
        o_part = torch.from_numpy(np.concatenate(o_rows)).to(torch.float32)
        lse = torch.from_numpy(np.concatenate(l_rows)).to(torch.float32)
        o_all, l_all = gather_parts(o_part, lse)
        merged = O.merge_partials(o_all.numpy(), l_all.numpy())          # [rows, d_c]
        got = merged.reshape(len(LENS), TQ, H, D_C)
        err = 0.0
        for b in range(len(LENS)):
            proj = np.einsum("thd,hvd->thv", got[b], W_UV)
            ref = O.decode_expanded(q[b], rows[b], W_UK, W_UV, 0.25, 10000.0)
            err = max(err, float(np.max(np.abs(proj - ref)) / np.max(np.abs(ref))))
        out[rank] = err
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_exchange_partials_and_reproduce_the_decode():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        errs = dict(out)
    assert sorted(errs) == [0, 1]
    # fp32 transport of fp64 partials: relative error at fp32 rounding level
    assert max(errs.values()) < 1e-6, errs
