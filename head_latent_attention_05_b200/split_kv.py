"""Split-KV decode across GPUs for long contexts: the host side of the one exchange step.

Each GPU holds whole 64-token pages of a contiguous key range of every sequence. A decode step
runs mla_decode_partial on every GPU over its range (latent output O / l and its log-sum-exp per
query row), gathers the partials of all GPUs with one all-gather (NCCL over NVLink / NVSwitch),
and runs mla_combine, which merges them in rank order and applies W_UV; every GPU then holds the
same output. The pages are silent on splitting one sequence's keys; the merge is the same
log-sum-exp merge the library uses between the splits of one GPU.
"""

from __future__ import annotations

import torch
import torch.distributed as dist

from . import mla_combine, mla_combine_workspace_size, mla_decode_partial


def kv_ranges(seq_lens, world: int, page_size: int = 64):
    """[begin, end) key range of every sequence on every rank: the sequence's pages are dealt
    out in contiguous, near-equal runs (rank r gets pages [r*n/world, (r+1)*n/world)), so
    ranges start on page boundaries and every key belongs to exactly one rank. Returns
    ranges[rank][b] = (begin, end); a rank may get an empty range (begin == end)."""
    out = [[] for _ in range(world)]
    for L in (int(v) for v in seq_lens):
        n = (L + page_size - 1) // page_size
        for r in range(world):
            p0, p1 = (r * n) // world, ((r + 1) * n) // world
            out[r].append((min(L, p0 * page_size), min(L, p1 * page_size)))
    return out


def gather_parts(o_part: torch.Tensor, lse: torch.Tensor, group=None):
    """All-gather every rank's partial (o_part [rows, d_c], lse [rows]) into [world, rows, d_c]
    and [world, rows], in rank order."""
    world = dist.get_world_size(group)
    # the concatenated output form (every backend takes it), viewed as stacked
    o_all = torch.empty((world * o_part.shape[0],) + tuple(o_part.shape[1:]), dtype=o_part.dtype,
                        device=o_part.device)
    l_all = torch.empty((world * lse.shape[0],), dtype=lse.dtype, device=lse.device)
    dist.all_gather_into_tensor(o_all, o_part.contiguous(), group=group)
    dist.all_gather_into_tensor(l_all, lse.contiguous(), group=group)
    return o_all.view((world,) + tuple(o_part.shape)), l_all.view(world, lse.shape[0])


def decode_split_kv(cfg, q, cache, block_table, seq_lens, seq_lens_host, w_uk_t, w_uv,
                    workspace, out, group=None):
    """One decode step whose keys are split over the ranks of `group`. This rank's cache holds
    the pages of its range (kv_ranges; block_table entries of other pages are never read).
    q, seq_lens, w_uk_t, w_uv are the same on every rank; out [B, Tq, H, d_v] ends up identical
    on every rank. workspace: mla_decode_workspace_size bytes."""
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    B, Tq, H = q.shape[0], q.shape[1], q.shape[2]
    rng = kv_ranges(seq_lens_host, world, cfg.page_size)[rank]
    kv_b = torch.tensor([a for a, _ in rng], dtype=torch.int32, device=q.device)
    kv_e = torch.tensor([b for _, b in rng], dtype=torch.int32, device=q.device)
    rows = B * Tq * H
    o_part = torch.empty((rows, cfg.d_c), dtype=q.dtype, device=q.device)
    lse = torch.empty((rows,), dtype=torch.float32, device=q.device)
    mla_decode_partial(cfg, q, cache, block_table, seq_lens, kv_b, kv_e, w_uk_t, workspace,
                       o_part, lse)
    o_all, l_all = gather_parts(o_part, lse, group)
    n = mla_combine_workspace_size(cfg, B, Tq)
    ws = torch.empty(max(n, 0), dtype=torch.uint8, device=q.device) if n > 0 else None
    mla_combine(cfg, o_all, l_all, w_uv, ws, out)
    return out
