"""Seeded synthetic workloads for MLA decode: shapes, lengths, page tables and random tensors.

This module is shared by the tests, the benchmark and the oracle checks. It holds none of the
attention arithmetic: it only draws random numbers (torch CPU generator, fixed seed), rounds
them to the storage dtype, and lays out the paged cache bookkeeping (lengths, block tables).

Distributions (chosen to match what the module on the pages produces with random weights):
  * x ~ N(0, 1)                                   -- token hidden states
  * every weight ~ N(0, 1/fan_in), RMSNorm gains 1 -- nn.Linear-style random init
  * cache rows [c_KV | k_R] ~ N(0, 1)              -- c_KV after RMSNorm has unit RMS, and a
                                                    RoPE rotation of N(0,1) is again N(0,1)
  * q = [q_nope | q_rope] ~ N(0, 1)                -- RMSNorm'd q_a times a 1/fan_in weight
The cache pool is filled i.i.d. page by page, so a shuffled page order is just a relabelling.

A quantised cache (kv = "fp8": E4M3 codes plus one float32 scale per token, the page layout of
include/mla.h) is drawn the same way: codes are N(0,1) draws times 448/4.5 cast to float8_e4m3fn
by torch (so a row's codes reach about ±448, as a row quantised to its own maximum does), and
each token's scale is 4.5/448 times a uniform factor in [0.75, 1.25].
"""

from __future__ import annotations

import dataclasses
import math

import torch

PAGE_SIZE = 64


@dataclasses.dataclass(frozen=True)
class Workload:
    """One decode workload. Sizes follow DeepSeek-V2 naming (d_c = kv_lora_rank, d_r = rope dim)."""

    name: str
    B: int
    H: int
    d_model: int
    d_c: int
    d_r: int
    d_nope: int
    d_v: int
    q_lora: int
    Tq: int
    lens: tuple            # ("fixed", L) | ("uniform", lo, hi) | ("loguniform", lo, hi)
    dtype: str             # "f32" | "bf16"
    pages: str             # "identity" | "shuffled"
    seed: int
    rms_eps: float = 1e-6
    rope_theta: float = 10000.0
    kv: str = "plain"      # cache rows: "plain" (in dtype) | "fp8" (E4M3 codes + token scales)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d_nope + self.d_r)

    @property
    def row(self) -> int:
        return self.d_c + self.d_r

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def fp8_page_bytes(self) -> int:
        """Bytes of one quantised cache page: 64 rows of codes, then 64 float32 scales."""
        return PAGE_SIZE * (self.row + 4)


# The five workloads: a tiny fp32 case, DeepSeek-V2 shape at batch 16 x 4096, the 32-head
# module shape with shuffled pages, a V2 serving mix with log-uniform lengths, and a long
# context case with two causal query tokens per sequence.
WORKLOADS = {
    "tiny_f32_b1_h4_ctx128": Workload(
        "tiny_f32_b1_h4_ctx128", B=1, H=4, d_model=128, d_c=64, d_r=16, d_nope=32, d_v=32,
        q_lora=48, Tq=1, lens=("fixed", 128), dtype="f32", pages="identity", seed=0),
    "v2_bf16_b16_ctx4096": Workload(
        "v2_bf16_b16_ctx4096", B=16, H=128, d_model=5120, d_c=512, d_r=64, d_nope=128,
        d_v=128, q_lora=1536, Tq=1, lens=("fixed", 4096), dtype="bf16", pages="identity",
        seed=1),
    "h32_bf16_b32_ctx512to8192_shuffled": Workload(
        "h32_bf16_b32_ctx512to8192_shuffled", B=32, H=32, d_model=4096, d_c=512, d_r=64,
        d_nope=128, d_v=128, q_lora=512, Tq=1, lens=("uniform", 512, 8192), dtype="bf16",
        pages="shuffled", seed=2),
    "v2_bf16_b64_ctx1kto32k_mix": Workload(
        "v2_bf16_b64_ctx1kto32k_mix", B=64, H=128, d_model=5120, d_c=512, d_r=64,
        d_nope=128, d_v=128, q_lora=1536, Tq=1, lens=("loguniform", 1024, 32768),
        dtype="bf16", pages="shuffled", seed=3),
    "v2_bf16_b4_ctx131072_tq2": Workload(
        "v2_bf16_b4_ctx131072_tq2", B=4, H=128, d_model=5120, d_c=512, d_r=64, d_nope=128,
        d_v=128, q_lora=1536, Tq=2, lens=("fixed", 131072), dtype="bf16", pages="identity",
        seed=4),
}

WORKLOAD_ORDER = list(WORKLOADS)

# The serving mix again over a quantised (FP8 E4M3, per-token scale) latent cache.
EXTRA_WORKLOADS = {
    "v2_fp8_b64_ctx1kto32k_mix": Workload(
        "v2_fp8_b64_ctx1kto32k_mix", B=64, H=128, d_model=5120, d_c=512, d_r=64,
        d_nope=128, d_v=128, q_lora=1536, Tq=1, lens=("loguniform", 1024, 32768),
        dtype="bf16", pages="shuffled", seed=3, kv="fp8"),
}


def get(name: str) -> Workload:
    """A workload by name, from WORKLOADS or EXTRA_WORKLOADS."""
    return WORKLOADS[name] if name in WORKLOADS else EXTRA_WORKLOADS[name]


def small_variant(w: Workload, **over) -> Workload:
    """Same workload with some fields replaced (smaller batch, shorter context, ...)."""
    return dataclasses.replace(w, **over)


def _gen(seed: int, stream: int) -> torch.Generator:
    g = torch.Generator()
    g.manual_seed(seed * 1_000_003 + stream)
    return g


def seq_lens(w: Workload) -> torch.Tensor:
    """Context length of each sequence, counting the Tq new tokens (int32 [B])."""
    g = _gen(w.seed, 1)
    kind = w.lens[0]
    if kind == "fixed":
        L = torch.full((w.B,), w.lens[1], dtype=torch.int64)
    elif kind == "uniform":
        lo, hi = w.lens[1], w.lens[2]
        L = torch.randint(lo, hi + 1, (w.B,), generator=g, dtype=torch.int64)
    elif kind == "loguniform":
        lo, hi = w.lens[1], w.lens[2]
        u = torch.rand((w.B,), generator=g, dtype=torch.float64)
        L = torch.exp(math.log(lo) + u * (math.log(hi) - math.log(lo))).round().to(torch.int64)
        L = L.clamp(lo, hi)
    else:
        raise ValueError(kind)
    return torch.clamp(L, min=w.Tq).to(torch.int32)


@dataclasses.dataclass
class PageTable:
    block_table: torch.Tensor   # int32 [B, max_pages]; -1 where unused
    num_pages: int
    max_pages: int


def page_table(w: Workload, lens: torch.Tensor, spare_pages: int = 0) -> PageTable:
    """Assign whole 64-token pages to each sequence; identity or Fisher-Yates shuffled order."""
    need = [(int(L) + PAGE_SIZE - 1) // PAGE_SIZE for L in lens.tolist()]
    total = sum(need) + spare_pages
    max_pages = max(need) if need else 1
    if w.pages == "shuffled":
        perm = torch.randperm(total, generator=_gen(w.seed, 2)).to(torch.int32)
    else:
        perm = torch.arange(total, dtype=torch.int32)
    bt = torch.full((w.B, max_pages), -1, dtype=torch.int32)
    off = 0
    for b, n in enumerate(need):
        bt[b, :n] = perm[off:off + n]
        off += n
    return PageTable(bt, total, max_pages)


def randn(shape, seed: int, stream: int, std: float = 1.0, dtype=torch.float32) -> torch.Tensor:
    """N(0, std^2) drawn in fp32 from a seeded CPU generator, then rounded (RNE) to dtype."""
    t = torch.randn(shape, generator=_gen(seed, stream), dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


@dataclasses.dataclass
class Weights:
    w_dkv: torch.Tensor     # [d_c + d_r, d_model]        (wkv_a)
    kv_gain: torch.Tensor   # [d_c]                       (kv_norm weight)
    wkv_b: torch.Tensor     # [H*(d_nope+d_v), d_c]
    w_qa: torch.Tensor      # [q_lora, d_model]
    q_gain: torch.Tensor    # [q_lora]
    w_qb: torch.Tensor      # [H*(d_nope+d_r), q_lora]


def weights(w: Workload) -> Weights:
    dt = w.torch_dtype
    return Weights(
        w_dkv=randn((w.row, w.d_model), w.seed, 10, 1.0 / math.sqrt(w.d_model), dt),
        kv_gain=torch.ones(w.d_c, dtype=dt),
        wkv_b=randn((w.H * (w.d_nope + w.d_v), w.d_c), w.seed, 11, 1.0 / math.sqrt(w.d_c), dt),
        w_qa=randn((w.q_lora, w.d_model), w.seed, 12, 1.0 / math.sqrt(w.d_model), dt),
        q_gain=torch.ones(w.q_lora, dtype=dt),
        w_qb=randn((w.H * (w.d_nope + w.d_r), w.q_lora), w.seed, 13,
                   1.0 / math.sqrt(w.q_lora), dt),
    )


def output_weight(w: Workload) -> torch.Tensor:
    """wo weight [d_model, H*d_v] ~ N(0, 1/(H*d_v)), in dtype (drawn only when asked for: it is
    the largest tensor of the layer, 168 MB in bf16 at DeepSeek-V2 shape)."""
    return randn((w.d_model, w.H * w.d_v), w.seed, 14, 1.0 / math.sqrt(w.H * w.d_v),
                 w.torch_dtype)


def cache_pool(w: Workload, num_pages: int, chunk_pages: int = 2048) -> torch.Tensor:
    """Page pool [num_pages, 64, d_c+d_r] filled i.i.d. N(0,1) (the history rows), in dtype."""
    out = torch.empty((num_pages, PAGE_SIZE, w.row), dtype=w.torch_dtype)
    for i, p0 in enumerate(range(0, num_pages, chunk_pages)):
        p1 = min(num_pages, p0 + chunk_pages)
        out[p0:p1] = randn((p1 - p0, PAGE_SIZE, w.row), w.seed, 1000 + i, 1.0, w.torch_dtype)
    return out


def cache_pool_fp8(w: Workload, num_pages: int, chunk_pages: int = 2048) -> torch.Tensor:
    """Quantised page pool as bytes [num_pages, fp8_page_bytes]: per page 64 rows of E4M3 codes
    (row after row), then the 64 float32 token scales (see the module docstring)."""
    n_codes = PAGE_SIZE * w.row
    out = torch.empty((num_pages, w.fp8_page_bytes), dtype=torch.uint8)
    for i, p0 in enumerate(range(0, num_pages, chunk_pages)):
        p1 = min(num_pages, p0 + chunk_pages)
        v = randn((p1 - p0, n_codes), w.seed, 1000 + i, 448.0 / 4.5, torch.float32)
        out[p0:p1, :n_codes] = v.clamp_(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8)
        u = torch.rand((p1 - p0, PAGE_SIZE), generator=_gen(w.seed, 3000 + i), dtype=torch.float32)
        scales = (4.5 / 448.0) * (0.75 + 0.5 * u)
        out[p0:p1, n_codes:] = scales.view(torch.uint8).view(p1 - p0, 4 * PAGE_SIZE)
    return out


def tail_slots(lens: torch.Tensor, pt: PageTable):
    """(page, first_unused_slot) for every sequence whose last page is partly empty."""
    out = []
    for b, L in enumerate(lens.tolist()):
        n = (L + PAGE_SIZE - 1) // PAGE_SIZE
        if L % PAGE_SIZE:
            out.append((int(pt.block_table[b, n - 1]), L % PAGE_SIZE))
    return out


def new_token_inputs(w: Workload, lens: torch.Tensor):
    """Hidden states of the Tq new tokens, their (sequence, position) and their queries.

    Returns x_new [B*Tq, d_model], seq_idx int32 [B*Tq], pos int32 [B*Tq] (0-based position in
    the sequence: L_b - Tq + t), and q [B, Tq, H, d_nope + d_r] (un-rotated).
    """
    dt = w.torch_dtype
    x_new = randn((w.B * w.Tq, w.d_model), w.seed, 20, 1.0, dt)
    seq_idx = torch.arange(w.B, dtype=torch.int32).repeat_interleave(w.Tq)
    t = torch.arange(w.Tq, dtype=torch.int32).repeat(w.B)
    pos = lens.to(torch.int32).repeat_interleave(w.Tq) - w.Tq + t
    q = randn((w.B, w.Tq, w.H, w.d_nope + w.d_r), w.seed, 21, 1.0, dt)
    return x_new, seq_idx, pos, q


def full_sequence_x(w: Workload, lens: torch.Tensor) -> torch.Tensor:
    """Hidden states of every context token, [B, max(L), d_model] (used by the tiny workload)."""
    Lmax = int(lens.max())
    return randn((w.B, Lmax, w.d_model), w.seed, 30, 1.0, w.torch_dtype)
