#!/usr/bin/env python3
"""Benchmark of one MLA decode step on B200: append the new tokens' latents, then decode.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

A step is one pass of the whole hot path over one batch of synthetic input:
mla_append_latent (down-projection GEMM + RMSNorm/RoPE/scatter) then mla_decode (query
absorption with the split-KV planner, latent attention, split merge fused with the value
projection), five kernel launches through the C ABI (six over a quantised cache, whose
query rows are split into E4M3 parts by one more kernel). The metric
is cache-tokens x heads per second: sum_b L_b * Tq * H / step time, summed over all GPUs
(each GPU decodes its own batch: weak scaling, no data-path collective).

Timing: the K timed steps are captured once into a CUDA graph (so host launch latency stays
out of device time) and replayed; before every step the graph writes 256 MiB to flush the
126 MB L2 and then reads another 256 MiB so that the written lines are drained to HBM before
the step rather than during it, all outside the step's CUDA events, which bracket each step and nothing inside it.
Per-kernel times (and the attention kernel's time in the roofline) come from a second replay
of the same steps in which the library records events between its kernels (those marks stop
consecutive kernels from overlapping their start and end, so they are not in the headline).
`e2e` repeats the step through the plain API from pinned
host buffers, with the host->device copies of the step's inputs and the device->host copy of
its output inside the timed region. rank 0 prints one JSON line.
"""

from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import workloads as WL  # noqa: E402

METRIC = "MLA decode cache-tokens/s (×heads) on 1 B200; % of HBM/tensor roofline"
UNIT = "cache_tokens*heads/s"
DEFAULT_WORKLOAD = "v2_bf16_b64_ctx1kto32k_mix"
# measured after the headline, each with its own attention roofline
EXTRA_WORKLOADS = ("v2_bf16_b16_ctx4096", "h32_bf16_b32_ctx512to8192_shuffled",
                   "v2_bf16_b4_ctx131072_tq2", "v2_fp8_b64_ctx1kto32k_mix")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
ATTN_PROFILE = os.path.join(ROOT, "profiles", "attn_kernel_traffic.json")


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    choices=WL.WORKLOAD_ORDER + list(WL.EXTRA_WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="budget of the oracle CPU-baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="launch the timed steps eagerly")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the other workloads measured after the headline")
    ap.add_argument("--extra-steps", type=int, default=40,
                    help="timed steps of each extra workload")
    return ap.parse_args()


# --------------------------------------------------------------------------- bookkeeping

def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def work_of(w: WL.Workload, lens: torch.Tensor) -> dict:
    """Algorithmic work of one step (per GPU)."""
    Ls = [int(v) for v in lens.tolist()]
    tokens = sum(Ls)
    elem = 4 if w.dtype == "f32" else 2
    # a quantised cache row: one byte per code plus its float32 scale
    cache_bytes = tokens * (w.row + 4) if w.kv == "fp8" else tokens * w.row * elem
    w_bytes = 2 * w.H * w.d_nope * w.d_c * elem          # W_UK + W_UV
    attn_flops = sum(L * w.Tq for L in Ls) * w.H * 2 * (w.row + w.d_c)
    proj_flops = 2 * (2 * w.B * w.Tq * w.H * w.d_nope * w.d_c)
    return dict(units=sum(L * w.Tq for L in Ls) * w.H, tokens=tokens, cache_bytes=cache_bytes,
                weight_bytes=w_bytes, attn_flops=attn_flops, proj_flops=proj_flops)


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 10 ms while running."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,"
             "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "10"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.05)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 10:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}

        def num(v):
            try:
                return float(v)
            except ValueError:
                return None
        busy = [r for r in rows if (num(r[4]) or 0) > 0] or rows
        sm = [num(r[1]) for r in busy if num(r[1]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in busy for i in range(4) if r[6 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": num(rows[0][2]), "reasons": reasons,
                "samples": len(rows), "samples_busy": len(busy),
                "power_w_max": max((num(r[3]) or 0.0) for r in rows)}


def cpu_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


# ------------------------------------------------------------------ oracle (CPU baseline)

def oracle_sample(w: WL.Workload, lens, pt, weights, cache_host, x_new, pos, q, seconds: float,
                  max_units: int | None = None, form: str = "expanded"):
    """Time the fp64 oracle (as it stands; the expanded form unless form == "absorbed") on
    (sequence, head) units of the workload for about `seconds`; returns (rate in
    cache-tokens*heads/s, units, description)."""
    from oracle import mla_oracle as O
    decode = O.decode_absorbed if form == "absorbed" else O.decode_expanded
    W_UK, W_UV = O.split_wkv_b(weights.wkv_b, w.H, w.d_nope, w.d_v)
    new_rows = O.latent_rows(x_new, weights.w_dkv, weights.kv_gain, pos.numpy(), w.d_c,
                             w.rms_eps, w.rope_theta)
    if w.kv == "fp8":   # the stored rows: the new ones quantised, the history dequantised
        new_rows = O.dequantize_rows_e4m3(*O.quantize_rows_e4m3(new_rows.astype("float32")))
        n = WL.PAGE_SIZE * w.row
        codes = cache_host[:, :n].view(cache_host.shape[0], WL.PAGE_SIZE, w.row).numpy()
        scales = cache_host[:, n:].view(torch.float32).numpy()
    heads = [0, w.H // 2, w.H - 1, w.H // 3, (2 * w.H) // 3]
    done_units, done_work, elapsed = 0, 0, 0.0
    rows_cache = {}
    i = 0
    while elapsed < seconds and (max_units is None or done_units < max_units):
        b = i % w.B
        h = heads[(i // w.B) % len(heads)]
        i += 1
        L = int(lens[b])
        if b not in rows_cache:
            if w.kv == "fp8":
                r = O.gather_rows_fp8(codes, scales, pt.block_table[b].numpy(), L, WL.PAGE_SIZE)
            else:
                r = O.gather_rows(cache_host, pt.block_table[b].numpy(), L, WL.PAGE_SIZE)
            r[L - w.Tq:] = new_rows[b * w.Tq:(b + 1) * w.Tq]
            rows_cache = {b: r}
        t0 = time.perf_counter()
        decode(q[b], rows_cache[b], W_UK, W_UV, w.scale, w.rope_theta, heads=[h])
        elapsed += time.perf_counter() - t0
        done_units += 1
        done_work += L * w.Tq
    rate = done_work / elapsed if elapsed > 0 else 0.0
    desc = (f"{done_units} (sequence, head) units of {w.name} through the fp64 {form}-form "
            f"oracle ({done_work} cache-token*heads, {elapsed:.1f} s); rate scales to the full "
            f"workload because the work per cache-token*head is uniform")
    return rate, done_units, desc


# ------------------------------------------------------------------------------- setup

def build_inputs(w: WL.Workload, device):
    lens = WL.seq_lens(w)
    pt = WL.page_table(w, lens)
    weights = WL.weights(w)
    cache_host = (WL.cache_pool_fp8(w, pt.num_pages) if w.kv == "fp8"
                  else WL.cache_pool(w, pt.num_pages))
    x_new, seq_idx, pos, q = WL.new_token_inputs(w, lens)
    return lens, pt, weights, cache_host, x_new, seq_idx, pos, q


def max_over_ranks(x: float, world: int, device) -> float:
    """The largest x over all ranks (the job's time is the slowest rank's); x itself at N=1."""
    if world <= 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank: float, ms_per_step: float, world: int) -> float:
    """Whole-job throughput: every rank processes its own units_per_rank each step."""
    return world * units_per_rank / (ms_per_step / 1e3)


def run_reference(args, rank: int, world: int):
    """Reference arm: the fp64 oracle on this host's cores, same workload / metric / unit."""
    if rank != 0:
        return
    w = WL.get(args.workload)
    lens, pt, weights, cache_host, x_new, seq_idx, pos, q = build_inputs(w, "cpu")
    # each step: one (sequence, head) unit; the metric is total work / total time
    for _ in range(max(0, args.warmup)):
        oracle_sample(w, lens, pt, weights, cache_host, x_new, pos, q, 0.0, max_units=1)
    t0 = time.perf_counter()
    rate, units, desc = oracle_sample(w, lens, pt, weights, cache_host, x_new, pos, q,
                                      float("inf"), max_units=args.steps)
    wall = time.perf_counter() - t0
    cores = cpu_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": rate, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * wall / max(1, units),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": w.name, "batch_per_gpu": w.B, "heads": w.H, "tq": w.Tq,
                   "context": list(w.lens)},
        "cpu_baseline": {"value": rate, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": rate, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


class DeviceCase:
    """One workload's inputs on the device, the library's buffers and the step functions."""

    def __init__(self, mla, w: WL.Workload, dev):
        self.w, self.dev = w, dev
        (self.lens, self.pt, self.weights, self.cache_host, self.x_new_h, self.seq_idx_h,
         self.pos_h, self.q_h) = build_inputs(w, dev)
        self.cfg = mla.make_config(w.H, w.d_model, w.d_c, w.d_r, w.d_nope, w.d_v, WL.PAGE_SIZE,
                                   w.dtype, w.scale, w.rms_eps, w.rope_theta, kv_format=w.kv)
        dt = w.torch_dtype
        self.cache = self.cache_host.to(dev)
        self.bt = self.pt.block_table.to(dev)
        self.seq_lens = self.lens.to(dev)
        self.x_new, self.seq_idx, self.pos, self.q = (
            t.contiguous().to(dev) for t in (self.x_new_h, self.seq_idx_h, self.pos_h, self.q_h))
        self.w_dkv, self.kv_gain = self.weights.w_dkv.to(dev), self.weights.kv_gain.to(dev)
        self.w_uk_t = torch.empty((w.H, w.d_c, w.d_nope), dtype=dt, device=dev)
        self.w_uv = torch.empty((w.H, w.d_v, w.d_c), dtype=dt, device=dev)
        mla.mla_absorb_weights(self.cfg, self.weights.wkv_b.to(dev), self.w_uk_t, self.w_uv)
        n_tok = w.B * w.Tq
        self.ws_a = mla.workspace(mla.mla_append_workspace_size(self.cfg, n_tok), dev)
        self.ws_d = mla.workspace(mla.mla_decode_workspace_size(self.cfg, w.B, w.Tq), dev)
        self.out = torch.empty((w.B, w.Tq, w.H, w.d_v), dtype=dt, device=dev)
        self.work = work_of(w, self.lens)
        self.mla = mla

    def step(self, evs=None, marks=None):
        mla = self.mla
        if evs is not None:
            evs[0].record()
        if marks is not None:
            marks[0].record()
        mla.mla_append_latent(self.cfg, self.x_new, self.w_dkv, self.kv_gain, self.seq_idx,
                              self.pos, self.bt, self.cache, self.ws_a)
        if marks is not None:
            mla.mla_decode_profiled(self.cfg, self.q, self.cache, self.bt, self.seq_lens,
                                    self.w_uk_t, self.w_uv, self.ws_d, self.out, marks[1:5])
        else:
            self.decode()
        if evs is not None:
            evs[1].record()

    def decode(self):
        self.mla.mla_decode(self.cfg, self.q, self.cache, self.bt, self.seq_lens, self.w_uk_t,
                            self.w_uv, self.ws_d, self.out)


class L2Flush:
    """Before a step: write a buffer twice the L2 size (the step's inputs leave L2), then read
    another as large, so that the written buffer's dirty lines drain to HBM here and not inside
    the next step."""

    def __init__(self, dev):
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        self.flush = torch.empty(max(2 * l2, 256 << 20), dtype=torch.uint8, device=dev)
        self.drain = torch.zeros_like(self.flush)

    def __call__(self, i):
        self.flush.fill_(i & 0xFF)
        self.drain.max()


def attn_roofline(w: WL.Workload, work: dict, t_attn_s: float, ms_per_step: float) -> dict:
    """Roofline block of the latent attention kernel: its algorithmic bytes (or FLOPs) over its
    own CUDA-event time, against the measured HBM copy rate (or bf16 tensor peak)."""
    pk, pk_kind = peaks()
    hbm_peak = float(pk["hbm_gbs"])
    tc_peak = float(pk["bf16_tflops"])
    t_mem = work["cache_bytes"] / (hbm_peak * 1e9)
    t_tc = work["attn_flops"] / (tc_peak * 1e12)
    bound = "hbm" if t_mem >= t_tc else "tensor"
    if bound == "hbm":
        roof = {"bound": "hbm", "achieved": work["cache_bytes"] / t_attn_s / 1e9,
                "peak": hbm_peak, "unit": "GB/s"}
    else:
        roof = {"bound": "tensor", "achieved": work["attn_flops"] / t_attn_s / 1e12,
                "peak": tc_peak, "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = stored_traffic(w.name)
    roof["peak_source"] = (f"{pk_kind} (MEASURED_PEAKS.json: burst bf16 GEMM, copy HBM)"
                           if pk_kind == "measured" else "fallback")
    roof["kernel"] = "mla_decode_attn_fp8_kernel" if w.kv == "fp8" else "mla_decode_attn_kernel"
    roof["kernel_us"] = t_attn_s * 1e6
    roof["algorithmic_bytes_per_launch"] = work["cache_bytes"]
    roof["algorithmic_flops_per_launch"] = work["attn_flops"]
    roof["hbm_frac"] = (work["cache_bytes"] / t_attn_s / 1e9) / hbm_peak
    roof["tensor_frac"] = (work["attn_flops"] / t_attn_s / 1e12) / tc_peak
    roof["step_roofline_frac"] = max(
        (work["cache_bytes"] + work["weight_bytes"]) / (hbm_peak * 1e9),
        (work["attn_flops"] + work["proj_flops"]) / (tc_peak * 1e12)) / (ms_per_step / 1e3)
    return roof


def decode_roofline_ms(work: dict) -> float:
    """The path's roofline time for mla_decode: the larger of (cache + W_UK + W_UV bytes) over
    the HBM rate and (attention + projection FLOPs) over the tensor peak."""
    pk, _ = peaks()
    return 1e3 * max((work["cache_bytes"] + work["weight_bytes"]) / (float(pk["hbm_gbs"]) * 1e9),
                     (work["attn_flops"] + work["proj_flops"]) / (float(pk["bf16_tflops"]) * 1e12))


def measure_device(c: DeviceCase, flush_l2: L2Flush, K: int, Wm: int, world: int, use_graph: bool,
                   local_rank: int):
    """Warm up, then time K steps (append + decode) with CUDA events around each step, a marked
    replay for the per-kernel breakdown and a decode-only replay. Returns a dict of results."""
    mla = c.mla
    ev = lambda: torch.cuda.Event(enable_timing=True, external=True)
    step_ev = [[ev() for _ in range(2)] for _ in range(K)]
    prof_ev = [[ev() for _ in range(5)] for _ in range(K)]
    dec_ev = [[ev() for _ in range(2)] for _ in range(K)]
    # torch creates events lazily: record every event once so it exists before capture
    for evs in step_ev + prof_ev + dec_ev:
        for e in evs:
            e.record()
    torch.cuda.synchronize()
    for i in range(Wm):
        flush_l2(i)
        c.step()
    err = mla.mla_get_device_error()
    if err != 0:
        raise RuntimeError(f"device error during warm-up: {mla.mla_status_string(err)}")

    def capture(fn):
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream(device=c.dev)
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                fn()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        return g

    def timed_steps():
        for i in range(K):
            flush_l2(i * 7)
            c.step(evs=step_ev[i])

    def marked_steps():
        for i in range(K):
            flush_l2(i * 7)
            c.step(marks=prof_ev[i])

    def decode_steps():
        for i in range(K):
            flush_l2(i * 7)
            dec_ev[i][0].record()
            c.decode()
            dec_ev[i][1].record()

    graphs = [capture(f) for f in (timed_steps, marked_steps, decode_steps)] if use_graph else None
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.03)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t_wall0 = time.perf_counter()
    if graphs is not None:
        graphs[0].replay()
    else:
        timed_steps()
    torch.cuda.synchronize()
    t_wall = time.perf_counter() - t_wall0
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop()
    err = mla.mla_get_device_error()
    if err != 0:
        raise RuntimeError(f"device error in the timed region: {mla.mla_status_string(err)}")
    # the breakdown replay (same steps, event marks between the kernels), then decode alone
    if graphs is not None:
        graphs[1].replay()
        graphs[2].replay()
    else:
        marked_steps()
        decode_steps()
    torch.cuda.synchronize()
    del graphs

    names = ["append", "q_absorb_plan", "attention", "merge_value_proj"]
    per = {n: [] for n in names}
    steps_ms = [evs[0].elapsed_time(evs[1]) for evs in step_ev]
    for evs in prof_ev:
        for j, n in enumerate(names):
            per[n].append(evs[j].elapsed_time(evs[j + 1]))
    ms_per_step = max_over_ranks(sum(steps_ms), world, c.dev) / K
    kernel_ms = {n: statistics.fmean(v) for n, v in per.items()}
    kernel_ms["marked_step"] = statistics.fmean(evs[0].elapsed_time(evs[4]) for evs in prof_ev)
    decode_ms = max_over_ranks(statistics.fmean(e[0].elapsed_time(e[1]) for e in dec_ev), world,
                               c.dev)
    t_roof = decode_roofline_ms(c.work)
    decode_only = {"value": job_rate(c.work["units"], decode_ms, world), "unit": UNIT,
                   "ms_per_step": decode_ms, "roofline_frac": t_roof / decode_ms,
                   "roofline_ms": t_roof,
                   "what": "mla_decode alone (query absorption + planner, attention, merge + "
                           "value projection), same L2 flush, graph-timed"}
    return dict(ms_per_step=ms_per_step, value=job_rate(c.work["units"], ms_per_step, world),
                kernel_ms=kernel_ms, decode_only=decode_only, clocks=clk, wall=t_wall,
                roofline=attn_roofline(c.w, c.work, kernel_ms["attention"] / 1e3, ms_per_step))


def measure_e2e(c: DeviceCase, flush_l2: L2Flush, K: int, world: int) -> dict:
    """The same step through the plain API from pinned host memory: every step copies its
    inputs in and its output back inside the timed region. The append's inputs (x, seq_idx,
    pos) go in one copy on the step's stream, the decode's (q, seq_lens) in one copy on a
    second stream that runs while the append kernels do (mla_decode waits for it), the output
    in one copy that the host waits for."""
    mla, dev = c.mla, c.dev

    def staged(parts):
        offs, off = [], 0
        for t in parts:
            offs.append(off)
            off += (t.numel() * t.element_size() + 255) // 256 * 256
        host = torch.empty(off, dtype=torch.uint8).pin_memory()
        devb = torch.empty(off, dtype=torch.uint8, device=dev)
        views = []
        for t, o in zip(parts, offs):
            nb = t.numel() * t.element_size()
            host[o:o + nb].view(t.dtype).view(t.shape).copy_(t)
            views.append(devb[o:o + nb].view(t.dtype).view(t.shape))
        return host, devb, views

    app_h, app_d, (x_e, si_e, pos_e) = staged(
        [c.x_new_h.contiguous(), c.seq_idx_h.contiguous(), c.pos_h.contiguous()])
    dec_h, dec_d, (q_e, lens_e) = staged([c.q_h.contiguous(), c.lens.contiguous()])
    out_pin = torch.empty(c.out.shape, dtype=c.out.dtype).pin_memory()
    h2d = app_h.numel() + dec_h.numel()
    d2h = out_pin.numel() * out_pin.element_size()
    main_s = torch.cuda.current_stream(dev)
    side_s = torch.cuda.Stream(device=dev)
    q_ready = torch.cuda.Event()
    K2 = min(K, 50)
    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(K2)]
    e2e_ms = []
    for i in range(K2):
        flush_l2(i)
        a, b = e2e_ev[i]
        a.record()
        side_s.wait_stream(main_s)   # after the start mark and the previous step's reads
        with torch.cuda.stream(side_s):
            dec_d.copy_(dec_h, non_blocking=True)
            q_ready.record(side_s)
        app_d.copy_(app_h, non_blocking=True)
        mla.mla_append_latent(c.cfg, x_e, c.w_dkv, c.kv_gain, si_e, pos_e, c.bt, c.cache, c.ws_a)
        main_s.wait_event(q_ready)
        mla.mla_decode(c.cfg, q_e, c.cache, c.bt, lens_e, c.w_uk_t, c.w_uv, c.ws_d, c.out)
        out_pin.copy_(c.out, non_blocking=True)
        b.record()
        b.synchronize()
        e2e_ms.append(a.elapsed_time(b))
    e2e_step = max_over_ranks(statistics.fmean(e2e_ms), world, dev)
    err = mla.mla_get_device_error()
    if err != 0:
        raise RuntimeError(f"device error in the e2e loop: {mla.mla_status_string(err)}")
    return {"value": job_rate(c.work["units"], e2e_step, world), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_step}


def launches_per_step(w: WL.Workload) -> int:
    """The library's kernel launches in one step: append GEMM + finish, query absorption,
    attention, merge + value projection; a quantised cache adds the query split."""
    return 6 if w.kv == "fp8" else 5


def run_ours(args, rank: int, world: int, local_rank: int):
    import head_latent_attention_05_b200 as mla

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = WL.get(args.workload)
    K, Wm = args.steps, max(3, args.warmup)
    flush_l2 = L2Flush(dev)
    c = DeviceCase(mla, w, dev)
    m = measure_device(c, flush_l2, K, Wm, world, not args.no_graph, local_rank)
    e2e = measure_e2e(c, flush_l2, K, world)
    work = c.work

    line = {
        "metric": METRIC, "value": m["value"], "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": Wm, "ms_per_step": m["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": w.name, "batch_per_gpu": w.B, "global_batch": w.B * world,
                   "heads": w.H, "tq": w.Tq, "context": list(w.lens),
                   "cache_tokens_per_gpu": work["tokens"], "parallelism": f"dp{world}",
                   "l2": "flushed before every step, outside the step events: 256 MiB write, then a "
                         "256 MiB read that drains the written lines",
                   "timing": ("CUDA graph of the K steps" if not args.no_graph else "eager")
                   + "; kernel_ms and the roofline's kernel time from a second replay of the same"
                   " steps with event marks between the kernels",
                   "step": "mla_append_latent + mla_decode"},
        "roofline": m["roofline"],
        "kernel_ms": m["kernel_ms"],
        "decode_only": m["decode_only"],
        "e2e": e2e,
        "gpu_launches": K * launches_per_step(w),
        "clocks": m["clocks"],
        "wall_s_timed_region": m["wall"],
    }
    cpu_case = (c.lens, c.pt, c.weights, c.cache_host, c.x_new_h, c.pos_h, c.q_h)
    del c

    # the other bench-relevant workloads (the batch-16 x 4096 V2 shape, the 32-head module
    # shape, the tensor-bound long-context case, the quantised-cache mix), each with its own
    # attention roofline (fewer steps); one that fails is reported as such, the headline stands
    if not args.no_extra:
        extra = {}
        for name in EXTRA_WORKLOADS:
            if name == w.name:
                continue
            try:
                ce = DeviceCase(mla, WL.get(name), dev)
                me = measure_device(ce, flush_l2, min(K, args.extra_steps), Wm, world,
                                    not args.no_graph, local_rank)
                extra[name] = {"value": me["value"], "unit": UNIT,
                               "ms_per_step": me["ms_per_step"],
                               "steps": min(K, args.extra_steps), "roofline": me["roofline"],
                               "kernel_ms": me["kernel_ms"], "decode_only": me["decode_only"],
                               "clocks": me["clocks"],
                               "gpu_launches": min(K, args.extra_steps) * launches_per_step(ce.w)}
                del ce
            except Exception as e:   # reported in the line, never silently dropped
                extra[name] = {"error": f"{type(e).__name__}: {e}"}
            torch.cuda.empty_cache()
        line["other_workloads"] = extra

    if world == 1 and not args.no_extra:
        line["layer_calls"] = measure_layer_calls(mla, dev, flush_l2, min(K, 20))

    if rank == 0 and world == 1 and not args.no_cpu_baseline and w.kv == "plain":
        lens, pt, weights, cache_host, x_new_h, pos_h, q_h = cpu_case
        threading = ("serial loop over (sequence, head) units; cores = the BLAS thread count that "
                     "numpy's matrix products may use inside one unit")
        rate, units, desc = oracle_sample(w, lens, pt, weights, cache_host, x_new_h, pos_h, q_h,
                                          args.cpu_seconds)
        line["cpu_baseline"] = {"value": rate, "unit": UNIT, "cores": cpu_threads(),
                                "kind": "oracle", "sample": desc, "threading": threading}
        # the same oracle's absorbed (latent-space) form, a second CPU number
        rate_a, _, desc_a = oracle_sample(w, lens, pt, weights, cache_host, x_new_h, pos_h, q_h,
                                          args.cpu_seconds / 3, form="absorbed")
        line["cpu_baseline_absorbed"] = {"value": rate_a, "unit": UNIT, "cores": cpu_threads(),
                                         "kind": "oracle", "sample": desc_a,
                                         "threading": threading}
    if rank == 0:
        print(json.dumps(line), flush=True)


def graph_time_ms(fn, flush_l2, K: int, dev) -> float:
    """Mean device time of fn() over K calls captured in one CUDA graph, each after an L2 flush
    that lies outside its events (3 eager warm-up calls first)."""
    ev = lambda: torch.cuda.Event(enable_timing=True, external=True)
    evs = [(ev(), ev()) for _ in range(K)]
    for a, b in evs:
        a.record()
        b.record()
    for i in range(3):
        flush_l2(i)
        fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream(device=dev)
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            for i in range(K):
                flush_l2(i * 7)
                evs[i][0].record()
                fn()
                evs[i][1].record()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    ms = statistics.fmean(a.elapsed_time(b) for a, b in evs)
    del g
    return ms


def measure_layer_calls(mla, dev, flush_l2, K: int) -> dict:
    """Device times of the layer's other calls at DeepSeek-V2 shape, each against its own
    roofline: the q path and the output projection for the 16 query tokens of a batch-16
    decode step (weight-streaming, HBM-bound), a tensor-core prefill of 2 prompts of 256 tokens
    (tensor-bound) and a windowed decode (window 1024) of 16 sequences of 4096 tokens. Each
    item is measured on its own; one that fails reports its error."""
    pk, _ = peaks()
    hbm, tc = float(pk["hbm_gbs"]), float(pk["bf16_tflops"])
    bf = torch.bfloat16
    res = {}
    w = WL.get("v2_bf16_b16_ctx4096")
    cfg = mla.make_config(w.H, w.d_model, w.d_c, w.d_r, w.d_nope, w.d_v, WL.PAGE_SIZE, w.dtype,
                          w.scale, w.rms_eps, w.rope_theta)
    n = w.B * w.Tq
    try:
        wt = WL.weights(w)
        x = WL.randn((n, w.d_model), w.seed, 40, 1.0, bf).to(dev)
        w_qa, q_gain, w_qb = wt.w_qa.to(dev), wt.q_gain.to(dev), wt.w_qb.to(dev)
        q_out = torch.empty((n, w.H, w.d_nope + w.d_r), dtype=bf, device=dev)
        ws = mla.workspace(mla.mla_query_workspace_size(cfg, w.q_lora, n), dev)
        ms = graph_time_ms(lambda: mla.mla_query(cfg, x, w_qa, q_gain, w_qb, ws, q_out), flush_l2, K, dev)
        nbytes = 2 * (w_qa.numel() + w_qb.numel() + x.numel() + q_out.numel())
        res["query"] = {"what": f"mla_query, {n} tokens: wq_a, q_norm, wq_b", "ms_per_call": ms,
                        "bound": "hbm", "algorithmic_bytes": nbytes,
                        "roofline_frac": nbytes / (ms / 1e3) / 1e9 / hbm}
        del wt, x, w_qa, q_gain, w_qb, q_out, ws
    except Exception as e:
        res["query"] = {"error": f"{type(e).__name__}: {e}"}
    try:
        attn = WL.randn((n, w.H, w.d_v), w.seed, 41, 1.0, bf).to(dev)
        w_o = WL.output_weight(w).to(dev)
        y = torch.empty((n, w.d_model), dtype=bf, device=dev)
        ws = mla.workspace(mla.mla_output_workspace_size(cfg, n), dev)
        ms = graph_time_ms(lambda: mla.mla_output(cfg, attn, w_o, ws, y), flush_l2, K, dev)
        nbytes = 2 * (w_o.numel() + attn.numel() + y.numel())
        res["output"] = {"what": f"mla_output, {n} tokens: wo", "ms_per_call": ms, "bound": "hbm",
                         "algorithmic_bytes": nbytes,
                         "roofline_frac": nbytes / (ms / 1e3) / 1e9 / hbm}
        del attn, w_o, y, ws
    except Exception as e:
        res["output"] = {"error": f"{type(e).__name__}: {e}"}
    try:
        B, T = 2, 256
        wp = WL.small_variant(WL.get("v2_bf16_b16_ctx4096"), B=B, Tq=T, lens=("fixed", T))
        lens = WL.seq_lens(wp)
        pt = WL.page_table(wp, lens)
        wt = WL.weights(wp)
        cache = WL.cache_pool(wp, pt.num_pages).to(dev)
        x_new, _, _, q = WL.new_token_inputs(wp, lens)
        x = x_new.view(B, T, wp.d_model).to(dev)
        q = q.contiguous().to(dev)
        w_uk_t = torch.empty((wp.H, wp.d_c, wp.d_nope), dtype=bf, device=dev)
        w_uv = torch.empty((wp.H, wp.d_v, wp.d_c), dtype=bf, device=dev)
        mla.mla_absorb_weights(cfg, wt.wkv_b.to(dev), w_uk_t, w_uv)
        w_dkv, kv_gain = wt.w_dkv.to(dev), wt.kv_gain.to(dev)
        bt, sl = pt.block_table.to(dev), lens.to(dev)
        out = torch.empty((B, T, wp.H, wp.d_v), dtype=bf, device=dev)
        ws = mla.workspace(mla.mla_prefill_workspace_size(cfg, B, T), dev)
        ms = graph_time_ms(lambda: mla.mla_prefill(cfg, x, q, w_dkv, kv_gain, w_uk_t, w_uv, sl, bt,
                                                   cache, ws, out), flush_l2, K, dev)
        n_tok = B * T
        flops = (wp.H * 2 * (wp.row + wp.d_c) * B * T * (T + 1) // 2     # causal attention
                 + 2 * n_tok * wp.row * wp.d_model                         # down-projection
                 + 2 * 2 * n_tok * wp.H * wp.d_nope * wp.d_c)              # W_UK and W_UV
        res["prefill"] = {"what": f"mla_prefill, {B} prompts of {T} tokens (append, absorbed "
                                  "query, causal latent attention, W_UV)",
                          "ms_per_call": ms, "prompt_tokens_per_s": n_tok / (ms / 1e3),
                          "bound": "tensor", "algorithmic_flops": flops,
                          "roofline_frac": flops / (ms / 1e3) / 1e12 / tc}
        del cache, x, q, w_uk_t, w_uv, w_dkv, kv_gain, bt, sl, out, ws, wt
    except Exception as e:
        res["prefill"] = {"error": f"{type(e).__name__}: {e}"}
    try:
        ww = WL.get("v2_bf16_b16_ctx4096")
        cw = DeviceCase(mla, ww, dev)
        cw.cfg.window = 1024
        mla.mla_append_latent(cw.cfg, cw.x_new, cw.w_dkv, cw.kv_gain, cw.seq_idx, cw.pos, cw.bt,
                              cw.cache, cw.ws_a)
        ms = graph_time_ms(cw.decode, flush_l2, K, dev)
        keys = sum(min(int(L), 1024) for L in cw.lens.tolist())
        nbytes = keys * ww.row * 2
        res["window_decode"] = {"what": "mla_decode, 16 sequences of 4096 tokens, window 1024",
                                "ms_per_call": ms,
                                "value": keys * ww.Tq * ww.H / (ms / 1e3), "unit": UNIT,
                                "bound": "hbm", "algorithmic_bytes": nbytes + cw.work["weight_bytes"],
                                "roofline_frac": (nbytes + cw.work["weight_bytes"]) / (ms / 1e3) / 1e9 / hbm}
        del cw
    except Exception as e:
        res["window_decode"] = {"error": f"{type(e).__name__}: {e}"}
    torch.cuda.empty_cache()
    return res


def stored_traffic(workload: str):
    """DRAM bytes per launch of the attention kernel from the committed ncu capture of this
    workload, while the kernel's code still matches the one measured; else None."""
    if not os.path.exists(ATTN_PROFILE):
        return None
    with open(ATTN_PROFILE) as f:
        prof = json.load(f)
    sha = kernel_sha(fp8=WL.get(workload).kv == "fp8")
    for e in prof.get("captures", []):
        if e.get("workload") == workload and e.get("kernel_source_sha") == sha:
            return e.get("dram_bytes_per_launch")
    return None


def kernel_sha(fp8: bool = False) -> str:
    """Hash of the attention kernel's code (its source with // comments and blank lines
    dropped), to tell whether stored counters are still current. The quantised-cache kernel
    is hashed together with the file it builds on."""
    import hashlib
    import re
    files = ["tc_decode.cuh"] + (["tc_decode_fp8.cuh", "fp8_cache.cuh"] if fp8 else [])
    code = ""
    for name in files:
        path = os.path.join(ROOT, "head_latent_attention_05_b200", "csrc", name)
        with open(path, encoding="utf-8") as f:
            lines = [re.sub(r"//.*", "", ln).rstrip() for ln in f]
        code += "\n".join(ln for ln in lines if ln.strip())
    return hashlib.sha256(code.encode()).hexdigest()[:16]


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the library has no CPU path)")
    from head_latent_attention_05_b200 import build as _b
    if rank == 0 or world == 1:
        _b.build()
    if world > 1:
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group(
            "nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local_rank))
        torch.distributed.barrier()
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
