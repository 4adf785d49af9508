"""The host logic of bench.py on CPU. With two gloo ranks: the job's step time is the slowest
rank's, the job's rate sums every rank's units, and the reference arm runs on rank 0 only (the
other ranks return at once, without work or output). And the CPU baseline's oracle sampler in
both of the oracle's forms."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r measured a step of 1 + r ms: the job took the slowest rank's time
        t = bench.max_over_ranks(1.0 + rank, world, torch.device("cpu"))
        rate = bench.job_rate(1000.0, t, world)
        out[rank] = (t, rate)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank_and_sum_the_work():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0] == res[1]
    t, rate = res[0]
    assert t == 2.0                          # slowest rank: 1 + (world - 1) ms
    assert rate == pytest.approx(world * 1000.0 / 2e-3)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5
    assert bench.job_rate(10.0, 2.0, 1) == pytest.approx(5000.0)


class _Args:   # the fields run_reference reads
    workload = "v2_bf16_b16_ctx4096"
    steps = 1
    warmup = 0
    gpus = 2


def test_reference_arm_runs_on_rank_zero_only(capsys):
    bench.run_reference(_Args(), rank=1, world=2)
    assert capsys.readouterr().out == ""


@pytest.mark.parametrize("form", ["expanded", "absorbed"])
def test_oracle_sample_times_both_forms(form):
    w = bench.WL.WORKLOADS["tiny_f32_b1_h4_ctx128"]
    lens, pt, weights, cache_host, x_new, seq_idx, pos, q = bench.build_inputs(w, "cpu")
    rate, units, desc = bench.oracle_sample(w, lens, pt, weights, cache_host, x_new, pos, q,
                                            float("inf"), max_units=3, form=form)
    assert units == 3 and rate > 0.0 and form in desc


def test_reference_arm_prints_one_json_line():
    """`bench.py --impl reference` (the fp64 oracle on the host) runs without a GPU and prints
    the contract's line: metric, value, unit, impl, cpu_baseline and a zero-copy e2e."""
    import json
    import subprocess
    import sys
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload",
                        "tiny_f32_b1_h4_ctx128", "--steps", "2", "--warmup", "1"],
                       cwd=bench.ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == bench.UNIT
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_bench_accounts_for_the_quantised_cache():
    """bench.py counts a quantised row as its codes plus one float32 scale, and one more
    launch per step (the query split)."""
    plain = bench.WL.get("v2_bf16_b64_ctx1kto32k_mix")
    fp8 = bench.WL.get("v2_fp8_b64_ctx1kto32k_mix")
    lens = torch.tensor([1000, 3000], dtype=torch.int32)
    wp, wf = bench.work_of(plain, lens), bench.work_of(fp8, lens)
    assert wp["cache_bytes"] == 4000 * 576 * 2
    assert wf["cache_bytes"] == 4000 * (576 + 4)
    assert wf["attn_flops"] == wp["attn_flops"] and wf["weight_bytes"] == wp["weight_bytes"]
    assert bench.launches_per_step(plain) == 5 and bench.launches_per_step(fp8) == 6
