"""The attention kernel's abort path: a bounded pipeline wait that runs out.

libmla_shortwait.so is the same sources with the attention kernels' pipeline waits limited to
200 ns (their drains keep the 2 s limit); both the bf16-cache and the quantised-cache kernel
are run through it. A decode through it has some wait for a TMA load or an
MMA run out: the kernel records MLA_ERR_DEVICE_TIMEOUT, drains the copies and MMAs it has in
flight, frees its tensor memory and leaves; nothing faults or hangs. The product library then
decodes the same case in the same process and matches the oracle, so the context is still
usable.
"""

import pytest
import torch

import head_latent_attention_05_b200 as mla
from head_latent_attention_05_b200 import build as B
import workloads as W
import harness as Hs

pytestmark = pytest.mark.gpu

V2 = W.WORKLOADS["v2_bf16_b16_ctx4096"]
TIMEOUT = {name: code for code, name in mla.STATUS.items()}["MLA_ERR_DEVICE_TIMEOUT"]


@pytest.mark.parametrize("kv", ["plain", "fp8"])
def test_pipeline_wait_timeout_drains_and_reports(kv):
    w = W.small_variant(V2, B=4, pages="shuffled", kv=kv)
    c = Hs.make_case(w, torch.tensor([4096, 1500, 700, 65], dtype=torch.int32))
    Hs.run_append(c)
    assert mla.mla_get_device_error() == 0
    product = mla.LIB_PATH
    short = B.build_shortwait()
    try:
        mla.use_library(short)
        Hs.run_decode(c)
        torch.cuda.synchronize()
        err = mla.mla_get_device_error()
        assert err == TIMEOUT, mla.mla_status_string(err)
    finally:
        mla.use_library(product)
    torch.cuda.synchronize()   # the context survived the abort
    out = Hs.run_decode(c).float().cpu()
    assert mla.mla_get_device_error() == 0
    new_rows = Hs.oracle_new_rows(c)
    for b in range(w.B):
        ref = Hs.oracle_out(c, b, [0, 64, 127], new_rows)
        Hs.assert_parity(out[b][:, [0, 64, 127]], ref, "bf16", f"{kv} b={b} after the abort")
