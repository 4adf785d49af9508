"""CPU-only checks of the C ABI: the library loads, exports every function include/mla.h
declares, and rejects bad arguments on the host before launching anything."""

import ctypes
import os
import re

import pytest

import head_latent_attention_05_b200 as mla
from head_latent_attention_05_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return mla.load_library()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "mla.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mla_[a-z_]+)\s*\(", text)))


def test_header_and_binding_agree():
    assert declared_functions() == sorted(mla.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code, name in mla.STATUS.items():
        assert mla.mla_status_string(code) == name


def _cfg(**over):
    base = dict(n_heads=128, d_model=5120, d_c=512, d_rope=64, d_nope=128, d_v=128)
    base.update(over)
    return mla.make_config(**base)


FAKE = ctypes.c_void_p(0x10000)      # aligned, never dereferenced: calls fail validation first
ODD = ctypes.c_void_p(0x10008)


def _decode(lib, cfg, q=FAKE, batch=2, tq=1, ws_bytes=1 << 40, out=FAKE):
    return lib.mla_decode(ctypes.byref(cfg), q, batch, tq, FAKE, 8, FAKE, 4, FAKE, FAKE, FAKE,
                          FAKE, ws_bytes, out, None)


def test_decode_rejects_bad_arguments(lib):
    cfg = _cfg()
    assert _decode(lib, cfg, q=None) == 1                       # null pointer
    assert _decode(lib, cfg, out=ODD) == 1                      # unaligned pointer
    assert _decode(lib, cfg, batch=0) == 1
    assert _decode(lib, cfg, tq=0) == 1
    assert _decode(lib, _cfg(n_heads=0)) == 1                   # bad config
    assert _decode(lib, _cfg(d_rope=63)) == 1                   # odd rope width
    assert _decode(lib, _cfg(d_rope=130, d_c=510)) == 2         # rope wider than 128
    assert _decode(lib, _cfg(d_c=256)) == 2                     # bf16 path is V2-shaped only
    assert _decode(lib, cfg, ws_bytes=16) == 3                  # workspace too small
    assert lib.mla_decode(None, FAKE, 1, 1, FAKE, 1, FAKE, 1, FAKE, FAKE, FAKE, FAKE, 1, FAKE,
                          None) == 1


def test_append_and_prefill_reject_bad_arguments(lib):
    cfg = _cfg()
    args = [ctypes.byref(cfg), FAKE, 4, FAKE, FAKE, FAKE, FAKE, FAKE, 2, 4, FAKE, 8, FAKE, 1 << 40, None]
    bad = list(args)
    bad[2] = 0
    assert lib.mla_append_latent(*bad) == 1
    bad = list(args)
    bad[6] = None
    assert lib.mla_append_latent(*bad) == 1
    bad = list(args)
    bad[13] = 8
    assert lib.mla_append_latent(*bad) == 3
    cfg2 = _cfg(d_model=100)                                    # bf16 GEMM needs d_model % 64
    bad = list(args)
    bad[0] = ctypes.byref(cfg2)
    assert lib.mla_append_latent(*bad) == 2
    assert lib.mla_prefill_ref(ctypes.byref(cfg), FAKE, FAKE, 1, 0, FAKE, FAKE, FAKE, FAKE, FAKE,
                               FAKE, 1, FAKE, 1, FAKE, 1 << 30, FAKE, None) == 1
    assert lib.mla_absorb_weights(ctypes.byref(cfg), FAKE, None, FAKE, None) == 1


def test_workspace_sizes_are_consistent(lib):
    cfg = _cfg()
    a = mla.mla_decode_workspace_size(cfg, 16, 1)
    b = mla.mla_decode_workspace_size(cfg, 64, 1)
    assert 0 < a < b and a % 256 == 0
    assert mla.mla_decode_workspace_size(cfg, 0, 1) == 0
    assert mla.mla_decode_workspace_size(_cfg(d_c=256), 4, 1) == 0
    f32 = mla.make_config(4, 128, 64, 16, 32, 32, dtype="f32")
    assert mla.mla_decode_workspace_size(f32, 1, 1) >= (4 * (80 + 64)) * 4
    assert mla.mla_append_workspace_size(cfg, 16) >= 16 * 576 * 4
    assert mla.mla_prefill_ref_workspace_size(f32, 1, 128) > 0


def test_quantised_cache_config_is_validated(lib):
    fp8 = _cfg(kv_format="fp8")
    assert _decode(lib, fp8, q=None) == 1                       # still validates pointers
    assert _decode(lib, fp8, ws_bytes=16) == 3
    bad = _cfg()
    bad.kv_format = 2                                           # unknown row format
    assert _decode(lib, bad) == 1
    f32_fp8 = mla.make_config(4, 128, 64, 16, 32, 32, dtype="f32", kv_format="fp8")
    assert _decode(lib, f32_fp8) == 2                           # quantised cache needs bf16
    # the quantised path adds the split query rows (1152 bytes) and their scales per query row
    extra = mla.mla_decode_workspace_size(fp8, 16, 1) - mla.mla_decode_workspace_size(_cfg(), 16, 1)
    assert 16 * 128 * (1152 + 4) <= extra <= 16 * 128 * (1152 + 4) + 512
    # mla_quantize_latent: only for a quantised cache, pointers checked before any launch
    q = lambda cfg, rows=FAKE, n=4: lib.mla_quantize_latent(ctypes.byref(cfg), rows, n, FAKE, FAKE,
                                                              FAKE, 2, 4, FAKE, 8, None)
    assert q(_cfg()) == 1
    assert q(fp8, rows=None) == 1
    assert q(fp8, rows=ODD) == 1
    assert q(fp8, n=0) == 1
    # prefill_ref does not take a quantised cache
    assert lib.mla_prefill_ref(ctypes.byref(fp8), FAKE, FAKE, 1, 1, FAKE, FAKE, FAKE, FAKE, FAKE,
                               FAKE, 1, FAKE, 1, FAKE, 1 << 30, FAKE, None) == 2
    assert mla.fp8_page_bytes(fp8) == 64 * (576 + 4)
