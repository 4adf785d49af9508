"""Python binding of libmla.so (MLA decode over a paged latent KV cache on B200).

The functions below carry the names of the C ABI in include/mla.h and only marshal arguments:
torch tensors are passed as raw device pointers with the current CUDA stream, and a non-zero
status raises MlaError. All computation happens in the CUDA library; there is no fallback.
If libmla.so has not been built, importing works but every call raises.
"""

from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmla.so")

MLA_DTYPE_F32 = 0
MLA_DTYPE_BF16 = 1
MLA_KV_PLAIN = 0
MLA_KV_FP8_E4M3 = 1

STATUS = {
    0: "MLA_OK", 1: "MLA_ERR_INVALID_ARG", 2: "MLA_ERR_UNSUPPORTED",
    3: "MLA_ERR_WORKSPACE_TOO_SMALL", 4: "MLA_ERR_CUDA", 5: "MLA_ERR_DEVICE_TIMEOUT",
    6: "MLA_ERR_DEVICE_OOB", 7: "MLA_ERR_DEVICE_BAD_LENGTH",
}

# Every symbol include/mla.h declares (checked by the tests against the built library).
EXPORTED = (
    "mla_status_string", "mla_absorb_weights", "mla_append_workspace_size", "mla_append_latent",
    "mla_decode_workspace_size", "mla_decode", "mla_decode_profiled", "mla_decode_noalloc",
    "mla_prefill_ref_workspace_size",
    "mla_prefill_ref", "mla_get_device_error", "mla_query_workspace_size", "mla_query",
    "mla_output_workspace_size", "mla_output", "mla_decode_partial", "mla_combine_workspace_size",
    "mla_combine", "mla_prefill_workspace_size", "mla_prefill", "mla_quantize_latent",
)


class MlaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS.get(code, code)}")


class MlaConfig(ctypes.Structure):
    _fields_ = [
        ("n_heads", ctypes.c_int32), ("d_model", ctypes.c_int32), ("d_c", ctypes.c_int32),
        ("d_rope", ctypes.c_int32), ("d_nope", ctypes.c_int32), ("d_v", ctypes.c_int32),
        ("page_size", ctypes.c_int32), ("dtype", ctypes.c_int32),
        ("softmax_scale", ctypes.c_float), ("rms_eps", ctypes.c_float),
        ("rope_theta", ctypes.c_float), ("window", ctypes.c_int32),
        ("kv_format", ctypes.c_int32),
    ]


def make_config(n_heads, d_model, d_c, d_rope, d_nope, d_v, page_size=64, dtype="bf16",
                softmax_scale=None, rms_eps=1e-6, rope_theta=10000.0, window=0,
                kv_format="plain") -> MlaConfig:
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d_nope + d_rope)
    dt = {"bf16": MLA_DTYPE_BF16, "f32": MLA_DTYPE_F32,
          torch.bfloat16: MLA_DTYPE_BF16, torch.float32: MLA_DTYPE_F32}[dtype]
    kf = {"plain": MLA_KV_PLAIN, "fp8": MLA_KV_FP8_E4M3}[kv_format]
    return MlaConfig(n_heads, d_model, d_c, d_rope, d_nope, d_v, page_size, dt,
                     softmax_scale, rms_eps, rope_theta, window, kf)


def fp8_page_bytes(cfg: MlaConfig) -> int:
    """Bytes of one page of a quantised cache: page_size rows of d_c + d_rope codes, then the
    page_size float32 scales (include/mla.h, mla_kv_format)."""
    return cfg.page_size * (cfg.d_c + cfg.d_rope + 4)


def fp8_cache_views(cfg: MlaConfig, cache: torch.Tensor):
    """(codes [num_pages, page_size, d_c + d_rope] uint8, scales [num_pages, page_size] float32):
    views of a quantised cache held as a uint8 tensor [num_pages, fp8_page_bytes(cfg)]."""
    row, ps = cfg.d_c + cfg.d_rope, cfg.page_size
    codes = cache[:, :ps * row].view(cache.shape[0], ps, row)
    scales = cache[:, ps * row:].view(torch.float32)
    return codes, scales


_lib = None


def use_library(path: str) -> None:
    """Load the C ABI from another build of the same sources (e.g. the short-wait test build)
    for the calls that follow; use_library(LIB_PATH) goes back to the product library. Each
    library keeps its own device error word."""
    global LIB_PATH, _lib
    LIB_PATH = path
    _lib = None
    load_library()


def load_library() -> ctypes.CDLL:
    """Load libmla.so from the package directory; raise if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python head_latent_attention_05_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, SZ, CFG = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t, ctypes.POINTER(MlaConfig)
    sig = {
        "mla_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "mla_absorb_weights": (ctypes.c_int, [CFG, P, P, P, P]),
        "mla_append_workspace_size": (SZ, [CFG, I32]),
        "mla_append_latent": (ctypes.c_int, [CFG, P, I32, P, P, P, P, P, I32, I32, P, I32, P, SZ, P]),
        "mla_decode_workspace_size": (SZ, [CFG, I32, I32]),
        "mla_decode": (ctypes.c_int, [CFG, P, I32, I32, P, I32, P, I32, P, P, P, P, SZ, P, P]),
        "mla_decode_profiled": (ctypes.c_int,
                                [CFG, P, I32, I32, P, I32, P, I32, P, P, P, P, SZ, P, P, P]),
        "mla_decode_noalloc": (ctypes.c_int, [CFG, P, I32, I32, P, I32, P, I32, P, P, P, P, P]),
        "mla_prefill_ref_workspace_size": (SZ, [CFG, I32, I32]),
        "mla_prefill_ref": (ctypes.c_int, [CFG, P, P, I32, I32, P, P, P, P, P, P, I32, P, I32, P, SZ, P, P]),
        "mla_get_device_error": (ctypes.c_int, [P]),
        "mla_query_workspace_size": (SZ, [CFG, I32, I32]),
        "mla_query": (ctypes.c_int, [CFG, I32, P, I32, P, P, P, P, SZ, P, P]),
        "mla_output_workspace_size": (SZ, [CFG, I32]),
        "mla_output": (ctypes.c_int, [CFG, P, I32, P, P, SZ, P, P]),
        "mla_decode_partial": (ctypes.c_int, [CFG, P, I32, I32, P, I32, P, I32, P, P, P, P, P, SZ,
                                              P, P, P]),
        "mla_combine_workspace_size": (SZ, [CFG, I32, I32]),
        "mla_combine": (ctypes.c_int, [CFG, I32, I32, I32, P, P, P, P, SZ, P, P]),
        "mla_prefill_workspace_size": (SZ, [CFG, I32, I32]),
        "mla_prefill": (ctypes.c_int, [CFG, P, P, I32, I32, P, P, P, P, P, P, I32, P, I32, P, SZ,
                                       P, P]),
        "mla_quantize_latent": (ctypes.c_int, [CFG, P, I32, P, P, P, I32, I32, P, I32, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    _lib = lib
    return lib


def _ptr(t: torch.Tensor):
    if not t.is_contiguous():
        raise ValueError("tensors passed to libmla must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(code: int, where: str):
    if code != 0:
        raise MlaError(code, where)


def mla_status_string(code: int) -> str:
    return load_library().mla_status_string(code).decode()


def mla_absorb_weights(cfg: MlaConfig, wkv_b, w_uk_t, w_uv, stream=None):
    _check(load_library().mla_absorb_weights(ctypes.byref(cfg), _ptr(wkv_b), _ptr(w_uk_t),
                                             _ptr(w_uv), _stream(stream)), "mla_absorb_weights")


def mla_append_workspace_size(cfg: MlaConfig, n_tok: int) -> int:
    return int(load_library().mla_append_workspace_size(ctypes.byref(cfg), n_tok))


def mla_append_latent(cfg: MlaConfig, x, w_dkv, kv_gain, seq_idx, pos, block_table, cache,
                      workspace, stream=None):
    batch, max_pages = block_table.shape
    _check(load_library().mla_append_latent(
        ctypes.byref(cfg), _ptr(x), x.shape[0], _ptr(w_dkv), _ptr(kv_gain), _ptr(seq_idx),
        _ptr(pos), _ptr(block_table), batch, max_pages, _ptr(cache), cache.shape[0],
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)),
        "mla_append_latent")


def mla_quantize_latent(cfg: MlaConfig, rows, seq_idx, pos, block_table, cache, stream=None):
    """Quantise float32 rows [n_tok, d_c + d_rope] into their slots of a quantised cache."""
    batch, max_pages = block_table.shape
    _check(load_library().mla_quantize_latent(
        ctypes.byref(cfg), _ptr(rows), rows.shape[0], _ptr(seq_idx), _ptr(pos), _ptr(block_table),
        batch, max_pages, _ptr(cache), cache.shape[0], _stream(stream)), "mla_quantize_latent")


def mla_decode_workspace_size(cfg: MlaConfig, batch: int, tq: int) -> int:
    return int(load_library().mla_decode_workspace_size(ctypes.byref(cfg), batch, tq))


def mla_decode(cfg: MlaConfig, q, cache, block_table, seq_lens, w_uk_t, w_uv, workspace, out,
               stream=None):
    batch, tq = q.shape[0], q.shape[1]
    _check(load_library().mla_decode(
        ctypes.byref(cfg), _ptr(q), batch, tq, _ptr(cache), cache.shape[0], _ptr(block_table),
        block_table.shape[1], _ptr(seq_lens), _ptr(w_uk_t), _ptr(w_uv), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(out), _stream(stream)), "mla_decode")


def mla_decode_profiled(cfg: MlaConfig, q, cache, block_table, seq_lens, w_uk_t, w_uv,
                        workspace, out, events, stream=None):
    """mla_decode that also records 4 torch.cuda.Event objects at its kernel boundaries
    (before the query absorption, the attention, the merge + value projection, and after).

    The events must already exist on the device (torch creates them lazily: record each once
    before the first call). Create them with external=True to time inside a CUDA graph."""
    if len(events) != 4 or any(e.cuda_event == 0 for e in events):
        raise ValueError("mla_decode_profiled needs 4 already-created CUDA events")
    arr = (ctypes.c_void_p * 4)(*[ctypes.c_void_p(e.cuda_event) for e in events])
    batch, tq = q.shape[0], q.shape[1]
    _check(load_library().mla_decode_profiled(
        ctypes.byref(cfg), _ptr(q), batch, tq, _ptr(cache), cache.shape[0], _ptr(block_table),
        block_table.shape[1], _ptr(seq_lens), _ptr(w_uk_t), _ptr(w_uv), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(out), _stream(stream), arr),
        "mla_decode_profiled")


# Bytes of the library's built-in scratch used by mla_decode_noalloc.
MLA_DECODE_NOALLOC_MAX_SCRATCH = 32 << 20


def mla_decode_noalloc(cfg: MlaConfig, q, cache, block_table, seq_lens, w_uk_t, w_uv, out,
                       stream=None):
    """mla_decode without a workspace argument: the scratch is a fixed device array inside the
    library (see include/mla.h), for callers that cannot allocate device memory."""
    batch, tq = q.shape[0], q.shape[1]
    _check(load_library().mla_decode_noalloc(
        ctypes.byref(cfg), _ptr(q), batch, tq, _ptr(cache), cache.shape[0], _ptr(block_table),
        block_table.shape[1], _ptr(seq_lens), _ptr(w_uk_t), _ptr(w_uv), _ptr(out),
        _stream(stream)), "mla_decode_noalloc")


def mla_prefill_ref_workspace_size(cfg: MlaConfig, batch: int, t_new: int) -> int:
    return int(load_library().mla_prefill_ref_workspace_size(ctypes.byref(cfg), batch, t_new))


def mla_prefill_ref(cfg: MlaConfig, x, q, w_dkv, kv_gain, w_uk_t, w_uv, seq_lens, block_table,
                    cache, workspace, out, stream=None):
    batch, t_new = q.shape[0], q.shape[1]
    _check(load_library().mla_prefill_ref(
        ctypes.byref(cfg), _ptr(x), _ptr(q), batch, t_new, _ptr(w_dkv), _ptr(kv_gain),
        _ptr(w_uk_t), _ptr(w_uv), _ptr(seq_lens), _ptr(block_table), block_table.shape[1],
        _ptr(cache), cache.shape[0], _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(out), _stream(stream)),
        "mla_prefill_ref")


def mla_query_workspace_size(cfg: MlaConfig, q_lora: int, n_tok: int) -> int:
    return int(load_library().mla_query_workspace_size(ctypes.byref(cfg), q_lora, n_tok))


def mla_query(cfg: MlaConfig, x, w_qa, q_gain, w_qb, workspace, q_out, stream=None):
    """q path: q_out [n_tok, H, d_nope + d_rope] from hidden states x [n_tok, d_model]."""
    n_tok, q_lora = x.shape[0], w_qa.shape[0]
    _check(load_library().mla_query(
        ctypes.byref(cfg), q_lora, _ptr(x), n_tok, _ptr(w_qa), _ptr(q_gain), _ptr(w_qb),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(q_out),
        _stream(stream)), "mla_query")


def mla_output_workspace_size(cfg: MlaConfig, n_tok: int) -> int:
    return int(load_library().mla_output_workspace_size(ctypes.byref(cfg), n_tok))


def mla_output(cfg: MlaConfig, attn, w_o, workspace, y, stream=None):
    """Output projection: y [n_tok, d_model] from attention outputs attn [n_tok, H, d_v]."""
    _check(load_library().mla_output(
        ctypes.byref(cfg), _ptr(attn), attn.shape[0], _ptr(w_o), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(y), _stream(stream)), "mla_output")


def mla_decode_partial(cfg: MlaConfig, q, cache, block_table, seq_lens, kv_begin, kv_end, w_uk_t,
                       workspace, o_part, lse, stream=None):
    """Decode over keys kv_begin[b] <= j < kv_end[b] only: o_part [B*Tq*H, d_c] (O / l) and
    lse [B*Tq*H] (natural log), to be merged with other ranges' partials by mla_combine."""
    batch, tq = q.shape[0], q.shape[1]
    _check(load_library().mla_decode_partial(
        ctypes.byref(cfg), _ptr(q), batch, tq, _ptr(cache), cache.shape[0], _ptr(block_table),
        block_table.shape[1], _ptr(seq_lens), _ptr(kv_begin), _ptr(kv_end), _ptr(w_uk_t),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(o_part), _ptr(lse),
        _stream(stream)), "mla_decode_partial")


def mla_combine_workspace_size(cfg: MlaConfig, batch: int, tq: int) -> int:
    return int(load_library().mla_combine_workspace_size(ctypes.byref(cfg), batch, tq))


def mla_combine(cfg: MlaConfig, o_parts, lse_parts, w_uv, workspace, out, stream=None):
    """Merge n_parts partials (o_parts [n_parts, B*Tq*H, d_c], lse_parts [n_parts, B*Tq*H]) and
    project into out [B, Tq, H, d_v]."""
    n_parts, batch, tq = o_parts.shape[0], out.shape[0], out.shape[1]
    ws = workspace if workspace is not None else torch.empty(0, dtype=torch.uint8)
    _check(load_library().mla_combine(
        ctypes.byref(cfg), n_parts, batch, tq, _ptr(o_parts), _ptr(lse_parts), _ptr(w_uv),
        ctypes.c_void_p(ws.data_ptr()) if ws.numel() else None, ws.numel() * ws.element_size(),
        _ptr(out), _stream(stream)), "mla_combine")


def mla_prefill_workspace_size(cfg: MlaConfig, batch: int, t_new: int) -> int:
    return int(load_library().mla_prefill_workspace_size(ctypes.byref(cfg), batch, t_new))


def mla_prefill(cfg: MlaConfig, x, q, w_dkv, kv_gain, w_uk_t, w_uv, seq_lens, block_table, cache,
                workspace, out, stream=None):
    """Tensor-core prefill: same arguments and results as mla_prefill_ref."""
    batch, t_new = q.shape[0], q.shape[1]
    _check(load_library().mla_prefill(
        ctypes.byref(cfg), _ptr(x), _ptr(q), batch, t_new, _ptr(w_dkv), _ptr(kv_gain),
        _ptr(w_uk_t), _ptr(w_uv), _ptr(seq_lens), _ptr(block_table), block_table.shape[1],
        _ptr(cache), cache.shape[0], _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(out), _stream(stream)), "mla_prefill")


def mla_get_device_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the library's device error code."""
    return int(load_library().mla_get_device_error(_stream(stream)))


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A 256-byte-aligned byte buffer of at least nbytes (torch's allocator aligns to 512)."""
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)
