"""Python binding of libmla: MLA latent-KV decode on B200 (sm_100a).

Argument marshalling only: every function here forwards torch tensors (device memory owned
by the caller) and integers to the C ABI of the same name in ``include/mla.h`` and raises
``MlaError`` on a non-OK status.  All computation happens in the library's CUDA kernels;
there is no fallback: importing works without a GPU, but calling anything needs the built
``libmla.so`` (``python -m mla_latent_kv_24_b200.build``) and a CUDA device.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np

__all__ = [
    "MlaError", "mla_dims", "make_dims", "load", "LIB_PATH", "STATUS",
    "mla_cache_append", "mla_decode_workspace_size", "mla_decode_absorbed",
    "gqla_expand_cache", "gqla_decode_workspace_size", "gqla_decode_grouped",
    "mla_get_device_status", "mla_last_error_string", "mla_version", "mla_set_profile_events",
    "mla_decode_absorbed_noalloc", "NOALLOC_SCRATCH_BYTES", "EXPORTED_SYMBOLS", "mla_select_path",
    "mla_prefill_workspace_size", "mla_prefill_expanded", "gqla_expand_tokens", "mla_debug_decode_fault",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmla.so")

STATUS = {0: "MLA_OK", 1: "MLA_ERR_INVALID_ARG", 2: "MLA_ERR_UNSUPPORTED", 3: "MLA_ERR_WORKSPACE",
          4: "MLA_ERR_CUDA", 5: "MLA_ERR_DEVICE_BOUNDS", 6: "MLA_ERR_TIMEOUT"}
MLA_BF16, MLA_FP32 = 0, 1

EXPORTED_SYMBOLS = ["mla_cache_append", "mla_decode_workspace_size", "mla_decode_absorbed",
                    "gqla_expand_cache", "gqla_decode_workspace_size", "gqla_decode_grouped",
                    "mla_get_device_status", "mla_last_error_string", "mla_version", "mla_set_profile_events",
                    "mla_decode_absorbed_noalloc", "mla_select_path", "mla_prefill_workspace_size",
                    "mla_prefill_expanded", "gqla_expand_tokens", "mla_debug_decode_fault"]
NOALLOC_SCRATCH_BYTES = 32 << 20


class MlaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


class mla_dims(ctypes.Structure):
    _fields_ = [("n_heads", ctypes.c_int32), ("heads_per_group", ctypes.c_int32), ("d_c", ctypes.c_int32),
                ("d_rope", ctypes.c_int32), ("d_nope", ctypes.c_int32), ("d_v", ctypes.c_int32),
                ("page_size", ctypes.c_int32), ("softmax_scale", ctypes.c_float), ("rope_base", ctypes.c_float),
                ("dtype", ctypes.c_int32)]


def make_dims(n_heads=128, heads_per_group=1, d_c=512, d_rope=64, d_nope=128, d_v=128, page_size=64,
              softmax_scale=0.0, rope_base=10000.0, dtype="bf16") -> mla_dims:
    return mla_dims(n_heads, heads_per_group, d_c, d_rope, d_nope, d_v, page_size, softmax_scale, rope_base,
                    MLA_BF16 if dtype == "bf16" else MLA_FP32)


_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int32
_S = ctypes.c_size_t


def load() -> ctypes.CDLL:
    """Loads libmla.so (once).  Raises ImportError if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m mla_latent_kv_24_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    D = ctypes.POINTER(mla_dims)
    sig = {
        "mla_cache_append": [D, _P, _I, _P, _P, _P, _P, _I, _P, _I, _I, _I, _P, _P],
        "mla_decode_workspace_size": [D, _I, _I, _P, ctypes.POINTER(_S)],
        "mla_decode_absorbed": [D, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _S, _P],
        "gqla_expand_cache": [D, _P, _P, _P, _P, _I, _I, _P, _P],
        "gqla_expand_tokens": [D, _P, _P, _P, _P, _P, _I, _P, _I, _I, _I, _P, _P],
        "gqla_decode_workspace_size": [D, _I, _I, _P, ctypes.POINTER(_S)],
        "gqla_decode_grouped": [D, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _S, _P],
        "mla_get_device_status": [_P],
        "mla_last_error_string": [],
        "mla_version": [],
        "mla_set_profile_events": [_P, _P],
        "mla_decode_absorbed_noalloc": [D, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P],
        "mla_select_path": [D, _I, _I, _P, ctypes.c_double, ctypes.c_double, _I, ctypes.POINTER(ctypes.c_int),
                            ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double)],
        "mla_prefill_workspace_size": [D, _I, _I, _P, ctypes.POINTER(_S)],
        "mla_prefill_expanded": [D, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _S, _P],
        "mla_debug_decode_fault": [_I, ctypes.c_uint32],
    }
    for name, args in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = ctypes.c_char_p if name == "mla_last_error_string" else ctypes.c_int
    _lib = lib
    return lib


def _check(status: int):
    if status != 0:
        raise MlaError(status, load().mla_last_error_string().decode())


def _dev(t) -> Optional[int]:
    """Device address of a CUDA tensor (None stays NULL)."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def _host_i32(x: Sequence[int]):
    a = np.ascontiguousarray(np.asarray(x, dtype=np.int32))
    return a, a.ctypes.data_as(ctypes.c_void_p)


def mla_cache_append(dims, h, hidden, W_dkv, W_kr, req_idx, positions, n_tok, page_table, batch, max_pages,
                     n_pages_total, latent_cache, stream=None) -> None:
    _check(load().mla_cache_append(ctypes.byref(dims), _dev(h), hidden, _dev(W_dkv), _dev(W_kr), _dev(req_idx),
                                   _dev(positions), n_tok, _dev(page_table), batch, max_pages, n_pages_total,
                                   _dev(latent_cache), _stream(stream)))


def mla_decode_workspace_size(dims, batch, s_q, seq_lens_host) -> int:
    arr, p = _host_i32(seq_lens_host)
    out = _S(0)
    _check(load().mla_decode_workspace_size(ctypes.byref(dims), batch, s_q, p, ctypes.byref(out)))
    return out.value


def gqla_decode_workspace_size(dims, batch, s_q, seq_lens_host) -> int:
    arr, p = _host_i32(seq_lens_host)
    out = _S(0)
    _check(load().gqla_decode_workspace_size(ctypes.byref(dims), batch, s_q, p, ctypes.byref(out)))
    return out.value


def mla_decode_absorbed(dims, q, W_uk, W_uv, latent_cache, page_table, seq_lens, seq_lens_host, batch, s_q,
                        max_pages, n_pages_total, out, workspace, workspace_bytes=None, stream=None) -> None:
    arr, p = _host_i32(seq_lens_host)
    nbytes = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    _check(load().mla_decode_absorbed(ctypes.byref(dims), _dev(q), _dev(W_uk), _dev(W_uv), _dev(latent_cache),
                                      _dev(page_table), _dev(seq_lens), p, batch, s_q, max_pages, n_pages_total,
                                      _dev(out), _dev(workspace), nbytes, _stream(stream)))


def gqla_expand_cache(dims, W_uk, W_uv, latent_cache, page_ids, n_ids, n_pages_total, expanded_cache,
                      stream=None) -> None:
    _check(load().gqla_expand_cache(ctypes.byref(dims), _dev(W_uk), _dev(W_uv), _dev(latent_cache), _dev(page_ids),
                                    n_ids, n_pages_total, _dev(expanded_cache), _stream(stream)))


def gqla_expand_tokens(dims, W_uk, W_uv, latent_cache, req_idx, positions, n_tok, page_table, batch, max_pages,
                       n_pages_total, expanded_cache, stream=None) -> None:
    _check(load().gqla_expand_tokens(ctypes.byref(dims), _dev(W_uk), _dev(W_uv), _dev(latent_cache), _dev(req_idx),
                                     _dev(positions), n_tok, _dev(page_table), batch, max_pages, n_pages_total,
                                     _dev(expanded_cache), _stream(stream)))


def gqla_decode_grouped(dims, q, expanded_cache, latent_cache, page_table, seq_lens, seq_lens_host, batch, s_q,
                        max_pages, n_pages_total, out, workspace, workspace_bytes=None, stream=None) -> None:
    arr, p = _host_i32(seq_lens_host)
    nbytes = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    _check(load().gqla_decode_grouped(ctypes.byref(dims), _dev(q), _dev(expanded_cache), _dev(latent_cache),
                                      _dev(page_table), _dev(seq_lens), p, batch, s_q, max_pages, n_pages_total,
                                      _dev(out), _dev(workspace), nbytes, _stream(stream)))


def mla_get_device_status(stream=None) -> None:
    _check(load().mla_get_device_status(_stream(stream)))


def mla_last_error_string() -> str:
    return load().mla_last_error_string().decode()


def mla_version() -> int:
    return int(load().mla_version())


def mla_set_profile_events(start=None, stop=None) -> None:
    """Records torch.cuda.Event `start`/`stop` around the main attention kernel of later decode
    calls on this thread (None, None turns it off).  The events must already exist: record
    each once before passing it."""
    s = None if start is None else ctypes.c_void_p(start.cuda_event)
    e = None if stop is None else ctypes.c_void_p(stop.cuda_event)
    _check(load().mla_set_profile_events(s, e))


def mla_decode_absorbed_noalloc(dims, q, W_uk, W_uv, latent_cache, page_table, seq_lens, seq_lens_host, batch, s_q,
                                max_pages, n_pages_total, out, stream=None) -> None:
    """mla_decode_absorbed without a workspace argument, for callers that cannot allocate device
    memory: the library's own static scratch (NOALLOC_SCRATCH_BYTES per device) is used.  Calls
    that overlap on the GPU race on that scratch; batches that need more raise MlaError."""
    arr, p = _host_i32(seq_lens_host)
    _check(load().mla_decode_absorbed_noalloc(ctypes.byref(dims), _dev(q), _dev(W_uk), _dev(W_uv), _dev(latent_cache),
                                              _dev(page_table), _dev(seq_lens), p, batch, s_q, max_pages,
                                              n_pages_total, _dev(out), _stream(stream)))


def mla_select_path(dims, batch, s_q, seq_lens_host, hbm_bytes_per_s, flops_per_s, tp=1):
    """Roofline choice between the two decoding paths (host arithmetic only, no GPU needed).
    Returns ("absorbed" | "grouped", modelled seconds of the absorbed path, of the grouped path)."""
    lens, lp = _host_i32(seq_lens_host)
    path = ctypes.c_int(0)
    ta, tg = ctypes.c_double(0.0), ctypes.c_double(0.0)
    _check(load().mla_select_path(ctypes.byref(dims), batch, s_q, lp, float(hbm_bytes_per_s), float(flops_per_s), tp,
                                  ctypes.byref(path), ctypes.byref(ta), ctypes.byref(tg)))
    return ("grouped" if path.value == 1 else "absorbed"), ta.value, tg.value


def mla_prefill_workspace_size(dims, batch, n_q, seq_lens_host) -> int:
    arr, p = _host_i32(seq_lens_host)
    n = _S(0)
    _check(load().mla_prefill_workspace_size(ctypes.byref(dims), batch, n_q, p, ctypes.byref(n)))
    return n.value


def mla_prefill_expanded(dims, q, expanded_cache, latent_cache, page_table, seq_lens, seq_lens_host, batch, n_q,
                         max_pages, n_pages_total, out, workspace, workspace_bytes=None, stream=None) -> None:
    arr, p = _host_i32(seq_lens_host)
    nbytes = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    _check(load().mla_prefill_expanded(ctypes.byref(dims), _dev(q), _dev(expanded_cache), _dev(latent_cache),
                                       _dev(page_table), _dev(seq_lens), p, batch, n_q, max_pages, n_pages_total,
                                       _dev(out), _dev(workspace), nbytes, _stream(stream)))


def mla_debug_decode_fault(withhold_step: int, wait_us: int = 0) -> None:
    """Test hook: later tensor-core absorbed decodes on this thread withhold the completion signal
    of pipeline step `withhold_step` (-1 restores normal operation) and give up every device wait
    after `wait_us` microseconds (0: the 2 s default).  See include/mla.h."""
    _check(load().mla_debug_decode_fault(withhold_step, wait_us))
