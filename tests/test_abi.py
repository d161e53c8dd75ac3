"""C-ABI library checks that need no GPU: it loads, exports every entry point include/mla.h
declares, and rejects bad arguments with the documented status before touching a device."""
import ctypes
import os
import re

import numpy as np
import pytest

import mla_latent_kv_24_b200 as mla

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "mla.h")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"MLA_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)))


def test_library_is_built_and_loads():
    assert os.path.exists(mla.LIB_PATH), "run python -m mla_latent_kv_24_b200.build"
    lib = mla.load()
    assert lib.mla_version() == 100


def test_every_declared_symbol_is_exported():
    syms = declared_symbols()
    assert len(syms) >= 9
    assert sorted(mla.EXPORTED_SYMBOLS) == sorted(syms)
    lib = ctypes.CDLL(mla.LIB_PATH)
    for s in syms:
        assert hasattr(lib, s), s


def _call_absorbed(dims, batch=1, s_q=1, lens=(64,), max_pages=1, q=1, ws=256, wsb=1 << 20):
    lib = mla.load()
    arr = np.asarray(lens, np.int32)
    return lib.mla_decode_absorbed(ctypes.byref(dims), q, 256, 256, 256, 256, 256,
                                   arr.ctypes.data_as(ctypes.c_void_p), batch, s_q, max_pages, 1, 256, ws, wsb, None)


def test_invalid_arguments_return_status_without_device():
    good = mla.make_dims()
    assert _call_absorbed(mla.make_dims(heads_per_group=3)) == 1           # does not divide H
    assert _call_absorbed(mla.make_dims(d_c=1024)) == 2                    # unsupported dims
    assert _call_absorbed(mla.make_dims(page_size=48)) == 2
    assert _call_absorbed(good, s_q=5, lens=(64,)) == 1                    # s_q out of range (1..4)
    assert _call_absorbed(good, s_q=2, lens=(1,)) == 1                     # seq_len < s_q
    assert _call_absorbed(good, lens=(65,), max_pages=1) == 1              # seq_len > max_pages * page
    assert _call_absorbed(good, q=None) == 1                               # NULL pointer
    assert _call_absorbed(good, q=8) == 1                                  # misaligned pointer
    lib = mla.load()
    assert lib.mla_decode_absorbed(None, 1, 1, 1, 1, 1, 1, None, 1, 1, 1, 1, 1, 1, 1, None) == 1
    assert "dims is NULL" in mla.mla_last_error_string()


def test_append_argument_checks():
    lib = mla.load()
    d = mla.make_dims()
    # W_dkv set but W_kr NULL
    assert lib.mla_cache_append(ctypes.byref(d), 256, 5120, 256, None, 256, 256, 4, 256, 1, 1, 1, 256, None) == 1
    # pre-projected input must be d_c + d_rope wide
    assert lib.mla_cache_append(ctypes.byref(d), 256, 5120, None, None, 256, 256, 4, 256, 1, 1, 1, 256, None) == 1
    # zero tokens is a no-op
    assert lib.mla_cache_append(ctypes.byref(d), None, 5120, None, None, None, None, 0, None, 1, 1, 1, None, None) == 0


def test_binding_raises_mla_error():
    d = mla.make_dims(heads_per_group=5)
    with pytest.raises(mla.MlaError) as e:
        mla.mla_decode_workspace_size(d, 1, 1, [64])
    assert e.value.status == 1


def test_prefill_argument_checks_without_device():
    import mla_latent_kv_24_b200 as mla
    dims = mla.make_dims()
    with pytest.raises(mla.MlaError) as e:
        mla.mla_prefill_workspace_size(dims, 2, 300, [100, 500])          # n_q > seq_len
    assert e.value.status == 1
    with pytest.raises(mla.MlaError) as e:
        mla.mla_prefill_workspace_size(mla.make_dims(dtype="fp32"), 1, 4, [64])   # not built for fp32
    assert e.value.status == 2
    # scratch is linear in n_q: q_rot + partials + (m, l) per query row, one work item per request
    a = mla.mla_prefill_workspace_size(dims, 2, 16, [100, 500])
    b = mla.mla_prefill_workspace_size(dims, 2, 32, [100, 500])
    assert 1.9 < b / a < 2.1


def test_expand_tokens_argument_checks():
    lib = mla.load()
    d = mla.make_dims()
    # zero tokens is a no-op, whatever the pointers
    assert lib.gqla_expand_tokens(ctypes.byref(d), None, None, None, None, None, 0, None, 1, 1, 1, None, None) == 0
    assert lib.gqla_expand_tokens(ctypes.byref(d), 256, 256, 256, 256, 256, -1, 256, 1, 1, 1, 256, None) == 1
    assert lib.gqla_expand_tokens(ctypes.byref(d), 256, 256, 256, None, 256, 4, 256, 1, 1, 1, 256, None) == 1
    assert lib.gqla_expand_tokens(ctypes.byref(d), 256, 256, 256, 256, 256, 4, 256, 0, 1, 1, 256, None) == 1
    assert lib.gqla_expand_tokens(ctypes.byref(d), 256, 256, 8, 256, 256, 4, 256, 1, 1, 1, 256, None) == 1
    assert "aligned" in mla.mla_last_error_string()


def test_noalloc_scratch_size_matches_the_header():
    # The binding's copy of the static scratch size must be the header's, or the rejection test of
    # the no-allocation entry point would probe the wrong bound.
    m = re.search(r"#define\s+MLA_NOALLOC_SCRATCH_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", open(HEADER).read())
    assert m, "MLA_NOALLOC_SCRATCH_BYTES not found in include/mla.h"
    assert int(m.group(1)) << int(m.group(2)) == mla.NOALLOC_SCRATCH_BYTES


def test_debug_fault_hook_argument_checks():
    # thread-local host state only: no device is touched
    assert mla.load().mla_debug_decode_fault(-2, 0) == 1
    assert mla.load().mla_debug_decode_fault(0, 2000001) == 1
    mla.mla_debug_decode_fault(3, 1000)
    mla.mla_debug_decode_fault(-1, 0)
