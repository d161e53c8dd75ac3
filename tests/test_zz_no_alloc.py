"""The no-allocation decode entry point against the workspace entry point.

mla_decode_absorbed_noalloc exists for callers that cannot allocate device memory (an engine
whose allocator already owns all of HBM, or a hot loop that must not pay cudaMalloc's implicit
synchronisation): it uses the library's static scratch instead of a caller workspace.  This file
is named to be collected last, so a run that stops at the first failure has run every other test
before it.  It passes alone in a fresh process and after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import mla_latent_kv_24_b200 as mla
import workloads as wl
from _gpu import BF16_MAE, BF16_REL, Dev, errors

pytestmark = pytest.mark.gpu


def _noalloc(dev: Dev):
    w = dev.inp.w
    out = torch.full((w.B, w.s_q, w.H, w.d_v), float("nan"), dtype=dev.tdtype, device=dev.q.device)
    mla.mla_decode_absorbed_noalloc(dev.dims, dev.q, dev.W_uk, dev.W_uv, dev.cache, dev.page_table, dev.seq_lens,
                                    dev.inp.seq_lens, w.B, w.s_q, dev.max_pages, dev.inp.n_pages, out)
    return out


def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row():
    # Two different batches, larger first, so the second call runs over the first call's leftovers.
    shapes = [dict(B=4, s_q=2, lens=[3000, 70, 1500, 4096], seed=31),
              dict(B=2, s_q=1, lens=[65, 700], seed=32)]
    for kw in shapes:
        w = wl.small_workload(wl.WORKLOADS["4"], B=kw["B"], s_q=kw["s_q"], lens=kw["lens"], lens_loguniform=None,
                              shuffle_pages=True, seed=kw["seed"])
        dev = Dev(wl.make_inputs(w))
        ref = wl.from_torch_f64(dev.decode_absorbed())
        got = wl.from_torch_f64(_noalloc(dev))
        mla.mla_get_device_status()
        rel, mae = errors(got, ref)
        assert np.isfinite(got).all()
        assert rel <= BF16_REL and mae <= BF16_MAE, (rel, mae)


def test_same_batch_twice_gives_the_same_output():
    w = wl.small_workload(wl.WORKLOADS["2"], B=3, lens=[100, 2048, 5], seed=33)
    dev = Dev(wl.make_inputs(w))
    ref = wl.from_torch_f64(dev.decode_absorbed())
    first = wl.from_torch_f64(_noalloc(dev))
    second = wl.from_torch_f64(_noalloc(dev))
    mla.mla_get_device_status()
    for got in (first, second):
        rel, mae = errors(got, ref)
        assert rel <= BF16_REL and mae <= BF16_MAE, (rel, mae)


def test_a_call_takes_no_device_memory():
    # After a first call (which looks up the static scratch's address), a call with its output
    # already allocated must leave the device's free memory exactly where it was.
    w = wl.small_workload(wl.WORKLOADS["4"], B=3, s_q=2, lens=[900, 64, 2500], lens_loguniform=None, seed=35)
    dev = Dev(wl.make_inputs(w))
    out = torch.empty((w.B, w.s_q, w.H, w.d_v), dtype=dev.tdtype, device=dev.q.device)
    call = lambda: mla.mla_decode_absorbed_noalloc(dev.dims, dev.q, dev.W_uk, dev.W_uv, dev.cache, dev.page_table,  # noqa: E731
                                                   dev.seq_lens, dev.inp.seq_lens, w.B, w.s_q, dev.max_pages,
                                                   dev.inp.n_pages, out)
    call()
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    call()
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    mla.mla_get_device_status()
    assert free_after == free_before, (free_before, free_after)


def test_batch_too_large_for_the_static_scratch_is_rejected():
    w = wl.small_workload(wl.WORKLOADS["2"], B=1, lens=[64], seed=34)
    dev = Dev(wl.make_inputs(w))
    big = 512
    lens = np.full(big, 131072, dtype=np.int32)
    need = mla.mla_decode_workspace_size(dev.dims, big, 2, lens)
    assert need > mla.NOALLOC_SCRATCH_BYTES
    out = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    # Rejected before anything is enqueued, so the small tensors are never read.
    with pytest.raises(mla.MlaError) as e:
        mla.mla_decode_absorbed_noalloc(dev.dims, dev.q, dev.W_uk, dev.W_uv, dev.cache, dev.page_table,
                                        dev.seq_lens, lens, big, 2, 2048, dev.inp.n_pages, out)
    assert e.value.status == 3
    mla.mla_get_device_status()
