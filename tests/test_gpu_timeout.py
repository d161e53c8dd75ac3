"""Failure detection of the tcgen05 decode's bounded waits, without a GPU fault.

A test hook makes the PV issuer withhold one pipeline completion signal, so the waits on it run
out after a short limit: the kernel must record MLA_ERR_TIMEOUT, stop, free its tensor memory
and return, and the same context must then decode correctly."""
import time

import numpy as np
import pytest

import mla_latent_kv_24_b200 as mla
import workloads as wl
from _gpu import Dev, assert_close, oracle_decode

pytestmark = pytest.mark.gpu


def _timed_out(dev, withhold):
    mla.mla_debug_decode_fault(withhold, 2000)   # every wait gives up after 2 ms
    try:
        t0 = time.perf_counter()
        dev.decode_absorbed()
        with pytest.raises(mla.MlaError) as e:
            mla.mla_get_device_status()
        elapsed = time.perf_counter() - t0
    finally:
        mla.mla_debug_decode_fault(-1, 0)
    assert e.value.status == 6, e.value          # MLA_ERR_TIMEOUT
    assert elapsed < 5.0, elapsed                  # the short limit applied, not the 2 s default


def test_withheld_first_step_times_out_and_the_context_recovers():
    # short requests: every CTA pair decodes one 128-token step, so step 0 is every pair's step
    w = wl.small_workload(wl.WORKLOADS["2"], B=2, lens=[300, 4000], seed=41)
    inp = wl.make_inputs(w)
    dev = Dev(inp)
    mla.mla_get_device_status()
    _timed_out(dev, 0)
    got = wl.from_torch_f64(dev.decode_absorbed())
    mla.mla_get_device_status()
    assert_close(got, oracle_decode(inp), "bf16", "after a timeout at step 0")


def test_withheld_later_step_times_out_and_the_next_call_is_bit_identical():
    # long requests: each pair runs several steps, and the signal of its fourth step is withheld
    w = wl.small_workload(wl.WORKLOADS["2"], B=2, lens=[40000, 20000], seed=42)
    dev = Dev(wl.make_inputs(w))
    ref = wl.from_torch_f64(dev.decode_absorbed())
    mla.mla_get_device_status()
    _timed_out(dev, 3)
    got = wl.from_torch_f64(dev.decode_absorbed())
    mla.mla_get_device_status()
    assert np.array_equal(got, ref)
