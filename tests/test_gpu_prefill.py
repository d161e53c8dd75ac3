"""Head-expanded prefill (mla_prefill_expanded) against the fp64 oracle: the last n_q tokens of
every request attend causally over keys and values up-projected per head (MLA weights, expanded
per head) or per group (GQLA weights)."""
import numpy as np
import pytest

import workloads as wl
from _gpu import Dev, assert_close, oracle_decode, prefill

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n_q,lens", [(1, (100, 300)), (17, (100, 300)), (64, (64, 520))])
def test_prefill_mla_weights_per_head_cache(n_q, lens):
    w = wl.small_workload(wl.WORKLOADS["2"], B=len(lens), s_q=n_q, lens=list(lens), shuffle_pages=True, seed=200 + n_q)
    inp = wl.make_inputs(w)
    dev = Dev(inp)
    got = wl.from_torch_f64(prefill(dev, dev.expand()))       # expand with heads_per_group = 1: per head
    assert_close(got, oracle_decode(inp), "bf16", f"MLA prefill n_q={n_q}")


@pytest.mark.parametrize("n_q", [3, 40])
def test_prefill_gqla_weights_per_group_cache(n_q):
    w = wl.small_workload(wl.WORKLOADS["5_8192_1"], B=3, s_q=n_q, lens=[n_q, 150, 700], shuffle_pages=True,
                          seed=300 + n_q)
    inp = wl.make_inputs(w)
    dev = Dev(inp)
    got = wl.from_torch_f64(prefill(dev, dev.expand()))
    ref = oracle_decode(inp)
    assert_close(got, ref, "bf16", f"GQLA prefill n_q={n_q}")


def test_full_prefill_from_an_empty_context():
    # n_q = L: every token attends to its own prefix, the first one to itself only
    L = 90
    w = wl.small_workload(wl.WORKLOADS["2"], B=1, s_q=L, lens=[L], seed=404)
    inp = wl.make_inputs(w)
    dev = Dev(inp)
    got = wl.from_torch_f64(prefill(dev, dev.expand()))
    ref = oracle_decode(inp)
    assert_close(got, ref, "bf16", "full prefill")
    # query 0 sees only token 0, so each head's output is its V row of token 0 (one-key softmax)
    np.testing.assert_allclose(got[0, 0], ref[0, 0], rtol=0, atol=2 ** -7 * np.abs(ref[0, 0]).max())


def test_prefill_full_size_sampled():
    # the size the prefill is timed at: B = 2, L = 4096, n_q = 512 (per-head cache), sampled rows
    from _gpu import compare_sampled, oracle_decode_sampled, sample_outputs
    w = wl.small_workload(wl.WORKLOADS["2"], B=2, s_q=512, lens=[4096, 4096], seed=7)
    inp = wl.make_inputs(w)
    dev = Dev(inp)
    got = wl.from_torch_f64(prefill(dev, dev.expand()))
    assert np.isfinite(got).all()
    sample = sample_outputs(inp, 24)
    compare_sampled(got, oracle_decode_sampled(inp, sample), "bf16", "prefill B=2 L=4096 n_q=512")
