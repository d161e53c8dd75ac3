"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Small shapes compare every output element; the full-size workloads compare sampled output
rows (the oracle computes them one request at a time).  Tolerances: bf16 inputs with fp32
accumulation, normwise max relative error <= 1e-2 and mean absolute error <= 1e-3; the fp32
workload <= 1e-5.
"""
import numpy as np
import pytest
import torch

import mla_latent_kv_24_b200 as mla
import workloads as wl
from _gpu import (Dev, assert_close, compare_sampled, oracle_decode, oracle_decode_sampled, sample_outputs)

pytestmark = pytest.mark.gpu

_CACHE = {}


def full_inputs(key):
    if key not in _CACHE:
        _CACHE.clear()
        _CACHE[key] = wl.make_inputs(wl.WORKLOADS[key])
    return _CACHE[key]


def test_tiny_fp32_workload_matches_oracle():
    inp = wl.make_inputs(wl.WORKLOADS["1"])
    got = wl.from_torch_f64(Dev(inp).decode_absorbed())
    rel, _ = assert_close(got, oracle_decode(inp), "fp32", "tiny fp32")
    assert rel <= 1e-5


SMALL = [
    # (B, s_q, hpw, lens, shuffle)
    (3, 1, 1, (1, 64, 65), False),
    (4, 2, 1, (2, 63, 129, 700), True),
    (2, 1, 8, (128, 1000), True),
    (5, 2, 8, (2, 3, 64, 130, 257), False),
]


@pytest.mark.parametrize("B,s_q,hpw,lens,shuffle", SMALL)
def test_absorbed_small_shapes_match_oracle(B, s_q, hpw, lens, shuffle):
    w = wl.small_workload(wl.WORKLOADS["4"], B=B, s_q=s_q, hpw=hpw, lens=list(lens), lens_loguniform=None,
                          shuffle_pages=shuffle, seed=1000 + B)
    inp = wl.make_inputs(w)
    got = wl.from_torch_f64(Dev(inp).decode_absorbed())
    assert_close(got, oracle_decode(inp), "bf16", f"absorbed {B}x{s_q} hpw{hpw}")


def test_absorbed_fp32_general_shapes():
    w = wl.small_workload(wl.WORKLOADS["1"], B=3, s_q=2, H=8, hpw=2, lens=[2, 40, 150], page=32, seed=7)
    inp = wl.make_inputs(w)
    got = wl.from_torch_f64(Dev(inp).decode_absorbed())
    assert_close(got, oracle_decode(inp), "fp32", "fp32 general")


@pytest.mark.parametrize("key", ["2", "3", "4"])
def test_absorbed_full_size_sampled(key):
    inp = full_inputs(key)
    got = wl.from_torch_f64(Dev(inp).decode_absorbed())
    assert np.isfinite(got).all()
    sample = sample_outputs(inp, 12)
    compare_sampled(got, oracle_decode_sampled(inp, sample), "bf16", f"workload {key}")


@pytest.mark.parametrize("B,s_q,lens", [(2, 1, (64, 200)), (3, 2, (2, 65, 511))])
def test_grouped_small_shapes_match_oracle(B, s_q, lens):
    w = wl.small_workload(wl.WORKLOADS["5_8192_1"], B=B, s_q=s_q, lens=list(lens), shuffle_pages=True, seed=77 + B)
    inp = wl.make_inputs(w)
    dev = Dev(inp)
    exp = dev.expand()
    got = wl.from_torch_f64(dev.decode_grouped(exp))
    ref = oracle_decode(inp)
    assert_close(got, ref, "bf16", "grouped small")
    # the absorbed path on the same GQLA weights agrees with the same oracle
    assert_close(wl.from_torch_f64(dev.decode_absorbed()), ref, "bf16", "absorbed on GQLA weights")


@pytest.mark.parametrize("B,s_q,lens", [(1, 2, (5000,)), (4, 2, (129, 4097, 64, 3000)), (6, 1, (1, 63, 64, 65, 700, 2049))])
def test_grouped_multi_chunk_shapes_match_oracle(B, s_q, lens):
    # few requests against a whole GPU: every request is cut into many chunks, some of which end
    # between the two queries' visible lengths
    w = wl.small_workload(wl.WORKLOADS["5_8192_1"], B=B, s_q=s_q, lens=list(lens), shuffle_pages=True, seed=131 + B)
    inp = wl.make_inputs(w)
    dev = Dev(inp)
    got = wl.from_torch_f64(dev.decode_grouped(dev.expand()))
    assert_close(got, oracle_decode(inp), "bf16", f"grouped multi-chunk {lens}")


@pytest.mark.parametrize("s_q,lens", [(2, (70, 130, 1000)), (1, (84, 127, 1111, 64)), (4, (70, 150, 1000, 1087))])
def test_grouped_ignores_nonfinite_stale_slots(s_q, lens):
    # slots past a request's length in its last page are never read as keys or values: the page
    # arrives whole by tensor copy and each warp zeroes its own rows past the end (last pages with
    # 2 to 63 valid rows put the end inside every warp's 16-row band; s_q = 4 runs two row tiles)
    w = wl.small_workload(wl.WORKLOADS["5_8192_1"], B=len(lens), s_q=s_q, lens=list(lens), shuffle_pages=True,
                          seed=21 + s_q)
    inp = wl.make_inputs(w)
    dev = Dev(inp)
    exp = dev.expand()
    for b, L in enumerate(inp.seq_lens):
        last = int(inp.page_table[b, (int(L) - 1) // w.page])
        used = int(L) - ((int(L) - 1) // w.page) * w.page
        exp[last, :, used:, :] = float("nan")
        dev.cache.view(inp.n_pages, w.page, w.d_row)[last, used:, :] = float("nan")
    got = wl.from_torch_f64(dev.decode_grouped(exp))
    mla.mla_get_device_status()
    assert_close(got, oracle_decode(inp), "bf16", f"grouped with NaN stale slots s_q={s_q}")


@pytest.mark.parametrize("s_q,lens", [(1, (70, 130, 1000, 64)), (2, (70, 129, 1000, 5))])
def test_absorbed_ignores_nonfinite_stale_slots(s_q, lens):
    # slots past a request's length in its last page hold NaN; the tensor-core kernel loads whole
    # pages, so it must clear those rows before P.V (a zero probability times NaN is NaN)
    w = wl.small_workload(wl.WORKLOADS["4"], B=len(lens), s_q=s_q, lens=list(lens), lens_loguniform=None,
                          shuffle_pages=True, seed=23 + s_q)
    inp = wl.make_inputs(w)
    dev = Dev(inp)
    for b, L in enumerate(inp.seq_lens):
        last = int(inp.page_table[b, (int(L) - 1) // w.page])
        used = int(L) - ((int(L) - 1) // w.page) * w.page
        dev.cache.view(inp.n_pages, w.page, w.d_row)[last, used:, :] = float("nan")
    got = wl.from_torch_f64(dev.decode_absorbed())
    mla.mla_get_device_status()
    assert_close(got, oracle_decode(inp), "bf16", f"absorbed with NaN stale slots s_q={s_q}")


@pytest.mark.parametrize("s_q", [3, 4])
def test_deeper_mtp_both_paths_match_oracle(s_q):
    # s_q = 3, 4: the absorbed path decodes every query row; the grouped path runs two 16-row
    # tensor-core tiles (queries 0-1 and 2-3) over each K/V tile.  One request has exactly s_q tokens.
    w = wl.small_workload(wl.WORKLOADS["5_8192_1"], B=3, s_q=s_q, lens=[s_q, 130, 700], shuffle_pages=True,
                          seed=60 + s_q)
    inp = wl.make_inputs(w)
    dev = Dev(inp)
    ref = oracle_decode(inp)
    assert_close(wl.from_torch_f64(dev.decode_absorbed()), ref, "bf16", f"absorbed s_q={s_q}")
    assert_close(wl.from_torch_f64(dev.decode_grouped(dev.expand())), ref, "bf16", f"grouped s_q={s_q}")


@pytest.mark.parametrize("s_q,lens", [(4, (5000, 64)), (3, (129, 4097, 3)), (4, (4, 70, 2049, 1000))])
def test_deeper_mtp_grouped_multi_chunk_matches_oracle(s_q, lens):
    # long requests split into many chunks, some of which end between the queries' visible
    # lengths; NaN in the stale slots of every last page must not reach the output
    w = wl.small_workload(wl.WORKLOADS["5_8192_1"], B=len(lens), s_q=s_q, lens=list(lens), shuffle_pages=True,
                          seed=90 + s_q + len(lens))
    inp = wl.make_inputs(w)
    dev = Dev(inp)
    exp = dev.expand()
    for b, L in enumerate(inp.seq_lens):
        last = int(inp.page_table[b, (int(L) - 1) // w.page])
        used = int(L) - ((int(L) - 1) // w.page) * w.page
        exp[last, :, used:, :] = float("nan")
        dev.cache.view(inp.n_pages, w.page, w.d_row)[last, used:, :] = float("nan")
    assert_close(wl.from_torch_f64(dev.decode_grouped(exp)), oracle_decode(inp), "bf16",
                 f"grouped s_q={s_q} multi-chunk {lens}")


def test_deeper_mtp_mla_weights_match_oracle():
    w = wl.small_workload(wl.WORKLOADS["2"], B=2, s_q=4, lens=[4, 300], seed=64)
    inp = wl.make_inputs(w)
    assert_close(wl.from_torch_f64(Dev(inp).decode_absorbed()), oracle_decode(inp), "bf16", "MLA s_q=4")


def test_expand_cache_matches_oracle():
    import oracle
    w = wl.small_workload(wl.WORKLOADS["5_8192_1"], B=2, lens=[100, 64], seed=5)
    inp = wl.make_inputs(w)
    exp = wl.from_torch_f64(Dev(inp).expand())            # [n_pages, G, page, 256]
    rows = inp.cache.f64().reshape(-1, w.d_row)
    Kg, Vg = oracle.expand_group_cache(rows, inp.W_uk.f64(), inp.W_uv.f64())   # [G, T, 128]
    ref = np.concatenate([Kg, Vg], axis=2).reshape(w.n_w, inp.n_pages, w.page, 256).transpose(1, 0, 2, 3)
    rel = np.abs(exp - ref).max() / np.abs(ref).max()
    assert rel <= 2 ** -8, rel


@pytest.mark.parametrize("key", ["5_8192_1", "5_65536_2"])
def test_grouped_full_size_sampled(key):
    inp = full_inputs(key)
    dev = Dev(inp)
    exp = dev.expand()
    got_g = wl.from_torch_f64(dev.decode_grouped(exp))
    del exp
    torch.cuda.empty_cache()
    got_a = wl.from_torch_f64(dev.decode_absorbed())
    sample = sample_outputs(inp, 8)
    ref = oracle_decode_sampled(inp, sample)
    compare_sampled(got_g, ref, "bf16", f"grouped {key}")
    compare_sampled(got_a, ref, "bf16", f"absorbed {key}")


def test_out_of_range_page_id_is_reported_not_faulted():
    w = wl.small_workload(wl.WORKLOADS["2"], B=2, lens=[100, 100], seed=3)
    inp = wl.make_inputs(w)
    dev = Dev(inp)
    dev.page_table[1, 1] = inp.n_pages + 5
    dev.decode_absorbed()
    with pytest.raises(mla.MlaError) as e:
        mla.mla_get_device_status()
    assert e.value.status == 5
    dev.page_table[1, 1] = int(inp.page_table[1, 1])      # the context stays usable
    got = wl.from_torch_f64(dev.decode_absorbed())
    mla.mla_get_device_status()
    assert_close(got, oracle_decode(inp), "bf16", "after bounds error")


def test_grouped_out_of_range_page_id_is_reported_not_faulted():
    # the grouped path's tensor copies read an out-of-range page as zeros and report the id
    w = wl.small_workload(wl.WORKLOADS["5_8192_2"], B=2, lens=[200, 300], shuffle_pages=True, seed=13)
    inp = wl.make_inputs(w)
    dev = Dev(inp)
    exp = dev.expand()
    dev.page_table[0, 2] = inp.n_pages + 7
    dev.decode_grouped(exp)
    with pytest.raises(mla.MlaError) as e:
        mla.mla_get_device_status()
    assert e.value.status == 5
    dev.page_table[0, 2] = int(inp.page_table[0, 2])      # the context stays usable
    got = wl.from_torch_f64(dev.decode_grouped(exp))
    mla.mla_get_device_status()
    assert_close(got, oracle_decode(inp), "bf16", "grouped after bounds error")


def test_device_seq_lens_disagreeing_with_host_is_reported():
    w = wl.small_workload(wl.WORKLOADS["2"], B=2, lens=[100, 300], seed=4)
    inp = wl.make_inputs(w)
    dev = Dev(inp)
    dev.seq_lens[1] = 64
    dev.decode_absorbed()
    with pytest.raises(mla.MlaError) as e:
        mla.mla_get_device_status()
    assert e.value.status == 1


def test_request_alone_equals_request_in_batch():
    w = wl.small_workload(wl.WORKLOADS["4"], B=4, s_q=2, lens=[3000, 70, 1500, 4096], lens_loguniform=None,
                          shuffle_pages=True, seed=9)
    inp = wl.make_inputs(w)
    dev = Dev(inp)
    full = wl.from_torch_f64(dev.decode_absorbed())
    for b in (1, 3):
        sub = Dev(inp)
        sub.q = dev.q[b:b + 1].contiguous()
        sub.page_table = dev.page_table[b:b + 1].contiguous()
        sub.seq_lens = dev.seq_lens[b:b + 1].contiguous()
        sub.inp = wl.DecodeInputs(**{**inp.__dict__, "seq_lens": inp.seq_lens[b:b + 1],
                                     "page_table": inp.page_table[b:b + 1], "w": wl.small_workload(w, B=1)})
        one = wl.from_torch_f64(sub.decode_absorbed())
        # Different batches get different split plans, so fp32 sums run in another order and a
        # bf16 output may move by an ulp; anything beyond two ulps of the largest value is a bug.
        diff = np.abs(one[0] - full[b])
        assert diff.max() / np.abs(full[b]).max() <= 2 ** -6, diff.max()
        assert diff.mean() <= 1e-4, diff.mean()
