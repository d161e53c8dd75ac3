"""GPU checks of mla_cache_append: slot placement is bit-exact, projected values are exact when
they are representable, RoPE'd values match the oracle, untouched rows stay unchanged."""
import numpy as np
import pytest
import torch

import mla_latent_kv_24_b200 as mla
import oracle
import workloads as wl
from _gpu import assert_close, dims_of

pytestmark = pytest.mark.gpu


def _setup(hidden, seed, int_valued):
    w = wl.small_workload(wl.WORKLOADS["4"], B=3, s_q=2, lens=[70, 5, 200], lens_loguniform=None,
                          shuffle_pages=True, hidden=hidden, seed=seed)
    inp = wl.make_inputs(w)
    rng = np.random.default_rng(seed)
    if int_valued:
        h = rng.integers(-1, 2, size=inp.h.shape).astype(np.float32)
        Wd = rng.integers(-1, 2, size=inp.W_dkv.shape).astype(np.float32)
        Wr = rng.integers(-1, 2, size=inp.W_kr.shape).astype(np.float32)
        inp.h = wl.Tensor(wl.f32_to_bf16_bits(h), "bf16")
        inp.W_dkv = wl.Tensor(wl.f32_to_bf16_bits(Wd), "bf16")
        inp.W_kr = wl.Tensor(wl.f32_to_bf16_bits(Wr), "bf16")
    return w, inp


def _run(w, inp, pre_projected=False):
    req, pos = wl.new_token_positions(inp.seq_lens, w.s_q)
    cache = wl.to_torch(inp.cache)
    before = cache.clone()
    h = wl.to_torch(inp.h)
    if pre_projected:
        h = h[:, :w.d_row].contiguous()
    mla.mla_cache_append(dims_of(w), h, h.shape[1], None if pre_projected else wl.to_torch(inp.W_dkv),
                         None if pre_projected else wl.to_torch(inp.W_kr), torch.from_numpy(req).cuda(),
                         torch.from_numpy(pos).cuda(), len(req), torch.from_numpy(inp.page_table).cuda(), w.B,
                         inp.page_table.shape[1], inp.n_pages, cache)
    mla.mla_get_device_status()
    return req, pos, before, cache


def test_placement_and_exact_values():
    w, inp = _setup(hidden=64, seed=21, int_valued=True)
    req, pos, before, cache = _run(w, inp)
    ref = oracle.cache_append(inp.cache.f64(), inp.h.f64(), inp.W_dkv.f64(), inp.W_kr.f64(), req, pos,
                              inp.page_table, w.rope_base, w.d_c)
    got = wl.from_torch_f64(cache)
    written = np.zeros(got.shape[:2], dtype=bool)
    for b, p in zip(req, pos):
        pg, r = oracle.slot_of(inp.page_table, int(b), int(p), w.page)
        written[pg, r] = True
        assert np.array_equal(got[pg, r, :w.d_c], ref[pg, r, :w.d_c])        # exact integer sums
        k_ref = wl.bf16_bits_to_f64(wl.f32_to_bf16_bits(ref[pg, r, w.d_c:].astype(np.float32)))
        assert np.abs(got[pg, r, w.d_c:] - k_ref).max() <= 2 ** -7 * max(1.0, np.abs(k_ref).max())
    # every other row keeps its bytes
    assert torch.equal(cache.view(torch.int16)[torch.from_numpy(~written).cuda()],
                       before.view(torch.int16)[torch.from_numpy(~written).cuda()])


def test_pre_projected_rows_at_position_zero_are_stored_unchanged():
    w = wl.small_workload(wl.WORKLOADS["2"], B=2, lens=[1, 1], seed=3)
    inp = wl.make_inputs(w)
    req, pos = wl.new_token_positions(inp.seq_lens, 1)
    assert (pos == 0).all()
    _, _, _, cache = _run(w, inp, pre_projected=True)
    for i, (b, p) in enumerate(zip(req, pos)):
        pg, r = oracle.slot_of(inp.page_table, int(b), int(p), w.page)
        assert np.array_equal(cache[pg, r].view(torch.int16).cpu().numpy().view(np.uint16), inp.h.data[i, :w.d_row])


def test_full_hidden_projection_matches_oracle():
    w, inp = _setup(hidden=5120, seed=22, int_valued=False)
    req, pos, _, cache = _run(w, inp)
    ref = oracle.cache_append(inp.cache.f64(), inp.h.f64(), inp.W_dkv.f64(), inp.W_kr.f64(), req, pos,
                              inp.page_table, w.rope_base, w.d_c)
    got = wl.from_torch_f64(cache)
    sl = [oracle.slot_of(inp.page_table, int(b), int(p), w.page) for b, p in zip(req, pos)]
    g = np.stack([got[pg, r] for pg, r in sl])
    r_ = np.stack([ref[pg, r] for pg, r in sl])
    rel = np.abs(g - r_).max() / np.abs(r_).max()
    assert rel <= 2 ** -8, rel


def test_out_of_range_position_is_skipped_and_reported():
    w, inp = _setup(hidden=64, seed=23, int_valued=True)
    req, pos = wl.new_token_positions(inp.seq_lens, w.s_q)
    pos = pos.copy()
    pos[0] = inp.page_table.shape[1] * w.page + 3
    cache = wl.to_torch(inp.cache)
    before = cache.clone()
    h = wl.to_torch(inp.h)
    mla.mla_cache_append(dims_of(w), h, h.shape[1], wl.to_torch(inp.W_dkv), wl.to_torch(inp.W_kr),
                         torch.from_numpy(req).cuda(), torch.from_numpy(pos).cuda(), 1,
                         torch.from_numpy(inp.page_table).cuda(), w.B, inp.page_table.shape[1], inp.n_pages, cache)
    with pytest.raises(mla.MlaError) as e:
        mla.mla_get_device_status()
    assert e.value.status == 5
    assert torch.equal(cache.view(torch.int16), before.view(torch.int16))
