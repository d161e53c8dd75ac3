"""GPU checks of the GQA path's cache expansion by token (gqla_expand_tokens): the rows that a
cache append wrote get the same [K_g | V_g] bits as expanding their whole pages, the oracle's
values within bf16 rounding, and every other row keeps its bytes ("GQLA: Group-Query Latent
Attention ..." abstract: the GQA path's per-group expanded cache)."""
import numpy as np
import pytest
import torch

import mla_latent_kv_24_b200 as mla
import oracle
import workloads as wl
from _gpu import Dev

pytestmark = pytest.mark.gpu


def _tokens(inp, s_q):
    req, pos = wl.new_token_positions(inp.seq_lens, s_q)
    return req, pos, torch.from_numpy(req).cuda(), torch.from_numpy(pos).cuda()


def _expand_tokens(dev, req_d, pos_d, n, exp):
    w = dev.inp.w
    mla.gqla_expand_tokens(dev.dims, dev.W_uk, dev.W_uv, dev.cache, req_d, pos_d, n, dev.page_table, w.B,
                           dev.max_pages, dev.inp.n_pages, exp)


@pytest.mark.parametrize("dtype,s_q", [("bf16", 1), ("bf16", 2), ("fp32", 2)])
def test_token_rows_equal_page_expansion_and_others_untouched(dtype, s_q):
    w = wl.small_workload(wl.WORKLOADS["5_8192_1"], B=3, s_q=s_q, lens=[130, 64, 7], shuffle_pages=True,
                          dtype=dtype, seed=71)
    inp = wl.make_inputs(w)
    dev = Dev(inp)
    req, pos, req_d, pos_d = _tokens(inp, s_q)
    full = dev.expand()                                   # every page
    exp = torch.full_like(full, 3.0)                      # sentinel rows
    _expand_tokens(dev, req_d, pos_d, len(req), exp)
    mla.mla_get_device_status()
    written = torch.zeros(exp.shape[0], exp.shape[2], dtype=torch.bool)
    for b, p in zip(req, pos):
        pg, r = oracle.slot_of(inp.page_table, int(b), int(p), w.page)
        written[pg, r] = True
        # same kernel arithmetic per row: identical bits to the page expansion
        assert torch.equal(exp[pg, :, r], full[pg, :, r])
    keep = (~written).cuda()
    assert (exp.permute(0, 2, 1, 3)[keep] == 3.0).all()


def test_token_rows_match_oracle():
    w = wl.small_workload(wl.WORKLOADS["5_8192_1"], B=4, s_q=2, lens=[65, 300, 2, 1000], shuffle_pages=True,
                          seed=72)
    inp = wl.make_inputs(w)
    dev = Dev(inp)
    req, pos, req_d, pos_d = _tokens(inp, 2)
    G = w.H // w.hpw
    exp = torch.zeros((inp.n_pages, G, w.page, w.d_n + w.d_v), dtype=torch.bfloat16, device="cuda")
    _expand_tokens(dev, req_d, pos_d, len(req), exp)
    mla.mla_get_device_status()
    got = wl.from_torch_f64(exp)
    sl = [oracle.slot_of(inp.page_table, int(b), int(p), w.page) for b, p in zip(req, pos)]
    rows = np.stack([inp.cache.f64()[pg, r] for pg, r in sl])
    Kg, Vg = oracle.expand_group_cache(rows, inp.W_uk.f64(), inp.W_uv.f64())      # [G, n, 128]
    ref = np.concatenate([Kg, Vg], axis=2)
    g = np.stack([got[pg, :, r] for pg, r in sl], axis=1)                           # [G, n, 256]
    rel = np.abs(g - ref).max() / np.abs(ref).max()
    assert rel <= 2 ** -8, rel


def test_out_of_range_token_is_reported_and_skipped():
    w = wl.small_workload(wl.WORKLOADS["5_8192_1"], B=2, lens=[100, 40], seed=73)
    inp = wl.make_inputs(w)
    dev = Dev(inp)
    req, pos, _, _ = _tokens(inp, 1)
    pos = pos.copy()
    pos[1] = dev.max_pages * w.page            # one past the page table
    G = w.H // w.hpw
    exp = torch.zeros((inp.n_pages, G, w.page, w.d_n + w.d_v), dtype=torch.bfloat16, device="cuda")
    _expand_tokens(dev, torch.from_numpy(req).cuda(), torch.from_numpy(pos).cuda(), len(req), exp)
    with pytest.raises(mla.MlaError) as e:
        mla.mla_get_device_status()
    assert e.value.status == 5
    pg, r = oracle.slot_of(inp.page_table, int(req[0]), int(pos[0]), w.page)
    assert exp[pg, :, r].abs().sum() > 0                    # the valid token was still expanded
    exp[pg, :, r] = 0
    assert exp.abs().sum() == 0                             # nothing else written
