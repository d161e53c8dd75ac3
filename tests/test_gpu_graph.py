"""A whole decode step (cache append, then the decode call) captured in a CUDA graph and replayed
gives the bits of the same step run eagerly, on both paths.  The library's kernels are launched
with programmatic stream serialisation, which stream capture records as programmatic edges."""
import pytest
import torch

import mla_latent_kv_24_b200 as mla
import workloads as wl
from _gpu import Dev

pytestmark = pytest.mark.gpu


def _step_fn(dev, grouped):
    w, inp = dev.inp.w, dev.inp
    req_np, pos_np = wl.new_token_positions(inp.seq_lens, w.s_q)
    req, pos = torch.from_numpy(req_np).cuda(), torch.from_numpy(pos_np).cuda()
    h, W_dkv, W_kr = wl.to_torch(inp.h), wl.to_torch(inp.W_dkv), wl.to_torch(inp.W_kr)
    out = torch.empty((w.B, w.s_q, w.H, w.d_v), dtype=dev.tdtype, device="cuda")
    if grouped:
        exp = dev.expand()
        nb = mla.gqla_decode_workspace_size(dev.dims, w.B, w.s_q, inp.seq_lens)
    else:
        nb = mla.mla_decode_workspace_size(dev.dims, w.B, w.s_q, inp.seq_lens)
    ws = torch.empty(max(nb, 256), dtype=torch.uint8, device="cuda")

    def step():
        mla.mla_cache_append(dev.dims, h, w.hidden, W_dkv, W_kr, req, pos, len(req_np), dev.page_table, w.B,
                             dev.max_pages, inp.n_pages, dev.cache)
        if grouped:
            mla.gqla_expand_tokens(dev.dims, dev.W_uk, dev.W_uv, dev.cache, req, pos, len(req_np), dev.page_table,
                                   w.B, dev.max_pages, inp.n_pages, exp)
            mla.gqla_decode_grouped(dev.dims, dev.q, exp, dev.cache, dev.page_table, dev.seq_lens, inp.seq_lens, w.B,
                                    w.s_q, dev.max_pages, inp.n_pages, out, ws)
        else:
            mla.mla_decode_absorbed(dev.dims, dev.q, dev.W_uk, dev.W_uv, dev.cache, dev.page_table, dev.seq_lens,
                                    inp.seq_lens, w.B, w.s_q, dev.max_pages, inp.n_pages, out, ws)
    return step, out


@pytest.mark.parametrize("key,grouped", [("2", False), ("4", False), ("5_8192_1", True)])
def test_captured_step_replays_bit_exact(key, grouped):
    w = wl.small_workload(wl.WORKLOADS[key], B=3, s_q=2 if key == "4" else 1, lens=[300, 64, 1000],
                          lens_loguniform=None, shuffle_pages=True, seed=81)
    dev = Dev(wl.make_inputs(w))
    mla.mla_set_profile_events(None, None)
    step, out = _step_fn(dev, grouped)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()                                   # eager, on the capture stream's pool
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    mla.mla_get_device_status()
    eager = out.clone()
    out.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    mla.mla_get_device_status()
    assert torch.equal(out.view(torch.int16), eager.view(torch.int16))
    del g
