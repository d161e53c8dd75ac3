"""Group-sharded GQA-path decode (mla_latent_kv_24_b200.tp): shard ranges, the head all-gather on
two gloo ranks (CPU, oracle outputs per shard), and the real kernels per shard on one GPU."""
import os
import socket
import sys
import tempfile

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import mla_latent_kv_24_b200 as mla  # noqa: E402
from mla_latent_kv_24_b200 import tp  # noqa: E402
import workloads as wl  # noqa: E402

GQLA = mla.make_dims(n_heads=128, heads_per_group=8)


@pytest.mark.parametrize("n", [1, 2, 4, 8, 16])
def test_shards_cover_heads_and_groups_once(n):
    heads, groups = [], []
    for r in range(n):
        s = tp.shard(GQLA, n, r)
        assert s.head1 - s.head0 == 128 // n and s.group1 - s.group0 == 16 // n
        assert s.head0 == 8 * s.group0   # a rank's heads are exactly its groups' heads
        heads += list(range(s.head0, s.head1))
        groups += list(range(s.group0, s.group1))
    assert heads == list(range(128)) and groups == list(range(16))
    assert tp.local_dims(GQLA, n).n_heads == 128 // n


@pytest.mark.parametrize("n,rank", [(3, 0), (32, 0), (2, 2), (0, 0)])
def test_bad_shards_are_rejected(n, rank):
    with pytest.raises(ValueError):
        tp.shard(GQLA, n, rank)


def _small_gqla():
    w = wl.small_workload(wl.WORKLOADS["5_8192_2"], B=2, lens=[70, 130], shuffle_pages=True, seed=91)
    return w, wl.make_inputs(w)


def _oracle(inp, w, h0=0, h1=None, g0=0, g1=None):
    import oracle
    h1 = w.H if h1 is None else h1
    g1 = w.n_w if g1 is None else g1
    return oracle.decode_expanded(inp.q.f64()[:, :, h0:h1], inp.W_uk.f64()[g0:g1], inp.W_uv.f64()[g0:g1],
                                  inp.cache.f64(), inp.page_table, inp.seq_lens, w.hpw, w.softmax_scale, w.rope_base)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, inp = _small_gqla()
        s = tp.shard(GQLA, world, rank)
        local = torch.from_numpy(_oracle(inp, w, s.head0, s.head1, s.group0, s.group1))
        full = tp.gather_heads(local)
        np.save(os.path.join(out_dir, f"r{rank}.npy"), full.numpy())
    finally:
        dist.destroy_process_group()


def test_gather_heads_reassembles_the_oracle_on_two_gloo_ranks():
    world = 2
    w, inp = _small_gqla()
    ref = _oracle(inp, w)
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_rank_main, args=(world, _free_port(), d), nprocs=world, start_method="spawn", join=True)
        for r in range(world):
            got = np.load(os.path.join(d, f"r{r}.npy"))
            # the per-shard oracle is the same arithmetic on a head subset: equal to fp64 rounding
            np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12 * np.abs(ref).max())


@pytest.mark.gpu
@pytest.mark.parametrize("n", [2, 8])
def test_every_shard_decoded_on_one_gpu_matches_the_oracle(n):
    from _gpu import Dev, assert_close
    w, inp = _small_gqla()
    dev = Dev(inp)
    out = torch.empty((w.B, w.s_q, w.H, w.d_v), dtype=torch.bfloat16, device="cuda")
    for r in range(n):
        s = tp.shard(GQLA, n, r)
        dims = tp.local_dims(dev.dims, n)
        W_uk, W_uv = dev.W_uk[s.group0:s.group1].contiguous(), dev.W_uv[s.group0:s.group1].contiguous()
        exp = torch.empty((inp.n_pages, s.group1 - s.group0, w.page, w.d_n + w.d_v), dtype=torch.bfloat16,
                          device="cuda")
        mla.gqla_expand_cache(dims, W_uk, W_uv, dev.cache, None, 0, inp.n_pages, exp)
        q = dev.q[:, :, s.head0:s.head1].contiguous()
        nb = mla.gqla_decode_workspace_size(dims, w.B, w.s_q, inp.seq_lens)
        ws = torch.empty(max(nb, 256), dtype=torch.uint8, device="cuda")
        o = torch.empty((w.B, w.s_q, s.head1 - s.head0, w.d_v), dtype=torch.bfloat16, device="cuda")
        mla.gqla_decode_grouped(dims, q, exp, dev.cache, dev.page_table, dev.seq_lens, inp.seq_lens, w.B, w.s_q,
                                dev.max_pages, inp.n_pages, o, ws)
        out[:, :, s.head0:s.head1] = o
    assert_close(wl.from_torch_f64(out), _oracle(inp, w), "bf16", f"tp={n} shards")
