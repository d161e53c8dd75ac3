"""Multi-rank (torchrun) logic of bench.py on CPU: two gloo ranks, no GPU.

Every rank decodes its own seeded batch with no collective on the data path; the only exchange is
the reduction of the timing (max over ranks) and of the cache-token count (sum over ranks)."""
import importlib.util
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
import workloads as wl  # noqa: E402


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench = _bench()
        # rank r took (r + 1) ms per step, its kernel 10 (r + 1) ms, and decoded 100 (r + 1) tokens
        times, tokens = bench.reduce_over_ranks(dist, torch.device("cpu"), [rank + 1.0, 10.0 * (rank + 1), 0.0],
                                                100 * (rank + 1))
        np.save(os.path.join(out_dir, f"r{rank}.npy"), np.array(times + [tokens]))
    finally:
        dist.destroy_process_group()


def test_reduce_over_ranks_two_gloo_ranks():
    world = 2
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_rank_main, args=(world, _free_port(), d), nprocs=world, start_method="spawn", join=True)
        for r in range(world):
            got = np.load(os.path.join(d, f"r{r}.npy"))
            # max over ranks of every time, sum of the tokens, identical on every rank
            np.testing.assert_array_equal(got, [2.0, 20.0, 0.0, 300.0])


def test_reduce_over_ranks_single_rank_is_identity():
    times, tokens = _bench().reduce_over_ranks(None, torch.device("cpu"), [1.5, 0.25, 3.0], 42)
    assert times == [1.5, 0.25, 3.0] and tokens == 42.0


@pytest.mark.parametrize("key", ["2", "4"])
def test_rank_batches_are_distinct_and_same_shape(key):
    # bench.py seeds rank r with workload seed + 1009 r: same shapes and sizes, different data
    # (and, for the ragged workload, different lengths, hence the token sum above).
    w = wl.small_workload(wl.WORKLOADS[key], B=3, lens=None if key == "4" else [100, 200, 300])
    a, b = wl.make_inputs(w, seed=w.seed), wl.make_inputs(w, seed=w.seed + 1009)
    assert a.q.data.shape == b.q.data.shape and a.W_uk.data.shape == b.W_uk.data.shape
    assert not np.array_equal(a.q.data, b.q.data)
    assert not np.array_equal(a.cache.data[:1], b.cache.data[:1])
