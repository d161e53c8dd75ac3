"""bench.py's algorithmic accounting (the numerators of every roofline fraction), checked against
the per-token byte and flop counts written out by hand ("MLA and GRPO architecture", "The
Mathematics of MLA": the cache row is [c^KV (512) | k^R (64)]; "GQLA ..." abstract: the GQA path
reads per group K_g and V_g plus the shared RoPE key).  Host arithmetic only."""
import importlib.util
import os

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_absorbed_long_context_bytes_and_flops():
    b = _bench()
    w = b.wl.WORKLOADS["3"]                          # B = 4, L = 131072, s_q = 1, 128 heads
    lens = np.full(w.B, 131072, dtype=np.int64)
    a = b.algorithmic(w, lens, "absorbed")
    # every cached row once (576 bf16 = 1152 B) plus the absorbed queries (rows x heads x 576 x 2 B)
    assert a["kernel_bytes"] == 4 * 131072 * 1152 + 4 * 128 * 1152 == 604_569_600
    # per visible (query, token) pair and head: 2 x 576 for q.k plus 2 x 512 for p.v
    assert a["kernel_flops"] == 4 * 131072 * 128 * 2 * (576 + 512)
    assert a["tokens"] == 4 * 131072


def test_grouped_bytes_per_token_and_step_terms():
    b = _bench()
    w = b.wl.WORKLOADS["5_8192_1"]                   # B = 32, L = 8192, 16 groups of 8 heads
    lens = np.full(w.B, 8192, dtype=np.int64)
    a = b.algorithmic(w, lens, "grouped")
    tokens = 32 * 8192
    # per token: 16 groups x (128 + 128) x 2 B of expanded K|V plus the 64-wide RoPE key: 8320 B
    assert a["kernel_bytes"] == tokens * 8320 + 32 * 128 * 192 * 2 == 2_182_610_944
    assert a["kernel_flops"] == tokens * 128 * 2 * (192 + 128)
    # the step adds the output, the append's W_DKV|W_KR and hidden rows, and the new tokens'
    # expansion (both weight sets, their latent rows, 16 x 256 outputs per token)
    rows, e = 32, 2
    extra = (rows * 128 * 128 * e + 576 * w.hidden * e + rows * w.hidden * e
             + (16 * 512 * 256 + rows * 576 + rows * 16 * 256) * e)
    assert a["step_bytes"] - a["kernel_bytes"] == extra


def test_mtp_visible_pairs_are_causal():
    b = _bench()
    w = b.wl.small_workload(b.wl.WORKLOADS["4"], B=2, s_q=2)
    lens = np.array([10, 3])
    a = b.algorithmic(w, lens, "absorbed")
    visible = (9 + 10) + (2 + 3)                     # query j of a request sees L - s_q + j + 1 tokens
    assert a["kernel_flops"] == visible * 128 * 2 * (576 + 512)


def test_committed_traffic_records_read_the_cache_once():
    # each committed ncu record (profiles/traffic_*.txt) of a main kernel's DRAM bytes per launch is
    # the algorithmic bytes plus at most 2 % (the cache is read once; the partials stay in L2)
    b = _bench()
    for path, key in (("absorbed", "3"), ("grouped", "5_8192_1")):
        fn = os.path.join(ROOT, "profiles", f"traffic_{path}_{key}.txt")
        vals = dict(line.split(":", 1) for line in open(fn) if ":" in line and not line.startswith("#"))
        traffic = float(vals["dram_bytes_per_launch"])
        w = b.wl.WORKLOADS[key]
        alg = b.algorithmic(w, np.asarray(w.lens, dtype=np.int64), path)["kernel_bytes"]
        assert 1.0 <= traffic / alg <= 1.02, (path, key, traffic, alg)


def test_a_traffic_record_is_ignored_once_the_kernel_source_changes(monkeypatch):
    b = _bench()
    current = b.recorded_traffic("absorbed", "3")
    monkeypatch.setattr(b, "source_hash", lambda names: "0000000000000000")
    assert b.recorded_traffic("absorbed", "3") is None
    assert b.recorded_traffic("absorbed", "no_such_workload") is None
    assert current is None or current > 0
