"""The seeded input generator: determinism, shapes, bf16 rounding, page tables."""
import numpy as np
import torch

import workloads as wl


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10,
                        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8, 0.0, -0.0], np.float32)])
    ours = wl.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    assert np.array_equal(wl.bf16_bits_to_f64(ours), torch.from_numpy(x).to(torch.bfloat16).double().numpy())


def test_small_workload_deterministic_and_shaped():
    w = wl.small_workload(wl.WORKLOADS["4"], B=5, lens_loguniform=(10, 300), H=8)
    a, b = wl.make_inputs(w), wl.make_inputs(w)
    assert np.array_equal(a.cache.data, b.cache.data) and np.array_equal(a.q.data, b.q.data)
    assert a.q.shape == (5, 2, 8, 192) and a.cache.shape[1:] == (64, 576)
    assert ((a.seq_lens >= 10) & (a.seq_lens <= 300)).all()
    used = np.concatenate([a.page_table[i, :(int(L) + 63) // 64] for i, L in enumerate(a.seq_lens)])
    assert sorted(used.tolist()) == list(range(a.n_pages))


def test_full_workload_lengths():
    rng = np.random.default_rng(wl.WORKLOADS["4"].seed)
    L = wl.seq_lens(wl.WORKLOADS["4"], rng)
    assert L.shape == (64,) and L.min() >= 1024 and L.max() <= 32768
    assert list(wl.WORKLOADS["3"].lens) == [131072] * 4
    assert wl.WORKLOADS["5_65536_2"].hpw == 8 and wl.WORKLOADS["5_65536_2"].n_w == 16
