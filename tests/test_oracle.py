"""Pins for the CPU oracle: checks it against things other than itself.

- a pure-Python brute force on tiny shapes;
- closed forms (one cached token, zero query, identical rows);
- the equivalence of the absorbed, head-expanded and grouped forms that the GQLA abstract
  states ("two algebraically equivalent decoding paths over the same parameters");
- RoPE identities and an independent complex-number form of the rotation;
- the split-softmax merge identity;
- the cache-size figures the pages print (tests/golden/cache_arithmetic.txt);
- planted mistakes in the oracle, each of which some pin must catch.
"""
import math
import os

import numpy as np
import pytest

import oracle
from oracle import brute
from oracle import mla as om

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "cache_arithmetic.txt")


def _rand_problem(rng, B=2, s_q=2, H=4, hpw=2, d_c=6, d_n=4, d_r=4, d_v=3, lens=(3, 17), page=4):
    n_w = H // hpw
    lens = np.asarray(lens, dtype=np.int32)[:B]
    n_pages = sum((int(L) + page - 1) // page for L in lens) + 1
    perm = rng.permutation(n_pages)
    pt = np.zeros((B, max((int(L) + page - 1) // page for L in lens)), dtype=np.int32)
    off = 0
    for b, L in enumerate(lens):
        n = (int(L) + page - 1) // page
        pt[b, :n] = perm[off:off + n]
        off += n
    return dict(
        q=rng.standard_normal((B, s_q, H, d_n + d_r)),
        W_uk=rng.standard_normal((n_w, d_n, d_c)) * 0.5,
        W_uv=rng.standard_normal((n_w, d_v, d_c)) * 0.5,
        cache=rng.standard_normal((n_pages, page, d_c + d_r)),
        page_table=pt, seq_lens=lens, hpw=hpw, d_c=d_c, d_n=d_n,
        scale=1.0 / math.sqrt(d_n + d_r), base=10000.0, s_q=s_q)


def _oracle_out(p):
    return om.decode_expanded(p["q"], p["W_uk"], p["W_uv"], p["cache"], p["page_table"], p["seq_lens"],
                              p["hpw"], p["scale"], p["base"])


def _brute_out(p):
    rows = [om.request_rows(p["cache"], p["page_table"], b, int(L)).tolist() for b, L in enumerate(p["seq_lens"])]
    return np.asarray(brute.decode(p["q"].tolist(), p["W_uk"].tolist(), p["W_uv"].tolist(), rows, p["s_q"],
                                   p["hpw"], p["d_c"], p["d_n"], p["scale"], p["base"]))


# ----------------------------------------------------------------------------- pins
# Each pin returns True when the oracle passes it; tests assert them and the planted-
# mistake test checks that each mistake makes at least one of them fail.

def pin_brute_force():
    rng = np.random.default_rng(11)
    ok = True
    for (H, hpw, s_q, lens) in [(1, 1, 1, (1, 2)), (2, 1, 2, (2, 17)), (4, 2, 1, (3, 5)), (4, 4, 2, (17, 3))]:
        p = _rand_problem(rng, H=H, hpw=hpw, s_q=s_q, lens=lens)
        ok &= np.allclose(_oracle_out(p), _brute_out(p), rtol=0, atol=1e-12)
    return bool(ok)


def pin_single_token():
    rng = np.random.default_rng(12)
    p = _rand_problem(rng, B=1, s_q=1, lens=(1,))
    out = _oracle_out(p)
    c0 = om.request_rows(p["cache"], p["page_table"], 0, 1)[0, :p["d_c"]]
    exp = np.stack([p["W_uv"][h // p["hpw"]] @ c0 for h in range(p["q"].shape[2])])
    return bool(np.allclose(out[0, 0], exp, rtol=0, atol=1e-13))


def pin_zero_query():
    rng = np.random.default_rng(13)
    p = _rand_problem(rng, s_q=2, lens=(9, 14))
    p["q"][:] = 0.0
    out = _oracle_out(p)
    ok = True
    for b, L in enumerate(p["seq_lens"]):
        rows = om.request_rows(p["cache"], p["page_table"], b, int(L))
        for j in range(2):
            pj = int(L) - 2 + j
            mean_c = rows[:pj + 1, :p["d_c"]].mean(axis=0)
            for h in range(p["q"].shape[2]):
                ok &= np.allclose(out[b, j, h], p["W_uv"][h // p["hpw"]] @ mean_c, rtol=0, atol=1e-13)
    return bool(ok)


def pin_identical_rows():
    rng = np.random.default_rng(14)
    p = _rand_problem(rng, B=1, s_q=1, lens=(7,))
    row = rng.standard_normal(p["cache"].shape[2])
    p["cache"][:] = row
    out = _oracle_out(p)
    exp = np.stack([p["W_uv"][h // p["hpw"]] @ row[:p["d_c"]] for h in range(p["q"].shape[2])])
    return bool(np.allclose(out[0, 0], exp, rtol=0, atol=1e-12))


def pin_query_positions():
    """With s_q = 2, query 0 equals an s_q = 1 decode over the first L - 1 tokens."""
    rng = np.random.default_rng(15)
    p = _rand_problem(rng, B=1, s_q=2, lens=(13,))
    out2 = _oracle_out(p)
    rows = om.request_rows(p["cache"], p["page_table"], 0, 13)
    out1 = om.decode_request_expanded(p["q"][0, :1], rows[:12], p["W_uk"], p["W_uv"], p["hpw"], p["scale"], p["base"])
    return bool(np.allclose(out2[0, 0], out1[0], rtol=0, atol=1e-13))


def pin_paths_equivalent():
    rng = np.random.default_rng(16)
    ok = True
    for hpw in (1, 2, 4):
        p = _rand_problem(rng, B=1, s_q=2, H=4, hpw=hpw, lens=(19,))
        rows = om.request_rows(p["cache"], p["page_table"], 0, 19)
        e = om.decode_request_expanded(p["q"][0], rows, p["W_uk"], p["W_uv"], hpw, p["scale"], p["base"])
        a = om.decode_request_absorbed(p["q"][0], rows, p["W_uk"], p["W_uv"], hpw, p["scale"], p["base"])
        Kg, Vg = om.expand_group_cache(rows, p["W_uk"], p["W_uv"])
        g = om.decode_request_grouped(p["q"][0], Kg, Vg, rows[:, p["d_c"]:], hpw, p["scale"], p["base"])
        ok &= np.allclose(e, a, rtol=0, atol=1e-12) and np.allclose(e, g, rtol=0, atol=1e-12)
    return bool(ok)


def pin_rope_complex():
    """RoPE pair (x0, x1) at angle a equals the complex product (x0 + i x1) e^{i a}."""
    rng = np.random.default_rng(17)
    d, base = 8, 10000.0
    x = rng.standard_normal((5, d))
    pos = np.array([0, 1, 7, 1000, 131071])
    r = om.rope(x, pos, base)
    z = x[:, 0::2] + 1j * x[:, 1::2]
    theta = np.array([base ** (-(2.0 * i) / d) for i in range(d // 2)])
    zr = z * np.exp(1j * pos[:, None] * theta[None, :])
    return bool(np.allclose(r[:, 0::2], zr.real, atol=1e-12) and np.allclose(r[:, 1::2], zr.imag, atol=1e-12))


def pin_rope_relative():
    """<RoPE(q, m), RoPE(k, n)> depends only on m - n; position 0 is the identity; norms kept."""
    rng = np.random.default_rng(18)
    q, k = rng.standard_normal(8), rng.standard_normal(8)
    a = om.rope(q, 10, 10000.0) @ om.rope(k, 3, 10000.0)
    b = om.rope(q, 1007, 10000.0) @ om.rope(k, 1000, 10000.0)
    ok = abs(a - b) < 1e-10
    ok &= np.array_equal(om.rope(q, 0, 10000.0), q)
    ok &= abs(np.linalg.norm(om.rope(q, 12345, 10000.0)) - np.linalg.norm(q)) < 1e-12
    return bool(ok)


def pin_split_merge():
    rng = np.random.default_rng(19)
    K, V, q = rng.standard_normal((40, 6)), rng.standard_normal((40, 5)), rng.standard_normal(6) * 3
    full = om.attention_weights(q, K, 39, 0.7) @ V
    ok = True
    for cuts in ([0, 40], [0, 1, 40], [0, 13, 14, 27, 40], list(range(0, 41, 8))):
        parts = [om.partial_attention(q, K, V, a, b, 0.7) for a, b in zip(cuts[:-1], cuts[1:])]
        ok &= np.allclose(om.combine_partials(parts), full, rtol=0, atol=1e-13)
    return bool(ok)


def pin_masking():
    """Rows after a query's position (and page-tail rows beyond L) do not change its output;
    the row at the position does."""
    rng = np.random.default_rng(20)
    p = _rand_problem(rng, B=1, s_q=2, lens=(10,), page=4)
    base_out = _oracle_out(p)
    pg, r = om.slot_of(p["page_table"], 0, 9, 4)
    p2 = dict(p, cache=p["cache"].copy())
    p2["cache"][pg, r] += 5.0                  # token 9: seen by query 1 only
    out2 = _oracle_out(p2)
    ok = np.allclose(out2[0, 0], base_out[0, 0], atol=1e-14) and not np.allclose(out2[0, 1], base_out[0, 1])
    pg, r = om.slot_of(p["page_table"], 0, 11, 4)
    p3 = dict(p, cache=p["cache"].copy())
    p3["cache"][pg, r] += 5.0                  # row 11 is beyond L = 10
    ok &= np.array_equal(_oracle_out(p3), base_out)
    return bool(ok)


ALL_PINS = [pin_brute_force, pin_single_token, pin_zero_query, pin_identical_rows, pin_query_positions,
            pin_paths_equivalent, pin_rope_complex, pin_rope_relative, pin_split_merge, pin_masking]


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    assert pin()


def test_softmax_rows_sum_to_one():
    rng = np.random.default_rng(21)
    for _ in range(5):
        K, q = rng.standard_normal((50, 7)), rng.standard_normal(7) * 10
        p = om.attention_weights(q, K, int(rng.integers(0, 50)), 0.4)
        assert abs(p.sum() - 1.0) < 1e-15 and (p > 0).all()


def test_softmax_large_scores_one_hot():
    """With huge scores the weights go to the arg-max token (no overflow from exp)."""
    K = np.array([[1.0, 0.0], [0.0, 1.0], [3.0, 0.0]])
    p = om.attention_weights(np.array([1.0, 0.0]), K, 2, 1e4)
    assert np.array_equal(p, [0.0, 0.0, 1.0])


def test_rope_does_not_commute_with_up_projection():
    """Rotating before an up-projection differs from rotating after it ("MLA's 512-Scalar KV
    Latent ..." RoPE paragraph), unless the projection commutes with the rotation."""
    rng = np.random.default_rng(22)
    W, x = rng.standard_normal((8, 8)), rng.standard_normal(8)
    assert not np.allclose(om.rope(W @ x, 5, 10000.0), W @ om.rope(x, 5, 10000.0))
    S = 2.5 * np.eye(8)
    assert np.allclose(om.rope(S @ x, 5, 10000.0), S @ om.rope(x, 5, 10000.0))


def test_rope_frequencies_endpoints():
    th = om.rope_frequencies(64, 10000.0)
    assert th.shape == (32,) and th[0] == 1.0
    assert abs(th[-1] - 10000.0 ** (-62.0 / 64.0)) < 1e-18


def test_cache_append_placement_and_values():
    rng = np.random.default_rng(23)
    page, d_c, d_r, hidden = 4, 6, 4, 5
    cache = rng.standard_normal((5, page, d_c + d_r))
    pt = np.array([[3, 1], [0, 4]], dtype=np.int32)
    h = rng.integers(-3, 4, size=(3, hidden)).astype(np.float64)
    W_dkv = rng.integers(-2, 3, size=(d_c, hidden)).astype(np.float64)
    W_kr = rng.integers(-2, 3, size=(d_r, hidden)).astype(np.float64)
    req, pos = np.array([0, 1, 1]), np.array([5, 0, 7])
    out = om.cache_append(cache, h, W_dkv, W_kr, req, pos, pt, 10000.0, d_c)
    # token 5 of request 0 -> page pt[0][1] = 1, row 1; token 0 of req 1 -> page 0 row 0; token 7 -> page 4 row 3
    assert np.array_equal(out[1, 1, :d_c], W_dkv @ h[0])
    assert np.array_equal(out[0, 0], np.concatenate([W_dkv @ h[1], W_kr @ h[1]]))   # pos 0: no rotation
    assert np.array_equal(out[4, 3, :d_c], W_dkv @ h[2])
    assert np.allclose(out[4, 3, d_c:], om.rope(W_kr @ h[2], 7, 10000.0))
    touched = {(1, 1), (0, 0), (4, 3)}
    for pg in range(5):
        for r in range(page):
            if (pg, r) not in touched:
                assert np.array_equal(out[pg, r], cache[pg, r])
    # pre-projected input at position 0 stores the input unchanged
    pre = rng.standard_normal((1, d_c + d_r))
    out2 = om.cache_append(cache, pre, None, None, [1], [0], pt, 10000.0, d_c)
    assert np.array_equal(out2[0, 0], pre[0])


def _golden():
    rows = {}
    with open(GOLDEN) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            key, val, _inputs, cite = [s.strip() for s in line.split("|")]
            assert cite
            rows[key] = float(val)
    return rows


def test_cache_size_arithmetic_matches_pages():
    g = _golden()
    mha = om.mha_scalars_per_token(1, 128, 128)
    lat = om.mla_scalars_per_token(512, 0)
    assert mha == g["mha_scalars_per_token_128x128"]
    assert lat == g["mla_latent_scalars"]
    assert round(100.0 * lat / mha, 2) == g["content_latent_percent_2dp"]
    assert round(100.0 - 100.0 * lat / mha, 2) == g["latent_reduction_percent_2dp"]
    assert mha // lat == g["compression_fold"] and mha % lat == 0
    assert 8 * (mha // lat) == g["concurrent_streams"]
    assert 100.0 * om.mla_scalars_per_token(512, 64) / om.gqa_scalars_per_token(8, 128) == g["gqla_absorb_cache_percent"]
    assert 100.0 * (1 - 768 / 2048) == g["converted_saving_percent"]
    assert 100.0 * om.gqa_scalars_per_token(128 // 8, 128) / om.mha_scalars_per_token(1, 128, 128) == g["gqa8_relative_percent"]
    assert om.mha_scalars_per_token(80, 64, 128) == g["mha_70b_scalars_per_token"]


def test_bytes_per_token_of_both_paths():
    assert om.absorbed_path_bytes_per_token(512, 64, 2) == 1152
    assert om.gqa_path_bytes_per_token(16, 128, 128, 64, 2) == 8320
    # at 8-way group sharding each rank holds 2 groups + the shared RoPE key: 1152 B, as much as the latent
    assert om.gqa_path_bytes_per_token(2, 128, 128, 64, 2) == 1152


# ----------------------------------------------------------------------- planted mistakes
def _bad_rope_sign(x, pos, base):
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    ang = np.asarray(pos, dtype=np.float64)[..., None] * om.rope_frequencies(d, base)
    out = np.empty(np.broadcast_shapes(x.shape, ang.shape[:-1] + (d,)))
    out[..., 0::2] = x[..., 0::2] * np.cos(ang) + x[..., 1::2] * np.sin(ang)
    out[..., 1::2] = -x[..., 0::2] * np.sin(ang) + x[..., 1::2] * np.cos(ang)
    return out


def _bad_rope_halves(x, pos, base):
    """Rotates (i, i + d/2) pairs instead of interleaved ones."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    ang = np.asarray(pos, dtype=np.float64)[..., None] * om.rope_frequencies(d, base)
    a, b = x[..., : d // 2], x[..., d // 2:]
    return np.concatenate([a * np.cos(ang) - b * np.sin(ang), a * np.sin(ang) + b * np.cos(ang)], axis=-1)


def _bad_weights_no_max(q_tilde, K, p_j, scale):
    s = scale * (K[: p_j + 1] @ q_tilde)
    e = np.exp(s)
    return e / e.sum()


def _bad_weights_off_by_one(q_tilde, K, p_j, scale):
    s = scale * (K[: p_j] @ q_tilde) if p_j > 0 else scale * (K[:1] @ q_tilde)
    e = np.exp(s - s.max())
    p = e / e.sum()
    return np.concatenate([p, np.zeros(p_j + 1 - len(p))])


def _bad_weights_no_scale(q_tilde, K, p_j, scale):
    s = K[: p_j + 1] @ q_tilde
    e = np.exp(s - s.max())
    return e / e.sum()


def _bad_qtilde_drop_rope(q_row, d_n, pos, base):
    return np.concatenate([q_row[:d_n], np.zeros(len(q_row) - d_n)])


def _bad_qtilde_wrong_pos(q_row, d_n, pos, base):
    return np.concatenate([q_row[:d_n], om.rope(q_row[d_n:], pos + 1, base)])


def _bad_combine(parts):
    M = max(m for _, m, _ in parts)
    num = sum(np.exp(m - M) * o for o, m, _ in parts)
    den = sum(l for _, m, l in parts)
    return num / den


MISTAKES = [
    ("rope", _bad_rope_sign), ("rope", _bad_rope_halves), ("attention_weights", _bad_weights_off_by_one),
    ("attention_weights", _bad_weights_no_scale), ("_q_tilde", _bad_qtilde_drop_rope),
    ("_q_tilde", _bad_qtilde_wrong_pos), ("combine_partials", _bad_combine),
]


@pytest.mark.parametrize("name,bad", MISTAKES, ids=[f"{n}:{b.__name__}" for n, b in MISTAKES])
def test_planted_mistake_is_caught(monkeypatch, name, bad):
    monkeypatch.setattr(om, name, bad)
    assert not all(pin() for pin in ALL_PINS)


def test_planted_transposed_operand_is_caught(monkeypatch):
    """Using W_UK without the transpose on a square latent (d_n == d_c) changes the result."""
    orig = om.decode_request_expanded

    def bad(q_b, rows, W_uk, W_uv, hpw, scale, base, heads=None, queries=None):
        return orig(q_b, rows, np.swapaxes(np.asarray(W_uk), 1, 2), W_uv, hpw, scale, base, heads, queries)

    monkeypatch.setattr(om, "decode_request_expanded", bad)
    rng = np.random.default_rng(30)
    p = _rand_problem(rng, d_c=4, d_n=4, lens=(5, 9))
    assert not np.allclose(_oracle_out(p), _brute_out(p), atol=1e-9)


def test_no_max_subtraction_overflows():
    """Dropping the max subtraction is caught by large scores (inf/nan instead of one-hot)."""
    K = np.array([[1.0, 0.0], [0.0, 1.0], [3.0, 0.0]])
    with np.errstate(over="ignore", invalid="ignore"):
        bad = _bad_weights_no_max(np.array([1.0, 0.0]), K, 2, 1e4)
    assert not np.array_equal(bad, [0.0, 0.0, 1.0])
