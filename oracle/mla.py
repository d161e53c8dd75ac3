"""Plain fp64 numpy oracle for MLA latent-KV decode (test infrastructure only).

The reference form is the head-expanded (non-absorbed) one: keys and values of every head
are up-projected from the cached latent, the cached RoPE key is concatenated to the key,
softmax is taken over the visible tokens and the probabilities weight the values
("MLA and GRPO architecture", "The Mathematics of MLA" and "Decoupled Rotary Position
Embeddings (RoPE)"; the paper abstract on the AI Radio GQLA episode names the
"head-expanded" form beside the absorbed one).

The absorbed and grouped forms below exist only so tests can check the pages' claim that
the decoding paths are algebraically equivalent ("GQLA: Group-Query Latent Attention for
Hardware-Adaptive Large Language Model Decoding", abstract); they are never the reference.
"""
from __future__ import annotations

import math
from typing import Iterable, List, Optional, Sequence, Tuple

import numpy as np

F64 = np.float64


# ---------------------------------------------------------------------------------------
# RoPE ("MLA and GRPO architecture", "Decoupled Rotary Position Embeddings (RoPE)":
# RoPE is applied only to the small positional vector k_t^R).  The page gives no formula;
# reading: interleaved pairs (2i, 2i+1) rotated by pos * theta_i, theta_i = base^(-2i/d).
# ---------------------------------------------------------------------------------------
def rope_frequencies(d_r: int, base: float) -> np.ndarray:
    """theta_i = base^(-2i/d_r) for i < d_r/2."""
    i = np.arange(d_r // 2, dtype=F64)
    return np.power(F64(base), -2.0 * i / d_r)


def rope(x: np.ndarray, pos, base: float) -> np.ndarray:
    """Rotate the interleaved pairs of x[..., d_r] by angle pos*theta_i (pos broadcast over x[..., 0])."""
    x = np.asarray(x, dtype=F64)
    d = x.shape[-1]
    ang = np.asarray(pos, dtype=F64)[..., None] * rope_frequencies(d, base)
    c, s = np.cos(ang), np.sin(ang)
    x0, x1 = x[..., 0::2], x[..., 1::2]
    out = np.empty(np.broadcast_shapes(x.shape, ang.shape[:-1] + (d,)), dtype=F64)
    out[..., 0::2] = x0 * c - x1 * s
    out[..., 1::2] = x0 * s + x1 * c
    return out


# ---------------------------------------------------------------------------------------
# Down-projection and the cached state ("MLA and GRPO architecture", "The Mathematics of
# MLA": c_t^KV = W_DKV h_t; "Decoupled RoPE": cached state [c_t^KV, k_t^R]).  The page does
# not name the projection that produces k_t^R; reading: k_t^R = RoPE(W_KR h_t, t).
# ---------------------------------------------------------------------------------------
def down_project(h: np.ndarray, W_dkv: Optional[np.ndarray], W_kr: Optional[np.ndarray],
                 pos, base: float, d_c: int) -> np.ndarray:
    """Cache rows [n, d_c + d_r] = [W_DKV h | RoPE(W_KR h, pos)].

    With W_dkv None, h already holds [c | k_rope before rotation] (width d_c + d_r).
    """
    h = np.asarray(h, dtype=F64)
    if W_dkv is None:
        c, kr = h[:, :d_c], h[:, d_c:]
    else:
        c = h @ np.asarray(W_dkv, F64).T
        kr = h @ np.asarray(W_kr, F64).T
    return np.concatenate([c, rope(kr, pos, base)], axis=1)


def slot_of(page_table: np.ndarray, b: int, pos: int, page: int) -> Tuple[int, int]:
    """(page id, row in page) of token ``pos`` of request ``b`` in a paged cache."""
    return int(page_table[b][pos // page]), int(pos % page)


def cache_append(cache: np.ndarray, h, W_dkv, W_kr, req_idx, positions, page_table,
                 base: float, d_c: int) -> np.ndarray:
    """Returns a copy of ``cache`` [n_pages, page, d_row] with the new rows written (fp64)."""
    out = np.array(cache, dtype=F64, copy=True)
    page = out.shape[1]
    rows = down_project(h, W_dkv, W_kr, np.asarray(positions), base, d_c)
    for i, (b, p) in enumerate(zip(req_idx, positions)):
        pg, r = slot_of(page_table, int(b), int(p), page)
        out[pg, r, :] = rows[i]
    return out


def request_rows(cache: np.ndarray, page_table: np.ndarray, b: int, L: int) -> np.ndarray:
    """The first L cached rows [L, d_row] of request b, in token order."""
    page = cache.shape[1]
    n = (L + page - 1) // page
    rows = np.concatenate([np.asarray(cache[int(page_table[b][i])], dtype=F64) for i in range(n)], axis=0)
    return rows[:L]


# ---------------------------------------------------------------------------------------
# Attention.  Query j of a request whose cache holds L tokens (the s_q current tokens
# included) sits at position p_j = L - s_q + j and sees keys t <= p_j.  Scores use the
# softmax scale given by the caller (reading: 1/sqrt(d_nope + d_rope)).
# ---------------------------------------------------------------------------------------
def attention_weights(q_tilde: np.ndarray, K: np.ndarray, p_j: int, scale: float) -> np.ndarray:
    """softmax_t( scale * q_tilde . K_t ) over t <= p_j, with max subtraction."""
    s = scale * (K[: p_j + 1] @ q_tilde)
    s = s - s.max()
    e = np.exp(s)
    return e / e.sum()


def _q_tilde(q_row: np.ndarray, d_n: int, pos: int, base: float) -> np.ndarray:
    return np.concatenate([q_row[:d_n], rope(q_row[d_n:], pos, base)])


def decode_request_expanded(q_b: np.ndarray, rows: np.ndarray, W_uk: np.ndarray, W_uv: np.ndarray,
                            hpw: int, scale: float, base: float,
                            heads: Optional[Iterable[int]] = None,
                            queries: Optional[Iterable[int]] = None) -> np.ndarray:
    """Head-expanded MLA attention of one request.

    q_b [s_q, H, d_n + d_r]; rows [L, d_c + d_r]; W_uk [n_w, d_n, d_c]; W_uv [n_w, d_v, d_c].
    Per head h (weight group w = h // hpw): K_t = [W_UK^w c_t ; k_t^R], V_t = W_UV^w c_t
    ("The Mathematics of MLA": k^C = W_UK c, v^C = W_UV c); o_h = sum_t softmax(s)_t V_t.
    Returns out [s_q, H, d_v] (rows of heads / queries not requested are NaN).
    """
    q_b = np.asarray(q_b, F64)
    rows = np.asarray(rows, F64)
    W_uk = np.asarray(W_uk, F64)
    W_uv = np.asarray(W_uv, F64)
    s_q, H, _ = q_b.shape
    n_w, d_n, d_c = W_uk.shape
    d_v = W_uv.shape[1]
    L = rows.shape[0]
    heads = list(range(H)) if heads is None else list(heads)
    queries = list(range(s_q)) if queries is None else list(queries)
    c, kr = rows[:, :d_c], rows[:, d_c:]
    out = np.full((s_q, H, d_v), np.nan)
    for w in sorted({h // hpw for h in heads}):
        K = np.concatenate([c @ W_uk[w].T, kr], axis=1)      # [L, d_n + d_r]
        V = c @ W_uv[w].T                                      # [L, d_v]
        for h in heads:
            if h // hpw != w:
                continue
            for j in queries:
                p_j = L - s_q + j
                p = attention_weights(_q_tilde(q_b[j, h], d_n, p_j, base), K, p_j, scale)
                out[j, h] = p @ V[: p_j + 1]
    return out


def decode_expanded(q, W_uk, W_uv, cache, page_table, seq_lens, hpw: int, scale: float, base: float,
                    sample: Optional[Sequence[Tuple[int, int, int]]] = None) -> np.ndarray:
    """Whole-batch decode out [B, s_q, H, d_v]; with ``sample`` = [(b, j, h), ...] only those
    outputs are computed (the rest are NaN)."""
    q = np.asarray(q, F64)
    B, s_q, H, _ = q.shape
    d_v = np.asarray(W_uv).shape[1]
    out = np.full((B, s_q, H, d_v), np.nan)
    for b in range(B):
        if sample is None:
            heads, queries = None, None
        else:
            sel = [(j, h) for (bb, j, h) in sample if bb == b]
            if not sel:
                continue
            heads = sorted({h for _, h in sel})
            queries = sorted({j for j, _ in sel})
        rows = request_rows(cache, page_table, b, int(seq_lens[b]))
        out[b] = decode_request_expanded(q[b], rows, W_uk, W_uv, hpw, scale, base, heads, queries)
    return out


# ---------------------------------------------------------------------------------------
# Alternative forms, used only to check the equivalence the GQLA pages state.
# ---------------------------------------------------------------------------------------
def decode_request_absorbed(q_b, rows, W_uk, W_uv, hpw: int, scale: float, base: float) -> np.ndarray:
    """MQA-absorb form ("Decompression Multiplex": W_UK folded into the query; the latent is the
    shared key and value): q_lat = W_UK^T q_nope, s_t = scale (q_lat . c_t + q_rope' . k_t^R),
    o = W_UV (sum_t p_t c_t)."""
    q_b, rows = np.asarray(q_b, F64), np.asarray(rows, F64)
    W_uk, W_uv = np.asarray(W_uk, F64), np.asarray(W_uv, F64)
    s_q, H, _ = q_b.shape
    n_w, d_n, d_c = W_uk.shape
    L = rows.shape[0]
    out = np.empty((s_q, H, W_uv.shape[1]))
    for h in range(H):
        w = h // hpw
        for j in range(s_q):
            p_j = L - s_q + j
            q_lat = W_uk[w].T @ q_b[j, h, :d_n]
            q_rot = rope(q_b[j, h, d_n:], p_j, base)
            s = scale * (rows[: p_j + 1, :d_c] @ q_lat + rows[: p_j + 1, d_c:] @ q_rot)
            e = np.exp(s - s.max())
            p = e / e.sum()
            out[j, h] = W_uv[w] @ (p @ rows[: p_j + 1, :d_c])
    return out


def expand_group_cache(rows, W_uk, W_uv) -> Tuple[np.ndarray, np.ndarray]:
    """Per-group expanded cache of the GQA path: K_g [n_w, L, d_n], V_g [n_w, L, d_v]."""
    rows = np.asarray(rows, F64)
    W_uk, W_uv = np.asarray(W_uk, F64), np.asarray(W_uv, F64)
    d_c = W_uk.shape[2]
    c = rows[:, :d_c]
    return np.einsum("gnc,tc->gtn", W_uk, c), np.einsum("gvc,tc->gtv", W_uv, c)


def decode_request_grouped(q_b, Kg, Vg, kr, hpw: int, scale: float, base: float) -> np.ndarray:
    """GQA path over the per-group expanded cache: head h attends to group h // hpw's K and V,
    with the shared RoPE key kr [L, d_r] concatenated to every group's key."""
    q_b = np.asarray(q_b, F64)
    s_q, H, _ = q_b.shape
    d_n = Kg.shape[2]
    L = kr.shape[0]
    out = np.empty((s_q, H, Vg.shape[2]))
    for h in range(H):
        g = h // hpw
        K = np.concatenate([Kg[g], kr], axis=1)
        for j in range(s_q):
            p_j = L - s_q + j
            p = attention_weights(_q_tilde(q_b[j, h], d_n, p_j, base), K, p_j, scale)
            out[j, h] = p @ Vg[g][: p_j + 1]
    return out


def partial_attention(q_tilde, K, V, t0: int, t1: int, scale: float):
    """Unnormalised partial softmax over keys [t0, t1): (o = sum e_t V_t, m = max s, l = sum e_t)."""
    s = scale * (K[t0:t1] @ q_tilde)
    m = s.max()
    e = np.exp(s - m)
    return e @ V[t0:t1], m, e.sum()


def combine_partials(parts) -> np.ndarray:
    """Merge partial softmaxes: M = max m_i; o = sum e^{m_i - M} o_i / sum e^{m_i - M} l_i."""
    M = max(m for _, m, _ in parts)
    num = sum(np.exp(m - M) * o for o, m, _ in parts)
    den = sum(np.exp(m - M) * l for _, m, l in parts)
    return num / den


# ---------------------------------------------------------------------------------------
# Cache-size arithmetic ("MLA and GRPO architecture" section 1 formula and "Memory Footprint
# Comparison" table; "MLA's 512-Scalar KV Latent ..." 32,768 vs 512; GQLA abstract 28.125 %).
# ---------------------------------------------------------------------------------------
def mha_scalars_per_token(n_layers: int, n_heads: int, d_head: int) -> int:
    """2 x n_layers x n_heads x d_head (one key and one value per head and layer)."""
    return 2 * n_layers * n_heads * d_head


def gqa_scalars_per_token(n_kv_heads: int, d_head: int) -> int:
    return 2 * n_kv_heads * d_head


def mla_scalars_per_token(d_c: int, d_r: int) -> int:
    """Cached state [c^KV, k^R]: d_c + d_R scalars per token and layer."""
    return d_c + d_r


def absorbed_path_bytes_per_token(d_c: int, d_r: int, elt_bytes: int) -> int:
    return (d_c + d_r) * elt_bytes


def gqa_path_bytes_per_token(n_groups: int, d_n: int, d_v: int, d_r: int, elt_bytes: int) -> int:
    """Per-group K and V plus the one shared RoPE key."""
    return (n_groups * (d_n + d_v) + d_r) * elt_bytes
