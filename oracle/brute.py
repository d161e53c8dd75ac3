"""Pure-Python brute-force MLA decode for tiny inputs (test infrastructure only).

Written with Python floats and explicit index loops, no numpy, straight from the
definitions in "MLA and GRPO architecture" ("The Mathematics of MLA": k^C = W_UK c,
v^C = W_UV c; "Decoupled RoPE": key = [k^C ; k^R]).  It pins the numpy oracle in
``oracle/mla.py``; it is far too slow for anything but tiny shapes.
"""
from __future__ import annotations

import math


def rope_pairs(x, pos, base):
    """Rotate interleaved pairs (2i, 2i+1) of list x by pos * base^(-2i/d)."""
    d = len(x)
    out = [0.0] * d
    for i in range(d // 2):
        ang = pos * base ** (-2.0 * i / d)
        c, s = math.cos(ang), math.sin(ang)
        a, b = x[2 * i], x[2 * i + 1]
        out[2 * i] = a * c - b * s
        out[2 * i + 1] = a * s + b * c
    return out


def decode_one(q_row, rows, W_uk_w, W_uv_w, d_c, d_n, pos, scale, base):
    """One head, one query at position ``pos``; rows = list of cache rows [c | k_r]."""
    d_v = len(W_uv_w)
    q_n = q_row[:d_n]
    q_r = rope_pairs(q_row[d_n:], pos, base)
    scores = []
    values = []
    for t in range(pos + 1):
        c = rows[t][:d_c]
        kr = rows[t][d_c:]
        s = 0.0
        for i in range(d_n):
            k_i = 0.0
            for k in range(d_c):
                k_i += W_uk_w[i][k] * c[k]
            s += q_n[i] * k_i
        for i in range(len(kr)):
            s += q_r[i] * kr[i]
        scores.append(scale * s)
        v = []
        for o in range(d_v):
            acc = 0.0
            for k in range(d_c):
                acc += W_uv_w[o][k] * c[k]
            v.append(acc)
        values.append(v)
    mx = max(scores)
    e = [math.exp(s - mx) for s in scores]
    z = sum(e)
    return [sum(e[t] / z * values[t][o] for t in range(len(e))) for o in range(d_v)]


def decode(q, W_uk, W_uv, rows_per_request, s_q, hpw, d_c, d_n, scale, base):
    """q[b][j][h] lists; rows_per_request[b] = the L_b cache rows of request b."""
    out = []
    for b, rows in enumerate(rows_per_request):
        L = len(rows)
        ob = []
        for j in range(s_q):
            pos = L - s_q + j
            oj = []
            for h in range(len(q[b][j])):
                w = h // hpw
                oj.append(decode_one(q[b][j][h], rows, W_uk[w], W_uv[w], d_c, d_n, pos, scale, base))
            ob.append(oj)
        out.append(ob)
    return out
