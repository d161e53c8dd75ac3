"""Helpers for the GPU parity tests: upload seeded inputs, call the C ABI through the binding,
and compare with the oracle under the stated tolerances."""
import numpy as np
import torch

import mla_latent_kv_24_b200 as mla
import workloads as wl

# bf16 inputs, fp32 accumulation: normwise max relative error and mean absolute error.
BF16_REL, BF16_MAE = 1e-2, 1e-3
FP32_REL = 1e-5
# Scale-free mean error for bf16: the GPU rounds q_abs, P and the output to bf16 (unit roundoff
# 2^-9 each), which moves the mean relative error by a few 1e-3 at most; 1e-2 leaves a margin of
# several times that while still failing a dropped term or a wrong index at any output scale.
BF16_MAE_REL = 1e-2


def dims_of(w: wl.Workload):
    return mla.make_dims(n_heads=w.H, heads_per_group=w.hpw, d_c=w.d_c, d_rope=w.d_r, d_nope=w.d_n, d_v=w.d_v,
                         page_size=w.page, softmax_scale=w.softmax_scale, rope_base=w.rope_base, dtype=w.dtype)


class Dev:
    """Device copies of one workload's inputs."""

    def __init__(self, inp: wl.DecodeInputs, device="cuda"):
        self.inp = inp
        w = inp.w
        self.q = wl.to_torch(inp.q, device)
        self.W_uk = wl.to_torch(inp.W_uk, device)
        self.W_uv = wl.to_torch(inp.W_uv, device)
        self.cache = wl.to_torch(inp.cache, device)
        self.page_table = torch.from_numpy(inp.page_table).to(device)
        self.seq_lens = torch.from_numpy(inp.seq_lens).to(device)
        self.max_pages = inp.page_table.shape[1]
        self.dims = dims_of(w)
        self.tdtype = torch.bfloat16 if w.dtype == "bf16" else torch.float32

    def decode_absorbed(self, out=None, lens_host=None):
        w = self.inp.w
        lens_host = self.inp.seq_lens if lens_host is None else lens_host
        nb = mla.mla_decode_workspace_size(self.dims, w.B, w.s_q, self.inp.seq_lens)
        ws = torch.empty(max(nb, 256), dtype=torch.uint8, device=self.q.device)
        out = torch.empty((w.B, w.s_q, w.H, w.d_v), dtype=self.tdtype, device=self.q.device) if out is None else out
        mla.mla_decode_absorbed(self.dims, self.q, self.W_uk, self.W_uv, self.cache, self.page_table, self.seq_lens,
                                lens_host, w.B, w.s_q, self.max_pages, self.inp.n_pages, out, ws)
        return out

    def expand(self):
        w = self.inp.w
        G = w.H // w.hpw
        exp = torch.empty((self.inp.n_pages, G, w.page, w.d_n + w.d_v), dtype=self.tdtype, device=self.q.device)
        mla.gqla_expand_cache(self.dims, self.W_uk, self.W_uv, self.cache, None, 0, self.inp.n_pages, exp)
        return exp

    def decode_grouped(self, expanded):
        w = self.inp.w
        nb = mla.gqla_decode_workspace_size(self.dims, w.B, w.s_q, self.inp.seq_lens)
        ws = torch.empty(max(nb, 256), dtype=torch.uint8, device=self.q.device)
        out = torch.empty((w.B, w.s_q, w.H, w.d_v), dtype=self.tdtype, device=self.q.device)
        mla.gqla_decode_grouped(self.dims, self.q, expanded, self.cache, self.page_table, self.seq_lens,
                                self.inp.seq_lens, w.B, w.s_q, self.max_pages, self.inp.n_pages, out, ws)
        return out


def prefill(dev: "Dev", expanded):
    """Head-expanded prefill of the workload's last s_q tokens (n_q = s_q) through the C ABI."""
    w = dev.inp.w
    nb = mla.mla_prefill_workspace_size(dev.dims, w.B, w.s_q, dev.inp.seq_lens)
    ws = torch.empty(max(nb, 256), dtype=torch.uint8, device=dev.q.device)
    out = torch.empty((w.B, w.s_q, w.H, w.d_v), dtype=dev.tdtype, device=dev.q.device)
    mla.mla_prefill_expanded(dev.dims, dev.q, expanded, dev.cache, dev.page_table, dev.seq_lens, dev.inp.seq_lens,
                             w.B, w.s_q, dev.max_pages, dev.inp.n_pages, out, ws)
    return out


def errors(got: np.ndarray, ref: np.ndarray):
    """(normwise max relative error, mean absolute error) over the finite entries of ref."""
    f = figures(got, ref)
    return f["rel"], f["mae"]


def figures(got: np.ndarray, ref: np.ndarray) -> dict:
    """Every error figure of one comparison, over the finite entries of ref:
    rel       max|g - o| / max|o|              (normwise; gated in every test)
    mae       mean|g - o|                      (absolute; gated for bf16)
    mae_rel   mean|g - o| / mean|o|            (scale-free: at long contexts |o| is ~1e-3, where an
                                                absolute MAE bound says little)
    elem_max  max |g - o| / |o| over entries with |o| > 0.1 rms(o)   (element-wise, reported)
    elem_p99  its 99th percentile                                      (reported)"""
    m = np.isfinite(ref)
    g, r = got[m].astype(np.float64), ref[m].astype(np.float64)
    d = np.abs(g - r)
    a = np.abs(r)
    big = a > 0.1 * np.sqrt(np.mean(r * r))
    el = d[big] / a[big] if big.any() else np.zeros(1)
    return {"rel": float(d.max() / a.max()), "mae": float(d.mean()), "mae_rel": float(d.mean() / a.mean()),
            "elem_max": float(el.max()), "elem_p99": float(np.percentile(el, 99)), "n": int(d.size)}


# Figures of every comparison in this process, printed as a table at the end of the run.
REPORT = []


def assert_close(got: np.ndarray, ref: np.ndarray, dtype: str, what: str = ""):
    assert np.isfinite(got[np.isfinite(ref)]).all(), f"{what}: non-finite GPU output"
    f = figures(got, ref)
    REPORT.append((what, dtype, f))
    rel, mae = f["rel"], f["mae"]
    msg = f"{what}: rel {rel:.3e} mae {mae:.3e} mae_rel {f['mae_rel']:.3e} elem_max {f['elem_max']:.3e}"
    if dtype == "bf16":
        assert rel <= BF16_REL and mae <= BF16_MAE, msg
        assert f["mae_rel"] <= BF16_MAE_REL, msg
    else:
        assert rel <= FP32_REL, msg
    return rel, mae


def oracle_decode(inp: wl.DecodeInputs, sample=None):
    import oracle
    w = inp.w
    return oracle.decode_expanded(inp.q.f64(), inp.W_uk.f64(), inp.W_uv.f64(), inp.cache.f64(), inp.page_table,
                                  inp.seq_lens, w.hpw, w.softmax_scale, w.rope_base, sample=sample)


def sample_outputs(inp: wl.DecodeInputs, n: int, seed: int = 99):
    """n distinct (b, j, h) output rows, always including the longest request and the last head."""
    w = inp.w
    rng = np.random.default_rng(seed)
    picks = {(int(np.argmax(inp.seq_lens)), w.s_q - 1, w.H - 1), (0, 0, 0)}
    while len(picks) < n:
        picks.add((int(rng.integers(w.B)), int(rng.integers(w.s_q)), int(rng.integers(w.H))))
    return sorted(picks)


def oracle_decode_sampled(inp: wl.DecodeInputs, sample):
    """Oracle outputs for the sampled (b, j, h) rows only, converting just the cache rows of the
    sampled requests to float64 (full-size caches do not fit in memory as float64)."""
    import oracle
    w = inp.w
    q = inp.q.f64()
    W_uk, W_uv = inp.W_uk.f64(), inp.W_uv.f64()
    out = {}
    for b in sorted({s[0] for s in sample}):
        L = int(inp.seq_lens[b])
        n = (L + w.page - 1) // w.page
        bits = inp.cache.data[inp.page_table[b, :n]].reshape(n * w.page, w.d_row)[:L]
        rows = wl.bf16_bits_to_f64(bits) if w.dtype == "bf16" else bits.astype(np.float64)
        sel = [(j, h) for (bb, j, h) in sample if bb == b]
        res = oracle.decode_request_expanded(q[b], rows, W_uk, W_uv, w.hpw, w.softmax_scale, w.rope_base,
                                             heads=sorted({h for _, h in sel}), queries=sorted({j for j, _ in sel}))
        for j, h in sel:
            out[(b, j, h)] = res[j, h]
    return out


def compare_sampled(got: np.ndarray, ref: dict, dtype: str, what: str):
    keys = sorted(ref)
    g = np.stack([got[k] for k in keys])
    r = np.stack([ref[k] for k in keys])
    return assert_close(g, r, dtype, what)
