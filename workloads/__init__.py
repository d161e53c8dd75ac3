"""Seeded synthetic inputs for MLA latent-KV decode workloads.

This module is shared by the tests, the bench and the CPU oracle's callers.  It only
draws random numbers, rounds them to the storage dtype and lays them out (page tables,
sequence lengths).  It holds none of the attention arithmetic: no projection, no RoPE,
no softmax.

Recipe (the pages fix none of it, so it is this repository's own):
  * one ``numpy.random.default_rng(seed)`` (PCG64) per workload, drawn in the fixed
    order: sequence lengths -> page permutation -> W_UK -> W_UV -> W_DKV -> W_KR ->
    latent cache (row chunks of 65536 rows, c_kv and k_rope together) -> q -> h;
  * float32 standard normals scaled by the stated standard deviation, then rounded once
    to bfloat16 (round to nearest even) for the bf16 workloads; the fp32 workload keeps
    the float32 values;
  * weights std 0.02, latents / RoPE keys / queries / hidden states std 1 (bf16 workloads);
    the tiny fp32 workload uses std 1/sqrt(fan_in) with fan_in = d_c for W_UK/W_UV and the
    vector's own length for c_kv (d_c), k_rope (d_rope) and q (d_nope + d_rope);
  * ragged lengths are log-uniform: round(exp(U[ln lo, ln hi])), clipped to [lo, hi];
  * a shuffled page table is a random permutation of a pool of exactly
    sum_b ceil(L_b / page) pages; otherwise request b owns consecutive pages.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional, Sequence

import numpy as np

PAGE = 64


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and distribution of one decode workload."""

    name: str
    dtype: str            # "bf16" or "fp32"
    B: int
    H: int
    d_c: int
    d_r: int
    d_n: int
    d_v: int
    hpw: int              # query heads per weight group: 1 = MLA, 8 = GQLA
    s_q: int
    seed: int
    hidden: int = 5120
    lens: Optional[Sequence[int]] = None     # uniform lengths if given
    lens_loguniform: Optional[Sequence[int]] = None  # (lo, hi)
    shuffle_pages: bool = False
    page: int = PAGE
    rope_base: float = 10000.0

    @property
    def n_w(self) -> int:
        return self.H // self.hpw

    @property
    def d_qk(self) -> int:
        return self.d_n + self.d_r

    @property
    def d_row(self) -> int:
        return self.d_c + self.d_r

    @property
    def softmax_scale(self) -> float:
        # Length of the head-expanded dot product: no-position part + RoPE part.
        return 1.0 / math.sqrt(self.d_n + self.d_r)


def _mla(name, **kw) -> Workload:
    base = dict(dtype="bf16", H=128, d_c=512, d_r=64, d_n=128, d_v=128, hpw=1, hidden=5120)
    base.update(kw)
    return Workload(name=name, **base)


#: The five workloads.  Keys are the workload numbers used on the command line.
WORKLOADS: Dict[str, Workload] = {
    "1": Workload(name="tiny_fp32_b1_h4_l64", dtype="fp32", B=1, H=4, d_c=32, d_r=8, d_n=16,
                  d_v=16, hpw=1, s_q=1, seed=0, hidden=64, lens=[64]),
    "2": _mla("dsv2_b8_l4096_sq1", B=8, s_q=1, seed=1, lens=[4096] * 8),
    "3": _mla("longctx_b4_l131072_sq1", B=4, s_q=1, seed=2, lens=[131072] * 4),
    "4": _mla("ragged_b64_l1k_32k_sq2_shuffled", B=64, s_q=2, seed=3,
              lens_loguniform=(1024, 32768), shuffle_pages=True),
}
for _L in (8192, 16384, 32768, 65536):
    for _sq in (1, 2):
        WORKLOADS[f"5_{_L}_{_sq}"] = _mla(f"gqla_16x8_b32_l{_L}_sq{_sq}", B=32, s_q=_sq, seed=4,
                                          hpw=8, lens=[_L] * 32)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest, ties to even); returns the uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float64."""
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32)


class Tensor:
    """Host array in storage form: ``bits`` (uint16 for bf16, float32 for fp32)."""

    def __init__(self, data: np.ndarray, dtype: str):
        self.data = data
        self.dtype = dtype

    @property
    def shape(self):
        return self.data.shape

    def f64(self) -> np.ndarray:
        if self.dtype == "bf16":
            return bf16_bits_to_f64(self.data)
        return self.data.astype(np.float64)


def _draw(rng: np.random.Generator, shape, std: float, dtype: str) -> Tensor:
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    if dtype == "bf16":
        return Tensor(f32_to_bf16_bits(x), "bf16")
    return Tensor(x, "fp32")


def seq_lens(w: Workload, rng: np.random.Generator) -> np.ndarray:
    if w.lens is not None:
        return np.asarray(w.lens, dtype=np.int32)
    lo, hi = w.lens_loguniform
    u = rng.uniform(math.log(lo), math.log(hi), size=w.B)
    return np.clip(np.rint(np.exp(u)), lo, hi).astype(np.int32)


def page_table(w: Workload, lens: np.ndarray, rng: np.random.Generator):
    """Returns (page_table [B, max_pages] int32, n_pages_total)."""
    n_per = [(int(L) + w.page - 1) // w.page for L in lens]
    total = int(sum(n_per))
    max_pages = max(n_per)
    ids = np.arange(total, dtype=np.int32)
    if w.shuffle_pages:
        ids = rng.permutation(total).astype(np.int32)
    pt = np.zeros((w.B, max_pages), dtype=np.int32)
    off = 0
    for b, n in enumerate(n_per):
        pt[b, :n] = ids[off:off + n]
        off += n
    return pt, total


@dataclasses.dataclass
class DecodeInputs:
    w: Workload
    seq_lens: np.ndarray          # [B] int32
    page_table: np.ndarray        # [B, max_pages] int32
    n_pages: int
    W_uk: Tensor                  # [n_w, d_n, d_c]
    W_uv: Tensor                  # [n_w, d_v, d_c]
    W_dkv: Tensor                 # [d_c, hidden]
    W_kr: Tensor                  # [d_r, hidden]
    cache: Tensor                 # [n_pages, page, d_c + d_r]
    q: Tensor                     # [B, s_q, H, d_n + d_r]
    h: Tensor                     # [B * s_q, hidden] hidden states of the new tokens


CHUNK_ROWS = 65536


def make_inputs(w: Workload, seed: Optional[int] = None, lens: Optional[Sequence[int]] = None) -> DecodeInputs:
    """Draws every input of one workload (see the module docstring for the recipe)."""
    rng = np.random.default_rng(w.seed if seed is None else seed)
    L = np.asarray(lens, dtype=np.int32) if lens is not None else seq_lens(w, rng)
    pt, n_pages = page_table(w, L, rng)
    if w.dtype == "fp32":
        s_w, s_c, s_r, s_q = 1 / math.sqrt(w.d_c), 1 / math.sqrt(w.d_c), 1 / math.sqrt(w.d_r), 1 / math.sqrt(w.d_qk)
        s_p, s_h = 1 / math.sqrt(w.hidden), 1.0
    else:
        s_w = s_p = 0.02
        s_c = s_r = s_q = s_h = 1.0
    W_uk = _draw(rng, (w.n_w, w.d_n, w.d_c), s_w, w.dtype)
    W_uv = _draw(rng, (w.n_w, w.d_v, w.d_c), s_w, w.dtype)
    W_dkv = _draw(rng, (w.d_c, w.hidden), s_p, w.dtype)
    W_kr = _draw(rng, (w.d_r, w.hidden), s_p, w.dtype)
    rows = n_pages * w.page
    store = np.uint16 if w.dtype == "bf16" else np.float32
    cache = np.empty((rows, w.d_row), dtype=store)
    for r0 in range(0, rows, CHUNK_ROWS):
        r1 = min(rows, r0 + CHUNK_ROWS)
        x = rng.standard_normal(size=(r1 - r0, w.d_row), dtype=np.float32)
        if s_c != 1.0:
            x[:, :w.d_c] *= np.float32(s_c)
        if s_r != 1.0:
            x[:, w.d_c:] *= np.float32(s_r)
        cache[r0:r1] = f32_to_bf16_bits(x) if w.dtype == "bf16" else x
    cache = Tensor(cache.reshape(n_pages, w.page, w.d_row), w.dtype)
    q = _draw(rng, (w.B, w.s_q, w.H, w.d_qk), s_q, w.dtype)
    h = _draw(rng, (w.B * w.s_q, w.hidden), s_h, w.dtype)
    return DecodeInputs(w=w, seq_lens=L, page_table=pt, n_pages=n_pages, W_uk=W_uk, W_uv=W_uv,
                        W_dkv=W_dkv, W_kr=W_kr, cache=cache, q=q, h=h)


def small_workload(base: Workload, **kw) -> Workload:
    """A copy of ``base`` with some fields replaced (test-sized variants)."""
    return dataclasses.replace(base, **kw)


def new_token_positions(lens: np.ndarray, s_q: int):
    """(request index, position) of the s_q newest tokens of each request, request-major."""
    req, pos = [], []
    for b, L in enumerate(lens):
        for j in range(s_q):
            req.append(b)
            pos.append(int(L) - s_q + j)
    return np.asarray(req, dtype=np.int32), np.asarray(pos, dtype=np.int32)


__all__ = ["Workload", "WORKLOADS", "DecodeInputs", "make_inputs", "Tensor", "PAGE",
           "f32_to_bf16_bits", "bf16_bits_to_f64", "bf16_bits_to_f32", "small_workload",
           "new_token_positions", "seq_lens", "page_table"]


def to_torch(t: Tensor, device="cuda"):
    """Copies a host tensor to torch (bf16 bit patterns become torch.bfloat16)."""
    import torch
    if t.dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(t.data).view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(t.data)).to(device)


def from_torch_f64(x) -> np.ndarray:
    """Exact float64 copy of a torch tensor (bf16 or fp32) on any device."""
    import torch
    return x.detach().to("cpu", torch.float64).numpy()
