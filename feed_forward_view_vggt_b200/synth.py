"""Seeded synthetic inputs of VGGT shape for the attention hot path.

This module only draws random numbers and picks sample rows; it holds none
of the attention arithmetic, so both the CUDA path and the fp64 oracle can
be fed from it without sharing any of the method's code.

Token layout: N frames, each n_special = 5 special tokens (camera/register
style; 17 in the VGGT-Omega layout) followed by an h x w grid of
14x14-pixel patch tokens, row-major;
a 518x518 view gives 37 x 37 = 1369 patches ("Vggt cvpr2025 dissection",
section 2.5 worked example).  Tensors are bf16 [S, H, d], S = N * L,
L = 5 + h * w, token-major (the global-attention view of [N, L, H, d]).

Value recipe (stand-ins for the pages' datasets, which are not available):
  * tiny: Q, K, V i.i.d. N(0, 1), drawn in that order.
  * other workloads: Q, V ~ N(0, 1); K = b[p] + 0.5 * e with the base b ~
    N(0, 1) shared by the same in-frame position p across all frames
    (cross-frame correspondence structure) and e ~ N(0, 1) per token.
    Draw order: Q, base, noise, V (then outliers).
  * "outliers": exactly floor(0.1 * S) tokens, chosen uniformly without
    replacement, get K redrawn i.i.d. N(0, 1) for all heads.
All draws come from one torch CPU generator seeded per workload, one frame
at a time (so memory stays bounded at N = 800), then round to bf16
(round-to-nearest-even).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    N: int
    h: int
    w: int
    H: int
    seed: int
    structure: str  # "iid" | "corr" | "corr_outliers"
    sga_strides: tuple = ((2, 2),)
    n_special: int = 5
    d: int = 64
    ops: tuple = ("frame", "global", "sga")
    note: str = field(default="", compare=False)

    @property
    def L(self) -> int:
        return self.n_special + self.h * self.w

    @property
    def S(self) -> int:
        return self.N * self.L


WORKLOADS = {
    "tiny": Workload("tiny", N=2, h=8, w=8, H=2, seed=0, structure="iid",
                     note="N=2, 8x8 patches + 5 specials = 69 tokens/frame, H=2, d=64"),
    "n4": Workload("n4", N=4, h=37, w=37, H=16, seed=1, structure="corr",
                   note="worked example: 4 views of 518x518, 1374 tokens/frame"),
    "n32": Workload("n32", N=32, h=37, w=37, H=16, seed=2, structure="corr",
                    sga_strides=((2, 2), (3, 3))),
    "n100": Workload("n100", N=100, h=37, w=37, H=16, seed=3, structure="corr_outliers",
                     note="headline: 137,400 tokens"),
    "n300": Workload("n300", N=300, h=37, w=37, H=16, seed=6, structure="corr",
                     note="412,200 tokens: the 300-frame point of the AVGGT speedup figures"),
    "n800": Workload("n800", N=800, h=37, w=37, H=16, seed=4, structure="corr",
                     sga_strides=((3, 3), (2, 2)), note="1,099,200 tokens"),
    # VGGT-Omega token layout: 16 registers + 1 camera token per frame
    "omega100": Workload("omega100", N=100, h=37, w=37, H=16, seed=5, structure="corr", n_special=17,
                         note="register-attention layout: 17 special tokens per frame, 138,600 tokens"),
}


def _randn_bf16(gen: torch.Generator, *shape) -> torch.Tensor:
    return torch.randn(*shape, generator=gen, dtype=torch.float32).to(torch.bfloat16)


def make_qkv(wl: Workload):
    """Seeded (Q, K, V) as CPU bf16 tensors of shape [S, H, d]."""
    g = torch.Generator().manual_seed(wl.seed)
    S, L, H, d = wl.S, wl.L, wl.H, wl.d
    if wl.structure == "iid":
        q = _randn_bf16(g, S, H, d)
        k = _randn_bf16(g, S, H, d)
        v = _randn_bf16(g, S, H, d)
        return q, k, v
    q = torch.empty(S, H, d, dtype=torch.bfloat16)
    k = torch.empty(S, H, d, dtype=torch.bfloat16)
    v = torch.empty(S, H, d, dtype=torch.bfloat16)
    for n in range(wl.N):
        q[n * L:(n + 1) * L] = _randn_bf16(g, L, H, d)
    base = torch.randn(L, H, d, generator=g, dtype=torch.float32)
    for n in range(wl.N):
        e = torch.randn(L, H, d, generator=g, dtype=torch.float32)
        k[n * L:(n + 1) * L] = (base + 0.5 * e).to(torch.bfloat16)
    for n in range(wl.N):
        v[n * L:(n + 1) * L] = _randn_bf16(g, L, H, d)
    if wl.structure == "corr_outliers":
        n_out = int(math.floor(0.1 * S))
        idx = torch.randperm(S, generator=g)[:n_out]
        k[idx] = _randn_bf16(g, n_out, H, d)
    elif wl.structure != "corr":
        raise ValueError(f"unknown structure {wl.structure!r}")
    return q, k, v


def make_qkv_heads(wl: Workload, h0: int, h1: int):
    """Heads [h0, h1) of make_qkv(wl): the seeded (Q, K, V) of one
    head-sharded rank, each [S, h1 - h0, d].  The correspondence workloads
    are drawn from the same random stream one frame at a time, so only the
    slice is held."""
    if not 0 <= h0 < h1 <= wl.H:
        raise ValueError("head range must satisfy 0 <= h0 < h1 <= H")
    g = torch.Generator().manual_seed(wl.seed)
    S, L, H, d = wl.S, wl.L, wl.H, wl.d
    hs = h1 - h0
    q = torch.empty(S, hs, d, dtype=torch.bfloat16)
    k = torch.empty(S, hs, d, dtype=torch.bfloat16)
    v = torch.empty(S, hs, d, dtype=torch.bfloat16)
    if wl.structure == "iid":  # small workloads only: the same three whole draws as make_qkv
        return tuple(_randn_bf16(g, S, H, d)[:, h0:h1].contiguous() for _ in range(3))
    for n in range(wl.N):
        q[n * L:(n + 1) * L] = _randn_bf16(g, L, H, d)[:, h0:h1]
    base = torch.randn(L, H, d, generator=g, dtype=torch.float32)
    for n in range(wl.N):
        e = torch.randn(L, H, d, generator=g, dtype=torch.float32)
        k[n * L:(n + 1) * L] = (base + 0.5 * e).to(torch.bfloat16)[:, h0:h1]
    for n in range(wl.N):
        v[n * L:(n + 1) * L] = _randn_bf16(g, L, H, d)[:, h0:h1]
    if wl.structure == "corr_outliers":
        n_out = int(math.floor(0.1 * S))
        idx = torch.randperm(S, generator=g)[:n_out]
        k[idx] = _randn_bf16(g, n_out, H, d)[:, h0:h1]
    elif wl.structure != "corr":
        raise ValueError(f"unknown structure {wl.structure!r}")
    return q, k, v


def sample_rows(S: int, L: int, n_special: int = 5, count: int = 4096, seed: int = 1234):
    """Seeded query-token sample, ascending int64.

    Always contains token 0, token S-1, the special tokens of frame 0, the
    ragged tail of frame 0 (tokens past its last multiple of 256) and the
    ragged tail of the whole sequence; the rest are uniform without
    replacement from a numpy generator seeded with ``seed``."""
    if count >= S:
        return np.arange(S, dtype=np.int64)
    forced = {0, S - 1}
    forced.update(range(min(n_special, S)))
    tail_f = L % 256
    forced.update(range(max(0, L - (tail_f or 256)), min(L, S)))
    tail_s = S % 256
    forced.update(range(max(0, S - (tail_s or 256)), S))
    forced = sorted(forced)[:count]
    rng = np.random.default_rng(seed)
    pool = np.setdiff1d(np.arange(S, dtype=np.int64), np.asarray(forced, dtype=np.int64))
    extra = rng.choice(pool, size=count - len(forced), replace=False)
    return np.sort(np.concatenate([np.asarray(forced, dtype=np.int64), extra]))
