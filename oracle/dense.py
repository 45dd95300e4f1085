"""fp64 attention for sampled query rows, with each head's logits for a
block of rows taken from one matrix product.

TEST INFRASTRUCTURE ONLY.  Same callers as the rest of ``oracle/``: the
test-suite, the smoke check and the benchmark's CPU-baseline leg; the CUDA
library and its binding never import it, and it imports nothing from them.

What it computes is what ``vggt_oracle.c`` computes, for the same four
modes (sources cited there and in ``oracle/__init__.py``):
  * frame attention -- keys = the query's own frame ("VGGT CVPR25 Best
    Paper" notes, "Alternating-Attention");
  * global attention -- keys = all S tokens (same section);
  * SGA -- keys = the kept set, plus the query's own key when it was
    dropped, plus the mean column with logit scale * q.kbar + ln M_i
    ("AVGGT: Rethinking Global Attention for Accelerating VGGT", technical
    summary section 3 step two; readings as in ``vggt_oracle.c``);
  * register attention -- queries and keys = the special tokens of all
    frames (VGGT-Omega notes, improvement one "Register Attention").

Why a second form: the C oracle walks one (row, head) at a time with scalar
dot products, about 0.3 s per global-attention row at N = 800 (1,099,200
keys) on 16 cores, so a 4096-row sample would take twenty minutes.  Here
the dot products of a block of query rows with all keys of one head are one
fp64 ``torch.matmul`` (a library primitive, run on the host's cores), and
the value sum is another.  Nothing else changes: per (row, head) the logit
list is the same, the softmax is two-pass (the row maximum first, then the
sum of exp(logit - max)) in fp64, and the kept list, the multiplicities and
the means over the dropped set come from the C oracle's own functions
(``sga_build_index``, ``sga_means``).  Query rows are independent, so
cutting them into blocks reorders no sum.

Every bf16 input is widened exactly to fp64 before any arithmetic.
"""
from __future__ import annotations

import math

import numpy as np
import torch

from . import FRAME, GLOBAL, REGISTER, SGA, Shape, _bits, sga_build_index, sga_means, special_rows

# Query rows per matrix product (the fastest of 8 to 128 on the host: the
# logits of 16 rows stay in the last-level cache at N = 100).
ROW_BLOCK = 16


def _as_bf16(x) -> torch.Tensor:
    """uint16 bit patterns (or a CPU bf16 tensor) as a torch bf16 view."""
    return torch.from_numpy(_bits(x).view(np.int16)).view(torch.bfloat16)


def _softmax_rows(logits: torch.Tensor, values: torch.Tensor, extra_l=None, extra_v=None):
    """Two-pass softmax over each row of `logits` [B, n] (fp64) with
    `values` [n, d]; `extra_l` [B, e] / `extra_v` [B, e, d] are further
    columns with their own value vectors (-inf logits are absent columns).
    Returns (out [B, d], lse [B])."""
    m = logits.max(dim=1).values
    if extra_l is not None:
        m = torch.maximum(m, extra_l.max(dim=1).values)
    p = logits.sub_(m[:, None]).exp_()  # in place: the logits are not needed again
    denom = p.sum(dim=1)
    acc = p @ values
    if extra_l is not None:
        pe = torch.exp(extra_l - m[:, None])  # exp(-inf) = 0: an absent column adds nothing
        denom = denom + pe.sum(dim=1)
        acc = acc + (pe[:, :, None] * extra_v).sum(dim=1)
    return acc / denom[:, None], m + torch.log(denom)


def attention(mode: int, q, k, v, shape: Shape, scale: float | None = None,
              s_h: int = 1, s_w: int = 1, rows=None, row_block: int = ROW_BLOCK):
    """fp64 attention outputs for query tokens ``rows`` (default: all S), all
    heads.  Same arguments and results as ``oracle.attention``:
    (out [nrows, H, d] float64, lse [nrows, H] float64)."""
    if mode not in (FRAME, GLOBAL, SGA, REGISTER):
        raise ValueError(f"unknown mode {mode}")
    qt, kt, vt = _as_bf16(q), _as_bf16(k), _as_bf16(v)
    S, H, d, L = shape.S, shape.H, shape.d, shape.L
    for name, a in (("q", qt), ("k", kt), ("v", vt)):
        if tuple(a.shape) != (S, H, d):
            raise ValueError(f"{name} has shape {tuple(a.shape)}, expected {(S, H, d)}")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    rows = np.arange(S, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64)
    if rows.size and (rows.min() < 0 or rows.max() >= S):
        raise ValueError("row index out of range")
    if mode == REGISTER and rows.size and (rows % L >= shape.n_special).any():
        raise ValueError("register attention is defined for special-token rows only")
    rows_t = torch.from_numpy(rows)
    out = torch.zeros(len(rows), H, d, dtype=torch.float64)
    lse = torch.zeros(len(rows), H, dtype=torch.float64)

    if mode == SGA:
        kept, mult, n_kept, n_dropped = sga_build_index(shape, s_h, s_w)
        kept_t = torch.from_numpy(kept.astype(np.int64))
        mult_rows = torch.from_numpy(mult[rows].astype(np.int64))
        means = sga_means(k, v, shape, s_h, s_w) if n_dropped > 0 else None
        # the query's own key is a column only when it was dropped
        dropped_rows = mult_rows == n_dropped - 1 if n_dropped > 0 else torch.zeros(len(rows), dtype=torch.bool)
    elif mode == REGISTER:
        key_tokens = torch.from_numpy(special_rows(shape))

    for h in range(H):
        qh = qt[rows_t, h, :].double()
        if mode == FRAME:
            frames = rows // L
            for f in np.unique(frames):
                sel = torch.from_numpy(np.nonzero(frames == f)[0])
                kh = kt[f * L:(f + 1) * L, h, :].double()
                vh = vt[f * L:(f + 1) * L, h, :].double()
                o_, l_ = _softmax_rows((qh[sel] @ kh.T) * scale, vh)
                out[sel, h], lse[sel, h] = o_, l_
            continue
        if mode == GLOBAL:
            kh, vh = kt[:, h, :].double(), vt[:, h, :].double()
        elif mode == REGISTER:
            kh, vh = kt[key_tokens, h, :].double(), vt[key_tokens, h, :].double()
        else:
            kh, vh = kt[kept_t, h, :].double(), vt[kept_t, h, :].double()
        for b0 in range(0, len(rows), row_block):
            b1 = min(len(rows), b0 + row_block)
            logits = (qh[b0:b1] @ kh.T) * scale
            if mode != SGA:
                o_, l_ = _softmax_rows(logits, vh)
            else:
                nb = b1 - b0
                blk = rows_t[b0:b1]
                extra_l = torch.full((nb, 2), -math.inf, dtype=torch.float64)
                extra_v = torch.zeros(nb, 2, d, dtype=torch.float64)
                own_k = kt[blk, h, :].double()
                own_v = vt[blk, h, :].double()
                diag = (qh[b0:b1] * own_k).sum(dim=1) * scale
                dr = dropped_rows[b0:b1]
                extra_l[:, 0] = torch.where(dr, diag, torch.tensor(-math.inf, dtype=torch.float64))
                extra_v[:, 0] = own_v
                if means is not None:
                    kbar = torch.from_numpy(means[0][h])
                    vbar = torch.from_numpy(means[1][h])
                    M = mult_rows[b0:b1]
                    mean_l = (qh[b0:b1] @ kbar) * scale + torch.log(M.clamp(min=1).double())
                    extra_l[:, 1] = torch.where(M > 0, mean_l, torch.tensor(-math.inf, dtype=torch.float64))
                    extra_v[:, 1] = vbar
                o_, l_ = _softmax_rows(logits, vh, extra_l, extra_v)
            out[b0:b1, h], lse[b0:b1, h] = o_, l_
    return out.numpy(), lse.numpy()


def frame_attention(q, k, v, shape, scale=None, rows=None):
    return attention(FRAME, q, k, v, shape, scale, rows=rows)


def global_attention(q, k, v, shape, scale=None, rows=None):
    return attention(GLOBAL, q, k, v, shape, scale, rows=rows)


def sga_attention(q, k, v, shape, s_h, s_w, scale=None, rows=None):
    return attention(SGA, q, k, v, shape, scale, s_h=s_h, s_w=s_w, rows=rows)


def register_attention(q, k, v, shape, scale=None, rows=None):
    if rows is None:
        rows = special_rows(shape)
    return attention(REGISTER, q, k, v, shape, scale, rows=rows)
