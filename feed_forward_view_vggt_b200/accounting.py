"""Closed-form work accounting for the attention hot path.

Counts only the method's own work (the dense work SGA avoids is not
counted).  FLOPs count a multiply-add as 2.

  frame   : 4 * N * L^2 * H * d        (QK^T and PV within each frame)
  global  : 4 * S^2 * H * d            (all S = N*L tokens as one sequence)
  SGA     : 4 * S * (n_kept + 1) * H * d   (kept keys + the mean column)
            + 4 * |D| * H * d              (diagonal term of dropped queries)
  mean-fill bytes read: 2 tensors (K, V) * N*h*w patch tokens * H*d * 2 B

The dense attention-matrix size reproduces the memory estimate in the
"VGGT CVPR25 Best Paper" notes ("Alternating-Attention" section):
102,400 tokens -> 1.05e10 entries -> 21 GB fp16 / 42 GB fp32.
"""
from __future__ import annotations


def attention_matrix_entries(tokens: int) -> int:
    return tokens * tokens


def attention_matrix_bytes(tokens: int, bytes_per_entry: int) -> int:
    return attention_matrix_entries(tokens) * bytes_per_entry


def axis_windows(n: int, s: int) -> int:
    """Number of stride-s windows on an axis of length n (a shorter last
    window counts)."""
    return -(-n // s)


def sga_counts(N: int, n_special: int, h: int, w: int, s_h: int, s_w: int):
    """(n_kept, n_dropped) for SGA with stride (s_h, s_w): every special
    token plus one patch per window is kept in each frame."""
    kept_patches = axis_windows(h, s_h) * axis_windows(w, s_w)
    n_kept = N * (n_special + kept_patches)
    n_dropped = N * (h * w - kept_patches)
    return n_kept, n_dropped


def flops_frame(N: int, L: int, H: int, d: int) -> int:
    return 4 * N * L * L * H * d


def flops_global(S: int, H: int, d: int) -> int:
    return 4 * S * S * H * d


def flops_sga(S: int, n_kept: int, n_dropped: int, H: int, d: int) -> int:
    return 4 * S * (n_kept + 1) * H * d + 4 * n_dropped * H * d


def meanfill_read_bytes(N: int, h: int, w: int, H: int, d: int) -> int:
    return 2 * N * h * w * H * d * 2


def exps(S: int, keys_per_query: int, H: int) -> int:
    return S * keys_per_query * H


def flops_register(N: int, n_special: int, H: int, d: int) -> int:
    """Register attention: global attention over the N * n_special special
    tokens only."""
    return flops_global(N * n_special, H, d)


def flops_schedule(layers, N: int, n_special: int, h: int, w: int, H: int, d: int) -> int:
    """Algorithmic FLOP of a layer schedule (see schedules.py)."""
    L = n_special + h * w
    S = N * L
    total = 0
    for ly in layers:
        kind = ly if isinstance(ly, str) else ly[0]
        if kind == "frame":
            total += flops_frame(N, L, H, d)
        elif kind == "global":
            total += flops_global(S, H, d)
        elif kind == "register":
            total += flops_register(N, n_special, H, d)
        elif kind == "sga":
            kept, dropped = sga_counts(N, n_special, h, w, int(ly[1]), int(ly[2]))
            total += flops_sga(S, kept, dropped, H, d)
        else:
            raise ValueError(f"unknown layer kind {kind!r}")
    return total
