"""Attention-layer schedules of an alternating-attention trunk.

Host logic only: lists of layer descriptors for ``vggt_attn_schedule``
(``"frame"``, ``"global"``, ``"register"`` or ``("sga", s_h, s_w)``), in
trunk order.  Sources, cited by page title and section:

* "VGGT CVPR25 Best Paper" notes, "Alternating-Attention": the trunk is a
  stack of blocks, each a frame-wise attention layer followed by a global
  attention layer.
* "AVGGT: Rethinking Global Attention for Accelerating VGGT", sections 2
  and 3.  The global layers play three roles by depth (early, middle,
  last).  Step one turns the early global layers into frame attention.
  Step two runs SGA in the remaining global layers.
* VGGT-Omega notes, improvement one "Register Attention": a quarter of the
  global layers become register attention.

Readings where the pages are silent:

* The number of blocks is not given.  ``DEPTH = 24`` is the default, and
  every builder takes the depth as an argument.
* How many global layers count as "early" is not given.  The first third
  is taken, i.e. the first of the three roles the analysis names.
* Which global layers become register attention is not given.  Every
  fourth one is taken (global layers 3, 7, 11, ... counted from 0), which
  spreads the quarter evenly over depth.
"""
from __future__ import annotations

DEPTH = 24


def vggt_trunk(depth: int = DEPTH):
    """VGGT: ``depth`` blocks of (frame, global)."""
    if depth < 0:
        raise ValueError("depth must be >= 0")
    out = []
    for _ in range(depth):
        out += ["frame", "global"]
    return out


def avggt_trunk(depth: int = DEPTH, converted: int | None = None, stride=(2, 2)):
    """AVGGT: the first ``converted`` global layers become frame attention
    (default: the first third) and the others SGA with ``stride``."""
    if depth < 0:
        raise ValueError("depth must be >= 0")
    converted = depth // 3 if converted is None else int(converted)
    if not 0 <= converted <= depth:
        raise ValueError("converted must lie in [0, depth]")
    s_h, s_w = int(stride[0]), int(stride[1])
    out = []
    for i in range(depth):
        out += ["frame", "frame" if i < converted else ("sga", s_h, s_w)]
    return out


def omega_trunk(depth: int = DEPTH, every: int = 4):
    """VGGT-Omega: every ``every``-th global layer (counted from 0, the
    last of each group) becomes register attention."""
    if depth < 0 or every < 1:
        raise ValueError("depth must be >= 0 and every >= 1")
    out = []
    for i in range(depth):
        out += ["frame", "register" if i % every == every - 1 else "global"]
    return out


def kind_counts(layers):
    """{kind: count} of a schedule, SGA layers keyed by (\"sga\", s_h, s_w)."""
    counts: dict = {}
    for ly in layers:
        key = ly if isinstance(ly, str) else tuple(ly)
        counts[key] = counts.get(key, 0) + 1
    return counts
