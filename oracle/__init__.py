"""Plain fp64 CPU oracle for VGGT frame / global attention and AVGGT SGA.

TEST INFRASTRUCTURE ONLY.  Callers: the test-suite (``tests/``), the smoke
check in ``__graft_entry__.smoke()`` and the CPU-baseline / reference leg of
``bench.py``.  The CUDA library and its Python binding never import this
package, and this package never imports them: the two share only the seeded
input generator, which holds none of the method's arithmetic.

The arithmetic lives in ``vggt_oracle.c`` (fp64, two-pass softmax, libm
``exp``); this module builds it with gcc and marshals numpy arrays.
``dense.py`` holds the same attention definitions with each head's logits
for a block of query rows taken from one fp64 matrix product, for samples
too large for the scalar C loops (N = 800); it is pinned against them.

Sources followed (cited by page title and section):
  * "VGGT CVPR25 Best Paper" notes, "Alternating-Attention": frame-wise vs
    global self-attention.
  * VGGT-Omega notes, improvement one "Register Attention": cross-frame
    attention restricted to the register/camera (special) tokens.
  * "AVGGT: Rethinking Global Attention for Accelerating VGGT", section 3
    step two (SGA): query retention, grid K/V sampling, diagonal
    preservation, mean-fill, shared softmax normalisation.
  * "Feed-forward optimization in Visual Geometry Grounded and 3DGS", Cut3R
    part, section 3.5 (position encoding): RoPE on Q and K before every
    attention (``qkv_rope``: the projection that produces Q, K, V, with a
    2D rotary embedding; the exact form is a reading).

Inputs are bf16 bit patterns as ``numpy.uint16`` arrays of shape [S, H, d]
(token-major, S = N * L, L = n_special + h * w).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "vggt_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

FRAME, GLOBAL, SGA, REGISTER = 0, 1, 2, 3

_lib = None


@dataclass(frozen=True)
class Shape:
    """Token layout of one attention layer: N frames of n_special special
    tokens followed by an h x w patch grid, H heads of width d."""

    N: int
    n_special: int
    h: int
    w: int
    H: int
    d: int

    @property
    def L(self) -> int:
        return self.n_special + self.h * self.w

    @property
    def S(self) -> int:
        return self.N * self.L


def build(force: bool = False) -> str:
    """Compile vggt_oracle.c into liboracle.so (portable x86-64-v2 code)."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    tmp = _LIB + ".tmp.%d" % os.getpid()
    cmd = ["gcc", "-O3", "-march=x86-64-v2", "-mtune=generic", "-std=c11", "-fPIC",
           "-shared", "-pthread", "-Wall", "-Wno-unused-function", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    i32, i64, dbl, vp = ctypes.c_int, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
    lib.oracle_hardware_threads.restype = i32
    lib.oracle_axis_kept.argtypes = [i32, i32, vp]
    lib.oracle_axis_kept.restype = i32
    lib.oracle_sga_build_index.argtypes = [i32, i32, i32, i32, i32, i32, vp, vp, vp, vp]
    lib.oracle_sga_build_index.restype = i32
    lib.oracle_sga_means.argtypes = [vp, vp, i32, i32, i32, i32, i32, i32, i32, i32, vp, vp]
    lib.oracle_sga_means.restype = i32
    lib.oracle_attn.argtypes = [i32, vp, vp, vp, i32, i32, i32, i32, i32, i32, dbl,
                                i32, i32, vp, i64, vp, vp, i32]
    lib.oracle_attn.restype = i32
    lib.oracle_qkv_rope.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, i32, dbl, vp, i64, vp, vp, vp, i32]
    lib.oracle_qkv_rope.restype = i32
    lib.oracle_linear.argtypes = [vp, vp, vp, i64, i32, i32, vp, i64, vp]
    lib.oracle_linear.restype = i32
    _lib = lib
    return lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def _bits(x) -> np.ndarray:
    """bf16 input as a C-contiguous uint16 array (accepts numpy uint16 or a
    CPU torch.bfloat16 tensor)."""
    if isinstance(x, np.ndarray):
        if x.dtype != np.uint16:
            raise TypeError("oracle inputs are bf16 bit patterns (uint16)")
        return np.ascontiguousarray(x)
    import torch  # only for the CPU tensor view

    if x.dtype != torch.bfloat16 or x.is_cuda:
        raise TypeError("oracle inputs must be CPU bf16 tensors or uint16 arrays")
    return np.ascontiguousarray(x.contiguous().view(torch.int16).numpy().view(np.uint16))


def hardware_threads() -> int:
    return int(_load().oracle_hardware_threads())


def axis_kept(n: int, s: int) -> np.ndarray:
    """Kept coordinates on one grid axis (one per window, the window centre)."""
    lib = _load()
    cnt = lib.oracle_axis_kept(n, s, None)
    out = np.zeros(max(cnt, 1), dtype=np.int32)
    lib.oracle_axis_kept(n, s, _ptr(out))
    return out[:cnt]


def sga_build_index(shape: Shape, s_h: int, s_w: int):
    """(kept_idx int32[n_kept] ascending, mult int32[S], n_kept, n_dropped)."""
    lib = _load()
    nk, nd = ctypes.c_int64(0), ctypes.c_int64(0)
    rc = lib.oracle_sga_build_index(shape.N, shape.n_special, shape.h, shape.w, s_h, s_w,
                                    None, None, ctypes.byref(nk), ctypes.byref(nd))
    if rc != 0:
        raise ValueError("invalid SGA index arguments")
    kept = np.zeros(max(nk.value, 1), dtype=np.int32)
    mult = np.zeros(max(shape.S, 1), dtype=np.int32)
    lib.oracle_sga_build_index(shape.N, shape.n_special, shape.h, shape.w, s_h, s_w,
                               _ptr(kept), _ptr(mult), None, None)
    return kept[: nk.value], mult[: shape.S], int(nk.value), int(nd.value)


def sga_means(k, v, shape: Shape, s_h: int, s_w: int):
    """fp64 (kbar, vbar), each [H, d], summed directly over the dropped set;
    None when no token is dropped."""
    kb, vb = _bits(k), _bits(v)
    kbar = np.zeros((shape.H, shape.d), dtype=np.float64)
    vbar = np.zeros((shape.H, shape.d), dtype=np.float64)
    rc = _load().oracle_sga_means(_ptr(kb), _ptr(vb), shape.N, shape.n_special, shape.h,
                                  shape.w, shape.H, shape.d, s_h, s_w, _ptr(kbar), _ptr(vbar))
    return None if rc != 0 else (kbar, vbar)


def attention(mode: int, q, k, v, shape: Shape, scale: float | None = None,
              s_h: int = 1, s_w: int = 1, rows=None, nthreads: int = 0):
    """fp64 attention outputs for query tokens ``rows`` (default: all S).

    Returns (out [nrows, H, d] float64, lse [nrows, H] float64)."""
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    expect = (shape.S, shape.H, shape.d)
    for name, a in (("q", qb), ("k", kb), ("v", vb)):
        if a.shape != expect:
            raise ValueError(f"{name} has shape {a.shape}, expected {expect}")
    if scale is None:
        scale = 1.0 / np.sqrt(shape.d)
    if rows is None:
        rows = np.arange(shape.S, dtype=np.int64)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    out = np.zeros((len(rows), shape.H, shape.d), dtype=np.float64)
    lse = np.zeros((len(rows), shape.H), dtype=np.float64)
    rc = _load().oracle_attn(mode, _ptr(qb), _ptr(kb), _ptr(vb), shape.N, shape.n_special,
                             shape.h, shape.w, shape.H, shape.d, float(scale), s_h, s_w,
                             _ptr(rows), len(rows), _ptr(out), _ptr(lse), int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle_attn failed with code {rc}")
    return out, lse


def frame_attention(q, k, v, shape, scale=None, rows=None, nthreads=0):
    return attention(FRAME, q, k, v, shape, scale, rows=rows, nthreads=nthreads)


def global_attention(q, k, v, shape, scale=None, rows=None, nthreads=0):
    return attention(GLOBAL, q, k, v, shape, scale, rows=rows, nthreads=nthreads)


def sga_attention(q, k, v, shape, s_h, s_w, scale=None, rows=None, nthreads=0):
    return attention(SGA, q, k, v, shape, scale, s_h=s_h, s_w=s_w, rows=rows, nthreads=nthreads)


def special_rows(shape: Shape):
    """Token indices of every special token, frame by frame."""
    return (np.arange(shape.N, dtype=np.int64)[:, None] * shape.L +
            np.arange(shape.n_special, dtype=np.int64)[None, :]).reshape(-1)


def register_attention(q, k, v, shape, scale=None, rows=None, nthreads=0):
    """Register attention for special-token rows (default: all of them)."""
    if rows is None:
        rows = special_rows(shape)
    return attention(REGISTER, q, k, v, shape, scale, rows=rows, nthreads=nthreads)


def qkv_rope(x, w, bias, shape: Shape, base: float = 100.0, rows=None, nthreads: int = 0):
    """fp64 fused QKV projection + 2D RoPE (see vggt_oracle.c).

    x: bf16 [S, C] (C = H*d); w: bf16 [3C, C]; bias: float32 [3C] or None.
    Returns (q, k, v), each float64 [nrows, H, d]."""
    xb, wb = _bits(x), _bits(w)
    C = shape.H * shape.d
    if xb.shape != (shape.S, C) or wb.shape != (3 * C, C):
        raise ValueError(f"x {xb.shape} / w {wb.shape} do not match S={shape.S}, C={C}")
    b = None if bias is None else np.ascontiguousarray(np.asarray(bias, dtype=np.float32).reshape(3 * C))
    if rows is None:
        rows = np.arange(shape.S, dtype=np.int64)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    q, k, v = (np.zeros((len(rows), C), dtype=np.float64) for _ in range(3))
    rc = _load().oracle_qkv_rope(_ptr(xb), _ptr(wb), None if b is None else _ptr(b), shape.N, shape.n_special,
                                 shape.h, shape.w, shape.H, shape.d, float(base), _ptr(rows), len(rows),
                                 _ptr(q), _ptr(k), _ptr(v), int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle_qkv_rope failed with code {rc}")
    return tuple(a.reshape(len(rows), shape.H, shape.d) for a in (q, k, v))


def linear(x, w, bias=None, rows=None):
    """fp64 y = x W^T + b for the rows ``rows`` of x (bf16 [R, n_in]);
    w bf16 [n_out, n_in]; bias float32 [n_out] or None."""
    xb, wb = _bits(x), _bits(w)
    n_rows, n_in = xb.shape
    n_out = wb.shape[0]
    if wb.shape[1] != n_in:
        raise ValueError("w does not match x")
    b = None if bias is None else np.ascontiguousarray(np.asarray(bias, dtype=np.float32).reshape(n_out))
    rows = np.arange(n_rows, dtype=np.int64) if rows is None else np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    y = np.zeros((len(rows), n_out), dtype=np.float64)
    rc = _load().oracle_linear(_ptr(xb), _ptr(wb), None if b is None else _ptr(b), n_rows, n_in, n_out, _ptr(rows),
                               len(rows), _ptr(y))
    if rc != 0:
        raise ValueError(f"oracle_linear failed with code {rc}")
    return y
