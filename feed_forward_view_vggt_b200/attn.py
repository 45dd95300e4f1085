"""ctypes binding of ``libvggt_attn.so`` -- argument marshalling only.

Every function named ``vggt_*`` mirrors the C entry point of the same name in
``include/vggt_attn.h`` and returns its status code (an int; 0 = VGGT_OK).
Tensor arguments may be CUDA ``torch`` tensors (their ``data_ptr()`` is
passed) or raw integer device addresses; ``stream`` may be a
``torch.cuda.Stream``, a raw ``cudaStream_t`` integer, or None for torch's
current stream.  The library is loaded on first use; if it has not been
built this raises -- there is no CPU fallback.

The helpers at the bottom (``frame``, ``global_``, ``sga``) allocate the
outputs with torch, call the entry points and raise ``VggtError`` on a
non-zero status.
"""
from __future__ import annotations

import ctypes
import math
import os
import re

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libvggt_attn.so")
DEBUG_LIB_PATH = os.path.join(_HERE, "libvggt_attn_debug.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "vggt_attn.h")

# The ABI this binding marshals for (VGGT_ABI_VERSION of include/vggt_attn.h);
# a library reporting another version is refused at load.
ABI_VERSION = 3

VGGT_OK = 0
VGGT_ERR_INVALID_ARG = 1
VGGT_ERR_UNSUPPORTED = 2
VGGT_ERR_WORKSPACE = 3
VGGT_ERR_CUDA = 4
VGGT_ERR_TIMEOUT = 5
VGGT_ERR_BOUNDS = 6


class VggtError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = int(status)
        super().__init__(f"{what}: {vggt_status_string(status)} ({status})" if what else
                         f"{vggt_status_string(status)} ({status})")


class vggt_shape(ctypes.Structure):
    _fields_ = [("n_frames", ctypes.c_int32), ("n_special", ctypes.c_int32),
                ("patch_h", ctypes.c_int32), ("patch_w", ctypes.c_int32),
                ("n_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32)]


class vggt_layer(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("s_h", ctypes.c_int32), ("s_w", ctypes.c_int32)]


VGGT_LAYER_FRAME, VGGT_LAYER_GLOBAL, VGGT_LAYER_SGA, VGGT_LAYER_REGISTER = 0, 1, 2, 3
_LAYER_KINDS = {"frame": VGGT_LAYER_FRAME, "global": VGGT_LAYER_GLOBAL, "sga": VGGT_LAYER_SGA,
                "register": VGGT_LAYER_REGISTER}

_lib = None


def load():
    """Loads the in-tree library (raises if it is missing).  With the
    environment variable VGGT_DEBUG=1 the library with device index checks
    (libvggt_attn_debug.so) is loaded instead."""
    global _lib
    if _lib is not None:
        return _lib
    _lib = load_library(DEBUG_LIB_PATH if os.environ.get("VGGT_DEBUG") == "1" else LIB_PATH)
    return _lib


def load_library(path: str):
    """A separate ctypes handle on one build of the library, with every
    entry point's signature set (raises if it is missing)."""
    if not os.path.exists(path):
        flag = " --debug" if path == DEBUG_LIB_PATH else ""
        raise RuntimeError(f"{path} is not built; run `python -m feed_forward_view_vggt_b200.build{flag}`")
    lib = ctypes.CDLL(path)
    i32, i64, sz, vp, f32 = ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_float
    S = vggt_shape
    sigs = {
        "vggt_status_string": ([i32], ctypes.c_char_p),
        "vggt_abi_version": ([], i32),
        "vggt_num_tokens": ([S], i64),
        "vggt_sga_num_kept": ([S, i32, i32], i64),
        "vggt_sga_num_dropped": ([S, i32, i32], i64),
        "vggt_sga_workspace_bytes": ([S, i32, i32], sz),
        "vggt_sga_build_index": ([S, i32, i32, vp, vp, vp], i32),
        "vggt_attn_frame": ([vp, vp, vp, vp, vp, S, f32, vp], i32),
        "vggt_attn_global": ([vp, vp, vp, vp, vp, S, f32, vp], i32),
        "vggt_attn_sga": ([vp, vp, vp, vp, vp, S, i32, i32, vp, vp, vp, sz, f32, vp], i32),
        "vggt_attn_sga_noalloc": ([vp, vp, vp, vp, vp, S, i32, i32, vp, vp, f32, vp], i32),
        "vggt_attn_global_rows": ([vp, i32, vp, vp, vp, vp, S, f32, vp], i32),
        "vggt_attn_sga_rows": ([vp, i32, i32, vp, vp, vp, vp, S, i32, i32, vp, vp, vp, sz, f32, vp], i32),
        "vggt_attn_register": ([vp, vp, vp, vp, vp, S, f32, vp], i32),
        "vggt_sga_partial_workspace_bytes": ([S], sz),
        "vggt_sga_gather_partial": ([vp, vp, S, i32, i32, vp, vp, vp, vp, sz, vp], i32),
        "vggt_attn_sga_gathered": ([vp, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, S, i32, i32, f32, vp], i32),
        "vggt_test_attn_global_stall": ([vp, vp, vp, vp, S, f32, ctypes.c_uint64, vp], i32),
        "vggt_check": ([vp, vp], i32),
        "vggt_schedule_workspace_bytes": ([S, vp, i32], i64),
        "vggt_qkv_rope": ([vp, vp, vp, vp, vp, vp, S, f32, vp], i32),
        "vggt_out_proj": ([vp, vp, vp, vp, S, vp], i32),
        "vggt_attn_schedule": ([vp, vp, vp, vp, S, vp, i32, f32, vp, sz, vp], i32),
        "vggt_debug_checks": ([], i32),
    }
    for name, (args, res) in sigs.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    if lib.vggt_abi_version() != ABI_VERSION:
        raise RuntimeError(f"{path} has ABI version {lib.vggt_abi_version()}, the binding expects {ABI_VERSION}; "
                           "rebuild it")
    return lib


def declared_symbols(header: str = HEADER_PATH):
    """Names of the functions declared in the public header."""
    text = open(header).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(vggt_[a-z0-9_]+)\s*\(", text)))


# ------------------------------------------------------------- marshalling

def _shape(shape) -> vggt_shape:
    if isinstance(shape, vggt_shape):
        return shape
    if isinstance(shape, (tuple, list)):
        return vggt_shape(*[int(x) for x in shape])
    # objects with N, n_special, h, w, H, d (synth.Workload, oracle.Shape)
    return vggt_shape(int(shape.N), int(shape.n_special), int(shape.h), int(shape.w), int(shape.H),
                      int(shape.d))


def _ptr(x, dtype=None, name="argument"):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    import torch

    if not isinstance(x, torch.Tensor):
        raise TypeError(f"{name}: expected a CUDA tensor or an integer device address")
    if not x.is_cuda:
        raise ValueError(f"{name}: tensor must live on a CUDA device")
    if not x.is_contiguous():
        raise ValueError(f"{name}: tensor must be contiguous")
    if dtype is not None and x.dtype != dtype:
        raise ValueError(f"{name}: expected dtype {dtype}, got {x.dtype}")
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch

        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _bf16():
    import torch

    return torch.bfloat16


def _i32():
    import torch

    return torch.int32


def _f32():
    import torch

    return torch.float32


def _layers(layers):
    """ctypes array of vggt_layer from descriptors: a vggt_layer, a kind name
    ("frame", "global", "register"), or a tuple (kind[, s_h, s_w])."""
    out = (vggt_layer * max(len(layers), 1))()
    for i, ly in enumerate(layers):
        if isinstance(ly, vggt_layer):
            out[i] = ly
            continue
        if isinstance(ly, str):
            ly = (ly,)
        kind = _LAYER_KINDS[ly[0]] if isinstance(ly[0], str) else int(ly[0])
        s_h, s_w = (int(ly[1]), int(ly[2])) if len(ly) >= 3 else (0, 0)
        out[i] = vggt_layer(kind, s_h, s_w)
    return out


def _ptr_array(xs, dtype, name):
    return (ctypes.c_void_p * max(len(xs), 1))(*[_ptr(x, dtype, name) for x in xs])


# ------------------------------------------------- entry points, same names

def vggt_status_string(status: int) -> str:
    return load().vggt_status_string(int(status)).decode()


def vggt_abi_version() -> int:
    return int(load().vggt_abi_version())


def vggt_num_tokens(shape) -> int:
    return int(load().vggt_num_tokens(_shape(shape)))


def vggt_sga_num_kept(shape, s_h: int, s_w: int) -> int:
    return int(load().vggt_sga_num_kept(_shape(shape), s_h, s_w))


def vggt_sga_num_dropped(shape, s_h: int, s_w: int) -> int:
    return int(load().vggt_sga_num_dropped(_shape(shape), s_h, s_w))


def vggt_sga_workspace_bytes(shape, s_h: int, s_w: int) -> int:
    return int(load().vggt_sga_workspace_bytes(_shape(shape), s_h, s_w))


def vggt_sga_build_index(shape, s_h, s_w, kept_idx, mult, stream=None) -> int:
    return int(load().vggt_sga_build_index(_shape(shape), s_h, s_w, _ptr(kept_idx, _i32(), "kept_idx"),
                                           _ptr(mult, _i32(), "mult"), _stream(stream)))


def vggt_attn_frame(q, k, v, o, lse, shape, scale, stream=None) -> int:
    b = _bf16()
    return int(load().vggt_attn_frame(_ptr(q, b, "q"), _ptr(k, b, "k"), _ptr(v, b, "v"), _ptr(o, b, "o"),
                                      _ptr(lse, _f32(), "lse"), _shape(shape), float(scale), _stream(stream)))


def vggt_attn_global(q, k, v, o, lse, shape, scale, stream=None) -> int:
    b = _bf16()
    return int(load().vggt_attn_global(_ptr(q, b, "q"), _ptr(k, b, "k"), _ptr(v, b, "v"), _ptr(o, b, "o"),
                                       _ptr(lse, _f32(), "lse"), _shape(shape), float(scale), _stream(stream)))


def vggt_attn_sga(q, k, v, o, lse, shape, s_h, s_w, kept_idx, mult, workspace, workspace_bytes, scale,
                  stream=None) -> int:
    b = _bf16()
    return int(load().vggt_attn_sga(_ptr(q, b, "q"), _ptr(k, b, "k"), _ptr(v, b, "v"), _ptr(o, b, "o"),
                                    _ptr(lse, _f32(), "lse"), _shape(shape), int(s_h), int(s_w),
                                    _ptr(kept_idx, _i32(), "kept_idx"), _ptr(mult, _i32(), "mult"),
                                    _ptr(workspace, None, "workspace"), int(workspace_bytes), float(scale),
                                    _stream(stream)))


def vggt_attn_sga_noalloc(q, k, v, o, lse, shape, s_h, s_w, kept_idx, mult, scale, stream=None) -> int:
    """SGA for callers that cannot allocate: the library's built-in 16 MiB
    device scratch array stands in for the workspace (see the header)."""
    b = _bf16()
    return int(load().vggt_attn_sga_noalloc(_ptr(q, b, "q"), _ptr(k, b, "k"), _ptr(v, b, "v"),
                                            _ptr(o, b, "o"), _ptr(lse, _f32(), "lse"), _shape(shape),
                                            int(s_h), int(s_w), _ptr(kept_idx, _i32(), "kept_idx"),
                                            _ptr(mult, _i32(), "mult"), float(scale), _stream(stream)))


def vggt_attn_global_rows(q_rows, n_rows, k, v, o_rows, lse_rows, shape, scale, stream=None) -> int:
    b = _bf16()
    return int(load().vggt_attn_global_rows(_ptr(q_rows, b, "q_rows"), int(n_rows), _ptr(k, b, "k"), _ptr(v, b, "v"),
                                            _ptr(o_rows, b, "o_rows"), _ptr(lse_rows, _f32(), "lse_rows"),
                                            _shape(shape), float(scale), _stream(stream)))


def vggt_attn_sga_rows(q_rows, row0, n_rows, k, v, o_rows, lse_rows, shape, s_h, s_w, kept_idx, mult, workspace,
                       workspace_bytes, scale, stream=None) -> int:
    b = _bf16()
    return int(load().vggt_attn_sga_rows(_ptr(q_rows, b, "q_rows"), int(row0), int(n_rows), _ptr(k, b, "k"),
                                         _ptr(v, b, "v"), _ptr(o_rows, b, "o_rows"), _ptr(lse_rows, _f32(), "lse_rows"),
                                         _shape(shape), int(s_h), int(s_w), _ptr(kept_idx, _i32(), "kept_idx"),
                                         _ptr(mult, _i32(), "mult"), _ptr(workspace, None, "workspace"),
                                         int(workspace_bytes), float(scale), _stream(stream)))


def vggt_sga_partial_workspace_bytes(local_shape) -> int:
    return int(load().vggt_sga_partial_workspace_bytes(_shape(local_shape)))


def vggt_sga_gather_partial(k, v, local_shape, s_h, s_w, kept_k, kept_v, dropped_sums, workspace, workspace_bytes,
                            stream=None) -> int:
    b = _bf16()
    return int(load().vggt_sga_gather_partial(_ptr(k, b, "k"), _ptr(v, b, "v"), _shape(local_shape), int(s_h),
                                              int(s_w), _ptr(kept_k, b, "kept_k"), _ptr(kept_v, b, "kept_v"),
                                              _ptr(dropped_sums, _f32(), "dropped_sums"),
                                              _ptr(workspace, None, "workspace"), int(workspace_bytes),
                                              _stream(stream)))


def vggt_attn_sga_gathered(q_rows, row0, n_rows, k_rows, v_rows, kept_k, kept_v, dropped_sums, mult, means, o_rows,
                           lse_rows, shape, s_h, s_w, scale, stream=None) -> int:
    b = _bf16()
    return int(load().vggt_attn_sga_gathered(_ptr(q_rows, b, "q_rows"), int(row0), int(n_rows),
                                             _ptr(k_rows, b, "k_rows"), _ptr(v_rows, b, "v_rows"),
                                             _ptr(kept_k, b, "kept_k"), _ptr(kept_v, b, "kept_v"),
                                             _ptr(dropped_sums, _f32(), "dropped_sums"), _ptr(mult, _i32(), "mult"),
                                             _ptr(means, _f32(), "means"), _ptr(o_rows, b, "o_rows"),
                                             _ptr(lse_rows, _f32(), "lse_rows"), _shape(shape), int(s_h), int(s_w),
                                             float(scale), _stream(stream)))


def vggt_test_attn_global_stall(q, k, v, o, shape, scale, wait_limit_ns, stream=None) -> int:
    """Failure-path test hook: global attention whose first scores are never
    signalled, with in-kernel waits bounded by wait_limit_ns (see header)."""
    b = _bf16()
    return int(load().vggt_test_attn_global_stall(_ptr(q, b, "q"), _ptr(k, b, "k"), _ptr(v, b, "v"),
                                                  _ptr(o, b, "o"), _shape(shape), float(scale),
                                                  int(wait_limit_ns), _stream(stream)))


def vggt_attn_register(q, k, v, o, lse, shape, scale, stream=None) -> int:
    b = _bf16()
    return int(load().vggt_attn_register(_ptr(q, b, "q"), _ptr(k, b, "k"), _ptr(v, b, "v"), _ptr(o, b, "o"),
                                         _ptr(lse, _f32(), "lse"), _shape(shape), float(scale), _stream(stream)))


def vggt_schedule_workspace_bytes(shape, layers) -> int:
    return int(load().vggt_schedule_workspace_bytes(_shape(shape), _layers(layers), len(layers)))


def vggt_attn_schedule(qs, ks, vs, os_, shape, layers, scale, workspace, workspace_bytes, stream=None) -> int:
    b = _bf16()
    n = len(layers)
    return int(load().vggt_attn_schedule(_ptr_array(qs, b, "q"), _ptr_array(ks, b, "k"), _ptr_array(vs, b, "v"),
                                         _ptr_array(os_, b, "o"), _shape(shape), _layers(layers), n, scale,
                                         _ptr(workspace, None, "workspace"), workspace_bytes, _stream(stream)))


def vggt_qkv_rope(x, w, bias, q, k, v, shape, rope_base, stream=None) -> int:
    b = _bf16()
    return int(load().vggt_qkv_rope(_ptr(x, b, "x"), _ptr(w, b, "w"), _ptr(bias, _f32(), "bias"), _ptr(q, b, "q"),
                                    _ptr(k, b, "k"), _ptr(v, b, "v"), _shape(shape), rope_base, _stream(stream)))


def vggt_out_proj(o, w, bias, y, shape, stream=None) -> int:
    b = _bf16()
    return int(load().vggt_out_proj(_ptr(o, b, "o"), _ptr(w, b, "w"), _ptr(bias, _f32(), "bias"), _ptr(y, b, "y"),
                                    _shape(shape), _stream(stream)))


def vggt_check(stream=None):
    """(status, detail word); synchronises the stream."""
    detail = ctypes.c_uint32(0)
    st = int(load().vggt_check(_stream(stream), ctypes.byref(detail)))
    return st, int(detail.value)


# ----------------------------------------------------------- conveniences

def _raise(status: int, what: str):
    if status != VGGT_OK:
        raise VggtError(status, what)


def default_scale(head_dim: int = 64) -> float:
    return 1.0 / math.sqrt(head_dim)


def frame(q, k, v, shape, scale=None, want_lse=False, stream=None):
    import torch

    o = torch.empty_like(q)
    sh = _shape(shape)
    lse = torch.empty(q.shape[0], q.shape[1], dtype=torch.float32, device=q.device) if want_lse else None
    _raise(vggt_attn_frame(q, k, v, o, lse, sh, default_scale(sh.head_dim) if scale is None else scale, stream), "vggt_attn_frame")
    return (o, lse) if want_lse else o


def global_(q, k, v, shape, scale=None, want_lse=False, stream=None):
    import torch

    o = torch.empty_like(q)
    sh = _shape(shape)
    lse = torch.empty(q.shape[0], q.shape[1], dtype=torch.float32, device=q.device) if want_lse else None
    _raise(vggt_attn_global(q, k, v, o, lse, sh, default_scale(sh.head_dim) if scale is None else scale, stream),
           "vggt_attn_global")
    return (o, lse) if want_lse else o


class SgaIndex:
    """Device-side SGA index (kept list + multiplicities) for one shape and
    stride, built once by vggt_sga_build_index and reusable across heads and
    layers; also owns a workspace of vggt_sga_workspace_bytes."""

    def __init__(self, shape, s_h: int, s_w: int, device=None, stream=None):
        import torch

        self.shape = _shape(shape)
        self.s_h, self.s_w = int(s_h), int(s_w)
        self.n_kept = vggt_sga_num_kept(self.shape, s_h, s_w)
        self.n_dropped = vggt_sga_num_dropped(self.shape, s_h, s_w)
        if self.n_kept < 0:
            raise VggtError(VGGT_ERR_INVALID_ARG, "SgaIndex")
        S = vggt_num_tokens(self.shape)
        device = device or torch.device("cuda")
        self.kept_idx = torch.empty(max(self.n_kept, 1), dtype=torch.int32, device=device)
        self.mult = torch.empty(S, dtype=torch.int32, device=device)
        self.workspace_bytes = vggt_sga_workspace_bytes(self.shape, s_h, s_w)
        self.workspace = torch.empty(self.workspace_bytes, dtype=torch.uint8, device=device)
        _raise(vggt_sga_build_index(self.shape, s_h, s_w, self.kept_idx, self.mult, stream),
               "vggt_sga_build_index")

    def means(self):
        """(kbar, vbar) fp32 [H, 64] as left in the workspace by the last call."""
        hd = self.shape.n_heads * 64
        f = self.workspace[: 8 * hd].view(_f32())
        return f[:hd].view(self.shape.n_heads, 64), f[hd:2 * hd].view(self.shape.n_heads, 64)


def sga(q, k, v, index: SgaIndex, scale=None, want_lse=False, stream=None):
    import torch

    o = torch.empty_like(q)
    lse = torch.empty(q.shape[0], q.shape[1], dtype=torch.float32, device=q.device) if want_lse else None
    _raise(vggt_attn_sga(q, k, v, o, lse, index.shape, index.s_h, index.s_w, index.kept_idx, index.mult,
                         index.workspace, index.workspace_bytes,
                         default_scale(index.shape.head_dim) if scale is None else scale, stream), "vggt_attn_sga")
    return (o, lse) if want_lse else o


def register(q, k, v, shape, scale=None, want_lse=False, o=None, stream=None):
    """Register attention; returns O (patch-token rows are those of ``o`` if
    given, else uninitialised)."""
    import torch

    sh = _shape(shape)
    o = torch.empty_like(q) if o is None else o
    lse = torch.empty(q.shape[0], q.shape[1], dtype=torch.float32, device=q.device) if want_lse else None
    _raise(vggt_attn_register(q, k, v, o, lse, sh, default_scale(sh.head_dim) if scale is None else scale, stream),
           "vggt_attn_register")
    return (o, lse) if want_lse else o


def schedule(qs, ks, vs, shape, layers, os_=None, scale=None, stream=None):
    """Runs a layer schedule: layer i reads qs[i], ks[i], vs[i] and writes
    os_[i] (allocated if not given; register layers write only the
    special-token rows).  Returns the list of outputs."""
    import torch

    sh = _shape(shape)
    n = len(layers)
    if not (len(qs) == len(ks) == len(vs) == n):
        raise ValueError("one q, k and v per layer")
    os_ = [torch.empty_like(q) for q in qs] if os_ is None else os_
    nbytes = vggt_schedule_workspace_bytes(sh, layers)
    if nbytes < 0:
        raise VggtError(VGGT_ERR_INVALID_ARG, "vggt_schedule_workspace_bytes")
    ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=qs[0].device) if n else None
    _raise(vggt_attn_schedule(qs, ks, vs, os_, sh, layers, default_scale(sh.head_dim) if scale is None else scale,
                              ws, nbytes, stream), "vggt_attn_schedule")
    return os_


def qkv_rope(x, w, shape, bias=None, rope_base=100.0, stream=None):
    """Fused QKV projection + 2D RoPE; returns (q, k, v), each [S, H, 64]."""
    import torch

    sh = _shape(shape)
    S = x.shape[0]
    q, k, v = (torch.empty(S, sh.n_heads, sh.head_dim, dtype=x.dtype, device=x.device) for _ in range(3))
    _raise(vggt_qkv_rope(x, w, bias, q, k, v, sh, rope_base, stream), "vggt_qkv_rope")
    return q, k, v


def out_proj(o, w, shape, bias=None, stream=None):
    """Output projection y = o W^T + b; returns y, [S, C]."""
    import torch

    sh = _shape(shape)
    y = torch.empty(o.shape[0], sh.n_heads * sh.head_dim, dtype=o.dtype, device=o.device)
    _raise(vggt_out_proj(o, w, bias, y, sh, stream), "vggt_out_proj")
    return y
