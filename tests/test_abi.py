"""C-ABI boundary checks that need no GPU: the library loads, exports every
symbol the header declares, computes the closed-form SGA counts, rejects bad
arguments before queuing anything, and fails loudly (VGGT_ERR_CUDA) when no
device is present -- there is no CPU fallback."""
import numpy as np
import pytest
import torch

import oracle
from feed_forward_view_vggt_b200 import accounting, attn
from feed_forward_view_vggt_b200 import build as vbuild

SHAPE = attn.vggt_shape(4, 5, 37, 37, 16, 64)
A = 1 << 28  # fake, 16-byte aligned "device" addresses: never dereferenced on these paths


@pytest.fixture(scope="module", autouse=True)
def built():
    vbuild.build()
    attn.load()


def no_gpu():
    return not torch.cuda.is_available()


def test_exports_every_declared_symbol():
    names = attn.declared_symbols()
    assert {"vggt_attn_frame", "vggt_attn_global", "vggt_attn_sga", "vggt_sga_build_index"} <= set(names)
    lib = attn.load()
    for n in names:
        assert hasattr(lib, n), n


def test_debug_build_loads_and_reports_itself():
    # the -DVGGT_DEBUG library: same exports, device index checks compiled in
    vbuild.build(debug=True)
    dbg = attn.load_library(attn.DEBUG_LIB_PATH)
    for n in attn.declared_symbols():
        assert hasattr(dbg, n), n
    assert dbg.vggt_debug_checks() == 1 and attn.load().vggt_debug_checks() == 0
    assert dbg.vggt_status_string(attn.VGGT_ERR_BOUNDS) == b"VGGT_ERR_BOUNDS"
    # argument checks are the same in both builds
    assert dbg.vggt_attn_global(None, None, None, None, None, SHAPE, 0.125, None) == attn.VGGT_ERR_INVALID_ARG


def test_status_strings_and_version():
    import re

    header_version = int(re.search(r"#define VGGT_ABI_VERSION (\d+)", open(attn.HEADER_PATH).read()).group(1))
    assert attn.vggt_abi_version() == header_version == attn.ABI_VERSION == 3
    for code, name in [(0, "VGGT_OK"), (1, "VGGT_ERR_INVALID_ARG"), (2, "VGGT_ERR_UNSUPPORTED"),
                       (3, "VGGT_ERR_WORKSPACE"), (4, "VGGT_ERR_CUDA"), (5, "VGGT_ERR_TIMEOUT"),
                       (6, "VGGT_ERR_BOUNDS")]:
        assert attn.vggt_status_string(code) == name
    assert attn.vggt_status_string(99) == "VGGT_ERR_UNKNOWN"


@pytest.mark.parametrize("N,ns,h,w,sh,sw", [(100, 5, 37, 37, 2, 2), (800, 5, 37, 37, 3, 3),
                                            (2, 5, 8, 8, 2, 2), (3, 0, 7, 5, 4, 2), (1, 5, 1, 2, 1, 2),
                                            (2, 5, 8, 8, 1, 1), (2, 3, 6, 4, 8, 8)])
def test_counts_match_oracle(N, ns, h, w, sh, sw):
    shape = attn.vggt_shape(N, ns, h, w, 16, 64)
    _, _, nk, nd = oracle.sga_build_index(oracle.Shape(N, ns, h, w, 16, 64), sh, sw)
    assert attn.vggt_sga_num_kept(shape, sh, sw) == nk
    assert attn.vggt_sga_num_dropped(shape, sh, sw) == nd
    assert attn.vggt_num_tokens(shape) == N * (ns + h * w)
    ws = attn.vggt_sga_workspace_bytes(shape, sh, sw)
    assert ws >= 2 * nk * 16 * 64 * 2 + 8 * 16 * 64 and ws % 256 == 0


def test_invalid_shapes_and_strides():
    assert attn.vggt_sga_num_kept(SHAPE, 0, 2) == -1
    assert attn.vggt_sga_num_kept(SHAPE, 2, -1) == -1
    assert attn.vggt_num_tokens(attn.vggt_shape(0, 5, 37, 37, 16, 64)) == -1
    assert attn.vggt_num_tokens(attn.vggt_shape(1, 0, 0, 0, 16, 64)) == -1
    assert attn.vggt_sga_workspace_bytes(attn.vggt_shape(4, 5, 37, 37, 16, 128), 2, 2) == 0


def call_frame(q=A, k=2 * A, v=3 * A, o=4 * A, lse=None, shape=SHAPE, scale=0.125):
    return attn.load().vggt_attn_frame(q, k, v, o, lse, shape, scale, None)


def call_sga(ws=8 * A, ws_bytes=None, kept=5 * A, mult=6 * A, sh=2, sw=2, shape=SHAPE, o=4 * A):
    if ws_bytes is None:
        ws_bytes = attn.vggt_sga_workspace_bytes(shape, sh, sw)
    return attn.load().vggt_attn_sga(A, 2 * A, 3 * A, o, None, shape, sh, sw, kept, mult, ws,
                                     ws_bytes, 0.125, None)


def test_rejects_bad_pointers_before_launch():
    E = attn.VGGT_ERR_INVALID_ARG
    assert call_frame(q=None) == E
    assert call_frame(o=None) == E
    assert call_frame(k=2 * A + 8) == E           # misaligned
    assert call_frame(lse=5 * A + 2) == E         # misaligned lse
    assert call_frame(o=A + 64) == E              # O overlaps Q
    assert call_frame(scale=0.0) == E
    assert call_frame(scale=float("nan")) == E
    assert call_frame(scale=-1.0) == E
    lib = attn.load()
    for fn in (lib.vggt_attn_global,):
        assert fn(None, 2 * A, 3 * A, 4 * A, None, SHAPE, 0.125, None) == E


def test_rejects_unsupported_shapes():
    U = attn.VGGT_ERR_UNSUPPORTED
    assert call_frame(shape=attn.vggt_shape(4, 5, 37, 37, 16, 128)) == U
    assert call_frame(shape=attn.vggt_shape(4, 5, 37, 37, 65, 64)) == U
    assert call_frame(shape=attn.vggt_shape(3000, 5, 1000, 1000, 1, 64)) == U
    assert call_frame(shape=attn.vggt_shape(0, 5, 37, 37, 16, 64)) == attn.VGGT_ERR_INVALID_ARG


def test_sga_argument_checks():
    assert call_sga(ws_bytes=1024) == attn.VGGT_ERR_WORKSPACE
    assert call_sga(ws=8 * A + 16) == attn.VGGT_ERR_INVALID_ARG     # not 256-aligned
    assert call_sga(ws=None) == attn.VGGT_ERR_INVALID_ARG
    assert call_sga(kept=None) == attn.VGGT_ERR_INVALID_ARG
    assert call_sga(mult=6 * A + 2) == attn.VGGT_ERR_INVALID_ARG
    assert call_sga(sh=0) == attn.VGGT_ERR_INVALID_ARG
    # workspace overlapping the output
    assert call_sga(ws=4 * A) == attn.VGGT_ERR_INVALID_ARG
    lib = attn.load()
    assert lib.vggt_sga_build_index(SHAPE, 2, 2, None, 6 * A, None) == attn.VGGT_ERR_INVALID_ARG
    assert lib.vggt_sga_build_index(SHAPE, 2, 0, 5 * A, 6 * A, None) == attn.VGGT_ERR_INVALID_ARG


def test_noalloc_argument_checks_come_before_the_device():
    # The allocation-free SGA entry point checks the size limit, then the
    # same pointers, scale and index arrays as vggt_attn_sga, all before it
    # looks up its scratch array on the device.
    lib = attn.load()
    tiny = attn.vggt_shape(2, 5, 8, 8, 2, 64)
    n100 = attn.vggt_shape(100, 5, 37, 37, 16, 64)
    assert lib.vggt_attn_sga_noalloc(None, None, None, None, None, n100, 2, 2, None, None, 0.125,
                                     None) == attn.VGGT_ERR_WORKSPACE
    assert lib.vggt_attn_sga_noalloc(None, None, None, None, None, tiny, 2, 2, None, None, 0.125,
                                     None) == attn.VGGT_ERR_INVALID_ARG
    assert lib.vggt_attn_sga_noalloc(A, 2 * A, 3 * A, 4 * A, None, tiny, 2, 2, None, 6 * A, 0.125,
                                     None) == attn.VGGT_ERR_INVALID_ARG
    assert lib.vggt_attn_sga_noalloc(A, 2 * A, 3 * A, 4 * A, None, tiny, 2, 2, 5 * A, 6 * A, -1.0,
                                     None) == attn.VGGT_ERR_INVALID_ARG
    assert lib.vggt_attn_sga_noalloc(A, 2 * A, 3 * A, A + 16, None, tiny, 2, 2, 5 * A, 6 * A, 0.125,
                                     None) == attn.VGGT_ERR_INVALID_ARG  # O overlaps Q


@pytest.mark.skipif(not no_gpu(), reason="checks the behaviour without a CUDA device")
def test_valid_call_without_gpu_fails_loudly():
    # Valid arguments reach the CUDA runtime, which finds no device: the
    # library reports VGGT_ERR_CUDA instead of computing anything on the host.
    assert call_frame() == attn.VGGT_ERR_CUDA
    assert call_sga() == attn.VGGT_ERR_CUDA
    lib = attn.load()
    assert lib.vggt_sga_build_index(SHAPE, 2, 2, 5 * A, 6 * A, None) == attn.VGGT_ERR_CUDA


def test_stall_hook_argument_checks():
    lib = attn.load()
    # the wait bound must lie in [1 ms, 4 s]; checked before anything is queued
    assert lib.vggt_test_attn_global_stall(A, 2 * A, 3 * A, 4 * A, SHAPE, 0.125, 0, None) == attn.VGGT_ERR_INVALID_ARG
    assert lib.vggt_test_attn_global_stall(A, 2 * A, 3 * A, 4 * A, SHAPE, 0.125, 10 ** 10, None) == \
        attn.VGGT_ERR_INVALID_ARG
    assert lib.vggt_test_attn_global_stall(None, 2 * A, 3 * A, 4 * A, SHAPE, 0.125, 10 ** 8, None) == \
        attn.VGGT_ERR_INVALID_ARG


def test_register_argument_checks():
    lib = attn.load()
    no_special = attn.vggt_shape(4, 0, 37, 37, 16, 64)
    many_special = attn.vggt_shape(4, 129, 37, 37, 16, 64)
    assert lib.vggt_attn_register(A, 2 * A, 3 * A, 4 * A, None, no_special, 0.125, None) == attn.VGGT_ERR_INVALID_ARG
    assert lib.vggt_attn_register(A, 2 * A, 3 * A, 4 * A, None, many_special, 0.125, None) == \
        attn.VGGT_ERR_UNSUPPORTED
    assert lib.vggt_attn_register(A, 2 * A, 3 * A, 4 * A, None, SHAPE, 0.0, None) == attn.VGGT_ERR_INVALID_ARG
    assert lib.vggt_attn_register(A, 2 * A, 3 * A, A + 32, None, SHAPE, 0.125, None) == \
        attn.VGGT_ERR_INVALID_ARG  # O overlaps Q
    assert lib.vggt_attn_register(None, 2 * A, 3 * A, 4 * A, None, SHAPE, 0.125, None) == attn.VGGT_ERR_INVALID_ARG


def test_row_block_argument_checks():
    lib = attn.load()
    S = attn.vggt_num_tokens(SHAPE)
    assert lib.vggt_attn_global_rows(A, 0, 2 * A, 3 * A, 4 * A, None, SHAPE, 0.125, None) == attn.VGGT_ERR_INVALID_ARG
    assert lib.vggt_attn_global_rows(A, S + 1, 2 * A, 3 * A, 4 * A, None, SHAPE, 0.125, None) == \
        attn.VGGT_ERR_INVALID_ARG
    assert lib.vggt_attn_global_rows(None, 10, 2 * A, 3 * A, 4 * A, None, SHAPE, 0.125, None) == \
        attn.VGGT_ERR_INVALID_ARG
    # the output block overlaps the (full) keys
    assert lib.vggt_attn_global_rows(A, 10, 2 * A, 3 * A, 2 * A + 64, None, SHAPE, 0.125, None) == \
        attn.VGGT_ERR_INVALID_ARG
    nb = attn.vggt_sga_workspace_bytes(SHAPE, 2, 2)
    args = dict(q=A, row0=100, n=10, k=2 * A, v=3 * A, o=4 * A, kept=5 * A, mult=6 * A, ws=8 * A, wsb=nb)

    def sga_rows(**kw):
        a = {**args, **kw}
        return lib.vggt_attn_sga_rows(a["q"], a["row0"], a["n"], a["k"], a["v"], a["o"], None, SHAPE, 2, 2,
                                      a["kept"], a["mult"], a["ws"], a["wsb"], 0.125, None)

    assert sga_rows(row0=-1) == attn.VGGT_ERR_INVALID_ARG
    assert sga_rows(row0=S - 5) == attn.VGGT_ERR_INVALID_ARG  # past the end of the sequence
    assert sga_rows(n=0) == attn.VGGT_ERR_INVALID_ARG
    assert sga_rows(wsb=256) == attn.VGGT_ERR_WORKSPACE
    assert sga_rows(mult=None) == attn.VGGT_ERR_INVALID_ARG


def test_kept_exchange_argument_checks():
    # the query-split SGA entry points reject bad arguments before any launch
    lib = attn.load()
    S = attn.vggt_num_tokens(SHAPE)
    loc = attn.vggt_shape(2, SHAPE.n_special, SHAPE.patch_h, SHAPE.patch_w, SHAPE.n_heads, 64)
    nb = attn.vggt_sga_partial_workspace_bytes(loc)
    assert nb > 0 and nb % 256 == 0
    assert attn.vggt_sga_partial_workspace_bytes(attn.vggt_shape(0, 5, 4, 4, 2, 64)) == 0

    def gather(**kw):
        a = dict(k=A, v=2 * A, sh=2, sw=2, kk=3 * A, kv=4 * A, sums=5 * A, ws=6 * A, wsb=nb, shape=loc)
        a.update(kw)
        return lib.vggt_sga_gather_partial(a["k"], a["v"], a["shape"], a["sh"], a["sw"], a["kk"], a["kv"],
                                           a["sums"], a["ws"], a["wsb"], None)

    assert gather(sh=0) == attn.VGGT_ERR_INVALID_ARG
    assert gather(k=None) == attn.VGGT_ERR_INVALID_ARG
    assert gather(kk=3 * A + 8) == attn.VGGT_ERR_INVALID_ARG          # misaligned output
    assert gather(ws=6 * A + 64) == attn.VGGT_ERR_INVALID_ARG         # workspace not 256-byte aligned
    assert gather(wsb=nb - 256) == attn.VGGT_ERR_WORKSPACE
    assert gather(kv=A + 64) == attn.VGGT_ERR_INVALID_ARG             # output inside the keys
    assert gather(sums=3 * A) == attn.VGGT_ERR_INVALID_ARG            # two outputs overlap

    def gathered(**kw):
        a = dict(q=A, row0=10, n=20, kr=2 * A, vr=3 * A, kk=4 * A, kv=5 * A, sums=6 * A, mult=7 * A, means=8 * A,
                 o=9 * A, sh=2, sw=2, scale=0.125)
        a.update(kw)
        return lib.vggt_attn_sga_gathered(a["q"], a["row0"], a["n"], a["kr"], a["vr"], a["kk"], a["kv"], a["sums"],
                                          a["mult"], a["means"], a["o"], None, SHAPE, a["sh"], a["sw"], a["scale"],
                                          None)

    assert gathered(row0=-1) == attn.VGGT_ERR_INVALID_ARG
    assert gathered(row0=S - 5) == attn.VGGT_ERR_INVALID_ARG          # past the end of the sequence
    assert gathered(n=0) == attn.VGGT_ERR_INVALID_ARG
    assert gathered(mult=None) == attn.VGGT_ERR_INVALID_ARG
    assert gathered(means=8 * A + 4) == attn.VGGT_ERR_INVALID_ARG     # misaligned
    assert gathered(means=4 * A) == attn.VGGT_ERR_INVALID_ARG         # means inside the kept keys
    assert gathered(scale=0.0) == attn.VGGT_ERR_INVALID_ARG
    assert gathered(sw=0) == attn.VGGT_ERR_INVALID_ARG


def test_binding_refuses_host_tensors():
    q = torch.zeros(10, 2, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        attn.vggt_attn_frame(q, q, q, q, None, (1, 5, 1, 5, 2, 64), 0.125, stream=0)


def test_accounting_flops():
    assert accounting.flops_global(137400, 16, 64) == 4 * 137400 ** 2 * 16 * 64
    assert abs(accounting.flops_global(137400, 16, 64) - 7.73e13) / 7.73e13 < 1e-3
    assert abs(accounting.flops_frame(100, 1374, 16, 64) - 7.73e11) / 7.73e11 < 1e-3
    nk, nd = accounting.sga_counts(100, 5, 37, 37, 2, 2)
    assert abs(accounting.flops_sga(137400, nk, nd, 16, 64) - 2.06e13) / 2.06e13 < 2e-3
    assert abs(accounting.meanfill_read_bytes(100, 37, 37, 16, 64) - 560.7e6) / 560.7e6 < 1e-3


def test_qkv_rope_rejects_bad_arguments_before_queuing():
    lib = attn.load()
    sh16 = attn.vggt_shape(4, 5, 37, 37, 16, 64)
    C = 16 * 64
    x, w, q, k, v = A, A + (1 << 30), A + (2 << 30), A + (3 << 30), A + (4 << 30)
    call = lambda shape=sh16, base=100.0, **kw: lib.vggt_qkv_rope(
        kw.get("x", x), kw.get("w", w), kw.get("bias", None), kw.get("q", q), kw.get("k", k), kw.get("v", v),
        shape, base, None)
    assert call(shape=attn.vggt_shape(4, 5, 37, 37, 3, 64)) == attn.VGGT_ERR_UNSUPPORTED  # odd H
    assert call(shape=attn.vggt_shape(1, 5, 200, 4, 16, 64)) == attn.VGGT_ERR_UNSUPPORTED  # grid > 128
    assert call(base=0.0) == attn.VGGT_ERR_INVALID_ARG
    assert call(base=float("inf")) == attn.VGGT_ERR_INVALID_ARG
    assert call(x=None) == attn.VGGT_ERR_INVALID_ARG
    assert call(q=A + 8) == attn.VGGT_ERR_INVALID_ARG          # misaligned
    assert call(bias=A + 2) == attn.VGGT_ERR_INVALID_ARG       # misaligned bias
    assert call(k=q) == attn.VGGT_ERR_INVALID_ARG              # outputs overlap
    assert call(v=x) == attn.VGGT_ERR_INVALID_ARG              # output overlaps the input
    assert C == 1024


def test_out_proj_rejects_bad_arguments_before_queuing():
    lib = attn.load()
    sh16 = attn.vggt_shape(4, 5, 37, 37, 16, 64)
    o, w, y = A, A + (1 << 30), A + (2 << 30)
    call = lambda shape=sh16, **kw: lib.vggt_out_proj(kw.get("o", o), kw.get("w", w), kw.get("bias", None),
                                                      kw.get("y", y), shape, None)
    assert call(shape=attn.vggt_shape(4, 5, 37, 37, 3, 64)) == attn.VGGT_ERR_UNSUPPORTED
    assert call(y=None) == attn.VGGT_ERR_INVALID_ARG
    assert call(y=o) == attn.VGGT_ERR_INVALID_ARG
    assert call(bias=A + 6) == attn.VGGT_ERR_INVALID_ARG
