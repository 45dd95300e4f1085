"""The debug build (libvggt_attn_debug.so, -DVGGT_DEBUG): every kernel
checks its computed indices on the device before the guarded accesses.  On
valid inputs no check may fail (vggt_check stays VGGT_OK) and every output
must equal the release library's bit for bit, for every entry point, on the
tiny workload, the worked example and a ragged shape."""
import ctypes

import pytest
import torch

from feed_forward_view_vggt_b200 import attn, synth
from feed_forward_view_vggt_b200 import build as vbuild

pytestmark = pytest.mark.gpu

CASES = [synth.WORKLOADS["tiny"], synth.WORKLOADS["n4"],
         synth.Workload("ragged", N=3, h=7, w=5, H=3, seed=9, structure="iid")]


@pytest.fixture(scope="module")
def libs():
    vbuild.build(debug=True)
    return attn.load(), attn.load_library(attn.DEBUG_LIB_PATH)


def check(lib):
    d = ctypes.c_uint32(0)
    st = lib.vggt_check(None, ctypes.byref(d))
    assert st == attn.VGGT_OK, (attn.vggt_status_string(st), hex(d.value))


def run_all(lib, wl, q, k, v):
    sh, sc = attn._shape(wl), attn.default_scale(64)
    S, H = q.shape[0], q.shape[1]
    out = {}
    for name in ("frame", "global"):
        o = torch.empty_like(q)
        lse = torch.empty(S, H, dtype=torch.float32, device=q.device)
        assert getattr(lib, f"vggt_attn_{name}")(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                                  lse.data_ptr(), sh, sc, None) == attn.VGGT_OK
        out[name], out[name + "_lse"] = o, lse
    for s_h, s_w in ((2, 2), (3, 2)):
        nk = lib.vggt_sga_num_kept(sh, s_h, s_w)
        kept = torch.empty(nk, dtype=torch.int32, device=q.device)
        mult = torch.empty(S, dtype=torch.int32, device=q.device)
        assert lib.vggt_sga_build_index(sh, s_h, s_w, kept.data_ptr(), mult.data_ptr(), None) == attn.VGGT_OK
        nbytes = lib.vggt_sga_workspace_bytes(sh, s_h, s_w)
        ws = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
        o = torch.empty_like(q)
        assert lib.vggt_attn_sga(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), None, sh, s_h, s_w,
                                 kept.data_ptr(), mult.data_ptr(), ws.data_ptr(), nbytes, sc, None) == attn.VGGT_OK
        out[f"sga{s_h}x{s_w}"], out[f"kept{s_h}x{s_w}"], out[f"mult{s_h}x{s_w}"] = o, kept, mult
    # the kept-row exchange of the query-row split, two ranks run in turn
    s_h = s_w = 2
    L, hd = S // wl.N, H * 64
    cuts = [0, wl.N // 2, wl.N] if wl.N > 1 else [0, wl.N]
    parts, sums = [], torch.zeros(2, hd, dtype=torch.float32, device=q.device)
    for f0, f1 in zip(cuts[:-1], cuts[1:]):
        loc = attn.vggt_shape(f1 - f0, sh.n_special, sh.patch_h, sh.patch_w, H, 64)
        nk = lib.vggt_sga_num_kept(loc, s_h, s_w)
        kk, kv = (torch.empty(nk, H, 64, dtype=torch.bfloat16, device=q.device) for _ in range(2))
        ds = torch.empty(2, hd, dtype=torch.float32, device=q.device)
        nb = lib.vggt_sga_partial_workspace_bytes(loc)
        ws = torch.empty(nb, dtype=torch.uint8, device=q.device)
        assert lib.vggt_sga_gather_partial(k[f0 * L:].data_ptr(), v[f0 * L:].data_ptr(), loc, s_h, s_w, kk.data_ptr(),
                                           kv.data_ptr(), ds.data_ptr(), ws.data_ptr(), nb, None) == attn.VGGT_OK
        parts.append((kk, kv))
        sums += ds
    kept_k, kept_v = torch.cat([p[0] for p in parts]), torch.cat([p[1] for p in parts])
    means = torch.empty(2, hd, dtype=torch.float32, device=q.device)
    o = torch.empty_like(q)
    for f0, f1 in zip(cuts[:-1], cuts[1:]):
        r0, r1 = f0 * L, f1 * L
        assert lib.vggt_attn_sga_gathered(q[r0:].data_ptr(), r0, r1 - r0, k[r0:].data_ptr(), v[r0:].data_ptr(),
                                          kept_k.data_ptr(), kept_v.data_ptr(), sums.data_ptr(),
                                          out["mult2x2"].data_ptr(), means.data_ptr(), o[r0:].data_ptr(), None, sh,
                                          s_h, s_w, sc, None) == attn.VGGT_OK
    out["kept_exchange"], out["kept_exchange_rows"] = o, kept_k
    if wl.n_special > 0:
        o = torch.zeros_like(q)
        assert lib.vggt_attn_register(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), None, sh, sc,
                                      None) == attn.VGGT_OK
        out["register"] = o
    if H % 2 == 0:
        C = H * 64
        g = torch.Generator().manual_seed(5)
        x = torch.randn(S, C, generator=g).to(torch.bfloat16).cuda()
        w = (torch.randn(3 * C, C, generator=g) / C ** 0.5).to(torch.bfloat16).cuda()
        qq, kk, vv = (torch.empty_like(q) for _ in range(3))
        assert lib.vggt_qkv_rope(x.data_ptr(), w.data_ptr(), None, qq.data_ptr(), kk.data_ptr(), vv.data_ptr(), sh,
                                 100.0, None) == attn.VGGT_OK
        out["qkv"] = torch.cat([qq, kk, vv])
    check(lib)
    return out


@pytest.mark.parametrize("wl", CASES, ids=[w.name for w in CASES])
def test_debug_build_checks_pass_and_match_release(libs, wl):
    rel, dbg = libs
    assert dbg.vggt_debug_checks() == 1
    q, k, v = (x.cuda() for x in synth.make_qkv(wl))
    a, b = run_all(rel, wl, q, k, v), run_all(dbg, wl, q, k, v)
    assert a.keys() == b.keys()
    for name in a:
        assert torch.equal(a[name], b[name]), name
