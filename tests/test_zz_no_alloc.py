"""The allocation-free SGA entry point, vggt_attn_sga_noalloc.

It is meant for callers that cannot allocate device memory when they call
SGA (a fixed memory budget, a runtime that owns every allocation, or code
where cudaMalloc is not allowed); instead of a caller workspace it uses the
library's built-in 16 MiB device scratch array.  Here it is called through
the C ABI and its output is checked against the workspace entry point,
vggt_attn_sga, on several calls in a row (the scratch array is shared and
keeps the previous call's contents), and a shape whose scratch need exceeds
the array is refused before anything is queued.

This file is collected last so that a run stopping at the first failure has
already run every other test."""
import numpy as np
import pytest
import torch

from feed_forward_view_vggt_b200 import attn, synth

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
REL_FRO = 5e-3


def check_ok():
    st, detail = attn.vggt_check()
    assert st == attn.VGGT_OK, (attn.vggt_status_string(st), hex(detail))


def run_noalloc(q, k, v, wl, index):
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[0], q.shape[1], dtype=torch.float32, device=q.device)
    st = attn.vggt_attn_sga_noalloc(q, k, v, o, lse, wl, index.s_h, index.s_w, index.kept_idx, index.mult,
                                    attn.default_scale(64))
    assert st == attn.VGGT_OK, attn.vggt_status_string(st)
    check_ok()
    return o, lse


def assert_close(got, ref):
    g, r = got.double().cpu().numpy(), ref.double().cpu().numpy()
    err = np.abs(g - r)
    rel = np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30)
    assert np.isfinite(g).all() and err.max() <= MAX_ABS and rel <= REL_FRO, (err.max(), rel)


def test_noalloc_matches_workspace_entry_on_calls_in_a_row():
    first = None
    # The stride-1x1 call comes right after a 2x2 call: with nothing dropped
    # it computes no means, so the array still holds the previous call's
    # kbar/vbar, and the result must not depend on them.
    for name, stride in (("n4", (2, 2)), ("tiny", (3, 3)), ("n4", (2, 2)), ("tiny", (1, 1))):
        wl = synth.WORKLOADS[name]
        q, k, v = (x.cuda() for x in synth.make_qkv(wl))
        index = attn.SgaIndex(wl, *stride)
        assert index.workspace_bytes <= 16 << 20
        ref, ref_lse = attn.sga(q, k, v, index, want_lse=True)
        check_ok()
        o, lse = run_noalloc(q, k, v, wl, index)
        assert_close(o.float(), ref.float())
        assert_close(lse, ref_lse)
        if stride == (1, 1):
            # nothing dropped: SGA is global attention, and equal to the
            # workspace entry point bit for bit
            glob, glob_lse = attn.global_(q, k, v, wl, want_lse=True)
            check_ok()
            assert_close(o.float(), glob.float())
            assert_close(lse, glob_lse)
            assert torch.equal(o, ref)
        elif first is None:
            first = o.clone()
        elif name == "n4":
            # same inputs as the first call, after a call of another size
            assert torch.equal(o, first)


def test_noalloc_refuses_shapes_beyond_the_scratch_array():
    wl = synth.WORKLOADS["n100"]  # needs ~152 MB of scratch
    assert attn.vggt_sga_workspace_bytes(wl, 2, 2) > 16 << 20
    lib = attn.load()
    st = lib.vggt_attn_sga_noalloc(None, None, None, None, None, attn._shape(wl), 2, 2, None, None, 0.125, None)
    assert st == attn.VGGT_ERR_WORKSPACE
