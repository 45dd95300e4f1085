"""Parity at the largest configuration, N=800 frames (1,099,200 tokens,
H=16, d=64): sampled query rows against the fp64 oracle (token 0, token S-1,
the frame-0 specials and the ragged tails always included), plus a property
that holds at any size (V == 1 gives O == 1) on the full output."""
import numpy as np
import pytest
import torch

import oracle
from feed_forward_view_vggt_b200 import attn, synth

pytestmark = pytest.mark.gpu

_case = {}


def case():
    if not _case:
        wl = synth.WORKLOADS["n800"]
        q, k, v = synth.make_qkv(wl)
        _case.update(wl=wl, bits=[x.view(torch.int16).numpy().view(np.uint16) for x in (q, k, v)],
                     dev=[x.cuda() for x in (q, k, v)],
                     shape=oracle.Shape(wl.N, wl.n_special, wl.h, wl.w, wl.H, wl.d))
    return _case


def check(o, rows, ref):
    assert attn.vggt_check()[0] == attn.VGGT_OK
    got = o[torch.as_tensor(rows).cuda()].float().cpu().double().numpy()
    err = np.abs(got - ref)
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert np.isfinite(got).all() and err.max() <= 2e-2 and rel <= 5e-3, (err.max(), rel)


@pytest.mark.parametrize("op,stride,count", [("frame", None, 2048), ("global", None, 256),
                                             ("sga", (3, 3), 512), ("sga", (2, 2), 256)])
def test_n800_sampled(op, stride, count):
    c = case()
    wl, sh = c["wl"], c["shape"]
    q, k, v = c["dev"]
    rows = synth.sample_rows(wl.S, wl.L, wl.n_special, count=count, seed=1234)
    if op == "frame":
        o = attn.frame(q, k, v, wl)
        ref, _ = oracle.frame_attention(*c["bits"], sh, rows=rows)
    elif op == "global":
        o = attn.global_(q, k, v, wl)
        ref, _ = oracle.global_attention(*c["bits"], sh, rows=rows)
    else:
        o = attn.sga(q, k, v, attn.SgaIndex(wl, *stride))
        ref, _ = oracle.sga_attention(*c["bits"], sh, *stride, rows=rows)
    check(o, rows, ref)


def test_n800_values_one_give_one_everywhere():
    c = case()
    q, k, v = c["dev"]
    ones = torch.ones_like(v)
    o = attn.sga(q, k, ones, attn.SgaIndex(c["wl"], 3, 3))
    assert attn.vggt_check()[0] == attn.VGGT_OK
    assert (o.float() - 1.0).abs().max().item() <= 1e-2
