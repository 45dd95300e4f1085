"""Parity at the largest configuration, N=800 frames (1,099,200 tokens,
H=16, d=64): every op on 4096 seeded query rows x all 16 heads, compared
element by element with the fp64 oracle (token 0, token S-1, the frame-0
specials and the ragged tails always included), plus a property that holds
at any size (V == 1 gives O == 1) on the full output.

The oracle here is its matrix-product form (oracle/dense.py, pinned against
the scalar C oracle in test_oracle_dense.py): the scalar form needs about
0.3 s per global-attention row at this size, the matrix-product form a few
hundredths.  Each op is its own test; the device run and the inputs are
shared through a module-level cache."""
import numpy as np
import pytest
import torch

import oracle
from oracle import dense
from feed_forward_view_vggt_b200 import attn, synth

pytestmark = pytest.mark.gpu

ROWS = 4096
MAX_ABS = 2e-2
REL_FRO = 5e-3

_case = {}


def case():
    if not _case:
        wl = synth.WORKLOADS["n800"]
        q, k, v = synth.make_qkv(wl)
        _case.update(wl=wl, bits=[x.view(torch.int16).numpy().view(np.uint16) for x in (q, k, v)],
                     dev=[x.cuda() for x in (q, k, v)],
                     shape=oracle.Shape(wl.N, wl.n_special, wl.h, wl.w, wl.H, wl.d),
                     rows=synth.sample_rows(wl.S, wl.L, wl.n_special, count=ROWS, seed=1234))
    return _case


def check(o, lse, rows, ref, ref_lse):
    assert attn.vggt_check()[0] == attn.VGGT_OK
    assert len(rows) == ROWS
    idx = torch.as_tensor(rows).cuda()
    got = o[idx].float().cpu().double().numpy()
    err = np.abs(got - ref)
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert np.isfinite(got).all() and err.max() <= MAX_ABS and rel <= REL_FRO, (err.max(), rel)
    got_lse = lse[idx].cpu().double().numpy()
    assert np.abs(got_lse - ref_lse).max() <= MAX_ABS


def test_n800_frame():
    c = case()
    o, lse = attn.frame(*c["dev"], c["wl"], want_lse=True)
    check(o, lse, c["rows"], *dense.frame_attention(*c["bits"], c["shape"], rows=c["rows"]))


def test_n800_global():
    c = case()
    o, lse = attn.global_(*c["dev"], c["wl"], want_lse=True)
    check(o, lse, c["rows"], *dense.global_attention(*c["bits"], c["shape"], rows=c["rows"]))


@pytest.mark.parametrize("stride", [(3, 3), (2, 2)])
def test_n800_sga(stride):
    c = case()
    o, lse = attn.sga(*c["dev"], attn.SgaIndex(c["wl"], *stride), want_lse=True)
    check(o, lse, c["rows"], *dense.sga_attention(*c["bits"], c["shape"], *stride, rows=c["rows"]))


def test_n800_values_one_give_one_everywhere():
    c = case()
    q, k, v = c["dev"]
    ones = torch.ones_like(v)
    o = attn.sga(q, k, ones, attn.SgaIndex(c["wl"], 3, 3))
    assert attn.vggt_check()[0] == attn.VGGT_OK
    assert (o.float() - 1.0).abs().max().item() <= 1e-2
