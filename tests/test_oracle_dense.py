"""Pins for oracle/dense.py, the matrix-product form of the fp64 oracle used
for the large sampled parity cases (N = 800).

It must agree with the scalar C oracle (vggt_oracle.c, pinned on its own in
test_oracle.py by hand-derived index lists, closed forms and brute force) to
fp64 rounding on every mode, including ragged grids, strides that leave
short windows, M_i = 0 and |D| = 0; and it must satisfy the invariants the
definition fixes by itself (V == 1 gives O == 1; SGA at stride 1x1 is global
attention; global attention over one frame is frame attention)."""
import numpy as np
import pytest
import torch

import oracle
from oracle import dense
from feed_forward_view_vggt_b200 import synth

TOL = 1e-11


def bits(x):
    return x.contiguous().view(torch.int16).numpy().view(np.uint16)


def random_case(N, ns, h, w, H, seed):
    g = torch.Generator().manual_seed(seed)
    S = N * (ns + h * w)
    q, k, v = (torch.randn(S, H, 64, generator=g).to(torch.bfloat16) for _ in range(3))
    return [bits(x) for x in (q, k, v)], oracle.Shape(N, ns, h, w, H, 64)


def close(a, b, tol=TOL):
    (oa, la), (ob, lb) = a, b
    assert oa.shape == ob.shape and la.shape == lb.shape
    assert np.abs(oa - ob).max() <= tol, np.abs(oa - ob).max()
    assert np.abs(la - lb).max() <= tol, np.abs(la - lb).max()


@pytest.mark.parametrize("mode", [oracle.FRAME, oracle.GLOBAL, oracle.REGISTER])
def test_dense_matches_c_oracle_tiny(mode):
    wl = synth.WORKLOADS["tiny"]
    b = [bits(x) for x in synth.make_qkv(wl)]
    sh = oracle.Shape(wl.N, wl.n_special, wl.h, wl.w, wl.H, wl.d)
    rows = oracle.special_rows(sh) if mode == oracle.REGISTER else None
    close(dense.attention(mode, *b, sh, rows=rows), oracle.attention(mode, *b, sh, rows=rows))


@pytest.mark.parametrize("stride", [(1, 1), (2, 2), (3, 3), (2, 3), (8, 8), (9, 1)])
def test_dense_sga_matches_c_oracle_tiny(stride):
    wl = synth.WORKLOADS["tiny"]
    b = [bits(x) for x in synth.make_qkv(wl)]
    sh = oracle.Shape(wl.N, wl.n_special, wl.h, wl.w, wl.H, wl.d)
    close(dense.sga_attention(*b, sh, *stride), oracle.sga_attention(*b, sh, *stride))


@pytest.mark.parametrize("N,ns,h,w,stride", [(3, 5, 7, 5, (3, 2)),   # short last windows on both axes
                                              (2, 0, 4, 4, (2, 2)),   # no special tokens
                                              (3, 1, 1, 2, (1, 2)),   # |D| = 3 = N: M_i = 2 for dropped rows
                                              (1, 2, 1, 2, (1, 2))])  # |D| = 1: M_i = 0 on the dropped row
def test_dense_sga_matches_c_oracle_ragged(N, ns, h, w, stride):
    b, sh = random_case(N, ns, h, w, 3, seed=N * 100 + h * 10 + w)
    close(dense.sga_attention(*b, sh, *stride), oracle.sga_attention(*b, sh, *stride))
    close(dense.global_attention(*b, sh), oracle.global_attention(*b, sh))
    close(dense.frame_attention(*b, sh), oracle.frame_attention(*b, sh))


def test_dense_matches_c_oracle_on_sampled_rows_at_the_worked_example():
    wl = synth.WORKLOADS["n4"]
    b = [bits(x) for x in synth.make_qkv(wl)]
    sh = oracle.Shape(wl.N, wl.n_special, wl.h, wl.w, wl.H, wl.d)
    rows = synth.sample_rows(wl.S, wl.L, wl.n_special, count=48, seed=7)
    for mode, st in ((oracle.FRAME, (1, 1)), (oracle.GLOBAL, (1, 1)), (oracle.SGA, (2, 2)), (oracle.SGA, (3, 3))):
        close(dense.attention(mode, *b, sh, s_h=st[0], s_w=st[1], rows=rows),
              oracle.attention(mode, *b, sh, s_h=st[0], s_w=st[1], rows=rows))
    # the rows may come in any order, and in blocks of any size
    perm = rows[::-1].copy()
    o1, l1 = dense.attention(oracle.SGA, *b, sh, s_h=2, s_w=2, rows=perm, row_block=5)
    o2, l2 = dense.attention(oracle.SGA, *b, sh, s_h=2, s_w=2, rows=rows)
    assert np.abs(o1[::-1] - o2).max() <= TOL and np.abs(l1[::-1] - l2).max() <= TOL


def test_dense_invariants():
    b, sh = random_case(3, 5, 6, 6, 2, seed=11)
    q, k, v = b
    ones = np.full_like(v, 0x3F80)  # bf16 1.0
    for mode, st in ((oracle.FRAME, (1, 1)), (oracle.GLOBAL, (1, 1)), (oracle.SGA, (2, 2)), (oracle.SGA, (3, 2))):
        o, _ = dense.attention(mode, q, k, ones, sh, s_h=st[0], s_w=st[1])
        assert np.abs(o - 1.0).max() <= 1e-13
    # stride 1x1 drops nothing: SGA is global attention
    close(dense.sga_attention(q, k, v, sh, 1, 1), dense.global_attention(q, k, v, sh))
    # one frame: global attention is frame attention
    b1, sh1 = random_case(1, 5, 6, 6, 2, seed=12)
    close(dense.global_attention(*b1, sh1), dense.frame_attention(*b1, sh1))


def test_dense_refuses_bad_rows():
    b, sh = random_case(2, 5, 4, 4, 2, seed=13)
    with pytest.raises(ValueError):
        dense.global_attention(*b, sh, rows=[sh.S])
    with pytest.raises(ValueError):
        dense.register_attention(*b, sh, rows=[sh.n_special])
