"""Seeded input generator: determinism, shapes and the stated structure."""
import math

import numpy as np
import torch

from feed_forward_view_vggt_b200 import synth


def test_tiny_shapes_and_determinism():
    wl = synth.WORKLOADS["tiny"]
    a = synth.make_qkv(wl)
    b = synth.make_qkv(wl)
    for x, y in zip(a, b):
        assert x.shape == (138, 2, 64) and x.dtype == torch.bfloat16
        assert torch.equal(x.view(torch.int16), y.view(torch.int16))
    assert not torch.equal(a[0], a[1])


def test_correspondence_structure_n4():
    wl = synth.WORKLOADS["n4"]
    q, k, v = synth.make_qkv(wl)
    assert q.shape == (5496, 16, 64)
    kf = k.float().view(wl.N, wl.L, wl.H, wl.d)
    # same in-frame position across frames shares a base: correlation ~ 1/(1+0.25)
    x, y = kf[0].flatten(), kf[1].flatten()
    corr = torch.corrcoef(torch.stack([x, y]))[0, 1].item()
    assert abs(corr - 0.8) < 0.02
    # different positions are uncorrelated
    corr2 = torch.corrcoef(torch.stack([kf[0, :-1].flatten(), kf[1, 1:].flatten()]))[0, 1]
    assert abs(corr2.item()) < 0.02
    assert abs(q.float().std().item() - 1.0) < 0.01


def test_outlier_recipe_counts():
    wl = synth.Workload("mini_out", N=10, h=5, w=5, H=2, seed=3, structure="corr_outliers")
    q, k, v = synth.make_qkv(wl)
    base = synth.Workload("mini", N=10, h=5, w=5, H=2, seed=3, structure="corr")
    q0, k0, v0 = synth.make_qkv(base)
    assert torch.equal(q, q0) and torch.equal(v, v0)
    changed = (k.view(torch.int16) != k0.view(torch.int16)).any(dim=2).any(dim=1)
    assert int(changed.sum()) == math.floor(0.1 * wl.S)


def test_sample_rows():
    S, L = 137400, 1374
    r = synth.sample_rows(S, L)
    assert len(r) == 4096 and np.all(np.diff(r) > 0)
    assert r[0] == 0 and r[-1] == S - 1
    for t in list(range(5)) + list(range(1280, 1374)) + list(range(S - 184, S)):
        assert t in set(r.tolist())
    assert np.array_equal(r, synth.sample_rows(S, L))
    assert np.array_equal(synth.sample_rows(100, 50), np.arange(100))
