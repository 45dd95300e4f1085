"""Layer schedule on the GPU.

* Every layer of a mixed schedule equals the single-layer call on the same
  inputs bit for bit: the SGA index built once per stride is the one each
  layer would build.
* Every layer matches the fp64 oracle.
* A register layer leaves patch-token rows untouched.
* AVGGT and VGGT-Omega trunks at N=4 reproduce per-layer calls."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from feed_forward_view_vggt_b200 import attn, schedules, synth

pytestmark = pytest.mark.gpu

MIXED = ["frame", "global", ("sga", 2, 2), "register", ("sga", 3, 3), ("sga", 2, 2), "global"]


def close(got, ref):
    got = got.float().cpu().double().numpy()
    err = np.abs(got - ref)
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert np.isfinite(got).all() and err.max() <= 2e-2 and rel <= 5e-3, (err.max(), rel)


def single(ly, q, k, v, wl, o_init=None):
    kind = ly if isinstance(ly, str) else ly[0]
    if kind == "frame":
        return attn.frame(q, k, v, wl)
    if kind == "global":
        return attn.global_(q, k, v, wl)
    if kind == "register":
        return attn.register(q, k, v, wl, o=o_init.clone())
    return attn.sga(q, k, v, attn.SgaIndex(wl, ly[1], ly[2]))


def test_mixed_schedule_equals_single_layer_calls_and_the_oracle():
    wl = synth.WORKLOADS["tiny"]
    sh = oracle.Shape(wl.N, wl.n_special, wl.h, wl.w, wl.H, wl.d)
    inputs = [synth.make_qkv(dataclasses.replace(wl, seed=100 + i)) for i in range(len(MIXED))]
    dev = [[x.cuda() for x in qkv] for qkv in inputs]
    qs, ks, vs = ([d[j] for d in dev] for j in range(3))
    sentinel = torch.full_like(qs[0], 7.0)
    os_ = [torch.empty_like(q) for q in qs]
    os_[3] = sentinel.clone()
    attn.schedule(qs, ks, vs, wl, MIXED, os_=os_)
    assert attn.vggt_check()[0] == attn.VGGT_OK
    for i, ly in enumerate(MIXED):
        q, k, v = dev[i]
        assert torch.equal(os_[i], single(ly, q, k, v, wl, sentinel)), (i, ly)
        bits = [x.view(torch.int16).numpy().view(np.uint16) for x in inputs[i]]
        kind = ly if isinstance(ly, str) else ly[0]
        if kind == "frame":
            close(os_[i], oracle.frame_attention(*bits, sh)[0])
        elif kind == "global":
            close(os_[i], oracle.global_attention(*bits, sh)[0])
        elif kind == "sga":
            close(os_[i], oracle.sga_attention(*bits, sh, ly[1], ly[2])[0])
        else:
            rows = oracle.special_rows(sh)
            close(os_[i][torch.as_tensor(rows).cuda()], oracle.register_attention(*bits, sh)[0])
            patch = np.setdiff1d(np.arange(sh.S), rows)
            assert bool((os_[i][torch.as_tensor(patch).cuda()] == 7.0).all())
    assert attn.vggt_check()[0] == attn.VGGT_OK


@pytest.mark.parametrize("trunk", ["avggt", "omega"])
def test_trunks_at_n4_reproduce_per_layer_calls(trunk):
    wl = synth.WORKLOADS["n4"]
    q, k, v = (x.cuda() for x in synth.make_qkv(wl))
    layers = schedules.avggt_trunk(6, stride=(3, 3)) if trunk == "avggt" else schedules.omega_trunk(4, every=2)
    n = len(layers)
    base = torch.full_like(q, -3.0)
    os_ = [base.clone() for _ in range(n)]
    attn.schedule([q] * n, [k] * n, [v] * n, wl, layers, os_=os_)
    assert attn.vggt_check()[0] == attn.VGGT_OK
    for i, ly in enumerate(layers):
        assert torch.equal(os_[i], single(ly, q, k, v, wl, base)), (i, ly)


def test_empty_schedule_is_a_no_op():
    wl = synth.WORKLOADS["tiny"]
    assert attn.schedule([], [], [], wl, []) == []
    assert attn.vggt_check()[0] == attn.VGGT_OK
