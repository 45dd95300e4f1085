"""GPU parity of register attention (VGGT-Omega) against the fp64 oracle:
every special-token row of O and lse, and patch-token rows left untouched."""
import numpy as np
import pytest
import torch

import oracle
from feed_forward_view_vggt_b200 import attn, synth

pytestmark = pytest.mark.gpu


def bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("wl", [
    synth.WORKLOADS["tiny"],
    synth.Workload("omega8", N=8, h=37, w=37, H=16, seed=6, structure="corr", n_special=17),
    synth.WORKLOADS["omega100"],
    synth.Workload("one_special", N=300, h=3, w=3, H=2, seed=7, structure="iid", n_special=1),
], ids=lambda w: w.name)
def test_register_attention_matches_oracle(wl):
    q, k, v = synth.make_qkv(wl)
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    sentinel = torch.full_like(qd, 7.0)
    o, lse = attn.register(qd, kd, vd, wl, want_lse=True, o=sentinel.clone())
    st, detail = attn.vggt_check()
    assert st == attn.VGGT_OK, hex(detail)
    sh = oracle.Shape(wl.N, wl.n_special, wl.h, wl.w, wl.H, wl.d)
    rows = oracle.special_rows(sh)
    ref, ref_lse = oracle.register_attention(bits(q), bits(k), bits(v), sh)
    got = o[torch.as_tensor(rows).cuda()].float().cpu().double().numpy()
    err = np.abs(got - ref)
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert err.max() <= 2e-2 and rel <= 5e-3, (err.max(), rel)
    got_lse = lse[torch.as_tensor(rows).cuda()].double().cpu().numpy()
    assert np.abs(got_lse - ref_lse).max() <= 2e-2
    patch = torch.ones(wl.S, dtype=torch.bool)
    patch[torch.as_tensor(rows)] = False
    assert torch.equal(o[patch.cuda()], sentinel[patch.cuda()])


@pytest.mark.parametrize("N,ns,h,w,seed", [(40, 17, 4, 4, 11), (300, 1, 3, 3, 12)])
def test_register_attention_large_logits(N, ns, h, w, seed):
    # q scaled by 6: logits spread over ~+-40, so key tiles after the first
    # push a row's tile sum of P past 2^15 and the softmax's exact slow path
    # (tile max, O/l rescale, P again) runs -- 30 and 2 row-steps by a CPU
    # emulation of the rule on these inputs
    wl = synth.Workload("regx6", N=N, h=h, w=w, H=2, seed=seed, structure="iid", n_special=ns)
    q, k, v = synth.make_qkv(wl)
    q = (q.float() * 6.0).to(torch.bfloat16)
    o, lse = attn.register(q.cuda(), k.cuda(), v.cuda(), wl, want_lse=True)
    st, detail = attn.vggt_check()
    assert st == attn.VGGT_OK, hex(detail)
    sh = oracle.Shape(wl.N, wl.n_special, wl.h, wl.w, wl.H, wl.d)
    rows = oracle.special_rows(sh)
    ref, ref_lse = oracle.register_attention(bits(q), bits(k), bits(v), sh)
    got = o[torch.as_tensor(rows).cuda()].float().cpu().double().numpy()
    err = np.abs(got - ref)
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert err.max() <= 2e-2 and rel <= 5e-3, (err.max(), rel)
    got_lse = lse[torch.as_tensor(rows).cuda()].double().cpu().numpy()
    assert np.abs(got_lse - ref_lse).max() <= 2e-2
