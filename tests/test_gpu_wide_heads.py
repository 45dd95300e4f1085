"""Head counts above 16 on the GPU against the fp64 oracle: H = 32 and the
largest supported H = 64 (C = 4096).  These take the mean-fill's wide form
(one block of 2 * H * 64 / 8 = 512 or 1024 threads per SM, a thread per
16-byte column vector of K or V), attention tensor maps with more heads
per token row, the projection GEMM's pair form at C = 2048 / 4096, and the
kept-row exchange of the query-row split."""
import numpy as np
import pytest
import torch

import oracle
from feed_forward_view_vggt_b200 import attn, synth

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
REL_FRO = 5e-3


def bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def compare(got, ref):
    got = got.float().cpu().double().numpy().reshape(ref.shape)
    err = np.abs(got - ref)
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert np.isfinite(got).all() and err.max() <= MAX_ABS and rel <= REL_FRO, (err.max(), rel)


WIDE = [synth.Workload("wide32", N=3, h=7, w=6, H=32, seed=41, structure="iid"),
        synth.Workload("wide64", N=2, h=5, w=5, H=64, seed=42, structure="iid")]


@pytest.mark.parametrize("wl", WIDE, ids=[w.name for w in WIDE])
def test_attention_with_many_heads(wl):
    q, k, v = synth.make_qkv(wl)
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    sh = oracle.Shape(wl.N, wl.n_special, wl.h, wl.w, wl.H, wl.d)
    qb, kb, vb = bits(q), bits(k), bits(v)
    compare(attn.frame(qd, kd, vd, wl), oracle.frame_attention(qb, kb, vb, sh)[0])
    compare(attn.global_(qd, kd, vd, wl), oracle.global_attention(qb, kb, vb, sh)[0])
    for stride in ((2, 2), (3, 2)):
        idx = attn.SgaIndex(wl, *stride)
        compare(attn.sga(qd, kd, vd, idx), oracle.sga_attention(qb, kb, vb, sh, *stride)[0])
    assert attn.vggt_check()[0] == attn.VGGT_OK


@pytest.mark.parametrize("wl", WIDE, ids=[w.name for w in WIDE])
def test_kept_row_exchange_with_many_heads(wl):
    q, k, v = (x.cuda() for x in synth.make_qkv(wl))
    idx = attn.SgaIndex(wl, 2, 2)
    full = attn.sga(q, k, v, idx)
    hd = wl.H * wl.d
    cut = [0, 1, wl.N]
    parts, sums = [], torch.zeros(2, hd, dtype=torch.float32, device=q.device)
    for f0, f1 in zip(cut[:-1], cut[1:]):
        r0, r1 = f0 * wl.L, f1 * wl.L
        loc = attn.vggt_shape(f1 - f0, wl.n_special, wl.h, wl.w, wl.H, wl.d)
        nk = attn.vggt_sga_num_kept(loc, 2, 2)
        kk, kv = (torch.empty(nk, wl.H, wl.d, dtype=torch.bfloat16, device=q.device) for _ in range(2))
        ds = torch.empty(2, hd, dtype=torch.float32, device=q.device)
        nb = attn.vggt_sga_partial_workspace_bytes(loc)
        ws = torch.empty(nb, dtype=torch.uint8, device=q.device)
        assert attn.vggt_sga_gather_partial(k[r0:r1], v[r0:r1], loc, 2, 2, kk, kv, ds, ws, nb) == attn.VGGT_OK
        parts.append((kk, kv))
        sums += ds
    kept_k, kept_v = torch.cat([p[0] for p in parts]), torch.cat([p[1] for p in parts])
    assert torch.equal(kept_k, k[idx.kept_idx.long()]) and torch.equal(kept_v, v[idx.kept_idx.long()])
    o = torch.empty_like(q)
    means = torch.empty(2, hd, dtype=torch.float32, device=q.device)
    for f0, f1 in zip(cut[:-1], cut[1:]):
        r0, r1 = f0 * wl.L, f1 * wl.L
        assert attn.vggt_attn_sga_gathered(q[r0:r1], r0, r1 - r0, k[r0:r1], v[r0:r1], kept_k, kept_v, sums,
                                           idx.mult, means, o[r0:r1], None, wl, 2, 2,
                                           attn.default_scale(64)) == attn.VGGT_OK
    assert attn.vggt_check()[0] == attn.VGGT_OK
    assert (o.float() - full.float()).abs().max().item() <= 1e-2


@pytest.mark.parametrize("wl", WIDE, ids=[w.name for w in WIDE])
def test_projections_with_many_heads(wl):
    sh = oracle.Shape(wl.N, wl.n_special, wl.h, wl.w, wl.H, wl.d)
    C = wl.H * wl.d
    g = torch.Generator().manual_seed(3)
    x = torch.randn(wl.S, C, generator=g).to(torch.bfloat16)
    w = (torch.randn(3 * C, C, generator=g) / np.sqrt(C)).to(torch.bfloat16)
    b = (0.1 * torch.randn(3 * C, generator=g)).float()
    qq, kk, vv = attn.qkv_rope(x.cuda(), w.cuda(), wl, bias=b.cuda(), rope_base=100.0)
    assert attn.vggt_check()[0] == attn.VGGT_OK
    for got, ref in zip((qq, kk, vv), oracle.qkv_rope(x, w, b.numpy(), sh, 100.0)):
        compare(got, ref)
    y = attn.out_proj(x.cuda(), w[:C].contiguous().cuda(), wl, bias=b[:C].contiguous().cuda())
    assert attn.vggt_check()[0] == attn.VGGT_OK
    compare(y, oracle.linear(x, w[:C], b[:C].numpy()))
