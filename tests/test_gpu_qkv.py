"""Fused QKV projection + 2D RoPE on the GPU against the fp64 oracle: the
whole output at Tiny (H = 2, single-CTA form with 128-column tiles) and
N = 4 (H = 16, CTA-pair form with 256 x 256 tiles), sampled rows at
N = 100, without bias, with another rotation base, and ragged last row
blocks (one where the pair's second CTA holds a few rows, one where it
holds none)."""
import numpy as np
import pytest
import torch

import oracle
from feed_forward_view_vggt_b200 import attn, synth

pytestmark = pytest.mark.gpu


def inputs(wl, seed):
    g = torch.Generator().manual_seed(seed)
    C = wl.H * wl.d
    x = torch.randn(wl.S, C, generator=g).to(torch.bfloat16)
    w = (torch.randn(3 * C, C, generator=g) / np.sqrt(C)).to(torch.bfloat16)
    b = (0.1 * torch.randn(3 * C, generator=g)).float()
    return x, w, b


def check(got, ref):
    got = got.float().cpu().double().numpy().reshape(ref.shape)
    err = np.abs(got - ref)
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert np.isfinite(got).all() and err.max() <= 2e-2 and rel <= 5e-3, (err.max(), rel)


@pytest.mark.parametrize("name,rows,bias,base", [("tiny", None, True, 100.0), ("n4", None, True, 100.0),
                                                 ("tiny", None, False, 10000.0), ("n100", 256, True, 100.0)])
def test_qkv_rope_matches_oracle(name, rows, bias, base):
    wl = synth.WORKLOADS[name]
    sh = oracle.Shape(wl.N, wl.n_special, wl.h, wl.w, wl.H, wl.d)
    x, w, b = inputs(wl, 7)
    sel = None if rows is None else synth.sample_rows(wl.S, wl.L, wl.n_special, count=rows, seed=99)
    q, k, v = attn.qkv_rope(x.cuda(), w.cuda(), wl, bias=b.cuda() if bias else None, rope_base=base)
    assert attn.vggt_check()[0] == attn.VGGT_OK
    rq, rk, rv = oracle.qkv_rope(x, w, b.numpy() if bias else None, sh, base, rows=sel)
    if sel is not None:
        idx = torch.as_tensor(sel).cuda()
        q, k, v = q[idx], k[idx], v[idx]
    check(q, rq)
    check(k, rk)
    check(v, rv)


def test_ragged_last_row_block_and_specials():
    # S = 3 * (5 + 6*7) = 141 rows: the second 128-row block holds 13 rows
    wl = synth.Workload("qkv_ragged", N=3, h=6, w=7, H=4, seed=21, structure="iid")
    sh = oracle.Shape(wl.N, wl.n_special, wl.h, wl.w, wl.H, wl.d)
    x, w, b = inputs(wl, 3)
    # the three outputs sit in one buffer, each followed by a guard zone
    n, gap = wl.S * wl.H * wl.d, 4096
    buf = torch.full((3 * (n + gap),), 9.0, dtype=torch.bfloat16, device="cuda")
    out = [buf[i * (n + gap):i * (n + gap) + n].view(wl.S, wl.H, wl.d) for i in range(3)]
    st = attn.vggt_qkv_rope(x.cuda(), w.cuda(), b.cuda(), *out, wl, 100.0)
    assert st == attn.VGGT_OK and attn.vggt_check()[0] == attn.VGGT_OK
    for got, ref in zip(out, oracle.qkv_rope(x, w, b.numpy(), sh, 100.0)):
        check(got, ref)
    for i in range(3):
        assert bool((buf[i * (n + gap) + n:(i + 1) * (n + gap)] == 9.0).all()), "write past an output"


def test_bias_not_16_byte_aligned():
    # a bias 4 bytes past a 16-byte boundary takes the epilogue's scalar loads
    wl = synth.WORKLOADS["n4"]
    sh = oracle.Shape(wl.N, wl.n_special, wl.h, wl.w, wl.H, wl.d)
    x, w, b = inputs(wl, 8)
    buf = torch.zeros(b.numel() + 1, dtype=torch.float32, device="cuda")
    buf[1:] = b.cuda()
    bias = buf[1:]
    assert bias.data_ptr() % 16 == 4
    q, k, v = attn.qkv_rope(x.cuda(), w.cuda(), wl, bias=bias, rope_base=100.0)
    assert attn.vggt_check()[0] == attn.VGGT_OK
    for got, ref in zip((q, k, v), oracle.qkv_rope(x, w, b.numpy(), sh, 100.0)):
        check(got, ref)


def test_pair_tile_with_empty_second_half():
    # S = 7 * 47 = 329 rows: the second 256-row tile holds 73 rows, all in
    # the first CTA of the pair; C = 256 gives three 256-column tiles
    wl = synth.Workload("qkv_pair_tail", N=7, h=6, w=7, H=4, seed=22, structure="iid")
    sh = oracle.Shape(wl.N, wl.n_special, wl.h, wl.w, wl.H, wl.d)
    x, w, b = inputs(wl, 5)
    q, k, v = attn.qkv_rope(x.cuda(), w.cuda(), wl, bias=b.cuda(), rope_base=100.0)
    assert attn.vggt_check()[0] == attn.VGGT_OK
    for got, ref in zip((q, k, v), oracle.qkv_rope(x, w, b.numpy(), sh, 100.0)):
        check(got, ref)
    # output projection of the same rows: one 256-column tile
    o = torch.randn(wl.S, wl.H * wl.d, generator=torch.Generator().manual_seed(6)).to(torch.bfloat16)
    y = attn.out_proj(o.cuda(), w[: wl.H * wl.d].contiguous().cuda(), wl, bias=None)
    assert attn.vggt_check()[0] == attn.VGGT_OK
    check(y, oracle.linear(o, w[: wl.H * wl.d], None))


@pytest.mark.parametrize("name,bias", [("tiny", True), ("n4", True), ("n4", False)])
def test_out_proj_matches_oracle(name, bias):
    wl = synth.WORKLOADS[name]
    C = wl.H * wl.d
    g = torch.Generator().manual_seed(13)
    o = torch.randn(wl.S, C, generator=g).to(torch.bfloat16)
    w = (torch.randn(C, C, generator=g) / np.sqrt(C)).to(torch.bfloat16)
    b = (0.1 * torch.randn(C, generator=g)).float()
    y = attn.out_proj(o.cuda(), w.cuda(), wl, bias=b.cuda() if bias else None)
    assert attn.vggt_check()[0] == attn.VGGT_OK
    check(y, oracle.linear(o, w, b.numpy() if bias else None))
