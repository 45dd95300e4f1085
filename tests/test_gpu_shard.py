"""Head-sharded multi-GPU split, one rank at a time on one GPU: a rank's
head slice of the scene (synth.make_qkv_heads, H = h1 - h0 heads) runs
through vggt_attn_global and vggt_attn_sga exactly as bench.py --shard
heads runs it, and must match the oracle's output for heads [h0, h1) of
the whole scene.  Attention never mixes heads, so no rank needs another's
data; only the ranks' own runs are checked here (each one alone, so no
kernel waits on another)."""
import os
import sys

import numpy as np
import pytest
import torch

import oracle
from oracle import dense
from feed_forward_view_vggt_b200 import attn, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
REL_FRO = 5e-3


def compare(got, ref):
    err = np.abs(got - ref)
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert np.isfinite(got).all() and err.max() <= MAX_ABS and rel <= REL_FRO, (err.max(), rel)


@pytest.mark.parametrize("config,world,rank,count", [("n4", 4, 1, None), ("n4", 8, 7, None),
                                                     ("n4", 2, 0, None), ("n100", 8, 3, 512)])
def test_head_slice_matches_the_whole_scene(config, world, rank, count):
    full = synth.WORKLOADS[config]
    h0, h1 = bench.head_range(full.H, world, rank)
    wl, q, k, v = bench.rank_inputs(config, "heads", world, rank)
    assert wl.H == h1 - h0
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    o_glob = attn.global_(qd, kd, vd, wl)
    o_sga = attn.sga(qd, kd, vd, attn.SgaIndex(wl, 2, 2))
    assert attn.vggt_check()[0] == attn.VGGT_OK
    rows = (np.arange(full.S, dtype=np.int64) if count is None else
            synth.sample_rows(full.S, full.L, full.n_special, count=count, seed=1234))
    fq, fk, fv = synth.make_qkv(full)
    sh = oracle.Shape(full.N, full.n_special, full.h, full.w, full.H, full.d)
    idx = torch.as_tensor(rows).cuda()
    for o, (ref, _) in ((o_glob, dense.global_attention(fq, fk, fv, sh, rows=rows)),
                        (o_sga, dense.sga_attention(fq, fk, fv, sh, 2, 2, rows=rows))):
        compare(o[idx].double().cpu().numpy(), ref[:, h0:h1])


@pytest.mark.parametrize("config,world", [("n4", 2), ("n4", 3), ("tiny", 2), ("n32", 8)])
def test_query_row_blocks_reassemble_the_full_call(config, world):
    # Query-row split: each rank owns whole frames [f0, f1) and, after
    # gathering every K/V row, computes global attention and SGA for its
    # own query rows only.  Run here one rank at a time on one GPU: the
    # rank outputs, concatenated, must equal the full calls bit for bit
    # (each row's arithmetic is the same), and match the oracle.
    wl = synth.WORKLOADS[config]
    q, k, v = (x.cuda() for x in synth.make_qkv(wl))
    full_g, full_g_lse = attn.global_(q, k, v, wl, want_lse=True)
    idx = attn.SgaIndex(wl, 2, 2)
    full_s, full_s_lse = attn.sga(q, k, v, idx, want_lse=True)
    sc = attn.default_scale(64)
    og, os_ = torch.empty_like(q), torch.empty_like(q)
    lg = torch.empty(wl.S, wl.H, dtype=torch.float32, device=q.device)
    ls = torch.empty_like(lg)
    for rank in range(world):
        r0, r1 = (x * wl.L for x in bench.frame_range(wl.N, world, rank))
        if r1 == r0:
            continue
        assert attn.vggt_attn_global_rows(q[r0:r1], r1 - r0, k, v, og[r0:r1], lg[r0:r1], wl, sc) == attn.VGGT_OK
        assert attn.vggt_attn_sga_rows(q[r0:r1], r0, r1 - r0, k, v, os_[r0:r1], ls[r0:r1], wl, 2, 2, idx.kept_idx,
                                       idx.mult, idx.workspace, idx.workspace_bytes, sc) == attn.VGGT_OK
    assert attn.vggt_check()[0] == attn.VGGT_OK
    assert torch.equal(og, full_g) and torch.equal(lg, full_g_lse)
    assert torch.equal(os_, full_s) and torch.equal(ls, full_s_lse)
    rows = synth.sample_rows(wl.S, wl.L, wl.n_special, count=256, seed=5)
    fq, fk, fv = synth.make_qkv(wl)
    sh = oracle.Shape(wl.N, wl.n_special, wl.h, wl.w, wl.H, wl.d)
    idx_r = torch.as_tensor(rows).cuda()
    compare(og[idx_r].double().cpu().numpy(), dense.global_attention(fq, fk, fv, sh, rows=rows)[0])
    compare(os_[idx_r].double().cpu().numpy(), dense.sga_attention(fq, fk, fv, sh, 2, 2, rows=rows)[0])


@pytest.mark.parametrize("config,world,stride", [("n4", 3, (2, 2)), ("tiny", 2, (2, 2)), ("n32", 4, (3, 3)),
                                                 ("n4", 2, (1, 1)), ("n4", 8, (2, 2)), ("n100", 8, (2, 2))])
def test_kept_row_exchange_matches_the_full_call(config, world, stride):
    # The leaner query-row split for SGA: each rank gathers the kept K/V rows
    # and the dropped-token sums of its own frames (vggt_sga_gather_partial),
    # the ranks' kept rows are concatenated (the all-gather) and their sums
    # added (the all-reduce), and each rank runs SGA for its own query rows
    # (vggt_attn_sga_gathered).  One rank at a time on one GPU; the
    # collectives are done here with torch.cat and a sum.  The concatenated
    # kept rows must be exactly the index's kept rows, the output must match
    # the single-GPU call up to the rounding of k-bar / v-bar, and the oracle.
    wl = synth.WORKLOADS[config]
    s_h, s_w = stride
    q, k, v = (x.cuda() for x in synth.make_qkv(wl))
    idx = attn.SgaIndex(wl, s_h, s_w)
    full_s, full_lse = attn.sga(q, k, v, idx, want_lse=True)
    sc = attn.default_scale(64)
    hd = wl.H * wl.d
    kept_parts, sums = [], torch.zeros(2, hd, dtype=torch.float32, device=q.device)
    for rank in range(world):
        f0, f1 = bench.frame_range(wl.N, world, rank)
        if f1 == f0:
            continue
        r0, r1 = f0 * wl.L, f1 * wl.L
        loc = attn.vggt_shape(f1 - f0, wl.n_special, wl.h, wl.w, wl.H, wl.d)
        nk = attn.vggt_sga_num_kept(loc, s_h, s_w)
        kk = torch.empty(nk, wl.H, wl.d, dtype=torch.bfloat16, device=q.device)
        kv = torch.empty_like(kk)
        ds = torch.full((2, hd), float("nan"), dtype=torch.float32, device=q.device)
        nb = attn.vggt_sga_partial_workspace_bytes(loc)
        ws = torch.empty(nb, dtype=torch.uint8, device=q.device)
        assert attn.vggt_sga_gather_partial(k[r0:r1], v[r0:r1], loc, s_h, s_w, kk, kv, ds, ws, nb) == attn.VGGT_OK
        kept_parts.append((kk, kv))
        sums += ds
    kept_k = torch.cat([p[0] for p in kept_parts])
    kept_v = torch.cat([p[1] for p in kept_parts])
    rows_kept = idx.kept_idx.long()
    assert torch.equal(kept_k, k[rows_kept]) and torch.equal(kept_v, v[rows_kept])
    o = torch.empty_like(q)
    lse = torch.empty(wl.S, wl.H, dtype=torch.float32, device=q.device)
    means = torch.empty(2, hd, dtype=torch.float32, device=q.device)
    for rank in range(world):
        r0, r1 = (x * wl.L for x in bench.frame_range(wl.N, world, rank))
        if r1 == r0:
            continue
        assert attn.vggt_attn_sga_gathered(q[r0:r1], r0, r1 - r0, k[r0:r1], v[r0:r1], kept_k, kept_v, sums,
                                           idx.mult, means, o[r0:r1], lse[r0:r1], wl, s_h, s_w, sc) == attn.VGGT_OK
    assert attn.vggt_check()[0] == attn.VGGT_OK
    # k-bar / v-bar differ from the single-GPU ones only by the order of fp32 sums
    n_dropped = attn.vggt_sga_num_dropped(wl, s_h, s_w)
    if n_dropped > 0:
        ref_means = torch.stack([k[~torch.isin(torch.arange(wl.S, device=q.device), rows_kept)].float().sum(0)
                                 .reshape(-1), v[~torch.isin(torch.arange(wl.S, device=q.device), rows_kept)]
                                 .float().sum(0).reshape(-1)]) / n_dropped
        assert torch.allclose(means, ref_means, rtol=1e-5, atol=1e-6)
    assert (o.float() - full_s.float()).abs().max().item() <= 1e-2
    assert (lse - full_lse).abs().max().item() <= 1e-4
    rows = synth.sample_rows(wl.S, wl.L, wl.n_special, count=256, seed=9)
    fq, fk, fv = synth.make_qkv(wl)
    sh = oracle.Shape(wl.N, wl.n_special, wl.h, wl.w, wl.H, wl.d)
    idx_r = torch.as_tensor(rows).cuda()
    compare(o[idx_r].double().cpu().numpy(), dense.sga_attention(fq, fk, fv, sh, s_h, s_w, rows=rows)[0])
