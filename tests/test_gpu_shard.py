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
