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
