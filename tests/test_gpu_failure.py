"""Failure detection on the GPU without a fault: a launch whose first
scores are never signalled must end on its own (every in-kernel wait is
bounded), report VGGT_ERR_TIMEOUT through vggt_check with the wait site in
the detail word, and leave the CUDA context usable for correct work."""
import time

import numpy as np
import pytest
import torch

import oracle
from feed_forward_view_vggt_b200 import attn, synth

pytestmark = pytest.mark.gpu

SITES = {7: "p_ready", 8: "s_full"}


def test_stalled_wait_times_out_and_context_survives():
    wl = synth.WORKLOADS["tiny"]
    q, k, v = synth.make_qkv(wl)
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    assert attn.vggt_check()[0] == attn.VGGT_OK
    o = torch.empty_like(qd)
    t0 = time.perf_counter()
    st = attn.vggt_test_attn_global_stall(qd, kd, vd, o, wl, 0.125, 50_000_000)  # 50 ms bound
    assert st == attn.VGGT_OK
    st, detail = attn.vggt_check()
    elapsed = time.perf_counter() - t0
    assert st == attn.VGGT_ERR_TIMEOUT
    assert detail & 1 and ((detail >> 8) & 0xFF) in SITES, hex(detail)
    assert elapsed < 5.0
    # the error word was cleared and the context still computes correctly
    assert attn.vggt_check()[0] == attn.VGGT_OK
    good = attn.global_(qd, kd, vd, wl)
    assert attn.vggt_check()[0] == attn.VGGT_OK
    sh = oracle.Shape(wl.N, wl.n_special, wl.h, wl.w, wl.H, wl.d)
    bits = [x.view(torch.int16).numpy().view(np.uint16) for x in (q, k, v)]
    ref, _ = oracle.global_attention(*bits, sh)
    assert np.abs(good.float().cpu().double().numpy() - ref).max() <= 2e-2
