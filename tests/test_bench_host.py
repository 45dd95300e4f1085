"""Host-side logic of bench.py on CPU: argument parsing, clock-sample
parsing, the traffic record's source check, the max-over-ranks reduction
with world_size 2 (gloo), and the reference arm on the tiny workload."""
import json
import os
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_parse_args_defaults():
    a = bench.parse_args([])
    assert (a.gpus, a.warmup, a.config, a.s_h, a.s_w, a.impl) == (1, 3, "n100", 2, 2, "ours")
    a = bench.parse_args(["--stride", "3x3", "--config", "n800", "--impl", "reference"])
    assert (a.s_h, a.s_w, a.config, a.impl) == (3, 3, "n800", "reference")


def test_head_ranges_partition_the_heads():
    for H, world in ((16, 1), (16, 2), (16, 4), (16, 8), (2, 2)):
        got = [bench.head_range(H, world, r) for r in range(world)]
        assert got[0][0] == 0 and got[-1][1] == H
        assert all(a[1] == b[0] for a, b in zip(got, got[1:]))
        assert len({h1 - h0 for h0, h1 in got}) == 1
    with pytest.raises(ValueError):
        bench.head_range(16, 3, 0)
    a = bench.parse_args(["--shard", "heads"])
    assert a.shard == "heads" and bench.parse_args([]).shard == "replicas"


def test_head_shards_reassemble_the_scene():
    from feed_forward_view_vggt_b200 import synth

    wl = synth.WORKLOADS["n4"]
    full = synth.make_qkv(wl)
    parts = [synth.make_qkv_heads(wl, *bench.head_range(wl.H, 4, r)) for r in range(4)]
    for j in range(3):
        assert torch.equal(torch.cat([p[j] for p in parts], dim=1), full[j])


def test_clock_summary_parsing():
    c = bench.ClockSampler(0)
    c.lines = [
        "0, 1800, 1965, 900.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1300, 1965, 990.5, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1400, 1965, 995.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "garbage line",
    ]
    s = c.summary()
    assert s["sm_mhz"] == 1400 and s["sm_max_mhz"] == 1965 and s["reasons"] == ["sw_power_cap"]
    assert s["samples"] == 3


FAKE_SMI = """#!{python}
import sys, time
time.sleep(0.4)  # start-up delay, as nvidia-smi has
i = 0
while True:
    print("0, %d, 1965, 900.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active" % (1000 + i),
          flush=True)
    i += 1
    time.sleep(0.05)
"""


def test_clock_sampler_waits_for_the_first_sample_and_keeps_the_timed_region(tmp_path, monkeypatch):
    import time

    smi = tmp_path / "nvidia-smi"
    smi.write_text(FAKE_SMI.format(python=sys.executable))
    smi.chmod(0o755)
    monkeypatch.setenv("PATH", str(tmp_path) + os.pathsep + os.environ.get("PATH", ""))
    t = time.monotonic()
    c = bench.ClockSampler(0, period_ms=50)
    with c:
        entered = time.monotonic() - t
        assert c.stamped  # the region starts only after the first sample
        time.sleep(0.3)
    assert entered >= 0.35
    s = c.summary()
    # about 0.3 s / 0.05 s samples inside the region, none from before it
    assert 3 <= s["samples"] <= 9, s
    first_inside = int(c.lines[0].split(",")[1])
    assert first_inside > 1000, "the sample taken before the region must not count"
    assert s["reasons"] == ["sw_power_cap"] and s["sm_max_mhz"] == 1965


def test_traffic_record_requires_matching_kernel_source(tmp_path, monkeypatch):
    rec = tmp_path / "t.json"
    rec.write_text(json.dumps({"kernel_source_sha256_16": "0" * 16, "dram_bytes_per_launch": 123.0}))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(rec))
    assert bench.recorded_traffic() is None
    rec.write_text(json.dumps({"kernel_source_sha256_16": bench.kernel_source_hash(),
                               "dram_bytes_per_launch": 123.0}))
    assert bench.recorded_traffic() == 123.0


def test_workload_flops_n100():
    from feed_forward_view_vggt_b200 import synth

    flops, nk, nd = bench.workload_flops(synth.WORKLOADS["n100"], 2, 2)
    assert (nk, nd) == (36600, 100800)
    assert abs(flops["global"] / flops["sga"] - 3.75) < 0.01


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # each rank reports a different elapsed time; every rank gets the max
        got = bench.max_over_ranks(10.0 + 5.0 * rank, world)
        out[rank] = got
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    port = 29500 + (os.getpid() % 1000)
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(2, port, out), nprocs=2, join=True)
        assert dict(out) == {0: 15.0, 1: 15.0}
    assert bench.max_over_ranks(3.5, 1) == 3.5


def test_reference_arm_tiny_prints_one_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config",
                        "tiny", "--steps", "1", "--warmup", "3"], capture_output=True, text=True, timeout=600,
                       cwd=ROOT)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["unit"] == "TFLOP/s" and j["value"] > 0
    assert j["e2e"]["h2d_bytes_per_step"] == 0 and j["cpu_baseline"]["kind"] == "oracle"


def test_reference_arm_nonzero_rank_exits_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config",
                        "tiny", "--steps", "1", "--warmup", "3"], capture_output=True, text=True, timeout=600,
                       cwd=ROOT, env=env)
    assert r.returncode == 0 and r.stdout.strip() == ""


def _head_shard_main(rank, world, port, out):
    # The bench's head-sharded rank logic on CPU: each rank draws its heads
    # of the scene (bench.rank_inputs), runs attention on them -- the fp64
    # oracle stands in for the kernels, which need a GPU -- and the outputs
    # are all-gathered over gloo and reassembled along the head axis.
    import numpy as np

    import oracle
    from oracle import dense

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        res = {}
        for config, rows in (("tiny", None), ("n4", np.arange(0, 5496, 97))):
            wl, q, k, v = bench.rank_inputs(config, "heads", world, rank)
            sh = oracle.Shape(wl.N, wl.n_special, wl.h, wl.w, wl.H, wl.d)
            mine = [torch.from_numpy(dense.global_attention(q, k, v, sh, rows=rows)[0]),
                    torch.from_numpy(dense.sga_attention(q, k, v, sh, 2, 2, rows=rows)[0])]
            for name, o in zip(("global", "sga"), mine):
                parts = [torch.empty_like(o) for _ in range(world)]
                dist.all_gather(parts, o)
                if rank == 0:
                    res[(config, name)] = torch.cat(parts, dim=1).numpy()
        out[rank] = res
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_head_sharded_ranks_reassemble_the_scene_output_two_gloo_ranks():
    import numpy as np

    import oracle
    from oracle import dense
    from feed_forward_view_vggt_b200 import synth

    port = 29500 + ((os.getpid() + 500) % 1000)
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_head_shard_main, args=(2, port, out), nprocs=2, join=True)
        got = dict(out)[0]
    for config, rows in (("tiny", None), ("n4", np.arange(0, 5496, 97))):
        wl = synth.WORKLOADS[config]
        q, k, v = synth.make_qkv(wl)
        sh = oracle.Shape(wl.N, wl.n_special, wl.h, wl.w, wl.H, wl.d)
        ref = {"global": dense.global_attention(q, k, v, sh, rows=rows)[0],
               "sga": dense.sga_attention(q, k, v, sh, 2, 2, rows=rows)[0]}
        for name in ("global", "sga"):
            assert got[(config, name)].shape == ref[name].shape
            assert np.abs(got[(config, name)] - ref[name]).max() <= 1e-12


def test_rank_inputs_replicas_differ_and_heads_slice():
    wl0, q0, _, _ = bench.rank_inputs("tiny", "replicas", 2, 0)
    wl1, q1, _, _ = bench.rank_inputs("tiny", "replicas", 2, 1)
    assert wl0.H == wl1.H == 2 and wl1.seed == wl0.seed + 1000 and not torch.equal(q0, q1)
    wlh, qh, _, _ = bench.rank_inputs("tiny", "heads", 2, 1)
    assert wlh.H == 1 and torch.equal(qh[:, 0], q0[:, 1])
    with pytest.raises(ValueError):
        bench.rank_inputs("tiny", "frames", 2, 0)


def test_sweep_appends_one_line_per_op_and_resumes_after_an_interruption(tmp_path):
    from feed_forward_view_vggt_b200 import synth

    path = tmp_path / "results.jsonl"
    a = bench.parse_args(["--sweep", "tiny,n32", "--results", str(path)])
    calls = []

    def flaky(wl, op):
        calls.append((wl.name, op))
        if (wl.name, op) == ("n32", "global"):
            raise KeyboardInterrupt  # the run stops in the middle of the sweep
        return {"ms": 1.0}

    with pytest.raises(KeyboardInterrupt):
        bench.run_sweep(a, measure=flaky)
    # a torn line from the interrupted write must not count as done
    with open(path, "a") as f:
        f.write('{"workload": "n32", "op": "glo')
    first = [ln for ln in open(path) if ln.endswith("\n")]
    assert [json.loads(x)["op"] for x in first] == ["frame", "global", "sga2x2", "frame"]

    calls.clear()
    new = bench.run_sweep(a, measure=lambda wl, op: (calls.append((wl.name, op)) or {"ms": 2.0}))
    assert calls == [("n32", "global"), ("n32", "sga2x2"), ("n32", "sga3x3")]
    assert [r["op"] for r in new] == ["global", "sga2x2", "sga3x3"]
    done = bench.load_done(str(path))
    want = {(n, op) for n in ("tiny", "n32") for op in bench.sweep_ops(synth.WORKLOADS[n])}
    assert done == want
    # a third run finds nothing to do
    assert bench.run_sweep(a, measure=lambda wl, op: pytest.fail("nothing left to time")) == []


def _query_split_main(rank, world, port, out):
    # The bench's query-row split on CPU: each rank holds the K/V rows of its
    # frames, FrameExchange all-gathers them over gloo exactly as the GPU
    # ranks do over NCCL, and each rank attends its own query rows against
    # the gathered keys (the fp64 oracle stands in for the kernels); the
    # ranks' outputs are gathered the same way and reassembled on rank 0.
    import numpy as np

    import oracle
    from oracle import dense
    from feed_forward_view_vggt_b200 import synth

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        res = {}
        for config in ("tiny", "n4"):
            wl = synth.WORKLOADS[config]
            q, k, v = synth.make_qkv(wl)
            like = torch.empty(1, wl.H, wl.d, dtype=torch.bfloat16)
            xk, xv = bench.FrameExchange(wl.N, wl.L, world, like), bench.FrameExchange(wl.N, wl.L, world, like)
            r0, r1 = xk.rows(rank)
            xk.local[:r1 - r0].copy_(k[r0:r1])
            xv.local[:r1 - r0].copy_(v[r0:r1])
            k_all, v_all = xk.exchange(), xv.exchange()
            assert torch.equal(k_all, k) and torch.equal(v_all, v)
            q_mine = torch.zeros_like(q)
            q_mine[r0:r1] = q[r0:r1]  # the oracle reads only the listed rows
            sh = oracle.Shape(wl.N, wl.n_special, wl.h, wl.w, wl.H, wl.d)
            rows = np.arange(r0, r1, dtype=np.int64)
            for name in ("global", "sga"):
                xo = bench.FrameExchange(wl.N, wl.L, world, torch.empty(1, wl.H, wl.d, dtype=torch.float64))
                if r1 > r0:
                    o = (dense.global_attention(q_mine, k_all, v_all, sh, rows=rows)[0] if name == "global" else
                         dense.sga_attention(q_mine, k_all, v_all, sh, 2, 2, rows=rows)[0])
                    xo.local[:r1 - r0].copy_(torch.from_numpy(o))
                full = xo.exchange()
                if rank == 0:
                    res[(config, name)] = full.numpy().copy()
        out[rank] = res
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_query_row_split_three_gloo_ranks_uneven_frames():
    import numpy as np

    import oracle
    from oracle import dense
    from feed_forward_view_vggt_b200 import synth

    # tiny: 2 frames over 3 ranks (rank 0 holds none); n4: 4 frames as 1 / 1 / 2
    assert [bench.frame_range(2, 3, r) for r in range(3)] == [(0, 0), (0, 1), (1, 2)]
    assert [bench.frame_range(4, 3, r) for r in range(3)] == [(0, 1), (1, 2), (2, 4)]
    port = 29500 + ((os.getpid() + 250) % 1000)
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_query_split_main, args=(3, port, out), nprocs=3, join=True)
        got = dict(out)[0]
    for config in ("tiny", "n4"):
        wl = synth.WORKLOADS[config]
        q, k, v = synth.make_qkv(wl)
        sh = oracle.Shape(wl.N, wl.n_special, wl.h, wl.w, wl.H, wl.d)
        ref = {"global": dense.global_attention(q, k, v, sh)[0], "sga": dense.sga_attention(q, k, v, sh, 2, 2)[0]}
        for name in ("global", "sga"):
            assert np.abs(got[(config, name)] - ref[name]).max() <= 1e-12, (config, name)


def _kept_exchange_main(rank, world, port, out):
    # The kept-row exchange of the query-row split for SGA, on CPU: each rank
    # takes the kept K/V rows and the dropped-token sums of its own frames --
    # the oracle's index and means, applied to the rank's frames alone, stand
    # in for vggt_sga_gather_partial -- and KeptExchange all-gathers the rows
    # and all-reduces the sums over gloo exactly as the GPU ranks do over NCCL.
    import numpy as np

    import oracle
    from feed_forward_view_vggt_b200 import synth

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        res = {}
        for config, (s_h, s_w) in (("tiny", (2, 2)), ("n4", (2, 2)), ("n4", (3, 3))):
            wl = synth.WORKLOADS[config]
            q, k, v = synth.make_qkv(wl)
            f0, f1 = bench.frame_range(wl.N, world, rank)
            r0, r1 = f0 * wl.L, f1 * wl.L
            counts = bench.kept_counts(wl, world, s_h, s_w)
            x = bench.KeptExchange(counts, wl.H, wl.d, "cpu")
            if f1 > f0:
                loc = oracle.Shape(f1 - f0, wl.n_special, wl.h, wl.w, wl.H, wl.d)
                kept_loc, _, nk, nd = oracle.sga_build_index(loc, s_h, s_w)
                assert nk == counts[rank]
                ids = torch.as_tensor(kept_loc.astype(np.int64))
                x.local_k[:nk] = k[r0:r1][ids]
                x.local_v[:nk] = v[r0:r1][ids]
                if nd > 0:
                    kb, vb = oracle.sga_means(k[r0:r1], v[r0:r1], loc, s_h, s_w)
                    x.sums[0] = torch.from_numpy(kb.reshape(-1) * nd).float()
                    x.sums[1] = torch.from_numpy(vb.reshape(-1) * nd).float()
            full_k, full_v, sums = x.exchange()
            if rank == 0:
                res[(config, s_h)] = (full_k.clone(), full_v.clone(), sums.clone())
        out[rank] = res
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_kept_row_exchange_three_gloo_ranks_uneven_frames():
    import numpy as np

    import oracle
    from feed_forward_view_vggt_b200 import synth

    port = 29500 + ((os.getpid() + 750) % 1000)
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_kept_exchange_main, args=(3, port, out), nprocs=3, join=True)
        got = dict(out)[0]
    for config, (s_h, s_w) in (("tiny", (2, 2)), ("n4", (2, 2)), ("n4", (3, 3))):
        wl = synth.WORKLOADS[config]
        q, k, v = synth.make_qkv(wl)
        sh = oracle.Shape(wl.N, wl.n_special, wl.h, wl.w, wl.H, wl.d)
        kept, _, nk, nd = oracle.sga_build_index(sh, s_h, s_w)
        full_k, full_v, sums = got[(config, s_h)]
        ids = torch.as_tensor(kept.astype(np.int64))
        # the ranks' kept rows, in rank order, are the whole sequence's kept rows
        assert sum(bench.kept_counts(wl, 3, s_h, s_w)) == nk
        assert torch.equal(full_k, k[ids]) and torch.equal(full_v, v[ids])
        # the summed dropped-token sums give the whole sequence's means
        kb, vb = oracle.sga_means(k, v, sh, s_h, s_w)
        assert np.abs(sums[0].double().numpy() / nd - kb.reshape(-1)).max() <= 1e-5
        assert np.abs(sums[1].double().numpy() / nd - vb.reshape(-1)).max() <= 1e-5
