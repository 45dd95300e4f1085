#!/usr/bin/env python
"""Benchmark of the VGGT alternating-attention hot path on B200.

One step = every row of the hot path once over one synthetic batch:
frame attention, global attention, the SGA index build, the SGA gather +
mean-fill (+ finalisation) and SGA attention (stride 2x2), all through the
C ABI.  Default workload: N=100 frames x 1374 tokens (137,400 tokens), H=16,
d=64, bf16 -- the configuration the global-vs-SGA comparison is quoted on.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config n100]
    python bench.py --impl reference ...   # the fp64 CPU oracle as reference arm

Prints one JSON line (rank 0).  With N > 1 (launched by torchrun, one rank
per GPU) each rank runs an independent replica of the workload (different
seed); there is no collective on the data path; the timed region is
bracketed by a barrier and a device synchronize on every rank and the
reported time is the maximum over ranks (weak scaling).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "global-attn layer ms & TFLOP/s (frac. of BF16 peak) at N=100/800, SGA vs full"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 1024 * 1024
KERNEL_SOURCES = ["feed_forward_view_vggt_b200/csrc/attn_kernel.cuh", "feed_forward_view_vggt_b200/csrc/ptx.cuh"]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attn_global_n100_traffic.json")


# --------------------------------------------------------------- host logic

def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default="n100", choices=["tiny", "n4", "n32", "n100", "n300", "n800", "omega100"])
    ap.add_argument("--stride", default="2x2", help="SGA stride s_h x s_w")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle timing (profiling runs)")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end loop")
    ap.add_argument("--no-trunks", action="store_true", help="skip the whole-trunk schedule timings")
    ap.add_argument("--sweep", default="",
                    help="comma-separated workloads: time every op of each on its own and append one JSON line "
                         "per (workload, op) to --results, skipping the ones already there (resume)")
    ap.add_argument("--results", default="bench_results.jsonl", help="results file of --sweep")
    ap.add_argument("--shard", default="replicas", choices=["replicas", "heads", "queries"],
                    help="replicas: every rank runs its own scene (weak scaling); heads: the ranks split the "
                         "heads of one scene, with no exchange (strong scaling); queries: the ranks split the "
                         "frames of one scene, all-gather K and V every step and attend their own query rows "
                         "(strong scaling)")
    ap.add_argument("--layer", default="step", choices=["step", "sga"],
                    help="with --shard queries: step = frame + global + SGA with K and V all-gathered; sga = one "
                         "AVGGT SGA layer with only the kept K/V rows all-gathered and the dropped-token sums "
                         "all-reduced")
    a = ap.parse_args(argv)
    a.s_h, a.s_w = (int(x) for x in a.stride.lower().split("x"))
    return a


def head_range(H: int, world: int, rank: int):
    """Heads [h0, h1) of one rank when `world` ranks split H heads evenly."""
    if world < 1 or not 0 <= rank < world or H % world:
        raise ValueError(f"{H} heads do not split evenly over {world} ranks")
    per = H // world
    return rank * per, (rank + 1) * per


def frame_range(N: int, world: int, rank: int):
    """Frames [f0, f1) of one rank when `world` ranks split N frames as
    evenly as possible (query-row split)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank out of range")
    return rank * N // world, (rank + 1) * N // world


class FrameExchange:
    """The K/V exchange of the query-row split: rank r holds the K or V rows
    of its frames [f0, f1) (frame_range) in a buffer padded to the largest
    rank's row count; one all-gather brings every rank's buffer into
    `gathered` ([world * rows_max, H, d]), and a copy per rank packs the
    rows into the sequence order of `full` ([S, H, d]).  Works on any
    torch.distributed backend (NCCL on GPUs, gloo on the host)."""

    def __init__(self, N: int, L: int, world: int, like):
        import torch

        self.N, self.L, self.world = N, L, world
        self.ranges = [frame_range(N, world, r) for r in range(world)]
        self.rows_max = max(f1 - f0 for f0, f1 in self.ranges) * L
        shape = (self.rows_max,) + tuple(like.shape[1:])
        self.local = torch.zeros(shape, dtype=like.dtype, device=like.device)
        self.gathered = torch.empty((world * self.rows_max,) + shape[1:], dtype=like.dtype, device=like.device)
        self.full = torch.empty((N * L,) + shape[1:], dtype=like.dtype, device=like.device)

    def rows(self, rank: int):
        f0, f1 = self.ranges[rank]
        return f0 * self.L, f1 * self.L

    def exchange(self):
        """All-gather of every rank's `local` rows, packed into `full`."""
        if self.world > 1:
            import torch.distributed as dist

            dist.all_gather_into_tensor(self.gathered, self.local)
        else:
            self.gathered.copy_(self.local)
        for r in range(self.world):
            r0, r1 = self.rows(r)
            if r1 > r0:
                self.full[r0:r1].copy_(self.gathered[r * self.rows_max:r * self.rows_max + (r1 - r0)])
        return self.full


class KeptExchange:
    """The kept-row exchange of the query-row split for SGA: rank r gathers
    the kept K and V rows of its frames (n_kept[r] rows, sequence order) into
    `local_k` / `local_v`, padded to the largest rank's count; one all-gather
    each brings every rank's rows into `gathered_*`, a copy per rank packs
    them into `full_k` / `full_v` (the kept rows of the whole sequence, in
    sequence order), and one all-reduce adds the ranks' dropped-token sums
    ([2, H * d] fp32).  Works on any torch.distributed backend."""

    def __init__(self, n_kept, H: int, d: int, device, dtype=None):
        import torch

        dtype = dtype or torch.bfloat16
        self.n_kept = [int(x) for x in n_kept]
        self.world = len(self.n_kept)
        self.rows_max = max(max(self.n_kept), 1)
        self.local_k = torch.zeros(self.rows_max, H, d, dtype=dtype, device=device)
        self.local_v = torch.zeros_like(self.local_k)
        self.gathered_k = torch.empty(self.world * self.rows_max, H, d, dtype=dtype, device=device)
        self.gathered_v = torch.empty_like(self.gathered_k)
        total = max(sum(self.n_kept), 1)
        self.full_k = torch.empty(total, H, d, dtype=dtype, device=device)
        self.full_v = torch.empty_like(self.full_k)
        self.sums = torch.zeros(2, H * d, dtype=torch.float32, device=device)

    def exchange(self):
        """All-gather of the ranks' kept rows (packed into full_k / full_v) and
        all-reduce (sum) of `sums`."""
        if self.world > 1:
            import torch.distributed as dist

            dist.all_gather_into_tensor(self.gathered_k, self.local_k)
            dist.all_gather_into_tensor(self.gathered_v, self.local_v)
            dist.all_reduce(self.sums)
        else:
            self.gathered_k.copy_(self.local_k)
            self.gathered_v.copy_(self.local_v)
        at = 0
        for r, n in enumerate(self.n_kept):
            if n > 0:
                self.full_k[at:at + n].copy_(self.gathered_k[r * self.rows_max:r * self.rows_max + n])
                self.full_v[at:at + n].copy_(self.gathered_v[r * self.rows_max:r * self.rows_max + n])
            at += n
        return self.full_k, self.full_v, self.sums


def kept_counts(wl, world: int, s_h: int, s_w: int):
    """Kept rows of each rank's frames under the query-row split: the kept
    pattern repeats every frame, so a rank's count is its frame count times
    the per-frame count (closed form, host)."""
    from feed_forward_view_vggt_b200 import accounting

    per_frame = accounting.sga_counts(1, wl.n_special, wl.h, wl.w, s_h, s_w)[0]
    return [(f1 - f0) * per_frame for f0, f1 in (frame_range(wl.N, world, r) for r in range(world))]


def rank_inputs(config: str, shard: str, world: int, rank: int):
    """This rank's workload and seeded (Q, K, V), CPU bf16 [S, H, d].

    replicas: every rank draws its own scene (seed + 1000 * rank), all heads.
    heads:    the ranks split the heads of one scene; this rank draws exactly
              heads head_range(H, world, rank) of it (attention never mixes
              heads, so no rank needs another's data)."""
    from feed_forward_view_vggt_b200 import synth

    base = synth.WORKLOADS[config]
    if shard == "heads":
        h0, h1 = head_range(base.H, world, rank)
        wl = synth.Workload(base.name, base.N, base.h, base.w, h1 - h0, base.seed, base.structure,
                            base.sga_strides, base.n_special, base.d)
        return (wl, *synth.make_qkv_heads(base, h0, h1))
    if shard != "replicas":
        raise ValueError(f"unknown shard mode {shard!r}")
    wl = synth.Workload(base.name, base.N, base.h, base.w, base.H, base.seed + 1000 * rank, base.structure,
                        base.sga_strides, base.n_special, base.d)
    return (wl, *synth.make_qkv(wl))


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Maximum of a per-rank float over all ranks (identity for one rank)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic():
    """DRAM bytes per launch of the global-attention kernel from the committed
    ncu summary, or None when missing or taken on a different kernel source."""
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    if rec.get("kernel_source_sha256_16") != kernel_source_hash():
        return None
    return float(rec["dram_bytes_per_launch"])


def workload_flops(wl, s_h, s_w):
    from feed_forward_view_vggt_b200 import accounting as acc

    nk, nd = acc.sga_counts(wl.N, wl.n_special, wl.h, wl.w, s_h, s_w)
    return {
        "frame": acc.flops_frame(wl.N, wl.L, wl.H, wl.d),
        "global": acc.flops_global(wl.S, wl.H, wl.d),
        "sga": acc.flops_sga(wl.S, nk, nd, wl.H, wl.d),
    }, nk, nd


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs.

    nvidia-smi takes a few hundred ms to start, so it is started first and
    the timed region begins only after its first sample has arrived; each
    sample is stamped on arrival and only those inside the region count."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int, period_ms: int = 100):
        self.device_index = device_index
        self.period_ms = period_ms
        self.proc = None
        self.stamped = []
        self.lines = []
        self.t0 = self.t1 = None

    def _read(self):
        for ln in self.proc.stdout:
            if ln.strip():
                self.stamped.append((time.monotonic(), ln.strip()))

    def __enter__(self):
        import threading

        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.device_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", str(self.period_ms)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        if self.proc is not None:
            self.reader = threading.Thread(target=self._read, daemon=True)
            self.reader.start()
            deadline = time.monotonic() + 5.0
            while not self.stamped and time.monotonic() < deadline and self.proc.poll() is None:
                time.sleep(0.01)
        self.t0 = time.monotonic()
        return self

    def __exit__(self, *exc):
        self.t1 = time.monotonic()
        if self.proc is not None:
            # one more period so the last interval inside the region is reported
            time.sleep(self.period_ms / 1000.0)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.proc.wait()
            self.reader.join(timeout=5)
            inside = [ln for t, ln in self.stamped if self.t0 <= t <= self.t1 + self.period_ms / 1000.0]
            self.lines = inside or [ln for _, ln in self.stamped[-1:]]
        return False

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------- CPU oracle

def oracle_sample_timing(wl, s_h, s_w, rows_per_op, q, k, v, nthreads=0, measured=None):
    """Times the fp64 oracle on a bounded sample of query rows of every op;
    returns (seconds per op extrapolated to the whole layer, rows used,
    threads).  When `measured` is a dict, the seconds actually spent on each
    op's sample are stored in it."""
    import numpy as np

    import oracle
    from feed_forward_view_vggt_b200 import synth

    sh = oracle.Shape(wl.N, wl.n_special, wl.h, wl.w, wl.H, wl.d)
    bits = [x.contiguous().view(__import__("torch").int16).numpy().view(np.uint16) for x in (q, k, v)]
    threads = nthreads if nthreads > 0 else oracle.hardware_threads()
    full, used = {}, {}
    for op, mode in (("frame", oracle.FRAME), ("global", oracle.GLOBAL), ("sga", oracle.SGA)):
        n = min(rows_per_op[op], wl.S)
        rows = synth.sample_rows(wl.S, wl.L, wl.n_special, count=n, seed=4321)
        t0 = time.perf_counter()
        oracle.attention(mode, *bits, sh, s_h=s_h, s_w=s_w, rows=rows, nthreads=threads)
        dt = time.perf_counter() - t0
        full[op] = dt * wl.S / len(rows)
        used[op] = len(rows)
        if measured is not None:
            measured[op] = measured.get(op, 0.0) + dt
    return full, used, threads


def default_oracle_rows(wl):
    # about 10-30 s of host work on a 16-core box at N=100
    if wl.S <= 6000:
        return {"frame": wl.S, "global": wl.S, "sga": wl.S}
    scale = 137400 / wl.S
    return {"frame": 2048, "global": max(16, int(96 * scale)), "sga": max(16, int(256 * scale))}


def l2_note(wl):
    """How the timed steps keep L2 from serving inputs between steps."""
    qkv_bytes = wl.S * wl.H * wl.d * 2
    if 3 * qkv_bytes < 2 * L2_BYTES:
        return "flushed between steps"
    return f"inputs larger than L2 (Q/K/V {qkv_bytes / 1e6:.0f} MB each)"


def parallelism_note(shard, world, heads_per_rank):
    if shard == "heads":
        return f"heads split over {world} ranks, {heads_per_rank} each (no data-path collective)"
    return f"replicas x{world} (no data-path collective)"


def step_config(wl, s_h, s_w, n_kept, n_dropped, step_flops, l2, parallelism):
    """The `config` object both arms print for one workload."""
    return {"workload": f"{wl.name}: N={wl.N} frames x {wl.L} tokens ({wl.S} tokens), H={wl.H}, d={wl.d}",
            "ops": "frame + global + SGA index + SGA gather/mean-fill + SGA attention",
            "sga_stride": f"{s_h}x{s_w}", "n_kept": n_kept, "n_dropped": n_dropped,
            "step_flop": step_flops, "l2": l2, "parallelism": parallelism}


# --------------------------------------------------------------- GPU arm

TRUNK_MAX_TOKENS = 200_000


def time_projections(wl, dev, stream, call):
    import torch

    from feed_forward_view_vggt_b200 import attn

    C = wl.H * wl.d
    g = torch.Generator().manual_seed(wl.seed + 77)
    x = torch.randn(wl.S, C, generator=g).to(torch.bfloat16).to(dev)
    w = (torch.randn(3 * C, C, generator=g) / math.sqrt(C)).to(torch.bfloat16).to(dev)
    b = (0.1 * torch.randn(3 * C, generator=g)).float().to(dev)
    q, k, v = (torch.empty(wl.S, wl.H, wl.d, dtype=torch.bfloat16, device=dev) for _ in range(3))
    wo, bo = w[:C], b[:C]
    y = torch.empty(wl.S, C, dtype=torch.bfloat16, device=dev)

    def timed(fn):
        for _ in range(3):
            fn()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(10)]
        for a_, b_ in evs:
            a_.record(stream)
            fn()
            b_.record(stream)
        torch.cuda.synchronize(dev)
        return statistics.mean(a_.elapsed_time(b_) for a_, b_ in evs)

    ms = timed(lambda: call(attn.vggt_qkv_rope(x, w, b, q, k, v, wl, 100.0, stream), "qkv_rope"))
    flop = 2 * wl.S * C * 3 * C
    qkv = {"ms": round(ms, 4), "flop": flop, "tflops": round(flop / (ms * 1e-3) / 1e12, 1),
           "shape": f"[{wl.S} x {C}] x [{C} x {3 * C}] + bias, RoPE on Q and K", "launches": 1}
    ms = timed(lambda: call(attn.vggt_out_proj(q, wo, bo, y, wl, stream), "out_proj"))
    flop = 2 * wl.S * C * C
    out = {"ms": round(ms, 4), "flop": flop, "tflops": round(flop / (ms * 1e-3) / 1e12, 1),
           "shape": f"[{wl.S} x {C}] x [{C} x {C}] + bias", "launches": 1}
    return qkv, out


def time_trunks(wl, q, k, v, outs, s_h, s_w, scale, stream, call):
    """Attention time of whole VGGT / AVGGT / VGGT-Omega trunks through the
    schedule driver, every layer on this workload's Q/K/V.

    Up to TRUNK_MAX_TOKENS tokens each trunk runs whole (one untimed run,
    then one timed run).  Above it a 24-layer global trunk would take tens
    of seconds, so each distinct layer kind is timed as a one-layer
    schedule (one untimed run, then the mean of `reps` timed runs) and a
    trunk's time is the sum over its layers of its kind's time; the output
    says which ("timing")."""
    import torch

    from feed_forward_view_vggt_b200 import accounting, attn, schedules

    trunks = {"vggt": schedules.vggt_trunk(), "avggt": schedules.avggt_trunk(stride=(s_h, s_w))}
    if wl.n_special > 0:
        trunks["omega"] = schedules.omega_trunk()
    whole = wl.S <= TRUNK_MAX_TOKENS
    res = {"depth": schedules.DEPTH,
           "timing": ("whole trunks, one timed run each" if whole else
                      f"per layer kind: each kind timed as a one-layer schedule (mean of 3 runs), trunk time = "
                      f"sum over its layers (S = {wl.S} > {TRUNK_MAX_TOKENS} tokens)")}

    def timed_schedule(layers, reps):
        n = len(layers)
        nbytes = attn.vggt_schedule_workspace_bytes(wl, layers)
        ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=q.device)
        o_list = [outs[i % 2] for i in range(n)]

        def run():
            call(attn.vggt_attn_schedule([q] * n, [k] * n, [v] * n, o_list, wl, layers, scale, ws, nbytes, stream),
                 "schedule")

        run()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for e0, e1 in evs:
            e0.record(stream)
            run()
            e1.record(stream)
        torch.cuda.synchronize(q.device)
        del ws
        return statistics.mean(e0.elapsed_time(e1) for e0, e1 in evs)

    kind_ms = {}
    if not whole:
        for layers in trunks.values():
            for kind in schedules.kind_counts(layers):
                if kind not in kind_ms:
                    kind_ms[kind] = timed_schedule([kind if isinstance(kind, str) else list(kind)], 3)
        res["layer_ms"] = {(x if isinstance(x, str) else "sga%dx%d" % (x[1], x[2])): round(t, 3)
                           for x, t in kind_ms.items()}
    for name, layers in trunks.items():
        counts = schedules.kind_counts(layers)
        ms = timed_schedule(layers, 1) if whole else sum(c * kind_ms[x] for x, c in counts.items())
        fl = accounting.flops_schedule(layers, wl.N, wl.n_special, wl.h, wl.w, wl.H, wl.d)
        kinds = {(x if isinstance(x, str) else "sga%dx%d" % (x[1], x[2])): c for x, c in counts.items()}
        res[name] = {"layers": len(layers), "kinds": kinds, "ms": round(ms, 2), "flop": fl,
                     "tflops": round(fl / (ms * 1e-3) / 1e12, 1)}
    res["avggt_speedup_vs_vggt"] = round(res["vggt"]["ms"] / res["avggt"]["ms"], 3)
    if "omega" in res:
        res["omega_speedup_vs_vggt"] = round(res["vggt"]["ms"] / res["omega"]["ms"], 3)
    return res


def run_ours(a):
    import torch

    from feed_forward_view_vggt_b200 import attn, synth

    rank, world, local = dist_env()
    if world > 1:
        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=300))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    wl, q_h, k_h, v_h = rank_inputs(a.config, a.shard, world, rank)
    flops, n_kept, n_dropped = workload_flops(wl, a.s_h, a.s_w)
    step_flops = sum(flops.values())

    q, k, v = (x.to(dev) for x in (q_h, k_h, v_h))
    o_frame, o_global, o_sga = (torch.empty_like(q) for _ in range(3))
    index = attn.SgaIndex(wl, a.s_h, a.s_w, device=dev)
    in_bytes = 3 * q.numel() * 2
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev) if in_bytes < 2 * L2_BYTES else None
    stream = torch.cuda.current_stream(dev)
    scale = 1.0 / math.sqrt(wl.d)
    ops = ("frame", "global", "index", "sga")
    launches_per_step = 3 + 2 + (1 if n_dropped > 0 else 0)  # frame, global, index; gather, attn; finalize

    def call(status, what):
        if status != attn.VGGT_OK:
            raise attn.VggtError(status, what)

    def step(qq, kk, vv, ev=None, outs=None):
        of, og, os_ = (o_frame, o_global, o_sga) if outs is None else outs
        if ev is not None:
            ev[0].record(stream)
        call(attn.vggt_attn_frame(qq, kk, vv, of, None, wl, scale, stream), "frame")
        if ev is not None:
            ev[1].record(stream)
        call(attn.vggt_attn_global(qq, kk, vv, og, None, wl, scale, stream), "global")
        if ev is not None:
            ev[2].record(stream)
        call(attn.vggt_sga_build_index(wl, a.s_h, a.s_w, index.kept_idx, index.mult, stream), "index")
        if ev is not None:
            ev[3].record(stream)
        call(attn.vggt_attn_sga(qq, kk, vv, os_, None, wl, a.s_h, a.s_w, index.kept_idx, index.mult,
                                index.workspace, index.workspace_bytes, scale, stream), "sga")
        if ev is not None:
            ev[4].record(stream)

    def barrier():
        if world > 1:
            import torch.distributed as dist

            dist.barrier(device_ids=[local])

    for _ in range(max(a.warmup, 0)):
        step(q, k, v)
        if flush is not None:
            flush.zero_()
    st, detail = attn.vggt_check(stream)
    if st != attn.VGGT_OK:
        raise attn.VggtError(st, f"warm-up (detail {detail:#x})")

    events = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(a.steps)]
    barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index if dev.index is not None else 0) as clocks:
        for i in range(a.steps):
            step(q, k, v, events[i])
            if flush is not None:
                flush.zero_()
        torch.cuda.synchronize(dev)
    barrier()
    st, detail = attn.vggt_check(stream)
    if st != attn.VGGT_OK:
        raise attn.VggtError(st, f"timed region (detail {detail:#x})")

    per_op = {op: [] for op in ops}
    step_ms = []
    for ev in events:
        for j, op in enumerate(ops):
            per_op[op].append(ev[j].elapsed_time(ev[j + 1]))
        step_ms.append(ev[0].elapsed_time(ev[4]))
    local_total_ms = sum(step_ms)
    total_ms = max_over_ranks(local_total_ms, world, dev)
    ms_per_step = total_ms / a.steps

    # End to end through the public API with host buffers: every step copies
    # its inputs from pinned host memory, runs every op, and copies its three
    # outputs back.  The steps are pipelined as a serving loop would run them:
    # device buffers are double-buffered and the copies run on two copy
    # streams, so step i's H2D and step i-2's D2H overlap step i-1's compute.
    # The timed region spans the first H2D to the last D2H.
    e2e = None
    if not a.no_e2e:
        pin = [x.pin_memory() for x in (q_h, k_h, v_h)]
        outs_h = [torch.empty(q_h.shape, dtype=q_h.dtype).pin_memory() for _ in range(3)]
        ins_d = [[torch.empty_like(q) for _ in range(3)] for _ in range(2)]
        outs_d = [[torch.empty_like(q) for _ in range(3)] for _ in range(2)]
        h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev = lambda: torch.cuda.Event(enable_timing=False)
        h2d_done, comp_done, d2h_done = [None] * a.steps, [None] * a.steps, [None] * a.steps
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize(dev)
        t0.record(stream)
        h2d.wait_stream(stream)
        d2h.wait_stream(stream)
        for i in range(a.steps):
            b = i % 2
            if i >= 2:
                h2d.wait_event(comp_done[i - 2])  # ins_d[b] was last read by step i-2
            with torch.cuda.stream(h2d):
                for dst, src in zip(ins_d[b], pin):
                    dst.copy_(src, non_blocking=True)
            h2d_done[i] = ev()
            h2d_done[i].record(h2d)
            stream.wait_event(h2d_done[i])
            if i >= 2:
                stream.wait_event(d2h_done[i - 2])  # outs_d[b] was last read by step i-2's D2H
            step(*ins_d[b], outs=outs_d[b])
            if flush is not None:
                flush.zero_()
            comp_done[i] = ev()
            comp_done[i].record(stream)
            d2h.wait_event(comp_done[i])
            with torch.cuda.stream(d2h):
                for dst, src in zip(outs_h, outs_d[b]):
                    dst.copy_(src, non_blocking=True)
            d2h_done[i] = ev()
            d2h_done[i].record(d2h)
        stream.wait_event(d2h_done[-1])
        stream.wait_stream(h2d)
        t1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        e2e_ms = max_over_ranks(t0.elapsed_time(t1), world, dev) / a.steps
        e2e = {"value": round(world * step_flops / (e2e_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
               "ms_per_step": round(e2e_ms, 3), "h2d_bytes_per_step": int(in_bytes),
               "d2h_bytes_per_step": int(3 * q.numel() * 2),
               "pipeline": "double-buffered; H2D and D2H on two copy streams overlap the compute of "
                           "neighbouring steps; timed from the first H2D to the last D2H"}
        del ins_d, outs_d

    # Outside the step: register attention (VGGT-Omega) over this workload's
    # special tokens, timed after the step loop.
    extra = {}
    if wl.n_special > 0:
        o_reg = torch.empty_like(q)
        rows = wl.N * wl.n_special
        for _ in range(3):
            call(attn.vggt_attn_register(q, k, v, o_reg, None, wl, scale, stream), "register")
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(10)]
        for a_, b_ in evs:
            a_.record(stream)
            call(attn.vggt_attn_register(q, k, v, o_reg, None, wl, scale, stream), "register")
            b_.record(stream)
        torch.cuda.synchronize(dev)
        reg_ms = statistics.mean(a_.elapsed_time(b_) for a_, b_ in evs)
        reg_flop = 4 * rows * rows * wl.H * wl.d
        extra["register_attention"] = {
            "ms": round(reg_ms, 4), "tokens": rows, "flop": reg_flop,
            "tflops": round(reg_flop / (reg_ms * 1e-3) / 1e12, 2), "launches": 1,
            "global_over_register": round(statistics.mean(per_op["global"]) / reg_ms, 1)}

    # Outside the step: the fused QKV projection + 2D RoPE that would feed
    # this workload's attention (synthetic seeded weights, C = H * 64).
    if wl.H % 2 == 0:
        extra["qkv_rope"], extra["out_proj"] = time_projections(wl, dev, stream, call)
    else:
        extra["qkv_rope"] = extra["out_proj"] = {"skipped": f"{wl.H} heads per rank (needs an even count)"}

    # Outside the step: the attention layers of whole trunks through the
    # schedule driver (VGGT, AVGGT, VGGT-Omega; readings in schedules.py),
    # every layer on this workload's Q/K/V; one untimed run, then one timed
    # run each; above TRUNK_MAX_TOKENS, per layer kind, scaled by the layer
    # counts (see time_trunks).
    if not a.no_trunks:
        extra["trunks"] = time_trunks(wl, q, k, v, (o_frame, o_global), a.s_h, a.s_w, scale, stream, call)

    peaks, peaks_src = load_peaks()
    op_ms = {op: statistics.mean(v) for op, v in per_op.items()}
    glob_ms = max_over_ranks(op_ms["global"], world, dev)
    achieved = flops["global"] / (glob_ms * 1e-3) / 1e12
    per_op_out = {}
    for op in ("frame", "global", "sga"):
        ms = op_ms[op] + (op_ms["index"] if op == "sga" else 0.0)
        tf = flops[op] / (ms * 1e-3) / 1e12
        per_op_out[op] = {"ms": round(ms, 3), "tflops": round(tf, 1),
                          "frac_sustained": round(tf / peaks["bf16_tflops_sustained"], 4),
                          "frac_burst": round(tf / peaks["bf16_tflops"], 4)}
    per_op_out["sga"]["index_ms"] = round(op_ms["index"], 4)
    traffic = recorded_traffic()

    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        full, used, threads = oracle_sample_timing(wl, a.s_h, a.s_w, default_oracle_rows(wl), q_h, k_h, v_h)
        cpu_s = sum(full.values())
        cpu = {"value": round(step_flops / cpu_s / 1e12, 6), "unit": "TFLOP/s", "cores": threads,
               "kind": "oracle",
               "sample": (f"fp64 C oracle on {used['frame']}/{used['global']}/{used['sga']} seeded query rows "
                          f"(x all {wl.H} heads) of frame/global/SGA at {wl.name}; time extrapolated "
                          f"x S/rows to the whole step ({cpu_s:.0f} s)")}

    out = {
        "metric": METRIC,
        "value": round(world * step_flops / (ms_per_step * 1e-3) / 1e12, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": a.steps,
        "warmup": a.warmup,
        "ms_per_step": round(ms_per_step, 3),
        "higher_is_better": True,
        "scaling": "strong" if a.shard == "heads" else "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded, VGGT-shaped; correspondence-structured K)",
        "config": step_config(wl, a.s_h, a.s_w, n_kept, n_dropped, step_flops,
                              "flushed between steps" if flush is not None else l2_note(wl),
                              parallelism_note(a.shard, world, wl.H)),
        "per_op": per_op_out,
        "sga_speedup_vs_global": round(op_ms["global"] / (op_ms["sga"] + op_ms["index"]), 3),
        "roofline": {"bound": "tensor", "kernel": "attn_fwd_kernel (global attention)",
                     "achieved": round(achieved, 1), "peak": peaks["bf16_tflops_sustained"],
                     "unit": "TFLOP/s", "frac": round(achieved / peaks["bf16_tflops_sustained"], 4),
                     "peak_kind": f"bf16 dense, sustained ({peaks_src})",
                     "frac_of_burst": round(achieved / peaks["bf16_tflops"], 4),
                     "traffic": traffic},
        "extra_ops": extra,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": launches_per_step * a.steps,
        "clocks": clocks.summary(),
    }
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
    return out


# ------------------------------------------- query-row split across ranks

def run_queries_sga(a):
    """One AVGGT SGA layer with the frames of one scene split across the
    ranks and only the kept rows exchanged: each rank gathers the kept K/V
    rows and dropped-token sums of its own frames (vggt_sga_gather_partial),
    the ranks all-gather the kept rows and all-reduce the sums (NCCL), and
    each rank runs SGA for its own query rows (vggt_attn_sga_gathered).
    value = the layer's FLOP / the max over ranks of the layer time."""
    import datetime

    import torch

    from feed_forward_view_vggt_b200 import attn, synth

    rank, world, local = dist_env()
    if world > 1:
        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    wl = synth.WORKLOADS[a.config]
    flops, n_kept, n_dropped = workload_flops(wl, a.s_h, a.s_w)
    layer_flops = flops["sga"]
    q_h, k_h, v_h = synth.make_qkv(wl)  # every rank draws the scene and keeps its frames
    f0, f1 = frame_range(wl.N, world, rank)
    r0, r1 = f0 * wl.L, f1 * wl.L
    n_loc = r1 - r0
    q, k, v = (x[r0:r1].to(dev) for x in (q_h, k_h, v_h))
    counts = kept_counts(wl, world, a.s_h, a.s_w)
    x = KeptExchange(counts, wl.H, wl.d, dev)
    loc = attn.vggt_shape(max(f1 - f0, 1), wl.n_special, wl.h, wl.w, wl.H, wl.d)
    ws_bytes = attn.vggt_sga_partial_workspace_bytes(loc)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    means = torch.empty(2, wl.H * wl.d, dtype=torch.float32, device=dev)
    o = torch.empty_like(q)
    index = attn.SgaIndex(wl, a.s_h, a.s_w, device=dev)
    stream = torch.cuda.current_stream(dev)
    scale = 1.0 / math.sqrt(wl.d)
    ops = ("gather", "exchange", "sga")

    def call(status, what):
        if status != attn.VGGT_OK:
            raise attn.VggtError(status, what)

    def step(ev=None):
        rec = (lambda i: ev[i].record(stream)) if ev is not None else (lambda i: None)
        rec(0)
        if n_loc > 0:
            call(attn.vggt_sga_gather_partial(k, v, loc, a.s_h, a.s_w, x.local_k, x.local_v, x.sums, ws, ws_bytes,
                                              stream), "gather")
        else:
            x.sums.zero_()
        rec(1)
        kept_k, kept_v, sums = x.exchange()
        rec(2)
        if n_loc > 0:
            call(attn.vggt_attn_sga_gathered(q, r0, n_loc, k, v, kept_k, kept_v, sums, index.mult, means, o, None,
                                             wl, a.s_h, a.s_w, scale, stream), "sga")
        rec(3)

    def barrier():
        if world > 1:
            import torch.distributed as dist

            dist.barrier(device_ids=[local])

    for _ in range(max(a.warmup, 0)):
        step()
    st, detail = attn.vggt_check(stream)
    if st != attn.VGGT_OK:
        raise attn.VggtError(st, f"warm-up (detail {detail:#x})")
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(a.steps)]
    barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index if dev.index is not None else 0) as clocks:
        for i in range(a.steps):
            step(events[i])
        torch.cuda.synchronize(dev)
    barrier()
    st, detail = attn.vggt_check(stream)
    if st != attn.VGGT_OK:
        raise attn.VggtError(st, f"timed region (detail {detail:#x})")
    per_op = {op: statistics.mean(ev[j].elapsed_time(ev[j + 1]) for ev in events) for j, op in enumerate(ops)}
    local_ms = sum(ev[0].elapsed_time(ev[3]) for ev in events)
    ms_per_step = max_over_ranks(local_ms, world, dev) / a.steps
    launches = (2 if n_loc > 0 else 0) + ((2 if n_dropped > 0 else 1) if n_loc > 0 else 0)
    out = {
        "metric": METRIC,
        "value": round(layer_flops / (ms_per_step * 1e-3) / 1e12, 2),
        "unit": "TFLOP/s", "n_gpus": world, "steps": a.steps, "warmup": a.warmup,
        "ms_per_step": round(ms_per_step, 3), "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded, VGGT-shaped; correspondence-structured K)",
        "config": step_config(wl, a.s_h, a.s_w, n_kept, n_dropped, layer_flops, l2_note(wl),
                              f"one SGA layer; query rows split over {world} ranks by frames; the kept K/V rows "
                              f"all-gathered and the dropped-token sums all-reduced every step (NCCL)"),
        "per_op_rank0_ms": {op: round(v, 3) for op, v in per_op.items()},
        "exchange_bytes_per_rank": 2 * x.gathered_k.numel() * 2 + x.sums.numel() * 4,
        "roofline": None, "cpu_baseline": None,
        "e2e": None, "e2e_note": "not measured in the query-split mode",
        "gpu_launches": launches * a.steps,
        "clocks": clocks.summary(),
    }
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


def run_queries(a):
    """The step with the frames of one scene split across the ranks: every
    step all-gathers K and V (NCCL), then each rank runs frame attention on
    its own frames and global attention and SGA for its own query rows
    against all keys.  value = the whole problem's FLOP / the max over ranks
    of the step time (strong scaling)."""
    import datetime

    import torch

    from feed_forward_view_vggt_b200 import attn, synth

    rank, world, local = dist_env()
    if world > 1:
        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    wl = synth.WORKLOADS[a.config]
    flops, n_kept, n_dropped = workload_flops(wl, a.s_h, a.s_w)
    step_flops = sum(flops.values())
    q_h, k_h, v_h = synth.make_qkv(wl)  # every rank draws the scene and keeps its frames
    f0, f1 = frame_range(wl.N, world, rank)
    r0, r1 = f0 * wl.L, f1 * wl.L
    n_loc = r1 - r0
    xk = FrameExchange(wl.N, wl.L, world, torch.empty(1, wl.H, wl.d, dtype=torch.bfloat16, device=dev))
    xv = FrameExchange(wl.N, wl.L, world, torch.empty(1, wl.H, wl.d, dtype=torch.bfloat16, device=dev))
    xk.local[:n_loc].copy_(k_h[r0:r1])
    xv.local[:n_loc].copy_(v_h[r0:r1])
    q = q_h[r0:r1].to(dev)
    o_f, o_g, o_s = (torch.empty_like(q) for _ in range(3))
    loc_wl = synth.Workload(wl.name, max(f1 - f0, 1), wl.h, wl.w, wl.H, wl.seed, wl.structure, wl.sga_strides,
                            wl.n_special, wl.d)
    index = attn.SgaIndex(wl, a.s_h, a.s_w, device=dev)
    stream = torch.cuda.current_stream(dev)
    scale = 1.0 / math.sqrt(wl.d)
    ops = ("exchange", "frame", "global", "index", "sga")

    def call(status, what):
        if status != attn.VGGT_OK:
            raise attn.VggtError(status, what)

    def step(ev=None):
        rec = (lambda i: ev[i].record(stream)) if ev is not None else (lambda i: None)
        rec(0)
        k_all, v_all = xk.exchange(), xv.exchange()
        rec(1)
        if n_loc > 0:
            call(attn.vggt_attn_frame(q, xk.local, xv.local, o_f, None, loc_wl, scale, stream), "frame")
        rec(2)
        if n_loc > 0:
            call(attn.vggt_attn_global_rows(q, n_loc, k_all, v_all, o_g, None, wl, scale, stream), "global")
        rec(3)
        call(attn.vggt_sga_build_index(wl, a.s_h, a.s_w, index.kept_idx, index.mult, stream), "index")
        rec(4)
        if n_loc > 0:
            call(attn.vggt_attn_sga_rows(q, r0, n_loc, k_all, v_all, o_s, None, wl, a.s_h, a.s_w, index.kept_idx,
                                         index.mult, index.workspace, index.workspace_bytes, scale, stream), "sga")
        rec(5)

    def barrier():
        if world > 1:
            import torch.distributed as dist

            dist.barrier(device_ids=[local])

    for _ in range(max(a.warmup, 0)):
        step()
    st, detail = attn.vggt_check(stream)
    if st != attn.VGGT_OK:
        raise attn.VggtError(st, f"warm-up (detail {detail:#x})")
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(a.steps)]
    barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index if dev.index is not None else 0) as clocks:
        for i in range(a.steps):
            step(events[i])
        torch.cuda.synchronize(dev)
    barrier()
    st, detail = attn.vggt_check(stream)
    if st != attn.VGGT_OK:
        raise attn.VggtError(st, f"timed region (detail {detail:#x})")
    per_op = {op: statistics.mean(ev[j].elapsed_time(ev[j + 1]) for ev in events) for j, op in enumerate(ops)}
    local_ms = sum(ev[0].elapsed_time(ev[5]) for ev in events)
    ms_per_step = max_over_ranks(local_ms, world, dev) / a.steps
    peaks, peaks_src = load_peaks()
    launches = (1 if n_loc > 0 else 0) * 2 + 1 + ((2 + (1 if n_dropped > 0 else 0)) if n_loc > 0 else 0)
    out = {
        "metric": METRIC,
        "value": round(step_flops / (ms_per_step * 1e-3) / 1e12, 2),
        "unit": "TFLOP/s", "n_gpus": world, "steps": a.steps, "warmup": a.warmup,
        "ms_per_step": round(ms_per_step, 3), "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded, VGGT-shaped; correspondence-structured K)",
        "config": step_config(wl, a.s_h, a.s_w, n_kept, n_dropped, step_flops, l2_note(wl),
                              f"query rows split over {world} ranks by frames; K and V all-gathered every step "
                              f"(NCCL)"),
        "per_op_rank0_ms": {op: round(v, 3) for op, v in per_op.items()},
        "exchange_bytes_per_rank": 2 * xk.gathered.numel() * 2,
        "roofline": None, "cpu_baseline": None,
        "e2e": None, "e2e_note": "not measured in the query-split mode",
        "gpu_launches": launches * a.steps,
        "clocks": clocks.summary(),
    }
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
    return out


# ------------------------------------------------------ resumable op sweep

def sweep_ops(wl):
    """The ops a sweep times for one workload: frame, global and SGA at each
    of the workload's strides."""
    return ["frame", "global"] + ["sga%dx%d" % st for st in wl.sga_strides]


def load_done(path):
    """(workload, op) pairs already recorded in a results file; a torn last
    line (an interrupted write) is ignored."""
    done = set()
    try:
        with open(path) as f:
            for ln in f:
                try:
                    rec = json.loads(ln)
                except ValueError:
                    continue
                done.add((rec["workload"], rec["op"]))
    except OSError:
        pass
    return done


def append_result(path, rec):
    """Appends one record as one line and makes it durable before returning;
    a torn last line (no newline) is closed off first, so it stays one bad
    line instead of swallowing this record."""
    lead = ""
    try:
        with open(path, "rb") as f:
            f.seek(0, os.SEEK_END)
            if f.tell() > 0:
                f.seek(-1, os.SEEK_END)
                lead = "" if f.read(1) == b"\n" else "\n"
    except OSError:
        pass
    with open(path, "a") as f:
        f.write(lead + json.dumps(rec) + "\n")
        f.flush()
        os.fsync(f.fileno())


def run_sweep(a, measure=None):
    """Times every op of every workload in a.sweep on its own, appending one
    line per (workload, op) to a.results as soon as it is measured, and skips
    the pairs the file already holds -- an interrupted sweep (N = 800 global
    attention takes seconds per run) resumes where it stopped.  `measure(wl,
    op)` -> dict (defaults to CUDA-event timing on this GPU)."""
    from feed_forward_view_vggt_b200 import synth

    done = load_done(a.results)
    if measure is None:
        measure = GpuOpTimer(a)
    new = []
    for name in [c for c in a.sweep.split(",") if c]:
        wl = synth.WORKLOADS[name]
        for op in sweep_ops(wl):
            if (name, op) in done:
                continue
            rec = {"workload": name, "op": op, **measure(wl, op)}
            append_result(a.results, rec)
            done.add((name, op))
            new.append(rec)
    return new


class GpuOpTimer:
    """Per-op timing for the sweep: W untimed runs, then the median of K
    CUDA-event-timed runs of one op on the workload's seeded inputs (kept on
    the device while consecutive ops share a workload)."""

    def __init__(self, a):
        self.a = a
        self.wl = None

    def _inputs(self, wl):
        import torch

        from feed_forward_view_vggt_b200 import synth

        if self.wl is not wl:
            self.wl = None
            self.q = self.k = self.v = self.o = None
            torch.cuda.empty_cache()
            self.q, self.k, self.v = (x.cuda() for x in synth.make_qkv(wl))
            self.o = torch.empty_like(self.q)
            self.wl = wl
        return self.q, self.k, self.v, self.o

    def __call__(self, wl, op):
        import torch

        from feed_forward_view_vggt_b200 import accounting as acc
        from feed_forward_view_vggt_b200 import attn

        q, k, v, o = self._inputs(wl)
        scale = 1.0 / math.sqrt(wl.d)
        if op.startswith("sga"):
            s_h, s_w = (int(x) for x in op[3:].split("x"))
            idx = attn.SgaIndex(wl, s_h, s_w)
            nk, nd = acc.sga_counts(wl.N, wl.n_special, wl.h, wl.w, s_h, s_w)
            flop = acc.flops_sga(wl.S, nk, nd, wl.H, wl.d)

            def run():
                attn._raise(attn.vggt_sga_build_index(wl, s_h, s_w, idx.kept_idx, idx.mult), op)
                attn._raise(attn.vggt_attn_sga(q, k, v, o, None, wl, s_h, s_w, idx.kept_idx, idx.mult,
                                               idx.workspace, idx.workspace_bytes, scale), op)
        else:
            fn = attn.vggt_attn_frame if op == "frame" else attn.vggt_attn_global
            flop = (acc.flops_frame(wl.N, wl.L, wl.H, wl.d) if op == "frame" else acc.flops_global(wl.S, wl.H, wl.d))

            def run():
                attn._raise(fn(q, k, v, o, None, wl, scale), op)

        for _ in range(max(self.a.warmup, 0)):
            run()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(max(self.a.steps, 1))]
        for e0, e1 in evs:
            e0.record()
            run()
            e1.record()
        torch.cuda.synchronize()
        st, detail = attn.vggt_check()
        if st != attn.VGGT_OK:
            raise attn.VggtError(st, f"{op} (detail {detail:#x})")
        ms = statistics.median(e0.elapsed_time(e1) for e0, e1 in evs)
        peaks, src = load_peaks()
        tf = flop / (ms * 1e-3) / 1e12
        return {"ms": round(ms, 4), "reps": len(evs), "flop": flop, "tflops": round(tf, 1),
                "frac_sustained": round(tf / peaks["bf16_tflops_sustained"], 4),
                "frac_burst": round(tf / peaks["bf16_tflops"], 4), "peaks": src,
                "includes": "index build + gather/mean-fill + attention" if op.startswith("sga") else "one launch"}


# ---------------------------------------------------------- reference arm

def run_reference(a):
    """The fp64 CPU oracle timed as the reference arm, on rank 0 only."""
    rank, world, _ = dist_env()
    if rank != 0:
        return None
    from feed_forward_view_vggt_b200 import synth

    wl = synth.WORKLOADS[a.config]
    flops, n_kept, n_dropped = workload_flops(wl, a.s_h, a.s_w)
    step_flops = sum(flops.values())
    q, k, v = synth.make_qkv(wl)
    base_rows = default_oracle_rows(wl)
    # each step: a bounded sample (a quarter of the CPU-baseline sample)
    rows = {op: max(8, n // 4) if wl.S > 6000 else n for op, n in base_rows.items()}
    for _ in range(max(a.warmup, 0)):
        oracle_sample_timing(wl, a.s_h, a.s_w, {op: 8 for op in rows}, q, k, v)
    per_step = []
    used = threads = None
    measured = {}
    for _ in range(a.steps):
        full, used, threads = oracle_sample_timing(wl, a.s_h, a.s_w, rows, q, k, v, measured=measured)
        per_step.append(sum(full.values()))
    sec = statistics.mean(per_step)
    value = step_flops / sec / 1e12
    sample = (f"fp64 C oracle on {used['frame']}/{used['global']}/{used['sga']} seeded query rows (x all "
              f"{wl.H} heads) of frame/global/SGA per step; time extrapolated x S/rows to the whole step")
    out = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
        "n_gpus": world, "steps": a.steps, "warmup": a.warmup, "ms_per_step": round(sec * 1e3, 1),
        # ms_per_step is the sampled rows' time scaled by S / rows, not a
        # measured full step; the seconds actually measured are given too.
        "ms_per_step_extrapolated": any(n < wl.S for n in used.values()),
        "measured_s": {op: round(t, 3) for op, t in measured.items()},
        "measured_s_total": round(sum(measured.values()), 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded, VGGT-shaped; correspondence-structured K)",
        # the same config object as the GPU arm on this workload
        "config": step_config(wl, a.s_h, a.s_w, n_kept, n_dropped, step_flops, l2_note(wl),
                              parallelism_note("replicas", world, wl.H)),
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(out), flush=True)
    return out


def main(argv=None):
    a = parse_args(argv)
    if a.warmup < 3:
        print("warning: fewer than 3 warm-up steps; the number is not a valid bench value", file=sys.stderr)
    if a.impl == "reference":
        return run_reference(a)
    if a.sweep:
        for rec in run_sweep(a):
            print(json.dumps(rec), flush=True)
        return None
    if a.shard == "queries":
        return run_queries_sga(a) if a.layer == "sga" else run_queries(a)
    return run_ours(a)


if __name__ == "__main__":
    main()
