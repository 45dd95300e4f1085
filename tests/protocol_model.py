"""Discrete-event model of the attention kernel's synchronisation protocol,
for race detection on the CPU.

It models the roles of one CTA and their barriers as the kernel runs them:
* the TMA producer;
* the single-thread UMMA issuer: three rotating score buffers, S(k + 3)
  after PV(k) has completed, commits;
* two softmax warpgroups of four independent warps each;
* an asynchronous tensor pipe.

The model is conservative: a UMMA group or a TMA copy may touch its operands
at any time between its issue and its completion, and groups may complete
in any order.  A commit arrives only once every group issued before it has
completed, which is what tcgen05.commit guarantees.  The one ordering the
hardware does guarantee between UMMAs is kept: UMMAs issued by one thread
into the same accumulator with the same shape run in issue order (the PV
products of a warpgroup accumulating into its O), so those do not race.

Checks, under random timings (including warps of a warpgroup drifting apart
by whole steps):
* every mbarrier wait is by parity; when it returns, the phase the waiter
  meant must really have completed (no parity aliasing), and no waiter may
  start more than one phase behind (a missed phase);
* no two accesses to the same TMEM or shared-memory region overlap in time
  when one of them writes;
* every role finishes (no deadlock).

Work items are pairs of query tiles.  A pair inside one unit shares one
K/V stream (one ring stage per key tile, released by warpgroup 1's UMMAs);
a "split" pair straddling two units streams K/V per warpgroup (one stage
per step, each released by its own reader).  `splits` gives the flag of
every item.

Mutations reproduce earlier or plausible designs that have races, so the
tests can show the checker catches them:
* "single_p_ready": one P-ready barrier per warpgroup;
* "epilogue_o_done": the epilogue waits on o_done by parity instead of the
  per-item barrier;
* "split_shared_release": split items release K/V stages as a shared
  stream would (only after warpgroup 1), so warpgroup 0's stage is reused
  too early or the ring's phases slip;
* "defer_after_ready": the deferred epilogue reads O after the P-ready
  arrive, when the next item's first PV may already be overwriting it.
"""
from __future__ import annotations

import heapq
import random
from dataclasses import dataclass, field

STAGES = 4
BUFS = 3
EPI_WARPS = 8  # GEMM epilogue warps per CTA: two per TMEM lane quarter, each a share of the columns
P_HALF = 1  # the score-buffer half P is written over (split S)


class ProtocolError(AssertionError):
    pass


class Barrier:
    def __init__(self, name: str, count: int):
        self.name = name
        self.count = count
        self.pending = count
        self.completed = 0  # phases completed so far

    def arrive(self):
        self.pending -= 1
        if self.pending < 0:
            raise ProtocolError(f"{self.name}: more arrivals than expected")
        if self.pending == 0:
            self.completed += 1
            self.pending = self.count


@dataclass
class Access:
    resource: tuple
    write: bool
    t0: float
    t1: float
    who: str


@dataclass
class Sim:
    n_items: int
    n_kt: int
    rng: random.Random
    mutation: str = ""
    splits: tuple = ()
    # False (the shipped kernel): the whole S(k + 3) after PV(k) completes, P
    # in score columns 0..63.  True (an alternative measured slower on the
    # GPU): S issued as two halves, the first (columns 0..63) queued right
    # behind PV(k), the second after PV(k) completes, P in columns 64..127.
    split_s: bool = False
    # The general kernel (frame and register launches): the epilogue of
    # item i (wait for its last PV, read O) runs inside item i + 1's first
    # step, after that step's P is written and before its P-ready arrive.
    defer_epilogue: bool = False
    now: float = 0.0
    seq: int = 0
    queue: list = field(default_factory=list)
    accesses: list = field(default_factory=list)
    mma_done: list = field(default_factory=list)  # completion times of issued UMMA groups

    def __post_init__(self):
        B = Barrier
        if not self.splits:
            self.splits = (False,) * self.n_items
        self.q_full = [B(f"q_full{i}", 1) for i in range(2)]
        self.q_empty = [B(f"q_empty{i}", 1) for i in range(2)]
        self.k_full = [B(f"k_full{i}", 1) for i in range(STAGES)]
        self.k_empty = [B(f"k_empty{i}", 1) for i in range(STAGES)]
        self.v_full = [B(f"v_full{i}", 1) for i in range(STAGES)]
        self.v_empty = [B(f"v_empty{i}", 1) for i in range(STAGES)]
        self.s_full = [B(f"s_full{i}", 1) for i in range(BUFS)]
        n_p = 1 if self.mutation == "single_p_ready" else 2
        self.p_ready = [[B(f"p_ready{w}.{i}", 4) for i in range(n_p)] for w in range(2)]
        self.o_done = [B(f"o_done{w}", 1) for w in range(2)]
        self.o_final = [B(f"o_final{w}", 1) for w in range(2)]

    # ---------------------------------------------------------- event loop
    def at(self, t, fn):
        self.seq += 1
        heapq.heappush(self.queue, (t, self.seq, fn))

    def touch(self, resource, write, t0, t1, who):
        self.accesses.append(Access(resource, write, t0, t1, who))

    def commit(self, bar):
        t = max([self.now] + self.mma_done) + self.rng.uniform(0.0, 0.2)
        self.at(t, bar.arrive)

    def mma(self, reads, writes, who):
        t1 = self.now + self.rng.uniform(0.5, 3.0)  # any order of completion
        for r in reads:
            self.touch(r, False, self.now, t1, who)
        for w in writes:
            self.touch(w, True, self.now, t1, who)
        self.mma_done.append(t1)

    def tma(self, bar, writes, who):
        t1 = self.now + self.rng.uniform(0.5, 4.0)
        for w in writes:
            self.touch(w, True, self.now, t1, who)
        self.at(t1, bar.arrive)

    def run(self, actors, horizon=5000.0):
        waiting = {}
        for name, gen in actors.items():
            self.at(0.0, ("step", name))
        gens = dict(actors)
        done = set()
        while self.queue:
            t, _, ev = heapq.heappop(self.queue)
            if t > horizon:
                break
            self.now = t
            if callable(ev):
                ev()
                continue
            _, name = ev
            gen = gens[name]
            try:
                cmd = waiting.pop(name, None) or next(gen)
                while True:
                    if cmd[0] == "delay":
                        self.at(self.now + cmd[1], ("step", name))
                        break
                    if cmd[0] == "wait":
                        _, bar, n = cmd
                        if bar.completed > n + 1 or bar.completed < n - 1:
                            raise ProtocolError(f"{name}: waits for phase {n} of {bar.name}, which has "
                                                f"completed {bar.completed} phases (ambiguous or missed)")
                        if (bar.completed & 1) != (n & 1):  # try_wait.parity(n & 1) succeeds
                            if bar.completed != n + 1:
                                raise ProtocolError(f"{name}: parity wait for phase {n} of {bar.name} passed "
                                                    f"with {bar.completed} phases completed")
                            cmd = next(gen)
                            continue
                        waiting[name] = cmd
                        self.at(self.now + 0.05, ("step", name))
                        break
                    raise ProtocolError(f"unknown command {cmd}")
            except StopIteration:
                done.add(name)
        if len(done) != len(gens):
            raise ProtocolError(f"deadlock: {sorted(set(gens) - done)} never finished")
        self.check_accesses()

    def check_accesses(self):
        by_res = {}
        for a in self.accesses:
            by_res.setdefault(a.resource, []).append(a)
        for res, acc in by_res.items():
            acc.sort(key=lambda a: a.t0)
            for i, a in enumerate(acc):
                for b in acc[i + 1:]:
                    if b.t0 > a.t1:
                        break
                    same_acc = res[0] == "O" and a.who.startswith("PV") and b.who.startswith("PV")
                    if (a.write or b.write) and a.who != b.who and not same_acc:
                        raise ProtocolError(f"race on {res}: {a.who} [{a.t0:.2f}, {a.t1:.2f}] vs "
                                            f"{b.who} [{b.t0:.2f}, {b.t1:.2f}]")


# ------------------------------------------------------------------ roles

def producer(sim: Sim):
    u = 0
    for it in range(sim.n_items):
        qb = it & 1
        yield ("wait", sim.q_empty[qb], (it >> 1) - 1) if it >= 2 else ("delay", 0.0)
        sim.tma(sim.q_full[qb], [("Q", qb, 0), ("Q", qb, 1)], f"tmaQ{it}")
        for j in range(sim.n_kt):
            for _ in range(2 if sim.splits[it] else 1):
                st, n = u % STAGES, u // STAGES
                if n >= 1:
                    yield ("wait", sim.k_empty[st], n - 1)
                sim.tma(sim.k_full[st], [("K", st)], f"tmaK{u}")
                if n >= 1:
                    yield ("wait", sim.v_empty[st], n - 1)
                sim.tma(sim.v_full[st], [("V", st)], f"tmaV{u}")
                u += 1
            yield ("delay", sim.rng.uniform(0.0, 0.3))


def issuer(sim: Sim):
    T = sim.n_items * sim.n_kt
    steps = 2 * T
    # ring slot of every step: a shared stream advances after warpgroup 1's
    # step, a split item after every step
    slot, u = [], 0
    for k in range(steps):
        slot.append(u)
        if sim.splits[(k >> 1) // sim.n_kt] or (k & 1):
            u += 1

    def pos(k):
        c = k >> 1
        return k & 1, c, c // sim.n_kt, c % sim.n_kt, slot[k] % STAGES, slot[k] // STAGES, k % BUFS

    def own_stage(it, wg):
        # the step is a reader that waits for and releases its stage
        if sim.splits[it] and sim.mutation != "split_shared_release":
            return True
        return None

    def s_inputs(k):
        wg, c, it, j, st, ph, buf = pos(k)
        if wg == 0 or own_stage(it, wg):
            if wg == 0 and j == 0:
                yield ("wait", sim.q_full[it & 1], it >> 1)
            yield ("wait", sim.k_full[st], ph)

    def s_half(k, half):
        wg, c, it, j, st, ph, buf = pos(k)
        sim.mma([("K", st), ("Q", it & 1, wg)], [("S", buf, half, w) for w in range(4)], f"S{k}.{half}")

    def s_commit(k):
        wg, c, it, j, st, ph, buf = pos(k)
        sim.commit(sim.s_full[buf])
        if wg == 1 or own_stage(it, wg):
            sim.commit(sim.k_empty[st])
        if wg == 1 and j == sim.n_kt - 1:
            sim.commit(sim.q_empty[it & 1])

    def issue_s(k):
        yield from s_inputs(k)
        s_half(k, 0)
        s_half(k, 1)
        s_commit(k)

    for k in range(min(BUFS, steps)):
        yield from issue_s(k)
    for k in range(steps):
        wg, c, it, j, st, ph, buf = pos(k)
        own = own_stage(it, wg)
        if wg == 0 or own:
            yield ("wait", sim.v_full[st], ph)
        if sim.mutation == "single_p_ready":
            yield ("wait", sim.p_ready[wg][0], c)
        else:
            yield ("wait", sim.p_ready[wg][c & 1], c >> 1)
        sim.mma([("V", st)] + [("S", buf, P_HALF if sim.split_s else 0, w) for w in range(4)],
                [("O", wg, w) for w in range(4)], f"PV{k}")
        sim.commit(sim.o_done[wg])
        if j == sim.n_kt - 1:
            sim.commit(sim.o_final[wg])
        if wg == 1 or own:
            sim.commit(sim.v_empty[st])
        if k + BUFS < steps:
            if sim.split_s:
                # S(k + 3)'s first half does not touch P: it goes in now
                yield from s_inputs(k + BUFS)
                s_half(k + BUFS, 0)
                yield ("wait", sim.o_done[wg], c)
                s_half(k + BUFS, 1)
                s_commit(k + BUFS)
            else:
                yield ("wait", sim.o_done[wg], c)
                yield from issue_s(k + BUFS)
        yield ("delay", sim.rng.uniform(0.0, 0.2))


def softmax_warp(sim: Sim, wg: int, w: int, drift: float):
    who = f"wg{wg}.w{w}"
    c = o_seen = 0
    for it in range(sim.n_items):
        # per-item prologue (the SGA loads): occasionally long, per warp
        yield ("delay", sim.rng.uniform(0.0, drift if sim.rng.random() < 0.3 else 0.2))
        for j in range(sim.n_kt):
            k = 2 * c + wg
            buf = k % BUFS
            yield ("wait", sim.s_full[buf], k // BUFS)
            sim.touch(("S", buf, 0, w), False, sim.now, sim.now, who)
            sim.touch(("S", buf, 1, w), False, sim.now, sim.now, who)
            yield ("delay", sim.rng.uniform(0.1, 1.0))
            if j > 0 and sim.rng.random() < 0.3:  # lazy rescale of O
                if o_seen < c:
                    yield ("wait", sim.o_done[wg], c - 1)
                    o_seen = c
                sim.touch(("O", wg, w), True, sim.now, sim.now, who)
            yield ("delay", sim.rng.uniform(0.2, 2.0))
            sim.touch(("S", buf, P_HALF if sim.split_s else 0, w), True, sim.now, sim.now, who)  # P over S
            deferred = sim.defer_epilogue and j == 0 and it > 0
            if deferred and sim.mutation != "defer_after_ready":
                # the previous item's epilogue, before this step's P-ready
                yield ("wait", sim.o_final[wg], it - 1)
                o_seen = c
                sim.touch(("O", wg, w), False, sim.now, sim.now, who)
            if sim.mutation == "single_p_ready":
                sim.p_ready[wg][0].arrive()
            else:
                sim.p_ready[wg][c & 1].arrive()
            if deferred and sim.mutation == "defer_after_ready":
                yield ("wait", sim.o_final[wg], it - 1)
                o_seen = c
                yield ("delay", sim.rng.uniform(0.0, 1.0))
                sim.touch(("O", wg, w), False, sim.now, sim.now, who)
            c += 1
        if sim.defer_epilogue:
            continue
        if sim.mutation == "epilogue_o_done":
            if o_seen < c:
                yield ("wait", sim.o_done[wg], c - 1)
        else:
            yield ("wait", sim.o_final[wg], it)
        o_seen = c
        sim.touch(("O", wg, w), False, sim.now, sim.now, who)
    if sim.defer_epilogue and sim.n_items > 0:
        yield ("wait", sim.o_final[wg], sim.n_items - 1)
        sim.touch(("O", wg, w), False, sim.now, sim.now, who)


def simulate(seed: int, n_items: int = 4, n_kt: int = 3, drift: float = 6.0, mutation: str = "",
             splits=(), split_s: bool = False, defer_epilogue: bool = False):
    sim = Sim(n_items, n_kt, random.Random(seed), mutation, tuple(splits), split_s, defer_epilogue)
    actors = {"producer": producer(sim), "issuer": issuer(sim)}
    for wg in range(2):
        for w in range(4):
            actors[f"wg{wg}.w{w}"] = softmax_warp(sim, wg, w, drift)
    sim.run(actors)
    return sim


# ------------------------------------------- the QKV-projection GEMM kernel
#
# Roles: a TMA producer filling a 4-stage ring with an X and a W tile per K
# chunk; one issuer thread running a tile's UMMAs into one of two TMEM
# accumulators (acc_empty before, acc_full after); four epilogue warps, each
# reading its quarter of the accumulator rows, then arriving on acc_empty.
# Mutation "no_acc_empty": the issuer never waits for the epilogue.

class GemmSim(Sim):
    def __post_init__(self):
        B = Barrier
        self.full = [B(f"full{i}", 1) for i in range(STAGES)]
        self.empty = [B(f"empty{i}", 1) for i in range(STAGES)]
        self.acc_full = [B(f"acc_full{i}", 1) for i in range(2)]
        self.acc_empty = [B(f"acc_empty{i}", EPI_WARPS) for i in range(2)]


def gemm_producer(sim: GemmSim, n_tiles: int, k_chunks: int):
    u = 0
    for _ in range(n_tiles):
        for _ in range(k_chunks):
            st, n = u % STAGES, u // STAGES
            if n >= 1:
                yield ("wait", sim.empty[st], n - 1)
            sim.tma(sim.full[st], [("A", st), ("B", st)], f"tma{u}")
            u += 1
            yield ("delay", sim.rng.uniform(0.0, 0.3))


def gemm_issuer(sim: GemmSim, n_tiles: int, k_chunks: int):
    u = 0
    for tl in range(n_tiles):
        b, use = tl & 1, tl >> 1
        if use >= 1 and sim.mutation != "no_acc_empty":
            yield ("wait", sim.acc_empty[b], use - 1)
        for kc in range(k_chunks):
            st, n = u % STAGES, u // STAGES
            yield ("wait", sim.full[st], n)
            # the K chunks of one tile accumulate into one accumulator: in order
            sim.mma([("A", st), ("B", st)], [("ACC", b, w) for w in range(EPI_WARPS)], f"T{tl}")
            sim.commit(sim.empty[st])
            u += 1
        sim.commit(sim.acc_full[b])
        yield ("delay", sim.rng.uniform(0.0, 0.2))


def gemm_epilogue(sim: GemmSim, q: int, n_tiles: int, drift: float):
    """Epilogue warp q: its lane quarter's rows, its share of the columns."""
    who = f"epi{q}"
    for tl in range(n_tiles):
        b, use = tl & 1, tl >> 1
        yield ("wait", sim.acc_full[b], use)
        yield ("delay", sim.rng.uniform(0.0, drift if sim.rng.random() < 0.3 else 0.5))
        sim.touch(("ACC", b, q), False, sim.now, sim.now, who)
        sim.acc_empty[b].arrive()


def simulate_gemm(seed: int, n_tiles: int = 6, k_chunks: int = 5, drift: float = 8.0, mutation: str = ""):
    sim = GemmSim(0, 0, random.Random(seed), mutation)
    actors = {"producer": gemm_producer(sim, n_tiles, k_chunks), "issuer": gemm_issuer(sim, n_tiles, k_chunks)}
    for q in range(EPI_WARPS):
        actors[f"epi{q}"] = gemm_epilogue(sim, q, n_tiles, drift)
    sim.run(actors)
    return sim


# ------------------------------------------------------------ the CTA pair
# The GEMM's pair form: two CTAs (ranks 0 and 1) on two SMs, five stages.
# Each CTA's producer waits on its own empty barrier and loads its A and B
# halves; both copies complete on the leader's full barrier, which also
# takes the leader's expect-tx arrival (modelled as five arrivals: the
# expect-tx and the four copies' byte counts; the phase cannot complete
# before all five).  The leader's single issuer
# reads both CTAs' stages, writes both CTAs' accumulators, and its commits
# arrive on the barrier at the same offset in both CTAs (multicast).  The
# epilogue warps of both CTAs (EPI_WARPS each) read their own CTA's
# accumulator regions and arrive on the leader's acc_empty.
#
# Mutations:
# * "pair_follower_expects": the follower also arrives (expect-tx) on the
#   leader's full barrier;
# * "pair_commit_leader_only": stage releases arrive on the leader's empty
#   barrier only, so the follower's producer never sees its stage free;
# * "pair_local_release": the follower's epilogue releases the accumulator
#   on its own acc_empty instead of the leader's.

PAIR_STAGES = 5


class GemmPairSim(Sim):
    def __post_init__(self):
        B = Barrier
        self.full = [[B(f"full{i}.r{r}", 5) for i in range(PAIR_STAGES)] for r in range(2)]
        self.empty = [[B(f"empty{i}.r{r}", 1) for i in range(PAIR_STAGES)] for r in range(2)]
        self.acc_full = [[B(f"acc_full{i}.r{r}", 1) for i in range(2)] for r in range(2)]
        self.acc_empty = [[B(f"acc_empty{i}.r{r}", 2 * EPI_WARPS) for i in range(2)] for r in range(2)]

    def commit_pair(self, bars):
        targets = bars[:1] if self.mutation == "pair_commit_leader_only" and bars[0].name.startswith("empty") \
            else bars
        for bar in targets:
            self.commit(bar)


def pair_producer(sim: GemmPairSim, rank: int, n_tiles: int, k_chunks: int):
    u = 0
    for _ in range(n_tiles):
        for _ in range(k_chunks):
            st, n = u % PAIR_STAGES, u // PAIR_STAGES
            if n >= 1:
                yield ("wait", sim.empty[rank][st], n - 1)
            if rank == 0 or sim.mutation == "pair_follower_expects":
                sim.full[0][st].arrive()  # expect-tx on the leader's barrier
            sim.tma(sim.full[0][st], [("A", rank, st)], f"tma{u}.a.r{rank}")
            sim.tma(sim.full[0][st], [("B", rank, st)], f"tma{u}.b.r{rank}")
            u += 1
            yield ("delay", sim.rng.uniform(0.0, 0.3))


def pair_issuer(sim: GemmPairSim, n_tiles: int, k_chunks: int):
    u = 0
    for tl in range(n_tiles):
        b, use = tl & 1, tl >> 1
        if use >= 1:
            yield ("wait", sim.acc_empty[0][b], use - 1)
        for kc in range(k_chunks):
            st, n = u % PAIR_STAGES, u // PAIR_STAGES
            yield ("wait", sim.full[0][st], n)
            sim.mma([("A", r, st) for r in range(2)] + [("B", r, st) for r in range(2)],
                    [("ACC", r, b, w) for r in range(2) for w in range(EPI_WARPS)], f"T{tl}")
            sim.commit_pair([sim.empty[0][st], sim.empty[1][st]])
            u += 1
        sim.commit_pair([sim.acc_full[0][b], sim.acc_full[1][b]])
        yield ("delay", sim.rng.uniform(0.0, 0.2))


def pair_epilogue(sim: GemmPairSim, rank: int, q: int, n_tiles: int, drift: float):
    who = f"epi{q}.r{rank}"
    for tl in range(n_tiles):
        b, use = tl & 1, tl >> 1
        yield ("wait", sim.acc_full[rank][b], use)
        yield ("delay", sim.rng.uniform(0.0, drift if sim.rng.random() < 0.3 else 0.5))
        sim.touch(("ACC", rank, b, q), False, sim.now, sim.now, who)
        target = rank if sim.mutation == "pair_local_release" else 0
        sim.acc_empty[target][b].arrive()


def simulate_gemm_pair(seed: int, n_tiles: int = 6, k_chunks: int = 5, drift: float = 8.0, mutation: str = ""):
    sim = GemmPairSim(0, 0, random.Random(seed), mutation)
    actors = {"issuer": pair_issuer(sim, n_tiles, k_chunks)}
    for r in range(2):
        actors[f"producer.r{r}"] = pair_producer(sim, r, n_tiles, k_chunks)
        for q in range(EPI_WARPS):
            actors[f"epi{q}.r{r}"] = pair_epilogue(sim, r, q, n_tiles, drift)
    sim.run(actors)
    return sim
