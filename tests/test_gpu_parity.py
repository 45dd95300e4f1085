"""GPU parity: the sm_100a kernels, called through the C ABI, against the
fp64 CPU oracle on the same seeded inputs.

Bar (bf16 in, fp32 accumulate, bf16 out): max-abs <= 2e-2 and relative
Frobenius <= 5e-3 on the outputs; SGA index lists and multiplicities
bit-exact.  Small workloads are compared in full; large ones on 4096 seeded
query tokens x all heads (token 0, token S-1, the frame-0 specials and the
ragged tails always included)."""
import numpy as np
import pytest
import torch

import oracle
from feed_forward_view_vggt_b200 import attn, synth

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
REL_FRO = 5e-3
LSE_ABS = 2e-2


def bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def oshape(wl):
    return oracle.Shape(wl.N, wl.n_special, wl.h, wl.w, wl.H, wl.d)


def check_ok():
    st, detail = attn.vggt_check()
    assert st == attn.VGGT_OK, (attn.vggt_status_string(st), hex(detail))


def assert_close(got_dev, ref, rows, what, lse_dev=None, ref_lse=None):
    got = got_dev[torch.as_tensor(rows, device=got_dev.device)].float().cpu().double().numpy()
    assert np.isfinite(got).all(), what
    err = np.abs(got - ref)
    rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
    assert err.max() <= MAX_ABS and rel <= REL_FRO, f"{what}: max-abs {err.max():.3g}, rel-fro {rel:.3g}"
    if lse_dev is not None:
        gl = lse_dev[torch.as_tensor(rows, device=lse_dev.device)].double().cpu().numpy()
        assert np.abs(gl - ref_lse).max() <= LSE_ABS, f"{what} lse: {np.abs(gl - ref_lse).max():.3g}"


class Case:
    """Seeded inputs of one workload, on host (bf16 bits) and device."""

    def __init__(self, wl):
        self.wl = wl
        q, k, v = synth.make_qkv(wl)
        self.qb, self.kb, self.vb = bits(q), bits(k), bits(v)
        self.q, self.k, self.v = (x.cuda() for x in (q, k, v))
        self.shape = oshape(wl)


_cases = {}


def case(name):
    if name not in _cases:
        _cases[name] = Case(synth.WORKLOADS[name])
    return _cases[name]


def run_and_compare(c, op, rows, stride=(2, 2), nthreads=0):
    wl, sh = c.wl, c.shape
    if op == "frame":
        o, lse = attn.frame(c.q, c.k, c.v, wl, want_lse=True)
        ref, ref_lse = oracle.frame_attention(c.qb, c.kb, c.vb, sh, rows=rows, nthreads=nthreads)
    elif op == "global":
        o, lse = attn.global_(c.q, c.k, c.v, wl, want_lse=True)
        ref, ref_lse = oracle.global_attention(c.qb, c.kb, c.vb, sh, rows=rows, nthreads=nthreads)
    else:
        idx = attn.SgaIndex(wl, *stride)
        o, lse = attn.sga(c.q, c.k, c.v, idx, want_lse=True)
        ref, ref_lse = oracle.sga_attention(c.qb, c.kb, c.vb, sh, *stride, rows=rows, nthreads=nthreads)
    check_ok()
    assert_close(o, ref, rows, f"{wl.name} {op} {stride if op == 'sga' else ''}", lse, ref_lse)
    return o


# ------------------------------------------------------------ index parity

@pytest.mark.parametrize("N,ns,h,w,sh,sw", [
    (2, 5, 8, 8, 2, 2), (2, 5, 8, 8, 3, 3), (2, 5, 8, 8, 1, 1), (4, 5, 37, 37, 2, 2),
    (4, 5, 37, 37, 3, 3), (100, 5, 37, 37, 2, 2), (800, 5, 37, 37, 3, 3), (3, 0, 7, 5, 4, 2),
    (2, 3, 6, 4, 8, 8), (1, 5, 1, 2, 1, 2), (5, 1, 9, 1, 3, 1), (2, 5, 0, 0, 2, 2)])
def test_index_bit_exact(N, ns, h, w, sh, sw):
    shape = oracle.Shape(N, ns, h, w, 16, 64)
    kept, mult, nk, nd = oracle.sga_build_index(shape, sh, sw)
    idx = attn.SgaIndex(shape, sh, sw)
    check_ok()
    assert idx.n_kept == nk and idx.n_dropped == nd
    assert np.array_equal(idx.kept_idx[:nk].cpu().numpy(), kept)
    assert np.array_equal(idx.mult.cpu().numpy(), mult)


# ------------------------------------------------------ full comparisons

@pytest.mark.parametrize("op", ["frame", "global", "sga"])
def test_tiny_full(op):
    c = case("tiny")
    run_and_compare(c, op, np.arange(c.wl.S))


@pytest.mark.parametrize("op,stride", [("frame", None), ("global", None), ("sga", (2, 2)), ("sga", (3, 3))])
def test_n4_full(op, stride):
    c = case("n4")
    run_and_compare(c, op, np.arange(c.wl.S), stride or (2, 2))


# ------------------------------------------------------ sampled at scale

def sampled(wl, count=4096):
    return synth.sample_rows(wl.S, wl.L, wl.n_special, count=count)


@pytest.mark.parametrize("op,stride", [("frame", None), ("global", None), ("sga", (2, 2)), ("sga", (3, 3))])
def test_n32_sampled(op, stride):
    c = case("n32")
    run_and_compare(c, op, sampled(c.wl), stride or (2, 2))


@pytest.mark.parametrize("op,stride", [("global", None), ("sga", (2, 2)), ("frame", None)])
def test_n100_sampled(op, stride):
    c = case("n100")
    run_and_compare(c, op, sampled(c.wl), stride or (2, 2))


# ------------------------------------------------------------- mean-fill

@pytest.mark.parametrize("name,stride", [("tiny", (2, 2)), ("n4", (3, 3)), ("n100", (2, 2))])
def test_meanfill_matches_oracle(name, stride):
    c = case(name)
    idx = attn.SgaIndex(c.wl, *stride)
    attn.sga(c.q, c.k, c.v, idx)
    check_ok()
    kbar, vbar = (x.double().cpu().numpy() for x in idx.means())
    rk, rv = oracle.sga_means(c.kb, c.vb, c.shape, *stride)
    for got, ref in ((kbar, rk), (vbar, rv)):
        assert np.abs(got - ref).max() <= 1e-5 + 1e-4 * np.abs(ref).max()


# ------------------------------------------------------------ edge cases

def make_case(N, ns, h, w, H, seed=0, scale_q=1.0):
    wl = synth.Workload(f"edge{N}_{ns}_{h}x{w}_{H}", N=N, h=h, w=w, H=H, seed=seed, structure="iid",
                        n_special=ns)
    c = Case(wl)
    if scale_q != 1.0:
        q = (synth.make_qkv(wl)[0].float() * scale_q).to(torch.bfloat16)
        c.qb, c.q = bits(q), q.cuda()
    return c


@pytest.mark.parametrize("N,ns,h,w,H", [
    (3, 5, 5, 7, 3),      # L = 40: one ragged key tile, mostly empty second q tile
    (1, 0, 16, 16, 1),    # L = 256: exactly one item, no tail
    (2, 5, 20, 20, 2),    # L = 405: two items per frame, 4 key tiles with a tail
    (5, 1, 3, 3, 4),      # L = 10: tiny frames, global S = 50
    (7, 1, 0, 0, 2),      # L = 1: specials only (SGA keeps everything)
    (1, 5, 37, 37, 2),    # one VGGT frame: global == frame
])
@pytest.mark.parametrize("op", ["frame", "global", "sga"])
def test_ragged_shapes(N, ns, h, w, H, op):
    c = make_case(N, ns, h, w, H, seed=N * 131 + h)
    stride = (2, 3) if h and w else (2, 2)
    run_and_compare(c, op, np.arange(c.wl.S), stride)


def test_large_logits_exercise_rescaling():
    # q scaled by 6: logits spread over ~+-40, so the running max jumps
    # often and the O/l rescale path runs.
    c = make_case(4, 5, 12, 12, 2, seed=5, scale_q=6.0)
    for op in ("frame", "global", "sga"):
        run_and_compare(c, op, np.arange(c.wl.S))


def test_large_logits_lean_instantiation():
    # The same at N = 8 (S = 1192: 10 query tiles per head, an even count), so
    # global attention and SGA run the lean instantiation, whose slow path
    # keeps S in registers and overwrites the P chunks it stored early (63
    # global row-steps take it, by a CPU emulation of the rule on these
    # inputs); the N = 4 case above (5 tiles) runs the general one.
    c = make_case(8, 5, 12, 12, 2, seed=7, scale_q=6.0)
    for op in ("global", "sga"):
        run_and_compare(c, op, np.arange(c.wl.S))


@pytest.mark.parametrize("stride", [(1, 1), (8, 8), (2, 1)])
def test_sga_degenerate_strides(stride):
    c = make_case(3, 5, 6, 7, 2, seed=9)
    run_and_compare(c, "sga", np.arange(c.wl.S), stride)


def test_sga_stride_one_equals_global_on_gpu():
    c = case("n4")
    g = attn.global_(c.q, c.k, c.v, c.wl)
    s = attn.sga(c.q, c.k, c.v, attn.SgaIndex(c.wl, 1, 1))
    check_ok()
    assert (g.float() - s.float()).abs().max().item() <= MAX_ABS


def test_sga_single_dropped_token():
    c = make_case(1, 5, 1, 2, 2, seed=3)
    run_and_compare(c, "sga", np.arange(c.wl.S), (1, 2))


def test_values_all_one_give_one():
    c = case("n4")
    ones = torch.ones_like(c.v)
    idx = attn.SgaIndex(c.wl, 2, 2)
    for o in (attn.frame(c.q, c.k, ones, c.wl), attn.global_(c.q, c.k, ones, c.wl),
              attn.sga(c.q, c.k, ones, idx)):
        check_ok()
        assert (o.float() - 1.0).abs().max().item() <= 1e-2


def test_deterministic_and_frame_permutation_equivariant():
    c = case("n4")
    wl = c.wl
    a = attn.global_(c.q, c.k, c.v, wl)
    b = attn.global_(c.q, c.k, c.v, wl)
    check_ok()
    assert torch.equal(a, b)
    perm = torch.tensor([2, 0, 3, 1])
    tok = (perm[:, None] * wl.L + torch.arange(wl.L)[None, :]).reshape(-1).cuda()
    for fn in (attn.frame, attn.global_):
        o = fn(c.q, c.k, c.v, wl)
        op = fn(c.q[tok].contiguous(), c.k[tok].contiguous(), c.v[tok].contiguous(), wl)
        check_ok()
        assert (op.float() - o[tok].float()).abs().max().item() <= 2e-2
