"""Pins for the fp64 oracle, checked against things other than itself:
hand-derived index lists, closed forms, invariants of the definition, and
independent numpy brute force on tiny inputs.  CPU only."""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import FRAME, GLOBAL, SGA, Shape
from feed_forward_view_vggt_b200 import accounting

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
BF16_ONE = 0x3F80


def read_golden_pairs(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = line.split(None, 1)
            out[key] = val
    return out


def read_axis_golden():
    rows = []
    with open(os.path.join(GOLDEN, "sga_axis_kept.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            lhs, rhs = line.split(":")
            n, s = map(int, lhs.split())
            rows.append((n, s, [int(x) for x in rhs.split()]))
    return rows


def to_f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def to_bits(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16) \
        .view(torch.int16).numpy().view(np.uint16)


def rand_bits(rng, shape, scale=1.0):
    return to_bits(rng.standard_normal(shape) * scale)


def golden_keep_mask(shape, s_h, s_w):
    """Per-token keep mask assembled from the hand-derived axis coordinates."""
    table = {(n, s): ks for n, s, ks in read_axis_golden()}
    rk, ck = table[(shape.h, s_h)], table[(shape.w, s_w)]
    keep_frame = np.zeros(shape.L, dtype=bool)
    keep_frame[: shape.n_special] = True
    for r in rk:
        for c in ck:
            keep_frame[shape.n_special + r * shape.w + c] = True
    return np.tile(keep_frame, shape.N)


def dense_np(q, k, v, allowed, scale):
    """numpy fp64 dense softmax attention; allowed[i, j] masks keys."""
    S, H, d = q.shape
    out = np.empty((S, H, d))
    lse = np.empty((S, H))
    for h in range(H):
        logits = (q[:, h, :] @ k[:, h, :].T) * scale
        logits = np.where(allowed, logits, -np.inf)
        m = logits.max(axis=1, keepdims=True)
        p = np.exp(logits - m)
        den = p.sum(axis=1, keepdims=True)
        out[:, h, :] = (p @ v[:, h, :]) / den
        lse[:, h] = (m + np.log(den))[:, 0]
    return out, lse


TINY = Shape(N=2, n_special=5, h=8, w=8, H=2, d=64)


@pytest.fixture(scope="module")
def tiny_qkv():
    rng = np.random.default_rng(7)
    return tuple(rand_bits(rng, (TINY.S, TINY.H, TINY.d)) for _ in range(3))


# ---------------------------------------------------------------- index pins

def test_axis_kept_matches_hand_derived_golden():
    for n, s, expect in read_axis_golden():
        assert oracle.axis_kept(n, s).tolist() == expect, (n, s)


def test_build_index_8x8_stride2_handwritten():
    shape = Shape(N=2, n_special=5, h=8, w=8, H=1, d=64)
    kept, mult, nk, nd = oracle.sga_build_index(shape, 2, 2)
    frame0 = [0, 1, 2, 3, 4,
              5, 7, 9, 11, 21, 23, 25, 27, 37, 39, 41, 43, 53, 55, 57, 59]
    expect = frame0 + [69 + t for t in frame0]
    assert kept.tolist() == expect
    assert nk == 42 and nd == 2 * 64 - 2 * 16
    dropped = np.ones(shape.S, dtype=bool)
    dropped[expect] = False
    assert np.array_equal(mult, np.where(dropped, nd - 1, nd))


@pytest.mark.parametrize("N,ns,h,w,sh,sw", [
    (2, 5, 8, 8, 2, 2), (2, 5, 8, 8, 3, 3), (3, 5, 8, 8, 1, 1), (1, 5, 37, 37, 2, 2),
    (4, 5, 37, 37, 3, 3), (2, 0, 5, 7, 2, 3), (3, 2, 6, 4, 8, 8), (2, 5, 1, 9, 1, 4),
    (1, 1, 0, 0, 2, 2)])
def test_build_index_counts_and_structure(N, ns, h, w, sh, sw):
    shape = Shape(N=N, n_special=ns, h=h, w=w, H=1, d=64)
    kept, mult, nk, nd = oracle.sga_build_index(shape, sh, sw)
    closed = N * (ns + math.ceil(h / sh) * math.ceil(w / sw)) if h and w else N * ns
    assert nk == closed
    assert nk + nd == shape.S
    assert np.all(np.diff(kept) > 0)
    is_kept = np.zeros(shape.S, dtype=bool)
    is_kept[kept] = True
    assert np.array_equal(mult, np.where(is_kept, nd, nd - 1))
    # every special token is kept
    for n in range(N):
        assert is_kept[n * shape.L: n * shape.L + ns].all()
    # same kept pattern in every frame
    pat = is_kept.reshape(N, shape.L)
    assert (pat == pat[0]).all()


def test_worked_example_counts():
    g = read_golden_pairs("worked_example.txt")
    side = int(g["image_side"]) // int(g["patch_side"])
    assert side == int(g["patch_grid_side"])
    assert side * side == int(g["patches_per_view"])
    shape = Shape(N=int(g["views"]), n_special=5, h=side, w=side, H=16, d=64)
    assert shape.N * shape.h * shape.w == int(g["patch_tokens_total"])
    assert shape.L == 1374 and shape.S == 5496
    # 37x37 at stride 2 and 3 keep 19x19 and 13x13 patches per frame
    assert oracle.sga_build_index(shape, 2, 2)[2] == 4 * (5 + 361)
    assert oracle.sga_build_index(shape, 3, 3)[2] == 4 * (5 + 169)


def test_memory_arithmetic_closed_form():
    g = read_golden_pairs("memory_arithmetic.txt")
    tokens = int(g["images"]) * int(g["tokens_per_image"])
    assert tokens == int(g["total_tokens"])
    entries = accounting.attention_matrix_entries(tokens)
    assert round(entries / 1e10, 2) == float(g["entries"]) / 1e10
    assert round(accounting.attention_matrix_bytes(tokens, 2) / 1e9) == int(g["fp16_GB"])
    assert round(accounting.attention_matrix_bytes(tokens, 4) / 1e9) == int(g["fp32_GB"])


def test_accounting_counts_agree_with_oracle_index():
    for (N, ns, h, w, sh, sw) in [(100, 5, 37, 37, 2, 2), (800, 5, 37, 37, 3, 3),
                                  (2, 5, 8, 8, 3, 3), (3, 0, 7, 5, 4, 2)]:
        shape = Shape(N=N, n_special=ns, h=h, w=w, H=1, d=64)
        _, _, nk, nd = oracle.sga_build_index(shape, sh, sw)
        assert accounting.sga_counts(N, ns, h, w, sh, sw) == (nk, nd)
    assert accounting.sga_counts(100, 5, 37, 37, 2, 2) == (36600, 100800)


# ------------------------------------------------------- frame / global pins

def frame_ids(shape):
    return np.repeat(np.arange(shape.N), shape.L)


def test_frame_and_global_match_numpy_dense(tiny_qkv):
    q, k, v = tiny_qkv
    scale = 0.125
    fid = frame_ids(TINY)
    for mode, allowed in ((FRAME, fid[:, None] == fid[None, :]),
                          (GLOBAL, np.ones((TINY.S, TINY.S), dtype=bool))):
        out, lse = oracle.attention(mode, q, k, v, TINY, scale)
        ref, ref_lse = dense_np(to_f64(q), to_f64(k), to_f64(v), allowed, scale)
        assert np.abs(out - ref).max() < 1e-12
        assert np.abs(lse - ref_lse).max() < 1e-12


def test_rows_subset_matches_full(tiny_qkv):
    q, k, v = tiny_qkv
    rows = np.array([0, 3, 68, 69, 100, 137])
    for mode in (FRAME, GLOBAL, SGA):
        full, full_lse = oracle.attention(mode, q, k, v, TINY, s_h=2, s_w=2)
        part, part_lse = oracle.attention(mode, q, k, v, TINY, s_h=2, s_w=2, rows=rows)
        assert np.array_equal(part, full[rows]) and np.array_equal(part_lse, full_lse[rows])


def test_rows_sum_to_one(tiny_qkv):
    q, k, _ = tiny_qkv
    ones = np.full_like(q, BF16_ONE)
    for mode in (FRAME, GLOBAL, SGA):
        for sh, sw in ((2, 2), (3, 3)):
            out, _ = oracle.attention(mode, q, k, ones, TINY, s_h=sh, s_w=sw)
            assert np.abs(out - 1.0).max() < 1e-12


def test_zero_keys_give_key_set_mean(tiny_qkv):
    q, _, v = tiny_qkv
    zeros = np.zeros_like(q)
    vf = to_f64(v).reshape(TINY.N, TINY.L, TINY.H, TINY.d)
    out_f, lse_f = oracle.attention(FRAME, q, zeros, v, TINY)
    expect_f = np.repeat(vf.mean(axis=1), TINY.L, axis=0)
    assert np.abs(out_f - expect_f).max() < 1e-12
    assert np.abs(lse_f - math.log(TINY.L)).max() < 1e-12
    out_g, lse_g = oracle.attention(GLOBAL, q, zeros, v, TINY)
    expect_g = vf.reshape(TINY.S, TINY.H, TINY.d).mean(axis=0)
    assert np.abs(out_g - expect_g[None]).max() < 1e-12
    assert np.abs(lse_g - math.log(TINY.S)).max() < 1e-12


def test_two_key_logistic_closed_form():
    shape = Shape(N=1, n_special=2, h=0, w=0, H=1, d=64)
    a = 3.0
    q = np.zeros((2, 1, 64)); q[:, 0, 0] = a
    k = np.zeros((2, 1, 64)); k[0, 0, 0] = 1.0; k[1, 0, 0] = -1.0
    rng = np.random.default_rng(3)
    v = rng.standard_normal((2, 1, 64))
    qb, kb, vb = to_bits(q), to_bits(k), to_bits(v)
    vf = to_f64(vb)
    for scale in (0.125, 0.5):
        out, lse = oracle.attention(GLOBAL, qb, kb, vb, shape, scale)
        sig = 1.0 / (1.0 + math.exp(-2 * a * scale))
        expect = sig * vf[0, 0] + (1 - sig) * vf[1, 0]
        assert np.abs(out[:, 0, :] - expect[None]).max() < 1e-12
        assert abs(lse[0, 0] - math.log(math.exp(a * scale) + math.exp(-a * scale))) < 1e-12


def test_global_with_one_frame_equals_frame():
    shape = Shape(N=1, n_special=5, h=8, w=8, H=2, d=64)
    rng = np.random.default_rng(11)
    q, k, v = (rand_bits(rng, (shape.S, 2, 64)) for _ in range(3))
    f, fl = oracle.attention(FRAME, q, k, v, shape)
    g, gl = oracle.attention(GLOBAL, q, k, v, shape)
    assert np.abs(f - g).max() < 1e-13 and np.abs(fl - gl).max() < 1e-13


@pytest.mark.parametrize("mode", [FRAME, GLOBAL, SGA])
def test_frame_permutation_equivariance(mode):
    shape = Shape(N=3, n_special=5, h=4, w=6, H=2, d=64)
    rng = np.random.default_rng(5)
    q, k, v = (rand_bits(rng, (shape.S, 2, 64)) for _ in range(3))
    perm = np.array([2, 0, 1])
    tok = (perm[:, None] * shape.L + np.arange(shape.L)[None, :]).reshape(-1)
    out, _ = oracle.attention(mode, q, k, v, shape, s_h=2, s_w=3)
    outp, _ = oracle.attention(mode, q[tok], k[tok], v[tok], shape, s_h=2, s_w=3)
    assert np.abs(outp - out[tok]).max() < 1e-12


# ------------------------------------------------------------------ SGA pins

def test_sga_stride_one_equals_global(tiny_qkv):
    q, k, v = tiny_qkv
    g, gl = oracle.attention(GLOBAL, q, k, v, TINY)
    s, sl = oracle.attention(SGA, q, k, v, TINY, s_h=1, s_w=1)
    assert np.abs(g - s).max() < 1e-12 and np.abs(gl - sl).max() < 1e-12


def test_sga_identical_dropped_tokens_equals_global(tiny_qkv):
    q, k, v = (x.copy() for x in tiny_qkv)
    keep = golden_keep_mask(TINY, 2, 2)
    rng = np.random.default_rng(9)
    k_star = rand_bits(rng, (TINY.H, TINY.d))
    v_star = rand_bits(rng, (TINY.H, TINY.d))
    k[~keep] = k_star
    v[~keep] = v_star
    g, gl = oracle.attention(GLOBAL, q, k, v, TINY)
    s, sl = oracle.attention(SGA, q, k, v, TINY, s_h=2, s_w=2)
    assert np.abs(g - s).max() < 1e-12 and np.abs(gl - sl).max() < 1e-12


def test_sga_single_dropped_token_equals_global():
    shape = Shape(N=1, n_special=5, h=1, w=2, H=2, d=64)
    rng = np.random.default_rng(13)
    q, k, v = (rand_bits(rng, (shape.S, 2, 64)) for _ in range(3))
    kept, mult, nk, nd = oracle.sga_build_index(shape, 1, 2)
    assert nd == 1 and kept.tolist() == [0, 1, 2, 3, 4, 5]
    g, gl = oracle.attention(GLOBAL, q, k, v, shape)
    s, sl = oracle.attention(SGA, q, k, v, shape, s_h=1, s_w=2)
    assert np.abs(g - s).max() < 1e-12 and np.abs(gl - sl).max() < 1e-12


def test_sga_means_match_numpy(tiny_qkv):
    _, k, v = tiny_qkv
    for sh, sw in ((2, 2), (3, 3)):
        keep = golden_keep_mask(TINY, sh, sw)
        kbar, vbar = oracle.sga_means(k, v, TINY, sh, sw)
        assert np.abs(kbar - to_f64(k)[~keep].mean(axis=0)).max() < 1e-13
        assert np.abs(vbar - to_f64(v)[~keep].mean(axis=0)).max() < 1e-13
    assert oracle.sga_means(k, v, TINY, 1, 1) is None


@pytest.mark.parametrize("sh,sw", [(2, 2), (3, 3), (2, 3)])
def test_sga_matches_augmented_key_bruteforce(tiny_qkv, sh, sw):
    """Each dropped key/value other than the query's own is replaced by the
    mean (kbar, vbar); the query's own key stays; then plain softmax over
    all S columns.  Built literally per query with numpy."""
    q, k, v = tiny_qkv
    table = {(n, s): ks for n, s, ks in read_axis_golden()}
    if (8, sh) not in table or (8, sw) not in table:
        pytest.skip("no golden coordinates")
    keep = golden_keep_mask(TINY, sh, sw)
    qf, kf, vf = to_f64(q), to_f64(k), to_f64(v)
    kbar, vbar = kf[~keep].mean(axis=0), vf[~keep].mean(axis=0)
    scale = 0.125
    ref = np.empty_like(qf)
    for i in range(TINY.S):
        replace = ~keep.copy()
        replace[i] = False
        for h in range(TINY.H):
            kaug = np.where(replace[:, None], kbar[h][None, :], kf[:, h, :])
            vaug = np.where(replace[:, None], vbar[h][None, :], vf[:, h, :])
            lg = kaug @ qf[i, h] * scale
            p = np.exp(lg - lg.max())
            ref[i, h] = p @ vaug / p.sum()
    out, _ = oracle.attention(SGA, q, k, v, TINY, scale, s_h=sh, s_w=sw)
    assert np.abs(out - ref).max() < 1e-12


def test_sga_differs_from_global_when_dropping(tiny_qkv):
    # guards against an SGA that silently falls back to full attention
    q, k, v = tiny_qkv
    g, _ = oracle.attention(GLOBAL, q, k, v, TINY)
    s, _ = oracle.attention(SGA, q, k, v, TINY, s_h=2, s_w=2)
    assert np.abs(g - s).max() > 1e-3


# ------------------------------------------------------- register attention

REG = Shape(N=3, n_special=17, h=4, w=4, H=2, d=64)


@pytest.fixture(scope="module")
def reg_qkv():
    rng = np.random.default_rng(21)
    return tuple(rand_bits(rng, (REG.S, REG.H, REG.d)) for _ in range(3))


def test_register_matches_numpy_on_gathered_specials(reg_qkv):
    q, k, v = reg_qkv
    rows = oracle.special_rows(REG)
    out, lse = oracle.register_attention(q, k, v, REG)
    # numpy: dense attention over the gathered special tokens only
    allowed = np.ones((len(rows), len(rows)), dtype=bool)
    ref, ref_lse = dense_np(to_f64(q)[rows], to_f64(k)[rows], to_f64(v)[rows], allowed, 0.125)
    assert np.abs(out - ref).max() < 1e-12 and np.abs(lse - ref_lse).max() < 1e-12


def test_register_with_specials_only_equals_global():
    shape = Shape(N=4, n_special=17, h=0, w=0, H=2, d=64)
    rng = np.random.default_rng(22)
    q, k, v = (rand_bits(rng, (shape.S, 2, 64)) for _ in range(3))
    g, gl = oracle.attention(GLOBAL, q, k, v, shape)
    r, rl = oracle.register_attention(q, k, v, shape)
    assert np.abs(g - r).max() < 1e-13 and np.abs(gl - rl).max() < 1e-13


def test_register_ignores_patch_tokens_and_sums_to_one(reg_qkv):
    q, k, v = (x.copy() for x in reg_qkv)
    out, _ = oracle.register_attention(q, k, v, REG)
    patch = np.ones(REG.S, dtype=bool)
    patch[oracle.special_rows(REG)] = False
    rng = np.random.default_rng(23)
    k[patch] = rand_bits(rng, (patch.sum(), REG.H, REG.d))
    v[patch] = rand_bits(rng, (patch.sum(), REG.H, REG.d))
    out2, _ = oracle.register_attention(q, k, v, REG)
    assert np.array_equal(out, out2)
    ones = np.full_like(q, BF16_ONE)
    o1, _ = oracle.register_attention(q, k, ones, REG)
    assert np.abs(o1 - 1.0).max() < 1e-12


def test_register_rejects_patch_rows(reg_qkv):
    q, k, v = reg_qkv
    with pytest.raises(ValueError):
        oracle.register_attention(q, k, v, REG, rows=np.array([REG.n_special]))
