"""Pins of the oracle's fused QKV projection + 2D RoPE, each against
something other than the oracle's own formula:

* the projection against numpy's matmul (rows that are not rotated: the
  special tokens, and V everywhere);
* block-identity weights give exact multiples of the input;
* the rotation as complex multiplication, with the frequencies built as a
  geometric sequence;
* norm preservation per half-head;
* the relative-position property: the score between two rotated tokens
  depends only on their position difference;
* zero input gives the bias."""
import numpy as np
import pytest
import torch

import oracle

SH = oracle.Shape(N=2, n_special=2, h=3, w=4, H=2, d=64)  # C = 128, S = 28
C = SH.H * SH.d
BASE = 100.0


def bf16(a):
    return torch.as_tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


def widen(t):
    return t.float().double().numpy()


def special_rows():
    return np.array([t for t in range(SH.S) if t % SH.L < SH.n_special], dtype=np.int64)


def patch_rows():
    return np.array([t for t in range(SH.S) if t % SH.L >= SH.n_special], dtype=np.int64)


def grid_pos(t):
    g = t % SH.L - SH.n_special
    return g // SH.w, g % SH.w


@pytest.fixture(scope="module")
def rnd():
    g = torch.Generator().manual_seed(11)
    x = torch.randn(SH.S, C, generator=g).to(torch.bfloat16)
    w = (torch.randn(3 * C, C, generator=g) / np.sqrt(C)).to(torch.bfloat16)
    b = (0.1 * torch.randn(3 * C, generator=g)).numpy().astype(np.float32)
    return x, w, b


def test_projection_matches_numpy_matmul_where_nothing_rotates(rnd):
    x, w, b = rnd
    q, k, v = oracle.qkv_rope(x, w, b, SH, BASE)
    y = widen(x) @ widen(w).T + b.astype(np.float64)
    sr = special_rows()
    np.testing.assert_allclose(q[sr].reshape(len(sr), C), y[sr, :C], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(k[sr].reshape(len(sr), C), y[sr, C:2 * C], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(v.reshape(SH.S, C), y[:, 2 * C:], rtol=1e-12, atol=1e-12)


def test_block_identity_weights_give_exact_multiples(rnd):
    x = rnd[0]
    eye = np.eye(C, dtype=np.float32)
    w = bf16(np.concatenate([eye, 2 * eye, 3 * eye]))
    q, k, v = oracle.qkv_rope(x, w, None, SH, BASE)
    xs = widen(x)
    sr = special_rows()
    assert np.array_equal(q[sr].reshape(len(sr), C), xs[sr])
    assert np.array_equal(k[sr].reshape(len(sr), C), 2 * xs[sr])
    assert np.array_equal(v.reshape(SH.S, C), 3 * xs)


def test_rotation_is_complex_multiplication(rnd):
    x = rnd[0]
    eye = np.eye(C, dtype=np.float32)
    q, k, _ = oracle.qkv_rope(x, bf16(np.concatenate([eye, eye, eye])), None, SH, BASE)
    assert np.array_equal(q, k)
    xs = widen(x).reshape(SH.S, SH.H, SH.d)
    e = SH.d // 2
    freqs = np.geomspace(1.0, BASE ** (-(e // 2 - 1) / (e // 2)), e // 2)  # 1, base^-1/16, ...
    for t in patch_rows():
        r, c = grid_pos(t)
        for hh in range(SH.H):
            for half, pos in ((0, r), (1, c)):
                seg = xs[t, hh, half * e:(half + 1) * e]
                z = (seg[:e // 2] + 1j * seg[e // 2:]) * np.exp(1j * pos * freqs)
                got = q[t, hh, half * e:(half + 1) * e]
                np.testing.assert_allclose(got[:e // 2], z.real, atol=1e-12)
                np.testing.assert_allclose(got[e // 2:], z.imag, atol=1e-12)


def test_rotation_preserves_norms_per_half(rnd):
    x, w, b = rnd
    q, k, v = oracle.qkv_rope(x, w, b, SH, BASE)
    y = (widen(x) @ widen(w).T + b.astype(np.float64)).reshape(SH.S, 3, SH.H, 2, SH.d // 2)
    for part, got in ((0, q), (1, k)):
        g = got.reshape(SH.S, SH.H, 2, SH.d // 2)
        np.testing.assert_allclose(np.linalg.norm(g, axis=-1), np.linalg.norm(y[:, part], axis=-1), rtol=1e-12)


def test_scores_depend_only_on_the_position_difference():
    # every patch token of frame 0 carries the same vector u: q = k = R(pos) u
    g = torch.Generator().manual_seed(5)
    u = torch.randn(C, generator=g).numpy()
    xs = np.zeros((SH.S, C), dtype=np.float32)
    xs[:SH.L] = u
    eye = np.eye(C, dtype=np.float32)
    q, k, _ = oracle.qkv_rope(bf16(xs), bf16(np.concatenate([eye, eye, eye])), None, SH, BASE)

    def tok(r, c):
        return SH.n_special + r * SH.w + c

    def score(a, b):
        return float(np.sum(q[tok(*a)] * k[tok(*b)]))

    for d_r, d_c in ((1, 2), (0, 1), (2, 0), (1, -1)):
        pairs = [((r, c), (r + d_r, c + d_c)) for r in range(SH.h) for c in range(SH.w)
                 if 0 <= r + d_r < SH.h and 0 <= c + d_c < SH.w]
        vals = [score(a, b) for a, b in pairs]
        assert len(vals) >= 2
        np.testing.assert_allclose(vals, vals[0], rtol=1e-10)
    # and it does depend on the difference
    assert abs(score((0, 0), (1, 2)) - score((0, 0), (2, 1))) > 1e-3


def test_zero_input_gives_the_bias(rnd):
    _, w, b = rnd
    q, k, v = oracle.qkv_rope(bf16(np.zeros((SH.S, C))), w, b, SH, BASE)
    sr = special_rows()
    np.testing.assert_allclose(q[sr].reshape(len(sr), C), np.broadcast_to(b[:C], (len(sr), C)), atol=1e-12)
    np.testing.assert_allclose(v.reshape(SH.S, C), np.broadcast_to(b[2 * C:], (SH.S, C)), atol=1e-12)


def test_rejects_bad_arguments(rnd):
    x, w, b = rnd
    with pytest.raises(ValueError):
        oracle.qkv_rope(x, w, b, SH, base=0.0)
    with pytest.raises(ValueError):
        oracle.qkv_rope(x, w, b, SH, rows=[SH.S])


def test_linear_matches_numpy_matmul_and_identity(rnd):
    x, w, b = rnd
    wo = w[:C]
    y = oracle.linear(x, wo, b[:C])
    np.testing.assert_allclose(y, widen(x) @ widen(wo).T + b[:C].astype(np.float64), rtol=1e-12, atol=1e-12)
    eye = bf16(np.eye(C, dtype=np.float32))
    assert np.array_equal(oracle.linear(x, eye), widen(x))
    rows = np.array([3, 0, 27])
    np.testing.assert_array_equal(oracle.linear(x, wo, b[:C], rows=rows), y[rows])
