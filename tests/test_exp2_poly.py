"""The software 2^x used for part of the softmax exponentials: its
coefficients match the Remez fit in csrc/exp2_poly_fit.py, and the algorithm
(Cody-Waite reduction, degree-3 polynomial, exponent-field add), replayed in
float32 with numpy, stays within its relative error bound of exact 2^x."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "feed_forward_view_vggt_b200", "csrc")


def header_constants():
    text = open(os.path.join(CSRC, "attn_kernel.cuh")).read()
    c = [float(re.search(rf"kExp2C{k} = ([0-9.eE+-]+)f;", text).group(1)) for k in range(4)]
    magic = float(re.search(r"kRoundMagic = ([0-9.]+)f;", text).group(1))
    lo = float(re.search(r"kExp2MinArg = (-?[0-9.]+)f;", text).group(1))
    return np.array(c, dtype=np.float32), np.float32(magic), np.float32(lo)


def test_coefficients_match_remez_fit():
    spec = importlib.util.spec_from_file_location("fit", os.path.join(CSRC, "exp2_poly_fit.py"))
    fit = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(fit)
    c, err = fit.remez_relative()
    hc, _, _ = header_constants()
    assert np.array_equal(c.astype(np.float32), hc)
    assert err < 8e-5


def emulate(x):
    c, magic, lo = header_constants()
    f32 = np.float32
    x = np.maximum(x.astype(f32), lo)
    y = (x + magic).astype(f32)
    j = (y - magic).astype(f32)
    f = (x - j).astype(f32)
    q = (c[3] * f + c[2]).astype(f32)
    q = (q * f + c[1]).astype(f32)
    q = (q * f + c[0]).astype(f32)
    bits = (y.view(np.uint32).astype(np.uint64) * 8388608 + q.view(np.uint32)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(f32)


def test_relative_error_bound_over_the_softmax_range():
    x = np.concatenate([np.linspace(-125, 8, 2_000_001, dtype=np.float32),
                        np.float32(np.random.default_rng(0).uniform(-30, 8, 200_000))])
    got = emulate(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.abs(got / ref - 1).max() < 1e-4


def test_clamps_below_the_normal_range():
    got = emulate(np.array([-1e30, -np.inf, -200.0, -125.0], dtype=np.float32))
    assert np.all(got > 0) and np.all(got <= np.exp2(-125.0) * 1.0001)
    assert np.all(np.isfinite(got))
