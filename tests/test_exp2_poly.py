"""The FMA-pipe exponential of the flash kernels (exp2_poly2 in tc_ptx.cuh).

The device helper cannot run here, so its float32 steps are replayed in numpy
(round-to-nearest adds; each fused multiply-add as an exact float64 product
and sum rounded once to float32) and compared with 2^y in float64.  The
coefficients in the header must be the Remez script's output.
"""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "oracle_top_kv_b200", "csrc")


def _remez():
    spec = importlib.util.spec_from_file_location("exp2_poly", os.path.join(CSRC, "exp2_poly.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _header_coeffs():
    src = open(os.path.join(CSRC, "tc_ptx.cuh")).read()
    body = src[src.index("float2 exp2_poly2"):]
    body = body[:body.index("return")]
    vals = {k: np.float32(v) for k, v in re.findall(r"\b(c[0-3]) = ([0-9.e+-]+)f", body)}
    return [vals[f"c{i}"] for i in range(4)]


def _fma32(a, b, c):
    """float32 fused a*b + c: the float64 product of two float32 values is exact."""
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_poly_emulated(y):
    y = np.maximum(np.asarray(y, dtype=np.float32), np.float32(-125.0))
    shift = np.float32(12582912.0)
    t = (y + shift).astype(np.float32)
    r = (t - shift).astype(np.float32)
    f = _fma32(r, np.float32(-1.0), y)
    c0, c1, c2, c3 = _header_coeffs()
    p = _fma32(c3, f, c2)
    p = _fma32(p, f, c1)
    p = _fma32(p, f, c0)
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_header_coefficients_are_the_remez_output():
    c, err = _remez().minimax_exp2(3)
    assert err < 7.6e-5
    assert _header_coeffs() == [np.float32(v) for v in c]


def test_remez_degree3_equioscillates():
    c, err = _remez().minimax_exp2(3)
    g = np.linspace(-0.5, 0.5, 100001)
    e = np.polyval(c[::-1], g) / 2.0 ** g - 1.0
    # best approximation (Chebyshev alternation): the error reaches its bound
    # at n + 2 = 5 points (both ends and the interior extrema), alternating in sign
    s = np.sign(np.diff(e))
    ext = np.concatenate(([0], np.nonzero(s[1:] != s[:-1])[0] + 1, [len(g) - 1]))
    assert len(ext) == 5
    assert np.all(np.abs(np.abs(e[ext]) - err) < 1e-7)
    assert np.all(np.sign(e[ext][1:]) == -np.sign(e[ext][:-1]))


def test_shifter_exponent_identity():
    j = np.arange(-125, 9, dtype=np.int64)
    t = (j.astype(np.float32) + np.float32(12582912.0)).astype(np.float32)
    assert np.all(((t.view(np.uint32).astype(np.uint64) << 23) & 0xFFFFFFFF) ==
                  ((j << 23) & 0xFFFFFFFF))


def test_relative_error_over_the_softmax_range():
    # arguments a softmax tile can produce: up to +8 (lazy rescale) and down
    # to the clamp; dense grid plus the integers and half-integers
    y = np.concatenate([np.linspace(-125.0, 8.0, 2_000_001, dtype=np.float32),
                        np.arange(-125, 9, dtype=np.float32),
                        np.arange(-125, 8, dtype=np.float32) + np.float32(0.5),
                        np.float32([0.0, -0.0, 1e-7, -1e-7])])
    got = exp2_poly_emulated(y).astype(np.float64)
    want = 2.0 ** y.astype(np.float64)
    rel = np.abs(got / want - 1.0)
    assert rel.max() < 8e-5, rel.max()
    assert np.all(np.isfinite(got)) and np.all(got > 0)


def test_clamp_below_range():
    y = np.float32([-126.0, -200.0, -1e30, -np.inf])
    got = exp2_poly_emulated(y).astype(np.float64)
    assert np.all(np.abs(got / 2.0 ** -125 - 1.0) < 8e-5)
