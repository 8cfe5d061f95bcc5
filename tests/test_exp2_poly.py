"""The FMA-pipe 2^x of csrc/exp2_poly.cuh, checked on the CPU against exact 2^x.

The device function's constants are read from the header and its arithmetic is
replayed in fp32 (numpy float32 adds; fma as an exact float64 product-sum rounded
to float32): the shifter rounding, the reduced argument, Horner's rule and the
exponent-field add.  Bound: relative error within 2.5e-7 (about 2 ulp of 1) over
[-125, 0], and exactly 2^r for integer x (p(0) is c0 = 1 + 2^-23)."""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "long_context_kv_obs_b200", "csrc", "exp2_poly.cuh")


def _coeffs():
    src = open(HDR).read()
    body = src[src.index("float exp2_poly"):]
    assert "fmaxf(x, -125.f), 0.f" in body and "12582912.f" in body
    lead = re.findall(r"float p = ([0-9.eE+-]+)f;", body)
    rest = re.findall(r"p = fmaf\(p, f, ([0-9.eE+-]+)f\);", body)
    assert len(lead) == 1 and len(rest) == 5
    return np.array([float(v) for v in lead + rest], dtype=np.float32)     # c5 .. c0


def _fma32(a, b, c):
    return np.float32(np.float64(a) * np.float64(b) + np.float64(c))


def _exp2_poly(x):
    c = _coeffs()
    x = np.float32(min(max(np.float32(x), np.float32(-125.0)), np.float32(0.0)))
    sh = np.float32(12582912.0)
    t = np.float32(x + sh)
    f = np.float32(x - np.float32(t - sh))
    p = c[0]
    for ci in c[1:]:
        p = _fma32(p, f, ci)
    bits = (np.array(p, np.float32).view(np.int32).astype(np.int64)
            + ((np.array(t, np.float32).view(np.int32).astype(np.int64) << 23) & 0xFFFFFFFF))
    bits = ((bits + 2 ** 31) % 2 ** 32) - 2 ** 31
    return float(np.array(bits, np.int64).astype(np.int32).view(np.float32))


def test_exp2_poly_relative_error_bound():
    rng = np.random.default_rng(40)
    xs = np.concatenate([np.linspace(-125.0, 0.0, 40001), -rng.random(20000) * 3, [-0.5, 0.5 - 1, -1e-7, 0.0]])
    worst = 0.0
    for x in xs.astype(np.float32):
        want = 2.0 ** float(x)
        got = _exp2_poly(x)
        worst = max(worst, abs(got - want) / want)
    assert worst <= 2.5e-7, worst


def test_exp2_poly_integers_and_clamp():
    for r in range(-125, 1):
        assert abs(_exp2_poly(float(r)) / 2.0 ** r - 1.0) <= 2.0 ** -23 + 1e-12
    assert _exp2_poly(-1000.0) == _exp2_poly(-125.0)
    assert _exp2_poly(float("-inf")) == _exp2_poly(-125.0)
