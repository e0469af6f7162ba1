"""The FMA-pipe 2^x of the device code (ex2_fma in csrc/sm100.cuh): Cody-Waite
range reduction plus a fitted cubic.  Its steps are replayed here in IEEE
float32 with the coefficients read from the source, and checked against
numpy's exp2 over the range the softmax feeds it (no GPU)."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(__file__), "..", "attention_mqa_gqa_b200", "csrc", "sm100.cuh")


def _coefficients():
    src = open(SRC).read()
    body = src[src.index("float ex2_fma(float x)"):]
    body = body[: body.index("\n}\n")]
    c = [np.float32(v) for v in re.findall(r"(-?\d+\.\d*)f", body)]
    # clamp, rounding constant (twice), then the cubic c3, c2, c1, c0
    assert c[0] == np.float32(-125.0) and c[1] == c[2] == np.float32(12582912.0)
    return c[3:7]


def ex2_fma(x):
    c3, c2, c1, c0 = _coefficients()
    x = np.maximum(np.asarray(x, np.float32), np.float32(-125.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    f = (x - (t - np.float32(12582912.0))).astype(np.float32)
    q = (c3 * f + c2).astype(np.float32)
    q = (q * f + c1).astype(np.float32)
    q = (q * f + c0).astype(np.float32)
    bits = q.view(np.int32) + (t.view(np.int32) << np.int32(23))
    return bits.astype(np.int32).view(np.float32)


def test_relative_error_over_the_softmax_range():
    x = np.linspace(-124.0, 64.0, 2_000_001, dtype=np.float32)
    y = ex2_fma(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(y / ref - 1.0)) < 8e-5


def test_integers_and_halves():
    # at f = 0 the cubic's constant term, at f = +-1/2 its ends
    for n in range(-120, 60, 7):
        for d in (-0.5, -0.25, 0.0, 0.25, 0.4999):
            x = np.float32(n + d)
            assert abs(float(ex2_fma(x)) / 2.0 ** float(x) - 1.0) < 8e-5


def test_clamp_keeps_a_normal_number():
    y = ex2_fma(np.array([-np.inf, -1e30, -200.0, -125.0], np.float32))
    assert np.all(y > 0) and np.all(np.isfinite(y))
    assert np.all(y < 2.0 ** -124) and np.all(y >= np.finfo(np.float32).tiny)
