"""The FMA-pipe base-2 exponential the scan kernels use for a share of their decays
(``exp2_poly_pair`` in ``csrc/common.cuh``): its coefficients are read from the source and
the same steps are evaluated in single precision here, against 2^v in double precision.

The bound it must meet is the SFU's own: ``ex2.approx.f32`` is documented with a maximum
relative error of about 2^-22 (2.4e-7); the polynomial stays below 3e-7 over the range the
kernel admits, and the integer exponent add is exact.
"""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(__file__), "..", "selective_state_space_45_b200", "csrc", "common.cuh")


def _coefficients():
    text = open(SRC).read()
    body = text[text.index("exp2_poly_pair(float2 v)"):]
    body = body[:body.index("return f2(")]
    vals = re.findall(r"f2\(([-0-9.e]+)f, \1f\)", body)
    # q starts at the highest coefficient, then Horner steps down to the constant term
    return [np.float32(v) for v in vals if abs(float(v)) < 2.0 and float(v) != -1.0]


def _poly_exp2(v):
    v = np.clip(np.asarray(v, np.float32), np.float32(-126), np.float32(126))
    k = np.float32(12582912.0)
    t = (v + k).astype(np.float32)
    r = (t - k).astype(np.float32)
    f = (v - r).astype(np.float32)
    c = _coefficients()
    q = np.full_like(f, c[0])
    for ck in c[1:]:
        q = (q.astype(np.float64) * f + ck).astype(np.float32)   # fma: one rounding
    bits = q.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << np.uint64(23))
    return (bits & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32)


def test_six_coefficients_of_a_degree_five_fit():
    c = _coefficients()
    assert len(c) == 6
    assert abs(c[-1] - 1.0) < 1e-6 and abs(c[-2] - np.log(2)) < 1e-5   # 2^f = 1 + f ln 2 + ...


def test_relative_error_within_the_sfu_bound():
    v = np.linspace(-126.0, 126.0, 2_000_001, dtype=np.float64).astype(np.float32)
    v = np.concatenate([v, np.linspace(-1, 1, 200_001, dtype=np.float32),
                        np.float32([-126, -125.5, -0.5, 0.5, 0.0, 125.5, 126])])
    got = _poly_exp2(v).astype(np.float64)
    want = np.exp2(v.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() < 3e-7


def test_exact_powers_and_clamps():
    ints = np.arange(-126, 127, dtype=np.float32)
    got = _poly_exp2(ints).astype(np.float64)
    assert np.all(np.abs(got / np.exp2(ints.astype(np.float64)) - 1) < 2.5e-7)
    # below the range the result is (within the fit) the smallest normal, above it 2^126
    lo, hi = _poly_exp2(np.float32([-1000.0, 1000.0])).astype(np.float64)
    assert abs(lo / 2.0 ** -126 - 1) < 2.5e-7 and abs(hi / 2.0 ** 126 - 1) < 2.5e-7
