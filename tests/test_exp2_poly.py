"""The exponential the tensor-core feature map takes on the FMA pipe (CPU, no GPU).

The kernel computes part of its 2^x values as 2^round(x) * p(x - round(x)) with the cubic p of
csrc/slay_exp2_poly.h.  These tests pin p against numpy's exp2 (not against the fit that
produced it) and restate the kernel's float32 steps to check the range reduction, so a wrong
coefficient, a dropped term or a wrong exponent step fails here before any GPU run.
"""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "kernelized_linear_attention_unit_b200", "csrc", "slay_exp2_poly.h")


def _coeffs():
    txt = open(HDR).read()
    c = [np.float32(float(re.search(r"#define SLAY_EXP2_C%d ([-+0-9.eE]+)f" % k, txt).group(1)))
         for k in range(4)]
    bound = float(re.search(r"#define SLAY_EXP2_MAX_REL_ERR ([-+0-9.eE]+)", txt).group(1))
    return c, bound


def _horner(c, f):
    p = np.full_like(f, c[3])
    for ck in (c[2], c[1], c[0]):
        p = (p * f + ck).astype(np.float32)
    return p


def _ex2_poly(x):
    """The kernel's steps in float32: clamp, round by the 1.5 * 2^23 addition, polynomial of
    the remainder, exponent added to the bit pattern."""
    c, _ = _coeffs()
    x = np.clip(x.astype(np.float32), np.float32(-125.0), np.float32(126.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    f = (x - (t - magic).astype(np.float32)).astype(np.float32)
    p = _horner(c, f)
    bits = (t.view(np.uint32).astype(np.uint64) * np.uint64(8388608) +
            p.view(np.uint32).astype(np.uint64)) & np.uint64(0xFFFFFFFF)
    return bits.astype(np.uint32).view(np.float32)


def test_polynomial_relative_error_on_the_reduced_interval():
    c, bound = _coeffs()
    f = np.linspace(-0.5, 0.5, 400001).astype(np.float32)
    rel = np.abs(_horner(c, f).astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)
    assert rel.max() <= bound * 1.01
    assert bound < 1e-4   # far below bf16's half-ulp (2^-9), the precision the map stores


def test_coefficients_are_near_the_taylor_series():
    c, _ = _coeffs()
    ln2 = np.log(2.0)
    taylor = [1.0, ln2, ln2 ** 2 / 2, ln2 ** 3 / 6]
    for ck, tk in zip(c, taylor):
        assert abs(float(ck) - tk) < 0.02 * max(tk, 0.05)


def test_range_reduction_over_the_whole_exponent_range():
    rng = np.random.default_rng(7)
    x = np.concatenate([rng.uniform(-125.0, 126.0, 200000), np.arange(-125, 126) + 0.5,
                        np.arange(-125, 127).astype(np.float64), [-0.5, 0.5, -1e-8, 1e-8]])
    x32 = x.astype(np.float32)
    got = _ex2_poly(x32).astype(np.float64)
    want = np.exp2(x32.astype(np.float64))
    _, bound = _coeffs()
    # normal results: the polynomial's bound plus the rounding of f
    assert np.max(np.abs(got / want - 1.0)) <= bound + 1e-6


def test_clamped_ends_stay_finite_and_monotone():
    got = _ex2_poly(np.array([-1e30, -200.0, -125.0, 126.0, 200.0, 1e30], dtype=np.float32))
    assert np.all(np.isfinite(got))
    assert got[0] == got[1] == got[2] and got[3] == got[4] == got[5]
    assert 0.0 < got[2] < 1e-37 and got[3] > 1e37
