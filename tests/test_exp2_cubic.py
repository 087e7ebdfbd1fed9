"""The two-lane kernel's optional exp2 on the FMA pipe (a Cody-Waite range
reduction and a cubic), replayed step by step in float32 on the CPU.

The kernel rounds x to n with the 1.5 * 2^23 addition, evaluates
1 + c1 f + c2 f^2 + c3 f^3 on f = x - n in [-1/2, 1/2] and adds n to the result's
exponent field, after clamping x to -127.  The coefficients are read from the
kernel source.  Pinned here: the relative error against 2^x in float64 stays
under 1.1e-4 over the whole range the softmax produces (P is rounded to bf16,
whose half ulp is 2^-9 ~ 2e-3); the cubic's constant term is exactly 1, so
every x at or below -127 (a masked score, -inf) gives exactly +0; integers are
exact; and the coefficients are within 1 % of the error of a freshly solved
minimax problem (a linear program on a grid), so a mistyped digit fails.
"""
import os
import re

import numpy as np
import pytest

SRC = os.path.join(os.path.dirname(__file__), "..", "gqa_attention_forward_flash_b200", "csrc", "gqa_fwd2_kernel.cuh")


def _coeffs():
    text = open(SRC).read()
    c = []
    for name in ("kExp2C1", "kExp2C2", "kExp2C3"):
        m = re.search(r"constexpr float %s = ([0-9.eE+-]+)f;" % name, text)
        assert m, name
        c.append(np.float32(float(m.group(1))))
    m = re.search(r"constexpr float kRoundMagic = ([0-9.eE+-]+)f;", text)
    assert m
    return c, np.float32(float(m.group(1)))


def _cubic_exp2(x):
    (c1, c2, c3), magic = _coeffs()
    x = np.maximum(np.asarray(x, np.float32), np.float32(-127.0))
    j = (x + magic).astype(np.float32)
    f = (x - (j - magic).astype(np.float32)).astype(np.float32)
    q = (c3 * f + c2).astype(np.float32)
    q = (q * f + c1).astype(np.float32)
    q = (q * f + np.float32(1.0)).astype(np.float32)
    bits = q.view(np.uint32) + (j.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


def test_relative_error_over_the_softmax_range():
    x = np.linspace(-126.0, 40.0, 3_000_001).astype(np.float32)
    got = _cubic_exp2(x).astype(np.float64)
    rel = np.abs(got / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 1.1e-4, rel.max()


def test_masked_scores_give_exact_zero():
    x = np.array([-np.inf, -1e30, -300.0, -128.0, -127.0], np.float32)
    got = _cubic_exp2(x)
    assert np.all(got == 0.0) and not np.any(np.signbit(got))


def test_integers_are_exact():
    n = np.arange(-126, 41, dtype=np.float32)
    assert np.array_equal(_cubic_exp2(n), np.exp2(n.astype(np.float64)).astype(np.float32))


def test_coefficients_are_near_the_minimax_optimum():
    scipy_opt = pytest.importorskip("scipy.optimize")
    f = np.linspace(-0.5, 0.5, 4001)
    t = np.exp2(f)
    a = np.stack([f / t, f ** 2 / t, f ** 3 / t], 1)
    a_ub = np.vstack([np.hstack([a, -np.ones((len(f), 1))]), np.hstack([-a, -np.ones((len(f), 1))])])
    b_ub = np.concatenate([1 - 1 / t, -(1 - 1 / t)])
    res = scipy_opt.linprog([0, 0, 0, 1], A_ub=a_ub, b_ub=b_ub, bounds=[(None, None)] * 3 + [(0, None)])
    assert res.status == 0
    (c1, c2, c3), _ = _coeffs()
    p = 1 + float(c1) * f + float(c2) * f ** 2 + float(c3) * f ** 3
    err = np.abs(p / t - 1).max()
    assert err <= res.x[3] * 1.01, (err, res.x[3])
