"""Pins for the fp64 oracle, independent of the oracle's own code.

Each test checks the oracle against something the mathematics or the pages fix:
hand-computed values, closed forms of special cases, invariances of softmax
attention, and a high-precision brute force on tiny inputs.  A plausible slip
in the oracle (a dropped sink term, a causal off-by-one, a wrong head mapping,
a transposed operand, double normalisation, scale applied to the sink, padded
rows leaking in) fails at least one of them; ``test_planted_mistakes`` checks
that claim on mutated copies of the oracle source.
"""
import math
import os
import re
import subprocess
import tempfile
from decimal import Decimal, getcontext
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_two_keys.txt")


def bf(x):
    return torch.tensor(x, dtype=torch.float32).to(torch.bfloat16)


def rnd(shape, seed, sigma=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * sigma).to(torch.bfloat16)


def f64(t):
    return t.to(torch.float64).numpy()


# --------------------------------------------------------------------------
# hand-computed golden values
# --------------------------------------------------------------------------

def _parse_num(s):
    s = s.strip()
    if s == "-inf":
        return -math.inf
    if s.startswith("ln"):
        return math.log(float(s[2:]))
    return float(s)


def _golden_cases():
    cases = []
    for line in open(GOLDEN):
        if line.startswith("#") or not line.strip():
            continue
        name, tq, n, causal, sink, orows, lrows = [x.strip() for x in line.split("|")]
        o = [[_parse_num(x) for x in r.split()] for r in orows.split(";")]
        l = [_parse_num(x) for x in lrows.split(";")]
        cases.append((name, int(tq), int(n), int(causal), sink, o, l))
    return cases


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c[0])
def test_hand_computed(case):
    name, Tq, n, causal, sink, o_exp, l_exp = case
    q = bf([[[[1.0, 0.0]] * Tq]])
    k = bf([[[[1.0, 0.0], [0.0, 1.0]]]])
    v = bf([[[[4.0, 0.0], [0.0, 4.0]]]])
    kv = np.array([n], np.int32)
    sk = None if sink == "none" else np.array([_parse_num(sink)], np.float32)
    out, lse = oracle.attention(q, k, v, kv, sk, scale=math.log(3.0), causal=bool(causal))
    # the sink is stored as float32 (it is a float32 argument of the API)
    tol = 1e-6 if sk is not None else 1e-12
    np.testing.assert_allclose(out[0, 0], np.array(o_exp), rtol=tol, atol=tol)
    for got, exp in zip(lse[0, 0], l_exp):
        if exp == -math.inf:
            assert got == -math.inf
        else:
            assert abs(got - exp) < tol


# --------------------------------------------------------------------------
# closed forms of special cases
# --------------------------------------------------------------------------

def test_single_key_returns_its_value():
    q, k, v = rnd((2, 4, 3, 16), 1), rnd((2, 2, 1, 16), 2), rnd((2, 2, 1, 16), 3)
    out, lse = oracle.attention(q, k, v, None, None, scale=0.37, causal=False)
    for b in range(2):
        for h in range(4):
            g = h // 2
            for i in range(3):
                np.testing.assert_array_equal(out[b, h, i], f64(v[b, g, 0]))
                s = 0.37 * float(np.dot(f64(q[b, h, i]), f64(k[b, g, 0])))
                assert abs(lse[b, h, i] - s) < 1e-12


def test_two_keys_is_a_sigmoid_blend():
    q, k, v = rnd((1, 2, 2, 8), 4), rnd((1, 1, 2, 8), 5), rnd((1, 1, 2, 8), 6)
    out, lse = oracle.attention(q, k, v, None, None, scale=0.5, causal=False)
    for h in range(2):
        for i in range(2):
            s0 = 0.5 * float(np.dot(f64(q[0, h, i]), f64(k[0, 0, 0])))
            s1 = 0.5 * float(np.dot(f64(q[0, h, i]), f64(k[0, 0, 1])))
            w0 = 1.0 / (1.0 + math.exp(s1 - s0))
            np.testing.assert_allclose(out[0, h, i], w0 * f64(v[0, 0, 0]) + (1 - w0) * f64(v[0, 0, 1]),
                                       rtol=1e-12, atol=1e-12)
            assert abs(lse[0, h, i] - np.logaddexp(s0, s1)) < 1e-12


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("with_sink", [False, True])
def test_zero_query_averages_visible_values(causal, with_sink):
    """Q = 0 makes every visible logit 0: O is the mean of the visible V rows
    (shrunk by the sink weight), lse = ln(#visible [+ e^sink])."""
    B, Hq, Hkv, Tq, Tkv, d = 2, 6, 3, 5, 11, 8
    q = torch.zeros((B, Hq, Tq, d), dtype=torch.bfloat16)
    k, v = rnd((B, Hkv, Tkv, d), 7), rnd((B, Hkv, Tkv, d), 8)
    kv = np.array([9, 4], np.int32)
    sink = np.array([0.3, -1.0, 2.0, 0.0, -0.5, 1.5], np.float32) if with_sink else None
    out, lse = oracle.attention(q, k, v, kv, sink, scale=0.9, causal=causal)
    for b in range(B):
        n = int(kv[b])
        for h in range(Hq):
            g = h // (Hq // Hkv)
            for i in range(Tq):
                cnt = min(n, n - Tq + i + 1) if causal else n
                cnt = max(cnt, 0)
                extra = math.exp(float(sink[h])) if with_sink else 0.0
                z = cnt + extra
                if z == 0:
                    assert lse[b, h, i] == -math.inf
                    np.testing.assert_array_equal(out[b, h, i], 0.0)
                    continue
                exp_o = f64(v[b, g, :cnt]).sum(0) / z if cnt else np.zeros(d)
                np.testing.assert_allclose(out[b, h, i], exp_o, rtol=1e-12, atol=1e-12)
                assert abs(lse[b, h, i] - math.log(z)) < 1e-12


def test_constant_value_rows_return_that_row():
    """Catches double normalisation (dsv4 attention commit log: P normalised
    twice shrank O by the row sum)."""
    B, Hq, Hkv, Tq, Tkv, d = 1, 4, 2, 7, 33, 16
    q, k = rnd((B, Hq, Tq, d), 9, 2.0), rnd((B, Hkv, Tkv, d), 10, 2.0)
    row = rnd((d,), 11)
    v = row.expand(B, Hkv, Tkv, d).contiguous()
    out, _ = oracle.attention(q, k, v, None, None, scale=0.25, causal=True)
    np.testing.assert_allclose(out, np.broadcast_to(f64(row), out.shape), rtol=1e-12, atol=1e-12)


def test_peaked_query_selects_one_value():
    B, Hq, Hkv, Tkv, d = 1, 2, 1, 9, 16
    k = torch.eye(Tkv, d, dtype=torch.float32)[None, None].to(torch.bfloat16)
    v = rnd((B, Hkv, Tkv, d), 12)
    # q = 64 * k_5 with scale 1: logit 64 for key 5, 0 elsewhere
    q = (64.0 * k[:, :, 5:6, :].float()).expand(B, Hq, 1, d).contiguous().to(torch.bfloat16)
    out, lse = oracle.attention(q, k, v, None, None, scale=1.0, causal=False)
    w_other = math.exp(-64.0)
    for h in range(Hq):
        exp_o = (f64(v[0, 0, 5]) + w_other * (f64(v[0, 0]).sum(0) - f64(v[0, 0, 5]))) / (1 + 8 * w_other)
        np.testing.assert_allclose(out[0, h, 0], exp_o, rtol=1e-12, atol=1e-14)
        assert abs(lse[0, h, 0] - (64.0 + math.log1p(8 * w_other))) < 1e-12


# --------------------------------------------------------------------------
# invariances
# --------------------------------------------------------------------------

def test_key_permutation_invariance():
    B, Hq, Hkv, Tq, Tkv, d = 2, 4, 2, 3, 19, 16
    q, k, v = rnd((B, Hq, Tq, d), 13), rnd((B, Hkv, Tkv, d), 14), rnd((B, Hkv, Tkv, d), 15)
    perm = torch.randperm(Tkv, generator=torch.Generator().manual_seed(0))
    o1, l1 = oracle.attention(q, k, v, None, None, scale=0.3, causal=False)
    o2, l2 = oracle.attention(q, k[:, :, perm], v[:, :, perm], None, None, scale=0.3, causal=False)
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l1, l2, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_gqa_equals_mha_with_repeated_kv(causal):
    """Query head h reads KV head floor(h / G) (contiguous grouping)."""
    B, Hq, Hkv, Tq, Tkv, d = 2, 8, 2, 4, 13, 16
    q, k, v = rnd((B, Hq, Tq, d), 16), rnd((B, Hkv, Tkv, d), 17), rnd((B, Hkv, Tkv, d), 18)
    kv = np.array([13, 6], np.int32)
    sink = np.linspace(-1, 1, Hq).astype(np.float32)
    G = Hq // Hkv
    o1, l1 = oracle.attention(q, k, v, kv, sink, scale=0.2, causal=causal)
    o2, l2 = oracle.attention(q, k.repeat_interleave(G, 1), v.repeat_interleave(G, 1), kv, sink,
                              scale=0.2, causal=causal)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)
    # G = 1 with explicit per-head KV is the MHA case: head h uses KV head h
    o3, _ = oracle.attention(q[:, 3:4], k[:, 0:1], v[:, 0:1], kv, sink[3:4], scale=0.2, causal=causal)
    np.testing.assert_array_equal(o1[:, 3:4], o3)


def test_sink_minus_infinity_is_a_no_op():
    B, Hq, Hkv, Tq, Tkv, d = 1, 4, 1, 5, 17, 8
    q, k, v = rnd((B, Hq, Tq, d), 19), rnd((B, Hkv, Tkv, d), 20), rnd((B, Hkv, Tkv, d), 21)
    sink = np.full(Hq, -np.inf, np.float32)
    for causal in (False, True):
        o1, l1 = oracle.attention(q, k, v, None, None, scale=0.4, causal=causal)
        o2, l2 = oracle.attention(q, k, v, None, sink, scale=0.4, causal=causal)
        np.testing.assert_array_equal(o1, o2)
        np.testing.assert_array_equal(l1, l2)


def test_sink_is_in_the_scaled_domain():
    """Doubling `scale` must not change the sink's weight (dsv4 attention commit
    log, sink commit: the sink is compared with max(QK*scale) without another
    multiplication by scale).  With q = 0 every logit is 0 whatever the scale."""
    q = torch.zeros((1, 1, 1, 4), dtype=torch.bfloat16)
    k, v = rnd((1, 1, 3, 4), 22), rnd((1, 1, 3, 4), 23)
    sink = np.array([1.25], np.float32)
    o1, l1 = oracle.attention(q, k, v, None, sink, scale=0.5, causal=False)
    o2, l2 = oracle.attention(q, k, v, None, sink, scale=1.0, causal=False)
    np.testing.assert_array_equal(o1, o2)
    assert abs(l1[0, 0, 0] - math.log(3 + math.exp(1.25))) < 1e-12


def test_padded_rows_have_no_effect():
    """Rows at positions >= kv_len (NaN, inf, or other values) change nothing
    (dsv4 attention commit log, logical vs padded N)."""
    B, Hq, Hkv, Tq, Tkv, d = 2, 4, 2, 3, 20, 8
    q, k, v = rnd((B, Hq, Tq, d), 24), rnd((B, Hkv, Tkv, d), 25), rnd((B, Hkv, Tkv, d), 26)
    kv = np.array([11, 20], np.int32)
    o1, l1 = oracle.attention(q, k, v, kv, None, scale=0.3, causal=True)
    k2, v2 = k.clone(), v.clone()
    k2[0, :, 11:] = float("nan")
    v2[0, :, 11:] = float("inf")
    o2, l2 = oracle.attention(q, k2, v2, kv, None, scale=0.3, causal=True)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)
    # and equals a buffer that simply ends at kv_len
    o3, l3 = oracle.attention(q[0:1], k[0:1, :, :11], v[0:1, :, :11], None, None, scale=0.3, causal=True)
    np.testing.assert_array_equal(o1[0:1], o3)
    np.testing.assert_array_equal(l1[0:1], l3)


def test_logit_shift_invariance():
    """One extra feature with q_extra = c and k_extra = 1 adds scale*c to every
    logit of a row: O is unchanged and lse moves by exactly scale*c."""
    B, Hq, Hkv, Tq, Tkv, d = 1, 2, 1, 4, 10, 7
    q, k, v = rnd((B, Hq, Tq, d), 27), rnd((B, Hkv, Tkv, d), 28), rnd((B, Hkv, Tkv, d), 29)
    c = 3.0
    q2 = torch.cat([q, torch.full((B, Hq, Tq, 1), c).to(torch.bfloat16)], -1)
    k2 = torch.cat([k, torch.ones((B, Hkv, Tkv, 1)).to(torch.bfloat16)], -1)
    v2 = torch.cat([v, torch.zeros((B, Hkv, Tkv, 1)).to(torch.bfloat16)], -1)
    o1, l1 = oracle.attention(q, k, v, None, None, scale=0.5, causal=True)
    o2, l2 = oracle.attention(q2, k2, v2, None, None, scale=0.5, causal=True)
    np.testing.assert_allclose(o2[..., :d], o1, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l2, l1 + 0.5 * c, rtol=1e-12, atol=1e-12)


def test_causal_square_is_lower_triangular():
    """With Tq = kv_len the bottom-right causal mask is the usual i >= j mask."""
    B, Hq, Hkv, T, d = 1, 1, 1, 6, 4
    q, k, v = rnd((B, Hq, T, d), 30), rnd((B, Hkv, T, d), 31), rnd((B, Hkv, T, d), 32)
    out, _ = oracle.attention(q, k, v, None, None, scale=0.7, causal=True)
    for i in range(T):
        o_i, _ = oracle.attention(q[:, :, i:i + 1], k[:, :, :i + 1], v[:, :, :i + 1], None, None,
                                  scale=0.7, causal=False)
        np.testing.assert_allclose(out[0, 0, i], o_i[0, 0, 0], rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------------------
# split + merge (associativity of the (m, l, O) merge)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("causal,with_sink", [(False, False), (True, False), (True, True)])
def test_window_splits_merge_to_the_full_result(causal, with_sink):
    B, Hq, Hkv, Tq, Tkv, d = 2, 4, 2, 3, 23, 8
    q, k, v = rnd((B, Hq, Tq, d), 33), rnd((B, Hkv, Tkv, d), 34), rnd((B, Hkv, Tkv, d), 35)
    kv = np.array([23, 9], np.int32)
    sink = np.array([0.5, -0.25, 1.0, 0.0], np.float32) if with_sink else None
    full_o, full_l = oracle.attention(q, k, v, kv, sink, scale=0.6, causal=causal)
    for cuts in ([0, 23], [0, 5, 23], [0, 1, 2, 12, 20, 23], [0, 10, 10, 23]):
        parts_o, parts_l = [], []
        for a, b in zip(cuts[:-1], cuts[1:]):
            o, l = oracle.attention_window(q, k, v, kv, None, 0.6, causal, a, b)
            parts_o.append(o)
            parts_l.append(l)
        po = np.stack(parts_o, 3).astype(np.float32)
        pl = np.stack(parts_l, 3).astype(np.float32)
        mo, ml = oracle.combine(po, pl, sink)
        np.testing.assert_allclose(mo, full_o, rtol=2e-6, atol=2e-6)
        fin = np.isfinite(full_l)
        np.testing.assert_allclose(ml[fin], full_l[fin], rtol=2e-6, atol=2e-6)
        assert np.all(ml[~fin] == -np.inf)


def test_combine_of_one_partial_is_that_partial():
    o = np.random.default_rng(0).standard_normal((1, 2, 3, 1, 5)).astype(np.float32)
    l = np.random.default_rng(1).standard_normal((1, 2, 3, 1)).astype(np.float32)
    mo, ml = oracle.combine(o, l, None)
    np.testing.assert_array_equal(mo, o[:, :, :, 0].astype(np.float64))
    np.testing.assert_allclose(ml, l[..., 0].astype(np.float64), rtol=0, atol=1e-15)


def test_combine_ignores_empty_partials():
    o = np.random.default_rng(2).standard_normal((1, 1, 2, 3, 4)).astype(np.float32)
    l = np.random.default_rng(3).standard_normal((1, 1, 2, 3)).astype(np.float32)
    l[..., 1] = -np.inf
    o[..., 1, :] = 0.0
    mo, ml = oracle.combine(o, l, None)
    mo2, ml2 = oracle.combine(o[..., [0, 2], :], l[..., [0, 2]], None)
    np.testing.assert_allclose(mo, mo2, rtol=1e-15, atol=1e-15)
    np.testing.assert_allclose(ml, ml2, rtol=1e-15, atol=1e-15)


def test_rows_entry_matches_full_entry():
    B, Hq, Hkv, Tq, Tkv, d = 2, 4, 2, 5, 30, 8
    q, k, v = rnd((B, Hq, Tq, d), 36), rnd((B, Hkv, Tkv, d), 37), rnd((B, Hkv, Tkv, d), 38)
    kv = np.array([30, 3], np.int32)
    sink = np.array([0.1, 0.2, 0.3, 0.4], np.float32)
    full_o, full_l = oracle.attention(q, k, v, kv, sink, scale=0.3, causal=True)
    rows = np.array([0, 7, 19, 20, 33, 39])
    ro, rl = oracle.attention_rows(q, k, v, kv, sink, 0.3, True, rows)
    np.testing.assert_array_equal(ro, full_o.reshape(-1, d)[rows])
    np.testing.assert_array_equal(rl, full_l.reshape(-1)[rows])


# --------------------------------------------------------------------------
# brute force at 50 significant digits on tiny inputs
# --------------------------------------------------------------------------

def _brute_force(q, k, v, kv, sink, scale, causal):
    getcontext().prec = 50
    qf, kf, vf = f64(q), f64(k), f64(v)
    B, Hq, Tq, d = qf.shape
    Hkv, Tkv = kf.shape[1], kf.shape[2]
    G = Hq // Hkv
    out = np.zeros((B, Hq, Tq, d))
    lse = np.zeros((B, Hq, Tq))
    sc = Fraction(scale)
    for b in range(B):
        n = Tkv if kv is None else int(kv[b])
        for h in range(Hq):
            g = h // G
            for i in range(Tq):
                js = [j for j in range(n) if (not causal or j <= n - Tq + i)]
                logits = []
                for j in js:
                    dot = sum(Fraction(float(qf[b, h, i, c])) * Fraction(float(kf[b, g, j, c]))
                              for c in range(d))
                    logits.append(Decimal(sc.numerator) / Decimal(sc.denominator)
                                  * (Decimal(dot.numerator) / Decimal(dot.denominator)))
                ws = [x.exp() for x in logits]
                z = sum(ws, Decimal(0))
                if sink is not None:
                    z += Decimal(float(sink[h])).exp()
                for c in range(d):
                    num = sum((w * Decimal(float(vf[b, g, j, c])) for w, j in zip(ws, js)), Decimal(0))
                    out[b, h, i, c] = float(num / z)
                lse[b, h, i] = float(z.ln())
    return out, lse


@pytest.mark.parametrize("causal,with_sink", [(False, False), (True, True)])
def test_brute_force_high_precision(causal, with_sink):
    B, Hq, Hkv, Tq, Tkv, d = 2, 4, 2, 3, 7, 5
    q, k, v = rnd((B, Hq, Tq, d), 40, 2.0), rnd((B, Hkv, Tkv, d), 41, 2.0), rnd((B, Hkv, Tkv, d), 42)
    kv = np.array([7, 4], np.int32)
    sink = np.array([0.7, -0.3, 2.5, -2.0], np.float32) if with_sink else None
    o, l = oracle.attention(q, k, v, kv, sink, scale=0.45, causal=causal)
    bo, bl = _brute_force(q, k, v, kv, sink, 0.45, causal)
    np.testing.assert_allclose(o, bo, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l, bl, rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------------------
# the pins catch planted mistakes (mutations of a private copy of the oracle)
# --------------------------------------------------------------------------

MUTATIONS = {
    "causal_off_by_one": ("long last = causal ? (n - Tq + i) : (n - 1);",
                          "long last = causal ? (n - Tq + i - 1) : (n - 1);"),
    "head_mapping_modulo": ("const int g = h / G;", "const int g = h % Hkv;"),
    "sink_dropped_from_z": ("if (has_sink) Z += exp(sk - M);", "(void)0;"),
    "sink_scaled_again": ("const double sk = has_sink ? (double)sink[h] : -INFINITY;",
                          "const double sk = has_sink ? scale * (double)sink[h] : -INFINITY;"),
    "double_normalisation": ("for (int c = 0; c < d; ++c) o_row[c] /= Z;",
                             "for (int c = 0; c < d; ++c) o_row[c] /= Z * Z;"),
    "padded_length_used": ("long n = kv_lens ? (long)kv_lens[b] : (long)Tkv;", "long n = (long)Tkv;"),
    "k_transposed_index": ("const long kr = kb + j * (long)d;",
                           "const long kr = kb + (j % d) * (long)d;"),
    # the E4M3 decoder of the FP8 K/V path
    "e4m3_bias_8": ("v = ldexp(1.0 + (double)m / 8.0, e - 7);", "v = ldexp(1.0 + (double)m / 8.0, e - 8);"),
    "e4m3_subnormal_exponent": ("v = ldexp((double)m / 8.0, -6);", "v = ldexp((double)m / 8.0, -7);"),
    "e4m3_no_nan_code": ("else if (e == 15 && m == 7)\n        return NAN;", "else if (0)\n        return NAN;"),
    "fp8_v_scale_dropped": ("* s->v_scale", "* 1.0"),
    "fp8_k_scale_on_v": ("e4m3_to_double(((const uint8_t *)s->v)[idx]) * s->v_scale",
                         "e4m3_to_double(((const uint8_t *)s->v)[idx]) * s->k_scale"),
}


@pytest.mark.parametrize("mutation", sorted(MUTATIONS))
def test_planted_mistakes_are_caught(mutation, tmp_path):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "gqa_oracle.c")).read()
    old, new = MUTATIONS[mutation]
    assert old in src, mutation
    mutated = tmp_path / "m.c"
    mutated.write_text(src.replace(old, new))
    so = tmp_path / "m.so"
    subprocess.check_call(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", str(mutated), "-o", str(so), "-lm"])
    import importlib.util
    spec = importlib.util.spec_from_file_location("oracle_mut_%s" % mutation,
                                                  os.path.join(os.path.dirname(oracle.__file__), "__init__.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod._LIB = str(so)
    mod.build = lambda force=False: str(so)
    mod._lib = None
    real = oracle
    failures = 0
    pins = [
        lambda: _pin_golden(mod),
        lambda: _pin_zero_query(mod),
        lambda: _pin_gqa(mod),
        lambda: _pin_padded(mod),
        lambda: _pin_constant_v(mod),
        lambda: _pin_brute(mod),
        lambda: _pin_e4m3_table(mod),
        lambda: _pin_fp8kv_equals_dequantised(mod),
    ]
    for pin in pins:
        try:
            pin()
        except AssertionError:
            failures += 1
    assert real is oracle
    assert failures > 0, "mutation %s was not caught by any pin" % mutation


def _pin_golden(mod):
    for case in _golden_cases():
        name, Tq, n, causal, sink, o_exp, l_exp = case
        q = bf([[[[1.0, 0.0]] * Tq]])
        k = bf([[[[1.0, 0.0], [0.0, 1.0]]]])
        v = bf([[[[4.0, 0.0], [0.0, 4.0]]]])
        sk = None if sink == "none" else np.array([_parse_num(sink)], np.float32)
        out, lse = mod.attention(q, k, v, np.array([n], np.int32), sk, scale=math.log(3.0),
                                 causal=bool(causal))
        np.testing.assert_allclose(out[0, 0], np.array(o_exp), rtol=1e-6, atol=1e-6)
        np.testing.assert_allclose(lse[0, 0], np.array(l_exp), rtol=1e-6, atol=1e-6)


def _pin_zero_query(mod):
    B, Hq, Hkv, Tq, Tkv, d = 1, 4, 2, 5, 9, 4
    q = torch.zeros((B, Hq, Tq, d), dtype=torch.bfloat16)
    k, v = rnd((B, Hkv, Tkv, d), 7), rnd((B, Hkv, Tkv, d), 8)
    sink = np.array([0.3, -1.0, 2.0, 0.0], np.float32)
    out, lse = mod.attention(q, k, v, np.array([8], np.int32), sink, scale=0.9, causal=True)
    for h in range(Hq):
        for i in range(Tq):
            cnt = 8 - Tq + i + 1
            z = cnt + math.exp(float(sink[h]))
            np.testing.assert_allclose(out[0, h, i], f64(v[0, h // 2, :cnt]).sum(0) / z, rtol=1e-9, atol=1e-12)
            assert abs(lse[0, h, i] - math.log(z)) < 1e-9


def _pin_gqa(mod):
    B, Hq, Hkv, Tq, Tkv, d = 1, 4, 2, 2, 5, 4
    q, k, v = rnd((B, Hq, Tq, d), 16), rnd((B, Hkv, Tkv, d), 17), rnd((B, Hkv, Tkv, d), 18)
    o1, _ = mod.attention(q, k, v, None, None, scale=0.2, causal=False)
    o2, _ = oracle.attention(q, k.repeat_interleave(2, 1), v.repeat_interleave(2, 1), None, None,
                             scale=0.2, causal=False)
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-13)


def _pin_padded(mod):
    B, Hq, Hkv, Tq, Tkv, d = 1, 2, 1, 2, 8, 4
    q, k, v = rnd((B, Hq, Tq, d), 24), rnd((B, Hkv, Tkv, d), 25), rnd((B, Hkv, Tkv, d), 26)
    o1, _ = mod.attention(q, k, v, np.array([5], np.int32), None, scale=0.3, causal=True)
    o3, _ = oracle.attention(q, k[:, :, :5], v[:, :, :5], None, None, scale=0.3, causal=True)
    np.testing.assert_allclose(o1, o3, rtol=1e-12, atol=1e-13)


def _pin_constant_v(mod):
    q, k = rnd((1, 2, 3, 8), 9, 2.0), rnd((1, 1, 6, 8), 10, 2.0)
    row = rnd((8,), 11)
    v = row.expand(1, 1, 6, 8).contiguous()
    out, _ = mod.attention(q, k, v, None, None, scale=0.25, causal=True)
    np.testing.assert_allclose(out, np.broadcast_to(f64(row), out.shape), rtol=1e-12, atol=1e-12)


def _pin_brute(mod):
    B, Hq, Hkv, Tq, Tkv, d = 1, 2, 1, 2, 12, 3
    q, k, v = rnd((B, Hq, Tq, d), 40, 2.0), rnd((B, Hkv, Tkv, d), 41, 2.0), rnd((B, Hkv, Tkv, d), 42)
    kv = np.array([12], np.int32)
    o, l = mod.attention(q, k, v, kv, None, scale=0.45, causal=True)
    bo, bl = _brute_force(q, k, v, kv, None, 0.45, True)
    np.testing.assert_allclose(o, bo, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l, bl, rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------------------
# FP8 (E4M3) K/V: the decoder and the attention on dequantised values
# --------------------------------------------------------------------------

# bytes whose values follow directly from the format definition (sign, 4-bit
# exponent with bias 7, 3-bit mantissa; exponent field 0 is subnormal with
# exponent -6; exponent 15 with mantissa 7 is NaN; no infinities)
E4M3_HAND = {0x00: 0.0, 0x38: 1.0, 0xB8: -1.0, 0x3C: 1.5, 0x40: 2.0, 0x7E: 448.0, 0xFE: -448.0,
             0x08: 2.0 ** -6, 0x07: 7 * 2.0 ** -9, 0x01: 2.0 ** -9, 0x30: 0.5, 0x77: 240.0}


def _pin_e4m3_table(mod):
    codes = np.array(sorted(E4M3_HAND), np.uint8)
    np.testing.assert_array_equal(mod.e4m3_decode(codes), np.array([E4M3_HAND[c] for c in sorted(E4M3_HAND)]))
    assert np.isnan(mod.e4m3_decode(np.array([0x7F, 0xFF], np.uint8))).all()


def test_e4m3_decoder_hand_values():
    _pin_e4m3_table(oracle)


def test_e4m3_decoder_matches_torch_for_every_byte():
    """The oracle's decoder, written from the format definition, against torch's
    float8_e4m3fn -> float64 conversion (a library routine) on all 256 bytes."""
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    same = (ours == ref) | (np.isnan(ours) & np.isnan(ref))
    assert same.all(), codes[~same]


def _fp8_case(seed, B=2, Hq=8, Hkv=2, Tq=3, Tkv=40, d=16):
    g = torch.Generator().manual_seed(seed)
    k8 = (torch.randn((B, Hkv, Tkv, d), generator=g) * 60).to(torch.float8_e4m3fn)
    v8 = (torch.randn((B, Hkv, Tkv, d), generator=g) * 60).to(torch.float8_e4m3fn)
    q = rnd((B, Hq, Tq, d), seed + 1)
    return q, k8, v8


def _pin_fp8kv_equals_dequantised(mod):
    """With power-of-two scales every dequantised value is exactly a bf16, so the
    FP8 K/V attention must equal the bf16 attention on those values."""
    q, k8, v8 = _fp8_case(31)
    ks, vs = 2.0 ** -6, 2.0 ** -5
    kv = np.array([40, 17], np.int32)
    sink = np.linspace(-1, 1, 8).astype(np.float32)
    kd = torch.from_numpy(mod.e4m3_decode(k8) * ks).to(torch.bfloat16)
    vd = torch.from_numpy(mod.e4m3_decode(v8) * vs).to(torch.bfloat16)
    assert np.array_equal(kd.double().numpy(), mod.e4m3_decode(k8) * ks)  # exactly representable
    o8, l8 = mod.attention_fp8kv(q, k8, v8, ks, vs, kv, sink, scale=0.3, causal=True)
    ob, lb = mod.attention(q, kd, vd, kv, sink, scale=0.3, causal=True)
    np.testing.assert_array_equal(o8, ob)
    np.testing.assert_array_equal(l8, lb)


def test_fp8kv_equals_bf16_on_dequantised_values():
    _pin_fp8kv_equals_dequantised(oracle)


def test_fp8kv_scales():
    """v_scale multiplies O and leaves lse alone; k_scale acts as a factor of the
    logit scale."""
    q, k8, v8 = _fp8_case(33)
    o1, l1 = oracle.attention_fp8kv(q, k8, v8, 0.01, 0.02, None, None, scale=0.5)
    o2, l2 = oracle.attention_fp8kv(q, k8, v8, 0.01, 0.06, None, None, scale=0.5)
    np.testing.assert_allclose(o2, 3 * o1, rtol=1e-13, atol=1e-15)
    np.testing.assert_array_equal(l1, l2)
    o3, l3 = oracle.attention_fp8kv(q, k8, v8, 0.03, 0.02, None, None, scale=0.5 / 3)
    np.testing.assert_allclose(o3, o1, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(l3, l1, rtol=1e-12, atol=1e-12)


def test_fp8kv_padded_nan_bytes_have_no_effect():
    q, k8, v8 = _fp8_case(35)
    kv = np.array([23, 40], np.int32)
    o1, l1 = oracle.attention_fp8kv(q, k8, v8, 0.01, 0.02, kv, None, scale=0.5, causal=True)
    k8n, v8n = k8.clone().view(torch.uint8), v8.clone().view(torch.uint8)
    k8n[0, :, 23:] = 0x7F
    v8n[0, :, 23:] = 0xFF
    o2, l2 = oracle.attention_fp8kv(q, k8n, v8n, 0.01, 0.02, kv, None, scale=0.5, causal=True)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_fp8kv_rows_entry_matches_full_entry():
    q, k8, v8 = _fp8_case(37)
    kv = np.array([40, 9], np.int32)
    o, l = oracle.attention_fp8kv(q, k8, v8, 0.015, 0.025, kv, None, scale=0.4, causal=True)
    rows = np.array([0, 5, 17, 30, 47], np.int64)
    orow, lrow = oracle.attention_rows_fp8kv(q, k8, v8, 0.015, 0.025, kv, None, 0.4, True, rows)
    np.testing.assert_array_equal(orow, o.reshape(-1, o.shape[-1])[rows])
    np.testing.assert_array_equal(lrow, l.reshape(-1)[rows])
