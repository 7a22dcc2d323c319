"""Brute-force pin of the oracle's attention on tiny problems, in arithmetic
that shares nothing with it: the dequantized cache and the query are dyadic
rationals, so logits are exact `Fraction`s; exponentials, tanh and the
softmax are evaluated with Python's `decimal` at 60 significant digits.  The
oracle's fp64 result must agree to about fp64 rounding (1e-13 relative).
Covers GQA, an additive mask with -inf entries, the logit softcap and the
attention sinks."""
import decimal
from fractions import Fraction

import numpy as np
import pytest

from quantized_kv_attention_split_b200 import synthetic as S

decimal.getcontext().prec = 60
Dec = decimal.Decimal


def _dec(fr: Fraction) -> Dec:
    return Dec(fr.numerator) / Dec(fr.denominator)


def _exact_row(qrow, K, V, scale, madd, softcap, sink):
    """softmax over keys of scale*q.k (+ cap, + mask) with an optional sink."""
    logits = []
    for j in range(len(K)):
        if madd is not None and madd[j] == -np.inf:
            logits.append(None)
            continue
        x = _dec(sum((qrow[e] * scale) * K[j][e] for e in range(len(qrow))))
        if softcap:
            c = Dec(repr(softcap))
            t = (Dec(2) * x / c).exp()
            x = c * (t - 1) / (t + 1)
        if madd is not None:
            x += Dec(repr(float(madd[j])))
        logits.append(x)
    vis = [x for x in logits if x is not None]
    if not vis:
        return [Dec(0)] * len(V[0])
    M = max(vis + ([Dec(repr(sink))] if sink is not None else []))
    w = [None if x is None else (x - M).exp() for x in logits]
    den = sum(x for x in w if x is not None)
    if sink is not None:
        den += (Dec(repr(sink)) - M).exp()
    return [sum(w[j] * _dec(V[j][e]) for j in range(len(V)) if w[j] is not None) / den
            for e in range(len(V[0]))]


@pytest.mark.parametrize("fmt,bits,use_mask,softcap,use_sinks", [
    ("affine", 4, False, 0.0, False),
    ("affine", 8, True, 0.0, False),
    ("q8_0", 8, True, 1.5, False),
    ("affine", 3, False, 0.0, True),
    ("affine", 4, True, 2.0, True),
])
def test_attention_against_exact_arithmetic(orc, fmt, bits, use_mask, softcap, use_sinks):
    B, Hq, Hkv, Lq, D, L = 1, 4, 2, 2, 32, 6
    k = S.draw(81, "k", (B, Hkv, L, D), "normal", "f16")
    v = S.draw(81, "v", (B, Hkv, L, D), "normal", "f16")
    q = S.draw(82, "q", (B, Hq, Lq, D), "normal", "f16")
    kc = orc.quantize(k, "f16", fmt, 32, bits)
    vc = orc.quantize(v, "f16", fmt, 32, bits)
    scale = 0.25                                   # a power of two: q*scale exact
    Kd = orc.dequantize(kc, D)                     # fp64 values: exact dyadic rationals
    Vd = orc.dequantize(vc, D)
    qd = orc.to_f64(q, "f16")
    mask = None
    m = None
    if use_mask:
        rng = np.random.default_rng(5)
        m = rng.standard_normal((Lq, L)).astype(np.float32)
        m[0, 2] = -np.inf
        m[1, :] = -np.inf                          # a fully masked row
        mask = orc.Mask("additive", m, "f32", (0, 0, L))
    sinks = np.array([0.5, -1.0, 2.0, 0.0]) if use_sinks else None
    out = orc.attention(q, "f16", kc, vc, L, scale, mask=mask,
                        ext=orc.Ext(softcap=softcap, sinks=sinks))
    G = Hq // Hkv
    for h in range(Hq):
        K = [[Fraction(float(x)) for x in Kd[0, h // G, j]] for j in range(L)]
        V = [[Fraction(float(x)) for x in Vd[0, h // G, j]] for j in range(L)]
        for i in range(Lq):
            qrow = [Fraction(float(x)) for x in qd[0, h, i]]
            want = _exact_row(qrow, K, V, Fraction(scale), None if m is None else m[i],
                              softcap, None if sinks is None else float(sinks[h]))
            got = out[0, h, i]
            for e in range(D):
                w = float(want[e])
                assert abs(got[e] - w) <= 1e-13 * max(1.0, abs(w)), (h, i, e, got[e], w)


def test_values_as_a_view_of_the_keys_exact(orc):
    """The MLA shape (V = the first Dv elements of every K row) on a tiny
    problem, against the same exact arithmetic."""
    B, Hq, Hkv, Lq, Dk, Dv, L = 1, 2, 1, 2, 64, 32, 5
    k = S.draw(83, "k", (B, Hkv, L, Dk), "normal", "f16")
    q = S.draw(84, "q", (B, Hq, Lq, Dk), "normal", "f16")
    kc = orc.quantize(k, "f16", "q8_0")
    Kd = orc.dequantize(kc, Dk)
    qd = orc.to_f64(q, "f16")
    out = orc.attention_kview(q, "f16", kc, L, 0.125, Dv, ext=orc.Ext(sinks=np.array([0.3, -2.0])))
    assert out.shape == (B, Hq, Lq, Dv)
    K = [[Fraction(float(x)) for x in Kd[0, 0, j]] for j in range(L)]
    V = [row[:Dv] for row in K]
    for h in range(Hq):
        for i in range(Lq):
            qrow = [Fraction(float(x)) for x in qd[0, h, i]]
            want = _exact_row(qrow, K, V, Fraction(1, 8), None, 0.0, [0.3, -2.0][h])
            for e in range(Dv):
                assert abs(out[0, h, i, e] - float(want[e])) <= 1e-13 * max(1.0, abs(float(want[e])))


@pytest.mark.parametrize("fmt,bits,causal", [("affine", 4, False), ("q8_0", 8, True),
                                             ("affine", 3, True)])
def test_dense_form_against_exact_arithmetic(orc, fmt, bits, causal):
    """The matrix-product form of the oracle (attention_dense) on the same
    tiny problems, against exact logits and a 60-digit softmax; the causal
    limit is given to the exact side as -inf mask entries."""
    B, Hq, Hkv, Lq, D, L = 1, 4, 2, 3, 32, 6
    k = S.draw(85, "k", (B, Hkv, L, D), "normal", "f16")
    v = S.draw(85, "v", (B, Hkv, L, D), "normal", "f16")
    q = S.draw(86, "q", (B, Hq, Lq, D), "normal", "f16")
    kc = orc.quantize(k, "f16", fmt, 32, bits)
    vc = orc.quantize(v, "f16", fmt, 32, bits)
    Kd, Vd, qd = orc.dequantize(kc, D), orc.dequantize(vc, D), orc.to_f64(q, "f16")
    out = orc.attention_dense(q, "f16", kc, vc, L, 0.5, causal=causal)
    G = Hq // Hkv
    for h in range(Hq):
        K = [[Fraction(float(x)) for x in Kd[0, h // G, j]] for j in range(L)]
        V = [[Fraction(float(x)) for x in Vd[0, h // G, j]] for j in range(L)]
        for i in range(Lq):
            madd = None
            if causal:
                madd = np.array([0.0 if j <= L - Lq + i else -np.inf for j in range(L)])
            qrow = [Fraction(float(x)) for x in qd[0, h, i]]
            want = _exact_row(qrow, K, V, Fraction(1, 2), madd, 0.0, None)
            for e in range(D):
                w = float(want[e])
                assert abs(out[0, h, i, e] - w) <= 1e-13 * max(1.0, abs(w)), (h, i, e)
