"""Pins for the oracle's attention extensions (CPU only): logit softcap,
attention sinks and per-head slopes on the additive mask (ALiBi).

The llama.cpp PR ("Metal: Optimize q8_0 KV" and its follow-up) lists these
among the attention variants its tests cover but prints no formula, so the
oracle takes their usual definitions (stated in qkv_oracle.cpp).  They are
pinned here by what those definitions fix without the oracle's code:
 * a sink behaves exactly like one more key whose logit is the sink and whose
   value row is zero (built as a real cache row: constant groups dequantize
   exactly);
 * closed forms with a zero query (every logit 0) or with constant key rows
   (every logit known analytically);
 * limits: softcap -> infinity is plain attention, sink -> -inf is no sink;
 * a slope on the additive mask equals the same mask multiplied beforehand
   (that path is pinned against torch's SDPA in test_oracle_attention.py).
"""
import math

import numpy as np
import pytest

from quantized_kv_attention_split_b200 import synthetic as S


def _cache(orc, B, Hkv, L, D, fmt, bits, gs, seed, dist="normal"):
    k = S.draw(seed, "k", (B, Hkv, L, D), dist, "f16")
    v = S.draw(seed, "v", (B, Hkv, L, D), dist, "f16")
    return orc.quantize(k, "f16", fmt, gs, bits), orc.quantize(v, "f16", fmt, gs, bits)


MODES = (("two_pass", 1), ("online", 1), ("split", 3))


def test_sink_is_a_key_with_zero_value(orc):
    B, Hq, Hkv, D, L = 1, 4, 2, 64, 29
    G = Hq // Hkv
    # L ordinary keys plus one extra key row (index L) that is constant along
    # D, with a zero value row: both reconstruct exactly.
    k = S.draw(21, "k", (B, Hkv, L + 1, D), "normal", "f16")
    v = S.draw(21, "v", (B, Hkv, L + 1, D), "normal", "f16")
    a = np.float16(0.75)
    k[:, :, L, :] = np.full(D, a).view(np.uint16)
    v[:, :, L, :] = 0
    kc = orc.quantize(k, "f16", "affine", 64, 4)
    vc = orc.quantize(v, "f16", "affine", 64, 4)
    assert np.all(orc.dequantize(kc, D)[:, :, L] == 0.75)
    assert np.all(orc.dequantize(vc, D)[:, :, L] == 0.0)
    q = S.draw(22, "q", (B, Hq, 1, D), "normal", "f16")
    scale = 0.125
    qsum = orc.to_f64(q, "f16")[0, :, 0].sum(-1)            # per head
    # logit of the extra key for head h: scale * 0.75 * sum(q_h)
    sinks = np.array([(scale * 0.75) * qsum[h] for h in range(Hq)])
    with_key = orc.attention(q, "f16", kc, vc, L + 1, scale)
    for mode, ns in MODES:
        with_sink = orc.attention(q, "f16", kc, vc, L, scale, mode=mode, nsplit=ns,
                                  ext=orc.Ext(sinks=sinks))
        np.testing.assert_allclose(with_sink, with_key, rtol=0, atol=1e-13)
    assert G == 2


@pytest.mark.parametrize("sink", [-3.0, 0.0, 1.5, 6.0])
def test_sink_closed_form_with_zero_query(orc, sink):
    D, L, Hq = 64, 40, 4
    kc, vc = _cache(orc, 1, 1, L, D, "affine", 8, 32, seed=23)
    Vd = orc.dequantize(vc, D)[0, 0, :L]
    q = np.zeros((1, Hq, 1, D), np.uint16)
    sinks = np.full(Hq, sink)
    # every logit is 0: each key weighs 1 / (L + e^sink)
    want = Vd.sum(0) / (L + math.exp(sink))
    for mode, ns in MODES:
        out = orc.attention(q, "f16", kc, vc, L, 1.0, mode=mode, nsplit=ns,
                            ext=orc.Ext(sinks=sinks))
        np.testing.assert_allclose(out[0, :, 0], np.broadcast_to(want, (Hq, D)), rtol=0,
                                   atol=1e-14)
    p, _ = orc.attention_probs(q, "f16", kc, vc, L, 1.0, 0, 1, 0, ext=orc.Ext(sinks=sinks))
    assert abs(p.sum() - L / (L + math.exp(sink))) < 1e-14


def test_sink_limits_and_masked_rows(orc):
    D, L, Hq = 128, 33, 2
    kc, vc = _cache(orc, 1, 1, L, D, "q8_0", 8, 32, seed=24)
    q = S.draw(25, "q", (1, Hq, 1, D), "normal", "f16")
    plain = orc.attention(q, "f16", kc, vc, L, 0.1)
    none = orc.attention(q, "f16", kc, vc, L, 0.1, ext=orc.Ext(sinks=np.full(Hq, -np.inf)))
    assert np.array_equal(none, plain)
    big = orc.attention(q, "f16", kc, vc, L, 0.1, ext=orc.Ext(sinks=np.full(Hq, 60.0)))
    assert np.abs(big).max() < 1e-20
    # a row with no visible key stays zero with a sink
    m = np.full((L,), -np.inf, np.float32)
    out = orc.attention(q, "f16", kc, vc, L, 0.1, mask=orc.Mask("additive", m, "f32"),
                        ext=orc.Ext(sinks=np.zeros(Hq)))
    assert np.all(out == 0.0)


def test_softcap_closed_form_with_constant_keys(orc):
    D, L, Hq, c, scale = 64, 24, 2, 2.5, 0.5
    # key row j is the constant a_j along D (exact after quantization), so the
    # logit of head h is scale * a_j * sum(q_h)
    a = (np.arange(L, dtype=np.float32) - L / 2) / 4
    k = np.repeat(np.repeat(a[:, None], D, 1)[None, None], 1, 0).astype(np.float16).view(np.uint16)
    v = S.draw(26, "v", (1, 1, L, D), "normal", "f16")
    kc = orc.quantize(k, "f16", "affine", 64, 4)
    vc = orc.quantize(v, "f16", "affine", 64, 4)
    assert np.array_equal(orc.dequantize(kc, D)[0, 0, :, 0], a.astype(np.float64))
    Vd = orc.dequantize(vc, D)[0, 0]
    q = S.draw(27, "q", (1, Hq, 1, D), "uniform", "f16")
    qsum = orc.to_f64(q, "f16")[0, :, 0].sum(-1)
    out_by_mode = [orc.attention(q, "f16", kc, vc, L, scale, mode=m, nsplit=n,
                                 ext=orc.Ext(softcap=c)) for m, n in MODES]
    for h in range(Hq):
        x = [scale * float(a[j]) * qsum[h] for j in range(L)]
        y = [c * math.tanh(xj / c) for xj in x]
        mx = max(y)
        w = np.array([math.exp(yj - mx) for yj in y])
        want = (w[:, None] * Vd).sum(0) / w.sum()
        for out in out_by_mode:
            np.testing.assert_allclose(out[0, h, 0], want, rtol=0, atol=1e-13)
        assert max(abs(v) for v in x) > 2 * c          # the cap is active


def test_softcap_limits(orc):
    D, L, Hq = 128, 50, 4
    kc, vc = _cache(orc, 1, 2, L, D, "affine", 4, 64, seed=28)
    q = S.draw(29, "q", (1, Hq, 1, D), "normal", "f16")
    plain = orc.attention(q, "f16", kc, vc, L, 0.2)
    # c -> infinity: c*tanh(x/c) = x - x^3/(3c^2) + ...
    wide = orc.attention(q, "f16", kc, vc, L, 0.2, ext=orc.Ext(softcap=1e6))
    np.testing.assert_allclose(wide, plain, rtol=0, atol=1e-9)
    # tiny cap: every logit lies in (-c, c), so each weight is within e^(+-2c)
    # of 1/L and the output within that factor of the mean of V
    c = 1e-4
    Vd = orc.dequantize(vc, D)[0, :, :L]
    tight = orc.attention(q, "f16", kc, vc, L, 0.2, ext=orc.Ext(softcap=c))
    for h in range(Hq):
        mean = Vd[h // 2].mean(0)
        bound = (math.exp(2 * c) - 1) * np.abs(Vd[h // 2]).max() * 2
        assert np.abs(tight[0, h, 0] - mean).max() <= bound


def test_mask_slope_equals_premultiplied_mask(orc):
    B, Hq, Hkv, Lq, D, L = 1, 8, 2, 3, 64, 21
    kc, vc = _cache(orc, B, Hkv, L, D, "affine", 4, 32, seed=30)
    q = S.draw(31, "q", (B, Hq, Lq, D), "normal", "f16")
    rng = np.random.default_rng(3)
    m = rng.standard_normal((Lq, L)).astype(np.float32)
    m[1, 4] = -np.inf
    # ALiBi slopes for 8 heads (Press et al.): 2^-1 ... 2^-8, powers of two,
    # so slope * mask is exact in fp32
    slopes = 2.0 ** -np.arange(1, Hq + 1)
    shared = orc.Mask("additive", m, "f32", (0, 0, L))
    pre = (slopes[:, None, None] * m[None]).astype(np.float32)
    per_head = orc.Mask("additive", pre, "f32", (0, Lq * L, L))
    want = orc.attention(q, "f16", kc, vc, L, 0.3, mask=per_head)
    for mode, ns in MODES:
        got = orc.attention(q, "f16", kc, vc, L, 0.3, mask=shared, mode=mode, nsplit=ns,
                            ext=orc.Ext(slopes=slopes))
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-14)


def test_alibi_closed_form_with_zero_query(orc):
    D, L, Hq = 64, 30, 4
    kc, vc = _cache(orc, 1, 1, L, D, "q8_0", 8, 32, seed=32)
    Vd = orc.dequantize(vc, D)[0, 0, :L]
    q = np.zeros((1, Hq, 1, D), np.uint16)
    dist = -np.abs(np.arange(L) - (L - 1)).astype(np.float32)       # decode row at L-1
    slopes = 2.0 ** -np.arange(1, Hq + 1)
    out = orc.attention(q, "f16", kc, vc, L, 1.0, mask=orc.Mask("additive", dist, "f32"),
                        ext=orc.Ext(slopes=slopes))
    for h in range(Hq):
        r = math.exp(-slopes[h])                    # key j weighs r^(L-1-j)
        w = np.array([r ** (L - 1 - j) for j in range(L)])
        np.testing.assert_allclose(out[0, h, 0], (w[:, None] * Vd).sum(0) / w.sum(), rtol=0,
                                   atol=1e-13)


def test_all_extensions_agree_across_evaluation_orders(orc):
    B, Hq, Hkv, Lq, D, L = 2, 4, 2, 2, 128, 45
    kc, vc = _cache(orc, B, Hkv, L, D, "affine", 8, 64, seed=33)
    q = S.draw(34, "q", (B, Hq, Lq, D), "normal", "f16")
    m = -np.abs(np.arange(L)[None, :] - (L - Lq + np.arange(Lq))[:, None]).astype(np.float32)
    ext = orc.Ext(softcap=3.0, sinks=np.linspace(-1, 2, Hq), slopes=2.0 ** -np.arange(1, Hq + 1))
    mask = orc.Mask("additive", m, "f32", (0, 0, L))
    outs = [orc.attention(q, "f16", kc, vc, L, 0.15, mask=mask, mode=mo, nsplit=n, ext=ext)
            for mo, n in (("two_pass", 1), ("online", 1), ("split", 4), ("split", 9))]
    for o in outs[1:]:
        np.testing.assert_allclose(o, outs[0], rtol=0, atol=1e-13)
