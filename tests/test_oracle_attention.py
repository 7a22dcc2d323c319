"""Pins for the oracle's attention (CPU only).

The oracle dequantizes, then computes softmax(q*scale . K^T + mask) V in fp64
(MLX quantized-KV branch, fast.cpp fallback of
quantized_scaled_dot_product_attention).  It is checked against torch's
scaled_dot_product_attention in fp64 (a library routine) on the dequantized
cache, against closed forms (one key, uniform V, zero query, equal keys),
against invariants (softmax rows sum to one) and across its three independent
evaluation orders (two-pass, online, split + log-sum-exp merge).
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

from quantized_kv_attention_split_b200 import synthetic as S


def _cache(orc, B, Hkv, L, D, fmt, bits, gs, seed, dist="normal", dtype="f16", Lcap=None):
    Lcap = Lcap or L
    k = S.draw(seed, "k", (B, Hkv, Lcap, D), dist, dtype)
    v = S.draw(seed, "v", (B, Hkv, Lcap, D), dist, dtype)
    return orc.quantize(k, dtype, fmt, gs, bits), orc.quantize(v, dtype, fmt, gs, bits)


def _torch_ref(orc, q, qdt, kc, vc, L, scale, D, attn_mask=None):
    q64 = torch.from_numpy(orc.to_f64(q, qdt))
    K = torch.from_numpy(orc.dequantize(kc, D))[:, :, :L]
    V = torch.from_numpy(orc.dequantize(vc, D))[:, :, :L]
    G = q64.shape[1] // K.shape[1]
    K = K.repeat_interleave(G, dim=1)
    V = V.repeat_interleave(G, dim=1)
    return F.scaled_dot_product_attention(q64, K, V, attn_mask=attn_mask, scale=scale).numpy()


CASES = [
    # B, Hq, Hkv, Lq, D, L, Lcap, fmt, bits, gs, scale
    (1, 4, 1, 1, 64, 37, 40, "affine", 4, 64, 1.0),
    (2, 8, 2, 3, 128, 100, 128, "affine", 8, 32, 0.125),
    (1, 6, 3, 2, 64, 19, 19, "affine", 4, 32, 0.3),
    (1, 4, 2, 5, 256, 50, 64, "q8_0", 8, 32, 1.0 / 16),
    (2, 2, 2, 1, 128, 64, 64, "affine", 4, 128, 0.09),
    (1, 4, 2, 2, 64, 33, 40, "affine", 3, 32, 0.2),     # codes straddle words
    (1, 2, 1, 1, 128, 21, 24, "affine", 6, 64, 0.1),
    (1, 2, 1, 3, 64, 17, 24, "affine", 5, 32, 0.3),
    (1, 2, 2, 1, 64, 12, 16, "affine", 2, 64, 1.0),
]


@pytest.mark.parametrize("case", CASES)
def test_matches_torch_sdpa(orc, case):
    B, Hq, Hkv, Lq, D, L, Lcap, fmt, bits, gs, scale = case
    kc, vc = _cache(orc, B, Hkv, L, D, fmt, bits, gs, seed=B * 100 + D, Lcap=Lcap)
    q = S.draw(9, "q", (B, Hq, Lq, D), "normal", "f16")
    ref = _torch_ref(orc, q, "f16", kc, vc, L, scale, D)
    for mode, ns in (("two_pass", 1), ("online", 1), ("split", 3), ("split", 7)):
        out = orc.attention(q, "f16", kc, vc, L, scale, mode=mode, nsplit=ns, nthreads=4)
        np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_additive_mask_matches_torch(orc):
    B, Hq, Hkv, Lq, D, L = 2, 4, 2, 3, 64, 30
    kc, vc = _cache(orc, B, Hkv, L, D, "affine", 4, 64, seed=5)
    q = S.draw(10, "q", (B, Hq, Lq, D), "normal", "bf16")
    rng = np.random.default_rng(0)
    m = rng.standard_normal((B, Hq, Lq, L)).astype(np.float32)
    m[0, 1, 2, 5:9] = -np.inf
    mask = orc.Mask("additive", m, "f32", (Hq * Lq * L, Lq * L, L))
    ref = _torch_ref(orc, q, "bf16", kc, vc, L, 0.2, D, attn_mask=torch.from_numpy(m).double())
    out = orc.attention(q, "bf16", kc, vc, L, 0.2, mask=mask)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    # a broadcast (stride-0) fp16 mask
    mh = S.f32_to_half_bits(rng.standard_normal(L).astype(np.float32), "f16")
    mask = orc.Mask("additive", mh, "f16", (0, 0, 0))
    mt = torch.from_numpy(orc.to_f64(mh, "f16")).expand(B, Hq, Lq, L)
    ref = _torch_ref(orc, q, "bf16", kc, vc, L, 0.2, D, attn_mask=mt)
    out = orc.attention(q, "bf16", kc, vc, L, 0.2, mask=mask, mode="split", nsplit=4)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("Lq,L", [(5, 12), (12, 12), (1, 9)])
def test_causal_bottom_right_matches_torch(orc, Lq, L):
    B, Hq, Hkv, D = 1, 4, 1, 64
    kc, vc = _cache(orc, B, Hkv, L, D, "q8_0", 8, 32, seed=6)
    q = S.draw(11, "q", (B, Hq, Lq, D), "normal", "f16")
    i = np.arange(Lq)[:, None]
    j = np.arange(L)[None, :]
    allowed = torch.from_numpy(j <= L - Lq + i)          # bottom-right aligned
    ref = _torch_ref(orc, q, "f16", kc, vc, L, 0.125, D, attn_mask=allowed)
    for mode in ("two_pass", "online", "split"):
        out = orc.attention(q, "f16", kc, vc, L, 0.125, mask=orc.Mask("causal"), mode=mode,
                            nsplit=3)
        np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_fully_masked_rows_are_zero(orc):
    B, Hq, Hkv, Lq, D, L = 1, 2, 1, 4, 64, 3
    kc, vc = _cache(orc, B, Hkv, L, D, "affine", 4, 64, seed=7)
    q = S.draw(12, "q", (B, Hq, Lq, D), "normal", "f16")
    # causal with Lq > L: query i sees j <= L - Lq + i, so row 0 sees nothing
    for mode in ("two_pass", "online", "split"):
        out = orc.attention(q, "f16", kc, vc, L, 1.0, mask=orc.Mask("causal"), mode=mode,
                            nsplit=2)
        assert np.all(out[:, :, 0] == 0.0)
        assert np.all(np.abs(out[:, :, 1:]).sum(-1) > 0)
    m = np.full((L,), -np.inf, np.float32)
    out = orc.attention(q, "f16", kc, vc, L, 1.0, mask=orc.Mask("additive", m, "f32"))
    assert np.all(out == 0.0)


def test_single_key_returns_its_value(orc):
    D = 128
    kc, vc = _cache(orc, 1, 2, 1, D, "affine", 8, 64, seed=8, Lcap=8)
    q = S.draw(13, "q", (1, 8, 1, D), "uniform", "f16")
    out = orc.attention(q, "f16", kc, vc, 1, 1.0)
    Vd = orc.dequantize(vc, D)
    for h in range(8):
        np.testing.assert_allclose(out[0, h, 0], Vd[0, h // 4, 0], rtol=0, atol=1e-15)


def test_uniform_values_return_values(orc):
    D, L = 64, 77
    k = S.draw(1, "k", (1, 1, L, D), "uniform", "f16")
    row = S.draw(2, "v", (1, 1, 1, D), "uniform", "f16")
    v = np.repeat(row, L, axis=2)
    kc = orc.quantize(k, "f16", "affine", 64, 4)
    vc = orc.quantize(v, "f16", "affine", 64, 4)
    q = S.draw(3, "q", (1, 4, 1, D), "uniform", "f16")
    out = orc.attention(q, "f16", kc, vc, L, 1.0)
    Vd = orc.dequantize(vc, D)[0, 0, 0]
    np.testing.assert_allclose(out[0, :, 0], np.broadcast_to(Vd, (4, D)), rtol=0, atol=1e-14)


def test_zero_query_and_equal_keys_give_mean_of_values(orc):
    D, L = 64, 50
    kc, vc = _cache(orc, 1, 1, L, D, "affine", 4, 32, seed=9)
    Vd = orc.dequantize(vc, D)[0, 0, :L]
    q = np.zeros((1, 2, 1, D), np.uint16)
    out = orc.attention(q, "f16", kc, vc, L, 1.0)
    np.testing.assert_allclose(out[0, :, 0], np.broadcast_to(Vd.mean(0), (2, D)), atol=1e-14)
    # identical keys: every logit equal, so the weights are uniform
    k = np.repeat(S.draw(4, "k", (1, 1, 1, D), "normal", "f16"), L, axis=2)
    kc2 = orc.quantize(k, "f16", "affine", 32, 4)
    q = S.draw(5, "q", (1, 2, 1, D), "normal", "f16")
    out = orc.attention(q, "f16", kc2, vc, L, 1.0)
    np.testing.assert_allclose(out[0, :, 0], np.broadcast_to(Vd.mean(0), (2, D)), atol=1e-13)


def test_softmax_rows_sum_to_one(orc):
    D, L = 128, 300
    kc, vc = _cache(orc, 1, 2, L, D, "affine", 4, 64, seed=10, dist="uniform")
    q = S.draw(6, "q", (1, 8, 1, D), "uniform", "f16")
    for h in (0, 3, 7):
        p, o = orc.attention_probs(q, "f16", kc, vc, L, 1.0, 0, h, 0)
        assert abs(p.sum() - 1.0) < 1e-14
        assert np.all(p >= 0)
        Vd = orc.dequantize(vc, D)[0, h // 4, :L]
        np.testing.assert_allclose(o, p @ Vd, atol=1e-13)


def test_row_subset(orc):
    B, Hq, Hkv, Lq, D, L = 1, 4, 2, 3, 64, 20
    kc, vc = _cache(orc, B, Hkv, L, D, "affine", 4, 64, seed=11)
    q = S.draw(7, "q", (B, Hq, Lq, D), "normal", "f16")
    full = orc.attention(q, "f16", kc, vc, L, 1.0)
    rows = np.array([0, 5, 11])
    sub = orc.attention(q, "f16", kc, vc, L, 1.0, rows=rows)
    flat = sub.reshape(-1, D)
    assert np.array_equal(flat[rows], full.reshape(-1, D)[rows])
    assert np.isnan(flat[1]).all()


@pytest.mark.parametrize("causal", [False, True])
def test_values_as_a_view_of_the_keys_matches_torch(orc, causal):
    """MLA shape of the llama.cpp PR's follow-up tests: K rows of 576 (Q8_0),
    V the first 512 elements of each K row; torch's SDPA in fp64 with V given
    as that slice (a library routine that takes different K and V widths)."""
    B, Hq, Hkv, Lq, Dk, Dv, L = 1, 4, 1, 3, 576, 512, 40
    k = S.draw(91, "k", (B, Hkv, L, Dk), "normal", "f16")
    q = S.draw(92, "q", (B, Hq, Lq, Dk), "normal", "f16")
    kc = orc.quantize(k, "f16", "q8_0")
    K = torch.from_numpy(orc.dequantize(kc, Dk)).repeat_interleave(Hq // Hkv, dim=1)
    q64 = torch.from_numpy(orc.to_f64(q, "f16"))
    scale = 1.0 / 24
    mask = orc.Mask("causal") if causal else None
    tmask = None
    if causal:
        tmask = torch.ones(Lq, L, dtype=torch.bool).tril(diagonal=L - Lq)
    ref = F.scaled_dot_product_attention(q64, K, K[..., :Dv], attn_mask=tmask, scale=scale).numpy()
    for mode, ns in (("two_pass", 1), ("online", 1), ("split", 4)):
        out = orc.attention_kview(q, "f16", kc, L, scale, Dv, mask=mask, mode=mode, nsplit=ns)
        np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("causal", [False, True])
def test_dense_form_matches_torch_and_the_loops(orc, case, causal):
    """The matrix-product form (attention_dense, used to check every row of a
    large prefill) against torch's SDPA in fp64 and against the oracle's own
    per-row loops, with and without the bottom-right causal limit."""
    B, Hq, Hkv, Lq, D, L, Lcap, fmt, bits, gs, scale = case
    kc, vc = _cache(orc, B, Hkv, L, D, fmt, bits, gs, seed=B * 100 + D + 1, Lcap=Lcap)
    q = S.draw(19, "q", (B, Hq, Lq, D), "normal", "f16")
    tmask = torch.ones(Lq, L, dtype=torch.bool).tril(diagonal=L - Lq) if causal else None
    ref = _torch_ref(orc, q, "f16", kc, vc, L, scale, D, attn_mask=tmask)
    out = orc.attention_dense(q, "f16", kc, vc, L, scale, causal=causal, row_block=2)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    loops = orc.attention(q, "f16", kc, vc, L, scale,
                          mask=orc.Mask("causal") if causal else None)
    np.testing.assert_allclose(out, loops, rtol=0, atol=1e-12)


def test_dense_form_head_subset_and_rows_with_no_key(orc):
    """Only the requested heads are computed (the rest stay NaN); causal
    queries placed before the first key return zeros, as in the loops."""
    B, Hq, Hkv, Lq, D, L = 1, 4, 2, 7, 64, 5
    kc, vc = _cache(orc, B, Hkv, L, D, "q8_0", 8, 32, seed=23, Lcap=8)
    q = S.draw(24, "q", (B, Hq, Lq, D), "normal", "f16")
    out = orc.attention_dense(q, "f16", kc, vc, L, 0.2, causal=True, heads=[1, 2])
    assert np.isnan(out[0, 0]).all() and np.isnan(out[0, 3]).all()
    loops = orc.attention(q, "f16", kc, vc, L, 0.2, mask=orc.Mask("causal"))
    np.testing.assert_allclose(out[0, 1:3], loops[0, 1:3], rtol=0, atol=1e-12)
    assert np.all(out[0, 1:3, :Lq - L] == 0)
