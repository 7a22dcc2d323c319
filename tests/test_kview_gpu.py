"""Attention with the values as a view of the keys (K rows of 576, V their
first 512 elements: the "576/512 MLA" shape of the llama.cpp PR's follow-up
tests) through the C ABI (qsdpa_attention_kview), against the oracle's
attention_kview, element by element: Q8_0 and affine 4/8-bit caches, decode
(one query) and multi-query with and without the causal limit, one 64-row tile partly
filled and several (128 query heads over one KV head; 96 heads: a ragged
second tile), ragged L, units split over CTAs (merged by the merge kernel)
and whole."""
import numpy as np
import pytest
import torch

import oracle
from helpers import TOL, TORCH_DT, cache_to_dev, from_dev, max_err, out_err, to_dev
from quantized_kv_attention_split_b200 import synthetic as S

pytestmark = pytest.mark.gpu

DK, DV = 576, 512


def _problem(B, Hq, Hkv, Lq, L, fmt, bits, gs, seed, dist="normal", q_dtype="bf16"):
    Lcap = (L // 8 + 2) * 8
    k = S.draw(seed, "k", (B, Hkv, Lcap, DK), dist, "f16")
    q = S.draw(seed, "q", (B, Hq, Lq, DK), "normal", q_dtype)
    return q, oracle.quantize(k, "f16", fmt, gs, bits)


CASES = [
    # B, Hq, Hkv, Lq, L, fmt, bits, gs
    (1, 16, 1, 1, 4099, "q8_0", 8, 32),       # one tile, split over many CTAs
    (1, 128, 1, 1, 2048, "q8_0", 8, 32),      # 2 tiles (DeepSeek-like head count)
    (1, 96, 1, 1, 3001, "q8_0", 8, 32),       # a full tile and a half-filled one
    (1, 64, 1, 2, 700, "affine", 4, 64),      # multi-query: 128 rows, 2 tiles
    (2, 32, 2, 1, 777, "affine", 8, 64),
    (1, 16, 2, 1, 1000, "affine", 4, 32),
    (1, 8, 1, 1, 90, "affine", 4, 64),        # short: one CTA per unit, written whole
    (1, 16, 1, 8, 1500, "q8_0", 8, 32),       # multi-query
    (1, 4, 1, 20, 333, "affine", 8, 32),      # multi-query, ragged tile (80 rows)
]


# causal runs only where it differs from no mask (more than one query)
CASES_CAUSAL = [(c, False) for c in CASES] + [(c, True) for c in CASES if c[3] > 1]


@pytest.mark.parametrize("case,causal", CASES_CAUSAL,
                         ids=lambda c: "-".join(map(str, c)) if isinstance(c, tuple) else str(c))
def test_kview_matches_oracle(case, causal):
    from quantized_kv_attention_split_b200 import qkv
    B, Hq, Hkv, Lq, L, fmt, bits, gs = case
    q, kc = _problem(B, Hq, Hkv, Lq, L, fmt, bits, gs, seed=Hq + L)
    scale = 1.0 / np.sqrt(DK)
    mask = oracle.Mask("causal") if causal else None
    ref = oracle.attention_kview(q, "bf16", kc, L, scale, DV, mask=mask)
    qd, kd = to_dev(q, "bf16"), cache_to_dev(kc)
    for odt in ("bf16", "f16"):
        out = qkv.qsdpa_attention_kview(qd, kd, L, scale, causal=causal, out_dtype=TORCH_DT[odt])
        torch.cuda.synchronize()
        got = from_dev(out)
        assert got.shape == (B, Hq, Lq, DV)
        assert out_err(got, ref, odt) <= 1.0, (odt, max_err(got, ref))


def test_kview_uniform_inputs_and_lq_beyond_l():
    """U[0,1) keys (the decode benchmark's distribution) and causal queries
    before the first key, which see nothing and return zeros."""
    from quantized_kv_attention_split_b200 import qkv
    q, kc = _problem(1, 16, 1, 40, 24, "q8_0", 8, 32, seed=5, dist="uniform")
    ref = oracle.attention_kview(q, "bf16", kc, 24, 0.05, DV, mask=oracle.Mask("causal"))
    out = qkv.qsdpa_attention_kview(to_dev(q, "bf16"), cache_to_dev(kc), 24, 0.05, causal=True,
                                    out_dtype=torch.float16)
    torch.cuda.synchronize()
    got = from_dev(out)
    assert np.all(got[:, :, :40 - 24] == 0)
    assert max_err(got, ref) <= TOL["f16"]


def test_kview_refuses_what_it_does_not_build():
    from quantized_kv_attention_split_b200 import qkv
    q, kc = _problem(1, 16, 1, 1, 64, "q8_0", 8, 32, seed=6)
    qd, kd = to_dev(q, "bf16"), cache_to_dev(kc)
    with pytest.raises(qkv.QKVError, match="f16 or bf16"):
        qkv.qsdpa_attention_kview(qd, kd, 64, 0.1, out_dtype=torch.float32)


@pytest.mark.parametrize("fmt,bits,gs", [("q8_0", 8, 32), ("affine", 4, 64), ("affine", 8, 32)])
def test_kview_cache_written_by_the_quantizer(fmt, bits, gs):
    """576-element key rows appended by qkv_quantize_update (rows of 18
    threads) are bit-identical to the oracle's, and attended over."""
    from quantized_kv_attention_split_b200 import qkv
    B, Hq, L, Lcap = 1, 16, 301, 304
    x = S.draw(7, "k", (B, 1, L, DK), "normal", "bf16")
    f = qkv.Q8_0 if fmt == "q8_0" else qkv.AFFINE
    kd = qkv.QuantCache.empty(B, 1, Lcap, DK, f, bits, gs)
    vd = qkv.QuantCache.empty(B, 1, Lcap, DK, f, bits, gs)
    qkv.qkv_quantize_update(to_dev(x, "bf16"), to_dev(x, "bf16"), kd, vd, 0)
    torch.cuda.synchronize()
    ref_c = oracle.quantize(x, "bf16", fmt, gs, bits)
    from helpers import cache_from_dev
    got_c = cache_from_dev(kd, fmt)
    assert np.array_equal(got_c.codes[:, :, :L], ref_c.codes)
    assert np.array_equal(got_c.scales[:, :, :L], ref_c.scales)
    q = S.draw(8, "q", (B, Hq, 1, DK), "normal", "bf16")
    ref = oracle.attention_kview(q, "bf16", got_c, L, 0.04, DV)
    out = qkv.qsdpa_attention_kview(to_dev(q, "bf16"), kd, L, 0.04)
    torch.cuda.synchronize()
    assert out_err(from_dev(out), ref, "bf16") <= 1.0
