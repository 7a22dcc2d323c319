"""Affine codes stored 2, 3, 5 or 6 bits wide (one little-endian bit stream
per row, codes straddling 32-bit words for 3, 5 and 6 bits; MLX compare
v0.30.0...6c60bd1, quantized_utils.cuh get_pack_factor / get_bytes_per_pack
name these widths) through the C ABI: decode (the split-K kernel transcodes
each staged block to 8-bit codes), multi-query attention on the same kernel,
and the materialize-to-fp16 conversion -- against the CPU oracle, element by
element, at every width, group size 32/64/128 and head dimension 64/128/256."""
import numpy as np
import pytest
import torch

import oracle
from helpers import TOL, TORCH_DT, cache_from_dev, cache_to_dev, from_dev, make_problem, max_err, to_dev
from quantized_kv_attention_split_b200 import synthetic as S

pytestmark = pytest.mark.gpu

WIDTHS = [2, 3, 5, 6]
GEOM = [(64, 32), (64, 64), (128, 32), (128, 64), (128, 128), (256, 32), (256, 64), (256, 128)]


@pytest.fixture(scope="module")
def qkv():
    from quantized_kv_attention_split_b200 import qkv as m
    m.lib()
    return m


@pytest.mark.parametrize("bits", WIDTHS)
@pytest.mark.parametrize("D,gs", GEOM, ids=lambda x: str(x))
def test_decode_at_every_width(qkv, bits, D, gs):
    """Query heads per KV head 4, 16 and 40 (one, two and four 8-row chunks
    per CTA; 40 also takes two chunk groups), ragged L."""
    for Hq, Hkv, L in ((8, 2, 1333), (32, 2, 517), (40, 1, 203)):
        q, kc, vc = make_problem(1, Hq, Hkv, 1, D, L, "affine", bits, gs, "normal",
                                 Lcap=(L // 8 + 3) * 8, seed=bits * 7 + D + gs)
        scale = 1.0 / np.sqrt(D)
        ref = oracle.attention(q, "f16", kc, vc, L, scale)
        qd, kd, vd = to_dev(q, "f16"), cache_to_dev(kc), cache_to_dev(vc)
        for odt in ("f16", "f32"):
            out = qkv.qsdpa_decode(qd, kd, vd, L, scale, out_dtype=TORCH_DT[odt])
            torch.cuda.synchronize()
            assert max_err(from_dev(out), ref) <= TOL[odt], (Hq, L, odt, max_err(from_dev(out), ref))


@pytest.mark.parametrize("bits", WIDTHS)
def test_quantize_then_decode_short_and_full_blocks(qkv, bits):
    """The cache written by the GPU quantizer, read by the decode kernel, at
    lengths around the block sizes (the last block partly valid) and L = 0."""
    D, gs, B, Hq, Hkv = 128, 64, 2, 16, 4
    Lcap = 264
    src_k = S.draw(90 + bits, "k", (B, Hkv, Lcap, D), "uniform", "bf16")
    src_v = S.draw(90 + bits, "v", (B, Hkv, Lcap, D), "uniform", "bf16")
    kd = qkv.QuantCache.empty(B, Hkv, Lcap, D, qkv.AFFINE, bits, gs)
    vd = qkv.QuantCache.empty(B, Hkv, Lcap, D, qkv.AFFINE, bits, gs)
    qkv.qkv_quantize_update(to_dev(src_k, "bf16"), to_dev(src_v, "bf16"), kd, vd, 0)
    torch.cuda.synchronize()
    kc, vc = cache_from_dev(kd, "affine"), cache_from_dev(vd, "affine")
    ref_k = oracle.quantize(src_k, "bf16", "affine", gs, bits)
    assert np.array_equal(kc.codes, ref_k.codes) and np.array_equal(kc.scales, ref_k.scales)
    q = S.draw(95, "q", (B, Hq, 1, D), "normal", "bf16")
    for L in (0, 1, 15, 16, 17, 31, 32, 33, 257, 264):
        out = qkv.qsdpa_decode(to_dev(q, "bf16"), kd, vd, L, 0.1, out_dtype=torch.float32)
        torch.cuda.synchronize()
        if L == 0:
            assert torch.all(out == 0)
            continue
        ref = oracle.attention(q, "bf16", kc, vc, L, 0.1)
        assert max_err(from_dev(out), ref) <= TOL["f32"], (L, max_err(from_dev(out), ref))


@pytest.mark.parametrize("bits", WIDTHS)
@pytest.mark.parametrize("causal", [False, True])
def test_multi_query_at_every_width(qkv, bits, causal):
    """Multi-query attention over 2/3/5/6-bit caches runs on the split-K
    kernel (rows = (head, query) pairs), causal or not, 16-bit and fp32 out."""
    B, Hq, Hkv, Lq, D, L = 1, 8, 2, 24, 128, 700
    q, kc, vc = make_problem(B, Hq, Hkv, Lq, D, L, "affine", bits, 32, "normal", q_dtype="bf16",
                             Lcap=704, seed=bits + 40)
    mask = oracle.Mask("causal") if causal else None
    ref = oracle.attention(q, "bf16", kc, vc, L, 0.09, mask=mask)
    for odt in ("f16", "f32"):
        out = qkv.qsdpa_prefill(to_dev(q, "bf16"), cache_to_dev(kc), cache_to_dev(vc), L, 0.09,
                                causal=causal, out_dtype=TORCH_DT[odt])
        torch.cuda.synchronize()
        assert max_err(from_dev(out), ref) <= TOL[odt], (odt, max_err(from_dev(out), ref))


@pytest.mark.parametrize("bits", WIDTHS)
@pytest.mark.parametrize("D,gs", [(64, 32), (128, 64), (256, 128)])
def test_dequantize_at_every_width(qkv, bits, D, gs):
    """Materialize to fp16: the correctly rounded exact dequantization."""
    _, kc, _ = make_problem(2, 4, 2, 1, D, 77, "affine", bits, gs, "normal", Lcap=80, seed=3)
    out = qkv.qkv_dequantize(cache_to_dev(kc), 77)
    torch.cuda.synchronize()
    ref = oracle.dequantize(kc, D)[:, :, :77].astype(np.float16)      # one rounding from fp64
    assert np.array_equal(out.cpu().numpy().view(np.uint16), ref.view(np.uint16))


def test_unsupported_variants_are_refused(qkv):
    """Additive masks, attention extensions and the fused update step are not
    built for these widths: refused before any launch."""
    q, kc, vc = make_problem(1, 8, 2, 1, 128, 100, "affine", 3, 64, Lcap=104)
    qd, kd, vd = to_dev(q, "f16"), cache_to_dev(kc), cache_to_dev(vc)
    with pytest.raises(qkv.QKVError, match="2/3/5/6-bit"):
        qkv.qsdpa_decode(qd, kd, vd, 100, 0.1, softcap=30.0)
    with pytest.raises(qkv.QKVError, match="2/3/5/6-bit"):
        qkv.qsdpa_decode(qd, kd, vd, 100, 0.1, mask=torch.zeros(100, device="cuda"))
