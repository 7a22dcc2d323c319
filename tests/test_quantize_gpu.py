"""GPU quantize-and-append (qkv_quantize_update) must match the oracle's
quantizer bit for bit: codes, fp16 scales and fp16 biases, written only to
rows [offset, offset+Lnew) of each (batch, kv-head).  Affine codes of 2, 3, 4,
5, 6 and 8 bits (3, 5 and 6-bit codes straddle 32-bit words of the row's bit
stream) and Q8_0."""
import numpy as np
import pytest
import torch

import oracle
from helpers import cache_from_dev, to_dev
from quantized_kv_attention_split_b200 import synthetic as S

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def qkv():
    from quantized_kv_attention_split_b200 import qkv as m
    m.lib()
    return m


def _inputs(shape, kind, dtype, seed, fmt="affine", bits=4, gs=32):
    rng = np.random.default_rng(seed)
    if kind == "halfway":                    # codes exactly at and next to x.5
        return _halfway(shape, dtype, rng, fmt, bits, gs)
    if kind == "uniform":
        x = rng.random(shape, dtype=np.float32)
    elif kind == "normal":
        x = rng.standard_normal(shape).astype(np.float32)
    elif kind == "wide":
        x = (rng.standard_normal(shape) * 10.0 ** rng.uniform(-4, 3, shape[:-1] + (1,))).astype(
            np.float32)
    elif kind == "special":                  # constant groups, zeros, ties
        x = np.zeros(shape, np.float32)
        x[..., 1::4, :] = 0.5
        x[..., 2::4, :] = np.arange(shape[-1]) % 3 - 1.0
        x[..., 3::4, :] = rng.integers(-4, 5, shape[:-2] + (len(range(3, shape[-2], 4)), shape[-1]))
    return S.f32_to_half_bits(x, dtype)


def _halfway(shape, dtype, rng, fmt, bits, gs):
    """Groups whose scale is an exact power of two 2^e (affine: min 0 and max
    (2^bits - 1) * 2^e; Q8_0: max|x| = 127 * 2^e; all values representable in
    f16 and bf16), so that (x - bias) / scale is exactly k + 0.5 for the other
    elements, half of which are then moved one unit in the last place up or
    down: the quantizer's rounding decision at and right next to every tie."""
    lead = shape[:-1]
    ng = shape[-1] // gs
    e = rng.integers(-8, 5, lead + (ng, 1)).astype(np.float32)
    top = 127 if fmt == "q8_0" else (1 << bits) - 1
    k = rng.integers(0, min(top, 127), lead + (ng, gs)).astype(np.float32) + 0.5
    if fmt == "q8_0":
        k *= np.where(rng.random(k.shape) < 0.5, -1.0, 1.0)
    g = k * np.exp2(e)
    g[..., 0] = top * np.exp2(e[..., 0])
    if fmt != "q8_0":
        g[..., 1] = 0.0
    bits16 = S.f32_to_half_bits(g.reshape(shape), dtype).astype(np.int32)
    nudge = rng.integers(-1, 2, lead + (ng, gs))
    nudge[..., :2] = 0
    return (bits16 + nudge.reshape(shape)).astype(np.uint16)


CASES = [
    # fmt, bits, gs, D, dtype
    ("affine", 4, 64, 128, "f16"), ("affine", 4, 32, 64, "f16"), ("affine", 4, 128, 256, "bf16"),
    ("affine", 8, 64, 128, "bf16"), ("affine", 8, 32, 256, "f16"), ("affine", 8, 128, 128, "f16"),
    ("q8_0", 8, 32, 256, "f16"), ("q8_0", 8, 32, 64, "bf16"),
    # codes that straddle 32-bit words (3, 5, 6 bits) and 2-bit codes
    ("affine", 2, 64, 128, "f16"), ("affine", 2, 32, 256, "bf16"), ("affine", 3, 32, 64, "bf16"),
    ("affine", 3, 128, 256, "f16"), ("affine", 5, 64, 128, "bf16"), ("affine", 5, 32, 64, "f16"),
    ("affine", 6, 32, 128, "f16"), ("affine", 6, 128, 256, "bf16"),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c)))
@pytest.mark.parametrize("kind", ["uniform", "normal", "wide", "special", "halfway"])
def test_quantize_update_bit_exact(qkv, case, kind):
    fmt, bits, gs, D, dtype = case
    B, Hkv, Lnew, Lcap, offset = 2, 3, 37, 64, 19
    nk = _inputs((B, Hkv, Lnew, D), kind, dtype, 1, fmt, bits, gs)
    nv = _inputs((B, Hkv, Lnew, D), kind, dtype, 2, fmt, bits, gs)
    from quantized_kv_attention_split_b200.qkv import QuantCache, AFFINE, Q8_0
    f = Q8_0 if fmt == "q8_0" else AFFINE
    kd = QuantCache.empty(B, Hkv, Lcap, D, f, bits, gs)
    vd = QuantCache.empty(B, Hkv, Lcap, D, f, bits, gs)
    qkv.qkv_quantize_update(to_dev(nk, dtype), to_dev(nv, dtype), kd, vd, offset)
    torch.cuda.synchronize()
    for got_d, src in ((kd, nk), (vd, nv)):
        got = cache_from_dev(got_d, fmt)
        ref = oracle.quantize(src, dtype, fmt, gs, bits)
        sl = slice(offset, offset + Lnew)
        assert np.array_equal(got.codes[:, :, sl], ref.codes)
        assert np.array_equal(got.scales[:, :, sl], ref.scales)
        if fmt == "affine":
            assert np.array_equal(got.biases[:, :, sl], ref.biases)
        # nothing written outside the target rows
        assert not got.codes[:, :, :offset].any() and not got.codes[:, :, offset + Lnew:].any()
        assert not got.scales[:, :, :offset].any() and not got.scales[:, :, offset + Lnew:].any()


def test_single_token_update_matches_bulk(qkv):
    """Appending tokens one at a time gives the same cache as one bulk call."""
    from quantized_kv_attention_split_b200.qkv import QuantCache
    B, Hkv, D, Ln = 1, 8, 128, 24
    nk = _inputs((B, Hkv, Ln, D), "normal", "f16", 5)
    nv = _inputs((B, Hkv, Ln, D), "normal", "f16", 6)
    a_k, a_v = QuantCache.empty(B, Hkv, 32, D, bits=8), QuantCache.empty(B, Hkv, 32, D, bits=8)
    b_k, b_v = QuantCache.empty(B, Hkv, 32, D, bits=8), QuantCache.empty(B, Hkv, 32, D, bits=8)
    qkv.qkv_quantize_update(to_dev(nk, "f16"), to_dev(nv, "f16"), a_k, a_v, 3)
    for i in range(Ln):
        qkv.qkv_quantize_update(to_dev(nk[:, :, i:i + 1].copy(), "f16"),
                                to_dev(nv[:, :, i:i + 1].copy(), "f16"), b_k, b_v, 3 + i)
    torch.cuda.synchronize()
    for x, y in ((a_k, b_k), (a_v, b_v)):
        assert torch.equal(x.codes, y.codes) and torch.equal(x.scales, y.scales)
        assert torch.equal(x.biases, y.biases)


def test_quantize_rejects_bad_offset(qkv):
    from quantized_kv_attention_split_b200.qkv import QuantCache
    kd, vd = QuantCache.empty(1, 1, 16, 64), QuantCache.empty(1, 1, 16, 64)
    x = torch.zeros(1, 1, 4, 64, dtype=torch.float16, device="cuda")
    with pytest.raises(qkv.QKVError, match="offset"):
        qkv.qkv_quantize_update(x, x, kd, vd, 13)
