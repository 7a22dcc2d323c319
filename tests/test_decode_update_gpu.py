"""The fused decode step (qsdpa_decode_update) through the C ABI.

It must leave the cache exactly as the two separate calls leave it --
qkv_quantize_update of the new token at row L_old, then qsdpa_decode over
L_old + 1 keys -- with the same output bits, and both must match the oracle:
the cache bytes bit for bit (the quantizer contract) and the output within the
parity tolerance."""
import numpy as np
import pytest
import torch

import oracle
from helpers import cache_from_dev, cache_to_dev, from_dev, make_problem, out_err, to_dev
from quantized_kv_attention_split_b200 import synthetic as S

pytestmark = pytest.mark.gpu

CASES = [
    # B, Hq, Hkv, D, L_old, fmt, bits, gs, new-token dtype, out dtype
    (1, 32, 8, 128, 5000, "affine", 8, 64, "f16", "f16"),
    (1, 32, 8, 128, 4095, "affine", 4, 64, "f16", "f16"),     # new token ends a full block
    (1, 32, 8, 128, 0, "affine", 4, 64, "f16", "f16"),        # the new token is the only key
    (2, 16, 2, 64, 300, "affine", 4, 32, "bf16", "bf16"),
    (1, 8, 1, 128, 777, "affine", 8, 128, "f16", "f32"),
    (1, 32, 2, 256, 3000, "q8_0", 8, 32, "f16", "f32"),
    (1, 48, 1, 128, 2500, "affine", 4, 64, "f16", "f16"),     # two row chunk-groups per kv head
]


def _copy(c):
    from quantized_kv_attention_split_b200 import qkv
    return qkv.QuantCache(c.fmt, c.bits, c.group_size, c.codes.clone(), c.scales.clone(),
                          None if c.biases is None else c.biases.clone())


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c)))
def test_fused_update_decode_matches_two_calls_and_oracle(case):
    from quantized_kv_attention_split_b200 import qkv
    B, Hq, Hkv, D, L_old, fmt, bits, gs, ndt, odt = case
    L = L_old + 1
    dist = "normal" if fmt == "q8_0" else "uniform"
    q, kc, vc = make_problem(B, Hq, Hkv, 1, D, L, fmt, bits, gs, dist, seed=31)
    nk = S.draw(32, "new_k", (B, Hkv, 1, D), dist, ndt)
    nv = S.draw(32, "new_v", (B, Hkv, 1, D), dist, ndt)
    qd = to_dev(q, "f16")
    nkd, nvd = to_dev(nk, ndt), to_dev(nv, ndt)
    tdt = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}[odt]

    # two calls
    k2, v2 = cache_to_dev(kc), cache_to_dev(vc)
    qkv.qkv_quantize_update(nkd, nvd, k2, v2, L_old)
    ref2 = qkv.qsdpa_decode(qd, k2, v2, L, 0.0625, out_dtype=tdt)
    # fused
    k1, v1 = cache_to_dev(kc), cache_to_dev(vc)
    out = qkv.qsdpa_decode_update(qd, nkd, nvd, k1, v1, L_old, 0.0625, out_dtype=tdt)
    torch.cuda.synchronize()

    for a, b in ((k1, k2), (v1, v2)):
        assert torch.equal(a.codes, b.codes)
        assert torch.equal(a.scales.view(torch.int16), b.scales.view(torch.int16))
        if a.biases is not None:
            assert torch.equal(a.biases.view(torch.int16), b.biases.view(torch.int16))
    assert torch.equal(out.view(torch.int16 if odt != "f32" else torch.int32),
                       ref2.view(torch.int16 if odt != "f32" else torch.int32))

    # oracle: the new row bit for bit, the output within tolerance
    nq_k = oracle.quantize(nk, ndt, fmt, gs, bits)
    nq_v = oracle.quantize(nv, ndt, fmt, gs, bits)
    hk, hv = cache_from_dev(k1, fmt), cache_from_dev(v1, fmt)
    for h, nqc in ((hk, nq_k), (hv, nq_v)):
        assert np.array_equal(h.codes[:, :, L_old], nqc.codes[:, :, 0])
        assert np.array_equal(h.scales[:, :, L_old], nqc.scales[:, :, 0])
        if h.biases is not None:
            assert np.array_equal(h.biases[:, :, L_old], nqc.biases[:, :, 0])
    ref = oracle.attention(q, "f16", hk, hv, L, 0.0625)
    assert out_err(from_dev(out), ref, odt) <= 1.0


def test_fused_update_rejects_a_full_cache():
    from quantized_kv_attention_split_b200 import qkv
    q, kc, vc = make_problem(1, 8, 2, 1, 128, 64, "affine", 4, 64)
    qd = to_dev(q, "f16")
    kd, vd = cache_to_dev(kc), cache_to_dev(vc)
    n = torch.zeros(1, 2, 1, 128, dtype=torch.float16, device="cuda")
    with pytest.raises(qkv.QKVError, match="Lcap"):
        qkv.qsdpa_decode_update(qd, n, n, kd, vd, kd.Lcap, 1.0)
