"""qkv_dequantize (materialize a quantized cache as fp16) through the C ABI:
bit-exact against the correctly rounded fp16 of the oracle's exact (fp64)
dequantization, for every format, over rows [0, L) of a slab with Lcap > L."""
import numpy as np
import pytest
import torch

import oracle
from helpers import cache_to_dev
from quantized_kv_attention_split_b200 import synthetic as S

pytestmark = pytest.mark.gpu

CASES = [
    # B, Hkv, D, L, Lcap, fmt, bits, gs
    (1, 8, 128, 1000, 1024, "affine", 4, 64),
    (2, 2, 64, 77, 80, "affine", 4, 32),
    (1, 3, 256, 300, 304, "affine", 8, 128),
    (1, 2, 128, 513, 520, "affine", 8, 32),
    (1, 2, 256, 640, 640, "q8_0", 8, 32),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c)))
def test_dequantize_is_the_rounded_exact_value(case):
    from quantized_kv_attention_split_b200 import qkv
    B, Hkv, D, L, Lcap, fmt, bits, gs = case
    x = S.draw(41, "x", (B, Hkv, Lcap, D), "normal", "f16")
    c = oracle.quantize(x, "f16", fmt, gs, bits)
    ref = oracle.dequantize(c, D)[:, :, :L].astype(np.float16)
    out = qkv.qkv_dequantize(cache_to_dev(c), L)
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    assert got.shape == ref.shape
    assert np.array_equal(got.view(np.uint16), ref.view(np.uint16))
