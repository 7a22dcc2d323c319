"""Pins for the oracle's conversion between llama.cpp-style interleaved Q8_0
blocks (34 bytes: fp16 scale, then 32 int8 codes) and the library's planes
(CPU only): a hand-derived block, the dequantized values read straight from
the block bytes, and round trips."""
import numpy as np

from conftest import read_golden
from quantized_kv_attention_split_b200 import synthetic as S


def test_golden_block(orc):
    plane = read_golden("q8_0_block.txt")
    blk = read_golden("q8_0_aos_block.txt")
    raw = np.array([int(x, 16) for x in blk["block"]], np.uint8).reshape(1, 1, 1, 1, 34)
    c = orc.q8_0_from_blocks(raw)
    assert c.scales[0, 0, 0, 0] == int(plane["scale_bits"][0], 16)
    assert [int(w) for w in c.codes[0, 0, 0]] == [int(w, 16) for w in plane["words"]]
    assert np.array_equal(orc.q8_0_to_blocks(c, 1), raw)
    # the block's values are its codes times 1/8
    vals = orc.dequantize(c, 32)[0, 0, 0]
    assert np.array_equal(vals, np.array([int(x) for x in plane["codes"]]) / 8.0)


def test_block_bytes_give_the_dequantized_values(orc):
    B, Hkv, L, D = 2, 3, 21, 128
    x = S.draw(51, "x", (B, Hkv, L, D), "normal", "f16")
    c = orc.quantize(x, "f16", "q8_0")
    blocks = orc.q8_0_to_blocks(c, L)
    d = blocks[..., 0:2].copy().view(np.float16)[..., 0].astype(np.float64)   # little-endian fp16
    q = blocks[..., 2:].view(np.int8).astype(np.float64)
    direct = (d[..., None] * q).reshape(B, Hkv, L, D)
    assert np.array_equal(direct, orc.dequantize(c, D))


def test_round_trips(orc):
    B, Hkv, L, D = 1, 2, 40, 256
    x = S.draw(52, "x", (B, Hkv, L, D), "normal", "bf16")
    c = orc.quantize(x, "bf16", "q8_0")
    back = orc.q8_0_from_blocks(orc.q8_0_to_blocks(c, L), Lcap=L)
    assert np.array_equal(back.codes, c.codes) and np.array_equal(back.scales, c.scales)
    rng = np.random.default_rng(0)
    raw = rng.integers(0, 256, (2, 1, 5, 4, 34), dtype=np.uint8)
    assert np.array_equal(orc.q8_0_to_blocks(orc.q8_0_from_blocks(raw, Lcap=8), 5), raw)


import pytest


@pytest.mark.parametrize("kind", ["q4_0", "q4_1", "q5_0", "q5_1"])
def test_llama_block_golden_values(orc, kind):
    g = read_golden("llama_blocks.txt")
    raw = np.array([int(x, 16) for x in g[kind + "_block"]], np.uint8).reshape(1, 1, 1, 1, -1)
    want = np.array([float(v) for v in g[kind + "_values"]])
    assert np.array_equal(orc.llama_block_values(kind, raw).ravel(), want)
    # the affine cache it becomes holds exactly these values
    c = orc.llama_blocks_to_cache(kind, raw)
    assert c.bits == (4 if kind.startswith("q4") else 8) and c.gs == 32
    assert np.array_equal(orc.dequantize(c, 32).ravel(), want)


@pytest.mark.parametrize("kind", ["q4_0", "q4_1", "q5_0", "q5_1"])
def test_llama_blocks_to_cache_keeps_every_value(orc, kind):
    nbytes = orc.LLAMA_BLOCKS[kind][0]
    rng = np.random.default_rng(7)
    B, Hkv, L, nb = 2, 3, 9, 4
    raw = rng.integers(0, 256, (B, Hkv, L, nb, nbytes), dtype=np.uint8)
    # finite fp16 d (and m): drawn values, stored little-endian
    d = S.f32_to_half_bits(rng.uniform(-3, 3, (B, Hkv, L, nb)).astype(np.float32), "f16")
    raw[..., 0] = d & 0xFF
    raw[..., 1] = d >> 8
    if orc.LLAMA_BLOCKS[kind][1]:
        m = S.f32_to_half_bits(rng.uniform(-3, 3, (B, Hkv, L, nb)).astype(np.float32), "f16")
        raw[..., 2] = m & 0xFF
        raw[..., 3] = m >> 8
    c = orc.llama_blocks_to_cache(kind, raw, Lcap=16)
    vals = orc.llama_block_values(kind, raw)
    assert np.array_equal(orc.dequantize(c, 32 * nb)[:, :, :L], vals)
    assert not c.codes[:, :, L:].any()
