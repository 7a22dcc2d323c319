"""Pins for the oracle's llama.cpp block formats (CPU only):
 * Q8_0 blocks (34 bytes: fp16 scale, then 32 int8 codes) <-> the library's
   planes: a hand-derived block, the dequantized values read straight from the
   block bytes, round trips;
 * Q4_0/Q4_1/Q5_0/Q5_1 blocks: hand-built blocks and their values, the affine
   caches that hold exactly those values;
 * the reference quantizers for those blocks: the hand-built blocks are fixed
   points, and a per-element error bound."""
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


@pytest.mark.parametrize("kind", ["q4_0", "q4_1", "q5_0", "q5_1"])
def test_llama_quantizer_reproduces_the_hand_built_blocks(orc, kind):
    """Each hand-built block's values quantize back to exactly that block: its
    scale (and minimum) is what the reference quantizer derives from them, and
    every value sits on a code."""
    g = read_golden("llama_blocks.txt")
    raw = np.array([int(x, 16) for x in g[kind + "_block"]], np.uint8)
    vals = np.array([float(v) for v in g[kind + "_values"]], np.float32)
    x = S.f32_to_half_bits(vals, "f16")[None, :]
    assert np.array_equal(orc.llama_quantize_blocks(kind, x)[0, 0], raw)


@pytest.mark.parametrize("kind", ["q4_0", "q4_1", "q5_0", "q5_1"])
@pytest.mark.parametrize("dist", ["normal", "uniform"])
def test_llama_quantizer_error_bound(orc, kind, dist):
    """|x - xhat| <= the step (Q4_0/Q5_0: the code range is clamped on one
    side, so up to one step; Q4_1/Q5_1: half a step) plus what storing d and m
    in fp16 moves the levels."""
    D = 256
    x = S.draw(95, "x", (40, D), dist, "f16")
    blocks = orc.llama_quantize_blocks(kind, x)
    xh = orc.llama_block_values(kind, blocks)
    xf = orc.to_f64(x, "f16")
    nbytes, has_m, _, off, _ = orc.LLAMA_BLOCKS[kind]
    xb = xf.reshape(40, D // 32, 32).astype(np.float32)
    top = 15 if kind.startswith("q4") else 31
    if has_m:
        d = ((xb.max(-1) - xb.min(-1)) / np.float32(top)).astype(np.float64)
        half = 0.5
        lo = xb.min(-1).astype(np.float64)
        m16 = orc.f16_to_f32(blocks[..., 2].astype(np.uint16) | (blocks[..., 3].astype(np.uint16) << 8))
        shift = np.abs(lo - m16.astype(np.float64))
        reach = top
    else:
        i = np.abs(xb).argmax(-1)
        d = (np.take_along_axis(xb, i[..., None], -1)[..., 0] / np.float32(-off)).astype(np.float64)
        # half a step, except where the code would pass the top and is clamped
        t = xb.astype(np.float64) / np.where(d != 0, d, 1.0)[..., None] + off
        half = np.where(t + 0.5 >= top + 1, 1.0, 0.5)
        shift = 0.0
        reach = max(off, top - off)
    d16 = orc.f16_to_f32(blocks[..., 0].astype(np.uint16) | (blocks[..., 1].astype(np.uint16) << 8))
    dd = np.abs(d)[..., None]
    bound = dd * half * (1 + 2.0 ** -20) + (np.abs(d - d16.astype(np.float64)) * reach)[..., None]
    bound = bound + (shift[..., None] if has_m else 0.0)
    err = np.abs(xf - xh).reshape(40, D // 32, 32)
    assert np.all(err <= bound + 1e-12), (err - bound).max()


@pytest.mark.parametrize("kind,d_ok,d_over", [("q4_0", 8188.0, 8192.0), ("q5_0", 4094.0, 4096.0)])
def test_offset_bias_range_limit(orc, kind, d_ok, d_over):
    """The _0 blocks become affine groups with bias -8d (Q4_0) or -16d (Q5_0),
    stored in fp16: exact up to |bias| = 65504 (d = 8188 / 4094), and +-inf
    beyond (d = 8192 / 4096), where the block's own values leave the fp16
    range.  All codes zero: every value equals the bias."""
    nbytes, _, _, off, _ = orc.LLAMA_BLOCKS[kind]
    for d, finite in ((d_ok, True), (d_over, False), (-d_ok, True), (-d_over, False)):
        raw = np.zeros((1, 1, 1, 1, nbytes), np.uint8)
        db = int(S.f32_to_half_bits(np.array([d], np.float32), "f16")[0])
        raw[..., 0], raw[..., 1] = db & 0xFF, db >> 8
        c = orc.llama_blocks_to_cache(kind, raw)
        bias = float(orc.f16_to_f32(c.biases.ravel())[0])
        if finite:
            assert bias == -off * d and abs(bias) == 65504.0
            assert np.array_equal(orc.dequantize(c, 32).ravel(), orc.llama_block_values(kind, raw).ravel())
        else:
            assert np.isinf(bias) and np.sign(bias) == -np.sign(d)
            assert np.all(np.abs(orc.llama_block_values(kind, raw)) > 65504)
