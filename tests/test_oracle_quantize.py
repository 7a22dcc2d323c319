"""Pins for the oracle's conversions and quantizers (CPU only).

Each check ties the oracle to something other than itself: numpy / torch
half-precision conversion, hand-derived packed words (tests/golden), the
quantize-then-dequantize error bound, exact reconstruction of degenerate
groups, brute-force optimality of every code, and the pages' dequant formula
(scale * code + bias; MLX quantized-KV branch, quantized.h / sdpa_vector.h).
"""
import numpy as np
import pytest
import torch

from conftest import read_golden
from quantized_kv_attention_split_b200 import synthetic as S


# --------------------------------------------------------------------------
# conversions vs library routines
# --------------------------------------------------------------------------
def test_f16_roundtrip_all_patterns(orc):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    mine = orc.f16_to_f32(bits)
    ref = bits.view(np.float16).astype(np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan)
    assert np.array_equal(mine[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_f32_to_f16_matches_numpy(orc):
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(200000).astype(np.float32) * np.float32(3.0),
        (rng.random(100000) * 2.0 ** rng.integers(-30, 17, 100000)).astype(np.float32),
        np.array([0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e9, -1e9, 2.0 ** -24,
                  2.0 ** -25, 3 * 2.0 ** -26, 2.0 ** -14, np.inf, -np.inf, 1e-7], np.float32),
    ])
    # exact ties between halves: midpoints of adjacent half values
    h = rng.integers(0, 0x7bff, 50000).astype(np.uint16)
    lo = h.view(np.float16).astype(np.float64)
    hi = (h + 1).view(np.float16).astype(np.float64)
    x = np.concatenate([x, ((lo + hi) / 2).astype(np.float32)])
    assert np.array_equal(orc.f32_to_f16(x), x.astype(np.float16).view(np.uint16))


def test_bf16_matches_torch(orc):
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(100000).astype(np.float32),
        (rng.random(50000) * 2.0 ** rng.integers(-120, 120, 50000)).astype(np.float32),
        np.array([0.0, -0.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 3.4e38], np.float32),
    ])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(orc.f32_to_bf16(x), ref)
    back = orc.bf16_to_f32(ref)
    assert np.array_equal(back, torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16)
                          .float().numpy())


def test_synthetic_bf16_rounding_matches_torch():
    x = S.normal(7, 20000)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(S.f32_to_half_bits(x, "bf16"), ref)


# --------------------------------------------------------------------------
# golden fixtures (hand-derived from the pages' packing rules)
# --------------------------------------------------------------------------
def _golden_input(g):
    if "values" in g:
        vals = []
        for t in g["values"]:
            if "*" in t:
                v, n = t.split("*")
                vals += [float(v)] * int(n)
            else:
                vals.append(float(t))
        x = np.array(vals, np.float32)
    else:
        x = np.array([int(c) for c in g["codes"]], np.float32) / np.float32(
            float(g["value_divisor"][0]))
    return S.f32_to_half_bits(x, g["dtype"][0])[None, :]


@pytest.mark.parametrize("name", ["affine4_ramp.txt", "affine8_bytes.txt",
                                  "q8_0_block.txt", "affine4_constant.txt",
                                  "affine2_ramp.txt", "affine3_ramp.txt",
                                  "affine5_ramp.txt", "affine6_ramp.txt"])
def test_golden_packing(orc, name):
    g = read_golden(name)
    x = _golden_input(g)
    c = orc.quantize(x, g["dtype"][0], g["format"][0], int(g["group_size"][0]),
                     int(g["bits"][0]))
    words = np.array([int(w, 16) for w in g["words"]], np.uint32)
    assert np.array_equal(c.codes[0], words), [hex(w) for w in c.codes[0]]
    assert c.scales[0, 0] == int(g["scale_bits"][0], 16)
    if "bias_bits" in g:
        assert c.biases[0, 0] == int(g["bias_bits"][0], 16)
    # and dequantization reproduces the input exactly in these cases
    xd = orc.dequantize(c, x.shape[1])
    assert np.array_equal(xd[0], x.view(np.float16).astype(np.float64)[0])


# --------------------------------------------------------------------------
# properties of the quantizers
# --------------------------------------------------------------------------
def _unpack(codes, bits, D, signed=False):
    """Element e at bits [e*bits, (e+1)*bits) of the row's little-endian bit
    stream (for 2, 4 and 8 bits: element j of a word at bits [j*bits, ...))."""
    e = np.arange(D)
    pos = e * bits
    lo = codes[..., pos // 32].astype(np.uint64)
    hi_idx = np.minimum(pos // 32 + 1, codes.shape[-1] - 1)
    hi = codes[..., hi_idx].astype(np.uint64)
    both = lo | (hi << np.uint64(32))                 # 64-bit window over two words
    f = (both >> (pos % 32).astype(np.uint64)) & np.uint64((1 << bits) - 1)
    f = f.astype(np.int64)
    if signed:
        f = np.where(f >= 128, f - 256, f)
    return f


def _groups(seed, rows, D, kind, dtype="f16"):
    rng = np.random.default_rng(seed)
    if kind == "uniform":
        x = rng.random((rows, D)).astype(np.float32)
    elif kind == "normal":
        x = rng.standard_normal((rows, D)).astype(np.float32)
    elif kind == "wide":
        x = (rng.standard_normal((rows, D)) * 10.0 ** rng.uniform(-3, 3, (rows, 1))).astype(
            np.float32)
    elif kind == "offset":       # narrow spread far from zero
        x = (100.0 + rng.random((rows, D)) * 0.01).astype(np.float32)
    return S.f32_to_half_bits(x, dtype)


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 8])
@pytest.mark.parametrize("gs", [32, 64, 128])
@pytest.mark.parametrize("kind", ["uniform", "normal", "wide", "offset"])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_affine_error_bound_and_optimality(orc, bits, gs, kind, dtype):
    D = 128
    x = _groups(bits * 1000 + gs + len(kind), 64, D, kind, dtype)
    c = orc.quantize(x, dtype, "affine", gs, bits)
    xf = orc.to_f64(x, dtype)
    sf = orc.to_f64(c.scales, "f16")          # [rows, NG]
    bf = orc.to_f64(c.biases, "f16")
    q = _unpack(c.codes, bits, D)
    sfe = np.repeat(sf, gs, axis=1)
    bfe = np.repeat(bf, gs, axis=1)
    # pages' dequant formula: scale * code + bias
    xd = orc.dequantize(c, D)
    assert np.array_equal(xd, sfe * q + bfe)
    # bound |x - xhat| <= scale/2 (plus fp32 rounding of the division)
    err = np.abs(xf - xd)
    assert np.all(err <= sfe / 2 * (1 + 2.0 ** -20) + 1e-300), err.max()
    # each code is the best code for its element (brute force over all codes)
    levels = np.arange(1 << bits)
    best = np.abs(xf[..., None] - (sfe[..., None] * levels + bfe[..., None])).min(-1)
    assert np.all(err <= best * (1 + 2.0 ** -20) + 1e-300)
    # min-max reading: bias is the group minimum, and the maximum maps to the top
    # code unless the group is constant
    xg = xf.reshape(64, D // gs, gs)
    assert np.array_equal(bf, orc.to_f64(S.f32_to_half_bits(xg.min(-1).astype(np.float32),
                                                           "f16"), "f16"))
    qg = q.reshape(64, D // gs, gs)
    assert np.all(qg.min(-1) == 0)
    nonconst = xg.max(-1) > xg.min(-1)
    assert np.all(qg.max(-1)[nonconst] == (1 << bits) - 1)


@pytest.mark.parametrize("kind", ["uniform", "normal", "wide"])
def test_q8_0_error_bound_and_optimality(orc, kind):
    D = 256
    x = _groups(77 + len(kind), 64, D, kind, "f16")
    c = orc.quantize(x, "f16", "q8_0")
    assert c.biases is None and c.codes.shape == (64, D // 4) and c.scales.shape == (64, 8)
    xf = orc.to_f64(x, "f16")
    d = np.repeat(orc.to_f64(c.scales, "f16"), 32, axis=1)
    q = _unpack(c.codes, 8, D, signed=True)
    assert q.min() >= -127
    xd = orc.dequantize(c, D)
    assert np.array_equal(xd, d * q)
    err = np.abs(xf - xd)
    assert np.all(err <= d / 2 * (1 + 2.0 ** -20))
    levels = np.arange(-127, 128)
    best = np.abs(xf[..., None] - d[..., None] * levels).min(-1)
    assert np.all(err <= best * (1 + 2.0 ** -20) + 1e-300)
    # the element of largest magnitude in each block maps to +-127
    am = np.abs(xf).reshape(64, 8, 32).argmax(-1)
    qb = q.reshape(64, 8, 32)
    top = np.take_along_axis(qb, am[..., None], -1)[..., 0]
    assert np.all(np.abs(top) == 127)


def test_q8_0_zero_block(orc):
    x = np.zeros((2, 64), np.uint16)
    x[1, 32:] = S.f32_to_half_bits(np.linspace(-1, 1, 32, dtype=np.float32), "f16")
    c = orc.quantize(x, "f16", "q8_0")
    assert c.scales[0, 0] == 0 and c.scales[0, 1] == 0 and c.scales[1, 0] == 0
    assert np.all(c.codes[0] == 0) and np.all(c.codes[1, :8] == 0)
    assert c.scales[1, 1] != 0


def test_affine_constant_groups_reconstruct_exactly(orc):
    rng = np.random.default_rng(5)
    vals = rng.standard_normal(32).astype(np.float32)
    x = S.f32_to_half_bits(np.repeat(vals, 64).reshape(32, 64), "f16")
    for bits in (2, 3, 4, 5, 6, 8):
        c = orc.quantize(x, "f16", "affine", 64, bits)
        assert np.all(c.codes == 0)
        assert np.array_equal(orc.dequantize(c, 64), orc.to_f64(x, "f16"))


def test_affine_requantize_is_idempotent(orc):
    x = _groups(11, 256, 128, "normal")
    c = orc.quantize(x, "f16", "affine", 64, 4)
    xd = orc.dequantize(c, 128)
    xd32 = xd.astype(np.float32)
    exact = np.all(xd32.astype(np.float64) == xd, axis=1)
    c2 = orc.quantize(np.ascontiguousarray(xd32[exact]), "f32", "affine", 64, 4)
    assert exact.sum() > 100
    assert np.array_equal(c2.codes, c.codes[exact])
    assert np.array_equal(c2.scales, c.scales[exact])
    assert np.array_equal(c2.biases, c.biases[exact])


def test_affine_dot_identity(orc):
    """q . xhat == scale*(q . codes) + bias*sum(q) within a group: the identity
    the fused kernel uses for the key bias term (quant_sdpa_vector's
    query_sum in the MLX quantized-KV branch)."""
    x = _groups(12, 16, 128, "uniform")
    c = orc.quantize(x, "f16", "affine", 64, 4)
    rng = np.random.default_rng(3)
    q = rng.random(128)
    xd = orc.dequantize(c, 128)
    codes = _unpack(c.codes, 4, 128)
    s = orc.to_f64(c.scales, "f16")
    b = orc.to_f64(c.biases, "f16")
    for r in range(16):
        lhs = xd[r] @ q
        rhs = sum(s[r, g] * (codes[r, g * 64:(g + 1) * 64] @ q[g * 64:(g + 1) * 64])
                  + b[r, g] * q[g * 64:(g + 1) * 64].sum() for g in range(2))
        assert abs(lhs - rhs) <= 1e-12 * max(1.0, abs(lhs))



@pytest.mark.parametrize("bits", [3, 5, 6])
def test_odd_widths_pack_as_bit_stream(orc, bits):
    """3/5/6-bit codes straddle 32-bit words; every code survives the packing
    and a code's bits never touch its neighbours' (random codes planted through
    values whose group spans exactly 0..2^bits-1)."""
    rng = np.random.default_rng(bits)
    D, gs = 128, 32
    top = (1 << bits) - 1
    q = rng.integers(0, top + 1, (16, D))
    q[:, ::gs] = 0
    q[:, 1::gs] = top                           # each group spans the full code range
    x = S.f32_to_half_bits(q.astype(np.float32), "f16")
    c = orc.quantize(x, "f16", "affine", gs, bits)
    assert c.codes.shape[-1] == D * bits // 32
    assert np.array_equal(_unpack(c.codes, bits, D), q)
    assert np.array_equal(orc.dequantize(c, D), q.astype(np.float64))
