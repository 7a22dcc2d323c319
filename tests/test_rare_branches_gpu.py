"""GPU parity on inputs built to drive the kernels' rare numeric paths, which
homogeneous U[0,1) / N(0,1) caches never reach:

* decode, value-scale growth: the value operand of the decode kernel carries
  a per-warp power of two 2^tau sized by the largest value scale seen so far;
  a later block with a larger scale lowers tau and rescales the accumulated
  output by the exact power of two.  Value rows here carry spikes whose
  magnitude grows from 2^-10 to 2^12 along the cache (a spike every 97 rows),
  so every warp of every CTA of a split unit meets larger scales mid-stream.
* decode, moving maximum: the running maximum moves only when a block's
  logit exceeds it by more than 8 (base 2); the rescale of the output, the
  sum and the bias terms runs only then.  Isolated keys whose logits stand
  about 11 (base 2) above the rest, placed all along the cache (so in CTAs
  other than a unit's first and past their first block), and a ramp of key
  magnitudes that makes each warp move its maximum every block or two.
* prefill (tcgen05 kernel), moving maximum: the same spikes and ramp; the
  softmax threads rescale O in tensor memory when the maximum moves by more
  than 8 (base 2).

Each case runs on the plain decode kernel (the one the benchmark times) with
fp16 output (max-abs 2e-3) and fp32 output (1e-4) against the CPU oracle,
element by element, for affine 4-bit, affine 8-bit and Q8_0 caches at the
full decode benchmark shape (L = 65536, 32 query heads over 8 KV heads, so
each KV head is split over many CTAs)."""
import numpy as np
import pytest
import torch

import oracle
from helpers import TOL, TORCH_DT, cache_to_dev, from_dev, max_err, out_err, to_dev
from quantized_kv_attention_split_b200 import synthetic as S

pytestmark = pytest.mark.gpu

FORMATS = [("affine", 4, 64), ("affine", 8, 64), ("q8_0", 8, 32)]
B, HQ, HKV, D, L = 1, 32, 8, 128, 65536
SCALE = 1.0 / np.sqrt(D)


@pytest.fixture(scope="module")
def qkv():
    from quantized_kv_attention_split_b200 import qkv as m
    m.lib()
    return m


def _check_decode(qkv, q, kc, vc, L_, scale):
    ref = oracle.attention(q, "f16", kc, vc, L_, scale)
    qd, kd, vd = to_dev(q, "f16"), cache_to_dev(kc), cache_to_dev(vc)
    for odt in ("f16", "f32"):
        out = qkv.qsdpa_decode(qd, kd, vd, L_, scale, out_dtype=TORCH_DT[odt])
        torch.cuda.synchronize()
        got = from_dev(out)
        assert max_err(got, ref) <= TOL[odt], (odt, max_err(got, ref))
    return ref


@pytest.mark.parametrize("fmt,bits,gs", FORMATS)
def test_decode_value_scales_grow_along_the_cache(qkv, fmt, bits, gs):
    q = S.draw(31, "q", (B, HQ, 1, D), "uniform", "f16")
    k = S.draw(31, "k", (B, HKV, L, D), "uniform", "f16")
    v = S.value_spikes(31, (B, HKV, L, D), "f16", period=97, lo_exp=-10.0, hi_exp=12.0, gs=gs)
    kc = oracle.quantize(k, "f16", fmt, gs, bits)
    vc = oracle.quantize(v, "f16", fmt, gs, bits)
    ref = _check_decode(qkv, q, kc, vc, L, SCALE)
    # the spikes matter: the outputs are far from those of the spike-free rows
    assert np.abs(ref).max() > 1.5


@pytest.mark.parametrize("fmt,bits,gs", FORMATS)
def test_decode_isolated_logit_jumps(qkv, fmt, bits, gs):
    """24 keys whose logits stand ~11 (base 2) above the rest: together they
    weigh about as much as the other 65512 keys, so both the rescaled
    accumulators from before each jump and the spike rows show in the
    output."""
    q = S.draw(32, "q", (B, HQ, 1, D), "uniform", "f16")
    level = np.zeros(L, np.float32)
    level[S.spike_positions(32, L, 24, lo=2048)] = 1.84
    k = S.key_levels(32, (B, HKV, L, D), "f16", level, noise=1.0)
    k_spike = S.key_levels(33, (B, HKV, L, D), "f16", level, noise=0.1)
    k = np.where(level[None, None, :, None] > 0, k_spike, k)
    v = S.draw(32, "v", (B, HKV, L, D), "uniform", "f16")
    kc = oracle.quantize(k, "f16", fmt, gs, bits)
    vc = oracle.quantize(v, "f16", fmt, gs, bits)
    probs, _ = oracle.attention_probs(q, "f16", kc, vc, L, SCALE, 0, 0, 0)
    spike_mass = probs[level > 0].sum()
    assert 0.2 < spike_mass < 0.8, spike_mass                 # both parts weigh
    _check_decode(qkv, q, kc, vc, L, SCALE)


@pytest.mark.parametrize("fmt,bits,gs", FORMATS)
def test_decode_logit_ramp(qkv, fmt, bits, gs):
    """Key magnitudes grow linearly along the cache, so the logits rise by
    about 8 (base 2) every 700 keys: each warp moves its maximum every block
    or two, in every CTA of a unit."""
    q = S.draw(34, "q", (B, HQ, 1, D), "uniform", "f16")
    level = (92.0 * np.arange(L) / L).astype(np.float32)
    k = S.key_levels(34, (B, HKV, L, D), "f16", level, noise=0.25)
    v = S.draw(34, "v", (B, HKV, L, D), "uniform", "f16")
    kc = oracle.quantize(k, "f16", fmt, gs, bits)
    vc = oracle.quantize(v, "f16", fmt, gs, bits)
    _check_decode(qkv, q, kc, vc, L, SCALE)


# ---------------------------------------------------------------------------
# prefill (tcgen05 kernel: >= 64 rows per KV head, 16-bit output)
# ---------------------------------------------------------------------------
PB, PHQ, PHKV, PLQ, PD, PL = 1, 16, 2, 256, 128, 6000


@pytest.mark.parametrize("fmt,bits,gs", [("affine", 4, 64), ("q8_0", 8, 32)])
@pytest.mark.parametrize("shape", ["spikes", "ramp"])
@pytest.mark.parametrize("causal", [False, True])
def test_prefill_moving_maximum(qkv, fmt, bits, gs, shape, causal):
    q = S.draw(35, "q", (PB, PHQ, PLQ, PD), "uniform", "bf16")
    if shape == "spikes":
        level = np.zeros(PL, np.float32)
        level[S.spike_positions(35, PL, 12, lo=300)] = 1.84
        noise = 0.1
    else:
        level = (92.0 * np.arange(PL) / 65536).astype(np.float32)
        noise = 0.25
    k = S.key_levels(35, (PB, PHKV, PL, PD), "f16", level, noise=noise)
    if shape == "spikes":
        bulk = S.key_levels(36, (PB, PHKV, PL, PD), "f16", level * 0, noise=1.0)
        k = np.where(level[None, None, :, None] > 0, k, bulk)
    v = S.draw(35, "v", (PB, PHKV, PL, PD), "uniform", "f16")
    kc = oracle.quantize(k, "f16", fmt, gs, bits)
    vc = oracle.quantize(v, "f16", fmt, gs, bits)
    mask = oracle.Mask("causal") if causal else None
    ref = oracle.attention(q, "bf16", kc, vc, PL, SCALE, mask=mask)
    qd, kd, vd = to_dev(q, "bf16"), cache_to_dev(kc), cache_to_dev(vc)
    for odt in ("bf16", "f16"):
        out = qkv.qsdpa_prefill(qd, kd, vd, PL, SCALE, causal=causal, out_dtype=TORCH_DT[odt])
        torch.cuda.synchronize()
        got = from_dev(out)
        assert out_err(got, ref, odt) <= 1.0, (odt, max_err(got, ref))


# ---------------------------------------------------------------------------
# caches whose dequantized values leave the fp16 range
# ---------------------------------------------------------------------------
def _scaled_problem(fmt, bits, gs, ek, ev, L_, Hq, Hkv, Lq, D, seed):
    """bf16 q * 2^-ek, K * 2^ek, V * 2^ev (exact power-of-two scalings of
    bf16 draws): the logits are those of the unscaled problem and the output
    is 2^ev times its output.  K and V are N(0,1) for Q8_0 and U[0,1) for
    the affine format (whose fp16 bias, the group minimum, must stay finite)."""
    dist = "normal" if fmt == "q8_0" else "uniform"
    Lcap = (L_ + 7) // 8 * 8 + 8                   # rows past L hold values too
    q = S.draw(seed, "q", (1, Hq, Lq, D), "normal", "bf16")
    k = S.draw(seed, "k", (1, Hkv, Lcap, D), dist, "bf16")
    v = S.draw(seed, "v", (1, Hkv, Lcap, D), dist, "bf16")
    f = lambda x, e: S.f32_to_half_bits(oracle.bf16_to_f32(x) * np.float32(2.0 ** e), "bf16")
    q, k, v = f(q, -ek), f(k, ek), f(v, ev)
    kc = oracle.quantize(k, "bf16", fmt, gs, bits)
    vc = oracle.quantize(v, "bf16", fmt, gs, bits)
    return q, kc, vc


@pytest.mark.parametrize("fmt,bits,gs,ek,ev", [("q8_0", 8, 32, 14, 15), ("affine", 8, 64, 17, 17),
                                               ("affine", 4, 32, 17, 17), ("affine", 8, 32, 3, 18)])
def test_values_beyond_the_fp16_range(qkv, fmt, bits, gs, ek, ev):
    """Decode (fp32 scales in the kernel) and the tcgen05 prefill (fp16 tiles:
    each tile is brought below 2^15 by a power of two undone exactly on S and
    O) on caches whose values reach 2^ev * 4 > 65504; both must match the
    oracle to the order-one tolerance once divided by 2^ev."""
    Hq, Hkv, Lq, D, L_ = 8, 2, 64, 128, 700
    q, kc, vc = _scaled_problem(fmt, bits, gs, ek, ev, L_, Hq, Hkv, Lq, D, seed=41)
    kmax = np.abs(oracle.dequantize(kc, D)[:, :, :L_]).max()
    vmax = np.abs(oracle.dequantize(vc, D)[:, :, :L_]).max()
    assert vmax > 65504 and np.isfinite(vmax) and np.isfinite(kmax)
    assert kmax > 65504 or ek < 5                  # the last case keeps K in range
    c = 2.0 ** ev
    scale = 1.0 / np.sqrt(D)
    qd, kd, vd = to_dev(q, "bf16"), cache_to_dev(kc), cache_to_dev(vc)
    for causal in (False, True):
        mask = oracle.Mask("causal") if causal else None
        ref = oracle.attention(q, "bf16", kc, vc, L_, scale, mask=mask)
        out = qkv.qsdpa_prefill(qd, kd, vd, L_, scale, causal=causal, out_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        got = from_dev(out)
        assert np.all(np.isfinite(got))
        assert out_err(got / c, ref / c, "bf16") <= 1.0, (causal, max_err(got / c, ref / c))
    # decode: the last query of every head, fp32 and bf16 output
    q1 = np.ascontiguousarray(q[:, :, -1:])
    ref = oracle.attention(q1, "bf16", kc, vc, L_, scale)
    for odt in ("f32", "bf16"):
        out = qkv.qsdpa_decode(to_dev(q1, "bf16"), kd, vd, L_, scale, out_dtype=TORCH_DT[odt])
        torch.cuda.synchronize()
        got = from_dev(out)
        assert out_err(got / c, ref / c, odt) <= 1.0, (odt, max_err(got / c, ref / c))


def test_prefill_mixed_magnitudes_along_the_cache(qkv):
    """Tiles of very different magnitudes in one cache: keys [0, 200) of
    order one, [200, 450) scaled by 2^14 (values past 65504), [450, 900) by
    2^6, for K and V.  The per-tile K exponent changes from tile to tile and
    the V exponent grows mid-stream (O rescaled by the exact power of two).
    Tolerance: the order-one bound scaled by the largest factor, 2^14."""
    Hq, Hkv, Lq, D, L_ = 8, 2, 64, 128, 904
    q = S.draw(42, "q", (1, Hq, Lq, D), "normal", "bf16")
    Lcap = L_ + 8
    k = oracle.bf16_to_f32(S.draw(42, "k", (1, Hkv, Lcap, D), "normal", "bf16"))
    v = oracle.bf16_to_f32(S.draw(42, "v", (1, Hkv, Lcap, D), "normal", "bf16"))
    e = np.zeros(Lcap, np.float32)
    e[200:450], e[450:] = 14.0, 6.0
    f = np.exp2(e)[None, None, :, None].astype(np.float32)
    qs = S.f32_to_half_bits(oracle.bf16_to_f32(q) * np.float32(2.0 ** -14), "bf16")
    kc = oracle.quantize(S.f32_to_half_bits(k * f, "bf16"), "bf16", "q8_0")
    vc = oracle.quantize(S.f32_to_half_bits(v * f, "bf16"), "bf16", "q8_0")
    scale = 1.0 / np.sqrt(D)
    ref = oracle.attention(qs, "bf16", kc, vc, L_, scale, mask=oracle.Mask("causal"))
    out = qkv.qsdpa_prefill(to_dev(qs, "bf16"), cache_to_dev(kc), cache_to_dev(vc), L_, scale,
                            causal=True, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    got = from_dev(out)
    c = 2.0 ** 14
    assert np.all(np.isfinite(got))
    assert out_err(got / c, ref / c, "bf16") <= 1.0, max_err(got / c, ref / c)
