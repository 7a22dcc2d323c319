"""GPU parity of the attention extensions (qsdpa_decode_ext / qsdpa_prefill_ext:
logit softcap, attention sinks, per-head additive-mask slopes for ALiBi)
against the oracle, through the C ABI.  Decode runs the split-K kernel's
extension variant (whole-unit CTAs normalize with the sink themselves, split
units in the merge kernel); prefill runs the tcgen05 kernel for 16-bit output
and >= 64 rows per kv head, and the split-K kernel for fp32 output."""
import math

import numpy as np
import pytest
import torch

import oracle
from helpers import TORCH_DT, cache_to_dev, from_dev, make_problem, max_err, out_err, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def qkv():
    from quantized_kv_attention_split_b200 import qkv as m
    m.lib()
    return m


def _alibi_slopes(Hq):
    # Press et al.: 2^(-8(h+1)/n) for the nearest power of two n <= Hq, then the
    # odd-indexed slopes of the 2n schedule for the remaining heads
    n = 2 ** int(math.floor(math.log2(Hq)))
    s = [2.0 ** (-8.0 * (h + 1) / n) for h in range(n)]
    s += [2.0 ** (-4.0 * (2 * h + 1) / n) for h in range(Hq - n)]
    return np.array(s, np.float32)


def _sinks(Hq, L):
    # comparable to the softmax denominator, so that the sink matters
    return (math.log(max(L, 1)) + np.linspace(-3.0, 3.0, Hq)).astype(np.float32)


def _ext(Hq, L, softcap, use_sinks, use_slopes):
    sinks = _sinks(Hq, L) if use_sinks else None
    slopes = _alibi_slopes(Hq) if use_slopes else None
    dev = lambda a: None if a is None else torch.from_numpy(a).cuda()
    orc = oracle.Ext(softcap=softcap,
                     sinks=None if sinks is None else sinks.astype(np.float64),
                     slopes=None if slopes is None else slopes.astype(np.float64))
    return dict(softcap=softcap, sinks=dev(sinks), mask_slopes=dev(slopes)), orc


DEC_CASES = [
    # B, Hq, Hkv, D, L, fmt, bits, gs, q dtype, out dtype, softcap, sinks, alibi
    (1, 32, 8, 128, 5000, "affine", 4, 64, "f16", "f16", 2.0, False, False),
    (1, 32, 8, 128, 20000, "affine", 4, 64, "f16", "f16", 0.0, True, False),
    (8, 64, 32, 128, 200, "affine", 4, 64, "f16", "f16", 2.0, True, True),
    (2, 16, 2, 64, 3000, "affine", 4, 32, "bf16", "bf16", 0.0, False, True),
    (1, 32, 2, 256, 4000, "q8_0", 8, 32, "f16", "f32", 3.0, True, True),
    (1, 48, 1, 128, 2500, "affine", 8, 64, "f16", "f16", 5.0, True, True),
    (1, 8, 2, 128, 1, "affine", 4, 64, "f16", "f16", 1.0, True, False),
]


@pytest.mark.parametrize("case", DEC_CASES, ids=lambda c: "-".join(map(str, c)))
def test_decode_extensions_match_oracle(qkv, case):
    B, Hq, Hkv, D, L, fmt, bits, gs, qdt, odt, cap, use_sinks, alibi = case
    q, kc, vc = make_problem(B, Hq, Hkv, 1, D, L, fmt, bits, gs, "normal", q_dtype=qdt, seed=41)
    scale = 3.0 / math.sqrt(D)
    kw, ext = _ext(Hq, L, cap, use_sinks, alibi)
    mask_o = mask_d = None
    if alibi:
        dist = -np.abs(np.arange(L) - (L - 1)).astype(np.float32)   # the query sits at L - 1
        mask_o = oracle.Mask("additive", dist, "f32", (0, 0, 0))
        mask_d = (torch.from_numpy(dist).cuda(), (0, 0, 0))
    ref = oracle.attention(q, qdt, kc, vc, L, scale, mask=mask_o, ext=ext)
    out = qkv.qsdpa_decode(to_dev(q, qdt), cache_to_dev(kc), cache_to_dev(vc), L, scale,
                           mask=mask_d, out_dtype=TORCH_DT[odt], **kw)
    torch.cuda.synchronize()
    got = from_dev(out)
    assert out_err(got, ref, odt) <= 1.0, (max_err(got, ref), out_err(got, ref, odt))
    # the extension changes the result (the case tests something)
    plain = oracle.attention(q, qdt, kc, vc, L, scale)
    if L > 1:
        assert max_err(plain, ref) > 1e-2


def test_decode_sink_only_row_without_keys_is_zero(qkv):
    """A fully masked row stays zero with a sink (no value row is attached to it)."""
    B, Hq, Hkv, D, L = 1, 8, 2, 128, 700
    q, kc, vc = make_problem(B, Hq, Hkv, 1, D, L, "affine", 4, 64, "normal", seed=42)
    m = torch.full((L,), float("-inf"), device="cuda")
    kw, _ = _ext(Hq, L, 0.0, True, False)
    out = qkv.qsdpa_decode(to_dev(q, "f16"), cache_to_dev(kc), cache_to_dev(vc), L, 0.1,
                           mask=(m, (0, 0, 0)), **kw)
    torch.cuda.synchronize()
    assert torch.count_nonzero(out).item() == 0


PF_CASES = [
    # B, Hq, Hkv, Lq, D, L, fmt, bits, gs, out dtype, causal, softcap, sinks, alibi
    (1, 32, 2, 128, 256, 2048, "q8_0", 8, 32, "bf16", True, 2.0, True, False),
    (1, 8, 2, 64, 128, 700, "affine", 4, 64, "f16", True, 0.0, True, True),
    (1, 8, 2, 32, 128, 300, "q8_0", 8, 32, "bf16", False, 0.0, True, False),
    (2, 4, 1, 40, 64, 333, "affine", 8, 32, "f16", False, 4.0, False, False),
    (1, 8, 2, 20, 128, 257, "affine", 8, 64, "f32", True, 2.0, True, True),
]


@pytest.mark.parametrize("case", PF_CASES, ids=lambda c: "-".join(map(str, c)))
def test_prefill_extensions_match_oracle(qkv, case):
    B, Hq, Hkv, Lq, D, L, fmt, bits, gs, odt, causal, cap, use_sinks, alibi = case
    q, kc, vc = make_problem(B, Hq, Hkv, Lq, D, L, fmt, bits, gs, "normal", q_dtype="bf16",
                             Lcap=(L // 8 + 3) * 8, seed=43)
    # the plain prefill parity tests' scale: the tcgen05 kernel reads K as fp16
    # (11-bit significand), so its logit error grows with the logits' size
    scale = 1.0 / math.sqrt(D)
    kw, ext = _ext(Hq, L, cap, use_sinks, alibi)
    if alibi:
        # ALiBi distance of query i (position L - Lq + i) to key j; causal
        # positions hidden by -inf in the same additive mask
        pos = L - Lq + np.arange(Lq)[:, None]
        j = np.arange(L)[None, :]
        m = -np.abs(pos - j).astype(np.float32)
        if causal:
            m[j > pos] = -np.inf
        mask_o = oracle.Mask("additive", m, "f32", (0, 0, L))
        mask_d = (torch.from_numpy(m).cuda(), (0, 0, L))
        causal_d = False
    else:
        mask_o = oracle.Mask("causal") if causal else None
        mask_d = None
        causal_d = causal
    ref = oracle.attention(q, "bf16", kc, vc, L, scale, mask=mask_o, ext=ext)
    out = qkv.qsdpa_prefill(to_dev(q, "bf16"), cache_to_dev(kc), cache_to_dev(vc), L, scale,
                            mask=mask_d, causal=causal_d, out_dtype=TORCH_DT[odt], **kw)
    torch.cuda.synchronize()
    got = from_dev(out)
    assert out_err(got, ref, odt) <= 1.0, (max_err(got, ref), out_err(got, ref, odt))
    plain = oracle.attention(q, "bf16", kc, vc, L, scale, mask=mask_o)
    assert max_err(plain, ref) > 1e-2

