"""GPU parity of qsdpa_prefill (multi-query attention) against the oracle.
Calls with >= 64 (head, query) rows per kv head and 16-bit output run on the
tcgen05 kernel; smaller ones and fp32 output on the split-K kernel.  Both are
covered here."""
import numpy as np
import pytest
import torch

import oracle
from helpers import TOL, TORCH_DT, cache_to_dev, from_dev, make_problem, max_err, out_err, to_dev
from quantized_kv_attention_split_b200 import synthetic as S

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def qkv():
    from quantized_kv_attention_split_b200 import qkv as m
    m.lib()
    return m


def run_prefill(qkv, q, q_dtype, kc, vc, L, scale, out_dtype, causal=False, mask=None):
    out = qkv.qsdpa_prefill(to_dev(q, q_dtype), cache_to_dev(kc), cache_to_dev(vc), L, scale,
                            mask=mask, causal=causal, out_dtype=TORCH_DT[out_dtype])
    torch.cuda.synchronize()
    return from_dev(out)


CASES = [
    # B, Hq, Hkv, Lq, D, L, fmt, bits, gs   (rows per kv head = Hq/Hkv * Lq)
    (1, 8, 2, 32, 128, 300, "q8_0", 8, 32),       # 128 rows, tcgen05
    (1, 32, 2, 16, 256, 700, "q8_0", 8, 32),      # 256 rows, tcgen05
    (2, 4, 1, 40, 64, 333, "affine", 4, 64),      # 160 rows (ragged tile)
    (1, 8, 2, 20, 128, 257, "affine", 8, 64),     # 80 rows
    (1, 2, 1, 100, 256, 511, "affine", 4, 32),
    (1, 6, 3, 64, 128, 129, "affine", 4, 128),
    (1, 4, 1, 8, 128, 200, "affine", 4, 64),      # 32 rows: split-K path
    (1, 4, 4, 3, 64, 90, "q8_0", 8, 32),          # 3 rows: split-K path
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c)))
@pytest.mark.parametrize("causal", [False, True])
def test_prefill_matches_oracle(qkv, case, causal):
    B, Hq, Hkv, Lq, D, L, fmt, bits, gs = case
    q, kc, vc = make_problem(B, Hq, Hkv, Lq, D, L, fmt, bits, gs, "normal", q_dtype="bf16",
                             Lcap=(L // 8 + 3) * 8, seed=5)
    scale = 1.0 / np.sqrt(D)
    mask = oracle.Mask("causal") if causal else None
    ref = oracle.attention(q, "bf16", kc, vc, L, scale, mask=mask)
    got = run_prefill(qkv, q, "bf16", kc, vc, L, scale, "bf16", causal=causal)
    assert out_err(got, ref, "bf16") <= 1.0, (max_err(got, ref), out_err(got, ref, "bf16"))
    got = run_prefill(qkv, q, "bf16", kc, vc, L, scale, "f16", causal=causal)
    assert max_err(got, ref) <= TOL["f16"], max_err(got, ref)
    got = run_prefill(qkv, q, "bf16", kc, vc, L, scale, "f32", causal=causal)
    assert max_err(got, ref) <= TOL["f32"], max_err(got, ref)


def test_prefill_additive_mask_and_fp16(qkv):
    B, Hq, Hkv, Lq, D, L = 1, 16, 2, 16, 128, 400
    q, kc, vc = make_problem(B, Hq, Hkv, Lq, D, L, "affine", 8, 32, "normal", seed=8)
    rng = np.random.default_rng(2)
    m = rng.standard_normal((B, Hq, Lq, L)).astype(np.float32)
    m[0, 3, 5, :] = -np.inf                       # a fully masked row
    m[0, 7, :, 100:300] = -np.inf
    st = (Hq * Lq * L, Lq * L, L)
    ref = oracle.attention(q, "f16", kc, vc, L, 0.05, mask=oracle.Mask("additive", m, "f32", st))
    got = run_prefill(qkv, q, "f16", kc, vc, L, 0.05, "f16", mask=torch.from_numpy(m).cuda())
    assert np.all(got[0, 3, 5] == 0)
    assert max_err(got, ref) <= TOL["f16"]


def test_prefill_lq_greater_than_l_causal(qkv):
    """Queries before the first key see nothing and return zeros."""
    B, Hq, Hkv, Lq, D, L = 1, 8, 1, 40, 64, 24
    q, kc, vc = make_problem(B, Hq, Hkv, Lq, D, L, "q8_0", 8, 32, "normal", seed=9)
    ref = oracle.attention(q, "f16", kc, vc, L, 0.125, mask=oracle.Mask("causal"))
    got = run_prefill(qkv, q, "f16", kc, vc, L, 0.125, "f16", causal=True)
    assert np.all(got[:, :, :Lq - L] == 0)
    assert max_err(got, ref) <= TOL["f16"]


def test_prefill_q8_0_512_at_20k_full_kv_head(qkv):
    """The 512-query Q8_0 prompt at depth 20480 (Lk = 20992, causal over the
    last 512), full size, launched as the benchmark launches it: every output
    row of KV head 0 (its 16 query heads x 512 queries, the 64 CTAs of that
    head) against the oracle's matrix-product form, plus a sample of rows of
    the other head against the per-row loops."""
    w = S.WORKLOADS["prefill_q8_0_512_at_20k"]
    inp = S.make_inputs(w)
    kc = oracle.quantize(inp.k, w.kv_dtype, "q8_0")
    vc = oracle.quantize(inp.v, w.kv_dtype, "q8_0")
    got = run_prefill(qkv, inp.q, w.q_dtype, kc, vc, w.L, w.scale, w.out_dtype, causal=True)
    G = w.Hq // w.Hkv
    ref = oracle.attention_dense(inp.q, w.q_dtype, kc, vc, w.L, w.scale, causal=True,
                                 heads=range(G))
    assert out_err(got[:, :G], ref[:, :G], "bf16") <= 1.0, max_err(got[:, :G], ref[:, :G])
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([rng.integers(G * w.Lq, w.Hq * w.Lq, 48),
                                     [G * w.Lq, w.Hq * w.Lq - 1]]))
    ref = oracle.attention(inp.q, w.q_dtype, kc, vc, w.L, w.scale, mask=oracle.Mask("causal"),
                           rows=rows)
    g = got.reshape(-1, w.D)[rows]
    r = ref.reshape(-1, w.D)[rows]
    assert out_err(g, r, "bf16") <= 1.0, max_err(g, r)


@pytest.mark.parametrize("scale", [-0.09, 0.0])
def test_prefill_negative_and_zero_scale(qkv, scale):
    """A negative softmax scale flips which keys dominate; the tcgen05 kernel's
    shortcut of scaling the tile maximum of the raw products holds only for a
    non-negative scale, so such tiles take the per-element path.  Zero scale
    gives the mean of the visible values."""
    B, Hq, Hkv, Lq, D, L = 1, 8, 2, 64, 128, 500
    q, kc, vc = make_problem(B, Hq, Hkv, Lq, D, L, "affine", 4, 64, "normal", q_dtype="bf16",
                             Lcap=512, seed=6)
    for causal in (False, True):
        mask = oracle.Mask("causal") if causal else None
        ref = oracle.attention(q, "bf16", kc, vc, L, scale, mask=mask)
        got = run_prefill(qkv, q, "bf16", kc, vc, L, scale, "f16", causal=causal)
        assert max_err(got, ref) <= TOL["f16"], max_err(got, ref)


@pytest.mark.parametrize("mdt,L", [("f16", 333), ("bf16", 333), ("f16", 512), ("bf16", 520),
                                   ("f32", 301)])
def test_prefill_additive_mask_half_dtypes_and_alignment(qkv, mdt, L):
    """Additive masks in every dtype, on rows that are 16-byte aligned (read
    16 bytes at a time) and rows that are not (odd L: element reads), with a
    -inf band and a ragged last tile; tcgen05 kernel (64 rows per kv head)."""
    B, Hq, Hkv, Lq, D = 1, 8, 2, 16, 128
    q, kc, vc = make_problem(B, Hq, Hkv, Lq, D, L, "q8_0", 8, 32, "normal", q_dtype="bf16",
                             Lcap=(L // 8 + 2) * 8, seed=10)
    rng = np.random.default_rng(4)
    m32 = rng.standard_normal((Hq, Lq, L)).astype(np.float32)
    m32[2, :, 50:130] = -np.inf
    m32[5, 3, :] = -np.inf
    if mdt == "f32":
        mb, mt = m32, torch.from_numpy(m32).cuda()
    else:
        mb = S.f32_to_half_bits(m32, mdt)
        mt = to_dev(mb, mdt)
    st = (0, Lq * L, L)
    ref = oracle.attention(q, "bf16", kc, vc, L, 0.06, mask=oracle.Mask("additive", mb, mdt, st))
    got = run_prefill(qkv, q, "bf16", kc, vc, L, 0.06, "f16", mask=(mt, st))
    assert np.all(got[0, 5, 3] == 0)
    assert max_err(got, ref) <= TOL["f16"], max_err(got, ref)


@pytest.mark.parametrize("mdt", ["f32", "bf16"])
@pytest.mark.parametrize("negative", [False, True])
def test_prefill_mask_instance_one_pass_and_fallback(qkv, mdt, negative):
    """Additive masks without softcap or sinks run on the mask instance of the
    tcgen05 kernel: a tile whose keys are all visible to every row of a warp,
    with positive slopes, is scaled and masked in one pass (a -inf entry stays
    -inf through slope * mask); a negative slope in the warp, the ragged last
    tile and a causal-style -inf band meet the per-key path.  Many tiles (L =
    1000), a broadcast mask with per-head slopes, a query row hidden
    entirely (zeros) and scattered -inf keys."""
    B, Hq, Hkv, Lq, D, L = 1, 16, 2, 16, 128, 1000
    q, kc, vc = make_problem(B, Hq, Hkv, Lq, D, L, "affine", 4, 64, "normal", q_dtype="bf16",
                             Lcap=1008, seed=21)
    rng = np.random.default_rng(7)
    m32 = (4.0 * rng.standard_normal((Lq, L))).astype(np.float32)
    m32[:, 300:340] = -np.inf
    m32[3, :] = -np.inf
    m32[5, ::7] = -np.inf
    m32[9, 640:] = -np.inf
    if mdt == "f32":
        mb, mt = m32, torch.from_numpy(m32).cuda()
    else:
        mb = S.f32_to_half_bits(m32, mdt)
        mt = to_dev(mb, mdt)
    slopes = np.linspace(0.25, 1.5, Hq).astype(np.float32)
    if negative:
        slopes[1::5] *= -1.0
    st = (0, 0, L)
    scale = 1.0 / np.sqrt(D)
    ref = oracle.attention(q, "bf16", kc, vc, L, scale, mask=oracle.Mask("additive", mb, mdt, st),
                           ext=oracle.Ext(slopes=slopes.astype(np.float64)))
    out = qkv.qsdpa_prefill(to_dev(q, "bf16"), cache_to_dev(kc), cache_to_dev(vc), L, scale,
                            mask=(mt, st), mask_slopes=torch.from_numpy(slopes).cuda(),
                            out_dtype=torch.float16)
    torch.cuda.synchronize()
    got = from_dev(out)
    assert np.all(got[:, :, 3] == 0)
    assert max_err(got, ref) <= TOL["f16"], max_err(got, ref)
