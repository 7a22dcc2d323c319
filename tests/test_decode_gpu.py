"""GPU parity of qsdpa_decode against the CPU oracle (fp64), element by
element, through the C ABI (ctypes binding).  Tolerances: max-abs 2e-3 for
fp16/bf16 output, 1e-4 for fp32 output."""
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


def run_decode(qkv, q, q_dtype, kc, vc, L, scale, out_dtype="f16", mask=None, ws=None):
    qd = to_dev(q, q_dtype)
    out = qkv.qsdpa_decode(qd, cache_to_dev(kc), cache_to_dev(vc), L, scale, mask=mask,
                           out_dtype=TORCH_DT[out_dtype], workspace=ws)
    torch.cuda.synchronize()
    return from_dev(out)


SHAPES = [
    # B, Hq, Hkv, D, L, fmt, bits, gs
    (1, 4, 1, 64, 256, "affine", 4, 64),     # the tiny workload shape
    (1, 8, 8, 64, 100, "affine", 4, 32),
    (2, 8, 2, 64, 333, "affine", 8, 32),
    (1, 8, 1, 64, 1000, "affine", 8, 64),
    (1, 32, 8, 128, 4099, "affine", 4, 64),
    (2, 16, 4, 128, 777, "affine", 4, 32),
    (1, 12, 1, 128, 2049, "affine", 4, 128),
    (1, 8, 2, 128, 515, "affine", 8, 32),
    (1, 4, 1, 128, 1500, "affine", 8, 64),
    (3, 6, 3, 128, 97, "affine", 8, 128),
    (1, 32, 2, 256, 1037, "q8_0", 8, 32),
    (1, 16, 1, 256, 640, "affine", 4, 32),
    (1, 8, 2, 256, 300, "affine", 4, 64),
    (1, 2, 1, 256, 999, "affine", 4, 128),
    (1, 4, 4, 256, 129, "affine", 8, 32),
    (1, 24, 1, 256, 555, "affine", 8, 64),
    (1, 8, 1, 256, 2000, "affine", 8, 128),
    (1, 4, 2, 64, 77, "q8_0", 8, 32),
    (2, 40, 1, 128, 1024, "q8_0", 8, 32),     # 40 heads: two chunk-groups
    (1, 64, 1, 64, 450, "affine", 4, 64),     # 64 heads per kv head
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "-".join(map(str, s)))
def test_decode_matches_oracle(qkv, shape):
    B, Hq, Hkv, D, L, fmt, bits, gs = shape
    dist = "normal" if fmt == "q8_0" else "uniform"
    q, kc, vc = make_problem(B, Hq, Hkv, 1, D, L, fmt, bits, gs, dist, Lcap=(L // 8 + 5) * 8)
    scale = 1.0 / 16 if fmt == "q8_0" else 1.0 / np.sqrt(D)
    ref = oracle.attention(q, "f16", kc, vc, L, scale)
    got = run_decode(qkv, q, "f16", kc, vc, L, scale, "f16")
    assert max_err(got, ref) <= TOL["f16"], max_err(got, ref)


@pytest.mark.parametrize("out_dtype", ["f16", "bf16", "f32"])
@pytest.mark.parametrize("q_dtype", ["f16", "bf16"])
@pytest.mark.parametrize("fmt,bits,gs", [("affine", 4, 64), ("affine", 8, 32), ("q8_0", 8, 32)])
def test_decode_dtypes(qkv, out_dtype, q_dtype, fmt, bits, gs):
    B, Hq, Hkv, D, L = 1, 16, 2, 128, 1111
    q, kc, vc = make_problem(B, Hq, Hkv, 1, D, L, fmt, bits, gs, "normal", q_dtype=q_dtype,
                             kv_dtype=q_dtype, seed=11)
    ref = oracle.attention(q, q_dtype, kc, vc, L, 0.1)
    got = run_decode(qkv, q, q_dtype, kc, vc, L, 0.1, out_dtype)
    assert out_err(got, ref, out_dtype) <= 1.0, max_err(got, ref)


def test_tiny_workload_exact_config(qkv):
    w = S.WORKLOADS["tiny_decode"]
    inp = S.make_inputs(w)
    kc = oracle.quantize(inp.k, "f16", w.fmt, w.gs, w.bits)
    vc = oracle.quantize(inp.v, "f16", w.fmt, w.gs, w.bits)
    ref = oracle.attention(inp.q, "f16", kc, vc, w.L, w.scale)
    got = run_decode(qkv, inp.q, "f16", kc, vc, w.L, w.scale, "f16")
    assert max_err(got, ref) <= TOL["f16"]
    got32 = run_decode(qkv, inp.q, "f16", kc, vc, w.L, w.scale, "f32")
    assert max_err(got32, ref) <= TOL["f32"]


@pytest.mark.parametrize("L", [0, 1, 2, 15, 16, 17, 127, 128, 129])
def test_decode_short_and_ragged(qkv, L):
    q, kc, vc = make_problem(1, 8, 2, 1, 128, L, "affine", 4, 64, Lcap=136)
    got = run_decode(qkv, q, "f16", kc, vc, L, 0.125, "f32")
    if L == 0:
        assert np.all(got == 0)
        return
    ref = oracle.attention(q, "f16", kc, vc, L, 0.125)
    assert max_err(got, ref) <= TOL["f32"]


def test_decode_additive_mask(qkv):
    B, Hq, Hkv, D, L = 2, 8, 2, 128, 700
    q, kc, vc = make_problem(B, Hq, Hkv, 1, D, L, "affine", 8, 64, "normal")
    rng = np.random.default_rng(1)
    m = rng.standard_normal((B, Hq, 1, L)).astype(np.float32)
    m[0, 3, 0, 100:600] = -np.inf
    m[1, 5, 0, :] = -np.inf                                  # fully masked row
    ref = oracle.attention(q, "f16", kc, vc, L, 0.1,
                           mask=oracle.Mask("additive", m, "f32", (Hq * L, L, L)))
    md = torch.from_numpy(m).cuda()
    got = run_decode(qkv, q, "f16", kc, vc, L, 0.1, "f32", mask=md)
    assert np.all(got[1, 5] == 0)
    assert max_err(got, ref) <= TOL["f32"]
    # broadcast fp16 mask row (strides 0, 0, 0)
    mh = S.f32_to_half_bits(rng.standard_normal(L).astype(np.float32), "f16")
    ref = oracle.attention(q, "f16", kc, vc, L, 0.1, mask=oracle.Mask("additive", mh, "f16"))
    got = run_decode(qkv, q, "f16", kc, vc, L, 0.1, "f16", mask=(to_dev(mh, "f16"), (0, 0, 0)))
    assert max_err(got, ref) <= TOL["f16"]


def test_workspace_reuse_and_canaries(qkv):
    B, Hq, Hkv, D, L = 1, 32, 8, 128, 5000
    q, kc, vc = make_problem(B, Hq, Hkv, 1, D, L, "affine", 4, 64)
    ref = oracle.attention(q, "f16", kc, vc, L, 1.0)
    qd = to_dev(q, "f16")
    kd, vd = cache_to_dev(kc), cache_to_dev(vc)
    ws = qkv.make_workspace(B, Hq, Hkv, 1, D, L)
    nz = qkv.qsdpa_workspace_zero_bytes(B, Hq, Hkv, 1, D, L)
    n = B * Hq * D
    buf = torch.full((n + 64,), 7.0, dtype=torch.float16, device="cuda")
    out = buf[32:32 + n].view(B, Hq, 1, D)
    for _ in range(3):
        qkv.qsdpa_decode(qd, kd, vd, L, 1.0, out=out, workspace=ws)
        torch.cuda.synchronize()
        assert max_err(from_dev(out), ref) <= TOL["f16"]
        assert torch.all(ws[:nz] == 0), "the zeroed header must stay zero after a decode"
    assert torch.all(buf[:32] == 7.0) and torch.all(buf[32 + n:] == 7.0)


def test_decode_rejects_bad_arguments(qkv):
    q, kc, vc = make_problem(1, 8, 2, 1, 128, 64, "affine", 4, 64)
    qd = to_dev(q, "f16")
    kd, vd = cache_to_dev(kc), cache_to_dev(vc)
    with pytest.raises(qkv.QKVError, match="workspace"):
        qkv.qsdpa_decode(qd, kd, vd, 64, 1.0, workspace=torch.zeros(16, dtype=torch.uint8,
                                                                    device="cuda"))
    with pytest.raises(qkv.QKVError, match="L="):
        qkv.qsdpa_decode(qd, kd, vd, 10 ** 6, 1.0)
    bad = qkv.QuantCache(kd.fmt, 7, kd.group_size, kd.codes, kd.scales, kd.biases)
    with pytest.raises(qkv.QKVError, match="bits"):
        qkv.qsdpa_decode(qd, bad, vd, 64, 1.0)


# ---------------------------------------------------------------------------
# the benchmark workloads at full size
# ---------------------------------------------------------------------------
def _full(name):
    w = S.WORKLOADS[name]
    inp = S.make_inputs(w)
    return w, inp


def test_decode_64k_affine4_full(qkv):
    w, inp = _full("decode_64k_affine4")
    kc = oracle.quantize(inp.k, "f16", w.fmt, w.gs, w.bits)
    vc = oracle.quantize(inp.v, "f16", w.fmt, w.gs, w.bits)
    ref = oracle.attention(inp.q, "f16", kc, vc, w.L, w.scale)
    got = run_decode(qkv, inp.q, "f16", kc, vc, w.L, w.scale, "f16")
    assert max_err(got, ref) <= TOL["f16"], max_err(got, ref)
    got32 = run_decode(qkv, inp.q, "f16", kc, vc, w.L, w.scale, "f32")
    assert max_err(got32, ref) <= TOL["f32"], max_err(got32, ref)


def test_decode_64k_affine8_with_update_full(qkv):
    """Quantize and append one token per head at offset 65535 of a 65536-row
    cache on the GPU, check the written rows bit for bit, then decode."""
    from helpers import cache_from_dev
    w, inp = _full("decode_64k_affine8_update")
    Lold = w.L - w.update_tokens
    kfull = np.zeros((w.B, w.Hkv, w.Lcap, w.D), np.uint16)
    vfull = np.zeros_like(kfull)
    kfull[:, :, :Lold] = inp.k
    vfull[:, :, :Lold] = inp.v
    kc = oracle.quantize(kfull, "f16", w.fmt, w.gs, w.bits)
    vc = oracle.quantize(vfull, "f16", w.fmt, w.gs, w.bits)
    kd, vd = cache_to_dev(kc), cache_to_dev(vc)
    qkv.qkv_quantize_update(to_dev(inp.new_k, "f16"), to_dev(inp.new_v, "f16"), kd, vd, Lold)
    torch.cuda.synchronize()
    # expected cache after the update: the oracle quantizes the new rows
    kfull[:, :, Lold:] = inp.new_k
    vfull[:, :, Lold:] = inp.new_v
    kc2 = oracle.quantize(kfull, "f16", w.fmt, w.gs, w.bits)
    vc2 = oracle.quantize(vfull, "f16", w.fmt, w.gs, w.bits)
    kg, vg = cache_from_dev(kd, w.fmt), cache_from_dev(vd, w.fmt)
    for a, b in ((kg, kc2), (vg, vc2)):
        assert np.array_equal(a.codes, b.codes)
        assert np.array_equal(a.scales, b.scales)
        assert np.array_equal(a.biases, b.biases)
    ref = oracle.attention(inp.q, "f16", kc2, vc2, w.L, w.scale)
    out = qkv.qsdpa_decode(to_dev(inp.q, "f16"), kd, vd, w.L, w.scale)
    torch.cuda.synchronize()
    assert max_err(from_dev(out), ref) <= TOL["f16"]


@pytest.mark.parametrize("name", ["decode_q8_0_10k", "decode_q8_0_20k"])
def test_decode_q8_0_full(qkv, name):
    w, inp = _full(name)
    kc = oracle.quantize(inp.k, "f16", "q8_0")
    vc = oracle.quantize(inp.v, "f16", "q8_0")
    ref = oracle.attention(inp.q, "f16", kc, vc, w.L, w.scale)
    got = run_decode(qkv, inp.q, "f16", kc, vc, w.L, w.scale, "f16")
    assert max_err(got, ref) <= TOL["f16"], max_err(got, ref)
    got32 = run_decode(qkv, inp.q, "f16", kc, vc, w.L, w.scale, "f32")
    assert max_err(got32, ref) <= TOL["f32"], max_err(got32, ref)


def test_decode_negative_scale():
    from quantized_kv_attention_split_b200 import qkv
    q, kc, vc = make_problem(1, 32, 8, 1, 128, 3000, "affine", 4, 64, "normal", seed=7)
    ref = oracle.attention(q, "f16", kc, vc, 3000, -0.2)
    out = qkv.qsdpa_decode(to_dev(q, "f16"), cache_to_dev(kc), cache_to_dev(vc), 3000, -0.2)
    torch.cuda.synchronize()
    assert out_err(from_dev(out), ref, "f16") <= 1.0
