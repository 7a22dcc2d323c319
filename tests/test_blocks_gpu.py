"""llama.cpp-style interleaved Q8_0 blocks <-> the library's Q8_0 planes through
the C ABI (qkv_q8_0_from_blocks / qkv_q8_0_to_blocks): bit-exact against the
oracle's conversion, in llama.cpp's token-major layout and head-major, at an
offset into the cache, and as the input of a decode call."""
import numpy as np
import pytest
import torch

import oracle
from helpers import cache_from_dev, cache_to_dev, from_dev, make_problem, out_err, to_dev
from quantized_kv_attention_split_b200 import synthetic as S

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shift", [0, 2])
@pytest.mark.parametrize("B,Hkv,D,L", [(1, 2, 256, 777), (2, 3, 64, 40), (1, 8, 128, 1)])
def test_blocks_round_trip_token_major(B, Hkv, D, L, shift):
    """shift 0: 4-byte aligned blocks (moved in pairs, 32-bit words); shift 2:
    2-byte aligned only (moved block by block, 16-bit units)."""
    from quantized_kv_attention_split_b200 import qkv
    x = S.draw(61, "x", (B, Hkv, L, D), "normal", "f16")
    c = oracle.quantize(x, "f16", "q8_0")
    blocks = oracle.q8_0_to_blocks(c, L)                       # [B,Hkv,L,nb,34]
    nb = D // 32
    # llama.cpp keeps K as [token][kv head][blocks]: token-major bytes
    tm = np.ascontiguousarray(blocks.transpose(0, 2, 1, 3, 4)).reshape(B, L, Hkv * nb * 34)
    flat = torch.zeros(tm.size + 16, dtype=torch.uint8, device="cuda")
    dev = flat[shift:shift + tm.size].view(B, L, Hkv * nb * 34)
    dev.copy_(torch.from_numpy(tm).cuda())
    st = (L * Hkv * nb * 34, nb * 34, Hkv * nb * 34)
    off = 5
    Lcap = ((off + L) // 8 + 1) * 8
    dc = qkv.QuantCache.empty(B, Hkv, Lcap, D, qkv.Q8_0)
    qkv.qkv_q8_0_from_blocks(dev, dc, offset=off, L=L, strides=st)
    torch.cuda.synchronize()
    h = cache_from_dev(dc, "q8_0")
    assert np.array_equal(h.codes[:, :, off:off + L], c.codes)
    assert np.array_equal(h.scales[:, :, off:off + L], c.scales)
    assert not h.codes[:, :, :off].any() and not h.codes[:, :, off + L:].any()
    flat2 = torch.zeros(tm.size + 16, dtype=torch.uint8, device="cuda")
    back = flat2[shift:shift + tm.size].view(B, L, Hkv * nb * 34)
    qkv.qkv_q8_0_to_blocks(dc, L, offset=off, out=back, strides=st)
    torch.cuda.synchronize()
    assert torch.equal(back, dev)
    assert not flat2[:shift].any() and not flat2[shift + tm.size:].any()   # nothing written outside


def test_blocks_head_major_default_layout_and_decode():
    """Blocks in the default [B, Hkv, L, D/32*34] layout become a cache that the
    decode kernel reads like any other."""
    from quantized_kv_attention_split_b200 import qkv
    B, Hq, Hkv, D, L = 1, 32, 2, 256, 3000
    q, kc, vc = make_problem(B, Hq, Hkv, 1, D, L, "q8_0", 8, 32, "normal", seed=62)
    bk = torch.from_numpy(oracle.q8_0_to_blocks(kc, L).reshape(B, Hkv, L, -1)).cuda()
    bv = torch.from_numpy(oracle.q8_0_to_blocks(vc, L).reshape(B, Hkv, L, -1)).cuda()
    dk = qkv.QuantCache.empty(B, Hkv, kc.Lcap, D, qkv.Q8_0)
    dv = qkv.QuantCache.empty(B, Hkv, kc.Lcap, D, qkv.Q8_0)
    qkv.qkv_q8_0_from_blocks(bk, dk)
    qkv.qkv_q8_0_from_blocks(bv, dv)
    out = qkv.qsdpa_decode(to_dev(q, "f16"), dk, dv, L, 1.0 / 16)
    torch.cuda.synchronize()
    ref = oracle.attention(q, "f16", kc, vc, L, 1.0 / 16)
    assert out_err(from_dev(out), ref, "f16") <= 1.0
    assert torch.equal(qkv.qkv_q8_0_to_blocks(dk, L), bk)


def _random_llama_blocks(kind, B, Hkv, L, nb, seed):
    nbytes, has_m = oracle.LLAMA_BLOCKS[kind][0], oracle.LLAMA_BLOCKS[kind][1]
    rng = np.random.default_rng(seed)
    raw = rng.integers(0, 256, (B, Hkv, L, nb, nbytes), dtype=np.uint8)
    for lo in ((0, 2) if has_m else (0,)):
        h = S.f32_to_half_bits(rng.normal(0, 0.05, (B, Hkv, L, nb)).astype(np.float32), "f16")
        raw[..., lo] = h & 0xFF
        raw[..., lo + 1] = h >> 8
    return raw


@pytest.mark.parametrize("kind", ["q4_0", "q4_1", "q5_0", "q5_1"])
def test_llama_blocks_to_cache_matches_oracle_and_decodes(kind):
    """Random llama.cpp blocks (token-major, at a row offset) become exactly the
    oracle's affine cache; the decode kernel then matches the oracle on it."""
    from quantized_kv_attention_split_b200 import qkv
    B, Hq, Hkv, D, L, off = 1, 16, 2, 128, 1500, 3
    nb = D // 32
    nbytes, bits = oracle.LLAMA_BLOCKS[kind][0], oracle.LLAMA_BLOCKS[kind][4]
    Lcap = ((off + L) // 8 + 1) * 8
    caches = []
    for which in (0, 1):
        raw = _random_llama_blocks(kind, B, Hkv, L, nb, 70 + which)
        tm = np.ascontiguousarray(raw.transpose(0, 2, 1, 3, 4)).reshape(B, L, Hkv * nb * nbytes)
        st = (L * Hkv * nb * nbytes, nb * nbytes, Hkv * nb * nbytes)
        dc = qkv.QuantCache.empty(B, Hkv, Lcap, D, qkv.AFFINE, bits, 32)
        qkv.qkv_llama_blocks_to_cache(kind, torch.from_numpy(tm).cuda(), dc, offset=off, L=L,
                                      strides=st)
        torch.cuda.synchronize()
        ref = oracle.llama_blocks_to_cache(kind, raw)
        h = cache_from_dev(dc, "affine")
        assert np.array_equal(h.codes[:, :, off:off + L], ref.codes)
        assert np.array_equal(h.scales[:, :, off:off + L], ref.scales)
        assert np.array_equal(h.biases[:, :, off:off + L], ref.biases)
        caches.append((dc, h))
    (dk, hk), (dv, hv) = caches
    q = S.draw(71, "q", (B, Hq, 1, D), "normal", "f16")
    L_all = off + L
    out = qkv.qsdpa_decode(to_dev(q, "f16"), dk, dv, L_all, 0.125)
    torch.cuda.synchronize()
    ref = oracle.attention(q, "f16", hk, hv, L_all, 0.125)
    assert out_err(from_dev(out), ref, "f16") <= 1.0


# ---------------------------------------------------------------------------
# Q4_0 / Q4_1 / Q5_0 / Q5_1 written on the GPU
# ---------------------------------------------------------------------------
def _block_inputs(B, Hkv, L, D, dtype, seed):
    """Normal and uniform draws, plus blocks of special structure: all zeros,
    a constant block, a block whose largest magnitude appears twice with both
    signs (the first one sets d), and values on the half-way points of the
    codes of a previous quantization."""
    x = S.draw(seed, "x", (B, Hkv, L, D), "normal", dtype)
    u = S.draw(seed, "u", (B, Hkv, L, D), "uniform", dtype)
    x[:, :, 1::3] = u[:, :, 1::3]
    f = (oracle.f16_to_f32 if dtype == "f16" else oracle.bf16_to_f32)(x)
    f[0, 0, 0, :32] = 0.0
    f[0, 0, 0, 32:64] = 1.5
    if D >= 128:
        f[0, 0, 0, 64:96] = np.linspace(-1, 1, 32, dtype=np.float32)
        f[0, 0, 0, 70], f[0, 0, 0, 90] = -2.0, 2.0
    if L > 1:
        f[0, 0, 1, :32] = (np.arange(32, dtype=np.float32) - 8.0) * 0.125 + 0.0625
    return S.f32_to_half_bits(f, dtype)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("kind", ["q4_0", "q4_1", "q5_0", "q5_1"])
def test_llama_quantize_blocks_bit_exact(kind, dtype):
    """The GPU reference quantizer writes exactly the oracle's blocks, in
    llama.cpp's token-major layout (K: [token][kv head][blocks])."""
    from quantized_kv_attention_split_b200 import qkv
    B, Hkv, L, D = 2, 3, 57, 128
    nb, nbytes = D // 32, oracle.LLAMA_BLOCKS[kind][0]
    x = _block_inputs(B, Hkv, L, D, dtype, 81)
    want = oracle.llama_quantize_blocks(kind, x, dtype)           # [B,Hkv,L,nb,bytes]
    out = torch.zeros(B, L, Hkv, nb * nbytes, dtype=torch.uint8, device="cuda")
    st = (L * Hkv * nb * nbytes, nb * nbytes, Hkv * nb * nbytes)
    qkv.qkv_llama_quantize_blocks(kind, to_dev(x, dtype), out=out, strides=st)
    torch.cuda.synchronize()
    got = out.cpu().numpy().reshape(B, L, Hkv, nb, nbytes).transpose(0, 2, 1, 3, 4)
    assert np.array_equal(got, want), np.argwhere(got != want)[:5]


@pytest.mark.parametrize("kind", ["q4_0", "q4_1", "q5_0", "q5_1"])
def test_llama_quantize_update_extends_an_imported_cache(kind):
    """A cache imported from llama.cpp blocks is extended in its own format:
    new tokens quantized with the same reference quantizer land in the affine
    cache exactly as the import would write their blocks; the cache then
    exports back to exactly the blocks (old and new), and decodes like the
    oracle over all of it."""
    from quantized_kv_attention_split_b200 import qkv
    B, Hq, Hkv, D, L0, Lnew = 1, 16, 2, 128, 700, 37
    nb, nbytes, bits = D // 32, oracle.LLAMA_BLOCKS[kind][0], oracle.LLAMA_BLOCKS[kind][4]
    Lcap = ((L0 + Lnew) // 8 + 1) * 8
    dev_caches, all_blocks = [], []
    for which in (0, 1):
        old = oracle.llama_quantize_blocks(kind, S.draw(82 + which, "o", (B, Hkv, L0, D), "normal",
                                                        "f16"))
        new_x = _block_inputs(B, Hkv, Lnew, D, "f16", 84 + which)
        new = oracle.llama_quantize_blocks(kind, new_x)
        dc = qkv.QuantCache.empty(B, Hkv, Lcap, D, qkv.AFFINE, bits, 32)
        qkv.qkv_llama_blocks_to_cache(kind, torch.from_numpy(
            np.ascontiguousarray(old.reshape(B, Hkv, L0, nb * nbytes))).cuda(), dc)
        dev_caches.append((dc, to_dev(new_x, "f16")))
        all_blocks.append(np.concatenate([old, new], axis=2))
    (dk, nk), (dv, nv) = dev_caches
    qkv.qkv_llama_quantize_update(kind, nk, nv, dk, dv, L0)
    torch.cuda.synchronize()
    hosts = []
    for dc, blocks in zip((dk, dv), all_blocks):
        ref = oracle.llama_blocks_to_cache(kind, blocks)
        h = cache_from_dev(dc, "affine")
        L_all = L0 + Lnew
        assert np.array_equal(h.codes[:, :, :L_all], ref.codes)
        assert np.array_equal(h.scales[:, :, :L_all], ref.scales)
        assert np.array_equal(h.biases[:, :, :L_all], ref.biases)
        back = qkv.qkv_llama_cache_to_blocks(kind, dc, L_all)
        torch.cuda.synchronize()
        assert np.array_equal(back.cpu().numpy().reshape(blocks.shape), blocks)
        hosts.append(h)
    q = S.draw(86, "q", (B, Hq, 1, D), "normal", "f16")
    out = qkv.qsdpa_decode(to_dev(q, "f16"), dk, dv, L0 + Lnew, 0.125)
    torch.cuda.synchronize()
    ref = oracle.attention(q, "f16", hosts[0], hosts[1], L0 + Lnew, 0.125)
    assert out_err(from_dev(out), ref, "f16") <= 1.0
