"""CPU oracle for quantized-KV attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never calls it, and a
missing CUDA extension is an error there, never a reason to come here.

Thin ``ctypes`` wrapper around ``liboracle.so`` (built from ``qkv_oracle.cpp``
by ``oracle/build.py``).  All arrays are numpy; half-precision tensors are
passed as their raw ``uint16`` bit patterns together with a dtype name.

What each function follows is stated in ``qkv_oracle.cpp``: the MLX
quantized-KV branch ("add fast::quantized_kv_update": fast.cpp fallback math,
sdpa_vector.h packing and dequant, quantized.h eps), the MLX CUDA WIP page
(load_quantized dequant) and llama.cpp PR #25556 (the Q8_0 KV format).

Parity unpinned: agreement with MLX's or llama.cpp's own quantizer outputs
(the pages print no quantizer body and no worked example); the quantizers
(and the llama.cpp block quantizers below, a reading of the published
reference ones) are pinned only by what their definitions fix.
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass
from typing import Optional, Sequence

import numpy as np

from . import build as _build

_DT = {"f16": 0, "bf16": 1, "f32": 2}
_FMT = {"affine": 0, "q8_0": 1}

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        p = C.c_void_p
        i64 = C.c_int64
        i32 = C.c_int
        for name in ("orc_f32_to_f16", "orc_f16_to_f32", "orc_f32_to_bf16", "orc_bf16_to_f32"):
            getattr(L, name).argtypes = [p, p, i64]
            getattr(L, name).restype = None
        L.orc_quantize.argtypes = [i32, p, i32, i64, i32, i32, i32, p, p, p, i32]
        L.orc_quantize.restype = i32
        L.orc_dequantize.argtypes = [i32, i32, i32, p, p, p, i64, i32, p]
        L.orc_dequantize.restype = i32
        common = [p, i32, i32, i32, i32, i32,
                  i32, i32, i32, p, p, p,
                  i32, i32, i32, p, p, p,
                  i64, i64, C.c_double, i32, p, i32, i64, i64, i64,
                  C.c_double, p, p]
        L.orc_attention.argtypes = common + [i32, i32, p, i64, p, i32]
        L.orc_attention.restype = i32
        L.orc_attention_probs.argtypes = common + [i32, i32, i32, p, p]
        L.orc_attention_probs.restype = i32
        L.orc_attention_kview.argtypes = [p, i32, i32, i32, i32, i32, i32,
                                          i32, i32, i32, p, p, p,
                                          i64, i64, C.c_double, i32, p, i32, i64, i64, i64,
                                          C.c_double, p, p, i32, i32, p, i64, p, i32]
        L.orc_attention_kview.restype = i32
        _lib = L
    return _lib


def _ptr(a: Optional[np.ndarray]):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(C.c_void_p)


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


# ----------------------------------------------------------------------------
# half-precision conversions (IEEE-754, round-to-nearest-even)
# ----------------------------------------------------------------------------
def f32_to_f16(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    y = np.empty(x.shape, np.uint16)
    lib().orc_f32_to_f16(_ptr(x), _ptr(y), x.size)
    return y


def f16_to_f32(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.uint16)
    y = np.empty(x.shape, np.float32)
    lib().orc_f16_to_f32(_ptr(x), _ptr(y), x.size)
    return y


def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    y = np.empty(x.shape, np.uint16)
    lib().orc_f32_to_bf16(_ptr(x), _ptr(y), x.size)
    return y


def bf16_to_f32(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.uint16)
    y = np.empty(x.shape, np.float32)
    lib().orc_bf16_to_f32(_ptr(x), _ptr(y), x.size)
    return y


def to_f64(x: np.ndarray, dtype: str) -> np.ndarray:
    """Raw half bits (or float32) -> float64, exactly."""
    if dtype == "f16":
        return f16_to_f32(x).astype(np.float64)
    if dtype == "bf16":
        return bf16_to_f32(x).astype(np.float64)
    return np.asarray(x, dtype=np.float32).astype(np.float64)


# ----------------------------------------------------------------------------
# quantized cache
# ----------------------------------------------------------------------------
@dataclass
class QCache:
    """One of K or V: codes [B,Hkv,Lcap,D*bits/32] uint32, scales (and for the
    affine format biases) [B,Hkv,Lcap,D/gs] as fp16 bit patterns."""
    fmt: str
    bits: int
    gs: int
    codes: np.ndarray
    scales: np.ndarray
    biases: Optional[np.ndarray]

    @property
    def Lcap(self) -> int:
        return self.codes.shape[-2]


def quantize(x: np.ndarray, dtype: str, fmt: str = "affine", gs: int = 64,
             bits: int = 4, nthreads: Optional[int] = None) -> QCache:
    """Quantize x [..., D] (raw half bits, or float32 for dtype 'f32')."""
    if fmt == "q8_0":
        gs, bits = 32, 8
    x = np.ascontiguousarray(x)
    D = x.shape[-1]
    rows = x.size // D
    codes = np.zeros(x.shape[:-1] + (D * bits // 32,), np.uint32)
    scales = np.zeros(x.shape[:-1] + (D // gs,), np.uint16)
    biases = np.zeros_like(scales)
    rc = lib().orc_quantize(_FMT[fmt], _ptr(x), _DT[dtype], rows, D, gs, bits,
                            _ptr(codes), _ptr(scales), _ptr(biases),
                            nthreads or default_threads())
    if rc:
        raise ValueError("oracle quantize: unsupported shape/bits")
    return QCache(fmt, bits, gs, codes, scales, biases if fmt == "affine" else None)


def dequantize(c: QCache, D: int) -> np.ndarray:
    rows = c.codes.size // c.codes.shape[-1]
    out = np.empty(c.codes.shape[:-1] + (D,), np.float64)
    lib().orc_dequantize(_FMT[c.fmt], c.bits, c.gs, _ptr(c.codes), _ptr(c.scales),
                         _ptr(c.biases), rows, D, _ptr(out))
    return out


@dataclass
class Mask:
    kind: str = "none"                 # none | causal | additive
    add: Optional[np.ndarray] = None   # raw bits (f16/bf16) or float32
    dtype: str = "f32"
    strides: Sequence[int] = (0, 0, 0)  # element strides over (b, h, query)


@dataclass
class Ext:
    """Attention extensions (see qkv_oracle.cpp): logit softcap (0 = off),
    per-head sink logits [Hq] and per-head additive-mask slopes [Hq] (ALiBi)."""
    softcap: float = 0.0
    sinks: Optional[np.ndarray] = None
    slopes: Optional[np.ndarray] = None


def _common_args(q64, k: QCache, v: QCache, L, scale, mask: Optional[Mask],
                 ext: Optional[Ext] = None):
    B, Hq, Lq, D = q64.shape
    Hkv = k.codes.shape[1]
    mask = mask or Mask()
    ext = ext or Ext()
    kind = {"none": 0, "causal": 1, "additive": 2}[mask.kind]
    add = None if mask.add is None else np.ascontiguousarray(mask.add)
    sinks = None if ext.sinks is None else np.ascontiguousarray(ext.sinks, dtype=np.float64)
    slopes = None if ext.slopes is None else np.ascontiguousarray(ext.slopes, dtype=np.float64)
    for a in (sinks, slopes):
        if a is not None and a.size != Hq:
            raise ValueError("sinks and slopes hold one value per query head")
    return [
        _ptr(q64), B, Hq, Hkv, Lq, D,
        _FMT[k.fmt], k.bits, k.gs, _ptr(k.codes), _ptr(k.scales), _ptr(k.biases),
        _FMT[v.fmt], v.bits, v.gs, _ptr(v.codes), _ptr(v.scales), _ptr(v.biases),
        k.Lcap, L, float(scale), kind, _ptr(add), _DT[mask.dtype],
        int(mask.strides[0]), int(mask.strides[1]), int(mask.strides[2]),
        float(ext.softcap), _ptr(sinks), _ptr(slopes),
    ], (add, sinks, slopes)


def attention(q: np.ndarray, q_dtype: str, k: QCache, v: QCache, L: int,
              scale: float, mask: Optional[Mask] = None, mode: str = "two_pass",
              nsplit: int = 1, rows: Optional[np.ndarray] = None,
              nthreads: Optional[int] = None, ext: Optional[Ext] = None) -> np.ndarray:
    """fp64 attention output [B,Hq,Lq,D].  ``rows`` (flattened (b,h,i) ids)
    restricts the computation to a subset; other rows are left NaN."""
    q64 = np.ascontiguousarray(to_f64(q, q_dtype))
    B, Hq, Lq, D = q64.shape
    out = np.full((B, Hq, Lq, D), np.nan)
    args, keep = _common_args(q64, k, v, L, scale, mask, ext)
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    rc = lib().orc_attention(*args, {"two_pass": 0, "online": 1, "split": 2}[mode],
                             nsplit, _ptr(r), 0 if r is None else r.size, _ptr(out),
                             nthreads or default_threads())
    if rc:
        raise ValueError("oracle attention: invalid arguments")
    return out


def attention_dense(q: np.ndarray, q_dtype: str, k: QCache, v: QCache, L: int, scale: float,
                    causal: bool = False, heads: Optional[Sequence[int]] = None,
                    row_block: int = 1024) -> np.ndarray:
    """fp64 attention [B,Hq,Lq,D] evaluated as the definition reads, with
    library matrix products as its steps (MLX compare, mlx/fast.cpp fallback of
    quantized_scaled_dot_product_attention: q*scale, S = q K^T, the causal
    limit, a max-subtracted ("precise") softmax, then P V), over the cache
    dequantized once by the C oracle (exact fp64 values).  For checking many
    rows of a large problem in seconds: no additive mask and no extensions.
    ``heads``: the query heads to compute (others are left NaN).  A row that
    sees no key is zero, as in :func:`attention`."""
    q64 = to_f64(q, q_dtype)
    B, Hq, Lq, D = q64.shape
    Hkv = k.codes.shape[1]
    G = Hq // Hkv
    out = np.full((B, Hq, Lq, D), np.nan)
    Kd = dequantize(k, D)[:, :, :L]
    Vd = dequantize(v, D)[:, :, :L]
    sel = range(Hq) if heads is None else heads
    j = np.arange(L)
    for b in range(B):
        for h in sel:
            Kh, Vh = Kd[b, h // G], Vd[b, h // G]               # GQA: kv head h // G
            for i0 in range(0, Lq, row_block):
                i1 = min(Lq, i0 + row_block)
                S = (q64[b, h, i0:i1] * scale) @ Kh.T            # [rows, L]
                if causal:                                       # query i sees j <= L - Lq + i
                    lim = L - Lq + np.arange(i0, i1)
                    S = np.where(j[None, :] <= lim[:, None], S, -np.inf)
                m = S.max(axis=1, keepdims=True)
                vis = np.isfinite(m)
                P = np.exp(S - np.where(vis, m, 0.0))
                den = P.sum(axis=1, keepdims=True)
                O = (P @ Vh) / np.where(vis, den, 1.0)
                out[b, h, i0:i1] = np.where(vis, O, 0.0)
    return out


def attention_kview(q: np.ndarray, q_dtype: str, k: QCache, L: int, scale: float, Dv: int,
                    mask: Optional[Mask] = None, mode: str = "two_pass", nsplit: int = 1,
                    rows: Optional[np.ndarray] = None, nthreads: Optional[int] = None,
                    ext: Optional[Ext] = None) -> np.ndarray:
    """fp64 attention [B,Hq,Lq,Dv] whose values are the first Dv elements of
    the key rows (the MLA shape: K rows of Dk, V a view of K)."""
    q64 = np.ascontiguousarray(to_f64(q, q_dtype))
    B, Hq, Lq, Dk = q64.shape
    out = np.full((B, Hq, Lq, Dv), np.nan)
    args, keep = _common_args(q64, k, k, L, scale, mask, ext)
    # the common list holds both caches; the view entry takes the key cache once
    a = args[:5] + [Dk, Dv] + args[6:12] + args[18:]
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    rc = lib().orc_attention_kview(*a, {"two_pass": 0, "online": 1, "split": 2}[mode], nsplit,
                                   _ptr(r), 0 if r is None else r.size, _ptr(out),
                                   nthreads or default_threads())
    if rc:
        raise ValueError("oracle attention_kview: invalid arguments")
    return out


def attention_probs(q: np.ndarray, q_dtype: str, k: QCache, v: QCache, L: int,
                    scale: float, b: int, h: int, i: int,
                    mask: Optional[Mask] = None, ext: Optional[Ext] = None):
    """Softmax row (length L) and output (length D) of query row (b, h, i)."""
    q64 = np.ascontiguousarray(to_f64(q, q_dtype))
    D = q64.shape[-1]
    probs = np.empty(L, np.float64)
    o = np.empty(D, np.float64)
    args, keep = _common_args(q64, k, v, L, scale, mask, ext)
    rc = lib().orc_attention_probs(*args, b, h, i, _ptr(probs), _ptr(o))
    if rc:
        raise ValueError("oracle attention_probs: invalid arguments")
    return probs, o


# ----------------------------------------------------------------------------
# llama.cpp-style interleaved Q8_0 blocks <-> the library's planes
# ----------------------------------------------------------------------------
# Reading (the pages name the Q8_0 KV format -- llama.cpp PR #25556: one fp16
# scale per 32 int8 codes -- but not its bytes): the GGUF Q8_0 block, 34 bytes,
# the fp16 scale first (little-endian), then the 32 codes in element order as
# two's-complement bytes.  Plain numpy, element by element in its arithmetic.
Q8_0_BLOCK_BYTES = 34


def q8_0_to_blocks(c: QCache, L: int) -> np.ndarray:
    """Rows [0, L) of a Q8_0 cache -> blocks uint8 [B, Hkv, L, D/32, 34]."""
    assert c.fmt == "q8_0"
    B, Hkv, _, W = c.codes.shape
    nb = W * 4 // 32
    words = c.codes[:, :, :L].astype(np.uint64)             # [B,Hkv,L,W]
    scales = c.scales[:, :, :L].astype(np.uint64)           # [B,Hkv,L,nb]
    out = np.zeros((B, Hkv, L, nb, Q8_0_BLOCK_BYTES), np.uint8)
    out[..., 0] = scales & 0xFF
    out[..., 1] = scales >> 8
    for e in range(32):                                     # element e of each block
        for g in range(nb):
            d = 32 * g + e                                  # element index in the row
            out[:, :, :, g, 2 + e] = (words[..., d // 4] >> (8 * (d % 4))) & 0xFF
    return out


def q8_0_from_blocks(blocks: np.ndarray, Lcap: Optional[int] = None) -> QCache:
    """Blocks uint8 [B, Hkv, L, D/32, 34] -> a Q8_0 cache with Lcap rows (rows
    past L zero)."""
    B, Hkv, L, nb, nbytes = blocks.shape
    assert nbytes == Q8_0_BLOCK_BYTES
    Lcap = Lcap or L
    D = 32 * nb
    codes = np.zeros((B, Hkv, Lcap, D // 4), np.uint32)
    scales = np.zeros((B, Hkv, Lcap, nb), np.uint16)
    b = blocks.astype(np.uint32)
    scales[:, :, :L] = b[..., 0] | (b[..., 1] << 8)
    for g in range(nb):
        for e in range(32):
            d = 32 * g + e
            codes[:, :, :L, d // 4] |= b[:, :, :, g, 2 + e] << (8 * (d % 4))
    return QCache("q8_0", 8, 32, codes, scales, None)


# llama.cpp's other block formats (the PR's follow-up extends its conversion to
# Q4_0, Q4_1, Q5_0 and Q5_1; their bytes, not on the pages, are the GGUF
# blocks).  Reading: blocks of 32 elements, little-endian fp16 fields first;
#   Q4_0: d, qs[16]            x = d * (q - 8)
#   Q4_1: d, m, qs[16]         x = d * q + m
#   Q5_0: d, qh[4], qs[16]     x = d * (q - 16)
#   Q5_1: d, m, qh[4], qs[16]  x = d * q + m
# element j < 16 is the low nibble of qs[j], element j + 16 its high nibble;
# Q5's fifth bit of element e is bit e of qh (a little-endian 32-bit word).
# In the library they become affine caches with groups of 32: 4-bit codes for
# Q4 (bias -8d for Q4_0), 8-bit codes for Q5 (bias -16d for Q5_0).
LLAMA_BLOCKS = {  # name: (bytes, has m, has qh, code offset, cache bits)
    "q4_0": (18, False, False, 8, 4),
    "q4_1": (20, True, False, 0, 4),
    "q5_0": (22, False, True, 16, 8),
    "q5_1": (24, True, True, 0, 8),
}


def _llama_fields(kind: str, blocks: np.ndarray):
    nbytes, has_m, has_qh, off, _ = LLAMA_BLOCKS[kind]
    assert blocks.shape[-1] == nbytes
    b = blocks.astype(np.uint32)
    d = b[..., 0] | (b[..., 1] << 8)
    pos = 2
    m = None
    if has_m:
        m = b[..., pos] | (b[..., pos + 1] << 8)
        pos += 2
    qh = None
    if has_qh:
        qh = b[..., pos] | (b[..., pos + 1] << 8) | (b[..., pos + 2] << 16) | (b[..., pos + 3] << 24)
        pos += 4
    q = np.zeros(blocks.shape[:-1] + (32,), np.uint32)
    for j in range(16):
        q[..., j] = b[..., pos + j] & 0xF
        q[..., j + 16] = b[..., pos + j] >> 4
    if has_qh:
        for e in range(32):
            q[..., e] |= ((qh >> e) & 1) << 4
    return d.astype(np.uint16), None if m is None else m.astype(np.uint16), q, off


def llama_block_values(kind: str, blocks: np.ndarray) -> np.ndarray:
    """Exact values (fp64) of blocks uint8 [..., nb, bytes] -> [..., nb * 32]."""
    d, m, q, off = _llama_fields(kind, blocks)
    dv = f16_to_f32(d).astype(np.float64)[..., None]
    x = dv * (q.astype(np.float64) - off)
    if m is not None:
        x = x + f16_to_f32(m).astype(np.float64)[..., None]
    return x.reshape(blocks.shape[:-2] + (-1,))


def llama_blocks_to_cache(kind: str, blocks: np.ndarray, Lcap: Optional[int] = None) -> QCache:
    """Blocks uint8 [B, Hkv, L, nb, bytes] -> the affine cache (groups of 32)
    that holds the same values: scale d, bias m (or -off * d, exact in fp16
    while |off * d| <= 65504; beyond, the fp16 bias rounds to +-inf)."""
    B, Hkv, L, nb, _ = blocks.shape
    bits = LLAMA_BLOCKS[kind][4]
    Lcap = Lcap or L
    D = 32 * nb
    d, m, q, off = _llama_fields(kind, blocks)
    if m is None:
        m = f32_to_f16((-off * f16_to_f32(d).astype(np.float64)).astype(np.float32))
    codes = np.zeros((B, Hkv, Lcap, D * bits // 32), np.uint32)
    per = 32 // bits
    qq = q.reshape(B, Hkv, L, D)
    for e in range(D):
        codes[:, :, :L, e // per] |= qq[..., e] << (bits * (e % per))
    scales = np.zeros((B, Hkv, Lcap, nb), np.uint16)
    biases = np.zeros((B, Hkv, Lcap, nb), np.uint16)
    scales[:, :, :L] = d
    biases[:, :, :L] = m
    return QCache("affine", bits, 32, codes, scales, biases)


def llama_quantize_blocks(kind: str, x: np.ndarray, dtype: str = "f16") -> np.ndarray:
    """x [..., D] (raw half bits, or float32 for "f32") -> llama.cpp blocks
    uint8 [..., D/32, bytes] of the given kind.  Reading (the pages show no
    quantizer for these types): llama.cpp's published reference quantizers,
    in fp32, block by block of 32 --
      Q4_0 / Q5_0: m = the element of largest magnitude (first such), d = m / -8
        (or m / -16), id = 1/d (0 if d == 0), q = min(15 | 31, trunc(x*id + 8.5 | 16.5));
      Q4_1 / Q5_1: lo, hi = min, max, d = (hi - lo) / 15 (or 31), id = 1/d (0 if
        d == 0), q = min(15 | 31, trunc((x - lo)*id + 0.5)), m = lo;
    d (and m) stored as fp16 (round to nearest even), the codes computed with
    the fp32 d."""
    nbytes, has_m, has_qh, off, _ = LLAMA_BLOCKS[kind]
    xf = to_f64(x, dtype).astype(np.float32)
    D = xf.shape[-1]
    xb = xf.reshape(xf.shape[:-1] + (D // 32, 32))
    top = np.float32(2 * off - 1 if not has_m else (15 if kind == "q4_1" else 31))
    if has_m:
        lo = xb.min(-1)
        hi = xb.max(-1)
        d = ((hi - lo) / top).astype(np.float32)
        idv = np.where(d != 0, np.float32(1) / np.where(d != 0, d, np.float32(1)), np.float32(0))
        t = (xb - lo[..., None]) * idv[..., None] + np.float32(0.5)
        q = np.minimum(np.trunc(t), top).astype(np.uint32)
    else:
        amax_i = np.abs(xb).argmax(-1)
        mval = np.take_along_axis(xb, amax_i[..., None], -1)[..., 0]
        d = (mval / np.float32(-off)).astype(np.float32)
        idv = np.where(d != 0, np.float32(1) / np.where(d != 0, d, np.float32(1)), np.float32(0))
        t = xb * idv[..., None] + np.float32(off + 0.5)
        q = np.minimum(np.trunc(t), top).astype(np.uint32)
    out = np.zeros(xb.shape[:-1] + (nbytes,), np.uint8)
    d16 = f32_to_f16(d.astype(np.float32))
    out[..., 0] = d16 & 0xFF
    out[..., 1] = d16 >> 8
    pos = 2
    if has_m:
        m16 = f32_to_f16(lo.astype(np.float32))
        out[..., 2] = m16 & 0xFF
        out[..., 3] = m16 >> 8
        pos = 4
    if has_qh:
        qh = np.zeros(q.shape[:-1], np.uint64)
        for e in range(32):
            qh |= ((q[..., e].astype(np.uint64) >> 4) & 1) << e
        for k in range(4):
            out[..., pos + k] = (qh >> (8 * k)) & 0xFF
        pos += 4
    for j in range(16):
        out[..., pos + j] = (q[..., j] & 0xF) | ((q[..., j + 16] & 0xF) << 4)
    return out
