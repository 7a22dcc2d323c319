"""Python binding of ``libqkv.so`` (argument marshalling only).

The functions keep the names of the C entry points declared in
``include/qkv.h`` -- :func:`qkv_quantize_update`, :func:`qsdpa_decode`,
:func:`qsdpa_prefill` -- and take torch CUDA tensors (q and out of the
attention calls may also be pinned CPU tensors), passing their pointers,
sizes and the current CUDA stream to the library.  Every step of the
computation runs in the library's kernels; there is no fallback: if the
library is missing or a call fails, a Python exception is raised.
"""
from __future__ import annotations

import contextlib
import ctypes as C
import os
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqkv.so")

F16, BF16, F32 = 0, 1, 2
AFFINE, Q8_0 = 0, 1
MASK_NONE, MASK_CAUSAL, MASK_ADDITIVE = 0, 1, 2

_DTYPE = {torch.float16: F16, torch.bfloat16: BF16, torch.float32: F32}
_STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported", 3: "alignment",
           4: "workspace too small", 5: "CUDA error"}


class _Cache(C.Structure):
    _fields_ = [("fmt", C.c_int), ("bits", C.c_int), ("group_size", C.c_int),
                ("codes", C.c_void_p), ("scales", C.c_void_p), ("biases", C.c_void_p),
                ("Lcap", C.c_int64)]


class _Mask(C.Structure):
    _fields_ = [("kind", C.c_int), ("add", C.c_void_p), ("add_dtype", C.c_int),
                ("stride_b", C.c_int64), ("stride_h", C.c_int64), ("stride_q", C.c_int64)]


class _Ext(C.Structure):
    _fields_ = [("softcap", C.c_float), ("mask_slopes", C.c_void_p), ("sinks", C.c_void_p)]


class QKVError(RuntimeError):
    def __init__(self, status: int, detail: str):
        super().__init__(f"{_STATUS.get(status, status)}: {detail}")
        self.status = status


_lib = None


def lib() -> C.CDLL:
    """Load libqkv.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libqkv.so not found at {LIB_PATH}; build it with "
                              "`python quantized_kv_attention_split_b200/build.py`")
        L = C.CDLL(LIB_PATH)
        p, i32, i64, sz = C.c_void_p, C.c_int, C.c_int64, C.c_size_t
        cp = C.POINTER(_Cache)
        mp = C.POINTER(_Mask)
        L.qkv_quantize_update.argtypes = [p, p, i32, i32, i32, i32, i32, cp, cp, i64, p]
        L.qkv_quantize_update.restype = i32
        L.qsdpa_decode.argtypes = [p, i32, i32, i32, i32, i32, cp, cp, i64, C.c_float, mp,
                                   p, i32, p, sz, p]
        L.qsdpa_decode.restype = i32
        L.qsdpa_prefill.argtypes = [p, i32, i32, i32, i32, i32, i32, cp, cp, i64, C.c_float, mp,
                                    p, i32, p, sz, p]
        L.qsdpa_prefill.restype = i32
        ep = C.POINTER(_Ext)
        L.qsdpa_decode_ext.argtypes = [p, i32, i32, i32, i32, i32, cp, cp, i64, C.c_float, mp,
                                       ep, p, i32, p, sz, p]
        L.qsdpa_decode_ext.restype = i32
        L.qsdpa_prefill_ext.argtypes = [p, i32, i32, i32, i32, i32, i32, cp, cp, i64, C.c_float,
                                        mp, ep, p, i32, p, sz, p]
        L.qsdpa_prefill_ext.restype = i32
        L.qsdpa_decode_update.argtypes = [p, i32, p, p, i32, i32, i32, i32, i32, cp, cp, i64,
                                          C.c_float, mp, p, i32, p, sz, p]
        L.qsdpa_decode_update.restype = i32
        L.qkv_q8_0_from_blocks.argtypes = [p, i32, i32, i32, i64, i64, i64, i64, cp, i64, p]
        L.qkv_q8_0_from_blocks.restype = i32
        L.qkv_q8_0_to_blocks.argtypes = [cp, i32, i32, i32, i64, i64, p, i64, i64, i64, p]
        L.qkv_q8_0_to_blocks.restype = i32
        L.qkv_llama_blocks_to_cache.argtypes = [i32, p, i32, i32, i32, i64, i64, i64, i64, cp,
                                                i64, p]
        L.qkv_llama_blocks_to_cache.restype = i32
        L.qkv_llama_quantize_blocks.argtypes = [i32, p, i32, i32, i32, i32, i64, p, i64, i64, i64,
                                                p]
        L.qkv_llama_quantize_blocks.restype = i32
        L.qkv_llama_quantize_update.argtypes = [i32, p, p, i32, i32, i32, i32, i32, cp, cp, i64, p]
        L.qkv_llama_quantize_update.restype = i32
        L.qkv_llama_cache_to_blocks.argtypes = [i32, cp, i32, i32, i32, i64, i64, p, i64, i64, i64,
                                                p]
        L.qkv_llama_cache_to_blocks.restype = i32
        L.qsdpa_attention_kview.argtypes = [p, i32, i32, i32, i32, i32, i32, i32, cp, i64,
                                            C.c_float, mp, p, i32, p, sz, p]
        L.qsdpa_attention_kview.restype = i32
        L.qsdpa_kview_workspace_size.argtypes = [i32, i32, i32, i32, i32, i32, i64]
        L.qsdpa_kview_workspace_size.restype = sz
        L.qkv_dequantize.argtypes = [cp, i32, i32, i32, i64, p, p]
        L.qkv_dequantize.restype = i32
        L.qsdpa_workspace_size.argtypes = [i32, i32, i32, i32, i32, i64]
        L.qsdpa_workspace_size.restype = sz
        L.qsdpa_workspace_zero_bytes.argtypes = [i32, i32, i32, i32, i32, i64]
        L.qsdpa_workspace_zero_bytes.restype = sz
        L.qkv_status_string.argtypes = [i32]
        L.qkv_status_string.restype = C.c_char_p
        L.qkv_last_error.argtypes = []
        L.qkv_last_error.restype = C.c_char_p
        _lib = L
    return _lib


def _check(status: int):
    if status != 0:
        raise QKVError(status, lib().qkv_last_error().decode())


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _on(t: torch.Tensor):
    """Context in which t's device is the current one: the library launches on
    the current device (and the default stream is the current device's), so a
    call whose tensors live on another device switches to it first."""
    idx = t.device.index
    if idx is None or idx == torch.cuda.current_device():
        return contextlib.nullcontext()
    return torch.cuda.device(idx)


@dataclass
class QuantCache:
    """One of K or V in the library's layout (all tensors on one CUDA device):
    codes int32 [B,Hkv,Lcap,D*bits/32] (bit patterns of uint32 words), scales
    and biases float16 [B,Hkv,Lcap,D/group_size] (biases None for Q8_0)."""
    fmt: int
    bits: int
    group_size: int
    codes: torch.Tensor
    scales: torch.Tensor
    biases: Optional[torch.Tensor]

    @property
    def Lcap(self) -> int:
        return self.codes.shape[2]

    @staticmethod
    def empty(B: int, Hkv: int, Lcap: int, D: int, fmt: int = AFFINE, bits: int = 4,
              group_size: int = 64, device="cuda") -> "QuantCache":
        if fmt == Q8_0:
            bits, group_size = 8, 32
        codes = torch.zeros(B, Hkv, Lcap, D * bits // 32, dtype=torch.int32, device=device)
        scales = torch.zeros(B, Hkv, Lcap, D // group_size, dtype=torch.float16, device=device)
        biases = torch.zeros_like(scales) if fmt == AFFINE else None
        return QuantCache(fmt, bits, group_size, codes, scales, biases)

    def _struct(self) -> _Cache:
        # built once per set of buffers (decode calls are short: the host-side
        # marshalling is part of every call's latency)
        key = (self.fmt, self.bits, self.group_size, self.codes.data_ptr(),
               self.scales.data_ptr(), self.biases.data_ptr() if self.biases is not None else None,
               self.codes.shape[2])
        cached = self.__dict__.get("_cs")
        if cached is None or cached[0] != key:
            cached = (key, _Cache(*key))
            self.__dict__["_cs"] = cached
        return cached[1]


def qsdpa_workspace_size(B: int, Hq: int, Hkv: int, Lq: int, D: int, L: int) -> int:
    return int(lib().qsdpa_workspace_size(B, Hq, Hkv, Lq, D, L))


def qsdpa_workspace_zero_bytes(B: int, Hq: int, Hkv: int, Lq: int, D: int, L: int) -> int:
    return int(lib().qsdpa_workspace_zero_bytes(B, Hq, Hkv, Lq, D, L))


def make_workspace(B: int, Hq: int, Hkv: int, Lq: int, D: int, L: int,
                   device="cuda") -> torch.Tensor:
    """A zero-initialised workspace of the size the library asks for."""
    n = qsdpa_workspace_size(B, Hq, Hkv, Lq, D, L)
    return torch.zeros(max(n, 16), dtype=torch.uint8, device=device)


def qkv_quantize_update(new_k: torch.Tensor, new_v: torch.Tensor, k: QuantCache, v: QuantCache,
                        offset: int, stream=None) -> None:
    """Quantize new_k/new_v [B,Hkv,Lnew,D] (f16/bf16) into rows
    [offset, offset+Lnew) of the caches, in place."""
    assert new_k.is_contiguous() and new_v.is_contiguous()
    assert new_k.shape == new_v.shape and new_k.dtype == new_v.dtype
    B, Hkv, Lnew, D = new_k.shape
    ks, vs = k._struct(), v._struct()
    with _on(new_k):
        _check(lib().qkv_quantize_update(new_k.data_ptr(), new_v.data_ptr(), _DTYPE[new_k.dtype],
                                         B, Hkv, Lnew, D, C.byref(ks), C.byref(vs), int(offset),
                                         _stream(stream)))


def qkv_dequantize(c: QuantCache, L: int, out: Optional[torch.Tensor] = None,
                   stream=None) -> torch.Tensor:
    """Rows [0, L) of a cache as fp16 [B, Hkv, L, D]: the correctly rounded
    scale * code + bias (for "materialize, then dense attention")."""
    B, Hkv = c.codes.shape[0], c.codes.shape[1]
    D = c.codes.shape[3] * 32 // c.bits
    if out is None:
        out = torch.empty(B, Hkv, L, D, dtype=torch.float16, device=c.codes.device)
    assert out.is_contiguous() and out.dtype == torch.float16 and tuple(out.shape) == (B, Hkv, L, D)
    cs = c._struct()
    with _on(out):
        _check(lib().qkv_dequantize(C.byref(cs), B, Hkv, D, int(L), out.data_ptr(),
                                    _stream(stream)))
    return out


Q8_0_BLOCK_BYTES = 34


def _block_strides(blocks: torch.Tensor, strides):
    """Byte strides (b, kv head, token) of a uint8 block tensor [B,Hkv,L,D/32*34]
    (or [B,L,Hkv,D/32*34] when given explicitly as `strides`)."""
    if strides is not None:
        return tuple(int(x) for x in strides)
    s = blocks.stride()
    return s[0], s[1], s[2]


def qkv_q8_0_from_blocks(blocks: torch.Tensor, c: QuantCache, offset: int = 0,
                         L: Optional[int] = None, strides=None, stream=None) -> QuantCache:
    """Write llama.cpp-style Q8_0 blocks (uint8 CUDA tensor, by default
    [B, Hkv, L, D/32*34]; other layouts through `strides` = byte strides of
    (b, kv head, token) and an explicit L) into cache rows [offset, offset+L)."""
    assert blocks.dtype == torch.uint8 and blocks.is_cuda and c.fmt == Q8_0
    B, Hkv, D = c.codes.shape[0], c.codes.shape[1], c.codes.shape[3] * 4
    if L is None:
        L = blocks.shape[2]
    sb, sh, sl = _block_strides(blocks, strides)
    cs = c._struct()
    with _on(blocks):
        _check(lib().qkv_q8_0_from_blocks(blocks.data_ptr(), B, Hkv, D, int(L), sb, sh, sl,
                                          C.byref(cs), int(offset), _stream(stream)))
    return c


LLAMA_BLOCKS = {"q4_0": (0, 18, 4), "q4_1": (1, 20, 4), "q5_0": (2, 22, 8), "q5_1": (3, 24, 8)}


def qkv_llama_blocks_to_cache(kind: str, blocks: torch.Tensor, c: QuantCache, offset: int = 0,
                              L: Optional[int] = None, strides=None, stream=None) -> QuantCache:
    """Write llama.cpp Q4_0/Q4_1/Q5_0/Q5_1 blocks (uint8 CUDA tensor, by default
    [B, Hkv, L, D/32*bytes]) into rows [offset, offset+L) of an affine cache with
    group_size 32 (4-bit codes for Q4, 8-bit for Q5)."""
    code, nbytes, bits = LLAMA_BLOCKS[kind]
    assert blocks.dtype == torch.uint8 and blocks.is_cuda and c.fmt == AFFINE
    B, Hkv = c.codes.shape[0], c.codes.shape[1]
    D = c.codes.shape[3] * 32 // c.bits
    if L is None:
        L = blocks.shape[2]
    sb, sh, sl = _block_strides(blocks, strides)
    cs = c._struct()
    with _on(blocks):
        _check(lib().qkv_llama_blocks_to_cache(code, blocks.data_ptr(), B, Hkv, D, int(L), sb, sh,
                                               sl, C.byref(cs), int(offset), _stream(stream)))
    return c


def qkv_llama_quantize_blocks(kind: str, x: torch.Tensor, out: Optional[torch.Tensor] = None,
                              strides=None, stream=None) -> torch.Tensor:
    """llama.cpp's reference quantizer for Q4_0/Q4_1/Q5_0/Q5_1 on the GPU:
    x [B, Hkv, L, D] (f16/bf16) -> blocks (uint8, [B, Hkv, L, D/32*bytes]
    unless `out` and `strides` say otherwise)."""
    code, nbytes, _ = LLAMA_BLOCKS[kind]
    assert x.is_contiguous() and x.is_cuda
    B, Hkv, L, D = x.shape
    if out is None:
        out = torch.empty(B, Hkv, L, D // 32 * nbytes, dtype=torch.uint8, device=x.device)
    sb, sh, sl = _block_strides(out, strides)
    with _on(x):
        _check(lib().qkv_llama_quantize_blocks(code, x.data_ptr(), _DTYPE[x.dtype], B, Hkv, D,
                                               int(L), out.data_ptr(), sb, sh, sl,
                                               _stream(stream)))
    return out


def qkv_llama_quantize_update(kind: str, new_k: torch.Tensor, new_v: torch.Tensor, k: QuantCache,
                              v: QuantCache, offset: int, stream=None) -> None:
    """Quantize new_k/new_v [B, Hkv, Lnew, D] with llama.cpp's reference
    quantizer of `kind` and write rows [offset, offset+Lnew) of the affine
    caches (group 32; 4-bit for Q4, 8-bit for Q5) holding the blocks' values."""
    code, _, _ = LLAMA_BLOCKS[kind]
    assert new_k.is_contiguous() and new_v.is_contiguous() and new_k.shape == new_v.shape
    B, Hkv, Lnew, D = new_k.shape
    ks, vs = k._struct(), v._struct()
    with _on(new_k):
        _check(lib().qkv_llama_quantize_update(code, new_k.data_ptr(), new_v.data_ptr(),
                                               _DTYPE[new_k.dtype], B, Hkv, Lnew, D, C.byref(ks),
                                               C.byref(vs), int(offset), _stream(stream)))


def qkv_llama_cache_to_blocks(kind: str, c: QuantCache, L: int, offset: int = 0,
                              out: Optional[torch.Tensor] = None, strides=None,
                              stream=None) -> torch.Tensor:
    """Rows [offset, offset+L) of an affine cache (group 32) as llama.cpp blocks
    of `kind` (uint8, [B, Hkv, L, D/32*bytes] unless `out`/`strides` given)."""
    code, nbytes, _ = LLAMA_BLOCKS[kind]
    B, Hkv = c.codes.shape[0], c.codes.shape[1]
    D = c.codes.shape[3] * 32 // c.bits
    if out is None:
        out = torch.empty(B, Hkv, L, D // 32 * nbytes, dtype=torch.uint8, device=c.codes.device)
    sb, sh, sl = _block_strides(out, strides)
    cs = c._struct()
    with _on(out):
        _check(lib().qkv_llama_cache_to_blocks(code, C.byref(cs), B, Hkv, D, int(offset), int(L),
                                               out.data_ptr(), sb, sh, sl, _stream(stream)))
    return out


def qkv_q8_0_to_blocks(c: QuantCache, L: int, offset: int = 0,
                       out: Optional[torch.Tensor] = None, strides=None,
                       stream=None) -> torch.Tensor:
    """Cache rows [offset, offset+L) of a Q8_0 cache as llama.cpp-style blocks
    (uint8, [B, Hkv, L, D/32*34] unless `out` and `strides` say otherwise)."""
    assert c.fmt == Q8_0
    B, Hkv, D = c.codes.shape[0], c.codes.shape[1], c.codes.shape[3] * 4
    if out is None:
        out = torch.empty(B, Hkv, L, D // 32 * Q8_0_BLOCK_BYTES, dtype=torch.uint8,
                          device=c.codes.device)
    sb, sh, sl = _block_strides(out, strides)
    cs = c._struct()
    with _on(out):
        _check(lib().qkv_q8_0_to_blocks(C.byref(cs), B, Hkv, D, int(offset), int(L),
                                        out.data_ptr(), sb, sh, sl, _stream(stream)))
    return out


def _mask_struct(mask, causal: bool):
    if causal:
        return _Mask(MASK_CAUSAL, None, 0, 0, 0, 0)
    if mask is None:
        return None
    t, strides = mask if isinstance(mask, tuple) else (mask, None)
    if strides is None:                    # full [B,Hq,Lq,L] (or broadcastable) tensor
        s = t.stride()
        strides = (s[0], s[1], s[2]) if t.dim() == 4 else (0, 0, 0)
    return _Mask(MASK_ADDITIVE, t.data_ptr(), _DTYPE[t.dtype], *[int(x) for x in strides])


def _ext_struct(softcap, sinks, mask_slopes, Hq, device):
    """qkv_attn_ext for the optional extensions, or None when none is used.
    sinks / mask_slopes: fp32 CUDA tensors of Hq values."""
    if not softcap and sinks is None and mask_slopes is None:
        return None
    for t in (sinks, mask_slopes):
        if t is not None:
            assert t.is_cuda and t.dtype == torch.float32 and t.is_contiguous()
            assert t.numel() == Hq and t.device == device
    return _Ext(float(softcap or 0.0), None if mask_slopes is None else mask_slopes.data_ptr(),
                None if sinks is None else sinks.data_ptr())


def _io_ok(t: torch.Tensor) -> bool:
    """q and out of the attention calls: CUDA tensors, or page-locked CPU
    tensors, which the kernels read and write over the host link."""
    return t.is_contiguous() and (t.is_cuda or t.is_pinned())


def _attention(fn, q, k, v, L, scale, mask, causal, out, out_dtype, workspace, stream, decode,
               ext=None):
    assert _io_ok(q) and (out is None or _io_ok(out))
    B, Hq, Lq, D = q.shape
    Hkv = k.codes.shape[1]
    dev = k.codes.device                   # the device that runs the call
    if out is None:
        out = torch.empty(B, Hq, Lq, D, dtype=out_dtype or q.dtype, device=dev)
    if workspace is None:
        with _on(k.codes):                 # sized for the device that runs the call
            workspace = make_workspace(B, Hq, Hkv, Lq, D, L, dev)
    ks, vs = k._struct(), v._struct()
    m = _mask_struct(mask, causal)
    mp = C.byref(m) if m is not None else None
    common = (C.byref(ks), C.byref(vs), int(L), float(scale), mp)
    if ext is not None:
        common += (C.byref(ext),)
    with _on(k.codes):
        common += (out.data_ptr(), _DTYPE[out.dtype], workspace.data_ptr(), workspace.numel(),
                   _stream(stream))
        if decode:
            _check(fn(q.data_ptr(), _DTYPE[q.dtype], B, Hq, Hkv, D, *common))
        else:
            _check(fn(q.data_ptr(), _DTYPE[q.dtype], B, Hq, Hkv, Lq, D, *common))
    return out


def qsdpa_decode(q: torch.Tensor, k: QuantCache, v: QuantCache, L: int, scale: float,
                 mask=None, out: Optional[torch.Tensor] = None, out_dtype=None,
                 workspace: Optional[torch.Tensor] = None, stream=None, softcap: float = 0.0,
                 sinks: Optional[torch.Tensor] = None,
                 mask_slopes: Optional[torch.Tensor] = None) -> torch.Tensor:
    """softmax(q*scale . K^T + mask) V for q [B,Hq,1,D] over keys [0, L).
    ``softcap``, ``sinks`` and ``mask_slopes`` are the attention extensions
    of ``qkv_attn_ext`` (qsdpa_decode_ext).  ``q`` and ``out`` may be CUDA
    tensors on the caches' device or page-locked (pinned) CPU tensors: the
    kernels then read q and write out over the host link, with no separate
    copy.  The same holds for :func:`qsdpa_prefill`, whose calls with host
    tensors run on the split-K kernel."""
    assert q.shape[2] == 1
    ext = _ext_struct(softcap, sinks, mask_slopes, q.shape[1], k.codes.device)
    fn = lib().qsdpa_decode if ext is None else lib().qsdpa_decode_ext
    return _attention(fn, q, k, v, L, scale, mask, False, out, out_dtype, workspace, stream,
                      True, ext)


def qsdpa_decode_update(q: torch.Tensor, new_k: torch.Tensor, new_v: torch.Tensor,
                        k: QuantCache, v: QuantCache, L_old: int, scale: float, mask=None,
                        out: Optional[torch.Tensor] = None, out_dtype=None,
                        workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """One fused decode step: quantize new_k/new_v [B,Hkv,1,D] (f16/bf16) into
    cache row L_old, in place, and return softmax(q*scale . K^T + mask) V for
    q [B,Hq,1,D] over the L_old + 1 keys [0, L_old]."""
    assert q.is_contiguous() and q.is_cuda and q.shape[2] == 1
    assert new_k.is_contiguous() and new_v.is_contiguous()
    assert new_k.shape == new_v.shape and new_k.dtype == new_v.dtype and new_k.shape[2] == 1
    B, Hq, _, D = q.shape
    Hkv = k.codes.shape[1]
    if out is None:
        out = torch.empty(B, Hq, 1, D, dtype=out_dtype or q.dtype, device=q.device)
    if workspace is None:
        with _on(q):
            workspace = make_workspace(B, Hq, Hkv, 1, D, L_old + 1, q.device)
    ks, vs = k._struct(), v._struct()
    m = _mask_struct(mask, False)
    mp = C.byref(m) if m is not None else None
    with _on(q):
        _check(lib().qsdpa_decode_update(q.data_ptr(), _DTYPE[q.dtype], new_k.data_ptr(),
                                         new_v.data_ptr(), _DTYPE[new_k.dtype], B, Hq, Hkv, D,
                                         C.byref(ks), C.byref(vs), int(L_old), float(scale), mp,
                                         out.data_ptr(), _DTYPE[out.dtype], workspace.data_ptr(),
                                         workspace.numel(), _stream(stream)))
    return out


def qsdpa_prefill(q: torch.Tensor, k: QuantCache, v: QuantCache, L: int, scale: float,
                  mask=None, causal: bool = False, out: Optional[torch.Tensor] = None,
                  out_dtype=None, workspace: Optional[torch.Tensor] = None,
                  stream=None, softcap: float = 0.0, sinks: Optional[torch.Tensor] = None,
                  mask_slopes: Optional[torch.Tensor] = None) -> torch.Tensor:
    """softmax(q*scale . K^T + mask) V for q [B,Hq,Lq,D] over keys [0, L);
    ``causal`` aligns the Lq queries with the last Lq keys.  ``softcap``,
    ``sinks`` and ``mask_slopes`` as in :func:`qsdpa_decode`."""
    ext = _ext_struct(softcap, sinks, mask_slopes, q.shape[1], k.codes.device)
    fn = lib().qsdpa_prefill if ext is None else lib().qsdpa_prefill_ext
    return _attention(fn, q, k, v, L, scale, mask, causal, out, out_dtype, workspace, stream,
                      False, ext)


def qsdpa_decode_noalloc(q: torch.Tensor, k: QuantCache, v: QuantCache, L: int, scale: float,
                         mask=None, out: Optional[torch.Tensor] = None, out_dtype=None,
                         stream=None) -> torch.Tensor:
    """Like :func:`qsdpa_decode` but without a workspace: the library keeps the
    scratch in a fixed 8 MiB array of its own (for callers that cannot
    allocate device memory at decode time).  ``out`` should be passed by such
    callers; it is only allocated here when omitted.  Calls must not overlap
    on the GPU."""
    f = lib().qsdpa_decode_noalloc
    if f.argtypes is None:
        f.argtypes = [C.c_void_p, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int,
                      C.POINTER(_Cache), C.POINTER(_Cache), C.c_int64, C.c_float,
                      C.POINTER(_Mask), C.c_void_p, C.c_int, C.c_void_p]
        f.restype = C.c_int
    assert _io_ok(q) and (out is None or _io_ok(out)) and q.shape[2] == 1
    B, Hq, _, D = q.shape
    Hkv = k.codes.shape[1]
    if out is None:
        out = torch.empty(B, Hq, 1, D, dtype=out_dtype or q.dtype, device=k.codes.device)
    ks, vs = k._struct(), v._struct()
    m = _mask_struct(mask, False)
    with _on(k.codes):
        _check(f(q.data_ptr(), _DTYPE[q.dtype], B, Hq, Hkv, D, C.byref(ks), C.byref(vs), int(L),
                 float(scale), C.byref(m) if m is not None else None, out.data_ptr(),
                 _DTYPE[out.dtype], _stream(stream)))
    return out


def qsdpa_attention_kview(q: torch.Tensor, k: QuantCache, L: int, scale: float, Dv: int = 512,
                          causal: bool = False, out: Optional[torch.Tensor] = None, out_dtype=None,
                          workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """softmax(q*scale . K^T) V with V the first Dv elements of every key row
    (K rows of 576, Dv 512): q [B,Hq,Lq,576] -> out [B,Hq,Lq,512]; the cache
    holds K only.  ``causal`` aligns the Lq queries with the last Lq keys."""
    assert q.is_contiguous() and q.is_cuda
    B, Hq, Lq, Dk = q.shape
    Hkv = k.codes.shape[1]
    if out is None:
        out = torch.empty(B, Hq, Lq, Dv, dtype=out_dtype or q.dtype, device=q.device)
    with _on(q):
        if workspace is None:
            n = int(lib().qsdpa_kview_workspace_size(B, Hq, Hkv, Lq, Dk, Dv, int(L)))
            workspace = torch.empty(max(n, 16), dtype=torch.uint8, device=q.device)
        ks = k._struct()
        m = _mask_struct(None, causal)
        _check(lib().qsdpa_attention_kview(q.data_ptr(), _DTYPE[q.dtype], B, Hq, Hkv, Lq, Dk, Dv,
                                           C.byref(ks), int(L), float(scale),
                                           C.byref(m) if m is not None else None, out.data_ptr(),
                                           _DTYPE[out.dtype], workspace.data_ptr(),
                                           workspace.numel(), _stream(stream)))
    return out
