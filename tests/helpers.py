"""Shared helpers for the tests: moving oracle arrays to torch tensors and
building caches.  Expected values always come from the oracle (``oracle/``);
the CUDA path's results are only ever compared against them."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from quantized_kv_attention_split_b200 import synthetic as S

TOL = {"f16": 2e-3, "bf16": 2e-3, "f32": 1e-4}
TORCH_DT = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}


def to_dev(bits: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    """Raw half bits (uint16) -> torch f16/bf16 tensor on the device."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(TORCH_DT[dtype]).to(device)


def from_dev(t: torch.Tensor) -> np.ndarray:
    """Torch tensor -> float64 numpy (exact)."""
    return t.detach().float().cpu().numpy().astype(np.float64)


def cache_to_dev(c: oracle.QCache, device="cuda"):
    from quantized_kv_attention_split_b200 import qkv
    fmt = qkv.Q8_0 if c.fmt == "q8_0" else qkv.AFFINE
    codes = torch.from_numpy(c.codes.view(np.int32).copy()).to(device)
    scales = torch.from_numpy(c.scales.view(np.float16).copy()).to(device)
    biases = None if c.biases is None else torch.from_numpy(c.biases.view(np.float16).copy()).to(device)
    return qkv.QuantCache(fmt, c.bits, c.gs, codes, scales, biases)


def cache_from_dev(dc, fmt: str) -> oracle.QCache:
    codes = dc.codes.cpu().numpy().view(np.uint32)
    scales = dc.scales.cpu().numpy().view(np.uint16)
    biases = None if dc.biases is None else dc.biases.cpu().numpy().view(np.uint16)
    return oracle.QCache(fmt, dc.bits, dc.group_size, codes, scales, biases)


def make_problem(B, Hq, Hkv, Lq, D, L, fmt="affine", bits=4, gs=64, dist="uniform",
                 q_dtype="f16", kv_dtype="f16", Lcap=None, seed=3):
    """Seeded q (raw bits) and oracle-quantized K/V caches (rows past L are
    filled with quantized values too, so a kernel reading them by mistake
    would change the result)."""
    Lcap = Lcap or ((L + 7) // 8 * 8 if L > 0 else 8)
    q = S.draw(seed, "q", (B, Hq, Lq, D), dist, q_dtype)
    k = S.draw(seed, "k", (B, Hkv, Lcap, D), dist, kv_dtype)
    v = S.draw(seed, "v", (B, Hkv, Lcap, D), dist, kv_dtype)
    kc = oracle.quantize(k, kv_dtype, fmt, gs, bits)
    vc = oracle.quantize(v, kv_dtype, fmt, gs, bits)
    return q, kc, vc


def max_err(a: np.ndarray, b: np.ndarray) -> float:
    return float(np.max(np.abs(a - b))) if a.size else 0.0


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 values at |x| (8 significant bits; 2^-133 below the
    normal range)."""
    a = np.maximum(np.abs(x), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


def out_err(got: np.ndarray, ref: np.ndarray, dtype: str) -> float:
    """Largest error in units of the allowed error.  fp16 / fp32 outputs: max-abs
    error over 2e-3 / 1e-4.  bf16 outputs: within 2e-3 before one correct
    rounding, i.e. |got - ref| <= 2e-3 + half a bf16 ulp of got (a correctly
    rounded bf16 result of a value within 2e-3 of ref always passes; half an
    ulp is 2^-9 < 2e-3 for |x| in [0.5, 1), 2^-8 in [1, 2))."""
    err = np.abs(got - ref)
    if not err.size:
        return 0.0
    if dtype == "bf16":
        return float(np.max(err / (TOL["bf16"] + 0.5 * bf16_ulp(got))))
    return float(np.max(err / TOL[dtype]))
