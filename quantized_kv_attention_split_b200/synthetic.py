"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle.

This module holds random-number generation and the workload shapes only -- no
quantization, dequantization or attention arithmetic.  Values are produced by
a counter-based SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom
number generators", OOPSLA 2014): output i of a stream with seed s is the
SplitMix64 finalizer applied to s + (i+1)*0x9E3779B97F4A7C15.  Uniforms take
the top 24 bits (U[0,1) exactly representable in fp32); normals use the
Box-Muller transform on consecutive uniform pairs.  Draws are made in fp32 and
rounded to fp16 / bf16 with round-to-nearest-even.

The workload shapes mirror the pages' benchmarks: the MLX quantized SDPA
benchmark (L=65536, 32 query heads, 8 KV heads, D=128, uniform q/k/v, 4-bit
affine groups of 64, scale 1.0, seed 3) and the llama.cpp Q8_0 KV shapes
(D=256, 32 query heads over 2 KV heads, 10K/20K cache depth, 512-query
prompts).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np

GAMMA = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB
_CHUNK = 1 << 22


def _mix(z: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * np.uint64(_M1)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(_M2)
        return z ^ (z >> np.uint64(31))


def splitmix64(seed: int, n: int, offset: int = 0) -> np.ndarray:
    """Outputs offset .. offset+n-1 of the SplitMix64 stream with this seed."""
    out = np.empty(n, np.uint64)
    s = np.uint64(seed & 0xFFFFFFFFFFFFFFFF)
    for a in range(0, n, _CHUNK):
        b = min(n, a + _CHUNK)
        i = np.arange(offset + a + 1, offset + b + 1, dtype=np.uint64)
        with np.errstate(over="ignore"):
            z = s + i * np.uint64(GAMMA)
        out[a:b] = _mix(z)
    return out


def sub_seed(seed: int, name: str) -> int:
    """Independent stream seed for a named tensor (FNV-1a of the name, mixed)."""
    h = 0xCBF29CE484222325
    for ch in name.encode():
        h = ((h ^ ch) * 0x100000001B3) & 0xFFFFFFFFFFFFFFFF
    z = np.array([(seed ^ h) & 0xFFFFFFFFFFFFFFFF], np.uint64)
    return int(_mix(z)[0])


def uniform01(seed: int, n: int) -> np.ndarray:
    """U[0,1) in fp32: top 24 bits of each output times 2^-24."""
    u = splitmix64(seed, n) >> np.uint64(40)
    return u.astype(np.float32) * np.float32(2.0 ** -24)


def normal(seed: int, n: int) -> np.ndarray:
    """N(0,1) in fp32 via Box-Muller on pairs (u1, u2) of the stream."""
    m = (n + 1) // 2
    u = (splitmix64(seed, 2 * m) >> np.uint64(40)).astype(np.float64) * 2.0 ** -24
    u1, u2 = u[0::2], u[1::2]
    r = np.sqrt(-2.0 * np.log1p(-u1))          # 1-u1 in (0, 1]
    z = np.empty(2 * m, np.float64)
    z[0::2] = r * np.cos(2.0 * np.pi * u2)
    z[1::2] = r * np.sin(2.0 * np.pi * u2)
    return z[:n].astype(np.float32)


def f32_to_half_bits(x: np.ndarray, dtype: str) -> np.ndarray:
    """fp32 -> raw fp16 / bf16 bits, round-to-nearest-even."""
    x = np.asarray(x, np.float32)
    if dtype == "f16":
        return x.astype(np.float16).view(np.uint16)
    if dtype == "bf16":
        u = x.view(np.uint32).astype(np.uint64)
        lower = u & np.uint64(0xFFFF)
        upper = u >> np.uint64(16)
        up = (lower > 0x8000) | ((lower == 0x8000) & ((upper & np.uint64(1)) == 1))
        return (upper + up.astype(np.uint64)).astype(np.uint16)
    raise ValueError(dtype)


def draw(seed: int, name: str, shape, dist: str, dtype: str) -> np.ndarray:
    """Raw half bits (uint16) of a tensor drawn from U[0,1) or N(0,1)."""
    n = int(np.prod(shape))
    s = sub_seed(seed, name)
    x = uniform01(s, n) if dist == "uniform" else normal(s, n)
    return f32_to_half_bits(x, dtype).reshape(shape)


# ----------------------------------------------------------------------------
# workloads
# ----------------------------------------------------------------------------
@dataclass
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    Lq: int
    L: int                 # keys attended to
    Lcap: int              # cache row capacity
    fmt: str               # affine | q8_0
    bits: int
    gs: int
    dist: str              # uniform | normal
    q_dtype: str
    kv_dtype: str
    out_dtype: str
    scale: float
    mask: str = "none"     # none | causal
    update_tokens: int = 0  # tokens quantized and appended before attending
    seed: int = 3
    notes: str = ""

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def words(self) -> int:
        return self.D * self.bits // 32

    @property
    def ngroups(self) -> int:
        return self.D // self.gs

    def cache_bytes(self, L: Optional[int] = None) -> int:
        """Bytes of K+V codes and metadata for L keys (all heads)."""
        L = self.L if L is None else L
        per_row = self.words * 4 + self.ngroups * 2 * (2 if self.fmt == "affine" else 1)
        return 2 * self.B * self.Hkv * L * per_row


WORKLOADS = {
    "tiny_decode": Workload("tiny_decode", 1, 4, 1, 64, 1, 256, 256, "affine", 4, 64,
                            "uniform", "f16", "f16", "f16", 1.0),
    "decode_64k_affine4": Workload("decode_64k_affine4", 1, 32, 8, 128, 1, 65536, 65536,
                                   "affine", 4, 64, "uniform", "f16", "f16", "f16", 1.0),
    "decode_64k_affine8_update": Workload(
        "decode_64k_affine8_update", 1, 32, 8, 128, 1, 65536, 65536, "affine", 8, 64,
        "uniform", "f16", "f16", "f16", 1.0, update_tokens=1),
    "decode_q8_0_10k": Workload("decode_q8_0_10k", 1, 32, 2, 256, 1, 10240, 10240, "q8_0",
                                8, 32, "normal", "f16", "f16", "f16", 1.0 / 16),
    "decode_q8_0_20k": Workload("decode_q8_0_20k", 1, 32, 2, 256, 1, 20480, 20480, "q8_0",
                                8, 32, "normal", "f16", "f16", "f16", 1.0 / 16),
    "prefill_q8_0_512_at_20k": Workload(
        "prefill_q8_0_512_at_20k", 1, 32, 2, 256, 512, 20992, 20992, "q8_0", 8, 32,
        "normal", "bf16", "f16", "bf16", 1.0 / 16, mask="causal"),
}


@dataclass
class Inputs:
    q: np.ndarray                      # raw bits [B,Hq,Lq,D]
    k: np.ndarray                      # raw bits [B,Hkv,Lk,D] (source values)
    v: np.ndarray
    new_k: Optional[np.ndarray] = None  # [B,Hkv,update_tokens,D]
    new_v: Optional[np.ndarray] = None
    extra: dict = field(default_factory=dict)


def make_inputs(w: Workload, L: Optional[int] = None, seed: Optional[int] = None) -> Inputs:
    """Source tensors of a workload (before quantization).  ``L`` overrides the
    number of cached tokens drawn (defaults to the keys present before any
    update)."""
    seed = w.seed if seed is None else seed
    Lk = (w.L - w.update_tokens) if L is None else L
    q = draw(seed, "q", (w.B, w.Hq, w.Lq, w.D), w.dist, w.q_dtype)
    k = draw(seed, "k", (w.B, w.Hkv, Lk, w.D), w.dist, w.kv_dtype)
    v = draw(seed, "v", (w.B, w.Hkv, Lk, w.D), w.dist, w.kv_dtype)
    nk = nv = None
    if w.update_tokens:
        nk = draw(seed, "new_k", (w.B, w.Hkv, w.update_tokens, w.D), w.dist, w.kv_dtype)
        nv = draw(seed, "new_v", (w.B, w.Hkv, w.update_tokens, w.D), w.dist, w.kv_dtype)
    return Inputs(q, k, v, nk, nv)


# ----------------------------------------------------------------------------
# edge-case inputs (structure chosen to drive the kernels' rare paths; values
# are still seeded draws, rounded once to the half type)
# ----------------------------------------------------------------------------
def value_spikes(seed: int, shape, dtype: str, period: int, lo_exp: float, hi_exp: float,
                 gs: int) -> np.ndarray:
    """[B, Hkv, L, D] raw half bits: U[0,1) values, and in every `period`-th
    row (a seeded phase per head) one element of each group of `gs` (a
    seeded position) replaced by 2^e, e growing linearly from lo_exp at row 0
    to hi_exp at the last row -- magnitudes that grow along the cache."""
    B, H, L, D = shape
    x = uniform01(sub_seed(seed, "vs_base"), B * H * L * D).reshape(B, H, L, D)
    pick = splitmix64(sub_seed(seed, "vs_pick"), B * H * (1 + D // gs))
    rows = np.arange(L)
    e = lo_exp + (hi_exp - lo_exp) * rows / max(1, L - 1)
    k = 0
    for b in range(B):
        for h in range(H):
            phase = int(pick[k] % np.uint64(period)); k += 1
            sel = rows[(rows % period) == phase]
            for g in range(D // gs):
                col = g * gs + int(pick[k] % np.uint64(gs)); k += 1
                x[b, h, sel, col] = np.exp2(e[sel])
    return f32_to_half_bits(x, dtype)


def key_levels(seed: int, shape, dtype: str, level: np.ndarray, noise: float = 0.1) -> np.ndarray:
    """[B, Hkv, L, D] raw half bits: row j of every head is level[j] plus
    `noise` * U[0,1) per element (with queries of positive entries, a row's
    logit grows with its level, so `level` shapes the logits along the
    cache: steps, isolated spikes, ramps)."""
    B, H, L, D = shape
    u = uniform01(sub_seed(seed, "kl_noise"), B * H * L * D).reshape(B, H, L, D)
    x = np.asarray(level, np.float32)[None, None, :, None] + np.float32(noise) * u
    return f32_to_half_bits(x, dtype)


def spike_positions(seed: int, L: int, n: int, lo: int = 0) -> np.ndarray:
    """n distinct seeded row indices in [lo, L), sorted."""
    r = splitmix64(sub_seed(seed, "spk"), 4 * n)
    pos = np.unique((r % np.uint64(L - lo)).astype(np.int64) + lo)
    return pos[:n]
