"""Attention calls whose q and out live in page-locked host memory.

The C ABI accepts, for q and out of the attention calls, pinned host memory
that the device addresses at the same pointer: the split-K kernels read q and
write out over the host link themselves.  The results must match the CPU
oracle within the parity tolerance and the same call on device buffers; a
multi-query call with host buffers takes the split-K kernel (the tcgen05
kernel wants device memory); L = 0 zeroes a host output; pageable host memory
is refused before anything is launched."""
import numpy as np
import pytest
import torch

import oracle
from helpers import TOL, cache_to_dev, from_dev, make_problem, max_err, to_dev

pytestmark = pytest.mark.gpu


def _pinned(t: torch.Tensor) -> torch.Tensor:
    return t.cpu().pin_memory()


@pytest.mark.parametrize("where", ["both", "q", "out"])
@pytest.mark.parametrize("odt", [torch.float16, torch.float32])
def test_decode_with_host_buffers(where, odt):
    from quantized_kv_attention_split_b200 import qkv
    B, Hq, Hkv, D, L = 1, 32, 8, 128, 9000
    q, kc, vc = make_problem(B, Hq, Hkv, 1, D, L, "affine", 4, 64, seed=71)
    ref = oracle.attention(q, "f16", kc, vc, L, 0.0625)
    qd, kd, vd = to_dev(q, "f16"), cache_to_dev(kc), cache_to_dev(vc)
    dev_out = qkv.qsdpa_decode(qd, kd, vd, L, 0.0625, out_dtype=odt)
    qx = _pinned(qd) if where in ("both", "q") else qd
    if where in ("both", "out"):
        out = torch.full((B, Hq, 1, D), float("nan"), dtype=odt).pin_memory()
    else:
        out = torch.full((B, Hq, 1, D), float("nan"), dtype=odt, device="cuda")
    qkv.qsdpa_decode(qx, kd, vd, L, 0.0625, out=out)
    torch.cuda.synchronize()
    tol = TOL["f32" if odt == torch.float32 else "f16"]
    got = from_dev(out)
    assert max_err(got, ref) <= tol
    assert max_err(got, from_dev(dev_out)) <= tol


def test_multi_query_with_host_buffers_runs_split_k():
    """256 rows per KV head would take the tcgen05 kernel on device buffers."""
    from quantized_kv_attention_split_b200 import qkv
    B, Hq, Hkv, Lq, D, L = 1, 32, 2, 16, 128, 1500
    q, kc, vc = make_problem(B, Hq, Hkv, Lq, D, L, "q8_0", 8, 32, "normal", seed=72)
    ref = oracle.attention_dense(q, "f16", kc, vc, L, 1.0 / np.sqrt(D), causal=True)
    qh = _pinned(to_dev(q, "f16"))
    out = torch.full((B, Hq, Lq, D), float("nan"), dtype=torch.float16).pin_memory()
    qkv.qsdpa_prefill(qh, cache_to_dev(kc), cache_to_dev(vc), L, 1.0 / np.sqrt(D), causal=True,
                      out=out)
    torch.cuda.synchronize()
    assert max_err(from_dev(out), ref) <= TOL["f16"]


def test_noalloc_with_host_buffers():
    from quantized_kv_attention_split_b200 import qkv
    B, Hq, Hkv, D, L = 2, 16, 4, 64, 3000
    q, kc, vc = make_problem(B, Hq, Hkv, 1, D, L, "affine", 8, 32, seed=73)
    ref = oracle.attention(q, "f16", kc, vc, L, 0.125)
    out = torch.full((B, Hq, 1, D), float("nan"), dtype=torch.float32).pin_memory()
    qkv.qsdpa_decode_noalloc(_pinned(to_dev(q, "f16")), cache_to_dev(kc), cache_to_dev(vc), L,
                             0.125, out=out)
    torch.cuda.synchronize()
    assert max_err(from_dev(out), ref) <= TOL["f32"]


def test_empty_cache_zeroes_a_host_output():
    from quantized_kv_attention_split_b200 import qkv
    q, kc, vc = make_problem(1, 8, 2, 1, 128, 64, "affine", 4, 64, seed=74)
    out = torch.full((1, 8, 1, 128), float("nan"), dtype=torch.float16).pin_memory()
    qkv.qsdpa_decode(_pinned(to_dev(q, "f16")), cache_to_dev(kc), cache_to_dev(vc), 0, 1.0,
                     out=out)
    torch.cuda.synchronize()
    assert torch.count_nonzero(out).item() == 0


def test_pageable_host_memory_is_refused_before_launch():
    """Called through ctypes directly: the binding itself only passes CUDA or
    pinned tensors.  The library classifies the pointer and returns an error;
    nothing runs."""
    import ctypes as C
    from quantized_kv_attention_split_b200 import qkv
    B, Hq, Hkv, D, L = 1, 8, 2, 128, 64
    q, kc, vc = make_problem(B, Hq, Hkv, 1, D, L, "affine", 4, 64, seed=75)
    kd, vd = cache_to_dev(kc), cache_to_dev(vc)
    q_pageable = to_dev(q, "f16").cpu()
    assert not q_pageable.is_pinned()
    out = torch.empty(B, Hq, 1, D, dtype=torch.float16, device="cuda")
    ws = qkv.make_workspace(B, Hq, Hkv, 1, D, L)
    ks, vs = kd._struct(), vd._struct()
    lib = qkv.lib()
    st = lib.qsdpa_decode(q_pageable.data_ptr(), qkv.F16, B, Hq, Hkv, D, C.byref(ks), C.byref(vs),
                          L, 1.0, None, out.data_ptr(), qkv.F16, ws.data_ptr(), ws.numel(),
                          torch.cuda.current_stream().cuda_stream)
    assert st == 1, st
    assert b"page-locked" in lib.qkv_last_error()
    torch.cuda.synchronize()
