"""The allocation-free decode entry point (qsdpa_decode_noalloc) against the
regular one (qsdpa_decode, caller workspace), through the C ABI.

qsdpa_decode_noalloc exists for callers that cannot allocate device memory
when they decode (allocators that forbid cudaMalloc, pre-planned services,
plug-in interfaces that pass only inputs and outputs); its scratch is a fixed
array inside the library.  Two calls in a row, on different problems, must
each match the regular entry point within the parity tolerance, so nothing
left in the shared array by one call leaks into the next.  This file is named
to be collected last."""
import numpy as np
import pytest
import torch

from helpers import TOL, cache_to_dev, from_dev, make_problem, max_err, to_dev

pytestmark = pytest.mark.gpu


def test_noalloc_matches_workspace_entry_on_two_calls():
    from quantized_kv_attention_split_b200 import qkv
    qkv.lib()
    problems = [
        # B, Hq, Hkv, D, L, fmt, bits, gs, out dtype
        (1, 32, 8, 128, 20000, "affine", 4, 64, torch.float16),
        (2, 32, 2, 256, 3000, "q8_0", 8, 32, torch.float32),
    ]
    for call, (B, Hq, Hkv, D, L, fmt, bits, gs, odt) in enumerate(problems):
        q, kc, vc = make_problem(B, Hq, Hkv, 1, D, L, fmt, bits, gs,
                                 "normal" if fmt == "q8_0" else "uniform", seed=21 + call)
        qd, kd, vd = to_dev(q, "f16"), cache_to_dev(kc), cache_to_dev(vc)
        ref = qkv.qsdpa_decode(qd, kd, vd, L, 0.0625, out_dtype=odt)
        out = torch.full((B, Hq, 1, D), float("nan"), dtype=odt, device="cuda")
        qkv.qsdpa_decode_noalloc(qd, kd, vd, L, 0.0625, out=out)
        torch.cuda.synchronize()
        tol = TOL["f32" if odt == torch.float32 else "f16"]
        assert max_err(from_dev(out), from_dev(ref)) <= tol, (call, max_err(from_dev(out),
                                                                            from_dev(ref)))


def test_noalloc_rejects_shapes_beyond_its_scratch():
    from quantized_kv_attention_split_b200 import qkv
    q, kc, vc = make_problem(1, 64, 1, 1, 256, 64, "affine", 8, 64)
    qd, kd, vd = to_dev(q, "f16"), cache_to_dev(kc), cache_to_dev(vc)
    need = qkv.qsdpa_workspace_size(1, 64, 1, 1, 256, 64)
    if need <= 8 << 20:
        pytest.skip(f"shape fits the built-in scratch on this device ({need} bytes)")
    with pytest.raises(qkv.QKVError, match="scratch"):
        qkv.qsdpa_decode_noalloc(qd, kd, vd, 64, 1.0)
