"""The allocation-free decode entry point (qsdpa_decode_noalloc), through the
C ABI, against the CPU oracle and against the regular entry point
(qsdpa_decode, caller workspace).

qsdpa_decode_noalloc exists for callers that cannot allocate device memory
when they decode (allocators that forbid cudaMalloc, pre-planned services,
plug-in interfaces that pass only inputs and outputs); its scratch is a fixed
array inside the library.  Two calls in a row, on different problems, must
each match the oracle within the parity tolerance, and the regular entry point
within the same tolerance, so nothing left in the shared array by one call
leaks into the next.  (The two entry points run the same kernels with the same
plan, but not bit for bit alike: the decode kernel's warps take blocks of keys
from a shared counter as they become free, so the order of the fp32 sums, and
the last bits of a result, can change from run to run.)  This file is named
to be collected last; it also passes when run alone in a fresh process."""
import numpy as np
import pytest
import torch

import oracle
from helpers import TOL, cache_to_dev, from_dev, make_problem, max_err, to_dev

pytestmark = pytest.mark.gpu

NOALLOC_LIMIT = 8 << 20


def test_noalloc_matches_oracle_and_workspace_entry_on_two_calls():
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
        ref = oracle.attention(q, "f16", kc, vc, L, 0.0625)
        qd, kd, vd = to_dev(q, "f16"), cache_to_dev(kc), cache_to_dev(vc)
        regular = qkv.qsdpa_decode(qd, kd, vd, L, 0.0625, out_dtype=odt)
        out = torch.full((B, Hq, 1, D), float("nan"), dtype=odt, device="cuda")
        qkv.qsdpa_decode_noalloc(qd, kd, vd, L, 0.0625, out=out)
        torch.cuda.synchronize()
        tol = TOL["f32" if odt == torch.float32 else "f16"]
        assert max_err(from_dev(out), ref) <= tol, (call, max_err(from_dev(out), ref))
        assert max_err(from_dev(out), from_dev(regular)) <= tol, call


def test_noalloc_rejects_shapes_beyond_its_scratch():
    """32 rows per KV head at D = 256 need 2 partial slots of 32 x 256 fp32
    per CTA of a grid of one CTA per SM: more than 8 MiB on a 148-SM B200."""
    from quantized_kv_attention_split_b200 import qkv
    q, kc, vc = make_problem(1, 64, 1, 1, 256, 64, "affine", 8, 64)
    qd, kd, vd = to_dev(q, "f16"), cache_to_dev(kc), cache_to_dev(vc)
    need = qkv.qsdpa_workspace_size(1, 64, 1, 1, 256, 64)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert need > NOALLOC_LIMIT or sms < 128, (need, sms)
    if need <= NOALLOC_LIMIT:
        pytest.skip(f"shape fits the built-in scratch on this {sms}-SM device")
    with pytest.raises(qkv.QKVError, match="scratch"):
        qkv.qsdpa_decode_noalloc(qd, kd, vd, 64, 1.0)
    # a shape that fits runs (the same call with 8 query heads)
    q, kc, vc = make_problem(1, 8, 1, 1, 256, 64, "affine", 8, 64)
    out = qkv.qsdpa_decode_noalloc(to_dev(q, "f16"), cache_to_dev(kc), cache_to_dev(vc), 64,
                                   1.0, out_dtype=torch.float32)
    torch.cuda.synchronize()
    ref = oracle.attention(q, "f16", kc, vc, 64, 1.0)
    assert max_err(from_dev(out), ref) <= TOL["f32"]
