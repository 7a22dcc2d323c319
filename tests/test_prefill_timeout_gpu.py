"""The tcgen05 prefill kernel's bounded waits, made to run out on purpose
(no fault, no trap, no unbounded spin): the test hook QKV_PREFILL_STALL_HALF
makes the producer warp withhold the copy of one 32-key block, and
QKV_PREFILL_WAIT_NS shortens the limit of every wait to 100 us.  The dequant
warps' wait for that block times out, the CTA gives up (every later wait
returns at once, its own copies and tensor-core work are drained with the
same limit, TMEM is released), the first word of the workspace records the
time-out and the call returns promptly; the next call on a zeroed status word
is correct."""
import time

import numpy as np
import pytest
import torch

import oracle
from helpers import TOL, cache_to_dev, from_dev, make_problem, max_err, to_dev

pytestmark = pytest.mark.gpu


def test_prefill_wait_timeout_sets_status_and_recovers(monkeypatch):
    from quantized_kv_attention_split_b200 import qkv
    B, Hq, Hkv, Lq, D, L = 1, 8, 1, 16, 128, 1000          # 128 rows: the tcgen05 kernel
    q, kc, vc = make_problem(B, Hq, Hkv, Lq, D, L, "q8_0", 8, 32, "normal", q_dtype="bf16",
                             Lcap=1000, seed=12)
    qd, kd, vd = to_dev(q, "bf16"), cache_to_dev(kc), cache_to_dev(vc)
    ws = qkv.make_workspace(B, Hq, Hkv, Lq, D, L)
    monkeypatch.setenv("QKV_PREFILL_WAIT_NS", "100000")
    monkeypatch.setenv("QKV_PREFILL_STALL_HALF", "3")
    t0 = time.time()
    qkv.qsdpa_prefill(qd, kd, vd, L, 0.09, causal=True, out_dtype=torch.float16, workspace=ws)
    torch.cuda.synchronize()
    dt = time.time() - t0
    status = int(ws[:4].view(torch.int32).item())
    assert status & 1, hex(status)                        # the dequant warps' wait ran out
    assert dt < 5.0, dt
    monkeypatch.delenv("QKV_PREFILL_STALL_HALF")
    monkeypatch.delenv("QKV_PREFILL_WAIT_NS")
    ws.zero_()
    out = qkv.qsdpa_prefill(qd, kd, vd, L, 0.09, causal=True, out_dtype=torch.float16, workspace=ws)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0
    ref = oracle.attention(q, "bf16", kc, vc, L, 0.09, mask=oracle.Mask("causal"))
    assert max_err(from_dev(out), ref) <= TOL["f16"]
