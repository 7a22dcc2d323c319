"""Argument marshalling of the Python binding (CPU only: nothing is launched)."""
import ctypes as C

import pytest
import torch

from quantized_kv_attention_split_b200 import qkv


def test_mask_struct_from_tensors():
    m = torch.zeros(2, 4, 3, 10, dtype=torch.float16)
    s = qkv._mask_struct(m, False)
    assert s.kind == qkv.MASK_ADDITIVE and s.add_dtype == qkv.F16
    assert (s.stride_b, s.stride_h, s.stride_q) == (120, 30, 10)
    # explicit strides (broadcast over batch and heads), bf16
    mb = torch.zeros(3, 10, dtype=torch.bfloat16)
    s = qkv._mask_struct((mb, (0, 0, 10)), False)
    assert s.add_dtype == qkv.BF16 and (s.stride_b, s.stride_h, s.stride_q) == (0, 0, 10)
    # a 1-D mask broadcasts over everything
    s = qkv._mask_struct(torch.zeros(10), False)
    assert s.add_dtype == qkv.F32 and (s.stride_b, s.stride_h, s.stride_q) == (0, 0, 0)
    assert qkv._mask_struct(None, True).kind == qkv.MASK_CAUSAL
    assert qkv._mask_struct(None, False) is None


def test_ext_struct():
    assert qkv._ext_struct(0.0, None, None, 8, torch.device("cpu")) is None
    e = qkv._ext_struct(30.0, None, None, 8, torch.device("cpu"))
    assert abs(e.softcap - 30.0) < 1e-6 and not e.sinks and not e.mask_slopes
    with pytest.raises(AssertionError):      # sinks must be fp32 device tensors of Hq values
        qkv._ext_struct(0.0, torch.zeros(8), None, 8, torch.device("cpu"))


def test_cache_struct_is_cached_and_follows_the_buffers():
    c = qkv.QuantCache(qkv.AFFINE, 4, 64, torch.zeros(1, 2, 16, 16, dtype=torch.int32),
                       torch.zeros(1, 2, 16, 2, dtype=torch.float16),
                       torch.zeros(1, 2, 16, 2, dtype=torch.float16))
    a = c._struct()
    assert a is c._struct()
    assert (a.fmt, a.bits, a.group_size, a.Lcap) == (qkv.AFFINE, 4, 64, 16)
    assert a.codes == c.codes.data_ptr() and a.biases == c.biases.data_ptr()
    c.codes = torch.zeros(1, 2, 24, 16, dtype=torch.int32)   # new buffers: a new struct
    b = c._struct()
    assert b is not a and b.Lcap == 24 and b.codes == c.codes.data_ptr()


def test_block_strides():
    t = torch.zeros(2, 3, 5, 4 * 34, dtype=torch.uint8)
    assert qkv._block_strides(t, None) == (3 * 5 * 136, 5 * 136, 136)
    assert qkv._block_strides(t, (7, 8, 9)) == (7, 8, 9)
    assert qkv.LLAMA_BLOCKS["q5_1"] == (3, 24, 8) and qkv.Q8_0_BLOCK_BYTES == 34


def test_calls_switch_to_the_tensors_device(monkeypatch):
    """A call whose tensors live on a device that is not the current one runs
    with that device made current (launch, default stream, workspace size);
    on the current device nothing is switched."""
    import contextlib

    class Fake:
        def __init__(self, dev):
            self.device = dev
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    assert isinstance(qkv._on(Fake(torch.device("cuda", 0))), contextlib.nullcontext)
    assert isinstance(qkv._on(Fake(torch.device("cpu"))), contextlib.nullcontext)
    ctx = qkv._on(Fake(torch.device("cuda", 3)))
    assert isinstance(ctx, torch.cuda.device) and ctx.idx == 3
