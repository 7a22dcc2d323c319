"""The C-ABI library loads, exports every function include/qkv.h declares,
and rejects invalid arguments with the documented status codes before any
CUDA call (these run without a GPU: no compute is launched)."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    txt = open(os.path.join(ROOT, "include", "qkv.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(q\w+)\s*\(", txt)))


@pytest.fixture(scope="module")
def lib():
    from quantized_kv_attention_split_b200 import qkv
    return qkv.lib()


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert {"qkv_quantize_update", "qsdpa_decode", "qsdpa_prefill"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    assert lib.qkv_status_string(0) == b"ok"
    assert lib.qkv_status_string(4) == b"workspace too small"
    assert lib.qkv_status_string(99) == b"unknown status"


FAKE = 0x7f0000000000   # 16-byte aligned, never dereferenced: every call below fails validation


def _cache(qkv, fmt=0, bits=4, gs=64, Lcap=64, codes=FAKE, scales=FAKE + 4096, biases=FAKE + 8192):
    return qkv._Cache(fmt, bits, gs, codes, scales, biases, Lcap)


def _decode(lib, qkv, k, v, D=128, L=16, q=FAKE, out=FAKE + 65536, qdt=0, odt=0, Hq=8, Hkv=2):
    return lib.qsdpa_decode(q, qdt, 1, Hq, Hkv, D, C.byref(k), C.byref(v), L, 1.0, None,
                            out, odt, FAKE + 131072, 1 << 20, None)


def test_decode_validation_errors(lib):
    from quantized_kv_attention_split_b200 import qkv
    ok = _cache(qkv)
    assert _decode(lib, qkv, _cache(qkv, bits=7), ok) == 2                 # unsupported bits
    assert b"bits" in lib.qkv_last_error()
    assert _decode(lib, qkv, _cache(qkv, gs=48), ok) == 2                  # unsupported group
    assert _decode(lib, qkv, ok, ok, D=96) == 2                            # unsupported D
    assert _decode(lib, qkv, _cache(qkv, Lcap=60), _cache(qkv, Lcap=60)) == 3   # Lcap % 8
    assert _decode(lib, qkv, _cache(qkv, codes=FAKE + 4), ok) == 3         # misaligned codes
    assert _decode(lib, qkv, ok, ok, q=FAKE + 2) == 3                       # misaligned q
    assert _decode(lib, qkv, _cache(qkv, biases=0), ok) == 1               # affine without biases
    assert _decode(lib, qkv, _cache(qkv, fmt=1, bits=4, gs=32), ok) == 1    # bad Q8_0 bits
    assert _decode(lib, qkv, ok, _cache(qkv, bits=8)) == 2                  # k/v mismatch
    assert _decode(lib, qkv, ok, ok, L=65) == 1                             # L > Lcap
    assert _decode(lib, qkv, ok, ok, L=-1) == 1
    assert _decode(lib, qkv, ok, ok, Hq=6, Hkv=4) == 1                      # Hq % Hkv
    assert _decode(lib, qkv, ok, ok, qdt=2) == 1                            # q must be 16-bit
    assert _decode(lib, qkv, ok, ok, odt=7) == 1                            # unknown out dtype
    assert _decode(lib, qkv, ok, ok, q=0) == 1                              # NULL q
    m = qkv._Mask(9, None, 0, 0, 0, 0)
    assert lib.qsdpa_decode(FAKE, 0, 1, 8, 2, 128, C.byref(ok), C.byref(ok), 16, 1.0,
                            C.byref(m), FAKE, 0, FAKE, 1 << 20, None) == 1  # unknown mask kind


def test_quantize_validation_errors(lib):
    from quantized_kv_attention_split_b200 import qkv
    ok = _cache(qkv)
    f = lib.qkv_quantize_update
    assert f(FAKE, FAKE, 0, 1, 2, 4, 128, C.byref(ok), C.byref(ok), 61, None) == 1  # offset
    assert f(FAKE, FAKE, 2, 1, 2, 4, 128, C.byref(ok), C.byref(ok), 0, None) == 1   # f32 input
    assert f(FAKE + 8, FAKE, 0, 1, 2, 4, 128, C.byref(ok), C.byref(ok), 0, None) == 3
    assert f(0, FAKE, 0, 1, 2, 4, 128, C.byref(ok), C.byref(ok), 0, None) == 1
    assert f(FAKE, FAKE, 0, 1, 2, 4, 128, C.byref(_cache(qkv, bits=7)), C.byref(ok), 0, None) == 2
    assert f(FAKE, FAKE, 0, 1, 2, 0, 128, C.byref(ok), C.byref(ok), 0, None) == 0   # nothing to do


def test_quantize_rejects_too_many_slabs(lib):
    """The quantizer's grid holds (batch, kv head) slabs in its y dimension:
    more than 65535 of them is refused before any launch."""
    from quantized_kv_attention_split_b200 import qkv
    ok = _cache(qkv)
    f = lib.qkv_quantize_update
    assert f(FAKE, FAKE, 0, 65536, 1, 4, 128, C.byref(ok), C.byref(ok), 0, None) == 2
    assert b"65535" in lib.qkv_last_error()


def test_decode_update_validation_errors(lib):
    """The fused decode step validates the new-token arguments and the cache
    room before any launch."""
    from quantized_kv_attention_split_b200 import qkv
    ok = _cache(qkv)
    f = lib.qsdpa_decode_update

    def call(nk=FAKE + 1024, nv=FAKE + 2048, idt=0, L_old=16, k=ok):
        return f(FAKE, 0, nk, nv, idt, 1, 8, 2, 128, C.byref(k), C.byref(ok), L_old, 1.0, None,
                 FAKE + 65536, 0, FAKE + 131072, 1 << 20, None)
    assert call(L_old=64) == 1                     # no room for the new token (Lcap 64)
    assert b"Lcap" in lib.qkv_last_error()
    assert call(L_old=-1) == 1
    assert call(idt=2) == 1                        # new tokens must be 16-bit
    assert call(nk=0) == 1                         # NULL new_k
    assert call(nv=FAKE + 2056) == 3               # misaligned new_v
    assert call(k=_cache(qkv, bits=7)) == 2        # unsupported format


def test_dequantize_validation_errors(lib):
    from quantized_kv_attention_split_b200 import qkv
    ok = _cache(qkv)
    f = lib.qkv_dequantize
    assert f(C.byref(ok), 1, 2, 128, 65, FAKE, None) == 1                    # L > Lcap
    assert f(C.byref(ok), 1, 2, 128, 16, 0, None) == 1                       # NULL out
    assert f(C.byref(ok), 1, 2, 128, 16, FAKE + 8, None) == 3                # misaligned out
    assert f(C.byref(ok), 70000, 1, 128, 16, FAKE, None) == 2                # slabs > 65535
    assert f(C.byref(_cache(qkv, gs=48)), 1, 2, 128, 16, FAKE, None) == 2    # unsupported group
    assert f(C.byref(ok), 1, 2, 128, 0, FAKE, None) == 0                     # nothing to do


def test_extension_validation_errors(lib):
    """qsdpa_decode_ext / qsdpa_prefill_ext reject a negative, infinite or NaN
    softcap and misaligned extension arrays before any launch."""
    from quantized_kv_attention_split_b200 import qkv
    ok = _cache(qkv)

    def dec(ext):
        return lib.qsdpa_decode_ext(FAKE, 0, 1, 8, 2, 128, C.byref(ok), C.byref(ok), 16, 1.0,
                                    None, C.byref(ext), FAKE + 65536, 0, FAKE + 131072, 1 << 20,
                                    None)

    def pre(ext):
        return lib.qsdpa_prefill_ext(FAKE, 0, 1, 8, 2, 4, 128, C.byref(ok), C.byref(ok), 16, 1.0,
                                     None, C.byref(ext), FAKE + 65536, 0, FAKE + 131072, 1 << 20,
                                     None)
    for f in (dec, pre):
        assert f(qkv._Ext(-1.0, None, None)) == 1
        assert b"softcap" in lib.qkv_last_error()
        assert f(qkv._Ext(float("inf"), None, None)) == 1
        assert f(qkv._Ext(float("nan"), None, None)) == 1
        assert f(qkv._Ext(0.0, FAKE + 2, None)) == 3           # misaligned slopes
        assert f(qkv._Ext(30.0, None, FAKE + 6)) == 3          # misaligned sinks


def test_block_conversion_validation_errors(lib):
    from quantized_kv_attention_split_b200 import qkv
    q8 = _cache(qkv, fmt=1, bits=8, gs=32, biases=0)
    fb, tb = lib.qkv_q8_0_from_blocks, lib.qkv_q8_0_to_blocks
    st = (64 * 4 * 34, 4 * 34, 2 * 4 * 34)                      # token-major, Hkv 2, D 128
    assert fb(FAKE, 1, 2, 128, 16, *st, C.byref(_cache(qkv)), 0, None) == 2   # not Q8_0
    assert fb(FAKE, 1, 2, 128, 16, *st, C.byref(q8), 60, None) == 1           # past Lcap
    assert b"Lcap" in lib.qkv_last_error()
    assert fb(FAKE + 1, 1, 2, 128, 16, *st, C.byref(q8), 0, None) == 3        # odd address
    assert fb(FAKE, 1, 2, 128, 16, 1, 136, 272, C.byref(q8), 0, None) == 3    # odd stride
    assert fb(0, 1, 2, 128, 16, *st, C.byref(q8), 0, None) == 1               # NULL blocks
    assert tb(C.byref(q8), 1, 2, 128, -1, 4, FAKE, *st, None) == 1            # negative offset
    assert tb(C.byref(q8), 1, 2, 96, 0, 4, FAKE, *st, None) == 2              # unsupported D
    assert tb(C.byref(q8), 1, 2, 128, 0, 0, FAKE, *st, None) == 0             # nothing to do


def test_llama_blocks_validation_errors(lib):
    from quantized_kv_attention_split_b200 import qkv
    f = lib.qkv_llama_blocks_to_cache
    a4 = _cache(qkv, fmt=0, bits=4, gs=32)
    a8 = _cache(qkv, fmt=0, bits=8, gs=32)
    st = (64 * 4 * 18, 4 * 18, 2 * 4 * 18)
    assert f(9, FAKE, 1, 2, 128, 16, *st, C.byref(a4), 0, None) == 1          # unknown kind
    assert f(0, FAKE, 1, 2, 128, 16, *st, C.byref(a8), 0, None) == 2          # Q4 into 8-bit
    assert f(2, FAKE, 1, 2, 128, 16, *st, C.byref(a4), 0, None) == 2          # Q5 into 4-bit
    assert f(1, FAKE, 1, 2, 128, 16, *st, C.byref(_cache(qkv, gs=64)), 0, None) == 2  # group 64
    assert f(0, FAKE + 1, 1, 2, 128, 16, *st, C.byref(a4), 0, None) == 3      # odd address
    assert f(3, FAKE, 1, 2, 128, 70, *st, C.byref(a8), 0, None) == 1          # past Lcap


def test_header_is_plain_c(tmp_path):
    """include/qkv.h compiles as C99 (no C++ or CUDA types in the boundary),
    and a C program can take the address of every declared function."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    names = _declared()
    src = tmp_path / "use_qkv.c"
    src.write_text('#include "qkv.h"\ntypedef void (*fn_t)(void);\nfn_t fns[] = {\n' +
                   "".join(f"  (fn_t)&{n},\n" for n in names) + "};\n")
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-pedantic", "-c", str(src),
                        "-I", os.path.join(ROOT, "include"), "-o", str(tmp_path / "use_qkv.o")],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_noalloc_validation_matches_decode(lib):
    """qsdpa_decode_noalloc rejects what qsdpa_decode rejects, with the same
    status, before it looks up its scratch or launches anything."""
    from quantized_kv_attention_split_b200 import qkv
    f = lib.qsdpa_decode_noalloc
    f.argtypes = [C.c_void_p, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int,
                  C.POINTER(qkv._Cache), C.POINTER(qkv._Cache), C.c_int64, C.c_float,
                  C.POINTER(qkv._Mask), C.c_void_p, C.c_int, C.c_void_p]
    f.restype = C.c_int
    ok = _cache(qkv)

    def na(k, v, D=128, L=16, Hq=8, Hkv=2):
        return f(FAKE, 0, 1, Hq, Hkv, D, C.byref(k), C.byref(v), L, 1.0, None, FAKE + 65536, 0,
                 None)
    cases = [
        dict(k=ok, v=ok, D=96),                                   # unsupported D
        dict(k=_cache(qkv, bits=7), v=ok),                        # unsupported bits
        dict(k=_cache(qkv, gs=48), v=ok),                         # unsupported group
        dict(k=_cache(qkv, Lcap=60), v=_cache(qkv, Lcap=60)),     # Lcap alignment
        dict(k=_cache(qkv, biases=0), v=ok),                      # affine without biases
        dict(k=ok, v=ok, L=65),                                   # L > Lcap
        dict(k=ok, v=ok, L=-1),
        dict(k=ok, v=ok, Hq=6, Hkv=4),                            # Hq % Hkv
    ]
    for c in cases:
        want = _decode(lib, qkv, c["k"], c["v"], D=c.get("D", 128), L=c.get("L", 16),
                       Hq=c.get("Hq", 8), Hkv=c.get("Hkv", 2))
        assert want != 0
        assert na(**c) == want, c


def test_llama_quantize_and_export_validation_errors(lib):
    from quantized_kv_attention_split_b200 import qkv
    a4 = _cache(qkv, fmt=0, bits=4, gs=32)
    a8 = _cache(qkv, fmt=0, bits=8, gs=32)
    st = (64 * 4 * 18, 4 * 18, 2 * 4 * 18)
    qb, qu, ex = lib.qkv_llama_quantize_blocks, lib.qkv_llama_quantize_update, lib.qkv_llama_cache_to_blocks
    assert qb(7, FAKE, 0, 1, 2, 128, 16, FAKE, *st, None) == 1                # unknown kind
    assert qb(0, FAKE, 2, 1, 2, 128, 16, FAKE, *st, None) == 1                # f32 input
    assert qb(0, FAKE, 0, 1, 2, 96, 16, FAKE, *st, None) == 2                 # unsupported D
    assert qb(0, FAKE + 8, 0, 1, 2, 128, 16, FAKE, *st, None) == 3            # misaligned x
    assert qb(0, FAKE, 0, 1, 2, 128, 16, FAKE + 1, *st, None) == 3            # odd blocks address
    assert qb(0, FAKE, 0, 1, 2, 128, 0, FAKE, *st, None) == 0                 # nothing to do
    assert qu(0, FAKE, FAKE, 0, 1, 2, 4, 128, C.byref(a8), C.byref(a8), 0, None) == 2   # Q4 into 8-bit
    assert qu(2, FAKE, FAKE, 0, 1, 2, 4, 128, C.byref(a8), C.byref(a8), 61, None) == 1  # past Lcap
    assert qu(1, FAKE + 8, FAKE, 0, 1, 2, 4, 128, C.byref(a4), C.byref(a4), 0, None) == 3
    assert qu(3, FAKE, FAKE, 0, 1, 2, 0, 128, C.byref(a8), C.byref(a8), 0, None) == 0
    assert ex(1, C.byref(a8), 1, 2, 128, 0, 16, FAKE, *st, None) == 2        # Q4 from 8-bit
    assert ex(2, C.byref(a8), 1, 2, 128, 60, 16, FAKE, *st, None) == 1       # past Lcap
    assert ex(0, C.byref(a4), 1, 2, 128, 0, 16, FAKE + 1, *st, None) == 3    # odd address


def test_kview_validation_errors(lib):
    from quantized_kv_attention_split_b200 import qkv
    q8 = _cache(qkv, fmt=1, bits=8, gs=32, biases=0)
    f = lib.qsdpa_attention_kview

    def call(k=q8, Dk=576, Dv=512, odt=0, L=16, ws=1 << 26, mask=None):
        return f(FAKE, 0, 1, 16, 1, 1, Dk, Dv, C.byref(k), L, 0.1,
                 C.byref(mask) if mask is not None else None, FAKE + 65536, odt, FAKE + 131072, ws,
                 None)
    assert call(Dk=512) == 2 and call(Dv=256) == 2                          # shapes other than 576/512
    assert call(k=_cache(qkv, fmt=0, bits=4, gs=128)) == 2                  # group 128
    assert call(k=_cache(qkv, fmt=0, bits=3, gs=32)) == 2                   # 3-bit codes
    assert call(odt=2) == 2                                                 # fp32 out
    assert call(L=65) == 1                                                  # L > Lcap
    assert call(ws=16) == 4                                                 # workspace too small
    assert call(mask=qkv._Mask(2, FAKE, 2, 0, 0, 0)) == 2                   # additive mask
    assert lib.qsdpa_kview_workspace_size(1, 16, 1, 1, 576, 512, 100) > 0
    assert lib.qsdpa_kview_workspace_size(1, 16, 1, 1, 128, 128, 100) == 0
