"""Host-side checks of the C-ABI library (no GPU needed).

* libtq.so loads and exports every function include/tq.h declares.
* The library's host Lloyd-Max codebook (its own C++ implementation) agrees
  with the oracle's.
* Argument validation returns the documented status before any launch.
"""

import ctypes
import os
import re

import numpy as np
import pytest

from kv_cache_quantization_turboquantprod_b200 import tq
from oracle import codebook

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "tq.h")).read()
    return sorted(set(re.findall(r"TQ_API\s+[\w\s\*]*?\b(tq_\w+)\s*\(", src)))


def test_header_declares_the_binding_exports():
    assert _declared_functions() == sorted(tq.EXPORTS)


def test_library_exports_every_declared_symbol():
    lib = tq.load()
    for name in _declared_functions():
        assert hasattr(lib, name), name
    out = os.popen(f"nm -D --defined-only {tq.LIB_PATH}").read()
    exported = set(re.findall(r"\bT (tq_\w+)", out))
    assert set(_declared_functions()) <= exported
    # nothing else of ours leaks out of the library
    assert {s for s in exported if s.startswith("tq")} == set(_declared_functions())


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
@pytest.mark.parametrize("d", [64, 128])
def test_host_codebook_matches_oracle(bits, d):
    c, b = tq.tq_make_codebook(bits, d)
    oc, ob, _ = codebook.lloyd_max_gaussian(bits, d)
    assert np.allclose(c, oc, rtol=0, atol=1e-13)
    assert np.allclose(b, ob, rtol=0, atol=1e-13)
    # exactly antisymmetric in float64 and in the float32 the kernels read
    # (the kernels' symmetric fast paths test exactly that)
    c, b = np.asarray(c), np.asarray(b)
    assert np.array_equal(c, -c[::-1]) and np.array_equal(b, -b[::-1])
    c32, b32 = c.astype(np.float32), b.astype(np.float32)
    assert np.array_equal(c32, -c32[::-1]) and np.array_equal(b32, -b32[::-1])


def test_codebook_argument_errors():
    lib = tq.load()
    buf = (ctypes.c_double * 16)()
    assert lib.tq_make_codebook(0, 128, buf, buf) == 2
    assert lib.tq_make_codebook(5, 128, buf, buf) == 2
    assert lib.tq_make_codebook(2, 0, buf, buf) == 2
    assert lib.tq_make_codebook(2, 128, None, buf) == 1


def test_status_strings():
    for code, name in tq.STATUS.items():
        assert tq.tq_status_string(code) == name


def _params(d=128, kb=3, vb=2, g=32, ptr=256, mode=0, vptr=None, wptr=256, optr=None):
    return tq.Params(d, kb, vb, g, ptr, ptr, ptr, ptr, mode, vptr, vptr, wptr, optr)


def test_record_and_cache_bytes():
    lib = tq.load()
    P = _params()
    assert lib.tq_record_bytes(ctypes.byref(P)) == 100
    assert lib.tq_record_bytes(ctypes.byref(_params(kb=4))) == 116
    assert lib.tq_record_bytes(ctypes.byref(_params(vb=3))) == 116
    assert lib.tq_cache_bytes(ctypes.byref(P), 2, 8, 256) == 2 * 8 * 2 * 12800
    assert lib.tq_cache_bytes(ctypes.byref(P), 2, 8, 200) == 0     # not a tile multiple
    assert lib.tq_record_bytes(ctypes.byref(_params(d=64))) == 52       # head dims 64 and 256
    assert lib.tq_record_bytes(ctypes.byref(_params(d=256))) == 196
    assert lib.tq_record_bytes(ctypes.byref(_params(d=96))) == 0
    assert lib.tq_record_bytes(ctypes.byref(_params(g=16))) == 0
    assert lib.tq_record_bytes(ctypes.byref(_params(kb=5))) == 0
    # Pi and S must be 16-byte aligned (the kernels stage them with 16-byte loads)
    misaligned = tq.Params(128, 3, 2, 32, 264, 256, 256, 256)
    assert lib.tq_record_bytes(ctypes.byref(misaligned)) == 0
    misaligned = tq.Params(128, 3, 2, 32, 256, 260, 256, 256)
    assert lib.tq_record_bytes(ctypes.byref(misaligned)) == 0
    # TurboQuant-MSE values: 102-byte records, the values' codebook required
    assert lib.tq_record_bytes(ctypes.byref(_params(vb=3, mode=1, vptr=256))) == 102
    assert lib.tq_record_bytes(ctypes.byref(_params(vb=3, mode=1))) == 0
    assert lib.tq_record_bytes(ctypes.byref(_params(vb=3, mode=2, vptr=256))) == 0
    assert lib.tq_cache_bytes(ctypes.byref(_params(vb=3, mode=1, vptr=256)), 1, 2, 256) == 2 * 2 * 13056


def test_append_validation_before_launch():
    """Every error below is detected on the host; nothing touches a GPU."""
    lib = tq.load()
    P = _params()
    C = tq.Cache(2, 8, 256, 1 << 20)
    lens = (ctypes.c_int32 * 2)(0, 250)
    k = v = 1 << 21
    f = lib.tq_quantize_append
    assert f(None, ctypes.byref(C), k, v, 1, 4, lens, None, None) == 1
    assert f(ctypes.byref(_params(d=96)), ctypes.byref(C), k, v, 1, 4, lens, None, None) == 2
    assert f(ctypes.byref(P), None, k, v, 1, 4, lens, None, None) == 1
    assert f(ctypes.byref(P), ctypes.byref(C), k, v, 7, 4, lens, None, None) == 2   # dtype
    assert f(ctypes.byref(P), ctypes.byref(C), k, v, 1, -1, lens, None, None) == 1
    assert f(ctypes.byref(P), ctypes.byref(C), k, v, 1, 4, None, None, None) == 1
    assert f(ctypes.byref(P), ctypes.byref(C), None, v, 1, 4, lens, None, None) == 1
    assert f(ctypes.byref(P), ctypes.byref(C), k + 2, v, 1, 4, lens, None, None) == 1  # align
    assert f(ctypes.byref(P), ctypes.byref(C), k, v, 1, 7, lens, None, None) == 3   # 250+7>256
    nn = (ctypes.c_int32 * 2)(4, 9)
    assert f(ctypes.byref(P), ctypes.byref(C), k, v, 1, 8, lens, nn, None) == 1     # 9 > T
    nn = (ctypes.c_int32 * 2)(4, 7)
    assert f(ctypes.byref(P), ctypes.byref(C), k, v, 1, 8, lens, nn, None) == 3
    bad = (ctypes.c_int32 * 2)(-1, 0)
    assert f(ctypes.byref(P), ctypes.byref(C), k, v, 1, 4, bad, None, None) == 1
    Cmis = tq.Cache(2, 8, 256, (1 << 20) + 16)                                     # data align
    assert f(ctypes.byref(P), ctypes.byref(Cmis), k, v, 1, 4, lens, None, None) == 1
    Cbig = tq.Cache(tq.MAX_BATCH + 1, 1, 128, 1 << 20)
    big = (ctypes.c_int32 * (tq.MAX_BATCH + 1))()
    assert f(ctypes.byref(P), ctypes.byref(Cbig), k, v, 1, 4, big, None, None) == 3
    # T = 0 is a no-op that succeeds without launching
    assert f(ctypes.byref(P), ctypes.byref(C), None, None, 1, 0, lens, None, None) == 0
    # the float64 product S Pi^T is required, 16-byte aligned
    assert f(ctypes.byref(_params(wptr=None)), ctypes.byref(C), k, v, 1, 4, lens, None, None) == 1
    assert f(ctypes.byref(_params(wptr=264)), ctypes.byref(C), k, v, 1, 4, lens, None, None) == 1


def test_sketch_product_validation():
    lib = tq.load()
    f = lib.tq_sketch_product
    assert f(None, 1 << 20, None) == 1
    assert f(ctypes.byref(_params()), None, None) == 1
    assert f(ctypes.byref(_params()), (1 << 20) + 8, None) == 1         # output alignment
    assert f(ctypes.byref(_params(d=96)), 1 << 20, None) == 2
    assert f(ctypes.byref(_params(ptr=260)), 1 << 20, None) == 1        # Pi / S alignment


def test_prepare_operands_validation():
    lib = tq.load()
    f = lib.tq_prepare_operands
    assert f(None, 1 << 20, None) == 1
    assert f(ctypes.byref(_params()), None, None) == 1
    assert f(ctypes.byref(_params()), (1 << 20) + 64, None) == 1        # output alignment (128 bytes)
    assert f(ctypes.byref(_params(d=64)), 1 << 20, None) == 2          # the tensor-core append is d = 128 only
    assert f(ctypes.byref(_params(wptr=None)), 1 << 20, None) == 1     # needs W = S Pi^T
    assert f(ctypes.byref(_params(ptr=260)), 1 << 20, None) == 1       # Pi alignment
    assert tq.TQ_TC_OPERAND_BYTES == 5 * 128 * 128 * 2


def test_decode_validation_before_launch():
    lib = tq.load()
    P = _params()
    C = tq.Cache(2, 8, 256, 1 << 20)
    f = lib.tq_decode_attention
    q, ln, out, ws = 1 << 22, 1 << 23, 1 << 24, 1 << 25
    args = lambda **kw: [kw.get("p", ctypes.byref(P)), kw.get("c", ctypes.byref(C)),
                         kw.get("q", q), kw.get("dt", 1), kw.get("hq", 32), kw.get("ln", ln),
                         kw.get("ml", 256), kw.get("sc", 0.088), kw.get("out", out),
                         kw.get("ws", ws), kw.get("wsb", 1 << 20), None]
    assert f(*args(p=None)) == 1
    assert f(*args(q=None)) == 1
    assert f(*args(ln=None)) == 1
    assert f(*args(out=None)) == 1
    assert f(*args(hq=12)) == 1           # not a multiple of h_kv
    assert f(*args(hq=4)) == 1            # fewer than h_kv
    assert f(*args(hq=80)) == 2           # G = 10 not built
    assert f(*args(ml=257)) == 1          # beyond capacity
    assert f(*args(ml=-1)) == 1
    assert f(*args(sc=float("inf"))) == 1
    assert f(*args(ws=None)) == 4
    assert f(*args(ws=ws + 8)) == 4       # workspace alignment
    assert f(*args(dt=3)) == 2


def test_dequantize_validation_before_launch():
    lib = tq.load()
    P = _params()
    C = tq.Cache(2, 8, 256, 1 << 20)
    f = lib.tq_dequantize
    o = 1 << 22
    assert f(ctypes.byref(P), ctypes.byref(C), 2, 0, 1, o, o, None) == 1
    assert f(ctypes.byref(P), ctypes.byref(C), 0, 200, 57, o, o, None) == 1
    assert f(ctypes.byref(P), ctypes.byref(C), 0, -1, 1, o, o, None) == 1
    assert f(ctypes.byref(P), ctypes.byref(C), 0, 0, 1, None, o, None) == 1
    assert f(ctypes.byref(P), ctypes.byref(C), 0, 0, 0, None, None, None) == 0


def test_prefill_validation_before_launch():
    lib = tq.load()
    P = _params()
    C = tq.Cache(2, 8, 256, 1 << 20)
    f = lib.tq_prefill_attention
    q, ln, out, ws = 1 << 22, 1 << 23, 1 << 24, 1 << 25
    args = lambda **kw: [kw.get("p", ctypes.byref(P)), kw.get("c", ctypes.byref(C)),
                         kw.get("q", q), kw.get("dt", 1), kw.get("hq", 32), kw.get("t", 4),
                         kw.get("ln", ln), kw.get("ml", 256), kw.get("sc", 0.088), kw.get("out", out),
                         kw.get("ws", ws), kw.get("wsb", 1 << 20), None]
    assert f(*args(p=None)) == 1
    assert f(*args(q=None)) == 1
    assert f(*args(out=None)) == 1
    assert f(*args(hq=12)) == 1           # not a multiple of h_kv
    assert f(*args(hq=80)) == 2           # G = 10 not built
    assert f(*args(t=0)) == 1             # empty chunk
    assert f(*args(t=300)) == 1           # chunk longer than max_len
    assert f(*args(ml=257)) == 1          # beyond capacity
    assert f(*args(sc=float("nan"))) == 1
    assert f(*args(ws=None)) == 4
    assert f(*args(ws=ws + 8)) == 4
    assert f(*args(dt=3)) == 2


def test_prefill_tokens_per_pass():
    """Passes take the largest power of two of query tokens with G x tokens <= 4
    that the tensor-core kernel is built for (one token from GQA 4 up)."""
    lib = tq.load()
    P = _params()
    g = lib.tq_prefill_tokens_per_pass
    assert g(ctypes.byref(P), 32, 8, 8) == 1     # GQA 4
    assert g(ctypes.byref(P), 16, 8, 8) == 2     # GQA 2
    assert g(ctypes.byref(P), 8, 8, 8) == 4      # GQA 1
    assert g(ctypes.byref(P), 8, 8, 3) == 2      # capped by the chunk
    assert g(ctypes.byref(P), 8, 8, 1) == 1
    assert g(ctypes.byref(P), 64, 8, 8) == 1     # GQA 8
    assert g(ctypes.byref(P), 12, 8, 8) == 0     # not a multiple of h_kv
    assert g(ctypes.byref(P), 32, 8, 0) == 0
    assert g(None, 32, 8, 8) == 0


def test_noalloc_validation_before_launch():
    """The no-allocation entry point runs the same host checks as
    tq_decode_attention before it looks up its scratch or launches anything:
    a misaligned Pi or S (read with 16-byte loads) is rejected here rather
    than faulting on the device."""
    lib = tq.load()
    C = tq.Cache(2, 8, 256, 1 << 20)
    f = lib.tq_decode_attention_noalloc
    q, ln, out = 1 << 22, 1 << 23, 1 << 24

    def call(P, **kw):
        return f(ctypes.byref(P) if P is not None else None, ctypes.byref(C), kw.get("q", q), 1,
                 kw.get("hq", 32), ln, kw.get("ml", 256), 0.088, kw.get("out", out), None)

    assert call(tq.Params(128, 3, 2, 32, 264, 256, 256, 256, 0, None, None)) == 1   # Pi misaligned
    assert call(tq.Params(128, 3, 2, 32, 256, 260, 256, 256, 0, None, None)) == 1   # S misaligned
    assert call(None) == 1
    assert call(_params(d=96)) == 2
    assert call(_params(), q=None) == 1
    assert call(_params(), q=q + 4) == 1      # q alignment
    assert call(_params(), out=out + 4) == 1  # out alignment
    assert call(_params(), hq=12) == 1
    assert call(_params(), ml=257) == 1


def test_wait_limit_and_error_word_entry_points():
    lib = tq.load()
    assert lib.tq_set_wait_limit_ns(5000) == 0
    assert lib.tq_set_wait_limit_ns(0) == 0       # back to the default
    assert lib.tq_device_errors(None, 0) == 1     # null pointer, checked before the device


def test_refinement_test_hooks_validate():
    lib = tq.load()
    assert lib.tq_test_sign_refine_threshold(-1.0) == 1          # negative: invalid
    assert lib.tq_test_sign_refine_threshold(float("nan")) == 1
    assert lib.tq_test_sign_refine_threshold(1e-3) == 0
    assert lib.tq_test_sign_refine_threshold(0.0) == 0           # back to the default
    assert lib.tq_test_refine_count(None, 0) == 1                # null pointer, before the device
