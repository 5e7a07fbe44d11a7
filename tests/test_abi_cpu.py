"""The C-ABI library loads and exports every symbol include/fp4attn.h declares,
and argument validation rejects bad calls before anything is launched.
CPU only: no call here reaches the GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def fa():
    from nvfp4_precision_b200 import build
    build.build()
    from nvfp4_precision_b200 import fp4attn
    return fp4attn


def declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(fp4attn_[a-z0-9_]+)\s*\(", src))
    return names


def test_every_declared_symbol_is_exported(fa):
    names = declared_functions()
    assert {"fp4attn_quantize_qk", "fp4attn_forward", "fp4attn_dequant"} <= names
    lib = ctypes.CDLL(fa.LIB_PATH)
    for n in sorted(names):
        assert hasattr(lib, n), n
    assert set(fa.EXPORTS) >= names


def test_status_strings_and_workspace(fa):
    assert fa.status_string(0) == "ok"
    assert "wait" in fa.status_string(fa.ERR_TIMEOUT)
    assert fa.status_string(99) == "unknown status"
    ws = fa.fp4attn_workspace_bytes(1, 48, 109568)
    assert ws >= 48 * 128 * 8 + 4 and ws % 256 == 0
    assert fa.fp4attn_workspace_bytes(0, 0, 0) > 0


def _q(fa, shape, ws=ctypes.c_void_p(256), wsb=1 << 20, flags=0, ptr=ctypes.c_void_p(4096)):
    return fa.lib.fp4attn_quantize_qk(ptr, ptr, shape, None, None, flags, ptr, ptr, ptr, ptr, None, ws, wsb, None)


def test_quantize_validation_before_launch(fa):
    S = fa.Shape
    assert _q(fa, S(1, 1, 128, 96)) == fa.ERR_UNSUPPORTED          # D other than 64 or 128
    assert _q(fa, S(1, 1, 128, 256)) == fa.ERR_UNSUPPORTED
    assert fa.lib.fp4attn_quantize_qk_ex(ctypes.c_void_p(4096), fa.Strides(0, 0, 0), ctypes.c_void_p(4096),
                                         fa.Strides(0, 0, 0), S(1, 1, 128, 64), ctypes.c_void_p(4096),
                                         ctypes.c_void_p(4096), fa.DYNAMIC_GSCALE, *(4 * [ctypes.c_void_p(4096)]),
                                         None, ctypes.c_void_p(256), 1 << 20, None) \
        == fa.ERR_UNSUPPORTED                                       # dynamic scales: 128 channels only
    assert _q(fa, S(1, -1, 128, 128)) == fa.ERR_INVALID_ARG        # negative size
    assert _q(fa, S(1, 1, 1 << 19, 128)) == fa.ERR_UNSUPPORTED     # N beyond the exact-sum range
    assert _q(fa, S(1, 1, (1 << 18) + 1, 128)) == fa.ERR_UNSUPPORTED
    assert _q(fa, S(1, 1, 128, 128), flags=8) == fa.ERR_INVALID_ARG
    assert _q(fa, S(1, 1, 128, 128), ws=None) == fa.ERR_WORKSPACE
    assert _q(fa, S(1, 1, 128, 128), wsb=16) == fa.ERR_WORKSPACE
    assert _q(fa, S(1, 1, 128, 128), ws=ctypes.c_void_p(258)) == fa.ERR_WORKSPACE
    assert _q(fa, S(1, 1, 128, 128), ptr=ctypes.c_void_p(4100)) == fa.ERR_INVALID_ARG  # misaligned


def test_forward_validation_before_launch(fa):
    S = fa.Shape
    p = ctypes.c_void_p(4096)
    f = fa.lib.fp4attn_forward
    assert f(p, p, p, p, None, None, p, S(1, 1, 128, 96), 0.0, p, None, p, 1 << 20, None) == fa.ERR_UNSUPPORTED
    # the BF16-QK attention and the training backward take 128 channels only
    assert fa.lib.fp4attn_forward_bf16qk(p, p, p, S(1, 1, 128, 64), 0.0, p, None, p, 1 << 20, None) \
        == fa.ERR_UNSUPPORTED
    assert f(p, p, p, p, None, None, p, S(1, 1, 128, 128), 0.0, p, None, None, 0, None) == fa.ERR_WORKSPACE
    assert f(None, p, p, p, None, None, p, S(1, 1, 128, 128), 0.0, p, None, p, 1 << 20, None) == fa.ERR_INVALID_ARG
    assert f(p, p, p, p, None, None, p, S(1, 1, 128, 128), float("nan"), p, None, p, 1 << 20, None) \
        == fa.ERR_INVALID_ARG
    assert f(p, p, p, p, None, None, p, S(1, 1, 128, 128), 0.0, p, ctypes.c_void_p(4098), p, 1 << 20, None) \
        == fa.ERR_INVALID_ARG


def test_probe_validation(fa):
    assert fa.lib.fp4attn_probe_qk_tile(None, None, None, None, None, None) == fa.ERR_INVALID_ARG
    assert fa.lib.fp4attn_probe_wait_timeout(None, 1000, None) == fa.ERR_INVALID_ARG
    # the tensor-core rate probe: mode, repetition count and pointers are
    # checked before any CUDA call
    word = ctypes.c_int64(0)
    status = ctypes.c_int32(0)
    p64, p32 = ctypes.cast(ctypes.pointer(word), ctypes.c_void_p), ctypes.cast(ctypes.pointer(status), ctypes.c_void_p)
    assert fa.lib.fp4attn_probe_mma_rate(2, 10, p64, p32, None) == fa.ERR_INVALID_ARG
    assert fa.lib.fp4attn_probe_mma_rate(0, 0, p64, p32, None) == fa.ERR_INVALID_ARG
    assert fa.lib.fp4attn_probe_mma_rate(1, 1000001, p64, p32, None) == fa.ERR_INVALID_ARG
    assert fa.lib.fp4attn_probe_mma_rate(0, 10, None, p32, None) == fa.ERR_INVALID_ARG
    assert fa.lib.fp4attn_probe_mma_rate(0, 10, p64, None, None) == fa.ERR_INVALID_ARG
    assert fa.lib.fp4attn_encode_f32(None, 5, None, None, None) == fa.ERR_INVALID_ARG


def test_strided_and_dynamic_validation_before_launch(fa):
    """The strided entry points reject bad strides (not a positive multiple of 8
    elements, or 2^39 and above) and the dynamic scale without its outputs."""
    S, St = fa.Shape, fa.Strides
    p = ctypes.c_void_p(4096)
    ws = ctypes.c_void_p(256)
    shape = S(2, 3, 128, 128)
    good = St(3 * 128 * 128, 128 * 128, 128)

    def qex(qs, ks=good, flags=0, g=p):
        return fa.lib.fp4attn_quantize_qk_ex(p, qs, p, ks, shape, g, g, flags, p, p, p, p, None, ws, 1 << 20, None)

    for bad in (St(3 * 128 * 128, 128 * 128, 100), St(0, 128 * 128, 128), St(-8, 128 * 128, 128),
                St(3 * 128 * 128, 1 << 39, 128)):
        assert qex(bad) == fa.ERR_INVALID_ARG
        assert qex(good, ks=bad) == fa.ERR_INVALID_ARG
    assert qex(good, flags=fa.DYNAMIC_GSCALE, g=None) == fa.ERR_INVALID_ARG
    assert qex(good, flags=8) == fa.ERR_INVALID_ARG
    # the plain entry point takes its scales as inputs: no dynamic scale there
    assert _q(fa, S(1, 1, 128, 128), flags=fa.DYNAMIC_GSCALE) == fa.ERR_INVALID_ARG
    bad = St(3 * 128 * 128, 128 * 128, 12)
    fex = fa.lib.fp4attn_forward_ex
    assert fex(p, p, p, p, None, None, p, bad, shape, 0.0, p, good, None, p, 1 << 20, None) == fa.ERR_INVALID_ARG
    assert fex(p, p, p, p, None, None, p, good, shape, 0.0, p, bad, None, p, 1 << 20, None) == fa.ERR_INVALID_ARG
    bex = fa.lib.fp4attn_forward_bf16qk_ex
    for i in range(4):
        st = [good] * 4
        st[i] = bad
        assert bex(p, st[0], p, st[1], p, st[2], shape, 0.0, p, st[3], None, p, 1 << 20, None) == fa.ERR_INVALID_ARG


def test_backward_validation_before_launch(fa):
    S = fa.Shape
    p = ctypes.c_void_p(4096)
    f = fa.lib.fp4attn_backward
    shape = S(1, 2, 128, 128)
    wsb = fa.fp4attn_backward_workspace_bytes(1, 2, 128)
    assert wsb >= 256 + 2 * 128 * 4 + 2 * 128 * 4 + 2 * 128 * 128 * 4 + 2 * 2 * 128 * 128 * 2

    def b(codes=p, g=None, lse=p, dk=p, flags=0, scale=0.0, sh=shape, ws=wsb):
        return f(codes, p, p, p, g, None, p, p, p, lse, sh, scale, flags, p, dk, p, p, ws, None)

    assert b(sh=S(1, 2, 128, 64)) == fa.ERR_UNSUPPORTED
    assert b(ws=wsb - 16) == fa.ERR_WORKSPACE
    assert b(flags=8) == fa.ERR_INVALID_ARG
    assert b(scale=float("nan")) == fa.ERR_INVALID_ARG
    assert b(lse=None) == fa.ERR_INVALID_ARG
    assert b(codes=None) == fa.ERR_INVALID_ARG
    assert b(dk=ctypes.c_void_p(4104)) == fa.ERR_INVALID_ARG
    assert b(g=ctypes.c_void_p(4098)) == fa.ERR_INVALID_ARG
    d = fa.lib.fp4attn_dequant_bf16
    assert d(p, ctypes.c_void_p(4100), None, shape, p, None) == fa.ERR_INVALID_ARG
