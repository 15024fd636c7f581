"""The C-ABI library loads and exports every entry point of include/lightning_attn.h,
and its host-side argument validation rejects bad calls before any launch (CPU only).
"""
import ctypes
import os
import re

import pytest

from long_context_fwd_b200 import build, ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lightning_attn.h")

LA_ERR_NULL, LA_ERR_SHAPE, LA_ERR_ALIGN, LA_ERR_UNSUPPORTED = 1, 2, 3, 4


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(lightning_attn_\w+)\s*\(", text, flags=re.M)


@pytest.fixture(scope="module")
def lib():
    build.build()
    return ops.lib()


def test_header_lists_entry_points():
    names = header_functions()
    assert "lightning_attn_fwd" in names and "lightning_attn_decode" in names
    assert len(names) == len(set(names))


def test_library_exports_every_header_symbol(lib):
    for name in header_functions():
        assert hasattr(lib, name), name
        assert name in ops.SIGNATURES, f"binding lacks {name}"


def test_status_strings(lib):
    for code in range(8):
        s = ops.status_string(code)
        assert s.startswith("LA_")
    assert "unknown" in ops.status_string(99)


FAKE = 0x10000  # 16-byte aligned, never dereferenced: every call below fails validation first


def test_fwd_validation(lib):
    f = lib.lightning_attn_fwd
    assert f(None, FAKE, FAKE, FAKE, FAKE, 1, 1, 8, 128, 128, None) == LA_ERR_NULL
    assert f(FAKE, FAKE, FAKE, FAKE, None, 1, 1, 8, 128, 128, None) == LA_ERR_NULL
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 1, 8, 128, 128, None) == LA_ERR_SHAPE
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 0, 128, 128, None) == LA_ERR_SHAPE
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 1, -3, 8, 128, 128, None) == LA_ERR_SHAPE
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 8, 96, 128, None) == LA_ERR_UNSUPPORTED
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 8, 128, 96, None) == LA_ERR_UNSUPPORTED
    assert f(FAKE + 8, FAKE, FAKE, FAKE, FAKE, 1, 1, 8, 128, 128, None) == LA_ERR_ALIGN
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE + 4, 1, 1, 8, 128, 128, None) == LA_ERR_ALIGN
    assert f(FAKE, FAKE, FAKE, FAKE + 2, FAKE, 1, 1, 8, 128, 128, None) == LA_ERR_ALIGN
    big = 1 << 30
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, big, big, big, 128, 128, None) == LA_ERR_SHAPE
    g = lib.lightning_attn_fwd_ex
    assert g(FAKE, FAKE, FAKE, FAKE, None, None, FAKE, 1, 1, 8, 128, 128, 100, None) == LA_ERR_SHAPE
    assert g(FAKE, FAKE, FAKE, FAKE, FAKE + 8, None, FAKE, 1, 1, 8, 128, 128, 0, None) == LA_ERR_ALIGN
    assert g(FAKE, FAKE, FAKE, FAKE, None, FAKE + 8, FAKE, 1, 1, 8, 128, 128, 0, None) == LA_ERR_ALIGN


def test_fwd_f32_validation(lib):
    f = lib.lightning_attn_fwd_f32
    assert f(FAKE, None, FAKE, FAKE, FAKE, 1, 1, 8, 64, 64, None) == LA_ERR_NULL
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 0, 64, 64, None) == LA_ERR_SHAPE
    assert f(FAKE, FAKE, FAKE + 4, FAKE, FAKE, 1, 1, 8, 64, 64, None) == LA_ERR_ALIGN
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 8, 32, 64, None) == LA_ERR_UNSUPPORTED


def test_decode_validation(lib):
    f = lib.lightning_attn_decode
    assert f(FAKE, FAKE, FAKE, None, FAKE, FAKE, 1, 1, 128, 128, None) == LA_ERR_NULL
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 1, 128, 128, None) == LA_ERR_SHAPE
    assert f(FAKE, FAKE, FAKE, FAKE + 8, FAKE, FAKE, 1, 1, 128, 128, None) == LA_ERR_ALIGN
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 256, None) == LA_ERR_UNSUPPORTED


def test_device_status_null(lib):
    assert lib.lightning_attn_device_status(None, 0) == LA_ERR_NULL


def test_binding_rejects_cpu_tensors():
    import torch
    x = torch.zeros(1, 1, 4, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        ops.fwd(x, x, x, torch.zeros(1))


def test_binding_runs_each_entry_on_its_tensors_device():
    # every entry point is wrapped so it launches on the device of its tensors
    # and refuses tensors spread over devices (checked with real devices on GPU
    # boxes; here the wrapper's pass-through for non-CUDA tensors)
    for name in ("fwd", "fwd_strided", "fwd_anticausal", "fwd_fused", "fwd_fused_ex", "bwd",
                 "fwd_noalloc", "fwd_f32", "decode", "decode_fused", "state", "state_combine",
                 "fault_test_scan_stall"):
        fn = getattr(ops, name)
        assert getattr(fn, "__wrapped__", None) is not None, name
    import torch
    x = torch.zeros((1, 1, 4, 64))
    with pytest.raises(ValueError, match="CUDA tensor"):
        ops.fwd_f32(x, x, x, torch.zeros(1))


def test_fault_hook_validation(lib):
    f = lib.lightning_attn_fault_test_scan_stall
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 1024, 0, 100, None) == LA_ERR_SHAPE
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 256, 256, 100, None) == LA_ERR_SHAPE
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 1024, 256, 0, None) == LA_ERR_SHAPE
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 1024, 256, 20000, None) == LA_ERR_SHAPE


def test_noalloc_rejects_oversized_scratch_on_host(lib):
    # 200 sequences in 128-token chunks need 25 MiB of chunk states: rejected
    # before any launch.
    f = lib.lightning_attn_fwd_noalloc
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 200, 1024, 128, 128, 128, None) == 7


def test_strided_validation(lib):
    f = lib.lightning_attn_fwd_strided
    C = ctypes.c_longlong * 3
    ok = C(4 * 64 * 128, 64 * 128, 128)  # token-major-like, all multiples of 16 bytes
    ok_o = C(4 * 64 * 128, 64 * 128, 128)
    args = lambda qs, ks, vs, os: (FAKE, FAKE, FAKE, FAKE, None, None, FAKE, 1, 4, 64, 128, 128,
                                   qs, ks, vs, os, 0, None)
    assert f(*args(None, ok, ok, ok_o)) == LA_ERR_NULL
    bad_t = C(4 * 64 * 128, 64 * 128, 100)  # 200-byte token stride
    assert f(*args(bad_t, ok, ok, ok_o)) == LA_ERR_ALIGN
    neg = C(4 * 64 * 128, -128, 128)
    assert f(*args(ok, neg, ok, ok_o)) == LA_ERR_ALIGN
    bad_o = C(4 * 64 * 128, 64 * 128, 130)  # 520-byte fp32 token stride
    assert f(*args(ok, ok, ok, bad_o)) == LA_ERR_ALIGN
    assert f(FAKE, FAKE, FAKE, FAKE, None, None, FAKE, 1, 4, 64, 32, 128, ok, ok, ok, ok_o, 0,
             None) == LA_ERR_UNSUPPORTED


def test_backward_and_anticausal_validation(lib):
    f = lib.lightning_attn_bwd
    assert f(FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE, 1, 1, 8, 128, 128, None) == LA_ERR_NULL
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, 1, 1, 8, 128, 128, None) == LA_ERR_NULL
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 0, 128, 128, None) == LA_ERR_SHAPE
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 8, 96, 128, None) == LA_ERR_UNSUPPORTED
    # every pointer is checked before the first launch (q and dk, dv are not
    # operands of the dq launch)
    assert f(None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 8, 128, 128, None) == LA_ERR_NULL
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, 1, 1, 8, 128, 128, None) == LA_ERR_NULL
    assert f(FAKE + 8, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 8, 128, 128, None) == LA_ERR_ALIGN
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE + 8, 1, 1, 8, 128, 128, None) == LA_ERR_ALIGN
    g = lib.lightning_attn_fwd_anticausal
    assert g(None, FAKE, FAKE, FAKE, None, None, FAKE, 1, 1, 8, 128, 128, 0, None) == LA_ERR_NULL
    assert g(FAKE, FAKE, FAKE, FAKE, None, None, FAKE, 1, 1, 8, 128, 128, 100, None) == LA_ERR_SHAPE


def test_fused_layer_validation(lib):
    f = lib.lightning_attn_fwd_fused
    ok = (FAKE, FAKE, FAKE, FAKE, FAKE, FAKE)
    assert f(FAKE, FAKE, FAKE, None, FAKE, FAKE, 1e-6, FAKE, 1, 1, 8, 128, 128, None) == LA_ERR_NULL
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, None, 1e-6, FAKE, 1, 1, 8, 128, 128, None) == LA_ERR_NULL
    assert f(FAKE, FAKE, FAKE, FAKE + 8, FAKE, FAKE, 1e-6, FAKE, 1, 1, 8, 128, 128, None) == LA_ERR_ALIGN
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE + 4, 1e-6, FAKE, 1, 1, 8, 128, 128, None) == LA_ERR_ALIGN
    assert f(*ok[:6], -1.0, FAKE, 1, 1, 8, 128, 128, None) == LA_ERR_SHAPE
    assert f(*ok[:6], float("nan"), FAKE, 1, 1, 8, 128, 128, None) == LA_ERR_SHAPE
    assert f(*ok[:6], 1e-6, FAKE, 1, 1, 8, 128, 96, None) == LA_ERR_UNSUPPORTED


def test_cta_limit_setter(lib):
    prev = ops.set_cta_limit(0)
    try:
        assert ops.set_cta_limit(17) == 0
        assert ops.set_cta_limit(0) == 17
        with pytest.raises(ops.LightningAttnError) as err:
            ops.set_cta_limit(-1)
        assert err.value.code == LA_ERR_SHAPE
        assert ops.set_cta_limit(0) == 0  # a rejected call leaves the cap alone
    finally:
        ops.set_cta_limit(prev)


def test_fused_ex_and_decode_fused_validation(lib):
    C3, C2 = ctypes.c_longlong * 3, ctypes.c_longlong * 2
    f = lib.lightning_attn_fwd_fused_ex
    st = C3(64 * 8 * 128, 128, 8 * 128)
    args = lambda eps, strides: (FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, eps, None, None, FAKE, 1, 8,
                                 64, 128, 128, *strides, 0, None)
    assert f(*args(1e-6, (st, st, None, st, st))) == LA_ERR_NULL  # strides: all or none
    assert f(*args(-1.0, (None,) * 5)) == LA_ERR_SHAPE
    bad = C3(64 * 8 * 128, 128, 8 * 128 + 4)  # 8-byte token stride
    assert f(*args(1e-6, (st, st, st, bad, st))) == LA_ERR_ALIGN
    g = lib.lightning_attn_decode_fused
    s2 = C2(8 * 128, 128)
    dargs = lambda eps, strides, D=128: (FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, eps, FAKE, 2, 8,
                                         D, 128, *strides, None)
    assert g(*dargs(1e-6, (s2, None, s2, s2, s2))) == LA_ERR_NULL
    assert g(*dargs(float("nan"), (None,) * 5)) == LA_ERR_SHAPE
    assert g(*dargs(1e-6, (None,) * 5, D=96)) == LA_ERR_UNSUPPORTED
    assert g(*dargs(1e-6, (s2, s2, s2, C2(8 * 128, 132), s2))) == LA_ERR_ALIGN
    assert g(None, *dargs(1e-6, (None,) * 5)[1:]) == LA_ERR_NULL


def test_state_and_combine_validation(lib):
    f = lib.lightning_attn_state
    assert f(FAKE, FAKE, FAKE, None, None, 1, 2, 8, 128, 128, 0, None) == LA_ERR_NULL  # final_state
    assert f(None, FAKE, FAKE, None, FAKE, 1, 2, 8, 128, 128, 0, None) == LA_ERR_NULL
    assert f(FAKE, FAKE, FAKE, None, FAKE, 1, 2, 0, 128, 128, 0, None) == LA_ERR_SHAPE
    assert f(FAKE, FAKE, FAKE, None, FAKE, 1, 2, 8, 128, 128, 100, None) == LA_ERR_SHAPE
    assert f(FAKE, FAKE, FAKE, None, FAKE, 1, 2, 8, 96, 128, 0, None) == LA_ERR_UNSUPPORTED
    assert f(FAKE, FAKE, FAKE, FAKE + 8, FAKE, 1, 2, 8, 128, 128, 0, None) == LA_ERR_ALIGN
    g = lib.lightning_attn_state_combine
    C = ctypes.c_int * 3
    n = C(100, 200, 300)
    assert g(FAKE, 3, None, FAKE, None, FAKE, 1, 2, 128, 128, None) == LA_ERR_NULL
    assert g(None, 3, ctypes.cast(n, ctypes.c_void_p), FAKE, None, FAKE, 1, 2, 128, 128,
             None) == LA_ERR_NULL
    assert g(FAKE, 257, ctypes.cast(n, ctypes.c_void_p), FAKE, None, FAKE, 1, 2, 128, 128,
             None) == LA_ERR_SHAPE
    assert g(FAKE, -1, ctypes.cast(n, ctypes.c_void_p), FAKE, None, FAKE, 1, 2, 128, 128,
             None) == LA_ERR_SHAPE
    bad = C(100, -1, 300)
    assert g(FAKE, 3, ctypes.cast(bad, ctypes.c_void_p), FAKE, None, FAKE, 1, 2, 128, 128,
             None) == LA_ERR_SHAPE
    assert g(FAKE + 4, 3, ctypes.cast(n, ctypes.c_void_p), FAKE, None, FAKE, 1, 2, 128, 128,
             None) == LA_ERR_ALIGN
    assert g(FAKE, 3, ctypes.cast(n, ctypes.c_void_p), FAKE, None, FAKE, 1, 2, 128, 32,
             None) == LA_ERR_UNSUPPORTED
