"""Host-side checks of the C-ABI library, no GPU needed: it loads, it exports
every function include/moe_q4.h declares, the Python binding wraps them all,
and argument checks reject bad calls before any CUDA call is made."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "moe_q4_cuda_build", os.path.join(ROOT, "quantized_moe_q4_b200", "build.py"))
    build = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(build)
    path = build.build()
    return ctypes.CDLL(path)


def header_functions():
    src = open(os.path.join(ROOT, "include", "moe_q4.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_q4_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_three_core_calls():
    names = header_functions()
    for n in ("moe_q4_quantize_act", "moe_q4_route", "moe_q4_ffn_forward"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in header_functions():
        assert hasattr(lib, name), name


def test_binding_wraps_every_declared_symbol(lib):
    import quantized_moe_q4_b200 as m
    assert sorted(m.EXPORTS) == header_functions()
    for name in header_functions():
        assert callable(getattr(m, name, None)), name


def test_status_strings(lib):
    lib.moe_q4_status_string.restype = ctypes.c_char_p
    assert lib.moe_q4_status_string(0) == b"ok"
    for code in range(-7, 0):
        assert lib.moe_q4_status_string(code) not in (b"", b"unknown status")


class _L(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("hidden", "ffn", "n_experts", "top_k", "has_shared")] + \
               [(n, ctypes.c_void_p) for n in ("w_router", "router_bias", "w_gate", "w_up", "w_down",
                                                "sh_gate", "sh_up", "sh_down")]


FAKE = 0x7F0000000000  # a 256-byte aligned address that is never dereferenced


def make(**kw):
    d = dict(hidden=2048, ffn=512, n_experts=128, top_k=8, has_shared=1, w_router=FAKE, router_bias=None,
             w_gate=FAKE, w_up=FAKE, w_down=FAKE, sh_gate=FAKE, sh_up=FAKE, sh_down=FAKE)
    d.update(kw)
    return _L(**d)


def fwd(lib, L, x=FAKE + 0x1000000, T=4, y=FAKE + 0x2000000, ws=FAKE + 0x3000000, nbytes=1 << 40):
    f = lib.moe_q4_ffn_forward
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                  ctypes.c_size_t, ctypes.c_void_p]
    return f(ctypes.byref(L), x, T, y, ws, nbytes, None)


@pytest.mark.parametrize("kw,code", [
    (dict(top_k=0), -1), (dict(top_k=17, n_experts=32), -1), (dict(top_k=9, n_experts=8), -1),
    (dict(n_experts=0), -1), (dict(n_experts=257), -1), (dict(has_shared=2), -1),
    (dict(w_gate=None), -1), (dict(sh_up=None), -1), (dict(has_shared=0), -1),
    (dict(hidden=2000), -2), (dict(ffn=500), -2), (dict(hidden=0), -2), (dict(ffn=128), -2),
    (dict(hidden=32768), -2), (dict(w_up=FAKE + 8), -3), (dict(sh_down=FAKE + 2), -3),
])
def test_forward_rejects_bad_layers(lib, kw, code):
    assert fwd(lib, make(**kw)) == code


def test_forward_rejects_bad_calls(lib):
    L = make()
    assert fwd(lib, L, T=-1) == -1
    assert fwd(lib, L, T=(1 << 24) + 1) == -1
    assert fwd(lib, L, T=0) == 0                           # no-op, nothing touched
    assert fwd(lib, L, x=None) == -1
    assert fwd(lib, L, y=FAKE + 0x2000004) == -3
    assert fwd(lib, L, ws=FAKE + 0x3000010) == -3
    assert fwd(lib, L, nbytes=1000) == -4
    assert fwd(lib, L, y=FAKE + 0x1000000) == -7             # y == x
    assert fwd(lib, L, y=FAKE + 0x3000000, ws=FAKE + 0x3000000) == -7


def test_workspace_bytes_and_layout(lib):
    L = make()
    lib.moe_q4_ffn_workspace_bytes.restype = ctypes.c_size_t
    lib.moe_q4_ffn_workspace_bytes.argtypes = [ctypes.c_void_p, ctypes.c_int64]
    n1 = lib.moe_q4_ffn_workspace_bytes(ctypes.byref(L), 1)
    n947 = lib.moe_q4_ffn_workspace_bytes(ctypes.byref(L), 947)
    assert 0 < n1 < n947
    assert lib.moe_q4_ffn_workspace_bytes(ctypes.byref(make(top_k=0)), 4) == 0
    offs = (ctypes.c_size_t * 16)()
    lib.moe_q4_workspace_layout.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int]
    assert lib.moe_q4_workspace_layout(ctypes.byref(L), 947, offs, 16) == 0
    o = list(offs)
    assert o[0] == 0 and all(b > a for a, b in zip(o, o[1:])) and all(v % 256 == 0 for v in o)
    assert o[-1] == n947
    T, k, H, F = 947, 8, 2048, 512
    P = T * k
    # hq spans (P + T) slots of F bytes
    assert o[14] - o[13] >= (P + T) * F
    # dh: one binary16 scale per 32 values of hq
    assert o[15] - o[14] >= 2 * (P + T) * (F // 32)


def test_other_entry_points_reject_bad_args(lib):
    q = lib.moe_q4_quantize_act
    q.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_void_p]
    assert q(FAKE, 4, 48, FAKE, FAKE, None, None) == -1      # H not a multiple of 32
    assert q(FAKE + 4, 4, 64, FAKE, FAKE, None, None) == -3
    assert q(FAKE, 0, 64, None, None, None, None) == 0
    r = lib.moe_q4_route
    r.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_void_p]
    L = make()
    assert r(ctypes.byref(L), FAKE, 4, FAKE, FAKE, None, None) == -1
    b = lib.moe_q4_block_dots
    b.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p]
    assert b(FAKE, FAKE, 7, FAKE, None) == -1                # n not a multiple of 8
    assert b(FAKE + 2, FAKE, 8, FAKE, None) == -3
    rc = lib.moe_q4_rescale_ceiling
    rc.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    n = ctypes.c_int64(0)
    assert rc(0, 0, FAKE, ctypes.byref(n), None) == -1           # no stages
    assert rc(1, (1 << 20) + 1, FAKE, ctypes.byref(n), None) == -1
    assert rc(0, 8, None, ctypes.byref(n), None) == -1           # no sink
    assert rc(0, 8, FAKE, None, None) == -1                      # no element count
    assert rc(1, 8, FAKE + 2, ctypes.byref(n), None) == -3       # sink not 4-byte aligned
    d = lib.moe_q4_ffn_forward_debug
    d.argtypes = [ctypes.c_void_p] * 2 + [ctypes.c_int64] + [ctypes.c_void_p] * 2 + [ctypes.c_size_t] + \
                 [ctypes.c_void_p] * 2

    class _D(ctypes.Structure):
        _fields_ = [("h_out", ctypes.c_void_p), ("path", ctypes.c_int32), ("ev_start", ctypes.c_void_p),
                    ("ev_stop", ctypes.c_void_p), ("force_spin_timeout", ctypes.c_int32),
                    ("block_dots_out", ctypes.c_void_p), ("block_dots_down", ctypes.c_int32),
                    ("block_dots_group", ctypes.c_int32), ("block_dots_rb", ctypes.c_int32),
                    ("decode_kernel_ns", ctypes.c_void_p)]
    dbg = _D(None, 9, None, None, 0, None, 0, 0, 0, None)
    assert d(ctypes.byref(L), FAKE, 4, FAKE + 0x1000000, FAKE + 0x2000000, 1 << 40, ctypes.byref(dbg), None) == -1
    # block-dot capture of a group that does not exist (E = 128 routed + the shared group 128)
    dbg = _D(None, 0, None, None, 0, FAKE + 0x4000000, 0, 129, 0, None)
    assert d(ctypes.byref(L), FAKE, 4, FAKE + 0x1000000, FAKE + 0x2000000, 1 << 40, ctypes.byref(dbg), None) == -1
    dbg = _D(None, 0, None, None, 0, FAKE + 0x4000002, 0, 3, 0, None)     # misaligned capture buffer
    assert d(ctypes.byref(L), FAKE, 4, FAKE + 0x1000000, FAKE + 0x2000000, 1 << 40, ctypes.byref(dbg), None) == -1


def test_stack_entry_points_reject_bad_args(lib):
    n = lib.moe_q4_residual_rmsnorm
    n.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float,
                  ctypes.c_void_p, ctypes.c_void_p]
    X, Y, XN = FAKE, FAKE + 0x1000000, FAKE + 0x2000000
    assert n(X, Y, 4, 2000, 1e-6, XN, None) == -1            # H not a multiple of 256
    assert n(X, Y, 4, 2048, -1.0, XN, None) == -1            # negative eps
    assert n(X, Y, 4, 2048, float("nan"), XN, None) == -1
    assert n(None, Y, 4, 2048, 1e-6, XN, None) == -1
    assert n(X + 4, Y, 4, 2048, 1e-6, XN, None) == -3
    assert n(X, Y, 4, 2048, 1e-6, X + 4096, None) == -7      # xn overlaps x
    assert n(X, X, 4, 2048, 1e-6, XN, None) == -7            # y is x
    assert n(X, None, 0, 2048, 1e-6, None, None) == 0        # T == 0: no-op
    wb = lib.moe_q4_stack_workspace_bytes
    wb.argtypes, wb.restype = [ctypes.c_void_p, ctypes.c_int64], ctypes.c_size_t
    lib.moe_q4_ffn_workspace_bytes.argtypes = [ctypes.c_void_p, ctypes.c_int64]
    lib.moe_q4_ffn_workspace_bytes.restype = ctypes.c_size_t
    L = make()
    assert wb(ctypes.byref(L), 64) == lib.moe_q4_ffn_workspace_bytes(ctypes.byref(L), 64) + 2 * 64 * 2048 * 4
    assert wb(ctypes.byref(make(top_k=0)), 64) == 0
    f = lib.moe_q4_stack_forward
    f.argtypes = [ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p, ctypes.c_int64, ctypes.c_float,
                  ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
    arr = (_L * 3)(make(), make(), make())
    WS = FAKE + 0x10000000
    assert f(arr, 0, X, 4, 1e-6, WS, 1 << 40, None) == -1      # no layers
    assert f(None, 3, X, 4, 1e-6, WS, 1 << 40, None) == -1
    bad = (_L * 3)(make(), make(ffn=768), make())
    assert f(bad, 3, X, 4, 1e-6, WS, 1 << 40, None) == -2      # layers differ in shape
    bad = (_L * 2)(make(), make(top_k=0))
    assert f(bad, 2, X, 4, 1e-6, WS, 1 << 40, None) == -1      # an invalid layer
    assert f(arr, 3, X, 4, 1e-6, WS, 1000, None) == -4
    assert f(arr, 3, X + 8, 4, 1e-6, WS, 1 << 40, None) == -3
    assert f(arr, 3, WS, 4, 1e-6, WS, 1 << 40, None) == -7     # x inside the workspace
    assert f(arr, 3, X, 0, 1e-6, WS, 1 << 40, None) == 0       # T == 0: no-op


def test_gemv_rejects_bad_args(lib):
    wb = lib.moe_q4_gemv_workspace_bytes
    wb.argtypes, wb.restype = [ctypes.c_int64, ctypes.c_int32], ctypes.c_size_t
    assert wb(1, 2048) == 256 + 2048 + 256 and wb(9, 2048) == 0 and wb(1, 2000) == 0
    g = lib.moe_q4_gemv
    g.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
    Wp, X, Y, WS = FAKE, FAKE + 0x1000000, FAKE + 0x2000000, FAKE + 0x3000000
    assert g(Wp, 1000, 2048, X, 9, Y, WS, 1 << 20, None) == -1      # T > 8
    assert g(Wp, 0, 2048, X, 1, Y, WS, 1 << 20, None) == -1         # no rows
    assert g(Wp, 1000, 2000, X, 1, Y, WS, 1 << 20, None) == -2      # H not a multiple of 256
    assert g(None, 1000, 2048, X, 1, Y, WS, 1 << 20, None) == -1
    assert g(Wp + 8, 1000, 2048, X, 1, Y, WS, 1 << 20, None) == -3
    assert g(Wp, 1000, 2048, X, 1, Y, WS, 100, None) == -4
    assert g(Wp, 1000, 2048, X, 1, X, WS, 1 << 20, None) == -7      # y is x
    assert g(Wp, 1000, 2048, X, 0, Y, WS, 1 << 20, None) == 0       # T == 0: no-op


def test_product_package_does_not_use_the_oracle():
    pkg = os.path.join(ROOT, "quantized_moe_q4_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                src = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in src and "from oracle" not in src, f
                assert "libmoe_q4_oracle" not in src and "moe_q4_oracle" not in src, f


def test_arch_rejection_through_the_device_override(lib):
    """Every entry point refuses a device that is not compute capability
    10.0 with MOE_Q4_ERR_ARCH, before any CUDA call (this host has no GPU,
    so a CUDA call would return MOE_Q4_ERR_CUDA instead) and before anything
    is enqueued; the allocation-free entry checks the device before it looks
    up its scratch."""
    ov = lib.moe_q4_test_override_device
    ov.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32]
    L = make()
    X, Y, WS, ST = FAKE, FAKE + 0x1000000, FAKE + 0x2000000, FAKE + 0x40000000
    for major, minor in ((9, 0), (10, 3), (12, 0), (8, 9)):
        assert ov(1, major, minor) == 0
        try:
            assert fwd(lib, L) == -5
            q = lib.moe_q4_quantize_act
            q.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32] + [ctypes.c_void_p] * 4
            assert q(X, 4, 2048, Y, WS, None, None) == -5
            r = lib.moe_q4_route
            r.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64] + [ctypes.c_void_p] * 4
            assert r(ctypes.byref(L), X, 4, Y, Y + 4096, WS, None) == -5
            h = lib.moe_q4_ffn_forward_host
            h.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                          ctypes.c_size_t, ctypes.c_void_p]
            assert h(ctypes.byref(L), X, 4, Y, WS, 1 << 40, None) == -5
            n = lib.moe_q4_ffn_forward_noalloc
            n.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p]
            assert n(ctypes.byref(L), X, 4, Y, None) == -5
            nr = lib.moe_q4_residual_rmsnorm
            nr.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float,
                           ctypes.c_void_p, ctypes.c_void_p]
            assert nr(X, Y, 4, 2048, 1e-6, WS, None) == -5
            sf = lib.moe_q4_stack_forward
            sf.argtypes = [ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p, ctypes.c_int64, ctypes.c_float,
                           ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
            arr = (_L * 2)(make(), make())
            assert sf(arr, 2, X, 4, 1e-6, WS, 1 << 40, None) == -5
            g = lib.moe_q4_gemv
            g.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p, ctypes.c_int64,
                          ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
            assert g(ST, 1000, 2048, X, 1, Y, WS, 1 << 20, None) == -5
            st = lib.moe_q4_ffn_forward_streamed
            st.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                           ctypes.c_size_t, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
            assert st(ctypes.byref(L), X, 4, Y, WS, 1 << 40, ST, 1 << 40, None) == -5
            b = lib.moe_q4_block_dots
            b.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p]
            assert b(X, Y, 8, WS, None) == -5
            # argument errors still come first
            assert fwd(lib, make(top_k=0)) == -1
        finally:
            ov(0, 0, 0)
    # an override to 10.0 itself is not a rejection: on this GPU-less host the
    # call goes on to the (failing) driver query
    assert ov(1, 10, 0) == 0
    try:
        assert fwd(lib, L) == -6
    finally:
        ov(0, 0, 0)
