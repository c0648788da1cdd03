"""C-ABI checks that need no GPU: the library builds, loads and exports every
function declared in include/gdn.h, and host-side validation rejects bad
arguments before anything touches a device (no compute calls here)."""
import ctypes
import os
import re

import pytest
import torch

import gated_delta_rule_142_b200 as gdn
from gated_delta_rule_142_b200 import build as gdn_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER_DIR = os.path.join(ROOT, "include")

OK, NULL, SIZE, UNSUP, MISAL, ALLOC, LAUNCH, TIMEOUT, ALIAS, DEVICE = range(10)


def declared_functions():
    names = set()
    for h in os.listdir(HEADER_DIR):
        if not h.endswith(".h"):
            continue
        text = open(os.path.join(HEADER_DIR, h)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^[A-Za-z_][\w\s\*]*?\b(gdn_\w+)\s*\(", text, flags=re.M):
            names.add(m.group(1))
    return names


@pytest.fixture(scope="module")
def lib():
    gdn_build.build()
    return gdn.load()


def test_header_declares_the_entry_points():
    names = declared_functions()
    assert {"gdn_forward", "gdn_decode_step", "gdn_status_string", "gdn_version"} <= names


def test_library_exports_every_declared_function(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert getattr(lib, name) is not None
    assert set(gdn.EXPORTS) <= declared_functions()


def test_status_strings(lib):
    for s in range(10):
        assert gdn.status_string(s)
    assert gdn.status_string(0) == "ok"
    assert "unknown" in gdn.status_string(12345)
    assert lib.gdn_version() >= 100


# Fake, never dereferenced addresses: every call below is rejected by the host-side
# validation before any device or memory access.
A = 0x10000000


def fwd(lib, q=A, k=A + 0x1000000, v=A + 0x2000000, la=A + 0x3000000, be=A + 0x4000000, S0=None,
        out=A + 0x5000000, Sf=None, B=1, T=8, H=2, dk=16, dv=16, chunk=16, dtype=0):
    P = lambda x: None if x is None else ctypes.c_void_p(x)  # noqa: E731
    return lib.gdn_forward(P(q), P(k), P(v), P(la), P(be), P(S0), P(out), P(Sf), B, T, H, dk, dv, chunk, None, dtype)


def dec(lib, q=A, k=A + 0x1000000, v=A + 0x2000000, la=A + 0x3000000, be=A + 0x4000000, S=A + 0x6000000,
        out=A + 0x5000000, B=2, H=2, dk=16, dv=16, dtype=1):
    P = lambda x: None if x is None else ctypes.c_void_p(x)  # noqa: E731
    return lib.gdn_decode_step(P(q), P(k), P(v), P(la), P(be), P(S), P(out), B, H, dk, dv, None, dtype)


def test_forward_rejects_bad_arguments(lib):
    assert fwd(lib, dtype=7) == UNSUP
    assert fwd(lib, B=-1) == SIZE
    assert fwd(lib, T=-5) == SIZE
    assert fwd(lib, dk=48) == UNSUP
    assert fwd(lib, dv=256) == UNSUP
    assert fwd(lib, chunk=128) == UNSUP
    assert fwd(lib, chunk=0) == UNSUP
    assert fwd(lib, q=None) == NULL
    assert fwd(lib, out=None) == NULL
    assert fwd(lib, be=None) == NULL
    assert fwd(lib, q=A + 8) == MISAL
    assert fwd(lib, S0=A + 0x7000004) == MISAL
    assert fwd(lib, la=A + 0x3000002) == MISAL
    assert fwd(lib, la=A + 0x3000004, B=0) == OK
    assert fwd(lib, B=1 << 40, T=1 << 40) == SIZE
    # out overlapping an input, S_final partially overlapping S0
    assert fwd(lib, out=A + 0x2000000) == ALIAS
    assert fwd(lib, S0=A + 0x7000000, Sf=A + 0x7000010) == ALIAS
    assert fwd(lib, Sf=A + 0x1000000) == ALIAS


def fwd_varlen(lib, cu=(0, 3, 8), q=A, k=A + 0x1000000, v=A + 0x2000000, la=A + 0x3000000, be=A + 0x4000000,
               S0=None, out=A + 0x5000000, Sf=None, T=8, H=2, dk=16, dv=16, chunk=16, dtype=0):
    P = lambda x: None if x is None else ctypes.c_void_p(x)  # noqa: E731
    arr = (ctypes.c_int64 * len(cu))(*cu) if cu is not None else None
    n = len(cu) - 1 if cu is not None else 1
    return lib.gdn_forward_varlen(P(q), P(k), P(v), P(la), P(be), arr, n, P(S0), P(out), P(Sf), T, H, dk, dv,
                                  chunk, None, dtype)


def test_forward_varlen_rejects_bad_offsets(lib):
    lib.gdn_forward_varlen.argtypes = [ctypes.c_void_p] * 5 + [ctypes.POINTER(ctypes.c_int64), ctypes.c_int64] + \
        [ctypes.c_void_p] * 3 + [ctypes.c_int64] * 5 + [ctypes.c_void_p, ctypes.c_int]
    assert fwd_varlen(lib, cu=(1, 3, 8)) == SIZE   # must start at 0
    assert fwd_varlen(lib, cu=(0, 5, 3)) == SIZE   # decreasing
    assert fwd_varlen(lib, cu=(0, 3, 7)) == SIZE   # must end at T
    assert fwd_varlen(lib, cu=None) == SIZE        # NULL offsets with N > 0
    assert fwd_varlen(lib, dk=24) == UNSUP
    assert fwd_varlen(lib, q=A + 8) == MISAL
    assert fwd_varlen(lib, out=A + 0x2000000) == ALIAS
    assert fwd_varlen(lib, cu=(0,), T=0) == OK      # no sequences
    assert fwd_varlen(lib, H=0) == OK


def test_forward_empty_problems_are_noops(lib):
    assert fwd(lib, B=0) == OK
    assert fwd(lib, H=0, q=None, k=None, v=None, la=None, be=None, out=None) == OK


def test_decode_rejects_bad_arguments(lib):
    assert dec(lib, dtype=2) == UNSUP
    assert dec(lib, dk=8) == UNSUP
    assert dec(lib, H=-1) == SIZE
    assert dec(lib, S=None) == NULL
    assert dec(lib, out=None) == NULL
    assert dec(lib, v=A + 0x2000002) == MISAL
    assert dec(lib, out=A + 0x6000000) == ALIAS
    assert dec(lib, S=A) == ALIAS
    assert dec(lib, B=0) == OK


def test_raw_entry_points_validate_like_the_plain_ones(lib):
    """gdn_forward_raw, gdn_forward_varlen_raw and gdn_decode_step_raw take the same arguments (gate
    logits in place of the gates) and reject the same calls with the same status."""
    P = lambda x: None if x is None else ctypes.c_void_p(x)  # noqa: E731
    vp, i64 = ctypes.c_void_p, ctypes.c_int64
    lib.gdn_forward_raw.argtypes = [vp] * 8 + [i64] * 6 + [vp, ctypes.c_int]
    lib.gdn_decode_step_raw.argtypes = [vp] * 7 + [i64] * 4 + [vp, ctypes.c_int]
    lib.gdn_forward_varlen_raw.argtypes = [vp] * 5 + [ctypes.POINTER(i64), i64] + [vp] * 3 + [i64] * 5 + \
        [vp, ctypes.c_int]
    cases = [dict(dtype=7), dict(B=-1), dict(dk=48), dict(q=None), dict(q=A + 8), dict(la=A + 0x3000002),
             dict(out=A + 0x2000000), dict(Sf=A + 0x1000000), dict(B=0)]
    for kw in cases:
        a = dict(q=A, k=A + 0x1000000, v=A + 0x2000000, la=A + 0x3000000, be=A + 0x4000000, S0=None,
                 out=A + 0x5000000, Sf=None, B=1, T=8, H=2, dk=16, dv=16, chunk=16, dtype=0)
        a.update(kw)
        raw = lib.gdn_forward_raw(P(a["q"]), P(a["k"]), P(a["v"]), P(a["la"]), P(a["be"]), P(a["S0"]), P(a["out"]),
                                  P(a["Sf"]), a["B"], a["T"], a["H"], a["dk"], a["dv"], a["chunk"], None, a["dtype"])
        assert raw == fwd(lib, **a) and raw != OK or kw == dict(B=0), kw
    for kw in (dict(dk=8), dict(S=None), dict(out=A + 0x6000000), dict(B=0)):
        a = dict(q=A, k=A + 0x1000000, v=A + 0x2000000, la=A + 0x3000000, be=A + 0x4000000, S=A + 0x6000000,
                 out=A + 0x5000000, B=2, H=2, dk=16, dv=16, dtype=1)
        a.update(kw)
        raw = lib.gdn_decode_step_raw(P(a["q"]), P(a["k"]), P(a["v"]), P(a["la"]), P(a["be"]), P(a["S"]),
                                      P(a["out"]), a["B"], a["H"], a["dk"], a["dv"], None, a["dtype"])
        assert raw == dec(lib, **a), kw
    for cu in ((1, 3, 8), (0, 5, 3), (0, 3, 7)):
        arr = (ctypes.c_int64 * 3)(*cu)
        assert lib.gdn_forward_varlen_raw(P(A), P(A + 0x1000000), P(A + 0x2000000), P(A + 0x3000000),
                                          P(A + 0x4000000), arr, 2, None, P(A + 0x5000000), None, 8, 2, 16, 16, 16,
                                          None, 0) == SIZE


def bwd(lib, **kw):
    P = lambda x: None if x is None else ctypes.c_void_p(x)  # noqa: E731
    vp, i64 = ctypes.c_void_p, ctypes.c_int64
    lib.gdn_backward.argtypes = [vp] * 14 + [i64] * 6 + [vp, ctypes.c_int]
    a = dict(q=A, k=A + 0x1000000, v=A + 0x2000000, la=A + 0x3000000, be=A + 0x4000000, S0=None,
             go=A + 0x5000000, gSf=None, gq=A + 0x8000000, gk=A + 0x9000000, gv=A + 0xA000000,
             gla=A + 0xB000000, gbe=A + 0xC000000, gS0=None, B=1, T=8, H=2, dk=16, dv=16, chunk=16, dtype=0)
    a.update(kw)
    return lib.gdn_backward(*[P(a[n]) for n in ("q", "k", "v", "la", "be", "S0", "go", "gSf", "gq", "gk", "gv",
                                                 "gla", "gbe", "gS0")],
                            a["B"], a["T"], a["H"], a["dk"], a["dv"], a["chunk"], None, a["dtype"])


def test_backward_rejects_bad_arguments(lib):
    assert bwd(lib, dtype=5) == UNSUP
    assert bwd(lib, dk=24) == UNSUP
    assert bwd(lib, chunk=128) == UNSUP
    assert bwd(lib, T=-1) == SIZE
    assert bwd(lib, go=None) == NULL
    assert bwd(lib, gq=None) == NULL
    assert bwd(lib, gbe=None) == NULL
    assert bwd(lib, gk=A + 0x9000008) == MISAL
    assert bwd(lib, gla=A + 0xB000002) == MISAL
    assert bwd(lib, gq=A) == ALIAS                  # an output over an input
    assert bwd(lib, gk=A + 0x8000000) == ALIAS      # two outputs over each other
    assert bwd(lib, gS0=A + 0x5000000) == ALIAS     # dS0 over grad_out
    assert bwd(lib, B=0) == OK


def test_grouped_entry_points_reject_bad_head_counts(lib):
    P = lambda x: None if x is None else ctypes.c_void_p(x)  # noqa: E731
    vp, i64 = ctypes.c_void_p, ctypes.c_int64
    lib.gdn_forward_grouped.argtypes = [vp] * 8 + [i64] * 7 + [vp, ctypes.c_int]
    lib.gdn_decode_step_grouped.argtypes = [vp] * 7 + [i64] * 5 + [vp, ctypes.c_int]

    def fg(Hq, Hkv, **kw):
        a = dict(q=A, k=A + 0x1000000, v=A + 0x2000000, la=A + 0x3000000, be=A + 0x4000000, out=A + 0x5000000,
                 dk=16, dtype=0)
        a.update(kw)
        return lib.gdn_forward_grouped(P(a["q"]), P(a["k"]), P(a["v"]), P(a["la"]), P(a["be"]), None, P(a["out"]),
                                       None, 1, 8, Hq, Hkv, a["dk"], 16, 16, None, a["dtype"])

    def dg(Hq, Hkv):
        return lib.gdn_decode_step_grouped(P(A), P(A + 0x1000000), P(A + 0x2000000), P(A + 0x3000000),
                                           P(A + 0x4000000), P(A + 0x6000000), P(A + 0x5000000), 2, Hq, Hkv, 16, 16,
                                           None, 1)

    assert fg(6, 4) == SIZE      # not a multiple
    assert fg(4, 0) == SIZE      # no key-value heads
    assert fg(-8, 2) == SIZE
    assert fg(8, 2, dk=24) == UNSUP
    assert fg(8, 2, q=None) == NULL
    assert fg(8, 2, out=A + 0x1000000) == ALIAS
    assert fg(0, 0) == OK
    assert dg(6, 4) == SIZE
    assert dg(130, 2) == SIZE    # more than 64 query heads per memory
    assert dg(0, 0) == OK


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_valid_call_without_device_reports_device_error(lib):
    # S0 == S_final (in place) is allowed; with no CUDA device the call stops at the device check.
    assert fwd(lib, S0=A + 0x7000000, Sf=A + 0x7000000) == DEVICE
    assert dec(lib) == DEVICE


def test_binding_fails_loudly_without_library(tmp_path):
    import importlib
    saved = gdn._lib
    try:
        gdn._lib = None
        with pytest.raises(RuntimeError, match="libgdn.so not found"):
            gdn.load(os.path.join(str(tmp_path), "missing.so"))
    finally:
        gdn._lib = saved
    importlib.import_module("gated_delta_rule_142_b200")


def test_binding_validates_shapes_and_dtypes(lib):
    q = torch.zeros(1, 4, 2, 16)
    with pytest.raises(ValueError):
        gdn.forward(q, torch.zeros(1, 4, 2, 8), torch.zeros(1, 4, 2, 16), torch.zeros(1, 4, 2), torch.zeros(1, 4, 2))
    with pytest.raises(TypeError):
        gdn.forward(q.double(), q.double(), q.double(), torch.zeros(1, 4, 2), torch.zeros(1, 4, 2))
    with pytest.raises(ValueError):
        gdn.forward(q.transpose(1, 2), q, q, torch.zeros(1, 4, 2), torch.zeros(1, 4, 2))


def test_bindings_of_the_wider_entry_points_validate_before_calling(lib):
    """Shape and dtype errors in the raw, grouped, backward and convolution bindings are raised on the
    host, before any library call (so they need no device)."""
    z = torch.zeros
    q = z(1, 4, 8, 16)
    with pytest.raises(ValueError):  # gates with the query-head count instead of the key-value one
        gdn.forward_grouped(q, z(1, 4, 2, 16), z(1, 4, 2, 16), z(1, 4, 8), z(1, 4, 8))
    with pytest.raises(ValueError):  # S0 per query head
        gdn.forward_grouped(q, z(1, 4, 2, 16), z(1, 4, 2, 16), z(1, 4, 2), z(1, 4, 2), S0=z(1, 8, 16, 16))
    with pytest.raises(ValueError):
        gdn.decode_step_grouped(z(2, 8, 16), z(2, 2, 16), z(2, 2, 16), z(2, 2), z(2, 2), z(2, 8, 16, 16))
    with pytest.raises(ValueError):
        gdn.forward_raw(q, z(1, 4, 8, 8), z(1, 4, 8, 16), z(1, 4, 8), z(1, 4, 8))
    with pytest.raises(ValueError):  # grad_out shape
        gdn.backward(q, q, q, z(1, 4, 8), z(1, 4, 8), None, z(1, 4, 8, 8))
    with pytest.raises(TypeError):  # grad_out dtype differs from q
        gdn.backward(q, q, q, z(1, 4, 8), z(1, 4, 8), None, q.double())
    with pytest.raises(ValueError):  # weight [C, W] with the wrong C
        gdn.causal_conv(z(1, 4, 32), z(16, 4))
    with pytest.raises(ValueError):  # state [B, W-1, C]
        gdn.causal_conv(z(1, 4, 32), z(32, 4), state_in=z(1, 4, 32))


def test_forward_plan_argument_checks(lib):
    s, n = ctypes.c_int64(-1), ctypes.c_int(-1)
    assert lib.gdn_forward_plan(1, 8, 2, 48, 16, 16, 0, ctypes.byref(s), ctypes.byref(n)) == UNSUP
    assert (s.value, n.value) == (0, 0)
    assert lib.gdn_forward_plan(-1, 8, 2, 16, 16, 16, 0, None, None) == SIZE
    assert lib.gdn_forward_plan(0, 8, 2, 16, 16, 16, 1, ctypes.byref(s), ctypes.byref(n)) == OK
    assert (s.value, n.value) == (0, 0)


def test_head_count_overflow_is_rejected_even_with_no_tokens(lib):
    """B * H overflows int64 while T == 0: both forward entry points refuse the sizes before
    anything else (the token count is zero and would not reveal it)."""
    big = 1 << 40
    assert fwd(lib, B=big, H=big, T=0) == SIZE
    P = lambda x: None if x is None else ctypes.c_void_p(x)  # noqa: E731
    na = lib.gdn_forward_noalloc
    na.argtypes = [ctypes.c_void_p] * 8 + [ctypes.c_int64] * 6 + [ctypes.c_void_p, ctypes.c_int]
    na.restype = ctypes.c_int
    args = [P(A), P(A + 0x1000000), P(A + 0x2000000), P(A + 0x3000000), P(A + 0x4000000), None, P(A + 0x5000000),
            None]
    assert na(*args, big, 0, big, 16, 16, 16, None, 0) == SIZE
    # a token count beyond INT64_MAX / 8 is refused by both, as gdn_forward documents
    assert fwd(lib, B=1 << 31, T=1 << 31, H=2) == SIZE
    assert na(*args, 1 << 31, 1 << 31, 2, 16, 16, 16, None, 0) == SIZE


def test_forward_conv_validates_before_any_device_work(lib):
    """gdn_forward_conv: the convolution width and the usual sizes are checked on the host."""
    P = lambda x: None if x is None else ctypes.c_void_p(x)  # noqa: E731
    fc = lib.gdn_forward_conv

    def call(W=4, B=1, T=8, H=2, d=16, chunk=16, dtype=0, weight=A + 0x7000000):
        return fc(P(A), P(A + 0x1000000), P(A + 0x2000000), P(A + 0x3000000), P(A + 0x4000000), P(weight), None,
                  None, None, P(A + 0x5000000), None, B, T, H, d, d, W, chunk, None, dtype)

    assert call(W=5) == UNSUP
    assert call(W=0) == UNSUP
    assert call(W=-1) == SIZE
    assert call(dtype=7) == UNSUP
    assert call(weight=None) == NULL
    assert call(B=0) == OK
    assert call(weight=A + 0x7000001) == MISAL
