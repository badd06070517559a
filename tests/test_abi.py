"""The C ABI library without a GPU: it loads, exports every function the
headers declare, and rejects bad arguments on the host before any CUDA call."""
import ctypes
import os
import re

import pytest

from block_sparse_linear_router_b200 import build as B
from block_sparse_linear_router_b200 import sla2
from oracle import sla2_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return sla2.load_library()


def _declared():
    names = []
    for h in ("sla2.h", "sla2_test.h"):
        txt = open(os.path.join(ROOT, "include", h)).read()
        txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
        names += re.findall(r"\b(sla2_\w+)\s*\(", txt)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert {"sla2_forward", "sla2_router", "sla2_linear_state", "sla2_workspace_size", "sla2_topk_count",
            "sla2_status_string", "sla2_selftest_timeout"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    for code in range(6):
        assert lib.sla2_status_string(code)
    assert lib.sla2_status_string(99) == b"unknown status"


@pytest.mark.parametrize("nk,frac", [(32, 0.1), (512, 0.03), (512, 0.05), (512, 0.1), (512, 0.2), (512, 1.0),
                                     (1184, 0.05), (256, 0.1), (16, 0.001), (7, 0.5), (1, 1.0)])
def test_topk_count_matches_oracle(lib, nk, frac):
    assert lib.sla2_topk_count(nk, frac) == O.topk_count(nk, frac)


def test_topk_count_rejects_bad_fraction(lib):
    for f in (0.0, -0.1, 1.0001, float("nan")):
        assert lib.sla2_topk_count(32, f) == 0


def _desc(**kw):
    d = dict(B=1, H=2, N=1024, d=64, quantize=1, out_dtype=0)
    d.update(kw)
    return sla2.Desc(**d)


def test_workspace_size_valid_and_invalid(lib):
    ok = lib.sla2_workspace_size(ctypes.byref(_desc()), 0.1)
    assert ok > 0 and ok % 256 == 0
    assert lib.sla2_workspace_size(ctypes.byref(_desc(N=1000)), 0.1) == 0       # N % 128
    assert lib.sla2_workspace_size(ctypes.byref(_desc(d=96)), 0.1) == 0         # d
    assert lib.sla2_workspace_size(ctypes.byref(_desc()), 0.0) == 0             # frac
    assert lib.sla2_workspace_size(ctypes.byref(_desc(quantize=2)), 0.1) == 0
    assert lib.sla2_workspace_size(None, 0.1) == 0
    # the unquantised variant stores a bf16 V^T instead of INT8 Q/K and e4m3 V
    assert lib.sla2_workspace_size(ctypes.byref(_desc(quantize=0)), 0.1) != ok


def _fake(n=1 << 20):
    # a 16-byte aligned host address used only as a non-NULL token: the checks
    # below fail before anything would dereference it
    buf = ctypes.create_string_buffer(n + 256)
    return buf, (ctypes.addressof(buf) + 255) & ~255


def test_forward_argument_errors_are_host_side(lib):
    keep, p = _fake()
    d = _desc()
    args = [ctypes.c_void_p(p)] * 6
    assert lib.sla2_forward(ctypes.byref(_desc(N=1000)), *args, 0.1, ctypes.c_void_p(p), None) == 2
    assert lib.sla2_forward(ctypes.byref(_desc(d=32)), *args, 0.1, ctypes.c_void_p(p), None) == 2
    assert lib.sla2_forward(ctypes.byref(d), *args, 1.5, ctypes.c_void_p(p), None) == 1
    assert lib.sla2_forward(ctypes.byref(d), None, *args[1:], 0.1, ctypes.c_void_p(p), None) == 1
    mis = [ctypes.c_void_p(p + 4)] + args[1:]
    assert lib.sla2_forward(ctypes.byref(d), *mis, 0.1, ctypes.c_void_p(p), None) == 1
    # out aliasing q
    assert lib.sla2_forward(ctypes.byref(d), *args, 0.1, ctypes.c_void_p(p), None) == 1
    # missing / too small / misaligned workspace
    o = ctypes.c_void_p(p + 4096)
    assert lib.sla2_forward(ctypes.byref(d), *args, 0.1, o, None) == 3
    d.workspace, d.workspace_bytes = p, 1024
    assert lib.sla2_forward(ctypes.byref(d), *args, 0.1, o, None) == 3
    d.workspace, d.workspace_bytes = p + 16, 1 << 40
    assert lib.sla2_forward(ctypes.byref(d), *args, 0.1, o, None) == 3


def test_router_and_linear_state_argument_errors(lib):
    keep, p = _fake()
    v = ctypes.c_void_p(p)
    assert lib.sla2_router(ctypes.byref(_desc()), v, v, v, v, 0.0, v, v, None, None) == 1
    assert lib.sla2_router(ctypes.byref(_desc()), v, None, v, v, 0.1, v, v, None, None) == 1
    assert lib.sla2_router(ctypes.byref(_desc()), v, v, v, v, 0.1, v, v, None, None) == 3
    assert lib.sla2_linear_state(ctypes.byref(_desc(N=96)), v, v, v, v, v, v, v, None) == 2
    assert lib.sla2_linear_state(ctypes.byref(_desc()), v, v, None, v, v, v, v, None) == 1
    assert lib.sla2_linear_state(ctypes.byref(_desc()), v, v, v, v, v, v, v, None) == 3


def test_router_soft_argument_errors(lib):
    keep, p = _fake()
    v = ctypes.c_void_p(p)
    for tau in (0.0, -0.1, float("inf"), float("nan")):
        assert lib.sla2_router_soft(ctypes.byref(_desc()), v, v, v, v, 0.1, tau, v, None, None) == 1
    assert lib.sla2_router_soft(ctypes.byref(_desc()), v, v, v, v, 0.0, 0.1, v, None, None) == 1     # frac
    assert lib.sla2_router_soft(ctypes.byref(_desc()), v, v, v, v, 0.1, 0.1, None, None, None) == 1  # no output
    assert lib.sla2_router_soft(ctypes.byref(_desc(d=96)), v, v, v, v, 0.1, 0.1, v, None, None) == 2
    assert lib.sla2_router_soft(ctypes.byref(_desc()), v, v, v, v, 0.1, 0.1, v, None, None) == 3      # workspace


def test_selftest_rejects_bad_arguments(lib):
    lib.sla2_selftest_timeout.restype = ctypes.c_int
    lib.sla2_selftest_timeout.argtypes = [ctypes.c_void_p, ctypes.c_ulonglong, ctypes.c_void_p]
    keep, p = _fake()
    assert lib.sla2_selftest_timeout(None, 1000, None) == 1
    assert lib.sla2_selftest_timeout(ctypes.c_void_p(p), 0, None) == 1
    assert lib.sla2_selftest_timeout(ctypes.c_void_p(p), 20_000_000_000, None) == 1


def test_binding_refuses_cpu_tensors():
    import torch
    q = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16)
    with pytest.raises((ValueError, RuntimeError)):
        sla2.forward(q, q, q, torch.zeros(1, 64, 64), torch.zeros(1, 64, 64), torch.zeros(1, 1), 0.5)


def test_head_range_entry_point_rejects_bad_ranges_on_the_host(lib):
    buf, p = _fake()
    ws, pws = _fake()
    d = _desc(H=4)
    n = lib.sla2_workspace_size_heads(ctypes.byref(d), 2, 0.1)
    assert 0 < n < lib.sla2_workspace_size(ctypes.byref(d), 0.1)
    for hc in (0, -1, 5):
        assert lib.sla2_workspace_size_heads(ctypes.byref(d), hc, 0.1) == 0
    d.workspace, d.workspace_bytes = pws, 1 << 20
    args = [ctypes.c_void_p(p)] * 6 + [ctypes.c_float(0.1), ctypes.c_void_p(p + 4096), None]
    for hb, hc in ((-1, 2), (3, 2), (0, 0), (4, 1)):
        assert lib.sla2_forward_heads(ctypes.byref(d), hb, hc, *args) == 1      # invalid argument
    d.dbg_scores = p                                                             # debug exports refused
    assert lib.sla2_forward_heads(ctypes.byref(d), 0, 2, *args) == 1


def test_host_buffer_entry_point_rejects_bad_arguments_on_the_host(lib):
    buf, p = _fake()
    ws, pws = _fake()
    d = _desc(H=4)
    n2 = lib.sla2_forward_host_workspace_size(ctypes.byref(d), 2, 0.1)
    n4 = lib.sla2_forward_host_workspace_size(ctypes.byref(d), 4, 0.1)
    # the group's forward workspace plus two slots of group inputs and outputs
    slot2 = 2 * 2 * (3 * 1024 * 64 * 2 + 1024 * 64 * 2)
    assert n2 > lib.sla2_workspace_size_heads(ctypes.byref(d), 2, 0.1) + slot2
    assert n4 > n2
    for hpg in (0, -1, 5):
        assert lib.sla2_forward_host_workspace_size(ctypes.byref(d), hpg, 0.1) == 0
    args = [ctypes.c_void_p(p)] * 6 + [ctypes.c_float(0.1), ctypes.c_void_p(p + 4096), None]
    d.workspace, d.workspace_bytes = pws, n2
    for hpg in (0, 5):
        assert lib.sla2_forward_host(ctypes.byref(d), hpg, *args) == 1          # invalid argument
    d.workspace_bytes = n2 - 1
    assert lib.sla2_forward_host(ctypes.byref(d), 2, *args) == 3                 # workspace too small
    d.workspace_bytes = n2
    d.stage_events = p                                                           # per-stage events refused
    assert lib.sla2_forward_host(ctypes.byref(d), 2, *args) == 1
    d.stage_events = None
    bad = [None] + args[1:]
    assert lib.sla2_forward_host(ctypes.byref(d), 2, *bad) == 1


def test_host_binding_refuses_device_tensors_and_wrong_out():
    import torch
    q = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        sla2.forward_host(q, q, q, torch.zeros(1, 64, 64), torch.zeros(1, 64, 64), torch.zeros(1, 1), 0.5,
                          torch.zeros(1, 1, 128, 32, dtype=torch.bfloat16))
