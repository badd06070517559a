"""GPU test of sla2_router_noalloc, the router entry point for callers that
cannot allocate device memory: for example a plugin inside a host framework
that owns every device allocation, or a latency-critical path where
cudaMalloc is not allowed because it can synchronise the device. Its scratch
is a fixed device array inside libsla2.so instead of a caller workspace; it
must reproduce sla2_router (which takes a caller workspace) exactly, on two
calls in a row, and reject shapes whose scratch does not fit the array.

The file is named so that pytest collects it last."""
import ctypes

import pytest
import torch

from block_sparse_linear_router_b200.inputs import make_custom

pytestmark = pytest.mark.gpu

SLA2_ERR_WORKSPACE = 3


@pytest.fixture(scope="module")
def libs():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from block_sparse_linear_router_b200 import build
    build.build()
    from block_sparse_linear_router_b200 import sla2
    lib = sla2.load_library()
    fn = lib.sla2_router_noalloc
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.POINTER(sla2.Desc)] + [ctypes.c_void_p] * 4 + [ctypes.c_float] + [ctypes.c_void_p] * 4
    return sla2, fn


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


@pytest.mark.parametrize("shape", [(1, 1, 2048, 64, 0.1), (1, 2, 2048, 128, 0.05), (2, 3, 640, 64, 0.3)])
def test_noalloc_router_matches_workspace_router_on_two_calls(libs, shape):
    sla2, fn = libs
    B, H, N, d, frac = shape
    inp = make_custom(B, H, N, d, frac, seed=41)
    q, k, wq, wk = (getattr(inp, n).cuda() for n in ("q", "k", "proj_q", "proj_k"))
    ref = sla2.router(q, k, wq, wk, frac)          # caller-provided workspace
    torch.cuda.synchronize()
    nq, nk = N // 128, N // 64
    kk = sla2.topk_count(nk, frac)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        desc = sla2.make_desc(B, H, N, d, 0)       # no workspace
        mask = torch.full((B, H, nq, nk), 7, dtype=torch.uint8, device="cuda")
        idx = torch.full((B, H, nq, kk), -1, dtype=torch.int32, device="cuda")
        cm = torch.full((B, H, d), float("nan"), dtype=torch.float32, device="cuda")
        r = fn(ctypes.byref(desc), _p(q), _p(k), _p(wq), _p(wk), frac, _p(mask), _p(idx), _p(cm), stream)
        assert r == 0, f"call {call}: status {r}"
        torch.cuda.synchronize()
        assert torch.equal(mask, ref["mask"]), f"call {call}: mask differs"
        assert torch.equal(idx, ref["idx"]), f"call {call}: index list differs"
        assert torch.equal(cm, ref["colmean"]), f"call {call}: column mean differs"


def test_noalloc_router_rejects_shapes_beyond_the_array(libs):
    sla2, fn = libs
    t = torch.zeros(64, dtype=torch.float32, device="cuda")
    desc = sla2.make_desc(1, 16, 32768, 128, 0)    # about 29 MB of scratch > 16 MiB
    r = fn(ctypes.byref(desc), _p(t), _p(t), _p(t), _p(t), 0.03, _p(t), _p(t), None, None)
    assert r == SLA2_ERR_WORKSPACE
