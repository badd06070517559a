"""The polynomial 2^x that the sparse branch's softmax evaluates on the FMA pipe
for a share of its exponentials (device.cuh, exp2_poly_x2): 2^x = 2^j 2^f with
j = rint(x), f in [-1/2, 1/2] (Cody-Waite style range reduction) and a cubic
for 2^f whose coefficients were fitted by the Remez exchange on relative error.

CPU: the coefficients, read from the header, meet the stated bound (relative
error below 7.6e-5 on [-1/2, 1/2], in exact arithmetic and with an fp32
Horner evaluation). GPU: the device function, through the test hook, stays
within 1e-4 of exp2 over the range the softmax feeds it."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _coefficients():
    src = open(os.path.join(ROOT, "block_sparse_linear_router_b200", "csrc", "device.cuh")).read()
    body = src[src.index("uint64_t exp2_poly_x2("):]
    body = body[:body.index("\n}\n")]
    vals = [float(v) for v in re.findall(r"f2_pack\(([-0-9.e]+)f, \1f\)", body)]
    # Horner order in the source: c3, c2, c1, c0 (after the two reduction constants)
    consts = [v for v in vals if 0.0 < v < 2.0]
    assert len(consts) == 4, consts
    c3, c2, c1, c0 = consts
    return c0, c1, c2, c3


def test_cubic_meets_its_relative_error_bound():
    c0, c1, c2, c3 = _coefficients()
    f = np.linspace(-0.5, 0.5, 400001)
    exact = np.exp2(f)
    p64 = ((c3 * f + c2) * f + c1) * f + c0
    assert np.max(np.abs(p64 - exact) / exact) < 7.6e-5
    f32 = f.astype(np.float32)
    p32 = np.float32(c3)
    for c in (c2, c1, c0):
        p32 = (p32 * f32 + np.float32(c)).astype(np.float32)
    ex32 = np.exp2(f32.astype(np.float64))
    assert np.max(np.abs(p32.astype(np.float64) - ex32) / ex32) < 8e-5
    # equioscillation: the error reaches its bound with both signs (a minimax fit)
    err = (p64 - exact) / exact
    assert err.max() > 7e-5 and err.min() < -7e-5


@pytest.mark.gpu
def test_device_exp2_within_bound_of_exp2():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from block_sparse_linear_router_b200 import build, sla2
    build.build()
    lib = sla2.load_library()
    fn = lib.sla2_selftest_exp2
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]
    rng = np.random.default_rng(7)
    x = np.concatenate([np.linspace(-125.0, 9.0, 1 << 20), rng.uniform(-30, 9, 1 << 18),
                        np.arange(-125, 10, dtype=np.float64) + 0.5, np.array([-0.5, 0.5, 0.0, -1e-30])])
    x = x.astype(np.float32)
    xd = torch.from_numpy(x).cuda()
    yd = torch.empty_like(xd)
    assert fn(ctypes.c_void_p(xd.data_ptr()), ctypes.c_void_p(yd.data_ptr()), x.size,
              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)) == 0
    torch.cuda.synchronize()
    y = yd.cpu().numpy().astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    print(f"device exp2: max relative error {rel.max():.2e}")
    assert rel.max() < 1e-4
    # below the clamp the result stays tiny and positive
    z = torch.tensor([-200.0, -1e4, -126.0, float("-inf")], device="cuda")
    w = torch.empty_like(z)
    assert fn(ctypes.c_void_p(z.data_ptr()), ctypes.c_void_p(w.data_ptr()), 4,
              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)) == 0
    torch.cuda.synchronize()
    assert torch.all(w > 0) and torch.all(w < 2.0 ** -124)
