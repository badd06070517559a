"""GPU parity of the backward pass (sla2_backward, through the C ABI) against the
oracle's gradient of the unquantised forward for the same mask (SLA2 detail
page §7 note 3): dQ, dK, dV and dalpha within relative L2 1e-3, on shapes that
span several query and key blocks, both head dimensions, a batch, every block
selected (no linear branch) and more items than SMs."""
import numpy as np
import pytest
import torch

from block_sparse_linear_router_b200.inputs import make_custom
from oracle import sla2_oracle as O
from tests.gpu_helpers import head_np, rel_l2, to_dev

pytestmark = pytest.mark.gpu

REL_L2_BWD = 1e-3     # fp32 gradient against the fp64 oracle (h_j from fp16 tensor-core operands)


@pytest.fixture(scope="module")
def sla2():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from block_sparse_linear_router_b200 import build
    build.build()
    from block_sparse_linear_router_b200 import sla2 as S
    S.load_library()
    return S


@pytest.mark.parametrize("B,H,N,d,frac", [(1, 2, 512, 64, 0.25), (2, 1, 1024, 128, 0.1), (1, 1, 512, 64, 1.0),
                                          (1, 3, 640, 128, 0.3), (1, 2, 8192, 64, 0.05)])
def test_backward_matches_oracle_gradient(sla2, B, H, N, d, frac):
    inp = make_custom(B, H, N, d, frac, seed=61)
    dev = to_dev(inp)
    g = torch.Generator().manual_seed(62)
    dout = torch.randn(B, H, N, d, generator=g, dtype=torch.float32)
    dq, dk, dv, da = sla2.backward(dev["q"], dev["k"], dev["v"], dev["proj_q"], dev["proj_k"], dev["alpha"], frac,
                                   dout.cuda())
    r = sla2.router(dev["q"], dev["k"], dev["proj_q"], dev["proj_k"], frac)
    torch.cuda.synchronize()
    gmask = r["mask"].cpu().numpy()
    ref = {n: np.zeros((B, H, N, d)) for n in ("dQ", "dK", "dV")}
    ref_da = np.zeros((H, N // 128))
    for b in range(B):
        for h in range(H):
            Q, K, V, Wq, Wk, al = head_np(inp, b, h)
            s = O.router_scores(Q, K, Wq, Wk)
            mask, _ = O.topk_mask(s, O.topk_count(N // 64, frac))
            assert np.array_equal(mask, gmask[b, h]), "the GPU router's mask is the oracle's"
            res = O.head_backward(Q, K, V, al, mask, dout[b, h].double().numpy())
            for n in ("dQ", "dK", "dV"):
                ref[n][b, h] = res[n]
            ref_da[h] += res["dalpha"]
    errs = {"dQ": rel_l2(dq.cpu().numpy(), ref["dQ"]), "dK": rel_l2(dk.cpu().numpy(), ref["dK"]),
            "dV": rel_l2(dv.cpu().numpy(), ref["dV"]), "dalpha": rel_l2(da.cpu().numpy(), ref_da)}
    print(f"backward {(B, H, N, d, frac)}: " + " ".join(f"{n} {e:.2e}" for n, e in errs.items()))
    for n, e in errs.items():
        assert e <= REL_L2_BWD, (n, e)
