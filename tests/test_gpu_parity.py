"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs, stage by stage and end to end.

Bars: mask exact up to near-ties (oracle logits within 1e-6); Q-hat, V-hat
bit-exact; K-hat within 1 LSB; output within rel-L2 2e-2 and max-abs 5e-2 of
the quantisation-emulating oracle (mode qa); with quantisation off and fp32
output, within rel-L2 1e-3 of the exact oracle (mode u).
"""
import numpy as np
import pytest
import torch

from block_sparse_linear_router_b200.inputs import WORKLOADS, make_custom, make_inputs
from oracle import sla2_oracle as O
from tests.gpu_helpers import (MAX_ABS_Q, REL_L2_Q, REL_L2_U, check_mask_rows, head_np, rel_l2, to_dev)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sla2():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from block_sparse_linear_router_b200 import build
    build.build()
    from block_sparse_linear_router_b200 import sla2 as S
    S.load_library()
    return S


def _oracle_heads(inp, frac, mode, blocks=None):
    B, H = inp.q.shape[:2]
    res = {}
    for b in range(B):
        for h in range(H):
            res[(b, h)] = O.head_forward(*head_np(inp, b, h), frac, mode=mode, blocks=blocks)
    return res


def _compare_full(sla2, inp, frac, tag):
    """Quantised path, every stage, against oracle mode qa."""
    dev = to_dev(inp)
    out, dbg = sla2.forward(dev["q"], dev["k"], dev["v"], dev["proj_q"], dev["proj_k"], dev["alpha"], frac,
                            quantize=1, out_dtype=torch.float32, debug=True)
    torch.cuda.synchronize()
    B, H, N, d = inp.q.shape
    nq, nk = N // 128, N // 64
    ref = _oracle_heads(inp, frac, "qa")
    k = ref[(0, 0)]["k"]
    gm = dbg["mask"].cpu().numpy()
    rm = np.stack([np.stack([ref[(b, h)]["mask"] for h in range(H)]) for b in range(B)])
    rs = np.stack([np.stack([ref[(b, h)]["scores"] for h in range(H)]) for b in range(B)])
    near = check_mask_rows(gm, rm, rs, k)
    # logits: fp32 GPU vs fp64 oracle
    serr = np.max(np.abs(dbg["scores"].cpu().numpy() - rs))
    assert serr < 1e-5, serr
    # idx ascending and consistent with the mask
    gi = dbg["idx"].cpu().numpy()
    assert (np.diff(gi, axis=-1) > 0).all()
    for b in range(B):
        for h in range(H):
            for i in range(nq):
                assert (np.nonzero(gm[b, h, i])[0] == gi[b, h, i]).all()
    # quantised operands
    for b in range(B):
        for h in range(H):
            Q, K, V, *_ = head_np(inp, b, h)
            qh, sq = O.quantize_q(Q)
            np.testing.assert_array_equal(dbg["qhat"][b, h].cpu().numpy(), qh)
            np.testing.assert_array_equal(dbg["sq"][b, h].cpu().numpy(), sq)
            c = ref[(b, h)]["colmean"]
            kh, sk = O.quantize_k(K, c)
            gkh = dbg["khat"][b, h].cpu().numpy().astype(np.int32)
            assert np.abs(gkh - kh).max() <= 1
            assert (gkh != kh).mean() < 1e-3
            np.testing.assert_allclose(dbg["sk"][b, h].cpu().numpy(), sk, rtol=2e-7, atol=0)
            vc, sv = O.quantize_v(V)
            gv = dbg["vhatT"][b, h].cpu().numpy()               # [nk][d][64]
            gv_tok = gv.transpose(0, 2, 1).reshape(N, d)
            np.testing.assert_array_equal(gv_tok, vc)
            np.testing.assert_array_equal(dbg["sv"][b, h].cpu().numpy(), sv)
    # branches and output, skipping query blocks whose mask row is a near-tie swap
    gos, gol, go = dbg["O_s"].cpu().numpy(), dbg["O_l"].cpu().numpy(), out.cpu().numpy()
    errs = {"os": [], "ol": [], "o": []}
    keep_o, keep_ref = [], []
    for b in range(B):
        for h in range(H):
            r = ref[(b, h)]
            for i in range(nq):
                if (b, h, i) in near:
                    continue
                sl = slice(i * 128, (i + 1) * 128)
                keep_o.append(go[b, h, sl])
                keep_ref.append(r["O"][sl])
                errs["os"].append((gos[b, h, sl], r["O_s"][sl]))
                if k < nk:
                    errs["ol"].append((gol[b, h, sl], r["O_l"][sl]))
    e_o = rel_l2(np.concatenate(keep_o), np.concatenate(keep_ref))
    m_o = float(np.max(np.abs(np.concatenate(keep_o) - np.concatenate(keep_ref))))
    e_os = rel_l2(np.concatenate([a for a, _ in errs["os"]]), np.concatenate([b for _, b in errs["os"]]))
    print(f"[{tag}] k={k} rel-L2 O={e_o:.2e} max-abs O={m_o:.2e} O_s={e_os:.2e} near-tie rows={len(near)}")
    assert e_o <= REL_L2_Q and m_o <= MAX_ABS_Q
    assert e_os <= REL_L2_Q
    if errs["ol"]:
        e_ol = rel_l2(np.concatenate([a for a, _ in errs["ol"]]), np.concatenate([b for _, b in errs["ol"]]))
        print(f"[{tag}] rel-L2 O_l={e_ol:.2e}")
        assert e_ol <= 1e-3    # fp16 phi(Q) and fp16 operand tiles, fp32 accumulation
    return e_o


def test_small_workload_all_stages(sla2):
    w = WORKLOADS["small"]
    _compare_full(sla2, make_inputs(w), w.topk_frac, "small")


def test_d128_multi_head(sla2):
    _compare_full(sla2, make_custom(1, 2, 2048, 128, 0.05, seed=21), 0.05, "d128")


def test_batched_ragged_rows_d64(sla2):
    # nq = 5 (not a multiple of the 8-row top-k tile or the 32-row projection tile)
    _compare_full(sla2, make_custom(2, 3, 640, 64, 0.3, seed=22, offset_var=1.0), 0.3, "ragged")


def test_single_query_block_and_k1(sla2):
    _compare_full(sla2, make_custom(1, 2, 128, 64, 0.01, seed=23), 0.01, "N128-k1")
    _compare_full(sla2, make_custom(1, 1, 1024, 128, 0.01, seed=24), 0.01, "k1-d128")


@pytest.mark.parametrize("d", [64, 128])
def test_all_blocks_alpha_one_is_dense_attention(sla2, d):
    inp = make_custom(1, 2, 1024, d, 1.0, seed=25, alpha_one=True)
    dev = to_dev(inp)
    ref = torch.nn.functional.scaled_dot_product_attention(inp.q.double(), inp.k.double(), inp.v.double()).numpy()
    outq = sla2.forward(dev["q"], dev["k"], dev["v"], dev["proj_q"], dev["proj_k"], dev["alpha"], 1.0,
                        quantize=1, out_dtype=torch.float32).cpu().numpy()
    outu = sla2.forward(dev["q"], dev["k"], dev["v"], dev["proj_q"], dev["proj_k"], dev["alpha"], 1.0,
                        quantize=0, out_dtype=torch.float32).cpu().numpy()
    e_q, e_u = rel_l2(outq, ref), rel_l2(outu, ref)
    print(f"dense d={d}: quantised {e_q:.2e}, unquantised {e_u:.2e}")
    assert e_u <= REL_L2_U
    assert e_q <= 3e-2
    _compare_full(sla2, inp, 1.0, f"dense-d{d}")


@pytest.mark.parametrize("shape", [(1, 1, 2048, 64, 0.1), (1, 2, 2048, 128, 0.05), (2, 2, 640, 64, 0.3)])
def test_unquantised_fp32_matches_exact_oracle(sla2, shape):
    B, H, N, d, frac = shape
    inp = make_custom(B, H, N, d, frac, seed=26)
    dev = to_dev(inp)
    out = sla2.forward(dev["q"], dev["k"], dev["v"], dev["proj_q"], dev["proj_k"], dev["alpha"], frac,
                       quantize=0, out_dtype=torch.float32).cpu().numpy()
    ref = O.forward(inp.q, inp.k, inp.v, inp.proj_q, inp.proj_k, inp.alpha, frac, mode="u")
    e = rel_l2(out, ref)
    print(f"unquantised {shape}: rel-L2 {e:.2e}")
    assert e <= REL_L2_U


def test_bf16_output_is_rounded_fp32_output(sla2):
    inp = make_custom(1, 2, 1024, 128, 0.1, seed=27)
    dev = to_dev(inp)
    args = (dev["q"], dev["k"], dev["v"], dev["proj_q"], dev["proj_k"], dev["alpha"], 0.1)
    o32 = sla2.forward(*args, out_dtype=torch.float32)
    o16 = sla2.forward(*args, out_dtype=torch.bfloat16)
    assert torch.equal(o32.to(torch.bfloat16), o16)


def test_router_entry_point(sla2):
    inp = make_custom(2, 2, 1536, 128, 0.1, seed=28)
    dev = to_dev(inp)
    r = sla2.router(dev["q"], dev["k"], dev["proj_q"], dev["proj_k"], 0.1, scores=True)
    mask, idx, scores = O.router(inp.q, inp.k, inp.proj_q, inp.proj_k, 0.1)
    check_mask_rows(r["mask"].cpu().numpy(), mask, scores, O.topk_count(24, 0.1))
    cm = np.stack([np.stack([O.colmean(inp.k[b, h].double().numpy()) for h in range(2)]) for b in range(2)])
    np.testing.assert_array_equal(r["colmean"].cpu().numpy(), cm.astype(np.float32))


def test_router_identity_projection_is_heuristic_router(sla2):
    # proj = I: the learnable router reduces to the pooled-attention Top-k of SLA (detail page §2)
    inp = make_custom(1, 3, 2048, 64, 0.1, seed=31)
    eye = torch.eye(64).expand(3, 64, 64).contiguous()
    dev = to_dev(inp)
    r = sla2.router(dev["q"], dev["k"], eye.cuda(), eye.cuda(), 0.1, scores=True)
    mask, idx, scores = O.router(inp.q, inp.k, eye, eye, 0.1)
    check_mask_rows(r["mask"].cpu().numpy(), mask, scores, O.topk_count(32, 0.1))


@pytest.mark.parametrize("shape", [(1, 1, 2048, 64, 0.1, 0.1), (1, 2, 8192, 128, 0.03, 0.1), (2, 1, 1024, 64, 0.3, 0.5)])
def test_router_soft_matches_oracle(sla2, shape):
    B, H, N, d, frac, tau = shape
    inp = make_custom(B, H, N, d, frac, seed=32)
    dev = to_dev(inp)
    r = sla2.router_soft(dev["q"], dev["k"], dev["proj_q"], dev["proj_k"], frac, tau=tau)
    soft, lam = O.router_soft(inp.q, inp.k, inp.proj_q, inp.proj_k, frac, tau)
    got = r["soft"].cpu().numpy()
    kk = O.topk_count(N // 64, frac)
    e_soft = float(np.max(np.abs(got - soft)))
    e_lam = float(np.max(np.abs(r["lambda"].cpu().numpy() - lam)))
    e_sum = float(np.max(np.abs(got.sum(-1) - kk)))
    print(f"router_soft {shape}: max|soft| {e_soft:.2e} max|lambda| {e_lam:.2e} max|row sum - k| {e_sum:.2e}")
    assert e_soft < 2e-5          # fp32 logits, softmax and sigmoids against fp64
    assert e_lam < 1e-4
    assert e_sum < 1e-3


@pytest.mark.parametrize("d", [64, 128])
def test_linear_state_entry_point(sla2, d):
    inp = make_custom(1, 2, 1024, d, 0.1, seed=29)
    dev = to_dev(inp)
    cm = sla2.router(dev["q"], dev["k"], dev["proj_q"], dev["proj_k"], 0.1)["colmean"]
    st = sla2.linear_state(dev["k"], dev["v"], cm)
    for h in range(2):
        K = inp.k[0, h].double().numpy()
        V = inp.v[0, h].double().numpy()
        hh, zz = O.linear_states(K - O.colmean(K), V)
        hT = hh.transpose(0, 2, 1)                       # the library stores h_j^T
        e_h = rel_l2(st["h"][0, h].cpu().numpy(), hT)
        print(f"linear state d={d} head {h}: rel-L2 h {e_h:.2e}")
        assert e_h < 1e-3                                # fp16 phi operand, fp32 accumulation
        assert rel_l2(st["z"][0, h].cpu().numpy(), zz) < 1e-5
        assert rel_l2(st["Htot"][0, h].cpu().numpy(), hT.sum(0)) < 1e-3
        assert rel_l2(st["Ztot"][0, h].cpu().numpy(), zz.sum(0)) < 1e-5


def test_repeated_calls_are_deterministic(sla2):
    inp = make_custom(1, 2, 2048, 128, 0.05, seed=30)
    dev = to_dev(inp)
    ws = sla2.Workspace.for_shape(1, 2, 2048, 128, 0.05)
    args = (dev["q"], dev["k"], dev["v"], dev["proj_q"], dev["proj_k"], dev["alpha"], 0.05)
    a = sla2.forward(*args, workspace=ws)
    b = sla2.forward(*args, workspace=ws)
    assert torch.equal(a, b)


def test_bounded_wait_reports_timeout_and_context_survives(sla2):
    import ctypes
    lib = sla2.load_library()
    lib.sla2_selftest_timeout.restype = ctypes.c_int
    lib.sla2_selftest_timeout.argtypes = [ctypes.c_void_p, ctypes.c_ulonglong, ctypes.c_void_p]
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    r = lib.sla2_selftest_timeout(ctypes.c_void_p(st.data_ptr()), 2_000_000, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert r == 0
    torch.cuda.synchronize()
    assert int(st.item()) == 5
    # the context is still usable: a normal forward pass runs and reports status 0
    inp = make_custom(1, 1, 512, 64, 0.25, seed=31)
    dev = to_dev(inp)
    status = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    sla2.forward(dev["q"], dev["k"], dev["v"], dev["proj_q"], dev["proj_k"], dev["alpha"], 0.25, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0


@pytest.mark.parametrize("shape", [(1, 3, 8192, 128, 0.03), (1, 3, 8192, 64, 0.1), (1, 3, 8192, 128, 0.001),
                                   (1, 8, 8192, 128, 0.03)])
def test_more_query_blocks_than_sms(sla2, shape):
    """192 or 512 (head, query block) items: the persistent kernels walk several
    items per CTA (k = 1, 3 and 12 key blocks per item; up to four items, so that
    the epilogue's two-slot rings are each reused) and the linear-state pass splits
    heads into chunks."""
    B, H, N, d, frac = shape
    _compare_full(sla2, make_custom(B, H, N, d, frac, seed=32), frac, f"multiwave-d{d}")


def test_full_size_wan13b_sampled(sla2):
    """The benchmarked workload (Wan2.1-1.3B shape: 1 x 12 x 32768 x 128, k% = 3)
    in the same launch configuration as bench.py: the whole mask against the
    oracle router, and the output on sampled query blocks of sampled heads."""
    w = WORKLOADS["wan1.3b"]
    inp = make_inputs(w)
    dev = to_dev(inp)
    out, dbg = sla2.forward(dev["q"], dev["k"], dev["v"], dev["proj_q"], dev["proj_k"], dev["alpha"],
                            w.topk_frac, quantize=1, out_dtype=torch.bfloat16, debug=True)
    torch.cuda.synchronize()
    k = O.topk_count(w.nk, w.topk_frac)
    mask, idx, scores = O.router(inp.q, inp.k, inp.proj_q, inp.proj_k, w.topk_frac)
    near = check_mask_rows(dbg["mask"].cpu().numpy(), mask, scores, k)
    go = out.float().cpu().numpy()
    rng = np.random.default_rng(0)
    errs = []
    for h in (0, 5, 11):
        blocks = sorted(rng.choice(w.nq, size=4, replace=False).tolist())
        blocks = [i for i in blocks if (0, h, i) not in near]
        r = O.head_forward(*head_np(inp, 0, h), w.topk_frac, mode="qa", blocks=blocks)
        for n, i in enumerate(blocks):
            got = go[0, h, i * 128:(i + 1) * 128]
            ref = r["O"][n * 128:(n + 1) * 128]
            errs.append((got, ref))
    g = np.concatenate([a for a, _ in errs])
    rf = np.concatenate([b for _, b in errs])
    e, m = rel_l2(g, rf), float(np.max(np.abs(g - rf)))
    print(f"[wan1.3b sampled] rel-L2 {e:.2e} max-abs {m:.2e} near-tie rows {len(near)}")
    assert e <= REL_L2_Q and m <= MAX_ABS_Q


@pytest.mark.parametrize("name,heads,nblk", [("wan14b", ((0, 0), (0, 23), (0, 39)), 3),
                                             ("batched", ((0, 0), (1, 7), (1, 23)), 4)])
def test_full_size_other_workloads_sampled(sla2, name, heads, nblk):
    """The other evaluated configurations at full size (Wan2.1-14B shape 1 x 40 x
    75776 x 128 at k% = 5; the batched 2 x 24 x 16384 x 64 at k% = 10): the
    sampled heads' masks against the oracle router, and the output on sampled
    query blocks of those heads."""
    w = WORKLOADS[name]
    inp = make_inputs(w)
    dev = to_dev(inp)
    out, dbg = sla2.forward(dev["q"], dev["k"], dev["v"], dev["proj_q"], dev["proj_k"], dev["alpha"],
                            w.topk_frac, quantize=1, out_dtype=torch.bfloat16, debug=True)
    torch.cuda.synchronize()
    del dev
    k = O.topk_count(w.nk, w.topk_frac)
    gmask = dbg["mask"].cpu().numpy()
    go = out.float().cpu().numpy()
    del out, dbg
    rng = np.random.default_rng(1)
    errs, n_near = [], 0
    for b, h in heads:
        Q, K, V, Wq, Wk, al = head_np(inp, b, h)
        s = O.router_scores(Q, K, Wq, Wk)
        mask, _ = O.topk_mask(s, k)
        near = check_mask_rows(gmask[b, h][None], mask[None], s[None], k)
        n_near += len(near)
        near_rows = {r[-1] for r in near}
        blocks = sorted(i for i in rng.choice(w.nq, size=nblk, replace=False).tolist() if i not in near_rows)
        r = O.head_forward(Q, K, V, Wq, Wk, al, w.topk_frac, mode="qa", blocks=blocks)
        for n, i in enumerate(blocks):
            errs.append((go[b, h, i * 128:(i + 1) * 128], r["O"][n * 128:(n + 1) * 128]))
    g = np.concatenate([a for a, _ in errs])
    rf = np.concatenate([c for _, c in errs])
    e, m = rel_l2(g, rf), float(np.max(np.abs(g - rf)))
    print(f"[{name} sampled] rel-L2 {e:.2e} max-abs {m:.2e} near-tie rows {n_near}")
    assert e <= REL_L2_Q and m <= MAX_ABS_Q
