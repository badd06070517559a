"""Pins for the CPU oracle: facts fixed by the SLA2 pages, by mathematics and by
library routines, each independent of the oracle's own code path.

No GPU is used here. Sources: the SLA2 summary page (paper.rainbus.top, the
four-step forward pass) and the SLA2 detail page (zhaifeiyue.github.io: §3
flowchart, §4 symbol table, Eq. 9, Eq. 11, §7 implementation notes).
"""
import math
import os

import numpy as np
import pytest
import torch

from oracle import sla2_oracle as O
from block_sparse_linear_router_b200.inputs import make_custom, make_inputs, WORKLOADS

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _head(inp, b=0, h=0):
    f = lambda t: t[b, h].double().numpy()
    return f(inp.q), f(inp.k), f(inp.v), inp.proj_q[h].double().numpy(), inp.proj_k[h].double().numpy(), inp.alpha[h].double().numpy()


def _expand(mask, N):
    """M in {0,1}^{N x N} from M_c: each block entry covers 128 x 64 tokens
    ([D] §3 flowchart, 'Expand M_c -> M')."""
    return np.kron(mask.astype(np.float64), np.ones((O.BQ, O.BK)))


def _rel(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


# ---------------------------------------------------------------- golden files
def test_topk_counts_golden():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "topk_counts.txt")) if l.strip() and not l.startswith("#")]
    assert len(rows) >= 5
    for nk, frac, k in rows:
        assert O.topk_count(int(nk), float(frac)) == int(k), (nk, frac, k)


def test_e4m3_golden_points():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "e4m3_points.txt")) if l.strip() and not l.startswith("#")]
    assert len(rows) >= 15
    for x, dec, code in rows:
        x = np.float64(float(x))
        got = O.e4m3_round(x)
        assert got == float(dec) and np.signbit(got) == np.signbit(float(dec)), (x, got, dec)
        assert int(O.e4m3_code(x)) == int(code, 16), (x, hex(int(O.e4m3_code(x))), code)
        assert O.e4m3_decode(np.uint8(int(code, 16))) == float(dec)


# ---------------------------------------------------------------- codecs
def test_e4m3_matches_torch_cast_dense_sweep():
    """The oracle's e4m3 encoder against torch.float8_e4m3fn casts: every
    representable value, every midpoint, one fp32 ulp either side of each
    midpoint, and 400k log-uniform random values, all within [-448, 448]."""
    codes = np.arange(256, dtype=np.uint8)
    vals = O.e4m3_decode(codes)
    finite = np.isfinite(vals) & ((codes & 0x7F) != 0x7F)
    rep = np.unique(vals[finite])
    mids = (rep[:-1] + rep[1:]) / 2
    mids32 = mids.astype(np.float32)
    up = np.nextafter(mids32, np.float32(np.inf))
    dn = np.nextafter(mids32, np.float32(-np.inf))
    rng = np.random.default_rng(0)
    rnd = (np.exp(rng.uniform(np.log(1e-4), np.log(448.0), 400_000)) * rng.choice([-1, 1], 400_000)).astype(np.float32)
    x = np.concatenate([rep.astype(np.float32), mids32, up, dn, rnd]).astype(np.float32)
    x = x[np.abs(x) <= 448]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn)
    ref_codes = ref.view(torch.uint8).numpy()
    ref_vals = ref.to(torch.float64).numpy()
    got_codes = O.e4m3_code(x.astype(np.float64))
    np.testing.assert_array_equal(got_codes, ref_codes)
    np.testing.assert_array_equal(O.e4m3_round(x.astype(np.float64)), ref_vals)


def test_int8_quantiser_matches_torch_round_half_even():
    rng = np.random.default_rng(1)
    X = (rng.standard_normal((128, 64)) * 3).astype(np.float32)
    X[0, :8] = [0.5, -0.5, 1.5, -2.5, 3.0, 0.0, -0.0, 7.25]
    q, s = O.quant_int8(X)
    a = np.float32(np.abs(X).max())
    assert s == np.float32(a / np.float32(127))
    t = torch.from_numpy(X) * torch.tensor(np.float32(127) / a, dtype=torch.float32)
    ref = torch.round(t).clamp(-127, 127).to(torch.int8).numpy()     # torch.round: half to even
    np.testing.assert_array_equal(q, ref)
    assert np.abs(q).max() == 127
    z, sz = O.quant_int8(np.zeros((4, 4), np.float32))
    assert sz == 0 and not z.any()


def test_int8_products_are_exact():
    rng = np.random.default_rng(2)
    a = rng.integers(-127, 128, (8, 64))
    b = rng.integers(-127, 128, (5, 64))
    got = a.astype(np.int8).astype(np.float64) @ b.astype(np.int8).astype(np.float64).T
    brute = [[sum(int(x) * int(y) for x, y in zip(ra, rb)) for rb in b] for ra in a]
    np.testing.assert_array_equal(got, np.array(brute, dtype=np.float64))


def test_v_quantiser_per_channel_and_zero_channel():
    rng = np.random.default_rng(3)
    V = rng.standard_normal((256, 8)).astype(np.float32)
    V[:, 3] = 0.0
    codes, sv = O.quantize_v(V)
    assert sv[3] == 0 and not (codes[:, 3] & 0x7F).any()
    for e in (0, 5):
        a = np.abs(V[:, e]).max()
        assert sv[e] == np.float32(a / np.float32(448))
        # the largest-magnitude entry maps to +-448 and the dequantised column is within half a step
        deq = O.e4m3_decode(codes[:, e]) * float(sv[e])
        assert np.max(np.abs(O.e4m3_decode(codes[:, e]))) == 448
        assert np.all(np.abs(deq - V[:, e]) <= np.abs(V[:, e]) * 2 ** -4 + 2 ** -9 * float(sv[e]) + 1e-12)


def _scaled_integer_query_blocks():
    """Query rows whose 128-row blocks are integers times a power of two, so
    that symmetric INT8 with scale max|block| / 127 is exact: block i holds
    integers in [-127, 127] times 2^-i, with one +-127 in its SECOND 64-row
    half only (its first half stays within +-90). A block-wise quantiser
    must return those integers and the step 2^-i; a quantiser over 64-row
    groups would stretch the first half to +-127, and one over the whole
    tensor would use block 0's step everywhere."""
    rng = np.random.default_rng(17)
    nq, d = 4, 32
    ints = np.zeros((nq * O.BQ, d), np.int64)
    steps = np.zeros(nq)
    for i in range(nq):
        blk = rng.integers(-127, 128, (O.BQ, d))
        blk[:64] = rng.integers(-90, 91, (64, d))
        blk[64 + i, 3 + i] = 127 if i % 2 == 0 else -127
        ints[i * O.BQ:(i + 1) * O.BQ] = blk
        steps[i] = 2.0 ** -i
    Q = (ints * np.repeat(steps, O.BQ)[:, None]).astype(np.float64)
    return Q, ints, steps


def test_quantize_q_exact_on_scaled_integer_blocks():
    """Q-hat is per 128-token query block ([S] step 2: Q and K quantised to
    INT8 block-wise, with b_q = 128 the query block of [S] step 1): on blocks
    that are exact multiples of a power-of-two step with a +-127 entry, the
    codes are the integers and s_q the step, exactly."""
    Q, ints, steps = _scaled_integer_query_blocks()
    qh, sq = O.quantize_q(Q)
    assert qh.shape == Q.shape and sq.shape == (Q.shape[0] // O.BQ,)
    np.testing.assert_array_equal(qh.astype(np.int64), ints)
    np.testing.assert_array_equal(sq.astype(np.float64), steps)


def test_quantize_q_half_step_per_128_row_block():
    """On the seeded query rows (magnitudes varying per 64-token block), every
    128-row block dequantises with ONE scale to within half a step, and the
    block's largest code is +-127 (the step is as fine as the block allows)."""
    inp = make_custom(1, 1, 1024, 64, 0.1, seed=18, offset_var=4.0)
    Q = _head(inp)[0]
    Q[:64] *= 0.25                           # first half of block 0 much smaller
    Q = Q.astype(np.float32).astype(np.float64)
    qh, sq = O.quantize_q(Q)
    for i in range(Q.shape[0] // O.BQ):
        rows = slice(i * O.BQ, (i + 1) * O.BQ)
        deq = qh[rows].astype(np.float64) * float(sq[i])
        # half a step, plus the fp32 rounding of x * (127 / amax) (a few units in 2^-23 of 127)
        assert np.max(np.abs(deq - Q[rows])) <= 0.5 * float(sq[i]) * (1 + 1e-4)
        assert np.abs(qh[rows].astype(np.int64)).max() == 127


# ---------------------------------------------------------------- router
def test_pooling_and_colmean_bruteforce():
    rng = np.random.default_rng(4)
    X = rng.standard_normal((256, 4))
    p = O.pool(X, 64)
    for j in range(4):
        for e in range(4):
            assert abs(p[j, e] - sum(X[t, e] for t in range(64 * j, 64 * j + 64)) / 64) < 1e-14
    c = O.colmean(X)
    assert np.allclose(c, [sum(X[:, e]) / 256 for e in range(4)], rtol=0, atol=1e-14)


def test_router_identity_projection_is_heuristic_router():
    """With proj_q = proj_k = I the learnable router reduces to SLA's
    heuristic softmax(Qbar Kbar^T / sqrt d) router (detail page §2 table,
    'Routing' row); computed here with torch's softmax on explicit pooling."""
    inp = make_custom(1, 1, 512, 16, 0.25, seed=5)
    Q, K, V, _, _, _ = _head(inp)
    I = np.eye(16)
    s = O.router_scores(Q, K, I, I)
    Qt, Kt = torch.from_numpy(Q), torch.from_numpy(K)
    Qb = Qt.reshape(4, 128, 16).mean(1)
    Ks = Kt - Kt.mean(0)
    Kb = Ks.reshape(8, 64, 16).mean(1)
    Pc_ref = torch.softmax(Qb @ Kb.T / 4.0, dim=1).numpy()
    np.testing.assert_allclose(O.compressed_probs(s), Pc_ref, rtol=1e-12, atol=1e-15)


def test_router_projection_orientation_elementary_matrices():
    """y = x W with W stored [d_in][d_out]: with proj_q = E(0 -> 1) and proj_k =
    E(2 -> 1) (a single one at row 0 / row 2, column 1) the projected vectors meet
    only in feature 1, so s_ij = Qbar_i[0] * Kbar_s,j[2] / sqrt(d). A transposed or
    swapped projection moves the features elsewhere and fails this."""
    inp = make_custom(1, 1, 512, 16, 0.25, seed=15)
    Q, K, V, _, _, _ = _head(inp)
    Wq = np.zeros((16, 16)); Wq[0, 1] = 1.0
    Wk = np.zeros((16, 16)); Wk[2, 1] = 1.0
    s = O.router_scores(Q, K, Wq, Wk)
    Qt, Kt = torch.from_numpy(Q), torch.from_numpy(K)
    Qb = Qt.reshape(4, 128, 16).mean(1)
    Kb = (Kt - Kt.mean(0)).reshape(8, 64, 16).mean(1)
    ref = torch.outer(Qb[:, 0], Kb[:, 2]).numpy() / 4.0
    np.testing.assert_allclose(s, ref, rtol=1e-12, atol=1e-15)


def test_router_uses_each_batch_and_heads_own_inputs():
    """The [B, H] router takes head h's projections and head (b, h)'s Q, K:
    with elementary projections that differ per head (feature 0 of Q against
    feature h + 1 of K_s), each head's logits equal the outer product computed
    directly with torch pooling."""
    inp = make_custom(2, 3, 512, 16, 0.25, seed=16)
    H, d = 3, 16
    Wq = np.zeros((H, d, d)); Wk = np.zeros((H, d, d))
    for h in range(H):
        Wq[h, 0, 5] = 1.0
        Wk[h, h + 1, 5] = 1.0
    _, _, scores = O.router(inp.q, inp.k, Wq, Wk, 0.25)
    for b in range(2):
        for h in range(H):
            Qt, Kt = inp.q[b, h].double(), inp.k[b, h].double()
            Qb = Qt.reshape(4, 128, d).mean(1)
            Kb = (Kt - Kt.mean(0)).reshape(8, 64, d).mean(1)
            ref = torch.outer(Qb[:, 0], Kb[:, h + 1]).numpy() / 4.0
            np.testing.assert_allclose(scores[b, h], ref, rtol=1e-12, atol=1e-15)


def test_topk_matches_bruteforce_sort_and_counts():
    rng = np.random.default_rng(6)
    s = rng.standard_normal((16, 40))
    s[3, 10] = s[3, 2]           # an exact tie inside a row
    for k in (1, 5, 17, 40):
        mask, idx = O.topk_mask(s, k)
        assert (mask.sum(axis=1) == k).all()
        for i in range(16):
            brute = sorted(range(40), key=lambda j: (-s[i, j], j))[:k]
            assert list(idx[i]) == sorted(brute)
            assert (np.diff(idx[i]) > 0).all()


def test_topk_ties_go_to_lower_index():
    """Exactly duplicated key blocks give exactly equal logits; the lower
    block index must win every tie."""
    inp = make_custom(1, 1, 1024, 16, 0.25, seed=7)
    Q, K, V, Wq, Wk, _ = _head(inp)
    K = K.copy()
    K[:] = np.tile(K[:64], (16, 1))          # all 16 key blocks identical
    s = O.router_scores(Q, K, Wq, Wk)
    mask, idx = O.topk_mask(s, 4)
    assert (idx == np.arange(4)).all()
    K2 = _head(inp)[1].copy()
    K2[9 * 64:10 * 64] = K2[2 * 64:3 * 64]  # block 9 duplicates block 2
    s2 = O.router_scores(Q, K2, Wq, Wk)
    assert (s2[:, 9] == s2[:, 2]).all()
    for k in range(1, 16):
        m2, _ = O.topk_mask(s2, k)
        assert not np.any((m2[:, 9] == 1) & (m2[:, 2] == 0))


def test_router_mask_invariant_to_k_smoothing():
    """Each row's logits shift by a constant when K is smoothed, so the mask
    is unchanged (rows whose k-th and (k+1)-th logits are within 1e-9 skipped)."""
    inp = make_custom(1, 1, 2048, 32, 0.1, seed=8)
    Q, K, V, Wq, Wk, _ = _head(inp)
    s1 = O.router_scores(Q, K, Wq, Wk, smooth=True)
    s0 = O.router_scores(Q, K, Wq, Wk, smooth=False)
    d = s1 - s0
    assert np.allclose(d, d[:, :1], atol=1e-12)
    k = O.topk_count(32, 0.1)
    m1, _ = O.topk_mask(s1, k)
    m0, _ = O.topk_mask(s0, k)
    np.testing.assert_array_equal(m1, m0)


# ---------------------------------------------------------------- special cases
def test_all_blocks_alpha_one_is_dense_attention_sdpa():
    """k% = 100 and alpha = 1: the sparse branch covers every key and the
    output is ordinary softmax attention ([S] step 2 is FlashAttention over
    M = 1); compared with torch's scaled_dot_product_attention in fp64 on the
    UNsmoothed K (softmax shift invariance)."""
    inp = make_custom(1, 2, 512, 32, 1.0, seed=9, alpha_one=True)
    ref = torch.nn.functional.scaled_dot_product_attention(inp.q.double(), inp.k.double(), inp.v.double()).numpy()
    got = O.forward(inp.q, inp.k, inp.v, inp.proj_q, inp.proj_k, inp.alpha, 1.0, mode="u")
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-12)
    gq = O.forward(inp.q, inp.k, inp.v, inp.proj_q, inp.proj_k, inp.alpha, 1.0, mode="qa")
    assert _rel(gq, ref) < 3e-2          # INT8/FP8 emulation stays close to attention


def test_alpha_zero_is_masked_linear_attention_bruteforce():
    """alpha = 0: O = norm(phi(Q) phi(K)^T ⊙ (1 - M)) V over the full N x N
    matrix ([D] §3 flowchart, Linear Branch), with M expanded from M_c."""
    inp = make_custom(1, 1, 1024, 16, 0.25, seed=10)
    Q, K, V, Wq, Wk, _ = _head(inp)
    r = O.head_forward(Q, K, V, Wq, Wk, np.zeros(8), 0.25, mode="qa")
    Ks = K - K.mean(axis=0)
    eq = np.exp(Q - Q.max(1, keepdims=True)); phq = eq / eq.sum(1, keepdims=True)
    ek = np.exp(Ks - Ks.max(1, keepdims=True)); phk = ek / ek.sum(1, keepdims=True)
    L = (phq @ phk.T) * (1.0 - _expand(r["mask"], 1024))
    ref = (L @ V) / L.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(r["O"], ref, rtol=1e-11, atol=1e-13)


def test_no_selected_block_is_textbook_linear_attention():
    """With no block selected (test-only k = 0) the linear branch is plain
    linear attention phi(Q)(phi(K)^T V) / (phi(Q)(phi(K)^T 1)), using torch's
    softmax for phi."""
    inp = make_custom(1, 1, 512, 16, 0.25, seed=11)
    Q, K, V, Wq, Wk, _ = _head(inp)
    r = O.head_forward(Q, K, V, Wq, Wk, np.zeros(4), 0.25, mode="u", k_override=0)
    Kt = torch.from_numpy(K)
    phk = torch.softmax(Kt - Kt.mean(0), dim=1)
    phq = torch.softmax(torch.from_numpy(Q), dim=1)
    ref = (phq @ (phk.T @ torch.from_numpy(V))) / (phq @ phk.sum(0))[:, None]
    np.testing.assert_allclose(r["O"], ref.numpy(), rtol=1e-12, atol=1e-14)


def test_eq9_true_row_mass():
    """Eq. 9 of the detail page: P_1 V = alpha ⊙ O_s with alpha = P_1 1 the
    true row mass of the full attention P restricted to the mask."""
    inp = make_custom(1, 1, 1024, 16, 0.25, seed=12)
    Q, K, V, Wq, Wk, _ = _head(inp)
    r = O.head_forward(Q, K, V, Wq, Wk, np.ones(8), 0.25, mode="u")
    P = torch.softmax(torch.from_numpy(Q) @ torch.from_numpy(K).T / 4.0, dim=1).numpy()
    P1 = P * _expand(r["mask"], 1024)
    alpha_r = P1.sum(axis=1)
    np.testing.assert_allclose(alpha_r[:, None] * r["O_s"], P1 @ V, rtol=1e-11, atol=1e-14)
    # Eq. 11 with the true mass: alpha P_s + (1 - alpha) P_l keeps rows normalised,
    # shown on V = 1: every output entry is exactly 1.
    ones = np.ones_like(V)
    for a in (0.0, 0.3, 1.0):
        ro = O.head_forward(Q, K, ones, Wq, Wk, np.full(8, a), 0.25, mode="u")
        np.testing.assert_allclose(ro["O"], 1.0, rtol=0, atol=1e-12)


def test_constant_keys_closed_form():
    """All keys equal: K_s = 0, every logit is 0, every router score ties, so
    the first k blocks are selected; attention is uniform, O_s is the mean of
    V (of the dequantised V-hat in the quantised modes) over the selected
    tokens and O_l the mean of V over the rest."""
    inp = make_custom(1, 1, 1024, 16, 0.25, seed=13)
    Q, K, V, Wq, Wk, _ = _head(inp)
    K = np.tile(K[:1], (1024, 1))
    k = O.topk_count(16, 0.25)
    sel = np.arange(k * 64)
    for mode in ("u", "qa", "qb"):
        r = O.head_forward(Q, K, V, Wq, Wk, np.full(8, 0.25), 0.25, mode=mode)
        assert (r["idx"] == np.arange(k)).all()
        if mode == "u":
            os_ref = V[sel].mean(axis=0)
        else:
            codes, sv = O.quantize_v(V)
            os_ref = (O.e4m3_decode(codes[sel]) * sv.astype(np.float64)).mean(axis=0)
        ol_ref = V[k * 64:].mean(axis=0)
        np.testing.assert_allclose(r["O_s"], np.broadcast_to(os_ref, r["O_s"].shape), rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(r["O_l"], np.broadcast_to(ol_ref, r["O_l"].shape), rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(r["O"], 0.25 * r["O_s"] + 0.75 * r["O_l"], rtol=1e-12)


def test_total_minus_selected_equals_unselected_sum():
    """H_total - sum_{selected} h_j = sum_{unselected} h_j, the identity the
    GPU path uses for H_i ([D] §7 note 2: h_j precomputed then accumulated)."""
    inp = make_custom(1, 1, 1024, 16, 0.25, seed=14)
    Q, K, V, Wq, Wk, _ = _head(inp)
    r = O.head_forward(Q, K, V, Wq, Wk, np.ones(8), 0.25)
    h = r["h"]
    Ks = K - K.mean(0)
    ek = np.exp(Ks - Ks.max(1, keepdims=True)); phk = ek / ek.sum(1, keepdims=True)
    np.testing.assert_allclose(h.sum(0), phk.T @ V, rtol=1e-12, atol=1e-12)
    for i in range(8):
        sel = r["mask"][i] == 1
        np.testing.assert_allclose(h.sum(0) - h[sel].sum(0), h[~sel].sum(0), rtol=1e-10, atol=1e-12)


def test_single_selected_block_schedules_agree():
    """With one selected block the running max is the final max: modes qa and
    qb coincide exactly."""
    inp = make_custom(1, 1, 1024, 16, 1.0 / 16, seed=15)
    Q, K, V, Wq, Wk, al = _head(inp)
    a = O.head_forward(Q, K, V, Wq, Wk, al, 1.0 / 16, mode="qa")
    b = O.head_forward(Q, K, V, Wq, Wk, al, 1.0 / 16, mode="qb")
    assert a["k"] == 1
    np.testing.assert_array_equal(a["O"], b["O"])


def test_modes_agree_within_quantisation_error_small_workload():
    """The small workload (2048 tokens, d = 64, k% = 10): the quantised modes
    stay within a few percent of the exact one, and the schedule effect
    (qa vs qb) is well below the quantisation effect."""
    w = WORKLOADS["small"]
    inp = make_inputs(w)
    u = O.forward(inp.q, inp.k, inp.v, inp.proj_q, inp.proj_k, inp.alpha, w.topk_frac, mode="u")
    qa = O.forward(inp.q, inp.k, inp.v, inp.proj_q, inp.proj_k, inp.alpha, w.topk_frac, mode="qa")
    qb = O.forward(inp.q, inp.k, inp.v, inp.proj_q, inp.proj_k, inp.alpha, w.topk_frac, mode="qb")
    e_u = _rel(qa, u)
    e_b = _rel(qa, qb)
    assert 1e-4 < e_u < 3e-2, e_u
    assert e_b < e_u, (e_b, e_u)


def test_quantised_k_is_smoothed():
    inp = make_custom(1, 1, 512, 16, 0.25, seed=16)
    _, K, _, _, _, _ = _head(inp)
    c = O.colmean(K)
    kh, sk = O.quantize_k(K, c)
    Ks = K - c
    for j in range(8):
        deq = kh[j * 64:(j + 1) * 64].astype(np.float64) * float(sk[j])
        assert np.max(np.abs(deq - Ks[j * 64:(j + 1) * 64])) <= 0.5 * float(sk[j]) * 1.001 + 1e-6


# --------------------------------------------------------------------------
# SoftTop-k (detail page §4, Eq. 17): sigmoid(P_c / tau + lambda_i), lambda_i
# by bisection so that each row sums to k
# --------------------------------------------------------------------------
def test_soft_topk_rows_sum_to_k_and_lambda_in_bracket():
    rng = np.random.default_rng(11)
    for nk, frac, tau in ((32, 0.1, 0.1), (512, 0.03, 0.1), (256, 0.5, 0.05), (40, 0.25, 1.0)):
        k = O.topk_count(nk, frac)
        pc = rng.random(nk) ** 3
        pc /= pc.sum()
        m, lam = O.soft_topk(pc, k, tau)
        assert abs(m.sum() - k) < 1e-9
        assert np.all((m > 0) & (m < 1))
        base = math.log(k / (nk - k))
        assert base - 1.0 / tau - 1e-12 <= lam <= base + 1e-12


def test_soft_topk_constant_row_closed_form():
    # every P_c equal: sigmoid(c / tau + lambda) = k / nk for every entry
    for nk, k, tau in ((32, 3, 0.1), (512, 15, 0.1), (64, 40, 0.5)):
        m, lam = O.soft_topk(np.full(nk, 1.0 / nk), k, tau)
        np.testing.assert_allclose(m, k / nk, rtol=0, atol=1e-12)
        assert abs(lam - (math.log(k / (nk - k)) - 1.0 / (nk * tau))) < 1e-9


def test_soft_topk_small_tau_is_hard_topk():
    # well separated P_c and a tiny temperature: the relaxation reaches the hard mask
    rng = np.random.default_rng(12)
    nk, k = 64, 7
    pc = rng.permutation(np.arange(1, nk + 1, dtype=np.float64))
    pc /= pc.sum()                     # neighbouring values differ by 1 / sum = 4.8e-4
    m, _ = O.soft_topk(pc, k, 2e-5)
    hard = np.zeros(nk)
    hard[np.argsort(-pc)[:k]] = 1.0
    assert np.max(np.abs(m - hard)) < 1e-3


def test_soft_topk_preserves_order_and_full_selection():
    rng = np.random.default_rng(13)
    pc = rng.random(100)
    pc /= pc.sum()
    m, _ = O.soft_topk(pc, 10, 0.1)
    order = np.argsort(pc)
    assert np.all(np.diff(m[order]) >= 0)
    m_all, lam = O.soft_topk(pc, 100, 0.1)
    assert np.all(m_all == 1.0) and lam == math.inf
