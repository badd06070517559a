"""Plausible mistakes planted in the oracle (on the CPU, through monkeypatch)
must make at least one pin fail. This shows the pins constrain each part of
the oracle rather than restating it."""
import numpy as np
import pytest

from oracle import sla2_oracle as O
import tests.test_oracle_pins as pins


def _fails(fn):
    try:
        fn()
    except AssertionError:
        return True
    return False


def test_unselected_vs_selected_swap_is_caught(monkeypatch):
    orig = O.linear_branch

    def wrong(Q, h, z, mask_i, i):
        return orig(Q, h, z, 1 - mask_i, i)          # sums the SELECTED blocks
    monkeypatch.setattr(O, "linear_branch", wrong)
    assert _fails(pins.test_alpha_zero_is_masked_linear_attention_bruteforce)


def test_missing_online_rescale_is_caught(monkeypatch):
    def wrong(qh, sq, kh, sk, vcode, sv, idx_i, i, d, exact_max=False):
        # forgets to rescale l and acc when the running max grows
        rows = slice(i * O.BQ, (i + 1) * O.BQ)
        qi = qh[rows].astype(np.float64)
        vdec = O.e4m3_decode(vcode)
        m = np.full(O.BQ, -np.inf); l = np.zeros(O.BQ); acc = np.zeros((O.BQ, d))
        for j in idx_i:
            S = (qi @ kh[j * 64:(j + 1) * 64].astype(np.float64).T) * float(sq[i]) * float(sk[j]) / np.sqrt(d)
            m = np.maximum(m, S.max(1))
            p = np.exp(S - m[:, None])
            l = l + p.sum(1)
            acc = acc + O.e4m3_round(448 * p) @ vdec[j * 64:(j + 1) * 64]
        return acc * sv.astype(np.float64)[None, :] / 448 / l[:, None]
    monkeypatch.setattr(O, "sparse_quantized", wrong)
    assert _fails(pins.test_all_blocks_alpha_one_is_dense_attention_sdpa)


def test_ties_to_higher_index_is_caught(monkeypatch):
    def wrong(s, k):
        nq, nk = s.shape
        mask = np.zeros((nq, nk), np.uint8); idx = np.zeros((nq, k), np.int32)
        for i in range(nq):
            order = np.lexsort((-np.arange(nk), -s[i]))
            sel = np.sort(order[:k]); mask[i, sel] = 1; idx[i] = sel
        return mask, idx
    monkeypatch.setattr(O, "topk_mask", wrong)
    assert _fails(pins.test_topk_ties_go_to_lower_index)


def test_e4m3_ties_away_is_caught(monkeypatch):
    def wrong(x):
        x = np.asarray(x, dtype=np.float64)
        a = np.minimum(np.abs(x), 448.0)
        _, E = np.frexp(a)
        q = np.ldexp(1.0, np.maximum(E - 1, -6) - 3)
        r = np.minimum(np.floor(a / q + 0.5) * q, 448.0)
        return np.copysign(r, x)
    monkeypatch.setattr(O, "e4m3_round", wrong)
    assert _fails(pins.test_e4m3_golden_points)


def test_unnormalised_feature_map_is_caught(monkeypatch):
    def wrong(X):
        X = np.asarray(X, dtype=np.float64)
        return np.exp(X - X.max(axis=-1, keepdims=True))
    monkeypatch.setattr(O, "feature_softmax", wrong)
    assert _fails(pins.test_alpha_zero_is_masked_linear_attention_bruteforce)


def test_unsmoothed_quantised_k_is_caught(monkeypatch):
    monkeypatch.setattr(O, "smoothed_k_fp32", lambda K, c: np.asarray(K, dtype=np.float32))
    assert _fails(pins.test_quantised_k_is_smoothed)


def test_wrong_block_size_pooling_is_caught(monkeypatch):
    orig = O.pool
    monkeypatch.setattr(O, "pool", lambda X, b: orig(X, 64 if b == 128 else b) [: X.shape[0] // b])
    assert _fails(pins.test_router_identity_projection_is_heuristic_router)


def test_missing_mix_complement_is_caught(monkeypatch):
    orig = O.head_forward

    def wrong(*a, **kw):
        r = orig(*a, **kw)
        r["O"] = r["O_s"] * 0.25 + r["O_l"]        # forgets (1 - alpha)
        return r
    monkeypatch.setattr(O, "head_forward", wrong)
    assert _fails(pins.test_constant_keys_closed_form)


def test_soft_topk_temperature_multiplied_is_caught(monkeypatch):
    orig = O.soft_topk

    def wrong(pc_row, k, tau, iters=200):
        return orig(np.asarray(pc_row) * tau * tau, k, tau, iters)   # P_c * tau instead of P_c / tau
    monkeypatch.setattr(O, "soft_topk", wrong)
    assert _fails(pins.test_soft_topk_small_tau_is_hard_topk)


def test_transposed_projection_is_caught(monkeypatch):
    orig = O.router_scores

    def wrong(Q, K, Wq, Wk, smooth=True):
        return orig(Q, K, np.asarray(Wq).T, np.asarray(Wk).T, smooth)   # y = x W^T
    monkeypatch.setattr(O, "router_scores", wrong)
    assert _fails(pins.test_router_projection_orientation_elementary_matrices)


def test_swapped_projections_are_caught(monkeypatch):
    orig = O.router_scores

    def wrong(Q, K, Wq, Wk, smooth=True):
        return orig(Q, K, Wk, Wq, smooth)                               # proj_k applied to Q
    monkeypatch.setattr(O, "router_scores", wrong)
    assert _fails(pins.test_router_projection_orientation_elementary_matrices)


def test_first_heads_projection_everywhere_is_caught(monkeypatch):
    orig = O.router_scores
    first = {}

    def wrong(Q, K, Wq, Wk, smooth=True):
        first.setdefault("w", (Wq, Wk))                                  # head 0's matrices reused
        return orig(Q, K, first["w"][0], first["w"][1], smooth)
    monkeypatch.setattr(O, "router_scores", wrong)
    assert _fails(pins.test_router_uses_each_batch_and_heads_own_inputs)


def _quantize_q_in_groups(rows_per_group):
    """Q-hat with the scale taken over groups of `rows_per_group` rows (None:
    the whole tensor); each 128-row block reports the scale of the group
    holding its first row."""
    def wrong(Q):
        N, d = Q.shape
        Q32 = np.asarray(Q, dtype=np.float32)
        g = rows_per_group or N
        qh = np.zeros((N, d), np.int8)
        scale_of_row = np.zeros(N, np.float32)
        for r0 in range(0, N, g):
            qh[r0:r0 + g], s = O.quant_int8(Q32[r0:r0 + g])
            scale_of_row[r0:r0 + g] = s
        return qh, scale_of_row[::O.BQ].copy()
    return wrong


def test_query_quantised_per_64_rows_is_caught(monkeypatch):
    monkeypatch.setattr(O, "quantize_q", _quantize_q_in_groups(64))
    assert _fails(pins.test_quantize_q_exact_on_scaled_integer_blocks)
    assert _fails(pins.test_quantize_q_half_step_per_128_row_block)


def test_query_quantised_per_tensor_is_caught(monkeypatch):
    monkeypatch.setattr(O, "quantize_q", _quantize_q_in_groups(None))
    assert _fails(pins.test_quantize_q_exact_on_scaled_integer_blocks)
    assert _fails(pins.test_quantize_q_half_step_per_128_row_block)
