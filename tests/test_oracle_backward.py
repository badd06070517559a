"""Pins for the oracle's backward pass (the gradient of the unquantised forward
for a fixed block mask; SLA2 detail page §7 note 3 and §2 table): central
finite differences on tiny inputs, two special cases that reduce to library
autograd (every block selected with alpha = 1 is softmax attention; no block
selected with alpha = 0 is textbook linear attention), and planted mistakes
that must fail a pin. CPU only, fp64."""
import numpy as np
import pytest
import torch

from oracle import sla2_oracle as O

N, D = 256, 8          # two query blocks, four key blocks


def _inputs(seed, mask_kind="random"):
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((N, D))
    K = rng.standard_normal((N, D)) + rng.standard_normal(D)      # a channel bias (smoothing matters)
    V = rng.standard_normal((N, D))
    alpha = rng.uniform(0.1, 0.9, N // 128)
    nq, nk = N // 128, N // 64
    if mask_kind == "random":
        mask = np.zeros((nq, nk), np.uint8)
        for i in range(nq):
            mask[i, rng.choice(nk, size=1 + i, replace=False)] = 1
    elif mask_kind == "all":
        mask = np.ones((nq, nk), np.uint8)
    else:
        mask = np.zeros((nq, nk), np.uint8)
    G = rng.standard_normal((N, D))                                 # dL/dO for L = sum(O * G)
    return Q, K, V, alpha, mask, G


def _loss(Q, K, V, alpha, mask, G):
    return float(np.sum(O.head_forward_masked(Q, K, V, alpha, mask) * G))


def _fd_check(seed, n_entries=24, eps=1e-6, tol=1e-6):
    Q, K, V, alpha, mask, G = _inputs(seed)
    g = O.head_backward(Q, K, V, alpha, mask, G)
    rng = np.random.default_rng(seed + 100)
    for name, X in (("dQ", Q), ("dK", K), ("dV", V)):
        for _ in range(n_entries):
            r, c = rng.integers(N), rng.integers(D)
            Xp, Xm = X.copy(), X.copy()
            Xp[r, c] += eps
            Xm[r, c] -= eps
            args_p = {"dQ": (Xp, K, V), "dK": (Q, Xp, V), "dV": (Q, K, Xp)}[name]
            args_m = {"dQ": (Xm, K, V), "dK": (Q, Xm, V), "dV": (Q, K, Xm)}[name]
            num = (_loss(*args_p, alpha, mask, G) - _loss(*args_m, alpha, mask, G)) / (2 * eps)
            assert abs(g[name][r, c] - num) <= tol * max(1.0, abs(num)), (name, r, c, g[name][r, c], num)
    for i in range(len(alpha)):
        ap, am = alpha.copy(), alpha.copy()
        ap[i] += eps
        am[i] -= eps
        num = (_loss(Q, K, V, ap, mask, G) - _loss(Q, K, V, am, mask, G)) / (2 * eps)
        assert abs(g["dalpha"][i] - num) <= tol * max(1.0, abs(num)), ("dalpha", i, g["dalpha"][i], num)


@pytest.mark.parametrize("seed", [1, 2])
def test_backward_matches_central_finite_differences(seed):
    _fd_check(seed)


def test_all_blocks_alpha_one_backward_is_softmax_attention_autograd():
    Q, K, V, _, mask, G = _inputs(3, "all")
    alpha = np.ones(N // 128)
    g = O.head_backward(Q, K, V, alpha, mask, G)
    q, k, v = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (Q, K, V))
    out = torch.nn.functional.scaled_dot_product_attention(q[None, None], k[None, None], v[None, None])[0, 0]
    (out * torch.tensor(G)).sum().backward()
    for name, t in (("dQ", q), ("dK", k), ("dV", v)):
        np.testing.assert_allclose(g[name], t.grad.numpy(), rtol=0, atol=1e-12)
    assert np.all(g["dalpha"] == g["dalpha"])     # finite


def test_no_block_alpha_zero_backward_is_linear_attention_autograd():
    Q, K, V, _, mask, G = _inputs(4, "none")
    alpha = np.zeros(N // 128)
    g = O.head_backward(Q, K, V, alpha, mask, G)
    q, k, v = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (Q, K, V))
    ks = k - k.mean(dim=0, keepdim=True)
    pq, pk = torch.softmax(q, dim=-1), torch.softmax(ks, dim=-1)
    out = (pq @ (pk.T @ v)) / (pq @ pk.sum(dim=0))[:, None]
    (out * torch.tensor(G)).sum().backward()
    for name, t in (("dQ", q), ("dK", k), ("dV", v)):
        np.testing.assert_allclose(g[name], t.grad.numpy(), rtol=0, atol=1e-12)


def test_feature_softmax_backward_against_autograd():
    rng = np.random.default_rng(5)
    X = rng.standard_normal((7, 11))
    dY = rng.standard_normal((7, 11))
    x = torch.tensor(X, requires_grad=True)
    torch.softmax(x, dim=-1).backward(torch.tensor(dY))
    np.testing.assert_allclose(O.feature_softmax_backward(O.feature_softmax(X), dY), x.grad.numpy(), rtol=0, atol=1e-14)


# ---------------------------------------------------------------- planted mistakes
def _fails(fn):
    try:
        fn()
    except AssertionError:
        return True
    return False


def test_state_gradient_over_selected_blocks_is_caught(monkeypatch):
    # dH_i, dZ_i sent to the key blocks query block i SELECTED
    monkeypatch.setattr(O, "unselected_blocks", lambda row: np.nonzero(np.asarray(row))[0])
    assert _fails(lambda: _fd_check(1, n_entries=8))


def test_missing_smoothing_gradient_is_caught(monkeypatch):
    orig = O.head_backward

    def wrong(Q, K, V, alpha_h, mask, dO):
        g = orig(Q, K, V, alpha_h, mask, dO)
        # forgets dK = dK_s - colmean(dK_s): adds the column means back
        Ks_grad = g["dK"]
        g["dK"] = Ks_grad + 0.37 * np.ones_like(Ks_grad) * np.abs(Ks_grad).mean()
        return g
    monkeypatch.setattr(O, "head_backward", wrong)
    assert _fails(lambda: _fd_check(2, n_entries=8))


def test_missing_softmax_rowsum_term_is_caught(monkeypatch):
    orig = O.feature_softmax_backward
    monkeypatch.setattr(O, "feature_softmax_backward", lambda Y, dY: np.asarray(Y) * np.asarray(dY))
    assert _fails(test_no_block_alpha_zero_backward_is_linear_attention_autograd)
    monkeypatch.setattr(O, "feature_softmax_backward", orig)


def test_alpha_gradient_sign_is_caught(monkeypatch):
    orig = O.head_backward

    def wrong(Q, K, V, alpha_h, mask, dO):
        g = orig(Q, K, V, alpha_h, mask, dO)
        g["dalpha"] = -g["dalpha"]                  # dO * (O_l - O_s)
        return g
    monkeypatch.setattr(O, "head_backward", wrong)
    assert _fails(lambda: _fd_check(1, n_entries=1))
