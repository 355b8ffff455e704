"""Pins of the CPU oracle to things other than itself.

Each test checks the oracle against something the TTT pages or plain
mathematics fix: hand-worked numbers (tests/golden), central finite
differences of the loss, torch's own LayerNorm/GELU autograd (a separate
library), closed forms and special cases, and invariants (primal == dual,
resume, scale invariance). Page citations name "Test-Time Training: Linear
Complexity Beyond Attention" as P-TTT and its sections.
"""
from __future__ import annotations

import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(1234)


def rand_problem(B, H, T, d, *, dh=0, eta_scale=0.05, w_scale=0.3, seed=0):
    r = np.random.default_rng(seed)
    Q = r.standard_normal((B, H, T, d)) / np.sqrt(d)
    K = r.standard_normal((B, H, T, d)) / np.sqrt(d)
    V = r.standard_normal((B, H, T, d)) / np.sqrt(d)
    eta = eta_scale * (0.5 + r.random((B, H, T)))
    if dh:
        W1 = w_scale * r.standard_normal((H, d, dh)) / np.sqrt(d)
        W2 = w_scale * r.standard_normal((H, dh, d)) / np.sqrt(dh)
    else:
        W1 = w_scale * r.standard_normal((H, d, d)) / np.sqrt(d)
        W2 = None
    gamma = 1.0 + 0.1 * r.standard_normal((H, d))
    beta = 0.1 * r.standard_normal((H, d))
    return Q, K, V, eta, W1, W2, gamma, beta


# ---------------------------------------------------------------- torch helpers
# Independent definitions: torch's layer_norm and gelu, torch autograd for the
# gradient. Nothing here calls the oracle.

def t_f_linear(k, W, gamma, beta, ln, eps):
    x = k @ W
    if not ln:
        return x
    return k + F.layer_norm(x, (x.shape[-1],), gamma, beta, eps)


def t_f_mlp(k, W1, W2, gamma, beta, eps):
    x = F.gelu(k @ W1, approximate="none") @ W2
    return k + F.layer_norm(x, (x.shape[-1],), gamma, beta, eps)


def t(x):
    return torch.tensor(np.asarray(x), dtype=torch.float64)


def autograd_grad_linear(k, v, W, gamma, beta, ln, eps=1e-5):
    Wt = t(W).requires_grad_(True)
    f = t_f_linear(t(k), Wt, t(gamma) if ln else None, t(beta) if ln else None, ln, eps)
    loss = 0.5 * ((f - t(v)) ** 2).sum()
    (g,) = torch.autograd.grad(loss, Wt)
    return g.numpy()


# ---------------------------------------------------------------- golden, hand-worked

def _read_cases(path):
    cases, cur = [], None
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, *vals = line.split()
        if key == "case":
            cur = {"name": vals[0]}
            cases.append(cur)
        elif key == "mode":
            cur[key] = vals[0]
        else:
            cur[key] = [float(x) for x in vals]
    return cases


@pytest.mark.parametrize("case", _read_cases(os.path.join(GOLDEN, "linear_d1_hand.txt")),
                         ids=lambda c: c["name"])
def test_golden_d1_hand_worked(case):
    T = len(case["k"])
    sh = (1, 1, T, 1)
    Q, K, V = (np.array(case[x]).reshape(sh) for x in "qkv")
    eta = np.array(case["eta"]).reshape(1, 1, T)
    W0 = np.array(case["w0"]).reshape(1, 1, 1)
    b = int(case["b"][0])
    if case["mode"] == "chunk":
        Z, Wo = oracle.chunk_primal(Q, K, V, eta, W0, chunk=b)
    else:
        Z, Wo = oracle.linear_primal(Q, K, V, eta, W0, b=b, ln=False)
    np.testing.assert_allclose(Z.ravel(), case["z"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(Wo.ravel(), case["w_out"], rtol=0, atol=1e-15)


def test_golden_gelu_table():
    rows = np.loadtxt(os.path.join(GOLDEN, "gelu_normal_table.txt"))
    for h, g in rows:
        assert abs(oracle.gelu(h) - g) < 1e-10, (h, oracle.gelu(h), g)
    assert oracle.gelu_prime(0.0) == 0.5
    # large |h|: GELU(h) -> h for h >> 0 and -> 0 for h << 0
    assert abs(oracle.gelu(12.0) - 12.0) < 1e-12
    assert abs(oracle.gelu(-12.0)) < 1e-12


# ---------------------------------------------------------------- gradients

@pytest.mark.parametrize("ln", [False, True])
@pytest.mark.parametrize("d", [1, 2, 4, 8])
def test_grad_linear_finite_differences(ln, d):
    """P-TTT, Key Architectural Mechanics part 2: the gradient of
    1/2 ||f(k;W) - v||^2, checked by central differences of the loss alone."""
    if ln and d == 1:
        pytest.skip("LayerNorm over one element is constant")
    r = np.random.default_rng(d + 10 * ln)
    k, v = r.standard_normal(d), r.standard_normal(d)
    W = 0.5 * r.standard_normal((d, d))
    gamma, beta = 1 + 0.1 * r.standard_normal(d), 0.1 * r.standard_normal(d)
    G = oracle.grad_linear(k, v, W, gamma, beta, ln=ln)
    h = 1e-6
    FD = np.zeros_like(W)
    for i in range(d):
        for j in range(d):
            Wp, Wm = W.copy(), W.copy()
            Wp[i, j] += h
            Wm[i, j] -= h
            FD[i, j] = (oracle.loss_linear(k, v, Wp, gamma, beta, ln=ln)
                        - oracle.loss_linear(k, v, Wm, gamma, beta, ln=ln)) / (2 * h)
    scale = max(1.0, np.abs(G).max())
    assert np.abs(G - FD).max() / scale < 1e-7


@pytest.mark.parametrize("ln", [False, True])
def test_grad_linear_matches_torch_autograd(ln):
    d = 16
    r = np.random.default_rng(7)
    for _ in range(5):
        k, v = r.standard_normal(d) / 4, r.standard_normal(d) / 4
        W = 0.3 * r.standard_normal((d, d))
        gamma, beta = 1 + 0.1 * r.standard_normal(d), 0.1 * r.standard_normal(d)
        G = oracle.grad_linear(k, v, W, gamma, beta, ln=ln)
        Gt = autograd_grad_linear(k, v, W, gamma, beta, ln)
        np.testing.assert_allclose(G, Gt, rtol=1e-11, atol=1e-12 * np.abs(Gt).max())
        # the linear gradient is the outer product k^T (kW - v) (column form (Wk - v)k^T)
        if not ln:
            np.testing.assert_allclose(G, np.outer(k, k @ W - v), rtol=1e-13, atol=1e-15)


@pytest.mark.parametrize("d,dh", [(2, 8), (4, 16)])
def test_grad_mlp_finite_differences(d, dh):
    r = np.random.default_rng(d)
    k, v = r.standard_normal(d), r.standard_normal(d)
    W1, W2 = r.standard_normal((d, dh)), r.standard_normal((dh, d)) / 2
    gamma, beta = 1 + 0.1 * r.standard_normal(d), 0.1 * r.standard_normal(d)
    G1, G2 = oracle.grad_mlp(k, v, W1, W2, gamma, beta)
    h = 1e-6
    for W, G, which in ((W1, G1, 1), (W2, G2, 2)):
        FD = np.zeros_like(W)
        for idx in np.ndindex(W.shape):
            Wp, Wm = W.copy(), W.copy()
            Wp[idx] += h
            Wm[idx] -= h
            args_p = (Wp, W2) if which == 1 else (W1, Wp)
            args_m = (Wm, W2) if which == 1 else (W1, Wm)
            FD[idx] = (oracle.loss_mlp(k, v, *args_p, gamma, beta)
                       - oracle.loss_mlp(k, v, *args_m, gamma, beta)) / (2 * h)
        assert np.abs(G - FD).max() / max(1.0, np.abs(G).max()) < 1e-7


def test_grad_mlp_matches_torch_autograd():
    d, dh = 8, 32
    r = np.random.default_rng(3)
    k, v = r.standard_normal(d) / 3, r.standard_normal(d) / 3
    W1, W2 = 0.5 * r.standard_normal((d, dh)), 0.3 * r.standard_normal((dh, d))
    gamma, beta = 1 + 0.1 * r.standard_normal(d), 0.1 * r.standard_normal(d)
    G1, G2 = oracle.grad_mlp(k, v, W1, W2, gamma, beta)
    W1t, W2t = t(W1).requires_grad_(True), t(W2).requires_grad_(True)
    f = t_f_mlp(t(k), W1t, W2t, t(gamma), t(beta), 1e-5)
    g1, g2 = torch.autograd.grad(0.5 * ((f - t(v)) ** 2).sum(), (W1t, W2t))
    np.testing.assert_allclose(G1, g1.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(G2, g2.numpy(), rtol=1e-10, atol=1e-12)


def test_gelu_matches_torch_and_derivative_fd():
    hs = np.linspace(-6, 6, 97)
    ref = F.gelu(t(hs), approximate="none").numpy()
    ours = np.array([oracle.gelu(h) for h in hs])
    np.testing.assert_allclose(ours, ref, rtol=1e-14, atol=1e-15)
    eps = 1e-6
    fd = np.array([(oracle.gelu(h + eps) - oracle.gelu(h - eps)) / (2 * eps) for h in hs])
    der = np.array([oracle.gelu_prime(h) for h in hs])
    np.testing.assert_allclose(der, fd, atol=1e-8)


# ---------------------------------------------------------------- sequence-level pins

def _online_sgd_torch(Q, K, V, eta, W0, gamma, beta, ln, eps=1e-5):
    """Token-by-token online gradient descent (P-TTT, The Dual-Loop Structure and
    parts 2-3): W_t = W_{t-1} - eta_t grad l(W_{t-1}; x_t), then z_t = f(q_t; W_t).
    Gradients come from torch autograd."""
    B, H, T, d = Q.shape
    Z = np.zeros_like(Q)
    Wout = np.zeros((B, H, d, d))
    for bi in range(B):
        for h in range(H):
            W = t(W0[h]).clone()
            g_ = t(gamma[h]) if ln else None
            b_ = t(beta[h]) if ln else None
            for ti in range(T):
                Wr = W.clone().requires_grad_(True)
                f = t_f_linear(t(K[bi, h, ti]), Wr, g_, b_, ln, eps)
                loss = 0.5 * ((f - t(V[bi, h, ti])) ** 2).sum()
                (g,) = torch.autograd.grad(loss, Wr)
                W = W - float(eta[bi, h, ti]) * g
                Z[bi, h, ti] = t_f_linear(t(Q[bi, h, ti]), W, g_, b_, ln, eps).numpy()
            Wout[bi, h] = W.numpy()
    return Z, Wout


@pytest.mark.parametrize("ln", [False, True])
def test_b1_is_online_sgd(ln):
    Q, K, V, eta, W0, _, gamma, beta = rand_problem(2, 2, 12, 6, seed=5)
    Z, Wo = oracle.linear_primal(Q, K, V, eta, W0, gamma, beta, b=1, ln=ln)
    Zr, Wr = _online_sgd_torch(Q, K, V, eta, W0, gamma, beta, ln)
    np.testing.assert_allclose(Z, Zr, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(Wo, Wr, rtol=1e-11, atol=1e-12)


def _minibatch_gd_torch(Q, K, V, eta, W0, gamma, beta, b, ln, eps=1e-5):
    """Mini-batch rule (P-TTT part 4) via autograd of the eta-weighted loss of the
    first r tokens of each mini-batch at the mini-batch start weight: the weight
    after token t is W_m - grad_W sum_{s<=t} eta_s l_s(W_m)."""
    B, H, T, d = Q.shape
    Z = np.zeros_like(Q)
    Wout = np.zeros((B, H, d, d))
    for bi in range(B):
        for h in range(H):
            W = t(W0[h])
            g_ = t(gamma[h]) if ln else None
            b_ = t(beta[h]) if ln else None
            for m0 in range(0, T, b):
                Wm = W.clone()
                for r in range(b):
                    Wr = Wm.clone().requires_grad_(True)
                    s = slice(m0, m0 + r + 1)
                    f = t_f_linear(t(K[bi, h, s]), Wr, g_, b_, ln, eps)
                    per_tok = 0.5 * ((f - t(V[bi, h, s])) ** 2).sum(-1)
                    (g,) = torch.autograd.grad((t(eta[bi, h, s]) * per_tok).sum(), Wr)
                    W = Wm - g
                    Z[bi, h, m0 + r] = t_f_linear(t(Q[bi, h, m0 + r]), W, g_, b_, ln, eps).numpy()
            Wout[bi, h] = W.numpy()
    return Z, Wout


@pytest.mark.parametrize("ln", [False, True])
@pytest.mark.parametrize("b", [2, 4])
def test_minibatch_rule_matches_autograd_of_weighted_loss(ln, b):
    Q, K, V, eta, W0, _, gamma, beta = rand_problem(1, 2, 12, 5, seed=11)
    Z, Wo = oracle.linear_primal(Q, K, V, eta, W0, gamma, beta, b=b, ln=ln)
    Zr, Wr = _minibatch_gd_torch(Q, K, V, eta, W0, gamma, beta, b, ln)
    np.testing.assert_allclose(Z, Zr, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(Wo, Wr, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("ln", [False, True])
def test_eta_zero_gives_initial_weight(ln):
    """eta = 0: the weight never moves, so z_t = f(q_t; W0) and W_out = W0."""
    Q, K, V, eta, W0, _, gamma, beta = rand_problem(2, 3, 32, 8, seed=2)
    eta[:] = 0.0
    Z, Wo = oracle.linear_primal(Q, K, V, eta, W0, gamma, beta, b=8, ln=ln)
    for h in range(3):
        ref = t_f_linear(t(Q[:, h]), t(W0[h]), t(gamma[h]), t(beta[h]), ln, 1e-5).numpy()
        np.testing.assert_allclose(Z[:, h], ref, rtol=1e-13, atol=1e-14)
        np.testing.assert_array_equal(Wo[:, h], np.broadcast_to(W0[h], Wo[:, h].shape))


@pytest.mark.parametrize("b", [1, 3, 4, 12])
def test_linear_affine_closed_form(b):
    """No LayerNorm: each mini-batch is an affine map of the weight,
    W_{m+1} = (I - K^T E K) W_m + K^T E V, and the running weight after the
    first r tokens is the same expression over those tokens (E = diag(eta))."""
    Q, K, V, eta, W0, *_ = rand_problem(1, 1, 12, 4, seed=b)
    Z, Wo = oracle.linear_primal(Q, K, V, eta, W0, b=b, ln=False)
    W = W0[0].copy()
    I = np.eye(4)
    for m0 in range(0, 12, b):
        Wm = W
        for r in range(1, b + 1):
            Kr, Vr, Er = K[0, 0, m0:m0 + r], V[0, 0, m0:m0 + r], np.diag(eta[0, 0, m0:m0 + r])
            Wr = (I - Kr.T @ Er @ Kr) @ Wm + Kr.T @ Er @ Vr
            np.testing.assert_allclose(Z[0, 0, m0 + r - 1], Q[0, 0, m0 + r - 1] @ Wr,
                                       rtol=1e-12, atol=1e-14)
        W = Wr
    np.testing.assert_allclose(Wo[0, 0], W, rtol=1e-12, atol=1e-14)


def test_zero_initial_weight_first_minibatch_is_causal_linear_attention():
    """With W0 = 0 (the listing's init_hidden_state) and no LayerNorm, the first
    mini-batch outputs are z_t = sum_{s<=t} eta_s (q_t . k_s) v_s."""
    Q, K, V, eta, W0, *_ = rand_problem(1, 1, 8, 6, seed=4)
    W0[:] = 0.0
    Z, _ = oracle.linear_primal(Q, K, V, eta, W0, b=8, ln=False)
    q, k, v, e = Q[0, 0], K[0, 0], V[0, 0], eta[0, 0]
    A = np.tril(q @ k.T) * e[None, :]
    np.testing.assert_allclose(Z[0, 0], A @ v, rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("ln", [False, True])
@pytest.mark.parametrize("b", [1, 4, 16])
def test_primal_equals_dual(ln, b):
    Q, K, V, eta, W0, _, gamma, beta = rand_problem(2, 2, 32, 8, seed=b + 100 * ln)
    Zp, Wp = oracle.linear_primal(Q, K, V, eta, W0, gamma, beta, b=b, ln=ln)
    Zd, Wd = oracle.linear_dual(Q, K, V, eta, W0, gamma, beta, b=b, ln=ln)
    np.testing.assert_allclose(Zd, Zp, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(Wd, Wp, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("ln", [False, True])
def test_resume_invariance(ln):
    """The fast weight is the whole state: running T tokens equals running the
    first half, then the second half from the returned weight."""
    Q, K, V, eta, W0, _, gamma, beta = rand_problem(2, 2, 32, 6, seed=9)
    Z, Wo = oracle.linear_primal(Q, K, V, eta, W0, gamma, beta, b=4, ln=ln)
    h = 16
    Z1, W1 = oracle.linear_primal(Q[:, :, :h], K[:, :, :h], V[:, :, :h], eta[:, :, :h], W0,
                                  gamma, beta, b=4, ln=ln)
    Z2, W2 = oracle.linear_primal(Q[:, :, h:], K[:, :, h:], V[:, :, h:], eta[:, :, h:], W1,
                                  gamma, beta, b=4, ln=ln, w0_per_seq=True)
    np.testing.assert_allclose(np.concatenate([Z1, Z2], 2), Z, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(W2, Wo, rtol=1e-13, atol=1e-15)


def test_layernorm_scale_invariance_eps0():
    """With eps = 0, f(k; cW) = f(k; W) and Gamma(cW) = Gamma(W)/c for c > 0."""
    r = np.random.default_rng(8)
    d = 8
    k, v = r.standard_normal(d), r.standard_normal(d)
    W = r.standard_normal((d, d))
    gamma, beta = 1 + 0.1 * r.standard_normal(d), 0.1 * r.standard_normal(d)
    for c in (0.01, 3.0, 250.0):
        l1 = oracle.loss_linear(k, v, W, gamma, beta, ln=True, eps=0.0)
        l2 = oracle.loss_linear(k, v, c * W, gamma, beta, ln=True, eps=0.0)
        assert abs(l1 - l2) < 1e-12 * max(1, abs(l1))
        G1 = oracle.grad_linear(k, v, W, gamma, beta, ln=True, eps=0.0)
        G2 = oracle.grad_linear(k, v, c * W, gamma, beta, ln=True, eps=0.0)
        np.testing.assert_allclose(G2 * c, G1, rtol=1e-10, atol=1e-12)


def test_layernorm_two_features_eps0_is_frozen():
    """d = 2, eps = 0: LN(x) = gamma * (+-1, -+1) + beta is piecewise constant in
    x, so every gradient vanishes, W never moves and
    z = q + gamma * sign pattern of (qW) + beta."""
    Q, K, V, eta, W0, _, gamma, beta = rand_problem(1, 2, 16, 2, seed=21, eta_scale=0.5)
    Z, Wo = oracle.linear_primal(Q, K, V, eta, W0, gamma, beta, b=4, ln=True, eps=0.0)
    np.testing.assert_allclose(Wo[0], W0, rtol=0, atol=1e-12)
    for h in range(2):
        x = Q[0, h] @ W0[h]
        s = np.sign(x[:, 0] - x[:, 1])
        xhat = np.stack([s, -s], 1)
        np.testing.assert_allclose(Z[0, h], Q[0, h] + gamma[h] * xhat + beta[h], atol=1e-12)


# ---------------------------------------------------------------- large chunk

def test_chunk_single_chunk_closed_form():
    """T = chunk: outputs use W0 (Z = Q W0) and the weight takes one step on
    the eta-weighted sum of gradients: W0 - K^T E (K W0 - V)."""
    Q, K, V, eta, W0, *_ = rand_problem(1, 2, 16, 5, seed=31)
    Z, Wo = oracle.chunk_primal(Q, K, V, eta, W0, chunk=16)
    for h in range(2):
        np.testing.assert_allclose(Z[0, h], Q[0, h] @ W0[h], rtol=1e-13, atol=1e-15)
        E = np.diag(eta[0, h])
        ref = W0[h] - K[0, h].T @ E @ (K[0, h] @ W0[h] - V[0, h])
        np.testing.assert_allclose(Wo[0, h], ref, rtol=1e-12, atol=1e-15)


def test_chunk_affine_recursion():
    """Multi-chunk: Z_c = Q_c W_c and W_{c+1} = (I - K_c^T E K_c) W_c + K_c^T E V_c."""
    Q, K, V, eta, W0, *_ = rand_problem(1, 1, 32, 6, seed=32)
    Z, Wo = oracle.chunk_primal(Q, K, V, eta, W0, chunk=8)
    W = W0[0].copy()
    for c0 in range(0, 32, 8):
        s = slice(c0, c0 + 8)
        np.testing.assert_allclose(Z[0, 0, s], Q[0, 0, s] @ W, rtol=1e-12, atol=1e-15)
        Kc, Vc, E = K[0, 0, s], V[0, 0, s], np.diag(eta[0, 0, s])
        W = (np.eye(6) - Kc.T @ E @ Kc) @ W + Kc.T @ E @ Vc
    np.testing.assert_allclose(Wo[0, 0], W, rtol=1e-12, atol=1e-15)


def test_chunk_of_one_token_equals_apply_before_update_sgd():
    """chunk = 1: z_t = q_t W_{t-1} (read-out before the token's own step)."""
    Q, K, V, eta, W0, *_ = rand_problem(1, 1, 10, 4, seed=33)
    Z, Wo = oracle.chunk_primal(Q, K, V, eta, W0, chunk=1)
    Zu, Wu = oracle.linear_primal(Q, K, V, eta, W0, b=1, ln=False)
    # same weight trajectory; the read-outs differ by one step
    np.testing.assert_allclose(Wo, Wu, rtol=1e-13)
    W = W0[0]
    for ti in range(10):
        np.testing.assert_allclose(Z[0, 0, ti], Q[0, 0, ti] @ W, rtol=1e-12, atol=1e-15)
        k, v = K[0, 0, ti], V[0, 0, ti]
        W = W - eta[0, 0, ti] * np.outer(k, k @ W - v)


# ---------------------------------------------------------------- MLP

def _mlp_sgd_torch(Q, K, V, eta, W1, W2, gamma, beta, b, eps=1e-5):
    B, H, T, d = Q.shape
    Z = np.zeros_like(Q)
    for bi in range(B):
        for h in range(H):
            A1, A2 = t(W1[h]), t(W2[h])
            g_, b_ = t(gamma[h]), t(beta[h])
            for m0 in range(0, T, b):
                A1m, A2m = A1.clone(), A2.clone()
                for r in range(b):
                    p1, p2 = A1m.clone().requires_grad_(True), A2m.clone().requires_grad_(True)
                    s = slice(m0, m0 + r + 1)
                    f = t_f_mlp(t(K[bi, h, s]), p1, p2, g_, b_, eps)
                    per_tok = 0.5 * ((f - t(V[bi, h, s])) ** 2).sum(-1)
                    g1, g2 = torch.autograd.grad((t(eta[bi, h, s]) * per_tok).sum(), (p1, p2))
                    A1, A2 = A1m - g1, A2m - g2
                    Z[bi, h, m0 + r] = t_f_mlp(t(Q[bi, h, m0 + r]), A1, A2, g_, b_, eps).numpy()
    return Z


@pytest.mark.parametrize("b", [1, 4])
def test_mlp_minibatch_rule_matches_autograd(b):
    Q, K, V, eta, W1, W2, gamma, beta = rand_problem(1, 1, 8, 4, dh=16, seed=41, w_scale=1.0)
    Z, _, _ = oracle.mlp_primal(Q, K, V, eta, W1, W2, gamma, beta, b=b)
    Zr = _mlp_sgd_torch(Q, K, V, eta, W1, W2, gamma, beta, b)
    np.testing.assert_allclose(Z, Zr, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("b", [1, 4, 8])
def test_mlp_primal_equals_dual(b):
    Q, K, V, eta, W1, W2, gamma, beta = rand_problem(2, 2, 16, 8, dh=32, seed=b, w_scale=1.0)
    Zp, W1p, W2p = oracle.mlp_primal(Q, K, V, eta, W1, W2, gamma, beta, b=b)
    Zd, W1d, W2d = oracle.mlp_dual(Q, K, V, eta, W1, W2, gamma, beta, b=b)
    np.testing.assert_allclose(Zd, Zp, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(W1d, W1p, rtol=1e-10, atol=1e-13)
    np.testing.assert_allclose(W2d, W2p, rtol=1e-10, atol=1e-13)


def test_mlp_eta_zero():
    Q, K, V, eta, W1, W2, gamma, beta = rand_problem(1, 2, 8, 4, dh=16, seed=43)
    eta[:] = 0
    Z, W1o, W2o = oracle.mlp_primal(Q, K, V, eta, W1, W2, gamma, beta, b=4)
    for h in range(2):
        ref = t_f_mlp(t(Q[0, h]), t(W1[h]), t(W2[h]), t(gamma[h]), t(beta[h]), 1e-5).numpy()
        np.testing.assert_allclose(Z[0, h], ref, rtol=1e-13, atol=1e-14)
        np.testing.assert_array_equal(W1o[0, h], W1[h])
        np.testing.assert_array_equal(W2o[0, h], W2[h])


# ---------------------------------------------------------------- plumbing

def test_sequence_subset_and_threads_agree():
    Q, K, V, eta, W0, _, gamma, beta = rand_problem(3, 4, 16, 8, seed=51)
    Zall, Wall = oracle.linear_primal(Q, K, V, eta, W0, gamma, beta, b=4, ln=True, nthreads=1)
    Zthr, Wthr = oracle.linear_primal(Q, K, V, eta, W0, gamma, beta, b=4, ln=True, nthreads=5)
    np.testing.assert_array_equal(Zall, Zthr)
    np.testing.assert_array_equal(Wall, Wthr)
    seqs = [0, 5, 11]
    Zs, Ws = oracle.linear_primal(Q, K, V, eta, W0, gamma, beta, b=4, ln=True, seqs=seqs)
    for s in seqs:
        bi, h = divmod(s, 4)
        np.testing.assert_array_equal(Zs[bi, h], Zall[bi, h])
        np.testing.assert_array_equal(Ws[bi, h], Wall[bi, h])


def test_rejects_ragged_minibatch_where_undefined():
    """Only TTT-Linear defines a partial last mini-batch; the MLP and the
    large-chunk forms still require T to be a multiple of b."""
    Q, K, V, eta, W1, W2, gamma, beta = rand_problem(1, 1, 10, 4, dh=16)
    with pytest.raises(ValueError):
        oracle.mlp_primal(Q, K, V, eta, W1, W2, gamma, beta, b=4)
    Q, K, V, eta, W0, *_ = rand_problem(1, 1, 10, 4)
    with pytest.raises(ValueError):
        oracle.chunk_primal(Q, K, V, eta, W0, chunk=4)


@pytest.mark.parametrize("ln", [True, False])
def test_partial_last_minibatch_primal_equals_dual(ln):
    """T = 10 with b = 4: two full mini-batches and a partial one of 2 tokens;
    the token-by-token and the dual forms agree."""
    Q, K, V, eta, W0, _, gamma, beta = rand_problem(2, 2, 10, 6, seed=3)
    g, be = (gamma, beta) if ln else (None, None)
    Zp, Wp = oracle.linear_primal(Q, K, V, eta, W0, g, be, b=4, ln=ln)
    Zd, Wd = oracle.linear_dual(Q, K, V, eta, W0, g, be, b=4, ln=ln)
    np.testing.assert_allclose(Zd, Zp, rtol=0, atol=1e-12)
    np.testing.assert_allclose(Wd, Wp, rtol=0, atol=1e-12)


def test_partial_single_minibatch_is_one_batch_of_all_tokens():
    """T = 10 < b = 16: the only mini-batch holds all 10 tokens, the same
    computation as b = 10."""
    Q, K, V, eta, W0, _, gamma, beta = rand_problem(1, 2, 10, 6, seed=4)
    Z16, W16 = oracle.linear_primal(Q, K, V, eta, W0, gamma, beta, b=16, ln=True)
    Z10, W10 = oracle.linear_primal(Q, K, V, eta, W0, gamma, beta, b=10, ln=True)
    np.testing.assert_array_equal(Z16, Z10)
    np.testing.assert_array_equal(W16, W10)


@pytest.mark.parametrize("ln", [True, False])
def test_partial_minibatch_equals_zero_step_padding(ln):
    """A partial last mini-batch equals padding the sequence to a multiple of
    b with tokens of step size 0 (any q, k, v) under the full-batch rule: those
    tokens change no weight, and the real tokens' outputs are the same."""
    Q, K, V, eta, W0, _, gamma, beta = rand_problem(1, 2, 12, 6, seed=5)
    eta = eta.copy()
    eta[..., 10:] = 0.0
    g, be = (gamma, beta) if ln else (None, None)
    Zpad, Wpad = oracle.linear_primal(Q, K, V, eta, W0, g, be, b=4, ln=ln)
    Zr, Wr = oracle.linear_primal(Q[:, :, :10].copy(), K[:, :, :10].copy(), V[:, :, :10].copy(),
                                  eta[:, :, :10].copy(), W0, g, be, b=4, ln=ln)
    np.testing.assert_allclose(Zr, Zpad[:, :, :10], rtol=0, atol=1e-13)
    np.testing.assert_allclose(Wr, Wpad, rtol=0, atol=1e-13)
