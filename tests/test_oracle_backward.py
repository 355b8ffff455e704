"""Pins of the backward oracle (oracle/backward.py) to things other than itself:
its forwards against the C oracle's forwards, its outer gradients against
central finite differences (torch.autograd.gradcheck), and special cases the
method fixes (eta = 0 freezes the weight, so Z cannot depend on K or V; a
single large chunk reads out with W0 alone)."""
import os
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from oracle import backward as ob  # noqa: E402


def _inputs(seed, B, H, T, d, *, w0_per_seq=False, eta_scale=0.1):
    r = np.random.default_rng(seed)
    Q, K, V = (r.standard_normal((B, H, T, d)) for _ in range(3))
    eta = eta_scale * r.uniform(0.2, 1.0, (B, H, T))
    W0 = r.standard_normal((B, H, d, d) if w0_per_seq else (H, d, d)) / np.sqrt(d)
    gamma = 1.0 + 0.2 * r.standard_normal((H, d))
    beta = 0.2 * r.standard_normal((H, d))
    return Q, K, V, eta, W0, gamma, beta


@pytest.mark.parametrize("ln,b,w0_per_seq", [(True, 4, False), (False, 4, False), (True, 1, True),
                                             (True, 8, False)])
def test_forward_matches_c_oracle(ln, b, w0_per_seq):
    Q, K, V, eta, W0, gamma, beta = _inputs(1, 2, 2, 16, 8, w0_per_seq=w0_per_seq)
    Z, Wo = ob.linear_forward_np(Q, K, V, eta, W0, gamma, beta, b=b, ln=ln)
    Zc, Woc = oracle.linear_primal(Q, K, V, eta, W0, gamma if ln else None, beta if ln else None,
                                   b=b, ln=ln, w0_per_seq=w0_per_seq)
    assert np.abs(Z - Zc).max() <= 1e-12 * max(1.0, np.abs(Zc).max())
    assert np.abs(Wo - Woc).max() <= 1e-12 * max(1.0, np.abs(Woc).max())


@pytest.mark.parametrize("ln", [True, False])
def test_inner_gradient_matches_c_closed_form(ln):
    """The autograd inner gradient used by the oracle's forward equals the C
    oracle's closed-form k^T dl/dx."""
    r = np.random.default_rng(5)
    d = 6
    k, v = r.standard_normal(d), r.standard_normal(d)
    W = r.standard_normal((d, d)) / np.sqrt(d)
    gamma, beta = 1.0 + 0.3 * r.standard_normal(d), 0.3 * r.standard_normal(d)
    Wt = torch.tensor(W, requires_grad=True)
    kt, vt = torch.tensor(k), torch.tensor(v)
    x = kt @ Wt
    f = kt + torch.nn.functional.layer_norm(x, (d,), eps=ob.LN_EPS) * torch.tensor(gamma) \
        + torch.tensor(beta) if ln else x
    g = torch.autograd.grad(0.5 * ((f - vt) ** 2).sum(), Wt)[0].numpy()
    Gc = oracle.grad_linear(k, v, W, gamma if ln else None, beta if ln else None, ln=ln)
    assert np.abs(g - Gc).max() <= 1e-12 * np.abs(Gc).max()


@pytest.mark.parametrize("ln", [True, False])
def test_gradients_match_finite_differences(ln):
    """gradcheck: autograd through the unrolled inner loop (a gradient of a
    gradient) against central differences, for every input at once."""
    Q, K, V, eta, W0, gamma, beta = _inputs(2, 1, 1, 6, 3, eta_scale=0.5)
    ts = [torch.tensor(a, requires_grad=True) for a in (Q, K, V, eta, W0, gamma, beta)]
    r = np.random.default_rng(3)
    dZ = torch.tensor(r.standard_normal(Q.shape))
    dW = torch.tensor(r.standard_normal((1, 1, 3, 3)))

    def fn(*a):
        Z, Wo = ob.linear_forward(*a, b=2, ln=ln)
        return (Z * dZ).sum() + (Wo * dW).sum()

    inputs = tuple(ts if ln else ts[:5])
    if not ln:
        g0, b0 = ts[5].detach(), ts[6].detach()
        fn_noln = lambda *a: fn(*a, g0, b0)  # noqa: E731
        assert torch.autograd.gradcheck(fn_noln, inputs, eps=1e-6, atol=1e-7, rtol=1e-6)
    else:
        assert torch.autograd.gradcheck(fn, inputs, eps=1e-6, atol=1e-7, rtol=1e-6)


def test_linear_grads_equal_gradcheck_function():
    """linear_grads (the entry the GPU tests use) returns what autograd of the
    same scalar gives, key by key, and a zero dW_out equals no dW_out."""
    Q, K, V, eta, W0, gamma, beta = _inputs(4, 1, 2, 8, 4)
    r = np.random.default_rng(6)
    dZ = r.standard_normal(Q.shape)
    g1 = ob.linear_grads(Q, K, V, eta, W0, gamma, beta, dZ, None, b=4, ln=True)
    g2 = ob.linear_grads(Q, K, V, eta, W0, gamma, beta, dZ, np.zeros((1, 2, 4, 4)), b=4, ln=True)
    for n in g1:
        assert np.array_equal(g1[n], g2[n])
    assert set(g1) == {"Q", "K", "V", "eta", "W0", "gamma", "beta"}


def test_eta_zero_freezes_weight_so_k_and_v_get_no_gradient():
    """With eta = 0 the weight never moves, so Z depends on Q, W0, gamma and beta
    only: dK = dV = 0 exactly, dW_out flows straight to dW0, and deta is the
    first-order effect of each token's step (nonzero)."""
    Q, K, V, eta, W0, gamma, beta = _inputs(7, 1, 1, 8, 4, eta_scale=0.0)
    r = np.random.default_rng(8)
    dZ = r.standard_normal(Q.shape)
    dW = r.standard_normal((1, 1, 4, 4))
    g = ob.linear_grads(Q, K, V, eta, W0, gamma, beta, dZ * 0.0, dW, b=4, ln=True)
    assert np.abs(g["K"]).max() == 0.0 and np.abs(g["V"]).max() == 0.0
    assert np.allclose(g["W0"][0], dW[0, 0], rtol=0, atol=1e-15)
    g = ob.linear_grads(Q, K, V, eta, W0, gamma, beta, dZ, None, b=4, ln=True)
    assert np.abs(g["K"]).max() == 0.0 and np.abs(g["V"]).max() == 0.0
    assert np.abs(g["eta"]).max() > 0.0


# ------------------------------------------------------------ large-chunk form

def test_chunk_forward_matches_c_oracle():
    Q, K, V, eta, W0, _, _ = _inputs(9, 2, 2, 24, 6, eta_scale=0.05)
    Z, Wo = ob.chunk_forward_np(Q, K, V, eta, W0, chunk=8)
    Zc, Woc = oracle.chunk_primal(Q, K, V, eta, W0, chunk=8)
    assert np.abs(Z - Zc).max() <= 1e-12 * max(1.0, np.abs(Zc).max())
    assert np.abs(Wo - Woc).max() <= 1e-12 * max(1.0, np.abs(Woc).max())


def test_chunk_gradients_match_finite_differences():
    Q, K, V, eta, W0, _, _ = _inputs(10, 1, 1, 6, 3, eta_scale=0.4)
    ts = [torch.tensor(a, requires_grad=True) for a in (Q, K, V, eta, W0)]
    r = np.random.default_rng(11)
    dZ = torch.tensor(r.standard_normal(Q.shape))
    dW = torch.tensor(r.standard_normal((1, 1, 3, 3)))

    def fn(*a):
        Z, Wo = ob.chunk_forward(*a, chunk=2)
        return (Z * dZ).sum() + (Wo * dW).sum()

    assert torch.autograd.gradcheck(fn, tuple(ts), eps=1e-6, atol=1e-7, rtol=1e-6)


def test_chunk_single_chunk_closed_form():
    """One chunk: Z = Q W0 exactly, so with dW_out = 0 the gradients are
    dQ = dZ W0^T, dW0 = Q^T dZ and nothing reaches K, V or eta."""
    Q, K, V, eta, W0, _, _ = _inputs(12, 1, 1, 8, 4)
    dZ = np.random.default_rng(13).standard_normal(Q.shape)
    g = ob.chunk_grads(Q, K, V, eta, W0, dZ, None, chunk=8)
    np.testing.assert_allclose(g["Q"][0, 0], dZ[0, 0] @ W0[0].T, rtol=0, atol=1e-13)
    np.testing.assert_allclose(g["W0"][0], Q[0, 0].T @ dZ[0, 0], rtol=0, atol=1e-13)
    for k in ("K", "V", "eta"):
        assert np.abs(g[k]).max() == 0.0


def test_chunk_recurrences_and_s_form_reproduce_the_oracle():
    """The readings the large-chunk backward kernels compute, against the
    autograd oracle: W_c by the forward recurrence W - A_c W + B_c, Om_{c+1}
    by the reverse one Om - A_c Om + Q_c^T dZ_c (dW0 = Om_0), and per chunk
    dK = -diag(eta) (K S - V Om^T) with S = W Om^T + Om W^T, which equals
    -diag(eta) (R Om^T + P W^T) with R = K W - V, P = K Om; dV = diag(eta) P,
    deta = -P . R, dQ = dZ W^T. Each slice of columns of W or Om also evolves
    alone (the scans split the columns over blocks)."""
    B, H, T, d, C = 1, 2, 24, 5, 8
    Q, K, V, eta, W0, _, _ = _inputs(21, B, H, T, d, eta_scale=0.2)
    r = np.random.default_rng(22)
    dZ = r.standard_normal(Q.shape)
    dW = r.standard_normal((B, H, d, d))
    g = ob.chunk_grads(Q, K, V, eta, W0, dZ, dW, chunk=C)
    for h in range(H):
        q, k, v, e, dz = Q[0, h], K[0, h], V[0, h], eta[0, h], dZ[0, h]
        cs = [slice(c0, c0 + C) for c0 in range(0, T, C)]
        A = [k[c].T @ (e[c, None] * k[c]) for c in cs]
        Bc = [k[c].T @ (e[c, None] * v[c]) for c in cs]
        Ws, W = [], W0[h].copy()
        for i in range(len(cs)):
            Ws.append(W)
            W = W - A[i] @ W + Bc[i]
        Oms, Om = [None] * len(cs), dW[0, h].copy()
        for i in reversed(range(len(cs))):
            Oms[i] = Om
            Om = Om - A[i] @ Om + q[cs[i]].T @ dz[cs[i]]
        tol = 1e-10 * max(1.0, np.abs(g["W0"]).max())
        assert np.abs(Om - g["W0"][h]).max() <= tol
        # the first two columns alone follow the same recurrence
        Om2 = dW[0, h][:, :2].copy()
        for i in reversed(range(len(cs))):
            Om2 = Om2 - A[i] @ Om2 + (q[cs[i]].T @ dz[cs[i]])[:, :2]
        assert np.abs(Om2 - Om[:, :2]).max() <= tol
        for i, c in enumerate(cs):
            Wc, Oc = Ws[i], Oms[i]
            R, P = k[c] @ Wc - v[c], k[c] @ Oc
            S = Wc @ Oc.T + Oc @ Wc.T
            dk_s = -e[c, None] * (k[c] @ S - v[c] @ Oc.T)
            dk_rp = -e[c, None] * (R @ Oc.T + P @ Wc.T)
            np.testing.assert_allclose(dk_s, dk_rp, rtol=0, atol=1e-12 * np.abs(dk_rp).max())
            np.testing.assert_allclose(dk_s, g["K"][0, h, c], rtol=0, atol=1e-10 * np.abs(g["K"]).max())
            np.testing.assert_allclose(e[c, None] * P, g["V"][0, h, c], rtol=0,
                                       atol=1e-10 * np.abs(g["V"]).max())
            np.testing.assert_allclose(-(P * R).sum(1), g["eta"][0, h, c], rtol=0,
                                       atol=1e-10 * np.abs(g["eta"]).max())
            np.testing.assert_allclose(dz[c] @ Wc.T, g["Q"][0, h, c], rtol=0,
                                       atol=1e-10 * np.abs(g["Q"]).max())


# ------------------------------------------------------------ TTT-MLP form

def _mlp_inputs(seed, B, H, T, d, dh, eta_scale=0.1):
    r = np.random.default_rng(seed)
    Q, K, V = (r.standard_normal((B, H, T, d)) for _ in range(3))
    eta = eta_scale * r.uniform(0.2, 1.0, (B, H, T))
    W1 = 0.3 * r.standard_normal((H, d, dh)) / np.sqrt(d)
    W2 = 0.3 * r.standard_normal((H, dh, d)) / np.sqrt(dh)
    gamma, beta = 1.0 + 0.2 * r.standard_normal((H, d)), 0.2 * r.standard_normal((H, d))
    return Q, K, V, eta, W1, W2, gamma, beta


@pytest.mark.parametrize("b", [1, 4])
def test_mlp_forward_matches_c_oracle(b):
    args = _mlp_inputs(21, 2, 2, 8, 4, 16)
    Z, W1, W2 = ob.mlp_forward_np(*args, b=b)
    Zc, W1c, W2c = oracle.mlp_primal(*args, b=b)
    for x, y in ((Z, Zc), (W1, W1c), (W2, W2c)):
        assert np.abs(x - y).max() <= 1e-12 * max(1.0, np.abs(y).max())


def test_mlp_gradients_match_finite_differences():
    args = _mlp_inputs(22, 1, 1, 4, 2, 4, eta_scale=0.5)
    ts = [torch.tensor(a, requires_grad=True) for a in args]
    r = np.random.default_rng(23)
    dZ = torch.tensor(r.standard_normal(args[0].shape))
    dW1 = torch.tensor(r.standard_normal((1, 1, 2, 4)))

    def fn(*a):
        Z, W1, W2 = ob.mlp_forward(*a, b=2)
        return (Z * dZ).sum() + (W1 * dW1).sum() + W2.sum()

    assert torch.autograd.gradcheck(fn, tuple(ts), eps=1e-6, atol=1e-7, rtol=1e-6)
