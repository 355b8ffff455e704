"""Pins of the variant oracles (oracle/variants.py) to things other than
themselves.

L2-normalised keys: every normalised key has unit length; the variant's result
does not change when any key is scaled by a positive factor of its own (the
plain forward's does); a zero key stays zero.

Several steps per token: n = 1 is the C oracle's b = 1 forward; n steps at
token t equal the C oracle's b = 1 forward on the sequence with token t
repeated n times (its keys and values, each copy with the same eta), read out
after the last copy; for f(k) = k W the n-step update has the closed form
W_n = W_0 - k^T (k W_0 - v) (1 - rho^n) / ||k||^2 with rho = 1 - eta ||k||^2,
and for large n it fits the token exactly (k W_n -> v)."""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from oracle import variants  # noqa: E402


def _inputs(seed, B, H, T, d, eta_scale=0.05):
    r = np.random.default_rng(seed)
    Q, K, V = (r.standard_normal((B, H, T, d)) for _ in range(3))
    eta = eta_scale * r.uniform(0.2, 1.0, (B, H, T))
    W0 = r.standard_normal((H, d, d)) / np.sqrt(d)
    gamma = 1.0 + 0.2 * r.standard_normal((H, d))
    beta = 0.2 * r.standard_normal((H, d))
    return Q, K, V, eta, W0, gamma, beta


def _close(a, b, tol=1e-11):
    return np.abs(a - b).max() <= tol * max(1.0, np.abs(b).max())


def test_normalized_keys_have_unit_length_and_zero_stays_zero():
    K = np.random.default_rng(1).standard_normal((2, 3, 5, 7))
    K[0, 0, 0] = 0.0
    Kn = variants.normalize_keys(K)
    n = np.sqrt((Kn * Kn).sum(-1))
    assert np.all(Kn[0, 0, 0] == 0.0)
    n[0, 0, 0] = 1.0
    assert np.abs(n - 1.0).max() < 1e-15


@pytest.mark.parametrize("ln,b", [(True, 4), (False, 1), (False, 8)])
def test_normalized_key_variant_is_invariant_to_key_scale(ln, b):
    """Per-token positive scales of the keys leave the variant unchanged; the
    plain forward changes (so the normalisation is not a no-op)."""
    Q, K, V, eta, W0, gamma, beta = _inputs(2, 2, 2, 16, 6)
    c = np.random.default_rng(3).uniform(0.3, 3.0, K.shape[:3])[..., None]
    args = dict(b=b, ln=ln)
    g, be = (gamma, beta) if ln else (None, None)
    Z1, W1 = oracle.linear_primal(Q, variants.normalize_keys(K), V, eta, W0, g, be, **args)
    Z2, W2 = oracle.linear_primal(Q, variants.normalize_keys(c * K), V, eta, W0, g, be, **args)
    assert _close(Z1, Z2) and _close(W1, W2)
    Z3, _ = oracle.linear_primal(Q, c * K, V, eta, W0, g, be, **args)
    Z4, _ = oracle.linear_primal(Q, K, V, eta, W0, g, be, **args)
    assert not _close(Z3, Z4, 1e-6)


@pytest.mark.parametrize("ln", [True, False])
def test_one_step_is_the_b1_forward(ln):
    Q, K, V, eta, W0, gamma, beta = _inputs(4, 1, 2, 10, 5)
    g, be = (gamma, beta) if ln else (None, None)
    Z, W = variants.linear_multistep(Q, K, V, eta, W0, g, be, n_steps=1, ln=ln)
    Zc, Wc = oracle.linear_primal(Q, K, V, eta, W0, g, be, b=1, ln=ln)
    assert _close(Z, Zc) and _close(W, Wc)


@pytest.mark.parametrize("ln,n", [(True, 2), (True, 3), (False, 4)])
def test_n_steps_equal_the_b1_forward_on_repeated_tokens(ln, n):
    Q, K, V, eta, W0, gamma, beta = _inputs(5, 2, 1, 8, 4)
    g, be = (gamma, beta) if ln else (None, None)
    Z, W = variants.linear_multistep(Q, K, V, eta, W0, g, be, n_steps=n, ln=ln)
    rep = lambda a: np.repeat(a, n, axis=2)  # noqa: E731
    Zr, Wr = oracle.linear_primal(rep(Q), rep(K), rep(V), rep(eta), W0, g, be, b=1, ln=ln)
    assert _close(Z, Zr[:, :, n - 1::n]) and _close(W, Wr)


def test_linear_n_steps_closed_form_and_exact_fit():
    r = np.random.default_rng(6)
    d = 5
    k, v = r.standard_normal(d), r.standard_normal(d)
    W0 = r.standard_normal((d, d)) / np.sqrt(d)
    eta = 0.7 / (k @ k)                     # rho = 0.3
    one = lambda a: a.reshape(1, 1, 1, -1)  # noqa: E731
    for n in (1, 2, 5):
        _, W = variants.linear_multistep(one(k), one(k), one(v), np.full((1, 1, 1), eta),
                                         W0[None], n_steps=n, ln=False)
        rho = 1.0 - eta * (k @ k)
        closed = W0 - np.outer(k, k @ W0 - v) * (1.0 - rho ** n) / (k @ k)
        assert _close(W[0, 0], closed, 1e-13)
    _, W = variants.linear_multistep(one(k), one(k), one(v), np.full((1, 1, 1), eta), W0[None],
                                     n_steps=60, ln=False)
    assert np.abs(k @ W[0, 0] - v).max() < 1e-12 * np.abs(v).max()


def test_listing_recurrence_in_column_form():
    """An independent restatement of the per-token recurrence the PyTorch
    listing on "Test-Time Training: Linear Complexity Beyond Attention" runs
    (column form, prediction W k on a unit-length key, error W k - v,
    W <- W - lr (W k - v) k^T, read-out W q after the update, no LayerNorm
    inside the loss), against the oracle's b = 1 path on normalised keys with
    the weight transposed to the row form."""
    r = np.random.default_rng(12)
    d, T, lr = 4, 6, 0.05
    q, k, v = (r.standard_normal((T, d)) for _ in range(3))
    Wc = r.standard_normal((d, d)) * 0.3          # column form: prediction Wc @ k
    W = Wc.copy()
    zs = []
    for t in range(T):
        kn = k[t] / np.linalg.norm(k[t])
        W = W - lr * np.outer(W @ kn - v[t], kn)
        zs.append(W @ q[t])
    one = lambda a: a.reshape(1, 1, T, d)  # noqa: E731
    Zr, Wr = oracle.linear_primal(one(q), variants.normalize_keys(one(k)), one(v),
                                  np.full((1, 1, T), lr), Wc.T[None], b=1, ln=False)
    assert _close(Zr[0, 0], np.array(zs)) and _close(Wr[0, 0], W.T)
