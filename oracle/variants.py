"""Two variants of the TTT-Linear forward that the pages name, written out for
the tests (they come before any kernel that implements them).

TEST INFRASTRUCTURE ONLY: imported by the test suite, never by the library.
It shares nothing with the CUDA library and does not import it.

1. L2-normalised keys. The PyTorch listing on "Test-Time Training: Linear
   Complexity Beyond Attention" scales each key to unit Euclidean length
   before the inner prediction and its gradient; the query is used as given.
   Reading: the normalised key takes the key's place everywhere the inner
   loss and its gradient use it, in every form (TTT-Linear with or without
   LayerNorm, any mini-batch, large chunk); the read-out uses q as given. The
   scaling is k / max(||k||_2, 1e-12), the listing's normalisation defaults.
   The variant is therefore the plain forward applied to normalised keys, and
   that composition is what the oracle computes.

2. Several inner gradient steps per token. "How to Master Test-Time Training
   for LLMs", "How TTT Layers Actually Work": at each token the layer runs one
   or more gradient-descent steps on its reconstruction loss. Reading: online
   updates (b = 1); at token t the weight takes n steps
   W <- W - eta_t * grad l_t(W), each gradient at the weight the previous
   step left, then the token reads out z_t = f(q_t; W). With n = 1 this is the
   plain b = 1 forward.

Conventions as in ttt_oracle.c: row form x = k W with W[d_in][d_out],
Q/K/V [B][H][T][d], eta [B][H][T], W0 [H][d][d] (or [B][H][d][d]),
gamma/beta [H][d], LayerNorm eps 1e-5 with the biased variance. float64.
"""
from __future__ import annotations

import numpy as np

from . import LN_EPS, grad_linear

L2_EPS = 1e-12


def normalize_keys(K):
    """Every key row divided by max(||k||_2, 1e-12)."""
    K = np.asarray(K, dtype=np.float64)
    n = np.sqrt((K * K).sum(axis=-1, keepdims=True))
    return K / np.maximum(n, L2_EPS)


def _readout(q, W, gamma, beta, ln, eps):
    x = q @ W
    if not ln:
        return x
    mu = x.mean()
    var = ((x - mu) ** 2).mean()
    return q + gamma * (x - mu) / np.sqrt(var + eps) + beta


def linear_multistep(Q, K, V, eta, W0, gamma=None, beta=None, *, n_steps, ln, w0_per_seq=False,
                     eps=LN_EPS):
    """TTT-Linear, online, n_steps gradient steps per token before its
    read-out. The gradient of l = 1/2 ||f(k; W) - v||^2 at W is the C
    oracle's closed form (grad_linear). Returns (Z, W_out), float64."""
    Q, K, V = (np.asarray(a, dtype=np.float64) for a in (Q, K, V))
    eta = np.asarray(eta, dtype=np.float64)
    B, H, T, d = Q.shape
    Z = np.zeros((B, H, T, d))
    W_out = np.zeros((B, H, d, d))
    for b in range(B):
        for h in range(H):
            W = np.array(W0[b, h] if w0_per_seq else W0[h], dtype=np.float64)
            g = None if gamma is None else np.asarray(gamma[h], dtype=np.float64)
            be = None if beta is None else np.asarray(beta[h], dtype=np.float64)
            for t in range(T):
                for _ in range(n_steps):
                    W = W - eta[b, h, t] * grad_linear(K[b, h, t], V[b, h, t], W, g, be, ln=ln,
                                                       eps=eps)
                Z[b, h, t] = _readout(Q[b, h, t], W, g, be, ln, eps)
            W_out[b, h] = W
    return Z, W_out
