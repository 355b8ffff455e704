"""Affine segment maps of the large-chunk TTT update (and of TTT-Linear without
LayerNorm), for the tests of the sequence-parallel forward.

TEST INFRASTRUCTURE ONLY: imported by the test suite, never by the library.
It shares nothing with the CUDA library and does not import it.

Source: "Test-Time Training Done Right" (abstract). The tokens of chunk c read
out with W_c, then W_c takes one gradient step on the chunk's eta-weighted
reconstruction loss 1/2 sum_t eta_t ||k_t W - v_t||^2. Its gradient at W_c is
K_c^T diag(eta_c) (K_c W_c - V_c), so the step is affine in W_c:

    W_{c+1} = (I - A_c) W_c + B_c,   A_c = K_c^T diag(eta_c) K_c,
                                     B_c = K_c^T diag(eta_c) V_c.

(Reading: the pages give the gradient step; the affine form is that step
expanded.) The same holds for TTT-Linear without LayerNorm, whose mini-batch
of b tokens takes every gradient at the mini-batch's starting weight ("Test-Time
Training: Linear Complexity Beyond Attention", "Key Architectural Mechanics of
TTT-Linear", part 4), with chunk = b.

A run of consecutive chunks therefore maps its starting weight to its final
weight by W -> M W + N, where M is the ordered product of the (I - A_c) and N
is the run's final weight from W = 0. Doing run 1 then run 2 is the map
(M2 M1, M2 N1 + N2). Everything is float64 numpy, one sequence at a time.
Conventions as in ttt_oracle.c: row form x = k W with W[d_in][d_out],
K/V [B][H][T][d], eta [B][H][T], W0 [H][d][d] or [B][H][d][d].
"""
from __future__ import annotations

import numpy as np


def chunk_step(K_c, V_c, eta_c):
    """(A_c, B_c) of one chunk of one sequence: K_c, V_c [n][d], eta_c [n]."""
    K_c = np.asarray(K_c, dtype=np.float64)
    V_c = np.asarray(V_c, dtype=np.float64)
    e = np.asarray(eta_c, dtype=np.float64)[:, None]
    return K_c.T @ (e * K_c), K_c.T @ (e * V_c)


def segment_map(K, V, eta, *, chunk):
    """(M, N), each [B][H][d][d], of the chunks of K, V, eta [B][H][T(,d)]
    taken in order: starting from M = I, N = 0, every chunk does
    M <- M - A_c M and N <- N - A_c N + B_c. T must be a multiple of chunk."""
    B, H, T, d = K.shape
    if T % chunk:
        raise ValueError("T must be a multiple of chunk")
    M = np.zeros((B, H, d, d))
    N = np.zeros((B, H, d, d))
    for bb in range(B):
        for hh in range(H):
            m, n = np.eye(d), np.zeros((d, d))
            for c0 in range(0, T, chunk):
                sl = slice(c0, c0 + chunk)
                A, Bc = chunk_step(K[bb, hh, sl], V[bb, hh, sl], eta[bb, hh, sl])
                m = m - A @ m
                n = n - A @ n + Bc
            M[bb, hh], N[bb, hh] = m, n
    return M, N


def apply_map(M, N, W):
    """M W + N, batched over the leading axes."""
    return np.einsum("...ij,...jk->...ik", M, W) + N


def compose(first, second):
    """The map of `first` followed by `second` (each an (M, N) pair)."""
    M1, N1 = first
    M2, N2 = second
    return np.einsum("...ij,...jk->...ik", M2, M1), apply_map(M2, N2, N1)


def prefix_weights(maps, W0):
    """Starting weight of every segment and the final weight: W_in[0] = W0,
    W_in[j+1] = M_j W_in[j] + N_j; returns (list of W_in, W_end). maps is a
    list of (M, N) pairs [B][H][d][d] in sequence order; W0 is [B][H][d][d]."""
    W = np.asarray(W0, dtype=np.float64)
    W_in = []
    for M, N in maps:
        W_in.append(W)
        W = apply_map(M, N, W)
    return W_in, W
