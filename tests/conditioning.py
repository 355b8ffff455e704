"""Conditioning of the recurrence itself, measured with the oracle alone.

The inner loop is a nonlinear recurrence over thousands of steps; with a large
enough step size it amplifies small differences. Then no finite-precision
implementation (fp32 included) can track the exact result past some token,
and parity is only meaningful before it. `conditioned_horizon` measures that
token per sequence: the oracle runs on the inputs and on the inputs times
(1 + noise N(0,1)), and the horizon is the first mini-batch boundary after
which the two differ by more than `rel` of max|Z| (T if they never do).
"""
from __future__ import annotations

import dataclasses

import numpy as np

import oracle


def run_oracle(inp, seqs=None):
    wl = inp.wl
    if wl.kind == "linear":
        return oracle.linear_primal(inp.Q, inp.K, inp.V, inp.eta, inp.W1, inp.gamma, inp.beta,
                                    b=wl.b, ln=wl.ln, seqs=seqs)
    if wl.kind == "mlp":
        return oracle.mlp_primal(inp.Q, inp.K, inp.V, inp.eta, inp.W1, inp.W2, inp.gamma,
                                 inp.beta, b=wl.b, seqs=seqs)
    return oracle.chunk_primal(inp.Q, inp.K, inp.V, inp.eta, inp.W1, chunk=wl.b, seqs=seqs)


def perturbed(inp, noise=1e-7, seed=1):
    rng = np.random.default_rng(seed)
    p = lambda a: a.astype(np.float64) * (1.0 + noise * rng.standard_normal(a.shape))
    return dataclasses.replace(inp, Q=p(inp.Q), K=p(inp.K), V=p(inp.V))


def divergence(inp, seqs=None, ref=None, noise=1e-7):
    """Per sequence and token: max over d of |Z - Z_perturbed| / max|Z|.
    Returns (divergence [n_seq, T], oracle outputs on the unperturbed inputs)."""
    wl = inp.wl
    ref = ref if ref is not None else run_oracle(inp, seqs)
    alt = run_oracle(perturbed(inp, noise), seqs)
    n = wl.B * wl.H
    rows = np.arange(n) if seqs is None else np.asarray(seqs)
    Za = ref[0].reshape(n, wl.T, wl.d)[rows]
    Zb = alt[0].reshape(n, wl.T, wl.d)[rows]
    return np.abs(Za - Zb).max(axis=-1) / np.abs(Za).max(), ref


def conditioned_horizon(inp, seqs=None, rel=1e-6, noise=1e-7):
    """(horizon per listed sequence in tokens, oracle outputs)."""
    wl = inp.wl
    dev, ref = divergence(inp, seqs, noise=noise)
    bad = dev > rel
    h = np.where(bad.any(axis=1), bad.argmax(axis=1), wl.T)
    return (h // wl.b) * wl.b, ref
