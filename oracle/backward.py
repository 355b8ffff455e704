"""Outer gradients of the TTT-Linear layer, of TTT-MLP and of large-chunk TTT
(their backward passes), for the tests.

TEST INFRASTRUCTURE ONLY: imported by the test suite, never by the library.
It shares nothing with the CUDA library and does not import it.

The forward is written the way the pages define it, one token at a time, in
float64 with plain PyTorch CPU ops (sources, all on "Test-Time Training:
Linear Complexity Beyond Attention"):
  - "The Dual-Loop Structure": the inner loop is gradient descent on the fast
    weight with the self-supervised loss;
  - "Key Architectural Mechanics of TTT-Linear", parts 1-3: loss
    l(W; k, v) = 1/2 ||f(k; W) - v||^2 with f(k; W) = k W, or k + LN(k W)
    with the LayerNorm's gamma and beta; the read-out after the token's update,
    z_t = f(q_t; W_t), followed (with LayerNorm) by q + LN(.) gamma + beta;
  - part 4 "Mini-Batch Parallelism": inside a mini-batch every token's
    gradient is taken at the mini-batch's starting weight W_m, and token t
    reads out with W_m - sum_{s<=t} eta_s grad l_s(W_m).
The inner gradient is literally torch.autograd.grad of l at W_m (kept in the
graph), so the inner step is a gradient step by construction; the outer
gradients of  sum(Z * dZ) + sum(W_out * dW_out)  then come from autograd
through the whole unrolled loop. Conventions as in ttt_oracle.c: row form
x = k W with W[d_in][d_out], Q/K/V/Z [B][H][T][d], eta [B][H][T], W0 [H][d][d]
(or [B][H][d][d]), gamma/beta [H][d], LayerNorm eps 1e-5 with biased variance.
The large-chunk form (chunk_forward) is written the same way from "Test-Time
Training Done Right" (abstract): apply with the chunk's starting weight, then
one gradient step on the chunk's eta-weighted loss.
"""
from __future__ import annotations

import numpy as np
import torch
import torch.nn.functional as F

LN_EPS = 1e-5


def _t(x, grad=True):
    t = torch.as_tensor(np.asarray(x, dtype=np.float64)).clone()
    return t.requires_grad_(grad)


def linear_forward(Q, K, V, eta, W0, gamma, beta, *, b, ln, eps=LN_EPS):
    """Z [B,H,T,d] and W_out [B,H,d,d] as float64 tensors in an autograd graph.
    Every argument is a float64 tensor; W0 is [H,d,d] or [B,H,d,d]."""
    B, H, T, d = Q.shape
    W = W0.expand(B, H, d, d) if W0.dim() == 3 else W0
    g = gamma.view(1, H, d) if ln else None
    be = beta.view(1, H, d) if ln else None

    def f(k, Wt):
        x = torch.einsum("bhi,bhij->bhj", k, Wt)
        if not ln:
            return x
        return k + F.layer_norm(x, (d,), eps=eps) * g + be

    Z = []
    for m0 in range(0, T, b):
        Wm = W
        for t in range(m0, m0 + b):
            k, v = K[:, :, t], V[:, :, t]
            loss = 0.5 * ((f(k, Wm) - v) ** 2).sum()  # sum over (B, H): each term has its own W_m
            grad = torch.autograd.grad(loss, Wm, create_graph=True)[0]
            W = W - eta[:, :, t, None, None] * grad
            q = Q[:, :, t]
            x = torch.einsum("bhi,bhij->bhj", q, W)
            Z.append(q + F.layer_norm(x, (d,), eps=eps) * g + be if ln else x)
    return torch.stack(Z, dim=2), W


def linear_grads(Q, K, V, eta, W0, gamma, beta, dZ, dW_out=None, *, b, ln, eps=LN_EPS):
    """Gradients of L = sum(Z * dZ) + sum(W_out * dW_out) with respect to every
    input, as float64 numpy arrays: dict with keys Q, K, V, eta, W0 and (with
    LayerNorm) gamma, beta. Inputs are numpy arrays (any float dtype)."""
    H, d = Q.shape[1], Q.shape[3]
    if gamma is None:
        gamma = np.ones((H, d))
    if beta is None:
        beta = np.zeros((H, d))
    ts = {n: _t(a) for n, a in dict(Q=Q, K=K, V=V, eta=eta, W0=W0, gamma=gamma, beta=beta).items()}
    Z, Wo = linear_forward(ts["Q"], ts["K"], ts["V"], ts["eta"], ts["W0"], ts["gamma"],
                           ts["beta"], b=b, ln=ln, eps=eps)
    L = (Z * _t(dZ, False)).sum()
    if dW_out is not None:
        L = L + (Wo * _t(dW_out, False)).sum()
    names = ["Q", "K", "V", "eta", "W0"] + (["gamma", "beta"] if ln else [])
    grads = torch.autograd.grad(L, [ts[n] for n in names], allow_unused=True)
    out = {}
    for n, gr in zip(names, grads):
        out[n] = np.zeros(ts[n].shape) if gr is None else gr.detach().numpy()
    return out


def linear_forward_np(Q, K, V, eta, W0, gamma, beta, *, b, ln, eps=LN_EPS):
    """The same forward without a graph, as numpy (for pinning against the C oracle)."""
    H, d = Q.shape[1], Q.shape[3]
    gamma = np.ones((H, d)) if gamma is None else gamma
    beta = np.zeros((H, d)) if beta is None else beta
    ts = [_t(a) for a in (Q, K, V, eta, W0, gamma, beta)]
    Z, Wo = linear_forward(*ts, b=b, ln=ln, eps=eps)
    return Z.detach().numpy(), Wo.detach().numpy()


def chunk_forward(Q, K, V, eta, W0, *, chunk):
    """Large-chunk TTT ("Test-Time Training Done Right", abstract): the tokens
    of chunk c read out with W_c, then W_{c+1} = W_c - grad of
    sum_t eta_t 1/2 ||k_t W_c - v_t||^2 at W_c (autograd, kept in the graph).
    f(k) = k W (no LayerNorm). Returns (Z, W_out) as float64 tensors."""
    B, H, T, d = Q.shape
    W = W0.expand(B, H, d, d) if W0.dim() == 3 else W0
    Z = []
    for c0 in range(0, T, chunk):
        Wc = W
        sl = slice(c0, c0 + chunk)
        Z.append(torch.einsum("bhti,bhij->bhtj", Q[:, :, sl], Wc))
        r = torch.einsum("bhti,bhij->bhtj", K[:, :, sl], Wc) - V[:, :, sl]
        loss = 0.5 * (eta[:, :, sl, None] * r * r).sum()
        W = Wc - torch.autograd.grad(loss, Wc, create_graph=True)[0]
    return torch.cat(Z, dim=2), W


def chunk_grads(Q, K, V, eta, W0, dZ, dW_out=None, *, chunk):
    """Gradients of L = sum(Z * dZ) + sum(W_out * dW_out) for the large-chunk
    forward: dict with keys Q, K, V, eta, W0 (float64 numpy)."""
    ts = {n: _t(a) for n, a in dict(Q=Q, K=K, V=V, eta=eta, W0=W0).items()}
    Z, Wo = chunk_forward(ts["Q"], ts["K"], ts["V"], ts["eta"], ts["W0"], chunk=chunk)
    L = (Z * _t(dZ, False)).sum()
    if dW_out is not None:
        L = L + (Wo * _t(dW_out, False)).sum()
    names = ["Q", "K", "V", "eta", "W0"]
    grads = torch.autograd.grad(L, [ts[n] for n in names], allow_unused=True)
    return {n: (np.zeros(ts[n].shape) if g is None else g.detach().numpy())
            for n, g in zip(names, grads)}


def chunk_forward_np(Q, K, V, eta, W0, *, chunk):
    ts = [_t(a) for a in (Q, K, V, eta, W0)]
    Z, Wo = chunk_forward(*ts, chunk=chunk)
    return Z.detach().numpy(), Wo.detach().numpy()


def mlp_forward(Q, K, V, eta, W1_0, W2_0, gamma, beta, *, b, eps=LN_EPS):
    """TTT-MLP ("How to Master Test-Time Training for LLMs": the fast weight
    may be an MLP) with the TTT-Linear mini-batch rule: f(k) = k +
    LN(GELU(k W1) W2) gamma + beta, exact-erf GELU; every token's inner
    gradient (autograd, kept in the graph) at the mini-batch's starting
    weights, the read-out of token t after its own step. Returns (Z, W1_out,
    W2_out) as float64 tensors; W1_0 [H,d,dh] or [B,H,d,dh], W2_0 likewise."""
    B, H, T, d = Q.shape
    dh = W1_0.shape[-1]
    W1 = W1_0.expand(B, H, d, dh) if W1_0.dim() == 3 else W1_0
    W2 = W2_0.expand(B, H, dh, d) if W2_0.dim() == 3 else W2_0
    g, be = gamma.view(1, H, d), beta.view(1, H, d)

    def f(k, A1, A2):
        a = F.gelu(torch.einsum("bhi,bhij->bhj", k, A1))
        x = torch.einsum("bhi,bhij->bhj", a, A2)
        return k + F.layer_norm(x, (d,), eps=eps) * g + be

    Z = []
    for m0 in range(0, T, b):
        W1m, W2m = W1, W2
        for t in range(m0, m0 + b):
            k, v = K[:, :, t], V[:, :, t]
            loss = 0.5 * ((f(k, W1m, W2m) - v) ** 2).sum()
            g1, g2 = torch.autograd.grad(loss, (W1m, W2m), create_graph=True)
            e = eta[:, :, t, None, None]
            W1, W2 = W1 - e * g1, W2 - e * g2
            Z.append(f(Q[:, :, t], W1, W2))
    return torch.stack(Z, dim=2), W1, W2


def mlp_forward_np(Q, K, V, eta, W1_0, W2_0, gamma, beta, *, b, eps=LN_EPS):
    ts = [_t(a) for a in (Q, K, V, eta, W1_0, W2_0, gamma, beta)]
    Z, W1, W2 = mlp_forward(*ts, b=b, eps=eps)
    return Z.detach().numpy(), W1.detach().numpy(), W2.detach().numpy()


def mlp_grads(Q, K, V, eta, W1_0, W2_0, gamma, beta, dZ, dW1_out=None, dW2_out=None, *, b,
              eps=LN_EPS):
    """Gradients of L = sum(Z * dZ) + sum(W1_out * dW1_out) + sum(W2_out *
    dW2_out) for TTT-MLP: dict with keys Q, K, V, eta, W1, W2, gamma, beta."""
    names = ["Q", "K", "V", "eta", "W1", "W2", "gamma", "beta"]
    ts = dict(zip(names, (_t(a) for a in (Q, K, V, eta, W1_0, W2_0, gamma, beta))))
    Z, W1, W2 = mlp_forward(*(ts[n] for n in names), b=b, eps=eps)
    L = (Z * _t(dZ, False)).sum()
    if dW1_out is not None:
        L = L + (W1 * _t(dW1_out, False)).sum()
    if dW2_out is not None:
        L = L + (W2 * _t(dW2_out, False)).sum()
    grads = torch.autograd.grad(L, [ts[n] for n in names], allow_unused=True)
    return {n: (np.zeros(ts[n].shape) if gr is None else gr.detach().numpy())
            for n, gr in zip(names, grads)}
