"""ctypes wrapper of the CPU oracle (oracle/ttt_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by the test suite, the smoke check and the
benchmark's CPU-baseline leg, never by the library. Every array is widened to
float64 before the call; results come back as float64.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_lib = None
_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int)

LN_EPS = 1e-5  # torch nn.LayerNorm default, as in the pages' listing


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        c_int, c_double = ctypes.c_int, ctypes.c_double
        common = [_dp] * 7 + [_dp, _dp]
        L.orc_linear_primal.argtypes = common + [c_int] * 7 + [c_double, _ip, c_int, c_int]
        L.orc_linear_dual.argtypes = L.orc_linear_primal.argtypes
        L.orc_chunk_primal.argtypes = L.orc_linear_primal.argtypes
        mlp = [_dp] * 8 + [_dp, _dp, _dp] + [c_int] * 7 + [c_double, _ip, c_int, c_int]
        L.orc_mlp_primal.argtypes = mlp
        L.orc_mlp_dual.argtypes = mlp
        for f in ("orc_linear_primal", "orc_linear_dual", "orc_chunk_primal",
                  "orc_mlp_primal", "orc_mlp_dual", "orc_num_threads"):
            getattr(L, f).restype = c_int
        L.orc_loss_linear.argtypes = [_dp] * 5 + [c_int, c_int, c_double]
        L.orc_loss_linear.restype = c_double
        L.orc_grad_linear.argtypes = [_dp] * 5 + [c_int, c_int, c_double, _dp]
        L.orc_grad_linear.restype = None
        L.orc_loss_mlp.argtypes = [_dp] * 6 + [c_int, c_int, c_double]
        L.orc_loss_mlp.restype = c_double
        L.orc_grad_mlp.argtypes = [_dp] * 6 + [c_int, c_int, c_double, _dp, _dp]
        L.orc_grad_mlp.restype = None
        L.orc_gelu.argtypes = [c_double]
        L.orc_gelu.restype = c_double
        L.orc_gelu_prime.argtypes = [c_double]
        L.orc_gelu_prime.restype = c_double
        _lib = L
    return _lib


def num_threads() -> int:
    return lib().orc_num_threads()


def _d(x):
    """Contiguous float64 copy (or None) and its ctypes pointer."""
    if x is None:
        return None, None
    a = np.ascontiguousarray(x, dtype=np.float64)
    return a, a.ctypes.data_as(_dp)


def _seqs(seqs):
    if seqs is None:
        return None, None, 0
    a = np.ascontiguousarray(seqs, dtype=np.int32)
    return a, a.ctypes.data_as(_ip), int(a.size)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} failed with code {rc}")


def _linear_like(fn_name, Q, K, V, eta, W0, gamma, beta, b, ln, w0_per_seq, eps, seqs,
                 nthreads, with_w):
    B, H, T, d = Q.shape
    keep = []
    ptrs = []
    for x in (Q, K, V, eta, W0, gamma, beta):
        a, p = _d(x)
        keep.append(a)
        ptrs.append(p)
    Z = np.zeros((B, H, T, d))
    W_out = np.zeros((B, H, d, d)) if with_w else None
    sa, sp, ns = _seqs(seqs)
    rc = getattr(lib(), fn_name)(*ptrs, Z.ctypes.data_as(_dp),
                                 W_out.ctypes.data_as(_dp) if with_w else None,
                                 B, H, T, d, b, int(bool(ln)), int(bool(w0_per_seq)), eps,
                                 sp, ns, nthreads)
    _check(rc, fn_name)
    return Z, W_out


def linear_primal(Q, K, V, eta, W0, gamma=None, beta=None, *, b, ln, w0_per_seq=False,
                  eps=LN_EPS, seqs=None, nthreads=0, with_w=True):
    """TTT-Linear forward, update-then-apply with mini-batches of b (primal form).
    Returns (Z [B,H,T,d], W_out [B,H,d,d])."""
    return _linear_like("orc_linear_primal", Q, K, V, eta, W0, gamma, beta, b, ln, w0_per_seq,
                        eps, seqs, nthreads, with_w)


def linear_dual(Q, K, V, eta, W0, gamma=None, beta=None, *, b, ln, w0_per_seq=False,
                eps=LN_EPS, seqs=None, nthreads=0, with_w=True):
    """Same rule as linear_primal, computed in the mini-batch dual form."""
    return _linear_like("orc_linear_dual", Q, K, V, eta, W0, gamma, beta, b, ln, w0_per_seq,
                        eps, seqs, nthreads, with_w)


def chunk_primal(Q, K, V, eta, W0, gamma=None, beta=None, *, chunk, ln=False, w0_per_seq=False,
                 eps=LN_EPS, seqs=None, nthreads=0, with_w=True):
    """Large-chunk TTT (apply-then-update over chunks). Returns (Z, W_out)."""
    return _linear_like("orc_chunk_primal", Q, K, V, eta, W0, gamma, beta, chunk, ln, w0_per_seq,
                        eps, seqs, nthreads, with_w)


def _mlp(fn_name, Q, K, V, eta, W1, W2, gamma, beta, b, w0_per_seq, eps, seqs, nthreads):
    B, H, T, d = Q.shape
    dh = W1.shape[-1]
    keep, ptrs = [], []
    for x in (Q, K, V, eta, W1, W2, gamma, beta):
        a, p = _d(x)
        keep.append(a)
        ptrs.append(p)
    Z = np.zeros((B, H, T, d))
    W1o = np.zeros((B, H, d, dh))
    W2o = np.zeros((B, H, dh, d))
    sa, sp, ns = _seqs(seqs)
    rc = getattr(lib(), fn_name)(*ptrs, Z.ctypes.data_as(_dp), W1o.ctypes.data_as(_dp),
                                 W2o.ctypes.data_as(_dp), B, H, T, d, dh, b,
                                 int(bool(w0_per_seq)), eps, sp, ns, nthreads)
    _check(rc, fn_name)
    return Z, W1o, W2o


def mlp_primal(Q, K, V, eta, W1, W2, gamma, beta, *, b, w0_per_seq=False, eps=LN_EPS, seqs=None,
               nthreads=0):
    """TTT-MLP forward, f(k) = k + LN(GELU(k W1) W2), primal form.
    Returns (Z, W1_out [B,H,d,dh], W2_out [B,H,dh,d])."""
    return _mlp("orc_mlp_primal", Q, K, V, eta, W1, W2, gamma, beta, b, w0_per_seq, eps, seqs,
                nthreads)


def mlp_dual(Q, K, V, eta, W1, W2, gamma, beta, *, b, w0_per_seq=False, eps=LN_EPS, seqs=None,
             nthreads=0):
    """Same rule as mlp_primal in the two-stage dual form."""
    return _mlp("orc_mlp_dual", Q, K, V, eta, W1, W2, gamma, beta, b, w0_per_seq, eps, seqs,
                nthreads)


def loss_linear(k, v, W, gamma=None, beta=None, *, ln, eps=LN_EPS) -> float:
    d = k.shape[0]
    arrs = [_d(x) for x in (k, v, W, gamma, beta)]
    return lib().orc_loss_linear(*[p for _, p in arrs], d, int(bool(ln)), eps)


def grad_linear(k, v, W, gamma=None, beta=None, *, ln, eps=LN_EPS) -> np.ndarray:
    d = k.shape[0]
    arrs = [_d(x) for x in (k, v, W, gamma, beta)]
    G = np.zeros((d, d))
    lib().orc_grad_linear(*[p for _, p in arrs], d, int(bool(ln)), eps, G.ctypes.data_as(_dp))
    return G


def loss_mlp(k, v, W1, W2, gamma, beta, *, eps=LN_EPS) -> float:
    d, dh = W1.shape
    arrs = [_d(x) for x in (k, v, W1, W2, gamma, beta)]
    return lib().orc_loss_mlp(*[p for _, p in arrs], d, dh, eps)


def grad_mlp(k, v, W1, W2, gamma, beta, *, eps=LN_EPS):
    d, dh = W1.shape
    arrs = [_d(x) for x in (k, v, W1, W2, gamma, beta)]
    G1 = np.zeros((d, dh))
    G2 = np.zeros((dh, d))
    lib().orc_grad_mlp(*[p for _, p in arrs], d, dh, eps, G1.ctypes.data_as(_dp),
                       G2.ctypes.data_as(_dp))
    return G1, G2


def gelu(h: float) -> float:
    return lib().orc_gelu(float(h))


def gelu_prime(h: float) -> float:
    return lib().orc_gelu_prime(float(h))
