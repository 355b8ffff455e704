"""The fp32 CUDA-core kernels of ttt_simt.cu run on the host against the
oracles: TTT-Linear (the plain forward, with L2-normalised keys and with
several gradient steps per token), TTT-MLP and large-chunk TTT.
The kernel source is compiled with g++ into a test harness
(tests/host_emu/simt_emu.cpp): 256 OS threads per block, a std::barrier for
__syncthreads(), warp shuffles through per-warp buffers and barriers. It
checks the kernel's arithmetic and indexing without a GPU; the same cases run
on the GPU in tests/test_variants_gpu.py and tests/test_parity_gpu.py.
Tolerances: 1e-5 of the largest magnitude (fp32 arithmetic)."""
import ctypes
import os
import subprocess

import numpy as np
import pytest

import oracle
from oracle import variants

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "host_emu", "simt_emu.cpp")
TOL = 1e-5


@pytest.fixture(scope="module")
def emu(tmp_path_factory):
    so = str(tmp_path_factory.mktemp("emu") / "simt_emu.so")
    subprocess.run(["g++", "-std=c++20", "-O2", "-shared", "-fPIC", "-pthread",
                    "-I/usr/local/cuda/include", SRC, "-o", so], check=True)
    L = ctypes.CDLL(so)
    L.ttt_linear_simt_host_run.restype = ctypes.c_int
    L.ttt_linear_simt_host_run.argtypes = [ctypes.c_void_p] * 9 + [ctypes.c_int] * 11
    L.ttt_mlp_simt_host_run.restype = ctypes.c_int
    L.ttt_mlp_simt_host_run.argtypes = [ctypes.c_void_p] * 11 + [ctypes.c_int] * 6
    L.ttt_chunk_simt_host_run.restype = ctypes.c_int
    L.ttt_chunk_simt_host_run.argtypes = [ctypes.c_void_p] * 7 + [ctypes.c_int] * 5
    return L


def _inputs(seed, B, H, T, d, eta_scale):
    r = np.random.default_rng(seed)
    Q, K, V = (r.standard_normal((B, H, T, d)) / np.sqrt(d) for _ in range(3))
    eta = eta_scale * r.uniform(0.2, 1.0, (B, H, T))
    W0 = 0.3 * r.standard_normal((H, d, d)) / np.sqrt(d)
    g, be = 1 + 0.2 * r.standard_normal((H, d)), 0.2 * r.standard_normal((H, d))
    f = lambda a: np.ascontiguousarray(a, dtype=np.float32)  # noqa: E731
    return tuple(f(a) for a in (Q, K, V, eta, W0, g, be))


def _run(L, Q, K, V, eta, W0, g, be, *, b, ln, l2=False, steps=1):
    B, H, T, d = Q.shape
    Z = np.zeros((B, H, T, d), np.float32)
    W = np.zeros((B, H, d, d), np.float32)
    rc = L.ttt_linear_simt_host_run(*[a.ctypes.data for a in (Q, K, V, eta, W0, g, be, Z, W)],
                                    B, H, T, d, b, 0, int(ln), 0, 0, int(l2), steps)
    assert rc == 0
    return Z.astype(np.float64), W.astype(np.float64)


def _rel(g, r):
    return float(np.abs(g - r).max() / max(np.abs(r).max(), 1e-30))


@pytest.mark.parametrize("d,b,T,ln", [(16, 16, 64, False), (64, 16, 41, True), (32, 1, 12, True),
                                      (64, 8, 32, False)])
def test_plain_forward(emu, d, b, T, ln):
    Q, K, V, eta, W0, g, be = _inputs(d + T, 2, 2, T, d, 0.1)
    Z, W = _run(emu, Q, K, V, eta, W0, g, be, b=b, ln=ln)
    Zr, Wr = oracle.linear_primal(Q, K, V, eta, W0, g if ln else None, be if ln else None, b=b,
                                  ln=ln)
    assert _rel(Z, Zr) <= TOL and _rel(W, Wr) <= TOL


@pytest.mark.parametrize("d,b,T,ln", [(64, 16, 48, True), (16, 4, 19, False)])
def test_l2_keys(emu, d, b, T, ln):
    Q, K, V, eta, W0, g, be = _inputs(3 * d + T, 1, 2, T, d, 0.1)
    K = (K * np.random.default_rng(9).uniform(0.3, 3.0, K.shape[:3] + (1,))).astype(np.float32)
    Z, W = _run(emu, Q, K, V, eta, W0, g, be, b=b, ln=ln, l2=True)
    Zr, Wr = oracle.linear_primal(Q, variants.normalize_keys(K), V, eta, W0,
                                  g if ln else None, be if ln else None, b=b, ln=ln)
    assert _rel(Z, Zr) <= TOL and _rel(W, Wr) <= TOL


@pytest.mark.parametrize("d,n,ln,l2", [(64, 3, True, False), (16, 4, False, False),
                                       (32, 2, True, True)])
def test_several_steps_per_token(emu, d, n, ln, l2):
    Q, K, V, eta, W0, g, be = _inputs(5 * d + n, 2, 1, 10, d, 0.2)
    Z, W = _run(emu, Q, K, V, eta, W0, g, be, b=1, ln=ln, l2=l2, steps=n)
    Kr = variants.normalize_keys(K) if l2 else K
    Zr, Wr = variants.linear_multistep(Q, Kr, V, eta, W0, g if ln else None, be if ln else None,
                                       n_steps=n, ln=ln)
    assert _rel(Z, Zr) <= TOL and _rel(W, Wr) <= TOL


def test_mlp_kernel(emu):
    r = np.random.default_rng(41)
    B, H, T, d, dh, b = 1, 2, 32, 16, 64, 8
    f = lambda a: np.ascontiguousarray(a, dtype=np.float32)  # noqa: E731
    Q, K, V = (f(r.standard_normal((B, H, T, d)) / np.sqrt(d)) for _ in range(3))
    eta = f(0.1 * r.uniform(0.2, 1.0, (B, H, T)))
    W1 = f(0.5 * r.standard_normal((H, d, dh)) / np.sqrt(d))
    W2 = f(0.5 * r.standard_normal((H, dh, d)) / np.sqrt(dh))
    g, be = f(1 + 0.2 * r.standard_normal((H, d))), f(0.2 * r.standard_normal((H, d)))
    Z = np.zeros((B, H, T, d), np.float32)
    W1o, W2o = np.zeros((B, H, d, dh), np.float32), np.zeros((B, H, dh, d), np.float32)
    assert emu.ttt_mlp_simt_host_run(*[a.ctypes.data for a in (Q, K, V, eta, W1, W2, g, be, Z,
                                                                W1o, W2o)],
                                     B, H, T, d, dh, b) == 0
    Zr, W1r, W2r = oracle.mlp_primal(Q, K, V, eta, W1, W2, g, be, b=b)
    assert _rel(Z, Zr) <= TOL and _rel(W1o, W1r) <= TOL and _rel(W2o, W2r) <= TOL


def test_chunk_kernel(emu):
    r = np.random.default_rng(43)
    B, H, T, d, C = 2, 1, 128, 64, 64
    f = lambda a: np.ascontiguousarray(a, dtype=np.float32)  # noqa: E731
    Q, K, V = (f(r.standard_normal((B, H, T, d)) / np.sqrt(d)) for _ in range(3))
    eta = f(np.full((B, H, T), 1.0 / C))
    W0 = f(0.3 * r.standard_normal((H, d, d)) / np.sqrt(d))
    Z, W = np.zeros((B, H, T, d), np.float32), np.zeros((B, H, d, d), np.float32)
    assert emu.ttt_chunk_simt_host_run(*[a.ctypes.data for a in (Q, K, V, eta, W0, Z, W)],
                                       B, H, T, d, C) == 0
    Zr, Wr = oracle.chunk_primal(Q, K, V, eta, W0, chunk=C)
    assert _rel(Z, Zr) <= TOL and _rel(W, Wr) <= TOL
