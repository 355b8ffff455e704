"""The one-token TTT-Linear decode kernel (ttt_decode.cu) run on the host
(tests/host_emu/decode_emu.cpp: 128 OS threads per block, a std::barrier per
__syncthreads(), emulated warp shuffles): a loop of single-token calls, the
weight updated in place, against the C oracle's b = 1 forward over the same
tokens. Tolerance 1e-5 (fp32 inputs)."""
import ctypes
import os
import subprocess

import numpy as np
import pytest

import oracle
from oracle import variants

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "host_emu", "decode_emu.cpp")


@pytest.fixture(scope="module")
def emu(tmp_path_factory):
    so = str(tmp_path_factory.mktemp("emu") / "decode_emu.so")
    subprocess.run(["g++", "-std=c++20", "-O2", "-shared", "-fPIC", "-pthread",
                    "-I/usr/local/cuda/include", SRC, "-o", so], check=True)
    L = ctypes.CDLL(so)
    L.ttt_linear_decode_host_run.restype = ctypes.c_int
    L.ttt_linear_decode_host_run.argtypes = [ctypes.c_void_p] * 8 + [ctypes.c_int] * 5
    L.ttt_linear_decode_tokens_host_run.restype = ctypes.c_int
    L.ttt_linear_decode_tokens_host_run.argtypes = [ctypes.c_void_p] * 8 + [ctypes.c_int] * 6
    return L


@pytest.mark.parametrize("ln,l2", [(True, False), (False, False), (True, True)])
def test_token_loop_matches_oracle(emu, ln, l2):
    B, H, T, d = 2, 3, 12, 64
    r = np.random.default_rng(3 + int(ln))
    f = lambda a: np.ascontiguousarray(a, dtype=np.float32)  # noqa: E731
    Q, K, V = (f(r.standard_normal((B, H, T, d)) / np.sqrt(d)) for _ in range(3))
    eta = f(0.5 / d * r.uniform(0.2, 1.0, (B, H, T)))
    W0 = f(0.02 * r.standard_normal((B, H, d, d)))
    g, be = f(1 + 0.02 * r.standard_normal((H, d))), f(0.02 * r.standard_normal((H, d)))
    W = W0.copy()
    Z = np.zeros((B, H, T, d), np.float32)
    for t in range(T):
        q, k, v, e = (f(a[:, :, t]) for a in (Q, K, V, eta))
        z = np.zeros((B, H, d), np.float32)
        assert emu.ttt_linear_decode_host_run(q.ctypes.data, k.ctypes.data, v.ctypes.data,
                                              e.ctypes.data, g.ctypes.data, be.ctypes.data,
                                              W.ctypes.data, z.ctypes.data, B, H, 0, int(ln),
                                              int(l2)) == 0
        Z[:, :, t] = z
    Kr = variants.normalize_keys(K) if l2 else K
    Zr, Wr = oracle.linear_primal(Q, Kr, V, eta, W0, g if ln else None, be if ln else None, b=1,
                                  ln=ln, w0_per_seq=True)
    assert np.abs(Z - Zr).max() <= 1e-5 * np.abs(Zr).max()
    assert np.abs(W - Wr).max() <= 1e-5 * np.abs(Wr).max()


@pytest.mark.parametrize("ln,l2", [(True, False), (False, True)])
def test_tokens_in_one_call_match_oracle(emu, ln, l2):
    """All T tokens in one call (the weight kept in registers across them)
    against the oracle's b = 1 forward; a planted error in the token stride
    (every sequence reading token 0) fails it."""
    B, H, T, d = 2, 2, 9, 64
    r = np.random.default_rng(7 + int(ln))
    f = lambda a: np.ascontiguousarray(a, dtype=np.float32)  # noqa: E731
    Q, K, V = (f(r.standard_normal((B, H, T, d)) / np.sqrt(d)) for _ in range(3))
    eta = f(0.5 / d * r.uniform(0.2, 1.0, (B, H, T)))
    W0 = f(0.02 * r.standard_normal((B, H, d, d)))
    g, be = f(1 + 0.02 * r.standard_normal((H, d))), f(0.02 * r.standard_normal((H, d)))
    W = W0.copy()
    Z = np.zeros((B, H, T, d), np.float32)
    assert emu.ttt_linear_decode_tokens_host_run(Q.ctypes.data, K.ctypes.data, V.ctypes.data,
                                                 eta.ctypes.data, g.ctypes.data, be.ctypes.data,
                                                 W.ctypes.data, Z.ctypes.data, B, H, T, 0,
                                                 int(ln), int(l2)) == 0
    Kr = variants.normalize_keys(K) if l2 else K
    Zr, Wr = oracle.linear_primal(Q, Kr, V, eta, W0, g if ln else None, be if ln else None, b=1,
                                  ln=ln, w0_per_seq=True)
    assert np.abs(Z - Zr).max() <= 1e-5 * np.abs(Zr).max()
    assert np.abs(W - Wr).max() <= 1e-5 * np.abs(Wr).max()
    # the same call on inputs whose tokens all repeat token 0 differs (the kernel walks tokens)
    Q1, K1, V1 = (f(np.repeat(a[:, :, :1], T, axis=2)) for a in (Q, K, V))
    W1 = W0.copy()
    Z1 = np.zeros_like(Z)
    emu.ttt_linear_decode_tokens_host_run(Q1.ctypes.data, K1.ctypes.data, V1.ctypes.data,
                                          eta.ctypes.data, g.ctypes.data, be.ctypes.data,
                                          W1.ctypes.data, Z1.ctypes.data, B, H, T, 0, int(ln),
                                          int(l2))
    assert np.abs(Z1 - Zr).max() > 1e-3 * np.abs(Zr).max()
