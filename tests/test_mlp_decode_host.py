"""The one-token TTT-MLP decode kernel (ttt_mlp_decode.cu) run on the host
(tests/host_emu/mlp_decode_emu.cpp: 256 OS threads per block, a std::barrier
per __syncthreads(), emulated warp shuffles): a loop of single-token calls,
both layers updated in place, against the C oracle's b = 1 TTT-MLP forward
over the same tokens. Tolerance 1e-5 (fp32 inputs)."""
import ctypes
import os
import subprocess

import numpy as np
import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "host_emu", "mlp_decode_emu.cpp")


@pytest.fixture(scope="module")
def emu(tmp_path_factory):
    so = str(tmp_path_factory.mktemp("emu") / "mlp_decode_emu.so")
    subprocess.run(["g++", "-std=c++20", "-O2", "-shared", "-fPIC", "-pthread",
                    "-I/usr/local/cuda/include", SRC, "-o", so], check=True)
    L = ctypes.CDLL(so)
    L.ttt_mlp_decode_host_run.restype = ctypes.c_int
    L.ttt_mlp_decode_host_run.argtypes = [ctypes.c_void_p] * 9 + [ctypes.c_int] * 3
    L.ttt_mlp_decode_tokens_host_run.restype = ctypes.c_int
    L.ttt_mlp_decode_tokens_host_run.argtypes = [ctypes.c_void_p] * 9 + [ctypes.c_int] * 4
    return L


def test_token_loop_matches_oracle(emu):
    B, H, T, d, dh = 1, 2, 8, 64, 256
    r = np.random.default_rng(11)
    f = lambda a: np.ascontiguousarray(a, dtype=np.float32)  # noqa: E731
    Q, K, V = (f(r.standard_normal((B, H, T, d)) / np.sqrt(d)) for _ in range(3))
    eta = f(0.5 / d * r.uniform(0.2, 1.0, (B, H, T)))
    W1_0 = f(0.3 * r.standard_normal((B, H, d, dh)) / np.sqrt(d))
    W2_0 = f(0.3 * r.standard_normal((B, H, dh, d)) / np.sqrt(dh))
    g, be = f(1 + 0.1 * r.standard_normal((H, d))), f(0.1 * r.standard_normal((H, d)))
    W1, W2 = W1_0.copy(), W2_0.copy()
    Z = np.zeros((B, H, T, d), np.float32)
    for t in range(T):
        q, k, v, e = (f(a[:, :, t]) for a in (Q, K, V, eta))
        z = np.zeros((B, H, d), np.float32)
        assert emu.ttt_mlp_decode_host_run(q.ctypes.data, k.ctypes.data, v.ctypes.data,
                                           e.ctypes.data, g.ctypes.data, be.ctypes.data,
                                           W1.ctypes.data, W2.ctypes.data, z.ctypes.data, B, H,
                                           0) == 0
        Z[:, :, t] = z
    Zr, W1r, W2r = oracle.mlp_primal(Q, K, V, eta, W1_0, W2_0, g, be, b=1, w0_per_seq=True)
    for got, ref in ((Z, Zr), (W1, W1r), (W2, W2r)):
        assert np.abs(got - ref).max() <= 1e-5 * np.abs(ref).max()


def test_tokens_in_one_call_match_oracle(emu):
    """All T tokens in one call (both layers kept in registers across them)
    against the oracle's b = 1 TTT-MLP forward."""
    B, H, T, d, dh = 1, 2, 6, 64, 256
    r = np.random.default_rng(13)
    f = lambda a: np.ascontiguousarray(a, dtype=np.float32)  # noqa: E731
    Q, K, V = (f(r.standard_normal((B, H, T, d)) / np.sqrt(d)) for _ in range(3))
    eta = f(0.5 / d * r.uniform(0.2, 1.0, (B, H, T)))
    W1_0 = f(0.3 * r.standard_normal((B, H, d, dh)) / np.sqrt(d))
    W2_0 = f(0.3 * r.standard_normal((B, H, dh, d)) / np.sqrt(dh))
    g, be = f(1 + 0.1 * r.standard_normal((H, d))), f(0.1 * r.standard_normal((H, d)))
    W1, W2 = W1_0.copy(), W2_0.copy()
    Z = np.zeros((B, H, T, d), np.float32)
    assert emu.ttt_mlp_decode_tokens_host_run(Q.ctypes.data, K.ctypes.data, V.ctypes.data,
                                              eta.ctypes.data, g.ctypes.data, be.ctypes.data,
                                              W1.ctypes.data, W2.ctypes.data, Z.ctypes.data, B,
                                              H, T, 0) == 0
    Zr, W1r, W2r = oracle.mlp_primal(Q, K, V, eta, W1_0, W2_0, g, be, b=1, w0_per_seq=True)
    for got, ref in ((Z, Zr), (W1, W1r), (W2, W2r)):
        assert np.abs(got - ref).max() <= 1e-5 * np.abs(ref).max()
