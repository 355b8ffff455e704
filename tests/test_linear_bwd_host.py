"""The TTT-Linear backward kernels (ttt_linear_bwd.cu) run on the host
(tests/host_emu/linear_bwd_emu.cpp: 256 OS threads per block, a std::barrier
per __syncthreads(), emulated warp shuffles) against the backward oracle
(oracle/backward.py), on the shapes of the GPU cases in
tests/test_backward_gpu.py. Tolerance 1e-4 of each gradient's largest
magnitude, as on the GPU."""
import ctypes
import os
import subprocess

import numpy as np
import pytest

from oracle import backward as ob

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "host_emu", "linear_bwd_emu.cpp")
TOL = 1e-4


@pytest.fixture(scope="module")
def emu(tmp_path_factory):
    so = str(tmp_path_factory.mktemp("emu") / "linear_bwd_emu.so")
    subprocess.run(["g++", "-std=c++20", "-O2", "-shared", "-fPIC", "-pthread",
                    "-I/usr/local/cuda/include", SRC, "-o", so], check=True)
    L = ctypes.CDLL(so)
    L.ttt_linear_bwd_host_run.restype = ctypes.c_int
    L.ttt_linear_bwd_host_run.argtypes = [ctypes.c_void_p] * 16 + [ctypes.c_int] * 8
    return L


def _bf16(a):
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    bits = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    return bits, (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


@pytest.mark.parametrize("B,H,T,d,b,ln,bf16,w0seq,with_dw", [
    (2, 2, 16, 16, 4, True, False, False, True),
    (2, 2, 16, 16, 4, False, False, False, True),
    (2, 1, 32, 32, 8, True, False, True, False),
    (1, 2, 64, 64, 16, True, True, False, True),
    (1, 2, 48, 64, 16, False, True, False, False),
    (1, 1, 8, 64, 1, True, False, False, True),
])
def test_host_run_matches_oracle(emu, B, H, T, d, b, ln, bf16, w0seq, with_dw):
    r = np.random.default_rng(B + H + T + d + b)
    f = lambda a: np.ascontiguousarray(a, dtype=np.float32)  # noqa: E731
    Q, K, V = (r.standard_normal((B, H, T, d)) / np.sqrt(d) for _ in range(3))
    if bf16:
        (Qb, Q), (Kb, K), (Vb, V) = _bf16(Q), _bf16(K), _bf16(V)
        ins = [Qb, Kb, Vb]
    else:
        Q, K, V = (f(x).astype(np.float64) for x in (Q, K, V))
        ins = [f(Q), f(K), f(V)]
    eta = f(0.02 * r.uniform(0.2, 1.0, (B, H, T)))
    W0 = f(r.standard_normal((B, H, d, d) if w0seq else (H, d, d)) / np.sqrt(d))
    g, be = f(1 + 0.2 * r.standard_normal((H, d))), f(0.2 * r.standard_normal((H, d)))
    dZ = f(r.standard_normal((B, H, T, d)))
    dW = f(r.standard_normal((B, H, d, d))) if with_dw else None
    out = {k: np.zeros(s, np.float32) for k, s in dict(
        Q=(B, H, T, d), K=(B, H, T, d), V=(B, H, T, d), eta=(B, H, T), W0=W0.shape,
        gamma=(H, d), beta=(H, d)).items()}
    ptr = lambda a: None if a is None else a.ctypes.data  # noqa: E731
    rc = emu.ttt_linear_bwd_host_run(*[ptr(a) for a in ins + [eta, W0, g, be, dZ, dW]],
                                     *[ptr(out[k]) for k in ("Q", "K", "V", "eta", "W0", "gamma",
                                                             "beta")],
                                     B, H, T, d, b, int(bf16), int(ln), int(w0seq))
    assert rc == 0
    ref = ob.linear_grads(Q, K, V, eta, W0, g if ln else None, be if ln else None, dZ, dW, b=b,
                          ln=ln)
    for k, rv in ref.items():
        gv = out[k].astype(np.float64).reshape(rv.shape)
        assert np.abs(gv - rv).max() <= TOL * max(np.abs(rv).max(), 1e-30), k
