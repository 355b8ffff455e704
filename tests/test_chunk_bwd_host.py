"""The large-chunk backward's fp32 scan and per-token kernels (ttt_chunk_bwd.cu:
cb_scan_kernel with its column slices, cb_tok_kernel, the dW0 batch sum) run on
the host (tests/host_emu/chunk_bwd_emu.cpp: 256 OS threads per block, a
std::barrier per __syncthreads(), emulated warp shuffles), fed with the
per-chunk Gram products A_c = K_c^T diag(eta) K_c, B_c = K_c^T diag(eta) V_c,
D_c = Q_c^T dZ_c formed here in float64, against the backward oracle
(oracle/backward.py). Tolerance 1e-4 of each gradient's largest magnitude, as
on the GPU."""
import ctypes
import os
import subprocess

import numpy as np
import pytest

from oracle import backward as ob

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "host_emu", "chunk_bwd_emu.cpp")
TOL = 1e-4


@pytest.fixture(scope="module")
def emu(tmp_path_factory):
    so = str(tmp_path_factory.mktemp("emu") / "chunk_bwd_emu.so")
    subprocess.run(["g++", "-std=c++20", "-O2", "-shared", "-fPIC", "-pthread",
                    "-I/usr/local/cuda/include", SRC, "-o", so], check=True)
    L = ctypes.CDLL(so)
    L.ttt_chunk_bwd_scan_tok_host_run.restype = ctypes.c_int
    L.ttt_chunk_bwd_scan_tok_host_run.argtypes = [ctypes.c_void_p] * 12 + [ctypes.c_int] * 7
    return L


def _bf16(a):
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    bits = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    return bits, (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _gram(Q, K, V, eta, dZ, C):
    """[B*H*(T/C)][3][d][d]: A_c, B_c, D_c of every chunk, sequence-major."""
    B, H, T, d = Q.shape
    out = []
    for b in range(B):
        for h in range(H):
            for c0 in range(0, T, C):
                s = slice(c0, c0 + C)
                k, v, q, z, e = K[b, h, s], V[b, h, s], Q[b, h, s], dZ[b, h, s], eta[b, h, s, None]
                out.append(np.stack([k.T @ (e * k), k.T @ (e * v), q.T @ z]))
    return np.ascontiguousarray(np.stack(out), dtype=np.float32)


@pytest.mark.parametrize("B,H,T,d,C,bf16,w0seq,with_dw", [
    (2, 2, 96, 64, 32, False, False, True),
    (1, 2, 128, 64, 64, True, False, False),
    (2, 1, 64, 64, 32, False, True, True),
    (1, 1, 64, 128, 32, True, False, True),
])
def test_host_run_matches_oracle(emu, B, H, T, d, C, bf16, w0seq, with_dw):
    r = np.random.default_rng(B + H + T + d + C)
    f = lambda a: np.ascontiguousarray(a, dtype=np.float32)  # noqa: E731
    Q, K, V = (r.standard_normal((B, H, T, d)) / np.sqrt(d) for _ in range(3))
    if bf16:
        (_, Q), (Kb, K), (Vb, V) = _bf16(Q), _bf16(K), _bf16(V)
        ins = [Kb, Vb]
    else:
        Q, K, V = (f(x).astype(np.float64) for x in (Q, K, V))
        ins = [f(K), f(V)]
    eta = f(0.5 * r.uniform(0.2, 1.0, (B, H, T)) / C)
    W0 = f(r.standard_normal((B, H, d, d) if w0seq else (H, d, d)) / np.sqrt(d))
    dZ = f(r.standard_normal((B, H, T, d)))
    dW = f(r.standard_normal((B, H, d, d))) if with_dw else None
    gram = _gram(Q, K, V, eta.astype(np.float64), dZ.astype(np.float64), C)
    out = {n: np.zeros((B, H, T, d), np.float32) for n in ("Q", "K", "V")}
    deta = np.zeros((B, H, T), np.float32)
    dW0 = np.zeros(W0.shape, np.float32)
    p = lambda a: a.ctypes.data if a is not None else None  # noqa: E731
    rc = emu.ttt_chunk_bwd_scan_tok_host_run(p(ins[0]), p(ins[1]), p(eta), p(dZ), p(W0), p(dW),
                                             p(gram), p(out["Q"]), p(out["K"]), p(out["V"]),
                                             p(deta), p(dW0), B, H, T, d, C, int(bf16), int(w0seq))
    assert rc == 0
    ref = ob.chunk_grads(Q, K, V, eta.astype(np.float64), W0.astype(np.float64),
                         dZ.astype(np.float64), None if dW is None else dW.astype(np.float64),
                         chunk=C)
    got = {"Q": out["Q"], "K": out["K"], "V": out["V"], "eta": deta, "W0": dW0}
    for k, gv in got.items():
        rv = ref[k]
        assert np.abs(gv - rv).max() <= TOL * max(np.abs(rv).max(), 1e-30), k


def test_planted_error_fails(emu):
    """A wrong Gram product (B_c with a flipped sign in one chunk) must fail."""
    B, H, T, d, C = 1, 1, 64, 64, 32
    r = np.random.default_rng(5)
    f = lambda a: np.ascontiguousarray(a, dtype=np.float32)  # noqa: E731
    Q, K, V = (f(r.standard_normal((B, H, T, d)) / np.sqrt(d)).astype(np.float64) for _ in range(3))
    eta = f(0.5 * r.uniform(0.2, 1.0, (B, H, T)) / C)
    W0 = f(r.standard_normal((H, d, d)) / np.sqrt(d))
    dZ = f(r.standard_normal((B, H, T, d)))
    dW = f(r.standard_normal((B, H, d, d)))
    gram = _gram(Q, K, V, eta.astype(np.float64), dZ.astype(np.float64), C)
    gram[0, 1] *= -1.0
    outs = [np.zeros((B, H, T, d), np.float32) for _ in range(3)]
    deta, dW0 = np.zeros((B, H, T), np.float32), np.zeros(W0.shape, np.float32)
    rc = emu.ttt_chunk_bwd_scan_tok_host_run(f(K).ctypes.data, f(V).ctypes.data, eta.ctypes.data,
                                             dZ.ctypes.data, W0.ctypes.data, dW.ctypes.data,
                                             gram.ctypes.data, *(o.ctypes.data for o in outs),
                                             deta.ctypes.data, dW0.ctypes.data, B, H, T, d, C, 0, 0)
    assert rc == 0
    ref = ob.chunk_grads(Q, K, V, eta.astype(np.float64), W0.astype(np.float64),
                         dZ.astype(np.float64), dW.astype(np.float64), chunk=C)
    assert np.abs(outs[0] - ref["Q"]).max() > TOL * np.abs(ref["Q"]).max()
