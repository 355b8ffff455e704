"""The TTT-MLP backward kernel's body (ttt_mlp_bwd_body.inc) run on the host
against the backward oracle (oracle/backward.py: float64 autograd through the
unrolled inner loop). The body is compiled with g++ into a test harness
(tests/host_emu/mlp_bwd_emu.cpp) that runs each sequence as one block of 256
OS threads, a std::barrier standing for every __syncthreads(): the same
arithmetic, indexing and barrier placement as on the GPU, in fp32.

Tolerance 1e-4 of each gradient's largest magnitude (fp32 arithmetic through
second-order LayerNorm and GELU terms; as for the TTT-Linear backward)."""
import ctypes
import os
import subprocess

import numpy as np
import pytest

from oracle import backward as ob

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "host_emu", "mlp_bwd_emu.cpp")
TOL = 1e-4


@pytest.fixture(scope="module")
def emu(tmp_path_factory):
    so = str(tmp_path_factory.mktemp("emu") / "mlp_bwd_emu.so")
    subprocess.run(["g++", "-std=c++20", "-O2", "-shared", "-fPIC", "-pthread", SRC, "-o", so],
                   check=True)
    L = ctypes.CDLL(so)
    L.ttt_mlp_bwd_host_run.restype = ctypes.c_int
    L.ttt_mlp_bwd_host_run.argtypes = [ctypes.c_void_p] * 19 + [ctypes.c_int] * 8
    return L


def _inputs(seed, B, H, T, d, w0_per_seq, eta_scale=0.3):
    r = np.random.default_rng(seed)
    dh = 4 * d
    Q, K, V = (r.standard_normal((B, H, T, d)) / np.sqrt(d) for _ in range(3))
    eta = eta_scale * r.uniform(0.2, 1.0, (B, H, T))
    lead = (B, H) if w0_per_seq else (H,)
    W1 = 0.5 * r.standard_normal(lead + (d, dh)) / np.sqrt(d)
    W2 = 0.5 * r.standard_normal(lead + (dh, d)) / np.sqrt(dh)
    g, be = 1 + 0.2 * r.standard_normal((H, d)), 0.2 * r.standard_normal((H, d))
    dZ = r.standard_normal((B, H, T, d))
    dW1 = r.standard_normal((B, H, d, dh))
    dW2 = r.standard_normal((B, H, dh, d))
    return Q, K, V, eta, W1, W2, g, be, dZ, dW1, dW2


def _run(L, Q, K, V, eta, W1, W2, g, be, dZ, dW1, dW2, *, b, w0_per_seq, bf16):
    B, H, T, d = Q.shape
    dh = 4 * d
    f32 = lambda a: np.ascontiguousarray(a, dtype=np.float32)  # noqa: E731
    if bf16:  # inputs rounded to bf16 (round to nearest even), passed as raw bits
        def bits(a):
            u = f32(a).view(np.uint32)
            return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
        Qb, Kb, Vb = bits(Q), bits(K), bits(V)
        Q, K, V = ((x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
                   for x in (Qb, Kb, Vb))
        ins = [Qb, Kb, Vb]
    else:
        Q, K, V = (f32(x).astype(np.float64) for x in (Q, K, V))
        ins = [f32(Q), f32(K), f32(V)]
    rest = [f32(eta), f32(W1), f32(W2), f32(g), f32(be), f32(dZ),
            None if dW1 is None else f32(dW1), None if dW2 is None else f32(dW2)]
    out = dict(Q=np.zeros((B, H, T, d), np.float32), K=np.zeros((B, H, T, d), np.float32),
               V=np.zeros((B, H, T, d), np.float32), eta=np.zeros((B, H, T), np.float32),
               W1=np.zeros(W1.shape, np.float32), W2=np.zeros(W2.shape, np.float32),
               gamma=np.zeros((H, d), np.float32), beta=np.zeros((H, d), np.float32))
    ptr = lambda a: None if a is None else a.ctypes.data  # noqa: E731
    rc = L.ttt_mlp_bwd_host_run(*[ptr(a) for a in ins + rest],
                                *[ptr(out[k]) for k in ("Q", "K", "V", "eta", "W1", "W2", "gamma",
                                                        "beta")],
                                B, H, T, d, b, int(bf16), int(w0_per_seq), 256)
    assert rc == 0
    # the oracle sees exactly what the kernel saw (fp32-rounded weights and steps)
    ref = ob.mlp_grads(Q, K, V, f32(eta), f32(W1), f32(W2), f32(g), f32(be), f32(dZ),
                       None if dW1 is None else f32(dW1), None if dW2 is None else f32(dW2), b=b)
    return out, ref


@pytest.mark.parametrize("B,H,T,d,b,w0_per_seq,bf16,with_dw", [
    (1, 2, 8, 16, 4, False, False, True),
    (2, 1, 8, 16, 2, True, False, False),
    (2, 2, 6, 16, 3, False, True, True),
    (1, 1, 4, 32, 4, False, False, True),
    (1, 1, 32, 64, 16, False, True, True),   # the TTT-MLP workload's shape (d 64, dh 256, b 16)
])
def test_host_run_matches_oracle(emu, B, H, T, d, b, w0_per_seq, bf16, with_dw):
    Q, K, V, eta, W1, W2, g, be, dZ, dW1, dW2 = _inputs(7 + T + d, B, H, T, d, w0_per_seq)
    if not with_dw:
        dW1 = dW2 = None
    got, ref = _run(emu, Q, K, V, eta, W1, W2, g, be, dZ, dW1, dW2, b=b, w0_per_seq=w0_per_seq,
                    bf16=bf16)
    errs = {}
    for k, r in ref.items():
        gk = got[k].astype(np.float64).reshape(r.shape)
        errs[k] = float(np.abs(gk - r).max() / max(np.abs(r).max(), 1e-30))
    assert max(errs.values()) <= TOL, errs
