"""The affine-map kernels of the sequence-parallel forward (ttt_affine.cu) run
on the host (tests/host_emu/affine_emu.cpp, 256 OS threads per block and a
std::barrier per __syncthreads()) against the oracle's fold
(oracle/affine.py), in both stride layouts the library uses; the same cases
run on the GPU in tests/test_seqpar_gpu.py."""
import ctypes
import os
import subprocess

import numpy as np
import pytest

from oracle import affine

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "host_emu", "affine_emu.cpp")


@pytest.fixture(scope="module")
def emu(tmp_path_factory):
    so = str(tmp_path_factory.mktemp("emu") / "affine_emu.so")
    subprocess.run(["g++", "-std=c++20", "-O2", "-shared", "-fPIC", "-pthread",
                    "-I/usr/local/cuda/include", SRC, "-o", so], check=True)
    L = ctypes.CDLL(so)
    L.ttt_affine_prefix_host_run.restype = ctypes.c_int
    L.ttt_affine_prefix_host_run.argtypes = ([ctypes.c_void_p] * 5 + [ctypes.c_int] * 4
                                             + [ctypes.c_longlong] * 2 + [ctypes.c_int])
    L.ttt_affine_eye_host_run.restype = ctypes.c_int
    L.ttt_affine_eye_host_run.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int]
    return L


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("layout", ["sequence_major", "segment_major"])
@pytest.mark.parametrize("per_seq,with_end", [(False, True), (True, False)])
def test_fold_matches_oracle(emu, d, layout, per_seq, with_end):
    B, H, nseg = 1, 2, 3
    S = B * H
    r = np.random.default_rng(d + nseg + int(per_seq))
    Ms = (np.eye(d) + 0.3 * r.standard_normal((S, nseg, d, d)) / np.sqrt(d)).astype(np.float32)
    Ns = (0.1 * r.standard_normal((S, nseg, d, d))).astype(np.float32)
    W0 = (r.standard_normal((S, d, d) if per_seq else (H, d, d)) / np.sqrt(d)).astype(np.float32)
    dd = d * d
    if layout == "sequence_major":
        M, N = np.ascontiguousarray(Ms), np.ascontiguousarray(Ns)
        seq_stride, seg_stride = nseg * dd, dd
    else:
        M, N = (np.ascontiguousarray(a.transpose(1, 0, 2, 3)) for a in (Ms, Ns))
        seq_stride, seg_stride = dd, S * dd
    W_in = np.full(M.shape, np.nan, np.float32)
    W_end = np.zeros((S, d, d), np.float32)
    assert emu.ttt_affine_prefix_host_run(M.ctypes.data, N.ctypes.data, W0.ctypes.data,
                                          W_in.ctypes.data, W_end.ctypes.data if with_end else None,
                                          S, H, nseg, d, seq_stride, seg_stride, int(per_seq)) == 0
    got = W_in if layout == "sequence_major" else W_in.transpose(1, 0, 2, 3)
    w0 = W0 if per_seq else W0[np.arange(S) % H]
    ref_in, ref_end = affine.prefix_weights(
        [(Ms[:, j].astype(np.float64), Ns[:, j].astype(np.float64)) for j in range(nseg)], w0)
    for j in range(nseg):
        g = got[:, j].astype(np.float64)
        assert np.abs(g - ref_in[j]).max() <= 1e-5 * np.abs(ref_in[j]).max(), j
    if with_end:
        assert np.abs(W_end - ref_end).max() <= 1e-5 * np.abs(ref_end).max()


def test_identity_fill(emu):
    W = np.full((5, 64, 64), 7.0, np.float32)
    assert emu.ttt_affine_eye_host_run(W.ctypes.data, 5, 64) == 0
    assert np.array_equal(W, np.broadcast_to(np.eye(64, dtype=np.float32), W.shape))
