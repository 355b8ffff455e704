"""Sequence-parallel forward on one GPU, through the C ABI: ttt_chunk_map and
ttt_linear_map against the oracle's affine segment maps (oracle/affine.py),
ttt_affine_prefix against a float64 fold in both stride layouts, and the
segmented forwards (seqpar.chunk_fwd_segmented, seqpar.linear_fwd_segmented)
against the oracle's forward of the whole sequence. Error metric and
tolerances as in the other parity tests: max |gpu - ref| / max |ref| per
output, 2e-3 for bf16 inputs, 1e-5 for fp32 inputs (the fold itself, fp32
throughout, within 1e-5)."""
import numpy as np
import pytest
import torch

import oracle
import test_sequence_layers_layer_b200 as ttt
from oracle import affine
from test_sequence_layers_layer_b200 import seqpar, synth
from gpu_helpers import TOL, to_dev

pytestmark = pytest.mark.gpu

W = synth.WORKLOADS["chunk_d128_c2048_b4h8_t32768"]
CASES = {
    # d = 128 bf16 runs the tensor-core forward; d = 64 and fp32 the CUDA-core one
    "bf16_d128_c128": W.scaled(B=2, H=2, T=1024, b=128, eta="const:0.0078125"),
    "bf16_d128_c256_eta_varied": W.scaled(B=1, H=3, T=1024, b=256, eta="sigmoid_over_d"),
    "bf16_d64_c128": W.scaled(B=2, H=1, T=512, d=64, b=128, eta="const:0.0078125"),
    "fp32_d128_c128": W.scaled(B=1, H=2, T=512, b=128, dtype="fp32", eta="const:0.0078125"),
}


def _rel(g, r):
    return float(np.abs(g - r).max() / max(np.abs(r).max(), 1e-30))


def _np(t):
    return t.double().cpu().numpy()


@pytest.mark.parametrize("name", list(CASES))
def test_chunk_map_matches_oracle(name):
    wl = CASES[name]
    inp = synth.make_inputs(wl)
    x = to_dev(inp)
    M, N = ttt.chunk_map(x["K"], x["V"], x["eta"], chunk=wl.b)
    torch.cuda.synchronize()
    assert ttt.ttt_device_status() == 0
    Mr, Nr = affine.segment_map(inp.K, inp.V, inp.eta, chunk=wl.b)
    assert _rel(_np(M), Mr) <= TOL[wl.dtype]
    assert _rel(_np(N), Nr) <= TOL[wl.dtype]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("layout", ["sequence_major", "segment_major"])
@pytest.mark.parametrize("per_seq,with_end", [(False, True), (True, False)])
def test_affine_prefix_matches_float64_fold(d, layout, per_seq, with_end):
    B, H, nseg = 2, 3, 4
    S = B * H
    r = np.random.default_rng(d + nseg)
    Ms = (np.eye(d) + 0.3 * r.standard_normal((S, nseg, d, d)) / np.sqrt(d)).astype(np.float32)
    Ns = (0.1 * r.standard_normal((S, nseg, d, d))).astype(np.float32)
    W0 = (r.standard_normal((S, d, d) if per_seq else (H, d, d)) / np.sqrt(d)).astype(np.float32)
    dd = d * d
    if layout == "sequence_major":
        arr = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
        back = lambda t: _np(t).reshape(S, nseg, d, d)  # noqa: E731
        seq_stride, seg_stride = nseg * dd, dd
    else:
        arr = lambda a: torch.from_numpy(np.ascontiguousarray(a.transpose(1, 0, 2, 3))).cuda()  # noqa: E731
        back = lambda t: _np(t).reshape(nseg, S, d, d).transpose(1, 0, 2, 3)  # noqa: E731
        seq_stride, seg_stride = dd, S * dd
    M, N = arr(Ms), arr(Ns)
    W_in = torch.full_like(M, float("nan"))
    W_end = torch.empty((S, d, d), device="cuda") if with_end else None
    ttt.affine_prefix(M, N, torch.from_numpy(W0).cuda(), W_in, W_end, S=S, H=H, nseg=nseg,
                      seq_stride=seq_stride, seg_stride=seg_stride, w0_per_seq=per_seq)
    torch.cuda.synchronize()
    w0 = W0 if per_seq else W0[np.arange(S) % H]
    ref_in, ref_end = affine.prefix_weights(
        [(Ms[:, j].astype(np.float64), Ns[:, j].astype(np.float64)) for j in range(nseg)], w0)
    got = back(W_in)
    for j in range(nseg):
        assert _rel(got[:, j], ref_in[j]) <= 1e-5, j
    assert np.array_equal(got[:, 0], w0.astype(np.float64))  # W_in[0] is W0, copied
    if with_end:
        assert _rel(_np(W_end), ref_end) <= 1e-5


@pytest.mark.parametrize("name,nseg", [("bf16_d128_c128", 1), ("bf16_d128_c128", 2),
                                       ("bf16_d128_c128", 8), ("bf16_d128_c256_eta_varied", 4),
                                       ("bf16_d64_c128", 4), ("fp32_d128_c128", 2)])
def test_segmented_forward_matches_whole_sequence(name, nseg):
    wl = CASES[name]
    inp = synth.make_inputs(wl)
    x = to_dev(inp)
    Z, W_out = seqpar.chunk_fwd_segmented(x["Q"], x["K"], x["V"], x["eta"], x["W1"], chunk=wl.b,
                                          nseg=nseg)
    torch.cuda.synchronize()
    assert ttt.ttt_device_status() == 0
    Zr, Wr = oracle.chunk_primal(inp.Q, inp.K, inp.V, inp.eta, inp.W1, chunk=wl.b)
    assert _rel(_np(Z), Zr) <= TOL[wl.dtype]
    assert _rel(_np(W_out), Wr) <= TOL[wl.dtype]
    # and against the unsegmented library forward
    Zc, Wc = ttt.chunk_fwd(x["Q"], x["K"], x["V"], x["eta"], x["W1"], chunk=wl.b)
    assert _rel(_np(Z), _np(Zc)) <= TOL[wl.dtype]


def test_segmented_forward_per_sequence_w0_and_bf16_z():
    wl = CASES["bf16_d128_c128"]
    inp = synth.make_inputs(wl)
    x = to_dev(inp)
    r = np.random.default_rng(5)
    W0 = (np.broadcast_to(inp.W1[None], (wl.B,) + inp.W1.shape)
          + 0.01 * r.standard_normal((wl.B,) + inp.W1.shape)).astype(np.float32)
    W0d = torch.from_numpy(W0).cuda()
    Z, W_out = seqpar.chunk_fwd_segmented(x["Q"], x["K"], x["V"], x["eta"], W0d, chunk=wl.b,
                                          nseg=4, w0_per_seq=True)
    Zb, W_outb = seqpar.chunk_fwd_segmented(x["Q"], x["K"], x["V"], x["eta"], W0d, chunk=wl.b,
                                            nseg=4, w0_per_seq=True, z_bf16=True)
    torch.cuda.synchronize()
    assert ttt.ttt_device_status() == 0
    Zr, Wr = oracle.chunk_primal(inp.Q, inp.K, inp.V, inp.eta, W0, chunk=wl.b, w0_per_seq=True)
    assert _rel(_np(Z), Zr) <= TOL[wl.dtype] and _rel(_np(W_out), Wr) <= TOL[wl.dtype]
    assert torch.equal(Zb, Z.to(torch.bfloat16)) and torch.equal(W_outb, W_out)


def test_segmented_full_size_sampled_sequences():
    """The large-chunk workload (B=4, H=8, T=32768, d=128, chunk 2048, bf16)
    in four segments of four chunks: two sequences against the oracle."""
    wl = W
    inp = synth.make_inputs(wl)
    x = to_dev(inp)
    Z, W_out = seqpar.chunk_fwd_segmented(x["Q"], x["K"], x["V"], x["eta"], x["W1"], chunk=wl.b,
                                          nseg=4)
    torch.cuda.synchronize()
    assert ttt.ttt_device_status() == 0
    Zr, Wr = oracle.chunk_primal(inp.Q, inp.K, inp.V, inp.eta, inp.W1, chunk=wl.b, seqs=[0, 31])
    Zg = _np(Z).reshape(wl.B * wl.H, wl.T, wl.d)
    Wg = _np(W_out).reshape(wl.B * wl.H, wl.d, wl.d)
    Zo = Zr.reshape(wl.B * wl.H, wl.T, wl.d)
    Wo = Wr.reshape(wl.B * wl.H, wl.d, wl.d)
    for s in (0, 31):
        assert _rel(Zg[s], Zo[s]) <= TOL["bf16"] and _rel(Wg[s], Wo[s]) <= TOL["bf16"]


# ------------------------------------------------------- TTT-Linear without LN
L = synth.WORKLOADS["linear_ln_d64_b8h12_t2048"]
LINEAR_CASES = {
    # bf16, d = 64, b = 16 runs the tensor-core scan; fp32 the CUDA-core kernel
    "linear_noln_bf16_d64_b16": L.scaled(B=2, H=2, T=512, ln=False),
    "linear_noln_fp32_d64_b8": L.scaled(B=1, H=3, T=256, b=8, ln=False, dtype="fp32"),
}


@pytest.mark.late
@pytest.mark.parametrize("name", list(LINEAR_CASES))
def test_linear_map_matches_oracle(name):
    wl = LINEAR_CASES[name]
    inp = synth.make_inputs(wl)
    x = to_dev(inp)
    M, N = ttt.linear_map(x["K"], x["V"], x["eta"], b=wl.b)
    torch.cuda.synchronize()
    assert ttt.ttt_device_status() == 0
    Mr, Nr = affine.segment_map(inp.K, inp.V, inp.eta, chunk=wl.b)
    assert _rel(_np(M), Mr) <= TOL[wl.dtype]
    assert _rel(_np(N), Nr) <= TOL[wl.dtype]


@pytest.mark.late
@pytest.mark.parametrize("name,nseg", [("linear_noln_bf16_d64_b16", 2),
                                       ("linear_noln_bf16_d64_b16", 8),
                                       ("linear_noln_fp32_d64_b8", 4)])
def test_linear_segmented_forward_matches_whole_sequence(name, nseg):
    wl = LINEAR_CASES[name]
    inp = synth.make_inputs(wl)
    x = to_dev(inp)
    Z, W_out = seqpar.linear_fwd_segmented(x["Q"], x["K"], x["V"], x["eta"], x["W1"], b=wl.b,
                                           nseg=nseg)
    torch.cuda.synchronize()
    assert ttt.ttt_device_status() == 0
    Zr, Wr = oracle.linear_primal(inp.Q, inp.K, inp.V, inp.eta, inp.W1, b=wl.b, ln=False)
    assert _rel(_np(Z), Zr) <= TOL[wl.dtype]
    assert _rel(_np(W_out), Wr) <= TOL[wl.dtype]
    Zc, _ = ttt.linear_fwd(x["Q"], x["K"], x["V"], x["eta"], x["W1"], b=wl.b, ln=False)
    assert _rel(_np(Z), _np(Zc)) <= TOL[wl.dtype]
