"""Parity of the CUDA path (through the C ABI) against the CPU oracle.

Small cases span several mini-batches/chunks, sequence counts that do not
fill the machine evenly (150 > 148 SMs) and the degenerate shapes; the
full-size workloads are checked on sampled sequences (each sequence is
independent, so the oracle computes exactly those sequences)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import test_sequence_layers_layer_b200 as ttt
from test_sequence_layers_layer_b200 import synth

from conditioning import conditioned_horizon
from gpu_helpers import check_parity, run_gpu, to_dev, TOL, max_rel_err, run_oracle

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS

SMALL = {
    # fp32 CUDA-core path
    "linear_fp32_d16_full": W["linear_fp32_d16"],
    "linear_fp32_d64_noln": W["linear_fp32_d16"].scaled(B=2, H=3, T=128, d=64, b=16),
    "linear_fp32_d32_ln_b8": W["linear_fp32_d16"].scaled(B=2, H=2, T=64, d=32, b=8, ln=True,
                                                         eta="sigmoid_over_d"),
    "linear_fp32_d16_b1": W["linear_fp32_d16"].scaled(T=32, b=1),
    "linear_fp32_d64_ln_b64": W["linear_fp32_d16"].scaled(B=1, H=2, T=128, d=64, b=64, ln=True,
                                                          eta="sigmoid_over_d"),
    # bf16 linear + LN, d=64, b=16
    "linear_ln_small": W["linear_ln_d64_b8h12_t2048"].scaled(B=2, H=3, T=64),
    "linear_ln_T_eq_b": W["linear_ln_d64_b8h12_t2048"].scaled(B=1, H=5, T=16),
    "linear_ln_T_3b": W["linear_ln_d64_b8h12_t2048"].scaled(B=1, H=3, T=48),
    "linear_ln_150_seqs": W["linear_ln_d64_b8h12_t2048"].scaled(B=10, H=15, T=32),
    "linear_ln_long": W["linear_ln_d64_b8h12_t2048"].scaled(B=1, H=2, T=1024),
    "linear_noln_bf16": W["linear_ln_d64_b8h12_t2048"].scaled(B=2, H=2, T=128, ln=False),
    # partial last mini-batch (T not a multiple of b): tensor-core path with 3
    # full mini-batches + 2 tokens, a lone partial one, and one past a 64-token
    # TMA chunk; the fp32 path; and bf16 with b = 32 (fp32 kernel)
    "linear_ln_partial_T50": W["linear_ln_d64_b8h12_t2048"].scaled(B=2, H=3, T=50),
    "linear_ln_partial_T7": W["linear_ln_d64_b8h12_t2048"].scaled(B=1, H=2, T=7),
    "linear_ln_partial_T130": W["linear_ln_d64_b8h12_t2048"].scaled(B=1, H=3, T=130),
    "linear_noln_partial_T41": W["linear_ln_d64_b8h12_t2048"].scaled(B=2, H=1, T=41, ln=False),
    "linear_fp32_partial_T37": W["linear_fp32_d16"].scaled(B=2, H=2, T=37, d=32, b=8, ln=True,
                                                          eta="sigmoid_over_d"),
    "linear_bf16_b32_partial_T70": W["linear_ln_d64_b8h12_t2048"].scaled(B=1, H=2, T=70, b=32),
    # MLP
    "mlp_small": W["mlp_ln_d64_dh256_b4h12_t8192"].scaled(B=1, H=3, T=48),
    "mlp_fp32_d16": W["mlp_ln_d64_dh256_b4h12_t8192"].scaled(B=2, H=2, T=32, d=16, dh=64, b=4,
                                                             dtype="fp32"),
    "mlp_T_eq_b": W["mlp_ln_d64_dh256_b4h12_t8192"].scaled(B=1, H=2, T=16),
    "mlp_150_seqs": W["mlp_ln_d64_dh256_b4h12_t8192"].scaled(B=10, H=15, T=32),
    "mlp_long": W["mlp_ln_d64_dh256_b4h12_t8192"].scaled(B=1, H=2, T=1024),
    "mlp_eta_varied": W["mlp_ln_d64_dh256_b4h12_t8192"].scaled(B=2, H=2, T=256, eta="sigmoid_over_d"),
    # large chunk
    "chunk_small": W["chunk_d128_c2048_b4h8_t32768"].scaled(B=1, H=3, T=768, b=256,
                                                            eta="const:0.00390625"),
    "chunk_two_chunks": W["chunk_d128_c2048_b4h8_t32768"].scaled(B=1, H=2, T=4096),
    "chunk_d64": W["chunk_d128_c2048_b4h8_t32768"].scaled(B=2, H=1, T=512, d=64, b=128,
                                                          eta="const:0.0078125"),
    "chunk_c128": W["chunk_d128_c2048_b4h8_t32768"].scaled(B=2, H=2, T=512, b=128,
                                                           eta="const:0.0078125"),
    "chunk_single_chunk": W["chunk_d128_c2048_b4h8_t32768"].scaled(B=1, H=5, T=256, b=256,
                                                                   eta="const:0.00390625"),
    "chunk_150_chunks": W["chunk_d128_c2048_b4h8_t32768"].scaled(B=10, H=15, T=128, b=128,
                                                                 eta="const:0.0078125"),
    "chunk_eta_varied": W["chunk_d128_c2048_b4h8_t32768"].scaled(B=1, H=2, T=1024, b=512,
                                                                 eta="sigmoid_over_d"),
    "chunk_fp32": W["chunk_d128_c2048_b4h8_t32768"].scaled(B=1, H=2, T=512, b=256,
                                                           dtype="fp32", eta="const:0.00390625"),
}


# cases carrying the "late" marker, which conftest collects after all others
LATE_SMALL = {"linear_ln_T_3b"}


@pytest.mark.parametrize("name", [pytest.param(n, marks=pytest.mark.late) if n in LATE_SMALL
                                  else n for n in SMALL])
def test_small_parity(name):
    check_parity(synth.make_inputs(SMALL[name]))


FULL = [
    ("linear_fp32_d16", None),
    ("linear_ln_d64_b8h12_t2048", None),
    ("linear_ln_d64_b1h32_t32768", None),
    ("chunk_d128_c2048_b4h8_t32768", None),
]


@pytest.mark.parametrize("name,seqs", FULL, ids=[f[0] for f in FULL])
def test_full_size_parity(name, seqs):
    inp = synth.make_inputs(W[name])
    errs = check_parity(inp, seqs=seqs)
    print(f"{name}: max rel err {errs}")


def test_full_size_partial_last_minibatch():
    """The bench workload's shape with T = 2047 (127 full mini-batches and one
    of 15 tokens) in one launch, every sequence against the oracle."""
    inp = synth.make_inputs(W["linear_ln_d64_b8h12_t2048"].scaled(T=2047))
    errs = check_parity(inp)
    print(f"linear T=2047: max rel err {errs}")


def test_mlp_full_size_parity_conditioned():
    """Every sequence of the full MLP workload. The recurrence with this step
    size is chaotic on some sequences (see test_conditioning): there even the
    exact result moves by O(1) under rounding-size input changes after a few
    thousand tokens, so no finite-precision path can follow it. A sequence
    counts as conditioned when the oracle, fed inputs changed by 3e-5 relative
    (2^-15, the precision of a two-term bf16 operand), stays within half the
    tolerance over all tokens; those are compared over all tokens and their
    final weights. The others are compared over their first 2048 tokens, which
    the same probe shows the exact recurrence still tracks."""
    wl = W["mlp_ln_d64_dh256_b4h12_t8192"]
    tol = TOL[wl.dtype]
    inp = synth.make_inputs(wl)
    horizon, ref = conditioned_horizon(inp, noise=3e-5, rel=tol / 2)
    Z, W1o, W2o = run_gpu(inp)
    n = wl.B * wl.H
    Zg, Zr = Z.reshape(n, wl.T, wl.d), ref[0].reshape(n, wl.T, wl.d)
    scale = np.abs(Zr).max()
    full = horizon == wl.T
    prefix = np.where(full, wl.T, 2048)
    errs = np.array([np.abs(Zg[s, :p] - Zr[s, :p]).max() / scale for s, p in enumerate(prefix)])
    cond = np.where(full)[0]
    e1 = max_rel_err(W1o, ref[1], wl, cond)
    e2 = max_rel_err(W2o, ref[2], wl, cond)
    print(f"{len(cond)}/{n} sequences conditioned over all T (shortest horizon {horizon.min()}); "
          f"Z err conditioned {errs[full].max():.2e}, chaotic prefixes {errs[~full].max():.2e}; "
          f"W1 {e1:.2e} W2 {e2:.2e}")
    assert len(cond) >= 32 and horizon.min() >= 2560
    assert errs.max() <= tol and max(e1, e2) <= tol


def test_mlp_fp32_kernel_also_departs_on_a_chaotic_sequence():
    """The rule above rests on the recurrence, not on the bf16 kernel: the
    fp32 CUDA-core kernel, fed the same (bf16-valued) inputs in fp32, tracks
    the oracle on the chaotic sequence of the full MLP workload for its first
    1,024 tokens and then departs from it by O(1), while on a sequence the
    oracle's own perturbation probe calls conditioned it stays within the
    fp32 tolerance over all 8,192 tokens."""
    wl = W["mlp_ln_d64_dh256_b4h12_t8192"]
    inp = synth.make_inputs(wl)
    chaotic, calm = 20, 0
    horizon, _ = conditioned_horizon(inp, seqs=[calm])
    assert horizon[0] == wl.T
    ref = run_oracle(inp, seqs=[chaotic, calm])
    for k, seq in enumerate((chaotic, calm)):
        b, h = divmod(seq, wl.H)
        f = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()  # noqa: E731
        Q, K, V = (f(a[b:b + 1, h:h + 1]) for a in (inp.Q, inp.K, inp.V))
        eta = f(inp.eta[b:b + 1, h:h + 1])
        W1, W2 = f(inp.W1[h:h + 1]), f(inp.W2[h:h + 1])
        g, be = f(inp.gamma[h:h + 1]), f(inp.beta[h:h + 1])
        Z, _, _ = ttt.mlp_fwd(Q, K, V, eta, W1, W2, g, be, b=wl.b)
        torch.cuda.synchronize()
        assert ttt.ttt_device_status() == 0
        Zg = Z.double().cpu().numpy().reshape(wl.T, wl.d)
        Zr = ref[0].reshape(wl.B * wl.H, wl.T, wl.d)[seq]
        err = np.abs(Zg - Zr).max(axis=1) / np.abs(Zr).max()
        print(f"fp32 kernel, sequence {seq}: first 1024 tokens {err[:1024].max():.2e}, "
              f"all tokens {err.max():.2e}")
        if seq == chaotic:
            assert err[:1024].max() <= TOL["fp32"] and err.max() > 1e-2
        else:
            assert err.max() <= TOL["fp32"]


def test_mlp_full_size_parity_small_step():
    """The full MLP workload with a 10x smaller inner step, which is well
    conditioned on every sequence: all sequences, all tokens, final weights."""
    inp = synth.make_inputs(W["mlp_ln_d64_dh256_b4h12_t8192"].scaled(eta="sigmoid_over_d:0.1"))
    errs = check_parity(inp)
    print(f"mlp small step: max rel err {errs}")


# ------------------------------------------------------------------ edge cases

def test_eta_zero_keeps_initial_weight():
    wl = W["linear_ln_d64_b8h12_t2048"].scaled(B=1, H=2, T=64)
    inp = synth.make_inputs(wl)
    inp.eta[:] = 0
    Z, Wo = run_gpu(inp)
    np.testing.assert_array_equal(Wo[0], inp.W1.astype(np.float64))
    check_parity(inp)


@pytest.mark.parametrize("name", ["linear_ln_small", "linear_fp32_d64_noln"])
def test_resume_split_equals_whole(name):
    wl = SMALL[name]
    inp = synth.make_inputs(wl)
    x = to_dev(inp)
    Zw, Ww = ttt.linear_fwd(x["Q"], x["K"], x["V"], x["eta"], x["W1"], x["gamma"], x["beta"],
                            b=wl.b, ln=wl.ln)
    h = wl.T // 2
    sl = lambda t: t[:, :, :h].contiguous()
    sr = lambda t: t[:, :, h:].contiguous()
    Z1, W1 = ttt.linear_fwd(sl(x["Q"]), sl(x["K"]), sl(x["V"]), sl(x["eta"]), x["W1"],
                            x["gamma"], x["beta"], b=wl.b, ln=wl.ln)
    Z2, W2 = ttt.linear_fwd(sr(x["Q"]), sr(x["K"]), sr(x["V"]), sr(x["eta"]), W1,
                            x["gamma"], x["beta"], b=wl.b, ln=wl.ln, w0_per_seq=True)
    torch.cuda.synchronize()
    tol = TOL[wl.dtype]
    assert max_rel_err(torch.cat([Z1, Z2], 2).cpu().numpy(), Zw.cpu().numpy(), wl) <= tol
    assert max_rel_err(W2.cpu().numpy(), Ww.cpu().numpy(), wl) <= tol


def test_w_out_null_and_alias():
    wl = SMALL["linear_ln_small"]
    inp = synth.make_inputs(wl)
    x = to_dev(inp)
    Z0, W0o = ttt.linear_fwd(x["Q"], x["K"], x["V"], x["eta"], x["W1"], x["gamma"], x["beta"],
                             b=16, ln=True)
    Zn, none = ttt.linear_fwd(x["Q"], x["K"], x["V"], x["eta"], x["W1"], x["gamma"], x["beta"],
                              b=16, ln=True, want_w=False)
    assert none is None
    torch.testing.assert_close(Zn, Z0, rtol=0, atol=0)
    # in-place state update: W_out aliases a per-sequence W0
    Wps = x["W1"].unsqueeze(0).repeat(wl.B, 1, 1, 1)
    Z = torch.empty_like(Z0)
    ttt.ttt_linear_fwd(x["Q"], x["K"], x["V"], x["eta"], Wps, x["gamma"], x["beta"], Z, Wps,
                       wl.B, wl.H, wl.T, 64, 16, ttt.TTT_BF16, ttt.TTT_F_LN | ttt.TTT_F_W0_PER_SEQ)
    torch.cuda.synchronize()
    torch.testing.assert_close(Z, Z0, rtol=0, atol=0)
    torch.testing.assert_close(Wps, W0o, rtol=0, atol=0)


def test_deterministic():
    inp = synth.make_inputs(SMALL["linear_ln_150_seqs"])
    x = to_dev(inp)
    a = run_gpu(inp, x)
    b = run_gpu(inp, x)
    for u, v in zip(a, b):
        np.testing.assert_array_equal(u, v)


def test_rejects_host_and_misaligned_pointers():
    wl = SMALL["linear_ln_small"]
    inp = synth.make_inputs(wl)
    x = to_dev(inp)
    Z = torch.empty((wl.B, wl.H, wl.T, 64), device="cuda")
    host_q = torch.from_numpy(inp.Q_bits.view(np.int16)).view(torch.bfloat16)
    args = lambda Q, Zp: (Q, x["K"], x["V"], x["eta"], x["W1"], x["gamma"], x["beta"], Zp, None,
                          wl.B, wl.H, wl.T, 64, 16, ttt.TTT_BF16, ttt.TTT_F_LN)
    assert ttt.ttt_linear_fwd(*args(host_q, Z), check=False) == -5
    assert ttt.ttt_linear_fwd(*args(x["Q"].data_ptr() + 2, Z), check=False) == -4
    assert ttt.ttt_linear_fwd(*args(x["Q"], Z), check=False) == 0
    torch.cuda.synchronize()


def test_mlp_resume_split_equals_whole():
    wl = SMALL["mlp_long"].scaled(T=256)
    inp = synth.make_inputs(wl)
    x = to_dev(inp)
    args = (x["gamma"], x["beta"])
    Zw, W1w, W2w = ttt.mlp_fwd(x["Q"], x["K"], x["V"], x["eta"], x["W1"], x["W2"], *args, b=wl.b)
    h = wl.T // 2
    sl = lambda t: t[:, :, :h].contiguous()
    sr = lambda t: t[:, :, h:].contiguous()
    Z1, W1a, W2a = ttt.mlp_fwd(sl(x["Q"]), sl(x["K"]), sl(x["V"]), sl(x["eta"]), x["W1"], x["W2"],
                               *args, b=wl.b)
    Z2, W1b, W2b = ttt.mlp_fwd(sr(x["Q"]), sr(x["K"]), sr(x["V"]), sr(x["eta"]), W1a, W2a, *args,
                               b=wl.b, w0_per_seq=True)
    torch.cuda.synchronize()
    # The same kernel on the same values: the split run reproduces the whole run exactly.
    torch.testing.assert_close(torch.cat([Z1, Z2], 2), Zw, rtol=0, atol=0)
    torch.testing.assert_close(W1b, W1w, rtol=0, atol=0)
    torch.testing.assert_close(W2b, W2w, rtol=0, atol=0)


def test_mlp_deterministic_and_w_out_null():
    wl = SMALL["mlp_150_seqs"]
    inp = synth.make_inputs(wl)
    x = to_dev(inp)
    a = run_gpu(inp, x)
    b = run_gpu(inp, x)
    for u, v in zip(a, b):
        np.testing.assert_array_equal(u, v)
    Zn, n1, n2 = ttt.mlp_fwd(x["Q"], x["K"], x["V"], x["eta"], x["W1"], x["W2"], x["gamma"],
                             x["beta"], b=wl.b, want_w=False)
    torch.cuda.synchronize()
    assert n1 is None and n2 is None
    np.testing.assert_array_equal(Zn.cpu().numpy().astype(np.float64), a[0])


def test_chunk_resume_split_equals_whole():
    wl = SMALL["chunk_c128"]
    inp = synth.make_inputs(wl)
    x = to_dev(inp)
    Zw, Ww = ttt.chunk_fwd(x["Q"], x["K"], x["V"], x["eta"], x["W1"], chunk=wl.b)
    h = wl.T // 2
    sl = lambda t: t[:, :, :h].contiguous()
    sr = lambda t: t[:, :, h:].contiguous()
    Z1, W1 = ttt.chunk_fwd(sl(x["Q"]), sl(x["K"]), sl(x["V"]), sl(x["eta"]), x["W1"], chunk=wl.b)
    Z2, W2 = ttt.chunk_fwd(sr(x["Q"]), sr(x["K"]), sr(x["V"]), sr(x["eta"]), W1, chunk=wl.b,
                           w0_per_seq=True)
    torch.cuda.synchronize()
    assert max_rel_err(torch.cat([Z1, Z2], 2).cpu().numpy(), Zw.cpu().numpy(), wl) <= 1e-6
    assert max_rel_err(W2.cpu().numpy(), Ww.cpu().numpy(), wl) <= 1e-6


def test_chunk_rejects_small_workspace():
    wl = SMALL["chunk_c128"]
    inp = synth.make_inputs(wl)
    x = to_dev(inp)
    Z = torch.empty((wl.B, wl.H, wl.T, wl.d), device="cuda")
    need = ttt.ttt_chunk_workspace_bytes(wl.B, wl.H, wl.T, wl.d, wl.b)
    n = wl.B * wl.H * (wl.T // wl.b)
    assert need == n * 160 * 1024 + 256  # per chunk 160 KiB; flags, counts and counter: 256 B
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    args = (x["Q"], x["K"], x["V"], x["eta"], x["W1"], Z, None, wl.B, wl.H, wl.T, wl.d, wl.b,
            ttt.TTT_BF16, 0)
    assert ttt.ttt_chunk_fwd(*args, ws, need - 256, check=False) == -9
    assert ttt.ttt_chunk_fwd(*args, None, need, check=False) == -9
    assert ttt.ttt_chunk_fwd(*args, ws, need, check=False) == 0
    torch.cuda.synchronize()
