"""The single-issuer tensor-core TTT-MLP kernel (ttt_diag_mlp_fwd_tcgen05)
against the oracle, and the tcgen05 issue-cost probe that explains why
ttt_mlp_fwd runs the warp-level MMA kernel for these shapes instead.

The kernel computes the mini-batch dual form with every dense product as a
tcgen05.mma (hidden units on the MMA's M side, fp32 accumulators in tensor
memory) and the read-out of mini-batch m - 1 sharing a product with the key
side of mini-batch m (its causal term is then the strictly upper part of
Aq A^T against the next weights). It is held to the same tolerance as the
default kernel."""
import pytest
import torch

import test_sequence_layers_layer_b200 as ttt
from test_sequence_layers_layer_b200 import synth

from gpu_helpers import check_parity, run_gpu, to_dev

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS["mlp_ln_d64_dh256_b4h12_t8192"]

CASES = {
    "mlp_small": W.scaled(B=1, H=3, T=48),
    "mlp_T_eq_b": W.scaled(B=1, H=2, T=16),
    "mlp_150_seqs": W.scaled(B=10, H=15, T=32),
    "mlp_long": W.scaled(B=1, H=2, T=1024),
    "mlp_eta_varied": W.scaled(B=2, H=2, T=256, eta="sigmoid_over_d"),
}


@pytest.mark.parametrize("name", list(CASES))
def test_tcgen05_mlp_parity(name):
    inp = synth.make_inputs(CASES[name])
    check_parity(inp, gpu_out=run_gpu(inp, kernel="tcgen05"))


def test_tcgen05_mlp_full_size_small_step():
    """The full MLP workload with a 10x smaller inner step (well conditioned
    on every sequence): every sequence, every token, the final weights."""
    inp = synth.make_inputs(W.scaled(eta="sigmoid_over_d:0.1"))
    check_parity(inp, gpu_out=run_gpu(inp, kernel="tcgen05"))


def test_tcgen05_mlp_bf16_z_and_per_sequence_state():
    """bf16 Z is the fp32 run's Z rounded to bf16; per-sequence W0 matches
    the shared-W0 run."""
    wl = W.scaled(B=2, H=2, T=64)
    inp = synth.make_inputs(wl)
    x = to_dev(inp)
    args = (x["Q"], x["K"], x["V"], x["eta"], x["W1"], x["W2"], x["gamma"], x["beta"])
    Z, W1o, W2o = ttt.mlp_fwd(*args, b=16, kernel="tcgen05")
    Zb, _, _ = ttt.mlp_fwd(*args, b=16, kernel="tcgen05", z_bf16=True)
    W1s = x["W1"].unsqueeze(0).repeat(wl.B, 1, 1, 1)
    W2s = x["W2"].unsqueeze(0).repeat(wl.B, 1, 1, 1)
    Zs, W1p, W2p = ttt.mlp_fwd(x["Q"], x["K"], x["V"], x["eta"], W1s, W2s, x["gamma"], x["beta"],
                               b=16, kernel="tcgen05", w0_per_seq=True)
    torch.cuda.synchronize()
    assert ttt.ttt_device_status() == 0
    assert torch.equal(Zb, Z.to(torch.bfloat16))
    assert torch.equal(Zs, Z) and torch.equal(W1p, W1o) and torch.equal(W2p, W2o)


def test_tcgen05_mlp_rejects_other_shapes():
    wl = W.scaled(B=1, H=1, T=32, b=8)
    x = to_dev(synth.make_inputs(wl))
    Z = torch.empty((1, 1, 32, 64), device="cuda")
    rc = ttt.ttt_diag_mlp_fwd_tcgen05(x["Q"], x["K"], x["V"], x["eta"], x["W1"], x["W2"],
                                      x["gamma"], x["beta"], Z, None, None, 1, 1, 32, 64, 256, 8,
                                      ttt.TTT_BF16, ttt.TTT_F_LN, check=False)
    assert rc == -2


def test_umma_issue_cycles_probe():
    """The probe returns plausible cycle counts: issuing takes at most the
    time to completion, and 4x the instructions take at least 2x as long."""
    c = torch.zeros(2, dtype=torch.int64, device="cuda")
    ttt.ttt_diag_umma_issue_cycles(128, 32, 16, 1, c)
    torch.cuda.synchronize()
    few = c.cpu().numpy().copy()
    ttt.ttt_diag_umma_issue_cycles(128, 32, 64, 1, c)
    torch.cuda.synchronize()
    many = c.cpu().numpy().copy()
    assert ttt.ttt_device_status() == 0
    assert 0 < few[0] <= few[1] and 0 < many[0] <= many[1]
    assert many[1] >= 2 * few[1]
    assert ttt.ttt_diag_umma_issue_cycles(96, 32, 16, 1, c, check=False) == -2
    assert ttt.ttt_diag_umma_issue_cycles(128, 256, 16, 3, c, check=False) == -2
    assert ttt.ttt_diag_umma_issue_cycles(128, 32, 16, 1, None, check=False) == -5
