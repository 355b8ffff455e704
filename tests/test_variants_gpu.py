"""TTT-Linear variants through the C ABI against the variant oracle
(oracle/variants.py): L2-normalised keys (TTT_F_L2_KEYS; the plain forward on
keys scaled to unit length) and several gradient steps per token
(ttt_linear_fwd_steps). Tolerances as in the other parity tests: 2e-3 for
bf16 inputs, 1e-5 for fp32 inputs."""
import numpy as np
import pytest
import torch

import oracle
import test_sequence_layers_layer_b200 as ttt
from oracle import variants
from test_sequence_layers_layer_b200 import synth
from gpu_helpers import TOL, to_dev

pytestmark = [pytest.mark.gpu, pytest.mark.late]

L = synth.WORKLOADS["linear_ln_d64_b8h12_t2048"]
CASES = {
    "ln_bf16_d64_b16": L.scaled(B=2, H=3, T=256),           # the tensor-core shape
    "noln_bf16_d64_b16_partial": L.scaled(B=1, H=2, T=41, ln=False),
    "noln_fp32_d16_b16": synth.WORKLOADS["linear_fp32_d16"].scaled(B=2, H=2, T=128),
    "ln_fp32_d32_b8": L.scaled(B=1, H=2, T=96, d=32, b=8, dtype="fp32"),
}


def _rel(g, r):
    return float(np.abs(g - r).max() / max(np.abs(r).max(), 1e-30))


def _run(wl, x, K=None, w0_per_seq=False, W0=None):
    Z, W = ttt.linear_fwd(x["Q"], x["K"] if K is None else K, x["V"], x["eta"],
                          x["W1"] if W0 is None else W0, x["gamma"], x["beta"], b=wl.b, ln=wl.ln,
                          w0_per_seq=w0_per_seq, l2_keys=True)
    torch.cuda.synchronize()
    assert ttt.ttt_device_status() == 0
    return Z.double().cpu().numpy(), W.double().cpu().numpy()


@pytest.mark.parametrize("name", list(CASES))
def test_l2_keys_match_oracle(name):
    wl = CASES[name]
    inp = synth.make_inputs(wl)
    x = to_dev(inp)
    Z, W = _run(wl, x)
    g, be = (inp.gamma, inp.beta) if wl.ln else (None, None)
    Zr, Wr = oracle.linear_primal(inp.Q, variants.normalize_keys(inp.K), inp.V, inp.eta, inp.W1,
                                  g, be, b=wl.b, ln=wl.ln)
    assert _rel(Z, Zr) <= TOL[wl.dtype] and _rel(W, Wr) <= TOL[wl.dtype]
    # the plain forward differs: the normalisation is not a no-op here
    Zp, _ = ttt.linear_fwd(x["Q"], x["K"], x["V"], x["eta"], x["W1"], x["gamma"], x["beta"],
                           b=wl.b, ln=wl.ln)
    assert _rel(Zp.double().cpu().numpy(), Zr) > 2 * TOL[wl.dtype]


def test_l2_keys_ignore_key_scale():
    """Keys scaled per token by powers of two (exact in bf16) give the same
    result."""
    wl = CASES["ln_bf16_d64_b16"]
    inp = synth.make_inputs(wl)
    x = to_dev(inp)
    r = np.random.default_rng(3)
    c = torch.from_numpy(2.0 ** r.integers(-2, 3, (wl.B, wl.H, wl.T, 1))).to(torch.bfloat16).cuda()
    Z1, W1 = _run(wl, x)
    Z2, W2 = _run(wl, x, K=(x["K"] * c).contiguous())
    assert _rel(Z2, Z1) <= 1e-6 and _rel(W2, W1) <= 1e-6


def test_l2_keys_per_sequence_w0_and_rejected_elsewhere():
    wl = CASES["ln_fp32_d32_b8"]
    inp = synth.make_inputs(wl)
    x = to_dev(inp)
    r = np.random.default_rng(4)
    W0 = (np.broadcast_to(inp.W1[None], (wl.B,) + inp.W1.shape)
          + 0.01 * r.standard_normal((wl.B,) + inp.W1.shape)).astype(np.float32)
    Z, W = _run(wl, x, w0_per_seq=True, W0=torch.from_numpy(W0).cuda())
    Zr, Wr = oracle.linear_primal(inp.Q, variants.normalize_keys(inp.K), inp.V, inp.eta, W0,
                                  inp.gamma, inp.beta, b=wl.b, ln=True, w0_per_seq=True)
    assert _rel(Z, Zr) <= TOL["fp32"] and _rel(W, Wr) <= TOL["fp32"]
    # the flag belongs to ttt_linear_fwd only
    Zt = torch.empty(1 << 16, device="cuda")
    rc = ttt.ttt_chunk_fwd(x["Q"], x["K"], x["V"], x["eta"], x["W1"], Zt, None, wl.B, wl.H,
                           wl.T, wl.d, wl.b, ttt.TTT_FP32, ttt.TTT_F_L2_KEYS, None, 0, check=False)
    assert rc == -1


# ------------------------------------------------ several gradient steps per token
STEP_CASES = {
    "ln_bf16_d64": L.scaled(B=1, H=2, T=48, b=1),
    "noln_fp32_d16": synth.WORKLOADS["linear_fp32_d16"].scaled(B=2, H=1, T=40, b=1),
    "ln_fp32_d32": L.scaled(B=2, H=1, T=32, d=32, b=1, dtype="fp32"),
}


def _steps(wl, x, n, l2_keys=False):
    Z, W = ttt.linear_fwd_steps(x["Q"], x["K"], x["V"], x["eta"], x["W1"], x["gamma"], x["beta"],
                                n_steps=n, ln=wl.ln, l2_keys=l2_keys)
    torch.cuda.synchronize()
    assert ttt.ttt_device_status() == 0
    return Z, W


@pytest.mark.parametrize("name,n", [("ln_bf16_d64", 2), ("ln_bf16_d64", 4), ("noln_fp32_d16", 3),
                                    ("ln_fp32_d32", 2)])
def test_steps_match_oracle(name, n):
    wl = STEP_CASES[name]
    inp = synth.make_inputs(wl)
    x = to_dev(inp)
    Z, W = _steps(wl, x, n)
    g, be = (inp.gamma, inp.beta) if wl.ln else (None, None)
    Zr, Wr = variants.linear_multistep(inp.Q, inp.K, inp.V, inp.eta, inp.W1, g, be, n_steps=n,
                                       ln=wl.ln)
    assert _rel(Z.double().cpu().numpy(), Zr) <= TOL[wl.dtype]
    assert _rel(W.double().cpu().numpy(), Wr) <= TOL[wl.dtype]


def test_one_step_is_the_b1_forward_and_counts_are_checked():
    wl = STEP_CASES["ln_bf16_d64"]
    inp = synth.make_inputs(wl)
    x = to_dev(inp)
    Z1, W1 = _steps(wl, x, 1)
    Zb, Wb = ttt.linear_fwd(x["Q"], x["K"], x["V"], x["eta"], x["W1"], x["gamma"], x["beta"], b=1,
                            ln=True)
    torch.cuda.synchronize()
    assert torch.equal(Z1, Zb) and torch.equal(W1, Wb)  # the same kernel, one step
    for n in (0, 1025):
        rc = ttt.ttt_linear_fwd_steps(x["Q"], x["K"], x["V"], x["eta"], x["W1"], x["gamma"],
                                      x["beta"], Z1, None, wl.B, wl.H, wl.T, wl.d, n, ttt.TTT_BF16,
                                      ttt.TTT_F_LN, check=False)
        assert rc == -1


def test_steps_with_l2_keys():
    wl = STEP_CASES["ln_fp32_d32"]
    inp = synth.make_inputs(wl)
    x = to_dev(inp)
    Z, W = _steps(wl, x, 3, l2_keys=True)
    Zr, Wr = variants.linear_multistep(inp.Q, variants.normalize_keys(inp.K), inp.V, inp.eta,
                                       inp.W1, inp.gamma, inp.beta, n_steps=3, ln=True)
    assert _rel(Z.double().cpu().numpy(), Zr) <= TOL["fp32"]
    assert _rel(W.double().cpu().numpy(), Wr) <= TOL["fp32"]
