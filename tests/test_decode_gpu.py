"""Single-token decode (b = 1 streaming): one call per token, the state passed
in and updated in place (TTT_F_W0_PER_SEQ with W_out aliasing W0). The loop
must reproduce the whole-sequence call with b = 1 exactly, and the oracle's
token-by-token online update within the dtype's tolerance."""
import numpy as np
import pytest
import torch

import test_sequence_layers_layer_b200 as ttt
from test_sequence_layers_layer_b200 import synth

from gpu_helpers import TOL, max_rel_err, run_oracle, to_dev

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS


def _tok(t, i):
    return t[:, :, i:i + 1].contiguous()


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_linear_decode_loop(dtype):
    wl = W["linear_ln_d64_b8h12_t2048"].scaled(B=2, H=3, T=24, b=1, dtype=dtype)
    inp = synth.make_inputs(wl)
    x = to_dev(inp)
    Zw, Ww = ttt.linear_fwd(x["Q"], x["K"], x["V"], x["eta"], x["W1"], x["gamma"], x["beta"],
                            b=1, ln=True)
    state = x["W1"].unsqueeze(0).repeat(wl.B, 1, 1, 1)
    Z = torch.empty_like(Zw)
    for i in range(wl.T):
        z = torch.empty((wl.B, wl.H, 1, wl.d), dtype=torch.float32, device="cuda")
        ttt.ttt_linear_fwd(_tok(x["Q"], i), _tok(x["K"], i), _tok(x["V"], i), _tok(x["eta"], i),
                           state, x["gamma"], x["beta"], z, state, wl.B, wl.H, 1, wl.d, 1,
                           ttt.TTT_BF16 if dtype == "bf16" else ttt.TTT_FP32,
                           ttt.TTT_F_LN | ttt.TTT_F_W0_PER_SEQ)
        Z[:, :, i:i + 1] = z
    torch.cuda.synchronize()
    assert ttt.ttt_device_status() == 0
    torch.testing.assert_close(Z, Zw, rtol=0, atol=0)
    torch.testing.assert_close(state, Ww, rtol=0, atol=0)
    Zr, Wr = run_oracle(inp)
    assert max_rel_err(Z.double().cpu().numpy(), Zr, wl) <= TOL[dtype]
    assert max_rel_err(state.double().cpu().numpy(), Wr, wl) <= TOL[dtype]


def test_mlp_decode_loop():
    wl = W["mlp_ln_d64_dh256_b4h12_t8192"].scaled(B=1, H=2, T=12, b=1)
    inp = synth.make_inputs(wl)
    x = to_dev(inp)
    Zw, W1w, W2w = ttt.mlp_fwd(x["Q"], x["K"], x["V"], x["eta"], x["W1"], x["W2"], x["gamma"],
                               x["beta"], b=1)
    s1 = x["W1"].unsqueeze(0).repeat(wl.B, 1, 1, 1)
    s2 = x["W2"].unsqueeze(0).repeat(wl.B, 1, 1, 1)
    Z = torch.empty_like(Zw)
    for i in range(wl.T):
        z = torch.empty((wl.B, wl.H, 1, wl.d), dtype=torch.float32, device="cuda")
        ttt.ttt_mlp_fwd(_tok(x["Q"], i), _tok(x["K"], i), _tok(x["V"], i), _tok(x["eta"], i),
                        s1, s2, x["gamma"], x["beta"], z, s1, s2, wl.B, wl.H, 1, wl.d, wl.dh, 1,
                        ttt.TTT_BF16, ttt.TTT_F_LN | ttt.TTT_F_W0_PER_SEQ)
        Z[:, :, i:i + 1] = z
    torch.cuda.synchronize()
    assert ttt.ttt_device_status() == 0
    torch.testing.assert_close(Z, Zw, rtol=0, atol=0)
    torch.testing.assert_close(s1, W1w, rtol=0, atol=0)
    torch.testing.assert_close(s2, W2w, rtol=0, atol=0)
    Zr, W1r, W2r = run_oracle(inp)
    assert max_rel_err(Z.double().cpu().numpy(), Zr, wl) <= TOL["bf16"]
    assert max_rel_err(s2.double().cpu().numpy(), W2r, wl) <= TOL["bf16"]


@pytest.mark.late
@pytest.mark.parametrize("dtype,ln,l2", [("bf16", True, False), ("fp32", True, False),
                                         ("bf16", False, False), ("fp32", True, True)])
def test_decode_kernel_loop(dtype, ln, l2):
    """ttt_linear_decode (the one-token kernel, W in registers): a token loop
    against the oracle's online update and against the same loop through
    ttt_linear_fwd (T = 1), both within the dtype's tolerance."""
    wl = W["linear_ln_d64_b8h12_t2048"].scaled(B=2, H=3, T=24, b=1, dtype=dtype, ln=ln)
    inp = synth.make_inputs(wl)
    x = to_dev(inp)
    state = x["W1"].unsqueeze(0).repeat(wl.B, 1, 1, 1)
    Z = torch.empty((wl.B, wl.H, wl.T, wl.d), dtype=torch.float32, device="cuda")
    for i in range(wl.T):
        q, k, v = (x[n][:, :, i].contiguous() for n in ("Q", "K", "V"))
        e = x["eta"][:, :, i].contiguous()
        Z[:, :, i] = ttt.linear_decode(q, k, v, e, state, x["gamma"], x["beta"], ln=ln,
                                       l2_keys=l2)
    torch.cuda.synchronize()
    assert ttt.ttt_device_status() == 0
    if l2:
        from oracle import variants
        import oracle
        Zr, Wr = oracle.linear_primal(inp.Q, variants.normalize_keys(inp.K), inp.V, inp.eta,
                                      inp.W1, inp.gamma, inp.beta, b=1, ln=ln)
    else:
        Zr, Wr = run_oracle(inp)
    assert max_rel_err(Z.double().cpu().numpy(), Zr, wl) <= TOL[dtype]
    assert max_rel_err(state.double().cpu().numpy(), Wr, wl) <= TOL[dtype]
    Zw, Ww = ttt.linear_fwd(x["Q"], x["K"], x["V"], x["eta"], x["W1"], x["gamma"], x["beta"],
                            b=1, ln=ln, l2_keys=l2)
    torch.cuda.synchronize()
    assert max_rel_err(Z.double().cpu().numpy(), Zw.double().cpu().numpy(), wl) <= TOL[dtype]


@pytest.mark.late
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_mlp_decode_kernel_loop(dtype):
    """ttt_mlp_decode (the one-token TTT-MLP kernel): a token loop against the
    oracle's online update and against the same loop through ttt_mlp_fwd
    (T = 1), within the dtype's tolerance."""
    wl = W["mlp_ln_d64_dh256_b4h12_t8192"].scaled(B=1, H=2, T=12, b=1, dtype=dtype)
    inp = synth.make_inputs(wl)
    x = to_dev(inp)
    s1 = x["W1"].unsqueeze(0).repeat(wl.B, 1, 1, 1)
    s2 = x["W2"].unsqueeze(0).repeat(wl.B, 1, 1, 1)
    Z = torch.empty((wl.B, wl.H, wl.T, wl.d), dtype=torch.float32, device="cuda")
    for i in range(wl.T):
        q, k, v = (x[n][:, :, i].contiguous() for n in ("Q", "K", "V"))
        e = x["eta"][:, :, i].contiguous()
        Z[:, :, i] = ttt.mlp_decode(q, k, v, e, s1, s2, x["gamma"], x["beta"])
    torch.cuda.synchronize()
    assert ttt.ttt_device_status() == 0
    Zr, W1r, W2r = run_oracle(inp)
    assert max_rel_err(Z.double().cpu().numpy(), Zr, wl) <= TOL[dtype]
    assert max_rel_err(s1.double().cpu().numpy(), W1r, wl) <= TOL[dtype]
    assert max_rel_err(s2.double().cpu().numpy(), W2r, wl) <= TOL[dtype]
    Zw, _, _ = ttt.mlp_fwd(x["Q"], x["K"], x["V"], x["eta"], x["W1"], x["W2"], x["gamma"],
                           x["beta"], b=1)
    torch.cuda.synchronize()
    assert max_rel_err(Z.double().cpu().numpy(), Zw.double().cpu().numpy(), wl) <= TOL[dtype]


@pytest.mark.parametrize("kind,dtype", [("linear", "bf16"), ("linear", "fp32"), ("mlp", "bf16")])
def test_decode_tokens_in_one_call(kind, dtype):
    """ttt_linear_decode_tokens / ttt_mlp_decode_tokens (all tokens of the
    call with the weight kept on chip) equal the loop of one-token calls bit
    for bit, and match the oracle's online update."""
    name = "linear_ln_d64_b8h12_t2048" if kind == "linear" else "mlp_ln_d64_dh256_b4h12_t8192"
    wl = W[name].scaled(B=2, H=3, T=20, b=1, dtype=dtype)
    inp = synth.make_inputs(wl)
    x = to_dev(inp)
    s1 = x["W1"].unsqueeze(0).repeat(wl.B, 1, 1, 1)
    t1 = s1.clone()
    if kind == "mlp":
        s2 = x["W2"].unsqueeze(0).repeat(wl.B, 1, 1, 1)
        t2 = s2.clone()
        Z = ttt.mlp_decode_tokens(x["Q"], x["K"], x["V"], x["eta"], s1, s2, x["gamma"], x["beta"])
    else:
        Z = ttt.linear_decode_tokens(x["Q"], x["K"], x["V"], x["eta"], s1, x["gamma"], x["beta"],
                                     ln=True)
    Zl = torch.empty_like(Z)
    for i in range(wl.T):
        q, k, v = (x[n][:, :, i].contiguous() for n in ("Q", "K", "V"))
        e = x["eta"][:, :, i].contiguous()
        if kind == "mlp":
            Zl[:, :, i] = ttt.mlp_decode(q, k, v, e, t1, t2, x["gamma"], x["beta"])
        else:
            Zl[:, :, i] = ttt.linear_decode(q, k, v, e, t1, x["gamma"], x["beta"], ln=True)
    torch.cuda.synchronize()
    assert ttt.ttt_device_status() == 0
    assert torch.equal(Z, Zl) and torch.equal(s1, t1)
    outs = run_oracle(inp)
    assert max_rel_err(Z.double().cpu().numpy(), outs[0], wl) <= TOL[dtype]
    assert max_rel_err(s1.double().cpu().numpy(), outs[1], wl) <= TOL[dtype]
    if kind == "mlp":
        assert torch.equal(s2, t2)
        assert max_rel_err(s2.double().cpu().numpy(), outs[2], wl) <= TOL[dtype]


def test_decode_tokens_rejects_bad_n():
    wl = W["linear_ln_d64_b8h12_t2048"].scaled(B=1, H=1, T=4, b=1)
    x = to_dev(synth.make_inputs(wl))
    s = x["W1"].unsqueeze(0).repeat(1, 1, 1, 1)
    z = torch.empty((1, 1, 4, 64), device="cuda")
    rc = ttt.ttt_linear_decode_tokens(x["Q"], x["K"], x["V"], x["eta"], s, x["gamma"], x["beta"],
                                      z, 1, 1, 0, 64, ttt.TTT_BF16, ttt.TTT_F_LN, check=False)
    assert rc == -2
