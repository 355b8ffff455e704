"""TTT-Linear backward (ttt_linear_bwd), large-chunk backward (ttt_chunk_bwd)
and TTT-MLP backward (ttt_mlp_bwd) against the backward oracle
(oracle/backward.py: autograd through the float64 unrolled inner loop).

Tolerance: 1e-4 of each gradient's largest magnitude. The kernel works in
fp32 (unit roundoff 6e-8); a gradient here is a sum over the sequence of
products of a second-order LayerNorm derivative (itself a difference of terms
of size ~1/sigma) with length-d dot products, so its rounding error is a few
hundred ulps of its scale, ~2e-5; 1e-4 leaves a 5x margin. Inputs that the
kernel reads as bf16 are bf16-exact, so both sides see the same numbers."""
import numpy as np
import pytest
import torch

import test_sequence_layers_layer_b200 as ttt
from test_sequence_layers_layer_b200 import synth
from oracle import backward as ob

pytestmark = pytest.mark.gpu
TOL = 1e-4

CASES = {
    # name: (workload changes, ln, dtype, w0_per_seq, with dW_out)
    "ln_fp32_d16_b4": (dict(B=2, H=2, T=16, d=16, b=4), True, "fp32", False, True),
    "noln_fp32_d16_b4": (dict(B=2, H=2, T=16, d=16, b=4), False, "fp32", False, True),
    "ln_fp32_d32_b8_w0seq": (dict(B=2, H=1, T=32, d=32, b=8), True, "fp32", True, False),
    "ln_bf16_d64_b16": (dict(B=1, H=2, T=64, d=64, b=16), True, "bf16", False, True),
    "noln_bf16_d64_b16": (dict(B=1, H=2, T=48, d=64, b=16), False, "bf16", False, False),
    "ln_fp32_d64_b1": (dict(B=1, H=1, T=8, d=64, b=1), True, "fp32", False, True),
}


def _case(name, seed=11):
    ch, ln, dtype, w0seq, with_dw = CASES[name]
    base = synth.WORKLOADS["linear_ln_d64_b8h12_t2048"]
    wl = base.scaled(ln=ln, dtype=dtype, seed=seed, **ch)
    inp = synth.make_inputs(wl)
    r = np.random.default_rng(seed + 1)
    B, H, T, d = wl.B, wl.H, wl.T, wl.d
    dZ = r.standard_normal((B, H, T, d)).astype(np.float32)
    dW = r.standard_normal((B, H, d, d)).astype(np.float32) if with_dw else None
    W0 = inp.W1
    if w0seq:
        W0 = np.ascontiguousarray(np.broadcast_to(W0[None], (B,) + W0.shape)) + \
            0.01 * r.standard_normal((B,) + W0.shape)
        W0 = W0.astype(np.float32)
    return wl, inp, W0, dZ, dW, ln, w0seq


def _qkv(inp, wl):
    if wl.dtype == "bf16":
        q = lambda bits: torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()  # noqa: E731
        return q(inp.Q_bits), q(inp.K_bits), q(inp.V_bits)
    return tuple(torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()
                 for a in (inp.Q, inp.K, inp.V))


def _gpu(wl, inp, W0, dZ, dW, ln, w0seq):
    Q, K, V = _qkv(inp, wl)
    f = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()  # noqa: E731
    g = ttt.linear_bwd(Q, K, V, f(inp.eta), f(W0), f(inp.gamma) if ln else None,
                       f(inp.beta) if ln else None, f(dZ), f(dW), b=wl.b, ln=ln, w0_per_seq=w0seq)
    torch.cuda.synchronize()
    assert ttt.ttt_device_status() == 0
    return {k: v.double().cpu().numpy() for k, v in g.items()}


def _rel(g, r):
    return float(np.abs(g - r).max() / max(np.abs(r).max(), 1e-30))


@pytest.mark.parametrize("name", list(CASES))
def test_backward_matches_oracle(name):
    wl, inp, W0, dZ, dW, ln, w0seq = _case(name)
    got = _gpu(wl, inp, W0, dZ, dW, ln, w0seq)
    ref = ob.linear_grads(inp.Q, inp.K, inp.V, inp.eta, W0, inp.gamma if ln else None,
                          inp.beta if ln else None, dZ, dW, b=wl.b, ln=ln)
    if not w0seq:
        ref["W0"] = ref["W0"].reshape(W0.shape)
    errs = {k: _rel(got[k], ref[k]) for k in ref}
    assert set(got) == set(ref)
    assert max(errs.values()) <= TOL, errs


def test_backward_full_size_sampled_sequences():
    """The bench workload (B=8, H=12, T=2048, bf16, LN) in one launch; the
    per-token gradients of two sequences are checked against the oracle run
    on those sequences alone (they depend on nothing else)."""
    wl = synth.WORKLOADS["linear_ln_d64_b8h12_t2048"]
    inp = synth.make_inputs(wl)
    r = np.random.default_rng(21)
    dZ = r.standard_normal((wl.B, wl.H, wl.T, wl.d)).astype(np.float32)
    got = _gpu(wl, inp, inp.W1, dZ, None, True, False)
    for bb, hh in [(0, 0), (7, 11)]:
        sl = lambda a: a[bb:bb + 1, hh:hh + 1]  # noqa: E731
        ref = ob.linear_grads(sl(inp.Q), sl(inp.K), sl(inp.V), sl(inp.eta), inp.W1[hh:hh + 1],
                              inp.gamma[hh:hh + 1], inp.beta[hh:hh + 1], sl(dZ), None,
                              b=wl.b, ln=True)
        for k in ("Q", "K", "V", "eta"):
            e = _rel(sl(got[k]), ref[k])
            assert e <= TOL, (bb, hh, k, e)


def test_backward_deterministic_and_rejects_small_workspace():
    wl, inp, W0, dZ, dW, ln, w0seq = _case("ln_bf16_d64_b16")
    a = _gpu(wl, inp, W0, dZ, dW, ln, w0seq)
    b = _gpu(wl, inp, W0, dZ, dW, ln, w0seq)
    for k in a:
        assert np.array_equal(a[k], b[k]), k
    Q, K, V = _qkv(inp, wl)
    need = ttt.ttt_linear_bwd_workspace_bytes(wl.B, wl.H, wl.T, wl.d, wl.b)
    assert need == 4 * (wl.B * wl.H * (wl.T // wl.b) * wl.d ** 2 + wl.B * wl.H * wl.d ** 2
                        + 2 * wl.B * wl.H * wl.d)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    out = [torch.empty(1 << 20, device="cuda") for _ in range(7)]
    f = lambda x: torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()  # noqa: E731
    rc = ttt.ttt_linear_bwd(Q, K, V, f(inp.eta), f(W0), f(inp.gamma), f(inp.beta), f(dZ), None,
                            *out, wl.B, wl.H, wl.T, wl.d, wl.b, ttt.TTT_BF16, ttt.TTT_F_LN, ws,
                            need - 256, check=False)
    assert rc == -9  # TTT_ERR_WORKSPACE, nothing launched
    rc = ttt.ttt_linear_bwd(Q, K, V, f(inp.eta), f(W0), f(inp.gamma), f(inp.beta), f(dZ), None,
                            *out, wl.B, wl.H, wl.T + 1, wl.d, wl.b, ttt.TTT_BF16, ttt.TTT_F_LN, ws,
                            need, check=False)
    assert rc == -2  # TTT_ERR_SHAPE


# ------------------------------------------------------------ large-chunk TTT

CHUNK_CASES = {
    # name: (workload changes, w0_per_seq, with dW_out)
    "chunk_fp32_d64_c32": (dict(B=2, H=2, T=128, d=64, b=32, dtype="fp32"), False, True),
    "chunk_bf16_d128_c64": (dict(B=1, H=2, T=256, d=128, b=64), False, False),
    "chunk_fp32_d128_c128_w0seq": (dict(B=2, H=1, T=256, d=128, b=128, dtype="fp32"), True, True),
    # d = 128, bf16: the Gram products on the tensor cores (one eta per chunk:
    # raw K with eta on the fp32 accumulator; a varying eta: eta K as hi + lo)
    "chunk_bf16_d128_c64_eta_varied": (dict(B=1, H=2, T=256, d=128, b=64, eta="sigmoid_over_d"),
                                       False, True),
    "chunk_bf16_d128_c128_w0seq": (dict(B=2, H=1, T=512, d=128, b=128), True, True),
    "chunk_bf16_d128_c32_one_chunk": (dict(B=1, H=3, T=32, d=128, b=32), False, True),
    # chunk % 128 == 0: the per-token products on the tensor cores too
    "chunk_bf16_d128_c256_eta_varied": (dict(B=1, H=2, T=768, d=128, b=256, eta="sigmoid_over_d"),
                                        False, True),
    "chunk_bf16_d128_c128_one_chunk": (dict(B=2, H=1, T=128, d=128, b=128), True, False),
}


def _chunk_case(name, seed=31):
    ch, w0seq, with_dw = CHUNK_CASES[name]
    wl = synth.WORKLOADS["chunk_d128_c2048_b4h8_t32768"].scaled(seed=seed, **ch)
    inp = synth.make_inputs(wl)
    r = np.random.default_rng(seed + 1)
    dZ = r.standard_normal((wl.B, wl.H, wl.T, wl.d)).astype(np.float32)
    dW = r.standard_normal((wl.B, wl.H, wl.d, wl.d)).astype(np.float32) if with_dw else None
    W0 = inp.W1
    if w0seq:
        W0 = (np.broadcast_to(W0[None], (wl.B,) + W0.shape)
              + 0.01 * r.standard_normal((wl.B,) + W0.shape)).astype(np.float32)
    return wl, inp, W0, dZ, dW, w0seq


def _chunk_gpu(wl, inp, W0, dZ, dW, w0seq):
    Q, K, V = _qkv(inp, wl)
    f = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()  # noqa: E731
    g = ttt.chunk_bwd(Q, K, V, f(inp.eta), f(W0), f(dZ), f(dW), chunk=wl.b, w0_per_seq=w0seq)
    torch.cuda.synchronize()
    assert ttt.ttt_device_status() == 0
    return {k: v.double().cpu().numpy() for k, v in g.items()}


@pytest.mark.parametrize("name", list(CHUNK_CASES))
def test_chunk_backward_matches_oracle(name):
    wl, inp, W0, dZ, dW, w0seq = _chunk_case(name)
    got = _chunk_gpu(wl, inp, W0, dZ, dW, w0seq)
    ref = ob.chunk_grads(inp.Q, inp.K, inp.V, inp.eta, W0, dZ, dW, chunk=wl.b)
    if not w0seq:
        ref["W0"] = ref["W0"].reshape(W0.shape)
    errs = {k: _rel(got[k], ref[k]) for k in ref}
    assert set(got) == set(ref)
    assert max(errs.values()) <= TOL, errs


def test_chunk_backward_full_size_sampled_sequences():
    """The large-chunk bench workload (B=4, H=8, T=32768, d=128, chunk 2048,
    bf16) in one launch; two sequences' per-token gradients against the
    oracle run on those sequences alone."""
    wl = synth.WORKLOADS["chunk_d128_c2048_b4h8_t32768"]
    inp = synth.make_inputs(wl)
    r = np.random.default_rng(41)
    dZ = r.standard_normal((wl.B, wl.H, wl.T, wl.d)).astype(np.float32)
    got = _chunk_gpu(wl, inp, inp.W1, dZ, None, False)
    for bb, hh in [(0, 0), (3, 7)]:
        sl = lambda a: a[bb:bb + 1, hh:hh + 1]  # noqa: E731
        ref = ob.chunk_grads(sl(inp.Q), sl(inp.K), sl(inp.V), sl(inp.eta), inp.W1[hh:hh + 1],
                             sl(dZ), None, chunk=wl.b)
        for k in ("Q", "K", "V", "eta"):
            e = _rel(sl(got[k]), ref[k])
            assert e <= TOL, (bb, hh, k, e)


# ------------------------------------------------------------------- TTT-MLP

MLP_CASES = {
    # name: (workload changes, w0_per_seq, with dW1_out / dW2_out)
    "mlp_bf16_d64_b16": (dict(B=1, H=2, T=64), False, True),
    "mlp_fp32_d16_b4_w0seq": (dict(B=2, H=1, T=16, d=16, dh=64, b=4, dtype="fp32"), True, False),
    "mlp_bf16_d32_b8": (dict(B=2, H=1, T=32, d=32, dh=128, b=8), False, True),
}


def _mlp_case(name, seed=51):
    ch, w0seq, with_dw = MLP_CASES[name]
    wl = synth.WORKLOADS["mlp_ln_d64_dh256_b4h12_t8192"].scaled(seed=seed, **ch)
    inp = synth.make_inputs(wl)
    r = np.random.default_rng(seed + 1)
    B, H, T, d, dh = wl.B, wl.H, wl.T, wl.d, wl.dh
    dZ = r.standard_normal((B, H, T, d)).astype(np.float32)
    dW1 = r.standard_normal((B, H, d, dh)).astype(np.float32) if with_dw else None
    dW2 = r.standard_normal((B, H, dh, d)).astype(np.float32) if with_dw else None
    W1, W2 = inp.W1, inp.W2
    if w0seq:
        W1 = (np.broadcast_to(W1[None], (B,) + W1.shape)
              + 0.01 * r.standard_normal((B,) + W1.shape)).astype(np.float32)
        W2 = (np.broadcast_to(W2[None], (B,) + W2.shape)
              + 0.01 * r.standard_normal((B,) + W2.shape)).astype(np.float32)
    return wl, inp, W1, W2, dZ, dW1, dW2, w0seq


def _mlp_gpu(wl, inp, W1, W2, dZ, dW1, dW2, w0seq):
    Q, K, V = _qkv(inp, wl)
    f = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()  # noqa: E731
    g = ttt.mlp_bwd(Q, K, V, f(inp.eta), f(W1), f(W2), f(inp.gamma), f(inp.beta), f(dZ), f(dW1),
                    f(dW2), b=wl.b, w0_per_seq=w0seq)
    torch.cuda.synchronize()
    assert ttt.ttt_device_status() == 0
    return {k: v.double().cpu().numpy() for k, v in g.items()}


@pytest.mark.late
@pytest.mark.parametrize("name", list(MLP_CASES))
def test_mlp_backward_matches_oracle(name):
    wl, inp, W1, W2, dZ, dW1, dW2, w0seq = _mlp_case(name)
    got = _mlp_gpu(wl, inp, W1, W2, dZ, dW1, dW2, w0seq)
    ref = ob.mlp_grads(inp.Q, inp.K, inp.V, inp.eta, W1, W2, inp.gamma, inp.beta, dZ, dW1, dW2,
                       b=wl.b)
    errs = {k: _rel(got[k], ref[k]) for k in ref}
    assert set(got) == set(ref)
    assert max(errs.values()) <= TOL, errs
