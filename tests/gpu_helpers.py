"""Shared helpers of the GPU parity tests: put a workload's seeded inputs on
the device, run the CUDA path through the C ABI, run the oracle on the same
inputs, and measure the error.

Error metric, per output tensor: max_i |gpu_i - ref_i| / max_i |ref_i|
(a relative error normalised by the tensor's largest magnitude; pure
per-element relative error is meaningless near zeros). Tolerances: 1e-5 for
fp32 inputs, 2e-3 for bf16 inputs.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import test_sequence_layers_layer_b200 as ttt
from test_sequence_layers_layer_b200 import synth

TOL = {"fp32": 1e-5, "bf16": 2e-3}


def to_dev(inp: synth.Inputs, dev="cuda"):
    def qkv(vals, bits):
        if bits is not None:
            return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(vals).to(dev)

    d = dict(Q=qkv(inp.Q, inp.Q_bits), K=qkv(inp.K, inp.K_bits), V=qkv(inp.V, inp.V_bits),
             eta=torch.from_numpy(inp.eta).to(dev), W1=torch.from_numpy(inp.W1).to(dev),
             gamma=torch.from_numpy(inp.gamma).to(dev), beta=torch.from_numpy(inp.beta).to(dev))
    d["W2"] = torch.from_numpy(inp.W2).to(dev) if inp.W2 is not None else None
    return d


def run_gpu(inp: synth.Inputs, dev_inputs=None, **kw):
    """Returns a tuple of numpy float64 outputs: (Z, W_out) or (Z, W1_out, W2_out)."""
    wl = inp.wl
    x = dev_inputs or to_dev(inp)
    if wl.kind == "linear":
        outs = ttt.linear_fwd(x["Q"], x["K"], x["V"], x["eta"], x["W1"], x["gamma"], x["beta"],
                              b=wl.b, ln=wl.ln, **kw)
    elif wl.kind == "mlp":
        outs = ttt.mlp_fwd(x["Q"], x["K"], x["V"], x["eta"], x["W1"], x["W2"], x["gamma"],
                           x["beta"], b=wl.b, **kw)
    else:
        outs = ttt.chunk_fwd(x["Q"], x["K"], x["V"], x["eta"], x["W1"], chunk=wl.b, **kw)
    torch.cuda.synchronize()
    assert ttt.ttt_device_status() == 0
    return tuple(o.double().cpu().numpy() if o is not None else None for o in outs)


def run_oracle(inp: synth.Inputs, seqs=None):
    wl = inp.wl
    if wl.kind == "linear":
        return oracle.linear_primal(inp.Q, inp.K, inp.V, inp.eta, inp.W1, inp.gamma, inp.beta,
                                    b=wl.b, ln=wl.ln, seqs=seqs)
    if wl.kind == "mlp":
        return oracle.mlp_primal(inp.Q, inp.K, inp.V, inp.eta, inp.W1, inp.W2, inp.gamma,
                                 inp.beta, b=wl.b, seqs=seqs)
    return oracle.chunk_primal(inp.Q, inp.K, inp.V, inp.eta, inp.W1, chunk=wl.b, seqs=seqs)


def select(x, wl, seqs):
    """Rows of the listed sequences (batch*H + head) of a [B,H,...] array."""
    flat = x.reshape(wl.B * wl.H, *x.shape[2:])
    return flat if seqs is None else flat[np.asarray(seqs)]


def max_rel_err(gpu, ref, wl, seqs=None) -> float:
    g, r = select(gpu, wl, seqs), select(ref, wl, seqs)
    return float(np.abs(g - r).max() / max(np.abs(r).max(), 1e-30))


def elementwise_rel_err(gpu, ref, wl, seqs=None, floor=1e-3) -> float:
    """Largest per-element relative error, each element's denominator floored
    at floor * max |ref| (reported beside max_rel_err, not asserted)."""
    g, r = select(gpu, wl, seqs), select(ref, wl, seqs)
    den = np.maximum(np.abs(r), floor * max(np.abs(r).max(), 1e-30))
    return float((np.abs(g - r) / den).max())


def check_parity(inp, seqs=None, gpu_out=None):
    """Runs both sides, asserts every output within tolerance, returns errors.
    Prints, per output, the asserted error and the floored per-element one."""
    wl = inp.wl
    gpu_out = gpu_out or run_gpu(inp)
    ref_out = run_oracle(inp, seqs)
    tol = TOL[wl.dtype]
    errs = []
    for i, (g, r) in enumerate(zip(gpu_out, ref_out)):
        assert np.all(np.isfinite(select(g, wl, seqs)))
        errs.append(max_rel_err(g, r, wl, seqs))
        print(f"{wl.name} output {i}: max rel err {errs[-1]:.2e}, per-element (floor 1e-3) "
              f"{elementwise_rel_err(g, r, wl, seqs):.2e}")
    assert max(errs) <= tol, f"{wl.name}: errors {errs} > {tol}"
    return errs
