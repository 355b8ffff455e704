"""TTT_F_Z_BF16: the forward entry points store Z as bf16 (round to nearest
even) instead of fp32.

Every path computes Z in fp32 and rounds only at the store, so with the flag
the output must equal the fp32 run's Z rounded to bf16, bit for bit, and the
weights must not change. Against the oracle the bound is the fp32 path's
tolerance plus the rounding: |z16 - z| <= 2^-8 |z| + tol max|z| per element
(half a bf16 ulp is at most 2^-9 |z|; 2^-8 leaves room for a value the fp32
path already moved across a rounding boundary)."""
import numpy as np
import pytest
import torch

import test_sequence_layers_layer_b200 as ttt
from test_sequence_layers_layer_b200 import synth

from gpu_helpers import TOL, run_oracle, to_dev

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS

CASES = {
    "linear_tc": W["linear_ln_d64_b8h12_t2048"].scaled(B=2, H=2, T=96),
    "linear_simt_fp32": W["linear_fp32_d16"].scaled(B=2, H=2, T=40, d=32, b=8, ln=True,
                                                    eta="sigmoid_over_d"),
    "mlp_tc": W["mlp_ln_d64_dh256_b4h12_t8192"].scaled(B=1, H=2, T=64),
    "mlp_simt_fp32": W["mlp_ln_d64_dh256_b4h12_t8192"].scaled(B=1, H=2, T=32, d=16, dh=64, b=4,
                                                             dtype="fp32"),
    "chunk_tc": W["chunk_d128_c2048_b4h8_t32768"].scaled(B=1, H=2, T=512, b=256,
                                                         eta="const:0.00390625"),
    "chunk_simt_fp32": W["chunk_d128_c2048_b4h8_t32768"].scaled(B=1, H=2, T=512, b=256,
                                                                dtype="fp32", eta="const:0.00390625"),
}


def _run(wl, x, z_bf16):
    if wl.kind == "linear":
        out = ttt.linear_fwd(x["Q"], x["K"], x["V"], x["eta"], x["W1"], x["gamma"], x["beta"],
                             b=wl.b, ln=wl.ln, z_bf16=z_bf16)
    elif wl.kind == "mlp":
        out = ttt.mlp_fwd(x["Q"], x["K"], x["V"], x["eta"], x["W1"], x["W2"], x["gamma"],
                          x["beta"], b=wl.b, z_bf16=z_bf16)
    else:
        out = ttt.chunk_fwd(x["Q"], x["K"], x["V"], x["eta"], x["W1"], chunk=wl.b, z_bf16=z_bf16)
    torch.cuda.synchronize()
    assert ttt.ttt_device_status() == 0
    return out


@pytest.mark.parametrize("name", list(CASES))
def test_bf16_output_is_the_rounded_fp32_output(name):
    wl = CASES[name]
    inp = synth.make_inputs(wl)
    x = to_dev(inp)
    o32 = _run(wl, x, False)
    o16 = _run(wl, x, True)
    assert o16[0].dtype == torch.bfloat16 and o32[0].dtype == torch.float32
    assert torch.equal(o16[0], o32[0].to(torch.bfloat16)), name
    for w16, w32 in zip(o16[1:], o32[1:]):
        assert torch.equal(w16, w32)
    z = run_oracle(inp)[0]
    z16 = o16[0].double().cpu().numpy()
    bound = 2.0 ** -8 * np.abs(z) + TOL[wl.dtype] * np.abs(z).max()
    assert np.all(np.abs(z16 - z) <= bound), float(np.max(np.abs(z16 - z) / bound))
