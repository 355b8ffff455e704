"""Phase trace of the TTT-Linear tensor-core scan (profiling builds only).

Build the library with the trace compiled in, run this on a GPU, rebuild
without it afterwards:

    TTT_NVCC_DEFINES=TTT_TRACE python -m test_sequence_layers_layer_b200.build --force
    python -m test_sequence_layers_layer_b200.trace_linear linear_ln_d64_b8h12_t2048
    python -m test_sequence_layers_layer_b200.build --force

Block 0 of the kernel records the SM clock at each hand-off of its first 128
mini-batches. This prints, for mini-batches 20-99, the mean clock of each
event relative to the moment the scan warps publish G_j, and the period.
"""
from __future__ import annotations

import ctypes
import sys

import numpy as np

EVENTS = {0: "MMA thread sees G_j", 1: "W update issued", 9: "re-emit warp 0 sees the update",
          19: "re-emit: W loaded", 20: "re-emit: operand rows written", 13: "re-emit warp 0 done",
          18: "MMA thread sees the A tile", 2: "MMA thread sees W re-emitted",
          3: "product issued", 4: "copy-out of P_j and C_j done",
          5: "scan sees P_j", 21: "scan sees G_(j-1)", 6: "correction X = P - C G done",
          24: "LayerNorm row statistics", 7: "LayerNorm backward done", 25: "G stored (fp32)",
          26: "G stored (bf16 hi/lo)", 27: "async-proxy fence done", 8: "G_j published",
          17: "output warps: Z of mini-batch j stored"}


def main(workload: str = "linear_ln_d64_b8h12_t2048") -> None:
    import torch
    import test_sequence_layers_layer_b200 as ttt
    from test_sequence_layers_layer_b200 import synth

    L = ttt.lib()
    try:
        fetch = L.ttt_trace_fetch
    except AttributeError:
        sys.exit("libttt.so was built without TTT_TRACE")
    fetch.restype = ctypes.c_int
    fetch.argtypes = [ctypes.c_void_p, ctypes.c_int]
    wl = synth.WORKLOADS[workload]
    inp = synth.make_inputs(wl)

    def dev(vals, bits):
        if bits is not None:
            return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()
        return torch.from_numpy(vals).cuda()

    Q, K, V = dev(inp.Q, inp.Q_bits), dev(inp.K, inp.K_bits), dev(inp.V, inp.V_bits)
    eta, W0 = torch.from_numpy(inp.eta).cuda(), torch.from_numpy(inp.W1).cuda()
    gam, bet = torch.from_numpy(inp.gamma).cuda(), torch.from_numpy(inp.beta).cuda()
    for _ in range(3):
        ttt.linear_fwd(Q, K, V, eta, W0, gam, bet, b=wl.b, ln=wl.ln)
    torch.cuda.synchronize()
    tr = np.zeros(32 * 128, dtype=np.uint32)
    if fetch(tr.ctypes.data, tr.size) != 0:
        sys.exit("trace fetch failed")
    tr = tr.reshape(32, 128).astype(np.int64)
    js = np.arange(20, 100)
    print(f"{workload}: period {np.mean(np.diff(tr[8][js])):.0f} SM cycles per mini-batch")
    for ev, name in sorted(EVENTS.items(), key=lambda kv: np.mean(tr[kv[0]][js] - tr[8][js])):
        d = tr[ev][js] - tr[8][js]
        print(f"  {np.mean(d):8.0f}  {name}")


if __name__ == "__main__":
    main(*sys.argv[1:2])
