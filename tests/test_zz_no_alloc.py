"""The allocation-free large-chunk entry point (ttt_chunk_fwd_noalloc).

Some callers cannot allocate device memory themselves (for example a plugin
inside a host application whose allocator owns the whole GPU). For them the
library offers ttt_chunk_fwd_noalloc, which keeps its scratch in a buffer the
library declares statically instead of a caller workspace. This test calls it
through the C ABI twice in a row, on two different inputs, and checks each
result against the workspace entry point ttt_chunk_fwd: both run the same
kernels on the same inputs, so Z and W must agree bit for bit. It also checks that a problem too large for the static
buffer is refused before anything is launched. It lives in its own file,
collected last, and passes alone or after the other tests."""
import numpy as np
import pytest
import torch

import test_sequence_layers_layer_b200 as ttt
from test_sequence_layers_layer_b200 import synth

from gpu_helpers import to_dev

pytestmark = pytest.mark.gpu


def _case(seed):
    wl = synth.WORKLOADS["chunk_d128_c2048_b4h8_t32768"].scaled(B=2, H=3, T=1024, b=256,
                                                                 eta="sigmoid_over_d", seed=seed)
    return wl, to_dev(synth.make_inputs(wl))


def _with_workspace(wl, x):
    return ttt.chunk_fwd(x["Q"], x["K"], x["V"], x["eta"], x["W1"], chunk=wl.b)


def _noalloc(wl, x):
    Z = torch.empty((wl.B, wl.H, wl.T, wl.d), dtype=torch.float32, device="cuda")
    W = torch.empty((wl.B, wl.H, wl.d, wl.d), dtype=torch.float32, device="cuda")
    ttt.ttt_chunk_fwd_noalloc(x["Q"], x["K"], x["V"], x["eta"], x["W1"], Z, W, wl.B, wl.H, wl.T,
                              wl.d, wl.b, ttt.TTT_BF16, 0)
    return Z, W


def test_noalloc_matches_workspace_entry_point_twice():
    for seed in (3, 4):  # two calls in a row, different inputs, one shared buffer
        wl, x = _case(seed)
        need = ttt.ttt_chunk_workspace_bytes(wl.B, wl.H, wl.T, wl.d, wl.b)
        assert 0 < need <= (24 << 20) + 4096
        Zr, Wr = _with_workspace(wl, x)
        Z, W = _noalloc(wl, x)
        torch.cuda.synchronize()
        assert ttt.ttt_device_status() == 0
        assert torch.equal(Z, Zr), seed
        assert torch.equal(W, Wr), seed
        assert np.isfinite(Z.cpu().numpy()).all()


def test_noalloc_refuses_problems_beyond_its_buffer():
    wl, x = _case(5)
    big_T = 129 * 256  # 2 * 3 * 129 chunks of 160 KiB > 24 MiB + 4 KiB
    Z = torch.empty(1, device="cuda")
    n0 = ttt.ttt_launch_count()
    rc = ttt.ttt_chunk_fwd_noalloc(x["Q"], x["K"], x["V"], x["eta"], x["W1"], Z, None, wl.B,
                                   wl.H, big_T, wl.d, wl.b, ttt.TTT_BF16, 0, check=False)
    assert rc == -10
    assert ttt.ttt_launch_count() == n0
