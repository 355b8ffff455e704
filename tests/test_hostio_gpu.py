"""TTT-Linear forward from pinned host buffers with copies overlapped across
slices of the (batch, head) grid (hostio.linear_fwd_host): its outputs equal
one ttt_linear_fwd call on the device over the whole batch, bit for bit (a
sequence's result does not depend on which sequences share its call)."""
import pytest
import torch

import test_sequence_layers_layer_b200 as ttt
from test_sequence_layers_layer_b200 import hostio, synth
from gpu_helpers import to_dev

pytestmark = [pytest.mark.gpu, pytest.mark.late]

L = synth.WORKLOADS["linear_ln_d64_b8h12_t2048"]


@pytest.mark.parametrize("B,slices,z_bf16,ln", [(3, 1, False, True), (5, 3, False, True),
                                               (8, 4, True, True), (4, 4, False, False),
                                               (2, 5, False, True)])
def test_host_pipeline_equals_device_call(B, slices, z_bf16, ln):
    wl = L.scaled(B=B, H=3, T=160, ln=ln)
    x = to_dev(synth.make_inputs(wl))
    Zd, Wd = ttt.linear_fwd(x["Q"], x["K"], x["V"], x["eta"], x["W1"], x["gamma"], x["beta"],
                            b=wl.b, ln=ln, z_bf16=z_bf16)
    h = {k: x[k].cpu().pin_memory() for k in ("Q", "K", "V", "eta")}
    Zh, Wh = hostio.linear_fwd_host(h["Q"], h["K"], h["V"], h["eta"], x["W1"].cpu(),
                                    x["gamma"].cpu(), x["beta"].cpu(), b=wl.b, ln=ln,
                                    slices=slices, z_bf16=z_bf16)
    torch.cuda.current_stream().synchronize()
    assert ttt.ttt_device_status() == 0
    assert Zh.is_pinned() and Wh.is_pinned()
    assert torch.equal(Zh, Zd.cpu()) and torch.equal(Wh, Wd.cpu())


C = synth.WORKLOADS["chunk_d128_c2048_b4h8_t32768"]


@pytest.mark.parametrize("B,slices,z_bf16,per_seq", [(3, 3, False, False), (4, 2, True, False),
                                                    (2, 2, False, True), (2, 4, False, False),
                                                    (1, 2, True, True)])
def test_chunk_host_pipeline_equals_device_call(B, slices, z_bf16, per_seq):
    """Large-chunk forward from pinned host buffers, one workspace per slice,
    outputs written into caller-given pinned buffers: equal to one
    ttt_chunk_fwd call on the device, bit for bit."""
    wl = C.scaled(B=B, H=2, T=1024, b=256)
    x = to_dev(synth.make_inputs(wl))
    W0 = x["W1"].unsqueeze(0).repeat(B, 1, 1, 1) if per_seq else x["W1"]
    Zd, Wd = ttt.chunk_fwd(x["Q"], x["K"], x["V"], x["eta"], W0, chunk=wl.b, w0_per_seq=per_seq,
                           z_bf16=z_bf16)
    h = {k: x[k].cpu().pin_memory() for k in ("Q", "K", "V", "eta")}
    out = (torch.empty(tuple(Zd.shape), dtype=Zd.dtype, pin_memory=True),
           torch.empty(tuple(Wd.shape), dtype=torch.float32, pin_memory=True))
    Zh, Wh = hostio.chunk_fwd_host(h["Q"], h["K"], h["V"], h["eta"], W0.cpu(), chunk=wl.b,
                                   slices=slices, w0_per_seq=per_seq, z_bf16=z_bf16, out=out)
    torch.cuda.current_stream().synchronize()
    assert ttt.ttt_device_status() == 0
    assert Zh is out[0] and Wh is out[1]
    assert torch.equal(Zh, Zd.cpu()) and torch.equal(Wh, Wd.cpu())
