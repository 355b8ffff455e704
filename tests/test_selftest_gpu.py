"""The tensor-core plumbing (operand layouts, descriptors, TMEM) against torch.

Each case stages bf16 A and B in one canonical shared-memory layout, runs a
tcgen05 MMA chain into tensor memory through ttt_selftest_umma, and compares
D with torch's fp32 matmul of the same bf16 values."""
import pytest
import torch

import test_sequence_layers_layer_b200 as ttt

pytestmark = pytest.mark.gpu
KS, MS, KN = 0, 1, 2  # K-major 128B swizzle, MN-major 128B swizzle, K-major no swizzle

CASES = [
    (128, 64, 64, KS, MS), (64, 64, 64, KS, MS), (128, 64, 64, KS, KS),
    (64, 64, 16, MS, MS), (64, 64, 16, KN, MS), (128, 128, 64, KS, MS),
    (128, 256, 128, KS, MS), (128, 128, 128, MS, MS), (64, 16, 64, KS, KS),
    (128, 16, 64, KS, KS), (128, 64, 128, KN, MS), (64, 64, 32, MS, KS),
    # the TTT-MLP scan's product shapes
    (128, 32, 64, KS, KS), (64, 32, 256, MS, KS), (64, 16, 256, KS, KS),
    (128, 64, 16, KN, MS), (128, 64, 16, MS, MS),
]


@pytest.mark.parametrize("M,N,K,al,bl", CASES)
def test_umma_layouts(M, N, K, al, bl):
    g = torch.Generator(device="cuda").manual_seed(M * 1000 + N * 10 + K + al * 7 + bl)
    A = torch.randn(M, K, device="cuda", generator=g).to(torch.bfloat16)
    B = torch.randn(K, N, device="cuda", generator=g).to(torch.bfloat16)
    D = torch.full((M, N), float("nan"), device="cuda")
    ttt.ttt_selftest_umma(M, N, K, al, bl, A, B, D)
    torch.cuda.synchronize()
    assert ttt.ttt_device_status() == 0
    ref = A.double() @ B.double()
    err = (D.double() - ref).abs().max().item() / ref.abs().max().item()
    assert err < 1e-5, f"layout case {(M, N, K, al, bl)}: rel err {err}"


def test_mlp_gelu_against_exact():
    """The MLP kernel's GELU / GELU' (erf from Abramowitz & Stegun 7.1.26,
    |erf error| <= 1.5e-7) against the oracle's double-precision exact-erf
    GELU, on a dense grid over the range the scan sees and far tails."""
    import numpy as np
    import oracle
    h = np.concatenate([np.linspace(-12, 12, 200001), [0.0, -0.0, 1e-30, -1e-30, 40.0, -40.0]])
    h = h.astype(np.float32)
    x = torch.from_numpy(h).cuda()
    g = torch.empty_like(x)
    gp = torch.empty_like(x)
    ttt.ttt_diag_gelu(x, g, gp, x.numel())
    torch.cuda.synchronize()
    hd = h.astype(np.float64)
    ref_g = np.array([oracle.gelu(v) for v in hd[::7]])
    ref_gp = np.array([oracle.gelu_prime(v) for v in hd[::7]])
    g = g.double().cpu().numpy()[::7]
    gp = gp.double().cpu().numpy()[::7]
    # The formula in fp32 (evaluated off line on this grid) stays within 1.8e-7 * max(|h|, 1)
    # for GELU and 2.9e-7 for GELU'; the bounds leave room for the fast exp / reciprocal.
    assert np.all(np.abs(g - ref_g) <= 4e-7 * np.maximum(np.abs(hd[::7]), 1.0))
    assert np.all(np.abs(gp - ref_gp) <= 6e-7)


def test_bounded_wait_times_out_and_context_survives():
    """A device-side wait on a barrier nothing arrives on runs out after its
    limit, the kernel reports it through the status word and exits; the
    context stays usable (a TTT call afterwards is still correct)."""
    import time
    from test_sequence_layers_layer_b200 import synth
    from gpu_helpers import check_parity
    assert ttt.ttt_device_status() == 0
    assert ttt.ttt_diag_wait_timeout(0, check=False) == -1
    t0 = time.perf_counter()
    ttt.ttt_diag_wait_timeout(20000)  # 20 ms
    assert ttt.ttt_device_status() == -7  # TTT_ERR_DEVICE_TIMEOUT, read once and cleared
    elapsed = time.perf_counter() - t0
    assert 0.015 <= elapsed < 5.0
    assert ttt.ttt_device_status() == 0
    wl = synth.WORKLOADS["linear_ln_d64_b8h12_t2048"].scaled(B=1, H=2, T=64)
    check_parity(synth.make_inputs(wl))


def test_kernel_timing_sums_over_calls_without_sync():
    """Per-kernel event timing kept across several calls: one read after the
    loop returns, per kernel position, the summed durations; each is positive
    and together they fit inside the outer events around the calls. The
    large-chunk backward (d = 128, bf16, chunk 256) with a shared W0 launches
    six kernels (Gram, scan, the three token passes, sum over the batch)."""
    from test_sequence_layers_layer_b200 import synth
    from gpu_helpers import to_dev
    wl = synth.WORKLOADS["chunk_d128_c2048_b4h8_t32768"].scaled(B=1, H=2, T=1024, b=256)
    x = to_dev(synth.make_inputs(wl))
    dZ = torch.randn((wl.B, wl.H, wl.T, wl.d), device="cuda")
    ws = torch.empty(ttt.ttt_chunk_bwd_workspace_bytes(wl.B, wl.H, wl.T, wl.d, wl.b),
                     dtype=torch.uint8, device="cuda")

    def call():
        return ttt.chunk_bwd(x["Q"], x["K"], x["V"], x["eta"], x["W1"], dZ, chunk=wl.b, workspace=ws)

    call()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ttt.ttt_diag_kernel_timing(True)
    try:
        e0.record()
        for _ in range(3):
            call()
        e1.record()
        times = ttt.ttt_diag_kernel_times(8)
    finally:
        ttt.ttt_diag_kernel_timing(False)
    torch.cuda.synchronize()
    assert len(times) == 6 and all(t > 0 for t in times), times
    assert sum(times) <= e0.elapsed_time(e1) * 1.001 + 1e-3
    assert ttt.ttt_diag_kernel_times(8) == []  # disabled: nothing recorded
