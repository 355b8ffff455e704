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
