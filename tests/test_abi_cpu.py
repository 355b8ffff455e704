"""The C-ABI library without a GPU: it loads, exports every function
include/ttt.h declares, and rejects bad arguments on the host before any
launch."""
import ctypes

import pytest

import test_sequence_layers_layer_b200 as ttt

ALIGNED = 1 << 20  # a fake, 16-byte aligned "device" address; never dereferenced


def test_library_loads_and_exports_header_symbols():
    L = ttt.lib()
    syms = ttt.header_symbols()
    assert set(syms) >= {"ttt_linear_fwd", "ttt_mlp_fwd", "ttt_chunk_fwd",
                         "ttt_chunk_workspace_bytes", "ttt_status_string",
                         "ttt_abi_version", "ttt_device_status"}
    for s in syms:
        assert hasattr(L, s), s
    assert ttt.abi_version() == 1


def test_status_strings():
    for code in range(-9, 1):
        assert ttt.status_string(code) not in ("", "unknown status")
    assert ttt.status_string(-1234) == "unknown status"


def lin(**kw):
    args = dict(Q=ALIGNED, K=ALIGNED, V=ALIGNED, eta=ALIGNED, W0=ALIGNED, ln_gamma=ALIGNED,
                ln_beta=ALIGNED, Z=ALIGNED, W_out=None, B=1, H=1, T=64, d=64, b=16,
                dt=ttt.TTT_BF16, flags=ttt.TTT_F_LN, stream=0)
    args.update(kw)
    return ttt.ttt_linear_fwd(**args, check=False)


@pytest.mark.parametrize("kw,code", [
    (dict(T=0), -2),
    (dict(d=48), -2),              # unsupported d
    (dict(b=0), -2),
    (dict(B=0), -2),
    (dict(dt=7), -3),
    (dict(flags=16), -1),          # unknown flag bit
    (dict(flags=ttt.TTT_F_LN | ttt.TTT_F_L2_KEYS), -8),  # L2 keys pass the host checks
    (dict(Q=None), -5),
    (dict(ln_gamma=None), -5),     # LN requires gamma/beta
    (dict(Q=ALIGNED + 4), -4),     # misaligned
    (dict(Z=ALIGNED + 8), -4),
    (dict(W_out=ALIGNED, W0=ALIGNED), -1),  # aliasing W_out/W0 without per-seq W0
])
def test_linear_host_validation(kw, code):
    assert lin(**kw) == code


def test_linear_accepts_a_partial_last_minibatch():
    # T = 60 with b = 16: three full mini-batches and one of 12 tokens pass the
    # host checks; without a GPU the arch check then fails
    assert lin(T=60) in (-8, -5)
    assert lin(T=7) in (-8, -5)


def test_linear_without_ln_does_not_need_gamma():
    # validation passes; on a machine without a GPU the arch check then fails
    rc = lin(ln_gamma=None, ln_beta=None, flags=0)
    assert rc in (-8, -5)


def test_mlp_and_chunk_host_validation():
    m = dict(Q=ALIGNED, K=ALIGNED, V=ALIGNED, eta=ALIGNED, W1_0=ALIGNED, W2_0=ALIGNED,
             ln_gamma=ALIGNED, ln_beta=ALIGNED, Z=ALIGNED, W1_out=None, W2_out=None,
             B=1, H=1, T=32, d=64, dh=256, b=16, dt=ttt.TTT_BF16, flags=ttt.TTT_F_LN, stream=0)
    assert ttt.ttt_mlp_fwd(**{**m, "dh": 128}, check=False) == -2
    assert ttt.ttt_mlp_fwd(**{**m, "flags": 0}, check=False) == -1   # MLP needs LN
    assert ttt.ttt_mlp_fwd(**{**m, "b": 32}, check=False) == -2
    assert ttt.ttt_mlp_fwd(**{**m, "T": 40}, check=False) == -2   # MLP: T % b == 0
    c = dict(Q=ALIGNED, K=ALIGNED, V=ALIGNED, eta=ALIGNED, W0=ALIGNED, Z=ALIGNED, W_out=None,
             B=1, H=1, T=4096, d=128, chunk=2048, dt=ttt.TTT_BF16, flags=0,
             workspace=None, workspace_bytes=0, stream=0)
    assert ttt.ttt_chunk_fwd(**{**c, "chunk": 1000}, check=False) == -2
    assert ttt.ttt_chunk_fwd(**{**c, "T": 3000}, check=False) == -2
    assert ttt.ttt_chunk_fwd(**{**c, "flags": ttt.TTT_F_LN}, check=False) == -1


def test_no_gpu_means_unsupported_not_fallback():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert lin() == -8


def test_backward_host_validation():
    """ttt_linear_bwd and ttt_chunk_bwd reject bad arguments before any launch
    (the workspace check comes before the architecture check, so a too-small
    workspace is reported even without a GPU)."""
    A = ALIGNED
    lb = dict(Q=A, K=A, V=A, eta=A, W0=A, ln_gamma=A, ln_beta=A, dZ=A, dW_out=None, dQ=A, dK=A,
              dV=A, deta=A, dW0=A, dgamma=A, dbeta=A, B=1, H=2, T=64, d=64, b=16,
              dt=ttt.TTT_BF16, flags=ttt.TTT_F_LN, workspace=A, workspace_bytes=1 << 30, stream=0)
    call = lambda **kw: ttt.ttt_linear_bwd(**{**lb, **kw}, check=False)  # noqa: E731
    need = ttt.ttt_linear_bwd_workspace_bytes(1, 2, 64, 64, 16)
    assert need == 4 * (2 * 4 * 64 * 64 + 2 * 64 * 64 + 2 * 2 * 64)
    assert call(flags=ttt.TTT_F_Z_BF16) == -1        # not a backward flag
    assert call(dgamma=None) == -5                    # LN needs dgamma, dbeta
    assert call(T=60) == -2                           # backward: T % b == 0
    assert call(d=48) == -2
    assert call(workspace_bytes=need - 1) == -9
    assert call(workspace=A + 16) == -9               # not 256-byte aligned
    cb = dict(Q=A, K=A, V=A, eta=A, W0=A, dZ=A, dW_out=None, dQ=A, dK=A, dV=A, deta=A, dW0=A,
              B=1, H=2, T=4096, d=128, chunk=2048, dt=ttt.TTT_BF16, flags=0, workspace=A,
              workspace_bytes=1 << 34, stream=0)
    call = lambda **kw: ttt.ttt_chunk_bwd(**{**cb, **kw}, check=False)  # noqa: E731
    need = ttt.ttt_chunk_bwd_workspace_bytes(1, 2, 4096, 128, 2048)
    # fp32 per chunk (A_c, B_c, Q_c^T dZ_c, W_c, Om_{c+1}) and per sequence (dW0)
    assert need == 4 * (5 * 4 * 128 * 128 + 2 * 128 * 128)
    assert ttt.ttt_chunk_bwd_workspace_bytes(1, 2, 4096, 128, 32) == 4 * (5 * 256 * 128 * 128
                                                                         + 2 * 128 * 128)
    assert ttt.ttt_chunk_bwd_workspace_bytes(1, 2, 4096, 64, 2048) == 4 * (5 * 4 + 2) * 64 * 64
    assert ttt.ttt_chunk_bwd_workspace_bytes(1, 2, 4096, 96, 2048) == 0
    assert call(flags=ttt.TTT_F_LN) == -1
    assert call(dQ=None) == -5
    assert call(d=96) == -2
    assert call(chunk=48) == -2                       # chunk % 32 != 0
    assert call(T=5000) == -2                         # T % chunk != 0
    assert call(dQ=A + 4) == -4
    assert call(workspace_bytes=need - 1) == -9


def test_chunk_map_and_affine_prefix_host_validation():
    """ttt_chunk_map and ttt_affine_prefix reject bad arguments before any
    launch; arguments that pass every host check reach the architecture
    check, which fails without a GPU."""
    A = ALIGNED
    B, H, T, d, C = 1, 2, 4096, 128, 2048
    need = ttt.ttt_chunk_map_workspace_bytes(B, H, T, d, C, ttt.TTT_BF16)
    n = B * H * T * d
    r256 = lambda x: (x + 255) // 256 * 256  # noqa: E731
    # tensor-core shapes: one Gram pass and one [M | N] scan in the forward's workspace
    assert need == ttt.ttt_chunk_workspace_bytes(B, H, T, d, C)
    # fp32 runs the CUDA-core forward, which needs no workspace of its own
    assert ttt.ttt_chunk_map_workspace_bytes(B, H, T, d, C, ttt.TTT_FP32) == \
        r256(4 * n) + r256(2 * n) + r256(4 * B * H * d * d)
    assert ttt.ttt_chunk_map_workspace_bytes(B, H, T, 96, C, ttt.TTT_BF16) == 0
    assert ttt.ttt_chunk_map_workspace_bytes(B, H, 3000, d, C, ttt.TTT_BF16) == 0
    cm = dict(K=A, V=A, eta=A, M=A, N=A + (1 << 20), B=B, H=H, T=T, d=d, chunk=C,
              dt=ttt.TTT_BF16, workspace=A, workspace_bytes=need, stream=0)
    call = lambda **kw: ttt.ttt_chunk_map(**{**cm, **kw}, check=False)  # noqa: E731
    assert call(K=None) == -5
    assert call(T=3000) == -2
    assert call(chunk=1000) == -2
    assert call(d=96) == -2
    assert call(dt=7) == -3
    assert call(M=A + 4) == -4
    assert call(N=A) == -1                        # M and N must differ
    assert call(workspace_bytes=need - 1) == -9
    assert call(workspace=A + 16) == -9
    assert call() == -8                           # no GPU here
    dd = 64 * 64
    ap = dict(M=A, N=A + (1 << 22), W0=A + (2 << 22), W_in=A + (3 << 22), W_end=None, S=4, H=2,
              nseg=3, d=64, seq_stride=3 * dd, seg_stride=dd, flags=0, stream=0)
    call = lambda **kw: ttt.ttt_affine_prefix(**{**ap, **kw}, check=False)  # noqa: E731
    assert call() == -8                           # sequence-major layout passes
    assert call(seq_stride=dd, seg_stride=4 * dd) == -8   # segment-major layout passes
    assert call(seq_stride=dd, seg_stride=dd) == -1       # (s, j) blocks would overlap
    assert call(seq_stride=2 * dd) == -1                  # 3 segments do not fit
    assert call(seg_stride=dd - 4) == -1
    assert call(seq_stride=3 * dd + 2) == -4              # stride not a multiple of 4
    assert call(nseg=1, seq_stride=dd, seg_stride=0) == -8
    assert call(S=3) == -2                                # shared W0: S % H == 0
    assert call(S=3, flags=ttt.TTT_F_W0_PER_SEQ) == -8
    assert call(d=32) == -2
    assert call(flags=ttt.TTT_F_LN) == -1
    assert call(W_in=None) == -5
    assert call(W_in=A) == -1                             # output aliases M
    assert call(W_end=A + (1 << 22)) == -1                # output aliases N
    assert call(W0=A + 8) == -4


def test_linear_map_host_validation():
    A = ALIGNED
    B, H, T, d, b = 1, 2, 256, 64, 16
    need = ttt.ttt_linear_map_workspace_bytes(B, H, T, d, b, ttt.TTT_BF16)
    n = B * H * T * d
    r256 = lambda x: (x + 255) // 256 * 256  # noqa: E731
    assert need == r256(2 * n) + r256(2 * n) + r256(4 * B * H * d * d)
    assert ttt.ttt_linear_map_workspace_bytes(B, H, T, 48, b, ttt.TTT_BF16) == 0
    assert ttt.ttt_linear_map_workspace_bytes(B, H, T, d, 128, ttt.TTT_BF16) == 0
    lm = dict(K=A, V=A, eta=A, M=A, N=A + (1 << 20), B=B, H=H, T=T, d=d, b=b, dt=ttt.TTT_BF16,
              workspace=A, workspace_bytes=need, stream=0)
    call = lambda **kw: ttt.ttt_linear_map(**{**lm, **kw}, check=False)  # noqa: E731
    assert call(eta=None) == -5
    assert call(d=48) == -2
    assert call(b=0) == -2
    assert call(dt=5) == -3
    assert call(N=A) == -1
    assert call(V=A + 2) == -4
    assert call(workspace_bytes=need - 1) == -9
    assert call() == -8                           # no GPU here
    assert call(T=250) == -8                      # a partial last mini-batch is accepted


def test_linear_fwd_steps_host_validation():
    A = ALIGNED
    st = dict(Q=A, K=A, V=A, eta=A, W0=A, ln_gamma=A, ln_beta=A, Z=A, W_out=None, B=1, H=2, T=64,
              d=64, n_steps=2, dt=ttt.TTT_BF16, flags=ttt.TTT_F_LN, stream=0)
    call = lambda **kw: ttt.ttt_linear_fwd_steps(**{**st, **kw}, check=False)  # noqa: E731
    assert call(n_steps=0) == -1
    assert call(n_steps=1025) == -1
    assert call(flags=16) == -1
    assert call(d=128) == -2
    assert call(ln_beta=None) == -5
    assert call(Z=A + 4) == -4
    assert call(W_out=A) == -1                  # aliasing W0 without per-sequence W0
    assert call() == -8                         # no GPU here
    assert call(flags=ttt.TTT_F_L2_KEYS | ttt.TTT_F_Z_BF16, n_steps=1024) == -8


def test_mlp_backward_host_validation():
    A = ALIGNED
    B, H, T, d, b = 1, 2, 64, 64, 16
    need = ttt.ttt_mlp_bwd_workspace_bytes(B, H, T, d, 4 * d, b)
    assert need > 4 * B * H * (T // b) * 2 * d * 4 * d  # the checkpoints and more
    assert ttt.ttt_mlp_bwd_workspace_bytes(B, H, T, d, 3 * d, b) == 0
    assert ttt.ttt_mlp_bwd_workspace_bytes(B, H, T, 128, 512, b) == 0
    mb = dict(Q=A, K=A, V=A, eta=A, W1_0=A, W2_0=A, ln_gamma=A, ln_beta=A, dZ=A, dW1_out=None,
              dW2_out=None, dQ=A, dK=A, dV=A, deta=A, dW1_0=A, dW2_0=A, dgamma=A, dbeta=A, B=B,
              H=H, T=T, d=d, dh=4 * d, b=b, dt=ttt.TTT_BF16, flags=ttt.TTT_F_LN, workspace=A,
              workspace_bytes=need, stream=0)
    call = lambda **kw: ttt.ttt_mlp_bwd(**{**mb, **kw}, check=False)  # noqa: E731
    assert call(flags=0) == -1                        # TTT-MLP always has its LayerNorm
    assert call(flags=ttt.TTT_F_LN | ttt.TTT_F_Z_BF16) == -1
    assert call(dgamma=None) == -5
    assert call(T=60) == -2                           # T % b
    assert call(b=32, T=64) == -2                     # b <= 16
    assert call(dh=128) == -2
    assert call(dt=9) == -3
    assert call(workspace_bytes=need - 1) == -9
    assert call(workspace=A + 64) == -9
    assert call() == -8                               # no GPU here


def test_decode_host_validation():
    A = ALIGNED
    dc = dict(q=A, k=A, v=A, eta=A, W=A, ln_gamma=A, ln_beta=A, z=A, B=2, H=3, d=64,
              dt=ttt.TTT_BF16, flags=ttt.TTT_F_LN, stream=0)
    call = lambda **kw: ttt.ttt_linear_decode(**{**dc, **kw}, check=False)  # noqa: E731
    assert call(d=32) == -2                     # the decode kernel is d = 64
    assert call(flags=ttt.TTT_F_W0_PER_SEQ) == -1
    assert call(ln_gamma=None) == -5
    assert call(W=A + 8) == -4
    assert call(dt=4) == -3
    assert call(flags=0, ln_gamma=None, ln_beta=None) == -8   # valid without LN; no GPU here


def test_mlp_decode_host_validation():
    A = ALIGNED
    md = dict(q=A, k=A, v=A, eta=A, W1=A, W2=A + (1 << 20), ln_gamma=A, ln_beta=A, z=A, B=2,
              H=3, d=64, dh=256, dt=ttt.TTT_BF16, flags=ttt.TTT_F_LN, stream=0)
    call = lambda **kw: ttt.ttt_mlp_decode(**{**md, **kw}, check=False)  # noqa: E731
    assert call(flags=0) == -1                  # TTT-MLP always has its LayerNorm
    assert call(dh=128) == -2 and call(d=32, dh=128) == -2
    assert call(W2=A) == -1                     # W1 and W2 must differ
    assert call(ln_beta=None) == -5
    assert call(z=A + 2) == -4
    assert call() == -8                         # no GPU here
