"""Sequence-parallel forward of the TTT forms whose weight step is affine:
large-chunk TTT and TTT-Linear without LayerNorm.

Large-chunk TTT ("Test-Time Training Done Right", abstract) reads every chunk
out with the weight the chunks before it left, then takes one gradient step
on the chunk's eta-weighted reconstruction loss; TTT-Linear without LayerNorm
("Test-Time Training: Linear Complexity Beyond Attention", "Key Architectural
Mechanics of TTT-Linear", part 4) takes every gradient of a mini-batch at the
mini-batch's starting weight. Either way the step is affine in the weight,
W_{c+1} = (I - A_c) W_c + B_c, so a stretch of whole chunks (or mini-batches),
a segment, maps its starting weight to its final one by W -> M W + N, and a
long sequence's forward splits into three stages:

  1. every segment's (M, N), all segments at once   (ttt_chunk_map, ttt_linear_map)
  2. the fold of the maps into every segment's starting weight,
     W_in[j+1] = M_j W_in[j] + N_j                   (ttt_affine_prefix)
  3. every segment's forward from its starting weight, all at once
                                                     (ttt_chunk_fwd, ttt_linear_fwd)

Only stage 2 is sequential over segments, with nseg - 1 dependent d x d
products in place of the T / chunk dependent steps of the plain forward.

*_fwd_segmented run the three stages on one GPU, the segments of a sequence
becoming extra sequences of each call: [B][H][T][d] viewed, without a copy,
as [B][H * nseg][T / nseg][d]. *_fwd_seqpar run them with one process per
GPU, rank r holding tokens [r T_r, (r + 1) T_r) of every sequence; the maps
cross ranks once (an all-gather of 2 B H d^2 floats from each rank) and every
rank folds the same gathered maps, so every rank ends with the same final
weight.

Every arithmetic step runs in libttt.so's kernels; torch provides device
memory and torch.distributed the all-gather. Stage 1 costs two forwards (from
W = I with V = 0, and from W = 0), so a segment's work is about three
forwards of its tokens. The fold supports d = 64 and 128.
"""
from __future__ import annotations

import test_sequence_layers_layer_b200 as _lib


def _check(Q, K, V, eta, T_seg, size):
    if not (Q.shape == K.shape == V.shape) or Q.dim() != 4:
        raise ValueError("Q, K, V must be [B, H, T, d] of one shape")
    if tuple(eta.shape) != tuple(Q.shape[:3]):
        raise ValueError("eta must be [B, H, T]")
    for x in (Q, K, V, eta):
        if not x.is_contiguous():
            raise ValueError("Q, K, V and eta must be contiguous")
    if T_seg <= 0 or T_seg % size:
        raise ValueError("every segment must hold a whole number of chunks (mini-batches)")
    if Q.shape[3] not in (64, 128):
        raise ValueError("the fold of segment maps supports d = 64 and 128")


def _map(form, K, V, eta, size, stream):
    if form == "chunk":
        return _lib.chunk_map(K, V, eta, chunk=size, stream=stream)
    return _lib.linear_map(K, V, eta, b=size, stream=stream)


def _forward(form, Q, K, V, eta, W_in, size, z_bf16, stream):
    if form == "chunk":
        Z, _ = _lib.chunk_fwd(Q, K, V, eta, W_in, chunk=size, w0_per_seq=True, stream=stream,
                              want_w=False, z_bf16=z_bf16)
    else:
        Z, _ = _lib.linear_fwd(Q, K, V, eta, W_in, b=size, ln=False, w0_per_seq=True,
                               stream=stream, want_w=False, z_bf16=z_bf16)
    return Z


def _segmented(form, Q, K, V, eta, W0, size, nseg, w0_per_seq, z_bf16, stream):
    import torch
    B, H, T, d = Q.shape
    if nseg < 1 or T % nseg:
        raise ValueError("T must split into nseg equal segments")
    Ts = T // nseg
    _check(Q, K, V, eta, Ts, size)
    Qs, Ks, Vs = (x.view(B, H * nseg, Ts, d) for x in (Q, K, V))
    es = eta.view(B, H * nseg, Ts)
    M, N = _map(form, Ks, Vs, es, size, stream)  # [B][H][nseg][d][d]
    W_in = torch.empty_like(M)
    W_out = torch.empty((B, H, d, d), dtype=torch.float32, device=Q.device)
    _lib.affine_prefix(M, N, W0, W_in, W_out, S=B * H, H=H, nseg=nseg, seq_stride=nseg * d * d,
                       seg_stride=d * d, w0_per_seq=w0_per_seq, stream=stream)
    Z = _forward(form, Qs, Ks, Vs, es, W_in, size, z_bf16, stream)
    return Z.view(B, H, T, d), W_out


def _seqpar(form, Q, K, V, eta, W0, size, group, w0_per_seq, z_bf16):
    import torch
    import torch.distributed as dist
    R = dist.get_world_size(group)
    r = dist.get_rank(group)
    B, H, Tr, d = Q.shape
    _check(Q, K, V, eta, Tr, size)
    M, N = _map(form, K, V, eta, size, None)
    S = B * H
    Ms = torch.empty((R, B, H, d, d), dtype=torch.float32, device=Q.device)
    Ns = torch.empty_like(Ms)
    dist.all_gather(list(Ms.unbind(0)), M, group=group)
    dist.all_gather(list(Ns.unbind(0)), N, group=group)
    W_in = torch.empty_like(Ms)
    W_out = torch.empty((B, H, d, d), dtype=torch.float32, device=Q.device)
    _lib.affine_prefix(Ms, Ns, W0, W_in, W_out, S=S, H=H, nseg=R, seq_stride=d * d,
                       seg_stride=S * d * d, w0_per_seq=w0_per_seq)
    Z = _forward(form, Q, K, V, eta, W_in[r], size, z_bf16, None)
    return Z, W_out


def chunk_fwd_segmented(Q, K, V, eta, W0, *, chunk, nseg, w0_per_seq=False, z_bf16=False,
                        stream=None):
    """Large-chunk forward of [B, H, T, d] inputs split into nseg segments of
    T / nseg tokens (a multiple of chunk) on one GPU. W0 is [H, d, d], or
    [B, H, d, d] with w0_per_seq. Returns (Z [B, H, T, d], W_out [B, H, d, d])."""
    return _segmented("chunk", Q, K, V, eta, W0, chunk, nseg, w0_per_seq, z_bf16, stream)


def linear_fwd_segmented(Q, K, V, eta, W0, *, b, nseg, w0_per_seq=False, z_bf16=False,
                         stream=None):
    """TTT-Linear forward without LayerNorm (f(k) = k W, mini-batch b) split
    into nseg segments of T / nseg tokens (a multiple of b) on one GPU.
    Arguments and results as chunk_fwd_segmented."""
    return _segmented("linear", Q, K, V, eta, W0, b, nseg, w0_per_seq, z_bf16, stream)


def chunk_fwd_seqpar(Q, K, V, eta, W0, *, chunk, group=None, w0_per_seq=False, z_bf16=False):
    """Large-chunk forward with the sequence split across the ranks of
    `group` (one process per GPU): this rank's Q, K, V [B, H, T_r, d] and eta
    [B, H, T_r] are tokens [r T_r, (r + 1) T_r) of every sequence, T_r a
    multiple of chunk and equal on every rank; W0 ([H, d, d], or [B, H, d, d]
    with w0_per_seq) is the sequences' starting weight, the same on every
    rank. Returns (this rank's Z [B, H, T_r, d], the sequences' final weight
    [B, H, d, d], identical on every rank). Runs on torch's current stream;
    every rank must call it with the same shapes."""
    return _seqpar("chunk", Q, K, V, eta, W0, chunk, group, w0_per_seq, z_bf16)


def linear_fwd_seqpar(Q, K, V, eta, W0, *, b, group=None, w0_per_seq=False, z_bf16=False):
    """TTT-Linear forward without LayerNorm with the sequence split across
    the ranks of `group`; T_r a multiple of b. Arguments and results as
    chunk_fwd_seqpar."""
    return _seqpar("linear", Q, K, V, eta, W0, b, group, w0_per_seq, z_bf16)
