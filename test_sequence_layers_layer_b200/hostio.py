"""TTT-Linear and large-chunk forwards on inputs that live in host memory,
with the copies overlapped with the compute.

The (batch, head) grid is cut into `slices` groups: whole batch rows while
there are at least as many rows as groups, else each row's heads split into
runs (a run of heads of one row is contiguous in [B, H, T, d], and W0, gamma
and beta are cut to the same heads). Each group runs on its own CUDA stream:
its Q, K, V and eta are copied to the device, ttt_linear_fwd runs on them,
and its Z and W_out are copied back. The host-to-device copies are issued in
group order, each after the previous group's (so the first group's kernel
starts after 1/slices of the input has crossed, not all of it); the
host-to-device copies of later groups, the device-to-host copies of earlier
ones and the kernels of the groups in between then proceed at the same time.
A sequence's result does not depend on which other sequences share its call,
so the outputs equal those of one ttt_linear_fwd (ttt_chunk_fwd) call over
the whole batch.

Host tensors must be in pinned (page-locked) memory for the copies to run
asynchronously. torch provides the memory, the streams and the copies; every
step of the computation runs in libttt.so's kernels.
"""
from __future__ import annotations

import test_sequence_layers_layer_b200 as _lib


_STREAMS = {}


def _streams(dev, n):
    """n side streams of device dev, created once and reused."""
    import torch
    have = _STREAMS.setdefault(dev.index, [])
    while len(have) < n:
        have.append(torch.cuda.Stream(dev))
    return have[:n]


def _split(n: int, parts: int):
    """[0, n) cut into `parts` runs whose lengths differ by at most one."""
    q, r = divmod(n, parts)
    out, a = [], 0
    for i in range(parts):
        b = a + q + (1 if i < r else 0)
        out.append((a, b))
        a = b
    return out


def _bounds(B: int, H: int, slices: int):
    """Groups (b0, b1, h0, h1): whole batch rows when slices <= B, else runs
    of heads of one batch row each (about slices / B runs per row)."""
    if slices <= B:
        return [(b0, b1, 0, H) for b0, b1 in _split(B, max(1, slices))]
    per_row = min(H, -(-slices // B))
    return [(b, b + 1, h0, h1) for b in range(B) for h0, h1 in _split(H, per_row)]


def _outputs(Q, z_bf16, out):
    """(Z, W_out) pinned host tensors: the caller's `out` pair, else new ones."""
    import torch
    if out is not None:
        return out
    B, H, T, d = Q.shape
    Zh = torch.empty((B, H, T, d), dtype=torch.bfloat16 if z_bf16 else torch.float32,
                     pin_memory=True)
    Wh = torch.empty((B, H, d, d), dtype=torch.float32, pin_memory=True)
    return Zh, Wh


def linear_fwd_host(Q, K, V, eta, W0, ln_gamma=None, ln_beta=None, *, b, ln, slices=4,
                    z_bf16=False, device=None, out=None):
    """TTT-Linear forward of host tensors Q, K, V [B, H, T, d] (bf16 or fp32)
    and eta [B, H, T]; W0 [H, d, d] and the LayerNorm gain and bias [H, d] may
    be on the host or the device. Returns (Z, W_out) as pinned host tensors
    (`out`, a pinned (Z, W_out) pair of the right shapes, if given), valid once
    torch's current stream has reached the point of return (for example after
    torch.cuda.current_stream().synchronize())."""
    import torch
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    B, H, T, d = Q.shape
    cur = torch.cuda.current_stream(dev)
    W0d = W0.to(dev, non_blocking=True)
    gd = ln_gamma.to(dev, non_blocking=True) if ln_gamma is not None else None
    bd = ln_beta.to(dev, non_blocking=True) if ln_beta is not None else None
    Zh, Wh = _outputs(Q, z_bf16, out)
    bounds = _bounds(B, H, slices)
    streams = _streams(dev, len(bounds))
    prev = None  # the previous group's input copies
    for (b0, b1, h0, h1), st in zip(bounds, streams):
        st.wait_stream(cur)  # W0, gamma, beta are copied on the current stream
        if prev is not None:
            st.wait_event(prev)
        with torch.cuda.stream(st):
            q, k, v, e = (x[b0:b1, h0:h1].to(dev, non_blocking=True) for x in (Q, K, V, eta))
            prev = torch.cuda.Event()
            prev.record(st)
            Z, W = _lib.linear_fwd(q, k, v, e, W0d[h0:h1],
                                   gd[h0:h1] if gd is not None else None,
                                   bd[h0:h1] if bd is not None else None,
                                   b=b, ln=ln, stream=st, z_bf16=z_bf16)
            Zh[b0:b1, h0:h1].copy_(Z, non_blocking=True)
            Wh[b0:b1, h0:h1].copy_(W, non_blocking=True)
    for st in streams:
        cur.wait_stream(st)
    return Zh, Wh


def chunk_fwd_host(Q, K, V, eta, W0, *, chunk, slices=4, w0_per_seq=False, z_bf16=False,
                   device=None, out=None):
    """Large-chunk forward of host tensors Q, K, V [B, H, T, d] and eta
    [B, H, T]; W0 ([H, d, d], or [B, H, d, d] with w0_per_seq) on the host or
    the device. Each group of batch rows gets its own workspace (allocated by
    torch on its stream), so the groups' kernels may overlap. Returns (Z, W_out)
    as pinned host tensors (`out` if given), valid once torch's current stream
    has reached the point of return."""
    import torch
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    B = Q.shape[0]
    cur = torch.cuda.current_stream(dev)
    W0d = W0.to(dev, non_blocking=True)
    Zh, Wh = _outputs(Q, z_bf16, out)
    H = Q.shape[1]
    bounds = _bounds(B, H, slices)
    streams = _streams(dev, len(bounds))
    prev = None  # the previous group's input copies
    for (b0, b1, h0, h1), st in zip(bounds, streams):
        st.wait_stream(cur)  # W0 is copied on the current stream
        if prev is not None:
            st.wait_event(prev)
        with torch.cuda.stream(st):
            q, k, v, e = (x[b0:b1, h0:h1].to(dev, non_blocking=True) for x in (Q, K, V, eta))
            prev = torch.cuda.Event()
            prev.record(st)
            w0 = W0d[b0:b1, h0:h1] if w0_per_seq else W0d[h0:h1]
            Z, W = _lib.chunk_fwd(q, k, v, e, w0, chunk=chunk, w0_per_seq=w0_per_seq, stream=st,
                                  z_bf16=z_bf16)
            Zh[b0:b1, h0:h1].copy_(Z, non_blocking=True)
            Wh[b0:b1, h0:h1].copy_(W, non_blocking=True)
    for st in streams:
        cur.wait_stream(st)
    return Zh, Wh
