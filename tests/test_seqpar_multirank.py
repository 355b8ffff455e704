"""The sequence-parallel forward's host logic on CPU, with two and three gloo
ranks, for large-chunk TTT and TTT-Linear without LayerNorm. The library's
calls (chunk_map / linear_map, affine_prefix, chunk_fwd / linear_fwd) are
replaced in each rank by fakes built on the oracle, so what is
checked is the orchestration around them: the tokens each rank holds, the
order of the all-gathered maps, the strides handed to the fold (the fake
reads M, N and W_in at exactly the offsets the C ABI defines), and which
starting weight each rank runs from. The result must equal the oracle's
forward of the whole sequence, and every rank must end with the same final
weight."""
import os
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

B, H, T, d, CHUNK = 2, 2, 48, 64, 8


def _inputs(w0_per_seq):
    r = np.random.default_rng(17)
    Q, K, V = (r.standard_normal((B, H, T, d)) for _ in range(3))
    eta = 0.02 * r.uniform(0.2, 1.0, (B, H, T))
    K /= np.sqrt(d)
    W0 = r.standard_normal((B, H, d, d) if w0_per_seq else (H, d, d)) / np.sqrt(d)
    return Q, K, V, eta, W0


def _fakes():
    import oracle
    from oracle import affine

    def chunk_map(K, V, eta, *, chunk, workspace=None, stream=None):
        M, N = affine.segment_map(K.double().numpy(), V.double().numpy(), eta.double().numpy(),
                                  chunk=chunk)
        return torch.from_numpy(M).float(), torch.from_numpy(N).float()

    def affine_prefix(M, N, W0, W_in, W_end=None, *, S, H, nseg, seq_stride, seg_stride,
                      w0_per_seq=False, stream=None):
        dd = M.shape[-1] ** 2
        dm = M.shape[-1]
        m, n, wi = M.reshape(-1), N.reshape(-1), W_in.reshape(-1)
        w0 = W0.reshape(-1, dm, dm)
        for s in range(S):
            W = w0[s if w0_per_seq else s % H].double().numpy()
            for j in range(nseg):
                o = s * seq_stride + j * seg_stride
                wi[o:o + dd] = torch.from_numpy(W.reshape(-1)).float()
                W = affine.apply_map(m[o:o + dd].double().numpy().reshape(dm, dm),
                                     n[o:o + dd].double().numpy().reshape(dm, dm), W)
            if W_end is not None:
                W_end.reshape(-1, dm, dm)[s] = torch.from_numpy(W).float()

    def chunk_fwd(Q, K, V, eta, W0, *, chunk, w0_per_seq=False, workspace=None, stream=None,
                  want_w=True, z_bf16=False):
        Z, Wo = oracle.chunk_primal(Q.double().numpy(), K.double().numpy(), V.double().numpy(),
                                    eta.double().numpy(), W0.double().numpy(), chunk=chunk,
                                    w0_per_seq=w0_per_seq)
        return torch.from_numpy(Z).float(), (torch.from_numpy(Wo).float() if want_w else None)

    def linear_map(K, V, eta, *, b, workspace=None, stream=None):
        return chunk_map(K, V, eta, chunk=b)

    def linear_fwd(Q, K, V, eta, W0, ln_gamma=None, ln_beta=None, *, b, ln, w0_per_seq=False,
                   stream=None, want_w=True, z_bf16=False):
        assert not ln
        Z, Wo = oracle.linear_primal(Q.double().numpy(), K.double().numpy(), V.double().numpy(),
                                     eta.double().numpy(), W0.double().numpy(), b=b, ln=False,
                                     w0_per_seq=w0_per_seq)
        return torch.from_numpy(Z).float(), (torch.from_numpy(Wo).float() if want_w else None)

    return chunk_map, affine_prefix, chunk_fwd, linear_map, linear_fwd


def _rank_main(rank, world, port, w0_per_seq, form, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import test_sequence_layers_layer_b200 as ttt
        from test_sequence_layers_layer_b200 import seqpar
        (ttt.chunk_map, ttt.affine_prefix, ttt.chunk_fwd, ttt.linear_map,
         ttt.linear_fwd) = _fakes()
        Q, K, V, eta, W0 = _inputs(w0_per_seq)
        Tr = T // world
        sl = slice(rank * Tr, (rank + 1) * Tr)
        t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).float()  # noqa: E731
        args = (t(Q[:, :, sl]), t(K[:, :, sl]), t(V[:, :, sl]), t(eta[:, :, sl]), t(W0))
        if form == "chunk":
            Z, W_out = seqpar.chunk_fwd_seqpar(*args, chunk=CHUNK, w0_per_seq=w0_per_seq)
        else:
            Z, W_out = seqpar.linear_fwd_seqpar(*args, b=CHUNK, w0_per_seq=w0_per_seq)
        out[rank] = (Z.numpy(), W_out.numpy())
    finally:
        dist.destroy_process_group()


def _whole(form, Q, K, V, eta, W0, w0_per_seq):
    import oracle
    if form == "chunk":
        return oracle.chunk_primal(Q, K, V, eta, W0, chunk=CHUNK, w0_per_seq=w0_per_seq)
    return oracle.linear_primal(Q, K, V, eta, W0, b=CHUNK, ln=False, w0_per_seq=w0_per_seq)


@pytest.mark.parametrize("world,w0_per_seq,form", [(2, False, "chunk"), (3, True, "chunk"),
                                                   (2, True, "linear")])
def test_seqpar_ranks_reproduce_the_whole_sequence(world, w0_per_seq, form):
    port = 29600 + os.getpid() % 1000 + 7 * world + (50 if form == "linear" else 0)
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, port, w0_per_seq, form, out), nprocs=world, join=True)
        res = dict(out)
    Q, K, V, eta, W0 = _inputs(w0_per_seq)
    Z_ref, W_ref = _whole(form, Q, K, V, eta, W0, w0_per_seq)
    Z = np.concatenate([res[r][0] for r in range(world)], axis=2)
    scale = np.abs(Z_ref).max()
    assert np.abs(Z - Z_ref).max() <= 1e-5 * scale
    for r in range(world):
        assert np.array_equal(res[r][1], res[0][1])  # the same final weight on every rank
    assert np.abs(res[0][1] - W_ref).max() <= 1e-5 * np.abs(W_ref).max()
    # the later ranks' tokens really depend on the fold: from W0 instead they differ
    Tr = T // world
    sl = slice(Tr, 2 * Tr)
    Z_w0, _ = _whole(form, Q[:, :, sl], K[:, :, sl], V[:, :, sl], eta[:, :, sl], W0, w0_per_seq)
    assert np.abs(res[1][0] - Z_w0).max() > 1e-3 * scale
