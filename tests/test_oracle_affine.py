"""Pins of the affine segment maps (oracle/affine.py) to the C oracle's
token-by-token forwards, which share no code with them: the map applied to a
starting weight must give the weight the chunk-by-chunk (or mini-batch by
mini-batch) primal form ends with, for two different starting weights (so M
and N are both fixed); running the segments one after another from the
prefix weights must reproduce the whole sequence's Z and final weight; and
eta = 0 gives the identity map."""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from oracle import affine  # noqa: E402


def _inputs(seed, B, H, T, d, eta_scale=0.02):
    r = np.random.default_rng(seed)
    K, V, Q = (r.standard_normal((B, H, T, d)) for _ in range(3))
    eta = eta_scale * r.uniform(0.2, 1.0, (B, H, T))
    return Q, K, V, eta


def _close(a, b, tol=1e-11):
    return np.abs(a - b).max() <= tol * max(1.0, np.abs(b).max())


@pytest.mark.parametrize("chunk", [4, 8, 24])
def test_map_reproduces_chunk_primal_weight(chunk):
    B, H, T, d = 2, 2, 24, 5
    Q, K, V, eta = _inputs(1, B, H, T, d)
    M, N = affine.segment_map(K, V, eta, chunk=chunk)
    r = np.random.default_rng(2)
    for _ in range(2):
        W0 = r.standard_normal((B, H, d, d)) / np.sqrt(d)
        _, Wc = oracle.chunk_primal(Q, K, V, eta, W0, chunk=chunk, w0_per_seq=True)
        assert _close(affine.apply_map(M, N, W0), Wc)


def test_map_reproduces_linear_no_ln_weight():
    """TTT-Linear without LayerNorm: mini-batch b is a chunk of b."""
    B, H, T, d, b = 1, 2, 16, 4, 4
    Q, K, V, eta = _inputs(3, B, H, T, d, eta_scale=0.05)
    M, N = affine.segment_map(K, V, eta, chunk=b)
    W0 = np.random.default_rng(4).standard_normal((H, d, d)) / 2
    _, Wl = oracle.linear_primal(Q, K, V, eta, W0, b=b, ln=False)
    assert _close(affine.apply_map(M, N, np.broadcast_to(W0, (B, H, d, d))), Wl)


@pytest.mark.parametrize("nseg", [2, 3, 6])
def test_segments_from_prefix_weights_equal_whole_sequence(nseg):
    """Split T into nseg runs of whole chunks, map each run independently,
    fold the maps into every run's starting weight, run each segment alone
    from it: Z and the final weight equal the whole-sequence forward."""
    B, H, T, d, chunk = 2, 1, 48, 6, 8
    Q, K, V, eta = _inputs(5, B, H, T, d)
    W0 = np.random.default_rng(6).standard_normal((H, d, d)) / np.sqrt(d)
    Z_ref, W_ref = oracle.chunk_primal(Q, K, V, eta, W0, chunk=chunk)
    Ts = T // nseg
    segs = [slice(j * Ts, (j + 1) * Ts) for j in range(nseg)]
    maps = [affine.segment_map(K[:, :, s], V[:, :, s], eta[:, :, s], chunk=chunk) for s in segs]
    W_in, W_end = affine.prefix_weights(maps, np.broadcast_to(W0, (B, H, d, d)))
    Z = np.concatenate([oracle.chunk_primal(Q[:, :, s], K[:, :, s], V[:, :, s], eta[:, :, s],
                                            W_in[j], chunk=chunk, w0_per_seq=True)[0]
                        for j, s in enumerate(segs)], axis=2)
    assert _close(Z, Z_ref)
    assert _close(W_end, W_ref)


def test_compose_is_the_map_of_the_concatenation():
    B, H, T, d, chunk = 1, 2, 32, 4, 8
    _, K, V, eta = _inputs(7, B, H, T, d, eta_scale=0.1)
    h = T // 2
    first = affine.segment_map(K[:, :, :h], V[:, :, :h], eta[:, :, :h], chunk=chunk)
    second = affine.segment_map(K[:, :, h:], V[:, :, h:], eta[:, :, h:], chunk=chunk)
    whole = affine.segment_map(K, V, eta, chunk=chunk)
    Mc, Nc = affine.compose(first, second)
    assert _close(Mc, whole[0]) and _close(Nc, whole[1])
    # order matters: the other order is a different map for generic inputs
    Mr, _ = affine.compose(second, first)
    assert not _close(Mr, whole[0], 1e-6)


def test_eta_zero_is_the_identity_map():
    _, K, V, eta = _inputs(8, 1, 1, 16, 3)
    M, N = affine.segment_map(K, V, 0.0 * eta, chunk=4)
    assert np.array_equal(M[0, 0], np.eye(3)) and not N.any()


def test_scalar_case_by_hand():
    """d = 1, one chunk of two tokens: A = eta1 k1^2 + eta2 k2^2,
    B = eta1 k1 v1 + eta2 k2 v2, the map is w -> (1 - A) w + B."""
    K = np.array([2.0, -1.0]).reshape(1, 1, 2, 1)
    V = np.array([0.5, 3.0]).reshape(1, 1, 2, 1)
    eta = np.array([0.1, 0.2]).reshape(1, 1, 2)
    M, N = affine.segment_map(K, V, eta, chunk=2)
    A = 0.1 * 4.0 + 0.2 * 1.0
    Bc = 0.1 * 2.0 * 0.5 + 0.2 * (-1.0) * 3.0
    assert abs(M[0, 0, 0, 0] - (1 - A)) < 1e-15 and abs(N[0, 0, 0, 0] - Bc) < 1e-15
