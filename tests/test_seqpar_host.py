"""The sequence-parallel drivers reject inputs they cannot split before any
library call (CPU tensors here: nothing reaches the GPU)."""
import pytest
import torch

from test_sequence_layers_layer_b200 import seqpar


def _x(B=1, H=2, T=512, d=64):
    Q = torch.zeros(B, H, T, d, dtype=torch.bfloat16)
    return Q, Q.clone(), Q.clone(), torch.zeros(B, H, T), torch.zeros(H, d, d)


@pytest.mark.parametrize("kw,msg", [
    (dict(nseg=3), "equal segments"),           # 512 tokens do not split in 3
    (dict(nseg=8), "whole number"),             # 64-token segments, chunk 128
    (dict(nseg=0), "equal segments"),
])
def test_segmented_rejects_bad_splits(kw, msg):
    Q, K, V, eta, W0 = _x()
    with pytest.raises(ValueError, match=msg):
        seqpar.chunk_fwd_segmented(Q, K, V, eta, W0, chunk=128, **kw)


def test_segmented_rejects_bad_tensors():
    Q, K, V, eta, W0 = _x()
    with pytest.raises(ValueError, match="one shape"):
        seqpar.chunk_fwd_segmented(Q, K[:, :, :256], V, eta, W0, chunk=128, nseg=2)
    with pytest.raises(ValueError, match="eta"):
        seqpar.chunk_fwd_segmented(Q, K, V, eta[:, :1], W0, chunk=128, nseg=2)
    with pytest.raises(ValueError, match="contiguous"):
        seqpar.chunk_fwd_segmented(Q, K.transpose(2, 3).contiguous().transpose(2, 3), V, eta, W0,
                                   chunk=128, nseg=2)
    Q, K, V, eta, W0 = _x(d=32)
    with pytest.raises(ValueError, match="d = 64 and 128"):
        seqpar.linear_fwd_segmented(Q, K, V, eta, W0, b=16, nseg=2)
    Q, K, V, eta, W0 = _x()
    with pytest.raises(ValueError, match="whole number"):
        seqpar.linear_fwd_segmented(Q, K, V, eta, W0, b=48, nseg=2)
