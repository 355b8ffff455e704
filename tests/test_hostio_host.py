"""The host-buffer pipeline's batch slicing (no GPU): the slices are
contiguous, cover the batch once, differ in size by at most one row, and
there are never more slices than batch rows."""
import pytest

from test_sequence_layers_layer_b200 import hostio


@pytest.mark.parametrize("B,slices", [(8, 4), (5, 3), (2, 4), (7, 1), (1, 1), (9, 0), (16, 5)])
def test_bounds(B, slices):
    bounds = hostio._bounds(B, slices)
    assert bounds[0][0] == 0 and bounds[-1][1] == B
    assert all(a[1] == b[0] for a, b in zip(bounds, bounds[1:]))
    sizes = [b1 - b0 for b0, b1 in bounds]
    assert min(sizes) >= 1 and max(sizes) - min(sizes) <= 1
    assert len(bounds) == max(1, min(slices, B))
