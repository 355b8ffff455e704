"""The host-buffer pipeline's slicing of the (batch, head) grid (no GPU):
whole batch rows while there are at least as many rows as slices (contiguous,
covering the batch once, sizes within one row), else runs of heads within one
row each; either way every (b, h) pair lies in exactly one group."""
import pytest

from test_sequence_layers_layer_b200 import hostio


@pytest.mark.parametrize("B,H,slices", [(8, 3, 4), (5, 2, 3), (2, 8, 4), (7, 1, 1), (1, 1, 1),
                                        (9, 4, 0), (16, 2, 5), (4, 8, 16), (3, 3, 7), (1, 8, 8),
                                        (2, 3, 64)])
def test_bounds(B, H, slices):
    bounds = hostio._bounds(B, H, slices)
    seen = [(b, h) for b0, b1, h0, h1 in bounds for b in range(b0, b1) for h in range(h0, h1)]
    assert sorted(seen) == [(b, h) for b in range(B) for h in range(H)]
    if slices <= B:
        assert all(h0 == 0 and h1 == H for _, _, h0, h1 in bounds)
        assert bounds[0][0] == 0 and bounds[-1][1] == B
        assert all(a[1] == b[0] for a, b in zip(bounds, bounds[1:]))
        sizes = [b1 - b0 for b0, b1, _, _ in bounds]
        assert min(sizes) >= 1 and max(sizes) - min(sizes) <= 1
        assert len(bounds) == max(1, slices)
    else:
        assert all(b1 == b0 + 1 and h1 > h0 for b0, b1, h0, h1 in bounds)
        per_row = min(H, -(-slices // B))
        assert len(bounds) == B * per_row
        sizes = [h1 - h0 for _, _, h0, h1 in bounds]
        assert max(sizes) - min(sizes) <= 1
