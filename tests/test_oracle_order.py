"""Oracle pins for the space-filling (Z-order) token order.

AFFMAE notes, "Limitations": the lookup table and the gathers are bandwidth-bound and
space-filling curves are suggested to keep neighbouring tokens close in memory.  The oracle
orders tokens by the Morton code of their cell (column bits at even, row bits at odd
positions), ties by id.  Pinned by a hand-derived 4 x 4 fixture, by an independent recursive
quadrant traversal (top-left, top-right, bottom-left, bottom-right) on square and
rectangular grids, and by ties, clamping and permutation properties.
"""
import numpy as np
import pytest

import oracle
from tests import golden


def _grid_tokens(H, W):
    r, c = np.divmod(np.arange(H * W), W)
    return np.stack([c + 0.5, r + 0.5], axis=1).astype(np.float32)


def _quadrant_order(r0, c0, size, H, W, out):
    """Cells of the square [r0, r0+size) x [c0, c0+size) inside H x W, Z order."""
    if r0 >= H or c0 >= W:
        return
    if size == 1:
        out.append(r0 * W + c0)
        return
    h = size // 2
    for dr, dc in ((0, 0), (0, h), (h, 0), (h, h)):
        _quadrant_order(r0 + dr, c0 + dc, h, H, W, out)


def test_golden_4x4():
    g = golden.read("zorder_4x4.txt")
    H, W = int(g["grid"][0]), int(g["grid"][1])
    perm = oracle.token_order(_grid_tokens(H, W)[None], H, W)[0]
    assert perm.tolist() == [int(v) for v in g["order"][0]]


@pytest.mark.parametrize("H,W", [(8, 8), (16, 16), (8, 32), (32, 8), (13, 21), (64, 64)])
def test_matches_recursive_quadrants(H, W):
    size = 1
    while size < max(H, W):
        size *= 2
    ref = []
    _quadrant_order(0, 0, size, H, W, ref)
    perm = oracle.token_order(_grid_tokens(H, W)[None], H, W)[0]
    assert perm.tolist() == ref


def test_ties_by_id_clamping_and_permutation():
    rng = np.random.default_rng(3)
    N = 500
    xy = rng.uniform(-3.0, 19.0, size=(2, N, 2)).astype(np.float32)   # some off the grid
    xy[0, 10:20] = xy[0, 5]                                           # one crowded cell
    perm = oracle.token_order(xy, 16, 16)
    for b in range(2):
        assert sorted(perm[b].tolist()) == list(range(N))
        cy = np.clip(np.floor(xy[b, :, 1]), 0, 15).astype(int)
        cx = np.clip(np.floor(xy[b, :, 0]), 0, 15).astype(int)
        ref = []
        _quadrant_order(0, 0, 16, 16, 16, ref)
        rank = np.empty(256, dtype=int)
        rank[np.array(ref)] = np.arange(256)
        key = rank[cy * 16 + cx] * N + np.arange(N)       # cell's Z rank, then id
        assert perm[b].tolist() == np.argsort(key, kind="stable").tolist()
