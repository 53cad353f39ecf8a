"""Pins of the oracle's balanced clustering and neighbourhood table (CPU only).

The pages (AFFMAE notes, Method "Overall Architecture") say only that attention
runs over *local balanced clusters* of tokens with explicit 2D coordinates.  The
reading pinned here: recursive median bisection into clusters of exactly C slots
(padding only in the last cluster), and neighbourhoods of the R = M / C nearest
cluster centroids.  Pins: hand-derived goldens, and properties that fix the
output uniquely (partition, sizes, split separation by the stated key, leaf
order, k-nearest optimality) checked on the output rather than by re-running
the algorithm.
"""
import numpy as np
import pytest

import oracle
from off_grid_cluster_b200 import synth
from tests import golden


def _tree_nodes(G):
    """Internal nodes (c0, g, gl) of the fixed bisection tree over clusters [0, G)."""
    out, stack = [], [(0, G)]
    while stack:
        c0, g = stack.pop()
        if g == 1:
            continue
        gl = (g + 1) // 2
        out.append((c0, g, gl))
        stack.append((c0, gl))
        stack.append((c0 + gl, g - gl))
    return out


def check_clustering(xy, cl, C):
    """Assert every property that defines the recursive-median clustering."""
    N = xy.shape[0]
    G = (N + C - 1) // C
    assert cl.shape == (G, C)
    flat = cl.reshape(-1)
    valid = flat[flat >= 0]
    # partition of 0..N-1, padding only at the tail of the last cluster
    assert np.array_equal(np.sort(valid), np.arange(N))
    assert np.all(flat[:N] >= 0) and np.all(flat[N:] == -1)
    # leaves list ids ascending
    for g in range(G):
        ids = cl[g][cl[g] >= 0]
        assert np.all(np.diff(ids) > 0)
    # each internal node separates on its axis by the key (axis, other, id)
    x = xy[:, 0].astype(np.float64)
    y = xy[:, 1].astype(np.float64)
    for c0, g, gl in _tree_nodes(G):
        left = cl[c0:c0 + gl].reshape(-1)
        right = cl[c0 + gl:c0 + g].reshape(-1)
        left, right = left[left >= 0], right[right >= 0]
        allt = np.concatenate([left, right])
        ex = x[allt].max() - x[allt].min()
        ey = y[allt].max() - y[allt].min()
        a, b = (x, y) if ex >= ey else (y, x)
        assert left.size == gl * C
        kl = sorted(zip(a[left], b[left], left))
        kr = sorted(zip(a[right], b[right], right))
        assert kl[-1] < kr[0], (c0, g)


@pytest.mark.parametrize("name", ["cluster_grid8.txt", "cluster_grid4x16.txt",
                                  "cluster_line20.txt"])
def test_cluster_golden(name):
    gd = golden.read(name)
    rows, cols = (int(v) for v in gd["grid"])
    C = int(gd["C"][0])
    xy = golden.grid_coords(rows, cols)
    cl = oracle.cluster(xy, C)[0]
    assert np.array_equal(cl, np.array(gd["clusters"], dtype=np.int32))


def test_neighbors_golden():
    gd = golden.read("cluster_grid8.txt")
    xy = golden.grid_coords(8, 8)
    cl = oracle.cluster(xy, 8)
    nb = oracle.neighbors(xy, cl, 48)[0]
    want = np.array(gd["neighbour_clusters"], dtype=np.int64)
    for g in range(8):
        for r in range(6):
            assert np.array_equal(nb[g, r * 8:(r + 1) * 8], cl[0, want[g, r]])


@pytest.mark.parametrize("N", [1, 7, 8, 9, 31, 32, 33, 100, 517])
def test_cluster_properties_random(N):
    xy = synth.uniform(1234 + N, 2 * N, 0.0, 16.0).reshape(1, N, 2).astype(np.float32)
    for C in (1, 3, 8):
        cl = oracle.cluster(xy, C)[0]
        check_clustering(xy[0], cl, C)


def test_cluster_properties_workloads():
    a = synth.attn_tiny()
    check_clustering(a.coords[0], oracle.cluster(a.coords)[0], 8)
    xy = synth.stage1_coords(synth.WORKLOAD_ID["stage1"], 0)[None]
    check_clustering(xy[0], oracle.cluster(xy)[0], 8)
    for s, st in enumerate(synth.sweep_coords(B=1)):
        check_clustering(st[0], oracle.cluster(st)[0], 8)


def test_cluster_exact_ties_broken_by_id():
    # duplicated coordinates: the order falls through to the token id
    xy = np.zeros((1, 20, 2), dtype=np.float32)
    xy[0, :, 0] = np.repeat(np.arange(5), 4)
    cl = oracle.cluster(xy, 4)[0]
    check_clustering(xy[0], cl, 4)
    assert np.array_equal(cl.reshape(-1), np.arange(20))


def _centroids(xy, cl):
    out = []
    for row in cl:
        t = row[row >= 0]
        out.append(xy[t].astype(np.float64).mean(axis=0))
    return np.array(out)


def check_neighbors(xy, cl, nb, M):
    G, C = cl.shape
    R = M // C
    cen = _centroids(xy, cl)
    take = min(R, G)
    for g in range(G):
        blocks = []
        for r in range(R):
            blk = nb[g, r * C:(r + 1) * C]
            if r >= take:
                assert np.all(blk == -1)
                continue
            hits = [h for h in range(G) if np.array_equal(cl[h], blk)]
            assert len(hits) == 1
            blocks.append(hits[0])
        assert len(set(blocks)) == take
        d = ((cen - cen[g]) ** 2).sum(axis=1)
        chosen = d[blocks]
        assert np.all(np.diff(chosen) >= -1e-9)            # nearest first
        others = np.delete(d, blocks)
        if others.size:
            assert chosen.max() <= others.min() + 1e-9     # the R nearest
        assert blocks[0] == g or d[blocks[0]] <= 1e-12     # itself first


@pytest.mark.parametrize("N", [5, 48, 49, 200, 2048])
def test_neighbors_properties(N):
    if N == 2048:
        xy = synth.stage1_coords(synth.WORKLOAD_ID["stage1"], 3)[None]
    else:
        xy = synth.uniform(99 + N, 2 * N, 0.0, 12.0).reshape(1, N, 2).astype(np.float32)
    cl = oracle.cluster(xy, 8)
    for M in (8, 48, 64):
        nb = oracle.neighbors(xy, cl, M)
        check_neighbors(xy[0], cl[0], nb[0], M)


def test_stage_sizes_golden():
    gd = golden.read("stage_sizes.txt")
    want = [int(v) for v in gd["stages"]]
    assert synth.stage_sizes(int(gd["visible"][0]), 4, float(gd["retention"][0])) == want
    assert int(gd["visible"][0]) * 2 == int(gd["grid_tokens"][0])
    assert [int(v) for v in gd["dims"]] == list(synth.SWEEP_DIMS)
    assert [int(v) for v in gd["layers"]] == list(synth.SWEEP_LAYERS)
    st = synth.sweep_coords(B=1)
    assert [s.shape[1] for s in st] == want


def test_synth_bf16_and_masks():
    x = synth.normal_bf16(7, (1000,))
    bits = x.view(np.uint32)
    assert np.all(bits & 0xFFFF == 0)
    assert abs(x.mean()) < 0.1 and abs(x.std() - 1) < 0.1
    assert synth.noise_mask(3, 64, 64, 2048).size == 2048
    xy = synth.stage1_coords(2, 0)
    cells = synth.noise_mask(synth.stream_seed(2, 0, synth.TAG_MASK), 64, 64, 2048)
    assert np.array_equal(np.floor(xy[:, 0]) + 64 * np.floor(xy[:, 1]), cells)
