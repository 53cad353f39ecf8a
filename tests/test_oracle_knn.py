"""Pins of the oracle's KNN lookup table and distance-softmax gather (CPU only).

Sources: AFFMAE notes, "Key Designs" 2 (the decoder gathers the K nearest
visible tokens around q = r + Delta with weights w_i = softmax_i(-p d_i), an
exponential distance kernel described as a stable softmax with a temperature)
and "Key Designs" 3 (an H x W x K table of each grid cell's K nearest visible
tokens; the continuous query is quantised to the nearest cell).

Pins, each independent of the oracle's own code:
* the table equals scipy's KD-tree K-nearest search from the cell centres;
* p -> infinity gives the nearest token's feature, p = 0 the plain mean,
  K = 1 a copy, constant features come back unchanged (weights sum to one);
* queries outside the grid use the border cell (K = 1 copy);
* with queries on cell centres the gather is the softmax over the KD-tree's
  exact neighbours and distances;
* backward: central finite differences of L = <dOut, out> on the oracle.
"""
import numpy as np
import pytest
from scipy.spatial import cKDTree

import oracle
from off_grid_cluster_b200 import synth


def _centres(GH, GW):
    r, c = np.divmod(np.arange(GH * GW), GW)
    return np.stack([c + 0.5, r + 0.5], axis=1)


@pytest.mark.parametrize("N,GH,GW,K", [(50, 8, 8, 8), (131, 64, 64, 8), (2048, 64, 64, 8),
                                       (300, 16, 24, 5), (20, 10, 10, 1)])
def test_table_matches_kdtree(N, GH, GW, K):
    if N == 2048:
        xy = synth.stage1_coords(synth.WORKLOAD_ID["stage1"], 1)
    else:
        xy = synth.uniform(N * 31 + K, 2 * N, 0.0, float(max(GH, GW))).reshape(N, 2)
        xy = xy.astype(np.float32)
    table = oracle.knn_table(xy[None], GH, GW, K)[0]
    tree = cKDTree(xy.astype(np.float64))
    d, idx = tree.query(_centres(GH, GW), k=K)
    idx = idx.reshape(GH * GW, K)
    assert np.array_equal(table.reshape(GH * GW, K), idx)
    dd = np.sqrt(((xy[table.reshape(-1, K)].astype(np.float64)
                   - _centres(GH, GW)[:, None]) ** 2).sum(-1))
    assert np.all(np.diff(dd, axis=1) >= 0)


def test_table_fewer_tokens_than_k():
    xy = np.array([[3.2, 1.1], [0.4, 0.6], [2.2, 2.9]], dtype=np.float32)
    table = oracle.knn_table(xy[None], 4, 4, 5)[0]
    tree = cKDTree(xy.astype(np.float64))
    _, idx = tree.query(_centres(4, 4), k=3)
    assert np.array_equal(table[..., :3].reshape(16, 3), idx)
    assert np.all(table[..., 3:] == -1)


def test_table_ties_by_id():
    # two tokens at the same point: the lower id comes first
    xy = np.array([[1.5, 1.5], [1.5, 1.5], [0.2, 0.2]], dtype=np.float32)
    table = oracle.knn_table(xy[None], 2, 2, 3)[0]
    assert list(table[1, 1]) == [0, 1, 2]


def _problem(N=200, d=64, Q=300, K=8, GH=16, GW=16, seed=0):
    rng = np.random.default_rng(seed)
    xy = rng.uniform(0, GW, size=(1, N, 2)).astype(np.float32)
    feats = rng.standard_normal((1, N, d))
    q = (rng.uniform(0, GW, size=(1, Q, 2))).astype(np.float32)
    p = rng.uniform(0.5, 4.0, size=d // 32)
    table = oracle.knn_table(xy, GH, GW, K)
    return xy, feats, q, p, table


def _dists(q, xy, rows):
    return np.sqrt(((q[:, None, :].astype(np.float64)
                     - xy[rows].astype(np.float64)) ** 2).sum(-1))


def _rows(q, table, GH, GW):
    cy = np.clip(np.floor(q[:, 1]), 0, GH - 1).astype(int)
    cx = np.clip(np.floor(q[:, 0]), 0, GW - 1).astype(int)
    return table[cy, cx]


def test_limits_of_temperature():
    xy, feats, q, p, table = _problem()
    rows = _rows(q[0], table[0], 16, 16)
    d = _dists(q[0], xy[0], rows)
    # p = 0: plain mean of the K features
    out = oracle.knn_fwd(q, feats, xy, table, np.zeros_like(p))[0]
    np.testing.assert_allclose(out, feats[0][rows].mean(axis=1), rtol=1e-12, atol=1e-12)
    # p large: the nearest of the K (clear gaps only)
    out = oracle.knn_fwd(q, feats, xy, table, np.full_like(p, 1e4))[0]
    ds = np.sort(d, axis=1)
    clear = (ds[:, 1] - ds[:, 0]) > 0.02
    near = rows[np.arange(rows.shape[0]), np.argmin(d, axis=1)]
    np.testing.assert_allclose(out[clear], feats[0][near][clear], rtol=1e-9, atol=1e-9)
    # constant features stay constant: the weights sum to one
    out = oracle.knn_fwd(q, np.ones_like(feats), xy, table, p)[0]
    np.testing.assert_allclose(out, 1.0, rtol=1e-14)


def test_k1_is_copy_and_border_clamp():
    xy, feats, _, p, _ = _problem()
    table1 = oracle.knn_table(xy, 16, 16, 1)
    q = np.array([[[-5.0, 100.0], [40.0, -3.0], [7.3, 8.9], [np.nan, 2.5]]], dtype=np.float32)
    out = oracle.knn_fwd(q, feats, xy, table1, p)[0]
    want_cells = [(15, 0), (0, 15), (8, 7), (2, 0)]
    for i, (r, c) in enumerate(want_cells):
        if i == 3:
            continue          # NaN distance: only the cell choice is defined
        np.testing.assert_array_equal(out[i], feats[0, table1[0, r, c, 0]])


def test_cell_centre_queries_match_exact_knn():
    xy, feats, _, p, table = _problem(N=400, d=96, seed=4)
    cen = _centres(16, 16).astype(np.float32)
    out = oracle.knn_fwd(cen[None], feats, xy, table, p)[0]
    d, idx = cKDTree(xy[0].astype(np.float64)).query(cen.astype(np.float64), k=8)
    for h in range(3):
        z = -p[h] * d
        w = np.exp(z - z.max(axis=1, keepdims=True))
        w /= w.sum(axis=1, keepdims=True)
        ref = np.einsum("qk,qkc->qc", w, feats[0][idx][:, :, 32 * h:32 * h + 32])
        np.testing.assert_allclose(out[:, 32 * h:32 * h + 32], ref, rtol=1e-11, atol=1e-12)


def test_decoder_workload_runs():
    kb = synth.knn_decoder(B=1)[3]
    table = oracle.knn_table(kb.coords, kb.GH, kb.GW, kb.K)
    out = oracle.knn_fwd(kb.queries, kb.feats, kb.coords, table, kb.p)
    assert out.shape == (1, 4096, 768) and np.isfinite(out).all()


def _loss(q, feats, xy, table, p, dout):
    return float((oracle.knn_fwd(q, feats, xy, table, p) * dout).sum())


def test_backward_finite_differences():
    xy, feats, q, p, table = _problem(N=150, d=64, Q=120, seed=9)
    dout = np.random.default_rng(2).standard_normal((1, 120, 64))
    dF, dq, dp = oracle.knn_bwd(q, feats, xy, table, p, dout)
    rng = np.random.default_rng(1)
    eps = 1e-6
    for _ in range(60):
        idx = (0, int(rng.integers(0, 150)), int(rng.integers(0, 64)))
        fp, fm = feats.copy(), feats.copy()
        fp[idx] += eps
        fm[idx] -= eps
        fd = (_loss(q, fp, xy, table, p, dout) - _loss(q, fm, xy, table, p, dout)) / (2 * eps)
        assert dF[idx] == pytest.approx(fd, rel=1e-6, abs=1e-8)
    for h in range(2):
        pp, pm = p.copy(), p.copy()
        pp[h] += eps
        pm[h] -= eps
        fd = (_loss(q, feats, xy, table, pp, dout) - _loss(q, feats, xy, table, pm, dout)) / (2 * eps)
        assert dp[h] == pytest.approx(fd, rel=1e-6, abs=1e-8)
    # queries are fp32: step by an exactly representable 2^-12, away from cell edges
    e = 2.0 ** -12
    checked = 0
    for i in range(120):
        for j in range(2):
            v = float(q[0, i, j])
            if abs(v - np.round(v)) < 4 * e:
                continue
            qp, qm = q.copy(), q.copy()
            qp[0, i, j] = np.float32(v + e)
            qm[0, i, j] = np.float32(v - e)
            fd = (_loss(qp, feats, xy, table, p, dout) - _loss(qm, feats, xy, table, p, dout)) / (2 * e)
            assert dq[0, i, j] == pytest.approx(fd, rel=2e-4, abs=2e-5), (i, j)
            checked += 1
    assert checked > 200
