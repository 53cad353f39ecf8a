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
* backward: central finite differences of L = <dOut, out> on the oracle;
* a token repeated in a table row takes the weights of all its slots (closed form).
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


# ------------------------------------------------------------------ inverse-power kernel
# AFFMAE notes, "Key Designs" 2: the original AFF weighting w_i proportional to d_i^-p,
# which the notes replace by the exponential kernel because it overflows at short range and
# underflows at long range in mixed precision.

INV = oracle.KNN_INVPOW


def _one_row_table(GH, GW, ids):
    t = np.empty((1, GH, GW, len(ids)), dtype=np.int32)
    t[...] = np.asarray(ids, dtype=np.int32)
    return t


def test_invpow_two_neighbours_closed_form():
    # w_1 = 1 / (1 + (d1/d2)^p), w_2 = 1 - w_1 for two tokens at distances d1, d2
    xy = np.array([[[3.0, 2.0], [2.0, 6.0]]], dtype=np.float32)
    q = np.array([[[2.0, 2.5]]], dtype=np.float32)
    feats = np.random.default_rng(3).standard_normal((1, 2, 32))
    table = _one_row_table(8, 8, [0, 1])
    d1, d2 = np.hypot(1.0, 0.5), np.hypot(0.0, 3.5)
    for p in (0.5, 1.0, 2.5, 7.0):
        out = oracle.knn_fwd(q, feats, xy, table, np.array([p]), kind=INV)[0, 0]
        w1 = 1.0 / (1.0 + (d1 / d2) ** p)
        np.testing.assert_allclose(out, w1 * feats[0, 0] + (1 - w1) * feats[0, 1], rtol=1e-12)


def test_invpow_scale_invariance_and_exp_is_not():
    # d^-p weights only see distance ratios: scaling every token's offset from the query by
    # s leaves them unchanged; softmax(-p d) weights change
    rng = np.random.default_rng(5)
    K = 6
    off = rng.uniform(-1.5, 1.5, size=(K, 2))
    q = np.array([[[20.5, 20.5]]], dtype=np.float32)
    feats = rng.standard_normal((1, K, 64))
    table = _one_row_table(32, 32, list(range(K)))
    p = np.array([1.3, 3.0])
    outs = {}
    for kind in (oracle.KNN_EXP, INV):
        for s in (1.0, 4.0):
            xy = (q[0, 0].astype(np.float64) + s * off).astype(np.float32)[None]
            outs[kind, s] = oracle.knn_fwd(q, feats, xy, table, p, kind=kind)[0, 0]
    np.testing.assert_allclose(outs[INV, 1.0], outs[INV, 4.0], rtol=1e-6, atol=1e-6)
    assert np.abs(outs[oracle.KNN_EXP, 1.0] - outs[oracle.KNN_EXP, 4.0]).max() > 1e-2


def test_invpow_query_on_tokens_and_zero_temperature():
    # the limit d -> 0: a query on a token takes that token's features (shared equally by
    # coincident tokens); p = 0 gives the plain mean
    xy = np.array([[[1.25, 1.75], [1.25, 1.75], [3.0, 0.5], [0.1, 3.9]]], dtype=np.float32)
    feats = np.random.default_rng(7).standard_normal((1, 4, 32))
    table = _one_row_table(4, 4, [0, 1, 2, 3])
    q = np.array([[[1.25, 1.75], [3.0, 0.5]]], dtype=np.float32)
    out = oracle.knn_fwd(q, feats, xy, table, np.array([2.0]), kind=INV)[0]
    np.testing.assert_allclose(out[0], 0.5 * (feats[0, 0] + feats[0, 1]), rtol=1e-12)
    np.testing.assert_allclose(out[1], feats[0, 2], rtol=1e-12)
    out = oracle.knn_fwd(q, feats, xy, table, np.array([0.0]), kind=INV)[0]
    np.testing.assert_allclose(out[0], feats[0].mean(axis=0), rtol=1e-12)
    dF, dq, dp = oracle.knn_bwd(q, feats, xy, table, np.array([2.0]),
                                np.ones((1, 2, 32)), kind=INV)
    assert np.isfinite(dq).all() and np.isfinite(dp).all() and np.isfinite(dF).all()


def _loss_inv(q, feats, xy, table, p, dout):
    return float((oracle.knn_fwd(q, feats, xy, table, p, kind=INV) * dout).sum())


def test_invpow_backward_finite_differences():
    xy, feats, q, p, table = _problem(N=150, d=64, Q=120, seed=11)
    dout = np.random.default_rng(4).standard_normal((1, 120, 64))
    dF, dq, dp = oracle.knn_bwd(q, feats, xy, table, p, dout, kind=INV)
    rng = np.random.default_rng(8)
    eps = 1e-6
    for _ in range(40):
        idx = (0, int(rng.integers(0, 150)), int(rng.integers(0, 64)))
        fp, fm = feats.copy(), feats.copy()
        fp[idx] += eps
        fm[idx] -= eps
        fd = (_loss_inv(q, fp, xy, table, p, dout) - _loss_inv(q, fm, xy, table, p, dout)) / (2 * eps)
        assert dF[idx] == pytest.approx(fd, rel=1e-6, abs=1e-8)
    for h in range(2):
        pp, pm = p.copy(), p.copy()
        pp[h] += eps
        pm[h] -= eps
        fd = (_loss_inv(q, feats, xy, table, pp, dout) - _loss_inv(q, feats, xy, table, pm, dout)) / (2 * eps)
        assert dp[h] == pytest.approx(fd, rel=1e-6, abs=1e-8)
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
            fd = (_loss_inv(qp, feats, xy, table, p, dout) - _loss_inv(qm, feats, xy, table, p, dout)) / (2 * e)
            assert dq[0, i, j] == pytest.approx(fd, rel=5e-4, abs=5e-5), (i, j)
            checked += 1
    assert checked > 200


def test_invpow_half_precision_range_versus_exp_kernel():
    # the reason the notes give for the exponential kernel: evaluated directly in half
    # precision, d^-p overflows for close tokens and underflows for far ones, so the
    # normalised weights become nan or lose every term; softmax(-p d) with the minimum
    # subtracted stays in [0, 1].  (The oracle and the CUDA path evaluate the inverse power
    # as (d_min / d)^p, which stays in [0, 1] as well.)
    p = np.float16(4.0)
    near = np.array([0.05, 0.3, 0.6], dtype=np.float16)        # cell units
    far = np.array([40.0, 55.0, 60.0], dtype=np.float16)
    with np.errstate(over="ignore", divide="ignore", invalid="ignore"):
        w_near = near ** -p                                        # fp16: 0.05^-4 = 160000
        assert np.isinf(w_near[0])
        assert np.isnan(w_near / w_near.sum()).any()
        w_far = far ** -np.float16(8.0)                            # ~1e-13: below fp16 range
        assert (w_far == 0).all()
        bf_near = (near.astype(np.float32) ** -np.float32(30.0))   # bf16 range = fp32 range
        assert np.isinf(bf_near[0])
    for dist in (near, far):
        z = -p * (dist - dist.min())                                # exponential kernel
        w = np.exp(z.astype(np.float16))
        assert np.isfinite(w).all() and w.max() == np.float16(1.0)
        r = (dist.min() / dist) ** p                                # the ratio form
        assert np.isfinite(r).all() and r.max() == np.float16(1.0)


def test_repeated_token_in_a_row_counts_once_per_slot():
    """Table rows may repeat a token id (entries in [-1, N)); the softmax runs over the row's
    slots, so a token in two slots takes both slots' weights, and an empty slot (-1) none:
    closed form for the row [0, 0, 1, -1] at distances d0, d0, d1."""
    xy = np.array([[[3.0, 2.0], [2.0, 6.0]]], dtype=np.float32)
    q = np.array([[[2.0, 2.5]]], dtype=np.float32)
    rng = np.random.default_rng(11)
    feats = rng.standard_normal((1, 2, 32))
    dout = rng.standard_normal((1, 1, 32))
    table = _one_row_table(8, 8, [0, 0, 1, -1])
    d0, d1 = np.hypot(1.0, 0.5), np.hypot(0.0, 3.5)
    for p in (0.0, 0.7, 3.0):
        e0, e1 = np.exp(-p * d0), np.exp(-p * d1)
        w0, w1 = 2 * e0 / (2 * e0 + e1), e1 / (2 * e0 + e1)
        out = oracle.knn_fwd(q, feats, xy, table, np.array([p]))[0, 0]
        np.testing.assert_allclose(out, w0 * feats[0, 0] + w1 * feats[0, 1], rtol=1e-12)
        dF, _, _ = oracle.knn_bwd(q, feats, xy, table, np.array([p]), dout)
        np.testing.assert_allclose(dF[0, 0], w0 * dout[0, 0], rtol=1e-12)
        np.testing.assert_allclose(dF[0, 1], w1 * dout[0, 0], rtol=1e-12)
