"""Oracle pins for token merging between stages.

AFFMAE notes, "Key Designs" 1 (adaptive off-grid token merging): a lightweight MLP scores
the tokens, the top-k are kept as anchors at the retention rate, and the others are merged
differentiably into their nearest anchor, fusing features and coordinates.  Pinned by an
independent numpy/scipy evaluation of the MLP, brute-force selection and assignment, closed
forms of the merge (equal scores give the mean, a lone anchor keeps its features, a common
score shift changes nothing) and central finite differences of every gradient.
"""
import math

import numpy as np
import pytest
from scipy.special import erf

import oracle
from off_grid_cluster_b200 import synth


def _mb(B=2, N=300, d=64, seed=0):
    rng = np.random.default_rng(seed)
    xy = rng.uniform(0, 20, size=(B, N, 2)).astype(np.float32)
    return synth.merge_batch(xy, d=d)


def test_scores_match_numpy():
    mb = _mb()
    z = np.einsum("bnd,dh->bnh", mb.feats.astype(np.float64), mb.w1.astype(np.float64)) + mb.b1
    g = 0.5 * z * (1 + erf(z / math.sqrt(2)))
    ref = g @ mb.w2.astype(np.float64) + mb.b2
    np.testing.assert_allclose(oracle.merge_scores(mb.feats, mb.w1, mb.b1, mb.w2, mb.b2), ref,
                               rtol=1e-12, atol=1e-12)


def test_selection_matches_brute_force():
    mb = _mb(N=400, seed=1)
    s = oracle.merge_scores(mb.feats, mb.w1, mb.b1, mb.w2, mb.b2)
    s[0, 10:20] = s[0, 9]                       # ties by id
    anchors, assign = oracle.merge_select(s, mb.coords, mb.k)
    for b in range(mb.B):
        top = sorted(range(mb.N), key=lambda i: (-s[b, i], i))[:mb.k]
        assert anchors[b].tolist() == sorted(top)
        axy = mb.coords[b][anchors[b]].astype(np.float64)
        d2 = ((mb.coords[b].astype(np.float64)[:, None, :] - axy[None]) ** 2).sum(-1)
        ref = np.argmin(d2, axis=1)             # first minimum: the lower anchor id
        ref[anchors[b]] = np.arange(mb.k)       # an anchor is its own group
        assert assign[b].tolist() == ref.tolist()


def test_merge_closed_forms():
    mb = _mb(B=1, N=200, seed=2)
    s = oracle.merge_scores(mb.feats, mb.w1, mb.b1, mb.w2, mb.b2)
    anchors, assign = oracle.merge_select(s, mb.coords, mb.k)
    f = mb.feats.astype(np.float64)
    # equal scores: plain means of the groups
    m, mxy = oracle.merge_fwd(mb.feats, mb.coords, np.zeros_like(s), mb.k, assign)
    for j in range(mb.k):
        grp = np.nonzero(assign[0] == j)[0]
        np.testing.assert_allclose(m[0, j], f[0, grp].mean(0), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(mxy[0, j], mb.coords[0, grp].astype(np.float64).mean(0),
                                   rtol=1e-12, atol=1e-12)
    # a lone anchor keeps its own features; a common shift of the scores changes nothing
    m1, _ = oracle.merge_fwd(mb.feats, mb.coords, s, mb.k, assign)
    m2, _ = oracle.merge_fwd(mb.feats, mb.coords, s + 7.5, mb.k, assign)
    np.testing.assert_allclose(m1, m2, rtol=1e-12, atol=1e-12)
    sizes = np.bincount(assign[0], minlength=mb.k)
    lone = np.nonzero(sizes == 1)[0]
    assert lone.size > 0
    np.testing.assert_allclose(m1[0, lone], f[0, anchors[0, lone]], rtol=1e-12, atol=1e-12)
    # softmax weights: the group's weights sum to one
    ones, _ = oracle.merge_fwd(np.ones_like(mb.feats), mb.coords, s, mb.k, assign)
    np.testing.assert_allclose(ones, 1.0, rtol=1e-12)


def _loss(mb, assign, feats=None, xy=None, w1=None, b1=None, w2=None, b2=None):
    feats = mb.feats if feats is None else feats
    xy = mb.coords if xy is None else xy
    s = oracle.merge_scores(feats, mb.w1 if w1 is None else w1, mb.b1 if b1 is None else b1,
                            mb.w2 if w2 is None else w2, mb.b2 if b2 is None else b2)
    m, mxy = oracle.merge_fwd(feats, xy, s, mb.k, assign)
    return float((m * mb.dmerged).sum() + (mxy * mb.dmcoords).sum())


def test_backward_finite_differences():
    mb = _mb(B=1, N=120, d=32, seed=3)
    s = oracle.merge_scores(mb.feats, mb.w1, mb.b1, mb.w2, mb.b2)
    _, assign = oracle.merge_select(s, mb.coords, mb.k)
    df, dxy, dw1, db1, dw2, db2 = oracle.merge_bwd(mb.feats, mb.coords, mb.w1, mb.b1, mb.w2,
                                                   mb.b2, mb.k, assign, mb.dmerged, mb.dmcoords)
    rng = np.random.default_rng(4)
    eps = 1e-6

    def fd(**kw):
        key, arr, idx = kw["key"], kw["arr"], kw["idx"]
        a_p, a_m = arr.astype(np.float64).copy(), arr.astype(np.float64).copy()
        a_p[idx] += eps
        a_m[idx] -= eps
        return (_loss(mb, assign, **{key: a_p}) - _loss(mb, assign, **{key: a_m})) / (2 * eps)

    for _ in range(20):
        idx = (0, int(rng.integers(0, 120)), int(rng.integers(0, 32)))
        assert df[idx] == pytest.approx(fd(key="feats", arr=mb.feats, idx=idx), rel=1e-5, abs=1e-7)
    for _ in range(10):
        idx = (int(rng.integers(0, 32)), int(rng.integers(0, mb.h)))
        assert dw1[idx] == pytest.approx(fd(key="w1", arr=mb.w1, idx=idx), rel=1e-5, abs=1e-7)
    for u in range(mb.h):
        assert db1[u] == pytest.approx(fd(key="b1", arr=mb.b1, idx=(u,)), rel=1e-5, abs=1e-7)
        assert dw2[u] == pytest.approx(fd(key="w2", arr=mb.w2, idx=(u,)), rel=1e-5, abs=1e-7)
    b2p = (_loss(mb, assign, b2=mb.b2 + eps) - _loss(mb, assign, b2=mb.b2 - eps)) / (2 * eps)
    assert db2 == pytest.approx(b2p, abs=1e-7)           # a common shift: zero
    # coordinates enter only through the merged coordinates
    e = 2.0 ** -12
    for _ in range(20):
        i, c = int(rng.integers(0, 120)), int(rng.integers(0, 2))
        xp, xm = mb.coords.copy(), mb.coords.copy()
        xp[0, i, c] += np.float32(e)
        xm[0, i, c] -= np.float32(e)
        ref = (_loss(mb, assign, xy=xp) - _loss(mb, assign, xy=xm)) / (2 * e)
        assert dxy[0, i, c] == pytest.approx(ref, rel=1e-5, abs=1e-6)


def test_extreme_retention_rates():
    """k = N: every token is its own anchor, so merging is the identity and the MLP gets no
    gradient (a one-token group's softmax weight is constant); k = 1: one group, the merge is
    the softmax-of-scores average of all tokens (numpy)."""
    rng = np.random.default_rng(9)
    xy = rng.uniform(0, 10, size=(1, 60, 2)).astype(np.float32)
    mb = synth.merge_batch(xy, d=32, ds=1.0)
    assert mb.k == 60
    s = oracle.merge_scores(mb.feats, mb.w1, mb.b1, mb.w2, mb.b2)
    anchors, assign = oracle.merge_select(s, mb.coords, mb.k)
    np.testing.assert_array_equal(anchors[0], np.arange(60))
    np.testing.assert_array_equal(assign[0], np.arange(60))
    m, mxy = oracle.merge_fwd(mb.feats, mb.coords, s, mb.k, assign)
    np.testing.assert_allclose(m[0], mb.feats[0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(mxy[0], mb.coords[0], rtol=0, atol=1e-12)
    dm = np.ones((1, 60, 32))
    df, dxy, dw1, db1, dw2, db2 = oracle.merge_bwd(mb.feats, mb.coords, mb.w1, mb.b1, mb.w2, mb.b2,
                                                   mb.k, assign, dm, np.ones((1, 60, 2)))
    np.testing.assert_allclose(df[0], 1.0, rtol=0, atol=1e-12)
    np.testing.assert_allclose(dxy[0], 1.0, rtol=0, atol=1e-12)
    for g in (dw1, db1, dw2):
        assert np.abs(g).max() <= 1e-12
    assert abs(db2) <= 1e-12

    one = synth.merge_batch(xy, d=32, ds=1.0 / 60.0)
    assert one.k == 1
    s1 = oracle.merge_scores(one.feats, one.w1, one.b1, one.w2, one.b2)
    _, as1 = oracle.merge_select(s1, one.coords, 1)
    assert np.all(as1 == 0)
    m1, mxy1 = oracle.merge_fwd(one.feats, one.coords, s1, 1, as1)
    w = np.exp(s1[0] - s1[0].max())
    w /= w.sum()
    np.testing.assert_allclose(m1[0, 0], w @ one.feats[0].astype(np.float64), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(mxy1[0, 0], w @ one.coords[0].astype(np.float64), rtol=1e-12, atol=1e-12)
