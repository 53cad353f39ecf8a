"""Pins of the oracle's local cluster attention, forward and backward (CPU only).

Source: AFFMAE notes, Method "Overall Architecture" (Local Cluster Attention
over local balanced clusters); arXiv abstract page (Flash-style cluster
attention kernels).  Reading: per token, softmax over its cluster's
neighbourhood of scale*<q,k> + a_h dx + b_h dy - c_h (dx^2 + dy^2) with
dx = x_key - x_query.

Pins, each independent of the oracle's own code:
* neighbourhood = every token (G <= R) equals dense softmax attention computed
  by torch's scaled_dot_product_attention in fp64;
* closed forms: q = 0 and no bias gives the neighbourhood mean; two tokens give
  the logistic weights;
* derivative identities: d lse / d a_h = E_P[dx], d lse / d b_h = E_P[dy],
  d lse / d c_h = -E_P[dx^2 + dy^2], d lse / d scale = E_P[<q, k>], where the
  expectations come from the oracle's own output with V set to coordinates or
  keys -- a wrong sign, a swapped coefficient or a dropped term breaks them;
* permutation equivariance of cluster -> neighbours -> attention;
* backward: central finite differences of L = <dO, O> on the oracle itself.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from off_grid_cluster_b200 import synth


def _setup(N, H=2, D=32, seed=5, spread=6.0, C=8, M=48, bias_scale=1.0):
    rng = np.random.default_rng(seed)
    xy = rng.uniform(0, spread, size=(1, N, 2)).astype(np.float32)
    q = rng.standard_normal((1, N, H, D))
    k = rng.standard_normal((1, N, H, D))
    v = rng.standard_normal((1, N, H, D))
    bias = np.stack([rng.uniform(-.1, .1, H), rng.uniform(-.1, .1, H),
                     rng.uniform(0, .1, H)], axis=1) * bias_scale
    cl = oracle.cluster(xy, C)
    nb = oracle.neighbors(xy, cl, M)
    return xy, q, k, v, bias, cl, nb


@pytest.mark.parametrize("N", [1, 2, 9, 45, 48])
def test_dense_reduction_matches_sdpa(N):
    xy, q, k, v, bias, cl, nb = _setup(N, H=3)
    scale = 1 / math.sqrt(32)
    o, lse = oracle.attn_fwd(q, k, v, xy, cl, nb, bias, scale)
    x = torch.tensor(xy[0, :, 0], dtype=torch.float64)
    y = torch.tensor(xy[0, :, 1], dtype=torch.float64)
    dx = x[None, :] - x[:, None]
    dy = y[None, :] - y[:, None]
    for h in range(3):
        a, b, c = (float(t) for t in bias[h])
        mask = a * dx + b * dy - c * (dx * dx + dy * dy)
        qt = torch.tensor(q[0, :, h])[None, None]
        kt = torch.tensor(k[0, :, h])[None, None]
        vt = torch.tensor(v[0, :, h])[None, None]
        ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask,
                                                               scale=scale)[0, 0]
        np.testing.assert_allclose(o[0, :, h], ref.numpy(), rtol=1e-12, atol=1e-12)
        logits = scale * (qt[0, 0] @ kt[0, 0].T) + mask
        np.testing.assert_allclose(lse[0, :, h], torch.logsumexp(logits, 1).numpy(),
                                   rtol=1e-12, atol=1e-12)


def test_zero_query_no_bias_is_neighbourhood_mean():
    xy, q, k, v, bias, cl, nb = _setup(300, H=2)
    o, lse = oracle.attn_fwd(np.zeros_like(q), k, v, xy, cl, nb, np.zeros_like(bias), 0.17)
    G = cl.shape[1]
    for g in range(G):
        keys = nb[0, g][nb[0, g] >= 0]
        for i in cl[0, g][cl[0, g] >= 0]:
            np.testing.assert_allclose(o[0, i], v[0, keys].mean(axis=0), rtol=1e-12, atol=1e-13)
            np.testing.assert_allclose(lse[0, i], math.log(keys.size), rtol=1e-13)


def test_two_tokens_logistic_and_sign_convention():
    xy = np.array([[[1.25, 2.0], [3.75, 2.5]]], dtype=np.float32)
    D = 32
    q = np.zeros((1, 2, 1, D)); k = np.zeros((1, 2, 1, D)); v = np.zeros((1, 2, 1, D))
    q[0, 0, 0, 0] = 2.0
    k[0, 0, 0, 0] = 1.0            # s_00 = scale * 2, s_01 = bias only
    v[0, 0, 0, 0] = 1.0
    v[0, 1, 0, 1] = 1.0
    a, b, c, scale = 0.3, -0.2, 0.05, 0.5
    bias = np.array([[a, b, c]])
    cl = oracle.cluster(xy, 8)
    nb = oracle.neighbors(xy, cl, 48)
    o, lse = oracle.attn_fwd(q, k, v, xy, cl, nb, bias, scale)
    dx, dy = 3.75 - 1.25, 2.5 - 2.0          # key 1 minus query 0
    s0 = scale * 2.0
    s1 = a * dx + b * dy - c * (dx * dx + dy * dy)
    w0 = 1.0 / (1.0 + math.exp(s1 - s0))
    assert o[0, 0, 0, 0] == pytest.approx(w0, rel=1e-14)
    assert o[0, 0, 0, 1] == pytest.approx(1 - w0, rel=1e-14)
    assert lse[0, 0, 0] == pytest.approx(s0 + math.log1p(math.exp(s1 - s0)), rel=1e-14)


def test_lse_derivative_identities():
    xy, q, k, v, bias, cl, nb = _setup(120, H=2, seed=11)
    scale = 0.2
    N, H = 120, 2
    x = xy[0, :, 0].astype(np.float64)
    y = xy[0, :, 1].astype(np.float64)
    # V carrying (x, y, x^2, y^2) of the key in its first four channels
    vc = np.zeros_like(v)
    for h in range(H):
        vc[0, :, h, 0], vc[0, :, h, 1] = x, y
        vc[0, :, h, 2], vc[0, :, h, 3] = x * x, y * y
    oc, _ = oracle.attn_fwd(q, k, vc, xy, cl, nb, bias, scale)
    ok, _ = oracle.attn_fwd(q, k, k, xy, cl, nb, bias, scale)    # V = K
    Ex, Ey, Ex2, Ey2 = (oc[0, :, :, j] for j in range(4))
    xi, yi = x[:, None], y[:, None]
    want = {
        0: Ex - xi,
        1: Ey - yi,
        2: -((Ex2 - 2 * xi * Ex + xi * xi) + (Ey2 - 2 * yi * Ey + yi * yi)),
    }
    eps = 1e-6
    for h in range(H):
        for j in range(3):
            bp, bm = bias.copy(), bias.copy()
            bp[h, j] += eps
            bm[h, j] -= eps
            lp = oracle.attn_fwd(q, k, v, xy, cl, nb, bp, scale)[1]
            lm = oracle.attn_fwd(q, k, v, xy, cl, nb, bm, scale)[1]
            fd = (lp[0, :, h] - lm[0, :, h]) / (2 * eps)
            np.testing.assert_allclose(fd, want[j][:, h], rtol=1e-6, atol=1e-7)
    lp = oracle.attn_fwd(q, k, v, xy, cl, nb, bias, scale + eps)[1]
    lm = oracle.attn_fwd(q, k, v, xy, cl, nb, bias, scale - eps)[1]
    fd = (lp[0] - lm[0]) / (2 * eps)
    want_s = np.einsum("nhd,nhd->nh", q[0], ok[0])
    np.testing.assert_allclose(fd, want_s, rtol=1e-6, atol=1e-6)


def test_permutation_equivariance():
    a = synth.attn_tiny()
    cl = oracle.cluster(a.coords)
    nb = oracle.neighbors(a.coords, cl)
    o, lse = oracle.attn_fwd(a.q, a.k, a.v, a.coords, cl, nb, a.bias, a.scale)
    perm = np.random.default_rng(3).permutation(a.N)
    xy2 = a.coords[:, perm]
    cl2 = oracle.cluster(xy2)
    nb2 = oracle.neighbors(xy2, cl2)
    o2, lse2 = oracle.attn_fwd(a.q[:, perm], a.k[:, perm], a.v[:, perm], xy2, cl2, nb2,
                               a.bias, a.scale)
    np.testing.assert_allclose(o2, o[:, perm], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse2, lse[:, perm], rtol=1e-12, atol=1e-12)
    # the clustering itself is equivariant: same token sets
    sets = {frozenset(r[r >= 0]) for r in cl[0]}
    sets2 = {frozenset(perm[r[r >= 0]]) for r in cl2[0]}
    assert sets == sets2


def _loss(q, k, v, xy, cl, nb, bias, scale, dO):
    o, _ = oracle.attn_fwd(q, k, v, xy, cl, nb, bias, scale)
    return float((o * dO).sum())


@pytest.mark.parametrize("N", [37, 130])
def test_backward_finite_differences(N):
    xy, q, k, v, bias, cl, nb = _setup(N, H=2, seed=N)
    scale = 1 / math.sqrt(32)
    dO = np.random.default_rng(N + 1).standard_normal(q.shape)
    dq, dk, dv, db = oracle.attn_bwd(q, k, v, xy, cl, nb, bias, scale, dO)
    rng = np.random.default_rng(7)
    eps = 1e-6
    for name, t, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for _ in range(40):
            idx = tuple(int(rng.integers(0, s)) for s in t.shape)
            tp, tm = t.copy(), t.copy()
            tp[idx] += eps
            tm[idx] -= eps
            args = {"q": q, "k": k, "v": v}
            args[name] = tp
            lp = _loss(args["q"], args["k"], args["v"], xy, cl, nb, bias, scale, dO)
            args[name] = tm
            lm = _loss(args["q"], args["k"], args["v"], xy, cl, nb, bias, scale, dO)
            fd = (lp - lm) / (2 * eps)
            assert g[idx] == pytest.approx(fd, rel=1e-5, abs=1e-7), (name, idx)
    for h in range(2):
        for j in range(3):
            bp, bm = bias.copy(), bias.copy()
            bp[h, j] += eps
            bm[h, j] -= eps
            fd = (_loss(q, k, v, xy, cl, nb, bp, scale, dO)
                  - _loss(q, k, v, xy, cl, nb, bm, scale, dO)) / (2 * eps)
            assert db[h, j] == pytest.approx(fd, rel=1e-5, abs=1e-7), (h, j)


def test_backward_batch_sums_bias_gradient():
    xy, q, k, v, bias, cl, nb = _setup(60, H=2, seed=3)
    xy2, q2, k2, v2, _, cl2, nb2 = _setup(60, H=2, seed=4)
    dO = np.random.default_rng(0).standard_normal((2,) + q.shape[1:])
    cat = lambda a_, b_: np.concatenate([a_, b_])
    _, _, _, db = oracle.attn_bwd(cat(q, q2), cat(k, k2), cat(v, v2), cat(xy, xy2),
                                  cat(cl, cl2), cat(nb, nb2), bias, 0.3, dO)
    _, _, _, d1 = oracle.attn_bwd(q, k, v, xy, cl, nb, bias, 0.3, dO[:1])
    _, _, _, d2 = oracle.attn_bwd(q2, k2, v2, xy2, cl2, nb2, bias, 0.3, dO[1:])
    np.testing.assert_allclose(db, d1 + d2, rtol=1e-13, atol=1e-15)
