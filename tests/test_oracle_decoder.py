"""Pins of the oracle's decoder layer (AFFMAE notes, "Key Designs" 2, the point-wise
deformable cross-attention decoder: offset Delta = g(f), q = r + Delta, KNN distance-softmax
gather of an encoder stage at q, fused into the query feature).  Readings: g is linear, and
the gathered feature is projected by W_o and added: f_out = f + gather(q) W_o.

The gather itself is pinned in test_oracle_knn.py; here the offset head, the projection and
the chain rule of the whole layer are pinned by closed forms, a reduction to the gather, and
central finite differences."""
import numpy as np

import oracle


def tiny(seed=0, D=8, d=32, Q=5, N=10, G=6, K=4):
    rng = np.random.default_rng(seed)
    xy = rng.uniform(0, G, size=(1, N, 2)).astype(np.float32)
    cells = rng.choice(G * G, size=Q, replace=False)
    ref = np.stack([(cells % G) + 0.5, (cells // G) + 0.5], axis=1)[None].astype(np.float32)
    f = rng.normal(size=(1, Q, D))
    w_off = 0.03 * rng.normal(size=(D, 2))
    b_off = 0.02 * rng.normal(size=2)
    feats = rng.normal(size=(1, N, d))
    p = rng.uniform(0.5, 2.0, size=d // 32)
    w_o = rng.normal(size=(d, D)) / np.sqrt(d)
    table = oracle.knn_table(xy, G, G, K)
    df = rng.normal(size=(1, Q, D))
    return dict(ref=ref, f=f, w_off=w_off, b_off=b_off, feats=feats, xy=xy, table=table, p=p,
                w_o=w_o, df=df)


def test_offsets_closed_forms():
    t = tiny()
    ref, f, w, b = t["ref"], t["f"], t["w_off"], t["b_off"]
    # zero features: q = r + b
    np.testing.assert_allclose(oracle.decoder_offsets(ref, 0 * f, w, b)[0], ref[0] + b, rtol=0,
                               atol=1e-12)
    # a worked case: D = 2, f = (1, 2), W_off = [[1, -1], [0.5, 2]], b = (0.25, 0)
    q = oracle.decoder_offsets(np.array([[[3.5, 4.5]]], np.float32), np.array([[[1.0, 2.0]]]),
                               np.array([[1.0, -1.0], [0.5, 2.0]]), np.array([0.25, 0.0]))
    np.testing.assert_allclose(q[0, 0], [3.5 + 1.0 + 1.0 + 0.25, 4.5 - 1.0 + 4.0], rtol=0,
                               atol=1e-12)
    # linear in f
    f2 = np.random.default_rng(3).normal(size=f.shape)
    lhs = oracle.decoder_offsets(ref, f + f2, w, b) - oracle.decoder_offsets(ref, f2, w, b)
    rhs = oracle.decoder_offsets(ref, f, w, b) - oracle.decoder_offsets(ref, 0 * f, w, b)
    np.testing.assert_allclose(lhs, rhs, rtol=0, atol=1e-12)


def test_projection_reduces_to_the_gather():
    """W_o = I (d = D) and a zero offset head: the layer adds the plain gather at r."""
    t = tiny(D=32)
    eye = np.eye(32)
    zero = np.zeros((32, 2))
    q, v, f_out = oracle.decoder_layer_fwd(t["ref"], t["f"], zero, np.zeros(2), t["feats"],
                                           t["xy"], t["table"], t["p"], eye)
    np.testing.assert_array_equal(q.astype(np.float32), t["ref"])
    g = oracle.knn_fwd(t["ref"], t["feats"], t["xy"], t["table"], t["p"])
    np.testing.assert_allclose(v, g, rtol=0, atol=0)
    np.testing.assert_allclose(f_out, t["f"] + g, rtol=0, atol=1e-12)


def test_layer_backward_finite_differences():
    t = tiny()
    args = ("ref", "f", "w_off", "b_off", "feats", "xy", "table", "p", "w_o")

    def loss(**kw):
        a = {k: kw.get(k, t[k]) for k in args}
        return float(np.sum(t["df"] * oracle.decoder_layer_fwd(*[a[k] for k in args])[2]))

    q, v, _ = oracle.decoder_layer_fwd(*[t[k] for k in args])
    q32 = q.astype(np.float32)
    # the sample positions stay well inside their cells, so small steps keep the table rows
    frac = q32 - np.floor(q32)
    assert frac.min() > 0.05 and frac.max() < 0.95
    df_in, dw_off, db_off, dfeats, dp, dw_o = oracle.decoder_layer_bwd(
        t["f"], t["w_off"], t["feats"], t["xy"], t["table"], t["p"], t["w_o"], q32, v, t["df"])
    rng = np.random.default_rng(7)
    checks = [("f", df_in, 1e-3), ("w_off", dw_off, 1e-3), ("b_off", db_off, 1e-3),
              ("feats", dfeats, 1e-6), ("p", dp, 1e-6), ("w_o", dw_o, 1e-6)]
    for name, grad, eps in checks:
        x = t[name]
        scale = np.abs(grad).max()
        for _ in range(6):
            idx = tuple(rng.integers(0, s) for s in x.shape)
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            fd = (loss(**{name: xp}) - loss(**{name: xm})) / (2 * eps)
            assert abs(fd - grad[idx]) <= 1e-2 * scale, (name, idx, fd, grad[idx])


def test_two_layer_chain_finite_differences():
    """Two layers over two different stages: the gradient of the first layer's input, taken as
    layer 2's df_in fed to layer 1 as its df_out, against central differences of the composed
    loss (pins the coarse-to-fine chaining of the backward)."""
    t1, t2 = tiny(seed=1), tiny(seed=2, N=14)
    f0 = t1["f"]

    def chain(f):
        _, v1, f1 = oracle.decoder_layer_fwd(t1["ref"], f, t1["w_off"], t1["b_off"], t1["feats"],
                                             t1["xy"], t1["table"], t1["p"], t1["w_o"])
        q2, v2, f2 = oracle.decoder_layer_fwd(t2["ref"], f1, t2["w_off"], t2["b_off"], t2["feats"],
                                              t2["xy"], t2["table"], t2["p"], t2["w_o"])
        return v1, f1, q2, v2, f2

    v1, f1, q2, v2, f2 = chain(f0)
    q1 = oracle.decoder_offsets(t1["ref"], f0, t1["w_off"], t1["b_off"]).astype(np.float32)
    df1 = oracle.decoder_layer_bwd(f1, t2["w_off"], t2["feats"], t2["xy"], t2["table"], t2["p"],
                                   t2["w_o"], q2.astype(np.float32), v2, t2["df"])[0]
    df0 = oracle.decoder_layer_bwd(f0, t1["w_off"], t1["feats"], t1["xy"], t1["table"], t1["p"],
                                   t1["w_o"], q1, v1, df1)[0]
    scale = np.abs(df0).max()
    rng = np.random.default_rng(3)
    eps = 1e-3
    for _ in range(8):
        idx = tuple(rng.integers(0, s) for s in f0.shape)
        fp, fm = f0.copy(), f0.copy()
        fp[idx] += eps
        fm[idx] -= eps
        fd = (np.sum(t2["df"] * chain(fp)[4]) - np.sum(t2["df"] * chain(fm)[4])) / (2 * eps)
        assert abs(fd - df0[idx]) <= 1e-2 * scale, (idx, fd, df0[idx])
