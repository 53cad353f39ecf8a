"""fp64 CPU oracle for the off-grid cluster attention and KNN gather.

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check and by the
benchmark's CPU-baseline / reference leg.  The product library never imports
it and shares no code with it.  This module is argument marshalling around
oracle.c (numpy in, numpy out); all arithmetic lives in the C file, which
cites the passages it follows.

Array conventions (numpy): xy [B, N, 2] float32; q/k/v/dout [B, N, H, D]
(converted to float64); bias [H, 3]; clusters [B, G, C] int32; nbr [B, G, M]
int32; table [B, GH, GW, K] int32; queries [B, Q, 2] float32; feats
[B, N, d]; p [d/32].
"""
from __future__ import annotations

import ctypes as ct
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        so = _build.build()
        L = ct.CDLL(so)
        for name in ("orc_cluster_batch", "orc_neighbors_batch", "orc_attn_fwd_batch",
                     "orc_attn_bwd_batch", "orc_knn_table_batch", "orc_knn_fwd_batch",
                     "orc_knn_bwd_batch", "orc_set_threads", "orc_token_order_batch",
                     "orc_merge_scores", "orc_merge_select", "orc_merge_fwd", "orc_merge_bwd",
                     "orc_dec_offsets", "orc_dec_project", "orc_dec_project_bwd",
                     "orc_dec_offsets_bwd"):
            getattr(L, name).restype = ct.c_int
        _lib = L
    return _lib


def _p(a):
    return a.ctypes.data_as(ct.c_void_p)


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _i32(a):
    return np.ascontiguousarray(a, dtype=np.int32)


def _check(rc, what):
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with code {rc}")


def set_threads(n: int) -> int:
    """Set the OpenMP thread count of the batch drivers; returns the count in use."""
    return int(lib().orc_set_threads(int(n)))


def cluster(xy, C: int = 8) -> np.ndarray:
    xy = _f32(xy)
    B, N = xy.shape[:2]
    G = (N + C - 1) // C
    out = np.empty((B, G, C), dtype=np.int32)
    _check(lib().orc_cluster_batch(_p(xy), B, N, C, _p(out)), "cluster")
    return out


def neighbors(xy, clusters, M: int = 48) -> np.ndarray:
    xy, clusters = _f32(xy), _i32(clusters)
    B, N = xy.shape[:2]
    G, C = clusters.shape[1:]
    out = np.empty((B, G, M), dtype=np.int32)
    _check(lib().orc_neighbors_batch(_p(xy), _p(clusters), B, N, C, M, _p(out)), "neighbors")
    return out


def attn_fwd(q, k, v, xy, clusters, nbr, bias, scale: float):
    q, k, v, bias = _f64(q), _f64(k), _f64(v), _f64(bias)
    xy, clusters, nbr = _f32(xy), _i32(clusters), _i32(nbr)
    B, N, H, D = q.shape
    C, M = clusters.shape[2], nbr.shape[2]
    o = np.empty_like(q)
    lse = np.empty((B, N, H), dtype=np.float64)
    _check(lib().orc_attn_fwd_batch(_p(q), _p(k), _p(v), _p(xy), _p(clusters), _p(nbr),
                                    _p(bias), B, N, H, D, C, M, ct.c_double(scale),
                                    _p(o), _p(lse)), "attn_fwd")
    return o, lse


def attn_bwd(q, k, v, xy, clusters, nbr, bias, scale: float, dout):
    q, k, v, bias, dout = _f64(q), _f64(k), _f64(v), _f64(bias), _f64(dout)
    xy, clusters, nbr = _f32(xy), _i32(clusters), _i32(nbr)
    B, N, H, D = q.shape
    C, M = clusters.shape[2], nbr.shape[2]
    dq, dk, dv = np.empty_like(q), np.empty_like(q), np.empty_like(q)
    dbias = np.empty((H, 3), dtype=np.float64)
    _check(lib().orc_attn_bwd_batch(_p(q), _p(k), _p(v), _p(xy), _p(clusters), _p(nbr),
                                    _p(bias), B, N, H, D, C, M, ct.c_double(scale),
                                    _p(dout), _p(dq), _p(dk), _p(dv), _p(dbias)), "attn_bwd")
    return dq, dk, dv, dbias


def knn_table(xy, GH: int = 64, GW: int = 64, K: int = 8) -> np.ndarray:
    xy = _f32(xy)
    B, N = xy.shape[:2]
    out = np.empty((B, GH, GW, K), dtype=np.int32)
    _check(lib().orc_knn_table_batch(_p(xy), B, N, GH, GW, K, _p(out)), "knn_table")
    return out


KNN_EXP, KNN_INVPOW = 0, 1  # weight kernels: softmax(-p d) and d^-p / sum d^-p


def knn_fwd(queries, feats, xy, table, p, kind=KNN_EXP):
    queries, xy, table = _f32(queries), _f32(xy), _i32(table)
    feats, p = _f64(feats), _f64(p)
    B, Q = queries.shape[:2]
    N, d = feats.shape[1:]
    GH, GW, K = table.shape[1:]
    out = np.empty((B, Q, d), dtype=np.float64)
    _check(lib().orc_knn_fwd_batch(_p(queries), B, Q, _p(feats), _p(xy), N, d, _p(table),
                                   GH, GW, K, _p(p), int(kind), _p(out)), "knn_fwd")
    return out


def knn_bwd(queries, feats, xy, table, p, dout, kind=KNN_EXP):
    queries, xy, table = _f32(queries), _f32(xy), _i32(table)
    feats, p, dout = _f64(feats), _f64(p), _f64(dout)
    B, Q = queries.shape[:2]
    N, d = feats.shape[1:]
    GH, GW, K = table.shape[1:]
    dF = np.empty((B, N, d), dtype=np.float64)
    dq = np.empty((B, Q, 2), dtype=np.float64)
    dp = np.empty((d // 32,), dtype=np.float64)
    _check(lib().orc_knn_bwd_batch(_p(queries), B, Q, _p(feats), _p(xy), N, d, _p(table),
                                   GH, GW, K, _p(p), int(kind), _p(dout), _p(dF), _p(dq),
                                   _p(dp)),
           "knn_bwd")
    return dF, dq, dp


def token_order(xy, GH, GW):
    """Token ids of each image in Z-order of their cells on the GH x GW grid -> [B, N] int32."""
    xy = _f32(xy)
    B, N = xy.shape[:2]
    perm = np.empty((B, N), dtype=np.int32)
    _check(lib().orc_token_order_batch(_p(xy), B, N, GH, GW, _p(perm)), "token_order")
    return perm


# ------------------------------------------------------------------ token merging

def merge_scores(feats, w1, b1, w2, b2):
    """Importance scores s = w2 . gelu(W1^T f + b1) + b2 -> [B, N] fp64."""
    feats, w1, b1, w2 = _f64(feats), _f64(w1), _f64(b1), _f64(w2)
    B, N, d = feats.shape
    h = w1.shape[1]
    out = np.empty((B, N), dtype=np.float64)
    for b in range(B):
        _check(lib().orc_merge_scores(_p(feats[b]), N, d, _p(w1), _p(b1), _p(w2),
                                      ct.c_double(float(b2)), h, _p(out[b])), "merge_scores")
    return out


def merge_select(scores, xy, k):
    """Anchors (top-k scores, ties by id, ascending id) and nearest-anchor assignment."""
    scores, xy = _f64(scores), _f32(xy)
    B, N = scores.shape
    anchors = np.empty((B, k), dtype=np.int32)
    assign = np.empty((B, N), dtype=np.int32)
    for b in range(B):
        _check(lib().orc_merge_select(_p(scores[b]), _p(xy[b]), N, k, _p(anchors[b]),
                                      _p(assign[b])), "merge_select")
    return anchors, assign


def merge_fwd(feats, xy, scores, k, assign):
    """Merged features [B, k, d] and coordinates [B, k, 2] (softmax-of-score weights)."""
    feats, xy, scores, assign = _f64(feats), _f32(xy), _f64(scores), _i32(assign)
    B, N, d = feats.shape
    merged = np.empty((B, k, d), dtype=np.float64)
    mxy = np.empty((B, k, 2), dtype=np.float64)
    for b in range(B):
        _check(lib().orc_merge_fwd(_p(feats[b]), _p(xy[b]), N, d, _p(scores[b]), k,
                                   _p(assign[b]), _p(merged[b]), _p(mxy[b])), "merge_fwd")
    return merged, mxy


def merge_bwd(feats, xy, w1, b1, w2, b2, k, assign, dmerged, dmxy):
    """(dfeats, dcoords, dW1, db1, dw2, db2) for fixed anchors/assignment; parameter
    gradients summed over the images."""
    feats, xy, assign = _f64(feats), _f32(xy), _i32(assign)
    w1, b1, w2 = _f64(w1), _f64(b1), _f64(w2)
    dmerged, dmxy = _f64(dmerged), _f64(dmxy)
    B, N, d = feats.shape
    h = w1.shape[1]
    df = np.empty((B, N, d)); dxy = np.empty((B, N, 2))
    dw1 = np.zeros((d, h)); db1 = np.zeros(h); dw2 = np.zeros(h); db2 = 0.0
    for b in range(B):
        t1, t2, t3 = np.empty((d, h)), np.empty(h), np.empty(h)
        t4 = ct.c_double(0.0)
        _check(lib().orc_merge_bwd(_p(feats[b]), _p(xy[b]), N, d, _p(w1), _p(b1), _p(w2),
                                   ct.c_double(float(b2)), h, k, _p(assign[b]), _p(dmerged[b]),
                                   _p(dmxy[b]), _p(df[b]), _p(dxy[b]), _p(t1), _p(t2), _p(t3),
                                   ct.byref(t4)), "merge_bwd")
        dw1 += t1; db1 += t2; dw2 += t3; db2 += t4.value
    return df, dxy, dw1, db1, dw2, db2


def decoder_offsets(ref, f, w_off, b_off):
    """Sample positions q = r + f W_off + b_off in fp64 -> [B, Q, 2]."""
    ref, f, w_off, b_off = _f32(ref), _f64(f), _f64(w_off), _f64(b_off)
    B, Q, D = f.shape
    q = np.empty((B, Q, 2))
    for b in range(B):
        _check(lib().orc_dec_offsets(_p(ref[b]), _p(f[b]), Q, D, _p(w_off), _p(b_off), _p(q[b])),
               "dec_offsets")
    return q


def decoder_layer_fwd(ref, f, w_off, b_off, feats, xy, table, p, w_o, q=None):
    """One decoder layer: (q fp64, v = the stage gather at q, f_out = f + v W_o).  The gather
    samples at q rounded to fp32, or at the given fp32 q (the cell choice is an integer
    decision: a caller comparing with another implementation passes that one's q)."""
    q64 = decoder_offsets(ref, f, w_off, b_off)
    qs = q64.astype(np.float32) if q is None else _f32(q)
    v = knn_fwd(qs, feats, xy, table, p)
    f, w_o = _f64(f), _f64(w_o)
    B, Q, D = f.shape
    d = v.shape[2]
    f_out = np.empty((B, Q, D))
    for b in range(B):
        _check(lib().orc_dec_project(_p(f[b]), _p(v[b]), Q, D, d, _p(w_o), _p(f_out[b])),
               "dec_project")
    return q64, v, f_out


def decoder_layer_bwd(f, w_off, feats, xy, table, p, w_o, q, v, df_out):
    """Backward of one decoder layer at the fp32 sample positions q with gathered v:
    (df_in, dW_off, db_off, dfeats, dp, dW_o); parameter gradients summed over images."""
    f, w_off, w_o, v, df_out = _f64(f), _f64(w_off), _f64(w_o), _f64(v), _f64(df_out)
    B, Q, D = f.shape
    d = v.shape[2]
    dv = np.empty((B, Q, d))
    dw_o = np.zeros((d, D))
    for b in range(B):
        _check(lib().orc_dec_project_bwd(_p(v[b]), _p(df_out[b]), Q, D, d, _p(w_o), _p(dv[b]),
                                         _p(dw_o)), "dec_project_bwd")
    dfeats, dq, dp = knn_bwd(q, feats, xy, table, p, dv)
    df_in = np.empty((B, Q, D))
    dw_off = np.zeros((D, 2))
    db_off = np.zeros(2)
    for b in range(B):
        _check(lib().orc_dec_offsets_bwd(_p(f[b]), _p(dq[b]), _p(df_out[b]), Q, D, _p(w_off),
                                         _p(df_in[b]), _p(dw_off), _p(db_off)), "dec_offsets_bwd")
    return df_in, dw_off, db_off, dfeats, dp, dw_o
