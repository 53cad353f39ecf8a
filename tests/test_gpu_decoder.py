"""Decoder layer on the GPU against the oracle (AFFMAE notes, "Key Designs" 2, the point-wise
deformable cross-attention decoder; readings in the oracle: linear offset head, residual
projection of the gathered feature).  The table cell of each sample point is an integer
decision taken on the fp32 q: q is checked against the oracle's fp64 offsets, and the oracle
then gathers at the GPU's q.  Four layers run coarse to fine, each layer's input being the
previous layer's GPU output on both sides."""
import numpy as np
import pytest
import torch

import off_grid_cluster_b200 as acl
import oracle
from off_grid_cluster_b200 import synth
from tests.parity import FWD_ATOL, bf16, check_fwd, check_grad, dev, host

pytestmark = pytest.mark.gpu

Q_ATOL = 1e-4   # fp32 sample positions (|q| < 70) against the fp64 offsets


def layer_both(ref, f_in, w_off, b_off, w_o, st, df, table=None):
    """One layer forward + backward on both sides; returns the GPU's (f_out, df_in)."""
    table = oracle.knn_table(st.coords, st.GH, st.GW, st.K) if table is None else table
    g = dict(feats=bf16(st.feats), coords=dev(st.coords), table=dev(table), p=dev(st.p))
    f_d, wo_d, woff_d = dev(f_in), bf16(w_o), dev(w_off)
    q, v, f_out = acl.acl_decoder_layer_fwd(dev(ref), f_d, woff_d, dev(b_off), wo_d, **g)
    q_h = q.cpu().numpy()
    q64 = oracle.decoder_offsets(ref, f_in, w_off, b_off)
    assert np.abs(q_h - q64).max() <= Q_ATOL, "q"
    _, v_ref, f_ref = oracle.decoder_layer_fwd(ref, f_in, w_off, b_off, st.feats, st.coords, table,
                                               st.p, w_o, q=q_h)
    check_fwd(host(v), v_ref, "v")
    err = np.abs(host(f_out) - f_ref).max()
    assert err <= FWD_ATOL, f"f_out: max abs err {err:.3e}"
    grads = acl.acl_decoder_layer_bwd(f_d, woff_d, wo_d, q=q, v=v, df_out=dev(df), **g)
    acl.acl_device_check()  # no bounded tensor-core wait gave up
    refs = oracle.decoder_layer_bwd(f_in, w_off, st.feats, st.coords, table, st.p, w_o, q_h, v_ref, df)
    for name, got, want in zip(("df_in", "dW_off", "db_off", "dfeats", "dp", "dW_o"),
                               (grads[0], grads[1], grads[2], grads[4], grads[5], grads[3]), refs):
        check_grad(host(got), want, name)
    return host(f_out).astype(np.float32), host(grads[0]).astype(np.float32)


def run_decoder(db: synth.DecoderBatch):
    f = db.f0
    for layer, s in enumerate(db.layer_stage):
        f, _ = layer_both(db.ref, f, db.w_off[layer], db.b_off[layer], db.w_o[layer],
                          db.stages[s], db.df)


def test_decoder_four_layers_coarse_to_fine():
    run_decoder(synth.decoder_batch(B=2))


def test_decoder_backward_chain():
    """The gradient of layer l + 1's input is layer l's output gradient (GPU values on both
    sides), through all four layers."""
    db = synth.decoder_batch(B=1)
    fs = [db.f0]
    for layer, s in enumerate(db.layer_stage):
        f_d = dev(fs[-1])
        st = db.stages[s]
        table = oracle.knn_table(st.coords, st.GH, st.GW, st.K)
        _, _, f_out = acl.acl_decoder_layer_fwd(
            dev(db.ref), f_d, dev(db.w_off[layer]), dev(db.b_off[layer]), bf16(db.w_o[layer]),
            bf16(st.feats), dev(st.coords), dev(table), dev(st.p))
        fs.append(host(f_out).astype(np.float32))
    df = db.df
    for layer in reversed(range(4)):
        s = db.layer_stage[layer]
        _, df = layer_both(db.ref, fs[layer], db.w_off[layer], db.b_off[layer], db.w_o[layer],
                           db.stages[s], df)


def test_decoder_ragged_and_far_offsets():
    """37 queries (a ragged GEMM tile), D = 384 (three column tiles), one image, offsets of
    about 30 cells (many sample points clamped to the border), and a tiny stage."""
    db = synth.decoder_batch(B=1, D=384, offset_scale=30.0)
    ref = db.ref[:, :37].copy()
    f = db.f0[:, :37].copy()
    df = db.df[:, :37].copy()
    for layer, s in ((0, 3), (3, 0)):
        layer_both(ref, f, db.w_off[layer], db.b_off[layer], db.w_o[layer], db.stages[s], df)


def test_decoder_full_size_stage4():
    """The benchmark's size on the coarsest layer (8 images x 2048 queries, d = 768)."""
    db = synth.decoder_batch(B=8)
    layer_both(db.ref, db.f0, db.w_off[0], db.b_off[0], db.w_o[0], db.stages[3], db.df)


def test_decoder_is_bit_reproducible():
    db = synth.decoder_batch(B=2)
    st = db.stages[3]
    table = dev(oracle.knn_table(st.coords, st.GH, st.GW, st.K))
    g = dict(feats=bf16(st.feats), coords=dev(st.coords), table=table, p=dev(st.p))
    args = (dev(db.f0), dev(db.w_off[0]), bf16(db.w_o[0]))
    outs = []
    for _ in range(2):
        q, v, f_out = acl.acl_decoder_layer_fwd(dev(db.ref), args[0], args[1], dev(db.b_off[0]),
                                                args[2], **g)
        grads = acl.acl_decoder_layer_bwd(*args, q=q, v=v, df_out=dev(db.df), **g)
        outs.append((q, v, f_out) + tuple(grads))
    for x, y in zip(*outs):
        assert torch.equal(x, y)


def test_decoder_no_queries():
    """Q = 0: the forward has nothing to write; the backward's parameter and stage gradients
    are zero sums."""
    db = synth.decoder_batch(B=1)
    st = db.stages[3]
    table = dev(oracle.knn_table(st.coords, st.GH, st.GW, st.K))
    g = dict(feats=bf16(st.feats), coords=dev(st.coords), table=table, p=dev(st.p))
    ref = torch.empty((1, 0, 2), dtype=torch.float32, device="cuda")
    f0 = torch.empty((1, 0, db.D), dtype=torch.float32, device="cuda")
    q, v, f_out = acl.acl_decoder_layer_fwd(ref, f0, dev(db.w_off[0]), dev(db.b_off[0]),
                                            bf16(db.w_o[0]), **g)
    assert q.numel() == 0 and v.numel() == 0 and f_out.numel() == 0
    grads = acl.acl_decoder_layer_bwd(f0, dev(db.w_off[0]), bf16(db.w_o[0]), q=q, v=v,
                                      df_out=torch.empty_like(f0), **g)
    acl.acl_device_check()
    for t in grads[1:]:
        assert torch.count_nonzero(t).item() == 0
