"""Token merging between stages on the GPU against the oracle (AFFMAE notes, "Key
Designs" 1).  The anchor choice is an integer decision taken on the fp32 scores: the GPU's
anchors and assignment must equal the oracle's selection applied to the GPU's scores, and
the scores themselves must match the oracle's fp64 scores within fp32 rounding."""
import numpy as np
import pytest
import torch

import off_grid_cluster_b200 as acl
import oracle
from off_grid_cluster_b200 import synth
from tests.parity import bf16, check_fwd, check_grad, dev, host

pytestmark = pytest.mark.gpu


def merge_both(mb: synth.MergeBatch):
    f, xy = bf16(mb.feats), dev(mb.coords)
    w1, b1, w2 = dev(mb.w1), dev(mb.b1), dev(mb.w2)
    s, anchors, assign, merged, mxy = acl.acl_token_merge_fwd(f, xy, w1, b1, w2, mb.b2, mb.k)
    s_h = host(s)
    s_ref = oracle.merge_scores(mb.feats, mb.w1, mb.b1, mb.w2, mb.b2)
    assert np.abs(s_h - s_ref).max() <= 1e-4 * max(1.0, np.abs(s_ref).max()), "scores"
    a_ref, as_ref = oracle.merge_select(s_h, mb.coords, mb.k)
    assert np.array_equal(anchors.cpu().numpy(), a_ref), "anchors"
    assert np.array_equal(assign.cpu().numpy(), as_ref), "assignment"
    m_ref, mxy_ref = oracle.merge_fwd(mb.feats, mb.coords, s_h, mb.k, as_ref)
    check_fwd(host(merged), m_ref, "merged")
    np.testing.assert_allclose(host(mxy), mxy_ref, rtol=0, atol=2e-4 * max(1.0, np.abs(mxy_ref).max()))
    grads = acl.acl_token_merge_bwd(f, xy, w1, b1, w2, mb.b2, mb.k, s, assign, bf16(mb.dmerged),
                                    dev(mb.dmcoords))
    refs = oracle.merge_bwd(mb.feats, mb.coords, mb.w1, mb.b1, mb.w2, mb.b2, mb.k, as_ref,
                            mb.dmerged, mb.dmcoords)
    for name, got, ref in zip(("dfeats", "dcoords", "dW1", "db1", "dw2"), grads[:5], refs[:5]):
        check_grad(host(got), ref, name)
    # a common shift of the scores changes nothing: db2 vanishes up to rounding
    assert abs(float(grads[5][0])) <= 1e-3 * max(1.0, np.abs(refs[4]).max())
    return grads


def test_merge_stage1_step_workload():
    merge_both(synth.merge_batch(synth.step_batch(B=2).attn.coords, d=128))


@pytest.mark.parametrize("stage", [1, 2])
def test_merge_sweep_stages(stage):
    xy = synth.sweep_coords(B=2)[stage]
    merge_both(synth.merge_batch(xy, d=synth.SWEEP_DIMS[stage]))


def test_merge_small_odd_and_crowded():
    rng = np.random.default_rng(5)
    xy = rng.uniform(0, 6, size=(3, 37, 2)).astype(np.float32)
    xy[1, 5:15] = xy[1, 4]                      # coincident tokens: distance ties
    merge_both(synth.merge_batch(xy, d=32, hidden=8))
    merge_both(synth.merge_batch(xy, d=64, ds=1.0 / 37.0))   # k = 1: one group
    merge_both(synth.merge_batch(xy, d=64, ds=1.0))          # k = N: every token an anchor


def test_merge_is_bit_reproducible():
    mb = synth.merge_batch(synth.step_batch(B=2).attn.coords, d=128)
    f, xy = bf16(mb.feats), dev(mb.coords)
    w1, b1, w2 = dev(mb.w1), dev(mb.b1), dev(mb.w2)
    r1 = acl.acl_token_merge_fwd(f, xy, w1, b1, w2, mb.b2, mb.k)
    r2 = acl.acl_token_merge_fwd(f, xy, w1, b1, w2, mb.b2, mb.k)
    for x, y in zip(r1, r2):
        assert torch.equal(x, y)
    g1 = acl.acl_token_merge_bwd(f, xy, w1, b1, w2, mb.b2, mb.k, r1[0], r1[2], bf16(mb.dmerged),
                                 dev(mb.dmcoords))
    g2 = acl.acl_token_merge_bwd(f, xy, w1, b1, w2, mb.b2, mb.k, r1[0], r1[2], bf16(mb.dmerged),
                                 dev(mb.dmcoords))
    for x, y in zip(g1, g2):
        assert torch.equal(x, y)


@pytest.mark.parametrize("d,hidden", [(64, 100), (64, 256), (1024, 8), (64, 16), (192, 48)])
def test_merge_hidden_widths(d, hidden):
    """Hidden widths that are not a multiple of 32 (padded units), the widest (256), a W1 too
    large for shared memory (read from global memory), and the smallest and an odd-tile shape
    of the tensor-core MLP (d = 64, h = 16; d = 192, h = 48)."""
    rng = np.random.default_rng(11)
    xy = rng.uniform(0, 20, size=(2, 300, 2)).astype(np.float32)
    merge_both(synth.merge_batch(xy, d=d, hidden=hidden))


def test_merge_score_ties_and_many_tokens():
    """Tokens with identical features get bit-identical scores: the anchors among them are the
    lowest ids.  N = 5000 spans many CTAs of the counting and assignment kernels."""
    rng = np.random.default_rng(12)
    xy = rng.uniform(0, 70, size=(1, 5000, 2)).astype(np.float32)
    mb = synth.merge_batch(xy, d=32, hidden=8)
    mb.feats[:, 100:400] = mb.feats[:, 99:100]
    merge_both(mb)


def test_merge_binned_search_extremes():
    """The binned nearest-anchor search: 200 coincident tokens, far outliers (a bin grid
    stretched over 10^6 cells), and integer-lattice coordinates (many exact distance ties)."""
    rng = np.random.default_rng(21)
    xy = rng.uniform(0, 8, size=(2, 400, 2)).astype(np.float32)
    xy[0, :200] = 3.25
    xy[0, 390] = (1.0e6, -2.5e5)
    xy[0, 391] = (-7.0e5, 3.0e5)
    xy[1] = np.round(xy[1] * 2.0) / 2.0
    merge_both(synth.merge_batch(xy, d=32, hidden=8))


def test_merge_many_anchors_full_scan():
    """k above the binned search's limit (4500 anchors) takes the full-scan kernel."""
    rng = np.random.default_rng(22)
    xy = rng.uniform(0, 100, size=(1, 10000, 2)).astype(np.float32)
    merge_both(synth.merge_batch(xy, d=32, hidden=8, ds=0.45))
