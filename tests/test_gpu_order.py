"""Space-filling token order and the high-resolution table/gather on the GPU, against the
oracle (AFFMAE notes, "Limitations": space-filling curves; grids above ~1200 px)."""
import numpy as np
import pytest
import torch

import off_grid_cluster_b200 as acl
import oracle
from off_grid_cluster_b200 import synth
from tests.parity import bf16, check_fwd, check_grad, dev, host

pytestmark = pytest.mark.gpu


def order_both(xy: np.ndarray, H: int, W: int):
    ref = oracle.token_order(xy, H, W)
    got = acl.acl_token_order(dev(xy), H, W).cpu().numpy()
    assert np.array_equal(got, ref), "token order differs from the oracle"
    return ref


def test_order_hires_and_step_workloads():
    order_both(synth.hires_batch(B=2).coords, 128, 128)
    order_both(synth.step_batch(B=2).attn.coords, 64, 64)


def test_order_full_grid_and_rectangles():
    for H, W in ((32, 32), (8, 40), (45, 13)):
        r, c = np.divmod(np.arange(H * W), W)
        xy = np.stack([c + 0.5, r + 0.5], 1).astype(np.float32)[None]
        order_both(xy, H, W)


def test_order_crowded_cells_and_limits():
    rng = np.random.default_rng(0)
    xy = rng.uniform(-2.0, 10.0, size=(2, 3000, 2)).astype(np.float32)
    xy[0, :200] = xy[0, 7]                          # 200 tokens in one cell: bitonic path
    order_both(xy, 8, 8)
    xy = rng.uniform(0.0, 4096.0, size=(1, 16384, 2)).astype(np.float32)
    order_both(xy, 4096, 4096)                      # largest N and grid
    order_both(np.array([[[3.2, 1.1]]], dtype=np.float32), 4, 4)


def test_table_and_gather_at_128x128():
    kb = synth.hires_batch(B=2)
    table_ref = oracle.knn_table(kb.coords, 128, 128, 8)
    xy = dev(kb.coords)
    table = acl.acl_knn_table(xy, 128, 128, 8)
    assert np.array_equal(table.cpu().numpy(), table_ref)
    q, f, p, g = dev(kb.queries), bf16(kb.feats), dev(kb.p), bf16(kb.dout)
    out = acl.acl_knn_gather_fwd(q, f, xy, table, p)
    check_fwd(host(out), oracle.knn_fwd(kb.queries, kb.feats, kb.coords, table_ref, kb.p), "out")
    dF, dq, dp = acl.acl_knn_gather_bwd(q, f, xy, table, p, g)
    rF, rq, rp = oracle.knn_bwd(kb.queries, kb.feats, kb.coords, table_ref, kb.p, kb.dout)
    check_grad(host(dF), rF, "dfeats")
    check_grad(host(dq), rq, "dqueries")
    check_grad(host(dp), rp, "dp")


def test_gather_over_z_ordered_tokens_gives_the_same_results():
    kb = synth.hires_batch(B=2)
    xy, f = dev(kb.coords), bf16(kb.feats)
    perm = acl.acl_token_order(xy, 128, 128).long()
    bidx = torch.arange(2, device="cuda")[:, None]
    xy_z, f_z = xy[bidx, perm].contiguous(), f[bidx, perm].contiguous()
    q, p, g = dev(kb.queries), dev(kb.p), bf16(kb.dout)
    t_r = acl.acl_knn_table(xy, 128, 128, 8)
    t_z = acl.acl_knn_table(xy_z, 128, 128, 8)
    out_r = acl.acl_knn_gather_fwd(q, f, xy, t_r, p)
    out_z = acl.acl_knn_gather_fwd(q, f_z, xy_z, t_z, p)
    dF_r, dq_r, dp_r = acl.acl_knn_gather_bwd(q, f, xy, t_r, p, g)
    dF_z, dq_z, dp_z = acl.acl_knn_gather_bwd(q, f_z, xy_z, t_z, p, g)
    # same neighbours in the same slot order: identical sums (distance ties aside)
    torch.testing.assert_close(out_z, out_r, atol=1e-2, rtol=0)
    torch.testing.assert_close(dF_z, dF_r[bidx, perm], atol=2e-2, rtol=0)
    torch.testing.assert_close(dq_z, dq_r, atol=1e-3, rtol=1e-3)
    torch.testing.assert_close(dp_z, dp_r, atol=1e-3, rtol=1e-3)
