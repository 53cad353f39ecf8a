"""GPU parity of acl_cluster_attn_fwd / acl_cluster_attn_bwd with the fp64 oracle.

Both sides take the same seeded bf16 inputs.  The oracle computes its own
clusters and neighbourhood table (the GPU's are checked bit-exact against them
in test_gpu_cluster.py), and the GPU attention runs on that table.  The oracle's
backward recomputes its own forward; the GPU backward consumes the GPU forward's
O and lse, as a caller would.
"""
import math

import numpy as np
import pytest
import torch

import off_grid_cluster_b200 as acl
import oracle
from off_grid_cluster_b200 import synth
from tests.parity import LSE_ATOL, bf16, check_fwd, check_grad, dev, host

pytestmark = pytest.mark.gpu


def run_attn(a: synth.AttnBatch, M: int = 48, check_bwd: bool = True, scale=None, cl=None, nb=None):
    scale = a.scale if scale is None else scale
    if cl is None:
        cl = oracle.cluster(a.coords, 8)
    if nb is None:
        nb = oracle.neighbors(a.coords, cl, M)
    o_ref, lse_ref = oracle.attn_fwd(a.q, a.k, a.v, a.coords, cl, nb, a.bias, scale)
    Q, K, V, dO = bf16(a.q), bf16(a.k), bf16(a.v), bf16(a.do)
    xy, tcl, tnb, bias = dev(a.coords), dev(cl), dev(nb), dev(a.bias)
    O, lse = acl.acl_cluster_attn_fwd(Q, K, V, xy, tcl, tnb, bias, scale)
    stats = check_fwd(host(O), o_ref, "O")
    lse_g = host(lse)
    assert np.abs(lse_g - lse_ref).max() <= LSE_ATOL
    if not check_bwd:
        return stats
    dq_r, dk_r, dv_r, db_r = oracle.attn_bwd(a.q, a.k, a.v, a.coords, cl, nb, a.bias, scale, a.do)
    dQ, dK, dV, db = acl.acl_cluster_attn_bwd(Q, K, V, xy, tcl, tnb, bias, scale, O, dO, lse)
    for name, g, r in (("dQ", dQ, dq_r), ("dK", dK, dk_r), ("dV", dV, dv_r), ("dbias", db, db_r)):
        stats[name] = check_grad(host(g), r, name)
    return stats


def test_tiny():
    run_attn(synth.attn_tiny())


def ffma_fwd(a: synth.AttnBatch, M: int = 48):
    """The FMA-only forward (the tensor-core kernel's reference variant) against the oracle."""
    cl = oracle.cluster(a.coords, 8)
    nb = oracle.neighbors(a.coords, cl, M)
    o_ref, lse_ref = oracle.attn_fwd(a.q, a.k, a.v, a.coords, cl, nb, a.bias, a.scale)
    O, lse = acl.acl_cluster_attn_fwd_ffma(bf16(a.q), bf16(a.k), bf16(a.v), dev(a.coords), dev(cl), dev(nb),
                                           dev(a.bias), a.scale)
    check_fwd(host(O), o_ref, "O (FMA variant)")
    assert np.abs(host(lse) - lse_ref).max() <= LSE_ATOL


@pytest.mark.parametrize("case", ["stage1_b8", "stage3", "M64_ragged", "tiny"])
def test_ffma_forward_variant(case):
    if case == "stage1_b8":
        ffma_fwd(synth.attn_stage1(B=8))
    elif case == "stage3":
        ffma_fwd(synth.attn_stage3(B=8))
    elif case == "M64_ragged":
        ffma_fwd(synth.attn_stage1(B=2, N=701, H=3), M=64)
    else:
        ffma_fwd(synth.attn_tiny())


def test_stage1_full_batch():
    # 8 images x 2048 tokens x 4 heads: the benchmark workload's attention, every output
    run_attn(synth.attn_stage1())


def test_stage3_many_heads():
    run_attn(synth.attn_stage3())


@pytest.mark.parametrize("stage", [0, 1, 2, 3])
def test_sweep_layer_per_stage(stage):
    coords = synth.sweep_coords(B=16)[stage]
    run_attn(synth.attn_sweep_layer(coords, stage, 0))


@pytest.mark.parametrize("M", [8, 16, 24, 32, 40, 56, 64])
def test_neighbourhood_sizes(M):
    a = synth.attn_stage1(B=2, N=700, H=2)
    run_attn(a, M=M)


@pytest.mark.parametrize("N", [1, 5, 8, 9, 45, 48, 49, 131])
def test_small_and_ragged(N):
    full = synth.attn_stage1(B=2, N=N, H=3)
    run_attn(full)


def test_scale_and_strong_bias():
    a = synth.attn_stage1(B=1, N=512, H=4)
    a.bias = (a.bias * 20.0).astype(np.float32)         # sharply peaked softmax
    run_attn(a, scale=0.5)


def test_deterministic_and_overwrites():
    a = synth.attn_stage1(B=2, N=600, H=4)
    cl = oracle.cluster(a.coords, 8)
    nb = oracle.neighbors(a.coords, cl, 48)
    Q, K, V, dO = bf16(a.q), bf16(a.k), bf16(a.v), bf16(a.do)
    xy, tcl, tnb, bias = dev(a.coords), dev(cl), dev(nb), dev(a.bias)
    O, lse = acl.acl_cluster_attn_fwd(Q, K, V, xy, tcl, tnb, bias, a.scale)
    ws = torch.full((acl.acl_cluster_attn_workspace(2, 600, 4),), 0x7F, dtype=torch.uint8,
                    device="cuda")
    g1 = acl.acl_cluster_attn_bwd(Q, K, V, xy, tcl, tnb, bias, a.scale, O, dO, lse, workspace=ws)
    outs = [torch.full_like(t, float("nan")) for t in g1]
    g2 = acl.acl_cluster_attn_bwd(Q, K, V, xy, tcl, tnb, bias, a.scale, O, dO, lse, *outs,
                                  workspace=ws)
    for x, y in zip(g1, g2):
        assert torch.equal(x, y)          # bit-identical, and every element overwritten
    O2 = torch.full_like(O, float("nan"))
    acl.acl_cluster_attn_fwd(Q, K, V, xy, tcl, tnb, bias, a.scale, O=O2, lse=torch.empty_like(lse))
    assert torch.equal(O, O2)


def test_zero_query_zero_bias_is_mean():
    a = synth.attn_stage1(B=1, N=256, H=2)
    cl = oracle.cluster(a.coords, 8)
    nb = oracle.neighbors(a.coords, cl, 48)
    z = torch.zeros(1, 256, 2, 32, dtype=torch.bfloat16, device="cuda")
    O, lse = acl.acl_cluster_attn_fwd(z, bf16(a.k), bf16(a.v), dev(a.coords), dev(cl), dev(nb),
                                      torch.zeros(2, 3, device="cuda"), a.scale)
    assert torch.allclose(lse, torch.full_like(lse, math.log(48.0)), atol=1e-5)
    v = a.v[0]
    for g in range(cl.shape[1]):
        keys = nb[0, g]
        for i in cl[0, g]:
            np.testing.assert_allclose(host(O)[0, i], v[keys].mean(axis=0), atol=1e-2)


# The key pass walks a key cluster's reverse list in chunks of this many listed query
# clusters, carrying the dK / dV accumulators across chunks; its warps read list offsets
# through a window of this many consecutive key clusters.
KEY_CHUNK = 4
OFFSET_WINDOW = 32


def hub_table(cl: np.ndarray, M: int, seed: int) -> np.ndarray:
    """Neighbour table in which every cluster lists cluster 0 first, then itself, then
    R - 2 other clusters at random (whole cluster rows, as the backward requires)."""
    B, G, C = cl.shape
    R = M // C
    rng = np.random.default_rng(seed)
    nb = np.full((B, G, M), -1, np.int32)
    for b in range(B):
        for g in range(G):
            rest = [h for h in rng.permutation(G) if h not in (0, g)]
            lst = ([0, g] if g else [0]) + rest
            for r, h in enumerate(lst[:R]):
                nb[b, g, r * C:(r + 1) * C] = cl[b, h]
    return nb


@pytest.mark.parametrize("M", [48, 64])
def test_hub_table_long_reverse_lists(M):
    """A hand-built table in which every cluster lists cluster 0.  The reverse list of
    cluster 0 then holds every query cluster of the image, so its key-pass units run many
    chunks with accumulators carried between them, while the other key clusters have short
    lists; the per-warp plan balances chunk items, so one warp's range starts and ends in the
    middle of the hub's list and the offset window is refilled across image boundaries.  The
    assertions show the table has these shapes; the parity checks cover them against the
    oracle."""
    a = synth.attn_stage1(B=2, N=700, H=3)
    cl = oracle.cluster(a.coords, 8)
    nb = hub_table(cl, M, seed=11 + M)
    B, G, _ = cl.shape
    R = M // 8
    lens = []
    for b in range(B):
        first = {int(cl[b, g, 0]): g for g in range(G)}
        rev = [0] * G
        for g in range(G):
            for r in range(R):
                rev[first[int(nb[b, g, r * 8])]] += 1
        lens.append(rev)
    lens = np.array(lens)
    assert lens[:, 0].min() == G                          # the hub is listed by every cluster
    assert lens.max() > 4 * KEY_CHUNK                     # many chunks for one unit
    assert (lens <= KEY_CHUNK).sum() >= 10                 # and single-chunk units beside it
    assert B * G > OFFSET_WINDOW                          # window refills
    run_attn(a, M=M, cl=cl, nb=nb)
