"""GPU parity of acl_cluster and acl_neighbors with the oracle: bit-exact."""
import numpy as np
import pytest
import torch

import off_grid_cluster_b200 as acl
import oracle
from off_grid_cluster_b200 import synth
from tests import golden
from tests.parity import dev

pytestmark = pytest.mark.gpu


def run_both(xy: np.ndarray, C: int = 8, M: int = 48):
    cl_ref = oracle.cluster(xy, C)
    t = dev(xy)
    cl = acl.acl_cluster(t, C)
    assert np.array_equal(cl.cpu().numpy(), cl_ref), "clusters differ from the oracle"
    if M % C == 0 and M // C <= 16:
        nb_ref = oracle.neighbors(xy, cl_ref, M)
        nb = acl.acl_neighbors(t, cl, M)
        assert np.array_equal(nb.cpu().numpy(), nb_ref), "neighbour table differs from the oracle"
    return cl_ref


@pytest.mark.parametrize("name", ["cluster_grid8.txt", "cluster_grid4x16.txt", "cluster_line20.txt"])
def test_goldens(name):
    gd = golden.read(name)
    rows, cols = (int(v) for v in gd["grid"])
    xy = golden.grid_coords(rows, cols)
    cl = acl.acl_cluster(dev(xy), int(gd["C"][0])).cpu().numpy()[0]
    assert np.array_equal(cl, np.array(gd["clusters"], dtype=np.int32))


def test_workloads():
    run_both(synth.attn_tiny().coords)
    run_both(synth.attn_stage1().coords)                  # 8 x 2048
    run_both(synth.attn_stage3().coords)                  # 64 x 328
    for st in synth.sweep_coords(B=16):                   # 2048 / 819 / 328 / 131
        run_both(st)


@pytest.mark.parametrize("N", [1, 2, 7, 8, 9, 63, 64, 65, 100, 517, 1000, 4096, 8192])
def test_sizes_and_ragged_tails(N):
    xy = synth.uniform(77 + N, 2 * N * 3, -3.0, 40.0).reshape(3, N, 2).astype(np.float32)
    run_both(xy, 8, 48)


@pytest.mark.parametrize("C,M", [(1, 4), (3, 9), (4, 64), (8, 8), (8, 64), (8, 128), (16, 96),
                                 (64, 128)])
def test_cluster_sizes(C, M):
    xy = synth.uniform(5 * C + M, 2 * 2 * 700, 0.0, 30.0).reshape(2, 700, 2).astype(np.float32)
    run_both(xy, C, M)


@pytest.mark.parametrize("N,C", [(6000, 1), (8065, 63), (8192, 4), (3000, 5)])
def test_deep_trees_and_largest_warp_nodes(N, C):
    # the levels below the fifth run one warp per node; (8065, 63) gives the largest such
    # node (315 tokens), C = 1 the deepest tree
    xy = synth.uniform(1000 + N + C, 2 * N, -5.0, 70.0).reshape(1, N, 2).astype(np.float32)
    run_both(xy, C, 2 * C if C <= 8 else C)


def test_ties_negative_zero_and_duplicates():
    # exact duplicates, -0.0 vs +0.0, integer lattice: every tie-break path
    rng = np.random.default_rng(0)
    base = rng.integers(0, 6, size=(1, 300, 2)).astype(np.float32)
    base[0, :20] = 0.0
    base[0, 20:40] = -0.0
    run_both(base, 8, 48)
    grid = golden.grid_coords(32, 32)
    run_both(grid, 8, 48)


def test_batch_images_independent():
    xy = synth.attn_stage1(B=3).coords
    full = acl.acl_cluster(dev(xy)).cpu().numpy()
    for b in range(3):
        one = acl.acl_cluster(dev(xy[b:b + 1])).cpu().numpy()
        assert np.array_equal(one[0], full[b])


def test_repeatable_bits():
    xy = dev(synth.attn_stage1(B=2).coords)
    a = acl.acl_cluster(xy)
    b = acl.acl_cluster(xy)
    assert torch.equal(a, b)
    assert torch.equal(acl.acl_neighbors(xy, a), acl.acl_neighbors(xy, b))
