"""Run by tests/test_gpu_failure.py in a child process whose ACL_LIBRARY names the check build
(libacl_check.so): valid inputs match the oracle and leave no device-check flag; a token id
outside [-1, N) in a neighbour table, a KNN table and a cluster list is treated as an empty
slot, as in the regular build, and reported by acl_device_check as ACL_ERR_DEVICE_CHECK.
Prints one line per case and exits 0 when every case behaved so."""
import sys

import numpy as np
import torch

import off_grid_cluster_b200 as acl
import oracle
from off_grid_cluster_b200 import synth

DEVICE_CHECK = 5


def device_status() -> int:
    try:
        acl.acl_device_check()
        return 0
    except acl.AclError as e:
        return e.status


def main() -> int:
    assert acl.acl_device_checks_enabled(), "not the check build"
    T = lambda x, dt=None: torch.from_numpy(np.ascontiguousarray(x)).to(device="cuda", dtype=dt)
    bf = torch.bfloat16
    a = synth.attn_tiny()
    cl_ref = oracle.cluster(a.coords)
    nb_ref = oracle.neighbors(a.coords, cl_ref)
    xy = T(a.coords)
    cl = acl.acl_cluster(xy)
    nb = acl.acl_neighbors(xy, cl)
    assert np.array_equal(cl.cpu().numpy(), cl_ref) and np.array_equal(nb.cpu().numpy(), nb_ref)
    Q, K, V = T(a.q, bf), T(a.k, bf), T(a.v, bf)
    O, lse = acl.acl_cluster_attn_fwd(Q, K, V, xy, cl, nb, T(a.bias), a.scale)
    o_ref, _ = oracle.attn_fwd(a.q, a.k, a.v, a.coords, cl_ref, nb_ref, a.bias, a.scale)
    assert np.abs(O.float().cpu().numpy() - o_ref).max() <= 1e-2
    assert device_status() == 0, "valid inputs raised a device check"
    print("valid attention inputs: no flag")

    # a neighbour-table entry beyond N: an empty slot in the result, a flag on the device
    N = a.coords.shape[1]
    bad = nb_ref.copy()
    bad[0, 0, 5] = N + 3
    ref_nb = nb_ref.copy()
    ref_nb[0, 0, 5] = -1
    O2, _ = acl.acl_cluster_attn_fwd(Q, K, V, xy, cl, T(bad), T(a.bias), a.scale)
    o2_ref, _ = oracle.attn_fwd(a.q, a.k, a.v, a.coords, cl_ref, ref_nb, a.bias, a.scale)
    assert np.abs(O2.float().cpu().numpy() - o2_ref).max() <= 1e-2
    assert device_status() == DEVICE_CHECK, "out-of-range neighbour id not reported"
    print("neighbour id N + 3: treated as empty, ACL_ERR_DEVICE_CHECK")

    # a KNN-table entry below -1
    kb = synth.knn_batch(a.coords, 64, gh=16, gw=16)
    table = oracle.knn_table(kb.coords, 16, 16, 8)
    q, f, p = T(kb.queries), T(kb.feats, bf), T(kb.p)
    out = acl.acl_knn_gather_fwd(q, f, xy, T(table), p)
    assert np.abs(out.float().cpu().numpy() - oracle.knn_fwd(kb.queries, kb.feats, kb.coords, table, kb.p)).max() <= 1e-2
    assert device_status() == 0, "valid table raised a device check"
    tbad = table.copy()
    tbad[0, 3, 4, 2] = -7
    tref = table.copy()
    tref[0, 3, 4, 2] = -1
    out2 = acl.acl_knn_gather_fwd(q, f, xy, T(tbad), p)
    ref2 = oracle.knn_fwd(kb.queries, kb.feats, kb.coords, tref, kb.p)
    assert np.abs(out2.float().cpu().numpy() - ref2).max() <= 1e-2
    assert device_status() == DEVICE_CHECK, "out-of-range table id not reported"
    print("KNN table id -7: treated as empty, ACL_ERR_DEVICE_CHECK")

    # a cluster-list entry beyond N (read by the neighbour-table build)
    cbad = cl_ref.copy()
    cbad[0, 1, 0] = N + 100
    acl.acl_neighbors(xy, T(cbad))
    assert device_status() == DEVICE_CHECK, "out-of-range cluster id not reported"
    print("cluster id N + 100: ACL_ERR_DEVICE_CHECK")
    assert device_status() == 0, "flags not cleared"
    return 0


if __name__ == "__main__":
    sys.exit(main())
