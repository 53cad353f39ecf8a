"""GPU test of acl_cluster_attn_bwd_noalloc, the attention backward for callers that
cannot allocate device memory (it uses the library's own fixed scratch array).

It must give what acl_cluster_attn_bwd gives with a caller workspace, call after call:
both run the same kernels in the same order, so two calls in a row must equal the regular
entry point's results bit for bit.  The file sorts last so that a failure here does not
stop the rest of the suite; it also passes when run alone in a fresh process, where its
first call is the one that looks up the scratch array's address.
"""
import numpy as np
import pytest
import torch

import off_grid_cluster_b200 as acl
import oracle
from off_grid_cluster_b200 import synth
from tests.parity import bf16, dev

pytestmark = pytest.mark.gpu


def _inputs(B, N, H):
    a = synth.attn_stage1(B=B, N=N, H=H)
    cl = oracle.cluster(a.coords, 8)
    nb = oracle.neighbors(a.coords, cl, 48)
    t = dict(Q=bf16(a.q), K=bf16(a.k), V=bf16(a.v), dO=bf16(a.do), xy=dev(a.coords),
             cl=dev(cl), nb=dev(nb), bias=dev(a.bias))
    O, lse = acl.acl_cluster_attn_fwd(t["Q"], t["K"], t["V"], t["xy"], t["cl"], t["nb"], t["bias"],
                                      a.scale)
    return a, t, O, lse


def test_noalloc_matches_workspace_entry_point_twice():
    a, t, O, lse = _inputs(B=4, N=2048, H=4)
    args = (t["Q"], t["K"], t["V"], t["xy"], t["cl"], t["nb"], t["bias"], a.scale, O, t["dO"], lse)
    ref = acl.acl_cluster_attn_bwd(*args)
    for _ in range(2):
        outs = [torch.full_like(x, float("nan")) for x in ref]
        got = acl.acl_cluster_attn_bwd_noalloc(*args, *outs)
        torch.cuda.synchronize()
        for name, g, r in zip(("dQ", "dK", "dV", "dbias"), got, ref):
            assert torch.equal(g, r), f"{name} differs from the workspace entry point"


def test_noalloc_rejects_sizes_beyond_its_scratch():
    B, N, H = 64, 4096, 8
    assert acl.acl_cluster_attn_workspace(B, N, H) > acl.ACL_NOALLOC_ATTN_WS_BYTES
    Q = torch.zeros(B, N, H, 32, dtype=torch.bfloat16, device="cuda")
    xy = torch.zeros(B, N, 2, device="cuda")
    cl = torch.zeros(B, N // 8, 8, dtype=torch.int32, device="cuda")
    nb = torch.zeros(B, N // 8, 48, dtype=torch.int32, device="cuda")
    lse = torch.zeros(B, N, H, device="cuda")
    with pytest.raises(acl.AclError) as err:
        acl.acl_cluster_attn_bwd_noalloc(Q, Q, Q, xy, cl, nb, torch.zeros(H, 3, device="cuda"), 0.1,
                                         Q, Q, lse, Q, Q, Q)
    assert err.value.status == 3  # ACL_ERR_UNSUPPORTED
