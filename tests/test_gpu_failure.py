"""Failure paths of the library, exercised without faulting the GPU.

* Bounded waits: the tensor-core GEMM's main-loop mbarrier waits are given a zero budget
  through a test hook, so they give up; the kernel stops issuing MMAs, still waits (with
  the default budget) for the MMAs in flight, frees its tensor memory and leaves zero
  outputs; acl_device_check reports ACL_ERR_TIMEOUT and the context stays usable.
* Device-side range checks: the check build (libacl_check.so) runs, in a child process,
  cases with out-of-range token ids that acl_device_check must report as
  ACL_ERR_DEVICE_CHECK (tests/check_build_case.py)."""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import off_grid_cluster_b200 as acl
import oracle
from off_grid_cluster_b200 import synth
from tests.parity import dev

pytestmark = pytest.mark.gpu

TIMEOUT = 6
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _decoder_case(d=256, D=256, B=2):
    """One decoder layer over a 64 x 64 grid (d = 256: four 64-deep k-tiles in the GEMM, so
    its main loop waits on earlier stages)."""
    xy = synth.sweep_coords(B=B)[1]
    kb = synth.knn_batch(xy, d)
    rng = np.random.default_rng(3)
    f0 = rng.normal(size=(B, kb.Q, D)).astype(np.float32)
    w_off = (rng.normal(size=(D, 2)) / np.sqrt(D)).astype(np.float32)
    b_off = np.zeros(2, np.float32)
    w_o = synth.round_bf16(rng.normal(size=(d, D)) / np.sqrt(d))
    table = acl.acl_knn_table(dev(kb.coords), 64, 64, 8)
    args = (dev(kb.queries), dev(f0), dev(w_off), dev(b_off), dev(w_o, torch.bfloat16),
            dev(kb.feats, torch.bfloat16), dev(kb.coords), table, dev(kb.p))
    return args, (kb, f0, w_off, b_off, w_o, table)


def test_gemm_waits_that_run_out_report_timeout_and_leave_the_context_usable():
    args, (kb, f0, w_off, b_off, w_o, table) = _decoder_case()
    acl.acl_device_check()  # nothing pending
    acl.acl_test_set_wait_limit(0)
    try:
        q, v, f_out = acl.acl_decoder_layer_fwd(*args)
        with pytest.raises(acl.AclError) as err:
            acl.acl_device_check()
        assert err.value.status == TIMEOUT
        # the GEMM's output is zero: f_out = f_in + 0
        assert torch.equal(f_out, args[1])
    finally:
        acl.acl_test_set_wait_limit(-1)
    # default budget again: the same call completes and matches the oracle
    q, v, f_out = acl.acl_decoder_layer_fwd(*args)
    acl.acl_device_check()
    q_h = q.cpu().numpy()
    _, _, f_ref = oracle.decoder_layer_fwd(kb.queries, f0, w_off, b_off, kb.feats, kb.coords,
                                           table.cpu().numpy(), kb.p, w_o, q=q_h)
    assert np.abs(f_out.double().cpu().numpy() - f_ref).max() <= 1e-2


def test_check_build_reports_out_of_range_ids():
    assert os.path.exists(acl.CHECK_LIB_PATH), "check build missing (build(check=True))"
    env = dict(os.environ, ACL_LIBRARY=acl.CHECK_LIB_PATH, PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "check_build_case.py")], env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.count("ACL_ERR_DEVICE_CHECK") == 3, r.stdout


def test_regular_build_treats_out_of_range_ids_as_empty_without_a_flag():
    a = synth.attn_tiny()
    cl = oracle.cluster(a.coords)
    nb = oracle.neighbors(a.coords, cl)
    N = a.coords.shape[1]
    bad = nb.copy()
    bad[0, 0, 5] = N + 3
    ref_nb = nb.copy()
    ref_nb[0, 0, 5] = -1
    bf = torch.bfloat16
    O, _ = acl.acl_cluster_attn_fwd(dev(a.q, bf), dev(a.k, bf), dev(a.v, bf), dev(a.coords), dev(cl),
                                    dev(bad), dev(a.bias), a.scale)
    acl.acl_device_check()  # the regular build records nothing
    o_ref, _ = oracle.attn_fwd(a.q, a.k, a.v, a.coords, cl, ref_nb, a.bias, a.scale)
    assert np.abs(O.double().cpu().numpy() - o_ref).max() <= 1e-2
