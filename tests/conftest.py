import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


def pytest_sessionstart(session):
    # build the CUDA library and the oracle in-tree if missing or stale (nvcc and gcc are
    # available wherever the tests run; the GPU tests then load the in-tree libacl.so)
    from off_grid_cluster_b200 import build as acl_build
    from oracle import build as oracle_build
    acl_build.build()
    acl_build.build(check=True)
    oracle_build.build()


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Count of the forward outputs whose oracle value is >= 4 in magnitude: a bf16 result
    cannot be within 1e-2 of those, so the parity checks hold them to half a bf16 ulp +
    1e-3 instead (tests/parity.py); every such count is listed here."""
    try:
        from tests.parity import LARGE_OUTPUTS
    except Exception:  # pragma: no cover
        return
    if not LARGE_OUTPUTS:
        return
    n = sum(v[0] for v in LARGE_OUTPUTS.values())
    m = sum(v[1] for v in LARGE_OUTPUTS.values())
    tr = terminalreporter
    tr.write_line(f"forward outputs with |oracle| >= 4 (held to half a bf16 ulp + 1e-3): {n} of {m} "
                  f"checked over {len(LARGE_OUTPUTS)} output checks")
    for key, (k, tot) in sorted(LARGE_OUTPUTS.items()):
        if k:
            tr.write_line(f"  n_large {k:6d} / {tot:9d}  {key}")
