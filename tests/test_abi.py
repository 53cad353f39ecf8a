"""C-ABI checks that need no GPU: the library loads, exports every function the
header declares, and rejects bad arguments on the host before any launch.

Only argument validation runs here (fake but aligned device pointers are never
dereferenced because validation fails first); no kernel is launched.
"""
import ctypes as ct
import os
import re

import pytest

import off_grid_cluster_b200 as acl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "acl.h")

OK, INVALID, CUDA, UNSUPPORTED, WORKSPACE = 0, 1, 2, 3, 4
P = 1 << 20  # a fake, 256-byte-aligned "device" address; never dereferenced in these tests


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(acl_[a-z_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("acl_cluster", "acl_neighbors", "acl_cluster_attn_fwd", "acl_cluster_attn_bwd",
              "acl_cluster_attn_workspace", "acl_knn_table", "acl_knn_gather_fwd",
              "acl_knn_gather_bwd", "acl_knn_gather_workspace", "acl_knn_gather_index",
              "acl_knn_gather_bwd_indexed", "acl_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ct.CDLL(acl.LIB_PATH)
    for n in declared_functions():
        assert hasattr(lib, n), n
    assert set(declared_functions()) == set(acl.SIGNATURES)


def test_check_build_exports_the_same_symbols_and_reports_itself():
    """The check build (ACL_DEVICE_CHECKS: device-side range checks of index inputs) is
    built from the same sources and exports the same ABI; only it reports checks enabled."""
    assert os.path.exists(acl.CHECK_LIB_PATH)
    chk = ct.CDLL(acl.CHECK_LIB_PATH)
    for n in declared_functions():
        assert hasattr(chk, n), n
    chk.acl_device_checks_enabled.restype = ct.c_int
    assert chk.acl_device_checks_enabled() == 1
    assert acl.acl_device_checks_enabled() is False


def test_status_strings_and_version():
    for code in range(7):
        s = acl.acl_status_string(code)
        assert s.startswith("ACL_"), s
    assert "unknown" in acl.acl_status_string(99)
    assert acl.acl_version() >= 10000
    assert acl.acl_launch_count() >= 0


def _lib():
    return acl.lib()


def test_cluster_validation():
    L = _lib()
    assert L.acl_cluster(None, 1, 10, 8, P, None) == INVALID
    assert L.acl_cluster(P, 1, 0, 8, P, None) == INVALID
    assert L.acl_cluster(P, 0, 10, 8, P, None) == INVALID
    assert L.acl_cluster(P, 1, 8193, 8, P, None) == UNSUPPORTED
    assert L.acl_cluster(P, 1, 100, 65, P, None) == UNSUPPORTED
    assert L.acl_cluster(P, 1, 8192, 1, P, None) == UNSUPPORTED   # shared memory limit
    assert L.acl_cluster(P + 4, 1, 10, 8, P, None) == INVALID     # coords not 8-byte aligned


def test_neighbors_validation():
    L = _lib()
    assert L.acl_neighbors(P, P, 1, 100, 8, 44, P, None) == INVALID       # M % C
    assert L.acl_neighbors(P, P, 1, 100, 8, 136, P, None) == UNSUPPORTED  # R > 16
    assert L.acl_neighbors(P, None, 1, 100, 8, 48, P, None) == INVALID


def _attn_fwd(L, **kw):
    a = dict(Q=P, K=P, V=P, xy=P, cl=P, nb=P, bias=P, B=1, N=64, H=4, D=32, C=8, M=48,
             scale=0.1, O=P, lse=P)
    a.update(kw)
    return L.acl_cluster_attn_fwd(a["Q"], a["K"], a["V"], a["xy"], a["cl"], a["nb"], a["bias"],
                                  a["B"], a["N"], a["H"], a["D"], a["C"], a["M"], a["scale"],
                                  a["O"], a["lse"], None)


def test_attention_validation():
    L = _lib()
    assert _attn_fwd(L, D=64) == UNSUPPORTED
    assert _attn_fwd(L, C=4, M=48) == UNSUPPORTED
    assert _attn_fwd(L, M=72) == UNSUPPORTED
    assert _attn_fwd(L, M=44) == INVALID
    assert _attn_fwd(L, Q=None) == INVALID
    assert _attn_fwd(L, O=P + 8) == INVALID        # bf16 tensors need 16-byte alignment
    assert _attn_fwd(L, N=0) == INVALID
    ws = acl.acl_cluster_attn_workspace(2, 100, 4, 8, 48)
    assert ws > 0 and ws % 256 == 0
    assert acl.acl_cluster_attn_workspace(2, 100, 4, 8, 44) == 0
    args = [P] * 7 + [2, 100, 4, 32, 8, 48, ct.c_float(0.1)] + [P] * 7
    assert L.acl_cluster_attn_bwd(*args, P, ws - 1, None) == WORKSPACE
    assert L.acl_cluster_attn_bwd(*args, None, ws, None) == WORKSPACE
    assert L.acl_cluster_attn_bwd(*args, P + 16, ws, None) == WORKSPACE


def test_token_merge_validation():
    L = _lib()
    ws = acl.acl_token_merge_workspace(2, 2048, 128, 32, 819)
    assert ws > 0
    assert acl.acl_token_merge_workspace(2, 2048, 100, 32, 819) == 0
    assert acl.acl_token_merge_workspace(2, 2048, 128, 32, 4096) == 0
    fwd = lambda N=2048, d=128, h=32, k=819, f=P, wsb=ws, out=P: L.acl_token_merge_fwd(
        f, P, 2, N, d, P, P, P, 0.0, h, k, out, P, P, P, P, P, wsb, None)
    assert fwd(f=None) == INVALID
    assert fwd(d=100) == INVALID
    assert fwd(k=0) == INVALID and fwd(k=2049) == INVALID
    assert fwd(h=257) == UNSUPPORTED
    assert fwd(N=16385, k=10) == UNSUPPORTED
    assert fwd(f=P + 2) == INVALID
    assert fwd(wsb=16) == WORKSPACE
    assert fwd(out=None) == INVALID
    bwd = lambda wsb=ws, dw=P: L.acl_token_merge_bwd(P, P, 2, 2048, 128, P, P, P, 0.0, 32, 819,
                                                    P, P, P, P, P, P, dw, P, P, P, P, wsb, None)
    assert bwd(dw=None) == INVALID
    assert bwd(wsb=16) == WORKSPACE


def test_decoder_layer_validation():
    """Every case below is rejected before any launch (the pointers are fake)."""
    L = _lib()
    ws = acl.acl_decoder_layer_workspace(2, 2048, 131, 768, 256, 8)
    assert ws > 0
    assert acl.acl_decoder_layer_workspace(2, 2048, 131, 96, 256, 8) == 0   # d % 128
    assert acl.acl_decoder_layer_workspace(2, 2048, 131, 768, 200, 8) == 0  # D % 128
    fwd = lambda D=256, d=768, N=131, f=P, ref=P, out=P, wo=P: L.acl_decoder_layer_fwd(
        ref, f, 2, 2048, D, P, P, wo, P, P, N, d, P, 64, 64, 8, P, out, P, P, None)
    assert fwd(f=None) == INVALID and fwd(ref=None) == INVALID and fwd(wo=None) == INVALID
    assert fwd(D=200) == INVALID and fwd(d=96) == INVALID
    assert fwd(D=1152) == UNSUPPORTED
    assert fwd(N=16385) == UNSUPPORTED
    assert fwd(f=P + 8) == INVALID
    assert fwd(out=None) == INVALID
    bwd = lambda wsb=ws, w=P, dw=P: L.acl_decoder_layer_bwd(
        P, 2, 2048, 256, P, P, P, P, 131, 768, P, 64, 64, 8, P, P, P, P, P, dw, P, P, P, P, w,
        wsb, None)
    assert bwd(dw=None) == INVALID
    assert bwd(wsb=ws - 1) == WORKSPACE
    assert bwd(w=None) == WORKSPACE
    assert bwd(w=P + 16) == WORKSPACE


def test_token_order_validation():
    L = _lib()
    assert L.acl_token_order(None, 1, 10, 8, 8, P, None) == INVALID
    assert L.acl_token_order(P, 1, 10, 8, 8, None, None) == INVALID
    assert L.acl_token_order(P, 1, 0, 8, 8, P, None) == INVALID
    assert L.acl_token_order(P, 1, 10, 0, 8, P, None) == INVALID
    assert L.acl_token_order(P, 1, 16385, 8, 8, P, None) == UNSUPPORTED
    assert L.acl_token_order(P, 1, 10, 4097, 8, P, None) == UNSUPPORTED
    assert L.acl_token_order(P + 4, 1, 10, 8, 8, P, None) == INVALID


def test_knn_validation():
    L = _lib()
    assert L.acl_knn_table(P, 1, 0, 64, 64, 8, P, None) == INVALID
    assert L.acl_knn_table(P, 1, 100, 64, 64, 17, P, None) == UNSUPPORTED
    assert L.acl_knn_table(P, 1, 16385, 64, 64, 8, P, None) == UNSUPPORTED
    fwd = lambda d=128, K=8, feats=P, out=P: L.acl_knn_gather_fwd(
        P, 1, 10, feats, P, 100, d, P, 64, 64, K, P, out, None)
    assert fwd(d=100) == INVALID
    assert fwd(d=2048) == UNSUPPORTED
    assert fwd(K=17) == UNSUPPORTED
    assert fwd(feats=P + 2) == INVALID
    assert fwd(out=None) == INVALID
    ws = acl.acl_knn_gather_workspace(2, 4096, 2048, 128, 8)
    assert ws > 2 * 4096 * 8 * 4 * 4
    bwd = lambda Q=10, wsb=ws: L.acl_knn_gather_bwd(P, 1, Q, P, P, 100, 128, P, 64, 64, 8, P,
                                                    P, P, P, P, P, wsb, None)
    assert bwd(wsb=16) == WORKSPACE
    assert bwd(Q=70000, wsb=1 << 40) == UNSUPPORTED
    bwdi = lambda Q=10, wsb=ws: L.acl_knn_gather_bwd_indexed(P, 1, Q, P, P, 100, 128, P, 64, 64,
                                                             8, P, P, P, P, P, P, wsb, None)
    assert L.acl_knn_gather_fwd_ex(P, 1, 10, P, P, 100, 128, P, 64, 64, 8, P, 2, P, None) == INVALID
    assert L.acl_knn_gather_bwd_ex(P, 1, 10, P, P, 100, 128, P, 64, 64, 8, P, -1, P, P, P, P,
                                   P, ws, None) == INVALID
    assert L.acl_knn_gather_bwd_indexed_ex(P, 1, 10, P, P, 100, 128, P, 64, 64, 8, P, 7, P, P,
                                           P, P, P, ws, None) == INVALID
    assert L.acl_knn_gather_bwd_ex(P, 1, 10, P, P, 100, 128, P, 64, 64, 8, P, 1, P, P, P, P,
                                   P, 16, None) == WORKSPACE
    assert bwdi(wsb=16) == WORKSPACE
    assert bwdi(Q=70000, wsb=1 << 40) == UNSUPPORTED
    idx = lambda Q=10, d=128, K=8, q=P, t=P, wsb=ws, w=P: L.acl_knn_gather_index(
        q, 1, Q, 100, d, t, 64, 64, K, w, wsb, None)
    assert idx(t=None) == INVALID
    assert idx(q=None) == INVALID
    assert idx(d=100) == INVALID
    assert idx(K=17) == UNSUPPORTED
    assert idx(Q=70000) == UNSUPPORTED
    assert idx(q=P + 4) == INVALID
    assert idx(wsb=16) == WORKSPACE
    assert idx(w=P + 16) == WORKSPACE


def test_workspace_sizes_scale_with_inputs():
    # per-image parts grow linearly with the batch (a small fixed part does not)
    a = acl.acl_cluster_attn_workspace(1, 2048, 4, 8, 48)
    b = acl.acl_cluster_attn_workspace(2, 2048, 4, 8, 48)
    c = acl.acl_cluster_attn_workspace(4, 2048, 4, 8, 48)
    assert b > a and abs((c - b) - 2 * (b - a)) <= 8 * 256
    k1 = acl.acl_knn_gather_workspace(1, 4096, 2048, 128, 8)
    k2 = acl.acl_knn_gather_workspace(1, 4096, 2048, 768, 8)
    assert k2 > k1


def test_binding_rejects_cpu_tensors():
    import torch
    with pytest.raises(ValueError):
        acl.acl_cluster(torch.zeros(1, 10, 2))
