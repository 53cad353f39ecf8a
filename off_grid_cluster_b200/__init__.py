"""off_grid_cluster_b200 -- B200 (sm_100a) local cluster attention and KNN gather.

Python binding of libacl.so (the C ABI declared in include/acl.h).  Every
function here only marshals arguments: it checks shapes, dtypes and devices of
torch tensors, allocates outputs with torch when the caller passes none, and
calls the C entry point of the same name on the current CUDA stream.  All
arithmetic runs in the library's CUDA kernels.  There is no CPU path: the
library is loaded on first use, and if it is missing or fails to load that
first call raises ImportError.  (The seeded input generators in ``synth`` do
not need the library.)
"""
from __future__ import annotations

import ctypes as ct
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# the library to load: the regular build, or another build of the same sources named by
# ACL_LIBRARY (the check build libacl_check.so, whose kernels range-check their index inputs)
LIB_PATH = os.environ.get("ACL_LIBRARY") or os.path.join(_HERE, "libacl.so")
CHECK_LIB_PATH = os.path.join(_HERE, "libacl_check.so")

ACL_OK = 0
_STATUS = {0: "ACL_OK", 1: "ACL_ERR_INVALID_ARG", 2: "ACL_ERR_CUDA", 3: "ACL_ERR_UNSUPPORTED",
           4: "ACL_ERR_WORKSPACE", 5: "ACL_ERR_DEVICE_CHECK", 6: "ACL_ERR_TIMEOUT"}

# exported symbols and their ctypes signatures (kept in step with include/acl.h)
_P, _I, _F, _Z = ct.c_void_p, ct.c_int, ct.c_float, ct.c_size_t
SIGNATURES = {
    "acl_status_string": (ct.c_char_p, [_I]),
    "acl_version": (_I, []),
    "acl_launch_count": (ct.c_uint64, []),
    "acl_cluster": (_I, [_P, _I, _I, _I, _P, _P]),
    "acl_neighbors": (_I, [_P, _P, _I, _I, _I, _I, _P, _P]),
    "acl_cluster_attn_workspace": (_Z, [_I, _I, _I, _I, _I]),
    "acl_cluster_attn_fwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F,
                                  _P, _P, _P]),
    "acl_cluster_attn_fwd_ffma": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F,
                                       _P, _P, _P]),
    "acl_cluster_attn_bwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F,
                                  _P, _P, _P, _P, _P, _P, _P, _P, _Z, _P]),
    "acl_cluster_attn_bwd_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I,
                                          _F, _P, _P, _P, _P, _P, _P, _P, _P]),
    "acl_knn_table": (_I, [_P, _I, _I, _I, _I, _I, _P, _P]),
    "acl_token_order": (_I, [_P, _I, _I, _I, _I, _P, _P]),
    "acl_token_merge_workspace": (_Z, [_I, _I, _I, _I, _I]),
    "acl_token_merge_fwd": (_I, [_P, _P, _I, _I, _I, _P, _P, _P, _F, _I, _I, _P, _P, _P, _P, _P,
                                 _P, _Z, _P]),
    "acl_token_merge_bwd": (_I, [_P, _P, _I, _I, _I, _P, _P, _P, _F, _I, _I, _P, _P, _P, _P, _P,
                                 _P, _P, _P, _P, _P, _P, _Z, _P]),
    "acl_knn_gather_workspace": (_Z, [_I, _I, _I, _I, _I]),
    "acl_decoder_layer_workspace": (_Z, [_I, _I, _I, _I, _I, _I]),
    "acl_device_check": (_I, []),
    "acl_device_checks_enabled": (_I, []),
    "acl_test_set_wait_limit": (_I, [ct.c_longlong]),
    "acl_decoder_layer_fwd": (_I, [_P, _P, _I, _I, _I, _P, _P, _P, _P, _P, _I, _I, _P, _I, _I,
                                   _I, _P, _P, _P, _P, _P]),
    "acl_decoder_layer_bwd": (_I, [_P, _I, _I, _I, _P, _P, _P, _P, _I, _I, _P, _I, _I, _I, _P,
                                   _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _Z, _P]),
    "acl_knn_gather_fwd": (_I, [_P, _I, _I, _P, _P, _I, _I, _P, _I, _I, _I, _P, _P, _P]),
    "acl_knn_gather_bwd": (_I, [_P, _I, _I, _P, _P, _I, _I, _P, _I, _I, _I, _P, _P, _P, _P,
                                _P, _P, _Z, _P]),
    "acl_knn_gather_index": (_I, [_P, _I, _I, _I, _I, _P, _I, _I, _I, _P, _Z, _P]),
    "acl_knn_gather_fwd_ex": (_I, [_P, _I, _I, _P, _P, _I, _I, _P, _I, _I, _I, _P, _I, _P, _P]),
    "acl_knn_gather_bwd_ex": (_I, [_P, _I, _I, _P, _P, _I, _I, _P, _I, _I, _I, _P, _I, _P, _P,
                                   _P, _P, _P, _Z, _P]),
    "acl_knn_gather_bwd_indexed_ex": (_I, [_P, _I, _I, _P, _P, _I, _I, _P, _I, _I, _I, _P, _I,
                                           _P, _P, _P, _P, _P, _Z, _P]),
    "acl_knn_gather_bwd_indexed": (_I, [_P, _I, _I, _P, _P, _I, _I, _P, _I, _I, _I, _P, _P,
                                        _P, _P, _P, _P, _Z, _P]),
}


class AclError(RuntimeError):
    """A libacl call returned a status other than ACL_OK."""

    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {acl_status_string(status)}")


def _load() -> ct.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libacl.so not built at {LIB_PATH}: run `python "
                          f"off_grid_cluster_b200/build.py` (nvcc, sm_100a) first")
    lib = ct.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib: ct.CDLL | None = None


def lib() -> ct.CDLL:
    """The loaded libacl.so (loaded on first use; raises ImportError if absent)."""
    global _lib
    if _lib is None:
        _lib = _load()
    return _lib


def acl_status_string(status: int) -> str:
    return lib().acl_status_string(int(status)).decode()


def acl_version() -> int:
    return int(lib().acl_version())


def acl_launch_count() -> int:
    return int(lib().acl_launch_count())


def _call(name: str, *args) -> None:
    st = getattr(lib(), name)(*args)
    if st != ACL_OK:
        raise AclError(name, st)


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, shape: tuple | None = None) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (the library has no CPU path)")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _out(t, shape, dtype, like: torch.Tensor, name: str) -> torch.Tensor:
    if t is None:
        return torch.empty(shape, dtype=dtype, device=like.device)
    _need(t, name, dtype, shape)
    return t


# ---------------------------------------------------------------- clustering

def acl_cluster(coords: torch.Tensor, C: int = 8, clusters: torch.Tensor | None = None,
                stream=None) -> torch.Tensor:
    """Recursive-median balanced clustering: coords [B,N,2] f32 -> clusters [B,G,C] i32."""
    _need(coords, "coords", torch.float32)
    B, N = coords.shape[:2]
    G = (N + C - 1) // C
    clusters = _out(clusters, (B, G, C), torch.int32, coords, "clusters")
    _call("acl_cluster", _ptr(coords), B, N, C, _ptr(clusters), _stream(stream))
    return clusters


def acl_neighbors(coords: torch.Tensor, clusters: torch.Tensor, M: int = 48,
                  nbr: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Neighbourhood table: the M / C nearest clusters -> nbr [B,G,M] i32."""
    _need(coords, "coords", torch.float32)
    _need(clusters, "clusters", torch.int32)
    B, N = coords.shape[:2]
    G, C = clusters.shape[1:]
    nbr = _out(nbr, (B, G, M), torch.int32, coords, "nbr")
    _call("acl_neighbors", _ptr(coords), _ptr(clusters), B, N, C, M, _ptr(nbr), _stream(stream))
    return nbr


# ---------------------------------------------------------------- attention

def acl_cluster_attn_workspace(B: int, N: int, H: int, C: int = 8, M: int = 48) -> int:
    return int(lib().acl_cluster_attn_workspace(B, N, H, C, M))


def _attn_shapes(Q, K, V, coords, clusters, nbr, bias_coef):
    _need(Q, "Q", torch.bfloat16)
    B, N, H, D = Q.shape
    _need(K, "K", torch.bfloat16, (B, N, H, D))
    _need(V, "V", torch.bfloat16, (B, N, H, D))
    _need(coords, "coords", torch.float32, (B, N, 2))
    _need(clusters, "clusters", torch.int32)
    _need(nbr, "nbr", torch.int32)
    _need(bias_coef, "bias_coef", torch.float32, (H, 3))
    C, M = clusters.shape[2], nbr.shape[2]
    return B, N, H, D, C, M


def acl_cluster_attn_fwd(Q, K, V, coords, clusters, nbr, bias_coef, scale: float | None = None,
                         O=None, lse=None, stream=None):
    """Local cluster attention forward -> (O [B,N,H,D] bf16, lse [B,N,H] f32)."""
    B, N, H, D, C, M = _attn_shapes(Q, K, V, coords, clusters, nbr, bias_coef)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    O = _out(O, (B, N, H, D), torch.bfloat16, Q, "O")
    lse = _out(lse, (B, N, H), torch.float32, Q, "lse")
    _call("acl_cluster_attn_fwd", _ptr(Q), _ptr(K), _ptr(V), _ptr(coords), _ptr(clusters),
          _ptr(nbr), _ptr(bias_coef), B, N, H, D, C, M, scale, _ptr(O), _ptr(lse),
          _stream(stream))
    return O, lse


def acl_cluster_attn_fwd_ffma(Q, K, V, coords, clusters, nbr, bias_coef, scale: float | None = None,
                              O=None, lse=None, stream=None):
    """The forward on the FMA pipes only (the tensor-core kernel's reference variant)."""
    B, N, H, D, C, M = _attn_shapes(Q, K, V, coords, clusters, nbr, bias_coef)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    O = _out(O, (B, N, H, D), torch.bfloat16, Q, "O")
    lse = _out(lse, (B, N, H), torch.float32, Q, "lse")
    _call("acl_cluster_attn_fwd_ffma", _ptr(Q), _ptr(K), _ptr(V), _ptr(coords), _ptr(clusters),
          _ptr(nbr), _ptr(bias_coef), B, N, H, D, C, M, scale, _ptr(O), _ptr(lse),
          _stream(stream))
    return O, lse


def acl_cluster_attn_bwd(Q, K, V, coords, clusters, nbr, bias_coef, scale: float | None,
                         O, dO, lse, dQ=None, dK=None, dV=None, dbias_coef=None,
                         workspace: torch.Tensor | None = None, stream=None):
    """Local cluster attention backward -> (dQ, dK, dV, dbias_coef [H,3] f32)."""
    B, N, H, D, C, M = _attn_shapes(Q, K, V, coords, clusters, nbr, bias_coef)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    _need(O, "O", torch.bfloat16, (B, N, H, D))
    _need(dO, "dO", torch.bfloat16, (B, N, H, D))
    _need(lse, "lse", torch.float32, (B, N, H))
    dQ = _out(dQ, (B, N, H, D), torch.bfloat16, Q, "dQ")
    dK = _out(dK, (B, N, H, D), torch.bfloat16, Q, "dK")
    dV = _out(dV, (B, N, H, D), torch.bfloat16, Q, "dV")
    dbias_coef = _out(dbias_coef, (H, 3), torch.float32, Q, "dbias_coef")
    need = acl_cluster_attn_workspace(B, N, H, C, M)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=Q.device)
    _call("acl_cluster_attn_bwd", _ptr(Q), _ptr(K), _ptr(V), _ptr(coords), _ptr(clusters),
          _ptr(nbr), _ptr(bias_coef), B, N, H, D, C, M, scale, _ptr(O), _ptr(dO), _ptr(lse),
          _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(dbias_coef), _ptr(workspace),
          workspace.numel() * workspace.element_size(), _stream(stream))
    return dQ, dK, dV, dbias_coef


def acl_cluster_attn_bwd_noalloc(Q, K, V, coords, clusters, nbr, bias_coef, scale: float | None,
                                 O, dO, lse, dQ=None, dK=None, dV=None, dbias_coef=None,
                                 stream=None):
    """acl_cluster_attn_bwd with the library's own scratch array instead of a workspace.

    For callers that cannot allocate device scratch.  The outputs are allocated here only
    when not passed in (pass them to allocate nothing).  Raises AclError with
    ACL_ERR_UNSUPPORTED when the sizes need more than ACL_NOALLOC_ATTN_WS_BYTES.
    """
    B, N, H, D, C, M = _attn_shapes(Q, K, V, coords, clusters, nbr, bias_coef)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    _need(dO, "dO", torch.bfloat16, (B, N, H, D))
    _need(lse, "lse", torch.float32, (B, N, H))
    dQ = _out(dQ, (B, N, H, D), torch.bfloat16, Q, "dQ")
    dK = _out(dK, (B, N, H, D), torch.bfloat16, Q, "dK")
    dV = _out(dV, (B, N, H, D), torch.bfloat16, Q, "dV")
    dbias_coef = _out(dbias_coef, (H, 3), torch.float32, Q, "dbias_coef")
    _call("acl_cluster_attn_bwd_noalloc", _ptr(Q), _ptr(K), _ptr(V), _ptr(coords), _ptr(clusters),
          _ptr(nbr), _ptr(bias_coef), B, N, H, D, C, M, scale, _ptr(O), _ptr(dO), _ptr(lse),
          _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(dbias_coef), _stream(stream))
    return dQ, dK, dV, dbias_coef


ACL_NOALLOC_ATTN_WS_BYTES = 4 << 20


# ---------------------------------------------------------------- KNN gather

def acl_knn_table(coords: torch.Tensor, H: int = 64, W: int = 64, K: int = 8,
                  table: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """KNN cache lookup table -> table [B,H,W,K] i32."""
    _need(coords, "coords", torch.float32)
    B, N = coords.shape[:2]
    table = _out(table, (B, H, W, K), torch.int32, coords, "table")
    _call("acl_knn_table", _ptr(coords), B, N, H, W, K, _ptr(table), _stream(stream))
    return table


def acl_token_order(coords: torch.Tensor, H: int, W: int, perm: torch.Tensor | None = None,
                    stream=None) -> torch.Tensor:
    """Token ids of each image in Z-order of their cells on the H x W grid -> [B,N] int32."""
    _need(coords, "coords", torch.float32)
    B, N = coords.shape[:2]
    perm = _out(perm, (B, N), torch.int32, coords, "perm")
    _call("acl_token_order", _ptr(coords), B, N, H, W, _ptr(perm), _stream(stream))
    return perm


def acl_token_merge_workspace(B: int, N: int, d: int, h: int, k: int) -> int:
    return int(lib().acl_token_merge_workspace(B, N, d, h, k))


def _merge_shapes(feats, coords, w1, b1, w2):
    _need(feats, "feats", torch.bfloat16)
    B, N, d = feats.shape
    _need(coords, "coords", torch.float32, (B, N, 2))
    _need(w1, "w1", torch.float32)
    h = w1.shape[1]
    _need(w1, "w1", torch.float32, (d, h))
    _need(b1, "b1", torch.float32, (h,))
    _need(w2, "w2", torch.float32, (h,))
    return B, N, d, h


def acl_token_merge_fwd(feats, coords, w1, b1, w2, b2: float, k: int, workspace=None, stream=None):
    """Token merging -> (scores [B,N] f32, anchors [B,k] i32, assign [B,N] i32,
    merged [B,k,d] bf16, mcoords [B,k,2] f32)."""
    B, N, d, h = _merge_shapes(feats, coords, w1, b1, w2)
    dev = feats.device
    scores = torch.empty((B, N), dtype=torch.float32, device=dev)
    anchors = torch.empty((B, k), dtype=torch.int32, device=dev)
    assign = torch.empty((B, N), dtype=torch.int32, device=dev)
    merged = torch.empty((B, k, d), dtype=torch.bfloat16, device=dev)
    mcoords = torch.empty((B, k, 2), dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = torch.empty(max(acl_token_merge_workspace(B, N, d, h, k), 1),
                                dtype=torch.uint8, device=dev)
    _call("acl_token_merge_fwd", _ptr(feats), _ptr(coords), B, N, d, _ptr(w1), _ptr(b1),
          _ptr(w2), float(b2), h, k, _ptr(scores), _ptr(anchors), _ptr(assign), _ptr(merged),
          _ptr(mcoords), _ptr(workspace), workspace.numel(), _stream(stream))
    return scores, anchors, assign, merged, mcoords


def acl_token_merge_bwd(feats, coords, w1, b1, w2, b2: float, k: int, scores, assign, dmerged,
                        dmcoords, workspace=None, stream=None):
    """Token merging backward -> (dfeats [B,N,d] bf16, dcoords [B,N,2], dW1 [d,h], db1 [h],
    dw2 [h], db2 [1] f32)."""
    B, N, d, h = _merge_shapes(feats, coords, w1, b1, w2)
    dev = feats.device
    _need(dmerged, "dmerged", torch.bfloat16, (B, k, d))
    _need(dmcoords, "dmcoords", torch.float32, (B, k, 2))
    dfeats = torch.empty_like(feats)
    dcoords = torch.empty_like(coords)
    dw1, db1, dw2 = torch.empty_like(w1), torch.empty_like(b1), torch.empty_like(w2)
    db2 = torch.empty((1,), dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = torch.empty(max(acl_token_merge_workspace(B, N, d, h, k), 1),
                                dtype=torch.uint8, device=dev)
    _call("acl_token_merge_bwd", _ptr(feats), _ptr(coords), B, N, d, _ptr(w1), _ptr(b1),
          _ptr(w2), float(b2), h, k, _ptr(scores), _ptr(assign), _ptr(dmerged), _ptr(dmcoords),
          _ptr(dfeats), _ptr(dcoords), _ptr(dw1), _ptr(db1), _ptr(dw2), _ptr(db2),
          _ptr(workspace), workspace.numel(), _stream(stream))
    return dfeats, dcoords, dw1, db1, dw2, db2


def acl_knn_gather_workspace(B: int, Q: int, N: int, d: int, K: int = 8) -> int:
    return int(lib().acl_knn_gather_workspace(B, Q, N, d, K))


def _gather_shapes(queries, feats, coords, table, p):
    _need(queries, "queries", torch.float32)
    B, Q = queries.shape[:2]
    _need(feats, "feats", torch.bfloat16)
    N, d = feats.shape[1:]
    _need(coords, "coords", torch.float32, (B, N, 2))
    _need(table, "table", torch.int32)
    H, W, K = table.shape[1:]
    _need(p, "p", torch.float32, (d // 32,))
    return B, Q, N, d, H, W, K


ACL_KNN_EXP, ACL_KNN_INVPOW = 0, 1  # weight kernels: softmax(-p d), d^-p / sum d^-p


def acl_device_check() -> None:
    """Synchronise the device; raise AclError if a bounded device-side wait gave up
    (ACL_ERR_TIMEOUT) or, in the check build, an index input was out of range
    (ACL_ERR_DEVICE_CHECK)."""
    _call("acl_device_check")


def acl_device_checks_enabled() -> bool:
    """True in the check build of the library (device-side range checks)."""
    return bool(lib().acl_device_checks_enabled())


def acl_test_set_wait_limit(cycles: int) -> None:
    """Test hook: give-up limit (SM clocks) of the tensor-core GEMM's main-loop waits; a
    negative value restores the default."""
    _call("acl_test_set_wait_limit", int(cycles))


def acl_decoder_layer_workspace(B: int, Q: int, N: int, d: int, D: int, K: int = 8) -> int:
    return int(lib().acl_decoder_layer_workspace(B, Q, N, d, D, K))


def _decoder_shapes(f_in, w_off, w_o, feats, coords, table, p):
    _need(f_in, "f_in", torch.float32)
    B, Q, D = f_in.shape
    _need(feats, "feats", torch.bfloat16)
    N, d = feats.shape[1:]
    _need(coords, "coords", torch.float32, (B, N, 2))
    _need(table, "table", torch.int32)
    H, W, K = table.shape[1:]
    _need(p, "p", torch.float32, (d // 32,))
    _need(w_off, "w_off", torch.float32, (D, 2))
    _need(w_o, "w_o", torch.bfloat16, (d, D))
    return B, Q, D, N, d, H, W, K


def acl_decoder_layer_fwd(ref, f_in, w_off, b_off, w_o, feats, coords, table, p, f_out=None,
                          stream=None):
    """One decoder layer -> (q [B,Q,2] f32, v [B,Q,d] bf16, f_out [B,Q,D] f32)."""
    B, Q, D, N, d, H, W, K = _decoder_shapes(f_in, w_off, w_o, feats, coords, table, p)
    _need(ref, "ref", torch.float32, (B, Q, 2))
    _need(b_off, "b_off", torch.float32, (2,))
    dev = f_in.device
    q = torch.empty((B, Q, 2), dtype=torch.float32, device=dev)
    v = torch.empty((B, Q, d), dtype=torch.bfloat16, device=dev)
    f_out = _out(f_out, (B, Q, D), torch.float32, f_in, "f_out")
    _call("acl_decoder_layer_fwd", _ptr(ref), _ptr(f_in), B, Q, D, _ptr(w_off), _ptr(b_off),
          _ptr(w_o), _ptr(feats), _ptr(coords), N, d, _ptr(table), H, W, K, _ptr(p), _ptr(q),
          _ptr(v), _ptr(f_out), _stream(stream))
    return q, v, f_out


def acl_decoder_layer_bwd(f_in, w_off, w_o, feats, coords, table, p, q, v, df_out, df_in=None,
                          workspace=None, stream=None):
    """Decoder layer backward -> (df_in [B,Q,D] f32, dW_off [D,2], db_off [2], dW_o [d,D] f32,
    dfeats [B,N,d] bf16, dp [d/32] f32)."""
    B, Q, D, N, d, H, W, K = _decoder_shapes(f_in, w_off, w_o, feats, coords, table, p)
    _need(q, "q", torch.float32, (B, Q, 2))
    _need(v, "v", torch.bfloat16, (B, Q, d))
    _need(df_out, "df_out", torch.float32, (B, Q, D))
    dev = f_in.device
    df_in = _out(df_in, (B, Q, D), torch.float32, f_in, "df_in")
    dw_off = torch.empty((D, 2), dtype=torch.float32, device=dev)
    db_off = torch.empty((2,), dtype=torch.float32, device=dev)
    dw_o = torch.empty((d, D), dtype=torch.float32, device=dev)
    dfeats = torch.empty_like(feats)
    dp = torch.empty((d // 32,), dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = torch.empty(max(acl_decoder_layer_workspace(B, Q, N, d, D, K), 1),
                                dtype=torch.uint8, device=dev)
    _call("acl_decoder_layer_bwd", _ptr(f_in), B, Q, D, _ptr(w_off), _ptr(w_o), _ptr(feats),
          _ptr(coords), N, d, _ptr(table), H, W, K, _ptr(p), _ptr(q), _ptr(v), _ptr(df_out),
          _ptr(df_in), _ptr(dw_off), _ptr(db_off), _ptr(dw_o), _ptr(dfeats), _ptr(dp),
          _ptr(workspace), workspace.numel(), _stream(stream))
    return df_in, dw_off, db_off, dw_o, dfeats, dp


def acl_knn_gather_fwd(queries, feats, coords, table, p, out=None, stream=None,
                       kind: int = ACL_KNN_EXP):
    """KNN distance-weighted gather forward -> out [B,Q,d] bf16."""
    B, Q, N, d, H, W, K = _gather_shapes(queries, feats, coords, table, p)
    out = _out(out, (B, Q, d), torch.bfloat16, feats, "out")
    _call("acl_knn_gather_fwd_ex", _ptr(queries), B, Q, _ptr(feats), _ptr(coords), N, d,
          _ptr(table), H, W, K, _ptr(p), int(kind), _ptr(out), _stream(stream))
    return out


def acl_knn_gather_index(queries, table, N: int, d: int, workspace: torch.Tensor, stream=None):
    """Build the backward's inverse index (from the queries' cells and the table) in
    `workspace` (at least acl_knn_gather_workspace(B, Q, N, d, K) bytes)."""
    _need(queries, "queries", torch.float32)
    B, Q = queries.shape[:2]
    _need(table, "table", torch.int32)
    H, W, K = table.shape[1:]
    _call("acl_knn_gather_index", _ptr(queries), B, Q, N, d, _ptr(table), H, W, K,
          _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    return workspace


def acl_knn_gather_bwd_indexed(queries, feats, coords, table, p, dOut, workspace: torch.Tensor,
                               dfeats=None, dqueries=None, dp=None, stream=None,
                               kind: int = ACL_KNN_EXP):
    """acl_knn_gather_bwd reading the inverse index that acl_knn_gather_index wrote into
    `workspace` -> (dfeats, dqueries, dp)."""
    return _gather_bwd("acl_knn_gather_bwd_indexed_ex", queries, feats, coords, table, p, dOut,
                       dfeats, dqueries, dp, workspace, stream, kind)


def acl_knn_gather_bwd(queries, feats, coords, table, p, dOut, dfeats=None, dqueries=None,
                       dp=None, workspace: torch.Tensor | None = None, stream=None,
                       kind: int = ACL_KNN_EXP):
    """KNN gather backward -> (dfeats [B,N,d] bf16, dqueries [B,Q,2] f32, dp [d/32] f32)."""
    return _gather_bwd("acl_knn_gather_bwd_ex", queries, feats, coords, table, p, dOut, dfeats,
                       dqueries, dp, workspace, stream, kind)


def _gather_bwd(fn, queries, feats, coords, table, p, dOut, dfeats, dqueries, dp, workspace,
                stream, kind):
    B, Q, N, d, H, W, K = _gather_shapes(queries, feats, coords, table, p)
    _need(dOut, "dOut", torch.bfloat16, (B, Q, d))
    dfeats = _out(dfeats, (B, N, d), torch.bfloat16, feats, "dfeats")
    dqueries = _out(dqueries, (B, Q, 2), torch.float32, feats, "dqueries")
    dp = _out(dp, (d // 32,), torch.float32, feats, "dp")
    need = acl_knn_gather_workspace(B, Q, N, d, K)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=feats.device)
    _call(fn, _ptr(queries), B, Q, _ptr(feats), _ptr(coords), N, d,
          _ptr(table), H, W, K, _ptr(p), int(kind), _ptr(dOut), _ptr(dfeats), _ptr(dqueries),
          _ptr(dp),
          _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    return dfeats, dqueries, dp


__all__ = [n for n in list(globals()) if n.startswith("acl_")] + ["AclError", "lib", "LIB_PATH"]
