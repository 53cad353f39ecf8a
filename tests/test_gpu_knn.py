"""GPU parity of acl_knn_table (bit-exact) and acl_knn_gather_fwd / _bwd with the oracle."""
import numpy as np
import pytest
import torch

import off_grid_cluster_b200 as acl
import oracle
from off_grid_cluster_b200 import synth
from tests.parity import bf16, check_fwd, check_grad, dev, host

pytestmark = pytest.mark.gpu


def table_both(xy: np.ndarray, GH: int, GW: int, K: int) -> np.ndarray:
    ref = oracle.knn_table(xy, GH, GW, K)
    got = acl.acl_knn_table(dev(xy), GH, GW, K).cpu().numpy()
    assert np.array_equal(got, ref), f"table differs ({np.sum(got != ref)} entries)"
    return ref


def gather_both(kb: synth.KnnBatch, bwd: bool = True, kind: int = acl.ACL_KNN_EXP):
    table = table_both(kb.coords, kb.GH, kb.GW, kb.K)
    out_ref = oracle.knn_fwd(kb.queries, kb.feats, kb.coords, table, kb.p, kind=kind)
    q, f, xy, tt, p = dev(kb.queries), bf16(kb.feats), dev(kb.coords), dev(table), dev(kb.p)
    out = acl.acl_knn_gather_fwd(q, f, xy, tt, p, kind=kind)
    stats = check_fwd(host(out), out_ref, "out")
    if bwd:
        dF_r, dq_r, dp_r = oracle.knn_bwd(kb.queries, kb.feats, kb.coords, table, kb.p, kb.dout,
                                          kind=kind)
        dF, dq, dp = acl.acl_knn_gather_bwd(q, f, xy, tt, p, bf16(kb.dout), kind=kind)
        stats["dF"] = check_grad(host(dF), dF_r, "dfeats")
        stats["dq"] = check_grad(host(dq), dq_r, "dqueries")
        stats["dp"] = check_grad(host(dp), dp_r, "dp")
    return stats


def test_tables_of_the_decoder_stages():
    for st in synth.sweep_coords(B=16, wid=synth.WORKLOAD_ID["decoder"]):
        table_both(st, 64, 64, 8)


@pytest.mark.parametrize("N,GH,GW,K", [(1, 8, 8, 8), (5, 16, 16, 8), (7, 9, 13, 16), (300, 64, 64, 1),
                                       (300, 64, 64, 2), (300, 50, 70, 5), (2048, 64, 64, 16),
                                       (16384, 64, 64, 8), (64, 256, 256, 8)])
def test_table_sizes(N, GH, GW, K):
    xy = synth.uniform(N + 3 * K + GH, 2 * N * 2, -1.0, float(max(GH, GW)) + 1.0)
    table_both(xy.reshape(2, N, 2).astype(np.float32), GH, GW, K)


def test_table_ties_and_out_of_grid():
    rng = np.random.default_rng(1)
    xy = rng.integers(-3, 20, size=(2, 400, 2)).astype(np.float32) + 0.5   # duplicates, outside
    xy[0, :10] = 0.0
    xy[1, :10] = -0.0
    table_both(xy, 16, 16, 8)


def test_gather_step_workload():
    # the benchmark workload's gather: 8 images x 4096 queries over 2048 tokens, d = 128
    sb = synth.step_batch()
    gather_both(sb.knn)


@pytest.mark.parametrize("stage", [0, 1, 2, 3])
def test_gather_decoder_stage(stage):
    gather_both(synth.knn_decoder(B=16)[stage])


@pytest.mark.parametrize("d,K", [(32, 8), (64, 1), (96, 8), (160, 16), (288, 3), (1024, 8)])
def test_gather_shapes(d, K):
    xy = synth.sweep_coords(B=2)[1]
    kb = synth.knn_batch(xy, d, K=K)
    gather_both(kb)


def test_gather_fewer_tokens_than_k_and_far_queries():
    xy = synth.sweep_coords(B=2)[3][:, :5]                   # 5 tokens, K = 8
    kb = synth.knn_batch(np.ascontiguousarray(xy), 64)
    kb.queries[:, :64] *= np.float32(-1.0)                   # outside the grid
    kb.queries[:, 64:128] += np.float32(100.0)
    gather_both(kb)


def test_gather_temperature_limits():
    xy = synth.sweep_coords(B=1)[0]
    kb = synth.knn_batch(xy, 128)
    kb.p = np.zeros_like(kb.p)                               # plain mean
    gather_both(kb)
    kb.p = np.full_like(kb.p, 60.0)                          # near one-hot
    gather_both(kb, bwd=False)


def test_gather_no_queries():
    xy = synth.sweep_coords(B=2)[2]
    kb = synth.knn_batch(xy, 64)
    table = acl.acl_knn_table(dev(xy))
    q = torch.zeros(2, 0, 2, device="cuda")
    f = bf16(kb.feats)
    out = acl.acl_knn_gather_fwd(q, f, dev(xy), table, dev(kb.p))
    assert out.shape == (2, 0, 64)
    dF0 = torch.full_like(f, 7.0)
    dF, dq, dp = acl.acl_knn_gather_bwd(q, f, dev(xy), table, dev(kb.p),
                                        torch.zeros(2, 0, 64, dtype=torch.bfloat16, device="cuda"),
                                        dfeats=dF0)
    assert torch.count_nonzero(dF) == 0 and torch.count_nonzero(dp) == 0


def test_bwd_deterministic_and_overwrites():
    sb = synth.step_batch(B=2)
    kb = sb.knn
    xy = dev(kb.coords)
    table = acl.acl_knn_table(xy)
    q, f, p, g = dev(kb.queries), bf16(kb.feats), dev(kb.p), bf16(kb.dout)
    ws = torch.full((acl.acl_knn_gather_workspace(2, kb.Q, kb.N, kb.d, 8),), 0x55,
                    dtype=torch.uint8, device="cuda")
    r1 = acl.acl_knn_gather_bwd(q, f, xy, table, p, g, workspace=ws)
    outs = [torch.full_like(t, float("nan")) for t in r1]
    r2 = acl.acl_knn_gather_bwd(q, f, xy, table, p, g, *outs, workspace=ws)
    for x, y in zip(r1, r2):
        assert torch.equal(x, y)


def test_repeated_ids_beyond_16_bit_counts():
    """A hand-built table whose rows repeat token ids: every row lists token 0 six times, so
    token 0 collects 6 Q = 72000 (query, slot) entries in one image, more than a 16-bit count
    holds.  The inverse index and the token pass must still sum every entry once."""
    rng = np.random.default_rng(5)
    B, Q, N, d, K = 1, 12000, 16, 32, 8
    xy = np.stack([rng.uniform(0, 64, N), rng.uniform(0, 64, N)], -1)[None].astype(np.float32)
    queries = rng.uniform(0, 64, (B, Q, 2)).astype(np.float32)
    feats = synth.round_bf16(rng.standard_normal((B, N, d)).astype(np.float32))
    dout = synth.round_bf16(rng.standard_normal((B, Q, d)).astype(np.float32))
    p = np.array([1.5], np.float32)
    table = np.empty((B, 64, 64, K), np.int32)
    table[..., :6] = 0
    table[..., 6] = 1 + (np.arange(64 * 64).reshape(64, 64) % (N - 1))
    table[..., 7] = -1                                    # and one empty slot per row
    q, f, xyd, tt, pd = dev(queries), bf16(feats), dev(xy), dev(table), dev(p)
    check_fwd(host(acl.acl_knn_gather_fwd(q, f, xyd, tt, pd)),
              oracle.knn_fwd(queries, feats, xy, table, p), "out")
    dF_r, dq_r, dp_r = oracle.knn_bwd(queries, feats, xy, table, p, dout)
    dF, dq, dp = acl.acl_knn_gather_bwd(q, f, xyd, tt, pd, bf16(dout))
    check_grad(host(dF), dF_r, "dfeats")
    check_grad(host(dq), dq_r, "dqueries")
    check_grad(host(dp), dp_r, "dp")


@pytest.mark.parametrize("N,Q,K", [(1024, 1001, 8), (1025, 1001, 8), (700, 37, 5), (64, 145, 1)])
def test_gather_union_tiles_ragged_and_scattered(N, Q, K):
    """Images of at most 1024 tokens take the tensor-core union kernels, over tiles of 16
    consecutive queries: ragged last tiles (Q % 16 != 0), queries in random order so that a
    tile lists up to 16 x K distinct tokens, the 1024-token boundary (1025 takes the FMA
    kernels), K < 8, both weight kernels, p = 0, and a bit-identical repeated backward."""
    rng = np.random.default_rng(7 * N + Q)
    B, d = 2, 96
    xy = rng.uniform(0, 64, (B, N, 2)).astype(np.float32)
    queries = rng.uniform(-1, 65, (B, Q, 2)).astype(np.float32)
    feats = synth.round_bf16(rng.standard_normal((B, N, d)).astype(np.float32))
    dout = synth.round_bf16(rng.standard_normal((B, Q, d)).astype(np.float32))
    p = rng.uniform(0.5, 4.0, d // 32).astype(np.float32)
    kb = synth.KnnBatch(queries, xy, feats, dout, p, 64, 64, K)
    gather_both(kb)
    gather_both(kb, kind=acl.ACL_KNN_INVPOW)
    kb.p = np.zeros_like(kb.p)                               # plain mean
    gather_both(kb)
    kb.p = p
    table = acl.acl_knn_table(dev(xy), 64, 64, K)
    args = (dev(queries), bf16(feats), dev(xy), table, dev(p), bf16(dout))
    r1 = acl.acl_knn_gather_bwd(*args)
    r2 = acl.acl_knn_gather_bwd(*args)
    for x, y in zip(r1, r2):
        assert torch.equal(x, y)


def test_staged_backward_matches_one_call():
    """Index built on a side stream, then the indexed backward: bit-identical results."""
    sb = synth.step_batch(B=2)
    kb = sb.knn
    xy = dev(kb.coords)
    table = acl.acl_knn_table(xy)
    q, f, p, g = dev(kb.queries), bf16(kb.feats), dev(kb.p), bf16(kb.dout)
    need = acl.acl_knn_gather_workspace(2, kb.Q, kb.N, kb.d, 8)
    r1 = acl.acl_knn_gather_bwd(q, f, xy, table, p, g)
    ws = torch.full((need,), 0xAB, dtype=torch.uint8, device="cuda")
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    acl.acl_knn_gather_index(q, table, kb.N, kb.d, ws, stream=side)
    torch.cuda.current_stream().wait_stream(side)
    r2 = acl.acl_knn_gather_bwd_indexed(q, f, xy, table, p, g, ws)
    for x, y in zip(r1, r2):
        assert torch.equal(x, y)


# ------------------------------------------------------------------ inverse-power kernel

INV = acl.ACL_KNN_INVPOW


def test_invpow_step_workload():
    gather_both(synth.step_batch(B=2).knn, kind=INV)


@pytest.mark.parametrize("stage", [0, 3])
def test_invpow_decoder_stage(stage):
    gather_both(synth.knn_decoder(B=16)[stage], kind=INV)


@pytest.mark.parametrize("d,K", [(32, 8), (96, 8), (160, 16), (288, 3)])
def test_invpow_shapes(d, K):
    xy = synth.sweep_coords(B=2)[1]
    gather_both(synth.knn_batch(xy, d, K=K), kind=INV)


def test_invpow_queries_on_tokens_and_temperature_limits():
    xy = synth.sweep_coords(B=1)[1]
    kb = synth.knn_batch(xy, 128)
    kb.queries[:, :300] = kb.coords[:, :300]            # d_min = 0: the d -> 0 limit
    gather_both(kb, kind=INV)
    kb.p = np.zeros_like(kb.p)                           # plain mean
    gather_both(kb, kind=INV)
    kb.p = np.full_like(kb.p, 40.0)                      # near one-hot
    gather_both(kb, bwd=False, kind=INV)


def test_invpow_staged_backward_matches_one_call():
    kb = synth.step_batch(B=2).knn
    xy = dev(kb.coords)
    table = acl.acl_knn_table(xy)
    q, f, p, g = dev(kb.queries), bf16(kb.feats), dev(kb.p), bf16(kb.dout)
    r1 = acl.acl_knn_gather_bwd(q, f, xy, table, p, g, kind=INV)
    ws = torch.empty((acl.acl_knn_gather_workspace(2, kb.Q, kb.N, kb.d, 8),), dtype=torch.uint8,
                     device="cuda")
    acl.acl_knn_gather_index(q, table, kb.N, kb.d, ws)
    r2 = acl.acl_knn_gather_bwd_indexed(q, f, xy, table, p, g, ws, kind=INV)
    for x, y in zip(r1, r2):
        assert torch.equal(x, y)
