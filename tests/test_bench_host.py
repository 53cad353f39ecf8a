"""Host-side logic of the benchmark (no GPU): the algorithmic byte counts that the roofline
fractions divide by, the measured-peak loader, the traffic keying and the argument defaults."""
import os

import bench


def test_step_algorithmic_bytes():
    """The per-call bytes of the step workload (8 images x 2048 tokens, H = 4; Q = 4096,
    d = 128, K = 8 on a 64 x 64 grid), every tensor counted once."""
    by = bench.algorithmic_bytes(8, 2048, 4, 4096, 128, 8, 64, 64)
    B, N, H, Q, d, K = 8, 2048, 4, 4096, 128, 8
    G = N // 8
    meta = 8 + 4 + 4 * 48 * G / N
    assert by["cluster"] == B * N * 12
    assert by["attn_fwd"] == B * N * (H * (3 * 64 + 64 + 4) + meta) + H * 12
    assert by["attn_bwd"] == B * N * (H * (4 * 64 + 4 + 3 * 64) + meta) + 2 * H * 12
    assert by["knn_fwd"] == B * (Q * (8 + 4 * K + 2 * d) + N * (2 * d + 8)) + 4 * d // 32
    assert round(by["attn_bwd"] / 1e6, 3) == 30.212 and round(by["knn_fwd"] / 1e6, 3) == 14.025


def test_merge_bytes():
    b = bench.merge_bytes(8, 2048, 128, 819)
    T, A = 8 * 2048, 8 * 819
    assert b["fwd"] == T * (2 * 128 + 16) + A * (2 * 128 + 12)
    assert b["bwd"] == T * (4 * 128 + 24) + A * (2 * 128 + 8)


def test_peaks_have_both_denominators():
    p = bench.measured_peaks()
    assert p["hbm_gbs"] > 0 and p["bf16_tflops"] > 0 and p["source"]


def test_traffic_is_keyed_to_the_kernels_own_sources(tmp_path):
    names = bench.TRAFFIC_SOURCES["attn_bwd"]
    h = bench.source_hash(names)
    assert len(h) == 16 and h == bench.source_hash(names)
    assert h != bench.source_hash()  # a subset of the sources hashes differently
    for name in names:
        assert os.path.exists(os.path.join(bench.ROOT, "off_grid_cluster_b200", "csrc", name))


def test_argument_defaults():
    a = bench.parse_args([])
    assert (a.gpus, a.impl, a.only) == (1, "acl", None)
    assert a.warmup >= 3 and a.steps >= 1
    assert bench.parse_args(["--only", "configs"]).only == "configs"
