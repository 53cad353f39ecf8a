"""Host-side logic of the benchmark (no GPU): the algorithmic byte counts that the roofline
fractions divide by, the measured-peak loader, the DRAM-traffic summary keying, the clock
record and the argument defaults."""
import os

import bench


def test_attention_algorithmic_bytes():
    """Per (token, head): fwd Q, K, V, O + lse = 260 B, bwd Q, K, V, O, dO, lse + dQ, dK, dV =
    516 B; 72 B per token of coordinates, cluster list and neighbour-table share."""
    by = bench.attn_bytes(16, 328, 16)
    assert by["attn_fwd"] == 16 * 328 * (16 * (4 * 64 + 4) + 72)
    assert by["attn_bwd"] == 16 * 328 * (16 * (6 * 64 + 4 + 2 * 64) + 72)
    # the stage-1 layer of 8 images: 35.0 MB for the backward
    assert round(bench.attn_bytes(8, 2048, 4)["attn_bwd"] / 1e6, 1) == 35.0


def test_gather_algorithmic_bytes():
    B, Q, N, d, K = 16, 4096, 131, 768, 8
    by = bench.knn_bytes(B, Q, N, d, K)
    assert by["knn_fwd"] == B * (Q * (8 + 4 * K + 2 * d) + N * (2 * d + 8))
    assert by["knn_bwd"] == B * (Q * (8 + 4 * K + 8 + 2 * d) + N * (2 * d + 8 + 2 * d))
    tb = bench.table_bytes(16, 2048)
    assert tb["cluster"] == 16 * 2048 * 12 and tb["knn_table"] == 16 * (2048 * 8 + 64 * 64 * 8 * 4)


def test_merge_bytes():
    b = bench.merge_bytes(8, 2048, 128, 819)
    T, A = 8 * 2048, 8 * 819
    assert b["fwd"] == T * (2 * 128 + 16) + A * (2 * 128 + 12)
    assert b["bwd"] == T * (4 * 128 + 24) + A * (2 * 128 + 8)


def test_peaks_have_both_denominators():
    p = bench.measured_peaks()
    assert p["hbm_gbs"] > 0 and p["bf16_tflops"] > 0 and p["source"]


def test_traffic_is_keyed_to_call_shape_and_sources(tmp_path):
    names = bench.TRAFFIC_SOURCES["attn_bwd"]
    h = bench.source_hash(names)
    assert len(h) == 16 and h == bench.source_hash(names)
    assert h != bench.source_hash()  # a subset of the sources hashes differently
    for name in names:
        assert os.path.exists(os.path.join(bench.ROOT, "off_grid_cluster_b200", "csrc", name))
    w = bench.call_workload("attn_bwd", 16, 328, H=16)
    f = tmp_path / "t.txt"
    f.write_text("# comment\n"
                 f"traffic: call = attn_bwd; workload = {w}; read = 1000; write = 24; src = {h}\n"
                 f"traffic: call = attn_fwd; workload = {w}; read = 5; write = 5; src = 0000000000000000\n")
    rows = bench.read_traffic(str(f))
    assert len(rows) == 2
    assert bench.traffic_for("attn_bwd", w, rows) == {"read": 1000.0, "write": 24.0, "total": 1024.0}
    assert bench.traffic_for("attn_fwd", w, rows) is None          # stale sources
    assert bench.traffic_for("attn_bwd", "b8-n2048-h4", rows) is None
    assert bench.read_traffic(str(tmp_path / "missing.txt")) == []


def test_argument_defaults():
    a = bench.parse_args([])
    assert (a.gpus, a.impl, a.only, a.batch) == (1, "acl", None, 16)
    assert a.warmup >= 3 and a.steps >= 1
    assert bench.parse_args(["--only", "attn_stage", "--stage", "2"]).stage == 2


def test_workload_constants_match_the_generators():
    from off_grid_cluster_b200 import synth
    assert tuple(bench.STAGE_LAYERS) == tuple(synth.SWEEP_LAYERS)
    assert tuple(bench.STAGE_DIMS) == tuple(synth.SWEEP_DIMS)
    assert tuple(x.shape[1] for x in synth.sweep_coords(B=1)) == bench.STAGE_TOKENS


def test_clock_sampler_reads_median_max_and_reasons(tmp_path):
    """The clock record of a timed region: median SM clock under load, the highest
    clocks.max.sm seen, and every throttle reason that was Active in any sample."""
    path = tmp_path / "clocks.csv"
    path.write_text(
        "0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active\n"
        "0, 1900, 1965, 998.0, 0x4, Not Active, Not Active, Not Active, Active\n"
        "0, 1950, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active\n"
        "garbage line\n"
        "0, [N/A], 1965, 0, 0x0, Not Active, Active, Not Active, Not Active\n")

    class FakeProc:
        def terminate(self):
            pass

        def wait(self, timeout=None):
            return 0

    cs = bench.ClockSampler("GPU-0")
    cs.proc, cs.path = FakeProc(), str(path)
    rec = cs.stop()
    assert rec["samples"] == 4
    assert rec["sm_mhz"] == 1950.0 and rec["sm_max_mhz"] == 1965.0
    assert rec["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]
    assert not path.exists()
    assert bench.ClockSampler("GPU-0").stop()["reasons"] == ["nvidia-smi unavailable"]
