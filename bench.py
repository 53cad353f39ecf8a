#!/usr/bin/env python
"""Benchmark of the off-grid cluster attention + KNN gather hot path on B200.

One *step* is one pass of every step of the path over the two largest seeded synthetic
workloads, shaped like the AFFMAE pages' 1024 px encoder and decoder ("A Complete
Example": a 64 x 64 patch grid, 2048 visible tokens, then 819 / 328 / 131 after each
down-sampling):

  encoder sweep   16 images; four stages of 2048 / 819 / 328 / 131 tokens (nested random
                  subsets, ratio 0.4) with dims 128 / 256 / 512 / 768 (4 / 8 / 16 / 24
                  heads x 32) and 3 / 4 / 16 / 2 layers, C = 8, M = 48, distinct Q / K / V
                  / dO buffers per layer.  Forward over the stages (acl_cluster ->
                  acl_neighbors -> acl_cluster_attn_fwd per layer), then the backward in
                  reverse (acl_cluster_attn_bwd per layer).
  decoder gather  16 images x 4096 queries (cell centre + U(-1, 1)^2) over each of the
                  four stages' tokens (d = 128 ... 768), K = 8, one temperature per head:
                  acl_knn_table -> acl_knn_gather_fwd -> acl_knn_gather_bwd per stage.

`value` is the encoder sweep's cluster-attention tokens/s: token-layers (images x tokens,
summed over the 25 layers, all ranks) per second of the sweep's device time; the sweep's
time includes its clustering and neighbour tables.  `knn` gives the decoder gather's
queries/s the same way (queries x stages over the gather's device time, tables included).
Both spans are measured with CUDA events inside the timed steps; ms_per_step is their sum.
The inputs of one step (about 1.4 GB) are larger than the 126 MB L2, so no flush is
needed between steps; each step is one CUDA graph of the library calls with CUDA events
between the calls.  `roofline` and `roofline_knn` name the call with the largest share of
each span and divide its algorithmic bytes per launch by its mean launch time.  `e2e`
runs the same calls through the public entry points with every step's inputs copied in
from pinned host memory and all outputs read back, copies pipelined against compute.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl acl|reference]

With --impl reference the fp64 CPU oracle is timed on the host cores on a bounded sample
of the same workload (rank 0 only under torchrun).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "cluster-attn fwd+bwd tokens/s & KNN-gather queries/s; % of B200 HBM roofline"
IMAGES = 16                                   # images per rank
STAGE_TOKENS = (2048, 819, 328, 131)
STAGE_DIMS = (128, 256, 512, 768)
STAGE_LAYERS = (3, 4, 16, 2)
QUERIES, KNN_K, GRID = 4096, 8, 64
WORKLOAD = ("encoder-sweep-1024px-b16-n2048/819/328/131-d128/256/512/768-layers3/4/16/2-c8-m48"
            " + decoder-knn-gather-b16-q4096-k8-over-the-4-stages")
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
# the kernels behind each call
KERNELS = {
    "cluster": ["cluster_kernel"],
    "neighbors": ["neighbors_kernel"],
    "attn_fwd": ["attn_fwd_kernel"],
    "attn_bwd": ["attn_bwd_query_kernel", "attn_bwd_key_kernel"],
    "knn_table": ["knn_table_kernel"],
    "knn_fwd": ["knn_fwd_*"],
    "knn_index": ["knn_keys_kernel", "knn_csr_kernel"],
    "knn_bwd": ["knn_bwd_query_*", "knn_bwd_token_*"],
}
# the files whose code makes each call's kernels: a DRAM-traffic figure taken by ncu on
# other sources than the current ones is stale and is reported as null
TRAFFIC_SOURCES = {
    "attn_fwd": ("attn.cu", "common.cuh"),
    "attn_bwd": ("attn.cu", "common.cuh"),
    "knn_fwd": ("knn.cu", "common.cuh"),
    "knn_bwd": ("knn.cu", "common.cuh"),
}
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic.txt")


# --------------------------------------------------------------------------- helpers

def env_int(name: str, default: int) -> int:
    try:
        return int(os.environ.get(name, default))
    except ValueError:
        return default


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("acl", "reference"), default="acl")
    ap.add_argument("--batch", type=int, default=IMAGES, help="images per rank (default 16)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the extra parts (per-layer configurations, token merging, "
                         "high-resolution gather, decoder layers)")
    ap.add_argument("--e2e-steps", type=int, default=6)
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="bounded CPU work of the oracle baseline (seconds)")
    ap.add_argument("--only", choices=("token_merge", "decoder", "configs", "attn_stage", "knn_stage",
                                       "attn_traffic", "knn_traffic", "attn_fwd_units"),
                    default=None,
                    help="run one part alone on one GPU and print its JSON (a short command to "
                         "profile under ncu); no bench line.  attn_traffic / knn_traffic run one "
                         "stage's calls in the bench's order over inputs larger than L2, for a "
                         "DRAM-traffic capture whose cache state matches the bench's")
    ap.add_argument("--stage", type=int, default=3, help="stage (1-4) of --only attn_stage / knn_stage")
    return ap.parse_args(argv)


def shard_images(rank: int, world: int, per_rank: int) -> tuple[int, int]:
    """Images [first, first + per_rank) of the seeded workload handled by this rank.

    Images are independent problems, so ranks take disjoint image ranges and never
    exchange data: per-rank work is fixed as the rank count grows (weak scaling).
    """
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    return rank * per_rank, per_rank


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Maximum of a per-rank scalar over all ranks (the slowest rank's time)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def measured_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d.get("bf16_tflops", FALLBACK_BF16_TFLOPS)),
                "source": "measured (copy bandwidth and bf16 GEMM on this pool's B200s)"}
    return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
            "source": "fallback 6.65 TB/s, 1590 TFLOP/s"}


def source_hash(names=None) -> str:
    """Hash of the named CUDA sources (all of them when names is None)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "off_grid_cluster_b200", "csrc")
    for name in sorted(names if names is not None else os.listdir(csrc)):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


# --------------------------------------------------------------------------- byte counts

def attn_bytes(B: int, N: int, H: int) -> dict:
    """Algorithmic bytes of one attention call, every tensor once: per (token, head) the
    forward moves Q, K, V, O (64 B each in bf16) and the lse (4 B) = 260 B, the backward
    Q, K, V, O, dO, lse and dQ, dK, dV = 516 B; per token 72 B of coordinates, cluster
    list and neighbour-table share."""
    return {"attn_fwd": B * N * (260 * H + 72), "attn_bwd": B * N * (516 * H + 72)}


def knn_bytes(B: int, Q: int, N: int, d: int, K: int = KNN_K) -> dict:
    """Algorithmic bytes of one gather call: per query the forward reads its position (8 B)
    and table row (4K B) and writes d bf16 channels; the backward reads position, table row
    and dOut and writes dq (8 B); per token the features (2d B) and coordinates (8 B) are
    read once and the backward writes dF (2d B)."""
    return {"knn_fwd": B * (Q * (8 + 4 * K + 2 * d) + N * (2 * d + 8)),
            "knn_bwd": B * (Q * (8 + 4 * K + 8 + 2 * d) + N * (4 * d + 8)),
            # inverse index: positions and table rows in, the entries' tokens and their
            # token-sorted order out, one offset per token
            "knn_index": B * (Q * (8 + 12 * K) + 4 * (N + 1))}


def table_bytes(B: int, N: int, C: int = 8, M: int = 48, GH: int = GRID, GW: int = GRID,
                K: int = KNN_K) -> dict:
    """Clustering, neighbour table and KNN table: coordinates in, index tables out."""
    G = (N + C - 1) // C
    return {"cluster": B * N * (8 + 4), "neighbors": B * (N * 8 + G * C * 4 + G * M * 4),
            "knn_table": B * (N * 8 + GH * GW * K * 4)}


def merge_bytes(B: int, N: int, d: int, k: int) -> dict:
    """Algorithmic bytes of token merging, every tensor once: forward reads features (2d B)
    and coordinates (8 B) per token and writes score, assignment (8 B) per token and the merged
    row (2d + 8 B) and anchor id per anchor; backward reads features, coordinates, score and
    assignment and writes dfeats and dcoords per token (4d + 24 B), reads dmerged (2d + 8 B)
    per anchor."""
    T, A = B * N, B * k
    return {"fwd": T * (2 * d + 16) + A * (2 * d + 12), "bwd": T * (4 * d + 24) + A * (2 * d + 8)}


def read_traffic(path: str = TRAFFIC_FILE) -> list[dict]:
    """Rows of the committed ncu DRAM-traffic summary: lines `key = value; key = value ...`
    with call, workload, read, write (bytes per launch) and src (hash of the call's sources
    the counters were taken on); other lines are ignored."""
    rows = []
    if not os.path.exists(path):
        return rows
    with open(path) as f:
        for line in f:
            if not line.startswith("traffic:"):
                continue
            row = {}
            for part in line[len("traffic:"):].split(";"):
                if "=" in part:
                    k, v = part.split("=", 1)
                    row[k.strip()] = v.strip()
            if {"call", "workload", "read", "write", "src"} <= row.keys():
                rows.append(row)
    return rows


def traffic_for(call: str, workload: str, rows: list[dict]) -> dict | None:
    """DRAM bytes per launch of `call` on `workload` if a capture on the current sources
    exists, else None."""
    if call not in TRAFFIC_SOURCES:
        return None
    h = source_hash(TRAFFIC_SOURCES[call])
    for r in rows:
        if r["call"] == call and r["workload"] == workload and r["src"] == h:
            rd, wr = float(r["read"]), float(r["write"])
            return {"read": rd, "write": wr, "total": rd + wr}
    return None
class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 100 ms in the background."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu = gpu_id
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        return self

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"],
                    "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


# --------------------------------------------------------------------------- workload

def _pinned(torch, x: np.ndarray, dtype):
    t = torch.from_numpy(np.ascontiguousarray(x)).to(dtype)
    return t.pin_memory()


class HostWorkload:
    """The seeded inputs of one rank's step in pinned host memory (bf16 tensors as bf16):
    per encoder stage its coordinates, bias coefficients and every layer's Q / K / V / dO;
    per decoder stage its queries, token features, coordinates, temperatures and dOut."""

    def __init__(self, B: int, image0: int, torch, pin: bool = True, layers: int | None = None):
        """`layers` limits the layers generated per stage (the oracle's sample needs one);
        `pin` False keeps plain host tensors (no CUDA context needed)."""
        from off_grid_cluster_b200 import synth
        bf, f32 = torch.bfloat16, torch.float32
        self.B = B
        self.layer_counts = list(STAGE_LAYERS)
        host = _pinned if pin else (lambda _t, x, dt: torch.from_numpy(np.ascontiguousarray(x)).to(dt))
        self.stages = []
        for s, xy in enumerate(synth.sweep_coords(B, image0)):
            layers_s = []
            for layer in range(STAGE_LAYERS[s] if layers is None else min(layers, STAGE_LAYERS[s])):
                ab = synth.attn_sweep_layer(xy, s, layer, image0)
                layers_s.append({n: host(torch, getattr(ab, n), bf) for n in ("q", "k", "v", "do")})
            self.stages.append({"coords": host(torch, xy, f32), "bias": host(torch, ab.bias, f32),
                                "scale": float(ab.scale), "N": int(xy.shape[1]), "H": int(ab.q.shape[2]),
                                "layers": layers_s})
        self.knn = []
        for kb in synth.knn_decoder(B, image0):
            self.knn.append({"queries": host(torch, kb.queries, f32), "feats": host(torch, kb.feats, bf),
                             "coords": host(torch, kb.coords, f32), "p": host(torch, kb.p, f32),
                             "dout": host(torch, kb.dout, bf), "N": int(kb.N), "d": int(kb.d),
                             "Q": int(kb.Q), "GH": int(kb.GH), "GW": int(kb.GW), "K": int(kb.K)})

    def token_layers(self) -> int:
        return sum(self.B * st["N"] * L for st, L in zip(self.stages, self.layer_counts))

    def query_stages(self) -> int:
        return sum(self.B * k["Q"] for k in self.knn)


class DeviceStep:
    """Device copies of a HostWorkload's inputs, the outputs of every call and the calls of
    one step in order (`calls`: (kind, stage, fn) with fn(stream) issuing one library call)."""

    def __init__(self, hw: HostWorkload, device, torch, acl):
        self.torch, self.acl, self.B = torch, acl, hw.B
        dev = lambda t: t.to(device, non_blocking=False)
        e = lambda shape, dt: torch.empty(shape, dtype=dt, device=device)
        bf, f32, i32 = torch.bfloat16, torch.float32, torch.int32
        B = hw.B
        self.ins, self.outs = [], []            # (device, host) input pairs; device outputs
        self.stages = []
        ws_attn = 0
        for st in hw.stages:
            N, H = st["N"], st["H"]
            G = (N + 7) // 8
            d = {"coords": dev(st["coords"]), "bias": dev(st["bias"]), "scale": st["scale"], "N": N, "H": H,
                 "clusters": e((B, G, 8), i32), "nbr": e((B, G, 48), i32), "layers": []}
            self.ins += [(d["coords"], st["coords"]), (d["bias"], st["bias"])]
            self.outs += [d["clusters"], d["nbr"]]
            for hl in st["layers"]:
                L = {n: dev(hl[n]) for n in ("q", "k", "v", "do")}
                self.ins += [(L[n], hl[n]) for n in ("q", "k", "v", "do")]
                L.update(o=e((B, N, H, 32), bf), lse=e((B, N, H), f32), dq=e((B, N, H, 32), bf),
                         dk=e((B, N, H, 32), bf), dv=e((B, N, H, 32), bf), dbias=e((H, 3), f32))
                self.outs += [L[n] for n in ("o", "lse", "dq", "dk", "dv", "dbias")]
                d["layers"].append(L)
            ws_attn = max(ws_attn, acl.acl_cluster_attn_workspace(B, N, H, 8, 48))
            self.stages.append(d)
        self.knn = []
        ws_knn = 0
        for k in hw.knn:
            d = {n: dev(k[n]) for n in ("queries", "feats", "coords", "p", "dout")}
            self.ins += [(d[n], k[n]) for n in ("queries", "feats", "coords", "p", "dout")]
            d.update(GH=k["GH"], GW=k["GW"], K=k["K"],
                     table=e((B, k["GH"], k["GW"], k["K"]), i32), out=e((B, k["Q"], k["d"]), bf),
                     dfeats=e((B, k["N"], k["d"]), bf), dq=e((B, k["Q"], 2), f32), dp=e((k["d"] // 32,), f32))
            self.outs += [d[n] for n in ("table", "out", "dfeats", "dq", "dp")]
            # each stage's inverse index lives in its own workspace from its build to its backward
            d["ws"] = e((max(acl.acl_knn_gather_workspace(B, k["Q"], k["N"], k["d"], k["K"]), 1),), torch.uint8)
            ws_knn += d["ws"].numel()
            self.knn.append(d)
        # the attention calls run one at a time on one stream: one workspace serves them all
        self.ws_attn = e((max(ws_attn, 1),), torch.uint8)
        self.calls = self._calls()

    def bytes(self) -> int:
        ts = [t for t, _ in self.ins] + self.outs + [self.ws_attn] + [k["ws"] for k in self.knn]
        return sum(t.numel() * t.element_size() for t in ts)

    def _calls(self):
        acl, calls = self.acl, []
        for s, d in enumerate(self.stages):
            calls.append(("cluster", s, lambda st, d=d: acl.acl_cluster(d["coords"], 8, clusters=d["clusters"],
                                                                         stream=st)))
            calls.append(("neighbors", s, lambda st, d=d: acl.acl_neighbors(d["coords"], d["clusters"], 48,
                                                                             nbr=d["nbr"], stream=st)))
        for s, d in enumerate(self.stages):
            for L in d["layers"]:
                calls.append(("attn_fwd", s, lambda st, d=d, L=L: acl.acl_cluster_attn_fwd(
                    L["q"], L["k"], L["v"], d["coords"], d["clusters"], d["nbr"], d["bias"], d["scale"],
                    O=L["o"], lse=L["lse"], stream=st)))
        for s in reversed(range(len(self.stages))):
            d = self.stages[s]
            for L in reversed(d["layers"]):
                calls.append(("attn_bwd", s, lambda st, d=d, L=L: acl.acl_cluster_attn_bwd(
                    L["q"], L["k"], L["v"], d["coords"], d["clusters"], d["nbr"], d["bias"], d["scale"],
                    L["o"], L["do"], L["lse"], L["dq"], L["dk"], L["dv"], L["dbias"],
                    workspace=self.ws_attn, stream=st)))
        for s, k in enumerate(self.knn):
            calls.append(("knn_table", s, lambda st, k=k: acl.acl_knn_table(k["coords"], k["GH"], k["GW"], k["K"],
                                                                             table=k["table"], stream=st)))
            calls.append(("knn_index", s, lambda st, k=k: acl.acl_knn_gather_index(
                k["queries"], k["table"], k["feats"].shape[1], k["feats"].shape[2], k["ws"], stream=st)))
            calls.append(("knn_fwd", s, lambda st, k=k: acl.acl_knn_gather_fwd(
                k["queries"], k["feats"], k["coords"], k["table"], k["p"], out=k["out"], stream=st)))
            calls.append(("knn_bwd", s, lambda st, k=k: acl.acl_knn_gather_bwd_indexed(
                k["queries"], k["feats"], k["coords"], k["table"], k["p"], k["dout"], k["ws"], dfeats=k["dfeats"],
                dqueries=k["dq"], dp=k["dp"], stream=st)))
        return calls

    def first_knn(self) -> int:
        return next(i for i, c in enumerate(self.calls) if c[0].startswith("knn"))

    def step(self, stream, events=None, side=None):
        """Every call of the step on `stream`; events[2j], events[2j + 1] bracket call j (on the
        stream the call runs on).  With a `side` stream the clustering and neighbour tables of
        stages 2..4 run there, concurrently with the stage-1 layers (the clustering kernel
        takes one CTA per image), and each stage's first layer waits for its own tables."""
        torch = self.torch
        ready = {}
        if side is not None:
            side.wait_stream(stream)
        # decoder gather: the table of stage 1 on the main stream; every stage's inverse index
        # and the tables of stages 2..4 on the side stream (in stage order), so they overlap the
        # gathers; a stage's forward waits for its table, its backward for its index
        side_kinds = ("cluster", "neighbors", "knn_table", "knn_index")
        for j, (kind, s, fn) in enumerate(self.calls):
            on_side = side is not None and kind in side_kinds and (s > 0 or kind == "knn_index")
            st = side if on_side else stream
            if side is not None:
                if kind == "attn_fwd" and ("nbr", s) in ready:
                    stream.wait_event(ready.pop(("nbr", s)))
                if kind == "knn_fwd" and ("table", s) in ready:
                    stream.wait_event(ready.pop(("table", s)))
                if kind == "knn_bwd" and ("index", s) in ready:
                    stream.wait_event(ready.pop(("index", s)))
                if kind == "knn_index" and s == 0:
                    side.wait_event(ready.pop(("table0",)))
            if events is not None:
                events[2 * j].record(st)
            fn(st)
            if events is not None:
                events[2 * j + 1].record(st)
            if side is not None:
                tag = {"neighbors": "nbr", "knn_table": "table", "knn_index": "index"}.get(kind)
                if tag is not None:
                    ev = torch.cuda.Event()
                    ev.record(st)
                    ready[(tag, s) if (on_side or tag != "table") else ("table0",)] = ev
        if side is not None:
            stream.wait_stream(side)


def call_workload(kind: str, B: int, N: int, H: int = 0, d: int = 0, Q: int = QUERIES) -> str:
    """Canonical name of one launch shape (the key of the DRAM-traffic summary)."""
    if kind.startswith("attn") or kind in ("cluster", "neighbors"):
        return f"b{B}-n{N}-h{H}"
    return f"b{B}-q{Q}-n{N}-d{d}"


# --------------------------------------------------------------------------- GPU arm

def run_gpu(args, rank: int, world: int):
    import torch
    import torch.distributed as dist

    import off_grid_cluster_b200 as acl

    local = env_int("LOCAL_RANK", 0)
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=device)

    def barrier():
        if world > 1:
            dist.barrier()

    first, per_rank = shard_images(rank, world, args.batch)
    hw = HostWorkload(per_rank, first, torch)
    ds = DeviceStep(hw, device, torch, acl)
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    stream = torch.cuda.Stream(device)
    side = torch.cuda.Stream(device)
    # eager pass of every call (kernel attributes, lazy module loading), then capture
    with torch.cuda.stream(stream):
        ds.step(stream, side=side)
    stream.synchronize()
    n_calls = len(ds.calls)
    reps = max(1, min(args.steps, 3))       # graph copies with their own events, replayed in turn
    graphs, events = [], []
    launches0 = acl.acl_launch_count()
    for _ in range(reps):
        evs = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2 * n_calls)]
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            ds.step(stream, evs, side=side)
        graphs.append(g)
        events.append(evs)
    launches_per_step = (acl.acl_launch_count() - launches0) // reps
    torch.cuda.synchronize()

    def replay(i):
        with torch.cuda.stream(stream):
            graphs[i % reps].replay()

    for w in range(args.warmup):
        replay(w)
    torch.cuda.synchronize()
    props = torch.cuda.get_device_properties(device)
    uuid = getattr(props, "uuid", None)
    clocks = ClockSampler(f"GPU-{uuid}" if uuid is not None else str(local)).start()
    barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    # the last `reps` replays fill every graph copy's events
    for it in range(args.steps):
        replay(it)
    t1.record(stream)
    torch.cuda.synchronize()
    barrier()
    step_ms_local = t0.elapsed_time(t1) / max(args.steps, 1)
    # per-call durations of the last timed replay of every graph copy
    dur = np.zeros(n_calls)
    span_a, span_k = 0.0, 0.0
    kf = ds.first_knn()
    for evs in events:
        dur += np.array([evs[2 * j].elapsed_time(evs[2 * j + 1]) for j in range(n_calls)])
        span_a += evs[0].elapsed_time(evs[2 * kf - 1])
        span_k += evs[2 * kf].elapsed_time(evs[2 * n_calls - 1])
    dur /= reps
    span_a /= reps
    span_k /= reps
    # keep the same load on the GPU until the clock sampler has several samples
    t_wall = time.time()
    it = 0
    while time.time() - t_wall < 0.8:
        for _ in range(8):
            replay(it)
            it += 1
        stream.synchronize()
    torch.cuda.synchronize()
    clk = clocks.stop()

    step_ms = max_over_ranks(step_ms_local, world, device)
    span_a = max_over_ranks(span_a, world, device)
    span_k = max_over_ranks(span_k, world, device)
    peaks = measured_peaks()
    hbm = peaks["hbm_gbs"]
    B = per_rank
    token_layers = world * hw.token_layers()
    query_stages = world * hw.query_stages()
    value = token_layers / (span_a * 1e-3)
    knn_value = query_stages / (span_k * 1e-3)

    # per (call, stage) groups: launches, mean launch time, algorithmic bytes per launch
    groups = {}
    for j, (kind, s, _) in enumerate(ds.calls):
        g = groups.setdefault((kind, s), {"kind": kind, "stage": s, "launches": 0, "ms": 0.0})
        g["launches"] += 1
        g["ms"] += dur[j]
    for (kind, s), g in groups.items():
        if kind in ("knn_table", "knn_index", "knn_fwd", "knn_bwd"):
            k = hw.knn[s]
            by = {**knn_bytes(B, k["Q"], k["N"], k["d"], k["K"]), **table_bytes(B, k["N"])}
            g["workload"] = call_workload(kind, B, k["N"], d=k["d"], Q=k["Q"])
        else:
            st = hw.stages[s]
            by = {**attn_bytes(B, st["N"], st["H"]), **table_bytes(B, st["N"])}
            g["workload"] = call_workload(kind, B, st["N"], H=st["H"])
        g["bytes"] = by[kind]
        g["us"] = g["ms"] / g["launches"] * 1e3
        g["GB_s"] = g["bytes"] / (g["us"] * 1e-6) / 1e9
        g["frac"] = g["GB_s"] / hbm
    traffic_rows = read_traffic()

    def roofline(kinds, what):
        cand = [g for g in groups.values() if g["kind"] in kinds]
        g = max(cand, key=lambda x: x["ms"])
        tr = traffic_for(g["kind"], g["workload"], traffic_rows)
        return {"bound": "hbm", "achieved": round(g["GB_s"], 1), "peak": hbm, "unit": "GB/s",
                "frac": round(g["frac"], 4), "traffic": None if tr is None else int(tr["total"]),
                "traffic_read": None if tr is None else int(tr["read"]),
                "traffic_write": None if tr is None else int(tr["write"]),
                "traffic_basis": ("ncu dram__bytes_read.sum + dram__bytes_write.sum per launch, one eager "
                                  "launch of this shape on the current sources (--cache-control none)"
                                  if tr is not None else "no capture on the current sources"),
                "call": f"acl_{g['kind']}", "kernels": KERNELS[g["kind"]],
                "launch_workload": g["workload"], "stage": g["stage"] + 1,
                "launches_per_step": g["launches"], "share_of_span": round(g["ms"] / what, 4),
                "alg_bytes_per_launch": int(g["bytes"]), "launch_us": round(g["us"], 3),
                "peak_source": peaks["source"] + " (burst copy)", "of": "measured" if "measured" in peaks["source"]
                else "fallback"}

    attn_kinds = ("cluster", "neighbors", "attn_fwd", "attn_bwd")
    knn_kinds = ("knn_table", "knn_index", "knn_fwd", "knn_bwd")
    rf_attn = roofline(attn_kinds, span_a)
    rf_knn = roofline(knn_kinds, span_k)

    def span_of(kinds):
        """(device ms per step, fraction of HBM) of every launch of the given calls"""
        ms = sum(g["ms"] for g in groups.values() if g["kind"] in kinds)
        by = sum(g["bytes"] * g["launches"] for g in groups.values() if g["kind"] in kinds)
        return ms, by / (ms * 1e-3) / 1e9 / hbm
    attn_fb_ms, attn_fb_frac = span_of(("attn_fwd", "attn_bwd"))
    knn_fb_ms, knn_fb_frac = span_of(("knn_index", "knn_fwd", "knn_bwd"))
    per_stage = []
    for s, st in enumerate(hw.stages):
        f, b = groups[("attn_fwd", s)], groups[("attn_bwd", s)]
        per_stage.append({"stage": s + 1, "N": st["N"], "H": st["H"], "layers": f["launches"],
                          "cluster_us": round(groups[("cluster", s)]["us"], 2),
                          "neighbors_us": round(groups[("neighbors", s)]["us"], 2),
                          "fwd_us": round(f["us"], 2), "bwd_us": round(b["us"], 2),
                          "fwd_frac": round(f["frac"], 4), "bwd_frac": round(b["frac"], 4),
                          "fwd_bwd_frac": round((f["bytes"] + b["bytes"]) / ((f["us"] + b["us"]) * 1e-6)
                                                / 1e9 / hbm, 4)})
    knn_stage = []
    for s, k in enumerate(hw.knn):
        t, f, b = groups[("knn_table", s)], groups[("knn_fwd", s)], groups[("knn_bwd", s)]
        knn_stage.append({"stage": s + 1, "N": k["N"], "d": k["d"], "table_us": round(t["us"], 2),
                          "index_us": round(groups[("knn_index", s)]["us"], 2),
                          "fwd_us": round(f["us"], 2), "bwd_us": round(b["us"], 2),
                          "fwd_frac": round(f["frac"], 4), "bwd_frac": round(b["frac"], 4),
                          "fwd_bwd_frac": round((f["bytes"] + b["bytes"]) / ((f["us"] + b["us"]) * 1e-6)
                                                / 1e9 / hbm, 4)})

    extras = None
    if world == 1 and not args.no_extras:
        from off_grid_cluster_b200 import synth
        extras = {
            "configs": config_times(torch, acl, synth, device, stream, peaks),
            "token_merge_us": token_merge_times(torch, acl, synth, device, stream, peaks),
            "hires_gather_us": hires_gather_times(torch, acl, synth, device, stream),
            "decoder_us": decoder_times(torch, acl, synth, device, stream, peaks),
        }

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, hw, ds, stream, torch, acl, device)
        e2e_ms = max_over_ranks(e2e.pop("_ms"), world, device)
        e2e["ms_per_step"] = round(e2e_ms, 3)
        e2e["value"] = round(token_layers / (e2e_ms * 1e-3), 1)
        e2e["knn_value"] = round(query_stages / (e2e_ms * 1e-3), 1)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args, per_rank)

    set_mb = ds.bytes() / 1e6
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_ms, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; shapes of the pages' 1024 px encoder and decoder workloads)",
        "config": {"workload": WORKLOAD, "images_per_gpu": B, "stage_tokens": [st["N"] for st in hw.stages],
                   "stage_heads": [st["H"] for st in hw.stages],
                   "stage_layers": [len(st["layers"]) for st in hw.stages], "head_dim": 32, "C": 8, "M": 48,
                   "knn_queries_per_image": QUERIES, "knn_stage_d": [k["d"] for k in hw.knn], "K": KNN_K,
                   "grid": [GRID, GRID],
                   "l2": f"inputs + outputs of one step {set_mb:.0f} MB > L2 {l2 / 1e6:.0f} MB: no flush "
                         f"between steps",
                   "timing": f"one CUDA graph per step ({reps} copies replayed in turn), CUDA events on the "
                             f"launching stream around the steps and between the calls",
                   "parallelism": f"replicas x{world} (images sharded, no collective)"},
        "value_basis": "encoder token-layers of all ranks / the encoder sweep's device time per step "
                       "(clustering and neighbour tables included, those of stages 2-4 on a second stream "
                       "beside the stage-1 layers; mean of the last timed steps, max over ranks)",
        "segments_ms": {"encoder_sweep": round(span_a, 4), "decoder_gather": round(span_k, 4)},
        "knn": {"value": round(knn_value, 1), "unit": "queries/s",
                "basis": "decoder queries x stages of all ranks / the gather's device time per step "
                         "(KNN tables and inverse indexes included, those on a second stream beside "
                         "the gathers)",
                "gather_index_fwd_bwd_queries_per_s": round(query_stages / (knn_fb_ms * 1e-3), 1),
                "gather_index_fwd_bwd_frac": round(knn_fb_frac, 4), "stages": knn_stage},
        "roofline": rf_attn,
        "roofline_knn": rf_knn,
        "parts": {
            "attn_fwd_bwd_tokens_per_s": round(token_layers / (attn_fb_ms * 1e-3), 1),
            "attn_fwd_bwd_frac": round(attn_fb_frac, 4),
            "attn_stages": per_stage,
            "extras": extras,
        },
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": int(launches_per_step * args.steps),
        "clocks": clk,
    }
    for g in graphs:
        g.reset()
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def graph_time(torch, stream, fn, reps: int = 10) -> float:
    """Device time of one call of fn in microseconds: fn captured once as a CUDA graph and
    replayed `reps` times between CUDA events on `stream` (no host work inside)."""
    with torch.cuda.stream(stream):
        fn()
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    with torch.cuda.stream(stream):
        for _ in range(3):
            g.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
    e1.synchronize()
    g.reset()
    return round(e0.elapsed_time(e1) / reps * 1e3, 2)


def run_e2e(args, hw: HostWorkload, ds: DeviceStep, stream, torch, acl, device) -> dict:
    """The step through the public entry points from pinned host memory, copies inside.

    Every step copies all of its inputs host -> device and all of its outputs device ->
    host.  Two device sets and two copy streams pipeline the steps: the inputs of step
    k + 1 travel in and the outputs of step k - 1 travel out while step k computes (PCIe
    is full duplex), with events ordering each set's copy-in, compute and copy-out."""
    sets = [ds, DeviceStep(hw, device, torch, acl)]
    hout = [[torch.empty_like(t, device="cpu").pin_memory() for t in ds.outs] for _ in range(2)]
    h2d = sum(h.numel() * h.element_size() for _, h in ds.ins)
    d2h = sum(t.numel() * t.element_size() for t in ds.outs)
    cp_in, cp_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    side = torch.cuda.Stream(device)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    recorded = [False, False]

    def one(k):
        i = k % 2
        S = sets[i]
        if recorded[i]:
            cp_in.wait_event(ev_done[i])    # step k - 2 has finished reading set i's inputs
        with torch.cuda.stream(cp_in):
            for dv, hv in S.ins:
                dv.copy_(hv, non_blocking=True)
        ev_in[i].record(cp_in)
        stream.wait_event(ev_in[i])
        if recorded[i]:
            stream.wait_event(ev_out[i])    # step k - 2's outputs have left set i
        with torch.cuda.stream(stream):
            S.step(stream, side=side)
        ev_done[i].record(stream)
        cp_out.wait_event(ev_done[i])
        with torch.cuda.stream(cp_out):
            for dv, hv in zip(S.outs, hout[i]):
                hv.copy_(dv, non_blocking=True)
        ev_out[i].record(cp_out)
        recorded[i] = True

    def drain():
        stream.wait_stream(cp_out)
        stream.wait_stream(cp_in)

    for k in range(3):
        one(k)
    drain()
    torch.cuda.synchronize()
    n = max(1, args.e2e_steps)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    cp_in.wait_stream(stream)
    cp_out.wait_stream(stream)
    for k in range(n):
        one(k)
    drain()
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / n
    return {"unit": "tokens/s", "knn_unit": "queries/s", "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "steps": n, "_ms": ms,
            "pipelining": "2 device sets, copy-in / compute / copy-out streams; eager calls"}


# --------------------------------------------------------------------------- extra parts

def config_times(torch, acl, synth, device, stream, peaks: dict, reps: int = 10) -> dict:
    """One layer of the three smaller attention workloads (the tiny 16 x 16 grid; 8 images x
    2048 tokens, 4 heads; 64 images x 328 tokens, 16 heads), one call at a time, each
    captured as a CUDA graph and timed with CUDA events; tokens/s of fwd + bwd and the
    fraction of the measured HBM copy bandwidth on the algorithmic bytes (`attn_bytes`)."""
    T = lambda x, dt=None: torch.from_numpy(np.ascontiguousarray(x)).to(device=device, dtype=dt)
    timed = lambda fn: graph_time(torch, stream, fn, reps)
    hbm = peaks["hbm_gbs"]

    def attn_layer(ab, what):
        xy = T(ab.coords)
        q, k, v, do = (T(x, torch.bfloat16) for x in (ab.q, ab.k, ab.v, ab.do))
        bias = T(ab.bias)
        cl = acl.acl_cluster(xy, stream=stream)
        nb = acl.acl_neighbors(xy, cl, stream=stream)
        o, lse = acl.acl_cluster_attn_fwd(q, k, v, xy, cl, nb, bias, ab.scale, stream=stream)
        ws = torch.empty((acl.acl_cluster_attn_workspace(ab.B, ab.N, ab.H, 8, 48),), dtype=torch.uint8,
                         device=device)
        t_cl = timed(lambda: acl.acl_cluster(xy, clusters=cl, stream=stream))
        t_nb = timed(lambda: acl.acl_neighbors(xy, cl, nbr=nb, stream=stream))
        t_f = timed(lambda: acl.acl_cluster_attn_fwd(q, k, v, xy, cl, nb, bias, ab.scale, O=o, lse=lse,
                                                     stream=stream))
        t_b = timed(lambda: acl.acl_cluster_attn_bwd(q, k, v, xy, cl, nb, bias, ab.scale, o, do, lse,
                                                     workspace=ws, stream=stream))
        by = attn_bytes(ab.B, ab.N, ab.H)
        t = (t_f + t_b) * 1e-6
        gbs = (by["attn_fwd"] + by["attn_bwd"]) / t / 1e9
        return {"config": what, "tokens_per_s_fwd_bwd": round(ab.B * ab.N / t, 1), "cluster_us": t_cl,
                "neighbors_us": t_nb, "fwd_us": t_f, "bwd_us": t_b,
                "fwd_frac": round(by["attn_fwd"] / (t_f * 1e-6) / 1e9 / hbm, 4),
                "bwd_frac": round(by["attn_bwd"] / (t_b * 1e-6) / 1e9 / hbm, 4),
                "GB_s": round(gbs, 1), "frac": round(gbs / hbm, 4)}

    return {
        "tiny": attn_layer(synth.attn_tiny(), "1 image, 16 x 16 grid, H = 4 (launch-bound)"),
        "stage1_b8": attn_layer(synth.attn_stage1(B=8), "8 images x 2048 tokens, H = 4"),
        "stage3_b64": attn_layer(synth.attn_stage3(B=64), "64 images x 328 tokens, H = 16"),
    }


def token_merge_times(torch, acl, synth, device, stream, peaks: dict, reps: int = 10) -> dict:
    """Token merging of 8 images' stage-1 tokens into round(0.4 N) anchors (d = 128, hidden
    32), forward and backward, one call at a time with CUDA events; GB/s of the algorithmic
    bytes and the fraction of the measured HBM copy bandwidth."""
    mb = synth.merge_batch(synth.sweep_coords(B=8)[0], d=128)
    T = lambda x, dt=None: torch.from_numpy(np.ascontiguousarray(x)).to(device=device, dtype=dt)
    f, xy = T(mb.feats, torch.bfloat16), T(mb.coords)
    w1, b1, w2 = T(mb.w1), T(mb.b1), T(mb.w2)
    dm, dx = T(mb.dmerged, torch.bfloat16), T(mb.dmcoords)
    ws = torch.empty((acl.acl_token_merge_workspace(mb.B, mb.N, mb.d, mb.h, mb.k),),
                     dtype=torch.uint8, device=device)
    out = acl.acl_token_merge_fwd(f, xy, w1, b1, w2, mb.b2, mb.k, workspace=ws, stream=stream)
    timed = lambda fn: graph_time(torch, stream, fn, reps)
    res = {
        "workload": f"{mb.B} images, N = {mb.N} -> k = {mb.k}, d = {mb.d}, hidden {mb.h}",
        "fwd": timed(lambda: acl.acl_token_merge_fwd(f, xy, w1, b1, w2, mb.b2, mb.k, workspace=ws,
                                                     stream=stream)),
        "bwd": timed(lambda: acl.acl_token_merge_bwd(f, xy, w1, b1, w2, mb.b2, mb.k, out[0], out[2],
                                                     dm, dx, workspace=ws, stream=stream)),
    }
    nbytes = merge_bytes(mb.B, mb.N, mb.d, mb.k)
    res["roofline"] = {}
    for key in ("fwd", "bwd"):
        gbs = nbytes[key] / (res[key] * 1e-6) / 1e9
        res["roofline"][key] = {"alg_bytes": nbytes[key], "GB_s": round(gbs, 1),
                                "frac": round(gbs / peaks["hbm_gbs"], 4)}
    return res
def hires_gather_times(torch, acl, synth, device, stream, B: int = 4, reps: int = 10) -> dict:
    """Decoder gather at 128 x 128 cells (4 images, 8192 tokens, 16384 queries, d = 128):
    Z-order token order, then table + gather fwd + bwd in raster and in Z-order, one call at a
    time with CUDA events."""
    kb = synth.hires_batch(B=B)
    T = lambda x, dt=None: torch.from_numpy(np.ascontiguousarray(x)).to(device=device, dtype=dt)
    xy, f = T(kb.coords), T(kb.feats, torch.bfloat16)
    q, p, g = T(kb.queries), T(kb.p), T(kb.dout, torch.bfloat16)
    ws = torch.empty((acl.acl_knn_gather_workspace(B, kb.Q, kb.N, kb.d, 8),), dtype=torch.uint8,
                     device=device)

    timed = lambda fn: graph_time(torch, stream, fn, reps)
    res = {"workload": f"{B} images, 128x128 cells, {kb.N} tokens, {kb.Q} queries, d = {kb.d}, K = 8"}
    perm = acl.acl_token_order(xy, 128, 128, stream=stream)
    res["token_order"] = timed(lambda: acl.acl_token_order(xy, 128, 128, perm=perm, stream=stream))
    torch.cuda.synchronize()
    bidx = torch.arange(B, device=device)[:, None]
    pl = perm.long()
    variants = {"raster": (xy, f), "z_order": (xy[bidx, pl].contiguous(), f[bidx, pl].contiguous())}
    for name, (xv, fv) in variants.items():
        table = acl.acl_knn_table(xv, 128, 128, 8, stream=stream)
        out = acl.acl_knn_gather_fwd(q, fv, xv, table, p, stream=stream)
        dF, dq, dp = acl.acl_knn_gather_bwd(q, fv, xv, table, p, g, workspace=ws, stream=stream)
        res[name] = {
            "knn_table": timed(lambda: acl.acl_knn_table(xv, 128, 128, 8, table=table, stream=stream)),
            "knn_fwd": timed(lambda: acl.acl_knn_gather_fwd(q, fv, xv, table, p, out=out,
                                                            stream=stream)),
            "knn_bwd": timed(lambda: acl.acl_knn_gather_bwd(q, fv, xv, table, p, g, dF, dq, dp,
                                                            workspace=ws, stream=stream)),
        }
    return res


def decoder_times(torch, acl, synth, device, stream, peaks: dict, B: int = 8, reps: int = 10) -> dict:
    """The decoder's four layers (coarse to fine over stages 4..1; B images x 2048 mask-token
    queries, D = 256, K = 8), forward and backward per layer and the whole chain, each call
    captured as a CUDA graph and timed with CUDA events.  The projection GEMMs do
    2 T d D FLOPs forward and 4 T d D backward (T = B Q); their rate is given against the
    layer's whole time (a lower bound on the GEMM kernels' own rate) and the measured bf16
    peak."""
    db = synth.decoder_batch(B=B)
    T = lambda x, dt=None: torch.from_numpy(np.ascontiguousarray(x)).to(device=device, dtype=dt)
    ref, f0, df = T(db.ref), T(db.f0), T(db.df)
    layers = []
    for layer, s in enumerate(db.layer_stage):
        st = db.stages[s]
        xy = T(st.coords)
        table = acl.acl_knn_table(xy, st.GH, st.GW, st.K, stream=stream)
        layers.append(dict(w_off=T(db.w_off[layer]), b_off=T(db.b_off[layer]),
                           w_o=T(db.w_o[layer], torch.bfloat16), feats=T(st.feats, torch.bfloat16),
                           coords=xy, table=table, p=T(st.p), d=st.d, N=st.N))
    Tq = db.B * db.Q
    ws = torch.empty((max(acl.acl_decoder_layer_workspace(db.B, db.Q, L["N"], L["d"], db.D)
                          for L in layers),), dtype=torch.uint8, device=device)
    fs, saved = [f0], []
    for L in layers:
        q, v, f_out = acl.acl_decoder_layer_fwd(ref, fs[-1], L["w_off"], L["b_off"], L["w_o"],
                                                L["feats"], L["coords"], L["table"], L["p"], stream=stream)
        saved.append((q, v))
        fs.append(f_out)
    torch.cuda.synchronize()
    stage_of = lambda l: db.layer_stage[l] + 1

    def fwd(l):
        L = layers[l]
        return acl.acl_decoder_layer_fwd(ref, fs[l], L["w_off"], L["b_off"], L["w_o"], L["feats"],
                                         L["coords"], L["table"], L["p"], f_out=fs[l + 1], stream=stream)

    def bwd(l):
        L = layers[l]
        q, v = saved[l]
        return acl.acl_decoder_layer_bwd(fs[l], L["w_off"], L["w_o"], L["feats"], L["coords"],
                                         L["table"], L["p"], q, v, df, workspace=ws, stream=stream)

    res = {"workload": f"{db.B} images x {db.Q} queries, D = {db.D}, K = 8, stages 4..1 "
                       f"(N = {', '.join(str(L['N']) for L in layers)}; d = "
                       f"{', '.join(str(L['d']) for L in layers)})", "layers": []}
    tf, tb = 0.0, 0.0
    for l, L in enumerate(layers):
        uf = graph_time(torch, stream, lambda: fwd(l), reps)
        ub = graph_time(torch, stream, lambda: bwd(l), reps)
        tf += uf
        tb += ub
        flops_f, flops_b = 2.0 * Tq * L["d"] * db.D, 4.0 * Tq * L["d"] * db.D
        res["layers"].append({"stage": stage_of(l), "d": L["d"], "fwd": uf, "bwd": ub,
                              "gemm_tflops_fwd": round(flops_f / (uf * 1e-6) / 1e12, 1),
                              "gemm_tflops_bwd": round(flops_b / (ub * 1e-6) / 1e12, 1)})
    res["fwd_total"] = round(tf, 2)
    res["bwd_total"] = round(tb, 2)
    res["queries_per_s_fwd_bwd"] = round(Tq / ((tf + tb) * 1e-6), 1)
    res["peak_bf16_tflops"] = peaks["bf16_tflops"]
    return res




# --------------------------------------------------------------------------- CPU oracle

def oracle_pass(hw: HostWorkload, images: int) -> dict:
    """One pass of the hot path through the fp64 oracle on the first `images` images: per
    encoder stage the clustering and neighbour table (seconds) and one layer's forward +
    backward (seconds); per decoder stage the table, gather forward and backward."""
    import oracle
    sl = slice(0, images)
    res = {"tables_s": [], "layer_s": [], "knn_s": []}
    for st in hw.stages:
        xy = st["coords"][sl].numpy()
        L = st["layers"][0]
        q, k, v, do = (L[n][sl].float().numpy().astype(np.float64) for n in ("q", "k", "v", "do"))
        bias = st["bias"].numpy().astype(np.float64)
        t0 = time.perf_counter()
        cl = oracle.cluster(xy, 8)
        nb = oracle.neighbors(xy, cl, 48)
        t1 = time.perf_counter()
        oracle.attn_fwd(q, k, v, xy, cl, nb, bias, st["scale"])
        oracle.attn_bwd(q, k, v, xy, cl, nb, bias, st["scale"], do)
        t2 = time.perf_counter()
        res["tables_s"].append(t1 - t0)
        res["layer_s"].append(t2 - t1)
    for kd in hw.knn:
        qq, xy, p = kd["queries"][sl].numpy(), kd["coords"][sl].numpy(), kd["p"].numpy()
        f = kd["feats"][sl].float().numpy().astype(np.float64)
        g = kd["dout"][sl].float().numpy().astype(np.float64)
        t0 = time.perf_counter()
        table = oracle.knn_table(xy, kd["GH"], kd["GW"], kd["K"])
        oracle.knn_fwd(qq, f, xy, table, p)
        oracle.knn_bwd(qq, f, xy, table, p, g)
        res["knn_s"].append(time.perf_counter() - t0)
    return res


def oracle_rates(hw: HostWorkload, images: int, passes: list[dict]) -> tuple[float, float]:
    """(sweep tokens/s, gather queries/s) of the oracle from timed passes over `images`
    images: each stage's clustering + neighbour table once and its layer's time times the
    stage's layer count, as in the sweep."""
    n = len(passes)
    t_sweep = sum(sum(p["tables_s"][s] + hw.layer_counts[s] * p["layer_s"][s] for s in range(len(hw.stages)))
                  for p in passes) / n
    tokens = sum(images * st["N"] * L for st, L in zip(hw.stages, hw.layer_counts))
    t_knn = sum(sum(p["knn_s"]) for p in passes) / n
    queries = sum(images * kd["Q"] for kd in hw.knn)
    return tokens / t_sweep, queries / t_knn


def cpu_baseline(args, B: int) -> dict:
    """The oracle on the host cores over a bounded sample of the rank's workload: one layer
    of each encoder stage (scaled by the stage's layer count) and the gather over every
    stage, for the first images of the batch, repeated for about --cpu-seconds."""
    import torch

    import oracle
    hw = HostWorkload(B, 0, torch, pin=False, layers=1)
    cores = oracle.set_threads(os.cpu_count() or 1)
    images = min(B, max(1, cores))
    passes, t0 = [], time.perf_counter()
    while not passes or time.perf_counter() - t0 < args.cpu_seconds:
        passes.append(oracle_pass(hw, images))
    tok, qry = oracle_rates(hw, images, passes)
    oracle.set_threads(1)
    one = [oracle_pass(hw, 1)]
    tok1, qry1 = oracle_rates(hw, 1, one)
    oracle.set_threads(cores)
    return {"value": round(tok, 1), "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "knn_value": round(qry, 1), "knn_unit": "queries/s",
            "sample": f"{len(passes)} pass(es) over {images} of {B} images: each encoder stage's clustering, "
                      f"neighbour table and one layer fwd + bwd (layer time x the stage's layer count), and "
                      f"the decoder gather (table, fwd, bwd) over the four stages; fp64 C, OpenMP over "
                      f"image x head (attention) and images (the rest)",
            "value_1_thread": round(tok1, 1), "knn_value_1_thread": round(qry1, 1),
            "sample_1_thread": "one pass over 1 image on 1 thread"}


def run_reference(args, rank: int, world: int) -> None:
    if rank != 0:
        return
    import torch

    import oracle
    cores = oracle.set_threads(os.cpu_count() or 1)
    hw = HostWorkload(args.batch, 0, torch, pin=False, layers=1)
    # bounded sample: images per step chosen so that warm-up + steps take about 100 s
    n0 = min(args.batch, cores)
    t = time.perf_counter()
    oracle_pass(hw, n0)
    t0_pass = max(time.perf_counter() - t, 1e-3)
    total = args.steps + args.warmup
    images = int(max(1, min(args.batch, n0 * 100.0 / (total * t0_pass))))
    for _ in range(args.warmup):
        oracle_pass(hw, images)
    t0 = time.perf_counter()
    passes = [oracle_pass(hw, images) for _ in range(args.steps)]
    dt = (time.perf_counter() - t0) / max(args.steps, 1)
    tok, qry = oracle_rates(hw, images, passes)
    line = {
        "metric": METRIC, "value": round(tok, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; shapes of the pages' 1024 px encoder and decoder workloads)",
        "config": {"workload": WORKLOAD, "images_per_gpu": args.batch, "sample_images_per_step": images,
                   "stage_tokens": [st["N"] for st in hw.stages], "stage_layers": hw.layer_counts},
        "impl": "reference",
        "knn": {"value": round(qry, 1), "unit": "queries/s"},
        "cpu_baseline": {"value": round(tok, 1), "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"per step {images} of {args.batch} images: each encoder stage's "
                                   f"clustering, neighbour table and one layer fwd + bwd (layer time x the "
                                   f"stage's layer count) and the decoder gather over the four stages; "
                                   f"fp64 C oracle"},
        "e2e": {"value": round(tok, 1), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- one part alone

def stage_calls(torch, acl, synth, device, stream, which: str, stage: int, B: int = IMAGES):
    """The library calls of one encoder stage's layer (which = "attn") or one decoder stage's
    gather (which = "knn") of the benchmark workload, as closures, after one eager call of
    each; returns (name, fn) pairs."""
    T = lambda x, dt=None: torch.from_numpy(np.ascontiguousarray(x)).to(device=device, dtype=dt)
    s = stage - 1
    if which == "attn":
        xy_np = synth.sweep_coords(B)[s]
        ab = synth.attn_sweep_layer(xy_np, s, 0)
        xy, bias = T(xy_np), T(ab.bias)
        q, k, v, do = (T(x, torch.bfloat16) for x in (ab.q, ab.k, ab.v, ab.do))
        cl = acl.acl_cluster(xy, stream=stream)
        nb = acl.acl_neighbors(xy, cl, stream=stream)
        o, lse = acl.acl_cluster_attn_fwd(q, k, v, xy, cl, nb, bias, ab.scale, stream=stream)
        ws = torch.empty((acl.acl_cluster_attn_workspace(ab.B, ab.N, ab.H, 8, 48),), dtype=torch.uint8,
                         device=device)
        grads = acl.acl_cluster_attn_bwd(q, k, v, xy, cl, nb, bias, ab.scale, o, do, lse, workspace=ws,
                                         stream=stream)
        return [("attn_fwd", lambda: acl.acl_cluster_attn_fwd(q, k, v, xy, cl, nb, bias, ab.scale, O=o, lse=lse,
                                                              stream=stream)),
                ("attn_bwd", lambda: acl.acl_cluster_attn_bwd(q, k, v, xy, cl, nb, bias, ab.scale, o, do, lse,
                                                              *grads, workspace=ws, stream=stream))]
    kb = synth.knn_decoder(B)[s]
    xy, f = T(kb.coords), T(kb.feats, torch.bfloat16)
    qq, pp, g = T(kb.queries), T(kb.p), T(kb.dout, torch.bfloat16)
    table = acl.acl_knn_table(xy, kb.GH, kb.GW, kb.K, stream=stream)
    out = acl.acl_knn_gather_fwd(qq, f, xy, table, pp, stream=stream)
    ws = torch.empty((acl.acl_knn_gather_workspace(kb.B, kb.Q, kb.N, kb.d, kb.K),), dtype=torch.uint8,
                     device=device)
    grads = acl.acl_knn_gather_bwd(qq, f, xy, table, pp, g, workspace=ws, stream=stream)
    return [("knn_table", lambda: acl.acl_knn_table(xy, kb.GH, kb.GW, kb.K, table=table, stream=stream)),
            ("knn_fwd", lambda: acl.acl_knn_gather_fwd(qq, f, xy, table, pp, out=out, stream=stream)),
            ("knn_bwd", lambda: acl.acl_knn_gather_bwd(qq, f, xy, table, pp, g, *grads, workspace=ws,
                                                       stream=stream))]


def attn_traffic_run(torch, acl, synth, device, stream, stage: int, B: int = IMAGES) -> dict:
    """One encoder stage's layer, copied until the copies exceed 3 x L2, run as the bench runs
    its layers: every copy's forward, then the backward of the copies in reverse order.  The
    last forward and the last backward then read inputs that have left L2, while each
    backward's key pass still finds what its query pass brought in, as in the bench."""
    T = lambda x, dt=None: torch.from_numpy(np.ascontiguousarray(x)).to(device=device, dtype=dt)
    s = stage - 1
    xy_np = synth.sweep_coords(B)[s]
    ab = synth.attn_sweep_layer(xy_np, s, 0)
    xy, bias = T(xy_np), T(ab.bias)
    cl = acl.acl_cluster(xy, stream=stream)
    nb = acl.acl_neighbors(xy, cl, stream=stream)
    ws = torch.empty((acl.acl_cluster_attn_workspace(ab.B, ab.N, ab.H, 8, 48),), dtype=torch.uint8, device=device)
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    layer_bytes = 8 * ab.B * ab.N * ab.H * 64
    n = max(2, math.ceil(3 * l2 / layer_bytes))
    base = [T(x, torch.bfloat16) for x in (ab.q, ab.k, ab.v, ab.do)]
    copies = [[t.clone() for t in base] for _ in range(n)]
    outs = []
    with torch.cuda.stream(stream):
        for q, k, v, do in copies:
            outs.append(acl.acl_cluster_attn_fwd(q, k, v, xy, cl, nb, bias, ab.scale, stream=stream))
        for (q, k, v, do), (o, lse) in reversed(list(zip(copies, outs))):
            acl.acl_cluster_attn_bwd(q, k, v, xy, cl, nb, bias, ab.scale, o, do, lse, workspace=ws, stream=stream)
    stream.synchronize()
    return {"stage": stage, "copies": n, "order": f"attn_fwd x {n}, then attn_bwd x {n} (query, key passes)"}


def attn_fwd_units(torch, acl, synth, device, stream, peaks: dict) -> dict:
    """The attention forward on the tensor cores (acl_cluster_attn_fwd) and on the FMA pipes
    only (acl_cluster_attn_fwd_ffma), one layer of 8 images x 2048 tokens x 4 heads: each
    called eagerly twice (the second launches are the ones to profile), then timed as CUDA
    graphs."""
    T = lambda x, dt=None: torch.from_numpy(np.ascontiguousarray(x)).to(device=device, dtype=dt)
    ab = synth.attn_stage1(B=8)
    xy, bias = T(ab.coords), T(ab.bias)
    q, k, v = (T(x, torch.bfloat16) for x in (ab.q, ab.k, ab.v))
    cl = acl.acl_cluster(xy, stream=stream)
    nb = acl.acl_neighbors(xy, cl, stream=stream)
    o, lse = acl.acl_cluster_attn_fwd(q, k, v, xy, cl, nb, bias, ab.scale, stream=stream)
    calls = {"tensor_core": lambda: acl.acl_cluster_attn_fwd(q, k, v, xy, cl, nb, bias, ab.scale, O=o, lse=lse,
                                                             stream=stream),
             "ffma": lambda: acl.acl_cluster_attn_fwd_ffma(q, k, v, xy, cl, nb, bias, ab.scale, O=o, lse=lse,
                                                           stream=stream)}
    with torch.cuda.stream(stream):
        for _ in range(2):
            for fn in calls.values():
                fn()
    stream.synchronize()
    by = attn_bytes(ab.B, ab.N, ab.H)["attn_fwd"]
    res = {"workload": "8 images x 2048 tokens, H = 4, M = 48"}
    for name, fn in calls.items():
        us = graph_time(torch, stream, fn, 20)
        res[name] = {"us": us, "frac": round(by / (us * 1e-6) / 1e9 / peaks["hbm_gbs"], 4)}
    return res


def run_only(args):
    """One part on cuda:0 and its timing dict as JSON.  attn_stage / knn_stage run one
    stage's calls of the benchmark workload eagerly (one warm call each, then one more:
    a short command for ncu, whose launch shapes match the bench's), then time each call
    as a CUDA graph."""
    import torch

    import off_grid_cluster_b200 as acl
    from off_grid_cluster_b200 import synth

    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    stream = torch.cuda.Stream(device)
    peaks = measured_peaks()
    if args.only == "token_merge":
        res = token_merge_times(torch, acl, synth, device, stream, peaks)
    elif args.only == "decoder":
        res = decoder_times(torch, acl, synth, device, stream, peaks, B=8)
    elif args.only == "configs":
        res = config_times(torch, acl, synth, device, stream, peaks)
    elif args.only == "attn_fwd_units":
        res = attn_fwd_units(torch, acl, synth, device, stream, peaks)
    elif args.only == "attn_traffic":
        res = attn_traffic_run(torch, acl, synth, device, stream, args.stage, args.batch)
    elif args.only == "knn_traffic":
        calls = stage_calls(torch, acl, synth, device, stream, "knn", args.stage, args.batch)
        with torch.cuda.stream(stream):
            for _, fn in calls:  # table, fwd, bwd in the bench's order (inputs above L2 size)
                fn()
        stream.synchronize()
        res = {"stage": args.stage, "launches": [name for name, _ in calls] * 2}
    else:
        which = "attn" if args.only == "attn_stage" else "knn"
        calls = stage_calls(torch, acl, synth, device, stream, which, args.stage, args.batch)
        with torch.cuda.stream(stream):
            for _, fn in calls:
                fn()
        stream.synchronize()
        res = {"stage": args.stage, "us": {name: graph_time(torch, stream, fn) for name, fn in calls}}
    print(json.dumps({"part": args.only, **res}))


def main(argv=None):
    args = parse_args(argv)
    rank = env_int("RANK", 0)
    world = env_int("WORLD_SIZE", 1)
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.only:
        run_only(args)
        return
    run_gpu(args, rank, world)


if __name__ == "__main__":
    main()
