#!/usr/bin/env python
"""Benchmark of the off-grid cluster attention + KNN gather hot path on B200.

One *step* is one pass of every step of the path over one batch of seeded
synthetic input shaped like the AFFMAE pages' stage-1 workload at 1024 px
(8 images, a 64 x 64 patch grid with a value-noise mask keeping 2048 tokens per
image, dim 128 = 4 heads x 32, C = 8, M = 48), followed by the decoder's
KNN gather over that stage (4096 queries per image at cell centre + U(-1,1)^2,
K = 8, d = 128, one temperature per head):

    attention chain: acl_cluster -> acl_neighbors -> acl_cluster_attn_fwd
                     -> acl_cluster_attn_bwd
    KNN chain:       acl_knn_table -> (acl_knn_gather_index || acl_knn_gather_fwd)
                     -> acl_knn_gather_bwd_indexed

`value` is whole-job tokens/s: images x tokens processed by all ranks per second
of the slowest rank's device time.  Inputs sit in HBM before timing starts;
S input sets rotate so that the sets total at least 4x the L2 size.  Each set's
two chains are captured as two CUDA graphs and replayed on two streams (the
attention chain, the longer one, at the higher priority; the inverse index on a
third stream inside the KNN graph).  CUDA events inside the graphs time every
call; the roofline figure is taken for the call with the largest share of the
step.  `e2e` runs the same calls through the C entry points with every step's
inputs copied in from pinned host buffers and all of its outputs read back, the
copies pipelined against the neighbouring steps' compute.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl acl|reference]

With --impl reference the fp64 CPU oracle is timed on the host cores on a
bounded sample of the same workload (rank 0 only under torchrun).
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
WORKLOAD = "stage1-1024px-b8-n2048-d128-h4-c8-m48 + decoder-knn-gather-q4096-k8"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
OPS = ("cluster", "neighbors", "attn_fwd", "attn_bwd", "knn_table", "knn_index", "knn_fwd",
       "knn_bwd")
KERNELS = {
    "cluster": ["cluster_kernel"],
    "neighbors": ["neighbors_kernel"],
    "attn_fwd": ["attn_fwd_union_kernel"],
    "attn_bwd": ["attn_bwd_query_union_kernel", "attn_bwd_key_union_kernel"],
    "knn_table": ["knn_table_kernel"],
    "knn_index": ["knn_csr_kernel"],
    "knn_fwd": ["knn_fwd_shared_kernel"],
    "knn_bwd": ["knn_bwd_query_shared_kernel", "knn_bwd_token_kernel"],
}
# DRAM bytes per launch measured by ncu for each call (sum over its kernels), with the
# sha256 of the CUDA source the counters were taken on; a stale hash reports null.
NCU_TRAFFIC: dict[str, tuple[float, str, str]] = {
    # call: (DRAM bytes read + written per launch, hash of the sources of its kernels, summary)
    "attn_fwd": (13202176.0, "77c27f1c2b1cfe11", "profiles/attn_kernels_step_workload.md"),
    "attn_bwd": (35377408.0, "77c27f1c2b1cfe11", "profiles/attn_kernels_step_workload.md"),
}
# the files whose code makes each call's kernels (the traffic goes stale when they change)
TRAFFIC_SOURCES = {"attn_fwd": ("attn.cu", "common.cuh"), "attn_bwd": ("attn.cu", "common.cuh")}


# --------------------------------------------------------------------------- helpers

def env_int(name: str, default: int) -> int:
    try:
        return int(os.environ.get(name, default))
    except ValueError:
        return default


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("acl", "reference"), default="acl")
    ap.add_argument("--batch", type=int, default=8, help="images per rank (default 8)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--serial", action="store_true",
                    help="run all seven calls on one stream (default: the attention and KNN "
                         "chains run as two concurrent branches of the step graph)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="bounded CPU work of the oracle baseline (seconds)")
    ap.add_argument("--only", choices=("token_merge", "decoder", "configs"), default=None,
                    help="time one extra part alone on one GPU and print its JSON (a short "
                         "command to profile under ncu); no bench line")
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
                "source": "measured (MEASURED_PEAKS.json)"}
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


def algorithmic_bytes(B, N, H, Q, d, K, GH, GW, C=8, M=48) -> dict:
    """Bytes each call must move at least once (every tensor counted once)."""
    G = (N + C - 1) // C
    per_tok_meta = 8 + 4 + 4 * M * G / N           # coords, cluster slot, neighbour-table share
    return {
        "cluster": B * N * (8 + 4),
        "neighbors": B * (N * 8 + G * C * 4 + G * M * 4),
        "attn_fwd": B * N * (H * (3 * 64 + 64 + 4) + per_tok_meta) + H * 12,
        "attn_bwd": B * N * (H * (4 * 64 + 4 + 3 * 64) + per_tok_meta) + 2 * H * 12,
        "knn_table": B * (N * 8 + GH * GW * K * 4),
        "knn_index": B * (Q * 8 + GH * GW * K * 4 + Q * K * 4 + (N + 1) * 4),
        "knn_fwd": B * (Q * (8 + 4 * K + 2 * d) + N * (2 * d + 8)) + 4 * d // 32,
        "knn_bwd": B * (Q * (8 + 4 * K + 2 * d + 8) + N * (2 * d + 8 + 2 * d)) + 8 * d // 32,
    }


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


# --------------------------------------------------------------------------- GPU arm

class StepSet:
    """Device buffers of one input set plus the seven library calls of a step."""

    def __init__(self, sb, device, acl, torch):
        a, k = sb.attn, sb.knn
        T = lambda x, dt=None: torch.from_numpy(np.ascontiguousarray(x)).to(device=device, dtype=dt)
        bf = torch.bfloat16
        self.acl, self.torch = acl, torch
        self.B, self.N, self.H, self.Q, self.d, self.K = a.B, a.N, a.H, k.Q, k.d, k.K
        self.GH, self.GW, self.scale = k.GH, k.GW, a.scale
        self.inputs = {
            "coords": T(a.coords), "q": T(a.q, bf), "k": T(a.k, bf), "v": T(a.v, bf),
            "do": T(a.do, bf), "bias": T(a.bias), "queries": T(k.queries),
            "feats": T(k.feats, bf), "dout": T(k.dout, bf), "p": T(k.p),
        }
        B, N, H, G = self.B, self.N, self.H, (self.N + 7) // 8
        e = lambda shape, dt: torch.empty(shape, dtype=dt, device=device)
        self.outputs = {
            "clusters": e((B, G, 8), torch.int32), "nbr": e((B, G, 48), torch.int32),
            "o": e((B, N, H, 32), bf), "lse": e((B, N, H), torch.float32),
            "dq": e((B, N, H, 32), bf), "dk": e((B, N, H, 32), bf), "dv": e((B, N, H, 32), bf),
            "dbias": e((H, 3), torch.float32),
            "table": e((B, self.GH, self.GW, self.K), torch.int32),
            "out": e((B, self.Q, self.d), bf), "dfeats": e((B, N, self.d), bf),
            "dqueries": e((B, self.Q, 2), torch.float32), "dp": e((self.d // 32,), torch.float32),
        }
        self.ws_attn = e((acl.acl_cluster_attn_workspace(B, N, H, 8, 48),), torch.uint8)
        self.ws_knn = e((acl.acl_knn_gather_workspace(B, self.Q, N, self.d, self.K),), torch.uint8)

    def bytes(self) -> int:
        ts = list(self.inputs.values()) + list(self.outputs.values()) + [self.ws_attn, self.ws_knn]
        return sum(t.numel() * t.element_size() for t in ts)

    def op(self, name: str, stream, kind: int = 0):
        i, o, acl = self.inputs, self.outputs, self.acl
        if name == "cluster":
            acl.acl_cluster(i["coords"], 8, clusters=o["clusters"], stream=stream)
        elif name == "neighbors":
            acl.acl_neighbors(i["coords"], o["clusters"], 48, nbr=o["nbr"], stream=stream)
        elif name == "attn_fwd":
            acl.acl_cluster_attn_fwd(i["q"], i["k"], i["v"], i["coords"], o["clusters"], o["nbr"],
                                     i["bias"], self.scale, O=o["o"], lse=o["lse"], stream=stream)
        elif name == "attn_bwd":
            acl.acl_cluster_attn_bwd(i["q"], i["k"], i["v"], i["coords"], o["clusters"], o["nbr"],
                                     i["bias"], self.scale, o["o"], i["do"], o["lse"], o["dq"],
                                     o["dk"], o["dv"], o["dbias"], workspace=self.ws_attn,
                                     stream=stream)
        elif name == "knn_table":
            acl.acl_knn_table(i["coords"], self.GH, self.GW, self.K, table=o["table"], stream=stream)
        elif name == "knn_fwd":
            acl.acl_knn_gather_fwd(i["queries"], i["feats"], i["coords"], o["table"], i["p"],
                                   out=o["out"], stream=stream, kind=kind)
        elif name == "knn_index":
            acl.acl_knn_gather_index(i["queries"], o["table"], self.N, self.d, self.ws_knn,
                                     stream=stream)
        elif name == "knn_bwd":
            acl.acl_knn_gather_bwd_indexed(i["queries"], i["feats"], i["coords"], o["table"],
                                           i["p"], i["dout"], self.ws_knn, dfeats=o["dfeats"],
                                           dqueries=o["dqueries"], dp=o["dp"], stream=stream,
                                           kind=kind)
        else:
            raise KeyError(name)

    ATTN = ("cluster", "neighbors", "attn_fwd", "attn_bwd")
    KNN = ("knn_table", "knn_index", "knn_fwd", "knn_bwd")

    def chain(self, names, stream, events=None, s3=None):
        """The calls of one chain in order on `stream`; with s3 the inverse index runs on
        s3 after the table and the indexed backward waits for it."""
        torch = self.torch
        tab, idx = torch.cuda.Event(), torch.cuda.Event()
        for name in names:
            j = OPS.index(name)
            st = s3 if (name == "knn_index" and s3 is not None) else stream
            if name == "knn_index" and s3 is not None:
                s3.wait_event(tab)
            if name == "knn_bwd" and s3 is not None:
                stream.wait_event(idx)
            if events is not None:
                events[2 * j].record(st)
            self.op(name, st)
            if events is not None:
                events[2 * j + 1].record(st)
            if name == "knn_table":
                tab.record(stream)
            if name == "knn_index":
                idx.record(st)

    def step(self, stream, events=None, streams=None):
        """The eight calls.  With streams = (s2, s3) the KNN chain (table -> gather fwd ->
        indexed bwd; the inverse index on s3 after the table) runs on s2 concurrently with
        the attention chain (cluster -> neighbours -> attn fwd -> bwd) on stream;
        events[2j], events[2j+1] bracket call j on its stream."""
        if streams is None:
            self.chain(OPS, stream, events)
            return
        torch = self.torch
        s2, s3 = streams
        fork, join = torch.cuda.Event(), torch.cuda.Event()
        fork.record(stream)
        s2.wait_event(fork)
        self.chain(StepSet.ATTN, stream, events)
        self.chain(StepSet.KNN, s2, events, s3=s3)
        join.record(s2)
        stream.wait_event(join)


def run_gpu(args, rank: int, world: int):
    import torch
    import torch.distributed as dist

    import off_grid_cluster_b200 as acl
    from off_grid_cluster_b200 import synth

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
    sb = synth.step_batch(B=per_rank, image0=first)
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    base = StepSet(sb, device, acl, torch)
    set_bytes = base.bytes()
    n_sets = max(2, math.ceil(4 * l2 / set_bytes))
    sets = [base] + [StepSet(sb, device, acl, torch) for _ in range(n_sets - 1)]
    # the attention chain is the longer one: its stream gets the higher priority so its
    # CTAs are scheduled first and the KNN chain fills the remaining SMs
    # (a lower number is a higher priority; out-of-range values map to the nearest valid one)
    stream = torch.cuda.Stream(device, priority=-100)
    streams = None if args.serial else (torch.cuda.Stream(device, priority=0),
                                        torch.cuda.Stream(device, priority=0))

    # eager warm-up of every call (kernel attributes, lazy module loading), then capture
    with torch.cuda.stream(stream):
        for s in sets:
            s.step(stream)
    stream.synchronize()
    n_ev = 2 * len(OPS)
    graphs, events = [], []
    launches0 = acl.acl_launch_count()
    for s in sets:
        evs = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(n_ev)]
        if streams is None:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                s.step(stream, evs)
            graphs.append((g,))
        else:
            # one graph per chain, replayed on its own stream (graph nodes run at the
            # priority of the stream the graph is launched into)
            ga, gk = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
            with torch.cuda.graph(ga, stream=stream):
                s.chain(StepSet.ATTN, stream, evs)
            with torch.cuda.graph(gk, stream=streams[0]):
                s.chain(StepSet.KNN, streams[0], evs, s3=streams[1])
            graphs.append((ga, gk))
        events.append(evs)
    launches_per_step = (acl.acl_launch_count() - launches0) // len(sets)
    # single-stream graphs of the same sets: the per-call breakdown and the roofline come
    # from these, where no call shares the GPU with another
    serial_graphs, serial_events = [], []
    if streams is None:
        serial_graphs, serial_events = [gs[0] for gs in graphs], events
    else:
        for s in sets:
            evs = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(n_ev)]
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                s.step(stream, evs)
            serial_graphs.append(g)
            serial_events.append(evs)
    torch.cuda.synchronize()

    def replay(i):
        gs = graphs[i % n_sets]
        if len(gs) == 1:
            with torch.cuda.stream(stream):
                gs[0].replay()
            return
        with torch.cuda.stream(stream):
            gs[0].replay()
        with torch.cuda.stream(streams[0]):
            gs[1].replay()

    def fork():
        if streams is not None:
            streams[0].wait_stream(stream)

    def join():
        if streams is not None:
            stream.wait_stream(streams[0])

    fork()
    for w in range(args.warmup):
        replay(w)
    join()
    torch.cuda.synchronize()

    props = torch.cuda.get_device_properties(device)
    uuid = getattr(props, "uuid", None)
    clocks = ClockSampler(f"GPU-{uuid}" if uuid is not None else str(local)).start()
    barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    fork()
    for it in range(args.steps):
        replay(it)
    join()
    t1.record(stream)
    torch.cuda.synchronize()
    barrier()
    step_ms_local = t0.elapsed_time(t1) / max(args.steps, 1)
    def per_call(evsets, used):
        acc = np.zeros(len(OPS))
        for s_i in range(used):
            ev = evsets[s_i]
            acc += np.array([ev[2 * j].elapsed_time(ev[2 * j + 1]) for j in range(len(OPS))])
        return acc / max(used, 1)

    # per-call durations inside the timed region (the last replay of every set); with
    # concurrent chains each includes the time it shared the GPU with the other chain
    per_op_concurrent = per_call(events, min(n_sets, args.steps))
    # per-call durations with one call at a time: 2 rounds over the sets, after warm-up
    with torch.cuda.stream(stream):
        for it in range(3 * n_sets):
            serial_graphs[it % n_sets].replay()
    torch.cuda.synchronize()
    per_op = per_call(serial_events, n_sets)
    # the inverse-power weight kernel (the original AFF weighting) on the same gathers:
    # forward and backward of set 0, one call at a time
    inv_us = {}
    s0 = sets[0]
    for name in ("knn_fwd", "knn_bwd"):
        for kind, key in ((acl.ACL_KNN_EXP, "exp"), (acl.ACL_KNN_INVPOW, "invpow")):
            inv_us[f"{name}_{key}"] = graph_time(
                torch, stream, lambda: s0.op(name, stream, kind=kind), 20)
    hires = hires_gather_times(torch, acl, synth, device, stream) if world == 1 else None
    merge_us = (token_merge_times(torch, acl, synth, sb, device, stream, measured_peaks())
                if world == 1 else None)
    dec_us = decoder_times(torch, acl, synth, device, stream, measured_peaks()) if world == 1 else None
    cfg_us = config_times(torch, acl, synth, device, stream, measured_peaks()) if world == 1 else None
    # keep the same load on the GPU until the clock sampler has several samples
    t_wall = time.time()
    it = 0
    while time.time() - t_wall < 0.8:
        fork()
        for _ in range(64):
            replay(it)
            it += 1
        join()
        stream.synchronize()
    torch.cuda.synchronize()
    clk = clocks.stop()

    step_ms = max_over_ranks(step_ms_local, world, device)
    B, N, Q = per_rank, sb.attn.N, sb.knn.Q
    tokens = world * B * N
    value = tokens / (step_ms * 1e-3)
    abytes = algorithmic_bytes(B, N, sb.attn.H, Q, sb.knn.d, sb.knn.K, sb.knn.GH, sb.knn.GW)
    dom = int(np.argmax(per_op))
    dom_name = OPS[dom]
    peaks = measured_peaks()
    achieved = abytes[dom_name] / (per_op[dom] * 1e-3) / 1e9
    traffic = None
    traffic_src = None
    if dom_name in NCU_TRAFFIC and NCU_TRAFFIC[dom_name][1] == source_hash(TRAFFIC_SOURCES[dom_name]):
        traffic, traffic_src = NCU_TRAFFIC[dom_name][0], NCU_TRAFFIC[dom_name][2]
    breakdown = {}
    for j, name in enumerate(OPS):
        gbs = abytes[name] / (per_op[j] * 1e-3) / 1e9
        breakdown[name] = {"us": round(per_op[j] * 1e3, 2), "alg_MB": round(abytes[name] / 1e6, 3),
                           "GB_s": round(gbs, 1), "frac": round(gbs / peaks["hbm_gbs"], 4)}
    attn_ms = per_op[OPS.index("attn_fwd")] + per_op[OPS.index("attn_bwd")]
    knn_ms = sum(per_op[OPS.index(n)] for n in ("knn_index", "knn_fwd", "knn_bwd"))

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, base, stream, streams, torch, acl, tokens_per_step=world * B * N,
                      sb=sb, device=device)
        e2e_ms = max_over_ranks(e2e.pop("_ms"), world, device)
        e2e["value"] = round(world * B * N / (e2e_ms * 1e-3), 1)
        e2e["ms_per_step"] = round(e2e_ms, 4)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args, sb)

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_ms, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; shapes of the pages' 1024 px stage-1 workload)",
        "config": {"workload": WORKLOAD, "images_per_gpu": B, "tokens_per_image": N,
                   "heads": sb.attn.H, "head_dim": 32, "C": 8, "M": 48,
                   "queries_per_image": Q, "knn_d": sb.knn.d, "K": sb.knn.K, "grid": [64, 64],
                   "l2": f"rotating {n_sets} input sets, {n_sets * set_bytes / 1e6:.0f} MB total "
                         f">= 4 x L2 ({l2 / 1e6:.0f} MB)",
                   "timing": "CUDA graph per set, CUDA events on the launching stream",
                   "streams": "1" if args.serial else "3 (attention chain at high priority)",
                   "parallelism": f"replicas x{world} (images sharded, no collective)"},
        "parts": {
            "knn_queries_per_s": round(world * B * Q / (step_ms * 1e-3), 1),
            "cluster_attn_fwd_bwd_tokens_per_s": round(world * B * N / (attn_ms * 1e-3), 1),
            "knn_gather_fwd_bwd_queries_per_s": round(world * B * Q / (knn_ms * 1e-3), 1),
            "per_call": breakdown,
            "per_call_note": "one call at a time (single-stream graphs of the same sets, "
                             "after the timed region); the step overlaps the two chains",
            "per_call_concurrent_us": {n: round(per_op_concurrent[j] * 1e3, 2)
                                       for j, n in enumerate(OPS)},
            "knn_kernels_us": {**inv_us, "note": "exponential and inverse-power weight kernels "
                               "on the same gathers (set 0, one graph per call, L2-warm)"},
            "hires_gather_us": hires,
            "token_merge_us": merge_us,
            "decoder_us": dec_us,
            "configs": cfg_us,
        },
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                     "traffic": traffic, "traffic_unit": "bytes per launch (ncu DRAM read + write)",
                     "traffic_source": traffic_src, "kernel": f"acl_{dom_name} ({', '.join(KERNELS[dom_name])})",
                     "alg_bytes_per_launch": int(abytes[dom_name]),
                     "launch_us": round(per_op[dom] * 1e3, 3), "peak_source": peaks["source"]},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": int(launches_per_step * args.steps),
        "clocks": clk,
    }
    for gs in graphs:
        for g in gs:
            g.reset()
    if streams is not None:
        for g in serial_graphs:
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


def merge_bytes(B: int, N: int, d: int, k: int) -> dict:
    """Algorithmic bytes of token merging, every tensor once: forward reads features (2d B)
    and coordinates (8 B) per token and writes score, assignment (8 B) per token and the merged
    row (2d + 8 B) and anchor id per anchor; backward reads features, coordinates, score and
    assignment and writes dfeats and dcoords per token (4d + 24 B), reads dmerged (2d + 8 B)
    per anchor."""
    T, A = B * N, B * k
    return {"fwd": T * (2 * d + 16) + A * (2 * d + 12), "bwd": T * (4 * d + 24) + A * (2 * d + 8)}


def token_merge_times(torch, acl, synth, sb, device, stream, peaks: dict, reps: int = 10) -> dict:
    """Token merging of the stage-1 tokens into round(0.4 N) anchors (d = 128, hidden 32),
    forward and backward, one call at a time with CUDA events; GB/s of the algorithmic bytes
    and the fraction of the measured HBM copy bandwidth."""
    mb = synth.merge_batch(sb.attn.coords, d=128)
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


def run_e2e(args, s: StepSet, stream, streams, torch, acl, tokens_per_step: int, sb=None,
            device=None) -> dict:
    """The step through the public entry points from pinned host memory, copies inside.

    Every step copies its inputs host -> device and its results device -> host.  Two
    device sets and two copy streams pipeline the steps: the inputs of step k + 1 travel
    in and the results of step k - 1 travel out while step k computes (PCIe is full
    duplex), with events ordering each set's copy-in, compute and copy-out."""
    sets = [s, StepSet(sb, device, acl, torch)] if sb is not None else [s, s]
    hin = {k: torch.empty_like(v, device="cpu").pin_memory() for k, v in s.inputs.items()}
    for k, v in s.inputs.items():
        hin[k].copy_(v)
    hout = [{k: torch.empty_like(v, device="cpu").pin_memory() for k, v in s.outputs.items()}
            for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in hin.values())
    d2h = sum(t.numel() * t.element_size() for t in hout[0].values())
    cp_in, cp_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
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
            for name, v in hin.items():
                S.inputs[name].copy_(v, non_blocking=True)
        ev_in[i].record(cp_in)
        stream.wait_event(ev_in[i])
        if recorded[i]:
            stream.wait_event(ev_out[i])    # step k - 2's results have left set i
        with torch.cuda.stream(stream):
            S.step(stream, None, streams)
        ev_done[i].record(stream)
        cp_out.wait_event(ev_done[i])
        with torch.cuda.stream(cp_out):
            for name, v in S.outputs.items():
                hout[i][name].copy_(v, non_blocking=True)
        ev_out[i].record(cp_out)
        recorded[i] = True

    def drain():
        stream.wait_stream(cp_out)
        stream.wait_stream(cp_in)

    for k in range(4):
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
    return {"value": tokens_per_step / (ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "steps": n, "_ms": ms,
            "pipelining": "2 device sets, copy-in / compute / copy-out streams"}


# --------------------------------------------------------------------------- CPU oracle

def oracle_step(sb, images: slice | None = None) -> None:
    """One pass of the hot path through the fp64 oracle (optionally on a subset of images)."""
    import oracle
    a, k = sb.attn, sb.knn
    sl = images if images is not None else slice(None)
    xy = a.coords[sl]
    cl = oracle.cluster(xy, 8)
    nb = oracle.neighbors(xy, cl, 48)
    oracle.attn_fwd(a.q[sl], a.k[sl], a.v[sl], xy, cl, nb, a.bias, a.scale)
    oracle.attn_bwd(a.q[sl], a.k[sl], a.v[sl], xy, cl, nb, a.bias, a.scale, a.do[sl])
    table = oracle.knn_table(k.coords[sl], k.GH, k.GW, k.K)
    oracle.knn_fwd(k.queries[sl], k.feats[sl], k.coords[sl], table, k.p)
    oracle.knn_bwd(k.queries[sl], k.feats[sl], k.coords[sl], table, k.p, k.dout[sl])


def cpu_baseline(args, sb) -> dict:
    import oracle
    cores = oracle.set_threads(os.cpu_count() or 1)
    B, N = sb.attn.B, sb.attn.N
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle_step(sb)
        reps += 1
        if time.perf_counter() - t0 >= args.cpu_seconds:
            break
    dt = time.perf_counter() - t0
    # the same on one thread, over the first image only (a few seconds)
    oracle.set_threads(1)
    reps1, t1 = 0, time.perf_counter()
    while True:
        oracle_step(sb, images=slice(0, 1))
        reps1 += 1
        if time.perf_counter() - t1 >= max(2.0, args.cpu_seconds / 4):
            break
    dt1 = time.perf_counter() - t1
    oracle.set_threads(cores)
    return {"value": round(reps * B * N / dt, 1), "unit": "tokens/s", "cores": cores,
            "kind": "oracle",
            "sample": f"{reps} full step(s) of the workload ({B} images), fp64 C, OpenMP over images",
            "value_1_thread": round(reps1 * N / dt1, 1),
            "sample_1_thread": f"{reps1} step(s) of one image on 1 thread"}


def run_reference(args, rank: int, world: int) -> None:
    if rank != 0:
        return
    import oracle
    from off_grid_cluster_b200 import synth
    cores = oracle.set_threads(os.cpu_count() or 1)
    sb = synth.step_batch(B=args.batch)
    B, N = sb.attn.B, sb.attn.N
    # bounded sample: images per step chosen so that warm-up + steps take about two minutes
    t = time.perf_counter()
    oracle_step(sb, slice(0, 1))
    t_img = max(time.perf_counter() - t, 1e-3)
    total = args.steps + args.warmup
    per_step = int(max(1, min(B, 120.0 / (total * t_img))))
    sl = slice(0, per_step)
    for _ in range(args.warmup):
        oracle_step(sb, sl)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(sb, sl)
    dt = (time.perf_counter() - t0) / max(args.steps, 1)
    value = per_step * N / dt
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; shapes of the pages' 1024 px stage-1 workload)",
        "config": {"workload": WORKLOAD, "images_per_gpu": B, "tokens_per_image": N,
                   "sample_images_per_step": per_step},
        "impl": "reference",
        "cpu_baseline": {"value": round(value, 1), "unit": "tokens/s", "cores": cores,
                         "kind": "oracle",
                         "sample": f"{per_step} of {B} images per step, fp64 C oracle"},
        "e2e": {"value": round(value, 1), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


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


def config_times(torch, acl, synth, device, stream, peaks: dict, reps: int = 10) -> dict:
    """The five seeded configurations' hot-path calls, one call at a time, each captured as a
    CUDA graph and timed with CUDA events: cluster attention fwd + bwd tokens/s per layer
    (configs 1-4; the sweep as sum over stages of its layers x one layer's time, all layers of
    a stage having the same shapes) and the KNN gather fwd + bwd queries/s over the four stages
    (config 5), each with its fraction of the measured HBM copy bandwidth on the algorithmic
    bytes (`algorithmic_bytes`).  Clustering, neighbour and KNN tables are timed beside."""
    T = lambda x, dt=None: torch.from_numpy(np.ascontiguousarray(x)).to(device=device, dtype=dt)
    timed = lambda fn: graph_time(torch, stream, fn, reps)
    hbm = peaks["hbm_gbs"]

    def attn_layer(ab):
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
        by = algorithmic_bytes(ab.B, ab.N, ab.H, 1, 32, 8, 1, 1)
        return {"tokens": ab.B * ab.N, "cluster_us": t_cl, "neighbors_us": t_nb, "fwd_us": t_f, "bwd_us": t_b,
                "alg_MB": round((by["attn_fwd"] + by["attn_bwd"]) / 1e6, 2)}

    def attn_summary(r, layers=1):
        t = (r["fwd_us"] + r["bwd_us"]) * 1e-6
        gbs = r["alg_MB"] * 1e6 / t / 1e9
        return {"tokens_per_s_fwd_bwd": round(r["tokens"] / t, 1), "GB_s": round(gbs, 1),
                "frac": round(gbs / hbm, 4), **r}

    res = {}
    c1 = attn_summary(attn_layer(synth.attn_tiny()))
    c1["config"] = "tiny: 1 image, 16 x 16 grid, H = 4 (launch-bound)"
    res["c1"] = c1
    c2 = attn_summary(attn_layer(synth.attn_stage1(B=8)))
    c2["config"] = "stage 1: 8 images x 2048 tokens, H = 4"
    res["c2"] = c2
    c3 = attn_summary(attn_layer(synth.attn_stage3(B=64)))
    c3["config"] = "stage 3: 64 images x 328 tokens, H = 16"
    res["c3"] = c3
    coords = synth.sweep_coords(B=16)
    tot_t, tot_tok, tot_b, stages = 0.0, 0, 0.0, []
    for st, xy in enumerate(coords):
        r = attn_layer(synth.attn_sweep_layer(xy, st, 0))
        L = synth.SWEEP_LAYERS[st]
        t = (r["fwd_us"] + r["bwd_us"]) * 1e-6
        tot_t += L * t
        tot_tok += L * r["tokens"]
        tot_b += L * r["alg_MB"] * 1e6
        stages.append({"stage": st + 1, "N": xy.shape[1], "H": synth.SWEEP_DIMS[st] // 32, "layers": L,
                       "fwd_us": r["fwd_us"], "bwd_us": r["bwd_us"], "cluster_us": r["cluster_us"],
                       "neighbors_us": r["neighbors_us"],
                       "frac": round(r["alg_MB"] * 1e6 / t / 1e9 / hbm, 4)})
    res["c4"] = {"config": "sweep: 16 images, stages 2048/819/328/131, layers 3/4/16/2",
                 "tokens_per_s_fwd_bwd": round(tot_tok / tot_t, 1), "sweep_us": round(tot_t * 1e6, 1),
                 "GB_s": round(tot_b / tot_t / 1e9, 1), "frac": round(tot_b / tot_t / 1e9 / hbm, 4),
                 "stages": stages}
    kt, kq, kb, kst = 0.0, 0, 0.0, []
    for st, kbt in enumerate(synth.knn_decoder(B=16)):
        xy, f = T(kbt.coords), T(kbt.feats, torch.bfloat16)
        qq, pp, dout = T(kbt.queries), T(kbt.p), T(kbt.dout, torch.bfloat16)
        table = acl.acl_knn_table(xy, kbt.GH, kbt.GW, kbt.K, stream=stream)
        out = acl.acl_knn_gather_fwd(qq, f, xy, table, pp, stream=stream)
        ws = torch.empty((acl.acl_knn_gather_workspace(kbt.B, kbt.Q, kbt.N, kbt.d, kbt.K),),
                         dtype=torch.uint8, device=device)
        t_t = timed(lambda: acl.acl_knn_table(xy, kbt.GH, kbt.GW, kbt.K, table=table, stream=stream))
        t_f = timed(lambda: acl.acl_knn_gather_fwd(qq, f, xy, table, pp, out=out, stream=stream))
        t_b = timed(lambda: acl.acl_knn_gather_bwd(qq, f, xy, table, pp, dout, workspace=ws, stream=stream))
        by = algorithmic_bytes(kbt.B, kbt.N, 1, kbt.Q, kbt.d, kbt.K, kbt.GH, kbt.GW)
        bts = by["knn_fwd"] + by["knn_bwd"]
        t = (t_f + t_b) * 1e-6
        kt += t
        kq += kbt.B * kbt.Q
        kb += bts
        kst.append({"stage": st + 1, "N": kbt.N, "d": kbt.d, "table_us": t_t, "fwd_us": t_f, "bwd_us": t_b,
                    "frac": round(bts / t / 1e9 / hbm, 4)})
    res["c5"] = {"config": "decoder gather: 16 images x 4096 queries over the four stages, K = 8",
                 "queries_per_s_fwd_bwd": round(kq / kt, 1), "gather_us": round(kt * 1e6, 1),
                 "GB_s": round(kb / kt / 1e9, 1), "frac": round(kb / kt / 1e9 / hbm, 4), "stages": kst}
    return res


def run_only(args):
    """One extra part on cuda:0 (an eager call, then each call captured as a CUDA graph and
    replayed between CUDA events); prints its timing dict."""
    import torch

    import off_grid_cluster_b200 as acl
    from off_grid_cluster_b200 import synth

    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    stream = torch.cuda.Stream(device)
    if args.only == "token_merge":
        sb = synth.step_batch(B=args.batch)
        res = token_merge_times(torch, acl, synth, sb, device, stream, measured_peaks())
    elif args.only == "decoder":
        res = decoder_times(torch, acl, synth, device, stream, measured_peaks(), B=args.batch)
    else:
        res = config_times(torch, acl, synth, device, stream, measured_peaks())
    print(json.dumps({"part": args.only, **res}))


if __name__ == "__main__":
    main()
