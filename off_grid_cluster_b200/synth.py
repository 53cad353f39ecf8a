"""Seeded synthetic inputs for the off-grid cluster attention and KNN gather path.

This module only draws numbers and lays them out: it holds no step of the
method (no clustering, no distances, no softmax).  Both the CUDA path's tests
and benchmark and the CPU oracle's tests take their inputs from here, so the
two sides see identical values.

Generator
---------
SplitMix64 (Steele, Lea, Flood 2014): state_i = seed + i * 0x9E3779B97F4A7C15
(i = 1, 2, ...), each state mixed by the published two-multiply finaliser.
Every (workload, image, tensor) triple gets its own stream seed.  Uniforms take
the top 53 bits; normals are Box-Muller in fp64; bf16 tensors are fp64 ->
fp32 -> bf16, both roundings to nearest-even.  bf16 tensors are returned as
float32 numpy arrays whose values are exactly representable in bf16.

Workloads (shapes follow the AFFMAE pages' running example: a 64x64 patch grid,
about half of it visible, stage sizes 2048 -> 819 -> 328 -> 131 at a 40%
retention rate, dims 128/256/512/768, 32-channel heads):

* ``tiny``     -- 1 image, 16x16 grid, Bernoulli(0.5) mask, dim 128, 4 heads.
* ``stage1``   -- 8 images, 64x64 grid, value-noise mask keeping the 2048
                  lowest cells, dim 128, 4 heads.
* ``stage3``   -- 64 images, 328 tokens drawn from each image's stage-1 set,
                  dim 512, 16 heads.
* ``sweep``    -- 16 images, four stages 2048/819/328/131 by nested random
                  subsets, dims 128/256/512/768, layers 3/4/16/2.
* ``decoder``  -- the sweep's four stages as KNN sources, 4096 queries per
                  image at cell centre + U(-1,1)^2, K = 8, p_h ~ U(0.5, 4).
* ``dec_layer`` -- the decoder: the 2048 masked cells of each image as queries,
                  four layers over the sweep's stages coarse to fine (D = 256).
* ``step``     -- the stage1 batch plus a decoder gather over that same stage
                  (4096 queries per image, d = 128): one pass of every step.

Coordinates are fp32 in grid-cell units: x is the column, y the row, and cell
(r, c) covers [c, c+1) x [r, r+1) with centre (c + 0.5, r + 0.5).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

# tensor tags: one independent stream per (workload, image, tag)
TAG_MASK, TAG_JITTER, TAG_SUBSET, TAG_BIAS = 1, 2, 3, 4
TAG_Q, TAG_K, TAG_V, TAG_DO = 10, 11, 12, 13
TAG_QUERY, TAG_FEAT, TAG_P, TAG_DOUT = 20, 21, 22, 23

WORKLOAD_ID = {"tiny": 1, "stage1": 2, "stage3": 3, "sweep": 4, "decoder": 5,
               "step": 6, "hires": 7, "merge": 8, "dec_layer": 9}
TAG_F0, TAG_WOFF, TAG_WO, TAG_DF = 30, 31, 32, 33


def _mix(z: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        return z ^ (z >> np.uint64(31))


def splitmix64(seed: int, n: int) -> np.ndarray:
    """First ``n`` outputs of SplitMix64 started at ``seed`` (uint64 array)."""
    i = np.arange(1, n + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + i * _GAMMA
    return _mix(z)


def stream_seed(workload: int, image: int, tag: int, sub: int = 0) -> int:
    """Seed of the stream for one (workload, image, tensor[, layer]) tuple."""
    base = np.array([(((1000 * workload + image) << 24) + (tag << 12) + sub)],
                    dtype=np.uint64)
    return int(_mix(base)[0])


def uniform(seed: int, n: int, lo: float = 0.0, hi: float = 1.0) -> np.ndarray:
    """``n`` fp64 uniforms in [lo, hi) from the top 53 bits of SplitMix64."""
    u = (splitmix64(seed, n) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
    return lo + (hi - lo) * u


def normal(seed: int, n: int) -> np.ndarray:
    """``n`` fp64 standard normals, Box-Muller on consecutive uniform pairs."""
    m = (n + 1) // 2
    u = uniform(seed, 2 * m)
    u1 = 1.0 - u[0::2]                      # (0, 1]: log is finite
    u2 = u[1::2]
    r = np.sqrt(-2.0 * np.log(u1))
    z = np.empty(2 * m, dtype=np.float64)
    z[0::2] = r * np.cos(2.0 * np.pi * u2)
    z[1::2] = r * np.sin(2.0 * np.pi * u2)
    return z[:n]


def round_bf16(x: np.ndarray) -> np.ndarray:
    """fp64/fp32 -> fp32 -> bf16 (both nearest-even), returned as float32."""
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    b = f.view(np.uint32).astype(np.uint64)
    b = (b + np.uint64(0x7FFF) + ((b >> np.uint64(16)) & np.uint64(1))) & np.uint64(0xFFFF0000)
    return b.astype(np.uint32).view(np.float32).reshape(f.shape)


def normal_bf16(seed: int, shape) -> np.ndarray:
    n = int(np.prod(shape))
    return round_bf16(normal(seed, n)).reshape(shape)


# --------------------------------------------------------------------------
# masks and coordinates
# --------------------------------------------------------------------------

def bernoulli_mask(seed: int, gh: int, gw: int, p: float = 0.5) -> np.ndarray:
    """Visible cells (raster ids, ascending) of an i.i.d. Bernoulli(p) mask."""
    u = uniform(seed, gh * gw)
    return np.nonzero(u < p)[0].astype(np.int64)


def _fade(t: np.ndarray) -> np.ndarray:
    # Perlin's quintic 6t^5 - 15t^4 + 10t^3
    return t * t * t * (t * (t * 6.0 - 15.0) + 10.0)


def value_noise(seed: int, gh: int, gw: int, lattice: int = 8) -> np.ndarray:
    """Value noise sampled at the cell centres of a gh x gw grid.

    U(0,1) values on a (gh/lattice + 1) x (gw/lattice + 1) lattice, one
    lattice step every ``lattice`` cells, interpolated bilinearly with the
    quintic fade.  Returns a (gh, gw) fp64 array.
    """
    ly, lx = gh // lattice + 1, gw // lattice + 1
    lat = uniform(seed, ly * lx).reshape(ly, lx)
    r = (np.arange(gh, dtype=np.float64) + 0.5) / lattice
    c = (np.arange(gw, dtype=np.float64) + 0.5) / lattice
    r0 = np.floor(r).astype(np.int64)
    c0 = np.floor(c).astype(np.int64)
    tr = _fade(r - r0)[:, None]
    tc = _fade(c - c0)[None, :]
    v00 = lat[r0][:, c0]
    v01 = lat[r0][:, c0 + 1]
    v10 = lat[r0 + 1][:, c0]
    v11 = lat[r0 + 1][:, c0 + 1]
    top = v00 + (v01 - v00) * tc
    bot = v10 + (v11 - v10) * tc
    return top + (bot - top) * tr


def noise_mask(seed: int, gh: int, gw: int, keep: int, lattice: int = 8) -> np.ndarray:
    """Visible cells: the ``keep`` lowest value-noise cells, ties by cell id."""
    v = value_noise(seed, gh, gw, lattice).reshape(-1)
    order = np.lexsort((np.arange(v.size), v))
    return np.sort(order[:keep]).astype(np.int64)


def jittered_coords(seed: int, cells: np.ndarray, gw: int) -> np.ndarray:
    """(x, y) = cell centre + U(-0.5, 0.5)^2 for each visible cell, fp32 [n, 2]."""
    n = cells.size
    u = uniform(seed, 2 * n, -0.5, 0.5).reshape(n, 2)
    r = (cells // gw).astype(np.float64)
    c = (cells % gw).astype(np.float64)
    xy = np.stack([c + 0.5 + u[:, 0], r + 0.5 + u[:, 1]], axis=1)
    return xy.astype(np.float32)


def random_subset(seed: int, n: int, k: int) -> np.ndarray:
    """k of range(n) by a partial Fisher-Yates shuffle, returned ascending."""
    idx = np.arange(n, dtype=np.int64)
    u = uniform(seed, k)
    for i in range(k):
        j = i + int(u[i] * (n - i))
        idx[i], idx[j] = idx[j], idx[i]
    return np.sort(idx[:k])


def stage_sizes(n0: int, stages: int, ds: float = 0.4) -> list[int]:
    """Token counts per stage, each round(n * ds) of the previous one."""
    out = [n0]
    for _ in range(stages - 1):
        out.append(int(math.floor(out[-1] * ds + 0.5)))
    return out


# --------------------------------------------------------------------------
# workloads
# --------------------------------------------------------------------------

@dataclass
class AttnBatch:
    """One cluster-attention problem: B images of N tokens, H heads of 32."""
    coords: np.ndarray            # [B, N, 2] fp32
    q: np.ndarray                 # [B, N, H, 32] bf16 values in fp32
    k: np.ndarray
    v: np.ndarray
    do: np.ndarray
    bias: np.ndarray              # [H, 3] fp32: a_h, b_h, c_h
    C: int = 8
    M: int = 48
    scale: float = 1.0 / math.sqrt(32.0)

    @property
    def B(self): return self.coords.shape[0]

    @property
    def N(self): return self.coords.shape[1]

    @property
    def H(self): return self.q.shape[2]


@dataclass
class KnnBatch:
    """One KNN gather problem: B images, Q queries, N source tokens, d channels."""
    queries: np.ndarray           # [B, Q, 2] fp32
    coords: np.ndarray            # [B, N, 2] fp32
    feats: np.ndarray             # [B, N, d] bf16 values in fp32
    dout: np.ndarray              # [B, Q, d] bf16 values in fp32
    p: np.ndarray                 # [d / 32] fp32
    GH: int = 64
    GW: int = 64
    K: int = 8

    @property
    def B(self): return self.coords.shape[0]

    @property
    def N(self): return self.coords.shape[1]

    @property
    def Q(self): return self.queries.shape[1]

    @property
    def d(self): return self.feats.shape[2]


def _bias(wid: int, H: int) -> np.ndarray:
    u = uniform(stream_seed(wid, 0, TAG_BIAS), 3 * H).reshape(H, 3)
    a = -0.1 + 0.2 * u[:, 0]
    b = -0.1 + 0.2 * u[:, 1]
    c = 0.1 * u[:, 2]
    return np.stack([a, b, c], axis=1).astype(np.float32)


def _qkvdo(wid: int, images, N: int, H: int, sub: int = 0):
    outs = []
    for tag in (TAG_Q, TAG_K, TAG_V, TAG_DO):
        outs.append(np.stack([normal_bf16(stream_seed(wid, i, tag, sub), (N, H, 32))
                              for i in images]))
    return outs


def stage1_coords(wid: int, image: int, gh: int = 64, gw: int = 64,
                  keep: int = 2048) -> np.ndarray:
    cells = noise_mask(stream_seed(wid, image, TAG_MASK), gh, gw, keep)
    return jittered_coords(stream_seed(wid, image, TAG_JITTER), cells, gw)


def attn_tiny(image0: int = 0, seed_image: int | None = None) -> AttnBatch:
    """16x16 grid, Bernoulli(0.5) mask (about 128 tokens), dim 128, 4 heads."""
    wid = WORKLOAD_ID["tiny"]
    i = image0 if seed_image is None else seed_image
    cells = bernoulli_mask(stream_seed(wid, i, TAG_MASK), 16, 16)
    xy = jittered_coords(stream_seed(wid, i, TAG_JITTER), cells, 16)
    q, k, v, do = _qkvdo(wid, [i], xy.shape[0], 4)
    return AttnBatch(xy[None], q, k, v, do, _bias(wid, 4))


def attn_stage1(B: int = 8, image0: int = 0, N: int = 2048, H: int = 4) -> AttnBatch:
    """64x64 grid, value-noise mask keeping N cells, B images, H heads."""
    wid = WORKLOAD_ID["stage1"]
    imgs = range(image0, image0 + B)
    xy = np.stack([stage1_coords(wid, i, keep=N) for i in imgs])
    q, k, v, do = _qkvdo(wid, imgs, N, H)
    return AttnBatch(xy, q, k, v, do, _bias(wid, H))


def attn_stage3(B: int = 64, image0: int = 0, N: int = 328, H: int = 16) -> AttnBatch:
    """N tokens per image drawn from that image's stage-1 coordinates."""
    wid = WORKLOAD_ID["stage3"]
    imgs = range(image0, image0 + B)
    xys = []
    for i in imgs:
        full = stage1_coords(wid, i)
        sel = random_subset(stream_seed(wid, i, TAG_SUBSET), full.shape[0], N)
        xys.append(full[sel])
    xy = np.stack(xys)
    q, k, v, do = _qkvdo(wid, imgs, N, H)
    return AttnBatch(xy, q, k, v, do, _bias(wid, H))


SWEEP_DIMS = (128, 256, 512, 768)
SWEEP_LAYERS = (3, 4, 16, 2)


def sweep_coords(B: int = 16, image0: int = 0, n0: int = 2048, stages: int = 4,
                 wid: int | None = None) -> list[np.ndarray]:
    """Per-stage coordinates [B, N_s, 2]: nested random subsets of round(0.4 n)."""
    wid = WORKLOAD_ID["sweep"] if wid is None else wid
    sizes = stage_sizes(n0, stages)
    per_stage = [[] for _ in range(stages)]
    for i in range(image0, image0 + B):
        xy = stage1_coords(wid, i, keep=n0)
        per_stage[0].append(xy)
        for s in range(1, stages):
            sel = random_subset(stream_seed(wid, i, TAG_SUBSET, s), xy.shape[0], sizes[s])
            xy = xy[sel]
            per_stage[s].append(xy)
    return [np.stack(p) for p in per_stage]


def attn_sweep_layer(coords: np.ndarray, stage: int, layer: int, image0: int = 0) -> AttnBatch:
    """Q/K/V/dO of one encoder layer of the sweep (distinct per layer)."""
    wid = WORKLOAD_ID["sweep"]
    B, N = coords.shape[:2]
    H = SWEEP_DIMS[stage] // 32
    q, k, v, do = _qkvdo(wid, range(image0, image0 + B), N, H, sub=1 + 64 * stage + layer)
    return AttnBatch(coords, q, k, v, do, _bias(wid, H))


def knn_queries(wid: int, image: int, gh: int = 64, gw: int = 64) -> np.ndarray:
    """One query per cell: cell centre + U(-1, 1)^2, raster order, fp32 [gh*gw, 2]."""
    n = gh * gw
    u = uniform(stream_seed(wid, image, TAG_QUERY), 2 * n, -1.0, 1.0).reshape(n, 2)
    cells = np.arange(n)
    xy = np.stack([(cells % gw) + 0.5 + u[:, 0], (cells // gw) + 0.5 + u[:, 1]], axis=1)
    return xy.astype(np.float32)


def knn_batch(coords: np.ndarray, d: int, image0: int = 0, stage: int = 0,
              wid: int | None = None, K: int = 8, gh: int = 64, gw: int = 64) -> KnnBatch:
    """Decoder gather over one stage's tokens ``coords`` [B, N, 2] with d channels."""
    wid = WORKLOAD_ID["decoder"] if wid is None else wid
    B, N = coords.shape[:2]
    imgs = range(image0, image0 + B)
    queries = np.stack([knn_queries(wid, i, gh, gw) for i in imgs])
    Q = queries.shape[1]
    feats = np.stack([normal_bf16(stream_seed(wid, i, TAG_FEAT, stage), (N, d)) for i in imgs])
    dout = np.stack([normal_bf16(stream_seed(wid, i, TAG_DOUT, stage), (Q, d)) for i in imgs])
    p = uniform(stream_seed(wid, 0, TAG_P, stage), d // 32, 0.5, 4.0).astype(np.float32)
    return KnnBatch(queries, coords, feats, dout, p, gh, gw, K)


def knn_decoder(B: int = 16, image0: int = 0) -> list[KnnBatch]:
    """The decoder workload: one KnnBatch per sweep stage."""
    stages = sweep_coords(B, image0, wid=WORKLOAD_ID["decoder"])
    return [knn_batch(xy, SWEEP_DIMS[s], image0, s) for s, xy in enumerate(stages)]


@dataclass
class StepBatch:
    """Everything one pass of the hot path consumes (the benchmark step)."""
    attn: AttnBatch
    knn: KnnBatch
    meta: dict = field(default_factory=dict)


def step_batch(B: int = 8, image0: int = 0) -> StepBatch:
    """Stage-1 batch (B x 2048 tokens, dim 128, 4 heads) + its decoder gather."""
    a = attn_stage1(B, image0)
    kb = knn_batch(a.coords, 128, image0, 0, wid=WORKLOAD_ID["step"])
    return StepBatch(a, kb, {"workload": "stage1-1024px+decoder-gather", "B": B})


def hires_batch(B: int = 2, image0: int = 0, grid: int = 128, keep: int | None = None,
                d: int = 128) -> KnnBatch:
    """Decoder gather at high resolution: a grid x grid patch grid (128 x 128 = a 2048 px image
    at 16 px patches), the value-noise mask keeping half the cells, one query per cell."""
    wid = WORKLOAD_ID["hires"]
    keep = grid * grid // 2 if keep is None else keep
    xy = np.stack([stage1_coords(wid, i, grid, grid, keep) for i in range(image0, image0 + B)])
    return knn_batch(xy, d, image0, 0, wid=wid, gh=grid, gw=grid)


@dataclass
class MergeBatch:
    """Token merging between stages: B images of N tokens (d channels) -> k anchors, with a
    seeded random scoring MLP (W1 [d][h], b1 [h], w2 [h], b2) and upstream gradients."""
    coords: np.ndarray            # [B, N, 2] fp32
    feats: np.ndarray             # [B, N, d] bf16 values in fp32
    w1: np.ndarray                # [d, h] fp32
    b1: np.ndarray                # [h] fp32
    w2: np.ndarray                # [h] fp32
    b2: float
    k: int
    dmerged: np.ndarray           # [B, k, d] bf16 values in fp32
    dmcoords: np.ndarray          # [B, k, 2] fp32

    @property
    def B(self): return self.coords.shape[0]

    @property
    def N(self): return self.coords.shape[1]

    @property
    def d(self): return self.feats.shape[2]

    @property
    def h(self): return self.w1.shape[1]


def merge_batch(coords: np.ndarray, d: int = 128, ds: float = 0.4, image0: int = 0,
                hidden: int | None = None) -> MergeBatch:
    """Merge of one stage's tokens: k = round(ds N) anchors, hidden width d/4 by default;
    W1 ~ N(0, 1/d), w2 ~ N(0, 1/h), biases ~ 0.1 N(0, 1); features and gradients N(0, 1)."""
    wid = WORKLOAD_ID["merge"]
    B, N = coords.shape[:2]
    h = d // 4 if hidden is None else hidden
    k = int(math.floor(N * ds + 0.5))
    imgs = range(image0, image0 + B)
    feats = np.stack([normal_bf16(stream_seed(wid, i, TAG_FEAT), (N, d)) for i in imgs])
    w1 = (normal(stream_seed(wid, 0, TAG_Q, 1), d * h) / math.sqrt(d)).reshape(d, h).astype(np.float32)
    b1 = (0.1 * normal(stream_seed(wid, 0, TAG_K, 1), h)).astype(np.float32)
    w2 = (normal(stream_seed(wid, 0, TAG_V, 1), h) / math.sqrt(h)).astype(np.float32)
    b2 = float(np.float32(0.1 * normal(stream_seed(wid, 0, TAG_DO, 1), 1)[0]))
    dm = np.stack([normal_bf16(stream_seed(wid, i, TAG_DOUT), (k, d)) for i in imgs])
    dxy = np.stack([normal(stream_seed(wid, i, TAG_QUERY, 1), 2 * k).reshape(k, 2)
                    for i in imgs]).astype(np.float32)
    return MergeBatch(coords.astype(np.float32), feats, w1, b1, w2, b2, k, dm, dxy)


@dataclass
class DecoderBatch:
    """The decoder over four encoder stages: B images, Q mask-token queries per image (the
    masked cells of the 64 x 64 grid; reference positions at their centres) with D-channel
    features, and per layer an offset head (W_off [D, 2], b_off [2]) and a projection
    (W_o [d_s, D], bf16 values).  Layer l reads stage layer_stage[l]: coarse to fine."""
    ref: np.ndarray               # [B, Q, 2] fp32
    f0: np.ndarray                # [B, Q, D] fp32
    stages: list                  # KnnBatch per stage (0 = finest): coords, feats, p
    w_off: list                   # per layer [D, 2] fp32
    b_off: list                   # per layer [2] fp32
    w_o: list                     # per layer [d_s, D] bf16 values in fp32
    df: np.ndarray                # [B, Q, D] fp32, gradient of the last layer's output
    layer_stage: tuple = (3, 2, 1, 0)

    @property
    def B(self): return self.ref.shape[0]

    @property
    def Q(self): return self.ref.shape[1]

    @property
    def D(self): return self.f0.shape[2]


def decoder_batch(B: int = 8, image0: int = 0, D: int = 256, n0: int = 2048,
                  offset_scale: float = 1.0) -> DecoderBatch:
    """Stages as in the sweep (nested subsets, dims 128/256/512/768) of a value-noise mask
    keeping n0 of 4096 cells; the other cells are the queries.  f0, df ~ N(0, 1);
    W_off ~ offset_scale N(0, 1/D) (offsets of about offset_scale cells), b_off ~ 0.1 N(0, 1);
    W_o ~ N(0, 1/d_s) rounded to bf16."""
    wid = WORKLOAD_ID["dec_layer"]
    imgs = range(image0, image0 + B)
    coords = sweep_coords(B, image0, n0=n0, wid=wid)
    refs = []
    for i in imgs:
        vis = noise_mask(stream_seed(wid, i, TAG_MASK), 64, 64, n0)
        masked = np.setdiff1d(np.arange(64 * 64), vis)
        refs.append(np.stack([(masked % 64) + 0.5, (masked // 64) + 0.5], axis=1))
    ref = np.stack(refs).astype(np.float32)
    Q = ref.shape[1]
    stages = [knn_batch(xy, SWEEP_DIMS[s], image0, s, wid=wid) for s, xy in enumerate(coords)]
    f0 = np.stack([normal(stream_seed(wid, i, TAG_F0), Q * D).reshape(Q, D)
                   for i in imgs]).astype(np.float32)
    df = np.stack([normal(stream_seed(wid, i, TAG_DF), Q * D).reshape(Q, D)
                   for i in imgs]).astype(np.float32)
    w_off, b_off, w_o = [], [], []
    for layer, st in enumerate((3, 2, 1, 0)):
        w_off.append((offset_scale * normal(stream_seed(wid, 0, TAG_WOFF, layer), 2 * D)
                      / math.sqrt(D)).reshape(D, 2).astype(np.float32))
        b_off.append((0.1 * normal(stream_seed(wid, 0, TAG_WOFF, 16 + layer), 2)).astype(np.float32))
        d = SWEEP_DIMS[st]
        w_o.append(round_bf16(normal(stream_seed(wid, 0, TAG_WO, layer), d * D)
                              / math.sqrt(d)).reshape(d, D))
    return DecoderBatch(ref, f0, stages, w_off, b_off, w_o, df)
