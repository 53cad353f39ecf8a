// knn.cu -- KNN cache lookup table and the distance-softmax gather (fwd + bwd).
//
// AFFMAE notes, "Key Designs" 2: the decoder aggregates the K nearest visible
// tokens of a sample point q with w_i = softmax_i(-p d_i), the exponential
// distance kernel (a stable softmax with a temperature).  "Key Designs" 3: the
// neighbours come from an H x W x K table of every grid cell's K nearest tokens,
// q quantised to its cell, so the search becomes a lookup plus K distances.
//
// Table (bit-exact).  The tokens of an image are counting-sorted into square bins
// of s x s cells (s a power of two giving about two tokens per bin) in shared
// memory; each thread then searches one cell centre ring by ring.  A token in a
// bin at ring distance rho + 1 or more lies at least rho*s away on one axis, and
// correctly rounded fp64 arithmetic is monotone, so once the current K-th best
// fp64 squared distance is below (rho*s)^2 no unvisited token can enter the
// (distance, id) top-K: the result equals the brute-force definition.
//
// Gather.  A group of LPQ lanes (LPQ = d/8 rounded to a power of two, at most 32)
// owns one query; each lane owns 8 consecutive channels (one 16-byte bf16 load
// per neighbour row) for each 8*LPQ-channel chunk.  Every lane recomputes the K
// distances (same addresses across the group: broadcast loads), so no shuffles
// are needed in the forward.
//
// Backward without atomics.  Query side: recompute w, dw = <dOut, f> (reduced over
// the 4 lanes of a head), ds, dq, dp partials; store w and the token ids.  An
// inverse index -- for every token, its (query, slot) entries in ascending order --
// is built per image by a stable counting sort (per-warp chunk histograms with
// __match_any_sync, no floating point).  Token side: one lane group per token sums
// w * dOut over its entries in that fixed order.
#include <float.h>
#include <math.h>

#include "internal.h"

namespace acl {

namespace {

constexpr int kTableThreads = 256;
constexpr int kGatherWarps = 8;
constexpr int kGatherThreads = 32 * kGatherWarps;
constexpr int kCsrThreads = 1024;

__device__ __forceinline__ int quantise(float v, int n) {
    if (!(v >= 0.f)) return 0;
    if (v >= static_cast<float>(n)) return n - 1;
    const int i = static_cast<int>(v);
    return i > n - 1 ? n - 1 : i;
}

// Exclusive prefix sum in place by the whole block; returns the total.
__device__ int block_scan(int* data, int n, int* scratch) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    const int per = (n + blockDim.x - 1) / blockDim.x;
    const int p0 = tid * per;
    int local = 0;
    for (int i = 0; i < per; ++i)
        if (p0 + i < n) local += data[p0 + i];
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) scratch[warp] = incl;
    __syncthreads();
    if (tid == 0) {
        int run = 0;
        for (int w = 0; w < nw; ++w) {
            const int v = scratch[w];
            scratch[w] = run;
            run += v;
        }
        scratch[nw] = run;
    }
    __syncthreads();
    int run = scratch[warp] + incl - local;
    for (int i = 0; i < per; ++i) {
        if (p0 + i < n) {
            const int v = data[p0 + i];
            data[p0 + i] = run;
            run += v;
        }
    }
    const int total = scratch[nw];
    __syncthreads();
    return total;
}

// ------------------------------------------------------------------- table

struct BinGrid {
    float inv_s;   // 1 / s (exact: s is a power of two)
    int s, nbx, nby;
};

__device__ __forceinline__ int bin_coord(float v, float inv_s, int nb) {
    const float f = v * inv_s;
    if (!(f >= 0.f)) return 0;
    if (f >= static_cast<float>(nb)) return nb - 1;
    const int i = static_cast<int>(f);
    return i > nb - 1 ? nb - 1 : i;
}

template <int KMAX>
__device__ __forceinline__ void topk_insert(double (&bd)[KMAX], int (&bi)[KMAX], double d, int t) {
    if (d < bd[KMAX - 1] || (d == bd[KMAX - 1] && t < bi[KMAX - 1])) {
        bool placed = false;
#pragma unroll
        for (int r = KMAX - 1; r >= 0; --r) {
            if (!placed) {
                if (r > 0 && (bd[r - 1] > d || (bd[r - 1] == d && bi[r - 1] > t))) {
                    bd[r] = bd[r - 1];
                    bi[r] = bi[r - 1];
                } else {
                    bd[r] = d;
                    bi[r] = t;
                    placed = true;
                }
            }
        }
    }
}

// One warp per 8 x 4 tile of cells, one lane per cell.  Bin rows are contiguous runs of
// the bin-sorted tokens, and all lanes of the warp read the same candidate (a
// shared-memory broadcast).  A candidate whose fp32 squared distance exceeds the current K-th best by
// more than the fp32 rounding bound cannot enter the fp64 (distance, id) top-K and is
// skipped; the rest go through the exact fp64 comparison.  Bins are visited in rings
// around the tile's own bins, nearest first, so the lists fill with near tokens and the
// threshold tightens early.  After each ring every lane checks that its K-th distance is
// below its distance to the scanned rectangle's edge (tokens outside lie beyond it, and
// rounding is monotone); the warp stops once all lanes are proven.
template <int KMAX>
__global__ void __launch_bounds__(kTableThreads)
    knn_table_kernel(const float* __restrict__ xy, int N, int GH, int GW, int K, BinGrid bg,
                     int32_t* __restrict__ table) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int b = blockIdx.y, tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int nbins = bg.nbx * bg.nby;
    int* cnt = reinterpret_cast<int*>(smem);
    int* scratch = cnt + nbins;
    float2* txy = reinterpret_cast<float2*>(smem + ((4 * (nbins + 40) + 15) & ~15));
    uint16_t* tidv = reinterpret_cast<uint16_t*>(txy + N);
    const float2* img = reinterpret_cast<const float2*>(xy) + static_cast<size_t>(b) * N;

    for (int i = tid; i < nbins; i += kTableThreads) cnt[i] = 0;
    __syncthreads();
    for (int t = tid; t < N; t += kTableThreads) {
        const float2 p = img[t];
        atomicAdd(&cnt[bin_coord(p.y, bg.inv_s, bg.nby) * bg.nbx + bin_coord(p.x, bg.inv_s, bg.nbx)], 1);
    }
    __syncthreads();
    block_scan(cnt, nbins, scratch);
    for (int t = tid; t < N; t += kTableThreads) {
        const float2 p = img[t];
        const int bin = bin_coord(p.y, bg.inv_s, bg.nby) * bg.nbx + bin_coord(p.x, bg.inv_s, bg.nbx);
        const int pos = atomicAdd(&cnt[bin], 1);
        txy[pos] = p;
        tidv[pos] = static_cast<uint16_t>(t);
    }
    __syncthreads();  // cnt[bin] = end of bin; start = cnt[bin - 1]

    const int tiles_x = (GW + 7) >> 3, tiles_y = (GH + 3) >> 2;
    const int tile = blockIdx.x * (kTableThreads / 32) + warp;
    if (tile >= tiles_x * tiles_y) return;
    const int tx0 = (tile % tiles_x) * 8, ty0 = (tile / tiles_x) * 4;
    const int c = tx0 + (lane & 7), r = ty0 + (lane >> 3);
    const int cc = min(c, GW - 1), rr = min(r, GH - 1);  // lanes past the edge shadow a real cell
    const double px = static_cast<double>(cc) + 0.5, py = static_cast<double>(rr) + 0.5;
    const float pxf = static_cast<float>(cc) + 0.5f, pyf = static_cast<float>(rr) + 0.5f;

    double bd[KMAX];
    int bi[KMAX];
#pragma unroll
    for (int k = 0; k < KMAX; ++k) {
        bd[k] = DBL_MAX;
        bi[k] = 0x7fffffff;
    }
    float thr = INFINITY;
    // scan one contiguous run of bins [b0, b1] (one bin row): every lane reads the same token
    auto scan_run = [&](int b0, int b1) {
        const int s0 = b0 > 0 ? cnt[b0 - 1] : 0, s1 = cnt[b1];
        for (int i = s0; i < s1; ++i) {
            const float2 p = txy[i];
            const float dxf = p.x - pxf, dyf = p.y - pyf;
            const float d2f = fmaf(dxf, dxf, dyf * dyf);
            if (d2f <= thr) {
                const double dx = __dsub_rn(static_cast<double>(p.x), px);
                const double dy = __dsub_rn(static_cast<double>(p.y), py);
                topk_insert<KMAX>(bd, bi, __dadd_rn(__dmul_rn(dx, dx), __dmul_rn(dy, dy)), tidv[i]);
                if (bd[KMAX - 1] < DBL_MAX)
                    thr = static_cast<float>(bd[KMAX - 1]) * (1.0f + 1.0f / 1048576.0f);
            }
        }
    };
    // the tile's footprint in bins; rings of bins around it are scanned nearest first
    const int tbx0 = bin_coord(static_cast<float>(tx0) + 0.5f, bg.inv_s, bg.nbx);
    const int tbx1 = bin_coord(static_cast<float>(min(tx0 + 8, GW)) - 0.5f, bg.inv_s, bg.nbx);
    const int tby0 = bin_coord(static_cast<float>(ty0) + 0.5f, bg.inv_s, bg.nby);
    const int tby1 = bin_coord(static_cast<float>(min(ty0 + 4, GH)) - 0.5f, bg.inv_s, bg.nby);
    const double s = static_cast<double>(bg.s);
    const int maxring = max(bg.nbx, bg.nby);
    for (int rho = 0; rho <= maxring; ++rho) {
        const int bx_lo = tbx0 - rho, bx_hi = tbx1 + rho, by_lo = tby0 - rho, by_hi = tby1 + rho;
        const int cx_lo = max(bx_lo, 0), cx_hi = min(bx_hi, bg.nbx - 1);
        if (rho == 0) {
            for (int by = max(by_lo, 0); by <= min(by_hi, bg.nby - 1); ++by)
                scan_run(by * bg.nbx + cx_lo, by * bg.nbx + cx_hi);
        } else {
            if (by_lo >= 0) scan_run(by_lo * bg.nbx + cx_lo, by_lo * bg.nbx + cx_hi);
            if (by_hi < bg.nby) scan_run(by_hi * bg.nbx + cx_lo, by_hi * bg.nbx + cx_hi);
            for (int by = max(by_lo + 1, 0); by <= min(by_hi - 1, bg.nby - 1); ++by) {
                if (bx_lo >= 0) scan_run(by * bg.nbx + bx_lo, by * bg.nbx + bx_lo);
                if (bx_hi < bg.nbx) scan_run(by * bg.nbx + bx_hi, by * bg.nbx + bx_hi);
            }
        }
        // distance from the cell centre to the edge of the scanned rectangle; a side on the
        // grid border is unbounded (tokens outside the grid fall into border bins)
        double m = DBL_MAX;
        if (bx_lo > 0) m = fmin(m, px - bx_lo * s);
        if (bx_hi < bg.nbx - 1) m = fmin(m, (bx_hi + 1) * s - px);
        if (by_lo > 0) m = fmin(m, py - by_lo * s);
        if (by_hi < bg.nby - 1) m = fmin(m, (by_hi + 1) * s - py);
        const bool proven = (m == DBL_MAX) || (bd[KMAX - 1] < m * m);
        if (__all_sync(0xffffffffu, proven)) break;
    }
    if (c >= GW || r >= GH) return;
    int32_t* out = table + static_cast<size_t>(b) * GH * GW * K + (static_cast<size_t>(r) * GW + c) * K;
#pragma unroll
    for (int k = 0; k < KMAX; ++k)
        if (k < K) out[k] = (bi[k] == 0x7fffffff) ? -1 : bi[k];
}

BinGrid choose_bins(int N, int GH, int GW) {
    BinGrid g;
    int s = 1;
    const int gmax = GH > GW ? GH : GW;
    while (s < gmax && static_cast<double>(N) * s * s < 2.0 * GH * GW) s *= 2;
    g.s = s;
    g.inv_s = 1.0f / static_cast<float>(s);
    g.nbx = (GW + s - 1) / s;
    g.nby = (GH + s - 1) / s;
    return g;
}


// ------------------------------------------------------------------ gather

struct Nbrs {
    int t;
    float d, x, y;
};

// Lane-group prologue shared by the forward and the query side of the backward.
template <int KT>
__device__ __forceinline__ float load_neighbours(const KnnArgs& a, long long gq, float2 qp,
                                                 Nbrs (&nb)[KT]) {
    const int b = static_cast<int>(gq / a.Q);
    const int cy = quantise(qp.y, a.GH), cx = quantise(qp.x, a.GW);
    const int32_t* row = a.table + ((static_cast<size_t>(b) * a.GH + cy) * a.GW + cx) * a.K;
    const float2* xyb = reinterpret_cast<const float2*>(a.xy) + static_cast<size_t>(b) * a.N;
    float dmin = INFINITY;
#pragma unroll
    for (int j = 0; j < KT; ++j) {
        int t = (j < a.K) ? row[j] : -1;
        if (t >= a.N) t = -1;
        nb[j].t = t;
        if (t >= 0) {
            const float2 p = xyb[t];
            const float dx = qp.x - p.x, dy = qp.y - p.y;
            nb[j].x = p.x;
            nb[j].y = p.y;
            nb[j].d = sqrtf(dx * dx + dy * dy);
            dmin = fminf(dmin, nb[j].d);
        } else {
            nb[j].x = nb[j].y = 0.f;
            nb[j].d = INFINITY;
        }
    }
    return dmin;
}

__device__ __forceinline__ void fma8(float (&acc)[8], float w, uint4 f) {
    const uint32_t u[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        acc[2 * i] += w * bf16_lo(u[i]);
        acc[2 * i + 1] += w * bf16_hi(u[i]);
    }
}

__device__ __forceinline__ uint4 pack8(const float (&v)[8], float s) {
    uint4 o;
    o.x = pack_bf16(v[0] * s, v[1] * s);
    o.y = pack_bf16(v[2] * s, v[3] * s);
    o.z = pack_bf16(v[4] * s, v[5] * s);
    o.w = pack_bf16(v[6] * s, v[7] * s);
    return o;
}

template <int KT, int CH>
__global__ void __launch_bounds__(kGatherThreads) knn_fwd_kernel(const KnnArgs a, int lpq_log2) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int LPQ = 1 << lpq_log2;
    const int sub = lane & (LPQ - 1), grp = lane >> lpq_log2;
    const long long total = static_cast<long long>(a.B) * a.Q;
    const long long gq = (static_cast<long long>(blockIdx.x) * kGatherWarps + warp) * (32 >> lpq_log2) + grp;
    if (gq >= total) return;  // no cross-lane communication below
    const float2 qp = reinterpret_cast<const float2*>(a.queries)[gq];
    Nbrs nb[KT];
    const float dmin = load_neighbours<KT>(a, gq, qp, nb);
    const int b = static_cast<int>(gq / a.Q);
    const bf16* fb = a.feats + static_cast<size_t>(b) * a.N * a.d;
#pragma unroll
    for (int ch = 0; ch < CH; ++ch) {
        const int c0 = ch * LPQ * 8 + sub * 8;
        if (c0 >= a.d) break;
        const float ph = a.p[c0 >> 5] * kLog2e;
        uint4 f[KT];
#pragma unroll
        for (int j = 0; j < KT; ++j)
            f[j] = (nb[j].t >= 0) ? ldg16(fb + static_cast<size_t>(nb[j].t) * a.d + c0)
                                  : make_uint4(0u, 0u, 0u, 0u);
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        float sum = 0.f;
#pragma unroll
        for (int j = 0; j < KT; ++j) {
            const float w = (nb[j].t >= 0) ? exp2f(-ph * (nb[j].d - dmin)) : 0.f;
            sum += w;
            fma8(acc, w, f[j]);
        }
        const float inv = sum > 0.f ? 1.f / sum : 0.f;
        *reinterpret_cast<uint4*>(a.out + static_cast<size_t>(gq) * a.d + c0) = pack8(acc, inv);
    }
}

template <int KT, int CH>
__global__ void __launch_bounds__(kGatherThreads) knn_bwd_query_kernel(const KnnArgs a, int lpq_log2) {
    extern __shared__ __align__(16) float sdp[];  // [warps][groups][heads]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int LPQ = 1 << lpq_log2, QPW = 32 >> lpq_log2;
    const int sub = lane & (LPQ - 1), grp = lane >> lpq_log2;
    const int NH = a.d >> 5;
    const int nslots = kGatherWarps * QPW * NH;
    for (int i = threadIdx.x; i < nslots; i += kGatherThreads) sdp[i] = 0.f;
    __syncthreads();
    const long long total = static_cast<long long>(a.B) * a.Q;
    const long long gq = (static_cast<long long>(blockIdx.x) * kGatherWarps + warp) * QPW + grp;
    const bool live = gq < total;
    float2 qp = make_float2(0.f, 0.f);
    Nbrs nb[KT];
    float dmin = 0.f;
    int b = 0;
    if (live) {
        qp = reinterpret_cast<const float2*>(a.queries)[gq];
        dmin = load_neighbours<KT>(a, gq, qp, nb);
        b = static_cast<int>(gq / a.Q);
        if (sub == 0) {
#pragma unroll
            for (int j = 0; j < KT; ++j)
                if (j < a.K) a.keys[static_cast<size_t>(gq) * a.K + j] = nb[j].t;
        }
    } else {
#pragma unroll
        for (int j = 0; j < KT; ++j) {
            nb[j].t = -1;
            nb[j].d = INFINITY;
            nb[j].x = nb[j].y = 0.f;
        }
    }
    const bf16* fb = a.feats + static_cast<size_t>(b) * a.N * a.d;
    float dqx = 0.f, dqy = 0.f;
#pragma unroll
    for (int ch = 0; ch < CH; ++ch) {
        const int c0 = ch * LPQ * 8 + sub * 8;
        const bool on = live && c0 < a.d;
        const int hh = on ? (c0 >> 5) : 0;
        const float ph = on ? a.p[hh] : 0.f;
        float w[KT], dw[KT];
        float g[8];
        {
            const uint4 gv = on ? ldg16(a.dout + static_cast<size_t>(gq) * a.d + c0)
                                : make_uint4(0u, 0u, 0u, 0u);
            const uint32_t u[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                g[2 * i] = bf16_lo(u[i]);
                g[2 * i + 1] = bf16_hi(u[i]);
            }
        }
        float sum = 0.f;
#pragma unroll
        for (int j = 0; j < KT; ++j) {
            const bool v = on && nb[j].t >= 0;
            w[j] = v ? exp2f(-ph * kLog2e * (nb[j].d - dmin)) : 0.f;
            sum += w[j];
            const uint4 f = v ? ldg16(fb + static_cast<size_t>(nb[j].t) * a.d + c0)
                              : make_uint4(0u, 0u, 0u, 0u);
            const uint32_t u[4] = {f.x, f.y, f.z, f.w};
            float acc = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) acc += g[2 * i] * bf16_lo(u[i]) + g[2 * i + 1] * bf16_hi(u[i]);
            dw[j] = acc;
        }
        const float inv = sum > 0.f ? 1.f / sum : 0.f;
        float sdw = 0.f;
#pragma unroll
        for (int j = 0; j < KT; ++j) {
            dw[j] += __shfl_xor_sync(0xffffffffu, dw[j], 1);
            dw[j] += __shfl_xor_sync(0xffffffffu, dw[j], 2);
            w[j] *= inv;
            sdw += w[j] * dw[j];
        }
        if (on && (sub & 3) == 0) {
            float dph = 0.f;
            float* wout = a.w + static_cast<size_t>(gq) * a.K * NH + hh;
#pragma unroll
            for (int j = 0; j < KT; ++j) {
                if (j < a.K) wout[j * NH] = w[j];
                if (nb[j].t < 0) continue;
                const float ds = w[j] * (dw[j] - sdw);
                dph -= ds * nb[j].d;
                if (nb[j].d > 0.f) {
                    const float cf = -ds * ph / nb[j].d;
                    dqx += cf * (qp.x - nb[j].x);
                    dqy += cf * (qp.y - nb[j].y);
                }
            }
            sdp[(warp * QPW + grp) * NH + hh] = dph;
        }
    }
    // dq: sum over the group's head leaders
    for (int o = 1; o < LPQ; o <<= 1) {
        dqx += __shfl_xor_sync(0xffffffffu, dqx, o);
        dqy += __shfl_xor_sync(0xffffffffu, dqy, o);
    }
    if (live && sub == 0) reinterpret_cast<float2*>(a.dq)[gq] = make_float2(dqx, dqy);
    __syncthreads();
    for (int h = threadIdx.x; h < NH; h += kGatherThreads) {
        float acc = 0.f;
        for (int s = 0; s < kGatherWarps * QPW; ++s) acc += sdp[s * NH + h];
        a.dp_part[static_cast<size_t>(blockIdx.x) * NH + h] = acc;
    }
}

// Shared-neighbour variants (K <= lanes per query): lane j < K of a query's lane group
// looks up neighbour j, computes its distance once and the group exchanges ids and
// distances with width-limited shuffles, instead of every lane recomputing all K.  A CTA
// walks `iters` consecutive blocks of queries, so neighbouring queries (which share most
// of their tokens) run on one SM and find each other's feature rows in L1.
struct GroupNbrs {
    int t;
    float d, ux, uy;  // id, distance, unit vector (q - p) / d (0 when d == 0)
};

template <int KT>
__device__ __forceinline__ float group_neighbours(const KnnArgs& a, long long gq, bool live, float2 qp,
                                                  int sub, int LPQ, GroupNbrs (&nb)[KT]) {
    int t = -1;
    float d = INFINITY, ux = 0.f, uy = 0.f;
    if (live && sub < a.K) {
        const int b = static_cast<int>(gq / a.Q);
        const int cy = quantise(qp.y, a.GH), cx = quantise(qp.x, a.GW);
        t = a.table[((static_cast<size_t>(b) * a.GH + cy) * a.GW + cx) * a.K + sub];
        if (t >= a.N) t = -1;
        if (t >= 0) {
            const float2 p = reinterpret_cast<const float2*>(a.xy)[static_cast<size_t>(b) * a.N + t];
            const float dx = qp.x - p.x, dy = qp.y - p.y;
            d = sqrtf(dx * dx + dy * dy);
            if (d > 0.f) {
                ux = dx / d;
                uy = dy / d;
            }
        }
    }
    float dmin = d;
    for (int o = 1; o < LPQ; o <<= 1) dmin = fminf(dmin, __shfl_xor_sync(0xffffffffu, dmin, o, LPQ));
#pragma unroll
    for (int j = 0; j < KT; ++j) {
        nb[j].t = __shfl_sync(0xffffffffu, t, j, LPQ);
        nb[j].d = __shfl_sync(0xffffffffu, d, j, LPQ);
        nb[j].ux = __shfl_sync(0xffffffffu, ux, j, LPQ);
        nb[j].uy = __shfl_sync(0xffffffffu, uy, j, LPQ);
    }
    return dmin;
}

template <int KT, int CH>
__global__ void __launch_bounds__(kGatherThreads)
    knn_fwd_shared_kernel(const KnnArgs a, int lpq_log2, int iters) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int LPQ = 1 << lpq_log2, QPW = 32 >> lpq_log2;
    const int sub = lane & (LPQ - 1), grp = lane >> lpq_log2;
    const long long total = static_cast<long long>(a.B) * a.Q;
    for (int it = 0; it < iters; ++it) {
        const long long gq = ((static_cast<long long>(blockIdx.x) * iters + it) * kGatherWarps + warp) * QPW + grp;
        if ((gq - grp) >= total) break;  // whole warp past the end (uniform)
        const bool live = gq < total;
        const float2 qp = live ? reinterpret_cast<const float2*>(a.queries)[gq] : make_float2(0.f, 0.f);
        GroupNbrs nb[KT];
        const float dmin = group_neighbours<KT>(a, gq, live, qp, sub, LPQ, nb);
        if (!live) continue;
        const int b = static_cast<int>(gq / a.Q);
        const bf16* fb = a.feats + static_cast<size_t>(b) * a.N * a.d;
#pragma unroll
        for (int ch = 0; ch < CH; ++ch) {
            const int c0 = ch * LPQ * 8 + sub * 8;
            if (c0 >= a.d) break;
            const float ph = a.p[c0 >> 5] * kLog2e;
            uint4 f[KT];
#pragma unroll
            for (int j = 0; j < KT; ++j)
                f[j] = (nb[j].t >= 0) ? ldg16(fb + static_cast<size_t>(nb[j].t) * a.d + c0)
                                      : make_uint4(0u, 0u, 0u, 0u);
            float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            float sum = 0.f;
#pragma unroll
            for (int j = 0; j < KT; ++j) {
                const float w = (nb[j].t >= 0) ? exp2f(-ph * (nb[j].d - dmin)) : 0.f;
                sum += w;
                fma8(acc, w, f[j]);
            }
            const float inv = sum > 0.f ? 1.f / sum : 0.f;
            *reinterpret_cast<uint4*>(a.out + static_cast<size_t>(gq) * a.d + c0) = pack8(acc, inv);
        }
    }
}

template <int KT, int CH>
__global__ void __launch_bounds__(kGatherThreads)
    knn_bwd_query_shared_kernel(const KnnArgs a, int lpq_log2, int iters) {
    extern __shared__ __align__(16) float sdp[];  // [warps][groups][heads]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int LPQ = 1 << lpq_log2, QPW = 32 >> lpq_log2;
    const int sub = lane & (LPQ - 1), grp = lane >> lpq_log2;
    const int NH = a.d >> 5;
    const int nslots = kGatherWarps * QPW * NH;
    for (int i = threadIdx.x; i < nslots; i += kGatherThreads) sdp[i] = 0.f;
    __syncthreads();
    const long long total = static_cast<long long>(a.B) * a.Q;
    for (int it = 0; it < iters; ++it) {
        const long long gq = ((static_cast<long long>(blockIdx.x) * iters + it) * kGatherWarps + warp) * QPW + grp;
        if ((gq - grp) >= total) break;  // uniform per warp
        const bool live = gq < total;
        const float2 qp = live ? reinterpret_cast<const float2*>(a.queries)[gq] : make_float2(0.f, 0.f);
        GroupNbrs nb[KT];
        const float dmin = group_neighbours<KT>(a, gq, live, qp, sub, LPQ, nb);
        if (live && sub == 0) {
#pragma unroll
            for (int j = 0; j < KT; ++j)
                if (j < a.K) a.keys[static_cast<size_t>(gq) * a.K + j] = nb[j].t;
        }
        const int b = live ? static_cast<int>(gq / a.Q) : 0;
        const bf16* fb = a.feats + static_cast<size_t>(b) * a.N * a.d;
        float dqx = 0.f, dqy = 0.f;
#pragma unroll
        for (int ch = 0; ch < CH; ++ch) {
            const int c0 = ch * LPQ * 8 + sub * 8;
            const bool on = live && c0 < a.d;
            const int hh = on ? (c0 >> 5) : 0;
            const float ph = on ? a.p[hh] : 0.f;
            float g[8];
            {
                const uint4 gv = on ? ldg16(a.dout + static_cast<size_t>(gq) * a.d + c0)
                                    : make_uint4(0u, 0u, 0u, 0u);
                const uint32_t u[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    g[2 * i] = bf16_lo(u[i]);
                    g[2 * i + 1] = bf16_hi(u[i]);
                }
            }
            uint4 f[KT];
#pragma unroll
            for (int j = 0; j < KT; ++j)
                f[j] = (on && nb[j].t >= 0) ? ldg16(fb + static_cast<size_t>(nb[j].t) * a.d + c0)
                                            : make_uint4(0u, 0u, 0u, 0u);
            float w[KT], dw[KT];
            float sum = 0.f;
#pragma unroll
            for (int j = 0; j < KT; ++j) {
                w[j] = (on && nb[j].t >= 0) ? exp2f(-ph * kLog2e * (nb[j].d - dmin)) : 0.f;
                sum += w[j];
                const uint32_t u[4] = {f[j].x, f[j].y, f[j].z, f[j].w};
                float acc = 0.f;
#pragma unroll
                for (int i = 0; i < 4; ++i) acc += g[2 * i] * bf16_lo(u[i]) + g[2 * i + 1] * bf16_hi(u[i]);
                dw[j] = acc;
            }
            const float inv = sum > 0.f ? 1.f / sum : 0.f;
            float sdw = 0.f;
#pragma unroll
            for (int j = 0; j < KT; ++j) {
                dw[j] += __shfl_xor_sync(0xffffffffu, dw[j], 1);
                dw[j] += __shfl_xor_sync(0xffffffffu, dw[j], 2);
                w[j] *= inv;
                sdw += w[j] * dw[j];
            }
            if (on && (sub & 3) == 0) {
                float dph = 0.f;
                float* wout = a.w + static_cast<size_t>(gq) * a.K * NH + hh;
#pragma unroll
                for (int j = 0; j < KT; ++j) {
                    if (j < a.K) wout[j * NH] = w[j];
                    if (nb[j].t < 0) continue;
                    const float ds = w[j] * (dw[j] - sdw);
                    dph -= ds * nb[j].d;
                    const float cf = -ds * ph;
                    dqx += cf * nb[j].ux;
                    dqy += cf * nb[j].uy;
                }
                sdp[(warp * QPW + grp) * NH + hh] += dph;
            }
        }
        for (int o = 1; o < LPQ; o <<= 1) {
            dqx += __shfl_xor_sync(0xffffffffu, dqx, o);
            dqy += __shfl_xor_sync(0xffffffffu, dqy, o);
        }
        if (live && sub == 0) reinterpret_cast<float2*>(a.dq)[gq] = make_float2(dqx, dqy);
    }
    __syncthreads();
    for (int h = threadIdx.x; h < NH; h += kGatherThreads) {
        float acc = 0.f;
        for (int sl = 0; sl < kGatherWarps * QPW; ++sl) acc += sdp[sl * NH + h];
        a.dp_part[static_cast<size_t>(blockIdx.x) * NH + h] = acc;
    }
}

// Stable counting sort of an image's (query, slot) entries by token id, integer only,
// spread over `slices` CTAs per image: CTA (slice, b) owns the tokens [t_lo, t_hi).  Warp w
// owns the contiguous entry chunk [lo_w, hi_w) of the image:
//   compaction: one pass over its keys (16 per lane in flight) appends the entries of the
//     slice, in entry order, to the warp's shared-memory list (ballot + popc) and counts
//     the entries whose token lies below t_lo;
//   counts and prefix: per-(warp, token) counts of the lists; each warp's first slot per
//     token is (entries of smaller tokens) + (entries of this token in earlier warps);
//   placement: each listed entry goes to its warp's next slot for its token plus its rank
//     among equal tokens in its group of 32 (lanes OR their bit into a per-warp hashed
//     mask -- OR commutes, so the mask does not depend on timing).
// The list of a token ends up in ascending entry order; entries are stored packed as
// (query << 4) | slot.  CTA (0, 0) also resets the token kernel's work counter.
constexpr int kCsrSteps = 16;
constexpr int kCsrHash = 256;
constexpr int kCsrWarps = kCsrThreads / 32;
constexpr int kCsrCap = 384;  // listed entries per warp held in shared memory

struct CsrSmem {
    size_t pre, off, hash, lanes, ckey, cent, scratch, total;
};
__host__ __device__ __forceinline__ CsrSmem csr_smem_layout(int NS) {
    const size_t n2 = static_cast<size_t>((NS + 1) & ~1);
    CsrSmem L;
    L.pre = 0;
    L.off = (2 * kCsrWarps * n2 + 15) & ~size_t(15);
    L.hash = L.off + ((4 * static_cast<size_t>(NS + 1) + 15) & ~size_t(15));
    L.lanes = L.hash + 4 * static_cast<size_t>(kCsrHash) * kCsrWarps;
    L.ckey = L.lanes + 4 * 32 * static_cast<size_t>(kCsrWarps);
    L.cent = L.ckey + 2 * static_cast<size_t>(kCsrCap) * kCsrWarps;
    L.scratch = L.cent + 4 * static_cast<size_t>(kCsrCap) * kCsrWarps;
    L.total = L.scratch + 40 * 4;
    return L;
}

__global__ void __launch_bounds__(kCsrThreads) knn_csr_kernel(const KnnArgs a, int slices) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int b = blockIdx.y, sl = blockIdx.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int N = a.N, K = a.K;
    if (b == 0 && sl == 0 && tid == 0) *a.counter = 0;
    const int t_lo = static_cast<int>(static_cast<long long>(sl) * N / slices);
    const int t_hi = static_cast<int>(static_cast<long long>(sl + 1) * N / slices);
    const int NS = t_hi - t_lo;
    const int NS2 = (NS + 1) & ~1;
    const CsrSmem L = csr_smem_layout((N + slices - 1) / slices);
    uint16_t* pre = reinterpret_cast<uint16_t*>(smem + L.pre);  // [warps][NS2]
    int* off = reinterpret_cast<int*>(smem + L.off);
    uint32_t* hb = reinterpret_cast<uint32_t*>(smem + L.hash) + warp * kCsrHash;
    int* ks = reinterpret_cast<int*>(smem + L.lanes) + warp * 32;
    uint16_t* ckey = reinterpret_cast<uint16_t*>(smem + L.ckey) + warp * kCsrCap;  // key - t_lo
    int* cent = reinterpret_cast<int*>(smem + L.cent) + warp * kCsrCap;              // entry
    int* scratch = reinterpret_cast<int*>(smem + L.scratch);
    const int E = a.Q * K;
    const int32_t* keys = a.keys + static_cast<size_t>(b) * E;
    int32_t* csr = a.csr + static_cast<size_t>(b) * E;
    for (int i = tid; i < kCsrWarps * NS2; i += kCsrThreads) pre[i] = 0;
    for (int i = lane; i < kCsrHash; i += 32) hb[i] = 0u;
    const int lo = static_cast<int>(static_cast<long long>(warp) * E / kCsrWarps);
    const int hi = static_cast<int>(static_cast<long long>(warp + 1) * E / kCsrWarps);
    uint16_t* mine = pre + warp * NS2;
    const unsigned below_lanes = (1u << lane) - 1u;
    // compaction + count below the slice
    int ncomp = 0, below = 0;
    for (int base = lo; base < hi; base += 32 * kCsrSteps) {
        int k[kCsrSteps];
#pragma unroll
        for (int st = 0; st < kCsrSteps; ++st) {
            const int e = base + st * 32 + lane;
            const int v = (e < hi) ? __ldg(keys + e) : -1;
            k[st] = (v >= N) ? -1 : v;
        }
#pragma unroll
        for (int st = 0; st < kCsrSteps; ++st) {
            const int key = k[st];
            below += (key >= 0 && key < t_lo);
            const bool in = key >= t_lo && key < t_hi;
            const unsigned m = __ballot_sync(0xffffffffu, in);
            if (in) {
                const int pos = ncomp + __popc(m & below_lanes);
                if (pos < kCsrCap) {
                    ckey[pos] = static_cast<uint16_t>(key - t_lo);
                    cent[pos] = base + st * 32 + lane;
                }
            }
            ncomp += __popc(m);
        }
    }
    __syncthreads();  // pre / hash zeroed by all threads before any count
    const bool listed = ncomp <= kCsrCap;
    if (listed) {
        for (int i = lane; i < ncomp; i += 32) {
            const int idx = warp * NS2 + ckey[i];
            atomicAdd(reinterpret_cast<uint32_t*>(pre) + (idx >> 1), 1u << (16 * (idx & 1)));
        }
    } else {
        for (int base = lo; base < hi; base += 32) {
            const int e = base + lane;
            int key = (e < hi) ? __ldg(keys + e) : -1;
            if (key >= t_lo && key < t_hi) {
                const int idx = warp * NS2 + (key - t_lo);
                atomicAdd(reinterpret_cast<uint32_t*>(pre) + (idx >> 1), 1u << (16 * (idx & 1)));
            }
        }
    }
    below = __reduce_add_sync(0xffffffffu, below);
    if (lane == 0) scratch[warp] = below;
    __syncthreads();
    int base_slot = 0;
    for (int w = 0; w < kCsrWarps; ++w) base_slot += scratch[w];
    __syncthreads();
    for (int t = tid; t < NS; t += kCsrThreads) {
        int run = 0;
        for (int w = 0; w < kCsrWarps; ++w) {
            const int c = pre[w * NS2 + t];
            pre[w * NS2 + t] = static_cast<uint16_t>(run);
            run += c;
        }
        off[t] = run;
    }
    __syncthreads();
    const int tot = block_scan(off, NS, scratch);
    int32_t* coff = a.csr_off + static_cast<size_t>(b) * (N + 1);
    for (int t = tid; t < NS; t += kCsrThreads) {
        off[t] += base_slot;
        coff[t_lo + t] = off[t];
    }
    if (tid == 0 && sl == slices - 1) coff[N] = base_slot + tot;
    __syncthreads();
    auto place = [&](bool in, int kk, int e) {
        const int h = kk & (kCsrHash - 1);
        ks[lane] = in ? kk : -1;
        if (in) atomicOr(&hb[h], 1u << lane);
        __syncwarp();
        unsigned peers = 0u;
        int before = 0;
        if (in) {
            unsigned mm = hb[h];
            while (mm) {
                const int l = __ffs(mm) - 1;
                mm &= mm - 1u;
                if (ks[l] == kk) peers |= 1u << l;
            }
            before = mine[kk];
            const int q = e / K, j = e - q * K;
            csr[off[kk] + before + __popc(peers & below_lanes)] = (q << 4) | j;
        }
        __syncwarp();
        if (in && lane == __ffs(peers) - 1) {
            mine[kk] = static_cast<uint16_t>(before + __popc(peers));
            hb[h] = 0u;
        }
        __syncwarp();
    };
    if (listed) {
        for (int i0 = 0; i0 < ncomp; i0 += 32) {
            const int i = i0 + lane;
            const bool in = i < ncomp;
            place(in, in ? ckey[i] : -1, in ? cent[i] : 0);
        }
    } else {
        for (int base = lo; base < hi; base += 32) {
            const int e = base + lane;
            int key = (e < hi) ? __ldg(keys + e) : -1;
            if (key >= N) key = -1;
            const bool in = key >= t_lo && key < t_hi;
            if (__ballot_sync(0xffffffffu, in) == 0u) continue;
            place(in, in ? key - t_lo : -1, e);
        }
    }
}

// Token side of the gather backward.  dF_t = sum of w * dOut over the token's entries, in
// the entry order the CSR holds.  Entry counts are very uneven (tokens on the rim of an
// empty region are the neighbours of many cells), so warps are persistent and take
// tokens from a work counter; all 32 / LPQ lane groups of a warp work on the same token,
// each on every S-th entry, and the group sums are combined by a fixed shuffle tree.
// Only the scheduling uses an atomic: each token's sum is formed the same way whichever
// warp runs it, so the result is bit-reproducible.  The first NH CTAs first reduce dp.
template <int CH>
__global__ void __launch_bounds__(kGatherThreads)
    knn_bwd_token_kernel(const KnnArgs a, int lpq_log2, int query_blocks) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int NH = a.d >> 5;
    if (static_cast<int>(blockIdx.x) < NH) {
        __shared__ float red[kGatherWarps];
        const int h = blockIdx.x;
        float acc = 0.f;
        for (int i = threadIdx.x; i < query_blocks; i += kGatherThreads)
            acc += a.dp_part[static_cast<size_t>(i) * NH + h];
        acc = warp_sum(acc);
        if (lane == 0) red[warp] = acc;
        __syncthreads();
        if (threadIdx.x == 0) {
            float tot = 0.f;
            for (int w = 0; w < kGatherWarps; ++w) tot += red[w];
            a.dp[h] = tot;
        }
    }
    const int LPQ = 1 << lpq_log2, S = 32 >> lpq_log2;
    const int sub = lane & (LPQ - 1), grp = lane >> lpq_log2;
    const int total = a.B * a.N;
    const int KN = a.K * NH;
    int next = 0;
    if (lane == 0) next = atomicAdd(a.counter, 1);
    next = __shfl_sync(0xffffffffu, next, 0);
    while (next < total) {
        const int gt = next;
        if (lane == 0) next = atomicAdd(a.counter, 1);  // fetch the following token early
        const int b = gt / a.N, t = gt - b * a.N;
        const int32_t* coff = a.csr_off + static_cast<size_t>(b) * (a.N + 1);
        const int lo = coff[t], hi = coff[t + 1];
        const int32_t* csr = a.csr + static_cast<size_t>(b) * a.Q * a.K;
        const size_t qbase = static_cast<size_t>(b) * a.Q;
#pragma unroll
        for (int ch = 0; ch < CH; ++ch) {
            const int c0 = ch * LPQ * 8 + sub * 8;
            const bool on = c0 < a.d;
            const int hh = on ? (c0 >> 5) : 0;
            const float* wb = a.w + qbase * KN + hh;
            const bf16* gb = a.dout + qbase * a.d + (on ? c0 : 0);
            float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            int i = lo + grp;
            for (; i + 3 * S < hi; i += 4 * S) {
                int e[4];
                float wv[4];
                uint4 gv[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) e[u] = __ldg(csr + i + u * S);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int q = e[u] >> 4, j = e[u] & 15;
                    wv[u] = __ldg(wb + q * KN + j * NH);
                    gv[u] = on ? ldg16(gb + q * a.d) : make_uint4(0u, 0u, 0u, 0u);
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) fma8(acc, wv[u], gv[u]);
            }
            for (; i < hi; i += S) {
                const int e = __ldg(csr + i);
                const int q = e >> 4, j = e & 15;
                fma8(acc, __ldg(wb + q * KN + j * NH), on ? ldg16(gb + q * a.d) : make_uint4(0u, 0u, 0u, 0u));
            }
            for (int o = LPQ; o < 32; o <<= 1) {
#pragma unroll
                for (int v = 0; v < 8; ++v) acc[v] += __shfl_xor_sync(0xffffffffu, acc[v], o);
            }
            if (on && grp == 0)
                *reinterpret_cast<uint4*>(a.dfeats + static_cast<size_t>(gt) * a.d + c0) = pack8(acc, 1.f);
        }
        next = __shfl_sync(0xffffffffu, next, 0);
    }
}

// lanes per query: d/8 rounded up to a power of two, capped at 32
int lpq_log2_for(int d) {
    int lanes = d / 8;
    int l2 = 0;
    while ((1 << l2) < lanes && l2 < 5) ++l2;
    return l2;
}

// Launch shape of the query-side gather kernels (used by the workspace layout too).
struct GatherPlan {
    int l2, ch, iters, blocks;
    bool shared;  // lane j of a query group owns neighbour j (needs K <= lanes per query)
};
GatherPlan gather_plan(int B, int Q, int d, int K) {
    GatherPlan g;
    g.l2 = lpq_log2_for(d);
    const int lanes = 1 << g.l2;
    g.ch = (d + 8 * lanes - 1) / (8 * lanes);
    g.shared = K <= lanes;
    const long long per_iter = static_cast<long long>(kGatherWarps) * (32 >> g.l2);
    const long long total = static_cast<long long>(B) * Q;
    g.iters = (g.shared && total >= per_iter * 4 * 148 * 2) ? 4 : 1;
    g.blocks = static_cast<int>((total + per_iter * g.iters - 1) / (per_iter * g.iters));
    return g;
}

template <int KT>
cudaError_t fwd_shared_k(const KnnArgs& a, cudaStream_t st, const GatherPlan& g) {
    const unsigned blocks = static_cast<unsigned>(g.blocks);
    switch (g.ch) {
        case 1: knn_fwd_shared_kernel<KT, 1><<<blocks, kGatherThreads, 0, st>>>(a, g.l2, g.iters); break;
        case 2: knn_fwd_shared_kernel<KT, 2><<<blocks, kGatherThreads, 0, st>>>(a, g.l2, g.iters); break;
        case 3: knn_fwd_shared_kernel<KT, 3><<<blocks, kGatherThreads, 0, st>>>(a, g.l2, g.iters); break;
        default: knn_fwd_shared_kernel<KT, 4><<<blocks, kGatherThreads, 0, st>>>(a, g.l2, g.iters); break;
    }
    return cudaGetLastError();
}

template <int KT>
cudaError_t bwdq_shared_k(const KnnArgs& a, cudaStream_t st, const GatherPlan& g, size_t smem) {
    const unsigned blocks = static_cast<unsigned>(g.blocks);
    switch (g.ch) {
        case 1: knn_bwd_query_shared_kernel<KT, 1><<<blocks, kGatherThreads, smem, st>>>(a, g.l2, g.iters); break;
        case 2: knn_bwd_query_shared_kernel<KT, 2><<<blocks, kGatherThreads, smem, st>>>(a, g.l2, g.iters); break;
        case 3: knn_bwd_query_shared_kernel<KT, 3><<<blocks, kGatherThreads, smem, st>>>(a, g.l2, g.iters); break;
        default: knn_bwd_query_shared_kernel<KT, 4><<<blocks, kGatherThreads, smem, st>>>(a, g.l2, g.iters); break;
    }
    return cudaGetLastError();
}

template <int KT>
cudaError_t fwd_k(const KnnArgs& a, cudaStream_t st, int l2, int ch, unsigned blocks) {
    switch (ch) {
        case 1: knn_fwd_kernel<KT, 1><<<blocks, kGatherThreads, 0, st>>>(a, l2); break;
        case 2: knn_fwd_kernel<KT, 2><<<blocks, kGatherThreads, 0, st>>>(a, l2); break;
        case 3: knn_fwd_kernel<KT, 3><<<blocks, kGatherThreads, 0, st>>>(a, l2); break;
        default: knn_fwd_kernel<KT, 4><<<blocks, kGatherThreads, 0, st>>>(a, l2); break;
    }
    return cudaGetLastError();
}

template <int KT>
cudaError_t bwdq_k(const KnnArgs& a, cudaStream_t st, int l2, int ch, unsigned blocks, size_t smem) {
    switch (ch) {
        case 1: knn_bwd_query_kernel<KT, 1><<<blocks, kGatherThreads, smem, st>>>(a, l2); break;
        case 2: knn_bwd_query_kernel<KT, 2><<<blocks, kGatherThreads, smem, st>>>(a, l2); break;
        case 3: knn_bwd_query_kernel<KT, 3><<<blocks, kGatherThreads, smem, st>>>(a, l2); break;
        default: knn_bwd_query_kernel<KT, 4><<<blocks, kGatherThreads, smem, st>>>(a, l2); break;
    }
    return cudaGetLastError();
}


}  // namespace

size_t knn_table_smem_bytes(int N, int nbins) {
    return ((4 * static_cast<size_t>(nbins + 40) + 15) & ~size_t(15)) + 10 * static_cast<size_t>(N);
}

cudaError_t launch_knn_table(const float* xy, int B, int N, int GH, int GW, int K, int32_t* table,
                             cudaStream_t st) {
    const BinGrid bg = choose_bins(N, GH, GW);
    const size_t smem = knn_table_smem_bytes(N, bg.nbx * bg.nby);
    const int tiles = ((GW + 7) / 8) * ((GH + 3) / 4);
    dim3 grid((tiles + kTableThreads / 32 - 1) / (kTableThreads / 32), B);
    cudaError_t e;
#define ACL_TABLE_CASE(KM)                                                                        \
    e = ensure_smem<knn_table_kernel<KM>>(smem);                                                  \
    if (e != cudaSuccess) return e;                                                               \
    knn_table_kernel<KM><<<grid, kTableThreads, smem, st>>>(xy, N, GH, GW, K, bg, table);
    if (K <= 1) { ACL_TABLE_CASE(1) }
    else if (K <= 2) { ACL_TABLE_CASE(2) }
    else if (K <= 4) { ACL_TABLE_CASE(4) }
    else if (K <= 8) { ACL_TABLE_CASE(8) }
    else { ACL_TABLE_CASE(16) }
#undef ACL_TABLE_CASE
    note_launch();
    return cudaGetLastError();
}

KnnWorkspace knn_workspace_layout(int B, int Q, int N, int d, int K) {
    auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
    const size_t NH = static_cast<size_t>(d / 32);
    const size_t BQ = static_cast<size_t>(B) * Q;
    KnnWorkspace w;
    w.query_blocks = gather_plan(B, Q, d, K).blocks;
    size_t off = 0;
    w.w = off;       off += up(sizeof(float) * BQ * NH * K);
    w.keys = off;    off += up(sizeof(int32_t) * BQ * K);
    w.csr = off;     off += up(sizeof(int32_t) * BQ * K);
    w.csr_off = off; off += up(sizeof(int32_t) * static_cast<size_t>(B) * (N + 1));
    w.dp_part = off; off += up(sizeof(float) * static_cast<size_t>(w.query_blocks) * NH);
    w.counter = off; off += up(sizeof(int));
    w.total = off;
    return w;
}

cudaError_t launch_knn_fwd(const KnnArgs& a, cudaStream_t st) {
    const GatherPlan g = gather_plan(a.B, a.Q, a.d, a.K);
    if (g.blocks == 0) return cudaSuccess;
    cudaError_t e;
    if (g.shared)
        e = (a.K <= 8) ? fwd_shared_k<8>(a, st, g) : fwd_shared_k<16>(a, st, g);
    else
        e = (a.K <= 8) ? fwd_k<8>(a, st, g.l2, g.ch, g.blocks) : fwd_k<16>(a, st, g.l2, g.ch, g.blocks);
    note_launch();
    return e;
}

cudaError_t launch_knn_bwd(const KnnArgs& a, cudaStream_t st) {
    const int l2 = lpq_log2_for(a.d);
    const int lanes = 1 << l2;
    const int ch = (a.d + 8 * lanes - 1) / (8 * lanes);
    const int NH = a.d / 32;
    const KnnWorkspace ws = knn_workspace_layout(a.B, a.Q, a.N, a.d, a.K);
    const unsigned qblocks = static_cast<unsigned>(ws.query_blocks);
    const GatherPlan g = gather_plan(a.B, a.Q, a.d, a.K);
    cudaError_t e = cudaSuccess;
    if (qblocks > 0) {
        const size_t smem = sizeof(float) * kGatherWarps * (32 >> l2) * NH;
        if (g.shared)
            e = (a.K <= 8) ? bwdq_shared_k<8>(a, st, g, smem) : bwdq_shared_k<16>(a, st, g, smem);
        else
            e = (a.K <= 8) ? bwdq_k<8>(a, st, l2, ch, qblocks, smem) : bwdq_k<16>(a, st, l2, ch, qblocks, smem);
        note_launch();
        if (e != cudaSuccess) return e;
    }
    // the inverse index is built even for Q == 0 (it then writes empty lists)
    int slices = 148 / (a.B > 0 ? a.B : 1);
    if (slices > 8) slices = 8;
    if (slices < 1) slices = 1;
    if (slices > (a.N + 31) / 32) slices = (a.N + 31) / 32;
    const size_t csmem = csr_smem_layout((a.N + slices - 1) / slices).total;
    e = ensure_smem<knn_csr_kernel>(csmem);
    if (e != cudaSuccess) return e;
    knn_csr_kernel<<<dim3(slices, a.B), kCsrThreads, csmem, st>>>(a, slices);
    note_launch();
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int qb = static_cast<int>(qblocks);
    const unsigned tblocks = static_cast<unsigned>(148 * 4 > NH ? 148 * 4 : NH);
    switch (ch) {
        case 1: knn_bwd_token_kernel<1><<<tblocks, kGatherThreads, 0, st>>>(a, l2, qb); break;
        case 2: knn_bwd_token_kernel<2><<<tblocks, kGatherThreads, 0, st>>>(a, l2, qb); break;
        case 3: knn_bwd_token_kernel<3><<<tblocks, kGatherThreads, 0, st>>>(a, l2, qb); break;
        default: knn_bwd_token_kernel<4><<<tblocks, kGatherThreads, 0, st>>>(a, l2, qb); break;
    }
    note_launch();
    return cudaGetLastError();
}

}  // namespace acl
