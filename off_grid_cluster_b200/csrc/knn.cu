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
// is built per image by a stable counting sort (integer only).  Token side: a warp
// (or, for a token with many entries, a whole CTA) sums w * dOut over the token's
// entries in a fixed order of streams and combining steps.
#include <climits>
#include <float.h>
#include <math.h>


#include "internal.h"

namespace acl {

namespace {

constexpr int kTableThreads = 512;
constexpr int kTableSub = 4;  // lanes per cell in the table search
constexpr int kGatherWarps = 8;
constexpr int kGatherThreads = 32 * kGatherWarps;
constexpr int kCsrThreads = 1024;

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

// (d, t) < (d', t') in the table's order: distance, then token id
__device__ __forceinline__ bool dt_less(double d, int t, double d2, int t2) {
    return d < d2 || (d == d2 && t < t2);
}

// Insert (d, t) into the ascending top-K list: every slot compares with the new pair at
// once (the list is sorted, so the slots below it form a prefix), then shifts or takes it.
template <int KMAX>
__device__ __forceinline__ void topk_insert_par(double (&bd)[KMAX], int (&bi)[KMAX], double d, int t) {
    if (!dt_less(d, t, bd[KMAX - 1], bi[KMAX - 1])) return;
    bool lt[KMAX];
#pragma unroll
    for (int r = 0; r < KMAX; ++r) lt[r] = dt_less(bd[r], bi[r], d, t);
#pragma unroll
    for (int r = KMAX - 1; r >= 1; --r) {
        if (!lt[r]) {
            bd[r] = lt[r - 1] ? d : bd[r - 1];
            bi[r] = lt[r - 1] ? t : bi[r - 1];
        }
    }
    if (!lt[0]) {
        bd[0] = d;
        bi[0] = t;
    }
}

// In place: the K smallest of this lane's ascending list and the list of lane ^ o, as a
// bitonic sequence (element r is the smaller of A[r] and B[K-1-r]).
template <int KMAX>
__device__ __forceinline__ void merge_lows(double (&bd)[KMAX], int (&bi)[KMAX], int o) {
    double od[KMAX];
    int oi[KMAX];
#pragma unroll
    for (int r = 0; r < KMAX; ++r) {
        od[r] = __shfl_xor_sync(0xffffffffu, bd[r], o);
        oi[r] = __shfl_xor_sync(0xffffffffu, bi[r], o);
    }
#pragma unroll
    for (int r = 0; r < KMAX; ++r) {
        if (!dt_less(bd[r], bi[r], od[KMAX - 1 - r], oi[KMAX - 1 - r])) {
            bd[r] = od[KMAX - 1 - r];
            bi[r] = oi[KMAX - 1 - r];
        }
    }
}

// Sort a bitonic sequence ascending (half-cleaners of decreasing span).
template <int KMAX>
__device__ __forceinline__ void bitonic_finish(double (&cd)[KMAX], int (&ci)[KMAX]) {
#pragma unroll
    for (int span = KMAX / 2; span >= 1; span >>= 1) {
#pragma unroll
        for (int r = 0; r < KMAX; ++r) {
            if ((r & span) == 0) {
                const int u = r + span;
                if (dt_less(cd[u], ci[u], cd[r], ci[r])) {
                    const double td = cd[r]; cd[r] = cd[u]; cd[u] = td;
                    const int ti = ci[r]; ci[r] = ci[u]; ci[u] = ti;
                }
            }
        }
    }
}

// One warp per 4 x 2 tile of cells, kTableSub lanes per cell (lane = cell * kTableSub +
// sub).  Bin rows are contiguous runs of the bin-sorted tokens; sub-lane p of every cell
// takes the run's candidates i = p (mod kTableSub), all cells reading the same candidate
// (a shared-memory broadcast), and keeps its own ascending (fp64 distance, id) top-K.  A
// candidate whose fp32 squared distance exceeds a bound of the cell's K-th best by more
// than the fp32 rounding bound cannot enter the top-K and is skipped.  Bins are visited in
// rings around the tile's own bins, nearest first.  After each ring the cell's K-th best
// is bounded above by the largest of its sub-lanes' ceil(K / kTableSub)-th entries (those
// prefixes hold at least K distinct tokens); every cell checks that the bound is below its
// distance to the scanned rectangle's edge (tokens outside lie beyond it, and rounding is
// monotone), and the warp stops once all cells are proven.  The sub-lanes' lists are then
// merged (bitonic, over shuffles); each token was seen by exactly one sub-lane, so the
// merged list is the top-K of all candidates.
template <int KMAX>
__global__ void __launch_bounds__(kTableThreads, KMAX <= 8 ? 2 : 1)
    knn_table_kernel(const float* __restrict__ xy, int N, int GH, int GW, int K, BinGrid bg,
                     int32_t* __restrict__ table) {
    static_assert(kTableSub == 4, "the merge below takes two levels");
    extern __shared__ __align__(128) uint8_t smem[];
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

    const int tiles_x = (GW + 3) >> 2, tiles_y = (GH + 1) >> 1;
    const int tile = blockIdx.x * (kTableThreads / 32) + warp;
    if (tile >= tiles_x * tiles_y) return;
    const int tx0 = (tile % tiles_x) * 4, ty0 = (tile / tiles_x) * 2;
    const int cell = lane / kTableSub, sub = lane % kTableSub;
    const int c = tx0 + (cell & 3), r = ty0 + (cell >> 2);
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
    auto tighten = [&](double kth) {
        if (kth < DBL_MAX) thr = fminf(thr, static_cast<float>(kth) * (1.0f + 1.0f / 1048576.0f));
    };
    // scan one contiguous run of bins [b0, b1] (one bin row), this sub-lane's share
    auto scan_run = [&](int b0, int b1) {
        const int s0 = b0 > 0 ? cnt[b0 - 1] : 0, s1 = cnt[b1];
        for (int i = s0 + sub; i < s1; i += kTableSub) {
            const float2 p = txy[i];
            const float dxf = p.x - pxf, dyf = p.y - pyf;
            const float d2f = fmaf(dxf, dxf, dyf * dyf);
            if (d2f <= thr) {
                const double dx = __dsub_rn(static_cast<double>(p.x), px);
                const double dy = __dsub_rn(static_cast<double>(p.y), py);
                topk_insert_par<KMAX>(bd, bi, __dadd_rn(__dmul_rn(dx, dx), __dmul_rn(dy, dy)), tidv[i]);
                tighten(bd[KMAX - 1]);
            }
        }
    };
    // the tile's footprint in bins; rings of bins around it are scanned nearest first
    const int tbx0 = bin_coord(static_cast<float>(tx0) + 0.5f, bg.inv_s, bg.nbx);
    const int tbx1 = bin_coord(static_cast<float>(min(tx0 + 4, GW)) - 0.5f, bg.inv_s, bg.nbx);
    const int tby0 = bin_coord(static_cast<float>(ty0) + 0.5f, bg.inv_s, bg.nby);
    const int tby1 = bin_coord(static_cast<float>(min(ty0 + 2, GH)) - 0.5f, bg.inv_s, bg.nby);
    const double s = static_cast<double>(bg.s);
    const int maxring = max(bg.nbx, bg.nby);
    const int kq = (K + kTableSub - 1) / kTableSub - 1;
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
        // an upper bound of the cell's K-th best: the sub-lanes' first ceil(K / kTableSub)
        // entries are at least K distinct tokens, so the K-th best is at most their maximum
        double kth = DBL_MAX;
#pragma unroll
        for (int k = 0; k < KMAX; ++k)
            if (k == kq) kth = bd[k];
        kth = fmax(kth, __shfl_xor_sync(0xffffffffu, kth, 1));
        kth = fmax(kth, __shfl_xor_sync(0xffffffffu, kth, 2));
        tighten(kth);
        // distance from the cell centre to the edge of the scanned rectangle; a side on the
        // grid border is unbounded (tokens outside the grid fall into border bins)
        double m = DBL_MAX;
        if (bx_lo > 0) m = fmin(m, px - bx_lo * s);
        if (bx_hi < bg.nbx - 1) m = fmin(m, (bx_hi + 1) * s - px);
        if (by_lo > 0) m = fmin(m, py - by_lo * s);
        if (by_hi < bg.nby - 1) m = fmin(m, (by_hi + 1) * s - py);
        const bool proven = (m == DBL_MAX) || (kth < m * m);
        if (__all_sync(0xffffffffu, proven)) break;
    }
    // final list: merge the sub-lanes' lists (two levels), sub-lane 0 writes it
    merge_lows<KMAX>(bd, bi, 1);
    bitonic_finish<KMAX>(bd, bi);
    merge_lows<KMAX>(bd, bi, 2);
    bitonic_finish<KMAX>(bd, bi);
    if (sub != 0 || c >= GW || r >= GH) return;
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

// The two weight kernels share one form: w_k = 2^(-p (v_k - v_min)) / sum, with
// v = d log2(e) for the exponential kernel (exp(-p (d - d_min))) and v = log2(d) for the
// inverse power ((d_min / d)^p).  A neighbour at v_min gets 1 (for the inverse power at
// d_min = 0 that is the d -> 0 limit); p = 0 gives equal weights.
__device__ __forceinline__ float knn_v(float d, int kind) { return kind ? log2f(d) : d * kLog2e; }
__device__ __forceinline__ float knn_weight(float v, float vmin, float p) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(-p * (v - vmin)));
    return (v == vmin || p == 0.f) ? 1.f : y;
}
// -dz/dp for z = -p d (d) or z = -p ln d (ln d; 0 at d = 0), from v
__device__ __forceinline__ float knn_dzdp(float v) { return v == -INFINITY ? 0.f : v * kLn2; }
// f with dz/dq = -p f (q - x): 1 / d or 1 / d^2, 0 at d = 0
__device__ __forceinline__ float knn_dq_factor(float d, int kind) {
    return d > 0.f ? (kind ? 1.f / (d * d) : 1.f / d) : 0.f;
}

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
        ACL_DEVICE_CHECK(t >= -1 && t < a.N);
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

__device__ __forceinline__ uint4 pack8(const float (&v)[8], float s) {
    uint4 o;
    o.x = pack_bf16(v[0] * s, v[1] * s);
    o.y = pack_bf16(v[2] * s, v[3] * s);
    o.z = pack_bf16(v[4] * s, v[5] * s);
    o.w = pack_bf16(v[6] * s, v[7] * s);
    return o;
}

// Packed f32x2 arithmetic (fp32 pairs held in 64-bit registers).
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ float2 f2_unpack(uint64_t r) {
    float2 v;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(v.x), "=f"(v.y) : "l"(r));
    return v;
}
// acc[i] += ww * (the two bf16 of f word i, widened to fp32): one row of 8 channels
__device__ __forceinline__ void row_fma(uint64_t (&acc)[4], uint64_t ww, uint4 f) {
    asm("{\n\t.reg .b32 l0, h0, l1, h1, l2, h2, l3, h3;\n\t.reg .b64 p0, p1, p2, p3;\n\t"
        "shl.b32 l0, %5, 16;\n\tand.b32 h0, %5, 0xffff0000;\n\t"
        "shl.b32 l1, %6, 16;\n\tand.b32 h1, %6, 0xffff0000;\n\t"
        "shl.b32 l2, %7, 16;\n\tand.b32 h2, %7, 0xffff0000;\n\t"
        "shl.b32 l3, %8, 16;\n\tand.b32 h3, %8, 0xffff0000;\n\t"
        "mov.b64 p0, {l0, h0};\n\tmov.b64 p1, {l1, h1};\n\t"
        "mov.b64 p2, {l2, h2};\n\tmov.b64 p3, {l3, h3};\n\t"
        "fma.rn.f32x2 %0, %4, p0, %0;\n\tfma.rn.f32x2 %1, %4, p1, %1;\n\t"
        "fma.rn.f32x2 %2, %4, p2, %2;\n\tfma.rn.f32x2 %3, %4, p3, %3;\n\t}"
        : "+l"(acc[0]), "+l"(acc[1]), "+l"(acc[2]), "+l"(acc[3])
        : "l"(ww), "r"(f.x), "r"(f.y), "r"(f.z), "r"(f.w));
}
__device__ __forceinline__ void unpack_acc(const uint64_t (&acc)[4], float (&v)[8]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 x = f2_unpack(acc[i]);
        v[2 * i] = x.x;
        v[2 * i + 1] = x.y;
    }
}

// Neighbour j of a query: token id (-1 for an empty slot or an id >= N) and weight
// exponent v = knn_v(d) (+inf for an empty slot).
__device__ __forceinline__ void one_neighbour(const KnnArgs& a, const int32_t* row, const float2* xyb,
                                              float2 qp, int j, int& t, float& v) {
    t = __ldg(row + j);
    ACL_DEVICE_CHECK(t >= -1 && t < a.N);
    v = INFINITY;
    if (t >= a.N) t = -1;
    if (t >= 0) {
        const float2 p = __ldg(xyb + t);
        const float dx = qp.x - p.x, dy = qp.y - p.y;
        v = knn_v(sqrtf(dx * dx + dy * dy), a.kind);
    }
}

// All K neighbours of a query group's query in every lane of the group (slots K..KT-1
// empty); returns the minimum v.  With K <= LPQ lane j of the group looks up neighbour j
// and the group shares them by shuffles (all 32 lanes must call); otherwise every lane
// looks up all K.
template <int KT>
__device__ __forceinline__ float query_neighbours(const KnnArgs& a, int b, bool live, float2 qp,
                                                  int sub, int LPQ, int (&t)[KT], float (&v)[KT],
                                                  int* own_t = nullptr, float* own_v = nullptr) {
    const int cy = quantise(qp.y, a.GH), cx = quantise(qp.x, a.GW);
    const int32_t* row = a.table + ((static_cast<size_t>(b) * a.GH + cy) * a.GW + cx) * a.K;
    const float2* xyb = reinterpret_cast<const float2*>(a.xy) + static_cast<size_t>(b) * a.N;
    float vmin = INFINITY;
    if (a.K <= LPQ) {
        int my_t = -1;
        float my_v = INFINITY;
        if (live && sub < a.K) one_neighbour(a, row, xyb, qp, sub, my_t, my_v);
        if (own_t) *own_t = my_t;
        if (own_v) *own_v = my_v;
        vmin = my_v;
        for (int o = 1; o < LPQ; o <<= 1) vmin = fminf(vmin, __shfl_xor_sync(0xffffffffu, vmin, o, LPQ));
#pragma unroll
        for (int j = 0; j < KT; ++j) {
            const int tj = __shfl_sync(0xffffffffu, my_t, j, LPQ);
            const float vj = __shfl_sync(0xffffffffu, my_v, j, LPQ);
            t[j] = j < a.K ? tj : -1;
            v[j] = j < a.K ? vj : INFINITY;
        }
    } else {
#pragma unroll
        for (int j = 0; j < KT; ++j) {
            t[j] = -1;
            v[j] = INFINITY;
            if (live && j < a.K) one_neighbour(a, row, xyb, qp, j, t[j], v[j]);
            vmin = fminf(vmin, v[j]);
        }
    }
    return vmin;
}

// Forward.  A group of LPQ lanes owns a query; lane sub owns channels [8 (ch LPQ + sub),
// +8) of pass ch (one 16-byte load per neighbour row and pass).  The K weights of the
// lane's head are formed once per pass and the rows accumulate with packed f32x2 FMAs.
// CTA c takes the `span` consecutive queries from c * span, so neighbouring queries (which
// share most of their rows) run on one SM and meet each other's rows in L1.
template <int KT, int CH>
__global__ void __launch_bounds__(kGatherThreads, 2) knn_fwd_kernel(const KnnArgs a, int lpq_log2, long long span) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int LPQ = 1 << lpq_log2, QPW = 32 >> lpq_log2;
    const int sub = lane & (LPQ - 1), grp = lane >> lpq_log2;
    const long long total = static_cast<long long>(a.B) * a.Q;
    const long long q0 = static_cast<long long>(blockIdx.x) * span;
    const long long q1 = q0 + span < total ? q0 + span : total;
    long long gq = q0 + static_cast<long long>(warp) * QPW + grp;
    // image of query gq and its first query, advanced without divisions
    int b = static_cast<int>(gq / a.Q);
    long long qb = static_cast<long long>(b) * a.Q;
    for (; gq - grp < q1; gq += kGatherWarps * QPW) {
        while (gq - qb >= a.Q) {
            ++b;
            qb += a.Q;
        }
        const bool live = gq < q1;
        const float2 qp = live ? __ldg(reinterpret_cast<const float2*>(a.queries) + gq) : make_float2(0.f, 0.f);
        int t[KT];
        float v[KT];
        const float vmin = query_neighbours<KT>(a, live ? b : 0, live, qp, sub, LPQ, t, v);
        if (!live) continue;  // no shuffles below
        // per neighbour: the row's first channel of this lane and the weight exponent
        // e = v_min - v (0 at the nearest, -inf for an empty slot): w = 2^(p e)
        const bf16* rowp[KT];
        float e[KT];
        {
            const bf16* fb = a.feats + static_cast<size_t>(b) * a.N * a.d + sub * 8;
#pragma unroll
            for (int j = 0; j < KT; ++j) {
                rowp[j] = fb + static_cast<size_t>(t[j] < 0 ? 0 : t[j]) * a.d;
                e[j] = t[j] < 0 ? -INFINITY : (v[j] == vmin ? 0.f : vmin - v[j]);
            }
        }
        bf16* ob = a.out + static_cast<size_t>(gq) * a.d + sub * 8;
#pragma unroll
        for (int ch = 0; ch < CH; ++ch) {
            // passes after the first exist only with LPQ = 32: pass ch starts at channel 256 ch
            const int c0 = ch * 256 + sub * 8;
            if (c0 >= a.d) break;
            uint4 f[KT];
#pragma unroll
            for (int j = 0; j < KT; ++j) f[j] = t[j] >= 0 ? ldg16(rowp[j] + ch * 256) : make_uint4(0u, 0u, 0u, 0u);
            const float ph = __ldg(a.p + (c0 >> 5));
            const bool flat = ph == 0.f;  // p = 0: equal weights
            float w[KT];
            float sum = 0.f;
#pragma unroll
            for (int j = 0; j < KT; ++j) {
                float y;
                asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(ph * e[j]));
                w[j] = t[j] < 0 ? 0.f : (flat ? 1.f : y);
                sum += w[j];
            }
            uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
            for (int j = 0; j < KT; ++j) row_fma(acc, f2_pack(w[j], w[j]), f[j]);
            const float inv = sum > 0.f ? __fdividef(1.f, sum) : 0.f;
            const float2 a0 = f2_unpack(acc[0]), a1 = f2_unpack(acc[1]), a2 = f2_unpack(acc[2]),
                         a3 = f2_unpack(acc[3]);
            uint4 o;
            o.x = pack_bf16(a0.x * inv, a0.y * inv);
            o.y = pack_bf16(a1.x * inv, a1.y * inv);
            o.z = pack_bf16(a2.x * inv, a2.y * inv);
            o.w = pack_bf16(a3.x * inv, a3.y * inv);
            *reinterpret_cast<uint4*>(ob + ch * 256) = o;
        }
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
    } else {
#pragma unroll
        for (int j = 0; j < KT; ++j) {
            nb[j].t = -1;
            nb[j].d = INFINITY;
            nb[j].x = nb[j].y = 0.f;
        }
    }
    const bf16* fb = a.feats + static_cast<size_t>(b) * a.N * a.d;
    const float vmin = knn_v(dmin, a.kind);
    float v[KT];
#pragma unroll
    for (int j = 0; j < KT; ++j) v[j] = knn_v(nb[j].d, a.kind);
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
            const bool ok = on && nb[j].t >= 0;
            w[j] = ok ? knn_weight(v[j], vmin, ph) : 0.f;
            sum += w[j];
            const uint4 f = ok ? ldg16(fb + static_cast<size_t>(nb[j].t) * a.d + c0)
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
                dph -= ds * knn_dzdp(v[j]);
                const float cf = -ds * ph * knn_dq_factor(nb[j].d, a.kind);
                dqx += cf * (qp.x - nb[j].x);
                dqy += cf * (qp.y - nb[j].y);
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
// The neighbour that lane sub (< K) of a query's lane group owns: token id, weight
// exponent v = knn_v(d), and (q - p) * knn_dq_factor(d); returns the group's minimum v.
__device__ __forceinline__ float own_neighbour(const KnnArgs& a, int b, bool live, float2 qp,
                                               int sub, int LPQ, int& t, float& v, float& ux,
                                               float& uy) {
    if (live && sub < a.K) {
        const int cy = quantise(qp.y, a.GH), cx = quantise(qp.x, a.GW);
        t = a.table[((static_cast<size_t>(b) * a.GH + cy) * a.GW + cx) * a.K + sub];
        ACL_DEVICE_CHECK(t >= -1 && t < a.N);
        if (t >= a.N) t = -1;
        if (t >= 0) {
            const float2 p = reinterpret_cast<const float2*>(a.xy)[static_cast<size_t>(b) * a.N + t];
            const float dx = qp.x - p.x, dy = qp.y - p.y;
            const float d = sqrtf(dx * dx + dy * dy);
            v = knn_v(d, a.kind);
            const float f = knn_dq_factor(d, a.kind);
            ux = dx * f;
            uy = dy * f;
        }
    }
    float vmin = v;
    for (int o = 1; o < LPQ; o <<= 1) vmin = fminf(vmin, __shfl_xor_sync(0xffffffffu, vmin, o, LPQ));
    return vmin;
}

template <int KT, int CH>
__global__ void __launch_bounds__(kGatherThreads, (KT <= 8 && CH == 1) ? 4 : 2)
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
    // image of the lane's query and its first query, advanced without divisions
    const long long gq0 = (static_cast<long long>(blockIdx.x) * iters * kGatherWarps + warp) * QPW + grp;
    int bq = static_cast<int>(gq0 / a.Q);
    long long qb = static_cast<long long>(bq) * a.Q;
    for (int it = 0; it < iters; ++it) {
        const long long gq = gq0 + static_cast<long long>(it) * kGatherWarps * QPW;
        if ((gq - grp) >= total) break;  // uniform per warp
        while (gq - qb >= a.Q) {
            ++bq;
            qb += a.Q;
        }
        const bool live = gq < total;
        const int b = live ? bq : 0;
        const float2 qp = live ? reinterpret_cast<const float2*>(a.queries)[gq] : make_float2(0.f, 0.f);
        // lane j < K of the group owns neighbour j; every lane gets all K token ids
        int my_t = -1;
        float my_v = INFINITY, my_ux = 0.f, my_uy = 0.f;
        const float vmin = own_neighbour(a, b, live, qp, sub, LPQ, my_t, my_v, my_ux, my_uy);
        const int r = sub & 3;  // lane within the 4 lanes of a head
        constexpr int KQ = KT / 4;  // neighbours per lane after the reduce-scatter: j = r + 4 u
        // every neighbour's row (this lane's first channel; row 0 for an empty slot), and the
        // token, weight exponent and dq factor of this lane's neighbours j = r + 4 u: fixed for
        // the query, so taken once before the channel passes
        const bf16* rowp[KT];
        bool has[KT];
        {
            const bf16* fb = a.feats + static_cast<size_t>(b) * a.N * a.d + sub * 8;
#pragma unroll
            for (int j = 0; j < KT; ++j) {
                const int tj = __shfl_sync(0xffffffffu, my_t, j, LPQ);
                has[j] = live && tj >= 0;
                rowp[j] = fb + static_cast<size_t>(tj < 0 ? 0 : tj) * a.d;
            }
        }
        float vj[KQ], uxj[KQ], uyj[KQ];
        bool okq[KQ];
#pragma unroll
        for (int u = 0; u < KQ; ++u) {
            const int j = r + 4 * u;
            const int t = __shfl_sync(0xffffffffu, my_t, j, LPQ);
            vj[u] = __shfl_sync(0xffffffffu, my_v, j, LPQ);
            uxj[u] = __shfl_sync(0xffffffffu, my_ux, j, LPQ);
            uyj[u] = __shfl_sync(0xffffffffu, my_uy, j, LPQ);
            okq[u] = live && j < a.K && t >= 0;
        }
        const bf16* gb = a.dout + static_cast<size_t>(live ? gq : 0) * a.d + sub * 8;
        float dqx = 0.f, dqy = 0.f;
#pragma unroll
        for (int ch = 0; ch < CH; ++ch) {
            // passes after the first exist only with LPQ = 32: pass ch starts at channel 256 ch
            const int c0 = ch * 256 + sub * 8;
            const bool on = live && c0 < a.d;
            const int hh = on ? (c0 >> 5) : 0;
            const float ph = on ? a.p[hh] : 0.f;
            float g[8];
            {
                const uint4 gv = on ? ldg16(gb + ch * 256) : make_uint4(0u, 0u, 0u, 0u);
                const uint32_t u[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    g[2 * i] = bf16_lo(u[i]);
                    g[2 * i + 1] = bf16_hi(u[i]);
                }
            }
            // this lane's 8-channel share of dw_j = <dOut_h, f_j,h> for every neighbour
            float dwp[KT];
            {
                uint4 f[KT];
#pragma unroll
                for (int j = 0; j < KT; ++j)
                    f[j] = (on && has[j]) ? ldg16(rowp[j] + ch * 256) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                for (int j = 0; j < KT; ++j) {
                    const uint32_t u[4] = {f[j].x, f[j].y, f[j].z, f[j].w};
                    float acc = 0.f;
#pragma unroll
                    for (int i = 0; i < 4; ++i) acc += g[2 * i] * bf16_lo(u[i]) + g[2 * i + 1] * bf16_hi(u[i]);
                    dwp[j] = acc;
                }
            }
            // reduce-scatter over the head's 4 lanes: after the xor-2 step a lane holds the
            // j whose bit 1 matches bit 1 of r, after the xor-1 step the j = r + 4 u
            float dh[KT / 2];
#pragma unroll
            for (int s2 = 0; s2 < KT / 2; ++s2) {
                const int jlo = (s2 & 1) | ((s2 >> 1) << 2), jhi = jlo | 2;
                const float send = (r & 2) ? dwp[jlo] : dwp[jhi];
                const float keep = (r & 2) ? dwp[jhi] : dwp[jlo];
                dh[s2] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
            }
            float dw[KQ], w[KQ];
            bool okj[KQ];
            float sum = 0.f;
#pragma unroll
            for (int u = 0; u < KQ; ++u) {
                const float send = (r & 1) ? dh[2 * u] : dh[2 * u + 1];
                const float keep = (r & 1) ? dh[2 * u + 1] : dh[2 * u];
                dw[u] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
                okj[u] = on && okq[u];
                w[u] = okj[u] ? knn_weight(vj[u], vmin, ph) : 0.f;
                sum += w[u];
            }
            sum += __shfl_xor_sync(0xffffffffu, sum, 1);
            sum += __shfl_xor_sync(0xffffffffu, sum, 2);
            const float inv = sum > 0.f ? 1.f / sum : 0.f;
            float sdw = 0.f;
#pragma unroll
            for (int u = 0; u < KQ; ++u) {
                w[u] *= inv;
                sdw += w[u] * dw[u];
            }
            sdw += __shfl_xor_sync(0xffffffffu, sdw, 1);
            sdw += __shfl_xor_sync(0xffffffffu, sdw, 2);
            float dph = 0.f;
            float* wout = a.w + static_cast<size_t>(gq) * a.K * NH + hh;
#pragma unroll
            for (int u = 0; u < KQ; ++u) {
                const int j = r + 4 * u;
                if (on && j < a.K) wout[j * NH] = w[u];
                if (!okj[u]) continue;
                const float ds = w[u] * (dw[u] - sdw);
                dph -= ds * knn_dzdp(vj[u]);
                const float cf = -ds * ph;
                dqx += cf * uxj[u];
                dqy += cf * uyj[u];
            }
            dph += __shfl_xor_sync(0xffffffffu, dph, 1);
            dph += __shfl_xor_sync(0xffffffffu, dph, 2);
            if (on && r == 0) sdp[(warp * QPW + grp) * NH + hh] += dph;
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

// Query side of the backward on the tensor cores, for images of at most kUTMaxN tokens and
// K <= 8: a CTA takes tiles of 16 consecutive queries of one image.  The tile's (query, slot)
// entries name at most 128 tokens; their union U (ascending token id, found with a bitmap of
// the image's tokens and prefix popcounts) is the tile's set of F rows, so one row of F serves
// every query of the tile that lists it.  Per head, dW (16 x U) = dO_h (16 x 32) F_U,h^T is
// one row of m16n8k16 bf16 products (fp32 accumulation; both operands exact in bf16) whose
// operands are 16-byte loads of dO and F rows straight into the fragments, written to the
// warp's shared dW tile in fp32; each (query, slot) then reads its dw at its token's union
// position and the rest is the per-query algebra of the FMA query pass: w = 2^(p e) / S,
// ds = w (dw - sum w dw), dp and dq partials, w stored as [q][slot][head].  Thread (q, k) of
// the CTA's 128 builds the tile's entry (q, k); warp w takes heads w, w + 4, ...; dq adds the
// warps' partials in warp order and dp leaves each warp in a fixed order: bit-reproducible.
constexpr int kUTWarps = 4;
constexpr int kUTThreads = 32 * kUTWarps;
constexpr int kUTMaxN = 2048;             // bitmap capacity (tokens per image)
constexpr int kUTUseN = 1024;             // images of at most this many tokens take this pass
                                          // (at 2048 tokens the FMA passes measured as fast
                                          // or faster: forward 27 against 30 us at 16 x 4096
                                          // queries, backward equal)
constexpr int kUTMaxU = 128;              // 16 queries x 8 slots
constexpr int kUTDS = kUTMaxU + 4;        // row stride of a warp's dW tile (floats)
constexpr int kUTBatch = 4;               // n-tiles (8 union rows each) whose rows load together

struct UTSmem {
    size_t bits, pre, utok, qloc, qe, qz, qu, dqred, dw, wblk, total;
};
// wblk: the tile's w block, [query][slot][head] with rows of NH + 1 floats
__host__ __device__ __forceinline__ UTSmem ut_smem_layout(int NH) {
    UTSmem L;
    size_t o = 0;
    auto take = [&](size_t bytes) {
        const size_t at = o;
        o = (o + bytes + 127) & ~size_t(127);
        return at;
    };
    L.bits = take(4 * (kUTMaxN / 32));
    L.pre = take(4 * (kUTMaxN / 32 + 1));
    L.utok = take(4 * kUTMaxU);
    L.qloc = take(4 * kUTMaxU);
    L.qe = take(4 * kUTMaxU);
    L.qz = take(4 * kUTMaxU);
    L.qu = take(8 * kUTMaxU);
    L.dqred = take(8 * kUTWarps * 16);
    L.dw = take(4 * kUTWarps * 16 * kUTDS);
    L.wblk = take(4 * 16 * 8 * (NH + 1));
    L.total = o;
    return L;
}

__global__ void __launch_bounds__(kUTThreads)
    knn_bwd_query_union_kernel(const KnnArgs a, long long tiles_per_image, long long tile_span) {
    extern __shared__ __align__(128) uint8_t smem[];
    const UTSmem L = ut_smem_layout(a.d >> 5);
    uint32_t* bits = reinterpret_cast<uint32_t*>(smem + L.bits);
    int* pre = reinterpret_cast<int*>(smem + L.pre);
    int* utok = reinterpret_cast<int*>(smem + L.utok);
    int* qloc = reinterpret_cast<int*>(smem + L.qloc);
    float* qe = reinterpret_cast<float*>(smem + L.qe);
    float* qz = reinterpret_cast<float*>(smem + L.qz);
    float2* qu = reinterpret_cast<float2*>(smem + L.qu);
    float2* dqred = reinterpret_cast<float2*>(smem + L.dqred);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    float* dws = reinterpret_cast<float*>(smem + L.dw) + warp * 16 * kUTDS;
    float* wblk = reinterpret_cast<float*>(smem + L.wblk);
    const int NH = a.d >> 5, NW = (a.N + 31) >> 5;
    const int WS = NH + 1;  // row stride of the w block
    // the w block copy: this thread's first float (row, column) and its step of kUTThreads floats
    const int wr0 = tid / NH, wc0 = tid - (tid / NH) * NH;
    const int wdr = kUTThreads / NH, wdc = kUTThreads - (kUTThreads / NH) * NH;
    const int K = a.K;
    // this lane's four (query, slot) pairs in the per-head algebra: q = lane / 2, k = 4 (lane & 1) + i
    const int pq = lane >> 1, pk0 = 4 * (lane & 1);
    const int g = lane >> 2, tq = lane & 3;  // the mma fragments' row and column pair
    float dpa[8];  // dp partials of this warp's heads h = warp + 4 s (s < 8 covers NH <= 32)
#pragma unroll
    for (int s = 0; s < 8; ++s) dpa[s] = 0.f;
    const long long total_tiles = static_cast<long long>(a.B) * tiles_per_image;
    const long long t0 = static_cast<long long>(blockIdx.x) * tile_span;
    const long long t1 = t0 + tile_span < total_tiles ? t0 + tile_span : total_tiles;
    // image and first query of the tile, advanced without divisions
    int b = static_cast<int>(t0 / tiles_per_image);
    int qt0 = static_cast<int>(t0 - static_cast<long long>(b) * tiles_per_image) * 16;
    for (long long tile = t0; tile < t1; ++tile, qt0 += 16) {
        if (qt0 >= a.Q) {
            qt0 = 0;
            ++b;
        }
        const int nq = min(16, a.Q - qt0);
        // ---- the tile's entries: thread (q, k) = (tid / 8, tid % 8)
        const int eq = tid >> 3, ek = tid & 7;
        const bool qlive = eq < nq;
        const long long gq_e = static_cast<long long>(b) * a.Q + qt0 + eq;
        int t = -1;
        float v = INFINITY, z = 0.f;
        float2 u = make_float2(0.f, 0.f);
        if (qlive && ek < K) {
            const float2 qp = __ldg(reinterpret_cast<const float2*>(a.queries) + gq_e);
            const int cy = quantise(qp.y, a.GH), cx = quantise(qp.x, a.GW);
            t = __ldg(a.table + ((static_cast<size_t>(b) * a.GH + cy) * a.GW + cx) * K + ek);
            ACL_DEVICE_CHECK(t >= -1 && t < a.N);
            if (t >= a.N) t = -1;
            if (t >= 0) {
                const float2 p = __ldg(reinterpret_cast<const float2*>(a.xy) + static_cast<size_t>(b) * a.N + t);
                const float dx = qp.x - p.x, dy = qp.y - p.y;
                const float d = sqrtf(dx * dx + dy * dy);
                v = knn_v(d, a.kind);
                z = knn_dzdp(v);
                const float f = knn_dq_factor(d, a.kind);
                u = make_float2(dx * f, dy * f);
            }
        }
        float vmin = v;
        vmin = fminf(vmin, __shfl_xor_sync(0xffffffffu, vmin, 1));
        vmin = fminf(vmin, __shfl_xor_sync(0xffffffffu, vmin, 2));
        vmin = fminf(vmin, __shfl_xor_sync(0xffffffffu, vmin, 4));
        for (int i = tid; i < NW; i += kUTThreads) bits[i] = 0u;
        __syncthreads();
        if (t >= 0) atomicOr(&bits[t >> 5], 1u << (t & 31));
        __syncthreads();
        // exclusive prefix of the words' popcounts (warp 0; NW <= 64)
        if (warp == 0) {
            const int c0 = lane < NW ? __popc(bits[lane]) : 0;
            int s0 = c0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, s0, o);
                if (lane >= o) s0 += y;
            }
            const int tot0 = __shfl_sync(0xffffffffu, s0, 31);
            if (lane < NW) pre[lane] = s0 - c0;
            if (NW > 32) {
                const int c1 = lane + 32 < NW ? __popc(bits[lane + 32]) : 0;
                int s1 = c1;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int y = __shfl_up_sync(0xffffffffu, s1, o);
                    if (lane >= o) s1 += y;
                }
                if (lane + 32 < NW) pre[lane + 32] = tot0 + s1 - c1;
                if (lane == 31) pre[64] = tot0 + s1;
            } else if (lane == 0) {
                pre[64] = tot0;
            }
        }
        __syncthreads();
        const int U = pre[64];
        const int loc = t >= 0 ? pre[t >> 5] + __popc(bits[t >> 5] & ((1u << (t & 31)) - 1u)) : -1;
        if (t >= 0) utok[loc] = t;  // entries of one token write the same value
        qloc[tid] = loc;
        qe[tid] = t < 0 ? -INFINITY : (v == vmin ? 0.f : vmin - v);
        qz[tid] = z;
        qu[tid] = u;
        const int U8 = (U + 7) >> 3;  // n-tiles of 8 tokens
        __syncthreads();
        // this lane's pairs
        int lk[4];
        float le[4], lz[4];
        float2 lu[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int e = pq * 8 + pk0 + i;
            lk[i] = qloc[e];
            le[i] = qe[e];
            lz[i] = qz[e];
            lu[i] = qu[e];
        }
        float cq[4] = {0.f, 0.f, 0.f, 0.f};
        // rows of the lane's fragments: dO rows g and g + 8 of the tile (the tail repeats the
        // last query; those rows of dW are never read)
        const bf16* fimg = a.feats + static_cast<size_t>(b) * a.N * a.d + 8 * tq;
        const bf16* do0 = a.dout + (static_cast<size_t>(b) * a.Q + qt0 + min(g, nq - 1)) * a.d + 8 * tq;
        const bf16* do1 = a.dout + (static_cast<size_t>(b) * a.Q + qt0 + min(g + 8, nq - 1)) * a.d + 8 * tq;
        const long long gq0 = static_cast<long long>(b) * a.Q + qt0;
        // the fragments of a head: its dO rows and the first kUTBatch n-tiles of union rows
        // (rows past the union repeat its last row: those columns are never read); the next
        // head's are loaded while this one computes
        uint4 nq0 = make_uint4(0u, 0u, 0u, 0u), nq1 = nq0, nf[kUTBatch];
        auto fetch = [&](int hh) {
            nq0 = ldg16(do0 + hh * 32);
            nq1 = ldg16(do1 + hh * 32);
#pragma unroll
            for (int x = 0; x < kUTBatch; ++x)
                nf[x] = U8 > 0 ? ldg16(fimg + hh * 32 + static_cast<size_t>(utok[min(8 * x + g, U - 1)]) * a.d)
                               : make_uint4(0u, 0u, 0u, 0u);
        };
        if (warp < NH) fetch(warp);
        // warp w takes the heads h = w (mod 4)
        for (int h = warp; h < NH; h += kUTWarps) {
            {
                // dW_h = dO_h F_U,h^T into the warp's dW tile.  Lane (g, c) holds channels
                // 8c .. 8c + 7 of its rows as pairs e = 0..3; k-step s takes pairs 2s and 2s + 1
                // as its two k-halves, for dO and F alike, so the sum over channels is unchanged.
                const uint4 q0 = nq0, q1 = nq1;
                uint4 f[kUTBatch];
#pragma unroll
                for (int x = 0; x < kUTBatch; ++x) f[x] = nf[x];
                if (h + kUTWarps < NH) fetch(h + kUTWarps);
                const bf16* fh = fimg + h * 32;
                for (int n0 = 0; n0 < U8; n0 += kUTBatch) {
                    if (n0 > 0) {
#pragma unroll
                        for (int x = 0; x < kUTBatch; ++x) {
                            const int r = min(8 * (n0 + x) + g, U - 1);
                            f[x] = ldg16(fh + static_cast<size_t>(utok[r]) * a.d);
                        }
                    }
#pragma unroll
                    for (int x = 0; x < kUTBatch; ++x) {
                        const int nt = n0 + x;
                        if (nt >= U8) break;
                        float c[4] = {0.f, 0.f, 0.f, 0.f};
                        mma_bf16(c, q0.x, q1.x, q0.y, q1.y, f[x].x, f[x].y);
                        mma_bf16(c, q0.z, q1.z, q0.w, q1.w, f[x].z, f[x].w);
                        *reinterpret_cast<float2*>(dws + g * kUTDS + nt * 8 + 2 * tq) = make_float2(c[0], c[1]);
                        *reinterpret_cast<float2*>(dws + (g + 8) * kUTDS + nt * 8 + 2 * tq) = make_float2(c[2], c[3]);
                    }
                }
            }
            __syncwarp();
            // the per-query algebra of this head for the lane's four pairs
            const float ph = __ldg(a.p + h);
            float w[4], dw[4];
            float sum = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float y;
                asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(ph * le[i]));
                w[i] = lk[i] < 0 ? 0.f : (ph == 0.f ? 1.f : y);
                dw[i] = lk[i] < 0 ? 0.f : dws[pq * kUTDS + lk[i]];
                sum += w[i];
            }
            sum += __shfl_xor_sync(0xffffffffu, sum, 1);
            const float inv = sum > 0.f ? __fdividef(1.f, sum) : 0.f;
            float sdw = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                w[i] *= inv;
                sdw += w[i] * dw[i];
            }
            sdw += __shfl_xor_sync(0xffffffffu, sdw, 1);
            float dph = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float ds = w[i] * (dw[i] - sdw);
                dph -= w[i] > 0.f ? ds * lz[i] : 0.f;
                cq[i] -= ph * ds;
            }
            const int slot = (h - warp) >> 2;  // h = warp + 4 slot
#pragma unroll
            for (int s = 0; s < 8; ++s)
                if (s == slot) dpa[s] += dph;
#pragma unroll
            for (int i = 0; i < 4; ++i)
                if (pk0 + i < K) wblk[(pq * K + pk0 + i) * WS + h] = w[i];
            __syncwarp();
        }
        // dq: the lane's pairs, its partner lane, then the warps in order
        float dqx = 0.f, dqy = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            dqx += cq[i] * lu[i].x;
            dqy += cq[i] * lu[i].y;
        }
        dqx += __shfl_xor_sync(0xffffffffu, dqx, 1);
        dqy += __shfl_xor_sync(0xffffffffu, dqy, 1);
        if ((lane & 1) == 0) dqred[warp * 16 + pq] = make_float2(dqx, dqy);
        __syncthreads();
        // the tile's w block is contiguous in [q][slot][head]: float o of it sits at o + o / NH
        // in the padded rows; o advances by the CTA's width, its row and column without divisions
        {
            float* wout = a.w + static_cast<size_t>(gq0) * K * NH;
            const int n = nq * K * NH;
            int r = wr0, c = wc0;
            for (int o = tid; o < n; o += kUTThreads) {
                wout[o] = wblk[o + r];
                r += wdr;
                c += wdc;
                if (c >= NH) {
                    c -= NH;
                    ++r;
                }
            }
        }
        if (tid < nq) {
            float2 s = dqred[tid];
#pragma unroll
            for (int w2 = 1; w2 < kUTWarps; ++w2) {
                s.x += dqred[w2 * 16 + tid].x;
                s.y += dqred[w2 * 16 + tid].y;
            }
            reinterpret_cast<float2*>(a.dq)[gq0 + tid] = s;
        }
        __syncthreads();  // bits, lists and dq partials are rebuilt by the next tile
    }
    // dp: the lane partials of each of this warp's heads, summed over the warp in a fixed order
#pragma unroll
    for (int s = 0; s < 8; ++s) {
        const int h = warp + 4 * s;
        float x = dpa[s];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
        if (lane == 0 && h < NH) a.dp_part[static_cast<size_t>(blockIdx.x) * NH + h] = x;
    }
}

// Forward on the tensor cores, for the images the union query pass serves (at most kUTUseN
// tokens, K <= 8), over the same 16-query tiles and token unions.  Per head:
//   out (16 x 32) = W_h (16 x U) F_U,h (U x 32),
// W_h holding each query's normalised weights at the union positions of its tokens (slots
// that repeat a token add up in slot order), split into bf16 hi + lo (about 16 significant
// bits) and read by ldmatrix from a per-warp tile; m16n8k16 products accumulate in fp32.
// F_U,h never passes through shared memory: lane (g, c) loads 16 bytes, channels 8c .. 8c + 7,
// of union rows 16 s + g and 16 s + 8 + g, and movmatrix turns pair e of those registers
// into the B operand of column tile e, whose column n holds channel 8 (n / 2) + 2 e + n % 2.
// The accumulator of tile e then holds channels 8c + 2e, 8c + 2e + 1 of queries g and g + 8,
// so each lane stores 16 contiguous bytes per query.  Warp w takes heads w, w + 4, ...
constexpr int kUFDS = kUTMaxU + 8;  // row stride of a warp's W tiles (bf16; 272-byte rows)
constexpr int kUFBatch = 2;         // k-steps (16 union rows each) whose rows load together

struct UFSmem {
    size_t bits, pre, utok, qloc, qe, wt, total;
};
__host__ __device__ __forceinline__ UFSmem uf_smem_layout() {
    UFSmem L;
    size_t o = 0;
    auto take = [&](size_t bytes) {
        const size_t at = o;
        o = (o + bytes + 127) & ~size_t(127);
        return at;
    };
    L.bits = take(4 * (kUTMaxN / 32));
    L.pre = take(4 * (kUTMaxN / 32 + 1));
    L.utok = take(4 * kUTMaxU);
    L.qloc = take(4 * kUTMaxU);
    L.qe = take(4 * kUTMaxU);
    L.wt = take(2 * 2 * 16 * kUFDS * kUTWarps);  // hi and lo tiles per warp
    L.total = o;
    return L;
}

__global__ void __launch_bounds__(kUTThreads, 5)
    knn_fwd_union_kernel(const KnnArgs a, long long tiles_per_image, long long tile_span) {
    extern __shared__ __align__(128) uint8_t smem[];
    const UFSmem L = uf_smem_layout();
    uint32_t* bits = reinterpret_cast<uint32_t*>(smem + L.bits);
    int* pre = reinterpret_cast<int*>(smem + L.pre);
    int* utok = reinterpret_cast<int*>(smem + L.utok);
    int* qloc = reinterpret_cast<int*>(smem + L.qloc);
    float* qe = reinterpret_cast<float*>(smem + L.qe);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    bf16* wh = reinterpret_cast<bf16*>(smem + L.wt) + warp * 2 * 16 * kUFDS;
    bf16* wl = wh + 16 * kUFDS;
    const uint32_t wh0 = smem_addr(wh), wl0 = smem_addr(wl);
    const int NH = a.d >> 5, NW = (a.N + 31) >> 5;
    const int K = a.K;
    const int pq = lane >> 1, pk0 = 4 * (lane & 1);  // the lane's four (query, slot) pairs
    const int g = lane >> 2, tq = lane & 3;
    const uint32_t aoff = ((lane & 7) + ((lane >> 3) & 1) * 8) * (2 * kUFDS) + (lane >> 4) * 16;
    const long long total_tiles = static_cast<long long>(a.B) * tiles_per_image;
    const long long t0 = static_cast<long long>(blockIdx.x) * tile_span;
    const long long t1 = t0 + tile_span < total_tiles ? t0 + tile_span : total_tiles;
    // image and first query of the tile, advanced without divisions
    int b = static_cast<int>(t0 / tiles_per_image);
    int qt0 = static_cast<int>(t0 - static_cast<long long>(b) * tiles_per_image) * 16;
    for (long long tile = t0; tile < t1; ++tile, qt0 += 16) {
        if (qt0 >= a.Q) {
            qt0 = 0;
            ++b;
        }
        const int nq = min(16, a.Q - qt0);
        // ---- the tile's entries: thread (q, k) = (tid / 8, tid % 8)
        const int eq = tid >> 3, ek = tid & 7;
        const long long gq_e = static_cast<long long>(b) * a.Q + qt0 + eq;
        int t = -1;
        float v = INFINITY;
        if (eq < nq && ek < K) {
            const float2 qp = __ldg(reinterpret_cast<const float2*>(a.queries) + gq_e);
            const int cy = quantise(qp.y, a.GH), cx = quantise(qp.x, a.GW);
            t = __ldg(a.table + ((static_cast<size_t>(b) * a.GH + cy) * a.GW + cx) * K + ek);
            ACL_DEVICE_CHECK(t >= -1 && t < a.N);
            if (t >= a.N) t = -1;
            if (t >= 0) {
                const float2 p = __ldg(reinterpret_cast<const float2*>(a.xy) + static_cast<size_t>(b) * a.N + t);
                const float dx = qp.x - p.x, dy = qp.y - p.y;
                v = knn_v(sqrtf(dx * dx + dy * dy), a.kind);
            }
        }
        float vmin = v;
        vmin = fminf(vmin, __shfl_xor_sync(0xffffffffu, vmin, 1));
        vmin = fminf(vmin, __shfl_xor_sync(0xffffffffu, vmin, 2));
        vmin = fminf(vmin, __shfl_xor_sync(0xffffffffu, vmin, 4));
        // the entry is its token's first slot in the query's row unless an earlier slot holds
        // the token; a repeated token anywhere in the tile sends every warp down the summing path
        bool efirst = t >= 0, erep = false;
#pragma unroll
        for (int s = 1; s < 8; ++s) {
            const int ts = __shfl_sync(0xffffffffu, t, (lane & ~7) | ((lane + s) & 7));
            if (t >= 0 && ts == t) {
                erep = true;
                if (((lane + s) & 7) < ek) efirst = false;
            }
        }
        for (int i = tid; i < NW; i += kUTThreads) bits[i] = 0u;
        __syncthreads();
        if (t >= 0) atomicOr(&bits[t >> 5], 1u << (t & 31));
        __syncthreads();
        if (warp == 0) {  // exclusive prefix of the bitmap words' counts (NW <= 64)
            const int c0 = lane < NW ? __popc(bits[lane]) : 0;
            int s0 = c0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, s0, o);
                if (lane >= o) s0 += y;
            }
            const int tot0 = __shfl_sync(0xffffffffu, s0, 31);
            if (lane < NW) pre[lane] = s0 - c0;
            if (NW > 32) {
                const int c1 = lane + 32 < NW ? __popc(bits[lane + 32]) : 0;
                int s1 = c1;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int y = __shfl_up_sync(0xffffffffu, s1, o);
                    if (lane >= o) s1 += y;
                }
                if (lane + 32 < NW) pre[lane + 32] = tot0 + s1 - c1;
                if (lane == 31) pre[64] = tot0 + s1;
            } else if (lane == 0) {
                pre[64] = tot0;
            }
        }
        __syncthreads();
        const int U = pre[64];
        const int loc = t >= 0 ? pre[t >> 5] + __popc(bits[t >> 5] & ((1u << (t & 31)) - 1u)) : -1;
        if (t >= 0) utok[loc] = t;  // entries of one token write the same value
        qloc[tid] = efirst ? loc : (t >= 0 ? loc | 0x40000000 : -1);  // bit 30: a later slot
        qe[tid] = t < 0 ? -INFINITY : (v == vmin ? 0.f : vmin - v);
        const int nks = (U + 15) >> 4;  // k-steps of 16 union rows
        const bool dup = __syncthreads_or(erep) != 0;
        // the lane's slots: union position, whether it writes the token's summed weight, exponent
        int lk[4];
        bool first[4];
        float le[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = qloc[pq * 8 + pk0 + i];
            lk[i] = r < 0 ? -1 : (r & 0x3fffffff);
            first[i] = r >= 0 && !(r & 0x40000000);
            le[i] = qe[pq * 8 + pk0 + i];
        }
        // the warp's W tiles start at zero; every head of the tile writes the same positions,
        // so one clearing per tile suffices
        {
            bf16* zt = ((lane >> 4) ? wl : wh) + (lane & 15) * kUFDS;
            for (int c = 0; c < 2 * nks; ++c) *reinterpret_cast<uint4*>(zt + c * 8) = make_uint4(0u, 0u, 0u, 0u);
        }
        __syncwarp();
        const bf16* fimg = a.feats + static_cast<size_t>(b) * a.N * a.d + 8 * tq;
        bf16* oq = a.out + (static_cast<size_t>(b) * a.Q + qt0 + g) * a.d + 8 * tq;
        for (int h = warp; h < NH; h += kUTWarps) {
            const bf16* fh = fimg + h * 32;
            // the first k-steps' rows load while the weights form (rows past the union repeat
            // its last row: their W columns are zero)
            uint4 f0[kUFBatch], f1[kUFBatch];
            if (nks > 0) {
#pragma unroll
                for (int s = 0; s < kUFBatch; ++s) {
                    const int r0 = min(16 * s + g, U - 1), r1 = min(16 * s + 8 + g, U - 1);
                    f0[s] = ldg16(fh + static_cast<size_t>(utok[r0]) * a.d);
                    f1[s] = ldg16(fh + static_cast<size_t>(utok[r1]) * a.d);
                }
            }
            const float ph = __ldg(a.p + h);
            float w[4];
            float sum = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float y;
                asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(ph * le[i]));
                w[i] = lk[i] < 0 ? 0.f : (ph == 0.f ? 1.f : y);
                sum += w[i];
            }
            sum += __shfl_xor_sync(0xffffffffu, sum, 1);
            const float inv = sum > 0.f ? __fdividef(1.f, sum) : 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) w[i] *= inv;
            float x[4] = {w[0], w[1], w[2], w[3]};
            if (dup) {  // CTA-uniform: some query of the tile repeats a token
                float pw[4];
                int ok[4];  // the partner lane's slots: the query's other four
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    pw[i] = __shfl_xor_sync(0xffffffffu, w[i], 1);
                    ok[i] = __shfl_xor_sync(0xffffffffu, lk[i], 1);
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float s = 0.f;
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const bool mine = (lane & 1) ? (q >= 4) : (q < 4);
                        const int lq = mine ? lk[q & 3] : ok[q & 3];
                        if (lq == lk[i]) s += mine ? w[q & 3] : pw[q & 3];
                    }
                    x[i] = s;
                }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                if (!first[i]) continue;
                const bf16 hi = __float2bfloat16_rn(x[i]);
                wh[pq * kUFDS + lk[i]] = hi;
                wl[pq * kUFDS + lk[i]] = __float2bfloat16_rn(x[i] - __bfloat162float(hi));
            }
            __syncwarp();
            float acc[4][4];
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[e][0] = acc[e][1] = acc[e][2] = acc[e][3] = 0.f;
            for (int s0 = 0; s0 < nks; s0 += kUFBatch) {
                if (s0 > 0) {
#pragma unroll
                    for (int s = 0; s < kUFBatch; ++s) {
                        const int r0 = min(16 * (s0 + s) + g, U - 1), r1 = min(16 * (s0 + s) + 8 + g, U - 1);
                        f0[s] = ldg16(fh + static_cast<size_t>(utok[r0]) * a.d);
                        f1[s] = ldg16(fh + static_cast<size_t>(utok[r1]) * a.d);
                    }
                }
#pragma unroll
                for (int s = 0; s < kUFBatch; ++s) {
                    if (s0 + s >= nks) break;
                    uint32_t ah[4], al[4];
                    ldsm_x4(wh0 + aoff + (s0 + s) * 32, ah[0], ah[1], ah[2], ah[3]);
                    ldsm_x4(wl0 + aoff + (s0 + s) * 32, al[0], al[1], al[2], al[3]);
                    const uint32_t p0[4] = {f0[s].x, f0[s].y, f0[s].z, f0[s].w};
                    const uint32_t p1[4] = {f1[s].x, f1[s].y, f1[s].z, f1[s].w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const uint32_t b0 = movm_t(p0[e]), b1 = movm_t(p1[e]);
                        mma_bf16(acc[e], ah[0], ah[1], ah[2], ah[3], b0, b1);
                        mma_bf16(acc[e], al[0], al[1], al[2], al[3], b0, b1);
                    }
                }
            }
            if (g < nq)
                *reinterpret_cast<uint4*>(oq + h * 32) =
                    make_uint4(pack_bf16(acc[0][0], acc[0][1]), pack_bf16(acc[1][0], acc[1][1]),
                               pack_bf16(acc[2][0], acc[2][1]), pack_bf16(acc[3][0], acc[3][1]));
            if (g + 8 < nq)
                *reinterpret_cast<uint4*>(oq + static_cast<size_t>(8) * a.d + h * 32) =
                    make_uint4(pack_bf16(acc[0][2], acc[0][3]), pack_bf16(acc[1][2], acc[1][3]),
                               pack_bf16(acc[2][2], acc[2][3]), pack_bf16(acc[3][2], acc[3][3]));
            __syncwarp();  // the next head rewrites the W tiles
        }
        __syncthreads();  // utok, qloc and qe are rebuilt by the next tile
    }
}

// Stable counting sort of an image's (query, slot) entries by token id, integer only,
// spread over `slices` CTAs per image: CTA (slice, b) owns the tokens [t_lo, t_hi).
//   compaction: warp w scans the contiguous entry chunk [lo_w, hi_w) of the image twice
//     (16 keys per lane in flight): first it counts the slice's entries and the entries
//     whose token lies below t_lo, then, after a prefix over the warps' counts, it writes
//     the slice's entries in entry order into one shared-memory list (ballot + popc).
//     Queries come in raster order and tokens are numbered spatially, so a chunk's
//     entries cluster in one or two slices; the one list keeps the work per warp equal;
//   counts and prefix: warp w takes the w-th equal, contiguous share of the list; per-
//     (warp, token) counts of the shares; each warp's first slot per token is (entries of
//     smaller tokens) + (entries of this token in earlier shares);
//   placement: each listed entry goes to its warp's next slot for its token plus its rank
//     among equal tokens in its group of 32 (lanes OR their bit into a per-warp hashed
//     mask -- OR commutes, so the mask does not depend on timing).
//   A slice with more than kCsrListCap entries counts and places straight from the keys,
//     warp w over its own chunk.
// The list of a token ends up in ascending entry order; entries are stored packed as
// (query << 4) | slot.  Each CTA also lists its slice's tokens with more than
// kHeavyEntries entries (ascending) and writes the chunk starts of the token pass.
constexpr int kCsrSteps = 16;
constexpr int kCsrHash = 256;
constexpr int kCsrWarps = kCsrThreads / 32;
constexpr int kCsrListCap = 12288;  // entries of a slice listed in shared memory
constexpr int kHeavyEntries = 96;  // tokens with more entries are reduced by a whole CTA
constexpr int kChunkUnits = 64;   // work units (1 per token + 1 per entry) per light chunk
constexpr int kChunkIds = 192;    // staged ids per warp (>= kChunkUnits + kHeavyEntries)
constexpr int kHeavyCtas = 128;   // CTAs of the token pass that take the heavy tokens (default)
static_assert(kChunkUnits <= kHeavyEntries + 1, "a chunk's tokens other than its last must be light");
static_assert(kChunkIds >= kChunkUnits + kHeavyEntries, "a chunk's light entries must fit the staging");

struct CsrSmem {
    size_t pre, off, hash, lanes, ckey, cent, scratch, total;
};
__host__ __device__ __forceinline__ CsrSmem csr_smem_layout(int NS) {
    CsrSmem L;
    L.pre = 0;
    L.off = (4 * kCsrWarps * static_cast<size_t>(NS) + 15) & ~size_t(15);
    L.hash = L.off + ((4 * static_cast<size_t>(NS + 1) + 15) & ~size_t(15));
    L.lanes = L.hash + 4 * static_cast<size_t>(kCsrHash) * kCsrWarps;
    L.ckey = L.lanes + 4 * 32 * static_cast<size_t>(kCsrWarps);
    L.cent = L.ckey + 2 * static_cast<size_t>(kCsrListCap);
    L.scratch = L.cent + 4 * static_cast<size_t>(kCsrListCap);
    L.total = L.scratch + 80 * 4;
    return L;
}

// Token of every (query, slot) entry: the slot of the query's table row (-1 for an empty
// slot).  One thread per query; keys [B][Q * K].
__global__ void __launch_bounds__(256) knn_keys_kernel(const KnnArgs a) {
    const long long gq = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (gq >= static_cast<long long>(a.B) * a.Q) return;
    const int b = static_cast<int>(gq / a.Q);
    const float2 qp = reinterpret_cast<const float2*>(a.queries)[gq];
    const int cy = quantise(qp.y, a.GH), cx = quantise(qp.x, a.GW);
    const int32_t* row = a.table + ((static_cast<size_t>(b) * a.GH + cy) * a.GW + cx) * a.K;
    int32_t* out = a.keys + gq * a.K;
    for (int j = 0; j < a.K; ++j) {
        const int t = __ldg(row + j);
        ACL_DEVICE_CHECK(t >= -1 && t < a.N);
        out[j] = (t >= a.N) ? -1 : t;
    }
}

__global__ void __launch_bounds__(kCsrThreads)
    knn_csr_kernel(const KnnArgs a, int slices, int chunks) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int b = blockIdx.y, sl = blockIdx.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int N = a.N, K = a.K;
    const int t_lo = static_cast<int>(static_cast<long long>(sl) * N / slices);
    const int t_hi = static_cast<int>(static_cast<long long>(sl + 1) * N / slices);
    const int NS = t_hi - t_lo;
    const int NS2 = NS;
    const CsrSmem L = csr_smem_layout((N + slices - 1) / slices);
    // per (warp, token) entry counts, then prefixes: 32-bit, since a token repeated within
    // table rows can collect up to Q K entries
    uint32_t* pre = reinterpret_cast<uint32_t*>(smem + L.pre);  // [warps][NS]
    int* off = reinterpret_cast<int*>(smem + L.off);
    uint32_t* hb = reinterpret_cast<uint32_t*>(smem + L.hash) + warp * kCsrHash;
    int* ks = reinterpret_cast<int*>(smem + L.lanes) + warp * 32;
    uint16_t* ckey = reinterpret_cast<uint16_t*>(smem + L.ckey);  // [kCsrListCap] key - t_lo
    int* cent = reinterpret_cast<int*>(smem + L.cent);              // [kCsrListCap] entry
    int* scratch = reinterpret_cast<int*>(smem + L.scratch);        // [40] scan, [40..72) counts
    const int E = a.Q * K;
    const int32_t* keys = a.keys + static_cast<size_t>(b) * E;
    int32_t* csr = a.csr + static_cast<size_t>(b) * E;
    for (int i = tid; i < kCsrWarps * NS2; i += kCsrThreads) pre[i] = 0;
    for (int i = lane; i < kCsrHash; i += 32) hb[i] = 0u;
    const int lo = static_cast<int>(static_cast<long long>(warp) * E / kCsrWarps);
    const int hi = static_cast<int>(static_cast<long long>(warp + 1) * E / kCsrWarps);
    uint32_t* mine = pre + warp * NS2;
    const unsigned below_lanes = (1u << lane) - 1u;
    // pass 1: per warp, the entries of the slice and the entries below it
    int cnt = 0, below = 0;
    for (int base = lo; base < hi; base += 32 * kCsrSteps) {
        int k[kCsrSteps];
#pragma unroll
        for (int st = 0; st < kCsrSteps; ++st) {
            const int e = base + st * 32 + lane;
            k[st] = (e < hi) ? __ldg(keys + e) : -1;
        }
#pragma unroll
        for (int st = 0; st < kCsrSteps; ++st) {
            const int key = k[st];
            below += (key >= 0 && key < t_lo);
            cnt += __popc(__ballot_sync(0xffffffffu, key >= t_lo && key < t_hi));
        }
    }
    below = __reduce_add_sync(0xffffffffu, below);
    if (lane == 0) {
        scratch[warp] = below;
        scratch[40 + warp] = cnt;
    }
    __syncthreads();  // also: pre / hash zeroed by all threads before any count
    int wbase = 0, n = 0, base_slot = 0;
    for (int w = 0; w < kCsrWarps; ++w) {
        const int c = scratch[40 + w];
        wbase += (w < warp) ? c : 0;
        n += c;
        base_slot += scratch[w];
    }
    // pass 2: the slice's entries, in entry order, into one list (warps in order); each
    // warp then takes an equal, contiguous share of the list
    const bool listed = n <= kCsrListCap;
    if (listed) {
        int pos = wbase;
        for (int base = lo; base < hi; base += 32 * kCsrSteps) {
            int k[kCsrSteps];
#pragma unroll
            for (int st = 0; st < kCsrSteps; ++st) {
                const int e = base + st * 32 + lane;
                k[st] = (e < hi) ? __ldg(keys + e) : -1;
            }
#pragma unroll
            for (int st = 0; st < kCsrSteps; ++st) {
                const int key = k[st];
                const bool in = key >= t_lo && key < t_hi;
                const unsigned m = __ballot_sync(0xffffffffu, in);
                if (in) {
                    const int p = pos + __popc(m & below_lanes);
                    ckey[p] = static_cast<uint16_t>(key - t_lo);
                    cent[p] = base + st * 32 + lane;
                }
                pos += __popc(m);
            }
        }
    }
    __syncthreads();
    const int l0 = static_cast<int>(static_cast<long long>(warp) * n / kCsrWarps);
    const int l1 = static_cast<int>(static_cast<long long>(warp + 1) * n / kCsrWarps);
    if (listed) {
        for (int i = l0 + lane; i < l1; i += 32) {
            atomicAdd(pre + warp * NS2 + ckey[i], 1u);
        }
    } else {
        for (int base = lo; base < hi; base += 32) {
            const int e = base + lane;
            const int key = (e < hi) ? __ldg(keys + e) : -1;
            if (key >= t_lo && key < t_hi) {
                atomicAdd(pre + warp * NS2 + (key - t_lo), 1u);
            }
        }
    }
    __syncthreads();
    for (int t = tid; t < NS; t += kCsrThreads) {
        int run = 0;
        for (int w = 0; w < kCsrWarps; ++w) {
            const int c = static_cast<int>(pre[w * NS2 + t]);
            pre[w * NS2 + t] = static_cast<uint32_t>(run);
            run += c;
        }
        off[t] = run;
    }
    __syncthreads();
    const int tot = block_scan(off, NS, scratch);
    int32_t* coff = a.csr_off + static_cast<size_t>(b) * (N + 1);
    // tokens with many entries go to this slice's heavy list (token order), for the
    // token kernel's CTA-wide path
    if (warp == 0) {
        int nh = 0;
        int32_t* hl = a.heavy + (static_cast<size_t>(b) * slices + sl) * a.heavy_cap;
        for (int t0 = 0; t0 < NS; t0 += 32) {
            const int t = t0 + lane;
            const int cnt = (t < NS) ? ((t + 1 < NS ? off[t + 1] : tot) - off[t]) : 0;
            const bool hv = cnt > kHeavyEntries;
            const unsigned m = __ballot_sync(0xffffffffu, hv);
            if (hv) hl[nh + __popc(m & below_lanes)] = t_lo + t;
            nh += __popc(m);
        }
        if (lane == 0) a.heavy_count[static_cast<size_t>(b) * slices + sl] = nh;
    }
    __syncthreads();
    for (int t = tid; t < NS; t += kCsrThreads) {
        off[t] += base_slot;
        coff[t_lo + t] = off[t];
    }
    if (tid == 0 && sl == slices - 1) coff[N] = base_slot + tot;
    __syncthreads();
    // chunk starts of the token pass: chunk c begins at the first token t whose unit offset
    // start(t) + t reaches c * kChunkUnits (the boundaries inside (start(t) + t, start(t + 1)
    // + t + 1] belong to token t + 1); chunk_off[c] = start of that token
    int32_t* ctok = a.chunk_tok + static_cast<size_t>(b) * (chunks + 1);
    int32_t* cofs = a.chunk_off + static_cast<size_t>(b) * (chunks + 1);
    for (int t = tid; t < NS; t += kCsrThreads) {
        const int e1 = t + 1 < NS ? off[t + 1] : base_slot + tot;  // first entry of token t + 1
        const int s0 = off[t] + t_lo + t;
        const int s1 = e1 + t_lo + t + 1;
        for (int c = s0 / kChunkUnits + 1; c <= s1 / kChunkUnits; ++c) {
            ctok[c] = t_lo + t + 1;
            cofs[c] = e1;
        }
    }
    if (sl == 0 && tid == 0) {
        ctok[0] = 0;
        cofs[0] = 0;
    }
    if (sl == slices - 1)
        for (int c = (base_slot + tot + N) / kChunkUnits + 1 + tid; c <= chunks; c += kCsrThreads) {
            ctok[c] = N;
            cofs[c] = base_slot + tot;
        }
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
            before = static_cast<int>(mine[kk]);
            const int q = e / K, j = e - q * K;
            csr[off[kk] + before + __popc(peers & below_lanes)] = (q << 4) | j;
        }
        __syncwarp();
        if (in && lane == __ffs(peers) - 1) {
            mine[kk] = static_cast<uint32_t>(before + __popc(peers));
            hb[h] = 0u;
        }
        __syncwarp();
    };
    if (listed) {
        for (int i0 = l0; i0 < l1; i0 += 32) {
            const int i = i0 + lane;
            const bool in = i < l1;
            place(in, in ? ckey[i] : -1, in ? cent[i] : 0);
        }
    } else {
        for (int base = lo; base < hi; base += 32) {
            const int e = base + lane;
            const int key = (e < hi) ? __ldg(keys + e) : -1;
            const bool in = key >= t_lo && key < t_hi;
            if (__ballot_sync(0xffffffffu, in) == 0u) continue;
            place(in, in ? key - t_lo : -1, e);
        }
    }
}

// Token side of the gather backward.  dF_t = sum of w * dOut over the token's entries, with
// no atomics and a static, balanced split of the work:
//   light tokens (at most kHeavyEntries entries): the CSR build cuts each image's token
//     sequence into chunks of kChunkUnits "units" (a token weighs 1 + its entry count), so
//     every chunk holds about the same work, and lists for every chunk the first token that
//     starts in it.  One lane group per chunk stages the entry ids of its tokens in shared
//     memory (one round of independent loads), then walks them with the next batch's w and
//     dOut loads in flight, summing each token's entries in ascending order;
//   heavy tokens (listed per CSR slice): the first hctas CTAs (heavy_ctas) take them in a fixed
//     stride; all 8 warps x (32 / LPQ) lane groups stream every S-th entry, combined by a
//     fixed shuffle tree and a fixed-order pass over warps.
// Every token's sum is formed the same way on every run: bit-reproducible.  The first NH
// CTAs also reduce dp in a fixed order.
template <int CH>
__device__ __forceinline__ void token_streams(const KnnArgs& a, int b, int lo, int hi, int sid,
                                             int nstreams, int sub, int LPQ, int ch,
                                             uint64_t (&acc)[4]) {
    const int NH = a.d >> 5;
    const int KN = a.K * NH;
    const int c0 = ch * LPQ * 8 + sub * 8;
    const bool on = c0 < a.d;
    const int hh = on ? (c0 >> 5) : 0;
    const size_t qbase = static_cast<size_t>(b) * a.Q;
    const float* wb = a.w + qbase * KN + hh;
    const bf16* gb = a.dout + qbase * a.d + (on ? c0 : 0);
    const int32_t* csr = a.csr + static_cast<size_t>(b) * a.Q * a.K;
#pragma unroll
    for (int v = 0; v < 4; ++v) acc[v] = 0ull;
    // this stream's entries are lo + sid + nstreams * k; lanes of the group hold LPQ of them
    const int n = (hi - lo - sid + nstreams - 1) / nstreams;  // entries of this stream (>= 0)
    const unsigned gmask = (LPQ == 32) ? 0xffffffffu : (((1u << LPQ) - 1u) << (threadIdx.x & 31 & ~(LPQ - 1)));
    for (int k0 = 0; k0 < n; k0 += LPQ) {
        const int kk = k0 + sub;
        const int mine = (kk < n) ? __ldg(csr + lo + sid + nstreams * kk) : 0;
        const int cnt = min(LPQ, n - k0);
        int u = 0;
        for (; u + 4 <= cnt; u += 4) {
            float wv[4];
            uint4 gv[4];
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                const int e = __shfl_sync(gmask, mine, u + x, LPQ);
                const int q = e >> 4, j = e & 15;
                wv[x] = __ldg(wb + q * KN + j * NH);
                gv[x] = on ? ldg16(gb + q * a.d) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int x = 0; x < 4; ++x) row_fma(acc, f2_pack(wv[x], wv[x]), gv[x]);
        }
        for (; u < cnt; ++u) {
            const int e = __shfl_sync(gmask, mine, u, LPQ);
            const int q = e >> 4, j = e & 15;
            const float wv = __ldg(wb + q * KN + j * NH);
            row_fma(acc, f2_pack(wv, wv), on ? ldg16(gb + q * a.d) : make_uint4(0u, 0u, 0u, 0u));
        }
    }
}

// One heavy token by the whole CTA (all threads call).
__device__ void heavy_token(const KnnArgs& a, int b, int t, int l2, float (*part)[256]) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int LPQ = 1 << l2, S = 32 >> l2;
    const int sub = lane & (LPQ - 1), grp = lane >> l2;
    const int CH = (a.d + 8 * LPQ - 1) / (8 * LPQ);
    const int32_t* coff = a.csr_off + static_cast<size_t>(b) * (a.N + 1);
    const int lo = coff[t], hi = coff[t + 1];
    for (int ch = 0; ch < CH; ++ch) {
        uint64_t acc2[4];
        token_streams<1>(a, b, lo, hi, warp * S + grp, kGatherWarps * S, sub, LPQ, ch, acc2);
        float acc[8];
        unpack_acc(acc2, acc);
        for (int o = LPQ; o < 32; o <<= 1) {
#pragma unroll
            for (int v = 0; v < 8; ++v) acc[v] += __shfl_xor_sync(0xffffffffu, acc[v], o);
        }
        if (grp == 0) {
#pragma unroll
            for (int v = 0; v < 8; ++v) part[warp][sub * 8 + v] = acc[v];
        }
        __syncthreads();
        const int c0 = ch * LPQ * 8 + threadIdx.x * 8;
        if (threadIdx.x < LPQ && c0 < a.d) {
            float tot[8];
#pragma unroll
            for (int v = 0; v < 8; ++v) {
                float x = 0.f;
                for (int w = 0; w < kGatherWarps; ++w) x += part[w][threadIdx.x * 8 + v];
                tot[v] = x;
            }
            *reinterpret_cast<uint4*>(a.dfeats + (static_cast<size_t>(b) * a.N + t) * a.d + c0) =
                pack8(tot, 1.f);
        }
        __syncthreads();
    }
}

__global__ void __launch_bounds__(kGatherThreads, 4)
    knn_bwd_token_kernel(const KnnArgs a, int lpq_log2, int query_blocks, int nlists, int chunks,
                         int hctas) {
    constexpr int STEPS = 4;  // warp steps whose loads are in flight together
    __shared__ float part[kGatherWarps][256];
    __shared__ int hpre[kGatherThreads];
    __shared__ int scan_scratch[kGatherWarps + 1];
    __shared__ int ids_smem[kGatherWarps][kChunkIds];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int NH = a.d >> 5;
    if (static_cast<int>(blockIdx.x) < hctas) {
        const int h = blockIdx.x;
        if (h < NH) {
            float acc = 0.f;
            for (int i = threadIdx.x; i < query_blocks; i += kGatherThreads)
                acc += a.dp_part[static_cast<size_t>(i) * NH + h];
            acc = warp_sum(acc);
            if (lane == 0) part[warp][0] = acc;
            __syncthreads();
            if (threadIdx.x == 0) {
                float tot = 0.f;
                for (int w = 0; w < kGatherWarps; ++w) tot += part[w][0];
                a.dp[h] = tot;
            }
            __syncthreads();
        }
        // heavy items h, h + hctas, ... of the concatenated per-(image, slice) lists,
        // scanned kGatherThreads lists at a time
        const int slices = nlists / a.B;
        int run = 0;
        for (int l0 = 0; l0 < nlists; l0 += kGatherThreads) {
            const int nl = min(kGatherThreads, nlists - l0);
            hpre[threadIdx.x] = (static_cast<int>(threadIdx.x) < nl) ? a.heavy_count[l0 + threadIdx.x] : 0;
            __syncthreads();
            const int tot = block_scan(hpre, kGatherThreads, scan_scratch);  // hpre: exclusive
            int i = run + ((h - run % hctas) + hctas) % hctas;  // first i >= run, i = h mod hctas
            for (; i < run + tot; i += hctas) {
                const int r = i - run;
                int li = 0, hl = nl - 1;  // last list whose prefix is <= r
                while (li < hl) {
                    const int mid = (li + hl + 1) >> 1;
                    if (hpre[mid] <= r) li = mid; else hl = mid - 1;
                }
                const int lg = l0 + li;
                const int t = a.heavy[static_cast<size_t>(lg) * a.heavy_cap + (r - hpre[li])];
                heavy_token(a, lg / slices, t, lpq_log2, part);
            }
            run += tot;
            __syncthreads();
        }
        return;
    }
    // light tokens: warp gid owns chunk gid (image b, chunk c) and takes its tokens in order.
    // A token's entries are dealt round robin to the warp's EPS = 32 / LPQ slots (slot =
    // lane / LPQ; the lanes of a slot hold 8 channels each), STEPS entries per slot are
    // loaded together, and the slots are combined by a fixed xor tree at the token's end.
    const int LPQ = 1 << lpq_log2, EPS = 32 >> lpq_log2;
    const int slot = lane >> lpq_log2, sub = lane & (LPQ - 1);
    const int gid = (static_cast<int>(blockIdx.x) - hctas) * kGatherWarps + warp;
    const int b = gid / chunks;
    if (b >= a.B) return;  // whole warps leave together
    const int c = gid - b * chunks;
    int* ids = ids_smem[warp];
    const int32_t* ctok = a.chunk_tok + static_cast<size_t>(b) * (chunks + 1);
    const int32_t* coff = a.csr_off + static_cast<size_t>(b) * (a.N + 1);
    const int32_t* csr = a.csr + static_cast<size_t>(b) * a.Q * a.K;
    const int ta = ctok[c], tb = ctok[c + 1];
    const int* cofs = a.chunk_off + static_cast<size_t>(b) * (chunks + 1);
    const int C0 = cofs[c];
    const int KN = a.K * NH;
    const size_t qbase = static_cast<size_t>(b) * a.Q;
    bf16* dfb = a.dfeats + static_cast<size_t>(b) * a.N * a.d;
    const int passes = (a.d + 8 * LPQ - 1) / (8 * LPQ);
    {
        // the chunk's light entries all lie in its first kChunkUnits + kHeavyEntries entries
        const int nst = min(cofs[c + 1] - C0, kChunkIds);
        int v[kChunkIds / 32];
#pragma unroll
        for (int x = 0; x < kChunkIds / 32; ++x) {
            const int i = x * 32 + lane;
            v[x] = (i < nst) ? __ldg(csr + C0 + i) : 0;
        }
#pragma unroll
        for (int x = 0; x < kChunkIds / 32; ++x) {
            const int i = x * 32 + lane;
            if (i < nst) ids[i] = v[x];
        }
    }
    __syncwarp();
    for (int t0 = ta; t0 < tb; t0 += 31) {
        const int nt = min(31, tb - t0);
        const int offv = (lane <= nt) ? coff[t0 + lane] - C0 : 0;  // relative to the chunk
        // only the chunk's last token can be heavy; it is left to the heavy CTAs
        const int last_cnt = __shfl_sync(0xffffffffu, offv, nt) - __shfl_sync(0xffffffffu, offv, nt - 1);
        const int nl = (t0 + nt == tb && last_cnt > kHeavyEntries) ? nt - 1 : nt;
#pragma unroll 1
        for (int ps = 0; ps < passes; ++ps) {
            const int c0 = ps * LPQ * 8 + sub * 8;
            const bool on = c0 < a.d;
            const int hh = on ? (c0 >> 5) : 0;
            const float* wb = a.w + qbase * KN + hh;
            const bf16* gb = a.dout + qbase * a.d + (on ? c0 : 0);
            int lo = __shfl_sync(0xffffffffu, offv, 0);
            for (int k = 0; k < nl; ++k) {
                const int hi = __shfl_sync(0xffffffffu, offv, k + 1);
                uint64_t acc2[4] = {0ull, 0ull, 0ull, 0ull};
                for (int i0 = lo; i0 < hi; i0 += STEPS * EPS) {
                    float w[STEPS];
                    uint4 g[STEPS];
#pragma unroll
                    for (int x = 0; x < STEPS; ++x) {
                        const int i = i0 + x * EPS + slot;
                        w[x] = 0.f;
                        g[x] = make_uint4(0u, 0u, 0u, 0u);
                        if (i < hi) {
                            const int e = ids[i];
                            const int q = e >> 4, sl = e & 15;
                            w[x] = __ldg(wb + q * KN + sl * NH);
                            if (on) g[x] = ldg16(gb + static_cast<size_t>(q) * a.d);
                        }
                    }
#pragma unroll
                    for (int x = 0; x < STEPS; ++x) row_fma(acc2, f2_pack(w[x], w[x]), g[x]);
                }
                float acc[8];
                unpack_acc(acc2, acc);
                for (int o = LPQ; o < 32; o <<= 1) {
#pragma unroll
                    for (int v = 0; v < 8; ++v) acc[v] += __shfl_xor_sync(0xffffffffu, acc[v], o);
                }
                if (on && slot == 0)
                    *reinterpret_cast<uint4*>(dfb + static_cast<size_t>(t0 + k) * a.d + c0) = pack8(acc, 1.f);
                lo = hi;
            }
        }
        __syncwarp();
    }
}

// CTAs of the token pass that take the heavy tokens: kHeavyCtas when a token has few entries
// on average (heavy tokens are rare), four per SM when it has more than half the heavy
// threshold (most tokens heavy, e.g. a coarse stage gathered by many queries).  Every heavy
// token is summed by one CTA in the same order whatever this count.
int heavy_ctas(int Q, int K, int N) {
    const double mean = static_cast<double>(Q) * K / (N > 0 ? N : 1);
    return mean > 0.5 * kHeavyEntries ? 4 * 148 : kHeavyCtas;
}

// light chunks of the token pass per image: (Q*K entries + N tokens) / kChunkUnits + 1
int knn_chunks(int Q, int K, int N) {
    return static_cast<int>((static_cast<long long>(Q) * K + N) / kChunkUnits) + 1;
}

// token slices of the CSR build per image (B * slices <= 148 CTAs, at most 16)
// tokens per CSR slice at most, so that the build's shared memory (32-bit counts per warp
// and token) fits
constexpr int kCsrMaxSlice = 768;
int csr_slices(int B, int N) {
    int slices = 148 / (B > 0 ? B : 1);
    if (slices > 16) slices = 16;
    if (slices < 1) slices = 1;
    if (slices > (N + 31) / 32) slices = (N + 31) / 32;
    if (slices < 1) slices = 1;
    const int need = (N + kCsrMaxSlice - 1) / kCsrMaxSlice;
    return slices < need ? need : slices;
}

// lanes per query: d/8 rounded up to a power of two, capped at 32
int lpq_log2_for(int d) {
    int lanes = d / 8;
    int l2 = 0;
    while ((1 << l2) < lanes && l2 < 5) ++l2;
    return l2;
}

// Launch shape of the query-side gather kernels (the backward's also sizes the workspace).
struct GatherPlan {
    int l2, ch, iters, blocks;
    bool shared;  // lane j of a query group owns neighbour j (needs K <= lanes per query)
};
// Launch shape of the query-side gather kernels.  A CTA walks `iters` consecutive blocks of
// queries; iters is chosen so the grid fits one wave of the kernel's resident CTAs (4 per
// SM; 2 for the backward's query pass with K > 8 or more than one channel pass, which
// needs up to 128 registers).
GatherPlan gather_plan(int B, int Q, int d, int K, bool bwd) {
    GatherPlan g;
    g.l2 = lpq_log2_for(d);
    const int lanes = 1 << g.l2;
    g.ch = (d + 8 * lanes - 1) / (8 * lanes);
    g.shared = K <= lanes;
    const long long per_iter = static_cast<long long>(kGatherWarps) * (32 >> g.l2);
    const long long total = static_cast<long long>(B) * Q;
    const int resident = bwd ? ((K <= 8 && g.ch == 1) ? 4 : 2) : 4;
    long long it = 1;
    if (g.shared) {
        it = (total + per_iter * 148 * resident - 1) / (per_iter * 148 * resident);
        it = it < 1 ? 1 : (it > 8 ? 8 : it);
    }
    g.iters = static_cast<int>(it);
    g.blocks = static_cast<int>((total + per_iter * g.iters - 1) / (per_iter * g.iters));
    return g;
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

// The forward's persistent grid: at most one wave of resident CTAs, each taking a span of
// consecutive queries (a multiple of the queries one pass of its warps takes).
template <int KT, int CH>
cudaError_t fwd_launch(const KnnArgs& a, cudaStream_t st, int l2) {
    const long long total = static_cast<long long>(a.B) * a.Q;
    const long long per_pass = static_cast<long long>(kGatherWarps) * (32 >> l2);
    const long long passes = (total + per_pass - 1) / per_pass;
    const long long slots = static_cast<long long>(sm_count()) * resident<knn_fwd_kernel<KT, CH>>(kGatherThreads, 0);
    const long long blocks0 = passes < slots ? passes : slots;
    const long long span = (passes + blocks0 - 1) / blocks0 * per_pass;
    const unsigned blocks = static_cast<unsigned>((total + span - 1) / span);
    knn_fwd_kernel<KT, CH><<<blocks, kGatherThreads, 0, st>>>(a, l2, span);
    return cudaGetLastError();
}

template <int KT>
cudaError_t fwd_k(const KnnArgs& a, cudaStream_t st, int l2, int ch) {
    switch (ch) {
        case 1: return fwd_launch<KT, 1>(a, st, l2);
        case 2: return fwd_launch<KT, 2>(a, st, l2);
        case 3: return fwd_launch<KT, 3>(a, st, l2);
        default: return fwd_launch<KT, 4>(a, st, l2);
    }
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
    const int tiles = ((GW + 3) / 4) * ((GH + 1) / 2);
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
    w.query_blocks = gather_plan(B, Q, d, K, true).blocks;
    size_t off = 0;
    w.w = off;       off += up(sizeof(float) * BQ * NH * K);
    w.keys = off;    off += up(sizeof(int32_t) * BQ * K);
    w.csr = off;     off += up(sizeof(int32_t) * BQ * K);
    w.csr_off = off; off += up(sizeof(int32_t) * static_cast<size_t>(B) * (N + 1));
    w.dp_part = off; off += up(sizeof(float) * static_cast<size_t>(w.query_blocks) * NH);
    w.chunk_tok = off;
    off += up(sizeof(int32_t) * static_cast<size_t>(B) * (knn_chunks(Q, K, N) + 1));
    w.chunk_off = off;
    off += up(sizeof(int32_t) * static_cast<size_t>(B) * (knn_chunks(Q, K, N) + 1));
    {
        const int sl = csr_slices(B, N);
        w.heavy_cap = (N + sl - 1) / sl;
        w.heavy = off; off += up(sizeof(int32_t) * static_cast<size_t>(B) * sl * w.heavy_cap);
        w.heavy_count = off; off += up(sizeof(int32_t) * static_cast<size_t>(B) * sl);
    }
    w.total = off;
    return w;
}

cudaError_t launch_knn_fwd(const KnnArgs& a, cudaStream_t st) {
    if (static_cast<long long>(a.B) * a.Q == 0) return cudaSuccess;
    const int l2 = lpq_log2_for(a.d);
    const int ch = (a.d + (8 << l2) - 1) / (8 << l2);
    if (a.N <= kUTUseN && a.K <= 8) {
        // tensor-core forward over 16-query tiles, one wave of resident CTAs
        const size_t usmem = uf_smem_layout().total;
        const cudaError_t e = ensure_smem<knn_fwd_union_kernel>(usmem);
        if (e != cudaSuccess) return e;
        const long long tpi = (a.Q + 15) / 16;
        const long long tiles = static_cast<long long>(a.B) * tpi;
        long long grid = static_cast<long long>(sm_count()) * resident<knn_fwd_union_kernel>(kUTThreads, usmem);
        if (grid > tiles) grid = tiles;
        const long long span = (tiles + grid - 1) / grid;
        grid = (tiles + span - 1) / span;
        knn_fwd_union_kernel<<<static_cast<unsigned>(grid), kUTThreads, usmem, st>>>(a, tpi, span);
        note_launch();
        return cudaGetLastError();
    }
    const cudaError_t e = (a.K <= 8) ? fwd_k<8>(a, st, l2, ch) : fwd_k<16>(a, st, l2, ch);
    note_launch();
    return e;
}

cudaError_t launch_knn_index(const KnnArgs& a, cudaStream_t st) {
    // built even for Q == 0 (it then writes empty lists)
    const int slices = csr_slices(a.B, a.N);
    const size_t csmem = csr_smem_layout((a.N + slices - 1) / slices).total;
    cudaError_t e = ensure_smem<knn_csr_kernel>(csmem);
    if (e != cudaSuccess) return e;
    const long long nq = static_cast<long long>(a.B) * a.Q;
    if (nq > 0) {
        knn_keys_kernel<<<static_cast<unsigned>((nq + 255) / 256), 256, 0, st>>>(a);
        note_launch();
    }
    knn_csr_kernel<<<dim3(slices, a.B), kCsrThreads, csmem, st>>>(a, slices, knn_chunks(a.Q, a.K, a.N));
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_knn_bwd_indexed(const KnnArgs& a, cudaStream_t st) {
    const int l2 = lpq_log2_for(a.d);
    const int lanes = 1 << l2;
    const int ch = (a.d + 8 * lanes - 1) / (8 * lanes);
    const int NH = a.d / 32;
    const KnnWorkspace ws = knn_workspace_layout(a.B, a.Q, a.N, a.d, a.K);
    const unsigned qblocks = static_cast<unsigned>(ws.query_blocks);
    const GatherPlan g = gather_plan(a.B, a.Q, a.d, a.K, true);
    cudaError_t e = cudaSuccess;
    int qb_used = static_cast<int>(qblocks);
    if (qblocks > 0 && a.N <= kUTUseN && a.K <= 8) {
        // tensor-core query pass over 16-query tiles (grid within the workspace's dp rows)
        const size_t usmem = ut_smem_layout(a.d >> 5).total;
        e = ensure_smem<knn_bwd_query_union_kernel>(usmem);
        if (e != cudaSuccess) return e;
        const long long tpi = (a.Q + 15) / 16;
        const long long tiles = static_cast<long long>(a.B) * tpi;
        long long grid = static_cast<long long>(sm_count()) * resident<knn_bwd_query_union_kernel>(kUTThreads, usmem);
        if (grid > static_cast<long long>(qblocks)) grid = qblocks;
        if (grid > tiles) grid = tiles;
        const long long span = (tiles + grid - 1) / grid;
        grid = (tiles + span - 1) / span;
        qb_used = static_cast<int>(grid);
        knn_bwd_query_union_kernel<<<static_cast<unsigned>(grid), kUTThreads, usmem, st>>>(a, tpi, span);
        note_launch();
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    } else if (qblocks > 0) {
        const size_t smem = sizeof(float) * kGatherWarps * (32 >> l2) * NH;
        if (g.shared)
            e = (a.K <= 8) ? bwdq_shared_k<8>(a, st, g, smem) : bwdq_shared_k<16>(a, st, g, smem);
        else
            e = (a.K <= 8) ? bwdq_k<8>(a, st, l2, ch, qblocks, smem) : bwdq_k<16>(a, st, l2, ch, qblocks, smem);
        note_launch();
        if (e != cudaSuccess) return e;
    }
    const int slices = csr_slices(a.B, a.N);
    const int chunks = knn_chunks(a.Q, a.K, a.N);
    const int qb = qb_used;
    const long long warps = static_cast<long long>(a.B) * chunks;
    const int hctas = heavy_ctas(a.Q, a.K, a.N);
    const unsigned tblocks = static_cast<unsigned>(hctas + (warps + kGatherWarps - 1) / kGatherWarps);
    const int nlists = a.B * slices;
    knn_bwd_token_kernel<<<tblocks, kGatherThreads, 0, st>>>(a, l2, qb, nlists, chunks, hctas);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_knn_bwd(const KnnArgs& a, cudaStream_t st) {
    const cudaError_t e = launch_knn_index(a, st);
    if (e != cudaSuccess) return e;
    return launch_knn_bwd_indexed(a, st);
}

ACL_CHECK_READER(read_checks_knn)

}  // namespace acl
