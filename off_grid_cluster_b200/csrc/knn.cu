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

template <int KMAX>
__global__ void __launch_bounds__(kTableThreads)
    knn_table_kernel(const float* __restrict__ xy, int N, int GH, int GW, int K, BinGrid bg,
                     int32_t* __restrict__ table) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int b = blockIdx.y, tid = threadIdx.x;
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

    const int cell = blockIdx.x * kTableThreads + tid;
    if (cell >= GH * GW) return;
    const int r = cell / GW, c = cell - r * GW;
    const double px = static_cast<double>(c) + 0.5, py = static_cast<double>(r) + 0.5;
    const int qbx = bin_coord(static_cast<float>(c) + 0.5f, bg.inv_s, bg.nbx);
    const int qby = bin_coord(static_cast<float>(r) + 0.5f, bg.inv_s, bg.nby);
    double bd[KMAX];
    int bi[KMAX];
#pragma unroll
    for (int k = 0; k < KMAX; ++k) {
        bd[k] = DBL_MAX;
        bi[k] = 0x7fffffff;
    }
    const int maxring = max(bg.nbx, bg.nby);
    for (int rho = 0; rho <= maxring; ++rho) {
        const int by0 = qby - rho, by1 = qby + rho, bx0 = qbx - rho, bx1 = qbx + rho;
        const int ylo = max(by0, 0), yhi = min(by1, bg.nby - 1);
        for (int by = ylo; by <= yhi; ++by) {
            const bool full = (by == by0 || by == by1);
            const int xlo = max(bx0, 0), xhi = min(bx1, bg.nbx - 1);
            for (int bx = xlo; bx <= xhi; ++bx) {
                if (!full && bx != bx0 && bx != bx1) continue;
                const int bin = by * bg.nbx + bx;
                const int s0 = bin > 0 ? cnt[bin - 1] : 0, s1 = cnt[bin];
                for (int i = s0; i < s1; ++i) {
                    const float2 p = txy[i];
                    const double dx = __dsub_rn(static_cast<double>(p.x), px);
                    const double dy = __dsub_rn(static_cast<double>(p.y), py);
                    const double d = __dadd_rn(__dmul_rn(dx, dx), __dmul_rn(dy, dy));
                    topk_insert<KMAX>(bd, bi, d, tidv[i]);
                }
            }
        }
        const double lim = static_cast<double>(rho) * static_cast<double>(bg.s);
        if (bd[KMAX - 1] < lim * lim) break;
    }
    int32_t* out = table + static_cast<size_t>(b) * GH * GW * K + static_cast<size_t>(cell) * K;
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
            float* wout = a.w + (static_cast<size_t>(gq) * NH + hh) * a.K;
#pragma unroll
            for (int j = 0; j < KT; ++j) {
                if (j < a.K) wout[j] = w[j];
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

// Stable counting sort of an image's (query, slot) entries by token id.
__global__ void __launch_bounds__(kCsrThreads) knn_csr_kernel(const KnnArgs a, int nw) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int b = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int N = a.N;
    const long long E = static_cast<long long>(a.Q) * a.K;
    uint16_t* pre = reinterpret_cast<uint16_t*>(smem);
    int* off = reinterpret_cast<int*>(smem + ((2 * static_cast<size_t>(nw) * N + 15) & ~size_t(15)));
    int* scratch = off + N + 1;
    const int32_t* keys = a.keys + static_cast<size_t>(b) * E;
    int32_t* csr = a.csr + static_cast<size_t>(b) * E;
    for (int i = tid; i < nw * N; i += kCsrThreads) pre[i] = 0;
    __syncthreads();
    const long long lo = (warp < nw) ? warp * E / nw : 0;
    const long long hi = (warp < nw) ? (warp + 1) * E / nw : 0;
    uint16_t* mine = pre + static_cast<size_t>(warp) * N;
    if (warp < nw) {
        for (long long base = lo; base < hi; base += 32) {
            const long long e = base + lane;
            int key = (e < hi) ? keys[e] : -1;
            if (key >= N) key = -1;
            const unsigned peers = __match_any_sync(0xffffffffu, key);
            if (key >= 0 && lane == __ffs(peers) - 1) mine[key] += static_cast<uint16_t>(__popc(peers));
            __syncwarp();
        }
    }
    __syncthreads();
    for (int t = tid; t < N; t += kCsrThreads) {
        int run = 0;
        for (int w = 0; w < nw; ++w) {
            const int c = pre[static_cast<size_t>(w) * N + t];
            pre[static_cast<size_t>(w) * N + t] = static_cast<uint16_t>(run);
            run += c;
        }
        off[t] = run;
    }
    __syncthreads();
    const int tot = block_scan(off, N, scratch);
    int32_t* coff = a.csr_off + static_cast<size_t>(b) * (N + 1);
    for (int t = tid; t < N; t += kCsrThreads) coff[t] = off[t];
    if (tid == 0) coff[N] = tot;
    if (warp < nw) {
        const unsigned below = (1u << lane) - 1u;
        for (long long base = lo; base < hi; base += 32) {
            const long long e = base + lane;
            int key = (e < hi) ? keys[e] : -1;
            if (key >= N) key = -1;
            const unsigned peers = __match_any_sync(0xffffffffu, key);
            int before = 0;
            if (key >= 0) {
                before = mine[key];
                csr[off[key] + before + __popc(peers & below)] = static_cast<int32_t>(e);
            }
            __syncwarp();
            if (key >= 0 && lane == __ffs(peers) - 1)
                mine[key] = static_cast<uint16_t>(before + __popc(peers));
            __syncwarp();
        }
    }
}

template <int CH>
__global__ void __launch_bounds__(kGatherThreads)
    knn_bwd_token_kernel(const KnnArgs a, int lpq_log2, int token_blocks, int query_blocks) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int NH = a.d >> 5;
    if (static_cast<int>(blockIdx.x) >= token_blocks) {
        // dp reduction, one CTA per head, fixed order
        __shared__ float red[kGatherWarps];
        const int h = blockIdx.x - token_blocks;
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
        return;
    }
    const int LPQ = 1 << lpq_log2;
    const int sub = lane & (LPQ - 1), grp = lane >> lpq_log2;
    const long long total = static_cast<long long>(a.B) * a.N;
    const long long gt = (static_cast<long long>(blockIdx.x) * kGatherWarps + warp) * (32 >> lpq_log2) + grp;
    if (gt >= total) return;
    const int b = static_cast<int>(gt / a.N), t = static_cast<int>(gt - static_cast<long long>(b) * a.N);
    const int32_t* coff = a.csr_off + static_cast<size_t>(b) * (a.N + 1);
    const int lo = coff[t], hi = coff[t + 1];
    const size_t E = static_cast<size_t>(a.Q) * a.K;
    const int32_t* csr = a.csr + static_cast<size_t>(b) * E;
    const size_t qbase = static_cast<size_t>(b) * a.Q;
#pragma unroll
    for (int ch = 0; ch < CH; ++ch) {
        const int c0 = ch * LPQ * 8 + sub * 8;
        if (c0 >= a.d) break;
        const int hh = c0 >> 5;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        int i = lo;
        for (; i + 4 <= hi; i += 4) {
            int e[4];
            float wv[4];
            uint4 gv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) e[u] = csr[i + u];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int q = e[u] / a.K, j = e[u] - q * a.K;
                wv[u] = a.w[((qbase + q) * NH + hh) * a.K + j];
                gv[u] = ldg16(a.dout + (qbase + q) * a.d + c0);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) fma8(acc, wv[u], gv[u]);
        }
        for (; i < hi; ++i) {
            const int e = csr[i];
            const int q = e / a.K, j = e - q * a.K;
            fma8(acc, a.w[((qbase + q) * NH + hh) * a.K + j], ldg16(a.dout + (qbase + q) * a.d + c0));
        }
        *reinterpret_cast<uint4*>(a.dfeats + static_cast<size_t>(gt) * a.d + c0) = pack8(acc, 1.f);
    }
}

// lanes per query: d/8 rounded up to a power of two, capped at 32
int lpq_log2_for(int d) {
    int lanes = d / 8;
    int l2 = 0;
    while ((1 << l2) < lanes && l2 < 5) ++l2;
    return l2;
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

int csr_chunk_warps(int N) {
    const long long budget = 200 * 1024 - 4LL * (N + 1) - 256;
    long long nw = budget / (2LL * N);
    if (nw > 32) nw = 32;
    if (nw < 1) nw = 1;
    return static_cast<int>(nw);
}

}  // namespace

size_t knn_table_smem_bytes(int N, int nbins) {
    return ((4 * static_cast<size_t>(nbins + 40) + 15) & ~size_t(15)) + 10 * static_cast<size_t>(N);
}

cudaError_t launch_knn_table(const float* xy, int B, int N, int GH, int GW, int K, int32_t* table,
                             cudaStream_t st) {
    const BinGrid bg = choose_bins(N, GH, GW);
    const size_t smem = knn_table_smem_bytes(N, bg.nbx * bg.nby);
    dim3 grid((GH * GW + kTableThreads - 1) / kTableThreads, B);
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
    const int l2 = lpq_log2_for(d);
    const long long per_block = static_cast<long long>(kGatherWarps) * (32 >> l2);
    KnnWorkspace w;
    w.query_blocks = static_cast<int>((static_cast<long long>(BQ) + per_block - 1) / per_block);
    size_t off = 0;
    w.w = off;       off += up(sizeof(float) * BQ * NH * K);
    w.keys = off;    off += up(sizeof(int32_t) * BQ * K);
    w.csr = off;     off += up(sizeof(int32_t) * BQ * K);
    w.csr_off = off; off += up(sizeof(int32_t) * static_cast<size_t>(B) * (N + 1));
    w.dp_part = off; off += up(sizeof(float) * static_cast<size_t>(w.query_blocks) * NH);
    w.total = off;
    return w;
}

cudaError_t launch_knn_fwd(const KnnArgs& a, cudaStream_t st) {
    const int l2 = lpq_log2_for(a.d);
    const int lanes = 1 << l2;
    const int ch = (a.d + 8 * lanes - 1) / (8 * lanes);
    const long long per_block = static_cast<long long>(kGatherWarps) * (32 >> l2);
    const unsigned blocks = static_cast<unsigned>((static_cast<long long>(a.B) * a.Q + per_block - 1) / per_block);
    if (blocks == 0) return cudaSuccess;
    const cudaError_t e = (a.K <= 8) ? fwd_k<8>(a, st, l2, ch, blocks) : fwd_k<16>(a, st, l2, ch, blocks);
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
    cudaError_t e = cudaSuccess;
    if (qblocks > 0) {
        const size_t smem = sizeof(float) * kGatherWarps * (32 >> l2) * NH;
        e = (a.K <= 8) ? bwdq_k<8>(a, st, l2, ch, qblocks, smem) : bwdq_k<16>(a, st, l2, ch, qblocks, smem);
        note_launch();
        if (e != cudaSuccess) return e;
    }
    // the inverse index is built even for Q == 0 (it then writes empty lists)
    const int nw = csr_chunk_warps(a.N);
    const size_t csmem = ((2 * static_cast<size_t>(nw) * a.N + 15) & ~size_t(15)) +
                         4 * static_cast<size_t>(a.N + 1) + 40 * sizeof(int);
    e = ensure_smem<knn_csr_kernel>(csmem);
    if (e != cudaSuccess) return e;
    knn_csr_kernel<<<a.B, kCsrThreads, csmem, st>>>(a, nw);
    note_launch();
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const long long per_block = static_cast<long long>(kGatherWarps) * (32 >> l2);
    const int tblocks = static_cast<int>((static_cast<long long>(a.B) * a.N + per_block - 1) / per_block);
    const int qb = static_cast<int>(qblocks);
    switch (ch) {
        case 1: knn_bwd_token_kernel<1><<<tblocks + NH, kGatherThreads, 0, st>>>(a, l2, tblocks, qb); break;
        case 2: knn_bwd_token_kernel<2><<<tblocks + NH, kGatherThreads, 0, st>>>(a, l2, tblocks, qb); break;
        case 3: knn_bwd_token_kernel<3><<<tblocks + NH, kGatherThreads, 0, st>>>(a, l2, tblocks, qb); break;
        default: knn_bwd_token_kernel<4><<<tblocks + NH, kGatherThreads, 0, st>>>(a, l2, tblocks, qb); break;
    }
    note_launch();
    return cudaGetLastError();
}

}  // namespace acl
