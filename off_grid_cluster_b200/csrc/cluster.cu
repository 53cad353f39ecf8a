// cluster.cu -- local balanced clustering and the cluster-neighbourhood table.
//
// AFFMAE notes, Method "Overall Architecture": attention runs over local balanced
// clusters of tokens that carry explicit 2D coordinates.  The clustering here is
// recursive median bisection (split on the axis of larger extent, ties to x, by
// the key (axis coordinate, other coordinate, token id); the left part takes
// ceil(g/2) clusters of C tokens), and a cluster's neighbourhood is the R = M / C
// clusters of nearest centroid.  Both results are integer and bit-exact: the
// only floating point that decides them is fp64 arithmetic on fp32 inputs,
// written with explicitly rounded operations (no contraction) in the order the
// header states.
//
// GPU design.  One 1024-thread CTA per image holds all of the image in shared
// memory.  Instead of re-sorting every segment at every level (what a literal
// recursion does), the CTA sorts the tokens once by (x, y, id) and once by
// (y, x, id) -- a counting sort into N monotone buckets per axis followed by an
// exact insertion sort inside each bucket, or, when some bucket is crowded
// (repeated or tightly packed coordinates), a bitonic network over packed keys --
// and then walks the bisection tree breadth first: at each level a segment's extent is read off
// the ends of its two sorted lists, its left part is the first ceil(g/2)*C
// entries of the list on its split axis, and the other list is stably
// partitioned with one block-wide prefix sum.  Both lists stay sorted inside
// every segment, so each level costs O(N) work and a handful of barriers.  The
// shape of the tree depends only on (N, C), so no segment bookkeeping beyond a
// per-cluster (first cluster, cluster count) pair is needed.
#include <float.h>

#include "internal.h"

namespace acl {

namespace {

constexpr int kClusterThreads = 1024;

__device__ __forceinline__ uint32_t order_bits(float f) {
    uint32_t u = __float_as_uint(f);
    if ((u & 0x7FFFFFFFu) == 0) u = 0;  // -0 and +0 compare equal
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__host__ __device__ __forceinline__ int next_pow2(int n) {
    int p = 1;
    while (p < n) p <<= 1;
    return p;
}

constexpr int kBucketMax = 32;  // largest bucket the fast path sorts with one thread

// Byte offsets of the shared-memory regions of cluster_kernel:
//   xs, ys [N] f32 | L0 [2N] u16 (sorted X list, then Y list) |
//   U = union of { sort keys [2P] u64 (fallback) or bucket counts [2P] i32 (fast path) }
//             and { level arrays: L1 [2N], scanv [N], scanout [N], posX [N], posY [N],
//                   pos_cluster [N] (u16), seg_c0, seg_g [G] u16, seg_axis [G] u8 } |
//   scratch [160] i32
struct ClusterSmem {
    size_t l0, u, scratch, total;
};
__host__ __device__ __forceinline__ size_t round16(size_t x) { return (x + 15) & ~size_t(15); }
__host__ __device__ __forceinline__ ClusterSmem cluster_smem_layout(int N, int C) {
    const size_t P = static_cast<size_t>(next_pow2(N));
    const size_t G = static_cast<size_t>((N + C - 1) / C);
    const size_t n = static_cast<size_t>(N);
    ClusterSmem L;
    L.l0 = round16(8 * n);
    L.u = L.l0 + round16(4 * n);
    const size_t sort_bytes = 16 * P;
    const size_t level_bytes = 14 * n + 5 * G + 16;
    L.scratch = L.u + round16(sort_bytes > level_bytes ? sort_bytes : level_bytes);
    L.total = L.scratch + 160 * sizeof(int);
    return L;
}

__device__ __forceinline__ uint64_t full_key(float a, float b) {
    return (static_cast<uint64_t>(order_bits(a)) << 32) | order_bits(b);
}

// Block-wide min/max of x and y (all threads call; result broadcast through scratch).
__device__ void block_minmax(const float* xs, const float* ys, int N, int* scratch, float& xmin,
                             float& xmax, float& ymin, float& ymax) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    float a = INFINITY, b = -INFINITY, c = INFINITY, d = -INFINITY;
    for (int i = tid; i < N; i += blockDim.x) {
        a = fminf(a, xs[i]);
        b = fmaxf(b, xs[i]);
        c = fminf(c, ys[i]);
        d = fmaxf(d, ys[i]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        a = fminf(a, __shfl_xor_sync(0xffffffffu, a, o));
        b = fmaxf(b, __shfl_xor_sync(0xffffffffu, b, o));
        c = fminf(c, __shfl_xor_sync(0xffffffffu, c, o));
        d = fmaxf(d, __shfl_xor_sync(0xffffffffu, d, o));
    }
    float* f = reinterpret_cast<float*>(scratch);
    __syncthreads();
    if (lane == 0) {
        f[4 * warp] = a;
        f[4 * warp + 1] = b;
        f[4 * warp + 2] = c;
        f[4 * warp + 3] = d;
    }
    __syncthreads();
    if (warp == 0) {
        a = lane < nw ? f[4 * lane] : INFINITY;
        b = lane < nw ? f[4 * lane + 1] : -INFINITY;
        c = lane < nw ? f[4 * lane + 2] : INFINITY;
        d = lane < nw ? f[4 * lane + 3] : -INFINITY;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            a = fminf(a, __shfl_xor_sync(0xffffffffu, a, o));
            b = fmaxf(b, __shfl_xor_sync(0xffffffffu, b, o));
            c = fminf(c, __shfl_xor_sync(0xffffffffu, c, o));
            d = fmaxf(d, __shfl_xor_sync(0xffffffffu, d, o));
        }
        if (lane == 0) {
            f[128] = a;
            f[129] = b;
            f[130] = c;
            f[131] = d;
        }
    }
    __syncthreads();
    xmin = f[128];
    xmax = f[129];
    ymin = f[130];
    ymax = f[131];
    __syncthreads();
}

// Exclusive prefix sum of int data[0..n) in place (all threads call); returns the total.
__device__ int block_scan_int(int* data, int n, int* scratch) {
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
    if (warp == 0) {
        const int v = lane < nw ? scratch[lane] : 0;
        int sc = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, sc, o);
            if (lane >= o) sc += u;
        }
        scratch[lane] = sc - v;
        if (lane == 31) scratch[32] = sc;
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
    const int total = scratch[32];
    __syncthreads();
    return total;
}

// Exclusive prefix sum of vals[0..n) (uint16) into out[0..n); all threads call.
__device__ void block_exclusive_scan_u16(const uint16_t* vals, uint16_t* out, int n, int* scratch) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    const int per = (n + blockDim.x - 1) / blockDim.x;
    const int p0 = tid * per;
    int local = 0;
    for (int i = 0; i < per; ++i)
        if (p0 + i < n) local += vals[p0 + i];
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) scratch[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int v = lane < nw ? scratch[lane] : 0;
        int sc = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, sc, o);
            if (lane >= o) sc += u;
        }
        scratch[lane] = sc - v;
    }
    __syncthreads();
    int run = scratch[warp] + incl - local;
    for (int i = 0; i < per; ++i) {
        if (p0 + i < n) {
            out[p0 + i] = static_cast<uint16_t>(run);
            run += vals[p0 + i];
        }
    }
    __syncthreads();
}

// Bucket index of v: floor((v - vmin) * scale) clamped to [0, nb - 1].  Every step is
// monotone non-decreasing in v, so bucket order never contradicts coordinate order.
__device__ __forceinline__ int bucket_of(float v, float vmin, float scale, int nb) {
    const float t = (v - vmin) * scale;
    if (!(t >= 0.f)) return 0;
    if (t >= static_cast<float>(nb)) return nb - 1;
    const int i = static_cast<int>(t);
    return i > nb - 1 ? nb - 1 : i;
}

// Bitonic sort of 2P packed u64 values in shared memory, [0,P) and [P,2P) independently.
__device__ void bitonic_2lists(uint64_t* keys, int P) {
    const int tid = threadIdx.x, nt = blockDim.x;
    for (int k = 2; k <= P; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = tid; i < 2 * P; i += nt) {
                const int ixj = i ^ j;
                if (ixj > i) {
                    const bool up = ((i & (P - 1)) & k) == 0;
                    const uint64_t ka = keys[i], kb = keys[ixj];
                    if ((ka > kb) == up) {
                        keys[i] = kb;
                        keys[ixj] = ka;
                    }
                }
            }
            __syncthreads();
        }
    }
}

// Fallback sort for inputs with crowded buckets (many equal or clustered coordinates),
// with 48-bit packed keys only.  Pass 1 sorts (a, id) per list: T_x = tokens in (x, id)
// order, T_y = tokens in (y, id) order.  Pass 2 sorts the X list by (x, r) where r is a
// token's position in T_y -- so ties in x fall back to (y, id) -- and the Y list by (y, r)
// with r its position in T_x; mapping r back through T_y / T_x gives the tokens.
__device__ void fallback_sort(const float* xs, const float* ys, int N, int P, uint64_t* keys,
                              uint16_t* L0) {
    const int tid = threadIdx.x, nt = blockDim.x;
    for (int i = tid; i < 2 * P; i += nt) {
        const int li = i & (P - 1);
        keys[i] = (li < N) ? ((static_cast<uint64_t>(order_bits(i < P ? xs[li] : ys[li])) << 16) | li)
                           : ~uint64_t(0);
    }
    __syncthreads();
    bitonic_2lists(keys, P);
    for (int i = tid; i < N; i += nt) {
        L0[i] = static_cast<uint16_t>(keys[i] & 0xFFFFu);          // T_x
        L0[N + i] = static_cast<uint16_t>(keys[P + i] & 0xFFFFu);  // T_y
    }
    __syncthreads();
    for (int i = tid; i < 2 * P; i += nt) {
        const int li = i & (P - 1);
        uint64_t k = ~uint64_t(0);
        if (li < N) {
            if (i < P) {
                const int t = L0[N + li];  // li-th token of the (y, id) order
                k = (static_cast<uint64_t>(order_bits(xs[t])) << 16) | li;
            } else {
                const int t = L0[li];      // li-th token of the (x, id) order
                k = (static_cast<uint64_t>(order_bits(ys[t])) << 16) | li;
            }
        }
        keys[i] = k;
    }
    __syncthreads();
    bitonic_2lists(keys, P);
    for (int i = tid; i < N; i += nt) {
        const int rx = static_cast<int>(keys[i] & 0xFFFFu);
        const int ry = static_cast<int>(keys[P + i] & 0xFFFFu);
        keys[i] = L0[N + rx];
        keys[P + i] = L0[ry];
    }
    __syncthreads();
    for (int i = tid; i < N; i += nt) {
        L0[i] = static_cast<uint16_t>(keys[i]);
        L0[N + i] = static_cast<uint16_t>(keys[P + i]);
    }
    __syncthreads();
}

__global__ void __launch_bounds__(kClusterThreads)
    cluster_kernel(const float* __restrict__ xy, int N, int C, int32_t* __restrict__ clusters) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int b = blockIdx.x;
    const int tid = threadIdx.x;
    const int G = (N + C - 1) / C;
    const int P = next_pow2(N);
    const ClusterSmem L = cluster_smem_layout(N, C);
    float* xs = reinterpret_cast<float*>(smem);
    float* ys = xs + N;
    uint16_t* L0 = reinterpret_cast<uint16_t*>(smem + L.l0);  // [2N]: X list then Y list
    uint8_t* U = smem + L.u;
    int* scratch = reinterpret_cast<int*>(smem + L.scratch);

    const float2* img = reinterpret_cast<const float2*>(xy) + static_cast<size_t>(b) * N;
    for (int i = tid; i < N; i += kClusterThreads) {
        const float2 p = img[i];
        xs[i] = p.x;
        ys[i] = p.y;
    }
    __syncthreads();

    // ---- sort both lists: counting sort into N monotone buckets per axis, then an exact
    //      insertion sort inside each (small) bucket by (axis coord, other coord, id)
    float xmin, xmax, ymin, ymax;
    block_minmax(xs, ys, N, scratch, xmin, xmax, ymin, ymax);
    const int NB = N;
    const float sx = (float)NB / (xmax - xmin), sy = (float)NB / (ymax - ymin);
    int* cnt = reinterpret_cast<int*>(U);  // [2 NB]
    for (int i = tid; i < 2 * NB; i += kClusterThreads) cnt[i] = 0;
    __syncthreads();
    const bool sx_ok = isfinite(sx), sy_ok = isfinite(sy);
    for (int i = tid; i < N; i += kClusterThreads) {
        atomicAdd(&cnt[sx_ok ? bucket_of(xs[i], xmin, sx, NB) : 0], 1);
        atomicAdd(&cnt[NB + (sy_ok ? bucket_of(ys[i], ymin, sy, NB) : 0)], 1);
    }
    __syncthreads();
    int crowded = 0;
    for (int i = tid; i < 2 * NB; i += kClusterThreads) crowded |= (cnt[i] > kBucketMax);
    crowded = __syncthreads_or(crowded);
    if (!crowded) {
        block_scan_int(cnt, 2 * NB, scratch);
        for (int i = tid; i < N; i += kClusterThreads) {
            L0[atomicAdd(&cnt[sx_ok ? bucket_of(xs[i], xmin, sx, NB) : 0], 1)] = static_cast<uint16_t>(i);
            L0[atomicAdd(&cnt[NB + (sy_ok ? bucket_of(ys[i], ymin, sy, NB) : 0)], 1)] =
                static_cast<uint16_t>(i);
        }
        __syncthreads();  // cnt[bb] = end of bucket bb
        for (int bb = tid; bb < 2 * NB; bb += kClusterThreads) {
            const int s0 = bb > 0 ? cnt[bb - 1] : 0, s1 = cnt[bb];
            const bool isx = bb < NB;
            for (int i = s0 + 1; i < s1; ++i) {
                const int t = L0[i];
                const uint64_t kt = isx ? full_key(xs[t], ys[t]) : full_key(ys[t], xs[t]);
                int j = i - 1;
                while (j >= s0) {
                    const int u = L0[j];
                    const uint64_t ku = isx ? full_key(xs[u], ys[u]) : full_key(ys[u], xs[u]);
                    if (ku < kt || (ku == kt && u < t)) break;
                    L0[j + 1] = static_cast<uint16_t>(u);
                    --j;
                }
                L0[j + 1] = static_cast<uint16_t>(t);
            }
        }
        __syncthreads();
    } else {
        fallback_sort(xs, ys, N, P, reinterpret_cast<uint64_t*>(U), L0);
    }

    // ---- level arrays (overlay U now that the sort is done)
    uint16_t* L1 = reinterpret_cast<uint16_t*>(U);  // [2N]
    uint16_t* scanv = L1 + 2 * N;
    uint16_t* scanout = scanv + N;
    uint16_t* posX = scanout + N;
    uint16_t* posY = posX + N;
    uint16_t* pos_cluster = posY + N;
    uint16_t* seg_c0 = pos_cluster + N;
    uint16_t* seg_g = seg_c0 + G;
    uint8_t* seg_axis = reinterpret_cast<uint8_t*>(seg_g + G);
    for (int p = tid; p < N; p += kClusterThreads) {
        posX[L0[p]] = static_cast<uint16_t>(p);
        posY[L0[N + p]] = static_cast<uint16_t>(p);
        pos_cluster[p] = static_cast<uint16_t>(p / C);
    }
    for (int c = tid; c < G; c += kClusterThreads) {
        seg_c0[c] = 0;
        seg_g[c] = static_cast<uint16_t>(G);
    }
    __syncthreads();

    uint16_t *LX = L0, *LY = L0 + N, *NX = L1, *NY = L1 + N;
    bool first = true;
    for (int gmax = G; gmax > 1; gmax = (gmax + 1) / 2) {
        // A: the previous level's children become segments; then each segment's axis
        for (int c = tid; c < G; c += kClusterThreads) {
            int c0 = seg_c0[c], g = seg_g[c];
            if (!first && g >= 2) {
                const int gl = (g + 1) / 2;
                if (c < c0 + gl) {
                    g = gl;
                } else {
                    c0 += gl;
                    g -= gl;
                }
                seg_c0[c] = static_cast<uint16_t>(c0);
                seg_g[c] = static_cast<uint16_t>(g);
            }
            if (c == c0 && g >= 2) {
                const int lo = c0 * C, hi = min((c0 + g) * C, N) - 1;
                const double ex = __dsub_rn(static_cast<double>(xs[LX[hi]]), static_cast<double>(xs[LX[lo]]));
                const double ey = __dsub_rn(static_cast<double>(ys[LY[hi]]), static_cast<double>(ys[LY[lo]]));
                seg_axis[c0] = (ex >= ey) ? 0 : 1;
            }
        }
        first = false;
        __syncthreads();
        // C: is the other list's element in the left part?  (its rank on the split axis)
        for (int p = tid; p < N; p += kClusterThreads) {
            const int c = pos_cluster[p];
            const int c0 = seg_c0[c], g = seg_g[c];
            uint16_t v = 0;
            if (g >= 2) {
                const int lo = c0 * C, nl = ((g + 1) / 2) * C;
                const int ax = seg_axis[c0];
                const int t = ax ? LX[p] : LY[p];
                const int pa = ax ? posY[t] : posX[t];
                v = (pa - lo < nl) ? 1 : 0;
            }
            scanv[p] = v;
        }
        __syncthreads();
        block_exclusive_scan_u16(scanv, scanout, N, scratch);
        // D: stable partition of the other list; the axis list is already split
        for (int p = tid; p < N; p += kClusterThreads) {
            const int c = pos_cluster[p];
            const int c0 = seg_c0[c], g = seg_g[c];
            if (g < 2) {
                NX[p] = LX[p];
                NY[p] = LY[p];
                continue;
            }
            const int lo = c0 * C, nl = ((g + 1) / 2) * C;
            const int before = scanout[p] - scanout[lo];
            const int dst = scanv[p] ? lo + before : lo + nl + (p - lo - before);
            if (seg_axis[c0]) {
                NY[p] = LY[p];
                NX[dst] = LX[p];
                posX[LX[p]] = static_cast<uint16_t>(dst);
            } else {
                NX[p] = LX[p];
                NY[dst] = LY[p];
                posY[LY[p]] = static_cast<uint16_t>(dst);
            }
        }
        uint16_t* t0 = LX; LX = NX; NX = t0;
        uint16_t* t1 = LY; LY = NY; NY = t1;
        __syncthreads();
    }

    // leaves: ids ascending, padding (-1) after the valid ones; one thread per slot ranks
    // its id among its cluster's ids
    int32_t* out = clusters + static_cast<size_t>(b) * G * C;
    for (int q = tid; q < G * C; q += kClusterThreads) {
        const int lo = (q / C) * C;
        const int n = min(C, N - lo);
        if (q - lo >= n) {
            out[q] = -1;
            continue;
        }
        const int id = LX[q];
        int rank = 0;
        for (int u = 0; u < n; ++u) rank += (LX[lo + u] < id);
        out[lo + rank] = id;
    }
}

// ---------------------------------------------------------------------------
// neighbours: R nearest centroids per cluster
// ---------------------------------------------------------------------------

constexpr int kNbrThreads = 256;
constexpr int kNbrWarps = kNbrThreads / 32;

// (d, h) < (d', h') in the neighbour order
__device__ __forceinline__ bool nbr_less(double d, int h, double d2, int h2) {
    return d < d2 || (d == d2 && h < h2);
}

// One warp per query cluster g.  Every CTA first computes the G centroids of its image in
// shared memory (fp64, slot order, as the header states).  Lane l scores the candidate
// clusters h = l, l + 32, ... and keeps its own top-RMAX by (dist2, h); R rounds of a
// warp-wide argmin over the lanes' heads then pop the R nearest in order.
template <int RMAX>
__global__ void __launch_bounds__(kNbrThreads)
    neighbors_kernel(const float* __restrict__ xy, const int32_t* __restrict__ clusters, int N,
                     int C, int M, int32_t* __restrict__ nbr) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int b = blockIdx.y;
    const int G = (N + C - 1) / C;
    const int R = M / C;
    double* cx = reinterpret_cast<double*>(smem);
    double* cy = cx + G;
    const float* img = xy + static_cast<size_t>(b) * N * 2;
    const int32_t* cl = clusters + static_cast<size_t>(b) * G * C;

    for (int g = threadIdx.x; g < G; g += kNbrThreads) {
        double sx = 0.0, sy = 0.0;
        int cnt = 0;
        for (int s = 0; s < C; ++s) {
            const int t = cl[static_cast<size_t>(g) * C + s];
            ACL_DEVICE_CHECK(t >= -1 && t < N);
            if (t < 0 || t >= N) continue;
            sx = __dadd_rn(sx, static_cast<double>(img[2 * t]));
            sy = __dadd_rn(sy, static_cast<double>(img[2 * t + 1]));
            ++cnt;
        }
        const double dc = static_cast<double>(cnt > 0 ? cnt : 1);
        cx[g] = __ddiv_rn(sx, dc);
        cy[g] = __ddiv_rn(sy, dc);
    }
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = blockIdx.x * kNbrWarps + warp;
    if (g >= G) return;
    double bd[RMAX];
    int bh[RMAX];
#pragma unroll
    for (int r = 0; r < RMAX; ++r) {
        bd[r] = DBL_MAX;
        bh[r] = 0x7fffffff;
    }
    const double gx = cx[g], gy = cy[g];
    for (int h = lane; h < G; h += 32) {
        const double dx = __dsub_rn(cx[h], gx);
        const double dy = __dsub_rn(cy[h], gy);
        const double d = __dadd_rn(__dmul_rn(dx, dx), __dmul_rn(dy, dy));
        if (d < bd[RMAX - 1]) {  // h ascends within a lane, so equal d keeps the lower id
            bool placed = false;
#pragma unroll
            for (int r = RMAX - 1; r >= 0; --r) {
                if (!placed) {
                    if (r > 0 && bd[r - 1] > d) {
                        bd[r] = bd[r - 1];
                        bh[r] = bh[r - 1];
                    } else {
                        bd[r] = d;
                        bh[r] = h;
                        placed = true;
                    }
                }
            }
        }
    }
    int32_t* row = nbr + (static_cast<size_t>(b) * G + g) * M;
    for (int r = 0; r < R; ++r) {
        // warp argmin of the lanes' heads
        double d = bd[0];
        int h = bh[0];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const double d2 = __shfl_xor_sync(0xffffffffu, d, o);
            const int h2 = __shfl_xor_sync(0xffffffffu, h, o);
            if (nbr_less(d2, h2, d, h)) {
                d = d2;
                h = h2;
            }
        }
        const bool valid = (h != 0x7fffffff);
        if (valid && bh[0] == h) {  // the owner pops its head
#pragma unroll
            for (int q = 0; q < RMAX - 1; ++q) {
                bd[q] = bd[q + 1];
                bh[q] = bh[q + 1];
            }
            bd[RMAX - 1] = DBL_MAX;
            bh[RMAX - 1] = 0x7fffffff;
        }
        for (int s = lane; s < C; s += 32)
            row[r * C + s] = valid ? cl[static_cast<size_t>(h) * C + s] : -1;
    }
}

}  // namespace

size_t cluster_smem_bytes(int N, int C) { return cluster_smem_layout(N, C).total; }

cudaError_t launch_cluster(const float* xy, int B, int N, int C, int32_t* clusters,
                           cudaStream_t st) {
    const size_t smem = cluster_smem_bytes(N, C);
    cudaError_t e = ensure_smem<cluster_kernel>(smem);
    if (e != cudaSuccess) return e;
    cluster_kernel<<<B, kClusterThreads, smem, st>>>(xy, N, C, clusters);
    note_launch();
    return cudaGetLastError();
}

size_t neighbors_smem_bytes(int G) { return 16 * static_cast<size_t>(G); }

cudaError_t launch_neighbors(const float* xy, const int32_t* clusters, int B, int N, int C, int M,
                             int32_t* nbr, cudaStream_t st) {
    const int G = (N + C - 1) / C;
    const size_t smem = neighbors_smem_bytes(G);
    dim3 grid((G + kNbrWarps - 1) / kNbrWarps, B);
    cudaError_t e;
    if (M / C <= 8) {
        e = ensure_smem<neighbors_kernel<8>>(smem);
        if (e != cudaSuccess) return e;
        neighbors_kernel<8><<<grid, kNbrThreads, smem, st>>>(xy, clusters, N, C, M, nbr);
    } else {
        e = ensure_smem<neighbors_kernel<16>>(smem);
        if (e != cudaSuccess) return e;
        neighbors_kernel<16><<<grid, kNbrThreads, smem, st>>>(xy, clusters, N, C, M, nbr);
    }
    note_launch();
    return cudaGetLastError();
}

ACL_CHECK_READER(read_checks_cluster)

}  // namespace acl
