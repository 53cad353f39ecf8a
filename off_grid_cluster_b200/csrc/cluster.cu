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
// (y, x, id) -- one bitonic network over both lists -- and then walks the
// bisection tree breadth first: at each level a segment's extent is read off
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

// Byte offsets of the shared-memory regions of cluster_kernel.
struct ClusterSmem {
    size_t region, kid, warp, total;
};
__host__ __device__ __forceinline__ size_t round16(size_t x) { return (x + 15) & ~size_t(15); }
__host__ __device__ __forceinline__ ClusterSmem cluster_smem_layout(int N, int C) {
    const size_t P = static_cast<size_t>(next_pow2(N));
    const size_t G = static_cast<size_t>((N + C - 1) / C);
    const size_t n = static_cast<size_t>(N);
    ClusterSmem L;
    L.region = round16(8 * n);                                   // xs, ys
    const size_t sort_keys = 16 * P;                             // 2P u64
    const size_t levels = 12 * n + 4 * G + n + G + 16;           // lists, scans, segments, flags
    L.kid = L.region + round16(sort_keys > levels ? sort_keys : levels);
    L.warp = L.kid + round16(4 * P);                             // 2P u16 ids
    L.total = L.warp + 32 * sizeof(int);
    return L;
}

// Exclusive prefix sum of vals[0..n) (uint16) into out[0..n); all threads call.
__device__ void block_exclusive_scan_u16(const uint16_t* vals, uint16_t* out, int n,
                                         int* warp_tot) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int per = (n + kClusterThreads - 1) / kClusterThreads;
    const int p0 = tid * per;
    int local = 0;
    for (int i = 0; i < per; ++i)
        if (p0 + i < n) local += vals[p0 + i];
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int v = warp_tot[lane];
        int s = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int u = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += u;
        }
        warp_tot[lane] = s - v;  // exclusive prefix of warp totals
    }
    __syncthreads();
    int run = warp_tot[warp] + incl - local;
    for (int i = 0; i < per; ++i) {
        if (p0 + i < n) {
            out[p0 + i] = static_cast<uint16_t>(run);
            run += vals[p0 + i];
        }
    }
    __syncthreads();
}

// Shared memory: xs, ys [N] f32 | keys [2P] u64 | ids [2P] u16, where the level
// arrays (list ping-pong, flags, scan, segments) overlay the keys region once the
// sort is done.
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
    uint8_t* region = smem + L.region;
    uint64_t* keys = reinterpret_cast<uint64_t*>(region);
    uint16_t* kid = reinterpret_cast<uint16_t*>(smem + L.kid);
    // level arrays, inside the keys region (sized for both uses)
    uint16_t* lx0 = reinterpret_cast<uint16_t*>(region);
    uint16_t* ly0 = lx0 + N;
    uint16_t* lx1 = ly0 + N;
    uint16_t* ly1 = lx1 + N;
    uint16_t* scanv = ly1 + N;
    uint16_t* scanout = scanv + N;
    uint16_t* seg_c0 = scanout + N;
    uint16_t* seg_g = seg_c0 + G;
    uint8_t* flag = reinterpret_cast<uint8_t*>(seg_g + G);
    uint8_t* seg_axis = flag + N;
    int* warp_tot = reinterpret_cast<int*>(smem + L.warp);

    const float* img = xy + static_cast<size_t>(b) * N * 2;
    for (int i = tid; i < N; i += kClusterThreads) {
        float2 p = reinterpret_cast<const float2*>(img)[i];
        xs[i] = p.x;
        ys[i] = p.y;
    }
    __syncthreads();

    // ---- one bitonic network sorting both lists: [0,P) by (x,y,id), [P,2P) by (y,x,id)
    for (int i = tid; i < 2 * P; i += kClusterThreads) {
        const int li = i & (P - 1);
        if (li < N) {
            const uint32_t ox = order_bits(xs[li]), oy = order_bits(ys[li]);
            keys[i] = (i < P) ? ((uint64_t(ox) << 32) | oy) : ((uint64_t(oy) << 32) | ox);
            kid[i] = static_cast<uint16_t>(li);
        } else {
            keys[i] = ~uint64_t(0);
            kid[i] = 0xFFFFu;
        }
    }
    __syncthreads();
    for (int k = 2; k <= P; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = tid; i < 2 * P; i += kClusterThreads) {
                const int ixj = i ^ j;
                if (ixj > i) {
                    const bool up = ((i & (P - 1)) & k) == 0;
                    const uint64_t ka = keys[i], kb = keys[ixj];
                    const uint16_t ia = kid[i], ib = kid[ixj];
                    const bool gt = (ka > kb) || (ka == kb && ia > ib);
                    if (gt == up) {
                        keys[i] = kb;
                        keys[ixj] = ka;
                        kid[i] = ib;
                        kid[ixj] = ia;
                    }
                }
            }
            __syncthreads();
        }
    }
    // ids live above the keys region, so copying them into the level arrays is safe
    for (int i = tid; i < N; i += kClusterThreads) {
        lx0[i] = kid[i];
        ly0[i] = kid[P + i];
    }
    for (int c = tid; c < G; c += kClusterThreads) {
        seg_c0[c] = 0;
        seg_g[c] = static_cast<uint16_t>(G);
    }
    __syncthreads();

    uint16_t *LX = lx0, *LY = ly0, *NX = lx1, *NY = ly1;
    for (int gmax = G; gmax > 1; gmax = (gmax + 1) / 2) {
        // A: split axis of every segment, from the ends of its sorted lists
        for (int c = tid; c < G; c += kClusterThreads) {
            const int c0 = seg_c0[c], g = seg_g[c];
            if (c == c0 && g >= 2) {
                const int lo = c0 * C, hi = min((c0 + g) * C, N) - 1;
                const double ex = __dsub_rn(static_cast<double>(xs[LX[hi]]),
                                            static_cast<double>(xs[LX[lo]]));
                const double ey = __dsub_rn(static_cast<double>(ys[LY[hi]]),
                                            static_cast<double>(ys[LY[lo]]));
                seg_axis[c0] = (ex >= ey) ? 0 : 1;
            }
        }
        __syncthreads();
        // B: membership of the left part, read off the split-axis list
        for (int p = tid; p < N; p += kClusterThreads) {
            const int c = p / C;
            const int c0 = seg_c0[c], g = seg_g[c];
            if (g >= 2) {
                const int lo = c0 * C, nl = ((g + 1) / 2) * C;
                const uint16_t t = seg_axis[c0] ? LY[p] : LX[p];
                flag[t] = (p - lo < nl) ? 1 : 0;
            }
        }
        __syncthreads();
        // C: prefix count of left members along the other list
        for (int p = tid; p < N; p += kClusterThreads) {
            const int c = p / C;
            const int c0 = seg_c0[c], g = seg_g[c];
            uint16_t v = 0;
            if (g >= 2) {
                const uint16_t t = seg_axis[c0] ? LX[p] : LY[p];
                v = flag[t];
            }
            scanv[p] = v;
        }
        __syncthreads();
        block_exclusive_scan_u16(scanv, scanout, N, warp_tot);
        // D: stable partition of the other list; the axis list is already split
        for (int p = tid; p < N; p += kClusterThreads) {
            const int c = p / C;
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
            } else {
                NX[p] = LX[p];
                NY[dst] = LY[p];
            }
        }
        __syncthreads();
        // E: children become the segments of the next level
        for (int c = tid; c < G; c += kClusterThreads) {
            const int c0 = seg_c0[c], g = seg_g[c];
            if (g >= 2) {
                const int gl = (g + 1) / 2;
                if (c < c0 + gl) {
                    seg_g[c] = static_cast<uint16_t>(gl);
                } else {
                    seg_c0[c] = static_cast<uint16_t>(c0 + gl);
                    seg_g[c] = static_cast<uint16_t>(g - gl);
                }
            }
        }
        uint16_t* t0 = LX; LX = NX; NX = t0;
        uint16_t* t1 = LY; LY = NY; NY = t1;
        __syncthreads();
    }

    // leaves: ids ascending, padding (-1) after the valid ones
    int32_t* out = clusters + static_cast<size_t>(b) * G * C;
    for (int c = tid; c < G; c += kClusterThreads) {
        const int lo = c * C;
        const int n = min(C, N - lo);
        for (int s = 0; s < n; ++s) {
            const int id = LX[lo + s];
            int rank = 0;
            for (int u = 0; u < n; ++u) rank += (LX[lo + u] < id);
            out[lo + rank] = id;
        }
        for (int s = n; s < C; ++s) out[lo + s] = -1;
    }
}

// ---------------------------------------------------------------------------
// neighbours: R nearest centroids per cluster
// ---------------------------------------------------------------------------

constexpr int kNbrThreads = 128;

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

    const int g = blockIdx.x * kNbrThreads + threadIdx.x;
    if (g >= G) return;
    double bd[RMAX];
    int bh[RMAX];
#pragma unroll
    for (int r = 0; r < RMAX; ++r) {
        bd[r] = DBL_MAX;
        bh[r] = -1;
    }
    const double gx = cx[g], gy = cy[g];
    for (int h = 0; h < G; ++h) {
        const double dx = __dsub_rn(cx[h], gx);
        const double dy = __dsub_rn(cy[h], gy);
        const double d = __dadd_rn(__dmul_rn(dx, dx), __dmul_rn(dy, dy));
        if (d < bd[RMAX - 1]) {  // strict: an equal distance keeps the lower id already held
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
#pragma unroll
    for (int r = 0; r < RMAX; ++r) {
        if (r >= R) break;
        const int h = bh[r];
        for (int s = 0; s < C; ++s)
            row[r * C + s] = (h >= 0) ? cl[static_cast<size_t>(h) * C + s] : -1;
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
    dim3 grid((G + kNbrThreads - 1) / kNbrThreads, B);
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

}  // namespace acl
