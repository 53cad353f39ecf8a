// attn.cu -- local cluster attention, forward and backward (bf16 in, fp32 math).
//
// AFFMAE notes, Method "Overall Architecture" (stages of Local Cluster Attention
// over local balanced clusters); arXiv abstract page (Flash-style, numerically
// stable mixed-precision cluster attention kernels).  Per token i of cluster g and
// head h, over the keys j of nbr[g]:
//   s_ij = scale <q_i, k_j> + a_h dx + b_h dy - c_h (dx^2 + dy^2),  dx = x_j - x_i,
//   O_i = softmax_j(s_ij) V,  lse_i = log sum_j exp(s_ij).
//
// Work unit: one warp owns one (image, cluster, head): the cluster's C = 8 queries
// against its M <= 64 neighbourhood keys, D = 32.  The whole neighbourhood fits
// one tile, so the softmax is exact in registers (no running rescale).  The
// contractions run on the tensor cores as m16n8k16 bf16 MMAs with the operands
// swapped so that the 8 queries sit on the MMA's N = 8 side and keys on M:
//   S^T (M x 8)  = K (M x 32) . Q^T          -- 2 k-steps per 16-key tile
//   O^T (32 x 8) = V^T (32 x M) . P^T        -- P^T comes from the S^T
//                  accumulators by an in-register 8x8 transpose (movmatrix)
// so no tile is padded beyond M's rounding to 16.  K, V and Q rows are gathered
// by token id (nbr) with 16-byte cp.async into XOR-swizzled shared tiles that
// ldmatrix reads without bank conflicts.
//
// Backward (recompute, FA2-style, no atomics):
//   pass 1, query-major (same warp/tile as the forward): recompute P from lse,
//     dP^T = V . dO^T, Delta = rowsum(P o dP) (equal to <dO, O>, but exact in fp32
//     because the whole key row is in the tile, and O need not be read),
//     dS = P (dP - Delta),
//     dQ^T = K^T . dS^T, per-(cluster, head) partial sums of the bias gradient.
//     B extra CTAs build, per image, the reverse neighbourhood index: for every
//     key cluster, the query clusters whose table lists it (stable order).
//   pass 2, key-major: one warp per (image, key cluster, head) walks its reverse
//     list two query clusters at a time (16 queries = one MMA M tile):
//     S = Q K_h^T, dP = dO V_h^T, dV^T += dO^T P, dK^T += Q^T dS; 3H extra CTAs
//     reduce the bias-gradient partials in a fixed order.
#include <math.h>

#include "internal.h"

namespace acl {

namespace {

constexpr int kWarps = 4;
constexpr int kThreads = 32 * kWarps;

// ------------------------------------------------------------------ layouts

__host__ __device__ constexpr int fwd_warp_bytes(int MT) { return 140 * MT + 608; }
__host__ __device__ constexpr int bwdq_warp_bytes(int MT) { return 140 * MT + 1120; }
constexpr int kBwdKWarpBytes = 3584;

struct FwdTiles {
    uint8_t* ks;
    uint8_t* vs;
    uint8_t* qs;
    int* kid;
    float2* kxy;
    int* qid;
    float2* qxy;
};

__device__ __forceinline__ FwdTiles fwd_tiles(uint8_t* w, int MT) {
    FwdTiles t;
    t.ks = w;
    t.vs = w + MT * 64;
    t.qs = w + 2 * MT * 64;
    t.kid = reinterpret_cast<int*>(w + 2 * MT * 64 + 512);
    t.kxy = reinterpret_cast<float2*>(t.kid + MT);
    t.qid = reinterpret_cast<int*>(t.kxy + MT);
    t.qxy = reinterpret_cast<float2*>(t.qid + 8);
    return t;
}

// Gather the ids/coordinates of a (cluster, neighbourhood) and issue the cp.async of
// K, V (and Q) rows of head h.  Empty slots are zero-filled.
template <int MT>
__device__ __forceinline__ void load_cluster_tiles(const AttnArgs& a, int b, int g, int h, int lane,
                                                   const FwdTiles& t, const bf16* qsrc) {
    const float2* xyb = reinterpret_cast<const float2*>(a.xy) + static_cast<size_t>(b) * a.N;
    const int32_t* nrow = a.nbr + (static_cast<size_t>(b) * a.G + g) * a.M;
    for (int m = lane; m < MT; m += 32) {
        int id = (m < a.M) ? nrow[m] : -1;
        if (id < 0 || id >= a.N) id = -1;
        t.kid[m] = id;
        t.kxy[m] = (id >= 0) ? xyb[id] : make_float2(0.f, 0.f);
    }
    if (lane < 8) {
        int id = a.clusters[(static_cast<size_t>(b) * a.G + g) * 8 + lane];
        if (id < 0 || id >= a.N) id = -1;
        t.qid[lane] = id;
        t.qxy[lane] = (id >= 0) ? xyb[id] : make_float2(0.f, 0.f);
    }
    __syncwarp();
    const size_t tok0 = static_cast<size_t>(b) * a.N;
    const int H = a.H;
#pragma unroll
    for (int c = lane; c < MT * 4; c += 32) {
        const int row = c >> 2, ch = c & 3;
        const int id = t.kid[row];
        const size_t off = ((tok0 + (id >= 0 ? id : 0)) * H + h) * 32 + ch * 8;
        cp_async16(smem_addr(t.ks) + tile64_off(row, ch), a.k + off, id >= 0);
        cp_async16(smem_addr(t.vs) + tile64_off(row, ch), a.v + off, id >= 0);
    }
    {
        const int row = lane >> 2, ch = lane & 3;
        const int id = t.qid[row];
        const size_t off = ((tok0 + (id >= 0 ? id : 0)) * H + h) * 32 + ch * 8;
        cp_async16(smem_addr(t.qs) + tile64_off(row, ch), qsrc + off, id >= 0);
    }
}

// S^T = K . Q^T for all MT/16 key tiles (raw dot products).
template <int MTILES>
__device__ __forceinline__ void qk_tiles(float (&s)[MTILES][4], const uint8_t* ks, uint32_t qf0,
                                         uint32_t qf1, uint32_t qf2, uint32_t qf3, int lane) {
    const int mi = lane >> 3;
#pragma unroll
    for (int i = 0; i < MTILES; ++i) {
        s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
            const int row = 16 * i + (lane & 7) + 8 * (mi & 1);
            const int ch = 2 * kk + (mi >> 1);
            uint32_t a0, a1, a2, a3;
            ldsm_x4(smem_addr(ks) + tile64_off(row, ch), a0, a1, a2, a3);
            mma_bf16(s[i], a0, a1, a2, a3, kk ? qf2 : qf0, kk ? qf3 : qf1);
        }
    }
}

// acc^T (32 x 8) += X^T (32 x MT) . B^T where X is an MT x 32 row tile and bfr holds the
// transposed (k-major) B fragments of the MT x 8 matrix.
template <int MTILES>
__device__ __forceinline__ void xt_b(float (&acc)[2][4], const uint8_t* xs,
                                     const uint32_t (&bfr)[MTILES][2], int lane) {
    const int mi = lane >> 3;
#pragma unroll
    for (int m = 0; m < 2; ++m) {
        acc[m][0] = acc[m][1] = acc[m][2] = acc[m][3] = 0.f;
#pragma unroll
        for (int i = 0; i < MTILES; ++i) {
            const int row = 16 * i + (lane & 7) + 8 * (mi >> 1);
            const int ch = 2 * m + (mi & 1);
            uint32_t a0, a1, a2, a3;
            ldsm_x4_t(smem_addr(xs) + tile64_off(row, ch), a0, a1, a2, a3);
            mma_bf16(acc[m], a0, a1, a2, a3, bfr[i][0], bfr[i][1]);
        }
    }
}

// Same as xt_b with B = B_hi + B_lo given as two bf16 fragment sets (a split that keeps
// about 16 significant bits of B): each A fragment is loaded once and used twice.
template <int MTILES>
__device__ __forceinline__ void xt_b2(float (&acc)[2][4], const uint8_t* xs,
                                      const uint32_t (&bhi)[MTILES][2],
                                      const uint32_t (&blo)[MTILES][2], int lane) {
    const int mi = lane >> 3;
#pragma unroll
    for (int m = 0; m < 2; ++m) {
        acc[m][0] = acc[m][1] = acc[m][2] = acc[m][3] = 0.f;
#pragma unroll
        for (int i = 0; i < MTILES; ++i) {
            const int row = 16 * i + (lane & 7) + 8 * (mi >> 1);
            const int ch = 2 * m + (mi & 1);
            uint32_t a0, a1, a2, a3;
            ldsm_x4_t(smem_addr(xs) + tile64_off(row, ch), a0, a1, a2, a3);
            mma_bf16(acc[m], a0, a1, a2, a3, blo[i][0], blo[i][1]);
            mma_bf16(acc[m], a0, a1, a2, a3, bhi[i][0], bhi[i][1]);
        }
    }
}

// bf16 pair (hi) of two floats and the bf16 pair of their remainders (lo).
__device__ __forceinline__ void split_bf16(float x0, float x1, uint32_t& hi, uint32_t& lo) {
    hi = pack_bf16(x0, x1);
    lo = pack_bf16(x0 - bf16_lo(hi), x1 - bf16_hi(hi));
}

// Write an (e x 8-token) fp32 accumulator pair, transposed to token rows, as bf16 rows of
// `dst` (token-major [tok][H][32]) through a 512-byte staging tile.
__device__ __forceinline__ void store_rows_t(const float (&acc)[2][4], float s0, float s1,
                                             uint8_t* stage, const int* ids, size_t tok0, int H,
                                             int h, bf16* dst, int lane) {
    const int gq = lane >> 2, tq = lane & 3;
    const uint32_t w0 = movm_t(pack_bf16(acc[0][0] * s0, acc[0][1] * s1));
    const uint32_t w1 = movm_t(pack_bf16(acc[0][2] * s0, acc[0][3] * s1));
    const uint32_t w2 = movm_t(pack_bf16(acc[1][0] * s0, acc[1][1] * s1));
    const uint32_t w3 = movm_t(pack_bf16(acc[1][2] * s0, acc[1][3] * s1));
    __syncwarp();
    uint32_t* row = reinterpret_cast<uint32_t*>(stage + gq * 64);
    row[tq] = w0;
    row[4 + tq] = w1;
    row[8 + tq] = w2;
    row[12 + tq] = w3;
    __syncwarp();
    const int r = lane >> 2, ch = lane & 3;
    const int id = ids[r];
    if (id >= 0) {
        const uint4 v = *reinterpret_cast<const uint4*>(stage + r * 64 + ch * 16);
        *reinterpret_cast<uint4*>(dst + ((tok0 + id) * H + h) * 32 + ch * 8) = v;
    }
    __syncwarp();
}

// Same, for key-major accumulators whose per-column scale is uniform.
__device__ __forceinline__ void store_rows_t1(const float (&acc)[2][4], float s, uint8_t* stage,
                                              const int* ids, size_t tok0, int H, int h, bf16* dst,
                                              int lane) {
    store_rows_t(acc, s, s, stage, ids, tok0, H, h, dst, lane);
}

// --------------------------------------------------------------- forward

template <int MTILES>
__global__ void __launch_bounds__(kThreads) attn_fwd_kernel(const AttnArgs a) {
    constexpr int MT = 16 * MTILES;
    extern __shared__ __align__(16) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long task = static_cast<long long>(blockIdx.x) * kWarps + warp;
    if (task >= static_cast<long long>(a.B) * a.G * a.H) return;
    const int h = static_cast<int>(task % a.H);
    const long long bg = task / a.H;
    const int g = static_cast<int>(bg % a.G), b = static_cast<int>(bg / a.G);
    const FwdTiles t = fwd_tiles(smem + warp * fwd_warp_bytes(MT), MT);
    const size_t tok0 = static_cast<size_t>(b) * a.N;

    load_cluster_tiles<MT>(a, b, g, h, lane, t, a.q);
    cp_async_commit();
    cp_async_wait<0>();
    __syncwarp();

    const int gq = lane >> 2, tq = lane & 3;
    uint32_t qf0, qf1, qf2, qf3;
    ldsm_x4(smem_addr(t.qs) + tile64_off(lane & 7, lane >> 3), qf0, qf1, qf2, qf3);
    float s[MTILES][4];
    qk_tiles<MTILES>(s, t.ks, qf0, qf1, qf2, qf3, lane);

    // logits in log2 units
    const float sc = a.scale * kLog2e;
    const float ba = a.bias[3 * h] * kLog2e, bb = a.bias[3 * h + 1] * kLog2e,
                bc = a.bias[3 * h + 2] * kLog2e;
    const float2 qa = t.qxy[2 * tq], qb = t.qxy[2 * tq + 1];
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int i = 0; i < MTILES; ++i) {
#pragma unroll
        for (int hi = 0; hi < 2; ++hi) {
            const int key = 16 * i + gq + 8 * hi;
            const bool kv = t.kid[key] >= 0;
            const float2 kp = t.kxy[key];
            float dx = kp.x - qa.x, dy = kp.y - qa.y;
            const float v0 = s[i][2 * hi] * sc + ba * dx + bb * dy - bc * (dx * dx + dy * dy);
            dx = kp.x - qb.x;
            dy = kp.y - qb.y;
            const float v1 = s[i][2 * hi + 1] * sc + ba * dx + bb * dy - bc * (dx * dx + dy * dy);
            s[i][2 * hi] = kv ? v0 : -INFINITY;
            s[i][2 * hi + 1] = kv ? v1 : -INFINITY;
            mx0 = fmaxf(mx0, s[i][2 * hi]);
            mx1 = fmaxf(mx1, s[i][2 * hi + 1]);
        }
    }
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
    }
    const float m0 = (mx0 == -INFINITY) ? 0.f : mx0;
    const float m1 = (mx1 == -INFINITY) ? 0.f : mx1;
    float l0 = 0.f, l1 = 0.f;
    uint32_t pbh[MTILES][2], pbl[MTILES][2];
#pragma unroll
    for (int i = 0; i < MTILES; ++i) {
        const float p0 = exp2f(s[i][0] - m0), p1 = exp2f(s[i][1] - m1);
        const float p2 = exp2f(s[i][2] - m0), p3 = exp2f(s[i][3] - m1);
        l0 += p0 + p2;
        l1 += p1 + p3;
        uint32_t h01, l01, h23, l23;
        split_bf16(p0, p1, h01, l01);
        split_bf16(p2, p3, h23, l23);
        pbh[i][0] = movm_t(h01);
        pbl[i][0] = movm_t(l01);
        pbh[i][1] = movm_t(h23);
        pbl[i][1] = movm_t(l23);
    }
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
        l0 += __shfl_xor_sync(0xffffffffu, l0, o);
        l1 += __shfl_xor_sync(0xffffffffu, l1, o);
    }
    // P is split into bf16 hi + lo parts so that rounding P costs ~2^-17 relative
    // instead of 2^-9; the output's own bf16 rounding is then the only visible error.
    float oacc[2][4];
    xt_b2<MTILES>(oacc, t.vs, pbh, pbl, lane);
    const float i0 = l0 > 0.f ? 1.f / l0 : 0.f;
    const float i1 = l1 > 0.f ? 1.f / l1 : 0.f;
    store_rows_t(oacc, i0, i1, t.qs, t.qid, tok0, a.H, h, a.o, lane);
    if (gq == 0) {
        const int q0 = t.qid[2 * tq], q1 = t.qid[2 * tq + 1];
        if (q0 >= 0)
            a.lse[(tok0 + q0) * a.H + h] = l0 > 0.f ? (m0 + log2f(l0)) * kLn2 : -INFINITY;
        if (q1 >= 0)
            a.lse[(tok0 + q1) * a.H + h] = l1 > 0.f ? (m1 + log2f(l1)) * kLn2 : -INFINITY;
    }
}

// ------------------------------------------------------ block-wide int scan

// In-place exclusive prefix sum of data[0..n) by all threads of the block; returns the total.
__device__ int block_scan_excl(int* data, int n, int* scratch) {
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

// Reverse neighbourhood index of image b: for each key cluster h, the query clusters g
// whose table lists h, ascending in g.  Runs in one CTA; dynamic smem >= 4*(G+1)+160 B.
__device__ void build_reverse_index(const AttnArgs& a, int b, uint8_t* smem) {
    const int tid = threadIdx.x, nt = blockDim.x;
    const int N = a.N, G = a.G, R = a.R, M = a.M;
    int* cnt = reinterpret_cast<int*>(smem);
    int* scratch = cnt + G + 1;
    int32_t* tc = a.tok_cluster + static_cast<size_t>(b) * N;
    const int32_t* cl = a.clusters + static_cast<size_t>(b) * G * 8;
    const int32_t* nb = a.nbr + static_cast<size_t>(b) * G * M;
    int32_t* off = a.rev_off + static_cast<size_t>(b) * (G + 1);
    int32_t* lst = a.rev_list + static_cast<size_t>(b) * G * R;
    for (int i = tid; i < N; i += nt) tc[i] = -1;
    for (int i = tid; i <= G; i += nt) cnt[i] = 0;
    __syncthreads();
    for (int i = tid; i < G * 8; i += nt) {
        const int t = cl[i];
        if (t >= 0 && t < N) tc[t] = i >> 3;
    }
    __syncthreads();
    for (int e = tid; e < G * R; e += nt) {
        const int t0 = nb[static_cast<size_t>(e / R) * M + (e % R) * 8];
        const int h = (t0 >= 0 && t0 < N) ? tc[t0] : -1;
        if (h >= 0) atomicAdd(&cnt[h], 1);
    }
    __syncthreads();
    const int total = block_scan_excl(cnt, G, scratch);
    for (int i = tid; i < G; i += nt) off[i] = cnt[i];
    if (tid == 0) off[G] = total;
    __syncthreads();
    for (int e = tid; e < G * R; e += nt) {
        const int t0 = nb[static_cast<size_t>(e / R) * M + (e % R) * 8];
        const int h = (t0 >= 0 && t0 < N) ? tc[t0] : -1;
        if (h >= 0) lst[atomicAdd(&cnt[h], 1)] = e / R;
    }
    __syncthreads();
    // cnt[h] is now the end of list h; sort every list so the order is fixed
    for (int h = tid; h < G; h += nt) {
        const int lo = h > 0 ? cnt[h - 1] : 0, hi = cnt[h];
        for (int i = lo + 1; i < hi; ++i) {
            const int v = lst[i];
            int j = i - 1;
            while (j >= lo && lst[j] > v) {
                lst[j + 1] = lst[j];
                --j;
            }
            lst[j + 1] = v;
        }
    }
}

// ---------------------------------------------------- backward, query-major

template <int MTILES>
__global__ void __launch_bounds__(kThreads) attn_bwd_query_kernel(const AttnArgs a, int task_blocks) {
    constexpr int MT = 16 * MTILES;
    extern __shared__ __align__(16) uint8_t smem[];
    if (static_cast<int>(blockIdx.x) >= task_blocks) {
        build_reverse_index(a, blockIdx.x - task_blocks, smem);
        return;
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long task = static_cast<long long>(blockIdx.x) * kWarps + warp;
    if (task >= static_cast<long long>(a.B) * a.G * a.H) return;
    const int h = static_cast<int>(task % a.H);
    const long long bg = task / a.H;
    const int g = static_cast<int>(bg % a.G), b = static_cast<int>(bg / a.G);
    uint8_t* w = smem + warp * bwdq_warp_bytes(MT);
    const FwdTiles t = fwd_tiles(w, MT);
    uint8_t* dos = w + fwd_warp_bytes(MT);
    const size_t tok0 = static_cast<size_t>(b) * a.N;
    const int H = a.H;

    load_cluster_tiles<MT>(a, b, g, h, lane, t, a.q);
    {
        const int row = lane >> 2, ch = lane & 3;
        const int id = t.qid[row];
        const size_t off = ((tok0 + (id >= 0 ? id : 0)) * H + h) * 32 + ch * 8;
        cp_async16(smem_addr(dos) + tile64_off(row, ch), a.dout + off, id >= 0);
    }
    cp_async_commit();
    cp_async_wait<0>();
    __syncwarp();

    const int gq = lane >> 2, tq = lane & 3;
    const int q0 = t.qid[2 * tq], q1 = t.qid[2 * tq + 1];
    float L0 = q0 >= 0 ? a.lse_in[(tok0 + q0) * H + h] * kLog2e : INFINITY;
    float L1 = q1 >= 0 ? a.lse_in[(tok0 + q1) * H + h] * kLog2e : INFINITY;
    if (L0 == -INFINITY) L0 = INFINITY;  // empty neighbourhood: P = 0
    if (L1 == -INFINITY) L1 = INFINITY;

    uint32_t qf0, qf1, qf2, qf3, df0, df1, df2, df3;
    ldsm_x4(smem_addr(t.qs) + tile64_off(lane & 7, lane >> 3), qf0, qf1, qf2, qf3);
    ldsm_x4(smem_addr(dos) + tile64_off(lane & 7, lane >> 3), df0, df1, df2, df3);
    float s[MTILES][4], dp[MTILES][4];
    qk_tiles<MTILES>(s, t.ks, qf0, qf1, qf2, qf3, lane);
    qk_tiles<MTILES>(dp, t.vs, df0, df1, df2, df3, lane);

    const float sc = a.scale * kLog2e;
    const float ba = a.bias[3 * h] * kLog2e, bb = a.bias[3 * h + 1] * kLog2e,
                bc = a.bias[3 * h + 2] * kLog2e;
    const float2 qa = t.qxy[2 * tq], qb = t.qxy[2 * tq + 1];
    // P from the forward's lse; Delta_i = sum_j P_ij dP_ij (= <dO_i, O_i> exactly, since
    // the whole key row is in this tile -- no bf16-rounded O enters the gradient)
    float pd0 = 0.f, pd1 = 0.f;
#pragma unroll
    for (int i = 0; i < MTILES; ++i) {
#pragma unroll
        for (int hi = 0; hi < 2; ++hi) {
            const int key = 16 * i + gq + 8 * hi;
            const bool kv = t.kid[key] >= 0;
            const float2 kp = t.kxy[key];
#pragma unroll
            for (int qq = 0; qq < 2; ++qq) {
                const float2 qp = qq ? qb : qa;
                const float dx = kp.x - qp.x, dy = kp.y - qp.y;
                const int j = 2 * hi + qq;
                const float lg = s[i][j] * sc + ba * dx + bb * dy - bc * (dx * dx + dy * dy);
                const float p = kv ? exp2f(lg - (qq ? L1 : L0)) : 0.f;
                s[i][j] = p;
                if (qq) pd1 += p * dp[i][j];
                else pd0 += p * dp[i][j];
            }
        }
    }
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
        pd0 += __shfl_xor_sync(0xffffffffu, pd0, o);
        pd1 += __shfl_xor_sync(0xffffffffu, pd1, o);
    }
    if (gq == 0) {
        if (q0 >= 0) a.delta[(tok0 + q0) * H + h] = pd0;
        if (q1 >= 0) a.delta[(tok0 + q1) * H + h] = pd1;
    }
    float ga = 0.f, gb = 0.f, gc = 0.f;
    uint32_t db[MTILES][2];
#pragma unroll
    for (int i = 0; i < MTILES; ++i) {
        float ds[4];
#pragma unroll
        for (int hi = 0; hi < 2; ++hi) {
            const int key = 16 * i + gq + 8 * hi;
            const float2 kp = t.kxy[key];
#pragma unroll
            for (int qq = 0; qq < 2; ++qq) {
                const float2 qp = qq ? qb : qa;
                const float dx = kp.x - qp.x, dy = kp.y - qp.y;
                const int j = 2 * hi + qq;
                const float v = s[i][j] * (dp[i][j] - (qq ? pd1 : pd0));
                ds[j] = v;
                ga += v * dx;
                gb += v * dy;
                gc += v * (dx * dx + dy * dy);
            }
        }
        db[i][0] = movm_t(pack_bf16(ds[0], ds[1]));
        db[i][1] = movm_t(pack_bf16(ds[2], ds[3]));
    }
    ga = warp_sum(ga);
    gb = warp_sum(gb);
    gc = warp_sum(gc);
    if (lane == 0) {
        float* part = a.dbias_part + ((static_cast<size_t>(b) * a.G + g) * H + h) * 3;
        part[0] = ga;
        part[1] = gb;
        part[2] = -gc;
    }
    float dqacc[2][4];
    xt_b<MTILES>(dqacc, t.ks, db, lane);
    store_rows_t(dqacc, a.scale, a.scale, t.qs, t.qid, tok0, H, h, a.dq, lane);
}

// ------------------------------------------------------ backward, key-major

__global__ void __launch_bounds__(kThreads) attn_bwd_key_kernel(const AttnArgs a, int task_blocks) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (static_cast<int>(blockIdx.x) >= task_blocks) {
        // bias-gradient reduction: one CTA per (head, coefficient), fixed order
        const int hj = blockIdx.x - task_blocks;
        const int hh = hj / 3, j = hj % 3;
        const int n = a.B * a.G;
        float acc = 0.f;
#pragma unroll 4
        for (int i = threadIdx.x; i < n; i += kThreads)
            acc += a.dbias_part[(static_cast<size_t>(i) * a.H + hh) * 3 + j];
        acc = warp_sum(acc);
        float* red = reinterpret_cast<float*>(smem);
        if (lane == 0) red[warp] = acc;
        __syncthreads();
        if (threadIdx.x == 0) {
            float tot = 0.f;
            for (int w = 0; w < kWarps; ++w) tot += red[w];
            a.dbias[hh * 3 + j] = tot;
        }
        return;
    }
    const long long task = static_cast<long long>(blockIdx.x) * kWarps + warp;
    if (task >= static_cast<long long>(a.B) * a.G * a.H) return;
    const int h = static_cast<int>(task % a.H);
    const long long bk = task / a.H;
    const int kc = static_cast<int>(bk % a.G), b = static_cast<int>(bk / a.G);
    const int H = a.H;
    const size_t tok0 = static_cast<size_t>(b) * a.N;
    const float2* xyb = reinterpret_cast<const float2*>(a.xy) + tok0;

    uint8_t* w = smem + warp * kBwdKWarpBytes;
    uint8_t* ks = w;            // 8 rows
    uint8_t* vs = w + 512;      // 8 rows
    uint8_t* qs = w + 1024;     // 16 rows
    uint8_t* dos = w + 2048;    // 16 rows
    int* kid = reinterpret_cast<int*>(w + 3072);
    float2* kxy = reinterpret_cast<float2*>(w + 3104);
    int* qid = reinterpret_cast<int*>(w + 3168);
    float2* qxy = reinterpret_cast<float2*>(w + 3232);
    float* qL = reinterpret_cast<float*>(w + 3360);
    float* qD = reinterpret_cast<float*>(w + 3424);

    if (lane < 8) {
        int id = a.clusters[(static_cast<size_t>(b) * a.G + kc) * 8 + lane];
        if (id < 0 || id >= a.N) id = -1;
        kid[lane] = id;
        kxy[lane] = id >= 0 ? xyb[id] : make_float2(0.f, 0.f);
    }
    __syncwarp();
    {
        const int row = lane >> 2, ch = lane & 3;
        const int id = kid[row];
        const size_t off = ((tok0 + (id >= 0 ? id : 0)) * H + h) * 32 + ch * 8;
        cp_async16(smem_addr(ks) + tile64_off(row, ch), a.k + off, id >= 0);
        cp_async16(smem_addr(vs) + tile64_off(row, ch), a.v + off, id >= 0);
    }
    cp_async_commit();
    cp_async_wait<0>();
    __syncwarp();
    uint32_t kf0, kf1, kf2, kf3, vf0, vf1, vf2, vf3;
    ldsm_x4(smem_addr(ks) + tile64_off(lane & 7, lane >> 3), kf0, kf1, kf2, kf3);
    ldsm_x4(smem_addr(vs) + tile64_off(lane & 7, lane >> 3), vf0, vf1, vf2, vf3);

    const int gq = lane >> 2, tq = lane & 3;
    const float sc = a.scale * kLog2e;
    const float ba = a.bias[3 * h] * kLog2e, bb = a.bias[3 * h + 1] * kLog2e,
                bc = a.bias[3 * h + 2] * kLog2e;
    const float2 kp0 = kxy[2 * tq], kp1 = kxy[2 * tq + 1];
    const int lo = a.rev_off[static_cast<size_t>(b) * (a.G + 1) + kc];
    const int hi_ = a.rev_off[static_cast<size_t>(b) * (a.G + 1) + kc + 1];
    const int32_t* lst = a.rev_list + static_cast<size_t>(b) * a.G * a.R;
    float dk[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    float dv[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    const int mi = lane >> 3;

    for (int e = lo; e < hi_; e += 2) {
        if (lane < 16) {
            const int gg = (lane < 8) ? lst[e] : (e + 1 < hi_ ? lst[e + 1] : -1);
            int id = gg >= 0 ? a.clusters[(static_cast<size_t>(b) * a.G + gg) * 8 + (lane & 7)] : -1;
            if (id < 0 || id >= a.N) id = -1;
            qid[lane] = id;
            qxy[lane] = id >= 0 ? xyb[id] : make_float2(0.f, 0.f);
            float L = id >= 0 ? a.lse_in[(tok0 + id) * H + h] * kLog2e : INFINITY;
            if (L == -INFINITY) L = INFINITY;
            qL[lane] = L;
            qD[lane] = id >= 0 ? a.delta[(tok0 + id) * H + h] : 0.f;
        }
        __syncwarp();
#pragma unroll
        for (int c = lane; c < 64; c += 32) {
            const int row = c >> 2, ch = c & 3;
            const int id = qid[row];
            const size_t off = ((tok0 + (id >= 0 ? id : 0)) * H + h) * 32 + ch * 8;
            cp_async16(smem_addr(qs) + tile64_off(row, ch), a.q + off, id >= 0);
            cp_async16(smem_addr(dos) + tile64_off(row, ch), a.dout + off, id >= 0);
        }
        cp_async_commit();
        cp_async_wait<0>();
        __syncwarp();

        float sacc[4] = {0.f, 0.f, 0.f, 0.f}, pacc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
            const int row = (lane & 7) + 8 * (mi & 1);
            const int ch = 2 * kk + (mi >> 1);
            uint32_t a0, a1, a2, a3;
            ldsm_x4(smem_addr(qs) + tile64_off(row, ch), a0, a1, a2, a3);
            mma_bf16(sacc, a0, a1, a2, a3, kk ? kf2 : kf0, kk ? kf3 : kf1);
            ldsm_x4(smem_addr(dos) + tile64_off(row, ch), a0, a1, a2, a3);
            mma_bf16(pacc, a0, a1, a2, a3, kk ? vf2 : vf0, kk ? vf3 : vf1);
        }
        // element j: query row gq + 8*(j>>1), key 2*tq + (j&1)
        float p[4], ds[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int qr = gq + 8 * (j >> 1);
            const float2 qp = qxy[qr];
            const float2 kp = (j & 1) ? kp1 : kp0;
            const float dx = kp.x - qp.x, dy = kp.y - qp.y;
            const float lg = sacc[j] * sc + ba * dx + bb * dy - bc * (dx * dx + dy * dy);
            p[j] = exp2f(lg - qL[qr]);
            ds[j] = p[j] * (pacc[j] - qD[qr]);
        }
        const uint32_t pb0 = movm_t(pack_bf16(p[0], p[1]));
        const uint32_t pb1 = movm_t(pack_bf16(p[2], p[3]));
        const uint32_t sb0 = movm_t(pack_bf16(ds[0], ds[1]));
        const uint32_t sb1 = movm_t(pack_bf16(ds[2], ds[3]));
#pragma unroll
        for (int m = 0; m < 2; ++m) {
            const int row = (lane & 7) + 8 * (mi >> 1);
            const int ch = 2 * m + (mi & 1);
            uint32_t a0, a1, a2, a3;
            ldsm_x4_t(smem_addr(dos) + tile64_off(row, ch), a0, a1, a2, a3);
            mma_bf16(dv[m], a0, a1, a2, a3, pb0, pb1);
            ldsm_x4_t(smem_addr(qs) + tile64_off(row, ch), a0, a1, a2, a3);
            mma_bf16(dk[m], a0, a1, a2, a3, sb0, sb1);
        }
        __syncwarp();
    }
    store_rows_t1(dk, a.scale, qs, kid, tok0, H, h, a.dk, lane);
    store_rows_t1(dv, 1.f, qs, kid, tok0, H, h, a.dv, lane);
}

template <int MTILES>
cudaError_t fwd_dispatch(const AttnArgs& a, cudaStream_t st) {
    const size_t smem = static_cast<size_t>(kWarps) * fwd_warp_bytes(16 * MTILES);
    const long long tasks = static_cast<long long>(a.B) * a.G * a.H;
    const long long blocks = (tasks + kWarps - 1) / kWarps;
    attn_fwd_kernel<MTILES><<<static_cast<unsigned>(blocks), kThreads, smem, st>>>(a);
    note_launch();
    return cudaGetLastError();
}

template <int MTILES>
cudaError_t bwd_dispatch(const AttnArgs& a, cudaStream_t st) {
    const long long tasks = static_cast<long long>(a.B) * a.G * a.H;
    const int blocks = static_cast<int>((tasks + kWarps - 1) / kWarps);
    size_t smem = static_cast<size_t>(kWarps) * bwdq_warp_bytes(16 * MTILES);
    const size_t prep = 4 * static_cast<size_t>(a.G + 1) + 160;
    if (prep > smem) smem = prep;
    cudaError_t e = ensure_smem<attn_bwd_query_kernel<MTILES>>(smem);
    if (e != cudaSuccess) return e;
    attn_bwd_query_kernel<MTILES><<<blocks + a.B, kThreads, smem, st>>>(a, blocks);
    note_launch();
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const size_t smem2 = static_cast<size_t>(kWarps) * kBwdKWarpBytes;
    attn_bwd_key_kernel<<<blocks + 3 * a.H, kThreads, smem2, st>>>(a, blocks);
    note_launch();
    return cudaGetLastError();
}

}  // namespace

AttnWorkspace attn_workspace_layout(int B, int N, int H, int C, int M) {
    const size_t G = static_cast<size_t>((N + C - 1) / C);
    const size_t R = static_cast<size_t>(M / C);
    auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
    AttnWorkspace w;
    size_t off = 0;
    w.delta = off;       off += up(sizeof(float) * B * static_cast<size_t>(N) * H);
    w.dbias_part = off;  off += up(sizeof(float) * B * G * H * 3);
    w.tok_cluster = off; off += up(sizeof(int32_t) * B * static_cast<size_t>(N));
    w.rev_off = off;     off += up(sizeof(int32_t) * B * (G + 1));
    w.rev_list = off;    off += up(sizeof(int32_t) * B * G * R);
    w.total = off;
    return w;
}

cudaError_t launch_attn_fwd(const AttnArgs& a, cudaStream_t st) {
    switch ((a.M + 15) / 16) {
        case 1: return fwd_dispatch<1>(a, st);
        case 2: return fwd_dispatch<2>(a, st);
        case 3: return fwd_dispatch<3>(a, st);
        default: return fwd_dispatch<4>(a, st);
    }
}

cudaError_t launch_attn_bwd(const AttnArgs& a, cudaStream_t st) {
    switch ((a.M + 15) / 16) {
        case 1: return bwd_dispatch<1>(a, st);
        case 2: return bwd_dispatch<2>(a, st);
        case 3: return bwd_dispatch<3>(a, st);
        default: return bwd_dispatch<4>(a, st);
    }
}

}  // namespace acl
