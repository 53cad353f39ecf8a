// attn.cu -- local cluster attention, forward and backward (bf16 in, fp32 math).
//
// AFFMAE notes, Method "Overall Architecture" (stages of Local Cluster Attention
// over local balanced clusters); arXiv abstract page (Flash-style, numerically
// stable mixed-precision cluster attention kernels).  Per token i of cluster g and
// head h, over the keys j of nbr[g]:
//   s_ij = scale <q_i, k_j> + a_h dx + b_h dy - c_h (dx^2 + dy^2),  dx = x_j - x_i,
//   O_i = softmax_j(s_ij) V,  lse_i = log sum_j exp(s_ij).
//
// Work decomposition: every warp is an independent, persistent pipeline.  An item is one
// (image, cluster, head); a warp walks a contiguous range of items, cluster-major, so it
// takes consecutive heads of a cluster and then the next cluster.  Per item it gathers
// the cluster's M key rows of K and V and its 8 query rows of Q (64 bytes = one head of
// one token each) with 16-byte cp.async into one of two private stages, in slot order,
// while the previous item computes; the neighbour rows and coordinates of the clusters
// ahead are fetched into registers one and two clusters early.  No barrier, no shared
// state between warps: the only waits are the warp's own copies.
//
// Per warp and item: the cluster's 8 queries against its M <= 64 keys, D = 32, on the
// tensor cores as m16n8k16 bf16 MMAs with the operands swapped so that the 8 queries
// sit on the MMA's N = 8 side and keys on M (no padded rows):
//   S^T (M x 8)  = K (M x 32) . Q^T
//   O^T (32 x 8) = V^T (32 x M) . P^T        (P^T from the S^T accumulators by an
//                                             in-register 8x8 transpose, movmatrix;
//                                             P carried as bf16 hi + lo, ~16 bits)
//   l   (1 x 8)  = 1^T . P^T                 (row sums as one more MMA row)
// The bias is expanded around a local origin so that it costs three FMAs per score:
//   a dx + b dy - c (dx^2 + dy^2) = u_j + 2c x_i x_j + 2c y_i y_j + w_i,
//   u_j = a x_j + b y_j - c (x_j^2 + y_j^2),  w_i = -a x_i - b y_i - c (x_i^2 + y_i^2);
// w_i is constant along the softmax row, so it drops out of P and is added to lse.
//
// Backward (recompute, FA2-style, no atomics, every sum in a fixed order):
//   prep (one CTA per image): the reverse neighbourhood index -- for every key cluster,
//     the query clusters that list it, ascending, and their tokens.
//   query pass (the forward's items): P = exp(s - lse), dP^T = V . dO^T,
//     Delta_i = sum_j P dP (equal to <dO_i, O_i>, exact in fp32 because the whole key
//     row is in the tile, so O is not read), dS = P (dP - Delta), dQ^T = K^T . dS^T,
//     per-(cluster, head) partial sums of the bias gradient.
//   key pass: an item is (image, key cluster, head, chunk of up to kChunk listed query
//     clusters); the warp gathers its own K and V rows and the chunk's Q and dO rows and
//     walks the chunk two query clusters at a time (16 queries = one MMA M tile):
//     S = Q K^T, dP = dO V^T, dV^T += dO^T P, dK^T += Q^T dS, the sums carried over the
//     chunks of a (key cluster, head) in list order.  Extra CTAs reduce the bias partials
//     in a fixed order.
#include <math.h>

#include "internal.h"

namespace acl {

namespace {

constexpr int kWarps = 4;               // warps per CTA (independent pipelines)
constexpr int kThreads = 32 * kWarps;
constexpr int kRowB = 64;               // bytes of one head of one token (32 bf16)
constexpr int kChunk = 4;               // listed query clusters per key-pass item
constexpr int kMaxPlanWarps = 8192;     // key-pass warps a workspace plan can describe

// ---------------------------------------------------------------- small helpers

__device__ __forceinline__ float sfu_ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float sfu_lg2(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float sfu_rcp(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
    return y;
}

// 4-byte global->shared copy; zero-filled when !valid.
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src, bool valid) {
    int n = valid ? 4 : 0;
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(dst), "l"(src), "r"(n)
                 : "memory");
}

// bf16 pair (hi) of two floats and the bf16 pair of their remainders (lo).
__device__ __forceinline__ void split_bf16(float x0, float x1, uint32_t& hi, uint32_t& lo) {
    hi = pack_bf16(x0, x1);
    lo = pack_bf16(x0 - bf16_lo(hi), x1 - bf16_hi(hi));
}

// Sum of three per-lane values over the warp with 9 shuffles: after the first two rounds
// lane l holds a partial of value (l >> 3) & 3 (value 3 is a dummy zero).
__device__ __forceinline__ void warp_sum3(float& x0, float& x1, float& x2, int lane) {
    const bool hi16 = lane & 16;
    float k0 = hi16 ? x2 : x0, k1 = hi16 ? 0.f : x1;
    const float s0 = hi16 ? x0 : x2, s1 = hi16 ? x1 : 0.f;
    k0 += __shfl_xor_sync(0xffffffffu, s0, 16);
    k1 += __shfl_xor_sync(0xffffffffu, s1, 16);
    const bool hi8 = lane & 8;
    float k = hi8 ? k1 : k0;
    const float s = hi8 ? k0 : k1;
    k += __shfl_xor_sync(0xffffffffu, s, 8);
    k += __shfl_xor_sync(0xffffffffu, k, 4);
    k += __shfl_xor_sync(0xffffffffu, k, 2);
    k += __shfl_xor_sync(0xffffffffu, k, 1);
    x0 = __shfl_sync(0xffffffffu, k, 0);
    x1 = __shfl_sync(0xffffffffu, k, 8);
    x2 = __shfl_sync(0xffffffffu, k, 16);
}

__device__ __forceinline__ int valid_tok(int t, int N) {
    ACL_DEVICE_CHECK(t >= -1 && t < N);
    return (t >= 0 && t < N) ? t : -1;
}

__device__ __forceinline__ float2 sh2(float2 v, int src) {
    return make_float2(__shfl_sync(0xffffffffu, v.x, src), __shfl_sync(0xffffffffu, v.y, src));
}

// Tiles are rows of 64 bytes (one head of one token) in slot order; the 16-byte chunk c of
// row r sits at r * 64 + ((c ^ ((r >> 1) & 3)) << 4) (tile64_off), so the 8 rows of every
// ldmatrix fall in 8 distinct bank groups.  Lane l gathers chunk l & 3 of rows
// (l >> 2) + 8 k; for those rows the swizzle depends on the lane only.
__device__ __forceinline__ uint32_t gather_lane_off(int lane) {
    return static_cast<uint32_t>((lane >> 2) * kRowB + (((lane & 3) ^ ((lane >> 3) & 3)) << 4));
}

// ldmatrix lane offsets (bytes) of the tiles in slot order, for sub-matrix mi = lane >> 3:
//   ls[kk]: rows 16 i + 8 (mi & 1) + (lane & 7), chunk 2 kk + (mi >> 1)  (A operand, + 1024 i)
//   lt[m]:  rows 16 i + 8 (mi >> 1) + (lane & 7), chunk 2 m + (mi & 1)   (transposed A, + 1024 i)
//   oq:     row lane & 7, chunk mi                                        (B operand, 8 rows)
struct LaneOffs {
    uint32_t ls0, ls1, lt0, lt1, oq;
};
__device__ __forceinline__ LaneOffs lane_offs(int lane) {
    const int mi = lane >> 3, r7 = lane & 7, sw = (r7 >> 1) & 3;
    LaneOffs o;
    o.ls0 = (mi & 1) * 512 + r7 * kRowB + (((0 + (mi >> 1)) ^ sw) << 4);
    o.ls1 = (mi & 1) * 512 + r7 * kRowB + (((2 + (mi >> 1)) ^ sw) << 4);
    o.lt0 = (mi >> 1) * 512 + r7 * kRowB + (((0 + (mi & 1)) ^ sw) << 4);
    o.lt1 = (mi >> 1) * 512 + r7 * kRowB + (((2 + (mi & 1)) ^ sw) << 4);
    o.oq = r7 * kRowB + ((mi ^ sw) << 4);
    return o;
}

// The tokens of one cluster's neighbourhood as a warp holds them: lane l has slots l and
// l + 32 of the neighbour row (a, b) and slot l of the cluster row (q, lanes < 8); raw
// values, made valid where used.
struct Toks {
    int a, b, q;
};
__device__ __forceinline__ Toks load_toks(const AttnArgs& a, int b, int g, int lane) {
    Toks t;
    const int32_t* nb = a.nbr + (static_cast<size_t>(b) * a.G + g) * a.M;
    t.a = lane < a.M ? __ldg(nb + lane) : -1;
    t.b = lane + 32 < a.M ? __ldg(nb + lane + 32) : -1;
    t.q = lane < 8 ? __ldg(a.clusters + (static_cast<size_t>(b) * a.G + g) * 8 + lane) : -1;
    return t;
}
// Their coordinates (zero for empty slots).
struct TokXY {
    float2 a, b, q;
};
__device__ __forceinline__ TokXY load_xy(const AttnArgs& a, int b, const Toks& t) {
    const float2* xyb = reinterpret_cast<const float2*>(a.xy) + static_cast<size_t>(b) * a.N;
    const int ta = valid_tok(t.a, a.N), tb = valid_tok(t.b, a.N), tq = valid_tok(t.q, a.N);
    TokXY x;
    x.a = ta >= 0 ? __ldg(xyb + ta) : make_float2(0.f, 0.f);
    x.b = tb >= 0 ? __ldg(xyb + tb) : make_float2(0.f, 0.f);
    x.q = tq >= 0 ? __ldg(xyb + tq) : make_float2(0.f, 0.f);
    return x;
}

// The next cluster after (b, g).
__device__ __forceinline__ void next_cluster(int& b, int& g, int G) {
    if (++g == G) {
        g = 0;
        ++b;
    }
}

// ------------------------------------------------------------- cluster items

// Per-warp stage of the forward (BWD = false) and query pass (BWD = true): the M key rows of
// K and V, the 8 query rows of Q (and dO), and the 8 queries' lse.
template <int MT, bool BWD>
struct QTile {
    static constexpr int K = 0;
    static constexpr int V = MT * kRowB;
    static constexpr int Q = 2 * MT * kRowB;
    static constexpr int DO = Q + 8 * kRowB;
    static constexpr int LSE = DO + (BWD ? 8 * kRowB : 0);
    static constexpr int STAGE = LSE + (BWD ? 32 : 0);
    static constexpr int WARP = 2 * STAGE;
};

// One cluster's rows as the gather needs them: the byte offsets of rows gq + 8 k and of
// query row gq in a [B][N][H][32] bf16 tensor (at head 0), and a bit per row that marks a
// token.  Off is 32-bit when every such tensor is smaller than 4 GiB.
template <int NK, typename Off>
struct Rows {
    Off ro[NK];
    Off rq;
    unsigned valid;  // bit k: row gq + 8 k; bit NK: query row gq
};
template <int NK, typename Off>
__device__ __forceinline__ Rows<NK, Off> cluster_rows(const AttnArgs& a, const Toks& t, int b, int lane) {
    Rows<NK, Off> r;
    const Off rowb = static_cast<Off>(a.H) * 64u;
    const Off base = static_cast<Off>(b) * static_cast<Off>(a.N);
    r.valid = 0u;
#pragma unroll
    for (int k = 0; k < NK; ++k) {
        const int tk = __shfl_sync(0xffffffffu, k < 4 ? t.a : t.b, (lane >> 2) + 8 * (k & 3));
        const bool ok = static_cast<unsigned>(tk) < static_cast<unsigned>(a.N);
        r.ro[k] = ok ? (base + static_cast<Off>(tk)) * rowb : Off(0);
        r.valid |= ok ? (1u << k) : 0u;
    }
    const int tq = __shfl_sync(0xffffffffu, t.q, lane >> 2);
    const bool okq = static_cast<unsigned>(tq) < static_cast<unsigned>(a.N);
    r.rq = okq ? (base + static_cast<Off>(tq)) * rowb : Off(0);
    r.valid |= okq ? (1u << NK) : 0u;
    return r;
}

// Gather head h of a cluster into the stage at sb (a shared address): K and V rows, the Q
// row (query pass: the dO row and the lse of the query too).
template <int MT, bool BWD, typename Off>
__device__ __forceinline__ void gather_cluster(const AttnArgs& a, int h, const Rows<MT / 8, Off>& r, uint32_t sb,
                                               int lane) {
    using T = QTile<MT, BWD>;
    const uint32_t lo = gather_lane_off(lane);
    const size_t hb = static_cast<size_t>(h) * 64 + (lane & 3) * 16;
    const char* kp = reinterpret_cast<const char*>(a.k) + hb;
    const char* vp = reinterpret_cast<const char*>(a.v) + hb;
#pragma unroll
    for (int k = 0; k < MT / 8; ++k) {
        const bool ok = (r.valid >> k) & 1u;
        cp_async16(sb + T::K + 512 * k + lo, kp + r.ro[k], ok);
        cp_async16(sb + T::V + 512 * k + lo, vp + r.ro[k], ok);
    }
    const bool okq = (r.valid >> (MT / 8)) & 1u;
    cp_async16(sb + T::Q + lo, reinterpret_cast<const char*>(a.q) + hb + r.rq, okq);
    if (BWD) {
        cp_async16(sb + T::DO + lo, reinterpret_cast<const char*>(a.dout) + hb + r.rq, okq);
        // lse[tok][h] = element (row byte offset / 64 bytes per head-row) + h
        if ((lane & 3) == 0)
            cp_async4(sb + T::LSE + 4 * (lane >> 2), a.lse_in + (static_cast<size_t>(r.rq) >> 6) + h, okq);
    }
}

// Per-lane geometry of one cluster, reused for every head: the lane's keys k = 2 i + hi
// (slot gq + 8 k) and query columns 2 tq, 2 tq + 1 in local coordinates (origin: the
// cluster's first slot), and the query tokens the lane writes (lanes < 8 write query
// `lane`'s lse / Delta).
template <int MTILES>
struct Geo {
    float kx[2 * MTILES], ky[2 * MTILES], kr[2 * MTILES];  // kr = kx^2 + ky^2
    unsigned kval;
    float qx[2], qy[2];
    float sx, sy;  // query `lane` (lanes < 8)
    int qo;        // query row gq (O / dQ rows)
    int qs;        // query `lane` (lanes < 8)
};

template <int MTILES>
__device__ __forceinline__ Geo<MTILES> make_geo(const Toks& t, const TokXY& x, unsigned valid, int lane, int N) {
    const int gq = lane >> 2, tq = lane & 3;
    Geo<MTILES> g;
    const float2 o = sh2(x.q, 0);
    g.kval = valid;
#pragma unroll
    for (int k = 0; k < 2 * MTILES; ++k) {
        const float2 p = sh2(k < 4 ? x.a : x.b, gq + 8 * (k & 3));
        const bool ok = (valid >> k) & 1u;
        g.kx[k] = ok ? p.x - o.x : 0.f;
        g.ky[k] = ok ? p.y - o.y : 0.f;
        g.kr[k] = fmaf(g.kx[k], g.kx[k], g.ky[k] * g.ky[k]);
    }
#pragma unroll
    for (int c = 0; c < 2; ++c) {
        const float2 p = sh2(x.q, 2 * tq + c);
        g.qx[c] = p.x - o.x;
        g.qy[c] = p.y - o.y;
    }
    g.sx = x.q.x - o.x;
    g.sy = x.q.y - o.y;
    g.qs = valid_tok(t.q, N);
    // bits 16 + s: query slot s holds a token
    g.kval |= __ballot_sync(0xffffffffu, lane < 8 && g.qs >= 0) << 16;
    g.qo = valid_tok(__shfl_sync(0xffffffffu, t.q, gq), N);
    return g;
}

// ------------------------------------------------------------------ forward

template <int MTILES>
__device__ __forceinline__ void fwd_item(const AttnArgs& a, size_t tok0, int h, uint32_t sb, const LaneOffs& lo,
                                         const Geo<MTILES>& g, int lane) {
    using T = QTile<16 * MTILES, false>;
    const int gq = lane >> 2, tq = lane & 3;
    const uint32_t kb = sb + T::K, vb = sb + T::V, qb = sb + T::Q;
    const float an = __ldg(a.bias + 3 * h), bn = __ldg(a.bias + 3 * h + 1), cn = __ldg(a.bias + 3 * h + 2);
    const float a2 = an * kLog2e, b2 = bn * kLog2e, c2 = cn * kLog2e;
    const float sc = a.scale * kLog2e;
    float u[2 * MTILES];
#pragma unroll
    for (int k = 0; k < 2 * MTILES; ++k)
        u[k] = ((g.kval >> k) & 1u) ? fmaf(a2, g.kx[k], fmaf(b2, g.ky[k], -c2 * g.kr[k])) : -INFINITY;
    const float X[2] = {2.f * c2 * g.qx[0], 2.f * c2 * g.qx[1]};
    const float Y[2] = {2.f * c2 * g.qy[0], 2.f * c2 * g.qy[1]};

    uint32_t qf[4];
    ldsm_x4(qb + lo.oq, qf[0], qf[1], qf[2], qf[3]);
    float sacc[MTILES][4];
#pragma unroll
    for (int i = 0; i < MTILES; ++i) {
        sacc[i][0] = sacc[i][1] = sacc[i][2] = sacc[i][3] = 0.f;
        uint32_t r0, r1, r2, r3;
        ldsm_x4(kb + 1024 * i + lo.ls0, r0, r1, r2, r3);
        mma_bf16(sacc[i], r0, r1, r2, r3, qf[0], qf[1]);
        ldsm_x4(kb + 1024 * i + lo.ls1, r0, r1, r2, r3);
        mma_bf16(sacc[i], r0, r1, r2, r3, qf[2], qf[3]);
    }
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int i = 0; i < MTILES; ++i) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int k = 2 * i + (j >> 1), c = j & 1;
            const float t = fmaf(sacc[i][j], sc, fmaf(X[c], g.kx[k], fmaf(Y[c], g.ky[k], u[k])));
            sacc[i][j] = t;
            mx[c] = fmaxf(mx[c], t);
        }
    }
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
        mx[0] = fmaxf(mx[0], __shfl_xor_sync(0xffffffffu, mx[0], o));
        mx[1] = fmaxf(mx[1], __shfl_xor_sync(0xffffffffu, mx[1], o));
    }
    const float m0 = mx[0] == -INFINITY ? 0.f : mx[0];
    const float m1 = mx[1] == -INFINITY ? 0.f : mx[1];
    uint32_t ph[MTILES][2], pl[MTILES][2];
#pragma unroll
    for (int i = 0; i < MTILES; ++i) {
        const float p0 = sfu_ex2(sacc[i][0] - m0), p1 = sfu_ex2(sacc[i][1] - m1);
        const float p2 = sfu_ex2(sacc[i][2] - m0), p3 = sfu_ex2(sacc[i][3] - m1);
        uint32_t h01, l01, h23, l23;
        split_bf16(p0, p1, h01, l01);
        split_bf16(p2, p3, h23, l23);
        ph[i][0] = movm_t(h01);
        ph[i][1] = movm_t(h23);
        pl[i][0] = movm_t(l01);
        pl[i][1] = movm_t(l23);
    }
    float oacc[2][4], lacc[4] = {0.f, 0.f, 0.f, 0.f};
    const uint32_t ones = gq == 0 ? 0x3F803F80u : 0u;  // row 0 of the A operand = 1
#pragma unroll
    for (int m = 0; m < 2; ++m) {
        oacc[m][0] = oacc[m][1] = oacc[m][2] = oacc[m][3] = 0.f;
#pragma unroll
        for (int i = 0; i < MTILES; ++i) {
            uint32_t r0, r1, r2, r3;
            ldsm_x4_t(vb + 1024 * i + (m ? lo.lt1 : lo.lt0), r0, r1, r2, r3);
            mma_bf16(oacc[m], r0, r1, r2, r3, pl[i][0], pl[i][1]);
            mma_bf16(oacc[m], r0, r1, r2, r3, ph[i][0], ph[i][1]);
        }
    }
#pragma unroll
    for (int i = 0; i < MTILES; ++i) {
        mma_bf16(lacc, ones, 0u, ones, 0u, pl[i][0], pl[i][1]);
        mma_bf16(lacc, ones, 0u, ones, 0u, ph[i][0], ph[i][1]);
    }
    // lanes 0..3 hold l of columns 2 tq, 2 tq + 1
    const float l0 = __shfl_sync(0xffffffffu, lacc[0], tq);
    const float l1 = __shfl_sync(0xffffffffu, lacc[1], tq);
    const float i0 = l0 > 0.f ? sfu_rcp(l0) : 0.f;
    const float i1 = l1 > 0.f ? sfu_rcp(l1) : 0.f;
    // O^T (dims x queries) -> rows of O: after the transpose lane (g, t) holds dims
    // 2t, 2t + 1 (+ 8, + 16, + 24) of query g
    const uint32_t w0 = movm_t(pack_bf16(oacc[0][0] * i0, oacc[0][1] * i1));
    const uint32_t w1 = movm_t(pack_bf16(oacc[0][2] * i0, oacc[0][3] * i1));
    const uint32_t w2 = movm_t(pack_bf16(oacc[1][0] * i0, oacc[1][1] * i1));
    const uint32_t w3 = movm_t(pack_bf16(oacc[1][2] * i0, oacc[1][3] * i1));
    if (g.qo >= 0) {
        uint32_t* dst = reinterpret_cast<uint32_t*>(a.o + ((tok0 + g.qo) * a.H + h) * 32) + tq;
        dst[0] = w0;
        dst[4] = w1;
        dst[8] = w2;
        dst[12] = w3;
    }
    // lse of query `lane` (lanes < 8): its column max and sum sit at lane lane / 2
    {
        const int src = (lane >> 1) & 3;
        const float ma = __shfl_sync(0xffffffffu, m0, src), mb = __shfl_sync(0xffffffffu, m1, src);
        const float la = __shfl_sync(0xffffffffu, lacc[0], src), lb = __shfl_sync(0xffffffffu, lacc[1], src);
        const float mq = (lane & 1) ? mb : ma, lq = (lane & 1) ? lb : la;
        // w_i in natural units: the query-constant part of the expanded bias
        const float wq = -fmaf(an, g.sx, fmaf(bn, g.sy, cn * fmaf(g.sx, g.sx, g.sy * g.sy)));
        if (lane < 8 && g.qs >= 0)
            a.lse[(tok0 + g.qs) * a.H + h] = lq > 0.f ? fmaf(mq + sfu_lg2(lq), kLn2, wq) : -INFINITY;
    }
}

// ---------------------------------------------------------------- query pass

template <int MTILES>
__device__ __forceinline__ void query_item(const AttnArgs& a, size_t tok0, size_t crow, int h, uint32_t sb,
                                           const float* lse_s, const LaneOffs& lo, const Geo<MTILES>& g,
                                           int lane) {
    using T = QTile<16 * MTILES, true>;
    const int gq = lane >> 2, tq = lane & 3;
    const uint32_t kb = sb + T::K, vb = sb + T::V, qb = sb + T::Q, db_ = sb + T::DO;
    const float an = __ldg(a.bias + 3 * h), bn = __ldg(a.bias + 3 * h + 1), cn = __ldg(a.bias + 3 * h + 2);
    const float a2 = an * kLog2e, b2 = bn * kLog2e, c2 = cn * kLog2e;
    const float sc = a.scale * kLog2e;
    float u[2 * MTILES];
#pragma unroll
    for (int k = 0; k < 2 * MTILES; ++k)
        u[k] = ((g.kval >> k) & 1u) ? fmaf(a2, g.kx[k], fmaf(b2, g.ky[k], -c2 * g.kr[k])) : -INFINITY;
    float X[2], Y[2], Lq[2];
#pragma unroll
    for (int c = 0; c < 2; ++c) {
        X[c] = 2.f * c2 * g.qx[c];
        Y[c] = 2.f * c2 * g.qy[c];
        const float l = lse_s[2 * tq + c];
        // a padding query (no token) has its lse slot zero-filled: mask it through the
        // query-validity bits of the cluster
        const bool ok = ((g.kval >> (16 + 2 * tq + c)) & 1u) && l != -INFINITY;
        // P = exp2(t - L'), L' = lse log2e - w2 with w2 the query-constant bias part
        const float qr2 = fmaf(g.qx[c], g.qx[c], g.qy[c] * g.qy[c]);
        Lq[c] = ok ? fmaf(l, kLog2e, fmaf(a2, g.qx[c], fmaf(b2, g.qy[c], c2 * qr2))) : INFINITY;
    }
    uint32_t qf[4], df[4];
    ldsm_x4(qb + lo.oq, qf[0], qf[1], qf[2], qf[3]);
    ldsm_x4(db_ + lo.oq, df[0], df[1], df[2], df[3]);
    float sacc[MTILES][4], dp[MTILES][4];
#pragma unroll
    for (int i = 0; i < MTILES; ++i) {
        sacc[i][0] = sacc[i][1] = sacc[i][2] = sacc[i][3] = 0.f;
        dp[i][0] = dp[i][1] = dp[i][2] = dp[i][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
            uint32_t r0, r1, r2, r3;
            const uint32_t off = 1024 * i + (kk ? lo.ls1 : lo.ls0);
            ldsm_x4(kb + off, r0, r1, r2, r3);
            mma_bf16(sacc[i], r0, r1, r2, r3, qf[2 * kk], qf[2 * kk + 1]);
            ldsm_x4(vb + off, r0, r1, r2, r3);
            mma_bf16(dp[i], r0, r1, r2, r3, df[2 * kk], df[2 * kk + 1]);
        }
    }
    float pd[2] = {0.f, 0.f};
#pragma unroll
    for (int i = 0; i < MTILES; ++i) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int k = 2 * i + (j >> 1), c = j & 1;
            const float t = fmaf(sacc[i][j], sc, fmaf(X[c], g.kx[k], fmaf(Y[c], g.ky[k], u[k])));
            const float p = sfu_ex2(t - Lq[c]);
            sacc[i][j] = p;
            pd[c] = fmaf(p, dp[i][j], pd[c]);
        }
    }
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
        pd[0] += __shfl_xor_sync(0xffffffffu, pd[0], o);
        pd[1] += __shfl_xor_sync(0xffffffffu, pd[1], o);
    }
    // dS and the bias-gradient sums per query column: S0 = sum dS, Sx = sum dS x_j, ...
    float S0[2] = {0.f, 0.f}, Sx[2] = {0.f, 0.f}, Sy[2] = {0.f, 0.f}, Sr[2] = {0.f, 0.f};
    uint32_t dsb[MTILES][2];
#pragma unroll
    for (int i = 0; i < MTILES; ++i) {
        float ds[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int k = 2 * i + (j >> 1), c = j & 1;
            const float v = sacc[i][j] * (dp[i][j] - pd[c]);
            ds[j] = v;
            S0[c] += v;
            Sx[c] = fmaf(v, g.kx[k], Sx[c]);
            Sy[c] = fmaf(v, g.ky[k], Sy[c]);
            Sr[c] = fmaf(v, g.kr[k], Sr[c]);
        }
        dsb[i][0] = movm_t(pack_bf16(ds[0], ds[1]));
        dsb[i][1] = movm_t(pack_bf16(ds[2], ds[3]));
    }
    // sum_j dS (x_j - x_i) = Sx - x_i S0;  sum_j dS |p_j - p_i|^2 = Sr - 2 x_i Sx - 2 y_i Sy + r_i S0
    float ga = 0.f, gb = 0.f, gc = 0.f;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
        ga += Sx[c] - g.qx[c] * S0[c];
        gb += Sy[c] - g.qy[c] * S0[c];
        gc += Sr[c] - 2.f * (g.qx[c] * Sx[c] + g.qy[c] * Sy[c]) +
              fmaf(g.qx[c], g.qx[c], g.qy[c] * g.qy[c]) * S0[c];
    }
    warp_sum3(ga, gb, gc, lane);
    if (lane == 0) {
        float* part = a.dbias_part + (crow * a.H + h) * 3;
        part[0] = ga;
        part[1] = gb;
        part[2] = -gc;
    }
    {
        // Delta of query `lane` (lanes < 8) from the lanes holding its column
        const int src = (lane >> 1) & 3;
        const float da = __shfl_sync(0xffffffffu, pd[0], src), db = __shfl_sync(0xffffffffu, pd[1], src);
        if (lane < 8 && g.qs >= 0) a.delta[(tok0 + g.qs) * a.H + h] = (lane & 1) ? db : da;
    }
    float dq[2][4];
#pragma unroll
    for (int m = 0; m < 2; ++m) {
        dq[m][0] = dq[m][1] = dq[m][2] = dq[m][3] = 0.f;
#pragma unroll
        for (int i = 0; i < MTILES; ++i) {
            uint32_t r0, r1, r2, r3;
            ldsm_x4_t(kb + 1024 * i + (m ? lo.lt1 : lo.lt0), r0, r1, r2, r3);
            mma_bf16(dq[m], r0, r1, r2, r3, dsb[i][0], dsb[i][1]);
        }
    }
    const float scl = a.scale;
    const uint32_t w0 = movm_t(pack_bf16(dq[0][0] * scl, dq[0][1] * scl));
    const uint32_t w1 = movm_t(pack_bf16(dq[0][2] * scl, dq[0][3] * scl));
    const uint32_t w2 = movm_t(pack_bf16(dq[1][0] * scl, dq[1][1] * scl));
    const uint32_t w3 = movm_t(pack_bf16(dq[1][2] * scl, dq[1][3] * scl));
    if (g.qo >= 0) {
        uint32_t* dst = reinterpret_cast<uint32_t*>(a.dq + ((tok0 + g.qo) * a.H + h) * 32) + tq;
        dst[0] = w0;
        dst[4] = w1;
        dst[8] = w2;
        dst[12] = w3;
    }
}

// ------------------------------------------- forward / query pass: the warp pipeline

// One warp's items [i0, i1) (item = (image, cluster, head), cluster-major).  While item i
// computes, item i + 1 is in flight; the neighbour rows of the cluster after next and the
// coordinates of the next cluster load into registers at every cluster start.
template <int MTILES, bool BWD, typename Off>
__device__ __forceinline__ void cluster_items(const AttnArgs& a, long long i0, long long i1, uint8_t* wsm) {
    constexpr int MT = 16 * MTILES, NK = MT / 8;
    using T = QTile<MT, BWD>;
    const int lane = threadIdx.x & 31;
    const int H = a.H, G = a.G, N = a.N;
    const LaneOffs lo = lane_offs(lane);
    const uint32_t wb = smem_addr(wsm);
    const long long c0 = i0 / H;          // global cluster index b * G + g
    int h = static_cast<int>(i0 - c0 * H);
    // clusters left after the current one, and the end head of the last
    unsigned left = static_cast<unsigned>((i1 - 1) / H - c0);
    const int h_last_end = static_cast<int>(i1 - 1 - ((i1 - 1) / H) * H) + 1;
    int b = static_cast<int>(c0 / G), g = static_cast<int>(c0 - static_cast<long long>(b) * G);
    int b1 = b, g1 = g;
    next_cluster(b1, g1, G);
    int b2 = b1, g2 = g1;
    next_cluster(b2, g2, G);
    Toks cur = load_toks(a, b, g, lane);
    Toks nx = left >= 1 ? load_toks(a, b1, g1, lane) : Toks{-1, -1, -1};
    TokXY cxy = load_xy(a, b, cur);
    Rows<NK, Off> rows = cluster_rows<NK, Off>(a, cur, b, lane);
    int st = 0;
    gather_cluster<MT, BWD, Off>(a, h, rows, wb, lane);
    cp_async_commit();
    for (;;) {
        const int hend = left == 0 ? h_last_end : H;
        const Toks nn = left >= 2 ? load_toks(a, b2, g2, lane) : Toks{-1, -1, -1};
        const TokXY nxy = left >= 1 ? load_xy(a, b1, nx) : TokXY{};
        const Geo<MTILES> geo = make_geo<MTILES>(cur, cxy, rows.valid, lane, N);
        Rows<NK, Off> nrows = rows;
        const size_t tok0 = static_cast<size_t>(b) * N;
        for (; h < hend; ++h) {
            cp_async_wait<0>();
            __syncwarp();
            const uint32_t sb = wb + st * T::STAGE, nb = wb + (st ^ 1) * T::STAGE;
            if (h + 1 < hend) {
                gather_cluster<MT, BWD, Off>(a, h + 1, rows, nb, lane);
                cp_async_commit();
            } else if (left != 0) {
                nrows = cluster_rows<NK, Off>(a, nx, b1, lane);
                gather_cluster<MT, BWD, Off>(a, 0, nrows, nb, lane);
                cp_async_commit();
            }
            if (BWD)
                query_item<MTILES>(a, tok0, static_cast<size_t>(b) * G + g, h, sb,
                                   reinterpret_cast<const float*>(wsm + st * T::STAGE + T::LSE), lo, geo, lane);
            else
                fwd_item<MTILES>(a, tok0, h, sb, lo, geo, lane);
            __syncwarp();
            st ^= 1;
        }
        if (left == 0) break;
        --left;
        h = 0;
        b = b1;
        g = g1;
        b1 = b2;
        g1 = g2;
        next_cluster(b2, g2, G);
        cur = nx;
        nx = nn;
        cxy = nxy;
        rows = nrows;
    }
    cp_async_wait<0>();
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

// ------------------------------------------------------------------ prep

// Reverse neighbourhood index of image b: for each key cluster h, the query clusters g
// whose table lists h, ascending in g, and the 8 tokens of each listed cluster (made
// valid).  One CTA per image; dynamic smem >= 4 * (G + 1) + 160 bytes.
__global__ void __launch_bounds__(256) attn_bwd_prep_kernel(const AttnArgs a) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int b = blockIdx.x;
    const int tid = threadIdx.x, nt = blockDim.x;
    const int N = a.N, G = a.G, R = a.R, M = a.M;
    int* cnt = reinterpret_cast<int*>(smem);
    int* scratch = cnt + G + 1;
    int32_t* tc = a.tok_cluster + static_cast<size_t>(b) * N;
    const int32_t* cl = a.clusters + static_cast<size_t>(b) * G * 8;
    const int32_t* nb = a.nbr + static_cast<size_t>(b) * G * M;
    int32_t* off = a.rev_off + static_cast<size_t>(b) * (G + 1);
    int32_t* lst = a.rev_list + static_cast<size_t>(b) * G * R;
    int32_t* rtok = a.rev_tok + static_cast<size_t>(b) * G * R * 8;
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
    __syncthreads();
    for (int i = tid; i < total * 8; i += nt) rtok[i] = valid_tok(cl[lst[i >> 3] * 8 + (i & 7)], N);
}

// The same index built in shared memory (one CTA per image) when the image fits: the
// token -> cluster map, the cluster rows, the list entries and their key clusters all live
// on chip, so the kernel makes one pass over its inputs and one over its outputs.
// Shared ints: tc[N], cnt[G + 1], lst[G R], ek[G R], cls[8 G], pc[G + 1], scratch[40].
size_t prep_smem_ints(int N, int G, int R) {
    return static_cast<size_t>(N) + (G + 1) + 2ull * G * R + 8ull * G + (G + 1) + 40;
}

__device__ void prep_image_smem(const AttnArgs& a, int b, uint8_t* smem) {
    const int tid = threadIdx.x, nt = blockDim.x;
    const int N = a.N, G = a.G, R = a.R, M = a.M;
    int* tc = reinterpret_cast<int*>(smem);
    int* cnt = tc + N;
    int* lst = cnt + G + 1;
    int* ek = lst + G * R;
    int* cls = ek + G * R;
    int* pc = cls + 8 * G;
    int* scratch = pc + G + 1;
    const int32_t* cl = a.clusters + static_cast<size_t>(b) * G * 8;
    const int32_t* nb = a.nbr + static_cast<size_t>(b) * G * M;
    int32_t* off = a.rev_off + static_cast<size_t>(b) * (G + 1);
    int32_t* rlst = a.rev_list + static_cast<size_t>(b) * G * R;
    int32_t* rtok = a.rev_tok + static_cast<size_t>(b) * G * R * 8;
    for (int i = tid; i < N; i += nt) tc[i] = -1;
    for (int i = tid; i <= G; i += nt) cnt[i] = 0;
    // the first token of every neighbour block, eight loads in flight per thread
    constexpr int kB = 8;
    for (int e0 = tid; e0 < G * R; e0 += kB * nt) {
#pragma unroll
        for (int j = 0; j < kB; ++j) {
            const int e = e0 + j * nt;
            if (e < G * R) {
                const int q = e / R;
                ek[e] = __ldg(nb + static_cast<size_t>(q) * M + (e - q * R) * 8);
            }
        }
    }
    for (int i0 = tid; i0 < G * 8; i0 += kB * nt) {
        int v[kB];
#pragma unroll
        for (int j = 0; j < kB; ++j) v[j] = i0 + j * nt < G * 8 ? __ldg(cl + i0 + j * nt) : -1;
#pragma unroll
        for (int j = 0; j < kB; ++j)
            if (i0 + j * nt < G * 8) cls[i0 + j * nt] = valid_tok(v[j], N);
    }
    __syncthreads();
    for (int i = tid; i < G * 8; i += nt) {
        const int t = cls[i];
        if (t >= 0) tc[t] = i >> 3;
    }
    __syncthreads();
    for (int e = tid; e < G * R; e += nt) {
        const int t0 = valid_tok(ek[e], N);
        const int h = t0 >= 0 ? tc[t0] : -1;
        ek[e] = h;
        if (h >= 0) atomicAdd(&cnt[h], 1);
    }
    __syncthreads();
    const int total = block_scan_excl(cnt, G, scratch);
    for (int i = tid; i < G; i += nt) off[i] = cnt[i];
    if (tid == 0) off[G] = total;
    __syncthreads();  // every list start is read before the fill advances it
    for (int e = tid; e < G * R; e += nt) {
        const int h = ek[e];
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
    // key-pass plan: chunk counts per key cluster and their prefix
    for (int h = tid; h < G; h += nt) {
        const int E = cnt[h] - (h > 0 ? cnt[h - 1] : 0);
        pc[h] = E > 0 ? (E + kChunk - 1) / kChunk : 1;
    }
    __syncthreads();
    for (int i = tid; i < total; i += nt) rlst[i] = lst[i];
    for (int i = tid; i < total * 8; i += nt) rtok[i] = cls[lst[i >> 3] * 8 + (i & 7)];
    const int S = block_scan_excl(pc, G, scratch);
    if (tid == 0) pc[G] = S;
    __syncthreads();
    if (a.kwarps >= a.B) {
        // this image's warps of the key pass split its units (key cluster, head) in cluster-
        // major order so that each gets the same number of chunk items (a unit of key cluster
        // kc weighs its chunk count)
        const long long PW = a.kwarps;
        const int w0 = static_cast<int>((static_cast<long long>(b) * PW + a.B - 1) / a.B);
        const int w1 = static_cast<int>((static_cast<long long>(b + 1) * PW + a.B - 1) / a.B);
        const int k = w1 - w0;
        const long long T = static_cast<long long>(a.H) * S;
        const long long ub = static_cast<long long>(b) * G * a.H;
        auto unit_at = [&](long long tau) -> long long {
            int lo = 0, hi = G;  // largest kc with H pc[kc] <= tau
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (static_cast<long long>(a.H) * pc[mid] <= tau) lo = mid; else hi = mid;
            }
            const int nch = pc[lo + 1] - pc[lo];
            const long long hh = (tau - static_cast<long long>(a.H) * pc[lo]) / nch;
            return static_cast<long long>(lo) * a.H + hh;
        };
        for (int j = tid; j < k; j += nt) {
            const long long u0 = unit_at(T * j / k);
            const long long u1 = j + 1 == k ? static_cast<long long>(G) * a.H : unit_at(T * (j + 1) / k);
            a.kplan[2 * (w0 + j)] = ub + u0;
            a.kplan[2 * (w0 + j) + 1] = ub + u1;
        }
    }
}

__global__ void __launch_bounds__(256) attn_bwd_prep_smem_kernel(const AttnArgs a) {
    extern __shared__ __align__(16) uint8_t smem[];
    prep_image_smem(a, blockIdx.x, smem);
}

// ------------------------------------------------------------------ key pass

// Per-warp stage of the key pass: the key cluster's own K and V rows, the chunk's Q and dO
// rows (kChunk listed clusters), and the chunk rows' parameters (lse and Delta land in .x
// and .y and become (X, Y, L', Delta) in place).
struct KTile {
    static constexpr int K = 0;
    static constexpr int V = 8 * kRowB;
    static constexpr int Q = 16 * kRowB;
    static constexpr int DO = Q + 8 * kChunk * kRowB;
    static constexpr int PRM = DO + 8 * kChunk * kRowB;     // float4 [8 kChunk] row parameters
    static constexpr int LSE = PRM + 16 * 8 * kChunk;       // float [8 kChunk] raw lse
    static constexpr int DEL = LSE + 4 * 8 * kChunk;        // float [8 kChunk] raw Delta
    static constexpr int STAGE = DEL + 4 * 8 * kChunk;
    static constexpr int WARP = 2 * STAGE;
};

// One pair of query clusters (16 queries, rows 8 e .. 8 e + 15 of the Q / dO tiles at qb /
// dob, i.e. byte offset pe = 512 e) against the warp's 8 keys; p1 / p2: parameter rows
// (X, Y, L', Delta) of the lane's queries gq in each block.
__device__ __forceinline__ void key_pair(uint32_t qb, uint32_t dob, uint32_t pe, const LaneOffs& lo, float4 p1,
                                         float4 p2, const uint32_t (&kf)[4], const uint32_t (&vf)[4],
                                         const float (&kx)[2], const float (&ky)[2], const float (&u)[2], float sc,
                                         float (&dk)[2][4], float (&dv)[2][4]) {
    float sacc[4] = {0.f, 0.f, 0.f, 0.f}, pacc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
        const uint32_t off = pe + (kk ? lo.ls1 : lo.ls0);
        uint32_t r0, r1, r2, r3;
        ldsm_x4(qb + off, r0, r1, r2, r3);
        mma_bf16(sacc, r0, r1, r2, r3, kf[2 * kk], kf[2 * kk + 1]);
        ldsm_x4(dob + off, r0, r1, r2, r3);
        mma_bf16(pacc, r0, r1, r2, r3, vf[2 * kk], vf[2 * kk + 1]);
    }
    // element j: query row gq of block (j >> 1), key 2 tq + (j & 1)
    float p[4], ds[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float4 pr = (j >> 1) ? p2 : p1;
        const int c = j & 1;
        const float t = fmaf(sacc[j], sc, fmaf(pr.x, kx[c], fmaf(pr.y, ky[c], u[c])));
        p[j] = sfu_ex2(t - pr.z);
        ds[j] = p[j] * (pacc[j] - pr.w);
    }
    const uint32_t pb0 = movm_t(pack_bf16(p[0], p[1]));
    const uint32_t pb1 = movm_t(pack_bf16(p[2], p[3]));
    const uint32_t sb0 = movm_t(pack_bf16(ds[0], ds[1]));
    const uint32_t sb1 = movm_t(pack_bf16(ds[2], ds[3]));
#pragma unroll
    for (int m = 0; m < 2; ++m) {
        const uint32_t off = pe + (m ? lo.lt1 : lo.lt0);
        uint32_t r0, r1, r2, r3;
        ldsm_x4_t(dob + off, r0, r1, r2, r3);
        mma_bf16(dv[m], r0, r1, r2, r3, pb0, pb1);
        ldsm_x4_t(qb + off, r0, r1, r2, r3);
        mma_bf16(dk[m], r0, r1, r2, r3, sb0, sb1);
    }
}

// Row parameters of a query token for head h: X = 2 c x, Y = 2 c y (log2 units, local
// coordinates), L' = lse log2e - w2 (P = exp2(t - L')), Delta.
__device__ __forceinline__ float4 row_params(float x, float y, bool valid, float lse, float delta, float a2,
                                             float b2, float c2) {
    const bool ok = valid && lse != -INFINITY;
    float4 r;
    r.x = ok ? 2.f * c2 * x : 0.f;
    r.y = ok ? 2.f * c2 * y : 0.f;
    r.z = ok ? fmaf(lse, kLog2e, fmaf(a2, x, fmaf(b2, y, c2 * fmaf(x, x, y * y)))) : INFINITY;
    r.w = ok ? delta : 0.f;
    return r;
}

// Store one warp's dK^T / dV^T accumulators (dims x keys) as rows of dK / dV.
__device__ __forceinline__ void store_key_rows(const float (&acc)[2][4], float scl, int tok, size_t tok0,
                                               int H, int h, bf16* dst_base) {
    const int lane = threadIdx.x & 31, tq = lane & 3;
    const uint32_t w0 = movm_t(pack_bf16(acc[0][0] * scl, acc[0][1] * scl));
    const uint32_t w1 = movm_t(pack_bf16(acc[0][2] * scl, acc[0][3] * scl));
    const uint32_t w2 = movm_t(pack_bf16(acc[1][0] * scl, acc[1][1] * scl));
    const uint32_t w3 = movm_t(pack_bf16(acc[1][2] * scl, acc[1][3] * scl));
    if (tok >= 0) {
        uint32_t* dst = reinterpret_cast<uint32_t*>(dst_base + ((tok0 + tok) * H + h) * 32) + tq;
        dst[0] = w0;
        dst[4] = w1;
        dst[8] = w2;
        dst[12] = w3;
    }
}

// A key-pass item: (image b, key cluster kc, head h, chunk ch) over the list entries
// [e0, e0 + E) of kc (image-local).  It carries what the gather needs: the byte offsets
// (head 0) of the lane's gather rows -- own row gq, chunk rows gq + 8 k -- with a validity
// bit each, the tokens of the lane's parameter rows lane and lane + 32 and of the own
// cluster row (lanes < 8), and their coordinates (loaded an item later).
template <typename Off>
struct KItem {
    int b, kc, h, ch, nch, e0, E;
    Off qo[kChunk], ko;
    unsigned valid;  // bit k: chunk row gq + 8 k; bit kChunk: own row gq
    int pa, pb, kt;
    float2 pxa, pxb, kxy;
};

// The raw tokens of an item: the lane's parameter rows (chunk rows lane and lane + 32) and
// the own cluster row (lanes < 8).  Nothing uses them before the next item step, so the
// loads have a whole item to land.
template <typename Off>
__device__ __forceinline__ void kitem_tokens(const AttnArgs& a, KItem<Off>& it, int lane) {
    const int32_t* rtok = a.rev_tok + static_cast<size_t>(it.b) * a.G * a.R * 8;
    const size_t base = (static_cast<size_t>(it.e0) + static_cast<size_t>(kChunk) * it.ch) * 8;
    const int rem = (it.E - kChunk * it.ch) * 8;
    const int n = rem > 8 * kChunk ? 8 * kChunk : rem;
    it.pa = lane < n ? __ldg(rtok + base + lane) : -1;
    it.pb = lane + 32 < n ? __ldg(rtok + base + lane + 32) : -1;
    it.kt = lane < 8 ? __ldg(a.clusters + (static_cast<size_t>(it.b) * a.G + it.kc) * 8 + lane) : -1;
}
// An item step later: the tokens made valid, the coordinates requested.
template <typename Off>
__device__ __forceinline__ void kitem_coords(const AttnArgs& a, KItem<Off>& it) {
    const float2* xyb = reinterpret_cast<const float2*>(a.xy) + static_cast<size_t>(it.b) * a.N;
    it.kt = valid_tok(it.kt, a.N);
    it.pxa = it.pa >= 0 ? __ldg(xyb + it.pa) : make_float2(0.f, 0.f);
    it.pxb = it.pb >= 0 ? __ldg(xyb + it.pb) : make_float2(0.f, 0.f);
    it.kxy = it.kt >= 0 ? __ldg(xyb + it.kt) : make_float2(0.f, 0.f);
}
// The byte offsets (head 0) of the lane's gather rows: chunk rows gq + 8 k and own row gq.
template <typename Off>
__device__ __forceinline__ void kitem_rows(const AttnArgs& a, KItem<Off>& it, int lane) {
    const int gq = lane >> 2;
    const Off rowb = static_cast<Off>(a.H) * 64u;
    const Off tb = static_cast<Off>(it.b) * static_cast<Off>(a.N);
    it.valid = 0u;
#pragma unroll
    for (int k = 0; k < kChunk; ++k) {
        const int t = __shfl_sync(0xffffffffu, k < 4 ? it.pa : it.pb, gq + 8 * (k & 3));
        it.qo[k] = t >= 0 ? (tb + static_cast<Off>(t)) * rowb : Off(0);
        it.valid |= t >= 0 ? (1u << k) : 0u;
    }
    const int own = __shfl_sync(0xffffffffu, it.kt, gq);
    it.ko = own >= 0 ? (tb + static_cast<Off>(own)) * rowb : Off(0);
    it.valid |= own >= 0 ? (1u << kChunk) : 0u;
}

template <typename Off>
__device__ __forceinline__ void kitem_gather(const AttnArgs& a, const KItem<Off>& it, uint32_t sb, int lane) {
    const uint32_t lo = gather_lane_off(lane);
    const size_t hb = static_cast<size_t>(it.h) * 64 + (lane & 3) * 16;
    const char* kp = reinterpret_cast<const char*>(a.k) + hb;
    const char* vp = reinterpret_cast<const char*>(a.v) + hb;
    const char* qp = reinterpret_cast<const char*>(a.q) + hb;
    const char* dp = reinterpret_cast<const char*>(a.dout) + hb;
    const bool okk = (it.valid >> kChunk) & 1u;
    cp_async16(sb + KTile::K + lo, kp + it.ko, okk);
    cp_async16(sb + KTile::V + lo, vp + it.ko, okk);
#pragma unroll
    for (int k = 0; k < kChunk; ++k) {
        const bool ok = (it.valid >> k) & 1u;
        cp_async16(sb + KTile::Q + 512 * k + lo, qp + it.qo[k], ok);
        cp_async16(sb + KTile::DO + 512 * k + lo, dp + it.qo[k], ok);
    }
    const size_t tok0 = static_cast<size_t>(it.b) * a.N;
    const size_t sa = it.pa >= 0 ? (tok0 + it.pa) * a.H + it.h : 0;
    cp_async4(sb + KTile::LSE + 4 * lane, a.lse_in + sa, it.pa >= 0);
    cp_async4(sb + KTile::DEL + 4 * lane, a.delta + sa, it.pa >= 0);
    if (lane + 32 < 8 * kChunk) {
        const size_t s2 = it.pb >= 0 ? (tok0 + it.pb) * a.H + it.h : 0;
        cp_async4(sb + KTile::LSE + 4 * (lane + 32), a.lse_in + s2, it.pb >= 0);
        cp_async4(sb + KTile::DEL + 4 * (lane + 32), a.delta + s2, it.pb >= 0);
    }
}

// A window of list offsets held by the warp: lane j has (first entry, entry count) of the
// global key cluster base + j (global index b G + kc), so advancing to the next key cluster
// takes two shuffles instead of a dependent load.
struct OffWin {
    unsigned base;
    int e0, E;
};
__device__ __forceinline__ void load_win(const AttnArgs& a, OffWin& w, unsigned base, int lane) {
    w.base = base;
    const unsigned c = base + lane;
    const unsigned b = c / static_cast<unsigned>(a.G);
    w.e0 = 0;
    w.E = 0;
    if (b < static_cast<unsigned>(a.B)) {
        const int32_t* roff = a.rev_off + static_cast<size_t>(b) * (a.G + 1) + (c - b * a.G);
        w.e0 = __ldg(roff);
        w.E = __ldg(roff + 1) - w.e0;
    }
}

// Advance `it` (global key cluster c) to the next item of the warp's units (b, kc, h)
// (cluster-major), whose last is unit u_end - 1; returns false past the end.
template <typename Off>
__device__ __forceinline__ bool kitem_next(const AttnArgs& a, KItem<Off>& it, long long& unit, long long u_end,
                                           unsigned& c, OffWin& w, int lane) {
    if (it.ch + 1 < it.nch) {
        ++it.ch;
        return true;
    }
    if (unit + 1 >= u_end) return false;
    ++unit;
    it.ch = 0;
    if (++it.h == a.H) {
        it.h = 0;
        if (++it.kc == a.G) {
            it.kc = 0;
            ++it.b;
        }
        ++c;
        if (c - w.base >= 32u) load_win(a, w, c, lane);
        it.e0 = __shfl_sync(0xffffffffu, w.e0, c - w.base);
        it.E = __shfl_sync(0xffffffffu, w.E, c - w.base);
        it.nch = it.E > 0 ? (it.E + kChunk - 1) / kChunk : 1;
    }
    return true;
}

// One key-pass item: row parameters in place, then the chunk's pairs; the accumulators
// carry over the chunks of a (key cluster, head) and are stored after its last chunk.
template <typename Off>
__device__ __forceinline__ void key_item(const AttnArgs& a, const KItem<Off>& it, uint32_t sb, uint8_t* stage,
                                         const LaneOffs& lo, float (&dk)[2][4], float (&dv)[2][4], int lane) {
    const int gq = lane >> 2, tq = lane & 3;
    const float a2 = __ldg(a.bias + 3 * it.h) * kLog2e, b2 = __ldg(a.bias + 3 * it.h + 1) * kLog2e,
                c2 = __ldg(a.bias + 3 * it.h + 2) * kLog2e;
    const float sc = a.scale * kLog2e;
    float4* prm = reinterpret_cast<float4*>(stage + KTile::PRM);
    const float* lse = reinterpret_cast<const float*>(stage + KTile::LSE);
    const float* del = reinterpret_cast<const float*>(stage + KTile::DEL);
    // local origin: the key cluster's first slot
    const float2 org = sh2(it.kxy, 0);
    prm[lane] = row_params(it.pxa.x - org.x, it.pxa.y - org.y, it.pa >= 0, lse[lane], del[lane], a2, b2, c2);
    if (lane + 32 < 8 * kChunk)
        prm[lane + 32] = row_params(it.pxb.x - org.x, it.pxb.y - org.y, it.pb >= 0, lse[lane + 32], del[lane + 32], a2,
                                    b2, c2);
    __syncwarp();
    uint32_t kf[4], vf[4];
    ldsm_x4(sb + KTile::K + lo.oq, kf[0], kf[1], kf[2], kf[3]);
    ldsm_x4(sb + KTile::V + lo.oq, vf[0], vf[1], vf[2], vf[3]);
    float kx[2], ky[2], u[2];
#pragma unroll
    for (int c = 0; c < 2; ++c) {
        const float2 p = sh2(it.kxy, 2 * tq + c);
        const bool ok = __shfl_sync(0xffffffffu, it.kt, 2 * tq + c) >= 0;
        kx[c] = ok ? p.x - org.x : 0.f;
        ky[c] = ok ? p.y - org.y : 0.f;
        u[c] = ok ? fmaf(a2, kx[c], fmaf(b2, ky[c], -c2 * fmaf(kx[c], kx[c], ky[c] * ky[c]))) : -INFINITY;
    }
    // listed clusters of this chunk; rows of absent ones are zero and their parameters give P = 0
    const int n = min(it.E - kChunk * it.ch, kChunk);
#pragma unroll
    for (int e = 0; e < kChunk; e += 2) {
        if (e < n)
            key_pair(sb + KTile::Q, sb + KTile::DO, 512u * e, lo, prm[8 * e + gq], prm[8 * (e + 1) + gq], kf, vf, kx,
                     ky, u, sc, dk, dv);
    }
    if (it.ch + 1 == it.nch) {
        const int own = __shfl_sync(0xffffffffu, it.kt, gq);
        const size_t tok0 = static_cast<size_t>(it.b) * a.N;
        store_key_rows(dk, a.scale, own, tok0, a.H, it.h, a.dk);
        store_key_rows(dv, 1.f, own, tok0, a.H, it.h, a.dv);
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
            for (int j = 0; j < 4; ++j) dk[m][j] = dv[m][j] = 0.f;
    }
}

// One warp's units [u0, u1) of the key pass (unit = (image, key cluster, head)).  The
// item cursor runs two items ahead: tokens two items early, coordinates and the gather one.
template <typename Off>
__device__ __forceinline__ void key_units(const AttnArgs& a, long long u0, long long u1, uint8_t* wsm) {
    const int lane = threadIdx.x & 31;
    const int H = a.H, G = a.G;
    const uint32_t wb = smem_addr(wsm);
    const LaneOffs lo = lane_offs(lane);
    KItem<Off> cur;
    unsigned c = static_cast<unsigned>(u0 / H);  // global key cluster of the leading cursor
    OffWin win;
    load_win(a, win, c, lane);
    cur.h = static_cast<int>(u0 - static_cast<long long>(c) * H);
    cur.b = static_cast<int>(c / static_cast<unsigned>(G));
    cur.kc = static_cast<int>(c - static_cast<unsigned>(cur.b) * G);
    cur.ch = 0;
    cur.e0 = __shfl_sync(0xffffffffu, win.e0, 0);
    cur.E = __shfl_sync(0xffffffffu, win.E, 0);
    cur.nch = cur.E > 0 ? (cur.E + kChunk - 1) / kChunk : 1;
    kitem_tokens(a, cur, lane);
    kitem_coords(a, cur);
    KItem<Off> nx = cur;
    long long unx = u0;
    bool has_nx = kitem_next(a, nx, unx, u1, c, win, lane);
    if (has_nx) kitem_tokens(a, nx, lane);
    int st = 0;
    kitem_rows(a, cur, lane);
    kitem_gather(a, cur, wb, lane);
    cp_async_commit();
    float dk[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    float dv[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    for (;;) {
        KItem<Off> nn = nx;
        long long unn = unx;
        const bool has_nn = has_nx && kitem_next(a, nn, unn, u1, c, win, lane);
        if (has_nn) kitem_tokens(a, nn, lane);
        if (has_nx) kitem_coords(a, nx);
        cp_async_wait<0>();
        __syncwarp();
        if (has_nx) {
            kitem_rows(a, nx, lane);
            kitem_gather(a, nx, wb + (st ^ 1) * KTile::STAGE, lane);
            cp_async_commit();
        }
        key_item(a, cur, wb + st * KTile::STAGE, wsm + st * KTile::STAGE, lo, dk, dv, lane);
        __syncwarp();
        st ^= 1;
        if (!has_nx) break;
        cur = nx;
        nx = nn;
        unx = unn;
        has_nx = has_nn;
    }
    cp_async_wait<0>();
}

// ------------------------------------------------------------- entry kernels

// Resident warps per SM the kernels are built for: the forward 16 (4 CTAs of 4 warps, up
// to 128 registers), the query pass's larger stage 12, the key pass 16.
template <int MTILES, typename Off>
__global__ void __launch_bounds__(kThreads, MTILES <= 3 ? 4 : 2) attn_fwd_kernel(const AttnArgs a) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int warp = threadIdx.x >> 5;
    const long long PW = static_cast<long long>(gridDim.x) * kWarps;
    const long long gw = static_cast<long long>(blockIdx.x) * kWarps + warp;
    const long long W = static_cast<long long>(a.B) * a.G * a.H;
    const long long i0 = gw * W / PW, i1 = (gw + 1) * W / PW;
    if (i0 >= i1) return;
    cluster_items<MTILES, false, Off>(a, i0, i1, smem + warp * QTile<16 * MTILES, false>::WARP);
}

// The query pass; its first `nprep` CTAs build the reverse index of one image each (when
// the index fits the kernel's shared memory) while the others run the items.
template <int MTILES, typename Off>
__global__ void __launch_bounds__(kThreads, MTILES <= 3 ? 3 : 2) attn_bwd_query_kernel(const AttnArgs a, int nprep) {
    extern __shared__ __align__(16) uint8_t smem[];
    if (static_cast<int>(blockIdx.x) < nprep) {
        prep_image_smem(a, blockIdx.x, smem);
        return;
    }
    const int warp = threadIdx.x >> 5;
    const long long PW = static_cast<long long>(gridDim.x - nprep) * kWarps;
    const long long gw = static_cast<long long>(blockIdx.x - nprep) * kWarps + warp;
    const long long W = static_cast<long long>(a.B) * a.G * a.H;
    const long long i0 = gw * W / PW, i1 = (gw + 1) * W / PW;
    if (i0 >= i1) return;
    cluster_items<MTILES, true, Off>(a, i0, i1, smem + warp * QTile<16 * MTILES, true>::WARP);
}

template <typename Off>
__global__ void __launch_bounds__(kThreads, 4) attn_bwd_key_kernel(const AttnArgs a, int P) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (static_cast<int>(blockIdx.x) >= P) {
        // bias-gradient reduction: one CTA per (head, coefficient), fixed order
        const int hj = blockIdx.x - P;
        const int hh = hj / 3, j = hj % 3;
        const int n = a.B * a.G;
        float acc = 0.f;
#pragma unroll 4
        for (int i = tid; i < n; i += kThreads) acc += a.dbias_part[(static_cast<size_t>(i) * a.H + hh) * 3 + j];
        acc = warp_sum(acc);
        float* red = reinterpret_cast<float*>(smem);
        if (lane == 0) red[warp] = acc;
        __syncthreads();
        if (tid == 0) {
            float tot = 0.f;
            for (int w = 0; w < kWarps; ++w) tot += red[w];
            a.dbias[hh * 3 + j] = tot;
        }
        return;
    }
    const long long PW = static_cast<long long>(P) * kWarps;
    const long long gw = static_cast<long long>(blockIdx.x) * kWarps + warp;
    long long u0, u1;
    if (a.kwarps == PW && PW >= a.B) {
        // the plan the reverse-index builders made: equal chunk items per warp
        u0 = a.kplan[2 * gw];
        u1 = a.kplan[2 * gw + 1];
    } else {
        const long long W = static_cast<long long>(a.B) * a.G * a.H;
        u0 = gw * W / PW;
        u1 = (gw + 1) * W / PW;
    }
    if (u0 >= u1) return;
    key_units<Off>(a, u0, u1, smem + warp * KTile::WARP);
}

// ---------------------------------------------------------------- launchers


// Persistent grid: resident CTAs per SM times the SM count, or fewer when there are fewer
// items than warps.
int grid_for(long long items, int per_sm) {
    const long long slots = static_cast<long long>(sm_count()) * per_sm;
    const long long need = (items + kWarps - 1) / kWarps;
    return static_cast<int>(need < slots ? need : slots);
}

// The reverse index: in shared memory when an image fits, else through the workspace.
cudaError_t launch_prep(const AttnArgs& a, cudaStream_t st) {
    const size_t sm = 4 * prep_smem_ints(a.N, a.G, a.R);
    cudaError_t e;
    if (sm <= 200 * 1024) {
        e = ensure_smem<attn_bwd_prep_smem_kernel>(sm);
        if (e != cudaSuccess) return e;
        attn_bwd_prep_smem_kernel<<<a.B, 256, sm, st>>>(a);
    } else {
        const size_t prep = 4 * static_cast<size_t>(a.G + 1) + 160;
        e = ensure_smem<attn_bwd_prep_kernel>(prep);
        if (e != cudaSuccess) return e;
        attn_bwd_prep_kernel<<<a.B, 256, prep, st>>>(a);
    }
    note_launch();
    return cudaGetLastError();
}

// 32-bit row offsets when every [B][N][H][32] bf16 tensor is smaller than 4 GiB.
bool narrow_offsets(const AttnArgs& a) {
    return static_cast<unsigned long long>(a.B) * a.N * a.H * 64ull < (1ull << 32);
}

template <int MTILES, typename Off>
cudaError_t fwd_launch(const AttnArgs& a, cudaStream_t st) {
    const size_t smem = static_cast<size_t>(kWarps) * QTile<16 * MTILES, false>::WARP;
    cudaError_t e = ensure_smem<attn_fwd_kernel<MTILES, Off>>(smem);
    if (e != cudaSuccess) return e;
    const int per = resident<attn_fwd_kernel<MTILES, Off>>(kThreads, smem);
    const int grid = grid_for(static_cast<long long>(a.B) * a.G * a.H, per);
    attn_fwd_kernel<MTILES, Off><<<grid, kThreads, smem, st>>>(a);
    note_launch();
    return cudaGetLastError();
}

template <int MTILES>
cudaError_t fwd_dispatch(const AttnArgs& a, cudaStream_t st) {
    return narrow_offsets(a) ? fwd_launch<MTILES, uint32_t>(a, st) : fwd_launch<MTILES, uint64_t>(a, st);
}

// The query pass, with the reverse index built by its leading CTAs when an image's index
// fits the kernel's shared memory (those CTAs take resident slots from the query items for
// the few microseconds they run), else by a separate kernel first.
template <int MTILES, typename Off>
cudaError_t query_launch(const AttnArgs& a, cudaStream_t st) {
    const size_t smem = static_cast<size_t>(kWarps) * QTile<16 * MTILES, true>::WARP;
    cudaError_t e = ensure_smem<attn_bwd_query_kernel<MTILES, Off>>(smem);
    if (e != cudaSuccess) return e;
    const int per = resident<attn_bwd_query_kernel<MTILES, Off>>(kThreads, smem);
    const size_t prep = 4 * prep_smem_ints(a.N, a.G, a.R);
    const long long slots = static_cast<long long>(sm_count()) * per;
    int nprep = 0;
    if (prep <= smem && 2LL * a.B <= slots) {
        nprep = a.B;
    } else {
        const cudaError_t ep = launch_prep(a, st);
        if (ep != cudaSuccess) return ep;
    }
    const long long items = static_cast<long long>(a.B) * a.G * a.H;
    long long P = grid_for(items, per);
    if (nprep > 0 && P + nprep > slots) P = slots - nprep;
    attn_bwd_query_kernel<MTILES, Off><<<static_cast<unsigned>(P + nprep), kThreads, smem, st>>>(a, nprep);
    note_launch();
    return cudaGetLastError();
}

// Key pass (+ 3 H bias-reduction CTAs at the end of the grid).
template <typename Off>
int key_grid(const AttnArgs& a) {
    const size_t smem = static_cast<size_t>(kWarps) * KTile::WARP;
    if (ensure_smem<attn_bwd_key_kernel<Off>>(smem) != cudaSuccess) return 1;
    return grid_for(static_cast<long long>(a.B) * a.G * a.H, resident<attn_bwd_key_kernel<Off>>(kThreads, smem));
}

template <typename Off>
cudaError_t key_launch(const AttnArgs& a, cudaStream_t st) {
    const size_t smem = static_cast<size_t>(kWarps) * KTile::WARP;
    cudaError_t e = ensure_smem<attn_bwd_key_kernel<Off>>(smem);
    if (e != cudaSuccess) return e;
    const int P = key_grid<Off>(a);
    attn_bwd_key_kernel<Off><<<P + 3 * a.H, kThreads, smem, st>>>(a, P);
    note_launch();
    return cudaGetLastError();
}

template <int MTILES>
cudaError_t bwd_dispatch(const AttnArgs& a0, cudaStream_t st) {
    AttnArgs a = a0;
    const long long kw =
        static_cast<long long>(narrow_offsets(a) ? key_grid<uint32_t>(a) : key_grid<uint64_t>(a)) * kWarps;
    const bool plan = kw <= kMaxPlanWarps && 4 * prep_smem_ints(a.N, a.G, a.R) <= 200 * 1024;
    a.kwarps = plan ? static_cast<int>(kw) : 0;
    const cudaError_t e = narrow_offsets(a) ? query_launch<MTILES, uint32_t>(a, st) : query_launch<MTILES, uint64_t>(a, st);
    if (e != cudaSuccess) return e;
    return narrow_offsets(a) ? key_launch<uint32_t>(a, st) : key_launch<uint64_t>(a, st);
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
    w.rev_tok = off;     off += up(sizeof(int32_t) * B * G * R * 8);
    w.kplan = off;       off += up(sizeof(long long) * 2 * kMaxPlanWarps);
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

ACL_CHECK_READER(read_checks_attn)

}  // namespace acl
