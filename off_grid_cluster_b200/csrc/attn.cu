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
// so no tile is padded beyond M's rounding to 16.
//
// A CTA runs kUC = 4 consecutive clusters x kUH = 2 heads (8 warps).  Consecutive
// clusters are siblings of the bisection tree and their neighbourhoods overlap, so the
// CTA gathers the union of the group's neighbour blocks once (16-byte cp.async of
// 128-byte token rows = the two heads) into XOR-swizzled shared tiles, and each warp
// addresses its own 48 keys inside the union through a block map; ldmatrix reads them
// without bank conflicts.  This halves the L2 -> SM traffic of the 6x-reused rows.
//
// Backward (recompute, FA2-style, no atomics):
//   pass 1, query-major (same CTA shape as the forward): recompute P from lse,
//     dP^T = V . dO^T, Delta = rowsum(P o dP) (equal to <dO, O>, but exact in fp32
//     because the whole key row is in the tile, and O need not be read),
//     dS = P (dP - Delta), dQ^T = K^T . dS^T, per-(cluster, head) partial sums of the
//     bias gradient.  One extra column of CTAs builds, per image, the reverse
//     neighbourhood index: for every key cluster, the query clusters that list it.
//   pass 2, key-major: CTA = 4 key clusters x 2 heads; the union of the query clusters
//     in their reverse lists is gathered once, and each warp walks its own list two
//     query clusters at a time (16 queries = one MMA M tile): S = Q K_h^T,
//     dP = dO V_h^T, dV^T += dO^T P, dK^T += Q^T dS.  Extra CTAs reduce the bias
//     partials in a fixed order.  A group whose lists overflow the union tile falls back
//     to per-warp direct loads.
#include <math.h>

#include "internal.h"

namespace acl {

namespace {


// ------------------------------------------------------------------ layouts

constexpr int kBwdKWarpBytes = 3584;

// bf16 pair (hi) of two floats and the bf16 pair of their remainders (lo): hi + lo keeps
// about 16 significant bits.
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

// ------------------------------------------------- forward, neighbourhood unions
//
// One CTA per (image, group of kUC consecutive clusters, group of kUH heads); warp w owns
// cluster w / kUH and head w % kUH of the group.  Consecutive clusters are siblings of the
// bisection tree, so their neighbourhoods overlap: the CTA de-duplicates the group's
// neighbour blocks (a block is one whole cluster, named by its first token), gathers each
// union row's K and V once (kUH heads = 128 contiguous bytes per token) and every warp
// reads its own neighbourhood out of the union tile through a block map.  Rows are
// 128 bytes with the 16-byte chunk index XOR-ed by (row & 7); a neighbourhood block is 8
// consecutive union rows, so the 8 rows of every ldmatrix hit 8 distinct bank groups.
// Empty blocks map to 8 zero rows at the end of the tile.
constexpr int kUC = 4;
constexpr int kUH = 2;
constexpr int kUWarps = kUC * kUH;
constexpr int kUThreads = 32 * kUWarps;
constexpr int kURow = 64 * kUH;  // bytes per union row

struct UnionLayout {
    int ks, vs, qs, stage, utok, uxy, qtok, qxy, krow, nbs, total;
};
__host__ __device__ __forceinline__ UnionLayout union_layout(int R, int MT) {
    UnionLayout L;
    const int rows = kUC * R * 8 + 8;  // union rows + a zero block
    int o = 0;
    L.ks = o; o += rows * kURow;
    L.vs = o; o += rows * kURow;
    L.qs = o; o += kUC * 8 * kURow;
    L.stage = o; o += kUWarps * 512;
    L.utok = o; o += 4 * (rows - 8);
    L.uxy = o; o += 8 * (rows - 8);
    L.qtok = o; o += 4 * kUC * 8;
    L.qxy = o; o += 8 * kUC * 8;
    L.krow = o; o += 4 * kUC * MT;
    L.nbs = o; o += 4 * kUC * R * 8;        // the group's neighbour rows
    L.total = (o + 15) & ~15;
    return L;
}

__device__ __forceinline__ uint32_t urow_off(int row, int ch) {
    return static_cast<uint32_t>(row * kURow + ((ch ^ (row & 7)) << 4));
}

// Union setup shared by the forward-shaped kernels: the neighbour rows of the CTA's kUC
// clusters (one global round, into shared memory), their blocks de-duplicated by first
// token (every warp computes the same map in registers, so no barrier is needed before
// it is used), union row tokens, the per-cluster key-slot -> union row map and the
// group's query tokens.  Coordinates follow with the tiles (union_coords_async).  All
// threads of the CTA call it; returns the number of distinct blocks.
__device__ __forceinline__ int union_setup(const AttnArgs& a, int b, int g0, int MT, const UnionLayout& L,
                                           uint8_t* smem) {
    const int tid = threadIdx.x, lane = tid & 31;
    const int G = a.G, N = a.N, M = a.M, R = a.R;
    const int nblk = kUC * R;
    int* utok = reinterpret_cast<int*>(smem + L.utok);
    int* qtok = reinterpret_cast<int*>(smem + L.qtok);
    int* krow = reinterpret_cast<int*>(smem + L.krow);
    int* nbs = reinterpret_cast<int*>(smem + L.nbs);
    for (int i = tid; i < nblk * 8; i += blockDim.x) {
        const int cw = i / M, m = i - cw * M;
        const int g = g0 + cw;
        int t = -1;
        if (g < G) {
            t = a.nbr[(static_cast<size_t>(b) * G + g) * M + m];
            if (t < 0 || t >= N) t = -1;
        }
        nbs[i] = t;
    }
    for (int i = tid; i < kUC * 8; i += blockDim.x) {
        const int g = g0 + (i >> 3);
        int id = -1;
        if (g < G) {
            id = a.clusters[(static_cast<size_t>(b) * G + g) * 8 + (i & 7)];
            if (id < 0 || id >= N) id = -1;
        }
        qtok[i] = id;
    }
    __syncthreads();
    // lane j < nblk: block j's union index, or the index of its first occurrence (the
    // lowest lane holding the same first token)
    const int f = lane < nblk ? nbs[lane * 8] : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, f);
    const int lead = __ffs(peers) - 1;
    const int dup = (f >= 0 && lead != lane) ? lead : -1;
    const bool isnew = f >= 0 && lead == lane;
    const unsigned newmask = __ballot_sync(0xffffffffu, isnew);
    int u = isnew ? __popc(newmask & ((1u << lane) - 1u)) : -1;
    const int ud = __shfl_sync(0xffffffffu, u, dup >= 0 ? dup : 0);
    if (dup >= 0) u = ud;
    const int nU = __popc(newmask);
    for (int base = 0; base < nblk * 8; base += blockDim.x) {
        const int i = base + tid;
        const int blk = min(i >> 3, 31);
        const int ub = __shfl_sync(0xffffffffu, u, blk);
        const bool first = __shfl_sync(0xffffffffu, isnew ? 1 : 0, blk) != 0;
        if (i < nblk * 8 && first) utok[ub * 8 + (i & 7)] = nbs[i];
    }
    for (int base = 0; base < kUC * MT; base += blockDim.x) {
        const int i = base + tid;
        const int cw = i / MT, m = i - cw * MT;
        const int blk = min(cw * R + (m >> 3), 31);
        const int ub = __shfl_sync(0xffffffffu, u, blk);
        if (i < kUC * MT) krow[i] = (m < M && ub >= 0) ? ub * 8 + (m & 7) : -1;
    }
    __syncthreads();
    return nU;
}

// Coordinates of the union rows and of the group's queries, as asynchronous copies in
// the caller's current cp.async group (rows without a token read as (0, 0)).
__device__ __forceinline__ void union_coords_async(const AttnArgs& a, int b, int nU, const UnionLayout& L,
                                                   uint8_t* smem) {
    const int* utok = reinterpret_cast<const int*>(smem + L.utok);
    const int* qtok = reinterpret_cast<const int*>(smem + L.qtok);
    const float2* xyb = reinterpret_cast<const float2*>(a.xy) + static_cast<size_t>(b) * a.N;
    for (int i = threadIdx.x; i < nU * 8; i += blockDim.x) {
        const int t = utok[i];
        cp_async8(smem_addr(smem + L.uxy) + 8 * i, xyb + (t >= 0 ? t : 0), t >= 0);
    }
    for (int i = threadIdx.x; i < kUC * 8; i += blockDim.x) {
        const int t = qtok[i];
        cp_async8(smem_addr(smem + L.qxy) + 8 * i, xyb + (t >= 0 ? t : 0), t >= 0);
    }
}

template <int MTILES>
__global__ void __launch_bounds__(kUThreads) attn_fwd_union_kernel(const AttnArgs a) {
    constexpr int MT = 16 * MTILES;
    extern __shared__ __align__(16) uint8_t smem[];
    const int R = a.R;
    const UnionLayout L = union_layout(R, MT);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int cg = blockIdx.x, hg = blockIdx.y, b = blockIdx.z;
    const int G = a.G, N = a.N, H = a.H;
    const int g0 = cg * kUC;
    const int nblk = kUC * R;
    const int ZR = nblk * 8;
    uint8_t* ks = smem + L.ks;
    uint8_t* vs = smem + L.vs;
    uint8_t* qs = smem + L.qs;
    const int* utok = reinterpret_cast<const int*>(smem + L.utok);
    const float2* uxy = reinterpret_cast<const float2*>(smem + L.uxy);
    const int* qtok = reinterpret_cast<const int*>(smem + L.qtok);
    const float2* qxy = reinterpret_cast<const float2*>(smem + L.qxy);
    const int* krow = reinterpret_cast<const int*>(smem + L.krow);
    const size_t tok0 = static_cast<size_t>(b) * N;

    // 1-3. the group's neighbour rows, de-duplicated blocks, union rows and block map
    const int nU = union_setup(a, b, g0, MT, L, smem);
    // 4. gather the union's K and V rows, the group's Q rows, and zero the spare block;
    //    thread tid copies 16-byte chunk tid % 8 of rows tid / 8, tid / 8 + 32, ...
    const int hlo = hg * kUH;
    const int ch = tid & 7;
    const bool ch_ok = hlo + (ch >> 2) < H;
    const size_t cbase = (tok0 * H + hlo) * 32 + ch * 8;
    const size_t tstride = static_cast<size_t>(H) * 32;
    const int urows = nU * 8;
    for (int row = tid >> 3; row < urows + 8; row += kUThreads / 8) {
        const int t = row < urows ? utok[row] : -1;
        const bool ok = t >= 0 && ch_ok;
        const int drow = row < urows ? row : ZR + (row - urows);
        cp_async16(smem_addr(ks) + urow_off(drow, ch), a.k + (ok ? cbase + t * tstride : 0), ok);
    }
    for (int row = tid >> 3; row < kUC * 8; row += kUThreads / 8) {
        const int t = qtok[row];
        const bool ok = t >= 0 && ch_ok;
        cp_async16(smem_addr(qs) + urow_off(row, ch), a.q + (ok ? cbase + t * tstride : 0), ok);
    }
    union_coords_async(a, b, nU, L, smem);
    cp_async_commit();  // group 0: K, Q, coordinates
    for (int row = tid >> 3; row < urows + 8; row += kUThreads / 8) {
        const int t = row < urows ? utok[row] : -1;
        const bool ok = t >= 0 && ch_ok;
        const int drow = row < urows ? row : ZR + (row - urows);
        cp_async16(smem_addr(vs) + urow_off(drow, ch), a.v + (ok ? cbase + t * tstride : 0), ok);
    }
    cp_async_commit();  // group 1: V (lands while S and the softmax run)
    cp_async_wait<1>();
    __syncthreads();

    // 5. one (cluster, head) per warp
    const int cw = warp / kUH, hw = warp % kUH;
    const int g = g0 + cw;
    // a warp past the last cluster or head computes on masked data and stores nothing (it
    // must still reach the barrier before the V tile is read)
    const bool active = g < G && hlo + hw < H;
    const int h = active ? hlo + hw : 0;
    const int gq = lane >> 2, tq = lane & 3, mi = lane >> 3;
    const int* kr = krow + cw * MT;
    // row bases of the neighbourhood blocks this lane addresses
    // row 0 of each neighbourhood block this lane addresses: (mi & 1) picks the block of
    // the S / dQ operands, (mi >> 1) the block of the transposed V / K operands
    int base_s[MTILES], base_t[MTILES];
#pragma unroll
    for (int i = 0; i < MTILES; ++i) {
        const int s0 = 2 * i + (mi & 1), s1 = 2 * i + (mi >> 1);
        const int r0 = (s0 * 8 < a.M) ? kr[s0 * 8] : -1;
        const int r1 = (s1 * 8 < a.M) ? kr[s1 * 8] : -1;
        base_s[i] = r0 >= 0 ? r0 : ZR;
        base_t[i] = r1 >= 0 ? r1 : ZR;
    }
    uint32_t qf0, qf1, qf2, qf3;
    ldsm_x4(smem_addr(qs) + urow_off(cw * 8 + (lane & 7), hw * 4 + mi), qf0, qf1, qf2, qf3);
    float sacc[MTILES][4];
#pragma unroll
    for (int i = 0; i < MTILES; ++i) {
        sacc[i][0] = sacc[i][1] = sacc[i][2] = sacc[i][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
            const int row = base_s[i] + (lane & 7);
            uint32_t a0, a1, a2, a3;
            ldsm_x4(smem_addr(ks) + urow_off(row, hw * 4 + 2 * kk + (mi >> 1)), a0, a1, a2, a3);
            mma_bf16(sacc[i], a0, a1, a2, a3, kk ? qf2 : qf0, kk ? qf3 : qf1);
        }
    }
    const float sc = a.scale * kLog2e;
    const float ba = a.bias[3 * h] * kLog2e, bb = a.bias[3 * h + 1] * kLog2e,
                bc = a.bias[3 * h + 2] * kLog2e;
    const float2 qa = qxy[cw * 8 + 2 * tq], qb = qxy[cw * 8 + 2 * tq + 1];
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int i = 0; i < MTILES; ++i) {
#pragma unroll
        for (int hi = 0; hi < 2; ++hi) {
            const int row = kr[16 * i + gq + 8 * hi];
            const bool kv = row >= 0 && utok[row] >= 0;
            const float2 kp = kv ? uxy[row] : make_float2(0.f, 0.f);
            float dx = kp.x - qa.x, dy = kp.y - qa.y;
            const float v0 = sacc[i][2 * hi] * sc + ba * dx + bb * dy - bc * (dx * dx + dy * dy);
            dx = kp.x - qb.x;
            dy = kp.y - qb.y;
            const float v1 = sacc[i][2 * hi + 1] * sc + ba * dx + bb * dy - bc * (dx * dx + dy * dy);
            sacc[i][2 * hi] = kv ? v0 : -INFINITY;
            sacc[i][2 * hi + 1] = kv ? v1 : -INFINITY;
            mx0 = fmaxf(mx0, sacc[i][2 * hi]);
            mx1 = fmaxf(mx1, sacc[i][2 * hi + 1]);
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
        const float p0 = exp2f(sacc[i][0] - m0), p1 = exp2f(sacc[i][1] - m1);
        const float p2 = exp2f(sacc[i][2] - m0), p3 = exp2f(sacc[i][3] - m1);
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
    cp_async_wait<0>();
    __syncthreads();  // V tile complete (all threads reach this: no early exit above)
    float oacc[2][4];
#pragma unroll
    for (int m = 0; m < 2; ++m) {
        oacc[m][0] = oacc[m][1] = oacc[m][2] = oacc[m][3] = 0.f;
#pragma unroll
        for (int i = 0; i < MTILES; ++i) {
            const int row = base_t[i] + (lane & 7);
            uint32_t a0, a1, a2, a3;
            ldsm_x4_t(smem_addr(vs) + urow_off(row, hw * 4 + 2 * m + (mi & 1)), a0, a1, a2, a3);
            mma_bf16(oacc[m], a0, a1, a2, a3, pbl[i][0], pbl[i][1]);
            mma_bf16(oacc[m], a0, a1, a2, a3, pbh[i][0], pbh[i][1]);
        }
    }
    const float i0 = l0 > 0.f ? 1.f / l0 : 0.f;
    const float i1 = l1 > 0.f ? 1.f / l1 : 0.f;
    if (!active) return;
    store_rows_t(oacc, i0, i1, smem + L.stage + warp * 512, qtok + cw * 8, tok0, H, h, a.o, lane);
    if (gq == 0) {
        const int q0 = qtok[cw * 8 + 2 * tq], q1 = qtok[cw * 8 + 2 * tq + 1];
        if (q0 >= 0) a.lse[(tok0 + q0) * H + h] = l0 > 0.f ? (m0 + log2f(l0)) * kLn2 : -INFINITY;
        if (q1 >= 0) a.lse[(tok0 + q1) * H + h] = l1 > 0.f ? (m1 + log2f(l1)) * kLn2 : -INFINITY;
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

// ------------------------------------------------------ backward, key-major

// Key-major backward of one (image, key cluster, head) by one warp, loading the query
// rows of each pair of listed query clusters straight into its own 3.5 KB of shared memory.
__device__ void key_major_direct(const AttnArgs& a, int b, int kc, int h, int lane, uint8_t* w) {
    const int H = a.H;
    const size_t tok0 = static_cast<size_t>(b) * a.N;
    const float2* xyb = reinterpret_cast<const float2*>(a.xy) + tok0;

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


// ------------------------------------------------ backward with neighbourhood unions


// Query-major pass with neighbourhood unions (same CTA shape as the forward), plus one
// extra CTA column that builds each image's reverse neighbourhood index.
template <int MTILES>
__global__ void __launch_bounds__(kUThreads) attn_bwd_query_union_kernel(const AttnArgs a, int ncg) {
    constexpr int MT = 16 * MTILES;
    extern __shared__ __align__(16) uint8_t smem[];
    const int cg = blockIdx.x, hg = blockIdx.y, b = blockIdx.z;
    if (cg >= ncg) {
        if (hg == 0) build_reverse_index(a, b, smem);
        return;
    }
    const int R = a.R;
    const UnionLayout L = union_layout(R, MT);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = a.G, N = a.N, H = a.H;
    const int g0 = cg * kUC;
    const int ZR = kUC * R * 8;
    uint8_t* ks = smem + L.ks;
    uint8_t* vs = smem + L.vs;
    uint8_t* qs = smem + L.qs;
    uint8_t* dos = smem + L.stage;  // dO tile (kUC * 8 rows) in the staging area
    uint8_t* stage = smem + L.total;  // per-warp output staging after the layout
    const size_t tok0 = static_cast<size_t>(b) * N;
    const int nU = union_setup(a, b, g0, MT, L, smem);
    const int* utok = reinterpret_cast<const int*>(smem + L.utok);
    const float2* uxy = reinterpret_cast<const float2*>(smem + L.uxy);
    const int* qtok = reinterpret_cast<const int*>(smem + L.qtok);
    const float2* qxy = reinterpret_cast<const float2*>(smem + L.qxy);
    const int* krow = reinterpret_cast<const int*>(smem + L.krow);
    const int hlo = hg * kUH;
    {
        // thread tid copies 16-byte chunk tid % 8 of rows tid / 8, tid / 8 + 32, ...
        const int ch = tid & 7;
        const bool ch_ok = hlo + (ch >> 2) < H;
        const size_t cbase = (tok0 * H + hlo) * 32 + ch * 8;
        const size_t tstride = static_cast<size_t>(H) * 32;
        const int urows = nU * 8;
        for (int row = tid >> 3; row < urows + 8; row += kUThreads / 8) {
            const int t = row < urows ? utok[row] : -1;
            const bool ok = t >= 0 && ch_ok;
            const int drow = row < urows ? row : ZR + (row - urows);
            const size_t off = ok ? cbase + t * tstride : 0;
            cp_async16(smem_addr(ks) + urow_off(drow, ch), a.k + off, ok);
            cp_async16(smem_addr(vs) + urow_off(drow, ch), a.v + off, ok);
        }
        for (int row = tid >> 3; row < kUC * 8; row += kUThreads / 8) {
            const int t = qtok[row];
            const bool ok = t >= 0 && ch_ok;
            const size_t off = ok ? cbase + t * tstride : 0;
            cp_async16(smem_addr(qs) + urow_off(row, ch), a.q + off, ok);
            cp_async16(smem_addr(dos) + urow_off(row, ch), a.dout + off, ok);
        }
    }
    union_coords_async(a, b, nU, L, smem);
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();

    const int cw = warp / kUH, hw = warp % kUH;
    const int g = g0 + cw, h = hlo + hw;
    if (g >= G || h >= H) return;
    const int gq = lane >> 2, tq = lane & 3, mi = lane >> 3;
    const int* kr = krow + cw * MT;
    // row 0 of each neighbourhood block this lane addresses: (mi & 1) picks the block of
    // the S / dQ operands, (mi >> 1) the block of the transposed V / K operands
    int base_s[MTILES], base_t[MTILES];
#pragma unroll
    for (int i = 0; i < MTILES; ++i) {
        const int s0 = 2 * i + (mi & 1), s1 = 2 * i + (mi >> 1);
        const int r0 = (s0 * 8 < a.M) ? kr[s0 * 8] : -1;
        const int r1 = (s1 * 8 < a.M) ? kr[s1 * 8] : -1;
        base_s[i] = r0 >= 0 ? r0 : ZR;
        base_t[i] = r1 >= 0 ? r1 : ZR;
    }
    const int q0 = qtok[cw * 8 + 2 * tq], q1 = qtok[cw * 8 + 2 * tq + 1];
    float L0 = q0 >= 0 ? a.lse_in[(tok0 + q0) * H + h] * kLog2e : INFINITY;
    float L1 = q1 >= 0 ? a.lse_in[(tok0 + q1) * H + h] * kLog2e : INFINITY;
    if (L0 == -INFINITY) L0 = INFINITY;
    if (L1 == -INFINITY) L1 = INFINITY;
    uint32_t qf0, qf1, qf2, qf3, df0, df1, df2, df3;
    ldsm_x4(smem_addr(qs) + urow_off(cw * 8 + (lane & 7), hw * 4 + mi), qf0, qf1, qf2, qf3);
    ldsm_x4(smem_addr(dos) + urow_off(cw * 8 + (lane & 7), hw * 4 + mi), df0, df1, df2, df3);
    float sacc[MTILES][4], dp[MTILES][4];
#pragma unroll
    for (int i = 0; i < MTILES; ++i) {
        sacc[i][0] = sacc[i][1] = sacc[i][2] = sacc[i][3] = 0.f;
        dp[i][0] = dp[i][1] = dp[i][2] = dp[i][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
            const int row = base_s[i] + (lane & 7);
            const uint32_t off = urow_off(row, hw * 4 + 2 * kk + (mi >> 1));
            uint32_t a0, a1, a2, a3;
            ldsm_x4(smem_addr(ks) + off, a0, a1, a2, a3);
            mma_bf16(sacc[i], a0, a1, a2, a3, kk ? qf2 : qf0, kk ? qf3 : qf1);
            ldsm_x4(smem_addr(vs) + off, a0, a1, a2, a3);
            mma_bf16(dp[i], a0, a1, a2, a3, kk ? df2 : df0, kk ? df3 : df1);
        }
    }
    const float sc = a.scale * kLog2e;
    const float ba = a.bias[3 * h] * kLog2e, bb = a.bias[3 * h + 1] * kLog2e,
                bc = a.bias[3 * h + 2] * kLog2e;
    const float2 qa = qxy[cw * 8 + 2 * tq], qb = qxy[cw * 8 + 2 * tq + 1];
    float pd0 = 0.f, pd1 = 0.f;
#pragma unroll
    for (int i = 0; i < MTILES; ++i) {
#pragma unroll
        for (int hi = 0; hi < 2; ++hi) {
            const int row = kr[16 * i + gq + 8 * hi];
            const bool kv = row >= 0 && utok[row] >= 0;
            const float2 kp = kv ? uxy[row] : make_float2(0.f, 0.f);
#pragma unroll
            for (int qq = 0; qq < 2; ++qq) {
                const float2 qp = qq ? qb : qa;
                const float dx = kp.x - qp.x, dy = kp.y - qp.y;
                const int j = 2 * hi + qq;
                const float lg = sacc[i][j] * sc + ba * dx + bb * dy - bc * (dx * dx + dy * dy);
                const float p = kv ? exp2f(lg - (qq ? L1 : L0)) : 0.f;
                sacc[i][j] = p;
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
            const int row = kr[16 * i + gq + 8 * hi];
            const bool kv = row >= 0 && utok[row] >= 0;
            const float2 kp = kv ? uxy[row] : make_float2(0.f, 0.f);
#pragma unroll
            for (int qq = 0; qq < 2; ++qq) {
                const float2 qp = qq ? qb : qa;
                const float dx = kp.x - qp.x, dy = kp.y - qp.y;
                const int j = 2 * hi + qq;
                const float v = sacc[i][j] * (dp[i][j] - (qq ? pd1 : pd0));
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
        float* part = a.dbias_part + ((static_cast<size_t>(b) * G + g) * H + h) * 3;
        part[0] = ga;
        part[1] = gb;
        part[2] = -gc;
    }
    float dqacc[2][4];
#pragma unroll
    for (int m = 0; m < 2; ++m) {
        dqacc[m][0] = dqacc[m][1] = dqacc[m][2] = dqacc[m][3] = 0.f;
#pragma unroll
        for (int i = 0; i < MTILES; ++i) {
            const int row = base_t[i] + (lane & 7);
            uint32_t a0, a1, a2, a3;
            ldsm_x4_t(smem_addr(ks) + urow_off(row, hw * 4 + 2 * m + (mi & 1)), a0, a1, a2, a3);
            mma_bf16(dqacc[m], a0, a1, a2, a3, db[i][0], db[i][1]);
        }
    }
    store_rows_t(dqacc, a.scale, a.scale, stage + warp * 512, qtok + cw * 8, tok0, H, h, a.dq, lane);
}

// Key-major pass with query-cluster unions.  CTA = (kUC consecutive key clusters, kUH
// heads, image).  The reverse lists of its key clusters are concatenated and their query
// clusters de-duplicated; Q and dO rows of the union (plus lse and Delta) are gathered
// once and every warp walks its own list two query clusters at a time out of the union
// tile.  A group whose lists exceed the tile falls back to per-warp direct loading.
constexpr int kKQ = 24;       // union query clusters held per CTA
constexpr int kKEnt = 64;     // list entries per CTA
struct KeyLayout {
    int qs, dos, ks, vs, stage, ent, eu, es, qtok, qxy, qL, qD, ktok, kxy, misc, total;
};
__host__ __device__ __forceinline__ KeyLayout key_layout() {
    KeyLayout L;
    const int rows = kKQ * 8 + 8;
    int o = 0;
    L.qs = o; o += rows * kURow;
    L.dos = o; o += rows * kURow;
    L.ks = o; o += kUC * 8 * kURow;
    L.vs = o; o += kUC * 8 * kURow;
    L.stage = o; o += kUWarps * 512;
    L.ent = o; o += 4 * kKEnt;
    L.eu = o; o += 4 * kKEnt;
    L.es = o; o += 4 * (kUC + 1 + kKEnt);  // [kUC] count, then first-occurrence flags
    o = (o + 15) & ~15;
    L.qtok = o; o += 4 * rows;
    L.qxy = o; o += 8 * rows;
    L.qL = o; o += 4 * rows * kUH;
    L.qD = o; o += 4 * rows * kUH;
    L.ktok = o; o += 4 * kUC * 8;
    L.kxy = o; o += 8 * kUC * 8;
    L.misc = o; o += 16;
    L.total = (o + 15) & ~15;
    return L;
}

__global__ void __launch_bounds__(kUThreads) attn_bwd_key_union_kernel(const AttnArgs a, int ncg) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int cg = blockIdx.x, hg = blockIdx.y, b = blockIdx.z;
    const int G = a.G, N = a.N, H = a.H;
    if (cg >= ncg) {
        // bias-gradient reduction: one CTA per (head, coefficient), fixed order
        const int hj = cg - ncg;
        if (hg != 0 || b != 0 || hj >= 3 * H) return;
        const int hh = hj / 3, j = hj % 3;
        const int n = a.B * G;
        float acc = 0.f;
#pragma unroll 4
        for (int i = tid; i < n; i += kUThreads) acc += a.dbias_part[(static_cast<size_t>(i) * H + hh) * 3 + j];
        acc = warp_sum(acc);
        float* red = reinterpret_cast<float*>(smem);
        if (lane == 0) red[warp] = acc;
        __syncthreads();
        if (tid == 0) {
            float tot = 0.f;
            for (int w = 0; w < kUWarps; ++w) tot += red[w];
            a.dbias[hh * 3 + j] = tot;
        }
        return;
    }
    const KeyLayout L = key_layout();
    const int g0 = cg * kUC;
    const int hlo = hg * kUH;
    const int ZR = kKQ * 8;
    const size_t tok0 = static_cast<size_t>(b) * N;
    const float2* xyb = reinterpret_cast<const float2*>(a.xy) + tok0;
    int* ent = reinterpret_cast<int*>(smem + L.ent);
    int* eu = reinterpret_cast<int*>(smem + L.eu);
    int* es = reinterpret_cast<int*>(smem + L.es);
    int* qtok = reinterpret_cast<int*>(smem + L.qtok);
    float2* qxy = reinterpret_cast<float2*>(smem + L.qxy);
    float* qL = reinterpret_cast<float*>(smem + L.qL);
    float* qD = reinterpret_cast<float*>(smem + L.qD);
    int* ktok = reinterpret_cast<int*>(smem + L.ktok);
    float2* kxy = reinterpret_cast<float2*>(smem + L.kxy);
    int* misc = reinterpret_cast<int*>(smem + L.misc);
    const int32_t* roff = a.rev_off + static_cast<size_t>(b) * (G + 1);
    const int32_t* rlist = a.rev_list + static_cast<size_t>(b) * G * a.R;
    static_assert(kKEnt == 64 && kUC < 32, "warp 0 holds two list entries per lane");
    if (warp == 0) {
        // list offsets of the kUC key clusters (lane c), their prefix, then the entries
        // (lanes hold entries lane and lane + 32) and their de-duplication in registers
        int cnt = 0;
        if (lane < kUC && g0 + lane < G) cnt = roff[g0 + lane + 1] - roff[g0 + lane];
        const int start = (lane < kUC && g0 + lane < G) ? roff[g0 + lane] : 0;
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        const int ntot_w = __shfl_sync(0xffffffffu, incl, kUC - 1);
        int e[2] = {-1, -1};
        if (ntot_w <= kKEnt) {
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                const int i = x * 32 + lane;
                int c = 0;  // the key cluster whose list holds entry i (all lanes shuffle)
#pragma unroll
                for (int cc = 1; cc < kUC; ++cc)
                    c += (i >= __shfl_sync(0xffffffffu, incl - cnt, cc)) ? 1 : 0;
                const int es_c = __shfl_sync(0xffffffffu, incl - cnt, c);
                const int st_c = __shfl_sync(0xffffffffu, start, c);
                if (i < ntot_w) e[x] = rlist[st_c + (i - es_c)];
            }
            // first occurrence of each entry's value (src = its index), in list order
            int src[2] = {0x7fffffff, 0x7fffffff};
#pragma unroll 8
            for (int j = 0; j < kKEnt; ++j) {
                const int vj = __shfl_sync(0xffffffffu, j < 32 ? e[0] : e[1], j & 31);
#pragma unroll
                for (int x = 0; x < 2; ++x)
                    if (j < src[x] && vj == e[x] && j < ntot_w) src[x] = j;
            }
            int run = 0, ui[2];
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                const int i = x * 32 + lane;
                const bool first = i < ntot_w && src[x] == i;
                const unsigned m = __ballot_sync(0xffffffffu, first);
                ui[x] = first ? run + __popc(m & ((1u << lane) - 1u)) : -1;
                run += __popc(m);
            }
            // a repeated entry takes the union index of its first occurrence
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                const int i = x * 32 + lane;
                const int s2 = (i < ntot_w) ? src[x] : i;
                const int from0 = __shfl_sync(0xffffffffu, ui[0], s2 & 31);
                const int from1 = __shfl_sync(0xffffffffu, ui[1], s2 & 31);
                if (i < ntot_w) {
                    ent[i] = e[x];
                    eu[i] = (s2 < 32) ? from0 : from1;
                    es[kUC + 1 + i] = (src[x] == i) ? 1 : 0;  // first occurrence
                }
            }
            if (lane == 0) misc[0] = run;
        }
        if (lane <= kUC) es[lane] = incl - cnt;  // list start of key cluster lane; es[kUC] = total
    } else {
        for (int i = tid - 32; i < kUC * 8; i += kUThreads - 32) {
            const int kc = g0 + (i >> 3);
            int id = -1;
            if (kc < G) {
                id = a.clusters[(static_cast<size_t>(b) * G + kc) * 8 + (i & 7)];
                if (id < 0 || id >= N) id = -1;
            }
            ktok[i] = id;
            kxy[i] = id >= 0 ? xyb[id] : make_float2(0.f, 0.f);
        }
    }
    __syncthreads();
    const int ntot = es[kUC];
    const bool fits = ntot <= kKEnt && misc[0] <= kKQ;
    if (!fits) {
        // fallback: every warp handles its (key cluster, head) with direct loads
        const int cw = warp / kUH, hw = warp % kUH;
        const int kc = g0 + cw, h = hlo + hw;
        if (kc < G && h < H) key_major_direct(a, b, kc, h, lane, smem + warp * kBwdKWarpBytes);
        return;
    }
    const int nU = misc[0];
    // union query rows, their lse / Delta per head of the group
    for (int i = tid; i < ntot * 8; i += kUThreads) {
        const int e = i >> 3, sl = i & 7;
        if (!es[kUC + 1 + e]) continue;  // a repeated list entry
        const int row = eu[e] * 8 + sl;
        int t = a.clusters[(static_cast<size_t>(b) * G + ent[e]) * 8 + sl];
        if (t < 0 || t >= N) t = -1;
        qtok[row] = t;
        qxy[row] = t >= 0 ? xyb[t] : make_float2(0.f, 0.f);
        for (int hw = 0; hw < kUH; ++hw) {
            const int h = hlo + hw;
            float Lv = INFINITY, Dv = 0.f;
            if (t >= 0 && h < H) {
                Lv = a.lse_in[(tok0 + t) * H + h] * kLog2e;
                if (Lv == -INFINITY) Lv = INFINITY;
                Dv = a.delta[(tok0 + t) * H + h];
            }
            qL[row * kUH + hw] = Lv;
            qD[row * kUH + hw] = Dv;
        }
    }
    for (int i = tid; i < 8 * kUH; i += kUThreads) {
        qL[(ZR + (i / kUH)) * kUH + (i % kUH)] = INFINITY;
        qD[(ZR + (i / kUH)) * kUH + (i % kUH)] = 0.f;
    }
    if (tid < 8) {
        qtok[ZR + tid] = -1;
        qxy[ZR + tid] = make_float2(0.f, 0.f);
    }
    __syncthreads();
    uint8_t* qs = smem + L.qs;
    uint8_t* dos = smem + L.dos;
    uint8_t* ks = smem + L.ks;
    uint8_t* vs = smem + L.vs;
    {
        // thread tid copies 16-byte chunk tid % 8 of rows tid / 8, tid / 8 + 32, ...
        const int ch = tid & 7;
        const bool ch_ok = hlo + (ch >> 2) < H;
        const size_t cbase = (tok0 * H + hlo) * 32 + ch * 8;
        const size_t tstride = static_cast<size_t>(H) * 32;
        const int urows = nU * 8;
        for (int row = tid >> 3; row < urows + 8; row += kUThreads / 8) {
            const int drow = row < urows ? row : ZR + (row - urows);
            const int t = qtok[drow];
            const bool ok = t >= 0 && ch_ok;
            const size_t off = ok ? cbase + t * tstride : 0;
            cp_async16(smem_addr(qs) + urow_off(drow, ch), a.q + off, ok);
            cp_async16(smem_addr(dos) + urow_off(drow, ch), a.dout + off, ok);
        }
        for (int row = tid >> 3; row < kUC * 8; row += kUThreads / 8) {
            const int t = ktok[row];
            const bool ok = t >= 0 && ch_ok;
            const size_t off = ok ? cbase + t * tstride : 0;
            cp_async16(smem_addr(ks) + urow_off(row, ch), a.k + off, ok);
            cp_async16(smem_addr(vs) + urow_off(row, ch), a.v + off, ok);
        }
    }
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();

    const int cw = warp / kUH, hw = warp % kUH;
    const int kc = g0 + cw, h = hlo + hw;
    if (kc >= G || h >= H) return;
    const int gq = lane >> 2, tq = lane & 3, mi = lane >> 3;
    uint32_t kf0, kf1, kf2, kf3, vf0, vf1, vf2, vf3;
    ldsm_x4(smem_addr(ks) + urow_off(cw * 8 + (lane & 7), hw * 4 + mi), kf0, kf1, kf2, kf3);
    ldsm_x4(smem_addr(vs) + urow_off(cw * 8 + (lane & 7), hw * 4 + mi), vf0, vf1, vf2, vf3);
    const float sc = a.scale * kLog2e;
    const float ba = a.bias[3 * h] * kLog2e, bb = a.bias[3 * h + 1] * kLog2e,
                bc = a.bias[3 * h + 2] * kLog2e;
    const float2 kp0 = kxy[cw * 8 + 2 * tq], kp1 = kxy[cw * 8 + 2 * tq + 1];
    float dk[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    float dv[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    const int e_end = es[cw + 1];
    for (int e = es[cw]; e < e_end; e += 2) {
        const int b1 = eu[e] * 8;
        const int b2 = (e + 1 < e_end) ? eu[e + 1] * 8 : ZR;
        float sacc[4] = {0.f, 0.f, 0.f, 0.f}, pacc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
            const int row = ((mi & 1) ? b2 : b1) + (lane & 7);
            const uint32_t off = urow_off(row, hw * 4 + 2 * kk + (mi >> 1));
            uint32_t a0, a1, a2, a3;
            ldsm_x4(smem_addr(qs) + off, a0, a1, a2, a3);
            mma_bf16(sacc, a0, a1, a2, a3, kk ? kf2 : kf0, kk ? kf3 : kf1);
            ldsm_x4(smem_addr(dos) + off, a0, a1, a2, a3);
            mma_bf16(pacc, a0, a1, a2, a3, kk ? vf2 : vf0, kk ? vf3 : vf1);
        }
        float p[4], ds[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int qrow = ((j >> 1) ? b2 : b1) + gq;
            const float2 qp = qxy[qrow];
            const float2 kp = (j & 1) ? kp1 : kp0;
            const float dx = kp.x - qp.x, dy = kp.y - qp.y;
            const float lg = sacc[j] * sc + ba * dx + bb * dy - bc * (dx * dx + dy * dy);
            p[j] = exp2f(lg - qL[qrow * kUH + hw]);
            ds[j] = p[j] * (pacc[j] - qD[qrow * kUH + hw]);
        }
        const uint32_t pb0 = movm_t(pack_bf16(p[0], p[1]));
        const uint32_t pb1 = movm_t(pack_bf16(p[2], p[3]));
        const uint32_t sb0 = movm_t(pack_bf16(ds[0], ds[1]));
        const uint32_t sb1 = movm_t(pack_bf16(ds[2], ds[3]));
#pragma unroll
        for (int m = 0; m < 2; ++m) {
            const int row = ((mi >> 1) ? b2 : b1) + (lane & 7);
            const uint32_t off = urow_off(row, hw * 4 + 2 * m + (mi & 1));
            uint32_t a0, a1, a2, a3;
            ldsm_x4_t(smem_addr(dos) + off, a0, a1, a2, a3);
            mma_bf16(dv[m], a0, a1, a2, a3, pb0, pb1);
            ldsm_x4_t(smem_addr(qs) + off, a0, a1, a2, a3);
            mma_bf16(dk[m], a0, a1, a2, a3, sb0, sb1);
        }
    }
    uint8_t* stage = smem + L.stage + warp * 512;
    store_rows_t1(dk, a.scale, stage, ktok + cw * 8, tok0, H, h, a.dk, lane);
    store_rows_t1(dv, 1.f, stage, ktok + cw * 8, tok0, H, h, a.dv, lane);
}

template <int MTILES>
cudaError_t fwd_union_dispatch(const AttnArgs& a, cudaStream_t st) {
    const size_t smem = static_cast<size_t>(union_layout(a.R, 16 * MTILES).total);
    cudaError_t e = ensure_smem<attn_fwd_union_kernel<MTILES>>(smem);
    if (e != cudaSuccess) return e;
    dim3 grid((a.G + kUC - 1) / kUC, (a.H + kUH - 1) / kUH, a.B);
    attn_fwd_union_kernel<MTILES><<<grid, kUThreads, smem, st>>>(a);
    note_launch();
    return cudaGetLastError();
}

template <int MTILES>
cudaError_t bwd_dispatch(const AttnArgs& a, cudaStream_t st) {
    const int ncg = (a.G + kUC - 1) / kUC;
    const int nhg = (a.H + kUH - 1) / kUH;
    // query-major pass (+ one column of reverse-index CTAs)
    size_t smem = static_cast<size_t>(union_layout(a.R, 16 * MTILES).total) + kUWarps * 512;
    const size_t prep = 4 * static_cast<size_t>(a.G + 1) + 160;
    if (prep > smem) smem = prep;
    cudaError_t e = ensure_smem<attn_bwd_query_union_kernel<MTILES>>(smem);
    if (e != cudaSuccess) return e;
    attn_bwd_query_union_kernel<MTILES><<<dim3(ncg + 1, nhg, a.B), kUThreads, smem, st>>>(a, ncg);
    note_launch();
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // key-major pass (+ 3H bias-reduction CTAs in the first column block)
    size_t smem2 = static_cast<size_t>(key_layout().total);
    if (smem2 < static_cast<size_t>(kUWarps) * kBwdKWarpBytes) smem2 = static_cast<size_t>(kUWarps) * kBwdKWarpBytes;
    e = ensure_smem<attn_bwd_key_union_kernel>(smem2);
    if (e != cudaSuccess) return e;
    const int extra = (3 * a.H + 0);
    attn_bwd_key_union_kernel<<<dim3(ncg + extra, nhg, a.B), kUThreads, smem2, st>>>(a, ncg);
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
        case 1: return fwd_union_dispatch<1>(a, st);
        case 2: return fwd_union_dispatch<2>(a, st);
        case 3: return fwd_union_dispatch<3>(a, st);
        default: return fwd_union_dispatch<4>(a, st);
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
