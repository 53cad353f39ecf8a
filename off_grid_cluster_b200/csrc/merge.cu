// merge.cu -- token merging between stages, forward and backward.
//
// AFFMAE notes, "Key Designs" 1 (adaptive off-grid token merging): a lightweight MLP scores
// every token, the top-k by score are kept as anchors (k = the retention rate times N), and
// every other token is merged differentiably into its nearest anchor, fusing features and
// spatial support.  Here:
//   s_i = w2 . gelu(W1^T f_i + b1) + b2  (W1 [d][h] fp32, exact-erf gelu, fp32 math);
//   anchors = the k largest scores, ties by lower id, listed by ascending id;
//   assign_i = the rank of the nearest anchor (fp64 squared distance of the fp32 coordinates,
//     ties by lower anchor id; an anchor is its own group);
//   group G_j: w_i = softmax_{i in G_j}(s_i); merged F_j = sum w_i f_i, X_j = sum w_i x_i.
// Backward, for fixed anchors and assignment (both piecewise constant):
//   g_i = <dF_j, f_i> + <dX_j, x_i>, ds_i = w_i (g_i - sum_G w g), dx_i = w_i dX_j,
//   dh_i = ds_i w2 * gelu'(z_i), df_i = w_i dF_j + W1 dh_i,
//   dW1 = sum_i f_i dh_i^T, db1 = sum dh_i, dw2 = sum ds_i gelu(z_i), db2 = sum ds_i.
// No atomics in any sum: groups are listed by a sort, every token belongs to one group, and
// the parameter gradients are reduced in two fixed-order stages.
#include <float.h>

#include "internal.h"

namespace acl {

namespace {

constexpr int kMergeWarps = 8;
constexpr int kMergeThreads = 32 * kMergeWarps;
constexpr int kSortThreads = 1024;
constexpr int kParamParts = 64;   // token ranges of the first parameter-gradient stage
constexpr int kParamTile = 32;    // tokens staged per step of that stage

__device__ __forceinline__ float gelu_f(float z) { return 0.5f * z * (1.f + erff(z * 0.70710678118654752f)); }
__device__ __forceinline__ float gelu_grad_f(float z) {
    return 0.5f * (1.f + erff(z * 0.70710678118654752f)) + z * 0.39894228040143268f * expf(-0.5f * z * z);
}

__host__ __device__ __forceinline__ int pow2_ge(int n) {
    int p = 1;
    while (p < n) p <<= 1;
    return p;
}

// Hidden pre-activations z_u = b1_u + sum_c f_c W1[c][u] of one token, lane l holding
// u = l + 32 x (x < HP); f is read as bf16 pairs, two channels per lane, broadcast by shuffles.
template <int HP>
__device__ __forceinline__ void hidden_pre(const bf16* frow, int d, const float* w1, const float* b1,
                                           int h, int lane, float (&z)[HP]) {
#pragma unroll
    for (int x = 0; x < HP; ++x) {
        const int u = lane + 32 * x;
        z[x] = u < h ? __ldg(b1 + u) : 0.f;
    }
    for (int c0 = 0; c0 < d; c0 += 64) {
        const int c = c0 + 2 * lane;
        uint32_t pair = 0u;
        if (c < d) pair = *reinterpret_cast<const uint32_t*>(frow + c);
        const int cn = min(64, d - c0);
        for (int cc = 0; cc < cn; ++cc) {
            const uint32_t pw = __shfl_sync(0xffffffffu, pair, cc >> 1);
            const float fc = (cc & 1) ? bf16_hi(pw) : bf16_lo(pw);
            const float* wr = w1 + static_cast<size_t>(c0 + cc) * h;
#pragma unroll
            for (int x = 0; x < HP; ++x) {
                const int u = lane + 32 * x;
                if (u < h) z[x] = fmaf(fc, __ldg(wr + u), z[x]);
            }
        }
    }
}

// 1. scores: one warp per token.
template <int HP>
__global__ void __launch_bounds__(kMergeThreads)
    merge_scores_kernel(const bf16* __restrict__ feats, int T, int d, const float* __restrict__ w1,
                        const float* __restrict__ b1, const float* __restrict__ w2, float b2, int h,
                        float* __restrict__ scores) {
    const int lane = threadIdx.x & 31;
    const long long t = static_cast<long long>(blockIdx.x) * kMergeWarps + (threadIdx.x >> 5);
    if (t >= T) return;  // whole warps
    float z[HP];
    hidden_pre<HP>(feats + static_cast<size_t>(t) * d, d, w1, b1, h, lane, z);
    float s = 0.f;
#pragma unroll
    for (int x = 0; x < HP; ++x) {
        const int u = lane + 32 * x;
        if (u < h) s = fmaf(__ldg(w2 + u), gelu_f(z[x]), s);
    }
    s = warp_sum(s);
    if (lane == 0) scores[t] = s + b2;
}

__device__ __forceinline__ uint32_t order_bits_f(float f) {
    uint32_t u = __float_as_uint(f);
    if ((u & 0x7FFFFFFFu) == 0) u = 0;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Ascending bitonic sort of P u64 keys in shared memory by the whole block.
__device__ void bitonic_u64(uint64_t* keys, int P) {
    for (int k = 2; k <= P; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = threadIdx.x; i < P; i += blockDim.x) {
                const int ixj = i ^ j;
                if (ixj > i) {
                    const uint64_t a = keys[i], b = keys[ixj];
                    if ((a > b) == ((i & k) == 0)) {
                        keys[i] = b;
                        keys[ixj] = a;
                    }
                }
            }
            __syncthreads();
        }
    }
}

// Exclusive prefix sum of data[0..n) by the whole block; returns the total.
__device__ int merge_scan(int* data, int n, int* scratch) {
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

// 2. anchors: per image, the k largest scores (ties by id), listed by ascending id; rank[i]
//    = the anchor rank of token i, or -1.
__global__ void __launch_bounds__(kSortThreads)
    merge_topk_kernel(const float* __restrict__ scores, int N, int k, int32_t* __restrict__ anchors,
                      int32_t* __restrict__ rank) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int b = blockIdx.x, P = pow2_ge(N);
    uint64_t* keys = reinterpret_cast<uint64_t*>(smem);          // [P]
    int* flag = reinterpret_cast<int*>(keys + P);                 // [N]
    int* scratch = flag + N;                                      // [40]
    const float* sb = scores + static_cast<size_t>(b) * N;
    for (int i = threadIdx.x; i < P; i += kSortThreads)
        keys[i] = i < N ? ((static_cast<uint64_t>(~order_bits_f(sb[i])) << 32) | static_cast<uint32_t>(i))
                        : ~0ull;
    __syncthreads();
    bitonic_u64(keys, P);   // ascending: score descending, then id ascending
    for (int i = threadIdx.x; i < N; i += kSortThreads) flag[i] = 0;
    __syncthreads();
    for (int j = threadIdx.x; j < k; j += kSortThreads) flag[keys[j] & 0xffffffffu] = 1;
    __syncthreads();
    merge_scan(flag, N, scratch);   // flag[i] = number of anchors with a smaller id
    int32_t* ab = anchors + static_cast<size_t>(b) * k;
    int32_t* rb = rank + static_cast<size_t>(b) * N;
    for (int i = threadIdx.x; i < N; i += kSortThreads) {
        const int before = flag[i];
        const int after = i + 1 < N ? flag[i + 1] : k;
        const bool is_anchor = after > before;
        rb[i] = is_anchor ? before : -1;
        if (is_anchor) ab[before] = i;
    }
}

// 3. assignment: one thread per token; the CTA holds its image's anchor coordinates.
__global__ void __launch_bounds__(kMergeThreads)
    merge_assign_kernel(const float* __restrict__ xy, int N, int k, const int32_t* __restrict__ anchors,
                        const int32_t* __restrict__ rank, int32_t* __restrict__ assign) {
    extern __shared__ __align__(16) float2 axy[];  // [k]
    const int b = blockIdx.y;
    const float2* xb = reinterpret_cast<const float2*>(xy) + static_cast<size_t>(b) * N;
    const int32_t* ab = anchors + static_cast<size_t>(b) * k;
    for (int j = threadIdx.x; j < k; j += kMergeThreads) axy[j] = xb[ab[j]];
    __syncthreads();
    const int i = blockIdx.x * kMergeThreads + threadIdx.x;
    if (i >= N) return;
    const int r = rank[static_cast<size_t>(b) * N + i];
    if (r >= 0) {
        assign[static_cast<size_t>(b) * N + i] = r;
        return;
    }
    const float2 p = xb[i];
    const double px = p.x, py = p.y;
    double best = DBL_MAX;
    float bestf = FLT_MAX;
    int bj = 0;
    for (int j = 0; j < k; ++j) {
        const float2 a = axy[j];
        const float dxf = p.x - a.x, dyf = p.y - a.y;
        const float d2f = fmaf(dxf, dxf, dyf * dyf);
        if (d2f <= bestf) {   // a candidate beyond the fp32 bound cannot be nearer in fp64
            const double dx = __dsub_rn(px, static_cast<double>(a.x));
            const double dy = __dsub_rn(py, static_cast<double>(a.y));
            const double d2 = __dadd_rn(__dmul_rn(dx, dx), __dmul_rn(dy, dy));
            if (d2 < best) {  // strict: ties keep the lower anchor id
                best = d2;
                bj = j;
                bestf = static_cast<float>(best) * (1.0f + 1.0f / 1048576.0f);
            }
        }
    }
    assign[static_cast<size_t>(b) * N + i] = bj;
}

// 4. groups: per image, the tokens sorted by (assign, id) -> members [N] and the group
//    offsets goff [k + 1].
__global__ void __launch_bounds__(kSortThreads)
    merge_groups_kernel(const int32_t* __restrict__ assign, int N, int k, int32_t* __restrict__ members,
                        int32_t* __restrict__ goff) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int b = blockIdx.x, P = pow2_ge(N);
    uint64_t* keys = reinterpret_cast<uint64_t*>(smem);
    const int32_t* ab = assign + static_cast<size_t>(b) * N;
    for (int i = threadIdx.x; i < P; i += kSortThreads)
        keys[i] = i < N ? ((static_cast<uint64_t>(static_cast<uint32_t>(ab[i])) << 32) | static_cast<uint32_t>(i))
                        : ~0ull;
    __syncthreads();
    bitonic_u64(keys, P);
    int32_t* mb = members + static_cast<size_t>(b) * N;
    int32_t* gb = goff + static_cast<size_t>(b) * (k + 1);
    for (int i = threadIdx.x; i < N; i += kSortThreads) {
        const int a = static_cast<int>(keys[i] >> 32);
        mb[i] = static_cast<int32_t>(keys[i] & 0xffffffffu);
        const int prev = i > 0 ? static_cast<int>(keys[i - 1] >> 32) : -1;
        for (int g = prev + 1; g <= a; ++g) gb[g] = i;   // every group holds its anchor
    }
    if (threadIdx.x == 0) gb[k] = N;
}

// Softmax weights of a group's members, lanes over members (groups of any size).
__device__ __forceinline__ void group_softmax(const float* sb, const int32_t* mem, int n, int lane,
                                              float& gmax, float& gsum) {
    float m = -FLT_MAX;
    for (int x = lane; x < n; x += 32) m = fmaxf(m, sb[mem[x]]);
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float s = 0.f;
    for (int x = lane; x < n; x += 32) s += expf(sb[mem[x]] - m);
    gsum = warp_sum(s);
    gmax = m;
}

// 5. forward merge: one warp per anchor; lanes over channel pairs.
__global__ void __launch_bounds__(kMergeThreads)
    merge_fwd_kernel(const bf16* __restrict__ feats, const float* __restrict__ xy, int B, int N, int d,
                     int k, const float* __restrict__ scores, const int32_t* __restrict__ members,
                     const int32_t* __restrict__ goff, bf16* __restrict__ merged, float* __restrict__ mxy) {
    const int lane = threadIdx.x & 31;
    const long long ga = static_cast<long long>(blockIdx.x) * kMergeWarps + (threadIdx.x >> 5);
    if (ga >= static_cast<long long>(B) * k) return;
    const int b = static_cast<int>(ga / k), j = static_cast<int>(ga - static_cast<long long>(b) * k);
    const float* sb = scores + static_cast<size_t>(b) * N;
    const int32_t* mem = members + static_cast<size_t>(b) * N;
    const int32_t* gb = goff + static_cast<size_t>(b) * (k + 1);
    const int g0 = gb[j], n = gb[j + 1] - g0;
    float gmax, gsum;
    group_softmax(sb, mem + g0, n, lane, gmax, gsum);
    const float inv = 1.f / gsum;
    const bf16* fb = feats + static_cast<size_t>(b) * N * d;
    for (int c0 = 0; c0 < d; c0 += 64) {
        const int c = c0 + 2 * lane;
        float a0 = 0.f, a1 = 0.f;
        for (int x = 0; x < n; ++x) {
            const int t = mem[g0 + x];
            const float w = expf(sb[t] - gmax) * inv;
            if (c < d) {
                const uint32_t pr = *reinterpret_cast<const uint32_t*>(fb + static_cast<size_t>(t) * d + c);
                a0 = fmaf(w, bf16_lo(pr), a0);
                a1 = fmaf(w, bf16_hi(pr), a1);
            }
        }
        if (c < d) {
            const __nv_bfloat162 hv = __floats2bfloat162_rn(a0, a1);
            *reinterpret_cast<__nv_bfloat162*>(merged + (static_cast<size_t>(b) * k + j) * d + c) = hv;
        }
    }
    if (lane < 2) {
        const float2* xb = reinterpret_cast<const float2*>(xy) + static_cast<size_t>(b) * N;
        float acc = 0.f;
        for (int x = 0; x < n; ++x) {
            const int t = mem[g0 + x];
            const float2 p = xb[t];
            acc = fmaf(expf(sb[t] - gmax) * inv, lane ? p.y : p.x, acc);
        }
        mxy[(static_cast<size_t>(b) * k + j) * 2 + lane] = acc;
    }
}

// 6. backward per group: one warp per anchor, its members in order.  Writes dfeats (bf16),
//    dcoords, and per token ds and dh (fp32, workspace) for the parameter gradients.
template <int HP>
__global__ void __launch_bounds__(kMergeThreads)
    merge_bwd_group_kernel(const bf16* __restrict__ feats, const float* __restrict__ xy, int B, int N,
                           int d, int k, const float* __restrict__ w1, const float* __restrict__ b1,
                           const float* __restrict__ w2, int h, const float* __restrict__ scores,
                           const int32_t* __restrict__ members, const int32_t* __restrict__ goff,
                           const bf16* __restrict__ dmerged, const float* __restrict__ dmxy,
                           bf16* __restrict__ dfeats, float* __restrict__ dxy, float* __restrict__ ds_out,
                           float* __restrict__ dh_out, float* __restrict__ gz_out) {
    const int lane = threadIdx.x & 31;
    const long long ga = static_cast<long long>(blockIdx.x) * kMergeWarps + (threadIdx.x >> 5);
    if (ga >= static_cast<long long>(B) * k) return;
    const int b = static_cast<int>(ga / k), j = static_cast<int>(ga - static_cast<long long>(b) * k);
    const float* sb = scores + static_cast<size_t>(b) * N;
    const int32_t* mem = members + static_cast<size_t>(b) * N;
    const int32_t* gb = goff + static_cast<size_t>(b) * (k + 1);
    const int g0 = gb[j], n = gb[j + 1] - g0;
    float gmax, gsum;
    group_softmax(sb, mem + g0, n, lane, gmax, gsum);
    const float inv = 1.f / gsum;
    const bf16* fb = feats + static_cast<size_t>(b) * N * d;
    const bf16* dF = dmerged + (static_cast<size_t>(b) * k + j) * d;
    const float dX0 = dmxy[(static_cast<size_t>(b) * k + j) * 2], dX1 = dmxy[(static_cast<size_t>(b) * k + j) * 2 + 1];
    const float2* xb = reinterpret_cast<const float2*>(xy) + static_cast<size_t>(b) * N;
    // sum_G w g, g_i = <dF, f_i> + <dX, x_i>
    float sg = 0.f;
    for (int x = 0; x < n; ++x) {
        const int t = mem[g0 + x];
        float acc = 0.f;
        for (int c = 2 * lane; c < d; c += 64) {
            const uint32_t pf = *reinterpret_cast<const uint32_t*>(fb + static_cast<size_t>(t) * d + c);
            const uint32_t pg = *reinterpret_cast<const uint32_t*>(dF + c);
            acc = fmaf(bf16_lo(pf), bf16_lo(pg), acc);
            acc = fmaf(bf16_hi(pf), bf16_hi(pg), acc);
        }
        const float2 p = xb[t];
        const float gi = warp_sum(acc) + dX0 * p.x + dX1 * p.y;
        sg = fmaf(expf(sb[t] - gmax) * inv, gi, sg);
    }
    for (int x = 0; x < n; ++x) {
        const int t = mem[g0 + x];
        const size_t gt = static_cast<size_t>(b) * N + t;
        const bf16* frow = fb + static_cast<size_t>(t) * d;
        float acc = 0.f;
        for (int c = 2 * lane; c < d; c += 64) {
            const uint32_t pf = *reinterpret_cast<const uint32_t*>(frow + c);
            const uint32_t pg = *reinterpret_cast<const uint32_t*>(dF + c);
            acc = fmaf(bf16_lo(pf), bf16_lo(pg), acc);
            acc = fmaf(bf16_hi(pf), bf16_hi(pg), acc);
        }
        const float2 p = xb[t];
        const float gi = warp_sum(acc) + dX0 * p.x + dX1 * p.y;
        const float w = expf(sb[t] - gmax) * inv;
        const float ds = w * (gi - sg);
        // MLP backward of this token
        float z[HP], dh[HP];
        hidden_pre<HP>(frow, d, w1, b1, h, lane, z);
#pragma unroll
        for (int y = 0; y < HP; ++y) {
            const int u = lane + 32 * y;
            dh[y] = u < h ? ds * __ldg(w2 + u) * gelu_grad_f(z[y]) : 0.f;
            if (u < h) {
                dh_out[gt * h + u] = dh[y];
                gz_out[gt * h + u] = gelu_f(z[y]);
            }
        }
        if (lane == 0) ds_out[gt] = ds;
        if (lane < 2) reinterpret_cast<float*>(dxy)[gt * 2 + lane] = w * (lane ? dX1 : dX0);
        // df = w dF + W1 dh: lane owns channel pairs; dh broadcast by shuffles
        for (int c0 = 0; c0 < d; c0 += 64) {
            const int c = c0 + 2 * lane;
            float a0 = 0.f, a1 = 0.f;
            if (c < d) {
                const uint32_t pg = *reinterpret_cast<const uint32_t*>(dF + c);
                a0 = w * bf16_lo(pg);
                a1 = w * bf16_hi(pg);
            }
#pragma unroll
            for (int y = 0; y < HP; ++y) {
                for (int ul = 0; ul < 32; ++ul) {
                    const int u = ul + 32 * y;
                    const float dhu = __shfl_sync(0xffffffffu, dh[y], ul);
                    if (u < h && c < d) {
                        a0 = fmaf(__ldg(w1 + static_cast<size_t>(c) * h + u), dhu, a0);
                        a1 = fmaf(__ldg(w1 + static_cast<size_t>(c + 1) * h + u), dhu, a1);
                    }
                }
            }
            if (c < d)
                *reinterpret_cast<__nv_bfloat162*>(dfeats + gt * d + c) = __floats2bfloat162_rn(a0, a1);
        }
    }
}

// 7. parameter gradients, stage 1: CTA p sums tokens [p T / P, (p + 1) T / P) in order;
//    thread tid owns outputs o = tid, tid + 256, ... of [dW1 (d*h) | db1 (h) | dw2 (h) | db2].
__global__ void __launch_bounds__(kMergeThreads)
    merge_param_part_kernel(const bf16* __restrict__ feats, int T, int d, int h,
                            const float* __restrict__ ds, const float* __restrict__ dh,
                            const float* __restrict__ gz, float* __restrict__ part) {
    extern __shared__ __align__(16) float tile[];  // [kParamTile][d] f, then [kParamTile][h] dh, gz
    float* ft = tile;
    float* dht = ft + kParamTile * d;
    float* gzt = dht + kParamTile * h;
    float* dst = gzt + kParamTile * h;
    const int p = blockIdx.x;
    const int t0 = static_cast<int>(static_cast<long long>(p) * T / kParamParts);
    const int t1 = static_cast<int>(static_cast<long long>(p + 1) * T / kParamParts);
    const int nout = d * h + 2 * h + 1;
    constexpr int kPer = 16;  // outputs per thread held in registers per pass
    for (int ob = 0; ob < nout; ob += kMergeThreads * kPer) {
        float acc[kPer];
#pragma unroll
        for (int q = 0; q < kPer; ++q) acc[q] = 0.f;
        for (int tt = t0; tt < t1; tt += kParamTile) {
            const int nt = min(kParamTile, t1 - tt);
            __syncthreads();
            for (int i = threadIdx.x; i < nt * d; i += kMergeThreads) {
                const int r = i / d, c = i - r * d;
                ft[r * d + c] = __bfloat162float(feats[static_cast<size_t>(tt + r) * d + c]);
            }
            for (int i = threadIdx.x; i < nt * h; i += kMergeThreads) {
                const int r = i / h, u = i - r * h;
                dht[r * h + u] = dh[static_cast<size_t>(tt + r) * h + u];
                gzt[r * h + u] = gz[static_cast<size_t>(tt + r) * h + u];
            }
            for (int i = threadIdx.x; i < nt; i += kMergeThreads) dst[i] = ds[tt + i];
            __syncthreads();
#pragma unroll
            for (int q = 0; q < kPer; ++q) {
                const int o = ob + q * kMergeThreads + threadIdx.x;
                if (o >= nout) continue;
                float a = acc[q];
                if (o < d * h) {
                    const int c = o / h, u = o - c * h;
                    for (int r = 0; r < nt; ++r) a = fmaf(ft[r * d + c], dht[r * h + u], a);
                } else if (o < d * h + h) {
                    const int u = o - d * h;
                    for (int r = 0; r < nt; ++r) a += dht[r * h + u];
                } else if (o < d * h + 2 * h) {
                    const int u = o - d * h - h;
                    for (int r = 0; r < nt; ++r) a = fmaf(dst[r], gzt[r * h + u], a);
                } else {
                    for (int r = 0; r < nt; ++r) a += dst[r];
                }
                acc[q] = a;
            }
        }
#pragma unroll
        for (int q = 0; q < kPer; ++q) {
            const int o = ob + q * kMergeThreads + threadIdx.x;
            if (o < nout) part[static_cast<size_t>(p) * nout + o] = acc[q];
        }
    }
}

// 8. parameter gradients, stage 2: the parts summed in order.
__global__ void __launch_bounds__(kMergeThreads)
    merge_param_reduce_kernel(const float* __restrict__ part, int d, int h, float* __restrict__ dw1,
                              float* __restrict__ db1, float* __restrict__ dw2, float* __restrict__ db2) {
    const int nout = d * h + 2 * h + 1;
    const int o = blockIdx.x * kMergeThreads + threadIdx.x;
    if (o >= nout) return;
    float a = 0.f;
    for (int p = 0; p < kParamParts; ++p) a += part[static_cast<size_t>(p) * nout + o];
    if (o < d * h) dw1[o] = a;
    else if (o < d * h + h) db1[o - d * h] = a;
    else if (o < d * h + 2 * h) dw2[o - d * h - h] = a;
    else *db2 = a;
}

size_t sort_smem(int N) { return 8 * static_cast<size_t>(pow2_ge(N)) + 4 * static_cast<size_t>(N) + 40 * 4; }

}  // namespace

MergeWorkspace merge_workspace_layout(int B, int N, int d, int h, int k) {
    auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
    const size_t T = static_cast<size_t>(B) * N;
    MergeWorkspace w;
    size_t off = 0;
    w.rank = off;    off += up(sizeof(int32_t) * T);
    w.members = off; off += up(sizeof(int32_t) * T);
    w.goff = off;    off += up(sizeof(int32_t) * static_cast<size_t>(B) * (k + 1));
    w.ds = off;      off += up(sizeof(float) * T);
    w.dh = off;      off += up(sizeof(float) * T * h);
    w.gz = off;      off += up(sizeof(float) * T * h);
    w.part = off;    off += up(sizeof(float) * kParamParts * (static_cast<size_t>(d) * h + 2 * h + 1));
    w.total = off;
    return w;
}

size_t merge_smem_bytes(int N, int k, int d, int h) {
    const size_t s = sort_smem(N);
    const size_t a = 8 * static_cast<size_t>(k);
    const size_t p = sizeof(float) * (static_cast<size_t>(kParamTile) * (d + 2 * h) + kParamTile);
    size_t m = s > a ? s : a;
    return m > p ? m : p;
}

#define ACL_HP_SWITCH(h, CALL)                        \
    switch (((h) + 31) / 32) {                        \
        case 1: { constexpr int HP = 1; CALL; } break; \
        case 2: { constexpr int HP = 2; CALL; } break; \
        case 3: case 4: { constexpr int HP = 4; CALL; } break; \
        default: { constexpr int HP = 8; CALL; } break; \
    }

cudaError_t launch_merge_fwd(const MergeArgs& m, cudaStream_t st) {
    const int T = m.B * m.N;
    cudaError_t e;
    const unsigned sblocks = static_cast<unsigned>((T + kMergeWarps - 1) / kMergeWarps);
    ACL_HP_SWITCH(m.h, (merge_scores_kernel<HP><<<sblocks, kMergeThreads, 0, st>>>(
                           m.feats, T, m.d, m.w1, m.b1, m.w2, m.b2, m.h, m.scores)));
    note_launch();
    const size_t ssm = sort_smem(m.N);
    if ((e = ensure_smem<merge_topk_kernel>(ssm)) != cudaSuccess) return e;
    merge_topk_kernel<<<m.B, kSortThreads, ssm, st>>>(m.scores, m.N, m.k, m.anchors, m.rank);
    note_launch();
    const size_t asm_ = 8 * static_cast<size_t>(m.k);
    if ((e = ensure_smem<merge_assign_kernel>(asm_)) != cudaSuccess) return e;
    merge_assign_kernel<<<dim3((m.N + kMergeThreads - 1) / kMergeThreads, m.B), kMergeThreads, asm_, st>>>(
        m.xy, m.N, m.k, m.anchors, m.rank, m.assign);
    note_launch();
    if ((e = ensure_smem<merge_groups_kernel>(ssm)) != cudaSuccess) return e;
    merge_groups_kernel<<<m.B, kSortThreads, ssm, st>>>(m.assign, m.N, m.k, m.members, m.goff);
    note_launch();
    const long long na = static_cast<long long>(m.B) * m.k;
    merge_fwd_kernel<<<static_cast<unsigned>((na + kMergeWarps - 1) / kMergeWarps), kMergeThreads, 0, st>>>(
        m.feats, m.xy, m.B, m.N, m.d, m.k, m.scores, m.members, m.goff, m.merged, m.mxy);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_merge_bwd(const MergeArgs& m, cudaStream_t st) {
    const int T = m.B * m.N;
    cudaError_t e;
    const size_t ssm = sort_smem(m.N);
    if ((e = ensure_smem<merge_groups_kernel>(ssm)) != cudaSuccess) return e;
    merge_groups_kernel<<<m.B, kSortThreads, ssm, st>>>(m.assign, m.N, m.k, m.members, m.goff);
    note_launch();
    const long long na = static_cast<long long>(m.B) * m.k;
    const unsigned gblocks = static_cast<unsigned>((na + kMergeWarps - 1) / kMergeWarps);
    ACL_HP_SWITCH(m.h, (merge_bwd_group_kernel<HP><<<gblocks, kMergeThreads, 0, st>>>(
                           m.feats, m.xy, m.B, m.N, m.d, m.k, m.w1, m.b1, m.w2, m.h, m.scores,
                           m.members, m.goff, m.dmerged, m.dmxy, m.dfeats, m.dxy, m.ds, m.dh, m.gz)));
    note_launch();
    const size_t psm = sizeof(float) * (static_cast<size_t>(kParamTile) * (m.d + 2 * m.h) + kParamTile);
    if ((e = ensure_smem<merge_param_part_kernel>(psm)) != cudaSuccess) return e;
    merge_param_part_kernel<<<kParamParts, kMergeThreads, psm, st>>>(m.feats, T, m.d, m.h, m.ds, m.dh,
                                                                      m.gz, m.part);
    note_launch();
    const int nout = m.d * m.h + 2 * m.h + 1;
    merge_param_reduce_kernel<<<(nout + kMergeThreads - 1) / kMergeThreads, kMergeThreads, 0, st>>>(
        m.part, m.d, m.h, m.dw1, m.db1, m.dw2, m.db2);
    note_launch();
    return cudaGetLastError();
}

#undef ACL_HP_SWITCH

}  // namespace acl
