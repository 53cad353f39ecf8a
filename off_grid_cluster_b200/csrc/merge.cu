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
// No atomics in any sum: groups are listed by a counting sort whose order within a group is
// fixed by ranking ids, every token belongs to one group, and the parameter gradients are
// reduced in two fixed-order stages.
//
// Kernels.  Forward: scores (token-parallel, 4 lanes per token, W1 broadcast from shared
// memory) -> rank by counting (anchor flags) -> assignment (each CTA rebuilds the anchor list
// from the flags, then a nearest-anchor search with 4 lanes per token) -> groups (counting
// sort) -> merge (one warp per anchor).  Backward: groups -> group statistics (one warp per
// anchor: softmax max, 1/sum and sum_G w g) -> token pass (4 lanes per token: g, ds, the MLP
// backward, dfeats) -> parameter partial sums (4x4 register tiles over token ranges) -> the
// fixed-order sum of the parts.
#include <float.h>

#include "internal.h"

namespace acl {

namespace {

constexpr int kMergeWarps = 8;
constexpr int kMergeThreads = 32 * kMergeWarps;
constexpr int kSortThreads = 1024;
constexpr int kSub = 4;                               // lanes per token (token-parallel kernels)
constexpr int kTokPerWarp = 32 / kSub;
constexpr int kTokPerCta = kMergeWarps * kTokPerWarp;
constexpr int kTokCtasPerSm = 4;                      // grid cap of the token-parallel kernels
constexpr int kAssignSub = 4;                         // lanes per token in the nearest-anchor search
constexpr int kParamParts = 296;                      // token ranges of the parameter partial sums
constexpr int kParamTile = 32;                        // tokens staged per step of that stage
constexpr size_t kW1SmemMax = 96 * 1024;              // W1 staged in shared memory up to this size

__device__ __forceinline__ float gelu_f(float z) { return 0.5f * z * (1.f + erff(z * 0.70710678118654752f)); }
__device__ __forceinline__ float gelu_grad_f(float z) {
    return 0.5f * (1.f + erff(z * 0.70710678118654752f)) + z * 0.39894228040143268f * expf(-0.5f * z * z);
}

// Hidden units are held 8 HP per lane: lane sub-index s (of kSub) owns the float4 groups
// 4 s + 16 y (y < 2 HP), so the four lanes of a token read 64 contiguous bytes of a W1 row.
// W1 in shared memory: rows of kHS(HP) floats (h padded with zeros, +4 so that rows two
// apart start 32 bytes apart in the banks).
template <int HP>
constexpr int kHS = 32 * HP + 4;

template <int HP>
__device__ void stage_w1(float* w1s, const float* __restrict__ w1, int d, int h) {
#pragma unroll 4
    for (int i = threadIdx.x; i < d * kHS<HP>; i += blockDim.x) {
        const int c = i / kHS<HP>, u = i - c * kHS<HP>;
        w1s[i] = u < h ? w1[static_cast<size_t>(c) * h + u] : 0.f;
    }
}

// W1[c][u0 .. u0 + 3]: from the padded shared copy, or from global memory (rows of h).
template <bool SM>
__device__ __forceinline__ float4 w1_load4(const float* w, int stride, int h, int c, int u0) {
    if constexpr (SM) {
        return *reinterpret_cast<const float4*>(w + c * stride + u0);
    } else {
        const float* row = w + static_cast<size_t>(c) * h;
        return make_float4(u0 < h ? __ldg(row + u0) : 0.f, u0 + 1 < h ? __ldg(row + u0 + 1) : 0.f,
                           u0 + 2 < h ? __ldg(row + u0 + 2) : 0.f, u0 + 3 < h ? __ldg(row + u0 + 3) : 0.f);
    }
}

// Pre-activations z = b1 + W1^T f of one token for the units lane s owns (zero beyond h).
template <int HP, bool SM>
__device__ __forceinline__ void hidden4(const bf16* frow, int d, const float* w, int h,
                                        const float* b1s, int s, float (&z)[8 * HP]) {
#pragma unroll
    for (int y = 0; y < 2 * HP; ++y) {
        const float4 b = *reinterpret_cast<const float4*>(b1s + 4 * s + 16 * y);
        z[4 * y] = b.x;
        z[4 * y + 1] = b.y;
        z[4 * y + 2] = b.z;
        z[4 * y + 3] = b.w;
    }
    // 32 channels per step (d % 32 == 0), the next step's four 16-byte chunks loaded ahead
    uint4 cur[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) cur[q] = ldg16(frow + 8 * q);
    for (int c0 = 0; c0 < d; c0 += 32) {
        uint4 nxt[4];
        if (c0 + 32 < d) {
#pragma unroll
            for (int q = 0; q < 4; ++q) nxt[q] = ldg16(frow + c0 + 32 + 8 * q);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t fw[4] = {cur[q].x, cur[q].y, cur[q].z, cur[q].w};
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float fc = (e & 1) ? bf16_hi(fw[e >> 1]) : bf16_lo(fw[e >> 1]);
                const int c = c0 + 8 * q + e;
#pragma unroll
                for (int y = 0; y < 2 * HP; ++y) {
                    const float4 w4 = w1_load4<SM>(w, kHS<HP>, h, c, 4 * s + 16 * y);
                    z[4 * y] = fmaf(fc, w4.x, z[4 * y]);
                    z[4 * y + 1] = fmaf(fc, w4.y, z[4 * y + 1]);
                    z[4 * y + 2] = fmaf(fc, w4.z, z[4 * y + 2]);
                    z[4 * y + 3] = fmaf(fc, w4.w, z[4 * y + 3]);
                }
            }
        }
        if (c0 + 32 < d) {
#pragma unroll
            for (int q = 0; q < 4; ++q) cur[q] = nxt[q];
        }
    }
}

// b1 and w2 in shared memory, zero beyond h.
template <int HP>
__device__ __forceinline__ void stage_bias(float* b1s, float* w2s, const float* __restrict__ b1,
                                           const float* __restrict__ w2, int h) {
    for (int u = threadIdx.x; u < 32 * HP; u += blockDim.x) {
        b1s[u] = u < h ? b1[u] : 0.f;
        w2s[u] = u < h ? w2[u] : 0.f;
    }
}

// 1. scores: four lanes per token, eight tokens per warp, warps striding over the tokens.
template <int HP, bool SM>
__global__ void __launch_bounds__(kMergeThreads)
    merge_scores_kernel(const bf16* __restrict__ feats, int T, int d, const float* __restrict__ w1,
                        const float* __restrict__ b1, const float* __restrict__ w2, float b2, int h,
                        float* __restrict__ scores) {
    extern __shared__ __align__(16) float w1s[];  // [d][kHS] when SM
    __shared__ __align__(16) float b1s[32 * HP];
    __shared__ __align__(16) float w2s[32 * HP];
    stage_bias<HP>(b1s, w2s, b1, w2, h);
    if constexpr (SM) stage_w1<HP>(w1s, w1, d, h);
    __syncthreads();
    const float* w = SM ? w1s : w1;
    const int lane = threadIdx.x & 31, s = lane & (kSub - 1), tw = lane / kSub;
    const int warp_g = blockIdx.x * kMergeWarps + (threadIdx.x >> 5);
    for (int base = warp_g * kTokPerWarp; base < T; base += gridDim.x * kTokPerCta) {  // warp-uniform
        const int t = base + tw;
        const bool live = t < T;
        float z[8 * HP];
        hidden4<HP, SM>(feats + static_cast<size_t>(live ? t : base) * d, d, w, h, b1s, s, z);
        float acc = 0.f;
#pragma unroll
        for (int y = 0; y < 2 * HP; ++y)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc = fmaf(w2s[4 * s + 16 * y + e], gelu_f(z[4 * y + e]), acc);
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
        if (live && s == 0) scores[t] = acc + b2;
    }
}

// ---------------------------------------------------------- tensor-core MLP
//
// For d a multiple of 64 up to 256 and h a multiple of 16 up to 64, the hidden layer runs on
// the tensor cores:
// one warp per 16 tokens, z (16 x h) = F (16 x d, bf16: exact) . W1 by m16n8k16 bf16 MMAs with
// fp32 accumulation, W1 split into bf16 hi + lo (hi = bf16(w), lo = bf16(w - hi): about 16
// significant bits, two MMAs per tile).  The features are staged per warp by cp.async in
// shared-memory rows of d + 8 elements and W1 as [h][d + 8] (unit rows), both read by
// ldmatrix without bank conflicts.
constexpr int kMmaMaxD = 256, kMmaMaxH = 64;

// the backward's dfeats pass takes 64 channels at a time, so d % 64 == 0
bool mlp_mma_ok(int d, int h) { return d % 64 == 0 && d <= kMmaMaxD && h % 16 == 0 && h <= kMmaMaxH; }

struct MlpSmem {
    size_t w1t_hi, w1t_lo, w1_hi, w1_lo, b1, w2, f, total;
};
// bwd: also W1 as [d][h + 8] (channel rows) hi + lo, the B operand of dh . W1^T
__host__ __device__ inline MlpSmem mlp_smem(int d, int h, bool bwd) {
    MlpSmem L;
    size_t o = 0;
    const size_t wt = static_cast<size_t>(h) * (d + 8) * 2, w = static_cast<size_t>(d) * (h + 8) * 2;
    L.w1t_hi = o; o += wt;
    L.w1t_lo = o; o += wt;
    L.w1_hi = o; o += bwd ? w : 0;
    L.w1_lo = o; o += bwd ? w : 0;
    o = (o + 15) & ~size_t(15);
    L.b1 = o; o += 4 * static_cast<size_t>(h);
    L.w2 = o; o += 4 * static_cast<size_t>(h);
    o = (o + 15) & ~size_t(15);
    L.f = o; o += static_cast<size_t>(kMergeWarps) * 16 * (d + 8) * 2;
    L.total = o;
    return L;
}

__device__ void stage_mlp(const MlpSmem& L, uint8_t* sm, const float* __restrict__ w1, const float* __restrict__ b1,
                          const float* __restrict__ w2, int d, int h, bool bwd) {
    bf16* th = reinterpret_cast<bf16*>(sm + L.w1t_hi);
    bf16* tl = reinterpret_cast<bf16*>(sm + L.w1t_lo);
    bf16* wh = reinterpret_cast<bf16*>(sm + L.w1_hi);
    bf16* wl = reinterpret_cast<bf16*>(sm + L.w1_lo);
    for (int i = threadIdx.x; i < d * h; i += blockDim.x) {
        const int c = i / h, u = i - c * h;
        const float w = w1[i];
        const bf16 hi = __float2bfloat16_rn(w);
        const bf16 lo = __float2bfloat16_rn(w - __bfloat162float(hi));
        th[u * (d + 8) + c] = hi;
        tl[u * (d + 8) + c] = lo;
        if (bwd) {
            wh[c * (h + 8) + u] = hi;
            wl[c * (h + 8) + u] = lo;
        }
    }
    float* b1s = reinterpret_cast<float*>(sm + L.b1);
    float* w2s = reinterpret_cast<float*>(sm + L.w2);
    for (int u = threadIdx.x; u < h; u += blockDim.x) {
        b1s[u] = b1[u];
        w2s[u] = w2[u];
    }
}

// 16 feature rows (tokens t0 .. t0 + 15 of T) into the warp's tile; rows past T are zero.
__device__ __forceinline__ void load_f_tile(uint32_t tile, const bf16* __restrict__ feats, int t0, int T, int d,
                                            int lane) {
    const int cpr = d / 8;  // 16-byte chunks per row
    for (int q = lane; q < 16 * cpr; q += 32) {
        const int r = q / cpr, ch = q - r * cpr;
        const bool ok = t0 + r < T;
        cp_async16(tile + (r * (d + 8) + ch * 8) * 2, ok ? feats + static_cast<size_t>(t0 + r) * d + ch * 8 : feats, ok);
    }
    cp_async_commit();
}

// z = F . W1 for the warp's 16-token tile: lane (g, t) holds rows g and g + 8, units 8 nt + 2t, +1.
template <int NT>
__device__ __forceinline__ void z_mma(uint32_t ftile, uint32_t whi, uint32_t wlo, int d, int lane,
                                      float (&acc)[NT][4]) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
    const int rb = (d + 8) * 2;  // row bytes of the feature and W1 tiles
    const int mi = lane >> 3, r8 = lane & 7;
    for (int ks = 0; ks < d / 16; ++ks) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4(ftile + (lane & 15) * rb + (2 * ks + (lane >> 4)) * 16, a0, a1, a2, a3);
#pragma unroll
        for (int pr = 0; pr < NT / 2; ++pr) {
            const uint32_t off = (16 * pr + 8 * (mi >> 1) + r8) * rb + (2 * ks + (mi & 1)) * 16;
            uint32_t h0, h1, h2, h3, l0, l1, l2, l3;
            ldsm_x4(whi + off, h0, h1, h2, h3);
            ldsm_x4(wlo + off, l0, l1, l2, l3);
            mma_bf16(acc[2 * pr], a0, a1, a2, a3, h0, h1);
            mma_bf16(acc[2 * pr], a0, a1, a2, a3, l0, l1);
            mma_bf16(acc[2 * pr + 1], a0, a1, a2, a3, h2, h3);
            mma_bf16(acc[2 * pr + 1], a0, a1, a2, a3, l2, l3);
        }
    }
}

// 1'. scores on the tensor cores: warps stride over 16-token tiles.
template <int NT>
__global__ void __launch_bounds__(kMergeThreads)
    merge_scores_mma_kernel(const bf16* __restrict__ feats, int T, int d, const float* __restrict__ w1,
                            const float* __restrict__ b1, const float* __restrict__ w2, float b2,
                            float* __restrict__ scores) {
    extern __shared__ __align__(16) uint8_t msm[];
    constexpr int h = 8 * NT;
    const MlpSmem L = mlp_smem(d, h, false);
    stage_mlp(L, msm, w1, b1, w2, d, h, false);
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const uint32_t base = smem_addr(msm);
    const uint32_t ftile = base + static_cast<uint32_t>(L.f) + warp * 16 * (d + 8) * 2;
    const float* b1s = reinterpret_cast<const float*>(msm + L.b1);
    const float* w2s = reinterpret_cast<const float*>(msm + L.w2);
    for (int t0 = (blockIdx.x * kMergeWarps + warp) * 16; t0 < T; t0 += gridDim.x * kMergeWarps * 16) {
        load_f_tile(ftile, feats, t0, T, d, lane);
        cp_async_wait<0>();
        __syncwarp();
        float acc[NT][4];
        z_mma<NT>(ftile, base + static_cast<uint32_t>(L.w1t_hi), base + static_cast<uint32_t>(L.w1t_lo), d, lane, acc);
        float s0 = 0.f, s1 = 0.f;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int u = 8 * nt + 2 * t + e;
                s0 = fmaf(w2s[u], gelu_f(acc[nt][e] + b1s[u]), s0);
                s1 = fmaf(w2s[u], gelu_f(acc[nt][2 + e] + b1s[u]), s1);
            }
        s0 += __shfl_xor_sync(0xffffffffu, s0, 1);
        s0 += __shfl_xor_sync(0xffffffffu, s0, 2);
        s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
        s1 += __shfl_xor_sync(0xffffffffu, s1, 2);
        if (t == 0) {
            if (t0 + g < T) scores[t0 + g] = s0 + b2;
            if (t0 + g + 8 < T) scores[t0 + g + 8] = s1 + b2;
        }
        __syncwarp();  // the tile is read before the next one is loaded
    }
}

// 7'. backward token pass on the tensor cores: one warp per 16 tokens.  Lane (g, t) owns rows g
//     and g + 8: their weight, ds, dx; z again by z_mma; dh = ds w2 gelu'(z) and e = ds gelu(z)
//     for its units (written for the parameter sums); then dfeats = w dF + dh . W1^T with dh
//     (bf16 hi + lo, straight from the accumulator layout) as the A operand and W1 ([d][h + 8],
//     hi + lo) as B, 64 channels at a time, three MMAs per tile (hi.hi, hi.lo, lo.hi).
template <int NT>
__global__ void __launch_bounds__(kMergeThreads)
    merge_bwd_token_mma_kernel(const bf16* __restrict__ feats, const float* __restrict__ xy, int T, int N,
                               int d, int k, const float* __restrict__ w1, const float* __restrict__ b1,
                               const float* __restrict__ w2, const float* __restrict__ scores,
                               const int32_t* __restrict__ assign, const float4* __restrict__ gstat,
                               const float* __restrict__ gtok, const bf16* __restrict__ dmerged,
                               const float* __restrict__ dmxy, bf16* __restrict__ dfeats, float* __restrict__ dxy,
                               float* __restrict__ ds_out, float* __restrict__ dh_out, float* __restrict__ e_out) {
    extern __shared__ __align__(16) uint8_t msm[];
    constexpr int h = 8 * NT;
    const MlpSmem L = mlp_smem(d, h, true);
    stage_mlp(L, msm, w1, b1, w2, d, h, true);
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3, mi = lane >> 3, r8 = lane & 7;
    const uint32_t base = smem_addr(msm);
    const uint32_t ftile = base + static_cast<uint32_t>(L.f) + warp * 16 * (d + 8) * 2;
    const uint32_t wh = base + static_cast<uint32_t>(L.w1_hi), wl = base + static_cast<uint32_t>(L.w1_lo);
    const float* b1s = reinterpret_cast<const float*>(msm + L.b1);
    const float* w2s = reinterpret_cast<const float*>(msm + L.w2);
    constexpr int rbw = (h + 8) * 2;  // row bytes of W1 [d][h + 8]
    for (int t0 = (blockIdx.x * kMergeWarps + warp) * 16; t0 < T; t0 += gridDim.x * kMergeWarps * 16) {
        load_f_tile(ftile, feats, t0, T, d, lane);
        // rows g and g + 8: weight, ds, anchor row
        float wt[2], ds[2];
        size_t arow[2];
        bool live[2];
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
            const int tk = t0 + g + 8 * rr;
            live[rr] = tk < T;
            const int tc = live[rr] ? tk : t0;
            const int bimg = tc / N;
            const int a = assign[tc];
            const bool ok = live[rr] && a >= 0 && a < k;
            arow[rr] = static_cast<size_t>(bimg) * k + (ok ? a : 0);
            const float4 gs = gstat[arow[rr]];
            wt[rr] = ok ? expf(scores[tc] - gs.x) * gs.y : 0.f;
            ds[rr] = ok ? wt[rr] * (gtok[tc] - gs.z) : 0.f;
            if (live[rr] && t == 0) {
                ds_out[tk] = ds[rr];
                const float2 dX = reinterpret_cast<const float2*>(dmxy)[arow[rr]];
                reinterpret_cast<float2*>(dxy)[tk] = make_float2(wt[rr] * dX.x, wt[rr] * dX.y);
            }
        }
        cp_async_wait<0>();
        __syncwarp();
        float acc[NT][4];
        z_mma<NT>(ftile, base + static_cast<uint32_t>(L.w1t_hi), base + static_cast<uint32_t>(L.w1t_lo), d, lane, acc);
        // dh and e for the lane's units; dh packed as the A operand (hi, lo) of dh . W1^T
        uint32_t ahi[NT / 2][4], alo[NT / 2][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            float dh[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int u = 8 * nt + 2 * t + (e & 1), rr = e >> 1;
                const float z = acc[nt][e] + b1s[u];
                dh[e] = ds[rr] * w2s[u] * gelu_grad_f(z);
                if (live[rr]) {
                    const size_t o = static_cast<size_t>(t0 + g + 8 * rr) * h + u;
                    dh_out[o] = dh[e];
                    e_out[o] = ds[rr] * gelu_f(z);
                }
            }
            const uint32_t h01 = pack_bf16(dh[0], dh[1]), h23 = pack_bf16(dh[2], dh[3]);
            const uint32_t l01 = pack_bf16(dh[0] - bf16_lo(h01), dh[1] - bf16_hi(h01));
            const uint32_t l23 = pack_bf16(dh[2] - bf16_lo(h23), dh[3] - bf16_hi(h23));
            const int ks = nt >> 1, hf = nt & 1;  // n-tile 2 ks: A regs 0, 1; n-tile 2 ks + 1: regs 2, 3
            ahi[ks][2 * hf] = h01;
            ahi[ks][2 * hf + 1] = h23;
            alo[ks][2 * hf] = l01;
            alo[ks][2 * hf + 1] = l23;
        }
        // dfeats, 64 channels at a time
        for (int c0 = 0; c0 < d; c0 += 64) {
            float dfa[8][4];
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) dfa[nt][0] = dfa[nt][1] = dfa[nt][2] = dfa[nt][3] = 0.f;
#pragma unroll
            for (int ks = 0; ks < NT / 2; ++ks) {
#pragma unroll
                for (int pr = 0; pr < 4; ++pr) {
                    const uint32_t off = (c0 + 16 * pr + 8 * (mi >> 1) + r8) * rbw + (2 * ks + (mi & 1)) * 16;
                    uint32_t x0, x1, x2, x3, y0, y1, y2, y3;
                    ldsm_x4(wh + off, x0, x1, x2, x3);
                    ldsm_x4(wl + off, y0, y1, y2, y3);
                    mma_bf16(dfa[2 * pr], ahi[ks][0], ahi[ks][1], ahi[ks][2], ahi[ks][3], x0, x1);
                    mma_bf16(dfa[2 * pr], ahi[ks][0], ahi[ks][1], ahi[ks][2], ahi[ks][3], y0, y1);
                    mma_bf16(dfa[2 * pr], alo[ks][0], alo[ks][1], alo[ks][2], alo[ks][3], x0, x1);
                    mma_bf16(dfa[2 * pr + 1], ahi[ks][0], ahi[ks][1], ahi[ks][2], ahi[ks][3], x2, x3);
                    mma_bf16(dfa[2 * pr + 1], ahi[ks][0], ahi[ks][1], ahi[ks][2], ahi[ks][3], y2, y3);
                    mma_bf16(dfa[2 * pr + 1], alo[ks][0], alo[ks][1], alo[ks][2], alo[ks][3], x2, x3);
                }
            }
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                const int c = c0 + 8 * nt + 2 * t;
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) {
                    if (!live[rr]) continue;
                    const uint32_t pg = *reinterpret_cast<const uint32_t*>(dmerged + arow[rr] * d + c);
                    const float v0 = fmaf(wt[rr], bf16_lo(pg), dfa[nt][2 * rr]);
                    const float v1 = fmaf(wt[rr], bf16_hi(pg), dfa[nt][2 * rr + 1]);
                    *reinterpret_cast<uint32_t*>(dfeats + static_cast<size_t>(t0 + g + 8 * rr) * d + c) =
                        pack_bf16(v0, v1);
                }
            }
        }
        __syncwarp();
    }
}

// Order-preserving map of an fp32 score to uint32 (-0 and +0 equal).
__device__ __forceinline__ uint32_t order_bits_f(float f) {
    uint32_t u = __float_as_uint(f);
    if ((u & 0x7FFFFFFFu) == 0) u = 0;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// 2. anchors by counting: token i is ranked after every j with a larger score, or an equal
//    score and a lower id; it is an anchor when fewer than k tokens rank ahead of it.
//    kSub lanes per token, lane s over the 16-byte groups of scores = s (mod kSub).
//    flag[i] = 1 for anchors, else 0.
__global__ void __launch_bounds__(kMergeThreads)
    merge_rank_kernel(const float* __restrict__ scores, int N, int k, int32_t* __restrict__ flag) {
    extern __shared__ __align__(16) uint32_t ord[];  // [N rounded up to 4], zero padding
    const int b = blockIdx.y;
    const float* sb = scores + static_cast<size_t>(b) * N;
    const int N4 = (N + 3) & ~3;
    for (int j = threadIdx.x; j < N4; j += kMergeThreads) ord[j] = j < N ? order_bits_f(sb[j]) : 0u;
    __syncthreads();
    const int s = threadIdx.x & (kSub - 1);
    const int i = (blockIdx.x * kMergeThreads + threadIdx.x) / kSub;
    const int iw = i & ~(kTokPerWarp - 1);  // first token of this warp (a multiple of 8)
    if (iw >= N) return;                    // whole warps
    const uint32_t oi = i < N ? ord[i] : 0u;
    int ahead = 0;
    for (int g = s; g < iw / 4; g += kSub) {  // j < i: ahead iff o_j >= o_i
        const uint4 o = *reinterpret_cast<const uint4*>(ord + 4 * g);
        ahead += (o.x >= oi) + (o.y >= oi) + (o.z >= oi) + (o.w >= oi);
    }
    if (s == 0) {
        const int wend = min(iw + kTokPerWarp, N);
        for (int j = iw; j < wend; ++j) {
            const uint32_t o = ord[j];
            ahead += (o > oi) || (o == oi && j < i);
        }
    }
    for (int g = (iw + kTokPerWarp) / 4 + s; g < N4 / 4; g += kSub) {  // j > i: o_j > o_i (padding 0)
        const uint4 o = *reinterpret_cast<const uint4*>(ord + 4 * g);
        ahead += (o.x > oi) + (o.y > oi) + (o.z > oi) + (o.w > oi);
    }
    ahead += __shfl_xor_sync(0xffffffffu, ahead, 1);
    ahead += __shfl_xor_sync(0xffffffffu, ahead, 2);
    if (i < N && s == 0) flag[static_cast<size_t>(b) * N + i] = ahead < k ? 1 : 0;
}

// 3. assignment.  Every CTA rebuilds its image's anchor list (ascending id) from the flags
//    by a block scan; CTA 0 of the image writes it out.  Then kAssignSub lanes per token, lane
//    p scanning anchors j = p (mod kAssignSub) with an fp32 prefilter and the exact fp64
//    decision; the lanes' bests are combined by (fp64 distance, anchor id).
__global__ void __launch_bounds__(kMergeThreads)
    merge_assign_kernel(const float* __restrict__ xy, int N, int k, const int32_t* __restrict__ flag,
                        int32_t* __restrict__ anchors, int32_t* __restrict__ assign) {
    extern __shared__ __align__(16) float2 axy[];  // [k]
    constexpr int kTok = kMergeThreads / kAssignSub;
    __shared__ int wsum[kMergeWarps];
    __shared__ int myrank[kTok];
    const int b = blockIdx.y, i0 = blockIdx.x * kTok;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const float2* xb = reinterpret_cast<const float2*>(xy) + static_cast<size_t>(b) * N;
    const int32_t* fb = flag + static_cast<size_t>(b) * N;
    const int per = (N + kMergeThreads - 1) / kMergeThreads;
    const int j0 = min(N, threadIdx.x * per), j1 = min(N, j0 + per);
    int cnt = 0;
    for (int jb = j0; jb < j1; jb += 8) {
#pragma unroll
        for (int q = 0; q < 8; ++q) cnt += (jb + q < j1) ? (fb[jb + q] != 0) : 0;
    }
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    int r = incl - cnt;
    for (int w = 0; w < warp; ++w) r += wsum[w];
    for (int jb = j0; jb < j1; jb += 8) {  // flags and coordinates of 8 tokens loaded at once
        int f8[8];
        float2 p8[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            f8[q] = (jb + q < j1) ? fb[jb + q] : 0;
            p8[q] = (jb + q < j1) ? xb[jb + q] : make_float2(0.f, 0.f);
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const int j = jb + q;
            if (j >= j1) break;
            const bool is_anchor = f8[q] != 0 && r < k;
            if (j >= i0 && j < i0 + kTok) myrank[j - i0] = is_anchor ? r : -1;
            if (is_anchor) {
                axy[r] = p8[q];
                if (blockIdx.x == 0) anchors[static_cast<size_t>(b) * k + r] = j;
                ++r;
            }
        }
    }
    __syncthreads();
    const int sub = threadIdx.x % kAssignSub;
    const int i = i0 + threadIdx.x / kAssignSub;
    const bool live = i < N;
    const int ri = live ? myrank[i - i0] : 0;
    const float2 p = live ? xb[i] : make_float2(0.f, 0.f);
    const double px = p.x, py = p.y;
    double best = DBL_MAX;
    float bestf = FLT_MAX;
    int bj = 0x7fffffff;
    if (live && ri < 0) {
        for (int j = sub; j < k; j += kAssignSub) {
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
    }
#pragma unroll
    for (int o = 1; o < kAssignSub; o <<= 1) {
        const double ob = __shfl_xor_sync(0xffffffffu, best, o);
        const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
        if (ob < best || (ob == best && oj < bj)) {
            best = ob;
            bj = oj;
        }
    }
    if (live && sub == 0) assign[static_cast<size_t>(b) * N + i] = ri >= 0 ? ri : bj;
}

// Exclusive prefix sum of data[0..n) by the whole block; data[n] = the total.
__device__ void block_scan_excl(int* data, int n, int* scratch);

// 3b. assignment by a binned search, one thread per token (k <= kBinnedMaxK).  The CTA
//     rebuilds the anchor list as above, then counting-sorts the anchors into square bins of
//     side s, a power of two, aligned to multiples of s (bin = floor(x / s): exact), about two
//     anchors per bin over the anchors' bounding box.  A token scans rings of bins around its
//     own (clamped) bin, an fp32 prefilter before the exact fp64 (distance, anchor rank)
//     comparison; after each ring it stops once its best distance is below the squared
//     distance to the edge of the scanned rectangle (an anchor outside lies at least that far
//     on one axis, and rounding is monotone; a side on the grid's border bounds nothing).
//     The result equals the brute-force definition.  A CTA whose anchor box is not finite
//     falls back to the full scan.
constexpr int kBinThreads = 128;
constexpr int kBinnedMaxK = 4096;
constexpr int kBinsMax = 2048;

__global__ void __launch_bounds__(kBinThreads)
    merge_assign_binned_kernel(const float* __restrict__ xy, int N, int k, const int32_t* __restrict__ flag,
                               int32_t* __restrict__ anchors, int32_t* __restrict__ assign) {
    extern __shared__ __align__(16) uint8_t bsm[];
    float2* axy = reinterpret_cast<float2*>(bsm);   // [k] by rank
    float2* sxy = axy + k;                           // [k] in bin order
    int* srank = reinterpret_cast<int*>(sxy + k);    // [k] in bin order
    int* cnt = srank + k;                            // [kBinsMax + 1]
    __shared__ int wsum[kBinThreads / 32];
    __shared__ int myrank[kBinThreads];
    __shared__ float box[4][kBinThreads / 32];
    __shared__ int scan_scratch[40];
    __shared__ int grid_i[5];  // bx0, by0, nbx, nby, full scan
    __shared__ float grid_f[1];
    const int b = blockIdx.y, i0 = blockIdx.x * kBinThreads;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const float2* xb = reinterpret_cast<const float2*>(xy) + static_cast<size_t>(b) * N;
    const int32_t* fb = flag + static_cast<size_t>(b) * N;
    // anchor list (ascending id) by a block scan of the flags
    const int per = (N + kBinThreads - 1) / kBinThreads;
    const int j0 = min(N, tid * per), j1 = min(N, j0 + per);
    int c = 0;
    for (int j = j0; j < j1; ++j) c += fb[j] != 0;
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    int r = incl - c;
    for (int w = 0; w < warp; ++w) r += wsum[w];
    for (int jb = j0; jb < j1; jb += 8) {
        int f8[8];
        float2 p8[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            f8[q] = (jb + q < j1) ? fb[jb + q] : 0;
            p8[q] = (jb + q < j1) ? xb[jb + q] : make_float2(0.f, 0.f);
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const int j = jb + q;
            if (j >= j1) break;
            const bool is_anchor = f8[q] != 0 && r < k;
            if (j >= i0 && j < i0 + kBinThreads) myrank[j - i0] = is_anchor ? r : -1;
            if (is_anchor) {
                axy[r] = p8[q];
                if (blockIdx.x == 0) anchors[static_cast<size_t>(b) * k + r] = j;
                ++r;
            }
        }
    }
    __syncthreads();
    // bounding box of the anchors
    float mnx = FLT_MAX, mxx = -FLT_MAX, mny = FLT_MAX, mxy = -FLT_MAX;
    bool fin = true;
    for (int a = tid; a < k; a += kBinThreads) {
        const float2 p = axy[a];
        fin = fin && isfinite(p.x) && isfinite(p.y);
        mnx = fminf(mnx, p.x); mxx = fmaxf(mxx, p.x);
        mny = fminf(mny, p.y); mxy = fmaxf(mxy, p.y);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        mnx = fminf(mnx, __shfl_xor_sync(0xffffffffu, mnx, o));
        mxx = fmaxf(mxx, __shfl_xor_sync(0xffffffffu, mxx, o));
        mny = fminf(mny, __shfl_xor_sync(0xffffffffu, mny, o));
        mxy = fmaxf(mxy, __shfl_xor_sync(0xffffffffu, mxy, o));
    }
    const bool all_fin = __syncthreads_and(fin) != 0;
    if (lane == 0) {
        box[0][warp] = mnx; box[1][warp] = mxx; box[2][warp] = mny; box[3][warp] = mxy;
    }
    __syncthreads();
    if (tid == 0) {
        for (int w = 1; w < kBinThreads / 32; ++w) {
            mnx = fminf(mnx, box[0][w]); mxx = fmaxf(mxx, box[1][w]);
            mny = fminf(mny, box[2][w]); mxy = fmaxf(mxy, box[3][w]);
        }
        int full = !all_fin;
        float sv = 1.f;
        int bx0 = 0, by0 = 0, nbx = 1, nby = 1;
        if (!full) {
            // about two anchors per bin, at most kBinsMax bins, |bin index| < 2^30
            const int target = max(1, min(kBinsMax, k / 2));
            const float ext = fmaxf(fmaxf(mxx - mnx, mxy - mny), 1e-30f);
            sv = exp2f(ceilf(log2f(ext / sqrtf(static_cast<float>(target)))));
            for (int it = 0; it < 300; ++it) {
                const float fx0 = floorf(mnx / sv), fx1 = floorf(mxx / sv);
                const float fy0 = floorf(mny / sv), fy1 = floorf(mxy / sv);
                const bool ok = fabsf(fx0) < 1073741824.f && fabsf(fx1) < 1073741824.f &&
                                fabsf(fy0) < 1073741824.f && fabsf(fy1) < 1073741824.f &&
                                (fx1 - fx0 + 1.f) * (fy1 - fy0 + 1.f) <= static_cast<float>(target);
                if (ok) {
                    bx0 = static_cast<int>(fx0); by0 = static_cast<int>(fy0);
                    nbx = static_cast<int>(fx1 - fx0) + 1; nby = static_cast<int>(fy1 - fy0) + 1;
                    break;
                }
                sv *= 2.f;
                if (it == 299) full = 1;
            }
        }
        grid_i[0] = bx0; grid_i[1] = by0; grid_i[2] = nbx; grid_i[3] = nby; grid_i[4] = full;
        grid_f[0] = sv;
    }
    __syncthreads();
    const int bx0 = grid_i[0], by0 = grid_i[1], nbx = grid_i[2], nby = grid_i[3];
    const bool full = grid_i[4] != 0;
    const float sv = grid_f[0];
    const float inv_s = 1.f / sv;  // exact: a power of two
    auto bin_x = [&](float v) { return min(max(static_cast<int>(floorf(v * inv_s)) - bx0, 0), nbx - 1); };
    auto bin_y = [&](float v) { return min(max(static_cast<int>(floorf(v * inv_s)) - by0, 0), nby - 1); };
    const int nbins = nbx * nby;
    if (!full) {
        for (int i = tid; i <= nbins; i += kBinThreads) cnt[i] = 0;
        __syncthreads();
        for (int a = tid; a < k; a += kBinThreads) {
            const float2 p = axy[a];
            atomicAdd(&cnt[bin_y(p.y) * nbx + bin_x(p.x)], 1);
        }
        __syncthreads();
        block_scan_excl(cnt, nbins, scan_scratch);  // cnt[bin] = start
        for (int a = tid; a < k; a += kBinThreads) {
            const float2 p = axy[a];
            const int pos = atomicAdd(&cnt[bin_y(p.y) * nbx + bin_x(p.x)], 1);
            sxy[pos] = p;
            srank[pos] = a;
        }
        __syncthreads();  // cnt[bin] = end of bin; start = cnt[bin - 1]
    }
    const int i = i0 + tid;
    if (i >= N) return;
    const int ri = myrank[tid];
    if (ri >= 0) {
        assign[static_cast<size_t>(b) * N + i] = ri;
        return;
    }
    const float2 p = xb[i];
    const double px = p.x, py = p.y;
    double best = DBL_MAX;
    float bestf = FLT_MAX;
    int bj = 0x7fffffff;
    auto visit = [&](float2 a, int rank) {
        const float dxf = p.x - a.x, dyf = p.y - a.y;
        const float d2f = fmaf(dxf, dxf, dyf * dyf);
        if (d2f <= bestf) {   // a candidate beyond the fp32 bound cannot be nearer in fp64
            const double dx = __dsub_rn(px, static_cast<double>(a.x));
            const double dy = __dsub_rn(py, static_cast<double>(a.y));
            const double d2 = __dadd_rn(__dmul_rn(dx, dx), __dmul_rn(dy, dy));
            if (d2 < best || (d2 == best && rank < bj)) {
                best = d2;
                bj = rank;
                bestf = static_cast<float>(best) * (1.0f + 1.0f / 1048576.0f);
            }
        }
    };
    // a token whose scaled coordinates are not finite or not below 2^30 in magnitude takes the
    // full scan (its bin index would not be exact)
    const float fpx = floorf(p.x * inv_s), fpy = floorf(p.y * inv_s);
    if (full || !(fabsf(fpx) < 1073741824.f && fabsf(fpy) < 1073741824.f)) {
        for (int a = 0; a < k; ++a) visit(axy[a], a);
    } else {
        const int pbx = bin_x(p.x), pby = bin_y(p.y);
        const double s = static_cast<double>(sv);
        auto scan_bin = [&](int bx, int by) {
            const int bin = by * nbx + bx;
            const int a0 = bin > 0 ? cnt[bin - 1] : 0, a1 = cnt[bin];
            for (int a = a0; a < a1; ++a) visit(sxy[a], srank[a]);
        };
        const int maxring = max(nbx, nby);
        for (int rho = 0; rho <= maxring; ++rho) {
            const int xl = pbx - rho, xh = pbx + rho, yl = pby - rho, yh = pby + rho;
            const int cxl = max(xl, 0), cxh = min(xh, nbx - 1);
            if (rho == 0) {
                scan_bin(pbx, pby);
            } else {
                if (yl >= 0)
                    for (int bx = cxl; bx <= cxh; ++bx) scan_bin(bx, yl);
                if (yh < nby)
                    for (int bx = cxl; bx <= cxh; ++bx) scan_bin(bx, yh);
                for (int by = max(yl + 1, 0); by <= min(yh - 1, nby - 1); ++by) {
                    if (xl >= 0) scan_bin(xl, by);
                    if (xh < nbx) scan_bin(xh, by);
                }
            }
            double m = DBL_MAX;
            if (xl > 0) m = fmin(m, __dsub_rn(px, static_cast<double>(bx0 + xl) * s));
            if (xh < nbx - 1) m = fmin(m, __dsub_rn(static_cast<double>(bx0 + xh + 1) * s, px));
            if (yl > 0) m = fmin(m, __dsub_rn(py, static_cast<double>(by0 + yl) * s));
            if (yh < nby - 1) m = fmin(m, __dsub_rn(static_cast<double>(by0 + yh + 1) * s, py));
            if (m == DBL_MAX) break;                   // the whole grid is scanned
            if (best < __dmul_rn(m, m)) break;         // nothing outside can be nearer or tie
        }
    }
    assign[static_cast<size_t>(b) * N + i] = bj;
}

// Exclusive prefix sum of data[0..n) by the whole block; data[n] = the total.
__device__ void block_scan_excl(int* data, int n, int* scratch) {
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
    if (tid == 0) data[n] = scratch[32];
    __syncthreads();
}

// 4. groups: per image, a counting sort of the tokens by assignment -> members [N] (each
//    group's tokens by ascending id) and the offsets goff [k + 1].  Slots taken by shared-
//    memory atomics only place a token in its group's segment; its final position is its rank
//    by id within the group, so the result does not depend on the atomics' order.  A token
//    whose assignment is outside [0, k) is left out.
__global__ void __launch_bounds__(kSortThreads)
    merge_groups_kernel(const int32_t* __restrict__ assign, int N, int k, int32_t* __restrict__ members,
                        int32_t* __restrict__ goff) {
    extern __shared__ __align__(16) int gsm[];
    int* cnt = gsm;              // [k + 1]
    int* slot = cnt + k + 1;     // [N]
    int* seg = slot + N;         // [N]
    __shared__ int scratch[40];
    const int b = blockIdx.x;
    const int32_t* ab = assign + static_cast<size_t>(b) * N;
    for (int j = threadIdx.x; j <= k; j += kSortThreads) cnt[j] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < N; i += kSortThreads) {
        const int a = ab[i];
        slot[i] = (a >= 0 && a < k) ? atomicAdd(&cnt[a], 1) : -1;
    }
    __syncthreads();
    block_scan_excl(cnt, k, scratch);
    int32_t* gb = goff + static_cast<size_t>(b) * (k + 1);
    for (int j = threadIdx.x; j <= k; j += kSortThreads) gb[j] = cnt[j];
    for (int i = threadIdx.x; i < N; i += kSortThreads)
        if (slot[i] >= 0) seg[cnt[ab[i]] + slot[i]] = i;
    __syncthreads();
    int32_t* mb = members + static_cast<size_t>(b) * N;
    for (int i = threadIdx.x; i < N; i += kSortThreads) {
        if (slot[i] < 0) continue;
        const int a = ab[i], s0 = cnt[a], n = cnt[a + 1] - s0;
        int pos = 0;
        for (int x = 0; x < n; ++x) pos += seg[s0 + x] < i;
        mb[s0 + pos] = i;
    }
}

// Softmax of a group's scores, lanes over members: max m, inv = 1 / sum_x exp(s_x - m) (lane
// x adding members x, x + 32, ... in order, then a butterfly sum); member x's weight is
// exp(s_x - m) * inv.
__device__ __forceinline__ void group_softmax(const float* sb, const int32_t* mem, int n, int lane,
                                              float& gmax, float& inv) {
    float m = -FLT_MAX;
    for (int x = lane; x < n; x += 32) m = fmaxf(m, sb[mem[x]]);
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float s = 0.f;
    for (int x = lane; x < n; x += 32) s += expf(sb[mem[x]] - m);
    gmax = m;
    inv = 1.f / warp_sum(s);
}

// Members x0 + lane of a group (token id, weight, coordinates), 0 beyond n.
struct MemberLane {
    int t;
    float w;
    float2 p;
};
__device__ __forceinline__ MemberLane member_lane(const float* sb, const float2* xb, const int32_t* mem,
                                                  int x, int n, float gmax, float inv) {
    MemberLane r{0, 0.f, make_float2(0.f, 0.f)};
    if (x < n) {
        r.t = mem[x];
        r.w = expf(sb[r.t] - gmax) * inv;
        r.p = xb[r.t];
    }
    return r;
}

// Softmax statistics and the first round of members (lane x < 32) together: for a group of
// at most 32 members one round of loads serves both (the same operations in the same order
// as group_softmax followed by member_lane, which larger groups use).
__device__ __forceinline__ MemberLane group_first_round(const float* sb, const float2* xb, const int32_t* mem,
                                                        int n, int lane, float& gmax, float& inv) {
    if (n > 32) {
        group_softmax(sb, mem, n, lane, gmax, inv);
        return member_lane(sb, xb, mem, lane, n, gmax, inv);
    }
    MemberLane r{0, 0.f, make_float2(0.f, 0.f)};
    float sc = 0.f;
    if (lane < n) {
        r.t = mem[lane];
        sc = sb[r.t];
        r.p = xb[r.t];
    }
    float m = lane < n ? fmaxf(-FLT_MAX, sc) : -FLT_MAX;
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const float e = lane < n ? 0.f + expf(sc - m) : 0.f;
    gmax = m;
    inv = 1.f / warp_sum(e);
    if (lane < n) r.w = expf(sc - m) * inv;
    return r;
}

// 5. forward merge: one warp per anchor; members in rounds of 32 (lane x holding member x's
//    id and weight), lanes over 4-channel groups.
__global__ void __launch_bounds__(kMergeThreads)
    merge_fwd_kernel(const bf16* __restrict__ feats, const float* __restrict__ xy, int B, int N, int d,
                     int k, const float* __restrict__ scores, const int32_t* __restrict__ members,
                     const int32_t* __restrict__ goff, bf16* __restrict__ merged, float* __restrict__ mxy) {
    const int lane = threadIdx.x & 31;
    const long long ga = static_cast<long long>(blockIdx.x) * kMergeWarps + (threadIdx.x >> 5);
    if (ga >= static_cast<long long>(B) * k) return;
    const int b = static_cast<int>(ga / k), j = static_cast<int>(ga - static_cast<long long>(b) * k);
    const float* sb = scores + static_cast<size_t>(b) * N;
    const int32_t* gb = goff + static_cast<size_t>(b) * (k + 1);
    const int g0 = gb[j], n = gb[j + 1] - g0;
    const int32_t* mem = members + static_cast<size_t>(b) * N + g0;
    const float2* xb = reinterpret_cast<const float2*>(xy) + static_cast<size_t>(b) * N;
    float gmax, inv;
    const MemberLane ml0 = group_first_round(sb, xb, mem, n, lane, gmax, inv);
    const bf16* fb = feats + static_cast<size_t>(b) * N * d;
    bf16* out = merged + static_cast<size_t>(ga) * d;
    float mx = 0.f, my = 0.f;
    for (int c0 = 0; c0 < d; c0 += 128) {
        const int c = c0 + 4 * lane;
        float a[4] = {0.f, 0.f, 0.f, 0.f};
        for (int x0 = 0; x0 < n; x0 += 32) {
            const MemberLane ml = x0 == 0 ? ml0 : member_lane(sb, xb, mem, x0 + lane, n, gmax, inv);
            if (c0 == 0) {
                mx = fmaf(ml.w, ml.p.x, mx);
                my = fmaf(ml.w, ml.p.y, my);
            }
            const int nn = min(32, n - x0);
            for (int x = 0; x < nn; ++x) {
                const int t = __shfl_sync(0xffffffffu, ml.t, x);
                const float w = __shfl_sync(0xffffffffu, ml.w, x);
                if (c < d) {
                    const uint2 pr = *reinterpret_cast<const uint2*>(fb + static_cast<size_t>(t) * d + c);
                    a[0] = fmaf(w, bf16_lo(pr.x), a[0]);
                    a[1] = fmaf(w, bf16_hi(pr.x), a[1]);
                    a[2] = fmaf(w, bf16_lo(pr.y), a[2]);
                    a[3] = fmaf(w, bf16_hi(pr.y), a[3]);
                }
            }
        }
        if (c < d) {
            uint2 o;
            o.x = pack_bf16(a[0], a[1]);
            o.y = pack_bf16(a[2], a[3]);
            *reinterpret_cast<uint2*>(out + c) = o;
        }
    }
    mx = warp_sum(mx);
    my = warp_sum(my);
    if (lane == 0) reinterpret_cast<float2*>(mxy)[ga] = make_float2(mx, my);
}

// 6. backward group statistics: one warp per anchor -> gstat = {max score, 1 / sum of
//    exp(s - max), sum_G w g} with g_i = <dF_j, f_i> + <dX_j, x_i> (members four at a time,
//    lanes over 4-channel groups, then butterfly sums), summed in member order; g_i is stored
//    so that the token pass uses the very values summed here (a one-token group then gets
//    ds = 0 exactly).
__global__ void __launch_bounds__(kMergeThreads)
    merge_gstat_kernel(const bf16* __restrict__ feats, const float* __restrict__ xy, int B, int N, int d,
                       int k, const float* __restrict__ scores, const int32_t* __restrict__ members,
                       const int32_t* __restrict__ goff, const bf16* __restrict__ dmerged,
                       const float* __restrict__ dmxy, float4* __restrict__ gstat,
                       float* __restrict__ g_out) {
    const int lane = threadIdx.x & 31;
    const long long ga = static_cast<long long>(blockIdx.x) * kMergeWarps + (threadIdx.x >> 5);
    if (ga >= static_cast<long long>(B) * k) return;
    const int b = static_cast<int>(ga / k), j = static_cast<int>(ga - static_cast<long long>(b) * k);
    const float* sb = scores + static_cast<size_t>(b) * N;
    const int32_t* gb = goff + static_cast<size_t>(b) * (k + 1);
    const int g0 = gb[j], n = gb[j + 1] - g0;
    const int32_t* mem = members + static_cast<size_t>(b) * N + g0;
    const float2* xb = reinterpret_cast<const float2*>(xy) + static_cast<size_t>(b) * N;
    float gmax, inv;
    const MemberLane ml0 = group_first_round(sb, xb, mem, n, lane, gmax, inv);
    const bf16* fb = feats + static_cast<size_t>(b) * N * d;
    const bf16* dF = dmerged + static_cast<size_t>(ga) * d;
    const float2 dX = reinterpret_cast<const float2*>(dmxy)[ga];
    float* gb_out = g_out + static_cast<size_t>(b) * N;
    float sg = 0.f;
    for (int x0 = 0; x0 < n; x0 += 32) {
        const MemberLane ml = x0 == 0 ? ml0 : member_lane(sb, xb, mem, x0 + lane, n, gmax, inv);
        const int nn = min(32, n - x0);
        for (int x1 = 0; x1 < nn; x1 += 4) {
            int tq[4];
            float part[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                tq[q] = __shfl_sync(0xffffffffu, ml.t, min(x1 + q, nn - 1));
                part[q] = 0.f;
            }
            for (int c = 4 * lane; c < d; c += 128) {
                const uint2 g = *reinterpret_cast<const uint2*>(dF + c);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint2 f = *reinterpret_cast<const uint2*>(fb + static_cast<size_t>(tq[q]) * d + c);
                    part[q] = fmaf(bf16_lo(f.x), bf16_lo(g.x), part[q]);
                    part[q] = fmaf(bf16_hi(f.x), bf16_hi(g.x), part[q]);
                    part[q] = fmaf(bf16_lo(f.y), bf16_lo(g.y), part[q]);
                    part[q] = fmaf(bf16_hi(f.y), bf16_hi(g.y), part[q]);
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
#pragma unroll
                for (int q = 0; q < 4; ++q) part[q] += __shfl_xor_sync(0xffffffffu, part[q], o);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int x = x1 + q;
                const float px = __shfl_sync(0xffffffffu, ml.p.x, min(x, nn - 1));
                const float py = __shfl_sync(0xffffffffu, ml.p.y, min(x, nn - 1));
                const float wq = __shfl_sync(0xffffffffu, ml.w, min(x, nn - 1));
                if (x < nn) {
                    const float gi = part[q] + dX.x * px + dX.y * py;
                    if (lane == 0) gb_out[tq[q]] = gi;
                    sg = fmaf(wq, gi, sg);
                }
            }
        }
    }
    if (lane == 0) gstat[ga] = make_float4(gmax, inv, sg, 0.f);
}

// 7. backward token pass: four lanes per token.  w = exp(s - max) / sum, g from the group
//    statistics pass, ds = w (g - sum_G w g), dx = w dX;
//    z again, dh = ds w2 gelu'(z) and e = ds gelu(z) for the lane's units (written for the
//    parameter sums, and dh to shared memory for the token's four lanes); then dfeats = w dF
//    + W1 dh with lane s on the channel pairs 8 m + 2 s.  A token whose assignment is outside
//    [0, k) gets w = 0, so all its gradients are zero.
template <int HP, bool SM>
__global__ void __launch_bounds__(kMergeThreads)
    merge_bwd_token_kernel(const bf16* __restrict__ feats, const float* __restrict__ xy, int T, int N,
                           int d, int k, int h, const float* __restrict__ w1, const float* __restrict__ b1,
                           const float* __restrict__ w2, const float* __restrict__ scores,
                           const int32_t* __restrict__ assign, const float4* __restrict__ gstat,
                           const float* __restrict__ gtok, const bf16* __restrict__ dmerged, const float* __restrict__ dmxy,
                           bf16* __restrict__ dfeats, float* __restrict__ dxy, float* __restrict__ ds_out,
                           float* __restrict__ dh_out, float* __restrict__ e_out) {
    constexpr int HS = kHS<HP>;
    extern __shared__ __align__(16) float dyn[];
    float* dhs = dyn;                                 // [kTokPerCta][HS]
    float* w1s = dyn + kTokPerCta * HS;               // [d][HS] when SM
    __shared__ __align__(16) float b1s[32 * HP];
    __shared__ __align__(16) float w2s[32 * HP];
    stage_bias<HP>(b1s, w2s, b1, w2, h);
    if constexpr (SM) stage_w1<HP>(w1s, w1, d, h);
    __syncthreads();
    const float* w = SM ? w1s : w1;
    const int lane = threadIdx.x & 31, s = lane & (kSub - 1), tw = lane / kSub;
    float* mydh = dhs + ((threadIdx.x >> 5) * kTokPerWarp + tw) * HS;
    const int h4 = (h + 3) & ~3;
    const int warp_g = blockIdx.x * kMergeWarps + (threadIdx.x >> 5);
    for (int base = warp_g * kTokPerWarp; base < T; base += gridDim.x * kTokPerCta) {  // warp-uniform
        const int t0 = base + tw;
        const bool live = t0 < T;
        const int t = live ? t0 : base;
        const int b = t / N;
        const int a = assign[t];
        const bool ok = live && a >= 0 && a < k;
        const size_t ga = static_cast<size_t>(b) * k + (ok ? a : 0);
        const float4 gs = gstat[ga];
        const float wt = ok ? expf(scores[t] - gs.x) * gs.y : 0.f;
        const bf16* frow = feats + static_cast<size_t>(t) * d;
        const bf16* dF = dmerged + ga * d;
        const float2 dX = reinterpret_cast<const float2*>(dmxy)[ga];
        const float ds = ok ? wt * (gtok[t] - gs.z) : 0.f;
        float z[8 * HP];
        hidden4<HP, SM>(frow, d, w, h, b1s, s, z);
#pragma unroll
        for (int y = 0; y < 2 * HP; ++y) {
            const int u0 = 4 * s + 16 * y;
            float dh4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float zz = z[4 * y + e];
                dh4[e] = ds * w2s[u0 + e] * gelu_grad_f(zz);
                if (live && u0 + e < h) {
                    dh_out[static_cast<size_t>(t) * h + u0 + e] = dh4[e];
                    e_out[static_cast<size_t>(t) * h + u0 + e] = ds * gelu_f(zz);
                }
            }
            *reinterpret_cast<float4*>(mydh + u0) = make_float4(dh4[0], dh4[1], dh4[2], dh4[3]);
        }
        if (live && s == 0) {
            ds_out[t] = ds;
            reinterpret_cast<float2*>(dxy)[t] = make_float2(wt * dX.x, wt * dX.y);
        }
        __syncwarp();
        for (int c = 2 * s; c < d; c += 2 * kSub) {
            const uint32_t pg = *reinterpret_cast<const uint32_t*>(dF + c);
            float a0 = wt * bf16_lo(pg), a1 = wt * bf16_hi(pg);
#pragma unroll 4
            for (int u0 = 0; u0 < h4; u0 += 4) {
                const float4 dh4 = *reinterpret_cast<const float4*>(mydh + u0);
                const float4 wa = w1_load4<SM>(w, HS, h, c, u0);
                const float4 wb = w1_load4<SM>(w, HS, h, c + 1, u0);
                a0 = fmaf(wa.x, dh4.x, a0);
                a0 = fmaf(wa.y, dh4.y, a0);
                a0 = fmaf(wa.z, dh4.z, a0);
                a0 = fmaf(wa.w, dh4.w, a0);
                a1 = fmaf(wb.x, dh4.x, a1);
                a1 = fmaf(wb.y, dh4.y, a1);
                a1 = fmaf(wb.z, dh4.z, a1);
                a1 = fmaf(wb.w, dh4.w, a1);
            }
            if (live)
                *reinterpret_cast<__nv_bfloat162*>(dfeats + static_cast<size_t>(t) * d + c) =
                    __floats2bfloat162_rn(a0, a1);
        }
        __syncwarp();  // the token's dh is read before the next token overwrites it
    }
}

// 8. parameter gradients, stage 1: CTA x sums tokens [x T / P, (x + 1) T / P) in order into
//    4 x 4 register tiles of a (d + 3) x h output matrix: rows c < d give dW1 (left f_c,
//    right dh), row d gives db1 (left 1, right dh), row d + 1 gives dw2 (left 1, right e),
//    row d + 2 gives db2 (left ds, column 0).  Part layout [P][dW1 (d*h) | db1 | dw2 | db2].
__global__ void __launch_bounds__(1024)
    merge_param_part_kernel(const bf16* __restrict__ feats, int T, int d, int h,
                            const float* __restrict__ ds, const float* __restrict__ dh,
                            const float* __restrict__ ev, float* __restrict__ part) {
    extern __shared__ __align__(16) float tile[];
    const int h4 = (h + 3) & ~3;
    float* fs = tile;                        // [kParamTile][d]
    float* dhs = fs + kParamTile * d;        // [kParamTile][h4]
    float* es = dhs + kParamTile * h4;       // [kParamTile][h4]
    float* dss = es + kParamTile * h4;       // [kParamTile]
    const int RB = d / 4 + 1, CB = h4 / 4;
    const int tid = blockIdx.y * blockDim.x + threadIdx.x;
    const bool active = tid < RB * CB;
    const int rb = tid / CB, cb = tid - rb * CB;
    const int p = blockIdx.x;
    const int t0 = static_cast<int>(static_cast<long long>(p) * T / kParamParts);
    const int t1 = static_cast<int>(static_cast<long long>(p + 1) * T / kParamParts);
    const int d8 = d / 8;
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
    for (int tt = t0; tt < t1; tt += kParamTile) {
        const int nt = min(kParamTile, t1 - tt);
        __syncthreads();
#pragma unroll 4
        for (int q = threadIdx.x; q < nt * d8; q += blockDim.x) {
            const int r = q / d8, c8 = q - r * d8;
            const uint4 v = ldg16(feats + static_cast<size_t>(tt + r) * d + 8 * c8);
            float* dst = fs + r * d + 8 * c8;
            *reinterpret_cast<float4*>(dst) = make_float4(bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y));
            *reinterpret_cast<float4*>(dst + 4) = make_float4(bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w));
        }
#pragma unroll 4
        for (int q = threadIdx.x; q < nt * h4; q += blockDim.x) {
            const int r = q / h4, u = q - r * h4;
            const size_t g = static_cast<size_t>(tt + r) * h + u;
            dhs[q] = u < h ? dh[g] : 0.f;
            es[q] = u < h ? ev[g] : 0.f;
        }
        for (int q = threadIdx.x; q < nt; q += blockDim.x) dss[q] = ds[tt + q];
        __syncthreads();
        if (!active) continue;
        if (rb < RB - 1) {
            for (int r = 0; r < nt; ++r) {
                const float4 l = *reinterpret_cast<const float4*>(fs + r * d + 4 * rb);
                const float4 v = *reinterpret_cast<const float4*>(dhs + r * h4 + 4 * cb);
                const float lv[4] = {l.x, l.y, l.z, l.w}, rv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(lv[i], rv[j], acc[i][j]);
            }
        } else {
            for (int r = 0; r < nt; ++r) {
                const float4 v = *reinterpret_cast<const float4*>(dhs + r * h4 + 4 * cb);
                const float4 e4 = *reinterpret_cast<const float4*>(es + r * h4 + 4 * cb);
                const float sd = dss[r];
                acc[0][0] += v.x; acc[0][1] += v.y; acc[0][2] += v.z; acc[0][3] += v.w;
                acc[1][0] += e4.x; acc[1][1] += e4.y; acc[1][2] += e4.z; acc[1][3] += e4.w;
                acc[2][0] += sd;
            }
        }
    }
    if (!active) return;
    const size_t nout = static_cast<size_t>(d) * h + 2 * h + 1;
    float* pp = part + static_cast<size_t>(p) * nout;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int u = 4 * cb + j;
        if (u >= h) continue;
        if (rb < RB - 1) {
#pragma unroll
            for (int i = 0; i < 4; ++i) pp[static_cast<size_t>(4 * rb + i) * h + u] = acc[i][j];
        } else {
            pp[static_cast<size_t>(d) * h + u] = acc[0][j];
            pp[static_cast<size_t>(d) * h + h + u] = acc[1][j];
            if (u == 0) pp[static_cast<size_t>(d) * h + 2 * h] = acc[2][0];
        }
    }
}

// 9. parameter gradients, stage 2: CTA over 32 outputs; warp w sums parts w, w + 8, ... in
//    order, then the eight warp sums are added in warp order.
__global__ void __launch_bounds__(kMergeThreads)
    merge_param_reduce_kernel(const float* __restrict__ part, int d, int h, float* __restrict__ dw1,
                              float* __restrict__ db1, float* __restrict__ dw2, float* __restrict__ db2) {
    __shared__ float red[kMergeWarps][32];
    const int nout = d * h + 2 * h + 1;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int o = blockIdx.x * 32 + lane;
    float a = 0.f;
    if (o < nout)
#pragma unroll 8
        for (int p = warp; p < kParamParts; p += kMergeWarps) a += part[static_cast<size_t>(p) * nout + o];
    red[warp][lane] = a;
    __syncthreads();
    if (warp != 0 || o >= nout) return;
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kMergeWarps; ++w) s += red[w][lane];
    if (o < d * h) dw1[o] = s;
    else if (o < d * h + h) db1[o - d * h] = s;
    else if (o < d * h + 2 * h) dw2[o - d * h - h] = s;
    else *db2 = s;
}

int hp_of(int h) { return h <= 32 ? 1 : h <= 64 ? 2 : h <= 128 ? 4 : 8; }
size_t w1_smem(int d, int h) { return sizeof(float) * static_cast<size_t>(d) * (32 * hp_of(h) + 4); }
bool w1_in_smem(int d, int h) { return w1_smem(d, h) <= kW1SmemMax; }
size_t token_smem(int d, int h) {
    return sizeof(float) * static_cast<size_t>(kTokPerCta) * (32 * hp_of(h) + 4) + (w1_in_smem(d, h) ? w1_smem(d, h) : 0);
}
size_t rank_smem(int N) { return 4 * static_cast<size_t>((N + 3) & ~3); }
size_t binned_smem(int k) { return 20 * static_cast<size_t>(k) + 4 * (kBinsMax + 1); }
size_t groups_smem(int N, int k) { return 4 * (static_cast<size_t>(k) + 1 + 2 * static_cast<size_t>(N)); }
size_t param_smem(int d, int h) {
    return sizeof(float) * static_cast<size_t>(kParamTile) * (d + 2 * ((h + 3) & ~3) + 1);
}
int param_threads(int d, int h) {
    const int tiles = (d / 4 + 1) * (((h + 3) & ~3) / 4);
    return tiles >= 1024 ? 1024 : ((tiles + 31) / 32) * 32;
}
unsigned token_ctas(int T) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        sms = 148;
    const long long need = (static_cast<long long>(T) + kTokPerCta - 1) / kTokPerCta;
    const long long cap = static_cast<long long>(sms) * kTokCtasPerSm;
    return static_cast<unsigned>(need < cap ? need : cap);
}

}  // namespace

MergeWorkspace merge_workspace_layout(int B, int N, int d, int h, int k) {
    auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
    const size_t T = static_cast<size_t>(B) * N;
    MergeWorkspace w;
    size_t off = 0;
    w.flag = off;    off += up(sizeof(int32_t) * T);
    w.members = off; off += up(sizeof(int32_t) * T);
    w.goff = off;    off += up(sizeof(int32_t) * static_cast<size_t>(B) * (k + 1));
    w.gstat = off;   off += up(sizeof(float) * 4 * static_cast<size_t>(B) * k);
    w.g = off;       off += up(sizeof(float) * T);
    w.ds = off;      off += up(sizeof(float) * T);
    w.dh = off;      off += up(sizeof(float) * T * h);
    w.e = off;       off += up(sizeof(float) * T * h);
    w.part = off;    off += up(sizeof(float) * kParamParts * (static_cast<size_t>(d) * h + 2 * h + 1));
    w.total = off;
    return w;
}

size_t merge_smem_bytes(int N, int k, int d, int h) {
    const size_t c[] = {w1_in_smem(d, h) ? w1_smem(d, h) : 0, mlp_mma_ok(d, h) ? mlp_smem(d, h, true).total : 0,
                        rank_smem(N),
                        k <= kBinnedMaxK ? binned_smem(k) : 8 * static_cast<size_t>(k),
                        groups_smem(N, k), token_smem(d, h), param_smem(d, h)};
    size_t m = 0;
    for (size_t x : c) m = x > m ? x : m;
    return m;
}

#define ACL_HP_SWITCH(h, CALL)                                 \
    switch (hp_of(h)) {                                        \
        case 1: { constexpr int HP = 1; CALL; } break;         \
        case 2: { constexpr int HP = 2; CALL; } break;         \
        case 4: { constexpr int HP = 4; CALL; } break;         \
        default: { constexpr int HP = 8; CALL; } break;        \
    }

template <int HP, bool SM>
cudaError_t launch_scores(const MergeArgs& m, int T, cudaStream_t st) {
    const size_t sm = SM ? w1_smem(m.d, m.h) : 0;
    cudaError_t e = ensure_smem<merge_scores_kernel<HP, SM>>(sm);
    if (e != cudaSuccess) return e;
    merge_scores_kernel<HP, SM><<<token_ctas(T), kMergeThreads, sm, st>>>(m.feats, T, m.d, m.w1, m.b1, m.w2,
                                                                        m.b2, m.h, m.scores);
    note_launch();
    return cudaSuccess;
}

template <int NT>
cudaError_t launch_scores_mma_nt(const MergeArgs& m, int T, cudaStream_t st) {
    const size_t sm = mlp_smem(m.d, m.h, false).total;
    cudaError_t e = ensure_smem<merge_scores_mma_kernel<NT>>(sm);
    if (e != cudaSuccess) return e;
    const long long tiles = (static_cast<long long>(T) + 15) / 16;
    const long long need = (tiles + kMergeWarps - 1) / kMergeWarps;
    const unsigned ctas = static_cast<unsigned>(need < 2 * 148 ? need : 2 * 148);
    merge_scores_mma_kernel<NT><<<ctas, kMergeThreads, sm, st>>>(m.feats, T, m.d, m.w1, m.b1, m.w2, m.b2, m.scores);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_scores_mma(const MergeArgs& m, int T, cudaStream_t st) {
    switch (m.h / 8) {
        case 2: return launch_scores_mma_nt<2>(m, T, st);
        case 4: return launch_scores_mma_nt<4>(m, T, st);
        case 6: return launch_scores_mma_nt<6>(m, T, st);
        default: return launch_scores_mma_nt<8>(m, T, st);
    }
}

template <int NT>
cudaError_t launch_bwd_token_mma_nt(const MergeArgs& m, int T, cudaStream_t st) {
    const size_t sm = mlp_smem(m.d, m.h, true).total;
    cudaError_t e = ensure_smem<merge_bwd_token_mma_kernel<NT>>(sm);
    if (e != cudaSuccess) return e;
    const long long tiles = (static_cast<long long>(T) + 15) / 16;
    const long long need = (tiles + kMergeWarps - 1) / kMergeWarps;
    const unsigned ctas = static_cast<unsigned>(need < 2 * 148 ? need : 2 * 148);
    merge_bwd_token_mma_kernel<NT><<<ctas, kMergeThreads, sm, st>>>(
        m.feats, m.xy, T, m.N, m.d, m.k, m.w1, m.b1, m.w2, m.scores, m.assign,
        reinterpret_cast<const float4*>(m.gstat), m.g, m.dmerged, m.dmxy, m.dfeats, m.dxy, m.ds, m.dh, m.e);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_bwd_token_mma(const MergeArgs& m, int T, cudaStream_t st) {
    switch (m.h / 8) {
        case 2: return launch_bwd_token_mma_nt<2>(m, T, st);
        case 4: return launch_bwd_token_mma_nt<4>(m, T, st);
        case 6: return launch_bwd_token_mma_nt<6>(m, T, st);
        default: return launch_bwd_token_mma_nt<8>(m, T, st);
    }
}

template <int HP, bool SM>
cudaError_t launch_bwd_token(const MergeArgs& m, int T, cudaStream_t st) {
    const size_t sm = token_smem(m.d, m.h);
    cudaError_t e = ensure_smem<merge_bwd_token_kernel<HP, SM>>(sm);
    if (e != cudaSuccess) return e;
    merge_bwd_token_kernel<HP, SM><<<token_ctas(T), kMergeThreads, sm, st>>>(
        m.feats, m.xy, T, m.N, m.d, m.k, m.h, m.w1, m.b1, m.w2, m.scores, m.assign,
        reinterpret_cast<const float4*>(m.gstat), m.g, m.dmerged, m.dmxy, m.dfeats, m.dxy, m.ds, m.dh, m.e);
    note_launch();
    return cudaSuccess;
}

cudaError_t launch_groups(const MergeArgs& m, cudaStream_t st) {
    const size_t gsm = groups_smem(m.N, m.k);
    cudaError_t e = ensure_smem<merge_groups_kernel>(gsm);
    if (e != cudaSuccess) return e;
    merge_groups_kernel<<<m.B, kSortThreads, gsm, st>>>(m.assign, m.N, m.k, m.members, m.goff);
    note_launch();
    return cudaSuccess;
}

cudaError_t launch_merge_fwd(const MergeArgs& m, cudaStream_t st) {
    const int T = m.B * m.N;
    cudaError_t e = cudaSuccess;
    const bool sm = w1_in_smem(m.d, m.h);
    if (mlp_mma_ok(m.d, m.h)) {
        e = launch_scores_mma(m, T, st);
    } else {
        ACL_HP_SWITCH(m.h, (e = sm ? launch_scores<HP, true>(m, T, st) : launch_scores<HP, false>(m, T, st)));
    }
    if (e != cudaSuccess) return e;
    const size_t rsm = rank_smem(m.N);
    if ((e = ensure_smem<merge_rank_kernel>(rsm)) != cudaSuccess) return e;
    merge_rank_kernel<<<dim3((m.N + kTokPerCta - 1) / kTokPerCta, m.B), kMergeThreads, rsm, st>>>(
        m.scores, m.N, m.k, m.flag);
    note_launch();
    if (m.k <= kBinnedMaxK) {
        const size_t bsm = binned_smem(m.k);
        if ((e = ensure_smem<merge_assign_binned_kernel>(bsm)) != cudaSuccess) return e;
        merge_assign_binned_kernel<<<dim3((m.N + kBinThreads - 1) / kBinThreads, m.B), kBinThreads, bsm, st>>>(
            m.xy, m.N, m.k, m.flag, m.anchors, m.assign);
        note_launch();
        if ((e = launch_groups(m, st)) != cudaSuccess) return e;
        const long long na2 = static_cast<long long>(m.B) * m.k;
        merge_fwd_kernel<<<static_cast<unsigned>((na2 + kMergeWarps - 1) / kMergeWarps), kMergeThreads, 0, st>>>(
            m.feats, m.xy, m.B, m.N, m.d, m.k, m.scores, m.members, m.goff, m.merged, m.mxy);
        note_launch();
        return cudaGetLastError();
    }
    const size_t asm_ = 8 * static_cast<size_t>(m.k);
    if ((e = ensure_smem<merge_assign_kernel>(asm_)) != cudaSuccess) return e;
    constexpr int kAssignTok = kMergeThreads / kAssignSub;
    merge_assign_kernel<<<dim3((m.N + kAssignTok - 1) / kAssignTok, m.B), kMergeThreads, asm_, st>>>(
        m.xy, m.N, m.k, m.flag, m.anchors, m.assign);
    note_launch();
    if ((e = launch_groups(m, st)) != cudaSuccess) return e;
    const long long na = static_cast<long long>(m.B) * m.k;
    merge_fwd_kernel<<<static_cast<unsigned>((na + kMergeWarps - 1) / kMergeWarps), kMergeThreads, 0, st>>>(
        m.feats, m.xy, m.B, m.N, m.d, m.k, m.scores, m.members, m.goff, m.merged, m.mxy);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_merge_bwd(const MergeArgs& m, cudaStream_t st) {
    const int T = m.B * m.N;
    cudaError_t e = cudaSuccess;
    if ((e = launch_groups(m, st)) != cudaSuccess) return e;
    const long long na = static_cast<long long>(m.B) * m.k;
    merge_gstat_kernel<<<static_cast<unsigned>((na + kMergeWarps - 1) / kMergeWarps), kMergeThreads, 0, st>>>(
        m.feats, m.xy, m.B, m.N, m.d, m.k, m.scores, m.members, m.goff, m.dmerged, m.dmxy,
        reinterpret_cast<float4*>(m.gstat), m.g);
    note_launch();
    const bool sm = w1_in_smem(m.d, m.h);
    if (mlp_mma_ok(m.d, m.h)) {
        e = launch_bwd_token_mma(m, T, st);
    } else {
        ACL_HP_SWITCH(m.h, (e = sm ? launch_bwd_token<HP, true>(m, T, st) : launch_bwd_token<HP, false>(m, T, st)));
    }
    if (e != cudaSuccess) return e;
    const size_t psm = param_smem(m.d, m.h);
    if ((e = ensure_smem<merge_param_part_kernel>(psm)) != cudaSuccess) return e;
    const int pth = param_threads(m.d, m.h);
    const int tiles = (m.d / 4 + 1) * (((m.h + 3) & ~3) / 4);
    merge_param_part_kernel<<<dim3(kParamParts, (tiles + pth - 1) / pth), pth, psm, st>>>(
        m.feats, T, m.d, m.h, m.ds, m.dh, m.e, m.part);
    note_launch();
    const int nout = m.d * m.h + 2 * m.h + 1;
    merge_param_reduce_kernel<<<(nout + 31) / 32, kMergeThreads, 0, st>>>(m.part, m.d, m.h, m.dw1, m.db1,
                                                                        m.dw2, m.db2);
    note_launch();
    return cudaGetLastError();
}

#undef ACL_HP_SWITCH

}  // namespace acl
