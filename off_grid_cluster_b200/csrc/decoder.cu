// decoder.cu -- one layer of the point-wise deformable cross-attention decoder, forward and
// backward.
//
// AFFMAE notes, "Key Designs" 2: every mask-token query (feature f, reference position r)
// predicts a 2D offset Delta = g(f), samples q = r + Delta, gathers the nearest visible tokens
// of an encoder stage around q with distance-softmax weights, and the decoder fuses the
// stages coarse to fine ("A Complete Example": stage 4 first).  Here, per layer:
//   q = r + f W_off + b_off                     (offset head, fp32; W_off [D][2])
//   v = KNN gather of the stage at q            (the table/gather kernels of knn.cu, bf16)
//   f_out = f + v W_o                           (W_o [d][D] bf16, tensor cores, fp32 out)
// Backward:
//   dv = df_out W_o^T (bf16), dW_o = v^T df_out (split over the queries, fixed-order sum),
//   KNN backward of dv -> dfeats, dq, dp,
//   df_in = df_out + dq W_off^T, dW_off = f^T dq, db_off = sum dq (fixed-order sums).
//
// The GEMMs: mma.sync m16n8k16 bf16 -> fp32, 128 x 128 CTA tiles, 32-deep k-steps through a
// 3-stage cp.async pipeline; each operand is staged in its stored layout (k-contiguous rows
// of 64 bytes, or k-rows of 128 elements, 256 bytes) with an XOR swizzle and fragments are
// read by ldmatrix (.trans for k-row tiles), so no operand is transposed in memory.
#include <float.h>

#include "internal.h"

namespace acl {

namespace {

constexpr int kGM = 128, kGN = 128, kGK = 32, kGStages = 3, kGThreads = 256;
constexpr int kGTileBytes = kGM * kGK * 2;          // 8 KB, either layout
constexpr int kGStageBytes = 2 * kGTileBytes;       // A and B
constexpr int kGSmem = kGStages * kGStageBytes;     // 48 KB
constexpr int kDecParts = 296;                      // query ranges of the offset-head sums
constexpr int kMaxSplits = 16;                      // k-splits of the dW_o GEMM

enum { kEpiResid = 0, kEpiBf16 = 1, kEpiPart = 2 };

struct GemmArgs {
    const bf16* A;
    const bf16* B;
    int M, N, K;          // C[M][N] = sum_k A(m, k) B(k, n)
    int lda, ldb;         // row pitch (elements) of A and B as stored
    int kchunk;           // split z covers k in [z kchunk, min(K, (z + 1) kchunk))
    const float* R;       // kEpiResid: C = acc + R (pitch ldc)
    float* Cf;            // kEpiResid, kEpiPart (split z at Cf + z part_stride)
    bf16* Cb;             // kEpiBf16
    int ldc;
    size_t part_stride;
};

// k-row tile [32][128]: 16-byte chunk ch of k-row kr at chunk ch ^ (kr & 7), so the 8 rows an
// ldmatrix.trans reads fall in 8 distinct bank groups.
__device__ __forceinline__ uint32_t tile256_off(int kr, int ch) {
    return static_cast<uint32_t>(kr * 256 + ((ch ^ (kr & 7)) << 4));
}

// One operand tile, 512 chunks of 16 bytes (two per thread).  KROW: stored [K][rows] (rows
// contiguous; the tile is 32 k-rows x 128), else [rows][K] (the tile is 128 rows x 32 k).
// Chunks outside [0, rows) x [k0, kend) are zero-filled.  rows % 8 == 0 for KROW and
// kend % 8 == 0 otherwise, so a chunk is wholly inside or outside.
template <bool KROW>
__device__ __forceinline__ void gemm_load_tile(uint32_t sbase, const bf16* __restrict__ src, int ld,
                                               int row0, int rows, int k0, int kend, int tid) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int q = tid + i * kGThreads;
        if constexpr (!KROW) {
            const int r = q >> 2, ch = q & 3;
            const int gr = row0 + r, gk = k0 + 8 * ch;
            const bool ok = gr < rows && gk < kend;
            cp_async16(sbase + tile64_off(r, ch), ok ? src + static_cast<size_t>(gr) * ld + gk : src, ok);
        } else {
            const int kr = q >> 4, ch = q & 15;
            const int gk = k0 + kr, gc = row0 + 8 * ch;
            const bool ok = gk < kend && gc < rows;
            cp_async16(sbase + tile256_off(kr, ch), ok ? src + static_cast<size_t>(gk) * ld + gc : src, ok);
        }
    }
}

template <bool AKROW, bool BKROW, int EPI>
__global__ void __launch_bounds__(kGThreads)
    dec_gemm_kernel(const GemmArgs g) {
    extern __shared__ __align__(128) uint8_t gsm[];
    const uint32_t s0 = smem_addr(gsm);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int m0 = blockIdx.y * kGM, n0 = blockIdx.x * kGN;
    const int wm = (warp >> 2) * 64, wn = (warp & 3) * 32;
    const int kz0 = blockIdx.z * g.kchunk;
    const int kz1 = min(g.K, kz0 + g.kchunk);
    const int nk = kz1 > kz0 ? (kz1 - kz0 + kGK - 1) / kGK : 0;

    auto load_stage = [&](int stage, int kt) {
        const uint32_t sa = s0 + stage * kGStageBytes, sb = sa + kGTileBytes;
        const int k0 = kz0 + kt * kGK;
        gemm_load_tile<AKROW>(sa, g.A, g.lda, m0, g.M, k0, kz1, tid);
        gemm_load_tile<BKROW>(sb, g.B, g.ldb, n0, g.N, k0, kz1, tid);
    };

    float acc[4][4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.f;

#pragma unroll
    for (int s = 0; s < kGStages - 1; ++s) {
        if (s < nk) load_stage(s, s);
        cp_async_commit();
    }
    const int mi = lane >> 3, r8 = lane & 7;
    for (int kt = 0; kt < nk; ++kt) {
        cp_async_wait<kGStages - 2>();
        __syncthreads();
        const int nxt = kt + kGStages - 1;
        if (nxt < nk) load_stage(nxt % kGStages, nxt);
        cp_async_commit();
        const uint32_t sa = s0 + (kt % kGStages) * kGStageBytes, sb = sa + kGTileBytes;
#pragma unroll
        for (int kk = 0; kk < kGK; kk += 16) {
            uint32_t af[4][4], bfr[4][2];
#pragma unroll
            for (int mt = 0; mt < 4; ++mt) {
                if constexpr (!AKROW) {
                    const int row = wm + 16 * mt + (lane & 15), ch = (kk >> 3) + (lane >> 4);
                    ldsm_x4(sa + tile64_off(row, ch), af[mt][0], af[mt][1], af[mt][2], af[mt][3]);
                } else {
                    const int kr = kk + r8 + 8 * (mi >> 1), ch = ((wm + 16 * mt) >> 3) + (mi & 1);
                    ldsm_x4_t(sa + tile256_off(kr, ch), af[mt][0], af[mt][1], af[mt][2], af[mt][3]);
                }
            }
#pragma unroll
            for (int pr = 0; pr < 2; ++pr) {
                if constexpr (!BKROW) {
                    const int row = wn + 16 * pr + 8 * (mi >> 1) + r8, ch = (kk >> 3) + (mi & 1);
                    ldsm_x4(sb + tile64_off(row, ch), bfr[2 * pr][0], bfr[2 * pr][1], bfr[2 * pr + 1][0],
                            bfr[2 * pr + 1][1]);
                } else {
                    const int kr = kk + r8 + 8 * (mi & 1), ch = ((wn + 16 * pr) >> 3) + (mi >> 1);
                    ldsm_x4_t(sb + tile256_off(kr, ch), bfr[2 * pr][0], bfr[2 * pr][1], bfr[2 * pr + 1][0],
                              bfr[2 * pr + 1][1]);
                }
            }
#pragma unroll
            for (int mt = 0; mt < 4; ++mt)
#pragma unroll
                for (int nt = 0; nt < 4; ++nt)
                    mma_bf16(acc[mt][nt], af[mt][0], af[mt][1], af[mt][2], af[mt][3], bfr[nt][0], bfr[nt][1]);
        }
    }
    cp_async_wait<0>();

    const int gq = lane >> 2, tq = lane & 3;
#pragma unroll
    for (int mt = 0; mt < 4; ++mt)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int r = m0 + wm + 16 * mt + gq + 8 * h;
            if (r >= g.M) continue;
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                const int c = n0 + wn + 8 * nt + 2 * tq;
                const float x0 = acc[mt][nt][2 * h], x1 = acc[mt][nt][2 * h + 1];
                const size_t o = static_cast<size_t>(r) * g.ldc + c;
                if constexpr (EPI == kEpiResid) {
                    const float2 rv = *reinterpret_cast<const float2*>(g.R + o);
                    *reinterpret_cast<float2*>(g.Cf + o) = make_float2(x0 + rv.x, x1 + rv.y);
                } else if constexpr (EPI == kEpiBf16) {
                    *reinterpret_cast<uint32_t*>(g.Cb + o) = pack_bf16(x0, x1);
                } else {
                    *reinterpret_cast<float2*>(g.Cf + blockIdx.z * g.part_stride + o) = make_float2(x0, x1);
                }
            }
        }
}

template <bool AKROW, bool BKROW, int EPI>
cudaError_t launch_gemm(const GemmArgs& g, int splits, cudaStream_t st) {
    cudaError_t e = ensure_smem<dec_gemm_kernel<AKROW, BKROW, EPI>>(kGSmem);
    if (e != cudaSuccess) return e;
    const dim3 grid(g.N / kGN, (g.M + kGM - 1) / kGM, splits);
    dec_gemm_kernel<AKROW, BKROW, EPI><<<grid, kGThreads, kGSmem, st>>>(g);
    note_launch();
    return cudaGetLastError();
}

// Offsets: one warp per query, lane l holding channels 4 (l + 32 j) .. + 3.
__global__ void __launch_bounds__(256)
    dec_offsets_kernel(const float* __restrict__ ref, const float* __restrict__ f, int T, int D,
                       const float* __restrict__ w_off, const float* __restrict__ b_off, float* __restrict__ q) {
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (t >= T) return;
    const float* fr = f + static_cast<size_t>(t) * D;
    float ax = 0.f, ay = 0.f;
    for (int c = 4 * lane; c < D; c += 128) {
        const float4 fv = *reinterpret_cast<const float4*>(fr + c);
        const float4 w01 = __ldg(reinterpret_cast<const float4*>(w_off + 2 * c));
        const float4 w23 = __ldg(reinterpret_cast<const float4*>(w_off + 2 * c + 4));
        ax = fmaf(fv.x, w01.x, ax);
        ay = fmaf(fv.x, w01.y, ay);
        ax = fmaf(fv.y, w01.z, ax);
        ay = fmaf(fv.y, w01.w, ay);
        ax = fmaf(fv.z, w23.x, ax);
        ay = fmaf(fv.z, w23.y, ay);
        ax = fmaf(fv.w, w23.z, ax);
        ay = fmaf(fv.w, w23.w, ay);
    }
    ax = warp_sum(ax);
    ay = warp_sum(ay);
    if (lane == 0) {
        const float2 r = reinterpret_cast<const float2*>(ref)[t];
        reinterpret_cast<float2*>(q)[t] = make_float2(r.x + (b_off[0] + ax), r.y + (b_off[1] + ay));
    }
}

// df_out (fp32) -> bf16, eight elements per thread.
__global__ void __launch_bounds__(256)
    dec_to_bf16_kernel(const float* __restrict__ x, size_t n8, bf16* __restrict__ y) {
    for (size_t i = blockIdx.x * 256ull + threadIdx.x; i < n8; i += static_cast<size_t>(gridDim.x) * 256) {
        const float4 a = reinterpret_cast<const float4*>(x)[2 * i];
        const float4 b = reinterpret_cast<const float4*>(x)[2 * i + 1];
        uint4 o;
        o.x = pack_bf16(a.x, a.y);
        o.y = pack_bf16(a.z, a.w);
        o.z = pack_bf16(b.x, b.y);
        o.w = pack_bf16(b.z, b.w);
        reinterpret_cast<uint4*>(y)[i] = o;
    }
}

// Offset-head backward, stage 1: CTA p takes queries [p T / P, (p + 1) T / P); its D threads
// are 4 row groups x D/4 channel quads, row group r taking queries t0 + r, t0 + r + 4, ... in
// order: df_in = df_out + dq W_off^T (float4 rows), and per quad the sums of f_c dq and (quad
// 0) of dq; the four row groups' sums are then added in row-group order.
__global__ void __launch_bounds__(1024)
    dec_offsets_bwd_kernel(const float* __restrict__ f, const float* __restrict__ dq,
                           const float* __restrict__ df_out, int T, int D, const float* __restrict__ w_off,
                           float* __restrict__ df_in, float* __restrict__ part) {
    extern __shared__ float red[];  // [4][2 D + 2]
    const int nq = D / 4;
    const int rg = threadIdx.x / nq, cq = threadIdx.x - rg * nq;
    const int p = blockIdx.x;
    const int t0 = static_cast<int>(static_cast<long long>(p) * T / kDecParts);
    const int t1 = static_cast<int>(static_cast<long long>(p + 1) * T / kDecParts);
    const float4 wa = reinterpret_cast<const float4*>(w_off)[2 * cq];      // channels 4cq, 4cq+1
    const float4 wb = reinterpret_cast<const float4*>(w_off)[2 * cq + 1];  // channels 4cq+2, 4cq+3
    float sx[4] = {0.f, 0.f, 0.f, 0.f}, sy[4] = {0.f, 0.f, 0.f, 0.f}, bx = 0.f, by = 0.f;
#pragma unroll 2
    for (int t = t0 + rg; t < t1; t += 4) {
        const float2 g = reinterpret_cast<const float2*>(dq)[t];
        const size_t o = static_cast<size_t>(t) * nq + cq;
        const float4 fv = reinterpret_cast<const float4*>(f)[o];
        const float4 dv = reinterpret_cast<const float4*>(df_out)[o];
        float4 r;
        r.x = dv.x + (g.x * wa.x + g.y * wa.y);
        r.y = dv.y + (g.x * wa.z + g.y * wa.w);
        r.z = dv.z + (g.x * wb.x + g.y * wb.y);
        r.w = dv.w + (g.x * wb.z + g.y * wb.w);
        reinterpret_cast<float4*>(df_in)[o] = r;
        const float fa[4] = {fv.x, fv.y, fv.z, fv.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            sx[e] = fmaf(fa[e], g.x, sx[e]);
            sy[e] = fmaf(fa[e], g.y, sy[e]);
        }
        bx += g.x;
        by += g.y;
    }
    const int n = 2 * D + 2;
    float* my = red + rg * n;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        my[2 * (4 * cq + e)] = sx[e];
        my[2 * (4 * cq + e) + 1] = sy[e];
    }
    if (cq == 0) {
        my[2 * D] = bx;
        my[2 * D + 1] = by;
    }
    __syncthreads();
    float* pp = part + static_cast<size_t>(p) * n;
    for (int o = threadIdx.x; o < n; o += blockDim.x) pp[o] = ((red[o] + red[n + o]) + red[2 * n + o]) + red[3 * n + o];
}

// Stage 2: CTA over 32 outputs; warp w adds parts w, w + 8, ... in order, then the eight warp
// sums are added in warp order -> dW_off [D][2], db_off [2].
__global__ void __launch_bounds__(256)
    dec_offsets_reduce_kernel(const float* __restrict__ part, int D, float* __restrict__ dw_off,
                              float* __restrict__ db_off) {
    __shared__ float wsum[8][32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int o = blockIdx.x * 32 + lane;
    const int n = 2 * D + 2;
    float a = 0.f;
    if (o < n)
#pragma unroll 8
        for (int p = warp; p < kDecParts; p += 8) a += part[static_cast<size_t>(p) * n + o];
    wsum[warp][lane] = a;
    __syncthreads();
    if (warp != 0 || o >= n) return;
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) sum += wsum[w][lane];
    if (o < 2 * D) dw_off[o] = sum;
    else db_off[o - 2 * D] = sum;
}

// dW_o = the split parts summed in order.
__global__ void __launch_bounds__(256)
    dec_split_reduce_kernel(const float* __restrict__ part, size_t n, int splits, float* __restrict__ out) {
    const size_t o = blockIdx.x * 256ull + threadIdx.x;
    if (o >= n) return;
    float a = 0.f;
    for (int z = 0; z < splits; ++z) a += part[static_cast<size_t>(z) * n + o];
    out[o] = a;
}

int sm_count() {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        sms = 148;
    return sms;
}

}  // namespace

int dec_wo_splits(int T, int d, int D) {
    const int tiles = (d / kGM) * (D / kGN);
    int s = (2 * 148 + tiles - 1) / tiles;
    const int kt = (T + kGK - 1) / kGK;
    if (s > kt) s = kt;
    if (s > kMaxSplits) s = kMaxSplits;
    return s < 1 ? 1 : s;
}

DecWorkspace dec_workspace_layout(int B, int Q, int N, int d, int D, int K) {
    auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
    const size_t T = static_cast<size_t>(B) * Q;
    DecWorkspace w;
    size_t off = 0;
    w.dfb = off;    off += up(2 * T * D);
    w.dv = off;     off += up(2 * T * d);
    w.dq = off;     off += up(8 * T);
    w.wo_part = off; off += up(4 * static_cast<size_t>(dec_wo_splits(static_cast<int>(T), d, D)) * d * D);
    w.off_part = off; off += up(4 * static_cast<size_t>(kDecParts) * (2 * D + 2));
    w.knn = off;
    off += up(knn_workspace_layout(B, Q, N, d, K).total);
    w.total = off;
    return w;
}

cudaError_t launch_dec_fwd(const DecArgs& a, cudaStream_t st) {
    const int T = a.B * a.Q;
    if (T == 0) return cudaSuccess;
    dec_offsets_kernel<<<(T + 7) / 8, 256, 0, st>>>(a.ref, a.f_in, T, a.D, a.w_off, a.b_off, a.q);
    note_launch();
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    KnnArgs k = a.knn;
    k.queries = a.q;
    k.out = a.v;
    if ((e = launch_knn_fwd(k, st)) != cudaSuccess) return e;
    GemmArgs g = {};
    g.A = a.v; g.lda = a.d;                 // [T][d], k-contiguous
    g.B = a.w_o; g.ldb = a.D;               // [d][D], k-rows
    g.M = T; g.N = a.D; g.K = a.d; g.kchunk = a.d;
    g.R = a.f_in; g.Cf = a.f_out; g.ldc = a.D;
    return launch_gemm<false, true, kEpiResid>(g, 1, st);
}

cudaError_t launch_dec_bwd(const DecArgs& a, cudaStream_t st) {
    const int T = a.B * a.Q;
    cudaError_t e;
    if (T > 0) {
        const size_t n8 = static_cast<size_t>(T) * a.D / 8;
        const size_t want = (n8 + 255) / 256, cap = static_cast<size_t>(sm_count()) * 8;
        const unsigned cb = static_cast<unsigned>(want < cap ? want : cap);
        dec_to_bf16_kernel<<<cb, 256, 0, st>>>(a.df_out, n8, a.dfb);
        note_launch();
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        // dv = df W_o^T: A = df [T][D] (k-contiguous), B(k = D, n = d) = W_o[n][k] ([d][D], k-contiguous)
        GemmArgs g = {};
        g.A = a.dfb; g.lda = a.D;
        g.B = a.w_o; g.ldb = a.D;
        g.M = T; g.N = a.d; g.K = a.D; g.kchunk = a.D;
        g.Cb = a.dv; g.ldc = a.d;
        if ((e = launch_gemm<false, false, kEpiBf16>(g, 1, st)) != cudaSuccess) return e;
    }
    // dW_o = v^T df: A(m = d, k = T) = v[k][m] (k-rows), B(k = T, n = D) = df[k][n] (k-rows)
    const int splits = dec_wo_splits(T, a.d, a.D);
    const int kt = (T + kGK - 1) / kGK;
    GemmArgs w = {};
    w.A = a.v; w.lda = a.d;
    w.B = a.dfb; w.ldb = a.D;
    w.M = a.d; w.N = a.D; w.K = T; w.kchunk = ((kt + splits - 1) / splits) * kGK;
    w.Cf = a.wo_part; w.ldc = a.D; w.part_stride = static_cast<size_t>(a.d) * a.D;
    if ((e = launch_gemm<true, true, kEpiPart>(w, splits, st)) != cudaSuccess) return e;
    const size_t nw = static_cast<size_t>(a.d) * a.D;
    dec_split_reduce_kernel<<<static_cast<unsigned>((nw + 255) / 256), 256, 0, st>>>(a.wo_part, nw, splits, a.dw_o);
    note_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    KnnArgs k = a.knn;
    k.queries = a.q;
    k.dout = a.dv;
    k.dq = a.dq;
    if ((e = launch_knn_bwd(k, st)) != cudaSuccess) return e;
    const size_t osm = sizeof(float) * 4 * (2 * static_cast<size_t>(a.D) + 2);
    if ((e = ensure_smem<dec_offsets_bwd_kernel>(osm)) != cudaSuccess) return e;
    dec_offsets_bwd_kernel<<<kDecParts, a.D, osm, st>>>(a.f_in, a.dq, a.df_out, T, a.D, a.w_off, a.df_in,
                                                         a.off_part);
    note_launch();
    dec_offsets_reduce_kernel<<<(2 * a.D + 2 + 31) / 32, 256, 0, st>>>(a.off_part, a.D, a.dw_off, a.db_off);
    note_launch();
    return cudaGetLastError();
}

}  // namespace acl
