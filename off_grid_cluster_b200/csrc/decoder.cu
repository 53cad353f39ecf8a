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
// The GEMMs run on the tcgen05 tensor cores with the accumulator in tensor memory; each
// operand is staged in its stored layout (K-major or MN-major shared-memory descriptors), so
// no operand is transposed in memory.
#include <float.h>

#include "internal.h"

namespace acl {

namespace {

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

// ---------------------------------------------------------------- tcgen05 GEMM
//
// The same products on the 5th-generation tensor cores: a 128 x 128 fp32 accumulator in
// tensor memory (128 columns), 64-deep k-tiles staged by cp.async into shared memory in the
// canonical 128-byte-swizzle layouts (K-major: 128-byte rows, 16-byte chunk c of row r at
// c ^ (r mod 8); MN-major: two 64-element halves of 64 k-rows each, the same swizzle on the
// k-row), 3 stages.  One thread issues the four k16 MMAs of a stage and commits them to the
// stage's mbarrier; a stage is refilled only after that barrier completes.  Every wait is
// bounded: a wait that gives up counts in tc_timeouts (read by acl_device_check) and the CTA
// skips its remaining MMAs, waits once more for those in flight and frees its tensor memory.
constexpr int kTM = 128, kTN = 128, kTK = 64, kTStages = 3, kTThreads = 256;
constexpr int kTTileBytes = kTM * kTK * 2;                  // 16 KB, A or B
constexpr int kTStageBytes = 2 * kTTileBytes;
constexpr int kTSmem = kTStages * kTStageBytes + 1024 + 64;  // + alignment slack, barriers, slot
constexpr long long kTWaitCycles = 1000000000LL;
constexpr uint32_t kTmemCols = 128;

__device__ unsigned int tc_timeouts;
// SM clocks a main-loop wait may take before it gives up (kTWaitCycles unless a test lowers
// it; 0 gives up at once).  The final wait
// for the MMAs in flight always allows kTWaitCycles, so tensor memory is freed only after
// the MMAs that use it have completed.
__device__ long long tc_wait_cycles = kTWaitCycles;

// Shared-memory matrix descriptor: start, leading and stride byte offsets in 16-byte units,
// descriptor version 1, 128-byte swizzle.
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo16, uint32_t sbo16) {
    return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(lbo16 & 0x3FFFu) << 16) |
           (static_cast<uint64_t>(sbo16 & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
// Operand descriptor of k16 step j of a staged tile: K-major tiles advance 32 bytes inside the
// swizzle atom (8-row groups 1024 bytes apart); MN-major tiles advance 16 k-rows (2048 bytes),
// their two 64-element halves 8192 bytes apart and 8-k-row groups 1024 bytes apart.
template <bool MN>
__device__ __forceinline__ uint64_t tile_desc(uint32_t tile, int j) {
    return MN ? umma_desc(tile + 2048u * j, 8192u >> 4, 1024u >> 4) : umma_desc(tile + 32u * j, 1u, 1024u >> 4);
}
// Instruction descriptor, kind::f16: fp32 accumulator, bf16 A and B, majors, N / 8, M / 16.
template <bool AMN, bool BMN>
__host__ __device__ constexpr uint32_t tc_idesc() {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((AMN ? 1u : 0u) << 15) | ((BMN ? 1u : 0u) << 16) |
           (static_cast<uint32_t>(kTN >> 3) << 17) | (static_cast<uint32_t>(kTM >> 4) << 24);
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Wait for the phase of the given parity to complete, giving up after `limit` SM clocks
// (kTWaitCycles: about half a second): try_wait itself returns after a bounded suspension.
// A limit of 0 gives up at once (a test's way to make every main-loop wait run out).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, long long limit = kTWaitCycles) {
    if (limit <= 0) return false;
    const long long t0 = clock64();
    for (;;) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}\n"
            : "=r"(done)
            : "r"(bar), "r"(parity)
            : "memory");
        if (done) return true;
        if (clock64() - t0 > limit) return false;
    }
}

// Stage one operand tile (1024 chunks of 16 bytes, 4 per thread).  MN: stored [K][MN]
// (MN contiguous), rows = extent of MN; else stored [MN][K].  Out-of-range chunks are zeroed.
template <bool MN>
__device__ __forceinline__ void tc_load_tile(uint32_t tile, const bf16* __restrict__ src, int ld, int mn0,
                                             int rows, int k0, int kend, int tid) {
#pragma unroll
    for (int i = 0; i < 1024 / kTThreads; ++i) {
        const int q = tid + i * kTThreads;
        if constexpr (!MN) {
            const int r = q >> 3, c = q & 7;
            const int gr = mn0 + r, gk = k0 + 8 * c;
            const bool ok = gr < rows && gk < kend;
            cp_async16(tile + r * 128 + ((c ^ (r & 7)) << 4), ok ? src + static_cast<size_t>(gr) * ld + gk : src, ok);
        } else {
            const int kr = q >> 4, mc = q & 15, h = mc >> 3, c = mc & 7;
            const int gk = k0 + kr, gc = mn0 + 8 * mc;
            const bool ok = gk < kend && gc < rows;
            cp_async16(tile + h * 8192 + kr * 128 + ((c ^ (kr & 7)) << 4),
                       ok ? src + static_cast<size_t>(gk) * ld + gc : src, ok);
        }
    }
}

template <bool AMN, bool BMN, int EPI>
__global__ void __launch_bounds__(kTThreads)
    tc_gemm_kernel(const GemmArgs g) {
    extern __shared__ uint8_t tsm[];
    const uint32_t raw = smem_addr(tsm);
    const uint32_t s0 = (raw + 1023u) & ~1023u;
    const uint32_t bar0 = s0 + kTStages * kTStageBytes;
    const uint32_t slot = bar0 + 8 * kTStages;
    const volatile uint32_t* slot_p = reinterpret_cast<const volatile uint32_t*>(tsm + (slot - raw));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int m0 = blockIdx.x * kTM, n0 = blockIdx.y * kTN;  // M tiles on x: up to 2^31 - 1
    const int kz0 = blockIdx.z * g.kchunk;
    const int kz1 = min(g.K, kz0 + g.kchunk);
    const int nk = kz1 > kz0 ? (kz1 - kz0 + kTK - 1) / kTK : 0;

    if (tid == 0) {
        for (int s = 0; s < kTStages; ++s)
            asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar0 + 8 * s), "r"(1) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot), "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *slot_p;

    auto load = [&](int stage, int kt) {
        const uint32_t sa = s0 + stage * kTStageBytes, sb = sa + kTTileBytes;
        const int k0 = kz0 + kt * kTK;
        tc_load_tile<AMN>(sa, g.A, g.lda, m0, g.M, k0, kz1, tid);
        tc_load_tile<BMN>(sb, g.B, g.ldb, n0, g.N, k0, kz1, tid);
    };
#pragma unroll
    for (int s = 0; s < kTStages - 1; ++s) {
        if (s < nk) load(s, s);
        cp_async_commit();
    }
    const long long wait_limit = tc_wait_cycles;
    bool ok = true;
    int issued = 0;  // k-tiles whose MMAs were issued
    for (int kt = 0; kt < nk; ++kt) {
        cp_async_wait<kTStages - 2>();
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        if (!__syncthreads_and(ok)) break;  // a wait gave up somewhere: stop issuing
        if (tid == 0) {
            tc_fence_after();
            const uint32_t sa = s0 + (kt % kTStages) * kTStageBytes, sb = sa + kTTileBytes;
#pragma unroll
            for (int j = 0; j < kTK / 16; ++j) {
                const uint64_t ad = tile_desc<AMN>(sa, j), bd = tile_desc<BMN>(sb, j);
                const uint32_t acc = (kt > 0 || j > 0) ? 1u : 0u;
                asm volatile(
                    "{\n\t.reg .pred p;\n\t"
                    "setp.ne.b32 p, %4, 0;\n\t"
                    "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}\n"
                    ::"r"(tmem), "l"(ad), "l"(bd), "r"(tc_idesc<AMN, BMN>()), "r"(acc), "r"(0u), "r"(0u), "r"(0u),
                    "r"(0u)
                    : "memory");
            }
            asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                             bar0 + 8 * (kt % kTStages))
                         : "memory");
        }
        issued = kt + 1;
        const int nxt = kt + kTStages - 1;
        if (nxt < nk) {
            if (kt >= 1) ok = ok && mbar_wait(bar0 + 8 * ((kt - 1) % kTStages), ((kt - 1) / kTStages) & 1, wait_limit);
            if (ok) load(nxt % kTStages, nxt);
        }
        cp_async_commit();
    }
    cp_async_wait<0>();
    // the last commit covers every MMA issued before it
    if (issued > 0) {
        const bool done = mbar_wait(bar0 + 8 * ((issued - 1) % kTStages), ((issued - 1) / kTStages) & 1);
        ok = ok && done;
    }
    ok = __syncthreads_and(ok) != 0;
    tc_fence_after();
    const bool have = ok && nk > 0 && issued == nk;
    // warp w reads tensor-memory lanes 32 (w mod 4) .. + 31 (its rows), columns of half w / 4
    const int row = m0 + 32 * (warp & 3) + lane;
    const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16);
    const int c0 = (warp >> 2) * (kTN / 2);
    // the residual's 64 columns of this row, loaded before the accumulator is read back
    float4 rv[kTN / 8];
    if constexpr (EPI == kEpiResid) {
        if (row < g.M) {
            const float4* rp = reinterpret_cast<const float4*>(g.R + static_cast<size_t>(row) * g.ldc + n0 + c0);
#pragma unroll
            for (int e = 0; e < kTN / 8; ++e) rv[e] = rp[e];
        }
    }
#pragma unroll
    for (int cj = c0; cj < c0 + kTN / 2; cj += 16) {
        uint32_t v[16];
        if (have) {
            asm volatile(
                "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
                "%13, %14, %15}, [%16];\n"
                : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
                  "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]),
                  "=r"(v[15])
                : "r"(taddr + cj));
            asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) v[e] = 0u;
        }
        if (row >= g.M) continue;
        const size_t o = static_cast<size_t>(row) * g.ldc + n0 + cj;
        if constexpr (EPI == kEpiResid) {
#pragma unroll
            for (int e = 0; e < 16; e += 4) {
                const float4 r4 = rv[(cj - c0 + e) / 4];
                *reinterpret_cast<float4*>(g.Cf + o + e) =
                    make_float4(__uint_as_float(v[e]) + r4.x, __uint_as_float(v[e + 1]) + r4.y,
                                __uint_as_float(v[e + 2]) + r4.z, __uint_as_float(v[e + 3]) + r4.w);
            }
        } else if constexpr (EPI == kEpiBf16) {
            uint4 w0, w1;
            w0.x = pack_bf16(__uint_as_float(v[0]), __uint_as_float(v[1]));
            w0.y = pack_bf16(__uint_as_float(v[2]), __uint_as_float(v[3]));
            w0.z = pack_bf16(__uint_as_float(v[4]), __uint_as_float(v[5]));
            w0.w = pack_bf16(__uint_as_float(v[6]), __uint_as_float(v[7]));
            w1.x = pack_bf16(__uint_as_float(v[8]), __uint_as_float(v[9]));
            w1.y = pack_bf16(__uint_as_float(v[10]), __uint_as_float(v[11]));
            w1.z = pack_bf16(__uint_as_float(v[12]), __uint_as_float(v[13]));
            w1.w = pack_bf16(__uint_as_float(v[14]), __uint_as_float(v[15]));
            *reinterpret_cast<uint4*>(g.Cb + o) = w0;
            *reinterpret_cast<uint4*>(g.Cb + o + 8) = w1;
        } else {
            float* dst = g.Cf + blockIdx.z * g.part_stride + o;
#pragma unroll
            for (int e = 0; e < 16; e += 4)
                *reinterpret_cast<float4*>(dst + e) = make_float4(__uint_as_float(v[e]), __uint_as_float(v[e + 1]),
                                                                  __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
    }
    if (!ok && tid == 0) atomicAdd(&tc_timeouts, 1u);
}

template <bool AMN, bool BMN, int EPI>
cudaError_t launch_tc_gemm(const GemmArgs& g, int splits, cudaStream_t st) {
    cudaError_t e = ensure_smem<tc_gemm_kernel<AMN, BMN, EPI>>(kTSmem);
    if (e != cudaSuccess) return e;
    const dim3 grid((g.M + kTM - 1) / kTM, g.N / kTN, splits);
    tc_gemm_kernel<AMN, BMN, EPI><<<grid, kTThreads, kTSmem, st>>>(g);
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

}  // namespace

int dec_wo_splits(int T, int d, int D) {
    const int tiles = (d / kTM) * (D / kTN);
    int s = (2 * 148 + tiles - 1) / tiles;
    const int kt = (T + kTK - 1) / kTK;
    if (s > kt) s = kt;
    if (s > kMaxSplits) s = kMaxSplits;
    return s < 1 ? 1 : s;
}

cudaError_t set_tc_wait_cycles(long long cycles) {
    return cudaMemcpyToSymbol(tc_wait_cycles, &cycles, sizeof(long long));
}

cudaError_t read_tc_timeouts(unsigned int* count) {
    cudaError_t e = cudaMemcpyFromSymbol(count, tc_timeouts, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(tc_timeouts, &zero, sizeof(unsigned int));
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
    return launch_tc_gemm<false, true, kEpiResid>(g, 1, st);
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
        if ((e = launch_tc_gemm<false, false, kEpiBf16>(g, 1, st)) != cudaSuccess) return e;
    }
    // dW_o = v^T df: A(m = d, k = T) = v[k][m] (k-rows), B(k = T, n = D) = df[k][n] (k-rows)
    const int splits = dec_wo_splits(T, a.d, a.D);
    const int kt = (T + kTK - 1) / kTK;
    GemmArgs w = {};
    w.A = a.v; w.lda = a.d;
    w.B = a.dfb; w.ldb = a.D;
    w.M = a.d; w.N = a.D; w.K = T; w.kchunk = ((kt + splits - 1) / splits) * kTK;
    w.Cf = a.wo_part; w.ldc = a.D; w.part_stride = static_cast<size_t>(a.d) * a.D;
    if ((e = launch_tc_gemm<true, true, kEpiPart>(w, splits, st)) != cudaSuccess) return e;
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
