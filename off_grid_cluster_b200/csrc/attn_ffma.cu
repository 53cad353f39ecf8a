// attn_ffma.cu -- the cluster-attention forward on the FMA pipes only: the reference
// variant the tensor-core forward (attn.cu) is measured against.
//
// AFFMAE notes, Method "Overall Architecture" (local cluster attention over off-grid tokens)
// and the arXiv abstract page (mixed-precision Flash-style cluster attention kernels).  For a
// valid query i of cluster g, head h and every valid key j of the neighbourhood table row g:
//   s_ij = scale <q_i, k_j> + a_h dx + b_h dy - c_h (dx^2 + dy^2),  dx = x_j - x_i, dy = y_j - y_i
//   o_i = sum_j softmax_j(s_ij) v_j,  lse_i = log sum_j exp(s_ij)
// exactly what acl_cluster_attn_fwd computes; only the arithmetic units differ.
//
// One warp per (cluster, head) item: lane = 4 i + r holds query slot i (0..7) and scores the
// keys m = r, r + 4, ... of the row (fp32 dot products of bf16 rows read through L1), the four
// lanes of a query combine the row maximum and sum by shuffles, then lane r accumulates output
// channels 8 r .. 8 r + 7 over all M keys, taking each key's probability from the lane that
// scored it.  No shared memory and no tensor-core instruction.
#include "internal.h"

namespace acl {

namespace {

constexpr int kFfmaWarps = 8;
constexpr int kFfmaMaxKeysPerLane = 16;  // neighbourhood slots up to 64, four lanes per query

__device__ __forceinline__ void unpack8f(uint4 u, float (&f)[8]) {
    f[0] = bf16_lo(u.x);
    f[1] = bf16_hi(u.x);
    f[2] = bf16_lo(u.y);
    f[3] = bf16_hi(u.y);
    f[4] = bf16_lo(u.z);
    f[5] = bf16_hi(u.z);
    f[6] = bf16_lo(u.w);
    f[7] = bf16_hi(u.w);
}

__device__ __forceinline__ int ffma_tok(int t, int N) { return (t >= 0 && t < N) ? t : -1; }

__global__ void __launch_bounds__(32 * kFfmaWarps) attn_fwd_ffma_kernel(const AttnArgs a) {
    const int lane = threadIdx.x & 31;
    const int i = lane >> 2, r = lane & 3;
    const long long items = static_cast<long long>(a.B) * a.G * a.H;
    const long long stride = static_cast<long long>(gridDim.x) * kFfmaWarps;
    const float2* xy = reinterpret_cast<const float2*>(a.xy);
    const float kLog2 = kLog2e;
    for (long long it = static_cast<long long>(blockIdx.x) * kFfmaWarps + (threadIdx.x >> 5); it < items;
         it += stride) {
        const long long bg = it / a.H;
        const int h = static_cast<int>(it - bg * a.H);
        const int b = static_cast<int>(bg / a.G);
        const size_t tok0 = static_cast<size_t>(b) * a.N;
        const int qt = ffma_tok(__ldg(a.clusters + bg * 8 + i), a.N);
        const float ab = __ldg(a.bias + 3 * h), bb = __ldg(a.bias + 3 * h + 1), cb = __ldg(a.bias + 3 * h + 2);
        float q[32];
        float2 qxy = make_float2(0.f, 0.f);
        if (qt >= 0) {
            const uint4* qp = reinterpret_cast<const uint4*>(a.q + ((tok0 + qt) * a.H + h) * 32);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float f[8];
                unpack8f(__ldg(qp + c), f);
#pragma unroll
                for (int e = 0; e < 8; ++e) q[8 * c + e] = f[e] * a.scale;
            }
            qxy = __ldg(xy + tok0 + qt);
        } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) q[e] = 0.f;
        }
        // scores of this lane's keys m = r + 4 u
        const int32_t* row = a.nbr + bg * a.M;
        float s[kFfmaMaxKeysPerLane];
        int kt[kFfmaMaxKeysPerLane];
        float mx = -INFINITY;
#pragma unroll
        for (int u = 0; u < kFfmaMaxKeysPerLane; ++u) {
            const int m = r + 4 * u;
            const int t = (m < a.M) ? ffma_tok(__ldg(row + m), a.N) : -1;
            kt[u] = t;
            s[u] = -INFINITY;
            if (t >= 0 && qt >= 0) {
                const uint4* kp = reinterpret_cast<const uint4*>(a.k + ((tok0 + t) * a.H + h) * 32);
                float acc = 0.f;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    float f[8];
                    unpack8f(__ldg(kp + c), f);
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc = fmaf(q[8 * c + e], f[e], acc);
                }
                const float2 p = __ldg(xy + tok0 + t);
                const float dx = p.x - qxy.x, dy = p.y - qxy.y;
                s[u] = acc + ab * dx + bb * dy - cb * (dx * dx + dy * dy);
                mx = fmaxf(mx, s[u]);
            }
        }
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        float sum = 0.f;
#pragma unroll
        for (int u = 0; u < kFfmaMaxKeysPerLane; ++u) {
            s[u] = kt[u] >= 0 && qt >= 0 ? exp2f((s[u] - mx) * kLog2) : 0.f;
            sum += s[u];
        }
        sum += __shfl_xor_sync(0xffffffffu, sum, 1);
        sum += __shfl_xor_sync(0xffffffffu, sum, 2);
        // channels 8 r .. 8 r + 7 over every key of the row (probability and token from the
        // lane of this query that scored the key)
        float o[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        const int base = lane & ~3;
#pragma unroll
        for (int u = 0; u < kFfmaMaxKeysPerLane; ++u) {
            if (4 * u >= a.M) break;  // uniform
#pragma unroll
            for (int rr = 0; rr < 4; ++rr) {
                const float p = __shfl_sync(0xffffffffu, s[u], base + rr);
                const int t = __shfl_sync(0xffffffffu, kt[u], base + rr);
                if (t >= 0 && p != 0.f) {
                    float f[8];
                    unpack8f(__ldg(reinterpret_cast<const uint4*>(a.v + ((tok0 + t) * a.H + h) * 32 + 8 * r)), f);
#pragma unroll
                    for (int e = 0; e < 8; ++e) o[e] = fmaf(p, f[e], o[e]);
                }
            }
        }
        if (qt >= 0) {
            const float inv = sum > 0.f ? 1.f / sum : 0.f;
            uint4 w;
            w.x = pack_bf16(o[0] * inv, o[1] * inv);
            w.y = pack_bf16(o[2] * inv, o[3] * inv);
            w.z = pack_bf16(o[4] * inv, o[5] * inv);
            w.w = pack_bf16(o[6] * inv, o[7] * inv);
            const size_t orow = (tok0 + qt) * a.H + h;
            *reinterpret_cast<uint4*>(a.o + orow * 32 + 8 * r) = w;
            if (r == 0) a.lse[orow] = sum > 0.f ? mx + logf(sum) : -INFINITY;
        }
    }
}

}  // namespace

cudaError_t launch_attn_fwd_ffma(const AttnArgs& a, cudaStream_t st) {
    const long long items = static_cast<long long>(a.B) * a.G * a.H;
    if (items == 0) return cudaSuccess;
    const long long slots = static_cast<long long>(sm_count()) * resident<attn_fwd_ffma_kernel>(32 * kFfmaWarps, 0);
    const long long need = (items + kFfmaWarps - 1) / kFfmaWarps;
    const unsigned blocks = static_cast<unsigned>(need < slots ? need : slots);
    attn_fwd_ffma_kernel<<<blocks, 32 * kFfmaWarps, 0, st>>>(a);
    note_launch();
    return cudaGetLastError();
}

}  // namespace acl
