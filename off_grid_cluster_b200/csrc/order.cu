// order.cu -- space-filling (Z-order) token order.
//
// AFFMAE notes, "Limitations": the dense lookup table and the off-grid gathers are bound by
// memory traffic, and space-filling curves are suggested so that tokens that are close on
// the image are close in memory.  acl_token_order gives, per image, the token ids ordered by
// the Morton code of their cell on the H x W grid (column bit i at bit 2i, row bit i at bit
// 2i + 1), ties by id; permuting the tokens by it puts every 2^k x 2^k block of cells in one
// contiguous run.  Integer only and bit-exact.
//
// One 1024-thread CTA per image, all in shared memory: a counting sort of the tokens into
// P = next_pow2(N) buckets by the top bits of their code (a monotone bucket function), then
// an exact insertion sort of each bucket by (code, id).  When a bucket holds more than 32
// tokens (many tokens in a few cells) the CTA falls back to a bitonic sort of the P packed
// (code, id) keys.
#include "internal.h"

namespace acl {

namespace {

constexpr int kOrderThreads = 1024;
constexpr int kOrderBucketMax = 32;

__device__ __forceinline__ uint32_t spread_bits(uint32_t v) {  // bit i -> bit 2i (16 bits)
    v &= 0xFFFFu;
    v = (v | (v << 8)) & 0x00FF00FFu;
    v = (v | (v << 4)) & 0x0F0F0F0Fu;
    v = (v | (v << 2)) & 0x33333333u;
    v = (v | (v << 1)) & 0x55555555u;
    return v;
}

__host__ __device__ __forceinline__ int pow2_at_least(int n) {
    int p = 1;
    while (p < n) p <<= 1;
    return p;
}

// Exclusive prefix sum of data[0..n) in place by the whole block; returns the total.
__device__ int order_scan(int* data, int n, int* scratch) {
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

// Shared-memory layout: code [N] u32 | U = max(keys [P] u64, cnt [P] i32 + list [N] i32) |
// scratch [40] i32
struct OrderSmem {
    size_t u, scratch, total;
};
__host__ __device__ __forceinline__ OrderSmem order_smem_layout(int N) {
    const size_t P = static_cast<size_t>(pow2_at_least(N));
    const size_t n = static_cast<size_t>(N);
    OrderSmem L;
    L.u = (4 * n + 15) & ~size_t(15);
    const size_t ub = (8 * P > 4 * P + 4 * n) ? 8 * P : 4 * P + 4 * n;
    L.scratch = L.u + ((ub + 15) & ~size_t(15));
    L.total = L.scratch + 40 * 4;
    return L;
}

__global__ void __launch_bounds__(kOrderThreads)
    token_order_kernel(const float* __restrict__ xy, int N, int GH, int GW, int code_bits,
                       int32_t* __restrict__ perm) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int b = blockIdx.x, tid = threadIdx.x;
    const OrderSmem L = order_smem_layout(N);
    const int P = pow2_at_least(N);
    int lp = 0;
    while ((1 << lp) < P) ++lp;
    const int shift = code_bits > lp ? code_bits - lp : 0;
    uint32_t* code = reinterpret_cast<uint32_t*>(smem);
    int* cnt = reinterpret_cast<int*>(smem + L.u);  // [P]
    int* list = cnt + P;                           // [N]
    int* scratch = reinterpret_cast<int*>(smem + L.scratch);
    const float2* img = reinterpret_cast<const float2*>(xy) + static_cast<size_t>(b) * N;
    int32_t* out = perm + static_cast<size_t>(b) * N;

    for (int i = tid; i < P; i += kOrderThreads) cnt[i] = 0;
    for (int t = tid; t < N; t += kOrderThreads) {
        const float2 p = img[t];
        const uint32_t r = static_cast<uint32_t>(quantise(p.y, GH));
        const uint32_t c = static_cast<uint32_t>(quantise(p.x, GW));
        code[t] = spread_bits(c) | (spread_bits(r) << 1);
    }
    __syncthreads();
    for (int t = tid; t < N; t += kOrderThreads) atomicAdd(&cnt[code[t] >> shift], 1);
    __syncthreads();
    int crowded = 0;
    for (int i = tid; i < P; i += kOrderThreads) crowded |= (cnt[i] > kOrderBucketMax);
    crowded = __syncthreads_or(crowded);
    if (!crowded) {
        order_scan(cnt, P, scratch);
        for (int t = tid; t < N; t += kOrderThreads) list[atomicAdd(&cnt[code[t] >> shift], 1)] = t;
        __syncthreads();  // cnt[bb] = end of bucket bb
        for (int bb = tid; bb < P; bb += kOrderThreads) {
            const int s0 = bb > 0 ? cnt[bb - 1] : 0, s1 = cnt[bb];
            for (int i = s0 + 1; i < s1; ++i) {
                const int t = list[i];
                const uint32_t kt = code[t];
                int j = i - 1;
                while (j >= s0) {
                    const int u = list[j];
                    const uint32_t ku = code[u];
                    if (ku < kt || (ku == kt && u < t)) break;
                    list[j + 1] = u;
                    --j;
                }
                list[j + 1] = t;
            }
        }
        __syncthreads();
        for (int i = tid; i < N; i += kOrderThreads) out[i] = list[i];
        return;
    }
    // fallback: bitonic sort of P packed keys (code << 32 | id; padding sorts last)
    uint64_t* keys = reinterpret_cast<uint64_t*>(smem + L.u);
    for (int i = tid; i < P; i += kOrderThreads)
        keys[i] = i < N ? ((static_cast<uint64_t>(code[i]) << 32) | static_cast<uint32_t>(i)) : ~0ull;
    __syncthreads();
    for (int k = 2; k <= P; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = tid; i < P; i += kOrderThreads) {
                const int ixj = i ^ j;
                if (ixj > i) {
                    const uint64_t ka = keys[i], kb = keys[ixj];
                    const bool up = (i & k) == 0;
                    if ((ka > kb) == up) {
                        keys[i] = kb;
                        keys[ixj] = ka;
                    }
                }
            }
            __syncthreads();
        }
    }
    for (int i = tid; i < N; i += kOrderThreads) out[i] = static_cast<int32_t>(keys[i] & 0xffffffffu);
}

}  // namespace

size_t token_order_smem_bytes(int N) { return order_smem_layout(N).total; }

cudaError_t launch_token_order(const float* xy, int B, int N, int GH, int GW, int32_t* perm,
                               cudaStream_t st) {
    const size_t smem = token_order_smem_bytes(N);
    cudaError_t e = ensure_smem<token_order_kernel>(smem);
    if (e != cudaSuccess) return e;
    int bits = 0;
    const int g = GH > GW ? GH : GW;
    while ((1 << bits) < g) ++bits;
    token_order_kernel<<<B, kOrderThreads, smem, st>>>(xy, N, GH, GW, 2 * bits, perm);
    note_launch();
    return cudaGetLastError();
}

}  // namespace acl
