// internal.h -- launchers behind the C ABI (not exported).  Each returns the first
// CUDA error of its launches (cudaSuccess otherwise); argument checks live in api.cu.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>

#include "common.cuh"

namespace acl {

// counts every kernel launch issued by the library (see acl_launch_count)
void note_launch(int n = 1);

// Raise the dynamic shared-memory limit of kernel `Kern` on the current device to at
// least `bytes`, calling cudaFuncSetAttribute only the first time a larger value is
// needed on that device (so repeated calls, including calls made while a stream is
// being captured into a CUDA graph, do no driver work).
template <auto Kern>
cudaError_t ensure_smem(size_t bytes) {
    if (bytes <= 48 * 1024) return cudaSuccess;
    static std::atomic<int> done[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const int want = static_cast<int>(bytes);
    if (dev < 64 && done[dev].load(std::memory_order_acquire) >= want) return cudaSuccess;
    e = cudaFuncSetAttribute(Kern, cudaFuncAttributeMaxDynamicSharedMemorySize, want);
    if (e == cudaSuccess && dev < 64) {
        int cur = done[dev].load(std::memory_order_relaxed);
        while (cur < want && !done[dev].compare_exchange_weak(cur, want)) {
        }
    }
    return e;
}

// Streaming multiprocessors of the current device (asked of the runtime once per device).
inline int sm_count() {
    static int cached[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (cached[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

// Resident CTAs per SM of kernel `Kern` launched with `threads` threads and `smem` bytes of
// dynamic shared memory (asked of the runtime once per kernel and device: a kernel must be
// launched with one shape).
template <auto Kern>
int resident(int threads, size_t smem) {
    static int cached[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
    if (cached[dev] == 0) {
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, Kern, threads, smem) != cudaSuccess || n < 1) n = 1;
        cached[dev] = n;
    }
    return cached[dev];
}

size_t cluster_smem_bytes(int N, int C);
cudaError_t launch_cluster(const float* xy, int B, int N, int C, int32_t* clusters,
                           cudaStream_t st);
size_t neighbors_smem_bytes(int G);
cudaError_t launch_neighbors(const float* xy, const int32_t* clusters, int B, int N, int C,
                             int M, int32_t* nbr, cudaStream_t st);

struct AttnArgs {
    const bf16* q;
    const bf16* k;
    const bf16* v;
    const float* xy;
    const int32_t* clusters;
    const int32_t* nbr;
    const float* bias;
    int B, N, H, G, M, R;
    float scale;
    // forward outputs
    bf16* o;
    float* lse;
    // backward
    const bf16* dout;
    const float* lse_in;
    bf16* dq;
    bf16* dk;
    bf16* dv;
    float* dbias;
    // backward workspace
    float* delta;        // [B][N][H]
    float* dbias_part;   // [B][G][H][3]
    int32_t* tok_cluster;  // [B][N]
    int32_t* rev_off;    // [B][G + 1]
    int32_t* rev_list;   // [B][G * R]
    int32_t* rev_tok;    // [B][G * R][8] query tokens of every reverse-list entry
    long long* kplan;    // [kwarps][2] key-pass unit range of every warp (see attn.cu)
    int kwarps;          // warps of the key pass the plan is made for (0: no plan)
};

struct AttnWorkspace {
    size_t delta, dbias_part, tok_cluster, rev_off, rev_list, rev_tok, kplan, total;
};
AttnWorkspace attn_workspace_layout(int B, int N, int H, int C, int M);

cudaError_t launch_attn_fwd(const AttnArgs& a, cudaStream_t st);
// the same forward on the FMA pipes only (attn_ffma.cu): the tensor-core kernel's reference
cudaError_t launch_attn_fwd_ffma(const AttnArgs& a, cudaStream_t st);
cudaError_t launch_attn_bwd(const AttnArgs& a, cudaStream_t st);

struct KnnArgs {
    const float* queries;
    const bf16* feats;
    const float* xy;
    const int32_t* table;
    const float* p;
    int B, Q, N, d, GH, GW, K;
    int kind;           // 0: exponential kernel softmax(-p d); 1: inverse power d^-p / sum
    bf16* out;
    // backward
    const bf16* dout;
    bf16* dfeats;
    float* dq;
    float* dp;
    float* w;           // [B][Q][K][d/32]
    int32_t* keys;      // [B][Q*K] token of every (query, slot) entry
    int32_t* csr;       // [B][Q*K]
    int32_t* csr_off;   // [B][N + 1]
    float* dp_part;     // [query blocks][d/32]
    int32_t* chunk_tok;  // [B][chunks + 1] first token of every light chunk of the token pass
    int32_t* chunk_off;  // [B][chunks + 1] first entry of that token
    int32_t* heavy;     // [B][slices][heavy_cap] tokens with many entries, per CSR slice
    int32_t* heavy_count;  // [B][slices]
    int heavy_cap;
};

struct KnnWorkspace {
    size_t w, keys, csr, csr_off, dp_part, chunk_tok, chunk_off, heavy, heavy_count, total;
    int query_blocks, heavy_cap;
};
KnnWorkspace knn_workspace_layout(int B, int Q, int N, int d, int K);

struct MergeArgs {
    const bf16* feats;
    const float* xy;
    int B, N, d, h, k;
    const float* w1;
    const float* b1;
    const float* w2;
    float b2;
    float* scores;       // [B][N] (written by the forward, read by the backward)
    int32_t* anchors;    // [B][k]
    int32_t* assign;     // [B][N]
    bf16* merged;        // [B][k][d]
    float* mxy;          // [B][k][2]
    // backward
    const bf16* dmerged;
    const float* dmxy;
    bf16* dfeats;
    float* dxy;
    float* dw1;
    float* db1;
    float* dw2;
    float* db2;
    // workspace
    int32_t* flag;       // [B][N] 1 for anchors
    int32_t* members;    // [B][N] tokens by (assignment, id)
    int32_t* goff;       // [B][k + 1]
    float* gstat;        // [B][k][4] max score, 1 / sum, sum_G w g
    float* g;            // [B][N] <dF, f> + <dX, x>
    float* ds;           // [B][N]
    float* dh;           // [B][N][h]
    float* e;            // [B][N][h] ds * gelu(z)
    float* part;         // parameter partial sums
};

struct MergeWorkspace {
    size_t flag, members, goff, gstat, g, ds, dh, e, part, total;
};
MergeWorkspace merge_workspace_layout(int B, int N, int d, int h, int k);
size_t merge_smem_bytes(int N, int k, int d, int h);
cudaError_t launch_merge_fwd(const MergeArgs& m, cudaStream_t st);
cudaError_t launch_merge_bwd(const MergeArgs& m, cudaStream_t st);

struct DecArgs {
    const float* ref;     // [B][Q][2] reference positions
    const float* f_in;    // [B][Q][D] query features
    int B, Q, D, d;
    const float* w_off;   // [D][2]
    const float* b_off;   // [2]
    const bf16* w_o;      // [d][D]
    float* q;             // [B][Q][2] sample positions (forward out, backward in)
    bf16* v;              // [B][Q][d] gathered features (forward out, backward in)
    float* f_out;         // [B][Q][D]
    // backward
    const float* df_out;
    float* df_in;
    float* dw_off;
    float* db_off;
    float* dw_o;          // [d][D]
    // backward workspace
    bf16* dfb;            // [B][Q][D] df_out in bf16
    bf16* dv;             // [B][Q][d]
    float* dq;            // [B][Q][2]
    float* wo_part;       // [splits][d][D]
    float* off_part;      // [parts][2 D + 2]
    KnnArgs knn;          // the stage: feats, coords, table, p, sizes; dfeats, dp, workspace
};

struct DecWorkspace {
    size_t dfb, dv, dq, wo_part, off_part, knn, total;
};
DecWorkspace dec_workspace_layout(int B, int Q, int N, int d, int D, int K);
int dec_wo_splits(int T, int d, int D);
// reads and clears the count of bounded tensor-core waits that gave up (synchronous)
cudaError_t read_tc_timeouts(unsigned int* count);
// sets the give-up limit of the tensor-core GEMM's main-loop waits (synchronous; tests)
cudaError_t set_tc_wait_cycles(long long cycles);
// read and clear the device-check flags of each kernel file (always 0 in the regular build)
cudaError_t read_checks_attn(unsigned int* flags);
cudaError_t read_checks_knn(unsigned int* flags);
cudaError_t read_checks_cluster(unsigned int* flags);
cudaError_t launch_dec_fwd(const DecArgs& a, cudaStream_t st);
cudaError_t launch_dec_bwd(const DecArgs& a, cudaStream_t st);

size_t knn_table_smem_bytes(int N, int nbins);
size_t token_order_smem_bytes(int N);
cudaError_t launch_token_order(const float* xy, int B, int N, int GH, int GW, int32_t* perm,
                               cudaStream_t st);
cudaError_t launch_knn_table(const float* xy, int B, int N, int GH, int GW, int K,
                             int32_t* table, cudaStream_t st);
cudaError_t launch_knn_fwd(const KnnArgs& a, cudaStream_t st);
cudaError_t launch_knn_index(const KnnArgs& a, cudaStream_t st);
cudaError_t launch_knn_bwd_indexed(const KnnArgs& a, cudaStream_t st);
cudaError_t launch_knn_bwd(const KnnArgs& a, cudaStream_t st);

}  // namespace acl
