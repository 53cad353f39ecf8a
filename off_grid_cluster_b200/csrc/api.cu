// api.cu -- the exported C ABI (include/acl.h): argument validation, workspace
// sizing and dispatch to the kernel launchers.  No call allocates, synchronises or
// keeps state; every check runs on the host before the first launch.
#include <atomic>

#include "../../include/acl.h"
#include "internal.h"

namespace acl {

static std::atomic<uint64_t> g_launches{0};
void note_launch(int n) { g_launches.fetch_add(static_cast<uint64_t>(n), std::memory_order_relaxed); }

}  // namespace acl

namespace {

constexpr size_t kMaxSmem = 227 * 1024;
constexpr int kMaxAttnN = 262144;

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

acl_status cuda_status(cudaError_t e) { return e == cudaSuccess ? ACL_OK : ACL_ERR_CUDA; }

cudaStream_t S(acl_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

const acl::bf16* BF(const acl_bf16* p) { return reinterpret_cast<const acl::bf16*>(p); }
acl::bf16* BFm(acl_bf16* p) { return reinterpret_cast<acl::bf16*>(p); }

acl_status check_attn(const acl_bf16* Q, const acl_bf16* K, const acl_bf16* V, const float* coords,
                      const int32_t* clusters, const int32_t* nbr, const float* bias, int B, int N,
                      int H, int D, int C, int M) {
    if (!Q || !K || !V || !coords || !clusters || !nbr || !bias) return ACL_ERR_INVALID_ARG;
    if (B < 1 || N < 1 || H < 1 || D < 1 || C < 1 || M < 1) return ACL_ERR_INVALID_ARG;
    if (M % C != 0) return ACL_ERR_INVALID_ARG;
    if (D != ACL_ATTN_D || C != ACL_ATTN_C || M > ACL_ATTN_MAX_M || H > 1024 || N > kMaxAttnN ||
        B > 65535)
        return ACL_ERR_UNSUPPORTED;
    if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(coords, 8))
        return ACL_ERR_INVALID_ARG;
    return ACL_OK;
}

acl_status check_gather(const float* queries, int B, int Q, const acl_bf16* feats,
                        const float* coords, int N, int d, const int32_t* table, int H, int W,
                        int K, const float* p) {
    if ((Q > 0 && !queries) || !feats || !coords || !table || !p) return ACL_ERR_INVALID_ARG;
    if (B < 1 || Q < 0 || N < 1 || d < 1 || H < 1 || W < 1 || K < 1) return ACL_ERR_INVALID_ARG;
    if (d % 32 != 0) return ACL_ERR_INVALID_ARG;
    if (d > ACL_MAX_GATHER_D || K > ACL_MAX_KNN_K) return ACL_ERR_UNSUPPORTED;
    if (static_cast<long long>(H) * W * K > 0x7fffffffLL) return ACL_ERR_UNSUPPORTED;
    if (!aligned(feats, 16) || !aligned(queries, 8) || !aligned(coords, 8)) return ACL_ERR_INVALID_ARG;
    return ACL_OK;
}

void map_knn_workspace(acl::KnnArgs& a, uint8_t* ws, const acl::KnnWorkspace& L) {
    a.w = reinterpret_cast<float*>(ws + L.w);
    a.keys = reinterpret_cast<int32_t*>(ws + L.keys);
    a.csr = reinterpret_cast<int32_t*>(ws + L.csr);
    a.csr_off = reinterpret_cast<int32_t*>(ws + L.csr_off);
    a.dp_part = reinterpret_cast<float*>(ws + L.dp_part);
    a.chunk_tok = reinterpret_cast<int32_t*>(ws + L.chunk_tok);
    a.chunk_off = reinterpret_cast<int32_t*>(ws + L.chunk_off);
    a.heavy = reinterpret_cast<int32_t*>(ws + L.heavy);
    a.heavy_count = reinterpret_cast<int32_t*>(ws + L.heavy_count);
    a.heavy_cap = L.heavy_cap;
}

// Validation and argument set-up shared by the two backward entry points.
acl_status setup_gather_bwd(const float* queries, int B, int Q, const acl_bf16* feats,
                            const float* coords, int N, int d, const int32_t* table, int H, int W,
                            int K, const float* p, acl_knn_kernel kind, const acl_bf16* dOut,
                            acl_bf16* dfeats, float* dqueries, float* dp, void* workspace,
                            size_t ws_bytes, acl::KnnArgs& a) {
    acl_status st = check_gather(queries, B, Q, feats, coords, N, d, table, H, W, K, p);
    if (st != ACL_OK) return st;
    if (kind != ACL_KNN_EXP && kind != ACL_KNN_INVPOW) return ACL_ERR_INVALID_ARG;
    if ((Q > 0 && (!dOut || !dqueries)) || !dfeats || !dp) return ACL_ERR_INVALID_ARG;
    if (!aligned(dOut, 16) || !aligned(dfeats, 16) || !aligned(dqueries, 8)) return ACL_ERR_INVALID_ARG;
    if (Q > ACL_MAX_GATHER_Q || N > ACL_MAX_TABLE_N) return ACL_ERR_UNSUPPORTED;
    const acl::KnnWorkspace L = acl::knn_workspace_layout(B, Q, N, d, K);
    if (!workspace || !aligned(workspace, 256) || ws_bytes < L.total) return ACL_ERR_WORKSPACE;
    a.queries = queries; a.feats = BF(feats); a.xy = coords; a.table = table; a.p = p;
    a.B = B; a.Q = Q; a.N = N; a.d = d; a.GH = H; a.GW = W; a.K = K;
    a.dout = BF(dOut); a.dfeats = BFm(dfeats); a.dq = dqueries; a.dp = dp;
    a.kind = static_cast<int>(kind);
    map_knn_workspace(a, static_cast<uint8_t*>(workspace), L);
    return ACL_OK;
}

// Validation shared by the decoder-layer entry points (positions = ref or q).
acl_status check_decoder(const float* positions, const float* f_in, int B, int Q, int D,
                         const float* w_off, const acl_bf16* w_o, const acl_bf16* feats,
                         const float* coords, int N, int d, const int32_t* table, int H, int W,
                         int K, const float* p) {
    acl_status st = check_gather(positions, B, Q, feats, coords, N, d, table, H, W, K, p);
    if (st != ACL_OK) return st;
    if ((Q > 0 && !f_in) || !w_off || !w_o) return ACL_ERR_INVALID_ARG;
    if (D < 128 || D % 128 != 0 || d % 128 != 0) return ACL_ERR_INVALID_ARG;
    if (D > 1024 || Q > ACL_MAX_GATHER_Q || N > ACL_MAX_TABLE_N) return ACL_ERR_UNSUPPORTED;
    if (static_cast<long long>(B) * Q > (1LL << 24)) return ACL_ERR_UNSUPPORTED;
    if (!aligned(f_in, 16) || !aligned(w_off, 16) || !aligned(w_o, 16)) return ACL_ERR_INVALID_ARG;
    return ACL_OK;
}

void map_decoder_stage(acl::DecArgs& a, const float* f_in, int B, int Q, int D, const float* w_off,
                       const acl_bf16* w_o, const acl_bf16* feats, const float* coords, int N, int d,
                       const int32_t* table, int H, int W, int K, const float* p) {
    a.f_in = f_in; a.B = B; a.Q = Q; a.D = D; a.d = d; a.w_off = w_off; a.w_o = BF(w_o);
    acl::KnnArgs& k = a.knn;
    k.feats = BF(feats); k.xy = coords; k.table = table; k.p = p;
    k.B = B; k.Q = Q; k.N = N; k.d = d; k.GH = H; k.GW = W; k.K = K; k.kind = 0;
}

}  // namespace

extern "C" {

const char* acl_status_string(acl_status s) {
    switch (s) {
        case ACL_OK: return "ACL_OK";
        case ACL_ERR_INVALID_ARG: return "ACL_ERR_INVALID_ARG: null pointer, misaligned pointer or size out of range";
        case ACL_ERR_CUDA: return "ACL_ERR_CUDA: a CUDA call or kernel launch failed";
        case ACL_ERR_UNSUPPORTED: return "ACL_ERR_UNSUPPORTED: sizes outside the implemented limits";
        case ACL_ERR_WORKSPACE: return "ACL_ERR_WORKSPACE: workspace missing, misaligned or too small";
        case ACL_ERR_DEVICE_CHECK: return "ACL_ERR_DEVICE_CHECK: device-side consistency check failed";
        case ACL_ERR_TIMEOUT: return "ACL_ERR_TIMEOUT: a bounded device wait gave up";
    }
    return "unknown acl_status";
}

int acl_version(void) { return 10000; }

uint64_t acl_launch_count(void) { return acl::g_launches.load(std::memory_order_relaxed); }

acl_status acl_cluster(const float* coords, int B, int N, int C, int32_t* clusters,
                       acl_stream_t stream) {
    if (!coords || !clusters) return ACL_ERR_INVALID_ARG;
    if (B < 1 || N < 1 || C < 1) return ACL_ERR_INVALID_ARG;
    if (N > ACL_MAX_CLUSTER_N || C > ACL_MAX_CLUSTER_C) return ACL_ERR_UNSUPPORTED;
    if (acl::cluster_smem_bytes(N, C) > kMaxSmem) return ACL_ERR_UNSUPPORTED;
    if (!aligned(coords, 8)) return ACL_ERR_INVALID_ARG;
    return cuda_status(acl::launch_cluster(coords, B, N, C, clusters, S(stream)));
}

acl_status acl_neighbors(const float* coords, const int32_t* clusters, int B, int N, int C, int M,
                         int32_t* nbr, acl_stream_t stream) {
    if (!coords || !clusters || !nbr) return ACL_ERR_INVALID_ARG;
    if (B < 1 || N < 1 || C < 1 || M < 1 || M % C != 0) return ACL_ERR_INVALID_ARG;
    if (C > ACL_MAX_CLUSTER_C || M / C > ACL_MAX_NEIGHBOR_R || B > 65535) return ACL_ERR_UNSUPPORTED;
    const int G = (N + C - 1) / C;
    if (acl::neighbors_smem_bytes(G) > kMaxSmem) return ACL_ERR_UNSUPPORTED;
    return cuda_status(acl::launch_neighbors(coords, clusters, B, N, C, M, nbr, S(stream)));
}

size_t acl_cluster_attn_workspace(int B, int N, int H, int C, int M) {
    if (B < 1 || N < 1 || H < 1 || C < 1 || M < C || M % C != 0) return 0;
    return acl::attn_workspace_layout(B, N, H, C, M).total;
}

acl_status acl_cluster_attn_fwd(const acl_bf16* Q, const acl_bf16* K, const acl_bf16* V,
                                const float* coords, const int32_t* clusters, const int32_t* nbr,
                                const float* bias_coef, int B, int N, int H, int D, int C, int M,
                                float scale, acl_bf16* O, float* lse, acl_stream_t stream) {
    acl_status st = check_attn(Q, K, V, coords, clusters, nbr, bias_coef, B, N, H, D, C, M);
    if (st != ACL_OK) return st;
    if (!O || !lse) return ACL_ERR_INVALID_ARG;
    if (!aligned(O, 16)) return ACL_ERR_INVALID_ARG;
    acl::AttnArgs a = {};
    a.q = BF(Q); a.k = BF(K); a.v = BF(V);
    a.xy = coords; a.clusters = clusters; a.nbr = nbr; a.bias = bias_coef;
    a.B = B; a.N = N; a.H = H; a.G = (N + C - 1) / C; a.M = M; a.R = M / C;
    a.scale = scale;
    a.o = BFm(O); a.lse = lse;
    return cuda_status(acl::launch_attn_fwd(a, S(stream)));
}

acl_status acl_cluster_attn_fwd_ffma(const acl_bf16* Q, const acl_bf16* K, const acl_bf16* V,
                                     const float* coords, const int32_t* clusters, const int32_t* nbr,
                                     const float* bias_coef, int B, int N, int H, int D, int C, int M,
                                     float scale, acl_bf16* O, float* lse, acl_stream_t stream) {
    acl_status st = check_attn(Q, K, V, coords, clusters, nbr, bias_coef, B, N, H, D, C, M);
    if (st != ACL_OK) return st;
    if (!O || !lse) return ACL_ERR_INVALID_ARG;
    if (!aligned(O, 16)) return ACL_ERR_INVALID_ARG;
    acl::AttnArgs a = {};
    a.q = BF(Q); a.k = BF(K); a.v = BF(V);
    a.xy = coords; a.clusters = clusters; a.nbr = nbr; a.bias = bias_coef;
    a.B = B; a.N = N; a.H = H; a.G = (N + C - 1) / C; a.M = M; a.R = M / C;
    a.scale = scale;
    a.o = BFm(O); a.lse = lse;
    return cuda_status(acl::launch_attn_fwd_ffma(a, S(stream)));
}

acl_status acl_cluster_attn_bwd(const acl_bf16* Q, const acl_bf16* K, const acl_bf16* V,
                                const float* coords, const int32_t* clusters, const int32_t* nbr,
                                const float* bias_coef, int B, int N, int H, int D, int C, int M,
                                float scale, const acl_bf16* O, const acl_bf16* dO,
                                const float* lse, acl_bf16* dQ, acl_bf16* dK, acl_bf16* dV,
                                float* dbias_coef, void* workspace, size_t ws_bytes,
                                acl_stream_t stream) {
    acl_status st = check_attn(Q, K, V, coords, clusters, nbr, bias_coef, B, N, H, D, C, M);
    if (st != ACL_OK) return st;
    if (!dO || !lse || !dQ || !dK || !dV || !dbias_coef) return ACL_ERR_INVALID_ARG;
    if (!aligned(dO, 16) || !aligned(dQ, 16) || !aligned(dK, 16) || !aligned(dV, 16))
        return ACL_ERR_INVALID_ARG;
    const acl::AttnWorkspace L = acl::attn_workspace_layout(B, N, H, C, M);
    if (!workspace || !aligned(workspace, 256) || ws_bytes < L.total) return ACL_ERR_WORKSPACE;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    acl::AttnArgs a = {};
    a.q = BF(Q); a.k = BF(K); a.v = BF(V);
    a.xy = coords; a.clusters = clusters; a.nbr = nbr; a.bias = bias_coef;
    a.B = B; a.N = N; a.H = H; a.G = (N + C - 1) / C; a.M = M; a.R = M / C;
    a.scale = scale;
    (void)O;  // not read: Delta comes from the recomputed tile
    a.dout = BF(dO); a.lse_in = lse;
    a.dq = BFm(dQ); a.dk = BFm(dK); a.dv = BFm(dV); a.dbias = dbias_coef;
    a.delta = reinterpret_cast<float*>(ws + L.delta);
    a.dbias_part = reinterpret_cast<float*>(ws + L.dbias_part);
    a.tok_cluster = reinterpret_cast<int32_t*>(ws + L.tok_cluster);
    a.rev_off = reinterpret_cast<int32_t*>(ws + L.rev_off);
    a.rev_list = reinterpret_cast<int32_t*>(ws + L.rev_list);
    a.rev_tok = reinterpret_cast<int32_t*>(ws + L.rev_tok);
    a.kplan = reinterpret_cast<long long*>(ws + L.kplan);
    return cuda_status(acl::launch_attn_bwd(a, S(stream)));
}

acl_status acl_knn_table(const float* coords, int B, int N, int H, int W, int K, int32_t* table,
                         acl_stream_t stream) {
    if (!coords || !table) return ACL_ERR_INVALID_ARG;
    if (B < 1 || N < 1 || H < 1 || W < 1 || K < 1) return ACL_ERR_INVALID_ARG;
    if (N > ACL_MAX_TABLE_N || K > ACL_MAX_KNN_K || H > 4096 || W > 4096 || B > 65535)
        return ACL_ERR_UNSUPPORTED;
    if (!aligned(coords, 8)) return ACL_ERR_INVALID_ARG;
    return cuda_status(acl::launch_knn_table(coords, B, N, H, W, K, table, S(stream)));
}

acl_status acl_token_order(const float* coords, int B, int N, int H, int W, int32_t* perm,
                           acl_stream_t stream) {
    if (!coords || !perm) return ACL_ERR_INVALID_ARG;
    if (B < 1 || N < 1 || H < 1 || W < 1) return ACL_ERR_INVALID_ARG;
    if (N > ACL_MAX_TABLE_N || H > 4096 || W > 4096 || B > 65535) return ACL_ERR_UNSUPPORTED;
    if (acl::token_order_smem_bytes(N) > kMaxSmem) return ACL_ERR_UNSUPPORTED;
    if (!aligned(coords, 8)) return ACL_ERR_INVALID_ARG;
    return cuda_status(acl::launch_token_order(coords, B, N, H, W, perm, S(stream)));
}

size_t acl_token_merge_workspace(int B, int N, int d, int h, int k) {
    if (B < 1 || N < 1 || d < 32 || d % 32 != 0 || h < 1 || k < 1 || k > N) return 0;
    return acl::merge_workspace_layout(B, N, d, h, k).total;
}

}  // extern "C"

namespace {

acl_status check_merge(const acl_bf16* feats, const float* coords, int B, int N, int d,
                       const float* w1, const float* b1, const float* w2, int h, int k,
                       void* workspace, size_t ws_bytes) {
    if (!feats || !coords || !w1 || !b1 || !w2) return ACL_ERR_INVALID_ARG;
    if (B < 1 || N < 1 || d < 32 || d % 32 != 0 || h < 1 || k < 1 || k > N) return ACL_ERR_INVALID_ARG;
    if (N > ACL_MAX_TABLE_N || d > ACL_MAX_GATHER_D || h > 256 || B > 65535) return ACL_ERR_UNSUPPORTED;
    if (acl::merge_smem_bytes(N, k, d, h) > kMaxSmem) return ACL_ERR_UNSUPPORTED;
    if (!aligned(feats, 16) || !aligned(coords, 8)) return ACL_ERR_INVALID_ARG;
    const acl::MergeWorkspace L = acl::merge_workspace_layout(B, N, d, h, k);
    if (!workspace || !aligned(workspace, 256) || ws_bytes < L.total) return ACL_ERR_WORKSPACE;
    return ACL_OK;
}

void map_merge(acl::MergeArgs& m, const acl_bf16* feats, const float* coords, int B, int N, int d,
               const float* w1, const float* b1, const float* w2, float b2, int h, int k,
               void* workspace) {
    const acl::MergeWorkspace L = acl::merge_workspace_layout(B, N, d, h, k);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    m.feats = BF(feats); m.xy = coords; m.B = B; m.N = N; m.d = d; m.h = h; m.k = k;
    m.w1 = w1; m.b1 = b1; m.w2 = w2; m.b2 = b2;
    m.flag = reinterpret_cast<int32_t*>(ws + L.flag);
    m.members = reinterpret_cast<int32_t*>(ws + L.members);
    m.goff = reinterpret_cast<int32_t*>(ws + L.goff);
    m.gstat = reinterpret_cast<float*>(ws + L.gstat);
    m.g = reinterpret_cast<float*>(ws + L.g);
    m.ds = reinterpret_cast<float*>(ws + L.ds);
    m.dh = reinterpret_cast<float*>(ws + L.dh);
    m.e = reinterpret_cast<float*>(ws + L.e);
    m.part = reinterpret_cast<float*>(ws + L.part);
}

}  // namespace

extern "C" {

acl_status acl_token_merge_fwd(const acl_bf16* feats, const float* coords, int B, int N, int d,
                               const float* w1, const float* b1, const float* w2, float b2, int h,
                               int k, float* scores, int32_t* anchors, int32_t* assign,
                               acl_bf16* merged, float* mcoords, void* workspace, size_t ws_bytes,
                               acl_stream_t stream) {
    acl_status st = check_merge(feats, coords, B, N, d, w1, b1, w2, h, k, workspace, ws_bytes);
    if (st != ACL_OK) return st;
    if (!scores || !anchors || !assign || !merged || !mcoords) return ACL_ERR_INVALID_ARG;
    if (!aligned(merged, 16) || !aligned(mcoords, 8)) return ACL_ERR_INVALID_ARG;
    acl::MergeArgs m = {};
    map_merge(m, feats, coords, B, N, d, w1, b1, w2, b2, h, k, workspace);
    m.scores = scores; m.anchors = anchors; m.assign = assign; m.merged = BFm(merged); m.mxy = mcoords;
    return cuda_status(acl::launch_merge_fwd(m, S(stream)));
}

acl_status acl_token_merge_bwd(const acl_bf16* feats, const float* coords, int B, int N, int d,
                               const float* w1, const float* b1, const float* w2, float b2, int h,
                               int k, const float* scores, const int32_t* assign,
                               const acl_bf16* dmerged, const float* dmcoords, acl_bf16* dfeats,
                               float* dcoords, float* dw1, float* db1, float* dw2, float* db2,
                               void* workspace, size_t ws_bytes, acl_stream_t stream) {
    acl_status st = check_merge(feats, coords, B, N, d, w1, b1, w2, h, k, workspace, ws_bytes);
    if (st != ACL_OK) return st;
    if (!scores || !assign || !dmerged || !dmcoords || !dfeats || !dcoords || !dw1 || !db1 || !dw2 ||
        !db2)
        return ACL_ERR_INVALID_ARG;
    if (!aligned(dmerged, 16) || !aligned(dfeats, 16) || !aligned(dcoords, 8) || !aligned(dmcoords, 8))
        return ACL_ERR_INVALID_ARG;
    acl::MergeArgs m = {};
    map_merge(m, feats, coords, B, N, d, w1, b1, w2, b2, h, k, workspace);
    m.scores = const_cast<float*>(scores); m.assign = const_cast<int32_t*>(assign);
    m.dmerged = BF(dmerged); m.dmxy = dmcoords; m.dfeats = BFm(dfeats); m.dxy = dcoords;
    m.dw1 = dw1; m.db1 = db1; m.dw2 = dw2; m.db2 = db2;
    return cuda_status(acl::launch_merge_bwd(m, S(stream)));
}

size_t acl_knn_gather_workspace(int B, int Q, int N, int d, int K) {
    if (B < 1 || Q < 0 || N < 1 || d < 32 || d % 32 != 0 || K < 1) return 0;
    return acl::knn_workspace_layout(B, Q, N, d, K).total;
}

acl_status acl_knn_gather_fwd_ex(const float* queries, int B, int Q, const acl_bf16* feats,
                                 const float* coords, int N, int d, const int32_t* table, int H,
                                 int W, int K, const float* p, acl_knn_kernel kind, acl_bf16* out,
                                 acl_stream_t stream) {
    acl_status st = check_gather(queries, B, Q, feats, coords, N, d, table, H, W, K, p);
    if (st != ACL_OK) return st;
    if (kind != ACL_KNN_EXP && kind != ACL_KNN_INVPOW) return ACL_ERR_INVALID_ARG;
    if ((Q > 0 && !out) || !aligned(out, 16)) return ACL_ERR_INVALID_ARG;
    acl::KnnArgs a = {};
    a.queries = queries; a.feats = BF(feats); a.xy = coords; a.table = table; a.p = p;
    a.B = B; a.Q = Q; a.N = N; a.d = d; a.GH = H; a.GW = W; a.K = K;
    a.kind = static_cast<int>(kind);
    a.out = BFm(out);
    return cuda_status(acl::launch_knn_fwd(a, S(stream)));
}

acl_status acl_knn_gather_fwd(const float* queries, int B, int Q, const acl_bf16* feats,
                              const float* coords, int N, int d, const int32_t* table, int H, int W,
                              int K, const float* p, acl_bf16* out, acl_stream_t stream) {
    return acl_knn_gather_fwd_ex(queries, B, Q, feats, coords, N, d, table, H, W, K, p, ACL_KNN_EXP,
                                 out, stream);
}

acl_status acl_knn_gather_index(const float* queries, int B, int Q, int N, int d,
                                const int32_t* table, int H, int W, int K, void* workspace,
                                size_t ws_bytes, acl_stream_t stream) {
    if ((Q > 0 && !queries) || !table) return ACL_ERR_INVALID_ARG;
    if (B < 1 || Q < 0 || N < 1 || d < 32 || d % 32 != 0 || H < 1 || W < 1 || K < 1)
        return ACL_ERR_INVALID_ARG;
    if (d > ACL_MAX_GATHER_D || K > ACL_MAX_KNN_K || Q > ACL_MAX_GATHER_Q || N > ACL_MAX_TABLE_N)
        return ACL_ERR_UNSUPPORTED;
    if (static_cast<long long>(H) * W * K > 0x7fffffffLL) return ACL_ERR_UNSUPPORTED;
    if (!aligned(queries, 8)) return ACL_ERR_INVALID_ARG;
    const acl::KnnWorkspace L = acl::knn_workspace_layout(B, Q, N, d, K);
    if (!workspace || !aligned(workspace, 256) || ws_bytes < L.total) return ACL_ERR_WORKSPACE;
    acl::KnnArgs a = {};
    a.queries = queries; a.table = table;
    a.B = B; a.Q = Q; a.N = N; a.d = d; a.GH = H; a.GW = W; a.K = K;
    map_knn_workspace(a, static_cast<uint8_t*>(workspace), L);
    return cuda_status(acl::launch_knn_index(a, S(stream)));
}

acl_status acl_knn_gather_bwd_indexed_ex(const float* queries, int B, int Q,
                                         const acl_bf16* feats, const float* coords, int N, int d,
                                         const int32_t* table, int H, int W, int K, const float* p,
                                         acl_knn_kernel kind, const acl_bf16* dOut,
                                         acl_bf16* dfeats, float* dqueries, float* dp,
                                         void* workspace, size_t ws_bytes, acl_stream_t stream) {
    acl::KnnArgs a = {};
    const acl_status st = setup_gather_bwd(queries, B, Q, feats, coords, N, d, table, H, W, K, p,
                                           kind, dOut, dfeats, dqueries, dp, workspace, ws_bytes, a);
    if (st != ACL_OK) return st;
    return cuda_status(acl::launch_knn_bwd_indexed(a, S(stream)));
}

acl_status acl_knn_gather_bwd_indexed(const float* queries, int B, int Q, const acl_bf16* feats,
                                      const float* coords, int N, int d, const int32_t* table,
                                      int H, int W, int K, const float* p, const acl_bf16* dOut,
                                      acl_bf16* dfeats, float* dqueries, float* dp,
                                      void* workspace, size_t ws_bytes, acl_stream_t stream) {
    return acl_knn_gather_bwd_indexed_ex(queries, B, Q, feats, coords, N, d, table, H, W, K, p,
                                         ACL_KNN_EXP, dOut, dfeats, dqueries, dp, workspace,
                                         ws_bytes, stream);
}

acl_status acl_knn_gather_bwd_ex(const float* queries, int B, int Q, const acl_bf16* feats,
                                 const float* coords, int N, int d, const int32_t* table, int H,
                                 int W, int K, const float* p, acl_knn_kernel kind,
                                 const acl_bf16* dOut, acl_bf16* dfeats, float* dqueries, float* dp,
                                 void* workspace, size_t ws_bytes, acl_stream_t stream) {
    acl::KnnArgs a = {};
    const acl_status st = setup_gather_bwd(queries, B, Q, feats, coords, N, d, table, H, W, K, p,
                                           kind, dOut, dfeats, dqueries, dp, workspace, ws_bytes, a);
    if (st != ACL_OK) return st;
    return cuda_status(acl::launch_knn_bwd(a, S(stream)));
}

acl_status acl_knn_gather_bwd(const float* queries, int B, int Q, const acl_bf16* feats,
                              const float* coords, int N, int d, const int32_t* table, int H, int W,
                              int K, const float* p, const acl_bf16* dOut, acl_bf16* dfeats,
                              float* dqueries, float* dp, void* workspace, size_t ws_bytes,
                              acl_stream_t stream) {
    return acl_knn_gather_bwd_ex(queries, B, Q, feats, coords, N, d, table, H, W, K, p, ACL_KNN_EXP,
                                 dOut, dfeats, dqueries, dp, workspace, ws_bytes, stream);
}

acl_status acl_device_check(void) {
    if (cudaDeviceSynchronize() != cudaSuccess) return ACL_ERR_CUDA;
    unsigned int n = 0, fa = 0, fk = 0, fc = 0;
    if (acl::read_tc_timeouts(&n) != cudaSuccess || acl::read_checks_attn(&fa) != cudaSuccess ||
        acl::read_checks_knn(&fk) != cudaSuccess || acl::read_checks_cluster(&fc) != cudaSuccess)
        return ACL_ERR_CUDA;
    if (fa | fk | fc) return ACL_ERR_DEVICE_CHECK;
    return n ? ACL_ERR_TIMEOUT : ACL_OK;
}

int acl_device_checks_enabled(void) {
#ifdef ACL_DEVICE_CHECKS
    return 1;
#else
    return 0;
#endif
}

acl_status acl_test_set_wait_limit(long long cycles) {
    return acl::set_tc_wait_cycles(cycles < 0 ? 1000000000LL : cycles) == cudaSuccess ? ACL_OK : ACL_ERR_CUDA;
}

size_t acl_decoder_layer_workspace(int B, int Q, int N, int d, int D, int K) {
    if (B < 1 || Q < 0 || N < 1 || d < 128 || d % 128 != 0 || D < 128 || D % 128 != 0 || K < 1)
        return 0;
    return acl::dec_workspace_layout(B, Q, N, d, D, K).total;
}

acl_status acl_decoder_layer_fwd(const float* ref, const float* f_in, int B, int Q, int D,
                                 const float* w_off, const float* b_off, const acl_bf16* w_o,
                                 const acl_bf16* feats, const float* coords, int N, int d,
                                 const int32_t* table, int H, int W, int K, const float* p,
                                 float* q, acl_bf16* v, float* f_out, acl_stream_t stream) {
    acl_status st = check_decoder(ref, f_in, B, Q, D, w_off, w_o, feats, coords, N, d, table, H,
                                  W, K, p);
    if (st != ACL_OK) return st;
    if (!b_off || (Q > 0 && (!q || !v || !f_out))) return ACL_ERR_INVALID_ARG;
    if (!aligned(q, 8) || !aligned(v, 16) || !aligned(f_out, 16)) return ACL_ERR_INVALID_ARG;
    acl::DecArgs a = {};
    map_decoder_stage(a, f_in, B, Q, D, w_off, w_o, feats, coords, N, d, table, H, W, K, p);
    a.ref = ref; a.b_off = b_off; a.q = q; a.v = BFm(v); a.f_out = f_out;
    return cuda_status(acl::launch_dec_fwd(a, S(stream)));
}

acl_status acl_decoder_layer_bwd(const float* f_in, int B, int Q, int D, const float* w_off,
                                 const acl_bf16* w_o, const acl_bf16* feats, const float* coords,
                                 int N, int d, const int32_t* table, int H, int W, int K,
                                 const float* p, const float* q, const acl_bf16* v,
                                 const float* df_out, float* df_in, float* dw_off, float* db_off,
                                 float* dw_o, acl_bf16* dfeats, float* dp, void* workspace,
                                 size_t ws_bytes, acl_stream_t stream) {
    acl_status st = check_decoder(q, f_in, B, Q, D, w_off, w_o, feats, coords, N, d, table, H, W,
                                  K, p);
    if (st != ACL_OK) return st;
    if ((Q > 0 && (!v || !df_out || !df_in)) || !dw_off || !db_off || !dw_o || !dfeats || !dp)
        return ACL_ERR_INVALID_ARG;
    if (!aligned(v, 16) || !aligned(df_out, 16) || !aligned(df_in, 16) || !aligned(dfeats, 16) ||
        !aligned(dw_off, 8))
        return ACL_ERR_INVALID_ARG;
    const acl::DecWorkspace L = acl::dec_workspace_layout(B, Q, N, d, D, K);
    if (!workspace || !aligned(workspace, 256) || ws_bytes < L.total) return ACL_ERR_WORKSPACE;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    acl::DecArgs a = {};
    map_decoder_stage(a, f_in, B, Q, D, w_off, w_o, feats, coords, N, d, table, H, W, K, p);
    a.q = const_cast<float*>(q); a.v = const_cast<acl::bf16*>(BF(v)); a.df_out = df_out;
    a.df_in = df_in; a.dw_off = dw_off; a.db_off = db_off; a.dw_o = dw_o;
    a.dfb = reinterpret_cast<acl::bf16*>(ws + L.dfb);
    a.dv = reinterpret_cast<acl::bf16*>(ws + L.dv);
    a.dq = reinterpret_cast<float*>(ws + L.dq);
    a.wo_part = reinterpret_cast<float*>(ws + L.wo_part);
    a.off_part = reinterpret_cast<float*>(ws + L.off_part);
    a.knn.dfeats = BFm(dfeats); a.knn.dp = dp;
    map_knn_workspace(a.knn, ws + L.knn, acl::knn_workspace_layout(B, Q, N, d, K));
    return cuda_status(acl::launch_dec_bwd(a, S(stream)));
}

}  // extern "C"
