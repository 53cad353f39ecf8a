/*
 * acl.h -- C ABI of the off-grid local cluster attention and KNN gather library
 * (libacl.so, CUDA, sm_100a).
 *
 * What it computes follows the AFFMAE pages:
 *   "AFFMAE: Scalable Vision Pre-Training for High-Resolution Microscopy
 *   Segmentation on Desktop Hardware" (en.papernotes.org notes), Method:
 *   "Overall Architecture" -- every token keeps an explicit 2D coordinate and
 *   attention runs through local balanced clustering (stages of Local Cluster
 *   Attention); "Key Designs" 2 -- the decoder gathers the K nearest tokens of a
 *   sample point with the exponential distance kernel w_i = softmax_i(-p d_i);
 *   "Key Designs" 3 -- an H x W x K table of each grid cell's K nearest tokens,
 *   the query quantised to its cell.  The arXiv abstract page ("AFFMAE: Scalable
 *   and Efficient Vision Pretraining for Desktop Graphics Cards") names the
 *   Flash-style mixed-precision cluster attention kernels.
 *
 * Conventions shared by every call
 *   - Coordinates are fp32 in grid-cell units: x = column, y = row; cell (r, c)
 *     covers [c, c+1) x [r, r+1), centre (c + 0.5, r + 0.5).  They must be finite.
 *   - Feature tensors are bf16 (raw 16-bit patterns, acl_bf16), row-major.
 *     Attention Q/K/V/O and their gradients: [B][N][H][D] with D = 32.
 *     Gather features: [B][N][d], channel c belongs to head c / 32.
 *   - Index tensors are int32; -1 marks an empty slot.
 *   - Every pointer is a DEVICE pointer owned by the caller, including outputs
 *     and workspaces.  bf16 tensors must be 16-byte aligned, coordinate and
 *     query tensors 8-byte aligned, workspaces 256-byte aligned.  The library
 *     allocates nothing and keeps no state between calls (beyond raising a
 *     kernel's shared-memory limit once per device); calls are asynchronous on
 *     `stream` (NULL = legacy default stream) and may be captured into a CUDA
 *     graph once each call has been made once on the device outside capture.
 *   - Outputs are overwritten in full (gradients included: nothing accumulates).
 *   - Images in a batch are independent problems.
 *   - Host-side validation runs before any launch; a failed call launches
 *     nothing and returns the status.  After launching, a launch error maps to
 *     ACL_ERR_CUDA.  Nothing aborts and nothing throws across the ABI.
 *   - Floating-point results are deterministic: no floating-point atomics, every
 *     reduction runs in a fixed order; repeated calls give identical bits.
 */
#ifndef ACL_H
#define ACL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    ACL_OK = 0,
    ACL_ERR_INVALID_ARG = 1,   /* null pointer, size out of range, inconsistent sizes  */
    ACL_ERR_CUDA = 2,          /* a CUDA call or kernel launch failed                  */
    ACL_ERR_UNSUPPORTED = 3,   /* valid arguments outside what the kernels implement   */
    ACL_ERR_WORKSPACE = 4,     /* workspace pointer null or smaller than required     */
    ACL_ERR_DEVICE_CHECK = 5,  /* check build: a device-side range check failed        */
    ACL_ERR_TIMEOUT = 6        /* a bounded device wait gave up (acl_device_check)     */
} acl_status;

/* Same type as cudaStream_t (both are pointers to struct CUstream_st). */
struct CUstream_st;
typedef struct CUstream_st* acl_stream_t;

/* Raw bf16 bit pattern (1 sign, 8 exponent, 7 mantissa bits). */
typedef uint16_t acl_bf16;

/* Implementation limits (ACL_ERR_UNSUPPORTED beyond them). */
#define ACL_MAX_CLUSTER_N 8192   /* tokens per image for acl_cluster                     */
#define ACL_MAX_CLUSTER_C 64     /* cluster size for acl_cluster / acl_neighbors         */
#define ACL_MAX_NEIGHBOR_R 16    /* M / C neighbour clusters                             */
#define ACL_ATTN_D 32            /* head dim of the attention kernels                    */
#define ACL_ATTN_C 8             /* cluster size of the attention kernels                */
#define ACL_ATTN_MAX_M 64        /* neighbourhood slots of the attention kernels          */
#define ACL_MAX_TABLE_N 16384    /* tokens per image for acl_knn_table                   */
#define ACL_MAX_KNN_K 16         /* neighbours per cell                                  */
#define ACL_MAX_GATHER_D 1024    /* channels of the gather                               */
#define ACL_MAX_GATHER_Q 65535   /* queries per image for acl_knn_gather_bwd             */

/* Human-readable name of a status code (static string, never NULL). */
const char* acl_status_string(acl_status s);

/* Library ABI version (major * 10000 + minor * 100 + patch). */
int acl_version(void);

/* Number of kernels this process has launched through the library (diagnostic;
 * counts host-side launches, so a captured CUDA graph's replays add nothing). */
uint64_t acl_launch_count(void);

/*
 * acl_cluster -- local balanced clustering (a1).
 * Passage: AFF notes, Method "Overall Architecture" (attention through local
 * balanced clustering of tokens with 2D coordinates).  The pages give no
 * algorithm; this is recursive median bisection:
 *   split(S, g): if g == 1 emit S ordered by token id, padded with -1 to C slots;
 *   else cut on the axis of larger fp64 extent (max - min; ties -> x), ordering S
 *   by (coordinate on that axis, other coordinate, token id); the first
 *   ceil(g/2) * C tokens form the left part with ceil(g/2) clusters; recurse left
 *   then right.  The root is split(all N tokens, G = ceil(N / C)).
 * coords   [B][N][2] fp32.
 * clusters [B][G][C] int32 out: token ids; only the last cluster of an image may
 *          hold -1 (when N % C != 0).  Every token appears exactly once.
 * Limits: 1 <= N <= ACL_MAX_CLUSTER_N, 1 <= C <= ACL_MAX_CLUSTER_C, B >= 1.
 * The result is bit-exact: comparisons only, and fp64 extents of fp32 values.
 */
acl_status acl_cluster(const float* coords, int B, int N, int C,
                       int32_t* clusters, acl_stream_t stream);

/*
 * acl_neighbors -- cluster-neighbourhood table (a2).
 * Passage: AFF notes, Method "Overall Architecture" (Local Cluster Attention);
 * the pages do not define the neighbourhood.  Reading: the R = M / C clusters of
 * nearest centroid, the cluster itself first.
 *   centroid_g = (sum of its valid tokens' x in slot order, from 0.0) / count,
 *   likewise y, fp64; dist2 = dx*dx + dy*dy (dx = cx_h - cx_g), each operation
 *   rounded separately (no fused multiply-add); the first min(R, G) clusters by
 *   (dist2, cluster id).
 * coords [B][N][2]; clusters [B][G][C] as written by acl_cluster.
 * nbr    [B][G][M] int32 out: nbr[g][r*C + s] = clusters[h_r][s]; slots beyond
 *        min(R, G) clusters hold -1.
 * Limits: M % C == 0, 1 <= M / C <= ACL_MAX_NEIGHBOR_R, C <= ACL_MAX_CLUSTER_C,
 *         ceil(N / C) <= 14528 (centroids held in shared memory), B <= 65535.  Bit-exact.
 */
acl_status acl_neighbors(const float* coords, const int32_t* clusters, int B, int N,
                         int C, int M, int32_t* nbr, acl_stream_t stream);

/* Workspace bytes acl_cluster_attn_bwd needs for these sizes (0 on bad sizes). */
size_t acl_cluster_attn_workspace(int B, int N, int H, int C, int M);

/*
 * acl_cluster_attn_fwd -- local cluster attention, forward (a3).
 * Passage: AFF notes, Method "Overall Architecture" and the flowchart (Local
 * Cluster Attention blocks); arXiv abstract page (Flash-style cluster attention).
 * For each valid token i of cluster g, head h, over the valid keys j of nbr[g]:
 *   dx = x_j - x_i, dy = y_j - y_i                         (key minus query)
 *   s_ij = scale * <q_i, k_j> + a_h dx + b_h dy - c_h (dx^2 + dy^2)
 *   O_i = sum_j softmax_j(s_ij) v_j,   lse_i = log sum_j exp(s_ij)   (natural log)
 * Q, K, V [B][N][H][D] bf16 (any token order: nbr holds token ids);
 * coords [B][N][2]; clusters [B][G][C]; nbr [B][G][M] (any token ids, -1 = empty);
 * bias_coef [H][3] fp32 = (a_h, b_h, c_h); scale e.g. 1/sqrt(32).
 * O [B][N][H][D] bf16 out (rounded to nearest even), lse [B][N][H] fp32 out.
 * Rows of tokens that no cluster lists are left untouched; a token whose
 * neighbourhood is empty gets O = 0 and lse = -inf.
 * Arithmetic: bf16 tensor-core products with fp32 accumulation, fp32 softmax.
 * Limits: D == 32, C == 8, M % 8 == 0, 8 <= M <= 64, 1 <= H <= 1024, B <= 65535,
 *         N <= 262144.
 */
acl_status acl_cluster_attn_fwd(const acl_bf16* Q, const acl_bf16* K, const acl_bf16* V,
                                const float* coords, const int32_t* clusters,
                                const int32_t* nbr, const float* bias_coef,
                                int B, int N, int H, int D, int C, int M, float scale,
                                acl_bf16* O, float* lse, acl_stream_t stream);
/*
 * acl_cluster_attn_fwd_ffma -- the same forward computed on the FMA pipes only (fp32 dot
 * products and sums, no tensor-core instruction): the reference variant the tensor-core
 * kernel of acl_cluster_attn_fwd is measured against (the pages' kernel choice, tensor cores
 * or FMA on the 8 x 48 tiles, rests on that comparison).  Arguments, layouts, limits, errors
 * and results as acl_cluster_attn_fwd (results equal up to fp32 rounding order).
 */
acl_status acl_cluster_attn_fwd_ffma(const acl_bf16* Q, const acl_bf16* K, const acl_bf16* V,
                                     const float* coords, const int32_t* clusters,
                                     const int32_t* nbr, const float* bias_coef,
                                     int B, int N, int H, int D, int C, int M, float scale,
                                     acl_bf16* O, float* lse, acl_stream_t stream);

/*
 * acl_cluster_attn_bwd -- local cluster attention, backward (a4), recomputing
 * P_ij = exp(s_ij - lse_i) from the forward's lse:
 *   dP_ij = <dO_i, v_j>, Delta_i = <dO_i, O_i>, dS_ij = P_ij (dP_ij - Delta_i),
 *   dQ_i = scale sum_j dS_ij k_j,  dK_j = scale sum_i dS_ij q_i,
 *   dV_j = sum_i P_ij dO_i,
 *   dbias_coef[h] = (sum dS dx, sum dS dy, -sum dS (dx^2 + dy^2)) over all images.
 * Arguments as in the forward, plus lse from it and dO [B][N][H][D] bf16.  O is
 * accepted for interface symmetry but not read (may be NULL): the whole key row of a
 * query lies in one tile, so Delta_i is formed as sum_j P_ij dP_ij in fp32, which
 * equals <dO_i, O_i> without the bf16 rounding of the stored O.
 * dQ, dK, dV [B][N][H][D] bf16 out; dbias_coef [H][3] fp32 out.
 * nbr must be the table acl_neighbors built from `clusters` (each group of C
 * slots is a whole cluster row): dK/dV are reduced per key cluster over the
 * query clusters that list it, in a fixed order, without atomics.
 * workspace: device memory of at least acl_cluster_attn_workspace(B, N, H, C, M)
 * bytes, 256-byte aligned; its contents on entry do not matter.
 */
acl_status acl_cluster_attn_bwd(const acl_bf16* Q, const acl_bf16* K, const acl_bf16* V,
                                const float* coords, const int32_t* clusters,
                                const int32_t* nbr, const float* bias_coef,
                                int B, int N, int H, int D, int C, int M, float scale,
                                const acl_bf16* O, const acl_bf16* dO, const float* lse,
                                acl_bf16* dQ, acl_bf16* dK, acl_bf16* dV,
                                float* dbias_coef, void* workspace, size_t ws_bytes,
                                acl_stream_t stream);

/* Size of the library-owned scratch array used by acl_cluster_attn_bwd_noalloc. */
#define ACL_NOALLOC_ATTN_WS_BYTES (4u << 20)

/*
 * acl_cluster_attn_bwd_noalloc -- acl_cluster_attn_bwd without a caller workspace.
 * The pages have no counterpart: this entry point exists for callers that cannot
 * allocate device memory (a host framework that forbids allocation on its hot path, or a
 * runtime that only hands out pre-registered buffers).  It computes exactly what
 * acl_cluster_attn_bwd computes, with the same arguments minus workspace/ws_bytes; its
 * scratch is a file-scope device array of ACL_NOALLOC_ATTN_WS_BYTES (4 MiB) that every
 * GPU loading the library holds until the process exits.  Nothing is allocated.
 *  - Sizes whose acl_cluster_attn_workspace(B, N, H, C, M) exceeds
 *    ACL_NOALLOC_ATTN_WS_BYTES return ACL_ERR_UNSUPPORTED (the regular entry point with a
 *    caller workspace has no such limit); bad sizes return ACL_ERR_INVALID_ARG.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call before any
 *    stream capture on the device.
 *  - The array used is the current device's: `stream` must belong to the current device
 *    (a stream of another device returns ACL_ERR_INVALID_ARG; NULL is the current
 *    device's legacy stream).
 *  - All calls share the one array, which keeps the last call's contents; nothing in it
 *    needs to start at zero (every scratch value is written before it is read).  Calls
 *    that overlap on the GPU (on different streams, without ordering) race on it.
 */
acl_status acl_cluster_attn_bwd_noalloc(const acl_bf16* Q, const acl_bf16* K, const acl_bf16* V,
                                        const float* coords, const int32_t* clusters,
                                        const int32_t* nbr, const float* bias_coef,
                                        int B, int N, int H, int D, int C, int M, float scale,
                                        const acl_bf16* O, const acl_bf16* dO, const float* lse,
                                        acl_bf16* dQ, acl_bf16* dK, acl_bf16* dV,
                                        float* dbias_coef, acl_stream_t stream);

/*
 * acl_knn_table -- KNN cache lookup table (a5).
 * Passage: AFF notes, "Key Designs" 3 (KNN Cache Lookup): an H x W x K table of
 * the K nearest visible tokens of every grid cell.
 *   table[r][c][k] = the k-th token in the order (dist2, token id), where
 *   dist2 = dx*dx + dy*dy, dx = x_t - (c + 0.5), dy = y_t - (r + 0.5) in fp64,
 *   each operation rounded separately.  Slots k >= N hold -1.
 * coords [B][N][2]; table [B][H][W][K] int32 out.  Bit-exact (a binned search
 * whose cut-off is conservative in exact arithmetic returns the brute-force set).
 * Limits: 1 <= N <= ACL_MAX_TABLE_N, 1 <= K <= ACL_MAX_KNN_K, 1 <= H, W <= 4096,
 *         B <= 65535.
 */
acl_status acl_knn_table(const float* coords, int B, int N, int H, int W, int K,
                         int32_t* table, acl_stream_t stream);

/*
 * acl_token_order -- space-filling (Z-order) token order.  Passage: AFF notes,
 * "Limitations" (the lookup table and the gathers are bound by memory traffic; space-filling
 * curves are suggested so that tokens close on the image are close in memory).
 *   cell(t) = (clamp(floor(y_t), 0, H-1), clamp(floor(x_t), 0, W-1)) as for a query;
 *   code(t) = Morton code of the cell: column bit i at bit 2i, row bit i at bit 2i + 1;
 *   perm[b][i] = the id of the i-th token by (code, id) ascending.
 * Permuting a stage's tokens (coordinates, features) by perm before the table and the
 * gathers puts every aligned 2^k x 2^k block of cells in one contiguous run of tokens.
 * coords [B][N][2] fp32 (8-byte aligned); perm [B][N] int32 out (a permutation of 0..N-1).
 * Bit-exact (integer keys only).  Limits: 1 <= N <= ACL_MAX_TABLE_N, 1 <= H, W <= 4096,
 * B <= 65535.
 */
acl_status acl_token_order(const float* coords, int B, int N, int H, int W, int32_t* perm,
                           acl_stream_t stream);

/*
 * Token merging between stages -- AFF notes, "Key Designs" 1 (adaptive off-grid token
 * merging): a lightweight MLP scores every token, the top-k are kept as anchors at the
 * retention rate, and the other tokens are merged differentiably into their nearest anchor,
 * fusing features and spatial support.  The notes fix no more; this library takes:
 *   s_i = w2 . gelu(W1^T f_i + b1) + b2, gelu(z) = z (1 + erf(z / sqrt 2)) / 2, fp32;
 *   anchors: the k largest s_i, ties by lower id, listed by ascending token id;
 *   assign_i: the rank (0..k-1) of the anchor nearest to token i (squared distance of the
 *     fp32 coordinates in fp64, ties by lower anchor id); an anchor is its own group;
 *   merged_j = sum_{i in G_j} w_i f_i and mcoords_j = sum w_i x_i, w = softmax of the
 *     group's scores (so the scores, and the MLP, receive gradients).
 * feats [B][N][d] bf16 (16-byte aligned); coords [B][N][2] fp32; W1 [d][h], b1 [h], w2 [h]
 * fp32 (device); scores [B][N] fp32, anchors [B][k] int32, assign [B][N] int32, merged
 * [B][k][d] bf16, mcoords [B][k][2] fp32 out.  The anchor choice is an integer decision on
 * fp32 scores; ties and near-ties follow the fp32 values.
 * workspace: acl_token_merge_workspace(B, N, d, h, k) bytes, 256-byte aligned.
 * Limits: d % 32 == 0, 32 <= d <= ACL_MAX_GATHER_D, 1 <= h <= 256, 1 <= k <= N <=
 * ACL_MAX_TABLE_N.  No atomics in any sum: results are bit-reproducible.
 */
size_t acl_token_merge_workspace(int B, int N, int d, int h, int k);
acl_status acl_token_merge_fwd(const acl_bf16* feats, const float* coords, int B, int N, int d,
                               const float* w1, const float* b1, const float* w2, float b2,
                               int h, int k, float* scores, int32_t* anchors, int32_t* assign,
                               acl_bf16* merged, float* mcoords, void* workspace,
                               size_t ws_bytes, acl_stream_t stream);
/*
 * Backward for the forward's scores and assignment (anchors and assignment are piecewise
 * constant: no gradient flows through them):
 *   g_i = <dmerged_j, f_i> + <dmcoords_j, x_i>, ds_i = w_i (g_i - sum_G w g),
 *   dfeats_i = w_i dmerged_j + W1 dh_i, dh_i = ds_i w2 * gelu'(z_i), dcoords_i = w_i dmcoords_j,
 *   dW1 = sum_i f_i dh_i^T, db1 = sum dh_i, dw2 = sum ds_i gelu(z_i), db2 = sum ds_i
 *   (sums over all images).  All outputs are overwritten.
 * dmerged [B][k][d] bf16, dmcoords [B][k][2] fp32 in; dfeats [B][N][d] bf16, dcoords
 * [B][N][2], dW1 [d][h], db1 [h], dw2 [h], db2 [1] fp32 out.  scores and assign are the
 * forward's outputs; a token whose assign entry lies outside [0, k) belongs to no group and
 * gets zero gradients.
 */
acl_status acl_token_merge_bwd(const acl_bf16* feats, const float* coords, int B, int N, int d,
                               const float* w1, const float* b1, const float* w2, float b2,
                               int h, int k, const float* scores, const int32_t* assign,
                               const acl_bf16* dmerged, const float* dmcoords, acl_bf16* dfeats,
                               float* dcoords, float* dw1, float* db1, float* dw2, float* db2,
                               void* workspace, size_t ws_bytes, acl_stream_t stream);

/* Workspace bytes acl_knn_gather_bwd (and acl_knn_gather_index +
 * acl_knn_gather_bwd_indexed) need for these sizes (0 on bad sizes). */
size_t acl_knn_gather_workspace(int B, int Q, int N, int d, int K);

/*
 * acl_knn_gather_fwd -- KNN distance-softmax gather, forward (a6).
 * Passage: AFF notes, "Key Designs" 2 (w_i = softmax_i(-p d_i) over the K nearest
 * tokens of the sample point q) and 3 (q quantised to its grid cell, neighbours
 * read from the table).
 *   cell = (clamp(floor(q_y), 0, H-1), clamp(floor(q_x), 0, W-1)); a coordinate
 *   that is not >= 0 maps to 0;
 *   d_k = ||q - p_{t_k}|| (fp32); per head h: w_hk = softmax_k(-p_h d_k), computed
 *   as exp(-p_h (d_k - d_min)) / sum; out[h*32 + e] = sum_k w_hk f[t_k][h*32 + e].
 *   Table slots holding -1 are skipped; a row with no token gives out = 0.
 * queries [B][Q][2] fp32; feats [B][N][d] bf16; coords [B][N][2]; table
 * [B][H][W][K] (e.g. from acl_knn_table); p [d/32] fp32 (one temperature per head).
 * out [B][Q][d] bf16 out.
 * Limits: d % 32 == 0, 32 <= d <= ACL_MAX_GATHER_D, 1 <= K <= ACL_MAX_KNN_K,
 *         table entries in [-1, N).
 * Non-finite features: for N <= 1024 and K <= 8 the sum runs as a tensor-core product
 * over tiles of 16 consecutive queries, which multiplies every token listed by the tile
 * by every query's weight (zeros included); a feature row holding Inf or NaN then makes
 * the outputs of all 16 queries of such a tile non-finite.  Finite inputs are unaffected.
 */
acl_status acl_knn_gather_fwd(const float* queries, int B, int Q, const acl_bf16* feats,
                              const float* coords, int N, int d, const int32_t* table,
                              int H, int W, int K, const float* p, acl_bf16* out,
                              acl_stream_t stream);

/*
 * Weight kernels of the gather.  AFF notes, "Key Designs" 2: the method uses the
 * exponential distance kernel w_k = softmax_k(-p d_k); the original AFF weighting it
 * replaced is the inverse power w_k = d_k^-p / sum_k' d_k'^-p, which the notes describe as
 * overflowing at short range and underflowing at long range in mixed precision.  Here the
 * inverse power is evaluated as (d_min / d_k)^p / sum (the same ratio, in [0, 1]): a
 * neighbour at d_min gets 1 (a query on a token, d_min = 0, puts all weight on the tokens
 * at its position, the d -> 0 limit), p = 0 gives equal weights; p must be >= 0.  In the
 * backward, dz/dp = -ln d_k and dz/dq = -p (q - x_k) / d_k^2; terms of a neighbour at
 * d_k = 0 are 0.
 */
typedef enum {
    ACL_KNN_EXP = 0,     /* softmax(-p d): the method's kernel (the plain entry points)   */
    ACL_KNN_INVPOW = 1   /* d^-p / sum d^-p: the original AFF weighting                   */
} acl_knn_kernel;

/* acl_knn_gather_fwd with a choice of weight kernel (ACL_ERR_INVALID_ARG for any other). */
acl_status acl_knn_gather_fwd_ex(const float* queries, int B, int Q, const acl_bf16* feats,
                                 const float* coords, int N, int d, const int32_t* table,
                                 int H, int W, int K, const float* p, acl_knn_kernel kind,
                                 acl_bf16* out, acl_stream_t stream);

/*
 * acl_knn_gather_bwd -- KNN gather, backward (a7).  With z_hk = -p_h d_k:
 *   dw_hk = <dOut_h, f_{t_k},h>, ds_hk = w_hk (dw_hk - sum_k' w_hk' dw_hk'),
 *   dp_h = sum over all queries and k of ds_hk (-d_k),
 *   dq = sum_{h,k} ds_hk (-p_h) (q - p_{t_k}) / d_k (the term is 0 when d_k = 0),
 *   dF_t = sum over (query, k) with t_k = t of w_hk dOut_h.
 * The cell index is piecewise constant (no gradient); coords get none.
 * dF is reduced per token over an inverse index built by a stable counting sort
 * (fixed order, no atomics).
 * Arguments as in the forward plus dOut [B][Q][d] bf16.
 * dfeats [B][N][d] bf16 out; dqueries [B][Q][2] fp32 out; dp [d/32] fp32 out.
 * workspace: at least acl_knn_gather_workspace(B, Q, N, d, K) bytes, 256-byte
 * aligned; its contents on entry do not matter.
 * Limits: as the forward, plus Q <= ACL_MAX_GATHER_Q and N <= ACL_MAX_TABLE_N.
 */
acl_status acl_knn_gather_bwd(const float* queries, int B, int Q, const acl_bf16* feats,
                              const float* coords, int N, int d, const int32_t* table,
                              int H, int W, int K, const float* p, const acl_bf16* dOut,
                              acl_bf16* dfeats, float* dqueries, float* dp,
                              void* workspace, size_t ws_bytes, acl_stream_t stream);

/* acl_knn_gather_bwd with a choice of weight kernel (the kind of the forward). */
acl_status acl_knn_gather_bwd_ex(const float* queries, int B, int Q, const acl_bf16* feats,
                                 const float* coords, int N, int d, const int32_t* table,
                                 int H, int W, int K, const float* p, acl_knn_kernel kind,
                                 const acl_bf16* dOut, acl_bf16* dfeats, float* dqueries,
                                 float* dp, void* workspace, size_t ws_bytes,
                                 acl_stream_t stream);

/*
 * acl_knn_gather_index -- the first stage of acl_knn_gather_bwd on its own: the inverse
 * index (for every token, its (query, slot) entries in ascending order, by a stable
 * counting sort) built from the queries' cells and the table alone, written into the
 * workspace.  Passage: AFF notes, "Key Designs" 3 (q quantised to its cell; the cell's
 * table row names its K tokens).  The index depends neither on the features nor on dOut,
 * so it can be built as soon as the table exists, e.g. on another stream while the
 * forward gather runs.
 * queries [B][Q][2] fp32; table [B][H][W][K] int32 (entries in [-1, N)); d selects the
 * workspace layout and must equal the d of the backward call that uses the index.
 * workspace: as for acl_knn_gather_bwd (same sizes); only its index regions are written.
 * Limits: as acl_knn_gather_bwd.
 */
acl_status acl_knn_gather_index(const float* queries, int B, int Q, int N, int d,
                                const int32_t* table, int H, int W, int K, void* workspace,
                                size_t ws_bytes, acl_stream_t stream);

/*
 * acl_knn_gather_bwd_indexed -- acl_knn_gather_bwd without its first stage: the same
 * arguments and results, reading the inverse index that acl_knn_gather_index wrote into
 * this workspace for the same queries, table and sizes (stream-ordered before this call).
 * The workspace's other regions are overwritten.  An index built for other inputs gives
 * wrong dfeats; nothing checks this.
 */
acl_status acl_knn_gather_bwd_indexed(const float* queries, int B, int Q, const acl_bf16* feats,
                                      const float* coords, int N, int d, const int32_t* table,
                                      int H, int W, int K, const float* p, const acl_bf16* dOut,
                                      acl_bf16* dfeats, float* dqueries, float* dp,
                                      void* workspace, size_t ws_bytes, acl_stream_t stream);

/* acl_knn_gather_bwd_indexed with a choice of weight kernel (the index does not depend on
 * it). */
acl_status acl_knn_gather_bwd_indexed_ex(const float* queries, int B, int Q,
                                         const acl_bf16* feats, const float* coords, int N, int d,
                                         const int32_t* table, int H, int W, int K,
                                         const float* p, acl_knn_kernel kind,
                                         const acl_bf16* dOut, acl_bf16* dfeats, float* dqueries,
                                         float* dp, void* workspace, size_t ws_bytes,
                                         acl_stream_t stream);

/*
 * acl_decoder_layer_fwd -- one layer of the point-wise deformable cross-attention decoder
 * (NEXT row f4).  Passage: AFFMAE notes, "Key Designs" 2 (each mask-token query predicts a 2D
 * offset Delta = g(f) and samples q = r + Delta, gathers an encoder stage's nearest visible
 * tokens around q with distance-softmax weights, the stages fused coarse to fine) and "A
 * Complete Example" (stage 4 first, then stages 3 to 1).  Readings: g is linear, and the
 * gathered feature is projected to the decoder width and added to the query feature:
 *   q = r + f W_off + b_off                     (fp32)
 *   v = acl_knn_gather_fwd of the stage at q    (exponential kernel, bf16 out)
 *   f_out = f + v W_o                           (bf16 tensor-core products, fp32 sums)
 * ref [B][Q][2], f_in [B][Q][D] fp32; W_off [D][2], b_off [2] fp32; W_o [d][D] bf16; the
 * stage as for the gather (feats [B][N][d] bf16, coords [B][N][2], table [B][H][W][K], p
 * [d/32]).  Out: q [B][Q][2] fp32, v [B][Q][d] bf16 (both needed by the backward), f_out
 * [B][Q][D] fp32 (may equal f_in when no backward follows).  Stacking layers over stages 4..1
 * is the caller's loop.  Limits: D % 128 == 0, 128 <= D <= 1024; d % 128 == 0 and the
 * gather's limits; Q <= ACL_MAX_GATHER_Q, B Q <= 2^24.  The cell choice is an integer decision
 * on the fp32 q.
 */
size_t acl_decoder_layer_workspace(int B, int Q, int N, int d, int D, int K);
/*
 * acl_device_check -- synchronises the current device, then reports (and clears) what the
 * device recorded since the last call:
 *   ACL_ERR_DEVICE_CHECK  (check build only, see acl_device_checks_enabled) a kernel met an
 *                         index input outside its range: a token id outside [-1, N) in a
 *                         cluster list, neighbour table or KNN table.  The kernels treat such
 *                         an id as an empty slot in both builds; the check build reports it;
 *   ACL_ERR_TIMEOUT       a bounded device-side wait of the tensor-core kernels gave up (the
 *                         affected outputs are zero, not garbage);
 *   ACL_OK                neither; ACL_ERR_CUDA if synchronising failed.
 */
acl_status acl_device_check(void);
/*
 * acl_device_checks_enabled -- 1 in the check build of the library (libacl_check.so, compiled
 * with ACL_DEVICE_CHECKS: every token id read from a cluster list, neighbour table or KNN
 * table is range-checked on the device), 0 in the regular build.
 */
int acl_device_checks_enabled(void);
/*
 * acl_test_set_wait_limit -- test hook: the SM clocks after which a main-loop mbarrier wait of
 * the tensor-core GEMM gives up (default 1e9, about half a second; 0 = give up at once;
 * negative restores the default).  The wait for the MMAs
 * still in flight before tensor memory is freed always keeps the default, so a lowered limit
 * ends the kernel early with zero outputs and ACL_ERR_TIMEOUT from acl_device_check, never
 * with a fault.  Synchronous; affects the current device.
 */
acl_status acl_test_set_wait_limit(long long cycles);
acl_status acl_decoder_layer_fwd(const float* ref, const float* f_in, int B, int Q, int D,
                                 const float* w_off, const float* b_off, const acl_bf16* w_o,
                                 const acl_bf16* feats, const float* coords, int N, int d,
                                 const int32_t* table, int H, int W, int K, const float* p,
                                 float* q, acl_bf16* v, float* f_out, acl_stream_t stream);
/*
 * Backward of one decoder layer at the forward's q and v:
 *   dv = df_out W_o^T (bf16), dW_o = v^T df_out, the gather's backward of dv (dfeats, dq, dp),
 *   df_in = df_out + dq W_off^T, dW_off = f_in^T dq, db_off = sum dq
 * (parameter gradients summed over all queries in a fixed order: bit-reproducible).  Out:
 * df_in [B][Q][D] (may equal df_out), dW_off [D][2], db_off [2], dW_o [d][D] fp32, dfeats
 * [B][N][d] bf16, dp [d/32] fp32; all overwritten.  workspace: acl_decoder_layer_workspace
 * bytes, 256-byte aligned.
 */
acl_status acl_decoder_layer_bwd(const float* f_in, int B, int Q, int D, const float* w_off,
                                 const acl_bf16* w_o, const acl_bf16* feats, const float* coords,
                                 int N, int d, const int32_t* table, int H, int W, int K,
                                 const float* p, const float* q, const acl_bf16* v,
                                 const float* df_out, float* df_in, float* dw_off, float* db_off,
                                 float* dw_o, acl_bf16* dfeats, float* dp, void* workspace,
                                 size_t ws_bytes, acl_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* ACL_H */
