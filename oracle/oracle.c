/*
 * oracle.c -- plain, slow fp64 CPU reference for the off-grid cluster attention
 * and KNN distance-softmax gather.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file: only the tests, the smoke check and the benchmark's CPU-baseline
 * leg do.  It shares no code, header, table or helper with the CUDA library.
 *
 * Sources (page title, section):
 *   [AFF]  "AFFMAE: Scalable Vision Pre-Training for High-Resolution Microscopy
 *          Segmentation on Desktop Hardware" (en.papernotes.org notes), Method:
 *          "Overall Architecture" (tokens carry explicit 2D coordinates; attention
 *          through local balanced clustering; stages of Local Cluster Attention),
 *          "Key Designs" 2 (point-wise deformable cross-attention decoder, the
 *          exponential distance kernel w_i = softmax_i(-p d_i)), "Key Designs" 3
 *          (KNN cache lookup: an H x W x K table of the K nearest visible tokens
 *          per grid cell, queries quantised to a cell), "A Complete Example"
 *          (64 x 64 grid, ~2048 visible tokens, 819 / 328 / 131 after merging).
 *   [ABS]  "AFFMAE: Scalable and Efficient Vision Pretraining for Desktop
 *          Graphics Cards" (arXiv abstract page): mixed-precision Flash-style
 *          cluster attention kernels.
 * The pages name the operations but leave their details open.  The readings
 * taken here (recursive median bisection, C tokens per cluster, M = R*C slots
 * from the R nearest cluster centroids, the bias a*dx + b*dy - c*(dx^2+dy^2)
 * with dx = key - query, cell-centre lookup with clamping, per-head p) are the
 * plainest ones consistent with the pages; each is stated where it is used.
 *
 * Arithmetic: fp64 throughout; compiled with -ffp-contract=off so that every
 * product and sum is rounded on its own, in the order written.  Index-producing
 * geometry (extents, centroids, squared distances) is written as single
 * expressions whose rounding order the docstrings state.
 *
 * Pins: every function here is checked in tests/ against closed forms,
 * invariants, brute force on tiny inputs, library routines (dense softmax
 * attention, a KD-tree) and finite differences.  See the test files.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "oracle.h"

#ifdef _OPENMP
#include <omp.h>
#endif

/* Thread count of the batch drivers (OpenMP); returns the count in use. */
int orc_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}

/* ------------------------------------------------------------------------ */
/* a1: local balanced clustering                                             */
/* ------------------------------------------------------------------------ */

typedef struct {
    float a;      /* coordinate on the split axis   */
    float b;      /* coordinate on the other axis   */
    int32_t id;   /* token id: the final tie-break  */
} split_key;

static int cmp_split_key(const void* pa, const void* pb) {
    const split_key* x = (const split_key*)pa;
    const split_key* y = (const split_key*)pb;
    if (x->a < y->a) return -1;
    if (x->a > y->a) return 1;
    if (x->b < y->b) return -1;
    if (x->b > y->b) return 1;
    return (x->id > y->id) - (x->id < y->id);
}

static int cmp_i32(const void* pa, const void* pb) {
    int32_t x = *(const int32_t*)pa, y = *(const int32_t*)pb;
    return (x > y) - (x < y);
}

/*
 * split(S, g): cut the token set S (n tokens) into g clusters.
 *   g == 1: emit S sorted by token id, padded with -1 to C slots.
 *   else:   ex = max x - min x, ey = max y - min y over S (fp64 from fp32);
 *           axis = x when ex >= ey, else y;
 *           order S by (coordinate on axis, coordinate on the other axis, id);
 *           the first ceil(g/2)*C tokens form the left part (ceil(g/2)
 *           clusters), the rest the right part (g - ceil(g/2) clusters);
 *           recurse left, then right.
 * Clusters are numbered in emit order.  Because every left part is full, only
 * the last cluster of the image can hold padding.
 */
static void split(const float* xy, int32_t* ids, int n, int g, int C,
                  int32_t* out, int* next, split_key* keys) {
    if (g == 1) {
        int32_t* dst = out + (size_t)(*next) * C;
        qsort(ids, (size_t)n, sizeof(int32_t), cmp_i32);
        for (int s = 0; s < C; ++s) dst[s] = (s < n) ? ids[s] : -1;
        (*next)++;
        return;
    }
    double xmin = INFINITY, xmax = -INFINITY, ymin = INFINITY, ymax = -INFINITY;
    for (int i = 0; i < n; ++i) {
        double x = (double)xy[2 * ids[i]], y = (double)xy[2 * ids[i] + 1];
        if (x < xmin) xmin = x;
        if (x > xmax) xmax = x;
        if (y < ymin) ymin = y;
        if (y > ymax) ymax = y;
    }
    double ex = xmax - xmin, ey = ymax - ymin;
    int axis = (ex >= ey) ? 0 : 1;
    for (int i = 0; i < n; ++i) {
        keys[i].a = xy[2 * ids[i] + axis];
        keys[i].b = xy[2 * ids[i] + (1 - axis)];
        keys[i].id = ids[i];
    }
    qsort(keys, (size_t)n, sizeof(split_key), cmp_split_key);
    for (int i = 0; i < n; ++i) ids[i] = keys[i].id;
    int gl = (g + 1) / 2;
    int nl = gl * C;
    split(xy, ids, nl, gl, C, out, next, keys);
    split(xy, ids + nl, n - nl, g - gl, C, out, next, keys);
}

int orc_cluster(const float* xy, int N, int C, int32_t* clusters) {
    if (N < 1 || C < 1 || !xy || !clusters) return 1;
    int G = (N + C - 1) / C;
    int32_t* ids = (int32_t*)malloc(sizeof(int32_t) * (size_t)N);
    split_key* keys = (split_key*)malloc(sizeof(split_key) * (size_t)N);
    if (!ids || !keys) { free(ids); free(keys); return 2; }
    for (int i = 0; i < N; ++i) ids[i] = i;
    int next = 0;
    split(xy, ids, N, G, C, clusters, &next, keys);
    free(ids);
    free(keys);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* a2: cluster-neighbourhood table                                           */
/* ------------------------------------------------------------------------ */

/*
 * centroid_g = (sum of the valid slots' x, in slot order, from 0.0) / n_valid,
 * likewise y, fp64.  dist2(g, h) = dx*dx + dy*dy with dx = cx_h - cx_g,
 * dy = cy_h - cy_g, each product and the sum rounded separately.
 * The neighbourhood of g is the first min(R, G) clusters by (dist2, h),
 * R = M / C; nbr[g][r*C + s] = clusters[h_r][s]; remaining slots -1.
 */
int orc_neighbors(const float* xy, const int32_t* clusters, int N, int C, int M,
                  int32_t* nbr) {
    if (N < 1 || C < 1 || M < C || M % C != 0 || !xy || !clusters || !nbr) return 1;
    int G = (N + C - 1) / C;
    int R = M / C;
    double* cx = (double*)malloc(sizeof(double) * (size_t)G);
    double* cy = (double*)malloc(sizeof(double) * (size_t)G);
    double* d2 = (double*)malloc(sizeof(double) * (size_t)G);
    char* taken = (char*)malloc((size_t)G);
    if (!cx || !cy || !d2 || !taken) { free(cx); free(cy); free(d2); free(taken); return 2; }
    for (int g = 0; g < G; ++g) {
        double sx = 0.0, sy = 0.0;
        int cnt = 0;
        for (int s = 0; s < C; ++s) {
            int32_t t = clusters[(size_t)g * C + s];
            if (t < 0) continue;
            sx = sx + (double)xy[2 * t];
            sy = sy + (double)xy[2 * t + 1];
            cnt++;
        }
        cx[g] = sx / (double)cnt;
        cy[g] = sy / (double)cnt;
    }
    for (int g = 0; g < G; ++g) {
        for (int h = 0; h < G; ++h) {
            double dx = cx[h] - cx[g];
            double dy = cy[h] - cy[g];
            double px = dx * dx;
            double py = dy * dy;
            d2[h] = px + py;
            taken[h] = 0;
        }
        int32_t* row = nbr + (size_t)g * M;
        for (int m = 0; m < M; ++m) row[m] = -1;
        int take = R < G ? R : G;
        for (int r = 0; r < take; ++r) {
            int best = -1;
            for (int h = 0; h < G; ++h) {
                if (taken[h]) continue;
                if (best < 0 || d2[h] < d2[best]) best = h;   /* ties: lower h */
            }
            taken[best] = 1;
            for (int s = 0; s < C; ++s) row[r * C + s] = clusters[(size_t)best * C + s];
        }
    }
    free(cx); free(cy); free(d2); free(taken);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* a3 / a4: local cluster attention, forward and backward                    */
/* ------------------------------------------------------------------------ */

/*
 * For a valid token i of cluster g, head h, and every valid key j in nbr(g):
 *   dx = x_j - x_i, dy = y_j - y_i                       (key minus query)
 *   s_ij = scale * <q_i, k_j> + a_h dx + b_h dy - c_h (dx^2 + dy^2)
 *   o_i  = sum_j softmax_j(s_ij) v_j,   lse_i = log sum_j exp(s_ij)
 * Plain two-pass softmax (max, then exp-sum), no tiling.  A token whose
 * neighbourhood holds no valid key gets o = 0 and lse = -inf.
 * Layout: q, k, v, o as [N][H][D]; lse as [N][H]; bias as [H][3] = (a, b, c).
 */
static int attn_logits(const double* q, const double* k, const float* xy,
                       const int32_t* nrow, const double* bias, int i, int h,
                       int H, int D, int M, double scale, double* s, int* valid) {
    int any = 0;
    const double a = bias[3 * h], b = bias[3 * h + 1], c = bias[3 * h + 2];
    for (int m = 0; m < M; ++m) {
        int32_t j = nrow[m];
        valid[m] = (j >= 0);
        if (j < 0) { s[m] = -INFINITY; continue; }
        any = 1;
        double dx = (double)xy[2 * j] - (double)xy[2 * i];
        double dy = (double)xy[2 * j + 1] - (double)xy[2 * i + 1];
        double dot = 0.0;
        const double* qi = q + ((size_t)i * H + h) * D;
        const double* kj = k + ((size_t)j * H + h) * D;
        for (int e = 0; e < D; ++e) dot += qi[e] * kj[e];
        s[m] = scale * dot + a * dx + b * dy - c * (dx * dx + dy * dy);
    }
    return any;
}

/* The forward for heads [h0, h1) only (heads are independent; o and lse of the other
 * heads are left untouched). */
static int attn_fwd_heads(const double* q, const double* k, const double* v, const float* xy,
                          const int32_t* clusters, const int32_t* nbr, const double* bias,
                          int N, int H, int D, int C, int M, double scale, int h0, int h1,
                          double* o, double* lse) {
    if (N < 1 || H < 1 || D < 1 || C < 1 || M < 1 || h0 < 0 || h1 > H) return 1;
    int G = (N + C - 1) / C;
    double* s = (double*)malloc(sizeof(double) * (size_t)M);
    int* valid = (int*)malloc(sizeof(int) * (size_t)M);
    if (!s || !valid) { free(s); free(valid); return 2; }
    for (int g = 0; g < G; ++g) {
        const int32_t* nrow = nbr + (size_t)g * M;
        for (int sl = 0; sl < C; ++sl) {
            int32_t i = clusters[(size_t)g * C + sl];
            if (i < 0) continue;
            for (int h = h0; h < h1; ++h) {
                double* oi = o + ((size_t)i * H + h) * D;
                for (int e = 0; e < D; ++e) oi[e] = 0.0;
                if (!attn_logits(q, k, xy, nrow, bias, i, h, H, D, M, scale, s, valid)) {
                    lse[(size_t)i * H + h] = -INFINITY;
                    continue;
                }
                double mx = -INFINITY;
                for (int m = 0; m < M; ++m) if (valid[m] && s[m] > mx) mx = s[m];
                double sum = 0.0;
                for (int m = 0; m < M; ++m) if (valid[m]) sum += exp(s[m] - mx);
                for (int m = 0; m < M; ++m) {
                    if (!valid[m]) continue;
                    double p = exp(s[m] - mx) / sum;
                    const double* vj = v + ((size_t)nrow[m] * H + h) * D;
                    for (int e = 0; e < D; ++e) oi[e] += p * vj[e];
                }
                lse[(size_t)i * H + h] = mx + log(sum);
            }
        }
    }
    free(s); free(valid);
    return 0;
}

int orc_attn_fwd(const double* q, const double* k, const double* v, const float* xy,
                 const int32_t* clusters, const int32_t* nbr, const double* bias,
                 int N, int H, int D, int C, int M, double scale,
                 double* o, double* lse) {
    return attn_fwd_heads(q, k, v, xy, clusters, nbr, bias, N, H, D, C, M, scale, 0, H, o, lse);
}

/*
 * Backward by recomputation, from the definition of the forward:
 *   P_ij = exp(s_ij - lse_i), dP_ij = <dO_i, v_j>, Delta_i = <dO_i, o_i>,
 *   dS_ij = P_ij (dP_ij - Delta_i),
 *   dq_i = scale sum_j dS_ij k_j,  dk_j = scale sum_i dS_ij q_i,
 *   dv_j = sum_i P_ij dO_i,
 *   da_h = sum dS dx,  db_h = sum dS dy,  dc_h = -sum dS (dx^2 + dy^2).
 * o and lse are this oracle's own forward results.  Coordinates get no
 * gradient.  dq, dk, dv are overwritten; dbias [H][3] is overwritten.
 */
/* The backward for heads [h0, h1) only: dq, dk, dv of those heads and dbias[h0..h1)
 * are overwritten, the other heads are left untouched.  Every sum keeps the order of the
 * all-heads loop (clusters, slots, then keys), since a head's sums never mix with
 * another head's. */
static int attn_bwd_heads(const double* q, const double* k, const double* v, const float* xy,
                          const int32_t* clusters, const int32_t* nbr, const double* bias,
                          int N, int H, int D, int C, int M, double scale, int h0, int h1,
                          const double* dout, double* dq, double* dk, double* dv,
                          double* dbias) {
    if (N < 1 || H < 1 || D < 1 || C < 1 || M < 1 || h0 < 0 || h1 > H) return 1;
    int G = (N + C - 1) / C;
    size_t nel = (size_t)N * H * D;
    double* o = (double*)malloc(sizeof(double) * nel);
    double* lse = (double*)malloc(sizeof(double) * (size_t)N * H);
    double* s = (double*)malloc(sizeof(double) * (size_t)M);
    int* valid = (int*)malloc(sizeof(int) * (size_t)M);
    if (!o || !lse || !s || !valid) { free(o); free(lse); free(s); free(valid); return 2; }
    int rc = attn_fwd_heads(q, k, v, xy, clusters, nbr, bias, N, H, D, C, M, scale, h0, h1,
                            o, lse);
    if (rc) { free(o); free(lse); free(s); free(valid); return rc; }
    for (int t = 0; t < N; ++t)
        for (int h = h0; h < h1; ++h)
            for (int e = 0; e < D; ++e) {
                size_t x = ((size_t)t * H + h) * D + e;
                dq[x] = 0.0;
                dk[x] = 0.0;
                dv[x] = 0.0;
            }
    for (int h = h0; h < h1; ++h) dbias[3 * h] = dbias[3 * h + 1] = dbias[3 * h + 2] = 0.0;
    for (int g = 0; g < G; ++g) {
        const int32_t* nrow = nbr + (size_t)g * M;
        for (int sl = 0; sl < C; ++sl) {
            int32_t i = clusters[(size_t)g * C + sl];
            if (i < 0) continue;
            for (int h = h0; h < h1; ++h) {
                if (!attn_logits(q, k, xy, nrow, bias, i, h, H, D, M, scale, s, valid)) continue;
                const double L = lse[(size_t)i * H + h];
                const double* doi = dout + ((size_t)i * H + h) * D;
                const double* oi = o + ((size_t)i * H + h) * D;
                const double* qi = q + ((size_t)i * H + h) * D;
                double* dqi = dq + ((size_t)i * H + h) * D;
                double delta = 0.0;
                for (int e = 0; e < D; ++e) delta += doi[e] * oi[e];
                for (int m = 0; m < M; ++m) {
                    if (!valid[m]) continue;
                    int32_t j = nrow[m];
                    const double* vj = v + ((size_t)j * H + h) * D;
                    const double* kj = k + ((size_t)j * H + h) * D;
                    double* dkj = dk + ((size_t)j * H + h) * D;
                    double* dvj = dv + ((size_t)j * H + h) * D;
                    double p = exp(s[m] - L);
                    double dp = 0.0;
                    for (int e = 0; e < D; ++e) dp += doi[e] * vj[e];
                    double ds = p * (dp - delta);
                    for (int e = 0; e < D; ++e) {
                        dqi[e] += scale * ds * kj[e];
                        dkj[e] += scale * ds * qi[e];
                        dvj[e] += p * doi[e];
                    }
                    double dx = (double)xy[2 * j] - (double)xy[2 * i];
                    double dy = (double)xy[2 * j + 1] - (double)xy[2 * i + 1];
                    dbias[3 * h] += ds * dx;
                    dbias[3 * h + 1] += ds * dy;
                    dbias[3 * h + 2] -= ds * (dx * dx + dy * dy);
                }
            }
        }
    }
    free(o); free(lse); free(s); free(valid);
    return 0;
}

int orc_attn_bwd(const double* q, const double* k, const double* v, const float* xy,
                 const int32_t* clusters, const int32_t* nbr, const double* bias,
                 int N, int H, int D, int C, int M, double scale, const double* dout,
                 double* dq, double* dk, double* dv, double* dbias) {
    return attn_bwd_heads(q, k, v, xy, clusters, nbr, bias, N, H, D, C, M, scale, 0, H, dout,
                          dq, dk, dv, dbias);
}

/* ------------------------------------------------------------------------ */
/* a5: KNN cache lookup table                                                */
/* ------------------------------------------------------------------------ */

/*
 * table[r][c][k] = the k-th token in the order (dist2, id), where
 * dist2 = dx*dx + dy*dy, dx = x_t - (c + 0.5), dy = y_t - (r + 0.5), fp64,
 * each operation rounded on its own.  Slots k >= N hold -1.  The table stores
 * the neighbours of the cell centre (the lookup the pages describe), not of a
 * particular query.  Brute force over all tokens.
 */
int orc_knn_table(const float* xy, int N, int GH, int GW, int K, int32_t* table) {
    if (N < 1 || GH < 1 || GW < 1 || K < 1 || !xy || !table) return 1;
    double* d2 = (double*)malloc(sizeof(double) * (size_t)N);
    char* taken = (char*)malloc((size_t)N);
    if (!d2 || !taken) { free(d2); free(taken); return 2; }
    for (int r = 0; r < GH; ++r) {
        for (int c = 0; c < GW; ++c) {
            double ccx = (double)c + 0.5, ccy = (double)r + 0.5;
            for (int t = 0; t < N; ++t) {
                double dx = (double)xy[2 * t] - ccx;
                double dy = (double)xy[2 * t + 1] - ccy;
                double px = dx * dx;
                double py = dy * dy;
                d2[t] = px + py;
                taken[t] = 0;
            }
            int32_t* row = table + ((size_t)r * GW + c) * K;
            for (int kk = 0; kk < K; ++kk) {
                int best = -1;
                for (int t = 0; t < N; ++t) {
                    if (taken[t]) continue;
                    if (best < 0 || d2[t] < d2[best]) best = t;   /* ties: lower id */
                }
                row[kk] = best;
                if (best >= 0) taken[best] = 1;
            }
        }
    }
    free(d2); free(taken);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* a6 / a7: KNN distance-softmax gather, forward and backward                */
/* ------------------------------------------------------------------------ */

/*
 * Query quantisation: cell = (clamp(floor(qy), 0, GH-1), clamp(floor(qx), 0,
 * GW-1)); with cell centres at +0.5 this is the nearest cell, and clamping
 * keeps offsets that leave the grid on its border.  A coordinate that is not
 * >= 0 (negative or NaN) maps to 0.
 */
static int quantise(float v, int n) {
    if (!(v >= 0.0f)) return 0;
    if (v >= (float)n) return n - 1;
    int i = (int)floor((double)v);
    return i > n - 1 ? n - 1 : i;
}

/*
 * d_k = ||q - p_{t_k}|| (Euclidean, fp64); per head h (channels h*32..h*32+31) the
 * weights of the K neighbours, for the two kernels the AFFMAE notes compare ("Key Designs"
 * 2):
 *   kind 0, exponential (the method):  w_hk = exp(-p_h (d_k - d_min)) / sum_k' (same),
 *     i.e. softmax_k(-p_h d_k);
 *   kind 1, inverse power (the original AFF kernel the notes replace):
 *     w_hk = d_k^(-p_h) / sum_k' d_k'^(-p_h), evaluated as (d_min / d_k)^p_h / sum (same),
 *     the same ratio with both terms divided by d_min^(-p_h); a neighbour at d_min gets
 *     the factor 1 (so when the query sits on tokens, d_min = 0, they share the weight and
 *     the others get 0, the limit of the definition), and p_h = 0 gives equal weights.
 * out[q][h*32+e] = sum_k w_hk f[t_k][h*32+e].  Table slots holding -1 are skipped.  A
 * query whose row holds no token gets out = 0.
 */
static int knn_weights(const float* qxy, const float* xy, const int32_t* row, int K,
                       double ph, int kind, double* dist, double* w) {
    double dmin = INFINITY;
    int any = 0;
    for (int kk = 0; kk < K; ++kk) {
        int32_t t = row[kk];
        if (t < 0) { dist[kk] = INFINITY; continue; }
        double dx = (double)qxy[0] - (double)xy[2 * t];
        double dy = (double)qxy[1] - (double)xy[2 * t + 1];
        dist[kk] = sqrt(dx * dx + dy * dy);
        if (dist[kk] < dmin) dmin = dist[kk];
        any = 1;
    }
    if (!any) return 0;
    double sum = 0.0;
    for (int kk = 0; kk < K; ++kk) {
        if (row[kk] < 0) w[kk] = 0.0;
        else if (kind == 0) w[kk] = exp(-ph * (dist[kk] - dmin));
        else w[kk] = (dist[kk] == dmin || ph == 0.0) ? 1.0 : pow(dmin / dist[kk], ph);
        sum += w[kk];
    }
    for (int kk = 0; kk < K; ++kk) w[kk] /= sum;
    return 1;
}

int orc_knn_fwd(const float* queries, int Q, const double* feats, const float* xy,
                int N, int d, const int32_t* table, int GH, int GW, int K,
                const double* p, int kind, double* out) {
    if (Q < 0 || N < 1 || d < 32 || d % 32 != 0 || K < 1 || K > 64) return 1;
    int nh = d / 32;
    double dist[64], w[64];
    for (int qi = 0; qi < Q; ++qi) {
        const float* qxy = queries + 2 * (size_t)qi;
        int cy = quantise(qxy[1], GH), cx = quantise(qxy[0], GW);
        const int32_t* row = table + ((size_t)cy * GW + cx) * K;
        double* oq = out + (size_t)qi * d;
        for (int c = 0; c < d; ++c) oq[c] = 0.0;
        for (int h = 0; h < nh; ++h) {
            if (!knn_weights(qxy, xy, row, K, p[h], kind, dist, w)) break;
            for (int kk = 0; kk < K; ++kk) {
                int32_t t = row[kk];
                if (t < 0) continue;
                const double* f = feats + (size_t)t * d + 32 * h;
                for (int e = 0; e < 32; ++e) oq[32 * h + e] += w[kk] * f[e];
            }
        }
    }
    return 0;
}

/*
 * Backward of the gather.  With z_hk the logits of w_h (w_h = softmax_k(z_hk)):
 * z_hk = -p_h d_k (kind 0) or -p_h ln d_k (kind 1), and
 *   dw_hk = <dOut_q,h , f_{t_k},h>,  ds_hk = w_hk (dw_hk - sum_k' w_hk' dw_hk'),
 *   dp_h += sum_k ds_hk dz_hk/dp_h,  dz/dp = -d_k (kind 0), -ln d_k (kind 1),
 *   dq   += sum_{h,k} ds_hk dz_hk/dq, dz/dq = -p_h (q - p_{t_k}) / d_k (kind 0),
 *           -p_h (q - p_{t_k}) / d_k^2 (kind 1),
 *   dF_t += w_hk dOut_q,h for t = t_k.
 * Terms of a neighbour at d_k = 0 are taken as 0 in dq (both kinds) and in dp (kind 1),
 * where the derivatives are undefined.
 * The cell index is piecewise constant in q and has no gradient; token
 * coordinates get none.  dfeats [N][d], dq [Q][2] and dp [d/32] are overwritten.
 */
int orc_knn_bwd(const float* queries, int Q, const double* feats, const float* xy,
                int N, int d, const int32_t* table, int GH, int GW, int K,
                const double* p, int kind, const double* dout,
                double* dfeats, double* dq, double* dp) {
    if (Q < 0 || N < 1 || d < 32 || d % 32 != 0 || K < 1 || K > 64) return 1;
    int nh = d / 32;
    double dist[64], w[64], dw[64];
    memset(dfeats, 0, sizeof(double) * (size_t)N * d);
    memset(dq, 0, sizeof(double) * (size_t)Q * 2);
    memset(dp, 0, sizeof(double) * (size_t)nh);
    for (int qi = 0; qi < Q; ++qi) {
        const float* qxy = queries + 2 * (size_t)qi;
        int cy = quantise(qxy[1], GH), cx = quantise(qxy[0], GW);
        const int32_t* row = table + ((size_t)cy * GW + cx) * K;
        const double* g = dout + (size_t)qi * d;
        for (int h = 0; h < nh; ++h) {
            if (!knn_weights(qxy, xy, row, K, p[h], kind, dist, w)) break;
            double sdw = 0.0;
            for (int kk = 0; kk < K; ++kk) {
                int32_t t = row[kk];
                dw[kk] = 0.0;
                if (t < 0) continue;
                const double* f = feats + (size_t)t * d + 32 * h;
                for (int e = 0; e < 32; ++e) dw[kk] += g[32 * h + e] * f[e];
                sdw += w[kk] * dw[kk];
            }
            for (int kk = 0; kk < K; ++kk) {
                int32_t t = row[kk];
                if (t < 0) continue;
                double ds = w[kk] * (dw[kk] - sdw);
                if (kind == 0) dp[h] += ds * (-dist[kk]);
                else if (dist[kk] > 0.0) dp[h] += ds * (-log(dist[kk]));
                if (dist[kk] > 0.0) {
                    double r = kind == 0 ? dist[kk] : dist[kk] * dist[kk];
                    double ux = ((double)qxy[0] - (double)xy[2 * t]) / r;
                    double uy = ((double)qxy[1] - (double)xy[2 * t + 1]) / r;
                    dq[2 * qi] += ds * (-p[h]) * ux;
                    dq[2 * qi + 1] += ds * (-p[h]) * uy;
                }
                double* df = dfeats + (size_t)t * d + 32 * h;
                for (int e = 0; e < 32; ++e) df[e] += w[kk] * g[32 * h + e];
            }
        }
    }
    return 0;
}

/*
 * Space-filling token order (AFFMAE notes, "Limitations": the dense lookup table and the
 * gathers are bandwidth-bound, and space-filling curves are suggested to keep neighbouring
 * tokens close in memory).  Each token's cell on the H x W grid (quantised as the gather
 * quantises a query) gets its Z-order (Morton) code: bit i of the column goes to bit 2i,
 * bit i of the row to bit 2i + 1.  perm lists the token ids by (code, id) ascending.
 */
static uint32_t morton_code(uint32_t r, uint32_t c) {
    uint32_t code = 0;
    for (int i = 0; i < 16; ++i) {
        code |= ((c >> i) & 1u) << (2 * i);
        code |= ((r >> i) & 1u) << (2 * i + 1);
    }
    return code;
}

static int cmp_u64(const void* pa, const void* pb) {
    uint64_t a = *(const uint64_t*)pa, b = *(const uint64_t*)pb;
    return (a > b) - (a < b);
}

int orc_token_order(const float* xy, int N, int GH, int GW, int32_t* perm) {
    if (N < 1 || GH < 1 || GW < 1 || GH > 65536 || GW > 65536) return 1;
    uint64_t* key = (uint64_t*)malloc(sizeof(uint64_t) * (size_t)N);
    if (!key) return 2;
    for (int t = 0; t < N; ++t) {
        uint32_t r = (uint32_t)quantise(xy[2 * t + 1], GH), c = (uint32_t)quantise(xy[2 * t], GW);
        key[t] = ((uint64_t)morton_code(r, c) << 32) | (uint32_t)t;
    }
    qsort(key, (size_t)N, sizeof(uint64_t), cmp_u64);
    for (int i = 0; i < N; ++i) perm[i] = (int32_t)(key[i] & 0xffffffffu);
    free(key);
    return 0;
}

/*
 * Token merging between stages (AFFMAE notes, "Key Designs" 1, adaptive off-grid token
 * merging): a lightweight MLP scores every token, the top-k by score are kept as anchors
 * at the retention rate, and every other token is merged differentiably into its nearest
 * anchor, fusing features and spatial support.  The notes fix no more than that; the
 * readings taken:
 *   score s_i = w2 . gelu(W1^T f_i + b1) + b2, W1 [d][h], gelu(z) = z (1 + erf(z/sqrt 2))/2;
 *   anchors: the k largest scores, ties by lower id, listed by ascending id;
 *   assignment: the nearest anchor by squared distance (dx*dx + dy*dy in fp64, dx = x_i -
 *     x_a), ties by lower anchor id; an anchor is its own group;
 *   merge: group G_j of anchor j, weights w_i = exp(s_i - max_G s) / sum_G exp(.) (the
 *     softmax of the scores: differentiable in the scores, so the MLP is trained through
 *     the merge); merged feature F_j = sum_G w_i f_i, merged coordinate X_j = sum_G w_i x_i.
 */
static const double kPi = 3.14159265358979323846;
static double gelu(double z) { return 0.5 * z * (1.0 + erf(z / sqrt(2.0))); }
static double gelu_grad(double z) {
    return 0.5 * (1.0 + erf(z / sqrt(2.0))) + z * exp(-0.5 * z * z) / sqrt(2.0 * kPi);
}

int orc_merge_scores(const double* f, int N, int d, const double* w1, const double* b1,
                     const double* w2, double b2, int h, double* scores) {
    if (N < 1 || d < 1 || h < 1) return 1;
    for (int i = 0; i < N; ++i) {
        double s = b2;
        for (int u = 0; u < h; ++u) {
            double z = b1[u];
            for (int c = 0; c < d; ++c) z += f[(size_t)i * d + c] * w1[(size_t)c * h + u];
            s += w2[u] * gelu(z);
        }
        scores[i] = s;
    }
    return 0;
}

typedef struct { double s; int id; } score_id;
static int cmp_score_desc(const void* pa, const void* pb) {
    const score_id* a = (const score_id*)pa;
    const score_id* b = (const score_id*)pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    return (a->id > b->id) - (a->id < b->id);
}

int orc_merge_select(const double* scores, const float* xy, int N, int k, int32_t* anchors,
                     int32_t* assign) {
    if (N < 1 || k < 1 || k > N) return 1;
    score_id* o = (score_id*)malloc(sizeof(score_id) * (size_t)N);
    int32_t* rank = (int32_t*)malloc(sizeof(int32_t) * (size_t)N);
    if (!o || !rank) { free(o); free(rank); return 2; }
    for (int i = 0; i < N; ++i) { o[i].s = scores[i]; o[i].id = i; rank[i] = -1; }
    qsort(o, (size_t)N, sizeof(score_id), cmp_score_desc);
    for (int j = 0; j < k; ++j) anchors[j] = o[j].id;
    qsort(anchors, (size_t)k, sizeof(int32_t), cmp_i32);
    for (int j = 0; j < k; ++j) rank[anchors[j]] = j;
    for (int i = 0; i < N; ++i) {
        if (rank[i] >= 0) { assign[i] = rank[i]; continue; }
        double best = INFINITY;
        int bj = 0;
        for (int j = 0; j < k; ++j) {
            int a = anchors[j];
            double dx = (double)xy[2 * i] - (double)xy[2 * a];
            double dy = (double)xy[2 * i + 1] - (double)xy[2 * a + 1];
            double d2 = dx * dx + dy * dy;
            if (d2 < best) { best = d2; bj = j; }   /* strict: ties keep the lower id */
        }
        assign[i] = bj;
    }
    free(o);
    free(rank);
    return 0;
}

int orc_merge_fwd(const double* f, const float* xy, int N, int d, const double* scores, int k,
                  const int32_t* assign, double* merged, double* mxy) {
    if (N < 1 || d < 1 || k < 1) return 1;
    double* gmax = (double*)malloc(sizeof(double) * (size_t)k);
    double* gsum = (double*)calloc((size_t)k, sizeof(double));
    if (!gmax || !gsum) { free(gmax); free(gsum); return 2; }
    for (int j = 0; j < k; ++j) gmax[j] = -INFINITY;
    for (int i = 0; i < N; ++i) if (scores[i] > gmax[assign[i]]) gmax[assign[i]] = scores[i];
    for (int i = 0; i < N; ++i) gsum[assign[i]] += exp(scores[i] - gmax[assign[i]]);
    memset(merged, 0, sizeof(double) * (size_t)k * d);
    memset(mxy, 0, sizeof(double) * (size_t)k * 2);
    for (int i = 0; i < N; ++i) {
        int j = assign[i];
        double w = exp(scores[i] - gmax[j]) / gsum[j];
        for (int c = 0; c < d; ++c) merged[(size_t)j * d + c] += w * f[(size_t)i * d + c];
        mxy[2 * j] += w * (double)xy[2 * i];
        mxy[2 * j + 1] += w * (double)xy[2 * i + 1];
    }
    free(gmax);
    free(gsum);
    return 0;
}

/*
 * Backward of the merge and of the scoring MLP for fixed anchors and assignment (both are
 * piecewise constant in the inputs).  With g_i = <dF_j, f_i> + <dX_j, x_i> for i in G_j:
 *   df_i = w_i dF_j + W1 dh_i,  dx_i = w_i dX_j,
 *   ds_i = w_i (g_i - sum_G w g),  dh_i = ds_i w2 * gelu'(z_i),
 *   dW1 = sum_i f_i dh_i^T, db1 = sum_i dh_i, dw2 = sum_i ds_i gelu(z_i), db2 = sum_i ds_i.
 * The scores are recomputed from the MLP.  Outputs are overwritten; dW1 ... db2 hold this
 * image's sums.
 */
int orc_merge_bwd(const double* f, const float* xy, int N, int d, const double* w1,
                  const double* b1, const double* w2, double b2, int h, int k,
                  const int32_t* assign, const double* dmerged, const double* dmxy,
                  double* df, double* dxy, double* dw1, double* db1, double* dw2, double* db2) {
    if (N < 1 || d < 1 || h < 1 || k < 1) return 1;
    double* s = (double*)malloc(sizeof(double) * (size_t)N);
    double* z = (double*)malloc(sizeof(double) * (size_t)N * h);
    double* g = (double*)malloc(sizeof(double) * (size_t)N);
    double* gmax = (double*)malloc(sizeof(double) * (size_t)k);
    double* gsum = (double*)calloc((size_t)k, sizeof(double));
    double* gws = (double*)calloc((size_t)k, sizeof(double));
    if (!s || !z || !g || !gmax || !gsum || !gws) {
        free(s); free(z); free(g); free(gmax); free(gsum); free(gws);
        return 2;
    }
    for (int i = 0; i < N; ++i) {
        double si = b2;
        for (int u = 0; u < h; ++u) {
            double zz = b1[u];
            for (int c = 0; c < d; ++c) zz += f[(size_t)i * d + c] * w1[(size_t)c * h + u];
            z[(size_t)i * h + u] = zz;
            si += w2[u] * gelu(zz);
        }
        s[i] = si;
    }
    for (int j = 0; j < k; ++j) gmax[j] = -INFINITY;
    for (int i = 0; i < N; ++i) if (s[i] > gmax[assign[i]]) gmax[assign[i]] = s[i];
    for (int i = 0; i < N; ++i) gsum[assign[i]] += exp(s[i] - gmax[assign[i]]);
    for (int i = 0; i < N; ++i) {
        int j = assign[i];
        double gi = dmxy[2 * j] * (double)xy[2 * i] + dmxy[2 * j + 1] * (double)xy[2 * i + 1];
        for (int c = 0; c < d; ++c) gi += dmerged[(size_t)j * d + c] * f[(size_t)i * d + c];
        g[i] = gi;
        gws[j] += exp(s[i] - gmax[j]) / gsum[j] * gi;
    }
    memset(dw1, 0, sizeof(double) * (size_t)d * h);
    memset(db1, 0, sizeof(double) * (size_t)h);
    memset(dw2, 0, sizeof(double) * (size_t)h);
    *db2 = 0.0;
    for (int i = 0; i < N; ++i) {
        int j = assign[i];
        double w = exp(s[i] - gmax[j]) / gsum[j];
        double ds = w * (g[i] - gws[j]);
        dxy[2 * i] = w * dmxy[2 * j];
        dxy[2 * i + 1] = w * dmxy[2 * j + 1];
        for (int c = 0; c < d; ++c) df[(size_t)i * d + c] = w * dmerged[(size_t)j * d + c];
        *db2 += ds;
        for (int u = 0; u < h; ++u) {
            double zz = z[(size_t)i * h + u];
            double dh = ds * w2[u] * gelu_grad(zz);
            dw2[u] += ds * gelu(zz);
            db1[u] += dh;
            for (int c = 0; c < d; ++c) {
                df[(size_t)i * d + c] += w1[(size_t)c * h + u] * dh;
                dw1[(size_t)c * h + u] += f[(size_t)i * d + c] * dh;
            }
        }
    }
    free(s); free(z); free(g); free(gmax); free(gsum); free(gws);
    return 0;
}

/*
 * Decoder layer (AFFMAE notes, "Key Designs" 2, the point-wise deformable cross-attention
 * decoder): every mask-token query, with feature f and reference position r, predicts a 2D
 * offset Delta = g(f), samples q = r + Delta, gathers the nearest visible tokens of an
 * encoder stage around q with distance-softmax weights (the KNN gather above), and the
 * decoder fuses the stages coarse to fine ("A Complete Example": stage 4 first, then stages
 * 3 to 1).  The notes fix no more; the readings taken:
 *   g is one linear map: Delta = f W_off + b_off, W_off [D][2], b_off [2];
 *   the gathered feature v (the stage's d channels) is projected to the decoder width and
 *   added to the query feature: f_out = f + v W_o, W_o [d][D] (a residual cross-attention
 *   update whose attention weights are the distance softmax).
 * Plain loops in fp64; every sum in index order.
 */
int orc_dec_offsets(const float* ref, const double* f, int Q, int D, const double* w_off,
                    const double* b_off, double* q) {
    if (Q < 0 || D < 1) return 1;
    for (int i = 0; i < Q; ++i)
        for (int j = 0; j < 2; ++j) {
            double acc = (double)ref[(size_t)i * 2 + j] + b_off[j];
            for (int c = 0; c < D; ++c) acc += f[(size_t)i * D + c] * w_off[(size_t)c * 2 + j];
            q[(size_t)i * 2 + j] = acc;
        }
    return 0;
}

int orc_dec_project(const double* f, const double* v, int Q, int D, int d, const double* w_o,
                    double* f_out) {
    if (Q < 0 || D < 1 || d < 1) return 1;
    /* f_out[i][n] = f[i][n] + sum over c in order of v[i][c] w_o[c][n]; rows of w_o read whole */
    for (int i = 0; i < Q; ++i) {
        double* out = f_out + (size_t)i * D;
        for (int n = 0; n < D; ++n) out[n] = f[(size_t)i * D + n];
        for (int c = 0; c < d; ++c) {
            const double a = v[(size_t)i * d + c];
            for (int n = 0; n < D; ++n) out[n] += a * w_o[(size_t)c * D + n];
        }
    }
    return 0;
}

/* dv = df_out W_o^T; dW_o += v^T df_out (accumulated, so images can be summed) */
int orc_dec_project_bwd(const double* v, const double* df_out, int Q, int D, int d,
                        const double* w_o, double* dv, double* dw_o) {
    if (Q < 0 || D < 1 || d < 1) return 1;
    for (int i = 0; i < Q; ++i)
        for (int c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int n = 0; n < D; ++n) acc += df_out[(size_t)i * D + n] * w_o[(size_t)c * D + n];
            dv[(size_t)i * d + c] = acc;
        }
    /* each dW_o[c][n] sums v[i][c] df_out[i][n] over i in order, then joins the running total */
    double* acc = (double*)calloc((size_t)d * D, sizeof(double));
    if (!acc) return 2;
    for (int i = 0; i < Q; ++i)
        for (int c = 0; c < d; ++c) {
            const double a = v[(size_t)i * d + c];
            double* row = acc + (size_t)c * D;
            for (int n = 0; n < D; ++n) row[n] += a * df_out[(size_t)i * D + n];
        }
    for (size_t x = 0; x < (size_t)d * D; ++x) dw_o[x] += acc[x];
    free(acc);
    return 0;
}

/* df_in = df_out + dq W_off^T (the residual path plus the offset head);
 * dW_off += f^T dq, db_off += sum_i dq_i (accumulated) */
int orc_dec_offsets_bwd(const double* f, const double* dq, const double* df_out, int Q, int D,
                        const double* w_off, double* df_in, double* dw_off, double* db_off) {
    if (Q < 0 || D < 1) return 1;
    for (int i = 0; i < Q; ++i)
        for (int c = 0; c < D; ++c)
            df_in[(size_t)i * D + c] = df_out[(size_t)i * D + c] +
                                       dq[(size_t)i * 2] * w_off[(size_t)c * 2] +
                                       dq[(size_t)i * 2 + 1] * w_off[(size_t)c * 2 + 1];
    for (int c = 0; c < D; ++c)
        for (int j = 0; j < 2; ++j) {
            double acc = 0.0;
            for (int i = 0; i < Q; ++i) acc += f[(size_t)i * D + c] * dq[(size_t)i * 2 + j];
            dw_off[(size_t)c * 2 + j] += acc;
        }
    for (int j = 0; j < 2; ++j) {
        double acc = 0.0;
        for (int i = 0; i < Q; ++i) acc += dq[(size_t)i * 2 + j];
        db_off[j] += acc;
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* batch drivers: images are independent (attention: image x head)           */
/* ------------------------------------------------------------------------ */

int orc_cluster_batch(const float* xy, int B, int N, int C, int32_t* clusters) {
    int G = (N + C - 1) / C, rc = 0;
    #pragma omp parallel for schedule(dynamic) reduction(|:rc)
    for (int b = 0; b < B; ++b)
        rc |= orc_cluster(xy + (size_t)b * N * 2, N, C, clusters + (size_t)b * G * C);
    return rc;
}

int orc_neighbors_batch(const float* xy, const int32_t* clusters, int B, int N, int C,
                        int M, int32_t* nbr) {
    int G = (N + C - 1) / C, rc = 0;
    #pragma omp parallel for schedule(dynamic) reduction(|:rc)
    for (int b = 0; b < B; ++b)
        rc |= orc_neighbors(xy + (size_t)b * N * 2, clusters + (size_t)b * G * C, N, C, M,
                            nbr + (size_t)b * G * M);
    return rc;
}

int orc_attn_fwd_batch(const double* q, const double* k, const double* v, const float* xy,
                       const int32_t* clusters, const int32_t* nbr, const double* bias,
                       int B, int N, int H, int D, int C, int M, double scale,
                       double* o, double* lse) {
    int G = (N + C - 1) / C, rc = 0;
    size_t st = (size_t)N * H * D;
    #pragma omp parallel for collapse(2) schedule(dynamic) reduction(|:rc)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h)
            rc |= attn_fwd_heads(q + b * st, k + b * st, v + b * st, xy + (size_t)b * N * 2,
                                 clusters + (size_t)b * G * C, nbr + (size_t)b * G * M, bias,
                                 N, H, D, C, M, scale, h, h + 1, o + b * st,
                                 lse + (size_t)b * N * H);
    return rc;
}

/* dbias sums the images' partial sums in image order, after the parallel loop. */
int orc_attn_bwd_batch(const double* q, const double* k, const double* v, const float* xy,
                       const int32_t* clusters, const int32_t* nbr, const double* bias,
                       int B, int N, int H, int D, int C, int M, double scale,
                       const double* dout, double* dq, double* dk, double* dv,
                       double* dbias) {
    int G = (N + C - 1) / C, rc = 0;
    size_t st = (size_t)N * H * D;
    double* part = (double*)calloc((size_t)B * H * 3, sizeof(double));
    if (!part) return 2;
    #pragma omp parallel for collapse(2) schedule(dynamic) reduction(|:rc)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h)
            rc |= attn_bwd_heads(q + b * st, k + b * st, v + b * st, xy + (size_t)b * N * 2,
                                 clusters + (size_t)b * G * C, nbr + (size_t)b * G * M, bias,
                                 N, H, D, C, M, scale, h, h + 1, dout + b * st, dq + b * st,
                                 dk + b * st, dv + b * st, part + (size_t)b * H * 3);
    for (int j = 0; j < H * 3; ++j) {
        double acc = 0.0;
        for (int b = 0; b < B; ++b) acc += part[(size_t)b * H * 3 + j];
        dbias[j] = acc;
    }
    free(part);
    return rc;
}

int orc_knn_table_batch(const float* xy, int B, int N, int GH, int GW, int K,
                        int32_t* table) {
    int rc = 0;
    #pragma omp parallel for schedule(dynamic) reduction(|:rc)
    for (int b = 0; b < B; ++b)
        rc |= orc_knn_table(xy + (size_t)b * N * 2, N, GH, GW, K,
                            table + (size_t)b * GH * GW * K);
    return rc;
}

int orc_knn_fwd_batch(const float* queries, int B, int Q, const double* feats,
                      const float* xy, int N, int d, const int32_t* table, int GH, int GW,
                      int K, const double* p, int kind, double* out) {
    int rc = 0;
    #pragma omp parallel for schedule(dynamic) reduction(|:rc)
    for (int b = 0; b < B; ++b)
        rc |= orc_knn_fwd(queries + (size_t)b * Q * 2, Q, feats + (size_t)b * N * d,
                          xy + (size_t)b * N * 2, N, d, table + (size_t)b * GH * GW * K,
                          GH, GW, K, p, kind, out + (size_t)b * Q * d);
    return rc;
}

int orc_knn_bwd_batch(const float* queries, int B, int Q, const double* feats,
                      const float* xy, int N, int d, const int32_t* table, int GH, int GW,
                      int K, const double* p, int kind, const double* dout, double* dfeats,
                      double* dq, double* dp) {
    int rc = 0, nh = d / 32;
    double* part = (double*)calloc((size_t)B * nh, sizeof(double));
    if (!part) return 2;
    #pragma omp parallel for schedule(dynamic) reduction(|:rc)
    for (int b = 0; b < B; ++b)
        rc |= orc_knn_bwd(queries + (size_t)b * Q * 2, Q, feats + (size_t)b * N * d,
                          xy + (size_t)b * N * 2, N, d, table + (size_t)b * GH * GW * K,
                          GH, GW, K, p, kind, dout + (size_t)b * Q * d, dfeats + (size_t)b * N * d,
                          dq + (size_t)b * Q * 2, part + (size_t)b * nh);
    for (int h = 0; h < nh; ++h) {
        double acc = 0.0;
        for (int b = 0; b < B; ++b) acc += part[(size_t)b * nh + h];
        dp[h] = acc;
    }
    free(part);
    return rc;
}

int orc_token_order_batch(const float* xy, int B, int N, int GH, int GW, int32_t* perm) {
    int rc = 0;
    #pragma omp parallel for schedule(dynamic) reduction(|:rc)
    for (int b = 0; b < B; ++b)
        rc |= orc_token_order(xy + (size_t)b * N * 2, N, GH, GW, perm + (size_t)b * N);
    return rc;
}
