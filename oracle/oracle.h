/*
 * oracle.h -- declarations of the fp64 CPU reference (test infrastructure only;
 * the CUDA library neither includes nor links it).  Per-image functions take one
 * image; the *_batch drivers loop over B independent images (OpenMP).  Layouts:
 * xy [N][2] fp32 (x = column, y = row, grid-cell units); q/k/v/o/dout [N][H][D];
 * lse [N][H]; bias [H][3] = (a_h, b_h, c_h); clusters [G][C]; nbr [G][M];
 * table [GH][GW][K]; queries [Q][2]; feats/dfeats [N][d]; out/dout [Q][d];
 * p [d/32].  Return 0 on success, 1 on bad arguments, 2 on allocation failure.
 */
#ifndef ORACLE_H
#define ORACLE_H
#include <stdint.h>

int orc_set_threads(int n);
int orc_cluster(const float* xy, int N, int C, int32_t* clusters);
int orc_neighbors(const float* xy, const int32_t* clusters, int N, int C, int M, int32_t* nbr);
int orc_attn_fwd(const double* q, const double* k, const double* v, const float* xy,
                 const int32_t* clusters, const int32_t* nbr, const double* bias,
                 int N, int H, int D, int C, int M, double scale, double* o, double* lse);
int orc_attn_bwd(const double* q, const double* k, const double* v, const float* xy,
                 const int32_t* clusters, const int32_t* nbr, const double* bias,
                 int N, int H, int D, int C, int M, double scale, const double* dout,
                 double* dq, double* dk, double* dv, double* dbias);
int orc_knn_table(const float* xy, int N, int GH, int GW, int K, int32_t* table);
/* kind: 0 = exponential kernel softmax(-p d), 1 = inverse power d^-p / sum d^-p */
int orc_knn_fwd(const float* queries, int Q, const double* feats, const float* xy,
                int N, int d, const int32_t* table, int GH, int GW, int K,
                const double* p, int kind, double* out);
int orc_knn_bwd(const float* queries, int Q, const double* feats, const float* xy,
                int N, int d, const int32_t* table, int GH, int GW, int K,
                const double* p, int kind, const double* dout, double* dfeats, double* dq,
                double* dp);

/* token ids in Z-order of their cells on the GH x GW grid, ties by id */
int orc_token_order(const float* xy, int N, int GH, int GW, int32_t* perm);

/* token merging: MLP scores, top-k anchors + nearest-anchor assignment, merge, backward */
int orc_merge_scores(const double* f, int N, int d, const double* w1, const double* b1,
                     const double* w2, double b2, int h, double* scores);
int orc_merge_select(const double* scores, const float* xy, int N, int k, int32_t* anchors,
                     int32_t* assign);
int orc_merge_fwd(const double* f, const float* xy, int N, int d, const double* scores, int k,
                  const int32_t* assign, double* merged, double* mxy);
int orc_merge_bwd(const double* f, const float* xy, int N, int d, const double* w1,
                  const double* b1, const double* w2, double b2, int h, int k,
                  const int32_t* assign, const double* dmerged, const double* dmxy,
                  double* df, double* dxy, double* dw1, double* db1, double* dw2, double* db2);

int orc_cluster_batch(const float* xy, int B, int N, int C, int32_t* clusters);
int orc_neighbors_batch(const float* xy, const int32_t* clusters, int B, int N, int C,
                        int M, int32_t* nbr);
int orc_attn_fwd_batch(const double* q, const double* k, const double* v, const float* xy,
                       const int32_t* clusters, const int32_t* nbr, const double* bias,
                       int B, int N, int H, int D, int C, int M, double scale,
                       double* o, double* lse);
int orc_attn_bwd_batch(const double* q, const double* k, const double* v, const float* xy,
                       const int32_t* clusters, const int32_t* nbr, const double* bias,
                       int B, int N, int H, int D, int C, int M, double scale,
                       const double* dout, double* dq, double* dk, double* dv, double* dbias);
int orc_knn_table_batch(const float* xy, int B, int N, int GH, int GW, int K, int32_t* table);
int orc_knn_fwd_batch(const float* queries, int B, int Q, const double* feats,
                      const float* xy, int N, int d, const int32_t* table, int GH, int GW,
                      int K, const double* p, int kind, double* out);
int orc_knn_bwd_batch(const float* queries, int B, int Q, const double* feats,
                      const float* xy, int N, int d, const int32_t* table, int GH, int GW,
                      int K, const double* p, int kind, const double* dout, double* dfeats,
                      double* dq, double* dp);
int orc_token_order_batch(const float* xy, int B, int N, int GH, int GW, int32_t* perm);

/* decoder layer: offsets q = r + f W_off + b_off, projection f_out = f + v W_o, backward */
int orc_dec_offsets(const float* ref, const double* f, int Q, int D, const double* w_off,
                    const double* b_off, double* q);
int orc_dec_project(const double* f, const double* v, int Q, int D, int d, const double* w_o,
                    double* f_out);
int orc_dec_project_bwd(const double* v, const double* df_out, int Q, int D, int d,
                        const double* w_o, double* dv, double* dw_o);
int orc_dec_offsets_bwd(const double* f, const double* dq, const double* df_out, int Q, int D,
                        const double* w_off, double* df_in, double* dw_off, double* db_off);
#endif
