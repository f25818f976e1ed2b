/*
 * pariskv_oracle.h -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, single-threaded CPU restatement of ParisKV's decode-time
 * KV-cache retrieval (normalise + SRHT rotate, PolarANN sign-pattern codes,
 * multi-tier collision voting, integer Top-C, 4-bit RSQ-IP rerank, Top-k and
 * exact softmax attention over the selected rows).  It exists so that tests,
 * the smoke check and the CPU baseline of the benchmark can check the CUDA
 * library against an independent implementation.  It shares no code, header,
 * table or constant with the CUDA library and must never be called by it.
 *
 * Sources (page title, then section/equation/table on that page):
 *   [slides]  "ParisKV: Fast and Drift-Robust KV-Cache Retrieval" (reading of
 *             arXiv 2602.07721v3), frames for Sec. 3 Eqs. (1)-(3), Sec. 4.1.1-4.1.2
 *             Eqs. (5)-(6), Prop. 4.1 / App. B.1, Sec. 4.2.2 / App. B.2.1 Eq. (15),
 *             Eqs. (7)-(10) / App. B.2.2, Sec. 4.3.
 *   [readme]  "ParisKV" GitHub README (amy-77/ParisKV): pipeline prose, the
 *             parameter table and the adaptive ratio table.
 *
 * Floating point: the encode and query-preparation steps decide integers
 * (codes, level indices, bucket ranks), so they run in IEEE fp32 in one fixed
 * operation order (compile with -ffp-contract=off, no fast-math).  Scores and
 * attention are computed in fp64 from the stored fp32 values.
 */
#ifndef PARISKV_ORACLE_H
#define PARISKV_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- SRHT sign source ------------------------------------------------ */
/* First output of Vigna's splitmix64 generator whose state is x. */
uint64_t or_splitmix64(uint64_t x);
/* s_j = +1 when bit 63 of splitmix64(seed*D + j) is 0, else -1. */
void or_srht_signs(uint64_t seed, int D, int8_t *signs);

/* ---- magnitude prior and Lloyd-Max levels (slides, Prop. 4.1 / App. B.1) */
/* Density of y = |(u_b)_j| when (u_b)_j^2 ~ Beta(1/2,(m-1)/2), on [0,1]. */
double or_magnitude_density(int m, double y);
/* fp64 Lloyd-Max fixed point with L levels; returns iterations, -1 if no
 * convergence.  thresholds[t] = (levels[t]+levels[t+1])/2, t < L-1. */
int or_lloyd_max(int m, int L, double *levels, double *thresholds);
/* The same, rounded to fp32 (levels and midpoints rounded separately). */
int or_levels_f32(int m, int L, float *lev32, float *thr32);

/* ---- canonical fp32 normalise + rotate (slides, Eq. 5) --------------- */
/* xt = R (x / ||x||), R = H_D diag(s) / sqrt(D); returns ||x|| in fp32.
 * A zero vector gives ||x|| = 0 and xt = 0. */
float or_rotate(const float *x, int D, const int8_t *signs, float *xt);

/* ---- key encoding (slides, Eqs. 6-10) -------------------------------- */
/* For n keys of dimension D split into B = D/m blocks:
 *   codes[i*B+b]   sign-pattern centroid id (bit j set iff u_{i,b,j} < 0)
 *   tidx[i*D+j]    magnitude level index t in [0, L)   (quantize != 0)
 *   w[i*B+b]       ||k_i|| r_{i,b} / alpha_{i,b}
 *   occ[b*2^m+c]   += number of keys with code c in block b
 * Optional (nullable) debug outputs: knorm[i], rb[i*B+b], u[i*D+j].
 * quantize == 0 is the "no quantisation" limit v = u (alpha = <u,u>). */
void or_encode_keys(const float *K, int64_t n, int D, int m, const int8_t *signs,
                    const float *lev32, const float *thr32, int L, int quantize,
                    uint16_t *codes, uint16_t *tidx, float *w, uint32_t *occ,
                    float *knorm, float *rb, float *u);

/* ---- Stage I: bucket tiers and collision counts (slides, Sec. 4.2.2, Eq. 15) */
/* lut[b*2^m+c] = sum_j (bit_j(c) ? -qt_{b,j} : +qt_{b,j}) (fp32, j ascending);
 * buckets ranked by (lut desc, c asc); P(c) = keys in earlier buckets;
 * bonus = 6 - floor(6 P / R) when P < R, else 0. */
void or_bonus_from_qt(const float *qt, int D, int m, const uint32_t *occ, int64_t R,
                      float *lut, uint8_t *bonus);
/* q_agg = ((q_0 + q_1) + ...) + q_{G-1}; qt = rotate(q_agg); then bonus. */
void or_query_prep(const float *q, int G, int D, int m, const int8_t *signs,
                   const uint32_t *occ, int64_t R, float *qt, float *qnorm,
                   float *lut, uint8_t *bonus);
/* S_i = sum_b bonus[b][codes[i][b]]. */
void or_collision(const uint16_t *codes, int64_t n, int D, int m, const uint8_t *bonus,
                  uint8_t *S);
/* Top-C by (S desc, index asc); written in ascending index order; returns C. */
int64_t or_candidates(const uint8_t *S, int64_t n, int64_t C, int32_t *cand);

/* ---- Stage II: 4-bit estimator and Top-k (slides, Eqs. 7-10) ---------- */
/* v[i*D+j] = sigma_{i,j} * lev32[tidx] (fp64 copy of the fp32 level). */
void or_dequantize(const uint16_t *codes, const uint16_t *tidx, const float *lev32,
                   int64_t n, int D, int m, double *v);
/* est_c = qnorm * sum_b w_{i,b} * <v_{i,b}, qt_b>, i = cand[c], in fp64. */
void or_rerank(const int32_t *cand, int64_t C, const double *v, const float *w,
               int D, int m, const float *qt, float qnorm, double *est);
/* Top-k of (est desc, index asc); idx/score in that order. */
void or_topk(const int32_t *cand, const double *est, int64_t C, int k,
             int32_t *idx, double *score);

/* ---- exact attention over the selected rows (slides, Sec. 3 Eqs. 1-3) - */
/* o[g*D+d] = sum_r softmax_r(scale <q_g, K[idx_r]>) V[idx_r][d], fp64. */
void or_attend(const float *q, int G, int D, const float *K, const float *V,
               const int32_t *idx, int k, double scale, double *o);

/* ---- parameters (readme, adaptive ratio table) ------------------------ */
/* Candidate ratio beta and collision ratio rho for a retrieval zone of n keys. */
void or_ratio_table(int64_t n, double *beta, double *rho);
/* C = cand_budget or ceil(beta n); C = min(max(C, topk), n);
 * R = ceil(rho n) with rho = collision_ratio or the table's; 1 <= R <= n. */
void or_resolve(int64_t n, int64_t cand_budget, float collision_ratio, int topk,
                int64_t *C, int64_t *R);

#ifdef __cplusplus
}
#endif
#endif
