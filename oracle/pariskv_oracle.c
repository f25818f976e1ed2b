/*
 * pariskv_oracle.c -- TEST INFRASTRUCTURE ONLY (see pariskv_oracle.h).
 *
 * Plain, slow, obviously-correct CPU restatement of the ParisKV retrieval
 * path.  Build with:  gcc -O2 -std=c11 -ffp-contract=off -fPIC -shared -lm
 * (no -ffast-math: every fp32 step below is one IEEE round-to-nearest op).
 */
#include "pariskv_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ===================================================================== */
/* SRHT signs.  The pages state only that one orthogonal transform, an     */
/* SRHT, is shared by all keys (slides, Sec. 4.1.1, Eq. 5).  Reading: the   */
/* square SRHT H_D diag(s) / sqrt(D) with a seeded +-1 diagonal.  The       */
/* diagonal is drawn from splitmix64 (Vigna), counter-based per coordinate. */
/* ===================================================================== */
uint64_t or_splitmix64(uint64_t x)
{
    uint64_t z = x + 0x9e3779b97f4a7c15ULL;
    z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ULL;
    z = (z ^ (z >> 27)) * 0x94d049bb133111ebULL;
    return z ^ (z >> 31);
}

void or_srht_signs(uint64_t seed, int D, int8_t *signs)
{
    for (int j = 0; j < D; j++) {
        uint64_t r = or_splitmix64(seed * (uint64_t)D + (uint64_t)j);
        signs[j] = (r >> 63) ? (int8_t)-1 : (int8_t)1;
    }
}

/* ===================================================================== */
/* Magnitude prior (slides, Prop. 4.1 and App. B.1): for a Haar-rotated unit */
/* vector, (u_b)_j^2 ~ Beta(1/2, (m-1)/2).  Then y = |(u_b)_j| has density  */
/*   f(y) = 2 (1 - y^2)^((m-3)/2) / B(1/2, (m-1)/2),  0 <= y <= 1.           */
/* The 3-bit magnitude levels are the Lloyd-Max quantiser of f (slides,     */
/* same section; the readme ships a script that rebuilds the 8 levels).    */
/* Reading: the exact-density fixed point, found by adaptive Simpson        */
/* quadrature in fp64 and Lloyd's centroid / midpoint iteration.            */
/* ===================================================================== */
static double beta_fn(double a, double b)
{
    return exp(lgamma(a) + lgamma(b) - lgamma(a + b));
}

double or_magnitude_density(int m, double y)
{
    if (y < 0.0 || y > 1.0) return 0.0;
    double t = 1.0 - y * y;
    double a = 0.5 * (double)(m - 3);
    double un = (t <= 0.0) ? (a == 0.0 ? 1.0 : 0.0) : pow(t, a);
    return 2.0 * un / beta_fn(0.5, 0.5 * (double)(m - 1));
}

/* integrand selector: moment 0 -> f, moment 1 -> y f (unnormalised) */
static double integrand(int m, int moment, double y)
{
    double t = 1.0 - y * y;
    double a = 0.5 * (double)(m - 3);
    double un = (t <= 0.0) ? (a == 0.0 ? 1.0 : 0.0) : pow(t, a);
    return moment ? y * un : un;
}

static double simpson_rec(int m, int mom, double a, double b, double fa, double fm, double fb,
                          double whole, double eps, int depth)
{
    double c = 0.5 * (a + b);
    double l = 0.5 * (a + c), r = 0.5 * (c + b);
    double fl = integrand(m, mom, l), fr = integrand(m, mom, r);
    double left = (c - a) / 6.0 * (fa + 4.0 * fl + fm);
    double right = (b - c) / 6.0 * (fm + 4.0 * fr + fb);
    double diff = left + right - whole;
    if (depth <= 0 || fabs(diff) <= 15.0 * eps)
        return left + right + diff / 15.0;
    return simpson_rec(m, mom, a, c, fa, fl, fm, left, 0.5 * eps, depth - 1) +
           simpson_rec(m, mom, c, b, fm, fr, fb, right, 0.5 * eps, depth - 1);
}

static double integrate(int m, int mom, double a, double b)
{
    if (b <= a) return 0.0;
    double fa = integrand(m, mom, a), fb = integrand(m, mom, b);
    double c = 0.5 * (a + b), fm = integrand(m, mom, c);
    double whole = (b - a) / 6.0 * (fa + 4.0 * fm + fb);
    return simpson_rec(m, mom, a, b, fa, fm, fb, whole, 1e-17, 48);
}

int or_lloyd_max(int m, int L, double *levels, double *thresholds)
{
    if (m < 3 || L < 2) return -1;
    double *lev = (double *)malloc(sizeof(double) * (size_t)L);
    double *thr = (double *)malloc(sizeof(double) * (size_t)(L - 1));
    for (int t = 0; t < L; t++) lev[t] = ((double)t + 0.5) / (double)L;
    int it, done = 0;
    for (it = 1; it <= 200000 && !done; it++) {
        for (int t = 0; t < L - 1; t++) thr[t] = 0.5 * (lev[t] + lev[t + 1]);
        double delta = 0.0;
        for (int t = 0; t < L; t++) {
            double a = (t == 0) ? 0.0 : thr[t - 1];
            double b = (t == L - 1) ? 1.0 : thr[t];
            double num = integrate(m, 1, a, b);
            double den = integrate(m, 0, a, b);
            double nv = num / den;
            double d = fabs(nv - lev[t]);
            if (d > delta) delta = d;
            lev[t] = nv;
        }
        if (delta < 1e-15) done = 1;
    }
    for (int t = 0; t < L - 1; t++) thr[t] = 0.5 * (lev[t] + lev[t + 1]);
    memcpy(levels, lev, sizeof(double) * (size_t)L);
    memcpy(thresholds, thr, sizeof(double) * (size_t)(L - 1));
    free(lev);
    free(thr);
    return done ? it - 1 : -1;
}

int or_levels_f32(int m, int L, float *lev32, float *thr32)
{
    double *lev = (double *)malloc(sizeof(double) * (size_t)L);
    double *thr = (double *)malloc(sizeof(double) * (size_t)(L - 1));
    int it = or_lloyd_max(m, L, lev, thr);
    for (int t = 0; t < L; t++) lev32[t] = (float)lev[t];
    for (int t = 0; t < L - 1; t++) thr32[t] = (float)thr[t];
    free(lev);
    free(thr);
    return it;
}

/* ===================================================================== */
/* Normalise + rotate (slides, Sec. 4.1.1, Eq. 5): k^ = k/||k||,           */
/* k~ = R k^.  Canonical fp32 sequence (the pages give no operation order; */
/* this order is the reading both implementations follow):                 */
/*   (i)   s_j = x_j*x_j; for h = D/2 .. 1: s_j = s_j + s_{j+h} (j < h);    */
/*         ||x|| = sqrt(s_0)                                                */
/*   (ii)  y_j = x_j / ||x||                                                */
/*   (iii) y_j = s_j * y_j           (diag(s): a sign flip, exact)          */
/*   (iv)  Walsh-Hadamard butterflies for h = 1, 2, .., D/2:                */
/*         (y_j, y_{j+h}) = (y_j + y_{j+h}, y_j - y_{j+h}) for bit h of j 0  */
/*   (v)   y_j = y_j * c,  c = fp32(1/sqrt(D))                              */
/* ===================================================================== */
float or_rotate(const float *x, int D, const int8_t *signs, float *xt)
{
    float s[1024];
    if (D < 1 || D > 1024) return 0.0f;
    for (int j = 0; j < D; j++) s[j] = x[j] * x[j];
    for (int h = D / 2; h >= 1; h >>= 1)
        for (int j = 0; j < h; j++) s[j] = s[j] + s[j + h];
    float nrm = sqrtf(s[0]);
    if (nrm == 0.0f) {
        for (int j = 0; j < D; j++) xt[j] = 0.0f;
        return 0.0f;
    }
    for (int j = 0; j < D; j++) {
        float y = x[j] / nrm;
        xt[j] = (signs[j] < 0) ? -y : y;
    }
    for (int h = 1; h < D; h <<= 1)
        for (int j = 0; j < D; j++)
            if ((j & h) == 0) {
                float a = xt[j], b = xt[j + h];
                xt[j] = a + b;
                xt[j + h] = a - b;
            }
    float c = (float)(1.0 / sqrt((double)D));
    for (int j = 0; j < D; j++) xt[j] = xt[j] * c;
    return nrm;
}

/* sum of v[0..len) by the halving tree (len a power of two), fp32 */
static float tree_sum(float *v, int len)
{
    for (int h = len / 2; h >= 1; h >>= 1)
        for (int j = 0; j < h; j++) v[j] = v[j] + v[j + h];
    return v[0];
}

/* ===================================================================== */
/* Key encoding.  Block split D = B m (slides, Sec. 4.1.2 and the notation */
/* errata, which fix D as B times m).  Per block (slides, Eqs. 6-10):       */
/*   r_b = ||k~_b||, u_b = k~_b / r_b                                       */
/*   c_b = argmax_{w in {+-1/sqrt m}^m} <u_b, w>  = sign pattern of u_b     */
/*         (bit j set iff u_j < 0; u_j = 0 counts as +, lowest id on ties)  */
/*   t_j = #{t : |u_j| > theta_t}  (nearest Lloyd-Max level, ties low)      */
/*   v_j = sigma_j l_{t_j}   (raw levels: the estimate is scale-invariant   */
/*         in v because alpha divides it out)                               */
/*   alpha_b = <v_b, u_b> = sum_j l_{t_j} |u_j|  (tree order)               */
/*   w_b = (||k|| r_b) / alpha_b                                            */
/* A zero key or zero block encodes as code 0, levels 0, weight 0.          */
/* ===================================================================== */
void or_encode_keys(const float *K, int64_t n, int D, int m, const int8_t *signs,
                    const float *lev32, const float *thr32, int L, int quantize,
                    uint16_t *codes, uint16_t *tidx, float *w, uint32_t *occ,
                    float *knorm, float *rb, float *u)
{
    const int B = D / m;
    const int NC = 1 << m;
    float kt[1024], uu[1024], tmp[64];
    for (int64_t i = 0; i < n; i++) {
        const float *k = K + i * D;
        float nk = or_rotate(k, D, signs, kt);
        if (knorm) knorm[i] = nk;
        for (int b = 0; b < B; b++) {
            const float *x = kt + b * m;
            for (int j = 0; j < m; j++) tmp[j] = x[j] * x[j];
            float r = sqrtf(tree_sum(tmp, m));
            if (rb) rb[i * B + b] = r;
            uint16_t code = 0;
            if (nk == 0.0f || r == 0.0f) {
                codes[i * B + b] = 0;
                if (quantize && tidx)
                    for (int j = 0; j < m; j++) tidx[i * D + b * m + j] = 0;
                for (int j = 0; j < m; j++) uu[b * m + j] = 0.0f;
                w[i * B + b] = 0.0f;
                occ[(int64_t)b * NC + 0] += 1;
                continue;
            }
            for (int j = 0; j < m; j++) {
                uu[b * m + j] = x[j] / r;
                if (uu[b * m + j] < 0.0f) code |= (uint16_t)(1u << j);
            }
            codes[i * B + b] = code;
            occ[(int64_t)b * NC + code] += 1;
            float alpha;
            if (quantize) {
                for (int j = 0; j < m; j++) {
                    float a = fabsf(uu[b * m + j]);
                    int t = 0;
                    for (int q = 0; q < L - 1; q++)
                        if (a > thr32[q]) t++;
                    tidx[i * D + b * m + j] = (uint16_t)t;
                    tmp[j] = lev32[t] * a;
                }
                alpha = tree_sum(tmp, m);
            } else {
                for (int j = 0; j < m; j++) tmp[j] = uu[b * m + j] * uu[b * m + j];
                alpha = tree_sum(tmp, m);
            }
            w[i * B + b] = (nk * r) / alpha;
        }
        if (u)
            for (int j = 0; j < D; j++) u[i * D + j] = uu[j];
    }
}

/* ===================================================================== */
/* Stage I (slides, Sec. 4.2.2 and App. B.2.1 Eq. 15; readme, pipeline     */
/* step 2: per subspace the centroids nearest the query vote for keys):     */
/*   per block, keep the top-rho fraction of keys ranked by the score of    */
/*   their assigned centre; split it into six percentile tiers with bonuses */
/*   6..1;  S_i = sum_b 1{i in T_b(rho)} w_{l(i,b)}.                        */
/* Readings: keys of one bucket share a score, so tiers are decided per     */
/* bucket: buckets in (score desc, id asc) order, P(c) = keys in earlier    */
/* buckets, bucket active iff P(c) < R = ceil(rho n), tier floor(6 P / R).  */
/* The centre score <q~_b, w_c> is ranked without its 1/sqrt(m) factor.     */
/* ===================================================================== */
typedef struct { float l; int c; } bucket_t;

static int cmp_bucket(const void *pa, const void *pb)
{
    const bucket_t *a = (const bucket_t *)pa, *b = (const bucket_t *)pb;
    if (a->l > b->l) return -1;
    if (a->l < b->l) return 1;
    return (a->c < b->c) ? -1 : (a->c > b->c);
}

void or_bonus_from_qt(const float *qt, int D, int m, const uint32_t *occ, int64_t R,
                      float *lut, uint8_t *bonus)
{
    const int B = D / m;
    const int NC = 1 << m;
    bucket_t *bk = (bucket_t *)malloc(sizeof(bucket_t) * (size_t)NC);
    for (int b = 0; b < B; b++) {
        for (int c = 0; c < NC; c++) {
            float L = 0.0f;
            for (int j = 0; j < m; j++) {
                float x = qt[b * m + j];
                L = L + (((c >> j) & 1) ? -x : x);
            }
            lut[b * NC + c] = L;
            bk[c].l = L;
            bk[c].c = c;
        }
        qsort(bk, (size_t)NC, sizeof(bucket_t), cmp_bucket);
        int64_t P = 0;
        for (int r = 0; r < NC; r++) {
            int c = bk[r].c;
            uint8_t bon = 0;
            if (P < R) bon = (uint8_t)(6 - (int)((6 * P) / R));
            bonus[b * NC + c] = bon;
            P += occ[(int64_t)b * NC + c];
        }
    }
    free(bk);
}

void or_query_prep(const float *q, int G, int D, int m, const int8_t *signs,
                   const uint32_t *occ, int64_t R, float *qt, float *qnorm,
                   float *lut, uint8_t *bonus)
{
    float qa[1024];
    for (int j = 0; j < D; j++) {
        float a = q[j];
        for (int g = 1; g < G; g++) a = a + q[(int64_t)g * D + j];
        qa[j] = a;
    }
    *qnorm = or_rotate(qa, D, signs, qt);
    or_bonus_from_qt(qt, D, m, occ, R, lut, bonus);
}

void or_collision(const uint16_t *codes, int64_t n, int D, int m, const uint8_t *bonus,
                  uint8_t *S)
{
    const int B = D / m;
    const int NC = 1 << m;
    for (int64_t i = 0; i < n; i++) {
        int s = 0;
        for (int b = 0; b < B; b++) s += bonus[b * NC + codes[i * B + b]];
        S[i] = (uint8_t)s;
    }
}

/* Top-C of S (slides, Sec. 4.2.2: the keys with the largest S_i; Sec.    */
/* 4.3: C = ceil(beta n)).  Tie rule: higher S, then lower index.           */
typedef struct { int s; int32_t i; } sidx_t;

static int cmp_sidx(const void *pa, const void *pb)
{
    const sidx_t *a = (const sidx_t *)pa, *b = (const sidx_t *)pb;
    if (a->s != b->s) return (a->s > b->s) ? -1 : 1;
    return (a->i < b->i) ? -1 : (a->i > b->i);
}

static int cmp_i32(const void *pa, const void *pb)
{
    int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return (a < b) ? -1 : (a > b);
}

int64_t or_candidates(const uint8_t *S, int64_t n, int64_t C, int32_t *cand)
{
    if (C > n) C = n;
    sidx_t *v = (sidx_t *)malloc(sizeof(sidx_t) * (size_t)(n > 0 ? n : 1));
    for (int64_t i = 0; i < n; i++) {
        v[i].s = S[i];
        v[i].i = (int32_t)i;
    }
    qsort(v, (size_t)n, sizeof(sidx_t), cmp_sidx);
    for (int64_t c = 0; c < C; c++) cand[c] = v[c].i;
    qsort(cand, (size_t)C, sizeof(int32_t), cmp_i32);
    free(v);
    return C;
}

/* ===================================================================== */
/* Stage II (slides, Eqs. 7-10 / App. B.2.2):                              */
/*   <k_i, q>^ = ||q|| sum_b w_{i,b} <v_{i,b}, q~_b>                       */
/* evaluated in fp64 from the stored fp32 values.                           */
/* ===================================================================== */
void or_dequantize(const uint16_t *codes, const uint16_t *tidx, const float *lev32,
                   int64_t n, int D, int m, double *v)
{
    const int B = D / m;
    for (int64_t i = 0; i < n; i++)
        for (int b = 0; b < B; b++) {
            int code = codes[i * B + b];
            for (int j = 0; j < m; j++) {
                double l = (double)lev32[tidx[i * D + b * m + j]];
                v[i * D + b * m + j] = ((code >> j) & 1) ? -l : l;
            }
        }
}

void or_rerank(const int32_t *cand, int64_t C, const double *v, const float *w,
               int D, int m, const float *qt, float qnorm, double *est)
{
    const int B = D / m;
    for (int64_t c = 0; c < C; c++) {
        int64_t i = cand[c];
        double acc = 0.0;
        for (int b = 0; b < B; b++) {
            double dot = 0.0;
            for (int j = 0; j < m; j++)
                dot += v[i * D + b * m + j] * (double)qt[b * m + j];
            acc += (double)w[i * B + b] * dot;
        }
        est[c] = (double)qnorm * acc;
    }
}

typedef struct { double e; int32_t i; } eidx_t;

static int cmp_eidx(const void *pa, const void *pb)
{
    const eidx_t *a = (const eidx_t *)pa, *b = (const eidx_t *)pb;
    if (a->e != b->e) return (a->e > b->e) ? -1 : 1;
    return (a->i < b->i) ? -1 : (a->i > b->i);
}

void or_topk(const int32_t *cand, const double *est, int64_t C, int k,
             int32_t *idx, double *score)
{
    eidx_t *v = (eidx_t *)malloc(sizeof(eidx_t) * (size_t)(C > 0 ? C : 1));
    for (int64_t c = 0; c < C; c++) {
        v[c].e = est[c];
        v[c].i = cand[c];
    }
    qsort(v, (size_t)C, sizeof(eidx_t), cmp_eidx);
    for (int r = 0; r < k && r < C; r++) {
        idx[r] = v[r].i;
        score[r] = v[r].e;
    }
    free(v);
}

/* ===================================================================== */
/* Attention over the selected rows (slides, Sec. 3, Eqs. 1-3:             */
/* s_i = <k_i, q>, o = sum softmax(s)_i v_i, recomputed with full-precision */
/* K/V).  Reading: a scale factor (default 1/sqrt(D), standard decode       */
/* attention); scale = 1 is the printed formula.                            */
/* ===================================================================== */
void or_attend(const float *q, int G, int D, const float *K, const float *V,
               const int32_t *idx, int k, double scale, double *o)
{
    double *s = (double *)malloc(sizeof(double) * (size_t)(k > 0 ? k : 1));
    for (int g = 0; g < G; g++) {
        const float *qg = q + (int64_t)g * D;
        double mx = -INFINITY;
        for (int r = 0; r < k; r++) {
            const float *kr = K + (int64_t)idx[r] * D;
            double d = 0.0;
            for (int j = 0; j < D; j++) d += (double)qg[j] * (double)kr[j];
            s[r] = scale * d;
            if (s[r] > mx) mx = s[r];
        }
        double den = 0.0;
        for (int r = 0; r < k; r++) {
            s[r] = exp(s[r] - mx);
            den += s[r];
        }
        for (int j = 0; j < D; j++) {
            double acc = 0.0;
            for (int r = 0; r < k; r++) acc += s[r] * (double)V[(int64_t)idx[r] * D + j];
            o[(int64_t)g * D + j] = acc / den;
        }
    }
    free(s);
}

/* ===================================================================== */
/* Adaptive ratio table (readme, the table of candidate / collision ratio  */
/* by retrieval-zone length):                                               */
/*   < 5K: 0.50/0.50;  5K-10K: 0.25/0.30;  10K-30K: 0.20/0.25;             */
/*   >= 30K: 0.10/0.20.   Reading: K = 1000, half-open ranges.             */
/* ===================================================================== */
void or_ratio_table(int64_t n, double *beta, double *rho)
{
    if (n < 5000) { *beta = 0.50; *rho = 0.50; }
    else if (n < 10000) { *beta = 0.25; *rho = 0.30; }
    else if (n < 30000) { *beta = 0.20; *rho = 0.25; }
    else { *beta = 0.10; *rho = 0.20; }
}

void or_resolve(int64_t n, int64_t cand_budget, float collision_ratio, int topk,
                int64_t *C, int64_t *R)
{
    double beta, rho;
    or_ratio_table(n, &beta, &rho);
    int64_t c = (cand_budget > 0) ? cand_budget : (int64_t)ceil(beta * (double)n);
    if (c < topk) c = topk;
    if (c > n) c = n;
    double r = (collision_ratio > 0.0f) ? (double)collision_ratio : rho;
    int64_t rr = (int64_t)ceil(r * (double)n);
    if (rr < 1) rr = 1;
    if (rr > n) rr = n;
    *C = c;
    *R = rr;
}
