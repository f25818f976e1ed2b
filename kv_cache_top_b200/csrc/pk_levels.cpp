// pk_levels.cpp -- Lloyd-Max magnitude levels of the ParisKV 4-bit summary.
//
// ParisKV slides, Prop. 4.1 and App. B.1 (the codebook does not depend on the
// data; the quantiser is fitted to a prior): under a Haar rotation (u_b)_j^2 follows
// Beta(1/2, (m-1)/2), so y = |u_j| has density proportional to
// (1 - y^2)^((m-3)/2) on [0, 1], and offline Lloyd-Max quantisation gives the
// shared 3-bit magnitude levels (README, repository contents: a Lloyd-Max
// level file used by the 4-bit rerank).
//
// The cell integrals have closed forms: with y = sin(theta),
//   F0(Y) = int_0^Y (1-y^2)^((m-3)/2) dy = int_0^asin(Y) cos^(m-2)(theta) d theta
//         = I_{m-2}(asin Y),  I_p = cos^(p-1) sin / p + (p-1)/p I_{p-2},
//           I_0 = theta, I_1 = sin theta;
//   F1(Y) = int_0^Y y (1-y^2)^((m-3)/2) dy = (1 - (1-Y^2)^((m-1)/2)) / (m-1).
// Lloyd's iteration (centroids of the cells, then midpoints) from uniform
// levels to a fixed point in fp64; the index rounds the result to fp32.
#include <cmath>

namespace pk {

static double cos_power_integral(int p, double th)
{
    const double s = std::sin(th), c = std::cos(th);
    double i0 = th, i1 = s;
    if (p == 0) return i0;
    if (p == 1) return i1;
    double prev2 = (p % 2 == 0) ? i0 : i1;
    for (int q = (p % 2 == 0) ? 2 : 3; q <= p; q += 2) {
        const double cur = std::pow(c, q - 1) * s / q + (double)(q - 1) / q * prev2;
        prev2 = cur;
    }
    return prev2;
}

static double F0(int m, double y)
{
    if (y <= 0.0) return 0.0;
    if (y >= 1.0) y = 1.0;
    return cos_power_integral(m - 2, std::asin(y));
}

static double F1(int m, double y)
{
    if (y <= 0.0) return 0.0;
    if (y >= 1.0) y = 1.0;
    return (1.0 - std::pow(1.0 - y * y, 0.5 * (m - 1))) / (double)(m - 1);
}

int lloyd_max_levels(int m, int L, double *lev, double *thr)
{
    if (m < 3 || L < 2 || L > 4096) return -1;
    for (int t = 0; t < L; t++) lev[t] = (t + 0.5) / L;
    for (int it = 1; it <= 1000000; it++) {
        for (int t = 0; t < L - 1; t++) thr[t] = 0.5 * (lev[t] + lev[t + 1]);
        double delta = 0.0;
        for (int t = 0; t < L; t++) {
            const double a = (t == 0) ? 0.0 : thr[t - 1];
            const double b = (t == L - 1) ? 1.0 : thr[t];
            const double nv = (F1(m, b) - F1(m, a)) / (F0(m, b) - F0(m, a));
            delta = std::fmax(delta, std::fabs(nv - lev[t]));
            lev[t] = nv;
        }
        if (delta < 1e-15) {
            for (int t = 0; t < L - 1; t++) thr[t] = 0.5 * (lev[t] + lev[t + 1]);
            return it;
        }
    }
    return -1;
}

}  // namespace pk
