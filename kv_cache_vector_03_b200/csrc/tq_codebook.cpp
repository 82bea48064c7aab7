// Host Lloyd-Max codebook for one coordinate of a rotated unit vector.
//
// Law (a2a-mcp.org "What is TurboQuant", stage 1): after a random rotation each coordinate
// u of a unit vector in R^d follows Beta((d-1)/2, (d-1)/2) on [-1, 1], i.e.
// X = (u + 1)/2 ~ Beta(a, a) with a = (d-1)/2. The codebook is the Lloyd-Max (MSE-optimal)
// scalar quantizer of that law (blog.hotdry.top "TurboQuant vector-search compression",
// section "Random rotation and scalar quantization").
//
// Cell masses and first moments come from the regularised incomplete beta function
//   P(X in [x0, x1])        = I_x1(a, a) - I_x0(a, a)
//   E[X ; X in [x0, x1]]    = (1/2) (I_x1(a+1, a) - I_x0(a+1, a))
// (E[X 1{X <= x}] = a/(2a) I_x(a+1, a)), evaluated by the continued fraction of I_x
// (modified Lentz). Upper cells use the complements I_{1-x}(b, a) = 1 - I_x(a, b) so that
// tail masses keep their relative precision. The distortion at the fixed point is
//   D = 1 - d * sum_k c_k^2 P(cell k)   (E u^2 = 1/d and the centroid condition).
#include <cmath>
#include <cstring>

#include "tq_internal.h"

namespace {

// All incomplete-beta arithmetic runs in x87 extended precision (64-bit significand):
// the log-prefactor subtracts log-gamma terms of size ~a log a, whose rounding in plain
// double would limit the cell moments to ~1e-13 relative.
typedef long double ld;

ld lbeta(ld a, ld b) { return std::lgamma(a) + std::lgamma(b) - std::lgamma(a + b); }

// continued fraction of I_x(a,b) for x < (a+1)/(a+b+2) (modified Lentz)
ld betacf(ld a, ld b, ld x) {
    const ld tiny = 1e-300L;
    ld c = 1.0L, dd = 1.0L - (a + b) * x / (a + 1.0L);
    if (std::fabs(dd) < tiny) dd = tiny;
    dd = 1.0L / dd;
    ld h = dd;
    for (int k = 1; k <= 10000; ++k) {
        ld num = k * (b - k) * x / ((a + 2.0L * k - 1.0L) * (a + 2.0L * k));
        dd = 1.0L + num * dd; if (std::fabs(dd) < tiny) dd = tiny;
        c = 1.0L + num / c;  if (std::fabs(c) < tiny) c = tiny;
        dd = 1.0L / dd; h *= dd * c;
        num = -(a + k) * (a + b + k) * x / ((a + 2.0L * k) * (a + 2.0L * k + 1.0L));
        dd = 1.0L + num * dd; if (std::fabs(dd) < tiny) dd = tiny;
        c = 1.0L + num / c;  if (std::fabs(c) < tiny) c = tiny;
        dd = 1.0L / dd;
        ld del = dd * c;
        h *= del;
        if (std::fabs(del - 1.0L) < 1e-19L) break;
    }
    return h;
}

// I_x(a, b) for x <= (a+1)/(a+b+2), directly from the continued fraction
ld ibeta_cf(ld a, ld b, ld x) {
    if (x <= 0.0L) return 0.0L;
    ld lf = a * std::log(x) + b * std::log1p(-x) - lbeta(a, b) - std::log(a);
    return std::exp(lf) * betacf(a, b, x);
}

// I_x(a, b) and its complement 1 - I_x(a, b), each accurate in its own tail
void ibeta_pair(ld a, ld b, ld x, ld* lower, ld* upper) {
    if (x <= 0.0L) { *lower = 0.0L; *upper = 1.0L; return; }
    if (x >= 1.0L) { *lower = 1.0L; *upper = 0.0L; return; }
    if (x < (a + 1.0L) / (a + b + 2.0L)) {
        *lower = ibeta_cf(a, b, x);
        *upper = 1.0L - *lower;
    } else {
        *upper = ibeta_cf(b, a, 1.0L - x);
        *lower = 1.0L - *upper;
    }
}

// mass and first moment of u over [lo, hi] (u in [-1, 1]); cells entirely above 0 are
// computed from the upper tails
void cell_moments(double alpha, double lo, double hi, double* mass, double* first) {
    ld a = alpha, x0 = 0.5L * ((ld)lo + 1.0L), x1 = 0.5L * ((ld)hi + 1.0L);
    ld l0, u0, l1, u1, pl0, pu0, pl1, pu1;
    ibeta_pair(a, a, x0, &l0, &u0);
    ibeta_pair(a, a, x1, &l1, &u1);
    ibeta_pair(a + 1.0L, a, x0, &pl0, &pu0);
    ibeta_pair(a + 1.0L, a, x1, &pl1, &pu1);
    ld m, ex;  // mass and E[X ; cell]
    if (lo >= 0.0) {
        m = u0 - u1;
        ex = 0.5L * (pu0 - pu1);
    } else {
        m = l1 - l0;
        ex = 0.5L * (pl1 - pl0);
    }
    *mass = (double)m;
    *first = (double)(2.0L * ex - m);  // u = 2X - 1
}

}  // namespace

int tq_host_codebook(int d, int B, double* c, double* t, double* mse) {
    if (d < 3 || d > 4096 || B < 1 || B > 8) return -1;
    const int L = 1 << B;
    const double alpha = 0.5 * (d - 1);
    const double sigma = 1.0 / std::sqrt((double)d);
    // start: L equal-probability points of N(0, 1/d) (inverse of erfc by Newton)
    for (int k = 0; k < L; ++k) {
        double p = (k + 0.5) / L, z = 0.0;
        for (int it = 0; it < 60; ++it) {
            double f = 0.5 * std::erfc(-z / std::sqrt(2.0)) - p;
            double df = std::exp(-0.5 * z * z) / std::sqrt(2.0 * M_PI);
            z -= f / df;
        }
        c[k] = std::fmax(-0.999, std::fmin(0.999, sigma * z));
    }
    double mass[256], first[256];
    bool conv = false;
    for (int it = 0; it < 100000 && !conv; ++it) {
        double delta = 0.0;
        double lo = -1.0;
        for (int k = 0; k < L; ++k) {
            double hi = k + 1 < L ? 0.5 * (c[k] + c[k + 1]) : 1.0;
            cell_moments(alpha, lo, hi, &mass[k], &first[k]);
            lo = hi;
        }
        for (int k = 0; k < L; ++k) {
            double nc = first[k] / mass[k];
            delta = std::fmax(delta, std::fabs(nc - c[k]));
            c[k] = nc;
        }
        conv = delta < 1e-15;
    }
    for (int k = 0; k < L / 2; ++k) {
        double v = 0.5 * (c[L - 1 - k] - c[k]);
        c[L - 1 - k] = v;
        c[k] = -v;
    }
    for (int k = 0; k + 1 < L; ++k) t[k] = 0.5 * (c[k] + c[k + 1]);
    if (mse) {
        double acc = 0.0, lo = -1.0;
        for (int k = 0; k < L; ++k) {
            double hi = k + 1 < L ? t[k] : 1.0;
            double ms, fs;
            cell_moments(alpha, lo, hi, &ms, &fs);
            acc += c[k] * c[k] * ms;
            lo = hi;
        }
        *mse = 1.0 - d * acc;
    }
    return conv ? 0 : -6;
}
