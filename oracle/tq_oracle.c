/*
 * tq_oracle.c -- plain, slow fp64 CPU oracle of the TurboQuant KV-vector hot path.
 *
 * TEST INFRASTRUCTURE ONLY. It exists to check the CUDA library against the method as
 * the TurboQuant pages state it. Only tests/, the smoke entry point and the bench's CPU
 * baseline may load it. It shares no code, header, table or constant with the CUDA path.
 *
 * Every step follows the pages' order and notation, in fp64, one vector at a time,
 * with no blocking or reordering beyond what the definitions state. OpenMP only spreads
 * independent vectors / queries over cores.
 *
 * Sources (page title, section):
 *   [R]  blog.hotdry.top "TurboQuant vector-search compression", section
 *        "Random rotation and scalar quantization": rotate by a random orthogonal matrix;
 *        each coordinate then follows a fixed Beta law (-> N(0,1/d)); (b-1)-bit Lloyd-Max
 *        codebook computed offline; printed normalised MSE 0.36 / 0.117 / 0.03 / 0.009
 *        and 1-bit centroids +-sqrt(2/(pi d)).
 *   [Q]  same page, section "QJL residual correction": r = x - x_mse; S in R^{m x d}
 *        Gaussian; store sign(S r) and gamma = |r|_2; reconstruction
 *        x~ = x_mse + gamma sqrt(pi/2)/d S^T sign(S r); E<y,x~> = <y,x>.
 *   [B]  a2a-mcp.org "What is TurboQuant", stage 1: rotation from the QR of a Gaussian
 *        matrix; after rotation each coordinate follows Beta((d-1)/2,(d-1)/2) on [-1,1];
 *        Lloyd-Max quantizer for that law.
 *   [F]  same page, stage 2 + "fused Triton kernel": logits straight from the indices
 *        with the query pre-rotated once.
 *   [V]  friday-blog-bgf.pages.dev "TurboQuant deep dive II", section 1, step 1:
 *        values use the rotation + MSE scalar quantizer only.
 *
 * Readings where the pages are loose or silent:
 *   - the QJL factor is sqrt(pi/2)/m (the pages print /d; m = d in every workload);
 *   - vectors are normalised first: n = |x|, u = x/n, and gamma is |r| of the unit vector;
 *     scores are n * (<Pi q, c[idx]> + gamma sqrt(pi/2)/m <S q, s>);
 *   - idx_i = #{k : y_i > t_k} (a value on a boundary takes the lower cell); sign(0) = +1;
 *   - stored n and gamma are rounded to IEEE binary16, round-to-nearest-even.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_ERR_ARG -1
#define ORC_ERR_NOCONV -6

/* ------------------------------------------------------------------ binary16 rounding */
/* Round v to the nearest IEEE binary16 value (ties to even) and return it as a double.
 * Binary16 has 11 significant bits for normal numbers (|v| >= 2^-14) and a fixed quantum
 * of 2^-24 below that; anything that rounds above 65504 becomes +-inf. */
double orc_round_half(double v) {
    if (isnan(v)) return v;
    if (v == 0.0 || isinf(v)) return v;
    int e;
    frexp(v, &e);               /* v = f * 2^e, 0.5 <= |f| < 1 */
    int q = e - 11;             /* quantum of an 11-bit significand */
    if (q < -24) q = -24;       /* subnormal range */
    double r = ldexp(nearbyint(ldexp(v, -q)), q);
    if (fabs(r) > 65504.0) r = copysign(INFINITY, v);
    return r;
}

void orc_round_half_array(int64_t n, const double* in, double* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_round_half(in[i]);
}

/* ------------------------------------------------------------------ quadrature */
/* Gauss-Legendre nodes/weights on [-1,1] by Newton's method on P_n (three-term recurrence). */
#define GL_N 20
static double gl_x[GL_N], gl_w[GL_N];
static int gl_ready = 0;

static void gl_init(void) {
    if (gl_ready) return;
    const double pi = acos(-1.0);
    for (int i = 0; i < GL_N; ++i) {
        double x = cos(pi * (i + 0.75) / (GL_N + 0.5));
        double dp = 0.0;
        for (int it = 0; it < 100; ++it) {
            double p0 = 1.0, p1 = x;
            for (int k = 2; k <= GL_N; ++k) {
                double p2 = ((2.0 * k - 1.0) * x * p1 - (k - 1.0) * p0) / k;
                p0 = p1; p1 = p2;
            }
            dp = GL_N * (x * p1 - p0) / (x * x - 1.0);
            double dx = p1 / dp;
            x -= dx;
            if (fabs(dx) < 1e-16) break;
        }
        double p0 = 1.0, p1 = x;
        for (int k = 2; k <= GL_N; ++k) {
            double p2 = ((2.0 * k - 1.0) * x * p1 - (k - 1.0) * p0) / k;
            p0 = p1; p1 = p2;
        }
        dp = GL_N * (x * p1 - p0) / (x * x - 1.0);
        gl_x[i] = x;
        gl_w[i] = 2.0 / ((1.0 - x * x) * dp * dp);
    }
    gl_ready = 1;
}

/* ------------------------------------------------------------------ coordinate laws */
/* law 0: one coordinate of a uniform unit vector in R^d, density
 *        f(u) = (1-u^2)^((d-3)/2) / B(1/2, (d-1)/2) on [-1,1]      [B]
 * law 1: its large-d limit N(0, 1/d)                                [R]             */
typedef struct { int law; int d; double a; double log_norm; double sigma; double lim; } law_t;

static law_t law_make(int law, int d) {
    law_t L;
    L.law = law; L.d = d;
    L.a = 0.5 * (d - 3);
    L.log_norm = lgamma(0.5) + lgamma(0.5 * (d - 1)) - lgamma(0.5 * d); /* log B(1/2,(d-1)/2) */
    L.sigma = 1.0 / sqrt((double)d);
    /* beyond 40 sigma both densities are below e^-780 of their peak: integrate inside it */
    L.lim = law == 0 ? fmin(1.0, 40.0 * L.sigma) : 40.0 * L.sigma;
    return L;
}

static double law_pdf(const law_t* L, double u) {
    if (L->law == 0) {
        double s = 1.0 - u * u;
        if (s <= 0.0) return 0.0;
        return exp(L->a * log(s) - L->log_norm);
    }
    double z = u / L->sigma;
    return exp(-0.5 * z * z) / (L->sigma * sqrt(2.0 * acos(-1.0)));
}

/* integral of u^p f(u) (p = 0, 2) or (u-c)^2 f(u) (p = 3) over [lo, hi], composite
 * Gauss-Legendre with panels no wider than sigma/4 */
static double law_integral(const law_t* L, double lo, double hi, int p, double c) {
    gl_init();
    if (lo < -L->lim) lo = -L->lim;
    if (hi > L->lim) hi = L->lim;
    if (!(hi > lo)) return 0.0;
    int np = (int)ceil((hi - lo) / (0.25 * L->sigma));
    if (np < 1) np = 1;
    double h = (hi - lo) / np, acc = 0.0;
    for (int k = 0; k < np; ++k) {
        double a = lo + k * h, mid = a + 0.5 * h, part = 0.0;
        for (int i = 0; i < GL_N; ++i) {
            double u = mid + 0.5 * h * gl_x[i];
            double g = p == 0 ? 1.0 : p == 2 ? u * u : (u - c) * (u - c);
            part += gl_w[i] * g * law_pdf(L, u);
        }
        acc += 0.5 * h * part;
    }
    return acc;
}

/* cell mass: Gauss-Legendre for law 0, erfc for law 1 */
static double law_mass(const law_t* L, double lo, double hi) {
    if (L->law == 1) {
        double s2 = sqrt(2.0) * L->sigma;
        return 0.5 * (erfc(lo / s2) - erfc(hi / s2));
    }
    return law_integral(L, lo, hi, 0, 0.0);
}

/* cell first moment, closed form:
 *   law 0: int u (1-u^2)^a du = -(1-u^2)^(a+1) / (2(a+1))
 *   law 1: int u phi(u) du    = -sigma^2 phi(u)                                       */
static double law_first(const law_t* L, double lo, double hi) {
    if (L->law == 1) return L->sigma * L->sigma * (law_pdf(L, lo) - law_pdf(L, hi));
    double ap1 = L->a + 1.0;
    double flo = (1.0 - lo * lo) > 0.0 ? exp(ap1 * log1p(-lo * lo) - L->log_norm) : 0.0;
    double fhi = (1.0 - hi * hi) > 0.0 ? exp(ap1 * log1p(-hi * hi) - L->log_norm) : 0.0;
    return (flo - fhi) / (2.0 * ap1);
}

/* standard normal quantile by bisection on 0.5*erfc(-x/sqrt 2) */
static double norm_quantile(double p) {
    double lo = -40.0, hi = 40.0;
    for (int it = 0; it < 200; ++it) {
        double mid = 0.5 * (lo + hi);
        if (0.5 * erfc(-mid / sqrt(2.0)) < p) lo = mid; else hi = mid;
    }
    return 0.5 * (lo + hi);
}

/* ------------------------------------------------------------------ Lloyd-Max codebook */
/* [R][B] L = 2^B centroids c[0..L-1] (sorted) and L-1 boundaries t[k] = (c_k + c_{k+1})/2
 * for the coordinate law; Lloyd-Max fixed point: c_k = E[u | t_{k-1} < u < t_k] with
 * t_{-1} = -1, t_{L-1} = +1. Start at sigma * Phi^-1((k+1/2)/L); stop when max|dc| < 1e-15.
 * The law is symmetric, so the result is symmetrised (c_{L-1-k} = -c_k) before the
 * boundaries are formed; the middle boundary is then exactly 0.
 * mse = d * sum_k int_{cell k} (u - c_k)^2 f(u) du : the normalised distortion E|u - q(u)|^2
 * of a unit vector.                                                                       */
int orc_codebook(int d, int B, int law, double* c, double* t, double* mse, int* iters) {
    if (B < 1 || B > 8 || d < 3 || (law != 0 && law != 1)) return ORC_ERR_ARG;
    law_t L = law_make(law, d);
    int nl = 1 << B;
    double cn[256];
    for (int k = 0; k < nl; ++k) {
        double v = L.sigma * norm_quantile((k + 0.5) / nl);
        if (law == 0) v = fmax(-0.999, fmin(0.999, v));
        c[k] = v;
    }
    int it, conv = 0;
    for (it = 0; it < 100000; ++it) {
        double delta = 0.0;
        for (int k = 0; k < nl; ++k) {
            double lo = k == 0 ? -1.0 : 0.5 * (c[k - 1] + c[k]);
            double hi = k == nl - 1 ? 1.0 : 0.5 * (c[k] + c[k + 1]);
            if (law == 1) { if (k == 0) lo = -L.lim; if (k == nl - 1) hi = L.lim; }
            double mass = law_mass(&L, lo, hi);
            cn[k] = law_first(&L, lo, hi) / mass;
        }
        for (int k = 0; k < nl; ++k) { delta = fmax(delta, fabs(cn[k] - c[k])); c[k] = cn[k]; }
        if (delta < 1e-15) { conv = 1; ++it; break; }
    }
    if (iters) *iters = it;
    for (int k = 0; k < nl / 2; ++k) {
        double v = 0.5 * (c[nl - 1 - k] - c[k]);
        c[nl - 1 - k] = v;
        c[k] = -v;
    }
    for (int k = 0; k + 1 < nl; ++k) t[k] = 0.5 * (c[k] + c[k + 1]);
    double D = 0.0;
    for (int k = 0; k < nl; ++k) {
        double lo = k == 0 ? -1.0 : t[k - 1];
        double hi = k == nl - 1 ? 1.0 : t[k];
        if (law == 1) { if (k == 0) lo = -L.lim; if (k == nl - 1) hi = L.lim; }
        D += law_integral(&L, lo, hi, 3, c[k]);
    }
    if (mse) *mse = d * D;
    return conv ? ORC_OK : ORC_ERR_NOCONV;
}

/* mass of each cell under the law (diagnostic for the tests) */
int orc_cell_mass(int d, int B, int law, const double* t, double* mass) {
    law_t L = law_make(law, d);
    int nl = 1 << B;
    for (int k = 0; k < nl; ++k) {
        double lo = k == 0 ? -1.0 : t[k - 1];
        double hi = k == nl - 1 ? 1.0 : t[k];
        if (law == 1) { if (k == 0) lo = -L.lim; if (k == nl - 1) hi = L.lim; }
        mass[k] = law_mass(&L, lo, hi);
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------ quantize */
/* [R][Q] one vector x (fp64 copy of the exact input values):
 *   n = |x|, u = x / n (u = 0 for x = 0)
 *   y = Pi u                                  (Pi given in fp32, used in fp64)
 *   idx_i = #{k : y_i > t_k}                  (nearest centroid; B bits)
 *   x_mse = Pi^T c[idx],  r = u - x_mse,  gamma = |r|
 *   z = S r,  bit_j = [z_j >= 0]              (only when qjl)
 *   stored n^ = half(n), gamma^ = half(gamma)
 * Optional outputs y (n x d) and z (n x m) let the tests find coordinates that lie within
 * a tolerance band of a decision boundary. flags[v] bit 0: n^ overflowed binary16,
 * bit 1: non-finite input. When idx_in is given, those indices replace the nearest-centroid
 * step and the residual, gamma and signs follow from them (used to check the later steps
 * of a vector whose index was decided differently inside the tolerance band).            */
int orc_quantize(int64_t nv, int d, int m, int B, int qjl, const double* x, const float* pi,
                 const float* s, const double* c, const double* t, uint8_t* idx, uint8_t* sbit,
                 double* nhat, double* ghat, double* n_exact, double* g_exact, double* y_out,
                 double* z_out, int32_t* flags, const uint8_t* idx_in) {
    if (nv < 0 || d < 1 || d > 1024 || B < 1 || B > 8 || (qjl && (m < 1 || m > 1024))) return ORC_ERR_ARG;
    int nb = (1 << B) - 1;
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t v = 0; v < nv; ++v) {
        const double* xv = x + v * d;
        double* u = (double*)malloc(sizeof(double) * d * 4);
        double* y = u + d;
        double* xm = y + d;
        double* r = xm + d;
        int32_t fl = 0;
        double n2 = 0.0;
        for (int i = 0; i < d; ++i) { if (!isfinite(xv[i])) fl |= 2; n2 += xv[i] * xv[i]; }
        double n = sqrt(n2);
        for (int i = 0; i < d; ++i) u[i] = n > 0.0 ? xv[i] / n : 0.0;
        for (int i = 0; i < d; ++i) {
            double acc = 0.0;
            for (int j = 0; j < d; ++j) acc += (double)pi[(int64_t)i * d + j] * u[j];
            y[i] = acc;
        }
        for (int i = 0; i < d; ++i) {
            int k = 0;
            for (int b = 0; b < nb; ++b) k += y[i] > t[b];
            idx[v * d + i] = idx_in ? idx_in[v * d + i] : (uint8_t)k;
            if (y_out) y_out[v * d + i] = y[i];
        }
        for (int j = 0; j < d; ++j) {
            double acc = 0.0;
            for (int i = 0; i < d; ++i) acc += (double)pi[(int64_t)i * d + j] * c[idx[v * d + i]];
            xm[j] = acc;
        }
        double g2 = 0.0;
        for (int j = 0; j < d; ++j) { r[j] = u[j] - xm[j]; g2 += r[j] * r[j]; }
        double g = sqrt(g2);
        if (qjl) {
            for (int k = 0; k < m; ++k) {
                double acc = 0.0;
                for (int j = 0; j < d; ++j) acc += (double)s[(int64_t)k * d + j] * r[j];
                sbit[v * m + k] = acc >= 0.0;
                if (z_out) z_out[v * m + k] = acc;
            }
        }
        nhat[v] = orc_round_half(n);
        ghat[v] = orc_round_half(g);
        if (isinf(nhat[v])) fl |= 1;
        if (n_exact) n_exact[v] = n;
        if (g_exact) g_exact[v] = g;
        if (flags) flags[v] = fl;
        free(u);
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------ pre-rotated query */
/* [F] q' = Pi q and q'' = S q, once per query */
static void rotate_query(int d, int m, int qjl, const float* pi, const float* s, const double* q,
                         double* qp, double* qpp) {
    for (int i = 0; i < d; ++i) {
        double acc = 0.0;
        for (int j = 0; j < d; ++j) acc += (double)pi[(int64_t)i * d + j] * q[j];
        qp[i] = acc;
    }
    if (qjl)
        for (int k = 0; k < m; ++k) {
            double acc = 0.0;
            for (int j = 0; j < d; ++j) acc += (double)s[(int64_t)k * d + j] * q[j];
            qpp[k] = acc;
        }
}

/* score of one stored vector against a pre-rotated query [Q][F]:
 *   n^ * ( <q', c[idx]> + gamma^ * sqrt(pi/2)/m * <q'', s> ),  s_j = 2 bit_j - 1          */
static double score_one(int d, int m, int qjl, const uint8_t* idx, const uint8_t* sb, double nh,
                        double gh, const double* c, const double* qp, const double* qpp) {
    double a = 0.0;
    for (int i = 0; i < d; ++i) a += qp[i] * c[idx[i]];
    double b = 0.0;
    if (qjl) {
        for (int j = 0; j < m; ++j) b += qpp[j] * (sb[j] ? 1.0 : -1.0);
        b *= gh * sqrt(acos(-1.0) / 2.0) / m;
    }
    return nh * (a + b);
}

/* logits[q][k] = scale * score(q, key k) for every query against every key */
int orc_logits(int64_t nk, int d, int m, int B, int qjl, const uint8_t* idx, const uint8_t* sbit,
               const double* nhat, const double* ghat, const float* pi, const float* s,
               const double* c, int64_t nq, const double* q, double scale, double* out) {
    (void)B;
    if (nk < 0 || nq < 0 || d < 1) return ORC_ERR_ARG;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t iq = 0; iq < nq; ++iq) {
        double* qp = (double*)malloc(sizeof(double) * (d + (m > 0 ? m : 1)));
        double* qpp = qp + d;
        rotate_query(d, m, qjl, pi, s, q + iq * d, qp, qpp);
        for (int64_t k = 0; k < nk; ++k)
            out[iq * nk + k] = scale * score_one(d, m, qjl, idx + k * d, qjl ? sbit + k * m : NULL,
                                                 nhat[k], qjl ? ghat[k] : 0.0, c, qp, qpp);
        free(qp);
    }
    return ORC_OK;
}

/* exact logits of full-precision keys (the recent-token tail): scale * <q, k> */
int orc_exact_dot(int64_t nk, int d, const double* keys, int64_t nq, const double* q, double scale,
                  double* out) {
#pragma omp parallel for schedule(static)
    for (int64_t iq = 0; iq < nq; ++iq)
        for (int64_t k = 0; k < nk; ++k) {
            double acc = 0.0;
            for (int i = 0; i < d; ++i) acc += q[iq * d + i] * keys[k * d + i];
            out[iq * nk + k] = scale * acc;
        }
    return ORC_OK;
}

/* ------------------------------------------------------------------ reconstruction */
/* [Q] x~ = n^ (Pi^T c[idx] + gamma^ sqrt(pi/2)/m S^T s); values (no QJL): n^ Pi^T c[idx] [V] */
int orc_reconstruct(int64_t nv, int d, int m, int B, int qjl, const uint8_t* idx, const uint8_t* sbit,
                    const double* nhat, const double* ghat, const float* pi, const float* s,
                    const double* c, double* out) {
    (void)B;
    double kappa = qjl ? sqrt(acos(-1.0) / 2.0) / m : 0.0;
#pragma omp parallel for schedule(static)
    for (int64_t v = 0; v < nv; ++v) {
        for (int j = 0; j < d; ++j) {
            double acc = 0.0;
            for (int i = 0; i < d; ++i) acc += (double)pi[(int64_t)i * d + j] * c[idx[v * d + i]];
            if (qjl) {
                double b = 0.0;
                for (int k = 0; k < m; ++k) b += (double)s[(int64_t)k * d + j] * (sbit[v * m + k] ? 1.0 : -1.0);
                acc += ghat[v] * kappa * b;
            }
            out[v * d + j] = nhat[v] * acc;
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------ P.V */
/* [V] for each query head h: w = softmax(P[h, :]) (max subtracted, exp in fp64) and
 * o_h = sum_t w_t v^_t, with every value reconstructed on its own: v^_t = n^_t Pi^T c[idx_t].
 * All nh heads read the same tokens (one kv-head group).                                  */
int orc_pv(int64_t nt, int d, int B, const uint8_t* idx, const double* nhat, const float* pi,
           const double* c, int nh, const float* P, double* out) {
    (void)B;
    if (nt < 1 || nh < 1) return ORC_ERR_ARG;
    double* mx = (double*)malloc(sizeof(double) * nh * 2);
    double* zs = mx + nh;
    for (int h = 0; h < nh; ++h) {
        double m0 = -INFINITY;
        for (int64_t t = 0; t < nt; ++t) m0 = fmax(m0, (double)P[(int64_t)h * nt + t]);
        double z = 0.0;
        for (int64_t t = 0; t < nt; ++t) z += exp((double)P[(int64_t)h * nt + t] - m0);
        mx[h] = m0; zs[h] = z;
    }
    memset(out, 0, sizeof(double) * nh * d);
#pragma omp parallel
    {
        double* acc = (double*)calloc((size_t)nh * d + d, sizeof(double));
        double* vh = acc + (size_t)nh * d;
#pragma omp for schedule(static)
        for (int64_t t = 0; t < nt; ++t) {
            for (int j = 0; j < d; ++j) {
                double a = 0.0;
                for (int i = 0; i < d; ++i) a += (double)pi[(int64_t)i * d + j] * c[idx[t * d + i]];
                vh[j] = nhat[t] * a;
            }
            for (int h = 0; h < nh; ++h) {
                double w = exp((double)P[(int64_t)h * nt + t] - mx[h]) / zs[h];
                for (int j = 0; j < d; ++j) acc[(size_t)h * d + j] += w * vh[j];
            }
        }
#pragma omp critical
        for (int64_t i = 0; i < (int64_t)nh * d; ++i) out[i] += acc[i];
        free(acc);
    }
    free(mx);
    return ORC_OK;
}

/* ------------------------------------------------------------------ top-k */
/* keep the k best (score descending, ties -> lower index) in a sorted list */
static void topk_insert(int k, double* bs, int64_t* bi, double sc, int64_t id) {
    if (!(sc > bs[k - 1] || (sc == bs[k - 1] && id < bi[k - 1]))) return;
    int p = k - 1;
    while (p > 0 && (sc > bs[p - 1] || (sc == bs[p - 1] && id < bi[p - 1]))) {
        bs[p] = bs[p - 1]; bi[p] = bi[p - 1]; --p;
    }
    bs[p] = sc; bi[p] = id;
}

/* [Q][F] for each query: the inner-product estimator against every database vector, then
 * the k best. Used for vector search on a compressed database.                            */
int orc_topk(int64_t ndb, int d, int m, int B, int qjl, const uint8_t* idx, const uint8_t* sbit,
             const double* nhat, const double* ghat, const float* pi, const float* s,
             const double* c, int64_t nq, const double* q, int k, int64_t* out_idx, double* out_score) {
    (void)B;
    if (k < 1 || k > ndb) return ORC_ERR_ARG;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t iq = 0; iq < nq; ++iq) {
        double* qp = (double*)malloc(sizeof(double) * (d + m + 2 * k));
        double* qpp = qp + d;
        double* bs = qpp + m;
        int64_t* bi = (int64_t*)malloc(sizeof(int64_t) * k);
        for (int i = 0; i < k; ++i) { bs[i] = -INFINITY; bi[i] = INT64_MAX; }
        rotate_query(d, m, qjl, pi, s, q + iq * d, qp, qpp);
        for (int64_t v = 0; v < ndb; ++v) {
            double sc = score_one(d, m, qjl, idx + v * d, qjl ? sbit + v * m : NULL, nhat[v],
                                  qjl ? ghat[v] : 0.0, c, qp, qpp);
            topk_insert(k, bs, bi, sc, v);
        }
        for (int i = 0; i < k; ++i) { out_idx[iq * k + i] = bi[i]; out_score[iq * k + i] = bs[i]; }
        free(bi);
        free(qp);
    }
    return ORC_OK;
}

/* exact fp64 inner-product top-k of full-precision vectors (recall reference) */
int orc_exact_topk(int64_t ndb, int d, const float* xdb, int64_t nq, const double* q, int k,
                   int64_t* out_idx, double* out_score) {
    if (k < 1 || k > ndb) return ORC_ERR_ARG;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t iq = 0; iq < nq; ++iq) {
        double* bs = (double*)malloc(sizeof(double) * k);
        int64_t* bi = (int64_t*)malloc(sizeof(int64_t) * k);
        for (int i = 0; i < k; ++i) { bs[i] = -INFINITY; bi[i] = INT64_MAX; }
        for (int64_t v = 0; v < ndb; ++v) {
            double acc = 0.0;
            for (int i = 0; i < d; ++i) acc += q[iq * d + i] * (double)xdb[v * d + i];
            topk_insert(k, bs, bi, acc, v);
        }
        for (int i = 0; i < k; ++i) { out_idx[iq * k + i] = bi[i]; out_score[iq * k + i] = bs[i]; }
        free(bi);
        free(bs);
    }
    return ORC_OK;
}
