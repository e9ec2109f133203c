/*
 * slay_oracle.c -- plain, slow fp64 CPU oracle for SLAY spherical Yat-kernel
 * linear attention.  TEST INFRASTRUCTURE: only the tests, the package's smoke
 * check and the benchmark's CPU-baseline leg load this file's library.  It shares
 * no code, header or table with the CUDA library and includes none of its files.
 *
 * Citations (page title + section; see slay_oracle.h for the key):
 *   [ABS] SLAY abstract (paperdance card of arXiv 2602.04915)
 *   [REV] SLAY review (nubint.ai), section "Proposed method", steps 1-6
 *   [PHX] Salmon et al., SC'11, Philox4x32-10
 *
 * Readings taken where the pages are silent (each is listed in the design notes):
 *   - anchor feature = (a . x^)^2 with a ~ N(0, I/D), one positive degree-2 feature
 *   - quadrature substitution t = (2+eps)s, so s_r = t_r/(2+eps), wt_r = w_r/(2+eps)
 *   - one eps, used in the kernel (2 - 2x + eps) and in the denominator (+ eps)
 *   - causal sums are inclusive (j <= i); normalisation guard max(|x|, 1e-12)
 *   - omega and anchors independent per feature, shared by q and k, all b and h
 *
 * Pins (tests/test_oracle_pins.py): Philox known-answer vectors; Gauss-Laguerre
 * moments, the R=2 closed form and a library rule; quadrature convergence to the
 * closed-form kernel and its sign; per-node Monte-Carlo means of phi against the
 * closed form E = (1+2x^2)/D^2 * wt_r * exp(2 s_r x); positivity and scale
 * invariance of phi; quadratic == O(L) form; uniform-key and L=1 closed forms;
 * decode chain == causal rows; finite differences of the forward for the backward.
 * Every function here has at least one pin; none is "parity unpinned".
 */
#include "slay_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ Philox */

/* [PHX]: one round maps (c0,c1,c2,c3) with the two 32x32->64 products
 * M0*c0 and M1*c2 to (hi(M1 c2)^c1^k0, lo(M1 c2), hi(M0 c0)^c3^k1, lo(M0 c0));
 * between rounds the key is advanced by the Weyl constants. */
void orc_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    const uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;
    const uint32_t W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
    uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int round = 0; round < 10; ++round) {
        if (round > 0) { k0 += W0; k1 += W1; }
        uint64_t p0 = (uint64_t)M0 * (uint64_t)c0;
        uint64_t p1 = (uint64_t)M1 * (uint64_t)c2;
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t n0 = hi1 ^ c1 ^ k0;
        uint32_t n2 = hi0 ^ c3 ^ k1;
        c0 = n0; c1 = lo1; c2 = n2; c3 = lo0;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* One standard normal from the counter (idx, tag, 0, 0): Box-Muller on the first
 * two 32-bit outputs mapped to (0,1) as (x + 1/2) 2^-32. */
static double orc_normal(uint64_t seed, uint32_t idx, uint32_t tag)
{
    uint32_t ctr[4] = { idx, tag, 0u, 0u };
    uint32_t key[2] = { (uint32_t)(seed & 0xffffffffu), (uint32_t)(seed >> 32) };
    uint32_t o[4];
    orc_philox4x32_10(ctr, key, o);
    const double two_pi = 6.283185307179586476925286766559;
    double u1 = ((double)o[0] + 0.5) * (1.0 / 4294967296.0);
    double u2 = ((double)o[1] + 0.5) * (1.0 / 4294967296.0);
    return sqrt(-2.0 * log(u1)) * cos(two_pi * u2);
}

/* The same normal from the counter (idx, tag, head, 0): the per-head draw of a sketch
 * variant (head 0 is the counter above). */
static double orc_normal_h(uint64_t seed, uint32_t idx, uint32_t tag, uint32_t head)
{
    uint32_t ctr[4] = { idx, tag, head, 0u };
    uint32_t key[2] = { (uint32_t)(seed & 0xffffffffu), (uint32_t)(seed >> 32) };
    uint32_t o[4];
    orc_philox4x32_10(ctr, key, o);
    const double two_pi = 6.283185307179586476925286766559;
    double u1 = ((double)o[0] + 0.5) * (1.0 / 4294967296.0);
    double u2 = ((double)o[1] + 0.5) * (1.0 / 4294967296.0);
    return sqrt(-2.0 * log(u1)) * cos(two_pi * u2);
}

/* --------------------------------------------------------- Gauss-Laguerre */

/* L_n(t) and L_{n-1}(t) by the three-term recurrence
 * (k+1) L_{k+1} = (2k+1-t) L_k - k L_{k-1}, L_0 = 1, L_1 = 1 - t. */
static void laguerre_pair(int n, double t, double* ln, double* lnm1)
{
    double a = 1.0, b = 1.0 - t;  /* L_0, L_1 */
    if (n == 0) { *ln = 1.0; *lnm1 = 0.0; return; }
    for (int kk = 1; kk < n; ++kk) {
        double c = ((2.0 * kk + 1.0 - t) * b - kk * a) / (kk + 1.0);
        a = b; b = c;
    }
    *ln = b; *lnm1 = a;
}

/* [REV] step 4 discretises the Laplace integral with Gauss-Laguerre.  The R nodes
 * are the zeros of L_R; they are bracketed by sign changes on a grid uniform in
 * sqrt(t) (zeros are roughly evenly spaced there) over [0, 4R+10], refined by
 * bisection to the last bit, and the weights follow from
 * w = 1 / (t L_R'(t)^2) with L_R'(t) = -R L_{R-1}(t) / t at a zero. */
int orc_gauss_laguerre(int R, double* t, double* w)
{
    if (R < 1 || R > 64) return -1;
    const int G = 40000;
    double umax = sqrt(4.0 * R + 10.0);
    int found = 0;
    double ln, lm;
    double uprev = 0.0, fprev;
    laguerre_pair(R, 0.0, &fprev, &lm);
    for (int g = 1; g <= G && found < R; ++g) {
        double u = umax * g / G;
        double f;
        laguerre_pair(R, u * u, &f, &lm);
        if ((fprev < 0.0) != (f < 0.0)) {
            double lo = uprev * uprev, hi = u * u, flo = fprev;
            for (int it = 0; it < 200; ++it) {
                double mid = 0.5 * (lo + hi);
                if (mid <= lo || mid >= hi) break;
                double fm;
                laguerre_pair(R, mid, &fm, &lm);
                if ((fm < 0.0) == (flo < 0.0)) { lo = mid; flo = fm; } else { hi = mid; }
            }
            double root = 0.5 * (lo + hi);
            laguerre_pair(R, root, &ln, &lm);
            double dl = -R * lm / root;
            t[found] = root;
            w[found] = 1.0 / (root * dl * dl);
            ++found;
        }
        uprev = u; fprev = f;
    }
    return found == R ? 0 : -1;
}

int orc_sketch_params(int D, int R, int m, uint64_t seed, double eps,
                      double* omega, double* anchors, double* s, double* wt)
{
    double tn[64], wn[64];
    if (orc_gauss_laguerre(R, tn, wn) != 0) return -1;
    for (int r = 0; r < R; ++r) {
        s[r] = tn[r] / (2.0 + eps);
        wt[r] = wn[r] / (2.0 + eps);
    }
    const int64_t F = (int64_t)R * m;
    for (int64_t f = 0; f < F; ++f) {
        for (int d = 0; d < D; ++d) {
            uint32_t idx = (uint32_t)(f * D + d);
            double no = orc_normal(seed, idx, 0u);
            double na = orc_normal(seed, idx, 1u);
            omega[f * D + d] = (double)(float)no;
            anchors[f * D + d] = (double)(float)(na / sqrt((double)D));
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ kernels */

/* [ABS]: Yat kernel (q.k)^2 / (|q-k|^2 + eps); on the unit sphere
 * |q-k|^2 = 2 - 2x with x = q.k. */
double orc_yat_kernel(double x, double eps) { return x * x / (2.0 - 2.0 * x + eps); }

/* [REV] steps 2 and 4: 1/(2-2x+eps) = int_0^inf e^{-s(2+eps)} e^{2sx} ds, and with
 * t = (2+eps)s the e^{-t} weight is handled by the Gauss-Laguerre rule. */
double orc_quad_kernel(double x, int R, double eps)
{
    double tn[64], wn[64];
    if (orc_gauss_laguerre(R, tn, wn) != 0) return NAN;
    double acc = 0.0;
    for (int r = 0; r < R; ++r) {
        double sr = tn[r] / (2.0 + eps), wr = wn[r] / (2.0 + eps);
        acc += wr * exp(2.0 * sr * x);
    }
    return x * x * acc;
}

/* [REV] steps 1, 3, 4, 5: unit-sphere projection, positive exponential random
 * feature per node, anchor feature for the polynomial factor, elementwise
 * (tensor-sketch) product, node weight folded in as sqrt(wt_r/m). */
static void phi_row(const double* x, int D, int R, int m,
                    const double* omega, const double* anchors,
                    const double* s, const double* wt, double* phi)
{
    double nrm = 0.0;
    for (int d = 0; d < D; ++d) nrm += x[d] * x[d];
    nrm = sqrt(nrm);
    if (nrm < 1e-12) nrm = 1e-12;
    double xh[1024];
    for (int d = 0; d < D; ++d) xh[d] = x[d] / nrm;
    for (int r = 0; r < R; ++r) {
        double sq = sqrt(2.0 * s[r]);
        double scale = sqrt(wt[r] / m);
        for (int j = 0; j < m; ++j) {
            int64_t f = (int64_t)r * m + j;
            double u = 0.0, p = 0.0;
            for (int d = 0; d < D; ++d) {
                u += omega[f * D + d] * xh[d];
                p += anchors[f * D + d] * xh[d];
            }
            phi[f] = scale * exp(sq * u - s[r]) * p * p;
        }
    }
}

void orc_feature_map(const double* x, int64_t n, int D, int R, int m,
                     const double* omega, const double* anchors,
                     const double* s, const double* wt, double* phi)
{
    const int64_t F = (int64_t)R * m;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        phi_row(x + i * D, D, R, m, omega, anchors, s, wt, phi + i * F);
}

static double dot(const double* a, const double* b, int64_t n)
{
    double acc = 0.0;
    for (int64_t i = 0; i < n; ++i) acc += a[i] * b[i];
    return acc;
}

/* phi of every row of one (b,h) slice: returns a malloc'd [L, F] array. */
/* Sketch variants (the pages leave the anchor form and the feature bank open: review,
 * "Proposed method", steps 3 and 5; orthogonal banks appear as prior art on the LinSimp
 * page).  kind:
 *   0 positive anchor (the default above): iid omega, phi = c e^{...} (a.x^)^2;
 *   1 orthogonal: omega rows orthogonalised in blocks of D consecutive rows of a node by
 *     Gram-Schmidt in draw order, each row keeping the length of its own Gaussian draw
 *     (so every row is still N(0, I) marginally); anchors as kind 0;
 *   2 signed anchor: phi = c e^{...} (a.x^)(b.x^) with a second anchor set b (tag 2),
 *     unbiased for x^2 / D^2 but not positive;
 *   3 per head: kind 0 drawn per head h with the counter (f D + d, tag, h, 0);
 *   4 Performer FAVOR+: phi_f = exp(omega_f.x^ - 1/2) / sqrt(F), omega orthogonal as kind 1
 *     (no quadrature, no anchor; the estimator of exp(q^.k^)).
 * Values are rounded to float as in orc_sketch_params.  anchors_b is written for kind 2. */
int orc_sketch_params_kind(int D, int R, int m, uint64_t seed, double eps, int kind, int head,
                           double* omega, double* anchors, double* anchors_b, double* s,
                           double* wt)
{
    double tn[64], wn[64];
    if (kind < 0 || kind > 4 || head < 0 || D > 1024) return -1;
    if (orc_gauss_laguerre(R, tn, wn) != 0) return -1;
    for (int r = 0; r < R; ++r) {
        s[r] = tn[r] / (2.0 + eps);
        wt[r] = wn[r] / (2.0 + eps);
    }
    const int64_t F = (int64_t)R * m;
    const uint32_t h = kind == 3 ? (uint32_t)head : 0u;
    double* g = (double*)malloc(sizeof(double) * (size_t)F * D);
    for (int64_t f = 0; f < F; ++f)
        for (int d = 0; d < D; ++d) {
            uint32_t idx = (uint32_t)(f * D + d);
            g[f * D + d] = orc_normal_h(seed, idx, 0u, h);
            anchors[f * D + d] = (double)(float)(orc_normal_h(seed, idx, 1u, h) / sqrt((double)D));
            if (kind == 2)
                anchors_b[f * D + d] = (double)(float)(orc_normal_h(seed, idx, 2u, h) / sqrt((double)D));
        }
    if (kind == 1 || kind == 4) {
        /* classical Gram-Schmidt on each block: q_j = g_j - sum_{i<j} (g_j . e_i) e_i,
         * e_j = q_j / |q_j|, row j = e_j |g_j| */
        double* e = (double*)malloc(sizeof(double) * (size_t)D * D);
        for (int r = 0; r < R; ++r)
            for (int b0 = 0; b0 < m; b0 += D) {
                int nb = m - b0 < D ? m - b0 : D;
                for (int j = 0; j < nb; ++j) {
                    const double* gj = g + ((int64_t)r * m + b0 + j) * D;
                    double* ej = e + (int64_t)j * D;
                    for (int d = 0; d < D; ++d) ej[d] = gj[d];
                    for (int i = 0; i < j; ++i) {
                        double c = dot(gj, e + (int64_t)i * D, D);
                        for (int d = 0; d < D; ++d) ej[d] -= c * e[(int64_t)i * D + d];
                    }
                    double n = sqrt(dot(ej, ej, D));
                    for (int d = 0; d < D; ++d) ej[d] /= n;
                }
                for (int j = 0; j < nb; ++j) {
                    double* gj = g + ((int64_t)r * m + b0 + j) * D;
                    double len = sqrt(dot(gj, gj, D));
                    for (int d = 0; d < D; ++d) gj[d] = e[(int64_t)j * D + d] * len;
                }
            }
        free(e);
    }
    for (int64_t t = 0; t < F * D; ++t) omega[t] = (double)(float)g[t];
    free(g);
    return 0;
}

/* phi of one row for a sketch variant (kinds 0-3 share the quadrature; kind 4 is FAVOR+) */
static void phi_row_kind(const double* x, int D, int R, int m, const double* omega,
                         const double* anchors, const double* anchors_b, const double* s,
                         const double* wt, int kind, double* phi)
{
    double nrm = 0.0;
    for (int d = 0; d < D; ++d) nrm += x[d] * x[d];
    nrm = sqrt(nrm);
    if (nrm < 1e-12) nrm = 1e-12;
    double xh[1024];
    for (int d = 0; d < D; ++d) xh[d] = x[d] / nrm;
    const int64_t F = (int64_t)R * m;
    for (int r = 0; r < R; ++r) {
        double sq = sqrt(2.0 * s[r]);
        double scale = sqrt(wt[r] / m);
        for (int j = 0; j < m; ++j) {
            int64_t f = (int64_t)r * m + j;
            double u = dot(omega + f * D, xh, D);
            if (kind == 4) {
                phi[f] = exp(u - 0.5) / sqrt((double)F);
                continue;
            }
            double p = dot(anchors + f * D, xh, D);
            double pb = kind == 2 ? dot(anchors_b + f * D, xh, D) : p;
            phi[f] = scale * exp(sq * u - s[r]) * p * pb;
        }
    }
}

void orc_feature_map_kind(const double* x, int64_t n, int D, int R, int m,
                          const double* omega, const double* anchors, const double* anchors_b,
                          const double* s, const double* wt, int kind, double* phi)
{
    const int64_t F = (int64_t)R * m;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        phi_row_kind(x + i * D, D, R, m, omega, anchors, anchors_b, s, wt, kind, phi + i * F);
}

static double* phi_slice(const double* x, int L, int D, int R, int m,
                         const double* omega, const double* anchors,
                         const double* s, const double* wt)
{
    const int64_t F = (int64_t)R * m;
    double* p = (double*)malloc(sizeof(double) * (size_t)L * (size_t)F);
    for (int i = 0; i < L; ++i)
        phi_row(x + (int64_t)i * D, D, R, m, omega, anchors, s, wt, p + (int64_t)i * F);
    return p;
}

/* Quadratic definition of one output row i of one (b,h) slice. */
static void quad_row(const double* pq_i, const double* pk, const double* v,
                     int L, int Dv, int64_t F, double eps, int causal, int i,
                     double* out_i, double* den_i)
{
    int jend = causal ? i + 1 : L;
    double den = 0.0;
    for (int e = 0; e < Dv; ++e) out_i[e] = 0.0;
    for (int j = 0; j < jend; ++j) {
        double a = dot(pq_i, pk + (int64_t)j * F, F);
        den += a;
        for (int e = 0; e < Dv; ++e) out_i[e] += a * v[(int64_t)j * Dv + e];
    }
    for (int e = 0; e < Dv; ++e) out_i[e] /= (den + eps);
    if (den_i) *den_i = den;
}

void orc_attn_quadratic(const double* q, const double* k, const double* v,
                        int B, int H, int L, int D, int Dv, int R, int m,
                        const double* omega, const double* anchors,
                        const double* s, const double* wt, double eps, int causal,
                        double* out, double* den)
{
    const int64_t F = (int64_t)R * m;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < B * H; ++bh) {
        const double* qs = q + (int64_t)bh * L * D;
        const double* ks = k + (int64_t)bh * L * D;
        const double* vs = v + (int64_t)bh * L * Dv;
        double* pq = phi_slice(qs, L, D, R, m, omega, anchors, s, wt);
        double* pk = phi_slice(ks, L, D, R, m, omega, anchors, s, wt);
        for (int i = 0; i < L; ++i)
            quad_row(pq + (int64_t)i * F, pk, vs, L, Dv, F, eps, causal, i,
                     out + ((int64_t)bh * L + i) * Dv,
                     den ? den + (int64_t)bh * L + i : NULL);
        free(pq); free(pk);
    }
}

void orc_attn_quadratic_rows(const double* q, const double* k, const double* v,
                             int B, int H, int L, int D, int Dv, int R, int m,
                             const double* omega, const double* anchors,
                             const double* s, const double* wt, double eps, int causal,
                             const int64_t* rows, int nrows,
                             double* out_rows, double* den_rows)
{
    const int64_t F = (int64_t)R * m;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < B * H; ++bh) {
        const double* qs = q + (int64_t)bh * L * D;
        const double* ks = k + (int64_t)bh * L * D;
        const double* vs = v + (int64_t)bh * L * Dv;
        double* pk = phi_slice(ks, L, D, R, m, omega, anchors, s, wt);
        double* pq = (double*)malloc(sizeof(double) * (size_t)F);
        for (int r = 0; r < nrows; ++r) {
            int i = (int)rows[r];
            phi_row(qs + (int64_t)i * D, D, R, m, omega, anchors, s, wt, pq);
            quad_row(pq, pk, vs, L, Dv, F, eps, causal, i,
                     out_rows + ((int64_t)bh * nrows + r) * Dv,
                     den_rows ? den_rows + (int64_t)bh * nrows + r : NULL);
        }
        free(pq); free(pk);
    }
}

/* O(L) form of one (b,h) slice with state S [F, Dv] and z [F]. */
static void recurrent_slice(const double* pq, const double* pk, const double* vs,
                            int L, int Dv, int64_t F, double eps, int causal,
                            double* out, double* den)
{
    double* S = (double*)calloc((size_t)F * (size_t)Dv, sizeof(double));
    double* z = (double*)calloc((size_t)F, sizeof(double));
    if (!causal) {
        for (int j = 0; j < L; ++j)
            for (int64_t f = 0; f < F; ++f) {
                double a = pk[(int64_t)j * F + f];
                z[f] += a;
                for (int e = 0; e < Dv; ++e) S[f * Dv + e] += a * vs[(int64_t)j * Dv + e];
            }
    }
    for (int i = 0; i < L; ++i) {
        if (causal)
            for (int64_t f = 0; f < F; ++f) {
                double a = pk[(int64_t)i * F + f];
                z[f] += a;
                for (int e = 0; e < Dv; ++e) S[f * Dv + e] += a * vs[(int64_t)i * Dv + e];
            }
        const double* p = pq + (int64_t)i * F;
        double d = dot(p, z, F);
        for (int e = 0; e < Dv; ++e) {
            double acc = 0.0;
            for (int64_t f = 0; f < F; ++f) acc += p[f] * S[f * Dv + e];
            out[(int64_t)i * Dv + e] = acc / (d + eps);
        }
        if (den) den[i] = d;
    }
    free(S); free(z);
}

void orc_attn_recurrent(const double* q, const double* k, const double* v,
                        int B, int H, int L, int D, int Dv, int R, int m,
                        const double* omega, const double* anchors,
                        const double* s, const double* wt, double eps, int causal,
                        double* out, double* den)
{
    const int64_t F = (int64_t)R * m;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < B * H; ++bh) {
        double* pq = phi_slice(q + (int64_t)bh * L * D, L, D, R, m, omega, anchors, s, wt);
        double* pk = phi_slice(k + (int64_t)bh * L * D, L, D, R, m, omega, anchors, s, wt);
        recurrent_slice(pq, pk, v + (int64_t)bh * L * Dv, L, Dv, F, eps, causal,
                        out + (int64_t)bh * L * Dv, den ? den + (int64_t)bh * L : NULL);
        free(pq); free(pk);
    }
}

void orc_decode_step(const double* q, const double* k, const double* v,
                     double* S, double* z, double* out,
                     int N, int D, int Dv, int R, int m,
                     const double* omega, const double* anchors,
                     const double* s, const double* wt, double eps)
{
    const int64_t F = (int64_t)R * m;
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n) {
        double* pq = (double*)malloc(sizeof(double) * (size_t)F);
        double* pk = (double*)malloc(sizeof(double) * (size_t)F);
        phi_row(q + (int64_t)n * D, D, R, m, omega, anchors, s, wt, pq);
        phi_row(k + (int64_t)n * D, D, R, m, omega, anchors, s, wt, pk);
        double* Sn = S + (int64_t)n * F * Dv;
        double* zn = z + (int64_t)n * F;
        const double* vn = v + (int64_t)n * Dv;
        for (int64_t f = 0; f < F; ++f) {
            zn[f] += pk[f];
            for (int e = 0; e < Dv; ++e) Sn[f * Dv + e] += pk[f] * vn[e];
        }
        double d = dot(pq, zn, F);
        for (int e = 0; e < Dv; ++e) {
            double acc = 0.0;
            for (int64_t f = 0; f < F; ++f) acc += pq[f] * Sn[f * Dv + e];
            out[(int64_t)n * Dv + e] = acc / (d + eps);
        }
        free(pq); free(pk);
    }
}

/* ----------------------------------------------------------------- backward */

/* Chain rule through phi and the sphere projection for one row.  With
 * u = <omega_f, x^>, p = <a_f, x^>, E = exp(sqrt(2 s_r) u - s_r), c = sqrt(wt_r/m):
 *   d phi_f / d x^ = phi_f sqrt(2 s_r) omega_f + 2 c E p a_f
 * and x^ = x / n with n = max(|x|, 1e-12):
 *   dx = (dx^ - x^ <x^, dx^>) / n   (n = |x|),   dx = dx^ / 1e-12 (guard active). */
static void phi_backward_row(const double* x, const double* dphi, int D, int R, int m,
                             const double* omega, const double* anchors,
                             const double* s, const double* wt, double* dx)
{
    double nrm2 = 0.0;
    for (int d = 0; d < D; ++d) nrm2 += x[d] * x[d];
    double nrm = sqrt(nrm2);
    int guard = nrm < 1e-12;
    if (guard) nrm = 1e-12;
    double xh[1024], dxh[1024];
    for (int d = 0; d < D; ++d) { xh[d] = x[d] / nrm; dxh[d] = 0.0; }
    for (int r = 0; r < R; ++r) {
        double sq = sqrt(2.0 * s[r]);
        double c = sqrt(wt[r] / m);
        for (int j = 0; j < m; ++j) {
            int64_t f = (int64_t)r * m + j;
            const double* om = omega + f * D;
            const double* an = anchors + f * D;
            double u = dot(om, xh, D), p = dot(an, xh, D);
            double E = exp(sq * u - s[r]);
            double ph = c * E * p * p;
            double go = dphi[f] * ph * sq;
            double ga = dphi[f] * 2.0 * c * E * p;
            for (int d = 0; d < D; ++d) dxh[d] += go * om[d] + ga * an[d];
        }
    }
    if (guard) {
        for (int d = 0; d < D; ++d) dx[d] = dxh[d] / nrm;
    } else {
        double pr = dot(xh, dxh, D);
        for (int d = 0; d < D; ++d) dx[d] = (dxh[d] - xh[d] * pr) / nrm;
    }
}

/* Differentiating out_i = num_i / Z_i with num_i = sum_{j<=i} a_ij v_j,
 * Z_i = sum_{j<=i} a_ij + eps, a_ij = <phi(q_i), phi(k_j)>:
 *   dn_i = g_i / Z_i, delta_i = -<g_i, out_i> / Z_i, c_ij = <v_j, dn_i> + delta_i
 *   dphi(q_i) = sum_{j<=i} c_ij phi(k_j)
 *   dphi(k_j) = sum_{i>=j} c_ij phi(q_i)
 *   dv_j      = sum_{i>=j} a_ij dn_i                                          */
void orc_attn_causal_bwd(const double* q, const double* k, const double* v,
                         const double* dout,
                         int B, int H, int L, int D, int Dv, int R, int m,
                         const double* omega, const double* anchors,
                         const double* s, const double* wt, double eps,
                         double* dq, double* dk, double* dv)
{
    const int64_t F = (int64_t)R * m;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < B * H; ++bh) {
        const double* qs = q + (int64_t)bh * L * D;
        const double* ks = k + (int64_t)bh * L * D;
        const double* vs = v + (int64_t)bh * L * Dv;
        const double* gs = dout + (int64_t)bh * L * Dv;
        double* pq = phi_slice(qs, L, D, R, m, omega, anchors, s, wt);
        double* pk = phi_slice(ks, L, D, R, m, omega, anchors, s, wt);
        double* outv = (double*)malloc(sizeof(double) * (size_t)L * Dv);
        double* den = (double*)malloc(sizeof(double) * (size_t)L);
        for (int i = 0; i < L; ++i)
            quad_row(pq + (int64_t)i * F, pk, vs, L, Dv, F, eps, 1, i,
                     outv + (int64_t)i * Dv, den + i);
        double* dn = (double*)malloc(sizeof(double) * (size_t)L * Dv);
        double* delta = (double*)malloc(sizeof(double) * (size_t)L);
        for (int i = 0; i < L; ++i) {
            double Z = den[i] + eps;
            for (int e = 0; e < Dv; ++e) dn[(int64_t)i * Dv + e] = gs[(int64_t)i * Dv + e] / Z;
            delta[i] = -dot(gs + (int64_t)i * Dv, outv + (int64_t)i * Dv, Dv) / Z;
        }
        double* dpq = (double*)calloc((size_t)L * F, sizeof(double));
        double* dpk = (double*)calloc((size_t)L * F, sizeof(double));
        double* dvs = dv + (int64_t)bh * L * Dv;
        for (int64_t t = 0; t < (int64_t)L * Dv; ++t) dvs[t] = 0.0;
        for (int i = 0; i < L; ++i) {
            for (int j = 0; j <= i; ++j) {
                double c = dot(vs + (int64_t)j * Dv, dn + (int64_t)i * Dv, Dv) + delta[i];
                double a = dot(pq + (int64_t)i * F, pk + (int64_t)j * F, F);
                for (int64_t f = 0; f < F; ++f) {
                    dpq[(int64_t)i * F + f] += c * pk[(int64_t)j * F + f];
                    dpk[(int64_t)j * F + f] += c * pq[(int64_t)i * F + f];
                }
                for (int e = 0; e < Dv; ++e)
                    dvs[(int64_t)j * Dv + e] += a * dn[(int64_t)i * Dv + e];
            }
        }
        for (int i = 0; i < L; ++i) {
            phi_backward_row(qs + (int64_t)i * D, dpq + (int64_t)i * F, D, R, m,
                             omega, anchors, s, wt, dq + ((int64_t)bh * L + i) * D);
            phi_backward_row(ks + (int64_t)i * D, dpk + (int64_t)i * F, D, R, m,
                             omega, anchors, s, wt, dk + ((int64_t)bh * L + i) * D);
        }
        free(pq); free(pk); free(outv); free(den); free(dn); free(delta);
        free(dpq); free(dpk);
    }
}

/* The same gradients evaluated at a GIVEN forward output: out [B,H,L,Dv] and den [B,H,L]
 * are inputs here, as they are to the library's backward (which receives the forward's
 * stored out in the input dtype), instead of being recomputed.  dn_i = g_i/(den_i+eps),
 * delta_i = -<g_i, out_i>/(den_i+eps), then the contraction and the chain rule through phi
 * exactly as in orc_attn_causal_bwd (the derivative of the forward, reading 13 of the
 * design notes; the pages give no backward).  With the exact forward output it IS
 * orc_attn_causal_bwd; with a rounded copy it is the gradient formula the library evaluates
 * on that copy, so both sides see the same cancellation in <v_j, dn_i> + delta_i. */
void orc_attn_causal_bwd_given(const double* q, const double* k, const double* v,
                               const double* out, const double* den_in, const double* dout,
                               int B, int H, int L, int D, int Dv, int R, int m,
                               const double* omega, const double* anchors,
                               const double* s, const double* wt, double eps,
                               double* dq, double* dk, double* dv)
{
    const int64_t F = (int64_t)R * m;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < B * H; ++bh) {
        const double* qs = q + (int64_t)bh * L * D;
        const double* ks = k + (int64_t)bh * L * D;
        const double* vs = v + (int64_t)bh * L * Dv;
        const double* os = out + (int64_t)bh * L * Dv;
        const double* ds = den_in + (int64_t)bh * L;
        const double* gs = dout + (int64_t)bh * L * Dv;
        double* pq = phi_slice(qs, L, D, R, m, omega, anchors, s, wt);
        double* pk = phi_slice(ks, L, D, R, m, omega, anchors, s, wt);
        double* dn = (double*)malloc(sizeof(double) * (size_t)L * Dv);
        double* delta = (double*)malloc(sizeof(double) * (size_t)L);
        for (int i = 0; i < L; ++i) {
            double Z = ds[i] + eps;
            for (int e = 0; e < Dv; ++e) dn[(int64_t)i * Dv + e] = gs[(int64_t)i * Dv + e] / Z;
            delta[i] = -dot(gs + (int64_t)i * Dv, os + (int64_t)i * Dv, Dv) / Z;
        }
        double* dpq = (double*)calloc((size_t)L * F, sizeof(double));
        double* dpk = (double*)calloc((size_t)L * F, sizeof(double));
        double* dvs = dv + (int64_t)bh * L * Dv;
        for (int64_t t = 0; t < (int64_t)L * Dv; ++t) dvs[t] = 0.0;
        for (int i = 0; i < L; ++i) {
            for (int j = 0; j <= i; ++j) {
                double c = dot(vs + (int64_t)j * Dv, dn + (int64_t)i * Dv, Dv) + delta[i];
                double a = dot(pq + (int64_t)i * F, pk + (int64_t)j * F, F);
                for (int64_t f = 0; f < F; ++f) {
                    dpq[(int64_t)i * F + f] += c * pk[(int64_t)j * F + f];
                    dpk[(int64_t)j * F + f] += c * pq[(int64_t)i * F + f];
                }
                for (int e = 0; e < Dv; ++e)
                    dvs[(int64_t)j * Dv + e] += a * dn[(int64_t)i * Dv + e];
            }
        }
        for (int i = 0; i < L; ++i) {
            phi_backward_row(qs + (int64_t)i * D, dpq + (int64_t)i * F, D, R, m,
                             omega, anchors, s, wt, dq + ((int64_t)bh * L + i) * D);
            phi_backward_row(ks + (int64_t)i * D, dpk + (int64_t)i * F, D, R, m,
                             omega, anchors, s, wt, dk + ((int64_t)bh * L + i) * D);
        }
        free(pq); free(pk); free(dn); free(delta); free(dpq); free(dpk);
    }
}

/* The backward of one piece of a longer causal sequence, split over ranks (the prefix state
 * of the review's "Proposed method", step 6, carried across the split in both directions),
 * at the piece's given forward output out, den_in (its rows of the whole sequence's
 * forward).  S_in [BH][F][Dv], z_in [BH][F]: the sum of phi(k_j) [v_j, 1] over the tokens
 * before the piece; G_in [BH][F][Dv], zg_in [BH][F]: the sum of phi(q_i) [dn_i, delta_i] over
 * the tokens after it (NULL = zero).  The whole-sequence derivative of
 * orc_attn_causal_bwd_given, restricted to the piece's rows, is then
 *   dphi(q_i) = sum_{j<=i in the piece} c_ij phi(k_j) + S_in dn_i + z_in delta_i
 *   dphi(k_j) = sum_{i>=j in the piece} c_ij phi(q_i) + G_in v_j + zg_in
 *   dv_j      = sum_{i>=j in the piece} a_ij dn_i + G_in^T phi(k_j)
 * G_out, zg_out (NULL = not wanted): the piece's own sum of phi(q_i) [dn_i, delta_i], the
 * G_in of the pieces before it. */
void orc_attn_causal_bwd_state(const double* q, const double* k, const double* v,
                               const double* out, const double* den_in, const double* dout,
                               const double* S_in, const double* z_in,
                               const double* G_in, const double* zg_in,
                               int B, int H, int L, int D, int Dv, int R, int m,
                               const double* omega, const double* anchors,
                               const double* s, const double* wt, double eps,
                               double* dq, double* dk, double* dv,
                               double* G_out, double* zg_out)
{
    const int64_t F = (int64_t)R * m;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < B * H; ++bh) {
        const double* qs = q + (int64_t)bh * L * D;
        const double* ks = k + (int64_t)bh * L * D;
        const double* vs = v + (int64_t)bh * L * Dv;
        const double* os = out + (int64_t)bh * L * Dv;
        const double* ds = den_in + (int64_t)bh * L;
        const double* gs = dout + (int64_t)bh * L * Dv;
        const double* Si = S_in ? S_in + (int64_t)bh * F * Dv : NULL;
        const double* zi = z_in ? z_in + (int64_t)bh * F : NULL;
        const double* Gi = G_in ? G_in + (int64_t)bh * F * Dv : NULL;
        const double* zgi = zg_in ? zg_in + (int64_t)bh * F : NULL;
        double* pq = phi_slice(qs, L, D, R, m, omega, anchors, s, wt);
        double* pk = phi_slice(ks, L, D, R, m, omega, anchors, s, wt);
        double* dn = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1) * Dv);
        double* delta = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
        for (int i = 0; i < L; ++i) {
            double Z = ds[i] + eps;
            for (int e = 0; e < Dv; ++e) dn[(int64_t)i * Dv + e] = gs[(int64_t)i * Dv + e] / Z;
            delta[i] = -dot(gs + (int64_t)i * Dv, os + (int64_t)i * Dv, Dv) / Z;
        }
        double* dpq = (double*)calloc((size_t)(L > 0 ? L : 1) * F, sizeof(double));
        double* dpk = (double*)calloc((size_t)(L > 0 ? L : 1) * F, sizeof(double));
        double* dvs = dv + (int64_t)bh * L * Dv;
        for (int64_t t = 0; t < (int64_t)L * Dv; ++t) dvs[t] = 0.0;
        /* the piece's own pairs */
        for (int i = 0; i < L; ++i) {
            for (int j = 0; j <= i; ++j) {
                double c = dot(vs + (int64_t)j * Dv, dn + (int64_t)i * Dv, Dv) + delta[i];
                double a = dot(pq + (int64_t)i * F, pk + (int64_t)j * F, F);
                for (int64_t f = 0; f < F; ++f) {
                    dpq[(int64_t)i * F + f] += c * pk[(int64_t)j * F + f];
                    dpk[(int64_t)j * F + f] += c * pq[(int64_t)i * F + f];
                }
                for (int e = 0; e < Dv; ++e)
                    dvs[(int64_t)j * Dv + e] += a * dn[(int64_t)i * Dv + e];
            }
        }
        /* the pairs with tokens before the piece (through S_in, z_in) and after it (G_in,
         * zg_in) */
        for (int i = 0; i < L; ++i) {
            for (int64_t f = 0; f < F; ++f) {
                double sq = 0.0, sk = 0.0;
                if (Si) sq = dot(Si + f * Dv, dn + (int64_t)i * Dv, Dv) + zi[f] * delta[i];
                if (Gi) sk = dot(Gi + f * Dv, vs + (int64_t)i * Dv, Dv) + zgi[f];
                dpq[(int64_t)i * F + f] += sq;
                dpk[(int64_t)i * F + f] += sk;
            }
            if (Gi)
                for (int e = 0; e < Dv; ++e) {
                    double acc = 0.0;
                    for (int64_t f = 0; f < F; ++f) acc += Gi[f * Dv + e] * pk[(int64_t)i * F + f];
                    dvs[(int64_t)i * Dv + e] += acc;
                }
        }
        for (int i = 0; i < L; ++i) {
            phi_backward_row(qs + (int64_t)i * D, dpq + (int64_t)i * F, D, R, m,
                             omega, anchors, s, wt, dq + ((int64_t)bh * L + i) * D);
            phi_backward_row(ks + (int64_t)i * D, dpk + (int64_t)i * F, D, R, m,
                             omega, anchors, s, wt, dk + ((int64_t)bh * L + i) * D);
        }
        if (G_out)
            for (int64_t f = 0; f < F; ++f)
                for (int e = 0; e < Dv; ++e) {
                    double acc = 0.0;
                    for (int i = 0; i < L; ++i) acc += pq[(int64_t)i * F + f] * dn[(int64_t)i * Dv + e];
                    G_out[((int64_t)bh * F + f) * Dv + e] = acc;
                }
        if (zg_out)
            for (int64_t f = 0; f < F; ++f) {
                double acc = 0.0;
                for (int i = 0; i < L; ++i) acc += pq[(int64_t)i * F + f] * delta[i];
                zg_out[(int64_t)bh * F + f] = acc;
            }
        free(pq); free(pk); free(dn); free(delta); free(dpq); free(dpk);
    }
}

/* orc_attn_causal_bwd_given at the listed rows only (rows[r] is a query row for dq and a
 * key row for dk, dv), for sequences too long for the full form. */
void orc_attn_causal_bwd_given_rows(const double* q, const double* k, const double* v,
                                    const double* out, const double* den_in,
                                    const double* dout,
                                    int B, int H, int L, int D, int Dv, int R, int m,
                                    const double* omega, const double* anchors,
                                    const double* s, const double* wt, double eps,
                                    const int64_t* rows, int nrows,
                                    double* dq_rows, double* dk_rows, double* dv_rows)
{
    const int64_t F = (int64_t)R * m;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < B * H; ++bh) {
        const double* qs = q + (int64_t)bh * L * D;
        const double* ks = k + (int64_t)bh * L * D;
        const double* vs = v + (int64_t)bh * L * Dv;
        const double* os = out + (int64_t)bh * L * Dv;
        const double* ds = den_in + (int64_t)bh * L;
        const double* gs = dout + (int64_t)bh * L * Dv;
        double* pq = phi_slice(qs, L, D, R, m, omega, anchors, s, wt);
        double* pk = phi_slice(ks, L, D, R, m, omega, anchors, s, wt);
        double* dn = (double*)malloc(sizeof(double) * (size_t)L * Dv);
        double* delta = (double*)malloc(sizeof(double) * (size_t)L);
        for (int i = 0; i < L; ++i) {
            double Z = ds[i] + eps;
            for (int e = 0; e < Dv; ++e) dn[(int64_t)i * Dv + e] = gs[(int64_t)i * Dv + e] / Z;
            delta[i] = -dot(gs + (int64_t)i * Dv, os + (int64_t)i * Dv, Dv) / Z;
        }
        double* dph = (double*)malloc(sizeof(double) * (size_t)F);
        for (int r = 0; r < nrows; ++r) {
            int i = (int)rows[r];
            for (int64_t f = 0; f < F; ++f) dph[f] = 0.0;
            for (int j = 0; j <= i; ++j) {
                double c = dot(vs + (int64_t)j * Dv, dn + (int64_t)i * Dv, Dv) + delta[i];
                for (int64_t f = 0; f < F; ++f) dph[f] += c * pk[(int64_t)j * F + f];
            }
            phi_backward_row(qs + (int64_t)i * D, dph, D, R, m, omega, anchors, s, wt,
                             dq_rows + ((int64_t)bh * nrows + r) * D);
            int j = i;
            double* dvr = dv_rows + ((int64_t)bh * nrows + r) * Dv;
            for (int e = 0; e < Dv; ++e) dvr[e] = 0.0;
            for (int64_t f = 0; f < F; ++f) dph[f] = 0.0;
            for (int ii = j; ii < L; ++ii) {
                double c = dot(vs + (int64_t)j * Dv, dn + (int64_t)ii * Dv, Dv) + delta[ii];
                double a = dot(pq + (int64_t)ii * F, pk + (int64_t)j * F, F);
                for (int64_t f = 0; f < F; ++f) dph[f] += c * pq[(int64_t)ii * F + f];
                for (int e = 0; e < Dv; ++e) dvr[e] += a * dn[(int64_t)ii * Dv + e];
            }
            phi_backward_row(ks + (int64_t)j * D, dph, D, R, m, omega, anchors, s, wt,
                             dk_rows + ((int64_t)bh * nrows + r) * D);
        }
        free(dph); free(pq); free(pk); free(dn); free(delta);
    }
}

void orc_attn_causal_bwd_rows(const double* q, const double* k, const double* v,
                              const double* dout,
                              int B, int H, int L, int D, int Dv, int R, int m,
                              const double* omega, const double* anchors,
                              const double* s, const double* wt, double eps,
                              const int64_t* rows, int nrows,
                              double* dq_rows, double* dk_rows, double* dv_rows)
{
    const int64_t F = (int64_t)R * m;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < B * H; ++bh) {
        const double* qs = q + (int64_t)bh * L * D;
        const double* ks = k + (int64_t)bh * L * D;
        const double* vs = v + (int64_t)bh * L * Dv;
        const double* gs = dout + (int64_t)bh * L * Dv;
        double* pq = phi_slice(qs, L, D, R, m, omega, anchors, s, wt);
        double* pk = phi_slice(ks, L, D, R, m, omega, anchors, s, wt);
        double* outv = (double*)malloc(sizeof(double) * (size_t)L * Dv);
        double* den = (double*)malloc(sizeof(double) * (size_t)L);
        recurrent_slice(pq, pk, vs, L, Dv, F, eps, 1, outv, den);
        double* dn = (double*)malloc(sizeof(double) * (size_t)L * Dv);
        double* delta = (double*)malloc(sizeof(double) * (size_t)L);
        for (int i = 0; i < L; ++i) {
            double Z = den[i] + eps;
            for (int e = 0; e < Dv; ++e) dn[(int64_t)i * Dv + e] = gs[(int64_t)i * Dv + e] / Z;
            delta[i] = -dot(gs + (int64_t)i * Dv, outv + (int64_t)i * Dv, Dv) / Z;
        }
        double* dph = (double*)malloc(sizeof(double) * (size_t)F);
        for (int r = 0; r < nrows; ++r) {
            int i = (int)rows[r];
            /* dq at query row i */
            for (int64_t f = 0; f < F; ++f) dph[f] = 0.0;
            for (int j = 0; j <= i; ++j) {
                double c = dot(vs + (int64_t)j * Dv, dn + (int64_t)i * Dv, Dv) + delta[i];
                for (int64_t f = 0; f < F; ++f) dph[f] += c * pk[(int64_t)j * F + f];
            }
            phi_backward_row(qs + (int64_t)i * D, dph, D, R, m, omega, anchors, s, wt,
                             dq_rows + ((int64_t)bh * nrows + r) * D);
            /* dk, dv at key row j = i */
            int j = i;
            double* dvr = dv_rows + ((int64_t)bh * nrows + r) * Dv;
            for (int e = 0; e < Dv; ++e) dvr[e] = 0.0;
            for (int64_t f = 0; f < F; ++f) dph[f] = 0.0;
            for (int ii = j; ii < L; ++ii) {
                double c = dot(vs + (int64_t)j * Dv, dn + (int64_t)ii * Dv, Dv) + delta[ii];
                double a = dot(pq + (int64_t)ii * F, pk + (int64_t)j * F, F);
                for (int64_t f = 0; f < F; ++f) dph[f] += c * pq[(int64_t)ii * F + f];
                for (int e = 0; e < Dv; ++e) dvr[e] += a * dn[(int64_t)ii * Dv + e];
            }
            phi_backward_row(ks + (int64_t)j * D, dph, D, R, m, omega, anchors, s, wt,
                             dk_rows + ((int64_t)bh * nrows + r) * D);
        }
        free(dph); free(pq); free(pk); free(outv); free(den); free(dn); free(delta);
    }
}

/* The feature map's backward on its own: dx[n][D] from dphi[n][F] row by row through
 * phi_backward_row (the derivative of phi, steps 1, 3 and 5 of the review's "Proposed
 * method"; the pages give no backward). */
void orc_feature_map_bwd(const double* x, const double* dphi, int64_t n, int D, int R, int m,
                         const double* omega, const double* anchors, const double* s,
                         const double* wt, double* dx)
{
    const int64_t F = (int64_t)R * m;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        phi_backward_row(x + i * D, dphi + i * F, D, R, m, omega, anchors, s, wt, dx + i * D);
}

/* Backward of the bidirectional forward: out_i = num_i / Z_i with num_i = sum_j a_ij v_j and
 * Z_i = sum_j a_ij + eps over ALL keys j, a_ij = <phi(q_i), phi(k_j)>.  As in the causal
 * case (dn_i = g_i/Z_i, delta_i = -<g_i, out_i>/Z_i, c_ij = <v_j, dn_i> + delta_i), without
 * the mask:
 *   dphi(q_i) = sum_j c_ij phi(k_j),  dphi(k_j) = sum_i c_ij phi(q_i),  dv_j = sum_i a_ij dn_i. */
void orc_attn_bidir_bwd(const double* q, const double* k, const double* v, const double* dout,
                        int B, int H, int L, int D, int Dv, int R, int m,
                        const double* omega, const double* anchors,
                        const double* s, const double* wt, double eps,
                        double* dq, double* dk, double* dv)
{
    const int64_t F = (int64_t)R * m;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < B * H; ++bh) {
        const double* qs = q + (int64_t)bh * L * D;
        const double* ks = k + (int64_t)bh * L * D;
        const double* vs = v + (int64_t)bh * L * Dv;
        const double* gs = dout + (int64_t)bh * L * Dv;
        double* pq = phi_slice(qs, L, D, R, m, omega, anchors, s, wt);
        double* pk = phi_slice(ks, L, D, R, m, omega, anchors, s, wt);
        double* outv = (double*)malloc(sizeof(double) * (size_t)L * Dv);
        double* den = (double*)malloc(sizeof(double) * (size_t)L);
        for (int i = 0; i < L; ++i)
            quad_row(pq + (int64_t)i * F, pk, vs, L, Dv, F, eps, 0, i,
                     outv + (int64_t)i * Dv, den + i);
        double* dn = (double*)malloc(sizeof(double) * (size_t)L * Dv);
        double* delta = (double*)malloc(sizeof(double) * (size_t)L);
        for (int i = 0; i < L; ++i) {
            double Z = den[i] + eps;
            for (int e = 0; e < Dv; ++e) dn[(int64_t)i * Dv + e] = gs[(int64_t)i * Dv + e] / Z;
            delta[i] = -dot(gs + (int64_t)i * Dv, outv + (int64_t)i * Dv, Dv) / Z;
        }
        double* dpq = (double*)calloc((size_t)L * F, sizeof(double));
        double* dpk = (double*)calloc((size_t)L * F, sizeof(double));
        double* dvs = dv + (int64_t)bh * L * Dv;
        for (int64_t t = 0; t < (int64_t)L * Dv; ++t) dvs[t] = 0.0;
        for (int i = 0; i < L; ++i) {
            for (int j = 0; j < L; ++j) {
                double c = dot(vs + (int64_t)j * Dv, dn + (int64_t)i * Dv, Dv) + delta[i];
                double a = dot(pq + (int64_t)i * F, pk + (int64_t)j * F, F);
                for (int64_t f = 0; f < F; ++f) {
                    dpq[(int64_t)i * F + f] += c * pk[(int64_t)j * F + f];
                    dpk[(int64_t)j * F + f] += c * pq[(int64_t)i * F + f];
                }
                for (int e = 0; e < Dv; ++e)
                    dvs[(int64_t)j * Dv + e] += a * dn[(int64_t)i * Dv + e];
            }
        }
        for (int i = 0; i < L; ++i) {
            phi_backward_row(qs + (int64_t)i * D, dpq + (int64_t)i * F, D, R, m,
                             omega, anchors, s, wt, dq + ((int64_t)bh * L + i) * D);
            phi_backward_row(ks + (int64_t)i * D, dpk + (int64_t)i * F, D, R, m,
                             omega, anchors, s, wt, dk + ((int64_t)bh * L + i) * D);
        }
        free(pq); free(pk); free(outv); free(den); free(dn); free(delta);
        free(dpq); free(dpk);
    }
}

/* orc_attn_bidir_bwd at a GIVEN forward output (out [B,H,L,Dv], den [B,H,L] as inputs, as
 * the library's backward receives them); with the exact output it is orc_attn_bidir_bwd. */
void orc_attn_bidir_bwd_given(const double* q, const double* k, const double* v,
                              const double* out, const double* den_in, const double* dout,
                              int B, int H, int L, int D, int Dv, int R, int m,
                              const double* omega, const double* anchors,
                              const double* s, const double* wt, double eps,
                              double* dq, double* dk, double* dv)
{
    const int64_t F = (int64_t)R * m;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < B * H; ++bh) {
        const double* qs = q + (int64_t)bh * L * D;
        const double* ks = k + (int64_t)bh * L * D;
        const double* vs = v + (int64_t)bh * L * Dv;
        const double* os = out + (int64_t)bh * L * Dv;
        const double* ds = den_in + (int64_t)bh * L;
        const double* gs = dout + (int64_t)bh * L * Dv;
        double* pq = phi_slice(qs, L, D, R, m, omega, anchors, s, wt);
        double* pk = phi_slice(ks, L, D, R, m, omega, anchors, s, wt);
        double* dn = (double*)malloc(sizeof(double) * (size_t)L * Dv);
        double* delta = (double*)malloc(sizeof(double) * (size_t)L);
        for (int i = 0; i < L; ++i) {
            double Z = ds[i] + eps;
            for (int e = 0; e < Dv; ++e) dn[(int64_t)i * Dv + e] = gs[(int64_t)i * Dv + e] / Z;
            delta[i] = -dot(gs + (int64_t)i * Dv, os + (int64_t)i * Dv, Dv) / Z;
        }
        double* dpq = (double*)calloc((size_t)L * F, sizeof(double));
        double* dpk = (double*)calloc((size_t)L * F, sizeof(double));
        double* dvs = dv + (int64_t)bh * L * Dv;
        for (int64_t t = 0; t < (int64_t)L * Dv; ++t) dvs[t] = 0.0;
        for (int i = 0; i < L; ++i) {
            for (int j = 0; j < L; ++j) {
                double c = dot(vs + (int64_t)j * Dv, dn + (int64_t)i * Dv, Dv) + delta[i];
                double a = dot(pq + (int64_t)i * F, pk + (int64_t)j * F, F);
                for (int64_t f = 0; f < F; ++f) {
                    dpq[(int64_t)i * F + f] += c * pk[(int64_t)j * F + f];
                    dpk[(int64_t)j * F + f] += c * pq[(int64_t)i * F + f];
                }
                for (int e = 0; e < Dv; ++e)
                    dvs[(int64_t)j * Dv + e] += a * dn[(int64_t)i * Dv + e];
            }
        }
        for (int i = 0; i < L; ++i) {
            phi_backward_row(qs + (int64_t)i * D, dpq + (int64_t)i * F, D, R, m,
                             omega, anchors, s, wt, dq + ((int64_t)bh * L + i) * D);
            phi_backward_row(ks + (int64_t)i * D, dpk + (int64_t)i * F, D, R, m,
                             omega, anchors, s, wt, dk + ((int64_t)bh * L + i) * D);
        }
        free(pq); free(pk); free(dn); free(delta); free(dpq); free(dpk);
    }
}

/* The linear-attention contraction on given features (review, "Proposed method", step 6,
 * as its plain masked sum): out_i = sum_{j in J(i)} (pq_i . pk_j) v_j / (sum_{j in J(i)}
 * pq_i . pk_j + eps), J(i) = {j <= i} (causal) or all j.  pq, pk: [B,H,L,F]. */
void orc_attn_from_phi(const double* pq, const double* pk, const double* v,
                       int B, int H, int L, int F, int Dv, double eps, int causal,
                       double* out, double* den)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < B * H; ++bh) {
        const double* qs = pq + (int64_t)bh * L * F;
        const double* ks = pk + (int64_t)bh * L * F;
        const double* vs = v + (int64_t)bh * L * Dv;
        for (int i = 0; i < L; ++i)
            quad_row(qs + (int64_t)i * F, ks, vs, L, Dv, F, eps, causal, i,
                     out + ((int64_t)bh * L + i) * Dv, den + (int64_t)bh * L + i);
    }
}

/* The causal recurrence continued from a given state (review, "Proposed method", step 6:
 * the prefix state carries everything the earlier tokens contribute; abstract: O(L) time and
 * memory).  Per (b,h): S = S0, z = z0; for each token i: S += phi(k_i) v_i^T, z += phi(k_i),
 * out_i = phi(q_i)^T S / (phi(q_i)^T z + eps); S1, z1 = the state after the last token.
 * S0, z0: [B,H,F,Dv], [B,H,F] (NULL = zero); S1, z1 may be NULL. */
void orc_attn_causal_state(const double* q, const double* k, const double* v,
                           const double* S0, const double* z0,
                           int B, int H, int L, int D, int Dv, int R, int m,
                           const double* omega, const double* anchors,
                           const double* s, const double* wt, double eps,
                           double* out, double* den, double* S1, double* z1)
{
    const int64_t F = (int64_t)R * m;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < B * H; ++bh) {
        double* pq = phi_slice(q + (int64_t)bh * L * D, L, D, R, m, omega, anchors, s, wt);
        double* pk = phi_slice(k + (int64_t)bh * L * D, L, D, R, m, omega, anchors, s, wt);
        const double* vs = v + (int64_t)bh * L * Dv;
        double* S = (double*)calloc((size_t)F * (size_t)Dv, sizeof(double));
        double* z = (double*)calloc((size_t)F, sizeof(double));
        if (S0) for (int64_t t = 0; t < F * Dv; ++t) S[t] = S0[(int64_t)bh * F * Dv + t];
        if (z0) for (int64_t f = 0; f < F; ++f) z[f] = z0[(int64_t)bh * F + f];
        for (int i = 0; i < L; ++i) {
            for (int64_t f = 0; f < F; ++f) {
                double a = pk[(int64_t)i * F + f];
                z[f] += a;
                for (int e = 0; e < Dv; ++e) S[f * Dv + e] += a * vs[(int64_t)i * Dv + e];
            }
            const double* p = pq + (int64_t)i * F;
            double d = dot(p, z, F);
            for (int e = 0; e < Dv; ++e) {
                double acc = 0.0;
                for (int64_t f = 0; f < F; ++f) acc += p[f] * S[f * Dv + e];
                out[((int64_t)bh * L + i) * Dv + e] = acc / (d + eps);
            }
            if (den) den[(int64_t)bh * L + i] = d;
        }
        if (S1) for (int64_t t = 0; t < F * Dv; ++t) S1[(int64_t)bh * F * Dv + t] = S[t];
        if (z1) for (int64_t f = 0; f < F; ++f) z1[(int64_t)bh * F + f] = z[f];
        free(pq); free(pk); free(S); free(z);
    }
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
