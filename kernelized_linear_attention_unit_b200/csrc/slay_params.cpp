// slay_params.cpp -- host-side quadrature rule and seeded sketch draw of libslay.so.
//
// "SLAY: Geometry-Aware Spherical Linearized Attention with Yat-Kernel", review
// (nubint.ai), "Proposed method": step 4 discretises the Laplace integral with a
// Gauss-Laguerre rule; steps 3 and 5 draw the random exponential and anchor features
// that the tensor sketch multiplies.  The draw follows Philox4x32-10 from its
// definition (Salmon, Moraes, Dror, Shaw, SC'11) and Box-Muller.
//
// The Gauss-Laguerre rule here is computed the Golub-Welsch way: the nodes are the
// eigenvalues of the symmetric tridiagonal Jacobi matrix of the Laguerre polynomials
// (diagonal 2k+1, off-diagonal k), isolated by Sturm-sequence bisection, and the
// weights come from the Christoffel function w = 1 / sum_k L_k(t)^2 (the Laguerre
// polynomials are orthonormal for e^{-t}).
#include <algorithm>
#include <cmath>
#include <vector>
#include <cstdint>

#include "slay_internal.h"

namespace slay {

void philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    uint32_t x[4] = {ctr[0], ctr[1], ctr[2], ctr[3]};
    uint32_t k[2] = {key[0], key[1]};
    for (int i = 0; i < 10; ++i) {
        const uint64_t a = 0xD2511F53ull * x[0];
        const uint64_t b = 0xCD9E8D57ull * x[2];
        const uint32_t y0 = static_cast<uint32_t>(b >> 32) ^ x[1] ^ k[0];
        const uint32_t y1 = static_cast<uint32_t>(b);
        const uint32_t y2 = static_cast<uint32_t>(a >> 32) ^ x[3] ^ k[1];
        const uint32_t y3 = static_cast<uint32_t>(a);
        x[0] = y0; x[1] = y1; x[2] = y2; x[3] = y3;
        k[0] += 0x9E3779B9u;
        k[1] += 0xBB67AE85u;
    }
    for (int i = 0; i < 4; ++i) out[i] = x[i];
}

// Number of eigenvalues of the R x R Laguerre Jacobi matrix below `x` (Sturm count
// from the pivots of the LDL^T factorisation of J - xI).
static int sturm_count(int R, double x)
{
    int count = 0;
    double q = 1.0;
    for (int k = 0; k < R; ++k) {
        const double diag = 2.0 * k + 1.0 - x;
        const double off2 = (k == 0) ? 0.0 : static_cast<double>(k) * k;
        q = diag - ((k == 0) ? 0.0 : off2 / q);
        if (q == 0.0) q = -1e-300;
        if (q < 0.0) ++count;
    }
    return count;
}

bool gauss_laguerre(int R, double* t, double* w)
{
    if (R < 1 || R > kMaxR) return false;
    const double upper = 4.0 * R + 4.0;  // Gershgorin: every eigenvalue lies in [0, 4R]
    for (int i = 0; i < R; ++i) {
        double lo = 0.0, hi = upper;  // eigenvalue i (0-based, ascending) in (lo, hi]
        for (int it = 0; it < 200; ++it) {
            const double mid = 0.5 * (lo + hi);
            if (mid <= lo || mid >= hi) break;
            if (sturm_count(R, mid) > i) hi = mid; else lo = mid;
        }
        const double node = 0.5 * (lo + hi);
        // Christoffel weight from the orthonormal Laguerre polynomials at the node.
        double sum = 1.0, prev = 1.0, cur = 1.0 - node;
        if (R > 1) sum += cur * cur;
        for (int k = 1; k + 1 < R; ++k) {
            const double next = ((2.0 * k + 1.0 - node) * cur - k * prev) / (k + 1.0);
            prev = cur;
            cur = next;
            sum += cur * cur;
        }
        t[i] = node;
        w[i] = 1.0 / sum;
    }
    return true;
}

// Standard normal from one Philox block: counter (idx, tag, head, 0), Box-Muller on the
// first two words, each mapped to (0,1) as (word + 1/2) * 2^-32.
static double philox_normal(uint64_t seed, uint32_t idx, uint32_t tag, uint32_t head = 0)
{
    const uint32_t ctr[4] = {idx, tag, head, 0u};
    const uint32_t key[2] = {static_cast<uint32_t>(seed & 0xffffffffu),
                             static_cast<uint32_t>(seed >> 32)};
    uint32_t o[4];
    philox4x32_10(ctr, key, o);
    const double two_pi = 6.283185307179586476925286766559;
    const double u1 = (static_cast<double>(o[0]) + 0.5) * (1.0 / 4294967296.0);
    const double u2 = (static_cast<double>(o[1]) + 0.5) * (1.0 / 4294967296.0);
    return std::sqrt(-2.0 * std::log(u1)) * std::cos(two_pi * u2);
}

bool draw_sketch(int D, int R, int m, uint64_t seed, double eps, float* omega,
                 float* anchors, double* s, double* wt)
{
    double t[kMaxR], w[kMaxR];
    if (!gauss_laguerre(R, t, w)) return false;
    for (int r = 0; r < R; ++r) {
        if (s) s[r] = t[r] / (2.0 + eps);
        if (wt) wt[r] = w[r] / (2.0 + eps);
    }
    const int64_t F = static_cast<int64_t>(R) * m;
    const double rs = std::sqrt(static_cast<double>(D));
    for (int64_t f = 0; f < F; ++f)
        for (int d = 0; d < D; ++d) {
            const uint32_t idx = static_cast<uint32_t>(f * D + d);
            if (omega) omega[f * D + d] = static_cast<float>(philox_normal(seed, idx, 0u));
            if (anchors) anchors[f * D + d] = static_cast<float>(philox_normal(seed, idx, 1u) / rs);
        }
    return true;
}

bool draw_sketch_kind(int D, int R, int m, uint64_t seed, double eps, int kind, int head,
                      float* omega, float* anchors, float* anchors_b, double* s, double* wt)
{
    if (kind < 0 || kind > 4 || head < 0 || D <= 0) return false;
    double t[kMaxR], w[kMaxR];
    if (!gauss_laguerre(R, t, w)) return false;
    for (int r = 0; r < R; ++r) {
        if (s) s[r] = t[r] / (2.0 + eps);
        if (wt) wt[r] = w[r] / (2.0 + eps);
    }
    const int64_t F = static_cast<int64_t>(R) * m;
    const uint32_t h = kind == 3 ? static_cast<uint32_t>(head) : 0u;
    const double rs = std::sqrt(static_cast<double>(D));
    std::vector<double> g(static_cast<size_t>(F) * D);
    for (int64_t f = 0; f < F; ++f)
        for (int d = 0; d < D; ++d) {
            const uint32_t idx = static_cast<uint32_t>(f * D + d);
            g[f * D + d] = philox_normal(seed, idx, 0u, h);
            if (anchors) anchors[f * D + d] = static_cast<float>(philox_normal(seed, idx, 1u, h) / rs);
            if (anchors_b && kind == 2)
                anchors_b[f * D + d] = static_cast<float>(philox_normal(seed, idx, 2u, h) / rs);
        }
    if (kind == 1 || kind == 4) {
        // Blocks of D consecutive rows of a node made orthonormal by modified Gram-Schmidt
        // (each row is reduced against the finished ones one at a time), then each row
        // scaled back to the length of its own Gaussian draw.
        std::vector<double> len(static_cast<size_t>(D));
        for (int r = 0; r < R; ++r)
            for (int b0 = 0; b0 < m; b0 += D) {
                const int nb = std::min(D, m - b0);
                double* blk = g.data() + (static_cast<int64_t>(r) * m + b0) * D;
                for (int j = 0; j < nb; ++j) {
                    double* row = blk + static_cast<int64_t>(j) * D;
                    double l2 = 0.0;
                    for (int d = 0; d < D; ++d) l2 += row[d] * row[d];
                    len[j] = std::sqrt(l2);
                    for (int i = 0; i < j; ++i) {
                        const double* e = blk + static_cast<int64_t>(i) * D;
                        double c = 0.0;
                        for (int d = 0; d < D; ++d) c += row[d] * e[d];
                        for (int d = 0; d < D; ++d) row[d] -= c * e[d];
                    }
                    double n2 = 0.0;
                    for (int d = 0; d < D; ++d) n2 += row[d] * row[d];
                    const double inv = 1.0 / std::sqrt(n2);
                    for (int d = 0; d < D; ++d) row[d] *= inv;
                }
                for (int j = 0; j < nb; ++j)
                    for (int d = 0; d < D; ++d) blk[static_cast<int64_t>(j) * D + d] *= len[j];
            }
    }
    if (omega)
        for (int64_t i = 0; i < F * D; ++i) omega[i] = static_cast<float>(g[i]);
    return true;
}

}  // namespace slay
