/*
 * slay_oracle.h -- plain fp64 CPU oracle for SLAY (spherical Yat-kernel linear
 * attention).  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the
 * benchmark's CPU-baseline leg may call it; the library never does.
 *
 * Sources (cited by page title and section):
 *   [ABS] "SLAY: Geometry-Aware Spherical Linearized Attention with Yat-Kernel",
 *         arXiv 2602.04915, abstract (paperdance card): unit-sphere q/k, Bernstein
 *         mixture of polynomial-exponential kernels, strictly positive random
 *         features, O(L) attention, non-negative scores, PD + bounded kernel.
 *   [REV] the nubint.ai review of the same paper, section "Proposed method"
 *         (six steps: sphere, Laplace/Bernstein, PRF + anchor features,
 *         Gauss-Laguerre, tensor sketch, linear contraction without an LxL matrix).
 *   [PHX] Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy as 1, 2, 3",
 *         SC'11 -- definition of the Philox4x32-10 counter-based generator.
 *
 * Every array is fp64 and row-major; a tensor [B,H,L,D] has D innermost.
 * Parity status of each function is listed in the .c file header.
 */
#ifndef SLAY_ORACLE_H
#define SLAY_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* [PHX] Philox4x32 with 10 rounds: out = philox(ctr, key). */
void orc_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]);

/* R-point Gauss-Laguerre rule for weight e^{-t} on [0,inf): nodes t[R], weights w[R].
 * Found by bracketing sign changes of L_R on a fine grid and Newton/bisection.
 * Returns 0 on success, -1 if R is out of [1,64] or a root was missed. */
int orc_gauss_laguerre(int R, double* t, double* w);

/* Sketch parameters drawn from `seed`:
 *   omega[F*D]  : omega_{f,d} ~ N(0,1), rounded to fp32 (stored widened in double)
 *   anchors[F*D]: a_{f,d} ~ N(0,1)/sqrt(D), rounded to fp32
 *   s[R], wt[R] : quadrature after t = (2+eps)s:  s_r = t_r/(2+eps), wt_r = w_r/(2+eps)
 * Counter of each draw = (idx, tag, 0, 0) with idx = f*D + d, tag 0 for omega and
 * 1 for anchors; key = (seed low 32 bits, seed high 32 bits).  One normal per
 * counter by Box-Muller on the first two outputs.  Returns 0 or -1 (bad R). */
int orc_sketch_params(int D, int R, int m, uint64_t seed, double eps,
                      double* omega, double* anchors, double* s, double* wt);

/* The spherical Yat kernel x^2 / (2 - 2x + eps), x = <q^, k^> ([ABS]). */
double orc_yat_kernel(double x, double eps);
/* Its R-node quadrature with exact x^2 and no random features:
 *   sum_r wt_r x^2 exp(2 s_r x). */
double orc_quad_kernel(double x, int R, double eps);

/* phi[n, F] for rows x[n, D] ([REV] steps 1, 3, 4, 5):
 *   x^ = x / max(|x|, 1e-12)
 *   phi_{r*m+j} = sqrt(wt_r/m) * exp(sqrt(2 s_r) <omega_{rj}, x^> - s_r) * <a_{rj}, x^>^2 */
void orc_feature_map(const double* x, int64_t n, int D, int R, int m,
                     const double* omega, const double* anchors,
                     const double* s, const double* wt, double* phi);

/* Attention by the plain quadratic definition ([REV] step 6 computes this same sum
 * without forming LxL):
 *   a_ij = <phi(q_i), phi(k_j)>,  J(i) = {j <= i} (causal) or all j (bidirectional)
 *   den_i = sum_{j in J(i)} a_ij,  out_i = sum_{j in J(i)} a_ij v_j / (den_i + eps)
 * q,k [B,H,L,D], v [B,H,L,Dv] -> out [B,H,L,Dv], den [B,H,L] (den may be NULL). */
void orc_attn_quadratic(const double* q, const double* k, const double* v,
                        int B, int H, int L, int D, int Dv, int R, int m,
                        const double* omega, const double* anchors,
                        const double* s, const double* wt, double eps, int causal,
                        double* out, double* den);

/* Same definition evaluated only at query rows rows[0..nrows) of every (b,h):
 * out_rows [B,H,nrows,Dv], den_rows [B,H,nrows]. */
void orc_attn_quadratic_rows(const double* q, const double* k, const double* v,
                             int B, int H, int L, int D, int Dv, int R, int m,
                             const double* omega, const double* anchors,
                             const double* s, const double* wt, double eps, int causal,
                             const int64_t* rows, int nrows,
                             double* out_rows, double* den_rows);

/* The O(L) prefix-state form ([ABS] linear time; [REV] step 6):
 *   S_i = sum_{j<=i} phi(k_j) v_j^T, z_i = sum_{j<=i} phi(k_j),
 *   out_i = phi(q_i)^T S_i / (phi(q_i)^T z_i + eps); bidirectional uses S_L, z_L. */
void orc_attn_recurrent(const double* q, const double* k, const double* v,
                        int B, int H, int L, int D, int Dv, int R, int m,
                        const double* omega, const double* anchors,
                        const double* s, const double* wt, double eps, int causal,
                        double* out, double* den);

/* One recurrent decode step per (b,h), state updated in place, inclusive:
 *   S += phi(k) v^T; z += phi(k); out = phi(q)^T S / (phi(q)^T z + eps)
 * q,k [N,D], v [N,Dv], S [N,F,Dv], z [N,F], out [N,Dv], N = batch*heads. */
void orc_decode_step(const double* q, const double* k, const double* v,
                     double* S, double* z, double* out,
                     int N, int D, int Dv, int R, int m,
                     const double* omega, const double* anchors,
                     const double* s, const double* wt, double eps);

/* Gradient of sum_i <dout_i, out_i> for the causal form with respect to q, k, v,
 * by differentiating the quadratic definition (the pages give no backward).
 * Recomputes the forward itself.  dq,dk [B,H,L,D], dv [B,H,L,Dv]. */
void orc_attn_causal_bwd(const double* q, const double* k, const double* v,
                         const double* dout,
                         int B, int H, int L, int D, int Dv, int R, int m,
                         const double* omega, const double* anchors,
                         const double* s, const double* wt, double eps,
                         double* dq, double* dk, double* dv);

/* The same gradients at rows[0..nrows) only (dq at query rows, dk/dv at key rows);
 * out/den of every row come from the O(L) form above.
 * dq_rows, dk_rows [B,H,nrows,D], dv_rows [B,H,nrows,Dv]. */
/* The backward at a given forward output (out, den are inputs, as to the library's
 * backward): see slay_oracle.c. */
void orc_attn_causal_bwd_given(const double* q, const double* k, const double* v,
                               const double* out, const double* den, const double* dout,
                               int B, int H, int L, int D, int Dv, int R, int m,
                               const double* omega, const double* anchors,
                               const double* s, const double* wt, double eps,
                               double* dq, double* dk, double* dv);
void orc_attn_causal_bwd_state(const double* q, const double* k, const double* v,
                               const double* out, const double* den_in, const double* dout,
                               const double* S_in, const double* z_in,
                               const double* G_in, const double* zg_in,
                               int B, int H, int L, int D, int Dv, int R, int m,
                               const double* omega, const double* anchors,
                               const double* s, const double* wt, double eps,
                               double* dq, double* dk, double* dv,
                               double* G_out, double* zg_out);
void orc_attn_causal_bwd_given_rows(const double* q, const double* k, const double* v,
                                    const double* out, const double* den,
                                    const double* dout,
                                    int B, int H, int L, int D, int Dv, int R, int m,
                                    const double* omega, const double* anchors,
                                    const double* s, const double* wt, double eps,
                                    const int64_t* rows, int nrows,
                                    double* dq_rows, double* dk_rows, double* dv_rows);
void orc_attn_causal_bwd_rows(const double* q, const double* k, const double* v,
                              const double* dout,
                              int B, int H, int L, int D, int Dv, int R, int m,
                              const double* omega, const double* anchors,
                              const double* s, const double* wt, double eps,
                              const int64_t* rows, int nrows,
                              double* dq_rows, double* dk_rows, double* dv_rows);

/* Number of OpenMP threads the oracle uses (1 when built without OpenMP). */
/* Feature-map backward (dx from dphi, row by row) and the bidirectional backward: see
 * slay_oracle.c. */
void orc_feature_map_bwd(const double* x, const double* dphi, int64_t n, int D, int R, int m,
                         const double* omega, const double* anchors, const double* s,
                         const double* wt, double* dx);
void orc_attn_bidir_bwd(const double* q, const double* k, const double* v, const double* dout,
                        int B, int H, int L, int D, int Dv, int R, int m,
                        const double* omega, const double* anchors,
                        const double* s, const double* wt, double eps,
                        double* dq, double* dk, double* dv);
void orc_attn_bidir_bwd_given(const double* q, const double* k, const double* v,
                              const double* out, const double* den, const double* dout,
                              int B, int H, int L, int D, int Dv, int R, int m,
                              const double* omega, const double* anchors,
                              const double* s, const double* wt, double eps,
                              double* dq, double* dk, double* dv);
int orc_sketch_params_kind(int D, int R, int m, uint64_t seed, double eps, int kind, int head,
                           double* omega, double* anchors, double* anchors_b, double* s,
                           double* wt);
void orc_feature_map_kind(const double* x, int64_t n, int D, int R, int m,
                          const double* omega, const double* anchors, const double* anchors_b,
                          const double* s, const double* wt, int kind, double* phi);
void orc_attn_from_phi(const double* pq, const double* pk, const double* v,
                       int B, int H, int L, int F, int Dv, double eps, int causal,
                       double* out, double* den);
void orc_attn_causal_state(const double* q, const double* k, const double* v,
                           const double* S0, const double* z0,
                           int B, int H, int L, int D, int Dv, int R, int m,
                           const double* omega, const double* anchors,
                           const double* s, const double* wt, double eps,
                           double* out, double* den, double* S1, double* z1);
int orc_num_threads(void);

#ifdef __cplusplus
}
#endif
#endif
