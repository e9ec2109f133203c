/*
 * slay.h -- C ABI of libslay.so: SLAY spherical Yat-kernel linear attention on
 * NVIDIA B200 (sm_100a).
 *
 * The method ("SLAY: Geometry-Aware Spherical Linearized Attention with Yat-Kernel",
 * arXiv 2602.04915; abstract, and the nubint.ai review, section "Proposed method"):
 *   x^ = x / max(|x|, 1e-12)                           (queries/keys on the sphere)
 *   K(q,k) = x^2 / (2 - 2x + eps), x = q^ . k^         (spherical Yat kernel)
 *   1/(2-2x+eps) = int e^{-s(2+eps)} e^{2sx} ds         (Bernstein / Laplace)
 *   R-node Gauss-Laguerre rule (t_r, w_r) after t=(2+eps)s:
 *       s_r = t_r/(2+eps), wt_r = w_r/(2+eps)
 *   phi_{r*m+j}(x) = sqrt(wt_r/m) exp(sqrt(2 s_r) omega_{rj}.x^ - s_r) (a_{rj}.x^)^2
 *       (positive random feature x anchor feature, fused by an elementwise sketch)
 *   out_i = phi(q_i)^T S_i / (phi(q_i)^T z_i + eps),
 *       S_i = sum_{j in J(i)} phi(k_j) v_j^T, z_i = sum_{j in J(i)} phi(k_j)
 *   with J(i) = {j <= i} (causal) or all j (bidirectional).  F = R*m features.
 *
 * Sketch parameters: omega_{f,d} ~ N(0,1), a_{f,d} ~ N(0,1)/sqrt(D), f = r*m+j, drawn
 * from `seed` with Philox4x32-10 (Salmon et al., SC'11): counter (f*D+d, tag, 0, 0),
 * tag 0 for omega and 1 for anchors, key (seed & 0xffffffff, seed >> 32); one normal
 * per counter by Box-Muller on the first two words mapped to (0,1) as (w + 1/2) 2^-32,
 * computed in double and rounded to float.  The same draw serves q and k and every
 * batch and head.
 *
 * Conventions for every entry point:
 *   - Device pointers are caller-owned CUDA device memory; the library never frees or
 *     keeps them.  Tensors are contiguous row-major: [B,H,L,D] has D innermost.
 *     Every tensor base must be 16-byte aligned; `workspace` must be 256-byte aligned.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are
 *     asynchronous on it: a returned SLAY_OK means the work was enqueued.
 *   - dtype SLAY_F32: inputs/outputs fp32, all arithmetic fp32 on CUDA cores.
 *     dtype SLAY_BF16: q,k,v,out (and dout) bf16; arithmetic with fp32 accumulation,
 *     states S and z always fp32; gradients fp32.
 *   - Supported: D == Dv == 64, 1 <= R <= 16, 1 <= m, F = R*m <= 1024, eps > 0 and
 *     finite.  The bf16 tensor-core kernels take F % 128 == 0 and F <= 512 (the attention
 *     forward as feature chunks of at most 256 when F > 256), with m % 64 == 0 for the
 *     attention forward and m % 32 == 0 for the feature map and its backward; other sizes
 *     run on CUDA cores.
 *   - q and k rows (and the feature map's x rows) need not be unit length: every kernel
 *     projects them onto the sphere.  Supported row norms: up to 1e15.  Rows below 1e-12
 *     take the norm guard (x^ = x / 1e-12, a zero row maps to phi = 0).  The fp32 kernels
 *     divide by the norm before the projections.  The bf16 tensor-core kernels project the
 *     raw row and fold 1/|x|^2 into phi's exponent, so that exponent must stay inside
 *     fp32's range for every feature: at |x| = 2^50 (about 1e15) the row error is still
 *     fp32 rounding for R <= 16; from about 2^55 the smallest features are flushed or
 *     clamped and the error grows; at 1.8e19 the fp32 sum of squares overflows.
 *   - Errors are status codes, never exceptions or aborts.  On any error nothing is
 *     enqueued.  The library owns only its sketch-parameter cache: one small device
 *     buffer per (device, D, R, m, seed, eps), created on first use (synchronous
 *     allocation and upload; call slay_prepare before capturing a stream into a CUDA
 *     graph) and held until the process exits.  The cache is thread-safe.
 *   - Empty work (L == 0, n_rows == 0, B*H == 0) returns SLAY_OK and enqueues nothing (but
 *     for the calls whose outputs are states, which at L == 0 still write them); it leaves
 *     the workspace, and so its status word, as it was.
 */
#ifndef SLAY_H
#define SLAY_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SLAY_OK = 0,
    SLAY_ERR_INVALID_ARG = 1,   /* NULL pointer, misalignment, bad size, workspace too small */
    SLAY_ERR_UNSUPPORTED = 2,   /* a size or dtype combination this build does not offer */
    SLAY_ERR_CUDA = 3,          /* a CUDA runtime error (launch, allocation of the cache, no device) */
    SLAY_ERR_TIMEOUT = 4,       /* a kernel's bounded wait ran out (see slay_kernel_status) */
    SLAY_ERR_NO_MEMORY = 5      /* host allocation failed */
} slay_status;

typedef enum { SLAY_F32 = 0, SLAY_BF16 = 1 } slay_dtype;

typedef enum {
    SLAY_OP_FEATURE_MAP = 0,
    SLAY_OP_CAUSAL_FWD = 1,
    SLAY_OP_BIDIR_FWD = 2,
    SLAY_OP_CAUSAL_BWD = 3,
    SLAY_OP_DECODE = 4,
    SLAY_OP_BIDIR_BWD = 5,
    SLAY_OP_LINEAR_ATTN = 6,    /* slay_linear_attn_fwd: R * m = the number of features */
    SLAY_OP_CAUSAL_STATE = 7,   /* slay_causal_state */
    SLAY_OP_CAUSAL_FWD_SPLIT = 8, /* slay_attn_causal_fwd_begin / _finish (one workspace) */
    SLAY_OP_FEATURE_MAP_BWD = 9  /* slay_feature_map_bwd (no workspace; for slay_path) */
} slay_op;

/* Feature-map variants (slay_feature_map_ex).  The pages leave the form of the anchor
 * feature and of the random-feature bank open (review, "Proposed method", steps 3 and 5);
 * orthogonal banks and FAVOR+ features are prior art on the other pages and the abstract
 * compares SLAY with Performers.  Sketch draws follow the Philox spec above; "orthogonal"
 * rows are made orthonormal in blocks of D consecutive rows of a node (Gram-Schmidt in draw
 * order), each row keeping the length of its own Gaussian draw. */
typedef enum {
    SLAY_PHI_ANCHOR = 0,       /* SLAY: iid omega, positive anchor (a.x^)^2 (the default) */
    SLAY_PHI_ORTHOGONAL = 1,   /* SLAY with an orthogonal omega bank */
    SLAY_PHI_SIGNED = 2,       /* SLAY with (a.x^)(b.x^), b a second anchor set (counter tag 2):
                                  unbiased for (q^.k^)^2 / D^2, not positive */
    SLAY_PHI_PER_HEAD = 3,     /* SLAY with omega, a drawn per head h (counter (f*D+d, tag, h, 0)) */
    SLAY_PHI_PERFORMER = 4     /* Performer FAVOR+: exp(omega_f.x^ - 1/2) / sqrt(F), orthogonal
                                  omega, F = R*m features; estimates exp(q^.k^) */
} slay_phi_kind;

/* Feature map phi (review, "Proposed method", steps 1, 3, 4, 5).
 * x   : device [n_rows, D] in `in_dt` (rows need not be unit length; they are
 *       projected onto the sphere inside, a zero row maps to phi = 0).
 * phi : device [n_rows, R*m] in `out_dt`, written; feature index f = r*m + j.
 * in_dt/out_dt: (F32,F32), (BF16,BF16) or (BF16,F32).  No workspace. */
slay_status slay_feature_map(const void* x, void* phi, int64_t n_rows, int D,
                             slay_dtype in_dt, slay_dtype out_dt, int R, int m,
                             uint64_t seed, float eps, void* stream);

/* Causal SLAY attention forward (review, "Proposed method", step 6: the linear
 * contraction with prefix states, no LxL matrix; abstract: O(L) time and memory).
 * q,k : device [B,H,L,D], v : device [B,H,L,Dv], all in `dt`.
 * out : device [B,H,L,Dv] in `dt`, written.
 * den : device [B,H,L] fp32 or NULL; if given, den_i = phi(q_i)^T z_i (without eps)
 *       is written (the backward needs it).
 * workspace/ws_bytes: device scratch of at least
 *       slay_workspace_bytes(SLAY_OP_CAUSAL_FWD, dt, B, H, L, D, Dv, R, m) bytes;
 *       its contents on entry are ignored and on exit undefined. */
slay_status slay_attn_causal_fwd(const void* q, const void* k, const void* v, void* out,
                                 float* den, int B, int H, int L, int D, int Dv,
                                 slay_dtype dt, int R, int m, uint64_t seed, float eps,
                                 void* workspace, size_t ws_bytes, void* stream);

/* The causal forward continued from a state (review, "Proposed method", step 6: the
 * prefix state S_i = S_0 + sum_{j<=i} phi(k_j) v_j^T, z_i likewise, carries all earlier
 * tokens; abstract: O(L) time and memory).  With it a sequence can be processed in pieces --
 * prefill after a cached prefix, or one piece per GPU (sequence parallelism: each rank
 * takes the sum of the earlier ranks' slay_causal_state results, see slay_state_prefix).
 * Arguments as slay_attn_causal_fwd (same workspace size), plus:
 * S_in, z_in   : device [B,H,R*m,Dv] and [B,H,R*m] fp32, the state before the first token of
 *                this piece, or both NULL for a zero state (then the call equals
 *                slay_attn_causal_fwd);
 * S_out, z_out : device, same shapes, written with the state after the last token, or both
 *                NULL.  16-byte aligned.  They must not alias S_in, z_in. */
slay_status slay_attn_causal_fwd_state(const void* q, const void* k, const void* v, void* out,
                                       float* den, const float* S_in, const float* z_in,
                                       float* S_out, float* z_out, int B, int H, int L, int D,
                                       int Dv, slay_dtype dt, int R, int m, uint64_t seed,
                                       float eps, void* workspace, size_t ws_bytes, void* stream);

/* The causal state of a piece of a sequence without its outputs:
 *   S_out = S_in + sum_j phi(k_j) v_j^T,  z_out = z_in + sum_j phi(k_j)
 * over the L tokens of each (b,h) (S_in, z_in NULL: zero).  Layouts as
 * slay_attn_causal_fwd_state; workspace slay_workspace_bytes(SLAY_OP_CAUSAL_STATE, ...).
 * bf16 at tensor-core sizes: the state kernel of the causal forward over every segment
 * (phi(k) and the sums on tensor cores), then the total; otherwise CUDA cores. */
slay_status slay_causal_state(const void* k, const void* v, const float* S_in, const float* z_in,
                              float* S_out, float* z_out, int B, int H, int L, int D, int Dv,
                              slay_dtype dt, int R, int m, uint64_t seed, float eps,
                              void* workspace, size_t ws_bytes, void* stream);

/* Exclusive prefix over ranks of all-gathered piece states (sequence parallelism):
 *   S_in = sum_{r < rank} S_all[r],  z_in = sum_{r < rank} z_all[r]
 * S_all: device [nranks][BH][F][Dv] fp32, z_all: [nranks][BH][F]; S_in [BH][F][Dv],
 * z_in [BH][F] written (zero for rank 0).  F = R*m <= 1024, Dv == 64. */
slay_status slay_state_prefix(const float* S_all, const float* z_all, int nranks, int rank,
                              float* S_in, float* z_in, int BH, int F, int Dv, void* stream);

/* The sequence-parallel forward of one piece in two calls that share a workspace, so that the
 * piece's phi(k) and per-segment state sums are made once, for the exchange and the forward
 * alike (review, "Proposed method", step 6: the prefix state carries every earlier token, so
 * only the pieces' totals cross ranks).  Between the calls the caller exchanges the totals
 * and forms the prefix (slay_state_prefix).
 *
 * slay_attn_causal_fwd_begin writes this piece's state
 *     S_out = sum_j phi(k_j) v_j^T,  z_out = sum_j phi(k_j)   over its L tokens per (b,h)
 *   (slay_causal_state with S_in NULL; zero when L == 0) and leaves in `workspace` what the
 *   second call reads.  S_out [B,H,R*m,Dv], z_out [B,H,R*m] fp32, both required.
 * slay_attn_causal_fwd_finish writes out (and den, if not NULL) of the piece continued from
 *   S_in, z_in ([B,H,R*m,Dv], [B,H,R*m] fp32, or both NULL for a zero state): the values
 *   slay_attn_causal_fwd_state writes for the same arguments.  It must come after the first
 *   call in stream order, with the same k, v, B, H, L, D, Dv, dt, R, m, seed, eps and
 *   workspace, nothing else writing the workspace in between.  q, k, v, out, den as
 *   slay_attn_causal_fwd.
 * workspace: slay_workspace_bytes(SLAY_OP_CAUSAL_FWD_SPLIT, ...) bytes, caller-owned, its
 *   contents the library's from the first call to the second; its first int is the status
 *   word of both calls' tensor-core kernels (the first call clears it, the second does not).
 * bf16 at tensor-core sizes: the first call runs the causal forward's state kernel (phi(k)
 * stored, every segment's sum) and the totals, the second only its output kernel.  Otherwise
 * CUDA cores: the first call is slay_causal_state, the second slay_attn_causal_fwd_state.
 * Errors as slay_attn_causal_fwd; on an error nothing is enqueued. */
slay_status slay_attn_causal_fwd_begin(const void* k, const void* v, float* S_out, float* z_out,
                                       int B, int H, int L, int D, int Dv, slay_dtype dt, int R,
                                       int m, uint64_t seed, float eps, void* workspace,
                                       size_t ws_bytes, void* stream);
slay_status slay_attn_causal_fwd_finish(const void* q, const void* k, const void* v, void* out,
                                        float* den, const float* S_in, const float* z_in, int B,
                                        int H, int L, int D, int Dv, slay_dtype dt, int R, int m,
                                        uint64_t seed, float eps, void* workspace,
                                        size_t ws_bytes, void* stream);

/* The counterpart of slay_state_prefix for the backward (sequence parallelism):
 *   S_out = sum_{r > rank} S_all[r],  z_out = sum_{r > rank} z_all[r]
 * the sum of the states of the ranks after this one (zero for the last rank).  Layouts and
 * limits as slay_state_prefix. */
slay_status slay_state_suffix(const float* S_all, const float* z_all, int nranks, int rank,
                              float* S_out, float* z_out, int BH, int F, int Dv, void* stream);

/* Bidirectional SLAY attention forward: as above with S, z summed over all keys
 * (review, "Proposed method", step 6, non-causal form).  Same arguments; workspace
 * size from slay_workspace_bytes(SLAY_OP_BIDIR_FWD, ...). */
slay_status slay_attn_bidir_fwd(const void* q, const void* k, const void* v, void* out,
                                float* den, int B, int H, int L, int D, int Dv,
                                slay_dtype dt, int R, int m, uint64_t seed, float eps,
                                void* workspace, size_t ws_bytes, void* stream);

/* Backward of the causal forward: gradients of sum_i <dout_i, out_i> with respect to
 * q, k, v, through the contraction, the normaliser, phi and the sphere projection.
 * The pages give no backward; it is the derivative of the forward above.  omega and
 * anchors are fixed random draws and get no gradient.
 * out, den : the forward's outputs for the same inputs (out in `dt`, den fp32).
 * dout     : device [B,H,L,Dv] in `dt`.
 * dq, dk   : device [B,H,L,D] fp32, dv : device [B,H,L,Dv] fp32, all written.
 * workspace: slay_workspace_bytes(SLAY_OP_CAUSAL_BWD, ...) bytes; its first int is the
 *            status word of the tensor-core kernels (see slay_kernel_status).
 * bf16 mode with tensor-core sizes: the per-128-token-tile sums, the contraction and the
 * derivative through phi run on tensor cores with bf16 operands and fp32 accumulation;
 * dphi(q), dphi(k) pass between the last two as bf16. */
slay_status slay_attn_causal_bwd(const void* q, const void* k, const void* v,
                                 const void* out, const float* den, const void* dout,
                                 float* dq, float* dk, float* dv,
                                 int B, int H, int L, int D, int Dv,
                                 slay_dtype dt, int R, int m, uint64_t seed, float eps,
                                 void* workspace, size_t ws_bytes, void* stream);

/* Backward of one piece of a longer causal sequence (sequence parallelism: the prefix state
 * of the review's "Proposed method", step 6, split across ranks, in the backward direction).
 * Arguments as slay_attn_causal_bwd (same workspace size; out, den: this piece's rows of the
 * whole sequence's forward, e.g. from slay_attn_causal_fwd_state), plus:
 * S_in, z_in  : device [B,H,R*m,Dv] and [B,H,R*m] fp32, sum_j phi(k_j) [v_j, 1] over the tokens
 *               before the piece (the forward's S_in), or both NULL;
 * G_in, zg_in : same shapes, sum_i phi(q_i) [dn_i, delta_i] over the tokens after the piece
 *               (dn_i = dout_i / (den_i + eps), delta_i = -<dout_i, out_i> / (den_i + eps); the
 *               later ranks' slay_causal_bwd_state results summed, see slay_state_suffix), or
 *               both NULL.
 * Then dq, dk, dv of the piece's rows equal the whole sequence's.  With all four NULL the
 * call equals slay_attn_causal_bwd.  16-byte aligned. */
slay_status slay_attn_causal_bwd_state(const void* q, const void* k, const void* v,
                                       const void* out, const float* den, const void* dout,
                                       float* dq, float* dk, float* dv, const float* S_in,
                                       const float* z_in, const float* G_in, const float* zg_in,
                                       int B, int H, int L, int D, int Dv, slay_dtype dt, int R,
                                       int m, uint64_t seed, float eps, void* workspace,
                                       size_t ws_bytes, void* stream);

/* A piece's G state for the pieces before it:
 *   G_out = sum_i phi(q_i) dn_i^T,  zg_out = sum_i phi(q_i) delta_i
 * over its L tokens (dn, delta as in slay_attn_causal_bwd_state), G_out [B,H,R*m,Dv] and
 * zg_out [B,H,R*m] fp32, written (zero when L == 0).  q, out, dout in `dt`, den fp32; workspace
 * slay_workspace_bytes(SLAY_OP_CAUSAL_BWD, ...).  bf16 at tensor-core sizes: phi(q) and the
 * running sums on tensor cores; otherwise CUDA cores. */
slay_status slay_causal_bwd_state(const void* q, const void* out, const float* den,
                                  const void* dout, float* G_out, float* zg_out, int B, int H,
                                  int L, int D, int Dv, slay_dtype dt, int R, int m, uint64_t seed,
                                  float eps, void* workspace, size_t ws_bytes, void* stream);

/* The sequence-parallel backward of one piece in two calls that share a workspace, so that
 * phi(q) and the row statistics dn, delta (as in slay_attn_causal_bwd_state) are made once,
 * for the exchange and the backward alike.  Between the calls the caller
 * exchanges the G sums and forms the suffix (slay_state_suffix).
 * slay_attn_causal_bwd_begin: as slay_causal_bwd_state (same arguments, G_out and zg_out
 *   written), and it leaves phi(q) and the row statistics in `workspace`.
 * slay_attn_causal_bwd_finish: the gradients slay_attn_causal_bwd_state writes for the same
 *   arguments (same values), without recomputing phi(q) and the row statistics.  It must come
 *   after the first call in stream order, with the same q, out, den, dout, B, H, L, D, Dv, dt,
 *   R, m, seed, eps and workspace, nothing else writing the workspace in between.  It leaves
 *   the status word as the first call set it.
 * workspace: slay_workspace_bytes(SLAY_OP_CAUSAL_BWD, ...) bytes, caller-owned, its contents
 * the library's from the first call to the second.  Errors as slay_attn_causal_bwd_state. */
slay_status slay_attn_causal_bwd_begin(const void* q, const void* out, const float* den,
                                       const void* dout, float* G_out, float* zg_out, int B, int H,
                                       int L, int D, int Dv, slay_dtype dt, int R, int m,
                                       uint64_t seed, float eps, void* workspace, size_t ws_bytes,
                                       void* stream);
slay_status slay_attn_causal_bwd_finish(const void* q, const void* k, const void* v,
                                        const void* out, const float* den, const void* dout,
                                        float* dq, float* dk, float* dv, const float* S_in,
                                        const float* z_in, const float* G_in, const float* zg_in,
                                        int B, int H, int L, int D, int Dv, slay_dtype dt, int R,
                                        int m, uint64_t seed, float eps, void* workspace,
                                        size_t ws_bytes, void* stream);

/* Backward of the bidirectional forward: gradients of sum_i <dout_i, out_i> with respect
 * to q, k, v (the pages give no backward; it is the derivative of slay_attn_bidir_fwd).
 * With Z_i = den_i + eps, dn_i = dout_i / Z_i, delta_i = -<dout_i, out_i> / Z_i and the
 * whole-sequence sums S = sum_j phi(k_j) v_j^T, z = sum_j phi(k_j),
 * G = sum_i phi(q_i) dn_i^T, zg = sum_i phi(q_i) delta_i:
 *   dphi(q_i) = S dn_i + z delta_i,  dphi(k_j) = G v_j + zg,  dv_j = G^T phi(k_j),
 * then through phi and the sphere projection as in slay_attn_causal_bwd.
 * Arguments, layouts and dtypes: as slay_attn_causal_bwd (out, den: the bidirectional
 * forward's outputs for the same inputs); workspace:
 * slay_workspace_bytes(SLAY_OP_BIDIR_BWD, ...) bytes, its first int the kernel status word.
 * The sums and the per-row products run on CUDA cores in fp32; in bf16 mode phi and the
 * derivative through phi run on tensor cores where the sizes allow (as in the forward), with
 * dphi passed between them as bf16. */
slay_status slay_attn_bidir_bwd(const void* q, const void* k, const void* v,
                                const void* out, const float* den, const void* dout,
                                float* dq, float* dk, float* dv,
                                int B, int H, int L, int D, int Dv,
                                slay_dtype dt, int R, int m, uint64_t seed, float eps,
                                void* workspace, size_t ws_bytes, void* stream);

/* Feature map of a variant kind (slay_phi_kind), for the matched-feature-budget comparisons
 * and the sketch variants; arguments as slay_feature_map plus:
 *   kind          : the variant; SLAY_PHI_ANCHOR is slay_feature_map itself.
 *   heads, rows_per_head : for SLAY_PHI_PER_HEAD, the rows are sequences of rows_per_head
 *                   rows ([B,H,L,D] with rows_per_head = L) and sequence z uses head z % heads'
 *                   parameters (n_rows must be a multiple of rows_per_head); ignored otherwise.
 * Variants other than SLAY_PHI_ANCHOR run on CUDA cores in fp32; the library caches their
 * parameters per (device, D, R, m, seed, eps, kind, heads) like the default ones. */
slay_status slay_feature_map_ex(const void* x, void* phi, int64_t n_rows, int D,
                               slay_dtype in_dt, slay_dtype out_dt, int R, int m, uint64_t seed,
                               float eps, int kind, int heads, int64_t rows_per_head,
                               void* stream);

/* Host copy of a variant's sketch parameters (for tests): omega, anchors, anchors_b
 * [R*m, D] float (anchors_b only for SLAY_PHI_SIGNED; each may be NULL), s, w [R] double, for
 * head `head` (SLAY_PHI_PER_HEAD; other kinds ignore it).  Host only. */
slay_status slay_sketch_params_ex(int D, int R, int m, uint64_t seed, float eps, int kind,
                                  int head, float* omega_host, float* anchors_host,
                                  float* anchors_b_host, double* s_host, double* w_host);

/* The linear-attention contraction on given features (review, "Proposed method", step 6):
 *   out_i = sum_{j in J(i)} (phq_i . phk_j) v_j / (sum_{j in J(i)} phq_i . phk_j + eps)
 * computed in O(L) by 64-token chunks with fp32 states, J(i) = {j <= i} (causal != 0) or
 * all j.  Any feature map composes with it: slay_feature_map(_ex) for q and k, then this.
 * phq, phk : device [B,H,L,F] in dt;  v : device [B,H,L,Dv] in dt;  out : [B,H,L,Dv] in dt;
 * den      : device [B,H,L] fp32 or NULL (den_i without eps).  F <= 1024, Dv == 64.
 * workspace: slay_workspace_bytes(SLAY_OP_LINEAR_ATTN, dt, B, H, L, 64, Dv, 1, F) bytes.
 * CUDA cores, fp32 arithmetic (bf16 operands are widened on load). */
slay_status slay_linear_attn_fwd(const void* phq, const void* phk, const void* v, void* out,
                                 float* den, int B, int H, int L, int F, int Dv, slay_dtype dt,
                                 float eps, int causal, void* workspace, size_t ws_bytes,
                                 void* stream);

/* Backward of the feature map alone (review, "Proposed method", steps 1, 3, 4, 5; the
 * pages give no backward): dx = (d phi / d x)^T dphi for every row, through the sphere
 * projection (dx = (dx^ - x^ <x^, dx^>) / |x|, or dx^ / 1e-12 under the norm guard).
 * x    : device [n_rows, D] in x_dt (F32 or BF16), the rows slay_feature_map was given.
 * dphi : device [n_rows, R*m] in dphi_dt (F32 or BF16).
 * dx   : device [n_rows, D] fp32, written.  No workspace.
 * bf16 x and bf16 dphi with m % 32 == 0, F % 128 == 0, F <= 512 take the tensor-core kernel
 * (projection and its transpose on tcgen05, bf16 operands, fp32 accumulation; its bounded
 * waits report through slay_kernel_status(NULL, ...)); other combinations run on CUDA cores
 * in fp32. */
slay_status slay_feature_map_bwd(const void* x, const void* dphi, float* dx, int64_t n_rows,
                                 int D, slay_dtype x_dt, slay_dtype dphi_dt, int R, int m,
                                 uint64_t seed, float eps, void* stream);

/* One recurrent decode step for Bt*H independent sequences (abstract: linear time
 * and memory; the O(1)-per-token form of the causal contraction), inclusive:
 *   S += phi(k) v^T;  z += phi(k);  out = phi(q)^T S / (phi(q)^T z + eps)
 * q,k : device [Bt,H,D], v : device [Bt,H,Dv] in `dt`; out : device [Bt,H,Dv] in `dt`.
 * S   : device [Bt,H,F,Dv] fp32, z : device [Bt,H,F] fp32, updated in place
 *       (caller-owned; a checkpoint is a copy of S, z and the key (D,R,m,seed,eps)).
 * No workspace. */
slay_status slay_decode_step(const void* q, const void* k, const void* v,
                             float* S, float* z, void* out,
                             int Bt, int H, int D, int Dv, slay_dtype dt,
                             int R, int m, uint64_t seed, float eps, void* stream);

/* The causal forward above for callers that cannot allocate device memory: a host that
 * reserves all of HBM for its own pool at start-up, a plugin that is handed tensors but
 * no workspace, or a latency-bound loop that must not pay for cudaMalloc's implicit
 * synchronisation.  The pages of the method have no counterpart of this entry point; it
 * computes exactly what slay_attn_causal_fwd computes, with the same kernels.
 * Arguments: as slay_attn_causal_fwd without workspace/ws_bytes.
 * Memory: allocates nothing.  Its workspace is a file-scope device array of 32 MiB and its
 *   sketch parameters live in a second one of 2 MiB; every GPU that loads the library
 *   holds both (34 MiB) until the process exits.  Sizes whose workspace
 *   (slay_workspace_bytes(SLAY_OP_CAUSAL_FWD, ...)) exceeds 32 MiB are rejected with
 *   SLAY_ERR_UNSUPPORTED before anything is enqueued.
 * Set-up: the first call on a device looks up the arrays' device addresses; the first
 *   call with a new (D, R, m, seed, eps) uploads that key's parameters into the single
 *   parameter slot with a copy ordered on `stream`.  Make such calls before capturing the
 *   stream into a graph.
 * Sharing: all calls on a device share both arrays, which keep the last call's contents
 *   (no part of them needs to start at zero).  Calls that overlap on the GPU -- on
 *   different streams, or from different host threads -- race on them; calls in order on
 *   one stream do not.  The parameter upload of a call with a new key is ordered only on
 *   that call's stream: a later call with the same key on another stream must be ordered
 *   after it (an event, or a synchronisation), or it may read the slot before the copy
 *   has landed. */
slay_status slay_attn_causal_fwd_noalloc(const void* q, const void* k, const void* v,
                                         void* out, float* den, int B, int H, int L, int D,
                                         int Dv, slay_dtype dt, int R, int m, uint64_t seed,
                                         float eps, void* stream);

/* Kernel status of the last attention call that used `workspace` (or, with workspace ==
 * NULL, of the last slay_attn_causal_fwd_noalloc call and the last slay_feature_map call
 * on the current device: the library's own status words).
 * The tensor-core kernels coordinate their warps through shared-memory barriers; every
 * wait is bounded (2 s).  A wait that runs out makes the kernel stop early, leave its
 * outputs incomplete and set the status word, the first int of the workspace, which each
 * attention call clears when it is enqueued.  This call copies the word to the host on
 * `stream` and synchronizes the stream.  Returns SLAY_ERR_TIMEOUT if the word is set,
 * SLAY_OK if it is not (or if neither of those paths ran on this device),
 * SLAY_ERR_INVALID_ARG for a workspace that is not 256-byte aligned, SLAY_ERR_CUDA if the
 * copy fails.  The status of a call is only defined once it has been enqueued. */
slay_status slay_kernel_status(const void* workspace, void* stream);

/* Test hook for the failure path of the bounded waits (the pages have no counterpart;
 * off by default, for tests only).  With on != 0, the next slay_feature_map call that runs
 * the tensor-core kernel bounds every wait of that launch at 1 ms and has one warp
 * withhold one release of a projection buffer (a barrier that guards no copy or MMA in
 * flight), so that the issuing thread waits for a phase that never completes: the wait
 * runs out, the kernel stops early (its phi output is then incomplete), drains, frees its
 * tensor memory and sets the feature-map status word, which slay_kernel_status(NULL, ...)
 * reports as SLAY_ERR_TIMEOUT.  The hook disarms itself at that launch; on == 0 disarms
 * it earlier.  No GPU fault is involved and the context stays usable.  Returns SLAY_OK. */
slay_status slay_debug_expire_wait(int on);

/* Workspace bytes an entry point needs for these sizes (0 if none; SIZE_MAX if the
 * sizes are unsupported).  Feature map, its backward and decode need none. */
size_t slay_workspace_bytes(slay_op op, slay_dtype dt, int B, int H, int L, int D, int Dv,
                            int R, int m);

/* Which kernels a call takes at these sizes.  The call decides from its sizes and dtype alone,
 * by the same rule as this query, and never tells the caller: this is how to find out.
 * Returns a mask of slay_path_bit values (0: every step on the CUDA-core kernels), or -1 for
 * an op, size or dtype the call rejects.  Feature map and its backward: the rows are B*H*L
 * (pass B = H = 1, L = n_rows) and dt is the input and output dtype.  SLAY_OP_LINEAR_ATTN:
 * R*m is the number of features.  Host-only; enqueues nothing. */
typedef enum {
    SLAY_PATH_TC_FEATURE_MAP = 1,   /* phi of q and k (or x) by the tcgen05 projection: in
                                       the fused forward kernels, or the feature-map kernel
                                       ahead of CUDA-core contraction kernels */
    SLAY_PATH_TC_CONTRACTION = 2,   /* forward: state and output kernels; backward: the
                                       running sums and the contraction */
    SLAY_PATH_TC_PHI_BWD = 4        /* the chain rule through phi */
} slay_path_bit;
int slay_path(slay_op op, slay_dtype dt, int B, int H, int L, int D, int Dv, int R, int m);

/* Create (if absent) the device copy of the sketch parameters of this key on the
 * current device: synchronous; lets a caller warm the cache before stream capture. */
slay_status slay_prepare(int D, int R, int m, uint64_t seed, float eps);

/* Host copy of the sketch parameters the kernels use, for tests and checkpoints:
 * omega_host, anchors_host [R*m, D] float (each may be NULL), s_host, w_host [R] double
 * (each may be NULL): s_r = t_r/(2+eps), w_host[r] = wt_r = w_r/(2+eps).  Host only:
 * needs no GPU. */
slay_status slay_sketch_params(int D, int R, int m, uint64_t seed, float eps,
                               float* omega_host, float* anchors_host,
                               double* s_host, double* w_host);

/* Per-launch timing for profiling: while enabled (on != 0), every kernel this library
 * launches is bracketed by a pair of CUDA events recorded on its stream.  Host-side
 * bookkeeping only; results are unchanged.  Not for use during stream capture. */
slay_status slay_trace_enable(int on);

/* Waits for the recorded events, writes up to `cap` records (kernel name: a static
 * string owned by the library; duration in milliseconds, -1 if unavailable) into
 * names[] / ms[] (either may be NULL), clears the record list and returns the number of
 * records that were pending (which may exceed cap). */
int slay_trace_read(const char** names, float* ms, int cap);

/* Static description of a status code. */
const char* slay_status_string(slay_status st);

/* Text of the last CUDA error seen by this thread inside the library ("" if none). */
const char* slay_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* SLAY_H */
