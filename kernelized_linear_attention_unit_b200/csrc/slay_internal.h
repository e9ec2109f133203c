// slay_internal.h -- declarations shared by the files of libslay.so (not installed).
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

#include "slay.h"

namespace slay {

constexpr int kMaxR = 16;
constexpr int kMaxF = 1024;
constexpr int kD = 64;  // head dimension this build supports (D == Dv == 64)

// Device view of one sketch-parameter key.  The node constants travel by value.
struct Params {
    const float* omT;    // [D][F]   omega transposed (feature index fastest)
    const float* anT;    // [D][F]   anchors transposed
    const float* om;     // [F][D]   omega, row per feature
    const float* an;     // [F][D]   anchors, row per feature
    const uint16_t* wB;  // [F/32][64][D] bf16: per 32 features, 32 omega rows then 32
                         // anchor rows (tensor-core projection operand), may be null
    int D, R, m, F;
    // phi_f = exp2(a2[r] * u + b2[r]) * p^2 with u = omega_f . x^, p = a_f . x^, where
    // a2 = sqrt(2 s_r) log2(e), b2 = log2(sqrt(wt_r/m)) - s_r log2(e).
    float a2[kMaxR];
    float b2[kMaxR];
    // For the backward: sq = sqrt(2 s_r), c = sqrt(wt_r/m).
    float sq[kMaxR];
    float c[kMaxR];
};

// Device view of a sketch variant's parameters (slay_phi_kind): omega^T, anchors^T and, for
// the signed kind, the second anchors^T, each [H][D][F] (H heads for the per-head kind, else
// 1); phi_f = exp2(a2[r] u + b2[r]) times the anchor factor of the kind.
struct VarParams {
    const float* omT;
    const float* anT;
    const float* anbT;
    int F, m, R, H, kind;
    float a2[kMaxR];
    float b2[kMaxR];
};

// ---- per-launch timing (slay_trace.cpp) ----
// Brackets the kernel launched inside its scope with CUDA events while tracing is on.
class TraceScope {
public:
    TraceScope(const char* name, cudaStream_t st);
    ~TraceScope();
    TraceScope(const TraceScope&) = delete;
    TraceScope& operator=(const TraceScope&) = delete;

private:
    cudaStream_t st_;
    int idx_;
};

// ---- host math (slay_params.cpp): no CUDA calls ----
void philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]);
// Nodes/weights of the R-point Gauss-Laguerre rule; false on failure.
bool gauss_laguerre(int R, double* t, double* w);
// omega, anchors: [F*D] float, s, wt: [R] double.  false on failure.
bool draw_sketch(int D, int R, int m, uint64_t seed, double eps, float* omega,
                 float* anchors, double* s, double* wt);
// A sketch variant (kind 0-4, see slay_phi_kind) for one head; anchors_b only for kind 2.
bool draw_sketch_kind(int D, int R, int m, uint64_t seed, double eps, int kind, int head,
                      float* omega, float* anchors, float* anchors_b, double* s, double* wt);

// ---- argument checks and workspace sizing shared by the entry points (slay_api.cu) ----
bool eps_ok(float eps);
bool dtype_ok(slay_dtype d);
slay_status check_shape(int D, int Dv, int R, int m);
slay_status check_attn(const void* q, const void* k, const void* v, const void* out, int B,
                       int H, int L, int D, int Dv, slay_dtype dt, int R, int m, float eps);
// Every attention workspace starts with a 256-byte header whose first int is the
// kernel status word: 0 after a call is enqueued, set to 1 by a kernel whose bounded
// mbarrier wait ran out.  The path's own scratch follows the header.
constexpr size_t kWsHeader = 256;
size_t attn_ws(slay_op op, slay_dtype dt, int B, int H, int L, int Dv, int R, int m);
// Device address of the no-alloc path's status word on the current device, or nullptr
// when that path has not run on it.
const void* noalloc_status_word();

// ---- CUDA-core kernels (slay_simt.cu) ----
// Sizes of the workspace carve-outs of the CUDA-core path.
size_t simt_ws_causal(int B, int H, int L, int Dv, int F);
size_t simt_ws_bidir(int B, int H, int L, int Dv, int F);
size_t simt_ws_bwd(int B, int H, int L, int Dv, int F);
size_t simt_ws_bidir_bwd(int B, int H, int L, int Dv, int F);

cudaError_t simt_feature_map(const void* x, void* phi, int64_t n, slay_dtype in_dt,
                             slay_dtype out_dt, const Params& P, cudaStream_t st);
struct StateIO;
cudaError_t simt_attn_fwd(const void* q, const void* k, const void* v, void* out, float* den,
                          int B, int H, int L, slay_dtype dt, const Params& P, float eps,
                          bool causal, void* ws, cudaStream_t st, const StateIO* sio = nullptr);
size_t simt_ws_state(int B, int H, int L, int F);
cudaError_t simt_causal_state(const void* k, const void* v, int B, int H, int L, slay_dtype dt,
                              const Params& P, void* ws, cudaStream_t st, const StateIO& sio);
cudaError_t simt_state_prefix(const float* s_all, const float* z_all, int r0, int r1,
                              int64_t ns, int64_t nz, float* s_in, float* z_in, cudaStream_t st);
// The sums outside a piece of a causal sequence for its backward: s_in, z_in over the tokens
// before it (phi(k) [v, 1]), g_in, zg_in over the tokens after it (phi(q) [dn, delta]);
// [B,H,F,64] and [B,H,F] fp32, null = zero.
struct BwdStateIO {
    const float* s_in;
    const float* z_in;
    const float* g_in;
    const float* zg_in;
    // phi(q) and the row statistics of these q, out, den, dout are already in the workspace
    // (simt_causal_bwd_state on the same workspace left them there): not recomputed
    bool q_ready = false;
};
cudaError_t simt_attn_causal_bwd_state(const void* q, const void* k, const void* v,
                                       const void* out, const float* den, const void* dout,
                                       float* dq, float* dk, float* dv, int B, int H, int L,
                                       slay_dtype dt, const Params& P, float eps, void* ws,
                                       const BwdStateIO& sio, cudaStream_t st);
cudaError_t simt_causal_bwd_state(const void* q, const void* out, const float* den,
                                  const void* dout, float* g_out, float* zg_out, int B, int H,
                                  int L, slay_dtype dt, const Params& P, float eps, void* ws,
                                  cudaStream_t st);
cudaError_t simt_attn_causal_bwd(const void* q, const void* k, const void* v,
                                 const void* out, const float* den, const void* dout,
                                 float* dq, float* dk, float* dv, int B, int H, int L,
                                 slay_dtype dt, const Params& P, float eps, void* ws,
                                 cudaStream_t st);
cudaError_t simt_attn_bidir_bwd(const void* q, const void* k, const void* v,
                                const void* out, const float* den, const void* dout,
                                float* dq, float* dk, float* dv, int B, int H, int L,
                                slay_dtype dt, const Params& P, float eps, void* ws,
                                cudaStream_t st);
cudaError_t simt_feature_map_bwd(const void* x, const void* dphi, float* dx, int64_t n,
                                 slay_dtype x_dt, slay_dtype dphi_dt, const Params& P,
                                 cudaStream_t st);
cudaError_t simt_feature_map_kind(const void* x, void* phi, int64_t n, int64_t Lh,
                                  slay_dtype in_dt, slay_dtype out_dt, const VarParams& P,
                                  cudaStream_t st);
size_t simt_ws_linear(int B, int H, int L, int F);
cudaError_t simt_linear_attn(const void* phq, const void* phk, const void* v, void* out,
                             float* den, int B, int H, int L, int F, slay_dtype dt, float eps,
                             bool causal, void* ws, cudaStream_t st);
cudaError_t simt_decode_step(const void* q, const void* k, const void* v, float* S, float* z,
                             void* out, int N, slay_dtype dt, const Params& P, float eps,
                             cudaStream_t st);

}  // namespace slay
