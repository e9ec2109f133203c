// slay_api.cu -- C ABI entry points of libslay.so: argument checks, the per-key
// sketch-parameter cache and dispatch to the kernels.  See include/slay.h for the
// contract of each entry point.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <tuple>
#include <vector>

#include "slay.h"
#include "slay_internal.h"
#include "slay_tc.h"

namespace slay {
namespace {

thread_local std::string g_last_error;

slay_status cuda_fail(cudaError_t e)
{
    g_last_error = cudaGetErrorString(e);
    return SLAY_ERR_CUDA;
}

void set_last_error(const char* msg) { g_last_error = msg; }

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

using Key = std::tuple<int, int, int, int, uint64_t, uint32_t>;  // device, D, R, m, seed, eps bits

struct Entry {
    void* dev = nullptr;
    Params P{};
};

std::mutex g_mu;
std::map<Key, Entry>& cache()
{
    static std::map<Key, Entry>* c = new std::map<Key, Entry>();  // held until exit
    return *c;
}

uint32_t float_bits(float x)
{
    uint32_t b;
    std::memcpy(&b, &x, sizeof b);
    return b;
}

uint16_t to_bf16_bits(float x)
{
    uint32_t b = float_bits(x);
    b += 0x7FFFu + ((b >> 16) & 1u);
    return static_cast<uint16_t>(b >> 16);
}

// Build (or find) the device copy of the key's parameters on the current device.
slay_status get_params(int D, int R, int m, uint64_t seed, float eps, Params* out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    const Key key{dev, D, R, m, seed, float_bits(eps)};
    std::lock_guard<std::mutex> lock(g_mu);
    auto it = cache().find(key);
    if (it != cache().end()) { *out = it->second.P; return SLAY_OK; }

    const int F = R * m;
    std::vector<float> om(static_cast<size_t>(F) * D), an(static_cast<size_t>(F) * D);
    double s[kMaxR], wt[kMaxR];
    if (!draw_sketch(D, R, m, seed, static_cast<double>(eps), om.data(), an.data(), s, wt))
        return SLAY_ERR_INVALID_ARG;
    const size_t nF = static_cast<size_t>(F) * D;
    // layout: omT | anT | om | an (fp32), then wB (bf16 tensor-core operand)
    const size_t wb_elems = tc_wb_elems(D, R, m);
    const size_t bytes = 4 * nF * sizeof(float) + wb_elems * sizeof(uint16_t);
    std::vector<unsigned char> host(bytes);
    float* h = reinterpret_cast<float*>(host.data());
    for (int f = 0; f < F; ++f)
        for (int d = 0; d < D; ++d) {
            h[static_cast<size_t>(d) * F + f] = om[static_cast<size_t>(f) * D + d];
            h[nF + static_cast<size_t>(d) * F + f] = an[static_cast<size_t>(f) * D + d];
        }
    std::memcpy(h + 2 * nF, om.data(), nF * sizeof(float));
    std::memcpy(h + 3 * nF, an.data(), nF * sizeof(float));
    uint16_t* wb = reinterpret_cast<uint16_t*>(h + 4 * nF);
    if (wb_elems) {
        std::vector<uint16_t> omb(nF), anb(nF);
        for (size_t i = 0; i < nF; ++i) { omb[i] = to_bf16_bits(om[i]); anb[i] = to_bf16_bits(an[i]); }
        tc_pack_wb(D, R, m, omb.data(), anb.data(), wb);
    }

    Entry ent;
    e = cudaMalloc(&ent.dev, bytes);
    if (e != cudaSuccess) return cuda_fail(e);
    e = cudaMemcpy(ent.dev, host.data(), bytes, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) { cudaFree(ent.dev); return cuda_fail(e); }
    float* d = static_cast<float*>(ent.dev);
    Params& P = ent.P;
    P.omT = d;
    P.anT = d + nF;
    P.om = d + 2 * nF;
    P.an = d + 3 * nF;
    P.wB = wb_elems ? reinterpret_cast<const uint16_t*>(d + 4 * nF) : nullptr;
    P.D = D; P.R = R; P.m = m; P.F = F;
    const double log2e = 1.4426950408889634073599246810019;
    for (int r = 0; r < kMaxR; ++r) {
        if (r < R) {
            const double c = std::sqrt(wt[r] / m);
            const double sq = std::sqrt(2.0 * s[r]);
            P.a2[r] = static_cast<float>(sq * log2e);
            P.b2[r] = static_cast<float>(std::log2(c) - s[r] * log2e);
            P.sq[r] = static_cast<float>(sq);
            P.c[r] = static_cast<float>(c);
        } else {
            P.a2[r] = P.b2[r] = P.sq[r] = P.c[r] = 0.0f;
        }
    }
    cache()[key] = ent;
    *out = P;
    return SLAY_OK;
}

// ---- sketch variants: one cache entry per (device, D, R, m, seed, eps, kind, heads)
using VKey = std::tuple<int, int, int, int, uint64_t, uint32_t, int, int>;

struct VEntry {
    void* dev = nullptr;
    VarParams P{};
};

std::map<VKey, VEntry>& vcache()
{
    static std::map<VKey, VEntry>* c = new std::map<VKey, VEntry>();  // held until exit
    return *c;
}

slay_status get_var_params(int D, int R, int m, uint64_t seed, float eps, int kind, int H,
                           VarParams* out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    const VKey key{dev, D, R, m, seed, float_bits(eps), kind, H};
    std::lock_guard<std::mutex> lock(g_mu);
    auto it = vcache().find(key);
    if (it != vcache().end()) { *out = it->second.P; return SLAY_OK; }
    const int F = R * m;
    const size_t nF = static_cast<size_t>(F) * D;
    std::vector<float> om(nF), an(nF), anb(nF);
    // [3][H][D][F]: omega^T, anchors^T, second anchors^T
    std::vector<float> host(3 * static_cast<size_t>(H) * nF, 0.0f);
    double sr[kMaxR], wt[kMaxR];
    for (int h = 0; h < H; ++h) {
        if (!draw_sketch_kind(D, R, m, seed, static_cast<double>(eps), kind, h, om.data(),
                              an.data(), anb.data(), sr, wt))
            return SLAY_ERR_INVALID_ARG;
        for (int f = 0; f < F; ++f)
            for (int d = 0; d < D; ++d) {
                const size_t src = static_cast<size_t>(f) * D + d;
                const size_t dst = static_cast<size_t>(h) * nF + static_cast<size_t>(d) * F + f;
                host[dst] = om[src];
                host[static_cast<size_t>(H) * nF + dst] = an[src];
                host[2 * static_cast<size_t>(H) * nF + dst] = kind == 2 ? anb[src] : 0.0f;
            }
    }
    VEntry ent;
    const size_t bytes = host.size() * sizeof(float);
    e = cudaMalloc(&ent.dev, bytes);
    if (e != cudaSuccess) return cuda_fail(e);
    e = cudaMemcpy(ent.dev, host.data(), bytes, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) { cudaFree(ent.dev); return cuda_fail(e); }
    float* d = static_cast<float*>(ent.dev);
    VarParams& P = ent.P;
    P.omT = d;
    P.anT = d + static_cast<size_t>(H) * nF;
    P.anbT = d + 2 * static_cast<size_t>(H) * nF;
    P.F = F; P.m = m; P.R = R; P.H = H; P.kind = kind;
    const double log2e = 1.4426950408889634073599246810019;
    for (int r = 0; r < kMaxR; ++r) {
        if (r >= R) { P.a2[r] = P.b2[r] = 0.0f; continue; }
        if (kind == 4) {   // FAVOR+: exp(u - 1/2) / sqrt(F) = exp2(log2e u - (log2e + log2 F) / 2)
            P.a2[r] = static_cast<float>(log2e);
            P.b2[r] = static_cast<float>(-0.5 * (log2e + std::log2(static_cast<double>(F))));
        } else {
            P.a2[r] = static_cast<float>(std::sqrt(2.0 * sr[r]) * log2e);
            P.b2[r] = static_cast<float>(std::log2(std::sqrt(wt[r] / m)) - sr[r] * log2e);
        }
    }
    vcache()[key] = ent;
    *out = P;
    return SLAY_OK;
}

}  // namespace

bool eps_ok(float eps) { return std::isfinite(eps) && eps > 0.0f; }
bool dtype_ok(slay_dtype d) { return d == SLAY_F32 || d == SLAY_BF16; }

slay_status check_shape(int D, int Dv, int R, int m)
{
    if (D <= 0 || Dv <= 0 || R <= 0 || m <= 0) return SLAY_ERR_INVALID_ARG;
    if (D != kD || Dv != kD) return SLAY_ERR_UNSUPPORTED;
    if (R > kMaxR || static_cast<int64_t>(R) * m > kMaxF) return SLAY_ERR_UNSUPPORTED;
    return SLAY_OK;
}

slay_status check_attn(const void* q, const void* k, const void* v, const void* out, int B,
                       int H, int L, int D, int Dv, slay_dtype dt, int R, int m, float eps)
{
    if (B < 0 || H < 0 || L < 0) return SLAY_ERR_INVALID_ARG;
    slay_status s = check_shape(D, Dv, R, m);
    if (s != SLAY_OK) return s;
    if (!dtype_ok(dt) || !eps_ok(eps)) return SLAY_ERR_INVALID_ARG;
    if (static_cast<int64_t>(B) * H * L == 0) return SLAY_OK;
    if (!q || !k || !v || !out) return SLAY_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16))
        return SLAY_ERR_INVALID_ARG;
    // grid limits of the launches: (b,h) and 64-token chunks index grid y/z dimensions
    if (static_cast<int64_t>(B) * H > 65535 || (static_cast<int64_t>(L) + 63) / 64 > 65535)
        return SLAY_ERR_UNSUPPORTED;
    return SLAY_OK;
}

size_t attn_ws(slay_op op, slay_dtype dt, int B, int H, int L, int Dv, int R, int m)
{
    const int F = R * m;
    if (op == SLAY_OP_CAUSAL_STATE) {
        if (dt == SLAY_BF16 && tc_supported(SLAY_OP_CAUSAL_FWD, B, H, L, R, m))
            return tc_state_workspace_bytes(B, H, L, R, m);
    } else if (op == SLAY_OP_CAUSAL_FWD_SPLIT) {
        if (dt == SLAY_BF16 && tc_supported(SLAY_OP_CAUSAL_FWD, B, H, L, R, m))
            return tc_workspace_bytes(op, B, H, L, R, m);
        // CUDA cores: the piece-state call and the forward, one after the other
        return kWsHeader + std::max(simt_ws_causal(B, H, L, Dv, F), simt_ws_state(B, H, L, F));
    } else if (dt == SLAY_BF16 && tc_supported(op, B, H, L, R, m)) {
        return tc_workspace_bytes(op, B, H, L, R, m);
    }
    switch (op) {
        case SLAY_OP_CAUSAL_FWD: return kWsHeader + simt_ws_causal(B, H, L, Dv, F);
        case SLAY_OP_BIDIR_FWD: return kWsHeader + simt_ws_bidir(B, H, L, Dv, F);
        case SLAY_OP_CAUSAL_BWD: return kWsHeader + simt_ws_bwd(B, H, L, Dv, F);
        case SLAY_OP_BIDIR_BWD: return kWsHeader + simt_ws_bidir_bwd(B, H, L, Dv, F);
        case SLAY_OP_LINEAR_ATTN: return kWsHeader + simt_ws_linear(B, H, L, F);
        case SLAY_OP_CAUSAL_STATE: return kWsHeader + simt_ws_state(B, H, L, F);
        default: return 0;
    }
}

namespace {

slay_status attn_fwd(const void* q, const void* k, const void* v, void* out, float* den, int B,
                     int H, int L, int D, int Dv, slay_dtype dt, int R, int m, uint64_t seed,
                     float eps, void* ws, size_t ws_bytes, void* stream, bool causal)
{
    slay_status s = check_attn(q, k, v, out, B, H, L, D, Dv, dt, R, m, eps);
    if (s != SLAY_OK) return s;
    if (static_cast<int64_t>(B) * H * L == 0) return SLAY_OK;
    if (den && !aligned(den, 4)) return SLAY_ERR_INVALID_ARG;
    const slay_op op = causal ? SLAY_OP_CAUSAL_FWD : SLAY_OP_BIDIR_FWD;
    const size_t need = attn_ws(op, dt, B, H, L, Dv, R, m);
    if (need > 0 && (!ws || ws_bytes < need || !aligned(ws, 256))) return SLAY_ERR_INVALID_ARG;
    Params P;
    if ((s = get_params(D, R, m, seed, eps, &P)) != SLAY_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (dt == SLAY_BF16 && tc_supported(op, B, H, L, R, m)) {
        e = tc_attn_fwd(q, k, v, out, den, B, H, L, P, eps, causal, ws, st);
    } else {
        e = cudaMemsetAsync(ws, 0, sizeof(int), st);
        if (e == cudaSuccess)
            e = simt_attn_fwd(q, k, v, out, den, B, H, L, dt, P, eps, causal,
                              static_cast<char*>(ws) + kWsHeader, st);
    }
    return e == cudaSuccess ? SLAY_OK : cuda_fail(e);
}

}  // namespace
}  // namespace slay

using namespace slay;

extern "C" {

slay_status slay_feature_map(const void* x, void* phi, int64_t n_rows, int D, slay_dtype in_dt,
                             slay_dtype out_dt, int R, int m, uint64_t seed, float eps,
                             void* stream)
{
    if (n_rows < 0) return SLAY_ERR_INVALID_ARG;
    slay_status s = check_shape(D, kD, R, m);
    if (s != SLAY_OK) return s;
    if (!dtype_ok(in_dt) || !dtype_ok(out_dt) || !eps_ok(eps)) return SLAY_ERR_INVALID_ARG;
    if (in_dt == SLAY_F32 && out_dt == SLAY_BF16) return SLAY_ERR_UNSUPPORTED;
    if (n_rows == 0) return SLAY_OK;
    if (!x || !phi || !aligned(x, 16) || !aligned(phi, 16)) return SLAY_ERR_INVALID_ARG;
    if (n_rows > (int64_t(1) << 36)) return SLAY_ERR_UNSUPPORTED;
    Params P;
    if ((s = get_params(D, R, m, seed, eps, &P)) != SLAY_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (in_dt == SLAY_BF16 && out_dt == SLAY_BF16 && P.wB && tc_fmap_supported(D, R, m, n_rows))
        e = tc_feature_map(x, phi, n_rows, P, st);
    else
        e = simt_feature_map(x, phi, n_rows, in_dt, out_dt, P, st);
    return e == cudaSuccess ? SLAY_OK : cuda_fail(e);
}

slay_status slay_attn_causal_fwd(const void* q, const void* k, const void* v, void* out,
                                 float* den, int B, int H, int L, int D, int Dv, slay_dtype dt,
                                 int R, int m, uint64_t seed, float eps, void* workspace,
                                 size_t ws_bytes, void* stream)
{
    return attn_fwd(q, k, v, out, den, B, H, L, D, Dv, dt, R, m, seed, eps, workspace, ws_bytes,
                    stream, true);
}

slay_status slay_attn_bidir_fwd(const void* q, const void* k, const void* v, void* out,
                                float* den, int B, int H, int L, int D, int Dv, slay_dtype dt,
                                int R, int m, uint64_t seed, float eps, void* workspace,
                                size_t ws_bytes, void* stream)
{
    return attn_fwd(q, k, v, out, den, B, H, L, D, Dv, dt, R, m, seed, eps, workspace, ws_bytes,
                    stream, false);
}

}  // extern "C"

namespace slay {
namespace {

slay_status attn_bwd(const void* q, const void* k, const void* v, const void* out,
                     const float* den, const void* dout, float* dq, float* dk, float* dv, int B,
                     int H, int L, int D, int Dv, slay_dtype dt, int R, int m, uint64_t seed,
                     float eps, void* workspace, size_t ws_bytes, void* stream, bool causal,
                     const BwdStateIO* sio = nullptr)
{
    slay_status s = check_attn(q, k, v, out, B, H, L, D, Dv, dt, R, m, eps);
    if (s != SLAY_OK) return s;
    if (static_cast<int64_t>(B) * H * L == 0) return SLAY_OK;
    if (!den || !dout || !dq || !dk || !dv) return SLAY_ERR_INVALID_ARG;
    if (!aligned(den, 4) || !aligned(dout, 16) || !aligned(dq, 16) || !aligned(dk, 16) ||
        !aligned(dv, 16))
        return SLAY_ERR_INVALID_ARG;
    const size_t need = attn_ws(causal ? SLAY_OP_CAUSAL_BWD : SLAY_OP_BIDIR_BWD, dt, B, H, L, Dv,
                                R, m);
    if (need > 0 && (!workspace || ws_bytes < need || !aligned(workspace, 256)))
        return SLAY_ERR_INVALID_ARG;
    Params P;
    if ((s = get_params(D, R, m, seed, eps, &P)) != SLAY_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // the second call of the two-call backward keeps the status word the first one cleared
    cudaError_t e = (sio && sio->q_ready) ? cudaSuccess : cudaMemsetAsync(workspace, 0, sizeof(int), st);
    char* w = static_cast<char*>(workspace) + kWsHeader;
    if (e == cudaSuccess)
        e = sio ? simt_attn_causal_bwd_state(q, k, v, out, den, dout, dq, dk, dv, B, H, L, dt, P,
                                             eps, w, *sio, st)
            : causal ? simt_attn_causal_bwd(q, k, v, out, den, dout, dq, dk, dv, B, H, L, dt, P, eps,
                                            w, st)
                     : simt_attn_bidir_bwd(q, k, v, out, den, dout, dq, dk, dv, B, H, L, dt, P, eps,
                                           w, st);
    return e == cudaSuccess ? SLAY_OK : cuda_fail(e);
}

}  // namespace
}  // namespace slay

extern "C" {

slay_status slay_attn_causal_bwd(const void* q, const void* k, const void* v, const void* out,
                                 const float* den, const void* dout, float* dq, float* dk,
                                 float* dv, int B, int H, int L, int D, int Dv, slay_dtype dt,
                                 int R, int m, uint64_t seed, float eps, void* workspace,
                                 size_t ws_bytes, void* stream)
{
    return attn_bwd(q, k, v, out, den, dout, dq, dk, dv, B, H, L, D, Dv, dt, R, m, seed, eps,
                    workspace, ws_bytes, stream, true);
}

slay_status slay_attn_bidir_bwd(const void* q, const void* k, const void* v, const void* out,
                                const float* den, const void* dout, float* dq, float* dk,
                                float* dv, int B, int H, int L, int D, int Dv, slay_dtype dt,
                                int R, int m, uint64_t seed, float eps, void* workspace,
                                size_t ws_bytes, void* stream)
{
    return attn_bwd(q, k, v, out, den, dout, dq, dk, dv, B, H, L, D, Dv, dt, R, m, seed, eps,
                    workspace, ws_bytes, stream, false);
}

slay_status slay_feature_map_ex(const void* x, void* phi, int64_t n_rows, int D,
                               slay_dtype in_dt, slay_dtype out_dt, int R, int m, uint64_t seed,
                               float eps, int kind, int heads, int64_t rows_per_head,
                               void* stream)
{
    if (kind < SLAY_PHI_ANCHOR || kind > SLAY_PHI_PERFORMER) return SLAY_ERR_INVALID_ARG;
    if (kind == SLAY_PHI_ANCHOR)
        return slay_feature_map(x, phi, n_rows, D, in_dt, out_dt, R, m, seed, eps, stream);
    if (n_rows < 0) return SLAY_ERR_INVALID_ARG;
    slay_status s = check_shape(D, kD, R, m);
    if (s != SLAY_OK) return s;
    if (!dtype_ok(in_dt) || !dtype_ok(out_dt) || !eps_ok(eps)) return SLAY_ERR_INVALID_ARG;
    if (in_dt == SLAY_F32 && out_dt == SLAY_BF16) return SLAY_ERR_UNSUPPORTED;
    int H = 1;
    int64_t Lh = n_rows;
    if (kind == SLAY_PHI_PER_HEAD) {
        if (heads <= 0 || heads > 1024 || rows_per_head <= 0) return SLAY_ERR_INVALID_ARG;
        if (n_rows % rows_per_head != 0) return SLAY_ERR_INVALID_ARG;
        H = heads;
        Lh = rows_per_head;
    }
    if (n_rows == 0) return SLAY_OK;
    if (!x || !phi || !aligned(x, 16) || !aligned(phi, 16)) return SLAY_ERR_INVALID_ARG;
    if ((Lh + 63) / 64 > (int64_t(1) << 31) - 1 || n_rows / Lh > 65535) return SLAY_ERR_UNSUPPORTED;
    VarParams P;
    if ((s = get_var_params(D, R, m, seed, eps, kind, H, &P)) != SLAY_OK) return s;
    cudaError_t e = simt_feature_map_kind(x, phi, n_rows, Lh, in_dt, out_dt, P,
                                          static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SLAY_OK : cuda_fail(e);
}

slay_status slay_sketch_params_ex(int D, int R, int m, uint64_t seed, float eps, int kind,
                                  int head, float* omega_host, float* anchors_host,
                                  float* anchors_b_host, double* s_host, double* w_host)
{
    if (D <= 0 || D > 4096 || R <= 0 || R > kMaxR || m <= 0 || !eps_ok(eps) || head < 0)
        return SLAY_ERR_INVALID_ARG;
    if (kind < SLAY_PHI_ANCHOR || kind > SLAY_PHI_PERFORMER) return SLAY_ERR_INVALID_ARG;
    if (static_cast<int64_t>(R) * m * D > (int64_t(1) << 31)) return SLAY_ERR_UNSUPPORTED;
    if (!draw_sketch_kind(D, R, m, seed, static_cast<double>(eps), kind, head, omega_host,
                          anchors_host, anchors_b_host, s_host, w_host))
        return SLAY_ERR_INVALID_ARG;
    return SLAY_OK;
}

slay_status slay_linear_attn_fwd(const void* phq, const void* phk, const void* v, void* out,
                                 float* den, int B, int H, int L, int F, int Dv, slay_dtype dt,
                                 float eps, int causal, void* workspace, size_t ws_bytes,
                                 void* stream)
{
    if (B < 0 || H < 0 || L < 0 || F <= 0 || Dv <= 0) return SLAY_ERR_INVALID_ARG;
    if (Dv != kD) return SLAY_ERR_UNSUPPORTED;
    if (F > kMaxF) return SLAY_ERR_UNSUPPORTED;
    if (!dtype_ok(dt) || !eps_ok(eps)) return SLAY_ERR_INVALID_ARG;
    if (static_cast<int64_t>(B) * H * L == 0) return SLAY_OK;
    if (!phq || !phk || !v || !out) return SLAY_ERR_INVALID_ARG;
    if (!aligned(phq, 16) || !aligned(phk, 16) || !aligned(v, 16) || !aligned(out, 16) ||
        (den && !aligned(den, 4)))
        return SLAY_ERR_INVALID_ARG;
    if (static_cast<int64_t>(B) * H > 65535 || (static_cast<int64_t>(L) + 63) / 64 > 65535)
        return SLAY_ERR_UNSUPPORTED;
    const size_t need = kWsHeader + simt_ws_linear(B, H, L, F);
    if (!workspace || ws_bytes < need || !aligned(workspace, 256)) return SLAY_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(workspace, 0, sizeof(int), st);
    if (e == cudaSuccess)
        e = simt_linear_attn(phq, phk, v, out, den, B, H, L, F, dt, eps, causal != 0,
                             static_cast<char*>(workspace) + kWsHeader, st);
    return e == cudaSuccess ? SLAY_OK : cuda_fail(e);
}

namespace slay {
namespace {

// the state arguments of the state-continuation entry points: both of a pair or neither
slay_status check_state_ptrs(const float* s, const float* z)
{
    if ((s == nullptr) != (z == nullptr)) return SLAY_ERR_INVALID_ARG;
    if (s && (!aligned(s, 16) || !aligned(z, 16))) return SLAY_ERR_INVALID_ARG;
    return SLAY_OK;
}

}  // namespace
}  // namespace slay

slay_status slay_attn_causal_fwd_state(const void* q, const void* k, const void* v, void* out,
                                       float* den, const float* S_in, const float* z_in,
                                       float* S_out, float* z_out, int B, int H, int L, int D,
                                       int Dv, slay_dtype dt, int R, int m, uint64_t seed,
                                       float eps, void* workspace, size_t ws_bytes, void* stream)
{
    slay_status s = check_attn(q, k, v, out, B, H, L, D, Dv, dt, R, m, eps);
    if (s != SLAY_OK) return s;
    if ((s = check_state_ptrs(S_in, z_in)) != SLAY_OK) return s;
    if ((s = check_state_ptrs(S_out, z_out)) != SLAY_OK) return s;
    if (static_cast<int64_t>(B) * H * L == 0) return SLAY_OK;
    if (den && !aligned(den, 4)) return SLAY_ERR_INVALID_ARG;
    const size_t need = attn_ws(SLAY_OP_CAUSAL_FWD, dt, B, H, L, Dv, R, m);
    if (need > 0 && (!workspace || ws_bytes < need || !aligned(workspace, 256)))
        return SLAY_ERR_INVALID_ARG;
    Params P;
    if ((s = get_params(D, R, m, seed, eps, &P)) != SLAY_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const StateIO sio{S_in, z_in, S_out, z_out};
    cudaError_t e;
    if (dt == SLAY_BF16 && tc_supported(SLAY_OP_CAUSAL_FWD, B, H, L, R, m)) {
        e = tc_attn_fwd(q, k, v, out, den, B, H, L, P, eps, true, workspace, st, false, &sio);
    } else {
        e = cudaMemsetAsync(workspace, 0, sizeof(int), st);
        if (e == cudaSuccess)
            e = simt_attn_fwd(q, k, v, out, den, B, H, L, dt, P, eps, true,
                              static_cast<char*>(workspace) + kWsHeader, st, &sio);
    }
    return e == cudaSuccess ? SLAY_OK : cuda_fail(e);
}

slay_status slay_causal_state(const void* k, const void* v, const float* S_in, const float* z_in,
                              float* S_out, float* z_out, int B, int H, int L, int D, int Dv,
                              slay_dtype dt, int R, int m, uint64_t seed, float eps,
                              void* workspace, size_t ws_bytes, void* stream)
{
    slay_status s = check_attn(k, k, v, v, B, H, L, D, Dv, dt, R, m, eps);
    if (s != SLAY_OK) return s;
    if ((s = check_state_ptrs(S_in, z_in)) != SLAY_OK) return s;
    if (!S_out || !z_out) return SLAY_ERR_INVALID_ARG;
    if ((s = check_state_ptrs(S_out, z_out)) != SLAY_OK) return s;
    if (static_cast<int64_t>(B) * H == 0) return SLAY_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (L == 0) {   // an empty chunk: the state passes through unchanged
        const size_t bs = static_cast<size_t>(B) * H * R * m * Dv * sizeof(float);
        const size_t bz = static_cast<size_t>(B) * H * R * m * sizeof(float);
        cudaError_t e = S_in ? cudaMemcpyAsync(S_out, S_in, bs, cudaMemcpyDeviceToDevice, st)
                             : cudaMemsetAsync(S_out, 0, bs, st);
        if (e == cudaSuccess)
            e = S_in ? cudaMemcpyAsync(z_out, z_in, bz, cudaMemcpyDeviceToDevice, st)
                     : cudaMemsetAsync(z_out, 0, bz, st);
        return e == cudaSuccess ? SLAY_OK : cuda_fail(e);
    }
    const size_t need = attn_ws(SLAY_OP_CAUSAL_STATE, dt, B, H, L, Dv, R, m);
    if (!workspace || ws_bytes < need || !aligned(workspace, 256)) return SLAY_ERR_INVALID_ARG;
    Params P;
    if ((s = get_params(D, R, m, seed, eps, &P)) != SLAY_OK) return s;
    const StateIO sio{S_in, z_in, S_out, z_out};
    cudaError_t e;
    if (dt == SLAY_BF16 && tc_supported(SLAY_OP_CAUSAL_FWD, B, H, L, R, m)) {
        e = tc_causal_state(k, v, B, H, L, P, workspace, st, sio);
    } else {
        e = cudaMemsetAsync(workspace, 0, sizeof(int), st);
        if (e == cudaSuccess)
            e = simt_causal_state(k, v, B, H, L, dt, P, static_cast<char*>(workspace) + kWsHeader,
                                  st, sio);
    }
    return e == cudaSuccess ? SLAY_OK : cuda_fail(e);
}

slay_status slay_attn_causal_fwd_begin(const void* k, const void* v, float* S_out, float* z_out,
                                       int B, int H, int L, int D, int Dv, slay_dtype dt, int R,
                                       int m, uint64_t seed, float eps, void* workspace,
                                       size_t ws_bytes, void* stream)
{
    slay_status s = check_attn(k, k, v, v, B, H, L, D, Dv, dt, R, m, eps);
    if (s != SLAY_OK) return s;
    if (!S_out || !z_out) return SLAY_ERR_INVALID_ARG;
    if ((s = check_state_ptrs(S_out, z_out)) != SLAY_OK) return s;
    if (static_cast<int64_t>(B) * H == 0) return SLAY_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (L == 0) {   // an empty piece adds nothing to the state
        const size_t bs = static_cast<size_t>(B) * H * R * m * Dv * sizeof(float);
        const size_t bz = static_cast<size_t>(B) * H * R * m * sizeof(float);
        cudaError_t e = cudaMemsetAsync(S_out, 0, bs, st);
        if (e == cudaSuccess) e = cudaMemsetAsync(z_out, 0, bz, st);
        return e == cudaSuccess ? SLAY_OK : cuda_fail(e);
    }
    const size_t need = attn_ws(SLAY_OP_CAUSAL_FWD_SPLIT, dt, B, H, L, Dv, R, m);
    if (!workspace || ws_bytes < need || !aligned(workspace, 256)) return SLAY_ERR_INVALID_ARG;
    Params P;
    if ((s = get_params(D, R, m, seed, eps, &P)) != SLAY_OK) return s;
    cudaError_t e;
    if (dt == SLAY_BF16 && tc_supported(SLAY_OP_CAUSAL_FWD, B, H, L, R, m)) {
        e = tc_attn_fwd_begin(k, v, B, H, L, P, eps, workspace, st, S_out, z_out);
    } else {
        const StateIO sio{nullptr, nullptr, S_out, z_out};
        e = cudaMemsetAsync(workspace, 0, sizeof(int), st);
        if (e == cudaSuccess)
            e = simt_causal_state(k, v, B, H, L, dt, P, static_cast<char*>(workspace) + kWsHeader,
                                  st, sio);
    }
    return e == cudaSuccess ? SLAY_OK : cuda_fail(e);
}

slay_status slay_attn_causal_fwd_finish(const void* q, const void* k, const void* v, void* out,
                                        float* den, const float* S_in, const float* z_in, int B,
                                        int H, int L, int D, int Dv, slay_dtype dt, int R, int m,
                                        uint64_t seed, float eps, void* workspace,
                                        size_t ws_bytes, void* stream)
{
    slay_status s = check_attn(q, k, v, out, B, H, L, D, Dv, dt, R, m, eps);
    if (s != SLAY_OK) return s;
    if ((s = check_state_ptrs(S_in, z_in)) != SLAY_OK) return s;
    if (static_cast<int64_t>(B) * H * L == 0) return SLAY_OK;
    if (den && !aligned(den, 4)) return SLAY_ERR_INVALID_ARG;
    const size_t need = attn_ws(SLAY_OP_CAUSAL_FWD_SPLIT, dt, B, H, L, Dv, R, m);
    if (!workspace || ws_bytes < need || !aligned(workspace, 256)) return SLAY_ERR_INVALID_ARG;
    Params P;
    if ((s = get_params(D, R, m, seed, eps, &P)) != SLAY_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (dt == SLAY_BF16 && tc_supported(SLAY_OP_CAUSAL_FWD, B, H, L, R, m)) {
        e = tc_attn_fwd_finish(q, v, out, den, B, H, L, P, eps, workspace, st, S_in, z_in);
    } else {
        const StateIO sio{S_in, z_in, nullptr, nullptr};
        e = simt_attn_fwd(q, k, v, out, den, B, H, L, dt, P, eps, true,
                          static_cast<char*>(workspace) + kWsHeader, st, &sio);
    }
    return e == cudaSuccess ? SLAY_OK : cuda_fail(e);
}

slay_status slay_state_prefix(const float* S_all, const float* z_all, int nranks, int rank,
                              float* S_in, float* z_in, int BH, int F, int Dv, void* stream)
{
    if (nranks <= 0 || rank < 0 || rank >= nranks || BH < 0 || F <= 0 || Dv <= 0)
        return SLAY_ERR_INVALID_ARG;
    if (Dv != kD || F > kMaxF) return SLAY_ERR_UNSUPPORTED;
    if (BH == 0) return SLAY_OK;
    if (!S_all || !z_all || !S_in || !z_in) return SLAY_ERR_INVALID_ARG;
    const int64_t ns = static_cast<int64_t>(BH) * F * Dv, nz = static_cast<int64_t>(BH) * F;
    cudaError_t e = simt_state_prefix(S_all, z_all, 0, rank, ns, nz, S_in, z_in,
                                      static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SLAY_OK : cuda_fail(e);
}

slay_status slay_state_suffix(const float* S_all, const float* z_all, int nranks, int rank,
                              float* S_out, float* z_out, int BH, int F, int Dv, void* stream)
{
    if (nranks <= 0 || rank < 0 || rank >= nranks || BH < 0 || F <= 0 || Dv <= 0)
        return SLAY_ERR_INVALID_ARG;
    if (Dv != kD || F > kMaxF) return SLAY_ERR_UNSUPPORTED;
    if (BH == 0) return SLAY_OK;
    if (!S_all || !z_all || !S_out || !z_out) return SLAY_ERR_INVALID_ARG;
    const int64_t ns = static_cast<int64_t>(BH) * F * Dv, nz = static_cast<int64_t>(BH) * F;
    cudaError_t e = simt_state_prefix(S_all, z_all, rank + 1, nranks, ns, nz, S_out, z_out,
                                      static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SLAY_OK : cuda_fail(e);
}

slay_status slay_attn_causal_bwd_state(const void* q, const void* k, const void* v,
                                       const void* out, const float* den, const void* dout,
                                       float* dq, float* dk, float* dv, const float* S_in,
                                       const float* z_in, const float* G_in, const float* zg_in,
                                       int B, int H, int L, int D, int Dv, slay_dtype dt, int R,
                                       int m, uint64_t seed, float eps, void* workspace,
                                       size_t ws_bytes, void* stream)
{
    slay_status s = check_state_ptrs(S_in, z_in);
    if (s != SLAY_OK) return s;
    if ((s = check_state_ptrs(G_in, zg_in)) != SLAY_OK) return s;
    const BwdStateIO sio{S_in, z_in, G_in, zg_in};
    return attn_bwd(q, k, v, out, den, dout, dq, dk, dv, B, H, L, D, Dv, dt, R, m, seed, eps,
                    workspace, ws_bytes, stream, true, &sio);
}

slay_status slay_causal_bwd_state(const void* q, const void* out, const float* den,
                                  const void* dout, float* G_out, float* zg_out, int B, int H,
                                  int L, int D, int Dv, slay_dtype dt, int R, int m, uint64_t seed,
                                  float eps, void* workspace, size_t ws_bytes, void* stream)
{
    slay_status s = check_attn(q, q, out, out, B, H, L, D, Dv, dt, R, m, eps);
    if (s != SLAY_OK) return s;
    if (!G_out || !zg_out) return SLAY_ERR_INVALID_ARG;
    if ((s = check_state_ptrs(G_out, zg_out)) != SLAY_OK) return s;
    if (static_cast<int64_t>(B) * H == 0) return SLAY_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (L == 0) {   // an empty piece: its sum is zero
        cudaError_t e = cudaMemsetAsync(G_out, 0, static_cast<size_t>(B) * H * R * m * Dv * sizeof(float), st);
        if (e == cudaSuccess)
            e = cudaMemsetAsync(zg_out, 0, static_cast<size_t>(B) * H * R * m * sizeof(float), st);
        return e == cudaSuccess ? SLAY_OK : cuda_fail(e);
    }
    if (!den || !dout || !aligned(den, 4) || !aligned(dout, 16)) return SLAY_ERR_INVALID_ARG;
    const size_t need = attn_ws(SLAY_OP_CAUSAL_BWD, dt, B, H, L, Dv, R, m);
    if (!workspace || ws_bytes < need || !aligned(workspace, 256)) return SLAY_ERR_INVALID_ARG;
    Params P;
    if ((s = get_params(D, R, m, seed, eps, &P)) != SLAY_OK) return s;
    cudaError_t e = cudaMemsetAsync(workspace, 0, sizeof(int), st);
    if (e == cudaSuccess)
        e = simt_causal_bwd_state(q, out, den, dout, G_out, zg_out, B, H, L, dt, P, eps,
                                  static_cast<char*>(workspace) + kWsHeader, st);
    return e == cudaSuccess ? SLAY_OK : cuda_fail(e);
}

slay_status slay_attn_causal_bwd_begin(const void* q, const void* out, const float* den,
                                       const void* dout, float* G_out, float* zg_out, int B, int H,
                                       int L, int D, int Dv, slay_dtype dt, int R, int m,
                                       uint64_t seed, float eps, void* workspace, size_t ws_bytes,
                                       void* stream)
{
    // slay_causal_bwd_state leaves phi(q) and the row statistics where the backward reads them
    return slay_causal_bwd_state(q, out, den, dout, G_out, zg_out, B, H, L, D, Dv, dt, R, m, seed,
                                 eps, workspace, ws_bytes, stream);
}

slay_status slay_attn_causal_bwd_finish(const void* q, const void* k, const void* v,
                                        const void* out, const float* den, const void* dout,
                                        float* dq, float* dk, float* dv, const float* S_in,
                                        const float* z_in, const float* G_in, const float* zg_in,
                                        int B, int H, int L, int D, int Dv, slay_dtype dt, int R,
                                        int m, uint64_t seed, float eps, void* workspace,
                                        size_t ws_bytes, void* stream)
{
    slay_status s = check_state_ptrs(S_in, z_in);
    if (s != SLAY_OK) return s;
    if ((s = check_state_ptrs(G_in, zg_in)) != SLAY_OK) return s;
    BwdStateIO sio{S_in, z_in, G_in, zg_in};
    sio.q_ready = true;
    return attn_bwd(q, k, v, out, den, dout, dq, dk, dv, B, H, L, D, Dv, dt, R, m, seed, eps,
                    workspace, ws_bytes, stream, true, &sio);
}

slay_status slay_feature_map_bwd(const void* x, const void* dphi, float* dx, int64_t n_rows,
                                 int D, slay_dtype x_dt, slay_dtype dphi_dt, int R, int m,
                                 uint64_t seed, float eps, void* stream)
{
    if (n_rows < 0) return SLAY_ERR_INVALID_ARG;
    slay_status s = check_shape(D, kD, R, m);
    if (s != SLAY_OK) return s;
    if (!dtype_ok(x_dt) || !dtype_ok(dphi_dt) || !eps_ok(eps)) return SLAY_ERR_INVALID_ARG;
    if (n_rows == 0) return SLAY_OK;
    if (!x || !dphi || !dx || !aligned(x, 16) || !aligned(dphi, 16) || !aligned(dx, 16))
        return SLAY_ERR_INVALID_ARG;
    if (n_rows > (int64_t(1) << 36)) return SLAY_ERR_UNSUPPORTED;
    Params P;
    if ((s = get_params(D, R, m, seed, eps, &P)) != SLAY_OK) return s;
    cudaError_t e = simt_feature_map_bwd(x, dphi, dx, n_rows, x_dt, dphi_dt, P,
                                         static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SLAY_OK : cuda_fail(e);
}

slay_status slay_decode_step(const void* q, const void* k, const void* v, float* S, float* z,
                             void* out, int Bt, int H, int D, int Dv, slay_dtype dt, int R, int m,
                             uint64_t seed, float eps, void* stream)
{
    if (Bt < 0 || H < 0) return SLAY_ERR_INVALID_ARG;
    slay_status s = check_shape(D, Dv, R, m);
    if (s != SLAY_OK) return s;
    if (!dtype_ok(dt) || !eps_ok(eps)) return SLAY_ERR_INVALID_ARG;
    const int64_t N = static_cast<int64_t>(Bt) * H;
    if (N == 0) return SLAY_OK;
    if (N > (1 << 30)) return SLAY_ERR_UNSUPPORTED;
    if (!q || !k || !v || !S || !z || !out) return SLAY_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(S, 16) ||
        !aligned(z, 16) || !aligned(out, 16))
        return SLAY_ERR_INVALID_ARG;
    Params P;
    if ((s = get_params(D, R, m, seed, eps, &P)) != SLAY_OK) return s;
    cudaError_t e = simt_decode_step(q, k, v, S, z, out, static_cast<int>(N), dt, P, eps,
                                     static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SLAY_OK : cuda_fail(e);
}

slay_status slay_kernel_status(const void* workspace, void* stream)
{
    if (workspace && !aligned(workspace, 256)) return SLAY_ERR_INVALID_ARG;
    // the caller's workspace, or the library's own words: no-alloc scratch and feature map
    const void* words[2] = {workspace, nullptr};
    if (!workspace) {
        words[0] = noalloc_status_word();
        words[1] = fmap_status_word();
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int flags[2] = {0, 0};
    cudaError_t e = cudaSuccess;
    for (int i = 0; i < 2 && e == cudaSuccess; ++i)
        if (words[i])
            e = cudaMemcpyAsync(&flags[i], words[i], sizeof(int), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e);
    for (int i = 0; i < 2; ++i)
        if (flags[i]) {
            char msg[96];
            std::snprintf(msg, sizeof msg,
                          "a bounded wait ran out (barrier at shared-memory offset 0x%x)",
                          static_cast<unsigned>(flags[i]) & 0xFFFFu);
            set_last_error(msg);
            return SLAY_ERR_TIMEOUT;
        }
    return SLAY_OK;
}

size_t slay_workspace_bytes(slay_op op, slay_dtype dt, int B, int H, int L, int D, int Dv, int R,
                            int m)
{
    if (B < 0 || H < 0 || L < 0 || !dtype_ok(dt)) return SIZE_MAX;
    if (check_shape(D, Dv, R, m) != SLAY_OK) return SIZE_MAX;
    if (op == SLAY_OP_FEATURE_MAP || op == SLAY_OP_DECODE || op == SLAY_OP_FEATURE_MAP_BWD)
        return 0;
    if (op != SLAY_OP_CAUSAL_FWD && op != SLAY_OP_BIDIR_FWD && op != SLAY_OP_CAUSAL_BWD &&
        op != SLAY_OP_BIDIR_BWD && op != SLAY_OP_LINEAR_ATTN && op != SLAY_OP_CAUSAL_STATE &&
        op != SLAY_OP_CAUSAL_FWD_SPLIT)
        return SIZE_MAX;
    if (op == SLAY_OP_LINEAR_ATTN) {   // the contraction alone: F = R * m features given
        if (static_cast<int64_t>(B) * H * L == 0) return 0;
        return kWsHeader + simt_ws_linear(B, H, L, R * m);
    }
    if (static_cast<int64_t>(B) * H * L == 0) return 0;
    return attn_ws(op, dt, B, H, L, Dv, R, m);
}

int slay_path(slay_op op, slay_dtype dt, int B, int H, int L, int D, int Dv, int R, int m)
{
    if (B < 0 || H < 0 || L < 0 || !dtype_ok(dt)) return -1;
    if (op == SLAY_OP_LINEAR_ATTN) {   // R * m features given; the chunk kernels on CUDA cores
        if (R <= 0 || m <= 0 || Dv != kD || static_cast<int64_t>(R) * m > kMaxF) return -1;
        return 0;
    }
    if (check_shape(D, Dv, R, m) != SLAY_OK) return -1;
    const bool bf = dt == SLAY_BF16;
    const bool wb = tc_wb_elems(D, R, m) > 0;   // the packed projection operand exists
    const int64_t rows = static_cast<int64_t>(B) * H * L;
    const int fwd = SLAY_PATH_TC_FEATURE_MAP | SLAY_PATH_TC_CONTRACTION;
    // the tensor-core feature map, also ahead of the CUDA-core contraction kernels in bf16
    const int fm = bf && wb && tc_fmap_supported(D, R, m, rows) ? SLAY_PATH_TC_FEATURE_MAP : 0;
    switch (op) {
    case SLAY_OP_FEATURE_MAP:   // slay_feature_map: bf16 -> bf16 on tensor cores
        return fm;
    case SLAY_OP_FEATURE_MAP_BWD:
        return bf && wb && tc_phi_bwd_supported(D, R, m, rows) ? SLAY_PATH_TC_PHI_BWD : 0;
    case SLAY_OP_CAUSAL_FWD:
    case SLAY_OP_CAUSAL_STATE:
    case SLAY_OP_CAUSAL_FWD_SPLIT:   // phi inside the fused state and output kernels
        return bf && tc_supported(SLAY_OP_CAUSAL_FWD, B, H, L, R, m) ? fwd : fm;
    case SLAY_OP_BIDIR_FWD:
        return bf && tc_supported(SLAY_OP_BIDIR_FWD, B, H, L, R, m) ? fwd : fm;
    case SLAY_OP_CAUSAL_BWD:
    case SLAY_OP_BIDIR_BWD: {
        // the rule of the backward: phi maps, the tile contraction and the chain rule through
        // phi each on tensor cores where their sizes allow; bf16 dphi (which the tensor-core
        // chain rule reads) comes from the tile contraction, or the bidirectional chunk kernel
        if (!bf || rows == 0) return 0;
        const bool tcb = tc_bwd_tile_supported(R * m, L);
        const bool tcp = wb && tc_phi_bwd_supported(D, R, m, rows);
        int mask = fm;
        if (tcb) mask |= SLAY_PATH_TC_CONTRACTION;
        if ((tcb || op == SLAY_OP_BIDIR_BWD) && tcp) mask |= SLAY_PATH_TC_PHI_BWD;
        return mask;
    }
    case SLAY_OP_DECODE:
        return 0;
    default:
        return -1;
    }
}

slay_status slay_prepare(int D, int R, int m, uint64_t seed, float eps)
{
    slay_status s = check_shape(D, kD, R, m);
    if (s != SLAY_OK) return s;
    if (!eps_ok(eps)) return SLAY_ERR_INVALID_ARG;
    Params P;
    return get_params(D, R, m, seed, eps, &P);
}

slay_status slay_sketch_params(int D, int R, int m, uint64_t seed, float eps, float* omega_host,
                               float* anchors_host, double* s_host, double* w_host)
{
    if (D <= 0 || D > 4096 || R <= 0 || R > kMaxR || m <= 0 || !eps_ok(eps))
        return SLAY_ERR_INVALID_ARG;
    if (static_cast<int64_t>(R) * m * D > (int64_t(1) << 31)) return SLAY_ERR_UNSUPPORTED;
    if (!draw_sketch(D, R, m, seed, static_cast<double>(eps), omega_host, anchors_host, s_host,
                     w_host))
        return SLAY_ERR_INVALID_ARG;
    return SLAY_OK;
}

slay_status slay_debug_expire_wait(int on)
{
    fmap_arm_wait_fault(on);
    return SLAY_OK;
}

const char* slay_status_string(slay_status st)
{
    switch (st) {
        case SLAY_OK: return "ok";
        case SLAY_ERR_INVALID_ARG: return "invalid argument";
        case SLAY_ERR_UNSUPPORTED: return "unsupported size or dtype";
        case SLAY_ERR_CUDA: return "CUDA error";
        case SLAY_ERR_TIMEOUT: return "timeout";
        case SLAY_ERR_NO_MEMORY: return "out of host memory";
    }
    return "unknown status";
}

const char* slay_last_error(void) { return g_last_error.c_str(); }

}  // extern "C"
