// slay_simt.cu -- CUDA-core (FFMA) kernels of libslay.so.
//
// This path computes every SLAY step in fp32 on the CUDA cores.  It serves the fp32
// mode (whose tolerance rules out bf16/tf32 tensor-core products) and every shape the
// tensor-core path does not take.  Method: "SLAY: Geometry-Aware Spherical Linearized
// Attention with Yat-Kernel" (abstract; nubint.ai review, "Proposed method", steps 1-6).
//
// Chunked form of the causal contraction (step 6 computes the masked sum without an
// LxL matrix): with chunks of C = 64 tokens and per-chunk sums
//   dS_c = sum_{t in c} phi(k_t) [v_t, 1]^T            (F x (Dv+1), last column = z)
// an exclusive prefix over chunks gives the state entering each chunk, and
//   out_i = (sum_{j<=i, j in c} (phi_i . phi_j) v_j + phi(q_i)^T S_c)
//           / (sum_{j<=i, j in c} phi_i . phi_j + phi(q_i)^T z_c + eps).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <type_traits>

#include "slay_internal.h"
#include "slay_tc.h"

namespace slay {
namespace {

constexpr int C = 64;     // chunk / tile edge
constexpr int E = 65;     // Dv + 1 state columns (S | z) or (dn | delta)
constexpr int NT = 256;   // threads per block

__device__ __forceinline__ float ld(const float* p) { return *p; }
__device__ __forceinline__ float ld(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void st(float* p, float x) { *p = x; }
__device__ __forceinline__ void st(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
inline int nchunks(int L) { return (L + C - 1) / C; }

// Row norms of a 64 x 64 tile held in shared memory as xs[r][d] (row stride 65):
// inv[r] = 1 / max(|x_r|, 1e-12).  All 8 warps, 8 rows each.
__device__ void tile_inv_norms(const float (*xs)[65], float* inv)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int r = warp * 8; r < warp * 8 + 8; ++r) {
        float a = xs[r][lane], b = xs[r][lane + 32];
        float s = a * a + b * b;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) inv[r] = 1.0f / fmaxf(sqrtf(s), 1e-12f);
    }
}

// ---------------------------------------------------------------- feature map
// grid (ceil(n/64), ceil(F/64)); phi[row][f] = exp2(a2_r u + b2_r) p^2 with
// u = omega_f . x^, p = a_f . x^ (steps 1, 3-5 of the review's method).
struct FmSmem {
    float xs[C][65];
    float wo[C][C + 1];
    float wa[C][C + 1];
    float inv[C];
};

template <typename Tin, typename Tout>
__global__ void __launch_bounds__(NT) k_feature_map(const Tin* __restrict__ x,
                                                    Tout* __restrict__ phi, int64_t n,
                                                    Params P)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    FmSmem& sm = *reinterpret_cast<FmSmem*>(smem_raw);
    float (*xs)[65] = sm.xs;
    float (*wo)[C + 1] = sm.wo;   // [d][f_local]
    float (*wa)[C + 1] = sm.wa;
    float* inv = sm.inv;
    const int tid = threadIdx.x;
    const int64_t row0 = static_cast<int64_t>(blockIdx.x) * C;
    const int f0 = blockIdx.y * C;
    const int F = P.F;
    for (int idx = tid; idx < C * C; idx += NT) {
        const int r = idx >> 6, d = idx & 63;
        xs[r][d] = (row0 + r < n) ? ld(x + (row0 + r) * kD + d) : 0.0f;
        const int f = f0 + (idx & 63), dd = idx >> 6;
        wo[dd][idx & 63] = (f < F) ? P.omT[dd * F + f] : 0.0f;
        wa[dd][idx & 63] = (f < F) ? P.anT[dd * F + f] : 0.0f;
    }
    __syncthreads();
    tile_inv_norms(xs, inv);
    __syncthreads();
    const int ty = tid >> 4, tx = tid & 15;
    float au[4][4] = {}, ap[4][4] = {};
#pragma unroll 4
    for (int d = 0; d < C; ++d) {
        float xv[4], o[4], a[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) xv[i] = xs[ty + 16 * i][d];
#pragma unroll
        for (int j = 0; j < 4; ++j) { o[j] = wo[d][tx + 16 * j]; a[j] = wa[d][tx + 16 * j]; }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                au[i][j] = fmaf(xv[i], o[j], au[i][j]);
                ap[i][j] = fmaf(xv[i], a[j], ap[i][j]);
            }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = ty + 16 * i;
        if (row0 + r >= n) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int f = f0 + tx + 16 * j;
            if (f >= F) continue;
            const int node = f / P.m;
            const float u = au[i][j] * inv[r], p = ap[i][j] * inv[r];
            const float val = exp2f(fmaf(P.a2[node], u, P.b2[node])) * p * p;
            st(phi + (row0 + r) * F + f, val);
        }
    }
}

// --------------------------------------------------- feature map, sketch variants
// The CUDA-core feature map for a sketch variant (slay_phi_kind): grid (ceil(Lh/64),
// ceil(F/64), n/Lh) over rows grouped Lh to a sequence; sequence z uses head z % H's
// parameters (heads are H = 1 except for the per-head kind).  kSigned: the polynomial factor
// (a.x^)(b.x^) with the second anchor set; kPerformer: phi = exp2(a2 u + b2) with no anchor
// (the node constants then hold log2 e and -(log2 e + log2 F)/2).
struct FmKindSmem {
    float xs[C][65];
    float wo[C][C + 1];
    float wa[C][C + 1];
    float wb[C][C + 1];
    float inv[C];
};

template <typename Tin, typename Tout, bool kSigned, bool kPerformer>
__global__ void __launch_bounds__(NT) k_feature_map_kind(const Tin* __restrict__ x,
                                                         Tout* __restrict__ phi, int64_t Lh,
                                                         VarParams P)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    FmKindSmem& sm = *reinterpret_cast<FmKindSmem*>(smem_raw);
    const int tid = threadIdx.x;
    const int64_t seq = blockIdx.z;
    const int head = static_cast<int>(seq % P.H);
    const int64_t r0 = static_cast<int64_t>(blockIdx.x) * C;   // row within the sequence
    const int64_t base = seq * Lh;                               // first row of the sequence
    const int f0 = blockIdx.y * C;
    const int F = P.F;
    const size_t hoff = static_cast<size_t>(head) * kD * F;
    const float* omT = P.omT + hoff;
    const float* anT = P.anT + hoff;
    const float* anbT = kSigned ? P.anbT + hoff : nullptr;
    for (int idx = tid; idx < C * C; idx += NT) {
        const int r = idx >> 6, d = idx & 63;
        sm.xs[r][d] = (r0 + r < Lh) ? ld(x + (base + r0 + r) * kD + d) : 0.0f;
        const int f = f0 + (idx & 63), dd = idx >> 6;
        sm.wo[dd][idx & 63] = (f < F) ? omT[dd * F + f] : 0.0f;
        if (!kPerformer) sm.wa[dd][idx & 63] = (f < F) ? anT[dd * F + f] : 0.0f;
        if (kSigned) sm.wb[dd][idx & 63] = (f < F) ? anbT[dd * F + f] : 0.0f;
    }
    __syncthreads();
    tile_inv_norms(sm.xs, sm.inv);
    __syncthreads();
    const int ty = tid >> 4, tx = tid & 15;
    float au[4][4] = {}, ap[4][4] = {}, bp[4][4] = {};
#pragma unroll 4
    for (int d = 0; d < C; ++d) {
        float xv[4], o[4], a[4], b[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) xv[i] = sm.xs[ty + 16 * i][d];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            o[j] = sm.wo[d][tx + 16 * j];
            a[j] = kPerformer ? 0.0f : sm.wa[d][tx + 16 * j];
            b[j] = kSigned ? sm.wb[d][tx + 16 * j] : 0.0f;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                au[i][j] = fmaf(xv[i], o[j], au[i][j]);
                if (!kPerformer) ap[i][j] = fmaf(xv[i], a[j], ap[i][j]);
                if (kSigned) bp[i][j] = fmaf(xv[i], b[j], bp[i][j]);
            }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = ty + 16 * i;
        if (r0 + r >= Lh) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int f = f0 + tx + 16 * j;
            if (f >= F) continue;
            const int node = f / P.m;
            const float u = au[i][j] * sm.inv[r];
            float val = exp2f(fmaf(P.a2[node], u, P.b2[node]));
            if (!kPerformer) {
                const float p = ap[i][j] * sm.inv[r];
                val *= kSigned ? p * (bp[i][j] * sm.inv[r]) : p * p;
            }
            st(phi + (base + r0 + r) * F + f, val);
        }
    }
}

// ------------------------------------------------------------- chunk states// ------------------------------------------------------------- chunk states
// grid (ceil(F/64), NC, BH).  st[bh][c][f][e] = sum_{t in chunk c} phi[t][f] * Y[t][e],
// e < 64 from Y, e = 64 the "ones" column (Y1 == nullptr) or Y's own column 64.
// Y is either v (type T, 64 columns) or an fp32 [L][65] array.
template <typename TY, typename TP>
__global__ void __launch_bounds__(NT) k_chunk_state(const TP* __restrict__ phi,
                                                    const TY* __restrict__ Y, int ycols,
                                                    float* __restrict__ stt, int L, int F)
{
    __shared__ float ph[C][C + 1];  // [t][f_local]
    __shared__ float ys[C][E + 1];  // [t][e]
    const int tid = threadIdx.x;
    const int f0 = blockIdx.x * C, c = blockIdx.y, bh = blockIdx.z;
    const int NC = gridDim.y;
    const int t0 = c * C;
    const TP* phb = phi + static_cast<int64_t>(bh) * L * F;
    const TY* yb = Y + static_cast<int64_t>(bh) * L * ycols;
    for (int idx = tid; idx < C * C; idx += NT) {
        const int t = idx >> 6, fl = idx & 63;
        ph[t][fl] = (t0 + t < L && f0 + fl < F) ? ld(phb + static_cast<int64_t>(t0 + t) * F + f0 + fl) : 0.0f;
    }
    for (int idx = tid; idx < C * E; idx += NT) {
        const int t = idx / E, e = idx % E;
        float val = 0.0f;
        if (t0 + t < L) {
            if (e < ycols) val = ld(yb + static_cast<int64_t>(t0 + t) * ycols + e);
            else val = 1.0f;
        }
        ys[t][e] = val;
    }
    __syncthreads();
    const int ty = tid >> 4, tx = tid & 15;
    float acc[4][5] = {};
    for (int t = 0; t < C; ++t) {
        float a[4], b[5];
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = ph[t][ty + 16 * i];
#pragma unroll
        for (int j = 0; j < 4; ++j) b[j] = ys[t][tx + 16 * j];
        b[4] = ys[t][64];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 5; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    float* out = stt + (static_cast<int64_t>(bh) * NC + c) * F * E;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int f = f0 + ty + 16 * i;
        if (f >= F) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) out[static_cast<int64_t>(f) * E + tx + 16 * j] = acc[i][j];
        if (tx == 0) out[static_cast<int64_t>(f) * E + 64] = acc[i][4];
    }
}

// Prefix over chunks of st[bh][c][FE]: mode 0 exclusive forward, mode 1 exclusive
// reverse, mode 2 total into tot[bh][FE].
__global__ void k_scan(float* __restrict__ stt, float* __restrict__ tot, int BH, int NC,
                       int FE, int mode)
{
    const int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (gid >= static_cast<int64_t>(BH) * FE) return;
    const int bh = static_cast<int>(gid / FE), idx = static_cast<int>(gid % FE);
    float* base = stt + static_cast<int64_t>(bh) * NC * FE + idx;
    // chunks are read kBatch at a time (independent loads in flight), then summed in the
    // same sequential order as a one-by-one walk
    constexpr int kBatch = 16;
    float run = 0.0f;
    for (int c0 = 0; c0 < NC; c0 += kBatch) {
        float x[kBatch];
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
            const int cc = c0 + j;
            const int c = (mode == 1) ? NC - 1 - cc : cc;
            x[j] = (cc < NC) ? base[static_cast<int64_t>(c) * FE] : 0.0f;
        }
        if (mode == 2) {
#pragma unroll
            for (int j = 0; j < kBatch; ++j) run += x[j];
            continue;
        }
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
            const int cc = c0 + j;
            if (cc < NC) {
                const int c = (mode == 1) ? NC - 1 - cc : cc;
                base[static_cast<int64_t>(c) * FE] = run;
            }
            run += x[j];
        }
    }
    if (mode == 2) tot[static_cast<int64_t>(bh) * FE + idx] = run;
}

// Exclusive prefix over chunks of st[bh][c][f][65] (rev: exclusive suffix, chunks from the
// last) starting from a given state (s_in [bh][f][64], z_in [bh][f]; null = zero), with the
// state after the last chunk walked written to s_out / z_out (each may be null).  One
// thread per (bh, f, e).
__global__ void k_scan_state(float* __restrict__ stt, int BH, int NC, int F,
                             const float* __restrict__ s_in, const float* __restrict__ z_in,
                             float* __restrict__ s_out, float* __restrict__ z_out, int rev)
{
    const int FE = F * E;
    const int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (gid >= static_cast<int64_t>(BH) * FE) return;
    const int bh = static_cast<int>(gid / FE), idx = static_cast<int>(gid % FE);
    const int f = idx / E, e = idx % E;
    float run = 0.0f;
    if (s_in) run = e < kD ? s_in[(static_cast<int64_t>(bh) * F + f) * kD + e] : z_in[static_cast<int64_t>(bh) * F + f];
    float* base = stt + static_cast<int64_t>(bh) * NC * FE + idx;
    for (int cc = 0; cc < NC; ++cc) {
        const int c = rev ? NC - 1 - cc : cc;
        const float x = base[static_cast<int64_t>(c) * FE];
        base[static_cast<int64_t>(c) * FE] = run;
        run += x;
    }
    if (e < kD) {
        if (s_out) s_out[(static_cast<int64_t>(bh) * F + f) * kD + e] = run;
    } else if (z_out) {
        z_out[static_cast<int64_t>(bh) * F + f] = run;
    }
}

// --------------------------------------------------------------- chunk output
// grid (NC, BH), dynamic smem.  Causal: intra-chunk masked term + prefix state.
// Bidirectional: total state only.
struct OutSmem {
    float qs[C][C + 1];   // phi(q) tile [i][f_local]
    float kt[C][E + 1];   // phi(k) tile [j][f_local], or state tile [f_local][e]
    float ps[C][C + 1];   // masked P [i][j]
    float vs[C][E + 1];   // [v_j, 1]
    float dens[C];
};

template <typename T>
__global__ void __launch_bounds__(NT) k_chunk_out(const T* __restrict__ phq,
                                                  const T* __restrict__ phk,
                                                  const T* __restrict__ v,
                                                  const float* __restrict__ stt,
                                                  T* __restrict__ out, float* __restrict__ den,
                                                  int L, int F, float eps, int causal)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    OutSmem& sm = *reinterpret_cast<OutSmem*>(smem_raw);
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    const int c = blockIdx.x, bh = blockIdx.y, NC = gridDim.x;
    const int i0 = c * C;
    const T* qb = phq + static_cast<int64_t>(bh) * L * F;
    const T* kb = phk + static_cast<int64_t>(bh) * L * F;
    const T* vb = v + static_cast<int64_t>(bh) * L * kD;
    // state entering this chunk (causal: exclusive prefix of chunk c; bidir: total)
    const float* sb = causal ? stt + (static_cast<int64_t>(bh) * NC + c) * F * E
                             : stt + static_cast<int64_t>(bh) * F * E;

    for (int idx = tid; idx < C * E; idx += NT) {
        const int t = idx / E, e = idx % E;
        float val = 0.0f;
        if (i0 + t < L) val = (e < kD) ? ld(vb + static_cast<int64_t>(i0 + t) * kD + e) : 1.0f;
        sm.vs[t][e] = val;
    }
    float acc[4][5] = {};
    if (causal) {
        float pa[4][4] = {};
        for (int f0 = 0; f0 < F; f0 += C) {
            __syncthreads();
            for (int idx = tid; idx < C * C; idx += NT) {
                const int t = idx >> 6, fl = idx & 63;
                const bool ok = (i0 + t < L) && (f0 + fl < F);
                const int64_t off = static_cast<int64_t>(i0 + t) * F + f0 + fl;
                sm.qs[t][fl] = ok ? ld(qb + off) : 0.0f;
                sm.kt[t][fl] = ok ? ld(kb + off) : 0.0f;
            }
            __syncthreads();
#pragma unroll 4
            for (int fl = 0; fl < C; ++fl) {
                float a[4], b[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) a[i] = sm.qs[ty + 16 * i][fl];
#pragma unroll
                for (int j = 0; j < 4; ++j) b[j] = sm.kt[tx + 16 * j][fl];
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) pa[i][j] = fmaf(a[i], b[j], pa[i][j]);
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int r = ty + 16 * i, cc = tx + 16 * j;
                sm.ps[r][cc] = (cc <= r) ? pa[i][j] : 0.0f;
            }
        __syncthreads();
        // intra: sum_j P[i][j] [v_j, 1]
        for (int j = 0; j < C; ++j) {
            float a[4], b[5];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = sm.ps[ty + 16 * i][j];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) b[jj] = sm.vs[j][tx + 16 * jj];
            b[4] = sm.vs[j][64];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int jj = 0; jj < 5; ++jj) acc[i][jj] = fmaf(a[i], b[jj], acc[i][jj]);
        }
    }
    // inter: phi(q_i)^T [S | z]
    for (int f0 = 0; f0 < F; f0 += C) {
        __syncthreads();
        for (int idx = tid; idx < C * C; idx += NT) {
            const int t = idx >> 6, fl = idx & 63;
            sm.qs[t][fl] = (i0 + t < L && f0 + fl < F) ? ld(qb + static_cast<int64_t>(i0 + t) * F + f0 + fl) : 0.0f;
        }
        for (int idx = tid; idx < C * E; idx += NT) {
            const int fl = idx / E, e = idx % E;
            sm.kt[fl][e] = (f0 + fl < F) ? sb[static_cast<int64_t>(f0 + fl) * E + e] : 0.0f;
        }
        __syncthreads();
#pragma unroll 4
        for (int fl = 0; fl < C; ++fl) {
            float a[4], b[5];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = sm.qs[ty + 16 * i][fl];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) b[jj] = sm.kt[fl][tx + 16 * jj];
            b[4] = sm.kt[fl][64];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int jj = 0; jj < 5; ++jj) acc[i][jj] = fmaf(a[i], b[jj], acc[i][jj]);
        }
    }
    if (tx == 0)
#pragma unroll
        for (int i = 0; i < 4; ++i) sm.dens[ty + 16 * i] = acc[i][4];
    __syncthreads();
    T* ob = out + static_cast<int64_t>(bh) * L * kD;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = ty + 16 * i;
        if (i0 + r >= L) continue;
        const float d = sm.dens[r];
        const float rz = 1.0f / (d + eps);
#pragma unroll
        for (int jj = 0; jj < 4; ++jj)
            st(ob + static_cast<int64_t>(i0 + r) * kD + tx + 16 * jj, acc[i][jj] * rz);
        if (den && tx == 0) den[static_cast<int64_t>(bh) * L + i0 + r] = d;
    }
}

// ------------------------------------------------------------------ backward
// dn[row][e] = g[e] / Z (e < 64), dn[row][64] = -(g . out) / Z, Z = den + eps.
template <typename T>
__global__ void k_bwd_rowstats(const T* __restrict__ out, const float* __restrict__ den,
                               const T* __restrict__ g, float* __restrict__ dn, int64_t nrows,
                               float eps)
{
    const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= nrows) return;
    const float rz = 1.0f / (den[row] + eps);
    const float g0 = ld(g + row * kD + lane), g1 = ld(g + row * kD + lane + 32);
    float s = g0 * ld(out + row * kD + lane) + g1 * ld(out + row * kD + lane + 32);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    dn[row * E + lane] = g0 * rz;
    dn[row * E + lane + 32] = g1 * rz;
    if (lane == 0) dn[row * E + 64] = -s * rz;
}

// The same statistics for the tensor-core backward: dn as bf16 rows [row][64] (its MMA operand,
// loaded by TMA) and delta as fp32 [row].  bf16 rows only: eight lanes per row, each with 16
// bytes (eight values) of out, g and dn, so a warp serves four rows with full-width accesses.
__global__ void k_bwd_rowstats_tc(const __nv_bfloat16* __restrict__ out, const float* __restrict__ den,
                                  const __nv_bfloat16* __restrict__ g, __nv_bfloat16* __restrict__ dn16,
                                  float* __restrict__ delta, int64_t nrows, float eps)
{
    const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 3;
    const int part = threadIdx.x & 7;   // values 8 part .. 8 part + 7 of the row
    const bool ok = row < nrows;
    const int64_t r = ok ? row : nrows - 1;   // (the shuffles below need every lane)
    const uint4 gv = reinterpret_cast<const uint4*>(g + r * kD)[part];
    const uint4 ov = reinterpret_cast<const uint4*>(out + r * kD)[part];
    const float rz = 1.0f / (den[r] + eps);
    const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w}, ow[4] = {ov.x, ov.y, ov.z, ov.w};
    float s = 0.0f;
    uint32_t dw[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float g0 = __uint_as_float(gw[i] << 16), g1 = __uint_as_float(gw[i] & 0xFFFF0000u);
        s = fmaf(g0, __uint_as_float(ow[i] << 16), s);
        s = fmaf(g1, __uint_as_float(ow[i] & 0xFFFF0000u), s);
        const __nv_bfloat162 d = __floats2bfloat162_rn(g0 * rz, g1 * rz);
        dw[i] = *reinterpret_cast<const uint32_t*>(&d);
    }
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (!ok) return;
    reinterpret_cast<uint4*>(dn16 + row * kD)[part] = make_uint4(dw[0], dw[1], dw[2], dw[3]);
    if (part == 0) delta[row] = -s * rz;
}

struct BwdSmem {
    float a[C][C + 1];    // phi(q) tile [i][fl]
    float b[C][C + 1];    // phi(k) tile [j][fl]
    float st[C][E + 1];   // state tile [fl][e]
    float pm[C][C + 1];   // masked P [i][j]
    float cm[C][C + 1];   // masked c_ij = v_j . dn_i + delta_i
    float vs[C][E + 1];   // v [j][e], col 64 = 1
    float dn[C][E + 1];   // [dn_i, delta_i]
};

// grid (NC, BH).  With c_ij = v_j . dn_i + delta_i and P_ij = phi(q_i) . phi(k_j)
// restricted to j <= i inside the chunk:
//   dphi(q_i) = sum_j c_ij phi(k_j) + S_c [dn_i; delta_i]        (S_c = [S | z] entering)
//   dphi(k_j) = sum_i c_ij phi(q_i) + G_c [v_j; 1]               (G_c = sum over later
//   dv_j      = sum_i P_ij dn_i + G_c[:, :64]^T phi(k_j)           chunks of phi(q)[dn, delta]^T)
// kBidir: the bidirectional form, where every query sees every key: no masked intra-chunk
// terms, and S, G are the whole sequence's sums ([BH][F][E], one per sequence):
//   dphi(q_i) = S [dn_i; delta_i],  dphi(k_j) = G [v_j; 1],  dv_j = G[:, :64]^T phi(k_j).
// dphi is written in TD (fp32, or bf16 for the tensor-core feature-map backward).
template <typename T, bool kBidir, typename TD>
__global__ void __launch_bounds__(NT) k_bwd_chunk(const T* __restrict__ phq,
                                                  const T* __restrict__ phk,
                                                  const T* __restrict__ v,
                                                  const float* __restrict__ dn,
                                                  const float* __restrict__ sfw,
                                                  const float* __restrict__ gbw,
                                                  TD* __restrict__ dphq,
                                                  TD* __restrict__ dphk,
                                                  float* __restrict__ dv, int L, int F)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    BwdSmem& sm = *reinterpret_cast<BwdSmem*>(smem_raw);
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    const int c = blockIdx.x, bh = blockIdx.y, NC = gridDim.x;
    const int i0 = c * C;
    const int64_t rb = static_cast<int64_t>(bh) * L;
    const T* qb = phq + rb * F;
    const T* kb = phk + rb * F;
    const int64_t sidx = kBidir ? static_cast<int64_t>(bh) : static_cast<int64_t>(bh) * NC + c;
    const float* S = sfw + sidx * F * E;
    const float* G = gbw + sidx * F * E;

    for (int idx = tid; idx < C * E; idx += NT) {
        const int t = idx / E, e = idx % E;
        const bool ok = i0 + t < L;
        sm.vs[t][e] = ok ? ((e < kD) ? ld(v + (rb + i0 + t) * kD + e) : 1.0f) : 0.0f;
        sm.dn[t][e] = ok ? dn[(rb + i0 + t) * E + e] : 0.0f;
    }
    float dva[4][4] = {};   // dv rows j = ty + 16 i, cols e = tx + 16 jj
    if (!kBidir) {
    // P over all feature tiles
    float pa[4][4] = {};
    for (int f0 = 0; f0 < F; f0 += C) {
        __syncthreads();
        for (int idx = tid; idx < C * C; idx += NT) {
            const int t = idx >> 6, fl = idx & 63;
            const bool ok = (i0 + t < L) && (f0 + fl < F);
            const int64_t off = static_cast<int64_t>(i0 + t) * F + f0 + fl;
            sm.a[t][fl] = ok ? ld(qb + off) : 0.0f;
            sm.b[t][fl] = ok ? ld(kb + off) : 0.0f;
        }
        __syncthreads();
        for (int fl = 0; fl < C; ++fl) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = sm.a[ty + 16 * i][fl];
#pragma unroll
            for (int j = 0; j < 4; ++j) b[j] = sm.b[tx + 16 * j][fl];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) pa[i][j] = fmaf(a[i], b[j], pa[i][j]);
        }
    }
    // c_ij = v_j . dn_i + delta_i
    float ca[4][4] = {};
    for (int e = 0; e < kD; ++e) {
        float a[4], b[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = sm.dn[ty + 16 * i][e];
#pragma unroll
        for (int j = 0; j < 4; ++j) b[j] = sm.vs[tx + 16 * j][e];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) ca[i][j] = fmaf(a[i], b[j], ca[i][j]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int r = ty + 16 * i, cc = tx + 16 * j;
            const bool keep = (cc <= r) && (i0 + r < L) && (i0 + cc < L);
            sm.pm[r][cc] = keep ? pa[i][j] : 0.0f;
            sm.cm[r][cc] = keep ? ca[i][j] + sm.dn[r][64] : 0.0f;
        }
    // dv: sum_i P_ij dn_i
    __syncthreads();
    for (int i = 0; i < C; ++i) {
        float a[4], b[4];
#pragma unroll
        for (int jr = 0; jr < 4; ++jr) a[jr] = sm.pm[i][ty + 16 * jr];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) b[jj] = sm.dn[i][tx + 16 * jj];
#pragma unroll
        for (int jr = 0; jr < 4; ++jr)
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) dva[jr][jj] = fmaf(a[jr], b[jj], dva[jr][jj]);
    }
    }   // !kBidir
    for (int f0 = 0; f0 < F; f0 += C) {
        __syncthreads();
        for (int idx = tid; idx < C * C; idx += NT) {
            const int t = idx >> 6, fl = idx & 63;
            const bool ok = (i0 + t < L) && (f0 + fl < F);
            const int64_t off = static_cast<int64_t>(i0 + t) * F + f0 + fl;
            sm.a[t][fl] = ok ? ld(qb + off) : 0.0f;
            sm.b[t][fl] = ok ? ld(kb + off) : 0.0f;
        }
        for (int idx = tid; idx < C * E; idx += NT) {
            const int fl = idx / E, e = idx % E;
            sm.st[fl][e] = (f0 + fl < F) ? S[static_cast<int64_t>(f0 + fl) * E + e] : 0.0f;
        }
        __syncthreads();
        // dphi(q)[i][fl] (rows i = ty+16a, features fl = tx+16b)
        {
            float acc[4][4] = {};
            if (!kBidir)
            for (int j = 0; j < C; ++j) {
                float a[4], b[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) a[i] = sm.cm[ty + 16 * i][j];
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) b[jj] = sm.b[j][tx + 16 * jj];
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) acc[i][jj] = fmaf(a[i], b[jj], acc[i][jj]);
            }
            for (int e = 0; e < E; ++e) {
                float a[4], b[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) a[i] = sm.dn[ty + 16 * i][e];
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) b[jj] = sm.st[tx + 16 * jj][e];
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) acc[i][jj] = fmaf(a[i], b[jj], acc[i][jj]);
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = ty + 16 * i;
                if (i0 + r >= L) continue;
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const int f = f0 + tx + 16 * jj;
                    if (f < F) st(dphq + (rb + i0 + r) * F + f, acc[i][jj]);
                }
            }
        }
        __syncthreads();
        for (int idx = tid; idx < C * E; idx += NT) {
            const int fl = idx / E, e = idx % E;
            sm.st[fl][e] = (f0 + fl < F) ? G[static_cast<int64_t>(f0 + fl) * E + e] : 0.0f;
        }
        __syncthreads();
        // dphi(k)[j][fl]
        {
            float acc[4][4] = {};
            if (!kBidir)
            for (int i = 0; i < C; ++i) {
                float a[4], b[4];
#pragma unroll
                for (int jr = 0; jr < 4; ++jr) a[jr] = sm.cm[i][ty + 16 * jr];
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) b[jj] = sm.a[i][tx + 16 * jj];
#pragma unroll
                for (int jr = 0; jr < 4; ++jr)
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) acc[jr][jj] = fmaf(a[jr], b[jj], acc[jr][jj]);
            }
            for (int e = 0; e < E; ++e) {
                float a[4], b[4];
#pragma unroll
                for (int jr = 0; jr < 4; ++jr) a[jr] = sm.vs[ty + 16 * jr][e];
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) b[jj] = sm.st[tx + 16 * jj][e];
#pragma unroll
                for (int jr = 0; jr < 4; ++jr)
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) acc[jr][jj] = fmaf(a[jr], b[jj], acc[jr][jj]);
            }
#pragma unroll
            for (int jr = 0; jr < 4; ++jr) {
                const int r = ty + 16 * jr;
                if (i0 + r >= L) continue;
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const int f = f0 + tx + 16 * jj;
                    if (f < F) st(dphk + (rb + i0 + r) * F + f, acc[jr][jj]);
                }
            }
        }
        // dv += G[:, :64]^T phi(k_j) over this feature tile
        for (int fl = 0; fl < C; ++fl) {
            float a[4], b[4];
#pragma unroll
            for (int jr = 0; jr < 4; ++jr) a[jr] = sm.b[ty + 16 * jr][fl];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) b[jj] = sm.st[fl][tx + 16 * jj];
#pragma unroll
            for (int jr = 0; jr < 4; ++jr)
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) dva[jr][jj] = fmaf(a[jr], b[jj], dva[jr][jj]);
        }
    }
#pragma unroll
    for (int jr = 0; jr < 4; ++jr) {
        const int r = ty + 16 * jr;
        if (i0 + r >= L) continue;
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) dv[(rb + i0 + r) * kD + tx + 16 * jj] = dva[jr][jj];
    }
}

// Chain rule through phi and the sphere projection, 64 rows per block:
//   d phi_f / d x^ = phi_f sqrt(2 s_r) omega_f + 2 c_r E_f p_f a_f,  (c_r E_f = exp2(a2 u + b2))
//   dx = (dx^ - x^ (x^ . dx^)) / |x|   (or dx^ / 1e-12 when the norm guard is active)
struct PhiBwdSmem {
    float xs[C][65];
    float w1[C][C + 1];   // omega^T tile [d][fl], then omega tile [fl][d]
    float w2[C][C + 1];   // anchors^T tile, then anchors tile
    float go[C][C + 1];   // [row][fl]
    float ga[C][C + 1];
    float inv[C];
    float nrm[C];
};

template <typename Tin, typename TG>
__global__ void __launch_bounds__(NT) k_phi_bwd(const Tin* __restrict__ x,
                                                const TG* __restrict__ dphi,
                                                float* __restrict__ dx, int64_t n, Params P)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    PhiBwdSmem& sm = *reinterpret_cast<PhiBwdSmem*>(smem_raw);
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    const int64_t row0 = static_cast<int64_t>(blockIdx.x) * C;
    const int F = P.F;
    for (int idx = tid; idx < C * C; idx += NT) {
        const int r = idx >> 6, d = idx & 63;
        sm.xs[r][d] = (row0 + r < n) ? ld(x + (row0 + r) * kD + d) : 0.0f;
    }
    __syncthreads();
    {
        const int warp = tid >> 5, lane = tid & 31;
        for (int r = warp * 8; r < warp * 8 + 8; ++r) {
            float a = sm.xs[r][lane], b = sm.xs[r][lane + 32];
            float s = a * a + b * b;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
            if (lane == 0) { sm.nrm[r] = sqrtf(s); sm.inv[r] = 1.0f / fmaxf(sqrtf(s), 1e-12f); }
        }
    }
    __syncthreads();
    for (int idx = tid; idx < C * C; idx += NT) {
        const int r = idx >> 6, d = idx & 63;
        sm.xs[r][d] *= sm.inv[r];   // x^
    }
    float acc[4][4] = {};  // dx^[row ty+16i][d tx+16j]
    for (int f0 = 0; f0 < F; f0 += C) {
        __syncthreads();
        for (int idx = tid; idx < C * C; idx += NT) {
            const int dd = idx >> 6, fl = idx & 63;
            const int f = f0 + fl;
            sm.w1[dd][fl] = (f < F) ? P.omT[dd * F + f] : 0.0f;
            sm.w2[dd][fl] = (f < F) ? P.anT[dd * F + f] : 0.0f;
        }
        __syncthreads();
        float u[4][4] = {}, p[4][4] = {};
        for (int d = 0; d < C; ++d) {
            float xv[4], o[4], a[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) xv[i] = sm.xs[ty + 16 * i][d];
#pragma unroll
            for (int j = 0; j < 4; ++j) { o[j] = sm.w1[d][tx + 16 * j]; a[j] = sm.w2[d][tx + 16 * j]; }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    u[i][j] = fmaf(xv[i], o[j], u[i][j]);
                    p[i][j] = fmaf(xv[i], a[j], p[i][j]);
                }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = ty + 16 * i;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int fl = tx + 16 * j, f = f0 + fl;
                float gov = 0.0f, gav = 0.0f;
                if (f < F && row0 + r < n) {
                    const int node = f / P.m;
                    const float cE = exp2f(fmaf(P.a2[node], u[i][j], P.b2[node]));
                    const float g = ld(dphi + (row0 + r) * F + f);
                    gov = g * cE * p[i][j] * p[i][j] * P.sq[node];
                    gav = 2.0f * g * cE * p[i][j];
                }
                sm.go[r][fl] = gov;
                sm.ga[r][fl] = gav;
            }
        }
        __syncthreads();
        for (int idx = tid; idx < C * C; idx += NT) {
            const int fl = idx >> 6, dd = idx & 63;
            const int f = f0 + fl;
            sm.w1[fl][dd] = (f < F) ? P.om[static_cast<int64_t>(f) * kD + dd] : 0.0f;
            sm.w2[fl][dd] = (f < F) ? P.an[static_cast<int64_t>(f) * kD + dd] : 0.0f;
        }
        __syncthreads();
        for (int fl = 0; fl < C; ++fl) {
            float g1[4], g2[4], o[4], a[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) { g1[i] = sm.go[ty + 16 * i][fl]; g2[i] = sm.ga[ty + 16 * i][fl]; }
#pragma unroll
            for (int j = 0; j < 4; ++j) { o[j] = sm.w1[fl][tx + 16 * j]; a[j] = sm.w2[fl][tx + 16 * j]; }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(g1[i], o[j], fmaf(g2[i], a[j], acc[i][j]));
        }
    }
    __syncthreads();
    // stash dx^ in go, then project out the radial part
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) sm.go[ty + 16 * i][tx + 16 * j] = acc[i][j];
    __syncthreads();
    {
        const int warp = tid >> 5, lane = tid & 31;
        for (int r = warp * 8; r < warp * 8 + 8; ++r) {
            if (row0 + r >= n) continue;
            const float a0 = sm.go[r][lane], a1 = sm.go[r][lane + 32];
            const float x0 = sm.xs[r][lane], x1 = sm.xs[r][lane + 32];
            float s = a0 * x0 + a1 * x1;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
            const bool guard = !(sm.nrm[r] >= 1e-12f);
            const float iv = sm.inv[r];
            float* out = dx + (row0 + r) * kD;
            out[lane] = guard ? a0 * iv : (a0 - x0 * s) * iv;
            out[lane + 32] = guard ? a1 * iv : (a1 - x1 * s) * iv;
        }
    }
}

// -------------------------------------------------------------------- decode
// One block per group of G sequences (b,h).  Phase 1: phi of q and k of the group.
// Phase 2: stream S (read, add phi(k) v^T, write) and accumulate phi(q)^T S.
constexpr int G = 4;
constexpr int kDecodeBlocksPerSM = 5;   // register cap 51/thread: 5 resident blocks per SM

template <typename T>
__global__ void __launch_bounds__(NT, kDecodeBlocksPerSM) k_decode(const T* __restrict__ q, const T* __restrict__ k,
                                               const T* __restrict__ v, float* __restrict__ S,
                                               float* __restrict__ z, T* __restrict__ out, int N,
                                               Params P, float eps)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    float* ph = reinterpret_cast<float*>(smem_raw);   // [2G][F]: q rows then k rows
    __shared__ float xs[2 * G][kD];
    __shared__ float inv[2 * G];
    __shared__ float red[16][kD];
    __shared__ float dred[NT / 32];
    const int tid = threadIdx.x;
    const int F = P.F;
    // persistent: block b serves groups b, b + gridDim.x, ... of G sequences each
    for (int n0 = blockIdx.x * G; n0 < N; n0 += gridDim.x * G) {
    for (int idx = tid; idx < 2 * G * kD; idx += NT) {
        const int r = idx / kD, d = idx % kD;
        const int g = r % G, n = n0 + g;
        float val = 0.0f;
        if (n < N) val = (r < G) ? ld(q + static_cast<int64_t>(n) * kD + d) : ld(k + static_cast<int64_t>(n) * kD + d);
        xs[r][d] = val;
    }
    __syncthreads();
    if (tid < 2 * G) {
        float s = 0.0f;
        for (int d = 0; d < kD; ++d) s += xs[tid][d] * xs[tid][d];
        inv[tid] = 1.0f / fmaxf(sqrtf(s), 1e-12f);
    }
    __syncthreads();
    for (int f = tid; f < F; f += NT) {
        float u[2 * G] = {}, p[2 * G] = {};
        for (int d = 0; d < kD; ++d) {
            const float o = P.omT[d * F + f], a = P.anT[d * F + f];
#pragma unroll
            for (int r = 0; r < 2 * G; ++r) { u[r] = fmaf(xs[r][d], o, u[r]); p[r] = fmaf(xs[r][d], a, p[r]); }
        }
        const int node = f / P.m;
#pragma unroll
        for (int r = 0; r < 2 * G; ++r) {
            const float uu = u[r] * inv[r], pp = p[r] * inv[r];
            ph[r * F + f] = exp2f(fmaf(P.a2[node], uu, P.b2[node])) * pp * pp;
        }
    }
    __syncthreads();
    const int e4 = (tid & 15) * 4, fr = tid >> 4;
    for (int g = 0; g < G; ++g) {
        const int n = n0 + g;
        if (n >= N) break;   // uniform across the block
        const float* phq = ph + g * F;
        const float* phk = ph + (G + g) * F;
        float4 vv;
        {
            const T* vp = v + static_cast<int64_t>(n) * kD + e4;
            vv = make_float4(ld(vp), ld(vp + 1), ld(vp + 2), ld(vp + 3));
        }
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        float* Sn = S + static_cast<int64_t>(n) * F * kD;
#pragma unroll 8
        for (int f = fr; f < F; f += 16) {
            float4* sp = reinterpret_cast<float4*>(Sn + static_cast<int64_t>(f) * kD + e4);
            float4 s = *sp;
            const float a = phk[f], b = phq[f];
            s.x = fmaf(a, vv.x, s.x); s.y = fmaf(a, vv.y, s.y);
            s.z = fmaf(a, vv.z, s.z); s.w = fmaf(a, vv.w, s.w);
            *sp = s;
            acc.x = fmaf(b, s.x, acc.x); acc.y = fmaf(b, s.y, acc.y);
            acc.z = fmaf(b, s.z, acc.z); acc.w = fmaf(b, s.w, acc.w);
        }
        red[fr][e4] = acc.x; red[fr][e4 + 1] = acc.y; red[fr][e4 + 2] = acc.z; red[fr][e4 + 3] = acc.w;
        // z update and phi(q) . z
        float dp = 0.0f;
        float* zn = z + static_cast<int64_t>(n) * F;
        for (int f = tid; f < F; f += NT) {
            const float zz = zn[f] + phk[f];
            zn[f] = zz;
            dp = fmaf(phq[f], zz, dp);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) dp += __shfl_xor_sync(0xffffffffu, dp, o);
        if ((tid & 31) == 0) dred[tid >> 5] = dp;
        __syncthreads();
        if (tid < kD) {
            float num = 0.0f;
#pragma unroll
            for (int i = 0; i < 16; ++i) num += red[i][tid];
            float d = 0.0f;
#pragma unroll
            for (int w = 0; w < NT / 32; ++w) d += dred[w];
            st(out + static_cast<int64_t>(n) * kD + tid, num / (d + eps));
        }
        __syncthreads();
    }
    }
}

template <typename T>
inline const T* cp(const void* p) { return static_cast<const T*>(p); }
template <typename T>
inline T* mp(void* p) { return static_cast<T*>(p); }

}  // namespace

// ----------------------------------------------------------------- launchers

size_t simt_ws_causal(int B, int H, int L, int /*Dv*/, int F)
{
    const size_t BH = static_cast<size_t>(B) * H;
    const size_t phi = align256(BH * L * F * sizeof(float));
    const size_t stt = align256(BH * nchunks(L) * static_cast<size_t>(F) * E * sizeof(float));
    return 2 * phi + stt;
}

size_t simt_ws_bidir(int B, int H, int L, int Dv, int F)
{
    const size_t BH = static_cast<size_t>(B) * H;
    return simt_ws_causal(B, H, L, Dv, F) + align256(BH * F * E * sizeof(float));
}

size_t simt_ws_bwd(int B, int H, int L, int /*Dv*/, int F)
{
    const size_t BH = static_cast<size_t>(B) * H;
    const size_t phi = align256(BH * L * F * sizeof(float));
    const size_t stt = align256(BH * nchunks(L) * static_cast<size_t>(F) * E * sizeof(float));
    const size_t dn = align256(BH * L * E * sizeof(float));
    return 4 * phi + 2 * stt + dn;
}

// the causal backward's carve-outs plus the two whole-sequence sums [BH][F][E]
size_t simt_ws_bidir_bwd(int B, int H, int L, int Dv, int F)
{
    const size_t BH = static_cast<size_t>(B) * H;
    return simt_ws_bwd(B, H, L, Dv, F) + 2 * align256(BH * F * E * sizeof(float));
}

template <typename Tin, typename Tout>
static cudaError_t fm_launch(const void* x, void* phi, int64_t n, const Params& P, cudaStream_t st)
{
    const dim3 grid(static_cast<unsigned>((n + C - 1) / C), (P.F + C - 1) / C);
    const size_t smem = sizeof(FmSmem);
    cudaError_t err = cudaFuncSetAttribute(k_feature_map<Tin, Tout>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    {
        TraceScope trace_("simt_feature_map", st);
        k_feature_map<Tin, Tout><<<grid, NT, smem, st>>>(cp<Tin>(x), mp<Tout>(phi), n, P);
    }
    return cudaGetLastError();
}

cudaError_t simt_feature_map(const void* x, void* phi, int64_t n, slay_dtype in_dt,
                             slay_dtype out_dt, const Params& P, cudaStream_t st)
{
    if (in_dt == SLAY_F32 && out_dt == SLAY_F32) return fm_launch<float, float>(x, phi, n, P, st);
    if (in_dt == SLAY_BF16 && out_dt == SLAY_BF16)
        return fm_launch<__nv_bfloat16, __nv_bfloat16>(x, phi, n, P, st);
    return fm_launch<__nv_bfloat16, float>(x, phi, n, P, st);
}

// phi of `rows` rows of x in the mode's dtype: tensor cores for bf16 where the shape allows
template <typename T>
static cudaError_t phi_map(const void* x, T* phi, int64_t rows, const Params& P, cudaStream_t st)
{
    if (std::is_same<T, __nv_bfloat16>::value && P.wB && tc_fmap_supported(P.D, P.R, P.m, rows))
        return tc_feature_map(x, phi, rows, P, st);
    return fm_launch<T, T>(x, phi, rows, P, st);
}

template <typename T>
static cudaError_t attn_fwd_t(const void* q, const void* k, const void* v, void* out, float* den,
                              int B, int H, int L, const Params& P, float eps, bool causal,
                              void* ws, cudaStream_t st, const StateIO* sio)
{
    const int BH = B * H, F = P.F, NC = nchunks(L);
    const int64_t rows = static_cast<int64_t>(BH) * L;
    char* w = static_cast<char*>(ws);
    // phi(q), phi(k) in the mode's dtype (the buffers are sized for fp32)
    T* phq = reinterpret_cast<T*>(w);
    T* phk = reinterpret_cast<T*>(w + align256(rows * F * sizeof(float)));
    float* stt = reinterpret_cast<float*>(w + 2 * align256(rows * F * sizeof(float)));
    float* tot = reinterpret_cast<float*>(w + 2 * align256(rows * F * sizeof(float)) +
                                          align256(static_cast<size_t>(BH) * NC * F * E * sizeof(float)));
    cudaError_t err;
    if ((err = phi_map<T>(q, phq, rows, P, st)) != cudaSuccess) return err;
    if ((err = phi_map<T>(k, phk, rows, P, st)) != cudaSuccess) return err;
    {
        TraceScope trace_("simt_chunk_state", st);
        k_chunk_state<T, T><<<dim3((F + C - 1) / C, NC, BH), NT, 0, st>>>(phk, cp<T>(v), kD, stt, L, F);
    }
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    const int FE = F * E;
    const int64_t nth = static_cast<int64_t>(BH) * FE;
    {
        TraceScope trace_("simt_scan", st);
        if (causal && sio)
            k_scan_state<<<static_cast<unsigned>((nth + 255) / 256), 256, 0, st>>>(
                stt, BH, NC, F, sio->s_in, sio->z_in, sio->s_out, sio->z_out, 0);
        else
            k_scan<<<static_cast<unsigned>((nth + 255) / 256), 256, 0, st>>>(stt, tot, BH, NC, FE, causal ? 0 : 2);
    }
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    const size_t smem = sizeof(OutSmem);
    if ((err = cudaFuncSetAttribute(k_chunk_out<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>(smem))) != cudaSuccess)
        return err;
    {
        TraceScope trace_("simt_chunk_out", st);
        k_chunk_out<T><<<dim3(NC, BH), NT, smem, st>>>(phq, phk, cp<T>(v), causal ? stt : tot,
                                                       mp<T>(out), den, L, F, eps, causal ? 1 : 0);
    }
    return cudaGetLastError();
}

// The causal state of a whole sequence chunk, sum_j phi(k_j) [v_j, 1]^T -> S [bh][f][64],
// z [bh][f] (plus an optional initial state): phi(k), the chunk states, their total.
template <typename T>
static cudaError_t causal_state_t(const void* k, const void* v, int B, int H, int L,
                                  const Params& P, void* ws, cudaStream_t st, const StateIO& sio)
{
    const int BH = B * H, F = P.F, NC = nchunks(L);
    const int64_t rows = static_cast<int64_t>(BH) * L;
    char* w = static_cast<char*>(ws);
    T* phk = reinterpret_cast<T*>(w);
    float* stt = reinterpret_cast<float*>(w + align256(rows * F * sizeof(float)));
    cudaError_t err;
    if ((err = phi_map<T>(k, phk, rows, P, st)) != cudaSuccess) return err;
    {
        TraceScope trace_("simt_chunk_state", st);
        k_chunk_state<T, T><<<dim3((F + C - 1) / C, NC, BH), NT, 0, st>>>(phk, cp<T>(v), kD, stt, L, F);
    }
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    const int64_t nth = static_cast<int64_t>(BH) * F * E;
    TraceScope trace_("simt_scan", st);
    k_scan_state<<<static_cast<unsigned>((nth + 255) / 256), 256, 0, st>>>(stt, BH, NC, F, sio.s_in,
                                                                           sio.z_in, sio.s_out, sio.z_out, 0);
    return cudaGetLastError();
}

size_t simt_ws_state(int B, int H, int L, int F)
{
    const size_t BH = static_cast<size_t>(B) * H;
    return align256(BH * L * F * sizeof(float)) +
           align256(BH * nchunks(L) * static_cast<size_t>(F) * E * sizeof(float));
}

cudaError_t simt_causal_state(const void* k, const void* v, int B, int H, int L, slay_dtype dt,
                              const Params& P, void* ws, cudaStream_t st, const StateIO& sio)
{
    if (dt == SLAY_F32) return causal_state_t<float>(k, v, B, H, L, P, ws, st, sio);
    return causal_state_t<__nv_bfloat16>(k, v, B, H, L, P, ws, st, sio);
}

// S_in = sum of the per-rank states of the ranks before `rank` (an exclusive prefix over the
// all-gathered [nranks][BH][F][64] states and [nranks][BH][F] z), one thread per element
__global__ void k_state_prefix(const float* __restrict__ s_all, const float* __restrict__ z_all,
                               int r0, int r1, int64_t ns, int64_t nz,
                               float* __restrict__ s_in, float* __restrict__ z_in)
{
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < ns;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        float a = 0.0f;
        for (int r = r0; r < r1; ++r) a += s_all[static_cast<int64_t>(r) * ns + i];
        s_in[i] = a;
        if (i < nz) {
            float b = 0.0f;
            for (int r = r0; r < r1; ++r) b += z_all[static_cast<int64_t>(r) * nz + i];
            z_in[i] = b;
        }
    }
}

// The sum of the gathered states of ranks r0 .. r1 - 1 in rank order (the prefix of a rank
// is r0 = 0, r1 = rank; its suffix r0 = rank + 1, r1 = nranks).
cudaError_t simt_state_prefix(const float* s_all, const float* z_all, int r0, int r1,
                              int64_t ns, int64_t nz, float* s_in, float* z_in, cudaStream_t st)
{
    const int grid = static_cast<int>(std::min<int64_t>((ns + 255) / 256, 1184));
    TraceScope trace_("simt_state_prefix", st);
    k_state_prefix<<<grid, 256, 0, st>>>(s_all, z_all, r0, r1, ns, nz, s_in, z_in);
    return cudaGetLastError();
}

cudaError_t simt_attn_fwd(const void* q, const void* k, const void* v, void* out, float* den,
                          int B, int H, int L, slay_dtype dt, const Params& P, float eps,
                          bool causal, void* ws, cudaStream_t st, const StateIO* sio)
{
    if (dt == SLAY_F32) return attn_fwd_t<float>(q, k, v, out, den, B, H, L, P, eps, causal, ws, st, sio);
    return attn_fwd_t<__nv_bfloat16>(q, k, v, out, den, B, H, L, P, eps, causal, ws, st, sio);
}

template <typename Tin, typename Tout, bool kSigned, bool kPerformer>
static cudaError_t fm_kind_launch(const void* x, void* phi, int64_t n, int64_t Lh,
                                  const VarParams& P, cudaStream_t st)
{
    auto kern = k_feature_map_kind<Tin, Tout, kSigned, kPerformer>;
    const size_t smem = sizeof(FmKindSmem);
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    const dim3 grid(static_cast<unsigned>((Lh + C - 1) / C), (P.F + C - 1) / C,
                    static_cast<unsigned>(n / Lh));
    TraceScope trace_("simt_feature_map_kind", st);
    kern<<<grid, NT, smem, st>>>(cp<Tin>(x), mp<Tout>(phi), Lh, P);
    return cudaGetLastError();
}

template <typename Tin, typename Tout>
static cudaError_t fm_kind_t(const void* x, void* phi, int64_t n, int64_t Lh, const VarParams& P,
                             cudaStream_t st)
{
    if (P.kind == 2) return fm_kind_launch<Tin, Tout, true, false>(x, phi, n, Lh, P, st);
    if (P.kind == 4) return fm_kind_launch<Tin, Tout, false, true>(x, phi, n, Lh, P, st);
    return fm_kind_launch<Tin, Tout, false, false>(x, phi, n, Lh, P, st);
}

cudaError_t simt_feature_map_kind(const void* x, void* phi, int64_t n, int64_t Lh,
                                  slay_dtype in_dt, slay_dtype out_dt, const VarParams& P,
                                  cudaStream_t st)
{
    if (in_dt == SLAY_F32 && out_dt == SLAY_F32) return fm_kind_t<float, float>(x, phi, n, Lh, P, st);
    if (in_dt == SLAY_BF16 && out_dt == SLAY_BF16)
        return fm_kind_t<__nv_bfloat16, __nv_bfloat16>(x, phi, n, Lh, P, st);
    return fm_kind_t<__nv_bfloat16, float>(x, phi, n, Lh, P, st);
}

// The contraction on given features phi(q), phi(k) [BH][L][F] (in the mode's dtype): chunk
// states, the scan over chunks (causal prefix or whole-sequence total) and the chunk output.
size_t simt_ws_linear(int B, int H, int L, int F)
{
    const size_t BH = static_cast<size_t>(B) * H;
    return align256(BH * nchunks(L) * static_cast<size_t>(F) * E * sizeof(float)) +
           align256(BH * static_cast<size_t>(F) * E * sizeof(float));
}

template <typename T>
static cudaError_t linear_attn_t(const void* phq_, const void* phk_, const void* v, void* out,
                                 float* den, int B, int H, int L, int F, float eps, bool causal,
                                 void* ws, cudaStream_t st)
{
    const int BH = B * H, NC = nchunks(L);
    const T* phq = cp<T>(phq_);
    const T* phk = cp<T>(phk_);
    char* w = static_cast<char*>(ws);
    float* stt = reinterpret_cast<float*>(w);
    float* tot = reinterpret_cast<float*>(w + align256(static_cast<size_t>(BH) * NC * F * E * sizeof(float)));
    cudaError_t err;
    {
        TraceScope trace_("simt_chunk_state", st);
        k_chunk_state<T, T><<<dim3((F + C - 1) / C, NC, BH), NT, 0, st>>>(phk, cp<T>(v), kD, stt, L, F);
    }
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    const int64_t nth = static_cast<int64_t>(BH) * F * E;
    {
        TraceScope trace_("simt_scan", st);
        k_scan<<<static_cast<unsigned>((nth + 255) / 256), 256, 0, st>>>(stt, tot, BH, NC, F * E,
                                                                         causal ? 0 : 2);
    }
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    const size_t smem = sizeof(OutSmem);
    if ((err = cudaFuncSetAttribute(k_chunk_out<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>(smem))) != cudaSuccess)
        return err;
    {
        TraceScope trace_("simt_chunk_out", st);
        k_chunk_out<T><<<dim3(NC, BH), NT, smem, st>>>(phq, phk, cp<T>(v), causal ? stt : tot,
                                                       mp<T>(out), den, L, F, eps, causal ? 1 : 0);
    }
    return cudaGetLastError();
}

cudaError_t simt_linear_attn(const void* phq, const void* phk, const void* v, void* out,
                             float* den, int B, int H, int L, int F, slay_dtype dt, float eps,
                             bool causal, void* ws, cudaStream_t st)
{
    if (dt == SLAY_F32) return linear_attn_t<float>(phq, phk, v, out, den, B, H, L, F, eps, causal, ws, st);
    return linear_attn_t<__nv_bfloat16>(phq, phk, v, out, den, B, H, L, F, eps, causal, ws, st);
}

template <typename T>
static cudaError_t attn_bwd_t(const void* q, const void* k, const void* v, const void* out,
                              const float* den, const void* dout, float* dq, float* dk,
                              float* dv, int B, int H, int L, const Params& P, float eps,
                              void* ws, cudaStream_t st, bool bidir,
                              const BwdStateIO* sio = nullptr)
{
    const int BH = B * H, F = P.F, NC = nchunks(L);
    const int64_t rows = static_cast<int64_t>(BH) * L;
    const size_t phb = align256(rows * F * sizeof(float));
    const size_t stb = align256(static_cast<size_t>(BH) * NC * F * E * sizeof(float));
    char* w = static_cast<char*>(ws);
    T* phq = reinterpret_cast<T*>(w);   // phi in the mode's dtype (buffers sized for fp32)
    T* phk = reinterpret_cast<T*>(w + phb);
    float* dphq = reinterpret_cast<float*>(w + 2 * phb);
    float* dphk = reinterpret_cast<float*>(w + 3 * phb);
    float* sfw = reinterpret_cast<float*>(w + 4 * phb);
    float* gbw = reinterpret_cast<float*>(w + 4 * phb + stb);
    float* dn = reinterpret_cast<float*>(w + 4 * phb + 2 * stb);
    cudaError_t err;
    // phi(q) and the row statistics may be in the workspace already (the first call of the
    // two-call backward computed them at the same places)
    const bool q_ready = sio && sio->q_ready;
    if (!q_ready && (err = phi_map<T>(q, phq, rows, P, st)) != cudaSuccess) return err;
    if ((err = phi_map<T>(k, phk, rows, P, st)) != cudaSuccess) return err;
    // bf16 phi: states, contraction on tensor cores over 128-token tiles; else 64-token chunks
    // (the bidirectional form: the same kernels with whole-sequence sums and no masked term)
    const bool tcb = std::is_same<T, __nv_bfloat16>::value && tc_bwd_tile_supported(F, L);
    // tensor-core path: dn as bf16 rows and delta in the dn region (132 of its 260 bytes a row)
    __nv_bfloat16* dn16 = reinterpret_cast<__nv_bfloat16*>(dn);
    float* delta = reinterpret_cast<float*>(dn16 + rows * kD);
    if (!q_ready) {
        TraceScope trace_("simt_bwd_rowstats", st);
        if (tcb)
            k_bwd_rowstats_tc<<<static_cast<unsigned>((rows + 31) / 32), 256, 0, st>>>(
                reinterpret_cast<const __nv_bfloat16*>(out), den,
                reinterpret_cast<const __nv_bfloat16*>(dout), dn16, delta, rows, eps);
        else
            k_bwd_rowstats<T><<<static_cast<unsigned>((rows + 7) / 8), 256, 0, st>>>(
                cp<T>(out), den, cp<T>(dout), dn, rows, eps);
    }
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    // with the feature map's backward on tensor cores as well, dphi travels as bf16
    const bool tcp = std::is_same<T, __nv_bfloat16>::value && P.wB &&
                     tc_phi_bwd_supported(kD, P.R, P.m, rows);
    const bool dphi16 = (tcb || bidir) && tcp;
    const int NS = tcb ? (L + 127) / 128 : NC;   // state blocks per sequence
    int* status = reinterpret_cast<int*>(w - kWsHeader);
    if (!tcb) {   // (tensor-core path: the running sums below, after the total buffers)
        const dim3 sg((F + C - 1) / C, NC, BH);
        {
            TraceScope trace_("simt_chunk_state", st);
            k_chunk_state<T, T><<<sg, NT, 0, st>>>(phk, cp<T>(v), kD, sfw, L, F);
        }
        {
            TraceScope trace_("simt_chunk_state", st);
            k_chunk_state<float, T><<<sg, NT, 0, st>>>(phq, dn, E, gbw, L, F);
        }
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
    }
    const int FE = F * E;
    const int64_t nth = static_cast<int64_t>(BH) * FE;
    const unsigned sgrid = static_cast<unsigned>((nth + 255) / 256);
    // bidirectional: the whole-sequence sums, after the causal carve-outs
    float* stot = reinterpret_cast<float*>(w + simt_ws_bwd(B, H, L, kD, F));
    float* gtot = stot + align256(static_cast<size_t>(BH) * FE * sizeof(float)) / sizeof(float);
    if (tcb) {   // running sums over the tiles, written as the contraction's bf16 operands
        BwdSeeds seeds;   // a piece of a longer sequence: the sums outside it seed them
        if (sio) {
            seeds.s_in = sio->s_in;
            seeds.z_in = sio->z_in;
            seeds.g_in = sio->g_in;
            seeds.zg_in = sio->zg_in;
        }
        if ((err = tc_bwd_sums(phq, phk, v, dn16, delta, sfw, gbw, stot, gtot, BH, L, F, bidir,
                               status, st, &seeds)) != cudaSuccess)
            return err;
    } else if (sio) {   // causal piece: the chunk scans start from the outside sums
        {
            TraceScope trace_("simt_scan", st);
            k_scan_state<<<sgrid, 256, 0, st>>>(sfw, BH, NS, F, sio->s_in, sio->z_in, nullptr,
                                                nullptr, 0);
        }
        {
            TraceScope trace_("simt_scan", st);
            k_scan_state<<<sgrid, 256, 0, st>>>(gbw, BH, NS, F, sio->g_in, sio->zg_in, nullptr,
                                                nullptr, 1);
        }
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
    } else {
        {
            TraceScope trace_("simt_scan", st);
            k_scan<<<sgrid, 256, 0, st>>>(sfw, stot, BH, NS, FE, bidir ? 2 : 0);
        }
        {
            TraceScope trace_("simt_scan", st);
            k_scan<<<sgrid, 256, 0, st>>>(gbw, gtot, BH, NS, FE, bidir ? 2 : 1);
        }
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
    }
    if (tcb) {
        if ((err = tc_bwd_tile(phq, phk, v, dn16, delta, bidir ? stot : sfw, bidir ? gtot : gbw,
                               dphq, dphk, dphi16, dv, BH, L, F, status, st, bidir)) != cudaSuccess)
            return err;
    } else if (bidir) {
        // dphi as bf16 when the tensor-core feature-map backward takes it, else fp32
        if (dphi16) {
            auto kern = k_bwd_chunk<T, true, __nv_bfloat16>;
            const size_t smem = sizeof(BwdSmem);
            if ((err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            static_cast<int>(smem))) != cudaSuccess)
                return err;
            TraceScope trace_("simt_bwd_chunk", st);
            kern<<<dim3(NC, BH), NT, smem, st>>>(phq, phk, cp<T>(v), dn, stot, gtot,
                                                 reinterpret_cast<__nv_bfloat16*>(dphq),
                                                 reinterpret_cast<__nv_bfloat16*>(dphk), dv, L, F);
        } else {
            auto kern = k_bwd_chunk<T, true, float>;
            const size_t smem = sizeof(BwdSmem);
            if ((err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            static_cast<int>(smem))) != cudaSuccess)
                return err;
            TraceScope trace_("simt_bwd_chunk", st);
            kern<<<dim3(NC, BH), NT, smem, st>>>(phq, phk, cp<T>(v), dn, stot, gtot, dphq, dphk,
                                                 dv, L, F);
        }
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
    } else {
        const size_t smem = sizeof(BwdSmem);
        auto kern = k_bwd_chunk<T, false, float>;
        if ((err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        static_cast<int>(smem))) != cudaSuccess)
            return err;
        {
            TraceScope trace_("simt_bwd_chunk", st);
            kern<<<dim3(NC, BH), NT, smem, st>>>(phq, phk, cp<T>(v), dn, sfw, gbw, dphq, dphk, dv,
                                                 L, F);
        }
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
    }
    const size_t psm = sizeof(PhiBwdSmem);
    if ((err = cudaFuncSetAttribute(k_phi_bwd<T, float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>(psm))) != cudaSuccess)
        return err;
    // bf16 inputs: the feature map's backward on tensor cores when it takes these sizes
    if (dphi16) {
        if ((err = tc_phi_bwd(q, dphq, dq, rows, P, st)) != cudaSuccess) return err;
        return tc_phi_bwd(k, dphk, dk, rows, P, st);
    }
    const unsigned rg = static_cast<unsigned>((rows + C - 1) / C);
    {
        TraceScope trace_("simt_phi_bwd", st);
        k_phi_bwd<T, float><<<rg, NT, psm, st>>>(cp<T>(q), dphq, dq, rows, P);
    }
    {
        TraceScope trace_("simt_phi_bwd", st);
        k_phi_bwd<T, float><<<rg, NT, psm, st>>>(cp<T>(k), dphk, dk, rows, P);
    }
    return cudaGetLastError();
}

cudaError_t simt_attn_causal_bwd(const void* q, const void* k, const void* v, const void* out,
                                 const float* den, const void* dout, float* dq, float* dk,
                                 float* dv, int B, int H, int L, slay_dtype dt, const Params& P,
                                 float eps, void* ws, cudaStream_t st)
{
    if (dt == SLAY_F32)
        return attn_bwd_t<float>(q, k, v, out, den, dout, dq, dk, dv, B, H, L, P, eps, ws, st, false);
    return attn_bwd_t<__nv_bfloat16>(q, k, v, out, den, dout, dq, dk, dv, B, H, L, P, eps, ws, st,
                                     false);
}

cudaError_t simt_attn_bidir_bwd(const void* q, const void* k, const void* v, const void* out,
                                const float* den, const void* dout, float* dq, float* dk,
                                float* dv, int B, int H, int L, slay_dtype dt, const Params& P,
                                float eps, void* ws, cudaStream_t st)
{
    if (dt == SLAY_F32)
        return attn_bwd_t<float>(q, k, v, out, den, dout, dq, dk, dv, B, H, L, P, eps, ws, st, true);
    return attn_bwd_t<__nv_bfloat16>(q, k, v, out, den, dout, dq, dk, dv, B, H, L, P, eps, ws, st,
                                     true);
}

cudaError_t simt_attn_causal_bwd_state(const void* q, const void* k, const void* v,
                                       const void* out, const float* den, const void* dout,
                                       float* dq, float* dk, float* dv, int B, int H, int L,
                                       slay_dtype dt, const Params& P, float eps, void* ws,
                                       const BwdStateIO& sio, cudaStream_t st)
{
    if (dt == SLAY_F32)
        return attn_bwd_t<float>(q, k, v, out, den, dout, dq, dk, dv, B, H, L, P, eps, ws, st, false,
                                 &sio);
    return attn_bwd_t<__nv_bfloat16>(q, k, v, out, den, dout, dq, dk, dv, B, H, L, P, eps, ws, st,
                                     false, &sio);
}

// The piece's G = sum_i phi(q_i) [dn_i, delta_i] ([B,H,F,64] and [B,H,F] fp32): phi(q), the
// row statistics, then the G sums -- on tensor cores the running-sum kernel for G alone in
// its total form, else the chunk sums and a suffix scan whose final value is the total.
template <typename T>
static cudaError_t bwd_state_t(const void* q, const void* out, const float* den, const void* dout,
                               float* g_out, float* zg_out, int B, int H, int L, const Params& P,
                               float eps, void* ws, cudaStream_t st)
{
    const int BH = B * H, F = P.F, NC = nchunks(L);
    const int64_t rows = static_cast<int64_t>(BH) * L;
    const size_t phb = align256(rows * F * sizeof(float));
    const size_t stb = align256(static_cast<size_t>(BH) * NC * F * E * sizeof(float));
    char* w = static_cast<char*>(ws);
    T* phq = reinterpret_cast<T*>(w);
    float* gbw = reinterpret_cast<float*>(w + 4 * phb + stb);
    float* dn = reinterpret_cast<float*>(w + 4 * phb + 2 * stb);
    cudaError_t err;
    if ((err = phi_map<T>(q, phq, rows, P, st)) != cudaSuccess) return err;
    const bool tcb = std::is_same<T, __nv_bfloat16>::value && tc_bwd_tile_supported(F, L);
    __nv_bfloat16* dn16 = reinterpret_cast<__nv_bfloat16*>(dn);
    float* delta = reinterpret_cast<float*>(dn16 + rows * kD);
    {
        TraceScope trace_("simt_bwd_rowstats", st);
        if (tcb)
            k_bwd_rowstats_tc<<<static_cast<unsigned>((rows + 31) / 32), 256, 0, st>>>(
                reinterpret_cast<const __nv_bfloat16*>(out), den,
                reinterpret_cast<const __nv_bfloat16*>(dout), dn16, delta, rows, eps);
        else
            k_bwd_rowstats<T><<<static_cast<unsigned>((rows + 7) / 8), 256, 0, st>>>(
                cp<T>(out), den, cp<T>(dout), dn, rows, eps);
    }
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    if (tcb) {
        BwdSeeds only_g;
        only_g.sums = 2;
        only_g.g_out = g_out;
        only_g.zg_out = zg_out;
        int* status = reinterpret_cast<int*>(w - kWsHeader);
        // (the S-side operands are placeholders of the right shapes: no S CTA runs)
        return tc_bwd_sums(phq, phq, dn16, dn16, delta, nullptr, nullptr, nullptr, nullptr, BH, L,
                           F, true, status, st, &only_g);
    }
    const dim3 sg((F + C - 1) / C, NC, BH);
    {
        TraceScope trace_("simt_chunk_state", st);
        k_chunk_state<float, T><<<sg, NT, 0, st>>>(phq, dn, E, gbw, L, F);
    }
    const int64_t nth = static_cast<int64_t>(BH) * F * E;
    {
        TraceScope trace_("simt_scan", st);
        k_scan_state<<<static_cast<unsigned>((nth + 255) / 256), 256, 0, st>>>(
            gbw, BH, NC, F, nullptr, nullptr, g_out, zg_out, 1);
    }
    return cudaGetLastError();
}

cudaError_t simt_causal_bwd_state(const void* q, const void* out, const float* den,
                                  const void* dout, float* g_out, float* zg_out, int B, int H,
                                  int L, slay_dtype dt, const Params& P, float eps, void* ws,
                                  cudaStream_t st)
{
    if (dt == SLAY_F32)
        return bwd_state_t<float>(q, out, den, dout, g_out, zg_out, B, H, L, P, eps, ws, st);
    return bwd_state_t<__nv_bfloat16>(q, out, den, dout, g_out, zg_out, B, H, L, P, eps, ws, st);
}

template <typename Tin, typename TG>
static cudaError_t phi_bwd_launch(const void* x, const void* dphi, float* dx, int64_t n,
                                  const Params& P, cudaStream_t st)
{
    const size_t psm = sizeof(PhiBwdSmem);
    cudaError_t err = cudaFuncSetAttribute(k_phi_bwd<Tin, TG>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(psm));
    if (err != cudaSuccess) return err;
    TraceScope trace_("simt_phi_bwd", st);
    k_phi_bwd<Tin, TG><<<static_cast<unsigned>((n + C - 1) / C), NT, psm, st>>>(
        cp<Tin>(x), cp<TG>(dphi), dx, n, P);
    return cudaGetLastError();
}

cudaError_t simt_feature_map_bwd(const void* x, const void* dphi, float* dx, int64_t n,
                                 slay_dtype x_dt, slay_dtype dphi_dt, const Params& P,
                                 cudaStream_t st)
{
    // bf16 rows and bf16 dphi: the tensor-core kernel where it takes the sizes
    if (x_dt == SLAY_BF16 && dphi_dt == SLAY_BF16 && P.wB && tc_phi_bwd_supported(kD, P.R, P.m, n))
        return tc_phi_bwd(x, dphi, dx, n, P, st);
    if (x_dt == SLAY_F32)
        return dphi_dt == SLAY_F32 ? phi_bwd_launch<float, float>(x, dphi, dx, n, P, st)
                                   : phi_bwd_launch<float, __nv_bfloat16>(x, dphi, dx, n, P, st);
    return dphi_dt == SLAY_F32 ? phi_bwd_launch<__nv_bfloat16, float>(x, dphi, dx, n, P, st)
                               : phi_bwd_launch<__nv_bfloat16, __nv_bfloat16>(x, dphi, dx, n, P, st);
}

template <typename T>
static cudaError_t decode_t(const void* q, const void* k, const void* v, float* S, float* z,
                            void* out, int N, const Params& P, float eps, cudaStream_t st)
{
    const size_t smem = static_cast<size_t>(2 * G) * P.F * sizeof(float);
    cudaError_t err;
    if ((err = cudaFuncSetAttribute(k_decode<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>(smem))) != cudaSuccess)
        return err;
    {
        // one wave of resident blocks looping over the groups (no partial last wave)
        int per_sm = 0, sms = 0, dev = 0;
        if ((err = cudaGetDevice(&dev)) != cudaSuccess ||
            (err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
            (err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_decode<T>, NT, smem)) != cudaSuccess)
            return err;
        const int groups = (N + G - 1) / G;
        const int grid = std::max(1, std::min(groups, std::max(1, per_sm) * sms));
        TraceScope trace_("simt_decode", st);
        k_decode<T><<<grid, NT, smem, st>>>(cp<T>(q), cp<T>(k), cp<T>(v), S, z, mp<T>(out), N, P, eps);
    }
    return cudaGetLastError();
}

cudaError_t simt_decode_step(const void* q, const void* k, const void* v, float* S, float* z,
                             void* out, int N, slay_dtype dt, const Params& P, float eps,
                             cudaStream_t st)
{
    if (dt == SLAY_F32) return decode_t<float>(q, k, v, S, z, out, N, P, eps, st);
    return decode_t<__nv_bfloat16>(q, k, v, S, z, out, N, P, eps, st);
}

}  // namespace slay
