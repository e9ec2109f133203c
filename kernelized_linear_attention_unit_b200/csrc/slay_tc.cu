// slay_tc.cu -- tensor-core path (tcgen05 / TMEM / TMA, sm_100a) for bf16 inputs.
//
// Method: "SLAY: Geometry-Aware Spherical Linearized Attention with Yat-Kernel" (abstract;
// nubint.ai review, "Proposed method", steps 1-6).  The causal forward computes, per
// (b,h) sequence, out_i = phi(q_i)^T S_i / (phi(q_i)^T z_i + eps) with
// S_i = sum_{j<=i} phi(k_j) v_j^T, z_i = sum_{j<=i} phi(k_j), in 128-token tiles:
//
//   U   = X W_t^T                   projection of a 64-feature slice t (omega and anchor
//                                   rows of W_t), raw bf16 x; the 1/|x| scale is applied in
//                                   the epilogue, phi = exp2(a2 u/|x| + b2) (p/|x|)^2
//   P  += phiQ_t phiK_t^T           intra-tile scores, summed over feature slices
//   O  += phiQ_t S_t                inter-tile readout with the state entering the tile
//   O  += tril(P) V                 masked intra-tile term
//   S  += phiK^T V,  z += phiK^T 1  state update (fp32 in tensor memory)
//
// Sequences are split into L-segments so that every SM has work: a first kernel computes
// each segment's own sum of phi(k) [v, 1]^T, the second starts each segment from the sum
// of the earlier segments' contributions and produces the outputs.  Neither kernel waits on
// another CTA.  Every mbarrier wait is bounded in time; a timeout sets an error word in the
// workspace header and the kernel leaves after its in-flight copies have landed.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>

#include "slay_tc.h"
#include "slay_tc_ptx.cuh"

namespace slay {

using namespace tc;

namespace {

constexpr int kTile = 128;             // tokens per tile (MMA M)
constexpr int kSlice = 64;             // features per projection slice
constexpr int kTileBytes = kTile * 128;  // one [128 rows][64 bf16] swizzled tile = 16 KiB
constexpr int kThreads = 128;
constexpr size_t kWsHeader = 256;      // error word + padding at the start of the workspace
constexpr int kNumSMs = 148;

// TMEM column map (one CTA per SM, 512 columns allocated).
constexpr uint32_t kColU = 0;     // 128: projection of one slice (64 u | 64 p)
constexpr uint32_t kColP = 128;   // 128: intra-tile scores
constexpr uint32_t kColO = 256;   // 64 : output numerator
constexpr uint32_t kColS = 320;   // 2 x 64: state S, feature halves
constexpr uint32_t kColZ = 448;   // 2 x 16: state z (column 0 of each half is read)
constexpr uint32_t kColSA = 128;  // state kernel: S at 128.., z at 256..
constexpr uint32_t kColZA = 256;

enum { BAR_QK = 0, BAR_V = 1, BAR_W0 = 2, BAR_W1 = 3, BAR_MMA = 4, NUM_BARS = 8 };

struct SmemOut {
    uint32_t w, q, k, v, phik, phiq, sbf, ones, z, bar, tmem, total;
};

__host__ __device__ inline SmemOut smem_out_layout(int F)
{
    SmemOut s;
    s.w = 0;
    s.q = 2 * kTileBytes;
    s.k = s.q + kTileBytes;
    s.v = s.k + kTileBytes;
    s.phik = s.v + kTileBytes;
    s.phiq = s.phik + (F / kSlice) * kTileBytes;
    s.sbf = s.phiq + kTileBytes;
    s.ones = s.sbf + F * 128;
    s.z = s.ones + 4096;
    s.bar = s.z + F * 4;
    s.tmem = s.bar + NUM_BARS * 8;
    s.total = s.tmem + 16;
    return s;
}

struct SmemState {
    uint32_t w, k, v, phik, ones, bar, tmem, total;
};

__host__ __device__ inline SmemState smem_state_layout(int F)
{
    SmemState s;
    s.w = 0;
    s.k = 2 * kTileBytes;
    s.v = s.k + kTileBytes;
    s.phik = s.v + kTileBytes;
    s.ones = s.phik + (F / kSlice) * kTileBytes;
    s.bar = s.ones + 4096;
    s.tmem = s.bar + NUM_BARS * 8;
    s.total = s.tmem + 16;
    return s;
}

struct Seg {
    int bh, seg, t_begin, t_end;
};

__device__ __forceinline__ Seg segment_of(int block, int nseg, int ntiles)
{
    Seg s;
    s.bh = block / nseg;
    s.seg = block % nseg;
    s.t_begin = static_cast<int>((static_cast<int64_t>(s.seg) * ntiles) / nseg);
    s.t_end = static_cast<int>((static_cast<int64_t>(s.seg + 1) * ntiles) / nseg);
    return s;
}

// Sum of squares of one 64-element bf16 row (128 bytes; order does not matter, so the
// swizzle is irrelevant) -> (1/|x|, 2 log2(1/|x|)) with the 1e-12 norm guard.
__device__ __forceinline__ void row_scale(const unsigned char* row, float& inv, float& l2inv2)
{
    const uint4* p = reinterpret_cast<const uint4*>(row);
    float s = 0.0f;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const uint4 w = p[c];
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float lo = __uint_as_float(ws[e] << 16);
            const float hi = __uint_as_float(ws[e] & 0xFFFF0000u);
            s = fmaf(lo, lo, s);
            s = fmaf(hi, hi, s);
        }
    }
    const float n = fmaxf(sqrtf(s), 1e-12f);
    inv = 1.0f / n;
    l2inv2 = -2.0f * __log2f(n);
}

// Epilogue of one projection slice: TMEM columns [colU, colU+64) hold u, [colU+64, +128)
// hold p for this thread's row.  phi_j = exp2(a u_j + b) p_j^2 with a = a2[r]/|x| and
// b = b2[r] + 2 log2(1/|x|).  Writes the 64 bf16 values as row `row` of a 128-byte-swizzled
// K-major tile at `tile_addr`; if zs != nullptr also returns sum_j phi_j zs[j].
__device__ __forceinline__ float phi_slice_epilogue(uint32_t taddr_row, float a, float b,
                                                    uint32_t tile_addr, uint32_t row,
                                                    const float* zs)
{
    float dz = 0.0f;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
        uint32_t ur[32], pr[32];
        tmem_ld32(taddr_row + kColU + 32 * c, ur);
        tmem_ld32(taddr_row + kColU + 64 + 32 * c, pr);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
            const float u0 = __uint_as_float(ur[j]), u1 = __uint_as_float(ur[j + 1]);
            const float p0 = __uint_as_float(pr[j]), p1 = __uint_as_float(pr[j + 1]);
            const float f0 = ex2(fmaf(a, u0, b)) * p0 * p0;
            const float f1 = ex2(fmaf(a, u1, b)) * p1 * p1;
            if (zs) {
                dz = fmaf(f0, zs[32 * c + j], dz);
                dz = fmaf(f1, zs[32 * c + j + 1], dz);
            }
            pk[j >> 1] = pack_bf16(f0, f1);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q)
            st_shared_v4(tile_addr + sw128_off(row, 4 * c + q), pk[4 * q], pk[4 * q + 1],
                         pk[4 * q + 2], pk[4 * q + 3]);
    }
    return dz;
}

// After a timed-out wait: give copies and MMAs still in flight time to land (bounded)
// before the CTA releases its shared and tensor memory.
__device__ __forceinline__ void drain_after_failure(bool ok)
{
    if (ok) return;
    const uint64_t t0 = global_timer_ns();
    while (global_timer_ns() - t0 < 20000000ull) {
    }
}

struct KParams {
    int L, F, m, nseg, ntiles;
    float eps;
    float a2[kMaxR];
    float b2[kMaxR];
};

__device__ __forceinline__ void issue_projection(uint32_t tmem, uint32_t x_addr, uint32_t w_addr)
{
    constexpr uint32_t id = idesc_bf16(128, 128, 0, 0);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
        umma_bf16(tmem + kColU, sdesc(x_addr + 32 * kk, 16, 1024, kLayoutSW128),
                  sdesc(w_addr + 32 * kk, 16, 1024, kLayoutSW128), id, kk > 0 ? 1u : 0u);
}

// S_h (+)= phiK_h^T V and z_h (+)= phiK_h^T 1 for feature halves h (phiK as an MN-major
// A operand: 128 features = two 64-feature sub-tiles 16 KiB apart).
__device__ __forceinline__ void issue_state_update(uint32_t tmem, uint32_t colS, uint32_t colZ,
                                                   uint32_t phik, uint32_t vaddr, uint32_t ones,
                                                   int halves, bool first)
{
    constexpr uint32_t idS = idesc_bf16(128, 64, 1, 1);
    constexpr uint32_t idZ = idesc_bf16(128, 16, 1, 0);
    for (int h = 0; h < halves; ++h) {
        const uint32_t a0 = phik + 2 * h * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const uint64_t ad = sdesc(a0 + 2048 * kk, kTileBytes, 1024, kLayoutSW128);
            const uint32_t acc = (first && kk == 0) ? 0u : 1u;
            umma_bf16(tmem + colS + 64 * h, ad, sdesc(vaddr + 2048 * kk, kTileBytes, 1024, kLayoutSW128),
                      idS, acc);
            umma_bf16(tmem + colZ + 16 * h, ad, sdesc(ones + 256 * kk, 128, 256, kLayoutNone), idZ,
                      acc);
        }
    }
}

__device__ __forceinline__ void fill_ones(unsigned char* ones)
{
    uint32_t* p = reinterpret_cast<uint32_t*>(ones);
    for (int i = threadIdx.x; i < 1024; i += blockDim.x) p[i] = 0x3F803F80u;  // bf16 1.0 pairs
}

// ------------------------------------------------------------ state kernel
// grid = BH * (nseg - 1): segment seg of sequence bh writes
//   ws_S[bh][seg][f][e] = sum_{t in seg} phi(k_t)_f v_t[e],  ws_z[bh][seg][f] = sum phi(k_t)_f
__global__ void __launch_bounds__(kThreads, 1)
k_tc_causal_state(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                  const __grid_constant__ CUtensorMap tmw, KParams kp, float* __restrict__ wsS,
                  float* __restrict__ wsZ, int* __restrict__ err)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const SmemState L = smem_state_layout(kp.F);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + L.bar);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + L.tmem);
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int NT = kp.F / kSlice, halves = kp.F / 128;
    // the last segment's sum is never needed
    const Seg sg = segment_of(blockIdx.x + blockIdx.x / (kp.nseg - 1), kp.nseg, kp.ntiles);

    if (warp == 0) {
        tmem_alloc(tslot, 512);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < NUM_BARS; ++i) mbar_init(&bar[i], 1);
        mbar_fence_init();
        tma_prefetch_desc(&tmk);
        tma_prefetch_desc(&tmv);
        tma_prefetch_desc(&tmw);
    }
    fill_ones(sm + L.ones);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    const uint32_t trow = tmem + ((32u * warp) << 16);

    auto load_kv = [&](int tile) {
        mbar_arrive_expect_tx(&bar[BAR_QK], 2 * kTileBytes);
        tma_load_3d(sm + L.k, &tmk, &bar[BAR_QK], 0, tile * kTile, sg.bh);
        tma_load_3d(sm + L.v, &tmv, &bar[BAR_QK], 0, tile * kTile, sg.bh);
    };
    auto load_w = [&](int slice, int slot) {
        mbar_arrive_expect_tx(&bar[BAR_W0 + slot], kTileBytes);
        tma_load_2d(sm + L.w + slot * kTileBytes, &tmw, &bar[BAR_W0 + slot], 0, slice * 128);
    };
    if (tid == 0) {
        load_kv(sg.t_begin);
        for (int s = 0; s < 2 && s < NT; ++s) load_w(s, s);
    }
    bool ok = true;
    uint32_t ph_kv = 0, ph_w0 = 0, ph_w1 = 0, ph_mma = 0;
    for (int tile = sg.t_begin; tile < sg.t_end; ++tile) {
        ok = mbar_wait(&bar[BAR_QK], ph_kv, ok ? 2000000000ull : 0) && ok;
        ph_kv ^= 1;
        float inv, l2i;
        row_scale(sm + L.k + tid * 128, inv, l2i);
        for (int t = 0; t < NT; ++t) {
            const int slot = t & 1;
            ok = mbar_wait(&bar[BAR_W0 + slot], slot ? ph_w1 : ph_w0, ok ? 2000000000ull : 0) && ok;
            if (slot) ph_w1 ^= 1; else ph_w0 ^= 1;
            if (tid == 0) {
                tc_fence_after();
                issue_projection(tmem, sbase + L.k, sbase + L.w + slot * kTileBytes);
                umma_commit(&bar[BAR_MMA]);
            }
            ok = mbar_wait(&bar[BAR_MMA], ph_mma, ok ? 2000000000ull : 0) && ok;
            ph_mma ^= 1;
            tc_fence_after();
            const int node = (t * kSlice) / kp.m;
            phi_slice_epilogue(trow, kp.a2[node] * inv, kp.b2[node] + l2i,
                               sbase + L.phik + t * kTileBytes, tid, nullptr);
            fence_async_smem();
            tc_fence_before();
            __syncthreads();
            if (tid == 0 && t + 2 < NT) load_w(t + 2, slot);
        }
        if (tid == 0) {
            tc_fence_after();
            issue_state_update(tmem, kColSA, kColZA, sbase + L.phik, sbase + L.v, sbase + L.ones,
                               halves, tile == sg.t_begin);
            umma_commit(&bar[BAR_MMA]);
        }
        ok = mbar_wait(&bar[BAR_MMA], ph_mma, ok ? 2000000000ull : 0) && ok;
        ph_mma ^= 1;
        tc_fence_after();
        if (tid == 0 && tile + 1 < sg.t_end) {
            load_kv(tile + 1);
            for (int s = 0; s < 2 && s < NT; ++s) load_w(s, s);
        }
    }
    // write the segment sums: thread = TMEM lane = feature within a half
    const size_t segidx = static_cast<size_t>(sg.bh) * kp.nseg + sg.seg;
    for (int h = 0; h < halves; ++h) {
        const int f = 128 * h + tid;
        uint32_t r0[32], r1[32], zr;
        tmem_ld32(trow + kColSA + 64 * h, r0);
        tmem_ld32(trow + kColSA + 64 * h + 32, r1);
        tmem_ld1(trow + kColZA + 16 * h, zr);
        tmem_wait_ld();
        float4* dst = reinterpret_cast<float4*>(wsS + (segidx * kp.F + f) * 64);
#pragma unroll
        for (int q = 0; q < 8; ++q)
            dst[q] = make_float4(__uint_as_float(r0[4 * q]), __uint_as_float(r0[4 * q + 1]),
                                 __uint_as_float(r0[4 * q + 2]), __uint_as_float(r0[4 * q + 3]));
#pragma unroll
        for (int q = 0; q < 8; ++q)
            dst[8 + q] = make_float4(__uint_as_float(r1[4 * q]), __uint_as_float(r1[4 * q + 1]),
                                     __uint_as_float(r1[4 * q + 2]), __uint_as_float(r1[4 * q + 3]));
        wsZ[segidx * kp.F + f] = __uint_as_float(zr);
    }
    if (!ok) atomicExch(err, 1);
    drain_after_failure(ok);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

// ----------------------------------------------------------- output kernel
// grid = BH * nseg.  One CTA walks the tiles of one segment with the state entering it.
__global__ void __launch_bounds__(kThreads, 1)
k_tc_causal_out(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmw,
                KParams kp, const float* __restrict__ wsS, const float* __restrict__ wsZ,
                __nv_bfloat16* __restrict__ out, float* __restrict__ den, int* __restrict__ err)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const SmemOut L = smem_out_layout(kp.F);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + L.bar);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + L.tmem);
    float* zs = reinterpret_cast<float*>(sm + L.z);
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int NT = kp.F / kSlice, halves = kp.F / 128;
    const Seg sg = segment_of(blockIdx.x, kp.nseg, kp.ntiles);

    if (warp == 0) {
        tmem_alloc(tslot, 512);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < NUM_BARS; ++i) mbar_init(&bar[i], 1);
        mbar_fence_init();
        tma_prefetch_desc(&tmq);
        tma_prefetch_desc(&tmk);
        tma_prefetch_desc(&tmv);
        tma_prefetch_desc(&tmw);
    }
    fill_ones(sm + L.ones);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    const uint32_t trow = tmem + ((32u * warp) << 16);

    auto load_qkv = [&](int tile) {
        mbar_arrive_expect_tx(&bar[BAR_QK], 2 * kTileBytes);
        tma_load_3d(sm + L.q, &tmq, &bar[BAR_QK], 0, tile * kTile, sg.bh);
        tma_load_3d(sm + L.k, &tmk, &bar[BAR_QK], 0, tile * kTile, sg.bh);
        mbar_arrive_expect_tx(&bar[BAR_V], kTileBytes);
        tma_load_3d(sm + L.v, &tmv, &bar[BAR_V], 0, tile * kTile, sg.bh);
    };
    auto load_w = [&](int slice, int slot) {
        mbar_arrive_expect_tx(&bar[BAR_W0 + slot], kTileBytes);
        tma_load_2d(sm + L.w + slot * kTileBytes, &tmw, &bar[BAR_W0 + slot], 0, slice * 128);
    };
    if (tid == 0) {
        load_qkv(sg.t_begin);
        for (int s = 0; s < 2 && s < NT; ++s) load_w(s, s);
    }

    // state entering the segment: sum of the earlier segments' contributions
    for (int h = 0; h < halves; ++h) {
        const int f = 128 * h + tid;
        float acc[64];
#pragma unroll
        for (int e = 0; e < 64; ++e) acc[e] = 0.0f;
        float zf = 0.0f;
        for (int s = 0; s < sg.seg; ++s) {
            const size_t segidx = static_cast<size_t>(sg.bh) * kp.nseg + s;
            const float4* src = reinterpret_cast<const float4*>(wsS + (segidx * kp.F + f) * 64);
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                const float4 x = src[q];
                acc[4 * q] += x.x; acc[4 * q + 1] += x.y; acc[4 * q + 2] += x.z; acc[4 * q + 3] += x.w;
            }
            zf += wsZ[segidx * kp.F + f];
        }
        uint32_t r[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(acc[e]);
        tmem_st32(trow + kColS + 64 * h, r);
#pragma unroll
        for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(acc[32 + e]);
        tmem_st32(trow + kColS + 64 * h + 32, r);
#pragma unroll
        for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(e == 0 ? zf : 0.0f);
        tmem_st32(trow + kColZ + 16 * h, r);  // columns z_h .. z_h+31 (z_{h+1} is rewritten next)
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) pk[e] = pack_bf16(acc[2 * e], acc[2 * e + 1]);
#pragma unroll
        for (int q = 0; q < 8; ++q)
            st_shared_v4(sbase + L.sbf + sw128_off(f, q), pk[4 * q], pk[4 * q + 1], pk[4 * q + 2],
                         pk[4 * q + 3]);
        zs[f] = zf;
    }
    tmem_wait_st();
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    bool ok = true;
    uint32_t ph_qk = 0, ph_v = 0, ph_w0 = 0, ph_w1 = 0, ph_mma = 0;
    const int64_t rowbase = static_cast<int64_t>(sg.bh) * kp.L;
    for (int tile = sg.t_begin; tile < sg.t_end; ++tile) {
        ok = mbar_wait(&bar[BAR_QK], ph_qk, ok ? 2000000000ull : 0) && ok;
        ph_qk ^= 1;
        float invq, l2q, invk, l2k;
        row_scale(sm + L.q + tid * 128, invq, l2q);
        row_scale(sm + L.k + tid * 128, invk, l2k);
        float den_inter = 0.0f;
        for (int t = 0; t < NT; ++t) {
            const int slot = t & 1;
            const uint32_t waddr = sbase + L.w + slot * kTileBytes;
            ok = mbar_wait(&bar[BAR_W0 + slot], slot ? ph_w1 : ph_w0, ok ? 2000000000ull : 0) && ok;
            if (slot) ph_w1 ^= 1; else ph_w0 ^= 1;
            const int node = (t * kSlice) / kp.m;
            // q projection -> phiQ_t
            if (tid == 0) {
                tc_fence_after();
                issue_projection(tmem, sbase + L.q, waddr);
                umma_commit(&bar[BAR_MMA]);
            }
            ok = mbar_wait(&bar[BAR_MMA], ph_mma, ok ? 2000000000ull : 0) && ok;
            ph_mma ^= 1;
            tc_fence_after();
            den_inter += phi_slice_epilogue(trow, kp.a2[node] * invq, kp.b2[node] + l2q,
                                            sbase + L.phiq, tid, zs + t * kSlice);
            fence_async_smem();
            tc_fence_before();
            __syncthreads();
            // k projection -> phiK_t
            if (tid == 0) {
                tc_fence_after();
                issue_projection(tmem, sbase + L.k, waddr);
                umma_commit(&bar[BAR_MMA]);
            }
            ok = mbar_wait(&bar[BAR_MMA], ph_mma, ok ? 2000000000ull : 0) && ok;
            ph_mma ^= 1;
            tc_fence_after();
            phi_slice_epilogue(trow, kp.a2[node] * invk, kp.b2[node] + l2k,
                               sbase + L.phik + t * kTileBytes, tid, nullptr);
            fence_async_smem();
            tc_fence_before();
            __syncthreads();
            // P += phiQ_t phiK_t^T ; O += phiQ_t S_t
            if (tid == 0) {
                tc_fence_after();
                constexpr uint32_t idP = idesc_bf16(128, 128, 0, 0);
                constexpr uint32_t idO = idesc_bf16(128, 64, 0, 1);
                const uint32_t aq = sbase + L.phiq;
                const uint32_t bk = sbase + L.phik + t * kTileBytes;
                const uint32_t bs = sbase + L.sbf + t * kSlice * 128;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint32_t acc = (t > 0 || kk > 0) ? 1u : 0u;
                    const uint64_t ad = sdesc(aq + 32 * kk, 16, 1024, kLayoutSW128);
                    umma_bf16(tmem + kColP, ad, sdesc(bk + 32 * kk, 16, 1024, kLayoutSW128), idP, acc);
                    umma_bf16(tmem + kColO, ad, sdesc(bs + 2048 * kk, kTileBytes, 1024, kLayoutSW128),
                              idO, acc);
                }
                umma_commit(&bar[BAR_MMA]);
            }
            ok = mbar_wait(&bar[BAR_MMA], ph_mma, ok ? 2000000000ull : 0) && ok;
            ph_mma ^= 1;
            tc_fence_after();
            if (tid == 0 && t + 2 < NT) load_w(t + 2, slot);
        }
        // state update (asynchronous) while the masked scores are formed
        ok = mbar_wait(&bar[BAR_V], ph_v, ok ? 2000000000ull : 0) && ok;
        ph_v ^= 1;
        if (tid == 0) {
            tc_fence_after();
            issue_state_update(tmem, kColS, kColZ, sbase + L.phik, sbase + L.v, sbase + L.ones,
                               halves, false);
        }
        // P epilogue: mask j <= i, row sum, bf16 into the Q/K tile space (K-major, K = 128)
        float den_intra = 0.0f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            uint32_t pr[32];
            tmem_ld32(trow + kColP + 32 * c, pr);
            tmem_wait_ld();
            uint32_t pk[16];
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
                const int col = 32 * c + j;
                const float x0 = (col <= tid) ? __uint_as_float(pr[j]) : 0.0f;
                const float x1 = (col + 1 <= tid) ? __uint_as_float(pr[j + 1]) : 0.0f;
                den_intra += x0 + x1;
                pk[j >> 1] = pack_bf16(x0, x1);
            }
            const uint32_t base = sbase + ((c < 2) ? L.q : L.k);
#pragma unroll
            for (int q = 0; q < 4; ++q)
                st_shared_v4(base + sw128_off(tid, 4 * (c & 1) + q), pk[4 * q], pk[4 * q + 1],
                             pk[4 * q + 2], pk[4 * q + 3]);
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t idO = idesc_bf16(128, 64, 0, 1);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t a = sbase + ((kk < 4) ? L.q : L.k) + 32 * (kk & 3);
                umma_bf16(tmem + kColO, sdesc(a, 16, 1024, kLayoutSW128),
                          sdesc(sbase + L.v + 2048 * kk, kTileBytes, 1024, kLayoutSW128), idO, 1u);
            }
            umma_commit(&bar[BAR_MMA]);
        }
        ok = mbar_wait(&bar[BAR_MMA], ph_mma, ok ? 2000000000ull : 0) && ok;
        ph_mma ^= 1;
        tc_fence_after();
        if (tid == 0 && tile + 1 < sg.t_end) {
            load_qkv(tile + 1);
            for (int s = 0; s < 2 && s < NT; ++s) load_w(s, s);
        }
        // output epilogue
        {
            uint32_t o0[32], o1[32];
            tmem_ld32(trow + kColO, o0);
            tmem_ld32(trow + kColO + 32, o1);
            tmem_wait_ld();
            const float d = den_intra + den_inter;
            const float rz = 1.0f / (d + kp.eps);
            const int row = tile * kTile + tid;
            if (row < kp.L) {
                uint4* dst = reinterpret_cast<uint4*>(out + (rowbase + row) * 64);
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    dst[q] = make_uint4(pack_bf16(__uint_as_float(o0[8 * q]) * rz, __uint_as_float(o0[8 * q + 1]) * rz),
                                        pack_bf16(__uint_as_float(o0[8 * q + 2]) * rz, __uint_as_float(o0[8 * q + 3]) * rz),
                                        pack_bf16(__uint_as_float(o0[8 * q + 4]) * rz, __uint_as_float(o0[8 * q + 5]) * rz),
                                        pack_bf16(__uint_as_float(o0[8 * q + 6]) * rz, __uint_as_float(o0[8 * q + 7]) * rz));
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    dst[4 + q] = make_uint4(pack_bf16(__uint_as_float(o1[8 * q]) * rz, __uint_as_float(o1[8 * q + 1]) * rz),
                                            pack_bf16(__uint_as_float(o1[8 * q + 2]) * rz, __uint_as_float(o1[8 * q + 3]) * rz),
                                            pack_bf16(__uint_as_float(o1[8 * q + 4]) * rz, __uint_as_float(o1[8 * q + 5]) * rz),
                                            pack_bf16(__uint_as_float(o1[8 * q + 6]) * rz, __uint_as_float(o1[8 * q + 7]) * rz));
                if (den) den[rowbase + row] = d;
            }
        }
        // state after the tile -> bf16 operand copy and fp32 z
        if (tile + 1 < sg.t_end) {
            for (int h = 0; h < halves; ++h) {
                const int f = 128 * h + tid;
                uint32_t r0[32], r1[32], zr;
                tmem_ld32(trow + kColS + 64 * h, r0);
                tmem_ld32(trow + kColS + 64 * h + 32, r1);
                tmem_ld1(trow + kColZ + 16 * h, zr);
                tmem_wait_ld();
                uint32_t pk[32];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    pk[e] = pack_bf16(__uint_as_float(r0[2 * e]), __uint_as_float(r0[2 * e + 1]));
                    pk[16 + e] = pack_bf16(__uint_as_float(r1[2 * e]), __uint_as_float(r1[2 * e + 1]));
                }
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    st_shared_v4(sbase + L.sbf + sw128_off(f, q), pk[4 * q], pk[4 * q + 1],
                                 pk[4 * q + 2], pk[4 * q + 3]);
                zs[f] = __uint_as_float(zr);
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    if (!ok) atomicExch(err, 1);
    drain_after_failure(ok);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------ host side

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// [BH][L][64] bf16 viewed as a 3-D tensor, 128-token x 64 boxes, 128-byte swizzle;
// rows past L read as zero.
bool map_rows(CUtensorMap* m, const void* base, int L, int BH)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(L), static_cast<cuuint64_t>(BH)};
    const cuuint64_t strides[2] = {128, static_cast<cuuint64_t>(L) * 128};
    const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(kTile), 1};
    const cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
              es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// packed projection operand [F/64][128][64] bf16: per 64-feature slice, 64 omega rows then
// 64 anchor rows, each row the 64 input dimensions.
bool map_w(CUtensorMap* m, const void* base, int F)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {64, static_cast<cuuint64_t>(F / kSlice) * 128};
    const cuuint64_t strides[1] = {128};
    const cuuint32_t box[2] = {64, 128};
    const cuuint32_t es[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
              es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int choose_nseg(int BH, int ntiles)
{
    if (BH >= kNumSMs) return 1;
    return std::max(1, std::min(ntiles, kNumSMs / BH));
}

size_t smem_bytes_out(int F) { return smem_out_layout(F).total + 1024; }
size_t smem_bytes_state(int F) { return smem_state_layout(F).total + 1024; }

}  // namespace

bool tc_supported(slay_op op, int B, int H, int L, int R, int m)
{
    const int F = R * m;
    if (op != SLAY_OP_CAUSAL_FWD) return false;
    if (m % kSlice != 0 || F % 128 != 0 || F > 256) return false;
    if (static_cast<int64_t>(B) * H * L <= 0) return false;
    return smem_bytes_out(F) <= 232448;
}

size_t tc_workspace_bytes(slay_op op, int B, int H, int L, int R, int m)
{
    if (op != SLAY_OP_CAUSAL_FWD) return 0;
    const int F = R * m;
    const int BH = B * H;
    const int ntiles = (L + kTile - 1) / kTile;
    const int nseg = choose_nseg(BH, ntiles);
    const size_t per = static_cast<size_t>(BH) * nseg * F;
    return kWsHeader + ((per * 64 * sizeof(float) + 255) & ~size_t(255)) + per * sizeof(float);
}

size_t tc_wb_elems(int D, int R, int m)
{
    const int F = R * m;
    if (D != 64 || F % kSlice != 0) return 0;
    return static_cast<size_t>(F) * 2 * D;
}

void tc_pack_wb(int D, int R, int m, const uint16_t* om, const uint16_t* an, uint16_t* wb)
{
    const int F = R * m;
    for (int t = 0; t < F / kSlice; ++t)
        for (int r = 0; r < 128; ++r) {
            const int f = t * kSlice + (r & 63);
            const uint16_t* src = (r < 64) ? om : an;
            std::memcpy(wb + (static_cast<size_t>(t) * 128 + r) * D, src + static_cast<size_t>(f) * D,
                        D * sizeof(uint16_t));
        }
}

cudaError_t tc_feature_map(const void*, void*, int64_t, const Params&, cudaStream_t)
{
    return cudaErrorNotSupported;
}

cudaError_t tc_attn_fwd(const void* q, const void* k, const void* v, void* out, float* den, int B,
                        int H, int L, const Params& P, float eps, bool causal, void* ws,
                        cudaStream_t st)
{
    if (!causal || !P.wB) return cudaErrorNotSupported;
    const int BH = B * H, F = P.F;
    const int ntiles = (L + kTile - 1) / kTile;
    const int nseg = choose_nseg(BH, ntiles);
    CUtensorMap mq, mk, mv, mw;
    if (!map_rows(&mq, q, L, BH) || !map_rows(&mk, k, L, BH) || !map_rows(&mv, v, L, BH) ||
        !map_w(&mw, P.wB, F))
        return cudaErrorInvalidValue;
    KParams kp;
    kp.L = L; kp.F = F; kp.m = P.m; kp.nseg = nseg; kp.ntiles = ntiles; kp.eps = eps;
    for (int r = 0; r < kMaxR; ++r) { kp.a2[r] = P.a2[r]; kp.b2[r] = P.b2[r]; }
    char* w = static_cast<char*>(ws);
    int* err = reinterpret_cast<int*>(w);
    float* wsS = reinterpret_cast<float*>(w + kWsHeader);
    const size_t per = static_cast<size_t>(BH) * nseg * F;
    float* wsZ = reinterpret_cast<float*>(w + kWsHeader + ((per * 64 * sizeof(float) + 255) & ~size_t(255)));
    cudaError_t e = cudaMemsetAsync(err, 0, sizeof(int), st);
    if (e != cudaSuccess) return e;
    if (nseg > 1) {
        const size_t sm = smem_bytes_state(F);
        e = cudaFuncSetAttribute(k_tc_causal_state, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(sm));
        if (e != cudaSuccess) return e;
        TraceScope trace_("tc_causal_state", st);
        k_tc_causal_state<<<BH * (nseg - 1), kThreads, sm, st>>>(mk, mv, mw, kp, wsS, wsZ, err);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    const size_t sm = smem_bytes_out(F);
    e = cudaFuncSetAttribute(k_tc_causal_out, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(sm));
    if (e != cudaSuccess) return e;
    {
        TraceScope trace_("tc_causal_out", st);
        k_tc_causal_out<<<BH * nseg, kThreads, sm, st>>>(mq, mk, mv, mw, kp, wsS, wsZ,
                                                         static_cast<__nv_bfloat16*>(out), den, err);
    }
    return cudaGetLastError();
}

}  // namespace slay
