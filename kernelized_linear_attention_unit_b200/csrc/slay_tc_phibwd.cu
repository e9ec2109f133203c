// slay_tc_phibwd.cu -- tensor-core backward of the feature map: dx from dphi for bf16 rows.
//
// Method: "SLAY: Geometry-Aware Spherical Linearized Attention with Yat-Kernel" (nubint.ai
// review, "Proposed method", steps 1, 3, 4, 5) defines, per row x and feature f = r*m + j,
//   phi_f = c_r exp(sqrt(2 s_r) omega_f.x^ - s_r) (a_f.x^)^2,  x^ = x / |x|;
// the pages give no backward, so it is the chain rule of that definition.  With u = omega_f.x
// and p = a_f.x of the raw row, n = |x| and e = exp2(a2_r u/n + b2_r + 2 log2(1/n)) (so that
// phi = e p^2 and c_r exp(..) = e n^2):
//   dx^ = sum_f alpha_f omega_f + beta_f a_f,   t = dphi_f e p,
//   alpha_f = t p sqrt(2 s_r),  beta_f = 2 n t,
//   dx = (dx^ - x^ (x^ . dx^)) / n   (dx^ / 1e-12 below the norm guard |x| < 1e-12).
// Both contractions run on tensor cores: per 128-row tile and 64-feature group g (a job) the
// projections U = X W_g^T (N = 128: 64 omega and 64 anchor columns, as in the forward map),
// then dX^ += [alpha | beta]_g [Omega_g ; A_g] (K = 128, N = 64) with [alpha | beta] read from
// tensor memory and the same W tiles read as an MN-major shared-memory operand.  The kernel reads x (bf16), dphi (bf16, as the tensor-core
// contraction stores it) and writes dx (fp32): its DRAM traffic is dominated by the dphi
// reads (2F bytes per row).
//
// Persistent, one CTA per SM, 128-row tiles round-robin.  Warp 9 issues the TMA loads: X
// tiles, and per job the group's W operand (five slots, L2-resident) and the dphi tile
// [128 rows][64 features] (four slots: the dphi stream is the kernel's DRAM traffic, and the
// loads run up to four jobs ahead of the epilogue so that enough of it is in flight).  Warp 0
// issues the MMAs.  Warps 1-8 are the epilogue: warp w serves TMEM lanes 32 (w % 4).. (rows
// of the tile) and the 32-feature half (w - 1) / 4 of every group; per job it reads its rows'
// dphi from the shared-memory tile, its projections from tensor memory, and writes its block
// of [alpha | beta] back into tensor memory as the contraction's A operand (bf16 pairs, one
// row per lane); per tile, after the next tile's jobs, it turns dX^ into dx and stores its
// 32 x 32 block by TMA.  Every wait is bounded; a timeout sets the library's feature-map
// status word.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "slay_tc.h"
#include "slay_tc_common.cuh"
#include "slay_tc_ptx.cuh"

namespace slay {

using namespace tc;

namespace {

constexpr int kRows = 128;                  // rows per tile (MMA M)
constexpr int kBoxBytes = kRows * 128;      // [128 rows][64 bf16] swizzled X tile = 16 KiB
constexpr int kSubBytes = 64 * 128;         // packed W of 32 features = 8 KiB
constexpr int kGroupBytes = 2 * kSubBytes;  // 64 features = 16 KiB
constexpr int kEpiWarps = 8;
constexpr int kPbThreads = 32 * (2 + kEpiWarps);   // MMA warp, 8 epilogue warps, TMA warp
constexpr int kNumSMs = 148;
constexpr int kXBufs = 3;                   // X tiles in flight
constexpr int kRing = 5;                    // W groups in flight (slot = job % 5)
constexpr int kDRing = 4;                   // dphi tiles in flight (slot = job % 4)
constexpr int kStgBytes = 32 * 128;         // per epilogue warp: [32 rows][32 fp32] of dx
constexpr uint32_t kColU = 0;               // two 128-column projection buffers
constexpr uint32_t kColDX = 256;            // two 64-column dX^ accumulators
constexpr uint32_t kColA = 384;             // two 64-column [alpha | beta] operands (bf16 pairs)

enum {
    PB_XF = 0,                  // + slot (TMA: X tile)
    PB_XE = PB_XF + kXBufs,     // + slot (8 warp arrivals: dx of the tile written)
    PB_WF = PB_XE + kXBufs,     // + slot (TMA: W group)
    PB_WE = PB_WF + kRing,      // + slot (contraction MMA commit: the group's W free)
    PB_GF = PB_WE + kRing,      // + slot (TMA: dphi tile)
    PB_GE = PB_GF + kDRing,     // + slot (8 warp arrivals: dphi read)
    PB_UF = PB_GE + kDRing,     // + buffer (projection MMA commit)
    PB_AF = PB_UF + 2,          // + buffer (8 warp arrivals: [alpha | beta] in tensor memory)
    PB_AE = PB_AF + 2,          // + buffer (contraction MMA commit: operand free)
    PB_DF = PB_AE + 2,          // + buffer (dX^ of a tile complete)
    PB_DE = PB_DF + 2,          // + buffer (8 warp arrivals: dX^ read)
    PB_NUM = PB_DE + 2
};

struct PbLayout {
    uint32_t w, x, d, stg, bar, tmem, total;
};

__host__ __device__ inline PbLayout pb_layout(int /*F*/)
{
    PbLayout l;
    l.w = 0;                                // kRing W groups (16 KiB each)
    l.x = l.w + kRing * kGroupBytes;        // kXBufs X tiles
    l.d = l.x + kXBufs * kBoxBytes;         // kDRing dphi tiles [128 rows][64 features]
    l.stg = l.d + kDRing * kBoxBytes;       // kEpiWarps dx staging boxes (TMA stores)
    l.bar = l.stg + kEpiWarps * kStgBytes;
    l.tmem = l.bar + PB_NUM * 8;
    l.total = l.tmem + 16;
    return l;
}

struct PbParams {
    int F, ntiles;
    float a2[16];   // per 32-feature sub-slice: the scales of its node (F <= 512)
    float b2[16];
    float sq[16];   // sqrt(2 s_r)
};

// dphi value c = 0..31 of one row's 32-feature block held as four 16-byte words of bf16
__device__ __forceinline__ float dphi_val(const uint4 (&d)[4], int c)
{
    const uint4 w = d[c >> 3];
    const int k = (c >> 1) & 3;
    const uint32_t u = k == 0 ? w.x : k == 1 ? w.y : k == 2 ? w.z : w.w;
    return __uint_as_float((c & 1) ? (u & 0xFFFF0000u) : (u << 16));
}

// Slot and use count of a ring walked in order: the u-th use of slot s waits for phase u & 1
// of its full barrier and (u >= 1) phase (u - 1) & 1 of its empty barrier.
struct Ring {
    int slot = 0, use = 0, n;
    __device__ explicit Ring(int n_) : n(n_) {}
    __device__ void next()
    {
        if (++slot == n) {
            slot = 0;
            ++use;
        }
    }
};

__global__ void __launch_bounds__(kPbThreads, 1)
k_tc_phi_bwd(const __grid_constant__ CUtensorMap tmx, const __grid_constant__ CUtensorMap tmw,
             const __grid_constant__ CUtensorMap tmd, const __grid_constant__ CUtensorMap tmdx,
             PbParams pp, int* status)
{
    constexpr int kW = 4;     // 16-byte words per 32 bf16 dphi values
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* sm = aligned_smem(smem_raw);
    const PbLayout L = pb_layout(pp.F);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + L.bar);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + L.tmem);
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ng = pp.F / 64;

    if (warp == 0) {
        tmem_alloc(tslot, 512);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < PB_NUM; ++i) mbar_init(&bar[i], 1);
        for (int s = 0; s < kXBufs; ++s) mbar_init(&bar[PB_XE + s], kEpiWarps);
        for (int s = 0; s < kDRing; ++s) mbar_init(&bar[PB_GE + s], kEpiWarps);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bar[PB_AF + b], kEpiWarps);
            mbar_init(&bar[PB_DE + b], kEpiWarps);
        }
        mbar_fence_init();
        tma_prefetch_desc(&tmx);
        tma_prefetch_desc(&tmw);
        tma_prefetch_desc(&tmd);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem0 = *tslot;
    Waiter wt;
    const int nt = static_cast<int>(blockIdx.x) < pp.ntiles
                       ? (pp.ntiles - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1
                       : 0;
    const int njobs = nt * ng;   // job j = tile k (k-th of this CTA), group g: j = k ng + g
    auto row0_of = [&](int k) {
        return (k * static_cast<int>(gridDim.x) + static_cast<int>(blockIdx.x)) * kRows;
    };

    if (warp == 9) {
        // ---------------------------------------------------------------- TMA loads, in
        // job order: the X tile at each tile's first group (into the slot the tile kXBufs
        // before released), then per job its W group and its dphi tile (into the slots the
        // jobs kRing and kDRing before released)
        if (lane == 0) {
            Ring xr(kXBufs), rr(kRing), gr(kDRing);
            for (int j = 0, k = 0, g = 0; j < njobs && wt.ok; ++j) {
                if (g == 0) {
                    if (xr.use >= 1) {
                        uint32_t ph = static_cast<uint32_t>((xr.use - 1) & 1);
                        wt.wait(&bar[PB_XE + xr.slot], ph);
                    }
                    mbar_arrive_expect_tx(&bar[PB_XF + xr.slot], kBoxBytes);
                    tma_load_2d(sm + L.x + xr.slot * kBoxBytes, &tmx, &bar[PB_XF + xr.slot], 0, row0_of(k));
                    xr.next();
                }
                if (rr.use >= 1) {
                    uint32_t ph = static_cast<uint32_t>((rr.use - 1) & 1);
                    wt.wait(&bar[PB_WE + rr.slot], ph);
                }
                mbar_arrive_expect_tx(&bar[PB_WF + rr.slot], kGroupBytes);
                unsigned char* wd = sm + L.w + rr.slot * kGroupBytes;
                tma_load_2d(wd, &tmw, &bar[PB_WF + rr.slot], 0, (2 * g) * 64);
                tma_load_2d(wd + kSubBytes, &tmw, &bar[PB_WF + rr.slot], 0, (2 * g + 1) * 64);
                rr.next();
                if (gr.use >= 1) {
                    uint32_t ph = static_cast<uint32_t>((gr.use - 1) & 1);
                    wt.wait(&bar[PB_GE + gr.slot], ph);
                }
                mbar_arrive_expect_tx(&bar[PB_GF + gr.slot], kBoxBytes);
                tma_load_2d(sm + L.d + gr.slot * kBoxBytes, &tmd, &bar[PB_GF + gr.slot], 64 * g, row0_of(k));
                gr.next();
                if (++g == ng) {
                    g = 0;
                    ++k;
                }
            }
        }
        __syncwarp();
    } else if (warp == 0) {
        // ---------------------------------------------------------------- MMA issue
        if (lane == 0 && nt > 0) {
            constexpr uint32_t idU = idesc_bf16(128, 128, 0, 0);   // X (K-major) x W (K-major)
            constexpr uint32_t idD = idesc_bf16(128, 64, 0, 1);    // [alpha|beta] x W (MN-major)
            const uint64_t dx0 = sdesc(sbase + L.x, 16, 1024, kLayoutSW128);
            const uint64_t dw0 = sdesc(sbase + L.w, 16, 1024, kLayoutSW128);
            // projection job jp = (tile pk, group pg) from X slot px and W slot pw
            int jp = 0, pg = 0;
            Ring px(kXBufs), pw(kRing);
            auto proj = [&]() {   // U[jp & 1] = X_pk W_pg^T, then advance to the next job
                if (pg == 0) {
                    uint32_t ph = static_cast<uint32_t>(px.use & 1);
                    wt.wait(&bar[PB_XF + px.slot], ph);
                }
                {
                    uint32_t ph = static_cast<uint32_t>(pw.use & 1);
                    wt.wait(&bar[PB_WF + pw.slot], ph);
                }
                tc_fence_after();
                const uint64_t dx = dx0 + ((px.slot * kBoxBytes) >> 4);
                const uint64_t dw = dw0 + ((pw.slot * kGroupBytes) >> 4);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_bf16(tmem0 + kColU + 128u * (jp & 1), dx + 2 * kk, dw + 2 * kk, idU,
                              kk > 0 ? 1u : 0u);
                umma_commit(&bar[PB_UF + (jp & 1)]);
                ++jp;
                pw.next();
                if (++pg == ng) {
                    pg = 0;
                    px.next();
                }
            };
            proj();
            if (njobs > 1) proj();
            Ring cw(kRing);   // W slot of contraction job j
            for (int j = 0, k = 0, g = 0; j < njobs && wt.ok; ++j) {
                {
                    uint32_t ph = static_cast<uint32_t>((j >> 1) & 1);
                    wt.wait(&bar[PB_AF + (j & 1)], ph);   // [alpha|beta]_j written, U_j read
                }
                if (g == 0 && k >= 2) {   // dX^ buffer k & 1 read by the dx of tile k - 2
                    uint32_t ph = static_cast<uint32_t>(((k - 2) >> 1) & 1);
                    wt.wait(&bar[PB_DE + (k & 1)], ph);
                }
                tc_fence_after();
                // dX^_k += [alpha|beta]_j [Omega_g ; A_g]: K = 128, 16 per MMA (eight columns of
                // bf16 pairs of the tensor-memory operand; the W rows of the group 2 KiB per
                // 16-row K step)
                const uint32_t ta = tmem0 + kColA + 64u * (j & 1);
                const uint64_t dwm = dw0 + ((cw.slot * kGroupBytes) >> 4);   // same tiles, MN-major
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    umma_bf16_ts(tmem0 + kColDX + 64u * (k & 1), ta + 8 * kk, dwm + 128 * kk, idD,
                                 (g > 0 || kk > 0) ? 1u : 0u);
                umma_commit(&bar[PB_AE + (j & 1)]);
                umma_commit(&bar[PB_WE + cw.slot]);   // the group's W (projection and contraction) done
                if (g == ng - 1) umma_commit(&bar[PB_DF + (k & 1)]);
                cw.next();
                if (j + 2 < njobs) proj();   // job j + 2 into U[j & 1], read already (AF)
                if (++g == ng) {
                    g = 0;
                    ++k;
                }
            }
        }
        __syncwarp();
    } else {
        const int ew = warp - 1, q = warp & 3, half = ew >> 2;
        const uint32_t row = 32u * q + lane;
        const uint32_t trow = tmem0 + ((32u * q) << 16);
        // dx of tile k (X slot s, its rows' 1/|x| and |x|): dX^ (64 columns) -> (dX^ - x^
        // (x^ . dX^)) / n, this warp's half.  It runs after the next tile's jobs, so the wait
        // for the tile's last contraction is hidden behind them (dX^ is double buffered; the
        // X slot is released here, with kXBufs tiles in flight).
        auto dx_tile = [&](int k, int s, float inv, float nrm) {
            const unsigned char* xrow = sm + L.x + s * kBoxBytes + row * 128;
            {
                uint32_t ph = static_cast<uint32_t>((k >> 1) & 1);
                wt.wait(&bar[PB_DF + (k & 1)], ph);
            }
            tc_fence_after();
            uint32_t d0[32], d1[32];
            tmem_ld32(trow + kColDX + 64u * (k & 1), d0);
            tmem_ld32(trow + kColDX + 64u * (k & 1) + 32, d1);
            tmem_wait_ld();
            reg_fence(d0);
            reg_fence(d1);
            tc_fence_before();
            warp_arrive(&bar[PB_DE + (k & 1)]);
            // x^ of this row from the X tile (bf16, 128-byte swizzle: 16-byte chunk c of the
            // row at c ^ (row & 7)), read where it is used so that it holds no registers
            const uint4* xr = reinterpret_cast<const uint4*>(xrow);
            float dot[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint4 w4 = xr[c ^ (row & 7)];
                const uint32_t ws[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int i = 8 * c + 2 * e;   // element index 0..63
                    const float lo = __uint_as_float(ws[e] << 16);
                    const float hi = __uint_as_float(ws[e] & 0xFFFF0000u);
                    const float dlo = i < 32 ? __uint_as_float(d0[i]) : __uint_as_float(d1[i - 32]);
                    const float dhi = i < 32 ? __uint_as_float(d0[i + 1]) : __uint_as_float(d1[i - 31]);
                    dot[e] = fmaf(lo, dlo, dot[e]);
                    dot[e] = fmaf(hi, dhi, dot[e]);
                }
            }
            // below the 1e-12 norm guard x^ = x / 1e-12 is not a unit vector and its
            // derivative is the identity / 1e-12: no tangential projection there
            const float xd = nrm > 1e-12f ? ((dot[0] + dot[1]) + (dot[2] + dot[3])) * inv : 0.0f;
            // this warp's 32 rows x 32 columns through its staging box (128-byte swizzle:
            // 16-byte chunk c of row r at c ^ (r & 7)) and a TMA store; rows past the last row
            // are clipped by the tensor map
            const uint32_t box = sbase + L.stg + ew * kStgBytes;
            if (lane == 0) bulk_wait_read<0>();   // the previous tile's store has read it
            __syncwarp();
#pragma unroll
            for (int c = 0; c < 4; ++c) {   // this warp's 32 columns: chunks 4 half .. + 3
                const uint4 w4 = xr[(4 * half + c) ^ (row & 7)];
                const uint32_t ws[4] = {w4.x, w4.y, w4.z, w4.w};
                float o[8];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int i = 8 * c + 2 * e;   // column within the half
                    // selects, not an indexed pointer (local memory)
                    const float dlo = half ? __uint_as_float(d1[i]) : __uint_as_float(d0[i]);
                    const float dhi = half ? __uint_as_float(d1[i + 1]) : __uint_as_float(d0[i + 1]);
                    o[2 * e] = (dlo - __uint_as_float(ws[e] << 16) * inv * xd) * inv;
                    o[2 * e + 1] = (dhi - __uint_as_float(ws[e] & 0xFFFF0000u) * inv * xd) * inv;
                }
                st_shared_v4(box + sw128_off(lane, 2 * c), __float_as_uint(o[0]), __float_as_uint(o[1]),
                             __float_as_uint(o[2]), __float_as_uint(o[3]));
                st_shared_v4(box + sw128_off(lane, 2 * c + 1), __float_as_uint(o[4]), __float_as_uint(o[5]),
                             __float_as_uint(o[6]), __float_as_uint(o[7]));
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
                tma_store_2d(&tmdx, sm + L.stg + ew * kStgBytes, 32 * half, row0_of(k) + 32 * q);
                bulk_commit_group();
            }
            warp_arrive(&bar[PB_XE + s]);   // this warp is done with X slot s
        };
        Ring xring(kXBufs), dr(kDRing);
        int ps = 0;                     // X slot of the tile whose dx is pending
        float pinv = 1.0f, pnrm = 1.0f;
        for (int k = 0; k < nt; ++k) {
            const int s = xring.slot;
            {
                uint32_t ph = static_cast<uint32_t>(xring.use & 1);
                wt.wait(&bar[PB_XF + s], ph);
            }
            float inv, l2i;
            const unsigned char* xrow = sm + L.x + s * kBoxBytes + row * 128;
            row_scale(xrow, row, inv, l2i);
            const float nrm = 1.0f / inv, two_n = 2.0f * nrm;
            for (int g = 0; g < ng; ++g) {
                const int j = k * ng + g;
                // this row's 32 dphi of the group from the TMA tile (128-byte swizzle: 16-byte
                // chunk c of row r at c ^ (r & 7)); the slot is released at once
                uint4 dp[kW];
                {
                    uint32_t ph = static_cast<uint32_t>(dr.use & 1);
                    wt.wait(&bar[PB_GF + dr.slot], ph);
                }
                const uint4* drow = reinterpret_cast<const uint4*>(sm + L.d + dr.slot * kBoxBytes + row * 128);
#pragma unroll
                for (int i = 0; i < kW; ++i) dp[i] = drow[(4 * half + i) ^ (row & 7)];
                warp_arrive(&bar[PB_GE + dr.slot]);
                dr.next();
                {
                    uint32_t ph = static_cast<uint32_t>((j >> 1) & 1);
                    wt.wait(&bar[PB_UF + (j & 1)], ph);
                }
                tc_fence_after();
                uint32_t ur[32], pr[32];
                const uint32_t c0 = trow + kColU + 128u * (j & 1) + 64u * half;
                tmem_ld32(c0, ur);
                tmem_ld32(c0 + 32, pr);
                tmem_wait_ld();
                reg_fence(ur);
                reg_fence(pr);
                const int sub = 2 * g + half;
                const float a = pp.a2[sub] * inv, bb = pp.b2[sub] + l2i, sq = pp.sq[sub];
                const float2 a2 = make_float2(a, a), b2 = make_float2(bb, bb);
                const float2 sq2 = make_float2(sq, sq), tn2 = make_float2(two_n, two_n);
                uint32_t al[16], be[16];
#pragma unroll
                for (int c = 0; c < 32; c += 2) {
                    // pairs of features through the packed two-wide fp32 instructions (each
                    // lane rounds like the scalar form, in the same order)
                    const float2 d = make_float2(dphi_val(dp, c), dphi_val(dp, c + 1));
                    const float2 p = make_float2(__uint_as_float(pr[c]), __uint_as_float(pr[c + 1]));
                    const float2 y = ffma2(a2, make_float2(__uint_as_float(ur[c]), __uint_as_float(ur[c + 1])), b2);
                    // every exp2 on the special-function unit: moving a share onto the FMA pipe
                    // as a polynomial made this loop issue-bound (measured slower)
                    const float2 e = make_float2(ex2(y.x), ex2(y.y));
                    const float2 t = fmul2(fmul2(d, e), p);
                    const float2 af = fmul2(fmul2(t, p), sq2);
                    const float2 bf = fmul2(t, tn2);
                    al[c >> 1] = pack_bf16(af.x, af.y);
                    be[c >> 1] = pack_bf16(bf.x, bf.y);
                }
                if (j >= 2) {   // operand buffer j & 1 read by the contraction of job j - 2
                    uint32_t ph = static_cast<uint32_t>(((j - 2) >> 1) & 1);
                    wt.wait(&bar[PB_AE + (j & 1)], ph);
                }
                // K order of the operand: alpha then beta of sub-slice 2g in K 0..63 (columns
                // 0..31), of 2g+1 in K 64..127 -- the row order of the group's packed W (32
                // omega, 32 anchor); this warp writes its rows' 32 columns of sub-slice 2g+half
                const uint32_t acol = trow + kColA + 64u * (j & 1) + 32u * half;
                tmem_st16(acol, al);
                tmem_st16(acol + 16, be);
                tmem_wait_st();
                tc_fence_before();
                warp_arrive(&bar[PB_AF + (j & 1)]);
            }
            if (k >= 1) dx_tile(k - 1, ps, pinv, pnrm);
            ps = s;
            pinv = inv;
            pnrm = nrm;
            xring.next();
        }
        if (nt > 0) dx_tile(nt - 1, ps, pinv, pnrm);
        if (lane == 0) bulk_wait<0>();   // this warp's dx stores have landed
    }
    wt.report(status);
    drain_after_failure(wt.ok);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem0, 512);
}

// dx [n][64] fp32 for the TMA stores: boxes of 32 columns (128 bytes) x 32 rows, 128-byte
// swizzle; rows past n are not written.
bool map_dx(CUtensorMap* m, float* dx, int64_t n)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {64, static_cast<cuuint64_t>(n)};
    const cuuint64_t strides[1] = {64 * 4};
    const cuuint32_t box[2] = {32, 32};
    const cuuint32_t es[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, dx, dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool tc_phi_bwd_supported(int D, int R, int m, int64_t n_rows)
{
    const int F = R * m;
    return D == 64 && m % 32 == 0 && F % 128 == 0 && F <= 512 && n_rows > 0 &&
           n_rows <= (int64_t(1) << 31) - kRows && pb_layout(F).total + 1024 <= 232448;
}

cudaError_t tc_phi_bwd(const void* x, const void* dphi, float* dx, int64_t n, const Params& P,
                       cudaStream_t st)
{
    const int F = P.F;
    if (!P.wB || !tc_phi_bwd_supported(64, P.R, P.m, n)) return cudaErrorNotSupported;
    CUtensorMap mx, mw, md, mdx;
    if (!map_dx(&mdx, dx, n) ||
        !map_2d(&mx, x, 64, static_cast<uint64_t>(n), 64, kRows, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !map_2d(&mw, P.wB, 64, static_cast<uint64_t>(F / 32) * 64, 64, 64,
                CU_TENSOR_MAP_SWIZZLE_128B) ||
        !map_2d(&md, dphi, F, static_cast<uint64_t>(n), 64, kRows, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    PbParams pp;
    pp.F = F;
    pp.ntiles = static_cast<int>((n + kRows - 1) / kRows);
    for (int sub = 0; sub < 16; ++sub) {
        const int node = sub < F / 32 ? sub * 32 / P.m : 0;
        pp.a2[sub] = P.a2[node];
        pp.b2[sub] = P.b2[node];
        pp.sq[sub] = P.sq[node];
    }
    int* status = static_cast<int*>(const_cast<void*>(fmap_status_word()));
    if (!status) return cudaErrorInvalidValue;
    cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int), st);
    if (e != cudaSuccess) return e;
    const size_t smem = pb_layout(F).total + 1024;
    const int grid = pp.ntiles < kNumSMs ? pp.ntiles : kNumSMs;
    e = cudaFuncSetAttribute(k_tc_phi_bwd, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    TraceScope trace_("tc_phi_bwd", st);
    k_tc_phi_bwd<<<grid, kPbThreads, smem, st>>>(mx, mw, md, mdx, pp, status);
    return cudaGetLastError();
}

}  // namespace slay
