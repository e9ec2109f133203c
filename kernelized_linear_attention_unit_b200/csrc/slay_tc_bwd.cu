// slay_tc_bwd.cu -- tensor-core chunk contraction of the causal backward (bf16 mode).
//
// Method: "SLAY: Geometry-Aware Spherical Linearized Attention with Yat-Kernel" (nubint.ai
// review, "Proposed method", step 6: the linear-attention contraction); the pages give no
// backward, so this is the derivative of out_i = phi(q_i)^T S_i / (phi(q_i)^T z_i + eps).
// With dn_i = g_i / Z_i, delta_i = -(g_i . out_i) / Z_i and, inside a 128-token tile,
// P_ij = phi(q_i) . phi(k_j) and c_ij = v_j . dn_i + delta_i restricted to j <= i:
//   dphi(q_i) = sum_j c_ij phi(k_j) + S_c[:, :64] dn_i + z_c delta_i
//   dphi(k_j) = sum_i c_ij phi(q_i) + G_c[:, :64] v_j + zg_c
//   dv_j      = sum_i P_ij dn_i + G_c[:, :64]^T phi(k_j)
// where [S_c | z_c] = sum over earlier tokens of phi(k) [v, 1] (the state entering the tile)
// and [G_c | zg_c] = sum over later tokens of phi(q) [dn, delta], which k_tc_bwd_sums writes
// per tile as bf16 operands (and z in fp32).
//
// Per tile (M = 128 rows, all MMAs kind::f16, fp32 accumulators in tensor memory):
//   phase A: P = sum_s phiQ_s phiK_s^T (64-feature slices s), C0 = dn V^T;
//            the epilogue masks them (j <= i, inside L), adds delta_i to C0 and writes bf16
//            P~ and C~ into shared memory;
//   phase B: dV = P~^T dn, then per slice s: dphiQ_s = C~ phiK_s + dn S_s^T,
//            dphiK_s = C~^T phiQ_s + V G_s^T, dV += phiK_s G_s; the epilogue adds the z terms
//            and writes dphiQ, dphiK per slice (bf16 through TMA stores, or fp32), dV per
//            tile.
// The ones / delta columns never enter an MMA (their terms are rank one, added in fp32),
// so every contraction has K a multiple of 64.  The transposed products read the same
// shared-memory tiles as MN-major operands.
//
// Persistent, one CTA per SM over the (b, h, tile) items.  Warp 0 issues the MMAs, warp 9
// the TMA loads (V and dn (bf16 rows), the phi slice pairs of both phases through a ring of
// two, and per phase-B slice S_s and G_s from k_tc_bwd_sums' operand slabs), warps 1-8 are
// the epilogue (lane quadrant w % 4, column half (w - 1) / 4; delta per row from its fp32
// array).  Every wait is bounded; a timeout sets the workspace status word.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "slay_tc.h"
#include "slay_tc_common.cuh"
#include "slay_tc_ptx.cuh"

namespace slay {

using namespace tc;

namespace {

constexpr int kT = 128;                  // tokens per tile
constexpr int kTile = kT * 128;          // [128][64] bf16, 128-byte swizzle = 16 KiB
constexpr int kSG = 64 * 128;            // [64 f][64 e] bf16 = 8 KiB
constexpr int kE = 65;                   // [S | z] / [G | zg] columns
// The sums reach the contraction per 64-feature slab, kSlabF floats apart (the workspace is
// sized for fp32 [65][64] slabs): [64 f][64 e] bf16 (8 KiB, loaded by TMA) followed by z
// (e = 64) as fp32 [64 f] at float offset kZOff.
constexpr int kSlabF = 64 * kE;
constexpr int kZOff = 64 * 64 / 2;
constexpr int kBwThreads = 32 * 10;
constexpr int kNumSMs = 148;
// tensor memory: phase A P [0,128) and C0 [128,256); phase B per-slice buffers b: dphiQ at
// 128 b, dphiK at 128 b + 64; dV at 256
constexpr uint32_t kColP = 0, kColC = 128, kColDV = 256;

enum {
    BW_VF = 0, BW_VE, BW_PF0, BW_PF1, BW_PE0, BW_PE1, BW_PCF, BW_PCTF, BW_PCTE,
    BW_SGF0, BW_SGF1, BW_SGE0, BW_SGE1, BW_DQF0, BW_DQF1, BW_DQE0, BW_DQE1, BW_DVF, BW_DVE,
    BW_NUM
};

struct BwLayout {
    uint32_t phi, pt, ct, dn, v, sg, stg, bar, tmem, total;
};
constexpr int kStgBytes = 2 * 32 * 64;   // per epilogue warp: dphiQ, dphiK boxes [32 rows][32 bf16]

__host__ __device__ inline BwLayout bw_layout()
{
    BwLayout l;
    l.phi = 0;                    // 2 slots x (phiQ slice, phiK slice)
    l.pt = l.phi + 4 * kTile;     // P~ as two column halves [128 i][64 j]
    l.ct = l.pt + 2 * kTile;      // C~ likewise
    l.dn = l.ct + 2 * kTile;      // dn [128 i][64 e] (TMA, with V)
    l.v = l.dn + kTile;           // V [128 j][64 e]
    l.sg = l.v + kTile;           // 2 buffers x (S_s, G_s) [64 f][64 e]
    l.stg = l.sg + 4 * kSG;       // 8 epilogue warps x kStgBytes: bf16 dphi staged for TMA stores
    l.bar = l.stg + 8 * kStgBytes;
    l.tmem = l.bar + BW_NUM * 8;
    l.total = l.tmem + 16;
    return l;
}

struct BwParams {
    int L, F, ntiles, nitems;
    int dphi_bf16;   // contraction: store dphi(q), dphi(k) as bf16 (else fp32)
    int bidir;       // contraction: the bidirectional form (no masked intra-tile term; sfw,
                     // gbw hold each sequence's whole sums, not each tile's)
    // running sums (k_tc_bwd_sums): which sums (bit 0 S, bit 1 G), their starting values --
    // the sums over the tokens before this piece of the sequence (S) and after it (G),
    // [BH][F][64] and [BH][F] fp32, or null -- and, for G, an fp32 total out (same layout)
    int sums;
    const float* seed_s;
    const float* seed_z;
    const float* seed_g;
    const float* seed_zg;
    float* out_g;
    float* out_zg;
};

__global__ void __launch_bounds__(kBwThreads, 1)
k_tc_bwd_tile(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
              const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmdn,
              const __grid_constant__ CUtensorMap tms, const __grid_constant__ CUtensorMap tmg,
              const __grid_constant__ CUtensorMap tmdq, const __grid_constant__ CUtensorMap tmdk,
              const float* __restrict__ delta, const float* __restrict__ sfw,
              const float* __restrict__ gbw,
              void* __restrict__ dphq, void* __restrict__ dphk, float* __restrict__ dv,
              BwParams bp, int* err)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* sm = aligned_smem(smem_raw);
    const BwLayout Lo = bw_layout();
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + Lo.bar);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + Lo.tmem);
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ns = bp.F / 64;

    if (warp == 0) {
        tmem_alloc(tslot, 512);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < BW_NUM; ++i) mbar_init(&bar[i], 1);
        const int warp_counted[4] = {BW_PCTF, BW_DQE0, BW_DQE1, BW_DVE};
        for (int i = 0; i < 4; ++i) mbar_init(&bar[warp_counted[i]], 8);   // one arrival per epilogue warp
        mbar_fence_init();
        tma_prefetch_desc(&tmq);
        tma_prefetch_desc(&tmk);
        tma_prefetch_desc(&tmv);
        tma_prefetch_desc(&tmdn);
        tma_prefetch_desc(&tms);
        tma_prefetch_desc(&tmg);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    Waiter wt;
    // waits on the k-th completion (k >= 0) of a barrier
    auto wait_k = [&](int b, int k) {
        uint32_t ph = static_cast<uint32_t>(k & 1);
        wt.wait(&bar[b], ph);
    };

    if (warp == 9) {
        // ---------------------------------------------------------------- TMA loads
        if (lane == 0) {
            int use = 0, it = 0;   // phi slice-pair loads so far; items so far
            for (int item = blockIdx.x; item < bp.nitems && wt.ok; item += gridDim.x, ++it) {
                const int bh = item / bp.ntiles, t = item - bh * bp.ntiles;
                if (it >= 1) wait_k(BW_VE, it - 1);
                mbar_arrive_expect_tx(&bar[BW_VF], 2 * kTile);   // V and dn
                tma_load_3d(sm + Lo.v, &tmv, &bar[BW_VF], 0, t * kT, bh);
                tma_load_3d(sm + Lo.dn, &tmdn, &bar[BW_VF], 0, t * kT, bh);
                // operand slab of slice s: tile t's (bidirectional: the sequence's) slab s
                const int64_t slab0 = (bp.bidir ? static_cast<int64_t>(bh) : static_cast<int64_t>(bh) * bp.ntiles + t) * ns;
                for (int u = 0; u < 2 * ns; ++u, ++use) {   // phase A slices, then phase B
                    const int s = u < ns ? u : u - ns, slot = use & 1;
                    if (u >= ns) {   // S_s and G_s for phase B (buffer of slice k = it ns + s)
                        const int k = it * ns + s, sb = k & 1;
                        if (k >= 2) wait_k(BW_SGE0 + sb, (k >> 1) - 1);
                        mbar_arrive_expect_tx(&bar[BW_SGF0 + sb], 2 * kSG);
                        unsigned char* sgd = sm + Lo.sg + sb * 2 * kSG;
                        tma_load_3d(sgd, &tms, &bar[BW_SGF0 + sb], 0, 0, static_cast<int>(slab0 + s));
                        tma_load_3d(sgd + kSG, &tmg, &bar[BW_SGF0 + sb], 0, 0, static_cast<int>(slab0 + s));
                    }
                    if (use >= 2) wait_k(BW_PE0 + slot, (use >> 1) - 1);
                    mbar_arrive_expect_tx(&bar[BW_PF0 + slot], 2 * kTile);
                    unsigned char* dst = sm + Lo.phi + slot * 2 * kTile;
                    tma_load_3d(dst, &tmq, &bar[BW_PF0 + slot], 64 * s, t * kT, bh);
                    tma_load_3d(dst + kTile, &tmk, &bar[BW_PF0 + slot], 64 * s, t * kT, bh);
                }
            }
        }
        __syncwarp();
    } else if (warp == 0) {
        // ---------------------------------------------------------------- MMA issue
        if (lane == 0) {
            constexpr uint32_t idKK128 = idesc_bf16(128, 128, 0, 0);
            constexpr uint32_t idKK64 = idesc_bf16(128, 64, 0, 0);
            constexpr uint32_t idKM64 = idesc_bf16(128, 64, 0, 1);   // B MN-major
            constexpr uint32_t idMM64 = idesc_bf16(128, 64, 1, 1);   // A and B MN-major
            const uint64_t dphi0 = sdesc(sbase + Lo.phi, 16, 1024, kLayoutSW128);
            const uint64_t dct_k = sdesc(sbase + Lo.ct, 16, 1024, kLayoutSW128);
            const uint64_t dpt_m = sdesc(sbase + Lo.pt, kTile, 1024, kLayoutSW128);   // M = 128 over both halves
            const uint64_t dct_m = sdesc(sbase + Lo.ct, kTile, 1024, kLayoutSW128);
            const uint64_t ddn = sdesc(sbase + Lo.dn, 16, 1024, kLayoutSW128);
            const uint64_t dvv = sdesc(sbase + Lo.v, 16, 1024, kLayoutSW128);
            const uint64_t dsg0 = sdesc(sbase + Lo.sg, 16, 1024, kLayoutSW128);
            int use = 0, gs = 0, it = 0;   // phi uses, slice-accumulator uses, items
            for (int item = blockIdx.x; item < bp.nitems && wt.ok; item += gridDim.x, ++it) {
                wait_k(BW_VF, it);
                // P / C0 overwrite the slice buffers of the previous item: both read
                if (gs >= 1) wait_k(BW_DQE0 + ((gs - 1) & 1), (gs - 1) >> 1);
                if (gs >= 2) wait_k(BW_DQE0 + ((gs - 2) & 1), (gs - 2) >> 1);
                tc_fence_after();
                // phase A
                for (int s = 0; s < ns; ++s, ++use) {
                    const int slot = use & 1;
                    wait_k(BW_PF0 + slot, use >> 1);
                    tc_fence_after();
                    const uint64_t dq = dphi0 + ((slot * 2 * kTile) >> 4), dk = dq + (kTile >> 4);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_bf16(tmem + kColP, dq + 2 * kk, dk + 2 * kk, idKK128, (s > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&bar[BW_PE0 + slot]);
                }
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_bf16(tmem + kColC, ddn + 2 * kk, dvv + 2 * kk, idKK128, kk > 0 ? 1u : 0u);
                umma_commit(&bar[BW_PCF]);
                // phase B
                wait_k(BW_PCTF, it);
                if (it >= 1) wait_k(BW_DVE, it - 1);
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)   // dV = P~^T dn (K = i)
                    umma_bf16(tmem + kColDV, dpt_m + 128 * kk, ddn + 128 * kk, idMM64, kk > 0 ? 1u : 0u);
                for (int s = 0; s < ns; ++s, ++use, ++gs) {
                    // S/G buffer of slice k = it ns + s is k & 1 (gs == k: one per slice)
                    const int slot = use & 1, b = gs & 1, sb = gs & 1;
                    wait_k(BW_PF0 + slot, use >> 1);
                    wait_k(BW_SGF0 + sb, gs >> 1);
                    if (gs >= 2) wait_k(BW_DQE0 + b, (gs - 2) >> 1);
                    tc_fence_after();
                    const uint64_t dq = dphi0 + ((slot * 2 * kTile) >> 4), dk = dq + (kTile >> 4);
                    const uint64_t ds = dsg0 + ((sb * 2 * kSG) >> 4), dg = ds + (kSG >> 4);
                    const uint32_t cq = tmem + 128u * b, ck = cq + 64;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)   // dphiQ_s = C~ phiK_s (K = j)
                        umma_bf16(cq, dct_k + (kk >> 2) * (kTile >> 4) + 2 * (kk & 3), dk + 128 * kk,
                                  idKM64, kk > 0 ? 1u : 0u);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)   // += dn S_s^T (K = e)
                        umma_bf16(cq, ddn + 2 * kk, ds + 2 * kk, idKK64, 1u);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)   // dphiK_s = C~^T phiQ_s (K = i)
                        umma_bf16(ck, dct_m + 128 * kk, dq + 128 * kk, idMM64, kk > 0 ? 1u : 0u);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)   // += V G_s^T (K = e)
                        umma_bf16(ck, dvv + 2 * kk, dg + 2 * kk, idKK64, 1u);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)   // dV += phiK_s G_s (K = f)
                        umma_bf16(tmem + kColDV, dk + 2 * kk, dg + 128 * kk, idKM64, 1u);
                    umma_commit(&bar[BW_DQF0 + b]);
                    umma_commit(&bar[BW_SGE0 + sb]);
                    umma_commit(&bar[BW_PE0 + slot]);
                }
                umma_commit(&bar[BW_DVF]);
                umma_commit(&bar[BW_PCTE]);
                umma_commit(&bar[BW_VE]);   // V and dn free
            }
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- epilogue
        const int ew = warp - 1, q = warp & 3, half = ew >> 2;
        const uint32_t row = 32u * q + lane;
        const uint32_t trow = tmem + ((32u * q) << 16);
        int it = 0, gs = 0;
        for (int item = blockIdx.x; item < bp.nitems && wt.ok; item += gridDim.x, ++it) {
            const int bh = item / bp.ntiles, t = item - bh * bp.ntiles;
            const int i_abs = t * kT + static_cast<int>(row);   // this thread's token
            const bool valid = i_abs < bp.L;
            const int64_t grow = static_cast<int64_t>(bh) * bp.L + i_abs;
            const int64_t sidx = bp.bidir ? static_cast<int64_t>(bh) : static_cast<int64_t>(bh) * bp.ntiles + t;
            const float* Sb = sfw + sidx * bp.F * kE;
            const float* Gb = gbw + sidx * bp.F * kE;
            const bool intra = valid && !bp.bidir;   // the masked term exists only when causal
            const float dl = valid ? delta[grow] : 0.0f;   // dn itself arrives by TMA with V
            // masked P~ and C~ (this warp's half of the columns j)
            wait_k(BW_PCF, it);
            tc_fence_after();
            {
                uint32_t pr[32], p2[32], cr[32], c2[32];
                tmem_ld32(trow + kColP + 64 * half, pr);
                tmem_ld32(trow + kColP + 64 * half + 32, p2);
                tmem_ld32(trow + kColC + 64 * half, cr);
                tmem_ld32(trow + kColC + 64 * half + 32, c2);
                tmem_wait_ld();
                reg_fence(pr);
                reg_fence(p2);
                reg_fence(cr);
                reg_fence(c2);
                if (it >= 1) wait_k(BW_PCTE, it - 1);
                uint32_t pk[16], ck[16];
                const int j0 = t * kT + 64 * half;   // absolute token of column 64 half
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const uint32_t* P = hh ? p2 : pr;
                    const uint32_t* Cc = hh ? c2 : cr;
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        const int jl = 64 * half + 32 * hh + 2 * c;     // column within the tile
                        const bool k0 = intra && jl <= static_cast<int>(row) && j0 + 32 * hh + 2 * c < bp.L;
                        const bool k1 = intra && jl + 1 <= static_cast<int>(row) && j0 + 32 * hh + 2 * c + 1 < bp.L;
                        pk[c] = pack_bf16(k0 ? __uint_as_float(P[2 * c]) : 0.0f,
                                          k1 ? __uint_as_float(P[2 * c + 1]) : 0.0f);
                        ck[c] = pack_bf16(k0 ? __uint_as_float(Cc[2 * c]) + dl : 0.0f,
                                          k1 ? __uint_as_float(Cc[2 * c + 1]) + dl : 0.0f);
                    }
                    // column chunk 4 hh .. of the half tile
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        st_shared_v4(sbase + Lo.pt + half * kTile + sw128_off(row, 4 * hh + c),
                                     pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
                        st_shared_v4(sbase + Lo.ct + half * kTile + sw128_off(row, 4 * hh + c),
                                     ck[4 * c], ck[4 * c + 1], ck[4 * c + 2], ck[4 * c + 3]);
                    }
                }
            }
            fence_async_smem();
            tc_fence_before();
            warp_arrive(&bar[BW_PCTF]);
            // per slice the outputs (S_s and G_s reach the MMAs by TMA, already bf16).  The
            // rank-one terms' z_c and zg_c of the warp's 32 features: lane c loads feature
            // f0 + c from the slab's fp32 z (a slice ahead) and the warp broadcasts them.
            auto load_z = [&](int s, float& zsl, float& zgl) {
                zsl = Sb[static_cast<int64_t>(s) * kSlabF + kZOff + 32 * half + lane];
                zgl = Gb[static_cast<int64_t>(s) * kSlabF + kZOff + 32 * half + lane];
            };
            auto write_slice = [&](int s, int b, float zsl, float zgl) {
                wait_k(BW_DQF0 + b, gs >> 1);
                tc_fence_after();
                uint32_t qa[32], ka[32];
                tmem_ld32(trow + 128u * b + 32 * half, qa);
                tmem_ld32(trow + 128u * b + 64 + 32 * half, ka);
                tmem_wait_ld();
                reg_fence(qa);
                reg_fence(ka);
                tc_fence_before();
                warp_arrive(&bar[BW_DQE0 + b]);
                ++gs;
                const int f0 = 64 * s + 32 * half;
                float oq[32], ok[32];
#pragma unroll
                for (int c = 0; c < 32; ++c) {   // every lane takes part in the broadcasts
                    oq[c] = fmaf(dl, __shfl_sync(0xffffffffu, zsl, c), __uint_as_float(qa[c]));
                    ok[c] = __uint_as_float(ka[c]) + __shfl_sync(0xffffffffu, zgl, c);
                }
                if (bp.dphi_bf16) {
                    // this warp's 32 rows x 32 features of dphiQ and dphiK through its staging
                    // boxes (64-byte swizzle: chunk c of row r at c ^ ((r >> 1) & 3), so a
                    // warp's 16-byte writes spread over 8 bank groups) and two TMA stores;
                    // rows past L are clipped by the tensor map
                    const uint32_t qbuf = sbase + Lo.stg + ew * kStgBytes, kbuf = qbuf + 32 * 64;
                    if (lane == 0) bulk_wait_read<0>();   // the previous slice's stores read them
                    __syncwarp();
                    const uint32_t rsw = (static_cast<uint32_t>(lane) >> 1) & 3u;
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const uint32_t off = lane * 64u + ((static_cast<uint32_t>(c) ^ rsw) << 4);
                        st_shared_v4(qbuf + off, pack_bf16(oq[8 * c], oq[8 * c + 1]), pack_bf16(oq[8 * c + 2], oq[8 * c + 3]),
                                     pack_bf16(oq[8 * c + 4], oq[8 * c + 5]), pack_bf16(oq[8 * c + 6], oq[8 * c + 7]));
                        st_shared_v4(kbuf + off, pack_bf16(ok[8 * c], ok[8 * c + 1]), pack_bf16(ok[8 * c + 2], ok[8 * c + 3]),
                                     pack_bf16(ok[8 * c + 4], ok[8 * c + 5]), pack_bf16(ok[8 * c + 6], ok[8 * c + 7]));
                    }
                    fence_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        const int r0 = t * kT + 32 * q;
                        tma_store_3d(&tmdq, sm + Lo.stg + ew * kStgBytes, f0, r0, bh);
                        tma_store_3d(&tmdk, sm + Lo.stg + ew * kStgBytes + 32 * 64, f0, r0, bh);
                        bulk_commit_group();
                    }
                } else {
                    if (!valid) return;
                    float4* dq4 = reinterpret_cast<float4*>(static_cast<float*>(dphq) + grow * bp.F + f0);
                    float4* dk4 = reinterpret_cast<float4*>(static_cast<float*>(dphk) + grow * bp.F + f0);
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        dq4[c] = make_float4(oq[4 * c], oq[4 * c + 1], oq[4 * c + 2], oq[4 * c + 3]);
                        dk4[c] = make_float4(ok[4 * c], ok[4 * c + 1], ok[4 * c + 2], ok[4 * c + 3]);
                    }
                }
            };
            float zsl, zgl, zsn = 0.0f, zgn = 0.0f;
            load_z(0, zsl, zgl);
            for (int s = 0; s < ns; ++s) {
                if (s + 1 < ns) load_z(s + 1, zsn, zgn);
                write_slice(s, gs & 1, zsl, zgl);
                zsl = zsn;
                zgl = zgn;
            }
            // dV
            wait_k(BW_DVF, it);
            tc_fence_after();
            {
                uint32_t va[32];
                tmem_ld32(trow + kColDV + 32 * half, va);
                tmem_wait_ld();
                reg_fence(va);
                tc_fence_before();
                warp_arrive(&bar[BW_DVE]);
                if (valid) {
                    float4* o = reinterpret_cast<float4*>(dv + grow * 64 + 32 * half);
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        o[c] = make_float4(__uint_as_float(va[4 * c]), __uint_as_float(va[4 * c + 1]),
                                           __uint_as_float(va[4 * c + 2]), __uint_as_float(va[4 * c + 3]));
                }
            }
        }
        if (lane == 0) bulk_wait<0>();   // this warp's dphi stores have landed
    }
    wt.report(err);
    drain_after_failure(wt.ok);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------ running sums over tiles
// The contraction's S_c and G_c directly: one CTA per (sequence bh, 128-feature block mb,
// sum: blockIdx.x & 1 == 0 S, 1 G) walks the sequence's tiles (S forward, G backward),
// accumulates each tile's sum -- S_t = phiK_mb^T [V | 1], G_t = phiQ_mb^T [dn | delta] (M = 128
// features, N = 80, K = 128 tokens, phi read as an MN-major A operand, the extra column
// through a second tile at the B operand's leading-byte offset: constant ones, or delta in
// every column) -- into fp32 running sums held by the epilogue threads, and writes, per tile,
// the sum over the tiles before it (S) or after it (G) as an operand slab: [64 f][64 e] bf16
// and z fp32 (the form k_tc_bwd_tile loads by TMA).  total != 0 (bidirectional): only the
// whole-sequence sums, into tot_s / tot_g.  Tiles stream through two slots (phi block, V or
// dn, the extension tile) and two accumulators, so tile i + 1's MMAs run while tile i's sums
// are read.  Warp 0 issues the MMAs, warp 9 the TMA loads, warps 1-8 are the epilogue (lane
// quadrant w % 4 = 32 features, e half (w - 1) / 4; half 1 also e = 64) and, for G, write
// delta into the extension tile (row = token).
constexpr int kSumThreads = 32 * 10;

enum { SU_PF0 = 0, SU_PF1, SU_PE0, SU_PE1, SU_XF0, SU_XF1, SU_DF0, SU_DF1, SU_DE0, SU_DE1, SU_NUM };

struct SuLayout {
    uint32_t phi, y, stg, bar, tmem, total;
};

__host__ __device__ inline SuLayout su_layout()
{
    SuLayout l;
    l.phi = 0;                    // 2 slots x (two 64-feature tiles of the block)
    l.y = l.phi + 4 * kTile;      // 2 slots x (V or dn tile, then its extension tile at LBO)
    l.stg = l.y + 4 * kTile;      // 8 epilogue warps x [32 f][32 e] bf16 staged for TMA stores
    l.bar = l.stg + 8 * 32 * 64;
    l.tmem = l.bar + SU_NUM * 8;
    l.total = l.tmem + 16;
    return l;
}

__global__ void __launch_bounds__(kSumThreads, 1)
k_tc_bwd_sums(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
              const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmdn,
              const __grid_constant__ CUtensorMap tmso, const __grid_constant__ CUtensorMap tmgo,
              const float* __restrict__ delta, float* __restrict__ st_s, float* __restrict__ st_g,
              float* __restrict__ tot_s, float* __restrict__ tot_g, BwParams bp, int* err)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* sm = aligned_smem(smem_raw);
    const SuLayout Lo = su_layout();
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + Lo.bar);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + Lo.tmem);
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nb = bp.F / 128, NS = bp.ntiles, nsl = bp.F / 64;
    // 0: S (keys, forward), 1: G (queries, backward); one CTA of each per job unless only
    // one of the sums is wanted
    const int g = bp.sums == 3 ? static_cast<int>(blockIdx.x) & 1 : bp.sums >> 1;
    const int job = bp.sums == 3 ? static_cast<int>(blockIdx.x) >> 1 : static_cast<int>(blockIdx.x);
    const int bh = job / nb, mb = job - bh * nb;
    const bool total = bp.bidir != 0;
    auto tile_of = [&](int i) { return (g && !total) ? NS - 1 - i : i; };

    if (warp == 0) {
        tmem_alloc(tslot, 256);
        tmem_relinquish();
    }
    if (!g) {   // S: the extension tiles are constant bf16 ones
        for (int b = 0; b < 2; ++b) {
            uint32_t* p = reinterpret_cast<uint32_t*>(sm + Lo.y + (2 * b + 1) * kTile);
            for (int i = tid; i < kTile / 4; i += blockDim.x) p[i] = 0x3F803F80u;
        }
    }
    if (tid == 0) {
        for (int i = 0; i < SU_NUM; ++i) mbar_init(&bar[i], 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bar[SU_XF0 + b], 8);
            mbar_init(&bar[SU_DE0 + b], 8);
        }
        mbar_fence_init();
        tma_prefetch_desc(g ? &tmq : &tmk);
        tma_prefetch_desc(g ? &tmdn : &tmv);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    Waiter wt;
    auto wait_k = [&](int b, int k) {
        uint32_t ph = static_cast<uint32_t>(k & 1);
        wt.wait(&bar[b], ph);
    };

    if (warp == 9) {
        if (lane == 0) {
            const CUtensorMap* mphi = g ? &tmq : &tmk;
            const CUtensorMap* my = g ? &tmdn : &tmv;
            for (int i = 0; i < NS && wt.ok; ++i) {
                const int b = i & 1, t = tile_of(i);
                if (i >= 2) wait_k(SU_PE0 + b, (i >> 1) - 1);
                mbar_arrive_expect_tx(&bar[SU_PF0 + b], 3 * kTile);
                unsigned char* dp = sm + Lo.phi + b * 2 * kTile;
                tma_load_3d(dp, mphi, &bar[SU_PF0 + b], 128 * mb, t * kT, bh);
                tma_load_3d(dp + kTile, mphi, &bar[SU_PF0 + b], 128 * mb + 64, t * kT, bh);
                tma_load_3d(sm + Lo.y + 2 * b * kTile, my, &bar[SU_PF0 + b], 0, t * kT, bh);
            }
        }
        __syncwarp();
    } else if (warp == 0) {
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16(128, 80, 1, 1);   // A, B MN-major
            const uint64_t dphi0 = sdesc(sbase + Lo.phi, kTile, 1024, kLayoutSW128);
            const uint64_t dy0 = sdesc(sbase + Lo.y, kTile, 1024, kLayoutSW128);
            for (int i = 0; i < NS && wt.ok; ++i) {
                const int b = i & 1;
                wait_k(SU_PF0 + b, i >> 1);
                if (g) wait_k(SU_XF0 + b, i >> 1);
                if (i >= 2) wait_k(SU_DE0 + b, (i >> 1) - 1);
                tc_fence_after();
                const uint64_t da = dphi0 + ((b * 2 * kTile) >> 4), dbb = dy0 + ((b * 2 * kTile) >> 4);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    umma_bf16(tmem + 128u * b, da + 128 * kk, dbb + 128 * kk, idS, kk > 0 ? 1u : 0u);
                umma_commit(&bar[SU_PE0 + b]);
                umma_commit(&bar[SU_DF0 + b]);
            }
        }
        __syncwarp();
    } else {
        const int ew = warp - 1, q = warp & 3, half = ew >> 2;
        const uint32_t row = 32u * q + lane;   // TMEM lane: feature 128 mb + row; token row of delta
        const uint32_t trow = tmem + ((32u * q) << 16);
        const int f = 128 * mb + static_cast<int>(row);
        float run[33];
        {   // the sum over the tokens outside this piece of the sequence (zero when none)
            const float* sd = g ? bp.seed_g : bp.seed_s;
            const float* zd = g ? bp.seed_zg : bp.seed_z;
            const int64_t o = (static_cast<int64_t>(bh) * bp.F + f) * 64 + 32 * half;
#pragma unroll
            for (int c = 0; c < 32; ++c) run[c] = sd ? sd[o + c] : 0.0f;
            run[32] = (zd && half) ? zd[static_cast<int64_t>(bh) * bp.F + f] : 0.0f;
        }
        // delta of this thread's token in its 16-byte chunk `half` of the extension row (the
        // 16 columns the N = 80 operand reads), for walk step i
        auto write_delta = [&](int i) {
            const int b = i & 1, t = tile_of(i);
            if (i >= 2) wait_k(SU_PE0 + b, (i >> 1) - 1);   // the MMAs of step i - 2 read it
            const int i_abs = t * kT + static_cast<int>(row);
            const float dl = i_abs < bp.L ? delta[static_cast<int64_t>(bh) * bp.L + i_abs] : 0.0f;
            const uint32_t dd = pack_bf16(dl, dl);
            st_shared_v4(sbase + Lo.y + (2 * b + 1) * kTile + sw128_off(row, half), dd, dd, dd, dd);
            fence_async_smem();
            warp_arrive(&bar[SU_XF0 + b]);
        };
        // the operand slab form of feature f's running sums: row f % 64 of slab f / 64, this
        // warp's 32 e (64 bytes) through its staging box (64-byte swizzle: chunk c of row r
        // at c ^ ((r >> 1) & 3)) and a TMA store of [32 f][32 e]; z (half 1) stored directly
        const CUtensorMap* mout = g ? &tmgo : &tmso;
        const uint32_t sbox = sbase + Lo.stg + ew * 32 * 64;
        auto store = [&](int64_t slab, float* zdst) {
            if (lane == 0) bulk_wait_read<0>();   // the box's previous store has read it
            __syncwarp();
            const uint32_t rsw = (static_cast<uint32_t>(lane) >> 1) & 3u;
#pragma unroll
            for (int c = 0; c < 4; ++c)
                st_shared_v4(sbox + lane * 64u + ((static_cast<uint32_t>(c) ^ rsw) << 4),
                             pack_bf16(run[8 * c], run[8 * c + 1]), pack_bf16(run[8 * c + 2], run[8 * c + 3]),
                             pack_bf16(run[8 * c + 4], run[8 * c + 5]), pack_bf16(run[8 * c + 6], run[8 * c + 7]));
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
                tma_store_3d(mout, sm + Lo.stg + ew * 32 * 64, 32 * half, 32 * (q & 1), static_cast<int>(slab));
                bulk_commit_group();
            }
            if (half) zdst[kZOff + (f & 63)] = run[32];
        };
        float* sums = g ? st_g : st_s;
        if (g && NS > 0) write_delta(0);
        for (int i = 0; i < NS && wt.ok; ++i) {
            const int b = i & 1, t = tile_of(i);
            if (g && i + 1 < NS) write_delta(i + 1);
            // the sum over the tiles walked so far, before tile t: its operand (causal)
            if (!total) {
                const int64_t slab = (static_cast<int64_t>(bh) * NS + t) * nsl + (f >> 6);
                store(slab, sums + slab * kSlabF);
            }
            wait_k(SU_DF0 + b, i >> 1);
            tc_fence_after();
            uint32_t a[32], z = 0;
            tmem_ld32(trow + 128u * b + 32 * half, a);
            if (half) tmem_ld1(trow + 128u * b + 64, z);
            tmem_wait_ld();
            reg_fence(a);
            reg_fence1(z);
            tc_fence_before();
            warp_arrive(&bar[SU_DE0 + b]);
#pragma unroll
            for (int c = 0; c < 32; ++c) run[c] += __uint_as_float(a[c]);
            run[32] += __uint_as_float(z);
        }
        if (total && (g ? tot_g : tot_s)) {
            const int64_t slab = static_cast<int64_t>(bh) * nsl + (f >> 6);
            store(slab, (g ? tot_g : tot_s) + slab * kSlabF);
        }
        if (g && bp.out_g) {   // fp32 total of G (a piece's state for the other ranks)
            float4* o = reinterpret_cast<float4*>(bp.out_g + (static_cast<int64_t>(bh) * bp.F + f) * 64 + 32 * half);
#pragma unroll
            for (int c = 0; c < 8; ++c) o[c] = make_float4(run[4 * c], run[4 * c + 1], run[4 * c + 2], run[4 * c + 3]);
            if (half) bp.out_zg[static_cast<int64_t>(bh) * bp.F + f] = run[32];
        }
        if (lane == 0) bulk_wait<0>();   // this warp's stores have landed
    }
    wt.report(err);
    drain_after_failure(wt.ok);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

// bf16 dphi [BH][L][F] viewed as a 3-D tensor for the contraction's TMA stores: boxes of 32
// features x 32 tokens, 64-byte swizzle; rows past L are not written.
bool map_dphi(CUtensorMap* m, void* base, int F, int L, int BH)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(F), static_cast<cuuint64_t>(L),
                                static_cast<cuuint64_t>(BH)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(F) * 2, static_cast<cuuint64_t>(L) * F * 2};
    const cuuint32_t box[3] = {32, 32, 1};
    const cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
              CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Operand slabs ([nslabs] x [64 f][64 e] bf16, kSlabF floats apart) viewed as a 3-D tensor,
// one [64][64] box per slab, 128-byte swizzle.
bool map_slabs(CUtensorMap* m, const float* base, int64_t nslabs)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {64, 64, static_cast<cuuint64_t>(nslabs)};
    const cuuint64_t strides[2] = {128, static_cast<cuuint64_t>(kSlabF) * 4};
    const cuuint32_t box[3] = {64, 64, 1};
    const cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<float*>(base), dims, strides, box,
              es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The same slabs for k_tc_bwd_sums' TMA stores: boxes of 32 e x 32 f, 64-byte swizzle.
bool map_slabs_out(CUtensorMap* m, float* base, int64_t nslabs)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {64, 64, static_cast<cuuint64_t>(nslabs)};
    const cuuint64_t strides[2] = {128, static_cast<cuuint64_t>(kSlabF) * 4};
    const cuuint32_t box[3] = {32, 32, 1};
    const cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
              CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [BH][L][cols] bf16 viewed as a 3-D tensor, boxes of 64 columns x 128 tokens, 128-byte
// swizzle; rows past L read as zero.
bool map_seq(CUtensorMap* m, const void* base, int cols, int L, int BH)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(L),
                                static_cast<cuuint64_t>(BH)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(cols) * 2,
                                   static_cast<cuuint64_t>(L) * cols * 2};
    const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(kT), 1};
    const cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
              es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool tc_bwd_tile_supported(int F, int L)
{
    return F % 128 == 0 && F >= 128 && F <= 512 && L > 0 && bw_layout().total + 1024 <= 232448 &&
           su_layout().total + 1024 <= 232448;
}

cudaError_t tc_bwd_tile(const void* phq, const void* phk, const void* v, const void* dn16,
                        const float* delta, const float* sfw, const float* gbw, void* dphq,
                        void* dphk, bool dphi_bf16, float* dv, int BH, int L, int F, int* err,
                        cudaStream_t st, bool bidir)
{
    if (!tc_bwd_tile_supported(F, L)) return cudaErrorNotSupported;
    CUtensorMap mq, mk, mv, mdn;
    if (!map_seq(&mq, phq, F, L, BH) || !map_seq(&mk, phk, F, L, BH) || !map_seq(&mv, v, 64, L, BH) ||
        !map_seq(&mdn, dn16, 64, L, BH))
        return cudaErrorInvalidValue;
    BwParams bp{};
    bp.L = L;
    bp.F = F;
    bp.ntiles = (L + kT - 1) / kT;
    bp.nitems = BH * bp.ntiles;
    bp.dphi_bf16 = dphi_bf16 ? 1 : 0;
    bp.bidir = bidir ? 1 : 0;
    // the operand slabs k_tc_bwd_sums wrote: per tile (causal) or per sequence (bidirectional)
    const int64_t nslabs = static_cast<int64_t>(BH) * (bidir ? 1 : bp.ntiles) * (F / 64);
    CUtensorMap ms, mg, mdq = mq, mdk = mk;   // (mdq, mdk unused when dphi is fp32)
    if (!map_slabs(&ms, sfw, nslabs) || !map_slabs(&mg, gbw, nslabs)) return cudaErrorInvalidValue;
    if (dphi_bf16 && (!map_dphi(&mdq, dphq, F, L, BH) || !map_dphi(&mdk, dphk, F, L, BH)))
        return cudaErrorInvalidValue;
    const size_t smem = bw_layout().total + 1024;
    cudaError_t e = cudaFuncSetAttribute(k_tc_bwd_tile, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const int grid = bp.nitems < kNumSMs ? bp.nitems : kNumSMs;
    TraceScope trace_("tc_bwd_tile", st);
    k_tc_bwd_tile<<<grid, kBwThreads, smem, st>>>(mq, mk, mv, mdn, ms, mg, mdq, mdk, delta, sfw, gbw,
                                                  dphq, dphk, dv, bp, err);
    return cudaGetLastError();
}

cudaError_t tc_bwd_sums(const void* phq, const void* phk, const void* v, const void* dn16,
                        const float* delta, float* st_s, float* st_g, float* tot_s, float* tot_g,
                        int BH, int L, int F, bool bidir, int* err, cudaStream_t st,
                        const BwdSeeds* seeds)
{
    if (!tc_bwd_tile_supported(F, L)) return cudaErrorNotSupported;
    CUtensorMap mq, mk, mv, mdn;
    if (!map_seq(&mq, phq, F, L, BH) || !map_seq(&mk, phk, F, L, BH) || !map_seq(&mv, v, 64, L, BH) ||
        !map_seq(&mdn, dn16, 64, L, BH))
        return cudaErrorInvalidValue;
    BwParams bp{};
    bp.L = L;
    bp.F = F;
    bp.ntiles = (L + kT - 1) / kT;
    bp.nitems = BH * bp.ntiles;
    bp.dphi_bf16 = 0;
    bp.bidir = bidir ? 1 : 0;
    bp.sums = 3;
    if (seeds) {
        bp.sums = seeds->sums;
        bp.seed_s = seeds->s_in;
        bp.seed_z = seeds->z_in;
        bp.seed_g = seeds->g_in;
        bp.seed_zg = seeds->zg_in;
        bp.out_g = seeds->g_out;
        bp.out_zg = seeds->zg_out;
    }
    // outputs: every tile's slabs (causal) or every sequence's (bidirectional); a total-only
    // call (G state of a piece) writes no slabs and passes the inputs' maps as placeholders
    const int64_t nslabs = static_cast<int64_t>(BH) * (bidir ? 1 : bp.ntiles) * (F / 64);
    float* so = bidir ? tot_s : st_s;
    float* go = bidir ? tot_g : st_g;
    CUtensorMap mso = mq, mgo = mq;
    if ((so && !map_slabs_out(&mso, so, nslabs)) || (go && !map_slabs_out(&mgo, go, nslabs)))
        return cudaErrorInvalidValue;
    const size_t smem = su_layout().total + 1024;
    cudaError_t e = cudaFuncSetAttribute(k_tc_bwd_sums, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    TraceScope trace_("tc_bwd_sums", st);
    k_tc_bwd_sums<<<BH * (F / 128) * (bp.sums == 3 ? 2 : 1), kSumThreads, smem, st>>>(mq, mk, mv, mdn, mso, mgo, delta, st_s,
                                                                 st_g, tot_s, tot_g, bp, err);
    return cudaGetLastError();
}


}  // namespace slay
