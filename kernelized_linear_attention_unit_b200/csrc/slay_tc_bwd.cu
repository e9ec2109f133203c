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
// and [G_c | zg_c] = sum over later tokens of phi(q) [dn, delta]: the exclusive forward and
// reverse scans of the per-tile sums that k_tc_bwd_states computes.
//
// Per tile (M = 128 rows, all MMAs kind::f16, fp32 accumulators in tensor memory):
//   phase A: P = sum_s phiQ_s phiK_s^T (64-feature slices s), C0 = dn V^T;
//            the epilogue masks them (j <= i, inside L), adds delta_i to C0 and writes bf16
//            P~ and C~ into shared memory;
//   phase B: dV = P~^T dn, then per slice s: dphiQ_s = C~ phiK_s + dn S_s^T,
//            dphiK_s = C~^T phiQ_s + V G_s^T, dV += phiK_s G_s; the epilogue adds the z terms
//            and writes dphiQ, dphiK (fp32) per slice, dV per tile.
// The ones / delta columns never enter an MMA (their terms are rank one, added in fp32),
// so every contraction has K a multiple of 64.  The transposed products read the same
// shared-memory tiles as MN-major operands.
//
// Persistent, one CTA per SM over the (b, h, tile) items.  Warp 0 issues the MMAs, warp 9
// the TMA loads (V and dn (bf16 rows), and the phi slice pairs of both phases through a ring
// of two), warps 1-8 are the epilogue (lane quadrant w % 4, column half (w - 1) / 4; delta per
// row from its fp32 array).  Every wait is bounded; a timeout sets the workspace status word.
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
constexpr int kE = 65;                   // state / [dn | delta] columns in the scans' layout
// The per-tile sums are stored per 64-feature slab: [65 e][64 f] fp32 (kSlabF floats).  The
// scan rewrites each slab in place as the contraction's operand: [64 f][64 e] bf16 (8 KiB,
// loaded by TMA) followed by z (e = 64) as fp32 [64 f] at float offset kZOff.
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
    uint32_t phi, pt, ct, dn, v, sg, bar, tmem, total;
};

__host__ __device__ inline BwLayout bw_layout()
{
    BwLayout l;
    l.phi = 0;                    // 2 slots x (phiQ slice, phiK slice)
    l.pt = l.phi + 4 * kTile;     // P~ as two column halves [128 i][64 j]
    l.ct = l.pt + 2 * kTile;      // C~ likewise
    l.dn = l.ct + 2 * kTile;      // dn [128 i][64 e] (TMA, with V)
    l.v = l.dn + kTile;           // V [128 j][64 e]
    l.sg = l.v + kTile;           // 2 buffers x (S_s, G_s) [64 f][64 e]
    l.bar = l.sg + 4 * kSG;
    l.tmem = l.bar + BW_NUM * 8;
    l.total = l.tmem + 16;
    return l;
}

struct BwParams {
    int L, F, ntiles, nitems;
    int dphi_bf16;   // contraction: store dphi(q), dphi(k) as bf16 (else fp32)
    int bidir;       // contraction: the bidirectional form (no masked intra-tile term; sfw,
                     // gbw hold each sequence's whole sums [BH][65][F], not per-tile scans)
};

__global__ void __launch_bounds__(kBwThreads, 1)
k_tc_bwd_tile(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
              const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmdn,
              const __grid_constant__ CUtensorMap tms, const __grid_constant__ CUtensorMap tmg,
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
                if (!valid) return;
                if (bp.dphi_bf16) {
                    uint4* dq4 = reinterpret_cast<uint4*>(static_cast<uint16_t*>(dphq) + grow * bp.F + f0);
                    uint4* dk4 = reinterpret_cast<uint4*>(static_cast<uint16_t*>(dphk) + grow * bp.F + f0);
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        dq4[c] = make_uint4(pack_bf16(oq[8 * c], oq[8 * c + 1]), pack_bf16(oq[8 * c + 2], oq[8 * c + 3]),
                                            pack_bf16(oq[8 * c + 4], oq[8 * c + 5]), pack_bf16(oq[8 * c + 6], oq[8 * c + 7]));
                        dk4[c] = make_uint4(pack_bf16(ok[8 * c], ok[8 * c + 1]), pack_bf16(ok[8 * c + 2], ok[8 * c + 3]),
                                            pack_bf16(ok[8 * c + 4], ok[8 * c + 5]), pack_bf16(ok[8 * c + 6], ok[8 * c + 7]));
                    }
                } else {
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
    }
    wt.report(err);
    drain_after_failure(wt.ok);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------ tile states
// Per 128-token tile t of sequence bh: st_s[bh][t][slab][e][f] = sum_{j in t} phi(k_j)_f
// [v_j, 1]_e and st_g[bh][t][slab][e][f] = sum_{i in t} phi(q_i)_f [dn_i, delta_i]_e (fp32,
// 64-feature slabs, e = 64 the last row; e-major inside a slab so that a warp's 32 features
// store contiguously), the inputs of the scans (k_scan_slabs) that give the contraction S_c
// and G_c.
// Per item and 128-feature block mb: S = phiK_mb^T [V | 1] and G = phiQ_mb^T [dn | delta]
// (M = 128 features, N = 80, K = 128 tokens), phi read as an MN-major A operand (two 64-
// feature tiles), the extra column through a second 64-wide tile at the operand's leading
// byte offset: constant ones for [V | 1], delta_i in every column for [dn | delta].
// Warp 0 issues the MMAs, warp 9 the TMA loads (V and the bf16 dn rows with them), warps 1-8
// write delta into the extension tile and store the sums (lane quadrant w % 4 = 32
// features, half (w - 1) / 4 of the columns).
constexpr int kStThreads = 32 * 10;

enum {
    ST_VF = 0, ST_VE, ST_PF0, ST_PF1, ST_PE0, ST_PE1, ST_YF, ST_YE, ST_DF0, ST_DF1, ST_DE0, ST_DE1,
    ST_NUM
};

struct StLayout {
    uint32_t phi, v, ones, dn, dl, bar, tmem, total;
};

__host__ __device__ inline StLayout st_layout()
{
    StLayout l;
    l.phi = 0;                   // 2 slots x (phiQ 2 tiles, phiK 2 tiles) of one feature block
    l.v = l.phi + 8 * kTile;
    l.ones = l.v + kTile;        // right after V: [V | 1] at LBO = kTile
    l.dn = l.ones + kTile;       // dn (TMA, with V)
    l.dl = l.dn + kTile;         // right after dn: [dn | delta] at LBO = kTile
    l.bar = l.dl + kTile;
    l.tmem = l.bar + ST_NUM * 8;
    l.total = l.tmem + 16;
    return l;
}

__global__ void __launch_bounds__(kStThreads, 1)
k_tc_bwd_states(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmdn,
                const float* __restrict__ delta, float* __restrict__ st_s, float* __restrict__ st_g,
                BwParams bp, int* err)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* sm = aligned_smem(smem_raw);
    const StLayout Lo = st_layout();
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + Lo.bar);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + Lo.tmem);
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nb = bp.F / 128;                  // 128-feature blocks (jobs per item)

    if (warp == 0) {
        tmem_alloc(tslot, 512);
        tmem_relinquish();
    }
    {   // bf16 ones (the extra column of [V | 1], replicated over the tile)
        uint32_t* p = reinterpret_cast<uint32_t*>(sm + Lo.ones);
        for (int i = tid; i < kTile / 4; i += blockDim.x) p[i] = 0x3F803F80u;
    }
    if (tid == 0) {
        for (int i = 0; i < ST_NUM; ++i) mbar_init(&bar[i], 1);
        mbar_init(&bar[ST_YF], 8);
        mbar_init(&bar[ST_DE0], 8);
        mbar_init(&bar[ST_DE1], 8);
        mbar_fence_init();
        tma_prefetch_desc(&tmq);
        tma_prefetch_desc(&tmk);
        tma_prefetch_desc(&tmv);
        tma_prefetch_desc(&tmdn);
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
            int use = 0, it = 0;
            for (int item = blockIdx.x; item < bp.nitems && wt.ok; item += gridDim.x, ++it) {
                const int bh = item / bp.ntiles, t = item - bh * bp.ntiles;
                if (it >= 1) wait_k(ST_VE, it - 1);
                mbar_arrive_expect_tx(&bar[ST_VF], 2 * kTile);   // V and dn
                tma_load_3d(sm + Lo.v, &tmv, &bar[ST_VF], 0, t * kT, bh);
                tma_load_3d(sm + Lo.dn, &tmdn, &bar[ST_VF], 0, t * kT, bh);
                for (int mb = 0; mb < nb; ++mb, ++use) {
                    const int slot = use & 1;
                    if (use >= 2) wait_k(ST_PE0 + slot, (use >> 1) - 1);
                    mbar_arrive_expect_tx(&bar[ST_PF0 + slot], 4 * kTile);
                    unsigned char* dst = sm + Lo.phi + slot * 4 * kTile;
                    tma_load_3d(dst, &tmq, &bar[ST_PF0 + slot], 128 * mb, t * kT, bh);
                    tma_load_3d(dst + kTile, &tmq, &bar[ST_PF0 + slot], 128 * mb + 64, t * kT, bh);
                    tma_load_3d(dst + 2 * kTile, &tmk, &bar[ST_PF0 + slot], 128 * mb, t * kT, bh);
                    tma_load_3d(dst + 3 * kTile, &tmk, &bar[ST_PF0 + slot], 128 * mb + 64, t * kT, bh);
                }
            }
        }
        __syncwarp();
    } else if (warp == 0) {
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16(128, 80, 1, 1);   // A, B MN-major
            const uint64_t dphi0 = sdesc(sbase + Lo.phi, kTile, 1024, kLayoutSW128);
            const uint64_t dvb = sdesc(sbase + Lo.v, Lo.ones - Lo.v, 1024, kLayoutSW128);
            const uint64_t dyb = sdesc(sbase + Lo.dn, Lo.dl - Lo.dn, 1024, kLayoutSW128);
            int use = 0, it = 0, job = 0;
            for (int item = blockIdx.x; item < bp.nitems && wt.ok; item += gridDim.x, ++it) {
                wait_k(ST_VF, it);
                wait_k(ST_YF, it);
                for (int mb = 0; mb < nb; ++mb, ++use, ++job) {
                    const int slot = use & 1, b = job & 1;
                    wait_k(ST_PF0 + slot, use >> 1);
                    if (job >= 2) wait_k(ST_DE0 + b, (job >> 1) - 1);
                    tc_fence_after();
                    const uint64_t dq = dphi0 + ((slot * 4 * kTile) >> 4), dk = dq + ((2 * kTile) >> 4);
                    const uint32_t cs = tmem + 160u * b, cg = cs + 80;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        umma_bf16(cs, dk + 128 * kk, dvb + 128 * kk, idS, kk > 0 ? 1u : 0u);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        umma_bf16(cg, dq + 128 * kk, dyb + 128 * kk, idS, kk > 0 ? 1u : 0u);
                    umma_commit(&bar[ST_DF0 + b]);
                    umma_commit(&bar[ST_PE0 + slot]);
                }
                umma_commit(&bar[ST_VE]);
                umma_commit(&bar[ST_YE]);
            }
        }
        __syncwarp();
    } else {
        const int ew = warp - 1, q = warp & 3, half = ew >> 2;
        const uint32_t row = 32u * q + lane;
        const uint32_t trow = tmem + ((32u * q) << 16);
        int it = 0, job = 0;
        for (int item = blockIdx.x; item < bp.nitems && wt.ok; item += gridDim.x, ++it) {
            const int bh = item / bp.ntiles, t = item - bh * bp.ntiles;
            const int i_abs = t * kT + static_cast<int>(row);
            const bool valid = i_abs < bp.L;
            const int64_t grow = static_cast<int64_t>(bh) * bp.L + i_abs;
            // delta of this thread's token in the first 16 columns of its row of the extension
            // tile (the columns the N = 80 operand reads; dn itself arrives by TMA with V)
            if (it >= 1) wait_k(ST_YE, it - 1);
            {
                const float dl = valid ? delta[grow] : 0.0f;
                const uint32_t dd = pack_bf16(dl, dl);
                st_shared_v4(sbase + Lo.dl + sw128_off(row, half), dd, dd, dd, dd);
            }
            fence_async_smem();
            warp_arrive(&bar[ST_YF]);
            for (int mb = 0; mb < nb; ++mb, ++job) {
                const int b = job & 1;
                wait_k(ST_DF0 + b, job >> 1);
                tc_fence_after();
                // feature f = 128 mb + row; this warp writes columns 32 half .. (+ e = 64 for half 1)
                uint32_t sa[32], ga[32], sz = 0, gz = 0;
                const uint32_t cs = trow + 160u * b, cg = cs + 80;
                tmem_ld32(cs + 32 * half, sa);
                tmem_ld32(cg + 32 * half, ga);
                if (half) {
                    tmem_ld1(cs + 64, sz);
                    tmem_ld1(cg + 64, gz);
                }
                tmem_wait_ld();
                reg_fence(sa);
                reg_fence(ga);
                reg_fence1(sz);
                reg_fence1(gz);
                tc_fence_before();
                warp_arrive(&bar[ST_DE0 + b]);
                // slab f / 64, element (e, f % 64) at e * 64 + f % 64: for each e a warp's 32
                // consecutive features store 128 contiguous bytes
                const int f = 128 * mb + static_cast<int>(row);
                const int64_t o = (static_cast<int64_t>(bh) * bp.ntiles + t) * bp.F * kE +
                                  static_cast<int64_t>(f >> 6) * kSlabF + 64 * (32 * half) + (f & 63);
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    st_s[o + 64 * c] = __uint_as_float(sa[c]);
                    st_g[o + 64 * c] = __uint_as_float(ga[c]);
                }
                if (half) {
                    st_s[o + 64 * 32] = __uint_as_float(sz);
                    st_g[o + 64 * 32] = __uint_as_float(gz);
                }
            }
        }
    }
    wt.report(err);
    drain_after_failure(wt.ok);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------ scans over tiles
// One CTA per (sequence bh, 64-feature slab) and sum (blockIdx.y: 0 = S, 1 = G): walks the
// sequence's tiles in order (S: forward; G: backward) keeping fp32 running sums and writes,
// over each tile's slab, the sum over the tiles before it (S_c) or after it (G_c) -- the
// exclusive prefix / suffix -- as the contraction's operand: [64 f][64 e] bf16 and z fp32.
// total != 0 (the bidirectional form): the whole-sequence sums instead, written once to
// tot_s / tot_g ([BH][slabs] slabs of the same form); the per-tile sums are left as they are.
// Thread: feature fl = tid % 64 and the 16 e of group eg = tid / 64 (group 3 also e = 64),
// so its operand row piece is 32 contiguous bytes.  A tile's sums are all in registers (and
// added) before the barrier after which its slab is overwritten.
constexpr int kScanThreads = 256;

__global__ void __launch_bounds__(kScanThreads)
k_scan_slabs(float* __restrict__ st_s, float* __restrict__ st_g, float* __restrict__ tot_s,
             float* __restrict__ tot_g, int NS, int nsl, int total)
{
    const int which = blockIdx.y;
    const int bh = static_cast<int>(blockIdx.x) / nsl, slab = static_cast<int>(blockIdx.x) - bh * nsl;
    float* base = (which ? st_g : st_s) + (static_cast<int64_t>(bh) * NS * nsl + slab) * kSlabF;
    const int64_t tstride = static_cast<int64_t>(nsl) * kSlabF;   // floats from tile to tile
    const int fl = threadIdx.x & 63, eg = threadIdx.x >> 6;
    const bool hasz = eg == 3;
    const bool rev = !total && which == 1;
    float run[17], x[17];
#pragma unroll
    for (int c = 0; c < 17; ++c) run[c] = 0.0f;
    auto load = [&](int t) {
        const float* p = base + t * tstride + (16 * eg) * 64 + fl;
#pragma unroll
        for (int c = 0; c < 16; ++c) x[c] = p[64 * c];
        x[16] = hasz ? base[t * tstride + 64 * 64 + fl] : 0.0f;
    };
    auto store = [&](float* slab_base, const float (&val)[17]) {
        uint4* op = reinterpret_cast<uint4*>(reinterpret_cast<unsigned char*>(slab_base) + fl * 128 + 32 * eg);
        op[0] = make_uint4(pack_bf16(val[0], val[1]), pack_bf16(val[2], val[3]),
                           pack_bf16(val[4], val[5]), pack_bf16(val[6], val[7]));
        op[1] = make_uint4(pack_bf16(val[8], val[9]), pack_bf16(val[10], val[11]),
                           pack_bf16(val[12], val[13]), pack_bf16(val[14], val[15]));
        if (hasz) slab_base[kZOff + fl] = val[16];
    };
    const int t0 = rev ? NS - 1 : 0, step = rev ? -1 : 1;
    load(t0);
    for (int i = 0; i < NS; ++i) {
        const int t = t0 + i * step;
        float out[17];
#pragma unroll
        for (int c = 0; c < 17; ++c) {
            out[c] = run[c];
            run[c] += x[c];
        }
        if (i + 1 < NS) load(t + step);   // the next tile's sums, in flight during the stores
        if (!total) {
            __syncthreads();   // every thread has added tile t's sums: its slab may be overwritten
            store(base + t * tstride, out);
        }
    }
    if (total) store((which ? tot_g : tot_s) + (static_cast<int64_t>(bh) * nsl + slab) * kSlabF, run);
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
           st_layout().total + 1024 <= 232448;
}

cudaError_t tc_bwd_states(const void* phq, const void* phk, const void* v, const void* dn16,
                          const float* delta, float* st_s, float* st_g, int BH, int L, int F,
                          int* err, cudaStream_t st)
{
    if (!tc_bwd_tile_supported(F, L)) return cudaErrorNotSupported;
    CUtensorMap mq, mk, mv, mdn;
    if (!map_seq(&mq, phq, F, L, BH) || !map_seq(&mk, phk, F, L, BH) || !map_seq(&mv, v, 64, L, BH) ||
        !map_seq(&mdn, dn16, 64, L, BH))
        return cudaErrorInvalidValue;
    BwParams bp;
    bp.L = L;
    bp.F = F;
    bp.ntiles = (L + kT - 1) / kT;
    bp.nitems = BH * bp.ntiles;
    bp.dphi_bf16 = 0;
    bp.bidir = 0;
    const size_t smem = st_layout().total + 1024;
    cudaError_t e = cudaFuncSetAttribute(k_tc_bwd_states, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const int grid = bp.nitems < kNumSMs ? bp.nitems : kNumSMs;
    TraceScope trace_("tc_bwd_states", st);
    k_tc_bwd_states<<<grid, kStThreads, smem, st>>>(mq, mk, mv, mdn, delta, st_s, st_g, bp, err);
    return cudaGetLastError();
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
    BwParams bp;
    bp.L = L;
    bp.F = F;
    bp.ntiles = (L + kT - 1) / kT;
    bp.nitems = BH * bp.ntiles;
    bp.dphi_bf16 = dphi_bf16 ? 1 : 0;
    bp.bidir = bidir ? 1 : 0;
    // the operand slabs the scans wrote: per tile (causal) or per sequence (bidirectional)
    const int64_t nslabs = static_cast<int64_t>(BH) * (bidir ? 1 : bp.ntiles) * (F / 64);
    CUtensorMap ms, mg;
    if (!map_slabs(&ms, sfw, nslabs) || !map_slabs(&mg, gbw, nslabs)) return cudaErrorInvalidValue;
    const size_t smem = bw_layout().total + 1024;
    cudaError_t e = cudaFuncSetAttribute(k_tc_bwd_tile, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const int grid = bp.nitems < kNumSMs ? bp.nitems : kNumSMs;
    TraceScope trace_("tc_bwd_tile", st);
    k_tc_bwd_tile<<<grid, kBwThreads, smem, st>>>(mq, mk, mv, mdn, ms, mg, delta, sfw, gbw, dphq, dphk,
                                                  dv, bp, err);
    return cudaGetLastError();
}

cudaError_t tc_bwd_scan(float* st_s, float* st_g, float* tot_s, float* tot_g, int BH, int L, int F,
                        bool bidir, cudaStream_t st)
{
    if (!tc_bwd_tile_supported(F, L)) return cudaErrorNotSupported;
    const int NS = (L + kT - 1) / kT, nsl = F / 64;
    TraceScope trace_("tc_bwd_scan", st);
    k_scan_slabs<<<dim3(static_cast<unsigned>(BH * nsl), 2), kScanThreads, 0, st>>>(
        st_s, st_g, tot_s, tot_g, NS, nsl, bidir ? 1 : 0);
    return cudaGetLastError();
}

}  // namespace slay
