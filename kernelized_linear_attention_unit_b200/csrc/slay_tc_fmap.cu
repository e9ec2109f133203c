// slay_tc_fmap.cu -- tensor-core feature map phi(x) for bf16 rows, bf16 features.
//
// Method: "SLAY: Geometry-Aware Spherical Linearized Attention with Yat-Kernel" (nubint.ai
// review, "Proposed method", steps 1, 3, 4, 5): per row x and feature f = r*m + j,
//   phi_f(x) = sqrt(wt_r/m) exp(sqrt(2 s_r) omega_f.x^ - s_r) (a_f.x^)^2,  x^ = x/max(|x|,1e-12)
// written as exp2(a2_r u_f/|x| + b2_r + 2 log2(1/|x|)) (p_f/|x|)^2 with u = omega_f.x and
// p = a_f.x of the raw row.
//
// The map reads 128 bytes and writes 2F bytes per row, so it is bound by HBM bandwidth;
// the tensor cores only take the projections off the CUDA cores.  Persistent kernel, one
// CTA per SM holding the packed projection operand W (resident) and two independent teams
// of eight warps.  Each team owns 256 tensor-memory columns (two N = 128 buffers) and its
// own ring of row tiles, and takes 128-row tiles round-robin.  Warp w of a team serves the
// tensor-memory lanes 32 (w % 4) .. +31 (rows of the tile) and the 32-feature half w / 4 of
// every 64-feature group.  Per tile and group g:
//   - each warp waits for the projections U = X W_g^T of group g (an MMA issued two groups
//     earlier by the team's first thread), reads its 32 rows x 64 columns into registers
//     and signals the buffer's release barrier; once all eight warps have, the team's first
//     warp issues the next MMA into that buffer;
//   - each lane maps its row's 32 features and writes them into its warp's swizzled staging
//     box, stored by TMA (32 rows x 32 features per box).
// Each thread computes its own row's norm from the tile in shared memory.  Four warps per
// SM sub-partition hide one another's latencies; the two teams share nothing but W.
// Every wait is bounded; a timeout sets the library's feature-map status word.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "slay_tc.h"
#include "slay_tc_common.cuh"
#include "slay_tc_ptx.cuh"

namespace slay {

using namespace tc;

namespace {

constexpr int kRows = 128;                     // rows per tile (MMA M)
constexpr int kBoxBytes = kRows * 128;         // [128 rows][64 bf16] swizzled X tile = 16 KiB
constexpr int kSubBytes = 64 * 128;            // packed operand of 32 features = 8 KiB
constexpr int kGroupBytes = 2 * kSubBytes;     // 64 features (N = 128) = 16 KiB
constexpr int kTeams = 2;                      // independent teams of 8 warps per CTA
constexpr int kTeamThreads = 256;
constexpr int kComputeWarps = kTeams * kTeamThreads / 32;   // warps kTeams.. of the CTA
constexpr int kFmThreads = kTeamThreads * kTeams + 32 * kTeams;   // + one issuing warp per team
constexpr int kStageBytes = 32 * 64;           // one warp's [32 rows][32 bf16] output box
constexpr int kNumSMs = 148;
constexpr int kMaxXBufs = 4;

__device__ int g_fmap_status;                  // set to 1 by a kernel whose wait ran out

// barriers: W, then per team kMaxXBufs X-full, two U-full (MMA commit) and two U-empty
// (one arrival per warp of the team)
enum { FB_W = 0, FB_TEAM = 1, FB_XF = 0, FB_UF = kMaxXBufs, FB_UE = kMaxXBufs + 2,
       FB_PER_TEAM = kMaxXBufs + 4, FB_NUM = 1 + kTeams * FB_PER_TEAM };

struct FmLayout {
    uint32_t w, x, o, bar, tmem, total;
    int xbufs, obufs;
};

__host__ __device__ inline FmLayout fm_layout(int F)
{
    FmLayout l;
    l.xbufs = F <= 128 ? 4 : F <= 256 ? 3 : 2;   // X tiles in flight per team
    l.obufs = F <= 384 ? 2 : 1;                  // staging boxes per warp
    l.w = 0;                                     // F/32 packed sub-slices, resident
    l.x = (F / 32) * kSubBytes;
    l.o = l.x + kTeams * l.xbufs * kBoxBytes;
    l.bar = l.o + kComputeWarps * l.obufs * kStageBytes;
    l.tmem = l.bar + FB_NUM * 8;
    l.total = l.tmem + 16;
    return l;
}

// 64-byte swizzle of a [rows][64 B] box: 16-byte chunk c of row r sits at chunk
// c ^ ((r >> 1) & 3), the pattern TMA applies for CU_TENSOR_MAP_SWIZZLE_64B.
__device__ __forceinline__ uint32_t sw64_off(uint32_t row, uint32_t chunk)
{
    return row * 64u + ((chunk ^ ((row >> 1) & 3u)) << 4);
}

// Exponentials per pair of features taken by the polynomial below instead of the
// special-function unit: 0 (none), 1 (one of every two pairs' second element) or 2 (every
// pair's second element).  The special-function unit shares its issue queue with the
// shared-memory and barrier operations that pace the pipeline; with the packed two-wide
// fp32 arithmetic below, 0 and 1 measure the same and 2 is slower (the polynomial costs
// about a dozen instructions per value).
#ifndef SLAY_FM_POLY
#define SLAY_FM_POLY 1
#endif

struct FmParams {
    int F, ntiles;
    float a2[16];   // per 32-feature sub-slice (F <= 512): the scales of its node
    float b2[16];
    // Test hook of the failure path (0 in every normal call): the first compute warp of
    // CTA 0 withholds its release of projection buffer 0 after the tile's first group, so
    // team 0's issuer waits for a phase that never completes; every wait of the launch is
    // bounded by wait_ns.
    int withhold;
    unsigned long long wait_ns;
};

// Armed by slay_debug_expire_wait, consumed by the next tensor-core feature-map launch.
std::atomic<int> g_fmap_fault{0};

__global__ void __launch_bounds__(kFmThreads, 1)
k_tc_feature_map(const __grid_constant__ CUtensorMap tmx, const __grid_constant__ CUtensorMap tmw,
                 const __grid_constant__ CUtensorMap tmo, FmParams fp)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* sm = aligned_smem(smem_raw);
    const FmLayout L = fm_layout(fp.F);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + L.bar);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + L.tmem);
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // warp t < kTeams issues for team t; compute warp cw = warp - kTeams belongs to team
    // cw / 8; a warp reaches the TMEM lanes 32 (warp % 4).., and the two warps of a team on
    // the same lanes take the two 32-feature halves
    const int cw = warp - kTeams, team = cw >> 3, tw = cw & 7;
    const int q = warp & 3, half = tw >> 2;
    const int ng = fp.F / 64;                    // 64-feature groups (>= 2)
    const int xbufs = L.xbufs;

    if (warp == 0) {
        tmem_alloc(tslot, 512);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < FB_NUM; ++i) mbar_init(&bar[i], 1);
        for (int t = 0; t < kTeams; ++t)
            for (int b = 0; b < 2; ++b) mbar_init(&bar[FB_TEAM + t * FB_PER_TEAM + FB_UE + b], 8);
        mbar_fence_init();
        tma_prefetch_desc(&tmx);
        tma_prefetch_desc(&tmw);
        tma_prefetch_desc(&tmo);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem0 = *tslot;
    Waiter wt;
    wt.limit = fp.wait_ns;

    // tiles of team t: k-th = (k * gridDim.x + blockIdx.x) * kTeams + t
    const int stride = gridDim.x * kTeams;
    auto team_tiles = [&](int t) {
        const int first = blockIdx.x * kTeams + t;
        return first < fp.ntiles ? (fp.ntiles - 1 - first) / stride + 1 : 0;
    };

    if (warp < kTeams) {
        // Warp t issues for team t.  Job j = (tile k, group g) goes into buffer j & 1 once
        // every warp of the team has read job j - 2 from it (UE) and tile k is in shared
        // memory (XF); X slot k % xbufs takes tile k + xbufs once the team has read the last
        // group of tile k.  One issuer per team keeps each team's chain short: an issuer
        // waits only on its own team.
        const int t = warp;
        if (lane == 0) {
            const int nt = team_tiles(t);
            uint64_t* tb = bar + FB_TEAM + t * FB_PER_TEAM;
            const uint64_t dw0 = sdesc(sbase + L.w, 16, 1024, kLayoutSW128);
            const uint64_t dx0 = sdesc(sbase + L.x + t * xbufs * kBoxBytes, 16, 1024, kLayoutSW128);
            constexpr uint32_t idU = idesc_bf16(128, 128, 0, 0);
            auto load_x = [&](int k, int slot) {
                mbar_arrive_expect_tx(&tb[FB_XF + slot], kBoxBytes);
                tma_load_2d(sm + L.x + (t * xbufs + slot) * kBoxBytes, &tmx, &tb[FB_XF + slot], 0,
                            ((k * gridDim.x + blockIdx.x) * kTeams + t) * kRows);
            };
            if (t == 0 && nt > 0) {
                mbar_arrive_expect_tx(&bar[FB_W], (fp.F / 32) * kSubBytes);
                for (int n = 0; n < fp.F / 32; ++n)
                    tma_load_2d(sm + L.w + n * kSubBytes, &tmw, &bar[FB_W], 0, n * 64);
            }
            for (int k = 0; k < xbufs && k < nt; ++k) load_x(k, k);
            if (nt > 0) {
                uint32_t ph = 0;
                wt.wait(&bar[FB_W], ph);
            }
            int j = 0, sn = 0;                   // job, X slot of its tile
            uint32_t pn = 0;                     // that slot's phase
            for (int k = 0; k < nt && wt.ok; ++k) {
                {
                    uint32_t ph = pn;
                    wt.wait(&tb[FB_XF + sn], ph);
                }
                for (int g = 0; g < ng; ++g, ++j) {
                    if (j >= 2) {                // buffer j & 1 released by job j - 2
                        uint32_t ph = static_cast<uint32_t>(((j - 2) >> 1) & 1);
                        wt.wait(&tb[FB_UE + (j & 1)], ph);
                        // job j - 2 was the last group of tile k - 1 when g == 1 (ng >= 2):
                        // its X slot takes tile k - 1 + xbufs
                        if (g == 1 && k - 1 + xbufs < nt)
                            load_x(k - 1 + xbufs, sn == 0 ? xbufs - 1 : sn - 1);
                    }
                    tc_fence_after();
                    const uint64_t dx = dx0 + ((sn * kBoxBytes) >> 4);
                    const uint64_t dw = dw0 + ((g * kGroupBytes) >> 4);
                    const uint32_t d = tmem0 + 256u * t + 128u * (j & 1);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_bf16(d, dx + 2 * kk, dw + 2 * kk, idU, kk > 0 ? 1u : 0u);
                    umma_commit(&tb[FB_UF + (j & 1)]);
                }
                if (++sn == xbufs) {
                    sn = 0;
                    pn ^= 1u;
                }
            }
        }
        __syncwarp();
    } else {   // the two teams' warps
        uint64_t* tb = bar + FB_TEAM + team * FB_PER_TEAM;
        uint64_t* XF = tb + FB_XF;
        uint64_t* UF = tb + FB_UF;
        uint64_t* UE = tb + FB_UE;
        const unsigned char* xs = sm + L.x + team * xbufs * kBoxBytes;
        const int first = blockIdx.x * kTeams + team;
        const int nt = team_tiles(team);
        const uint32_t row = 32u * q + lane;
        const uint32_t tcol = tmem0 + 256u * team + ((32u * q) << 16) + 64u * half;
        const int obufs = L.obufs;
        const uint32_t obox = sbase + L.o + cw * obufs * kStageBytes;
        int js = 0;                                  // staging boxes used by this warp
        int s = 0;                                   // X slot of tile k and its phase
        uint32_t xph = 0;
        for (int k = 0; k < nt; ++k) {
            {
                uint32_t ph = xph;
                wt.wait(&XF[s], ph);
            }
            float inv, l2i;
            row_scale(xs + s * kBoxBytes + row * 128, row, inv, l2i);
            const int row0 = (first + k * stride) * kRows + 32 * q;
            for (int g = 0; g < ng; ++g, ++js) {
                const int j = k * ng + g;
                const uint32_t ph = static_cast<uint32_t>((j >> 1) & 1);
                {
                    uint32_t p = ph;
                    wt.wait(&UF[j & 1], p);
                }
                tc_fence_after();
                uint32_t ur[32], pr[32];
                tmem_ld32(tcol + 128u * (j & 1), ur);
                tmem_ld32(tcol + 128u * (j & 1) + 32, pr);
                tmem_wait_ld();
                reg_fence(ur);
                reg_fence(pr);
                tc_fence_before();
                // this warp's rows of buffer j & 1 are read (the test hook withholds one
                // release: it guards only the next MMA into the buffer, none in flight)
                if (!(fp.withhold && blockIdx.x == 0 && cw == 0 && j == 0))
                    warp_arrive(&UE[j & 1]);
                const float a = fp.a2[2 * g + half] * inv, bb = fp.b2[2 * g + half] + l2i;
                uint32_t pk[16];
                const float2 a2 = make_float2(a, a), b2 = make_float2(bb, bb);
#pragma unroll
                for (int c = 0; c < 32; c += 2) {
                    // pairs of features through the packed two-wide fp32 instructions
                    const float2 x =
                        make_float2(__uint_as_float(pr[c]), __uint_as_float(pr[c + 1]));
                    const float2 u =
                        make_float2(__uint_as_float(ur[c]), __uint_as_float(ur[c + 1]));
                    const float2 y = ffma2(a2, u, b2);
                    const bool poly = SLAY_FM_POLY == 2 || (SLAY_FM_POLY == 1 && (c & 2));
                    const float2 e = make_float2(ex2(y.x), poly ? ex2_poly(y.y) : ex2(y.y));
                    const float2 f = fmul2(fmul2(e, x), x);
                    pk[c >> 1] = pack_bf16(f.x, f.y);
                }
                // the box was stored obufs groups ago: its reads must be done before it is
                // rewritten
                if (lane == 0) {
                    if (obufs == 2)
                        bulk_wait_read<1>();
                    else
                        bulk_wait_read<0>();
                }
                __syncwarp();
                const uint32_t box = obox + (js & (obufs - 1)) * kStageBytes;
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    st_shared_v4(box + sw64_off(lane, c), pk[4 * c], pk[4 * c + 1], pk[4 * c + 2],
                                 pk[4 * c + 3]);
                fence_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(&tmo, sm + (box - sbase), 64 * g + 32 * half, row0);
                    bulk_commit_group();
                }
            }
            if (++s == xbufs) {
                s = 0;
                xph ^= 1u;
            }
        }
        if (lane == 0) bulk_wait<0>();
    }
    wt.report(&g_fmap_status);
    drain_after_failure(wt.ok);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem0, 512);
}

}  // namespace

bool tc_fmap_supported(int D, int R, int m, int64_t n_rows)
{
    const int F = R * m;
    return D == 64 && m % 32 == 0 && F % 128 == 0 && F <= 512 && n_rows > 0 &&
           n_rows <= (int64_t(1) << 31) - kRows && fm_layout(F).total + 1024 <= 232448;
}

const void* fmap_status_word()
{
    void* p = nullptr;
    return cudaGetSymbolAddress(&p, g_fmap_status) == cudaSuccess ? p : nullptr;
}

cudaError_t tc_feature_map(const void* x, void* phi, int64_t n, const Params& P, cudaStream_t st)
{
    const int F = P.F;
    if (!P.wB || !tc_fmap_supported(64, P.R, P.m, n)) return cudaErrorNotSupported;
    CUtensorMap mx, mw, mo;
    if (!map_2d(&mx, x, 64, static_cast<uint64_t>(n), 64, kRows, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !map_2d(&mw, P.wB, 64, static_cast<uint64_t>(F / 32) * 64, 64, 64,
                CU_TENSOR_MAP_SWIZZLE_128B) ||
        !map_2d(&mo, phi, static_cast<uint64_t>(F), static_cast<uint64_t>(n), 32, 32,
                CU_TENSOR_MAP_SWIZZLE_64B))
        return cudaErrorInvalidValue;
    FmParams fp;
    fp.F = F;
    fp.ntiles = static_cast<int>((n + kRows - 1) / kRows);
    fp.withhold = g_fmap_fault.exchange(0);
    fp.wait_ns = fp.withhold ? 1000000ull : kWaitNs;   // 1 ms under the test hook
    for (int sub = 0; sub < 16; ++sub) {
        const int node = sub < F / 32 ? sub * 32 / P.m : 0;
        fp.a2[sub] = P.a2[node];
        fp.b2[sub] = P.b2[node];
    }
    void* status = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&status, g_fmap_status);
    if (e != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(status, 0, sizeof(int), st)) != cudaSuccess) return e;
    const size_t smem = fm_layout(F).total + 1024;
    e = cudaFuncSetAttribute(k_tc_feature_map, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const int pairs = (fp.ntiles + kTeams - 1) / kTeams;
    const int grid = pairs < kNumSMs ? pairs : kNumSMs;
    TraceScope trace_("tc_feature_map", st);
    k_tc_feature_map<<<grid, kFmThreads, smem, st>>>(mx, mw, mo, fp);
    return cudaGetLastError();
}

void fmap_arm_wait_fault(int on) { g_fmap_fault.store(on ? 1 : 0); }

}  // namespace slay
