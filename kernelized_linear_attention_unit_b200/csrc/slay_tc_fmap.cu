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
// CTA per SM, 128-row tiles dealt round-robin:
//   warp 0      TMA: the packed projection operand once (resident), then row tiles into a
//               ring of 4 (F <= 256) or 2 buffers
//   warp 1      MMA: per tile and 64-feature group, U = X W_g^T with N = 128 (64 omega and
//               64 anchor columns), four buffers in tensor memory (4 x 128 columns)
//   warps 2-17  epilogue, four per SM sub-partition: warp w serves TMEM lanes 32*(w%4)
//               and one 32-feature sub-slice of every other group; it writes its 32 x 32 block of
//               phi to its own swizzled staging box and stores it by TMA (two boxes per
//               warp, so a store overlaps the next group; no CTA-wide barrier)
//   warp 18     the rows' norm scales, up to a ring of X tiles ahead of the epilogue
// Every wait is bounded; a timeout sets the library's feature-map status word.
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

constexpr int kRows = 128;                     // rows per tile (MMA M)
constexpr int kBoxBytes = kRows * 128;         // [128 rows][64 bf16] swizzled X tile = 16 KiB
constexpr int kSubBytes = 64 * 128;            // packed operand of 32 features = 8 KiB
constexpr int kGroupBytes = 2 * kSubBytes;     // 64 features (N = 128) = 16 KiB
constexpr int kUBufs = 4;                      // projection buffers of 128 TMEM columns
constexpr int kEpiWarps = 16;                  // 4 per SM sub-partition
constexpr int kNormWarp = 2 + kEpiWarps;       // row-norm scales, ahead of the epilogue
constexpr int kFmThreads = 32 * (3 + kEpiWarps);
constexpr int kWarpBoxBytes = 32 * 64;         // one warp's [32 rows][32 bf16] output box
constexpr int kNumSMs = 148;

__device__ int g_fmap_status;                  // set to 1 by a kernel whose wait ran out

enum { FB_W = 0, FB_XF = 1, FB_XE = 5, FB_RS = 9, FB_UF = 13, FB_UE = 17, FB_NUM = 21 };

struct FmLayout {
    uint32_t w, x, rs, o, bar, tmem, total;
    int xbufs, obufs;
};

__host__ __device__ inline FmLayout fm_layout(int F)
{
    FmLayout l;
    l.xbufs = F <= 256 ? 4 : 2;
    l.obufs = F <= 256 ? 2 : 1;
    l.w = 0;                                   // F/32 packed sub-slices, resident
    l.x = (F / 32) * kSubBytes;
    l.rs = l.x + l.xbufs * kBoxBytes;          // per X slot: (1/|x|, 2 log2(1/|x|)) per row
    l.o = l.rs + l.xbufs * kRows * 8;          // epilogue warps x obufs staging boxes of 2 KiB
    l.bar = l.o + kEpiWarps * l.obufs * kWarpBoxBytes;
    l.tmem = l.bar + FB_NUM * 8;
    l.total = l.tmem + 16;
    return l;
}

struct FmParams {
    int F, m, ntiles;
    float a2[kMaxR];
    float b2[kMaxR];
};

// 64-byte swizzle of a [rows][64 B] box: 16-byte chunk c of row r sits at chunk
// c ^ ((r >> 1) & 3), the pattern TMA applies for CU_TENSOR_MAP_SWIZZLE_64B.
__device__ __forceinline__ uint32_t sw64_off(uint32_t row, uint32_t chunk)
{
    return row * 64u + ((chunk ^ ((row >> 1) & 3u)) << 4);
}

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
    const int ngroups = fp.F / 64;
    const int xbufs = L.xbufs;

    if (warp == 1) {
        tmem_alloc(tslot, 512);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < FB_NUM; ++i) mbar_init(&bar[i], 1);
        for (int s = 0; s < 4; ++s) {
            mbar_init(&bar[FB_XE + s], 2 + kEpiWarps);
        }
        for (int b = 0; b < kUBufs; ++b) mbar_init(&bar[FB_UE + b], kEpiWarps / 2);
        mbar_fence_init();
        tma_prefetch_desc(&tmx);
        tma_prefetch_desc(&tmw);
        tma_prefetch_desc(&tmo);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    Waiter wt;

    if (warp == 0) {
        if (lane == 0) {
            mbar_arrive_expect_tx(&bar[FB_W], (fp.F / 32) * kSubBytes);
            for (int n = 0; n < fp.F / 32; ++n)
                tma_load_2d(sm + L.w + n * kSubBytes, &tmw, &bar[FB_W], 0, n * 64);
            uint32_t ph_xe = 0;   // one phase bit per ring slot
            int it = 0;
            for (int tile = blockIdx.x; tile < fp.ntiles; tile += gridDim.x, ++it) {
                const int s = it % xbufs;
                if (it >= xbufs) {
                    uint32_t ph = (ph_xe >> s) & 1u;
                    wt.wait(&bar[FB_XE + s], ph);
                    ph_xe ^= 1u << s;
                }
                mbar_arrive_expect_tx(&bar[FB_XF + s], kBoxBytes);
                tma_load_2d(sm + L.x + s * kBoxBytes, &tmx, &bar[FB_XF + s], 0, tile * kRows);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            uint32_t ph_w = 0, ph_xf = 0;
            wt.wait(&bar[FB_W], ph_w);
            constexpr uint32_t idU = idesc_bf16(128, 128, 0, 0);
            // descriptors built once, stepped by adds (see the causal kernels)
            const uint64_t dx0 = sdesc(sbase + L.x, 16, 1024, kLayoutSW128);
            const uint64_t dw0 = sdesc(sbase + L.w, 16, 1024, kLayoutSW128);
            int it = 0, j = 0;
            for (int tile = blockIdx.x; tile < fp.ntiles; tile += gridDim.x, ++it) {
                const int s = it % xbufs;
                uint32_t ph = (ph_xf >> s) & 1u;
                wt.wait(&bar[FB_XF + s], ph);
                ph_xf ^= 1u << s;
                const uint64_t dx = dx0 + ((s * kBoxBytes) >> 4);
                for (int g = 0; g < ngroups; ++g, ++j) {
                    const int b = j % kUBufs;
                    if (j >= kUBufs) {
                        uint32_t pu = static_cast<uint32_t>((j / kUBufs - 1) & 1);
                        wt.wait(&bar[FB_UE + b], pu);
                    }
                    tc_fence_after();
                    const uint64_t dw = dw0 + ((g * kGroupBytes) >> 4);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_bf16(tmem + 128 * b, dx + 2 * kk, dw + 2 * kk, idU, kk > 0 ? 1u : 0u);
                    umma_commit(&bar[FB_UF + b]);
                }
                umma_commit(&bar[FB_XE + s]);
            }
        }
    } else if (warp == kNormWarp) {
        // (1/|x|, 2 log2(1/|x|)) of the 128 rows of each X tile, four rows per lane
        uint32_t ph_xf = 0;
        int it = 0;
        for (int tile = blockIdx.x; tile < fp.ntiles; tile += gridDim.x, ++it) {
            const int s = it % xbufs;
            uint32_t ph = (ph_xf >> s) & 1u;
            wt.wait(&bar[FB_XF + s], ph);
            ph_xf ^= 1u << s;
            float2* rs = reinterpret_cast<float2*>(sm + L.rs + s * kRows * 8);
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int row = 32 * r + lane;
                float inv, l2i;
                row_scale(sm + L.x + s * kBoxBytes + row * 128, inv, l2i);
                rs[row] = make_float2(inv, l2i);
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bar[FB_RS + s]);
                mbar_arrive(&bar[FB_XE + s]);
            }
        }
    } else {
        // epilogue warp ew: TMEM lanes 32*(warp%4) (rows of the tile); warps with pair = 0
        // take the even 64-feature groups, pair = 1 the odd ones (the two pairs of a
        // sub-partition work on different buffers, out of step); sub-slice `sub` of each
        // group (u at columns 64 sub, p at 64 sub + 32 of the group's buffer)
        const int ew = warp - 2, q = warp & 3, e = ew >> 2, pair = e >> 1, sub = e & 1;
        const uint32_t row = 32u * q + lane;
        const uint32_t trow = tmem + ((32u * q) << 16);
        const int obufs = L.obufs;
        uint32_t ph_rs = 0;
        int it = 0, jw = 0;
        for (int tile = blockIdx.x; tile < fp.ntiles; tile += gridDim.x, ++it) {
            const int s = it % xbufs;
            uint32_t ph = (ph_rs >> s) & 1u;
            wt.wait(&bar[FB_RS + s], ph);
            ph_rs ^= 1u << s;
            const float2 v = reinterpret_cast<const float2*>(sm + L.rs + s * kRows * 8)[row];
            const float inv = v.x, l2i = v.y;
            warp_arrive(&bar[FB_XE + s]);
            for (int g = pair; g < ngroups; g += 2, ++jw) {
                const int j = it * ngroups + g;
                const int b = j % kUBufs;
                uint32_t pu = static_cast<uint32_t>((j / kUBufs) & 1);
                wt.wait(&bar[FB_UF + b], pu);
                tc_fence_after();
                uint32_t ur[32], pr[32];
                const uint32_t c0 = trow + 128 * b + 64 * sub;
                tmem_ld32(c0, ur);
                tmem_ld32(c0 + 32, pr);
                tmem_wait_ld();
                reg_fence(ur);
                reg_fence(pr);
                tc_fence_before();
                warp_arrive(&bar[FB_UE + b]);
                const int f0 = 64 * g + 32 * sub;
                const int node = f0 / fp.m;
                const float a = fp.a2[node] * inv, bb = fp.b2[node] + l2i;
                uint32_t pk[16];
#pragma unroll
                for (int c = 0; c < 32; c += 2) {
                    const float x0 = __uint_as_float(pr[c]), x1 = __uint_as_float(pr[c + 1]);
                    pk[c >> 1] = pack_bf16(ex2(fmaf(a, __uint_as_float(ur[c]), bb)) * x0 * x0,
                                           ex2(fmaf(a, __uint_as_float(ur[c + 1]), bb)) * x1 * x1);
                }
                // this warp's staging box was stored obufs groups ago: its reads must be done
                if (lane == 0) {
                    if (obufs == 2)
                        bulk_wait_read<1>();
                    else
                        bulk_wait_read<0>();
                }
                __syncwarp();
                const uint32_t box = sbase + L.o + (ew * obufs + jw % obufs) * kWarpBoxBytes;
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    st_shared_v4(box + sw64_off(lane, c), pk[4 * c], pk[4 * c + 1], pk[4 * c + 2],
                                 pk[4 * c + 3]);
                fence_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(&tmo, sm + L.o + (ew * obufs + jw % obufs) * kWarpBoxBytes, f0,
                                 tile * kRows + 32 * q);
                    bulk_commit_group();
                }
            }
        }
        if (lane == 0) bulk_wait<0>();
    }
    wt.report(&g_fmap_status);
    drain_after_failure(wt.ok);
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

// [rows][cols] bf16, row stride cols*2 bytes, boxes of box_cols x box_rows; out-of-range
// rows read as zero and are not written.
bool map_2d(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_cols,
            uint32_t box_rows, CUtensorMapSwizzle swz)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t es[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
              es, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
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
    fp.m = P.m;
    fp.ntiles = static_cast<int>((n + kRows - 1) / kRows);
    for (int r = 0; r < kMaxR; ++r) {
        fp.a2[r] = P.a2[r];
        fp.b2[r] = P.b2[r];
    }
    void* status = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&status, g_fmap_status);
    if (e != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(status, 0, sizeof(int), st)) != cudaSuccess) return e;
    const size_t smem = fm_layout(F).total + 1024;
    e = cudaFuncSetAttribute(k_tc_feature_map, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const int grid = fp.ntiles < kNumSMs ? fp.ntiles : kNumSMs;
    TraceScope trace_("tc_feature_map", st);
    k_tc_feature_map<<<grid, kFmThreads, smem, st>>>(mx, mw, mo, fp);
    return cudaGetLastError();
}

}  // namespace slay
