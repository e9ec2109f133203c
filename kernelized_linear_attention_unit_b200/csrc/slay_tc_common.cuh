// slay_tc_common.cuh -- pieces shared by the tensor-core kernels: bounded waits, the
// per-row norm scale, shared-memory alignment and the tensor-map encoder.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "slay_exp2_poly.h"
#include "slay_tc_ptx.cuh"

namespace slay {
namespace tc {

constexpr uint64_t kWaitNs = 2000000000ull;   // bound of every mbarrier wait (2 s)

// A waiter that stops waiting (and reports) once any wait of this thread timed out.
// `where` keeps the first barrier that ran out: 0x10000 | its shared-memory offset, the
// value a kernel puts in the status word.
struct Waiter {
    bool ok = true;
    uint32_t where = 0;
    uint64_t limit = kWaitNs;   // bound of each wait (only a test hook shortens it)
    __device__ __forceinline__ void wait(uint64_t* bar, uint32_t& phase)
    {
        const bool done = mbar_wait(bar, phase, ok ? limit : 0);
        if (!done && ok) where = 0x10000u | (smem_u32(bar) & 0xFFFFu);
        ok = done && ok;
        phase ^= 1u;
    }
    // record the first failure in the status word (0 = every wait completed)
    __device__ __forceinline__ void report(int* status) const
    {
        if (!ok) atomicCAS(status, 0, static_cast<int>(where));
    }
};

// One arrival per warp (lane 0 after the warp has converged).
__device__ __forceinline__ void warp_arrive(uint64_t* bar)
{
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

__device__ __forceinline__ void drain_after_failure(bool ok)
{
    if (ok) return;
    const uint64_t t0 = global_timer_ns();
    while (global_timer_ns() - t0 < 20000000ull) {
    }
}

// Sum of squares of one 64-element bf16 row (128 bytes) -> (1/|x|, 2 log2(1/|x|)) with the
// 1e-12 norm guard.  The order of the elements does not matter, so the row's 16-byte chunks
// are read in the order of the 128-byte swizzle (chunk c ^ (row & 7) first): the lanes of
// a warp, one row each, then hit distinct banks.
__device__ __forceinline__ void row_scale(const unsigned char* row_ptr, uint32_t row, float& inv,
                                          float& l2inv2)
{
    const uint4* p = reinterpret_cast<const uint4*>(row_ptr);
    const uint32_t rot = row & 7u;
    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};   // independent partial sums: short FMA chains
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const uint4 w = p[c ^ rot];
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float lo = __uint_as_float(ws[e] << 16);
            const float hi = __uint_as_float(ws[e] & 0xFFFF0000u);
            acc[e] = fmaf(lo, lo, acc[e]);
            acc[e] = fmaf(hi, hi, acc[e]);
        }
    }
    const float s = (acc[0] + acc[1]) + (acc[2] + acc[3]);
    const float n = fmaxf(sqrtf(s), 1e-12f);
    inv = 1.0f / n;
    l2inv2 = -2.0f * __log2f(n);
}

// 2^x on the FMA pipe: j = round(x) by adding 1.5 * 2^23 (the sum's low mantissa bits hold
// j), f = x - j in [-1/2, 1/2], 2^f from the degree-3 minimax polynomial of
// slay_exp2_poly.h, and 2^j applied by adding j to the exponent field (the sum's bit
// pattern times 2^23 is j << 23 modulo 2^32).  x is clamped to [-125, 126] so the exponent
// field stays in range; the relative error is the polynomial's, below 1e-4.
__device__ __forceinline__ float ex2_poly(float x)
{
    x = fminf(fmaxf(x, -125.0f), 126.0f);
    const float t = __fadd_rn(x, 12582912.0f);
    const float f = __fsub_rn(x, __fsub_rn(t, 12582912.0f));
    float p = fmaf(SLAY_EXP2_C3, f, SLAY_EXP2_C2);
    p = fmaf(p, f, SLAY_EXP2_C1);
    p = fmaf(p, f, SLAY_EXP2_C0);
    return __uint_as_float(__float_as_uint(t) * 8388608u + __float_as_uint(p));
}

__device__ __forceinline__ unsigned char* aligned_smem(unsigned char* raw)
{
    return reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(raw) + 1023) &
                                            ~uintptr_t(1023));
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn()
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

// [rows][cols] bf16, row stride cols*2 bytes, boxes of box_cols x box_rows; out-of-range
// rows read as zero and are not written.
inline bool map_2d(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_cols,
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

}  // namespace tc
}  // namespace slay
