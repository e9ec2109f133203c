// slay_tc.cu -- tensor-core path (tcgen05 / TMEM / TMA, sm_100a) for bf16 inputs.
//
// Method: "SLAY: Geometry-Aware Spherical Linearized Attention with Yat-Kernel" (abstract;
// nubint.ai review, "Proposed method", steps 1-6).  The causal forward computes, per
// (b,h) sequence, out_i = phi(q_i)^T S_i / (phi(q_i)^T z_i + eps) with
// S_i = sum_{j<=i} phi(k_j) v_j^T, z_i = sum_{j<=i} phi(k_j), in 128-token tiles:
//
//   U   = X W_n^T                   projection of a 32-feature sub-slice n (its omega and
//                                   anchor rows), raw bf16 x; the 1/|x| scale is applied in
//                                   the epilogue: phi = exp2(a2 u/|x| + b2) (p/|x|)^2
//   P  += phiQ_t phiK_t^T           intra-tile scores, summed over 64-feature slices t
//   O  += phiQ_t S_t                inter-tile readout with the state entering the tile
//   O  += tril(P) V                 masked intra-tile term
//   [S|z] += phiK^T [V|1]           state update, z as extra accumulator columns (fp32 in
//                                   tensor memory), one N=80 MMA per K step
//
// Sequences are split into L-segments so that every SM has work: a first kernel computes
// each segment's own sum of phi(k) [v, 1]^T, the second starts each segment from the sum
// of the earlier segments' contributions and produces the outputs.  Neither kernel waits on
// another CTA.
//
// Both kernels are warp-specialised: warp 0 issues TMA copies, warps 1, 10 and 11 issue
// tcgen05 MMAs (one elected thread each: the issue rate of a single thread, not the tensor
// pipe, limits narrow MMAs), warps 2-5 and 6-9 are two epilogue groups (one row of a 128-row
// tile per thread, one TMEM lane each).  In the output kernel the denominator is an extra
// accumulator column: O = [P | phiQ] . [[V | 1]; [S | z]], so no per-element dot product
// with z is needed and the phi(q) group never waits for the end of a tile.  Hand-offs go through mbarriers.  Every wait is
// bounded in time; a timeout sets an error word in the workspace header, later waits give
// up at once, and the CTA drains before releasing its memory.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>

#include "slay_tc.h"
#include "slay_tc_ptx.cuh"
#include "slay_tc_common.cuh"

namespace slay {

using namespace tc;

namespace {

constexpr int kTile = 128;                 // tokens per tile (MMA M)
constexpr int kSlice = 64;                 // features per phi tile (K of the P MMA)
constexpr int kSub = 32;                   // features per projection (N = 64 with anchors)
constexpr int kTileBytes = kTile * 128;    // one [128 rows][64 bf16] swizzled tile = 16 KiB
constexpr int kWBytes = 64 * 128;          // one projection operand [64 rows][64 bf16] = 8 KiB
constexpr int kWSlots = 3;                 // output kernel: 3 x 8 KiB projection operands
constexpr int kThreads = 384;              // 12 warps (state kernel)
constexpr int kOutThreads = 512;           // 16 warps (output kernel)
constexpr int kOnesBytes = kTileBytes;     // [128][64] bf16 ones: the z columns of [V | 1]
constexpr int kNumSMs = 148;

// TMEM column map (one CTA per SM, 512 columns allocated).
constexpr uint32_t kColU0 = 0;     // 64: q-side projection (32 u | 32 p)
constexpr uint32_t kColU1 = 64;    // 64: k-side projection
constexpr uint32_t kColP = 128;    // 128: intra-tile scores
constexpr uint32_t kColO = 256;    // 80 : output [numerator | denominator] (denominator column 64)
constexpr uint32_t kColS = 336;    // 2 x 80: state [S | z], feature halves (z in column 64)
constexpr int kStBytes = 80 * 128; // [S | z] rows of one 64-feature slice: 80 columns x 64 features bf16

// -------------------------------------------------------------- barriers
enum {
    B_QK_FULL = 0, B_QK_EMPTY, B_V_FULL, B_V_EMPTY,
    B_W_FULL0, B_W_FULL1, B_W_FULL2, B_W_FULL3,
    B_W_EMPTY0, B_W_EMPTY1, B_W_EMPTY2, B_W_EMPTY3,
    B_U_FULL0, B_U_FULL1, B_U_EMPTY0, B_U_EMPTY1,
    B_PQ_FULL0, B_PQ_FULL1, B_PQ_EMPTY0, B_PQ_EMPTY1,
    B_PK_FULL, B_P_FULL, B_PSM_FULL, B_TILE_DONE, B_O_EMPTY, B_SBF_READY,
    B_PK_FREE0, B_PK_FREE1, B_PK_FULL1, B_PK_FULL2, B_PK_FULL3,
    NUM_BARS
};

struct SmemOut {
    uint32_t w, q, k, v, ones, phik, phiq, st, bar, tmem, total;
};

// Output kernel: st = the state entering the tile in bf16, [S | z | 0] with 80 columns, as
// the B operand of the readout (MN-major, no swizzle: 8x8 core matrices, K groups of 8
// features 128 bytes apart, N groups of 8 columns F*16 bytes apart).
__host__ __device__ inline SmemOut smem_out_layout(int F)
{
    SmemOut s;
    s.w = 0;
    s.q = kWSlots * kWBytes;
    s.k = s.q + kTileBytes;
    s.v = s.k + kTileBytes;
    s.ones = s.v + kTileBytes;                         // right after V: fixed offset from it
    s.phik = s.ones + kOnesBytes;
    s.phiq = s.phik + (F / kSlice) * kTileBytes;
    s.st = s.phiq + 2 * kTileBytes;
    s.bar = s.st + (F / kSlice) * kStBytes;
    s.tmem = s.bar + NUM_BARS * 8;
    s.total = s.tmem + 16;
    return s;
}

// State kernel: two 16 KiB projection operands (64 features each); k tiles and phi(k) are
// double buffered (the projections of tile i+1 and its phi(k) proceed while tile i's state
// update runs); V, needed only by that update, has one buffer.
constexpr int kWStateBytes = 2 * kWBytes;
struct SmemState {
    uint32_t w, k, v, ones, phik, bar, tmem, total;
};

__host__ __device__ inline SmemState smem_state_layout(int F)
{
    SmemState s;
    s.w = 0;
    s.k = 2 * kWStateBytes;                 // 2 buffers
    s.v = s.k + 2 * kTileBytes;
    s.ones = s.v + kTileBytes;              // right after V: fixed offset from it
    s.phik = s.ones + kOnesBytes;           // 2 buffers of F/64 tiles
    s.bar = s.phik + 2 * (F / kSlice) * kTileBytes;
    s.tmem = s.bar + NUM_BARS * 8;
    s.total = s.tmem + 16;
    return s;
}

struct Seg {
    int bh, seg, t_begin, t_end;
};

// Segment `seg` of sequence bh: ntiles / nseg tiles each, the first ntiles % nseg segments one
// more.  The longer segments come first because a later segment's output CTA also sums the
// state of all earlier segments before its first tile.
__device__ __forceinline__ Seg segment_of(int index, int nseg, int ntiles)
{
    Seg s;
    s.bh = index / nseg;
    s.seg = index % nseg;
    const int q = ntiles / nseg, r = ntiles % nseg;
    s.t_begin = s.seg * q + (s.seg < r ? s.seg : r);
    s.t_end = s.t_begin + q + (s.seg < r ? 1 : 0);
    return s;
}

constexpr int kMaxSlices = 256 / kSlice;

struct KParams {
    int L, F, nseg, ntiles;   // F: the features of this launch (one chunk of at most 256)
    int all_segs;      // state kernel: 1 = every segment (bidirectional), 0 = all but the last
    float eps;
    float a2[kMaxSlices];   // per 64-feature slice (m % 64 == 0): the scales of its node
    float b2[kMaxSlices];
    // Feature chunks.  Scores, readouts, numerators and denominators are sums over features,
    // so a wider map runs as several chunks whose per-row numerators [rows][64] and
    // denominators [rows] (fp32) meet in part_num / part_den: acc_in adds the earlier
    // chunks' sums before the division, acc_out stores the sums there instead of the output.
    int acc_in, acc_out;
    float* part_num;
    float* part_den;
    // The state entering the sequence (causal forward continued from a state): S [bh][f][64]
    // and z [bh][f] of this launch's feature chunk, bh strides s_stride / z_stride floats;
    // null for a zero state.
    const float* s_in;
    const float* z_in;
    int s_stride, z_stride;
};

// The output row `g` (global row index over [BH][L]) from its numerator o0|o1 (64 fp32 bit
// patterns) and denominator d: out = num / (den + eps) in bf16 and den, or, with acc_out,
// the chunk's running sums.
__device__ __forceinline__ void finish_row(const KParams& kp, uint32_t (&o0)[32], uint32_t (&o1)[32],
                                           float d, size_t g, __nv_bfloat16* out, float* den)
{
    if (kp.acc_in) {
        const float4* src = reinterpret_cast<const float4*>(kp.part_num + g * 64);
#pragma unroll
        for (int q = 0; q < 16; ++q) {
            const float4 a = src[q];
            uint32_t* o = q < 8 ? o0 : o1;
            const int c = 4 * (q & 7);
            o[c] = __float_as_uint(__uint_as_float(o[c]) + a.x);
            o[c + 1] = __float_as_uint(__uint_as_float(o[c + 1]) + a.y);
            o[c + 2] = __float_as_uint(__uint_as_float(o[c + 2]) + a.z);
            o[c + 3] = __float_as_uint(__uint_as_float(o[c + 3]) + a.w);
        }
        d += kp.part_den[g];
    }
    if (kp.acc_out) {
        float4* dst = reinterpret_cast<float4*>(kp.part_num + g * 64);
#pragma unroll
        for (int q = 0; q < 16; ++q) {
            const uint32_t* o = q < 8 ? o0 : o1;
            const int c = 4 * (q & 7);
            dst[q] = make_float4(__uint_as_float(o[c]), __uint_as_float(o[c + 1]),
                                 __uint_as_float(o[c + 2]), __uint_as_float(o[c + 3]));
        }
        kp.part_den[g] = d;
        return;
    }
    const float rz = 1.0f / (d + kp.eps);
    uint4* dst = reinterpret_cast<uint4*>(out + g * 64);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const uint32_t* o = q < 4 ? o0 : o1;
        const int c = 8 * (q & 3);
        dst[q] = make_uint4(pack_bf16(__uint_as_float(o[c]) * rz, __uint_as_float(o[c + 1]) * rz),
                            pack_bf16(__uint_as_float(o[c + 2]) * rz, __uint_as_float(o[c + 3]) * rz),
                            pack_bf16(__uint_as_float(o[c + 4]) * rz, __uint_as_float(o[c + 5]) * rz),
                            pack_bf16(__uint_as_float(o[c + 6]) * rz, __uint_as_float(o[c + 7]) * rz));
    }
    if (den) den[g] = d;
}

// finish_row with the chunk mode fixed at compile time (no code, and no registers, for the
// modes a launch does not use)
template <bool kIn, bool kOut>
__device__ __forceinline__ void finish_row_t(const KParams& kp, uint32_t (&o0)[32], uint32_t (&o1)[32],
                                             float d, size_t g, __nv_bfloat16* out, float* den)
{
    if (kIn) {
        const float4* src = reinterpret_cast<const float4*>(kp.part_num + g * 64);
#pragma unroll
        for (int q = 0; q < 16; ++q) {
            const float4 a = src[q];
            uint32_t* o = q < 8 ? o0 : o1;
            const int c = 4 * (q & 7);
            o[c] = __float_as_uint(__uint_as_float(o[c]) + a.x);
            o[c + 1] = __float_as_uint(__uint_as_float(o[c + 1]) + a.y);
            o[c + 2] = __float_as_uint(__uint_as_float(o[c + 2]) + a.z);
            o[c + 3] = __float_as_uint(__uint_as_float(o[c + 3]) + a.w);
        }
        d += kp.part_den[g];
    }
    if (kOut) {
        float4* dst = reinterpret_cast<float4*>(kp.part_num + g * 64);
#pragma unroll
        for (int q = 0; q < 16; ++q) {
            const uint32_t* o = q < 8 ? o0 : o1;
            const int c = 4 * (q & 7);
            dst[q] = make_float4(__uint_as_float(o[c]), __uint_as_float(o[c + 1]),
                                 __uint_as_float(o[c + 2]), __uint_as_float(o[c + 3]));
        }
        kp.part_den[g] = d;
        return;
    }
    const float rz = 1.0f / (d + kp.eps);
    uint4* dst = reinterpret_cast<uint4*>(out + g * 64);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const uint32_t* o = q < 4 ? o0 : o1;
        const int c = 8 * (q & 3);
        dst[q] = make_uint4(pack_bf16(__uint_as_float(o[c]) * rz, __uint_as_float(o[c + 1]) * rz),
                            pack_bf16(__uint_as_float(o[c + 2]) * rz, __uint_as_float(o[c + 3]) * rz),
                            pack_bf16(__uint_as_float(o[c + 4]) * rz, __uint_as_float(o[c + 5]) * rz),
                            pack_bf16(__uint_as_float(o[c + 6]) * rz, __uint_as_float(o[c + 7]) * rz));
    }
    if (den) den[g] = d;
}

// v[t] for a slice index t < kMaxSlices, by selects (an indexed parameter array would be
// copied to local memory)
__device__ __forceinline__ float slice_val(const float (&v)[kMaxSlices], int t)
{
    static_assert(kMaxSlices == 4, "slice_val selects among four");
    return t < 2 ? (t == 0 ? v[0] : v[1]) : (t == 2 ? v[2] : v[3]);
}

// phi of one 32-feature sub-slice from registers holding u (32) and p (32) of this row:
// phi_j = exp2(a u_j + b) p_j^2, a = a2[r]/|x|, b = b2[r] + 2 log2(1/|x|).  Stores the 32
// bf16 values as chunks [4*half, 4*half+4) of row `row` of the swizzled tile at tile_addr.
// With zs != nullptr returns sum_j phi_j zs[j] (the inter-tile denominator term).
template <bool kPoly = false>
__device__ __forceinline__ float phi_sub_epilogue(const uint32_t (&ur)[32], const uint32_t (&pr)[32],
                                                  float a, float b, uint32_t tile_addr,
                                                  uint32_t row, int half, const float* zs)
{
    float dz = 0.0f;
    uint32_t pk[16];
#pragma unroll
    for (int j = 0; j < 32; j += 2) {
        const float p0 = __uint_as_float(pr[j]), p1 = __uint_as_float(pr[j + 1]);
        // with kPoly one exponential in four goes to the FMA pipe: the special-function
        // unit's queue is shared with the shared-memory and barrier traffic that paces these
        // kernels (the k side, which has the registers for it)
        const float2 y = ffma2(make_float2(a, a), make_float2(__uint_as_float(ur[j]), __uint_as_float(ur[j + 1])),
                               make_float2(b, b));
        const float2 pp = make_float2(p0, p1);
        const float2 e = make_float2(ex2(y.x), (kPoly && (j & 2)) ? ex2_poly(y.y) : ex2(y.y));
        const float2 ff = fmul2(fmul2(e, pp), pp);   // packed two-wide fp32
        const float f0 = ff.x, f1 = ff.y;
        if (zs) {
            dz = fmaf(f0, zs[j], dz);
            dz = fmaf(f1, zs[j + 1], dz);
        }
        pk[j >> 1] = pack_bf16(f0, f1);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q)
        st_shared_v4(tile_addr + sw128_off(row, 4 * half + q), pk[4 * q], pk[4 * q + 1],
                     pk[4 * q + 2], pk[4 * q + 3]);
    return dz;
}

// Shared-memory descriptors are built once per operand buffer and stepped with plain adds:
// the start-address field holds addr >> 4 in the low bits and every operand lies below
// 256 KiB, so adding bytes >> 4 never carries into the next field.  (Rebuilding a
// descriptor per MMA puts a chain of dependent integer ops in front of every issue and
// halves the single issuing thread's MMA rate.)
__device__ __forceinline__ uint64_t desc_add(uint64_t d, uint32_t bytes) { return d + (bytes >> 4); }

// K-major 128-byte-swizzled operand at `addr` (rows 128 bytes apart, 8-row groups 1 KiB apart)
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t addr) { return sdesc(addr, 16, 1024, kLayoutSW128); }

// U (64 columns: 32 u then 32 p) = X [128 x 64] . W_n^T [64 x 64]; dx, dw: K-major descriptors
__device__ __forceinline__ void issue_projection(uint32_t d_tmem, uint64_t dx, uint64_t dw)
{
    constexpr uint32_t id = idesc_bf16(128, 64, 0, 0);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) umma_bf16(d_tmem, dx + 2 * kk, dw + 2 * kk, id, kk > 0 ? 1u : 0u);
}

// [S|z]_h (+)= phiK_h^T [V | 1] for feature half h: phiK as an MN-major A operand
// (128 features = two 64-feature sub-tiles 16 KiB apart); B = V as an MN-major operand of
// width 80 whose columns 64..79 come from the ones tile at LBO (= ones - V) bytes.
// dphik: desc_phik(phik base), dv: desc_v(v, ones) (see below)
__device__ __forceinline__ void issue_state_half(uint32_t tmem, uint32_t colS, uint64_t dphik,
                                                 uint64_t dv, int h, bool first)
{
    constexpr uint32_t idS = idesc_bf16(128, 80, 1, 1);
    const uint64_t da = desc_add(dphik, 2 * h * kTileBytes);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
        umma_bf16(tmem + colS + 80 * h, da + 128 * kk, dv + 128 * kk, idS,
                  (first && kk == 0) ? 0u : 1u);
}

// phi(k) slices as the MN-major A operand of the state update (two 64-feature sub-tiles
// 16 KiB apart), and [V | 1] as an MN-major B operand (the ones tile at LBO = ones - v)
__device__ __forceinline__ uint64_t desc_phik(uint32_t phik) { return sdesc(phik, kTileBytes, 1024, kLayoutSW128); }
__device__ __forceinline__ uint64_t desc_v(uint32_t v, uint32_t ones) { return sdesc(v, ones - v, 1024, kLayoutSW128); }

__device__ __forceinline__ void fill_ones(unsigned char* ones)
{
    uint32_t* p = reinterpret_cast<uint32_t*>(ones);
    for (int i = threadIdx.x; i < kOnesBytes / 4; i += blockDim.x) p[i] = 0x3F803F80u;  // bf16 1.0
}


// Programmatic dependent launch: a grid launched with programmatic stream serialization may
// start before the grid ahead of it in the stream has finished; griddep_wait blocks until that
// grid has completed and its memory operations are visible (at once when there is none).
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;"); }

// State kernel projection order: the k-th projection of the li-th tile of a segment covers
// the 64-feature slice state_slice(li, k) and reads its operand from slot k % 2.  With four
// slices the odd tiles take them in the order 2, 3, 0, 1, so each slot's last slice of a tile
// is its first of the next and only two of the four operands are reloaded per tile; with two
// slices the slots never change.
__device__ __forceinline__ int state_slice(int li, int k, int NT)
{
    return (NT == 4 && (li & 1)) ? (k ^ 2) : k;
}
// whether projection (li, k) needs its slot (re)loaded (the slot held another slice before)
__device__ __forceinline__ bool state_reload(int li, int k, int NT)
{
    if (li == 0 && k < 2) return true;
    const int pli = k >= 2 ? li : li - 1, pk = k >= 2 ? k - 2 : k + NT - 2;
    return state_slice(pli, pk, NT) != state_slice(li, k, NT);
}

// ------------------------------------------------------------ state kernel
// grid = BH * (nseg - 1) (causal: the last segment's sum is never needed) or BH * nseg
// (bidirectional): segment seg of sequence bh writes
//   ws_S[bh][seg][f][e] = sum_{t in seg} phi(k_t)_f v_t[e],  ws_z[bh][seg][f] = sum phi(k_t)_f
// Projections are 64 features wide (N = 128: two packed 32-feature operands), double
// buffered in TMEM (warp 1 issues them); epilogue group g takes the projections k with
// k % 2 == g.  Tile i uses k and phi(k) buffer (i - first) % 2; warp 11 loads v and issues
// the state updates.
// kStorePhi: also write phi(k) of every tile (bf16, [BH][L][F]) through TMA for the output
// kernel that reads it instead of recomputing it; warp 10 issues those stores.
template <bool kStorePhi>
__global__ void __launch_bounds__(kThreads, 1)
k_tc_causal_state(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                  const __grid_constant__ CUtensorMap tmw, const __grid_constant__ CUtensorMap tmpk,
                  KParams kp, float* __restrict__ wsS, float* __restrict__ wsZ,
                  int* __restrict__ err)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* sm = aligned_smem(smem_raw);
    const SmemState L = smem_state_layout(kp.F);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + L.bar);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + L.tmem);
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int NT = kp.F / kSlice;
    const uint32_t phik_bytes = NT * kTileBytes;
    const Seg sg = kp.all_segs ? segment_of(blockIdx.x, kp.nseg, kp.ntiles)
                               : segment_of(blockIdx.x + blockIdx.x / (kp.nseg - 1), kp.nseg, kp.ntiles);
    // the readout kernel that follows may be scheduled now (onto SMs this grid leaves free,
    // then onto those its CTAs release); it waits for this grid's results before reading them
    griddep_launch_dependents();
    constexpr uint32_t kColUS = 0;     // 2 x 128: projections
    constexpr uint32_t kColST = 256;   // F: the transposed state, lanes 0-63 S^T, 64-127 z
    // barrier roles here: KF(b) / KE(b) the k buffers; VF / VE the V buffer; TD(b) = the
    // state update of a tile in phi(k) buffer b is done; PKF(b) = all phiK of a tile in
    // buffer b written (one barrier per buffer, so no waiter can fall two phases behind)
    auto KF = [bar](int b) { return &bar[b ? B_V_FULL : B_QK_FULL]; };
    auto KE = [bar](int b) { return &bar[b ? B_V_EMPTY : B_QK_EMPTY]; };
    uint64_t* VF = &bar[B_PQ_FULL0];
    uint64_t* VE = &bar[B_PQ_EMPTY0];
    uint64_t* TD = &bar[B_O_EMPTY];    // B_O_EMPTY, B_SBF_READY
    uint64_t* ST = &bar[B_PK_FREE0];   // ST(b): the phi(k) store from buffer b has read it
    auto PKF = [bar](int b) { return &bar[b ? B_PK_FULL1 : B_PK_FULL]; };
    if (warp == 1) {
        tmem_alloc(tslot, 512);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < NUM_BARS; ++i) mbar_init(&bar[i], 1);
        mbar_init(KE(0), 1 + 8);
        mbar_init(KE(1), 1 + 8);
        mbar_init(&bar[B_U_EMPTY0], 4);
        mbar_init(&bar[B_U_EMPTY1], 4);
        mbar_init(&bar[B_PK_FULL], 8);
        mbar_init(&bar[B_PK_FULL1], 8);
        mbar_fence_init();
        tma_prefetch_desc(&tmk);
        tma_prefetch_desc(&tmv);
        tma_prefetch_desc(&tmw);
        if (kStorePhi) tma_prefetch_desc(&tmpk);
    }
    fill_ones(sm + L.ones);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    Waiter wt;

    if (warp == 0) {
        // k tiles (two buffers) and the projection operands
        if (lane == 0) {
            uint32_t ph_ke = 0, ph_we = 0x3u;  // both operand slots start free
            for (int j = 0; j < 2 && sg.t_begin + j < sg.t_end; ++j) {
                mbar_arrive_expect_tx(KF(j), kTileBytes);
                tma_load_3d(sm + L.k + j * kTileBytes, &tmk, KF(j), 0, (sg.t_begin + j) * kTile, sg.bh);
            }
            for (int tile = sg.t_begin; tile < sg.t_end; ++tile) {
                const int li = tile - sg.t_begin, kb = li & 1;
                for (int k = 0; k < NT; ++k) {
                    if (!state_reload(li, k, NT)) continue;   // the slot already holds it
                    const int slot = k & 1, n = state_slice(li, k, NT);
                    uint32_t ph = (ph_we >> slot) & 1u;
                    wt.wait(&bar[B_W_EMPTY0 + slot], ph);
                    ph_we ^= (1u << slot);
                    mbar_arrive_expect_tx(&bar[B_W_FULL0 + slot], kWStateBytes);
                    unsigned char* dst = sm + L.w + slot * kWStateBytes;
                    tma_load_2d(dst, &tmw, &bar[B_W_FULL0 + slot], 0, (2 * n) * 64);
                    tma_load_2d(dst + kWBytes, &tmw, &bar[B_W_FULL0 + slot], 0, (2 * n + 1) * 64);
                }
                // k of tile + 2 into this tile's buffer once its projections and norms are done
                if (tile + 2 < sg.t_end) {
                    uint32_t pk = (ph_ke >> kb) & 1u;
                    wt.wait(KE(kb), pk);
                    ph_ke ^= 1u << kb;
                    mbar_arrive_expect_tx(KF(kb), kTileBytes);
                    tma_load_3d(sm + L.k + kb * kTileBytes, &tmk, KF(kb), 0, (tile + 2) * kTile, sg.bh);
                }
            }
        }
    } else if (warp == 11) {
        // v tiles (one buffer, refilled once the previous tile's state update has read it)
        // and the state updates, issued here so that they never hold up the projections
        if (lane == 0) {
            uint32_t ph_ve = 0, ph_vf = 0, ph_pk = 0;   // ph_pk: bit per phi(k) buffer
            // [S | z]^T += [V | 1]^T phi(k): M = 128 (v columns, then the ones tile at LBO),
            // N = F (all of phi(k) at once: its 64-feature tiles 16 KiB apart), K = 128 tokens
            const uint32_t idT = idesc_bf16(128, static_cast<uint32_t>(kp.F), 1, 1);
            const uint64_t dph0 = desc_phik(sbase + L.phik), dv = desc_v(sbase + L.v, sbase + L.ones);
            for (int tile = sg.t_begin; tile < sg.t_end; ++tile) {
                const int b = (tile - sg.t_begin) & 1;
                if (tile > sg.t_begin) wt.wait(VE, ph_ve);
                mbar_arrive_expect_tx(VF, kTileBytes);
                tma_load_3d(sm + L.v, &tmv, VF, 0, tile * kTile, sg.bh);
                {
                    uint32_t pp = (ph_pk >> b) & 1u;
                    wt.wait(PKF(b), pp);
                    ph_pk ^= 1u << b;
                }
                wt.wait(VF, ph_vf);
                tc_fence_after();
                const uint64_t dph = desc_add(dph0, b * phik_bytes);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    umma_bf16(tmem + kColST, dv + 128 * kk, dph + 128 * kk, idT,
                              (tile == sg.t_begin && kk == 0) ? 0u : 1u);
                umma_commit(VE);
                umma_commit(&TD[b]);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            uint32_t ph_kf = 0, ph_wf = 0, ph_ue0 = 1, ph_ue1 = 1;  // ph_kf: bit per buffer
            constexpr uint32_t idU = idesc_bf16(128, 128, 0, 0);
            const uint64_t dk0 = desc_kmajor(sbase + L.k), dw0 = desc_kmajor(sbase + L.w);
            // the projections only (warp 11 issues the state updates): the phi(k) warps never
            // wait for a projection behind an update
            // The first MMA of a launch takes ~7k cycles; a throwaway one issued now (operands
            // whatever the buffers hold) spends them while the first k tile and W load.  It
            // writes projection buffer 0, which this thread's first projection into it
            // overwrites (an MMA without accumulate, ordered after it).
            if (sg.t_end > sg.t_begin) umma_bf16(tmem + kColUS, dk0, dw0, idU, 0u);
            for (int tile = sg.t_begin; tile < sg.t_end; ++tile) {
                const int b = (tile - sg.t_begin) & 1;
                {
                    {
                        uint32_t pk = (ph_kf >> b) & 1u;
                        wt.wait(KF(b), pk);
                        ph_kf ^= 1u << b;
                    }
                    const uint64_t dk = desc_add(dk0, b * kTileBytes);
                    const int li = tile - sg.t_begin;
                    for (int k = 0; k < NT; ++k) {
                        const int slot = k & 1;
                        if (state_reload(li, k, NT)) {
                            uint32_t ph = (ph_wf >> slot) & 1u;
                            wt.wait(&bar[B_W_FULL0 + slot], ph);
                            ph_wf ^= (1u << slot);
                        }
                        const int ub = k & 1;
                        wt.wait(&bar[B_U_EMPTY0 + ub], ub ? ph_ue1 : ph_ue0);
                        tc_fence_after();
                        const uint64_t dw = desc_add(dw0, slot * kWStateBytes);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            umma_bf16(tmem + kColUS + 128 * ub, dk + 2 * kk, dw + 2 * kk, idU, kk > 0 ? 1u : 0u);
                        umma_commit(&bar[B_U_FULL0 + ub]);
                        // the slot is released when its next use reloads it
                        if (k + 2 < NT ? state_reload(li, k + 2, NT) : state_reload(li + 1, k + 2 - NT, NT))
                            umma_commit(&bar[B_W_EMPTY0 + slot]);
                    }
                    umma_commit(KE(b));
                }
            }
        }
    } else if (kStorePhi && warp == 10) {
        if (lane == 0) {
            uint32_t ph_pk = 0;
            for (int tile = sg.t_begin; tile < sg.t_end; ++tile) {
                const int b = (tile - sg.t_begin) & 1, li = tile - sg.t_begin;
                {   // all of phi(k) of this tile written
                    uint32_t pp = (ph_pk >> b) & 1u;
                    wt.wait(PKF(b), pp);
                    ph_pk ^= 1u << b;
                }
                // the next tile's operand reloads go first through this CTA's copy engine:
                // the projections wait for them, while this store has a tile of slack
                if (NT == 4 && tile + 1 < sg.t_end) {
                    // reload of slot s in tile j >= 1 is that slot's completion j + 1
                    for (int sl = 0; sl < 2; ++sl) {
                        uint32_t pw = static_cast<uint32_t>(li + 2) & 1u;
                        wt.wait(&bar[B_W_FULL0 + sl], pw);
                    }
                }
                for (int t = 0; t < NT; ++t)
                    tma_store_3d(&tmpk, sm + L.phik + b * phik_bytes + t * kTileBytes, kSlice * t,
                                 tile * kTile, sg.bh);
                bulk_commit_group();
                bulk_wait_read<0>();
                mbar_arrive(&ST[b]);
            }
            bulk_wait<0>();
        }
    } else if (warp < 10) {
        const int grp = (warp >= 6) ? 1 : 0;
        const int sp = warp & 3;
        const uint32_t row = 32u * sp + lane;
        const uint32_t trow = tmem + ((32u * sp) << 16);
        uint32_t ph_kf = 0, ph_uf = 0, ph_td = 0;
        for (int tile = sg.t_begin; tile < sg.t_end; ++tile) {
            const int li = tile - sg.t_begin, b = li & 1;
            {
                uint32_t pk = (ph_kf >> b) & 1u;
                wt.wait(KF(b), pk);
                ph_kf ^= 1u << b;
            }
            float inv, l2i;
            row_scale(sm + L.k + b * kTileBytes + row * 128, row, inv, l2i);
            warp_arrive(KE(b));
            if (li >= 2) {   // phiK buffer b free again (update and store of tile li-2 done)
                uint32_t pt = (ph_td >> b) & 1u, ps = pt;   // wait() flips its argument
                wt.wait(&TD[b], pt);
                if (kStorePhi) wt.wait(&ST[b], ps);
                ph_td ^= (1u << b);
            }
            for (int k = grp; k < NT; k += 2) {
                const int n = state_slice(li, k, NT);
                wt.wait(&bar[B_U_FULL0 + grp], ph_uf);
                tc_fence_after();
                const float a = slice_val(kp.a2, n) * inv, bb = slice_val(kp.b2, n) + l2i;
                const uint32_t col = kColUS + 128 * grp;
                uint32_t ua[32], pa[32], ub[32], pb[32];
                tmem_ld32(trow + col, ua);
                tmem_ld32(trow + col + 32, pa);
                tmem_ld32(trow + col + 64, ub);
                tmem_ld32(trow + col + 96, pb);
                tmem_wait_ld();
                reg_fence(ua);
                reg_fence(pa);
                reg_fence(ub);
                reg_fence(pb);
                tc_fence_before();
                warp_arrive(&bar[B_U_EMPTY0 + grp]);
                const uint32_t tile_addr = sbase + L.phik + b * phik_bytes + n * kTileBytes;
                phi_sub_epilogue<true>(ua, pa, a, bb, tile_addr, row, 0, nullptr);
                phi_sub_epilogue<true>(ub, pb, a, bb, tile_addr, row, 1, nullptr);
            }
            fence_async_smem();
            warp_arrive(PKF(b));
        }
        // the segment's sums once the last update is done (it follows all earlier ones)
        {
            const int lb = (sg.t_end - 1 - sg.t_begin) & 1;
            uint32_t pt = (ph_td >> lb) & 1u;
            wt.wait(&TD[lb], pt);
        }
        tc_fence_after();
        const size_t segidx = static_cast<size_t>(sg.bh) * kp.nseg + sg.seg;
        if (sp < 2) {
            // S[f][e] = S^T[e][f]: lane e of quadrants 0, 1; group g takes features
            // [g F/2, (g+1) F/2), 32 at a time (a warp's stores: 32 consecutive e of one f)
            const int fh = kp.F / 2;
            for (int f0 = grp * fh; f0 < (grp + 1) * fh; f0 += 32) {
                uint32_t r[32];
                tmem_ld32(trow + kColST + f0, r);
                tmem_wait_ld();
                reg_fence(r);
#pragma unroll
                for (int j = 0; j < 32; ++j) wsS[(segidx * kp.F + f0 + j) * 64 + row] = __uint_as_float(r[j]);
            }
        } else if (sp == 2 && grp == 0) {
            // z: every lane of quadrant 2 holds it (the ones rows); lane 0 writes it
            for (int f0 = 0; f0 < kp.F; f0 += 32) {
                uint32_t r[32];
                tmem_ld32(trow + kColST + f0, r);
                tmem_wait_ld();
                reg_fence(r);
                if (lane == 0) {
                    float4* dst = reinterpret_cast<float4*>(wsZ + segidx * kp.F + f0);
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        dst[q] = make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]),
                                             __uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3]));
                }
            }
        }
    }
    wt.report(err);
    drain_after_failure(wt.ok);
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

// ----------------------------------------------------------- output kernel
// Row f of the state copy [S | z]: columns 0..63 = S[f][:], column 64 = z[f], 65..71 = 0, in
// the no-swizzle MN-major layout (core matrix (n/8, f/8), row f%8, 16 bytes per row).
// Nine 16-byte stores; a warp's 32 consecutive features fill 512 contiguous bytes.
__device__ __forceinline__ void write_state_row(uint32_t st, int F, int f, const float* s, float z)
{
    const uint32_t base = st + (f >> 3) * 128 + (f & 7) * 16;
    const uint32_t sbo = static_cast<uint32_t>(F) * 16;
#pragma unroll
    for (int g = 0; g < 8; ++g)
        st_shared_v4(base + g * sbo, pack_bf16(s[8 * g], s[8 * g + 1]), pack_bf16(s[8 * g + 2], s[8 * g + 3]),
                     pack_bf16(s[8 * g + 4], s[8 * g + 5]), pack_bf16(s[8 * g + 6], s[8 * g + 7]));
    st_shared_v4(base + 8 * sbo, pack_bf16(z, 0.0f), 0u, 0u, 0u);
}

// Row f of the [S | z] copy (the layout of write_state_row) from the fp32 bit patterns of
// S[f][0..32) (s0) and S[f][32..64) (s1).
__device__ __forceinline__ void write_state_row_u(uint32_t st, int F, int f, const uint32_t (&s0)[32],
                                                  const uint32_t (&s1)[32], float z)
{
    const uint32_t base = st + (f >> 3) * 128 + (f & 7) * 16;
    const uint32_t sbo = static_cast<uint32_t>(F) * 16;
#pragma unroll
    for (int g = 0; g < 8; ++g) {
        const uint32_t* s = g < 4 ? s0 : s1;
        const int c = 8 * (g & 3);
        st_shared_v4(base + g * sbo,
                     pack_bf16(__uint_as_float(s[c]), __uint_as_float(s[c + 1])),
                     pack_bf16(__uint_as_float(s[c + 2]), __uint_as_float(s[c + 3])),
                     pack_bf16(__uint_as_float(s[c + 4]), __uint_as_float(s[c + 5])),
                     pack_bf16(__uint_as_float(s[c + 6]), __uint_as_float(s[c + 7])));
    }
    st_shared_v4(base + 8 * sbo, pack_bf16(z, 0.0f), 0u, 0u, 0u);
}

__device__ __forceinline__ uint32_t ld_shared_u32(uint32_t addr)
{
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}

// The sum over segments [0, nseg) of sequence bh of the per-segment sums S [BH][nseg][F][64]
// and z [BH][nseg][F], by all kOutThreads threads with 16-byte coalesced loads (one thread
// per piece, segments two at a time): S into sacc as fp32 [F][64] with the piece e4 of row f
// at piece position e4 ^ (f % 16) (read back one row per lane without bank conflicts, see
// read_state_sum), z into zacc.  The caller synchronises the block before reading them.
__device__ __forceinline__ void sum_segments(const float* __restrict__ wsS, const float* __restrict__ wsZ,
                                             int bh, int nseg, int nsum, int F, float* sacc, float* zacc,
                                             const KParams* kp = nullptr)
{
    const int tid = threadIdx.x;
    const int J = F / 32;   // pieces per thread: F * 16 / kOutThreads
    float4 acc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    float zsum = 0.0f;
    if (kp && kp->s_in) {   // the state the sequence starts from (same [F][64] piece order)
        const float4* src = reinterpret_cast<const float4*>(kp->s_in + static_cast<size_t>(bh) * kp->s_stride);
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (j < J) acc[j] = src[tid + kOutThreads * j];
        if (tid < F) zsum = kp->z_in[static_cast<size_t>(bh) * kp->z_stride + tid];
    }
#pragma unroll 2
    for (int s = 0; s < nsum; ++s) {
        const size_t segidx = static_cast<size_t>(bh) * nseg + s;
        const float4* src = reinterpret_cast<const float4*>(wsS + segidx * F * 64);
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (j < J) {
                const float4 x = src[tid + kOutThreads * j];
                acc[j].x += x.x; acc[j].y += x.y; acc[j].z += x.z; acc[j].w += x.w;
            }
        if (tid < F) zsum += wsZ[segidx * F + tid];
    }
#pragma unroll
    for (int j = 0; j < 8; ++j)
        if (j < J) {
            const int c = tid + kOutThreads * j, f = c >> 4, e4 = c & 15;
            *reinterpret_cast<float4*>(sacc + f * 64 + ((e4 ^ (f & 15)) << 2)) = acc[j];
        }
    if (tid < F) zacc[tid] = zsum;
}

// Row f of a sum_segments result as fp32 bit patterns: columns [0, 32) into r0, [32, 64) r1
__device__ __forceinline__ void read_state_sum(const float* sacc, int f, uint32_t (&r0)[32], uint32_t (&r1)[32])
{
#pragma unroll
    for (int e4 = 0; e4 < 16; ++e4) {
        const float4 x = *reinterpret_cast<const float4*>(sacc + f * 64 + ((e4 ^ (f & 15)) << 2));
        uint32_t* r = e4 < 8 ? r0 : r1;
        const int c = 4 * (e4 & 7);
        r[c] = __float_as_uint(x.x); r[c + 1] = __float_as_uint(x.y);
        r[c + 2] = __float_as_uint(x.z); r[c + 3] = __float_as_uint(x.w);
    }
}

// Output kernel: phi(k) slice t (of at most 4) is signalled on its own barrier, so the
// phi(k) warps, which may run a tile ahead, never complete a phase the MMA warp has not
// yet waited for.
__device__ __forceinline__ uint64_t* pk_full(uint64_t* bar, int t)
{
    return &bar[t == 0 ? B_PK_FULL : B_PK_FULL1 + t - 1];
}

// grid = BH * nseg.  One CTA walks the tiles of one segment with the state entering it.
// Warp 0 loads tiles; warp 1 issues the score, readout, state and P.V MMAs; warps 2 / 3
// issue the q / k projections (32 features each) into U0 / U1.  Warps 4-7 turn q
// projections into phi(q), warps 8-11 k projections into phi(k); warps 12-15 finish each
// tile (masked scores in place in tensor memory as bf16, the state copy for the next
// readout, the output), so the feature warps move on to the next tile meanwhile.
__global__ void __launch_bounds__(kOutThreads, 1)
k_tc_causal_out(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmw,
                KParams kp, const float* __restrict__ wsS, const float* __restrict__ wsZ,
                __nv_bfloat16* __restrict__ out, float* __restrict__ den, int* __restrict__ err)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* sm = aligned_smem(smem_raw);
    const SmemOut L = smem_out_layout(kp.F);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + L.bar);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + L.tmem);
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int NT = kp.F / kSlice, NS = kp.F / kSub, halves = kp.F / 128;
    const Seg sg = segment_of(blockIdx.x, kp.nseg, kp.ntiles);

    if (warp == 1) {
        tmem_alloc(tslot, 512);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < NUM_BARS; ++i) mbar_init(&bar[i], 1);
        mbar_init(&bar[B_QK_EMPTY], 2 + 8);
        for (int s = 0; s < kWSlots; ++s) mbar_init(&bar[B_W_EMPTY0 + s], 2);
        mbar_init(&bar[B_U_EMPTY0], 4);
        mbar_init(&bar[B_U_EMPTY1], 4);
        mbar_init(&bar[B_PQ_FULL0], 4);
        mbar_init(&bar[B_PQ_FULL1], 4);
        mbar_init(&bar[B_PK_FULL], 4);
        for (int t = 1; t < 4; ++t) mbar_init(&bar[B_PK_FULL1 + t - 1], 4);
        mbar_init(&bar[B_PSM_FULL], 4);
        mbar_init(&bar[B_O_EMPTY], 4);
        mbar_init(&bar[B_SBF_READY], 4);
        mbar_fence_init();
        tma_prefetch_desc(&tmq);
        tma_prefetch_desc(&tmk);
        tma_prefetch_desc(&tmv);
        tma_prefetch_desc(&tmw);
    }
    fill_ones(sm + L.ones);
    {   // the state copy: columns 65..79 stay zero
        uint4* p = reinterpret_cast<uint4*>(sm + L.st);
        for (int i = tid; i < NT * kStBytes / 16; i += kOutThreads) p[i] = make_uint4(0, 0, 0, 0);
    }
    // the state entering the segment (sum of the earlier segments' sums) into the phi(k)
    // space, z into the phi(q) space (neither is written before the next block barrier)
    sum_segments(wsS, wsZ, sg.bh, kp.nseg, sg.seg, kp.F, reinterpret_cast<float*>(sm + L.phik),
                 reinterpret_cast<float*>(sm + L.phiq));
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    // registers: 128 per thread at launch; the single-thread issuers of warpgroup 0 give
    // 32 of theirs to the three epilogue warpgroups (128*96 + 384*136 <= 65536).  Each role
    // stays inside the branch that set its budget.
    if (warp < 4) {
        regs_dec<96>();
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        Waiter wt;
        if (warp == 0) {
            // ---------------------------------------------------------------- TMA
            if (lane == 0) {
                uint32_t ph_qke = 0, ph_ve = 0, ph_we = (1u << kWSlots) - 1u;
                int n_glob = 0;
                const int vpoint = (NS < kWSlots ? NS : kWSlots) - 1;
                mbar_arrive_expect_tx(&bar[B_QK_FULL], 2 * kTileBytes);
                tma_load_3d(sm + L.q, &tmq, &bar[B_QK_FULL], 0, sg.t_begin * kTile, sg.bh);
                tma_load_3d(sm + L.k, &tmk, &bar[B_QK_FULL], 0, sg.t_begin * kTile, sg.bh);
                mbar_arrive_expect_tx(&bar[B_V_FULL], kTileBytes);
                tma_load_3d(sm + L.v, &tmv, &bar[B_V_FULL], 0, sg.t_begin * kTile, sg.bh);
                for (int tile = sg.t_begin; tile < sg.t_end; ++tile) {
                    for (int n = 0; n < NS; ++n, ++n_glob) {
                        const int slot = n_glob % kWSlots;
                        uint32_t ph = (ph_we >> slot) & 1u;
                        wt.wait(&bar[B_W_EMPTY0 + slot], ph);
                        ph_we ^= (1u << slot);
                        mbar_arrive_expect_tx(&bar[B_W_FULL0 + slot], kWBytes);
                        tma_load_2d(sm + L.w + slot * kWBytes, &tmw, &bar[B_W_FULL0 + slot], 0, n * 64);
                        // V of this tile once the previous tile's P.V and state update are done
                        if (tile > sg.t_begin && n == vpoint) {
                            wt.wait(&bar[B_V_EMPTY], ph_ve);
                            mbar_arrive_expect_tx(&bar[B_V_FULL], kTileBytes);
                            tma_load_3d(sm + L.v, &tmv, &bar[B_V_FULL], 0, tile * kTile, sg.bh);
                        }
                    }
                    if (tile + 1 < sg.t_end) {
                        wt.wait(&bar[B_QK_EMPTY], ph_qke);
                        mbar_arrive_expect_tx(&bar[B_QK_FULL], 2 * kTileBytes);
                        tma_load_3d(sm + L.q, &tmq, &bar[B_QK_FULL], 0, (tile + 1) * kTile, sg.bh);
                        tma_load_3d(sm + L.k, &tmk, &bar[B_QK_FULL], 0, (tile + 1) * kTile, sg.bh);
                    }
                }
            }
        } else if (warp == 1) {
            // ------------------------------------------------------ main MMA issuer
            if (lane == 0) {
                uint32_t ph_vf = 0, ph_pqf0 = 0, ph_pqf1 = 0, ph_pkf = 0, ph_psm = 0, ph_oe = 0,
                         ph_sbf = 0;
                constexpr uint32_t idP = idesc_bf16(128, 128, 0, 0);
                constexpr uint32_t idO = idesc_bf16(128, 80, 0, 1);
                constexpr uint32_t idPV = idesc_bf16(128, 80, 0, 1);
                const uint32_t st_sbo = static_cast<uint32_t>(kp.F) * 16;
                for (int tile = sg.t_begin; tile < sg.t_end; ++tile) {
                    const bool last = tile + 1 == sg.t_end;
                    for (int t = 0; t < NT; ++t) {
                        const int pslot = t & 1;
                        wt.wait(&bar[B_PQ_FULL0 + pslot], pslot ? ph_pqf1 : ph_pqf0);
                        {   // ph_pkf: one phase bit per phiK slice barrier
                            uint32_t ph = (ph_pkf >> t) & 1u;
                            wt.wait(pk_full(bar, t), ph);
                            ph_pkf ^= (1u << t);
                        }
                        if (t == 0 && tile > sg.t_begin) {
                            wt.wait(&bar[B_SBF_READY], ph_sbf);
                            wt.wait(&bar[B_O_EMPTY], ph_oe);
                        }
                        tc_fence_after();
                        // descriptors once per slice, stepped by adds over its 4 K steps
                        const uint64_t ad = desc_kmajor(sbase + L.phiq + pslot * kTileBytes);
                        const uint64_t bk = desc_kmajor(sbase + L.phik + t * kTileBytes);
                        const uint64_t bs = sdesc(sbase + L.st + t * (kSlice / 8) * 128, 128, st_sbo, kLayoutNone);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint32_t acc = (t > 0 || kk > 0) ? 1u : 0u;
                            umma_bf16(tmem + kColP, ad + 2 * kk, bk + 2 * kk, idP, acc);
                            umma_bf16(tmem + kColO, ad + 2 * kk, bs + 16 * kk, idO, acc);
                        }
                        umma_commit(&bar[B_PQ_EMPTY0 + pslot]);
                        // state update of a feature half once its phiK slices are in place; the
                        // half's phiK slices are free for the next tile once it has been read
                        if (!last && (t & 1) == 1) {
                            if (t == 1) wt.wait(&bar[B_V_FULL], ph_vf);
                            issue_state_half(tmem, kColS, desc_phik(sbase + L.phik),
                                                 desc_v(sbase + L.v, sbase + L.ones), t >> 1, false);
                            umma_commit(&bar[B_PK_FREE0 + (t >> 1)]);
                        }
                    }
                    umma_commit(&bar[B_P_FULL]);
                    if (last) wt.wait(&bar[B_V_FULL], ph_vf);
                    wt.wait(&bar[B_PSM_FULL], ph_psm);
                    tc_fence_after();
                    const uint64_t dvv = desc_v(sbase + L.v, sbase + L.ones);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        umma_bf16_ts(tmem + kColO, tmem + kColP + 8 * kk, dvv + 128 * kk, idPV, 1u);
                    umma_commit(&bar[B_TILE_DONE]);
                    umma_commit(&bar[B_V_EMPTY]);
                }
            }
        } else {
            // ------------------------------------------- projection issuers (q: 2, k: 3)
            if (lane == 0) {
                const int g = warp - 2;
                const uint64_t dx = desc_kmajor(sbase + (g ? L.k : L.q)), dw0 = desc_kmajor(sbase + L.w);
                uint32_t ph_qkf = 0, ph_wf = 0, ph_ue = 1;
                int n_glob = 0;
                for (int tile = sg.t_begin; tile < sg.t_end; ++tile) {
                    wt.wait(&bar[B_QK_FULL], ph_qkf);
                    for (int n = 0; n < NS; ++n, ++n_glob) {
                        const int slot = n_glob % kWSlots;
                        uint32_t ph = (ph_wf >> slot) & 1u;
                        wt.wait(&bar[B_W_FULL0 + slot], ph);
                        ph_wf ^= (1u << slot);
                        wt.wait(&bar[B_U_EMPTY0 + g], ph_ue);
                        tc_fence_after();
                        issue_projection(tmem + (g ? kColU1 : kColU0), dx, desc_add(dw0, slot * kWBytes));
                        umma_commit(&bar[B_U_FULL0 + g]);
                        umma_commit(&bar[B_W_EMPTY0 + slot]);
                    }
                    umma_commit(&bar[B_QK_EMPTY]);
                }
            }
        }
        wt.report(err);
        drain_after_failure(wt.ok);
    } else {
        regs_inc<136>();
        // state entering the segment (sum of the earlier segments), by the tail warps
        if (warp >= 12) {
            const int sp = warp & 3;
            const uint32_t row = 32u * sp + lane;
            const uint32_t trow = tmem + ((32u * sp) << 16);
            for (int h = 0; h < halves; ++h) {
                const int f = 128 * h + row;
                uint32_t r0[32], r1[32];
                read_state_sum(reinterpret_cast<const float*>(sm + L.phik), f, r0, r1);
                const float zf = reinterpret_cast<const float*>(sm + L.phiq)[f];
                tmem_st32(trow + kColS + 80 * h, r0);
                tmem_st32(trow + kColS + 80 * h + 32, r1);
                write_state_row_u(sbase + L.st, kp.F, f, r0, r1, zf);
#pragma unroll
                for (int e = 0; e < 32; ++e) r0[e] = __float_as_uint(zf);
                tmem_st32(trow + kColS + 80 * h + 64, r0);  // z columns (a later half rewrites its own)
            }
            tmem_wait_st();
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        Waiter wt;
        const int64_t rowbase = static_cast<int64_t>(sg.bh) * kp.L;
        if (warp < 12) {
            // ------------------------------------------------ feature epilogues
            const int grp = (warp >= 8) ? 1 : 0;
            const int sp = warp & 3;
            const uint32_t row = 32u * sp + lane;
            const uint32_t trow = tmem + ((32u * sp) << 16);
            uint32_t ph_qkf = 0, ph_uf = 0, ph_pqe0 = 0, ph_pqe1 = 0, ph_pkf0 = 0, ph_pkf1 = 0;
            int uses0 = 0, uses1 = 0;
            for (int tile = sg.t_begin; tile < sg.t_end; ++tile) {
                wt.wait(&bar[B_QK_FULL], ph_qkf);
                float inv, l2i;
                row_scale(sm + (grp ? L.k : L.q) + row * 128, row, inv, l2i);
                warp_arrive(&bar[B_QK_EMPTY]);
                for (int t = 0; t < NT; ++t) {
                    const float a = slice_val(kp.a2, t) * inv, b = slice_val(kp.b2, t) + l2i;
                    const int pslot = t & 1;
                    for (int half = 0; half < 2; ++half) {
                        wt.wait(&bar[B_U_FULL0 + grp], ph_uf);
                        tc_fence_after();
                        uint32_t ur[32], pr[32];
                        const uint32_t col = grp ? kColU1 : kColU0;
                        tmem_ld32(trow + col, ur);
                        tmem_ld32(trow + col + 32, pr);
                        tmem_wait_ld();
                        reg_fence(ur);
                        reg_fence(pr);
                        tc_fence_before();
                        warp_arrive(&bar[B_U_EMPTY0 + grp]);
                        if (grp == 0) {
                            if (half == 0) {
                                int& uses = pslot ? uses1 : uses0;
                                if (uses > 0) wt.wait(&bar[B_PQ_EMPTY0 + pslot], pslot ? ph_pqe1 : ph_pqe0);
                                ++uses;
                            }
                            phi_sub_epilogue(ur, pr, a, b, sbase + L.phiq + pslot * kTileBytes, row, half,
                                             nullptr);
                        } else {
                            if (half == 0 && pslot == 0 && tile > sg.t_begin)
                                wt.wait(&bar[B_PK_FREE0 + (t >> 1)], (t >> 1) ? ph_pkf1 : ph_pkf0);
                            phi_sub_epilogue(ur, pr, a, b, sbase + L.phik + t * kTileBytes, row, half,
                                             nullptr);
                        }
                    }
                    fence_async_smem();
                    warp_arrive(grp ? pk_full(bar, t) : &bar[B_PQ_FULL0 + pslot]);
                }
            }
        } else {
            // ------------------------------------------------------------ tile tail
            const int sp = warp & 3;
            const uint32_t row = 32u * sp + lane;
            const uint32_t trow = tmem + ((32u * sp) << 16);
            uint32_t ph_pf = 0, ph_td = 0;
            for (int tile = sg.t_begin; tile < sg.t_end; ++tile) {
                // masked scores -> bf16 in place (row i keeps keys j <= i), the A operand of P.V.
                // Key chunk c (32 keys) is below this warp's rows for c < sp, on the diagonal for
                // c == sp and above it (all zero, not read) for c > sp.
                wt.wait(&bar[B_P_FULL], ph_pf);
                tc_fence_after();
    #pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t pk[16];
                    if (c <= sp) {
                        uint32_t pv[32];
                        tmem_ld32(trow + kColP + 32 * c, pv);
                        tmem_wait_ld();
                        reg_fence(pv);
                        if (c < sp) {
    #pragma unroll
                            for (int j = 0; j < 16; ++j)
                                pk[j] = pack_bf16(__uint_as_float(pv[2 * j]), __uint_as_float(pv[2 * j + 1]));
                        } else {
    #pragma unroll
                            for (int j = 0; j < 16; ++j)
                                pk[j] = pack_bf16((2 * j <= lane) ? __uint_as_float(pv[2 * j]) : 0.0f,
                                                  (2 * j + 1 <= lane) ? __uint_as_float(pv[2 * j + 1]) : 0.0f);
                        }
                    } else {
    #pragma unroll
                        for (int j = 0; j < 16; ++j) pk[j] = 0u;
                    }
                    tmem_st16(trow + kColP + 16 * c, pk);
                }
                tmem_wait_st();
                tc_fence_before();
                warp_arrive(&bar[B_PSM_FULL]);
                if (tile + 1 < sg.t_end) {
                    // state after this tile (its update finished before the scores did) -> bf16
                    // copy for the next readout
                    for (int h = 0; h < halves; ++h) {
                        const int f = 128 * h + row;
                        uint32_t r0s[32], r1s[32], zr;
                        tmem_ld32(trow + kColS + 80 * h, r0s);
                        tmem_ld32(trow + kColS + 80 * h + 32, r1s);
                        tmem_ld1(trow + kColS + 80 * h + 64, zr);
                        tmem_wait_ld();
                        reg_fence(r0s);
                        reg_fence(r1s);
                        reg_fence1(zr);
                        float sv[64];
    #pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            sv[e] = __uint_as_float(r0s[e]);
                            sv[32 + e] = __uint_as_float(r1s[e]);
                        }
                        write_state_row(sbase + L.st, kp.F, f, sv, __uint_as_float(zr));
                    }
                    fence_async_smem();
                    tc_fence_before();
                    warp_arrive(&bar[B_SBF_READY]);
                }
                // output: O[:, :64] / (O[:, 64] + eps)
                wt.wait(&bar[B_TILE_DONE], ph_td);
                tc_fence_after();
                uint32_t o0[32], o1[32], dr;
                tmem_ld32(trow + kColO, o0);
                tmem_ld32(trow + kColO + 32, o1);
                tmem_ld1(trow + kColO + 64, dr);
                tmem_wait_ld();
                reg_fence(o0);
                reg_fence(o1);
                reg_fence1(dr);
                tc_fence_before();
                warp_arrive(&bar[B_O_EMPTY]);
                const int grow = tile * kTile + static_cast<int>(row);
                if (grow < kp.L)
                    finish_row(kp, o0, o1, __uint_as_float(dr), rowbase + grow, out, den);
            }
        }
        wt.report(err);
        drain_after_failure(wt.ok);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

// ------------------------------------------- causal output reading stored phi(k)
// grid = BH * nseg; one CTA walks the tiles of one segment with the state entering it, as
// k_tc_causal_out does, but phi(k) of every tile comes from HBM (written by the state
// kernel) instead of being recomputed, and phi(q) is written by its warps into tensor memory
// (bf16 pairs), where the score and readout MMAs read it as their A operand: phi(q) never
// passes through shared memory.  The projection operand W stays resident in shared memory
// and each 64-feature slice is one N = 128 projection.  Tensor memory holds no z and no ones
// column (to fit the phi(q) slot): the denominator is
//   den_i = phi(q_i) . z_tile + sum_{j <= i in the tile} P_ij,
// the first term from the readout against the state copy [S | z] (z_tile = z of the earlier
// segments + the column sums of this segment's earlier phi(k) tiles, which the output warps
// add up from the tiles in shared memory), the second summed in fp32 by the warps that mask
// the scores.
//
// Warps: 0 TMA (W once; q tiles, two buffers; phi(k) slices; v), 1 the score / readout /
// state / P.V MMAs, 2 the projections, 3 idle after setup; 4-11 phi(q) (group g = warp >= 8
// takes features [32g, 32g+32) of every slice) and, between the first two slices of a tile,
// the previous tile's masked bf16 scores; 12-15 the column sums of phi(k) (warp 12 + t sums
// slice t), the state copy for the next readout and the outputs.
constexpr uint32_t kTsU = 0;      // 128: projection of one 64-feature slice ([u | p] per 32)
constexpr uint32_t kTsP = 128;    // 128: intra-tile scores, then bf16 P in place
constexpr uint32_t kTsO = 256;    // 80 : numerator | phi(q) . z (column 64)
constexpr uint32_t kTsS = 336;    // 2 x 64: state S of the feature halves
constexpr uint32_t kTsQ = 464;    // 32 : phi(q) slice (64 features as 32 bf16 pairs)
constexpr uint32_t kTsFree = 496; // 16 : unused (the launch's throwaway first MMA)

enum {
    T_QF0 = 0, T_QF1, T_QE0, T_QE1, T_WF, T_UF, T_UE, T_PQF, T_PQE,
    T_PKF0, T_PKF1, T_PKF2, T_PKF3, T_PKFREE0, T_PKFREE1,
    T_VF, T_VE, T_PF, T_PSM, T_SD, T_TD, T_OE, T_SBF,
    T_DF0, T_DF1, T_DE0, T_DE1, T_ZC0, T_ZC1,
    NUM_TS_BARS
};

struct SmemOutTs {
    uint32_t w, q, v, phik, st, zpre, ztile, den, bar, tmem, total;
};

__host__ __device__ inline SmemOutTs smem_outts_layout(int F)
{
    SmemOutTs s;
    s.w = 0;                                     // F/32 sub-slices of 8 KiB, resident
    s.q = s.w + (F / kSub) * kWBytes;            // 2 buffers
    s.v = s.q + 2 * kTileBytes;
    s.phik = s.v + kTileBytes;                   // F/64 slices
    s.st = s.phik + (F / kSlice) * kTileBytes;   // [S | z] copy: F x 80 bf16 (write_state_row)
    s.zpre = s.st + (F / kSlice) * kStBytes;     // fp32 [F]: z of the earlier segments
    s.ztile = s.zpre + F * 4;                    // fp32 [2][F]: z entering the next tile
    s.den = s.ztile + 2 * F * 4;                 // fp32 [2 tile parities][2 groups][128 rows]
    s.bar = s.den + 2 * 2 * kTile * 4;
    s.tmem = s.bar + NUM_TS_BARS * 8;
    s.total = s.tmem + 16;
    return s;
}

// Columns [32 part, 32 part + 32) of row f of the [S | z] copy (four of its 16-byte pieces)
__device__ __forceinline__ void write_state_cols32(uint32_t st, int F, int f, int part, const uint32_t (&s)[32])
{
    const uint32_t sbo = static_cast<uint32_t>(F) * 16;
    const uint32_t base = st + (f >> 3) * 128 + (f & 7) * 16 + 4 * part * sbo;
#pragma unroll
    for (int q = 0; q < 4; ++q)
        st_shared_v4(base + q * sbo,
                     pack_bf16(__uint_as_float(s[8 * q]), __uint_as_float(s[8 * q + 1])),
                     pack_bf16(__uint_as_float(s[8 * q + 2]), __uint_as_float(s[8 * q + 3])),
                     pack_bf16(__uint_as_float(s[8 * q + 4]), __uint_as_float(s[8 * q + 5])),
                     pack_bf16(__uint_as_float(s[8 * q + 6]), __uint_as_float(s[8 * q + 7])));
}

// Column 64 (z) of row f of the [S | z] copy, with columns 65..71 zero
__device__ __forceinline__ void write_state_z(uint32_t st, int F, int f, float z)
{
    st_shared_v4(st + (f >> 3) * 128 + (f & 7) * 16 + 8 * static_cast<uint32_t>(F) * 16, pack_bf16(z, 0.0f), 0u, 0u, 0u);
}

// phi of 32 features (u, p of this row) packed as 16 bf16 pairs
__device__ __forceinline__ void phi_pack(const uint32_t (&ur)[32], const uint32_t (&pr)[32], float a, float b,
                                         uint32_t (&pk)[16])
{
#pragma unroll
    for (int j = 0; j < 32; j += 2) {
        const float2 y = ffma2(make_float2(a, a), make_float2(__uint_as_float(ur[j]), __uint_as_float(ur[j + 1])),
                               make_float2(b, b));
        const float2 pp = make_float2(__uint_as_float(pr[j]), __uint_as_float(pr[j + 1]));
        const float2 e = make_float2(ex2(y.x), ex2(y.y));
        const float2 ff = fmul2(fmul2(e, pp), pp);
        pk[j >> 1] = pack_bf16(ff.x, ff.y);
    }
}

// [S]_h += phiK_h^T V for feature half h (N = 64: no ones column here)
__device__ __forceinline__ void issue_state_half64(uint32_t tmem, uint64_t dphik, uint64_t dv, int h)
{
    constexpr uint32_t idS = idesc_bf16(128, 64, 1, 1);
    const uint64_t da = desc_add(dphik, 2 * h * kTileBytes);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) umma_bf16(tmem + kTsS + 64 * h, da + 128 * kk, dv + 128 * kk, idS, 1u);
}

// The masked scores of tile `pit` of the segment as bf16 in place, by the phi(q) warp of
// group g: the 32-column chunks c = g, g + 2 (chunks past the diagonal are zeros).  Chunk
// c (fp32 columns [32c, 32c+32)) goes to bf16 columns 32g + 16(c/2): a group writes only the
// columns of its own first chunk, after reading them, so the two groups of a quadrant never
// overwrite what the other still reads.  The row's sum of its unmasked scores in these
// chunks (fp32) goes to dens.
__device__ __forceinline__ void ts_mask_scores(uint64_t* bar, Waiter& wt, uint32_t& ph_pf, uint32_t& ph_de,
                                               uint32_t trow, uint32_t row, int lane, int sp, int g,
                                               float* dens, int pit)
{
    wt.wait(&bar[T_PF], ph_pf);
    tc_fence_after();
    float dint = 0.0f;
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
        const int c = g + 2 * cc;
        uint32_t pk[16];
        uint32_t pv[32];
        if (c <= sp) {
            tmem_ld32(trow + kTsP + 32 * c, pv);
            tmem_wait_ld();
            reg_fence(pv);
        }
        if (c < sp) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const float x0 = __uint_as_float(pv[2 * j]), x1 = __uint_as_float(pv[2 * j + 1]);
                dint += x0 + x1;
                pk[j] = pack_bf16(x0, x1);
            }
        } else if (c == sp) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const float x0 = (2 * j <= lane) ? __uint_as_float(pv[2 * j]) : 0.0f;
                const float x1 = (2 * j + 1 <= lane) ? __uint_as_float(pv[2 * j + 1]) : 0.0f;
                dint += x0 + x1;
                pk[j] = pack_bf16(x0, x1);
            }
        } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) pk[j] = 0u;
        }
        tmem_st16(trow + kTsP + 32 * g + 16 * cc, pk);
    }
    tmem_wait_st();
    tc_fence_before();
    warp_arrive(&bar[T_PSM]);
    const int par = pit & 1;
    if (pit >= 2) {
        uint32_t pd = (ph_de >> par) & 1u;
        wt.wait(&bar[T_DE0 + par], pd);
        ph_de ^= 1u << par;
    }
    dens[(2 * par + g) * kTile + row] = dint;
    warp_arrive(&bar[T_DF0 + par]);
}

template <int kAcc>   // bit 0: add the earlier chunks' sums; bit 1: store this chunk's sums
__global__ void __launch_bounds__(kOutThreads, 1)
k_tc_causal_out_ts(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmpk,
                   const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmw,
                   KParams kp, const float* __restrict__ wsS, const float* __restrict__ wsZ,
                   __nv_bfloat16* __restrict__ out, float* __restrict__ den, int* __restrict__ err)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* sm = aligned_smem(smem_raw);
    const SmemOutTs L = smem_outts_layout(kp.F);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + L.bar);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + L.tmem);
    float* zpre = reinterpret_cast<float*>(sm + L.zpre);
    float* ztile = reinterpret_cast<float*>(sm + L.ztile);
    float* dens = reinterpret_cast<float*>(sm + L.den);
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int NT = kp.F / kSlice, NS = kp.F / kSub, halves = kp.F / 128;
    const Seg sg = segment_of(blockIdx.x, kp.nseg, kp.ntiles);

    if (warp == 1) {
        tmem_alloc(tslot, 512);
        tmem_relinquish();
        // The first MMA of a launch takes ~7k cycles: a throwaway one into the unused columns
        // [kTsFree, 512) spends them while this CTA waits for the state kernel.  Later MMAs of
        // this thread are committed and waited for, so it has completed before the dealloc.
        tc_fence_before();
        __syncwarp();
        tc_fence_after();
        if (lane == 0 && sg.t_end > sg.t_begin) {
            uint32_t a = sbase;   // opaque: nothing computed here stays live for later code
            asm volatile("" : "+r"(a));
            umma_bf16(*tslot + kTsFree, desc_kmajor(a), desc_kmajor(a),
                      idesc_bf16(128, 512 - kTsFree, 0, 0), 0u);
        }
    }
    if (tid == 0) {
        for (int i = 0; i < NUM_TS_BARS; ++i) mbar_init(&bar[i], 1);
        mbar_init(&bar[T_QE0], 1 + 8);   // the projection issuer's commit + the phi(q) warps
        mbar_init(&bar[T_QE1], 1 + 8);
        mbar_init(&bar[T_UE], 8);
        mbar_init(&bar[T_PQF], 8);
        mbar_init(&bar[T_PSM], 8);
        mbar_init(&bar[T_OE], 4);
        mbar_init(&bar[T_SBF], 4);
        mbar_init(&bar[T_DF0], 8);
        mbar_init(&bar[T_DF1], 8);
        mbar_init(&bar[T_DE0], 4);
        mbar_init(&bar[T_DE1], 4);
        mbar_init(&bar[T_ZC0], 2);       // column sums of the two slices of a feature half
        mbar_init(&bar[T_ZC1], 2);
        mbar_fence_init();
        tma_prefetch_desc(&tmq);
        tma_prefetch_desc(&tmpk);
        tma_prefetch_desc(&tmv);
        tma_prefetch_desc(&tmw);
        // W and the first two q tiles (regions the prologue below does not touch) load while
        // the state entering the segment is summed
        mbar_arrive_expect_tx(&bar[T_WF], NS * kWBytes);
        for (int n = 0; n < NS; ++n) tma_load_2d(sm + L.w + n * kWBytes, &tmw, &bar[T_WF], 0, n * 64);
        for (int j = 0; j < 2 && sg.t_begin + j < sg.t_end; ++j) {
            mbar_arrive_expect_tx(&bar[T_QF0 + j], kTileBytes);
            tma_load_3d(sm + L.q + j * kTileBytes, &tmq, &bar[T_QF0 + j], 0, (sg.t_begin + j) * kTile, sg.bh);
        }
    }
    {   // the state copy: columns 65..79 stay zero
        uint4* p = reinterpret_cast<uint4*>(sm + L.st);
        for (int i = tid; i < NT * kStBytes / 16; i += kOutThreads) p[i] = make_uint4(0, 0, 0, 0);
    }
    // The state entering the segment, the sum of the earlier segments' sums, into the phi(k)
    // slices' space (no copy has reached it yet), z into zpre
    griddep_wait();   // the state kernel's sums and phi(k) (launched as its dependent)
    sum_segments(wsS, wsZ, sg.bh, kp.nseg, sg.seg, kp.F, reinterpret_cast<float*>(sm + L.phik), zpre, &kp);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    if (warp < 4) {
        regs_dec<96>();
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        Waiter wt;
        if (warp == 0) {
            // ---------------------------------------------------------------- TMA
            // per tile (W and the first two q tiles are loading since the start) the q tile two
            // ahead (two buffers, needed a tile ahead by the projections), the phi(k) slices
            // (each feature half once the previous tile's scores, state update and column sums
            // are done with it) and v (once the previous P.V is done)
            if (lane == 0) {
                uint32_t ph_qe = 0, ph_free = 0, ph_zc = 0, ph_ve = 0;
                auto load_q = [&](int it) {
                    const int qb = it & 1;
                    if (it >= 2) {
                        uint32_t ph = (ph_qe >> qb) & 1u;
                        wt.wait(&bar[T_QE0 + qb], ph);
                        ph_qe ^= 1u << qb;
                    }
                    mbar_arrive_expect_tx(&bar[T_QF0 + qb], kTileBytes);
                    tma_load_3d(sm + L.q + qb * kTileBytes, &tmq, &bar[T_QF0 + qb], 0,
                                (sg.t_begin + it) * kTile, sg.bh);
                };
                const int n = sg.t_end - sg.t_begin;
                for (int tile = sg.t_begin, it = 0; tile < sg.t_end; ++tile, ++it) {
                    for (int t = 0; t < NT; ++t) {
                        if (it > 0 && (t & 1) == 0) {   // MMAs and column sums done with the half
                            const int h = t >> 1;
                            uint32_t ph = (ph_free >> h) & 1u;
                            wt.wait(&bar[T_PKFREE0 + h], ph);
                            ph_free ^= 1u << h;
                            uint32_t pz = (ph_zc >> h) & 1u;
                            wt.wait(&bar[T_ZC0 + h], pz);
                            ph_zc ^= 1u << h;
                        }
                        mbar_arrive_expect_tx(&bar[T_PKF0 + t], kTileBytes);
                        tma_load_3d(sm + L.phik + t * kTileBytes, &tmpk, &bar[T_PKF0 + t], kSlice * t,
                                    tile * kTile, sg.bh);
                    }
                    if (it > 0) wt.wait(&bar[T_VE], ph_ve);
                    mbar_arrive_expect_tx(&bar[T_VF], kTileBytes);
                    tma_load_3d(sm + L.v, &tmv, &bar[T_VF], 0, tile * kTile, sg.bh);
                    if (it + 2 < n) load_q(it + 2);
                }
            }
        } else if (warp == 2) {
            // ---------------------------------- q projections, one 64-feature slice each
            if (lane == 0) {
                constexpr uint32_t idU = idesc_bf16(128, 128, 0, 0);
                uint32_t ph_qf = 0, ph_ue = 1, ph_wf = 0;
                const uint64_t dq0 = desc_kmajor(sbase + L.q), dw0 = desc_kmajor(sbase + L.w);
                wt.wait(&bar[T_WF], ph_wf);
                for (int tile = sg.t_begin, it = 0; tile < sg.t_end; ++tile, ++it) {
                    const int qb = it & 1;
                    uint32_t ph = (ph_qf >> qb) & 1u;
                    wt.wait(&bar[T_QF0 + qb], ph);
                    ph_qf ^= 1u << qb;
                    const uint64_t dq = desc_add(dq0, qb * kTileBytes);
                    for (int t = 0; t < NT; ++t) {
                        wt.wait(&bar[T_UE], ph_ue);
                        tc_fence_after();
                        const uint64_t dw = desc_add(dw0, t * 2 * kWBytes);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            umma_bf16(tmem + kTsU, dq + 2 * kk, dw + 2 * kk, idU, kk > 0 ? 1u : 0u);
                        umma_commit(&bar[T_UF]);
                    }
                    umma_commit(&bar[T_QE0 + qb]);
                }
            }
        } else if (warp == 1) {
            // ------------------------------------------------------ main MMA issuer
            if (lane == 0) {
                uint32_t ph_pqf = 0, ph_pkf = 0, ph_vf = 0, ph_psm = 0, ph_oe = 0, ph_sbf = 0;
                constexpr uint32_t idP = idesc_bf16(128, 128, 0, 0);
                constexpr uint32_t idO = idesc_bf16(128, 80, 0, 1);
                constexpr uint32_t idPV = idesc_bf16(128, 64, 0, 1);
                const uint32_t st_sbo = static_cast<uint32_t>(kp.F) * 16;
                const uint64_t dph = desc_phik(sbase + L.phik);
                const uint64_t dv = sdesc(sbase + L.v, kTileBytes, 1024, kLayoutSW128);
                const uint32_t aq = tmem + kTsQ;
                for (int tile = sg.t_begin; tile < sg.t_end; ++tile) {
                    const bool last = tile + 1 == sg.t_end;
                    bool have_v = false;
                    for (int t = 0; t < NT; ++t) {
                        wt.wait(&bar[T_PQF], ph_pqf);
                        {
                            uint32_t ph = (ph_pkf >> t) & 1u;
                            wt.wait(&bar[T_PKF0 + t], ph);
                            ph_pkf ^= 1u << t;
                        }
                        if (t == 0 && tile > sg.t_begin) {
                            wt.wait(&bar[T_SBF], ph_sbf);
                            wt.wait(&bar[T_OE], ph_oe);
                        }
                        tc_fence_after();
                        const uint64_t bk = desc_kmajor(sbase + L.phik + t * kTileBytes);
                        const uint64_t bs = sdesc(sbase + L.st + t * (kSlice / 8) * 128, 128, st_sbo, kLayoutNone);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint32_t acc = (t > 0 || kk > 0) ? 1u : 0u;
                            umma_bf16_ts(tmem + kTsP, aq + 8 * kk, bk + 2 * kk, idP, acc);
                            umma_bf16_ts(tmem + kTsO, aq + 8 * kk, bs + 16 * kk, idO, acc);
                        }
                        umma_commit(&bar[T_PQE]);
                        // every state half but the last right after its two slices; the last
                        // one after the scores, where it overlaps the masking
                        if ((t & 1) == 1 && !last && (t >> 1) + 1 < halves) {
                            if (!have_v) { wt.wait(&bar[T_VF], ph_vf); have_v = true; }
                            issue_state_half64(tmem, dph, dv, t >> 1);
                            umma_commit(&bar[T_PKFREE0 + (t >> 1)]);
                        }
                    }
                    umma_commit(&bar[T_PF]);
                    if (!have_v) { wt.wait(&bar[T_VF], ph_vf); have_v = true; }
                    if (!last) {
                        tc_fence_after();
                        issue_state_half64(tmem, dph, dv, halves - 1);
                        umma_commit(&bar[T_PKFREE0 + halves - 1]);
                        umma_commit(&bar[T_SD]);
                    }
                    wt.wait(&bar[T_PSM], ph_psm);
                    tc_fence_after();
                    // keys [16kk, 16kk+16): chunk c = kk/2 sits at bf16 columns 32(c%2) + 16(c/2)
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const int c = kk >> 1;
                        const uint32_t acol = 32 * (c & 1) + 16 * (c >> 1) + 8 * (kk & 1);
                        umma_bf16_ts(tmem + kTsO, tmem + kTsP + acol, dv + 128 * kk, idPV, 1u);
                    }
                    umma_commit(&bar[T_TD]);
                    umma_commit(&bar[T_VE]);
                }
            }
        }
        wt.report(err);
        drain_after_failure(wt.ok);
    } else {
        regs_inc<136>();
        if (warp >= 12) {   // state entering the segment (sum of the earlier segments)
            const int sp = warp & 3;
            const uint32_t row = 32u * sp + lane;
            const uint32_t trow = tmem + ((32u * sp) << 16);
            for (int h = 0; h < halves; ++h) {
                const int f = 128 * h + row;
                uint32_t r0[32], r1[32];
                read_state_sum(reinterpret_cast<const float*>(sm + L.phik), f, r0, r1);
                tmem_st32(trow + kTsS + 64 * h, r0);
                tmem_st32(trow + kTsS + 64 * h + 32, r1);
                write_state_row_u(sbase + L.st, kp.F, f, r0, r1, zpre[f]);
            }
            tmem_wait_st();
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        Waiter wt;
        const int64_t rowbase = static_cast<int64_t>(sg.bh) * kp.L;
        if (warp < 12) {
            // ---------------------------------------- phi(q) and the masked scores
            const int g = (warp >= 8) ? 1 : 0;
            const int sp = warp & 3;
            const uint32_t row = 32u * sp + lane;
            const uint32_t trow = tmem + ((32u * sp) << 16);
            uint32_t ph_qf = 0, ph_uf = 0, ph_pqe = 0, ph_de = 0, ph_pf = 0;
            bool slot_used = false;
            for (int tile = sg.t_begin, it = 0; tile < sg.t_end; ++tile, ++it) {
                const int qb = it & 1;
                uint32_t ph = (ph_qf >> qb) & 1u;
                wt.wait(&bar[T_QF0 + qb], ph);
                ph_qf ^= 1u << qb;
                float inv, l2i;
                row_scale(sm + L.q + qb * kTileBytes + row * 128, row, inv, l2i);
                warp_arrive(&bar[T_QE0 + qb]);
                for (int t = 0; t < NT; ++t) {
                    const float a = slice_val(kp.a2, t) * inv, b = slice_val(kp.b2, t) + l2i;
                    wt.wait(&bar[T_UF], ph_uf);
                    tc_fence_after();
                    uint32_t ur[32], pr[32];
                    tmem_ld32(trow + kTsU + 64 * g, ur);
                    tmem_ld32(trow + kTsU + 64 * g + 32, pr);
                    tmem_wait_ld();
                    reg_fence(ur);
                    reg_fence(pr);
                    tc_fence_before();
                    warp_arrive(&bar[T_UE]);
                    uint32_t pk[16];
                    phi_pack(ur, pr, a, b, pk);
                    // the previous tile's scores, complete with its last slice, are masked first:
                    // this slice's MMAs also wait for the readout of those scores' outputs
                    if (t == 0 && it > 0) ts_mask_scores(bar, wt, ph_pf, ph_de, trow, row, lane, sp, g, dens, it - 1);
                    // the slot is free once the MMAs of the previous slice have read it
                    if (slot_used) wt.wait(&bar[T_PQE], ph_pqe);
                    slot_used = true;
                    tmem_st16(trow + kTsQ + 16 * g, pk);
                    tmem_wait_st();
                    tc_fence_before();
                    warp_arrive(&bar[T_PQF]);
                }
            }
            ts_mask_scores(bar, wt, ph_pf, ph_de, trow, row, lane, sp, g, dens, sg.t_end - 1 - sg.t_begin);
        } else {
            // ------------------- column sums of phi(k), state copy for the next readout, outputs
            const int sp = warp & 3, w = warp - 12;
            const uint32_t row = 32u * sp + lane;
            const uint32_t trow = tmem + ((32u * sp) << 16);
            uint32_t ph_td = 0, ph_df = 0, ph_sd = 0, ph_pkf = 0;
            // warp w < F/64: this segment's running sum of phi(k) over the tokens of its
            // tiles so far, features 64w + 2 lane and 64w + 2 lane + 1
            float zr0 = 0.0f, zr1 = 0.0f;
            const int zf0 = kSlice * w + 2 * lane;
            const uint32_t zbase = sbase + L.phik + w * kTileBytes + (lane & 3) * 4;
            for (int tile = sg.t_begin, it = 0; tile < sg.t_end; ++tile, ++it) {
                const bool last = tile + 1 == sg.t_end;
                if (!last) {
                    const int zb = it & 1;
                    if (w < NT) {
                        wt.wait(&bar[T_PKF0 + w], ph_pkf);
                        float c0 = 0.0f, c1 = 0.0f;
                        // row r, features 2 lane, 2 lane + 1: 16-byte chunk lane/4 of the
                        // 128-byte swizzled row, at chunk (lane/4) ^ (r & 7)
#pragma unroll 8
                        for (int r = 0; r < kTile; ++r) {
                            const uint32_t v2 = ld_shared_u32(zbase + r * 128 + (((lane >> 2) ^ (r & 7)) << 4));
                            c0 += __uint_as_float(v2 << 16);
                            c1 += __uint_as_float(v2 & 0xFFFF0000u);
                        }
                        zr0 += c0;
                        zr1 += c1;
                        warp_arrive(&bar[T_ZC0 + (w >> 1)]);
                        ztile[zb * kp.F + zf0] = zpre[zf0] + zr0;
                        ztile[zb * kp.F + zf0 + 1] = zpre[zf0 + 1] + zr1;
                    }
                    named_bar_sync(2, 128);
                    wt.wait(&bar[T_SD], ph_sd);
                    tc_fence_after();
                    for (int h = 0; h < halves; ++h) {
                        const int f = 128 * h + static_cast<int>(row);
#pragma unroll 1
                        for (int part = 0; part < 2; ++part) {
                            uint32_t sv[32];
                            tmem_ld32(trow + kTsS + 64 * h + 32 * part, sv);
                            tmem_wait_ld();
                            reg_fence(sv);
                            write_state_cols32(sbase + L.st, kp.F, f, part, sv);
                        }
                        write_state_z(sbase + L.st, kp.F, f, ztile[zb * kp.F + f]);
                    }
                    fence_async_smem();
                    tc_fence_before();
                    warp_arrive(&bar[T_SBF]);
                }
                wt.wait(&bar[T_TD], ph_td);
                tc_fence_after();
                uint32_t o0[32], o1[32], dr;
                tmem_ld32(trow + kTsO, o0);
                tmem_ld32(trow + kTsO + 32, o1);
                tmem_ld1(trow + kTsO + 64, dr);
                tmem_wait_ld();
                reg_fence(o0);
                reg_fence(o1);
                reg_fence1(dr);
                tc_fence_before();
                warp_arrive(&bar[T_OE]);
                const int par = it & 1;
                {
                    uint32_t pd = (ph_df >> par) & 1u;
                    wt.wait(&bar[T_DF0 + par], pd);
                    ph_df ^= 1u << par;
                }
                const float d = __uint_as_float(dr) + dens[(2 * par) * kTile + row] + dens[(2 * par + 1) * kTile + row];
                warp_arrive(&bar[T_DE0 + par]);
                const int grow = tile * kTile + static_cast<int>(row);
                if (grow < kp.L) finish_row_t<(kAcc & 1) != 0, (kAcc & 2) != 0>(kp, o0, o1, d, rowbase + grow, out, den);
            }
        }
        wt.report(err);
        drain_after_failure(wt.ok);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------ bidirectional readout
// out_i = phi(q_i)^T S / (phi(q_i)^T z + eps) with the state [S | z] of the whole sequence.
// grid = BH * nseg; a CTA walks the tiles of one segment.  Warp 0 loads q tiles (two
// buffers) and projection operands; warp 2 issues the q projections alternately into U0 /
// U1; warps 4-7 and 8-11 turn them into phi(q) (group g writes the 32-feature half g of
// each 64-feature slice); warp 1 issues the readout O = phiQ [S | z] (N = 80) slice by slice;
// warps 12-15 first build the bf16 copy of the summed state, then write the outputs.
struct SmemBidir {
    uint32_t w, q, phiq, st, scr, zt, bar, tmem, total;
};

__host__ __device__ inline SmemBidir smem_bidir_layout(int F)
{
    SmemBidir s;
    s.w = 0;
    s.q = kWSlots * kWBytes;                // 2 buffers
    s.phiq = s.q + 2 * kTileBytes;          // 2 slots of 64 features
    s.st = s.phiq + 2 * kTileBytes;
    s.scr = s.st + (F / kSlice) * kStBytes;   // fp32 [F][64]: the summed state, once
    s.zt = s.scr + F * 256;                   // fp32 [F]: the summed z
    s.bar = s.zt + F * 4;
    s.tmem = s.bar + NUM_BARS * 8;
    s.total = s.tmem + 16;
    return s;
}

// barrier roles here: QK_FULL / QK_EMPTY and V_FULL / V_EMPTY hold q buffers 0 / 1
__global__ void __launch_bounds__(kOutThreads, 1)
k_tc_bidir_out(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmw,
               KParams kp, const float* __restrict__ wsS, const float* __restrict__ wsZ,
               __nv_bfloat16* __restrict__ out, float* __restrict__ den, int* __restrict__ err)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* sm = aligned_smem(smem_raw);
    const SmemBidir L = smem_bidir_layout(kp.F);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + L.bar);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + L.tmem);
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int NT = kp.F / kSlice, NS = kp.F / kSub, halves = kp.F / 128;
    const Seg sg = segment_of(blockIdx.x, kp.nseg, kp.ntiles);
    // q buffer b: full / empty barriers
    auto QF = [bar](int b) { return &bar[b ? B_V_FULL : B_QK_FULL]; };
    auto QE = [bar](int b) { return &bar[b ? B_V_EMPTY : B_QK_EMPTY]; };

    if (warp == 1) {
        tmem_alloc(tslot, 256);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < NUM_BARS; ++i) mbar_init(&bar[i], 1);
        mbar_init(QE(0), 1 + 8);
        mbar_init(QE(1), 1 + 8);
        mbar_init(&bar[B_U_EMPTY0], 4);
        mbar_init(&bar[B_U_EMPTY1], 4);
        mbar_init(&bar[B_PQ_FULL0], 8);
        mbar_init(&bar[B_PQ_FULL1], 8);
        mbar_init(&bar[B_O_EMPTY], 4);
        mbar_fence_init();
        tma_prefetch_desc(&tmq);
        tma_prefetch_desc(&tmw);
    }
    {   // the state copy: columns 65..79 stay zero
        uint4* p = reinterpret_cast<uint4*>(sm + L.st);
        for (int i = tid; i < NT * kStBytes / 16; i += kOutThreads) p[i] = make_uint4(0, 0, 0, 0);
    }
    // [S | z] of the whole sequence: the sum of all its segments
    griddep_wait();   // the state kernel's sums (launched as its dependent)
    sum_segments(wsS, wsZ, sg.bh, kp.nseg, kp.nseg, kp.F, reinterpret_cast<float*>(sm + L.scr),
                 reinterpret_cast<float*>(sm + L.zt));
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    if (warp >= 12) {
        const int sp = warp & 3;
        const uint32_t row = 32u * sp + lane;
        for (int h = 0; h < halves; ++h) {
            const int f = 128 * h + row;
            uint32_t r0[32], r1[32];
            read_state_sum(reinterpret_cast<const float*>(sm + L.scr), f, r0, r1);
            write_state_row_u(sbase + L.st, kp.F, f, r0, r1, reinterpret_cast<const float*>(sm + L.zt)[f]);
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    constexpr uint32_t kColO2 = 128;   // O after the two 64-column projection buffers
    Waiter wt;
    const int64_t rowbase = static_cast<int64_t>(sg.bh) * kp.L;
    if (warp == 0) {
        if (lane == 0) {
            uint32_t ph_qe = 0, ph_we = (1u << kWSlots) - 1u;
            int n_glob = 0;
            for (int tile = sg.t_begin, it = 0; tile < sg.t_end; ++tile, ++it) {
                const int qb = it & 1;
                if (it >= 2) {
                    uint32_t ph = (ph_qe >> qb) & 1u;
                    wt.wait(QE(qb), ph);
                    ph_qe ^= 1u << qb;
                }
                mbar_arrive_expect_tx(QF(qb), kTileBytes);
                tma_load_3d(sm + L.q + qb * kTileBytes, &tmq, QF(qb), 0, tile * kTile, sg.bh);
                for (int n = 0; n < NS; ++n, ++n_glob) {
                    const int slot = n_glob % kWSlots;
                    uint32_t ph = (ph_we >> slot) & 1u;
                    wt.wait(&bar[B_W_EMPTY0 + slot], ph);
                    ph_we ^= (1u << slot);
                    mbar_arrive_expect_tx(&bar[B_W_FULL0 + slot], kWBytes);
                    tma_load_2d(sm + L.w + slot * kWBytes, &tmw, &bar[B_W_FULL0 + slot], 0, n * 64);
                }
            }
        }
    } else if (warp == 2) {
        if (lane == 0) {
            uint32_t ph_qf = 0, ph_wf = 0, ph_ue = 0x3u;
            const uint64_t dqx0 = desc_kmajor(sbase + L.q), dw0 = desc_kmajor(sbase + L.w);
            int n_glob = 0;
            for (int tile = sg.t_begin, it = 0; tile < sg.t_end; ++tile, ++it) {
                const int qb = it & 1;
                uint32_t ph = (ph_qf >> qb) & 1u;
                wt.wait(QF(qb), ph);
                ph_qf ^= 1u << qb;
                for (int n = 0; n < NS; ++n, ++n_glob) {
                    const int slot = n_glob % kWSlots, g = n & 1;
                    uint32_t pw = (ph_wf >> slot) & 1u;
                    wt.wait(&bar[B_W_FULL0 + slot], pw);
                    ph_wf ^= (1u << slot);
                    uint32_t pu = (ph_ue >> g) & 1u;
                    wt.wait(&bar[B_U_EMPTY0 + g], pu);
                    ph_ue ^= 1u << g;
                    tc_fence_after();
                    issue_projection(tmem + 64 * g, desc_add(dqx0, qb * kTileBytes), desc_add(dw0, slot * kWBytes));
                    umma_commit(&bar[B_U_FULL0 + g]);
                    umma_commit(&bar[B_W_EMPTY0 + slot]);
                }
                umma_commit(QE(qb));
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            uint32_t ph_pqf = 0, ph_oe = 0;
            constexpr uint32_t idO = idesc_bf16(128, 80, 0, 1);
            const uint64_t dq0 = desc_kmajor(sbase + L.phiq);
            const uint64_t ds0 = sdesc(sbase + L.st, 128, static_cast<uint32_t>(kp.F) * 16, kLayoutNone);
            for (int tile = sg.t_begin; tile < sg.t_end; ++tile) {
                for (int t = 0; t < NT; ++t) {
                    const int pslot = t & 1;
                    uint32_t ph = (ph_pqf >> pslot) & 1u;
                    wt.wait(&bar[B_PQ_FULL0 + pslot], ph);
                    ph_pqf ^= 1u << pslot;
                    if (t == 0 && tile > sg.t_begin) wt.wait(&bar[B_O_EMPTY], ph_oe);
                    tc_fence_after();
                    const uint64_t ad = desc_add(dq0, pslot * kTileBytes);
                    const uint64_t bs = desc_add(ds0, t * (kSlice / 8) * 128);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_bf16(tmem + kColO2, ad + 2 * kk, bs + 16 * kk, idO, (t > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&bar[B_PQ_EMPTY0 + pslot]);
                }
                umma_commit(&bar[B_TILE_DONE]);
            }
        }
    } else if (warp >= 4 && warp < 12) {
        // phi(q): group g takes the projections n = 2t + g, i.e. half g of slice t
        const int g = (warp >= 8) ? 1 : 0;
        const int sp = warp & 3;
        const uint32_t row = 32u * sp + lane;
        const uint32_t trow = tmem + ((32u * sp) << 16);
        uint32_t ph_qf = 0, ph_uf = 0, ph_pqe = 0;
        int uses0 = 0, uses1 = 0;
        for (int tile = sg.t_begin, it = 0; tile < sg.t_end; ++tile, ++it) {
            const int qb = it & 1;
            uint32_t ph = (ph_qf >> qb) & 1u;
            wt.wait(QF(qb), ph);
            ph_qf ^= 1u << qb;
            float inv, l2i;
            row_scale(sm + L.q + qb * kTileBytes + row * 128, row, inv, l2i);
            warp_arrive(QE(qb));
            for (int t = 0; t < NT; ++t) {
                const float a = slice_val(kp.a2, t) * inv, b = slice_val(kp.b2, t) + l2i;
                const int pslot = t & 1;
                wt.wait(&bar[B_U_FULL0 + g], ph_uf);
                tc_fence_after();
                uint32_t ur[32], pr[32];
                tmem_ld32(trow + 64 * g, ur);
                tmem_ld32(trow + 64 * g + 32, pr);
                tmem_wait_ld();
                reg_fence(ur);
                reg_fence(pr);
                tc_fence_before();
                warp_arrive(&bar[B_U_EMPTY0 + g]);
                int& uses = pslot ? uses1 : uses0;
                if (uses > 0) {   // both groups wait for the same completion
                    uint32_t pe = (ph_pqe >> pslot) & 1u;
                    wt.wait(&bar[B_PQ_EMPTY0 + pslot], pe);
                    ph_pqe ^= 1u << pslot;
                }
                ++uses;
                phi_sub_epilogue(ur, pr, a, b, sbase + L.phiq + pslot * kTileBytes, row, g, nullptr);
                fence_async_smem();
                warp_arrive(&bar[B_PQ_FULL0 + pslot]);
            }
        }
    } else if (warp >= 12) {
        // output: O[:, :64] / (O[:, 64] + eps)
        const int sp = warp & 3;
        const uint32_t row = 32u * sp + lane;
        const uint32_t trow = tmem + ((32u * sp) << 16);
        uint32_t ph_td = 0;
        for (int tile = sg.t_begin; tile < sg.t_end; ++tile) {
            wt.wait(&bar[B_TILE_DONE], ph_td);
            tc_fence_after();
            uint32_t o0[32], o1[32], dr;
            tmem_ld32(trow + kColO2, o0);
            tmem_ld32(trow + kColO2 + 32, o1);
            tmem_ld1(trow + kColO2 + 64, dr);
            tmem_wait_ld();
            reg_fence(o0);
            reg_fence(o1);
            reg_fence1(dr);
            tc_fence_before();
            warp_arrive(&bar[B_O_EMPTY]);
            const int grow = tile * kTile + static_cast<int>(row);
            if (grow < kp.L) finish_row(kp, o0, o1, __uint_as_float(dr), rowbase + grow, out, den);
        }
    }
    wt.report(err);
    drain_after_failure(wt.ok);
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, 256);
}

// ------------------------------------------------------------------ host side

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

// packed projection operand [F/32][64][64] bf16: per 32-feature sub-slice, 32 omega rows
// then 32 anchor rows, each row the 64 input dimensions.
bool map_w(CUtensorMap* m, const void* base, int F)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {64, static_cast<cuuint64_t>(F / kSub) * 64};
    const cuuint64_t strides[1] = {128};
    const cuuint32_t box[2] = {64, 64};
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

namespace {

// Features per launch: the whole map up to 256, else chunks of 256 (or 128 when F is not a
// multiple of 256) whose sums meet in the partial numerator / denominator buffers.
int chunk_features(int F) { return F <= 256 ? F : (F % 256 == 0 ? 256 : 128); }

}  // namespace

bool tc_supported(slay_op op, int B, int H, int L, int R, int m, bool lowmem)
{
    const int F = R * m;
    if (op != SLAY_OP_CAUSAL_FWD && op != SLAY_OP_BIDIR_FWD) return false;
    if (m % kSlice != 0 || F % 128 != 0 || F > (lowmem ? 256 : 512)) return false;
    if (static_cast<int64_t>(B) * H * L <= 0) return false;
    return smem_bytes_out(chunk_features(F)) <= 232448;
}

namespace {

// Workspace: header | per-segment S [BH][nseg][Fc][64] fp32 | z [BH][nseg][Fc] fp32 | for the
// causal forward that stores phi(k): phi(k) [BH][L][Fc] bf16 | with more than one feature
// chunk: partial numerators [BH][L][64] and denominators [BH][L] fp32.  Fc is the chunk
// width; the chunks run one after another and reuse the per-chunk parts, except in the
// two-call forward (keep_chunks), which keeps every chunk's S, z and phi(k) from the first
// call to the second: chunk c's parts start c times the per-chunk size in (chunk_parts).
struct WsLayout {
    size_t s, z, phik, num, den, total;
};

WsLayout ws_layout(int BH, int L, int F, int nseg, bool with_phik, bool keep_chunks = false)
{
    const int Fc = chunk_features(F);
    const int kept = keep_chunks ? F / Fc : 1;
    const size_t per = static_cast<size_t>(BH) * nseg * Fc * kept;
    const size_t rows = static_cast<size_t>(BH) * L;
    auto up = [](size_t b) { return (b + 255) & ~size_t(255); };
    WsLayout w;
    w.s = kWsHeader;
    w.z = w.s + up(per * 64 * sizeof(float));
    w.phik = w.z + up(per * sizeof(float));
    w.num = w.phik + up(with_phik ? rows * Fc * kept * sizeof(uint16_t) : 0);
    const bool chunked = Fc < F;
    w.den = w.num + (chunked ? up(rows * 64 * sizeof(float)) : 0);
    w.total = w.den + (chunked ? up(rows * sizeof(float)) : 0);
    return w;
}

}  // namespace

size_t tc_workspace_bytes(slay_op op, int B, int H, int L, int R, int m, bool lowmem)
{
    const int BH = B * H;
    const int nseg = choose_nseg(BH, (L + kTile - 1) / kTile);
    if (op == SLAY_OP_CAUSAL_FWD_SPLIT) return ws_layout(BH, L, R * m, nseg, true, true).total;
    if (op != SLAY_OP_CAUSAL_FWD && op != SLAY_OP_BIDIR_FWD) return 0;
    return ws_layout(BH, L, R * m, nseg, op == SLAY_OP_CAUSAL_FWD && !lowmem).total;
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
    for (int n = 0; n < F / kSub; ++n)
        for (int r = 0; r < 64; ++r) {
            const int f = n * kSub + (r & 31);
            const uint16_t* src = (r < 32) ? om : an;
            std::memcpy(wb + (static_cast<size_t>(n) * 64 + r) * D, src + static_cast<size_t>(f) * D,
                        D * sizeof(uint16_t));
        }
}

// [BH][L][F] bf16 phi(k) viewed as a 3-D tensor, 64-feature x 128-token boxes, 128-byte
// swizzle (the layout the score and state MMAs read); rows past L read as zero, stores to
// them are dropped.
bool map_phik(CUtensorMap* m, const void* base, int F, int L, int BH)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(F), static_cast<cuuint64_t>(L),
                                static_cast<cuuint64_t>(BH)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(F) * 2, static_cast<cuuint64_t>(L) * F * 2};
    const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(kTile), 1};
    const cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
              es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Launch `kernel` as the programmatic dependent of the kernel before it on `st` (it may start
// while that one finishes and waits for its results with griddep_wait).
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), int grid, int block, size_t smem, cudaStream_t st,
                             Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

template <typename K>
cudaError_t set_smem(K kernel, size_t bytes)
{
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(bytes));
}

// The state after the whole sequence for one feature chunk: S_out[bh][c0 + f][e] = S_in +
// sum over the nseg per-segment sums (every segment's sum is in the workspace when the state
// kernel ran over all of them), z likewise, added in segment order.  One thread per four
// consecutive (f, e) with 16-byte loads and stores, four segments' loads in flight before
// their adds; the thread of e = 0..3 also sums z of its f, four loads deep as well.
__global__ void k_state_total(const float* __restrict__ wsS, const float* __restrict__ wsZ, int BH,
                              int nseg, int Fc, int Ftot, int c0, const float* __restrict__ s_in,
                              const float* __restrict__ z_in, float* __restrict__ s_out,
                              float* __restrict__ z_out)
{
    const int64_t q4 = static_cast<int64_t>(Fc) * 16;   // float4s of one sequence's chunk sum
    const int64_t n = static_cast<int64_t>(BH) * q4;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int bh = static_cast<int>(i / q4);
        const int j = static_cast<int>(i % q4);   // f = j / 16, e = 4 (j % 16) .. + 3
        const float4* src = reinterpret_cast<const float4*>(wsS) + static_cast<int64_t>(bh) * nseg * q4 + j;
        const int64_t dst = (static_cast<int64_t>(bh) * Ftot + c0) * 16 + j;
        float4 a = s_in ? reinterpret_cast<const float4*>(s_in)[dst] : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        int sg = 0;
        for (; sg + 4 <= nseg; sg += 4) {
            float4 x[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) x[u] = src[(sg + u) * q4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                a.x += x[u].x; a.y += x[u].y; a.z += x[u].z; a.w += x[u].w;
            }
        }
        for (; sg < nseg; ++sg) {
            const float4 x = src[sg * q4];
            a.x += x.x; a.y += x.y; a.z += x.z; a.w += x.w;
        }
        reinterpret_cast<float4*>(s_out)[dst] = a;
        if ((j & 15) == 0) {
            const int f = j >> 4;
            const int64_t dz = static_cast<int64_t>(bh) * Ftot + c0 + f;
            const float* zs = wsZ + static_cast<int64_t>(bh) * nseg * Fc + f;
            float az = z_in ? z_in[dz] : 0.0f;
            int t = 0;
            for (; t + 4 <= nseg; t += 4) {
                float y[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) y[u] = zs[static_cast<int64_t>(t + u) * Fc];
#pragma unroll
                for (int u = 0; u < 4; ++u) az += y[u];
            }
            for (; t < nseg; ++t) az += zs[static_cast<int64_t>(t) * Fc];
            z_out[dz] = az;
        }
    }
}

namespace {

// The parameters of feature chunk c of nch (features [c Fc, (c+1) Fc), packed W sub-slices
// from c Fc / 32 on): the node scales of its 64-feature slices, where its numerators and
// denominators go (the chunk sums in the workspace while more chunks follow) and the state
// entering the sequence (sio->s_in; null: zero).
KParams chunk_kparams(const Params& P, int L, int Fc, int nch, int nseg, int ntiles, float eps,
                      int c, char* w, const WsLayout& wl, const StateIO* sio)
{
    KParams kp{};
    kp.L = L; kp.F = Fc; kp.nseg = nseg; kp.ntiles = ntiles; kp.eps = eps;
    kp.all_segs = 1;
    for (int t = 0; t < kMaxSlices; ++t) {
        const int node = t < Fc / kSlice ? (c * Fc + t * kSlice) / P.m : 0;
        kp.a2[t] = P.a2[node];
        kp.b2[t] = P.b2[node];
    }
    kp.acc_in = c > 0;
    kp.acc_out = c + 1 < nch;
    kp.part_num = nch > 1 ? reinterpret_cast<float*>(w + wl.num) : nullptr;
    kp.part_den = nch > 1 ? reinterpret_cast<float*>(w + wl.den) : nullptr;
    const int F = Fc * nch;
    kp.s_in = (sio && sio->s_in) ? sio->s_in + static_cast<size_t>(c) * Fc * 64 : nullptr;
    kp.z_in = (sio && sio->s_in) ? sio->z_in + static_cast<size_t>(c) * Fc : nullptr;
    kp.s_stride = F * 64;
    kp.z_stride = F;
    return kp;
}

bool map_chunk_w(CUtensorMap* mw, const Params& P, int Fc, int c)
{
    return map_w(mw, P.wB + static_cast<size_t>(c) * (Fc / kSub) * 64 * 64, Fc);
}

// The causal output kernel on stored phi(k) for one chunk; `dependent`: launched as the
// dependent of the state kernel just ahead of it in the stream (its prologue overlaps that
// kernel's tail), else an ordinary launch.
cudaError_t launch_out_ts(const KParams& kp, int grid, bool dependent, cudaStream_t st,
                          const CUtensorMap& mq, const CUtensorMap& mpk, const CUtensorMap& mv,
                          const CUtensorMap& mw, const float* wsS, const float* wsZ,
                          __nv_bfloat16* o, float* den, int* err)
{
    const size_t smo = smem_outts_layout(kp.F).total + 1024;
    auto kern = k_tc_causal_out_ts<0>;
    switch ((kp.acc_in ? 1 : 0) | (kp.acc_out ? 2 : 0)) {
    case 1: kern = k_tc_causal_out_ts<1>; break;
    case 2: kern = k_tc_causal_out_ts<2>; break;
    case 3: kern = k_tc_causal_out_ts<3>; break;
    default: break;
    }
    cudaError_t e = set_smem(kern, smo);
    if (e != cudaSuccess) return e;
    TraceScope trace_("tc_qphi_out", st);
    if (dependent) {
        e = launch_dependent(kern, grid, kOutThreads, smo, st, mq, mpk, mv, mw, kp, wsS, wsZ, o, den, err);
    } else {
        kern<<<grid, kOutThreads, smo, st>>>(mq, mpk, mv, mw, kp, wsS, wsZ, o, den, err);
        e = cudaSuccess;
    }
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// The state after the sequence for one chunk: s_out/z_out = s_in + the sum of every segment's
// sum (null s_in: zero).
cudaError_t launch_state_total(const float* wsS, const float* wsZ, int BH, int nseg, int Fc, int F,
                               int c, const float* s_in, const float* z_in, float* s_out,
                               float* z_out, cudaStream_t st)
{
    TraceScope trace_("tc_state_total", st);
    const int64_t n = static_cast<int64_t>(BH) * Fc * 16;   // one thread per float4
    const int grid = static_cast<int>(std::min<int64_t>((n + 255) / 256, 8 * kNumSMs));
    k_state_total<<<grid, 256, 0, st>>>(wsS, wsZ, BH, nseg, Fc, F, c * Fc, s_in, z_in, s_out, z_out);
    return cudaGetLastError();
}

// Chunk c's per-segment sums and phi(k) in the two-call forward's workspace.
struct ChunkParts {
    float* s;
    float* z;
    void* phik;
};

ChunkParts chunk_parts(char* w, const WsLayout& wl, int BH, int L, int nseg, int Fc, int c)
{
    const size_t per = static_cast<size_t>(BH) * nseg * Fc;
    const size_t rows = static_cast<size_t>(BH) * L;
    ChunkParts p;
    p.s = reinterpret_cast<float*>(w + wl.s) + static_cast<size_t>(c) * per * 64;
    p.z = reinterpret_cast<float*>(w + wl.z) + static_cast<size_t>(c) * per;
    p.phik = reinterpret_cast<uint16_t*>(w + wl.phik) + static_cast<size_t>(c) * rows * Fc;
    return p;
}

}  // namespace

size_t tc_state_workspace_bytes(int B, int H, int L, int R, int m)
{
    const int BH = B * H;
    return ws_layout(BH, L, R * m, choose_nseg(BH, (L + kTile - 1) / kTile), false).total;
}

cudaError_t tc_causal_state(const void* k, const void* v, int B, int H, int L, const Params& P,
                            void* ws, cudaStream_t st, const StateIO& sio)
{
    if (!P.wB) return cudaErrorNotSupported;
    const int BH = B * H, F = P.F, Fc = chunk_features(F), nch = F / Fc;
    const int ntiles = (L + kTile - 1) / kTile;
    const int nseg = choose_nseg(BH, ntiles);
    const WsLayout wl = ws_layout(BH, L, F, nseg, false);
    char* w = static_cast<char*>(ws);
    CUtensorMap mk, mv, mpk;
    if (!map_rows(&mk, k, L, BH) || !map_rows(&mv, v, L, BH) || !map_phik(&mpk, P.wB, Fc, 1, 1))
        return cudaErrorInvalidValue;
    int* err = reinterpret_cast<int*>(w);
    float* wsS = reinterpret_cast<float*>(w + wl.s);
    float* wsZ = reinterpret_cast<float*>(w + wl.z);
    cudaError_t e = cudaMemsetAsync(err, 0, sizeof(int), st);
    if (e != cudaSuccess) return e;
    const size_t sms = smem_bytes_state(Fc);
    if ((e = set_smem(k_tc_causal_state<false>, sms)) != cudaSuccess) return e;
    for (int c = 0; c < nch; ++c) {
        CUtensorMap mw;
        if (!map_chunk_w(&mw, P, Fc, c)) return cudaErrorInvalidValue;
        const KParams kp = chunk_kparams(P, L, Fc, nch, nseg, ntiles, 0.0f, c, w, wl, nullptr);
        {
            TraceScope trace_("tc_state_sums", st);
            k_tc_causal_state<false><<<BH * nseg, kThreads, sms, st>>>(mk, mv, mw, mpk, kp, wsS, wsZ, err);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
        }
        e = launch_state_total(wsS, wsZ, BH, nseg, Fc, F, c, sio.s_in, sio.z_in, sio.s_out, sio.z_out, st);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t tc_attn_fwd(const void* q, const void* k, const void* v, void* out, float* den, int B,
                        int H, int L, const Params& P, float eps, bool causal, void* ws,
                        cudaStream_t st, bool lowmem, const StateIO* sio)
{
    if (!P.wB) return cudaErrorNotSupported;
    const int BH = B * H, F = P.F, Fc = chunk_features(F), nch = F / Fc;
    if (lowmem && nch > 1) return cudaErrorNotSupported;
    const int ntiles = (L + kTile - 1) / kTile;
    const int nseg = choose_nseg(BH, ntiles);
    const bool store_phik = causal && !lowmem;
    const WsLayout wl = ws_layout(BH, L, F, nseg, store_phik);
    char* w = static_cast<char*>(ws);
    CUtensorMap mq, mk, mv, mpk;
    if (!map_rows(&mq, q, L, BH) || !map_rows(&mk, k, L, BH) || !map_rows(&mv, v, L, BH))
        return cudaErrorInvalidValue;
    // without stored phi(k) the state kernel never touches this map: any valid one will do
    if (!map_phik(&mpk, store_phik ? static_cast<const void*>(w + wl.phik) : P.wB, Fc,
                  store_phik ? L : 1, store_phik ? BH : 1))
        return cudaErrorInvalidValue;
    int* err = reinterpret_cast<int*>(w);
    float* wsS = reinterpret_cast<float*>(w + wl.s);
    float* wsZ = reinterpret_cast<float*>(w + wl.z);
    __nv_bfloat16* o = static_cast<__nv_bfloat16*>(out);
    cudaError_t e = cudaMemsetAsync(err, 0, sizeof(int), st);
    if (e != cudaSuccess) return e;
    const size_t sms = smem_bytes_state(Fc);
    for (int c = 0; c < nch; ++c) {
        CUtensorMap mw;
        if (!map_chunk_w(&mw, P, Fc, c)) return cudaErrorInvalidValue;
        KParams kp = chunk_kparams(P, L, Fc, nch, nseg, ntiles, eps, c, w, wl, sio);
        kp.all_segs = (causal && lowmem) ? 0 : 1;
        if (!causal) {
            // every segment's sum, then the readout against their total
            if ((e = set_smem(k_tc_causal_state<false>, sms)) != cudaSuccess) return e;
            {
                TraceScope trace_("tc_bidir_state", st);
                k_tc_causal_state<false><<<BH * nseg, kThreads, sms, st>>>(mk, mv, mw, mpk, kp, wsS, wsZ, err);
                if ((e = cudaGetLastError()) != cudaSuccess) return e;
            }
            const size_t smb = smem_bidir_layout(Fc).total + 1024;
            if ((e = set_smem(k_tc_bidir_out, smb)) != cudaSuccess) return e;
            TraceScope trace_("tc_bidir_out", st);
            e = launch_dependent(k_tc_bidir_out, BH * nseg, kOutThreads, smb, st, mq, mw, kp, wsS, wsZ, o, den, err);
            if (e != cudaSuccess) return e;
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
            continue;
        }
        if (store_phik) {
            // phi(k) and every segment's sum once; the output kernel reads phi(k)
            if ((e = set_smem(k_tc_causal_state<true>, sms)) != cudaSuccess) return e;
            {
                TraceScope trace_("tc_kphi_state", st);
                k_tc_causal_state<true><<<BH * nseg, kThreads, sms, st>>>(mk, mv, mw, mpk, kp, wsS, wsZ, err);
                if ((e = cudaGetLastError()) != cudaSuccess) return e;
            }
            e = launch_out_ts(kp, BH * nseg, true, st, mq, mpk, mv, mw, wsS, wsZ, o, den, err);
            if (e != cudaSuccess) return e;
            if (sio && sio->s_out) {   // the state after the sequence, this chunk's features
                e = launch_state_total(wsS, wsZ, BH, nseg, Fc, F, c, kp.s_in ? sio->s_in : nullptr,
                                       kp.s_in ? sio->z_in : nullptr, sio->s_out, sio->z_out, st);
                if (e != cudaSuccess) return e;
            }
            continue;
        }
        // low-memory form (no phi(k) buffer): the output kernel recomputes phi(k)
        if (nseg > 1) {
            if ((e = set_smem(k_tc_causal_state<false>, sms)) != cudaSuccess) return e;
            TraceScope trace_("tc_causal_state", st);
            k_tc_causal_state<false><<<BH * (nseg - 1), kThreads, sms, st>>>(mk, mv, mw, mpk, kp, wsS, wsZ, err);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
        }
        const size_t smo = smem_bytes_out(Fc);
        if ((e = set_smem(k_tc_causal_out, smo)) != cudaSuccess) return e;
        {
            TraceScope trace_("tc_causal_out", st);
            k_tc_causal_out<<<BH * nseg, kOutThreads, smo, st>>>(mq, mk, mv, mw, kp, wsS, wsZ, o, den, err);
        }
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t tc_attn_fwd_begin(const void* k, const void* v, int B, int H, int L, const Params& P,
                              float eps, void* ws, cudaStream_t st, float* s_out, float* z_out)
{
    if (!P.wB) return cudaErrorNotSupported;
    const int BH = B * H, F = P.F, Fc = chunk_features(F), nch = F / Fc;
    const int ntiles = (L + kTile - 1) / kTile;
    const int nseg = choose_nseg(BH, ntiles);
    const WsLayout wl = ws_layout(BH, L, F, nseg, true, true);
    char* w = static_cast<char*>(ws);
    CUtensorMap mk, mv;
    if (!map_rows(&mk, k, L, BH) || !map_rows(&mv, v, L, BH)) return cudaErrorInvalidValue;
    int* err = reinterpret_cast<int*>(w);
    cudaError_t e = cudaMemsetAsync(err, 0, sizeof(int), st);
    if (e != cudaSuccess) return e;
    const size_t sms = smem_bytes_state(Fc);
    if ((e = set_smem(k_tc_causal_state<true>, sms)) != cudaSuccess) return e;
    for (int c = 0; c < nch; ++c) {
        const ChunkParts cp = chunk_parts(w, wl, BH, L, nseg, Fc, c);
        CUtensorMap mw, mpk;
        if (!map_chunk_w(&mw, P, Fc, c) || !map_phik(&mpk, cp.phik, Fc, L, BH)) return cudaErrorInvalidValue;
        const KParams kp = chunk_kparams(P, L, Fc, nch, nseg, ntiles, eps, c, w, wl, nullptr);
        {
            TraceScope trace_("tc_kphi_state", st);
            k_tc_causal_state<true><<<BH * nseg, kThreads, sms, st>>>(mk, mv, mw, mpk, kp, cp.s, cp.z, err);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
        }
        e = launch_state_total(cp.s, cp.z, BH, nseg, Fc, F, c, nullptr, nullptr, s_out, z_out, st);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t tc_attn_fwd_finish(const void* q, const void* v, void* out, float* den, int B, int H,
                               int L, const Params& P, float eps, void* ws, cudaStream_t st,
                               const float* s_in, const float* z_in)
{
    if (!P.wB) return cudaErrorNotSupported;
    const int BH = B * H, F = P.F, Fc = chunk_features(F), nch = F / Fc;
    const int ntiles = (L + kTile - 1) / kTile;
    const int nseg = choose_nseg(BH, ntiles);
    const WsLayout wl = ws_layout(BH, L, F, nseg, true, true);
    char* w = static_cast<char*>(ws);
    CUtensorMap mq, mv;
    if (!map_rows(&mq, q, L, BH) || !map_rows(&mv, v, L, BH)) return cudaErrorInvalidValue;
    int* err = reinterpret_cast<int*>(w);
    const StateIO sio{s_in, z_in, nullptr, nullptr};
    for (int c = 0; c < nch; ++c) {
        const ChunkParts cp = chunk_parts(w, wl, BH, L, nseg, Fc, c);
        CUtensorMap mw, mpk;
        if (!map_chunk_w(&mw, P, Fc, c) || !map_phik(&mpk, cp.phik, Fc, L, BH)) return cudaErrorInvalidValue;
        const KParams kp = chunk_kparams(P, L, Fc, nch, nseg, ntiles, eps, c, w, wl, &sio);
        // ordinary launches: whatever runs just ahead (the exchange, the caller's kernels)
        // may still be writing q, v or the state the prologue reads
        cudaError_t e = launch_out_ts(kp, BH * nseg, false, st, mq, mpk, mv, mw, cp.s, cp.z,
                                      static_cast<__nv_bfloat16*>(out), den, err);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace slay
