// slay_tc.h -- tensor-core (tcgen05/TMEM, TMA) path of libslay.so for bf16 inputs.
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

#include "slay.h"
#include "slay_internal.h"

namespace slay {

// Whether the tensor-core path takes this op at these sizes (bf16 mode only); F up to 512
// (as feature chunks of at most 256), or up to 256 in the low-memory form (lowmem).
bool tc_supported(slay_op op, int B, int H, int L, int R, int m, bool lowmem = false);
// Workspace bytes of the tensor-core path.  The causal forward stores phi(k) ([BH][L][F]
// bf16) unless `lowmem`, where the output kernel recomputes it instead.
size_t tc_workspace_bytes(slay_op op, int B, int H, int L, int R, int m, bool lowmem = false);
// Elements of the packed bf16 projection operand (0 when the path is not built).
size_t tc_wb_elems(int D, int R, int m);
// Pack bf16 omega / anchors ([F][D] row-major bit patterns) into the operand layout.
void tc_pack_wb(int D, int R, int m, const uint16_t* om, const uint16_t* an, uint16_t* wb);

// Feature map bf16 -> bf16 on tensor cores: D == 64, m % 32 == 0, F % 128 == 0, F <= 512.
bool tc_fmap_supported(int D, int R, int m, int64_t n_rows);
cudaError_t tc_feature_map(const void* x, void* phi, int64_t n, const Params& P, cudaStream_t st);
// Backward of the feature map on tensor cores (bf16 x, bf16 dphi [n][F] -> fp32 dx [n][64]):
// same sizes as the forward map.
bool tc_phi_bwd_supported(int D, int R, int m, int64_t n_rows);
// dphi is [n][F] bf16 (as the tensor-core contraction stores it)
cudaError_t tc_phi_bwd(const void* x, const void* dphi, float* dx, int64_t n, const Params& P,
                       cudaStream_t st);
// Causal backward on tensor cores over 128-token tiles (bf16 phi, v and dn rows, fp32 delta):
// the sums of phi(k) [v, 1] over the tokens before each tile and of phi(q) [dn, delta] over
// the tokens after it, then the contraction -> dphi(q), dphi(k), dv.
bool tc_bwd_tile_supported(int F, int L);
// The contraction's S_c and G_c in one launch: per (sequence, 128-feature block, sum) the
// tiles walked in order with the running sums on chip, written per tile as the contraction's
// operand slabs: [64 f][64 e] bf16 and z fp32 per 64 features, 65 x 64 floats apart (bidir:
// the whole-sequence sums into tot_s, tot_g).
// Sums over the tokens outside a piece of the sequence (sequence parallelism): s_in, z_in
// the S sums before it, g_in, zg_in the G sums after it ([BH][F][64], [BH][F] fp32; null =
// zero); g_out, zg_out: the piece's G total in fp32 (null = not wanted); sums: bit 0 S,
// bit 1 G (only those CTAs run).
struct BwdSeeds {
    const float* s_in = nullptr;
    const float* z_in = nullptr;
    const float* g_in = nullptr;
    const float* zg_in = nullptr;
    float* g_out = nullptr;
    float* zg_out = nullptr;
    int sums = 3;
};
cudaError_t tc_bwd_sums(const void* phq, const void* phk, const void* v, const void* dn16,
                        const float* delta, float* st_s, float* st_g, float* tot_s, float* tot_g,
                        int BH, int L, int F, bool bidir, int* err, cudaStream_t st,
                        const BwdSeeds* seeds = nullptr);
// bidir: the bidirectional form (no masked term; sfw, gbw are each sequence's whole sums).
// sfw, gbw hold tc_bwd_sums' operands.
cudaError_t tc_bwd_tile(const void* phq, const void* phk, const void* v, const void* dn16,
                        const float* delta, const float* sfw, const float* gbw, void* dphq,
                        void* dphk, bool dphi_bf16, float* dv, int BH, int L, int F, int* err,
                        cudaStream_t st, bool bidir = false);
// Test hook: the next tensor-core feature-map launch withholds one barrier arrival and
// bounds its waits at 1 ms, so that a wait runs out (on != 0 arms it, 0 disarms it).
void fmap_arm_wait_fault(int on);
// Device address of the status word of the feature-map kernels, forward and backward (set
// when a bounded wait ran out).
const void* fmap_status_word();
// A causal forward continued from a state and / or returning the final one: S [BH][F][64],
// z [BH][F] fp32 (s_in null: zero state; s_out null: not written).
struct StateIO {
    const float* s_in;
    const float* z_in;
    float* s_out;
    float* z_out;
};
cudaError_t tc_attn_fwd(const void* q, const void* k, const void* v, void* out, float* den,
                        int B, int H, int L, const Params& P, float eps, bool causal, void* ws,
                        cudaStream_t st, bool lowmem = false, const StateIO* sio = nullptr);
// The causal forward in two calls on one workspace (tc_workspace_bytes of
// SLAY_OP_CAUSAL_FWD_SPLIT): begin runs the state kernel over every segment of every feature
// chunk (phi(k) and the segment sums kept in the workspace) and writes the sequence's state
// into s_out, z_out; finish runs the output kernels on them from the state s_in, z_in (null:
// zero).  finish leaves the status word as begin set it.
cudaError_t tc_attn_fwd_begin(const void* k, const void* v, int B, int H, int L, const Params& P,
                              float eps, void* ws, cudaStream_t st, float* s_out, float* z_out);
cudaError_t tc_attn_fwd_finish(const void* q, const void* v, void* out, float* den, int B, int H,
                               int L, const Params& P, float eps, void* ws, cudaStream_t st,
                               const float* s_in, const float* z_in);

// The state of a whole sequence on tensor cores (k projections, phi(k) and per-segment sums
// by the state kernel over every segment, then their total plus sio.s_in into sio.s_out).
size_t tc_state_workspace_bytes(int B, int H, int L, int R, int m);
cudaError_t tc_causal_state(const void* k, const void* v, int B, int H, int L, const Params& P,
                            void* ws, cudaStream_t st, const StateIO& sio);

}  // namespace slay
