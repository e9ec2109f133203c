// slay_tc.cu -- tensor-core path (tcgen05 / TMEM / TMA) for bf16 inputs.
#include "slay_tc.h"

namespace slay {

bool tc_supported(slay_op, int, int, int, int, int) { return false; }
size_t tc_workspace_bytes(slay_op, int, int, int, int, int) { return 0; }
size_t tc_wb_elems(int, int, int) { return 0; }
void tc_pack_wb(int, int, int, const uint16_t*, const uint16_t*, uint16_t*) {}
cudaError_t tc_feature_map(const void*, void*, int64_t, const Params&, cudaStream_t)
{
    return cudaErrorNotSupported;
}
cudaError_t tc_attn_fwd(const void*, const void*, const void*, void*, float*, int, int, int,
                        const Params&, float, bool, void*, cudaStream_t)
{
    return cudaErrorNotSupported;
}

}  // namespace slay
