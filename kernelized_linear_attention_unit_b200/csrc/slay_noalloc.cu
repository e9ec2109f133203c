// slay_noalloc.cu -- a causal forward for callers that cannot allocate device memory.
//
// Who needs it: a host program that owns all device memory up front -- a serving engine
// that reserves HBM for its own pool at start-up, or a plugin whose host hands it
// tensors but no workspace -- cannot let a library call cudaMalloc, and a latency-bound
// loop cannot afford the device-wide synchronisation that cudaMalloc/cudaFree may
// cause.  slay_attn_causal_fwd needs a caller-provided workspace and, on the first call
// for a parameter key, allocates the sketch-parameter cache; this entry point does
// neither.  Its scratch and its one parameter slot are file-scope __device__ arrays that
// the CUDA runtime places when the library's module is loaded on a device, and that every
// GPU which loads the library holds until the process exits (34 MiB per device).
//
// There is no counterpart on the pages of the method; it is the same computation as
// slay_attn_causal_fwd, launched through the same kernels.
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <vector>

#include "slay.h"
#include "slay_internal.h"
#include "slay_tc.h"

namespace slay {
namespace {

constexpr size_t kScratchBytes = size_t(32) << 20;  // workspace of one call
constexpr size_t kParamBytes = size_t(2) << 20;     // one sketch-parameter set (F <= 1024, D = 64)

// Device-resident storage.  In host code these names are host-side stand-ins, not device
// addresses: host code must use the addresses returned by cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];
static __device__ __align__(256) unsigned char g_params[kParamBytes];

using Key = std::tuple<int, int, int, uint64_t, uint32_t>;  // D, R, m, seed, eps bits

struct DeviceSlot {
    unsigned char* scratch = nullptr;  // device address of g_scratch on this device
    unsigned char* params = nullptr;   // device address of g_params on this device
    bool loaded = false;               // g_params holds the parameters of `key`
    Key key{};
    Params P{};
};

std::mutex g_mu;
std::map<int, DeviceSlot>& slots()
{
    static auto* m = new std::map<int, DeviceSlot>();  // held until exit
    return *m;
}

uint32_t bits_of(float x)
{
    uint32_t b;
    std::memcpy(&b, &x, sizeof b);
    return b;
}

uint16_t bf16_bits(float x)
{
    uint32_t b = bits_of(x);
    b += 0x7FFFu + ((b >> 16) & 1u);
    return static_cast<uint16_t>(b >> 16);
}

// Fill the device's parameter slot for (D, R, m, seed, eps) with a stream-ordered copy
// (layout omega^T | anchors^T | omega | anchors in fp32, then the packed bf16 operand)
// and describe it in slot->P.
slay_status load_params(DeviceSlot* slot, int D, int R, int m, uint64_t seed, float eps,
                        cudaStream_t st)
{
    const int F = R * m;
    const size_t nF = static_cast<size_t>(F) * D;
    const size_t wb_elems = tc_wb_elems(D, R, m);
    const size_t bytes = 4 * nF * sizeof(float) + wb_elems * sizeof(uint16_t);
    if (bytes > kParamBytes) return SLAY_ERR_UNSUPPORTED;
    std::vector<float> om(nF), an(nF);
    double s[kMaxR], wt[kMaxR];
    if (!draw_sketch(D, R, m, seed, static_cast<double>(eps), om.data(), an.data(), s, wt))
        return SLAY_ERR_INVALID_ARG;
    std::vector<unsigned char> host(bytes);
    float* h = reinterpret_cast<float*>(host.data());
    for (int f = 0; f < F; ++f)
        for (int d = 0; d < D; ++d) {
            h[static_cast<size_t>(d) * F + f] = om[static_cast<size_t>(f) * D + d];
            h[nF + static_cast<size_t>(d) * F + f] = an[static_cast<size_t>(f) * D + d];
        }
    std::memcpy(h + 2 * nF, om.data(), nF * sizeof(float));
    std::memcpy(h + 3 * nF, an.data(), nF * sizeof(float));
    if (wb_elems) {
        std::vector<uint16_t> omb(nF), anb(nF);
        for (size_t i = 0; i < nF; ++i) { omb[i] = bf16_bits(om[i]); anb[i] = bf16_bits(an[i]); }
        tc_pack_wb(D, R, m, omb.data(), anb.data(), reinterpret_cast<uint16_t*>(h + 4 * nF));
    }
    // Pageable source: the call returns once the bytes are staged, so `host` may go; the
    // copy is ordered after earlier work on `st`.
    cudaError_t e = cudaMemcpyAsync(slot->params, host.data(), bytes, cudaMemcpyHostToDevice, st);
    if (e != cudaSuccess) return SLAY_ERR_CUDA;
    float* d = reinterpret_cast<float*>(slot->params);
    Params& P = slot->P;
    P.omT = d;
    P.anT = d + nF;
    P.om = d + 2 * nF;
    P.an = d + 3 * nF;
    P.wB = wb_elems ? reinterpret_cast<const uint16_t*>(d + 4 * nF) : nullptr;
    P.D = D; P.R = R; P.m = m; P.F = F;
    const double log2e = 1.4426950408889634073599246810019;
    for (int r = 0; r < kMaxR; ++r) {
        if (r < R) {
            const double c = std::sqrt(wt[r] / m);
            const double sq = std::sqrt(2.0 * s[r]);
            P.a2[r] = static_cast<float>(sq * log2e);
            P.b2[r] = static_cast<float>(std::log2(c) - s[r] * log2e);
            P.sq[r] = static_cast<float>(sq);
            P.c[r] = static_cast<float>(c);
        } else {
            P.a2[r] = P.b2[r] = P.sq[r] = P.c[r] = 0.0f;
        }
    }
    slot->key = Key{D, R, m, seed, bits_of(eps)};
    slot->loaded = true;
    return SLAY_OK;
}

}  // namespace

const void* noalloc_status_word()
{
    std::lock_guard<std::mutex> lock(g_mu);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
    return slots()[dev].scratch;
}

}  // namespace slay

using namespace slay;

extern "C" slay_status slay_attn_causal_fwd_noalloc(const void* q, const void* k, const void* v,
                                                    void* out, float* den, int B, int H, int L,
                                                    int D, int Dv, slay_dtype dt, int R, int m,
                                                    uint64_t seed, float eps, void* stream)
{
    slay_status s = check_attn(q, k, v, out, B, H, L, D, Dv, dt, R, m, eps);
    if (s != SLAY_OK) return s;
    if (static_cast<int64_t>(B) * H * L == 0) return SLAY_OK;
    if (den && (reinterpret_cast<uintptr_t>(den) % 4) != 0) return SLAY_ERR_INVALID_ARG;
    // the tensor-core path runs in its low-memory form here (phi(k) recomputed, not stored)
    const bool tc = dt == SLAY_BF16 && tc_supported(SLAY_OP_CAUSAL_FWD, B, H, L, R, m, true);
    // the size of the path that runs: bf16 sizes outside the low-memory tensor-core form
    // (F > 256 among them) take the CUDA-core kernels, whose scratch is far larger than
    // the regular tensor-core workspace for the same sizes
    const size_t need = tc ? tc_workspace_bytes(SLAY_OP_CAUSAL_FWD, B, H, L, R, m, true)
                           : kWsHeader + simt_ws_causal(B, H, L, Dv, R * m);
    if (need > kScratchBytes) return SLAY_ERR_UNSUPPORTED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    std::lock_guard<std::mutex> lock(g_mu);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SLAY_ERR_CUDA;
    DeviceSlot& slot = slots()[dev];
    if (!slot.scratch) {
        // once per device, with that device current: device addresses of the arrays
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) return SLAY_ERR_CUDA;
        void* w = nullptr;
        if (cudaGetSymbolAddress(&w, g_params) != cudaSuccess || !w) return SLAY_ERR_CUDA;
        slot.scratch = static_cast<unsigned char*>(p);
        slot.params = static_cast<unsigned char*>(w);
    }
    const Key key{D, R, m, seed, bits_of(eps)};
    if (!slot.loaded || slot.key != key) {
        if ((s = load_params(&slot, D, R, m, seed, eps, st)) != SLAY_OK) return s;
    }
    cudaError_t e;
    if (tc)
        e = tc_attn_fwd(q, k, v, out, den, B, H, L, slot.P, eps, true, slot.scratch, st, true);
    else if ((e = cudaMemsetAsync(slot.scratch, 0, sizeof(int), st)) == cudaSuccess)
        e = simt_attn_fwd(q, k, v, out, den, B, H, L, dt, slot.P, eps, true,
                          slot.scratch + kWsHeader, st);
    return e == cudaSuccess ? SLAY_OK : SLAY_ERR_CUDA;
}
