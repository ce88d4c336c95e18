// gdn_prefill_static_scratch: gdn_prefill for callers that cannot allocate device memory.
//
// Some callers have no way to call cudaMalloc when they run the mixer: a plugin whose
// host framework forbids device allocation inside its execute step, a runtime that
// reserves all device memory up front, or plain C code with no allocator at hand
// (cudaMalloc may also synchronise the device, which latency-bound callers avoid).
// This entry point takes the same inputs and outputs as gdn_prefill but keeps its
// scratch in a fixed array in device memory that the library owns, so it allocates
// nothing per call.
#include <mutex>

#include "gdn_internal.h"
#include "libgdn.h"

namespace {

// The scratch: one array per GPU on which this library's module is loaded, held
// until the process exits.  In host code `g_static_scratch` is only a host-side
// stand-in for the symbol; its device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_static_scratch[GDN_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_addr[kMaxDevices] = {};

}  // namespace

extern "C" gdn_status gdn_prefill_static_scratch(
    const gdn_config *cfg, gdn_dtype dtype, gdn_dtype out_dtype, const void *q, const void *k,
    const void *v, const float *conv_w_q, const float *conv_w_k, const float *conv_w_v,
    const void *alpha, const void *beta, const int32_t *cu_seqlens, int n_seqs,
    int64_t total_tokens, const float *initial_state, float *final_state,
    const void *conv_state_in, void *conv_state_out, void *out, cudaStream_t stream) {
    size_t need = 0;
    gdn_status st = gdn_prefill_workspace_size(cfg, dtype, total_tokens, n_seqs, 0, &need);
    if (st != GDN_OK) return st;
    // too large even with the shortest chunk ranges: rejected before anything else
    gdn::PrefillLayout plan;
    if (n_seqs > 0 && !gdn::prefill_layout(cfg->n_qk_heads, cfg->n_v_heads, total_tokens, n_seqs, 0,
                                           dtype == GDN_BF16, (size_t)GDN_STATIC_SCRATCH_BYTES, &plan))
        return GDN_ERR_WORKSPACE;

    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        gdn::record_cuda_error(e);
        return GDN_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return GDN_ERR_UNSUPPORTED;
    void *scratch = nullptr;
    {
        // set-up, once per device, with that device current: the array's device address
        std::lock_guard<std::mutex> lock(g_mu);
        if (!g_scratch_addr[dev]) {
            void *p = nullptr;
            e = cudaGetSymbolAddress(&p, g_static_scratch);
            if (e != cudaSuccess || p == nullptr) {
                gdn::record_cuda_error(e != cudaSuccess ? e : cudaErrorInvalidSymbol);
                return GDN_ERR_CUDA;
            }
            g_scratch_addr[dev] = p;
        }
        scratch = g_scratch_addr[dev];
    }
    // Every byte of the scratch that gdn_prefill reads is written earlier in the same
    // call (sequence tables, then the tiles of each chunk range, then the carried states),
    // so nothing has to be cleared.
    return gdn_prefill(cfg, dtype, out_dtype, q, k, v, conv_w_q, conv_w_k, conv_w_v, alpha, beta,
                       cu_seqlens, n_seqs, total_tokens, 0, initial_state, final_state, conv_state_in,
                       conv_state_out, out, scratch, (size_t)GDN_STATIC_SCRATCH_BYTES, stream);
}
