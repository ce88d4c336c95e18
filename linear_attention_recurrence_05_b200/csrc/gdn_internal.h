// Host-side declarations shared by the libgdn translation units (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "libgdn.h"

namespace gdn {

// Brackets one kernel launch with the active launch trace of this host thread (if any).
struct TraceLaunch {
    TraceLaunch(cudaStream_t s, const char *kernel);
    ~TraceLaunch();
    cudaStream_t stream;
    gdn_trace_entry *entry;
};

// Workspace carve-up of one gdn_prefill call (byte offsets from the workspace base).
struct PrefillLayout {
    int64_t max_chunks;   // upper bound of sum_b ceil(L_b / 64)
    size_t off_cu;        // int32 [n_seqs+1]   clamped, non-decreasing sequence bounds
    size_t off_cfirst;    // int32 [n_seqs+1]   first chunk index of each sequence
    size_t off_qh;        // [T, Hqk, 128] fp32 conv + L2 output
    size_t off_kh;        // [T, Hqk, 128]
    size_t off_vh;        // [T, Hv, 128]
    size_t off_tb;        // tensor-core path: [max_chunks, Hv, 64, 64] fp32 T diag(beta) tiles
    size_t off_pm;        // tensor-core path: [max_chunks, Hv, 64, 64] fp32 P tiles
    size_t bytes;
};

PrefillLayout prefill_layout(int n_qk, int n_v, int64_t T, int n_seqs, bool tc);

struct ConvParams {
    const void *q, *k, *v;                 // raw rows
    const float *wq, *wk, *wv;             // [ch, 4]
    const void *conv_in;                   // [n_seqs, 3, channels] or null
    float *qh, *kh, *vh;                   // fp32 outputs
    const int32_t *cu, *cfirst;            // workspace tables
    int n_seqs, n_qk, n_v;
    float q_scale, eps;
};

struct ScanParams {
    const float *qh, *kh, *vh;             // fp32 conv + L2 rows [T, H, 128]
    const void *alpha, *beta;              // [T, Hv]
    const int32_t *cu;                     // clamped bounds [n_seqs+1]
    const int32_t *cfirst;                 // first chunk index of each sequence [n_seqs+1]
    float *tb, *pm;                        // chunk-prep tiles (tensor-core path)
    int64_t max_chunks;
    const float *init;                     // [n_seqs, Hv, 128, 128] or null
    float *fin;                            // or null
    void *out;                             // [T, Hv, 128]
    int n_seqs, n_qk, n_v;
};

struct DecodeParams {
    const void *q, *k, *v;
    const float *wq, *wk, *wv;
    const void *alpha, *beta;
    float *state;
    void *conv;
    const int32_t *slots;
    int n_rows, batch, n_qk, n_v;
    float q_scale, eps;
    void *out;
};

// remembers `e` as this host thread's gdn_last_cuda_error()
void record_cuda_error(cudaError_t e);

// launchers: return the cudaError_t of the launch
cudaError_t launch_seq_table(const int32_t *cu_in, int n_seqs, int64_t T, int32_t *cu,
                             int32_t *cfirst, cudaStream_t s);
cudaError_t launch_conv_l2(const ConvParams &p, bool bf16, bool tf32, int64_t max_chunks,
                           cudaStream_t s);
cudaError_t launch_conv_state_out(const void *q, const void *k, const void *v,
                                  const void *conv_in, void *conv_out, const int32_t *cu,
                                  int n_seqs, int n_qk, int n_v, bool bf16, cudaStream_t s);
cudaError_t launch_scan_simt(const ScanParams &p, bool in_bf16, bool out_bf16, cudaStream_t s);
cudaError_t launch_chunk_prep(const ScanParams &p, int64_t total_tokens, bool in_bf16, cudaStream_t s);
cudaError_t launch_prefill_tc(const ScanParams &p, int64_t total_tokens, bool in_bf16, bool out_bf16,
                              cudaStream_t s);
cudaError_t launch_decode(const DecodeParams &p, bool in_bf16, bool out_bf16, cudaStream_t s);

}  // namespace gdn
