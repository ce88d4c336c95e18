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
    // fp32 path: conv + L2 rows
    size_t off_qh;        // [T, Hqk, 128] fp32 conv + L2 output
    size_t off_kh;        // [T, Hqk, 128]
    size_t off_vh;        // [T, Hv, 128]
    // tensor-core path: per-chunk tiles already in the shared-memory layout of the kernels
    // that read them (so each is one contiguous bulk copy); rows past a sequence's end are 0
    size_t off_kq;        // [max_chunks, Hqk] x 64 KB: [K;Q], K-major 128B-swizzled blocks
    size_t off_kmn;       // [max_chunks, Hqk] x 32 KB: K, MN-major 32B-granule swizzle
    size_t off_vi;        // [max_chunks, Hv]  x 32 KB: V, MN-major 32B-granule swizzle
    size_t off_tb;        // [max_chunks, Hv]  x 16 KB: T diag(beta), K-major 128B-swizzled
    size_t off_pm;        // [max_chunks, Hv]  x 16 KB: P, same
    size_t off_gr;        // [max_chunks, Hv]  x 640 B: gates record (gamma[64], kd[64], gamma_C)
    size_t off_cseq;      // int32 [max_chunks]: sequence of each chunk (written by the conv pass)
    size_t off_carry;     // [n_seqs, Hv, 128, 128] fp32 state between chunk ranges (segmented
                          // tensor-core path without a caller final-state buffer), else empty
    int n_segments;       // tensor-core path: chunk ranges run as a pipeline (1 = one pass)
    size_t bytes;
};

PrefillLayout prefill_layout(int n_qk, int n_v, int64_t T, int n_seqs, bool tc);

// Few (sequence, V head) chains leave most SMs idle while they run; the chunks are then
// cut into ranges so that the conv and chunk prep of range s+1 run on the idle SMs while
// the chains run range s.
constexpr int64_t kSegMaxChains = 96;     // at most this many chains (148 SMs)
constexpr int64_t kSegMinChunks = 32;     // chunks per range at least
constexpr int kSegMax = 8;                // ranges at most
int plan_segments(int n_v, int n_seqs, int64_t max_chunks);

struct ConvParams {
    const void *q, *k, *v;                 // raw rows
    const float *wq, *wk, *wv;             // [ch, 4]
    const void *conv_in;                   // [n_seqs, 3, channels] or null
    float *qh, *kh, *vh;                   // fp32 rows (fp32 path)
    float *kq, *kmn, *vi;                  // chunk tiles (tensor-core path), or null
    int32_t *cseq;                         // chunk -> sequence table, filled with the tiles
    const int32_t *cu, *cfirst;            // workspace tables
    int n_seqs, n_qk, n_v;
    float q_scale, eps;
    int64_t chunk_lo;                      // first global chunk index of this launch
};

struct ScanParams {
    const float *qh, *kh, *vh;             // fp32 conv + L2 rows [T, H, 128] (fp32 path)
    const float *kq, *kmn, *vi;            // chunk tiles (tensor-core path)
    const void *alpha, *beta;              // [T, Hv]
    const int32_t *cu;                     // clamped bounds [n_seqs+1]
    const int32_t *cfirst;                 // first chunk index of each sequence [n_seqs+1]
    const int32_t *cseq;                   // sequence of each chunk (tensor-core path)
    float *tb, *pm, *gr;                   // chunk-prep tiles and gates records (tensor-core path)
    int64_t max_chunks;
    int64_t chunk_lo, chunk_hi;            // global chunk range of one launch (tensor-core path)
    const float *carry_in;                 // state entering a chunk range that starts inside a
                                           // sequence (the previous range's output), or null
    float *carry_out;                      // state at the end of the range (fin or a workspace copy)
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
    int n_tok;                             // multi-token decode: tokens per row (1..kMaxDecTok)
    float *state_ckpt;                     //   or null: state after each token [B, n_tok, Hv, 128, 128]
    void *conv_ckpt;                       //   or null: conv state after each token [B, n_tok, 3, ch]
};
constexpr int kMaxDecTok = 8;

// remembers `e` as this host thread's gdn_last_cuda_error()
void record_cuda_error(cudaError_t e);

// gates record of one (chunk, V head), written by the chunk prep for the chain kernel
constexpr int kGateRec = 160;            // floats: gamma_t [64], kd_t [64], gamma_C, padding
constexpr int kGrGamma = 0, kGrKd = 64, kGrGammaC = 128;

// QSA indexer launchers (qsa_indexer.cu)
cudaError_t launch_qsa_block_keys(const void *k, const float *w, const int32_t *kpos, int B, int Tn,
                                  float eps, float theta, void *kbar, int nb_max, cudaStream_t s);
cudaError_t launch_qsa_scores(const void *q, const float *w, const int32_t *qpos, const void *kbar,
                              const int32_t *n_blocks, int B, int Qn, int nb_max, float eps, float theta,
                              float *scores, int64_t ld, cudaStream_t s);
// scores rows of stride ld: a multiple of 4 floats on a 16-byte aligned base
cudaError_t launch_qsa_topk(const float *scores, int64_t ld, const int32_t *qpos, const int32_t *n_blocks, int B,
                            int Qn, int nb_max, int32_t *blocks, int32_t *tokens, cudaStream_t s);

// launchers: return the cudaError_t of the launch
cudaError_t launch_seq_table(const int32_t *cu_in, int n_seqs, int64_t T, int32_t *cu,
                             int32_t *cfirst, cudaStream_t s);
// tiles: write the tensor-core chunk tiles (TF32-rounded) instead of fp32 rows
cudaError_t launch_conv_l2(const ConvParams &p, bool bf16, bool tiles, int64_t n_chunks,
                           int64_t total_tokens, cudaStream_t s);
cudaError_t launch_conv_state_out(const void *q, const void *k, const void *v,
                                  const void *conv_in, void *conv_out, const int32_t *cu,
                                  int n_seqs, int n_qk, int n_v, bool bf16, cudaStream_t s);
cudaError_t launch_scan_simt(const ScanParams &p, bool in_bf16, bool out_bf16, cudaStream_t s);
cudaError_t launch_chunk_prep(const ScanParams &p, int64_t total_tokens, bool in_bf16, cudaStream_t s);
cudaError_t launch_prefill_tc(const ScanParams &p, int64_t total_tokens, bool in_bf16, bool out_bf16,
                              cudaStream_t s);
cudaError_t launch_decode(const DecodeParams &p, bool in_bf16, bool out_bf16, cudaStream_t s);
cudaError_t launch_decode_multi(const DecodeParams &p, bool in_bf16, bool out_bf16, cudaStream_t s);
cudaError_t launch_output_gate(const void *y, bool y_bf16, const void *z, bool z_bf16, const float *w,
                               float eps, void *out, bool out_bf16, int64_t rows, cudaStream_t s);

}  // namespace gdn
