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

// Chunk ranges of the tensor-core prefill.  The chunks of a call are processed in ranges:
// range r holds chunks [r*R, (r+1)*R) of EVERY sequence ("sliced"), so the chains of all
// sequences advance together and the tiles of one range fit a fixed number of slots; chunk j
// of sequence b lives in slot b*R + (j - r*R) of the range's buffer.  When slicing would not
// save memory (one range covers everything) the chunks are numbered globally instead
// ("compact"): chunk j of sequence b lives in slot cfirst[b] + j.
struct ChunkRange {
    int compact;   // 1: one range, global chunk numbering
    int R;         // chunks per sequence per range (sliced)
    int r;         // range index (sliced)
    int last;      // 1 for the last range
};

// Workspace carve-up and range plan of one gdn_prefill call (byte offsets from the base).
struct PrefillLayout {
    int64_t max_chunks;   // upper bound of sum_b ceil(L_b / 64)
    size_t off_cu;        // int32 [n_seqs+1]   clamped, non-decreasing sequence bounds
    size_t off_cfirst;    // int32 [n_seqs+1]   first chunk index of each sequence
    // fp32 path: conv + L2 rows
    size_t off_qh;        // [T, Hqk, 128] fp32 conv + L2 output
    size_t off_kh;        // [T, Hqk, 128]
    size_t off_vh;        // [T, Hv, 128]
    // tensor-core path: n_buf buffers of `slots` chunk slots, each holding the tiles already in
    // the shared-memory layout of the kernels that read them (one contiguous bulk copy each);
    // rows past a sequence's end are 0.  Offsets inside a buffer:
    size_t off_tiles;     // first buffer
    size_t buf_bytes;     // distance between buffers
    size_t b_kq;          // [slots, Hqk] x 64 KB: [K;Q] TF32, K-major 128B-swizzled blocks
    size_t b_kmn;         // [slots, Hqk] x 16 KB: K fp16, MN-major 32B-granule swizzle
    size_t b_vi;          // [slots, Hv]  x 16 KB: V fp16, MN-major 32B-granule swizzle
    size_t b_tb;          // [slots, Hv]  x 8 KB: T diag(beta) fp16, K-major 128B-swizzled
    size_t b_tg;          // [slots, Hv]  x 16 KB: T diag(beta gamma) TF32, K-major 128B-swizzled
    size_t b_pm;          // [slots, Hv]  x 8 KB: P fp16, K-major 128B-swizzled
    size_t b_gr;          // [slots, Hv]  x 640 B: gates record (gamma[64], kd[64], gamma_C)
    size_t b_cseq;        // int32 [slots]: sequence of each chunk (compact numbering)
    size_t off_carry;     // [n_seqs, Hv, 128, 128] fp32 state between ranges (used when the
                          // caller passes no final-state buffer), else empty
    int64_t slots;        // chunk slots per buffer
    int n_buf;            // 1, or 2 (range r+1 is prepared while the chains run range r)
    int n_ranges;
    ChunkRange range0;    // compact flag and R (r = 0)
    size_t bytes;
};

// `ws_limit`: the plan shrinks the ranges to fit this many bytes (SIZE_MAX: preferred plan);
// returns false when even one chunk per sequence per range does not fit.
bool prefill_layout(int n_qk, int n_v, int64_t T, int n_seqs, int64_t max_seqlen, bool tc,
                    size_t ws_limit, PrefillLayout *out);

// Few (sequence, V head) chains leave most SMs idle while they run: the ranges then serve to
// overlap the conv and chunk prep of range r+1 with the chains of range r, and are sized for
// that; with many chains they bound the tile memory.
constexpr int64_t kFewChains = 96;        // at most this many chains (148 SMs)
constexpr int kMaxRanges = 64;            // ranges at most (when the longest sequence is known)
constexpr int kMaxRangesUnknown = 8;      // ranges at most when it is not

struct ConvParams {
    const void *q, *k, *v;                 // raw rows
    const float *wq, *wk, *wv;             // [ch, 4]
    const void *conv_in;                   // [n_seqs, 3, channels] or null
    float *qh, *kh, *vh;                   // fp32 rows (fp32 path)
    float *kq, *kmn, *vi;                  // chunk tiles (tensor-core path), or null
    int32_t *cseq;                         // slot -> sequence table (compact numbering)
    const int32_t *cu, *cfirst;            // workspace tables
    int n_seqs, n_qk, n_v;
    float q_scale, eps;
    int act;                               // 1: SiLU on the conv outputs
    ChunkRange rg;                         // tile path: the range this launch prepares
    int64_t slots;                         // tile path: slots of the range (grid x)
};

struct ScanParams {
    const float *qh, *kh, *vh;             // fp32 conv + L2 rows [T, H, 128] (fp32 path)
    const float *kq, *kmn, *vi;            // chunk tiles (tensor-core path)
    const void *alpha, *beta;              // [T, Hv]
    const int32_t *cu;                     // clamped bounds [n_seqs+1]
    const int32_t *cfirst;                 // first chunk index of each sequence [n_seqs+1]
    const int32_t *cseq;                   // slot -> sequence (tensor-core path, compact numbering)
    float *tb, *tg, *pm, *gr;              // chunk-prep tiles and gates records (tensor-core path)
    int64_t max_chunks;
    ChunkRange rg;                         // tensor-core path: the range of this launch
    int64_t slots;                         // its slots
    const float *carry_in;                 // state entering a range that starts inside a
                                           // sequence (the previous range's output), or null
    float *carry_out;                      // state at the end of the range (fin or a workspace copy)
    const float *init;                     // [n_seqs, Hv, 128, 128] or null
    float *fin;                            // or null
    void *out;                             // [T, Hv, 128]
    int n_seqs, n_qk, n_v;
    // gated output (tensor-core path): out = y / sqrt(mean(y^2) + gate_eps) * gate_w * SiLU(z)
    const void *gate_z;                    // [T, Hv, 128] or null (plain y)
    bool gate_z_bf16;
    const float *gate_w;                   // [128]
    float gate_eps;
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
    int act;                               // 1: SiLU on the conv outputs
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
// tiles: write the tensor-core chunk tiles ([K;Q] TF32-rounded, K and V fp16) instead of fp32 rows
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
cudaError_t launch_affine_combine(const float *M, const float *B, const float *S0, float *S_in, int n_spans,
                                  int n_v, cudaStream_t s);
cudaError_t launch_output_gate(const void *y, bool y_bf16, const void *z, bool z_bf16, const float *w,
                               float eps, void *out, bool out_bf16, int64_t rows, cudaStream_t s);

}  // namespace gdn
