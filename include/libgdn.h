/*
 * libgdn.h -- Gated DeltaNet (GDN) token mixer for NVIDIA B200 (sm_100a).
 *
 * The operation (page "ARCHITECTURE PREVIEW / FIELD NOTES", section 03 "Attention",
 * the GDN figure caption and the "GATED DELTANET" equations; section 01 config
 * table for the shapes: 48 value heads, 16 QK heads, head dim 128, conv kernel 4):
 *
 *   per token t of a sequence, raw rows q_t, k_t [Hqk, dk] and v_t [Hv, dv]:
 *     ShortConv   x'_t[c] = sum_{j=0..3} w[c][j] * x_{t-3+j}[c]   on every q, k, v channel
 *                 (causal, depthwise, tap 3 on the current row, no bias; no activation
 *                  unless cfg->conv_activation asks for SiLU; rows before the sequence
 *                  start come from the conv state, else zero)
 *     L2 norm     q^ = q' * q_scale / sqrt(|q'|^2 + l2_eps),  k^ = k' / sqrt(|k'|^2 + l2_eps)
 *                 per (token, QK head); v^ = v'
 *   per value head h, reading QK head g = h / (Hv / Hqk), with state S [dk][dv] (fp32):
 *     S~  = alpha_t S_{t-1}
 *     e_t = v^_t - S~^T k^_t
 *     S_t = S~ + beta_t k^_t e_t^T
 *     y_t = S_t^T q^_t                       (the read uses the updated state)
 *
 * Conventions shared by every entry point
 *  - Ownership: every buffer is a DEVICE pointer owned by the caller.  The library
 *    allocates no device memory for its data and calls on different streams are
 *    independent as long as their buffers do not overlap, with two exceptions, each
 *    described at its entry point: gdn_prefill keeps one auxiliary stream and five events
 *    per (host thread, device) for its chunk ranges (see "Auxiliary stream" there), and
 *    gdn_prefill_static_scratch shares one library-owned scratch array among all its
 *    calls on a device (see "Sharing" there).
 *  - Asynchrony: every call only enqueues work on `stream` (0 = legacy default stream)
 *    and returns; nothing synchronises.  Kernel faults surface at the caller's next
 *    synchronisation.
 *  - Validation: all argument checks run on the host before any launch; on failure
 *    nothing is enqueued and nothing is written.  Values stored in device memory
 *    (cu_seqlens, state_slots) cannot be checked on the host: the kernels clamp them
 *    so that no access leaves the buffers the host-side sizes describe.
 *  - Layout: token-major, row-major, innermost dimension last and contiguous.
 *  - Supported: d_k = d_v = 128, conv_width = 4, n_v_heads a multiple of n_qk_heads,
 *    compute capability 10.0 (B200).  Anything else returns GDN_ERR_UNSUPPORTED.
 *  - Errors: a failed launch returns GDN_ERR_CUDA; gdn_last_cuda_error() then gives
 *    the cudaError_t of the failing call (per host thread).
 */
#ifndef LIBGDN_H
#define LIBGDN_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GDN_API_VERSION 2

#if defined(__GNUC__)
#define GDN_EXPORT __attribute__((visibility("default")))
#else
#define GDN_EXPORT
#endif

typedef enum {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size, inconsistent config */
    GDN_ERR_UNSUPPORTED = 2,   /* shape or device this build does not implement */
    GDN_ERR_WORKSPACE = 3,     /* workspace missing, misaligned or too small */
    GDN_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed */
    GDN_ERR_TIMEOUT = 5        /* reserved: a bounded device-side wait gave up */
} gdn_status;

typedef enum {
    GDN_BF16 = 0,  /* bfloat16 storage */
    GDN_F32 = 1    /* float32 storage */
} gdn_dtype;
/* Every call takes two storage types: `dtype` for q, k, v, alpha, beta and the conv
 * state (the raw inputs), and `out_dtype` for y.  Whatever they are, accumulation and states
 * are fp32; the tensor-core products of the bf16 path take operands with an 11-bit
 * significand (TF32 for the state products and their [K;Q] and T_beta_gamma tiles, fp16 for
 * the other chunk tiles and the per-chunk vectors u), and the fp32 path computes in fp32 on
 * the CUDA cores.
 * Note on precision: rounding y to bfloat16 alone moves its largest entries by up to
 * 2^-9 of their magnitude, which on typical data is 2-3% of rms(y); use
 * out_dtype = GDN_F32 where y must stay within 1e-2 of rms(y) of the exact result. */

/* Activation of the ShortConv outputs (gdn_config.conv_activation).  The page names none
 * (GDN_ACT_NONE, the default reading); GDN_ACT_SILU applies SiLU(x) = x / (1 + e^-x) to every
 * conv output of q, k and v, before the L2 normalisation of q and k. */
typedef enum { GDN_ACT_NONE = 0, GDN_ACT_SILU = 1 } gdn_activation;

typedef struct {
    int n_qk_heads;   /* Hqk: QK heads (16 in the pages' layer)                      */
    int n_v_heads;    /* Hv: value heads (48); V head h reads QK head h/(Hv/Hqk)     */
    int d_k;          /* key/query head dim, must be 128                             */
    int d_v;          /* value head dim, must be 128                                 */
    int conv_width;   /* ShortConv kernel size, must be 4                            */
    float q_scale;    /* multiplies q^ after normalisation (1.0: the page has none)  */
    float l2_eps;     /* epsilon inside the L2 norm's square root (1e-6)             */
    int conv_activation;  /* gdn_activation of the conv outputs (GDN_ACT_NONE)       */
} gdn_config;

/* Human-readable name of a status code (static storage, never NULL). */
GDN_EXPORT const char *gdn_status_string(gdn_status status);

/* cudaError_t (as int) of the last CUDA failure seen by a libgdn call on this host thread. */
GDN_EXPORT int gdn_last_cuda_error(void);

/* GDN_API_VERSION of the loaded library. */
GDN_EXPORT int gdn_api_version(void);

/*
 * gdn_prefill_workspace_size -- bytes of device workspace that gdn_prefill prefers for
 * `total_tokens` tokens packed into `n_seqs` sequences, the longest of which has at most
 * `max_seqlen` tokens (0 = not known: total_tokens).  Writes *bytes.
 * The workspace is scratch only (no state persists between calls) and must not be shared
 * by two calls in flight.  For bf16 input it holds the sequence tables and the per-chunk
 * tiles of the tensor-core path for one or two chunk RANGES: range r covers chunks
 * [r*R, (r+1)*R) of every sequence (R chosen from n_seqs and max_seqlen), so its size grows
 * with n_seqs * R, not with total_tokens (about 3.7 MB per (sequence, chunk slot) at 16 QK /
 * 48 V heads, plus one fp32 state per (sequence, V head) carried between ranges).  Only when
 * one range covers the whole problem is it sized by the number of chunks instead.  For fp32
 * input (the fp32 CUDA-core path) it holds the convolved, normalised rows in fp32 (40 KB per
 * token at 16 QK / 48 V heads).
 */
GDN_EXPORT gdn_status gdn_prefill_workspace_size(const gdn_config *cfg, gdn_dtype dtype,
                                      int64_t total_tokens, int n_seqs, int64_t max_seqlen,
                                      size_t *bytes);

/*
 * gdn_prefill -- the mixer over packed variable-length sequences (chunked prefill).
 *
 * Page: "ARCHITECTURE PREVIEW / FIELD NOTES", section 03 (the GATED DELTANET
 * equations and the ShortConv of the GDN figure); chunked prefill is named in
 * section 03's performance note.  Internally the recurrence runs in chunks of
 * 64 tokens (WY/UT form: intra-chunk triangular solve, inter-chunk state scan),
 * which reaches the same result as the token-by-token recurrence up to rounding.
 *
 *   q, k            [T, Hqk, 128]  raw (pre-conv) rows, dtype      16-byte aligned
 *   v               [T, Hv, 128]   raw rows, dtype                 16-byte aligned
 *   conv_w_q, conv_w_k [Hqk*128, 4], conv_w_v [Hv*128, 4]  fp32, tap 3 = current row
 *   alpha, beta     [T, Hv] dtype: decay in (0, 1] and write strength, one per (token, V head)
 *   cu_seqlens      [n_seqs+1] int32 device: sequence b is rows cu[b] .. cu[b+1]-1;
 *                   non-decreasing, cu[0] = 0, cu[n_seqs] = total_tokens.  Zero-length
 *                   sequences are allowed (their final state equals the initial one).
 *                   Out-of-order values are clamped on the device, never dereferenced.
 *   total_tokens    T (>= 0, < 2^31)
 *   max_seqlen      an upper bound of the longest sequence's length, known on the host
 *                   (0 = not known: T).  It sets how many chunk ranges the call launches;
 *                   a sequence longer than the bound passed may get NaN for its tokens past
 *                   the bound and for its final state (never anything else).
 *   initial_state   [n_seqs, Hv, 128(dk), 128(dv)] fp32, dv fastest; NULL = zero state
 *   final_state     same shape; NULL = not returned; may alias initial_state
 *   conv_state_in   [n_seqs, 3, 2*Hqk*128 + Hv*128] dtype: the last 3 raw rows
 *                   (q | k | v channels), oldest first; NULL = zero history
 *   conv_state_out  same shape; NULL = not returned; may alias conv_state_in
 *   out             [T, Hv, 128] out_dtype: y
 *   workspace       256-byte aligned; gdn_prefill_workspace_size() bytes, or fewer: with
 *                   bf16 input a smaller workspace makes the chunk ranges shorter (more of
 *                   them, same results), down to one chunk per sequence per range;
 *                   GDN_ERR_WORKSPACE when even that does not fit
 * Returns GDN_OK after enqueueing; n_seqs == 0 or T == 0 with no states is a no-op.
 * Auxiliary stream: a bf16 call with more than one chunk range makes the tiles of range
 * r+1 on an auxiliary stream while the chains of range r run on `stream` (events order the
 * two).  The stream and five events are created by the first such call of a host thread on
 * a device (make it before any stream capture on that device) and kept until the process
 * exits.  Such calls of one host thread share that stream, so their tile work runs in
 * call order even when the calls use different streams.
 */
GDN_EXPORT gdn_status gdn_prefill(const gdn_config *cfg, gdn_dtype dtype, gdn_dtype out_dtype,
                       const void *q, const void *k, const void *v,
                       const float *conv_w_q, const float *conv_w_k, const float *conv_w_v,
                       const void *alpha, const void *beta,
                       const int32_t *cu_seqlens, int n_seqs, int64_t total_tokens,
                       int64_t max_seqlen,
                       const float *initial_state, float *final_state,
                       const void *conv_state_in, void *conv_state_out,
                       void *out, void *workspace, size_t workspace_bytes,
                       cudaStream_t stream);

/*
 * gdn_prefill_gated -- gdn_prefill with the mixer's output tail fused into the store of y
 * (page "ARCHITECTURE PREVIEW / FIELD NOTES", section 03, GDN figure caption: the readout
 * passes a normalisation and an output gate before the output projection; the page gives no
 * formula, this is the plainest reading, the same as gdn_output_gate's):
 *     out_t = y_t / sqrt(mean(y_t^2) + norm_eps) * norm_w * SiLU(z_t)   per (token, V head)
 * y never reaches memory.  Arguments as gdn_prefill, plus
 *   z         [T, Hv, 128] z_dtype: the output-gate input, 16-byte aligned
 *   norm_w    [128] fp32 (shared by the V heads), 16-byte aligned
 *   norm_eps  >= 0, finite
 *   out       [T, Hv, 128] out_dtype: the gated output
 * With fp32 input (the fp32 CUDA-core path) y is first written to `out` and the tail then
 * runs in place, so out_dtype must be GDN_F32 there (GDN_ERR_UNSUPPORTED otherwise).
 * Precision (bf16 input): SiLU is taken from the hardware tanh, z/2 (1 + tanh(z/2)), whose
 * error is at most |z| 2^-12 in absolute terms (gdn_output_gate uses the exponential); the
 * rest of the tail is fp32.
 */
GDN_EXPORT gdn_status gdn_prefill_gated(const gdn_config *cfg, gdn_dtype dtype, gdn_dtype out_dtype,
                             const void *q, const void *k, const void *v,
                             const float *conv_w_q, const float *conv_w_k, const float *conv_w_v,
                             const void *alpha, const void *beta,
                             const int32_t *cu_seqlens, int n_seqs, int64_t total_tokens,
                             int64_t max_seqlen,
                             const float *initial_state, float *final_state,
                             const void *conv_state_in, void *conv_state_out,
                             const void *z, gdn_dtype z_dtype, const float *norm_w, float norm_eps,
                             void *out, void *workspace, size_t workspace_bytes,
                             cudaStream_t stream);

/*
 * gdn_decode_step -- one token for each of `batch` sequences whose states stay
 * resident in device memory (the one-token case of the same recurrence: the
 * GATED DELTANET equations of section 03 with the ShortConv history shifted by one
 * row).  Each state is read once and written once, in place.
 *
 *   q, k            [batch, Hqk, 128] raw rows, dtype; v [batch, Hv, 128]
 *   conv_w_*        as in gdn_prefill
 *   alpha, beta     [batch, Hv] dtype
 *   state           [n_state_rows, Hv, 128, 128] fp32, updated in place
 *   conv_state      [n_state_rows, 3, 2*Hqk*128 + Hv*128] dtype, updated in place
 *                   (shifted by one row, the current raw row appended); NULL = zero
 *                   history and nothing written
 *   state_slots     [batch] int32 device, NULL = identity: row b uses state row
 *                   state_slots[b] (and the same conv-state row).  Slots of one call
 *                   must be distinct; a slot outside [0, n_state_rows) skips the row
 *                   (its out row is written as zeros, no state is touched).
 *   n_state_rows    rows in state / conv_state (>= batch when state_slots is NULL)
 *   out             [batch, Hv, 128] out_dtype: y
 */
GDN_EXPORT gdn_status gdn_decode_step(const gdn_config *cfg, gdn_dtype dtype, gdn_dtype out_dtype,
                           const void *q, const void *k, const void *v,
                           const float *conv_w_q, const float *conv_w_k, const float *conv_w_v,
                           const void *alpha, const void *beta,
                           float *state, void *conv_state,
                           const int32_t *state_slots, int n_state_rows,
                           void *out, int batch, cudaStream_t stream);

/*
 * gdn_decode_multi -- n_tok consecutive tokens for each of `batch` sequences whose states
 * stay resident (the verification step of speculative or multi-token decoding): the same
 * recurrence as gdn_decode_step, run over each row's tokens in order, token 0 first.  Each
 * state is read once and written once per call whatever n_tok is; optionally the state
 * and conv state after every token are written out, so that a caller that accepts only the
 * first m tokens can restore the row from checkpoint m-1 (no counterpart on the pages
 * beyond their use of multi-token speculative decoding).
 *
 *   q, k            [batch, n_tok, Hqk, 128] raw rows, dtype; v [batch, n_tok, Hv, 128]
 *   conv_w_*        as in gdn_prefill
 *   alpha, beta     [batch, n_tok, Hv] dtype
 *   state, conv_state, state_slots, n_state_rows
 *                   as in gdn_decode_step; both advance by all n_tok tokens
 *   state_ckpt      [batch, n_tok, Hv, 128, 128] fp32 or NULL: the state of row b after its
 *                   token j at [b][j] (not written for skipped rows)
 *   conv_ckpt       [batch, n_tok, 3, 2*Hqk*128 + Hv*128] dtype or NULL: the conv state
 *                   after token j (its last three raw rows, oldest first)
 *   out             [batch, n_tok, Hv, 128] out_dtype: y of every token
 *   n_tok           1 .. 8 (GDN_ERR_UNSUPPORTED above)
 * Errors as gdn_decode_step; the checkpoints must not overlap state or conv_state.
 */
GDN_EXPORT gdn_status gdn_decode_multi(const gdn_config *cfg, gdn_dtype dtype, gdn_dtype out_dtype,
                            const void *q, const void *k, const void *v,
                            const float *conv_w_q, const float *conv_w_k, const float *conv_w_v,
                            const void *alpha, const void *beta,
                            float *state, void *conv_state,
                            const int32_t *state_slots, int n_state_rows,
                            float *state_ckpt, void *conv_ckpt,
                            void *out, int batch, int n_tok, cudaStream_t stream);

/*
 * gdn_output_gate -- the mixer's output tail: gated RMS normalisation of y, per (token,
 * V head) over its 128 values (page "ARCHITECTURE PREVIEW / FIELD NOTES", section 03: the
 * readout passes a normalisation and an output gate before the output projection; the page
 * gives no formula, this is its plainest reading):
 *     out = y / sqrt(mean(y^2) + eps) * norm_w * SiLU(z),   SiLU(z) = z / (1 + exp(-z))
 *
 *   y        [n_tokens, Hv, 128] y_dtype (gdn_prefill's or gdn_decode_*'s out)
 *   z        [n_tokens, Hv, 128] z_dtype: the output-gate input
 *   norm_w   [128] fp32, shared by the V heads
 *   eps      >= 0, finite
 *   out      [n_tokens, Hv, 128] out_dtype; may be y itself when out_dtype == y_dtype
 * All pointers 16-byte aligned.  Only cfg->n_v_heads and cfg->d_v (128) are used.
 */
GDN_EXPORT gdn_status gdn_output_gate(const gdn_config *cfg, gdn_dtype y_dtype, gdn_dtype z_dtype,
                           gdn_dtype out_dtype, const void *y, const void *z, const float *norm_w,
                           float eps, void *out, int64_t n_tokens, cudaStream_t stream);

/*
 * gdn_affine_combine -- the states entering consecutive spans of one sequence, from the
 * spans' affine maps (the prefix combination of a context-parallel prefill).
 *
 * Page "ARCHITECTURE PREVIEW / FIELD NOTES", section 03 (GATED DELTANET equations): the
 * recurrence is affine in the state, so over a span of tokens, per V head,
 * S_out = M S_in + B, with M [dk x dk] the product of the span's per-token maps
 * alpha_t (I - beta_t k_t k_t^T) (gdn_prefill's final state for the span's keys and gates,
 * zero values and zero value history, from the identity state) and B the state the span
 * leaves from zero (its final state from a zero state).  This call computes
 *     S_in[0] = S0,   S_in[p+1] = M[p] S_in[p] + B[p],   p = 0 .. n_spans-1
 *   M, B    [n_spans, Hv, 128, 128] fp32 (row index first, as states are stored)
 *   S0      [Hv, 128, 128] fp32, or NULL for a zero state
 *   S_in    [n_spans + 1, Hv, 128, 128] fp32 out: entry p is the state entering span p,
 *           entry n_spans the state after the last span; must not overlap M, B or S0
 * fp32 arithmetic.  Only cfg->n_v_heads and the head dims (128) are used.  All pointers
 * 16-byte aligned.
 */
GDN_EXPORT gdn_status gdn_affine_combine(const gdn_config *cfg, const float *M, const float *B, int n_spans,
                                         const float *S0, float *S_in, cudaStream_t stream);

/*
 * gdn_prefill_static_scratch -- gdn_prefill without a caller-supplied workspace.
 *
 * No counterpart on the pages: it exists for callers that cannot call cudaMalloc
 * while they run the mixer (for example a plugin whose host framework forbids device
 * allocation in its execute step, a runtime that hands out all device memory up front,
 * or C code with no allocator at hand).  Inputs, outputs, layouts and results are
 * exactly those of gdn_prefill; only the scratch differs.  It lives in a fixed array
 * of GDN_STATIC_SCRATCH_BYTES in device memory owned by the library: one copy on each
 * GPU where the library's module holding it is loaded (with CUDA's default lazy module
 * loading, the GPUs on which this entry point is used), kept until the process exits.
 *  - Limit: the call runs gdn_prefill in GDN_STATIC_SCRATCH_BYTES of workspace, with chunk
 *    ranges as long as fit (longer inputs just take more ranges).  Problems that do not fit
 *    even with one chunk per sequence per range are rejected with GDN_ERR_WORKSPACE on the
 *    host, before anything is looked up or enqueued: at 16 QK / 48 V heads, bf16 input,
 *    a call takes up to 9 sequences of any length; fp32 input needs 40 KB per token
 *    (about 1,600 tokens per call).
 *  - Allocation: none; it calls no cudaMalloc, cudaFree or allocating library routine.
 *  - Set-up: the first call on each device (with that device current) looks up the
 *    array's device address with cudaGetSymbolAddress; a first call that takes more than
 *    one chunk range also creates gdn_prefill's auxiliary stream and events of the host
 *    thread (see gdn_prefill).  Make the first call before any stream capture on that
 *    device.
 *  - Sharing: every call on a device uses the same array, which keeps whatever the last
 *    call left in it (no byte of it needs to start at zero).  Calls whose work overlaps
 *    on the GPU (different streams, or different host threads) race on the array: order
 *    them on one stream or synchronise between them.
 */
#define GDN_STATIC_SCRATCH_BYTES (64u << 20)

GDN_EXPORT gdn_status gdn_prefill_static_scratch(
    const gdn_config *cfg, gdn_dtype dtype, gdn_dtype out_dtype,
    const void *q, const void *k, const void *v,
    const float *conv_w_q, const float *conv_w_k, const float *conv_w_v,
    const void *alpha, const void *beta,
    const int32_t *cu_seqlens, int n_seqs, int64_t total_tokens,
    const float *initial_state, float *final_state,
    const void *conv_state_in, void *conv_state_out,
    void *out, cudaStream_t stream);

/* ========================================================================== QSA indexer
 *
 * The block selector in front of the sparse attention layers (page "ARCHITECTURE
 * PREVIEW / FIELD NOTES", section 03: the QSA indexer figure with its BLOCK SCORE and
 * CAUSAL SPARSE SET formulas, and the five-step "QSA" list; section 01: 4 query heads
 * sharing 1 key head, head dim 128, budget 512 blocks = 2048 tokens):
 *
 *   block key     kbar_b = RoPE_{4b}( RMSNorm( mean of the indexer keys of tokens 4b..4b+3 ) * w_k )
 *   query heads   qh_i^h = RoPE_i( RMSNorm( q_i^h ) * w_q ),  h = 0..3
 *   block score   I[i][b] = sum_h ReLU(<qh_i^h, kbar_b>)  for the blocks complete at token i
 *                 (4b + 3 <= i); other blocks are not candidates
 *   block set     B_i = the 512 highest-scoring candidates (all of them when fewer)
 *   token set     S_i = tokens 4b..4b+3 of every b in B_i, then the tail 4 floor((i+1)/4) .. i
 *
 * with RMSNorm(x) = x / sqrt(mean(x^2) + eps) over the 128 dims, and RoPE_p rotating the
 * pairs (d, d+32), d < 32, by the angle p * theta^(-d/32) (x_d' = x_d cos - x_{d+32} sin,
 * x_{d+32}' = x_{d+32} cos + x_d sin); dims 64..127 are not rotated.  Equal scores rank the
 * lower block index first.  Arithmetic: fp32 (angles formed and reduced in fp64); the
 * rotated query heads and the block keys are rounded to bf16 and the scores are products
 * of those bf16 values accumulated in fp32 on the tensor cores (kind::f16).
 *
 * Layouts (all device memory, row-major, contiguous):
 *   k       bf16 [B][Tn][128]      indexer keys of tokens kpos[b] .. kpos[b] + Tn - 1
 *   kbar    bf16 [B][nb_max][128]  block-key cache: entry j of row b is block j (tokens 4j..4j+3)
 *   q       bf16 [B][Qn][4][128]   indexer query heads of tokens qpos[b] .. qpos[b] + Qn - 1
 *   w_k, w_q  fp32 [128]           RMSNorm weights (w_q shared by the 4 heads)
 *   kpos, qpos, n_blocks  int32 [B] (device): first token position of row b's keys /
 *           queries, and how many cache entries of row b are valid
 *   scores  fp32 [B][Qn][nb_max]
 *   blocks  int32 [B][Qn][512]     B_i in ascending block order, then -1
 *   tokens  int32 [B][Qn][2051]    S_i in ascending order, then -1
 * Device-side values are clamped, never trusted: a query at position i has
 * min(floor((i+1)/4), n_blocks[b], nb_max) candidate blocks (none when i < 0); a
 * key call whose kpos[b] is negative or not a multiple of 4 writes nothing for row b, and
 * blocks that would land at or past nb_max are not written.
 * Requirements: compute capability 10.0; pointers 16-byte aligned; B, Tn, Qn >= 0,
 * Tn % 4 == 0, nb_max >= 1, 4 * nb_max < 2^31; eps >= 0 and theta > 0 finite.
 * A bounded device-side wait that gives up (never expected) leaves NaN in the affected
 * scores and -2 in every entry of the affected rows of blocks and tokens.
 */

/* Writes the block keys of each row's Tn / 4 complete blocks into kbar (other entries untouched). */
GDN_EXPORT gdn_status gdn_qsa_block_keys(const void *k, const float *w_k, const int32_t *kpos,
                                         int B, int Tn, float eps, float theta,
                                         void *kbar, int nb_max, cudaStream_t stream);

/* I[i][b] of every query and every candidate block into `scores` (entries of non-candidate
 * blocks are unspecified).  Needs no workspace. */
GDN_EXPORT gdn_status gdn_qsa_block_scores(const void *q, const float *w_q, const int32_t *qpos,
                                           const void *kbar, const int32_t *n_blocks,
                                           int B, int Qn, int nb_max, float eps, float theta,
                                           float *scores, cudaStream_t stream);

/* Bytes of workspace gdn_qsa_select needs: the fp32 scores of every query row, each row
 * padded to a multiple of 32 floats (a 128-byte aligned start).  Writes *bytes. */
GDN_EXPORT gdn_status gdn_qsa_select_workspace_size(int B, int Qn, int nb_max, size_t *bytes);

/* B_i (and S_i when `tokens` is not NULL) of every query.  `workspace` (256-byte aligned,
 * at least gdn_qsa_select_workspace_size bytes) is scratch; it must not be shared by two
 * calls in flight. */
GDN_EXPORT gdn_status gdn_qsa_select(const void *q, const float *w_q, const int32_t *qpos,
                                     const void *kbar, const int32_t *n_blocks,
                                     int B, int Qn, int nb_max, float eps, float theta,
                                     int32_t *blocks, int32_t *tokens,
                                     void *workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Launch trace (a profiling aid; no counterpart on the pages).  While a trace is
 * active on a host thread, every kernel that a libgdn call made on that thread
 * launches is bracketed on its launch stream: entries[i].start is recorded just
 * before the i-th launch and entries[i].stop just after it, and entries[i].kernel is
 * set to the kernel's name (static storage).  The caller creates the events (with
 * timing enabled) and reads elapsed times after synchronising.  Launches beyond
 * `capacity` are counted but not recorded.  gdn_trace_end() stops the trace and
 * returns the number of launches seen since gdn_trace_begin().  Tracing never
 * changes what the kernels compute.
 */
typedef struct {
    cudaEvent_t start;
    cudaEvent_t stop;
    const char *kernel;
} gdn_trace_entry;

GDN_EXPORT void gdn_trace_begin(gdn_trace_entry *entries, int capacity);
GDN_EXPORT int gdn_trace_end(void);

#ifdef __cplusplus
}
#endif

#endif /* LIBGDN_H */
