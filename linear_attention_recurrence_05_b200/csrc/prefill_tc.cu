// Chunked gated-delta-rule prefill on the sm_100a tensor cores (TF32 and fp16 MMAs, fp32
// accumulators and state): the serial chain over the chunks of one (sequence, V head).
//
// The recurrence of the page "ARCHITECTURE PREVIEW / FIELD NOTES", section 03 (GATED
// DELTANET equations), in chunks of 64 tokens.  Within a chunk, with
// g_t = sum_{s<=t} log alpha_s, gamma_t = exp(g_t), kd_t = exp(g_C - g_t) and S the state
// entering the chunk:
//     u   = T_beta V - T_beta_gamma (K S),  T_beta = (I + A)^-1 diag(beta),
//                                           T_beta_gamma = T_beta diag(gamma)
//     y   = diag(gamma) (Q S) + P u,        P_ti = exp(g_t - g_i) q_t.k_i (i <= t)
//     S  <- gamma_C S + K^T diag(kd) u
// Every per-token factor applied here (gamma_t, kd_t, gamma_C) is at most 1, so no decay
// is ever divided out.  T_beta, T_beta_gamma, P and the gates (gamma, kd, gamma_C) of every
// chunk come from the chunk-prep pass; [K;Q], K and V as tiles from the conv + L2 pass, all
// already in the shared-memory layout the MMAs read ([K;Q] and K are the QK head's, shared by
// its V heads).
//
// One CTA owns one (sequence, V head) for one range of chunks.  All MMAs are M = 128 with
// the d_v index on the 128 tensor-memory lanes (transposed form), so every state-dependent
// A operand is read straight from tensor memory:
//   issuer (warp 0, one thread), per chunk c
//     MMA_1   [X | Y1] = S^T [K;Q]^T         (N=128, K=128)   X = (K S)^T, Y1 = (Q S)^T
//     MMA_2a  U^T      = V^T T_beta^T        (N=64,  K=64)    state-independent
//     MMA_2b  U^T     -= X T_beta_gamma^T    (N=64,  K=64)    -> u^T
//     MMA_3   S^T     += u~^T K              (N=128, K=64)    u~ = u diag(kd), onto gamma_C S^T
//     MMA_4   Y       += u^T P^T             (N=64,  K=64)    onto Y = Y1 diag(gamma)
//   MMA_1 and MMA_2b take TF32 operands (S and X are fp32 accumulators in tensor memory;
//   [K;Q] and T_beta_gamma fp32 tiles).  MMA_2a, MMA_3 and MMA_4 take fp16 operands
//   (kind::f16): V, T_beta, K and P as fp16 tiles, u~ and u as fp16 pairs in tensor memory,
//   written by the epilogue when it forms u~.  fp16 carries the 11-bit significand of TF32; its
//   range (|x| < 65504) holds the unit keys, P (|P| <= 1), T_beta (|T_beta| <= 1 for beta in
//   [0, 1], <= 4 for beta up to 2), V, u and u~ (u times decays <= 1) for activations of any
//   sensible size, and a value beyond it turns the state into inf/NaN rather than into a
//   wrong finite value.
//   V is double-buffered (a chunk ahead) and T_beta reloaded as soon as MMA_2a has read it, so
//   MMA_2a(c+1) is normally issued right after MMA_3(c) and MMA_4(c), and runs while the new
//   state is waited for; MMA_2b reads X straight from MMA_1's output.  The only epilogue step
//   left on the critical path is u~.  u^T is double-buffered in tensor memory (chunk parity).
//   epilogue (warps 1-4), in tensor memory: after MMA_1, Y = Y1 diag(gamma) (once the drain
//     group has read the previous Y) and S^T *= gamma_C; after MMA_2b, u~ (over X, which
//     MMA_2b has consumed); the state entering and leaving the range.
//   producer (warp 5): the tile loads, each issued as soon as its buffer is free.
//   drain group (warps 6-9): after MMA_4, reads Y and frees it at once, then writes y (or the
//     gated output) through shared memory with TMA stores; a bf16 gate input z arrives by
//     one TMA load per chunk, issued as soon as the previous chunk's rows have been read.
// All waits are bounded; a CTA that times out writes NaN to its outputs.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "chunk_range.cuh"
#include "gdn_common.cuh"
#include "gdn_internal.h"
#include "tc_sm100.cuh"
#include "tma_map.cuh"

namespace gdn {

namespace {
using namespace tc;

constexpr int kThr = 320;          // 10 warps
constexpr int kEpiWarp0 = 1;       // warps 1-4: epilogue
constexpr int kLoadWarp = 5;       // tile producer
constexpr int kDrainWarp0 = 6;     // warps 6-9: y out
constexpr int kEpiTid0 = kEpiWarp0 * 32;
constexpr int kDrainTid0 = kDrainWarp0 * 32;
constexpr int kBarEpi = 1;         // named barrier of the epilogue (128 threads)
constexpr int kBarDrain = 2;       // named barrier of the drain group (128 threads)

// shared-memory map (bytes from a 1024-aligned base)
constexpr uint32_t OFF_KQ = 0;          // [K;Q]   K-major, 4 blocks x (K 8 KB | Q 8 KB)       64 KB
constexpr uint32_t OFF_KMN = 65536;     // K       fp16, MN-major, 64 x 128                    16 KB
constexpr uint32_t OFF_Z = 81920;       // gate input z of a chunk, bf16, 64 rows x 256 B     16 KB
constexpr uint32_t OFF_V = 98304;       // V       fp16, MN-major, 2 buffers (chunk parity)  2 x 16 KB
constexpr uint32_t OFF_TB = 131072;     // T_beta        fp16, K-major [t][i]                   8 KB
constexpr uint32_t OFF_TG = 139264;     // T_beta_gamma  K-major [t][i]                        16 KB
constexpr uint32_t OFF_P = 155648;      // P       fp16, K-major [t][i]                         8 KB
constexpr uint32_t OFF_YST = 163840;    // y staging: 32 rows x 128 columns (TMA store box)    16 KB
constexpr uint32_t OFF_GR = 180224;     // gates records, 2 buffers                          1280 B
constexpr uint32_t OFF_BAR = OFF_GR + 2 * kGateRec * 4;   // mbarriers
constexpr uint32_t OFF_FLAGS = OFF_BAR + 176;             // TMEM base, abort flag
constexpr uint32_t kSmem = OFF_FLAGS + 16;
constexpr uint32_t kSmemAlloc = kSmem + 1024;              // slack to align the base to 1024
static_assert(kSmemAlloc <= 232448, "shared memory per CTA");

enum {
    B_KQ = 0, B_V0, B_V1, B_TB, B_TG,    // tile arrivals (B_KQ: features 0-63 of [K;Q]; B_V: V of
    B_KQ1,                               // buffer 0 / 1; B_KQ1: features 64-127 of [K;Q])
    B_KMN, B_PL,
    B_GR0, B_GR1,                        // gates record into buffer 0 / 1
    B_1A, B_1, B_2A, B_2, B_3, B_4,      // MMA completions (MMA_1 first half; MMA_1; 2a; up to 2b; 3; 4)
    B_Y1,                                // epilogue: Y = Y1 diag(gamma) stored, S scaled
    B_UT,                                // epilogue: u~ = u diag(kd) stored
    B_YF,                                // drain group: Y read (tensor memory free for the next chunk)
    B_DRAIN0,                            // drain on the failure path
    B_Z,                                 // gate input of a chunk arrived
    kNumBars
};
static_assert(kNumBars * 8 <= 176, "barrier area");

// tensor memory columns (all 128 lanes)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t T_S = 0;      // S^T                               128 cols
constexpr uint32_t T_XY = 128;   // [X | Y1]; fp16 u~^T over X once MMA_2b has read it  128 cols
constexpr uint32_t T_U = 256;    // u^T, two buffers (chunk parity), then fp16 u^T  2 x 64 cols
constexpr uint32_t T_Y = 384;    // gamma Y1, then y                    64 cols

constexpr uint32_t kWaitTries = 1u << 22;

__device__ __forceinline__ void bar_sync(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
// named barrier; returns true if any participating thread passed `pred`
__device__ __forceinline__ bool bar_or(int id, int count, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.b32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}\n"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(count)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ void mbar_arrive(uint64_t *m) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(m)) : "memory");
}
// Bounded wait that gives up early once another role has raised the abort flag.  Each
// poll may sleep up to 40 ns (a long suspend hint delays the wake-up well past the phase
// completion; none at all keeps the polling warp issuing at full rate).
__device__ __forceinline__ bool wait_or_abort(uint64_t *m, uint32_t par, volatile int *abort_flag) {
    if (mbar_try_wait(m, par)) return true;
    for (uint32_t i = 0; i < kWaitTries; ++i) {
        if (mbar_try_wait_sleep(m, par, 40)) return true;
        if ((i & 63) == 63 && *abort_flag) return false;
    }
    *abort_flag = 1;
    return false;
}

// SiLU(z) = z / (1 + e^-z) = z/2 (1 + tanh(z/2)) with the hardware tanh (tanh.approx.f32,
// relative error <= 2^-10.987): one special-function (MUFU) operation per element, whose
// issue rate in this kernel (~32 cycles per warp instruction on a sub-partition) is what the
// gated output is bound by.  The error is absolute in effect: |SiLU - exact| <= |z| 2^-12
// (largest where SiLU(z) -> 0 for z << 0, where 1 + tanh cancels).
__device__ __forceinline__ float silu_tanh(float z) {
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * z));
    return 0.5f * z * (1.f + t);
}

// Reduce-scatter of 32 rows over the 32 lanes of a warp: s[i] holds this lane's value of row i;
// returns the sum over the warp's lanes of row `lane` (31 shuffles: each step halves the rows a
// lane keeps and adds its partner's share of them).
__device__ __forceinline__ float warp_row_sums32(float (&s)[32], int lane) {
#pragma unroll
    for (int k = 16; k >= 1; k >>= 1) {
        const bool up = lane & k;
#pragma unroll
        for (int i = 0; i < k; ++i) {
            const float send = up ? s[i] : s[i + k];
            const float keep = up ? s[i + k] : s[i];
            s[i] = keep + __shfl_xor_sync(0xffffffffu, send, k);
        }
    }
    return s[0];
}

// A from tensor memory (K-major), B from a shared-memory descriptor
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t id, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d),
        "r"(a_tmem), "l"(b), "r"(id), "r"(acc));
}
// D[128 x N] (+)= (-)A_tmem[128 x K] B[K x N]; B K-major (b_arg = block stride) or MN-major
// (b_arg = its row count)
template <int N, int K, bool B_MN, bool NEG_A>
__device__ __forceinline__ void gemm_ts(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_base, uint32_t b_arg,
                                        bool accumulate) {
    constexpr uint32_t id = idesc_tf32(128, N, false, B_MN) | (NEG_A ? (1u << 13) : 0u);
    const uint64_t b0 = B_MN ? desc_mnmajor(b_base, (int)b_arg, 0) : desc_kmajor(b_base, b_arg, 0);
    const uint32_t b_blk16 = B_MN ? 0u : (b_arg >> 4);
#pragma unroll
    for (int s = 0; s < K / 8; ++s) {
        const uint32_t db = B_MN ? (uint32_t)(s * 64) : (uint32_t)((s >> 2) * b_blk16 + (s & 3) * 2);
        mma_ts(d_tmem, a_tmem + 8 * s, b0 + db, id, (accumulate || s > 0) ? 1u : 0u);
    }
}

}  // namespace

struct TcParams {
    CUtensorMap tm_out;   // y as [T, Hv*128] rows, boxes of 128 columns x 32 rows (no swizzle)
    CUtensorMap tm_z;     // bf16 z as [T, Hv*128] rows, boxes of 128 columns x 64 rows
    // per-chunk tiles of the range's buffer, by slot, in shared-memory layout: [K;Q] and K
    // (fp16) per (slot, QK head); V (fp16), T_beta (fp16), T_beta_gamma, P (fp16) and the gates
    // record per (slot, V head)
    const float *kq, *kmn, *vi, *tb, *tg, *pm, *gr;
    const int32_t *cu, *cfirst;
    const float *init, *carry_in;   // state entering chunk 0 / entering a later first chunk
    float *carry_out;               // state after the last chunk of the range
    void *out;
    int n_seqs, n_qk, n_v;
    ChunkRange rg;
    // gated output (GATED kernels): out = y / sqrt(mean(y^2) + norm_eps) * norm_w * SiLU(z)
    const void *z;          // [T, Hv, 128] gate input
    const float *norm_w;    // [128]
    float norm_eps;
};

template <class TO, class TZ, bool GATED>
__global__ void __launch_bounds__(kThr, 1) prefill_tc_kernel(const __grid_constant__ TcParams p) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    const uint32_t sb = smem_u32(sm);
    uint64_t *bar = (uint64_t *)(sm + OFF_BAR);
    uint32_t *tslot = (uint32_t *)(sm + OFF_FLAGS);
    volatile int *abort_flag = (volatile int *)(sm + OFF_FLAGS + 4);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int h = blockIdx.x % p.n_v;
    const int b = blockIdx.x / p.n_v;
    const int gq = h / (p.n_v / p.n_qk);
    const int seq0 = p.cu[b], L = p.cu[b + 1] - p.cu[b];
    const int seq_chunks = (L + kChunk - 1) / kChunk;
    // this range's chunks of the sequence: [cb, cb + nchunks); the state enters from the
    // initial state (cb = 0) or from the previous range's carry
    const bool first_range = p.rg.compact || p.rg.r == 0;
    const int cb = p.rg.compact ? 0 : p.rg.r * p.rg.R;
    const int nchunks = max(0, (p.rg.compact ? seq_chunks : min(seq_chunks, cb + p.rg.R)) - cb);
    // nothing in range (a zero-length sequence is handled by the first range)
    if (seq_chunks > 0 ? nchunks == 0 : !first_range) return;   // uniform per CTA
    const float *state_in = cb == 0 ? p.init : p.carry_in;
    // a sequence longer than the caller's bound on the longest one still has chunks after
    // the last range: its later tokens and its final state are set to NaN
    const bool overflow = !p.rg.compact && p.rg.last && seq_chunks > cb + nchunks;

    if (tid == 0) {
        // the y map is encoded only when the call has tokens (a CTA with chunks implies that)
        if (nchunks > 0) asm volatile("prefetch.tensormap [%0];" ::"l"(&p.tm_out) : "memory");
        for (int i = 0; i < kNumBars; ++i) mbar_init(&bar[i], 1);
        *abort_flag = 0;
    }
    if (warp == 0) {
        tmem_alloc(tslot, kTmemCols);
        tmem_relinquish();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tm = *tslot;

    // tile loads: one contiguous bulk copy each (thread 0 for the first chunks, then the producer)
    auto load = [&](int bar_i, uint32_t dst, const float *src, uint32_t bytes) {
        mbar_expect_tx(&bar[bar_i], bytes);
        bulk_load(sb + dst, src, bytes, &bar[bar_i]);
    };
    // (c counts this range's chunks from 0; the sequence's chunk is cb + c)
    auto slot = [&](int c) { return chunk_slot(p.rg, b, cb + c, p.cfirst); };
    auto qk_tile = [&](const float *base, int c, int64_t floats) { return base + (slot(c) * p.n_qk + gq) * floats; };
    auto v_tile = [&](const float *base, int c, int64_t floats) { return base + (slot(c) * p.n_v + h) * floats; };
    // [K;Q] in two halves by feature (blocks 0-1, 2-3): MMA_1 starts on the first half while
    // the second lands, and each half is reloaded as soon as MMA_1 has read it
    auto issue_kq0 = [&](int c) { load(B_KQ, OFF_KQ, qk_tile(p.kq, c, 16384), 32768); };
    auto issue_kq1 = [&](int c) { load(B_KQ1, OFF_KQ + 32768, qk_tile(p.kq, c, 16384) + 8192, 32768); };
    auto issue_kmn = [&](int c) { load(B_KMN, OFF_KMN, qk_tile(p.kmn, c, 4096), 16384); };
    auto issue_v = [&](int c) { load(B_V0 + (c & 1), OFF_V + (c & 1) * 16384, v_tile(p.vi, c, 4096), 16384); };
    auto issue_tb = [&](int c) { load(B_TB, OFF_TB, v_tile(p.tb, c, 2048), 8192); };
    auto issue_tg = [&](int c) { load(B_TG, OFF_TG, v_tile(p.tg, c, 4096), 16384); };
    auto issue_pm = [&](int c) { load(B_PL, OFF_P, v_tile(p.pm, c, 2048), 8192); };
    auto issue_gr = [&](int c) {  // gates record of chunk c into buffer c & 1
        load(B_GR0 + (c & 1), OFF_GR + (c & 1) * kGateRec * 4, v_tile(p.gr, c, kGateRec), kGateRec * 4);
    };

    // epilogue warps: initial state S^T (lane j = column j of S) into tensor memory
    if (warp >= kEpiWarp0 && warp < kLoadWarp) {
        const int q = warp & 3, j = 32 * q + lane;
        const uint32_t lrow = (uint32_t)(32 * q) << 16;
        const float *src = state_in ? state_in + ((int64_t)b * p.n_v + h) * kHeadDim * kHeadDim + j : nullptr;
#pragma unroll
        for (int d0 = 0; d0 < kHeadDim; d0 += 32) {
            float v[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = src ? src[(int64_t)(d0 + i) * kHeadDim] : 0.f;
            tmem_st32(tm + lrow + T_S + d0, v);
        }
        tmem_wait_st();
    }
    if (tid == 0 && nchunks > 0) {
        issue_v(0);
        issue_tb(0);
        issue_kq0(0);
        issue_kq1(0);
        if (nchunks > 1) issue_v(1);
        issue_tg(0);
        issue_kmn(0);
        issue_pm(0);
        issue_gr(0);
        if (nchunks > 1) issue_gr(1);
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();

    if (warp == 0) {
        // ================================================================ issuer
        if (lane == 0) {
            bool ok = true;
            bool a2_issued = false;   // MMA_2a of the current chunk already issued
            // V of chunk c sits in buffer c & 1; that buffer's barrier completes once per two
            // chunks, so chunk c waits for its phase c >> 1
            auto vpar = [](int c) { return (uint32_t)((c >> 1) & 1); };
            auto issue_2a = [&](int c) {   // into u^T buffer c & 1 (D), V of buffer c & 1
                const int bi = c & 1;
                fence_after_sync();
                gemm_f16<128, 64, 64, true, false>(tm + T_U + 64 * bi, sb + OFF_V + bi * 16384, 64, sb + OFF_TB, 0,
                                                   false);
                mma_commit(&bar[B_2A]);
            };
            // A wait costs ~100 cycles even when its phase is complete, so the waits for tiles
            // and for epilogue steps that are normally done sit right after an MMA group,
            // while the tensor pipe still has queued work.
            if (nchunks > 0) {
                ok = wait_or_abort(&bar[B_V0], 0, abort_flag) && wait_or_abort(&bar[B_TB], 0, abort_flag);
                if (ok) {
                    issue_2a(0);
                    a2_issued = true;
                    ok = wait_or_abort(&bar[B_KQ], 0, abort_flag);
                }
            }
            // MMA_1 over features 0-63 (A: S^T columns 0-63, B: [K;Q] blocks 0-1), then 64-127
            auto mma1_lo = [&]() {
                fence_after_sync();
                gemm_ts<128, 64, false, false>(tm + T_XY, tm + T_S, sb + OFF_KQ, 16384, false);
                mma_commit(&bar[B_1A]);
            };
            auto mma1_hi = [&]() {
                gemm_ts<128, 64, false, false>(tm + T_XY, tm + T_S + 64, sb + OFF_KQ + 32768, 16384, true);
                mma_commit(&bar[B_1]);
            };
            for (int c = 0; c < nchunks && ok; ++c) {
                const uint32_t par = c & 1;
                const int bi = c & 1;
                // MMA_1: needs S (MMA_3 of c-1, waited below) and [K;Q] of c (the first half
                // waited below, the second here)
                mma1_lo();
                if (!(ok = wait_or_abort(&bar[B_KQ1], par, abort_flag))) break;
                fence_after_sync();
                mma1_hi();
                // MMA_2a of c unless issued at the end of c-1 (its tiles came late)
                if (!a2_issued) {
                    if (!(ok = wait_or_abort(&bar[B_V0 + bi], vpar(c), abort_flag))) break;
                    if (!(ok = wait_or_abort(&bar[B_TB], par, abort_flag))) break;
                    issue_2a(c);
                }
                // MMA_2b: U^T -= X T_beta_gamma^T once MMA_1 has written X
                if (!(ok = wait_or_abort(&bar[B_TG], par, abort_flag))) break;
                if (!(ok = wait_or_abort(&bar[B_1], par, abort_flag))) break;
                fence_after_sync();
                gemm_ts<64, 64, false, true>(tm + T_U + 64 * bi, tm + T_XY, sb + OFF_TG, 8192, true);
                mma_commit(&bar[B_2]);
                // MMA_3: S^T += u~^T K onto gamma_C S^T (fp16: u~ from the epilogue, K tile
                // MN-major)
                if (!(ok = wait_or_abort(&bar[B_KMN], par, abort_flag))) break;
                if (!(ok = wait_or_abort(&bar[B_UT], par, abort_flag))) break;
                fence_after_sync();
                gemm_ts_f16<128, 64, true>(tm + T_S, tm + T_XY, sb + OFF_KMN, 64, true);
                mma_commit(&bar[B_3]);
                // MMA_4: Y += u^T P^T onto Y = Y1 diag(gamma) (fp16: u from the epilogue's u~
                // step, P tile); off the state's path, it runs while the new state is waited for
                if (!(ok = wait_or_abort(&bar[B_Y1], par, abort_flag))) break;
                if (!(ok = wait_or_abort(&bar[B_PL], par, abort_flag))) break;
                fence_after_sync();
                gemm_ts_f16<64, 64, false>(tm + T_Y, tm + T_U + 64 * bi, sb + OFF_P, 0, true);
                mma_commit(&bar[B_4]);
                a2_issued = false;
                if (c + 1 < nchunks) {
                    // MMA_2a of c+1 fills the wait for MMA_3 (its u^T buffer held u of c-1, read by
                    // MMA_4 and the epilogue of c-1, both complete before MMA_3 of c-1)
                    if (mbar_try_wait(&bar[B_V0 + (bi ^ 1)], vpar(c + 1)) && mbar_try_wait(&bar[B_TB], par ^ 1)) {
                        issue_2a(c + 1);
                        a2_issued = true;
                    }
                    if (!(ok = wait_or_abort(&bar[B_KQ], par ^ 1, abort_flag))) break;
                }
                if (!(ok = wait_or_abort(&bar[B_3], par, abort_flag))) break;
            }
            if (!ok) {  // drain this thread's MMAs (bounded)
                mma_commit(&bar[B_DRAIN0]);
                mbar_wait(&bar[B_DRAIN0], 0, kWaitTries);
            }
        }
    } else if (warp == kLoadWarp) {
        // ================================================================ tile producer
        if (lane == 0) {
            bool ok = true;
            int n_kq = nchunks > 0 ? 1 : 0, n_kq1 = n_kq, n_tb = n_kq, n_tg = n_kq, n_kmn = n_kq, n_pm = n_kq;
            int n_v[2] = {nchunks > 0 ? 1 : 0, nchunks > 1 ? 1 : 0};
            int n_gr[2] = {nchunks > 0 ? 1 : 0, nchunks > 1 ? 1 : 0};
            for (int c = 0; c < nchunks && ok; ++c) {
                const uint32_t par = c & 1;
                const bool more = c + 1 < nchunks;
                // MMA_2a of c has read T_beta and its V buffer: T_beta of c+1, V of c+2
                if (!(ok = wait_or_abort(&bar[B_2A], par, abort_flag))) break;
                if (more) { issue_tb(c + 1); ++n_tb; }
                if (c + 2 < nchunks) { issue_v(c + 2); ++n_v[c & 1]; }
                // each half of [K;Q] of c is consumed once its half of MMA_1 of c is done
                if (!(ok = wait_or_abort(&bar[B_1A], par, abort_flag))) break;
                if (more) { issue_kq0(c + 1); ++n_kq; }
                if (!(ok = wait_or_abort(&bar[B_1], par, abort_flag))) break;
                if (more) { issue_kq1(c + 1); ++n_kq1; }
                // T_beta_gamma once MMA_2b of c is done
                if (!(ok = wait_or_abort(&bar[B_2], par, abort_flag))) break;
                if (more) { issue_tg(c + 1); ++n_tg; }
                // K and this gates buffer once MMA_3 of c is done (the epilogue took the gates
                // of c before MMA_3 could start); P once MMA_4 of c is done
                if (!(ok = wait_or_abort(&bar[B_3], par, abort_flag))) break;
                if (more) { issue_kmn(c + 1); ++n_kmn; }
                if (c + 2 < nchunks) { issue_gr(c + 2); ++n_gr[c & 1]; }
                if (!(ok = wait_or_abort(&bar[B_4], par, abort_flag))) break;
                if (more) { issue_pm(c + 1); ++n_pm; }
            }
            if (!ok) {  // wait (bounded) for the copies this thread started
                const int counts[6] = {n_kq, n_kq1, n_tb, n_tg, n_kmn, n_pm};
                const int bars[6] = {B_KQ, B_KQ1, B_TB, B_TG, B_KMN, B_PL};
                for (int i = 0; i < 6; ++i)
                    if (counts[i]) mbar_wait(&bar[bars[i]], (uint32_t)(counts[i] - 1) & 1, kWaitTries);
                for (int i = 0; i < 2; ++i) {
                    if (n_v[i]) mbar_wait(&bar[B_V0 + i], (uint32_t)(n_v[i] - 1) & 1, kWaitTries);
                    if (n_gr[i]) mbar_wait(&bar[B_GR0 + i], (uint32_t)(n_gr[i] - 1) & 1, kWaitTries);
                }
            }
        }
    } else if (warp < kDrainWarp0) {
        // ================================================================ epilogue
        const int q = warp & 3;
        const uint32_t lrow = (uint32_t)(32 * q) << 16;
        const bool leader = tid == kEpiTid0;
        auto ewait = [&](int i, uint32_t par) -> bool {  // one thread polls, the group blocks
            const bool ok = leader ? wait_or_abort(&bar[i], par, abort_flag) : true;
            return !bar_or(kBarEpi, 128, !ok);
        };
        // the group's tensor-memory stores are done: tell the issuer through mbarrier i
        auto publish = [&](int i) {
            tmem_wait_st();
            fence_before_sync();
            bar_sync(kBarEpi, 128);
            if (leader) mbar_arrive(&bar[i]);
        };
        // columns [src, src + 64) of this warp's lanes, column i times f[i], stored at dst
        // (f: 16-byte aligned shared memory)
        auto scale64 = [&](uint32_t src, uint32_t dst, const float *f) {
            float v0[32], v1[32];
            tmem_ld32(tm + lrow + src, v0);
            tmem_ld32(tm + lrow + src + 32, v1);
            tmem_wait_ld();
            tmem_regs_after_wait(v0);
            tmem_regs_after_wait(v1);
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
                const float4 a = *reinterpret_cast<const float4 *>(f + i);
                const float4 b = *reinterpret_cast<const float4 *>(f + 32 + i);
                v0[i] *= a.x; v0[i + 1] *= a.y; v0[i + 2] *= a.z; v0[i + 3] *= a.w;
                v1[i] *= b.x; v1[i + 1] *= b.y; v1[i + 2] *= b.z; v1[i + 3] *= b.w;
            }
            tmem_st32(tm + lrow + dst, v0);
            tmem_st32(tm + lrow + dst + 32, v1);
        };
        for (int c = 0; c < nchunks; ++c) {
            const uint32_t par = c & 1;
            const int bsel = c & 1;
            {  // MMA_1 done, the gates record of c here, and Y of c-1 read by the drain group
                bool ok = true;
                if (leader) ok = wait_or_abort(&bar[B_1], par, abort_flag) &&
                                 wait_or_abort(&bar[B_GR0 + bsel], (c >> 1) & 1, abort_flag) &&
                                 (c == 0 || wait_or_abort(&bar[B_YF], par ^ 1, abort_flag));
                if (bar_or(kBarEpi, 128, !ok)) break;
            }
            fence_after_sync();
            const float *gr = (const float *)(sm + OFF_GR + bsel * kGateRec * 4);
            scale64(T_XY + 64, T_Y, gr + kGrGamma);        // Y = Y1 diag(gamma), for MMA_4
            {  // S^T *= gamma_C (last read by MMA_1; MMA_3 accumulates onto it)
                const float gc = gr[kGrGammaC];
#pragma unroll
                for (int d0 = 0; d0 < kHeadDim; d0 += 32) {
                    float v[32];
                    tmem_ld32(tm + lrow + T_S + d0, v);
                    tmem_wait_ld();
                    tmem_regs_after_wait(v);
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] *= gc;
                    tmem_st32(tm + lrow + T_S + d0, v);
                }
            }
            publish(B_Y1);
            if (!ewait(B_2, par)) break;
            fence_after_sync();
            {   // u (fp32, 64 columns) -> fp16 u over its first 32 columns, for MMA_4, and
                // fp16 u~ = u diag(kd) over X's first 32 columns, for MMA_3
                const uint32_t src = T_U + 64 * par;
                const float *kd = gr + kGrKd;
                float v0[32], v1[32], hu[32], ht[32];
                tmem_ld32(tm + lrow + src, v0);
                tmem_ld32(tm + lrow + src + 32, v1);
                tmem_wait_ld();
                tmem_regs_after_wait(v0);
                tmem_regs_after_wait(v1);
#pragma unroll
                for (int i = 0; i < 32; i += 4) {
                    const float4 a = *reinterpret_cast<const float4 *>(kd + i);
                    const float4 b = *reinterpret_cast<const float4 *>(kd + 32 + i);
                    hu[i / 2] = __uint_as_float(pack_f16x2(v0[i], v0[i + 1]));
                    hu[i / 2 + 1] = __uint_as_float(pack_f16x2(v0[i + 2], v0[i + 3]));
                    hu[16 + i / 2] = __uint_as_float(pack_f16x2(v1[i], v1[i + 1]));
                    hu[16 + i / 2 + 1] = __uint_as_float(pack_f16x2(v1[i + 2], v1[i + 3]));
                    ht[i / 2] = __uint_as_float(pack_f16x2(v0[i] * a.x, v0[i + 1] * a.y));
                    ht[i / 2 + 1] = __uint_as_float(pack_f16x2(v0[i + 2] * a.z, v0[i + 3] * a.w));
                    ht[16 + i / 2] = __uint_as_float(pack_f16x2(v1[i] * b.x, v1[i + 1] * b.y));
                    ht[16 + i / 2 + 1] = __uint_as_float(pack_f16x2(v1[i + 2] * b.z, v1[i + 3] * b.w));
                }
                tmem_st32(tm + lrow + T_XY, ht);
                tmem_st32(tm + lrow + src, hu);
            }
            publish(B_UT);
        }
    } else {
        // ================================================================ drain group (warps 6-9)
        // After MMA_4 of chunk c, read Y (this warp's 32 lanes = columns j of y, 64 tokens) and
        // free the tensor memory for chunk c+1 at once; then write y (gated when GATED) by 32-row
        // halves: staged in shared memory and written with one TMA store for a full chunk, or
        // stored directly (rows of the chunk only) for a sequence's last, partial chunk.
        const int q = warp & 3, j = 32 * q + lane;
        const uint32_t lrow = (uint32_t)(32 * q) << 16;
        const bool dleader = tid == kDrainTid0;
        const int64_t v_row = (int64_t)p.n_v * kHeadDim;
        float wj = 0.f;
        if constexpr (GATED) wj = p.norm_w[j];
        // bf16 z: the chunk's 64 rows by one TMA load into shared memory (rows past the last
        // token read as zero), issued as soon as the previous chunk's rows have been read
        constexpr bool kZTile = GATED && sizeof(TZ) == 2;
        int z_issued = 0, z_done = 0;
        auto issue_z = [&](int c) {
            mbar_expect_tx(&bar[B_Z], 64 * kHeadDim * 2);
            tma_load_2d(sb + OFF_Z, &p.tm_z, h * kHeadDim, (int)(seq0 + (int64_t)(cb + c) * kChunk), &bar[B_Z]);
            ++z_issued;
        };
        if constexpr (kZTile)
            if (dleader && nchunks > 0) issue_z(0);
        // fp32 z: read per column into registers, raw (converted where they are used): rows
        // past a partial chunk's end read its last row, so the 32 loads of a half carry no
        // condition and are all in flight at once
        TZ zr[2][32];
        auto load_z = [&](int c, int h2) {
            const int n = min(kChunk, L - (cb + c) * kChunk);
            const TZ *zp = (const TZ *)p.z + (seq0 + (int64_t)(cb + c) * kChunk) * v_row + h * kHeadDim + j;
#pragma unroll
            for (int i = 0; i < 32; ++i) zr[h2][i] = __ldg(zp + (int64_t)min(32 * h2 + i, n - 1) * v_row);
        };
        for (int c = 0; c < nchunks; ++c) {
            const int n = min(kChunk, L - (cb + c) * kChunk);
            const int64_t tok = seq0 + (int64_t)(cb + c) * kChunk;
            if constexpr (GATED && !kZTile) load_z(c, 0);   // in flight while MMA_4 runs
            {
                bool ok = true;
                if (dleader) {
                    ok = wait_or_abort(&bar[B_4], c & 1, abort_flag);
                    if (kZTile && ok) {
                        ok = wait_or_abort(&bar[B_Z], c & 1, abort_flag);
                        z_done += ok;
                    }
                }
                if (bar_or(kBarDrain, 128, !ok)) break;
            }
            fence_after_sync();
            float v[2][32];
            tmem_ld32(tm + lrow + T_Y, v[0]);
            tmem_ld32(tm + lrow + T_Y + 32, v[1]);
            tmem_wait_ld();
            tmem_regs_after_wait(v[0]);
            tmem_regs_after_wait(v[1]);
            fence_before_sync();
            bar_sync(kBarDrain, 128);
            if (dleader) mbar_arrive(&bar[B_YF]);              // the epilogue may rewrite Y
            if constexpr (GATED && !kZTile) load_z(c, 1);   // in flight while the first half is written
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                const int row0 = 32 * h2;
                // the staging (also the scratch of the gated rows) is free once the previous TMA
                // store has read it
                if (dleader) bulk_wait_read0();
                bar_sync(kBarDrain, 128);
                if constexpr (GATED) {
                    // out = y / sqrt(mean_j y^2 + eps) * w_j * SiLU(z): row sums over this warp's
                    // 32 columns in registers, over the 4 warps in a scratch in the staging
                    float sq[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) sq[i] = v[h2][i] * v[h2][i];
                    float *red = (float *)(sm + OFF_YST), *rinv = red + 128;
                    red[32 * q + lane] = warp_row_sums32(sq, lane);
                    bar_sync(kBarDrain, 128);
                    if (warp == kDrainWarp0)
                        rinv[lane] = rsqrtf((red[lane] + red[32 + lane] + red[64 + lane] + red[96 + lane]) *
                                                (1.f / kHeadDim) + p.norm_eps);
                    bar_sync(kBarDrain, 128);
                    float rw[32];   // 1 / rms of each row, times this column's weight
#pragma unroll
                    for (int i = 0; i < 32; i += 4) {
                        const float4 r4 = *reinterpret_cast<const float4 *>(rinv + i);
                        rw[i] = r4.x * wj; rw[i + 1] = r4.y * wj; rw[i + 2] = r4.z * wj; rw[i + 3] = r4.w * wj;
                    }
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        float zi;
                        if constexpr (kZTile)
                            zi = to_f32(reinterpret_cast<const bf16 *>(sm + OFF_Z)[(row0 + i) * kHeadDim + j]);
                        else
                            zi = to_f32(zr[h2][i]);
                        v[h2][i] *= rw[i] * silu_tanh(zi);
                    }
                    bar_sync(kBarDrain, 128);   // the scratch (and z) read before the staging is written
                    if constexpr (kZTile)
                        if (h2 == 1 && dleader && c + 1 < nchunks) issue_z(c + 1);
                }
                if (n == kChunk) {
                    TO *ys = (TO *)(sm + OFF_YST);
#pragma unroll
                    for (int i = 0; i < 32; ++i) ys[i * kHeadDim + j] = from_f32<TO>(v[h2][i]);
                    fence_smem_to_async();
                    bar_sync(kBarDrain, 128);
                    if (dleader) {
                        tma_store_2d(&p.tm_out, h * kHeadDim, (int)tok + row0, sb + OFF_YST);
                        bulk_commit();
                    }
                } else {
                    TO *o = (TO *)p.out + (tok + row0) * v_row + h * kHeadDim + j;
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (row0 + i < n) o[(int64_t)i * v_row] = from_f32<TO>(v[h2][i]);
                }
            }
        }
        if (dleader) bulk_wait0();   // this thread's y stores are complete
        if constexpr (kZTile)        // a z load still in flight after a failure
            if (dleader && z_issued > z_done) mbar_wait(&bar[B_Z], (uint32_t)(z_issued - 1) & 1, kWaitTries);
    }

    // ---------------------------------------------------------------- tear-down
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (warp >= kEpiWarp0 && warp < kLoadWarp) {
        const int q = warp & 3, j = 32 * q + lane;
        const uint32_t lrow = (uint32_t)(32 * q) << 16;
        const bool failed = *abort_flag != 0;
        if (p.carry_out) {
            const bool nan_state = failed || overflow;
            float *dst = p.carry_out + ((int64_t)b * p.n_v + h) * kHeadDim * kHeadDim + j;
#pragma unroll
            for (int d0 = 0; d0 < kHeadDim; d0 += 32) {
                float s[32];
                tmem_ld32(tm + lrow + T_S + d0, s);
                tmem_wait_ld();
                tmem_regs_after_wait(s);
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    dst[(int64_t)(d0 + i) * kHeadDim] = nan_state ? __int_as_float(0x7fc00000) : s[i];
            }
        }
        if (failed || overflow) {
            const int64_t v_row = (int64_t)p.n_v * kHeadDim;
            const int t0 = (failed ? cb : cb + nchunks) * kChunk;
            const int t1 = overflow ? L : min(L, (cb + nchunks) * kChunk);
            for (int e = tid - kEpiTid0 + t0 * kHeadDim; e < t1 * kHeadDim; e += 128) {
                const int t = e / kHeadDim, jj = e % kHeadDim;
                ((TO *)p.out)[(seq0 + t) * v_row + h * kHeadDim + jj] = from_f32<TO>(__int_as_float(0x7fc00000));
            }
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tm, kTmemCols);
}

// ---------------------------------------------------------------- host side
template <class TO, class TZ, bool GATED>
static cudaError_t launch_tc_t(TcParams p, int64_t total_tokens, cudaStream_t s) {
    const bool obf = sizeof(TO) == 2;
    const int64_t width = (int64_t)p.n_v * kHeadDim;
    if (total_tokens > 0 &&   // with no tokens there is no output (and `out` may be null)
        !encode_2d(&p.tm_out, obf ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, p.out,
                   width, total_tokens, width * (int64_t)sizeof(TO), kHeadDim, 32, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    if (GATED && sizeof(TZ) == 2 && total_tokens > 0 &&
        !encode_2d(&p.tm_z, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.z, width, total_tokens, width * 2, kHeadDim, 64,
                   CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    auto k = prefill_tc_kernel<TO, TZ, GATED>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemAlloc);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)((int64_t)p.n_seqs * p.n_v);
    TraceLaunch tl(s, GATED ? "prefill_tc_gated" : "prefill_tc");
    k<<<grid, kThr, kSmemAlloc, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_prefill_tc(const ScanParams &sp, int64_t total_tokens, bool /*in_bf16*/,
                              bool out_bf16, cudaStream_t s) {
    if (sp.n_seqs <= 0) return cudaSuccess;
    TcParams p{};
    p.kq = sp.kq; p.kmn = sp.kmn; p.vi = sp.vi; p.tb = sp.tb; p.tg = sp.tg; p.pm = sp.pm; p.gr = sp.gr;
    p.cu = sp.cu; p.cfirst = sp.cfirst; p.init = sp.init; p.carry_in = sp.carry_in; p.carry_out = sp.carry_out;
    p.rg = sp.rg;
    p.out = sp.out; p.n_seqs = sp.n_seqs; p.n_qk = sp.n_qk; p.n_v = sp.n_v;
    p.z = sp.gate_z; p.norm_w = sp.gate_w; p.norm_eps = sp.gate_eps;
    using gdn::bf16;
    if (!sp.gate_z)
        return out_bf16 ? launch_tc_t<bf16, float, false>(p, total_tokens, s)
                        : launch_tc_t<float, float, false>(p, total_tokens, s);
    if (sp.gate_z_bf16)
        return out_bf16 ? launch_tc_t<bf16, bf16, true>(p, total_tokens, s)
                        : launch_tc_t<float, bf16, true>(p, total_tokens, s);
    return out_bf16 ? launch_tc_t<bf16, float, true>(p, total_tokens, s)
                    : launch_tc_t<float, float, true>(p, total_tokens, s);
}

}  // namespace gdn
