// Chunked gated-delta-rule prefill on the sm_100a tensor cores (TF32 MMAs, fp32 state).
//
// The recurrence of the page "ARCHITECTURE PREVIEW / FIELD NOTES", section 03 (GATED
// DELTANET equations), in chunks of 64 tokens.  Within a chunk, with
// g_t = sum_{s<=t} log alpha_s, gamma_t = exp(g_t) and S the state entering the chunk:
//     A_ti = beta_t exp(g_t - g_i) k_t.k_i  (i < t),   T = (I + A)^-1,  T_beta = T diag(beta)
//     u    = T_beta V - T_beta diag(gamma) K S                         (the WY/UT solve)
//     y_t  = gamma_t S^T q_t + sum_{i<=t} exp(g_t - g_i)(q_t.k_i) u_i
//     S   <- gamma_C S + sum_i exp(g_C - g_i) k_i u_i^T
//
// Scaled state.  The CTA keeps S~ = S / G in tensor memory, with a running scalar G (a
// product of chunk decays, >= 2^-48; when it would drop below, S~ is rescaled once and G
// restarts at 1).  Every decay factor then moves into operands that are independent of
// the state, and the state update becomes a plain tensor-core accumulation:
//     u   = T_beta V - W2 (K S~),         W2 = G T_beta diag(gamma)
//     y   = G diag(gamma) (Q S~) + P u,   P_ti = exp(g_t - g_i) q_t.k_i (i <= t)
//     S~ += K~^T u,                       K~ = diag(exp(g_C - g) / G') K
//
// T_beta and P of every chunk come from the chunk-prep pass (64 x 64 TF32 tiles in the
// workspace).  One CTA owns one (sequence, V head); all MMAs are M = 128 with the d_v
// index on the 128 tensor-memory lanes (transposed form), so every state-dependent A
// operand is read straight from tensor memory:
//   issuer (warp 0, one thread), per chunk
//     MMA_1   [X | Y1] = S~^T [K;Q]^T           (N=128, K=128)   X = (K S~)^T, Y1 = (Q S~)^T
//     MMA_2a  U^T      = V^T T_beta^T           (N=64,  K=64)    V from shared memory
//     MMA_2b  U^T     -= X W2^T                 (N=64,  K=64)    -> u^T
//     MMA_3   S~^T    += u^T K~                 (N=128, K=64)
//     MMA_4   Y       += u^T P^T                (N=64,  K=64)    onto Y = G gamma Y1
//   scale (warps 5-12), ahead of the issuer: the gates and their scan, G, W2 from T_beta,
//     K~ from K (in place)
//   epilogue (warps 1-4): Y = G gamma Y1 into tensor memory for MMA_4, y to global memory,
//     the occasional rescale of S~, the initial and final state.
// Shared memory holds the K/Q, K (token-major view), V, T_beta and P tiles (TMA, no
// multicast) and W2; all waits are bounded and a timed-out CTA writes NaN to its outputs.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "gdn_common.cuh"
#include "gdn_internal.h"
#include "tc_sm100.cuh"
#include "tma_map.cuh"

namespace gdn {

namespace {
using namespace tc;

constexpr int kThr = 416;          // 13 warps
constexpr int kEpiWarp0 = 1;       // warps 1-4
constexpr int kPrepWarp0 = 5;      // warps 5-12 (scale role)
constexpr int kPrepTid0 = kPrepWarp0 * 32;
constexpr int kEpiTid0 = kEpiWarp0 * 32;
constexpr int kBarPrep = 1, kBarEpi = 2;  // named barriers

// shared-memory map (bytes from a 1024-aligned base)
constexpr uint32_t OFF_KQ = 0;          // [K;Q]   K-major, 4 blocks x (K 8 KB | Q 8 KB)       64 KB
constexpr uint32_t OFF_KMN = 65536;     // K~      MN-major (32-byte granules), 64 x 128       32 KB
constexpr uint32_t OFF_VMN = 98304;     // V       MN-major (32-byte granules), 64 x 128       32 KB
constexpr uint32_t OFF_TB = 131072;     // T_beta  K-major [t][i], 2 buffers                   32 KB
constexpr uint32_t OFF_P = 163840;      // P       K-major [t][i], 2 buffers                   32 KB
constexpr uint32_t OFF_W2 = 196608;     // W2      K-major [t][i]                              16 KB
constexpr uint32_t OFF_MISC = 212992;
constexpr uint32_t OFF_GATE = OFF_MISC;            // g, beta, ks, w2s: 4 x 64 floats
constexpr uint32_t OFF_INFO = OFF_MISC + 1024;     // 2 x ChunkInfo
constexpr uint32_t OFF_BAR = OFF_MISC + 2048;      // mbarriers
constexpr uint32_t OFF_FLAGS = OFF_BAR + 256;      // TMEM base, abort flag, final G
constexpr uint32_t kSmem = OFF_FLAGS + 16;
constexpr uint32_t kSmemAlloc = kSmem + 1024;      // slack to align the base to 1024

// per-chunk values the scale role hands to the issuer and the epilogue (double-buffered)
struct ChunkInfo {
    float yscale[64];   // G gamma_t
    float rfac;         // G gamma_C: factor of the rescale of S~, if any
    float gnext;        // G after the chunk
    int rflag;          // rescale S~ before MMA_3
    int pad[61];
};
static_assert(sizeof(ChunkInfo) == 512, "ChunkInfo layout");

enum {
    B_KQ = 0, B_V, B_KMN,        // TMA arrivals
    B_TBL0, B_TBL1,              // TMA arrivals of T_beta into buffer 0 / 1
    B_PL0, B_PL1,                // TMA arrivals of P into buffer 0 / 1
    B_1, B_2, B_34,              // MMA completions
    B_TB, B_PK,                  // scale role: W2 and chunk info ready; K~ ready
    B_Y1,                        // epilogue: Y1 taken, Y = G gamma Y1 stored, S~ rescaled
    B_DRAIN0,                    // drain on the failure path
    kNumBars
};
static_assert(kNumBars * 8 <= 256, "barrier area");

// tensor memory columns (all 128 lanes)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t T_S = 0;      // S~^T                 128 cols
constexpr uint32_t T_XY = 128;   // [X | Y1]             128 cols
constexpr uint32_t T_U = 256;    // u^T                   64 cols
constexpr uint32_t T_Y = 320;    // G gamma Y1, then y     64 cols

constexpr float kRescaleBelow = 0x1p-48f;
constexpr uint32_t kWaitTries = 1u << 22;

__device__ __forceinline__ float4 tf32x4(float a, float b, float c, float d) {
    return make_float4(to_tf32(a), to_tf32(b), to_tf32(c), to_tf32(d));
}

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
// Bounded wait (each poll may sleep up to 1 us, so at most a few seconds in all) that
// gives up early once another role has raised the abort flag.
__device__ __forceinline__ bool wait_or_abort(uint64_t *m, uint32_t par, volatile int *abort_flag) {
    if (mbar_try_wait(m, par)) return true;
    for (uint32_t i = 0; i < kWaitTries; ++i) {
        if (mbar_try_wait_sleep(m, par, 1000)) return true;
        if ((i & 15) == 15 && *abort_flag) return false;
    }
    *abort_flag = 1;
    return false;
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

__device__ __forceinline__ uint16_t ld_raw(const bf16 *p) {
    uint16_t r;
    asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(r) : "l"(p));
    return r;
}
__device__ __forceinline__ uint32_t ld_raw(const float *p) {
    uint32_t r;
    asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(r) : "l"(p));
    return r;
}
__device__ __forceinline__ float raw_to_f32(uint16_t r) { return __uint_as_float((uint32_t)r << 16); }
__device__ __forceinline__ float raw_to_f32(uint32_t r) { return __uint_as_float(r); }

template <class TI> struct RawT { typedef uint32_t type; };
template <> struct RawT<bf16> { typedef uint16_t type; };

}  // namespace

struct TcParams {
    CUtensorMap tm_k;     // k^ rows, K-major 128B swizzle boxes (32 x 64)
    CUtensorMap tm_q;     // q^ rows, same
    CUtensorMap tm_kmn;   // k^ rows, 32-byte-granule swizzle boxes (MN-major operand)
    CUtensorMap tm_vmn;   // v^ rows, same
    CUtensorMap tm_tb;    // T_beta tiles as [chunk*Hv*64, 64] rows, K-major 128B swizzle boxes
    CUtensorMap tm_pm;    // P tiles, same
    const void *alpha, *beta;
    const int32_t *cu, *cfirst;
    const float *init;
    float *fin;
    void *out;
    int n_seqs, n_qk, n_v;
};

template <class TI, class TO>
__global__ void __launch_bounds__(kThr, 1) prefill_tc_kernel(const __grid_constant__ TcParams p) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    const uint32_t sb = smem_u32(sm);
    uint64_t *bar = (uint64_t *)(sm + OFF_BAR);
    uint32_t *tslot = (uint32_t *)(sm + OFF_FLAGS);
    volatile int *abort_flag = (volatile int *)(sm + OFF_FLAGS + 4);
    float *s_gfinal = (float *)(sm + OFF_FLAGS + 8);   // G after the last chunk
    ChunkInfo *info = (ChunkInfo *)(sm + OFF_INFO);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int h = blockIdx.x % p.n_v;
    const int b = blockIdx.x / p.n_v;
    const int gq = h / (p.n_v / p.n_qk);
    const int seq0 = p.cu[b], L = p.cu[b + 1] - p.cu[b];
    const int64_t v_row = (int64_t)p.n_v * kHeadDim;
    const int nchunks = (L + kChunk - 1) / kChunk;
    const int tile0 = (p.cfirst[b] * p.n_v + h) * kChunk;   // T_beta / P row of chunk 0

    if (tid == 0) {
        for (int i = 0; i < kNumBars; ++i) mbar_init(&bar[i], 1);
        *abort_flag = 0;
        *s_gfinal = 1.f;
    }
    if (warp == 0) {
        tmem_alloc(tslot, kTmemCols);
        tmem_relinquish();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tm = *tslot;

    // TMA issue (thread 0 only)
    auto issue_kq = [&](int c) {
        const int tok = seq0 + c * kChunk;
        mbar_expect_tx(&bar[B_KQ], 65536);
#pragma unroll
        for (int kb = 0; kb < 4; ++kb) {
            tma_load_2d(sb + OFF_KQ + kb * 16384, &p.tm_k, gq * kHeadDim + 32 * kb, tok, &bar[B_KQ]);
            tma_load_2d(sb + OFF_KQ + kb * 16384 + 8192, &p.tm_q, gq * kHeadDim + 32 * kb, tok, &bar[B_KQ]);
        }
    };
    auto issue_v = [&](int c) {
        const int tok = seq0 + c * kChunk;
        mbar_expect_tx(&bar[B_V], 32768);
#pragma unroll
        for (int jb = 0; jb < 4; ++jb)
            tma_load_2d(sb + OFF_VMN + jb * 8192, &p.tm_vmn, h * kHeadDim + 32 * jb, tok, &bar[B_V]);
    };
    auto issue_kmn = [&](int c) {
        const int tok = seq0 + c * kChunk;
        mbar_expect_tx(&bar[B_KMN], 32768);
#pragma unroll
        for (int db = 0; db < 4; ++db)
            tma_load_2d(sb + OFF_KMN + db * 8192, &p.tm_kmn, gq * kHeadDim + 32 * db, tok, &bar[B_KMN]);
    };
    auto issue_tile = [&](const CUtensorMap *m, uint32_t dst, int bar_i, int c) {  // T_beta or P
        const int row = tile0 + c * p.n_v * kChunk;
        mbar_expect_tx(&bar[bar_i], 16384);
        tma_load_2d(dst, m, 0, row, &bar[bar_i]);
        tma_load_2d(dst + 8192, m, 32, row, &bar[bar_i]);
    };
    auto issue_tb = [&](int c) { issue_tile(&p.tm_tb, sb + OFF_TB + (c & 1) * 16384, B_TBL0 + (c & 1), c); };
    auto issue_pm = [&](int c) { issue_tile(&p.tm_pm, sb + OFF_P + (c & 1) * 16384, B_PL0 + (c & 1), c); };

    // epilogue warps: initial state S~^T (lane j = column j of S) into tensor memory
    if (warp >= kEpiWarp0 && warp < kPrepWarp0) {
        const int q = warp & 3, j = 32 * q + lane;
        const uint32_t lrow = (uint32_t)(32 * q) << 16;
        const float *src = p.init ? p.init + ((int64_t)b * p.n_v + h) * kHeadDim * kHeadDim + j : nullptr;
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
        issue_kq(0);
        issue_v(0);
        issue_kmn(0);
        issue_tb(0);
        issue_pm(0);
        if (nchunks > 1) {
            issue_tb(1);
            issue_pm(1);
        }
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();

    if (warp == 0) {
        // ================================================================ issuer
        if (lane == 0) {
            bool ok = true;
            int n_kq = nchunks > 0 ? 1 : 0, n_v = n_kq, n_kmn = n_kq;
            int n_tb[2] = {nchunks > 0 ? 1 : 0, nchunks > 1 ? 1 : 0}, n_pm[2] = {n_tb[0], n_tb[1]};
            for (int c = 0; c < nchunks; ++c) {
                const uint32_t par = c & 1, bpar = (c >> 1) & 1;
                const int bsel = c & 1;
                // MMA_1: needs S~ (previous MMA_3, waited below) and [K;Q] of c; Y1 of c-1 was
                // drained before MMA_4 of c-1
                if (!(ok = wait_or_abort(&bar[B_KQ], par, abort_flag))) break;
                fence_after_sync();
                gemm_ts<128, 128, false, false>(tm + T_XY, tm + T_S, sb + OFF_KQ, 16384, false);
                mma_commit(&bar[B_1]);
                // MMA_2a: U^T = V^T T_beta^T (state-independent)
                if (!(ok = wait_or_abort(&bar[B_TB], par, abort_flag))) break;   // W2, info of c
                if (!(ok = wait_or_abort(&bar[B_TBL0 + bsel], bpar, abort_flag))) break;
                if (!(ok = wait_or_abort(&bar[B_V], par, abort_flag))) break;
                fence_after_sync();
                gemm<128, 64, 64, true, false>(tm + T_U, sb + OFF_VMN, 64, sb + OFF_TB + bsel * 16384, 8192, false);
                // MMA_2b: U^T -= X W2^T
                if (!(ok = wait_or_abort(&bar[B_1], par, abort_flag))) break;
                if (c + 1 < nchunks) { issue_kq(c + 1); ++n_kq; }   // [K;Q] of c is consumed
                fence_after_sync();
                gemm_ts<64, 64, false, true>(tm + T_U, tm + T_XY, sb + OFF_W2, 8192, true);
                mma_commit(&bar[B_2]);
                if (!(ok = wait_or_abort(&bar[B_2], par, abort_flag))) break;
                if (c + 1 < nchunks) { issue_v(c + 1); ++n_v; }
                if (c + 2 < nchunks) { issue_tb(c + 2); ++n_tb[bsel]; }  // this T_beta buffer is consumed
                // MMA_3 / MMA_4: S~ += u^T K~ (after the rescale of S~, if any); Y += u^T P^T
                if (!(ok = wait_or_abort(&bar[B_Y1], par, abort_flag))) break;
                if (!(ok = wait_or_abort(&bar[B_PK], par, abort_flag))) break;
                if (!(ok = wait_or_abort(&bar[B_PL0 + bsel], bpar, abort_flag))) break;
                fence_after_sync();
                gemm_ts<128, 64, true, false>(tm + T_S, tm + T_U, sb + OFF_KMN, 64, true);
                gemm_ts<64, 64, false, false>(tm + T_Y, tm + T_U, sb + OFF_P + bsel * 16384, 8192, true);
                mma_commit(&bar[B_34]);
                if (!(ok = wait_or_abort(&bar[B_34], par, abort_flag))) break;
                if (c + 1 < nchunks) { issue_kmn(c + 1); ++n_kmn; }
                if (c + 2 < nchunks) { issue_pm(c + 2); ++n_pm[bsel]; }
            }
            if (!ok) {
                // drain this thread's MMAs and the TMA loads it issued, each wait bounded
                mma_commit(&bar[B_DRAIN0]);
                mbar_wait(&bar[B_DRAIN0], 0, kWaitTries);
                if (n_kq) mbar_wait(&bar[B_KQ], (uint32_t)(n_kq - 1) & 1, kWaitTries);
                if (n_v) mbar_wait(&bar[B_V], (uint32_t)(n_v - 1) & 1, kWaitTries);
                if (n_kmn) mbar_wait(&bar[B_KMN], (uint32_t)(n_kmn - 1) & 1, kWaitTries);
                for (int i = 0; i < 2; ++i) {
                    if (n_tb[i]) mbar_wait(&bar[B_TBL0 + i], (uint32_t)(n_tb[i] - 1) & 1, kWaitTries);
                    if (n_pm[i]) mbar_wait(&bar[B_PL0 + i], (uint32_t)(n_pm[i] - 1) & 1, kWaitTries);
                }
            }
        }
    } else if (warp < kPrepWarp0) {
        // ================================================================ epilogue
        const int q = warp & 3, j = 32 * q + lane;
        const uint32_t lrow = (uint32_t)(32 * q) << 16;
        const bool leader = tid == kEpiTid0;
        auto ewait = [&](int i, uint32_t par) -> bool {
            const bool ok = wait_or_abort(&bar[i], par, abort_flag);
            return !bar_or(kBarEpi, 128, !ok);
        };
        auto publish = [&](int i) {  // this group's tensor-memory accesses are done
            fence_before_sync();
            bar_sync(kBarEpi, 128);
            if (leader) mbar_arrive(&bar[i]);
        };
        float gfinal = 1.f;
        bool ok = true;
        for (int c = 0; c < nchunks; ++c) {
            const uint32_t par = c & 1;
            const int n = min(kChunk, L - c * kChunk);
            const int64_t tok = seq0 + (int64_t)c * kChunk;
            if (!(ok = ewait(B_1, par))) break;
            // this chunk's scales (written by the prep before it released B_TB)
            if (!(ok = ewait(B_TB, par))) break;
            fence_after_sync();
            const ChunkInfo &ci = info[par];
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {  // Y = G gamma Y1, the base MMA_4 accumulates onto
                float v[32];
                tmem_ld32(tm + lrow + T_XY + 64 + 32 * h2, v);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] *= ci.yscale[32 * h2 + i];
                tmem_st32(tm + lrow + T_Y + 32 * h2, v);
            }
            gfinal = ci.gnext;
            if (ci.rflag) {  // rescale S~ (last read by MMA_1) before MMA_3 accumulates into it
                const float rfac = ci.rfac;
#pragma unroll
                for (int d0 = 0; d0 < kHeadDim; d0 += 32) {
                    float v[32];
                    tmem_ld32(tm + lrow + T_S + d0, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] *= rfac;
                    tmem_st32(tm + lrow + T_S + d0, v);
                }
            }
            tmem_wait_st();
            publish(B_Y1);
            if (!(ok = ewait(B_34, par))) break;
            fence_after_sync();
            TO *o = (TO *)p.out + tok * v_row + h * kHeadDim + j;
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                float v[32];
                tmem_ld32(tm + lrow + T_Y + 32 * h2, v);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int t = 32 * h2 + i;
                    if (t < n) o[(int64_t)t * v_row] = from_f32<TO>(v[i]);
                }
            }
        }
        (void)ok;
        if (leader) *s_gfinal = gfinal;   // the final state is written after the tear-down barrier
    } else {
        // ================================================================ scale role
        const int ptid = tid - kPrepTid0;                // 0..255
        const TI *al = (const TI *)p.alpha;
        const TI *be = (const TI *)p.beta;
        typedef typename RawT<TI>::type raw_t;
        raw_t a_raw = 0, b_raw = 0;
        auto load_gates = [&](int c) {                   // raw bits; converted one chunk later
            const int n = min(kChunk, L - c * kChunk);
            const int64_t tok = seq0 + (int64_t)c * kChunk;
            if (ptid < n) {
                a_raw = ld_raw(al + (tok + ptid) * p.n_v + h);
                b_raw = ld_raw(be + (tok + ptid) * p.n_v + h);
            }
        };
        auto pwait = [&](int i, uint32_t par) -> bool {
            const bool ok = wait_or_abort(&bar[i], par, abort_flag);
            return !bar_or(kBarPrep, 256, !ok);
        };
        float *g_s = (float *)(sm + OFF_GATE);
        float *beta_s = g_s + 64, *ks_s = g_s + 128, *w2s_s = g_s + 192;
        float G = 1.f;                                   // scale of S~ entering the chunk
        if (nchunks > 0 && ptid < kChunk) load_gates(0);

        for (int c = 0; c < nchunks; ++c) {
            const int n = min(kChunk, L - c * kChunk);
            const uint32_t par = c & 1, ppar = par ^ 1;
            const int bsel = c & 1;
            ChunkInfo *ci = &info[par];
            // ---- gates, their scan and the chunk's scales.  info[par] was last read by the
            // epilogue for chunk c-2, which released B_Y1 before this role's previous B_TB.
            if (ptid < kChunk) {
                g_s[ptid] = ptid < n ? safe_log_alpha(raw_to_f32(a_raw)) : 0.f;
                beta_s[ptid] = ptid < n ? raw_to_f32(b_raw) : 0.f;
                if (c + 1 < nchunks) load_gates(c + 1);
            }
            bar_sync(kBarPrep, 256);
            if (ptid < 32) {  // inclusive scan of log alpha, two rows per lane
                const int t0 = 2 * lane, t1 = t0 + 1;
                const float a0 = g_s[t0], a1 = g_s[t1];
                float s = a0 + a1;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, s, o);
                    if (lane >= o) s += y;
                }
                const float g0 = s - a1, g1 = s;
                const float glast = __shfl_sync(0xffffffffu, ((n - 1) & 1) ? g1 : g0, (n - 1) >> 1);
                const float gam0 = expf(g0), gam1 = expf(g1), gC = expf(glast);
                const float Gn = G * gC;
                const bool rflag = Gn < kRescaleBelow;
                const float kscale = rflag ? 1.f : 1.f / Gn;
                ks_s[t0] = t0 < n ? expf(glast - g0) * kscale : 0.f;
                ks_s[t1] = t1 < n ? expf(glast - g1) * kscale : 0.f;
                w2s_s[t0] = G * gam0;
                w2s_s[t1] = G * gam1;
                ci->yscale[t0] = G * gam0;
                ci->yscale[t1] = G * gam1;
                if (lane == 0) {
                    ci->rflag = rflag ? 1 : 0;
                    ci->rfac = Gn;
                    ci->gnext = rflag ? 1.f : Gn;
                }
            }
            // ---- W2 = G T_beta diag(gamma) (its buffer is free once MMA_2b of c-1 is done)
            if (!pwait(B_TBL0 + bsel, (c >> 1) & 1)) break;   // also orders the scan
            if (c > 0 && !pwait(B_2, ppar)) break;
            {
                const int t = ptid >> 2, i0 = (ptid & 3) * 16;
                const unsigned char *Tb = sm + OFF_TB + bsel * 16384;
                unsigned char *W2 = sm + OFF_W2;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int i = i0 + 4 * k;
                    const uint32_t off = kmaj_off(t, i, 64);
                    const float4 x = *reinterpret_cast<const float4 *>(Tb + off);
                    *reinterpret_cast<float4 *>(W2 + off) =
                        tf32x4(x.x * w2s_s[i], x.y * w2s_s[i + 1], x.z * w2s_s[i + 2], x.w * w2s_s[i + 3]);
                }
            }
            fence_smem_to_async();
            // the epilogue must have taken chunk c-1's info before B_TB moves on
            if (c > 0) {
                if (!pwait(B_Y1, ppar)) break;
            } else {
                bar_sync(kBarPrep, 256);
            }
            if (ptid == 0) mbar_arrive(&bar[B_TB]);
            // ---- K~ = diag(exp(g_C - g) / G') K, in place in the MN-major tile
            if (!pwait(B_KMN, par)) break;
            {
                const int blk = ptid >> 6, t = ptid & 63;
                unsigned char *row = sm + OFF_KMN + blk * 8192 + t * 128;
                const float sc = ks_s[t];
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const int kk = (k + t) & 7;   // staggered: rows 128 B apart share banks
                    float4 x = *reinterpret_cast<const float4 *>(row + 16 * kk);
                    *reinterpret_cast<float4 *>(row + 16 * kk) = tf32x4(x.x * sc, x.y * sc, x.z * sc, x.w * sc);
                }
            }
            fence_smem_to_async();
            bar_sync(kBarPrep, 256);
            if (ptid == 0) mbar_arrive(&bar[B_PK]);
            G = ci->gnext;
        }
    }

    // ---------------------------------------------------------------- tear-down
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (warp >= kEpiWarp0 && warp < kPrepWarp0) {
        const int q = warp & 3, j = 32 * q + lane;
        const uint32_t lrow = (uint32_t)(32 * q) << 16;
        const bool failed = *abort_flag != 0;
        const float gf = *s_gfinal;
        if (p.fin) {
            float *dst = p.fin + ((int64_t)b * p.n_v + h) * kHeadDim * kHeadDim + j;
#pragma unroll
            for (int d0 = 0; d0 < kHeadDim; d0 += 32) {
                float s[32];
                tmem_ld32(tm + lrow + T_S + d0, s);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    dst[(int64_t)(d0 + i) * kHeadDim] = failed ? __int_as_float(0x7fc00000) : gf * s[i];
            }
        }
        if (failed) {
            for (int e = tid - kEpiTid0; e < L * kHeadDim; e += 128) {
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
template <class TI, class TO>
static cudaError_t launch_tc_t(const TcParams &p, cudaStream_t s) {
    auto k = prefill_tc_kernel<TI, TO>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemAlloc);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)((int64_t)p.n_seqs * p.n_v);
    TraceLaunch tl(s, "prefill_tc");
    k<<<grid, kThr, kSmemAlloc, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_prefill_tc(const ScanParams &sp, int64_t total_tokens, bool in_bf16,
                              bool out_bf16, cudaStream_t s) {
    if (sp.n_seqs <= 0) return cudaSuccess;
    TcParams p{};
    const int64_t T = total_tokens > 0 ? total_tokens : 1;
    const int64_t wqk = (int64_t)sp.n_qk * kHeadDim, wv = (int64_t)sp.n_v * kHeadDim;
    // T_beta / P tiles: rows (chunk * Hv + h) * 64 + t of a 64-wide matrix (int32 TMA coordinates)
    const int64_t tile_rows = (total_tokens > 0 ? sp.max_chunks : 1) * sp.n_v * kChunk;
    if (tile_rows >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
    if (!encode_rows(&p.tm_k, sp.kh, wqk, T, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_rows(&p.tm_q, sp.qh, wqk, T, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_rows(&p.tm_kmn, sp.kh, wqk, T, CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B) ||
        !encode_rows(&p.tm_vmn, sp.vh, wv, T, CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B) ||
        !encode_rows(&p.tm_tb, sp.tb, kChunk, tile_rows, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_rows(&p.tm_pm, sp.pm, kChunk, tile_rows, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    p.alpha = sp.alpha; p.beta = sp.beta; p.cu = sp.cu; p.cfirst = sp.cfirst;
    p.init = sp.init; p.fin = sp.fin;
    p.out = sp.out; p.n_seqs = sp.n_seqs; p.n_qk = sp.n_qk; p.n_v = sp.n_v;
    if (in_bf16) return out_bf16 ? launch_tc_t<gdn::bf16, gdn::bf16>(p, s) : launch_tc_t<gdn::bf16, float>(p, s);
    return out_bf16 ? launch_tc_t<float, gdn::bf16>(p, s) : launch_tc_t<float, float>(p, s);
}

}  // namespace gdn
