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
// One CTA owns one (sequence, V head); all MMAs are M = 128 with the d_v index on the
// 128 tensor-memory lanes (transposed form), so every state-dependent A operand is read
// straight from tensor memory:
//   issuer (warp 0, one thread), per chunk
//     MMA_1   [X | Y1] = S~^T [K;Q]^T           (N=128, K=128)   X = (K S~)^T, Y1 = (Q S~)^T
//     MMA_2a  U^T      = V^T T_beta^T           (N=64,  K=64)    V from shared memory
//     MMA_2b  U^T     -= X W2^T                 (N=64,  K=64)    -> u^T
//     MMA_3   S~^T    += u^T K~                 (N=128, K=64)
//     MMA_4   Y       += u^T P^T                (N=64,  K=64)    onto Y = G gamma Y1
//   prep (warps 5-12), the state-independent work of the same chunk, ahead of the issuer:
//     gates and their scan, MMA_a = [K;Q] K^T (M=128, N=64, K=128), A and P, the 64 x 64
//     unit-lower-triangular inverse on CUDA cores, T_beta, W2, K~
//   epilogue (warps 1-4): Y = G gamma Y1 into tensor memory for MMA_4, y to global memory,
//     the occasional rescale of S~, the initial and final state.
// Shared memory holds the K/Q, K (token-major view) and V tiles (TMA, no multicast) and
// the prep outputs; all waits are bounded and a timed-out CTA writes NaN to its outputs.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "gdn_common.cuh"
#include "gdn_internal.h"
#include "tc_sm100.cuh"

namespace gdn {

namespace {
using namespace tc;

constexpr int kThr = 416;          // 13 warps
constexpr int kEpiWarp0 = 1;       // warps 1-4
constexpr int kPrepWarp0 = 5;      // warps 5-12
constexpr int kPrepTid0 = kPrepWarp0 * 32;
constexpr int kEpiTid0 = kEpiWarp0 * 32;
constexpr int kBarPrep = 1, kBarEpi = 2;  // named barriers

// shared-memory map (bytes from a 1024-aligned base)
constexpr uint32_t OFF_KQ = 0;          // [K;Q]   K-major, 4 blocks x (K 8 KB | Q 8 KB)       64 KB
constexpr uint32_t OFF_KMN = 65536;     // K~      MN-major (32-byte granules), 64 x 128       32 KB
constexpr uint32_t OFF_VMN = 98304;     // V       MN-major (32-byte granules), 64 x 128       32 KB
constexpr uint32_t OFF_TB = 131072;     // T_beta  K-major [t][i]                              16 KB
constexpr uint32_t OFF_W2 = 147456;     // W2      K-major [t][i]                              16 KB
constexpr uint32_t OFF_P = 163840;      // P       K-major [t][i]                              16 KB
constexpr uint32_t OFF_AS = 180224;     // A scratch (fp32, swizzled rows)                     16 KB
constexpr uint32_t OFF_TS = 196608;     // T scratch (fp32, swizzled rows)                     16 KB
constexpr uint32_t OFF_MISC = 212992;
constexpr uint32_t OFF_GATE = OFF_MISC;            // g, beta, ks, w2s: 4 x 64 floats
constexpr uint32_t OFF_INFO = OFF_MISC + 1024;     // 2 x ChunkInfo
constexpr uint32_t OFF_INV = OFF_MISC + 2048;      // 2 x 256 floats (block products)
constexpr uint32_t OFF_BAR = OFF_MISC + 4096;      // mbarriers
constexpr uint32_t OFF_FLAGS = OFF_BAR + 128;      // TMEM base, abort flag
constexpr uint32_t kSmem = OFF_FLAGS + 16;
constexpr uint32_t kSmemAlloc = kSmem + 1024;      // slack to align the base to 1024

// per-chunk values the prep hands to the issuer and the epilogue (double-buffered)
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
    B_A, B_1, B_2, B_34,         // MMA completions
    B_TB, B_PK,                  // prep: T_beta/W2/info ready; K~/P ready
    B_Y1,                        // epilogue: Y1 taken, Y = G gamma Y1 stored, S~ rescaled
    B_DRAIN0, B_DRAIN1,          // drains on the failure path
    kNumBars
};

// tensor memory columns (all 128 lanes)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t T_S = 0;      // S~^T                 128 cols
constexpr uint32_t T_XY = 128;   // [X | Y1]             128 cols
constexpr uint32_t T_U = 256;    // u^T                   64 cols
constexpr uint32_t T_Y = 320;    // G gamma Y1, then y     64 cols
constexpr uint32_t T_A = 384;    // [K;Q] K^T             64 cols

constexpr float kRescaleBelow = 0x1p-48f;
constexpr uint32_t kWaitTries = 1u << 22;

// fp32 scratch [64][64] with 16-byte chunks XOR-swizzled by row
__device__ __forceinline__ int scr(int r, int c) { return r * 64 + ((((c >> 2) ^ (r & 7)) << 2) | (c & 3)); }

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
    const void *alpha, *beta;
    const int32_t *cu;
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
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();

    if (warp == 0) {
        // ================================================================ issuer
        if (lane == 0) {
            bool ok = true;
            int n_kq = nchunks > 0 ? 1 : 0, n_v = n_kq, n_kmn = n_kq;
            for (int c = 0; c < nchunks; ++c) {
                const uint32_t par = c & 1;
                // MMA_1: needs S~ (previous MMA_3, waited below) and [K;Q] of c; Y1 of c-1 was
                // drained before MMA_4 of c-1
                if (!(ok = wait_or_abort(&bar[B_KQ], par, abort_flag))) break;
                fence_after_sync();
                gemm_ts<128, 128, false, false>(tm + T_XY, tm + T_S, sb + OFF_KQ, 16384, false);
                mma_commit(&bar[B_1]);
                // MMA_2a: U^T = V^T T_beta^T (state-independent)
                if (!(ok = wait_or_abort(&bar[B_TB], par, abort_flag))) break;
                if (!(ok = wait_or_abort(&bar[B_V], par, abort_flag))) break;
                fence_after_sync();
                gemm<128, 64, 64, true, false>(tm + T_U, sb + OFF_VMN, 64, sb + OFF_TB, 8192, false);
                // MMA_2b: U^T -= X W2^T
                if (!(ok = wait_or_abort(&bar[B_1], par, abort_flag))) break;
                if (c + 1 < nchunks) { issue_kq(c + 1); ++n_kq; }   // [K;Q] is free (MMA_a(c) done before B_TB)
                fence_after_sync();
                gemm_ts<64, 64, false, true>(tm + T_U, tm + T_XY, sb + OFF_W2, 8192, true);
                mma_commit(&bar[B_2]);
                if (!(ok = wait_or_abort(&bar[B_2], par, abort_flag))) break;
                if (c + 1 < nchunks) { issue_v(c + 1); ++n_v; }
                // MMA_3 / MMA_4: S~ += u^T K~ (after the rescale of S~, if any); Y += u^T P^T
                if (!(ok = wait_or_abort(&bar[B_Y1], par, abort_flag))) break;
                if (!(ok = wait_or_abort(&bar[B_PK], par, abort_flag))) break;
                fence_after_sync();
                gemm_ts<128, 64, true, false>(tm + T_S, tm + T_U, sb + OFF_KMN, 64, true);
                gemm_ts<64, 64, false, false>(tm + T_Y, tm + T_U, sb + OFF_P, 8192, true);
                mma_commit(&bar[B_34]);
                if (!(ok = wait_or_abort(&bar[B_34], par, abort_flag))) break;
                if (c + 1 < nchunks) { issue_kmn(c + 1); ++n_kmn; }
            }
            if (!ok) {
                // drain this thread's MMAs and the TMA loads it issued, each wait bounded
                mma_commit(&bar[B_DRAIN0]);
                mbar_wait(&bar[B_DRAIN0], 0, kWaitTries);
                if (n_kq) mbar_wait(&bar[B_KQ], (uint32_t)(n_kq - 1) & 1, kWaitTries);
                if (n_v) mbar_wait(&bar[B_V], (uint32_t)(n_v - 1) & 1, kWaitTries);
                if (n_kmn) mbar_wait(&bar[B_KMN], (uint32_t)(n_kmn - 1) & 1, kWaitTries);
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
        // ================================================================ prep
        const int ptid = tid - kPrepTid0;                // 0..255
        const int q = warp & 3;                          // tensor-memory lane quarter
        const int ch = (warp - kPrepWarp0) >> 2;         // which 32 of the 64 columns of [K;Q]K^T
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
        auto pwait_or_sync = [&](bool need, int i, uint32_t par) -> bool {
            if (need) return pwait(i, par);
            bar_sync(kBarPrep, 256);
            return true;
        };
        float *g_s = (float *)(sm + OFF_GATE);
        float *beta_s = g_s + 64, *ks_s = g_s + 128, *w2s_s = g_s + 192;
        float *Ascr = (float *)(sm + OFF_AS);
        float *Tscr = (float *)(sm + OFF_TS);
        float *inv_s = (float *)(sm + OFF_INV);
        float G = 1.f;                                   // scale of S~ entering the chunk
        if (nchunks > 0 && ptid < kChunk) load_gates(0);

        for (int c = 0; c < nchunks; ++c) {
            const int n = min(kChunk, L - c * kChunk);
            const uint32_t par = c & 1, ppar = par ^ 1;
            ChunkInfo *ci = &info[par];

            // ---- gates, their scan and the chunk's scales
            if (!pwait(B_KQ, par)) break;
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
                g_s[t0] = g0;
                g_s[t1] = g1;
                ks_s[t0] = t0 < n ? expf(glast - g0) * kscale : 0.f;
                ks_s[t1] = t1 < n ? expf(glast - g1) * kscale : 0.f;
                w2s_s[t0] = G * gam0 * beta_s[t0];
                w2s_s[t1] = G * gam1 * beta_s[t1];
                ci->yscale[t0] = G * gam0;
                ci->yscale[t1] = G * gam1;
                if (lane == 0) {
                    ci->rflag = rflag ? 1 : 0;
                    ci->rfac = Gn;
                    ci->gnext = rflag ? 1.f : Gn;
                }
            }
            bar_sync(kBarPrep, 256);
            if (ptid == 0) {
                fence_after_sync();
                gemm<128, 64, 128, false, false>(tm + T_A, sb + OFF_KQ, 16384, sb + OFF_KQ, 16384, false);
                mma_commit(&bar[B_A]);
            }
            // ---- epilogue a: A (fp32 scratch) and P (K-major tile; free once MMA_4 of c-1 is done)
            if (c > 0 && !pwait(B_34, ppar)) break;
            if (!pwait(B_A, par)) break;
            fence_after_sync();
            {
                float v[32];
                tmem_ld32(taddr(tm + T_A, 32 * q, 32 * ch), v);
                tmem_wait_ld();
                if (q < 2) {  // K K^T rows
                    const int t = 32 * q + lane;
                    const float gt = g_s[t], bt = beta_s[t];
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        float a4[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int i = 32 * ch + 4 * k + e;
                            a4[e] = (i < t && t < n) ? bt * expf(gt - g_s[i]) * v[4 * k + e] : 0.f;
                        }
                        *reinterpret_cast<float4 *>(&Ascr[scr(t, 32 * ch + 4 * k)]) = make_float4(a4[0], a4[1], a4[2], a4[3]);
                    }
                } else {  // Q K^T rows
                    const int t = 32 * (q - 2) + lane;
                    const float gt = g_s[t];
                    unsigned char *Pt = sm + OFF_P;
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        float p4[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int i = 32 * ch + 4 * k + e;
                            p4[e] = (i <= t && t < n) ? expf(gt - g_s[i]) * v[4 * k + e] : 0.f;
                        }
                        *reinterpret_cast<float4 *>(Pt + kmaj_off(t, 32 * ch + 4 * k, 64)) = tf32x4(p4[0], p4[1], p4[2], p4[3]);
                    }
                }
            }
            fence_before_sync();
            bar_sync(kBarPrep, 256);
            // ---- T = (I + A)^-1: 16 x 16 diagonal blocks, two 32 x 32 halves, one merge
            if (ptid < 64) {  // diagonal blocks: column cc of block bb, right-looking updates
                const int bb = ptid >> 4, cc = ptid & 15, o = 16 * bb;
                float x[16];
#pragma unroll
                for (int r = 0; r < 16; ++r) x[r] = (r == cc) ? 1.f : 0.f;
#pragma unroll
                for (int m = 0; m < 15; ++m) {
                    const float xm = x[m];
#pragma unroll
                    for (int r = m + 1; r < 16; ++r) x[r] = fmaf(-Ascr[scr(o + r, o + m)], xm, x[r]);
                }
#pragma unroll
                for (int r = 0; r < 16; ++r) Tscr[scr(o + r, o + cc)] = x[r];
            } else {  // zero the 16 x 16 blocks above the diagonal that the products read
                for (int e = ptid - 64; e < 512; e += 192) {
                    const int blk = e >> 8, r = (e >> 4) & 15, cc = e & 15;
                    const int o = 32 * blk;
                    Tscr[scr(o + r, o + 16 + cc)] = 0.f;
                }
            }
            bar_sync(kBarPrep, 256);
            if (ptid < 128) {  // halves: M = A_10 T_00 (16 x 16 blocks)
                const int hh = ptid >> 6, rr = (ptid >> 2) & 15, c4 = (ptid & 3) * 4, o = 32 * hh;
                float a4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int m = 0; m < 16; ++m) {
                    const float a = Ascr[scr(o + 16 + rr, o + m)];
                    const float4 t4 = *reinterpret_cast<const float4 *>(&Tscr[scr(o + m, o + c4)]);
                    a4[0] = fmaf(a, t4.x, a4[0]); a4[1] = fmaf(a, t4.y, a4[1]);
                    a4[2] = fmaf(a, t4.z, a4[2]); a4[3] = fmaf(a, t4.w, a4[3]);
                }
                *reinterpret_cast<float4 *>(&inv_s[hh * 256 + rr * 16 + c4]) = make_float4(a4[0], a4[1], a4[2], a4[3]);
            }
            bar_sync(kBarPrep, 256);
            if (ptid < 128) {  // T_10 = -T_11 M
                const int hh = ptid >> 6, rr = (ptid >> 2) & 15, c4 = (ptid & 3) * 4, o = 32 * hh;
                float a4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int m = 0; m < 16; ++m) {
                    const float t = Tscr[scr(o + 16 + rr, o + 16 + m)];
                    const float4 m4 = *reinterpret_cast<const float4 *>(&inv_s[hh * 256 + m * 16 + c4]);
                    a4[0] = fmaf(t, m4.x, a4[0]); a4[1] = fmaf(t, m4.y, a4[1]);
                    a4[2] = fmaf(t, m4.z, a4[2]); a4[3] = fmaf(t, m4.w, a4[3]);
                }
                *reinterpret_cast<float4 *>(&Tscr[scr(o + 16 + rr, o + c4)]) = make_float4(-a4[0], -a4[1], -a4[2], -a4[3]);
            }
            bar_sync(kBarPrep, 256);
            {  // merge: M = A_bl T_top, parked in the (unused) upper-right block
                const int r = ptid >> 3, c4 = (ptid & 7) * 4;
                float a4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int m = 0; m < 32; ++m) {
                    const float a = Ascr[scr(32 + r, m)];
                    const float4 t4 = *reinterpret_cast<const float4 *>(&Tscr[scr(m, c4)]);
                    a4[0] = fmaf(a, t4.x, a4[0]); a4[1] = fmaf(a, t4.y, a4[1]);
                    a4[2] = fmaf(a, t4.z, a4[2]); a4[3] = fmaf(a, t4.w, a4[3]);
                }
                *reinterpret_cast<float4 *>(&Tscr[scr(r, 32 + c4)]) = make_float4(a4[0], a4[1], a4[2], a4[3]);
            }
            bar_sync(kBarPrep, 256);
            {  // T_bl = -T_br M
                const int r = ptid >> 3, c4 = (ptid & 7) * 4;
                float a4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int m = 0; m < 32; ++m) {
                    const float t = Tscr[scr(32 + r, 32 + m)];
                    const float4 m4 = *reinterpret_cast<const float4 *>(&Tscr[scr(m, 32 + c4)]);
                    a4[0] = fmaf(t, m4.x, a4[0]); a4[1] = fmaf(t, m4.y, a4[1]);
                    a4[2] = fmaf(t, m4.z, a4[2]); a4[3] = fmaf(t, m4.w, a4[3]);
                }
                *reinterpret_cast<float4 *>(&Tscr[scr(32 + r, c4)]) = make_float4(-a4[0], -a4[1], -a4[2], -a4[3]);
            }
            // ---- T_beta and W2 (their buffers are free once MMA_2b of c-1 is done)
            if (!pwait_or_sync(c > 0, B_2, ppar)) break;   // also orders the T products
            {
                const int t = ptid >> 2, i0 = (ptid & 3) * 16;
                const bool upper_right = t < 32 && i0 >= 32;
                unsigned char *Tb = sm + OFF_TB, *W2 = sm + OFF_W2;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int i = i0 + 4 * k;
                    float4 x = *reinterpret_cast<const float4 *>(&Tscr[scr(t, i)]);
                    if (upper_right) x = make_float4(0.f, 0.f, 0.f, 0.f);
                    *reinterpret_cast<float4 *>(Tb + kmaj_off(t, i, 64)) =
                        tf32x4(x.x * beta_s[i], x.y * beta_s[i + 1], x.z * beta_s[i + 2], x.w * beta_s[i + 3]);
                    *reinterpret_cast<float4 *>(W2 + kmaj_off(t, i, 64)) =
                        tf32x4(x.x * w2s_s[i], x.y * w2s_s[i + 1], x.z * w2s_s[i + 2], x.w * w2s_s[i + 3]);
                }
            }
            fence_smem_to_async();
            // the epilogue must have taken chunk c-1's info before B_TB moves on
            if (!pwait_or_sync(c > 0, B_Y1, ppar)) break;
            if (ptid == 0) mbar_arrive(&bar[B_TB]);
            // ---- K~ = diag(exp(g_C - g) / G') K, in place in the MN-major tile
            if (!pwait(B_KMN, par)) break;
            {
                const int blk = ptid >> 6, t = ptid & 63;
                unsigned char *row = sm + OFF_KMN + blk * 8192 + t * 128;
                const float s = ks_s[t];
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const int kk = (k + t) & 7;   // staggered: rows 128 B apart share banks
                    float4 x = *reinterpret_cast<const float4 *>(row + 16 * kk);
                    *reinterpret_cast<float4 *>(row + 16 * kk) = tf32x4(x.x * s, x.y * s, x.z * s, x.w * s);
                }
            }
            fence_smem_to_async();
            bar_sync(kBarPrep, 256);
            if (ptid == 0) mbar_arrive(&bar[B_PK]);
            G = ci->gnext;
        }
        if (*abort_flag && ptid == 0) {  // drain MMA_a
            mma_commit(&bar[B_DRAIN1]);
            mbar_wait(&bar[B_DRAIN1], 0, kWaitTries);
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
static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (PFN_cuTensorMapEncodeTiled_v12000)f;
    }
    return fn;
}

// 2-D map over a [rows x width] fp32 matrix, boxes of 32 columns x 64 rows
static bool encode_rows(CUtensorMap *m, const float *base, int64_t width, int64_t rows,
                        CUtensorMapSwizzle swz) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)width, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)width * 4};
    cuuint32_t box[2] = {32, 64}, es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, (void *)base, dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

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
    if (!encode_rows(&p.tm_k, sp.kh, wqk, T, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_rows(&p.tm_q, sp.qh, wqk, T, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_rows(&p.tm_kmn, sp.kh, wqk, T, CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B) ||
        !encode_rows(&p.tm_vmn, sp.vh, wv, T, CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B))
        return cudaErrorInvalidValue;
    p.alpha = sp.alpha; p.beta = sp.beta; p.cu = sp.cu; p.init = sp.init; p.fin = sp.fin;
    p.out = sp.out; p.n_seqs = sp.n_seqs; p.n_qk = sp.n_qk; p.n_v = sp.n_v;
    if (in_bf16) return out_bf16 ? launch_tc_t<gdn::bf16, gdn::bf16>(p, s) : launch_tc_t<gdn::bf16, float>(p, s);
    return out_bf16 ? launch_tc_t<float, gdn::bf16>(p, s) : launch_tc_t<float, float>(p, s);
}

}  // namespace gdn
