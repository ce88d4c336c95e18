// Chunked gated-delta-rule prefill on the sm_100a tensor cores (TF32 MMAs, fp32 state).
//
// The recurrence of the page "ARCHITECTURE PREVIEW / FIELD NOTES", section 03 (GATED
// DELTANET equations), in chunks of 64 tokens.  Within a chunk, with
// g_t = sum_{s<=t} log alpha_s, gamma_t = exp(g_t) and S the state entering the chunk:
//     A_ti = beta_t exp(g_t - g_i) k_t.k_i  (i < t),   T = (I + A)^-1,  T_beta = T diag(beta)
//     u    = T_beta (V - diag(gamma) K S)                             (the WY/UT solve)
//     y_t  = gamma_t S^T q_t + sum_{i<=t} exp(g_t - g_i)(q_t.k_i) u_i
//     S   <- gamma_C S + sum_i exp(g_C - g_i) k_i u_i^T
// (u = U - W S with U = T diag(beta) V and W = T diag(beta gamma) K, regrouped so that
// W never has to be formed).
//
// One CTA owns one (sequence, V head, 64-column slice j of d_v); the column split is
// exact.  Its 16 warps form two groups that run one chunk apart:
//  * prep (warps 8-15), state-independent, for chunk c+1:
//        MMA_a  [K;Q] K^T   (M=128, N=64, K=128)  -> A (strict lower), P (lower)
//        64 x 64 unit-lower-triangular inverse on CUDA cores -> T_beta
//  * chain (warps 0-7), the serial state recurrence of chunk c, in transposed form so
//    that every chain operand lives in tensor memory (A operands read from TMEM):
//        MMA_1  S^T [K;Q]^T   (M=64, N=128, K=128) -> (K S)^T, (Q S)^T
//        MMA_2  V'^T T_beta^T (M=64, N=64, K=64)   -> u^T        (V' = V - gamma*K S)
//        MMA_3  u~^T K        (M=64, N=128, K=64)  -> dS^T       (u~ = exp(g_C - g) u)
//        MMA_4  u^T P^T       (M=64, N=64, K=64)   accumulated onto (gamma*Q S)^T -> y^T
// Tensor memory (row j of an M=64 tile at lane 32*(j/16) + j%16 + base, base 0 or 16):
// the fp32 state lives in the upper half-lanes next to its TF32 operand copy.  Shared
// memory holds only the K/Q tiles (TMA, no multicast), the V tile and the
// double-buffered prep outputs.  All waits are bounded.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "gdn_common.cuh"
#include "gdn_internal.h"
#include "tc_sm100.cuh"

namespace gdn {

namespace {
using namespace tc;

constexpr int kN = 64;          // d_v columns per CTA
constexpr int kNS = kHeadDim / kN;
constexpr int kThr = 512;
constexpr int kGroup = 256;     // threads per group

// shared-memory map (bytes from a 1024-aligned base)
constexpr uint32_t OFF_KQ = 0;          // [K;Q]  K-major, 4 blocks x (K 8 KB | Q 8 KB)     64 KB
constexpr uint32_t OFF_KMN = 65536;     // K      MN-major R=64 (i) x 128 (d)              32 KB
constexpr uint32_t OFF_V = 98304;       // V      [t][j] K-major swizzle (read by threads)  16 KB
constexpr uint32_t OFF_TB = 114688;     // T_beta K-major [t][i], 2 buffers                 32 KB
constexpr uint32_t OFF_P = 147456;      // P      K-major [t][i], 2 buffers                 32 KB
constexpr uint32_t OFF_AS = 180224;     // A scratch (fp32, swizzled rows)                  16 KB
constexpr uint32_t OFF_TS = 196608;     // T scratch (fp32, swizzled rows)                  16 KB
constexpr uint32_t OFF_MISC = 212992;
constexpr uint32_t OFF_GATE = OFF_MISC;            // 2 buffers x {g, gamma, beta, kd}[64]  2 KB
constexpr uint32_t OFF_INV = OFF_MISC + 2048;      // 2 x 256 floats (block products)      2 KB
constexpr uint32_t OFF_BAR = OFF_MISC + 4096;      // mbarriers
constexpr uint32_t OFF_TSLOT = OFF_BAR + 128;
constexpr uint32_t kSmem = OFF_TSLOT + 16;
constexpr uint32_t kSmemAlloc = kSmem + 1024;      // slack to align the base to 1024

enum { B_KQ = 0, B_V, B_KMN, B_A, B_PREP, B_1, B_2, B_3, kNumBars };

// tensor memory: columns (lower half-lanes | upper half-lanes of each M=64 tile)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t T_A = 0;        // [K;Q]K^T, M=128 (all lanes)                        64 cols
constexpr uint32_t T_1 = 64;       // lower: [(K S)^T | (Q S)^T -> y^T]  upper: dS^T     128 cols
constexpr uint32_t T_S = 192;      // lower: S^T (TF32 operand)          upper: S^T fp32 128 cols
constexpr uint32_t T_V = 320;      // lower: V'^T (operand)              upper: u~^T      64 cols
constexpr uint32_t T_U = 384;      // lower: u^T (accumulator, then operand)              64 cols
constexpr uint32_t kUpper = 16u << 16;  // lane offset of the upper half-lanes

constexpr uint32_t kWaitTries = 1u << 22;

// fp32 scratch [64][64] with 16-byte chunks XOR-swizzled by row
__device__ __forceinline__ int scr(int r, int c) { return r * 64 + ((((c >> 2) ^ (r & 7)) << 2) | (c & 3)); }

__device__ __forceinline__ float4 tf32x4(float a, float b, float c, float d) {
    return make_float4(to_tf32(a), to_tf32(b), to_tf32(c), to_tf32(d));
}

// named barrier over one 256-thread group; returns true if any thread passed `pred`
__device__ __forceinline__ bool group_sync_or(int id, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.b32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, 256, p;\n\tselp.u32 %0, 1, 0, q;\n\t}\n"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ void group_sync(int id) {
    asm volatile("bar.sync %0, 256;" ::"r"(id) : "memory");
}

// A from tensor memory (K-major), B from a shared-memory descriptor
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t id, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d),
        "r"(a_tmem), "l"(b), "r"(id), "r"(acc));
}
// D[64 x N] (+)= A_tmem[64 x K] B[K x N]; B K-major (b_arg = block stride) or MN-major (b_arg = R)
template <int N, int K, bool B_MN>
__device__ __forceinline__ void gemm_ts(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_base, uint32_t b_arg,
                                        bool accumulate) {
    constexpr uint32_t id = idesc_tf32(64, N, false, B_MN);
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
    CUtensorMap tm_kmn;   // k^ rows, MN-major 32B-granule swizzle boxes
    CUtensorMap tm_v;     // v^ rows, K-major 128B swizzle boxes
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
    uint32_t *tslot = (uint32_t *)(sm + OFF_TSLOT);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int quarter = warp & 3;
    const int slice = blockIdx.x % kNS;
    const int h = (blockIdx.x / kNS) % p.n_v;
    const int b = blockIdx.x / (kNS * p.n_v);
    const int gq = h / (p.n_v / p.n_qk);
    const int seq0 = p.cu[b], L = p.cu[b + 1] - p.cu[b];
    const int col0 = slice * kN;
    const int64_t v_row = (int64_t)p.n_v * kHeadDim;
    const int nchunks = (L + kChunk - 1) / kChunk;

    if (tid == 0) {
        for (int i = 0; i < kNumBars; ++i) mbar_init(&bar[i], 1);
    }
    if (warp == 0) {
        tmem_alloc(tslot, kTmemCols);
        tmem_relinquish();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tm = *tslot;

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
        mbar_expect_tx(&bar[B_V], 16384);
#pragma unroll
        for (int jb = 0; jb < 2; ++jb)
            tma_load_2d(sb + OFF_V + jb * 8192, &p.tm_v, h * kHeadDim + col0 + 32 * jb, tok, &bar[B_V]);
    };
    auto issue_kmn = [&](int c) {
        const int tok = seq0 + c * kChunk;
        mbar_expect_tx(&bar[B_KMN], 32768);
#pragma unroll
        for (int db = 0; db < 4; ++db)
            tma_load_2d(sb + OFF_KMN + db * 8192, &p.tm_kmn, gq * kHeadDim + 32 * db, tok, &bar[B_KMN]);
    };

    bool failed = false;

    if (warp < 8) {
        // ================================================================ chain group
        const int ch = warp >> 2;                      // which 32 of each 64 columns
        const bool upper = lane >= 16;
        const int j = 16 * quarter + (lane & 15);      // row of the M=64 tiles (column of d_v)
        const int tcol = 32 * ch;                      // this thread's 32 columns of 64
        const uint32_t lrow = (uint32_t)(32 * quarter) << 16;  // warp's lane quarter
        auto wait_all = [&](int i, uint32_t par) -> bool {
            const bool ok = mbar_wait(&bar[i], par, kWaitTries);
            return !group_sync_or(1, !ok);
        };
        // initial state: lower lanes the TF32 copy of S^T, upper lanes S^T in fp32
        {
            const float *src = p.init ? p.init + ((int64_t)b * p.n_v + h) * kHeadDim * kHeadDim + col0 + j : nullptr;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int d0 = 64 * ch + 32 * half;
                float v[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const float s = src ? src[(int64_t)(d0 + i) * kHeadDim] : 0.f;
                    v[i] = upper ? s : to_tf32(s);
                }
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
        group_sync(1);

        for (int c = 0; c < nchunks; ++c) {
            const int n = min(kChunk, L - c * kChunk);
            const int64_t tok = seq0 + (int64_t)c * kChunk;
            const uint32_t par = c & 1;
            const float *gate = (const float *)(sm + OFF_GATE + (c & 1) * 1024);
            const float *gam_s = gate + 64, *kd_s = gate + 192;

            // ---- MMA_1: S^T [K;Q]^T
            if (!wait_all(B_KQ, par)) { failed = true; break; }
            if (tid == 0) {
                fence_after_sync();
                gemm_ts<128, 128, false>(tm + T_1, tm + T_S, sb + OFF_KQ, 16384, false);
                mma_commit(&bar[B_1]);
            }
            if (!wait_all(B_1, par)) { failed = true; break; }
            if (!wait_all(B_PREP, par)) { failed = true; break; }  // gates, T_beta, P of chunk c
            if (tid == 0 && c + 1 < nchunks) issue_kq(c + 1);      // prep and chain are done with [K;Q]
            if (!wait_all(B_V, par)) { failed = true; break; }
            fence_after_sync();

            // ---- epilogue 1: V'^T = V^T - gamma * (K S)^T ; (Q S)^T *= gamma
            {
                float v[32];
                tmem_ld32(tm + lrow + T_1 + tcol, v);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int t = tcol + i;
                    const float x = *(const float *)(sm + OFF_V + kmaj_off(t, j, 64));
                    v[i] = to_tf32(x - gam_s[t] * v[i]);
                }
                tmem_st32(tm + lrow + T_V + tcol, v);  // upper half-lanes: u~^T slot, not live yet
                float w[32];
                tmem_ld32(tm + lrow + T_1 + 64 + tcol, w);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) w[i] *= gam_s[tcol + i];
                tmem_st32(tm + lrow + T_1 + 64 + tcol, w);  // upper half-lanes: dS^T slot, dead
                tmem_wait_st();
            }
            fence_before_sync();
            group_sync(1);
            if (tid == 0) {
                if (c + 1 < nchunks) issue_v(c + 1);  // V of this chunk has been read
                fence_after_sync();
                gemm_ts<64, 64, false>(tm + T_U, tm + T_V, sb + OFF_TB + (c & 1) * 16384, 8192, false);
                mma_commit(&bar[B_2]);
            }
            // ---- epilogue 2: u^T rounded in place (operand of MMA_4); u~^T = u^T * kd (upper lanes)
            if (!wait_all(B_2, par)) { failed = true; break; }
            fence_after_sync();
            {
                float v[32];
                tmem_ld32(tm + lrow + T_U + tcol, v);
                tmem_wait_ld();
                float ut[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const float x = v[i];
                    v[i] = to_tf32(x);
                    // the upper thread of each pair takes the scaled copy of the lower thread's row
                    const float xs = __shfl_xor_sync(0xffffffffu, x, 16);
                    ut[i] = to_tf32(xs * kd_s[tcol + i]);
                }
                tmem_st32(tm + lrow + T_U + tcol, v);   // upper half-lanes unused
                tmem_st32(tm + lrow + T_V + tcol, ut);  // lower: V'^T (consumed); upper: u~^T
                tmem_wait_st();
            }
            fence_before_sync();
            if (!wait_all(B_KMN, par)) { failed = true; break; }
            if (tid == 0) {
                fence_after_sync();
                gemm_ts<128, 64, true>(tm + kUpper + T_1, tm + kUpper + T_V, sb + OFF_KMN, 64, false);
                gemm_ts<64, 64, false>(tm + T_1 + 64, tm + T_U, sb + OFF_P + (c & 1) * 16384, 8192, true);
                mma_commit(&bar[B_3]);
            }
            if (!wait_all(B_3, par)) { failed = true; break; }
            fence_after_sync();
            if (tid == 0 && c + 1 < nchunks) issue_kmn(c + 1);
            // ---- epilogue 3: S^T <- gamma_C S^T + dS^T (upper lanes fp32, lower lanes TF32); y^T out
            {
                const float gc = gam_s[n - 1];
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int d0 = 64 * ch + 32 * half;
                    float ds[32], s[32];
                    tmem_ld32(tm + lrow + T_1 + d0, ds);   // upper half-lanes hold dS^T
                    tmem_ld32(tm + lrow + T_S + d0, s);    // upper half-lanes hold S^T fp32
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const float sn = fmaf(gc, s[i], ds[i]);           // meaningful on upper lanes
                        const float from_upper = __shfl_xor_sync(0xffffffffu, sn, 16);
                        s[i] = upper ? sn : to_tf32(from_upper);
                    }
                    tmem_st32(tm + lrow + T_S + d0, s);
                }
                float y[32];
                tmem_ld32(tm + lrow + T_1 + 64 + tcol, y);
                tmem_wait_ld();
                tmem_wait_st();
                if (!upper) {
                    TO *o = (TO *)p.out + tok * v_row + h * kHeadDim + col0 + j;
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int t = tcol + i;
                        if (t < n) o[(int64_t)t * v_row] = from_f32<TO>(y[i]);
                    }
                }
            }
            fence_before_sync();
            group_sync(1);
        }
        // ---- final state (upper half-lanes) -> fin;  on failure poison this CTA's outputs
        if (p.fin) {
            float *dst = p.fin + ((int64_t)b * p.n_v + h) * kHeadDim * kHeadDim + col0 + j;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int d0 = 64 * ch + 32 * half;
                float s[32];
                tmem_ld32(tm + lrow + T_S + d0, s);
                tmem_wait_ld();
                if (upper) {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        dst[(int64_t)(d0 + i) * kHeadDim] = failed ? __int_as_float(0x7fc00000) : s[i];
                }
            }
        }
        if (failed) {
            for (int e = tid; e < L * kN; e += kGroup) {
                const int t = e / kN, jj = e % kN;
                ((TO *)p.out)[(seq0 + t) * v_row + h * kHeadDim + col0 + jj] =
                    from_f32<TO>(__int_as_float(0x7fc00000));
            }
        }
    } else {
        // ================================================================ prep group
        const int ptid = tid - kGroup;                 // 0..255
        const int ch = (warp - 8) >> 2;                // which 32 of the 64 columns of [K;Q]K^T
        const TI *al = (const TI *)p.alpha;
        const TI *be = (const TI *)p.beta;
        typedef typename RawT<TI>::type raw_t;
        raw_t a_raw = 0, b_raw = 0;
        auto load_gates = [&](int c) {                 // raw bits; converted one chunk later
            const int n = min(kChunk, L - c * kChunk);
            const int64_t tok = seq0 + (int64_t)c * kChunk;
            if (ptid < n) {
                a_raw = ld_raw(al + (tok + ptid) * p.n_v + h);
                b_raw = ld_raw(be + (tok + ptid) * p.n_v + h);
            }
        };
        auto wait_all = [&](int i, uint32_t par) -> bool {
            const bool ok = mbar_wait(&bar[i], par, kWaitTries);
            return !group_sync_or(2, !ok);
        };
        float *Ascr = (float *)(sm + OFF_AS);
        float *Tscr = (float *)(sm + OFF_TS);
        float *inv_s = (float *)(sm + OFF_INV);
        if (nchunks > 0 && ptid < kChunk) load_gates(0);

        for (int c = 0; c < nchunks; ++c) {
            const int n = min(kChunk, L - c * kChunk);
            const uint32_t par = c & 1;
            float *gate = (float *)(sm + OFF_GATE + (c & 1) * 1024);
            float *g_s = gate, *gam_s = gate + 64, *beta_s = gate + 128, *kd_s = gate + 192;
            unsigned char *Pt = sm + OFF_P + (c & 1) * 16384;
            unsigned char *Tb = sm + OFF_TB + (c & 1) * 16384;

            // ---- gates of chunk c.  [K;Q] of chunk c is issued only after the chain has
            // finished chunk c-1, so its arrival also frees this gate buffer, P and T_beta.
            if (!wait_all(B_KQ, par)) { failed = true; break; }
            if (ptid < kChunk) {
                g_s[ptid] = ptid < n ? safe_log_alpha(raw_to_f32(a_raw)) : 0.f;
                beta_s[ptid] = ptid < n ? raw_to_f32(b_raw) : 0.f;
                if (c + 1 < nchunks) load_gates(c + 1);
            }
            group_sync(2);
            if (ptid < 32) {  // inclusive scan of log alpha, two rows per lane
                const float a0 = g_s[2 * lane], a1 = g_s[2 * lane + 1];
                float s = a0 + a1;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, s, o);
                    if (lane >= o) s += y;
                }
                const float g0 = s - a1;
                const float glast = __shfl_sync(0xffffffffu, ((n - 1) & 1) ? s : g0, (n - 1) >> 1);
                g_s[2 * lane] = g0;
                g_s[2 * lane + 1] = s;
                gam_s[2 * lane] = expf(g0);
                gam_s[2 * lane + 1] = expf(s);
                kd_s[2 * lane] = 2 * lane < n ? expf(glast - g0) : 0.f;
                kd_s[2 * lane + 1] = 2 * lane + 1 < n ? expf(glast - s) : 0.f;
            }
            group_sync(2);
            if (ptid == 0) {
                fence_after_sync();
                gemm<128, 64, 128, false, false>(tm + T_A, sb + OFF_KQ, 16384, sb + OFF_KQ, 16384, false);
                mma_commit(&bar[B_A]);
            }
            // ---- epilogue a: A (fp32 scratch) and P (K-major tile)
            if (!wait_all(B_A, par)) { failed = true; break; }
            fence_after_sync();
            {
                float v[32];
                tmem_ld32(taddr(tm + T_A, 32 * quarter, 32 * ch), v);
                tmem_wait_ld();
                if (quarter < 2) {  // K K^T rows
                    const int t = 32 * quarter + lane;
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
                    const int t = 32 * quarter + lane - 64;
                    const float gt = g_s[t];
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
            group_sync(2);
            // ---- T = (I + A)^-1: 16 x 16 diagonal blocks, two 32 x 32 halves, one merge
            if (ptid < 64) {
                const int bb = ptid >> 4, cc = ptid & 15;
                float x[16];
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    float a0 = (r == cc) ? 1.f : 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
                    for (int m = 0; m + 3 < r; m += 4) {
                        const float4 a4 = *reinterpret_cast<const float4 *>(&Ascr[scr(16 * bb + r, 16 * bb + m)]);
                        a0 = fmaf(-a4.x, x[m], a0);
                        a1 = fmaf(-a4.y, x[m + 1], a1);
                        a2 = fmaf(-a4.z, x[m + 2], a2);
                        a3 = fmaf(-a4.w, x[m + 3], a3);
                    }
#pragma unroll
                    for (int m = r & ~3; m < r; ++m) a0 = fmaf(-Ascr[scr(16 * bb + r, 16 * bb + m)], x[m], a0);
                    x[r] = (r < cc) ? 0.f : (a0 + a1) + (a2 + a3);
                }
#pragma unroll
                for (int r = 0; r < 16; ++r) Tscr[scr(16 * bb + r, 16 * bb + cc)] = x[r];
            } else {
                for (int e = ptid - 64; e < 64 * 64; e += kGroup - 64) {
                    const int r = e >> 6, cc = e & 63;
                    if ((r >> 4) < (cc >> 4)) Tscr[scr(r, cc)] = 0.f;
                }
            }
            group_sync(2);
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
            group_sync(2);
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
            group_sync(2);
            {  // merge: M = A_bl T_top into the (zero) upper-right block
                const int r = ptid >> 3, c4 = (ptid & 7) * 4;
                float a4[4] = {0.f, 0.f, 0.f, 0.f};
                for (int m = c4; m < 32; ++m) {
                    const float a = Ascr[scr(32 + r, m)];
                    const float4 t4 = *reinterpret_cast<const float4 *>(&Tscr[scr(m, c4)]);
                    a4[0] = fmaf(a, t4.x, a4[0]); a4[1] = fmaf(a, t4.y, a4[1]);
                    a4[2] = fmaf(a, t4.z, a4[2]); a4[3] = fmaf(a, t4.w, a4[3]);
                }
                *reinterpret_cast<float4 *>(&Tscr[scr(r, 32 + c4)]) = make_float4(a4[0], a4[1], a4[2], a4[3]);
            }
            group_sync(2);
            {  // T_bl = -T_br M
                const int r = ptid >> 3, c4 = (ptid & 7) * 4;
                float a4[4] = {0.f, 0.f, 0.f, 0.f};
                for (int m = 0; m <= r; ++m) {
                    const float t = Tscr[scr(32 + r, 32 + m)];
                    const float4 m4 = *reinterpret_cast<const float4 *>(&Tscr[scr(m, 32 + c4)]);
                    a4[0] = fmaf(t, m4.x, a4[0]); a4[1] = fmaf(t, m4.y, a4[1]);
                    a4[2] = fmaf(t, m4.z, a4[2]); a4[3] = fmaf(t, m4.w, a4[3]);
                }
                *reinterpret_cast<float4 *>(&Tscr[scr(32 + r, c4)]) = make_float4(-a4[0], -a4[1], -a4[2], -a4[3]);
            }
            group_sync(2);
            {  // T_beta = T diag(beta) as a K-major tile (the upper-right block is zero)
                const int t = ptid >> 2, i0 = (ptid & 3) * 16;
                const bool upper_right = t < 32 && i0 >= 32;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    float4 x = *reinterpret_cast<const float4 *>(&Tscr[scr(t, i0 + 4 * k)]);
                    if (upper_right) x = make_float4(0.f, 0.f, 0.f, 0.f);
                    *reinterpret_cast<float4 *>(Tb + kmaj_off(t, i0 + 4 * k, 64)) =
                        tf32x4(x.x * beta_s[i0 + 4 * k], x.y * beta_s[i0 + 4 * k + 1],
                               x.z * beta_s[i0 + 4 * k + 2], x.w * beta_s[i0 + 4 * k + 3]);
                }
            }
            fence_smem_to_async();  // P and T_beta are read by the chain's MMAs
            group_sync(2);
            if (ptid == 0) {
                asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&bar[B_PREP])) : "memory");
            }
        }
    }

    // ---------------------------------------------------------------- tear-down
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
    const unsigned grid = (unsigned)((int64_t)p.n_seqs * p.n_v * kNS);
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
        !encode_rows(&p.tm_v, sp.vh, wv, T, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    p.alpha = sp.alpha; p.beta = sp.beta; p.cu = sp.cu; p.init = sp.init; p.fin = sp.fin;
    p.out = sp.out; p.n_seqs = sp.n_seqs; p.n_qk = sp.n_qk; p.n_v = sp.n_v;
    if (in_bf16) return out_bf16 ? launch_tc_t<gdn::bf16, gdn::bf16>(p, s) : launch_tc_t<gdn::bf16, float>(p, s);
    return out_bf16 ? launch_tc_t<float, gdn::bf16>(p, s) : launch_tc_t<float, float>(p, s);
}

}  // namespace gdn
