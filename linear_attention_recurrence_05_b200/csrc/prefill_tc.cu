// Chunked gated-delta-rule prefill on the sm_100a tensor cores (TF32 MMAs, fp32 state).
//
// The recurrence of the page "ARCHITECTURE PREVIEW / FIELD NOTES", section 03 (GATED
// DELTANET equations), in chunks of 64 tokens.  Within a chunk, with
// g_t = sum_{s<=t} log alpha_s, gamma_t = exp(g_t) and S the state entering the chunk:
//     A_ti = beta_t exp(g_t - g_i) k_t.k_i  (i < t),   T = (I + A)^-1
//     u    = T diag(beta) (V - diag(gamma) K S)                      (the WY/UT solve)
//     y_t  = gamma_t S^T q_t + sum_{i<=t} exp(g_t - g_i)(q_t.k_i) u_i
//     S   <- gamma_C S + sum_i exp(g_C - g_i) k_i u_i^T
// (u = U - W S with U = T diag(beta) V and W = T diag(beta gamma) K, regrouped so
// that W never has to be formed).
//
// One CTA owns one (sequence, V head, 64-column half of d_v) and walks the sequence's
// chunks in order; the column split is exact.  Per chunk, on the tensor core:
//     MMA_a  [K;Q] K^T        128 x 64 x 128   -> A (strict lower) and P (lower)
//     MMA_1  K S, Q S          64 x 64 x 128   -> V' = V - gamma*KS ; gamma*QS kept in TMEM
//     MMA_2  T_beta V'         64 x 64 x 64    -> u, u~ = exp(g_C - g) u
//     MMA_3  K^T u~           128 x 64 x 64    -> S update (state stays fp32 in registers)
//     MMA_4  P u (accumulate)  64 x 64 x 64    -> y = gamma*QS + P u
// and on the CUDA cores the 64 x 64 unit-lower-triangular inverse (16 x 16 blocks).
// The next chunk's K/Q, V and K (token-major copy) are fetched with cp.async into
// each buffer as soon as its last reader has finished.
#include "gdn_common.cuh"
#include "gdn_internal.h"
#include "tc_sm100.cuh"

namespace gdn {

namespace {
using namespace tc;

constexpr int kN = 64;          // d_v columns per CTA
constexpr int kNS = kHeadDim / kN;
constexpr int kThr = 256;

// shared-memory map (bytes from a 1024-aligned base)
constexpr uint32_t OFF_S = 0;          // S        MN-major  [128 d][64 j]            32 KB
constexpr uint32_t OFF_KQ = 32768;     // [K;Q]    K-major   [128 rows][128 d]        64 KB
constexpr uint32_t OFF_KMN = 98304;    // K        MN-major  [64 i][128 d]            32 KB
constexpr uint32_t OFF_V = 131072;     // V plain [64][64] fp32, then V' MN-major      16 KB
constexpr uint32_t OFF_TB = 147456;    // T plain, then T_beta K-major, then u~ MN-major 16 KB
constexpr uint32_t OFF_P = 163840;     // P        K-major   [64 t][64 i]             16 KB
constexpr uint32_t OFF_U = 180224;     // A plain [64][64] fp32, then u MN-major      16 KB
constexpr uint32_t OFF_MISC = 196608;  // gates, inverse scratch, barriers
constexpr uint32_t OFF_G = OFF_MISC;            // g[64]
constexpr uint32_t OFF_GAM = OFF_MISC + 256;    // gamma[64]
constexpr uint32_t OFF_BETA = OFF_MISC + 512;   // beta[64]
constexpr uint32_t OFF_KD = OFF_MISC + 768;     // exp(g_last - g)[64]
constexpr uint32_t OFF_INV = OFF_MISC + 1024;   // 3 x 256 floats (block products)
constexpr uint32_t OFF_BAR = OFF_MISC + 4096;   // 5 mbarriers
constexpr uint32_t OFF_TSLOT = OFF_BAR + 64;  // after 5 x 8 bytes
constexpr uint32_t kSmem = OFF_MISC + 4096 + 128;
constexpr uint32_t kSmemAlloc = kSmem + 1024;   // slack to align the base to 1024

// tensor-memory columns
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t T_A = 0;      // [K;Q]K^T  M=128
constexpr uint32_t T_KS = 64;    // K S       M=64
constexpr uint32_t T_QS = 128;   // Q S, then y  M=64
constexpr uint32_t T_U = 192;    // u         M=64
constexpr uint32_t T_DS = 256;   // K^T u~    M=128

constexpr uint32_t kWaitTries = 1u << 22;

__device__ __forceinline__ void cp_async16_zfill(uint32_t dst, const void *src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
                 "r"(valid ? 16 : 0)
                 : "memory");
}

template <class TO>
__device__ __forceinline__ void store_out(TO *p, float v) { *p = from_f32<TO>(v); }

}  // namespace

struct TcParams {
    const float *qh, *kh, *vh;
    const void *alpha, *beta;
    const int32_t *cu;
    const float *init;
    float *fin;
    void *out;
    int n_seqs, n_qk, n_v;
};

template <class TI, class TO>
__global__ void __launch_bounds__(kThr, 1) prefill_tc_kernel(TcParams p) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    const uint32_t sb = smem_u32(sm);
    float *g_s = (float *)(sm + OFF_G);
    float *gam_s = (float *)(sm + OFF_GAM);
    float *beta_s = (float *)(sm + OFF_BETA);
    float *kd_s = (float *)(sm + OFF_KD);
    float *inv_s = (float *)(sm + OFF_INV);
    // one phase per chunk each: 0 MMA_a, 1 K S, 2 Q S, 3 MMA_2, 4 MMA_3 + MMA_4
    uint64_t *bar = (uint64_t *)(sm + OFF_BAR);
    uint32_t *tslot = (uint32_t *)(sm + OFF_TSLOT);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int quarter = warp & 3, half = warp >> 2;   // TMEM lane quarter, 32-column half
    const int slice = blockIdx.x % kNS;
    const int h = (blockIdx.x / kNS) % p.n_v;
    const int b = blockIdx.x / (kNS * p.n_v);
    const int gq = h / (p.n_v / p.n_qk);
    const int seq0 = p.cu[b], L = p.cu[b + 1] - p.cu[b];
    const int col0 = slice * kN;
    const int64_t qk_row = (int64_t)p.n_qk * kHeadDim, v_row = (int64_t)p.n_v * kHeadDim;
    const TI *al = (const TI *)p.alpha;
    const TI *be = (const TI *)p.beta;
    TO *out = (TO *)p.out;
    const int nchunks = (L + kChunk - 1) / kChunk;

    // ---------------------------------------------------------------- set-up
    if (tid == 0) {
        for (int i = 0; i < 5; ++i) mbar_init(&bar[i], 1);
    }
    if (warp == 0) {
        tmem_alloc(tslot, kTmemCols);
        tmem_relinquish();
    }
    // state: this thread owns S[d][32*half .. 32*half+31] with d = 32*quarter + lane
    const int d_own = 32 * quarter + lane;
    float S[32];
    {
        const int64_t st_off = (((int64_t)b * p.n_v + h) * kHeadDim + d_own) * kHeadDim + col0 + 32 * half;
#pragma unroll
        for (int j = 0; j < 32; ++j) S[j] = p.init ? p.init[st_off + j] : 0.f;
#pragma unroll
        for (int j = 0; j < 32; ++j)
            *(float *)(sm + OFF_S + mn_off(d_own, 32 * half + j, kHeadDim)) = to_tf32(S[j]);
    }

    // chunk loaders ----------------------------------------------------------
    auto load_kq = [&](int c) {  // [K;Q] rows, K-major core-matrix layout (group 1)
        const int n = min(kChunk, L - c * kChunk);
        const int64_t tok = seq0 + (int64_t)c * kChunk;
        for (int e = tid; e < 128 * 32; e += kThr) {
            const int r = e >> 5, q4 = (e & 31) * 4;
            const int t = r & 63;
            const float *src = (r < 64 ? p.kh : p.qh) + (tok + (t < n ? t : 0)) * qk_row +
                               gq * kHeadDim + q4;
            cp_async16_zfill(sb + OFF_KQ + cm_off(r, q4, 128), src, t < n);
        }
    };
    auto load_v = [&](int c) {  // V rows, plain [64][64] (group 2)
        const int n = min(kChunk, L - c * kChunk);
        const int64_t tok = seq0 + (int64_t)c * kChunk;
        for (int e = tid; e < 64 * 16; e += kThr) {
            const int t = e >> 4, q4 = (e & 15) * 4;
            const float *src = p.vh + (tok + (t < n ? t : 0)) * v_row + h * kHeadDim + col0 + q4;
            cp_async16_zfill(sb + OFF_V + (t * 64 + q4) * 4, src, t < n);
        }
    };
    auto load_kmn = [&](int c) {  // K rows, MN-major swizzled layout (group 3)
        const int n = min(kChunk, L - c * kChunk);
        const int64_t tok = seq0 + (int64_t)c * kChunk;
        for (int e = tid; e < 64 * 32; e += kThr) {
            const int t = e >> 5, q4 = (e & 31) * 4;
            const float *src = p.kh + (tok + (t < n ? t : 0)) * qk_row + gq * kHeadDim + q4;
            cp_async16_zfill(sb + OFF_KMN + mn_off(t, q4, 64), src, t < n);
        }
    };
    // gate prefetch: thread t < 64 holds alpha/beta of row t of the next chunk
    float a_next = 1.f, b_next = 0.f;
    auto load_gates = [&](int c) {
        const int n = min(kChunk, L - c * kChunk);
        const int64_t tok = seq0 + (int64_t)c * kChunk;
        if (tid < kChunk) {
            a_next = tid < n ? to_f32(al[(tok + tid) * p.n_v + h]) : 1.f;
            b_next = tid < n ? to_f32(be[(tok + tid) * p.n_v + h]) : 0.f;
        }
    };

    if (nchunks > 0) {
        load_kq(0);
        cp_async_commit();
        load_v(0);
        cp_async_commit();
        load_kmn(0);
        cp_async_commit();
        load_gates(0);
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tm = *tslot;
    bool failed = false;

    // waits for barrier `i` phase `par` on every thread; all threads agree on failure
    auto wait_bar = [&](int i, uint32_t par) -> bool {
        bool ok = mbar_wait(&bar[i], par, kWaitTries);
        return __syncthreads_or(!ok) == 0;
    };

    for (int c = 0; c < nchunks && !failed; ++c) {
        const int n = min(kChunk, L - c * kChunk);
        const int64_t tok = seq0 + (int64_t)c * kChunk;
        const uint32_t par = c & 1;

        // ---- gates of this chunk, K/Q tile
        if (tid < kChunk) {
            g_s[tid] = safe_log_alpha(a_next);
            beta_s[tid] = b_next;
        }
        cp_async_wait<2>();  // group 1 of this chunk ([K;Q]) has landed
        fence_smem_to_async();
        __syncthreads();
        if (warp == 0) {  // inclusive scan of log alpha, two rows per lane
            float a0 = g_s[2 * lane], a1 = g_s[2 * lane + 1];
            float s = a0 + a1;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                float y = __shfl_up_sync(0xffffffffu, s, o);
                if (lane >= o) s += y;
            }
            const float base = s - (a0 + a1);
            g_s[2 * lane] = base + a0;
            g_s[2 * lane + 1] = s;
            __syncwarp();
            const float glast = __shfl_sync(0xffffffffu, (n - 1) & 1 ? s : base + a0, (n - 1) >> 1);
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int t = 2 * lane + k;
                const float gt = k ? s : base + a0;
                gam_s[t] = expf(gt);
                kd_s[t] = t < n ? expf(glast - gt) : 0.f;
            }
        }
        __syncthreads();

        // ---- MMA_a: [K;Q] K^T ; MMA_1: K S, Q S
        if (tid == 0) {
            fence_after_sync();
            gemm<128, 64, 128, false, false>(tm + T_A, sb + OFF_KQ, 128, sb + OFF_KQ, 128, false);
            mma_commit(&bar[0]);
            gemm<64, 64, 128, false, true>(tm + T_KS, sb + OFF_KQ, 128, sb + OFF_S, kHeadDim, false);
            mma_commit(&bar[1]);
            gemm<64, 64, 128, false, true>(tm + T_QS, sb + OFF_KQ + 64 * 128 * 4, 128, sb + OFF_S,
                                           kHeadDim, false);
            mma_commit(&bar[2]);
        }

        // ---- epilogue a: A (fp32 scratch in OFF_U) and P (K-major tile)
        if (!wait_bar(0, par)) { failed = true; break; }
        fence_after_sync();
        {
            float v[32];
            tmem_ld32(taddr(tm + T_A, 32 * quarter, 32 * half), v);
            tmem_wait_ld();
            const int row = 32 * quarter + lane;
            if (row < 64) {  // K K^T rows -> A
                const int t = row;
                float *A = (float *)(sm + OFF_U);
                const float gt = g_s[t], bt = beta_s[t];
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int i = 32 * half + j;
                    A[t * 64 + i] = (i < t && t < n) ? bt * expf(gt - g_s[i]) * v[j] : 0.f;
                }
            } else {  // Q K^T rows -> P
                const int t = row - 64;
                const float gt = g_s[t];
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int i = 32 * half + j;
                    const float pv = (i <= t && t < n) ? expf(gt - g_s[i]) * v[j] : 0.f;
                    *(float *)(sm + OFF_P + cm_off(t, i, 64)) = to_tf32(pv);
                }
            }
        }
        // ---- epilogue 1: V' = V - gamma * K S  (M=64 layout: row t at lane 16*quarter + l)
        cp_async_wait<1>();  // group 2 (V) of this chunk; made visible by the barrier below
        if (!wait_bar(1, par)) { failed = true; break; }
        fence_after_sync();
        {
            float v[32];
            tmem_ld32(taddr(tm + T_KS, 32 * quarter, 32 * half), v);
            tmem_wait_ld();
            const int t = 16 * quarter + lane;
            float vp[32];
            if (lane < 16) {
                const float gt = gam_s[t];
                const float *V = (const float *)(sm + OFF_V);
#pragma unroll
                for (int j = 0; j < 32; ++j) vp[j] = V[t * 64 + 32 * half + j] - gt * v[j];
            }
            __syncthreads();  // every V value has been read before V' overwrites it
            if (lane < 16) {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    *(float *)(sm + OFF_V + mn_off(t, 32 * half + j, 64)) = to_tf32(vp[j]);
            }
        }
        __syncthreads();  // A complete

        // ---- T = (I + A)^-1 by 16 x 16 blocks (plain fp32 in OFF_TB)
        {
            const float *A = (const float *)(sm + OFF_U);
            float *T = (float *)(sm + OFF_TB);
            if (tid < 64) {  // diagonal blocks: column c of block bb by forward substitution
                const int bb = tid >> 4, cc = tid & 15;
                float x[16];
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    float acc = (r == cc) ? 1.f : 0.f;
#pragma unroll
                    for (int m = 0; m < r; ++m)
                        acc = fmaf(-A[(16 * bb + r) * 64 + 16 * bb + m], x[m], acc);
                    x[r] = (r < cc) ? 0.f : acc;
                }
#pragma unroll
                for (int r = 0; r < 16; ++r) T[(16 * bb + r) * 64 + 16 * bb + cc] = x[r];
            } else {  // zero the strictly upper blocks
                for (int e = tid - 64; e < 64 * 64; e += kThr - 64) {
                    const int r = e >> 6, cidx = e & 63;
                    if ((r >> 4) < (cidx >> 4)) T[e] = 0.f;
                }
            }
            __syncthreads();
            // off-diagonal blocks by distance: T_rc = -T_rr * sum_{k=c}^{r-1} A_rk T_kc
            for (int dist = 1; dist < 4; ++dist) {
                const int nb = 4 - dist;  // blocks at this distance: c = 0..nb-1, r = c + dist
                for (int e = tid; e < nb * 256; e += kThr) {
                    const int c = e >> 8, rr = (e >> 4) & 15, cc = e & 15;
                    const int r = c + dist;
                    float acc = 0.f;
                    for (int k = c; k < r; ++k) {
#pragma unroll
                        for (int m = 0; m < 16; ++m)
                            acc = fmaf(A[(16 * r + rr) * 64 + 16 * k + m], T[(16 * k + m) * 64 + 16 * c + cc], acc);
                    }
                    inv_s[e] = acc;
                }
                __syncthreads();
                for (int e = tid; e < nb * 256; e += kThr) {
                    const int c = e >> 8, rr = (e >> 4) & 15, cc = e & 15;
                    const int r = c + dist;
                    float acc = 0.f;
#pragma unroll
                    for (int m = 0; m < 16; ++m)
                        acc = fmaf(T[(16 * r + rr) * 64 + 16 * r + m], inv_s[(c << 8) + m * 16 + cc], acc);
                    T[(16 * r + rr) * 64 + 16 * c + cc] = -acc;
                }
                __syncthreads();
            }
            // T_beta = T diag(beta), rewritten in place as a K-major tile
            float tv[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const int e = tid + kThr * k;
                tv[k] = T[e] * beta_s[e & 63];
            }
            __syncthreads();
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const int e = tid + kThr * k;
                *(float *)(sm + OFF_TB + cm_off(e >> 6, e & 63, 64)) = to_tf32(tv[k]);
            }
        }
        // ---- gamma * Q S, scaled in place in TMEM
        if (!wait_bar(2, par)) { failed = true; break; }
        fence_after_sync();
        {
            float v[32];
            tmem_ld32(taddr(tm + T_QS, 32 * quarter, 32 * half), v);
            tmem_wait_ld();
            const float gt = gam_s[(16 * quarter + lane) & 63];
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] *= gt;
            tmem_st32(taddr(tm + T_QS, 32 * quarter, 32 * half), v);
            tmem_wait_st();
        }
        fence_smem_to_async();
        fence_before_sync();
        __syncthreads();
        // [K;Q] is free: fetch the next chunk's
        if (c + 1 < nchunks) {
            load_kq(c + 1);
            load_gates(c + 1);
        }
        cp_async_commit();

        // ---- MMA_2: u = T_beta V'
        if (tid == 0) {
            fence_after_sync();
            gemm<64, 64, 64, false, true>(tm + T_U, sb + OFF_TB, 64, sb + OFF_V, 64, false);
            mma_commit(&bar[3]);
        }
        if (!wait_bar(3, par)) { failed = true; break; }
        fence_after_sync();
        // V and T_beta are free: next chunk's V
        if (c + 1 < nchunks) load_v(c + 1);
        cp_async_commit();
        {
            float v[32];
            tmem_ld32(taddr(tm + T_U, 32 * quarter, 32 * half), v);
            tmem_wait_ld();
            if (lane < 16) {
                const int t = 16 * quarter + lane;
                const float kd = kd_s[t];
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int jj = 32 * half + j;
                    *(float *)(sm + OFF_U + mn_off(t, jj, 64)) = to_tf32(v[j]);
                    *(float *)(sm + OFF_TB + mn_off(t, jj, 64)) = to_tf32(kd * v[j]);
                }
            }
        }
        cp_async_wait<2>();  // group 3 (K, token-major copy) of this chunk
        fence_smem_to_async();
        fence_before_sync();
        __syncthreads();

        // ---- MMA_3: dS = K^T u~ ; MMA_4: y = gamma QS + P u
        if (tid == 0) {
            fence_after_sync();
            gemm<128, 64, 64, true, true>(tm + T_DS, sb + OFF_KMN, 64, sb + OFF_TB, 64, false);
            gemm<64, 64, 64, false, true>(tm + T_QS, sb + OFF_P, 64, sb + OFF_U, 64, true);
            mma_commit(&bar[4]);
        }
        if (!wait_bar(4, par)) { failed = true; break; }
        fence_after_sync();
        if (c + 1 < nchunks) load_kmn(c + 1);
        cp_async_commit();
        {
            // state: S <- gamma_C S + dS (fp32 in registers), tf32 copy for the next MMAs
            float v[32];
            tmem_ld32(taddr(tm + T_DS, 32 * quarter, 32 * half), v);
            tmem_wait_ld();
            const float gc = gam_s[n - 1];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                S[j] = fmaf(gc, S[j], v[j]);
                *(float *)(sm + OFF_S + mn_off(d_own, 32 * half + j, kHeadDim)) = to_tf32(S[j]);
            }
            // outputs of this chunk
            float y[32];
            tmem_ld32(taddr(tm + T_QS, 32 * quarter, 32 * half), y);
            tmem_wait_ld();
            const int t = 16 * quarter + lane;
            if (lane < 16 && t < n) {
                TO *o = out + (tok + t) * v_row + h * kHeadDim + col0 + 32 * half;
#pragma unroll
                for (int j = 0; j < 32; ++j) store_out(o + j, y[j]);
            }
        }
        fence_smem_to_async();
        fence_before_sync();
        __syncthreads();
    }

    // ---------------------------------------------------------------- tear-down
    cp_async_wait<0>();
    const int64_t st_off = (((int64_t)b * p.n_v + h) * kHeadDim + d_own) * kHeadDim + col0 + 32 * half;
    if (p.fin) {
#pragma unroll
        for (int j = 0; j < 32; ++j) p.fin[st_off + j] = failed ? __int_as_float(0x7fc00000) : S[j];
    }
    if (failed) {  // a tensor-core wait gave up: poison this CTA's outputs
        for (int e = tid; e < L * kN; e += kThr) {
            const int t = e / kN, j = e % kN;
            store_out(out + (seq0 + t) * v_row + h * kHeadDim + col0 + j, __int_as_float(0x7fc00000));
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tm, kTmemCols);
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

cudaError_t launch_prefill_tc(const ScanParams &sp, bool in_bf16, bool out_bf16, cudaStream_t s) {
    if (sp.n_seqs <= 0) return cudaSuccess;
    TcParams p{sp.qh, sp.kh, sp.vh, sp.alpha, sp.beta, sp.cu, sp.init, sp.fin, sp.out,
               sp.n_seqs, sp.n_qk, sp.n_v};
    if (in_bf16) return out_bf16 ? launch_tc_t<gdn::bf16, gdn::bf16>(p, s) : launch_tc_t<gdn::bf16, float>(p, s);
    return out_bf16 ? launch_tc_t<float, gdn::bf16>(p, s) : launch_tc_t<float, float>(p, s);
}

}  // namespace gdn
