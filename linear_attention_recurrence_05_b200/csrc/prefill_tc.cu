// Chunked gated-delta-rule prefill on the sm_100a tensor cores (TF32 MMAs, fp32 state).
//
// The recurrence of the page "ARCHITECTURE PREVIEW / FIELD NOTES", section 03 (GATED
// DELTANET equations), in chunks of 64 tokens.  Within a chunk, with
// g_t = sum_{s<=t} log alpha_s, gamma_t = exp(g_t) and S the state entering the chunk:
//     A_ti = beta_t exp(g_t - g_i) k_t.k_i  (i < t),   T = (I + A)^-1
//     u    = T diag(beta) (V - diag(gamma) K S)                      (the WY/UT solve)
//     y_t  = gamma_t S^T q_t + sum_{i<=t} exp(g_t - g_i)(q_t.k_i) u_i
//     S   <- gamma_C S + sum_i exp(g_C - g_i) k_i u_i^T
// (u = U - W S with U = T diag(beta) V and W = T diag(beta gamma) K, regrouped so that
// W never has to be formed).
//
// One CTA (16 warps) owns one (sequence, V head, 64-column half of d_v) and walks the
// sequence's chunks in order; the column split is exact.  Per chunk, on the tensor core:
//     MMA_a  [K;Q] K^T      M=128 N=64 K=128 -> A (strict lower) and P (lower)
//     MMA_1  [K;Q] S        M=128 N=64 K=128 -> V' = V - gamma*KS ; gamma*QS kept in TMEM
//     MMA_2  T_beta V'      M=64  N=64 K=64  -> u, u~ = exp(g_C - g) u
//     MMA_3  K^T u~         M=128 N=64 K=64  -> S update (the state stays fp32 in registers)
//     MMA_4  [*;P] u        M=128 N=64 K=64  -> accumulated onto gamma*QS: y
// MMA_4 reads P through a 128-row view whose upper 64 rows are whatever precedes P in
// shared memory; they land on rows 0-63 of the accumulator, which hold K S and are
// already consumed.  On the CUDA cores: the 64 x 64 unit-lower-triangular inverse
// (16 x 16 blocks) and the element-wise epilogues.  Operand tiles arrive by TMA
// (2-D boxes of 32 fp32 x 64 tokens), each reloaded as soon as its last reader is done.
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

// shared-memory map (bytes from a 1024-aligned base)
constexpr uint32_t OFF_S = 0;          // S       MN-major R=128 (d) x 64 (j)               32 KB
constexpr uint32_t OFF_KQ = 32768;     // [K;Q]   K-major, 4 blocks x (K 8 KB | Q 8 KB)      64 KB
constexpr uint32_t OFF_KMN = 98304;    // K       MN-major R=64 (i) x 128 (d)               32 KB
constexpr uint32_t OFF_V = 131072;     // V (K-major swizzle, read by threads), then V' MN  16 KB
constexpr uint32_t OFF_TB = 147456;    // T (fp32 scratch), then T_beta K-major, then u~ MN 16 KB
constexpr uint32_t OFF_P = 163840;     // P       K-major R=64                               16 KB
constexpr uint32_t OFF_U = 180224;     // A (fp32 scratch), then u MN-major                16 KB
constexpr uint32_t OFF_MISC = 196608;
constexpr uint32_t OFF_G = OFF_MISC;            // g[64]
constexpr uint32_t OFF_GAM = OFF_MISC + 256;    // gamma[64]
constexpr uint32_t OFF_BETA = OFF_MISC + 512;   // beta[64]
constexpr uint32_t OFF_KD = OFF_MISC + 768;     // exp(g_last - g)[64]
constexpr uint32_t OFF_INV = OFF_MISC + 1024;   // 3 x 256 floats (block products)
constexpr uint32_t OFF_BAR = OFF_MISC + 4096;   // mbarriers
constexpr uint32_t OFF_TSLOT = OFF_BAR + 128;
constexpr uint32_t kSmem = OFF_TSLOT + 16;
constexpr uint32_t kSmemAlloc = kSmem + 1024;   // slack to align the base to 1024

enum { B_KQ = 0, B_V, B_KMN, B_A, B_1, B_2, B_3, kNumBars };

// tensor-memory columns
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t T_A = 0;      // [K;Q]K^T    M=128
constexpr uint32_t T_1 = 64;     // [K;Q]S, then rows 64.. = y   M=128
constexpr uint32_t T_U = 128;    // u           M=64
constexpr uint32_t T_DS = 192;   // K^T u~      M=128

constexpr uint32_t kWaitTries = 1u << 22;

// fp32 scratch [64][64] with 16-byte chunks XOR-swizzled by row (conflict-free rows and columns)
__device__ __forceinline__ int scr(int r, int c) { return r * 64 + ((((c >> 2) ^ (r & 7)) << 2) | (c & 3)); }

__device__ __forceinline__ float4 tf32x4(float a, float b, float c, float d) {
    return make_float4(to_tf32(a), to_tf32(b), to_tf32(c), to_tf32(d));
}

template <class TO>
__device__ __forceinline__ void store_row16(TO *dst, const float (&v)[16]);
template <>
__device__ __forceinline__ void store_row16<float>(float *dst, const float (&v)[16]) {
#pragma unroll
    for (int k = 0; k < 4; ++k)
        *reinterpret_cast<float4 *>(dst + 4 * k) = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
}
template <>
__device__ __forceinline__ void store_row16<bf16>(bf16 *dst, const float (&v)[16]) {
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        uint4 w;
        __nv_bfloat162 h0 = __floats2bfloat162_rn(v[8 * k], v[8 * k + 1]);
        __nv_bfloat162 h1 = __floats2bfloat162_rn(v[8 * k + 2], v[8 * k + 3]);
        __nv_bfloat162 h2 = __floats2bfloat162_rn(v[8 * k + 4], v[8 * k + 5]);
        __nv_bfloat162 h3 = __floats2bfloat162_rn(v[8 * k + 6], v[8 * k + 7]);
        w.x = *reinterpret_cast<uint32_t *>(&h0);
        w.y = *reinterpret_cast<uint32_t *>(&h1);
        w.z = *reinterpret_cast<uint32_t *>(&h2);
        w.w = *reinterpret_cast<uint32_t *>(&h3);
        *reinterpret_cast<uint4 *>(dst + 8 * k) = w;
    }
}

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
    float *g_s = (float *)(sm + OFF_G);
    float *gam_s = (float *)(sm + OFF_GAM);
    float *beta_s = (float *)(sm + OFF_BETA);
    float *kd_s = (float *)(sm + OFF_KD);
    float *inv_s = (float *)(sm + OFF_INV);
    uint64_t *bar = (uint64_t *)(sm + OFF_BAR);
    uint32_t *tslot = (uint32_t *)(sm + OFF_TSLOT);
    float *Ascr = (float *)(sm + OFF_U);   // A scratch (fp32, swizzled rows)
    float *Tscr = (float *)(sm + OFF_TB);  // T scratch (fp32, swizzled rows)

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int quarter = warp & 3, cg = warp >> 2;   // TMEM lane quarter, 16-column group
    const int col = 16 * cg;                        // first accumulator column of this thread
    const int slice = blockIdx.x % kNS;
    const int h = (blockIdx.x / kNS) % p.n_v;
    const int b = blockIdx.x / (kNS * p.n_v);
    const int gq = h / (p.n_v / p.n_qk);
    const int seq0 = p.cu[b], L = p.cu[b + 1] - p.cu[b];
    const int col0 = slice * kN;
    const int64_t v_row = (int64_t)p.n_v * kHeadDim;
    const TI *al = (const TI *)p.alpha;
    const TI *be = (const TI *)p.beta;
    TO *out = (TO *)p.out;
    const int nchunks = (L + kChunk - 1) / kChunk;

    // ---------------------------------------------------------------- set-up
    if (tid == 0) {
        for (int i = 0; i < kNumBars; ++i) mbar_init(&bar[i], 1);
    }
    if (warp == 0) {
        tmem_alloc(tslot, kTmemCols);
        tmem_relinquish();
    }
    // this thread owns S[d_own][col .. col+15]
    const int d_own = 32 * quarter + lane;
    const int64_t st_off = (((int64_t)b * p.n_v + h) * kHeadDim + d_own) * kHeadDim + col0 + col;
    float S[16];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        float4 v4 = p.init ? *reinterpret_cast<const float4 *>(p.init + st_off + 4 * k)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
        S[4 * k] = v4.x; S[4 * k + 1] = v4.y; S[4 * k + 2] = v4.z; S[4 * k + 3] = v4.w;
    }
#pragma unroll
    for (int k = 0; k < 4; ++k)
        *reinterpret_cast<float4 *>(sm + OFF_S + mn_off(d_own, col + 4 * k, kHeadDim)) =
            tf32x4(S[4 * k], S[4 * k + 1], S[4 * k + 2], S[4 * k + 3]);

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

    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tm = *tslot;
    if (nchunks > 0) {
        if (tid == 0) {
            issue_kq(0);
            issue_v(0);
            issue_kmn(0);
        }
        load_gates(0);
    }
    bool failed = false;
    // every thread waits; all agree on success
    auto wait_bar = [&](int i, uint32_t par) -> bool {
        bool ok = mbar_wait(&bar[i], par, kWaitTries);
        return __syncthreads_or(!ok) == 0;
    };

    for (int c = 0; c < nchunks; ++c) {
        const int n = min(kChunk, L - c * kChunk);
        const int64_t tok = seq0 + (int64_t)c * kChunk;
        const uint32_t par = c & 1;

        // ---- gates, and this chunk's [K;Q]
        if (tid < kChunk) {
            g_s[tid] = safe_log_alpha(a_next);
            beta_s[tid] = b_next;
        }
        if (c + 1 < nchunks) load_gates(c + 1);  // a whole chunk ahead of their use
        fence_smem_to_async();  // S tile written by the previous chunk (or the set-up)
        if (!wait_bar(B_KQ, par)) { failed = true; break; }
        if (warp == 0) {  // inclusive scan of log alpha, two rows per lane
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
        __syncthreads();

        // ---- MMA_a: [K;Q] K^T ; MMA_1: [K;Q] S
        if (tid == 0) {
            fence_after_sync();
            gemm<128, 64, 128, false, false>(tm + T_A, sb + OFF_KQ, 16384, sb + OFF_KQ, 16384, false);
            mma_commit(&bar[B_A]);
            gemm<128, 64, 128, false, true>(tm + T_1, sb + OFF_KQ, 16384, sb + OFF_S, kHeadDim, false);
            mma_commit(&bar[B_1]);
        }

        // ---- epilogue a: A (fp32 scratch) and P (K-major tile)
        if (!wait_bar(B_A, par)) { failed = true; break; }
        fence_after_sync();
        {
            float v[16];
            tmem_ld16(taddr(tm + T_A, 32 * quarter, col), v);
            tmem_wait_ld();
            if (quarter < 2) {  // K K^T rows -> A = strict lower beta_t exp(g_t - g_i) k_t.k_i
                const int t = 32 * quarter + lane;
                const float gt = g_s[t], bt = beta_s[t];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    float a4[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int i = col + 4 * k + e;
                        a4[e] = (i < t && t < n) ? bt * expf(gt - g_s[i]) * v[4 * k + e] : 0.f;
                    }
                    *reinterpret_cast<float4 *>(&Ascr[scr(t, col + 4 * k)]) = make_float4(a4[0], a4[1], a4[2], a4[3]);
                }
            } else {  // Q K^T rows -> P = lower exp(g_t - g_i) q_t.k_i
                const int t = 32 * quarter + lane - 64;
                const float gt = g_s[t];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    float p4[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int i = col + 4 * k + e;
                        p4[e] = (i <= t && t < n) ? expf(gt - g_s[i]) * v[4 * k + e] : 0.f;
                    }
                    *reinterpret_cast<float4 *>(sm + OFF_P + kmaj_off(t, col + 4 * k, 64)) =
                        tf32x4(p4[0], p4[1], p4[2], p4[3]);
                }
            }
        }
        // ---- epilogue 1: V' = V - gamma * K S (rows 0-63); gamma * Q S in place (rows 64-127)
        if (!wait_bar(B_1, par)) { failed = true; break; }
        if (tid == 0 && c + 1 < nchunks) issue_kq(c + 1);  // MMA_a and MMA_1 are done with [K;Q]
        if (!wait_bar(B_V, par)) { failed = true; break; }
        fence_after_sync();
        {
            float v[16];
            tmem_ld16(taddr(tm + T_1, 32 * quarter, col), v);
            tmem_wait_ld();
            if (quarter < 2) {
                const int t = 32 * quarter + lane;
                const float gt = gam_s[t];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float4 x = *reinterpret_cast<const float4 *>(sm + OFF_V + kmaj_off(t, col + 4 * k, 64));
                    v[4 * k] = x.x - gt * v[4 * k];
                    v[4 * k + 1] = x.y - gt * v[4 * k + 1];
                    v[4 * k + 2] = x.z - gt * v[4 * k + 2];
                    v[4 * k + 3] = x.w - gt * v[4 * k + 3];
                }
            } else {
                const float gt = gam_s[32 * quarter + lane - 64];
#pragma unroll
                for (int j = 0; j < 16; ++j) v[j] *= gt;
                tmem_st16(taddr(tm + T_1, 32 * quarter, col), v);
                tmem_wait_st();
            }
            __syncthreads();  // all of V has been read before V' overwrites it
            if (quarter < 2) {
                const int t = 32 * quarter + lane;
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    *reinterpret_cast<float4 *>(sm + OFF_V + mn_off(t, col + 4 * k, 64)) =
                        tf32x4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
            }
        }

        // ---- T = (I + A)^-1 (fp32 scratch in OFF_TB): 16 x 16 diagonal blocks by forward
        // substitution, then the two 32 x 32 halves, then the lower-left 32 x 32 block:
        //   [[X, 0], [Y, Z]]^-1 = [[X^-1, 0], [-Z^-1 Y X^-1, Z^-1]]
        if (tid < 64) {  // diagonal blocks: column cc of block bb
            const int bb = tid >> 4, cc = tid & 15;
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
        } else {  // zero the strictly upper part outside the diagonal blocks
            for (int e = tid - 64; e < 64 * 64; e += kThr - 64) {
                const int r = e >> 6, cc = e & 63;
                if ((r >> 4) < (cc >> 4)) Tscr[scr(r, cc)] = 0.f;
            }
        }
        __syncthreads();
        // 32 x 32 halves hh = 0, 1 (rows/cols 32hh..32hh+31): T_10 = -T_11 A_10 T_00 in
        // 16-blocks; then the lower-left 32 x 32 block T_bl = -T_br A_bl T_top.  Each
        // thread computes a 4-column strip of one row (float4 operand loads).
        if (tid < 128) {
            const int hh = tid >> 6, rr = (tid >> 2) & 15, c4 = (tid & 3) * 4, o = 32 * hh;
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
        __syncthreads();
        if (tid < 128) {
            const int hh = tid >> 6, rr = (tid >> 2) & 15, c4 = (tid & 3) * 4, o = 32 * hh;
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
        __syncthreads();
        // M = A_bl T_top, kept in the (zero) upper-right block of T
        if (tid < 256) {
            const int r = tid >> 3, c4 = (tid & 7) * 4;
            float a4[4] = {0.f, 0.f, 0.f, 0.f};
            for (int m = c4; m < 32; ++m) {  // T_top is lower triangular
                const float a = Ascr[scr(32 + r, m)];
                const float4 t4 = *reinterpret_cast<const float4 *>(&Tscr[scr(m, c4)]);
                a4[0] = fmaf(a, t4.x, a4[0]); a4[1] = fmaf(a, t4.y, a4[1]);
                a4[2] = fmaf(a, t4.z, a4[2]); a4[3] = fmaf(a, t4.w, a4[3]);
            }
            *reinterpret_cast<float4 *>(&Tscr[scr(r, 32 + c4)]) = make_float4(a4[0], a4[1], a4[2], a4[3]);
        }
        __syncthreads();
        // T_bl = -T_br M
        if (tid < 256) {
            const int r = tid >> 3, c4 = (tid & 7) * 4;
            float a4[4] = {0.f, 0.f, 0.f, 0.f};
            for (int m = 0; m <= r; ++m) {  // T_br is lower triangular
                const float t = Tscr[scr(32 + r, 32 + m)];
                const float4 m4 = *reinterpret_cast<const float4 *>(&Tscr[scr(m, 32 + c4)]);
                a4[0] = fmaf(t, m4.x, a4[0]); a4[1] = fmaf(t, m4.y, a4[1]);
                a4[2] = fmaf(t, m4.z, a4[2]); a4[3] = fmaf(t, m4.w, a4[3]);
            }
            *reinterpret_cast<float4 *>(&Tscr[scr(32 + r, c4)]) = make_float4(-a4[0], -a4[1], -a4[2], -a4[3]);
        }
        __syncthreads();
        // T_beta = T diag(beta), rewritten in place as a K-major tile
        {
            const int t = tid >> 3, i0 = (tid & 7) * 8;
            const bool upper_right = t < 32 && i0 >= 32;  // zero in T; held the merge product
            float tv[8];
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                float4 x = *reinterpret_cast<const float4 *>(&Tscr[scr(t, i0 + 4 * k)]);
                if (upper_right) x = make_float4(0.f, 0.f, 0.f, 0.f);
                tv[4 * k] = x.x * beta_s[i0 + 4 * k];
                tv[4 * k + 1] = x.y * beta_s[i0 + 4 * k + 1];
                tv[4 * k + 2] = x.z * beta_s[i0 + 4 * k + 2];
                tv[4 * k + 3] = x.w * beta_s[i0 + 4 * k + 3];
            }
            __syncthreads();
#pragma unroll
            for (int k = 0; k < 2; ++k)
                *reinterpret_cast<float4 *>(sm + OFF_TB + kmaj_off(t, i0 + 4 * k, 64)) =
                    tf32x4(tv[4 * k], tv[4 * k + 1], tv[4 * k + 2], tv[4 * k + 3]);
        }
        fence_smem_to_async();
        fence_before_sync();
        __syncthreads();

        // ---- MMA_2: u = T_beta V'
        if (tid == 0) {
            fence_after_sync();
            gemm<64, 64, 64, false, true>(tm + T_U, sb + OFF_TB, 8192, sb + OFF_V, 64, false);
            mma_commit(&bar[B_2]);
        }
        if (!wait_bar(B_2, par)) { failed = true; break; }
        fence_after_sync();
        if (tid == 0 && c + 1 < nchunks) issue_v(c + 1);  // V' consumed
        {
            float v[16];
            tmem_ld16(taddr(tm + T_U, 32 * quarter, col), v);
            tmem_wait_ld();
            if (lane < 16) {  // M=64 layout: row t at lane 16*quarter + l of quarter `quarter`
                const int t = 16 * quarter + lane;
                const float kd = kd_s[t];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    *reinterpret_cast<float4 *>(sm + OFF_U + mn_off(t, col + 4 * k, 64)) =
                        tf32x4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
                    *reinterpret_cast<float4 *>(sm + OFF_TB + mn_off(t, col + 4 * k, 64)) =
                        tf32x4(kd * v[4 * k], kd * v[4 * k + 1], kd * v[4 * k + 2], kd * v[4 * k + 3]);
                }
            }
        }
        fence_smem_to_async();
        if (!wait_bar(B_KMN, par)) { failed = true; break; }
        fence_before_sync();
        __syncthreads();

        // ---- MMA_3: dS = K^T u~ ; MMA_4: y = gamma QS + P u (128-row view of P)
        if (tid == 0) {
            fence_after_sync();
            gemm<128, 64, 64, true, true>(tm + T_DS, sb + OFF_KMN, 64, sb + OFF_TB, 64, false);
            gemm<128, 64, 64, false, true>(tm + T_1, sb + OFF_P - 8192, 8192, sb + OFF_U, 64, true);
            mma_commit(&bar[B_3]);
        }
        if (!wait_bar(B_3, par)) { failed = true; break; }
        fence_after_sync();
        if (tid == 0 && c + 1 < nchunks) issue_kmn(c + 1);  // K (token-major copy) consumed
        {
            float v[16];
            tmem_ld16(taddr(tm + T_DS, 32 * quarter, col), v);
            tmem_wait_ld();
            const float gc = gam_s[n - 1];
#pragma unroll
            for (int j = 0; j < 16; ++j) S[j] = fmaf(gc, S[j], v[j]);
#pragma unroll
            for (int k = 0; k < 4; ++k)
                *reinterpret_cast<float4 *>(sm + OFF_S + mn_off(d_own, col + 4 * k, kHeadDim)) =
                    tf32x4(S[4 * k], S[4 * k + 1], S[4 * k + 2], S[4 * k + 3]);
            float y[16];
            tmem_ld16(taddr(tm + T_1, 32 * quarter, col), y);
            tmem_wait_ld();
            const int t = 32 * quarter + lane - 64;
            if (quarter >= 2 && t < n) store_row16<TO>(out + (tok + t) * v_row + h * kHeadDim + col0 + col, y);
        }
        fence_before_sync();
        __syncthreads();
    }

    // ---------------------------------------------------------------- tear-down
    if (p.fin) {
        if (failed) {
#pragma unroll
            for (int j = 0; j < 16; ++j) S[j] = __int_as_float(0x7fc00000);
        }
#pragma unroll
        for (int k = 0; k < 4; ++k)
            *reinterpret_cast<float4 *>(p.fin + st_off + 4 * k) = make_float4(S[4 * k], S[4 * k + 1], S[4 * k + 2], S[4 * k + 3]);
    }
    if (failed) {  // a wait gave up: poison this CTA's outputs
        for (int e = tid; e < L * kN; e += kThr) {
            const int t = e / kN, j = e % kN;
            out[(seq0 + t) * v_row + h * kHeadDim + col0 + j] = from_f32<TO>(__int_as_float(0x7fc00000));
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
