// Chunked gated-delta-rule prefill on CUDA cores (fp32 arithmetic).
//
// This is the fp32-storage path and the reference-precision path of libgdn.  It
// implements the chunk-64 WY/UT form of the recurrence of the page "ARCHITECTURE
// PREVIEW / FIELD NOTES", section 03 (GATED DELTANET equations).  Within a chunk,
// with g_t = sum_{s<=t} log alpha_s and gamma_t = exp(g_t):
//     A_ti = beta_t exp(g_t - g_i) k_t.k_i   (i < t),    T = (I + A)^-1
//     W = T diag(beta gamma) K,   U = T diag(beta) V,    u = U - W S
//     y_t = gamma_t S^T q_t + sum_{i<=t} exp(g_t - g_i) (q_t.k_i) u_i
//     S  <- gamma_C S + sum_i exp(g_C - g_i) k_i u_i^T
// which unrolls the token recurrence exactly; only rounding differs.
//
// One CTA owns one (sequence, V head, 32-column slice of d_v) and walks the
// sequence's chunks in order.  The column slice is exact: column j of e, u, S and y
// depends only on column j of v and S.  Everything stays in shared memory.
#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {

namespace {
constexpr int kSlice = 32;                 // d_v columns per CTA
constexpr int kNSlice = kHeadDim / kSlice; // CTAs per (sequence, V head)
constexpr int kThreads = 256;
constexpr int kKP = kHeadDim + 1;          // padded row of K/Q (bank-conflict free)
constexpr int kAP = kChunk + 1;
constexpr int kXW = kHeadDim + kSlice;     // columns of [W | U]

struct SimtSmem {
    float K[kChunk][kKP];
    float Q[kChunk][kKP];
    float V[kChunk][kSlice];
    float A[kChunk][kAP];
    float P[kChunk][kAP];
    float X[kChunk][kXW];
    float S[kHeadDim][kSlice];
    float u[kChunk][kSlice];
    // g_t = sum_{s<=t} log alpha_s in fp64: with strong decay g reaches -100 and beyond inside
    // a chunk, and fp32 sums would leave ~1e-4 relative error in the ratios exp(g_t - g_i)
    double g[kChunk];
    float gam[kChunk];
    float beta[kChunk];
    float kd[kChunk];
};
}  // namespace

template <class T, class TO>
__global__ void __launch_bounds__(kThreads, 1) scan_simt_kernel(ScanParams p) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    SimtSmem &sm = *reinterpret_cast<SimtSmem *>(smem_raw);
    const int tid = threadIdx.x;
    const int slice = blockIdx.x % kNSlice;
    const int h = (blockIdx.x / kNSlice) % p.n_v;
    const int b = blockIdx.x / (kNSlice * p.n_v);
    const int g_qk = h / (p.n_v / p.n_qk);
    const int seq0 = p.cu[b], L = p.cu[b + 1] - p.cu[b];
    const int col0 = slice * kSlice;
    const int64_t qk_row = (int64_t)p.n_qk * kHeadDim, v_row = (int64_t)p.n_v * kHeadDim;
    const float *qh = p.qh, *kh = p.kh, *vh = p.vh;
    const T *al = (const T *)p.alpha, *be = (const T *)p.beta;
    TO *out = (TO *)p.out;

    const int64_t st_off = ((int64_t)b * p.n_v + h) * kHeadDim * kHeadDim;
    for (int e = tid; e < kHeadDim * kSlice; e += kThreads) {
        const int r = e / kSlice, j = e % kSlice;
        sm.S[r][j] = p.init ? p.init[st_off + (int64_t)r * kHeadDim + col0 + j] : 0.f;
    }

    for (int c0 = 0; c0 < L; c0 += kChunk) {
        const int n = min(kChunk, L - c0);
        const int64_t tok = seq0 + c0;
        __syncthreads();
        // ---- load K, Q (full rows), V slice, gates
        for (int e = tid; e < kChunk * (kHeadDim / 4); e += kThreads) {
            const int t = e / (kHeadDim / 4), c = 4 * (e % (kHeadDim / 4));
            float kv[4] = {0.f, 0.f, 0.f, 0.f}, qv[4] = {0.f, 0.f, 0.f, 0.f};
            if (t < n) {
                ld4(kh + (tok + t) * qk_row + g_qk * kHeadDim + c, kv);
                ld4(qh + (tok + t) * qk_row + g_qk * kHeadDim + c, qv);
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) { sm.K[t][c + i] = kv[i]; sm.Q[t][c + i] = qv[i]; }
        }
        for (int e = tid; e < kChunk * (kSlice / 4); e += kThreads) {
            const int t = e / (kSlice / 4), c = 4 * (e % (kSlice / 4));
            float vv[4] = {0.f, 0.f, 0.f, 0.f};
            if (t < n) ld4(vh + (tok + t) * v_row + h * kHeadDim + col0 + c, vv);
#pragma unroll
            for (int i = 0; i < 4; ++i) sm.V[t][c + i] = vv[i];
        }
        if (tid < kChunk) {
            float la = 0.f, bb = 0.f;
            if (tid < n) {
                la = safe_log_alpha(to_f32(al[(tok + tid) * p.n_v + h]));
                bb = to_f32(be[(tok + tid) * p.n_v + h]);
            }
            sm.g[tid] = la;
            sm.beta[tid] = bb;
        }
        __syncthreads();
        if (tid < 32) {  // inclusive scan of log alpha over 64 rows (two per lane), in fp64
            const double a0 = sm.g[2 * tid], a1 = sm.g[2 * tid + 1];
            double s = a0 + a1;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const double y = __shfl_up_sync(0xffffffffu, s, o);
                if (tid >= o) s += y;
            }
            const double base = s - (a0 + a1);
            sm.g[2 * tid] = base + a0;
            sm.g[2 * tid + 1] = s;
        }
        __syncthreads();
        if (tid < kChunk) {
            sm.gam[tid] = expf((float)sm.g[tid]);
            sm.kd[tid] = tid < n ? expf((float)(sm.g[n - 1] - sm.g[tid])) : 0.f;
        }
        // ---- A = strict-lower beta exp(g_t - g_i) K K^T ;  P = lower exp(g_t - g_i) Q K^T
        for (int e = tid; e < kChunk * kChunk; e += kThreads) {
            const int t = e / kChunk, i = e % kChunk;
            float a = 0.f, pq = 0.f;
            if (i <= t && t < n) {
                float dk = 0.f, dq = 0.f;
#pragma unroll 8
                for (int r = 0; r < kHeadDim; ++r) {
                    const float ki = sm.K[i][r];
                    dk = fmaf(sm.K[t][r], ki, dk);
                    dq = fmaf(sm.Q[t][r], ki, dq);
                }
                const float dec = expf((float)(sm.g[t] - sm.g[i]));
                pq = dec * dq;
                if (i < t) a = sm.beta[t] * dec * dk;
            }
            sm.A[t][i] = a;
            sm.P[t][i] = pq;
        }
        __syncthreads();
        // ---- forward substitution (I + A) X = [diag(beta gamma) K | diag(beta) V]
        if (tid < kXW) {
            const int col = tid;
            for (int t = 0; t < n; ++t) {
                float x = col < kHeadDim ? sm.beta[t] * sm.gam[t] * sm.K[t][col]
                                         : sm.beta[t] * sm.V[t][col - kHeadDim];
                float x1 = 0.f, x2 = 0.f, x3 = 0.f;
                int i = 0;
                for (; i + 4 <= t; i += 4) {
                    x = fmaf(-sm.A[t][i], sm.X[i][col], x);
                    x1 = fmaf(-sm.A[t][i + 1], sm.X[i + 1][col], x1);
                    x2 = fmaf(-sm.A[t][i + 2], sm.X[i + 2][col], x2);
                    x3 = fmaf(-sm.A[t][i + 3], sm.X[i + 3][col], x3);
                }
                for (; i < t; ++i) x = fmaf(-sm.A[t][i], sm.X[i][col], x);
                sm.X[t][col] = x + x1 + x2 + x3;
            }
        }
        __syncthreads();
        // ---- u = U - W S   (rows >= n are zero)
        {
            const int j = tid % kSlice;
            for (int t = tid / kSlice; t < kChunk; t += kThreads / kSlice) {
                float acc = 0.f;
                if (t < n) {
                    acc = sm.X[t][kHeadDim + j];
#pragma unroll 8
                    for (int r = 0; r < kHeadDim; ++r) acc = fmaf(-sm.X[t][r], sm.S[r][j], acc);
                }
                sm.u[t][j] = acc;
            }
        }
        __syncthreads();
        // ---- y = gamma Q S + P u  -> out
        {
            const int j = tid % kSlice;
            for (int t = tid / kSlice; t < n; t += kThreads / kSlice) {
                float qs = 0.f;
#pragma unroll 8
                for (int r = 0; r < kHeadDim; ++r) qs = fmaf(sm.Q[t][r], sm.S[r][j], qs);
                float acc = sm.gam[t] * qs;
                for (int i = 0; i <= t; ++i) acc = fmaf(sm.P[t][i], sm.u[i][j], acc);
                out[(tok + t) * v_row + h * kHeadDim + col0 + j] = from_f32<TO>(acc);
            }
        }
        __syncthreads();
        // ---- S <- gamma_C S + sum_i exp(g_C - g_i) k_i u_i^T
        {
            const int j = tid % kSlice;
            const float gc = sm.gam[n - 1];
            for (int r = tid / kSlice; r < kHeadDim; r += kThreads / kSlice) {
                float acc = gc * sm.S[r][j];
                for (int i = 0; i < n; ++i) acc = fmaf(sm.kd[i] * sm.K[i][r], sm.u[i][j], acc);
                sm.S[r][j] = acc;
            }
        }
    }
    __syncthreads();
    if (p.fin) {
        for (int e = tid; e < kHeadDim * kSlice; e += kThreads) {
            const int r = e / kSlice, j = e % kSlice;
            p.fin[st_off + (int64_t)r * kHeadDim + col0 + j] = sm.S[r][j];
        }
    }
}

template <class T, class TO>
static cudaError_t launch_scan_simt_t(const ScanParams &p, cudaStream_t s) {
    const size_t smem = sizeof(SimtSmem);
    const unsigned grid = (unsigned)((int64_t)p.n_seqs * p.n_v * kNSlice);
    cudaError_t e = cudaFuncSetAttribute(scan_simt_kernel<T, TO>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    TraceLaunch tl(s, "scan_simt");
    scan_simt_kernel<T, TO><<<grid, kThreads, smem, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_scan_simt(const ScanParams &p, bool in_bf16, bool out_bf16, cudaStream_t s) {
    if (p.n_seqs <= 0) return cudaSuccess;
    if (in_bf16) return out_bf16 ? launch_scan_simt_t<gdn::bf16, gdn::bf16>(p, s)
                                 : launch_scan_simt_t<gdn::bf16, float>(p, s);
    return out_bf16 ? launch_scan_simt_t<float, gdn::bf16>(p, s) : launch_scan_simt_t<float, float>(p, s);
}

}  // namespace gdn
