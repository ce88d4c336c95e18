// Entering states of consecutive spans of one sequence from the spans' affine maps (the
// prefix combination of the context-parallel prefill).
//
// The gated delta rule of the page "ARCHITECTURE PREVIEW / FIELD NOTES", section 03 (GATED
// DELTANET equations) is affine in the state: over a span of tokens, per V head,
// S_out = M S_in + B with M [d_k x d_k] the product of the span's maps alpha_t (I - beta_t
// k_t k_t^T) and B the state the span leaves from zero.  Given every span's (M, B), the state
// entering span p is
//     S_in[0] = S0,   S_in[p+1] = M[p] S_in[p] + B[p].
// The columns of S (the d_v index) do not mix, so one CTA owns one V head and 32 columns and
// walks the spans in order, keeping its 128 x 32 block of S in shared memory; each span's M
// is staged transposed in shared memory (64 KB) so that the threads of a warp read
// consecutive rows of it.  fp32 FMAs on the CUDA cores: the work (2 x 128^3 flop per span and
// V head) is far too small for the tensor cores to matter, and fp32 keeps the combination as
// exact as the maps it combines.
#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {

namespace {
constexpr int kCols = 32;                 // columns of S per CTA
constexpr int kThreads = 256;             // 128 rows x 2 half-blocks of 16 columns
constexpr uint32_t kSmemMt = 128 * 129 * 4;   // M^T, rows padded by one float
constexpr uint32_t kSmemS = 128 * kCols * 4;  // the S block
}  // namespace

__global__ void __launch_bounds__(kThreads) affine_combine_kernel(const float *__restrict__ M,
                                                                  const float *__restrict__ B,
                                                                  const float *__restrict__ S0,
                                                                  float *__restrict__ S_in, int n_spans,
                                                                  int n_v) {
    extern __shared__ float sm[];
    float *mt = sm;                        // mt[k * 129 + r] = M[r][k]
    float *s = sm + kSmemMt / 4;           // s[k * 32 + c] = S[k][c0 + c]
    const int h = blockIdx.x, c0 = blockIdx.y * kCols;
    const int t = threadIdx.x, r = t >> 1, cb = (t & 1) * 16;
    const int64_t mat = (int64_t)128 * 128;
    const int64_t head = (int64_t)h * mat;

    // S_in[0] = S0 (or zero)
    for (int e = t; e < 128 * kCols; e += kThreads) {
        const int k = e / kCols, c = e % kCols;
        const float v = S0 ? S0[head + (int64_t)k * 128 + c0 + c] : 0.f;
        s[e] = v;
        S_in[head + (int64_t)k * 128 + c0 + c] = v;
    }
    for (int p = 0; p < n_spans; ++p) {
        const int64_t span = (int64_t)p * n_v * mat + head;
        __syncthreads();   // the previous span's reads of mt are done
        for (int e = t; e < 128 * 128; e += kThreads) {
            const int rr = e >> 7, k = e & 127;   // coalesced read of row rr
            mt[k * 129 + rr] = M[span + e];
        }
        __syncthreads();
        float acc[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) acc[c] = B[span + (int64_t)r * 128 + c0 + cb + c];
#pragma unroll 4
        for (int k = 0; k < 128; ++k) {
            const float m = mt[k * 129 + r];
            const float4 *sk = reinterpret_cast<const float4 *>(s + k * kCols + cb);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float4 x = sk[q];
                acc[4 * q] = fmaf(m, x.x, acc[4 * q]);
                acc[4 * q + 1] = fmaf(m, x.y, acc[4 * q + 1]);
                acc[4 * q + 2] = fmaf(m, x.z, acc[4 * q + 2]);
                acc[4 * q + 3] = fmaf(m, x.w, acc[4 * q + 3]);
            }
        }
        __syncthreads();   // every thread has read the old S block
        float *dst = S_in + (int64_t)(p + 1) * n_v * mat + head + (int64_t)r * 128 + c0 + cb;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 v = make_float4(acc[4 * q], acc[4 * q + 1], acc[4 * q + 2], acc[4 * q + 3]);
            *reinterpret_cast<float4 *>(s + r * kCols + cb + 4 * q) = v;
            *reinterpret_cast<float4 *>(dst + 4 * q) = v;
        }
    }
}

cudaError_t launch_affine_combine(const float *M, const float *B, const float *S0, float *S_in, int n_spans,
                                  int n_v, cudaStream_t s) {
    const uint32_t smem = kSmemMt + kSmemS;
    cudaError_t e = cudaFuncSetAttribute(affine_combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)n_v, 128 / kCols);
    TraceLaunch tl(s, "affine_combine");
    affine_combine_kernel<<<grid, kThreads, smem, s>>>(M, B, S0, S_in, n_spans, n_v);
    return cudaGetLastError();
}

}  // namespace gdn
