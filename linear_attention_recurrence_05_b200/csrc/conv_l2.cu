// ShortConv(4) + per-head L2 normalisation, and the sequence/chunk tables of a prefill.
//
// Page "ARCHITECTURE PREVIEW / FIELD NOTES", section 03: q, k and v each pass a
// kernel-4 ShortConv before the gated delta rule.  The conv is causal and depthwise
// with tap 3 on the current row; q and k are then L2-normalised per (token, head).
// Memory-bound: each raw row is read once (plus a 3-row halo per 16-row strip, served
// by L2) and each normalised row written once, in fp32 (rounding these rows to bf16
// would by itself move y by several percent of its rms).
#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {

// ------------------------------------------------------------------------ tables
// One CTA.  cu[b] = running max of clamp(cu_in[b], 0, T) (so lengths are >= 0 and
// every row index stays inside [0, T)); cfirst = exclusive scan of ceil(L_b / 64).
template <int NT>
__device__ __forceinline__ int block_scan_incl(int x, bool is_max, int *tmp) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x = is_max ? max(x, y) : x + y;
    }
    if (lane == 31) tmp[w] = x;
    __syncthreads();
    if (w == 0) {
        int y = lane < NT / 32 ? tmp[lane] : (is_max ? INT32_MIN : 0);
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int z = __shfl_up_sync(0xffffffffu, y, o);
            if (lane >= o) y = is_max ? max(y, z) : y + z;
        }
        tmp[lane] = y;
    }
    __syncthreads();
    if (w > 0) x = is_max ? max(x, tmp[w - 1]) : x + tmp[w - 1];
    __syncthreads();
    return x;
}

__global__ void __launch_bounds__(1024) seq_table_kernel(const int32_t *__restrict__ cu_in,
                                                         int n_seqs, int T, int32_t *cu,
                                                         int32_t *cfirst) {
    __shared__ int tmp[32];
    __shared__ int carry;
    if (threadIdx.x == 0) carry = 0;
    __syncthreads();
    // pass 1: clamped running max over n_seqs + 1 entries
    for (int base = 0; base <= n_seqs; base += 1024) {
        const int i = base + threadIdx.x;
        int x = i <= n_seqs ? min(max(cu_in[i], 0), T) : 0;
        x = block_scan_incl<1024>(x, true, tmp);
        x = max(x, carry);
        if (i <= n_seqs) cu[i] = x;
        __syncthreads();
        if (threadIdx.x == 1023) carry = x;
        __syncthreads();
    }
    __syncthreads();
    if (threadIdx.x == 0) carry = 0;
    __syncthreads();
    // pass 2: chunk counts, exclusive scan into cfirst[0..n_seqs]
    for (int base = 0; base < n_seqs; base += 1024) {
        const int b = base + threadIdx.x;
        int c = 0;
        if (b < n_seqs) c = (cu[b + 1] - cu[b] + kChunk - 1) / kChunk;
        int incl = block_scan_incl<1024>(c, false, tmp);
        if (b < n_seqs) cfirst[b] = carry + incl - c;
        __syncthreads();
        if (threadIdx.x == 1023) carry += incl;
        __syncthreads();
    }
    if (threadIdx.x == 0) cfirst[n_seqs] = carry;
}

cudaError_t launch_seq_table(const int32_t *cu_in, int n_seqs, int64_t T, int32_t *cu,
                             int32_t *cfirst, cudaStream_t s) {
    TraceLaunch tl(s, "seq_table");
    seq_table_kernel<<<1, 1024, 0, s>>>(cu_in, n_seqs, (int)T, cu, cfirst);
    return cudaGetLastError();
}

// ------------------------------------------------------------------------ conv + L2
// grid (max_chunks, 2*Hqk + Hv): CTA = one 64-row chunk of one head slot (q heads,
// then k heads, then v heads).  Warp w walks rows 16w..16w+15 in order, keeping the
// 3-row conv history of its lane's 4 channels in registers.
// kTiles: instead of fp32 rows, write the tensor-core path's chunk tiles, TF32-rounded (the
// MMAs read them as TF32; rounding here gives round-to-nearest instead of truncation), in
// the shared-memory layouts the tensor-core kernels copy them into:
//   [K;Q] of (chunk, QK head): 4 blocks of 32 features x (K 64 rows | Q 64 rows), 128-byte
//     rows with 16-byte chunks XOR-swizzled by row (K-major operand layout);
//   K of (chunk, QK head) and V of (chunk, V head): 4 blocks of 32 features x 64 rows,
//     128-byte rows with 32-byte granules XOR-swizzled by row (MN-major operand layout).
// Rows past the end of the sequence are written as zeros.
template <class T, bool kTiles>
__global__ void __launch_bounds__(128) conv_l2_kernel(ConvParams p) {
    const int n_chunks = p.cfirst[p.n_seqs];
    const int ci = (int)(p.chunk_lo + blockIdx.x);
    if (ci >= n_chunks) return;
    const int b = upper_index(p.cfirst, p.n_seqs, ci);
    const int seq0 = p.cu[b], seq1 = p.cu[b + 1];
    const int r0 = (ci - p.cfirst[b]) * kChunk;  // chunk start within the sequence
    const int len = min(kChunk, seq1 - seq0 - r0);
    if (kTiles && blockIdx.y == 0 && threadIdx.x == 0) p.cseq[ci] = b;   // for the chunk-prep pass

    const int slot = blockIdx.y;
    const T *x;
    float *dst;
    const float *w;
    int64_t row_stride;
    int chan, cs_chan;
    bool norm;
    float scale = 1.f;
    const int qkc = p.n_qk * kHeadDim;
    if (slot < p.n_qk) {
        x = (const T *)p.q; dst = p.qh; w = p.wq; row_stride = qkc;
        chan = slot * kHeadDim; cs_chan = chan; norm = true; scale = p.q_scale;
    } else if (slot < 2 * p.n_qk) {
        x = (const T *)p.k; dst = p.kh; w = p.wk; row_stride = qkc;
        chan = (slot - p.n_qk) * kHeadDim; cs_chan = qkc + chan; norm = true;
    } else {
        x = (const T *)p.v; dst = p.vh; w = p.wv; row_stride = (int64_t)p.n_v * kHeadDim;
        chan = (slot - 2 * p.n_qk) * kHeadDim; cs_chan = 2 * qkc + chan; norm = false;
    }
    const int64_t cs_row = 2 * (int64_t)qkc + (int64_t)p.n_v * kHeadDim;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int c4 = chan + 4 * lane;  // first of this lane's 4 channels

    float wt[4][4];  // wt[channel][tap]
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        float4 t = *reinterpret_cast<const float4 *>(w + (int64_t)(c4 + c) * kConvW);
        wt[c][0] = t.x; wt[c][1] = t.y; wt[c][2] = t.z; wt[c][3] = t.w;
    }
    const int rs = r0 + wid * 16;                  // first row of this warp (in sequence)
    const int re = min(rs + 16, r0 + len);
    if (!kTiles && rs >= re) return;
    // tile destinations (float offsets of this lane's 4 features, row 0)
    float *t_a = nullptr, *t_b = nullptr;          // K-major ([K;Q]) and MN-major (K or V) tile
    if (kTiles) {
        if (slot < p.n_qk) {
            t_a = p.kq + ((int64_t)ci * p.n_qk + slot) * 16384 + 2048;
        } else if (slot < 2 * p.n_qk) {
            t_a = p.kq + ((int64_t)ci * p.n_qk + slot - p.n_qk) * 16384;
            t_b = p.kmn + ((int64_t)ci * p.n_qk + slot - p.n_qk) * 8192;
        } else {
            t_b = p.vi + ((int64_t)ci * p.n_v + slot - 2 * p.n_qk) * 8192;
        }
    }
    auto put_tile = [&](int t, const float y[4]) {  // row t of the chunk
        if (t_a) st4(t_a + (lane >> 3) * 4096 + t * 32 + (((lane & 7) ^ (t & 7)) << 2), y);
        if (t_b) st4(t_b + (lane >> 3) * 2048 + t * 32 + ((((lane & 7) >> 1) ^ (t & 3)) << 3) + (lane & 1) * 4, y);
    };
    if (kTiles) {  // rows of this warp past the end of the sequence
        const float z[4] = {0.f, 0.f, 0.f, 0.f};
        for (int s = max(rs, r0 + len); s < r0 + wid * 16 + 16; ++s) put_tile(s - r0, z);
        if (rs >= re) return;
    }
    // history rows rs-3, rs-2, rs-1
    float h[3][4];
#pragma unroll
    for (int j = 0; j < 3; ++j) {
        const int s = rs - 3 + j;
        if (s >= 0) {
            ld4(x + (int64_t)(seq0 + s) * row_stride + c4, h[j]);
        } else if (p.conv_in) {
            ld4((const T *)p.conv_in + ((int64_t)b * 3 + (3 + s)) * cs_row + cs_chan + 4 * lane, h[j]);
        } else {
            h[j][0] = h[j][1] = h[j][2] = h[j][3] = 0.f;
        }
    }
    for (int s = rs; s < re; ++s) {
        float cur[4], y[4];
        ld4(x + (int64_t)(seq0 + s) * row_stride + c4, cur);
        float ss = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            y[c] = wt[c][0] * h[0][c] + wt[c][1] * h[1][c] + wt[c][2] * h[2][c] + wt[c][3] * cur[c];
            ss += y[c] * y[c];
            h[0][c] = h[1][c]; h[1][c] = h[2][c]; h[2][c] = cur[c];
        }
        if (norm) {
            ss = warp_sum(ss);
            const float inv = scale * rsqrtf(ss + p.eps);
#pragma unroll
            for (int c = 0; c < 4; ++c) y[c] *= inv;
        }
        if (kTiles) {
#pragma unroll
            for (int c = 0; c < 4; ++c)  // TF32, nearest with ties away (integer ops)
                y[c] = __uint_as_float((__float_as_uint(y[c]) + 0x1000u) & 0xFFFFE000u);
            put_tile(s - r0, y);
        } else {
            st4(dst + (int64_t)(seq0 + s) * row_stride + c4, y);
        }
    }
}

cudaError_t launch_conv_l2(const ConvParams &p, bool bf16, bool tiles, int64_t n_chunks,
                           cudaStream_t s) {
    if (n_chunks <= 0) return cudaSuccess;
    dim3 grid((unsigned)n_chunks, 2 * p.n_qk + p.n_v);
    TraceLaunch tl(s, "conv_l2");
    if (bf16) {
        if (tiles) conv_l2_kernel<gdn::bf16, true><<<grid, 128, 0, s>>>(p);
        else conv_l2_kernel<gdn::bf16, false><<<grid, 128, 0, s>>>(p);
    } else {
        if (tiles) conv_l2_kernel<float, true><<<grid, 128, 0, s>>>(p);
        else conv_l2_kernel<float, false><<<grid, 128, 0, s>>>(p);
    }
    return cudaGetLastError();
}

// ------------------------------------------------------------------------ conv state out
// Last 3 raw rows of each sequence (history rows first when the sequence is short).
// One thread owns 4 channels of one sequence and reads all 3 source rows before it
// writes, so conv_out may alias conv_in.
template <class T>
__global__ void conv_state_out_kernel(const T *q, const T *k, const T *v, const T *conv_in,
                                      T *conv_out, const int32_t *cu, int n_seqs, int n_qk,
                                      int n_v) {
    const int b = blockIdx.x;
    const int qkc = n_qk * kHeadDim;
    const int64_t ch = 2 * (int64_t)qkc + (int64_t)n_v * kHeadDim;
    const int64_t c = 4 * ((int64_t)blockIdx.y * blockDim.x + threadIdx.x);
    if (c >= ch) return;
    const int seq0 = cu[b], L = cu[b + 1] - cu[b];
    const T *x;
    int64_t stride, cc;
    if (c < qkc) { x = q; stride = qkc; cc = c; }
    else if (c < 2 * qkc) { x = k; stride = qkc; cc = c - qkc; }
    else { x = v; stride = (int64_t)n_v * kHeadDim; cc = c - 2 * qkc; }
    alignas(16) T rows[3][4];
#pragma unroll
    for (int r = 0; r < 3; ++r) {
        const int s = L - 3 + r;
        if (s >= 0) cp4(rows[r], x + (int64_t)(seq0 + s) * stride + cc);
        else if (conv_in) cp4(rows[r], conv_in + ((int64_t)b * 3 + (3 + s)) * ch + c);
        else zero4(rows[r]);
    }
#pragma unroll
    for (int r = 0; r < 3; ++r) cp4(conv_out + ((int64_t)b * 3 + r) * ch + c, rows[r]);
}

cudaError_t launch_conv_state_out(const void *q, const void *k, const void *v,
                                  const void *conv_in, void *conv_out, const int32_t *cu,
                                  int n_seqs, int n_qk, int n_v, bool bf16, cudaStream_t s) {
    if (n_seqs <= 0) return cudaSuccess;
    const int64_t ch4 = (2 * (int64_t)n_qk * kHeadDim + (int64_t)n_v * kHeadDim) / 4;
    dim3 grid((unsigned)n_seqs, (unsigned)((ch4 + 255) / 256));
    TraceLaunch tl(s, "conv_state_out");
    if (bf16)
        conv_state_out_kernel<gdn::bf16><<<grid, 256, 0, s>>>(
            (const gdn::bf16 *)q, (const gdn::bf16 *)k, (const gdn::bf16 *)v,
            (const gdn::bf16 *)conv_in, (gdn::bf16 *)conv_out, cu, n_seqs, n_qk, n_v);
    else
        conv_state_out_kernel<float><<<grid, 256, 0, s>>>(
            (const float *)q, (const float *)k, (const float *)v, (const float *)conv_in,
            (float *)conv_out, cu, n_seqs, n_qk, n_v);
    return cudaGetLastError();
}

}  // namespace gdn
