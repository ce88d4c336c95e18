// ShortConv(4) + per-head L2 normalisation, and the sequence/chunk tables of a prefill.
//
// Page "ARCHITECTURE PREVIEW / FIELD NOTES", section 03: q, k and v each pass a
// kernel-4 ShortConv before the gated delta rule.  The conv is causal and depthwise
// with tap 3 on the current row; q and k are then L2-normalised per (token, head).
// Memory-bound: each raw row is read once (plus a 3-row halo per chunk or 16-row strip,
// served by L2) and each normalised row written once: as fp32 rows (fp32 input) or into the
// chain's tiles ([K;Q] rounded to TF32, K and V to fp16, both 11-bit significands; bf16's 8
// bits would by themselves move y by several percent of its rms).
#include <cuda.h>
#include <cudaTypedefs.h>

#include "gdn_common.cuh"
#include "gdn_internal.h"
#include "chunk_range.cuh"
#include "tc_sm100.cuh"
#include "tma_map.cuh"

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
// fp32 rows (fp32-input path).  grid (max_chunks, 2*Hqk + Hv): CTA = one 64-row chunk of
// one head slot (q heads, then k heads, then v heads).  Warp w walks rows 16w..16w+15 in
// order, keeping the 3-row conv history of its lane's 4 channels in registers.
template <class T>
__global__ void __launch_bounds__(128) conv_l2_kernel(ConvParams p) {
    const int n_chunks = p.cfirst[p.n_seqs];
    const int ci = (int)blockIdx.x;
    if (ci >= n_chunks) return;
    const int b = upper_index(p.cfirst, p.n_seqs, ci);
    const int seq0 = p.cu[b], seq1 = p.cu[b + 1];
    const int r0 = (ci - p.cfirst[b]) * kChunk;  // chunk start within the sequence
    const int len = min(kChunk, seq1 - seq0 - r0);

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
    if (rs >= re) return;
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
            y[c] = conv_act(wt[c][0] * h[0][c] + wt[c][1] * h[1][c] + wt[c][2] * h[2][c] + wt[c][3] * cur[c],
                            p.act);
            ss += y[c] * y[c];
            h[0][c] = h[1][c]; h[1][c] = h[2][c]; h[2][c] = cur[c];
        }
        if (norm) {
            ss = warp_sum(ss);
            const float inv = scale * rsqrtf(ss + p.eps);
#pragma unroll
            for (int c = 0; c < 4; ++c) y[c] *= inv;
        }
        st4(dst + (int64_t)(seq0 + s) * row_stride + c4, y);
    }
}

// ------------------------------------------------------------------------ conv + L2, tiles
// The tensor-core path's tiles from bf16 input.  CTA = one 64-row chunk of one head slot:
// q heads ([K;Q] tile, Q half), k heads ([K;Q] tile, K half, and the fp16 K tile, MN-major),
// v heads (the fp16 V tile, MN-major).  One TMA copy brings the chunk's rows and the 3 rows before
// them (rows outside the tensor read as zero; at a sequence's start the 3 history rows are
// replaced by the conv state or zeros); each warp then walks 16 rows from shared memory and
// stores each row straight into the tiles, TF32-rounded for [K;Q], fp16 for the K and V tiles:
// the 32 lanes of a warp cover one row, whole 128-byte lines.
namespace {
using namespace tc;

constexpr int kSlabRows = kChunk + 3;
constexpr uint32_t kSlabBytes = kSlabRows * kHeadDim * 2;   // bf16 rows, 17,152 B
constexpr uint32_t C_SLAB = 0;
constexpr uint32_t C_BAR = 17408;
constexpr uint32_t kConvSmem = C_BAR + 16;
constexpr uint32_t kConvSmemAlloc = kConvSmem + 1024;
constexpr uint32_t kConvWaitTries = 1u << 24;

struct ConvTileParams {
    CUtensorMap tm_q, tm_k, tm_v;   // [T, H*128] bf16 rows, boxes of 128 columns x 67 rows
    const float *wq, *wk, *wv;      // [ch, 4]
    const void *conv_in;            // [n_seqs, 3, channels] bf16 or null
    float *kq, *kmn, *vi;
    int32_t *cseq;
    const int32_t *cu, *cfirst;
    int n_seqs, n_qk, n_v;
    float q_scale, eps;
    int act;
    ChunkRange rg;
};

// largest b in [0, n) with first[b] <= i (first non-decreasing, first[0] <= i < first[n]),
// found by the whole warp: each step reads 32 points of the remaining range at once
__device__ __forceinline__ int upper_index_warp(const int32_t *first, int n, int i) {
    const int lane = threadIdx.x & 31;
    int lo = 0, hi = n;   // first[lo] <= i, answer in [lo, hi)
    while (hi - lo > 32) {
        const int step = (hi - lo + 31) / 32;
        const int k = lo + lane * step;
        const unsigned m = __ballot_sync(0xffffffffu, k < hi && __ldg(first + k) <= i);
        lo += (31 - __clz(m)) * step;
        hi = min(hi, lo + step);
    }
    const int k = lo + lane;
    const unsigned m = __ballot_sync(0xffffffffu, k < hi && __ldg(first + k) <= i);
    return lo + (31 - __clz(m));
}

__device__ __forceinline__ void bf16x4_to_f32(uint2 r, float v[4]) {
    v[0] = __uint_as_float(r.x << 16);
    v[1] = __uint_as_float(r.x & 0xffff0000u);
    v[2] = __uint_as_float(r.y << 16);
    v[3] = __uint_as_float(r.y & 0xffff0000u);
}

}  // namespace

__global__ void __launch_bounds__(128) conv_tiles_kernel(const __grid_constant__ ConvTileParams p) {
    const int64_t ci = blockIdx.x;   // slot of the range
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int b, jc;
    if (p.rg.compact) {
        if (ci >= p.cfirst[p.n_seqs]) return;   // uniform per CTA
        b = upper_index_warp(p.cfirst, p.n_seqs, (int)ci);
        jc = (int)ci - p.cfirst[b];
        if (blockIdx.y == 0 && threadIdx.x == 0) p.cseq[ci] = b;   // for the chunk-prep pass
    } else if (!sliced_slot_chunk(p.rg, ci, p.cfirst, &b, &jc)) {
        return;   // uniform per CTA
    }
    const int seq0 = p.cu[b], seq1 = p.cu[b + 1];
    const int r0 = jc * kChunk;   // chunk start within the sequence
    const int len = min(kChunk, seq1 - seq0 - r0);

    // slot kinds: 0 q ([K;Q] Q half), 1 k ([K;Q] K half + K tile), 3 v (V tile)
    const int slot = blockIdx.y, nq = p.n_qk;
    const int kind = slot < nq ? 0 : slot < 2 * nq ? 1 : 3;
    const int head = kind == 3 ? slot - 2 * nq : slot - kind * nq;
    const CUtensorMap *tm = kind == 0 ? &p.tm_q : kind == 3 ? &p.tm_v : &p.tm_k;
    const float *w = kind == 0 ? p.wq : kind == 3 ? p.wv : p.wk;
    const int qkc = nq * kHeadDim;
    const int cs_chan = (kind == 0 ? 0 : kind == 3 ? 2 * qkc : qkc) + head * kHeadDim;
    const bool norm = kind != 3;
    const float scale = kind == 0 ? p.q_scale : 1.f;

    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    uint64_t *bar = (uint64_t *)(sm + C_BAR);
    if (threadIdx.x == 0) {
        mbar_init(bar, 1);
        mbar_expect_tx(bar, kSlabBytes);
        tma_load_2d(smem_u32(sm + C_SLAB), tm, head * kHeadDim, seq0 + r0 - 3, bar);
    }
    float wt[4][4];  // wt[channel][tap], this lane's 4 channels
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const float4 t = *reinterpret_cast<const float4 *>(w + (int64_t)(head * kHeadDim + 4 * lane + c) * kConvW);
        wt[c][0] = t.x; wt[c][1] = t.y; wt[c][2] = t.z; wt[c][3] = t.w;
    }
    __syncthreads();   // the barrier is initialised
    const bool ok = mbar_wait(bar, 0, kConvWaitTries);
    if (r0 == 0 && threadIdx.x < 96) {   // history rows of a sequence's first chunk
        const int j = threadIdx.x >> 5;   // slab row j = row j - 3 of the sequence
        uint2 h = make_uint2(0u, 0u);
        if (p.conv_in) {
            const int64_t cs_row = 2 * (int64_t)qkc + (int64_t)p.n_v * kHeadDim;
            h = *reinterpret_cast<const uint2 *>((const bf16 *)p.conv_in + ((int64_t)b * 3 + j) * cs_row +
                                                 cs_chan + 4 * lane);
        }
        *reinterpret_cast<uint2 *>(sm + C_SLAB + j * 256 + lane * 8) = h;
    }
    __syncthreads();

    const unsigned char *slab = sm + C_SLAB + lane * 8;
    float h[3][4];
#pragma unroll
    for (int j = 0; j < 3; ++j) bf16x4_to_f32(*reinterpret_cast<const uint2 *>(slab + (16 * wid + j) * 256), h[j]);
    const bool mn = kind == 3;
    const float nan = __int_as_float(0x7fc00000);
#pragma unroll 4
    for (int i = 0; i < 16; ++i) {
        const int t = 16 * wid + i;
        float cur[4], y[4];
        bf16x4_to_f32(*reinterpret_cast<const uint2 *>(slab + (t + 3) * 256), cur);
        float ss = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            y[c] = conv_act(wt[c][0] * h[0][c] + wt[c][1] * h[1][c] + wt[c][2] * h[2][c] + wt[c][3] * cur[c],
                            p.act);
            ss += y[c] * y[c];
            h[0][c] = h[1][c]; h[1][c] = h[2][c]; h[2][c] = cur[c];
        }
        if (norm) {
            ss = warp_sum(ss);
            const float inv = scale * rsqrtf(ss + p.eps);
#pragma unroll
            for (int c = 0; c < 4; ++c) y[c] *= inv;
        }
        float4 o;   // TF32, nearest with ties away (integer ops); rows past the end are zero
        o.x = t < len ? __uint_as_float((__float_as_uint(y[0]) + 0x1000u) & 0xFFFFE000u) : 0.f;
        o.y = t < len ? __uint_as_float((__float_as_uint(y[1]) + 0x1000u) & 0xFFFFE000u) : 0.f;
        o.z = t < len ? __uint_as_float((__float_as_uint(y[2]) + 0x1000u) & 0xFFFFE000u) : 0.f;
        o.w = t < len ? __uint_as_float((__float_as_uint(y[3]) + 0x1000u) & 0xFFFFE000u) : 0.f;
        if (!ok) o = make_float4(nan, nan, nan, nan);
        if (mn) {   // the V tile, fp16 (nearest even), MN-major
            const float4 f = ok ? make_float4(t < len ? y[0] : 0.f, t < len ? y[1] : 0.f,
                                              t < len ? y[2] : 0.f, t < len ? y[3] : 0.f)
                                : o;
            *reinterpret_cast<uint2 *>(reinterpret_cast<unsigned char *>(p.vi + ((int64_t)ci * p.n_v + head) * 4096) +
                                       tc::mn16_off(t, 4 * lane, kChunk)) =
                make_uint2(tc::pack_f16x2(f.x, f.y), tc::pack_f16x2(f.z, f.w));
        } else {
            unsigned char *kq = reinterpret_cast<unsigned char *>(p.kq + ((int64_t)ci * nq + head) * 16384 +
                                                                 (kind == 0 ? 2048 : 0));
            *reinterpret_cast<float4 *>(kq + (lane >> 3) * 16384 + t * 128 + (((lane & 7) ^ (t & 7)) << 4)) = o;
            if (kind == 1) {   // the K tile, fp16 (nearest even), MN-major
                const float4 f = ok ? make_float4(t < len ? y[0] : 0.f, t < len ? y[1] : 0.f,
                                                  t < len ? y[2] : 0.f, t < len ? y[3] : 0.f)
                                    : o;
                *reinterpret_cast<uint2 *>(reinterpret_cast<unsigned char *>(
                    p.kmn + ((int64_t)ci * nq + head) * 4096) + tc::mn16_off(t, 4 * lane, kChunk)) =
                    make_uint2(tc::pack_f16x2(f.x, f.y), tc::pack_f16x2(f.z, f.w));
            }
        }
    }
    if (!ok && threadIdx.x == 0) mbar_wait(bar, 0, kConvWaitTries);   // the copy is done before exit
}

cudaError_t launch_conv_l2(const ConvParams &p, bool bf16, bool tiles, int64_t n_chunks,
                           int64_t total_tokens, cudaStream_t s) {
    if (n_chunks <= 0) return cudaSuccess;
    if (tiles) {   // tensor-core path: bf16 input only
        if (!bf16) return cudaErrorInvalidValue;
        ConvTileParams tp{};
        const int64_t qkc = (int64_t)p.n_qk * kHeadDim, vc = (int64_t)p.n_v * kHeadDim;
        if (!encode_2d(&tp.tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.q, qkc, total_tokens, qkc * 2, kHeadDim,
                       kSlabRows, CU_TENSOR_MAP_SWIZZLE_NONE) ||
            !encode_2d(&tp.tm_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.k, qkc, total_tokens, qkc * 2, kHeadDim,
                       kSlabRows, CU_TENSOR_MAP_SWIZZLE_NONE) ||
            !encode_2d(&tp.tm_v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.v, vc, total_tokens, vc * 2, kHeadDim,
                       kSlabRows, CU_TENSOR_MAP_SWIZZLE_NONE))
            return cudaErrorInvalidValue;
        tp.wq = p.wq; tp.wk = p.wk; tp.wv = p.wv; tp.conv_in = p.conv_in;
        tp.kq = p.kq; tp.kmn = p.kmn; tp.vi = p.vi; tp.cseq = p.cseq; tp.cu = p.cu; tp.cfirst = p.cfirst;
        tp.n_seqs = p.n_seqs; tp.n_qk = p.n_qk; tp.n_v = p.n_v; tp.q_scale = p.q_scale; tp.eps = p.eps; tp.act = p.act;
        tp.rg = p.rg;
        cudaError_t e = cudaFuncSetAttribute(conv_tiles_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)kConvSmemAlloc);
        if (e != cudaSuccess) return e;
        dim3 grid((unsigned)n_chunks, 2 * p.n_qk + p.n_v);
        TraceLaunch tl(s, "conv_l2");
        conv_tiles_kernel<<<grid, 128, kConvSmemAlloc, s>>>(tp);
        return cudaGetLastError();
    }
    dim3 grid((unsigned)n_chunks, 2 * p.n_qk + p.n_v);
    TraceLaunch tl(s, "conv_l2");
    if (bf16) conv_l2_kernel<gdn::bf16><<<grid, 128, 0, s>>>(p);
    else conv_l2_kernel<float><<<grid, 128, 0, s>>>(p);
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
