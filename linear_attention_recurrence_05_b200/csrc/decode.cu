// Single-token decode step on resident fp32 states (HBM-bound).
//
// The one-token case of the GATED DELTANET equations (page "ARCHITECTURE PREVIEW /
// FIELD NOTES", section 03) with the kernel-4 ShortConv history shifted by one row.
// With r = S^T k, p = S^T q (both over the OLD state S):
//     e = v - alpha r,      y = S_t^T q = alpha p + beta (k.q) e,
//     S_t = alpha S + beta k e^T.
// so one read pass over S gives both reductions, and each state is read once and
// written once.  S rows are streamed with 16-byte loads: warp w owns rows
// 16w..16w+15 and lane l owns columns 4l..4l+3, so one warp instruction moves one
// full 512-byte row.
//
// One CTA owns one decode row b and one QK head g with its Hv/Hqk value heads: it is
// the only CTA that touches that row's q/k conv-state channels, so the in-place
// conv-state shift needs no cross-CTA ordering.
#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {

namespace {
constexpr int kDecThreads = 256;
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kRowsPerWarp = kHeadDim / kDecWarps;  // 16
}  // namespace

template <class T, class TO>
__global__ void __launch_bounds__(kDecThreads, 2) decode_kernel(DecodeParams p) {
    __shared__ __align__(16) float qs[kHeadDim], ks[kHeadDim], vs[kHeadDim], es[kHeadDim];
    __shared__ __align__(16) float red_r[kDecWarps][kHeadDim], red_p[kDecWarps][kHeadDim];
    __shared__ float kq_s;

    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int b = blockIdx.x / p.n_qk, g = blockIdx.x % p.n_qk;
    const int G = p.n_v / p.n_qk;
    const int slot = p.slots ? p.slots[b] : b;
    const int qkc = p.n_qk * kHeadDim;
    const int64_t ch = 2 * (int64_t)qkc + (int64_t)p.n_v * kHeadDim;
    TO *outp = (TO *)p.out;

    if (slot < 0 || slot >= p.n_rows) {  // skipped row: zero output, touch no state
        for (int e = tid; e < G * kHeadDim; e += kDecThreads)
            outp[(int64_t)b * p.n_v * kHeadDim + (int64_t)g * G * kHeadDim + e] = from_f32<TO>(0.f);
        return;
    }
    T *cs = p.conv ? (T *)p.conv + (int64_t)slot * 3 * ch : nullptr;

    // ---- q and k: conv (+ shift of their conv-state channels) and L2, warps 0 and 1
    if (wid < 2) {
        const bool isq = wid == 0;
        const T *x = (const T *)(isq ? p.q : p.k) + ((int64_t)b * p.n_qk + g) * kHeadDim;
        const float *w = isq ? p.wq : p.wk;
        const int cc = (isq ? 0 : qkc) + g * kHeadDim + 4 * lane;  // conv-state channel
        const int wc = g * kHeadDim + 4 * lane;                    // weight row
        float cur[4], hst[3][4], y[4];
        ld4(x + 4 * lane, cur);
#pragma unroll
        for (int j = 0; j < 3; ++j) {
            if (cs) ld4(cs + (int64_t)j * ch + cc, hst[j]);
            else hst[j][0] = hst[j][1] = hst[j][2] = hst[j][3] = 0.f;
        }
        float ss = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            float4 wt = *reinterpret_cast<const float4 *>(w + (int64_t)(wc + c) * kConvW);
            y[c] = conv_act(wt.x * hst[0][c] + wt.y * hst[1][c] + wt.z * hst[2][c] + wt.w * cur[c], p.act);
            ss += y[c] * y[c];
        }
        ss = warp_sum(ss);
        const float inv = (isq ? p.q_scale : 1.f) * rsqrtf(ss + p.eps);
        float *dst = isq ? qs : ks;
#pragma unroll
        for (int c = 0; c < 4; ++c) dst[4 * lane + c] = y[c] * inv;
        if (cs) {  // shift: rows 1,2 move to 0,1; the raw current row becomes row 2
            st4(cs + 0 * ch + cc, hst[1]);
            st4(cs + 1 * ch + cc, hst[2]);
            cp4(cs + 2 * ch + cc, x + 4 * lane);
        }
    }
    __syncthreads();
    if (wid == 0) {
        float d = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) d += qs[4 * lane + c] * ks[4 * lane + c];
        d = warp_sum(d);
        if (lane == 0) kq_s = d;
    }

    for (int hh = 0; hh < G; ++hh) {
        const int h = g * G + hh;
        // ---- v conv for this V head (warp 2), overlapped with the state loads below
        if (wid == 2) {
            const T *x = (const T *)p.v + ((int64_t)b * p.n_v + h) * kHeadDim;
            const int cc = 2 * qkc + h * kHeadDim + 4 * lane;
            const int wc = h * kHeadDim + 4 * lane;
            float cur[4], hst[3][4], y[4];
            ld4(x + 4 * lane, cur);
#pragma unroll
            for (int j = 0; j < 3; ++j) {
                if (cs) ld4(cs + (int64_t)j * ch + cc, hst[j]);
                else hst[j][0] = hst[j][1] = hst[j][2] = hst[j][3] = 0.f;
            }
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float4 wt = *reinterpret_cast<const float4 *>(p.wv + (int64_t)(wc + c) * kConvW);
                y[c] = conv_act(wt.x * hst[0][c] + wt.y * hst[1][c] + wt.z * hst[2][c] + wt.w * cur[c], p.act);
                vs[4 * lane + c] = y[c];
            }
            if (cs) {
                st4(cs + 0 * ch + cc, hst[1]);
                st4(cs + 1 * ch + cc, hst[2]);
                cp4(cs + 2 * ch + cc, x + 4 * lane);
            }
        }
        float *S = p.state + ((int64_t)slot * p.n_v + h) * kHeadDim * kHeadDim;
        const int r0 = wid * kRowsPerWarp;
        float4 s[kRowsPerWarp];
#pragma unroll
        for (int i = 0; i < kRowsPerWarp; ++i)
            s[i] = __ldcs(reinterpret_cast<const float4 *>(S + (int64_t)(r0 + i) * kHeadDim + 4 * lane));
        const float a = to_f32(((const T *)p.alpha)[(int64_t)b * p.n_v + h]);
        const float be = to_f32(((const T *)p.beta)[(int64_t)b * p.n_v + h]);
        float rr[4] = {0.f, 0.f, 0.f, 0.f}, pp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < kRowsPerWarp; ++i) {
            const float kr = ks[r0 + i], qr = qs[r0 + i];
            rr[0] = fmaf(s[i].x, kr, rr[0]); rr[1] = fmaf(s[i].y, kr, rr[1]);
            rr[2] = fmaf(s[i].z, kr, rr[2]); rr[3] = fmaf(s[i].w, kr, rr[3]);
            pp[0] = fmaf(s[i].x, qr, pp[0]); pp[1] = fmaf(s[i].y, qr, pp[1]);
            pp[2] = fmaf(s[i].z, qr, pp[2]); pp[3] = fmaf(s[i].w, qr, pp[3]);
        }
        *reinterpret_cast<float4 *>(&red_r[wid][4 * lane]) = make_float4(rr[0], rr[1], rr[2], rr[3]);
        *reinterpret_cast<float4 *>(&red_p[wid][4 * lane]) = make_float4(pp[0], pp[1], pp[2], pp[3]);
        __syncthreads();
        if (tid < kHeadDim) {
            float r = 0.f, pq = 0.f;
#pragma unroll
            for (int w = 0; w < kDecWarps; ++w) { r += red_r[w][tid]; pq += red_p[w][tid]; }
            const float e = vs[tid] - a * r;
            es[tid] = e;
            outp[((int64_t)b * p.n_v + h) * kHeadDim + tid] = from_f32<TO>(a * pq + be * kq_s * e);
        }
        __syncthreads();
        const float4 e4 = *reinterpret_cast<const float4 *>(&es[4 * lane]);
#pragma unroll
        for (int i = 0; i < kRowsPerWarp; ++i) {
            const float bk = be * ks[r0 + i];
            float4 o;
            o.x = fmaf(bk, e4.x, a * s[i].x);
            o.y = fmaf(bk, e4.y, a * s[i].y);
            o.z = fmaf(bk, e4.z, a * s[i].z);
            o.w = fmaf(bk, e4.w, a * s[i].w);
            __stcs(reinterpret_cast<float4 *>(S + (int64_t)(r0 + i) * kHeadDim + 4 * lane), o);
        }
    }
}

cudaError_t launch_decode(const DecodeParams &p, bool in_bf16, bool out_bf16, cudaStream_t s) {
    if (p.batch <= 0) return cudaSuccess;
    const unsigned grid = (unsigned)((int64_t)p.batch * p.n_qk);
    TraceLaunch tl(s, "decode");
    if (in_bf16) {
        if (out_bf16) decode_kernel<gdn::bf16, gdn::bf16><<<grid, kDecThreads, 0, s>>>(p);
        else decode_kernel<gdn::bf16, float><<<grid, kDecThreads, 0, s>>>(p);
    } else {
        if (out_bf16) decode_kernel<float, gdn::bf16><<<grid, kDecThreads, 0, s>>>(p);
        else decode_kernel<float, float><<<grid, kDecThreads, 0, s>>>(p);
    }
    return cudaGetLastError();
}

}  // namespace gdn

// ---------------------------------------------------------------- multi-token decode
// n_tok consecutive tokens per row (speculative or multi-token verification): the same
// recurrence run over the row's tokens in order.  One CTA per (row, QK head) as in the
// single-token kernel, but each V head's state is held by columns (two threads per column,
// each with half of the rows; a warp holds 32 adjacent columns, so every state access is a
// whole 128-byte line) for the whole token loop: loaded once (copied into shared memory while the previous head
// is computed), advanced token by token (the reductions of token j read the state after
// token j-1) and stored once, so the state traffic of a call does not grow with n_tok.
// Optionally the state and the conv state after every token are written out, for rolling
// back to an accepted prefix.
namespace gdn {

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(smem)),
                 "l"(gmem)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

template <class T, class TO>
__global__ void __launch_bounds__(kDecThreads, 2) decode_multi_kernel(DecodeParams p) {
    // s_tile: one V head's state [128][128] fp32 (64 KB), the next head's, copied in while the
    // current one is computed; then alpha and beta of the CTA's heads [2][G][n_tok], then v of
    // every (head, token) [G][n_tok][128]
    extern __shared__ float4 s_tile4[];
    float *s_tile = reinterpret_cast<float *>(s_tile4);
    __shared__ __align__(16) float qs[kMaxDecTok][kHeadDim], ks[kMaxDecTok][kHeadDim];
    __shared__ float kq_s[kMaxDecTok];
    __shared__ __align__(16) float xr[2][2][kHeadDim], xp[2][2][kHeadDim];   // [token parity][half][column]

    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int b = blockIdx.x / p.n_qk, g = blockIdx.x % p.n_qk;
    const int G = p.n_v / p.n_qk, nt = p.n_tok;
    const int slot = p.slots ? p.slots[b] : b;
    const int qkc = p.n_qk * kHeadDim;
    const int64_t ch = 2 * (int64_t)qkc + (int64_t)p.n_v * kHeadDim;
    TO *outp = (TO *)p.out;

    if (slot < 0 || slot >= p.n_rows) {  // skipped row: zero output, touch no state
        for (int j = 0; j < nt; ++j)
            for (int e = tid; e < G * kHeadDim; e += kDecThreads)
                outp[((int64_t)b * nt + j) * p.n_v * kHeadDim + (int64_t)g * G * kHeadDim + e] = from_f32<TO>(0.f);
        return;
    }
    T *cs = p.conv ? (T *)p.conv + (int64_t)slot * 3 * ch : nullptr;
    T *cck = (T *)p.conv_ckpt;
    // the state tile of head h into s_tile, in 16-byte pieces spread over all threads
    auto prefetch = [&](int h) {
        const float *S = p.state + ((int64_t)slot * p.n_v + h) * kHeadDim * kHeadDim;
#pragma unroll 4
        for (int i = 0; i < kHeadDim * kHeadDim / 4 / kDecThreads; ++i) {
            const int c = i * kDecThreads + tid;   // 16-byte piece: row c / 32, columns 4 (c % 32) ..
            cp_async16(s_tile + 4 * c, S + 4 * c);
        }
        cp_async_commit();
    };
    prefetch(g * G);   // the first head's state, while q and k are computed
    float *ab = s_tile + kHeadDim * kHeadDim;
    float (*vs_all)[kHeadDim] = reinterpret_cast<float (*)[kHeadDim]>(ab + 2 * G * nt);   // [G * nt][128]
    for (int e = tid; e < G * nt; e += kDecThreads) {   // gates of every (head, token)
        const int hh = e / nt, j = e % nt;
        const int64_t tv = ((int64_t)b * nt + j) * p.n_v + g * G + hh;
        ab[e] = to_f32(((const T *)p.alpha)[tv]);
        ab[G * nt + e] = to_f32(((const T *)p.beta)[tv]);
    }

    // conv of one channel group over the row's tokens: history rows 0..2 from the conv state
    // (oldest first), then the tokens; writes y of token j to dst[j]; shifts the conv state
    // by nt rows and writes the checkpoints (the last 3 rows after each token)
    auto conv_tokens = [&](const T *x0, int64_t x_stride, const float *w, int wc, int cc, bool norm, float scale,
                           float (*dst)[kHeadDim]) {
        float h[3][4];
#pragma unroll
        for (int j = 0; j < 3; ++j) {
            if (cs) ld4(cs + (int64_t)j * ch + cc, h[j]);
            else h[j][0] = h[j][1] = h[j][2] = h[j][3] = 0.f;
        }
        float wt[4][4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const float4 t4 = *reinterpret_cast<const float4 *>(w + (int64_t)(wc + c) * kConvW);
            wt[c][0] = t4.x; wt[c][1] = t4.y; wt[c][2] = t4.z; wt[c][3] = t4.w;
        }
        for (int j = 0; j < nt; ++j) {
            float cur[4], y[4];
            ld4(x0 + (int64_t)j * x_stride, cur);
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
#pragma unroll
            for (int c = 0; c < 4; ++c) dst[j][4 * lane + c] = y[c];
            if (cck) {   // conv state after token j: the last three raw rows
                T *ck = cck + ((int64_t)b * nt + j) * 3 * ch + cc;
#pragma unroll
                for (int r = 0; r < 3; ++r) st4(ck + (int64_t)r * ch, h[r]);
            }
        }
        if (cs) {
#pragma unroll
            for (int r = 0; r < 3; ++r) st4(cs + (int64_t)r * ch + cc, h[r]);
        }
    };

    // ---- q and k of every token (warps 0 and 1: conv, conv-state shift, L2) and v of every
    // (head, token) (the other warps, one head each in turn)
    if (wid < 2) {
        const bool isq = wid == 0;
        const T *x = (const T *)(isq ? p.q : p.k) + ((int64_t)b * nt * p.n_qk + g) * kHeadDim + 4 * lane;
        conv_tokens(x, (int64_t)p.n_qk * kHeadDim, isq ? p.wq : p.wk, g * kHeadDim + 4 * lane,
                    (isq ? 0 : qkc) + g * kHeadDim + 4 * lane, true, isq ? p.q_scale : 1.f, isq ? qs : ks);
    } else {
        for (int hh = wid - 2; hh < G; hh += kDecWarps - 2) {
            const int h = g * G + hh;
            const T *x = (const T *)p.v + ((int64_t)b * nt * p.n_v + h) * kHeadDim + 4 * lane;
            conv_tokens(x, (int64_t)p.n_v * kHeadDim, p.wv, h * kHeadDim + 4 * lane,
                        2 * qkc + h * kHeadDim + 4 * lane, false, 1.f, vs_all + hh * nt);
        }
    }
    __syncthreads();
    if (wid < nt) {   // k.q of token wid
        float d = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) d += qs[wid][4 * lane + c] * ks[wid][4 * lane + c];
        d = warp_sum(d);
        if (lane == 0) kq_s[wid] = d;
    }

    // Thread (jc, hf) = (tid % 128, tid / 128) owns rows 64 hf .. 64 hf + 63 of state column jc:
    // the two halves of each reduction meet through a small exchange (one block barrier per
    // token, double-buffered by token parity), e and y of column jc are the thread's own, and
    // the update needs nothing from other threads.
    const int jc = tid & (kHeadDim - 1), hf = tid >> 7, rb = 64 * hf;
    for (int hh = 0; hh < G; ++hh) {
        const int h = g * G + hh;
        float (*vs)[kHeadDim] = vs_all + hh * nt;
        float *S = p.state + ((int64_t)slot * p.n_v + h) * kHeadDim * kHeadDim;
        cp_async_wait0();
        __syncthreads();   // head h's tile is in shared memory (kq_s, v and the gates are ready)
        float s[64];
#pragma unroll
        for (int r = 0; r < 64; ++r) s[r] = s_tile[(rb + r) * kHeadDim + jc];
        __syncthreads();   // every thread has its column: the tile may be refilled
        if (hh + 1 < G) prefetch(h + 1);   // overlaps the tokens of head h
        for (int j = 0; j < nt; ++j) {
            const int64_t tv = ((int64_t)b * nt + j) * p.n_v + h;
            const float a = ab[hh * nt + j], be = ab[G * nt + hh * nt + j];
            const float4 *k4 = reinterpret_cast<const float4 *>(&ks[j][rb]);
            const float4 *q4 = reinterpret_cast<const float4 *>(&qs[j][rb]);
            float r0 = 0.f, r1 = 0.f, p0 = 0.f, p1 = 0.f;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float4 kk = k4[i], qq = q4[i];
                r0 = fmaf(s[4 * i], kk.x, r0); r1 = fmaf(s[4 * i + 1], kk.y, r1);
                r0 = fmaf(s[4 * i + 2], kk.z, r0); r1 = fmaf(s[4 * i + 3], kk.w, r1);
                p0 = fmaf(s[4 * i], qq.x, p0); p1 = fmaf(s[4 * i + 1], qq.y, p1);
                p0 = fmaf(s[4 * i + 2], qq.z, p0); p1 = fmaf(s[4 * i + 3], qq.w, p1);
            }
            float r = r0 + r1, pq = p0 + p1;
            xr[j & 1][hf][jc] = r;
            xp[j & 1][hf][jc] = pq;
            __syncthreads();
            r += xr[j & 1][hf ^ 1][jc];
            pq += xp[j & 1][hf ^ 1][jc];
            const float e = vs[j][jc] - a * r;
            if (hf == 0) outp[tv * kHeadDim + jc] = from_f32<TO>(a * pq + be * kq_s[j] * e);
            const float be_e = be * e;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float4 kk = k4[i];
                s[4 * i] = fmaf(kk.x, be_e, a * s[4 * i]);
                s[4 * i + 1] = fmaf(kk.y, be_e, a * s[4 * i + 1]);
                s[4 * i + 2] = fmaf(kk.z, be_e, a * s[4 * i + 2]);
                s[4 * i + 3] = fmaf(kk.w, be_e, a * s[4 * i + 3]);
            }
            if (p.state_ckpt) {
                float *ck = p.state_ckpt + tv * kHeadDim * kHeadDim + (int64_t)rb * kHeadDim + jc;
#pragma unroll
                for (int r2 = 0; r2 < 64; ++r2) __stcs(ck + (int64_t)r2 * kHeadDim, s[r2]);
            }
        }
#pragma unroll
        for (int r = 0; r < 64; ++r) __stcs(S + (int64_t)(rb + r) * kHeadDim + jc, s[r]);
    }
}

cudaError_t launch_decode_multi(const DecodeParams &p, bool in_bf16, bool out_bf16, cudaStream_t s) {
    if (p.batch <= 0) return cudaSuccess;
    if (p.n_tok < 1 || p.n_tok > kMaxDecTok) return cudaErrorInvalidValue;
    const unsigned grid = (unsigned)((int64_t)p.batch * p.n_qk);
    const int G = p.n_v / p.n_qk;
    // one state tile + gates + v of every (head, token)
    const int kPrefetch = kHeadDim * kHeadDim * 4 + 2 * G * p.n_tok * 4 + G * p.n_tok * kHeadDim * 4;
    if (kPrefetch > 200 * 1024) return cudaErrorInvalidValue;
    auto k = in_bf16 ? (out_bf16 ? decode_multi_kernel<gdn::bf16, gdn::bf16> : decode_multi_kernel<gdn::bf16, float>)
                     : (out_bf16 ? decode_multi_kernel<float, gdn::bf16> : decode_multi_kernel<float, float>);
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kPrefetch);
    if (e != cudaSuccess) return e;
    TraceLaunch tl(s, "decode_multi");
    k<<<grid, kDecThreads, kPrefetch, s>>>(p);
    return cudaGetLastError();
}

}  // namespace gdn
