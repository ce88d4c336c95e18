// State-independent work of the chunked prefill, for every (chunk, V head) at once.
//
// For a chunk of n <= 64 tokens of one sequence and one V head h (QK head g = h / (Hv/Hqk)),
// following the chunked form of the gated delta rule of the page "ARCHITECTURE PREVIEW /
// FIELD NOTES", section 03 (GATED DELTANET), with g_t = sum_{s<=t} log alpha_s inside the
// chunk, gamma_t = exp(g_t) and kd_t = exp(g_{n-1} - g_t):
//     A_ti = beta_t exp(g_t - g_i) k_t.k_i        (i < t < n, else 0)
//     T    = (I + A)^-1,   T_beta = T diag(beta),   W2 = T_beta diag(gamma)
//     P_ti = exp(g_t - g_i) q_t.k_i               (i <= t < n, else 0)
//     K~   = diag(kd) K                            (rows t >= n zero)
// T_beta, W2 and P (64 x 64) and K~ (64 x 128) are written as fp32 tiles rounded to TF32 (the
// precision the tensor-core chain reads them in), already in the shared-memory layout of
// an MMA operand (T_beta, W2, P: K-major, 128-byte rows with 16-byte chunks XOR-swizzled by
// row; K~: MN-major with 32-byte granules, like the V tile), for the chain kernel to stream in with one bulk
// copy each.  A gates record per (chunk, head) carries gamma_t, kd_t and gamma_C = exp(g_{n-1}).
//
// One CTA per (chunk, V head), 256 threads, about 70 KB of shared memory (three CTAs per
// SM): one bulk copy brings the chunk's [K;Q] tile, one tcgen05 MMA forms [K;Q] K^T in
// tensor memory while the warps write K~, the warps turn K K^T and Q K^T into A and P, and
// the inverse runs on CUDA cores in fp32 (16 x 16 diagonal blocks by forward substitution,
// then two block-merge levels).  The [K;Q] tile's space is reused for the scratch and the
// output staging; the tiles leave by bulk stores.
#include "gdn_common.cuh"
#include "gdn_internal.h"
#include "tc_sm100.cuh"

namespace gdn {

namespace {
using namespace tc;

constexpr int kPThr = 256;

// shared-memory map (bytes from a 1024-aligned base).  [0, 64 KB) first holds the [K;Q]
// tile; once the MMA has read it and K~ has been written, it holds the scratch and staging.
constexpr uint32_t P_KQ = 0;          // [K;Q] K-major, 4 blocks x (K 8 KB | Q 8 KB)   64 KB
constexpr uint32_t P_AS = 0;          // A (fp32, swizzled rows), then the W2 staging   16 KB
constexpr uint32_t P_TS = 16384;      // T (fp32, swizzled rows)                       16 KB
constexpr uint32_t P_PST = 32768;     // P staging (K-major image)                     16 KB
constexpr uint32_t P_TBST = 49152;    // T_beta staging (K-major image)                16 KB
constexpr uint32_t P_INV = 65536;     // 2 x 256 floats (block products)                2 KB
constexpr uint32_t P_GATE = 67584;    // g, beta, gamma, kd, 1/gamma: 5 x 64 floats    1280 B
constexpr uint32_t P_BAR = 68864;     // 2 mbarriers
constexpr uint32_t P_SLOT = 68880;    // TMEM base
constexpr uint32_t kPSmem = P_SLOT + 16;
constexpr uint32_t kPSmemAlloc = kPSmem + 1024;
constexpr uint32_t kPTmemCols = 64;
constexpr uint32_t kPWaitTries = 1u << 24;
constexpr float kMaxChunkDecay = 80.f;  // factor exp(g_t - g_i) = gamma_t / gamma_i below this

// fp32 scratch [64][64] with 16-byte chunks XOR-swizzled by row
__device__ __forceinline__ int scr(int r, int c) { return r * 64 + ((((c >> 2) ^ (r & 7)) << 2) | (c & 3)); }

__device__ __forceinline__ float4 tf32x4(float4 x) {
    return make_float4(to_tf32(x.x), to_tf32(x.y), to_tf32(x.z), to_tf32(x.w));
}

// contiguous bulk copy shared (this CTA) -> global, tracked as a bulk async-group
__device__ __forceinline__ void bulk_store(void *dst, uint32_t src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src), "r"(bytes)
                 : "memory");
}

struct PrepParams {
    const float *kq;      // [chunk, Hqk] [K;Q] tiles (64 KB each)
    float *kt;            // [chunk, Hv] K~ tiles (32 KB each)
    const void *alpha, *beta;
    const int32_t *cu, *cfirst;
    float *tb, *w2, *pm;  // [chunk, Hv] tiles (16 KB each)
    float *gr;            // [chunk, Hv] gates records
    int n_seqs, n_qk, n_v;
    int64_t chunk_lo;     // first global chunk index of this launch
};

}  // namespace

template <class TI>
__global__ void __launch_bounds__(kPThr) chunk_prep_kernel(const __grid_constant__ PrepParams p) {
    const int h = blockIdx.x % p.n_v;
    const int u = (int)(p.chunk_lo + blockIdx.x / p.n_v);   // global chunk index
    if (u >= p.cfirst[p.n_seqs]) return;               // uniform per CTA
    const int b = upper_index(p.cfirst, p.n_seqs, u);
    const int seq0 = p.cu[b];
    const int r0 = (u - p.cfirst[b]) * kChunk;
    const int n = min(kChunk, p.cu[b + 1] - seq0 - r0);
    const int tok = seq0 + r0;
    const int gq = h / (p.n_v / p.n_qk);

    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    const uint32_t sb = smem_u32(sm);
    uint64_t *bar = (uint64_t *)(sm + P_BAR);
    uint32_t *tslot = (uint32_t *)(sm + P_SLOT);
    float *g_s = (float *)(sm + P_GATE), *beta_s = g_s + 64, *gam_s = g_s + 128, *kd_s = g_s + 192,
          *ig_s = g_s + 256;
    float *Ascr = (float *)(sm + P_AS), *Tscr = (float *)(sm + P_TS), *inv_s = (float *)(sm + P_INV);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t tile = (int64_t)u * p.n_v + h;
    float *gr = p.gr + tile * kGateRec;

    if (tid == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        mbar_expect_tx(&bar[0], 65536);
        bulk_load(sb + P_KQ, p.kq + ((int64_t)u * p.n_qk + gq) * 16384, 65536, &bar[0]);
    }
    if (warp == 0) {
        tmem_alloc(tslot, kPTmemCols);
        tmem_relinquish();
    }
    // gates of the chunk: log alpha and beta, zero past n
    if (tid < kChunk) {
        const TI *al = (const TI *)p.alpha, *be = (const TI *)p.beta;
        const int64_t e = (int64_t)(tok + tid) * p.n_v + h;
        g_s[tid] = tid < n ? safe_log_alpha(to_f32(al[e])) : 0.f;
        beta_s[tid] = tid < n ? to_f32(be[e]) : 0.f;
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tm = *tslot;

    // [K;Q] K^T (M=128: rows 0-63 K K^T, rows 64-127 Q K^T; N=64) into tensor memory
    bool ok = true;
    if (tid == 0) {
        ok = mbar_wait(&bar[0], 0, kPWaitTries);
        if (ok) {
            fence_after_sync();
            gemm<128, 64, 128, false, false>(tm, sb + P_KQ, 16384, sb + P_KQ, 16384, false);
            mma_commit(&bar[1]);
        }
    }
    if (warp == 1) {  // gates: inclusive scan of log alpha, two rows per lane (meanwhile)
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
        g_s[t0] = g0;
        g_s[t1] = g1;
        const float gam0 = expf(g0), gam1 = expf(g1);
        gam_s[t0] = gam0;
        gam_s[t1] = gam1;
        ig_s[t0] = expf(-g0);      // used only when the chunk's decay stays below kMaxChunkDecay
        ig_s[t1] = expf(-g1);
        const float kd0 = t0 < n ? expf(glast - g0) : 0.f, kd1 = t1 < n ? expf(glast - g1) : 0.f;
        kd_s[t0] = kd0;
        kd_s[t1] = kd1;
        gr[kGrGamma + t0] = gam0;
        gr[kGrGamma + t1] = gam1;
        gr[kGrKd + t0] = kd0;
        gr[kGrKd + t1] = kd1;
        if (lane == 0) gr[kGrGammaC] = expf(glast);
    }
    if (__syncthreads_or(!ok)) {  // also publishes the gates and the arrived [K;Q] tile
        if (tid == 0) mbar_wait(&bar[0], 0, kPWaitTries);  // drain the copy
        ok = false;
    }
    // K~ = diag(kd) K from the K-major K tile, written in the MN-major layout (coalesced)
    {
        float4 *dst = reinterpret_cast<float4 *>(p.kt + tile * 8192);
        const float nan = __int_as_float(0x7fc00000);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int i4 = tid + kPThr * k;                       // float4 of the MN-major tile
            const int o = 4 * i4, blk = o >> 11, t = (o >> 5) & 63, w = o & 31;
            const int dl = 8 * ((w >> 3) ^ (t & 3)) + (w & 4);    // its first feature in the block
            float4 x = *reinterpret_cast<const float4 *>(sm + P_KQ + blk * 16384 + t * 128 +
                                                         ((((dl >> 2) ^ (t & 7))) << 4));
            const float sc = ok ? kd_s[t] : nan;
            dst[i4] = tf32x4(make_float4(x.x * sc, x.y * sc, x.z * sc, x.w * sc));
        }
    }
    if (ok) ok = tid == 0 ? mbar_wait(&bar[1], 0, kPWaitTries) : true;
    ok = !__syncthreads_or(!ok);  // the MMA is done and K~ has read the K tile
    fence_after_sync();
    if (ok) {
        // A (fp32 scratch) from the K K^T rows, P (TF32, staged as a K-major image) from the
        // Q K^T rows.  exp(g_t - g_i) = gamma_t / gamma_i while the chunk's total decay keeps
        // 1 / gamma finite; otherwise one exponential per element.
        const int q = warp & 3, ch = warp >> 2;
        float v[32];
        tmem_ld32(taddr(tm, 32 * q, 32 * ch), v);
        tmem_wait_ld();
        const int t = 32 * (q & 1) + lane;
        const bool factored = -g_s[n - 1] < kMaxChunkDecay;
        const float gt = g_s[t], rowf = gam_s[t] * (q < 2 ? beta_s[t] : 1.f), bt = q < 2 ? beta_s[t] : 1.f;
        float out[32];
        const int lim = t < n ? (q < 2 ? t : t + 1) : 0;   // columns i < lim are kept
        if (factored) {   // uniform per CTA
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const int i = 32 * ch + e;
                out[e] = i < lim ? rowf * ig_s[i] * v[e] : 0.f;
            }
        } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const int i = 32 * ch + e;
                out[e] = i < lim ? bt * expf(gt - g_s[i]) * v[e] : 0.f;
            }
        }
        if (q < 2) {
#pragma unroll
            for (int k = 0; k < 8; ++k)
                *reinterpret_cast<float4 *>(&Ascr[scr(t, 32 * ch + 4 * k)]) =
                    make_float4(out[4 * k], out[4 * k + 1], out[4 * k + 2], out[4 * k + 3]);
        } else {
#pragma unroll
            for (int k = 0; k < 8; ++k)
                *reinterpret_cast<float4 *>(sm + P_PST + kmaj_off(t, 32 * ch + 4 * k, 64)) =
                    tf32x4(make_float4(out[4 * k], out[4 * k + 1], out[4 * k + 2], out[4 * k + 3]));
        }
        fence_smem_to_async();
    }
    fence_before_sync();
    __syncthreads();
    if (ok && tid == 0) bulk_store(p.pm + tile * 4096, sb + P_PST, 16384);
    if (ok) {
        // ---- T = (I + A)^-1.  Diagonal 16 x 16 blocks: column cc of block bb by forward
        // substitution with right-looking updates; the other threads clear the two blocks
        // above the diagonal that the merge products read.
        if (tid < 64) {
            const int bb = tid >> 4, cc = tid & 15, o = 16 * bb;
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
        } else {
            for (int e = tid - 64; e < 512; e += kPThr - 64) {
                const int blk = e >> 8, r = (e >> 4) & 15, cc = e & 15, o = 32 * blk;
                Tscr[scr(o + r, o + 16 + cc)] = 0.f;
            }
        }
        __syncthreads();
        if (tid < 128) {  // 32 x 32 halves: M = A_10 T_00
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
        if (tid < 128) {  // T_10 = -T_11 M
            const int hh = tid >> 6, rr = (tid >> 2) & 15, c4 = (tid & 3) * 4, o = 32 * hh;
            float a4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int m = 0; m < 16; ++m) {
                const float tv = Tscr[scr(o + 16 + rr, o + 16 + m)];
                const float4 m4 = *reinterpret_cast<const float4 *>(&inv_s[hh * 256 + m * 16 + c4]);
                a4[0] = fmaf(tv, m4.x, a4[0]); a4[1] = fmaf(tv, m4.y, a4[1]);
                a4[2] = fmaf(tv, m4.z, a4[2]); a4[3] = fmaf(tv, m4.w, a4[3]);
            }
            *reinterpret_cast<float4 *>(&Tscr[scr(o + 16 + rr, o + c4)]) = make_float4(-a4[0], -a4[1], -a4[2], -a4[3]);
        }
        __syncthreads();
        {  // merge: M = A_bl T_top, parked in the (otherwise unused) upper-right block
            const int r = tid >> 3, c4 = (tid & 7) * 4;
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
        __syncthreads();
        {  // T_bl = -T_br M
            const int r = tid >> 3, c4 = (tid & 7) * 4;
            float a4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int m = 0; m < 32; ++m) {
                const float tv = Tscr[scr(32 + r, 32 + m)];
                const float4 m4 = *reinterpret_cast<const float4 *>(&Tscr[scr(m, 32 + c4)]);
                a4[0] = fmaf(tv, m4.x, a4[0]); a4[1] = fmaf(tv, m4.y, a4[1]);
                a4[2] = fmaf(tv, m4.z, a4[2]); a4[3] = fmaf(tv, m4.w, a4[3]);
            }
            *reinterpret_cast<float4 *>(&Tscr[scr(32 + r, c4)]) = make_float4(-a4[0], -a4[1], -a4[2], -a4[3]);
        }
        __syncthreads();
    }
    {  // T_beta = T diag(beta) and W2 = T_beta diag(gamma), staged (the upper-right block of
       // T is zero; W2 reuses the A scratch, dead since the merge); NaN if the CTA failed
        const int t = tid >> 2, i0 = (tid & 3) * 16;
        const bool upper_right = t < 32 && i0 >= 32;
        const float nan = __int_as_float(0x7fc00000);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int i = i0 + 4 * k;
            float4 x = *reinterpret_cast<const float4 *>(&Tscr[scr(t, i)]);
            if (upper_right) x = make_float4(0.f, 0.f, 0.f, 0.f);
            x = make_float4(x.x * beta_s[i], x.y * beta_s[i + 1], x.z * beta_s[i + 2], x.w * beta_s[i + 3]);
            if (!ok) x = make_float4(nan, nan, nan, nan);
            const float4 w = make_float4(x.x * gam_s[i], x.y * gam_s[i + 1], x.z * gam_s[i + 2], x.w * gam_s[i + 3]);
            *reinterpret_cast<float4 *>(sm + P_TBST + kmaj_off(t, i, 64)) = tf32x4(x);
            *reinterpret_cast<float4 *>(sm + P_AS + kmaj_off(t, i, 64)) = tf32x4(w);
        }
        fence_smem_to_async();
    }
    fence_before_sync();
    __syncthreads();
    if (tid == 0) {
        bulk_store(p.tb + tile * 4096, sb + P_TBST, 16384);
        bulk_store(p.w2 + tile * 4096, sb + P_AS, 16384);
        bulk_commit();
        bulk_wait0();   // the stores are complete before the CTA's shared memory goes away
    }
    __syncthreads();
    if (warp == 0) tmem_dealloc(tm, kPTmemCols);
}

cudaError_t launch_chunk_prep(const ScanParams &sp, int64_t total_tokens, bool in_bf16, cudaStream_t s) {
    if (sp.n_seqs <= 0 || total_tokens <= 0) return cudaSuccess;
    PrepParams p{};
    p.kq = sp.kq; p.kt = sp.kt;
    p.alpha = sp.alpha; p.beta = sp.beta; p.cu = sp.cu; p.cfirst = sp.cfirst;
    p.tb = sp.tb; p.w2 = sp.w2; p.pm = sp.pm; p.gr = sp.gr; p.n_seqs = sp.n_seqs; p.n_qk = sp.n_qk; p.n_v = sp.n_v;
    p.chunk_lo = sp.chunk_lo;
    const int64_t grid = (sp.chunk_hi - sp.chunk_lo) * sp.n_v;
    if (grid <= 0) return cudaSuccess;
    if (grid >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
    auto k = in_bf16 ? chunk_prep_kernel<bf16> : chunk_prep_kernel<float>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kPSmemAlloc);
    if (e != cudaSuccess) return e;
    TraceLaunch tl(s, "chunk_prep");
    k<<<(unsigned)grid, kPThr, kPSmemAlloc, s>>>(p);
    return cudaGetLastError();
}

}  // namespace gdn
