// QSA indexer: block keys, block scores and the top-512 block selection.
//
// Page "ARCHITECTURE PREVIEW / FIELD NOTES", section 03, the QSA indexer figure (BLOCK
// SCORE, CAUSAL SPARSE SET) and the five-step "QSA" list; section 01 for the shapes (4
// query heads over 1 shared key head, head dim 128, 512 blocks of 4 tokens).
//
//   qsa_block_keys_kernel   warp per block: mean of 4 key rows, RMSNorm, rotary encoding at
//                           the block's first token, bf16 into the block-key cache
//   qsa_scores_kernel       CTA per (row, 4..64 queries, share of the block range): the
//                           query heads are normalised and rotated into shared memory once;
//                           128-block key tiles stream in by TMA; one kind::f16 MMA chain per
//                           tile gives every (block, query head) dot product in tensor
//                           memory; the epilogue sums the ReLUs of the 4 heads and stores the
//                           fp32 scores, query-major
//   qsa_topk_kernel         CTA per query: the 512th largest score by a 3-digit radix select
//                           (11 + 10 + 10 bits of the non-negative score's bit pattern) over
//                           a sampled candidate set, then the selected blocks in ascending
//                           order (equal scores: lower index first) and the tokens
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include <algorithm>
#include <cmath>

#include "gdn_internal.h"
#include "tc_sm100.cuh"
#include "tma_map.cuh"

namespace gdn {
namespace qsa {

using namespace tc;

constexpr int kR = 4;                       // tokens per block
constexpr int kD = 128;                     // indexer head dim
constexpr int kHeads = 4;                   // indexer query heads
constexpr int kKB = 512;                    // block budget
constexpr int kTok = kR * kKB + kR - 1;     // token-set slots per query
constexpr uint32_t kWaitTries = 1u << 22;

// ------------------------------------------------------------------ shared pieces
__device__ __forceinline__ double inv_freq(int d, double log2_theta) {
    return exp2(-(double)d * (log2_theta / 32.0));
}
// cos and sin of pos * f: the angle is formed and reduced to [-pi, pi] in fp64, where the
// hardware sine/cosine is within about 2^-21 (far below the bf16 rounding that follows)
__device__ __forceinline__ void rope_cs(int64_t pos, double f, float &c, float &s) {
    const double two_pi = 6.283185307179586;
    const double a = (double)pos * f;
    const double n = rint(a * (1.0 / two_pi));
    __sincosf((float)fma(-n, two_pi, a), &s, &c);
}
__device__ __forceinline__ void unpack4(uint2 u, float (&x)[4]) {
    x[0] = __uint_as_float(u.x << 16);
    x[1] = __uint_as_float(u.x & 0xFFFF0000u);
    x[2] = __uint_as_float(u.y << 16);
    x[3] = __uint_as_float(u.y & 0xFFFF0000u);
}
__device__ __forceinline__ uint2 pack4(const float (&x)[4]) {
    __nv_bfloat162 a = __floats2bfloat162_rn(x[0], x[1]), b = __floats2bfloat162_rn(x[2], x[3]);
    return make_uint2(*reinterpret_cast<uint32_t *>(&a), *reinterpret_cast<uint32_t *>(&b));
}
// RMSNorm * w, then the rotary encoding, of one 128-dim row held by a warp, 4 dims per lane
// (lane l: dims 4l..4l+3).  c, s: this lane's 4 cos/sin (lanes 0..15; dims d and d + 32 of
// a pair sit in lanes l and l + 8).
__device__ __forceinline__ void norm_rope_row(float (&x)[4], const float4 w, float eps,
                                              const float (&c)[4], const float (&s)[4], int lane) {
    float ss = x[0] * x[0] + x[1] * x[1] + x[2] * x[2] + x[3] * x[3];
#pragma unroll
    for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float r = rsqrtf(ss * (1.f / kD) + eps);
    x[0] *= r * w.x;
    x[1] *= r * w.y;
    x[2] *= r * w.z;
    x[3] *= r * w.w;
    float o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) o[e] = __shfl_xor_sync(0xffffffffu, x[e], 8);
    if (lane < 8) {
#pragma unroll
        for (int e = 0; e < 4; ++e) x[e] = x[e] * c[e] - o[e] * s[e];
    } else if (lane < 16) {
#pragma unroll
        for (int e = 0; e < 4; ++e) x[e] = x[e] * c[e] + o[e] * s[e];
    }
}
// candidate blocks of a query at position pos: complete blocks, capped by the valid cache
__device__ __forceinline__ int64_t n_cand(int64_t pos, int64_t cap) {
    return pos < 0 ? 0 : min((pos + 1) >> 2, cap);
}

// ------------------------------------------------------------------ block keys
struct KeyParams {
    const __nv_bfloat16 *k;
    const float *w;
    const int32_t *kpos;
    __nv_bfloat16 *kbar;
    int B, Tn, nb_max;
    float eps, theta;
};

__global__ void __launch_bounds__(256) qsa_block_keys_kernel(const __grid_constant__ KeyParams p) {
    const int lane = threadIdx.x & 31;
    const int nbj = p.Tn / kR;
    const int64_t gw = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (gw >= (int64_t)p.B * nbj) return;                  // whole warps leave together
    const int b = (int)(gw / nbj), j = (int)(gw % nbj);
    const int kp = p.kpos[b];
    if (kp < 0 || (kp & 3)) return;
    const int64_t blk = (int64_t)(kp >> 2) + j;
    if (blk >= p.nb_max) return;
    const uint2 *src = reinterpret_cast<const uint2 *>(p.k + ((int64_t)b * p.Tn + (int64_t)j * kR) * kD) + lane;
    float x[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int t = 0; t < kR; ++t) {
        float r[4];
        unpack4(__ldg(src + t * (kD / 4)), r);
#pragma unroll
        for (int e = 0; e < 4; ++e) x[e] += r[e];
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) x[e] *= 1.f / kR;
    float c[4] = {1.f, 1.f, 1.f, 1.f}, s[4] = {0.f, 0.f, 0.f, 0.f};
    if (lane < 16) {
        const double l2t = log2((double)p.theta);
#pragma unroll
        for (int e = 0; e < 4; ++e) rope_cs(kR * blk, inv_freq(4 * (lane & 7) + e, l2t), c[e], s[e]);
    }
    const float4 w = __ldg(reinterpret_cast<const float4 *>(p.w) + lane);
    norm_rope_row(x, w, p.eps, c, s, lane);
    reinterpret_cast<uint2 *>(p.kbar + ((int64_t)b * p.nb_max + blk) * kD)[lane] = pack4(x);
}

// ------------------------------------------------------------------ block scores
constexpr int kStages = 4;
constexpr uint32_t kTileBytes = 128 * kD * 2;      // 128 blocks x 128 dims, bf16
constexpr uint32_t kHalf = kTileBytes / 2;         // one 64-dim column block (128-byte rows)
constexpr uint32_t OFF_Q = 0;                      // query heads: <= 256 rows x 256 B
constexpr uint32_t OFF_K = 65536;                  // key tiles, kStages deep
constexpr uint32_t OFF_BAR = OFF_K + kStages * kTileBytes;
enum { BAR_FULL = 0, BAR_EMPTY = kStages, BAR_TFULL = 2 * kStages, BAR_TEMPTY = 2 * kStages + 2,
       BAR_Q = 2 * kStages + 4, kNumBars };
constexpr uint32_t OFF_FLAG = OFF_BAR + 8 * 16;    // TMEM base, abort flag
constexpr uint32_t kScoreSmem = OFF_FLAG + 16;
// Warps: n_epi epilogue warps (4 per group of 16-column chunks, up to 4 groups: one warp
// per TMEM lane quadrant in each), then the producer, then the MMA issuer; the launch picks
// n_epi = 4 min(4, N / 16).
constexpr int kMaxEpiWarps = 16;
constexpr int kScoreThrMax = 32 * (kMaxEpiWarps + 2);
constexpr int kMaxQT = 64;                         // queries per CTA (N = 4 x 64 = 256)

struct ScoreParams {
    CUtensorMap tm_kbar;        // kbar as [B * nb_max, 128] bf16 rows, boxes 64 x 128, 128B swizzle
    const __nv_bfloat16 *q;
    const float *w;
    const int32_t *qpos, *n_blocks;
    float *scores;
    int64_t ld;                 // row stride of scores (>= nb_max)
    int B, Qn, nb_max, qt, n_split;
    float eps, theta;
};

__device__ __forceinline__ void arrive(uint64_t *m) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(m)) : "memory");
}
// bounded wait that gives up early once another role has raised the abort flag
__device__ __forceinline__ bool wait_abort(uint64_t *m, uint32_t par, volatile int *abort_flag) {
    if (mbar_try_wait(m, par)) return true;
    for (uint32_t i = 0; i < kWaitTries; ++i) {
        if (mbar_try_wait_sleep(m, par, 40)) return true;
        if ((i & 63) == 63 && *abort_flag) return false;
    }
    *abort_flag = 1;
    return false;
}

__global__ void __launch_bounds__(kScoreThrMax, 1) qsa_scores_kernel(const __grid_constant__ ScoreParams p) {
    extern __shared__ __align__(1024) unsigned char sm[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_epi = (int)(blockDim.x >> 5) - 2, kLoadWarp = n_epi, kMmaWarp = n_epi + 1;
    const int b = blockIdx.y, q0 = blockIdx.x * p.qt;
    const int nq = min(p.qt, p.Qn - q0);
    const int N = kHeads * p.qt;                               // MMA N: (query, head) rows
    const int64_t pos0 = p.qpos[b];
    const int64_t cap = max(0, min(p.n_blocks[b], p.nb_max));
    const int64_t ncand = n_cand(pos0 + q0 + nq - 1, cap);     // the tile's last query sees most
    const int ntiles = (int)((ncand + 127) / 128);
    const int per = (ntiles + p.n_split - 1) / p.n_split;
    const int t0 = blockIdx.z * per, t1 = min(ntiles, t0 + per);
    if (t0 >= t1) return;                                      // uniform per CTA
    const int nt = t1 - t0;

    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + OFF_FLAG);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + OFF_FLAG + 4);
    uint32_t tcols = 32;
    while (tcols < 2u * (uint32_t)N) tcols <<= 1;

    if (threadIdx.x == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(&p.tm_kbar) : "memory");
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bar[BAR_FULL + s], 1);
            mbar_init(&bar[BAR_EMPTY + s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bar[BAR_TFULL + i], 1);
            mbar_init(&bar[BAR_TEMPTY + i], 32 * n_epi);
        }
        mbar_init(&bar[BAR_Q], 32 * n_epi);
        *abort_flag = 0;
    }
    if (warp == kMmaWarp) {
        tmem_alloc(tslot, tcols);
        tmem_relinquish();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tslot;

    if (warp == kLoadWarp) {
        // ================================================================ producer
        if (lane == 0) {
            int issued = 0;
            bool ok = true;
            for (int it = 0; it < nt; ++it) {
                const int s = it % kStages;
                if (it >= kStages && !(ok = wait_abort(&bar[BAR_EMPTY + s], (uint32_t)((it / kStages) - 1) & 1, abort_flag)))
                    break;
                const uint32_t dst = smem_u32(sm + OFF_K + s * kTileBytes);
                const int y = b * p.nb_max + (t0 + it) * 128;
                mbar_expect_tx(&bar[BAR_FULL + s], kTileBytes);
                tma_load_2d(dst, &p.tm_kbar, 0, y, &bar[BAR_FULL + s]);
                tma_load_2d(dst + kHalf, &p.tm_kbar, 64, y, &bar[BAR_FULL + s]);
                ++issued;
            }
            if (!ok)  // wait (bounded) for the copies still in flight
                for (int it = max(0, issued - kStages); it < issued; ++it)
                    mbar_wait(&bar[BAR_FULL + it % kStages], (uint32_t)(it / kStages) & 1, kWaitTries);
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ================================================================ MMA issuer
        if (lane == 0) {
            const uint32_t id = idesc_bf16(128, N);
            const uint32_t qb = smem_u32(sm + OFF_Q);
            const uint64_t b0 = desc_kmajor(qb, (uint32_t)N * 128, 0);
            const uint32_t b_blk16 = ((uint32_t)N * 128) >> 4;
            int issued = 0;
            bool ok = wait_abort(&bar[BAR_Q], 0, abort_flag);
            for (int it = 0; ok && it < nt; ++it) {
                const int s = it % kStages, buf = it & 1;
                if (!(ok = wait_abort(&bar[BAR_FULL + s], (uint32_t)(it / kStages) & 1, abort_flag))) break;
                if (it >= 2 && !(ok = wait_abort(&bar[BAR_TEMPTY + buf], (uint32_t)((it >> 1) - 1) & 1, abort_flag))) break;
                fence_after_sync();
                const uint64_t a0 = desc_kmajor(smem_u32(sm + OFF_K + s * kTileBytes), kHalf, 0);
#pragma unroll
                for (int st = 0; st < kD / 16; ++st) {
                    const uint32_t da = (uint32_t)(st >> 2) * (kHalf >> 4) + (uint32_t)(st & 3) * 2;
                    const uint32_t db = (uint32_t)(st >> 2) * b_blk16 + (uint32_t)(st & 3) * 2;
                    mma_bf16(tmem + (uint32_t)(buf * N), a0 + da, b0 + db, id, st > 0 ? 1u : 0u);
                }
                mma_commit(&bar[BAR_EMPTY + s]);
                mma_commit(&bar[BAR_TFULL + buf]);
                ++issued;
            }
            // the tensor memory is released only after the last issued MMAs have completed
            if (issued) mbar_wait(&bar[BAR_TFULL + ((issued - 1) & 1)], (uint32_t)((issued - 1) >> 1) & 1, kWaitTries);
        }
        __syncwarp();
    } else {
        // ================================================================ epilogue
        // 1. the CTA's query heads, normalised and rotated, as the MMA's B operand (K-major,
        //    128-byte swizzle: row n = 4 query + head, two 64-dim column blocks)
        {
            double f[4];
            const double l2t = log2((double)p.theta);
#pragma unroll
            for (int e = 0; e < 4; ++e) f[e] = inv_freq(4 * (lane & 7) + e, l2t);
            const float4 w = __ldg(reinterpret_cast<const float4 *>(p.w) + lane);
            const int d = 4 * lane;
            for (int qi = warp; qi < p.qt; qi += n_epi) {
                const bool live = qi < nq;
                float c[4] = {1.f, 1.f, 1.f, 1.f}, s[4] = {0.f, 0.f, 0.f, 0.f};
                if (live && lane < 16) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) rope_cs(pos0 + q0 + qi, f[e], c[e], s[e]);
                }
                const uint2 *src = reinterpret_cast<const uint2 *>(p.q + ((int64_t)b * p.Qn + q0 + qi) * kHeads * kD) + lane;
#pragma unroll
                for (int h = 0; h < kHeads; ++h) {
                    const int n = kHeads * qi + h;
                    float x[4] = {0.f, 0.f, 0.f, 0.f};
                    if (live) {
                        unpack4(__ldg(src + h * (kD / 4)), x);
                        norm_rope_row(x, w, p.eps, c, s, lane);
                    }
                    const uint32_t off = (uint32_t)(d >> 6) * (uint32_t)(N * 128) + (uint32_t)n * 128 +
                                         ((((uint32_t)(d & 63) >> 3) ^ (uint32_t)(n & 7)) << 4) + ((uint32_t)(d & 7) << 1);
                    *reinterpret_cast<uint2 *>(sm + OFF_Q + off) = pack4(x);
                }
            }
            fence_smem_to_async();
            arrive(&bar[BAR_Q]);
        }
        // 2. per key tile: sum over heads of ReLU(dot), one fp32 score per (query, block).
        //    Warp w reads TMEM lanes 32 (w % 4) .. (its 32 blocks) and one quarter of the
        //    16-column chunks (4 queries each).
        const int qd = warp & 3, part = warp >> 2;
        const uint32_t lrow = (uint32_t)(32 * qd) << 16;
        const int nch = N / 16, nparts = n_epi / 4, share = (nch + nparts - 1) / nparts;
        const int c0 = min(nch, part * share), c1 = min(nch, c0 + share);
        bool ok = true;
        for (int it = 0; it < nt; ++it) {
            const int buf = it & 1;
            const int blk = (t0 + it) * 128 + 32 * qd + lane;
            const bool in = blk < p.nb_max;
            float *dst = p.scores + ((int64_t)b * p.Qn + q0) * p.ld + blk;
            if (ok) ok = wait_abort(&bar[BAR_TFULL + buf], (uint32_t)(it >> 1) & 1, abort_flag);
            if (!ok) {   // leave NaN where this tile's scores belong
                if (in)
                    for (int qi = 4 * c0; qi < min(nq, 4 * c1); ++qi) dst[(int64_t)qi * p.ld] = __int_as_float(0x7fc00000);
                continue;
            }
            fence_after_sync();
            float *dq = dst + (int64_t)(4 * c0) * p.ld;
            // up to 2 loads of 16 columns (8 queries) in flight per wait
            for (int c = c0; c < c1; c += 2) {
                const int g = min(2, c1 - c);                // warp-uniform
                float v[2][16];
#pragma unroll
                for (int u = 0; u < 2; ++u)
                    if (u < g) tmem_ld16(tmem + lrow + (uint32_t)(buf * N + 16 * (c + u)), v[u]);
                tmem_wait_ld();
                tmem_regs_after_wait(v[0]);
                if (g > 1) tmem_regs_after_wait(v[1]);
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    if (u >= g) break;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int qi = 4 * (c + u) + j;
                        float sc = 0.f;
#pragma unroll
                        for (int h = 0; h < kHeads; ++h) {
                            const float t = v[u][kHeads * j + h];
                            sc += t > 0.f ? t : 0.f;
                        }
                        if (in && qi < nq) __stcs(dq, sc);
                        dq += p.ld;
                    }
                }
            }
            fence_before_sync();
            arrive(&bar[BAR_TEMPTY + buf]);
        }
    }

    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (warp == kMmaWarp) tmem_dealloc(tmem, tcols);
}

// ------------------------------------------------------------------ top-512 selection
// Per query: the 512th largest score is found exactly by a radix select on a candidate set:
// a strided sample (1 element in 17) sets a threshold that the top ~1200 scores clear
// (expected; at least 512 with a margin of about 5 standard deviations), one coalesced pass
// collects the scores above it, and the radix select runs over those only.  Bitmaps of the
// selected and of the equal-to-threshold blocks then give the ascending output, equal
// scores taken from the lowest block index up.  When the candidate set misses the budget or
// overflows (ties, unusual distributions), the row falls back to the radix select over all
// of its scores; both paths give the same result.
constexpr int kTopThr = 512;
constexpr int kTopWarps = kTopThr / 32;
constexpr int kHist = 2048;
constexpr int kCandCap = 4096;     // candidate keys kept in shared memory
constexpr int kSampleStride = 17;  // odd: the strided sample reads distinct banks
constexpr int kSampleMargin = 40;  // extra sample ranks above the budget's share

struct TopkParams {
    const float *scores;        // rows of stride ld (a multiple of 4, 16-byte aligned rows)
    const int32_t *qpos, *n_blocks;
    int32_t *blocks, *tokens;
    int64_t ld;
    int B, Qn, nb_max;
};

constexpr int kBinsPerThr = kHist / kTopThr;

// exclusive prefix sum over the CTA's threads (sw: one int per warp of scratch)
__device__ __forceinline__ int excl_scan_cta(int x, int *sw) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int v = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += y;
    }
    if (lane == 31) sw[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int t = lane < kTopWarps ? sw[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, t, o);
            if (lane >= o) t += y;
        }
        if (lane < kTopWarps) sw[lane] = t;
    }
    __syncthreads();
    const int before = (warp ? sw[warp - 1] : 0) + v - x;
    __syncthreads();
    return before;
}

// The k-th largest of n keys (k <= n) by radix digits of 11, 10 and 10 bits of a
// non-negative float's bit pattern; also returns how many keys equal to it rank within the
// k (kk).  With passes < 3 the result is the lower edge of the k-th largest key's 11- or
// 21-bit prefix (a lower bound; kk is then not meaningful).  Called by all threads of the CTA.
__device__ uint32_t radix_select(const uint32_t *keys, int n, int k, int *hist, int *sw, int *sel, int &kk,
                                 int passes = 3) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint32_t hi = 0;
    kk = k;
#pragma unroll 1
    for (int pass = 0; pass < passes; ++pass) {
        const int shift = pass == 0 ? 20 : pass == 1 ? 10 : 0;
        const int width = pass == 0 ? 11 : 10;
        const int nbins = 1 << width;
        for (int i = tid; i < nbins; i += kTopThr) hist[i] = 0;
        __syncthreads();
        for (int base = warp * 32; base < n; base += kTopThr) {
            const int e = base + lane;
            uint32_t dg = 0xFFFFFFFFu;
            if (e < n) {
                const uint32_t key = keys[e];
                if ((key >> (shift + width)) == hi) dg = (key >> shift) & (uint32_t)(nbins - 1);
            }
            const uint32_t m = __match_any_sync(0xffffffffu, dg);
            if (dg != 0xFFFFFFFFu && lane == __ffs(m) - 1) atomicAdd(&hist[dg], __popc(m));
        }
        __syncthreads();
        // bins from the top: thread t holds bins nbins-1-kB t .. nbins-kB(t+1) (kB = kBinsPerThr)
        int loc[kBinsPerThr], sum = 0;
#pragma unroll
        for (int j = 0; j < kBinsPerThr; ++j) {
            const int bin = nbins - 1 - kBinsPerThr * tid - j;
            loc[j] = bin >= 0 ? hist[bin] : 0;
            sum += loc[j];
        }
        const int before = excl_scan_cta(sum, sw);
        if (before < kk && kk <= before + sum) {
            int cum = before;
#pragma unroll
            for (int j = 0; j < kBinsPerThr; ++j) {
                if (cum + loc[j] >= kk) {
                    sel[0] = nbins - 1 - kBinsPerThr * tid - j;
                    sel[1] = cum;
                    break;
                }
                cum += loc[j];
            }
        }
        __syncthreads();
        hi = (hi << width) | (uint32_t)sel[0];
        kk -= sel[1];
        __syncthreads();
    }
    return passes == 3 ? hi : passes == 2 ? hi << 10 : hi << 20;
}

__global__ void __launch_bounds__(kTopThr) qsa_topk_kernel(const __grid_constant__ TopkParams p) {
    extern __shared__ __align__(16) unsigned char smt[];
    int *hist = reinterpret_cast<int *>(smt);                          // [kHist]
    int *sw = hist + kHist;                                            // [32] scan scratch
    int *sel = sw + 32;                                                // [32] digit, count above, count
    int *wcnt = sel + 32;                                              // [32] per-warp counts
    uint32_t *ckey = reinterpret_cast<uint32_t *>(wcnt + 32);          // [kCandCap]
    int *cidx = reinterpret_cast<int *>(ckey + kCandCap);              // [kCandCap]
    uint32_t *bm_sel = reinterpret_cast<uint32_t *>(cidx + kCandCap);  // [ceil(nb_max / 32)]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t lt = (1u << lane) - 1u;
    const int64_t row = blockIdx.x;
    const int b = (int)(row / p.Qn);
    const int64_t pos = (int64_t)p.qpos[b] + row % p.Qn;
    const int64_t cap = max(0, min(p.n_blocks[b], p.nb_max));
    const int nvis = (int)n_cand(pos, cap);
    const int nwords = (p.nb_max + 31) >> 5;
    uint32_t *bm_eq = bm_sel + nwords;
    int32_t *ob = p.blocks + row * kKB;
    int32_t *ot = p.tokens ? p.tokens + row * kTok : nullptr;
    const int64_t tail0 = pos < 0 ? 0 : ((pos + 1) >> 2) * kR;
    const int tail_n = pos < 0 ? 0 : (int)(pos - tail0 + 1);
    const int count = min(nvis, kKB);
    // token slots after the selected blocks' 4 count: the tail, then -1
    auto tail_fill = [&]() {
        if (!ot) return;
        for (int t = kR * count + tid; t < kTok; t += kTopThr)
            ot[t] = t - kR * count < tail_n ? (int32_t)(tail0 + (t - kR * count)) : -1;
    };
    auto emit = [&](int o, int e) {
        ob[o] = e;
        if (ot) {
            ot[kR * o] = kR * e;
            ot[kR * o + 1] = kR * e + 1;
            ot[kR * o + 2] = kR * e + 2;
            ot[kR * o + 3] = kR * e + 3;
        }
    };
    auto fail = [&]() {   // a score computation gave up: mark the whole row
        for (int t = tid; t < kKB; t += kTopThr) ob[t] = -2;
        if (ot)
            for (int t = tid; t < kTok; t += kTopThr) ot[t] = -2;
    };
    if (nvis <= kKB) {   // every candidate is selected
        for (int t = tid; t < kKB; t += kTopThr) ob[t] = t < nvis ? t : -1;
        if (ot)
            for (int t = tid; t < kR * count; t += kTopThr) ot[t] = t;
        tail_fill();
        return;
    }
    const uint32_t *keys = reinterpret_cast<const uint32_t *>(p.scores + row * p.ld);

    // 1. threshold from a strided sample (all scores are candidates when few)
    uint32_t t_low = 0;
    if (nvis > kCandCap) {
        const int S = min(nvis / kSampleStride, kCandCap);
        for (int j = tid; j < S; j += kTopThr) ckey[j] = keys[kSampleStride * j + kSampleStride / 2];
        __syncthreads();
        const int rs = min(S, (int)(((int64_t)kKB * S + nvis - 1) / nvis) + kSampleMargin);
        int kk_s;
        t_low = radix_select(ckey, S, rs, hist, sw, sel, kk_s, 2);
    }
    // 2. candidates: every score >= t_low, 4 keys per lane per load (NaN or a set sign bit
    //    marks a failed score computation)
    if (tid == 0) sel[2] = 0;
    __syncthreads();
    uint32_t mx = 0;
    for (int base = warp * 128; base < nvis; base += 4 * kTopThr) {
        const int e = base + 4 * lane;
        uint4 kv = make_uint4(0u, 0u, 0u, 0u);
        if (e < nvis) kv = __ldcs(reinterpret_cast<const uint4 *>(keys + e));   // e + 3 < ld
        const uint32_t k4[4] = {kv.x, kv.y, kv.z, kv.w};
        uint32_t cm = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const bool v = e + j < nvis;
            if (v) mx = max(mx, k4[j]);
            if (v && k4[j] >= t_low) cm |= 1u << j;
        }
        const int cnt = __popc(cm);
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        const int tot = __shfl_sync(0xffffffffu, incl, 31);
        int at = 0;
        if (lane == 31 && tot) at = atomicAdd(&sel[2], tot);
        at = __shfl_sync(0xffffffffu, at, 31);
        int o = at + incl - cnt;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if ((cm >> j) & 1u) {
                if (o < kCandCap) {
                    ckey[o] = k4[j];
                    cidx[o] = e + j;
                }
                ++o;
            }
        }
    }
    const bool bad = mx > 0x7F800000u;
    if (__syncthreads_or(bad)) {
        fail();
        return;
    }
    const int C = sel[2];
    __syncthreads();

    if (C >= kKB && C <= kCandCap) {
        // 3. exact select among the candidates, then the ordered output from bitmaps
        int kk;
        const uint32_t thr = radix_select(ckey, C, kKB, hist, sw, sel, kk);
        const int W = (nvis + 31) >> 5;
        for (int w = tid; w < W; w += kTopThr) bm_sel[w] = bm_eq[w] = 0u;
        __syncthreads();
        for (int c = tid; c < C; c += kTopThr) {
            const uint32_t key = ckey[c];
            const int e = cidx[c];
            if (key > thr) atomicOr(&bm_sel[e >> 5], 1u << (e & 31));
            else if (key == thr) atomicOr(&bm_eq[e >> 5], 1u << (e & 31));
        }
        __syncthreads();
        const int wpt = (W + kTopThr - 1) / kTopThr;
        const int w0 = min(W, tid * wpt), w1 = min(W, w0 + wpt);
        int eqc = 0;
        for (int w = w0; w < w1; ++w) eqc += __popc(bm_eq[w]);
        int need = kk - excl_scan_cta(eqc, sw);      // equal keys this thread may still take
        int selc = 0;
        for (int w = w0; w < w1; ++w) {
            uint32_t e = bm_eq[w], take = 0u;
            if (need > 0) {
                if (__popc(e) <= need) {
                    take = e;
                    need -= __popc(e);
                } else {
                    while (need > 0) {
                        const uint32_t lb = e & (0u - e);
                        take |= lb;
                        e ^= lb;
                        --need;
                    }
                }
            }
            const uint32_t m = bm_sel[w] | take;
            bm_sel[w] = m;
            selc += __popc(m);
        }
        int o = excl_scan_cta(selc, sw);
        for (int w = w0; w < w1; ++w) {
            uint32_t m = bm_sel[w];
            while (m) {
                const int bit = __ffs(m) - 1;
                m &= m - 1u;
                emit(o++, 32 * w + bit);
            }
        }
        tail_fill();
        return;
    }

    // 4. fallback: radix select over the whole row, then one ordered pass (warp w covers
    //    [w Ew, (w+1) Ew): its counts first, then the writes)
    int kk;
    const uint32_t thr = radix_select(keys, nvis, kKB, hist, sw, sel, kk);
    const int ew = ((nvis + kTopWarps - 1) / kTopWarps + 31) & ~31;
    const int e0 = warp * ew, e1 = min(nvis, e0 + ew);
    int gt = 0, eq = 0;
    for (int base = e0; base < e1; base += 32) {
        const int e = base + lane;
        const uint32_t key = e < e1 ? keys[e] : 0u;
        gt += __popc(__ballot_sync(0xffffffffu, e < e1 && key > thr));
        eq += __popc(__ballot_sync(0xffffffffu, e < e1 && key == thr));
    }
    if (lane == 0) {
        wcnt[warp] = gt;
        sw[16 + warp] = eq;
    }
    __syncthreads();
    int gt_run = 0, eq_run = 0;
    for (int w = 0; w < warp; ++w) {
        gt_run += wcnt[w];
        eq_run += sw[16 + w];
    }
    for (int base = e0; base < e1; base += 32) {
        const int e = base + lane;
        const uint32_t key = e < e1 ? keys[e] : 0u;
        const bool g = e < e1 && key > thr, q = e < e1 && key == thr;
        const uint32_t gb = __ballot_sync(0xffffffffu, g), qb = __ballot_sync(0xffffffffu, q);
        const bool take = g || (q && eq_run + __popc(qb & lt) < kk);
        const uint32_t sb = __ballot_sync(0xffffffffu, take);
        if (take) emit(gt_run + min(eq_run, kk) + __popc(sb & lt), e);
        gt_run += __popc(gb);
        eq_run += __popc(qb);
    }
    tail_fill();
}

}  // namespace qsa

// ------------------------------------------------------------------ launchers
cudaError_t launch_qsa_block_keys(const void *k, const float *w, const int32_t *kpos, int B, int Tn,
                                  float eps, float theta, void *kbar, int nb_max, cudaStream_t s) {
    qsa::KeyParams p{static_cast<const __nv_bfloat16 *>(k), w, kpos, static_cast<__nv_bfloat16 *>(kbar),
                     B, Tn, nb_max, eps, theta};
    const int64_t warps = (int64_t)B * (Tn / qsa::kR);
    if (warps == 0) return cudaSuccess;
    TraceLaunch tl(s, "qsa_block_keys");
    qsa::qsa_block_keys_kernel<<<(unsigned)((warps + 7) / 8), 256, 0, s>>>(p);
    return cudaGetLastError();
}

// queries per scores CTA: the smallest multiple of 4 that covers Qn, at most 64
static int score_qt(int Qn) { return std::min(qsa::kMaxQT, (Qn + 3) & ~3); }

cudaError_t launch_qsa_scores(const void *q, const float *w, const int32_t *qpos, const void *kbar,
                              const int32_t *n_blocks, int B, int Qn, int nb_max, float eps, float theta,
                              float *scores, int64_t ld, cudaStream_t s) {
    if (B == 0 || Qn == 0) return cudaSuccess;
    qsa::ScoreParams p{};
    if (!encode_2d(&p.tm_kbar, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kbar, qsa::kD, (int64_t)B * nb_max,
                   qsa::kD * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    p.q = static_cast<const __nv_bfloat16 *>(q);
    p.w = w;
    p.qpos = qpos;
    p.n_blocks = n_blocks;
    p.scores = scores;
    p.ld = ld;
    p.B = B;
    p.Qn = Qn;
    p.nb_max = nb_max;
    p.eps = eps;
    p.theta = theta;
    // queries per CTA (a multiple of 4, at most 64) and the split of each query tile's block
    // range: the fewest estimated time units over whole waves of one CTA per SM, a 128-block
    // tile costing ~ qt + 16 units (the epilogue of its 4 qt columns and a fixed share) and a
    // CTA's query-head preparation ~ 2 qt
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t tiles = (nb_max + 127) / 128;
    double best_cost = 1e300;
    p.qt = 4;
    p.n_split = 1;
    for (int qt = score_qt(Qn); qt >= 4; qt -= 4) {
        const int64_t ctas1 = (int64_t)((Qn + qt - 1) / qt) * B;
        for (int ns = 1; ns <= 16 && ns <= tiles; ++ns) {
            const double waves = std::ceil((double)(ctas1 * ns) / sms);
            const double cost = waves * (std::ceil((double)tiles / ns) * (qt + 16.0) + 2.0 * qt);
            if (cost < best_cost - 1e-9) {
                best_cost = cost;
                p.qt = qt;
                p.n_split = ns;
            }
        }
    }
    const int nqt = (Qn + p.qt - 1) / p.qt;
    auto kern = qsa::qsa_scores_kernel;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)qsa::kScoreSmem);
    if (e != cudaSuccess) return e;
    const int n_epi = 4 * std::min(4, p.qt / 4);
    TraceLaunch tl(s, "qsa_scores");
    kern<<<dim3((unsigned)nqt, (unsigned)B, (unsigned)p.n_split), 32 * (n_epi + 2), qsa::kScoreSmem, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_qsa_topk(const float *scores, int64_t ld, const int32_t *qpos, const int32_t *n_blocks, int B,
                            int Qn, int nb_max, int32_t *blocks, int32_t *tokens, cudaStream_t s) {
    if (B == 0 || Qn == 0) return cudaSuccess;
    qsa::TopkParams p{scores, qpos, n_blocks, blocks, tokens, ld, B, Qn, nb_max};
    const size_t smem = (size_t)(qsa::kHist + 96) * 4 + (size_t)qsa::kCandCap * 8 +
                        (size_t)2 * ((nb_max + 31) / 32) * 4;
    auto kern = qsa::qsa_topk_kernel;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    TraceLaunch tl(s, "qsa_topk");
    kern<<<(unsigned)((int64_t)B * Qn), qsa::kTopThr, smem, s>>>(p);
    return cudaGetLastError();
}

}  // namespace gdn
