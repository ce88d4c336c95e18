// State-independent work of the chunked prefill, for every (chunk, V head) at once.
//
// For a chunk of n <= 64 tokens of one sequence and one V head h (QK head g = h / (Hv/Hqk)),
// following the chunked form of the gated delta rule of the page "ARCHITECTURE PREVIEW /
// FIELD NOTES", section 03 (GATED DELTANET), with g_t = sum_{s<=t} log alpha_s inside the
// chunk, gamma_t = exp(g_t) and kd_t = exp(g_{n-1} - g_t):
//     A_ti = beta_t exp(g_t - g_i) k_t.k_i        (i < t < n, else 0)
//     T    = (I + A)^-1,   T_beta = T diag(beta),   T_beta_gamma = T diag(beta gamma)
//     P_ti = exp(g_t - g_i) q_t.k_i               (i <= t < n, else 0)
// T_beta and P (64 x 64) are written as fp16 tiles and T_beta_gamma as an fp32 tile rounded to
// TF32 (the precisions the tensor-core chain reads them in), already in the shared-memory
// layout of an MMA operand (K-major, 128-byte rows with 16-byte chunks XOR-swizzled by row),
// for the chain kernel to stream in with one bulk copy each.  A gates record per (chunk, head) carries gamma_t,
// kd_t and gamma_C = exp(g_{n-1}), the per-token factors the chain applies in tensor memory.
//
// One CTA per (chunk, group of up to 3 V heads of one QK head): K K^T and Q K^T do not
// depend on the gates, so one bulk copy of the chunk's [K;Q] tile and one tcgen05 MMA
// ([K;Q] K^T into tensor memory) serve all the CTA's heads.  Each head then has a group of
// 4 warps: the warps turn the MMA rows into A (kept in shared memory, transposed) and P
// (stored straight to global memory), and invert I + A in registers, two threads per
// column of T (even and odd rows) by forward substitution.  T_beta and T_beta_gamma are
// staged in turn over the head's scratch and each leaves by one bulk store.
#include "gdn_common.cuh"
#include "chunk_range.cuh"
#include "gdn_internal.h"
#include "tc_sm100.cuh"

namespace gdn {

namespace {
using namespace tc;

constexpr int kGroupThr = 128;   // 4 warps per V head
constexpr int kMaxGroups = 3;    // V heads per CTA

// shared-memory map (bytes from a 1024-aligned base).  [0, 64 KB) holds the [K;Q] tile until
// the MMA has read it, then one scratch per group: -A^T split by row parity, array p holding
// -A[2s + p][m] at row m, column s (64 x 32 floats), the odd array 64 bytes past a multiple
// of 8 KB so that the two parities fall in different banks; after the inverse, the staging
// of T_beta (K-major fp16 image, 8 KB), then of T_beta_gamma (K-major TF32 image, 16 KB).
constexpr uint32_t P_KQ = 0;
constexpr uint32_t kParStride = 8192 + 64;
constexpr uint32_t kScrBytes = 2 * kParStride;
constexpr uint32_t P_GATE = 65536;                 // per group: g, beta, gamma, 1/gamma
constexpr uint32_t kGateBytes = 4 * 64 * 4;
constexpr uint32_t P_BAR = P_GATE + kMaxGroups * kGateBytes;   // 2 mbarriers
constexpr uint32_t P_SLOT = P_BAR + 16;            // TMEM base
constexpr uint32_t kPSmem = P_SLOT + 16;
constexpr uint32_t kPSmemAlloc = kPSmem + 1024;
constexpr uint32_t kPTmemCols = 64;
constexpr uint32_t kPWaitTries = 1u << 24;
constexpr float kMaxChunkDecay = 80.f;  // factor exp(g_t - g_i) = gamma_t / gamma_i below this
static_assert(kMaxGroups * kScrBytes <= 65536, "group scratch inside the tile area");

__device__ __forceinline__ float4 tf32x4(float4 x) {
    return make_float4(to_tf32(x.x), to_tf32(x.y), to_tf32(x.z), to_tf32(x.w));
}

// contiguous bulk copy shared (this CTA) -> global, tracked as a bulk async-group
__device__ __forceinline__ void bulk_store(void *dst, uint32_t src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void group_sync(int id) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(kGroupThr) : "memory");
}

struct PrepParams {
    const float *kq;      // [chunk, Hqk] [K;Q] tiles (64 KB each)
    const void *alpha, *beta;
    const int32_t *cu, *cfirst;
    const int32_t *cseq;  // sequence of each slot (compact numbering)
    float *tb, *tg, *pm;  // [slot, Hv] tiles (T_beta_gamma 16 KB; T_beta and P fp16, 8 KB)
    float *gr;            // [slot, Hv] gates records
    int n_seqs, n_qk, n_v;
    ChunkRange rg;        // the range of this launch
};

}  // namespace

// blockDim.x = 128 x G, G dividing Hv / Hqk; CTA x covers V heads G*(x mod Hv/G) + [0, G)
// of the chunk in slot x / (Hv/G) of the range
template <class TI>
__global__ void __launch_bounds__(kGroupThr * kMaxGroups, 2) chunk_prep_kernel(const __grid_constant__ PrepParams p) {
    const int G = blockDim.x / kGroupThr;
    const int per_chunk = p.n_v / G;
    const int64_t u = blockIdx.x / per_chunk;   // slot
    int b, cj;
    if (p.rg.compact) {
        if (u >= p.cfirst[p.n_seqs]) return;   // uniform per CTA
        b = p.cseq[u];
        cj = (int)u - p.cfirst[b];
    } else if (!sliced_slot_chunk(p.rg, u, p.cfirst, &b, &cj)) {
        return;   // uniform per CTA
    }
    const int h0 = (int)(blockIdx.x % per_chunk) * G;
    const int gq = h0 / (p.n_v / p.n_qk);
    const int seq0 = p.cu[b];
    const int r0 = cj * kChunk;
    const int n = min(kChunk, p.cu[b + 1] - seq0 - r0);
    const int tok = seq0 + r0;

    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    const uint32_t sb = smem_u32(sm);
    uint64_t *bar = (uint64_t *)(sm + P_BAR);
    uint32_t *tslot = (uint32_t *)(sm + P_SLOT);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int grp = tid / kGroupThr, gt = tid % kGroupThr;   // group grp: V head h0 + grp
    const int h = h0 + grp;
    const int64_t tile = (int64_t)u * p.n_v + h;
    float *g_s = (float *)(sm + P_GATE + grp * kGateBytes), *beta_s = g_s + 64, *gam_s = g_s + 128,
          *ig_s = g_s + 192;
    unsigned char *scr = sm + grp * kScrBytes;
    const int gbar = 1 + grp;   // named barrier of the group
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
    if (gt < kChunk) {
        const TI *al = (const TI *)p.alpha, *be = (const TI *)p.beta;
        const int64_t e = (int64_t)(tok + gt) * p.n_v + h;
        g_s[gt] = gt < n ? safe_log_alpha(to_f32(al[e])) : 0.f;
        beta_s[gt] = gt < n ? to_f32(be[e]) : 0.f;
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
    // warp 1 of each group: inclusive scan of log alpha, two rows per lane, summed in fp64 (with
    // strong decay g reaches -100 and beyond inside a chunk, and fp32 partial sums would leave
    // ~1e-4 relative error in the ratios exp(g_t - g_i); each g_t rounded once to fp32 leaves
    // ~1e-5 at g = -100)
    if ((gt >> 5) == 1) {
        const int t0 = 2 * lane, t1 = t0 + 1;
        const double a0 = g_s[t0], a1 = g_s[t1];
        double s = a0 + a1;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const double y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        const double g0 = s - a1, g1 = s;
        const double glast = __shfl_sync(0xffffffffu, ((n - 1) & 1) ? g1 : g0, (n - 1) >> 1);
        g_s[t0] = (float)g0;
        g_s[t1] = (float)g1;
        const float gam0 = expf((float)g0), gam1 = expf((float)g1);
        gam_s[t0] = gam0;
        gam_s[t1] = gam1;
        ig_s[t0] = expf((float)-g0);      // used only when the chunk's decay stays below kMaxChunkDecay
        ig_s[t1] = expf((float)-g1);
        gr[kGrGamma + t0] = gam0;
        gr[kGrGamma + t1] = gam1;
        gr[kGrKd + t0] = t0 < n ? expf((float)(glast - g0)) : 0.f;
        gr[kGrKd + t1] = t1 < n ? expf((float)(glast - g1)) : 0.f;
        if (lane == 0) gr[kGrGammaC] = expf((float)glast);
    }
    if (tid == 0) {
        if (ok) ok = mbar_wait(&bar[1], 0, kPWaitTries);
        else mbar_wait(&bar[0], 0, kPWaitTries);   // drain the copy
    }
    ok = !__syncthreads_or(!ok);  // the MMA is done (the tile area is free); gates published
    fence_after_sync();
    if (ok) {
        // Row t of K K^T (lane quarters 0-1) becomes row t of -A, written transposed into the
        // parity arrays; row t of Q K^T (quarters 2-3) becomes row t of P, fp16, stored to
        // global memory in the K-major image.  exp(g_t - g_i) = gamma_t / gamma_i while the
        // chunk's total decay keeps 1 / gamma finite; otherwise one exponential per element.
        const int q = warp & 3;
        const bool is_a = q < 2;
        const int t = 32 * (q & 1) + lane;
        const bool factored = -g_s[n - 1] < kMaxChunkDecay;
        const float bt = is_a ? -beta_s[t] : 1.f, rowf = gam_s[t] * bt, gtv = g_s[t];
        const int lim = t < n ? (is_a ? t : t + 1) : 0;   // columns i < lim are kept
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {   // columns 32*h2 .. 32*h2 + 31
            float v[32];
            tmem_ld32(taddr(tm, 32 * q, 32 * h2), v);
            tmem_wait_ld();
            tmem_regs_after_wait(v);
            if (factored) {   // uniform per CTA
#pragma unroll
                for (int e = 0; e < 32; e += 4) {
                    const float4 f = *reinterpret_cast<const float4 *>(ig_s + 32 * h2 + e);
                    const int i = 32 * h2 + e;
                    v[e] = i < lim ? rowf * f.x * v[e] : 0.f;
                    v[e + 1] = i + 1 < lim ? rowf * f.y * v[e + 1] : 0.f;
                    v[e + 2] = i + 2 < lim ? rowf * f.z * v[e + 2] : 0.f;
                    v[e + 3] = i + 3 < lim ? rowf * f.w * v[e + 3] : 0.f;
                }
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int i = 32 * h2 + e;
                    v[e] = i < lim ? bt * expf(gtv - g_s[i]) * v[e] : 0.f;
                }
            }
            if (is_a) {
                float *at = (float *)(scr + (t & 1) * kParStride) + (t >> 1) + 32 * 32 * h2;
#pragma unroll
                for (int e = 0; e < 32; ++e) at[e * 32] = v[e];
            } else {   // fp16 (nearest even), K-major
                unsigned char *dst = (unsigned char *)(p.pm + tile * 2048);
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    *reinterpret_cast<uint2 *>(dst + kmaj16_off(t, 32 * h2 + 4 * k)) =
                        make_uint2(pack_f16x2(v[4 * k], v[4 * k + 1]), pack_f16x2(v[4 * k + 2], v[4 * k + 3]));
            }
        }
    }
    group_sync(gbar);   // the group's A^T is complete

    // ---- T = (I + A)^-1, column jc by forward substitution with right-looking updates:
    // once row m of the column is final, every later row r loses A[r][m] T[m][jc].  This
    // thread holds the rows of parity par (x[s] = T[2s + par][jc], as pairs for the packed
    // FMA) and takes row m from its partner lane when m has the other parity.  Entries of A
    // on or above the diagonal are zero in the scratch, so the updates may start at a
    // multiple of 4; a warp skips the steps before its first column, where its rows are 0.
    const int jc = gt >> 1, par = gt & 1;
    const int m_first = 16 * (gt >> 5);   // this warp's columns are m_first .. m_first + 15
    float2 x[16];
#pragma unroll
    for (int s = 0; s < 16; ++s)
        x[s] = make_float2(2 * (2 * s) + par == jc ? 1.f : 0.f, 2 * (2 * s + 1) + par == jc ? 1.f : 0.f);
    if (ok) {
        const float *atp = (const float *)(scr + par * kParStride);
#pragma unroll
        for (int m = 0; m < 63; ++m) {
            if (m < m_first) continue;   // warp-uniform
            const float2 xs = x[m >> 2];
            const float mine = (m >> 1) & 1 ? xs.y : xs.x;
            const float other = __shfl_xor_sync(0xffffffffu, mine, 1);
            const float xm = (par == (m & 1)) ? mine : other;
            const float2 xm2 = make_float2(xm, xm);
#pragma unroll
            for (int s0 = (m >> 1) & ~3; s0 < 32; s0 += 4) {
                const float4 a = *reinterpret_cast<const float4 *>(atp + m * 32 + s0);
                x[s0 >> 1] = __ffma2_rn(make_float2(a.x, a.y), xm2, x[s0 >> 1]);
                x[(s0 >> 1) + 1] = __ffma2_rn(make_float2(a.z, a.w), xm2, x[(s0 >> 1) + 1]);
            }
        }
    }
    // T_beta = T diag(beta) as fp16 and T_beta_gamma = T diag(beta gamma) as TF32, each a
    // K-major image staged over the group's scratch and stored with one bulk copy; NaN if the
    // CTA failed.  fp16 holds T_beta: |T_beta| <= 1 for beta in [0, 1] (and <= 4 for beta up
    // to 2), and an entry beyond 65504 would become inf, so NaN downstream, never a wrong
    // finite value.
    const float nan = __int_as_float(0x7fc00000);
    const float bj = beta_s[jc];
#pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {
        group_sync(gbar);   // the scratch is free (A^T read, or the previous store has read it)
        if (pass == 0) {
#pragma unroll
            for (int s = 0; s < 32; s += 2) {
                // rows 2s + par and 2s + 2 + par of column jc: two separate fp16 (columns are
                // what this thread owns, so no pairs can be packed)
                const float2 xv = x[s >> 1];
                *reinterpret_cast<__half *>(scr + kmaj16_off(2 * s + par, jc)) =
                    __float2half_rn(ok ? xv.x * bj : nan);
                *reinterpret_cast<__half *>(scr + kmaj16_off(2 * s + 2 + par, jc)) =
                    __float2half_rn(ok ? xv.y * bj : nan);
            }
        } else {
            const float fj = bj * gam_s[jc];
#pragma unroll
            for (int s = 0; s < 32; ++s) {
                const float xv = (s & 1) ? x[s >> 1].y : x[s >> 1].x;
                *reinterpret_cast<float *>(scr + kmaj_off(2 * s + par, jc, 64)) = ok ? to_tf32(xv * fj) : nan;
            }
        }
        fence_smem_to_async();
        group_sync(gbar);
        if (gt == 0) {
            if (pass == 0) bulk_store(p.tb + tile * 2048, smem_u32(scr), 8192);
            else bulk_store(p.tg + tile * 4096, smem_u32(scr), 16384);
            bulk_commit();
            bulk_wait_read0();   // the staging may be overwritten once the copy has read it
        }
    }
    if (gt == 0) bulk_wait0();   // the stores are complete before the CTA's shared memory goes away
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tm, kPTmemCols);
}

cudaError_t launch_chunk_prep(const ScanParams &sp, int64_t total_tokens, bool in_bf16, cudaStream_t s) {
    if (sp.n_seqs <= 0 || total_tokens <= 0) return cudaSuccess;
    PrepParams p{};
    p.kq = sp.kq;
    p.alpha = sp.alpha; p.beta = sp.beta; p.cu = sp.cu; p.cfirst = sp.cfirst; p.cseq = sp.cseq;
    p.tb = sp.tb; p.tg = sp.tg; p.pm = sp.pm; p.gr = sp.gr; p.n_seqs = sp.n_seqs; p.n_qk = sp.n_qk; p.n_v = sp.n_v;
    p.rg = sp.rg;
    // V heads per CTA: 3, 2 or 1, whichever first divides the V heads of a QK head
    const int ratio = sp.n_v / sp.n_qk;
    const int G = ratio % 3 == 0 ? 3 : (ratio % 2 == 0 ? 2 : 1);
    const int64_t grid = sp.slots * (sp.n_v / G);
    if (grid <= 0) return cudaSuccess;
    if (grid >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
    auto k = in_bf16 ? chunk_prep_kernel<bf16> : chunk_prep_kernel<float>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kPSmemAlloc);
    if (e != cudaSuccess) return e;
    TraceLaunch tl(s, "chunk_prep");
    k<<<(unsigned)grid, kGroupThr * G, kPSmemAlloc, s>>>(p);
    return cudaGetLastError();
}

}  // namespace gdn
