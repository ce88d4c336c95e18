// C ABI of libgdn: argument validation, workspace layout and kernel launches.
// The declarations and the contract of every entry point are in include/libgdn.h.
#include <algorithm>
#include <cmath>
#include <cstring>

#include "gdn_common.cuh"
#include "gdn_internal.h"
#include "libgdn.h"

namespace gdn {

static thread_local int t_last_cuda_error = 0;

// per-host-thread launch trace (see gdn_trace_begin)
static thread_local gdn_trace_entry *t_trace = nullptr;
static thread_local int t_trace_cap = 0;
static thread_local int t_trace_n = 0;
static thread_local bool t_trace_on = false;

void record_cuda_error(cudaError_t e) { t_last_cuda_error = (int)e; }

TraceLaunch::TraceLaunch(cudaStream_t s, const char *kernel) : stream(s), entry(nullptr) {
    if (!t_trace_on) return;
    if (t_trace_n < t_trace_cap && t_trace) {
        entry = &t_trace[t_trace_n];
        entry->kernel = kernel;
        cudaEventRecord(entry->start, s);
    }
    ++t_trace_n;
}

TraceLaunch::~TraceLaunch() {
    if (entry) cudaEventRecord(entry->stop, stream);
}

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Carve the tile buffers for `slots` chunk slots, `n_buf` buffers, starting at `off`.
static size_t carve_tiles(PrefillLayout &L, int n_qk, int n_v, int64_t slots, int n_buf, size_t off) {
    const size_t ns = (size_t)slots;
    size_t o = 0;
    L.b_kq = o;   o = align_up(o + ns * n_qk * 65536, 256);
    L.b_kmn = o;  o = align_up(o + ns * n_qk * 16384, 256);   // fp16
    L.b_vi = o;   o = align_up(o + ns * n_v * 16384, 256);    // fp16
    L.b_tb = o;   o = align_up(o + ns * n_v * 8192, 256);     // fp16
    L.b_tg = o;   o = align_up(o + ns * n_v * 16384, 256);
    L.b_pm = o;   o = align_up(o + ns * n_v * 8192, 256);    // fp16
    L.b_gr = o;   o = align_up(o + ns * n_v * kGateRec * sizeof(float), 256);
    L.b_cseq = o; o = align_up(o + ns * sizeof(int32_t), 256);
    L.buf_bytes = o;
    L.off_tiles = off;
    L.slots = slots;
    L.n_buf = n_buf;
    return off + (size_t)n_buf * o;
}

// The tensor-core layout for a given range plan: compact (one range over every chunk) or
// sliced with R chunks per sequence per range and n_buf buffers.
static void tc_layout(PrefillLayout &L, int n_qk, int n_v, int n_seqs, int64_t maxc, bool compact, int R,
                      int n_buf, size_t off) {
    if (compact) {
        L.range0 = ChunkRange{1, 0, 0, 1};
        L.n_ranges = 1;
        off = carve_tiles(L, n_qk, n_v, L.max_chunks, 1, off);
    } else {
        L.range0 = ChunkRange{0, R, 0, 0};
        L.n_ranges = (int)((maxc + R - 1) / R);
        off = carve_tiles(L, n_qk, n_v, (int64_t)n_seqs * R, std::min(n_buf, L.n_ranges), off);
    }
    const size_t carry = L.n_ranges > 1 ? (size_t)n_seqs * n_v * 128 * 128 * sizeof(float) : 0;
    L.off_carry = off;
    off = align_up(off + carry, 256);
    L.bytes = off;
}

bool prefill_layout(int n_qk, int n_v, int64_t T, int n_seqs, int64_t max_seqlen, bool tc, size_t ws_limit,
                    PrefillLayout *out) {
    PrefillLayout L{};
    L.max_chunks = (T + kChunk - 1) / kChunk + n_seqs;
    size_t off = 0;
    L.off_cu = off;      off = align_up(off + sizeof(int32_t) * (size_t)(n_seqs + 1), 256);
    L.off_cfirst = off;  off = align_up(off + sizeof(int32_t) * (size_t)(n_seqs + 1), 256);
    const size_t qk_bytes = tc ? 0 : (size_t)T * n_qk * 128 * sizeof(float);
    const size_t v_bytes = tc ? 0 : (size_t)T * n_v * 128 * sizeof(float);
    L.off_qh = off;      off = align_up(off + qk_bytes, 256);
    L.off_kh = off;      off = align_up(off + qk_bytes, 256);
    L.off_vh = off;      off = align_up(off + v_bytes, 256);
    if (!tc || T == 0 || n_seqs == 0) {   // fp32 rows (one pass), or nothing to tile
        L.range0 = ChunkRange{1, 0, 0, 1};
        L.n_ranges = 1;
        L.n_buf = 1;
        L.off_tiles = L.off_carry = off;
        L.bytes = off;
        *out = L;
        return L.bytes <= ws_limit;
    }
    // preferred plan: few chains -> ranges sized to overlap prep with the chains; many chains
    // -> ranges that bound the tile memory while every sequence still advances in each range
    const int64_t ms = (max_seqlen > 0 && max_seqlen < T) ? max_seqlen : T;
    const int64_t maxc = (ms + kChunk - 1) / kChunk;
    const bool few = (int64_t)n_seqs * n_v <= kFewChains;
    int64_t R = few ? std::min<int64_t>(128, std::max<int64_t>(32, (maxc + 3) / 4))
                    : std::min<int64_t>(64, std::max<int64_t>(8, 512 / n_seqs));
    R = std::min(R, maxc);
    const int64_t cap = max_seqlen > 0 ? kMaxRanges : kMaxRangesUnknown;
    if ((maxc + R - 1) / R > cap) R = (maxc + cap - 1) / cap;
    const int nr = (int)((maxc + R - 1) / R);
    // one range, or many chains and no memory to save: global chunk numbering
    const bool compact = nr == 1 || (!few && (int64_t)std::min(2, nr) * n_seqs * R >= L.max_chunks);
    tc_layout(L, n_qk, n_v, n_seqs, maxc, compact, (int)std::min<int64_t>(R, INT32_MAX), 2, off);
    if (L.bytes > ws_limit) {
        // shrink the ranges to the workspace given: two buffers if one chunk per sequence fits
        // twice, else one (range r+1 is then prepared after the chains of range r)
        bool fit = false;
        for (int nb = 2; nb >= 1 && !fit; --nb) {
            const size_t per = (size_t)n_seqs * ((size_t)n_qk * 81920 + (size_t)n_v * (49152 + kGateRec * 4)) * nb;
            const size_t avail = ws_limit > off ? ws_limit - off : 0;
            int64_t r = std::min<int64_t>(R, (int64_t)(avail / per) + 1);
            for (; r >= 1; --r) {
                tc_layout(L, n_qk, n_v, n_seqs, maxc, false, (int)r, nb, off);
                if (L.bytes <= ws_limit) { fit = true; break; }
            }
        }
        if (!fit) {
            *out = L;
            return false;
        }
    }
    *out = L;
    return true;
}

// One auxiliary stream and a few events per (host thread, device) for the chunk ranges:
// created on the first multi-range prefill of the thread on that device, kept for the life
// of the process.
struct AuxStream {
    cudaStream_t stream = nullptr;
    cudaEvent_t ev_tab = nullptr;       // sequence tables ready (caller's stream)
    cudaEvent_t ev_prep[2] = {};        // tiles of the range in buffer i ready (auxiliary stream)
    cudaEvent_t ev_chain[2] = {};       // chains done with buffer i (caller's stream)
};
static thread_local AuxStream t_aux[64];

static cudaError_t aux_stream(AuxStream **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    AuxStream &a = t_aux[dev];
    if (!a.stream) {
        AuxStream fresh;
        cudaEvent_t *evs[5] = {&fresh.ev_tab, &fresh.ev_prep[0], &fresh.ev_prep[1], &fresh.ev_chain[0],
                               &fresh.ev_chain[1]};
        e = cudaStreamCreateWithFlags(&fresh.stream, cudaStreamNonBlocking);
        for (auto *ev : evs)
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
        if (e != cudaSuccess) {
            for (auto *ev : evs)
                if (*ev) cudaEventDestroy(*ev);
            if (fresh.stream) cudaStreamDestroy(fresh.stream);
            return e;
        }
        a = fresh;
    }
    *out = &a;
    return cudaSuccess;
}

}  // namespace gdn

using namespace gdn;

static gdn_status cuda_fail(cudaError_t e) {
    t_last_cuda_error = (int)e;
    return GDN_ERR_CUDA;
}

static bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

static gdn_status check_config(const gdn_config *cfg, gdn_dtype dtype) {
    if (!cfg) return GDN_ERR_INVALID_ARG;
    if (dtype != GDN_BF16 && dtype != GDN_F32) return GDN_ERR_INVALID_ARG;
    if (cfg->n_qk_heads <= 0 || cfg->n_v_heads <= 0) return GDN_ERR_INVALID_ARG;
    if (cfg->n_v_heads % cfg->n_qk_heads != 0) return GDN_ERR_INVALID_ARG;
    if (!std::isfinite(cfg->q_scale) || !std::isfinite(cfg->l2_eps) || cfg->l2_eps < 0.f)
        return GDN_ERR_INVALID_ARG;
    if (cfg->conv_activation != GDN_ACT_NONE && cfg->conv_activation != GDN_ACT_SILU) return GDN_ERR_INVALID_ARG;
    if (cfg->d_k != 128 || cfg->d_v != 128 || cfg->conv_width != 4) return GDN_ERR_UNSUPPORTED;
    // keep channel counts and grid dimensions inside int range
    // grid dimensions: 2*Hqk + Hv head slots ride in gridDim.y (<= 65535)
    if (cfg->n_qk_heads > 4096 || cfg->n_v_heads > 16384) return GDN_ERR_UNSUPPORTED;
    return GDN_OK;
}

static gdn_status check_device() {
    int dev = 0, major = 0, minor = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e != cudaSuccess) return cuda_fail(e);
    e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (major != 10 || minor != 0) return GDN_ERR_UNSUPPORTED;  // built for sm_100a only
    return GDN_OK;
}

extern "C" {

const char *gdn_status_string(gdn_status s) {
    switch (s) {
        case GDN_OK: return "GDN_OK";
        case GDN_ERR_INVALID_ARG: return "GDN_ERR_INVALID_ARG";
        case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED";
        case GDN_ERR_WORKSPACE: return "GDN_ERR_WORKSPACE";
        case GDN_ERR_CUDA: return "GDN_ERR_CUDA";
        case GDN_ERR_TIMEOUT: return "GDN_ERR_TIMEOUT";
    }
    return "GDN_ERR_UNKNOWN";
}

int gdn_last_cuda_error(void) { return t_last_cuda_error; }

int gdn_api_version(void) { return GDN_API_VERSION; }

void gdn_trace_begin(gdn_trace_entry *entries, int capacity) {
    t_trace = entries;
    t_trace_cap = entries ? (capacity > 0 ? capacity : 0) : 0;
    t_trace_n = 0;
    t_trace_on = true;
}

int gdn_trace_end(void) {
    t_trace_on = false;
    t_trace = nullptr;
    t_trace_cap = 0;
    return t_trace_n;
}

gdn_status gdn_prefill_workspace_size(const gdn_config *cfg, gdn_dtype dtype, int64_t total_tokens,
                                      int n_seqs, int64_t max_seqlen, size_t *bytes) {
    gdn_status st = check_config(cfg, dtype);
    if (st != GDN_OK) return st;
    if (!bytes || total_tokens < 0 || total_tokens >= ((int64_t)1 << 31) || n_seqs < 0 || max_seqlen < 0)
        return GDN_ERR_INVALID_ARG;
    PrefillLayout L;
    prefill_layout(cfg->n_qk_heads, cfg->n_v_heads, total_tokens, n_seqs, max_seqlen, dtype == GDN_BF16,
                   SIZE_MAX, &L);
    *bytes = L.bytes;
    return GDN_OK;
}

}  // extern "C"

// gated output of gdn_prefill_gated (z == null: plain y)
struct GateArgs {
    const void *z = nullptr;
    gdn_dtype z_dtype = GDN_BF16;
    const float *w = nullptr;
    float eps = 0.f;
};

static gdn_status prefill_impl(const gdn_config *cfg, gdn_dtype dtype, gdn_dtype out_dtype,
                               const void *q, const void *k,
                               const void *v, const float *conv_w_q, const float *conv_w_k,
                               const float *conv_w_v, const void *alpha, const void *beta,
                               const int32_t *cu_seqlens, int n_seqs, int64_t total_tokens, int64_t max_seqlen,
                               const float *initial_state, float *final_state, const void *conv_state_in,
                               void *conv_state_out, void *out, void *workspace, size_t workspace_bytes,
                               const GateArgs &gate, cudaStream_t stream) {
    gdn_status st = check_config(cfg, dtype);
    if (st != GDN_OK) return st;
    if (out_dtype != GDN_BF16 && out_dtype != GDN_F32) return GDN_ERR_INVALID_ARG;
    if (n_seqs < 0 || total_tokens < 0 || total_tokens >= ((int64_t)1 << 31) || max_seqlen < 0)
        return GDN_ERR_INVALID_ARG;
    if (n_seqs == 0) return GDN_OK;
    if ((int64_t)n_seqs * cfg->n_v_heads * 4 >= ((int64_t)1 << 31)) return GDN_ERR_UNSUPPORTED;
    const size_t eb = dtype == GDN_BF16 ? 2 : 4;
    if (!cu_seqlens || !aligned(cu_seqlens, 4)) return GDN_ERR_INVALID_ARG;
    if (total_tokens > 0) {
        if (!q || !k || !v || !alpha || !beta || !out) return GDN_ERR_INVALID_ARG;
        if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16))
            return GDN_ERR_INVALID_ARG;
        if (!aligned(alpha, eb) || !aligned(beta, eb)) return GDN_ERR_INVALID_ARG;
    }
    if (!conv_w_q || !conv_w_k || !conv_w_v) return GDN_ERR_INVALID_ARG;
    if (!aligned(conv_w_q, 16) || !aligned(conv_w_k, 16) || !aligned(conv_w_v, 16))
        return GDN_ERR_INVALID_ARG;
    if ((initial_state && !aligned(initial_state, 16)) || (final_state && !aligned(final_state, 16)))
        return GDN_ERR_INVALID_ARG;
    if ((conv_state_in && !aligned(conv_state_in, 16)) ||
        (conv_state_out && !aligned(conv_state_out, 16)))
        return GDN_ERR_INVALID_ARG;
    if (gate.z) {
        if (gate.z_dtype != GDN_BF16 && gate.z_dtype != GDN_F32) return GDN_ERR_INVALID_ARG;
        if (!gate.w || !aligned(gate.w, 16) || !std::isfinite(gate.eps) || gate.eps < 0.f) return GDN_ERR_INVALID_ARG;
        if (total_tokens > 0 && !aligned(gate.z, 16)) return GDN_ERR_INVALID_ARG;
        // fp32 input: y in fp32 in `out`, then the tail in place
        if (dtype == GDN_F32 && out_dtype != GDN_F32) return GDN_ERR_UNSUPPORTED;
    }
    if (!workspace || !aligned(workspace, 256)) return GDN_ERR_WORKSPACE;
    const bool bf = dtype == GDN_BF16;
    PrefillLayout L;
    if (!prefill_layout(cfg->n_qk_heads, cfg->n_v_heads, total_tokens, n_seqs, max_seqlen, bf, workspace_bytes, &L))
        return GDN_ERR_WORKSPACE;
    st = check_device();
    if (st != GDN_OK) return st;

    unsigned char *ws = (unsigned char *)workspace;
    int32_t *cu = (int32_t *)(ws + L.off_cu);
    int32_t *cfirst = (int32_t *)(ws + L.off_cfirst);
    cudaError_t e = launch_seq_table(cu_seqlens, n_seqs, total_tokens, cu, cfirst, stream);
    if (e != cudaSuccess) return cuda_fail(e);

    ConvParams cp{};
    cp.q = q; cp.k = k; cp.v = v;
    cp.wq = conv_w_q; cp.wk = conv_w_k; cp.wv = conv_w_v;
    cp.conv_in = conv_state_in;
    cp.qh = (float *)(ws + L.off_qh); cp.kh = (float *)(ws + L.off_kh);
    cp.vh = (float *)(ws + L.off_vh);
    cp.cu = cu; cp.cfirst = cfirst;
    cp.n_seqs = n_seqs; cp.n_qk = cfg->n_qk_heads; cp.n_v = cfg->n_v_heads;
    cp.q_scale = cfg->q_scale; cp.eps = cfg->l2_eps; cp.act = cfg->conv_activation;
    ScanParams sp{};
    sp.qh = (const float *)(ws + L.off_qh); sp.kh = (const float *)(ws + L.off_kh);
    sp.vh = (const float *)(ws + L.off_vh);
    sp.alpha = alpha; sp.beta = beta; sp.cu = cu; sp.cfirst = cfirst;
    sp.max_chunks = L.max_chunks;
    sp.init = initial_state; sp.fin = final_state; sp.out = out;
    sp.n_seqs = n_seqs; sp.n_qk = cfg->n_qk_heads; sp.n_v = cfg->n_v_heads;
    if (!bf) {
        // fp32 inputs: conv + L2 rows, then the fp32 CUDA-core chunked scan (one pass)
        if (total_tokens > 0) {
            e = launch_conv_l2(cp, false, /*tiles=*/false, L.max_chunks, total_tokens, stream);
            if (e != cudaSuccess) return cuda_fail(e);
        }
        e = launch_scan_simt(sp, false, out_dtype == GDN_BF16, stream);
        if (e == cudaSuccess && gate.z && total_tokens > 0)
            e = launch_output_gate(out, false, gate.z, gate.z_dtype == GDN_BF16, gate.w, gate.eps, out, false,
                                   total_tokens * cfg->n_v_heads, stream);
        if (e != cudaSuccess) return cuda_fail(e);
    } else {
        // bf16 inputs: per chunk range, conv + L2 tiles and the state-independent chunk work of
        // every chunk of the range at once, then the chains of the range.  With several ranges
        // the tiles of range r+1 are made on an auxiliary stream into the other buffer while
        // the chains run range r on the caller's stream; the state passes from range to range
        // through the final-state buffer (or a workspace carry).
        sp.gate_z = gate.z; sp.gate_z_bf16 = gate.z_dtype == GDN_BF16;
        sp.gate_w = gate.w; sp.gate_eps = gate.eps;
        sp.carry_in = sp.carry_out = final_state;
        if (L.n_ranges > 1 && !final_state) sp.carry_in = sp.carry_out = (float *)(ws + L.off_carry);
        AuxStream *aux = nullptr;
        if (L.n_ranges > 1) {
            e = aux_stream(&aux);
            if (e == cudaSuccess) e = cudaEventRecord(aux->ev_tab, stream);   // the tables are ready
            if (e == cudaSuccess) e = cudaStreamWaitEvent(aux->stream, aux->ev_tab, 0);
            if (e != cudaSuccess) return cuda_fail(e);
        }
        for (int r = 0; r < L.n_ranges && e == cudaSuccess; ++r) {
            const int buf = r % L.n_buf;
            unsigned char *tb = ws + L.off_tiles + (size_t)buf * L.buf_bytes;
            ChunkRange rg = L.range0;
            rg.r = r;
            rg.last = r == L.n_ranges - 1;
            cp.rg = sp.rg = rg;
            cp.slots = sp.slots = L.slots;
            cp.kq = (float *)(tb + L.b_kq); cp.kmn = (float *)(tb + L.b_kmn); cp.vi = (float *)(tb + L.b_vi);
            cp.cseq = (int32_t *)(tb + L.b_cseq);
            sp.kq = cp.kq; sp.kmn = cp.kmn; sp.vi = cp.vi; sp.cseq = cp.cseq;
            sp.tb = (float *)(tb + L.b_tb); sp.tg = (float *)(tb + L.b_tg); sp.pm = (float *)(tb + L.b_pm);
            sp.gr = (float *)(tb + L.b_gr);
            cudaStream_t ps = aux ? aux->stream : stream;   // where this range's tiles are made
            if (aux && r >= L.n_buf) e = cudaStreamWaitEvent(ps, aux->ev_chain[buf], 0);   // buffer free
            if (e == cudaSuccess && total_tokens > 0) e = launch_conv_l2(cp, true, /*tiles=*/true, L.slots, total_tokens, ps);
            if (e == cudaSuccess && total_tokens > 0) e = launch_chunk_prep(sp, total_tokens, true, ps);
            if (e == cudaSuccess && aux) e = cudaEventRecord(aux->ev_prep[buf], ps);
            if (e == cudaSuccess && aux) e = cudaStreamWaitEvent(stream, aux->ev_prep[buf], 0);
            if (e == cudaSuccess) e = launch_prefill_tc(sp, total_tokens, true, out_dtype == GDN_BF16, stream);
            if (e == cudaSuccess && aux) e = cudaEventRecord(aux->ev_chain[buf], stream);
        }
        if (e != cudaSuccess) return cuda_fail(e);
    }
    // last, on the caller's stream: every kernel that reads conv_state_in (the conv passes on
    // either stream) is ordered before this one, so conv_state_out may alias it
    if (conv_state_out) {
        e = launch_conv_state_out(q, k, v, conv_state_in, conv_state_out, cu, n_seqs,
                                  cfg->n_qk_heads, cfg->n_v_heads, bf, stream);
        if (e != cudaSuccess) return cuda_fail(e);
    }
    return GDN_OK;
}

extern "C" {

gdn_status gdn_prefill(const gdn_config *cfg, gdn_dtype dtype, gdn_dtype out_dtype, const void *q, const void *k,
                       const void *v, const float *conv_w_q, const float *conv_w_k, const float *conv_w_v,
                       const void *alpha, const void *beta, const int32_t *cu_seqlens, int n_seqs,
                       int64_t total_tokens, int64_t max_seqlen, const float *initial_state, float *final_state,
                       const void *conv_state_in, void *conv_state_out, void *out, void *workspace,
                       size_t workspace_bytes, cudaStream_t stream) {
    return prefill_impl(cfg, dtype, out_dtype, q, k, v, conv_w_q, conv_w_k, conv_w_v, alpha, beta, cu_seqlens,
                        n_seqs, total_tokens, max_seqlen, initial_state, final_state, conv_state_in,
                        conv_state_out, out, workspace, workspace_bytes, GateArgs{}, stream);
}

gdn_status gdn_prefill_gated(const gdn_config *cfg, gdn_dtype dtype, gdn_dtype out_dtype, const void *q,
                             const void *k, const void *v, const float *conv_w_q, const float *conv_w_k,
                             const float *conv_w_v, const void *alpha, const void *beta, const int32_t *cu_seqlens,
                             int n_seqs, int64_t total_tokens, int64_t max_seqlen, const float *initial_state,
                             float *final_state, const void *conv_state_in, void *conv_state_out, const void *z,
                             gdn_dtype z_dtype, const float *norm_w, float norm_eps, void *out, void *workspace,
                             size_t workspace_bytes, cudaStream_t stream) {
    if (!z) return GDN_ERR_INVALID_ARG;
    GateArgs g;
    g.z = z; g.z_dtype = z_dtype; g.w = norm_w; g.eps = norm_eps;
    return prefill_impl(cfg, dtype, out_dtype, q, k, v, conv_w_q, conv_w_k, conv_w_v, alpha, beta, cu_seqlens,
                        n_seqs, total_tokens, max_seqlen, initial_state, final_state, conv_state_in,
                        conv_state_out, out, workspace, workspace_bytes, g, stream);
}

gdn_status gdn_decode_step(const gdn_config *cfg, gdn_dtype dtype, gdn_dtype out_dtype,
                           const void *q, const void *k,
                           const void *v, const float *conv_w_q, const float *conv_w_k,
                           const float *conv_w_v, const void *alpha, const void *beta, float *state,
                           void *conv_state, const int32_t *state_slots, int n_state_rows,
                           void *out, int batch, cudaStream_t stream) {
    gdn_status st = check_config(cfg, dtype);
    if (st != GDN_OK) return st;
    if (out_dtype != GDN_BF16 && out_dtype != GDN_F32) return GDN_ERR_INVALID_ARG;
    if (batch < 0 || n_state_rows < 0) return GDN_ERR_INVALID_ARG;
    if (batch == 0) return GDN_OK;
    if (!state_slots && n_state_rows < batch) return GDN_ERR_INVALID_ARG;
    if ((int64_t)batch * cfg->n_qk_heads >= ((int64_t)1 << 31)) return GDN_ERR_UNSUPPORTED;
    const size_t eb = dtype == GDN_BF16 ? 2 : 4;
    if (!q || !k || !v || !alpha || !beta || !state || !out) return GDN_ERR_INVALID_ARG;
    if (!conv_w_q || !conv_w_k || !conv_w_v) return GDN_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
        !aligned(state, 16) || !aligned(conv_w_q, 16) || !aligned(conv_w_k, 16) ||
        !aligned(conv_w_v, 16))
        return GDN_ERR_INVALID_ARG;
    if (!aligned(alpha, eb) || !aligned(beta, eb)) return GDN_ERR_INVALID_ARG;
    if (conv_state && !aligned(conv_state, 16)) return GDN_ERR_INVALID_ARG;
    if (state_slots && !aligned(state_slots, 4)) return GDN_ERR_INVALID_ARG;
    st = check_device();
    if (st != GDN_OK) return st;

    DecodeParams p{};
    p.q = q; p.k = k; p.v = v;
    p.wq = conv_w_q; p.wk = conv_w_k; p.wv = conv_w_v;
    p.alpha = alpha; p.beta = beta;
    p.state = state; p.conv = conv_state; p.slots = state_slots;
    p.n_rows = n_state_rows; p.batch = batch;
    p.n_qk = cfg->n_qk_heads; p.n_v = cfg->n_v_heads;
    p.q_scale = cfg->q_scale; p.eps = cfg->l2_eps; p.act = cfg->conv_activation;
    p.out = out;
    cudaError_t e = launch_decode(p, dtype == GDN_BF16, out_dtype == GDN_BF16, stream);
    if (e != cudaSuccess) return cuda_fail(e);
    return GDN_OK;
}

gdn_status gdn_decode_multi(const gdn_config *cfg, gdn_dtype dtype, gdn_dtype out_dtype,
                            const void *q, const void *k, const void *v, const float *conv_w_q,
                            const float *conv_w_k, const float *conv_w_v, const void *alpha,
                            const void *beta, float *state, void *conv_state,
                            const int32_t *state_slots, int n_state_rows, float *state_ckpt,
                            void *conv_ckpt, void *out, int batch, int n_tok, cudaStream_t stream) {
    gdn_status st = check_config(cfg, dtype);
    if (st != GDN_OK) return st;
    if (out_dtype != GDN_BF16 && out_dtype != GDN_F32) return GDN_ERR_INVALID_ARG;
    if (batch < 0 || n_state_rows < 0 || n_tok < 1) return GDN_ERR_INVALID_ARG;
    if (n_tok > gdn::kMaxDecTok) return GDN_ERR_UNSUPPORTED;
    if (batch == 0) return GDN_OK;
    if (!state_slots && n_state_rows < batch) return GDN_ERR_INVALID_ARG;
    if ((int64_t)batch * cfg->n_qk_heads >= ((int64_t)1 << 31)) return GDN_ERR_UNSUPPORTED;
    const size_t eb = dtype == GDN_BF16 ? 2 : 4;
    if (!q || !k || !v || !alpha || !beta || !state || !out) return GDN_ERR_INVALID_ARG;
    if (!conv_w_q || !conv_w_k || !conv_w_v) return GDN_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
        !aligned(state, 16) || !aligned(conv_w_q, 16) || !aligned(conv_w_k, 16) ||
        !aligned(conv_w_v, 16))
        return GDN_ERR_INVALID_ARG;
    if (!aligned(alpha, eb) || !aligned(beta, eb)) return GDN_ERR_INVALID_ARG;
    if (conv_state && !aligned(conv_state, 16)) return GDN_ERR_INVALID_ARG;
    if (state_ckpt && !aligned(state_ckpt, 16)) return GDN_ERR_INVALID_ARG;
    if (conv_ckpt && !aligned(conv_ckpt, 16)) return GDN_ERR_INVALID_ARG;
    if (state_slots && !aligned(state_slots, 4)) return GDN_ERR_INVALID_ARG;
    st = check_device();
    if (st != GDN_OK) return st;

    DecodeParams p{};
    p.q = q; p.k = k; p.v = v;
    p.wq = conv_w_q; p.wk = conv_w_k; p.wv = conv_w_v;
    p.alpha = alpha; p.beta = beta;
    p.state = state; p.conv = conv_state; p.slots = state_slots;
    p.n_rows = n_state_rows; p.batch = batch;
    p.n_qk = cfg->n_qk_heads; p.n_v = cfg->n_v_heads;
    p.q_scale = cfg->q_scale; p.eps = cfg->l2_eps; p.act = cfg->conv_activation;
    p.out = out;
    p.n_tok = n_tok; p.state_ckpt = state_ckpt; p.conv_ckpt = conv_ckpt;
    cudaError_t e = launch_decode_multi(p, dtype == GDN_BF16, out_dtype == GDN_BF16, stream);
    if (e != cudaSuccess) return cuda_fail(e);
    return GDN_OK;
}

gdn_status gdn_output_gate(const gdn_config *cfg, gdn_dtype y_dtype, gdn_dtype z_dtype,
                           gdn_dtype out_dtype, const void *y, const void *z, const float *norm_w,
                           float eps, void *out, int64_t n_tokens, cudaStream_t stream) {
    if (!cfg) return GDN_ERR_INVALID_ARG;
    if (cfg->n_v_heads <= 0) return GDN_ERR_INVALID_ARG;
    if (cfg->d_v != 128) return GDN_ERR_UNSUPPORTED;
    for (gdn_dtype d : {y_dtype, z_dtype, out_dtype})
        if (d != GDN_BF16 && d != GDN_F32) return GDN_ERR_INVALID_ARG;
    if (n_tokens < 0 || !(eps >= 0.f) || !std::isfinite(eps)) return GDN_ERR_INVALID_ARG;
    if (n_tokens == 0) return GDN_OK;
    if (!y || !z || !norm_w || !out) return GDN_ERR_INVALID_ARG;
    if (!aligned(y, 16) || !aligned(z, 16) || !aligned(norm_w, 16) || !aligned(out, 16)) return GDN_ERR_INVALID_ARG;
    if (n_tokens > ((int64_t)1 << 40) / cfg->n_v_heads) return GDN_ERR_UNSUPPORTED;
    gdn_status st = check_device();
    if (st != GDN_OK) return st;
    cudaError_t e = launch_output_gate(y, y_dtype == GDN_BF16, z, z_dtype == GDN_BF16, norm_w, eps, out,
                                       out_dtype == GDN_BF16, n_tokens * cfg->n_v_heads, stream);
    if (e != cudaSuccess) return cuda_fail(e);
    return GDN_OK;
}

gdn_status gdn_affine_combine(const gdn_config *cfg, const float *M, const float *B, int n_spans, const float *S0,
                              float *S_in, cudaStream_t stream) {
    if (!cfg || cfg->n_v_heads <= 0) return GDN_ERR_INVALID_ARG;
    if (cfg->d_k != 128 || cfg->d_v != 128) return GDN_ERR_UNSUPPORTED;
    if (cfg->n_v_heads > 65535) return GDN_ERR_UNSUPPORTED;
    if (n_spans < 0 || !S_in || !aligned(S_in, 16)) return GDN_ERR_INVALID_ARG;
    if (n_spans > 0 && (!M || !B || !aligned(M, 16) || !aligned(B, 16))) return GDN_ERR_INVALID_ARG;
    if (S0 && !aligned(S0, 16)) return GDN_ERR_INVALID_ARG;
    gdn_status st = check_device();
    if (st != GDN_OK) return st;
    cudaError_t e = launch_affine_combine(M, B, S0, S_in, n_spans, cfg->n_v_heads, stream);
    if (e != cudaSuccess) return cuda_fail(e);
    return GDN_OK;
}

// ------------------------------------------------------------------ QSA indexer
static bool qsa_scalars_ok(float eps, float theta) {
    return std::isfinite(eps) && eps >= 0.f && std::isfinite(theta) && theta > 0.f;
}
// the select workspace keeps each query's scores on a 128-byte aligned row
static int64_t qsa_row_stride(int nb_max) { return ((int64_t)nb_max + 31) & ~(int64_t)31; }
static bool qsa_sizes_ok(int B, int n, int nb_max) {
    return B >= 0 && n >= 0 && nb_max >= 1 && B <= 65535 && nb_max < (1 << 29) &&
           (int64_t)B * nb_max < ((int64_t)1 << 31) - 256;
}

gdn_status gdn_qsa_block_keys(const void *k, const float *w_k, const int32_t *kpos, int B, int Tn,
                              float eps, float theta, void *kbar, int nb_max, cudaStream_t stream) {
    if (!qsa_sizes_ok(B, Tn, nb_max) || Tn % 4 != 0 || !qsa_scalars_ok(eps, theta)) return GDN_ERR_INVALID_ARG;
    if ((int64_t)B * Tn > ((int64_t)1 << 36)) return GDN_ERR_UNSUPPORTED;
    if (B == 0 || Tn == 0) return GDN_OK;
    if (!k || !w_k || !kpos || !kbar) return GDN_ERR_INVALID_ARG;
    if (!aligned(k, 16) || !aligned(w_k, 16) || !aligned(kpos, 16) || !aligned(kbar, 16)) return GDN_ERR_INVALID_ARG;
    gdn_status st = check_device();
    if (st != GDN_OK) return st;
    cudaError_t e = launch_qsa_block_keys(k, w_k, kpos, B, Tn, eps, theta, kbar, nb_max, stream);
    if (e != cudaSuccess) return cuda_fail(e);
    return GDN_OK;
}

static gdn_status qsa_query_args(const void *q, const float *w_q, const int32_t *qpos, const void *kbar,
                                 const int32_t *n_blocks, int B, int Qn, int nb_max, float eps, float theta) {
    if (!qsa_sizes_ok(B, Qn, nb_max) || !qsa_scalars_ok(eps, theta)) return GDN_ERR_INVALID_ARG;
    if ((int64_t)B * Qn >= ((int64_t)1 << 31)) return GDN_ERR_UNSUPPORTED;
    if (B == 0 || Qn == 0) return GDN_OK;
    if (!q || !w_q || !qpos || !kbar || !n_blocks) return GDN_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(w_q, 16) || !aligned(qpos, 16) || !aligned(kbar, 16) || !aligned(n_blocks, 16))
        return GDN_ERR_INVALID_ARG;
    return GDN_OK;
}

gdn_status gdn_qsa_block_scores(const void *q, const float *w_q, const int32_t *qpos, const void *kbar,
                                const int32_t *n_blocks, int B, int Qn, int nb_max, float eps, float theta,
                                float *scores, cudaStream_t stream) {
    gdn_status st = qsa_query_args(q, w_q, qpos, kbar, n_blocks, B, Qn, nb_max, eps, theta);
    if (st != GDN_OK) return st;
    if (B == 0 || Qn == 0) return GDN_OK;
    if (!scores || !aligned(scores, 16)) return GDN_ERR_INVALID_ARG;
    st = check_device();
    if (st != GDN_OK) return st;
    cudaError_t e = launch_qsa_scores(q, w_q, qpos, kbar, n_blocks, B, Qn, nb_max, eps, theta, scores, nb_max, stream);
    if (e != cudaSuccess) return cuda_fail(e);
    return GDN_OK;
}

gdn_status gdn_qsa_select_workspace_size(int B, int Qn, int nb_max, size_t *bytes) {
    if (!bytes) return GDN_ERR_INVALID_ARG;
    if (!qsa_sizes_ok(B, Qn, nb_max)) return GDN_ERR_INVALID_ARG;
    *bytes = (((size_t)B * Qn * qsa_row_stride(nb_max) * 4) + 255) & ~(size_t)255;
    return GDN_OK;
}

gdn_status gdn_qsa_select(const void *q, const float *w_q, const int32_t *qpos, const void *kbar,
                          const int32_t *n_blocks, int B, int Qn, int nb_max, float eps, float theta,
                          int32_t *blocks, int32_t *tokens, void *workspace, size_t workspace_bytes,
                          cudaStream_t stream) {
    gdn_status st = qsa_query_args(q, w_q, qpos, kbar, n_blocks, B, Qn, nb_max, eps, theta);
    if (st != GDN_OK) return st;
    if (B == 0 || Qn == 0) return GDN_OK;
    if (!blocks || !aligned(blocks, 16) || (tokens && !aligned(tokens, 16))) return GDN_ERR_INVALID_ARG;
    size_t need = 0;
    gdn_qsa_select_workspace_size(B, Qn, nb_max, &need);
    if (!workspace || !aligned(workspace, 256) || workspace_bytes < need) return GDN_ERR_WORKSPACE;
    st = check_device();
    if (st != GDN_OK) return st;
    float *scores = static_cast<float *>(workspace);
    const int64_t ld = qsa_row_stride(nb_max);
    cudaError_t e = launch_qsa_scores(q, w_q, qpos, kbar, n_blocks, B, Qn, nb_max, eps, theta, scores, ld, stream);
    if (e != cudaSuccess) return cuda_fail(e);
    e = launch_qsa_topk(scores, ld, qpos, n_blocks, B, Qn, nb_max, blocks, tokens, stream);
    if (e != cudaSuccess) return cuda_fail(e);
    return GDN_OK;
}

}  // extern "C"
