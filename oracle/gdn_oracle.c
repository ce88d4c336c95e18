/*
 * gdn_oracle.c -- plain, slow, fp64 reference ("oracle") of the Gated DeltaNet
 * token mixer.  TEST INFRASTRUCTURE ONLY: it is built and called by the tests,
 * by the package's smoke check and by the benchmark's CPU-baseline leg, never by
 * the product path.  It shares no code, header or table with the CUDA library.
 *
 * What it computes, per packed sequence b and per value head h (QK head
 * g = h / (Hv/Hqk)), everything in double precision on the stored input values:
 *
 *  1. ShortConv (the page "ARCHITECTURE PREVIEW / FIELD NOTES", section 03
 *     "Attention", figure caption of the GDN diagram: q, k and v each pass a
 *     kernel-4 ShortConv first; config table of section 01: conv kernel 4).
 *     Read as a causal depthwise convolution without bias or activation:
 *         x'_t[c] = sum_{j=0..W-1} w[c][j] * x_{t-(W-1)+j}[c]
 *     so tap W-1 multiplies the current row.  Rows before the start of a
 *     sequence come from the conv state (oldest row first) when one is given,
 *     else they are zero.  Packed sequences never see each other's rows.
 *     Optionally (conv_silu = 1, off by default: the page names no activation) every
 *     conv output passes SiLU(x) = x / (1 + e^-x) before step 2.
 *  2. Per-head L2 normalisation of q and k after the conv:
 *         q^ = q' * q_scale / sqrt(sum q'^2 + eps),  k^ = k' / sqrt(sum k'^2 + eps).
 *     v is not normalised.
 *  3. The gated delta rule in its four-equation form (same page, section 03,
 *     "GATED DELTANET" equations), with the state S indexed [d_k][d_v]:
 *         S~  = alpha_t * S_{t-1}
 *         e_t = v_t - S~^T k_t
 *         S_t = S~ + beta_t * k_t e_t^T
 *         y_t = S_t^T q_t            (the read uses the updated state S_t)
 *     S starts from the initial state (or zero) and the last S is returned.
 *  4. The returned conv state holds the last W-1 raw rows seen by the sequence
 *     (the given conv-state rows followed by the sequence's own rows).
 *
 * Parity pins (tests/test_oracle_pins.py) hold this file to what the page and
 * the mathematics fix: the page's expanded one-step form, brute-force transition
 * products on tiny inputs, the beta=0 closed form, exact recall with
 * orthonormal keys at alpha=beta=1, chunked == sequential, split == whole.
 *
 * Compile-time planted mistakes (-DGDN_ORACLE_MUTANT=n) exist only so that a
 * test can show that the pins catch each of them; the normal build has none.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#ifndef GDN_ORACLE_MUTANT
#define GDN_ORACLE_MUTANT 0
#endif

typedef struct {
    int n_qk_heads, n_v_heads, d_k, d_v, conv_width;
    double q_scale, l2_eps;
    int conv_silu;   /* 1: SiLU on every conv output (before the L2 norm of q, k) */
} oracle_shape;

/* raw value of channel c of conv input row s of sequence b (s < 0: history) */
static double conv_row_value(const double *x, int64_t row_stride, int64_t tok0, int s, int c,
                             const double *conv_state, int64_t cs_row_stride, int cs_offset,
                             int b, int W)
{
    if (s >= 0) return x[(tok0 + s) * row_stride + c];
    if (!conv_state) return 0.0;
    /* conv state rows: index 0 is the oldest, W-2 the newest (row s = -1) */
    int r = (W - 1) + s;
    if (r < 0) return 0.0;
    return conv_state[((int64_t)b * (W - 1) + r) * cs_row_stride + cs_offset + c];
}

/* ShortConv of one channel at position s of sequence b */
static double short_conv(const double *x, int64_t row_stride, int64_t tok0, int s, int c,
                         const double *w, const double *conv_state, int64_t cs_row_stride,
                         int cs_offset, int b, int W)
{
    double acc = 0.0;
    for (int j = 0; j < W; ++j) {
#if GDN_ORACLE_MUTANT == 4
        /* planted: taps reversed (tap 0 on the current row) */
        double xv = conv_row_value(x, row_stride, tok0, s - j, c, conv_state, cs_row_stride,
                                   cs_offset, b, W);
#else
        double xv = conv_row_value(x, row_stride, tok0, s - (W - 1) + j, c, conv_state,
                                   cs_row_stride, cs_offset, b, W);
#endif
        acc += w[(int64_t)c * W + j] * xv;
    }
    return acc;
}

/* SiLU(x) = x * sigmoid(x) = x / (1 + e^-x) */
static double silu(double x) { return x / (1.0 + exp(-x)); }

/* conv (then SiLU when `act`) then L2 over the head's d channels starting at channel c0 */
static void conv_l2_head(double *dst, const double *x, int64_t row_stride, int64_t tok0, int s,
                         int c0, int d, const double *w, const double *conv_state,
                         int64_t cs_row_stride, int cs_offset, int b, int W, int normalize,
                         double scale, double eps, int act)
{
    double ss = 0.0;
    for (int i = 0; i < d; ++i) {
        dst[i] = short_conv(x, row_stride, tok0, s, c0 + i, w, conv_state, cs_row_stride,
                            cs_offset, b, W);
#if GDN_ORACLE_MUTANT != 7
        if (act) dst[i] = silu(dst[i]);
#endif
        ss += dst[i] * dst[i];
    }
    if (normalize) {
        double inv = scale / sqrt(ss + eps);
        for (int i = 0; i < d; ++i) dst[i] *= inv;
    }
#if GDN_ORACLE_MUTANT == 7
    /* planted: the activation after the normalisation */
    if (act)
        for (int i = 0; i < d; ++i) dst[i] = silu(dst[i]);
#endif
}

/*
 * oracle_gdn_prefill: the full mixer over packed sequences.
 *   q, k        [T, Hqk, dk]      raw (pre-conv) values
 *   v           [T, Hv, dv]
 *   wq, wk      [Hqk*dk, W]       wv [Hv*dv, W]
 *   alpha, beta [T, Hv]
 *   cu_seqlens  [n_seqs+1]        non-decreasing, cu[0] = 0
 *   init_state  [n_seqs, Hv, dk, dv] or NULL (zero)
 *   conv_state  [n_seqs, W-1, 2*Hqk*dk + Hv*dv] raw rows q|k|v, oldest first, or NULL
 *   heads       list of V heads to compute (NULL: all Hv); outputs of other heads
 *               are left untouched
 *   out         [T, Hv, dv]
 *   final_state [n_seqs, Hv, dk, dv] (may be NULL)
 *   conv_state_out [n_seqs, W-1, channels] (may be NULL; may alias conv_state only
 *               if the caller copies first -- this oracle reads conv_state while
 *               writing conv_state_out at the end)
 * Returns 0, or -1 on a bad argument.
 */
int oracle_gdn_prefill(const oracle_shape *sh,
                       const double *q, const double *k, const double *v,
                       const double *wq, const double *wk, const double *wv,
                       const double *alpha, const double *beta,
                       const int32_t *cu_seqlens, int n_seqs,
                       const double *init_state, const double *conv_state,
                       const int32_t *heads, int n_heads_sel,
                       double *out, double *final_state, double *conv_state_out,
                       int n_threads)
{
    const int H = sh->n_qk_heads, Hv = sh->n_v_heads, dk = sh->d_k, dv = sh->d_v;
    const int W = sh->conv_width;
    if (H <= 0 || Hv <= 0 || Hv % H != 0 || dk <= 0 || dv <= 0 || W < 1 || n_seqs < 0)
        return -1;
    const int G = Hv / H;
    const int64_t chans = (int64_t)2 * H * dk + (int64_t)Hv * dv;
    const int nsel = heads ? n_heads_sel : Hv;
    const int64_t units = (int64_t)n_seqs * nsel;

#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#else
    (void)n_threads;
#endif

    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t u = 0; u < units; ++u) {
        const int b = (int)(u / nsel);
        const int h = heads ? heads[u % nsel] : (int)(u % nsel);
        if (h < 0 || h >= Hv) { bad |= 1; continue; }
#if GDN_ORACLE_MUTANT == 5
        const int g = h % H;            /* planted: interleaved head mapping */
#else
        const int g = h / G;            /* V heads [g*G, (g+1)*G) share QK head g */
#endif
        const int64_t tok0 = cu_seqlens[b];
        const int L = cu_seqlens[b + 1] - cu_seqlens[b];
        double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
        double *qh = (double *)malloc(sizeof(double) * dk);
        double *kh = (double *)malloc(sizeof(double) * dk);
        double *vh = (double *)malloc(sizeof(double) * dv);
        double *e = (double *)malloc(sizeof(double) * dv);
        if (init_state)
            for (int64_t i = 0; i < (int64_t)dk * dv; ++i)
                S[i] = init_state[(((int64_t)b * Hv + h) * dk) * dv + i];
        else
            memset(S, 0, sizeof(double) * (size_t)dk * dv);

        for (int t = 0; t < L; ++t) {
            /* 1-2: ShortConv then L2 norm (q, k) */
            conv_l2_head(qh, q, (int64_t)H * dk, tok0, t, g * dk, dk, wq, conv_state, chans, 0,
                         b, W, 1, sh->q_scale, sh->l2_eps, sh->conv_silu);
            conv_l2_head(kh, k, (int64_t)H * dk, tok0, t, g * dk, dk, wk, conv_state, chans,
                         H * dk, b, W, 1, 1.0, sh->l2_eps, sh->conv_silu);
            conv_l2_head(vh, v, (int64_t)Hv * dv, tok0, t, h * dv, dv, wv, conv_state, chans,
                         2 * H * dk, b, W, 0, 1.0, 0.0, sh->conv_silu);
            const double a = alpha[(tok0 + t) * Hv + h];
            const double be = beta[(tok0 + t) * Hv + h];

            /* 3: S~ = alpha S */
            for (int64_t i = 0; i < (int64_t)dk * dv; ++i) S[i] *= a;
            /* e = v - S~^T k */
            for (int j = 0; j < dv; ++j) {
                double p = 0.0;
                for (int i = 0; i < dk; ++i)
#if GDN_ORACLE_MUTANT == 3
                    p += S[(int64_t)j * dv + i] * kh[i];   /* planted: transposed state */
#else
                    p += S[(int64_t)i * dv + j] * kh[i];
#endif
#if GDN_ORACLE_MUTANT == 1
                e[j] = vh[j] - p / a;                      /* planted: error from undecayed S */
#else
                e[j] = vh[j] - p;
#endif
            }
#if GDN_ORACLE_MUTANT == 2
            /* planted: read before the write (y from S~) */
            for (int j = 0; j < dv; ++j) {
                double y = 0.0;
                for (int i = 0; i < dk; ++i) y += S[(int64_t)i * dv + j] * qh[i];
                if (out) out[((tok0 + t) * Hv + h) * dv + j] = y;
            }
#endif
            /* S = S~ + beta k e^T */
            for (int i = 0; i < dk; ++i) {
#if GDN_ORACLE_MUTANT == 6
                const double bk = kh[i];                   /* planted: beta dropped */
#else
                const double bk = be * kh[i];
#endif
                for (int j = 0; j < dv; ++j) S[(int64_t)i * dv + j] += bk * e[j];
            }
#if GDN_ORACLE_MUTANT != 2
            /* y = S^T q */
            for (int j = 0; j < dv; ++j) {
                double y = 0.0;
                for (int i = 0; i < dk; ++i) y += S[(int64_t)i * dv + j] * qh[i];
                if (out) out[((tok0 + t) * Hv + h) * dv + j] = y;
            }
#endif
        }
        if (final_state)
            for (int64_t i = 0; i < (int64_t)dk * dv; ++i)
                final_state[(((int64_t)b * Hv + h) * dk) * dv + i] = S[i];
        free(S); free(qh); free(kh); free(vh); free(e);
    }
    if (bad) return -1;

    /* 4: returned conv state = last W-1 raw rows (history rows, then the sequence's) */
    if (conv_state_out && W > 1) {
        for (int b = 0; b < n_seqs; ++b) {
            const int64_t tok0 = cu_seqlens[b];
            const int L = cu_seqlens[b + 1] - cu_seqlens[b];
            for (int r = 0; r < W - 1; ++r) {
                const int s = L - (W - 1) + r;   /* position of this row in the sequence */
                double *dst = conv_state_out + ((int64_t)b * (W - 1) + r) * chans;
                for (int64_t c = 0; c < chans; ++c) {
                    const double *x; int64_t stride, cc; int off;
                    if (c < (int64_t)H * dk) { x = q; stride = (int64_t)H * dk; cc = c; off = 0; }
                    else if (c < (int64_t)2 * H * dk) {
                        x = k; stride = (int64_t)H * dk; cc = c - (int64_t)H * dk; off = H * dk;
                    } else {
                        x = v; stride = (int64_t)Hv * dv; cc = c - (int64_t)2 * H * dk;
                        off = 2 * H * dk;
                    }
                    dst[c] = conv_row_value(x, stride, tok0, s, (int)cc, conv_state, chans, off,
                                            b, W);
                }
            }
        }
    }
    return 0;
}

/* The conv + L2 stage alone, for all tokens: qh,kh [T,Hqk,dk], vh [T,Hv,dv]. */
int oracle_gdn_conv_l2(const oracle_shape *sh,
                       const double *q, const double *k, const double *v,
                       const double *wq, const double *wk, const double *wv,
                       const int32_t *cu_seqlens, int n_seqs, const double *conv_state,
                       double *qh, double *kh, double *vh, int n_threads)
{
    const int H = sh->n_qk_heads, Hv = sh->n_v_heads, dk = sh->d_k, dv = sh->d_v;
    const int W = sh->conv_width;
    if (H <= 0 || Hv <= 0 || dk <= 0 || dv <= 0 || W < 1 || n_seqs < 0) return -1;
    const int64_t chans = (int64_t)2 * H * dk + (int64_t)Hv * dv;
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#else
    (void)n_threads;
#endif
#pragma omp parallel for schedule(dynamic, 1)
    for (int b = 0; b < n_seqs; ++b) {
        const int64_t tok0 = cu_seqlens[b];
        const int L = cu_seqlens[b + 1] - cu_seqlens[b];
        for (int t = 0; t < L; ++t) {
            for (int g = 0; g < H; ++g) {
                conv_l2_head(qh + ((tok0 + t) * H + g) * dk, q, (int64_t)H * dk, tok0, t, g * dk,
                             dk, wq, conv_state, chans, 0, b, W, 1, sh->q_scale, sh->l2_eps, sh->conv_silu);
                conv_l2_head(kh + ((tok0 + t) * H + g) * dk, k, (int64_t)H * dk, tok0, t, g * dk,
                             dk, wk, conv_state, chans, H * dk, b, W, 1, 1.0, sh->l2_eps, sh->conv_silu);
            }
            for (int h = 0; h < Hv; ++h)
                conv_l2_head(vh + ((tok0 + t) * Hv + h) * dv, v, (int64_t)Hv * dv, tok0, t,
                             h * dv, dv, wv, conv_state, chans, 2 * H * dk, b, W, 0, 1.0, 0.0,
                             sh->conv_silu);
        }
    }
    return 0;
}

int oracle_mutant_id(void) { return GDN_ORACLE_MUTANT; }
