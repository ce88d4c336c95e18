// GDN output tail: gated RMS normalisation of the state readout y, per (token, V head).
//
// Page "ARCHITECTURE PREVIEW / FIELD NOTES", section 03 (figure caption): y passes a
// normalisation and an output gate before the output projection (the page gives no
// formula; this is the plainest reading):
//     o = y / sqrt(mean(y^2) + eps) * w * SiLU(z),     SiLU(z) = z / (1 + exp(-z))
// over the 128 values of one (token, V head), w [128] shared by the heads.
// Memory-bound: one warp per (token, head) row, 4 channels per lane, each value read once
// and written once with 8- or 16-byte accesses; out may be y itself (same dtype).
#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {

namespace {
constexpr int kGateThreads = 256;
constexpr int kRowsPerCta = kGateThreads / 32;
}  // namespace

template <class TY, class TZ, class TO>
__global__ void __launch_bounds__(kGateThreads) output_gate_kernel(const TY *y, const TZ *z, const float *w,
                                                                   float eps, TO *out, int64_t rows) {
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * kRowsPerCta + (threadIdx.x >> 5);
    if (row >= rows) return;
    const int64_t off = row * kHeadDim + 4 * lane;
    float yv[4], zv[4];
    ld4(y + off, yv);
    ld4(z + off, zv);
    const float4 wv = *reinterpret_cast<const float4 *>(w + 4 * lane);
    float ss = yv[0] * yv[0] + yv[1] * yv[1] + yv[2] * yv[2] + yv[3] * yv[3];
    ss = warp_sum(ss);
    const float inv = rsqrtf(ss * (1.f / kHeadDim) + eps);
    const float ww[4] = {wv.x, wv.y, wv.z, wv.w};
    float o[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) o[c] = yv[c] * inv * ww[c] * (zv[c] / (1.f + __expf(-zv[c])));
    st4(out + off, o);
}

cudaError_t launch_output_gate(const void *y, bool y_bf16, const void *z, bool z_bf16, const float *w,
                               float eps, void *out, bool out_bf16, int64_t rows, cudaStream_t s) {
    if (rows <= 0) return cudaSuccess;
    const int64_t grid = (rows + kRowsPerCta - 1) / kRowsPerCta;
    if (grid >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
    TraceLaunch tl(s, "output_gate");
#define GDN_GATE(TY, TZ, TO)                                                                   \
    output_gate_kernel<TY, TZ, TO><<<(unsigned)grid, kGateThreads, 0, s>>>((const TY *)y, (const TZ *)z, w, eps, \
                                                                          (TO *)out, rows)
    if (y_bf16) {
        if (z_bf16) { if (out_bf16) GDN_GATE(bf16, bf16, bf16); else GDN_GATE(bf16, bf16, float); }
        else        { if (out_bf16) GDN_GATE(bf16, float, bf16); else GDN_GATE(bf16, float, float); }
    } else {
        if (z_bf16) { if (out_bf16) GDN_GATE(float, bf16, bf16); else GDN_GATE(float, bf16, float); }
        else        { if (out_bf16) GDN_GATE(float, float, bf16); else GDN_GATE(float, float, float); }
    }
#undef GDN_GATE
    return cudaGetLastError();
}

}  // namespace gdn
