// Shared device helpers of libgdn (storage-type loads/stores, warp reductions).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gdn {

constexpr int kHeadDim = 128;   // d_k = d_v
constexpr int kConvW = 4;       // ShortConv taps
constexpr int kChunk = 64;      // tokens per chunk of the chunked prefill
constexpr float kMinLogAlpha = -80.0f;  // log(alpha) floor: alpha <= e^-80 acts as a full reset

typedef __nv_bfloat16 bf16;

// ---------------------------------------------------------------- scalar conversions
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(bf16 x) { return __bfloat162float(x); }

template <class T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ bf16 from_f32<bf16>(float x) { return __float2bfloat16_rn(x); }

// ---------------------------------------------------------------- 4-wide vector access
// 4 consecutive elements: 16 B for fp32, 8 B for bf16 (caller guarantees alignment).
__device__ __forceinline__ void ld4(const float *p, float v[4]) {
    float4 t = *reinterpret_cast<const float4 *>(p);
    v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
}
__device__ __forceinline__ void ld4(const bf16 *p, float v[4]) {
    uint2 t = *reinterpret_cast<const uint2 *>(p);
    __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162 *>(&t.x);
    __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162 *>(&t.y);
    float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    v[0] = fa.x; v[1] = fa.y; v[2] = fb.x; v[3] = fb.y;
}
__device__ __forceinline__ void st4(float *p, const float v[4]) {
    *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
__device__ __forceinline__ void st4(bf16 *p, const float v[4]) {
    __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]);
    __nv_bfloat162 b = __floats2bfloat162_rn(v[2], v[3]);
    uint2 t;
    t.x = *reinterpret_cast<uint32_t *>(&a);
    t.y = *reinterpret_cast<uint32_t *>(&b);
    *reinterpret_cast<uint2 *>(p) = t;
}
// raw copy of 4 stored elements (no rounding): 16 B fp32 / 8 B bf16
__device__ __forceinline__ void cp4(float *dst, const float *src) {
    *reinterpret_cast<float4 *>(dst) = *reinterpret_cast<const float4 *>(src);
}
__device__ __forceinline__ void cp4(bf16 *dst, const bf16 *src) {
    *reinterpret_cast<uint2 *>(dst) = *reinterpret_cast<const uint2 *>(src);
}
__device__ __forceinline__ void zero4(float *dst) {
    *reinterpret_cast<float4 *>(dst) = make_float4(0.f, 0.f, 0.f, 0.f);
}
__device__ __forceinline__ void zero4(bf16 *dst) { *reinterpret_cast<uint2 *>(dst) = make_uint2(0u, 0u); }

// ---------------------------------------------------------------- reductions
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// the optional activation of the ShortConv outputs: SiLU(y) = y / (1 + e^-y) when act != 0
__device__ __forceinline__ float conv_act(float y, int act) { return act ? y / (1.f + expf(-y)) : y; }

__device__ __forceinline__ float safe_log_alpha(float a) {
    // alpha in (0, 1]; non-positive or tiny values act as a full reset
    return a > 0.f ? fmaxf(logf(a), kMinLogAlpha) : kMinLogAlpha;
}

// largest b in [0, n) with first[b] <= i, for a non-decreasing first[0..n]
__device__ __forceinline__ int upper_index(const int32_t *first, int n, int i) {
    int lo = 0, hi = n;  // invariant: first[lo] <= i < first[hi]
    while (hi - lo > 1) {
        int mid = (lo + hi) >> 1;
        if (__ldg(first + mid) <= i) lo = mid; else hi = mid;
    }
    return lo;
}

}  // namespace gdn
