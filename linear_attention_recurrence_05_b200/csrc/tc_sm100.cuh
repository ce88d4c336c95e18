// Thin wrappers over the sm_100a tensor-core (tcgen05) and mbarrier PTX used by the
// chunked prefill.  Operands are fp32 values read as TF32 (kind::tf32, 8 K-elements per
// instruction) or fp16 values (kind::f16, 16 K-elements per instruction); accumulators are
// fp32 in tensor memory.
//
// Shared-memory operand layouts for fp32 elements, made of 128-byte rows grouped in blocks
// of 32 columns (a [R x C] tile is C/32 blocks of R*128 bytes):
//  * K-major operands (rows = M or N index, columns = K index): 128-byte swizzle with
//    16-byte chunks, chunk c of row r at c ^ (r % 8) (what TMA's SWIZZLE_128B writes).
//    K step s (8 columns) starts at block(s/4) + (s%4)*32 B; SBO = 1024 B (8 rows).
//  * MN-major operands (rows = K index, columns = M or N index): 128-byte swizzle with
//    32-byte granules, granule g of row r at g ^ (r % 4) -- the only MN-major layout
//    the tensor core takes for 32-bit elements (TMA: SWIZZLE_128B_ATOM_32B).
//    K step s (8 rows) starts at +1024*s; LBO = R*128 B (next 32 columns), SBO = 512 B.
// A matrix contracted over both of its indices (K of a chunk: over features in K K^T
// and K S, over tokens in K^T u) is staged once per layout (here: [K;Q] K-major in fp32 for
// the feature contractions, K MN-major in fp16 for the token contraction).
//
// fp16 operands (kind::f16, 16 K-elements per instruction): 128-byte rows of 64 elements,
// 128-byte swizzle with 16-byte chunks (chunk c of row r at c ^ (r % 8)).
//  * K-major [R x 64]: element (r, c) at r*128 + ((c/8) ^ (r%8))*16 + (c%8)*2; K step s
//    (16 columns) starts at +32*s; SBO = 1024 B.
//  * MN-major [R x C] (rows = K index): blocks of 64 columns, R*128 bytes each; K step s
//    (16 rows) starts at +2048*s; LBO = R*128 B (next 64 columns), SBO = 1024 B (8 rows).
// A from tensor memory holds two fp16 per 32-bit column, the lower K index in the low half.
#pragma once

#include <stdint.h>
#include <cuda_fp16.h>

namespace gdn {
namespace tc {

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

// byte offset of element (r, c) of a [R x C] fp32 tile, K-major 128B swizzle
__host__ __device__ __forceinline__ uint32_t kmaj_off(int r, int c, int R) {
    return (uint32_t)((c >> 5) * R * 128 + r * 128 + ((((c & 31) >> 2) ^ (r & 7)) << 4) +
                      ((c & 3) << 2));
}

// byte offset of element (r, c) of a [R x 64] fp16 tile, K-major 128B swizzle
__host__ __device__ __forceinline__ uint32_t kmaj16_off(int r, int c) {
    return (uint32_t)(r * 128 + ((((c & 63) >> 3) ^ (r & 7)) << 4) + ((c & 7) << 1));
}
// byte offset of element (r, c) of a [R x C] fp16 tile, MN-major 128B swizzle
__host__ __device__ __forceinline__ uint32_t mn16_off(int r, int c, int R) {
    return (uint32_t)((c >> 6) * R * 128 + r * 128 + ((((c & 63) >> 3) ^ (r & 7)) << 4) + ((c & 7) << 1));
}
// two fp16 (nearest even) in one 32-bit word, `lo` in the low half
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// ------------------------------------------------------------------ descriptors
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo,
                                              uint32_t layout) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;                  // descriptor version for sm_100
    d |= (uint64_t)(layout & 7u) << 61;      // 2: 128B swizzle, 1: 128B with 32B granules
    return d;
}

// K-major view of a tile whose 32-column blocks are `blk` bytes apart, K step s
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t base, uint32_t blk, int s) {
    return smem_desc(base + (uint32_t)(s >> 2) * blk + (uint32_t)(s & 3) * 32, 16, 1024, 2);
}
// MN-major view of a tile with R rows (= K extent), K step s (8 rows)
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t base, int R, int s) {
    return smem_desc(base + (uint32_t)(s * 1024), (uint32_t)(R * 128), 512, 1);
}

// instruction descriptor: kind::tf32, fp32 accumulator, M x N, operand majors
__host__ __device__ constexpr uint32_t idesc_tf32(int M, int N, bool a_mn, bool b_mn) {
    return (1u << 4)                       // D format: f32
           | (2u << 7) | (2u << 10)        // A, B format: tf32
           | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16)
           | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// instruction descriptor: kind::f16 with fp16 A and B, fp32 accumulator, operand majors
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, bool a_mn, bool b_mn) {
    return (1u << 4)                       // D format: f32 (A, B format 0: f16)
           | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16)
           | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// instruction descriptor: kind::f16 with bf16 A and B, fp32 accumulator, both K-major
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
    return (1u << 4)                       // D format: f32
           | (1u << 7) | (1u << 10)        // A, B format: bf16
           | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// ------------------------------------------------------------------ MMA
__device__ __forceinline__ void mma_tf32(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate));
}

// one kind::f16 MMA, both operands from shared memory (K = 16 16-bit elements = 32 bytes of
// each operand row; fp16 or bf16 as the instruction descriptor says)
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate));
}

// D[M x N] (+)= A[M x K] B[K x N], K a multiple of 8, issued by one thread.
// A K-major: a_arg = byte distance between its 32-column blocks; A MN-major: a_arg = its
// row count R (= K).  Same for B.  Only the 14-bit start-address field changes from one
// K step to the next, so each step's descriptors are the first step's plus a constant.
template <int M, int N, int K, bool A_MN, bool B_MN>
__device__ __forceinline__ void gemm(uint32_t d_tmem, uint32_t a_base, uint32_t a_arg,
                                     uint32_t b_base, uint32_t b_arg, bool accumulate) {
    constexpr uint32_t id = idesc_tf32(M, N, A_MN, B_MN);
    const uint64_t a0 = A_MN ? desc_mnmajor(a_base, (int)a_arg, 0) : desc_kmajor(a_base, a_arg, 0);
    const uint64_t b0 = B_MN ? desc_mnmajor(b_base, (int)b_arg, 0) : desc_kmajor(b_base, b_arg, 0);
    const uint32_t a_blk16 = A_MN ? 0u : (a_arg >> 4), b_blk16 = B_MN ? 0u : (b_arg >> 4);
#pragma unroll
    for (int s = 0; s < K / 8; ++s) {
        // start-address step (16-byte units): MN-major +1024 B per step; K-major +32 B per
        // step inside a 32-column block, +block per 4 steps
        const uint32_t da = A_MN ? (uint32_t)(s * 64) : (uint32_t)((s >> 2) * a_blk16 + (s & 3) * 2);
        const uint32_t db = B_MN ? (uint32_t)(s * 64) : (uint32_t)((s >> 2) * b_blk16 + (s & 3) * 2);
        mma_tf32(d_tmem, a0 + da, b0 + db, id, (accumulate || s > 0) ? 1u : 0u);
    }
}

// D[128 x N] (+)= A[128 x K] B[K x N] in fp16 (kind::f16), A from tensor memory (K/2
// columns of packed pairs), B from shared memory: K-major [N x 64] (b_rows unused) or
// MN-major [K x N] with b_rows = K.
template <int N, int K, bool B_MN>
__device__ __forceinline__ void gemm_ts_f16(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_base, int b_rows,
                                            bool accumulate) {
    constexpr uint32_t id = idesc_f16(128, N, false, B_MN);
    const uint64_t b0 = B_MN ? smem_desc(b_base, (uint32_t)b_rows * 128u, 1024, 2) : smem_desc(b_base, 16, 1024, 2);
#pragma unroll
    for (int s = 0; s < K / 16; ++s) {
        const uint32_t db = B_MN ? (uint32_t)(s * 128) : (uint32_t)(s * 2);   // 16-byte units
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
            "r"(a_tmem + 8u * s), "l"(b0 + db), "r"(id), "r"((accumulate || s > 0) ? 1u : 0u));
    }
}

// D[M x N] (+)= A[M x K] B[K x N] in fp16 (kind::f16), both operands in shared memory: each
// K-major [rows x 64] (rows argument unused) or MN-major [K x M|N] with rows = K.
template <int M, int N, int K, bool A_MN, bool B_MN>
__device__ __forceinline__ void gemm_f16(uint32_t d_tmem, uint32_t a_base, int a_rows, uint32_t b_base, int b_rows,
                                         bool accumulate) {
    constexpr uint32_t id = idesc_f16(M, N, A_MN, B_MN);
    const uint64_t a0 = A_MN ? smem_desc(a_base, (uint32_t)a_rows * 128u, 1024, 2) : smem_desc(a_base, 16, 1024, 2);
    const uint64_t b0 = B_MN ? smem_desc(b_base, (uint32_t)b_rows * 128u, 1024, 2) : smem_desc(b_base, 16, 1024, 2);
#pragma unroll
    for (int s = 0; s < K / 16; ++s) {
        const uint32_t da = A_MN ? (uint32_t)(s * 128) : (uint32_t)(s * 2);   // 16-byte units
        const uint32_t db = B_MN ? (uint32_t)(s * 128) : (uint32_t)(s * 2);
        mma_bf16(d_tmem, a0 + da, b0 + db, id, (accumulate || s > 0) ? 1u : 0u);
    }
}

__device__ __forceinline__ void mma_commit(uint64_t *mbar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(mbar))
        : "memory");
}

// ------------------------------------------------------------------ fences
__device__ __forceinline__ void fence_before_sync() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after_sync() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// make this thread's generic-proxy shared-memory writes visible to the tensor core
__device__ __forceinline__ void fence_smem_to_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint64_t *m, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(m)), "r"(count));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *m, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(m)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Same, but the thread may sleep up to `hint_ns` nanoseconds inside the poll instead of
// returning at once, so that waiting warps leave the issue slots to the working ones.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t *m, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(m)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}
// Bounded wait on phase `parity`: returns false if it has not completed after
// `max_tries` polls (each poll itself blocks for a hardware-defined short time).
__device__ __forceinline__ bool mbar_wait(uint64_t *m, uint32_t parity, uint32_t max_tries) {
    for (uint32_t i = 0; i < max_tries; ++i)
        if (mbar_try_wait(m, parity)) return true;
    return false;
}

// ------------------------------------------------------------------ tensor memory
__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

// 32 consecutive columns of this thread's lane (32x32b shape): lane = warp quarter base + laneid
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
// 16 consecutive columns of this thread's lane
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
        "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15]))
        : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// Registers written by tcgen05.ld are valid only after tcgen05.wait::ld, but the wait
// carries no register dependence, so the compiler may schedule arithmetic on them before
// it.  Passing each register through an empty volatile asm placed after the wait (volatile
// asm statements keep their order) makes every use depend on the wait.
template <int N>
__device__ __forceinline__ void tmem_regs_after_wait(float (&v)[N]) {
#pragma unroll
    for (int i = 0; i < N; ++i) asm volatile("" : "+f"(v[i])::"memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
        "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
        "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
        "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
        "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
        "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
        "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
        : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// TMEM address of (lane, column)
__device__ __forceinline__ uint32_t taddr(uint32_t base, int lane, int col) {
    return base + ((uint32_t)lane << 16) + (uint32_t)col;
}

// ------------------------------------------------------------------ tf32 rounding
// Round a finite fp32 value to TF32 (10 explicit mantissa bits), nearest with ties away
// from zero: add half a unit of the kept last place to the magnitude bits, then drop the 13
// low bits.  Two integer ops on the ALU pipe (a carry into the exponent is the correct
// rounding up to the next binade).
__device__ __forceinline__ float to_tf32(float x) {
    return __uint_as_float((__float_as_uint(x) + 0x1000u) & 0xFFFFE000u);
}

// ------------------------------------------------------------------ TMA (no multicast)
__device__ __forceinline__ void mbar_expect_tx(uint64_t *m, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(m)),
                 "r"(bytes)
                 : "memory");
}
// 2D tile load global -> shared (this CTA), completion counted on mbarrier `m`
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void *tmap, int x, int y,
                                            uint64_t *m) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(tmap), "r"(x), "r"(y), "r"(smem_u32(m))
        : "memory");
}

// contiguous bulk copy global -> shared (this CTA), completion counted on mbarrier `m`;
// both addresses 16-byte aligned, `bytes` a multiple of 16
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint64_t *m) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(smem_u32(m))
        : "memory");
}
// 2D tile store shared (this CTA) -> global, tracked as a bulk async-group of this thread
__device__ __forceinline__ void tma_store_2d(const void *tmap, int x, int y, uint32_t src) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(tmap),
                 "r"(x), "r"(y), "r"(src)
                 : "memory");
}
// contiguous bulk copy shared (this CTA) -> global, tracked as a bulk async-group; both
// addresses 16-byte aligned, `bytes` a multiple of 16
__device__ __forceinline__ void bulk_store_s2g(void *dst, uint32_t src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// wait until this thread's bulk groups have finished reading shared memory
__device__ __forceinline__ void bulk_wait_read0() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// wait until at most one of this thread's bulk groups is still reading shared memory
__device__ __forceinline__ void bulk_wait_read1() {
    asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
// wait until this thread's bulk groups are complete
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// ------------------------------------------------------------------ cp.async (16 B)
__device__ __forceinline__ void cp_async16(uint32_t dst_smem, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst_smem), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

}  // namespace tc
}  // namespace gdn
