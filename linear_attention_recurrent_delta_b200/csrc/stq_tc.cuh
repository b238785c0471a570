// stq_tc.cuh -- fifth-generation tensor-core (tcgen05) building blocks for
// sm_100a: tensor-memory allocation, shared-memory matrix descriptors for the
// 128-byte-swizzled K-major layout, the tf32 MMA, its completion on an
// mbarrier, and tensor-memory loads.
//
// Conventions used by every caller:
//   * an operand tile is 128 rows x 32 fp32 (one 128-byte swizzle atom per
//     row, 16 KB) at a 1024-byte-aligned shared address; row r, element k sits
//     at byte  r * 128 + (((k >> 2) ^ (r & 7)) << 4) + (k & 3) * 4;
//     a K extent of 32 n is n such tiles, 16 KB apart;
//   * one MMA consumes K = 8 (32 bytes) of each operand: the descriptor's start
//     address moves 32 bytes per K step inside a tile;
//   * D (M = 128 rows) lives in tensor memory with row i in lane i, column j in
//     column (base + j); warp w reads lanes 32 (w % 4) .. + 31.
#pragma once

#include <cstdint>

namespace stq {
namespace tc {

constexpr uint32_t kTileBytes = 128 * 128;   // 128 rows x 128 bytes

// byte offset of element (row r, k in 0..31) inside a swizzled tile
__host__ __device__ __forceinline__ uint32_t sw128_offset(uint32_t r, uint32_t k) {
    return r * 128u + ((((k >> 2) ^ (r & 7u)) & 7u) << 4) + (k & 3u) * 4u;
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (SBO), leading offset unused by this layout (1), version 1.
__device__ __forceinline__ uint64_t desc_k_sw128(uint32_t smem_addr) {
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);
    d |= (uint64_t)1u << 16;                   // LBO = 16 bytes (unused for this layout)
    d |= (uint64_t)(1024u >> 4) << 32;         // SBO = 1024 bytes
    d |= (uint64_t)1u << 46;                   // descriptor version
    d |= (uint64_t)2u << 61;                   // 128-byte swizzle
    return d;
}

// Instruction descriptor of kind::tf32 with fp32 accumulation, both operands
// K-major; neg_a negates A.
__host__ __device__ constexpr uint32_t idesc_tf32(int M, int N, bool neg_a = false) {
    return (1u << 4)                            // D format: f32
           | (2u << 7)                          // A format: tf32
           | (2u << 10)                         // B format: tf32
           | ((neg_a ? 1u : 0u) << 13)
           | ((uint32_t)(N >> 3) << 17)
           | ((uint32_t)(M >> 4) << 24);
}

// warp-wide: allocate ncols (a power of two >= 32) tensor-memory columns; the
// address is written to *dst (shared memory)
__device__ __forceinline__ void tmem_alloc(uint32_t *dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void fence_before_sync() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void fence_after_sync() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D (+)= A * B^T, tf32 inputs, fp32 accumulation (one thread issues)
__device__ __forceinline__ void mma_tf32(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         bool accumulate) {
    const uint32_t acc = accumulate ? 1u : 0u;
    const uint32_t z = 0;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}"
                 :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(acc), "r"(z), "r"(z), "r"(z), "r"(z)
                 : "memory");
}

// arrive once on the mbarrier when every MMA this thread issued so far is done
__device__ __forceinline__ void commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 :: "r"(static_cast<uint32_t>(__cvta_generic_to_shared(bar))) : "memory");
}

// 32 consecutive columns of this warp's 32 lanes: thread t gets row (lane base + t)
__device__ __forceinline__ void ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 "
                 "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
                 "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
                   "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
                   "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
                   "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// 16 consecutive columns of this warp's 32 lanes (waits for them)
__device__ __forceinline__ void ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                 "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
                   "=r"(r[14]), "=r"(r[15])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// store 32 consecutive columns of this warp's 32 lanes (thread t: row lane
// base + t) and wait until the stores are done
__device__ __forceinline__ void st32(uint32_t taddr, const float (&v)[32]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
                 "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
                 "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
                 :: "r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
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
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// the tf32 part of x (low 13 mantissa bits cleared, round to nearest on the
// cleared bits) and the remainder x - hi, exact in fp32
__device__ __forceinline__ void split_tf32(float x, float &hi, float &lo) {
    const uint32_t u = __float_as_uint(x);
    const uint32_t h = (u + 0x1000u) & 0xFFFFE000u;
    hi = __uint_as_float(h);
    lo = __fsub_rn(x, hi);
}

}  // namespace tc
}  // namespace stq
