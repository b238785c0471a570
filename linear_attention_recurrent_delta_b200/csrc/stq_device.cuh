// stq_device.cuh -- device building blocks of the quantized Delta-rule
// decode step for sm_100a: page format, plane unpack/pack, dequant/requant,
// the pcg4d stochastic-rounding hash, bulk-copy staging with bounded mbarrier waits.
//
// In every page kernel lane l of a warp owns value columns 4l .. 4l+3.  The
// packed layout is built so that a lane reads and writes its columns as
// whole 16-byte chunks (or aligned parts of one) and one mask + shift yields
// the four columns of a row.  The quantize and dequantize kernels give warp w
// the 16-row blocks 2w and 2w+1; the decode kernel gives warp w slice w
// (rows 4w .. 4w+3) of every block.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>

namespace stq {

constexpr int kD = 128;
constexpr int kThreads = 128;
constexpr int kWarps = 4;
constexpr int kRowsPerWarp = 32;
constexpr int kBlocks = 8;          // 16-row blocks per page

enum : int { kKindInt = 0, kKindFp16 = 1 };

// Status word bits (state header).
enum : uint32_t { kStatusTimeout = 1u, kStatusBadSlot = 2u };

// Per-format constants, passed by value to every kernel.
struct DevFormat {
    int page_bytes;
    int r_off;                 // byte offset of the r region
    int c_off;                 // byte offset of the c region (col_scales)
    int col_scales, stochastic, gate_vector;
    int n_int_rows;
    // Per 16-row block, packed so that a run-time block index is a shift
    // (an indexed array in the by-value parameter would go to local memory):
    uint64_t bits8;      // byte i: bits of block i (16 = FP16)
    uint64_t rbase8;     // byte i: r index of block i's first row (INT blocks)
    uint64_t off_lo, off_hi;   // 16-bit field i: byte offset of block i (0-3, 4-7)

    __host__ __device__ int blk_bits(int i) const { return (int)((bits8 >> (8 * i)) & 0xFF); }
    __host__ __device__ int blk_kind(int i) const { return blk_bits(i) == 16 ? 1 : 0; }
    __host__ __device__ int blk_rbase(int i) const { return (int)((rbase8 >> (8 * i)) & 0xFF); }
    __host__ __device__ int blk_off(int i) const {
        return (int)((((i < 4) ? off_lo : off_hi) >> (16 * (i & 3))) & 0xFFFF);
    }
};

// ---------------------------------------------------------------- planes --
// A plane of width W (bits) over 16 rows: quad l owns 2W words; words come in
// 16-byte chunks (8 bytes when W == 1), chunk t of quad l at (32t + l) * chunk.
template <int W>
__device__ __forceinline__ void load_plane(const uint8_t *plane, int lane, uint32_t (&w)[2 * W]) {
    if constexpr (W == 1) {
        uint2 c = *reinterpret_cast<const uint2 *>(plane + lane * 8);
        w[0] = c.x; w[1] = c.y;
    } else {
#pragma unroll
        for (int t = 0; t < W / 2; ++t) {
            uint4 c = *reinterpret_cast<const uint4 *>(plane + (t * 32 + lane) * 16);
            w[4 * t + 0] = c.x; w[4 * t + 1] = c.y; w[4 * t + 2] = c.z; w[4 * t + 3] = c.w;
        }
    }
}

template <int W>
__device__ __forceinline__ void store_plane(uint8_t *plane, int lane, const uint32_t (&w)[2 * W]) {
    if constexpr (W == 1) {
        *reinterpret_cast<uint2 *>(plane + lane * 8) = make_uint2(w[0], w[1]);
    } else {
#pragma unroll
        for (int t = 0; t < W / 2; ++t)
            *reinterpret_cast<uint4 *>(plane + (t * 32 + lane) * 16) =
                make_uint4(w[4 * t + 0], w[4 * t + 1], w[4 * t + 2], w[4 * t + 3]);
    }
}

template <int W>
__host__ __device__ constexpr uint32_t plane_mask() { return 0x01010101u * ((1u << W) - 1u); }

// x moved from bit `from` to bit `to` of every byte (a shift of the word).
template <int FROM, int TO>
__device__ __forceinline__ uint32_t move_bits(uint32_t x) {
    if constexpr (TO >= FROM) return x << (TO - FROM);
    else return x >> (FROM - TO);
}

// Biased b-bit codes of a 16-row INT block, as byte vectors: ub[rho] holds the
// codes of row rho for columns 4l .. 4l+3 in bytes 0..3.  Planes are the
// binary decomposition of B, widest plane first, holding the low bits.
template <int B>
__device__ __forceinline__ void unpack_int_block(const uint8_t *blk, int lane, uint32_t (&ub)[16]) {
    if constexpr (B == 8) {
        uint32_t w[16];
        load_plane<8>(blk, lane, w);
#pragma unroll
        for (int r = 0; r < 16; ++r) ub[r] = w[r];
    } else {
        constexpr bool p4 = (B & 4) != 0, p2 = (B & 2) != 0, p1 = (B & 1) != 0;
        constexpr int lo2 = p4 ? 4 : 0;
        constexpr int lo1 = lo2 + (p2 ? 2 : 0);
        constexpr int off2 = p4 ? 1024 : 0;
        constexpr int off1 = off2 + (p2 ? 512 : 0);
        uint32_t w4[8], w2[4], w1[2];
        if constexpr (p4) load_plane<4>(blk, lane, w4);
        if constexpr (p2) load_plane<2>(blk + off2, lane, w2);
        if constexpr (p1) load_plane<1>(blk + off1, lane, w1);
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            uint32_t x = 0;
            if constexpr (p4) {
                // rows 2n (low nibbles) and 2n+1 (high nibbles) of word n
                x = (r & 1) ? (w4[r >> 1] >> 4) & plane_mask<4>() : w4[r >> 1] & plane_mask<4>();
            }
            if constexpr (p2) {
                const uint32_t src = w2[r >> 2];
                uint32_t f;
                switch (r & 3) {
                    case 0: f = move_bits<0, lo2>(src); break;
                    case 1: f = move_bits<2, lo2>(src); break;
                    case 2: f = move_bits<4, lo2>(src); break;
                    default: f = move_bits<6, lo2>(src); break;
                }
                x |= f & (plane_mask<2>() << lo2);
            }
            if constexpr (p1) {
                const uint32_t src = w1[r >> 3];
                uint32_t f;
                switch (r & 7) {
                    case 0: f = move_bits<0, lo1>(src); break;
                    case 1: f = move_bits<1, lo1>(src); break;
                    case 2: f = move_bits<2, lo1>(src); break;
                    case 3: f = move_bits<3, lo1>(src); break;
                    case 4: f = move_bits<4, lo1>(src); break;
                    case 5: f = move_bits<5, lo1>(src); break;
                    case 6: f = move_bits<6, lo1>(src); break;
                    default: f = move_bits<7, lo1>(src); break;
                }
                x |= f & (plane_mask<1>() << lo1);
            }
            ub[r] = x;
        }
    }
}

// Inverse of unpack_int_block; ub bytes hold values < 2^B.
template <int B>
__device__ __forceinline__ void pack_int_block(uint8_t *blk, int lane, const uint32_t (&ub)[16]) {
    if constexpr (B == 8) {
        uint32_t w[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) w[r] = ub[r];
        store_plane<8>(blk, lane, w);
    } else {
        constexpr bool p4 = (B & 4) != 0, p2 = (B & 2) != 0, p1 = (B & 1) != 0;
        constexpr int lo2 = p4 ? 4 : 0;
        constexpr int lo1 = lo2 + (p2 ? 2 : 0);
        constexpr int off2 = p4 ? 1024 : 0;
        constexpr int off1 = off2 + (p2 ? 512 : 0);
        if constexpr (p4) {
            uint32_t w[8];
#pragma unroll
            for (int n = 0; n < 8; ++n) {
                if constexpr (B == 4)   // codes < 16: the nibbles need no mask
                    w[n] = ub[2 * n] | (ub[2 * n + 1] << 4);
                else
                    w[n] = (ub[2 * n] & plane_mask<4>()) | ((ub[2 * n + 1] << 4) & ~plane_mask<4>());
            }
            store_plane<4>(blk, lane, w);
        }
        if constexpr (p2) {
            uint32_t w[4];
#pragma unroll
            for (int n = 0; n < 4; ++n) {
                uint32_t x;
                if constexpr (B == 2) {   // codes < 4: fields never spill
                    x = ub[4 * n] | (ub[4 * n + 1] << 2) | (ub[4 * n + 2] << 4) | (ub[4 * n + 3] << 6);
                } else {
                    x = move_bits<lo2, 0>(ub[4 * n]) & plane_mask<2>();
                    x |= move_bits<lo2, 2>(ub[4 * n + 1]) & (plane_mask<2>() << 2);
                    x |= move_bits<lo2, 4>(ub[4 * n + 2]) & (plane_mask<2>() << 4);
                    x |= move_bits<lo2, 6>(ub[4 * n + 3]) & (plane_mask<2>() << 6);
                }
                w[n] = x;
            }
            store_plane<2>(blk + off2, lane, w);
        }
        if constexpr (p1) {
            uint32_t w[2];
#pragma unroll
            for (int n = 0; n < 2; ++n) {
                uint32_t x = move_bits<lo1, 0>(ub[8 * n]) & plane_mask<1>();
                x |= move_bits<lo1, 1>(ub[8 * n + 1]) & (plane_mask<1>() << 1);
                x |= move_bits<lo1, 2>(ub[8 * n + 2]) & (plane_mask<1>() << 2);
                x |= move_bits<lo1, 3>(ub[8 * n + 3]) & (plane_mask<1>() << 3);
                x |= move_bits<lo1, 4>(ub[8 * n + 4]) & (plane_mask<1>() << 4);
                x |= move_bits<lo1, 5>(ub[8 * n + 5]) & (plane_mask<1>() << 5);
                x |= move_bits<lo1, 6>(ub[8 * n + 6]) & (plane_mask<1>() << 6);
                x |= move_bits<lo1, 7>(ub[8 * n + 7]) & (plane_mask<1>() << 7);
                w[n] = x;
            }
            store_plane<1>(blk + off1, lane, w);
        }
    }
}

// FP16 block: 128 bytes per quad = 8 chunks; word 2*rho + h holds row rho,
// columns 4l + 2h (low half) and 4l + 2h + 1 (high half).
__device__ __forceinline__ void unpack_fp16_block(const uint8_t *blk, int lane, uint32_t (&w)[32]) {
#pragma unroll
    for (int t = 0; t < 8; ++t) {
        uint4 c = *reinterpret_cast<const uint4 *>(blk + (t * 32 + lane) * 16);
        w[4 * t + 0] = c.x; w[4 * t + 1] = c.y; w[4 * t + 2] = c.z; w[4 * t + 3] = c.w;
    }
}

__device__ __forceinline__ void pack_fp16_block(uint8_t *blk, int lane, const uint32_t (&w)[32]) {
#pragma unroll
    for (int t = 0; t < 8; ++t)
        *reinterpret_cast<uint4 *>(blk + (t * 32 + lane) * 16) =
            make_uint4(w[4 * t + 0], w[4 * t + 1], w[4 * t + 2], w[4 * t + 3]);
}

// --------------------------------------------------------------- numerics --
// Exact integer -> float: bits 0x4B000000 | u is the float 2^23 + u (u < 2^23).
__device__ __forceinline__ float magic_byte(uint32_t ub, int beta) {
    return __int_as_float(__byte_perm(ub, 0x4B000000u, 0x7650u | beta));
}

// The four columns of a row as exact floats z = u - bias, in pairs.
__device__ __forceinline__ void codes_to_float(uint32_t ub, float bias_magic, float2 &z01, float2 &z23) {
    const float2 m = make_float2(-bias_magic, -bias_magic);
    z01 = __fadd2_rn(make_float2(magic_byte(ub, 0), magic_byte(ub, 1)), m);
    z23 = __fadd2_rn(make_float2(magic_byte(ub, 2), magic_byte(ub, 3)), m);
}

// Low bytes of four floats gathered into one word.
__device__ __forceinline__ uint32_t low_bytes(float y0, float y1, float y2, float y3) {
    uint32_t lo = __byte_perm(__float_as_uint(y0), __float_as_uint(y1), 0x0040u);
    uint32_t hi = __byte_perm(__float_as_uint(y2), __float_as_uint(y3), 0x0040u);
    return __byte_perm(lo, hi, 0x5410u);
}

// ------------------------------------------------- stochastic-rounding hash --
// pcg4d (Jarzynski and Olano, "Hash Functions for GPU Rendering", JCGT 9(3),
// 2020): a linear congruential step on each word, each word plus the product
// of two others, a 16-bit xorshift of every word, the products once more.
// Input: the counter (x, step, request, head), the last two words xor the
// 64-bit seed (k0, k1).  Within a page only x changes, so the terms the
// other three words fix -- their congruential step and the product y w of
// the first mixing round -- are formed once per page (sr_fix) and each hash
// starts from x alone (sr_hash4_fixed): the same operations modulo 2^32,
// the constant terms added first.
struct SrFixed {
    uint32_t y1, z1, w1, cx;
};

__device__ __forceinline__ SrFixed sr_fix(uint32_t y, uint32_t z, uint32_t w, uint32_t k0, uint32_t k1) {
    SrFixed f;
    f.y1 = y * 1664525u + 1013904223u;
    f.z1 = (z ^ k0) * 1664525u + 1013904223u;
    f.w1 = (w ^ k1) * 1664525u + 1013904223u;
    f.cx = 1013904223u + f.y1 * f.w1;
    return f;
}

__device__ __forceinline__ uint4 sr_hash4_fixed(uint32_t x0, const SrFixed &f) {
    uint32_t x = x0 * 1664525u + f.cx;
    uint32_t y = f.y1 + f.z1 * x;
    uint32_t z = f.z1 + x * y;
    uint32_t w = f.w1 + y * z;
    x ^= x >> 16;
    y ^= y >> 16;
    z ^= z >> 16;
    w ^= w >> 16;
    x += y * w;
    y += z * x;
    z += x * y;
    w += y * z;
    return make_uint4(x, y, z, w);
}

// Stochastic-rounding offsets of the two columns held by one 32-bit word, as
// the floats 128 + u, u = h16 / 65536 in [0, 1) for the high and the low
// 16-bit half: a byte permute puts h16 under the exponent of 128.0f (the
// float 128 (1 + h16 2^-23) = 128 + h16 2^-16, exact).
__device__ __forceinline__ float2 sr_offset_pair(uint32_t word) {
    const float hi = __int_as_float(__byte_perm(word, 0x43000000u, 0x7632u));   // 128 + high half / 2^16
    const float lo = __int_as_float(__byte_perm(word, 0x43000000u, 0x7610u));   // 128 + low half / 2^16
    return make_float2(hi, lo);
}

// ------------------------------------------------------- bulk-copy staging --
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                 :: "r"(smem_u32(bar)), "r"(bytes) : "memory");
}

// Global -> shared bulk copy (no multicast); bytes and both addresses are
// multiples of 16.  Completion is counted on `bar`.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile("cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 :: "r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}

// Shared -> global bulk copy, tracked as a bulk async-group of the issuing
// thread; bytes and both addresses are multiples of 16.
__device__ __forceinline__ void bulk_s2g(void *dst, const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                 :: "l"(dst), "r"(smem_u32(src)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void bulk_commit() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Wait until at most N of this thread's bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" :: "n"(N) : "memory");
}

// Wait until at most N of this thread's bulk groups are incomplete.
template <int N>
__device__ __forceinline__ void bulk_wait() {
    asm volatile("cp.async.bulk.wait_group %0;" :: "n"(N) : "memory");
}

// ------------------------------------------------------- small reductions --
// max(|x|) over the 32 lanes of a full warp, in every lane (sm_100a).
__device__ __forceinline__ float warp_absmax(float x) {
    float r;
    asm volatile("redux.sync.max.abs.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(x));
    return r;
}

// max of three floats (one instruction on sm_100a); the result for NaN
// inputs is left unspecified.
__device__ __forceinline__ float max3f(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Bounded wait on a phase of an mbarrier.  Returns false if the phase did not
// complete within limit_ns.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (;;) {
#pragma unroll 1
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (global_ns() - t0 > limit_ns) return false;
    }
}

}  // namespace stq
