// stq_slices.cuh -- per-slice device pieces of the packed-state kernels (sm_100a):
// the compile-time formats, plane unpack / pack of one slice (rows 4w .. 4w+3 of a
// 16-row block, lane l holding columns 4l .. 4l+3), dequantization, requantization
// (round to nearest or pcg4d stochastic rounding), the readout chains and the
// divisions of the row-scale step.  Included by the decode and window kernels.
#pragma once

#include <type_traits>

#include "stq_internal.h"

namespace stq {

// ---- formats: widths per 16-row block (16 = FP16) known at compile time,
// or read from DevFormat at run time (any other valid format)
// Per-format code-placement choices (measured per format on a B200; each
// changes only where independent work sits, never the arithmetic):
//   kOLate   all readout chains beside S6's division (gives its latency work)
//   kOSplit  the second readout chain (blocks 4-7) beside S6
//   kFastRcp S6's division starts from the approximate hardware reciprocal
//   kEarlyRefill a stage is refilled during the page after its own, after
//            the update (its bulk store has read it by then); otherwise at
//            the barrier of the page after that (one page less of look-ahead)
enum Tune : int { kTuneNone = 0, kOLate = 1, kOSplit = 2, kFastRcp = 4, kEarlyRefill = 8 };

template <int W0, int W1, int W2, int W3, int W4, int W5, int W6, int W7, bool COLS, bool GVEC, bool SR, int TUNE>
struct StaticFmt {
    static constexpr bool kRuntime = false;
    static constexpr bool kCols = COLS, kGvec = GVEC, kSr = SR;
    static constexpr int kTune = TUNE;
    __host__ __device__ static constexpr int width(int b) {
        return b == 0 ? W0 : b == 1 ? W1 : b == 2 ? W2 : b == 3 ? W3 : b == 4 ? W4 : b == 5 ? W5 : b == 6 ? W6 : W7;
    }
    // offset of block b's codes and index of its first r (INT rows, stored order)
    __host__ __device__ static constexpr int offset(int b) {
        int off = 0;
        for (int i = 0; i < b; ++i) off += 256 * width(i);
        return off;
    }
    __host__ __device__ static constexpr int rbase(int b) {
        int r = 0;
        for (int i = 0; i < b; ++i) r += width(i) == 16 ? 0 : 16;
        return r;
    }
};

template <bool SR>
struct RuntimeFmt {
    static constexpr bool kRuntime = true;
    static constexpr bool kSr = SR;
    static constexpr int kTune = kTuneNone;
};

// (the stepquant6 instantiation sits at the register limit: each move made
// it spill and run 3-6 % slower; kda likewise with kFastRcp or kEarlyRefill)
using FmtStepQuant6 = StaticFmt<8, 8, 6, 6, 6, 6, 4, 4, true, false, false, kTuneNone>;
using FmtInt8Row = StaticFmt<8, 8, 8, 8, 8, 8, 8, 8, false, false, false, kOLate | kFastRcp | kEarlyRefill>;
using FmtStepQuant4Kda = StaticFmt<8, 4, 4, 4, 3, 3, 3, 3, true, true, false, kOSplit>;
using FmtDamp = StaticFmt<16, 8, 8, 8, 8, 8, 8, 8, false, false, true, kFastRcp | kEarlyRefill>;

// m / qmax rounded to nearest, for qmax = 2^(b-1) - 1: one correction step on
// m * RN(1/qmax) (Markstein's division by a constant); equal to IEEE division
// for every positive finite float m and every qmax of 2..8-bit codes (checked
// exhaustively on the GPU against __fdiv_rn).
__device__ __forceinline__ float div_by_qmax(float m, float qmax, float rcp_qmax) {
    const float q0 = __fmul_rn(m, rcp_qmax);
    return __fmaf_rn(__fmaf_rn(-q0, qmax, m), rcp_qmax, q0);
}

// qmax / m rounded toward zero, for finite m > 0 and qmax = 2^(b-1) - 1:
// a Markstein step on qmax * y, y a reciprocal of m, gives q1 within half an
// ulp of the quotient, and the exact residual qmax - q1 m says whether q1
// lies above it (then the next float below is the result).  y is RN(1/m),
// or with FAST the hardware approximation (within an ulp: the step still
// lands within half an ulp).  Outside [2^-100, 2^126] (1/m near overflow, or
// an approximate 1/m flushed to zero) the library division is used.  Equal
// to __fdiv_rz for every m >= 2^-100 and every qmax of 2..8-bit codes, both
// ways (checked exhaustively on the GPU).
template <bool FAST>
__device__ __forceinline__ float div_rz_qmax(float qmax, float m) {
    if (m < 0x1p-100f || (FAST && m > 0x1p126f)) return __fdiv_rz(qmax, m);
    float y;
    if constexpr (FAST) asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(m));
    else y = __frcp_rn(m);
    const float q0 = __fmul_rn(qmax, y);
    const float q1 = __fmaf_rn(__fmaf_rn(-q0, m, qmax), y, q0);
    const float r1 = __fmaf_rn(-q1, m, qmax);
    return r1 < 0.f ? __int_as_float(__float_as_int(q1) - 1) : q1;
}

// ---- S1 / S8 on one slice: rows 4w .. 4w+3 of a 16-row block.
// Plane words of a slice (quad l): width 8: the whole chunk w; width 4: the
// half chunk holding rows (0,1), (2,3); width 2: one word, row i at bits 2i
// of each byte; width 1: half the bits of one word (bits 4(w&1) + i), shared
// with the partner slice w ^ 1.
template <int B>
__device__ __forceinline__ void unpack_int_slice(const uint8_t *blk, int w, int lane, uint32_t (&ub)[4]) {
    if constexpr (B == 8) {
        const uint4 c = *reinterpret_cast<const uint4 *>(blk + (32 * w + lane) * 16);
        ub[0] = c.x; ub[1] = c.y; ub[2] = c.z; ub[3] = c.w;
    } else {
        constexpr bool p4 = (B & 4) != 0, p2 = (B & 2) != 0, p1 = (B & 1) != 0;
        constexpr int lo2 = p4 ? 4 : 0;
        constexpr int lo1 = lo2 + (p2 ? 2 : 0);
        constexpr int off2 = p4 ? 1024 : 0;
        constexpr int off1 = off2 + (p2 ? 512 : 0);
#pragma unroll
        for (int i = 0; i < 4; ++i) ub[i] = 0;
        if constexpr (p4) {
            const uint2 c = *reinterpret_cast<const uint2 *>(blk + (32 * (w >> 1) + lane) * 16 + 8 * (w & 1));
            ub[0] = c.x & plane_mask<4>();
            ub[1] = (c.x >> 4) & plane_mask<4>();
            ub[2] = c.y & plane_mask<4>();
            ub[3] = (c.y >> 4) & plane_mask<4>();
        }
        if constexpr (p2) {
            const uint32_t c = *reinterpret_cast<const uint32_t *>(blk + off2 + lane * 16 + 4 * w);
            ub[0] |= move_bits<0, lo2>(c) & (plane_mask<2>() << lo2);
            ub[1] |= move_bits<2, lo2>(c) & (plane_mask<2>() << lo2);
            ub[2] |= move_bits<4, lo2>(c) & (plane_mask<2>() << lo2);
            ub[3] |= move_bits<6, lo2>(c) & (plane_mask<2>() << lo2);
        }
        if constexpr (p1) {
            const uint32_t c = *reinterpret_cast<const uint32_t *>(blk + off1 + lane * 8 + 4 * (w >> 1)) >>
                               (4 * (w & 1));
            ub[0] |= move_bits<0, lo1>(c) & (plane_mask<1>() << lo1);
            ub[1] |= move_bits<1, lo1>(c) & (plane_mask<1>() << lo1);
            ub[2] |= move_bits<2, lo1>(c) & (plane_mask<1>() << lo1);
            ub[3] |= move_bits<3, lo1>(c) & (plane_mask<1>() << lo1);
        }
    }
}

// Inverse of unpack_int_slice (ub bytes < 2^B), in place in the stage.  The
// 1-bit plane's word is shared with the partner slice: only this slice's
// bits are flipped, by an atomic xor, so the two slices may write in any order.
template <int B>
__device__ __forceinline__ void pack_int_slice(uint8_t *blk, int w, int lane, const uint32_t (&ub)[4]) {
    if constexpr (B == 8) {
        *reinterpret_cast<uint4 *>(blk + (32 * w + lane) * 16) = make_uint4(ub[0], ub[1], ub[2], ub[3]);
    } else {
        constexpr bool p4 = (B & 4) != 0, p2 = (B & 2) != 0, p1 = (B & 1) != 0;
        constexpr int lo2 = p4 ? 4 : 0;
        constexpr int lo1 = lo2 + (p2 ? 2 : 0);
        constexpr int off2 = p4 ? 1024 : 0;
        constexpr int off1 = off2 + (p2 ? 512 : 0);
        if constexpr (p4) {
            uint32_t x0, x1;
            if constexpr (B == 4) {   // codes < 16: the nibbles need no mask
                x0 = ub[0] | (ub[1] << 4);
                x1 = ub[2] | (ub[3] << 4);
            } else {
                x0 = (ub[0] & plane_mask<4>()) | ((ub[1] << 4) & ~plane_mask<4>());
                x1 = (ub[2] & plane_mask<4>()) | ((ub[3] << 4) & ~plane_mask<4>());
            }
            *reinterpret_cast<uint2 *>(blk + (32 * (w >> 1) + lane) * 16 + 8 * (w & 1)) = make_uint2(x0, x1);
        }
        if constexpr (p2) {
            uint32_t x;
            if constexpr (B == 2) {   // codes < 4: fields never spill
                x = ub[0] | (ub[1] << 2) | (ub[2] << 4) | (ub[3] << 6);
            } else {
                x = move_bits<lo2, 0>(ub[0]) & plane_mask<2>();
                x |= move_bits<lo2, 2>(ub[1]) & (plane_mask<2>() << 2);
                x |= move_bits<lo2, 4>(ub[2]) & (plane_mask<2>() << 4);
                x |= move_bits<lo2, 6>(ub[3]) & (plane_mask<2>() << 6);
            }
            *reinterpret_cast<uint32_t *>(blk + off2 + lane * 16 + 4 * w) = x;
        }
        if constexpr (p1) {
            uint32_t x = move_bits<lo1, 0>(ub[0]) & plane_mask<1>();
            x |= move_bits<lo1, 1>(ub[1]) & (plane_mask<1>() << 1);
            x |= move_bits<lo1, 2>(ub[2]) & (plane_mask<1>() << 2);
            x |= move_bits<lo1, 3>(ub[3]) & (plane_mask<1>() << 3);
            uint32_t *word = reinterpret_cast<uint32_t *>(blk + off1 + lane * 8 + 4 * (w >> 1));
            const int sh = 4 * (w & 1);
            const uint32_t mine = (*word >> sh) & 0x0F0F0F0Fu;   // this slice's bits: no one else writes them
            atomicXor(word, (mine ^ x) << sh);
        }
    }
}

// FP16 slice: words 8w .. 8w+7 of the quad (chunks 2w, 2w+1); word 2i + h
// holds row 4w + i, columns 4l + 2h (low half) and 4l + 2h + 1.
__device__ __forceinline__ void load_fp16_slice(const uint8_t *blk, int w, int lane, uint32_t (&x)[8]) {
    const uint4 c0 = *reinterpret_cast<const uint4 *>(blk + (32 * (2 * w) + lane) * 16);
    const uint4 c1 = *reinterpret_cast<const uint4 *>(blk + (32 * (2 * w + 1) + lane) * 16);
    x[0] = c0.x; x[1] = c0.y; x[2] = c0.z; x[3] = c0.w;
    x[4] = c1.x; x[5] = c1.y; x[6] = c1.z; x[7] = c1.w;
}

__device__ __forceinline__ void store_fp16_slice(uint8_t *blk, int w, int lane, const uint32_t (&x)[8]) {
    *reinterpret_cast<uint4 *>(blk + (32 * (2 * w) + lane) * 16) = make_uint4(x[0], x[1], x[2], x[3]);
    *reinterpret_cast<uint4 *>(blk + (32 * (2 * w + 1) + lane) * 16) = make_uint4(x[4], x[5], x[6], x[7]);
}

// ---- per-block dispatch: fn(std::integral_constant<int, width>) for block B
template <int V>
using IC = std::integral_constant<int, V>;

template <class FMT, int B, class Fn>
__device__ __forceinline__ void with_width(const DevFormat &F, Fn &&fn) {
    if constexpr (!FMT::kRuntime) {
        fn(IC<FMT::width(B)>{});
    } else {
        switch (F.blk_bits(B)) {
            case 16: fn(IC<16>{}); break;
            case 8: fn(IC<8>{}); break;
            case 7: fn(IC<7>{}); break;
            case 6: fn(IC<6>{}); break;
            case 5: fn(IC<5>{}); break;
            case 4: fn(IC<4>{}); break;
            case 3: fn(IC<3>{}); break;
            default: fn(IC<2>{}); break;
        }
    }
}

template <int I, int N, class Fn>
__device__ __forceinline__ void static_for(Fn &&fn) {
    if constexpr (I < N) {
        fn(IC<I>{});
        static_for<I + 1, N>(fn);
    }
}

template <class FMT, int B>
__device__ __forceinline__ int fmt_offset(const DevFormat &F) {
    if constexpr (FMT::kRuntime) {
        return F.blk_off(B);
    } else {
        constexpr int off = FMT::offset(B);
        return off;
    }
}

using Tile = float2[kBlocks][4][2];   // a thread's T: [block][row of the slice][column pair]

// ---- S1 + S2 on slice w of block B (a4: the four rows' alpha * r)
template <int W, int B>
__device__ __forceinline__ void dequant_slice(const uint8_t *blk, int w, int lane, const float4 a4, Tile &T) {
    const float av[4] = {a4.x, a4.y, a4.z, a4.w};
    if constexpr (W == 16) {
        uint32_t x[8];
        load_fp16_slice(blk, w, lane, x);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 as = make_float2(av[i], av[i]);
            T[B][i][0] = __fmul2_rn(__half22float2(*reinterpret_cast<const __half2 *>(&x[2 * i])), as);
            T[B][i][1] = __fmul2_rn(__half22float2(*reinterpret_cast<const __half2 *>(&x[2 * i + 1])), as);
        }
    } else {
        uint32_t ub[4];
        unpack_int_slice<W>(blk, w, lane, ub);
        const float bm = 8388608.0f + (float)(1 << (W - 1));
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float2 z01, z23;
            codes_to_float(ub[i], bm, z01, z23);
            T[B][i][0] = __fmul2_rn(z01, make_float2(av[i], av[i]));
            T[B][i][1] = __fmul2_rn(z23, make_float2(av[i], av[i]));
        }
    }
}

// ---- S7 + S8 on slice w of block B, in place in the stage
struct SrCtx {
    uint32_t k0, k1, step, b, h;
    SrFixed f;   // the hash's terms fixed by (step, b, h) and the seed: set by fix()
    __device__ __forceinline__ void fix() { f = sr_fix(step, b, h, k0, k1); }
};

template <int W, int B, bool SR>
__device__ __forceinline__ void requant_slice(uint8_t *blk, int w, int lane, const float4 inv4, const Tile &T,
                                              const SrCtx sr) {
    if constexpr (W == 16) {
        uint32_t x[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __half2 h01 = __floats2half2_rn(T[B][i][0].x, T[B][i][0].y);
            __half2 h23 = __floats2half2_rn(T[B][i][1].x, T[B][i][1].y);
            x[2 * i] = *reinterpret_cast<uint32_t *>(&h01);
            x[2 * i + 1] = *reinterpret_cast<uint32_t *>(&h23);
        }
        store_fp16_slice(blk, w, lane, x);
    } else {
        const float M = 12582912.0f + (float)(1 << (W - 1));   // 1.5 * 2^23 + bias
        const float2 M2 = make_float2(M, M);
        // stochastic rounding: floor(x + u) of the exact x = T inv.  The fma
        // rounds x + 128 + u down (in [1, 256): |x| <= qmax < 128), which keeps
        // its floor, and the add of M - 128 rounds down to the integer grid
        // of [2^23, 2^24): floor(x + u) + M in one rounding each.
        const float2 Mf2 = make_float2(M - 128.0f, M - 128.0f);
        const float iv[4] = {inv4.x, inv4.y, inv4.z, inv4.w};
        uint32_t ub[4];
#pragma unroll
        for (int i = 0; i < 4; i += 2) {
            const float2 i0 = make_float2(iv[i], iv[i]), i1 = make_float2(iv[i + 1], iv[i + 1]);
            float2 y0, y1, y2, y3;
            if constexpr (SR) {
                const uint32_t s = 16u * B + 4u * (uint32_t)w + (uint32_t)i;   // stored row, even
                const uint4 h = sr_hash4_fixed((s >> 1) * 32u + (uint32_t)lane, sr.f);
                y0 = __fadd2_rd(__ffma2_rd(T[B][i][0], i0, sr_offset_pair(h.x)), Mf2);
                y1 = __fadd2_rd(__ffma2_rd(T[B][i][1], i0, sr_offset_pair(h.y)), Mf2);
                y2 = __fadd2_rd(__ffma2_rd(T[B][i + 1][0], i1, sr_offset_pair(h.z)), Mf2);
                y3 = __fadd2_rd(__ffma2_rd(T[B][i + 1][1], i1, sr_offset_pair(h.w)), Mf2);
            } else {
                y0 = __ffma2_rn(T[B][i][0], i0, M2);
                y1 = __ffma2_rn(T[B][i][1], i0, M2);
                y2 = __ffma2_rn(T[B][i + 1][0], i1, M2);
                y3 = __ffma2_rn(T[B][i + 1][1], i1, M2);
            }
            ub[i] = low_bytes(y0.x, y0.y, y1.x, y1.y);
            ub[i + 1] = low_bytes(y2.x, y2.y, y3.x, y3.y);
        }
        pack_int_slice<W>(blk, w, lane, ub);
    }
}

// S5's chains over block B of the slice (q of the slice's rows in qp)
template <int B>
__device__ __forceinline__ void readout_block(const float *qp, const Tile &T, float2 (&co)[2]) {
    const float4 q4 = *reinterpret_cast<const float4 *>(&qp[4 * B]);
    const float qv[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        co[0] = __ffma2_rn(make_float2(qv[i], qv[i]), T[B][i][0], co[0]);
        co[1] = __ffma2_rn(make_float2(qv[i], qv[i]), T[B][i][1], co[1]);
    }
}

// the warp's readout partial: chain over blocks 0-3 plus chain over 4-7
__device__ __forceinline__ void store_readout(float *red, int lane, const float2 (&co)[2][2]) {
    const float2 w01 = __fadd2_rn(co[0][0], co[1][0]), w23 = __fadd2_rn(co[0][1], co[1][1]);
    *reinterpret_cast<float4 *>(&red[4 * lane]) = make_float4(w01.x, w01.y, w23.x, w23.y);
}

// max |x| over a row's four columns held by one lane
__device__ __forceinline__ float absmax4(float2 a, float2 b) {
    return fmaxf(max3f(fabsf(a.x), fabsf(a.y), fabsf(b.x)), fabsf(b.y));
}

template <class FMT>
inline bool format_is(const DevFormat &F) {
    for (int b = 0; b < kBlocks; ++b)
        if (F.blk_bits(b) != FMT::width(b)) return false;
    return (F.col_scales != 0) == FMT::kCols && (F.gate_vector != 0) == FMT::kGvec &&
           (F.stochastic != 0) == FMT::kSr;
}

}  // namespace stq
