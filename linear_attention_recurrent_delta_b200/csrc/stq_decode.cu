// stq_decode.cu -- the fused decode-step kernel (sm_100a).
//
// One persistent CTA of 128 threads walks pages p = blockIdx.x + i*gridDim.x.
// Each page's bytes and its q, k, v (and KDA alpha) rows are brought into a
// shared-memory ring by one thread with cp.async.bulk (no multicast), counted
// on an mbarrier; the ring is 2..4 deep so the copies of later pages overlap
// the math of the current one.  Per page, all in registers / shared memory:
//   S1 unpack planes -> S2 dequant + decay T = z (alpha r)
//   S3 column sums u = sum_s k_s T_s (one fma chain per 16-row block, then
//      ((P0+P1)+(P2+P3))+((P4+P5)+(P6+P7))),  e = v (1/c) - u
//   S4 T' = T + (beta k_s) e      S5 o = c * sum_s q_s T'_s (same order)
//   S6 row absmax -> r' = m/qmax, inv = qmax/m rounded toward zero
//   S7 requant (RNE of the exact product, or Philox stochastic rounding on
//      INT rows; binary16 on FP16 rows)   S8 repack and store in place.
// The state crosses HBM once each way per step.  No tensor cores: the work
// is rank-1 updates and mat-vecs.
//
// Warp w owns the 16-row blocks 2w and 2w+1 and dispatches on their widths at
// run time.  All warps share one copy of the loop: per-warp copies specialised
// to each warp's widths were measured slower, the larger code overflowing the
// instruction cache the SM's warps share.
//
// One CTA-wide barrier per page: each warp prepares the operands of its own
// rows (thread 32w + l: stored row 32w + l) and syncs within the warp; the
// column sums' block partials and 1/c are double-buffered by page parity, so
// the only cross-warp dependency is u (and o, finished after the next page's
// barrier).  Warps of a CTA drift apart by up to a page.
#include "stq_internal.h"

namespace stq {

struct DecodeArgs {
    uint8_t *pages;
    const uint8_t *perm;
    uint32_t *status;
    const float *q, *k, *v, *alpha, *beta;
    float *o;
    int n_pages;                  // < 2^31 (checked when the state is bound)
    int heads;
    int n_stages;                 // ring depth, 2 .. kMaxStages
    uint32_t stage_bytes;
    uint32_t seed_lo, seed_hi, step;
    uint64_t wait_limit_ns;
    int stall_first_wait;
};

constexpr int kMaxStages = 4;
constexpr int kRmxPitch = 36;     // words per row of the row-max tile

struct SmemFixed {
    // per stored row (a 16-byte load serves 4 rows; an f32x2 operation takes
    // the value duplicated without a move):
    float a[kD];                            // alpha * r (decay x row scale)
    float kp[kD];                           // k of the row's key channel
    float bk[kD];                           // beta * k
    float qp[kD];                           // q
    float red_u[2][kWarps][kD];             // per page parity and warp: P_2w + P_2w+1 of u
    float red_o[2][kWarps][kD];             // the same for o
    // row-partial maxima: row r of a warp at r * kRmxPitch, one word per lane;
    // the pitch keeps both the per-row stores and the 16-byte row reads
    // free of bank conflicts
    float rmx[kWarps][kRowsPerWarp * kRmxPitch];
    float inv[kWarps][kRowsPerWarp];        // requant multipliers
    float ic[2][kD];                        // per page parity: 1 / c per column
    float c_prev[kD];                       // c of the page whose o is pending
    uint64_t full[kMaxStages];              // stage-full barriers
    uint64_t never;                         // a barrier nothing completes (test hook)
};

constexpr size_t kFixedBytes = (sizeof(SmemFixed) + 127) / 128 * 128;

__host__ __device__ inline uint32_t decode_stage_bytes(const DevFormat &F) {
    return (uint32_t)F.page_bytes + 3u * 512u + (F.gate_vector ? 512u : 0u);
}

// m / qmax rounded to nearest, for qmax = 2^(b-1) - 1: one correction step on
// m * RN(1/qmax) (Markstein's division by a constant); equal to IEEE division
// for every positive finite float m and every qmax of 2..8-bit codes (checked
// exhaustively on the GPU against __fdiv_rn).
__device__ __forceinline__ float div_by_qmax(float m, float qmax, float rcp_qmax) {
    const float q0 = __fmul_rn(m, rcp_qmax);
    return __fmaf_rn(__fmaf_rn(-q0, qmax, m), rcp_qmax, q0);
}

// ---- S1 + S2: one 16-row block into T[r0 .. r0+15] (a: the block's alpha * r)
template <int B>
__device__ __forceinline__ void dequant_int(const uint8_t *blk, int lane, const float *a,
                                            float2 (&T)[kRowsPerWarp][2], int r0) {
    uint32_t ub[16];
    unpack_int_block<B>(blk, lane, ub);
    const float bm = 8388608.0f + (float)(1 << (B - 1));
#pragma unroll
    for (int r = 0; r < 16; r += 4) {
        const float4 aa = *reinterpret_cast<const float4 *>(a + r);   // rows r .. r+3
        const float av[4] = {aa.x, aa.y, aa.z, aa.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float2 z01, z23;
            codes_to_float(ub[r + i], bm, z01, z23);
            T[r0 + r + i][0] = __fmul2_rn(z01, make_float2(av[i], av[i]));
            T[r0 + r + i][1] = __fmul2_rn(z23, make_float2(av[i], av[i]));
        }
    }
}

__device__ __forceinline__ void dequant_fp16(const uint8_t *blk, int lane, const float *a,
                                             float2 (&T)[kRowsPerWarp][2], int r0) {
    uint32_t w[32];
    unpack_fp16_block(blk, lane, w);
#pragma unroll
    for (int r = 0; r < 16; ++r) {
        const float2 as = make_float2(a[r], a[r]);
        float2 x01 = __half22float2(*reinterpret_cast<const __half2 *>(&w[2 * r]));
        float2 x23 = __half22float2(*reinterpret_cast<const __half2 *>(&w[2 * r + 1]));
        T[r0 + r][0] = __fmul2_rn(x01, as);
        T[r0 + r][1] = __fmul2_rn(x23, as);
    }
}

// BITS: the block's width (16 = FP16), or 0 to read `bits` at run time.
template <int BITS, int R0>
__device__ __forceinline__ void dequant_block(int bits, const uint8_t *blk, int lane, const float *a,
                                              float2 (&T)[kRowsPerWarp][2]) {
    if constexpr (BITS == 16) dequant_fp16(blk, lane, a, T, R0);
    else if constexpr (BITS != 0) dequant_int<BITS>(blk, lane, a, T, R0);
    else {
        switch (bits) {
            case 16: dequant_fp16(blk, lane, a, T, R0); break;
            case 8: dequant_int<8>(blk, lane, a, T, R0); break;
            case 7: dequant_int<7>(blk, lane, a, T, R0); break;
            case 6: dequant_int<6>(blk, lane, a, T, R0); break;
            case 5: dequant_int<5>(blk, lane, a, T, R0); break;
            case 4: dequant_int<4>(blk, lane, a, T, R0); break;
            case 3: dequant_int<3>(blk, lane, a, T, R0); break;
            default: dequant_int<2>(blk, lane, a, T, R0); break;
        }
    }
}

// ---- S7 + S8: requantize one 16-row block of T' and store its planes.
struct SrCtx {
    uint32_t k0, k1, step, b, h;
};

template <int B, bool SR>
__device__ __forceinline__ void requant_int(uint8_t *blk, int lane, const float *inv,
                                            const float2 (&T)[kRowsPerWarp][2], int r0, int s0,
                                            const SrCtx sr) {
    const float M = 12582912.0f + (float)(1 << (B - 1));   // 1.5 * 2^23 + bias
    const float2 M2 = make_float2(M, M);
    uint32_t ub[16];
#pragma unroll
    for (int r = 0; r < 16; r += 2) {
        const float4 i4 = *reinterpret_cast<const float4 *>(inv + (r & ~3));   // rows r & ~3 .. +3
        const float ia = (r & 2) ? i4.z : i4.x, ib = (r & 2) ? i4.w : i4.y;
        const float2 i0 = make_float2(ia, ia), i1 = make_float2(ib, ib);
        float2 y0, y1, y2, y3;
        if constexpr (SR) {
            const int s = s0 + r;   // even
            const uint4 h = philox4x32_10(
                make_uint4((uint32_t)(s >> 1) * 32u + (uint32_t)lane, sr.step, sr.b, sr.h), sr.k0, sr.k1);
            y0 = __fadd2_rn(__ffma2_rn(T[r0 + r][0], i0, sr_delta_pair(h.x)), M2);
            y1 = __fadd2_rn(__ffma2_rn(T[r0 + r][1], i0, sr_delta_pair(h.y)), M2);
            y2 = __fadd2_rn(__ffma2_rn(T[r0 + r + 1][0], i1, sr_delta_pair(h.z)), M2);
            y3 = __fadd2_rn(__ffma2_rn(T[r0 + r + 1][1], i1, sr_delta_pair(h.w)), M2);
        } else {
            y0 = __ffma2_rn(T[r0 + r][0], i0, M2);
            y1 = __ffma2_rn(T[r0 + r][1], i0, M2);
            y2 = __ffma2_rn(T[r0 + r + 1][0], i1, M2);
            y3 = __ffma2_rn(T[r0 + r + 1][1], i1, M2);
        }
        ub[r] = low_bytes(y0.x, y0.y, y1.x, y1.y);
        ub[r + 1] = low_bytes(y2.x, y2.y, y3.x, y3.y);
    }
    pack_int_block<B>(blk, lane, ub);
}

__device__ __forceinline__ void requant_fp16(uint8_t *blk, int lane, const float2 (&T)[kRowsPerWarp][2],
                                             int r0) {
    uint32_t w[32];
#pragma unroll
    for (int r = 0; r < 16; ++r) {
        __half2 h01 = __floats2half2_rn(T[r0 + r][0].x, T[r0 + r][0].y);
        __half2 h23 = __floats2half2_rn(T[r0 + r][1].x, T[r0 + r][1].y);
        w[2 * r] = *reinterpret_cast<uint32_t *>(&h01);
        w[2 * r + 1] = *reinterpret_cast<uint32_t *>(&h23);
    }
    pack_fp16_block(blk, lane, w);
}

template <int BITS, int R0, bool SR>
__device__ __forceinline__ void requant_block(int bits, uint8_t *blk, int lane, const float *inv,
                                              const float2 (&T)[kRowsPerWarp][2], int s0, const SrCtx sr) {
    if constexpr (BITS == 16) requant_fp16(blk, lane, T, R0);
    else if constexpr (BITS != 0) requant_int<BITS, SR>(blk, lane, inv, T, R0, s0, sr);
    else {
        switch (bits) {
            case 16: requant_fp16(blk, lane, T, R0); break;
            case 8: requant_int<8, SR>(blk, lane, inv, T, R0, s0, sr); break;
            case 7: requant_int<7, SR>(blk, lane, inv, T, R0, s0, sr); break;
            case 6: requant_int<6, SR>(blk, lane, inv, T, R0, s0, sr); break;
            case 5: requant_int<5, SR>(blk, lane, inv, T, R0, s0, sr); break;
            case 4: requant_int<4, SR>(blk, lane, inv, T, R0, s0, sr); break;
            case 3: requant_int<3, SR>(blk, lane, inv, T, R0, s0, sr); break;
            default: requant_int<2, SR>(blk, lane, inv, T, R0, s0, sr); break;
        }
    }
}

// ---- S3 / S5 partial sums of one 16-row block: chains p = fma(w_s, X_s, p)
// from 0 in ascending row order, two column pairs.
template <int R0>
__device__ __forceinline__ void block_chain(const float *w, const float2 (&X)[kRowsPerWarp][2],
                                            float2 &p01, float2 &p23) {
    p01 = make_float2(0.f, 0.f);
    p23 = make_float2(0.f, 0.f);
#pragma unroll
    for (int r = 0; r < 16; r += 4) {
        const float4 ww = *reinterpret_cast<const float4 *>(w + r);
        const float wv[4] = {ww.x, ww.y, ww.z, ww.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            p01 = __ffma2_rn(make_float2(wv[i], wv[i]), X[R0 + r + i][0], p01);
            p23 = __ffma2_rn(make_float2(wv[i], wv[i]), X[R0 + r + i][1], p23);
        }
    }
}

__device__ __forceinline__ void issue_stage(const DevFormat &F, const DecodeArgs &A, uint8_t *dst, int p,
                                            uint64_t *bar) {
    mbar_expect_tx(bar, decode_stage_bytes(F));
    bulk_g2s(dst, A.pages + (size_t)p * F.page_bytes, (uint32_t)F.page_bytes, bar);
    uint8_t *rows = dst + F.page_bytes;
    bulk_g2s(rows, A.q + (size_t)p * kD, 512, bar);
    bulk_g2s(rows + 512, A.k + (size_t)p * kD, 512, bar);
    bulk_g2s(rows + 1024, A.v + (size_t)p * kD, 512, bar);
    if (F.gate_vector) bulk_g2s(rows + 1536, A.alpha + (size_t)p * kD, 512, bar);
}

// o of a finished page: the tree over the warps' block-pair partials, times c.
__device__ __forceinline__ void write_o(const float (*red_o)[kD], const DecodeArgs &A, int p, int lane,
                                        const float *c_prev, int col_scales) {
    const float4 o0 = *reinterpret_cast<const float4 *>(&red_o[0][4 * lane]);
    const float4 o1 = *reinterpret_cast<const float4 *>(&red_o[1][4 * lane]);
    const float4 o2 = *reinterpret_cast<const float4 *>(&red_o[2][4 * lane]);
    const float4 o3 = *reinterpret_cast<const float4 *>(&red_o[3][4 * lane]);
    float2 oa = __fadd2_rn(__fadd2_rn(make_float2(o0.x, o0.y), make_float2(o1.x, o1.y)),
                           __fadd2_rn(make_float2(o2.x, o2.y), make_float2(o3.x, o3.y)));
    float2 ob = __fadd2_rn(__fadd2_rn(make_float2(o0.z, o0.w), make_float2(o1.z, o1.w)),
                           __fadd2_rn(make_float2(o2.z, o2.w), make_float2(o3.z, o3.w)));
    if (col_scales) {
        const float4 c = *reinterpret_cast<const float4 *>(&c_prev[4 * lane]);
        oa = __fmul2_rn(make_float2(c.x, c.y), oa);
        ob = __fmul2_rn(make_float2(c.z, c.w), ob);
    }
    *reinterpret_cast<float4 *>(A.o + (size_t)p * kD + 4 * lane) = make_float4(oa.x, oa.y, ob.x, ob.y);
}

// Resident CTAs per SM the register budget is sized for: 3 (168 registers);
// the stochastic-rounding variant carries the Philox state and gets 2.
template <bool SR>
constexpr int decode_ctas_per_sm() { return SR ? 2 : 3; }

// Iteration index at which a CTA processed page p.
__device__ __forceinline__ int it_last(int p, unsigned first, unsigned stride) {
    return (p - (int)first) / (int)stride;
}

__device__ __forceinline__ float absmax4(float2 a, float2 b) {
    return fmaxf(fmaxf(fabsf(a.x), fabsf(a.y)), fmaxf(fabsf(b.x), fabsf(b.y)));
}

// The per-page loop (every warp runs this one body; warp w owns blocks 2w, 2w+1).
template <bool SR>
__global__ void __launch_bounds__(kThreads, decode_ctas_per_sm<SR>())
decode_kernel(const DevFormat F, const DecodeArgs A) {
    extern __shared__ __align__(128) uint8_t smem[];
    SmemFixed &S = *reinterpret_cast<SmemFixed *>(smem);
    uint8_t *stages = smem + kFixedBytes;
    const int warp = threadIdx.x >> 5;
    constexpr int BA = 0, BB = 0;   // block widths come from F at run time

    if (threadIdx.x == 0) {
        for (int st = 0; st < A.n_stages; ++st) mbar_init(&S.full[st], 1);
        mbar_init(&S.never, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int i = 0; i < A.n_stages; ++i) {
            const int p = (int)blockIdx.x + i * (int)gridDim.x;
            if (p < A.n_pages) issue_stage(F, A, stages + i * A.stage_bytes, p, &S.full[i]);
        }
    }
    const int tid = threadIdx.x, lane = tid & 31;
    const int stride = (int)gridDim.x;
    const int n = A.n_pages;
    const int NS = A.n_stages;
    // (request, head) of a page is carried along: p advances by `stride`,
    // i.e. by (stride / H, stride % H) with a carry
    const int H = A.heads;
    const int sb = stride / H, sh = stride % H;

    int p = (int)blockIdx.x;
    int pb = p / H, ph = p % H;            // request and head of page p
    float alpha_s = 0.f, beta_s = 0.f;
    int kap = 0;
    if (p < n) {
        beta_s = __ldg(A.beta + p);
        if (!F.gate_vector) alpha_s = __ldg(A.alpha + p);
        kap = __ldg(A.perm + ph * kD + tid) & (kD - 1);
    }
    const int b0 = 2 * warp, b1 = 2 * warp + 1;
    const int bits0 = BA ? BA : F.blk_bits(b0), bits1 = BB ? BB : F.blk_bits(b1);
    const int off0 = F.blk_off(b0), off1 = F.blk_off(b1);
    // this lane's row of S6 (row 32w + lane) and its scales' constants
    const int my_bits = (lane < 16) ? bits0 : bits1;
    const float my_qmax = (my_bits == 16) ? 0.f : (float)((1 << (my_bits - 1)) - 1);
    const float my_rcp = (my_bits == 16) ? 0.f : __frcp_rn(my_qmax);
    const int my_r = F.blk_rbase(lane < 16 ? b0 : b1) + (lane & 15);
    float *rmx = S.rmx[warp];
    int p_prev = -1;                  // page whose o is still to be written
    int st = 0;
    uint32_t parity = 0;

    for (int it = 0; p < n; ++it) {
        // scalars of the next page, loaded early
        const int pn = p + stride;
        int pnb = pb + sb, pnh = ph + sh;
        if (pnh >= H) { pnh -= H; ++pnb; }
        float alpha_n = 0.f, beta_n = 0.f;
        int kap_n = 0;
        if (pn < n) {
            beta_n = __ldg(A.beta + pn);
            if (!F.gate_vector) alpha_n = __ldg(A.alpha + pn);
            kap_n = __ldg(A.perm + pnh * kD + tid) & (kD - 1);
        }

        // a wait that runs out is voted on at the page's barrier, before
        // anything of the page is written
        bool ok;
        if (A.stall_first_wait && it == 0) ok = mbar_wait_bounded(&S.never, 0, A.wait_limit_ns);
        else ok = mbar_wait_bounded(&S.full[st], parity, A.wait_limit_ns);
        const int par = it & 1;
        const uint8_t *stg = stages + st * A.stage_bytes;
        const float *q_s = reinterpret_cast<const float *>(stg + F.page_bytes);
        const float *k_s = q_s + kD;
        const float *v_s = q_s + 2 * kD;
        const float *al_s = q_s + 3 * kD;

        // per stored row s = tid: decay x row scale, permuted k and q, beta k
        {
            const int s = tid, blk = s >> 4;
            const float kk = k_s[kap], qq = q_s[kap];
            const float al = F.gate_vector ? al_s[kap] : alpha_s;
            float a = al;
            if (F.blk_kind(blk) == kKindInt) {
                const float r = reinterpret_cast<const float *>(stg + F.r_off)[F.blk_rbase(blk) + (s & 15)];
                a = __fmul_rn(al, r);
            }
            const float bk = __fmul_rn(beta_s, kk);
            if (F.col_scales)   // thread s also inverts the scale of column s
                S.ic[par][s] = __frcp_rn(reinterpret_cast<const float *>(stg + F.c_off)[s]);
            S.a[s] = a;
            S.kp[s] = kk;
            S.qp[s] = qq;
            S.bk[s] = bk;
        }
        __syncwarp();   // the warp's rows' operands come from its own lanes

        // S1 + S2, and S3's block chains
        float2 T[kRowsPerWarp][2];
        dequant_block<BA, 0>(bits0, stg + off0, lane, &S.a[32 * warp], T);
        dequant_block<BB, 16>(bits1, stg + off1, lane, &S.a[32 * warp + 16], T);
        {
            float2 pa01, pa23, pb01, pb23;
            block_chain<0>(&S.kp[32 * warp], T, pa01, pa23);
            block_chain<16>(&S.kp[32 * warp + 16], T, pb01, pb23);
            const float2 w01 = __fadd2_rn(pa01, pb01), w23 = __fadd2_rn(pa23, pb23);
            *reinterpret_cast<float4 *>(&S.red_u[par][warp][4 * lane]) = make_float4(w01.x, w01.y, w23.x, w23.y);
        }
        const float4 v4 = *reinterpret_cast<const float4 *>(v_s + 4 * lane);
        float4 c4 = make_float4(1.f, 1.f, 1.f, 1.f);
        if (F.col_scales) c4 = *reinterpret_cast<const float4 *>(stg + F.c_off + 16 * lane);
        if (__syncthreads_or(!ok)) {
            // a stage never arrived: record it, let the copies already issued
            // into the ring land, and leave; nothing of this page was written
            if (tid == 0) {
                atomicOr(A.status, kStatusTimeout);
                for (int i = 0; i < NS; ++i) {
                    const int pi = p + i * stride;
                    if (pi < n) {
                        const int ii = it + i;
                        mbar_wait_bounded(&S.full[ii % NS], (uint32_t)((ii / NS) & 1), A.wait_limit_ns);
                    }
                }
            }
            __syncthreads();
            return;
        }

        // the stage is no longer read: refill it with the page NS iterations ahead
        if (tid == 0) {
            const int pr = p + NS * stride;
            if (pr < n) {
                fence_proxy_async_smem();
                issue_stage(F, A, stages + st * A.stage_bytes, pr, &S.full[st]);
            }
        }
        // o of the previous page (its block partials were stored before this barrier)
        if (warp == 0 && p_prev >= 0) {
            write_o(S.red_o[par ^ 1], A, p_prev, lane, S.c_prev, F.col_scales);
            if (F.col_scales) *reinterpret_cast<float4 *>(&S.c_prev[4 * lane]) = c4;
        }

        // u = ((P0+P1)+(P2+P3))+((P4+P5)+(P6+P7)); e = v (1/c) - u
        float2 e01, e23;
        {
            const float4 u0 = *reinterpret_cast<const float4 *>(&S.red_u[par][0][4 * lane]);
            const float4 u1 = *reinterpret_cast<const float4 *>(&S.red_u[par][1][4 * lane]);
            const float4 u2 = *reinterpret_cast<const float4 *>(&S.red_u[par][2][4 * lane]);
            const float4 u3 = *reinterpret_cast<const float4 *>(&S.red_u[par][3][4 * lane]);
            const float2 ua = __fadd2_rn(__fadd2_rn(make_float2(u0.x, u0.y), make_float2(u1.x, u1.y)),
                                         __fadd2_rn(make_float2(u2.x, u2.y), make_float2(u3.x, u3.y)));
            const float2 ub = __fadd2_rn(__fadd2_rn(make_float2(u0.z, u0.w), make_float2(u1.z, u1.w)),
                                         __fadd2_rn(make_float2(u2.z, u2.w), make_float2(u3.z, u3.w)));
            float4 ic = make_float4(1.f, 1.f, 1.f, 1.f);
            if (F.col_scales) ic = *reinterpret_cast<const float4 *>(&S.ic[par][4 * lane]);
            // two roundings, scalar: an f32x2 multiply feeding an f32x2 add is
            // fused by the compiler into one f32x2 fma
            e01 = make_float2(__fsub_rn(__fmul_rn(v4.x, ic.x), ua.x), __fsub_rn(__fmul_rn(v4.y, ic.y), ua.y));
            e23 = make_float2(__fsub_rn(__fmul_rn(v4.z, ic.z), ub.x), __fsub_rn(__fmul_rn(v4.w, ic.w), ub.y));
        }

        // S4: T' = T + (beta k) e; row partial maxima into the row-max tile
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; r += 4) {
            const float4 bb = *reinterpret_cast<const float4 *>(&S.bk[32 * warp + r]);
            const float bv[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                T[r + i][0] = __ffma2_rn(make_float2(bv[i], bv[i]), e01, T[r + i][0]);
                T[r + i][1] = __ffma2_rn(make_float2(bv[i], bv[i]), e23, T[r + i][1]);
                rmx[(r + i) * kRmxPitch + lane] = absmax4(T[r + i][0], T[r + i][1]);
            }
        }
        // S5: block chains of o, finished at the next page's first barrier
        {
            float2 pa01, pa23, pb01, pb23;
            block_chain<0>(&S.qp[32 * warp], T, pa01, pa23);
            block_chain<16>(&S.qp[32 * warp + 16], T, pb01, pb23);
            const float2 w01 = __fadd2_rn(pa01, pb01), w23 = __fadd2_rn(pa23, pb23);
            *reinterpret_cast<float4 *>(&S.red_o[par][warp][4 * lane]) = make_float4(w01.x, w01.y, w23.x, w23.y);
        }
        __syncwarp();

        // S6: lane l reduces row l of its warp: r' = m / qmax, inv = qmax / m (toward zero)
        uint8_t *page = A.pages + (size_t)p * (size_t)F.page_bytes;
        {
            const float4 *row = reinterpret_cast<const float4 *>(rmx + lane * kRmxPitch);
            float m = 0.f;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const float4 x = row[c];
                m = fmaxf(m, fmaxf(fmaxf(x.x, x.y), fmaxf(x.z, x.w)));
            }
            float inv = 0.f;
            if (my_bits != 16) {
                float r = 0.f;
                if (m > 0.f) {
                    r = div_by_qmax(m, my_qmax, my_rcp);
                    inv = __fdiv_rz(my_qmax, m);
                }
                reinterpret_cast<float *>(page + F.r_off)[my_r] = r;
            }
            S.inv[warp][lane] = inv;
        }
        __syncwarp();

        // S7 + S8
        SrCtx sr;
        sr.k0 = A.seed_lo; sr.k1 = A.seed_hi; sr.step = A.step;
        sr.b = (uint32_t)pb; sr.h = (uint32_t)ph;
        requant_block<BA, 0, SR>(bits0, page + off0, lane, &S.inv[warp][0], T, 32 * warp, sr);
        requant_block<BB, 16, SR>(bits1, page + off1, lane, &S.inv[warp][16], T, 32 * warp + 16, sr);

        if (warp == 0 && p_prev < 0 && F.col_scales) *reinterpret_cast<float4 *>(&S.c_prev[4 * lane]) = c4;
        p_prev = p;
        alpha_s = alpha_n;
        beta_s = beta_n;
        kap = kap_n;
        p = pn;
        pb = pnb;
        ph = pnh;
        if (++st == NS) { st = 0; parity ^= 1u; }
    }
    __syncthreads();
    if (warp == 0 && p_prev >= 0) write_o(S.red_o[(it_last(p_prev, blockIdx.x, gridDim.x)) & 1], A, p_prev, lane,
                                          S.c_prev, F.col_scales);
}

static int decode_stages(size_t stride, int ctas_per_sm) {
    // as many ring stages as fit next to the fixed part at the target occupancy
    int dev = 0, smem_sm = 0, reserved = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
    cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
    const long budget = (long)smem_sm / ctas_per_sm - reserved - (long)kFixedBytes;
    long ns = budget / (long)stride;
    if (ns > kMaxStages) ns = kMaxStages;
    if (ns < 2) ns = 2;
    return (int)ns;
}

cudaError_t launch_decode(const stq_state *s, const float *q, const float *k, const float *v,
                          const float *alpha, const float *beta, float *o, uint64_t seed, uint32_t step,
                          int stall_first_wait, cudaStream_t stream) {
    const DevFormat &F = s->dev;
    DecodeArgs A;
    A.pages = s->base + s->pages_offset;
    A.perm = s->base + s->perm_offset;
    A.status = reinterpret_cast<uint32_t *>(s->base + s->status_offset);
    A.q = q; A.k = k; A.v = v; A.alpha = alpha; A.beta = beta; A.o = o;
    A.n_pages = s->batch * s->heads;
    A.heads = s->heads;
    A.stage_bytes = (decode_stage_bytes(F) + 127) / 128 * 128;
    A.n_stages = decode_stages(A.stage_bytes, F.stochastic ? decode_ctas_per_sm<true>() : decode_ctas_per_sm<false>());
    A.seed_lo = (uint32_t)seed;
    A.seed_hi = (uint32_t)(seed >> 32);
    A.step = step;
    A.wait_limit_ns = s->wait_limit_ns;
    A.stall_first_wait = stall_first_wait;
    const size_t smem = kFixedBytes + (size_t)A.n_stages * A.stage_bytes;
    const void *fn = F.stochastic ? (const void *)decode_kernel<true> : (const void *)decode_kernel<false>;
    cudaError_t err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    const int grid = persistent_grid(fn, kThreads, smem, A.n_pages);
    if (grid <= 0) return cudaErrorInvalidConfiguration;
    if (F.stochastic)
        decode_kernel<true><<<grid, kThreads, smem, stream>>>(F, A);
    else
        decode_kernel<false><<<grid, kThreads, smem, stream>>>(F, A);
    return cudaGetLastError();
}

}  // namespace stq
