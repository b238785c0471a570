// stq_decode.cu -- the fused decode-step kernel (sm_100a).
//
// One persistent CTA of 128 threads walks pages p = blockIdx.x + i*gridDim.x.
// Each page's bytes and its q, k, v (and KDA alpha) rows are brought into a
// shared-memory ring by one thread with cp.async.bulk (no multicast), counted
// on an mbarrier; the ring is kStages deep so copies of later pages overlap
// the math of the current one.  Per page, all in registers / shared memory:
//   S1 unpack planes -> S2 dequant + decay T = z (alpha r)
//   S3 column sums u = sum_s k_s T_s (blocks of 32 rows, one per warp, then
//      (P0+P1)+(P2+P3)),  e = v (1/c) - u
//   S4 T' = T + (beta k_s) e      S5 o = c * sum_s q_s T'_s
//   S6 row absmax -> r' = m/qmax, inv = qmax/m rounded toward zero
//   S7 requant (RNE of the exact product, or Philox stochastic rounding on
//      INT rows; binary16 on FP16 rows)   S8 repack and store in place.
// The state crosses HBM once each way per step.  No tensor cores: the work
// is rank-1 updates and mat-vecs.
#include "stq_internal.h"

#include <cstdio>

namespace stq {

struct DecodeArgs {
    uint8_t *pages;
    const uint8_t *perm;
    uint32_t *status;
    const float *q, *k, *v, *alpha, *beta;
    float *o;
    long n_pages;
    int heads;
    uint32_t stage_bytes;
    uint32_t seed_lo, seed_hi, step;
    uint64_t wait_limit_ns;
    int stall_first_wait;
};

struct SmemFixed {
    float kp[kD], qp[kD], a[kD], bk[kD];   // per stored row: k, q, alpha*r, beta*k
    float red_u[kWarps][kD];                // block partials of u
    float red_o[kWarps][kD];                // block partials of o
    float inv[kWarps][kRowsPerWarp];        // per-row requant multipliers
    uint64_t full[kStages];                 // stage-full barriers
    uint64_t never;                         // a barrier nothing completes (test hook)
};

constexpr size_t kFixedBytes = (sizeof(SmemFixed) + 127) / 128 * 128;

__host__ __device__ inline uint32_t decode_stage_bytes(const DevFormat &F) {
    return (uint32_t)F.page_bytes + 3u * 512u + (F.gate_vector ? 512u : 0u);
}

// ---- S1 + S2: one 16-row block into T (rows 16*half .. 16*half+15 of the warp)
template <int B>
__device__ __forceinline__ void dequant_int(const uint8_t *blk, int lane, const float *a,
                                            float2 (&T)[kRowsPerWarp][2], int r0) {
    uint32_t ub[16];
    unpack_int_block<B>(blk, lane, ub);
    const float bm = 8388608.0f + (float)(1 << (B - 1));
#pragma unroll
    for (int r = 0; r < 16; ++r) {
        float2 z01, z23;
        codes_to_float(ub[r], bm, z01, z23);
        const float as = a[r];
        T[r0 + r][0] = __fmul2_rn(z01, make_float2(as, as));
        T[r0 + r][1] = __fmul2_rn(z23, make_float2(as, as));
    }
}

__device__ __forceinline__ void dequant_fp16(const uint8_t *blk, int lane, const float *a,
                                             float2 (&T)[kRowsPerWarp][2], int r0) {
    uint32_t w[32];
    unpack_fp16_block(blk, lane, w);
#pragma unroll
    for (int r = 0; r < 16; ++r) {
        const float as = a[r];
        float2 x01 = __half22float2(*reinterpret_cast<const __half2 *>(&w[2 * r]));
        float2 x23 = __half22float2(*reinterpret_cast<const __half2 *>(&w[2 * r + 1]));
        T[r0 + r][0] = __fmul2_rn(x01, make_float2(as, as));
        T[r0 + r][1] = __fmul2_rn(x23, make_float2(as, as));
    }
}

template <int R0>
__device__ __forceinline__ void dequant_block(int kind, int bits, const uint8_t *blk, int lane,
                                              const float *a, float2 (&T)[kRowsPerWarp][2]) {
    if (kind == kKindFp16) { dequant_fp16(blk, lane, a, T, R0); return; }
    switch (bits) {
        case 8: dequant_int<8>(blk, lane, a, T, R0); break;
        case 7: dequant_int<7>(blk, lane, a, T, R0); break;
        case 6: dequant_int<6>(blk, lane, a, T, R0); break;
        case 5: dequant_int<5>(blk, lane, a, T, R0); break;
        case 4: dequant_int<4>(blk, lane, a, T, R0); break;
        case 3: dequant_int<3>(blk, lane, a, T, R0); break;
        default: dequant_int<2>(blk, lane, a, T, R0); break;
    }
}

// ---- S7 + S8: requantize one 16-row block of T' and store its planes.
struct SrCtx {
    uint32_t k0, k1, step, b, h;
};

template <int B, bool SR>
__device__ __forceinline__ void requant_int(uint8_t *blk, int lane, const float *inv,
                                            const float2 (&T)[kRowsPerWarp][2], int r0, int s0,
                                            const SrCtx &sr) {
    const float M = 12582912.0f + (float)(1 << (B - 1));   // 1.5 * 2^23 + bias
    const float2 M2 = make_float2(M, M);
    uint32_t ub[16];
#pragma unroll
    for (int r = 0; r < 16; r += 2) {
        const float i0 = inv[r], i1 = inv[r + 1];
        float2 y0, y1, y2, y3;
        if constexpr (SR) {
            const int s = s0 + r;   // even
            const uint4 h = philox4x32_10(
                make_uint4((uint32_t)(s >> 1) * 32u + (uint32_t)lane, sr.step, sr.b, sr.h), sr.k0, sr.k1);
            y0 = __fadd2_rn(__ffma2_rn(T[r0 + r][0], make_float2(i0, i0), sr_delta_pair(h.x)), M2);
            y1 = __fadd2_rn(__ffma2_rn(T[r0 + r][1], make_float2(i0, i0), sr_delta_pair(h.y)), M2);
            y2 = __fadd2_rn(__ffma2_rn(T[r0 + r + 1][0], make_float2(i1, i1), sr_delta_pair(h.z)), M2);
            y3 = __fadd2_rn(__ffma2_rn(T[r0 + r + 1][1], make_float2(i1, i1), sr_delta_pair(h.w)), M2);
        } else {
            y0 = __ffma2_rn(T[r0 + r][0], make_float2(i0, i0), M2);
            y1 = __ffma2_rn(T[r0 + r][1], make_float2(i0, i0), M2);
            y2 = __ffma2_rn(T[r0 + r + 1][0], make_float2(i1, i1), M2);
            y3 = __ffma2_rn(T[r0 + r + 1][1], make_float2(i1, i1), M2);
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

template <int R0, bool SR>
__device__ __forceinline__ void requant_block(int kind, int bits, uint8_t *blk, int lane, const float *inv,
                                              const float2 (&T)[kRowsPerWarp][2], int s0, const SrCtx &sr) {
    if (kind == kKindFp16) { requant_fp16(blk, lane, T, R0); return; }
    switch (bits) {
        case 8: requant_int<8, SR>(blk, lane, inv, T, R0, s0, sr); break;
        case 7: requant_int<7, SR>(blk, lane, inv, T, R0, s0, sr); break;
        case 6: requant_int<6, SR>(blk, lane, inv, T, R0, s0, sr); break;
        case 5: requant_int<5, SR>(blk, lane, inv, T, R0, s0, sr); break;
        case 4: requant_int<4, SR>(blk, lane, inv, T, R0, s0, sr); break;
        case 3: requant_int<3, SR>(blk, lane, inv, T, R0, s0, sr); break;
        default: requant_int<2, SR>(blk, lane, inv, T, R0, s0, sr); break;
    }
}

__device__ __forceinline__ void issue_stage(const DevFormat &F, const DecodeArgs &A, uint8_t *dst, long p,
                                            uint64_t *bar) {
    mbar_expect_tx(bar, decode_stage_bytes(F));
    bulk_g2s(dst, A.pages + (size_t)p * F.page_bytes, (uint32_t)F.page_bytes, bar);
    uint8_t *rows = dst + F.page_bytes;
    bulk_g2s(rows, A.q + (size_t)p * kD, 512, bar);
    bulk_g2s(rows + 512, A.k + (size_t)p * kD, 512, bar);
    bulk_g2s(rows + 1024, A.v + (size_t)p * kD, 512, bar);
    if (F.gate_vector) bulk_g2s(rows + 1536, A.alpha + (size_t)p * kD, 512, bar);
}

template <bool SR>
__global__ void __launch_bounds__(kThreads, 2)
decode_kernel(const DevFormat F, const DecodeArgs A) {
    extern __shared__ __align__(128) uint8_t smem[];
    SmemFixed &S = *reinterpret_cast<SmemFixed *>(smem);
    uint8_t *stages = smem + kFixedBytes;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const long stride = gridDim.x;
    const long n = A.n_pages;

    if (tid == 0) {
        for (int st = 0; st < kStages; ++st) mbar_init(&S.full[st], 1);
        mbar_init(&S.never, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            long p = blockIdx.x + i * stride;
            if (p < n) issue_stage(F, A, stages + i * A.stage_bytes, p, &S.full[i]);
        }
    }

    long p = blockIdx.x;
    float alpha_s = 0.f, beta_s = 0.f;
    int kap = 0;
    if (p < n) {
        beta_s = __ldg(A.beta + p);
        if (!F.gate_vector) alpha_s = __ldg(A.alpha + p);
        kap = __ldg(A.perm + (size_t)(p % A.heads) * kD + tid) & (kD - 1);
    }

    for (long it = 0; p < n; ++it, p += stride) {
        const int st = (int)(it % kStages);
        const uint32_t parity = (uint32_t)((it / kStages) & 1);
        // scalars of the next page, loaded early
        const long pn = p + stride;
        float alpha_n = 0.f, beta_n = 0.f;
        int kap_n = 0;
        if (pn < n) {
            beta_n = __ldg(A.beta + pn);
            if (!F.gate_vector) alpha_n = __ldg(A.alpha + pn);
            kap_n = __ldg(A.perm + (size_t)(pn % A.heads) * kD + tid) & (kD - 1);
        }

        bool ok;
        if (A.stall_first_wait && it == 0) ok = mbar_wait_bounded(&S.never, 0, A.wait_limit_ns);
        else ok = mbar_wait_bounded(&S.full[st], parity, A.wait_limit_ns);
        if (__syncthreads_or(!ok)) {
            if (tid == 0) {
                atomicOr(A.status, kStatusTimeout);
                // let the copies already issued into the ring land before exiting
                for (int i = 0; i < kStages; ++i) {
                    long pi = p + i * stride;
                    if (pi < n) {
                        long ii = it + i;
                        mbar_wait_bounded(&S.full[ii % kStages], (uint32_t)((ii / kStages) & 1), A.wait_limit_ns);
                    }
                }
            }
            __syncthreads();
            return;
        }
        const uint8_t *stg = stages + st * A.stage_bytes;
        const float *q_s = reinterpret_cast<const float *>(stg + F.page_bytes);
        const float *k_s = q_s + kD;
        const float *v_s = q_s + 2 * kD;
        const float *al_s = q_s + 3 * kD;

        // per stored row s = tid: permuted k, q, decay x row scale, beta k
        {
            const int s = tid, blk = s >> 4;
            const float kk = k_s[kap], qq = q_s[kap];
            const float al = F.gate_vector ? al_s[kap] : alpha_s;
            float a = al;
            if (F.blk_kind(blk) == kKindInt) {
                const float r = reinterpret_cast<const float *>(stg + F.r_off)[F.blk_rbase(blk) + (s & 15)];
                a = __fmul_rn(al, r);
            }
            S.kp[s] = kk;
            S.qp[s] = qq;
            S.a[s] = a;
            S.bk[s] = __fmul_rn(beta_s, kk);
        }
        __syncthreads();

        // S1 + S2
        float2 T[kRowsPerWarp][2];
        const int b0 = 2 * warp, b1 = 2 * warp + 1;
        dequant_block<0>(F.blk_kind(b0), F.blk_bits(b0), stg + F.blk_off(b0), lane, &S.a[32 * warp], T);
        dequant_block<16>(F.blk_kind(b1), F.blk_bits(b1), stg + F.blk_off(b1), lane, &S.a[32 * warp + 16], T);

        // S3: this warp's block partial of u
        {
            float2 P0 = make_float2(0.f, 0.f), P1 = make_float2(0.f, 0.f);
#pragma unroll
            for (int r = 0; r < kRowsPerWarp; ++r) {
                const float kk = S.kp[32 * warp + r];
                P0 = __ffma2_rn(make_float2(kk, kk), T[r][0], P0);
                P1 = __ffma2_rn(make_float2(kk, kk), T[r][1], P1);
            }
            *reinterpret_cast<float4 *>(&S.red_u[warp][4 * lane]) = make_float4(P0.x, P0.y, P1.x, P1.y);
        }
        const float4 v4 = *reinterpret_cast<const float4 *>(v_s + 4 * lane);
        float4 c4 = make_float4(1.f, 1.f, 1.f, 1.f);
        if (F.col_scales) c4 = *reinterpret_cast<const float4 *>(stg + F.c_off + 16 * lane);
        __syncthreads();

        // the stage is no longer read: refill it with the page kStages iterations ahead
        if (tid == 0) {
            long pr = p + kStages * stride;
            if (pr < n) {
                fence_proxy_async_smem();
                issue_stage(F, A, stages + st * A.stage_bytes, pr, &S.full[st]);
            }
        }

        float2 e01, e23;
        {
            const float4 u0 = *reinterpret_cast<const float4 *>(&S.red_u[0][4 * lane]);
            const float4 u1 = *reinterpret_cast<const float4 *>(&S.red_u[1][4 * lane]);
            const float4 u2 = *reinterpret_cast<const float4 *>(&S.red_u[2][4 * lane]);
            const float4 u3 = *reinterpret_cast<const float4 *>(&S.red_u[3][4 * lane]);
            const float2 ua = __fadd2_rn(__fadd2_rn(make_float2(u0.x, u0.y), make_float2(u1.x, u1.y)),
                                         __fadd2_rn(make_float2(u2.x, u2.y), make_float2(u3.x, u3.y)));
            const float2 ub = __fadd2_rn(__fadd2_rn(make_float2(u0.z, u0.w), make_float2(u1.z, u1.w)),
                                         __fadd2_rn(make_float2(u2.z, u2.w), make_float2(u3.z, u3.w)));
            float4 ic = make_float4(1.f, 1.f, 1.f, 1.f);
            if (F.col_scales)
                ic = make_float4(__fdiv_rn(1.f, c4.x), __fdiv_rn(1.f, c4.y), __fdiv_rn(1.f, c4.z),
                                 __fdiv_rn(1.f, c4.w));
            // e = v (1/c) - u with two roundings.  Scalar __fmul_rn/__fsub_rn:
            // the compiler fuses an f32x2 multiply feeding an f32x2 add into one
            // f32x2 fma, which would round once.
            e01 = make_float2(__fsub_rn(__fmul_rn(v4.x, ic.x), ua.x), __fsub_rn(__fmul_rn(v4.y, ic.y), ua.y));
            e23 = make_float2(__fsub_rn(__fmul_rn(v4.z, ic.z), ub.x), __fsub_rn(__fmul_rn(v4.w, ic.w), ub.y));
        }

        // S4 + S5 partial + row absmax partial
        float rm[kRowsPerWarp];
        {
            float2 P0 = make_float2(0.f, 0.f), P1 = make_float2(0.f, 0.f);
#pragma unroll
            for (int r = 0; r < kRowsPerWarp; ++r) {
                const float bk = S.bk[32 * warp + r];
                T[r][0] = __ffma2_rn(make_float2(bk, bk), e01, T[r][0]);
                T[r][1] = __ffma2_rn(make_float2(bk, bk), e23, T[r][1]);
                const float qq = S.qp[32 * warp + r];
                P0 = __ffma2_rn(make_float2(qq, qq), T[r][0], P0);
                P1 = __ffma2_rn(make_float2(qq, qq), T[r][1], P1);
                rm[r] = fmaxf(fmaxf(fabsf(T[r][0].x), fabsf(T[r][0].y)),
                              fmaxf(fabsf(T[r][1].x), fabsf(T[r][1].y)));
            }
            *reinterpret_cast<float4 *>(&S.red_o[warp][4 * lane]) = make_float4(P0.x, P0.y, P1.x, P1.y);
        }
        __syncthreads();

        if (warp == 0) {
            const float4 o0 = *reinterpret_cast<const float4 *>(&S.red_o[0][4 * lane]);
            const float4 o1 = *reinterpret_cast<const float4 *>(&S.red_o[1][4 * lane]);
            const float4 o2 = *reinterpret_cast<const float4 *>(&S.red_o[2][4 * lane]);
            const float4 o3 = *reinterpret_cast<const float4 *>(&S.red_o[3][4 * lane]);
            float2 oa = __fadd2_rn(__fadd2_rn(make_float2(o0.x, o0.y), make_float2(o1.x, o1.y)),
                                   __fadd2_rn(make_float2(o2.x, o2.y), make_float2(o3.x, o3.y)));
            float2 ob = __fadd2_rn(__fadd2_rn(make_float2(o0.z, o0.w), make_float2(o1.z, o1.w)),
                                   __fadd2_rn(make_float2(o2.z, o2.w), make_float2(o3.z, o3.w)));
            if (F.col_scales) {
                oa = __fmul2_rn(make_float2(c4.x, c4.y), oa);
                ob = __fmul2_rn(make_float2(c4.z, c4.w), ob);
            }
            *reinterpret_cast<float4 *>(A.o + (size_t)p * kD + 4 * lane) = make_float4(oa.x, oa.y, ob.x, ob.y);
        }

        // S6: row absmax over the warp (reduce-scatter: lane ends with row `lane`)
#pragma unroll
        for (int off = 16, cnt = 32; off >= 1; off >>= 1, cnt >>= 1) {
            const bool upper = (lane & off) != 0;
#pragma unroll
            for (int i = 0; i < cnt / 2; ++i) {
                const float send = upper ? rm[i] : rm[i + cnt / 2];
                const float keep = upper ? rm[i + cnt / 2] : rm[i];
                rm[i] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, off));
            }
        }
        uint8_t *page = A.pages + (size_t)p * F.page_bytes;
        {
            const int s = 32 * warp + lane, blk = s >> 4;
            const float m = rm[0];
            float inv = 0.f;
            if (F.blk_kind(blk) == kKindInt) {
                const float qmax = (float)((1 << (F.blk_bits(blk) - 1)) - 1);
                float r = 0.f;
                if (m > 0.f) {
                    r = __fdiv_rn(m, qmax);
                    inv = __fdiv_rz(qmax, m);
                }
                reinterpret_cast<float *>(page + F.r_off)[F.blk_rbase(blk) + (s & 15)] = r;
            }
            S.inv[warp][lane] = inv;
        }
        __syncwarp();

        // S7 + S8
        SrCtx sr;
        sr.k0 = A.seed_lo; sr.k1 = A.seed_hi; sr.step = A.step;
        sr.b = (uint32_t)(p / A.heads); sr.h = (uint32_t)(p % A.heads);
        requant_block<0, SR>(F.blk_kind(b0), F.blk_bits(b0), page + F.blk_off(b0), lane, &S.inv[warp][0],
                             T, 32 * warp, sr);
        requant_block<16, SR>(F.blk_kind(b1), F.blk_bits(b1), page + F.blk_off(b1), lane, &S.inv[warp][16],
                              T, 32 * warp + 16, sr);

        alpha_s = alpha_n;
        beta_s = beta_n;
        kap = kap_n;
    }
}

static size_t decode_smem(const DevFormat &F) {
    return kFixedBytes + (size_t)kStages * ((decode_stage_bytes(F) + 127) / 128 * 128);
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
    A.n_pages = (long)s->batch * s->heads;
    A.heads = s->heads;
    A.stage_bytes = (decode_stage_bytes(F) + 127) / 128 * 128;
    A.seed_lo = (uint32_t)seed;
    A.seed_hi = (uint32_t)(seed >> 32);
    A.step = step;
    A.wait_limit_ns = s->wait_limit_ns;
    A.stall_first_wait = stall_first_wait;
    const size_t smem = decode_smem(F);
    const void *kern = F.stochastic ? (const void *)decode_kernel<true> : (const void *)decode_kernel<false>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    const int grid = persistent_grid(kern, smem, A.n_pages);
    if (grid <= 0) return cudaErrorInvalidConfiguration;
    if (F.stochastic)
        decode_kernel<true><<<grid, kThreads, smem, stream>>>(F, A);
    else
        decode_kernel<false><<<grid, kThreads, smem, stream>>>(F, A);
    return cudaGetLastError();
}

}  // namespace stq
