// stq_fit.cu -- joint fit of the row and column scales at quantization time
// (STEPQuant's scale fitting; cold path, once per calibration).
//
// STEPQuant fits key-row and value-column scales jointly from the state's
// distribution and each key row's impact on the output error.  The objective
// taken here is the impact-weighted squared reconstruction error over the INT
// rows,  E = sum_kappa w_kappa sum_j (S_kappa,j - z r c)^2,  minimized from the
// absmax scales by alternating exact steps, none of which can raise E:
//   z   <- the nearest codes for (r, c), clamped to [-qmax, qmax];
//   r_s <- sum_j S z c / sum_j (z c)^2                    (least squares per row)
//   c_j <- sum_k w S z r / sum_k w (z r)^2 over INT rows  (weighted, per column)
// and after the last round the codes once more for the final scales.
//
// One CTA of 128 threads per page (grid-stride).  The page's fp32 state sits
// in shared memory in natural key order; thread s owns stored row s for the
// codes and the row update, thread j owns column j for the column update.
// Every sum runs in double in a fixed order (j ascending for a row, kappa
// ascending for a column), each scale is rounded to float once per update,
// and a code is S / (r c) by one correctly rounded double division, so the
// result does not depend on the thread mapping.  The packed page is written
// with the quantizer's layout (warp w packs blocks 2w and 2w + 1).
#include "stq_internal.h"

namespace stq {

constexpr int kFitStride = kD + 1;        // floats per state row in shared memory (bank spread)
constexpr int kFitZStride = kD + 4;       // bytes per code row

struct FitSmem {
    float S[kD * kFitStride];             // the page's state, natural key order
    int8_t z[kD * kFitZStride];           // codes, stored row order
    float r[kD], c[kD], ic[kD], w[kD];    // scales (stored rows / columns), 1/c, impact (natural)
    int kap[kD];                          // stored row -> key channel
    int row_of[kD];                       // key channel -> stored row
};

__device__ __forceinline__ void fit_codes_row(FitSmem &M, int s, float qmax) {
    const float *Sr = M.S + M.kap[s] * kFitStride;
    const double r = (double)M.r[s];
    int8_t *zr = M.z + s * kFitZStride;
    for (int j = 0; j < kD; ++j) {
        const double d = __dmul_rn(r, (double)M.c[j]);
        double n = 0.0;
        if (d > 0.0) {
            n = rint(__ddiv_rn((double)Sr[j], d));
            n = fmin(fmax(n, -(double)qmax), (double)qmax);
        }
        zr[j] = (int8_t)(int)n;
    }
}

template <int B>
__device__ __forceinline__ void fit_pack_int(const FitSmem &M, uint8_t *blk, int s0, int lane) {
    uint32_t ub[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) {
        const int8_t *zr = M.z + (s0 + r) * kFitZStride + 4 * lane;
        uint32_t x = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) x |= (uint32_t)(uint8_t)(zr[b] + (1 << (B - 1))) << (8 * b);
        ub[r] = x;
    }
    pack_int_block<B>(blk, lane, ub);
}

__global__ void __launch_bounds__(kThreads) fit_kernel(const DevFormat F, const float *S, const float *impact,
                                                        const uint8_t *perm, uint8_t *pages, long n_pages,
                                                        int heads, int iters) {
    extern __shared__ __align__(16) uint8_t fit_smem[];
    FitSmem &M = *reinterpret_cast<FitSmem *>(fit_smem);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // this thread's stored row
    const int my_blk = tid >> 4;
    const bool my_int = F.blk_kind(my_blk) == kKindInt;
    const float my_qmax = my_int ? (float)((1 << (F.blk_bits(my_blk) - 1)) - 1) : 0.f;
    for (long p = blockIdx.x; p < n_pages; p += gridDim.x) {
        const int h = (int)(p % heads);
        __syncthreads();
        {
            const int k = perm[(size_t)h * kD + tid] & (kD - 1);   // a map byte is a channel < 128
            M.kap[tid] = k;
            M.row_of[k] = tid;
            M.w[tid] = impact ? impact[(size_t)h * kD + tid] : 1.f;
        }
        const float4 *Sp = reinterpret_cast<const float4 *>(S + (size_t)p * kD * kD);
#pragma unroll 4
        for (int i = 0; i < kD * kD / 4 / kThreads; ++i) {
            const int q = i * kThreads + tid;            // float4 index: row q / 32, columns 4 (q % 32) ..
            const float4 x = __ldg(Sp + q);
            float *dst = M.S + (q >> 5) * kFitStride + 4 * (q & 31);
            dst[0] = x.x; dst[1] = x.y; dst[2] = x.z; dst[3] = x.w;
        }
        __syncthreads();
        // the absmax start: c_j = max_kappa |S| (1 if zero), r_s = max_j |S / c| / qmax
        {
            float c = 1.f;
            if (F.col_scales) {
                float m = 0.f;
                for (int k = 0; k < kD; ++k) m = fmaxf(m, fabsf(M.S[k * kFitStride + tid]));
                c = m > 0.f ? m : 1.f;
            }
            M.c[tid] = c;
            M.ic[tid] = F.col_scales ? __fdiv_rn(1.f, c) : 1.f;
        }
        __syncthreads();
        {
            const float *Sr = M.S + M.kap[tid] * kFitStride;
            float m = 0.f;
            for (int j = 0; j < kD; ++j) m = fmaxf(m, fabsf(__fmul_rn(Sr[j], M.ic[j])));
            M.r[tid] = (my_int && m > 0.f) ? __fdiv_rn(m, my_qmax) : 0.f;
        }
        __syncthreads();
        for (int it = 0; it < iters; ++it) {
            if (my_int) {
                fit_codes_row(M, tid, my_qmax);
                // row scale: least squares for the codes with c fixed
                const float *Sr = M.S + M.kap[tid] * kFitStride;
                const int8_t *zr = M.z + tid * kFitZStride;
                double num = 0.0, den = 0.0;
                for (int j = 0; j < kD; ++j) {
                    const double zc = __dmul_rn((double)zr[j], (double)M.c[j]);
                    num = __dadd_rn(num, __dmul_rn((double)Sr[j], zc));
                    den = __dadd_rn(den, __dmul_rn(zc, zc));
                }
                if (den > 0.0) M.r[tid] = __double2float_rn(__ddiv_rn(num, den));
            }
            __syncthreads();
            if (F.col_scales) {
                // column scale: impact-weighted least squares with the codes and r fixed
                double num = 0.0, den = 0.0;
                for (int k = 0; k < kD; ++k) {
                    const int s = M.row_of[k];
                    if (F.blk_kind(s >> 4) != kKindInt) continue;
                    const double w = (double)M.w[k];
                    const double zr = __dmul_rn((double)M.z[s * kFitZStride + tid], (double)M.r[s]);
                    num = __dadd_rn(num, __dmul_rn(w, __dmul_rn((double)M.S[k * kFitStride + tid], zr)));
                    den = __dadd_rn(den, __dmul_rn(w, __dmul_rn(zr, zr)));
                }
                if (den > 0.0) M.c[tid] = __double2float_rn(__ddiv_rn(num, den));
            }
            __syncthreads();
        }
        // the final codes for the fitted scales; the packed page
        uint8_t *page = pages + (size_t)p * F.page_bytes;
        if (F.col_scales) {
            M.ic[tid] = __fdiv_rn(1.f, M.c[tid]);
            reinterpret_cast<float *>(page + F.c_off)[tid] = M.c[tid];
        }
        if (my_int) {
            fit_codes_row(M, tid, my_qmax);
            reinterpret_cast<float *>(page + F.r_off)[F.blk_rbase(my_blk) + (tid & 15)] = M.r[tid];
        }
        __syncthreads();
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const int blk = 2 * warp + half, s0 = 16 * blk;
            uint8_t *dst = page + F.blk_off(blk);
            if (F.blk_kind(blk) == kKindFp16) {
                // binary16 of S / c, as the quantizer stores FP16 rows
                uint32_t wd[32];
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    const float *Sr = M.S + M.kap[s0 + r] * kFitStride + 4 * lane;
                    const float *ic = M.ic + 4 * lane;
                    __half2 h01 = __floats2half2_rn(__fmul_rn(Sr[0], ic[0]), __fmul_rn(Sr[1], ic[1]));
                    __half2 h23 = __floats2half2_rn(__fmul_rn(Sr[2], ic[2]), __fmul_rn(Sr[3], ic[3]));
                    wd[2 * r] = *reinterpret_cast<uint32_t *>(&h01);
                    wd[2 * r + 1] = *reinterpret_cast<uint32_t *>(&h23);
                }
                pack_fp16_block(dst, lane, wd);
                continue;
            }
            switch (F.blk_bits(blk)) {
                case 8: fit_pack_int<8>(M, dst, s0, lane); break;
                case 7: fit_pack_int<7>(M, dst, s0, lane); break;
                case 6: fit_pack_int<6>(M, dst, s0, lane); break;
                case 5: fit_pack_int<5>(M, dst, s0, lane); break;
                case 4: fit_pack_int<4>(M, dst, s0, lane); break;
                case 3: fit_pack_int<3>(M, dst, s0, lane); break;
                default: fit_pack_int<2>(M, dst, s0, lane); break;
            }
        }
    }
}

cudaError_t launch_fit(const stq_state *s, const float *S, const float *impact, int iters, cudaStream_t stream) {
    if (iters == 0) return launch_quantize(s, S, stream);
    const long n = (long)s->batch * s->heads;
    const size_t smem = sizeof(FitSmem);
    cudaError_t err = cudaFuncSetAttribute((const void *)fit_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem);
    if (err != cudaSuccess) return err;
    const int grid = persistent_grid((const void *)fit_kernel, kThreads, smem, n);
    if (grid <= 0) return cudaErrorInvalidConfiguration;
    fit_kernel<<<grid, kThreads, smem, stream>>>(s->dev, S, impact, s->base + s->perm_offset,
                                                  s->base + s->pages_offset, n, s->heads, iters);
    return cudaGetLastError();
}

}  // namespace stq
