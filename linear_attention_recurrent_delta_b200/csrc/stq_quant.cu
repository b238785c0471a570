// stq_quant.cu -- cold-path kernels: precision map (calibration), quantize,
// dequantize.  One CTA of 128 threads per page: warp w owns the 16-row blocks
// 2w and 2w+1, lane l columns 4l .. 4l+3, and the whole-block plane packers of
// stq_device.cuh write the same byte layout the decode kernel reads and writes
// slice by slice.
#include "stq_internal.h"

#include <map>
#include <mutex>

namespace stq {

constexpr int kCalibChunk = 32;   // requests summed per partial score

size_t calibrate_workspace_bytes(int batch, int heads) {
    const size_t chunks = ((size_t)batch + kCalibChunk - 1) / kCalibChunk;
    return chunks * (size_t)heads * kD * sizeof(double);
}

// Partial score of key channel kappa = tid over one chunk of requests:
// sum over b in the chunk (ascending) of sum_j S[b][h][kappa][j]^2 (ascending j),
// in double.  grid = (chunks, H).
__global__ void __launch_bounds__(kThreads) calib_partial_kernel(const float *S, int batch, int heads,
                                                                 double *ws) {
    const int c = blockIdx.x, h = blockIdx.y, kap = threadIdx.x;
    const int b0 = c * kCalibChunk, b1 = min(batch, b0 + kCalibChunk);
    double acc = 0.0;
    for (int b = b0; b < b1; ++b) {
        const float4 *row = reinterpret_cast<const float4 *>(S + (((size_t)b * heads + h) * kD + kap) * kD);
        double rs = 0.0;
#pragma unroll 8
        for (int j4 = 0; j4 < kD / 4; ++j4) {
            const float4 x = __ldg(row + j4);
            rs = __fma_rn((double)x.x, (double)x.x, rs);
            rs = __fma_rn((double)x.y, (double)x.y, rs);
            rs = __fma_rn((double)x.z, (double)x.z, rs);
            rs = __fma_rn((double)x.w, (double)x.w, rs);
        }
        acc += rs;
    }
    ws[((size_t)c * heads + h) * kD + kap] = acc;
}

struct GroupEnds {
    int n;
    int end[STQ_MAX_GROUPS];   // cumulative row counts
};

// Ranks key channels of head h = blockIdx.x and writes the precision map.
__global__ void __launch_bounds__(kThreads) calib_rank_kernel(const double *ws, int chunks, int heads,
                                                              const float *row_weight, GroupEnds G,
                                                              uint8_t *perm) {
    __shared__ double score[kD];
    __shared__ int grp[kD];
    const int h = blockIdx.x, kap = threadIdx.x;
    double acc = 0.0;
    for (int c = 0; c < chunks; ++c) acc += ws[((size_t)c * heads + h) * kD + kap];
    if (row_weight) acc *= (double)row_weight[(size_t)h * kD + kap];
    if (!(acc == acc)) acc = -1.0;   // a non-finite state still yields a permutation
    score[kap] = acc;
    __syncthreads();
    int rank = 0;
    for (int i = 0; i < kD; ++i) {
        const double si = score[i];
        rank += (si > acc) || (si == acc && i < kap);
    }
    int g = 0;
    while (g < G.n - 1 && rank >= G.end[g]) ++g;
    grp[kap] = g;
    __syncthreads();
    int pos = 0;
    for (int i = 0; i < kap; ++i) pos += (grp[i] == g);
    const int start = g ? G.end[g - 1] : 0;
    perm[(size_t)h * kD + start + pos] = (uint8_t)kap;
}

cudaError_t launch_calibrate(const stq_state *s, const float *S, const float *row_weight, double *ws,
                             cudaStream_t stream) {
    const int chunks = (s->batch + kCalibChunk - 1) / kCalibChunk;
    calib_partial_kernel<<<dim3(chunks, s->heads), kThreads, 0, stream>>>(S, s->batch, s->heads, ws);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    GroupEnds G;
    G.n = s->fmt.n_groups;
    int acc = 0;
    for (int g = 0; g < STQ_MAX_GROUPS; ++g) {
        if (g < G.n) acc += s->fmt.group_rows[g];
        G.end[g] = acc;
    }
    calib_rank_kernel<<<s->heads, kThreads, 0, stream>>>(ws, chunks, s->heads, row_weight, G,
                                                          s->base + s->perm_offset);
    return cudaGetLastError();
}

// ------------------------------------------------ calibration, no allocation --
// Scratch of stq_calibrate_noalloc: one fixed array in every GPU that loads the
// library, held until the process exits.  Every call shares it; the partial
// kernel writes each entry the rank kernel reads, so nothing in it has to
// start at zero, and two calls that overlap on the GPU would race on it.
static __device__ __align__(256) double g_calib_scratch[STQ_CALIBRATE_NOALLOC_MAX_BYTES / sizeof(double)];

// Device address of g_calib_scratch on the current device.  Host code must
// not hand the symbol itself to a kernel (on the host it names a host-side
// stand-in).  The address is looked up with the device current, on every
// call whose stream is not being captured (so a context rebuilt after a
// device reset, which loads the module again, is seen), and kept per device
// for calls made while a stream is captured, which use the address of the
// device's last uncaptured call.
static cudaError_t noalloc_scratch(cudaStream_t stream, double **out) {
    static std::mutex mu;
    static std::map<int, double *> addr;
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    err = cudaStreamIsCapturing(stream, &cs);
    if (err != cudaSuccess) return err;
    std::lock_guard<std::mutex> lock(mu);
    auto it = addr.find(dev);
    if (cs == cudaStreamCaptureStatusNone || it == addr.end()) {
        void *p = nullptr;
        err = cudaGetSymbolAddress(&p, g_calib_scratch);
        if (err != cudaSuccess) return err;
        addr[dev] = static_cast<double *>(p);
        it = addr.find(dev);
    }
    *out = it->second;
    return cudaSuccess;
}

}  // namespace stq

extern "C" stq_status stq_calibrate_noalloc(stq_state *s, const float *d_S, const float *d_row_weight,
                                            void *stream) {
    using namespace stq;
    const stq_status in = check_calibrate_input(s, d_S, d_row_weight);
    if (in != STQ_OK) return in;
    if (calibrate_workspace_bytes(s->batch, s->heads) > STQ_CALIBRATE_NOALLOC_MAX_BYTES)
        return STQ_ERR_BUFFER_TOO_SMALL;
    double *ws = nullptr;
    if (noalloc_scratch(static_cast<cudaStream_t>(stream), &ws) != cudaSuccess) return STQ_ERR_CUDA;
    return launch_calibrate(s, d_S, d_row_weight, ws, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? STQ_OK : STQ_ERR_CUDA;
}

namespace stq {

// ------------------------------------------------------------- quantize --
template <int B>
__device__ __forceinline__ void quant_int(uint8_t *blk, int lane, const float *inv,
                                          const float2 (&T)[kRowsPerWarp][2], int r0) {
    const float M = 12582912.0f + (float)(1 << (B - 1));
    const float2 M2 = make_float2(M, M);
    uint32_t ub[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) {
        const float i0 = inv[r];
        const float2 y0 = __ffma2_rn(T[r0 + r][0], make_float2(i0, i0), M2);
        const float2 y1 = __ffma2_rn(T[r0 + r][1], make_float2(i0, i0), M2);
        ub[r] = low_bytes(y0.x, y0.y, y1.x, y1.y);
    }
    pack_int_block<B>(blk, lane, ub);
}

template <int R0>
__device__ __forceinline__ void quant_block(int kind, int bits, uint8_t *blk, int lane, const float *inv,
                                            const float2 (&T)[kRowsPerWarp][2]) {
    if (kind == kKindFp16) {
        uint32_t w[32];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            __half2 h01 = __floats2half2_rn(T[R0 + r][0].x, T[R0 + r][0].y);
            __half2 h23 = __floats2half2_rn(T[R0 + r][1].x, T[R0 + r][1].y);
            w[2 * r] = *reinterpret_cast<uint32_t *>(&h01);
            w[2 * r + 1] = *reinterpret_cast<uint32_t *>(&h23);
        }
        pack_fp16_block(blk, lane, w);
        return;
    }
    switch (bits) {
        case 8: quant_int<8>(blk, lane, inv, T, R0); break;
        case 7: quant_int<7>(blk, lane, inv, T, R0); break;
        case 6: quant_int<6>(blk, lane, inv, T, R0); break;
        case 5: quant_int<5>(blk, lane, inv, T, R0); break;
        case 4: quant_int<4>(blk, lane, inv, T, R0); break;
        case 3: quant_int<3>(blk, lane, inv, T, R0); break;
        default: quant_int<2>(blk, lane, inv, T, R0); break;
    }
}

// One CTA per page (grid-stride).  S: [B][H][128][128] natural key order.
__global__ void __launch_bounds__(kThreads, 2) quantize_kernel(const DevFormat F, const float *S,
                                                               const uint8_t *perm, uint8_t *pages,
                                                               long n_pages, int heads) {
    __shared__ int kap_s[kD];
    __shared__ float4 red[kWarps][32];
    __shared__ float inv_s[kWarps][kRowsPerWarp];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (long p = blockIdx.x; p < n_pages; p += gridDim.x) {
        const int h = (int)(p % heads);
        __syncthreads();
        kap_s[tid] = perm[(size_t)h * kD + tid] & (kD - 1);   // a map byte is a channel < 128
        __syncthreads();
        const float *Sp = S + (size_t)p * kD * kD;
        float2 T[kRowsPerWarp][2];
        float4 cm = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r) {
            const float4 x = __ldg(reinterpret_cast<const float4 *>(Sp + (size_t)kap_s[32 * warp + r] * kD) + lane);
            T[r][0] = make_float2(x.x, x.y);
            T[r][1] = make_float2(x.z, x.w);
            cm = make_float4(fmaxf(cm.x, fabsf(x.x)), fmaxf(cm.y, fabsf(x.y)), fmaxf(cm.z, fabsf(x.z)),
                             fmaxf(cm.w, fabsf(x.w)));
        }
        uint8_t *page = pages + (size_t)p * F.page_bytes;
        if (F.col_scales) {
            red[warp][lane] = cm;
            __syncthreads();
            float4 c = red[0][lane];
            for (int w = 1; w < kWarps; ++w) {
                const float4 t = red[w][lane];
                c = make_float4(fmaxf(c.x, t.x), fmaxf(c.y, t.y), fmaxf(c.z, t.z), fmaxf(c.w, t.w));
            }
            c.x = c.x > 0.f ? c.x : 1.f;
            c.y = c.y > 0.f ? c.y : 1.f;
            c.z = c.z > 0.f ? c.z : 1.f;
            c.w = c.w > 0.f ? c.w : 1.f;
            const float2 ic01 = make_float2(__fdiv_rn(1.f, c.x), __fdiv_rn(1.f, c.y));
            const float2 ic23 = make_float2(__fdiv_rn(1.f, c.z), __fdiv_rn(1.f, c.w));
#pragma unroll
            for (int r = 0; r < kRowsPerWarp; ++r) {
                T[r][0] = __fmul2_rn(T[r][0], ic01);
                T[r][1] = __fmul2_rn(T[r][1], ic23);
            }
            if (warp == 0) *reinterpret_cast<float4 *>(page + F.c_off + 16 * lane) = c;
        }
        float rm[kRowsPerWarp];
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r)
            rm[r] = fmaxf(fmaxf(fabsf(T[r][0].x), fabsf(T[r][0].y)), fmaxf(fabsf(T[r][1].x), fabsf(T[r][1].y)));
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
            inv_s[warp][lane] = inv;
        }
        __syncwarp();
        const int b0 = 2 * warp, b1 = 2 * warp + 1;
        quant_block<0>(F.blk_kind(b0), F.blk_bits(b0), page + F.blk_off(b0), lane, &inv_s[warp][0], T);
        quant_block<16>(F.blk_kind(b1), F.blk_bits(b1), page + F.blk_off(b1), lane, &inv_s[warp][16], T);
    }
}

cudaError_t launch_quantize(const stq_state *s, const float *S, cudaStream_t stream) {
    const long n = (long)s->batch * s->heads;
    const int grid = persistent_grid((const void *)quantize_kernel, kThreads, 0, n);
    if (grid <= 0) return cudaErrorInvalidConfiguration;
    quantize_kernel<<<grid, kThreads, 0, stream>>>(s->dev, S, s->base + s->perm_offset,
                                                   s->base + s->pages_offset, n, s->heads);
    return cudaGetLastError();
}

// ----------------------------------------------------------- dequantize --
template <int B>
__device__ __forceinline__ void dequant_rows_int(const uint8_t *blk, int lane, const float *rs,
                                                 float2 (&X)[16][2]) {
    uint32_t ub[16];
    unpack_int_block<B>(blk, lane, ub);
    const float bm = 8388608.0f + (float)(1 << (B - 1));
#pragma unroll
    for (int r = 0; r < 16; ++r) {
        float2 z01, z23;
        codes_to_float(ub[r], bm, z01, z23);
        X[r][0] = __fmul2_rn(z01, make_float2(rs[r], rs[r]));
        X[r][1] = __fmul2_rn(z23, make_float2(rs[r], rs[r]));
    }
}

__global__ void __launch_bounds__(kThreads) dequantize_kernel(const DevFormat F, const uint8_t *perm,
                                                              const uint8_t *pages, float *S, long n_pages,
                                                              int heads) {
    __shared__ int kap_s[kD];
    __shared__ float r_s[kD];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (long p = blockIdx.x; p < n_pages; p += gridDim.x) {
        const int h = (int)(p % heads);
        const uint8_t *page = pages + (size_t)p * F.page_bytes;
        __syncthreads();
        kap_s[tid] = perm[(size_t)h * kD + tid] & (kD - 1);   // a map byte is a channel < 128
        {
            const int blk = tid >> 4;
            r_s[tid] = F.blk_kind(blk) == kKindInt
                           ? reinterpret_cast<const float *>(page + F.r_off)[F.blk_rbase(blk) + (tid & 15)]
                           : 1.f;
        }
        __syncthreads();
        float4 c = make_float4(1.f, 1.f, 1.f, 1.f);
        if (F.col_scales) c = *reinterpret_cast<const float4 *>(page + F.c_off + 16 * lane);
        float *Sp = S + (size_t)p * kD * kD;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const int blk = 2 * warp + half;
            const int s0 = 16 * blk;
            float2 X[16][2];
            const uint8_t *src = page + F.blk_off(blk);
            if (F.blk_kind(blk) == kKindFp16) {
                uint32_t w[32];
                unpack_fp16_block(src, lane, w);
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    X[r][0] = __half22float2(*reinterpret_cast<const __half2 *>(&w[2 * r]));
                    X[r][1] = __half22float2(*reinterpret_cast<const __half2 *>(&w[2 * r + 1]));
                }
            } else {
                switch (F.blk_bits(blk)) {
                    case 8: dequant_rows_int<8>(src, lane, &r_s[s0], X); break;
                    case 7: dequant_rows_int<7>(src, lane, &r_s[s0], X); break;
                    case 6: dequant_rows_int<6>(src, lane, &r_s[s0], X); break;
                    case 5: dequant_rows_int<5>(src, lane, &r_s[s0], X); break;
                    case 4: dequant_rows_int<4>(src, lane, &r_s[s0], X); break;
                    case 3: dequant_rows_int<3>(src, lane, &r_s[s0], X); break;
                    default: dequant_rows_int<2>(src, lane, &r_s[s0], X); break;
                }
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                float2 a = X[r][0], b = X[r][1];
                if (F.col_scales) {
                    a = __fmul2_rn(a, make_float2(c.x, c.y));
                    b = __fmul2_rn(b, make_float2(c.z, c.w));
                }
                *reinterpret_cast<float4 *>(Sp + (size_t)kap_s[s0 + r] * kD + 4 * lane) = make_float4(a.x, a.y, b.x, b.y);
            }
        }
    }
}

cudaError_t launch_dequantize(const stq_state *s, float *S, cudaStream_t stream) {
    const long n = (long)s->batch * s->heads;
    const int grid = persistent_grid((const void *)dequantize_kernel, kThreads, 0, n);
    if (grid <= 0) return cudaErrorInvalidConfiguration;
    dequantize_kernel<<<grid, kThreads, 0, stream>>>(s->dev, s->base + s->perm_offset, s->base + s->pages_offset,
                                                     S, n, s->heads);
    return cudaGetLastError();
}

}  // namespace stq
