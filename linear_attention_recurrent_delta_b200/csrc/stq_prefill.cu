// stq_prefill.cu -- prefill: a prompt of L tokens through every page (sm_100a).
//
// The step before decode that builds the state from a prompt ("repeated
// prefill" on the DASC card page): each page's state runs through L decode
// steps in fp32 and is requantized once, after the last token.  One
// persistent CTA of 128 threads walks pages p = blockIdx.x + i*gridDim.x
// with the decode kernel's mapping (warp w: slice w of every 16-row block,
// lane l: columns 4l .. 4l+3) and keeps the page's state T in registers for
// the whole prompt:
//   token 0   T = z (alpha r)          (the page, decayed as the decode step)
//   token l   T = RN(alpha T)          (the fp32 state decayed in place)
//   each      u = T^T k (canonical column sums), e = v (1/c) - u,
//             T = fma(beta k, e, T), o = c T^T q
// then the decode step's row scales and requantization (RTN or pcg4d SR
// with `step`), in place in the page's buffer, and one bulk store.
// Pages are double-buffered in shared memory; each token's q, k, v (and KDA
// gate) rows stream through a ring of token stages, all by cp.async.bulk (no
// multicast) counted on mbarriers with bounded waits.  One CTA barrier per
// token (the cross-warp sum of u); o of a token is finished after the next
// token's barrier.
#include "stq_rows.cuh"

namespace stq {

constexpr int kTokenStages = 4;

struct PrefillArgs {
    uint8_t *pages;
    const uint8_t *perm;
    uint32_t *status;
    const float *q, *k, *v, *alpha, *beta;   // [L][pages][128] (scalar alpha, beta: [L][pages])
    float *o;                                // [L][pages][128]
    float *S_out;                            // optional [pages][128][128], natural key order
    int L, n_pages, heads;
    uint32_t tok_bytes;                      // bytes a token stage receives
    uint32_t tok_stride;                     // token stage stride (a multiple of 128)
    uint32_t page_stride;                    // page buffer stride (a multiple of 128)
    uint32_t store_bytes;                    // codes + r
    uint32_t seed_lo, seed_hi, step;
    uint64_t wait_limit_ns;
    int stall_first_wait;
};

struct PrefillSmem {
    // per warp, its 32 rows in slice order (row 4b + i = block b, row i):
    float a[kWarps][kRowsPerWarp];           // decay (token 0: alpha r)
    float kp[kWarps][kRowsPerWarp];          // k of the row's key channel
    float bk[kWarps][kRowsPerWarp];          // beta k
    float qp[kWarps][kRowsPerWarp];          // q
    float inv[kWarps][kRowsPerWarp];         // row maxima, then requant multipliers
    float red_u[2][kWarps][kD];              // per token parity and warp: chain sums of u
    float red_o[2][kWarps][kD];              // the same for o
    float beta_t[kD];                        // beta of the page's tokens 128 m .. 128 m + 127
    float alpha_t[kD];                       // the scalar gate of the same tokens (GDN)
    float ic[kD];                            // the page's 1 / c
    float cpg[kD];                           // the page's c
    uint64_t pfull[2];                       // page buffers
    uint64_t tfull[kTokenStages];            // token stages
    uint64_t never;                          // a barrier nothing completes (test hook)
    int g_next;                              // thread 0: tokens 0 .. g_next - 1 of the stream are loaded
    int last_item[2];                        // thread 0: the last page item loaded into each buffer
};

constexpr size_t kPrefillFixedBytes = (sizeof(PrefillSmem) + 127) / 128 * 128;

__device__ __forceinline__ void issue_page(const DevFormat &F, const PrefillArgs &A, uint8_t *dst, int p,
                                           uint64_t *bar) {
    mbar_expect_tx(bar, (uint32_t)F.page_bytes);
    bulk_g2s(dst, A.pages + (size_t)p * F.page_bytes, (uint32_t)F.page_bytes, bar);
}

// Token g of this CTA's stream: page item g / L, token g % L.
__device__ __forceinline__ void issue_token(const DevFormat &F, const PrefillArgs &A, uint8_t *dst, int g,
                                            uint64_t *bar) {
    const int item = g / A.L, l = g % A.L;
    const int p = (int)blockIdx.x + item * (int)gridDim.x;
    const size_t row = ((size_t)l * A.n_pages + p) * kD;
    mbar_expect_tx(bar, A.tok_bytes);
    bulk_g2s(dst, A.q + row, 512, bar);
    bulk_g2s(dst + 512, A.k + row, 512, bar);
    bulk_g2s(dst + 1024, A.v + row, 512, bar);
    if (F.gate_vector) bulk_g2s(dst + 1536, A.alpha + row, 512, bar);
}

// Is token g of this CTA's stream a real one (its page exists)?
__device__ __forceinline__ bool token_exists(const PrefillArgs &A, int g) {
    return (long)blockIdx.x + (long)(g / A.L) * (long)gridDim.x < (long)A.n_pages;
}

// o of token l of page p: the tree over the warps' chain sums, times c.
__device__ __forceinline__ void prefill_write_o(const float (*red_o)[kD], const PrefillArgs &A, int l, int p,
                                                int lane, const float *cpg, bool col_scales) {
    const float4 o0 = *reinterpret_cast<const float4 *>(&red_o[0][4 * lane]);
    const float4 o1 = *reinterpret_cast<const float4 *>(&red_o[1][4 * lane]);
    const float4 o2 = *reinterpret_cast<const float4 *>(&red_o[2][4 * lane]);
    const float4 o3 = *reinterpret_cast<const float4 *>(&red_o[3][4 * lane]);
    float2 oa = __fadd2_rn(__fadd2_rn(make_float2(o0.x, o0.y), make_float2(o1.x, o1.y)),
                           __fadd2_rn(make_float2(o2.x, o2.y), make_float2(o3.x, o3.y)));
    float2 ob = __fadd2_rn(__fadd2_rn(make_float2(o0.z, o0.w), make_float2(o1.z, o1.w)),
                           __fadd2_rn(make_float2(o2.z, o2.w), make_float2(o3.z, o3.w)));
    if (col_scales) {
        const float4 c = *reinterpret_cast<const float4 *>(cpg + 4 * lane);
        oa = __fmul2_rn(make_float2(c.x, c.y), oa);
        ob = __fmul2_rn(make_float2(c.z, c.w), ob);
    }
    *reinterpret_cast<float4 *>(A.o + ((size_t)l * A.n_pages + p) * kD + 4 * lane) = make_float4(oa.x, oa.y, ob.x, ob.y);
}

template <class FMT>
__global__ void __launch_bounds__(kThreads, 3) prefill_kernel(const DevFormat F, const PrefillArgs A) {
    extern __shared__ __align__(128) uint8_t smem[];
    PrefillSmem &S = *reinterpret_cast<PrefillSmem *>(smem);
    uint8_t *pbufs = smem + kPrefillFixedBytes;
    uint8_t *tstages = pbufs + 2 * A.page_stride;
    constexpr bool SR = FMT::kSr;
    bool col_scales, gate_vector;
    format_flags<FMT>(F, col_scales, gate_vector);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int L = A.L, n = A.n_pages, stride = (int)gridDim.x, H = A.heads;
    if (tid == 0) {
        mbar_init(&S.pfull[0], 1);
        mbar_init(&S.pfull[1], 1);
        for (int st = 0; st < kTokenStages; ++st) mbar_init(&S.tfull[st], 1);
        mbar_init(&S.never, 1);
        fence_mbar_init();
    }
    __syncthreads();
    asm volatile("griddepcontrol.wait;" ::: "memory");   // see the decode kernel
    if (tid == 0) {
        S.last_item[0] = S.last_item[1] = -1;
        S.g_next = 0;
        for (int i = 0; i < 2; ++i) {
            const int p = (int)blockIdx.x + i * stride;
            if (p < n) {
                issue_page(F, A, pbufs + i * A.page_stride, p, &S.pfull[i]);
                S.last_item[i] = i;
            }
        }
        for (int g = 0; g < kTokenStages && token_exists(A, g); ++g) {
            issue_token(F, A, tstages + g * A.tok_stride, g, &S.tfull[g]);
            S.g_next = g + 1;
        }
    }
    const RowCtx R = row_ctx<FMT>(F, warp, lane);
    const int sb = stride / H, sh = stride % H;
    int p = (int)blockIdx.x;
    int pb = p / H, ph = p % H;
    int g = 0;           // this CTA's token index
    bool failed = false;

    for (int item = 0; p < n; ++item) {
        uint8_t *pbuf = pbufs + (item & 1) * A.page_stride;
        const bool okp = mbar_wait_bounded(&S.pfull[item & 1], (uint32_t)((item >> 1) & 1), A.wait_limit_ns);
        const int kap = __ldg(A.perm + ph * kD + R.s) & (kD - 1);
        float *r_s = reinterpret_cast<float *>(pbuf + F.r_off);
        const float r_me = (R.all_int || R.is_int) ? r_s[R.rix] : 1.f;
        if (col_scales) {   // thread t keeps and inverts the scale of column t
            const float c = reinterpret_cast<const float *>(pbuf + F.c_off)[tid];
            S.cpg[tid] = c;
            S.ic[tid] = __frcp_rn(c);
        }
        Tile T;
        for (int l = 0; l < L; ++l) {
            if ((l & (kD - 1)) == 0) {
                // beta (and a scalar gate) of the next 128 tokens of the page,
                // thread t: token l + t
                __syncthreads();   // every warp is done with the previous ones
                if (l + tid < L) {
                    const size_t si = (size_t)(l + tid) * n + p;
                    S.beta_t[tid] = __ldg(A.beta + si);
                    if (!gate_vector) S.alpha_t[tid] = __ldg(A.alpha + si);
                }
                __syncthreads();
            }
            const bool first = l == 0;   // token 0 dequantizes the page, later ones decay T
            const int st = g & (kTokenStages - 1);
            const int par = g & 1;
            bool ok;
            if (A.stall_first_wait && g == 0) ok = mbar_wait_bounded(&S.never, 0, A.wait_limit_ns);
            else ok = mbar_wait_bounded(&S.tfull[st], (uint32_t)((g / kTokenStages) & 1), A.wait_limit_ns);
            if (first) ok = ok && okp;
            const float *q_s = reinterpret_cast<const float *>(tstages + st * A.tok_stride);
            const float *k_s = q_s + kD;
            const float *v_s = q_s + 2 * kD;
            const float *al_s = q_s + 3 * kD;
            const float beta = S.beta_t[l & (kD - 1)];
            {
                const float al = gate_vector ? al_s[kap] : S.alpha_t[l & (kD - 1)];
                const float kk = k_s[kap];
                S.a[warp][lane] = (first && (R.all_int || R.is_int)) ? __fmul_rn(al, r_me) : al;
                S.kp[warp][lane] = kk;
                S.qp[warp][lane] = q_s[kap];
                S.bk[warp][lane] = __fmul_rn(beta, kk);
            }
            __syncwarp();   // the warp's rows' operands come from its own lanes

            // decay (token 0: dequantize the page) and u's chains
            float2 cu[2][2];
#pragma unroll
            for (int h = 0; h < 2; ++h) cu[h][0] = cu[h][1] = make_float2(0.f, 0.f);
            static_for<0, kBlocks>([&](auto bc) {
                constexpr int b = decltype(bc)::value;
                const float4 a4 = *reinterpret_cast<const float4 *>(&S.a[warp][4 * b]);
                if (first) {
                    const uint8_t *blk = pbuf + fmt_offset<FMT, b>(F);
                    with_width<FMT, b>(F, [&](auto wc) {
                        constexpr int W = decltype(wc)::value;
                        dequant_slice<W, b>(blk, warp, lane, a4, T);
                    });
                } else {
                    const float av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        T[b][i][0] = __fmul2_rn(make_float2(av[i], av[i]), T[b][i][0]);
                        T[b][i][1] = __fmul2_rn(make_float2(av[i], av[i]), T[b][i][1]);
                    }
                }
                const float4 k4 = *reinterpret_cast<const float4 *>(&S.kp[warp][4 * b]);
                const float kv[4] = {k4.x, k4.y, k4.z, k4.w};
                constexpr int h = b >> 2;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    cu[h][0] = __ffma2_rn(make_float2(kv[i], kv[i]), T[b][i][0], cu[h][0]);
                    cu[h][1] = __ffma2_rn(make_float2(kv[i], kv[i]), T[b][i][1], cu[h][1]);
                }
            });
            store_readout(S.red_u[par][warp], lane, cu);
            const float4 v4 = *reinterpret_cast<const float4 *>(v_s + 4 * lane);
            if (__syncthreads_or(!ok)) {
                failed = true;
                break;
            }
            if (tid == 0 && g >= 1) {
                // every warp is done with the previous token's stage: refill it
                const int gr = g - 1 + kTokenStages;
                if (token_exists(A, gr)) {
                    fence_proxy_async_smem();
                    const int sr = gr & (kTokenStages - 1);
                    issue_token(F, A, tstages + sr * A.tok_stride, gr, &S.tfull[sr]);
                    S.g_next = gr + 1;
                }
            }
            if (!first && warp == kWarps - 1)
                prefill_write_o(S.red_o[par ^ 1], A, l - 1, p, lane, S.cpg, col_scales);

            // u = (W0 + W1) + (W2 + W3); e = v (1/c) - u
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
                if (col_scales) ic = *reinterpret_cast<const float4 *>(&S.ic[4 * lane]);
                e01 = make_float2(__fsub_rn(__fmul_rn(v4.x, ic.x), ua.x), __fsub_rn(__fmul_rn(v4.y, ic.y), ua.y));
                e23 = make_float2(__fsub_rn(__fmul_rn(v4.z, ic.z), ub.x), __fsub_rn(__fmul_rn(v4.w, ic.w), ub.y));
            }
            // T = T + (beta k) e; o's chains
            float2 co[2][2];
#pragma unroll
            for (int h = 0; h < 2; ++h) co[h][0] = co[h][1] = make_float2(0.f, 0.f);
            static_for<0, kBlocks>([&](auto bc) {
                constexpr int b = decltype(bc)::value;
                const float4 b4 = *reinterpret_cast<const float4 *>(&S.bk[warp][4 * b]);
                const float bv[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    T[b][i][0] = __ffma2_rn(make_float2(bv[i], bv[i]), e01, T[b][i][0]);
                    T[b][i][1] = __ffma2_rn(make_float2(bv[i], bv[i]), e23, T[b][i][1]);
                }
                readout_block<b>(S.qp[warp], T, co[b >> 2]);
            });
            store_readout(S.red_o[par][warp], lane, co);
            __syncwarp();   // every lane is done with the warp's operands
            ++g;
        }
        if (failed) break;

        // the page's end: o of its last token, the state (optional), the one
        // requantization in the page's buffer and its store
        __syncthreads();
        if (warp == kWarps - 1) prefill_write_o(S.red_o[(g - 1) & 1], A, L - 1, p, lane, S.cpg, col_scales);
        if (A.S_out) {
            // S = T c in natural key order: row (b, i) holds the key channel of lane 4b + i
            float4 c4 = make_float4(1.f, 1.f, 1.f, 1.f);
            if (col_scales) c4 = *reinterpret_cast<const float4 *>(&S.cpg[4 * lane]);
            static_for<0, kBlocks>([&](auto bc) {
                constexpr int b = decltype(bc)::value;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int kr = __shfl_sync(0xffffffffu, kap, 4 * b + i);
                    const float2 x = __fmul2_rn(T[b][i][0], make_float2(c4.x, c4.y));
                    const float2 y = __fmul2_rn(T[b][i][1], make_float2(c4.z, c4.w));
                    *reinterpret_cast<float4 *>(A.S_out + ((size_t)p * kD + kr) * kD + 4 * lane) =
                        make_float4(x.x, x.y, y.x, y.y);
                }
            });
        }
        static_for<0, kBlocks>([&](auto bc) {
            constexpr int b = decltype(bc)::value;
#pragma unroll
            for (int i = 0; i < 4; ++i) S.inv[warp][4 * b + i] = warp_absmax(absmax4(T[b][i][0], T[b][i][1]));
        });
        __syncwarp();
        {
            // lane l finishes row l of the slice: r' = m / qmax, inv = qmax / m (toward zero)
            const float m = S.inv[warp][lane];
            float inv = 0.f;
            if (R.all_int || R.is_int) {
                const float r = div_by_qmax(m, R.qmax, R.rcp_qmax);
                inv = m > 0.f ? div_rz_qmax<(FMT::kTune & kFastRcp) != 0>(R.qmax, m) : 0.f;
                r_s[R.rix] = r;
            }
            S.inv[warp][lane] = inv;
        }
        __syncwarp();
        SrCtx sr;
        sr.k0 = A.seed_lo; sr.k1 = A.seed_hi; sr.step = A.step;
        sr.b = (uint32_t)pb;
        sr.h = (uint32_t)ph;
        if constexpr (SR) sr.fix();
        static_for<0, kBlocks>([&](auto bc) {
            constexpr int b = decltype(bc)::value;
            const float4 i4 = *reinterpret_cast<const float4 *>(&S.inv[warp][4 * b]);
            uint8_t *blk = pbuf + fmt_offset<FMT, b>(F);
            with_width<FMT, b>(F, [&](auto wc) {
                constexpr int W = decltype(wc)::value;
                requant_slice<W, b, SR>(blk, warp, lane, i4, T, sr);
            });
        });
        fence_proxy_async_smem();   // the buffer's new bytes are read by the bulk store
        __syncthreads();
        if (tid == 0) {
            bulk_s2g(A.pages + (size_t)p * F.page_bytes, pbuf, A.store_bytes);
            bulk_commit();
            const int p2 = p + 2 * stride;
            if (p2 < n) {
                // the buffer takes the page two items ahead once the store has read it
                bulk_wait_read<0>();
                fence_proxy_async_smem();
                issue_page(F, A, pbuf, p2, &S.pfull[item & 1]);
                S.last_item[item & 1] = item + 2;
            }
        }
        p += stride;
        pb += sb;
        ph += sh;
        if (ph >= H) { ph -= H; ++pb; }
    }
    asm volatile("griddepcontrol.launch_dependents;");
    __syncthreads();
    if (tid == 0) {
        if (failed) {
            // record it; the loads in flight land before the CTA exits
            atomicOr(A.status, kStatusTimeout);
            for (int j = g; j < S.g_next; ++j)
                mbar_wait_bounded(&S.tfull[j & (kTokenStages - 1)], (uint32_t)((j / kTokenStages) & 1),
                                  A.wait_limit_ns);
            for (int i = 0; i < 2; ++i)
                if (S.last_item[i] >= 0)
                    mbar_wait_bounded(&S.pfull[i], (uint32_t)((S.last_item[i] >> 1) & 1), A.wait_limit_ns);
        }
        bulk_wait<0>();
    }
}

template <class FMT>
static cudaError_t launch_prefill_with(const DevFormat &F, const PrefillArgs &A, bool early_launch,
                                       cudaStream_t stream) {
    const size_t smem = kPrefillFixedBytes + 2 * (size_t)A.page_stride + kTokenStages * (size_t)A.tok_stride;
    const void *fn = (const void *)prefill_kernel<FMT>;
    cudaError_t err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    const int grid = persistent_grid(fn, kThreads, smem, A.n_pages);
    if (grid <= 0) return cudaErrorInvalidConfiguration;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = early_launch ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, prefill_kernel<FMT>, F, A);
}

cudaError_t launch_prefill(const stq_state *s, int L, const float *q, const float *k, const float *v,
                           const float *alpha, const float *beta, float *o, float *S_out, uint64_t seed,
                           uint32_t step, int stall_first_wait, bool early_launch, cudaStream_t stream) {
    const DevFormat &F = s->dev;
    PrefillArgs A;
    A.pages = s->base + s->pages_offset;
    A.perm = s->base + s->perm_offset;
    A.status = reinterpret_cast<uint32_t *>(s->base + s->status_offset);
    A.q = q; A.k = k; A.v = v; A.alpha = alpha; A.beta = beta; A.o = o; A.S_out = S_out;
    A.L = L;
    A.n_pages = s->batch * s->heads;
    A.heads = s->heads;
    A.tok_bytes = 1536u + (F.gate_vector ? 512u : 0u);
    A.tok_stride = (A.tok_bytes + 127u) / 128u * 128u;
    A.page_stride = ((uint32_t)F.page_bytes + 127u) / 128u * 128u;
    A.store_bytes = (uint32_t)(F.col_scales ? F.c_off : F.page_bytes);
    A.seed_lo = (uint32_t)seed;
    A.seed_hi = (uint32_t)(seed >> 32);
    A.step = step;
    A.wait_limit_ns = s->wait_limit_ns;
    A.stall_first_wait = stall_first_wait;
    if (format_is<FmtStepQuant6>(F)) return launch_prefill_with<FmtStepQuant6>(F, A, early_launch, stream);
    if (format_is<FmtInt8Row>(F)) return launch_prefill_with<FmtInt8Row>(F, A, early_launch, stream);
    if (format_is<FmtStepQuant4Kda>(F)) return launch_prefill_with<FmtStepQuant4Kda>(F, A, early_launch, stream);
    if (format_is<FmtDamp>(F)) return launch_prefill_with<FmtDamp>(F, A, early_launch, stream);
    if (F.stochastic) return launch_prefill_with<RuntimeFmt<true>>(F, A, early_launch, stream);
    return launch_prefill_with<RuntimeFmt<false>>(F, A, early_launch, stream);
}

}  // namespace stq
