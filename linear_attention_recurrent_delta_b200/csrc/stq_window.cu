// stq_window.cu -- the per-window decode kernels (sm_100a).
//
// Per-window quantization (LeapQuant abstract, paper-cards page): within a
// window of W steps the packed page stays fixed; step t (0-based) of a window
// reads the page together with a per-page fp32 buffer of the window's earlier
// updates, and only the window's committing step writes the page, requantized
// once.  Buffer of page p (buf + p * stride, stride = 512 (1 + 2W) bytes):
//   P[128]     cumulative decay per key channel (natural order); not read at t = 0
//   K[W][128]  entry tau's key, decayed to the current step (natural order)
//   D[W][128]  entry tau's delta beta_tau e_tau, column-normalised units
// Step t, with T0 = z r the fixed page (FP16 rows: h; stored order, the row
// of stored index s holding key channel perm[s]):
//   P' = P alpha;   K[tau] <- RN(K[tau] alpha)                  (tau < t)
//   u = T0^T RN(P' k) + sum_{tau<t} (K[tau] . k) D[tau]
//   D[t] = RN(beta (v (1/c) - u));   K[t] = k
//   o = c (T0^T RN(P' q) + sum_{tau<=t} (K[tau] . q) D[tau])
// The column sums over T0 are the decode kernel's (same slices, chains and
// tree); both run in one pass over the page, since the page does not change
// within a window.  A buffer dot product is a 4-channel fma chain per lane
// (lane l: channels 4l .. 4l+3) and an xor butterfly over the warp; buffer
// terms are added by fma in entry order.  A committing step then rebuilds
// T = RN(P' T0), T <- fma(K[tau], D[tau], T) for tau = 0 .. t, in registers,
// and requantizes it exactly as the decode step requantizes T'; it writes
// nothing to the buffer (a window's first step reads none of it).
//
// Staging is the decode kernel's: one thread copies the page, the input rows
// and the buffer rows a step reads into a shared-memory ring with
// cp.async.bulk (no multicast), counted on an mbarrier with a bounded wait.
#include "stq_slices.cuh"

namespace stq {

constexpr int kWindowMax = STQ_WINDOW_MAX;
constexpr int kWindowStages = 4;          // ring depth at most

struct WindowArgs {
    uint8_t *pages;
    const uint8_t *perm;
    uint32_t *status;
    const float *q, *k, *v, *alpha, *beta;
    float *o;
    uint8_t *buf;                 // window buffer, stride bytes per page
    uint32_t stride;
    int t;                        // position of this step in its window
    int n_pages, heads, n_stages;
    uint32_t stage_bytes;         // ring stride (a multiple of 128)
    uint32_t tx_bytes;            // bytes a stage receives
    uint32_t store_bytes;         // codes + r: the part of a page a commit rewrites
    uint32_t p_off, k_off, d_off; // buffer rows inside a stage
    uint32_t buf_d_off;           // D inside a page's buffer: 512 (1 + W)
    uint32_t kd_bytes;            // per-warp key table of a commit (0 otherwise)
    uint32_t seed_lo, seed_hi, step;
    uint64_t wait_limit_ns;
};

struct WindowSmem {
    // per warp, its 32 rows in slice order (row 4b + i = block b, row i):
    float rw[kWarps][kRowsPerWarp];         // r (FP16 rows: 1)
    float kp[kWarps][kRowsPerWarp];         // RN(P' k) of the row's key channel
    float qp[kWarps][kRowsPerWarp];         // RN(P' q)
    float pk[kWarps][kRowsPerWarp];         // P' (commit)
    float inv[kWarps][kRowsPerWarp];        // commit: row maxima, then requant multipliers
    float red_u[2][kWarps][kD];             // per page parity and warp: chain sums of u
    float red_o[2][kWarps][kD];             // the same for o
    float da[2][kWindowMax];                // per page parity: K[tau] . k
    float dq[2][kWindowMax];                // K[tau] . q
    uint64_t full[kWindowStages];           // stage-full barriers
};

constexpr size_t kWindowFixedBytes = (sizeof(WindowSmem) + 127) / 128 * 128;

// Stage layout: page, q, k, v (, alpha), then (t > 0) P, K[0 .. t-1], D[0 .. t-1].
__device__ __forceinline__ void issue_window_stage(const DevFormat &F, const WindowArgs &A, uint8_t *dst, int p,
                                                   uint64_t *bar) {
    mbar_expect_tx(bar, A.tx_bytes);
    bulk_g2s(dst, A.pages + (size_t)p * F.page_bytes, (uint32_t)F.page_bytes, bar);
    uint8_t *rows = dst + F.page_bytes;
    bulk_g2s(rows, A.q + (size_t)p * kD, 512, bar);
    bulk_g2s(rows + 512, A.k + (size_t)p * kD, 512, bar);
    bulk_g2s(rows + 1024, A.v + (size_t)p * kD, 512, bar);
    if (F.gate_vector) bulk_g2s(rows + 1536, A.alpha + (size_t)p * kD, 512, bar);
    if (A.t > 0) {
        const uint8_t *b = A.buf + (size_t)p * A.stride;
        const uint32_t rows_t = (uint32_t)A.t * 512u;
        bulk_g2s(dst + A.p_off, b, 512, bar);
        bulk_g2s(dst + A.k_off, b + 512, rows_t, bar);
        bulk_g2s(dst + A.d_off, b + A.buf_d_off, rows_t, bar);
    }
}

// x . y over the 128 channels: this lane's chain over channels 4l .. 4l+3
// from +0, then an xor butterfly (the sum is the same in every lane)
__device__ __forceinline__ float lane_dot(float4 x, float4 y) {
    float acc = __fmaf_rn(x.x, y.x, 0.f);
    acc = __fmaf_rn(x.y, y.y, acc);
    acc = __fmaf_rn(x.z, y.z, acc);
    acc = __fmaf_rn(x.w, y.w, acc);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, off));
    return acc;
}

__device__ __forceinline__ float4 mul4(float4 a, float4 b) {
    return make_float4(__fmul_rn(a.x, b.x), __fmul_rn(a.y, b.y), __fmul_rn(a.z, b.z), __fmul_rn(a.w, b.w));
}

// the warps' four chain sums of one page: (W0 + W1) + (W2 + W3), columns 4l .. 4l+3
__device__ __forceinline__ float4 tree4(const float (*red)[kD], int lane) {
    const float4 x0 = *reinterpret_cast<const float4 *>(&red[0][4 * lane]);
    const float4 x1 = *reinterpret_cast<const float4 *>(&red[1][4 * lane]);
    const float4 x2 = *reinterpret_cast<const float4 *>(&red[2][4 * lane]);
    const float4 x3 = *reinterpret_cast<const float4 *>(&red[3][4 * lane]);
    const float2 a = __fadd2_rn(__fadd2_rn(make_float2(x0.x, x0.y), make_float2(x1.x, x1.y)),
                                __fadd2_rn(make_float2(x2.x, x2.y), make_float2(x3.x, x3.y)));
    const float2 b = __fadd2_rn(__fadd2_rn(make_float2(x0.z, x0.w), make_float2(x1.z, x1.w)),
                                __fadd2_rn(make_float2(x2.z, x2.w), make_float2(x3.z, x3.w)));
    return make_float4(a.x, a.y, b.x, b.y);
}

__device__ __forceinline__ float4 fma4(float s, float4 d, float4 acc) {
    return make_float4(__fmaf_rn(s, d.x, acc.x), __fmaf_rn(s, d.y, acc.y), __fmaf_rn(s, d.z, acc.z),
                       __fmaf_rn(s, d.w, acc.w));
}

// This step's delta for columns 4l .. 4l+3: u from the tree and the earlier
// entries, e = v (1/c) - u (two roundings), D[t] = RN(beta e).
__device__ __forceinline__ float4 window_delta(const WindowSmem &S, int par, const float *v_s, const float *d_s,
                                               const float *c_s, int t, float beta, int lane) {
    float4 u = tree4(S.red_u[par], lane);
    for (int tau = 0; tau < t; ++tau)
        u = fma4(S.da[par][tau], *reinterpret_cast<const float4 *>(d_s + tau * kD + 4 * lane), u);
    float4 ic = make_float4(1.f, 1.f, 1.f, 1.f);
    if (c_s) {
        const float4 c = *reinterpret_cast<const float4 *>(c_s + 4 * lane);
        ic = make_float4(__frcp_rn(c.x), __frcp_rn(c.y), __frcp_rn(c.z), __frcp_rn(c.w));
    }
    const float4 v = *reinterpret_cast<const float4 *>(v_s + 4 * lane);
    const float4 e = make_float4(__fsub_rn(__fmul_rn(v.x, ic.x), u.x), __fsub_rn(__fmul_rn(v.y, ic.y), u.y),
                                 __fsub_rn(__fmul_rn(v.z, ic.z), u.z), __fsub_rn(__fmul_rn(v.w, ic.w), u.w));
    return make_float4(__fmul_rn(beta, e.x), __fmul_rn(beta, e.y), __fmul_rn(beta, e.z), __fmul_rn(beta, e.w));
}

// o of a page for columns 4l .. 4l+3: the tree, every entry's term, times c
__device__ __forceinline__ void window_out(const WindowSmem &S, int par, const float *d_s, const float *c_s,
                                           int t, float4 dt, float *o, int lane) {
    float4 ot = tree4(S.red_o[par], lane);
    for (int tau = 0; tau < t; ++tau)
        ot = fma4(S.dq[par][tau], *reinterpret_cast<const float4 *>(d_s + tau * kD + 4 * lane), ot);
    ot = fma4(S.dq[par][t], dt, ot);
    if (c_s) ot = mul4(*reinterpret_cast<const float4 *>(c_s + 4 * lane), ot);
    *reinterpret_cast<float4 *>(o + 4 * lane) = ot;
}

// Resident CTAs per SM the register budget is sized for: a step that does
// not commit keeps no tile of the state in registers (4); a committing step
// keeps T as the decode step does (2).
template <bool COMMIT>
constexpr int window_ctas_per_sm() { return COMMIT ? 2 : 4; }

// The per-page loop (same persistent walk and page -> (request, head) carry
// as the decode kernel).  One CTA barrier per page, after the column sums;
// everything of a page that needs the warps' sums happens after it.
template <class FMT, bool COMMIT>
__global__ void __launch_bounds__(kThreads, window_ctas_per_sm<COMMIT>())
window_kernel(const DevFormat F, const WindowArgs A) {
    extern __shared__ __align__(128) uint8_t smem[];
    WindowSmem &S = *reinterpret_cast<WindowSmem *>(smem);
    float *kd_tab = reinterpret_cast<float *>(smem + kWindowFixedBytes);   // commit: [warp][tau][32]
    uint8_t *stages = smem + kWindowFixedBytes + A.kd_bytes;
    constexpr bool SR = FMT::kSr;
    bool col_scales, gate_vector;
    if constexpr (FMT::kRuntime) {
        col_scales = F.col_scales != 0;
        gate_vector = F.gate_vector != 0;
    } else {
        col_scales = FMT::kCols;
        gate_vector = FMT::kGvec;
    }

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int t = A.t;
    if (tid == 0) {
        for (int st = 0; st < A.n_stages; ++st) mbar_init(&S.full[st], 1);
        fence_mbar_init();
    }
    __syncthreads();
    asm volatile("griddepcontrol.wait;" ::: "memory");   // see the decode kernel
    const int stride = (int)gridDim.x;
    const int n = A.n_pages;
    const int NS = A.n_stages;
    if (tid == 0) {
        for (int i = 0; i < NS; ++i) {
            const int p = (int)blockIdx.x + i * stride;
            if (p < n) issue_window_stage(F, A, stages + i * A.stage_bytes, p, &S.full[i]);
        }
    }
    const int H = A.heads;
    const int sb = stride / H, sh = stride % H;

    // this lane's row of the slice: block my_blk = lane / 4, stored row my_s
    const int my_blk = lane >> 2;
    const int my_s = 16 * my_blk + 4 * warp + (lane & 3);
    int my_bits, my_rbase;
    if constexpr (FMT::kRuntime) {
        my_bits = F.blk_bits(my_blk);
        my_rbase = F.blk_rbase(my_blk);
    } else {
        my_bits = 0;
        my_rbase = 0;
#pragma unroll
        for (int b = 0; b < kBlocks; ++b) {
            if (b == my_blk) my_bits = FMT::width(b);
            if (b < my_blk && FMT::width(b) != 16) my_rbase += 16;
        }
    }
    const bool my_int = my_bits != 16;
    bool all_int = false;
    if constexpr (!FMT::kRuntime) {
        all_int = true;
        for (int b = 0; b < kBlocks; ++b) all_int = all_int && FMT::width(b) != 16;
    }
    const int my_r = my_rbase + 4 * warp + (lane & 3);
    const float my_qmax = my_int ? (float)((1 << (my_bits - 1)) - 1) : 0.f;
    const float my_rcp = my_int ? __frcp_rn(my_qmax) : 0.f;

    int p = (int)blockIdx.x;
    int pb = p / H, ph = p % H;
    float alpha_s = 0.f, beta_s = 0.f;
    int kap = 0;
    if (p < n) {
        beta_s = __ldg(A.beta + p);
        if (!gate_vector) alpha_s = __ldg(A.alpha + p);
        kap = __ldg(A.perm + ph * kD + my_s) & (kD - 1);
    }
    int p_prev = -1, st = 0, st_prev = 0;
    uint32_t parity = 0;
    int it = 0;

    for (; p < n; ++it) {
        const int pn = p + stride;
        int pnb = pb + sb, pnh = ph + sh;
        if (pnh >= H) { pnh -= H; ++pnb; }
        float alpha_n = 0.f, beta_n = 0.f;
        int kap_n = 0;
        if (pn < n) {
            beta_n = __ldg(A.beta + pn);
            if (!gate_vector) alpha_n = __ldg(A.alpha + pn);
            kap_n = __ldg(A.perm + pnh * kD + my_s) & (kD - 1);
        }

        // a wait that runs out is voted on at the page's barrier, before
        // anything of the page is written to global memory
        const bool ok = mbar_wait_bounded(&S.full[st], parity, A.wait_limit_ns);
        const int par = it & 1;
        uint8_t *stg = stages + st * A.stage_bytes;
        const float *q_s = reinterpret_cast<const float *>(stg + F.page_bytes);
        const float *k_s = q_s + kD;
        const float *v_s = q_s + 2 * kD;
        const float *al_s = q_s + 3 * kD;
        const float *P_s = reinterpret_cast<const float *>(stg + A.p_off);
        const float *K_s = reinterpret_cast<const float *>(stg + A.k_off);
        const float *D_s = reinterpret_cast<const float *>(stg + A.d_off);
        float *r_s = reinterpret_cast<float *>(stg + F.r_off);
        const float *c_s = col_scales ? reinterpret_cast<const float *>(stg + F.c_off) : nullptr;

        // operands of this lane's row: r, RN(P' k), RN(P' q) (and for a
        // commit P' and the row's decayed keys)
        {
            const float al = gate_vector ? al_s[kap] : alpha_s;
            const float pp = t > 0 ? __fmul_rn(P_s[kap], al) : al;
            S.rw[warp][lane] = (all_int || my_int) ? r_s[my_r] : 1.f;
            S.kp[warp][lane] = __fmul_rn(pp, k_s[kap]);
            S.qp[warp][lane] = __fmul_rn(pp, q_s[kap]);
            if constexpr (COMMIT) {
                float *kd = kd_tab + warp * (t + 1) * kRowsPerWarp;
                S.pk[warp][lane] = pp;
                for (int tau = 0; tau < t; ++tau) kd[tau * kRowsPerWarp + lane] = __fmul_rn(K_s[tau * kD + kap], al);
                kd[t * kRowsPerWarp + lane] = k_s[kap];
            }
        }
        // the entries' dot products: warp w takes entries w, w + 4, ...
        {
            const float4 al4 = gate_vector ? *reinterpret_cast<const float4 *>(al_s + 4 * lane)
                                           : make_float4(alpha_s, alpha_s, alpha_s, alpha_s);
            const float4 k4 = *reinterpret_cast<const float4 *>(k_s + 4 * lane);
            const float4 q4 = *reinterpret_cast<const float4 *>(q_s + 4 * lane);
            for (int tau = warp; tau <= t; tau += kWarps) {
                const float4 kk = tau < t ? mul4(*reinterpret_cast<const float4 *>(K_s + tau * kD + 4 * lane), al4) : k4;
                const float a = lane_dot(kk, k4);
                const float b = lane_dot(kk, q4);
                if (lane == 0) {
                    S.da[par][tau] = a;
                    S.dq[par][tau] = b;
                }
            }
        }
        __syncwarp();

        // one pass over the page: dequantize, u's and o's chains
        Tile T;
        float2 cu[2][2], co[2][2];
#pragma unroll
        for (int h = 0; h < 2; ++h) cu[h][0] = cu[h][1] = co[h][0] = co[h][1] = make_float2(0.f, 0.f);
        static_for<0, kBlocks>([&](auto bc) {
            constexpr int b = decltype(bc)::value;
            const float4 a4 = *reinterpret_cast<const float4 *>(&S.rw[warp][4 * b]);
            const uint8_t *blk = stg + fmt_offset<FMT, b>(F);
            with_width<FMT, b>(F, [&](auto wc) {
                constexpr int W = decltype(wc)::value;
                dequant_slice<W, b>(blk, warp, lane, a4, T);
            });
            const float4 k4 = *reinterpret_cast<const float4 *>(&S.kp[warp][4 * b]);
            const float4 q4 = *reinterpret_cast<const float4 *>(&S.qp[warp][4 * b]);
            const float kv[4] = {k4.x, k4.y, k4.z, k4.w};
            const float qv[4] = {q4.x, q4.y, q4.z, q4.w};
            constexpr int h = b >> 2;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                cu[h][0] = __ffma2_rn(make_float2(kv[i], kv[i]), T[b][i][0], cu[h][0]);
                cu[h][1] = __ffma2_rn(make_float2(kv[i], kv[i]), T[b][i][1], cu[h][1]);
                co[h][0] = __ffma2_rn(make_float2(qv[i], qv[i]), T[b][i][0], co[h][0]);
                co[h][1] = __ffma2_rn(make_float2(qv[i], qv[i]), T[b][i][1], co[h][1]);
            }
        });
        store_readout(S.red_u[par][warp], lane, cu);
        store_readout(S.red_o[par][warp], lane, co);

        if (__syncthreads_or(!ok)) {
            // a stage never arrived: record it, store the previous page (a
            // commit), let the copies in flight land and leave
            if (tid == 0) {
                atomicOr(A.status, kStatusTimeout);
                if (COMMIT && p_prev >= 0) {
                    bulk_s2g(A.pages + (size_t)p_prev * F.page_bytes, stages + st_prev * A.stage_bytes, A.store_bytes);
                    bulk_commit();
                }
                const int last = COMMIT ? (it < 3 ? NS - 1 : it - 3 + NS) : (it < 2 ? NS - 1 : it - 2 + NS);
                for (int j = it; j <= last; ++j) {
                    if ((int)blockIdx.x + j * stride < n)
                        mbar_wait_bounded(&S.full[j % NS], (uint32_t)((j / NS) & 1), A.wait_limit_ns);
                }
                bulk_wait<0>();
            }
            __syncthreads();
            return;
        }

        if (tid == 0) {
            // a commit stores the previous page and refills the stage of the
            // one before once its store has read it; otherwise the previous
            // page's stage is free now
            int j = -1;
            if constexpr (COMMIT) {
                if (p_prev >= 0) {
                    bulk_s2g(A.pages + (size_t)p_prev * F.page_bytes, stages + st_prev * A.stage_bytes, A.store_bytes);
                    bulk_commit();
                }
                if (it >= 2) {
                    bulk_wait_read<1>();
                    j = it - 2 + NS;
                }
            } else {
                if (it >= 1) j = it - 1 + NS;
            }
            const int pr = (int)blockIdx.x + j * stride;
            if (j >= 0 && pr < n) {
                fence_proxy_async_smem();
                issue_window_stage(F, A, stages + (j % NS) * A.stage_bytes, pr, &S.full[j % NS]);
            }
        }

        uint8_t *bp = A.buf + (size_t)p * A.stride;
        if constexpr (!COMMIT) {
            // the buffer rows of channel tid: P', the decayed keys, K[t] = k
            const float al = gate_vector ? al_s[tid] : alpha_s;
            reinterpret_cast<float *>(bp)[tid] = t > 0 ? __fmul_rn(P_s[tid], al) : al;
            float *Kg = reinterpret_cast<float *>(bp + 512);
            for (int tau = 0; tau < t; ++tau) Kg[tau * kD + tid] = __fmul_rn(K_s[tau * kD + tid], al);
            Kg[t * kD + tid] = k_s[tid];
        }
        // D[t] and o by one warp (a commit: D[t] in every warp)
        const int fw = it & (kWarps - 1);
        if (COMMIT || warp == fw) {
            const float4 dt = window_delta(S, par, v_s, D_s, c_s, t, beta_s, lane);
            if (warp == fw) {
                if constexpr (!COMMIT)
                    *reinterpret_cast<float4 *>(bp + A.buf_d_off + (size_t)t * 512 + 16 * lane) = dt;
                window_out(S, par, D_s, c_s, t, dt, A.o + (size_t)p * kD, lane);
            }
            if constexpr (COMMIT) {
                // T = RN(P' T0), then the entries in order (per element the
                // same chain; block by block, so that a block's keys are the
                // only operands in registers), and the row maxima
                const float *kd = kd_tab + warp * (t + 1) * kRowsPerWarp;
                const float2 dt01 = make_float2(dt.x, dt.y), dt23 = make_float2(dt.z, dt.w);
                static_for<0, kBlocks>([&](auto bc) {
                    constexpr int b = decltype(bc)::value;
                    const float4 p4 = *reinterpret_cast<const float4 *>(&S.pk[warp][4 * b]);
                    const float pv[4] = {p4.x, p4.y, p4.z, p4.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        T[b][i][0] = __fmul2_rn(T[b][i][0], make_float2(pv[i], pv[i]));
                        T[b][i][1] = __fmul2_rn(T[b][i][1], make_float2(pv[i], pv[i]));
                    }
#pragma unroll 1
                    for (int tau = 0; tau < t; ++tau) {
                        const float4 d = *reinterpret_cast<const float4 *>(D_s + tau * kD + 4 * lane);
                        const float4 k4 = *reinterpret_cast<const float4 *>(kd + tau * kRowsPerWarp + 4 * b);
                        const float kv[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            T[b][i][0] = __ffma2_rn(make_float2(kv[i], kv[i]), make_float2(d.x, d.y), T[b][i][0]);
                            T[b][i][1] = __ffma2_rn(make_float2(kv[i], kv[i]), make_float2(d.z, d.w), T[b][i][1]);
                        }
                    }
                    const float4 k4 = *reinterpret_cast<const float4 *>(kd + t * kRowsPerWarp + 4 * b);
                    const float kv[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        T[b][i][0] = __ffma2_rn(make_float2(kv[i], kv[i]), dt01, T[b][i][0]);
                        T[b][i][1] = __ffma2_rn(make_float2(kv[i], kv[i]), dt23, T[b][i][1]);
                        S.inv[warp][4 * b + i] = warp_absmax(absmax4(T[b][i][0], T[b][i][1]));
                    }
                });
                __syncwarp();
                // lane l finishes row l of the slice: r' = m / qmax, inv = qmax / m (toward zero)
                {
                    const float m = S.inv[warp][lane];
                    float inv = 0.f;
                    if (all_int || my_int) {
                        const float r = div_by_qmax(m, my_qmax, my_rcp);
                        inv = m > 0.f ? div_rz_qmax<(FMT::kTune & kFastRcp) != 0>(my_qmax, m) : 0.f;
                        r_s[my_r] = r;
                    }
                    S.inv[warp][lane] = inv;
                }
                __syncwarp();
                SrCtx sr;
                sr.k0 = A.seed_lo; sr.k1 = A.seed_hi; sr.step = A.step;
                sr.b = (uint32_t)pb;
                sr.h = (uint32_t)ph;
                static_for<0, kBlocks>([&](auto bc) {
                    constexpr int b = decltype(bc)::value;
                    const float4 i4 = *reinterpret_cast<const float4 *>(&S.inv[warp][4 * b]);
                    uint8_t *blk = stg + fmt_offset<FMT, b>(F);
                    with_width<FMT, b>(F, [&](auto wc) {
                        constexpr int W = decltype(wc)::value;
                        requant_slice<W, b, SR>(blk, warp, lane, i4, T, sr);
                    });
                });
                fence_proxy_async_smem();   // the stage's new bytes are read by the bulk store
            }
        }

        p_prev = p;
        st_prev = st;
        alpha_s = alpha_n;
        beta_s = beta_n;
        kap = kap_n;
        p = pn;
        pb = pnb;
        ph = pnh;
        if (++st == NS) { st = 0; parity ^= 1u; }
    }
    asm volatile("griddepcontrol.launch_dependents;");
    __syncthreads();
    if (tid == 0) {
        if (COMMIT && p_prev >= 0) {
            bulk_s2g(A.pages + (size_t)p_prev * F.page_bytes, stages + st_prev * A.stage_bytes, A.store_bytes);
            bulk_commit();
        }
        bulk_wait<0>();
    }
}

// Ring depth and residency: the most pages in flight per SM (resident CTAs x
// pages of look-ahead: NS - 1, a commit NS - 2 since a stage is refilled only
// after its page's store has read it), at most `ctas` CTAs.
static void window_ring(size_t fixed, size_t stage, int ctas, bool commit, int *ns_out) {
    int dev = 0, smem_sm = 0, reserved = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
    cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
    const int min_ns = commit ? 3 : 2;
    int best_ns = min_ns, best_score = -1;
    for (int c = ctas; c >= 1; --c) {
        long ns = ((long)smem_sm / c - reserved - (long)fixed) / (long)stage;
        if (ns > kWindowStages) ns = kWindowStages;
        if (ns < min_ns) continue;
        const int score = c * (int)(ns - (commit ? 2 : 1));
        if (score > best_score) {
            best_score = score;
            best_ns = (int)ns;
        }
    }
    *ns_out = best_ns;
}

template <class FMT, bool COMMIT>
static cudaError_t launch_window_with(const DevFormat &F, const WindowArgs &A0, bool early_launch,
                                      cudaStream_t stream) {
    WindowArgs A = A0;
    const size_t fixed = kWindowFixedBytes + A.kd_bytes;
    window_ring(fixed, A.stage_bytes, window_ctas_per_sm<COMMIT>(), COMMIT, &A.n_stages);
    const size_t smem = fixed + (size_t)A.n_stages * A.stage_bytes;
    const void *fn = (const void *)window_kernel<FMT, COMMIT>;
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
    return cudaLaunchKernelEx(&cfg, window_kernel<FMT, COMMIT>, F, A);
}

template <bool COMMIT>
static cudaError_t launch_window_fmt(const DevFormat &F, const WindowArgs &A, bool early_launch, cudaStream_t stream) {
    if (format_is<FmtStepQuant6>(F)) return launch_window_with<FmtStepQuant6, COMMIT>(F, A, early_launch, stream);
    if (format_is<FmtInt8Row>(F)) return launch_window_with<FmtInt8Row, COMMIT>(F, A, early_launch, stream);
    if (format_is<FmtStepQuant4Kda>(F)) return launch_window_with<FmtStepQuant4Kda, COMMIT>(F, A, early_launch, stream);
    if (format_is<FmtDamp>(F)) return launch_window_with<FmtDamp, COMMIT>(F, A, early_launch, stream);
    if (F.stochastic) return launch_window_with<RuntimeFmt<true>, COMMIT>(F, A, early_launch, stream);
    return launch_window_with<RuntimeFmt<false>, COMMIT>(F, A, early_launch, stream);
}

size_t window_buffer_stride(int window) { return 512u * (1u + 2u * (size_t)window); }

cudaError_t launch_window(const stq_state *s, uint8_t *buf, int window, int t, bool commit, const float *q,
                          const float *k, const float *v, const float *alpha, const float *beta, float *o,
                          uint64_t seed, uint32_t step, bool early_launch, cudaStream_t stream) {
    const DevFormat &F = s->dev;
    WindowArgs A;
    A.pages = s->base + s->pages_offset;
    A.perm = s->base + s->perm_offset;
    A.status = reinterpret_cast<uint32_t *>(s->base + s->status_offset);
    A.q = q; A.k = k; A.v = v; A.alpha = alpha; A.beta = beta; A.o = o;
    A.buf = buf;
    A.stride = (uint32_t)window_buffer_stride(window);
    A.buf_d_off = 512u * (1u + (uint32_t)window);
    A.t = t;
    A.n_pages = s->batch * s->heads;
    A.heads = s->heads;
    A.n_stages = 0;
    const uint32_t rows = (uint32_t)F.page_bytes + 1536u + (F.gate_vector ? 512u : 0u);
    A.p_off = rows;
    A.k_off = rows + 512u;
    A.d_off = A.k_off + 512u * (uint32_t)t;
    A.tx_bytes = rows + (t > 0 ? 512u + 1024u * (uint32_t)t : 0u);
    A.stage_bytes = (A.tx_bytes + 127u) / 128u * 128u;
    A.store_bytes = (uint32_t)(F.col_scales ? F.c_off : F.page_bytes);
    A.kd_bytes = commit ? 512u * (uint32_t)(t + 1) : 0u;
    A.seed_lo = (uint32_t)seed;
    A.seed_hi = (uint32_t)(seed >> 32);
    A.step = step;
    A.wait_limit_ns = s->wait_limit_ns;
    if (commit) return launch_window_fmt<true>(F, A, early_launch, stream);
    return launch_window_fmt<false>(F, A, early_launch, stream);
}

}  // namespace stq
