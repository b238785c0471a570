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
// Step t, with z the fixed page's exact codes (FP16 rows: h; stored order,
// the row of stored index s holding key channel perm[s]) and one factor per
// stored row, a'_s = RN(P'_kappa r_s) (FP16 rows: P'_kappa), the window's
// decay folded into the row scale as the decode step folds alpha into r:
//   P' = P alpha;   K[tau] <- RN(K[tau] alpha)                  (tau < t)
//   u = z^T RN(k a') + sum_{tau<t} (K[tau] . k) D[tau]
//   D[t] = RN(beta (v (1/c) - u));   K[t] = k
//   o = c (z^T RN(q a') + sum_{tau<=t} (K[tau] . q) D[tau])
// The column sums over the page are the decode kernel's (same slices, chains
// and tree); both run in one pass, since the page does not change within a
// window.  A buffer dot product is a 4-channel fma chain per lane (lane l:
// channels 4l .. 4l+3) and an xor butterfly over the warp; buffer terms are
// added by fma in entry order.  A committing step then rebuilds
// T = RN(z a'), T <- fma(K[tau], D[tau], T) for tau = 0 .. t, in registers,
// and requantizes it exactly as the decode step requantizes T'; it writes
// nothing to the buffer (a window's first step reads none of it).
//
// Staging is the decode kernel's: the page, the input rows and the buffer rows
// a step reads are copied into a shared-memory ring with cp.async.bulk (no
// multicast), counted on an mbarrier with a bounded wait.
#include "stq_rows.cuh"

namespace stq {

constexpr int kWindowMax = STQ_WINDOW_MAX;
constexpr int kWindowStages = 4;          // ring depth at most
constexpr int kRebuildGroup = 4;          // blocks per pass of a commit's entry loop (measured: 1, 2, 4, 8)

struct WindowArgs {
    uint8_t *pages;
    const uint8_t *perm;
    uint32_t *status;
    const float *q, *k, *v, *alpha, *beta;
    float *o;
    uint8_t *buf;                 // window buffer, stride bytes per page
    uint32_t stride;
    uint32_t buf_d_off;           // D inside a page's buffer: 512 (1 + W)
    int t;                        // position of this step in its window
    int n_pages, heads, n_stages;
    uint32_t stage_bytes;         // ring stride (a multiple of 128)
    uint32_t tx_bytes;            // bytes a stage receives
    uint32_t store_bytes;         // codes + r: the part of a page a commit rewrites
    uint32_t p_off, k_off, d_off; // buffer rows inside a stage
    uint32_t scr_off;             // the stage's scratch (the warps' sums)
    uint32_t kd_bytes;            // per-warp key table of a commit (0 otherwise)
    uint32_t seed_lo, seed_hi, step;
    uint64_t wait_limit_ns;
    int stall_first_wait;
};

struct WindowSmem {
    // per warp, its 32 rows in slice order (row 4b + i = block b, row i):
    float kp[kWarps][kRowsPerWarp];         // RN(k a') of the row's key channel
    float qp[kWarps][kRowsPerWarp];         // RN(q a')
    float pk[kWarps][kRowsPerWarp];         // a' = RN(P' r), FP16 rows P' (commit)
    float inv[kWarps][kRowsPerWarp];        // commit: row maxima, then requant multipliers
    uint64_t full[kWindowStages];           // stage-full barriers
    uint64_t never;                         // a barrier nothing completes (test hook)
    uint32_t phase[kWindowStages];          // parity of the stage's latest load
    int issued[kWindowStages];              // the stage has had a load
};

// A stage's scratch, after the bytes its load brings: the warps' chain sums
// of the page and the entries' dot products.
struct WindowScratch {
    float red_u[kWarps][kD];
    float red_o[kWarps][kD];
    float da[kWindowMax];                   // K[tau] . k
    float dq[kWindowMax];                   // K[tau] . q
};

constexpr size_t kWindowFixedBytes = (sizeof(WindowSmem) + 127) / 128 * 128;
constexpr uint32_t kScratchBytes = (uint32_t)((sizeof(WindowScratch) + 127) / 128 * 128);

// Stage layout: page, q, k, v (, alpha), then (t > 0) P, K[0 .. t-1],
// D[0 .. t-1]; then the scratch.
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
__device__ __forceinline__ float4 window_delta(const WindowScratch &X, const float *v_s, const float *d_s,
                                               const float *c_s, int t, float beta, int lane) {
    float4 u = tree4(X.red_u, lane);
    for (int tau = 0; tau < t; ++tau)
        u = fma4(X.da[tau], *reinterpret_cast<const float4 *>(d_s + tau * kD + 4 * lane), u);
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
__device__ __forceinline__ float4 window_out(const WindowScratch &X, const float *d_s, const float *c_s, int t,
                                             float4 dt, int lane) {
    float4 ot = tree4(X.red_o, lane);
    for (int tau = 0; tau < t; ++tau)
        ot = fma4(X.dq[tau], *reinterpret_cast<const float4 *>(d_s + tau * kD + 4 * lane), ot);
    ot = fma4(X.dq[t], dt, ot);
    if (c_s) ot = mul4(*reinterpret_cast<const float4 *>(c_s + 4 * lane), ot);
    return ot;
}

// The page's pointers inside a stage.
struct StageView {
    const float *q, *k, *v, *al, *P, *K, *D, *c;
    float *r;
    WindowScratch *X;
};

__device__ __forceinline__ StageView stage_view(const DevFormat &F, const WindowArgs &A, uint8_t *stg,
                                                bool col_scales) {
    StageView V;
    V.q = reinterpret_cast<const float *>(stg + F.page_bytes);
    V.k = V.q + kD;
    V.v = V.q + 2 * kD;
    V.al = V.q + 3 * kD;
    V.P = reinterpret_cast<const float *>(stg + A.p_off);
    V.K = reinterpret_cast<const float *>(stg + A.k_off);
    V.D = reinterpret_cast<const float *>(stg + A.d_off);
    V.c = col_scales ? reinterpret_cast<const float *>(stg + F.c_off) : nullptr;
    V.r = reinterpret_cast<float *>(stg + F.r_off);
    V.X = reinterpret_cast<WindowScratch *>(stg + A.scr_off);
    return V;
}

// The exact values of slice w of block B: the codes z (FP16 rows: h) as floats.
template <int W, int B>
__device__ __forceinline__ void codes_slice(const uint8_t *blk, int w, int lane, Tile &T) {
    if constexpr (W == 16) {
        uint32_t x[8];
        load_fp16_slice(blk, w, lane, x);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            T[B][i][0] = __half22float2(*reinterpret_cast<const __half2 *>(&x[2 * i]));
            T[B][i][1] = __half22float2(*reinterpret_cast<const __half2 *>(&x[2 * i + 1]));
        }
    } else {
        uint32_t ub[4];
        unpack_int_slice<W>(blk, w, lane, ub);
        const float bm = 8388608.0f + (float)(1 << (W - 1));
#pragma unroll
        for (int i = 0; i < 4; ++i) codes_to_float(ub[i], bm, T[B][i][0], T[B][i][1]);
    }
}

// The first phase of a page, per warp: the operands of this lane's row, the
// entries' dot products (warp w: entries w, w + 4, ...) and one pass over the
// warp's slices (dequantize, u's and o's chains), whose sums go to the
// stage's scratch.  A commit also keeps the row factor a' and the row's
// decayed keys (kd: this warp's [tau][32] table).
template <class FMT, bool COMMIT>
__device__ __forceinline__ void window_first_phase(const DevFormat &F, const WindowArgs &A, WindowSmem &S,
                                                   const uint8_t *stg, const StageView &V, const RowCtx &R,
                                                   int kap, float alpha_s, bool gate_vector, int warp, int lane,
                                                   float *kd) {
    const int t = A.t;
    {
        const float al = gate_vector ? V.al[kap] : alpha_s;
        const float pp = t > 0 ? __fmul_rn(V.P[kap], al) : al;
        const float af = (R.all_int || R.is_int) ? __fmul_rn(pp, V.r[R.rix]) : pp;   // a'
        S.kp[warp][lane] = __fmul_rn(V.k[kap], af);
        S.qp[warp][lane] = __fmul_rn(V.q[kap], af);
        if constexpr (COMMIT) {
            S.pk[warp][lane] = af;
            for (int tau = 0; tau < t; ++tau) kd[tau * kRowsPerWarp + lane] = __fmul_rn(V.K[tau * kD + kap], al);
            kd[t * kRowsPerWarp + lane] = V.k[kap];
        }
    }
    {
        const float4 al4 = gate_vector ? *reinterpret_cast<const float4 *>(V.al + 4 * lane)
                                       : make_float4(alpha_s, alpha_s, alpha_s, alpha_s);
        const float4 k4 = *reinterpret_cast<const float4 *>(V.k + 4 * lane);
        const float4 q4 = *reinterpret_cast<const float4 *>(V.q + 4 * lane);
        for (int tau = warp; tau <= t; tau += kWarps) {
            float4 kk = k4;
            if (tau < t) kk = mul4(*reinterpret_cast<const float4 *>(V.K + tau * kD + 4 * lane), al4);
            const float a = lane_dot(kk, k4);
            const float b = lane_dot(kk, q4);
            if (lane == 0) {
                V.X->da[tau] = a;
                V.X->dq[tau] = b;
            }
        }
    }
    __syncwarp();   // the warp's rows' operands come from its own lanes

    float2 cu[2][2], co[2][2];
#pragma unroll
    for (int h = 0; h < 2; ++h) cu[h][0] = cu[h][1] = co[h][0] = co[h][1] = make_float2(0.f, 0.f);
    static_for<0, kBlocks>([&](auto bc) {
        constexpr int b = decltype(bc)::value;
        const uint8_t *blk = stg + fmt_offset<FMT, b>(F);
        Tile T;   // only block b of it is live: the exact codes
        with_width<FMT, b>(F, [&](auto wc) {
            constexpr int W = decltype(wc)::value;
            codes_slice<W, b>(blk, warp, lane, T);
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
    store_readout(V.X->red_u[warp], lane, cu);
    store_readout(V.X->red_o[warp], lane, co);
}

// Barriers, counters and the first loads of the ring (thread 0), then the
// wait for the previous kernel on the stream (see the decode kernel).
__device__ __forceinline__ void window_start(const DevFormat &F, const WindowArgs &A, WindowSmem &S,
                                             uint8_t *stages) {
    const int stride = (int)gridDim.x;
    if (threadIdx.x == 0) {
        for (int st = 0; st < A.n_stages; ++st) {
            mbar_init(&S.full[st], 1);
            S.phase[st] = 0;
            S.issued[st] = 0;
        }
        mbar_init(&S.never, 1);
        fence_mbar_init();
    }
    __syncthreads();
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (threadIdx.x == 0) {
        for (int i = 0; i < A.n_stages; ++i) {
            const int p = (int)blockIdx.x + i * stride;
            if (p < A.n_pages) {
                issue_window_stage(F, A, stages + i * A.stage_bytes, p, &S.full[i]);
                S.issued[i] = 1;
            }
        }
    }
}

// Loads in flight when the CTA stops early (a wait ran out) land before it
// exits: thread 0 waits, bounded, for each stage's latest load.
__device__ __forceinline__ void window_drain(const WindowArgs &A, WindowSmem &S) {
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int st = 0; st < A.n_stages; ++st)
            if (S.issued[st]) mbar_wait_bounded(&S.full[st], S.phase[st], A.wait_limit_ns);
    }
}

// A step that does not commit: one CTA barrier per page, after the first
// phase.  After it, thread c writes channel c's buffer rows (P', the decayed
// keys, K[t] = k) and finishes column c: D[t] and o; one warp per page, in
// turn, refills the previous page's stage.
template <class FMT>
__global__ void __launch_bounds__(kThreads, 4) window_step_kernel(const DevFormat F, const WindowArgs A) {
    extern __shared__ __align__(128) uint8_t smem[];
    WindowSmem &S = *reinterpret_cast<WindowSmem *>(smem);
    uint8_t *stages = smem + kWindowFixedBytes;
    bool col_scales, gate_vector;
    format_flags<FMT>(F, col_scales, gate_vector);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int t = A.t;
    window_start(F, A, S, stages);
    const int stride = (int)gridDim.x;
    const int n = A.n_pages;
    const int NS = A.n_stages;
    const int H = A.heads;
    const int sh = stride % H;
    const RowCtx R = row_ctx<FMT>(F, warp, lane);

    int p = (int)blockIdx.x;
    int ph = p % H;
    float alpha_s = 0.f, beta_s = 0.f;
    int kap = 0;
    if (p < n) {
        beta_s = __ldg(A.beta + p);
        if (!gate_vector) alpha_s = __ldg(A.alpha + p);
        kap = __ldg(A.perm + ph * kD + R.s) & (kD - 1);
    }
    int st = 0, st_prev = 0;
    uint32_t parity = 0;
    for (int it = 0; p < n; ++it) {
        const int pn = p + stride;
        int pnh = ph + sh;   // the head advances by stride mod H
        if (pnh >= H) pnh -= H;
        float alpha_n = 0.f, beta_n = 0.f;
        int kap_n = 0;
        if (pn < n) {
            beta_n = __ldg(A.beta + pn);
            if (!gate_vector) alpha_n = __ldg(A.alpha + pn);
            kap_n = __ldg(A.perm + pnh * kD + R.s) & (kD - 1);
        }
        // a wait that runs out is voted on at the page's barrier, before
        // anything of the page is written to global memory
        bool ok;
        if (A.stall_first_wait && it == 0) ok = mbar_wait_bounded(&S.never, 0, A.wait_limit_ns);
        else ok = mbar_wait_bounded(&S.full[st], parity, A.wait_limit_ns);
        uint8_t *stg = stages + st * A.stage_bytes;
        const StageView V = stage_view(F, A, stg, col_scales);
        window_first_phase<FMT, false>(F, A, S, stg, V, R, kap, alpha_s, gate_vector, warp, lane, nullptr);
        if (__syncthreads_or(!ok)) {
            if (tid == 0) atomicOr(A.status, kStatusTimeout);
            break;   // the loads in flight land in the drain below
        }
        if (it >= 1 && tid == 32 * (it & (kWarps - 1))) {
            // every warp is done with the previous page: refill its stage
            const int pr = p + (NS - 1) * stride;
            if (pr < n) {
                fence_proxy_async_smem();
                issue_window_stage(F, A, stages + st_prev * A.stage_bytes, pr, &S.full[st_prev]);
                S.phase[st_prev] ^= 1u;
            }
        }
        uint8_t *bp = A.buf + (size_t)p * A.stride;
        {
            const float al = gate_vector ? V.al[tid] : alpha_s;
            reinterpret_cast<float *>(bp)[tid] = t > 0 ? __fmul_rn(V.P[tid], al) : al;
            float *Kg = reinterpret_cast<float *>(bp + 512);
            for (int tau = 0; tau < t; ++tau) Kg[tau * kD + tid] = __fmul_rn(V.K[tau * kD + tid], al);
            Kg[t * kD + tid] = V.k[tid];
        }
        {
            // column c = tid: u = (W0 + W1) + (W2 + W3) + the earlier entries,
            // e = v (1/c) - u, D[t] = RN(beta e); o = c (tree + every entry's term)
            const WindowScratch &X = *V.X;
            const int col = tid;
            float u = __fadd_rn(__fadd_rn(X.red_u[0][col], X.red_u[1][col]),
                                __fadd_rn(X.red_u[2][col], X.red_u[3][col]));
            float ot = __fadd_rn(__fadd_rn(X.red_o[0][col], X.red_o[1][col]),
                                 __fadd_rn(X.red_o[2][col], X.red_o[3][col]));
            for (int tau = 0; tau < t; ++tau) {
                const float d = V.D[tau * kD + col];
                u = __fmaf_rn(X.da[tau], d, u);
                ot = __fmaf_rn(X.dq[tau], d, ot);
            }
            const float c = col_scales ? V.c[col] : 1.f;
            const float ic = col_scales ? __frcp_rn(c) : 1.f;
            const float dtc = __fmul_rn(beta_s, __fsub_rn(__fmul_rn(V.v[col], ic), u));
            ot = __fmaf_rn(X.dq[t], dtc, ot);
            reinterpret_cast<float *>(bp + A.buf_d_off + (size_t)t * 512)[col] = dtc;
            A.o[(size_t)p * kD + col] = col_scales ? __fmul_rn(c, ot) : ot;
        }
        st_prev = st;
        alpha_s = alpha_n;
        beta_s = beta_n;
        kap = kap_n;
        p = pn;
        ph = pnh;
        if (++st == NS) { st = 0; parity ^= 1u; }
    }
    asm volatile("griddepcontrol.launch_dependents;");
    window_drain(A, S);
}

// A committing step: one CTA barrier per page, after the first phase, since
// every warp needs this step's delta D[t] for its own rows.  After it each
// warp dequantizes its slices again with the row factor, T = RN(z a') (the
// page is intact in the stage until the warp requantizes them), adds the
// entries in order, takes the row maxima and requantizes in place; the
// stage is stored at the next page's barrier and refilled once the store has
// read it.
template <class FMT>
__global__ void __launch_bounds__(kThreads, 3) window_commit_kernel(const DevFormat F, const WindowArgs A) {
    extern __shared__ __align__(128) uint8_t smem[];
    WindowSmem &S = *reinterpret_cast<WindowSmem *>(smem);
    float *kd_tab = reinterpret_cast<float *>(smem + kWindowFixedBytes);   // [warp][tau][32]
    uint8_t *stages = smem + kWindowFixedBytes + A.kd_bytes;
    constexpr bool SR = FMT::kSr;
    bool col_scales, gate_vector;
    format_flags<FMT>(F, col_scales, gate_vector);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int t = A.t;
    window_start(F, A, S, stages);
    const int stride = (int)gridDim.x;
    const int n = A.n_pages;
    const int NS = A.n_stages;
    const int H = A.heads;
    const int sb = stride / H, sh = stride % H;
    const RowCtx R = row_ctx<FMT>(F, warp, lane);
    float *kd = kd_tab + warp * (t + 1) * kRowsPerWarp;

    int p = (int)blockIdx.x;
    int pb = p / H, ph = p % H;
    float alpha_s = 0.f, beta_s = 0.f;
    int kap = 0;
    if (p < n) {
        beta_s = __ldg(A.beta + p);
        if (!gate_vector) alpha_s = __ldg(A.alpha + p);
        kap = __ldg(A.perm + ph * kD + R.s) & (kD - 1);
    }
    int p_prev = -1, st = 0, st_prev = 0;
    uint32_t parity = 0;
    for (int it = 0; p < n; ++it) {
        const int pn = p + stride;
        int pnb = pb + sb, pnh = ph + sh;
        if (pnh >= H) { pnh -= H; ++pnb; }
        float alpha_n = 0.f, beta_n = 0.f;
        int kap_n = 0;
        if (pn < n) {
            beta_n = __ldg(A.beta + pn);
            if (!gate_vector) alpha_n = __ldg(A.alpha + pn);
            kap_n = __ldg(A.perm + pnh * kD + R.s) & (kD - 1);
        }
        // a wait that runs out is voted on at the page's barrier, before
        // anything of the page is written to global memory
        bool ok;
        if (A.stall_first_wait && it == 0) ok = mbar_wait_bounded(&S.never, 0, A.wait_limit_ns);
        else ok = mbar_wait_bounded(&S.full[st], parity, A.wait_limit_ns);
        uint8_t *stg = stages + st * A.stage_bytes;
        const StageView V = stage_view(F, A, stg, col_scales);
        window_first_phase<FMT, true>(F, A, S, stg, V, R, kap, alpha_s, gate_vector, warp, lane, kd);

        if (__syncthreads_or(!ok)) {
            // record it, store the previous (finished) page and leave; the
            // loads in flight land in the drain below
            if (tid == 0) {
                atomicOr(A.status, kStatusTimeout);
                if (p_prev >= 0) {
                    bulk_s2g(A.pages + (size_t)p_prev * F.page_bytes, stages + st_prev * A.stage_bytes,
                             A.store_bytes);
                    bulk_commit();
                }
                bulk_wait<0>();
            }
            break;
        }
        if (tid == 0 && p_prev >= 0) {
            // the previous page is complete in its stage: store it
            bulk_s2g(A.pages + (size_t)p_prev * F.page_bytes, stages + st_prev * A.stage_bytes, A.store_bytes);
            bulk_commit();
        }
        const WindowScratch &X = *V.X;
        // o of columns 4l .. 4l+3 by one warp (in turn); D[t] of them in every warp
        const float4 dt = window_delta(X, V.v, V.D, V.c, t, beta_s, lane);
        if (warp == (it & (kWarps - 1)))
            *reinterpret_cast<float4 *>(A.o + (size_t)p * kD + 4 * lane) = window_out(X, V.D, V.c, t, dt, lane);

        // T = RN(z a'), then the entries in order (per element one chain;
        // a group of blocks at a time, so that the group's keys and one
        // delta row are the only operands in registers besides T), and the
        // row maxima
        const float2 dt01 = make_float2(dt.x, dt.y), dt23 = make_float2(dt.z, dt.w);
        Tile T;
        // blocks in groups of kRebuildGroup: each entry's delta row is read
        // once per group
        static_for<0, kBlocks / kRebuildGroup>([&](auto gc) {
            constexpr int g = decltype(gc)::value;
            static_for<0, kRebuildGroup>([&](auto jc) {
                constexpr int b = g * kRebuildGroup + decltype(jc)::value;
                const float4 a4 = *reinterpret_cast<const float4 *>(&S.pk[warp][4 * b]);
                const uint8_t *blk = stg + fmt_offset<FMT, b>(F);
                with_width<FMT, b>(F, [&](auto wc) {
                    constexpr int W = decltype(wc)::value;
                    dequant_slice<W, b>(blk, warp, lane, a4, T);   // RN(z a')
                });
            });
#pragma unroll 1
            for (int tau = 0; tau < t; ++tau) {
                const float4 d = *reinterpret_cast<const float4 *>(V.D + tau * kD + 4 * lane);
                static_for<0, kRebuildGroup>([&](auto jc) {
                    constexpr int b = g * kRebuildGroup + decltype(jc)::value;
                    const float4 k4 = *reinterpret_cast<const float4 *>(kd + tau * kRowsPerWarp + 4 * b);
                    const float kv[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        T[b][i][0] = __ffma2_rn(make_float2(kv[i], kv[i]), make_float2(d.x, d.y), T[b][i][0]);
                        T[b][i][1] = __ffma2_rn(make_float2(kv[i], kv[i]), make_float2(d.z, d.w), T[b][i][1]);
                    }
                });
            }
            static_for<0, kRebuildGroup>([&](auto jc) {
                constexpr int b = g * kRebuildGroup + decltype(jc)::value;
                const float4 k4 = *reinterpret_cast<const float4 *>(kd + t * kRowsPerWarp + 4 * b);
                const float kv[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    T[b][i][0] = __ffma2_rn(make_float2(kv[i], kv[i]), dt01, T[b][i][0]);
                    T[b][i][1] = __ffma2_rn(make_float2(kv[i], kv[i]), dt23, T[b][i][1]);
                    S.inv[warp][4 * b + i] = warp_absmax(absmax4(T[b][i][0], T[b][i][1]));
                }
            });
        });
        if (tid == 0 && p_prev >= 0) {
            // refill the previous page's stage with the page NS - 1 ahead of this one
            bulk_wait_read<0>();
            const int pr = p + (NS - 1) * stride;
            if (pr < n) {
                fence_proxy_async_smem();
                issue_window_stage(F, A, stages + st_prev * A.stage_bytes, pr, &S.full[st_prev]);
                S.phase[st_prev] ^= 1u;
            }
        }
        __syncwarp();
        // lane l finishes row l of the slice: r' = m / qmax, inv = qmax / m (toward zero)
        {
            const float m = S.inv[warp][lane];
            float inv = 0.f;
            if (R.all_int || R.is_int) {
                const float r = div_by_qmax(m, R.qmax, R.rcp_qmax);
                inv = m > 0.f ? div_rz_qmax<(FMT::kTune & kFastRcp) != 0>(R.qmax, m) : 0.f;
                V.r[R.rix] = r;
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
            uint8_t *blk = stg + fmt_offset<FMT, b>(F);
            with_width<FMT, b>(F, [&](auto wc) {
                constexpr int W = decltype(wc)::value;
                requant_slice<W, b, SR>(blk, warp, lane, i4, T, sr);
            });
        });
        fence_proxy_async_smem();   // the stage's new bytes are read by the bulk store

        p_prev = p;
        st_prev = st;
        alpha_s = alpha_n;
        beta_s = beta_n;
        kap = kap_n;
        p = pn;
        pb = pnb;
        ph = pnh;
        if (++st == NS) { st = 0; parity ^= 1u; }
        if (p >= n) {
            // the last page: store it once every warp has requantized its slices
            asm volatile("griddepcontrol.launch_dependents;");
            __syncthreads();
            if (tid == 0) {
                bulk_s2g(A.pages + (size_t)p_prev * F.page_bytes, stages + st_prev * A.stage_bytes, A.store_bytes);
                bulk_commit();
                bulk_wait<0>();
            }
        }
    }
    window_drain(A, S);
}

// Ring depth and residency: the most resident CTAs (up to `ctas`) whose ring
// holds at least two stages, then the deepest ring at that residency (at most
// kWindowStages).  Measured on a B200: residency beats look-ahead here.
static int window_ring(size_t fixed, size_t stage, int ctas) {
    int dev = 0, smem_sm = 0, reserved = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
    cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
    for (int c = ctas; c >= 1; --c) {
        long ns = ((long)smem_sm / c - reserved - (long)fixed) / (long)stage;
        if (ns >= 2) return ns > kWindowStages ? kWindowStages : (int)ns;
    }
    return 2;
}

template <class FMT, bool COMMIT>
static cudaError_t launch_window_with(const DevFormat &F, const WindowArgs &A0, bool early_launch,
                                      cudaStream_t stream) {
    WindowArgs A = A0;
    const size_t fixed = kWindowFixedBytes + A.kd_bytes;
    A.n_stages = window_ring(fixed, A.stage_bytes, COMMIT ? 3 : 4);
    const size_t smem = fixed + (size_t)A.n_stages * A.stage_bytes;
    const void *fn = COMMIT ? (const void *)window_commit_kernel<FMT> : (const void *)window_step_kernel<FMT>;
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
    if constexpr (COMMIT) return cudaLaunchKernelEx(&cfg, window_commit_kernel<FMT>, F, A);
    else return cudaLaunchKernelEx(&cfg, window_step_kernel<FMT>, F, A);
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
                          uint64_t seed, uint32_t step, int stall_first_wait, bool early_launch,
                          cudaStream_t stream) {
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
    A.scr_off = (A.tx_bytes + 127u) / 128u * 128u;
    A.stage_bytes = A.scr_off + kScratchBytes;
    A.store_bytes = (uint32_t)(F.col_scales ? F.c_off : F.page_bytes);
    A.kd_bytes = commit ? 512u * (uint32_t)(t + 1) : 0u;
    A.seed_lo = (uint32_t)seed;
    A.seed_hi = (uint32_t)(seed >> 32);
    A.step = step;
    A.wait_limit_ns = s->wait_limit_ns;
    A.stall_first_wait = stall_first_wait;
    if (commit) return launch_window_fmt<true>(F, A, early_launch, stream);
    return launch_window_fmt<false>(F, A, early_launch, stream);
}

}  // namespace stq
