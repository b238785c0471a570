// stq_prefill_tc.cu -- the chunkwise prefill on the fifth-generation tensor
// cores (sm_100a, tcgen05): a prompt of L tokens through every page of a
// state, 128 tokens per chunk, one requantization after the last token.
//
// Per chunk of n <= 128 tokens from the state S0 (T = S / c units, key rows
// in natural order), with gam_i = prod of the gates of tokens 0..i of the
// chunk (per key channel for gate vectors; the UT-transform form of the
// delta rule, "repeated prefill": DASC):
//   G  = K K^T,  A_ij = beta_i rho_ij G_ij  (j < i)
//   E  = (I + A)^-1 R,  R_i = beta_i (v_i / c - gam_i (S0^T k_i))
//   o_i = c (gam_i S0^T q_i + sum_{j<=i} rho_ij (q_i . k_j) E_j)
//   S  <- gam_n S0 + sum_j rho_nj k_j E_j^T
// with rho_ij = gam_i / gam_j.  Scalar gates take it as gam_i (1 / gam_j)
// while every cumulative decay of the chunk lies in [2^-100, 2^100]
// (otherwise a second launch forms it as the product of the gates of tokens
// j + 1 .. i).  Gate vectors fold gam into the operands, G = (K Gam)(K /
// Gam)^T and so on, while every gate lies in [0, 1] and every cumulative
// decay in [2^-100, 1] (tested on the staged decays, slab by slab; a chunk
// that fails runs token by token on the CUDA cores).
// The products run on the tensor cores in tf32 with each fp32 operand split
// into a tf32 part and its remainder (three MMAs per product: hi hi, hi lo,
// lo hi), which keeps fp32-level accuracy; the triangular solve runs on the
// CUDA cores (thread v owns value column v of E).
//
// One CTA of 256 threads per page (persistent over pages; 170-216 KB of
// shared memory and all 512 tensor-memory columns keep it alone on its SM).
// Thread t of each 128-thread half owns row t of whatever a phase computes:
// token t, value column t, or key channel t, which is also tensor-memory
// lane t (warps w and w + 4 see the same 32 lanes); the two halves split the
// row's columns between them.  The triangular solve runs on the first half.
//   shared memory: six (gate vectors: eight) 16 KB operand tiles (128 rows x
//   32 fp32, 128-byte swizzled, K-major), reused as the solve's matrix A and
//   as the page buffer; the state X = S^T (X[v][kappa], fp32, rows padded to
//   129 floats); per-token scalars; (gate vectors) one slab's decays.
//   tensor memory: G | Y^T | P | O^T, then the state's increment in G's
//   columns.
#include "stq_rows.cuh"
#include "stq_tc.cuh"

namespace stq {

constexpr int kChunk = 128;                    // tokens per chunk
constexpr int kTcThreads = 256;                // two halves of 128 threads
static_assert(kTcThreads == 2 * kChunk, "a page's gates are staged two chunks at a time");
constexpr int kXStride = kD + 1;               // floats per state row
constexpr int kAStride = kChunk + 4;           // floats per row of the solve's matrix (16-byte rows)
// operand tiles: six for scalar gates (K, gam Q, X as hi / lo pairs), eight
// for gate vectors (K Gam, Q Gam, X, K / Gam)
template <bool GV>
__host__ __device__ constexpr uint32_t tile_region() { return (GV ? 8u : 6u) * tc::kTileBytes; }
constexpr int kGsStride = 33;                  // floats per token row of the staged decays

struct TcArgs {
    uint8_t *pages;
    const uint8_t *perm;
    uint32_t *status;
    uint32_t *pending;       // == call when the quotient launch left pages to the product launch
    uint32_t call;           // this call's mark (never 0)
    const float *q, *k, *v, *alpha, *beta;
    float *o, *S_out;
    int L, n_pages, heads;
    uint32_t store_bytes;
    uint32_t seed_lo, seed_hi, step;
    uint64_t wait_limit_ns;
    int stall_first_wait;
};

struct TcSmall {
    float gam[kChunk];       // cumulative gate of the chunk's tokens
    float al[kChunk];        // the gate of each token (1 for padding)
    float bet[kChunk];       // beta (0 for padding)
    float kts[kChunk];       // a key's decay to the chunk's end: the gates of tokens j + 1 .. n - 1
    float igam[kChunk];      // 1 / gam (chunks whose decays stay in range)
    float c[kD], ic[kD];     // column scale and its inverse
    alignas(16) float inv[kWarps][kRowsPerWarp];   // read as float4
    int kap[kD];             // stored row -> key channel
    uint64_t mma_bar, page_bar, never;
    uint32_t tmem;
    int in_range;            // this chunk's cumulative decays lie in [2^-100, 2^100]
    float gn[kD];            // gate vectors: each key channel's decay to the chunk's end
    float segp[8][32];       // gate vectors: products of 16-token segments of one slab's channels
    float red[2][2][kD];     // gate vectors, token by token: the halves' partial sums (u, o)
    alignas(16) float tok[2][4][kD];   // gate vectors, token by token: k, q, gate, v / c (two buffers; float4 reads)
};

static_assert(offsetof(TcSmall, inv) % 16 == 0, "inv is read as float4");
static_assert(offsetof(TcSmall, mma_bar) % 8 == 0, "mbarriers are 8-byte aligned");
static_assert((tile_region<false>() + (size_t)kD * kXStride * 4) % alignof(TcSmall) == 0, "TcSmall follows X aligned");
static_assert((tile_region<true>() + (size_t)kD * kXStride * 4) % alignof(TcSmall) == 0, "TcSmall follows X aligned");
static_assert(sizeof(TcSmall) % 16 == 0, "the staged decays follow TcSmall 16-byte aligned");
static_assert(offsetof(TcSmall, tok) % 16 == 0, "tok is read as float4");
// shared memory: tiles, X, TcSmall, (gate vectors) one slab's decays of the
// chunk's tokens, 1 KB for the alignment of the tiles
template <bool GV>
constexpr size_t tc_smem() {
    return tile_region<GV>() + (size_t)kD * kXStride * 4 + sizeof(TcSmall) +
           (GV ? (size_t)kChunk * kGsStride * 4 : 0) + 1024;
}
static_assert(tc_smem<true>() <= 227 * 1024, "shared memory of one CTA");

// four consecutive columns k .. k + 3 (k a multiple of 4) of a row: one
// 16-byte unit of the swizzled row, so a warp's 32 rows take 4 conflict-free
// shared-memory wavefronts (a float at a time, 8 banks serve the 32 rows)
__device__ __forceinline__ float4 mul4e(float4 a, float4 x) {
    return make_float4(__fmul_rn(a.x, x.x), __fmul_rn(a.y, x.y), __fmul_rn(a.z, x.z), __fmul_rn(a.w, x.w));
}

__device__ __forceinline__ float4 mul4(float a, float4 x) {
    return make_float4(__fmul_rn(a, x.x), __fmul_rn(a, x.y), __fmul_rn(a, x.z), __fmul_rn(a, x.w));
}

__device__ __forceinline__ void put_split4(uint8_t *hi_tile, uint8_t *lo_tile, uint32_t row, uint32_t k, float4 x) {
    float4 h, l;
    tc::split_tf32(x.x, h.x, l.x);
    tc::split_tf32(x.y, h.y, l.y);
    tc::split_tf32(x.z, h.z, l.z);
    tc::split_tf32(x.w, h.w, l.w);
    const uint32_t off = tc::sw128_offset(row, k);
    *reinterpret_cast<float4 *>(hi_tile + off) = h;
    *reinterpret_cast<float4 *>(lo_tile + off) = l;
}

// D (+)= A B^T over one 32-wide K slab, split operands: hi hi, hi lo, lo hi
__device__ __forceinline__ void mma_split(uint32_t d, uint32_t a_hi, uint32_t a_lo, uint32_t b_hi, uint32_t b_lo,
                                          bool accumulate) {
    const uint32_t idesc = tc::idesc_tf32(128, 128);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
        const uint32_t off = 32u * kk;
        tc::mma_tf32(d, tc::desc_k_sw128(a_hi + off), tc::desc_k_sw128(b_hi + off), idesc, accumulate || kk > 0);
        tc::mma_tf32(d, tc::desc_k_sw128(a_hi + off), tc::desc_k_sw128(b_lo + off), idesc, true);
        tc::mma_tf32(d, tc::desc_k_sw128(a_lo + off), tc::desc_k_sw128(b_hi + off), idesc, true);
    }
}

// 128 columns of this thread's tensor-memory lane, 32 at a time
template <class Fn>
__device__ __forceinline__ void tmem_row(uint32_t taddr_lane, Fn &&fn) {
#pragma unroll
    for (int c = 0; c < kChunk; c += 32) {
        float x[32];
        tc::ld32(taddr_lane + (uint32_t)c, x);
        fn(c, x);
    }
}

// the test a chunk's cumulative decays (gam_0, gam_1, ... as thread 0 forms
// them, padding gates 1) pass for the quotient form
__device__ __forceinline__ bool decay_in_range(float g) { return g >= 0x1p-100f && g <= 0x1p100f; }

// QUOT: every page, the decay from token j to token i taken as gam_i (1 /
// gam_j) with gam_i folded into q; a page with a chunk whose cumulative
// decays leave [2^-100, 2^100] is left as it was (before that chunk's first
// product; its page bytes are not written) and *A.pending is set to A.call.
// !QUOT (launched next, as a programmatic dependent launch: its CTAs may wait
// on the SMs the first leaves idle): once the first has completed, nothing
// unless *A.pending == A.call; then the pages the first launch left, each
// decay the product of the gates of tokens j + 1 .. i (defined for zero gates
// and decays below the float range).
// GV (gate vectors, KDA): QUOT only; a chunk whose per-channel cumulative
// decays leave the range runs token by token on the CUDA cores instead.
template <class FMT, bool QUOT, bool GV>
__global__ void __launch_bounds__(kTcThreads, 1) prefill_tc_kernel(const DevFormat F, const TcArgs A) {
    static_assert(QUOT || !GV, "gate vectors take the quotient form or the token recurrence");
    extern __shared__ uint8_t tc_smem_raw[];
    const uint32_t raw = smem_u32(tc_smem_raw);
    uint8_t *base = tc_smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint8_t *tiles = base;                                            // operand tiles / A / page buffer
    float *XS = reinterpret_cast<float *>(base + tile_region<GV>());  // X[v][kappa]
    TcSmall &M = *reinterpret_cast<TcSmall *>(base + tile_region<GV>() + (size_t)kD * kXStride * 4);
    float *Gs = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(&M) + sizeof(TcSmall));   // GV: [token][33]
    float *Amat = reinterpret_cast<float *>(tiles);
    const uint32_t t_base = smem_u32(tiles);
    auto tile = [&](int i) { return tiles + i * tc::kTileBytes; };
    auto tile_addr = [&](int i) { return t_base + (uint32_t)i * tc::kTileBytes; };

    if constexpr (QUOT) {
        asm volatile("griddepcontrol.launch_dependents;");
    } else {
        asm volatile("griddepcontrol.wait;" ::: "memory");   // the quotient launch has completed
        if (*reinterpret_cast<volatile const uint32_t *>(A.pending) != A.call) return;   // nothing was left
    }
    constexpr bool SR = FMT::kSr;
    bool col_scales, gate_vector;
    format_flags<FMT>(F, col_scales, gate_vector);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int t = tid & (kD - 1), hf = tid >> 7;   // row t, half hf of its columns
    const int wq = warp & 3;                        // lanes 32 wq .. + 31; slice wq of the page
    const RowCtx R = row_ctx<FMT>(F, wq, lane);

    if (tid == 0) {
        mbar_init(&M.mma_bar, 1);
        mbar_init(&M.page_bar, 1);
        mbar_init(&M.never, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tc::tmem_alloc(&M.tmem, 512);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = M.tmem;
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * wq) << 16);     // this thread's lane, column 0
    const uint32_t RG = 0, RY = 128, RP = 256, RO = 384;               // column regions

    const int n = A.n_pages, H = A.heads;
    uint32_t mma_phase = 0, page_phase = 0;
    bool failed = false;
    int pending_mma = -1, pending_page = -1;      // a phase this thread gave up on (exit path waits again)

    auto wait_mma = [&]() {
        const uint32_t ph = mma_phase;
        mma_phase ^= 1u;
        const bool ok = mbar_wait_bounded(&M.mma_bar, ph, A.wait_limit_ns);
        if (!ok) pending_mma = (int)ph;
        tc::fence_after_sync();
        return ok;
    };

    for (int p = blockIdx.x; p < n; p += gridDim.x) {
        if (!QUOT) {
            // was this page left by the quotient launch?  Its rule, replayed:
            // a chunk's gates staged in shared memory, then one thread per
            // chunk forms the cumulative decays in the same order
            float *gst = reinterpret_cast<float *>(tiles);
            bool left = false;
            for (int base = 0; base < A.L; base += kTcThreads) {
                const int i = base + tid;
                gst[tid] = i < A.L ? __ldg(A.alpha + (size_t)i * n + p) : 1.f;
                __syncthreads();
                if (tid < 2 && base + kChunk * tid < A.L) {
                    float g = 1.f;
                    for (int k = 0; k < kChunk; ++k) {
                        g = __fmul_rn(g, gst[kChunk * tid + k]);
                        left = left || !decay_in_range(g);
                    }
                }
                __syncthreads();
            }
            fence_proxy_async_smem();   // the staging writes before the page's bulk copy
            if (!__syncthreads_or(left)) continue;
        }
        const int ph = p % H, pb = p / H;
        // ---- the page: bulk copy into the tile region, dequantize into X
        if (tid == 0) {
            mbar_expect_tx(&M.page_bar, (uint32_t)F.page_bytes);
            bulk_g2s(tiles, A.pages + (size_t)p * F.page_bytes, (uint32_t)F.page_bytes, &M.page_bar);
        }
        if (tid < kD) M.kap[tid] = A.perm[(size_t)ph * kD + tid] & (kD - 1);
        bool ok;
        const uint32_t pp = page_phase;
        page_phase ^= 1u;
        if (A.stall_first_wait && p == (int)blockIdx.x) ok = mbar_wait_bounded(&M.never, 0, A.wait_limit_ns);
        else ok = mbar_wait_bounded(&M.page_bar, pp, A.wait_limit_ns);
        if (!ok) pending_page = (int)pp;
        if (tid < kD) {
            const float c = col_scales ? reinterpret_cast<const float *>(tiles + F.c_off)[tid] : 1.f;
            M.c[tid] = c;
            M.ic[tid] = col_scales ? __frcp_rn(c) : 1.f;
        }
        if (__syncthreads_or(!ok)) { failed = true; break; }
        {
            // warp w dequantizes slice w % 4 (rows 16 b + 4 (w % 4) + i) of
            // blocks 4 (w / 4) .. + 3: T = z r (FP16 rows: h), written to
            // X[v][kappa]
            const float *r_s = reinterpret_cast<const float *>(tiles + F.r_off);
            static_for<0, kBlocks>([&](auto bc) {
                constexpr int b = decltype(bc)::value;
                if ((b >> 2) != hf) return;
                float av[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int blk_r = (R.all_int || F.blk_kind(b) == kKindInt) ? F.blk_rbase(b) + 4 * wq + i : -1;
                    av[i] = blk_r >= 0 ? r_s[blk_r] : 1.f;
                }
                Tile T;
                const uint8_t *blk = tiles + fmt_offset<FMT, b>(F);
                with_width<FMT, b>(F, [&](auto wc) {
                    constexpr int W = decltype(wc)::value;
                    dequant_slice<W, b>(blk, wq, lane, make_float4(av[0], av[1], av[2], av[3]), T);
                });
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int kap = M.kap[16 * b + 4 * wq + i];
                    XS[(4 * lane + 0) * kXStride + kap] = T[b][i][0].x;
                    XS[(4 * lane + 1) * kXStride + kap] = T[b][i][0].y;
                    XS[(4 * lane + 2) * kXStride + kap] = T[b][i][1].x;
                    XS[(4 * lane + 3) * kXStride + kap] = T[b][i][1].y;
                }
            });
        }
        __syncthreads();

        bool leave = false;   // the quotient launch leaves this page to the product launch
        // Gate vectors, a chunk whose per-channel decays leave the range: the
        // delta rule token by token on the CUDA cores, in the state's own
        // units (X = S^T / c).  Thread (v, hf) holds X[v][64 hf .. + 63] in
        // registers; each token: decay, prediction u = X k, e = beta (v / c -
        // u), update X += e k^T, readout o = c X q, the halves' partial sums
        // through shared memory.  The next token's vectors are staged while
        // this one runs.
        auto gv_tokens = [&](int t0, int cn) {
            auto stage = [&](int i, int b) {
                if (tid < kD) {
                    const size_t row = ((size_t)(t0 + i) * n + p) * kD + tid;
                    M.tok[b][0][tid] = __ldg(A.k + row);
                    M.tok[b][1][tid] = __ldg(A.q + row);
                    M.tok[b][2][tid] = __ldg(A.alpha + row);
                    M.tok[b][3][tid] = __fmul_rn(__ldg(A.v + row), M.ic[tid]);
                }
            };
            float x[64];
            const float *xr = XS + t * kXStride + 64 * hf;
#pragma unroll
            for (int c = 0; c < 64; ++c) x[c] = xr[c];
            stage(0, 0);
            __syncthreads();
            for (int i = 0; i < cn; ++i) {
                const int b = i & 1;
                if (i + 1 < cn) stage(i + 1, b ^ 1);   // read after the next token's first barrier
                const float *kb = &M.tok[b][0][64 * hf], *qb = &M.tok[b][1][64 * hf], *ab = &M.tok[b][2][64 * hf];
                float u = 0.f;
#pragma unroll
                for (int c = 0; c < 64; c += 4) {
                    const float4 a4 = *reinterpret_cast<const float4 *>(ab + c);
                    const float4 k4 = *reinterpret_cast<const float4 *>(kb + c);
                    x[c] = __fmul_rn(x[c], a4.x);
                    x[c + 1] = __fmul_rn(x[c + 1], a4.y);
                    x[c + 2] = __fmul_rn(x[c + 2], a4.z);
                    x[c + 3] = __fmul_rn(x[c + 3], a4.w);
                    u = __fmaf_rn(k4.x, x[c], u);
                    u = __fmaf_rn(k4.y, x[c + 1], u);
                    u = __fmaf_rn(k4.z, x[c + 2], u);
                    u = __fmaf_rn(k4.w, x[c + 3], u);
                }
                M.red[0][hf][t] = u;
                __syncthreads();
                const float e = __fmul_rn(M.bet[i], __fsub_rn(M.tok[b][3][t], __fadd_rn(M.red[0][0][t], M.red[0][1][t])));
                float o = 0.f;
#pragma unroll
                for (int c = 0; c < 64; c += 4) {
                    const float4 k4 = *reinterpret_cast<const float4 *>(kb + c);
                    const float4 q4 = *reinterpret_cast<const float4 *>(qb + c);
                    x[c] = __fmaf_rn(k4.x, e, x[c]);
                    x[c + 1] = __fmaf_rn(k4.y, e, x[c + 1]);
                    x[c + 2] = __fmaf_rn(k4.z, e, x[c + 2]);
                    x[c + 3] = __fmaf_rn(k4.w, e, x[c + 3]);
                    o = __fmaf_rn(q4.x, x[c], o);
                    o = __fmaf_rn(q4.y, x[c + 1], o);
                    o = __fmaf_rn(q4.z, x[c + 2], o);
                    o = __fmaf_rn(q4.w, x[c + 3], o);
                }
                M.red[1][hf][t] = o;
                __syncthreads();
                if (hf == 0)
                    A.o[((size_t)(t0 + i) * n + p) * kD + t] =
                        __fmul_rn(M.c[t], __fadd_rn(M.red[1][0][t], M.red[1][1][t]));
            }
            float *xw = XS + t * kXStride + 64 * hf;
#pragma unroll
            for (int c = 0; c < 64; ++c) xw[c] = x[c];
            __syncthreads();   // X is whole again before the next chunk
        };
        for (int t0 = 0; t0 < A.L && !failed; t0 += kChunk) {
            const int cn = min(kChunk, A.L - t0);
            // ---- per-token scalars of the chunk
            if (tid < kChunk) {
                const bool real = tid < cn;
                const size_t row = (size_t)(t0 + tid) * n + p;
                M.bet[tid] = real ? A.beta[row] : 0.f;
                if constexpr (!GV) M.al[tid] = real ? A.alpha[row] : 1.f;
            }
            if constexpr (GV) {
                // (the decays are staged, and their range tested, per slab in
                // phase A; a chunk out of range switches to gv_tokens there)
            } else {
                __syncthreads();
                if (tid == 0) {
                    float g = 1.f;
                    bool in_range = true;
                    for (int i = 0; i < kChunk; ++i) {
                        g = __fmul_rn(g, M.al[i]);
                        M.gam[i] = g;
                        in_range = in_range && decay_in_range(g);
                    }
                    M.in_range = in_range ? 1 : 0;
                }
                __syncthreads();
                if (QUOT && M.in_range == 0) {   // for the product launch
                    leave = true;
                    break;
                }
            }
            bool gv_fallback = false;   // gate vectors: this chunk's decays left the range
            auto chunk_body = [&]() {
                constexpr bool quot = QUOT;
                if constexpr (GV) {
                    // (the decays come per slab below)
                } else if (quot) {
                    if (tid < kChunk) {
                        const float gi = M.gam[tid];
                        M.igam[tid] = __frcp_rn(gi);
                        M.kts[tid] = __fdiv_rn(M.gam[kChunk - 1], gi);
                    }
                } else if (tid == 32) {
                    float g = 1.f;
                    M.kts[kChunk - 1] = g;
                    for (int j = kChunk - 2; j >= 0; --j) {
                        g = __fmul_rn(g, M.al[j + 1]);
                        M.kts[j] = g;
                    }
                }
                __syncthreads();

                // ---- phase A: G = K K^T, Y^T = X K^T, P = (gam Q) K^T and
                // O^T = X (gam Q)^T (gam = 1 here for a chunk of products)
                // row t of the K and Q slabs, columns 16 hf .. + 15: the next slab's
                // are loaded while the tensor cores work on this one
                float4 kx[4], qx[4];
                auto load_kq = [&](int ks) {
                    const bool real = t < cn;
                    const size_t row = ((size_t)(t0 + t) * n + p) * kD + 32 * ks + 16 * hf;
#pragma unroll
                    for (int j4 = 0; j4 < 4; ++j4) {
                        kx[j4] = qx[j4] = make_float4(0.f, 0.f, 0.f, 0.f);
                        if (real) {
                            kx[j4] = __ldg(reinterpret_cast<const float4 *>(A.k + row) + j4);
                            qx[j4] = __ldg(reinterpret_cast<const float4 *>(A.q + row) + j4);
                        }
                    }
                };
                // gate vectors: the decays Gam[token][channel] of one slab's 32
                // channels staged in Gs; warp s takes tokens 16 s .. + 15 of
                // channel 32 ks + lane (segment products, then their prefixes)
                // Returns (CTA-wide) whether every gate lies in [0, 1] and every
                // decay it formed in [2^-100, 2^100] (so 1 / Gam is finite and
                // the decays to the chunk's end, products of gates, are at
                // most 1); the last segment's warp records those decays.
                auto stage_gam = [&](int ks) -> bool {
                    float av[16];
                    float pr = 1.f;
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int tk = 16 * warp + i;
                        av[i] = tk < cn ? __ldg(A.alpha + ((size_t)(t0 + tk) * n + p) * kD + 32 * ks + lane) : 1.f;
                        pr = __fmul_rn(pr, av[i]);
                    }
                    M.segp[warp][lane] = pr;
                    __syncthreads();
                    float g = 1.f;
                    for (int s2 = 0; s2 < warp; ++s2) g = __fmul_rn(g, M.segp[s2][lane]);
                    bool in_range = true;   // a NaN fails the test too
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        g = __fmul_rn(g, av[i]);
                        in_range = in_range && av[i] >= 0.f && av[i] <= 1.f && decay_in_range(g);
                        Gs[(16 * warp + i) * kGsStride + lane] = g;
                    }
                    if (warp == kTcThreads / 32 - 1) M.gn[32 * ks + lane] = g;
                    return __syncthreads_and(in_range) != 0;
                };
                load_kq(0);
                bool gam_ok = true;
                if constexpr (GV) {
                    if (!stage_gam(0)) {
                        gv_fallback = true;   // before any product of the chunk
                        return;
                    }
                }
                for (int ks = 0; ks < kD / 32; ++ks) {
                    if constexpr (GV) {
                        // row t of the K Gam, Q Gam, X and K / Gam slabs, columns 16 hf .. + 15
                        const float *xr = XS + t * kXStride + 32 * ks;
                        const float *gr = Gs + t * kGsStride;
#pragma unroll
                        for (int j4 = 0; j4 < 4; ++j4) {
                            const int j = 16 * hf + 4 * j4;
                            const float4 g4 = make_float4(gr[j], gr[j + 1], gr[j + 2], gr[j + 3]);
                            const float4 ig4 = make_float4(__frcp_rn(g4.x), __frcp_rn(g4.y), __frcp_rn(g4.z), __frcp_rn(g4.w));
                            put_split4(tile(0), tile(1), t, j, mul4e(kx[j4], g4));
                            put_split4(tile(2), tile(3), t, j, mul4e(qx[j4], g4));
                            put_split4(tile(4), tile(5), t, j, make_float4(xr[j], xr[j + 1], xr[j + 2], xr[j + 3]));
                            put_split4(tile(6), tile(7), t, j, mul4e(kx[j4], ig4));
                        }
                    } else {
                        // row t of the K, gam Q and X slabs, columns 16 hf .. + 15
                        const float gi = quot ? M.gam[t] : 1.f;
                        const float *xr = XS + t * kXStride + 32 * ks;
#pragma unroll
                        for (int j4 = 0; j4 < 4; ++j4) {
                            const int j = 16 * hf + 4 * j4;
                            put_split4(tile(0), tile(1), t, j, kx[j4]);
                            put_split4(tile(2), tile(3), t, j, quot ? mul4(gi, qx[j4]) : qx[j4]);
                            put_split4(tile(4), tile(5), t, j, make_float4(xr[j], xr[j + 1], xr[j + 2], xr[j + 3]));
                        }
                    }
                    fence_proxy_async_smem();
                    tc::fence_before_sync();
                    __syncthreads();
                    tc::fence_after_sync();
                    if (tid == 0) {
                        const bool acc = ks > 0;
                        if constexpr (GV) {
                            // G = (K Gam)(K / Gam)^T, Y^T = X (K Gam)^T, P = (Q Gam)(K / Gam)^T, O^T = X (Q Gam)^T
                            mma_split(tmem + RG, tile_addr(0), tile_addr(1), tile_addr(6), tile_addr(7), acc);
                            mma_split(tmem + RY, tile_addr(4), tile_addr(5), tile_addr(0), tile_addr(1), acc);
                            mma_split(tmem + RP, tile_addr(2), tile_addr(3), tile_addr(6), tile_addr(7), acc);
                            mma_split(tmem + RO, tile_addr(4), tile_addr(5), tile_addr(2), tile_addr(3), acc);
                        } else {
                            mma_split(tmem + RG, tile_addr(0), tile_addr(1), tile_addr(0), tile_addr(1), acc);
                            mma_split(tmem + RY, tile_addr(4), tile_addr(5), tile_addr(0), tile_addr(1), acc);
                            mma_split(tmem + RP, tile_addr(2), tile_addr(3), tile_addr(0), tile_addr(1), acc);
                            mma_split(tmem + RO, tile_addr(4), tile_addr(5), tile_addr(2), tile_addr(3), acc);
                        }
                        tc::commit(&M.mma_bar);
                    }
                    if (ks + 1 < kD / 32) load_kq(ks + 1);
                    if constexpr (GV) {
                        if (ks + 1 < kD / 32) gam_ok = stage_gam(ks + 1);   // Gs is free: this slab's tiles are written
                    }
                    if (__syncthreads_or(!wait_mma())) { failed = true; break; }
                    if (GV && !gam_ok) {
                        gv_fallback = true;   // the products so far wrote only tensor memory
                        return;
                    }
                }
                if (failed) return;

                // ---- phase B: R from Y^T in place (thread v), then the solve
                // (I + A) E = R in two halves of 64 tokens: each half by forward
                // substitution with thread v holding column v of the half in
                // registers; between them the off-diagonal block, R2 -= A21 E1,
                // as a tensor-core product.  E^T ends up in Y^T's columns.
                {
                    // column t of R, tokens 64 hf .. + 63; in a chunk of products
                    // the same columns of O^T get their token's decay (o_i's first
                    // part is gam_i S0^T q_i)
                    const float icv = M.ic[t];
                    const uint32_t ry = lane_addr + RY, ro = lane_addr + RO;
#pragma unroll
                    for (int c0 = 64 * hf; c0 < 64 * hf + 64; c0 += 32) {
                        float x[32];
                        tc::ld32(ry + c0, x);
#pragma unroll
                        for (int jj = 0; jj < 32; ++jj) {
                            const int i = c0 + jj;
                            const float vv = (i < cn) ? __ldg(A.v + ((size_t)(t0 + i) * n + p) * kD + t) : 0.f;
                            // R_i = beta_i (v_i / c - gam_i y_i) (gate vectors: the decay is in y)
                            const float gy = GV ? x[jj] : __fmul_rn(M.gam[i], x[jj]);
                            x[jj] = __fmul_rn(M.bet[i], __fsub_rn(__fmul_rn(vv, icv), gy));
                        }
                        tc::st32(ry + c0, x);
                        if (!quot) {
                            tc::ld32(ro + c0, x);
#pragma unroll
                            for (int jj = 0; jj < 32; ++jj) x[jj] = __fmul_rn(M.gam[c0 + jj], x[jj]);
                            tc::st32(ro + c0, x);
                        }
                    }
                }
                for (int sb = 0; sb < 2; ++sb) {
                    // the diagonal block of this half: A_ij, i, j in [64 sb, 64 sb + 64)
                    // (row t, columns 32 hf .. + 31 of the block).  rho = the decay
                    // from token j to t, walked down from j = t: rho_{t,j-1} =
                    // rho_{t,j} al_j
                    if (t >= 64 * sb && t < 64 * sb + 64) {
                        const float bi = M.bet[t];
                        float *arow = Amat + (t - 64 * sb) * kAStride;
                        const int c0 = 32 * hf;
                        const int jlo = 64 * sb + c0;
                        float x[32];
                        tc::ld32(lane_addr + RG + jlo, x);
                        float a[32];
                        if constexpr (GV) {
#pragma unroll
                            for (int jj = 0; jj < 32; ++jj) a[jj] = jlo + jj < t ? __fmul_rn(bi, x[jj]) : 0.f;
                        } else if (quot) {
                            const float gi = M.gam[t];
#pragma unroll
                            for (int jj = 0; jj < 32; ++jj) {
                                const int j = jlo + jj;
                                a[jj] = j < t ? __fmul_rn(bi, __fmul_rn(__fmul_rn(gi, M.igam[j]), x[jj])) : 0.f;
                            }
                        } else {
                            float rho = 1.f;   // rho_{t, jlo+31} when t is above the columns: the gates jlo+32 .. t
#pragma unroll
                            for (int d = 0; d < 32; ++d)
                                if (jlo + 32 + d <= t) rho = __fmul_rn(rho, M.al[jlo + 32 + d]);
#pragma unroll
                            for (int jj = 31; jj >= 0; --jj) {
                                const int j = jlo + jj;
                                a[jj] = j < t ? __fmul_rn(bi, __fmul_rn(rho, x[jj])) : 0.f;
                                if (j <= t) rho = __fmul_rn(rho, M.al[j]);
                            }
                        }
#pragma unroll
                        for (int u = 0; u < 8; ++u)
                            *reinterpret_cast<float4 *>(arow + c0 + 4 * u) =
                                make_float4(a[4 * u], a[4 * u + 1], a[4 * u + 2], a[4 * u + 3]);
                    }
                    __syncthreads();
                    float e[64];   // the first half's threads: column t of this half of E
                    if (hf == 0) {
                        {
                            float x[32];
                            tc::ld32(lane_addr + RY + 64 * sb, x);
#pragma unroll
                            for (int jj = 0; jj < 32; ++jj) e[jj] = x[jj];
                            tc::ld32(lane_addr + RY + 64 * sb + 32, x);
#pragma unroll
                            for (int jj = 0; jj < 32; ++jj) e[32 + jj] = x[jj];
                        }
                        // forward substitution: E_i = R_i - sum_{j<i} A_ij E_j
#pragma unroll
                        for (int i = 1; i < 64; ++i) {
                            const float *arow = Amat + i * kAStride;
                            float acc = e[i];
#pragma unroll
                            for (int j4 = 0; j4 < (i + 3) / 4; ++j4) {
                                const float4 a4 = *reinterpret_cast<const float4 *>(arow + 4 * j4);
                                const float av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
                                for (int jj = 0; jj < 4; ++jj)
                                    if (4 * j4 + jj < i) acc = __fmaf_rn(-av[jj], e[4 * j4 + jj], acc);
                            }
                            e[i] = acc;
                        }
                        {
                            float x[32];
#pragma unroll
                            for (int jj = 0; jj < 32; ++jj) x[jj] = e[jj];
                            tc::st32(lane_addr + RY + 64 * sb, x);
#pragma unroll
                            for (int jj = 0; jj < 32; ++jj) x[jj] = e[32 + jj];
                            tc::st32(lane_addr + RY + 64 * sb + 32, x);
                        }
                    }
                    if (sb == 1) break;
                    __syncthreads();   // the diagonal block's space becomes operand tiles
                    // R2 -= A21 E1 on the tensor cores: D = R2^T (columns 64..127 of
                    // Y^T) += (-E1^T) A21^T, M = 128 (v), N = 64 (i), K = 64 (j).
                    // Tiles: E1^T hi / lo (rows v, two K slabs) at 0 .. 64 KB, written
                    // by the first half from its columns of E; A21 hi / lo (rows
                    // i - 64, 64-row tiles of 8 KB) at 64 .. 96 KB, by the second.
                    if (hf == 0) {
#pragma unroll
                        for (int kb = 0; kb < 2; ++kb) {
#pragma unroll
                            for (int u = 0; u < 8; ++u) {
                                const int j = 32 * kb + 4 * u;
                                put_split4(tile(2 * kb), tile(2 * kb + 1), t, 4 * u,
                                           make_float4(e[j], e[j + 1], e[j + 2], e[j + 3]));
                            }
                        }
                    } else if (t >= 64) {
                        // rho walked down from j = t to the block's columns 63 .. 0
                        const float bi = M.bet[t];
                        uint8_t *a21 = tiles + 4 * tc::kTileBytes;
                        const float gi = GV ? 1.f : M.gam[t];
                        float rho = 1.f;   // rho_{t, 63}: the gates 64 .. t
                        if (!quot) {
#pragma unroll
                            for (int d = 0; d < 64; ++d)
                                if (64 + d <= t) rho = __fmul_rn(rho, M.al[64 + d]);
                        }
#pragma unroll
                        for (int kb = 1; kb >= 0; --kb) {
                            float x[32];
                            tc::ld32(lane_addr + RG + 32 * kb, x);
                            float a[32];
                            if constexpr (GV) {
#pragma unroll
                                for (int jj = 0; jj < 32; ++jj) a[jj] = __fmul_rn(bi, x[jj]);
                            } else if (quot) {
#pragma unroll
                                for (int jj = 0; jj < 32; ++jj)
                                    a[jj] = __fmul_rn(bi, __fmul_rn(__fmul_rn(gi, M.igam[32 * kb + jj]), x[jj]));
                            } else {
#pragma unroll
                                for (int jj = 31; jj >= 0; --jj) {
                                    const int j = 32 * kb + jj;
                                    a[jj] = __fmul_rn(bi, __fmul_rn(rho, x[jj]));
                                    rho = __fmul_rn(rho, M.al[j]);
                                }
                            }
#pragma unroll
                            for (int u = 0; u < 8; ++u)
                                put_split4(a21 + (2 * kb) * (tc::kTileBytes / 2), a21 + (2 * kb + 1) * (tc::kTileBytes / 2),
                                           t - 64, 4 * u, make_float4(a[4 * u], a[4 * u + 1], a[4 * u + 2], a[4 * u + 3]));
                        }
                    }
                    fence_proxy_async_smem();
                    tc::fence_before_sync();
                    __syncthreads();
                    tc::fence_after_sync();
                    if (tid == 0) {
                        const uint32_t idesc = tc::idesc_tf32(128, 64, true);
                        const uint32_t a21 = tile_addr(4);
#pragma unroll
                        for (int kb = 0; kb < 2; ++kb) {
                            const uint32_t e_hi = tile_addr(2 * kb), e_lo = tile_addr(2 * kb + 1);
                            const uint32_t b_hi = a21 + (2 * kb) * (tc::kTileBytes / 2);
                            const uint32_t b_lo = a21 + (2 * kb + 1) * (tc::kTileBytes / 2);
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk) {
                                const uint32_t off = 32u * kk;
                                tc::mma_tf32(tmem + RY + 64, tc::desc_k_sw128(e_hi + off), tc::desc_k_sw128(b_hi + off),
                                             idesc, true);
                                tc::mma_tf32(tmem + RY + 64, tc::desc_k_sw128(e_hi + off), tc::desc_k_sw128(b_lo + off),
                                             idesc, true);
                                tc::mma_tf32(tmem + RY + 64, tc::desc_k_sw128(e_lo + off), tc::desc_k_sw128(b_hi + off),
                                             idesc, true);
                            }
                        }
                        tc::commit(&M.mma_bar);
                    }
                    if (__syncthreads_or(!wait_mma())) { failed = true; break; }
                }
                if (failed) return;
                // the solve's space becomes operand tiles again; E^T (stored by the
                // first half) is read by both halves
                tc::fence_before_sync();
                __syncthreads();
                tc::fence_after_sync();

                // ---- phase C: O^T += E^T P~^T, dX = E^T K~ (K = tokens); in a
                // chunk of products the token slabs go from the last to the first,
                // so that each thread walks the decay rho_{t,j} down from j = t.
                // k of key channel t, tokens 32 js + 16 hf .. + 15: the next
                // slab's loaded while the tensor cores work on this one
                float kk[16];
                auto load_kt = [&](int js) {
#pragma unroll
                    for (int jj = 0; jj < 16; ++jj) {
                        const int j = 32 * js + 16 * hf + jj;
                        kk[jj] = (j < cn) ? __ldg(A.k + ((size_t)(t0 + j) * n + p) * kD + t) : 0.f;
                    }
                };
                // slab order: ascending for quotients, descending for products
                constexpr int kSlabs = kChunk / 32;
                // (gate vectors: descending too, a key's decay to the chunk's end
                // being the product of the gates after it)
                auto slab = [&](int n_done) { return (quot && !GV) ? n_done : kSlabs - 1 - n_done; };
                load_kt(slab(0));
                float rho = 1.f;   // rho_{t, j} for the next j below the columns done
                float gk = 1.f;    // gate vectors: channel t's gates after the next token down
                for (int sdone = 0; sdone < kSlabs; ++sdone) {
                    const int js = slab(sdone);
                    {
                        // columns 16 hf .. + 15 of the slab
                        const int c0 = 16 * hf;
                        // E^T row v (thread v), from Y^T's columns
                        float x[16];
                        tc::ld16(lane_addr + RY + 32 * js + c0, x);
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            put_split4(tile(0), tile(1), t, c0 + 4 * u,
                                       make_float4(x[4 * u], x[4 * u + 1], x[4 * u + 2], x[4 * u + 3]));
                        // P~ row i (thread i), j <= i (else 0): P_ij / gam_j, or in a
                        // chunk of products rho_ij P_ij, rho running through the
                        // other half's columns of the slab too
                        tc::ld16(lane_addr + RP + 32 * js + c0, x);
                        float pv[16];
                        if constexpr (GV) {
#pragma unroll
                            for (int e = 0; e < 16; ++e) pv[e] = 32 * js + c0 + e <= t ? x[e] : 0.f;
                        } else if (quot) {
#pragma unroll
                            for (int e = 0; e < 16; ++e) {
                                const int j = 32 * js + c0 + e;
                                pv[e] = j <= t ? __fmul_rn(x[e], M.igam[j]) : 0.f;
                            }
                        } else {
#pragma unroll
                            for (int e = 0; e < 16; ++e) pv[e] = 0.f;
#pragma unroll
                            for (int part = 1; part >= 0; --part) {
#pragma unroll
                                for (int e = 15; e >= 0; --e) {
                                    const int j = 32 * js + 16 * part + e;
                                    if (part == hf && j <= t) pv[e] = __fmul_rn(rho, x[e]);
                                    if (j <= t) rho = __fmul_rn(rho, M.al[j]);
                                }
                            }
                        }
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            put_split4(tile(2), tile(3), t, c0 + 4 * u,
                                       make_float4(pv[4 * u], pv[4 * u + 1], pv[4 * u + 2], pv[4 * u + 3]));
                        // K~^T row kappa (thread kappa): k_j[kappa] times the decay of
                        // token j to the chunk's end (gate vectors: Gam_n / Gam_j of
                        // channel kappa, Gam walked through the slab's tokens)
                        if constexpr (GV) {
                            // the slab's gates of every channel, [32 tokens][128] in
                            // tile 6 (free in this phase): thread (t, hf) loads
                            // channel t of tokens 16 hf .. + 15 in one batch
                            float *ga = reinterpret_cast<float *>(tile(6));
                            {
                                float av[16];
#pragma unroll
                                for (int e = 0; e < 16; ++e) {
                                    const int j = 32 * js + 16 * hf + e;
                                    av[e] = j < cn ? __ldg(A.alpha + ((size_t)(t0 + j) * n + p) * kD + t) : 1.f;
                                }
#pragma unroll
                                for (int e = 0; e < 16; ++e) ga[(16 * hf + e) * kD + t] = av[e];
                            }
                            __syncthreads();
                            // Gam_n / Gam_j = the gates of tokens j + 1 .. n - 1, walked
                            // down (padding gates are 1)
                            float rt[16];
#pragma unroll
                            for (int e = 0; e < 16; ++e) rt[e] = 0.f;
#pragma unroll
                            for (int part = 1; part >= 0; --part) {
#pragma unroll
                                for (int e = 15; e >= 0; --e) {
                                    if (part == hf) rt[e] = gk;
                                    gk = __fmul_rn(gk, ga[(16 * part + e) * kD + t]);
                                }
                            }
#pragma unroll
                            for (int u = 0; u < 4; ++u)
                                put_split4(tile(4), tile(5), t, c0 + 4 * u,
                                           make_float4(__fmul_rn(kk[4 * u], rt[4 * u]), __fmul_rn(kk[4 * u + 1], rt[4 * u + 1]),
                                                       __fmul_rn(kk[4 * u + 2], rt[4 * u + 2]),
                                                       __fmul_rn(kk[4 * u + 3], rt[4 * u + 3])));
                        } else {
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                const float *kt = M.kts + 32 * js + c0 + 4 * u;
                                put_split4(tile(4), tile(5), t, c0 + 4 * u,
                                           make_float4(__fmul_rn(kk[4 * u], kt[0]), __fmul_rn(kk[4 * u + 1], kt[1]),
                                                       __fmul_rn(kk[4 * u + 2], kt[2]), __fmul_rn(kk[4 * u + 3], kt[3])));
                            }
                        }
                    }
                    fence_proxy_async_smem();
                    tc::fence_before_sync();
                    __syncthreads();
                    tc::fence_after_sync();
                    if (tid == 0) {
                        mma_split(tmem + RO, tile_addr(0), tile_addr(1), tile_addr(2), tile_addr(3), true);
                        mma_split(tmem + RG, tile_addr(0), tile_addr(1), tile_addr(4), tile_addr(5), sdone > 0);
                        tc::commit(&M.mma_bar);
                    }
                    if (sdone + 1 < kSlabs) load_kt(slab(sdone + 1));
                    if (__syncthreads_or(!wait_mma())) { failed = true; break; }
                }
                if (failed) return;

                // ---- phase D: o of the chunk's tokens; X <- gam_n X + dX
                {
                    // column t: tokens (o) and key channels (X) 64 hf .. + 63
                    const float cv = M.c[t];
#pragma unroll
                    for (int c0 = 64 * hf; c0 < 64 * hf + 64; c0 += 32) {
                        float x[32];
                        tc::ld32(lane_addr + RO + c0, x);
#pragma unroll
                        for (int jj = 0; jj < 32; ++jj) {
                            const int i = c0 + jj;
                            if (i < cn) A.o[((size_t)(t0 + i) * n + p) * kD + t] = __fmul_rn(cv, x[jj]);
                        }
                    }
                    const float gn = M.gam[kChunk - 1];
                    float *xr = XS + t * kXStride;
#pragma unroll
                    for (int c0 = 64 * hf; c0 < 64 * hf + 64; c0 += 32) {
                        float x[32];
                        tc::ld32(lane_addr + RG + c0, x);
#pragma unroll
                        for (int jj = 0; jj < 32; ++jj)
                        xr[c0 + jj] = __fmaf_rn(GV ? M.gn[c0 + jj] : gn, xr[c0 + jj], x[jj]);
                    }
                }
                tc::fence_before_sync();
                __syncthreads();
                tc::fence_after_sync();
            };
            chunk_body();
            if (GV && gv_fallback && !failed) gv_tokens(t0, cn);   // this chunk token by token
        }
        if (failed) break;
        if (QUOT && leave) {
            // nothing of the page is stored (o of its earlier chunks is
            // written again by the product launch)
            if (tid == 0) *reinterpret_cast<volatile uint32_t *>(A.pending) = A.call;
            fence_proxy_async_smem();   // the tiles' generic writes before the next bulk copy
            __syncthreads();
            continue;
        }

        // ---- the page's end: the state (optional), one requantization, the store
        if (A.S_out) {
            const float cv = M.c[t];
            const float *xr = XS + t * kXStride;
            for (int kap = 64 * hf; kap < 64 * hf + 64; ++kap)
                A.S_out[((size_t)p * kD + kap) * kD + t] = __fmul_rn(xr[kap], cv);
        }
        // the page buffer starts from zero (the 1-bit plane's words are
        // updated by xor of each slice's bits)
        for (int i = tid; i < (int)(F.page_bytes / 16); i += kTcThreads)
            reinterpret_cast<uint4 *>(tiles)[i] = make_uint4(0u, 0u, 0u, 0u);
        __syncthreads();   // the buffer is zero before any slice packs into it
        // warp w: slice w % 4 of blocks 4 (w / 4) .. + 3, as at the page's
        // start; its lanes 0 .. 15 finish those blocks' 16 rows (row maxima
        // in M.inv[w % 4][4 b + i])
        SrCtx sr;
        sr.k0 = A.seed_lo; sr.k1 = A.seed_hi; sr.step = A.step;
        sr.b = (uint32_t)pb;
        sr.h = (uint32_t)ph;
        if constexpr (SR) sr.fix();
        auto finish_half = [&](auto hc) {
            constexpr int H = decltype(hc)::value;
            Tile T;
            static_for<4 * H, 4 * H + 4>([&](auto bc) {
                constexpr int b = decltype(bc)::value;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int kap = M.kap[16 * b + 4 * wq + i];
                    T[b][i][0] = make_float2(XS[(4 * lane + 0) * kXStride + kap], XS[(4 * lane + 1) * kXStride + kap]);
                    T[b][i][1] = make_float2(XS[(4 * lane + 2) * kXStride + kap], XS[(4 * lane + 3) * kXStride + kap]);
                    M.inv[wq][4 * b + i] = warp_absmax(absmax4(T[b][i][0], T[b][i][1]));
                }
            });
            __syncwarp();
            if (lane < 16) {
                const int vl = 16 * H + lane;   // row vl of the slice: block vl / 4, row vl % 4
                const RowCtx Rv = row_ctx<FMT>(F, wq, vl);
                float *r_s = reinterpret_cast<float *>(tiles + F.r_off);
                const float m = M.inv[wq][vl];
                float inv = 0.f;
                if (Rv.all_int || Rv.is_int) {
                    const float r = div_by_qmax(m, Rv.qmax, Rv.rcp_qmax);
                    inv = m > 0.f ? div_rz_qmax<false>(Rv.qmax, m) : 0.f;
                    r_s[Rv.rix] = r;
                }
                M.inv[wq][vl] = inv;
            }
            __syncwarp();
            static_for<4 * H, 4 * H + 4>([&](auto bc) {
                constexpr int b = decltype(bc)::value;
                const float4 i4 = *reinterpret_cast<const float4 *>(&M.inv[wq][4 * b]);
                uint8_t *blk = tiles + fmt_offset<FMT, b>(F);
                with_width<FMT, b>(F, [&](auto wc) {
                    constexpr int W = decltype(wc)::value;
                    requant_slice<W, b, SR>(blk, wq, lane, i4, T, sr);
                });
            });
        };
        if (hf == 0) finish_half(IC<0>{});
        else finish_half(IC<1>{});
        fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) {
            bulk_s2g(A.pages + (size_t)p * F.page_bytes, tiles, A.store_bytes);
            bulk_commit();
            bulk_wait<0>();
        }
        __syncthreads();
    }
    if (failed && tid == 0) {
        atomicOr(A.status, kStatusTimeout);
        // the MMAs or the page copy still outstanding get a second bounded
        // wait before the tensor memory is released and the CTA exits
        if (pending_mma >= 0) mbar_wait_bounded(&M.mma_bar, (uint32_t)pending_mma, A.wait_limit_ns);
        if (pending_page >= 0) mbar_wait_bounded(&M.page_bar, (uint32_t)pending_page, A.wait_limit_ns);
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 0) tc::tmem_dealloc(tmem, 512);
}

template <class FMT, bool QUOT, bool GV>
static cudaError_t launch_prefill_tc_form(const DevFormat &F, const TcArgs &A, cudaStream_t stream) {
    const void *fn = (const void *)prefill_tc_kernel<FMT, QUOT, GV>;
    constexpr size_t smem = tc_smem<GV>();
    cudaError_t err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    const int grid = persistent_grid(fn, kTcThreads, smem, A.n_pages);
    if (grid <= 0) return cudaErrorInvalidConfiguration;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kTcThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = QUOT ? 0 : 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, prefill_tc_kernel<FMT, QUOT, GV>, F, A);
}

// the quotient form on every page it can take, then the pages it left (the
// second launch returns at once when there are none)
template <class FMT>
static cudaError_t launch_prefill_tc_scalar(const DevFormat &F, const TcArgs &A, cudaStream_t stream) {
    cudaError_t err = launch_prefill_tc_form<FMT, true, false>(F, A, stream);
    if (err != cudaSuccess) return err;
    return launch_prefill_tc_form<FMT, false, false>(F, A, stream);
}

// gate vectors: one launch (the token recurrence takes the chunks out of range)
template <class FMT>
static cudaError_t launch_prefill_tc_with(const DevFormat &F, const TcArgs &A, cudaStream_t stream) {
    if constexpr (FMT::kRuntime) {
        if (F.gate_vector) return launch_prefill_tc_form<FMT, true, true>(F, A, stream);
        return launch_prefill_tc_scalar<FMT>(F, A, stream);
    } else if constexpr (FMT::kGvec) {
        return launch_prefill_tc_form<FMT, true, true>(F, A, stream);
    } else {
        return launch_prefill_tc_scalar<FMT>(F, A, stream);
    }
}

cudaError_t launch_prefill_tc(const stq_state *s, int L, const float *q, const float *k, const float *v,
                              const float *alpha, const float *beta, float *o, float *S_out, uint64_t seed,
                              uint32_t step, int stall_first_wait, cudaStream_t stream) {
    const DevFormat &F = s->dev;
    TcArgs A;
    A.pages = s->base + s->pages_offset;
    A.perm = s->base + s->perm_offset;
    A.status = reinterpret_cast<uint32_t *>(s->base + s->status_offset);
    A.pending = A.status + 1;   // the header's second word
    A.call = ++s->chunked_calls;
    if (A.call == 0) A.call = ++s->chunked_calls;   // a zeroed header never matches
    A.q = q; A.k = k; A.v = v; A.alpha = alpha; A.beta = beta; A.o = o; A.S_out = S_out;
    A.L = L;
    A.n_pages = s->batch * s->heads;
    A.heads = s->heads;
    A.store_bytes = (uint32_t)(F.col_scales ? F.c_off : F.page_bytes);
    A.seed_lo = (uint32_t)seed;
    A.seed_hi = (uint32_t)(seed >> 32);
    A.step = step;
    A.wait_limit_ns = s->wait_limit_ns;
    A.stall_first_wait = stall_first_wait;
    if (format_is<FmtStepQuant6>(F)) return launch_prefill_tc_with<FmtStepQuant6>(F, A, stream);
    if (format_is<FmtInt8Row>(F)) return launch_prefill_tc_with<FmtInt8Row>(F, A, stream);
    if (format_is<FmtDamp>(F)) return launch_prefill_tc_with<FmtDamp>(F, A, stream);
    if (format_is<FmtStepQuant4Kda>(F)) return launch_prefill_tc_with<FmtStepQuant4Kda>(F, A, stream);
    if (F.stochastic) return launch_prefill_tc_with<RuntimeFmt<true>>(F, A, stream);
    return launch_prefill_tc_with<RuntimeFmt<false>>(F, A, stream);
}

}  // namespace stq
