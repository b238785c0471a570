// stq_decode.cu -- the fused decode-step kernel (sm_100a).
//
// One persistent CTA of 128 threads walks pages p = blockIdx.x + i*gridDim.x.
// Each page's bytes and its q, k, v (and KDA alpha) rows are brought into a
// shared-memory ring by one thread with cp.async.bulk (no multicast), counted
// on an mbarrier.  Per page, all in registers / shared memory:
//   S1 unpack planes -> S2 dequant + decay T = z (alpha r)
//   S3 column sums u = sum_s k_s T_s        e = v (1/c) - u
//   S4 T' = T + (beta k_s) e                 S5 o = c * sum_s q_s T'_s
//   S6 row absmax -> r' = m/qmax, inv = qmax/m rounded toward zero
//   S7 requant (RNE of the exact product, or pcg4d stochastic rounding on
//      INT rows; binary16 on FP16 rows)    S8 repack.
// The requantized codes and r' are written back into the page's ring stage,
// and one bulk copy stores the stage to HBM at the next page's barrier, so
// the state crosses HBM once each way per step in whole 16-byte chunks.  No
// tensor cores: the work is rank-1 updates and mat-vecs.
//
// Thread mapping: lane l owns value columns 4l .. 4l+3; warp w owns slice w
// of every 16-row block, i.e. stored rows 16b + 4w + i (b = 0..7, i = 0..3).
// Every warp therefore meets the blocks' widths in the same order and all
// warps of the SM run one instruction stream; for the formats known at
// compile time that stream has no branch on a width.  Column sums follow
// the canonical order of the oracle: per thread one fma chain over blocks
// 0-3 and one over blocks 4-7 (16 rows each, ascending), their sum per warp,
// then (W0 + W1) + (W2 + W3) over the warps.
//
// One CTA-wide barrier per page: each warp prepares the operands of its own
// rows and syncs within the warp; the warps' column-sum partials and 1/c are
// double-buffered by page parity, so the only cross-warp dependency is u
// (and o, finished after the next page's barrier).
#include "stq_slices.cuh"

namespace stq {

struct DecodeArgs {
    uint8_t *pages;
    const uint8_t *perm;
    uint32_t *status;
    const float *q, *k, *v, *alpha, *beta;
    float *o;
    int n_pages;                  // work items = input rows x heads, < 2^31
    int heads;
    int n_stages;                 // ring depth, 3 .. kMaxStages
    uint32_t stage_bytes;
    uint32_t store_bytes;         // codes + r: the part of a page a step rewrites
    uint32_t seed_lo, seed_hi, step;
    uint64_t wait_limit_ns;
    int stall_first_wait;
    int n_slots;                  // requests in the state (valid slots: 0 .. n_slots-1)
    const int32_t *slots;         // slot table of a paged step (else null)
};

constexpr int kMaxStages = 4;
constexpr int kSlotThread = 32;   // paged step: the thread (warp 1) that fetches and resolves slots

struct SmemFixed {
    // per warp, its 32 rows in slice order (row 4b + i = block b, row i):
    float a[kWarps][kRowsPerWarp];          // alpha * r (decay x row scale)
    float kp[kWarps][kRowsPerWarp];         // k of the row's key channel
    float bk[kWarps][kRowsPerWarp];         // beta * k
    float qp[kWarps][kRowsPerWarp];         // q
    float inv[kWarps][kRowsPerWarp];        // requant multipliers
    float red_u[2][kWarps][kD];             // per page parity and warp: chain sums of u
    float red_o[2][kWarps][kD];             // the same for o
    float ic[2][kD];                        // per page parity: 1 / c per column
    float cpg[2][kD];                       // per page parity: c (o of a page is finished a page later)
    uint64_t full[kMaxStages];              // stage-full barriers
    uint64_t never;                         // a barrier nothing completes (test hook)
    int pg[kMaxStages];                     // paged step: page in each stage (-1: bad slot)
    int slot[kMaxStages];                   // paged step: the request's slot in each stage
    int bad[2];                             // paged step, per page parity: the page's slot was bad
    int pf_slot;                            // paged step: slot of a later refill's item (async copy)
    int pf_b, pf_h;                         // paged step: that item's input row and head
    int next_pg[2], next_slot[2];           // paged step, per page parity: the refill item's page, slot
};

constexpr size_t kFixedBytes = (sizeof(SmemFixed) + 127) / 128 * 128;

__host__ __device__ inline uint32_t decode_stage_bytes(const DevFormat &F) {
    return (uint32_t)F.page_bytes + 3u * 512u + (F.gate_vector ? 512u : 0u);
}

// Stage the page `pg` (paged step: none if pg < 0; else pg == p) and the
// input rows of work item p.
template <bool SLOTS>
__device__ __forceinline__ void issue_stage(const DevFormat &F, const DecodeArgs &A, uint8_t *dst, int p,
                                            uint64_t *bar, int pg) {
    if constexpr (SLOTS) {
        mbar_expect_tx(bar, decode_stage_bytes(F) - (pg < 0 ? (uint32_t)F.page_bytes : 0u));
        if (pg >= 0) bulk_g2s(dst, A.pages + (size_t)pg * F.page_bytes, (uint32_t)F.page_bytes, bar);
    } else {
        mbar_expect_tx(bar, decode_stage_bytes(F));
        bulk_g2s(dst, A.pages + (size_t)p * F.page_bytes, (uint32_t)F.page_bytes, bar);
    }
    uint8_t *rows = dst + F.page_bytes;
    bulk_g2s(rows, A.q + (size_t)p * kD, 512, bar);
    bulk_g2s(rows + 512, A.k + (size_t)p * kD, 512, bar);
    bulk_g2s(rows + 1024, A.v + (size_t)p * kD, 512, bar);
    if (F.gate_vector) bulk_g2s(rows + 1536, A.alpha + (size_t)p * kD, 512, bar);
}

// Paged step: the page of work item p (input row p / H, head p % H) is
// slot(row) * H + head, or -1 when the row's slot is out of range.
__device__ __forceinline__ int slot_page(const DecodeArgs &A, int p, int slot) {
    return (slot >= 0 && slot < A.n_slots) ? slot * A.heads + p % A.heads : -1;
}

__device__ __forceinline__ int item_slot(const DecodeArgs &A, int p) {
    return __ldg(A.slots + p / A.heads);
}

// Start copying the slot of input row `row` into *dst (4-byte async copy;
// no register holds it while it is in flight); cp_async_wait() before reading.
__device__ __forceinline__ void prefetch_slot(const DecodeArgs &A, int row, int *dst) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n\tcp.async.commit_group;"
                 :: "r"(smem_u32(dst)), "l"(A.slots + row) : "memory");
}

__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_all;" ::: "memory");
}

// o of a finished page: the tree over the warps' chain sums, times c.
__device__ __forceinline__ void write_o(const float (*red_o)[kD], const DecodeArgs &A, int p, int lane,
                                        const float *cpg, bool col_scales, bool bad = false) {
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
    if (bad) oa = ob = make_float2(__int_as_float(0x7FC00000), __int_as_float(0x7FC00000));   // NaN
    *reinterpret_cast<float4 *>(A.o + (size_t)p * kD + 4 * lane) = make_float4(oa.x, oa.y, ob.x, ob.y);
}

// Resident CTAs per SM the register budget is sized for: 3 (168 registers);
// the stochastic-rounding variant carries the hash state and gets 2.
template <bool SR>
constexpr int decode_ctas_per_sm() { return SR ? 2 : 3; }

// The per-page loop.
// SLOTS: the paged step (pages found through the slot table); otherwise
// page index = work item.
template <class FMT, bool SLOTS>
__global__ void __launch_bounds__(kThreads, decode_ctas_per_sm<FMT::kSr>())
decode_kernel(const DevFormat F, const DecodeArgs A) {
    extern __shared__ __align__(128) uint8_t smem[];
    SmemFixed &S = *reinterpret_cast<SmemFixed *>(smem);
    uint8_t *stages = smem + kFixedBytes;
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
    if (tid == 0) {
        for (int st = 0; st < A.n_stages; ++st) mbar_init(&S.full[st], 1);
        mbar_init(&S.never, 1);
        fence_mbar_init();
    }
    __syncthreads();
    // Launched early (programmatic dependent launch), the CTA may start
    // while the previous kernel on the stream finishes; nothing in global
    // memory is read before that kernel is complete and its writes visible
    // (a no-op for a plain launch).
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int stride = (int)gridDim.x;
    const int n = A.n_pages;
    const int NS = A.n_stages;
    if constexpr (SLOTS) {
        // lanes of warp 0 look up the first stages' pages in parallel; warp
        // 1 starts fetching the slot of the first refill's item
        if (tid < NS) {
            const int p = (int)blockIdx.x + tid * stride;
            if (p < n) {
                const int sl = item_slot(A, p);
                const int pg = slot_page(A, p, sl);
                S.pg[tid] = pg;
                S.slot[tid] = sl;
                if (pg < 0) atomicOr(A.status, kStatusBadSlot);
            }
        }
        if (tid == kSlotThread) {
            const int p = (int)blockIdx.x + NS * stride;
            if (p < n) {
                S.pf_b = p / A.heads;
                S.pf_h = p % A.heads;
                prefetch_slot(A, S.pf_b, &S.pf_slot);
            }
        }
        __syncwarp();
    }
    if (tid == 0) {
        for (int i = 0; i < NS; ++i) {
            const int p = (int)blockIdx.x + i * stride;
            if (p < n) {
                int pg = p;
                if constexpr (SLOTS) pg = S.pg[i];
                issue_stage<SLOTS>(F, A, stages + i * A.stage_bytes, p, &S.full[i], pg);
            }
        }
    }
    // (request, head) of a page is carried along: p advances by `stride`,
    // i.e. by (stride / H, stride % H) with a carry
    const int H = A.heads;
    const int sb = stride / H, sh = stride % H;

    // this lane's row of the slice (operand preparation and S6): block
    // my_blk = lane / 4, stored row my_s
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
        for (int b = 0; b < kBlocks; ++b) {   // selects, not a table in local memory
            if (b == my_blk) my_bits = FMT::width(b);
            if (b < my_blk && FMT::width(b) != 16) my_rbase += 16;
        }
    }
    const bool my_int = my_bits != 16;
    bool all_int = false;   // every row INT: the S6 test on my_int folds away
    if constexpr (!FMT::kRuntime) {
        all_int = true;
        for (int b = 0; b < kBlocks; ++b) all_int = all_int && FMT::width(b) != 16;
    }
    const int my_r = my_rbase + 4 * warp + (lane & 3);
    const float my_qmax = my_int ? (float)((1 << (my_bits - 1)) - 1) : 0.f;
    const float my_rcp = my_int ? __frcp_rn(my_qmax) : 0.f;

    int p = (int)blockIdx.x;
    int pb = p / H, ph = p % H;            // request and head of page p
    float alpha_s = 0.f, beta_s = 0.f;
    int kap = 0;
    if (p < n) {
        beta_s = __ldg(A.beta + p);
        if (!gate_vector) alpha_s = __ldg(A.alpha + p);
        kap = __ldg(A.perm + ph * kD + my_s) & (kD - 1);
    }
    int p_prev = -1;                  // work item whose codes and o are still to be stored
    int st = 0, st_prev = 0;
    uint32_t parity = 0;
    int it = 0;

    for (; p < n; ++it) {
        // scalars of the next page, loaded early
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
        // anything of the page is written
        bool ok;
        if (A.stall_first_wait && it == 0) ok = mbar_wait_bounded(&S.never, 0, A.wait_limit_ns);
        else ok = mbar_wait_bounded(&S.full[st], parity, A.wait_limit_ns);
        const int par = it & 1;
        uint8_t *stg = stages + st * A.stage_bytes;
        if constexpr (SLOTS) {
            // the stage's page was recorded before its barrier was armed
            if (tid == 0) S.bad[par] = S.pg[st] < 0;
        }
        const float *q_s = reinterpret_cast<const float *>(stg + F.page_bytes);
        const float *k_s = q_s + kD;
        const float *v_s = q_s + 2 * kD;
        const float *al_s = q_s + 3 * kD;
        float *r_s = reinterpret_cast<float *>(stg + F.r_off);

        // operands of this lane's row: decay x row scale, permuted k and q, beta k
        {
            const float kk = k_s[kap], qq = q_s[kap];
            const float al = gate_vector ? al_s[kap] : alpha_s;
            const float a = (all_int || my_int) ? __fmul_rn(al, r_s[my_r]) : al;
            if (col_scales) {   // thread t also keeps and inverts the scale of column t
                const float c = reinterpret_cast<const float *>(stg + F.c_off)[tid];
                S.cpg[par][tid] = c;
                S.ic[par][tid] = __frcp_rn(c);
            }
            S.a[warp][lane] = a;
            S.kp[warp][lane] = kk;
            S.qp[warp][lane] = qq;
            S.bk[warp][lane] = __fmul_rn(beta_s, kk);
        }
        __syncwarp();   // the warp's rows' operands come from its own lanes

        // S1 + S2 and S3's chains: blocks 0-3 feed chain 0, blocks 4-7 chain 1
        Tile T;
        float2 cu[2][2];   // chains from +0, as p = fma(w, x, p) from 0
#pragma unroll
        for (int h = 0; h < 2; ++h) cu[h][0] = cu[h][1] = make_float2(0.f, 0.f);
        static_for<0, kBlocks>([&](auto bc) {
            constexpr int b = decltype(bc)::value;
            const float4 a4 = *reinterpret_cast<const float4 *>(&S.a[warp][4 * b]);
            const uint8_t *blk = stg + fmt_offset<FMT, b>(F);
            with_width<FMT, b>(F, [&](auto wc) {
                constexpr int W = decltype(wc)::value;
                dequant_slice<W, b>(blk, warp, lane, a4, T);
            });
            const float4 k4 = *reinterpret_cast<const float4 *>(&S.kp[warp][4 * b]);
            const float kv[4] = {k4.x, k4.y, k4.z, k4.w};
            constexpr int h = b >> 2;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                cu[h][0] = __ffma2_rn(make_float2(kv[i], kv[i]), T[b][i][0], cu[h][0]);
                cu[h][1] = __ffma2_rn(make_float2(kv[i], kv[i]), T[b][i][1], cu[h][1]);
            }
        });
        {
            const float2 w01 = __fadd2_rn(cu[0][0], cu[1][0]), w23 = __fadd2_rn(cu[0][1], cu[1][1]);
            *reinterpret_cast<float4 *>(&S.red_u[par][warp][4 * lane]) = make_float4(w01.x, w01.y, w23.x, w23.y);
        }
        const float4 v4 = *reinterpret_cast<const float4 *>(v_s + 4 * lane);
        if (__syncthreads_or(!ok)) {
            // a stage never arrived: record it, finish the previous page, let
            // the copies in flight land and leave; nothing of this page (or
            // a later one) is written
            if (warp == kWarps - 1 && p_prev >= 0)
                write_o(S.red_o[par ^ 1], A, p_prev, lane, S.cpg[par ^ 1], col_scales, SLOTS && S.bad[par ^ 1]);
            if (tid == 0) {
                atomicOr(A.status, kStatusTimeout);
                if (SLOTS ? S.pg[st_prev] >= 0 : p_prev >= 0) {
                    bulk_s2g(A.pages + (size_t)(SLOTS ? S.pg[st_prev] : p_prev) * F.page_bytes, stages + st_prev * A.stage_bytes,
                             A.store_bytes);
                    bulk_commit();
                }
                // last ring slot whose load was issued
                const int last = it < 2 ? NS - 1 : ((FMT::kTune & kEarlyRefill) ? it - 2 + NS : it - 3 + NS);
                for (int j = it; j <= last; ++j) {
                    if ((int)blockIdx.x + j * stride < n)
                        mbar_wait_bounded(&S.full[j % NS], (uint32_t)((j / NS) & 1), A.wait_limit_ns);
                }
                bulk_wait<0>();
            }
            if (SLOTS && tid == kSlotThread) cp_async_wait();   // no copy outlives the CTA
            __syncthreads();
            return;
        }

        constexpr bool kEarly = (FMT::kTune & kEarlyRefill) != 0;
        if (tid == 0) {
            // the previous page is complete in its stage: store it; its stage
            // is refilled once the store has read it (see kEarlyRefill)
            if (SLOTS ? p_prev >= 0 && S.pg[st_prev] >= 0 : p_prev >= 0) {
                bulk_s2g(A.pages + (size_t)(SLOTS ? S.pg[st_prev] : p_prev) * F.page_bytes, stages + st_prev * A.stage_bytes,
                         A.store_bytes);
                bulk_commit();
            }
            if (!kEarly && it >= 2) {
                bulk_wait_read<1>();
                const int j = it - 2 + NS;
                const int pr = (int)blockIdx.x + j * stride;
                if (pr < n) {
                    int pg = pr;
                    if constexpr (SLOTS) {   // looked up by the slot thread a page ago
                        pg = S.next_pg[it & 1];
                        S.pg[j % NS] = pg;
                        S.slot[j % NS] = S.next_slot[it & 1];
                    }
                    fence_proxy_async_smem();
                    issue_stage<SLOTS>(F, A, stages + (j % NS) * A.stage_bytes, pr, &S.full[j % NS], pg);
                }
            }
        }
        if constexpr (SLOTS) {
            // the slot thread (off the copy thread's path) looks up the page
            // of the item the next page's refill loads, from the slot fetched
            // a page ago, and starts fetching the one after it
            if (tid == kSlotThread && (kEarly || it >= 1)) {
                const int j = kEarly ? it + NS : it - 1 + NS;
                const int pr = (int)blockIdx.x + j * stride;
                if (pr < n) {
                    // item pr is (row pf_b, head pf_h); the next one is
                    // `stride` further: (stride / H, stride % H) with a carry
                    cp_async_wait();
                    const int sl = S.pf_slot, rb = S.pf_b, rh = S.pf_h;
                    const int pg = (sl >= 0 && sl < A.n_slots) ? sl * H + rh : -1;
                    S.next_pg[(it + 1) & 1] = pg;
                    S.next_slot[(it + 1) & 1] = sl;
                    if (pg < 0) atomicOr(A.status, kStatusBadSlot);
                    if (pr + stride < n) {
                        int nb = rb + sb, nh = rh + sh;
                        if (nh >= H) { nh -= H; ++nb; }
                        S.pf_b = nb;
                        S.pf_h = nh;
                        prefetch_slot(A, nb, &S.pf_slot);
                    }
                }
            }
        }
        // o of the previous page (its chain sums were stored before this
        // barrier), by the last warp: warp 0's first thread handles the copies
        if (warp == kWarps - 1 && p_prev >= 0)
            write_o(S.red_o[par ^ 1], A, p_prev, lane, S.cpg[par ^ 1], col_scales, SLOTS && S.bad[par ^ 1]);

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
            if (col_scales) ic = *reinterpret_cast<const float4 *>(&S.ic[par][4 * lane]);
            // two roundings, scalar: an f32x2 multiply feeding an f32x2 add is
            // fused by the compiler into one f32x2 fma
            e01 = make_float2(__fsub_rn(__fmul_rn(v4.x, ic.x), ua.x), __fsub_rn(__fmul_rn(v4.y, ic.y), ua.y));
            e23 = make_float2(__fsub_rn(__fmul_rn(v4.z, ic.z), ub.x), __fsub_rn(__fmul_rn(v4.w, ic.w), ub.y));
        }

        // S4: T' = T + (beta k) e; S6's row maxima (one warp reduction per
        // row, kept in the row's inv slot); S5's chains
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
                S.inv[warp][4 * b + i] = warp_absmax(absmax4(T[b][i][0], T[b][i][1]));
            }
            if constexpr (!(FMT::kTune & kOLate) && !((FMT::kTune & kOSplit) && b >= 4))
                readout_block<b>(S.qp[warp], T, co[b >> 2]);
        });
        if constexpr (!(FMT::kTune & (kOLate | kOSplit))) store_readout(S.red_o[par][warp], lane, co);
        if (kEarly && tid == 0 && p_prev >= 0) {
            // refill the previous page's stage with the page NS - 1 ahead of this one
            bulk_wait_read<0>();
            {
                const int j = it - 1 + NS;
                const int pr = (int)blockIdx.x + j * stride;
            if (pr < n) {
                int pg = pr;
                if constexpr (SLOTS) {   // looked up by the slot thread a page ago
                    pg = S.next_pg[it & 1];
                    S.pg[j % NS] = pg;
                    S.slot[j % NS] = S.next_slot[it & 1];
                }
                fence_proxy_async_smem();
                issue_stage<SLOTS>(F, A, stages + (j % NS) * A.stage_bytes, pr, &S.full[j % NS], pg);
            }
            }
        }
        __syncwarp();

        // S6: lane l finishes row l of the slice: r' = m / qmax, inv = qmax / m (toward zero)
        {
            const float m = S.inv[warp][lane];
            float inv = 0.f;
            if (all_int || my_int) {
                // m = 0 (a zero row): r' = 0 and inv = 0, codes 0
                const float r = div_by_qmax(m, my_qmax, my_rcp);
                inv = m > 0.f ? div_rz_qmax<(FMT::kTune & kFastRcp) != 0>(my_qmax, m) : 0.f;
                r_s[my_r] = r;
            }
            if constexpr ((FMT::kTune & (kOLate | kOSplit)) != 0) {
                static_for<((FMT::kTune & kOLate) ? 0 : 4), kBlocks>([&](auto bc) {
                    constexpr int b = decltype(bc)::value;
                    readout_block<b>(S.qp[warp], T, co[b >> 2]);
                });
                store_readout(S.red_o[par][warp], lane, co);
            }
            S.inv[warp][lane] = inv;
        }
        __syncwarp();

        // S7 + S8, into the stage
        SrCtx sr;
        sr.k0 = A.seed_lo; sr.k1 = A.seed_hi; sr.step = A.step;
        if constexpr (SLOTS) sr.b = (uint32_t)S.slot[st];   // the request's slot in the state
        else sr.b = (uint32_t)pb;
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
    }
    // the next kernel on the stream may start its own set-up now
    asm volatile("griddepcontrol.launch_dependents;");
    __syncthreads();
    if (p_prev >= 0) {
        if (tid == 0 && (SLOTS ? S.pg[st_prev] >= 0 : true)) {
            bulk_s2g(A.pages + (size_t)(SLOTS ? S.pg[st_prev] : p_prev) * F.page_bytes, stages + st_prev * A.stage_bytes, A.store_bytes);
            bulk_commit();
        }
        if (warp == kWarps - 1)
            write_o(S.red_o[(it - 1) & 1], A, p_prev, lane, S.cpg[(it - 1) & 1], col_scales, SLOTS && S.bad[(it - 1) & 1]);
    }
    if (tid == 0) bulk_wait<0>();
    if (SLOTS && tid == kSlotThread) cp_async_wait();   // no copy outlives the CTA
}

static int decode_stages(size_t stride, int ctas_per_sm) {
    // as many ring stages as fit next to the fixed part at the target
    // occupancy, at least 3 (a stage is written back during the page after
    // its own and refilled then or one page later)
    int dev = 0, smem_sm = 0, reserved = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
    cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
    const long budget = (long)smem_sm / ctas_per_sm - reserved - (long)kFixedBytes;
    long ns = budget / (long)stride;
    if (ns > kMaxStages) ns = kMaxStages;
    if (ns < 3) ns = 3;
    return (int)ns;
}

template <class FMT, bool SLOTS>
static cudaError_t launch_with(const DevFormat &F, const DecodeArgs &A0, bool early_launch, cudaStream_t stream) {
    DecodeArgs A = A0;
    A.n_stages = decode_stages(A.stage_bytes, decode_ctas_per_sm<FMT::kSr>());
    const size_t smem = kFixedBytes + (size_t)A.n_stages * A.stage_bytes;
    const void *fn = (const void *)decode_kernel<FMT, SLOTS>;
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
    return cudaLaunchKernelEx(&cfg, decode_kernel<FMT, SLOTS>, F, A);
}

template <bool SLOTS>
static cudaError_t launch_fmt(const DevFormat &F, const DecodeArgs &A, bool early_launch, cudaStream_t stream) {
    if (format_is<FmtStepQuant6>(F)) return launch_with<FmtStepQuant6, SLOTS>(F, A, early_launch, stream);
    if (format_is<FmtInt8Row>(F)) return launch_with<FmtInt8Row, SLOTS>(F, A, early_launch, stream);
    if (format_is<FmtStepQuant4Kda>(F)) return launch_with<FmtStepQuant4Kda, SLOTS>(F, A, early_launch, stream);
    if (format_is<FmtDamp>(F)) return launch_with<FmtDamp, SLOTS>(F, A, early_launch, stream);
    if (F.stochastic) return launch_with<RuntimeFmt<true>, SLOTS>(F, A, early_launch, stream);
    return launch_with<RuntimeFmt<false>, SLOTS>(F, A, early_launch, stream);
}

cudaError_t launch_decode(const stq_state *s, const float *q, const float *k, const float *v,
                          const float *alpha, const float *beta, float *o, uint64_t seed, uint32_t step,
                          int stall_first_wait, bool early_launch, const int32_t *slots, int n_rows,
                          cudaStream_t stream) {
    const DevFormat &F = s->dev;
    DecodeArgs A;
    A.pages = s->base + s->pages_offset;
    A.perm = s->base + s->perm_offset;
    A.status = reinterpret_cast<uint32_t *>(s->base + s->status_offset);
    A.q = q; A.k = k; A.v = v; A.alpha = alpha; A.beta = beta; A.o = o;
    A.slots = slots;
    A.n_slots = s->batch;
    A.n_pages = (slots ? n_rows : s->batch) * s->heads;
    A.heads = s->heads;
    A.stage_bytes = (decode_stage_bytes(F) + 127) / 128 * 128;
    A.store_bytes = (uint32_t)(F.col_scales ? F.c_off : F.page_bytes);
    A.n_stages = 0;
    A.seed_lo = (uint32_t)seed;
    A.seed_hi = (uint32_t)(seed >> 32);
    A.step = step;
    A.wait_limit_ns = s->wait_limit_ns;
    A.stall_first_wait = stall_first_wait;
    if (slots) return launch_fmt<true>(F, A, early_launch, stream);
    return launch_fmt<false>(F, A, early_launch, stream);
}

}  // namespace stq
