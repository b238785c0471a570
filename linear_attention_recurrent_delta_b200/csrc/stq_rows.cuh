// stq_rows.cuh -- per-lane row context and format flags shared by the
// per-window and prefill kernels (sm_100a).  Lane l of warp w owns stored
// row 16 (l / 4) + 4 w + (l % 4) for its row-wise work (operands, row scale).
#pragma once

#include "stq_slices.cuh"

namespace stq {

// This lane's row of the slice: block lane / 4, stored row s, r index rix.
struct RowCtx {
    int s, rix;
    bool is_int, all_int;
    float qmax, rcp_qmax;
};

template <class FMT>
__device__ __forceinline__ RowCtx row_ctx(const DevFormat &F, int warp, int lane) {
    RowCtx R;
    const int blk = lane >> 2;
    R.s = 16 * blk + 4 * warp + (lane & 3);
    int bits, rbase;
    if constexpr (FMT::kRuntime) {
        bits = F.blk_bits(blk);
        rbase = F.blk_rbase(blk);
        R.all_int = false;
    } else {
        bits = 0;
        rbase = 0;
#pragma unroll
        for (int b = 0; b < kBlocks; ++b) {   // selects, not a table in local memory
            if (b == blk) bits = FMT::width(b);
            if (b < blk && FMT::width(b) != 16) rbase += 16;
        }
        R.all_int = true;
        for (int b = 0; b < kBlocks; ++b) R.all_int = R.all_int && FMT::width(b) != 16;
    }
    R.is_int = bits != 16;
    R.rix = rbase + 4 * warp + (lane & 3);
    R.qmax = R.is_int ? (float)((1 << (bits - 1)) - 1) : 0.f;
    R.rcp_qmax = R.is_int ? __frcp_rn(R.qmax) : 0.f;
    return R;
}

template <class FMT>
__device__ __forceinline__ void format_flags(const DevFormat &F, bool &col_scales, bool &gate_vector) {
    if constexpr (FMT::kRuntime) {
        col_scales = F.col_scales != 0;
        gate_vector = F.gate_vector != 0;
    } else {
        col_scales = FMT::kCols;
        gate_vector = FMT::kGvec;
    }
}

}  // namespace stq
