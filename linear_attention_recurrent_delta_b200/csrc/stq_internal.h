// stq_internal.h -- host-side internals shared by the library's .cu files.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/stq.h"
#include "stq_device.cuh"

struct stq_state {
    stq_format fmt;
    int batch, heads;
    uint8_t *base;               // caller's device buffer
    size_t buf_bytes;
    size_t page_bytes, perm_offset, pages_offset, status_offset;
    stq::DevFormat dev;
    uint64_t wait_limit_ns;
    int stall_first_wait;
    mutable uint32_t chunked_calls = 0;   // stq_prefill_chunked calls (the mark its two launches share)
};

namespace stq {

constexpr size_t kHeaderBytes = 256;

// Validate a format and build its device constants.  Returns STQ_OK,
// STQ_ERR_INVALID_ARG or STQ_ERR_UNSUPPORTED.
stq_status build_dev_format(const stq_format *f, DevFormat *out);

// Persistent-grid size for a kernel: SM count x resident CTAs of `threads`
// threads with `dyn_smem` dynamic shared memory, at most n_units.
int persistent_grid(const void *kernel, int threads, size_t dyn_smem, long n_units);

// Launchers (return cudaError_t of the launch).
cudaError_t launch_decode(const stq_state *s, const float *q, const float *k, const float *v,
                          const float *alpha, const float *beta, float *o, uint64_t seed,
                          uint32_t step, int stall_first_wait, bool early_launch, const int32_t *slots,
                          int n_rows, cudaStream_t stream);
// Per-window decode: step t of a window of `window` steps (commit: requantize
// and store the pages); buf holds window_buffer_stride(window) bytes per page.
size_t window_buffer_stride(int window);
cudaError_t launch_window(const stq_state *s, uint8_t *buf, int window, int t, bool commit, const float *q,
                          const float *k, const float *v, const float *alpha, const float *beta, float *o,
                          uint64_t seed, uint32_t step, int stall_first_wait, bool early_launch,
                          cudaStream_t stream);
// Prefill: a prompt of L tokens through every page, one requantization.
cudaError_t launch_prefill(const stq_state *s, int L, const float *q, const float *k, const float *v,
                           const float *alpha, const float *beta, float *o, float *S_out, uint64_t seed,
                           uint32_t step, int stall_first_wait, bool early_launch, cudaStream_t stream);
// Prefill in chunkwise form on the tensor cores (scalar-gate formats).
cudaError_t launch_prefill_tc(const stq_state *s, int L, const float *q, const float *k, const float *v,
                              const float *alpha, const float *beta, float *o, float *S_out, uint64_t seed,
                              uint32_t step, int stall_first_wait, cudaStream_t stream);
cudaError_t launch_calibrate(const stq_state *s, const float *S, const float *row_weight,
                             double *workspace, cudaStream_t stream);
// The checks every calibration entry point makes of its fp32 state and row
// weight: d_S non-null, 16-byte aligned and clear of the state's bytes;
// d_row_weight (may be null) 4-byte aligned.  STQ_OK or the error to return.
stq_status check_calibrate_input(const stq_state *s, const float *d_S, const float *d_row_weight);
size_t calibrate_workspace_bytes(int batch, int heads);
cudaError_t launch_quantize(const stq_state *s, const float *S, cudaStream_t stream);
// Quantize with jointly fitted scales (iters rounds; 0: launch_quantize).
cudaError_t launch_fit(const stq_state *s, const float *S, const float *impact, int iters, cudaStream_t stream);
cudaError_t launch_dequantize(const stq_state *s, float *S, cudaStream_t stream);

}  // namespace stq
