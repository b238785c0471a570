// stq_lifetime.h -- launcher of the lifetime row weights (stq_lifetime.cu).
#pragma once

#include "stq_internal.h"

namespace stq {

// Row weights [H][128] from gate samples [n_samples][B][H] (or [..][128]).
cudaError_t launch_lifetime(const stq_state *s, const float *alpha, int n_samples, float *row_weight,
                            cudaStream_t stream);

}  // namespace stq
