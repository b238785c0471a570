// stq_lifetime.cu -- lifetime row weights from gate samples (sm_100a).
//
// STEPQuant's temporal allocation (landing page, Figure B1): errors in
// long-lived memory persist, so key channels whose gates keep their content
// longer deserve wider rows.  Per head h and key channel kappa the weight is
// the expected persistence under geometric decay with the mean gate,
// 1 / (1 - mean alpha), capped at 2^24; it is the row_weight stq_calibrate
// multiplies the row energy by.  One CTA of 1,024 threads per head: thread
// (j, kappa) sums slice j of the requests, [j B / 8, (j + 1) B / 8), in double
// (samples, then its requests, ascending) and the eight slice sums are added
// as a fixed pairwise tree -- the oracle's order, so the weights are
// bit-identical.  A cold-path kernel, run once per calibration.
#include "stq_lifetime.h"

namespace stq {

constexpr int kLifetimeSlices = 8;

__global__ void __launch_bounds__(kD * kLifetimeSlices) lifetime_kernel(const float *alpha, int n_samples, int B,
                                                                        int H, int gate_vector, float *row_weight) {
    __shared__ double part[kLifetimeSlices][kD];
    const int h = blockIdx.x, kap = threadIdx.x & (kD - 1), j = threadIdx.x / kD;
    const int na = gate_vector ? kD : 1;
    const int col = gate_vector ? kap : 0;
    const int b0 = j * B / kLifetimeSlices, b1 = (j + 1) * B / kLifetimeSlices;
    double acc = 0.0;
    for (int t = 0; t < n_samples; ++t)
        for (int b = b0; b < b1; ++b)
            acc = __dadd_rn(acc, (double)__ldg(alpha + (((size_t)t * B + b) * H + h) * na + col));
    part[j][kap] = acc;
    __syncthreads();
    if (j == 0) {
        const double sum = __dadd_rn(__dadd_rn(__dadd_rn(part[0][kap], part[1][kap]), __dadd_rn(part[2][kap], part[3][kap])),
                                     __dadd_rn(__dadd_rn(part[4][kap], part[5][kap]), __dadd_rn(part[6][kap], part[7][kap])));
        const double mean = __ddiv_rn(sum, __dmul_rn((double)n_samples, (double)B));
        const double gap = __dsub_rn(1.0, mean);
        const double w = (gap <= 0x1p-24) ? 0x1p24 : __ddiv_rn(1.0, gap);
        row_weight[(size_t)h * kD + kap] = __double2float_rn(w);
    }
}

cudaError_t launch_lifetime(const stq_state *s, const float *alpha, int n_samples, float *row_weight,
                            cudaStream_t stream) {
    lifetime_kernel<<<s->heads, kD * kLifetimeSlices, 0, stream>>>(alpha, n_samples, s->batch, s->heads, s->fmt.gate_vector,
                                                 row_weight);
    return cudaGetLastError();
}

}  // namespace stq
