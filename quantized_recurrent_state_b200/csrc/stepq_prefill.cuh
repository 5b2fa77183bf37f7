// Launch arguments of the chunked prefill (stepq_prefill.cu), shared with the
// C ABI that fills them.
#pragma once

namespace stepq {

// Device error word bit set by the prefill: a gate outside (0, 1], or per-row gates whose
// running log-products leave the range the fp32 factors hold (see k_prefill).
constexpr int kErrGateRange = 8;

// d = 128; per-head gates (rows = 0) or one gate per key row (rows = 1).
struct PrefillArgs {
    float *S;                  // [n_req][nL][H][D][D] fp32 states, read (unless zero_init) and written
    const float *q, *k, *v;    // [n_req][T][nL_in][H][D]
    const float *alpha;        // [n_req][T][nL_in][H], or [..][H][D] when rows
    const float *beta;         // [n_req][T][nL_in][H]
    float *o;                  // [n_req][T][nL_in][H][D]
    int n_req, T, nL, nL_in, l_in0, H;
    int zero_init;
    int rows;
    int *err;                  // device error word (kErrGateRange)
};

}  // namespace stepq
