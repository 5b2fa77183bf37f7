// Launch arguments of the chunked prefill (stepq_prefill.cu), shared with the
// C ABI that fills them.
#pragma once

namespace stepq {

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
};

}  // namespace stepq
