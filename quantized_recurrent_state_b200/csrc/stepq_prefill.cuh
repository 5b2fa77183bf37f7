// Launch arguments of the chunked prefill (stepq_prefill.cu), shared with the
// C ABI that fills them.
#pragma once

namespace stepq {

// Per-head units, d = 128.
struct PrefillArgs {
    float *S;                  // [n_req][nL][H][D][D] fp32 states, read (unless zero_init) and written
    const float *q, *k, *v;    // [n_req][T][nL_in][H][D]
    const float *alpha, *beta; // [n_req][T][nL_in][H]
    float *o;                  // [n_req][T][nL_in][H][D]
    int n_req, T, nL, nL_in, l_in0, H;
    int zero_init;
};

}  // namespace stepq
