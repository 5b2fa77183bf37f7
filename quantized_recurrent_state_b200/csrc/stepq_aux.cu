// FP32-state reference step, HBM copy probe and calibration kernels.
//
// STEPQuant paper digest (vibe-research): the FP32-state decode is the
// unquantized baseline the pages compare against (背景与动机, 实验); the
// calibration statistics are those of 方法-1 (mean log gate, distortion per
// width) and 方法-2 (row impact omega_i = E[g_i^2], g = A_t^T q_t).
#include "stepq_dev.cuh"

namespace stepq {

// Scratch shared with the step kernels' layout assumptions (fp64 partials).
template <int D>
struct Fp32Scratch {
    double pU[8][D];
    double pO[8][D];
    float wv[D];
    float kf[D];
    float qf[D];
};

template <int D>
struct GeoA {
    static constexpr int NT = 2 * D, RT = D / 8, LANES = D / 4;
};

// One (request, layer, head) fp32 state per CTA:
//   S'_ij = fl(alpha_i S_ij); u_j = fl32(sum_i k_i S'_ij) (fp64 sum);
//   w_j = fl(beta fl(v_j - u_j)); S_ij = fma(k_i, w_j, S'_ij);
//   o_j = fl32(sum_i q_i S_ij) (fp64 sum).
template <int D>
__global__ void __launch_bounds__(2 * D) k_fp32_step(Args a, float *S_pool, int n_layers_total, int kda) {
    __shared__ Fp32Scratch<D> sc;
    using G = GeoA<D>;
    const int tid = threadIdx.x;
    const int g = tid / G::LANES, l = tid % G::LANES;
    const int it = blockIdx.x;
    const int per_req = a.nL * a.H;
    const int n = it / per_req;
    const int rem = it - n * per_req;
    const int ll = rem / a.H, h = rem - (rem / a.H) * a.H;
    const int row = (n * a.nL_in + a.l_in0 + ll) * a.H + h;
    const int slot = a.slots[n];
    if (slot < 0 || slot >= a.n_slots) {
        if (tid == 0) flag_error(a.err, kErrBadSlot);
        return;
    }
    float *S = S_pool + (((size_t)slot * n_layers_total + (a.lb + ll)) * a.H + h) * (size_t)D * D;
    const float *q = a.q + (size_t)row * D;
    const float *k = a.k + (size_t)row * D;
    const float *v = a.v + (size_t)row * D;
    const float beta = a.beta[row];
    if (tid < D) {
        sc.kf[tid] = k[tid];
        sc.qf[tid] = q[tid];
    }
    __syncthreads();
    float Sr[G::RT][4];
    double accU[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
    for (int r = 0; r < G::RT; ++r) {
        const int i = g * G::RT + r;
        const float al = kda ? a.alpha[(size_t)row * D + i] : a.alpha[row];
        const float4 x = *reinterpret_cast<const float4 *>(S + (size_t)i * D + 4 * l);
        Sr[r][0] = __fmul_rn(al, x.x); Sr[r][1] = __fmul_rn(al, x.y);
        Sr[r][2] = __fmul_rn(al, x.z); Sr[r][3] = __fmul_rn(al, x.w);
        const double ki = (double)sc.kf[i];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) accU[jj] = fma(ki, (double)Sr[r][jj], accU[jj]);
    }
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) sc.pU[g][4 * l + jj] = accU[jj];
    __syncthreads();
    if (tid < D) {
        double s = 0.0;
#pragma unroll
        for (int b = 0; b < 8; ++b) s += sc.pU[b][tid];
        const float u = __double2float_rn(s);
        sc.wv[tid] = __fmul_rn(beta, __fsub_rn(v[tid], u));
    }
    __syncthreads();
    double accO[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
    for (int r = 0; r < G::RT; ++r) {
        const int i = g * G::RT + r;
        const float ki = sc.kf[i];
        const double qi = (double)sc.qf[i];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            Sr[r][jj] = __fmaf_rn(ki, sc.wv[4 * l + jj], Sr[r][jj]);
            accO[jj] = fma(qi, (double)Sr[r][jj], accO[jj]);
        }
        *reinterpret_cast<float4 *>(S + (size_t)i * D + 4 * l) = make_float4(Sr[r][0], Sr[r][1], Sr[r][2], Sr[r][3]);
    }
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) sc.pO[g][4 * l + jj] = accO[jj];
    __syncthreads();
    if (tid < D) {
        double s = 0.0;
#pragma unroll
        for (int b = 0; b < 8; ++b) s += sc.pO[b][tid];
        a.o[(size_t)row * D + tid] = __double2float_rn(s);
    }
}

cudaError_t launch_fp32_step(int D, const Args &a, float *S_pool, int n_layers_total, cudaStream_t st) {
    if (a.n_items <= 0) return cudaSuccess;
    const int kda = a.mode == 1;
    switch (D) {
        case 16: k_fp32_step<16><<<a.n_items, 32, 0, st>>>(a, S_pool, n_layers_total, kda); break;
        case 32: k_fp32_step<32><<<a.n_items, 64, 0, st>>>(a, S_pool, n_layers_total, kda); break;
        case 64: k_fp32_step<64><<<a.n_items, 128, 0, st>>>(a, S_pool, n_layers_total, kda); break;
        case 128: k_fp32_step<128><<<a.n_items, 256, 0, st>>>(a, S_pool, n_layers_total, kda); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// HBM copy probe: grid-stride 16-byte copy.
// ---------------------------------------------------------------------------
__global__ void k_copy(uint4 *__restrict__ dst, const uint4 *__restrict__ src, size_t n) {
    size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    for (; i + 3 * stride < n; i += 4 * stride) {
        const uint4 a0 = src[i], a1 = src[i + stride], a2 = src[i + 2 * stride], a3 = src[i + 3 * stride];
        dst[i] = a0; dst[i + stride] = a1; dst[i + 2 * stride] = a2; dst[i + 3 * stride] = a3;
    }
    for (; i < n; i += stride) dst[i] = src[i];
}

cudaError_t launch_copy(void *dst, const void *src, size_t bytes, int n_sms, cudaStream_t st) {
    const size_t n = bytes / 16;
    if (n == 0) return cudaSuccess;
    int grid = n_sms * 8;
    k_copy<<<grid, 512, 0, st>>>(reinterpret_cast<uint4 *>(dst), reinterpret_cast<const uint4 *>(src), n);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Calibration: omega and log-gate accumulation (one CTA per (req, layer, head),
// max(D, 32) threads, thread i < D owns key row i).
// ---------------------------------------------------------------------------
template <int D>
__global__ void k_calib_acc(Args a, double *omega_acc, double *lsum_acc, int kda) {
    constexpr int NTH = D < 32 ? 32 : D;
    __shared__ double red[NTH / 32];
    const int tid = threadIdx.x;
    const int it = blockIdx.x;
    const int per_req = a.nL * a.H;
    const int n = it / per_req;
    const int rem = it - n * per_req;
    const int ll = rem / a.H, h = rem - (rem / a.H) * a.H;
    const int row = (n * a.nL_in + a.l_in0 + ll) * a.H + h;
    const int gl = (a.lb + ll) * a.H + h;
    const bool on = tid < D;
    const double qi = on ? (double)a.q[(size_t)row * D + tid] : 0.0;
    const double ki = on ? (double)a.k[(size_t)row * D + tid] : 0.0;
    double kq = ki * qi;
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, m);
    if ((tid & 31) == 0) red[tid >> 5] = kq;
    __syncthreads();
    double s = 0.0;
    for (int w = 0; w < NTH / 32; ++w) s += red[w];
    if (!on) return;
    const double al = kda ? (double)a.alpha[(size_t)row * D + tid] : (double)a.alpha[row];
    const double beta = (double)a.beta[row];
    const double gv = al * (qi - beta * ki * s);
    atomicAdd(&omega_acc[(size_t)gl * D + tid], gv * gv);
    atomicAdd(&lsum_acc[(size_t)gl * D + tid], log(al));
}

cudaError_t launch_calib_acc(int D, const Args &a, double *om, double *ls, cudaStream_t st) {
    if (a.n_items <= 0) return cudaSuccess;
    const int kda = a.mode == 1;
    switch (D) {
        case 16: k_calib_acc<16><<<a.n_items, 32, 0, st>>>(a, om, ls, kda); break;
        case 32: k_calib_acc<32><<<a.n_items, 32, 0, st>>>(a, om, ls, kda); break;
        case 64: k_calib_acc<64><<<a.n_items, 64, 0, st>>>(a, om, ls, kda); break;
        case 128: k_calib_acc<128><<<a.n_items, 128, 0, st>>>(a, om, ls, kda); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace stepq
