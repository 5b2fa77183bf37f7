// FP32-state reference step, HBM copy probe and calibration kernels.
//
// STEPQuant paper digest (vibe-research): the FP32-state decode is the
// unquantized baseline the pages compare against (背景与动机, 实验); the
// calibration statistics are those of 方法-1 (mean log gate, distortion per
// width) and 方法-2 (row impact omega_i = E[g_i^2], g = A_t^T q_t).
#include "stepq_dev.cuh"

namespace stepq {



// FP32-state step: a persistent grid streams the (request, layer, head)
// states through a ring of shared-memory stages (the D x D fp32 tile, q, k,
// v and the gates by 1-D bulk copies, completion on an mbarrier).  Thread t
// owns rows [g RT, g RT + RT) of columns [4l, 4l + 4), g = t / (D/4),
// l = t % (D/4): at D = 128 a warp holds one band of 16 whole rows, so its
// shared-memory reads of the tile are consecutive 16-byte chunks.  Per state:
//   S'_ij = fl(alpha_i S_ij); u_j = band_i(k_i S'_ij);
//   w_j = fl(beta fl(v_j - u_j)); S_ij = fma(k_i, w_j, S'_ij); o_j = band_i(q_i S_ij)
// (band order: in each band of RT rows the even and the odd rows form fma
// chains that are added; the 8 band values are added in a balanced tree).
template <int D>
struct Fp32Geo {
    static constexpr int NT = 2 * D, RT = D / 8, LANES = D / 4;
    static constexpr int STAGES = D == 128 ? 3 : 4;
    static constexpr uint32_t TILE = (uint32_t)D * D * 4;
    static constexpr uint32_t TAIL = 4u * D * 4 + 16;       // q, k, v, alpha rows, {alpha, beta}
    static constexpr uint32_t STAGE = TILE + TAIL;
};

template <int D>
struct __align__(16) Fp32Scratch {
    float pb[8][D];    // band values of u, then of o
    float wv[D];
    float2 k2[D];      // (k_i, k_i)
    float2 q2[D];      // (q_i, q_i)
    float2 a2[D];      // (alpha_i, alpha_i)
    int meta[Fp32Geo<D>::STAGES][4];  // valid, input row, state element offset lo, hi
};

template <int D>
__device__ __forceinline__ void fp32_issue(const Args &a, float *S_pool, int n_layers_total, int kda, int it,
                                           uint8_t *stage, uint64_t *bar, int *meta) {
    using G = Fp32Geo<D>;
    const int per_req = a.nL * a.H;
    const int n = it / per_req;
    const int rem = it - n * per_req;
    const int ll = rem / a.H, h = rem - ll * a.H;
    const int row = (n * a.nL_in + a.l_in0 + ll) * a.H + h;
    const int slot = a.slots[n];
    const bool ok = slot >= 0 && slot < a.n_slots;
    const size_t soff = (((size_t)slot * n_layers_total + (a.lb + ll)) * a.H + h) * (size_t)D * D;
    meta[0] = ok ? 1 : 0;
    meta[1] = row;
    meta[2] = (int)(uint32_t)soff;
    meta[3] = (int)(uint32_t)(soff >> 32);
    if (!ok) {
        flag_error(a.err, kErrBadSlot);
        mbar_arrive(bar);
        return;
    }
    float *tf = reinterpret_cast<float *>(stage + G::TILE);
    float *ab = tf + 4 * D;
    if (!kda) cp_async4(ab, a.alpha + row);
    cp_async4(ab + 1, a.beta + row);
    cp_async_mbar_arrive(bar);
    fence_proxy_async();
    constexpr uint32_t RB = D * 4;
    mbar_arrive_expect(bar, G::TILE + 3 * RB + (kda ? RB : 0) + a.phantom_tx);
    bulk_g2s(stage, S_pool + soff, G::TILE, bar);
    bulk_g2s(tf, a.q + (size_t)row * D, RB, bar);
    bulk_g2s(tf + D, a.k + (size_t)row * D, RB, bar);
    bulk_g2s(tf + 2 * D, a.v + (size_t)row * D, RB, bar);
    if (kda) bulk_g2s(tf + 3 * D, a.alpha + (size_t)row * D, RB, bar);
}

template <int D>
__global__ void __launch_bounds__(2 * D, 1) k_fp32_step(Args a, float *S_pool, int n_layers_total, int kda) {
    using G = Fp32Geo<D>;
    constexpr int RT = G::RT, LANES = G::LANES, ST = G::STAGES;
    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t *stages = smem;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + ST * G::STAGE);
    Fp32Scratch<D> &sc = *reinterpret_cast<Fp32Scratch<D> *>(smem + ST * G::STAGE + 64);
    const int tid = threadIdx.x;
    const int g = tid / LANES, l = tid % LANES, j0 = 4 * l;
    const int Gd = gridDim.x;
    if (tid == 0) {
        for (int s = 0; s < ST; ++s) mbar_init(&bars[s], 1);
        fence_mbar_init();
        for (int s = 0; s < ST; ++s) {
            const int it = blockIdx.x + s * Gd;
            if (it >= a.n_items) break;
            fp32_issue<D>(a, S_pool, n_layers_total, kda, it, stages + s * G::STAGE, &bars[s], sc.meta[s]);
        }
    }
    __syncthreads();
    int s = 0;
    uint32_t phase = 0;
    for (int it = blockIdx.x; it < a.n_items; it += Gd) {
        const bool ok = mbar_wait_bounded(&bars[s], phase, a.wait_polls);
        const uint8_t *stage = stages + s * G::STAGE;
        const int valid = sc.meta[s][0], row = sc.meta[s][1];
        float *Sg = S_pool + ((size_t)(uint32_t)sc.meta[s][2] | ((size_t)(uint32_t)sc.meta[s][3] << 32));
        const float *tile = reinterpret_cast<const float *>(stage);
        const float *tf = reinterpret_cast<const float *>(stage + G::TILE);
        bool abort = false;
        if (valid) {
            const float *qs = tf, *ks = tf + D, *vs = tf + 2 * D, *als = tf + 3 * D;
            const float beta = tf[4 * D + 1];
            if (l < RT) {  // this band's rows (read by the band's own warp), duplicated for the packed products
                const int i = g * RT + l;
                const float al = kda ? als[i] : tf[4 * D];
                sc.k2[i] = make_float2(ks[i], ks[i]);
                sc.q2[i] = make_float2(qs[i], qs[i]);
                sc.a2[i] = make_float2(al, al);
            }
            __syncwarp();
            float2 S[RT][2];
            float2 E[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)}, O[2] = {E[0], E[1]};
#pragma unroll
            for (int r = 0; r < RT; ++r) {
                const int i = g * RT + r;
                const float4 x = *reinterpret_cast<const float4 *>(tile + (size_t)i * D + j0);
                const float2 a2 = sc.a2[i], k2 = sc.k2[i];
                S[r][0] = mul2(a2, make_float2(x.x, x.y));
                S[r][1] = mul2(a2, make_float2(x.z, x.w));
#pragma unroll
                for (int hp = 0; hp < 2; ++hp) {
                    if (r & 1) O[hp] = fma2(k2, S[r][hp], O[hp]);
                    else E[hp] = fma2(k2, S[r][hp], E[hp]);
                }
            }
            *reinterpret_cast<float4 *>(&sc.pb[g][j0]) =
                make_float4(E[0].x + O[0].x, E[0].y + O[0].y, E[1].x + O[1].x, E[1].y + O[1].y);
            abort = __syncthreads_or(!ok);
            if (!abort) {
                {  // u and w, two threads per column
                    const int j = tid >> 1, b0 = 4 * (tid & 1);
                    float u = (sc.pb[b0][j] + sc.pb[b0 + 1][j]) + (sc.pb[b0 + 2][j] + sc.pb[b0 + 3][j]);
                    u = u + __shfl_xor_sync(0xffffffffu, u, 1);
                    if ((tid & 1) == 0) sc.wv[j] = __fmul_rn(beta, __fsub_rn(vs[j], u));
                }
                __syncthreads();
                // every read of this stage is done: put item it + ST G into it
                if (tid == 0 && it + ST * Gd < a.n_items)
                    fp32_issue<D>(a, S_pool, n_layers_total, kda, it + ST * Gd, stages + s * G::STAGE, &bars[s],
                                  sc.meta[s]);
                const float4 w4 = *reinterpret_cast<const float4 *>(&sc.wv[j0]);
                const float2 w01 = make_float2(w4.x, w4.y), w23 = make_float2(w4.z, w4.w);
                E[0] = E[1] = O[0] = O[1] = make_float2(0.0f, 0.0f);
#pragma unroll
                for (int r = 0; r < RT; ++r) {
                    const int i = g * RT + r;
                    const float2 k2 = sc.k2[i], q2 = sc.q2[i];
                    S[r][0] = fma2(k2, w01, S[r][0]);
                    S[r][1] = fma2(k2, w23, S[r][1]);
#pragma unroll
                    for (int hp = 0; hp < 2; ++hp) {
                        if (r & 1) O[hp] = fma2(q2, S[r][hp], O[hp]);
                        else E[hp] = fma2(q2, S[r][hp], E[hp]);
                    }
                    *reinterpret_cast<float4 *>(Sg + (size_t)i * D + j0) = make_float4(S[r][0].x, S[r][0].y, S[r][1].x, S[r][1].y);
                }
                *reinterpret_cast<float4 *>(&sc.pb[g][j0]) =
                    make_float4(E[0].x + O[0].x, E[0].y + O[0].y, E[1].x + O[1].x, E[1].y + O[1].y);
                __syncthreads();
                {
                    const int j = tid >> 1, b0 = 4 * (tid & 1);
                    float o = (sc.pb[b0][j] + sc.pb[b0 + 1][j]) + (sc.pb[b0 + 2][j] + sc.pb[b0 + 3][j]);
                    o = o + __shfl_xor_sync(0xffffffffu, o, 1);
                    if ((tid & 1) == 0) a.o[(size_t)row * D + j] = o;
                }
                __syncthreads();
            }
        } else {
            abort = __syncthreads_or(!ok);
            if (!abort && tid == 0 && it + ST * Gd < a.n_items)
                fp32_issue<D>(a, S_pool, n_layers_total, kda, it + ST * Gd, stages + s * G::STAGE, &bars[s], sc.meta[s]);
        }
        if (abort) {
            if (tid == 0) {
                flag_error(a.err, kErrWait);
                cp_async_wait_all();
                for (int k = 0; k < ST; ++k) mbar_wait_bounded(&bars[k], phase ^ (k < s ? 1u : 0u), a.wait_polls);
            }
            return;
        }
        if (++s == ST) {
            s = 0;
            phase ^= 1u;
        }
    }
}

template <int D>
static cudaError_t launch_fp32_d(const Args &a, float *S_pool, int n_layers_total, int n_sms, cudaStream_t st) {
    using G = Fp32Geo<D>;
    const size_t smem = (size_t)G::STAGES * G::STAGE + 64 + sizeof(Fp32Scratch<D>);
    const int kda = a.mode == 1;
    cudaError_t e = cudaFuncSetAttribute(k_fp32_step<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_fp32_step<D>, 2 * D, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    int grid = n_sms * per_sm;
    if (grid > a.n_items) grid = a.n_items;
    k_fp32_step<D><<<grid, 2 * D, smem, st>>>(a, S_pool, n_layers_total, kda);
    return cudaGetLastError();
}

cudaError_t launch_fp32_step(int D, const Args &a, float *S_pool, int n_layers_total, int n_sms, cudaStream_t st) {
    if (a.n_items <= 0) return cudaSuccess;
    switch (D) {
        case 16: return launch_fp32_d<16>(a, S_pool, n_layers_total, n_sms, st);
        case 32: return launch_fp32_d<32>(a, S_pool, n_layers_total, n_sms, st);
        case 64: return launch_fp32_d<64>(a, S_pool, n_layers_total, n_sms, st);
        case 128: return launch_fp32_d<128>(a, S_pool, n_layers_total, n_sms, st);
        default: return cudaErrorInvalidValue;
    }
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
