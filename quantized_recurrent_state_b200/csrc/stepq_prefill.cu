// Chunked prefill of per-head states (the step before decode).
//
// A prompt of T tokens runs the same gated delta rule as the decode step
// (STEPQuant paper digest page, 背景与动机), with a scalar gate alpha_t per
// (token, head):  S_t = (I - beta_t k_t k_t^T) alpha_t S_{t-1} + beta_t k_t v_t^T,
// o_t = S_t^T q_t.  In chunks of C = 64 tokens from S_0, with gamma_t the
// running gate product inside the chunk and Gamma_ts = gamma_t / gamma_s:
//   (I + M) U = V - diag(gamma) K S_0,   M_ts = Gamma_ts beta_s (k_t . k_s), s < t
//   O   = diag(gamma) Q S_0 + (L_incl(Q K^T o Gamma) diag(beta)) U
//   S_C = gamma_C S_0 + K^T diag(beta gamma_C / gamma) U
// The seven dense products per chunk run on the tensor cores as
// mma.m16n8k8 TF32 with each fp32 operand split into a TF32 high part and a
// TF32 remainder (three products per tile: hi*hi + hi*lo + lo*hi), which keeps
// them near fp32 accuracy; the unit-lower-triangular solve for U runs on the
// CUDA cores, each warp owning 16 value columns.
//
// One CTA of 256 threads per (request, layer, head) prompt, the fp32 state
// and the chunk's Q, K, V in shared memory (rows padded to avoid bank
// conflicts).  Head dimension 128.
#include "stepq_dev.cuh"
#include "stepq_prefill.cuh"

namespace stepq {

namespace pf {

constexpr int D = 128;         // d_k = d_v
constexpr int C = 64;          // tokens per chunk
constexpr int NT = 256;        // threads
constexpr int SD = D + 4;      // padded row of a 128-wide tile
constexpr int SC = C + 4;      // padded row of a 64-wide tile

struct Smem {
    float S[D * SD];           // state, row i (key) x column j (value)
    float K[C * SD];
    float Q[C * SD];
    float V[C * SD];           // V, then R = V - diag(gamma) K S, then U
    float M[C * SC];           // M (strict lower), then A (lower incl.)
    float lg[C];               // inclusive running sum of log alpha in the chunk
    float beta[C];
    float f[C];                // beta_s gamma_C / gamma_s
};

__device__ __forceinline__ uint32_t tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ void split(float x, uint32_t &hi, uint32_t &lo) {
    hi = tf32(x);
    lo = tf32(x - __uint_as_float(hi));
}

__device__ __forceinline__ void mma(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// acc[nt] += A[m0 .. m0+16, 0 .. KK) B[0 .. KK, n0 + 8 nt .. + 8) for one warp.
// A(r, c) = sA[r ars + c acs]; B(r, c) = sB[r brs + c bcs] (times bsc[r] when given).
// Fragment of acc[nt]: [0] (m0+g, n0+8nt+2t), [1] (.., +1), [2] (m0+g+8, ..), [3] (.., +1).
template <int NTILE, int KK>
__device__ __forceinline__ void warp_gemm(float (&acc)[NTILE][4], const float *sA, int ars, int acs, const float *sB,
                                          int brs, int bcs, const float *bsc, int m0, int n0, int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll 1
    for (int k0 = 0; k0 < KK; k0 += 8) {
        uint32_t ah[4], al[4];
        split(sA[(m0 + g) * ars + (k0 + t) * acs], ah[0], al[0]);
        split(sA[(m0 + g + 8) * ars + (k0 + t) * acs], ah[1], al[1]);
        split(sA[(m0 + g) * ars + (k0 + t + 4) * acs], ah[2], al[2]);
        split(sA[(m0 + g + 8) * ars + (k0 + t + 4) * acs], ah[3], al[3]);
        const float s0 = bsc ? bsc[k0 + t] : 1.0f, s1 = bsc ? bsc[k0 + t + 4] : 1.0f;
#pragma unroll
        for (int nt = 0; nt < NTILE; ++nt) {
            const int n = n0 + 8 * nt + g;
            uint32_t bh[2], bl[2];
            split(sB[(k0 + t) * brs + n * bcs] * s0, bh[0], bl[0]);
            split(sB[(k0 + t + 4) * brs + n * bcs] * s1, bh[1], bl[1]);
            mma(acc[nt], ah, bh);
            mma(acc[nt], ah, bl);
            mma(acc[nt], al, bh);
        }
    }
}

template <int NTILE>
__device__ __forceinline__ void zero(float (&acc)[NTILE][4]) {
#pragma unroll
    for (int nt = 0; nt < NTILE; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.0f;
}

}  // namespace pf

__global__ void __launch_bounds__(pf::NT, 1) k_prefill(PrefillArgs a) {
    using namespace pf;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int g = lane >> 2, t4 = lane & 3;
    const int item = blockIdx.x;               // (n, ll, h)
    const int per_req = a.nL * a.H;
    const int n = item / per_req, rem = item - n * per_req, ll = rem / a.H, h = rem - ll * a.H;
    float *Sg = a.S + (size_t)item * D * D;

    // the state
    for (int e = tid; e < D * D / 4; e += NT) {
        const int i = e / (D / 4), j4 = e % (D / 4);
        const float4 x = a.zero_init ? make_float4(0.f, 0.f, 0.f, 0.f) : reinterpret_cast<const float4 *>(Sg)[e];
        *reinterpret_cast<float4 *>(&sm.S[i * SD + 4 * j4]) = x;
    }

    for (int c0 = 0; c0 < a.T; c0 += C) {
        const int cc = min(C, a.T - c0);
        __syncthreads();  // the previous chunk is done with K, Q, V, M
        // 1. the chunk's rows (padded rows: zeros, alpha = 1, beta = 0)
        for (int e = tid; e < C * D / 4; e += NT) {
            const int r = e / (D / 4), j4 = e % (D / 4);
            float4 kx = make_float4(0.f, 0.f, 0.f, 0.f), qx = kx, vx = kx;
            if (r < cc) {
                const size_t row = ((size_t)(n * a.T + c0 + r) * a.nL_in + a.l_in0 + ll) * a.H + h;
                kx = reinterpret_cast<const float4 *>(a.k + row * D)[j4];
                qx = reinterpret_cast<const float4 *>(a.q + row * D)[j4];
                vx = reinterpret_cast<const float4 *>(a.v + row * D)[j4];
            }
            *reinterpret_cast<float4 *>(&sm.K[r * SD + 4 * j4]) = kx;
            *reinterpret_cast<float4 *>(&sm.Q[r * SD + 4 * j4]) = qx;
            *reinterpret_cast<float4 *>(&sm.V[r * SD + 4 * j4]) = vx;
        }
        if (w == 0) {  // gates: inclusive scan of log alpha over the 64 tokens, 2 per lane
            float l2[2], b2[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int r = 2 * lane + u;
                l2[u] = 0.0f;
                b2[u] = 0.0f;
                if (r < cc) {
                    const size_t row = ((size_t)(n * a.T + c0 + r) * a.nL_in + a.l_in0 + ll) * a.H + h;
                    l2[u] = logf(a.alpha[row]);
                    b2[u] = a.beta[row];
                }
            }
            float s = l2[0] + l2[1];
#pragma unroll
            for (int m = 1; m < 32; m <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, s, m);
                if (lane >= m) s += y;
            }
            const float excl = s - (l2[0] + l2[1]);
            sm.lg[2 * lane] = excl + l2[0];
            sm.lg[2 * lane + 1] = s;
            sm.beta[2 * lane] = b2[0];
            sm.beta[2 * lane + 1] = b2[1];
        }
        __syncthreads();
        if (tid < C) sm.f[tid] = sm.beta[tid] * expf(sm.lg[C - 1] - sm.lg[tid]);
        // 2. M = strict_lower(K K^T o Gamma) diag(beta)  and  R = V - diag(gamma) K S
        {
            float acc[4][4];
            zero(acc);
            const int m0 = 16 * (w >> 1), n0 = 32 * (w & 1);
            warp_gemm<4, D>(acc, sm.K, SD, 1, sm.K, 1, SD, nullptr, m0, n0, lane);
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int r = m0 + g + 8 * (e >> 1), s = n0 + 8 * nt + 2 * t4 + (e & 1);
                    sm.M[r * SC + s] = (s < r) ? acc[nt][e] * expf(sm.lg[r] - sm.lg[s]) * sm.beta[s] : 0.0f;
                }
        }
        {
            float acc[8][4];
            zero(acc);
            const int m0 = 16 * (w >> 1), n0 = 64 * (w & 1);
            warp_gemm<8, D>(acc, sm.K, SD, 1, sm.S, SD, 1, nullptr, m0, n0, lane);
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int r = m0 + g + 8 * (e >> 1), j = n0 + 8 * nt + 2 * t4 + (e & 1);
                    sm.V[r * SD + j] -= expf(sm.lg[r]) * acc[nt][e];
                }
        }
        __syncthreads();
        // 3. U = (I + M)^-1 R in place: warp w owns value columns [16 w, 16 w + 16),
        //    two lanes per column (even / odd s), rows in order
        {
            const int j = 16 * w + (lane & 15), hs = lane >> 4;
            for (int r = 1; r < C; ++r) {
                float part = 0.0f;
                for (int s = hs; s < r; s += 2) part += sm.M[r * SC + s] * sm.V[s * SD + j];
                part += __shfl_xor_sync(0xffffffffu, part, 16);
                if (hs == 0) sm.V[r * SD + j] -= part;
                __syncwarp();
            }
        }
        __syncthreads();
        // 4. A = L_incl(Q K^T o Gamma) diag(beta) into M
        {
            float acc[4][4];
            zero(acc);
            const int m0 = 16 * (w >> 1), n0 = 32 * (w & 1);
            warp_gemm<4, D>(acc, sm.Q, SD, 1, sm.K, 1, SD, nullptr, m0, n0, lane);
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int r = m0 + g + 8 * (e >> 1), s = n0 + 8 * nt + 2 * t4 + (e & 1);
                    sm.M[r * SC + s] = (s <= r) ? acc[nt][e] * expf(sm.lg[r] - sm.lg[s]) * sm.beta[s] : 0.0f;
                }
        }
        __syncthreads();
        // 5. O = diag(gamma) Q S + A U, rows of this chunk to global
        {
            float acc[8][4], acc2[8][4];
            zero(acc);
            zero(acc2);
            const int m0 = 16 * (w >> 1), n0 = 64 * (w & 1);
            warp_gemm<8, D>(acc, sm.Q, SD, 1, sm.S, SD, 1, nullptr, m0, n0, lane);
            warp_gemm<8, C>(acc2, sm.M, SC, 1, sm.V, SD, 1, nullptr, m0, n0, lane);
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int e2 = 0; e2 < 2; ++e2) {
                    const int r = m0 + g + 8 * e2, j = n0 + 8 * nt + 2 * t4;
                    if (r < cc) {
                        const float gm = expf(sm.lg[r]);
                        const size_t row = ((size_t)(n * a.T + c0 + r) * a.nL_in + a.l_in0 + ll) * a.H + h;
                        *reinterpret_cast<float2 *>(a.o + row * D + j) =
                            make_float2(gm * acc[nt][2 * e2] + acc2[nt][2 * e2], gm * acc[nt][2 * e2 + 1] + acc2[nt][2 * e2 + 1]);
                    }
                }
        }
        __syncthreads();  // every read of the old state is done
        // 6. S = gamma_C S + K^T diag(f) U, warp w updates state rows [16 w, 16 w + 16)
        {
            const float gC = expf(sm.lg[C - 1]);
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                float acc[8][4];
                zero(acc);
                const int m0 = 16 * w, n0 = 64 * half;
                warp_gemm<8, C>(acc, sm.K, 1, SD, sm.V, SD, 1, sm.f, m0, n0, lane);
#pragma unroll
                for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int i = m0 + g + 8 * (e >> 1), j = n0 + 8 * nt + 2 * t4 + (e & 1);
                        sm.S[i * SD + j] = gC * sm.S[i * SD + j] + acc[nt][e];
                    }
            }
        }
    }
    __syncthreads();
    for (int e = tid; e < D * D / 4; e += NT) {
        const int i = e / (D / 4), j4 = e % (D / 4);
        reinterpret_cast<float4 *>(Sg)[e] = *reinterpret_cast<const float4 *>(&sm.S[i * SD + 4 * j4]);
    }
}

size_t prefill_smem_bytes() { return sizeof(pf::Smem); }

cudaError_t launch_prefill(const PrefillArgs &a, cudaStream_t st) {
    const int items = a.n_req * a.nL * a.H;
    if (items <= 0 || a.T <= 0) return cudaSuccess;
    const size_t smem = sizeof(pf::Smem);
    cudaError_t e = cudaFuncSetAttribute(k_prefill, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k_prefill<<<items, pf::NT, smem, st>>>(a);
    return cudaGetLastError();
}

}  // namespace stepq
