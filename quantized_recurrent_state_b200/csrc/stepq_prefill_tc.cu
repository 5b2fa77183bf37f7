// Chunked prefill of per-head states with the state in tensor memory (tcgen05).
//
// The same chunk form as k_prefill (stepq_prefill.cu) for per-head gates, d = 128,
// C = 64, one CTA of 256 threads per (request, layer, head).  The state S^T
// (lane j = value column, column i = key row) lives in tensor memory in fp32 with its
// TF32 remainder beside it; it is the A operand of the two state products
// W^T = S^T K^T and Y^T = S^T Q^T and the accumulator of the update
// S^T <- Gamma_C S^T + (U diag(f))^T K, all three on tcgen05 kind::tf32 in three passes
// (hi*hi, hi*lo, lo*hi).  K and Q arrive once per chunk as TF32 hi/lo tiles in the
// K-major core layout (stepq_tc.cuh), which the tcgen05 products read as their B
// operand and the mma.sync products (K K^T, Q K^T) read as pre-split fragments; K^T
// is built from them for the update.  The block solve and A U stay on mma.sync.
//
// Tensor memory: S^T 0..127, its remainder 128..255, W^T 256..319, Y^T 320..383,
// (U f)^T hi 384..447 and lo 448..511 (all 512 columns: one CTA per SM, which the
// shared memory (about 181 KB) guarantees).  Every tcgen05 wait is bounded; a wait
// that gives up sets kErrWait, lets the issued products finish (bounded) and frees the
// columns.
#include "stepq_dev.cuh"
#include "stepq_prefill.cuh"
#include "stepq_tc.cuh"

namespace stepq {

namespace tcpf {

constexpr int D = 128, C = 64, NT = 256;
constexpr int SV = D + 8, SC = C + 4;
constexpr uint32_t kPolls = 1u << 24;
// tensor-memory columns
constexpr uint32_t TS = 0, TSL = 128, TW = 256, TY = 320, TUH = 384, TUL = 448, NCOLS = 512;

struct Smem {
    alignas(1024) float Xhi[C * D];   // K then Q, K-major cores: tc::kmajor_off(t, i, D)
    alignas(1024) float Xlo[C * D];
    alignas(1024) float KThi[D * C];  // K^T: tc::kmajor_off(i, t, C)
    alignas(1024) float KTlo[D * C];
    float V[C * SV];                  // V, R, U, then A U
    float M[C * SC];
    float lg[C], gam[C], beta[C], f[C];
    alignas(8) uint64_t bar[3];
    uint32_t taddr;
};

__device__ __forceinline__ uint32_t tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ void split(float x, float &hi, float &lo) {
    hi = __uint_as_float(tf32(x));
    lo = __uint_as_float(tf32(x - hi));
}
__device__ __forceinline__ void split_u(float x, uint32_t &hi, uint32_t &lo) {
    hi = tf32(x);
    lo = tf32(x - __uint_as_float(hi));
}
__device__ __forceinline__ void mma(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
template <int NTILE>
__device__ __forceinline__ void zero(float (&acc)[NTILE][4]) {
#pragma unroll
    for (int nt = 0; nt < NTILE; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.0f;
}

// fp32 operands split on the fly: acc[nt] += A[m0.., 0..kk) B[0..kk, n0 + 8 nt ..]
template <int NTILE>
__device__ __forceinline__ void warp_gemm(float (&acc)[NTILE][4], const float *sA, int ars, int acs, const float *sB,
                                          int brs, int bcs, int m0, int n0, int kk, int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll 1
    for (int k0 = 0; k0 < kk; k0 += 8) {
        uint32_t ah[4], al[4];
        split_u(sA[(m0 + g) * ars + (k0 + t) * acs], ah[0], al[0]);
        split_u(sA[(m0 + g + 8) * ars + (k0 + t) * acs], ah[1], al[1]);
        split_u(sA[(m0 + g) * ars + (k0 + t + 4) * acs], ah[2], al[2]);
        split_u(sA[(m0 + g + 8) * ars + (k0 + t + 4) * acs], ah[3], al[3]);
        uint32_t bh[NTILE][2], bl[NTILE][2];
#pragma unroll
        for (int nt = 0; nt < NTILE; ++nt) {
            const int n = n0 + 8 * nt + g;
            split_u(sB[(k0 + t) * brs + n * bcs], bh[nt][0], bl[nt][0]);
            split_u(sB[(k0 + t + 4) * brs + n * bcs], bh[nt][1], bl[nt][1]);
        }
#pragma unroll
        for (int nt = 0; nt < NTILE; ++nt) mma(acc[nt], ah, bh[nt]);
#pragma unroll
        for (int nt = 0; nt < NTILE; ++nt) mma(acc[nt], ah, bl[nt]);
#pragma unroll
        for (int nt = 0; nt < NTILE; ++nt) mma(acc[nt], al, bh[nt]);
    }
}

// Pre-split operands in core layout: A(r, c) at offset aoff(r, c) of Ah/Al, B(k, n) at
// boff(k, n) of Bh/Bl (word offsets).  acc[nt] += A[m0.., 0..kk) B[0..kk, n0 + 8 nt ..]
template <int NTILE, class AOFF, class BOFF>
__device__ __forceinline__ void warp_gemm_split(float (&acc)[NTILE][4], const float *Ah, const float *Al, AOFF aoff,
                                                const float *Bh, const float *Bl, BOFF boff, int m0, int n0, int kk,
                                                int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll 2
    for (int k0 = 0; k0 < kk; k0 += 8) {
        uint32_t ah[4], al[4];
        const int ao[4] = {aoff(m0 + g, k0 + t), aoff(m0 + g + 8, k0 + t), aoff(m0 + g, k0 + t + 4),
                           aoff(m0 + g + 8, k0 + t + 4)};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            ah[u] = __float_as_uint(Ah[ao[u]]);
            al[u] = __float_as_uint(Al[ao[u]]);
        }
        uint32_t bh[NTILE][2], bl[NTILE][2];
#pragma unroll
        for (int nt = 0; nt < NTILE; ++nt) {
            const int n = n0 + 8 * nt + g;
            const int b0 = boff(k0 + t, n), b1 = boff(k0 + t + 4, n);
            bh[nt][0] = __float_as_uint(Bh[b0]);
            bl[nt][0] = __float_as_uint(Bl[b0]);
            bh[nt][1] = __float_as_uint(Bh[b1]);
            bl[nt][1] = __float_as_uint(Bl[b1]);
        }
#pragma unroll
        for (int nt = 0; nt < NTILE; ++nt) mma(acc[nt], ah, bh[nt]);
#pragma unroll
        for (int nt = 0; nt < NTILE; ++nt) mma(acc[nt], ah, bl[nt]);
#pragma unroll
        for (int nt = 0; nt < NTILE; ++nt) mma(acc[nt], al, bh[nt]);
    }
}

__device__ __forceinline__ int xoff(int t, int i) { return (int)(tc::kmajor_off(t, i, D) >> 2); }   // X[t][i]
__device__ __forceinline__ int ktoff(int i, int t) { return (int)(tc::kmajor_off(i, t, C) >> 2); }  // KT[i][t]

// TF32 hi/lo split of the chunk's rows of x (K or Q) into X (rows past cc are 0).  An
// iteration covers one 8-row core group: thread -> row 8 it + (tid % 8), columns
// 4 (tid / 8) .. + 3, so a quarter warp writes eight consecutive 16-byte core rows.
template <class RowOf>
__device__ __forceinline__ void split_rows(Smem &sm, const float *x, RowOf row_of, int c0, int cc, int tid) {
#pragma unroll 4
    for (int it = 0; it < C / 8; ++it) {
        const int r = 8 * it + (tid & 7), i = 4 * (tid >> 3);
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (r < cc) v = *reinterpret_cast<const float4 *>(x + row_of(c0 + r) + i);
        float4 hi, lo;
        split(v.x, hi.x, lo.x); split(v.y, hi.y, lo.y); split(v.z, hi.z, lo.z); split(v.w, hi.w, lo.w);
        *reinterpret_cast<float4 *>(&sm.Xhi[xoff(r, i)]) = hi;
        *reinterpret_cast<float4 *>(&sm.Xlo[xoff(r, i)]) = lo;
    }
}

__global__ void __launch_bounds__(NT, 1) k_prefill_tc(PrefillArgs a) {
    extern __shared__ __align__(1024) uint8_t smraw[];
    Smem &sm = *reinterpret_cast<Smem *>(smraw);
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int g = lane >> 2, t4 = lane & 3;
    const int item = blockIdx.x;
    const int per_req = a.nL * a.H;
    const int n = item / per_req, rem = item - n * per_req, ll = rem / a.H, h = rem - ll * a.H;
    float *Sg = a.S + (size_t)item * D * D;
    auto row_of = [&](int tok) { return (((size_t)(n * a.T + tok) * a.nL_in + a.l_in0 + ll) * a.H + h) * D; };
    // the k, q, v rows of the chunk from token c0 into L2 ahead of their (synchronous) loads
    auto prefetch_chunk = [&](int c0) {
        const int cc = min(C, a.T - c0);
        if (tid < 3 * cc) {
            const int r = tid / 3, which = tid - 3 * r;
            const float *base = which == 0 ? a.k : which == 1 ? a.q : a.v;
            asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(base + row_of(c0 + r)), "r"(D * 4)
                         : "memory");
        }
    };
    const int q4 = w & 3, hh = w >> 2;               // this warp's lane quadrant and half
    const int j = 32 * q4 + lane;                    // the lane (value column j) this thread reads in tensor memory
    const uint32_t quad = (uint32_t)(32 * q4) << 16;
    auto xo = [](int r, int c) { return xoff(r, c); };
    auto xo_t = [](int k, int nn) { return xoff(nn, k); };
    auto kto = [](int k, int nn) { return ktoff(k, nn); };

    prefetch_chunk(0);
    if (tid == 0)
        for (int b = 0; b < 3; ++b) tc::mbar_init(&sm.bar[b]);
    if (w == 0) tc::alloc(&sm.taddr, NCOLS);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tm = sm.taddr;

    // S_0 into TS (lane j, column i) and its remainder into TSL
#pragma unroll 1
    for (int p = 0; p < 2; ++p) {
        const int i0 = 64 * hh + 32 * p;
        uint32_t v[32], l[32];
#pragma unroll
        for (int u = 0; u < 32; ++u) {
            const float s = a.zero_init ? 0.0f : Sg[(size_t)(i0 + u) * D + j];
            v[u] = __float_as_uint(s);
            l[u] = __float_as_uint(s - __uint_as_float(v[u] & 0xFFFFE000u));
        }
        tc::st32(tm + quad + TS + i0, v);
        tc::st32(tm + quad + TSL + i0, l);
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();

    bool ok = true;
    int ci = 0;
#pragma unroll 1
    for (int c0 = 0; c0 < a.T && ok; c0 += C, ++ci) {
        const int cc = min(C, a.T - c0);
        const uint32_t par = ci & 1;
        if (c0 + C < a.T) prefetch_chunk(c0 + C);
        // 1. K split into X, V, gates.  The split tiles are written 8 rows x 4 columns per
        // quarter warp (row fastest): eight consecutive 16-byte core rows, free of bank
        // conflicts; V keeps rows of consecutive columns per warp.
        split_rows(sm, a.k, row_of, c0, cc, tid);
#pragma unroll 4
        for (int e = tid; e < C * D / 4; e += NT) {
            const int r = e / (D / 4), i = 4 * (e % (D / 4));
            float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
            if (r < cc) y = *reinterpret_cast<const float4 *>(a.v + row_of(c0 + r) + i);
            *reinterpret_cast<float4 *>(&sm.V[r * SV + i]) = y;
        }
        if (w == 0) {
            float l2[2], b2[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int r = 2 * lane + u;
                l2[u] = 0.0f;
                b2[u] = 0.0f;
                if (r < cc) {
                    const size_t gi = row_of(c0 + r) / D;
                    l2[u] = logf(a.alpha[gi]);
                    b2[u] = a.beta[gi];
                }
            }
            if (!(isfinite(l2[0]) && isfinite(l2[1]))) atomicOr(a.err, kErrGateRange);
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
        // K^T from X: warp w fills whole 8 x 4 cores (lane = i offset * 4 + t offset)
        for (int cidx = w; cidx < (D / 8) * (C / 4); cidx += NT / 32) {
            const int i = 8 * (cidx / (C / 4)) + (lane >> 2), t = 4 * (cidx % (C / 4)) + (lane & 3);
            sm.KThi[ktoff(i, t)] = sm.Xhi[xoff(t, i)];
            sm.KTlo[ktoff(i, t)] = sm.Xlo[xoff(t, i)];
        }
        if (tid < C) {
            sm.f[tid] = sm.beta[tid] * expf(sm.lg[C - 1] - sm.lg[tid]);
            sm.gam[tid] = expf(sm.lg[tid]);
        }
        tc::fence_smem_to_async();
        tc::fence_before();
        __syncthreads();
        tc::fence_after();
        // 2. W^T = S^T K^T on tcgen05 (three passes), meanwhile M = K K^T on mma.sync
        if (tid == 0) {
            const uint32_t id = tc::idesc_tf32(128, C);
            const uint32_t xh = tc::smem_addr(sm.Xhi), xl = tc::smem_addr(sm.Xlo);
            for (int kk = 0; kk < D / 8; ++kk) tc::mma_ts(tm + TW, tm + TS + 8 * kk, tc::kmajor_desc(xh, D, kk), id, kk > 0);
            for (int kk = 0; kk < D / 8; ++kk) tc::mma_ts(tm + TW, tm + TS + 8 * kk, tc::kmajor_desc(xl, D, kk), id, 1);
            for (int kk = 0; kk < D / 8; ++kk) tc::mma_ts(tm + TW, tm + TSL + 8 * kk, tc::kmajor_desc(xh, D, kk), id, 1);
            tc::commit(&sm.bar[0]);
        }
        {
            float acc[4][4];
            zero(acc);
            const int m0 = 16 * (w >> 1), n0 = 32 * (w & 1);
            warp_gemm_split<4>(acc, sm.Xhi, sm.Xlo, xo, sm.Xhi, sm.Xlo, xo_t, m0, n0, D, lane);
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int r = m0 + g + 8 * (e >> 1), s = n0 + 8 * nt + 2 * t4 + (e & 1);
                    sm.M[r * SC + s] = (s < r) ? acc[nt][e] * expf(sm.lg[r] - sm.lg[s]) * sm.beta[s] : 0.0f;
                }
        }
        // 3. R = V - gamma_t W
        ok = tc::mbar_wait(&sm.bar[0], par, kPolls);
        ok = __syncthreads_and(ok);
        if (!ok) break;
        tc::fence_after();
        {
            uint32_t v[32];
            tc::ld32(tm + quad + TW + 32 * hh, v);
#pragma unroll
            for (int u = 0; u < 32; ++u) {
                const int t = 32 * hh + u;
                sm.V[t * SV + j] -= sm.gam[t] * __uint_as_float(v[u]);
            }
        }
        __syncthreads();
        // Q split into X
        split_rows(sm, a.q, row_of, c0, cc, tid);
        tc::fence_smem_to_async();
        tc::fence_before();
        __syncthreads();
        tc::fence_after();
        // 4. Y^T = S^T Q^T on tcgen05, meanwhile the block solve
        if (tid == 0) {
            const uint32_t id = tc::idesc_tf32(128, C);
            const uint32_t xh = tc::smem_addr(sm.Xhi), xl = tc::smem_addr(sm.Xlo);
            for (int kk = 0; kk < D / 8; ++kk) tc::mma_ts(tm + TY, tm + TS + 8 * kk, tc::kmajor_desc(xh, D, kk), id, kk > 0);
            for (int kk = 0; kk < D / 8; ++kk) tc::mma_ts(tm + TY, tm + TS + 8 * kk, tc::kmajor_desc(xl, D, kk), id, 1);
            for (int kk = 0; kk < D / 8; ++kk) tc::mma_ts(tm + TY, tm + TSL + 8 * kk, tc::kmajor_desc(xh, D, kk), id, 1);
            tc::commit(&sm.bar[1]);
        }
        if (w < 4) {   // diagonal block inverses
            const int r0 = 16 * w, c = lane & 15;
            float tc_[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                float acc = 0.0f;
#pragma unroll
                for (int s2 = 0; s2 < r; ++s2) acc = fmaf(sm.M[(r0 + r) * SC + r0 + s2], tc_[s2], acc);
                tc_[r] = (r == c) ? 1.0f : (r < c ? 0.0f : -acc);
            }
            __syncwarp();
            if (lane < 16) {
#pragma unroll
                for (int r = 0; r < 16; ++r) sm.M[(r0 + r) * SC + r0 + c] = tc_[r];
            }
        }
        __syncthreads();
        {
            const int jw = 16 * w;
#pragma unroll 1
            for (int r0 = 0; r0 < C; r0 += 16) {
                if (r0 > 0) {
                    float acc[2][4];
                    zero(acc);
                    warp_gemm<2>(acc, sm.M, SC, 1, sm.V, SV, 1, r0, jw, r0, lane);
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            sm.V[(r0 + g + 8 * (e >> 1)) * SV + jw + 8 * nt + 2 * t4 + (e & 1)] -= acc[nt][e];
                    __syncwarp();
                }
                float acc[2][4];
                zero(acc);
                warp_gemm<2>(acc, sm.M + r0, SC, 1, sm.V + r0 * SV, SV, 1, r0, jw, 16, lane);
                __syncwarp();
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        sm.V[(r0 + g + 8 * (e >> 1)) * SV + jw + 8 * nt + 2 * t4 + (e & 1)] = acc[nt][e];
                __syncwarp();
            }
        }
        __syncthreads();
        // 5. U f into tensor memory (split), A = L_incl(Q K^T o Gamma) beta, then A U
        {
            uint32_t vh[32], vl[32];
#pragma unroll
            for (int u = 0; u < 32; ++u) {
                const int t = 32 * hh + u;
                split_u(sm.V[t * SV + j] * sm.f[t], vh[u], vl[u]);
            }
            tc::st32(tm + quad + TUH + 32 * hh, vh);
            tc::st32(tm + quad + TUL + 32 * hh, vl);
        }
        {
            float acc[4][4];
            zero(acc);
            const int m0 = 16 * (w >> 1), n0 = 32 * (w & 1);
            warp_gemm_split<4>(acc, sm.Xhi, sm.Xlo, xo, sm.KThi, sm.KTlo, kto, m0, n0, D, lane);
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int r = m0 + g + 8 * (e >> 1), s = n0 + 8 * nt + 2 * t4 + (e & 1);
                    sm.M[r * SC + s] = (s <= r) ? acc[nt][e] * expf(sm.lg[r] - sm.lg[s]) * sm.beta[s] : 0.0f;
                }
        }
        __syncthreads();
        {
            float acc[8][4];
            zero(acc);
            const int m0 = 16 * (w >> 1), n0 = 64 * (w & 1);
            warp_gemm<8>(acc, sm.M, SC, 1, sm.V, SV, 1, m0, n0, C, lane);
            __syncthreads();   // every read of U is done
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    sm.V[(m0 + g + 8 * (e >> 1)) * SV + n0 + 8 * nt + 2 * t4 + (e & 1)] = acc[nt][e];
        }
        __syncthreads();
        // 6. o = gamma_t Y + A U; S^T *= gamma_C
        ok = tc::mbar_wait(&sm.bar[1], par, kPolls);
        ok = __syncthreads_and(ok);
        if (!ok) break;
        tc::fence_after();
        {
            uint32_t v[32];
            tc::ld32(tm + quad + TY + 32 * hh, v);
#pragma unroll
            for (int u = 0; u < 32; ++u) {
                const int t = 32 * hh + u;
                if (t < cc) a.o[row_of(c0 + t) + j] = sm.gam[t] * __uint_as_float(v[u]) + sm.V[t * SV + j];
            }
            const float gC = expf(sm.lg[C - 1]);
#pragma unroll 1
            for (int p = 0; p < 2; ++p) {
                uint32_t s[32];
                tc::ld32(tm + quad + TS + 64 * hh + 32 * p, s);
#pragma unroll
                for (int u = 0; u < 32; ++u) s[u] = __float_as_uint(gC * __uint_as_float(s[u]));
                tc::st32(tm + quad + TS + 64 * hh + 32 * p, s);
            }
        }
        tc::fence_before();
        __syncthreads();
        tc::fence_after();
        // 7. S^T += (U f)^T K on tcgen05 (three passes, N = 128)
        if (tid == 0) {
            const uint32_t id = tc::idesc_tf32(128, D);
            const uint32_t kh = tc::smem_addr(sm.KThi), kl = tc::smem_addr(sm.KTlo);
            for (int kk = 0; kk < C / 8; ++kk) tc::mma_ts(tm + TS, tm + TUH + 8 * kk, tc::kmajor_desc(kh, C, kk), id, 1);
            for (int kk = 0; kk < C / 8; ++kk) tc::mma_ts(tm + TS, tm + TUH + 8 * kk, tc::kmajor_desc(kl, C, kk), id, 1);
            for (int kk = 0; kk < C / 8; ++kk) tc::mma_ts(tm + TS, tm + TUL + 8 * kk, tc::kmajor_desc(kh, C, kk), id, 1);
            tc::commit(&sm.bar[2]);
        }
        // 8. the remainder of the new state for the next chunk's products
        ok = tc::mbar_wait(&sm.bar[2], par, kPolls);
        ok = __syncthreads_and(ok);
        if (!ok) break;
        tc::fence_after();
#pragma unroll 1
        for (int p = 0; p < 2; ++p) {
            uint32_t s[32];
            tc::ld32(tm + quad + TS + 64 * hh + 32 * p, s);
#pragma unroll
            for (int u = 0; u < 32; ++u) s[u] = __float_as_uint(__uint_as_float(s[u]) - __uint_as_float(s[u] & 0xFFFFE000u));
            tc::st32(tm + quad + TSL + 64 * hh + 32 * p, s);
        }
        tc::fence_before();
        __syncthreads();
        tc::fence_after();
    }
    if (ok) {
#pragma unroll 1
        for (int p = 0; p < 2; ++p) {
            uint32_t s[32];
            const int i0 = 64 * hh + 32 * p;
            tc::ld32(tm + quad + TS + i0, s);
#pragma unroll
            for (int u = 0; u < 32; ++u) Sg[(size_t)(i0 + u) * D + j] = __uint_as_float(s[u]);
        }
    } else {
        if (tid == 0) atomicOr(a.err, kErrWait);
        // let the products already issued finish (bounded) before the columns are freed;
        // if one of these waits gives up too, the columns are freed with a product possibly
        // still writing them, which the error word records as its own (fatal) condition
        bool drained = true;
        for (int b = 0; b < 3; ++b) drained = tc::mbar_wait(&sm.bar[b], ci & 1, kPolls) && drained;
        if (!drained && tid == 0) atomicOr(a.err, kErrTmemDrain);
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    if (w == 0) tc::dealloc(tm, NCOLS);
}

}  // namespace tcpf


size_t prefill_tc_smem_bytes() { return sizeof(tcpf::Smem); }

cudaError_t launch_prefill_tc(const PrefillArgs &a, cudaStream_t st) {
    const int items = a.n_req * a.nL * a.H;
    if (items <= 0 || a.T <= 0) return cudaSuccess;
    const size_t smem = sizeof(tcpf::Smem);
    cudaError_t e = cudaFuncSetAttribute(tcpf::k_prefill_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    tcpf::k_prefill_tc<<<items, tcpf::NT, smem, st>>>(a);
    return cudaGetLastError();
}

}  // namespace stepq
