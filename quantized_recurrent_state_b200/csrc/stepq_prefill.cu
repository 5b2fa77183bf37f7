// Chunked prefill of per-head and per-key-row states (the step before decode).
//
// A prompt of T tokens runs the same gated delta rule as the decode step
// (STEPQuant paper digest page, 背景与动机), gate first:
// S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T and
// o_t = S_t^T q_t, with alpha_t a scalar per (token, head) for per-head units
// or a vector over the key rows for per-row units.  In chunks of C = 64
// tokens from S_0, with Gamma_t the running gate product inside the chunk
// (per key row for per-row gates):
//   (I + M) U = V - (K o Gamma) S_0,  M_ts = beta_s sum_i k_ti k_si Gamma_ti / Gamma_si, s < t
//   O   = (Q o Gamma) S_0 + L_incl(A) U,  A_ts = beta_s sum_i q_ti k_si Gamma_ti / Gamma_si
//   S_C = Diag(Gamma_C) S_0 + (K o (Gamma_C / Gamma) o beta)^T U
// For per-head gates the ratios are one factor per (t, s) pair; per-row gates
// are factored per key row around the chunk's middle token (see k_prefill).
//
// The dense products run on the tensor cores as mma.m16n8k8 TF32 warp tiles
// with each fp32 operand split into a TF32 high part and a TF32 remainder
// (three products per tile: hi*hi + hi*lo + lo*hi), which keeps them near
// fp32 accuracy.  The unit lower triangular solve for U goes in blocks of 16
// rows: four warps invert the diagonal blocks by substitution in registers,
// then each warp forms its 16 value columns of every block with two small
// tensor-core products.
//
// One CTA of 256 threads per (request, layer, head) prompt holds the fp32
// state and the chunk's K, Q, V, M in shared memory (row strides chosen for
// conflict-free fragment loads); the next chunk's K (per-head gates) and Q
// arrive by cp.async while the current chunk is computed.  Head dimension 128.
#include "stepq_dev.cuh"
#include "stepq_prefill.cuh"

namespace stepq {

namespace pf {

constexpr int D = 128;         // d_k = d_v
constexpr int C = 64;          // tokens per chunk
constexpr int NT = 256;        // threads
constexpr int SD = D + 4;      // row of K, Q: read as A (row, k) and as B (n, k) fragments
constexpr int SV = D + 8;      // row of S, V: read as B (k, n) fragments
constexpr int SC = C + 4;      // row of M

// Row strides in 4-byte words, chosen so that a warp's fragment loads hit 32
// distinct banks: an A fragment reads (g, t) at g * stride + t (stride = 4
// mod 32), a B fragment from a row-major [k][n] tile reads (t, g) at
// t * stride + g (stride = 8 mod 32); g < 8, t < 4.
static_assert(SD % 32 == 4 && SC % 32 == 4 && SV % 32 == 8, "bank-conflict-free strides");

struct Smem {
    float S[D * SV];           // state, row i (key) x column j (value)
    float K[2][C * SD];        // per-head gates: this chunk's K and the next chunk's, fetched ahead;
                               // per-row gates: K o e^(g - g_ref) and K o e^(g_ref - g) (see k_prefill)
    float Q[C * SD];           // Q (per-row gates: Q o e^(g - g_ref))
    float V[C * SV];           // V, then R = V - (gated K) S, then U
    float M[C * SC];           // M (strict lower; diagonal 16 x 16 blocks then (I + M_bb)^-1), then A
    float lg[C];               // per-head gates: inclusive running sum of log alpha in the chunk
    float beta[C];
    float f[C];                // per-head gates: beta_s gamma_C / gamma_s
    float gref[D];             // per-row gates, per key row i: g_ref, e^(g_ref), e^(g_C), e^(g_C - g_ref)
    float eref[D];
    float egC[D];
    float egCr[D];
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

// Not volatile: a pure function of its operands, so the compiler may
// interleave independent tiles.
__device__ __forceinline__ void mma(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// 16-byte asynchronous copy global -> shared; src_bytes = 0 writes zeros.
__device__ __forceinline__ void cp16(float *dst, const float *src, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
                 : "memory");
}

// acc[nt] += A[m0 .. m0+16, 0 .. kk) B[0 .. kk, n0 + 8 nt .. + 8) for one warp, kk a multiple of 8.
// A(r, c) = sA[r ars + c acs] (times asc[c] when given); B(r, c) = sB[r brs + c bcs].
// Fragment of acc[nt]: [0] (m0+g, n0+8nt+2t), [1] (.., +1), [2] (m0+g+8, ..), [3] (.., +1).
// Each product is hi*hi + hi*lo + lo*hi of the TF32 splits, issued as three
// passes over the n-tiles so that consecutive MMAs never share an accumulator.
template <int NTILE>
__device__ __forceinline__ void warp_gemm(float (&acc)[NTILE][4], const float *sA, int ars, int acs, const float *asc,
                                          const float *sB, int brs, int bcs, int m0, int n0, int kk, int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll 2
    for (int k0 = 0; k0 < kk; k0 += 8) {
        float x[4];
        x[0] = sA[(m0 + g) * ars + (k0 + t) * acs];
        x[1] = sA[(m0 + g + 8) * ars + (k0 + t) * acs];
        x[2] = sA[(m0 + g) * ars + (k0 + t + 4) * acs];
        x[3] = sA[(m0 + g + 8) * ars + (k0 + t + 4) * acs];
        if (asc) {
            const float s0 = asc[k0 + t], s1 = asc[k0 + t + 4];
            x[0] *= s0; x[1] *= s0; x[2] *= s1; x[3] *= s1;
        }
        uint32_t ah[4], al[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) split(x[u], ah[u], al[u]);
        uint32_t bh[NTILE][2], bl[NTILE][2];
#pragma unroll
        for (int nt = 0; nt < NTILE; ++nt) {
            const int n = n0 + 8 * nt + g;
            split(sB[(k0 + t) * brs + n * bcs], bh[nt][0], bl[nt][0]);
            split(sB[(k0 + t + 4) * brs + n * bcs], bh[nt][1], bl[nt][1]);
        }
#pragma unroll
        for (int nt = 0; nt < NTILE; ++nt) mma(acc[nt], ah, bh[nt]);
#pragma unroll
        for (int nt = 0; nt < NTILE; ++nt) mma(acc[nt], ah, bl[nt]);
#pragma unroll
        for (int nt = 0; nt < NTILE; ++nt) mma(acc[nt], al, bh[nt]);
    }
}

template <int NTILE>
__device__ __forceinline__ void zero(float (&acc)[NTILE][4]) {
#pragma unroll
    for (int nt = 0; nt < NTILE; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.0f;
}

}  // namespace pf

// One CTA per (request, layer, head).  Per-row gates (ROWS): with g_ti the
// running sum of log alpha_ti over the chunk's tokens and g_ref,i its value at
// the chunk's middle token, the gate ratios factor per key row as
// e^(g_ti - g_ref,i) e^(g_ref,i - g_si), so with Kt = K o e^(g - g_ref),
// Kh = K o e^(g_ref - g) and Qt = Q o e^(g - g_ref):
//   M = strict_lower(Kt Kh^T) diag(beta),  R = V - (Kt diag(e^g_ref)) S_0,
//   A = L_incl(Qt Kh^T) diag(beta),        O = (Qt diag(e^g_ref)) S_0 + A U,
//   S_C = Diag(e^g_C) S_0 + Diag(e^(g_C - g_ref)) (Kh^T diag(beta)) U.
// The exponents stay within the gates of half a chunk (32 tokens) of the
// reference, so fp32 holds them while the sum of |log alpha_i| over any 32
// consecutive tokens stays below about 80; a chunk where a row's gates leave
// that range (or any gate is not in (0, 1]) sets kErrGateRange in the device
// error word.
template <bool ROWS>
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
    // element offset of token tok's row of this (request, layer, head) in q, k, v, o
    auto row_of = [&](int tok) { return (((size_t)(n * a.T + tok) * a.nL_in + a.l_in0 + ll) * a.H + h) * D; };
    // the q, k, v rows of the chunk from token c0 into L2 ahead of their loads
    auto prefetch_chunk = [&](int c0) {
        const int cc = min(C, a.T - c0);
        if (tid < 3 * cc) {
            const int r = tid / 3, which = tid - 3 * r;
            const float *base = which == 0 ? a.k : which == 1 ? a.q : a.v;
            asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(base + row_of(c0 + r)), "r"(D * 4)
                         : "memory");
        }
    };

    // asynchronous copy of the chunk from token c0 of one of q, k, v into rows of buf (zeros past T)
    auto fetch_rows = [&](float *buf, int stride, const float *base, int c0) {
        const int cc = min(C, a.T - c0);
        for (int e = tid; e < C * D / 4; e += NT) {
            const int r = e / (D / 4), j4 = e % (D / 4);
            const bool ok = r < cc;
            cp16(buf + r * stride + 4 * j4, ok ? base + row_of(c0 + r) + 4 * j4 : base, ok ? 16 : 0);
        }
    };

    prefetch_chunk(0);
    if (!ROWS) fetch_rows(sm.K[0], SD, a.k, 0);   // per-row gates fetch K with the chunk's gates
    fetch_rows(sm.Q, SD, a.q, 0);
    cp_async_commit();
    // the state
    for (int e = tid; e < D * D / 4; e += NT) {
        const int i = e / (D / 4), j4 = e % (D / 4);
        const float4 x = a.zero_init ? make_float4(0.f, 0.f, 0.f, 0.f) : reinterpret_cast<const float4 *>(Sg)[e];
        *reinterpret_cast<float4 *>(&sm.S[i * SV + 4 * j4]) = x;
    }

#pragma unroll 1
    for (int c0 = 0, ci = 0; c0 < a.T; c0 += C, ++ci) {
        const int cc = min(C, a.T - c0);
        // K as the row operand (A side) and as the column operand (B side) of K K^T and Q K^T
        const float *Ka = ROWS ? sm.K[0] : sm.K[ci & 1];
        const float *Kb = ROWS ? sm.K[1] : Ka;
        __syncthreads();  // the previous chunk is done with V, M and its K buffers
        // 1. the chunk's rows: Q (and per-head K) were fetched ahead, V now; per-row gates:
        //    K and the gate rows now.  Rows past T: zeros, alpha = 1, beta = 0.
        fetch_rows(sm.V, SV, a.v, c0);
        if (ROWS) {
            fetch_rows(sm.K[1], SD, a.k, c0);
            fetch_rows(sm.K[0], SD, a.alpha, c0);
        }
        cp_async_commit();
        if (w == 0) {  // beta; per-head gates: inclusive scan of log alpha over the 64 tokens, 2 per lane
            float l2[2], b2[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int r = 2 * lane + u;
                l2[u] = 0.0f;
                b2[u] = 0.0f;
                if (r < cc) {
                    const size_t gi = row_of(c0 + r) / D;
                    if (!ROWS) l2[u] = logf(a.alpha[gi]);
                    b2[u] = a.beta[gi];
                }
            }
            if (!ROWS) {
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
            }
            sm.beta[2 * lane] = b2[0];
            sm.beta[2 * lane + 1] = b2[1];
        }
        cp_async_wait_all();
        __syncthreads();
        if (c0 + C < a.T) {  // the next chunk into L2 (per-head gates: and its K into the other buffer)
            prefetch_chunk(c0 + C);
            if (!ROWS) {
                fetch_rows(sm.K[(ci + 1) & 1], SD, a.k, c0 + C);
                cp_async_commit();
            }
        }
        if (ROWS) {
            // per key row i (thread i): g_ti = running sum of log alpha_ti in place of the gate
            // rows, the reference g at the middle real token, and the row factors
            if (tid < D) {
                float *gcol = sm.K[0] + tid;
                float gs = 0.0f;
#pragma unroll 4
                for (int t = 0; t < C; ++t) {
                    if (t < cc) gs += logf(gcol[t * SD]);
                    gcol[t * SD] = gs;
                }
                const float gr = gcol[((cc - 1) >> 1) * SD];
                // the factors e^(g - g_ref), e^(g_ref - g) and e^(g_ref) must stay finite
                if (!(gcol[0] - gr <= 80.0f && gr - gs <= 80.0f && -gr <= 80.0f)) atomicOr(a.err, kErrGateRange);
                sm.gref[tid] = gr;
                sm.eref[tid] = expf(gr);
                sm.egC[tid] = expf(gs);
                sm.egCr[tid] = expf(gs - gr);
            }
            __syncthreads();
            {  // Kt = K o e^(g - g_ref) over the gates, Kh = K o e^(g_ref - g) over K, Qt = Q o e^(g - g_ref)
                const int i = tid & (D - 1), tb = (tid / D) * (C / 2);
                const float gr = sm.gref[i];
#pragma unroll 4
                for (int t = tb; t < tb + C / 2; ++t) {
                    const float gt = sm.K[0][t * SD + i], kr = sm.K[1][t * SD + i];
                    const float up = expf(gt - gr);
                    sm.K[0][t * SD + i] = kr * up;
                    sm.K[1][t * SD + i] = kr * expf(gr - gt);
                    sm.Q[t * SD + i] *= up;
                }
            }
            __syncthreads();
        } else if (tid < C) {
            sm.f[tid] = sm.beta[tid] * expf(sm.lg[C - 1] - sm.lg[tid]);
        }
        // 2. M = strict_lower(K K^T o Gamma) diag(beta)  and  R = V - (K o Gamma) S
        {
            float acc[4][4];
            zero(acc);
            const int m0 = 16 * (w >> 1), n0 = 32 * (w & 1);
            warp_gemm<4>(acc, Ka, SD, 1, nullptr, Kb, 1, SD, m0, n0, D, lane);
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int r = m0 + g + 8 * (e >> 1), s = n0 + 8 * nt + 2 * t4 + (e & 1);
                    const float x = ROWS ? acc[nt][e] : acc[nt][e] * expf(sm.lg[r] - sm.lg[s]);
                    sm.M[r * SC + s] = (s < r) ? x * sm.beta[s] : 0.0f;
                }
        }
        {
            float acc[8][4];
            zero(acc);
            const int m0 = 16 * (w >> 1), n0 = 64 * (w & 1);
            warp_gemm<8>(acc, Ka, SD, 1, ROWS ? sm.eref : nullptr, sm.S, SV, 1, m0, n0, D, lane);
            const float gm0 = ROWS ? 1.0f : expf(sm.lg[m0 + g]), gm1 = ROWS ? 1.0f : expf(sm.lg[m0 + g + 8]);
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int r = m0 + g + 8 * (e >> 1), j = n0 + 8 * nt + 2 * t4 + (e & 1);
                    sm.V[r * SV + j] -= ((e >> 1) ? gm1 : gm0) * acc[nt][e];
                }
        }
        __syncthreads();
        // 3. U = (I + M)^-1 R in blocks of 16 rows.  (a) Warps 0-3 each invert one unit
        //    lower triangular diagonal block, T_bb = (I + M_bb)^-1, by substitution down its
        //    columns (lane c holds column c), and store it over M_bb.
        if (w < 4) {
            const int r0 = 16 * w, c = lane & 15;
            float tc[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                float acc = 0.0f;
#pragma unroll
                for (int s2 = 0; s2 < r; ++s2) acc = fmaf(sm.M[(r0 + r) * SC + r0 + s2], tc[s2], acc);
                tc[r] = (r == c) ? 1.0f : (r < c ? 0.0f : -acc);
            }
            __syncwarp();
            if (lane < 16) {
#pragma unroll
                for (int r = 0; r < 16; ++r) sm.M[(r0 + r) * SC + r0 + c] = tc[r];
            }
        }
        __syncthreads();
        //    (b) Warp w owns value columns [16 w, 16 w + 16); block by block,
        //    U_b = T_bb (R_b - M[b, < b] U[< b]), both products on the tensor cores.
        {
            const int jw = 16 * w;
#pragma unroll 1
            for (int r0 = 0; r0 < C; r0 += 16) {
                if (r0 > 0) {
                    float acc[2][4];
                    zero(acc);
                    warp_gemm<2>(acc, sm.M, SC, 1, nullptr, sm.V, SV, 1, r0, jw, r0, lane);
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            sm.V[(r0 + g + 8 * (e >> 1)) * SV + jw + 8 * nt + 2 * t4 + (e & 1)] -= acc[nt][e];
                    __syncwarp();
                }
                float acc[2][4];
                zero(acc);
                warp_gemm<2>(acc, sm.M + r0, SC, 1, nullptr, sm.V + r0 * SV, SV, 1, r0, jw, 16, lane);
                __syncwarp();  // every lane has read R_b
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        sm.V[(r0 + g + 8 * (e >> 1)) * SV + jw + 8 * nt + 2 * t4 + (e & 1)] = acc[nt][e];
                __syncwarp();
            }
        }
        __syncthreads();
        // 4. A = L_incl(Q K^T o Gamma) diag(beta) into M
        {
            float acc[4][4];
            zero(acc);
            const int m0 = 16 * (w >> 1), n0 = 32 * (w & 1);
            warp_gemm<4>(acc, sm.Q, SD, 1, nullptr, Kb, 1, SD, m0, n0, D, lane);
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int r = m0 + g + 8 * (e >> 1), s = n0 + 8 * nt + 2 * t4 + (e & 1);
                    const float x = ROWS ? acc[nt][e] : acc[nt][e] * expf(sm.lg[r] - sm.lg[s]);
                    sm.M[r * SC + s] = (s <= r) ? x * sm.beta[s] : 0.0f;
                }
        }
        __syncthreads();
        // 5. O = (Q o Gamma) S + A U, rows of this chunk to global
        {
            float acc[8][4], acc2[8][4];
            zero(acc);
            zero(acc2);
            const int m0 = 16 * (w >> 1), n0 = 64 * (w & 1);
            warp_gemm<8>(acc, sm.Q, SD, 1, ROWS ? sm.eref : nullptr, sm.S, SV, 1, m0, n0, D, lane);
            warp_gemm<8>(acc2, sm.M, SC, 1, nullptr, sm.V, SV, 1, m0, n0, C, lane);
#pragma unroll
            for (int e2 = 0; e2 < 2; ++e2) {
                const int r = m0 + g + 8 * e2;
                if (r < cc) {
                    const float gm = ROWS ? 1.0f : expf(sm.lg[r]);
                    float *orow = a.o + row_of(c0 + r);
#pragma unroll
                    for (int nt = 0; nt < 8; ++nt) {
                        const int j = n0 + 8 * nt + 2 * t4;
                        *reinterpret_cast<float2 *>(orow + j) = make_float2(gm * acc[nt][2 * e2] + acc2[nt][2 * e2],
                                                                            gm * acc[nt][2 * e2 + 1] + acc2[nt][2 * e2 + 1]);
                    }
                }
            }
        }
        __syncthreads();  // every read of the old state and of Q is done
        if (c0 + C < a.T) {  // the next chunk's Q, during the state update
            fetch_rows(sm.Q, SD, a.q, c0 + C);
            cp_async_commit();
        }
        // 6. S = Gamma_C S + (K^T diag(beta Gamma_C / Gamma)) U, warp w updates state rows
        //    [16 w, 16 w + 16); per-row gates: the row factors e^(g_C), e^(g_C - g_ref)
        {
            const float gC = ROWS ? 0.0f : expf(sm.lg[C - 1]);
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                float acc[8][4];
                zero(acc);
                const int m0 = 16 * w, n0 = 64 * half;
                warp_gemm<8>(acc, Kb, 1, SD, ROWS ? sm.beta : sm.f, sm.V, SV, 1, m0, n0, C, lane);
#pragma unroll
                for (int e2 = 0; e2 < 2; ++e2) {
                    const int i = m0 + g + 8 * e2;
                    const float dS = ROWS ? sm.egC[i] : gC, dU = ROWS ? sm.egCr[i] : 1.0f;
#pragma unroll
                    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                        for (int e1 = 0; e1 < 2; ++e1) {
                            const int j = n0 + 8 * nt + 2 * t4 + e1;
                            sm.S[i * SV + j] = dS * sm.S[i * SV + j] + dU * acc[nt][2 * e2 + e1];
                        }
                }
            }
        }
    }
    cp_async_wait_all();
    __syncthreads();
    for (int e = tid; e < D * D / 4; e += NT) {
        const int i = e / (D / 4), j4 = e % (D / 4);
        reinterpret_cast<float4 *>(Sg)[e] = *reinterpret_cast<const float4 *>(&sm.S[i * SV + 4 * j4]);
    }
}

size_t prefill_smem_bytes() { return sizeof(pf::Smem); }

cudaError_t launch_prefill(const PrefillArgs &a, cudaStream_t st) {
    const int items = a.n_req * a.nL * a.H;
    if (items <= 0 || a.T <= 0) return cudaSuccess;
    const size_t smem = sizeof(pf::Smem);
    auto kern = a.rows ? k_prefill<true> : k_prefill<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<items, pf::NT, smem, st>>>(a);
    return cudaGetLastError();
}

}  // namespace stepq
