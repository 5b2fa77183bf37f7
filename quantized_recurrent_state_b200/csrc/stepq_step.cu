// Packed-state decode step kernels for per-key-row units (KDA, plan mode 1),
// and the launchers of the step and pack kernels of both unit kinds.
//
// STEPQuant paper digest (vibe-research), 方法-1 (KDA: a single key row is
// the allocation unit, each with its own width 2/4/6/8 or FP16) and 方法-4
// (reconstruct -> retention + delta update + readout -> refit -> pack ->
// write back).  Arithmetic definitions: include/stepq.h.
//
// One CTA of 2D threads handles one (request, layer, head) record.  Thread t
// owns rows [g RT, g RT + RT) x columns [4l, 4l + 4) with RT = D/8,
// g = t / (D/4), l = t % (D/4): a warp holds one band of whole key rows, so
// the per-row branches (width, pivot row) are uniform across a warp.  The
// column sums of the band order (u, o and the two least-squares sums) take
// a band's even-row and odd-row chains in registers and add the 8 band values
// across warps through shared memory, two threads per column.
#include "stepq_pipe.cuh"

namespace stepq {

template <int D>
struct Geo {
    static constexpr int NT = 2 * D;       // threads per CTA
    static constexpr int RT = D / 8;       // rows per thread
    static constexpr int LANES = D / 4;    // threads across a row band
    static constexpr int BANDS = 8;
};

// Shared memory besides the stages.  Per-row factors that multiply a pair
// of columns are kept duplicated ((x_i, x_i) pairs), so a 16-byte load gives
// two rows' packed operands without register moves.
template <int D>
struct __align__(16) Scratch {
    static constexpr int RT = D / 8, LANES = D / 4, RS = D / 4 + 4;  // RS: padded row of the transpose
    union {
        struct {
            float pU[8][D];  // per-band column values of u (then o)
        } col;
        float pmax[4][8][D];  // column absmax per width class and band
    } u;
    float rsum[8][RT][RS];  // per-thread row partials, transposed for the row reduction
    float pf0[8][D];
    float pf1[8][D];
    float2 a2[D];     // (a_i, a_i), a_i = fl(alpha_i r_i) (FP16 rows: alpha_i)
    float2 k2[D];     // (k_i, k_i)
    float2 q2[D];     // (q_i, q_i)
    float rho[D];     // (requant kernel; the step reads them from the stage)
    float wbar[D];
    float2 rinv2[D];  // (fl(1/r_i), fl(1/r_i)) of the refit
    float2 bw2[D];    // (b_i, b_i) of the refit
    float rowr[D];    // r_i of the refit
    float cold[D];    // c_j refitted
    float wv[D];      // w_j
    float ic0[D];
    float c0[D];
    float ic[D];
    uint4 dring[2];    // prefetched item descriptors (thread 0)
    int dslot[2];
    int meta[kStages][8];
    uint32_t roff[D];  // requant kernel: row byte offset in the codes block
    uint8_t rw[D];     // requant kernel: row width (16 = FP16 row)
};

template <int D>
constexpr bool scratch_aligned() {
    using S = Scratch<D>;
    return offsetof(S, u) % 16 == 0 && offsetof(S, rsum) % 16 == 0 && offsetof(S, pf0) % 16 == 0 &&
           offsetof(S, pf1) % 16 == 0 && offsetof(S, a2) % 16 == 0 && offsetof(S, k2) % 16 == 0 &&
           offsetof(S, q2) % 16 == 0 && offsetof(S, rinv2) % 16 == 0 && offsetof(S, bw2) % 16 == 0 &&
           offsetof(S, cold) % 16 == 0 && offsetof(S, wv) % 16 == 0 && offsetof(S, ic0) % 16 == 0 &&
           offsetof(S, ic) % 16 == 0 && offsetof(S, dring) % 16 == 0 && (sizeof(float) * Scratch<D>::RS) % 16 == 0;
}
static_assert(scratch_aligned<128>(), "scratch arrays must stay 16-byte aligned");

template <int N>
__device__ __forceinline__ float tree_sum1(float (&x)[N]) {
#pragma unroll
    for (int s = 1; s < N; s <<= 1)
#pragma unroll
        for (int i = 0; i + s < N; i += 2 * s) x[i] = x[i] + x[i + s];
    return x[0];
}

// Column value of the band order from the 8 per-band values in p[8][D]:
// two threads per column, four bands each in a pair tree, then the halves.
template <int D>
__device__ __forceinline__ float band_column(const float (*p)[D], int tid) {
    const int j = tid >> 1, b0 = 4 * (tid & 1);
    const float s = (p[b0][j] + p[b0 + 1][j]) + (p[b0 + 2][j] + p[b0 + 3][j]);
    return s + __shfl_xor_sync(0xffffffffu, s, 1);
}

// Band values of this thread's four columns: fl(even chain + odd chain).
template <int D>
__device__ __forceinline__ void put_band(float (*p)[D], int g, int j0, const float2 (&E)[2], const float2 (&O)[2]) {
    *reinterpret_cast<float4 *>(&p[g][j0]) = make_float4(E[0].x + O[0].x, E[0].y + O[0].y, E[1].x + O[1].x, E[1].y + O[1].y);
}

// Column refit from the band values in pf0 (numerator) and pf1
// (denominator): c_j = num / den (c0_j when den = 0), two threads per column.
template <int D, int s16>
__device__ __forceinline__ void column_ls_fit(Scratch<D> &sc, int tid, uint8_t *rec_c) {
    const int j = tid >> 1;
    const float num = band_column<D>(sc.pf0, tid);
    const float den = band_column<D>(sc.pf1, tid);
    if ((tid & 1) == 0) {
        const float c = scale_round((den > 0.0f) ? __fdiv_rn(num, den) : sc.c0[j], s16);
        sc.ic[j] = __frcp_rn(c);
        sc.cold[j] = c;
        if (rec_c) scale_put(rec_c, j, c, s16);
    }
    __syncthreads();
}

// ---------------------------------------------------------------------------
// Row-major codes of per-row units: lane l's four codes of a row are row
// bits [4 b l, 4 b l + 4 b).  The width of a row is the same for all lanes of
// a band, so the per-row branches below are uniform across a warp.
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t row_field(const uint8_t *row, int b, int l) {
    const int bit = 4 * b * l;
    const uint32_t *wp = reinterpret_cast<const uint32_t *>(row);  // rows start 16-byte aligned
    const int w = bit >> 5, sh = bit & 31;
    const uint32_t lo = wp[w];
    const uint32_t hi = (sh + 4 * b > 32) ? wp[w + 1] : 0u;
    return __funnelshift_r(lo, hi, sh);
}

// Store lane l's 4b-bit field of a row (row bits [4 b l, 4 b l + 4 b)).
__device__ __forceinline__ void row_field_store(uint8_t *row, int b, int l, uint32_t f) {
    if (b == 8) {
        reinterpret_cast<uint32_t *>(row)[l] = f;
    } else if (b == 4) {
        reinterpret_cast<uint16_t *>(row)[l] = (uint16_t)f;
    } else if (b == 2) {
        row[l] = (uint8_t)f;
    } else {  // b == 6: three bytes at byte 3l
        uint8_t *p = row + 3 * l;
        p[0] = (uint8_t)f;
        p[1] = (uint8_t)(f >> 8);
        p[2] = (uint8_t)(f >> 16);
    }
}

// Final code e = z + qmax in [0, 2 qmax] of a row of width b from
// t = fma(y, 1/c, kMagic + 2^(b-1)): bits(t) = 0x4B400000 + 2^(b-1) + rint(y/c).
__device__ __forceinline__ uint32_t final_e_rt(float y, float ic, int b) {
    const int off = 1 << (b - 1);
    const float t = __fmaf_rn(y, ic, kMagic + (float)off);
    return (uint32_t)__viaddmin_s32_relu(__float_as_int(t), -(0x4B400000 + 1), 2 * (off - 1));
}

// Refit of a tile of per-row units held in registers; writes r and c to
// rec_r / rec_c (global, may be null) and the packed rows into `codes`
// (shared memory holding the codes block; it is copied out by the caller).
// FP16 rows keep S_t and are stored as binary16; they take no part in the
// column fit and carry r = 0.
template <int D, int s16>
__device__ void fit_rows(float2 (&S)[D / 8][2], Scratch<D> &sc, int tid, const uint8_t *rw, const uint32_t *roff,
                         const float *rho, const float *wbar, uint8_t *codes, uint8_t *rec_r, uint8_t *rec_c) {
    using G = Geo<D>;
    constexpr int RT = G::RT, LANES = G::LANES, RS = Scratch<D>::RS, HALF = LANES / 2;
    const int g = tid / LANES, l = tid % LANES;
    const int j0 = 4 * l;

    // 1. row sums (pairwise over the columns) and row factors
    float *rs = &sc.rsum[g][0][0];
#pragma unroll
    for (int r = 0; r < RT; ++r)
        rs[r * RS + l] = (fabsf(S[r][0].x) + fabsf(S[r][0].y)) + (fabsf(S[r][1].x) + fabsf(S[r][1].y));
    __syncwarp();
    {
        const int rr = l >> 1, hh = l & 1;
        const float *src = rs + rr * RS + hh * HALF;
        float v[HALF];
#pragma unroll
        for (int k = 0; k < HALF; ++k) v[k] = src[k];
        float s = tree_sum1<HALF>(v);
        s = s + __shfl_xor_sync(0xffffffffu, s, 1);
        const int i = g * RT + rr;
        float ri = 0.0f, inv = 0.0f, bw = 0.0f;
        if (rw[i] != kPivotBits) {
            float m = __fmul_rn(s, 1.0f / (float)D);
            m = fmaxf(m, 1e-12f);
            ri = scale_round(__fmul_rn(m, rho[i]), s16);
            inv = __frcp_rn(ri);
            bw = __fmul_rn(wbar[i], __fmul_rn(ri, ri));
        }
        if (hh == 0) {
            sc.rinv2[i] = make_float2(inv, inv);
            sc.bw2[i] = make_float2(bw, bw);
            sc.rowr[i] = ri;
            if (rec_r) scale_put(rec_r, i, ri, s16);
        }
    }
    __syncwarp();
    // 2. y = fl(S * (1/r)) on quantized rows; 3. column absmax per width class
    {
        float m[4][4];
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) m[c][jj] = 0.0f;
#pragma unroll
        for (int r = 0; r < RT; ++r) {
            const int i = g * RT + r;
            const int b = rw[i];
            if (b == kPivotBits) continue;
            const float2 i2 = sc.rinv2[i];
            S[r][0] = mul2(S[r][0], i2);
            S[r][1] = mul2(S[r][1], i2);
            const float a0 = fabsf(S[r][0].x), a1 = fabsf(S[r][0].y), a2 = fabsf(S[r][1].x), a3 = fabsf(S[r][1].y);
            switch (b) {
                case 2: m[0][0] = fmaxf(m[0][0], a0); m[0][1] = fmaxf(m[0][1], a1); m[0][2] = fmaxf(m[0][2], a2); m[0][3] = fmaxf(m[0][3], a3); break;
                case 4: m[1][0] = fmaxf(m[1][0], a0); m[1][1] = fmaxf(m[1][1], a1); m[1][2] = fmaxf(m[1][2], a2); m[1][3] = fmaxf(m[1][3], a3); break;
                case 6: m[2][0] = fmaxf(m[2][0], a0); m[2][1] = fmaxf(m[2][1], a1); m[2][2] = fmaxf(m[2][2], a2); m[2][3] = fmaxf(m[2][3], a3); break;
                default: m[3][0] = fmaxf(m[3][0], a0); m[3][1] = fmaxf(m[3][1], a1); m[3][2] = fmaxf(m[3][2], a2); m[3][3] = fmaxf(m[3][3], a3); break;
            }
        }
#pragma unroll
        for (int c = 0; c < 4; ++c)
            *reinterpret_cast<float4 *>(&sc.u.pmax[c][g][j0]) = make_float4(m[c][0], m[c][1], m[c][2], m[c][3]);
    }
    __syncthreads();
    {  // two threads per column, four bands each; c0_j = max over width classes of fl(max |y| fl(1/qmax))
        const int j = tid >> 1, h = tid & 1, b0 = 4 * h;
        float mm[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            mm[c] = fmaxf(fmaxf(sc.u.pmax[c][b0][j], sc.u.pmax[c][b0 + 1][j]),
                          fmaxf(sc.u.pmax[c][b0 + 2][j], sc.u.pmax[c][b0 + 3][j]));
            mm[c] = fmaxf(mm[c], __shfl_xor_sync(0xffffffffu, mm[c], 1));
        }
        if (h == 0) {
            constexpr float IQ[4] = {1.0f / 1.0f, 1.0f / 7.0f, 1.0f / 31.0f, 1.0f / 127.0f};  // widths 2, 4, 6, 8
            float c0 = 0.0f;
#pragma unroll
            for (int c = 0; c < 4; ++c) c0 = fmaxf(c0, __fmul_rn(mm[c], IQ[c]));
            if (c0 == 0.0f) c0 = 1.0f;
            sc.c0[j] = c0;
            sc.ic0[j] = __frcp_rn(c0);
        }
    }
    __syncthreads();
    // 4. z0, t = fl(b z0) and the least-squares chains over the quantized rows
    {
        const float2 mg = make_float2(kMagic, kMagic);
        const float2 nmg = make_float2(-kMagic, -kMagic);
        const float4 ic4 = *reinterpret_cast<const float4 *>(&sc.ic0[j0]);
        float2 nE[2], nO[2], dE[2], dO[2];
#pragma unroll
        for (int hp = 0; hp < 2; ++hp) nE[hp] = nO[hp] = dE[hp] = dO[hp] = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int r = 0; r < RT; ++r) {
            const int i = g * RT + r;
            if (rw[i] == kPivotBits) continue;
            const float2 b2 = sc.bw2[i];
#pragma unroll
            for (int hp = 0; hp < 2; ++hp) {
                const float2 ic = hp ? make_float2(ic4.z, ic4.w) : make_float2(ic4.x, ic4.y);
                const float2 y = S[r][hp];
                const float2 z0 = add2(fma2(y, ic, mg), nmg);
                const float2 t = mul2(b2, z0);
                if (r & 1) {
                    nO[hp] = fma2(t, y, nO[hp]);
                    dO[hp] = fma2(t, z0, dO[hp]);
                } else {
                    nE[hp] = fma2(t, y, nE[hp]);
                    dE[hp] = fma2(t, z0, dE[hp]);
                }
            }
        }
        put_band<D>(sc.pf0, g, j0, nE, nO);
        put_band<D>(sc.pf1, g, j0, dE, dO);
    }
    __syncthreads();
    column_ls_fit<D, s16>(sc, tid, rec_c);
    // 5. final codes (or binary16) of every row into the shared codes block
    {
        const float4 ic4 = *reinterpret_cast<const float4 *>(&sc.ic[j0]);
        const float icj[4] = {ic4.x, ic4.y, ic4.z, ic4.w};
#pragma unroll
        for (int r = 0; r < RT; ++r) {
            const int i = g * RT + r;
            const int b = rw[i];
            uint8_t *row = codes + roff[i];
            if (b == kPivotBits) {
                const __half2 h01 = __float22half2_rn(S[r][0]);
                const __half2 h23 = __float22half2_rn(S[r][1]);
                uint2 v;
                v.x = *reinterpret_cast<const uint32_t *>(&h01);
                v.y = *reinterpret_cast<const uint32_t *>(&h23);
                *reinterpret_cast<uint2 *>(row + 8 * l) = v;
            } else {
                const float y4[4] = {S[r][0].x, S[r][0].y, S[r][1].x, S[r][1].y};
                uint32_t f = 0u;
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) f |= (final_e_rt(y4[jj], icj[jj], b) + 1u) << (b * jj);
                row_field_store(row, b, l, f);
            }
        }
    }
    __syncthreads();
}

// Copy `bytes` (a multiple of 16) from shared to global memory, all threads.
template <int D>
__device__ __forceinline__ void copy_out(uint8_t *dst, const uint8_t *src, uint32_t bytes, int tid) {
    for (uint32_t o = 16u * tid; o < bytes; o += 16u * (2 * D))
        *reinterpret_cast<uint4 *>(dst + o) = *reinterpret_cast<const uint4 *>(src + o);
}

// Column phase of the step: u and w (KIND != kFitPack) of column j from the
// band values in pU; w to shared memory (and the workspace for kDecode).
template <int D, int KIND>
__device__ __forceinline__ void finish_w(const Args &a, Scratch<D> &sc, int tid, int row, float beta, const float *vs) {
    const int j = tid >> 1;
    const float u = band_column<D>(sc.u.col.pU, tid);
    const float w = __fmul_rn(beta, __fsub_rn(vs[j], u));
    if ((tid & 1) == 0) {
        if (KIND == kDecode) a.w[(size_t)row * D + j] = w;
        sc.wv[j] = w;
    }
}

// One head of per-row units: decode / fit-pack / fused.
template <int D, int KIND, int s16>
__device__ void item_rows(const Args &a, uint8_t *stage, uint8_t *rec_g, int row, uint32_t codes_bytes,
                          Scratch<D> &sc, int tid) {
    using G = Geo<D>;
    constexpr int RT = G::RT, LANES = G::LANES;
    const int g = tid / LANES, l = tid % LANES;
    const int j0 = 4 * l;
    const uint8_t *st_r = stage + codes_bytes;              // staged r[D] and c[D]
    const uint8_t *st_c = st_r + D * (s16 ? 2 : 4);
    const float *tf = stage_tail<D>(a, stage);
    const float *qs = tf + kTailQ * D;
    const float *ks = tf + kTailK * D;
    const float *vs = tf + kTailV * D;
    const float *xs = tf + kTailX * D;
    const float *als = tf + kTailAlpha * D;
    const uint32_t *roff = reinterpret_cast<const uint32_t *>(tf + kTailRoff * D);
    const uint8_t *rw = reinterpret_cast<const uint8_t *>(tf + kTailRw * D);
    const float beta = stage_ab<D>(a, stage)[1];

    if ((tid & 31) < 16) {  // this warp's 16 rows
        const int i = 16 * (tid >> 5) + (tid & 31);
        const int b = rw[i];
        const float al = als[i];
        const float ai = (b == kPivotBits) ? al : __fmul_rn(al, scale_at(st_r, i, s16));
        sc.a2[i] = make_float2(ai, ai);
        sc.k2[i] = make_float2(ks[i], ks[i]);
        if (KIND != kFitPack) sc.q2[i] = make_float2(qs[i], qs[i]);
    }
    __syncwarp();

    // reconstruct S' (fl(fl(a_i c_j) z); FP16 rows fl(alpha_i h)), u chains
    float2 S[RT][2];
    float2 E[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)}, O[2] = {E[0], E[1]};
    const float4 c4 = scale4_at(st_c, j0, s16);
    const float2 c01 = make_float2(c4.x, c4.y), c23 = make_float2(c4.z, c4.w);
#pragma unroll
    for (int r = 0; r < RT; ++r) {
        const int i = g * RT + r;
        const int b = rw[i];
        const float2 a2 = sc.a2[i];
        if (b == kPivotBits) {
            const uint2 v = *reinterpret_cast<const uint2 *>(stage + roff[i] + 8 * l);
            S[r][0] = mul2(a2, __half22float2(*reinterpret_cast<const __half2 *>(&v.x)));
            S[r][1] = mul2(a2, __half22float2(*reinterpret_cast<const __half2 *>(&v.y)));
        } else {
            const uint32_t f = row_field(stage + roff[i], b, l);
            const uint32_t mask = (1u << b) - 1u;
            const float zb = 8388608.0f + (float)(1 << (b - 1));  // 2^23 + 2^(b-1)
            float z[4];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) z[jj] = __fsub_rn(__uint_as_float(((f >> (b * jj)) & mask) | 0x4B000000u), zb);
            S[r][0] = mul2(mul2(a2, c01), make_float2(z[0], z[1]));
            S[r][1] = mul2(mul2(a2, c23), make_float2(z[2], z[3]));
        }
        if (KIND != kFitPack) {
            const float2 k2 = sc.k2[i];
#pragma unroll
            for (int hp = 0; hp < 2; ++hp) {
                if (r & 1) O[hp] = fma2(k2, S[r][hp], O[hp]);
                else E[hp] = fma2(k2, S[r][hp], E[hp]);
            }
        }
    }
    if (KIND != kFitPack) {
        put_band<D>(sc.u.col.pU, g, j0, E, O);
        __syncthreads();
        finish_w<D, KIND>(a, sc, tid, row, beta, vs);
        __syncthreads();
    }
    // S = fma(k, w, S'); o chains
    {
        const float4 w4 = *reinterpret_cast<const float4 *>(KIND == kFitPack ? &xs[j0] : &sc.wv[j0]);
        const float2 w01 = make_float2(w4.x, w4.y), w23 = make_float2(w4.z, w4.w);
        E[0] = E[1] = O[0] = O[1] = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int r = 0; r < RT; ++r) {
            const int i = g * RT + r;
            const float2 k2 = sc.k2[i];
            S[r][0] = fma2(k2, w01, S[r][0]);
            S[r][1] = fma2(k2, w23, S[r][1]);
            if (KIND != kFitPack) {
                const float2 q2 = sc.q2[i];
#pragma unroll
                for (int hp = 0; hp < 2; ++hp) {
                    if (r & 1) O[hp] = fma2(q2, S[r][hp], O[hp]);
                    else E[hp] = fma2(q2, S[r][hp], E[hp]);
                }
            }
        }
    }
    if (KIND != kFitPack) {
        put_band<D>(sc.u.col.pU, g, j0, E, O);
        __syncthreads();
        const float o = band_column<D>(sc.u.col.pU, tid);
        if ((tid & 1) == 0) a.o[(size_t)row * D + (tid >> 1)] = o;
        __syncthreads();
    }
    if (KIND != kDecode) {
        // the staged codes are no longer read: assemble the new rows there
        uint8_t *rec_r = rec_g + codes_bytes;
        fit_rows<D, s16>(S, sc, tid, rw, roff, tf + kTailRho * D, tf + kTailWbar * D, stage, rec_r,
                         rec_r + D * (s16 ? 2 : 4));
        copy_out<D>(rec_g, stage, codes_bytes, tid);
    }
}

// ---------------------------------------------------------------------------
// Persistent pipeline kernel for per-row units.  Every item opens with a
// block barrier (the vote on the copy wait); right after it thread 0 puts
// item it + (kStages-1) G into the stage the previous item used.
// ---------------------------------------------------------------------------
template <int D, int KIND, int S16>
__global__ void __launch_bounds__(2 * D, 2) k_step_rows(Args a) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x;
    const int G = gridDim.x;
    uint8_t *stages = smem;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kStages * a.stage_bytes);
    Scratch<D> &sc = *reinterpret_cast<Scratch<D> *>(smem + kStages * a.stage_bytes + 64);

    int dsel = 0;
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(&bars[s], 1);
        fence_mbar_init();
        for (int s = 0; s < kStages; ++s) {
            const int it = blockIdx.x + s * G;
            if (it >= a.n_items) break;
            int n, ll, di;
            step_coords<D>(a, it, n, ll, di);
            issue_item<D, KIND, 1>(a, it, a.t.desc[di], a.slots[n], stages + s * a.stage_bytes, &bars[s], sc.meta[s]);
        }
        const int nx = blockIdx.x + kStages * G;
        if (nx < a.n_items) prefetch_desc<D>(a, nx, sc.dring, sc.dslot, 0);
    }
    __syncthreads();
    int s = 0;
    uint32_t phase = 0;
    for (int it = blockIdx.x; it < a.n_items; it += G) {
        const bool ok = mbar_wait_bounded(&bars[s], phase, a.wait_polls);
        if (__syncthreads_or(!ok)) {
            if (tid == 0) {
                flag_error(a.err, kErrWait);
                drain_copies(bars, s, phase, a.wait_polls);
            }
            return;
        }
        if (tid == 0 && it != (int)blockIdx.x) {
            const int ps = (s + kStages - 1) % kStages;
            const int nx = it + (kStages - 1) * G;
            if (nx < a.n_items) {
                cp_async_wait_all();
                issue_item<D, KIND, 1>(a, nx, sc.dring[dsel], sc.dslot[dsel], stages + ps * a.stage_bytes, &bars[ps],
                                       sc.meta[ps]);
                dsel ^= 1;
                if (nx + G < a.n_items) prefetch_desc<D>(a, nx + G, sc.dring, sc.dslot, dsel);
            }
        }
        uint8_t *stage = stages + s * a.stage_bytes;
        uint8_t *rec_g = reinterpret_cast<uint8_t *>((uintptr_t)(uint32_t)sc.meta[s][kMetaRecLo] |
                                                     ((uintptr_t)(uint32_t)sc.meta[s][kMetaRecHi] << 32));
        if (sc.meta[s][kMetaValid])
            item_rows<D, KIND, S16>(a, stage, rec_g, sc.meta[s][kMetaRow], (uint32_t)sc.meta[s][kMetaCodes], sc, tid);
        if (++s == kStages) {
            s = 0;
            phase ^= 1u;
        }
    }
}

// ---------------------------------------------------------------------------
// Pack fp32 states (S_0) and unpack records of per-row units: one CTA per head.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(2 * D) k_requant_rows(Args a) {
    extern __shared__ __align__(128) uint8_t smem[];
    Scratch<D> &sc = *reinterpret_cast<Scratch<D> *>(smem);
    uint8_t *codes = smem + ((sizeof(Scratch<D>) + 127) / 128) * 128;  // D*D*2 bytes
    using G = Geo<D>;
    const int tid = threadIdx.x;
    const int g = tid / G::LANES, l = tid % G::LANES;
    int n, ll, h, gl, row;
    item_coords<D>(a, blockIdx.x, n, ll, h, gl, row);
    const int slot = a.slots[n];
    if (slot < 0 || slot >= a.n_slots) {
        if (tid == 0) flag_error(a.err, kErrBadSlot);
        return;
    }
    uint8_t *rec = a.pool + (uint64_t)slot * a.slot_bytes + a.t.rec_off[gl];
    const float *Sg = a.S_in + (size_t)row * D * D;
    float2 S[G::RT][2];
#pragma unroll
    for (int r = 0; r < G::RT; ++r) {
        const float4 v = *reinterpret_cast<const float4 *>(Sg + (size_t)(g * G::RT + r) * D + 4 * l);
        S[r][0] = make_float2(v.x, v.y);
        S[r][1] = make_float2(v.z, v.w);
    }
    if (tid < D) {
        sc.rw[tid] = a.t.row_width[(size_t)gl * D + tid];
        sc.roff[tid] = a.t.row_off[(size_t)gl * D + tid];
        sc.rho[tid] = a.t.rho[(size_t)gl * D + tid];
        sc.wbar[tid] = a.t.wbar[(size_t)gl * D + tid];
    }
    __syncthreads();
    const uint32_t codes_bytes = a.t.codes_bytes[gl];
    uint8_t *rec_r = rec + codes_bytes;
    if (a.scale16) fit_rows<D, 1>(S, sc, tid, sc.rw, sc.roff, sc.rho, sc.wbar, codes, rec_r, rec_r + 2 * D);
    else fit_rows<D, 0>(S, sc, tid, sc.rw, sc.roff, sc.rho, sc.wbar, codes, rec_r, rec_r + 4 * D);
    copy_out<D>(rec, codes, codes_bytes, tid);
}

template <int D>
__global__ void __launch_bounds__(2 * D) k_unpack_rows(Args a) {
    using G = Geo<D>;
    const int tid = threadIdx.x;
    const int g = tid / G::LANES, l = tid % G::LANES;
    int n, ll, h, gl, row;
    item_coords<D>(a, blockIdx.x, n, ll, h, gl, row);
    const int slot = a.slots[n];
    if (slot < 0 || slot >= a.n_slots) {
        if (tid == 0) flag_error(a.err, kErrBadSlot);
        return;
    }
    const uint8_t *rec = a.pool + (uint64_t)slot * a.slot_bytes + a.t.rec_off[gl];
    float *out = a.S_out + (size_t)row * D * D;
    const uint32_t codes_bytes = a.t.codes_bytes[gl];
    const int s16 = a.scale16;
    const uint8_t *rr = rec + codes_bytes;
    const uint8_t *cc = rr + D * (s16 ? 2 : 4);
    const float4 c4 = scale4_at(cc, 4 * l, s16);
    const float2 c01 = make_float2(c4.x, c4.y), c23 = make_float2(c4.z, c4.w);
#pragma unroll
    for (int r = 0; r < G::RT; ++r) {
        const int i = g * G::RT + r;
        const int b = a.t.row_width[(size_t)gl * D + i];
        const uint8_t *rowp = rec + a.t.row_off[(size_t)gl * D + i];
        float2 s01, s23;
        if (b == kPivotBits) {
            const uint2 v = *reinterpret_cast<const uint2 *>(rowp + 8 * l);
            s01 = __half22float2(*reinterpret_cast<const __half2 *>(&v.x));
            s23 = __half22float2(*reinterpret_cast<const __half2 *>(&v.y));
        } else {
            const uint32_t f = row_field(rowp, b, l);
            const uint32_t mask = (1u << b) - 1u;
            const float zb = 8388608.0f + (float)(1 << (b - 1));
            float z[4];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) z[jj] = __fsub_rn(__uint_as_float(((f >> (b * jj)) & mask) | 0x4B000000u), zb);
            const float ri = scale_at(rr, i, s16);
            const float2 r2 = make_float2(ri, ri);
            s01 = mul2(mul2(r2, c01), make_float2(z[0], z[1]));
            s23 = mul2(mul2(r2, c23), make_float2(z[2], z[3]));
        }
        *reinterpret_cast<float4 *>(out + (size_t)i * D + 4 * l) = make_float4(s01.x, s01.y, s23.x, s23.y);
    }
}

// ---------------------------------------------------------------------------
// Host-side launchers (called by the C ABI in stepq_api.cu).  Per-head units
// run the kernels of stepq_head.cu.
// ---------------------------------------------------------------------------
cudaError_t launch_step_head(int kind, int D, const Args &a, int n_sms, cudaStream_t st, int *grid);
cudaError_t launch_pack_head(int D, const Args &a, bool unpack, cudaStream_t st);
size_t step_smem_head_bytes(int D, uint32_t stage_bytes);

template <int KIND>
static cudaError_t launch_rows_kind(const Args &a, int n_sms, cudaStream_t st, int *grid_out) {
    constexpr int D = 128;
    const size_t smem = (size_t)kStages * a.stage_bytes + 64 + sizeof(Scratch<D>);
    auto kern = a.scale16 ? k_step_rows<D, KIND, 1> : k_step_rows<D, KIND, 0>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 2 * D, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    int grid = n_sms * per_sm;
    if (grid > a.n_items) grid = a.n_items;
    if (grid_out) *grid_out = grid;
    if (grid <= 0) return cudaSuccess;
    kern<<<grid, 2 * D, smem, st>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_step(int kind, int D, const Args &a, int n_sms, cudaStream_t st, int *grid) {
    if (a.mode == 0) return launch_step_head(kind, D, a, n_sms, st, grid);
    if (D != 128) return cudaErrorInvalidValue;
    switch (kind) {
        case kDecode: return launch_rows_kind<kDecode>(a, n_sms, st, grid);
        case kFitPack: return launch_rows_kind<kFitPack>(a, n_sms, st, grid);
        case kFused: return launch_rows_kind<kFused>(a, n_sms, st, grid);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_pack(int D, const Args &a, bool unpack, cudaStream_t st) {
    if (a.mode == 0) return launch_pack_head(D, a, unpack, st);
    if (D != 128) return cudaErrorInvalidValue;
    if (a.n_items <= 0) return cudaSuccess;
    if (unpack) {
        k_unpack_rows<128><<<a.n_items, 2 * 128, 0, st>>>(a);
    } else {
        const size_t smem = ((sizeof(Scratch<128>) + 127) / 128) * 128 + (size_t)128 * 128 * 2;
        cudaError_t e = cudaFuncSetAttribute(k_requant_rows<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        k_requant_rows<128><<<a.n_items, 2 * 128, smem, st>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace stepq
