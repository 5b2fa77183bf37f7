// Building blocks of the per-head-unit (GDN, plan mode 0) step kernels: the
// tile geometry, the band-order column reductions, the code-field codec of
// the tile-major layout, the row phase and the refit.  Used by the
// register-resident kernels (stepq_head.cu) and the tensor-memory kernel
// (stepq_head_tm.cu).
//
// STEPQuant paper digest (vibe-research), 方法-3 (X_hat = r_i c_j z_ij; row
// factors from the row means, column factors by an omega-weighted fit) and
// 方法-4 (reconstruct -> update -> readout -> refit -> pack).  Arithmetic
// definitions: include/stepq.h.
#pragma once

#include "stepq_pipe.cuh"

namespace stepq {

template <int D>
struct GeoH {
    static constexpr int NT = 2 * D;  // threads = tiles
    static constexpr int RT = D / 8;  // rows of a tile (one band)
    static constexpr int NP = RT / 2; // row pairs of a tile
    static constexpr int NCB = D / 4; // column blocks
    static constexpr int PS = D + 4;  // row of the partial array (floats)
};

// Shared memory besides the stages.
template <int D>
struct __align__(16) ScratchH {
    // partial row sums (or row maxima) per column block: part[pidx(cb, i)];
    // the upper half of the column blocks sits 16 floats further on, so the
    // two threads of a row read different banks
    float part[GeoH<D>::NCB * GeoH<D>::PS + 16];
    float rinv[D];  // fl(1/r_i)
    float bw[D];    // b_i = fl(wbar_i fl(r_i r_i))
    float rowr[D];  // r_i (calibration)
    float rho[D];   // the head's rho_i and wbar_i (requant and calibration kernels)
    float wbar[D];
    uint4 dring[2];  // prefetched item descriptors (thread 0)
    int dslot[2];
    int meta[kStages][8];
};

template <int D>
__device__ __forceinline__ int pidx(int cb, int i) {
    return cb * GeoH<D>::PS + (cb >= GeoH<D>::NCB / 2 ? 16 : 0) + i;
}

constexpr unsigned kFull = 0xffffffffu;

// Tile of thread t (tile t of the code layout): band g = lane bits [2, 5),
// column block cb = 4 (t / 32) + (t % 4).  The 8 lanes of a quarter warp then
// cover two bands and four column blocks, so the per-row operand loads (two
// distinct 16-byte addresses per quarter) and the row-partial stores are free
// of bank conflicts.
__device__ __forceinline__ int band_of(int t) { return (t >> 2) & 7; }
__device__ __forceinline__ int cblk_of(int t) { return ((t >> 5) << 2) | (t & 3); }
// Lane xor masks that reach band g ^ 1, g ^ 2, g ^ 4 of the same column block.
constexpr int kX1 = 4, kX2 = 8, kX4 = 16;
// Lane of band gs in the column block of `lane`.
__device__ __forceinline__ int band_lane(int lane, int gs) { return (lane & ~28) | (gs << 2); }

// ---------------------------------------------------------------------------
// Column reductions over the 8 bands of a column group (bands g ^ 1, g ^ 2,
// g ^ 4).  Level 1 adds bands (g, g^1), level 2 pairs of those, level 3 the
// halves: ((b0 + b1) + (b2 + b3)) + ((b4 + b5) + (b6 + b7)).  Each level keeps
// half of the lane's columns and sends the other half to its partner, so
// after the three levels the lane holds one finished column.
// ---------------------------------------------------------------------------

// After band_sum4 / band_max4 the lane with band g holds column 2 (g & 1) + ((g >> 1) & 1).
__device__ __forceinline__ int col4_of(int g) { return 2 * (g & 1) + ((g >> 1) & 1); }
// Lane of the same column block that holds column c after band_sum4 / band_max4.
__device__ __forceinline__ int col4_src(int lane, int c) { return band_lane(lane, (c >> 1) | ((c & 1) << 1)); }

__device__ __forceinline__ float band_sum4(float v0, float v1, float v2, float v3, int g) {
    const bool h1 = g & 1, h2 = g & 2;
    float ka = h1 ? v2 : v0, kb = h1 ? v3 : v1;
    const float sa = h1 ? v0 : v2, sb = h1 ? v1 : v3;
    ka = ka + __shfl_xor_sync(kFull, sa, kX1);
    kb = kb + __shfl_xor_sync(kFull, sb, kX1);
    float k = h2 ? kb : ka;
    const float s = h2 ? ka : kb;
    k = k + __shfl_xor_sync(kFull, s, kX2);
    return k + __shfl_xor_sync(kFull, k, kX4);
}

__device__ __forceinline__ float band_max4(float v0, float v1, float v2, float v3, int g) {
    const bool h1 = g & 1, h2 = g & 2;
    float ka = h1 ? v2 : v0, kb = h1 ? v3 : v1;
    const float sa = h1 ? v0 : v2, sb = h1 ? v1 : v3;
    ka = fmaxf(ka, __shfl_xor_sync(kFull, sa, kX1));
    kb = fmaxf(kb, __shfl_xor_sync(kFull, sb, kX1));
    float k = h2 ? kb : ka;
    const float s = h2 ? ka : kb;
    k = fmaxf(k, __shfl_xor_sync(kFull, s, kX2));
    return fmaxf(k, __shfl_xor_sync(kFull, k, kX4));
}

// The two least-squares sums of four columns: the lane with band g ends with
// N (g even) or D (g odd) of column 2 ((g >> 1) & 1) + ((g >> 2) & 1); its
// partner lane g ^ 1 holds the other sum of the same column.
__device__ __forceinline__ int col8_of(int g) { return 2 * ((g >> 1) & 1) + ((g >> 2) & 1); }
__device__ __forceinline__ int col8_src(int lane, int c) { return band_lane(lane, ((c >> 1) << 1) | ((c & 1) << 2)); }

__device__ __forceinline__ float band_sum8(const float (&N)[4], const float (&Dn)[4], int g) {
    const bool h1 = g & 1, h2 = g & 2, h4 = g & 4;
    float k[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const float keep = h1 ? Dn[c] : N[c], send = h1 ? N[c] : Dn[c];
        k[c] = keep + __shfl_xor_sync(kFull, send, kX1);
    }
    float ka = h2 ? k[2] : k[0], kb = h2 ? k[3] : k[1];
    const float sa = h2 ? k[0] : k[2], sb = h2 ? k[1] : k[3];
    ka = ka + __shfl_xor_sync(kFull, sa, kX2);
    kb = kb + __shfl_xor_sync(kFull, sb, kX2);
    float kk = h4 ? kb : ka;
    const float s = h4 ? ka : kb;
    return kk + __shfl_xor_sync(kFull, s, kX4);
}

__device__ __forceinline__ float2 abs2(float2 x) { return make_float2(fabsf(x.x), fabsf(x.y)); }

// max(m, |x|, |y|)
__device__ __forceinline__ float max3abs(float m, float x, float y) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(m), "f"(fabsf(x)), "f"(fabsf(y)));
    return d;
}

// ---------------------------------------------------------------------------
// Codes of a tile.  A field is turned into an fp32 number by OR-ing it, at
// its bit position p, into the bit pattern of 2^(23-p): the result is
// 2^(23-p) + u exactly, and one subtraction of 2^(23-p) + 2^(b-1) leaves z.
// The row pair (2k, 2k+1) of a column sits at the same p for every width,
// so one packed subtraction serves both rows.
// ---------------------------------------------------------------------------

__host__ __device__ constexpr uint32_t mbits(int p) { return (uint32_t)(150 - p) << 23; }
__host__ __device__ constexpr float mval(int p, int off) { return (float)(1 << (23 - p)) + (float)off; }

__device__ __forceinline__ float2 zpair(uint32_t xa, uint32_t xb, float nk) {
    return add2(make_float2(__uint_as_float(xa), __uint_as_float(xb)), make_float2(nk, nk));
}

// The four codes of a 6-bit row value (24 bits: code c in bits [6c, 6c + 6)).
__device__ __forceinline__ void row6_x(uint32_t R, uint32_t (&X)[4]) {
    X[0] = (R & 0x3Fu) | mbits(0);
    X[1] = (R & 0xFC0u) | mbits(6);
    X[2] = (R & 0x3F000u) | mbits(12);
    X[3] = ((R >> 12) & 0xFC0u) | mbits(6);
}

// z of rows (2k, 2k+1) x the tile's 4 columns.
template <int D, int B>
__device__ __forceinline__ void unpack_pair(const uint32_t (&W)[Stream<D, B>::NW], int k, float2 (&z)[4]) {
    constexpr int OFF = 1 << (B - 1);
    if constexpr (B == 4) {
        const uint32_t w = W[k], wh = w >> 16;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const uint32_t m = 0xFu << (4 * c);
            z[c] = zpair((w & m) | mbits(4 * c), (wh & m) | mbits(4 * c), -mval(4 * c, OFF));
        }
    } else if constexpr (B == 8) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
            z[c] = zpair(__byte_perm(W[2 * k], 0x4B000000u, 0x7540u | c), __byte_perm(W[2 * k + 1], 0x4B000000u, 0x7540u | c),
                         -mval(0, OFF));
    } else if constexpr (B == 2) {
        const uint32_t w = (k & 1) ? (W[k >> 1] >> 16) : W[k >> 1];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int pa = 2 * c, pb = 8 + 2 * c;
            z[c] = add2(make_float2(__uint_as_float((w & (3u << pa)) | mbits(pa)), __uint_as_float((w & (3u << pb)) | mbits(pb))),
                        make_float2(-mval(pa, OFF), -mval(pb, OFF)));
        }
    } else {  // B == 6
        uint32_t Ra, Rb;
        if constexpr (D / 8 >= 4) {
            const int q = k >> 1;
            if ((k & 1) == 0) {
                Ra = W[3 * q];
                Rb = W[3 * q + 1];
            } else {  // row 2 of the group: its bytes are the top bytes of the group's words
                Ra = __byte_perm(__byte_perm(W[3 * q], W[3 * q + 1], 0x0073u), W[3 * q + 2], 0x0710u);
                Rb = W[3 * q + 2];
            }
        } else {  // RT = 2: plain stream, row 0 in bits [0, 24), row 1 in [24, 48)
            Ra = W[0];
            Rb = __funnelshift_r(W[0], W[1], 24);
        }
        uint32_t Xa[4], Xb[4];
        row6_x(Ra, Xa);
        row6_x(Rb, Xb);
        z[0] = zpair(Xa[0], Xb[0], -mval(0, OFF));
        z[1] = zpair(Xa[1], Xb[1], -mval(6, OFF));
        z[2] = zpair(Xa[2], Xb[2], -mval(12, OFF));
        z[3] = zpair(Xa[3], Xb[3], -mval(6, OFF));
    }
}

// Final codes of rows (2k, 2k+1) from T = fma(y, 1/c, kMagic + 2^(b-1)) per
// element: bits(T) = 0x4B400000 + 2^(b-1) + rint(y/c), and |rint(y/c)| <=
// 2 qmax + 1 (the refit c is at least c0/2), so the low 16 bits hold
// 2^(b-1) + rint(y/c) as a signed 16-bit value.  e = clamp(rint + qmax, 0,
// 2 qmax); the stored field is e + 1 = z + 2^(b-1).
template <int B>
__device__ __forceinline__ uint32_t clamp_pair16(float2 T) {
    constexpr uint32_t Q = (1u << (B - 1)) - 1u;
    return __viaddmin_s16x2_relu(__byte_perm(__float_as_uint(T.x), __float_as_uint(T.y), 0x5410u), 0xFFFFFFFFu,
                                 (2u * Q) | ((2u * Q) << 16));
}

template <int B>
__device__ __forceinline__ uint32_t clamp1(float t) {
    constexpr int Q = (1 << (B - 1)) - 1;
    return (uint32_t)__viaddmin_s32_relu(__float_as_int(t), -(0x4B400000 + 1), 2 * Q);
}

template <int D, int B>
__device__ __forceinline__ void pack_pair(uint32_t (&W)[Stream<D, B>::NW], int k, const float2 (&T)[4], uint32_t &hold_a,
                                          uint32_t &hold_b) {
    if constexpr (B == 4) {
        uint32_t w = 0x11111111u;
#pragma unroll
        for (int c = 0; c < 4; ++c) w += clamp_pair16<4>(T[c]) << (4 * c);
        W[k] = w;
    } else if constexpr (B == 8) {
        uint32_t v[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) v[c] = clamp_pair16<8>(T[c]);
        const uint32_t t01 = __byte_perm(v[0], v[1], 0x6240u), t23 = __byte_perm(v[2], v[3], 0x6240u);
        W[2 * k] = __byte_perm(t01, t23, 0x5410u) + 0x01010101u;
        W[2 * k + 1] = __byte_perm(t01, t23, 0x7632u) + 0x01010101u;
    } else if constexpr (B == 2) {
        uint32_t w = (k & 1) ? W[k >> 1] : 0x55555555u;
        const int sh = 16 * (k & 1);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            w += clamp1<2>(T[c].x) << (sh + 2 * c);
            w += clamp1<2>(T[c].y) << (sh + 8 + 2 * c);
        }
        W[k >> 1] = w;
    } else {  // B == 6: 24-bit row values, then the group's words
        uint32_t Ra = 0x41041u, Rb = 0x41041u;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            Ra += clamp1<6>(T[c].x) << (6 * c);
            Rb += clamp1<6>(T[c].y) << (6 * c);
        }
        if constexpr (D / 8 >= 4) {
            const int q = k >> 1;
            if ((k & 1) == 0) {
                hold_a = Ra;  // rows 0 and 1 of the group wait for row 2's bytes
                hold_b = Rb;
            } else {
                W[3 * q] = __byte_perm(hold_a, Ra, 0x4210u);
                W[3 * q + 1] = __byte_perm(hold_b, Ra, 0x5210u);
                W[3 * q + 2] = __byte_perm(Rb, Ra, 0x6210u);
            }
        } else {
            W[0] = Ra | (Rb << 24);
            W[1] = Rb >> 8;
        }
    }
}

// (x_i, x_{i+1}) of a scale array (fp32 or bfloat16).
__device__ __forceinline__ float2 scale2_at(const uint8_t *base, int i, int s16) {
    if (s16) {
        const uint32_t v = *reinterpret_cast<const uint32_t *>(base + 2 * i);
        return make_float2(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u));
    }
    return *reinterpret_cast<const float2 *>(base + 4 * i);
}

// Row pairs (x_i, x_{i+1}), i = i0 + 2k, of NP pairs from a 16-byte aligned
// row array (16-byte loads, two pairs each).
template <int NP>
__device__ __forceinline__ void load_pairs(const float *p, float2 (&out)[NP]) {
    if constexpr (NP % 2 == 0) {
#pragma unroll
        for (int k = 0; k < NP; k += 2) {
            const float4 v = *reinterpret_cast<const float4 *>(p + 2 * k);
            out[k] = make_float2(v.x, v.y);
            out[k + 1] = make_float2(v.z, v.w);
        }
    } else {
#pragma unroll
        for (int k = 0; k < NP; ++k) out[k] = *reinterpret_cast<const float2 *>(p + 2 * k);
    }
}

// The same from a scale array (fp32 or bfloat16) at row i0.
template <int NP>
__device__ __forceinline__ void load_scale_pairs(const uint8_t *base, int i0, int s16, float2 (&out)[NP]) {
    if (!s16) {
        load_pairs<NP>(reinterpret_cast<const float *>(base) + i0, out);
        return;
    }
    if constexpr (NP % 4 == 0) {
#pragma unroll
        for (int k = 0; k < NP; k += 4) {
            const uint4 v = *reinterpret_cast<const uint4 *>(base + 2 * (i0 + 2 * k));
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int t = 0; t < 4; ++t) out[k + t] = make_float2(__uint_as_float(w[t] << 16), __uint_as_float(w[t] & 0xffff0000u));
        }
    } else {
#pragma unroll
        for (int k = 0; k < NP; ++k) out[k] = scale2_at(base, i0 + 2 * k, 1);
    }
}

// ---------------------------------------------------------------------------
// Requantization of the fp32 tile S (registers) into codes, r and c.
// ---------------------------------------------------------------------------

// This thread's partial row sums (QUANT dual-axis) or maxima (absmax) of its
// RT rows over its 4 columns, into the partial array.
template <int D, int QUANT>
__device__ __forceinline__ void row_partials(const float2 (&S)[D / 16][4], ScratchH<D> &sc, int g, int cb) {
    constexpr int NP = D / 16;
    float rs[2 * NP];
#pragma unroll
    for (int k = 0; k < NP; ++k) {
        if (QUANT == kQuantAbsmax) {
            rs[2 * k] = fmaxf(fmaxf(fabsf(S[k][0].x), fabsf(S[k][1].x)), fmaxf(fabsf(S[k][2].x), fabsf(S[k][3].x)));
            rs[2 * k + 1] = fmaxf(fmaxf(fabsf(S[k][0].y), fabsf(S[k][1].y)), fmaxf(fabsf(S[k][2].y), fabsf(S[k][3].y)));
        } else {  // pairwise over the four columns, both rows of the pair in one packed add
            const float2 p01 = add2(abs2(S[k][0]), abs2(S[k][1]));
            const float2 p23 = add2(abs2(S[k][2]), abs2(S[k][3]));
            const float2 r = add2(p01, p23);
            rs[2 * k] = r.x;
            rs[2 * k + 1] = r.y;
        }
    }
    float *dst = &sc.part[pidx<D>(cb, g * (D / 8))];
    if constexpr (NP % 2 == 0) {
#pragma unroll
        for (int k = 0; k < NP; k += 2)
            *reinterpret_cast<float4 *>(dst + 2 * k) = make_float4(rs[2 * k], rs[2 * k + 1], rs[2 * k + 2], rs[2 * k + 3]);
    } else {
#pragma unroll
        for (int k = 0; k < NP; ++k) *reinterpret_cast<float2 *>(dst + 2 * k) = make_float2(rs[2 * k], rs[2 * k + 1]);
    }
}

template <int N>
__device__ __forceinline__ float pairwise_tree(float (&x)[N]) {
#pragma unroll
    for (int s = 1; s < N; s <<= 1)
#pragma unroll
        for (int i = 0; i + s < N; i += 2 * s) x[i] = x[i] + x[i + s];
    return x[0];
}

// Row phase (between the first and the second block barrier of a record):
// two threads per row finish the row sum (pairwise over the column blocks,
// each thread one half, then the two halves) or the row maximum, form r_i,
// 1/r_i and b_i, and write r_i to the record.  Ends with the second barrier.
template <int D, int B, int S16, int QUANT>
__device__ __forceinline__ void row_phase(ScratchH<D> &sc, int tid, const float *rho, const float *wbar, uint8_t *rec_r) {
    constexpr int HB = GeoH<D>::NCB / 2;
    constexpr int Q = (1 << (B - 1)) - 1;
    const int i = tid >> 1, h = tid & 1;
    float v[HB];
#pragma unroll
    for (int m = 0; m < HB; ++m) v[m] = sc.part[pidx<D>(h * HB + m, i)];
    float ri, bw = 0.0f;
    if (QUANT == kQuantAbsmax) {
        float mx = v[0];
#pragma unroll
        for (int m = 1; m < HB; ++m) mx = fmaxf(mx, v[m]);
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
        ri = scale_round((mx > 0.0f) ? __fdiv_rn(mx, (float)Q) : 1.0f, S16);
    } else {
        float s = pairwise_tree<HB>(v);
        s = s + __shfl_xor_sync(kFull, s, 1);
        const float m = fmaxf(__fmul_rn(s, 1.0f / (float)D), 1e-12f);
        ri = scale_round(__fmul_rn(m, rho[i]), S16);
        bw = __fmul_rn(wbar[i], __fmul_rn(ri, ri));
    }
    if (h == 0) {
        sc.rinv[i] = __frcp_rn(ri);
        sc.rowr[i] = ri;
        if (rec_r) scale_put(rec_r, i, ri, S16);
    } else {
        sc.bw[i] = bw;
    }
    __syncthreads();
}

// After the row phase: y = fl(S fl(1/r)) in place, the initial column factor,
// the initial codes and the least-squares refinement of c, then the final
// codes of the tile into W.  c_j goes to rec_c (may be null); cq (may be
// null) receives c of the thread's four columns.
template <int D, int B, int S16>
__device__ __forceinline__ void fit_codes(float2 (&S)[D / 16][4], ScratchH<D> &sc, int tid, uint8_t *rec_c,
                                          uint32_t (&W)[Stream<D, B>::NW], float *cq = nullptr) {
    constexpr int NP = D / 16, RT = D / 8;
    constexpr int OFF = 1 << (B - 1), Q = OFF - 1;
    constexpr float IQ = 1.0f / (float)Q;
    const int g = band_of(tid), lane = tid & 31, i0 = g * RT, j0 = 4 * cblk_of(tid);
    // y and the column maxima of |y|
    float m[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    float2 pr[NP];
    load_pairs<NP>(&sc.rinv[i0], pr);
#pragma unroll
    for (int k = 0; k < NP; ++k) {
        const float2 ir = pr[k];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            S[k][c] = mul2(S[k][c], ir);
            m[c] = max3abs(m[c], S[k][c].x, S[k][c].y);
        }
    }
    const float mx = band_max4(m[0], m[1], m[2], m[3], g);
    const float c0 = (mx == 0.0f) ? 1.0f : __fmul_rn(mx, IQ);
    const float ic0 = __frcp_rn(c0);
    float2 ic0d[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const float t = __shfl_sync(kFull, ic0, col4_src(lane, c));
        ic0d[c] = make_float2(t, t);
    }
    // z0 = rint(y fl(1/c0)); t = fl(b z0); N = sum t y, D = sum t z0 (band order)
    const float2 mg = make_float2(kMagic, kMagic), nmg = make_float2(-kMagic, -kMagic);
    float2 na[4], da[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) na[c] = da[c] = make_float2(0.0f, 0.0f);
    load_pairs<NP>(&sc.bw[i0], pr);
#pragma unroll
    for (int k = 0; k < NP; ++k) {
        const float2 b2 = pr[k];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const float2 z0 = add2(fma2(S[k][c], ic0d[c], mg), nmg);
            const float2 t = mul2(b2, z0);
            na[c] = fma2(t, S[k][c], na[c]);
            da[c] = fma2(t, z0, da[c]);
        }
    }
    float N[4], Dn[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        N[c] = na[c].x + na[c].y;
        Dn[c] = da[c].x + da[c].y;
    }
    const float mine = band_sum8(N, Dn, g);
    const float other = __shfl_xor_sync(kFull, mine, kX1);
    const float num = (g & 1) ? other : mine, den = (g & 1) ? mine : other;
    const int c8 = col8_of(g);
    const float c0c = __shfl_sync(kFull, c0, col4_src(lane, c8));
    const float cj = scale_round((den > 0.0f) ? __fdiv_rn(num, den) : c0c, S16);
    const float icj = __frcp_rn(cj);
    if ((g & 1) == 0 && rec_c) scale_put(rec_c, j0 + c8, cj, S16);
    float2 icd[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const float t = __shfl_sync(kFull, icj, col8_src(lane, c));
        icd[c] = make_float2(t, t);
        if (cq) cq[c] = __shfl_sync(kFull, cj, col8_src(lane, c));
    }
    // final codes
    const float2 mg2 = make_float2(kMagic + (float)OFF, kMagic + (float)OFF);
    uint32_t ha = 0u, hb = 0u;
#pragma unroll
    for (int k = 0; k < NP; ++k) {
        float2 T[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) T[c] = fma2(S[k][c], icd[c], mg2);
        pack_pair<D, B>(W, k, T, ha, hb);
    }
}

// Per-row absmax codes (the baseline quantizer): z = clamp(rint(S fl(1/r_i))).
template <int D, int B>
__device__ __forceinline__ void absmax_codes(const float2 (&S)[D / 16][4], const ScratchH<D> &sc, int tid,
                                             uint32_t (&W)[Stream<D, B>::NW]) {
    constexpr int NP = D / 16, RT = D / 8, OFF = 1 << (B - 1);
    const int i0 = band_of(tid) * RT;
    const float2 mg2 = make_float2(kMagic + (float)OFF, kMagic + (float)OFF);
    uint32_t ha = 0u, hb = 0u;
    float2 pr[NP];
    load_pairs<NP>(&sc.rinv[i0], pr);
#pragma unroll
    for (int k = 0; k < NP; ++k) {
        const float2 ir = pr[k];
        float2 T[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) T[c] = fma2(S[k][c], ir, mg2);
        pack_pair<D, B>(W, k, T, ha, hb);
    }
}

}  // namespace stepq
