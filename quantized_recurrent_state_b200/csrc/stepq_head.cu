// Packed-state decode step of per-head units (GDN, plan mode 0): the fused
// step, the two-stream decode and fit-and-pack kernels, the requantizer of
// fp32 states, the unpacker and the calibration distortion kernel.
//
// STEPQuant paper digest (vibe-research), 方法-4: reconstruct the state tile
// from integer codes, row/column scales and FP16 pivots; retention, delta
// update and readout on the floating-point tile; the readout goes on at once;
// refit the row/column factors (方法-3); pack codes and scales; write back
// before the next read.  Arithmetic definitions: include/stepq.h.
//
// Mapping.  One CTA of NT = 2D threads works on one (request, layer, head)
// record at a time.  Thread t owns tile t of the tile-major code layout:
// rows [g RT, g RT + RT) (band g = t & 7, RT = D/8) of columns
// [4 cb, 4 cb + 4) (cb = t >> 3).  A warp therefore holds 16 whole value
// columns: every column reduction (u, o, the initial column factor and the
// two least-squares sums) runs over the 8 bands of a column group inside one
// warp (lanes xor 1, 2, 4), in the balanced tree of the band order; only the
// row sums cross warps (one shared-memory exchange, two block barriers per
// record).  The state lives in registers as row pairs: S[k][c] holds rows
// g RT + 2k and g RT + 2k + 1 of column 4 cb + c, so the even/odd row chains
// of the band order are the two halves of one packed fp32x2 accumulator.
//
// Persistent CTAs stream records through a ring of shared-memory stages
// filled by 1-D bulk copies (cp.async.bulk, completion on an mbarrier); the
// stage of a record is refilled right after the last block barrier that
// follows its last read.
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

// ---------------------------------------------------------------------------
// Column reductions over the 8 bands of a column group (lanes xor 1, 2, 4).
// Level 1 adds bands (g, g^1), level 2 pairs of those, level 3 the halves:
// ((b0 + b1) + (b2 + b3)) + ((b4 + b5) + (b6 + b7)).  Each level keeps half
// of the lane's columns and sends the other half to its partner, so after
// the three levels the lane holds one finished column.
// ---------------------------------------------------------------------------

// After band_sum4 / band_max4 the lane with band g holds column 2 (g & 1) + ((g >> 1) & 1).
__device__ __forceinline__ int col4_of(int g) { return 2 * (g & 1) + ((g >> 1) & 1); }
// Lane of the same column group that holds column c after band_sum4 / band_max4.
__device__ __forceinline__ int col4_src(int lane, int c) { return (lane & ~7) | (c >> 1) | ((c & 1) << 1); }

__device__ __forceinline__ float band_sum4(float v0, float v1, float v2, float v3, int g) {
    const bool h1 = g & 1, h2 = g & 2;
    float ka = h1 ? v2 : v0, kb = h1 ? v3 : v1;
    const float sa = h1 ? v0 : v2, sb = h1 ? v1 : v3;
    ka = ka + __shfl_xor_sync(kFull, sa, 1);
    kb = kb + __shfl_xor_sync(kFull, sb, 1);
    float k = h2 ? kb : ka;
    const float s = h2 ? ka : kb;
    k = k + __shfl_xor_sync(kFull, s, 2);
    return k + __shfl_xor_sync(kFull, k, 4);
}

__device__ __forceinline__ float band_max4(float v0, float v1, float v2, float v3, int g) {
    const bool h1 = g & 1, h2 = g & 2;
    float ka = h1 ? v2 : v0, kb = h1 ? v3 : v1;
    const float sa = h1 ? v0 : v2, sb = h1 ? v1 : v3;
    ka = fmaxf(ka, __shfl_xor_sync(kFull, sa, 1));
    kb = fmaxf(kb, __shfl_xor_sync(kFull, sb, 1));
    float k = h2 ? kb : ka;
    const float s = h2 ? ka : kb;
    k = fmaxf(k, __shfl_xor_sync(kFull, s, 2));
    return fmaxf(k, __shfl_xor_sync(kFull, k, 4));
}

// The two least-squares sums of four columns: the lane with band g ends with
// N (g even) or D (g odd) of column 2 ((g >> 1) & 1) + ((g >> 2) & 1); its
// partner lane g ^ 1 holds the other sum of the same column.
__device__ __forceinline__ int col8_of(int g) { return 2 * ((g >> 1) & 1) + ((g >> 2) & 1); }
__device__ __forceinline__ int col8_src(int lane, int c) { return (lane & ~7) | ((c >> 1) << 1) | ((c & 1) << 2); }

__device__ __forceinline__ float band_sum8(const float (&N)[4], const float (&Dn)[4], int g) {
    const bool h1 = g & 1, h2 = g & 2, h4 = g & 4;
    float k[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const float keep = h1 ? Dn[c] : N[c], send = h1 ? N[c] : Dn[c];
        k[c] = keep + __shfl_xor_sync(kFull, send, 1);
    }
    float ka = h2 ? k[2] : k[0], kb = h2 ? k[3] : k[1];
    const float sa = h2 ? k[0] : k[2], sb = h2 ? k[1] : k[3];
    ka = ka + __shfl_xor_sync(kFull, sa, 2);
    kb = kb + __shfl_xor_sync(kFull, sb, 2);
    float kk = h4 ? kb : ka;
    const float s = h4 ? ka : kb;
    return kk + __shfl_xor_sync(kFull, s, 4);
}

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
        } else {  // pairwise over the four columns
            rs[2 * k] = (fabsf(S[k][0].x) + fabsf(S[k][1].x)) + (fabsf(S[k][2].x) + fabsf(S[k][3].x));
            rs[2 * k + 1] = (fabsf(S[k][0].y) + fabsf(S[k][1].y)) + (fabsf(S[k][2].y) + fabsf(S[k][3].y));
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
    const int g = tid & 7, lane = tid & 31, i0 = g * RT, j0 = 4 * (tid >> 3);
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
    const float other = __shfl_xor_sync(kFull, mine, 1);
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
    const int i0 = (tid & 7) * RT;
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

// ---------------------------------------------------------------------------
// One quantized head of width B: decode / fit-pack / fused.  Returns true
// when a copy wait of the block gave up (the caller ends the kernel).  `ok`
// is this thread's wait result; `rel` refills the record's stage (thread 0)
// and is called right after the last block barrier that follows the last
// read of the stage.  No global memory is written before the vote.
// ---------------------------------------------------------------------------
template <int D, int B, int KIND, int S16, int QUANT, class Rel>
__device__ bool item_head(const Args &a, const uint8_t *stage, uint8_t *rec_g, int row, ScratchH<D> &sc, int tid,
                          bool ok, Rel &rel) {
    constexpr int NP = D / 16, RT = D / 8;
    const int g = tid & 7, cb = tid >> 3, lane = tid & 31, i0 = g * RT, j0 = 4 * cb;
    const uint32_t codes_bytes = (uint32_t)D * D * B / 8;
    const uint8_t *st_r = stage + codes_bytes;
    const uint8_t *st_c = st_r + D * (S16 ? 2 : 4);
    const float *tf = stage_tail<D>(a, stage);
    const float *qs = tf + kTailQ * D, *ks = tf + kTailK * D, *vs = tf + kTailV * D, *xs = tf + kTailX * D;
    const float *ab = stage_ab<D>(a, stage);
    const float alpha = ab[0];

    uint32_t W[Stream<D, B>::NW];
    load_stream<D, B>(stage, tid, W);
    const float4 c4 = scale4_at(st_c, j0, S16);
    const float2 cd[4] = {make_float2(c4.x, c4.x), make_float2(c4.y, c4.y), make_float2(c4.z, c4.z),
                          make_float2(c4.w, c4.w)};
    const float2 al2 = make_float2(alpha, alpha);

    // reconstruct S' = fl(fl(a_i c_j) z), a_i = fl(alpha r_i); u chains
    float2 S[NP][4];
    float2 acc[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[c] = make_float2(0.0f, 0.0f);
    float2 rp[NP], kp[NP];
    load_scale_pairs<NP>(st_r, i0, S16, rp);
    load_pairs<NP>(ks + i0, kp);
#pragma unroll
    for (int k = 0; k < NP; ++k) {
        const float2 a2 = mul2(rp[k], al2);
        float2 z[4];
        unpack_pair<D, B>(W, k, z);
        const float2 k2 = kp[k];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            S[k][c] = mul2(mul2(a2, cd[c]), z[c]);
            if (KIND != kFitPack) acc[c] = fma2(k2, S[k][c], acc[c]);
        }
    }
    // w of the four columns
    float2 wd[4];
    float w_mine = 0.0f;
    const int cs = col4_of(g);
    if (KIND != kFitPack) {
        const float u = band_sum4(acc[0].x + acc[0].y, acc[1].x + acc[1].y, acc[2].x + acc[2].y, acc[3].x + acc[3].y, g);
        w_mine = __fmul_rn(ab[1], __fsub_rn(vs[j0 + cs], u));
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const float t = __shfl_sync(kFull, w_mine, col4_src(lane, c));
            wd[c] = make_float2(t, t);
        }
    } else {
        const float4 w4 = *reinterpret_cast<const float4 *>(xs + j0);
        wd[0] = make_float2(w4.x, w4.x);
        wd[1] = make_float2(w4.y, w4.y);
        wd[2] = make_float2(w4.z, w4.z);
        wd[3] = make_float2(w4.w, w4.w);
    }
    // S = fma(k, w, S'); o chains
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[c] = make_float2(0.0f, 0.0f);
    load_pairs<NP>(ks + i0, kp);
    if (KIND != kFitPack) load_pairs<NP>(qs + i0, rp);
#pragma unroll
    for (int k = 0; k < NP; ++k) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            S[k][c] = fma2(kp[k], wd[c], S[k][c]);
            if (KIND != kFitPack) acc[c] = fma2(rp[k], S[k][c], acc[c]);
        }
    }
    // the row partials go out first: the readout's shuffles then overlap the
    // stores and the wait at the block barrier
    if (KIND != kDecode) row_partials<D, QUANT>(S, sc, g, cb);
    float o_mine = 0.0f;
    if (KIND != kFitPack)
        o_mine = band_sum4(acc[0].x + acc[0].y, acc[1].x + acc[1].y, acc[2].x + acc[2].y, acc[3].x + acc[3].y, g);
    if (KIND == kDecode) {
        if (__syncthreads_or(!ok)) return true;
        rel();
        if ((g & 4) == 0) {
            a.o[(size_t)row * D + j0 + cs] = o_mine;
            a.w[(size_t)row * D + j0 + cs] = w_mine;
        }
        return false;
    }
    if (__syncthreads_or(!ok)) return true;
    if (KIND == kFused && (g & 4) == 0) a.o[(size_t)row * D + j0 + cs] = o_mine;
    uint8_t *rec_r = rec_g + codes_bytes;
    uint8_t *rec_c = rec_r + D * (S16 ? 2 : 4);
    row_phase<D, B, S16, QUANT>(sc, tid, tf + kTailRho * D, tf + kTailWbar * D, rec_r);
    rel();
    if (QUANT == kQuantAbsmax) {
        if (tid < D) scale_put(rec_c, tid, 1.0f, S16);
        absmax_codes<D, B>(S, sc, tid, W);
    } else {
        fit_codes<D, B, S16>(S, sc, tid, rec_c, W);
    }
    store_stream<D, B>(rec_g, tid, W);
    return false;
}

// One FP16 pivot head (binary16 tile, row-major, read and written in place).
template <int D, int KIND, class Rel>
__device__ bool item_pivot(const Args &a, const uint8_t *stage, uint8_t *rec_g, int row, int tid, bool ok, Rel &rel) {
    constexpr int NP = D / 16, RT = D / 8;
    const int g = tid & 7, lane = tid & 31, i0 = g * RT, j0 = 4 * (tid >> 3);
    const float *tf = stage_tail<D>(a, stage);
    const float *qs = tf + kTailQ * D, *ks = tf + kTailK * D, *vs = tf + kTailV * D, *xs = tf + kTailX * D;
    const float *ab = stage_ab<D>(a, stage);
    const float alpha = ab[0];
    float2 S[NP][4];
    float2 acc[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[c] = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int k = 0; k < NP; ++k) {
        const int i = i0 + 2 * k;
        const uint2 ha = *reinterpret_cast<const uint2 *>(rec_g + ((size_t)i * D + j0) * 2);
        const uint2 hb = *reinterpret_cast<const uint2 *>(rec_g + ((size_t)(i + 1) * D + j0) * 2);
        const float2 a01 = __half22float2(*reinterpret_cast<const __half2 *>(&ha.x));
        const float2 a23 = __half22float2(*reinterpret_cast<const __half2 *>(&ha.y));
        const float2 b01 = __half22float2(*reinterpret_cast<const __half2 *>(&hb.x));
        const float2 b23 = __half22float2(*reinterpret_cast<const __half2 *>(&hb.y));
        const float2 al2 = make_float2(alpha, alpha);
        S[k][0] = mul2(al2, make_float2(a01.x, b01.x));
        S[k][1] = mul2(al2, make_float2(a01.y, b01.y));
        S[k][2] = mul2(al2, make_float2(a23.x, b23.x));
        S[k][3] = mul2(al2, make_float2(a23.y, b23.y));
        if (KIND != kFitPack) {
            const float2 k2 = *reinterpret_cast<const float2 *>(ks + i);
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[c] = fma2(k2, S[k][c], acc[c]);
        }
    }
    float2 wd[4];
    float w_mine = 0.0f;
    const int cs = col4_of(g);
    if (KIND != kFitPack) {
        const float u = band_sum4(acc[0].x + acc[0].y, acc[1].x + acc[1].y, acc[2].x + acc[2].y, acc[3].x + acc[3].y, g);
        w_mine = __fmul_rn(ab[1], __fsub_rn(vs[j0 + cs], u));
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const float t = __shfl_sync(kFull, w_mine, col4_src(lane, c));
            wd[c] = make_float2(t, t);
        }
    } else {
        const float4 w4 = *reinterpret_cast<const float4 *>(xs + j0);
        wd[0] = make_float2(w4.x, w4.x);
        wd[1] = make_float2(w4.y, w4.y);
        wd[2] = make_float2(w4.z, w4.z);
        wd[3] = make_float2(w4.w, w4.w);
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[c] = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int k = 0; k < NP; ++k) {
        const int i = i0 + 2 * k;
        const float2 k2 = *reinterpret_cast<const float2 *>(ks + i);
        float2 q2;
        if (KIND != kFitPack) q2 = *reinterpret_cast<const float2 *>(qs + i);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            S[k][c] = fma2(k2, wd[c], S[k][c]);
            if (KIND != kFitPack) acc[c] = fma2(q2, S[k][c], acc[c]);
        }
    }
    float o_mine = 0.0f;
    if (KIND != kFitPack)
        o_mine = band_sum4(acc[0].x + acc[0].y, acc[1].x + acc[1].y, acc[2].x + acc[2].y, acc[3].x + acc[3].y, g);
    if (__syncthreads_or(!ok)) return true;
    rel();
    if (KIND != kFitPack && (g & 4) == 0) {
        a.o[(size_t)row * D + j0 + cs] = o_mine;
        if (KIND == kDecode) a.w[(size_t)row * D + j0 + cs] = w_mine;
    }
    if (KIND != kDecode) {
#pragma unroll
        for (int k = 0; k < NP; ++k) {
            const int i = i0 + 2 * k;
            const __half2 a01 = __floats2half2_rn(S[k][0].x, S[k][1].x), a23 = __floats2half2_rn(S[k][2].x, S[k][3].x);
            const __half2 b01 = __floats2half2_rn(S[k][0].y, S[k][1].y), b23 = __floats2half2_rn(S[k][2].y, S[k][3].y);
            *reinterpret_cast<uint2 *>(rec_g + ((size_t)i * D + j0) * 2) =
                make_uint2(*reinterpret_cast<const uint32_t *>(&a01), *reinterpret_cast<const uint32_t *>(&a23));
            *reinterpret_cast<uint2 *>(rec_g + ((size_t)(i + 1) * D + j0) * 2) =
                make_uint2(*reinterpret_cast<const uint32_t *>(&b01), *reinterpret_cast<const uint32_t *>(&b23));
        }
    }
    return false;
}

// ---------------------------------------------------------------------------
// Persistent pipeline kernel for per-head units.
// ---------------------------------------------------------------------------
template <int D, int KIND, int S16, int QUANT>
__global__ void __launch_bounds__(2 * D, 2) k_step_head(Args a) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x;
    const int G = gridDim.x;
    uint8_t *stages = smem;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kStages * a.stage_bytes);
    ScratchH<D> &sc = *reinterpret_cast<ScratchH<D> *>(smem + kStages * a.stage_bytes + 64);

    int dsel = 0;
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(&bars[s], 1);
        fence_mbar_init();
        for (int s = 0; s < kStages; ++s) {
            const int it = blockIdx.x + s * G;
            if (it >= a.n_items) break;
            int n, ll, di;
            step_coords<D>(a, it, n, ll, di);
            issue_item<D, KIND, 0>(a, it, a.t.desc[di], a.slots[n], stages + s * a.stage_bytes, &bars[s], sc.meta[s]);
        }
        const int nx = blockIdx.x + kStages * G;
        if (nx < a.n_items) prefetch_desc<D>(a, nx, sc.dring, sc.dslot, 0);
    }
    __syncthreads();
    int s = 0;
    uint32_t phase = 0;
    for (int it = blockIdx.x; it < a.n_items; it += G) {
        const bool ok = mbar_wait_bounded(&bars[s], phase, a.wait_polls);
        const int width = sc.meta[s][kMetaWidth];
        const int valid = sc.meta[s][kMetaValid];
        const int row = sc.meta[s][kMetaRow];
        uint8_t *rec_g = reinterpret_cast<uint8_t *>((uintptr_t)(uint32_t)sc.meta[s][kMetaRecLo] |
                                                     ((uintptr_t)(uint32_t)sc.meta[s][kMetaRecHi] << 32));
        uint8_t *stage = stages + s * a.stage_bytes;
        // thread 0: put item it + kStages G into this stage (every thread is past its reads)
        auto rel = [&]() {
            if (tid != 0) return;
            const int nx = it + kStages * G;
            if (nx >= a.n_items) return;
            cp_async_wait_all();
            issue_item<D, KIND, 0>(a, nx, sc.dring[dsel], sc.dslot[dsel], stage, &bars[s], sc.meta[s]);
            dsel ^= 1;
            if (nx + G < a.n_items) prefetch_desc<D>(a, nx + G, sc.dring, sc.dslot, dsel);
        };
        bool abort = false;
        if (!valid) {
            abort = __syncthreads_or(!ok);
            if (!abort) rel();
        } else {
            switch (width) {
                case 2: abort = item_head<D, 2, KIND, S16, QUANT>(a, stage, rec_g, row, sc, tid, ok, rel); break;
                case 4: abort = item_head<D, 4, KIND, S16, QUANT>(a, stage, rec_g, row, sc, tid, ok, rel); break;
                case 6: abort = item_head<D, 6, KIND, S16, QUANT>(a, stage, rec_g, row, sc, tid, ok, rel); break;
                case 8: abort = item_head<D, 8, KIND, S16, QUANT>(a, stage, rec_g, row, sc, tid, ok, rel); break;
                case kPivotBits: abort = item_pivot<D, KIND>(a, stage, rec_g, row, tid, ok, rel); break;
                default:
                    if (tid == 0) flag_error(a.err, kErrArgs);
                    abort = __syncthreads_or(!ok);
                    if (!abort) rel();
                    break;
            }
        }
        if (abort) {
            if (tid == 0) {
                flag_error(a.err, kErrWait);
                drain_copies(bars, s, phase, a.wait_polls);
            }
            return;
        }
        if (++s == kStages) {
            s = 0;
            phase ^= 1u;
        }
    }
}

// ---------------------------------------------------------------------------
// Pack fp32 states (S_0) and unpack records: one CTA per head, no pipeline.
// ---------------------------------------------------------------------------

// The fp32 tile of this thread from a row-major D x D state.
template <int D>
__device__ __forceinline__ void load_tile(const float *Sg, int tid, float2 (&S)[D / 16][4]) {
    constexpr int NP = D / 16, RT = D / 8;
    const int i0 = (tid & 7) * RT, j0 = 4 * (tid >> 3);
#pragma unroll
    for (int k = 0; k < NP; ++k) {
        const float4 x = *reinterpret_cast<const float4 *>(Sg + (size_t)(i0 + 2 * k) * D + j0);
        const float4 y = *reinterpret_cast<const float4 *>(Sg + (size_t)(i0 + 2 * k + 1) * D + j0);
        S[k][0] = make_float2(x.x, y.x);
        S[k][1] = make_float2(x.y, y.y);
        S[k][2] = make_float2(x.z, y.z);
        S[k][3] = make_float2(x.w, y.w);
    }
}

template <int D, int B, int S16, int QUANT>
__device__ void requant_head(float2 (&S)[D / 16][4], uint8_t *rec, ScratchH<D> &sc, int tid) {
    const uint32_t codes_bytes = (uint32_t)D * D * B / 8;
    uint8_t *rec_r = rec + codes_bytes;
    uint8_t *rec_c = rec_r + D * (S16 ? 2 : 4);
    row_partials<D, QUANT>(S, sc, tid & 7, tid >> 3);
    __syncthreads();
    row_phase<D, B, S16, QUANT>(sc, tid, sc.rho, sc.wbar, rec_r);
    uint32_t W[Stream<D, B>::NW];
    if (QUANT == kQuantAbsmax) {
        if (tid < D) scale_put(rec_c, tid, 1.0f, S16);
        absmax_codes<D, B>(S, sc, tid, W);
    } else {
        fit_codes<D, B, S16>(S, sc, tid, rec_c, W);
    }
    store_stream<D, B>(rec, tid, W);
}

template <int D, int S16, int QUANT>
__device__ void requant_width(int width, float2 (&S)[D / 16][4], uint8_t *rec, ScratchH<D> &sc, int tid, int *err) {
    switch (width) {
        case 2: requant_head<D, 2, S16, QUANT>(S, rec, sc, tid); break;
        case 4: requant_head<D, 4, S16, QUANT>(S, rec, sc, tid); break;
        case 6: requant_head<D, 6, S16, QUANT>(S, rec, sc, tid); break;
        case 8: requant_head<D, 8, S16, QUANT>(S, rec, sc, tid); break;
        default: if (tid == 0) flag_error(err, kErrArgs); break;
    }
}

template <int D>
__global__ void __launch_bounds__(2 * D) k_requant_head(Args a) {
    __shared__ ScratchH<D> sc;
    constexpr int NP = D / 16, RT = D / 8;
    const int tid = threadIdx.x;
    int n, ll, h, gl, row;
    item_coords<D>(a, blockIdx.x, n, ll, h, gl, row);
    const int slot = a.slots[n];
    if (slot < 0 || slot >= a.n_slots) {
        if (tid == 0) flag_error(a.err, kErrBadSlot);
        return;
    }
    uint8_t *rec = a.pool + (uint64_t)slot * a.slot_bytes + a.t.rec_off[gl];
    float2 S[NP][4];
    load_tile<D>(a.S_in + (size_t)row * D * D, tid, S);
    const int width = a.t.width[gl];
    if (width == kPivotBits) {
        const int i0 = (tid & 7) * RT, j0 = 4 * (tid >> 3);
#pragma unroll
        for (int k = 0; k < NP; ++k) {
            const int i = i0 + 2 * k;
            const __half2 a01 = __floats2half2_rn(S[k][0].x, S[k][1].x), a23 = __floats2half2_rn(S[k][2].x, S[k][3].x);
            const __half2 b01 = __floats2half2_rn(S[k][0].y, S[k][1].y), b23 = __floats2half2_rn(S[k][2].y, S[k][3].y);
            *reinterpret_cast<uint2 *>(rec + ((size_t)i * D + j0) * 2) =
                make_uint2(*reinterpret_cast<const uint32_t *>(&a01), *reinterpret_cast<const uint32_t *>(&a23));
            *reinterpret_cast<uint2 *>(rec + ((size_t)(i + 1) * D + j0) * 2) =
                make_uint2(*reinterpret_cast<const uint32_t *>(&b01), *reinterpret_cast<const uint32_t *>(&b23));
        }
        return;
    }
    if (tid < D) {
        sc.rho[tid] = a.t.rho[(size_t)gl * D + tid];
        sc.wbar[tid] = a.t.wbar[(size_t)gl * D + tid];
    }
    __syncthreads();
    if (a.scale16) {
        if (a.quantizer == kQuantAbsmax) requant_width<D, 1, kQuantAbsmax>(width, S, rec, sc, tid, a.err);
        else requant_width<D, 1, kQuantDualAxis>(width, S, rec, sc, tid, a.err);
    } else {
        if (a.quantizer == kQuantAbsmax) requant_width<D, 0, kQuantAbsmax>(width, S, rec, sc, tid, a.err);
        else requant_width<D, 0, kQuantDualAxis>(width, S, rec, sc, tid, a.err);
    }
}

// X_hat = fl(fl(r_i c_j) z_ij) of one record into a row-major fp32 D x D array.
template <int D, int B>
__device__ void unpack_head(const uint8_t *rec, float *out, int tid, int s16) {
    constexpr int NP = D / 16, RT = D / 8;
    const int i0 = (tid & 7) * RT, j0 = 4 * (tid >> 3);
    const uint32_t codes_bytes = (uint32_t)D * D * B / 8;
    const uint8_t *rr = rec + codes_bytes;
    const uint8_t *cc = rr + D * (s16 ? 2 : 4);
    uint32_t W[Stream<D, B>::NW];
    load_stream<D, B>(rec, tid, W);
    const float4 c4 = scale4_at(cc, j0, s16);
    const float2 cd[4] = {make_float2(c4.x, c4.x), make_float2(c4.y, c4.y), make_float2(c4.z, c4.z),
                          make_float2(c4.w, c4.w)};
#pragma unroll
    for (int k = 0; k < NP; ++k) {
        const int i = i0 + 2 * k;
        const float2 r2 = scale2_at(rr, i, s16);
        float2 z[4], x[4];
        unpack_pair<D, B>(W, k, z);
#pragma unroll
        for (int c = 0; c < 4; ++c) x[c] = mul2(mul2(r2, cd[c]), z[c]);
        *reinterpret_cast<float4 *>(out + (size_t)i * D + j0) = make_float4(x[0].x, x[1].x, x[2].x, x[3].x);
        *reinterpret_cast<float4 *>(out + (size_t)(i + 1) * D + j0) = make_float4(x[0].y, x[1].y, x[2].y, x[3].y);
    }
}

template <int D>
__global__ void __launch_bounds__(2 * D) k_unpack_head(Args a) {
    constexpr int RT = D / 8;
    const int tid = threadIdx.x;
    int n, ll, h, gl, row;
    item_coords<D>(a, blockIdx.x, n, ll, h, gl, row);
    const int slot = a.slots[n];
    if (slot < 0 || slot >= a.n_slots) {
        if (tid == 0) flag_error(a.err, kErrBadSlot);
        return;
    }
    const uint8_t *rec = a.pool + (uint64_t)slot * a.slot_bytes + a.t.rec_off[gl];
    float *out = a.S_out + (size_t)row * D * D;
    switch (a.t.width[gl]) {
        case 2: unpack_head<D, 2>(rec, out, tid, a.scale16); break;
        case 4: unpack_head<D, 4>(rec, out, tid, a.scale16); break;
        case 6: unpack_head<D, 6>(rec, out, tid, a.scale16); break;
        case 8: unpack_head<D, 8>(rec, out, tid, a.scale16); break;
        case kPivotBits: {
            const int i0 = (tid & 7) * RT, j0 = 4 * (tid >> 3);
#pragma unroll
            for (int r = 0; r < RT; ++r) {
                const int i = i0 + r;
                const uint2 v = *reinterpret_cast<const uint2 *>(rec + ((size_t)i * D + j0) * 2);
                const float2 x01 = __half22float2(*reinterpret_cast<const __half2 *>(&v.x));
                const float2 x23 = __half22float2(*reinterpret_cast<const __half2 *>(&v.y));
                *reinterpret_cast<float4 *>(out + (size_t)i * D + j0) = make_float4(x01.x, x01.y, x23.x, x23.y);
            }
            break;
        }
        default: if (tid == 0) flag_error(a.err, kErrArgs); break;
    }
}

// ---------------------------------------------------------------------------
// Calibration distortion d_u(b) (方法-1): squared reconstruction error per key
// row when the whole head is quantized at uniform width B, accumulated into
// dist_acc[(gl*D + i)*n_bits + m].  Row weights: wbar from the calibration,
// rho_i = fl32(1/sqrt(sqrt(wbar_i))) (fp64).  One CTA per (item, width).
// ---------------------------------------------------------------------------
struct BitList {
    int b[4];
    int n;
};

template <int D, int B>
__device__ void dist_head(const float *Sg, int gl, int m, int n_bits, double *dist_acc, ScratchH<D> &sc, int tid) {
    constexpr int NP = D / 16, RT = D / 8, Q = (1 << (B - 1)) - 1;
    const int g = tid & 7, lane = tid & 31, i0 = g * RT, j0 = 4 * (tid >> 3);
    float2 S[NP][4];
    load_tile<D>(Sg, tid, S);
    row_partials<D, kQuantDualAxis>(S, sc, g, tid >> 3);
    __syncthreads();
    row_phase<D, B, 0, kQuantDualAxis>(sc, tid, sc.rho, sc.wbar, nullptr);
    uint32_t W[Stream<D, B>::NW];
    float cq[4];
    fit_codes<D, B, 0>(S, sc, tid, nullptr, W, cq);
    // the codes again from the tile's stream, the reconstruction and its error
    float2 z[NP][4];
#pragma unroll
    for (int k = 0; k < NP; ++k) unpack_pair<D, B>(W, k, z[k]);
    const float4 *src = nullptr;
    (void)src;
#pragma unroll
    for (int k = 0; k < NP; ++k) {
        const int i = i0 + 2 * k;
        const float2 r2 = make_float2(sc.rowr[i], sc.rowr[i + 1]);
        const float4 xa = *reinterpret_cast<const float4 *>(Sg + (size_t)i * D + j0);
        const float4 xb = *reinterpret_cast<const float4 *>(Sg + (size_t)(i + 1) * D + j0);
        const float oa[4] = {xa.x, xa.y, xa.z, xa.w}, ob[4] = {xb.x, xb.y, xb.z, xb.w};
        double ea = 0.0, eb = 0.0;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const float2 sh = mul2(mul2(r2, make_float2(cq[c], cq[c])), z[k][c]);
            const double da = (double)sh.x - (double)oa[c], db = (double)sh.y - (double)ob[c];
            ea = fma(da, da, ea);
            eb = fma(db, db, eb);
        }
        // the row's other column blocks of this warp (lanes xor 8, 16)
        ea += __shfl_xor_sync(kFull, ea, 8);
        ea += __shfl_xor_sync(kFull, ea, 16);
        eb += __shfl_xor_sync(kFull, eb, 8);
        eb += __shfl_xor_sync(kFull, eb, 16);
        if ((lane >> 3) == 0) {
            atomicAdd(&dist_acc[((size_t)gl * D + i) * n_bits + m], ea);
            atomicAdd(&dist_acc[((size_t)gl * D + i + 1) * n_bits + m], eb);
        }
    }
    (void)Q;
}

template <int D>
__global__ void __launch_bounds__(2 * D) k_calib_dist(Args a, BitList bl, double *dist_acc) {
    __shared__ ScratchH<D> sc;
    const int tid = threadIdx.x;
    const int m = blockIdx.y;
    int n, ll, h, gl, row;
    item_coords<D>(a, blockIdx.x, n, ll, h, gl, row);
    if (tid < D) {
        const float wb = a.t.wbar[(size_t)gl * D + tid];
        sc.wbar[tid] = wb;
        sc.rho[tid] = (float)(1.0 / sqrt(sqrt((double)wb)));
    }
    __syncthreads();
    const float *Sg = a.S_in + (size_t)row * D * D;
    switch (bl.b[m]) {
        case 2: dist_head<D, 2>(Sg, gl, m, bl.n, dist_acc, sc, tid); break;
        case 4: dist_head<D, 4>(Sg, gl, m, bl.n, dist_acc, sc, tid); break;
        case 6: dist_head<D, 6>(Sg, gl, m, bl.n, dist_acc, sc, tid); break;
        case 8: dist_head<D, 8>(Sg, gl, m, bl.n, dist_acc, sc, tid); break;
        default: if (tid == 0) flag_error(a.err, kErrArgs); break;
    }
}

// ---------------------------------------------------------------------------
// Host-side launchers.
// ---------------------------------------------------------------------------
template <int D>
size_t step_smem_head(uint32_t stage_bytes) {
    return (size_t)kStages * stage_bytes + 64 + sizeof(ScratchH<D>);
}

template <int D, int KIND, int S16, int QUANT>
static cudaError_t launch_head_k(const Args &a, int n_sms, cudaStream_t st, int *grid_out) {
    const size_t smem = step_smem_head<D>(a.stage_bytes);
    auto kern = k_step_head<D, KIND, S16, QUANT>;
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

template <int D, int KIND>
static cudaError_t launch_head_d(const Args &a, int n_sms, cudaStream_t st, int *grid) {
    if (a.scale16) {
        return a.quantizer == kQuantAbsmax ? launch_head_k<D, KIND, 1, kQuantAbsmax>(a, n_sms, st, grid)
                                           : launch_head_k<D, KIND, 1, kQuantDualAxis>(a, n_sms, st, grid);
    }
    return a.quantizer == kQuantAbsmax ? launch_head_k<D, KIND, 0, kQuantAbsmax>(a, n_sms, st, grid)
                                       : launch_head_k<D, KIND, 0, kQuantDualAxis>(a, n_sms, st, grid);
}

template <int KIND>
static cudaError_t launch_head_kind(int D, const Args &a, int n_sms, cudaStream_t st, int *grid) {
    switch (D) {
        case 16: return launch_head_d<16, KIND>(a, n_sms, st, grid);
        case 32: return launch_head_d<32, KIND>(a, n_sms, st, grid);
        case 64: return launch_head_d<64, KIND>(a, n_sms, st, grid);
        case 128: return launch_head_d<128, KIND>(a, n_sms, st, grid);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_step_head(int kind, int D, const Args &a, int n_sms, cudaStream_t st, int *grid) {
    switch (kind) {
        case kDecode: return launch_head_kind<kDecode>(D, a, n_sms, st, grid);
        case kFitPack: return launch_head_kind<kFitPack>(D, a, n_sms, st, grid);
        case kFused: return launch_head_kind<kFused>(D, a, n_sms, st, grid);
        default: return cudaErrorInvalidValue;
    }
}

size_t step_smem_head_bytes(int D, uint32_t stage_bytes) {
    switch (D) {
        case 16: return step_smem_head<16>(stage_bytes);
        case 32: return step_smem_head<32>(stage_bytes);
        case 64: return step_smem_head<64>(stage_bytes);
        default: return step_smem_head<128>(stage_bytes);
    }
}

template <int D>
static cudaError_t launch_pack_head_d(const Args &a, bool unpack, cudaStream_t st) {
    if (a.n_items <= 0) return cudaSuccess;
    if (unpack) k_unpack_head<D><<<a.n_items, 2 * D, 0, st>>>(a);
    else k_requant_head<D><<<a.n_items, 2 * D, 0, st>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_pack_head(int D, const Args &a, bool unpack, cudaStream_t st) {
    switch (D) {
        case 16: return launch_pack_head_d<16>(a, unpack, st);
        case 32: return launch_pack_head_d<32>(a, unpack, st);
        case 64: return launch_pack_head_d<64>(a, unpack, st);
        case 128: return launch_pack_head_d<128>(a, unpack, st);
        default: return cudaErrorInvalidValue;
    }
}

template <int D>
static cudaError_t launch_dist_d(const Args &a, const BitList &bl, double *acc, cudaStream_t st) {
    if (a.n_items <= 0) return cudaSuccess;
    k_calib_dist<D><<<dim3(a.n_items, bl.n), 2 * D, 0, st>>>(a, bl, acc);
    return cudaGetLastError();
}

cudaError_t launch_calib_dist(int D, const Args &a, const int *bits, int n_bits, double *acc, cudaStream_t st) {
    BitList bl{};
    if (n_bits < 1 || n_bits > 4) return cudaErrorInvalidValue;
    for (int i = 0; i < n_bits; ++i) bl.b[i] = bits[i];
    bl.n = n_bits;
    switch (D) {
        case 16: return launch_dist_d<16>(a, bl, acc, st);
        case 32: return launch_dist_d<32>(a, bl, acc, st);
        case 64: return launch_dist_d<64>(a, bl, acc, st);
        case 128: return launch_dist_d<128>(a, bl, acc, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace stepq
