// Packed-state decode step kernels for per-key-row units (KDA, plan mode 1),
// and the launchers of the step and pack kernels of both unit kinds.
//
// STEPQuant paper digest (vibe-research), 方法-1 (KDA: a single key row is
// the allocation unit, each with its own width 2/4/6/8 or FP16) and 方法-4
// (reconstruct -> retention + delta update + readout -> refit -> pack ->
// write back).  Arithmetic definitions: include/stepq.h.
//
// Mapping: the one of the per-head kernels (stepq_head.cuh).  Thread t owns
// tile t of the band-tile code layout: rows [16 g, 16 g + 16) x columns
// [4 cb, 4 cb + 4), g = band_of(t), cb = cblk_of(t); a warp holds 16 whole
// value columns, so u, o, the column maxima and the least-squares sums are
// warp shuffles in the band order and only the row sums cross warps.  Every
// row has its own width: a thread walks its tile stream row by row with the
// row's width in a register (widths differ from lane to lane, so the code
// fields are cut with run-time shifts and masks), and the lanes holding an
// FP16 row take a branch of their own for it.  A tile stream is the tile's
// own run of 32-bit words, so the new codes go straight from registers to
// the record, word by word.
#include "stepq_head.cuh"

namespace stepq {
namespace kda {

constexpr int D = 128, NT = 2 * D, RT = D / 8, NP = D / 16, NCB = D / 4;

// Shared memory besides the stages.
struct __align__(16) ScratchR {
    ScratchH<D> h;     // row partials, 1/r, b, r, rho, wbar, descriptors, stage metadata
    float iq[D];       // fl(1/qmax_i); 0 for FP16 rows
    uint32_t mgb[D];   // bits of 1.5 2^23 + 2^(b_i - 1): the rounding constant of row i's final codes
    uint32_t ones[D];  // sum_c 2^(c b_i): the offset 1 of each of the row's four fields
    uint16_t bnd[D];   // 2 qmax_i: the clamp bound of e = z + qmax_i (0 for FP16 rows, like the two above)
    uint8_t rw[D];     // row widths (16 = FP16 row)
    uint32_t roff[D];  // (first word of the row's band block) << 11 | stream bit of the row
};

// Width of row r of this thread's band from its 16 width bytes.
__device__ __forceinline__ uint32_t wid(const uint4 &w, int r) {
    const uint32_t x = r < 4 ? w.x : r < 8 ? w.y : r < 12 ? w.z : w.w;
    return __byte_perm(x, 0u, 0x4440u | (uint32_t)(r & 3));
}

// Byte offset of this thread's tile word 0 in the codes block (band block of
// g, then the tile's rotated column position).
__device__ __forceinline__ uint32_t tile_byte0(uint32_t roff_band, int g, int cb) {
    return 4u * ((roff_band >> 11) + (uint32_t)((cb + 4 * g) & (NCB - 1)));
}

// 32 stream bits of the tile from stream bit P on.
__device__ __forceinline__ uint32_t bits32(const uint8_t *tile0, uint32_t P) {
    const uint32_t *p = reinterpret_cast<const uint32_t *>(tile0 + (P >> 5) * (4u * NCB));
    return __funnelshift_r(p[0], p[NCB], P & 31u);
}

// The four binary16 values (64 stream bits) of an FP16 row from stream bit P on.
__device__ __forceinline__ void halves4(const uint8_t *tile0, uint32_t P, float (&h)[4]) {
    const uint32_t *p = reinterpret_cast<const uint32_t *>(tile0 + (P >> 5) * (4u * NCB));
    const uint32_t s = P & 31u;
    const uint32_t lo = __funnelshift_r(p[0], p[NCB], s), hi = __funnelshift_r(p[NCB], p[2 * NCB], s);
    h[0] = __half2float(__ushort_as_half((unsigned short)(lo & 0xffffu)));
    h[1] = __half2float(__ushort_as_half((unsigned short)(lo >> 16)));
    h[2] = __half2float(__ushort_as_half((unsigned short)(hi & 0xffffu)));
    h[3] = __half2float(__ushort_as_half((unsigned short)(hi >> 16)));
}

// z of rows (2k, 2k+1) x the tile's 4 columns, rows of widths ba, bb at
// stream bits P and P + 4 ba.  A field u goes into the low mantissa bits of
// 2^23 (exact 2^23 + u), and one packed subtraction of 2^23 + 2^(b-1) leaves
// z.  An FP16 row gives finite values here that its caller replaces.
__device__ __forceinline__ void unpack_pair_rows(const uint8_t *tile0, uint32_t P, uint32_t ba, uint32_t bb,
                                                 float2 (&z)[4]) {
    uint32_t xa = bits32(tile0, P), xb = bits32(tile0, P + 4u * ba);
    const uint32_t ma = (1u << ba) - 1u, mb = (1u << bb) - 1u;
    const float2 nb = make_float2(__uint_as_float(0xCB000000u | (1u << (ba - 1u))),
                                  __uint_as_float(0xCB000000u | (1u << (bb - 1u))));
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        z[c] = add2(make_float2(__uint_as_float((xa & ma) | 0x4B000000u), __uint_as_float((xb & mb) | 0x4B000000u)), nb);
        xa >>= ba;
        xb >>= bb;
    }
}

// The codes of this tile, appended to its stream and written to the record
// word by word (own words only: word m of the tile at tile0 + 4 NCB m).  Every
// put stores the word it reaches, complete or not (a partial word is stored
// again once more bits have joined it), so the lanes of a warp, whose rows
// have different widths, run it without a branch.
struct StreamOut {
    uint8_t *tile0;
    uint32_t acc = 0, fill = 0, m = 0;
    __device__ __forceinline__ void put(uint32_t f, uint32_t nbits) {  // 0 < nbits <= 32
        acc |= f << fill;
        *reinterpret_cast<uint32_t *>(tile0 + m * (4u * NCB)) = acc;
        const uint32_t nf = fill + nbits;
        const bool full = nf >= 32u;
        const uint32_t spill = __funnelshift_l(f, 0u, fill);  // the bits of f past the word end (0 when fill = 0)
        acc = full ? spill : acc;
        m += full ? 1u : 0u;
        fill = nf & 31u;
    }
    __device__ __forceinline__ void flush() {
        if (fill) *reinterpret_cast<uint32_t *>(tile0 + m * (4u * NCB)) = acc;
    }
};

// sum_c e_c 2^(c b) of a row of width b from its four clamped codes e_c in
// [0, 2 qmax], held in the low (hi = false) or high 16 bits of e[c]; adding
// the row's `ones` gives the field, u_c = e_c + 1 at bits [c b, c b + b).
__device__ __forceinline__ uint32_t field4(const uint32_t (&e)[4], bool hi, uint32_t b) {
    const uint32_t M = 1u << b;
    uint32_t f = hi ? (e[3] >> 16) : (e[3] & 0xffffu);
    f = f * M + (hi ? (e[2] >> 16) : (e[2] & 0xffffu));
    f = f * M + (hi ? (e[1] >> 16) : (e[1] & 0xffffu));
    f = f * M + (hi ? (e[0] >> 16) : (e[0] & 0xffffu));
    return f;
}

// Row phase of per-row units (between the first and the second block barrier
// of a record): two threads per row finish the pairwise row sum and form r_i,
// 1/r_i, b_i and fl(1/qmax_i).  FP16 rows get r = b = fl(1/qmax) = 0 and a
// factor 1 in place of 1/r, so that the binary16 pattern their registers hold
// passes the fit unchanged and adds exact zeros to its sums.  The row widths
// and offsets are copied out of the stage for the passes after its release.
// Ends with the second barrier.
template <int S16>
__device__ __forceinline__ void row_phase_rows(ScratchR &sc, int tid, const float *rho, const float *wbar,
                                               const uint8_t *rw, const uint32_t *roff, uint8_t *rec_r) {
    constexpr int HB = NCB / 2;
    const int i = tid >> 1, h = tid & 1;
    float v[HB];
#pragma unroll
    for (int m = 0; m < HB; ++m) v[m] = sc.h.part[pidx<D>(h * HB + m, i)];
    float s = pairwise_tree<HB>(v);
    s = s + __shfl_xor_sync(kFull, s, 1);
    const uint32_t b = rw[i];
    float ri = 0.0f, inv = 0.0f, bw = 0.0f, iq = 0.0f;
    uint32_t mgb = 0u, ones = 0u, bnd = 0u;
    if (b == (uint32_t)kPivotBits) {
        inv = 1.0f;  // y = S: an FP16 row's register holds its binary16 pattern as a tiny fp32 value
    } else {
        const float m = fmaxf(__fmul_rn(s, 1.0f / (float)D), 1e-12f);
        ri = scale_round(__fmul_rn(m, rho[i]), S16);
        inv = __frcp_rn(ri);
        bw = __fmul_rn(wbar[i], __fmul_rn(ri, ri));
        iq = __frcp_rn((float)((1u << (b - 1u)) - 1u));
        mgb = 0x4B400000u + (1u << (b - 1u));
        ones = 1u + (1u << b) + (1u << (2u * b)) + (1u << (3u * b));
        bnd = (1u << b) - 2u;
    }
    if (h == 0) {
        sc.h.rinv[i] = inv;
        sc.h.rowr[i] = ri;
        sc.rw[i] = (uint8_t)b;
        sc.mgb[i] = mgb;
        sc.ones[i] = ones;
        if (rec_r) scale_put(rec_r, i, ri, S16);
    } else {
        sc.h.bw[i] = bw;
        sc.iq[i] = iq;
        sc.bnd[i] = (uint16_t)bnd;
        sc.roff[i] = roff[i];
    }
    __syncthreads();
}

// After the row phase: y = fl(S fl(1/r)), c0_j = max_i fl(|y_ij| iq_i), the
// initial codes, the least-squares refinement of c, then the final codes of
// the tile written to the record (codes block at rec, c to rec_c).
template <int S16, bool HAS16>
__device__ __forceinline__ void fit_pack_rows(float2 (&S)[NP][4], const ScratchR &sc, int tid, uint8_t *rec,
                                              uint8_t *rec_c) {
    const int g = band_of(tid), cb = cblk_of(tid), lane = tid & 31, i0 = g * RT, j0 = 4 * cb;
    float m[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    {
        float2 pr[NP], qi[NP];
        load_pairs<NP>(&sc.h.rinv[i0], pr);
        load_pairs<NP>(&sc.iq[i0], qi);
#pragma unroll
        for (int k = 0; k < NP; ++k) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                S[k][c] = mul2(S[k][c], pr[k]);
                const float2 a = mul2(S[k][c], qi[k]);  // |fl(y iq)| = fl(|y| iq)
                m[c] = max3abs(m[c], a.x, a.y);
            }
        }
    }
    const float mx = band_max4(m[0], m[1], m[2], m[3], g);
    const float c0 = (mx == 0.0f) ? 1.0f : mx;
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
    {
        float2 pr[NP];
        load_pairs<NP>(&sc.h.bw[i0], pr);
#pragma unroll
        for (int k = 0; k < NP; ++k) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float2 z0 = add2(fma2(S[k][c], ic0d[c], mg), nmg);
                const float2 t = mul2(pr[k], z0);
                na[c] = fma2(t, S[k][c], na[c]);
                da[c] = fma2(t, z0, da[c]);
            }
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
    }
    // final codes: T = fma(y, 1/c, 1.5 2^23 + 2^(b-1)) per element (the offset
    // lands in the mantissa of 1.5 2^23, 0x4B400000); the low 16 bits of a row
    // pair's two results are joined and clamped to [0, 2 qmax]
    const uint4 wv = *reinterpret_cast<const uint4 *>(&sc.rw[i0]);
    StreamOut out;
    out.tile0 = rec + tile_byte0(sc.roff[i0], g, cb);
#pragma unroll
    for (int k = 0; k < NP; ++k) {
        const uint32_t ba = wid(wv, 2 * k), bb = wid(wv, 2 * k + 1);
        const uint2 mgp = *reinterpret_cast<const uint2 *>(&sc.mgb[i0 + 2 * k]);
        const uint2 onp = *reinterpret_cast<const uint2 *>(&sc.ones[i0 + 2 * k]);
        const uint32_t bound = *reinterpret_cast<const uint32_t *>(&sc.bnd[i0 + 2 * k]);
        const float2 mg2 = make_float2(__uint_as_float(mgp.x), __uint_as_float(mgp.y));
        uint32_t e[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const float2 T = fma2(S[k][c], icd[c], mg2);
            e[c] = __viaddmin_s16x2_relu(__byte_perm(__float_as_uint(T.x), __float_as_uint(T.y), 0x5410u), 0xFFFFFFFFu, bound);
        }
        if (!HAS16 || (ba != (uint32_t)kPivotBits && bb != (uint32_t)kPivotBits)) {
            out.put(field4(e, false, ba) + onp.x, 4u * ba);
            out.put(field4(e, true, bb) + onp.y, 4u * bb);
        } else {  // FP16 rows carry their binary16 patterns in the low bits of S (see item_rows)
#pragma unroll
            for (int hs = 0; hs < 2; ++hs) {
                const uint32_t b = hs ? bb : ba;
                if (b == (uint32_t)kPivotBits) {
                    const uint32_t x0 = __float_as_uint(hs ? S[k][0].y : S[k][0].x), x1 = __float_as_uint(hs ? S[k][1].y : S[k][1].x);
                    const uint32_t x2 = __float_as_uint(hs ? S[k][2].y : S[k][2].x), x3 = __float_as_uint(hs ? S[k][3].y : S[k][3].x);
                    out.put(__byte_perm(x0, x1, 0x5410u), 32u);
                    out.put(__byte_perm(x2, x3, 0x5410u), 32u);
                } else {
                    out.put(field4(e, hs != 0, b) + (hs ? onp.y : onp.x), 4u * b);
                }
            }
        }
    }
    out.flush();
}

// ---------------------------------------------------------------------------
// One head of per-row units: decode / fit-pack / fused.  Returns true when a
// copy wait of the block gave up.  `ok` is this thread's wait result; `rel`
// refills the record's stage (thread 0) and is called right after the last
// block barrier that follows the last read of the stage.  No global memory
// is written before the vote.
// ---------------------------------------------------------------------------
template <int KIND, int S16, bool HAS16, class Rel>
__device__ bool item_rows(const Args &a, const uint8_t *stage, uint8_t *rec_g, int row, uint32_t codes_bytes,
                          ScratchR &sc, int tid, bool ok, Rel &rel) {
    const int g = band_of(tid), cb = cblk_of(tid), lane = tid & 31, i0 = g * RT, j0 = 4 * cb;
    const uint8_t *st_r = stage + codes_bytes;
    const uint8_t *st_c = st_r + D * (S16 ? 2 : 4);
    const float *tf = stage_tail<D>(a, stage);
    const float *qs = tf + kTailQ * D, *ks = tf + kTailK * D, *vs = tf + kTailV * D, *xs = tf + kTailX * D;
    const float *als = tf + kTailAlpha * D;
    const uint32_t *roff = reinterpret_cast<const uint32_t *>(tf + kTailRoff * D);
    const uint8_t *rw = reinterpret_cast<const uint8_t *>(tf + kTailRw * D);
    const float *ab = stage_ab<D>(a, stage);

    const uint4 wv = *reinterpret_cast<const uint4 *>(rw + i0);
    const uint8_t *tile0 = stage + tile_byte0(roff[i0], g, cb);
    const float4 c4 = scale4_at(st_c, j0, S16);
    const float2 cd[4] = {make_float2(c4.x, c4.x), make_float2(c4.y, c4.y), make_float2(c4.z, c4.z),
                          make_float2(c4.w, c4.w)};

    // reconstruct S' = fl(fl(a_i c_j) z), a_i = fl(alpha_i r_i); FP16 rows
    // S' = fl(alpha_i h); u chains
    float2 S[NP][4];
    float2 acc[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[c] = make_float2(0.0f, 0.0f);
    {
        float2 ap[NP], rp[NP], kp[NP];
        load_pairs<NP>(als + i0, ap);
        load_scale_pairs<NP>(st_r, i0, S16, rp);
        load_pairs<NP>(ks + i0, kp);
        uint32_t P = 0;
#pragma unroll
        for (int k = 0; k < NP; ++k) {
            const uint32_t ba = wid(wv, 2 * k), bb = wid(wv, 2 * k + 1);
            float2 z[4];
            unpack_pair_rows(tile0, P, ba, bb, z);
            const float2 a2 = mul2(ap[k], rp[k]);
#pragma unroll
            for (int c = 0; c < 4; ++c) S[k][c] = mul2(mul2(a2, cd[c]), z[c]);
            if (HAS16 && (ba == (uint32_t)kPivotBits || bb == (uint32_t)kPivotBits)) {
                float h[4];
                if (ba == (uint32_t)kPivotBits) {
                    halves4(tile0, P, h);
#pragma unroll
                    for (int c = 0; c < 4; ++c) S[k][c].x = __fmul_rn(ap[k].x, h[c]);
                }
                if (bb == (uint32_t)kPivotBits) {
                    halves4(tile0, P + 4u * ba, h);
#pragma unroll
                    for (int c = 0; c < 4; ++c) S[k][c].y = __fmul_rn(ap[k].y, h[c]);
                }
            }
            if (KIND != kFitPack) {
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[c] = fma2(kp[k], S[k][c], acc[c]);
            }
            P += 4u * (ba + bb);
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
    // S = fma(k, w, S'); o chains; then FP16 rows keep their binary16 pattern
    // in the register for the refit to pass through
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[c] = make_float2(0.0f, 0.0f);
    {
        float2 kp[NP], qp[NP];
        load_pairs<NP>(ks + i0, kp);
        if (KIND != kFitPack) load_pairs<NP>(qs + i0, qp);
#pragma unroll
        for (int k = 0; k < NP; ++k) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                S[k][c] = fma2(kp[k], wd[c], S[k][c]);
                if (KIND != kFitPack) acc[c] = fma2(qp[k], S[k][c], acc[c]);
            }
            if (HAS16 && KIND != kDecode) {
                const uint32_t ba = wid(wv, 2 * k), bb = wid(wv, 2 * k + 1);
                if (ba == (uint32_t)kPivotBits || bb == (uint32_t)kPivotBits) {
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        if (ba == (uint32_t)kPivotBits)
                            S[k][c].x = __uint_as_float((uint32_t)__half_as_ushort(__float2half_rn(S[k][c].x)));
                        if (bb == (uint32_t)kPivotBits)
                            S[k][c].y = __uint_as_float((uint32_t)__half_as_ushort(__float2half_rn(S[k][c].y)));
                    }
                }
            }
        }
    }
    if (KIND != kDecode) row_partials<D, kQuantDualAxis>(S, sc.h, g, cb);
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
    row_phase_rows<S16>(sc, tid, tf + kTailRho * D, tf + kTailWbar * D, rw, roff, rec_r);
    rel();
    fit_pack_rows<S16, HAS16>(S, sc, tid, rec_g, rec_c);
    return false;
}

// ---------------------------------------------------------------------------
// Persistent pipeline kernel for per-row units (the protocol of k_step_head).
// ---------------------------------------------------------------------------
template <int KIND, int S16>
__global__ void __launch_bounds__(NT, 2) k_step_rows(Args a) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x;
    const int G = gridDim.x;
    uint8_t *stages = smem;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kStages * a.stage_bytes);
    ScratchR &sc = *reinterpret_cast<ScratchR *>(smem + kStages * a.stage_bytes + 64);

    int dsel = 0;
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(&bars[s], 1);
        fence_mbar_init();
        for (int s = 0; s < kStages; ++s) {
            const int it = blockIdx.x + s * G;
            if (it >= a.n_items) break;
            int n, ll, di;
            step_coords<D>(a, it, n, ll, di);
            issue_item<D, KIND, 1>(a, it, a.t.desc[di], a.slots[n], stages + s * a.stage_bytes, &bars[s], sc.h.meta[s]);
        }
        const int nx = blockIdx.x + kStages * G;
        if (nx < a.n_items) prefetch_desc<D>(a, nx, sc.h.dring, sc.h.dslot, 0);
    }
    __syncthreads();
    int s = 0;
    uint32_t phase = 0;
    for (int it = blockIdx.x; it < a.n_items; it += G) {
        const bool ok = mbar_wait_bounded(&bars[s], phase, a.wait_polls);
        const int valid = sc.h.meta[s][kMetaValid];
        const int row = sc.h.meta[s][kMetaRow];
        const uint32_t codes_bytes = (uint32_t)sc.h.meta[s][kMetaCodes];
        uint8_t *rec_g = reinterpret_cast<uint8_t *>((uintptr_t)(uint32_t)sc.h.meta[s][kMetaRecLo] |
                                                     ((uintptr_t)(uint32_t)sc.h.meta[s][kMetaRecHi] << 32));
        uint8_t *stage = stages + s * a.stage_bytes;
        // thread 0: put item it + kStages G into this stage (every thread is past its reads)
        auto rel = [&]() {
            if (tid != 0) return;
            const int nx = it + kStages * G;
            if (nx >= a.n_items) return;
            cp_async_wait_all();
            issue_item<D, KIND, 1>(a, nx, sc.h.dring[dsel], sc.h.dslot[dsel], stage, &bars[s], sc.h.meta[s]);
            dsel ^= 1;
            if (nx + G < a.n_items) prefetch_desc<D>(a, nx + G, sc.h.dring, sc.h.dslot, dsel);
        };
        bool abort;
        if (!valid) {
            abort = __syncthreads_or(!ok);
            if (!abort) rel();
        } else {
            // the descriptor's width byte is 16 for a head with FP16 rows, else 0
            abort = sc.h.meta[s][kMetaWidth] == kPivotBits
                        ? item_rows<KIND, S16, true>(a, stage, rec_g, row, codes_bytes, sc, tid, ok, rel)
                        : item_rows<KIND, S16, false>(a, stage, rec_g, row, codes_bytes, sc, tid, ok, rel);
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
// Pack fp32 states (S_0) and unpack records of per-row units: one CTA per head.
// ---------------------------------------------------------------------------
template <int S16>
__global__ void __launch_bounds__(NT) k_requant_rows(Args a) {
    __shared__ ScratchR sc;
    const int tid = threadIdx.x;
    const int g = band_of(tid), cb = cblk_of(tid), i0 = g * RT, j0 = 4 * cb;
    int n, ll, h, gl, row;
    item_coords<D>(a, blockIdx.x, n, ll, h, gl, row);
    const int slot = a.slots[n];
    if (slot < 0 || slot >= a.n_slots) {
        if (tid == 0) flag_error(a.err, kErrBadSlot);
        return;
    }
    uint8_t *rec = a.pool + (uint64_t)slot * a.slot_bytes + a.t.rec_off[gl];
    if (tid < D) {
        sc.h.rho[tid] = a.t.rho[(size_t)gl * D + tid];
        sc.h.wbar[tid] = a.t.wbar[(size_t)gl * D + tid];
    }
    const uint4 wv = *reinterpret_cast<const uint4 *>(a.t.row_width + (size_t)gl * D + i0);
    const float *Sg = a.S_in + (size_t)row * D * D;
    float2 S[NP][4];
#pragma unroll
    for (int k = 0; k < NP; ++k) {
        const float4 x = *reinterpret_cast<const float4 *>(Sg + (size_t)(i0 + 2 * k) * D + j0);
        const float4 y = *reinterpret_cast<const float4 *>(Sg + (size_t)(i0 + 2 * k + 1) * D + j0);
        S[k][0] = make_float2(x.x, y.x);
        S[k][1] = make_float2(x.y, y.y);
        S[k][2] = make_float2(x.z, y.z);
        S[k][3] = make_float2(x.w, y.w);
        const uint32_t ba = wid(wv, 2 * k), bb = wid(wv, 2 * k + 1);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            if (ba == (uint32_t)kPivotBits) S[k][c].x = __uint_as_float((uint32_t)__half_as_ushort(__float2half_rn(S[k][c].x)));
            if (bb == (uint32_t)kPivotBits) S[k][c].y = __uint_as_float((uint32_t)__half_as_ushort(__float2half_rn(S[k][c].y)));
        }
    }
    row_partials<D, kQuantDualAxis>(S, sc.h, g, cb);
    __syncthreads();
    const uint32_t codes_bytes = a.t.codes_bytes[gl];
    uint8_t *rec_r = rec + codes_bytes;
    row_phase_rows<S16>(sc, tid, sc.h.rho, sc.h.wbar, a.t.row_width + (size_t)gl * D, a.t.row_off + (size_t)gl * D, rec_r);
    fit_pack_rows<S16, true>(S, sc, tid, rec, rec_r + D * (S16 ? 2 : 4));
}

__global__ void __launch_bounds__(NT) k_unpack_rows(Args a) {
    const int tid = threadIdx.x;
    const int g = band_of(tid), cb = cblk_of(tid), i0 = g * RT, j0 = 4 * cb;
    int n, ll, h, gl, row;
    item_coords<D>(a, blockIdx.x, n, ll, h, gl, row);
    const int slot = a.slots[n];
    if (slot < 0 || slot >= a.n_slots) {
        if (tid == 0) flag_error(a.err, kErrBadSlot);
        return;
    }
    const uint8_t *rec = a.pool + (uint64_t)slot * a.slot_bytes + a.t.rec_off[gl];
    float *out = a.S_out + (size_t)row * D * D;
    const int s16 = a.scale16;
    const uint8_t *rr = rec + a.t.codes_bytes[gl];
    const uint8_t *cc = rr + D * (s16 ? 2 : 4);
    const uint4 wv = *reinterpret_cast<const uint4 *>(a.t.row_width + (size_t)gl * D + i0);
    const uint8_t *tile0 = rec + tile_byte0(a.t.row_off[(size_t)gl * D + i0], g, cb);
    const float4 c4 = scale4_at(cc, j0, s16);
    const float2 cd[4] = {make_float2(c4.x, c4.x), make_float2(c4.y, c4.y), make_float2(c4.z, c4.z),
                          make_float2(c4.w, c4.w)};
    uint32_t P = 0;
#pragma unroll
    for (int k = 0; k < NP; ++k) {
        const int i = i0 + 2 * k;
        const uint32_t ba = wid(wv, 2 * k), bb = wid(wv, 2 * k + 1);
        float2 z[4], x[4];
        unpack_pair_rows(tile0, P, ba, bb, z);
        const float2 r2 = scale2_at(rr, i, s16);
#pragma unroll
        for (int c = 0; c < 4; ++c) x[c] = mul2(mul2(r2, cd[c]), z[c]);
        if (ba == (uint32_t)kPivotBits || bb == (uint32_t)kPivotBits) {
            float hv[4];
            if (ba == (uint32_t)kPivotBits) {
                halves4(tile0, P, hv);
#pragma unroll
                for (int c = 0; c < 4; ++c) x[c].x = hv[c];
            }
            if (bb == (uint32_t)kPivotBits) {
                halves4(tile0, P + 4u * ba, hv);
#pragma unroll
                for (int c = 0; c < 4; ++c) x[c].y = hv[c];
            }
        }
        *reinterpret_cast<float4 *>(out + (size_t)i * D + j0) = make_float4(x[0].x, x[1].x, x[2].x, x[3].x);
        *reinterpret_cast<float4 *>(out + (size_t)(i + 1) * D + j0) = make_float4(x[0].y, x[1].y, x[2].y, x[3].y);
        P += 4u * (ba + bb);
    }
}

}  // namespace kda

// ---------------------------------------------------------------------------
// Host-side launchers (called by the C ABI in stepq_api.cu).  Per-head units
// run the kernels of stepq_head.cu.
// ---------------------------------------------------------------------------
cudaError_t launch_step_head(int kind, int D, const Args &a, int n_sms, cudaStream_t st, int *grid);
cudaError_t launch_pack_head(int D, const Args &a, bool unpack, cudaStream_t st);
size_t step_smem_head_bytes(int D, uint32_t stage_bytes);

template <int KIND>
static cudaError_t launch_rows_kind(const Args &a, int n_sms, cudaStream_t st, int *grid_out) {
    const size_t smem = (size_t)kStages * a.stage_bytes + 64 + sizeof(kda::ScratchR);
    auto kern = a.scale16 ? kda::k_step_rows<KIND, 1> : kda::k_step_rows<KIND, 0>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kda::NT, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    int grid = n_sms * per_sm;
    if (grid > a.n_items) grid = a.n_items;
    if (grid_out) *grid_out = grid;
    if (grid <= 0) return cudaSuccess;
    kern<<<grid, kda::NT, smem, st>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_step(int kind, int D, const Args &a, int n_sms, cudaStream_t st, int *grid) {
    if (a.mode == 0) return launch_step_head(kind, D, a, n_sms, st, grid);
    if (D != kda::D) return cudaErrorInvalidValue;
    switch (kind) {
        case kDecode: return launch_rows_kind<kDecode>(a, n_sms, st, grid);
        case kFitPack: return launch_rows_kind<kFitPack>(a, n_sms, st, grid);
        case kFused: return launch_rows_kind<kFused>(a, n_sms, st, grid);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_pack(int D, const Args &a, bool unpack, cudaStream_t st) {
    if (a.mode == 0) return launch_pack_head(D, a, unpack, st);
    if (D != kda::D) return cudaErrorInvalidValue;
    if (a.n_items <= 0) return cudaSuccess;
    if (unpack) {
        kda::k_unpack_rows<<<a.n_items, kda::NT, 0, st>>>(a);
    } else if (a.scale16) {
        kda::k_requant_rows<1><<<a.n_items, kda::NT, 0, st>>>(a);
    } else {
        kda::k_requant_rows<0><<<a.n_items, kda::NT, 0, st>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace stepq
