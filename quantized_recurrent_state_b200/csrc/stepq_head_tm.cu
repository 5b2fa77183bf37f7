// Fused packed-state decode step of per-head units (GDN, plan mode 0) with
// the fp32 state tile held in tensor memory, d = 128.
//
// STEPQuant paper digest (vibe-research), 方法-4: reconstruct the state tile
// from codes, row/column scales and FP16 pivots; retention, delta update and
// readout; refit (方法-3); pack and write back before the next read.
// Arithmetic definitions: include/stepq.h.
//
// Same mapping, arithmetic and order of operations as k_step_head (thread t
// owns tile t: rows [16 g, 16 g + 16) x columns [4 cb, 4 cb + 4), g = band_of(t),
// cb = cblk_of(t); warps hold whole value columns), but the 64 state values of a
// thread live in its own tensor-memory lane between the passes, 16 at a time
// in registers.  That frees the registers the state would hold, so three
// CTAs (24 warps) share an SM instead of two and the column reductions and
// block barriers of one record overlap the arithmetic of the others.
//
// Tensor-memory map (128 columns per CTA): warp w reads and writes lane
// 32 (w % 4) + laneid, columns [64 (w / 4), 64 (w / 4) + 64); chunk m (row
// pairs 2m and 2m + 1 of the tile) is columns 16 m .. 16 m + 15, entry
// (k - 2m) 8 + 2c + {0, 1} holding rows (2k, 2k + 1) of column c.
#include "stepq_head.cuh"
#include "stepq_tc.cuh"

namespace stepq {
namespace tm {

constexpr int D = 128, NT = 256, RT = 16;

#define STEPQ_TM_R16 "=f"(v[0].x), "=f"(v[0].y), "=f"(v[1].x), "=f"(v[1].y), "=f"(v[2].x), "=f"(v[2].y), "=f"(v[3].x), \
    "=f"(v[3].y), "=f"(v[4].x), "=f"(v[4].y), "=f"(v[5].x), "=f"(v[5].y), "=f"(v[6].x), "=f"(v[6].y), "=f"(v[7].x), "=f"(v[7].y)
#define STEPQ_TM_W16 "f"(v[0].x), "f"(v[0].y), "f"(v[1].x), "f"(v[1].y), "f"(v[2].x), "f"(v[2].y), "f"(v[3].x), \
    "f"(v[3].y), "f"(v[4].x), "f"(v[4].y), "f"(v[5].x), "f"(v[5].y), "f"(v[6].x), "f"(v[6].y), "f"(v[7].x), "f"(v[7].y)

// 16 consecutive columns of this thread's lane (one chunk); the values are
// usable after wait_ld().
__device__ __forceinline__ void ld16(uint32_t taddr, float2 (&v)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
                 : STEPQ_TM_R16
                 : "r"(taddr)
                 : "memory");
}
__device__ __forceinline__ void wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void st16(uint32_t taddr, const float2 (&v)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
                 ::"r"(taddr), STEPQ_TM_W16
                 : "memory");
}
__device__ __forceinline__ void wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

#undef STEPQ_TM_R16
#undef STEPQ_TM_W16

// Byte offset of stream word w of tile t in the codes block (RT = 16: 16-byte chunks).
__device__ __forceinline__ uint32_t word_off(int t, int w) { return (uint32_t)((((w >> 2) * NT + t) << 4) + ((w & 3) << 2)); }

// The B/2 stream words of chunk m (row pairs 2m, 2m + 1) of tile t.
template <int B>
__device__ __forceinline__ void load_words(const uint8_t *blk, int t, int m, uint32_t (&w)[B / 2]) {
    if constexpr (B == 8) {
        const uint4 v = *reinterpret_cast<const uint4 *>(blk + word_off(t, 4 * m));
        w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else if constexpr (B == 4) {
        const uint2 v = *reinterpret_cast<const uint2 *>(blk + word_off(t, 2 * m));
        w[0] = v.x; w[1] = v.y;
    } else if constexpr (B == 2) {
        w[0] = *reinterpret_cast<const uint32_t *>(blk + word_off(t, m));
    } else {
#pragma unroll
        for (int i = 0; i < 3; ++i) w[i] = *reinterpret_cast<const uint32_t *>(blk + word_off(t, 3 * m + i));
    }
}

template <int B>
__device__ __forceinline__ void store_words(uint8_t *blk, int t, int m, const uint32_t (&w)[B / 2]) {
    if constexpr (B == 8) {
        *reinterpret_cast<uint4 *>(blk + word_off(t, 4 * m)) = make_uint4(w[0], w[1], w[2], w[3]);
    } else if constexpr (B == 4) {
        *reinterpret_cast<uint2 *>(blk + word_off(t, 2 * m)) = make_uint2(w[0], w[1]);
    } else if constexpr (B == 2) {
        *reinterpret_cast<uint32_t *>(blk + word_off(t, m)) = w[0];
    } else {
#pragma unroll
        for (int i = 0; i < 3; ++i) *reinterpret_cast<uint32_t *>(blk + word_off(t, 3 * m + i)) = w[i];
    }
}

// z of row pair 2m + tt of a chunk (the chunk's words in w).
template <int B, int TT>
__device__ __forceinline__ void unpack_chunk(const uint32_t (&w)[B / 2], float2 (&z)[4]) {
    constexpr int OFF = 1 << (B - 1);
    if constexpr (B == 4) {
        const uint32_t lo = w[TT], hi = w[TT] >> 16;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const uint32_t m = 0xFu << (4 * c);
            z[c] = zpair((lo & m) | mbits(4 * c), (hi & m) | mbits(4 * c), -mval(4 * c, OFF));
        }
    } else if constexpr (B == 8) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
            z[c] = zpair(__byte_perm(w[2 * TT], 0x4B000000u, 0x7540u | c), __byte_perm(w[2 * TT + 1], 0x4B000000u, 0x7540u | c),
                         -mval(0, OFF));
    } else if constexpr (B == 2) {
        const uint32_t x = TT ? (w[0] >> 16) : w[0];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int pa = 2 * c, pb = 8 + 2 * c;
            z[c] = add2(make_float2(__uint_as_float((x & (3u << pa)) | mbits(pa)), __uint_as_float((x & (3u << pb)) | mbits(pb))),
                        make_float2(-mval(pa, OFF), -mval(pb, OFF)));
        }
    } else {
        uint32_t Ra, Rb;
        if (TT == 0) {
            Ra = w[0];
            Rb = w[1];
        } else {
            Ra = __byte_perm(__byte_perm(w[0], w[1], 0x0073u), w[2], 0x0710u);
            Rb = w[2];
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

// Stream words of a chunk from T = fma(y, 1/c, kMagic + 2^(b-1)) of its two row
// pairs (see clamp_pair16 / clamp1 for the field values).
template <int B>
__device__ __forceinline__ void pack_chunk(const float2 (&T)[8], uint32_t (&w)[B / 2]) {
    if constexpr (B == 4) {
#pragma unroll
        for (int tt = 0; tt < 2; ++tt) {
            uint32_t x = 0x11111111u;
#pragma unroll
            for (int c = 0; c < 4; ++c) x += clamp_pair16<4>(T[4 * tt + c]) << (4 * c);
            w[tt] = x;
        }
    } else if constexpr (B == 8) {
#pragma unroll
        for (int tt = 0; tt < 2; ++tt) {
            uint32_t v[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) v[c] = clamp_pair16<8>(T[4 * tt + c]);
            const uint32_t t01 = __byte_perm(v[0], v[1], 0x6240u), t23 = __byte_perm(v[2], v[3], 0x6240u);
            w[2 * tt] = __byte_perm(t01, t23, 0x5410u) + 0x01010101u;
            w[2 * tt + 1] = __byte_perm(t01, t23, 0x7632u) + 0x01010101u;
        }
    } else if constexpr (B == 2) {
        uint32_t x = 0x55555555u;
#pragma unroll
        for (int tt = 0; tt < 2; ++tt)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                x += clamp1<2>(T[4 * tt + c].x) << (16 * tt + 2 * c);
                x += clamp1<2>(T[4 * tt + c].y) << (16 * tt + 8 + 2 * c);
            }
        w[0] = x;
    } else {
        uint32_t R[4];
#pragma unroll
        for (int tt = 0; tt < 2; ++tt) {
            uint32_t Ra = 0x41041u, Rb = 0x41041u;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                Ra += clamp1<6>(T[4 * tt + c].x) << (6 * c);
                Rb += clamp1<6>(T[4 * tt + c].y) << (6 * c);
            }
            R[2 * tt] = Ra;
            R[2 * tt + 1] = Rb;
        }
        // rows 0, 1, 3 of the group keep their value, row 2 (R[2]) gives the top bytes
        w[0] = __byte_perm(R[0], R[2], 0x4210u);
        w[1] = __byte_perm(R[1], R[2], 0x5210u);
        w[2] = __byte_perm(R[3], R[2], 0x6210u);
    }
}

// Four consecutive rows of a scale array (fp32 or bfloat16) as two row pairs.
__device__ __forceinline__ void scale_pairs4(const uint8_t *base, int i, int s16, float2 &p0, float2 &p1) {
    if (s16) {
        const uint2 v = *reinterpret_cast<const uint2 *>(base + 2 * i);
        p0 = make_float2(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u));
        p1 = make_float2(__uint_as_float(v.y << 16), __uint_as_float(v.y & 0xffff0000u));
    } else {
        const float4 v = *reinterpret_cast<const float4 *>(base + 4 * i);
        p0 = make_float2(v.x, v.y);
        p1 = make_float2(v.z, v.w);
    }
}
__device__ __forceinline__ void pairs4(const float *p, float2 &p0, float2 &p1) {
    const float4 v = *reinterpret_cast<const float4 *>(p);
    p0 = make_float2(v.x, v.y);
    p1 = make_float2(v.z, v.w);
}

// One quantized head of width B, fused.  tb: this thread's tensor-memory
// address (lane quadrant and column base folded in).
template <int B, int S16, int QUANT, class Rel>
__device__ bool item(const Args &a, const uint8_t *stage, uint8_t *rec_g, int row, ScratchH<D> &sc, int tid, bool ok,
                     Rel &rel, uint32_t tb) {
    constexpr int OFF = 1 << (B - 1), Q = OFF - 1;
    constexpr float IQ = 1.0f / (float)Q;
    const int g = band_of(tid), cb = cblk_of(tid), lane = tid & 31, i0 = g * RT, j0 = 4 * cb;
    const uint32_t codes_bytes = (uint32_t)D * D * B / 8;
    const uint8_t *st_r = stage + codes_bytes;
    const uint8_t *st_c = st_r + D * (S16 ? 2 : 4);
    const float *tf = stage_tail<D>(a, stage);
    const float *qs = tf + kTailQ * D, *ks = tf + kTailK * D, *vs = tf + kTailV * D;
    const float *ab = stage_ab<D>(a, stage);
    const float2 al2 = make_float2(ab[0], ab[0]);

    // reconstruct S' = fl(fl(a_i c_j) z) into tensor memory; u chains
    float2 cd[4];
    {
        const float4 c4 = scale4_at(st_c, j0, S16);
        cd[0] = make_float2(c4.x, c4.x);
        cd[1] = make_float2(c4.y, c4.y);
        cd[2] = make_float2(c4.z, c4.z);
        cd[3] = make_float2(c4.w, c4.w);
    }
    float2 acc[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[c] = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const int i = i0 + 4 * m;
        uint32_t w[B / 2];
        load_words<B>(stage, tid, m, w);
        float2 r0, r1, k0, k1;
        scale_pairs4(st_r, i, S16, r0, r1);
        pairs4(ks + i, k0, k1);
        float2 v[8], z[4];
        const float2 a0 = mul2(r0, al2), a1 = mul2(r1, al2);
        unpack_chunk<B, 0>(w, z);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            v[c] = mul2(mul2(a0, cd[c]), z[c]);
            acc[c] = fma2(k0, v[c], acc[c]);
        }
        unpack_chunk<B, 1>(w, z);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            v[4 + c] = mul2(mul2(a1, cd[c]), z[c]);
            acc[c] = fma2(k1, v[4 + c], acc[c]);
        }
        st16(tb + 16 * m, v);
    }
    // w of the four columns
    const int cs = col4_of(g);
    float2 wd[4];
    {
        const float u = band_sum4(acc[0].x + acc[0].y, acc[1].x + acc[1].y, acc[2].x + acc[2].y, acc[3].x + acc[3].y, g);
        const float wm = __fmul_rn(ab[1], __fsub_rn(vs[j0 + cs], u));
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const float t = __shfl_sync(kFull, wm, col4_src(lane, c));
            wd[c] = make_float2(t, t);
        }
    }
    wait_st();
    // S = fma(k, w, S'); o chains; row partials
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[c] = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const int i = i0 + 4 * m;
        float2 v[8], k0, k1, q0, q1;
        ld16(tb + 16 * m, v);
        pairs4(ks + i, k0, k1);
        pairs4(qs + i, q0, q1);
        wait_ld();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            v[c] = fma2(k0, wd[c], v[c]);
            acc[c] = fma2(q0, v[c], acc[c]);
            v[4 + c] = fma2(k1, wd[c], v[4 + c]);
            acc[c] = fma2(q1, v[4 + c], acc[c]);
        }
        float4 rs;
        if (QUANT == kQuantAbsmax) {
            rs.x = fmaxf(fmaxf(fabsf(v[0].x), fabsf(v[1].x)), fmaxf(fabsf(v[2].x), fabsf(v[3].x)));
            rs.y = fmaxf(fmaxf(fabsf(v[0].y), fabsf(v[1].y)), fmaxf(fabsf(v[2].y), fabsf(v[3].y)));
            rs.z = fmaxf(fmaxf(fabsf(v[4].x), fabsf(v[5].x)), fmaxf(fabsf(v[6].x), fabsf(v[7].x)));
            rs.w = fmaxf(fmaxf(fabsf(v[4].y), fabsf(v[5].y)), fmaxf(fabsf(v[6].y), fabsf(v[7].y)));
        } else {
            rs.x = (fabsf(v[0].x) + fabsf(v[1].x)) + (fabsf(v[2].x) + fabsf(v[3].x));
            rs.y = (fabsf(v[0].y) + fabsf(v[1].y)) + (fabsf(v[2].y) + fabsf(v[3].y));
            rs.z = (fabsf(v[4].x) + fabsf(v[5].x)) + (fabsf(v[6].x) + fabsf(v[7].x));
            rs.w = (fabsf(v[4].y) + fabsf(v[5].y)) + (fabsf(v[6].y) + fabsf(v[7].y));
        }
        *reinterpret_cast<float4 *>(&sc.part[pidx<D>(cb, i)]) = rs;
        st16(tb + 16 * m, v);
    }
    const float o_mine =
        band_sum4(acc[0].x + acc[0].y, acc[1].x + acc[1].y, acc[2].x + acc[2].y, acc[3].x + acc[3].y, g);
    wait_st();
    if (__syncthreads_or(!ok)) return true;
    if ((g & 4) == 0) a.o[(size_t)row * D + j0 + cs] = o_mine;
    uint8_t *rec_r = rec_g + codes_bytes;
    uint8_t *rec_c = rec_r + D * (S16 ? 2 : 4);
    row_phase<D, B, S16, QUANT>(sc, tid, tf + kTailRho * D, tf + kTailWbar * D, rec_r);
    rel();
    const float2 mg2 = make_float2(kMagic + (float)OFF, kMagic + (float)OFF);
    if (QUANT == kQuantAbsmax) {
        if (tid < D) scale_put(rec_c, tid, 1.0f, S16);
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const int i = i0 + 4 * m;
            float2 v[8], ir0, ir1;
            ld16(tb + 16 * m, v);
            pairs4(&sc.rinv[i], ir0, ir1);
            wait_ld();
            float2 T[8];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                T[c] = fma2(v[c], ir0, mg2);
                T[4 + c] = fma2(v[4 + c], ir1, mg2);
            }
            uint32_t w[B / 2];
            pack_chunk<B>(T, w);
            store_words<B>(rec_g, tid, m, w);
        }
        return false;
    }
    // y = fl(S fl(1/r)) into tensor memory; column maxima
    float mx4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const int i = i0 + 4 * m;
        float2 v[8], ir0, ir1;
        ld16(tb + 16 * m, v);
        pairs4(&sc.rinv[i], ir0, ir1);
        wait_ld();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            v[c] = mul2(v[c], ir0);
            v[4 + c] = mul2(v[4 + c], ir1);
            mx4[c] = max3abs(mx4[c], v[c].x, v[c].y);
            mx4[c] = max3abs(mx4[c], v[4 + c].x, v[4 + c].y);
        }
        st16(tb + 16 * m, v);
    }
    const float mx = band_max4(mx4[0], mx4[1], mx4[2], mx4[3], g);
    const float c0 = (mx == 0.0f) ? 1.0f : __fmul_rn(mx, IQ);
    float2 icd[4];
    {
        const float ic0 = __frcp_rn(c0);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const float t = __shfl_sync(kFull, ic0, col4_src(lane, c));
            icd[c] = make_float2(t, t);
        }
    }
    wait_st();
    // z0 = rint(y fl(1/c0)); t = fl(b z0); N = sum t y, D = sum t z0 (band order)
    const float2 mg = make_float2(kMagic, kMagic), nmg = make_float2(-kMagic, -kMagic);
    float2 na[4], da[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) na[c] = da[c] = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const int i = i0 + 4 * m;
        float2 v[8], b0, b1;
        ld16(tb + 16 * m, v);
        pairs4(&sc.bw[i], b0, b1);
        wait_ld();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            float2 z0 = add2(fma2(v[c], icd[c], mg), nmg);
            float2 t = mul2(b0, z0);
            na[c] = fma2(t, v[c], na[c]);
            da[c] = fma2(t, z0, da[c]);
            z0 = add2(fma2(v[4 + c], icd[c], mg), nmg);
            t = mul2(b1, z0);
            na[c] = fma2(t, v[4 + c], na[c]);
            da[c] = fma2(t, z0, da[c]);
        }
    }
    {
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
        if ((g & 1) == 0) scale_put(rec_c, j0 + c8, cj, S16);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const float t = __shfl_sync(kFull, icj, col8_src(lane, c));
            icd[c] = make_float2(t, t);
        }
    }
    // final codes, packed and written chunk by chunk
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        float2 v[8];
        ld16(tb + 16 * m, v);
        wait_ld();
        float2 T[8];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            T[c] = fma2(v[c], icd[c], mg2);
            T[4 + c] = fma2(v[4 + c], icd[c], mg2);
        }
        uint32_t w[B / 2];
        pack_chunk<B>(T, w);
        store_words<B>(rec_g, tid, m, w);
    }
    return false;
}

// One FP16 pivot head (binary16 tile, row-major, in place).
template <class Rel>
__device__ bool item_pivot(const Args &a, const uint8_t *stage, uint8_t *rec_g, int row, int tid, bool ok, Rel &rel,
                           uint32_t tb) {
    const int g = band_of(tid), lane = tid & 31, i0 = g * RT, j0 = 4 * cblk_of(tid);
    const float *tf = stage_tail<D>(a, stage);
    const float *qs = tf + kTailQ * D, *ks = tf + kTailK * D, *vs = tf + kTailV * D;
    const float *ab = stage_ab<D>(a, stage);
    const float2 al2 = make_float2(ab[0], ab[0]);
    float2 acc[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[c] = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        float2 v[8];
#pragma unroll
        for (int tt = 0; tt < 2; ++tt) {
            const int i = i0 + 4 * m + 2 * tt;
            const uint2 ha = *reinterpret_cast<const uint2 *>(rec_g + ((size_t)i * D + j0) * 2);
            const uint2 hb = *reinterpret_cast<const uint2 *>(rec_g + ((size_t)(i + 1) * D + j0) * 2);
            const float2 a01 = __half22float2(*reinterpret_cast<const __half2 *>(&ha.x));
            const float2 a23 = __half22float2(*reinterpret_cast<const __half2 *>(&ha.y));
            const float2 b01 = __half22float2(*reinterpret_cast<const __half2 *>(&hb.x));
            const float2 b23 = __half22float2(*reinterpret_cast<const __half2 *>(&hb.y));
            v[4 * tt + 0] = mul2(al2, make_float2(a01.x, b01.x));
            v[4 * tt + 1] = mul2(al2, make_float2(a01.y, b01.y));
            v[4 * tt + 2] = mul2(al2, make_float2(a23.x, b23.x));
            v[4 * tt + 3] = mul2(al2, make_float2(a23.y, b23.y));
            const float2 k2 = *reinterpret_cast<const float2 *>(ks + i);
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[c] = fma2(k2, v[4 * tt + c], acc[c]);
        }
        st16(tb + 16 * m, v);
    }
    const int cs = col4_of(g);
    float2 wd[4];
    {
        const float u = band_sum4(acc[0].x + acc[0].y, acc[1].x + acc[1].y, acc[2].x + acc[2].y, acc[3].x + acc[3].y, g);
        const float wm = __fmul_rn(ab[1], __fsub_rn(vs[j0 + cs], u));
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const float t = __shfl_sync(kFull, wm, col4_src(lane, c));
            wd[c] = make_float2(t, t);
        }
    }
    wait_st();
    if (__syncthreads_or(!ok)) return true;
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[c] = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        float2 v[8];
        ld16(tb + 16 * m, v);
        wait_ld();
#pragma unroll
        for (int tt = 0; tt < 2; ++tt) {
            const int i = i0 + 4 * m + 2 * tt;
            const float2 k2 = *reinterpret_cast<const float2 *>(ks + i);
            const float2 q2 = *reinterpret_cast<const float2 *>(qs + i);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                v[4 * tt + c] = fma2(k2, wd[c], v[4 * tt + c]);
                acc[c] = fma2(q2, v[4 * tt + c], acc[c]);
            }
            const float2 *s = &v[4 * tt];
            const __half2 a01 = __floats2half2_rn(s[0].x, s[1].x), a23 = __floats2half2_rn(s[2].x, s[3].x);
            const __half2 b01 = __floats2half2_rn(s[0].y, s[1].y), b23 = __floats2half2_rn(s[2].y, s[3].y);
            *reinterpret_cast<uint2 *>(rec_g + ((size_t)i * D + j0) * 2) =
                make_uint2(*reinterpret_cast<const uint32_t *>(&a01), *reinterpret_cast<const uint32_t *>(&a23));
            *reinterpret_cast<uint2 *>(rec_g + ((size_t)(i + 1) * D + j0) * 2) =
                make_uint2(*reinterpret_cast<const uint32_t *>(&b01), *reinterpret_cast<const uint32_t *>(&b23));
        }
    }
    const float o_mine =
        band_sum4(acc[0].x + acc[0].y, acc[1].x + acc[1].y, acc[2].x + acc[2].y, acc[3].x + acc[3].y, g);
    __syncthreads();  // every thread is past its reads of the stage
    rel();
    if ((g & 4) == 0) a.o[(size_t)row * D + j0 + cs] = o_mine;
    return false;
}

constexpr uint32_t kCols = 128;  // tensor-memory columns per CTA

struct __align__(16) Extra {
    uint32_t taddr;
};

template <int S16, int QUANT>
__global__ void __launch_bounds__(NT, 3) k_step_tm(Args a) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5;
    const int G = gridDim.x;
    uint8_t *stages = smem;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kStages * a.stage_bytes);
    Extra &ex = *reinterpret_cast<Extra *>(smem + kStages * a.stage_bytes + 32);
    ScratchH<D> &sc = *reinterpret_cast<ScratchH<D> *>(smem + kStages * a.stage_bytes + 64);

    if (warp == 0) tc::alloc(&ex.taddr, kCols);
    int dsel = 0;
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(&bars[s], 1);
        fence_mbar_init();
        for (int s = 0; s < kStages; ++s) {
            const int it = blockIdx.x + s * G;
            if (it >= a.n_items) break;
            int n, ll, di;
            step_coords<D>(a, it, n, ll, di);
            issue_item<D, kFused, 0>(a, it, a.t.desc[di], a.slots[n], stages + s * a.stage_bytes, &bars[s], sc.meta[s]);
        }
        const int nx = blockIdx.x + kStages * G;
        if (nx < a.n_items) prefetch_desc<D>(a, nx, sc.dring, sc.dslot, 0);
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tb = ex.taddr + ((uint32_t)(32 * (warp & 3)) << 16) + 64u * (uint32_t)(warp >> 2);
    int s = 0;
    uint32_t phase = 0;
    bool abort = false;
    for (int it = blockIdx.x; it < a.n_items && !abort; it += G) {
        const bool ok = mbar_wait_bounded(&bars[s], phase, a.wait_polls);
        const int width = sc.meta[s][kMetaWidth];
        const int valid = sc.meta[s][kMetaValid];
        const int row = sc.meta[s][kMetaRow];
        uint8_t *rec_g = reinterpret_cast<uint8_t *>((uintptr_t)(uint32_t)sc.meta[s][kMetaRecLo] |
                                                     ((uintptr_t)(uint32_t)sc.meta[s][kMetaRecHi] << 32));
        uint8_t *stage = stages + s * a.stage_bytes;
        auto rel = [&]() {
            if (tid != 0) return;
            const int nx = it + kStages * G;
            if (nx >= a.n_items) return;
            cp_async_wait_all();
            issue_item<D, kFused, 0>(a, nx, sc.dring[dsel], sc.dslot[dsel], stage, &bars[s], sc.meta[s]);
            dsel ^= 1;
            if (nx + G < a.n_items) prefetch_desc<D>(a, nx + G, sc.dring, sc.dslot, dsel);
        };
        if (!valid) {
            abort = __syncthreads_or(!ok);
            if (!abort) rel();
        } else {
            switch (width) {
                case 2: abort = item<2, S16, QUANT>(a, stage, rec_g, row, sc, tid, ok, rel, tb); break;
                case 4: abort = item<4, S16, QUANT>(a, stage, rec_g, row, sc, tid, ok, rel, tb); break;
                case 6: abort = item<6, S16, QUANT>(a, stage, rec_g, row, sc, tid, ok, rel, tb); break;
                case 8: abort = item<8, S16, QUANT>(a, stage, rec_g, row, sc, tid, ok, rel, tb); break;
                case kPivotBits: abort = item_pivot(a, stage, rec_g, row, tid, ok, rel, tb); break;
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
        } else if (++s == kStages) {
            s = 0;
            phase ^= 1u;
        }
    }
    // every thread's tensor-memory accesses are complete (waited) before the columns go back
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    if (warp == 0) tc::dealloc(ex.taddr, kCols);
}

}  // namespace tm

size_t step_smem_tm(uint32_t stage_bytes) { return (size_t)kStages * stage_bytes + 64 + sizeof(ScratchH<tm::D>); }

template <int S16, int QUANT>
static cudaError_t launch_tm_k(const Args &a, int n_sms, cudaStream_t st, int *grid_out) {
    const size_t smem = step_smem_tm(a.stage_bytes);
    auto kern = tm::k_step_tm<S16, QUANT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    // Three CTAs per SM: the kernel's register bound (80 per thread) and its shared memory
    // allow three, and three hold 384 of the SM's 512 tensor-memory columns.  (The
    // occupancy calculator reports one CTA per SM for this kernel.)
    int per_sm = 3;
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return e;
    if (fa.numRegs * tm::NT * per_sm > 65536 || (smem + 1024) * per_sm > 232448) per_sm = 2;
    int grid = n_sms * per_sm;
    if (grid > a.n_items) grid = a.n_items;
    if (grid_out) *grid_out = grid;
    if (grid <= 0) return cudaSuccess;
    kern<<<grid, tm::NT, smem, st>>>(a);
    return cudaGetLastError();
}

// The fused step with the state in tensor memory (d = 128 per-head units).
cudaError_t launch_step_tm(const Args &a, int n_sms, cudaStream_t st, int *grid) {
    if (a.scale16)
        return a.quantizer == kQuantAbsmax ? launch_tm_k<1, kQuantAbsmax>(a, n_sms, st, grid)
                                           : launch_tm_k<1, kQuantDualAxis>(a, n_sms, st, grid);
    return a.quantizer == kQuantAbsmax ? launch_tm_k<0, kQuantAbsmax>(a, n_sms, st, grid)
                                       : launch_tm_k<0, kQuantDualAxis>(a, n_sms, st, grid);
}

}  // namespace stepq
