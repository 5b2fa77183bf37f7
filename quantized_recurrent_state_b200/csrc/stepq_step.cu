// Packed-state decode step kernels for per-head units (GDN, mode 0).
//
// STEPQuant paper digest (vibe-research), 方法-4: reconstruct the state tile
// from integer codes, row/column scales and FP16 pivots; retention, delta
// update and readout on the floating-point tile; the readout goes on at once;
// refit the row/column factors; pack codes and scales; write back before the
// next read.  Arithmetic definitions: include/stepq.h.
//
// One CTA of NT = 2D threads handles one (request, layer, head) record at a
// time.  Thread t owns rows [g RT, g RT + RT) x columns [4l, 4l + 4) with
// RT = D/8, g = t / (D/4), l = t % (D/4); the packed layout stores thread t's
// codes as its own bit stream, so its chunks come straight out of a 16-byte
// shared-memory load.  Persistent CTAs stream records through a ring of
// shared-memory stages filled by 1-D bulk copies (cp.async.bulk, completion
// on an mbarrier).  Kernels:
//   kDecode   reconstruct -> u, w -> o (readout) ; writes o and w
//   kFitPack  reconstruct -> S_t = S' + k w^T -> refit r, c -> pack, in place
//   kFused    both in one pass over the record
#include <cstddef>

#include "stepq_dev.cuh"

namespace stepq {

enum Kind { kDecode = 0, kFitPack = 1, kFused = 2 };

constexpr int kStages = 2;  // one item in flight while the other is worked on
constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23: fl(x + kMagic) - kMagic = rint(x), |x| < 2^22

template <int D>
struct Geo {
    static constexpr int NT = 2 * D;       // threads per CTA
    static constexpr int RT = D / 8;       // rows per thread
    static constexpr int LANES = D / 4;    // threads across a row band
    static constexpr int BANDS = 8;
};

template <int D, int B>
struct Stream {
    static constexpr int RT = D / 8;
    static constexpr int WORDS = (RT * B + 7) / 8;  // 32-bit words of a thread stream (4 RT B bits)
    static constexpr int NW = WORDS + 1;                                // + guard word
    static constexpr int NCH = B / 2;                                   // chunks of RT bytes
};

// Shared memory besides the stages.  Per-row factors that multiply a pair
// of columns are kept duplicated ((x_i, x_i) pairs), so a 16-byte load gives
// two rows' packed operands without register moves.
template <int D>
struct __align__(16) Scratch {
    static constexpr int RT = D / 8, LANES = D / 4, RS = D / 4 + 4;  // RS: padded row of the transpose
    union {
        struct {
            double pU[8][D];  // per-band column partials of u and o
            double pO[8][D];
        } col;
        float pmax[4][8][D];  // per-row records: column absmax per width class and band
    } u;
    float rsum[8][RT][RS];  // per-thread row partials, transposed for the row reduction
    float pf0[8][D];
    float pf1[8][D];
    float2 a2[D];     // (a_i, a_i), a_i = fl(alpha_i r_i)
    float2 k2[D];     // (k_i, k_i)
    double kap[D];    // k_i a_i 2^-12   (FP16 rows and heads: k_i alpha_i)
    double qt[D];     // q_i a_i 2^-12   (FP16 rows and heads: q_i alpha_i)
    float rho[D];     // (requant and calibration kernels; the step reads them from the stage)
    float wbar[D];
    float2 rinv2[D];  // (fl(1/r_i), fl(1/r_i)) of the refit
    float2 bw2[D];    // (b_i, b_i) of the refit
    float rowr[D];    // r_i of the refit
    float cold[D];    // c_j (old on entry, refitted after fit_scales)
    float wv[D];      // w_j
    float ic0[D];
    float c0[D];
    float ic[D];
    double bandQK[8];  // per band: sum_i q_i k_i
    uint4 dring[2];    // prefetched item descriptors (thread 0)
    int dslot[2];
    int meta[kStages][8];  // slot, width, valid, codes bytes, record address lo, hi
    uint32_t roff[D];  // per-row records (requant kernel): row byte offset in the codes block
    uint8_t rw[D];     // per-row records (requant kernel): row width (16 = FP16 row)
    float nz;          // -0.0f, read at run time (see fit_scales)
};

// Every array read or written with 8- or 16-byte vector accesses starts on a
// 16-byte boundary of the (16-byte aligned) scratch block.
template <int D>
constexpr bool scratch_aligned() {
    using S = Scratch<D>;
    return offsetof(S, u) % 16 == 0 && offsetof(S, rsum) % 16 == 0 && offsetof(S, pf0) % 16 == 0 &&
           offsetof(S, pf1) % 16 == 0 && offsetof(S, a2) % 16 == 0 && offsetof(S, k2) % 16 == 0 &&
           offsetof(S, kap) % 16 == 0 && offsetof(S, qt) % 16 == 0 && offsetof(S, rinv2) % 16 == 0 &&
           offsetof(S, bw2) % 16 == 0 && offsetof(S, cold) % 16 == 0 &&
           offsetof(S, wv) % 16 == 0 && offsetof(S, ic0) % 16 == 0 && offsetof(S, ic) % 16 == 0 &&
           offsetof(S, dring) % 16 == 0 && (sizeof(float) * Scratch<D>::RS) % 16 == 0;
}
static_assert(scratch_aligned<16>() && scratch_aligned<32>() && scratch_aligned<64>() && scratch_aligned<128>(),
              "scratch arrays must stay 16-byte aligned");

template <int D>
__device__ __forceinline__ void item_coords(const Args &a, int it, int &n, int &ll, int &h, int &gl, int &row) {
    const int per_req = a.nL * a.H;
    n = it / per_req;
    const int rem = it - n * per_req;
    ll = rem / a.H;
    h = rem - ll * a.H;
    gl = (a.lb + ll) * a.H + h;
    row = (n * a.nL_in + a.l_in0 + ll) * a.H + h;  // index of the (request, layer, head) input row
}

// Item order of the step kernels: requests fastest, then the layer's heads
// in the order of its descriptor table (sorted by width on the host, so the
// CTAs of an SM run one width's code at a time), then layers.  Returns the
// request n, the layer ll inside the launch and the descriptor index.
template <int D>
__device__ __forceinline__ void step_coords(const Args &a, int it, int &n, int &ll, int &di) {
    const int k = (int)fast_div((uint32_t)it, a.div_nreq);
    n = it - k * a.n_req;
    ll = (int)fast_div((uint32_t)k, a.div_h);
    di = (a.lb + ll) * a.H + (k - ll * a.H);
}

// Thread 0: start the 16-byte descriptor and the slot of item `it` on their
// way into the descriptor ring entry e (cp.async, completion by group).
template <int D>
__device__ __forceinline__ void prefetch_desc(const Args &a, int it, Scratch<D> &sc, int e) {
    int n, ll, di;
    step_coords<D>(a, it, n, ll, di);
    cp_async16(&sc.dring[e], &a.t.desc[di]);
    cp_async4(&sc.dslot[e], &a.slots[n]);
    cp_async_commit();
}

// Thread 0: stage item `it` (descriptor dsc, slot) into `stage`: the record,
// the input rows and the head's tables by bulk copies, the per-item scalars
// by cp.async, all completing on `bar`; or mark the item invalid.
template <int D, int KIND, int MODE>
__device__ void issue_item(const Args &a, int it, uint4 dsc, int slot, uint8_t *stage, uint64_t *bar, int *meta) {
    int n, ll, di;
    step_coords<D>(a, it, n, ll, di);
    const int h = (int)(dsc.y >> 16);
    const int gl = (a.lb + ll) * a.H + h;
    const int row = (n * a.nL_in + a.l_in0 + ll) * a.H + h;  // the (request, layer, head) input row
    const bool ok = slot >= 0 && slot < a.n_slots;
    const uint8_t *rec = a.pool + (uint64_t)slot * a.slot_bytes + ((uint64_t)(dsc.y & 0xffffu) << 32 | dsc.x);
    meta[0] = slot;
    meta[1] = (int)(dsc.w & 0xffu);
    meta[2] = ok ? 1 : 0;
    meta[3] = (int)(dsc.w >> 8);
    meta[4] = (int)(uint32_t)(uintptr_t)rec;
    meta[5] = (int)(uint32_t)((uintptr_t)rec >> 32);
    meta[6] = row;
    if (!ok) {
        flag_error(a.err, kErrBadSlot);
        mbar_arrive(bar);
        return;
    }
    uint8_t *tail = stage + a.rec_stage_bytes;
    float *ab = reinterpret_cast<float *>(tail + 4 * kTailRw * D + D);
    if (MODE == 0) cp_async4(ab, a.alpha + row);
    if (KIND != kFitPack) cp_async4(ab + 1, a.beta + row);
    cp_async_mbar_arrive(bar);  // before the expect-tx arrival, so the phase waits for them
    fence_proxy_async();
    constexpr uint32_t RB = D * 4;
    const uint32_t rec_bytes = dsc.z;
    uint32_t total = rec_bytes + (KIND != kFitPack ? 3 * RB : 2 * RB);
    if (KIND != kDecode) total += 2 * RB;
    if (MODE == 1) total += 2 * RB + D;
    mbar_arrive_expect(bar, total + a.phantom_tx);
    if (rec_bytes) bulk_g2s(stage, rec, rec_bytes, bar);
    const size_t off = (size_t)row * D;
    const size_t goff = (size_t)gl * D;
    float *tf = reinterpret_cast<float *>(tail);
    if (KIND != kFitPack) {
        bulk_g2s(tf + kTailQ * D, a.q + off, RB, bar);
        bulk_g2s(tf + kTailV * D, a.v + off, RB, bar);
    } else {
        bulk_g2s(tf + kTailX * D, a.w + off, RB, bar);
    }
    bulk_g2s(tf + kTailK * D, a.k + off, RB, bar);
    if (KIND != kDecode) {
        bulk_g2s(tf + kTailRho * D, a.t.rho + goff, RB, bar);
        bulk_g2s(tf + kTailWbar * D, a.t.wbar + goff, RB, bar);
    }
    if (MODE == 1) {
        bulk_g2s(tf + kTailAlpha * D, a.alpha + off, RB, bar);
        bulk_g2s(tail + 4 * kTailRw * D, a.t.row_width + goff, D, bar);
        bulk_g2s(tf + kTailRoff * D, a.t.row_off + goff, RB, bar);
    }
}

// Load thread t's code stream (NCH chunks of RT bytes) from the codes block.
template <int D, int B>
__device__ __forceinline__ void load_stream(const uint8_t *blk, int t, uint32_t (&W)[Stream<D, B>::NW]) {
    constexpr int RT = D / 8, NT = 2 * D, NCH = B / 2;
#pragma unroll
    for (int i = 0; i < Stream<D, B>::NW; ++i) W[i] = 0u;
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
        const uint8_t *p = blk + (size_t)(c * NT + t) * RT;
        if constexpr (RT == 16) {
            const uint4 v = *reinterpret_cast<const uint4 *>(p);
            W[4 * c] = v.x; W[4 * c + 1] = v.y; W[4 * c + 2] = v.z; W[4 * c + 3] = v.w;
        } else if constexpr (RT == 8) {
            const uint2 v = *reinterpret_cast<const uint2 *>(p);
            W[2 * c] = v.x; W[2 * c + 1] = v.y;
        } else if constexpr (RT == 4) {
            W[c] = *reinterpret_cast<const uint32_t *>(p);
        } else {
            const uint32_t v = *reinterpret_cast<const uint16_t *>(p);
            W[c >> 1] |= v << (16 * (c & 1));
        }
    }
}

// Load chunk c of thread t's code stream into W (RT bytes per chunk).
template <int D, int B>
__device__ __forceinline__ void load_chunk(const uint8_t *blk, int t, int c, uint32_t (&W)[Stream<D, B>::NW]) {
    constexpr int RT = D / 8, NT = 2 * D;
    const uint8_t *p = blk + (size_t)(c * NT + t) * RT;
    if constexpr (RT == 16) {
        const uint4 v = *reinterpret_cast<const uint4 *>(p);
        W[4 * c] = v.x; W[4 * c + 1] = v.y; W[4 * c + 2] = v.z; W[4 * c + 3] = v.w;
    } else if constexpr (RT == 8) {
        const uint2 v = *reinterpret_cast<const uint2 *>(p);
        W[2 * c] = v.x; W[2 * c + 1] = v.y;
    } else if constexpr (RT == 4) {
        W[c] = *reinterpret_cast<const uint32_t *>(p);
    } else {
        const uint32_t v = *reinterpret_cast<const uint16_t *>(p);
        if (c & 1) W[c >> 1] |= v << 16;
        else W[c >> 1] = v;
    }
}

template <int D, int B>
__device__ __forceinline__ void store_stream(uint8_t *blk, int t, const uint32_t (&W)[Stream<D, B>::NW]) {
    constexpr int RT = D / 8, NT = 2 * D, NCH = B / 2;
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
        uint8_t *p = blk + (size_t)(c * NT + t) * RT;
        if constexpr (RT == 16) {
            *reinterpret_cast<uint4 *>(p) = make_uint4(W[4 * c], W[4 * c + 1], W[4 * c + 2], W[4 * c + 3]);
        } else if constexpr (RT == 8) {
            *reinterpret_cast<uint2 *>(p) = make_uint2(W[2 * c], W[2 * c + 1]);
        } else if constexpr (RT == 4) {
            *reinterpret_cast<uint32_t *>(p) = W[c];
        } else {
            *reinterpret_cast<uint16_t *>(p) = (uint16_t)(W[c >> 1] >> (16 * (c & 1)));
        }
    }
}

template <int N>
__device__ __forceinline__ float tree_sum1(float (&x)[N]) {
#pragma unroll
    for (int s = 1; s < N; s <<= 1)
#pragma unroll
        for (int i = 0; i + s < N; i += 2 * s) x[i] = x[i] + x[i + s];
    return x[0];
}

// Balanced pairwise tree over terms pushed in index order, holding only
// log2(N) + 1 partial sums (push(r, v) with r = 0, 1, ..., N-1 unrolled).
template <int N>
struct PairTree {
    static constexpr int LV = (N >= 16) ? 5 : (N >= 8) ? 4 : (N >= 4) ? 3 : (N >= 2) ? 2 : 1;
    float2 s[LV];
    __device__ __forceinline__ void push(int r, float2 v) {
        int lvl = 0;
#pragma unroll
        for (int b = 0; b < LV - 1; ++b) {
            if (r & (1 << b)) {
                v = add2(s[lvl], v);
                ++lvl;
            } else {
                break;
            }
        }
        s[lvl] = v;
    }
    __device__ __forceinline__ float2 total() const { return s[LV - 1]; }
};

// Packing of e = z + qmax in [0, 2 qmax] (the stored field is e + 1): e is
// added into the stream at its bit offset, the +1 of every field is a
// per-word constant folded in at the end.
template <int D, int B>
__host__ __device__ constexpr uint32_t pack_ones(int w) {
    uint32_t c = 0;
    for (int p = 0; p < 4 * (D / 8); ++p) {
        const int bit = p * B;
        if ((bit >> 5) == w && (bit & 31) + B <= 32) c += 1u << (bit & 31);
    }
    return c;
}

template <int D, int B, int W>
struct PackOnes {
    static constexpr uint32_t value = pack_ones<D, B>(W);
};

template <int D, int B, int W = 0>
__device__ __forceinline__ void add_pack_ones(uint32_t *w) {
    if constexpr (W < Stream<D, B>::WORDS) {
        w[W] += PackOnes<D, B, W>::value;
        add_pack_ones<D, B, W + 1>(w);
    }
}

template <int B>
__device__ __forceinline__ void field_acc(uint32_t *W, int p, uint32_t e) {
    const int bit = p * B;
    const int w = bit >> 5;
    const int s = bit & 31;
    if (s + B <= 32) {
        W[w] += e << s;
    } else {  // a field split across two words carries its own +1
        const uint32_t v = e + 1u;
        W[w] += v << s;
        W[w + 1] += v >> (32 - s);
    }
}

// Final code as e = z + qmax, clamped to [0, 2 qmax], from t = fma(y, 1/c,
// kMagic + 2^(B-1)): bits(t) = 0x4B400000 + 2^(B-1) + rint(y/c), and
// |y/c| <= 2 qmax because the refit c is at least c0/2, so the difference
// below cannot overflow.
template <int B>
__device__ __forceinline__ uint32_t final_e(float t) {
    constexpr int Q = (1 << (B - 1)) - 1;
    constexpr int LO = 0x4B400000 + (1 << (B - 1)) - Q;
    return (uint32_t)__viaddmin_s32_relu(__float_as_int(t), -LO, 2 * Q);
}

// Column refit from the per-band least-squares partials in pf0 (numerator)
// and pf1 (denominator): c_j = num / den (c0_j when den = 0), two threads
// per column; each sums four bands pairwise and the pair adds the halves,
// which is the balanced tree over the eight bands.
template <int D, int s16>
__device__ __forceinline__ void column_ls_fit(Scratch<D> &sc, int tid, uint8_t *rec_c) {
    const int j = tid >> 1, h = tid & 1, b0 = 4 * h;
    float num = (sc.pf0[b0][j] + sc.pf0[b0 + 1][j]) + (sc.pf0[b0 + 2][j] + sc.pf0[b0 + 3][j]);
    float den = (sc.pf1[b0][j] + sc.pf1[b0 + 1][j]) + (sc.pf1[b0 + 2][j] + sc.pf1[b0 + 3][j]);
    num = num + __shfl_xor_sync(0xffffffffu, num, 1);
    den = den + __shfl_xor_sync(0xffffffffu, den, 1);
    if (h == 0) {
        const float c = scale_round((den > 0.0f) ? __fdiv_rn(num, den) : sc.c0[j], s16);
        sc.ic[j] = __frcp_rn(c);
        sc.cold[j] = c;
        if (rec_c) scale_put(rec_c, j, c, s16);
    }
    __syncthreads();
}

// ---------------------------------------------------------------------------
// Refit of the fp32 tile S held in registers as column pairs (all rows at
// width B).  On return S holds y = fl(S * fl(1/r)); sc.rowr[i] = r_i,
// sc.cold[j] = c_j, sc.ic[j] = fl(1/c_j) (r and c rounded to the stored
// precision first when s16).  rec_r / rec_c (global scale arrays, may be
// null) receive r and c.  rho / wbar: the head's rho_i and wbar_i (shared
// memory).
// ---------------------------------------------------------------------------
template <int D, int B, int s16>
__device__ void fit_scales(float2 (&S)[D / 8][2], Scratch<D> &sc, int tid, const float *rho, const float *wbar,
                           uint8_t *rec_r, uint8_t *rec_c) {
    using G = Geo<D>;
    constexpr int RT = G::RT, LANES = G::LANES, RS = Scratch<D>::RS, HALF = LANES / 2;
    constexpr int Q = (1 << (B - 1)) - 1;
    const int g = tid / LANES, l = tid % LANES;
    const int j0 = 4 * l;

    // 1. row sums: thread partial over its 4 columns, then the other lanes'
    //    partials of the row through shared memory (pairwise in lane order)
    float *rs = &sc.rsum[g][0][0];
#pragma unroll
    for (int r = 0; r < RT; ++r)
        rs[r * RS + l] = (fabsf(S[r][0].x) + fabsf(S[r][0].y)) + (fabsf(S[r][1].x) + fabsf(S[r][1].y));
    __syncwarp();
    {
        const int rr = l >> 1, hh = l & 1;
        const float *src = rs + rr * RS + hh * HALF;
        float v[HALF];
        if constexpr (HALF % 4 == 0) {
#pragma unroll
            for (int k = 0; k < HALF / 4; ++k) {
                const float4 x = *reinterpret_cast<const float4 *>(src + 4 * k);
                v[4 * k] = x.x; v[4 * k + 1] = x.y; v[4 * k + 2] = x.z; v[4 * k + 3] = x.w;
            }
        } else {
#pragma unroll
            for (int k = 0; k < HALF; ++k) v[k] = src[k];
        }
        float s = tree_sum1<HALF>(v);
        s = s + __shfl_xor_sync(0xffffffffu, s, 1);
        const int i = g * RT + rr;
        float m = __fmul_rn(s, 1.0f / (float)D);
        m = fmaxf(m, 1e-12f);
        const float ri = scale_round(__fmul_rn(m, rho[i]), s16);
        const float inv = __frcp_rn(ri);
        const float bw = __fmul_rn(wbar[i], __fmul_rn(ri, ri));
        if (hh == 0) {
            sc.rinv2[i] = make_float2(inv, inv);
            sc.bw2[i] = make_float2(bw, bw);
            sc.rowr[i] = ri;
            if (rec_r) scale_put(rec_r, i, ri, s16);
        }
    }
    __syncwarp();
    // 2. y = fl(S * (1/r)) in place; 3. column absmax partials
    {
        float2 m01 = make_float2(0.0f, 0.0f), m23 = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int r = 0; r < RT; r += 2) {
            const float4 f = *reinterpret_cast<const float4 *>(&sc.rinv2[g * RT + r]);
            const float2 i0 = make_float2(f.x, f.y), i1 = make_float2(f.z, f.w);
            S[r][0] = mul2(S[r][0], i0);
            S[r][1] = mul2(S[r][1], i0);
            S[r + 1][0] = mul2(S[r + 1][0], i1);
            S[r + 1][1] = mul2(S[r + 1][1], i1);
            m01.x = fmaxf(m01.x, fmaxf(fabsf(S[r][0].x), fabsf(S[r + 1][0].x)));
            m01.y = fmaxf(m01.y, fmaxf(fabsf(S[r][0].y), fabsf(S[r + 1][0].y)));
            m23.x = fmaxf(m23.x, fmaxf(fabsf(S[r][1].x), fabsf(S[r + 1][1].x)));
            m23.y = fmaxf(m23.y, fmaxf(fabsf(S[r][1].y), fabsf(S[r + 1][1].y)));
        }
        *reinterpret_cast<float4 *>(&sc.pf0[g][j0]) = make_float4(m01.x, m01.y, m23.x, m23.y);
    }
    __syncthreads();
    {  // two threads per column, four bands each
        const int j = tid >> 1, h = tid & 1;
        float m = fmaxf(fmaxf(sc.pf0[4 * h][j], sc.pf0[4 * h + 1][j]), fmaxf(sc.pf0[4 * h + 2][j], sc.pf0[4 * h + 3][j]));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
        if (h == 0) {
            const float c0 = (m == 0.0f) ? 1.0f : __fdiv_rn(m, (float)Q);
            sc.c0[j] = c0;
            sc.ic0[j] = __frcp_rn(c0);
        }
    }
    __syncthreads();
    // 4. z0 and the weighted least-squares sums (pairwise over rows)
    {
        const float2 mg = make_float2(kMagic, kMagic);
        const float2 nmg = make_float2(-kMagic, -kMagic);
        const float2 nz2 = make_float2(sc.nz, sc.nz);
        const float4 ic4 = *reinterpret_cast<const float4 *>(&sc.ic0[j0]);
#pragma unroll
        for (int hp = 0; hp < 2; ++hp) {
            const int jA = j0 + 2 * hp;
            const float2 ic = hp ? make_float2(ic4.z, ic4.w) : make_float2(ic4.x, ic4.y);
            PairTree<RT> tn, td;
            float4 f;
#pragma unroll
            for (int r = 0; r < RT; ++r) {
                if ((r & 1) == 0) f = *reinterpret_cast<const float4 *>(&sc.bw2[g * RT + r]);
                const float2 b2 = (r & 1) ? make_float2(f.z, f.w) : make_float2(f.x, f.y);
                const float2 y = S[r][hp];
                const float2 z0 = add2(fma2(y, ic, mg), nmg);
                // fl(b * p) written as fma(b, p, -0) with a run-time -0: the
                // product is rounded once and cannot be contracted into the
                // pairwise additions that follow
                tn.push(r, fma2(b2, mul2(z0, y), nz2));
                td.push(r, fma2(b2, mul2(z0, z0), nz2));
            }
            *reinterpret_cast<float2 *>(&sc.pf0[g][jA]) = tn.total();
            *reinterpret_cast<float2 *>(&sc.pf1[g][jA]) = td.total();
        }
    }
    __syncthreads();
    column_ls_fit<D, s16>(sc, tid, rec_c);
}

// Refit and pack into the record at `rec` (global): codes, r, c.
template <int D, int B, int s16>
__device__ void fit_pack(float2 (&S)[D / 8][2], uint8_t *rec, Scratch<D> &sc, int tid, const float *rho,
                         const float *wbar) {
    using G = Geo<D>;
    constexpr int RT = G::RT, LANES = G::LANES;
    constexpr int OFF = 1 << (B - 1);
    constexpr float MG2 = kMagic + (float)OFF;
    const int l = tid % LANES;
    const int j0 = 4 * l;
    const uint32_t codes_bytes = (uint32_t)D * D * B / 8;
    uint8_t *rec_r = rec + codes_bytes;
    uint8_t *rec_c = rec_r + D * (s16 ? 2 : 4);
    fit_scales<D, B, s16>(S, sc, tid, rho, wbar, rec_r, rec_c);
    uint32_t W[Stream<D, B>::NW];
#pragma unroll
    for (int i = 0; i < Stream<D, B>::NW; ++i) W[i] = 0u;
    const float4 ic4 = *reinterpret_cast<const float4 *>(&sc.ic[j0]);
    const float2 mg2 = make_float2(MG2, MG2);
#pragma unroll
    for (int hp = 0; hp < 2; ++hp) {
        const float2 ic = hp ? make_float2(ic4.z, ic4.w) : make_float2(ic4.x, ic4.y);
#pragma unroll
        for (int r = 0; r < RT; ++r) {
            const float2 t = fma2(S[r][hp], ic, mg2);
            field_acc<B>(W, 4 * r + 2 * hp, final_e<B>(t.x));
            field_acc<B>(W, 4 * r + 2 * hp + 1, final_e<B>(t.y));
        }
    }
    add_pack_ones<D, B>(W);
    store_stream<D, B>(rec, tid, W);
}

// Per-row absmax requantization (the baseline quantizer of the plan's
// quantizer field): r_i = fl(max_j |S_ij| / qmax) (1 for a zero row), codes
// = clamp(rne(S_ij * fl(1/r_i))), c = 1.  Rows live inside one warp, so the
// whole fit needs no block barrier.  Writes codes, r and c to `rec`.
template <int D, int B, int s16>
__device__ void fit_pack_absmax(float2 (&S)[D / 8][2], uint8_t *rec, Scratch<D> &sc, int tid) {
    using G = Geo<D>;
    constexpr int RT = G::RT, LANES = G::LANES, RS = Scratch<D>::RS, HALF = LANES / 2;
    constexpr int Q = (1 << (B - 1)) - 1;
    constexpr float MG2 = kMagic + (float)(1 << (B - 1));
    const int g = tid / LANES, l = tid % LANES;
    const uint32_t codes_bytes = (uint32_t)D * D * B / 8;
    uint8_t *rec_r = rec + codes_bytes;
    uint8_t *rec_c = rec_r + D * (s16 ? 2 : 4);
    // 1. row maxima: this thread's 4 columns, then the row's lanes (transpose)
    float *rs = &sc.rsum[g][0][0];
#pragma unroll
    for (int r = 0; r < RT; ++r)
        rs[r * RS + l] = fmaxf(fmaxf(fabsf(S[r][0].x), fabsf(S[r][0].y)), fmaxf(fabsf(S[r][1].x), fabsf(S[r][1].y)));
    __syncwarp();
    {
        const int rr = l >> 1, hh = l & 1;
        const float *src = rs + rr * RS + hh * HALF;
        float m = 0.0f;
#pragma unroll
        for (int k = 0; k < HALF; ++k) m = fmaxf(m, src[k]);
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
        const int i = g * RT + rr;
        const float ri = scale_round((m > 0.0f) ? __fdiv_rn(m, (float)Q) : 1.0f, s16);
        const float inv = __frcp_rn(ri);
        if (hh == 0) {
            sc.rinv2[i] = make_float2(inv, inv);
            scale_put(rec_r, i, ri, s16);
        }
    }
    __syncwarp();
    if (tid < D) scale_put(rec_c, tid, 1.0f, s16);
    // 2. codes e = rne(S * fl(1/r)) + qmax, clamped, packed into the stream
    uint32_t W[Stream<D, B>::NW];
#pragma unroll
    for (int i = 0; i < Stream<D, B>::NW; ++i) W[i] = 0u;
    const float2 mg2 = make_float2(MG2, MG2);
#pragma unroll
    for (int r = 0; r < RT; r += 2) {
        const float4 f = *reinterpret_cast<const float4 *>(&sc.rinv2[g * RT + r]);
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
            const float2 inv2 = rr ? make_float2(f.z, f.w) : make_float2(f.x, f.y);
#pragma unroll
            for (int hp = 0; hp < 2; ++hp) {
                const float2 t = fma2(S[r + rr][hp], inv2, mg2);
                field_acc<B>(W, 4 * (r + rr) + 2 * hp, final_e<B>(t.x));
                field_acc<B>(W, 4 * (r + rr) + 2 * hp + 1, final_e<B>(t.y));
            }
        }
    }
    add_pack_ones<D, B>(W);
    store_stream<D, B>(rec, tid, W);
    (void)Q;
}

// Pivot head (binary16 tile): S_t -> fp16 RNE, written in place.
template <int D>
__device__ __forceinline__ void store_pivot(float2 (&S)[D / 8][2], uint8_t *rec, int tid) {
    using G = Geo<D>;
    const int g = tid / G::LANES, l = tid % G::LANES;
#pragma unroll
    for (int r = 0; r < G::RT; ++r) {
        const int i = g * G::RT + r;
        const __half2 h01 = __float22half2_rn(S[r][0]);
        const __half2 h23 = __float22half2_rn(S[r][1]);
        uint2 v;
        v.x = *reinterpret_cast<const uint32_t *>(&h01);
        v.y = *reinterpret_cast<const uint32_t *>(&h23);
        *reinterpret_cast<uint2 *>(rec + ((size_t)i * D + 4 * l) * 2) = v;
    }
}

template <int D>
__device__ __forceinline__ void load_pivot(const uint8_t *rec, int tid, float2 (&h)[D / 8][2]) {
    using G = Geo<D>;
    const int g = tid / G::LANES, l = tid % G::LANES;
#pragma unroll
    for (int r = 0; r < G::RT; ++r) {
        const int i = g * G::RT + r;
        const uint2 v = *reinterpret_cast<const uint2 *>(rec + ((size_t)i * D + 4 * l) * 2);
        h[r][0] = __half22float2(*reinterpret_cast<const __half2 *>(&v.x));
        h[r][1] = __half22float2(*reinterpret_cast<const __half2 *>(&v.y));
    }
}

// Per-band fp64 sums of sum_i q_i k_i.  Warp w holds rows [16 w, 16 w + 16):
// lane L < 16 carries row 16 w + L (lanes 16..31 carry zeros); a band is RT
// consecutive rows, so the butterfly over RT lanes stays inside the warp.
template <int D>
__device__ __forceinline__ void band_sums(Scratch<D> &sc, int tid, double x2) {
    constexpr int RT = D / 8;
#pragma unroll
    for (int m = 1; m < RT; m <<= 1) x2 += __shfl_xor_sync(0xffffffffu, x2, m);
    const int lane = tid & 31, i = 16 * (tid >> 5) + lane;
    if (lane < 16 && (lane % RT) == 0) sc.bandQK[i / RT] = x2;
}

// Column phase of the decode: u, w, o of column j from the band partials
// (already relative to the offset-binary bias), two threads per column.
template <int D, int KIND, int s16 = 0>
__device__ __forceinline__ void finish_columns(const Args &a, Scratch<D> &sc, int tid, int row, float beta,
                                               const float *vs, const uint8_t *cs) {
    const int j = tid >> 1, h = tid & 1, b0 = 4 * h;
    double su = (sc.u.col.pU[b0][j] + sc.u.col.pU[b0 + 1][j]) + (sc.u.col.pU[b0 + 2][j] + sc.u.col.pU[b0 + 3][j]);
    double so = (sc.u.col.pO[b0][j] + sc.u.col.pO[b0 + 1][j]) + (sc.u.col.pO[b0 + 2][j] + sc.u.col.pO[b0 + 3][j]);
    double qk = (sc.bandQK[b0] + sc.bandQK[b0 + 1]) + (sc.bandQK[b0 + 2] + sc.bandQK[b0 + 3]);
    su += __shfl_xor_sync(0xffffffffu, su, 1);
    so += __shfl_xor_sync(0xffffffffu, so, 1);
    qk += __shfl_xor_sync(0xffffffffu, qk, 1);
    const double cj = cs ? (double)scale_at(cs, j, s16) : 1.0;
    const float u = __double2float_rn(cj * su);
    const float w = __fmul_rn(beta, __fsub_rn(vs[j], u));
    const float o = __double2float_rn(cj * so + qk * (double)w);
    if (h == 0) {
        a.o[(size_t)row * D + j] = o;
        if (KIND == kDecode) a.w[(size_t)row * D + j] = w;
        else sc.wv[j] = w;
    }
}

// ---------------------------------------------------------------------------
// One quantized head of width B: decode / fit-pack / fused.
// ---------------------------------------------------------------------------
template <int D, int B, int KIND, int s16>
__device__ void item_uniform(const Args &a, uint8_t *stage, uint8_t *rec_g, int row, Scratch<D> &sc, int tid) {
    using G = Geo<D>;
    constexpr int RT = G::RT, LANES = G::LANES;
    constexpr int OFF = 1 << (B - 1);
    const int g = tid / LANES, l = tid % LANES;
    const int j0 = 4 * l;
    const uint32_t codes_bytes = (uint32_t)D * D * B / 8;
    const uint8_t *st_r = stage + codes_bytes;              // staged r[D] and c[D]
    const uint8_t *st_c = st_r + D * (s16 ? 2 : 4);
    const float *tf = reinterpret_cast<const float *>(stage + a.rec_stage_bytes);
    const float *qs = tf + kTailQ * D;
    const float *ks = tf + kTailK * D;
    const float *vs = tf + kTailV * D;
    const float *xs = tf + kTailX * D;
    const float *ab = tf + kTailRw * D + D / 4;
    const float alpha = ab[0];
    const float beta = ab[1];

    // per-row parameters of this warp's 16 rows (only this warp reads them)
    double bqk = 0.0;
    if ((tid & 31) < 16) {
        const int i = 16 * (tid >> 5) + (tid & 31);
        const float ai = __fmul_rn(alpha, scale_at(st_r, i, s16));
        const float ki = ks[i];
        sc.a2[i] = make_float2(ai, ai);
        sc.k2[i] = make_float2(ki, ki);
        if (KIND != kFitPack) {
            // k_i a_i and q_i a_i (exact in fp64) times 2^-12: the fp64 operand below is z 2^12
            sc.kap[i] = (double)ks[i] * (double)ai * (1.0 / 4096.0);
            sc.qt[i] = (double)qs[i] * (double)ai * (1.0 / 4096.0);
            bqk = (double)qs[i] * (double)ks[i];
        }
    }
    if (KIND != kFitPack) band_sums<D>(sc, tid, bqk);
    __syncwarp();

    uint32_t W[Stream<D, B>::NW];
    W[Stream<D, B>::NW - 1] = 0u;
    const uint32_t xb = a.x_bits;
    int loaded = -1;  // chunks are loaded as the rows reach them (fewer live registers)

    float2 S[RT][2];
    double accU[4] = {0.0, 0.0, 0.0, 0.0}, accO[4] = {0.0, 0.0, 0.0, 0.0};
    float2 cp01, cp23;
    if (KIND != kDecode) {  // c_j 2^-12 of this thread's columns (exact scaling)
        const float4 c4 = scale4_at(st_c, j0, s16);
        const float2 s12 = make_float2(1.0f / 4096.0f, 1.0f / 4096.0f);
        cp01 = mul2(make_float2(c4.x, c4.y), s12);
        cp23 = mul2(make_float2(c4.z, c4.w), s12);
    }
    constexpr float ZB = 8388608.0f + (float)OFF * 4096.0f;
    const float2 nzb = make_float2(-ZB, -ZB);
#pragma unroll
    for (int r = 0; r < RT; r += 2) {
        const int i = g * RT + r;
        double2 kap2, qt2;
        if (KIND != kFitPack) {
            kap2 = *reinterpret_cast<const double2 *>(&sc.kap[i]);
            qt2 = *reinterpret_cast<const double2 *>(&sc.qt[i]);
        }
        float4 a4;
        if (KIND != kDecode) a4 = *reinterpret_cast<const float4 *>(&sc.a2[i]);
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
            {
                constexpr int CB = D / 8;  // chunk bytes
                const int last = ((4 * (r + rr + 1) * B - 1) / 8) / CB;
#pragma unroll
                for (int c = 0; c < B / 2; ++c)
                    if (c > loaded && c <= last) load_chunk<D, B>(stage, tid, c, W);
                if (last > loaded) loaded = last;
            }
            uint32_t X[4];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) X[jj] = field_x<B>(W, 4 * (r + rr) + jj, xb);
            // z 2^12, exact in fp32
            const float2 z01 = add2(make_float2(__uint_as_float(X[0]), __uint_as_float(X[1])), nzb);
            const float2 z23 = add2(make_float2(__uint_as_float(X[2]), __uint_as_float(X[3])), nzb);
            if (KIND != kFitPack) {
                // u and o partials: sums of the exact products (k_i a_i 2^-12) (z_ij 2^12) in fp64
                const double kap = rr ? kap2.y : kap2.x, qt = rr ? qt2.y : qt2.x;
                const double d[4] = {(double)z01.x, (double)z01.y, (double)z23.x, (double)z23.y};
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    accU[jj] = fma(kap, d[jj], accU[jj]);
                    accO[jj] = fma(qt, d[jj], accO[jj]);
                }
            }
            if (KIND != kDecode) {
                const float2 a2 = rr ? make_float2(a4.z, a4.w) : make_float2(a4.x, a4.y);
                S[r + rr][0] = mul2(mul2(a2, cp01), z01);
                S[r + rr][1] = mul2(mul2(a2, cp23), z23);
            }
        }
    }

    if (KIND != kFitPack) {
        // hand this band's partials over
        *reinterpret_cast<double2 *>(&sc.u.col.pU[g][j0]) = make_double2(accU[0], accU[1]);
        *reinterpret_cast<double2 *>(&sc.u.col.pU[g][j0 + 2]) = make_double2(accU[2], accU[3]);
        *reinterpret_cast<double2 *>(&sc.u.col.pO[g][j0]) = make_double2(accO[0], accO[1]);
        *reinterpret_cast<double2 *>(&sc.u.col.pO[g][j0 + 2]) = make_double2(accO[2], accO[3]);
        __syncthreads();
        finish_columns<D, KIND, s16>(a, sc, tid, row, beta, vs, st_c);
        if (KIND == kFused) __syncthreads();
    }

    if (KIND != kDecode) {
        const float4 w4 = *reinterpret_cast<const float4 *>(KIND == kFitPack ? &xs[j0] : &sc.wv[j0]);
        const float2 w01 = make_float2(w4.x, w4.y);
        const float2 w23 = make_float2(w4.z, w4.w);
#pragma unroll
        for (int r = 0; r < RT; r += 2) {
            const float4 k4 = *reinterpret_cast<const float4 *>(&sc.k2[g * RT + r]);
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                const float2 k2 = rr ? make_float2(k4.z, k4.w) : make_float2(k4.x, k4.y);
                S[r + rr][0] = fma2(k2, w01, S[r + rr][0]);
                S[r + rr][1] = fma2(k2, w23, S[r + rr][1]);
            }
        }
        if (a.quantizer == kQuantAbsmax) fit_pack_absmax<D, B, s16>(S, rec_g, sc, tid);
        else fit_pack<D, B, s16>(S, rec_g, sc, tid, tf + kTailRho * D, tf + kTailWbar * D);
    }
}

// One FP16 pivot head.
template <int D, int KIND>
__device__ void item_pivot(const Args &a, uint8_t *stage, uint8_t *rec_g, int row, Scratch<D> &sc, int tid) {
    using G = Geo<D>;
    constexpr int RT = G::RT, LANES = G::LANES;
    const int g = tid / LANES, l = tid % LANES;
    const int j0 = 4 * l;
    const float *tf = reinterpret_cast<const float *>(stage + a.rec_stage_bytes);
    const float *qs = tf + kTailQ * D;
    const float *ks = tf + kTailK * D;
    const float *vs = tf + kTailV * D;
    const float *xs = tf + kTailX * D;
    const float *ab = tf + kTailRw * D + D / 4;
    const float alpha = ab[0];
    const float beta = ab[1];
    double bqk = 0.0;
    if ((tid & 31) < 16) {  // this warp's 16 rows
        const int i = 16 * (tid >> 5) + (tid & 31);
        sc.k2[i] = make_float2(ks[i], ks[i]);
        if (KIND != kFitPack) {
            sc.kap[i] = (double)ks[i] * (double)alpha;
            sc.qt[i] = (double)qs[i] * (double)alpha;
            bqk = (double)qs[i] * (double)ks[i];
        }
    }
    if (KIND != kFitPack) band_sums<D>(sc, tid, bqk);
    __syncwarp();
    float2 S[RT][2];
    load_pivot<D>(rec_g, tid, S);
    if (KIND != kFitPack) {
        double accU[4] = {0.0, 0.0, 0.0, 0.0}, accO[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
        for (int r = 0; r < RT; ++r) {
            const int i = g * RT + r;
            const double kap = sc.kap[i], qt = sc.qt[i];
            const double d[4] = {(double)S[r][0].x, (double)S[r][0].y, (double)S[r][1].x, (double)S[r][1].y};
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                accU[jj] = fma(kap, d[jj], accU[jj]);
                accO[jj] = fma(qt, d[jj], accO[jj]);
            }
        }
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            sc.u.col.pU[g][j0 + jj] = accU[jj];
            sc.u.col.pO[g][j0 + jj] = accO[jj];
        }
        __syncthreads();
        finish_columns<D, KIND>(a, sc, tid, row, beta, vs, nullptr);
        if (KIND == kFused) __syncthreads();
    }
    if (KIND != kDecode) {
        const float2 al = make_float2(alpha, alpha);
        const float4 w4 = *reinterpret_cast<const float4 *>(KIND == kFitPack ? &xs[j0] : &sc.wv[j0]);
        const float2 w01 = make_float2(w4.x, w4.y);
        const float2 w23 = make_float2(w4.z, w4.w);
#pragma unroll
        for (int r = 0; r < RT; ++r) {
            const float2 k2 = sc.k2[g * RT + r];
            S[r][0] = fma2(k2, w01, mul2(al, S[r][0]));
            S[r][1] = fma2(k2, w23, mul2(al, S[r][1]));
        }
        store_pivot<D>(S, rec_g, tid);
    }
}

// ---------------------------------------------------------------------------
// Per-key-row units (KDA, mode 1): every key row has its own width b_i
// (2, 4, 6, 8, or 16 for an FP16 pivot row) and its own retention gate.
// Row-major codes: lane l's four codes of a row are row bits [4 b l, 4 b l + 4 b).
// The width of a row is the same for all lanes of a band, so the per-row
// branches below are uniform across a warp.
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

// Final code e = z + qmax in [0, 2 qmax] of a row of width b (see final_e).
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

    // 1. row sums and row factors
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
    {  // two threads per column, four bands each
        const int j = tid >> 1, h = tid & 1, b0 = 4 * h;
        float mm[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            mm[c] = fmaxf(fmaxf(sc.u.pmax[c][b0][j], sc.u.pmax[c][b0 + 1][j]),
                          fmaxf(sc.u.pmax[c][b0 + 2][j], sc.u.pmax[c][b0 + 3][j]));
            mm[c] = fmaxf(mm[c], __shfl_xor_sync(0xffffffffu, mm[c], 1));
        }
        if (h == 0) {
            float c0 = 0.0f;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int q = (1 << (2 * c + 1)) - 1;  // widths 2, 4, 6, 8
                if (mm[c] > 0.0f) c0 = fmaxf(c0, __fdiv_rn(mm[c], (float)q));
            }
            if (c0 == 0.0f) c0 = 1.0f;
            sc.c0[j] = c0;
            sc.ic0[j] = __frcp_rn(c0);
        }
    }
    __syncthreads();
    // 4. z0 and the weighted least-squares sums over the quantized rows
    {
        const float2 mg = make_float2(kMagic, kMagic);
        const float2 nmg = make_float2(-kMagic, -kMagic);
        const float2 nz2 = make_float2(sc.nz, sc.nz);
        const float4 ic4 = *reinterpret_cast<const float4 *>(&sc.ic0[j0]);
#pragma unroll
        for (int hp = 0; hp < 2; ++hp) {
            const int jA = j0 + 2 * hp;
            const float2 ic = hp ? make_float2(ic4.z, ic4.w) : make_float2(ic4.x, ic4.y);
            PairTree<RT> tn, td;
#pragma unroll
            for (int r = 0; r < RT; ++r) {
                const int i = g * RT + r;
                float2 vn = make_float2(0.0f, 0.0f), vd = make_float2(0.0f, 0.0f);
                if (rw[i] != kPivotBits) {
                    const float2 b2 = sc.bw2[i];
                    const float2 y = S[r][hp];
                    const float2 z0 = add2(fma2(y, ic, mg), nmg);
                    vn = fma2(b2, mul2(z0, y), nz2);
                    vd = fma2(b2, mul2(z0, z0), nz2);
                }
                tn.push(r, vn);
                td.push(r, vd);
            }
            *reinterpret_cast<float2 *>(&sc.pf0[g][jA]) = tn.total();
            *reinterpret_cast<float2 *>(&sc.pf1[g][jA]) = td.total();
        }
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

template <int D>
__device__ __forceinline__ void rows_prologue_tables(const Args &a, Scratch<D> &sc, int tid, int gl) {
    if (tid < D) {
        sc.rw[tid] = a.t.row_width[(size_t)gl * D + tid];
        sc.roff[tid] = a.t.row_off[(size_t)gl * D + tid];
        sc.rho[tid] = a.t.rho[(size_t)gl * D + tid];
        sc.wbar[tid] = a.t.wbar[(size_t)gl * D + tid];
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
    const float *tf = reinterpret_cast<const float *>(stage + a.rec_stage_bytes);
    const float *qs = tf + kTailQ * D;
    const float *ks = tf + kTailK * D;
    const float *vs = tf + kTailV * D;
    const float *xs = tf + kTailX * D;
    const float *als = tf + kTailAlpha * D;
    const uint32_t *roff = reinterpret_cast<const uint32_t *>(tf + kTailRoff * D);
    const uint8_t *rw = reinterpret_cast<const uint8_t *>(tf + kTailRw * D);
    const float beta = (tf + kTailRw * D + D / 4)[1];

    double bqk = 0.0;
    if ((tid & 31) < 16) {  // this warp's 16 rows
        const int i = 16 * (tid >> 5) + (tid & 31);
        const int b = rw[i];
        const float al = als[i];
        const float ai = (b == kPivotBits) ? al : __fmul_rn(al, scale_at(st_r, i, s16));
        sc.a2[i] = make_float2(ai, ai);
        sc.k2[i] = make_float2(ks[i], ks[i]);
        if (KIND != kFitPack) {
            const double ka = (double)ks[i] * (double)ai;
            const double qa = (double)qs[i] * (double)ai;
            // quantized rows: times 2^-12, the fp64 operand below being z 2^12
            const double sk = (b == kPivotBits) ? 1.0 : 1.0 / 4096.0;
            sc.kap[i] = ka * sk;
            sc.qt[i] = qa * sk;
            bqk = (double)qs[i] * (double)ks[i];
        }
    }
    if (KIND != kFitPack) band_sums<D>(sc, tid, bqk);
    __syncwarp();

    float2 S[RT][2];
    double accU[4] = {0.0, 0.0, 0.0, 0.0}, accO[4] = {0.0, 0.0, 0.0, 0.0};
    double accUp[4] = {0.0, 0.0, 0.0, 0.0}, accOp[4] = {0.0, 0.0, 0.0, 0.0};
    const uint32_t xb = a.x_bits;
    const float4 c4 = scale4_at(st_c, j0, s16);
    const float2 s12 = make_float2(1.0f / 4096.0f, 1.0f / 4096.0f);
    const float2 cp01 = mul2(make_float2(c4.x, c4.y), s12), cp23 = mul2(make_float2(c4.z, c4.w), s12);
#pragma unroll
    for (int r = 0; r < RT; ++r) {
        const int i = g * RT + r;
        const int b = rw[i];
        const float2 a2 = sc.a2[i];
        if (b == kPivotBits) {
            const uint2 v = *reinterpret_cast<const uint2 *>(stage + roff[i] + 8 * l);
            const float2 h01 = __half22float2(*reinterpret_cast<const __half2 *>(&v.x));
            const float2 h23 = __half22float2(*reinterpret_cast<const __half2 *>(&v.y));
            if (KIND != kFitPack) {
                const double kap = sc.kap[i], qt = sc.qt[i];
                const double d[4] = {(double)h01.x, (double)h01.y, (double)h23.x, (double)h23.y};
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    accUp[jj] = fma(kap, d[jj], accUp[jj]);
                    accOp[jj] = fma(qt, d[jj], accOp[jj]);
                }
            }
            S[r][0] = mul2(a2, h01);
            S[r][1] = mul2(a2, h23);
        } else {
            const uint32_t f = row_field(stage + roff[i], b, l);
            // field jj of f moved to bits [12, 12 + b): a funnel shift of the 64-bit f << 12
            const uint32_t flo = f << 12, fhi = f >> 20;
            const uint32_t m12 = ((1u << b) - 1u) << 12;
            const float zb = __uint_as_float(0x4B000000u | (1u << (b + 11)));  // 2^23 + 2^(b-1) 2^12
            uint32_t X[4];
            X[0] = (flo & m12) | xb;
#pragma unroll
            for (int jj = 1; jj < 4; ++jj) X[jj] = (__funnelshift_r(flo, fhi, b * jj) & m12) | xb;
            const float2 nzb = make_float2(-zb, -zb);
            const float2 z01 = add2(make_float2(__uint_as_float(X[0]), __uint_as_float(X[1])), nzb);
            const float2 z23 = add2(make_float2(__uint_as_float(X[2]), __uint_as_float(X[3])), nzb);
            if (KIND != kFitPack) {
                const double kap = sc.kap[i], qt = sc.qt[i];
                const double d[4] = {(double)z01.x, (double)z01.y, (double)z23.x, (double)z23.y};
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    accU[jj] = fma(kap, d[jj], accU[jj]);
                    accO[jj] = fma(qt, d[jj], accO[jj]);
                }
            }
            S[r][0] = mul2(mul2(a2, cp01), z01);
            S[r][1] = mul2(mul2(a2, cp23), z23);
        }
    }

    if (KIND != kFitPack) {
        // quantized rows carry c_j; FP16 rows do not: scale the band partial here
        double pu[4], po[4];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            const double cj = (double)scale_at(st_c, j0 + jj, s16);
            pu[jj] = cj * accU[jj] + accUp[jj];
            po[jj] = cj * accO[jj] + accOp[jj];
        }
        *reinterpret_cast<double2 *>(&sc.u.col.pU[g][j0]) = make_double2(pu[0], pu[1]);
        *reinterpret_cast<double2 *>(&sc.u.col.pU[g][j0 + 2]) = make_double2(pu[2], pu[3]);
        *reinterpret_cast<double2 *>(&sc.u.col.pO[g][j0]) = make_double2(po[0], po[1]);
        *reinterpret_cast<double2 *>(&sc.u.col.pO[g][j0 + 2]) = make_double2(po[2], po[3]);
        __syncthreads();
        finish_columns<D, KIND>(a, sc, tid, row, beta, vs, nullptr);
        if (KIND == kFused) __syncthreads();
    }

    if (KIND != kDecode) {
        const float4 w4 = *reinterpret_cast<const float4 *>(KIND == kFitPack ? &xs[j0] : &sc.wv[j0]);
        const float2 w01 = make_float2(w4.x, w4.y);
        const float2 w23 = make_float2(w4.z, w4.w);
#pragma unroll
        for (int r = 0; r < RT; ++r) {
            const float2 k2 = sc.k2[g * RT + r];
            S[r][0] = fma2(k2, w01, S[r][0]);
            S[r][1] = fma2(k2, w23, S[r][1]);
        }
        // the staged codes are no longer read: assemble the new rows there
        uint8_t *rec_r = rec_g + codes_bytes;
        fit_rows<D, s16>(S, sc, tid, rw, roff, tf + kTailRho * D, tf + kTailWbar * D, stage, rec_r,
                         rec_r + D * (s16 ? 2 : 4));
        copy_out<D>(rec_g, stage, codes_bytes, tid);
    }
}

// ---------------------------------------------------------------------------
// Persistent pipeline kernel.
// ---------------------------------------------------------------------------
template <int D, int KIND, int MODE, int S16>
__global__ void __launch_bounds__(2 * D, 2) k_step(Args a) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x;
    const int G = gridDim.x;
    uint8_t *stages = smem;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kStages * a.stage_bytes);
    Scratch<D> &sc = *reinterpret_cast<Scratch<D> *>(smem + kStages * a.stage_bytes + 64);

    // Thread 0 keeps the ring full: the first kStages items here, then the
    // item kStages - 1 ahead right after the barrier that opens each item
    // (every thread is past the previous item, so its stage is free).  The
    // descriptor of the item after that is fetched one item ahead by
    // cp.async, so thread 0 never waits on a global load on this path.
    int dsel = 0;
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(&bars[s], 1);
        fence_mbar_init();
        sc.nz = a.neg_zero;
        for (int s = 0; s < kStages; ++s) {
            const int it = blockIdx.x + s * G;
            if (it >= a.n_items) break;
            int n, ll, di;
            step_coords<D>(a, it, n, ll, di);
            issue_item<D, KIND, MODE>(a, it, a.t.desc[di], a.slots[n], stages + s * a.stage_bytes, &bars[s],
                                      sc.meta[s]);
        }
        const int nx = blockIdx.x + kStages * G;
        if (nx < a.n_items) prefetch_desc<D>(a, nx, sc, 0);
    }
    __syncthreads();
    int s = 0;
    uint32_t phase = 0;
    for (int it = blockIdx.x; it < a.n_items; it += G) {
        const bool ok = mbar_wait_bounded(&bars[s], phase, a.wait_polls);
        if (__syncthreads_or(!ok)) {
            if (tid == 0) {
                flag_error(a.err, kErrWait);
                // let every copy still in flight land before shared memory goes away
                cp_async_wait_all();
                for (int k = 0; k < kStages; ++k) mbar_wait_bounded(&bars[k], phase ^ (k < s ? 1u : 0u), a.wait_polls);
            }
            return;
        }
        if (tid == 0 && it != (int)blockIdx.x) {
            const int ps = (s + kStages - 1) % kStages;
            const int nx = it + (kStages - 1) * G;
            if (nx < a.n_items) {
                cp_async_wait_all();
                issue_item<D, KIND, MODE>(a, nx, sc.dring[dsel], sc.dslot[dsel], stages + ps * a.stage_bytes,
                                          &bars[ps], sc.meta[ps]);
                dsel ^= 1;
                if (nx + G < a.n_items) prefetch_desc<D>(a, nx + G, sc, dsel);
            }
        }
        uint8_t *stage = stages + s * a.stage_bytes;
        const int width = sc.meta[s][1];
        const int valid = sc.meta[s][2];
        uint8_t *rec_g = reinterpret_cast<uint8_t *>((uintptr_t)(uint32_t)sc.meta[s][4] |
                                                     ((uintptr_t)(uint32_t)sc.meta[s][5] << 32));
        if (valid) {
            const int row = sc.meta[s][6];
            if (MODE == 1) {
                item_rows<D, KIND, S16>(a, stage, rec_g, row, (uint32_t)sc.meta[s][3], sc, tid);
            } else {
                switch (width) {
                    case 2: item_uniform<D, 2, KIND, S16>(a, stage, rec_g, row, sc, tid); break;
                    case 4: item_uniform<D, 4, KIND, S16>(a, stage, rec_g, row, sc, tid); break;
                    case 6: item_uniform<D, 6, KIND, S16>(a, stage, rec_g, row, sc, tid); break;
                    case 8: item_uniform<D, 8, KIND, S16>(a, stage, rec_g, row, sc, tid); break;
                    case kPivotBits: item_pivot<D, KIND>(a, stage, rec_g, row, sc, tid); break;
                    default: if (tid == 0) flag_error(a.err, kErrArgs); break;
                }
            }
        }
        if (++s == kStages) { s = 0; phase ^= 1u; }
    }
}

// ---------------------------------------------------------------------------
// Pack fp32 states (S_0) and unpack records: one CTA per head, no pipeline.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(2 * D) k_requant_pack(Args a) {
    extern __shared__ __align__(128) uint8_t smem[];
    Scratch<D> &sc = *reinterpret_cast<Scratch<D> *>(smem);
    uint8_t *codes = smem + ((sizeof(Scratch<D>) + 127) / 128) * 128;  // per-row records: D*D*2 bytes
    using G = Geo<D>;
    const int tid = threadIdx.x;
    const int g = tid / G::LANES, l = tid % G::LANES;
    const int it = blockIdx.x;
    int n, ll, h, gl, row;
    item_coords<D>(a, it, n, ll, h, gl, row);
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
    if (a.mode == 1) {
        rows_prologue_tables<D>(a, sc, tid, gl);
        if (tid == 0) sc.nz = a.neg_zero;
        __syncthreads();
        const uint32_t codes_bytes = a.t.codes_bytes[gl];
        uint8_t *rec_r = rec + codes_bytes;
        if (a.scale16) fit_rows<D, 1>(S, sc, tid, sc.rw, sc.roff, sc.rho, sc.wbar, codes, rec_r, rec_r + 2 * D);
        else fit_rows<D, 0>(S, sc, tid, sc.rw, sc.roff, sc.rho, sc.wbar, codes, rec_r, rec_r + 4 * D);
        copy_out<D>(rec, codes, codes_bytes, tid);
        return;
    }
    const int width = a.t.width[gl];
    if (width == kPivotBits) {
        store_pivot<D>(S, rec, tid);
        return;
    }
    if (tid < D) {
        sc.rho[tid] = a.t.rho[(size_t)gl * D + tid];
        sc.wbar[tid] = a.t.wbar[(size_t)gl * D + tid];
    }
    if (tid == 0) sc.nz = a.neg_zero;
    __syncthreads();
    switch (width) {
        case 2:
            if (a.scale16) {
                if (a.quantizer == kQuantAbsmax) fit_pack_absmax<D, 2, 1>(S, rec, sc, tid);
                else fit_pack<D, 2, 1>(S, rec, sc, tid, sc.rho, sc.wbar);
            } else {
                if (a.quantizer == kQuantAbsmax) fit_pack_absmax<D, 2, 0>(S, rec, sc, tid);
                else fit_pack<D, 2, 0>(S, rec, sc, tid, sc.rho, sc.wbar);
            }
            break;
        case 4:
            if (a.scale16) {
                if (a.quantizer == kQuantAbsmax) fit_pack_absmax<D, 4, 1>(S, rec, sc, tid);
                else fit_pack<D, 4, 1>(S, rec, sc, tid, sc.rho, sc.wbar);
            } else {
                if (a.quantizer == kQuantAbsmax) fit_pack_absmax<D, 4, 0>(S, rec, sc, tid);
                else fit_pack<D, 4, 0>(S, rec, sc, tid, sc.rho, sc.wbar);
            }
            break;
        case 6:
            if (a.scale16) {
                if (a.quantizer == kQuantAbsmax) fit_pack_absmax<D, 6, 1>(S, rec, sc, tid);
                else fit_pack<D, 6, 1>(S, rec, sc, tid, sc.rho, sc.wbar);
            } else {
                if (a.quantizer == kQuantAbsmax) fit_pack_absmax<D, 6, 0>(S, rec, sc, tid);
                else fit_pack<D, 6, 0>(S, rec, sc, tid, sc.rho, sc.wbar);
            }
            break;
        case 8:
            if (a.scale16) {
                if (a.quantizer == kQuantAbsmax) fit_pack_absmax<D, 8, 1>(S, rec, sc, tid);
                else fit_pack<D, 8, 1>(S, rec, sc, tid, sc.rho, sc.wbar);
            } else {
                if (a.quantizer == kQuantAbsmax) fit_pack_absmax<D, 8, 0>(S, rec, sc, tid);
                else fit_pack<D, 8, 0>(S, rec, sc, tid, sc.rho, sc.wbar);
            }
            break;
        default: if (tid == 0) flag_error(a.err, kErrArgs); break;
    }
}

template <int D, int B>
__device__ void unpack_uniform(const uint8_t *rec, float *out, int tid, int s16) {
    using G = Geo<D>;
    const int g = tid / G::LANES, l = tid % G::LANES;
    const uint32_t codes_bytes = (uint32_t)D * D * B / 8;
    const uint8_t *rr = rec + codes_bytes;
    const uint8_t *cc = rr + D * (s16 ? 2 : 4);
    uint32_t W[Stream<D, B>::NW];
    load_stream<D, B>(rec, tid, W);
    const float4 c4 = scale4_at(cc, 4 * l, s16);
    const float2 c01 = make_float2(__fmul_rn(c4.x, 1.0f / 4096.0f), __fmul_rn(c4.y, 1.0f / 4096.0f));
    const float2 c23 = make_float2(__fmul_rn(c4.z, 1.0f / 4096.0f), __fmul_rn(c4.w, 1.0f / 4096.0f));
#pragma unroll
    for (int r = 0; r < G::RT; ++r) {
        const int i = g * G::RT + r;
        const float ri = scale_at(rr, i, s16);
        const float2 r2 = make_float2(ri, ri);
        const float2 A01 = mul2(r2, c01), A23 = mul2(r2, c23);
        const float2 z01 = make_float2(x_as_zscaled<B>(field_x<B>(W, 4 * r)), x_as_zscaled<B>(field_x<B>(W, 4 * r + 1)));
        const float2 z23 = make_float2(x_as_zscaled<B>(field_x<B>(W, 4 * r + 2)), x_as_zscaled<B>(field_x<B>(W, 4 * r + 3)));
        const float2 s01 = mul2(A01, z01), s23 = mul2(A23, z23);
        *reinterpret_cast<float4 *>(out + (size_t)i * D + 4 * l) = make_float4(s01.x, s01.y, s23.x, s23.y);
    }
}

template <int D>
__device__ void unpack_rows(const Args &a, const uint8_t *rec, float *out, int gl, int tid) {
    using G = Geo<D>;
    const int g = tid / G::LANES, l = tid % G::LANES;
    const uint32_t codes_bytes = a.t.codes_bytes[gl];
    const int s16 = a.scale16;
    const uint8_t *rr = rec + codes_bytes;
    const uint8_t *cc = rr + D * (s16 ? 2 : 4);
    const float4 c4 = scale4_at(cc, 4 * l, s16);
    const float2 c01 = make_float2(__fmul_rn(c4.x, 1.0f / 4096.0f), __fmul_rn(c4.y, 1.0f / 4096.0f));
    const float2 c23 = make_float2(__fmul_rn(c4.z, 1.0f / 4096.0f), __fmul_rn(c4.w, 1.0f / 4096.0f));
#pragma unroll
    for (int r = 0; r < G::RT; ++r) {
        const int i = g * G::RT + r;
        const int b = a.t.row_width[(size_t)gl * D + i];
        const uint8_t *row = rec + a.t.row_off[(size_t)gl * D + i];
        float2 s01, s23;
        if (b == kPivotBits) {
            const uint2 v = *reinterpret_cast<const uint2 *>(row + 8 * l);
            s01 = __half22float2(*reinterpret_cast<const __half2 *>(&v.x));
            s23 = __half22float2(*reinterpret_cast<const __half2 *>(&v.y));
        } else {
            const uint32_t f = row_field(row, b, l);
            const uint32_t mask = (1u << b) - 1u;
            const float zb = 8388608.0f + (float)(1 << (b - 1)) * 4096.0f;
            float z[4];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj)
                z[jj] = __fsub_rn(__uint_as_float((((f >> (b * jj)) & mask) << 12) | 0x4B000000u), zb);
            const float ri = scale_at(rr, i, s16);
            const float2 r2 = make_float2(ri, ri);
            s01 = mul2(mul2(r2, c01), make_float2(z[0], z[1]));
            s23 = mul2(mul2(r2, c23), make_float2(z[2], z[3]));
        }
        *reinterpret_cast<float4 *>(out + (size_t)i * D + 4 * l) = make_float4(s01.x, s01.y, s23.x, s23.y);
    }
}

template <int D>
__global__ void __launch_bounds__(2 * D) k_unpack(Args a) {
    using G = Geo<D>;
    const int tid = threadIdx.x;
    const int it = blockIdx.x;
    int n, ll, h, gl, row;
    item_coords<D>(a, it, n, ll, h, gl, row);
    const int slot = a.slots[n];
    if (slot < 0 || slot >= a.n_slots) {
        if (tid == 0) flag_error(a.err, kErrBadSlot);
        return;
    }
    const uint8_t *rec = a.pool + (uint64_t)slot * a.slot_bytes + a.t.rec_off[gl];
    float *out = a.S_out + (size_t)row * D * D;
    if (a.mode == 1) {
        unpack_rows<D>(a, rec, out, gl, tid);
        return;
    }
    switch (a.t.width[gl]) {
        case 2: unpack_uniform<D, 2>(rec, out, tid, a.scale16); break;
        case 4: unpack_uniform<D, 4>(rec, out, tid, a.scale16); break;
        case 6: unpack_uniform<D, 6>(rec, out, tid, a.scale16); break;
        case 8: unpack_uniform<D, 8>(rec, out, tid, a.scale16); break;
        case kPivotBits: {
            float2 S[G::RT][2];
            load_pivot<D>(rec, tid, S);
            const int g = tid / G::LANES, l = tid % G::LANES;
#pragma unroll
            for (int r = 0; r < G::RT; ++r)
                *reinterpret_cast<float4 *>(out + (size_t)(g * G::RT + r) * D + 4 * l) =
                    make_float4(S[r][0].x, S[r][0].y, S[r][1].x, S[r][1].y);
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
__device__ void dist_uniform(const float *Sg, int gl, int m, int n_bits, double *dist_acc, Scratch<D> &sc, int tid) {
    using G = Geo<D>;
    constexpr int RT = G::RT, LANES = G::LANES;
    constexpr int OFF = 1 << (B - 1);
    constexpr int Q = (1 << (B - 1)) - 1;
    constexpr float MG2 = kMagic + (float)OFF;
    const int g = tid / LANES, l = tid % LANES;
    const int j0 = 4 * l;
    float2 S[RT][2];
#pragma unroll
    for (int r = 0; r < RT; ++r) {
        const float4 v = *reinterpret_cast<const float4 *>(Sg + (size_t)(g * RT + r) * D + j0);
        S[r][0] = make_float2(v.x, v.y);
        S[r][1] = make_float2(v.z, v.w);
    }
    fit_scales<D, B, 0>(S, sc, tid, sc.rho, sc.wbar, nullptr, nullptr);
    float cc[4], icc[4];
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) { cc[jj] = sc.cold[j0 + jj]; icc[jj] = sc.ic[j0 + jj]; }
#pragma unroll
    for (int r = 0; r < RT; ++r) {
        const int i = g * RT + r;
        const float ri = sc.rowr[i];
        const float4 orig = *reinterpret_cast<const float4 *>(Sg + (size_t)i * D + j0);
        const float o4[4] = {orig.x, orig.y, orig.z, orig.w};
        const float y4[4] = {S[r][0].x, S[r][0].y, S[r][1].x, S[r][1].y};
        double e = 0.0;
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            const float t = __fmaf_rn(y4[jj], icc[jj], MG2);
            const float z = (float)((int)final_e<B>(t) - Q);
            const float sh = __fmul_rn(__fmul_rn(ri, cc[jj]), z);
            const double d = (double)sh - (double)o4[jj];
            e = fma(d, d, e);
        }
        e = lane_sum_f64<LANES>(e);
        if (l == (r % LANES)) atomicAdd(&dist_acc[((size_t)gl * D + i) * n_bits + m], e);
    }
}

template <int D>
__global__ void __launch_bounds__(2 * D) k_calib_dist(Args a, BitList bl, double *dist_acc) {
    extern __shared__ __align__(128) uint8_t smem[];
    Scratch<D> &sc = *reinterpret_cast<Scratch<D> *>(smem);
    const int tid = threadIdx.x;
    const int it = blockIdx.x;
    const int m = blockIdx.y;
    int n, ll, h, gl, row;
    item_coords<D>(a, it, n, ll, h, gl, row);
    if (tid < D) {
        const float wb = a.t.wbar[(size_t)gl * D + tid];
        sc.wbar[tid] = wb;
        sc.rho[tid] = (float)(1.0 / sqrt(sqrt((double)wb)));
    }
    if (tid == 0) sc.nz = a.neg_zero;
    __syncthreads();
    const float *Sg = a.S_in + (size_t)row * D * D;
    switch (bl.b[m]) {
        case 2: dist_uniform<D, 2>(Sg, gl, m, bl.n, dist_acc, sc, tid); break;
        case 4: dist_uniform<D, 4>(Sg, gl, m, bl.n, dist_acc, sc, tid); break;
        case 6: dist_uniform<D, 6>(Sg, gl, m, bl.n, dist_acc, sc, tid); break;
        case 8: dist_uniform<D, 8>(Sg, gl, m, bl.n, dist_acc, sc, tid); break;
        default: if (tid == 0) flag_error(a.err, kErrArgs); break;
    }
}

template <int D>
static cudaError_t launch_dist_d(const Args &a, const BitList &bl, double *acc, cudaStream_t st) {
    if (a.n_items <= 0) return cudaSuccess;
    const size_t smem = sizeof(Scratch<D>);
    cudaError_t e = cudaFuncSetAttribute(k_calib_dist<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k_calib_dist<D><<<dim3(a.n_items, bl.n), 2 * D, smem, st>>>(a, bl, acc);
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

// ---------------------------------------------------------------------------
// Host-side launchers (called by the C ABI in stepq_api.cpp).
// ---------------------------------------------------------------------------
template <int D>
static size_t step_smem(uint32_t stage_bytes) {
    return (size_t)kStages * stage_bytes + 64 + sizeof(Scratch<D>);
}

template <int D, int KIND>
static cudaError_t launch_step_d(Args a, int n_sms, cudaStream_t st, int *grid_out) {
    const size_t smem = step_smem<D>(a.stage_bytes);
    auto kern = a.mode == 1 ? (a.scale16 ? k_step<D, KIND, 1, 1> : k_step<D, KIND, 1, 0>)
                            : (a.scale16 ? k_step<D, KIND, 0, 1> : k_step<D, KIND, 0, 0>);
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

template <int KIND>
static cudaError_t launch_step_kind(int D, Args a, int n_sms, cudaStream_t st, int *grid) {
    switch (D) {
        case 16: return launch_step_d<16, KIND>(a, n_sms, st, grid);
        case 32: return launch_step_d<32, KIND>(a, n_sms, st, grid);
        case 64: return launch_step_d<64, KIND>(a, n_sms, st, grid);
        case 128: return launch_step_d<128, KIND>(a, n_sms, st, grid);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_step(int kind, int D, const Args &a, int n_sms, cudaStream_t st, int *grid) {
    switch (kind) {
        case kDecode: return launch_step_kind<kDecode>(D, a, n_sms, st, grid);
        case kFitPack: return launch_step_kind<kFitPack>(D, a, n_sms, st, grid);
        case kFused: return launch_step_kind<kFused>(D, a, n_sms, st, grid);
        default: return cudaErrorInvalidValue;
    }
}

template <int D>
static cudaError_t launch_pack_d(const Args &a, bool unpack, cudaStream_t st) {
    if (a.n_items <= 0) return cudaSuccess;
    if (unpack) {
        k_unpack<D><<<a.n_items, 2 * D, 0, st>>>(a);
    } else {
        const size_t smem = ((sizeof(Scratch<D>) + 127) / 128) * 128 + (a.mode == 1 ? (size_t)D * D * 2 : 0);
        cudaError_t e = cudaFuncSetAttribute(k_requant_pack<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        k_requant_pack<D><<<a.n_items, 2 * D, smem, st>>>(a);
    }
    return cudaGetLastError();
}

cudaError_t launch_pack(int D, const Args &a, bool unpack, cudaStream_t st) {
    switch (D) {
        case 16: return launch_pack_d<16>(a, unpack, st);
        case 32: return launch_pack_d<32>(a, unpack, st);
        case 64: return launch_pack_d<64>(a, unpack, st);
        case 128: return launch_pack_d<128>(a, unpack, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace stepq
