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
// rows [g RT, g RT + RT) (band g = (t / 4) % 8, RT = D/8) of columns
// [4 cb, 4 cb + 4) (cb = 4 (t / 32) + t % 4).  A warp therefore holds 16 whole
// value columns: every column reduction (u, o, the initial column factor and
// the two least-squares sums) runs over the 8 bands of a column group inside
// one warp (lanes xor 4, 8, 16), in the balanced tree of the band order; only the
// row sums cross warps (one shared-memory exchange, two block barriers per
// record).  The state lives in registers as row pairs: S[k][c] holds rows
// g RT + 2k and g RT + 2k + 1 of column 4 cb + c, so the even/odd row chains
// of the band order are the two halves of one packed fp32x2 accumulator.
//
// Persistent CTAs stream records through a ring of shared-memory stages
// filled by 1-D bulk copies (cp.async.bulk, completion on an mbarrier); the
// stage of a record is refilled right after the last block barrier that
// follows its last read.
#include "stepq_head.cuh"

namespace stepq {

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
    const int g = band_of(tid), cb = cblk_of(tid), lane = tid & 31, i0 = g * RT, j0 = 4 * cb;
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
    const int g = band_of(tid), lane = tid & 31, i0 = g * RT, j0 = 4 * cblk_of(tid);
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
    const int i0 = band_of(tid) * RT, j0 = 4 * cblk_of(tid);
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
    row_partials<D, QUANT>(S, sc, band_of(tid), cblk_of(tid));
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
        const int i0 = band_of(tid) * RT, j0 = 4 * cblk_of(tid);
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
    const int i0 = band_of(tid) * RT, j0 = 4 * cblk_of(tid);
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
            const int i0 = band_of(tid) * RT, j0 = 4 * cblk_of(tid);
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
    const int g = band_of(tid), lane = tid & 31, i0 = g * RT, j0 = 4 * cblk_of(tid);
    float2 S[NP][4];
    load_tile<D>(Sg, tid, S);
    row_partials<D, kQuantDualAxis>(S, sc, g, cblk_of(tid));
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
        // the row's other column blocks of this warp (lanes xor 1, 2)
        ea += __shfl_xor_sync(kFull, ea, 1);
        ea += __shfl_xor_sync(kFull, ea, 2);
        eb += __shfl_xor_sync(kFull, eb, 1);
        eb += __shfl_xor_sync(kFull, eb, 2);
        if ((lane & 3) == 0) {
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
