// Pipeline pieces shared by the step kernels of both unit kinds: item
// coordinates, the 16-byte step descriptors, the staging of one item (the
// packed record, the input rows, the head's tables) into a shared-memory
// stage by 1-D bulk copies, and the tile-major code streams.
//
// STEPQuant paper digest (vibe-research), 方法-4: every decode step reads the
// packed record, updates, reads out and writes the record back before the
// next step reads it.
#pragma once

#include <cstddef>

#include "stepq_dev.cuh"

namespace stepq {

enum Kind { kDecode = 0, kFitPack = 1, kFused = 2 };

constexpr int kStages = 2;             // one item in flight while the other is worked on
constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23: fl(x + kMagic) - kMagic = rint(x), |x| < 2^22

// Words of one thread's (one tile's) code stream: RT rows x 4 columns of b-bit codes.
template <int D, int B>
struct Stream {
    static constexpr int RT = D / 8;
    static constexpr int WORDS = (RT * B + 7) / 8;  // 32-bit words (4 RT B bits, rounded up)
    static constexpr int NW = WORDS + 1;            // + guard word
    static constexpr int NCH = B / 2;               // chunks of RT bytes
};

// Load tile t's code stream (NCH chunks of RT bytes; chunk c of tile t at
// block byte (c NT + t) RT) into W.
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

// (request, layer in launch, head, global head index, input row) of item `it`
// in plain (request-major) order.
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
// way into descriptor ring entry e (cp.async, completion by group).
template <int D>
__device__ __forceinline__ void prefetch_desc(const Args &a, int it, uint4 *dring, int *dslot, int e) {
    int n, ll, di;
    step_coords<D>(a, it, n, ll, di);
    cp_async16(&dring[e], &a.t.desc[di]);
    cp_async4(&dslot[e], &a.slots[n]);
    cp_async_commit();
}

// Item metadata left in shared memory by issue_item.
enum Meta { kMetaSlot = 0, kMetaWidth, kMetaValid, kMetaCodes, kMetaRecLo, kMetaRecHi, kMetaRow };

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
    meta[kMetaSlot] = slot;
    meta[kMetaWidth] = (int)(dsc.w & 0xffu);
    meta[kMetaValid] = ok ? 1 : 0;
    meta[kMetaCodes] = (int)(dsc.w >> 8);
    meta[kMetaRecLo] = (int)(uint32_t)(uintptr_t)rec;
    meta[kMetaRecHi] = (int)(uint32_t)((uintptr_t)rec >> 32);
    meta[kMetaRow] = row;
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

// The staged item's per-item scalars {alpha (per-head records), beta}.
template <int D>
__device__ __forceinline__ const float *stage_ab(const Args &a, const uint8_t *stage) {
    return reinterpret_cast<const float *>(stage + a.rec_stage_bytes + 4 * kTailRw * D + D);
}

template <int D>
__device__ __forceinline__ const float *stage_tail(const Args &a, const uint8_t *stage) {
    return reinterpret_cast<const float *>(stage + a.rec_stage_bytes);
}

// Thread 0, on the error path: let every copy still in flight land before
// shared memory goes away (stage k's pending phase is `phase`, or the next
// one for the stages before s).
__device__ __forceinline__ void drain_copies(uint64_t *bars, int s, uint32_t phase, uint32_t polls) {
    cp_async_wait_all();
    for (int k = 0; k < kStages; ++k) mbar_wait_bounded(&bars[k], phase ^ (k < s ? 1u : 0u), polls);
}

}  // namespace stepq
