// Device-side helpers of libstepq: launch arguments, the bulk-copy pipeline
// (cp.async.bulk into shared memory, mbarrier completion, bounded waits),
// packed-code field extraction and packing, and pairwise reductions.
//
// Method: STEPQuant paper digest (vibe-research), 方法-3 (X_hat = r c z) and
// 方法-4 (fused read -> update -> readout; refit and packed writeback).  The
// arithmetic definitions are stated in include/stepq.h.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace stepq {

constexpr int kPivotBits = 16;
constexpr int kQuantDualAxis = 0;  // plan quantizer: STEPQuant row/column fit
constexpr int kQuantAbsmax = 1;    // plan quantizer: per-row absmax, c = 1
constexpr int kErrBadSlot = 1;
constexpr int kErrWait = 2;
constexpr int kErrArgs = 4;
// A tensor-memory kernel freed its columns although a product it had issued
// might still have been writing them (a bounded wait gave up): later results
// of that memory cannot be trusted; the context refuses further work.
constexpr int kErrTmemDrain = 16;

// Device copy of the plan tables.
struct Tables {
    const uint4 *desc;           // [L*H] {record offset lo, hi, staged record bytes (0 for an FP16
                                 //  head), head width | codes-block bytes << 8}: one 16-byte read
    const uint64_t *rec_off;     // [L*H] record offset inside a slot
    const uint32_t *rec_bytes;   // [L*H]
    const uint32_t *codes_bytes; // [L*H] bytes of the codes block
    const uint8_t *width;        // [L*H] mode 0 unit width (16 = pivot head)
    const uint8_t *row_width;    // [L*H*D] mode 1 row widths (else null)
    const uint32_t *row_off;     // [L*H*D] mode 1: (first word of the row's band block) << 11 | (stream bit of the row in its tile); else null
    const float *wbar;           // [L*H*D]
    const float *rho;            // [L*H*D]
};

struct Args {
    uint8_t *pool;
    uint64_t slot_bytes;
    const int32_t *slots;
    int n_slots;
    int n_req;
    int lb;   // first layer of the launch (absolute)
    int nL;   // layers in the launch
    int nL_in;  // layers in the layout of the input/output arrays
    int l_in0;  // index of layer lb inside that layout
    int H;
    int mode;
    int quantizer;           // kQuantDualAxis or kQuantAbsmax (per-head units)
    int scale16;             // 1: r and c stored as bfloat16 (else fp32)
    int n_items;             // n_req * nL * H
    uint64_t div_nreq;       // floor(2^64 / n_req) + 1 (0 when n_req == 1): n / n_req = umul64hi(n, div_nreq)
    uint64_t div_h;          // the same for H
    const float *q, *k, *v, *alpha, *beta;
    float *o;
    float *w;                // workspace (decode writes, fit-pack reads)
    const float *S_in;       // requant_pack input
    float *S_out;            // unpack output
    Tables t;
    int *err;
    uint32_t wait_polls;     // polls before a copy wait gives up (error kErrWait)
    uint32_t phantom_tx;     // extra expected bytes per stage that never arrive (0: none; timeout test)
    uint32_t stage_bytes;    // bytes of one pipeline stage
    uint32_t rec_stage_bytes;// bytes reserved for the record in a stage
};

// Tail of a pipeline stage (after the staged record), in 4-byte words of D:
// q, k, v, x (the w workspace), rho, wbar, the per-row alpha (per-row
// records), row byte offsets (per-row records), then D bytes of row widths
// and a 16-byte block {alpha (per-head records), beta}.
enum StageTail { kTailQ = 0, kTailK, kTailV, kTailX, kTailRho, kTailWbar, kTailAlpha, kTailRoff, kTailRw };

__host__ __device__ constexpr uint32_t stage_tail_bytes(int D) { return 4u * kTailRw * D + D + 16u; }

// ---------------------------------------------------------------------------
// PTX wrappers: mbarrier + 1-D bulk copy (no multicast).
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// global -> shared bulk copy; dst, src 16-byte aligned, bytes a multiple of 16
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// 4- and 16-byte asynchronous copies global -> shared (non-bulk).  Their
// completion is handed to an mbarrier (cp_async_mbar_arrive: an arrival
// that lands once every earlier cp.async of this thread has) or to a group
// (cp_async_commit / cp_async_wait_all).
__device__ __forceinline__ void cp_async4(void *dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_mbar_arrive(uint64_t *bar) {
    asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t phase) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(phase)
        : "memory");
    return ok != 0;
}

// Bounded wait: gives up after `limit` polls (each poll may suspend the
// thread for a hardware-chosen interval), so a lost copy cannot hang the GPU.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t phase, uint32_t limit = (1u << 22)) {
    for (uint32_t i = 0; i < limit; ++i)
        if (mbar_try_wait(bar, phase)) return true;
    return false;
}

// ---------------------------------------------------------------------------
// Packed fp32x2 arithmetic with an explicit round-to-nearest modifier.  The
// .rn form keeps ptxas from contracting a multiply into a following add, so
// every product and sum rounds exactly where the arithmetic definition says.
// ---------------------------------------------------------------------------

__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
    float2 d;
    asm("{\n .reg .b64 ra, rb, rd;\n mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n"
        " mul.rn.f32x2 rd, ra, rb;\n mov.b64 {%0, %1}, rd;\n}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

__device__ __forceinline__ float2 add2(float2 a, float2 b) {
    float2 d;
    asm("{\n .reg .b64 ra, rb, rd;\n mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n"
        " add.rn.f32x2 rd, ra, rb;\n mov.b64 {%0, %1}, rd;\n}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n .reg .b64 ra, rb, rc, rd;\n mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n"
        " mov.b64 rc, {%6, %7};\n fma.rn.f32x2 rd, ra, rb, rc;\n mov.b64 {%0, %1}, rd;\n}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

__device__ __forceinline__ void flag_error(int *err, int code) { atomicOr(err, code); }

// Scale storage: fp32, or bfloat16 (the top half of an fp32, RNE).
__device__ __forceinline__ float scale_at(const uint8_t *base, int i, int s16) {
    return s16 ? __uint_as_float((uint32_t)reinterpret_cast<const uint16_t *>(base)[i] << 16)
               : reinterpret_cast<const float *>(base)[i];
}

// Four consecutive scales from index j0 (a multiple of 4; base 8-byte aligned).
__device__ __forceinline__ float4 scale4_at(const uint8_t *base, int j0, int s16) {
    if (s16) {
        const uint2 v = *reinterpret_cast<const uint2 *>(base + 2 * j0);
        return make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u),
                           __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xffff0000u));
    }
    return *reinterpret_cast<const float4 *>(base + 4 * j0);
}

// x rounded to the stored scale precision.
__device__ __forceinline__ float scale_round(float x, int s16) {
    return s16 ? __uint_as_float((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(x)) << 16) : x;
}

// Store a scale already rounded by scale_round.
__device__ __forceinline__ void scale_put(uint8_t *base, int i, float x, int s16) {
    if (s16) reinterpret_cast<uint16_t *>(base)[i] = (uint16_t)(__float_as_uint(x) >> 16);
    else reinterpret_cast<float *>(base)[i] = x;
}

// n / d for n < 2^32 with m = div_magic(d): floor(n m / 2^64) differs from
// n / d by less than n / 2^64 < 1 / d, which cannot cross an integer.
__device__ __forceinline__ uint32_t fast_div(uint32_t n, uint64_t m) {
    return m ? (uint32_t)__umul64hi((unsigned long long)n, (unsigned long long)m) : n;
}

__host__ __forceinline__ uint64_t div_magic(uint32_t d) {
    if (d <= 1) return 0;
    return (uint64_t)(((unsigned __int128)1 << 64) / d) + 1;
}

}  // namespace stepq
