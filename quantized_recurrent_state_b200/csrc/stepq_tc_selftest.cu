// Self-test of the tcgen05 building blocks (stepq_tc.cuh): one CTA computes
//   D1 = A B1^T   (both operands K-major in shared memory, accumulator in tensor memory),
//   D2 = D1 B2^T  (A read from tensor memory where the first product left it),
//   D3 = A B2^T   (A written to tensor memory by tcgen05.st),
// with A [128][32], B1 [32][32], B2 [64][32].  Every wait is bounded; on a timeout the
// kernel sets the error word, waits once more (bounded) and frees its tensor memory.
#include "stepq_tc.cuh"

namespace stepq {
namespace {

constexpr int kM = 128, kK = 32, kN1 = 32, kN2 = 64;
constexpr uint32_t kCols = 256;        // D1 [0, 32), D2 [64, 128), D3 [128, 192), A copy [192, 224)
constexpr uint32_t kPolls = 1u << 22;

__device__ int g_tc_err;

struct TcSmem {
    alignas(128) float A[kM * kK];
    alignas(128) float B1[kN1 * kK];
    alignas(128) float B2[kN2 * kK];
    alignas(8) uint64_t bar[3];
    uint32_t taddr;
};

__global__ void __launch_bounds__(128, 1) k_tc_selftest(const float *A, const float *B1, const float *B2, float *D1,
                                                        float *D2, float *D3) {
    __shared__ TcSmem sm;
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    uint8_t *sa = reinterpret_cast<uint8_t *>(sm.A), *sb1 = reinterpret_cast<uint8_t *>(sm.B1),
            *sb2 = reinterpret_cast<uint8_t *>(sm.B2);
    for (int e = tid; e < kM * kK; e += 128)
        *reinterpret_cast<float *>(sa + tc::kmajor_off(e / kK, e % kK, kK)) = A[e];
    for (int e = tid; e < kN1 * kK; e += 128)
        *reinterpret_cast<float *>(sb1 + tc::kmajor_off(e / kK, e % kK, kK)) = B1[e];
    for (int e = tid; e < kN2 * kK; e += 128)
        *reinterpret_cast<float *>(sb2 + tc::kmajor_off(e / kK, e % kK, kK)) = B2[e];
    if (tid == 0)
        for (int b = 0; b < 3; ++b) tc::mbar_init(&sm.bar[b]);
    if (w == 0) tc::alloc(&sm.taddr, kCols);
    tc::fence_smem_to_async();
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = sm.taddr, quad = (uint32_t)(32 * w) << 16;
    {   // row 32 w + lane of A into columns [192, 224) of its lane
        uint32_t v[32];
        for (int k = 0; k < kK; ++k) v[k] = __float_as_uint(A[(32 * w + lane) * kK + k]);
        tc::st32(tmem + quad + 192, v);
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    if (tid == 0) {
        for (int kk = 0; kk < kK / 8; ++kk)
            tc::mma_ss(tmem, tc::kmajor_desc(tc::smem_addr(sa), kK, kk), tc::kmajor_desc(tc::smem_addr(sb1), kK, kk),
                       tc::idesc_tf32(kM, kN1), kk > 0);
        tc::commit(&sm.bar[0]);
        for (int kk = 0; kk < kK / 8; ++kk)
            tc::mma_ts(tmem + 128, tmem + 192 + 8 * kk, tc::kmajor_desc(tc::smem_addr(sb2), kK, kk),
                       tc::idesc_tf32(kM, kN2), kk > 0);
        tc::commit(&sm.bar[1]);
    }
    bool ok = tc::mbar_wait(&sm.bar[0], 0, kPolls);     // D1 complete
    tc::fence_before();
    ok = __syncthreads_and(ok);
    tc::fence_after();
    if (ok && tid == 0) {
        for (int kk = 0; kk < kK / 8; ++kk)
            tc::mma_ts(tmem + 64, tmem + 8 * kk, tc::kmajor_desc(tc::smem_addr(sb2), kK, kk), tc::idesc_tf32(kM, kN2),
                       kk > 0);
        tc::commit(&sm.bar[2]);
    }
    if (ok) ok = tc::mbar_wait(&sm.bar[1], 0, kPolls) && tc::mbar_wait(&sm.bar[2], 0, kPolls);
    if (ok) {
        tc::fence_after();
        const int m = 32 * w + lane;
        uint32_t v[32];
        tc::ld32(tmem + quad, v);
        for (int n = 0; n < kN1; ++n) D1[m * kN1 + n] = __uint_as_float(v[n]);
        for (int h = 0; h < 2; ++h) {
            tc::ld32(tmem + quad + 64 + 32 * h, v);
            for (int n = 0; n < 32; ++n) D2[m * kN2 + 32 * h + n] = __uint_as_float(v[n]);
            tc::ld32(tmem + quad + 128 + 32 * h, v);
            for (int n = 0; n < 32; ++n) D3[m * kN2 + 32 * h + n] = __uint_as_float(v[n]);
        }
    } else if (lane == 0) {
        atomicOr(&g_tc_err, 1);
    }
    tc::fence_before();
    if (!__syncthreads_and(ok)) {   // gave up: let whatever was issued finish (bounded), then free
        for (int b = 0; b < 3; ++b) tc::mbar_wait(&sm.bar[b], 0, kPolls);
        __syncthreads();
    }
    tc::fence_after();
    if (w == 0) tc::dealloc(tmem, kCols);
}

}  // namespace

// Runs the self-test kernel on the default stream and waits; *word receives the kernel's error
// word (1: a wait gave up).
cudaError_t run_tc_selftest(const float *A, const float *B1, const float *B2, float *D1, float *D2, float *D3,
                            int *word) {
    const int zero = 0;
    cudaError_t e = cudaMemcpyToSymbol(g_tc_err, &zero, sizeof zero);
    if (e != cudaSuccess) return e;
    k_tc_selftest<<<1, 128>>>(A, B1, B2, D1, D2, D3);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = cudaDeviceSynchronize()) != cudaSuccess) return e;
    return cudaMemcpyFromSymbol(word, g_tc_err, sizeof *word);
}

}  // namespace stepq
