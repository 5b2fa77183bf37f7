// C ABI of libstepq (include/stepq.h): plan parsing and validation, the
// offline planner, per-device contexts (tables, streams, events, error word)
// and the launch sequencing of the decode step.
//
// STEPQuant paper digest (vibe-research): 方法-1 (precision map, pivots,
// budget, DP / Lagrangian allocation, bit/value accounting) and 方法-4
// (fused decode on one stream, scale fitting and packed writeback on a
// separate stream, finished before the next read).
#include <cuda_runtime.h>

#include <algorithm>
#include <chrono>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <limits>
#include <mutex>
#include <new>
#include <string>
#include <thread>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "../../include/stepq.h"
#include "stepq_dev.cuh"
#include "stepq_prefill.cuh"

namespace stepq {
cudaError_t launch_step(int kind, int D, const Args &a, int n_sms, cudaStream_t st, int *grid);
cudaError_t launch_pack(int D, const Args &a, bool unpack, cudaStream_t st);
cudaError_t launch_fp32_step(int D, const Args &a, float *S_pool, int n_layers_total, int n_sms, cudaStream_t st);
cudaError_t launch_copy(void *dst, const void *src, size_t bytes, int n_sms, cudaStream_t st);
cudaError_t launch_calib_acc(int D, const Args &a, double *om, double *ls, cudaStream_t st);
cudaError_t launch_calib_dist(int D, const Args &a, const int *bits, int n_bits, double *acc, cudaStream_t st);
cudaError_t launch_prefill(const PrefillArgs &a, cudaStream_t st);
cudaError_t launch_prefill_tc(const PrefillArgs &a, cudaStream_t st);
cudaError_t launch_step_tm(const Args &a, int n_sms, cudaStream_t st, int *grid);
cudaError_t run_tc_selftest(const float *A, const float *B1, const float *B2, float *D1, float *D2, float *D3,
                            int *word);
}  // namespace stepq

namespace {

thread_local std::string g_err;

int fail(int code, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return code;
}

int cuda_fail(cudaError_t e, const char *what) {
    return fail(STEPQ_ECUDA, "%s: %s", what, cudaGetErrorString(e));
}

// CRC-32 (IEEE 802.3, reflected polynomial 0xEDB88320).
uint32_t crc32(const uint8_t *p, size_t n) {
    static uint32_t table[256];
    static bool init = false;
    if (!init) {
        for (uint32_t i = 0; i < 256; ++i) {
            uint32_t c = i;
            for (int k = 0; k < 8; ++k) c = (c & 1) ? 0xEDB88320u ^ (c >> 1) : c >> 1;
            table[i] = c;
        }
        init = true;
    }
    uint32_t c = 0xFFFFFFFFu;
    for (size_t i = 0; i < n; ++i) c = table[(c ^ p[i]) & 0xFF] ^ (c >> 8);
    return c ^ 0xFFFFFFFFu;
}

inline uint64_t align_up(uint64_t x, uint64_t a) { return (x + a - 1) / a * a; }

template <class T>
T rd(const uint8_t *p) {
    T v;
    std::memcpy(&v, p, sizeof v);
    return v;
}

}  // namespace

// ---------------------------------------------------------------------------
// plan
// ---------------------------------------------------------------------------

// NVTX range around a public call (a no-op unless a profiler is attached).
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};

struct stepq_plan {
    int mode = 0, L = 0, H = 0, D = 0, n_units = 0, n_pivots = 0;
    int quantizer = 0;                // 0 dual-axis fit, 1 per-row absmax (mode 0)
    int scale_bits = 32;              // storage of r and c: 32 (fp32) or 16 (bfloat16)
    uint32_t bitset = 0;
    float nominal = 0.f;
    uint64_t horizon = 0;
    std::vector<uint8_t> width;       // [n_units]
    std::vector<float> wbar, rho;     // [L*H*D]
    std::vector<double> lgate, life;  // [n_units]
    // derived layout
    std::vector<uint64_t> rec_off;    // [L*H]
    std::vector<uint32_t> rec_bytes, codes_bytes;
    std::vector<uint8_t> head_width;  // [L*H] (mode 0: unit width; mode 1: 0)
    std::vector<uint8_t> row_width;   // [L*H*D] (mode 1)
    std::vector<uint32_t> row_off;    // [L*H*D] (mode 1)
    uint64_t slot_bytes = 0;
    double bpv = 0, bpv16 = 0;
};

/*
 * Plan file, little-endian:
 *   0  8 magic "STEPQPL1" | 8 u32 version=1 | 12 u32 mode | 16 u32 n_layers
 *   20 u32 n_heads | 24 u32 d_k | 28 u32 d_v | 32 u32 n_units | 36 u32 n_pivots
 *   40 u32 bitset | 44 f32 nominal bits | 48 u64 horizon | 56 u32 quantizer
 *   (0 dual-axis fit, 1 per-row absmax; mode 0 only) | 60 u32 scale storage
 *   (0: fp32 r and c, 16: bfloat16 r and c)
 *   64 u8 width[n_units], zero pad to 4 | f32 wbar[L*H*d] | f32 rho[L*H*d]
 *   f64 lgate[n_units] | f64 lifetime[n_units] | u32 CRC-32 of all before it
 */
static int plan_parse(const uint8_t *d, size_t n, stepq_plan *p) {
    if (n < 68) return fail(STEPQ_EFORMAT, "plan: %zu bytes is shorter than the header", n);
    if (std::memcmp(d, "STEPQPL1", 8) != 0) return fail(STEPQ_EFORMAT, "plan: bad magic");
    if (rd<uint32_t>(d + 8) != 1) return fail(STEPQ_EFORMAT, "plan: unsupported version %u", rd<uint32_t>(d + 8));
    const uint32_t crc = rd<uint32_t>(d + n - 4);
    if (crc != crc32(d, n - 4)) return fail(STEPQ_EFORMAT, "plan: CRC mismatch");
    p->mode = (int)rd<uint32_t>(d + 12);
    p->L = (int)rd<uint32_t>(d + 16);
    p->H = (int)rd<uint32_t>(d + 20);
    const uint32_t dk = rd<uint32_t>(d + 24), dv = rd<uint32_t>(d + 28);
    p->n_units = (int)rd<uint32_t>(d + 32);
    p->n_pivots = (int)rd<uint32_t>(d + 36);
    p->bitset = rd<uint32_t>(d + 40);
    p->nominal = rd<float>(d + 44);
    p->horizon = rd<uint64_t>(d + 48);
    p->quantizer = (int)rd<uint32_t>(d + 56);
    if (p->mode != 0 && p->mode != 1) return fail(STEPQ_EFORMAT, "plan: mode %d", p->mode);
    if (p->quantizer != 0 && !(p->quantizer == 1 && p->mode == 0))
        return fail(STEPQ_EFORMAT, "plan: quantizer %d with mode %d", p->quantizer, p->mode);
    const uint32_t sw = rd<uint32_t>(d + 60);
    if (sw != 0 && sw != 16) return fail(STEPQ_EFORMAT, "plan: scale storage word %u (0 or 16)", sw);
    p->scale_bits = sw == 16 ? 16 : 32;
    if (dk != dv) return fail(STEPQ_EFORMAT, "plan: d_k %u != d_v %u", dk, dv);
    if (dk != 16 && dk != 32 && dk != 64 && dk != 128) return fail(STEPQ_EFORMAT, "plan: d = %u unsupported", dk);
    p->D = (int)dk;
    if (p->L <= 0 || p->H <= 0 || p->L > 4096 || p->H > 4096) return fail(STEPQ_EFORMAT, "plan: bad layer/head counts");
    const uint64_t heads = (uint64_t)p->L * p->H;
    const uint64_t units = p->mode == 0 ? heads : heads * p->D;
    if ((uint64_t)p->n_units != units) return fail(STEPQ_EFORMAT, "plan: n_units %d != %llu", p->n_units, (unsigned long long)units);
    if (p->bitset & ~((1u << 2) | (1u << 4) | (1u << 6) | (1u << 8)))
        return fail(STEPQ_EFORMAT, "plan: bitset 0x%x allows widths outside {2,4,6,8}", p->bitset);
    if (!(p->nominal > 0.f) || !std::isfinite(p->nominal)) return fail(STEPQ_EFORMAT, "plan: bad nominal bits");
    const uint64_t nrow = heads * p->D;
    const uint64_t off_w = 64, off_f = align_up(off_w + units, 4);
    const uint64_t need = off_f + 8 * nrow + 16 * units + 4;
    if (n != need) return fail(STEPQ_EFORMAT, "plan: size %zu, expected %llu", n, (unsigned long long)need);
    p->width.assign(d + off_w, d + off_w + units);
    p->wbar.resize(nrow);
    p->rho.resize(nrow);
    std::memcpy(p->wbar.data(), d + off_f, 4 * nrow);
    std::memcpy(p->rho.data(), d + off_f + 4 * nrow, 4 * nrow);
    p->lgate.resize(units);
    p->life.resize(units);
    std::memcpy(p->lgate.data(), d + off_f + 8 * nrow, 8 * units);
    std::memcpy(p->life.data(), d + off_f + 8 * nrow + 8 * units, 8 * units);
    // widths, pivot count, budget
    int piv = 0;
    uint64_t bits_sum = 0, n_q = 0;
    for (uint64_t u = 0; u < units; ++u) {
        const int w = p->width[u];
        if (w == STEPQ_PIVOT_BITS) { ++piv; continue; }
        if (w > 8 || !((p->bitset >> w) & 1u)) return fail(STEPQ_EFORMAT, "plan: unit %llu has width %d outside the bitset", (unsigned long long)u, w);
        bits_sum += (uint64_t)w;
        ++n_q;
    }
    if (piv != p->n_pivots) return fail(STEPQ_EFORMAT, "plan: %d FP16 units but n_pivots = %d", piv, p->n_pivots);
    const uint64_t cap = (uint64_t)std::floor((double)p->nominal * (double)n_q);
    if (bits_sum > cap) return fail(STEPQ_EFORMAT, "plan: widths sum %llu exceed the budget %llu", (unsigned long long)bits_sum, (unsigned long long)cap);
    for (uint64_t i = 0; i < nrow; ++i)
        if (!(p->wbar[i] > 0.f) || !std::isfinite(p->wbar[i]) || !(p->rho[i] > 0.f) || !std::isfinite(p->rho[i]))
            return fail(STEPQ_EFORMAT, "plan: row weight %llu not finite and positive", (unsigned long long)i);
    // layout
    const int D = p->D;
    p->rec_off.resize(heads);
    p->rec_bytes.resize(heads);
    p->codes_bytes.resize(heads);
    p->head_width.assign(heads, 0);
    if (p->mode == 1) {
        p->row_width.assign(p->width.begin(), p->width.end());
        p->row_off.resize(nrow);
    }
    uint64_t off = 0;
    for (uint64_t hd = 0; hd < heads; ++hd) {
        uint64_t codes;
        uint64_t rec;
        if (p->mode == 0) {
            const int w = p->width[hd];
            p->head_width[hd] = (uint8_t)w;
            codes = (uint64_t)D * D * w / 8;
            rec = (w == STEPQ_PIVOT_BITS) ? align_up(codes, 128) : align_up(codes + 2ull * (p->scale_bits / 8) * D, 128);
        } else {
            // band-tile layout: band g's tiles take NW_g = ceil(4 sum_r b_r / 32) words each;
            // row_off = (first word of the band's block) << 11 | (stream bit of the row)
            const int RT = D / 8, NCB = D / 4;
            uint64_t words = 0;
            for (int g = 0; g < 8; ++g) {
                uint32_t bit = 0;
                for (int r = 0; r < RT; ++r) {
                    p->row_off[hd * D + g * RT + r] = (uint32_t)(words << 11) | bit;
                    bit += 4u * p->width[hd * D + g * RT + r];
                }
                words += (uint64_t)NCB * ((bit + 31) / 32);
            }
            codes = 4 * words;
            rec = align_up(codes + 2ull * (p->scale_bits / 8) * D, 128);
        }
        p->rec_off[hd] = off;
        p->codes_bytes[hd] = (uint32_t)codes;
        p->rec_bytes[hd] = (uint32_t)rec;
        off += rec;
    }
    p->slot_bytes = off;
    // bit/value: codes + FP16 pivots + scales (r per non-pivot row, c per head with one)
    double code_bits = 0, scale_rows = 0, scale_heads = 0;
    for (uint64_t hd = 0; hd < heads; ++hd) {
        int nonpiv_rows = 0;
        for (int i = 0; i < D; ++i) {
            const int w = p->mode == 0 ? p->width[hd] : p->width[hd * D + i];
            code_bits += (double)w * D;
            if (w != STEPQ_PIVOT_BITS) ++nonpiv_rows;
        }
        scale_rows += nonpiv_rows;
        if (nonpiv_rows) scale_heads += 1;
    }
    const double values = (double)heads * D * D;
    p->bpv = (code_bits + (double)p->scale_bits * (scale_rows + D * scale_heads)) / values;
    p->bpv16 = (code_bits + 16.0 * (scale_rows + D * scale_heads)) / values;
    return STEPQ_OK;
}

extern "C" int stepq_plan_load_mem(const void *data, size_t bytes, stepq_plan **out) {
    if (!data || !out) return fail(STEPQ_EINVAL, "plan_load_mem: null argument");
    stepq_plan *p = new (std::nothrow) stepq_plan;
    if (!p) return fail(STEPQ_ENOMEM, "plan_load_mem: out of memory");
    const int rc = plan_parse(static_cast<const uint8_t *>(data), bytes, p);
    if (rc != STEPQ_OK) {
        delete p;
        return rc;
    }
    *out = p;
    return STEPQ_OK;
}

extern "C" int stepq_plan_load(const char *path, stepq_plan **out) {
    if (!path || !out) return fail(STEPQ_EINVAL, "plan_load: null argument");
    FILE *f = std::fopen(path, "rb");
    if (!f) return fail(STEPQ_EINVAL, "plan_load: cannot open %s", path);
    std::vector<uint8_t> buf;
    uint8_t tmp[1 << 16];
    size_t n;
    while ((n = std::fread(tmp, 1, sizeof tmp, f)) > 0) buf.insert(buf.end(), tmp, tmp + n);
    std::fclose(f);
    return stepq_plan_load_mem(buf.data(), buf.size(), out);
}

extern "C" void stepq_plan_free(stepq_plan *plan) { delete plan; }

extern "C" int stepq_plan_get_info(const stepq_plan *p, stepq_plan_info *o) {
    if (!p || !o) return fail(STEPQ_EINVAL, "plan_get_info: null argument");
    std::memset(o, 0, sizeof *o);
    o->mode = p->mode;
    o->n_layers = p->L;
    o->n_heads = p->H;
    o->d = p->D;
    o->n_units = p->n_units;
    o->n_pivots = p->n_pivots;
    o->bitset = p->bitset;
    o->nominal_bits = p->nominal;
    o->horizon = p->horizon;
    o->slot_bytes = p->slot_bytes;
    o->bits_per_value = p->bpv;
    o->bits_per_value_s16 = p->bpv16;
    o->quantizer = p->quantizer;
    o->scale_bits = p->scale_bits;
    for (int w : p->width) o->units_by_width[w <= 16 ? w : 0]++;
    return STEPQ_OK;
}

extern "C" int stepq_plan_widths(const stepq_plan *p, uint8_t *out) {
    if (!p || !out) return fail(STEPQ_EINVAL, "plan_widths: null argument");
    std::memcpy(out, p->width.data(), p->width.size());
    return STEPQ_OK;
}

extern "C" int stepq_plan_record(const stepq_plan *p, int layer, int head, uint64_t *offset, uint64_t *bytes) {
    if (!p || !offset || !bytes) return fail(STEPQ_EINVAL, "plan_record: null argument");
    if (layer < 0 || layer >= p->L || head < 0 || head >= p->H) return fail(STEPQ_EINVAL, "plan_record: (%d, %d) out of range", layer, head);
    const size_t hd = (size_t)layer * p->H + head;
    *offset = p->rec_off[hd];
    *bytes = p->rec_bytes[hd];
    return STEPQ_OK;
}

// ---------------------------------------------------------------------------
// offline planner (方法-1)
// ---------------------------------------------------------------------------

namespace {

double lifetime_weight(double l, uint64_t H) {
    if (l == 0.0) return (double)H;
    return std::expm1(2.0 * (double)H * l) / std::expm1(2.0 * l);
}

// Multiple-choice DP over units, capacity in 2-bit steps above the smallest
// width; value (cost, bits) compared lexicographically; reconstruction takes
// the smallest width reaching the optimum at each unit.
bool dp_allocate(const std::vector<double> &cost, int N, const std::vector<int> &w, long long cap,
                 std::vector<int> &out) {
    const int M = (int)w.size();
    const int bmin = w[0];
    std::vector<int> st(M);
    for (int m = 0; m < M; ++m) st[m] = (w[m] - bmin) / 2;
    long long C = cap - (long long)bmin * N;
    if (C < 0) return false;
    C /= 2;
    C = std::min<long long>(C, (long long)st[M - 1] * N);
    const size_t W = (size_t)C + 1;
    std::vector<double> Vc((size_t)(N + 1) * W, 0.0);
    std::vector<long long> Vb((size_t)(N + 1) * W, 0);
    const double INF = std::numeric_limits<double>::infinity();
    for (int u = N - 1; u >= 0; --u) {
        double *bc = &Vc[(size_t)u * W];
        long long *bb = &Vb[(size_t)u * W];
        const double *nc = &Vc[(size_t)(u + 1) * W];
        const long long *nb = &Vb[(size_t)(u + 1) * W];
        for (size_t c = 0; c < W; ++c) {
            double best = INF;
            long long bestb = 0;
            for (int m = 0; m < M; ++m) {
                double cc = INF;
                long long cb = 0;
                if ((size_t)st[m] <= c) {
                    cc = cost[(size_t)u * M + m] + nc[c - st[m]];
                    cb = w[m] + nb[c - st[m]];
                }
                if (cc < best || (cc == best && cb < bestb)) {
                    best = cc;
                    bestb = cb;
                }
            }
            bc[c] = best;
            bb[c] = bestb;
        }
    }
    out.assign((size_t)std::max(N, 0), 0);
    size_t c = (size_t)C;
    for (int u = 0; u < N; ++u) {
        const double tc = Vc[(size_t)u * W + c];
        const long long tb = Vb[(size_t)u * W + c];
        bool found = false;
        for (int m = 0; m < M && !found; ++m) {
            if ((size_t)st[m] > c) continue;
            const double cc = cost[(size_t)u * M + m] + Vc[(size_t)(u + 1) * W + c - st[m]];
            const long long cb = w[m] + Vb[(size_t)(u + 1) * W + c - st[m]];
            if (cc == tc && cb == tb) {
                out[u] = w[m];
                c -= st[m];
                found = true;
            }
        }
        if (!found) return false;
    }
    return true;
}

void lagrange_choice(const std::vector<double> &cost, int N, const std::vector<int> &w, double lam,
                     std::vector<int> &b) {
    const int M = (int)w.size();
    b.resize(N);
    for (int u = 0; u < N; ++u) {
        int best = 0;
        double bv = cost[(size_t)u * M] + lam * (double)w[0];
        for (int m = 1; m < M; ++m) {
            const double v = cost[(size_t)u * M + m] + lam * (double)w[m];
            if (v < bv) { bv = v; best = m; }
        }
        b[u] = w[best];
    }
}

long long sum_bits(const std::vector<int> &b) {
    long long s = 0;
    for (int x : b) s += x;
    return s;
}

bool lagrangian_allocate(const std::vector<double> &cost, int N, const std::vector<int> &w, long long cap,
                         std::vector<int> &b) {
    const int M = (int)w.size();
    if ((long long)w[0] * N > cap) return false;
    lagrange_choice(cost, N, w, 0.0, b);
    if (sum_bits(b) > cap) {
        double lo = 0.0, hi = 1.0;
        std::vector<int> t;
        for (;;) {
            lagrange_choice(cost, N, w, hi, t);
            if (sum_bits(t) <= cap) break;
            hi *= 2.0;
        }
        for (int it = 0; it < 200; ++it) {
            const double mid = 0.5 * (lo + hi);
            lagrange_choice(cost, N, w, mid, t);
            if (sum_bits(t) <= cap) hi = mid;
            else lo = mid;
        }
        lagrange_choice(cost, N, w, hi, b);
    }
    std::vector<int> idx(N);
    for (int u = 0; u < N; ++u)
        for (int m = 0; m < M; ++m)
            if (w[m] == b[u]) idx[u] = m;
    long long slack = cap - sum_bits(b);
    while (slack >= 2) {
        int bu = -1;
        double bd = 0.0;
        for (int u = 0; u < N; ++u) {
            if (idx[u] + 1 >= M) continue;
            const double drop = cost[(size_t)u * M + idx[u]] - cost[(size_t)u * M + idx[u] + 1];
            if (drop > bd) { bd = drop; bu = u; }
        }
        if (bu < 0) break;
        idx[bu] += 1;
        b[bu] = w[idx[bu]];
        slack -= 2;
    }
    return true;
}

void put_u32(std::vector<uint8_t> &v, uint32_t x) { v.insert(v.end(), (uint8_t *)&x, (uint8_t *)&x + 4); }
void put_u64(std::vector<uint8_t> &v, uint64_t x) { v.insert(v.end(), (uint8_t *)&x, (uint8_t *)&x + 8); }

// The plan file image (format above); rho_i = fl32(1/sqrt(sqrt(wbar_i))).
std::vector<uint8_t> serialize_plan(int mode, int n_layers, int n_heads, int d, int n_pivots, uint32_t bitset,
                                    float nominal_bits, uint64_t horizon, int quantizer, int scale_bits,
                                    const std::vector<uint8_t> &width, const float *wbar, const double *lgate,
                                    const std::vector<double> &life) {
    const size_t heads = (size_t)n_layers * n_heads, nrow = heads * d, units = width.size();
    std::vector<uint8_t> f;
    f.insert(f.end(), (const uint8_t *)"STEPQPL1", (const uint8_t *)"STEPQPL1" + 8);
    put_u32(f, 1);
    put_u32(f, (uint32_t)mode);
    put_u32(f, (uint32_t)n_layers);
    put_u32(f, (uint32_t)n_heads);
    put_u32(f, (uint32_t)d);
    put_u32(f, (uint32_t)d);
    put_u32(f, (uint32_t)units);
    put_u32(f, (uint32_t)n_pivots);
    put_u32(f, bitset);
    uint32_t nb;
    std::memcpy(&nb, &nominal_bits, 4);
    put_u32(f, nb);
    put_u64(f, horizon);
    put_u32(f, (uint32_t)quantizer);
    put_u32(f, scale_bits == 16 ? 16u : 0u);
    f.insert(f.end(), width.begin(), width.end());
    while (f.size() % 4) f.push_back(0);
    const size_t off_wb = f.size();
    f.resize(off_wb + 8 * nrow);
    std::memcpy(&f[off_wb], wbar, 4 * nrow);
    for (size_t i = 0; i < nrow; ++i) {
        const float r = (float)(1.0 / std::sqrt(std::sqrt((double)wbar[i])));
        std::memcpy(&f[off_wb + 4 * nrow + 4 * i], &r, 4);
    }
    const size_t off_l = f.size();
    f.resize(off_l + 16 * units);
    std::memcpy(&f[off_l], lgate, 8 * units);
    std::memcpy(&f[off_l + 8 * units], life.data(), 8 * units);
    put_u32(f, crc32(f.data(), f.size()));
    return f;
}

int write_plan_file(const char *path, const std::vector<uint8_t> &f, const char *who) {
    if (!path) return STEPQ_OK;
    FILE *fp = std::fopen(path, "wb");
    if (!fp) return fail(STEPQ_EINVAL, "%s: cannot write %s", who, path);
    const size_t wr = std::fwrite(f.data(), 1, f.size(), fp);
    std::fclose(fp);
    if (wr != f.size()) return fail(STEPQ_EINVAL, "%s: short write to %s", who, path);
    return STEPQ_OK;
}

}  // namespace

extern "C" int stepq_plan_build(int mode, int n_layers, int n_heads, int d, const int *bits, int n_bits,
                                float nominal_bits, int n_pivots, uint64_t horizon, const double *lgate,
                                const double *dist, const float *wbar, int scale_bits, const char *path,
                                stepq_plan **out) {
    if (!bits || !lgate || !dist || !wbar || !out) return fail(STEPQ_EINVAL, "plan_build: null argument");
    if (scale_bits != 16 && scale_bits != 32) return fail(STEPQ_EINVAL, "plan_build: scale_bits %d", scale_bits);
    if (mode != 0 && mode != 1) return fail(STEPQ_EINVAL, "plan_build: mode %d", mode);
    if (n_layers <= 0 || n_heads <= 0 || (d != 16 && d != 32 && d != 64 && d != 128))
        return fail(STEPQ_EINVAL, "plan_build: bad dims");
    if (n_bits < 1 || n_bits > 4) return fail(STEPQ_EINVAL, "plan_build: n_bits %d", n_bits);
    std::vector<int> w(bits, bits + n_bits);
    std::sort(w.begin(), w.end());
    uint32_t bitset = 0;
    for (int m = 0; m < n_bits; ++m) {
        if (w[m] != 2 && w[m] != 4 && w[m] != 6 && w[m] != 8) return fail(STEPQ_EINVAL, "plan_build: width %d", w[m]);
        if (m && w[m] != w[m - 1] + 2) return fail(STEPQ_EINVAL, "plan_build: widths must be spaced by 2");
        bitset |= 1u << w[m];
    }
    const int heads = n_layers * n_heads;
    const int units = mode == 0 ? heads : heads * d;
    if (n_pivots < 0 || n_pivots > units) return fail(STEPQ_EINVAL, "plan_build: n_pivots %d", n_pivots);
    const int M = n_bits;
    std::vector<double> life(units);
    for (int u = 0; u < units; ++u) life[u] = lifetime_weight(lgate[u], horizon);
    // pivots: top n_pivots by L_u d_u(b_max), ties to the lower index
    std::vector<int> order(units);
    for (int u = 0; u < units; ++u) order[u] = u;
    std::vector<double> score(units);
    for (int u = 0; u < units; ++u) score[u] = life[u] * dist[(size_t)u * M + (M - 1)];
    std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return score[a] > score[b]; });
    std::vector<uint8_t> width(units, 0);
    for (int i = 0; i < n_pivots; ++i) width[order[i]] = STEPQ_PIVOT_BITS;
    std::vector<int> keep;
    for (int u = 0; u < units; ++u)
        if (width[u] != STEPQ_PIVOT_BITS) keep.push_back(u);
    const int N = (int)keep.size();
    std::vector<double> cost((size_t)N * M);
    for (int k = 0; k < N; ++k)
        for (int m = 0; m < M; ++m) cost[(size_t)k * M + m] = life[keep[k]] * dist[(size_t)keep[k] * M + m];
    const long long cap = (long long)std::floor((double)nominal_bits * (double)N);
    std::vector<int> alloc;
    const bool ok = mode == 0 ? dp_allocate(cost, N, w, cap, alloc) : lagrangian_allocate(cost, N, w, cap, alloc);
    if (!ok) return fail(STEPQ_EINVAL, "plan_build: budget %lld below the smallest width", cap);
    for (int k = 0; k < N; ++k) width[keep[k]] = (uint8_t)alloc[k];
    const std::vector<uint8_t> f = serialize_plan(mode, n_layers, n_heads, d, n_pivots, bitset, nominal_bits, horizon,
                                                  0, scale_bits, width, wbar, lgate, life);
    if (int rc = write_plan_file(path, f, "plan_build")) return rc;
    return stepq_plan_load_mem(f.data(), f.size(), out);
}

extern "C" int stepq_plan_build_uniform(int mode, int n_layers, int n_heads, int d, int bits, int quantizer,
                                        uint64_t horizon, const float *wbar, int scale_bits, const char *path,
                                        stepq_plan **out) {
    if (!out) return fail(STEPQ_EINVAL, "plan_build_uniform: null argument");
    if (scale_bits != 16 && scale_bits != 32) return fail(STEPQ_EINVAL, "plan_build_uniform: scale_bits %d", scale_bits);
    if (mode != 0 && mode != 1) return fail(STEPQ_EINVAL, "plan_build_uniform: mode %d", mode);
    if (n_layers <= 0 || n_heads <= 0 || (d != 16 && d != 32 && d != 64 && d != 128))
        return fail(STEPQ_EINVAL, "plan_build_uniform: bad dims");
    if (bits != 2 && bits != 4 && bits != 6 && bits != 8) return fail(STEPQ_EINVAL, "plan_build_uniform: width %d", bits);
    if (quantizer != 0 && !(quantizer == 1 && mode == 0))
        return fail(STEPQ_EINVAL, "plan_build_uniform: quantizer %d with mode %d", quantizer, mode);
    const size_t heads = (size_t)n_layers * n_heads, nrow = heads * d, units = mode == 0 ? heads : nrow;
    std::vector<float> ones;
    if (!wbar) {
        ones.assign(nrow, 1.0f);
        wbar = ones.data();
    }
    const std::vector<uint8_t> width(units, (uint8_t)bits);
    const std::vector<double> lgate(units, 0.0);
    const std::vector<double> life(units, lifetime_weight(0.0, horizon));
    const std::vector<uint8_t> f = serialize_plan(mode, n_layers, n_heads, d, 0, 1u << bits, (float)bits, horizon,
                                                  quantizer, scale_bits, width, wbar, lgate.data(), life);
    if (int rc = write_plan_file(path, f, "plan_build_uniform")) return rc;
    return stepq_plan_load_mem(f.data(), f.size(), out);
}

extern "C" int stepq_plan_slice(const stepq_plan *p, int lb, int le, stepq_plan **out) {
    if (!p || !out) return fail(STEPQ_EINVAL, "plan_slice: null argument");
    if (lb < 0 || le > p->L || lb >= le) return fail(STEPQ_EINVAL, "plan_slice: layers [%d, %d) of %d", lb, le, p->L);
    const size_t H = (size_t)p->H, D = (size_t)p->D;
    const size_t per_layer_units = p->mode == 0 ? H : H * D, per_layer_rows = H * D;
    const size_t u0 = (size_t)lb * per_layer_units, u1 = (size_t)le * per_layer_units;
    const std::vector<uint8_t> width(p->width.begin() + u0, p->width.begin() + u1);
    const std::vector<double> lgate(p->lgate.begin() + u0, p->lgate.begin() + u1);
    const std::vector<double> life(p->life.begin() + u0, p->life.begin() + u1);
    const std::vector<float> wbar(p->wbar.begin() + (size_t)lb * per_layer_rows, p->wbar.begin() + (size_t)le * per_layer_rows);
    int piv = 0;
    uint64_t bits = 0, n_q = 0;
    for (uint8_t w : width) {
        if (w == STEPQ_PIVOT_BITS) { ++piv; continue; }
        bits += w;
        ++n_q;
    }
    // the global budget is not a per-layer constraint: the slice carries its own average,
    // the smallest float whose floor(nominal * N) still covers its widths
    float nominal = p->nominal;
    if (n_q) {
        nominal = (float)((double)bits / (double)n_q);
        while ((uint64_t)std::floor((double)nominal * (double)n_q) < bits) nominal = std::nextafter(nominal, 1e30f);
    }
    const std::vector<uint8_t> f = serialize_plan(p->mode, le - lb, p->H, p->D, piv, p->bitset, nominal, p->horizon,
                                                  p->quantizer, p->scale_bits, width, wbar.data(), lgate.data(), life);
    return stepq_plan_load_mem(f.data(), f.size(), out);
}

// ---------------------------------------------------------------------------
// context
// ---------------------------------------------------------------------------

struct stepq_ctx {
    const stepq_plan *plan = nullptr;
    int device = 0, n_sms = 0, n_slots = 0, chunk = 4;
    cudaStream_t main = nullptr, side = nullptr;
    std::vector<cudaEvent_t> side_done;  // per layer
    std::vector<cudaEvent_t> dec_done;   // per chunk index
    cudaEvent_t ev_main = nullptr, ev_side = nullptr;
    int *err = nullptr;
    void *tables_mem = nullptr;
    stepq::Tables t{};
    std::vector<uint32_t> layer_max_rec;  // max non-pivot record bytes per layer
    uint64_t launches = 0;
    bool timing = false;
    uint32_t wait_polls = 1u << 22, phantom_tx = 0;
    int prefill_kernel = STEPQ_PREFILL_TCGEN05;
    int step_kernel = STEPQ_STEP_REGISTERS;
    bool poisoned = false;  // a tensor-memory drain failure was reported: refuse further work
    struct Timed { int kind; cudaEvent_t a, b; };
    std::vector<Timed> timed;
    std::vector<cudaEvent_t> ev_pool;
};

namespace {

int check_ptr(const void *p, size_t align, const char *name) {
    if (!p) return fail(STEPQ_EINVAL, "%s is null", name);
    if (reinterpret_cast<uintptr_t>(p) % align) return fail(STEPQ_EINVAL, "%s is not %zu-byte aligned", name, align);
    return STEPQ_OK;
}

int check_range(const stepq_ctx *c, int n_req, int lb, int le) {
    if (!c) return fail(STEPQ_EINVAL, "null context");
    if (c->poisoned)
        return fail(STEPQ_EDEVICE, "context unusable: a tensor-memory kernel freed columns a product may still have "
                                   "been writing (reported by an earlier stepq_sync); create a new context");
    if (n_req < 0) return fail(STEPQ_EINVAL, "n_req %d < 0", n_req);
    if (lb < 0 || le > c->plan->L || lb >= le) return fail(STEPQ_EINVAL, "layer range [%d, %d) outside [0, %d)", lb, le, c->plan->L);
    return STEPQ_OK;
}

int set_device(const stepq_ctx *c) {
    const cudaError_t e = cudaSetDevice(c->device);
    return e == cudaSuccess ? STEPQ_OK : cuda_fail(e, "cudaSetDevice");
}

stepq::Args base_args(stepq_ctx *c, void *pool, const int32_t *slots, int n_req, int lb, int le) {
    stepq::Args a{};
    a.pool = static_cast<uint8_t *>(pool);
    a.slot_bytes = c->plan->slot_bytes;
    a.slots = slots;
    a.n_slots = c->n_slots;
    a.n_req = n_req;
    a.lb = lb;
    a.nL = le - lb;
    a.nL_in = le - lb;
    a.l_in0 = 0;
    a.H = c->plan->H;
    a.mode = c->plan->mode;
    a.quantizer = c->plan->quantizer;
    a.wait_polls = c->wait_polls;
    a.phantom_tx = c->phantom_tx;
    a.scale16 = c->plan->scale_bits == 16 ? 1 : 0;
    a.n_items = n_req * (le - lb) * c->plan->H;
    a.div_nreq = stepq::div_magic((uint32_t)n_req);
    a.div_h = stepq::div_magic((uint32_t)c->plan->H);
    a.t = c->t;
    a.err = c->err;
    return a;
}

void set_stages(stepq_ctx *c, stepq::Args &a, int lb, int le) {
    uint32_t m = 128;
    for (int l = lb; l < le; ++l) m = std::max(m, c->layer_max_rec[l]);
    a.rec_stage_bytes = (uint32_t)align_up(m, 128);
    a.stage_bytes = a.rec_stage_bytes + (uint32_t)align_up(stepq::stage_tail_bytes(c->plan->D), 128);
}

cudaEvent_t take_event(stepq_ctx *c) {
    if (!c->ev_pool.empty()) {
        cudaEvent_t e = c->ev_pool.back();
        c->ev_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}

// Bracket one launch with timing events when timing is on.
struct LaunchTimer {
    stepq_ctx *c;
    int kind;
    cudaStream_t st;
    cudaEvent_t a = nullptr, b = nullptr;
    LaunchTimer(stepq_ctx *c_, int kind_, cudaStream_t st_) : c(c_), kind(kind_), st(st_) {
        if (c->timing) {
            a = take_event(c);
            b = take_event(c);
            cudaEventRecord(a, st);
        }
    }
    void done() {
        c->launches++;
        if (a && b) {
            cudaEventRecord(b, st);
            c->timed.push_back({kind, a, b});
        }
    }
};

// The tensor-memory prefill kernel serves per-head units; per-row plans keep the other one.
bool use_tc_prefill(const stepq_ctx *c) { return c->prefill_kernel == STEPQ_PREFILL_TCGEN05 && c->plan->mode == 0; }

int wait_side(stepq_ctx *c, int lb, int le) {
    for (int l = lb; l < le; ++l) {
        const cudaError_t e = cudaStreamWaitEvent(c->main, c->side_done[l], 0);
        if (e != cudaSuccess) return cuda_fail(e, "cudaStreamWaitEvent");
    }
    return STEPQ_OK;
}

}  // namespace

extern "C" int stepq_ctx_create(const stepq_plan *plan, void *main_stream, void *side_stream, int n_slots,
                                int chunk_layers, stepq_ctx **out) {
    if (!plan || !out) return fail(STEPQ_EINVAL, "ctx_create: null argument");
    if (!main_stream || !side_stream) return fail(STEPQ_EINVAL, "ctx_create: pass two real CUDA streams");
    if (main_stream == side_stream) return fail(STEPQ_EINVAL, "ctx_create: main and side streams must differ");
    if (n_slots <= 0) return fail(STEPQ_EINVAL, "ctx_create: n_slots %d", n_slots);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    cudaDeviceProp prop;
    e = cudaGetDeviceProperties(&prop, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDeviceProperties");
    if (prop.major < 10) return fail(STEPQ_ECUDA, "ctx_create: device %d is sm_%d%d; this library is built for sm_100a", dev, prop.major, prop.minor);
    if (plan->mode == 1 && plan->D != 128)
        return fail(STEPQ_EINVAL, "ctx_create: per-key-row plans run on the device at d = 128 only (d = %d)", plan->D);
    stepq_ctx *c = new (std::nothrow) stepq_ctx;
    if (!c) return fail(STEPQ_ENOMEM, "ctx_create: out of memory");
    c->plan = plan;
    c->device = dev;
    c->n_sms = prop.multiProcessorCount;
    c->n_slots = n_slots;
    c->chunk = chunk_layers > 0 ? chunk_layers : 4;
    c->main = static_cast<cudaStream_t>(main_stream);
    c->side = static_cast<cudaStream_t>(side_stream);
    const stepq_plan *p = plan;
    const size_t heads = (size_t)p->L * p->H, nrow = heads * p->D;
    const size_t sz_off = 8 * heads, sz_u32 = 4 * heads, sz_hw = align_up(heads, 16), sz_rw = align_up(p->mode == 1 ? nrow : 16, 16),
                 sz_ro = 4 * (p->mode == 1 ? nrow : 4), sz_f = 4 * nrow;
    const size_t sz_desc = 16 * heads;
    const size_t total = sz_desc + sz_off + 2 * sz_u32 + sz_hw + sz_rw + sz_ro + 2 * sz_f + 64 * 9;
    e = cudaMalloc(&c->tables_mem, total);
    if (e != cudaSuccess) { delete c; return cuda_fail(e, "cudaMalloc(tables)"); }
    uint8_t *m = static_cast<uint8_t *>(c->tables_mem);
    size_t o = 0;
    auto put = [&](const void *src, size_t bytes, size_t reserve) -> void * {
        void *dst = m + o;
        if (src && bytes) cudaMemcpy(dst, src, bytes, cudaMemcpyHostToDevice);
        o += align_up(reserve, 64);
        return dst;
    };
    // Step-kernel descriptors, one 16-byte read per item: per layer, the
    // heads in width order (per-head units; per-row units keep head order),
    // so concurrently running items mostly share one width's code path.
    // Entry: record offset low word, (offset bits 32..47) | head << 16,
    // staged record bytes (0 for an FP16 head), width | codes bytes << 8
    // (per-row units: 16 if the head has an FP16 row, else 0).
    if (p->slot_bytes >> 48) { cudaFree(c->tables_mem); delete c; return fail(STEPQ_EFORMAT, "ctx_create: slot above 2^48 bytes"); }
    std::vector<uint32_t> desc(4 * heads);
    for (int l = 0; l < p->L; ++l) {
        std::vector<int> order(p->H);
        for (int h = 0; h < p->H; ++h) order[h] = h;
        if (p->mode == 0)
            std::stable_sort(order.begin(), order.end(), [&](int x, int y) {
                return p->head_width[(size_t)l * p->H + x] < p->head_width[(size_t)l * p->H + y];
            });
        for (int k = 0; k < p->H; ++k) {
            const size_t hd = (size_t)l * p->H + order[k], e = 4 * ((size_t)l * p->H + k);
            const bool staged = !(p->mode == 0 && p->head_width[hd] == STEPQ_PIVOT_BITS);
            desc[e] = (uint32_t)p->rec_off[hd];
            desc[e + 1] = (uint32_t)((p->rec_off[hd] >> 32) & 0xffffu) | ((uint32_t)order[k] << 16);
            desc[e + 2] = staged ? p->rec_bytes[hd] : 0u;
            uint32_t wbyte = p->mode == 0 ? p->head_width[hd] : 0u;
            if (p->mode == 1)  // per-row units: 16 marks a head with FP16 rows (the step kernels' FP16 path)
                for (int i = 0; i < p->D; ++i)
                    if (p->row_width[hd * p->D + i] == STEPQ_PIVOT_BITS) wbyte = STEPQ_PIVOT_BITS;
            desc[e + 3] = wbyte | (p->codes_bytes[hd] << 8);
        }
    }
    c->t.desc = (const uint4 *)put(desc.data(), sz_desc, sz_desc);
    c->t.rec_off = (const uint64_t *)put(p->rec_off.data(), sz_off, sz_off);
    c->t.rec_bytes = (const uint32_t *)put(p->rec_bytes.data(), sz_u32, sz_u32);
    c->t.codes_bytes = (const uint32_t *)put(p->codes_bytes.data(), sz_u32, sz_u32);
    c->t.width = (const uint8_t *)put(p->head_width.data(), heads, sz_hw);
    c->t.row_width = (const uint8_t *)put(p->mode == 1 ? p->row_width.data() : nullptr, p->mode == 1 ? nrow : 0, sz_rw);
    c->t.row_off = (const uint32_t *)put(p->mode == 1 ? p->row_off.data() : nullptr, p->mode == 1 ? 4 * nrow : 0, sz_ro);
    c->t.wbar = (const float *)put(p->wbar.data(), sz_f, sz_f);
    c->t.rho = (const float *)put(p->rho.data(), sz_f, sz_f);
    e = cudaGetLastError();
    if (e != cudaSuccess || o > total) { cudaFree(c->tables_mem); delete c; return cuda_fail(e, "table upload"); }
    e = cudaMalloc(&c->err, sizeof(int));
    if (e == cudaSuccess) e = cudaMemset(c->err, 0, sizeof(int));
    if (e != cudaSuccess) { cudaFree(c->tables_mem); delete c; return cuda_fail(e, "cudaMalloc(error word)"); }
    c->side_done.resize(p->L);
    c->dec_done.resize(p->L);
    for (int l = 0; l < p->L && e == cudaSuccess; ++l) {
        e = cudaEventCreateWithFlags(&c->side_done[l], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c->dec_done[l], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventRecord(c->side_done[l], c->side);
    }
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c->ev_main, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c->ev_side, cudaEventDisableTiming);
    if (e != cudaSuccess) { stepq_ctx_free(c); return cuda_fail(e, "event creation"); }
    c->layer_max_rec.assign(p->L, 128);
    for (int l = 0; l < p->L; ++l)
        for (int h = 0; h < p->H; ++h) {
            const size_t hd = (size_t)l * p->H + h;
            if (p->mode == 0 && p->head_width[hd] == STEPQ_PIVOT_BITS) continue;
            c->layer_max_rec[l] = std::max(c->layer_max_rec[l], p->rec_bytes[hd]);
        }
    *out = c;
    return STEPQ_OK;
}

extern "C" void stepq_ctx_free(stepq_ctx *c) {
    if (!c) return;
    cudaSetDevice(c->device);
    if (c->main) cudaStreamSynchronize(c->main);
    if (c->side) cudaStreamSynchronize(c->side);
    for (auto &t : c->timed) { cudaEventDestroy(t.a); cudaEventDestroy(t.b); }
    for (auto ev : c->ev_pool) cudaEventDestroy(ev);
    for (auto ev : c->side_done) if (ev) cudaEventDestroy(ev);
    for (auto ev : c->dec_done) if (ev) cudaEventDestroy(ev);
    if (c->ev_main) cudaEventDestroy(c->ev_main);
    if (c->ev_side) cudaEventDestroy(c->ev_side);
    if (c->err) cudaFree(c->err);
    if (c->tables_mem) cudaFree(c->tables_mem);
    delete c;
}

extern "C" size_t stepq_workspace_bytes(const stepq_ctx *c, int n_req, int nL) {
    if (!c || n_req < 0 || nL < 0) return 0;
    return (size_t)n_req * nL * c->plan->H * c->plan->D * sizeof(float);
}

extern "C" uint64_t stepq_launch_count(const stepq_ctx *c) { return c ? c->launches : 0; }

// ---------------------------------------------------------------------------
// the step
// ---------------------------------------------------------------------------

extern "C" int stepq_requant_pack(stepq_ctx *c, void *pool, const int32_t *slots, int n_req, int lb, int le,
                                  const float *S) {
    NvtxRange nvtx_range("stepq_requant_pack");
    int rc = check_range(c, n_req, lb, le);
    if (rc) return rc;
    if ((rc = check_ptr(pool, 128, "pool")) || (rc = check_ptr(slots, 4, "slots")) || (rc = check_ptr(S, 16, "S"))) return rc;
    if ((rc = set_device(c))) return rc;
    if (n_req == 0) return STEPQ_OK;
    if ((rc = wait_side(c, lb, le))) return rc;
    stepq::Args a = base_args(c, pool, slots, n_req, lb, le);
    a.S_in = S;
    LaunchTimer lt(c, 3, c->main);
    const cudaError_t e = stepq::launch_pack(c->plan->D, a, false, c->main);
    if (e != cudaSuccess) return cuda_fail(e, "requant_pack launch");
    lt.done();
    return STEPQ_OK;
}

extern "C" int stepq_unpack(stepq_ctx *c, const void *pool, const int32_t *slots, int n_req, int lb, int le, float *S) {
    NvtxRange nvtx_range("stepq_unpack");
    int rc = check_range(c, n_req, lb, le);
    if (rc) return rc;
    if ((rc = check_ptr(pool, 128, "pool")) || (rc = check_ptr(slots, 4, "slots")) || (rc = check_ptr(S, 16, "S"))) return rc;
    if ((rc = set_device(c))) return rc;
    if (n_req == 0) return STEPQ_OK;
    if ((rc = wait_side(c, lb, le))) return rc;
    stepq::Args a = base_args(c, const_cast<void *>(pool), slots, n_req, lb, le);
    a.S_out = S;
    LaunchTimer lt(c, 3, c->main);
    const cudaError_t e = stepq::launch_pack(c->plan->D, a, true, c->main);
    if (e != cudaSuccess) return cuda_fail(e, "unpack launch");
    lt.done();
    return STEPQ_OK;
}

static int check_step_io(stepq_ctx *c, void *pool, const int32_t *slots, const float *q, const float *k,
                         const float *v, const float *alpha, const float *beta, float *o) {
    int rc;
    if ((rc = check_ptr(pool, 128, "pool")) || (rc = check_ptr(slots, 4, "slots")) || (rc = check_ptr(q, 16, "q")) ||
        (rc = check_ptr(k, 16, "k")) || (rc = check_ptr(v, 16, "v")) ||
        (rc = check_ptr(alpha, c->plan->mode == 1 ? 16 : 4, "alpha")) ||  // per-row alpha rows are bulk-copied
        (rc = check_ptr(beta, 4, "beta")) || (rc = check_ptr(o, 16, "o")))
        return rc;
    return STEPQ_OK;
}

extern "C" int stepq_decode_step(stepq_ctx *c, void *pool, const int32_t *slots, int n_req, int lb, int le,
                                 const float *q, const float *k, const float *v, const float *alpha,
                                 const float *beta, float *o, void *workspace) {
    NvtxRange nvtx_range("stepq_decode_step");
    int rc = check_range(c, n_req, lb, le);
    if (rc) return rc;
    if ((rc = check_step_io(c, pool, slots, q, k, v, alpha, beta, o))) return rc;
    if ((rc = check_ptr(workspace, 16, "workspace"))) return rc;
    if ((rc = set_device(c))) return rc;
    if (n_req == 0) return STEPQ_OK;
    for (int c0 = lb; c0 < le; c0 += c->chunk) {
        const int c1 = std::min(le, c0 + c->chunk);
        if ((rc = wait_side(c, c0, c1))) return rc;
        stepq::Args a = base_args(c, pool, slots, n_req, c0, c1);
        a.nL_in = le - lb;
        a.l_in0 = c0 - lb;
        a.q = q; a.k = k; a.v = v; a.alpha = alpha; a.beta = beta; a.o = o;
        a.w = static_cast<float *>(workspace);
        set_stages(c, a, c0, c1);
        LaunchTimer t0(c, 0, c->main);
        cudaError_t e = stepq::launch_step(0, c->plan->D, a, c->n_sms, c->main, nullptr);
        if (e != cudaSuccess) return cuda_fail(e, "decode launch");
        t0.done();
        cudaEvent_t ev = c->dec_done[c0];
        if ((e = cudaEventRecord(ev, c->main)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
        if ((e = cudaStreamWaitEvent(c->side, ev, 0)) != cudaSuccess) return cuda_fail(e, "cudaStreamWaitEvent");
        LaunchTimer t1(c, 1, c->side);
        e = stepq::launch_step(1, c->plan->D, a, c->n_sms, c->side, nullptr);
        if (e != cudaSuccess) return cuda_fail(e, "fit-pack launch");
        t1.done();
        for (int l = c0; l < c1; ++l)
            if ((e = cudaEventRecord(c->side_done[l], c->side)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
    }
    return STEPQ_OK;
}

extern "C" int stepq_decode_step_fused(stepq_ctx *c, void *pool, const int32_t *slots, int n_req, int lb, int le,
                                       const float *q, const float *k, const float *v, const float *alpha,
                                       const float *beta, float *o) {
    NvtxRange nvtx_range("stepq_decode_step_fused");
    int rc = check_range(c, n_req, lb, le);
    if (rc) return rc;
    if ((rc = check_step_io(c, pool, slots, q, k, v, alpha, beta, o))) return rc;
    if ((rc = set_device(c))) return rc;
    if (n_req == 0) return STEPQ_OK;
    if ((rc = wait_side(c, lb, le))) return rc;
    stepq::Args a = base_args(c, pool, slots, n_req, lb, le);
    a.q = q; a.k = k; a.v = v; a.alpha = alpha; a.beta = beta; a.o = o;
    set_stages(c, a, lb, le);
    LaunchTimer lt(c, 2, c->main);
    const cudaError_t e = (c->step_kernel == STEPQ_STEP_TMEM && c->plan->mode == 0 && c->plan->D == 128)
                              ? stepq::launch_step_tm(a, c->n_sms, c->main, nullptr)
                              : stepq::launch_step(2, c->plan->D, a, c->n_sms, c->main, nullptr);
    if (e != cudaSuccess) return cuda_fail(e, "fused launch");
    lt.done();
    return STEPQ_OK;
}

extern "C" int stepq_fp32_decode_step(stepq_ctx *c, float *S_pool, const int32_t *slots, int n_req, int lb, int le,
                                      const float *q, const float *k, const float *v, const float *alpha,
                                      const float *beta, float *o) {
    NvtxRange nvtx_range("stepq_fp32_decode_step");
    int rc = check_range(c, n_req, lb, le);
    if (rc) return rc;
    if ((rc = check_ptr(S_pool, 16, "S_pool")) || (rc = check_ptr(slots, 4, "slots")) || (rc = check_ptr(q, 16, "q")) ||
        (rc = check_ptr(k, 16, "k")) || (rc = check_ptr(v, 16, "v")) || (rc = check_ptr(alpha, 4, "alpha")) ||
        (rc = check_ptr(beta, 4, "beta")) || (rc = check_ptr(o, 16, "o")))
        return rc;
    if ((rc = set_device(c))) return rc;
    if (n_req == 0) return STEPQ_OK;
    stepq::Args a = base_args(c, nullptr, slots, n_req, lb, le);
    a.q = q; a.k = k; a.v = v; a.alpha = alpha; a.beta = beta; a.o = o;
    LaunchTimer lt(c, 3, c->main);
    const cudaError_t e = stepq::launch_fp32_step(c->plan->D, a, S_pool, c->plan->L, c->n_sms, c->main);
    if (e != cudaSuccess) return cuda_fail(e, "fp32 step launch");
    lt.done();
    return STEPQ_OK;
}

extern "C" int stepq_ctx_set_wait_limit(stepq_ctx *c, uint32_t polls, uint32_t phantom_bytes) {
    if (!c) return fail(STEPQ_EINVAL, "set_wait_limit: null context");
    if (phantom_bytes >= (1u << 16)) return fail(STEPQ_EINVAL, "set_wait_limit: phantom_bytes %u", phantom_bytes);
    c->wait_polls = polls ? polls : (1u << 22);
    c->phantom_tx = phantom_bytes;
    return STEPQ_OK;
}

extern "C" int stepq_ctx_set_step_kernel(stepq_ctx *c, int kernel) {
    if (!c) return fail(STEPQ_EINVAL, "set_step_kernel: null context");
    if (kernel != STEPQ_STEP_REGISTERS && kernel != STEPQ_STEP_TMEM)
        return fail(STEPQ_EINVAL, "set_step_kernel: kernel %d", kernel);
    c->step_kernel = kernel;
    return STEPQ_OK;
}

extern "C" int stepq_ctx_set_prefill_kernel(stepq_ctx *c, int kernel) {
    if (!c) return fail(STEPQ_EINVAL, "set_prefill_kernel: null context");
    if (kernel != STEPQ_PREFILL_MMA_SYNC && kernel != STEPQ_PREFILL_TCGEN05)
        return fail(STEPQ_EINVAL, "set_prefill_kernel: kernel %d", kernel);
    c->prefill_kernel = kernel;
    return STEPQ_OK;
}

extern "C" int stepq_sync(stepq_ctx *c, int timeout_ms) {
    if (!c) return fail(STEPQ_EINVAL, "sync: null context");
    int rc = set_device(c);
    if (rc) return rc;
    cudaError_t e = cudaEventRecord(c->ev_main, c->main);
    if (e == cudaSuccess) e = cudaEventRecord(c->ev_side, c->side);
    if (e != cudaSuccess) return cuda_fail(e, "sync: cudaEventRecord");
    const auto t0 = std::chrono::steady_clock::now();
    for (;;) {
        const cudaError_t a = cudaEventQuery(c->ev_main), b = cudaEventQuery(c->ev_side);
        if (a == cudaSuccess && b == cudaSuccess) break;
        if (a != cudaSuccess && a != cudaErrorNotReady) return cuda_fail(a, "sync: main stream");
        if (b != cudaSuccess && b != cudaErrorNotReady) return cuda_fail(b, "sync: side stream");
        if (timeout_ms > 0 &&
            std::chrono::duration_cast<std::chrono::milliseconds>(std::chrono::steady_clock::now() - t0).count() > timeout_ms)
            return fail(STEPQ_ETIMEDOUT, "sync: work still running after %d ms", timeout_ms);
        std::this_thread::sleep_for(std::chrono::microseconds(20));
    }
    int word = 0;
    e = cudaMemcpy(&word, c->err, sizeof word, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "sync: read error word");
    if (word) {
        cudaMemset(c->err, 0, sizeof(int));
        if (word & stepq::kErrTmemDrain) c->poisoned = true;
        return fail(STEPQ_EDEVICE, "device error word 0x%x (%s%s%s%s%s)", word,
                    (word & stepq::kErrBadSlot) ? "slot out of range " : "", (word & stepq::kErrWait) ? "copy wait gave up " : "",
                    (word & stepq::kErrArgs) ? "bad width " : "", (word & stepq::kErrGateRange) ? "prefill gate out of range " : "",
                    (word & stepq::kErrTmemDrain) ? "tensor memory freed with a product in flight (context now unusable) " : "");
    }
    return STEPQ_OK;
}

extern "C" int stepq_prefill_fp32(stepq_ctx *c, float *S, int n_req, int lb, int le, int T, const float *q,
                                  const float *k, const float *v, const float *alpha, const float *beta, float *o,
                                  int zero_init) {
    NvtxRange nvtx_range("stepq_prefill_fp32");
    int rc = check_range(c, n_req, lb, le);
    if (rc) return rc;
    if (c->plan->D != 128) return fail(STEPQ_EINVAL, "prefill: d = 128 only (d %d)", c->plan->D);
    if (T < 0) return fail(STEPQ_EINVAL, "prefill: T = %d", T);
    if ((rc = check_ptr(S, 16, "S")) || (rc = check_ptr(q, 16, "q")) || (rc = check_ptr(k, 16, "k")) ||
        (rc = check_ptr(v, 16, "v")) || (rc = check_ptr(alpha, c->plan->mode ? 16 : 4, "alpha")) ||
        (rc = check_ptr(beta, 4, "beta")) || (rc = check_ptr(o, 16, "o")))
        return rc;
    if ((rc = set_device(c))) return rc;
    if (n_req == 0 || T == 0) return STEPQ_OK;
    stepq::PrefillArgs a{};
    a.S = S; a.q = q; a.k = k; a.v = v; a.alpha = alpha; a.beta = beta; a.o = o;
    a.n_req = n_req; a.T = T; a.nL = le - lb; a.nL_in = le - lb; a.l_in0 = 0; a.H = c->plan->H;
    a.zero_init = zero_init ? 1 : 0;
    a.rows = c->plan->mode == 1;
    a.err = c->err;
    LaunchTimer lt(c, 4, c->main);
    const cudaError_t e = use_tc_prefill(c) ? stepq::launch_prefill_tc(a, c->main) : stepq::launch_prefill(a, c->main);
    if (e != cudaSuccess) return cuda_fail(e, "prefill launch");
    lt.done();
    return STEPQ_OK;
}

extern "C" size_t stepq_prefill_workspace_bytes(const stepq_ctx *c, int n_req, int n_layers) {
    if (!c || n_req < 0 || n_layers < 0) return 0;
    return (size_t)n_req * n_layers * c->plan->H * c->plan->D * c->plan->D * sizeof(float);
}

extern "C" int stepq_prefill(stepq_ctx *c, void *pool, const int32_t *slots, int n_req, int lb, int le, int T,
                             const float *q, const float *k, const float *v, const float *alpha, const float *beta,
                             float *o, float *workspace, int from_zero) {
    NvtxRange nvtx_range("stepq_prefill");
    int rc = check_range(c, n_req, lb, le);
    if (rc) return rc;
    if (c->plan->D != 128) return fail(STEPQ_EINVAL, "prefill: d = 128 only (d %d)", c->plan->D);
    if (T < 0) return fail(STEPQ_EINVAL, "prefill: T = %d", T);
    if ((rc = check_ptr(pool, 128, "pool")) || (rc = check_ptr(slots, 4, "slots")) || (rc = check_ptr(q, 16, "q")) ||
        (rc = check_ptr(k, 16, "k")) || (rc = check_ptr(v, 16, "v")) ||
        (rc = check_ptr(alpha, c->plan->mode ? 16 : 4, "alpha")) || (rc = check_ptr(beta, 4, "beta")) ||
        (rc = check_ptr(o, 16, "o")) || (rc = check_ptr(workspace, 16, "workspace")))
        return rc;
    if ((rc = set_device(c))) return rc;
    if (n_req == 0 || T == 0) return STEPQ_OK;
    if ((rc = wait_side(c, lb, le))) return rc;
    // the whole layer range at once (n_req * layers * H CTAs per launch): states -> fp32
    // workspace, the chunked prefill, requantize into the pool
    stepq::Args a = base_args(c, pool, slots, n_req, lb, le);
    cudaError_t e = cudaSuccess;
    if (!from_zero) {
        a.S_out = workspace;
        LaunchTimer lt(c, 3, c->main);
        e = stepq::launch_pack(c->plan->D, a, true, c->main);
        if (e != cudaSuccess) return cuda_fail(e, "prefill: unpack launch");
        lt.done();
    }
    stepq::PrefillArgs p{};
    p.S = workspace; p.q = q; p.k = k; p.v = v; p.alpha = alpha; p.beta = beta; p.o = o;
    p.n_req = n_req; p.T = T; p.nL = le - lb; p.nL_in = le - lb; p.l_in0 = 0; p.H = c->plan->H;
    p.zero_init = from_zero ? 1 : 0;
    p.rows = c->plan->mode == 1;
    p.err = c->err;
    {
        LaunchTimer lt(c, 4, c->main);
        e = use_tc_prefill(c) ? stepq::launch_prefill_tc(p, c->main) : stepq::launch_prefill(p, c->main);
        if (e != cudaSuccess) return cuda_fail(e, "prefill launch");
        lt.done();
    }
    a.S_in = workspace;
    LaunchTimer lt(c, 3, c->main);
    e = stepq::launch_pack(c->plan->D, a, false, c->main);
    if (e != cudaSuccess) return cuda_fail(e, "prefill: requant_pack launch");
    lt.done();
    return STEPQ_OK;
}

extern "C" int stepq_selftest_tc(const float *A, const float *B1, const float *B2, float *D1, float *D2, float *D3) {
    int rc;
    if ((rc = check_ptr(A, 16, "A")) || (rc = check_ptr(B1, 16, "B1")) || (rc = check_ptr(B2, 16, "B2")) ||
        (rc = check_ptr(D1, 16, "D1")) || (rc = check_ptr(D2, 16, "D2")) || (rc = check_ptr(D3, 16, "D3")))
        return rc;
    int word = 0;
    const cudaError_t e = stepq::run_tc_selftest(A, B1, B2, D1, D2, D3, &word);
    if (e != cudaSuccess) return cuda_fail(e, "selftest_tc");
    if (word) return fail(STEPQ_EDEVICE, "selftest_tc: a tensor-core wait gave up");
    return STEPQ_OK;
}

extern "C" int stepq_calib_accumulate(stepq_ctx *c, int n_req, int lb, int le, const float *q, const float *k,
                                      const float *alpha, const float *beta, double *omega_acc, double *lsum_acc) {
    int rc = check_range(c, n_req, lb, le);
    if (rc) return rc;
    if ((rc = check_ptr(q, 16, "q")) || (rc = check_ptr(k, 16, "k")) || (rc = check_ptr(alpha, 4, "alpha")) ||
        (rc = check_ptr(beta, 4, "beta")) || (rc = check_ptr(omega_acc, 8, "omega_acc")) || (rc = check_ptr(lsum_acc, 8, "lsum_acc")))
        return rc;
    if ((rc = set_device(c))) return rc;
    if (n_req == 0) return STEPQ_OK;
    stepq::Args a = base_args(c, nullptr, nullptr, n_req, lb, le);
    a.q = q; a.k = k; a.alpha = alpha; a.beta = beta;
    LaunchTimer lt(c, 3, c->main);
    const cudaError_t e = stepq::launch_calib_acc(c->plan->D, a, omega_acc, lsum_acc, c->main);
    if (e != cudaSuccess) return cuda_fail(e, "calib_accumulate launch");
    lt.done();
    return STEPQ_OK;
}

extern "C" int stepq_calib_distortion(stepq_ctx *c, int n_req, int lb, int le, const float *S, const float *wbar,
                                      const int *bits, int n_bits, double *dist_acc) {
    int rc = check_range(c, n_req, lb, le);
    if (rc) return rc;
    if ((rc = check_ptr(S, 16, "S")) || (rc = check_ptr(wbar, 4, "wbar")) || (rc = check_ptr(dist_acc, 8, "dist_acc"))) return rc;
    if (!bits || n_bits < 1 || n_bits > 4) return fail(STEPQ_EINVAL, "calib_distortion: bits");
    for (int m = 0; m < n_bits; ++m)
        if (bits[m] != 2 && bits[m] != 4 && bits[m] != 6 && bits[m] != 8) return fail(STEPQ_EINVAL, "calib_distortion: width %d", bits[m]);
    if ((rc = set_device(c))) return rc;
    if (n_req == 0) return STEPQ_OK;
    stepq::Args a = base_args(c, nullptr, nullptr, n_req, lb, le);
    a.S_in = S;
    a.t.wbar = wbar;
    LaunchTimer lt(c, 3, c->main);
    const cudaError_t e = stepq::launch_calib_dist(c->plan->D, a, bits, n_bits, dist_acc, c->main);
    if (e != cudaSuccess) return cuda_fail(e, "calib_distortion launch");
    lt.done();
    return STEPQ_OK;
}

extern "C" int stepq_copy_probe(void *dst, const void *src, size_t bytes, void *stream) {
    int rc;
    if ((rc = check_ptr(dst, 16, "dst")) || (rc = check_ptr(src, 16, "src"))) return rc;
    if (bytes % 16) return fail(STEPQ_EINVAL, "copy_probe: %zu bytes is not a multiple of 16", bytes);
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "copy_probe: device query");
    e = stepq::launch_copy(dst, src, bytes, sms, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? STEPQ_OK : cuda_fail(e, "copy_probe launch");
}

extern "C" int stepq_ctx_set_timing(stepq_ctx *c, int enable) {
    if (!c) return fail(STEPQ_EINVAL, "set_timing: null context");
    c->timing = enable != 0;
    return STEPQ_OK;
}

extern "C" int stepq_kernel_stats(stepq_ctx *c, double *ms, uint64_t *launches) {
    if (!c || !ms || !launches) return fail(STEPQ_EINVAL, "kernel_stats: null argument");
    int rc = set_device(c);
    if (rc) return rc;
    for (int k = 0; k < 5; ++k) { ms[k] = 0.0; launches[k] = 0; }
    for (auto &t : c->timed) {
        cudaError_t e = cudaEventSynchronize(t.b);
        if (e != cudaSuccess) return cuda_fail(e, "kernel_stats: cudaEventSynchronize");
        float dt = 0.f;
        e = cudaEventElapsedTime(&dt, t.a, t.b);
        if (e != cudaSuccess) return cuda_fail(e, "kernel_stats: cudaEventElapsedTime");
        ms[t.kind] += dt;
        launches[t.kind] += 1;
        c->ev_pool.push_back(t.a);
        c->ev_pool.push_back(t.b);
    }
    c->timed.clear();
    return STEPQ_OK;
}

extern "C" const char *stepq_last_error(void) { return g_err.c_str(); }

// ---------------------------------------------------------------------------
// Allocation-free variant of the two-stream step: the decode -> fit-pack
// hand-off values w live in a fixed device array owned by the library, for
// callers that cannot allocate device memory themselves.
// ---------------------------------------------------------------------------

static __device__ __align__(256) float g_noalloc_w[STEPQ_NOALLOC_SCRATCH_BYTES / sizeof(float)];

namespace {
std::mutex g_noalloc_mu;
constexpr int kMaxDevices = 128;
struct NoallocEntry {
    void *ctx = nullptr;  // the CUDA context the address belongs to
    float *addr = nullptr;
};
NoallocEntry g_noalloc[kMaxDevices];

// The driver's current context, read through the runtime's driver entry
// point (no link against the driver library).
void *current_cu_context() {
    using GetCurrent = int (*)(void **);
    static GetCurrent fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return static_cast<GetCurrent>(nullptr);
        return reinterpret_cast<GetCurrent>(p);
    }();
    void *ctx = nullptr;
    if (fn) fn(&ctx);
    return ctx;
}

// Device address of g_noalloc_w on the current device `dev` and its current
// context.  In host code the symbol is only a host-side stand-in; the address
// is looked up on the first call per device and again whenever the current
// context of that device is not the one it was looked up in (a device reset
// or a context made current through the driver API).
int noalloc_scratch(int dev, float **out) {
    if (dev < 0 || dev >= kMaxDevices) return fail(STEPQ_EINVAL, "decode_step_noalloc: device ordinal %d", dev);
    void *ctx = current_cu_context();
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    NoallocEntry &e = g_noalloc[dev];
    if (!e.addr || e.ctx != ctx) {
        void *p = nullptr;
        const cudaError_t err = cudaGetSymbolAddress(&p, g_noalloc_w);
        if (err != cudaSuccess) return cuda_fail(err, "decode_step_noalloc: cudaGetSymbolAddress");
        e.addr = static_cast<float *>(p);
        e.ctx = ctx;
    }
    *out = e.addr;
    return STEPQ_OK;
}
}  // namespace

extern "C" int stepq_decode_step_noalloc(stepq_ctx *c, void *pool, const int32_t *slots, int n_req, int lb, int le,
                                         const float *q, const float *k, const float *v, const float *alpha,
                                         const float *beta, float *o) {
    NvtxRange nvtx_range("stepq_decode_step_noalloc");
    int rc = check_range(c, n_req, lb, le);
    if (rc) return rc;
    if ((rc = check_step_io(c, pool, slots, q, k, v, alpha, beta, o))) return rc;
    const size_t need = stepq_workspace_bytes(c, n_req, le - lb);
    if (need > STEPQ_NOALLOC_SCRATCH_BYTES)
        return fail(STEPQ_EINVAL,
                    "decode_step_noalloc: this call needs %zu bytes of scratch, more than the built-in %u bytes; "
                    "split it into calls over fewer requests or layers",
                    need, (unsigned)STEPQ_NOALLOC_SCRATCH_BYTES);
    if ((rc = set_device(c))) return rc;
    if (n_req == 0) return STEPQ_OK;
    float *scratch = nullptr;
    if ((rc = noalloc_scratch(c->device, &scratch))) return rc;
    // every earlier fit-pack of this context may still read the shared array
    if ((rc = wait_side(c, 0, c->plan->L))) return rc;
    return stepq_decode_step(c, pool, slots, n_req, lb, le, q, k, v, alpha, beta, o, scratch);
}
