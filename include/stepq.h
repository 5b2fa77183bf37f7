/*
 * stepq.h -- C ABI of libstepq.so, the B200 (sm_100a) packed recurrent-state
 * decode step of STEPQuant.
 *
 * Source of the method: "STEPQuant: When and Where Errors Matter in
 * Delta-Rule Recurrent State Quantization", paper digest page
 * (vibe-research):
 *   - 背景与动机: one state S_t in R^{dk x dv} per (request, head), updated
 *     each decode step with the key, value and retention gate and read out
 *     with the query; E_t = A_t E_{t-1} + eps_t;
 *   - 方法-1 Lifetime-aware Bit Allocation: per-unit widths {2,4,6,8} from an
 *     offline precision map, FP16 pivot units, a fixed average-bit budget;
 *   - 方法-2 Row-impact: omega_i = E[g_{t,i}^2], g_t = A_t^T q_t;
 *   - 方法-3 Key-Row-Aware Dual-Axis Fitting: X_hat_ij = r_i c_j z_ij;
 *   - 方法-4 per-step path: reconstruct the tile from codes, scales and FP16
 *     pivots -> retention + delta update + readout in floating point -> the
 *     readout goes on at once -> refit r and c -> pack -> asynchronous
 *     writeback before the next read, scale fitting on a separate stream.
 *
 * Arithmetic (the pages print no formulas for it; this library and its CPU
 * checker implement the same definitions independently):
 *   recurrence  S_t = (I - beta k k^T) Diag(alpha) S_{t-1} + beta k v^T,
 *               o_t = S_t^T q_t  (GDN: alpha scalar per head; KDA: per key row)
 *   decode      a_i = fl(alpha_i r_i);  S'_ij = fl(fl(a_i c_j) z_ij)
 *               (16-bit rows: S'_ij = fl(alpha_i h_ij))
 *               u_j = band_i(k_i S'_ij)
 *               w_j = fl(beta fl(v_j - u_j));  S_t,ij = fma(k_i, w_j, S'_ij)
 *               o_j = band_i(q_i S_t,ij)
 *   requantize  r_i = fl(max(pairwise_j |S_ij| / D, 1e-12) rho_i)
 *               y = fl(S fl(1/r));  c0_j = max_i fl(|y_ij| fl(1/qmax_i)) (0 -> 1)
 *               z0 = rint(y * fl(1/c0))   (exact product, ties to even)
 *               t_ij = fl(b_i z0_ij), b_i = fl(wbar_i fl(r_i r_i))
 *               c_j = fl(band_i(t_ij y_ij) / band_i(t_ij z0_ij)); a zero
 *                     denominator keeps c0
 *               z = clamp(rint(y * fl(1/c)), -qmax, qmax); 16-bit rows: fp16 RNE
 *   qmax(b) = 2^(b-1) - 1.  pairwise = fp32 sum in balanced binary-tree order.
 *   band_i(x_i y_i) = fp32 sum over the D rows in band order: 8 bands of D/8
 *     consecutive rows; in a band the even rows and the odd rows each form a
 *     chain acc = fma(x_i, y_i, acc) from +0, the band's value is the sum of
 *     the two chains, and the 8 band values are added in a balanced binary
 *     tree in band order.
 *
 * Packed format (decided offline, 方法-4 "fixed packed layout").  Codes are
 * stored offset-binary, u = z + 2^(b-1).
 *   per-head units (mode 0), width b in {2,4,6,8}: tile-major layout with
 *     RT = D/8, NT = 2D tiles: element (i,j) -> tile
 *     t = 32 (j/16) + 4 (i/RT) + (j/4)%4, tile code (r, c) = (i%RT, j%4); tile stream bits [(4r + c) b, +b), LSB first,
 *     except b = 6 with RT >= 4, where the rows of a tile go in groups of four
 *     over three 32-bit words (rows 0, 1, 3 of a group in bits [0, 24) of
 *     words 0, 1, 2 as 24-bit row values sum_c u_c 2^(6c); the 24-bit value of
 *     row 2 byte by byte in bits [24, 32) of the same words); stream byte B
 *     of tile t at block byte ((B/RT) NT + t) RT + B%RT.
 *   per-row units (mode 1): band-tile layout.  Band g = rows [g RT, g RT + RT),
 *     RT = D/8; tile (g, cb) = the band's rows x columns [4 cb, 4 cb + 4), NCB = D/4
 *     tiles per band.  A tile's stream holds, row after row, the row's four codes
 *     of b_r bits each (LSB first; a 16-bit row holds binary16 values): row r at
 *     stream bits [P_r, P_r + 4 b_r), P_r = 4 sum_{r'<r} b_r'.  Each tile takes
 *     NW_g = ceil(P_RT / 32) 32-bit words; band g's block starts at word
 *     W_g = NCB sum_{g'<g} NW_g', and stream word m of tile cb is word
 *     W_g + m NCB + (cb + 4 g) mod NCB of the codes block, little endian.
 *   record = codes | r[D] | c[D], zero-padded to 128 bytes, r and c fp32, or
 *     bfloat16 in plans with 16-bit scales (header word at byte 60 = 16: r_i
 *     is rounded to bfloat16, RNE, as soon as it is formed and used rounded
 *     from then on; c_j likewise after the refinement); a mode-0 pivot head's
 *     record is its binary16 tile, row-major, D*D*2 bytes.  Per-row units
 *     (mode 1) run on the device at D = 128 only (stepq_ctx_create).
 *   pool   = n_slots slots of slot_bytes each; inside a slot the records of
 *     (layer, head) follow layer-major (offsets: stepq_plan_record).
 *
 * Plan file: see the byte table in the implementation's plan parser
 * (magic "STEPQPL1", version 1, CRC-32 trailer); fields are listed with
 * stepq_plan_info.
 *
 * Conventions for every call:
 *   - Device pointers are plain CUDA device addresses on the context's
 *     device, owned by the caller; the library never frees them.  The
 *     library allocates only its plan tables, events and a 4-byte error
 *     word per context.
 *   - Alignment: pool 128 bytes; all other arrays 16 bytes.
 *   - q, k, v, o, workspace: [n_req][n_layers_launched][n_heads][D] fp32.
 *     alpha: mode 0 [n_req][nL][n_heads], mode 1 [n_req][nL][n_heads][D].
 *     beta: [n_req][nL][n_heads].  S (fp32 states): [n_req][nL][n_heads][D][D].
 *     slots: device int32[n_req], each in [0, n_slots) (a slot outside it sets
 *     the device error word and its records are skipped); the slots of one
 *     call must be distinct: two requests on one slot would update the same
 *     records concurrently (not checked, the array lives on the device).
 *   - Calls are asynchronous on the context's streams, except stepq_sync,
 *     the plan functions and stepq_last_error.
 *   - Return 0 (STEPQ_OK) or a negative STEPQ_E* code; stepq_last_error()
 *     gives a thread-local message.  No C++ exception crosses the ABI.
 *   - No CPU fallback: without a usable sm_100 device, calls that launch
 *     work return STEPQ_ECUDA.
 */
#ifndef STEPQ_H
#define STEPQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define STEPQ_OK 0
#define STEPQ_EINVAL (-1)    /* bad argument: null/misaligned pointer, range, dims */
#define STEPQ_EFORMAT (-2)   /* plan file malformed: magic, version, CRC, budget ... */
#define STEPQ_ECUDA (-3)     /* CUDA runtime error (message has the CUDA string) */
#define STEPQ_ETIMEDOUT (-4) /* stepq_sync gave up waiting */
#define STEPQ_EDEVICE (-5)   /* a kernel flagged a bad slot or a stalled copy */
#define STEPQ_ENOMEM (-6)    /* host allocation failed */

#define STEPQ_PIVOT_BITS 16

/* Requantizer of a plan (plan header word at byte 56).
 * STEPQ_QUANT_DUAL_AXIS: the STEPQuant row/column fit above (方法-3).
 * STEPQ_QUANT_ABSMAX: the ordinary per-row absmax baseline the pages compare
 *   against (实验: uniform INT4/INT6/INT8), per-head units only:
 *   r_i = fl(max_j |S_ij| / qmax) (1 for a zero row), z_ij = clamp(nearest
 *   integer, ties to even, to the exact S_ij * fl(1/r_i), +-qmax), c_j = 1;
 *   the record keeps the codes | r | c layout and decodes unchanged. */
#define STEPQ_QUANT_DUAL_AXIS 0
#define STEPQ_QUANT_ABSMAX 1

typedef struct stepq_plan stepq_plan; /* opaque, host-side plan */
typedef struct stepq_ctx stepq_ctx;   /* opaque, per device: tables, streams, events */

typedef struct stepq_plan_info {
    int mode;            /* 0 per-head units (GDN), 1 per-key-row units (KDA) */
    int n_layers;
    int n_heads;
    int d;               /* d_k == d_v: 16, 32, 64 or 128 */
    int n_units;         /* mode 0: n_layers*n_heads; mode 1: times d */
    int n_pivots;        /* units stored as FP16 */
    uint32_t bitset;     /* bit b set: width b allowed */
    float nominal_bits;  /* average-bit budget of the non-pivot units */
    uint64_t horizon;    /* H of the lifetime weight */
    uint64_t slot_bytes; /* bytes of one request's packed state */
    double bits_per_value;       /* codes + FP16 pivots + the plan's stored scales */
    double bits_per_value_s16;   /* the same with 16-bit scale accounting */
    int units_by_width[17];      /* histogram of unit widths (index = bits) */
    int quantizer;               /* STEPQ_QUANT_DUAL_AXIS or STEPQ_QUANT_ABSMAX */
    int scale_bits;              /* storage of r and c: 32 (fp32) or 16 (bfloat16) */
} stepq_plan_info;

/* ---- plan (方法-1 offline precision map) -------------------------------- */

/* Parse and validate a plan file.  Checks magic, version, CRC-32, dims, that
 * every width is allowed by the bitset or is 16, that the number of 16-bit
 * units equals n_pivots, that the non-pivot widths sum to at most
 * floor(nominal * N), and that wbar and rho are finite and positive.
 * Errors: STEPQ_EINVAL (null args, unreadable file), STEPQ_EFORMAT. */
int stepq_plan_load(const char *path, stepq_plan **out);
/* Same from a memory image of the file. */
int stepq_plan_load_mem(const void *data, size_t bytes, stepq_plan **out);
void stepq_plan_free(stepq_plan *plan);
int stepq_plan_get_info(const stepq_plan *plan, stepq_plan_info *out);
/* Copy the unit widths (n_units bytes: 2,4,6,8 or 16). */
int stepq_plan_widths(const stepq_plan *plan, uint8_t *out);
/* Byte offset inside a slot and size of the record of (layer, head). */
int stepq_plan_record(const stepq_plan *plan, int layer, int head, uint64_t *offset, uint64_t *bytes);

/* Build a plan from calibration statistics (方法-1): pivots are the top
 * n_pivots units by L_u * d_u(b_max) (ties to the lower index); the rest get
 * widths from `bits` (ascending, spaced by 2) minimising sum L_u d_u(b_u)
 * with sum b_u <= floor(nominal * N): multiple-choice DP for mode 0, the
 * Lagrangian with discrete repair for mode 1 (ties: smaller cost, then fewer
 * bits, then the lexicographically smaller width vector; Lagrangian ties to
 * the smaller width and the lower index).  L_u = sum_{j<H} exp(2 j l_u),
 * evaluated in closed form.
 *   lgate[n_units]            mean log retention gate l_u
 *   dist[n_units][n_bits]     distortion d_u(b) per allowed width
 *   wbar[n_layers*n_heads*d]  normalised row impact omega_i / mean omega
 * rho_i = fl32(1/sqrt(sqrt(wbar_i))) is derived.  scale_bits: 32 (fp32 r, c)
 * or 16 (bfloat16 r, c).  Host pointers.  Writes the plan file to `path`
 * (NULL: none) and returns the parsed plan in *out. */
int stepq_plan_build(int mode, int n_layers, int n_heads, int d, const int *bits, int n_bits,
                     float nominal_bits, int n_pivots, uint64_t horizon, const double *lgate,
                     const double *dist, const float *wbar, int scale_bits, const char *path,
                     stepq_plan **out);

/* A baseline plan (实验: uniform INT-b): every unit at width `bits` (2, 4, 6
 * or 8), no pivots, the given quantizer (STEPQ_QUANT_ABSMAX needs mode 0).
 * wbar[n_layers*n_heads*d] (host, NULL: all ones) feeds rho for the
 * dual-axis fit; lgate is 0 for every unit; scale_bits 32 or 16 as for
 * stepq_plan_build.  Writes the plan file to `path`
 * (NULL: none) and returns the parsed plan.  Errors: STEPQ_EINVAL. */
int stepq_plan_build_uniform(int mode, int n_layers, int n_heads, int d, int bits, int quantizer,
                             uint64_t horizon, const float *wbar, int scale_bits, const char *path,
                             stepq_plan **out);

/* The plan of layers [lb, le) of `plan` (a head- or layer-sharded pool: each
 * GPU holds the records of its own layers).  Units, wbar, rho, l_u and L_u
 * of those layers, the parent's mode, dims, bitset, horizon, requantizer and
 * scale storage; n_pivots counts the slice's FP16 units; nominal bits become
 * the slice's own average width (the parent's budget is global, not per
 * layer), the smallest float whose floor(nominal * N) covers the widths.
 * Errors: STEPQ_EINVAL. */
int stepq_plan_slice(const stepq_plan *plan, int lb, int le, stepq_plan **out);

/* ---- context ------------------------------------------------------------ */

/* Bind a plan to the current CUDA device (paper digest page, 方法-4: the
 * decode runs on one stream while scale fitting and packing run on a separate
 * one; the context holds those two streams, the device copy of the plan's
 * tables and the per-layer events that order them).  main/side are
 * cudaStream_t (NULL for the legacy default stream is rejected: pass real
 * streams).  n_slots is the capacity of every pool used with this context.
 * chunk_layers groups layers per launch pair in stepq_decode_step (<= 0: 4). */
int stepq_ctx_create(const stepq_plan *plan, void *main_stream, void *side_stream, int n_slots,
                     int chunk_layers, stepq_ctx **out);
void stepq_ctx_free(stepq_ctx *ctx);
/* Bytes of fp32 workspace stepq_decode_step needs for a launch of n_req
 * requests over nL layers (= n_req*nL*n_heads*d*4). */
size_t stepq_workspace_bytes(const stepq_ctx *ctx, int n_req, int n_layers_launched);

/* ---- prefill (the step before decode) ----------------------------------- */
/* Source: the STEPQuant project page, 快速上手 (the serving command prefills prompts in
 * chunks of 2,048 tokens), with the recurrence of the paper digest page, 背景与动机; the
 * chunk form below restates that recurrence over a block of tokens (no requantization
 * between tokens; the packed entry point requantizes the final state once). */

/* Chunked prefill of T tokens on fp32 states (d = 128, either unit kind):
 * for every (request, layer in [lb, le), head) the gated delta rule above,
 * token by token in meaning, S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1}
 * + beta_t k_t v_t^T and o_t = S_t^T q_t, evaluated in chunks of 64 tokens:
 * with Gamma_t the running gate product in the chunk (per key row for
 * per-row plans), (I + M) U = V - (K o Gamma) S_0 with M_ts = beta_s
 * sum_i k_ti k_si Gamma_ti/Gamma_si (s < t), O = (Q o Gamma) S_0 + L_incl(A) U
 * with A_ts = beta_s sum_i q_ti k_si Gamma_ti/Gamma_si, and S_C = Diag(Gamma_C)
 * S_0 + (K o (Gamma_C/Gamma) o beta)^T U.  The dense products run on the
 * tensor cores (TF32 with a TF32 remainder, near fp32), the triangular solve
 * in fp32; results match the token-by-token fp64 recurrence to the
 * tolerance stated in the tests, not bit for bit.
 *   S: [n_req][le-lb][n_heads][D][D] fp32, read (unless zero_init) and written.
 *   q, k, v, o: [n_req][T][le-lb][n_heads][D];  beta: [n_req][T][le-lb][n_heads];
 *   alpha: [n_req][T][le-lb][n_heads] for per-head plans, [..][n_heads][D]
 *   (16-byte aligned) for per-row plans; alpha in (0, 1] (its logarithm is
 *   taken).  Per-row gates are factored around the chunk's middle token, so
 *   they need the sum of |ln alpha_i| over any 32 consecutive tokens of a row
 *   below about 80 (any alpha >= 0.083 meets it); beyond that the fp32 gate
 *   factors overflow.  A gate outside (0, 1], or per-row gates beyond that
 *   range, set the context's device error word: the next stepq_sync returns
 *   STEPQ_EDEVICE ("prefill gate out of range") and the affected outputs are
 *   not valid.  Enqueued on main. */
int stepq_prefill_fp32(stepq_ctx *ctx, float *S, int n_req, int lb, int le, int T, const float *q,
                       const float *k, const float *v, const float *alpha, const float *beta, float *o,
                       int zero_init);
/* Which kernel the prefill of per-head plans runs (per-row plans always use the first):
 * STEPQ_PREFILL_TCGEN05 (default): the state in tensor memory as the A operand of K S
 *   and Q S and the accumulator of the update, those three products on tcgen05
 *   (kind::tf32, operands from shared memory), the rest on mma.sync;
 * STEPQ_PREFILL_MMA_SYNC: the chunk's products as mma.sync TF32 warp tiles, the state
 *   in shared memory; same results within the tolerance stated in the tests.
 * Applies to later calls. */
#define STEPQ_PREFILL_MMA_SYNC 0
#define STEPQ_PREFILL_TCGEN05 1
int stepq_ctx_set_prefill_kernel(stepq_ctx *ctx, int kernel);
/* Bytes of the fp32 workspace stepq_prefill needs for n_layers layers of the
 * batch (n_req * n_layers * n_heads * D * D * 4); 0 for a null context or a
 * negative count. */
size_t stepq_prefill_workspace_bytes(const stepq_ctx *ctx, int n_req, int n_layers);
/* Prefill into packed states: the pool records of (slots, layers [lb, le))
 * are unpacked into the workspace (from_zero: S_0 = 0 instead), prefilled as
 * in stepq_prefill_fp32, and requantized into the pool (the plan's
 * requantizer): three launches over the whole range.  The workspace, of
 * stepq_prefill_workspace_bytes(ctx, n_req, le - lb) bytes and owned by the
 * caller, holds the final fp32 states [n_req][le-lb][n_heads][D][D] on
 * return.  Same input layouts; enqueued on main after the side stream's last
 * work on those layers. */
int stepq_prefill(stepq_ctx *ctx, void *pool, const int32_t *slots, int n_req, int lb, int le, int T,
                  const float *q, const float *k, const float *v, const float *alpha, const float *beta,
                  float *o, float *workspace, int from_zero);

/* Pack fp32 states S into the pool records of (slots, layers [lb, le)):
 * the requantizer of the header comment (used for S_0).  Enqueued on main. */
int stepq_requant_pack(stepq_ctx *ctx, void *pool, const int32_t *slots, int n_req, int lb, int le,
                       const float *S);

/* ---- the decode step (方法-4) --------------------------------------------- */

/* One decode step over (slots, layers [lb, le), all heads), two streams:
 * per layer chunk, the decode kernel (reconstruct -> retention + delta ->
 * readout o, and w for the fit) runs on `main`, and the fit-and-pack kernel
 * (recompute S_t from the same record and w, refit r and c, pack, write the
 * record in place) runs on `side` after it.  Before reading a chunk, `main`
 * waits for the previous call's side work on the same layers.  o is valid on
 * `main` when the call returns (enqueue order); the pool is valid after
 * stepq_sync.  workspace: stepq_workspace_bytes() bytes. */
int stepq_decode_step(stepq_ctx *ctx, void *pool, const int32_t *slots, int n_req, int lb, int le,
                      const float *q, const float *k, const float *v, const float *alpha,
                      const float *beta, float *o, void *workspace);

/* The same step in one fused pass per record on `main` (no re-read of the
 * record, no workspace).  Results are bit-identical to stepq_decode_step. */
int stepq_decode_step_fused(stepq_ctx *ctx, void *pool, const int32_t *slots, int n_req, int lb,
                            int le, const float *q, const float *k, const float *v,
                            const float *alpha, const float *beta, float *o);

/* Which kernel stepq_decode_step_fused runs for per-head plans at d = 128 (other plans
 * always use the first; results are bit-identical):
 * STEPQ_STEP_REGISTERS: each thread keeps its 64 state values in registers between the
 *   passes over a record (two CTAs of 256 threads per SM);
 * STEPQ_STEP_TMEM: each thread keeps them in its own tensor-memory lane (128 columns per
 *   CTA, tcgen05.ld/st of 16 values at a time), which frees the registers for three CTAs
 *   per SM.  Applies to later calls. */
#define STEPQ_STEP_REGISTERS 0
#define STEPQ_STEP_TMEM 1
int stepq_ctx_set_step_kernel(stepq_ctx *ctx, int kernel);

/* Allocation-free variant of stepq_decode_step (the paper has no
 * counterpart; it exists for callers that cannot allocate device memory,
 * such as plugins whose host framework owns every allocation, or latency-
 * critical loops where an allocator call is not allowed).  The caller passes
 * the same inputs and outputs but no workspace: the w values the decode
 * kernel hands to the fit-and-pack kernel live in a fixed array of
 * STEPQ_NOALLOC_SCRATCH_BYTES inside the library, which every GPU that loads
 * the library holds until the process exits.  The call allocates nothing.
 *   - Limit: n_req * (le - lb) * n_heads * d * 4 bytes must not exceed
 *     STEPQ_NOALLOC_SCRATCH_BYTES; larger calls return STEPQ_EINVAL (split
 *     them, e.g. one layer range at a time).
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.  The address is looked up again when the
 *     device's current context is no longer the one it was looked up in
 *     (after a cudaDeviceReset, or a context made current through the driver
 *     API); a device reset also invalidates every stepq_ctx of that device,
 *     so create new contexts after one.
 *   - All calls on a device share the array and it keeps the last call's
 *     contents (nothing in it needs to start at zero: every value is written
 *     before it is read).  Before launching, the call makes `main` wait for
 *     all earlier side-stream (fit-and-pack) work of this context, on every
 *     layer and not only on [lb, le): unlike stepq_decode_step, a call does
 *     not overlap the previous call's fit-and-pack of other layers.  Calls
 *     from different contexts, threads or processes' streams that overlap on
 *     the GPU race on the array.
 * Results are bit-identical to stepq_decode_step. */
#define STEPQ_NOALLOC_SCRATCH_BYTES (8u << 20)
int stepq_decode_step_noalloc(stepq_ctx *ctx, void *pool, const int32_t *slots, int n_req, int lb, int le,
                              const float *q, const float *k, const float *v, const float *alpha,
                              const float *beta, float *o);

/* Wait for all work of the context (both streams) with a host-side timeout
 * (<= 0: wait without limit), then return the device error word:
 * STEPQ_OK, STEPQ_ETIMEDOUT, STEPQ_EDEVICE (the word is cleared) or ECUDA.
 * Paper digest page, 方法-4: the refitted, packed records are written back
 * asynchronously and must be complete before the next read; this is the
 * point where the host knows they are. */
int stepq_sync(stepq_ctx *ctx, int timeout_ms);

/* Reconstruct X_hat_ij = fl(fl(r_i c_j) z_ij) (16-bit rows: their value) into S
 * (paper digest page, 方法-3 Key-Row-Aware Dual-Axis Fitting: X_hat = r_i c_j z_ij). */
int stepq_unpack(stepq_ctx *ctx, const void *pool, const int32_t *slots, int n_req, int lb, int le,
                 float *S);

/* FP32-state reference step on an fp32 pool of [n_slots][n_layers][n_heads][D][D]:
 * the unquantized recurrence the pages set the packed state against (paper
 * digest page, 背景与动机 and 实验: the FP32 state pool), S'_ij =
 * fl(alpha_i S_ij), u_j = band_i(k_i S'_ij), w_j = fl(beta fl(v_j - u_j)),
 * S_ij = fma(k_i, w_j, S'_ij), o_j = band_i(q_i S_ij).  On main. */
int stepq_fp32_decode_step(stepq_ctx *ctx, float *S_pool, const int32_t *slots, int n_req, int lb,
                           int le, const float *q, const float *k, const float *v,
                           const float *alpha, const float *beta, float *o);

/* ---- calibration statistics on the device (方法-1, 方法-2) ---------------- */

/* Accumulate, for one calibration step, omega_acc[l][h][i] += g_i^2 with
 * g = alpha (.) (q - beta k (k^T q)) and lsum_acc[l][h][i] += log alpha_i,
 * over n_req requests and layers [lb, le).  Accumulators: device fp64
 * [n_layers][n_heads][d]. */
int stepq_calib_accumulate(stepq_ctx *ctx, int n_req, int lb, int le, const float *q,
                           const float *k, const float *alpha, const float *beta,
                           double *omega_acc, double *lsum_acc);
/* Accumulate dist_acc[l][h][i][m] += squared reconstruction error of row i
 * when head (l, h) of each fp32 state in S ([n_req][nL][H][D][D]) is
 * quantized at uniform width bits[m] with the row weights wbar (device fp32
 * [n_layers][n_heads][d]). */
int stepq_calib_distortion(stepq_ctx *ctx, int n_req, int lb, int le, const float *S,
                           const float *wbar, const int *bits, int n_bits, double *dist_acc);

/* ---- measurement -------------------------------------------------------- */

/* Plain device copy of `bytes` (multiple of 16, 16-byte aligned) on `stream`
 * (a cudaStream_t): the in-run HBM bandwidth probe. */
int stepq_copy_probe(void *dst, const void *src, size_t bytes, void *stream);

/* Number of kernel launches this context has issued so far. */
uint64_t stepq_launch_count(const stepq_ctx *ctx);

/* Kernel timing.  While enabled, every launch of the context is bracketed by
 * two CUDA events on the stream it runs on.  stepq_kernel_stats waits for
 * them, adds up the device time per kernel kind (0 decode, 1 fit-pack,
 * 2 fused, 3 pack/unpack/fp32/calibration, 4 chunked prefill), writes
 * ms[5] and launches[5] (host arrays) and forgets the recorded launches. */
int stepq_ctx_set_timing(stepq_ctx *ctx, int enable);
/* Bounded copy waits of the step kernels.  Every wait of a kernel on its
 * shared-memory copies gives up after `polls` polls of the barrier (0: the
 * default, 2^22), sets the device error word (stepq_sync then returns
 * STEPQ_EDEVICE, "copy wait gave up") and ends its block without touching
 * the pool.  phantom_bytes (< 65536, normally 0) adds bytes that never
 * arrive to every stage's expected count, so every wait runs out: the test
 * of that path.  Applies to later launches of the context. */
int stepq_ctx_set_wait_limit(stepq_ctx *ctx, uint32_t polls, uint32_t phantom_bytes);
int stepq_kernel_stats(stepq_ctx *ctx, double *ms, uint64_t *launches);

const char *stepq_last_error(void);

/* Self-test of the fifth-generation tensor-core path (tcgen05, kind::tf32) on this device:
 * one CTA computes D1 = A B1^T with both operands K-major in shared memory and the
 * accumulator in tensor memory, D2 = D1 B2^T with A read from tensor memory where the first
 * product left it, and D3 = A B2^T with A written to tensor memory by tcgen05.st.
 * A [128][32], B1 [32][32], B2 [64][32] (row-major fp32, device, 16-byte aligned);
 * D1 [128][32], D2 and D3 [128][64] (device, written).  The tensor cores read the fp32
 * operands truncated to TF32 (the low 13 mantissa bits are dropped).  Synchronous (default
 * stream); every wait is bounded: STEPQ_EDEVICE if one gave up, tensor memory freed. */
int stepq_selftest_tc(const float *A, const float *B1, const float *B2, float *D1, float *D2, float *D3);

#ifdef __cplusplus
}
#endif
#endif /* STEPQ_H */
