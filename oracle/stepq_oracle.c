/*
 * STEPQuant CPU oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * Only tests/, __graft_entry__.smoke() and the cpu_baseline leg of bench.py
 * may load this file's library.  The product path (libstepq.so) shares no
 * code with it: both sides implement the arithmetic and the packed format
 * from the written definition, each on its own.
 *
 * Source: "STEPQuant: When and Where Errors Matter in Delta-Rule Recurrent
 * State Quantization" (paper digest page, vibe-research), sections
 * "背景与动机" (the state S_t in R^{dk x dv}, update with key/value/gate,
 * readout with the query; error recursion E_t = A_t E_{t-1} + eps_t),
 * "方法-3 Key-Row-Aware Dual-Axis Fitting" (X_hat = r_i c_j z_ij) and
 * "方法-4 每个 decode step 的执行路径" (reconstruct -> retention + delta +
 * readout -> refit r, c -> pack).  The update formula, the quantizer formulas
 * and the numeric precision are not printed on the pages; the readings used
 * here are stated beside each function.
 *
 * Build: gcc -O2 -ffp-contract=off -fno-fast-math -shared -fPIC
 * (no contraction: every fp32 operation below rounds exactly where written).
 *
 * Parity status of each function is stated in its comment.  Functions not
 * marked otherwise are pinned by tests/test_oracle_*.py.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define SQ_PIVOT_BITS 16

/* ------------------------------------------------------------------------ */
/* IEEE 754 binary16 <-> binary32, written from the format definition       */
/* (1 sign bit, 5 exponent bits with bias 15, 10 fraction bits).             */
/* Pivot units are stored in FP16 ("方法-1": FP16 pivots).                    */
/* ------------------------------------------------------------------------ */

float sq_f16_to_f32(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);                 /* subnormal: f * 2^-24 */
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + f), e - 25);     /* (1 + f/1024) * 2^(e-15) */
    return (float)(sign ? -v : v);
}

/* Round-to-nearest-even conversion; overflow goes to +-inf. */
uint16_t sq_f32_to_f16(float x)
{
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs((double)x);
    if (isnan(x)) return 0x7e00;
    if (a == 0.0) return sign;
    /* quantum of the binade that holds a (subnormal range uses 2^-24) */
    int ex;
    frexp(a, &ex);                 /* a = m * 2^ex, m in [0.5, 1) */
    int e = ex - 1;                /* a in [2^e, 2^(e+1)) */
    if (e < -14) e = -14;          /* subnormal quantum */
    double q = ldexp(1.0, e - 10);
    double n = a / q;              /* exact: power-of-two scaling */
    double fl = floor(n);
    double rem = n - fl;
    if (rem > 0.5 || (rem == 0.5 && fmod(fl, 2.0) != 0.0)) fl += 1.0;
    double r = fl * q;
    if (r >= 65520.0 || r > 65504.0) return sign | 0x7c00;
    /* encode r */
    if (r < ldexp(1.0, -14)) {
        int f = (int)(r / ldexp(1.0, -24));
        return sign | (uint16_t)f;
    }
    frexp(r, &ex);
    e = ex - 1;
    int f = (int)(r / ldexp(1.0, e - 10)) - 1024;
    return sign | (uint16_t)(((e + 15) << 10) | f);
}

/* ------------------------------------------------------------------------ */
/* bfloat16 (the top 16 bits of a binary32: 1 sign, 8 exponent, 7 fraction) */
/* with round to nearest, ties to even, written from the format definition. */
/* Storage of the r and c scales in plans with 16-bit scales.               */
/* ------------------------------------------------------------------------ */

uint16_t sq_f32_to_bf16(float x)
{
    uint32_t u;
    memcpy(&u, &x, 4);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x0040u); /* NaN */
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

float sq_bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float x;
    memcpy(&x, &u, 4);
    return x;
}

static float round_scale(float x, int scale_bits)
{
    return scale_bits == 16 ? sq_bf16_to_f32(sq_f32_to_bf16(x)) : x;
}

/* ------------------------------------------------------------------------ */
/* Packed format (our own; the pages fix only that the layout is decided     */
/* offline, "方法-4": 离线分配固定 packed layout).                             */
/*                                                                          */
/* Codes are offset-binary: the stored field of a b-bit code z is          */
/* u = z + 2^(b-1), in [1, 2^b - 1] for |z| <= qmax = 2^(b-1) - 1.            */
/*                                                                          */
/* Uniform-width unit (a head whose rows all share width b):                */
/*   RT = D/8 rows per band, NT = 2D tiles.  Tile                           */
/*   tau = 32*(j/16) + 4*(i/RT) + (j/4)%4 holds the RT x 4 block of rows     */
/*   [RT*(i/RT), +RT) and columns [4*(j/4), +4); inside it (i,j) is the     */
/*   tile code (r, c) = (i%RT, j%4).                                        */
/*   Tile tau's codes form a bit stream; stream byte B lives at block byte   */
/*   ((B/RT)*NT + tau)*RT + B%RT.  Inside the stream, code (r, c):           */
/*     b = 2, 4, 8, and b = 6 with RT < 4: bits [(4r+c)*b, +b), LSB first;   */
/*     b = 6 with RT >= 4: rows go in groups of four, r = 4g + s, over the    */
/*       32-bit little-endian stream words 3g, 3g+1, 3g+2.  Rows s = 0, 1, 3 */
/*       have their 24-bit row value V = sum_c u_c 2^(6c) in bits [0, 24) of */
/*       words 3g, 3g+1, 3g+2; the 24-bit value of row s = 2 is stored byte  */
/*       by byte in bits [24, 32) of the same three words (byte m in word     */
/*       3g+m).                                                             */
/* Row-major tile (a pivot head): row i starts at the sum of the byte sizes */
/*   D*b/8 of the rows before it; code j occupies row bits [b*j, b*j+b).    */
/*   A 16-bit row holds binary16 values, 2 bytes per column.                */
/* Band-tile unit (per-row units, rows of mixed width): RT = D/8 rows per   */
/*   band, NCB = D/4 tiles per band; tile (g, cb) holds rows [g*RT, +RT) x   */
/*   columns [4*cb, +4).  Its stream: for r = 0 .. RT-1 the four codes of    */
/*   row g*RT + r (columns 4cb .. 4cb+3), b_r bits each, LSB first, at       */
/*   stream bits [P_r + c*b_r, +b_r), P_r = 4 * sum_{r' < r} b_r'; a 16-bit  */
/*   row stores its binary16 patterns.  A tile stream takes                 */
/*   NW_g = ceil(P_RT / 32) 32-bit words (the rest of the last word is 0).   */
/*   Band g's block starts at word W_g = NCB * sum_{g' < g} NW_g'; stream    */
/*   word m of tile cb is block word W_g + m*NCB + (cb + 4g) mod NCB, little */
/*   endian.                                                                */
/* ------------------------------------------------------------------------ */

static int get_bit(const uint8_t *blk, long bit) { return (blk[bit >> 3] >> (bit & 7)) & 1; }
static void set_bit(uint8_t *blk, long bit, int v)
{
    if (v) blk[bit >> 3] |= (uint8_t)(1u << (bit & 7));
    else   blk[bit >> 3] &= (uint8_t)~(1u << (bit & 7));
}

/* Stream bit of bit k (0 = least significant) of tile code (r, c). */
static long tile_stream_bit(int D, int b, int r, int c, int k)
{
    int RT = D / 8;
    if (b != 6 || RT < 4) return (long)(4 * r + c) * b + k;
    int g = r / 4, s = r % 4;
    int v = 6 * c + k;                        /* bit of the 24-bit row value */
    if (s == 2) return (long)(3 * g + v / 8) * 32 + 24 + v % 8;
    int word = 3 * g + (s == 3 ? 2 : s);
    return (long)word * 32 + v;
}

/* Block bit address of bit k of code (i, j) of a uniform-width unit. */
static long uniform_bit_addr(int D, int b, int i, int j, int k)
{
    int RT = D / 8, NT = 2 * D;
    long tau = (long)(j / 16) * 32 + (i / RT) * 4 + (j / 4) % 4;
    long s = tile_stream_bit(D, b, i % RT, j % 4, k);
    long B = s >> 3;
    long byte = ((B / RT) * NT + tau) * RT + (B % RT);
    return byte * 8 + (s & 7);
}

long sq_codes_bytes_uniform(int D, int b) { return (long)D * D * b / 8; }

void sq_pack_uniform(int D, int b, const int32_t *z, uint8_t *blk)
{
    memset(blk, 0, (size_t)sq_codes_bytes_uniform(D, b));
    for (int i = 0; i < D; i++)
        for (int j = 0; j < D; j++) {
            unsigned u = (unsigned)(z[i * D + j] + (1 << (b - 1)));
            for (int k = 0; k < b; k++)
                set_bit(blk, uniform_bit_addr(D, b, i, j, k), (u >> k) & 1);
        }
}

void sq_unpack_uniform(int D, int b, const uint8_t *blk, int32_t *z)
{
    for (int i = 0; i < D; i++)
        for (int j = 0; j < D; j++) {
            unsigned u = 0;
            for (int k = 0; k < b; k++)
                u |= (unsigned)get_bit(blk, uniform_bit_addr(D, b, i, j, k)) << k;
            z[i * D + j] = (int32_t)u - (1 << (b - 1));
        }
}

long sq_row_bytes(int D, int b) { return (long)D * b / 8; }

long sq_codes_bytes_rows(int D, const int *widths)
{
    long n = 0;
    for (int i = 0; i < D; i++) n += sq_row_bytes(D, widths[i]);
    return n;
}

/* Row-major pack.  z holds codes for quantized rows; h holds binary16
 * patterns for 16-bit rows (entries of other rows are ignored). */
void sq_pack_rows(int D, const int *widths, const int32_t *z, const uint16_t *h, uint8_t *blk)
{
    long off = 0;
    memset(blk, 0, (size_t)sq_codes_bytes_rows(D, widths));
    for (int i = 0; i < D; i++) {
        int b = widths[i];
        uint8_t *row = blk + off;
        for (int j = 0; j < D; j++) {
            if (b == SQ_PIVOT_BITS) {
                row[2 * j] = (uint8_t)(h[i * D + j] & 0xff);
                row[2 * j + 1] = (uint8_t)(h[i * D + j] >> 8);
            } else {
                unsigned u = (unsigned)(z[i * D + j] + (1 << (b - 1)));
                for (int k = 0; k < b; k++) set_bit(row, (long)b * j + k, (u >> k) & 1);
            }
        }
        off += sq_row_bytes(D, b);
    }
}

void sq_unpack_rows(int D, const int *widths, const uint8_t *blk, int32_t *z, uint16_t *h)
{
    long off = 0;
    for (int i = 0; i < D; i++) {
        int b = widths[i];
        const uint8_t *row = blk + off;
        for (int j = 0; j < D; j++) {
            if (b == SQ_PIVOT_BITS) {
                h[i * D + j] = (uint16_t)(row[2 * j] | (row[2 * j + 1] << 8));
                z[i * D + j] = 0;
            } else {
                unsigned u = 0;
                for (int k = 0; k < b; k++) u |= (unsigned)get_bit(row, (long)b * j + k) << k;
                z[i * D + j] = (int32_t)u - (1 << (b - 1));
                h[i * D + j] = 0;
            }
        }
        off += sq_row_bytes(D, b);
    }
}

/* Stream words of a tile of band g. */
static long band_tile_words(int D, const int *widths, int g)
{
    int RT = D / 8;
    long bits = 0;
    for (int r = 0; r < RT; r++) bits += 4L * widths[g * RT + r];
    return (bits + 31) / 32;
}

long sq_codes_bytes_bands(int D, const int *widths)
{
    long words = 0;
    for (int g = 0; g < 8; g++) words += (long)(D / 4) * band_tile_words(D, widths, g);
    return 4 * words;
}

/* Block bit address of bit k of the field of element (i, j). */
static long band_bit_addr(int D, const int *widths, int i, int j, int k)
{
    int RT = D / 8, NCB = D / 4;
    int g = i / RT, r = i % RT, cb = j / 4, c = j % 4;
    long base = 0;
    for (int gg = 0; gg < g; gg++) base += (long)NCB * band_tile_words(D, widths, gg);
    long p = 0;
    for (int rr = 0; rr < r; rr++) p += 4L * widths[g * RT + rr];
    long s = p + (long)c * widths[i] + k;           /* stream bit */
    long word = base + (s / 32) * NCB + (cb + 4 * g) % NCB;
    return word * 32 + s % 32;
}

/* Band-tile pack.  z holds codes for quantized rows; h holds binary16
 * patterns for 16-bit rows (entries of other rows are ignored). */
void sq_pack_bands(int D, const int *widths, const int32_t *z, const uint16_t *h, uint8_t *blk)
{
    memset(blk, 0, (size_t)sq_codes_bytes_bands(D, widths));
    for (int i = 0; i < D; i++) {
        int b = widths[i];
        for (int j = 0; j < D; j++) {
            unsigned u = (b == SQ_PIVOT_BITS) ? (unsigned)h[i * D + j] : (unsigned)(z[i * D + j] + (1 << (b - 1)));
            for (int k = 0; k < b; k++) set_bit(blk, band_bit_addr(D, widths, i, j, k), (u >> k) & 1);
        }
    }
}

void sq_unpack_bands(int D, const int *widths, const uint8_t *blk, int32_t *z, uint16_t *h)
{
    for (int i = 0; i < D; i++) {
        int b = widths[i];
        for (int j = 0; j < D; j++) {
            unsigned u = 0;
            for (int k = 0; k < b; k++) u |= (unsigned)get_bit(blk, band_bit_addr(D, widths, i, j, k)) << k;
            if (b == SQ_PIVOT_BITS) {
                h[i * D + j] = (uint16_t)u;
                z[i * D + j] = 0;
            } else {
                z[i * D + j] = (int32_t)u - (1 << (b - 1));
                h[i * D + j] = 0;
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Reductions.                                                               */
/* ------------------------------------------------------------------------ */

/* fp32 pairwise sum of n = 2^m terms: sum(x[0:n]) = sum(x[0:n/2]) +
 * sum(x[n/2:n]), each addition rounded to fp32.  This is the summation order
 * of the quantizer's row sums (the row mean of r_i). */
float sq_pairwise_sum(const float *x, int n)
{
    if (n == 1) return x[0];
    float a = sq_pairwise_sum(x, n / 2);
    float b = sq_pairwise_sum(x + n / 2, n / 2);
    return a + b;
}

/* Band-order dot product over the D rows of a column: sum_i x_i y_i in fp32,
 * the order in which u, o and the two refinement sums are defined.
 *   - The rows form 8 bands of RT = D/8 consecutive rows.
 *   - Inside band g the even rows (g*RT + 0, 2, ...) and the odd rows
 *     (g*RT + 1, 3, ...) are each accumulated by a chain of fused
 *     multiply-adds that starts at +0: acc = fma(x_i, y_i, acc), rows in
 *     increasing order.  The band's value is fl(even chain + odd chain).
 *   - The 8 band values are added in a balanced binary tree in band order:
 *     ((b0 + b1) + (b2 + b3)) + ((b4 + b5) + (b6 + b7)).
 * x and y are read with strides sx and sy (a column of a row-major D x D
 * array has stride D). */
float sq_band_dot(int D, const float *x, int sx, const float *y, int sy)
{
    int RT = D / 8;
    float band[8];
    for (int g = 0; g < 8; g++) {
        float even = 0.0f, odd = 0.0f;
        for (int m = 0; m < RT; m += 2) {
            int i = g * RT + m;
            even = fmaf(x[(long)i * sx], y[(long)i * sy], even);
            odd = fmaf(x[(long)(i + 1) * sx], y[(long)(i + 1) * sy], odd);
        }
        band[g] = even + odd;
    }
    return sq_pairwise_sum(band, 8);
}

/* ------------------------------------------------------------------------ */
/* Quantizer (section 方法-3): X_hat_ij = r_i * c_j * z_ij.                   */
/*   rho_i   = (omega_i / mean omega)^(-1/4)          (from the plan)         */
/*   r_i     = max(mean_j |S_ij|, 1e-12) * rho_i                              */
/*   c0_j    = max_i |S_ij / r_i| / qmax_i                                    */
/*   z0      = rhe(S / (r c0))                                                */
/*   c_j     = sum_i w_i r_i z0_ij S_ij / sum_i w_i r_i^2 z0_ij^2  (w = omega) */
/*   z       = clamp(rhe(S / (r c)), -qmax, qmax)                             */
/* Readings (the pages print none of these formulas):                        */
/*   - the row mean is the fp32 pairwise sum of |S_ij| over j, times 1/D;     */
/*   - S/(r c) is taken as y = fl(S * fl(1/r)) and then the exact product    */
/*     y * fl(1/c) is rounded to the nearest integer, ties to even;          */
/*   - dividing by qmax is a product with fl(1/qmax):                        */
/*     c0_j = max_i fl(|y_ij| * fl(1/qmax_i)); an all-zero column gets 1;     */
/*   - with t_ij = fl(b_i * z0_ij), b_i = fl(wbar_i * fl(r_i * r_i)), the     */
/*     refinement is c_j = fl(N_j / D_j) with N_j = sum_i t_ij y_ij and       */
/*     D_j = sum_i t_ij z0_ij in band order (sq_band_dot); these equal        */
/*     sum w r z0 S and sum w r^2 z0^2 up to the common factor 1/r;          */
/*     rows of 16-bit (pivot) width have t = 0; a zero denominator keeps c0; */
/*   - c_j is rounded to fp32 before the final codes are taken.               */
/*   - 16-bit scale storage (scale_bits = 16, the pages' 16-bit scale        */
/*     accounting, 局限): r_i is rounded                                      */
/*     to bfloat16 (RNE) as soon as it is formed and that value is used      */
/*     everywhere after (1/r, b_i, the record); c_j likewise after the        */
/*     refinement, before the final codes.  sq_quantize = scale_bits 32.      */
/* 16-bit rows are stored as binary16 (RNE) and carry no row factor (r = 0).  */
/* tie_out (optional, D*D): bit0 = final code within 1e-6 relative of a .5   */
/* boundary; bit1 = its column had such a tie in z0 (column tie-affected).   */
/* z0_out (optional, D*D): the initial codes z0 (exposed for the LS pin).     */
/* ------------------------------------------------------------------------ */

static int qmax_of(int b) { return (1 << (b - 1)) - 1; }

static int near_half(double x)
{
    double ax = fabs(x);
    double f = floor(ax);
    return fabs(ax - (f + 0.5)) <= 1e-6 * ax;
}

void sq_quantize_s(int D, const int *widths, const float *rho, const float *wbar,
                   const float *S, int32_t *z, uint16_t *h, float *r, float *c,
                   uint8_t *tie_out, int32_t *z0_out, int scale_bits)
{
    float *absrow = (float *)malloc(sizeof(float) * D);
    float *y = (float *)malloc(sizeof(float) * D * D);
    float *bw = (float *)malloc(sizeof(float) * D);
    float *t = (float *)malloc(sizeof(float) * D);
    float *z0f = (float *)malloc(sizeof(float) * D);
    float *ycol = (float *)malloc(sizeof(float) * D);
    int32_t *z0 = (int32_t *)malloc(sizeof(int32_t) * D * D);
    uint8_t *coltie = (uint8_t *)calloc(D, 1);

    /* row factors */
    for (int i = 0; i < D; i++) {
        if (widths[i] == SQ_PIVOT_BITS) {
            r[i] = 0.0f;
            bw[i] = 0.0f;
            for (int j = 0; j < D; j++) {
                h[i * D + j] = sq_f32_to_f16(S[i * D + j]);
                z[i * D + j] = 0;
                y[i * D + j] = 0.0f;
            }
            continue;
        }
        for (int j = 0; j < D; j++) absrow[j] = fabsf(S[i * D + j]);
        float m = sq_pairwise_sum(absrow, D) * (1.0f / (float)D);
        if (!(m > 1e-12f)) m = 1e-12f;
        r[i] = round_scale(m * rho[i], scale_bits);
        float inv_r = 1.0f / r[i];
        for (int j = 0; j < D; j++) {
            y[i * D + j] = S[i * D + j] * inv_r;
            h[i * D + j] = 0;
        }
        float rr = r[i] * r[i];
        bw[i] = wbar[i] * rr;
    }

    for (int j = 0; j < D; j++) {
        /* initial column factor */
        float c0 = 0.0f;
        for (int i = 0; i < D; i++) {
            if (widths[i] == SQ_PIVOT_BITS) continue;
            float iq = 1.0f / (float)qmax_of(widths[i]);
            float v = fabsf(y[i * D + j]) * iq;
            if (v > c0) c0 = v;
        }
        if (c0 == 0.0f) c0 = 1.0f;
        float inv_c0 = 1.0f / c0;
        /* initial codes and the weighted least-squares refinement */
        for (int i = 0; i < D; i++) {
            ycol[i] = y[i * D + j];
            if (widths[i] == SQ_PIVOT_BITS) { z0[i * D + j] = 0; z0f[i] = 0.0f; t[i] = 0.0f; continue; }
            double x0 = (double)y[i * D + j] * (double)inv_c0; /* exact: 24 x 24 bits */
            z0[i * D + j] = (int32_t)rint(x0);
            if (near_half(x0)) coltie[j] = 1;
            z0f[i] = (float)z0[i * D + j];
            t[i] = bw[i] * z0f[i];
        }
        float num = sq_band_dot(D, t, 1, ycol, 1);
        float den = sq_band_dot(D, t, 1, z0f, 1);
        float cj = round_scale((den > 0.0f) ? num / den : c0, scale_bits);
        c[j] = cj;
        float inv_c = 1.0f / cj;
        for (int i = 0; i < D; i++) {
            if (widths[i] == SQ_PIVOT_BITS) continue;
            int q = qmax_of(widths[i]);
            double x = (double)y[i * D + j] * (double)inv_c;
            double zr = rint(x);
            if (zr > q) zr = q;
            if (zr < -q) zr = -q;
            z[i * D + j] = (int32_t)zr;
            if (tie_out)
                tie_out[i * D + j] = (uint8_t)((near_half(x) ? 1 : 0) | (coltie[j] ? 2 : 0));
        }
    }
    if (tie_out)
        for (int i = 0; i < D; i++)
            if (widths[i] == SQ_PIVOT_BITS)
                for (int j = 0; j < D; j++) tie_out[i * D + j] = 0;
    if (z0_out)
        for (int i = 0; i < D; i++)
            for (int j = 0; j < D; j++)
                z0_out[i * D + j] = (widths[i] == SQ_PIVOT_BITS) ? 0 : z0[i * D + j];

    free(absrow); free(y); free(bw); free(t); free(z0f); free(ycol); free(z0); free(coltie);
}

void sq_quantize(int D, const int *widths, const float *rho, const float *wbar,
                 const float *S, int32_t *z, uint16_t *h, float *r, float *c,
                 uint8_t *tie_out, int32_t *z0_out)
{
    sq_quantize_s(D, widths, rho, wbar, S, z, h, r, c, tie_out, z0_out, 32);
}

/* ------------------------------------------------------------------------ */
/* Per-row absmax quantizer: the ordinary baseline the pages set against     */
/* STEPQuant (实验: uniform INT4 / INT6 / INT8 and the remark that plain      */
/* per-row absmax stays unstable even at 8 bits).  Reading, per row i of     */
/* width b (qmax = 2^(b-1) - 1):                                             */
/*   m_i = max_j |S_ij|;  r_i = fl(m_i / qmax), or 1 when m_i = 0;           */
/*   z_ij = clamp(nearest integer, ties to even, to the exact product        */
/*          S_ij * fl(1/r_i), -qmax, +qmax);  c_j = 1 for every column.      */
/* The record keeps the r | c layout, so X_hat = fl(fl(r_i c_j) z_ij) =      */
/* fl(r_i z_ij) decodes it unchanged.  16-bit rows as in sq_quantize.        */
/* tie_out (optional): bit0 = code within 1e-6 relative of a .5 boundary.    */
/* ------------------------------------------------------------------------ */

void sq_quantize_absmax_s(int D, const int *widths, const float *S, int32_t *z, uint16_t *h,
                          float *r, float *c, uint8_t *tie_out, int scale_bits)
{
    for (int j = 0; j < D; j++) c[j] = 1.0f;
    for (int i = 0; i < D; i++) {
        if (widths[i] == SQ_PIVOT_BITS) {
            r[i] = 0.0f;
            for (int j = 0; j < D; j++) {
                h[i * D + j] = sq_f32_to_f16(S[i * D + j]);
                z[i * D + j] = 0;
                if (tie_out) tie_out[i * D + j] = 0;
            }
            continue;
        }
        int q = qmax_of(widths[i]);
        float m = 0.0f;
        for (int j = 0; j < D; j++) {
            float a = fabsf(S[i * D + j]);
            if (a > m) m = a;
        }
        r[i] = round_scale((m > 0.0f) ? m / (float)q : 1.0f, scale_bits);
        float inv_r = 1.0f / r[i];
        for (int j = 0; j < D; j++) {
            double x = (double)S[i * D + j] * (double)inv_r; /* exact: 24 x 24 bits */
            double zr = rint(x);
            if (zr > q) zr = q;
            if (zr < -q) zr = -q;
            z[i * D + j] = (int32_t)zr;
            h[i * D + j] = 0;
            if (tie_out) tie_out[i * D + j] = (uint8_t)(near_half(x) ? 1 : 0);
        }
    }
}

void sq_quantize_absmax(int D, const int *widths, const float *S, int32_t *z, uint16_t *h,
                        float *r, float *c, uint8_t *tie_out)
{
    sq_quantize_absmax_s(D, widths, S, z, h, r, c, tie_out, 32);
}

/* Reconstruction X_hat_ij = fl(fl(r_i * c_j) * z_ij); 16-bit rows decode the
 * stored binary16 value. */
void sq_reconstruct(int D, const int *widths, const int32_t *z, const uint16_t *h,
                    const float *r, const float *c, float *S_hat)
{
    for (int i = 0; i < D; i++)
        for (int j = 0; j < D; j++) {
            if (widths[i] == SQ_PIVOT_BITS)
                S_hat[i * D + j] = sq_f16_to_f32(h[i * D + j]);
            else {
                float rc = r[i] * c[j];
                S_hat[i * D + j] = rc * (float)z[i * D + j];
            }
        }
}

/* ------------------------------------------------------------------------ */
/* One decode step of a packed head (sections 背景与动机 and 方法-4).           */
/*                                                                          */
/* Recurrence (gated delta rule; KDA reading with Diag(alpha) applied first): */
/*   S_t = (I - beta k k^T) Diag(alpha) S_{t-1} + beta k v^T,  o_t = S_t^T q  */
/* Readings (the pages fix the update in fp32 and no summation order):        */
/*   - retention is folded into the row factor: a_i = fl(alpha_i r_i) and      */
/*     S'_ij = fl(fl(a_i c_j) z_ij); 16-bit rows: S'_ij = fl(alpha_i h_ij);   */
/*   - u_j = sum_i k_i S'_ij in band order (sq_band_dot);                     */
/*   - w_j = fl(beta * fl(v_j - u_j));  S_ij = fma(k_i, w_j, S'_ij);           */
/*   - o_j = sum_i q_i S_ij in band order over the updated fp32 state: the    */
/*     readout of S_t, taken before requantization.                           */
/* alpha has D entries (GDN: all equal).  S_out receives the fp32 S_t that    */
/* the requantizer consumes.                                                 */
/* ------------------------------------------------------------------------ */

void sq_step_from_codes(int D, const int *widths, const int32_t *z, const uint16_t *h,
                        const float *r, const float *c,
                        const float *q, const float *k, const float *v,
                        const float *alpha, float beta,
                        float *S_out, float *o_out, float *u_out, float *w_out)
{
    float *w = (float *)malloc(sizeof(float) * D);
    for (int i = 0; i < D; i++) {
        if (widths[i] == SQ_PIVOT_BITS) {
            for (int j = 0; j < D; j++) S_out[i * D + j] = alpha[i] * sq_f16_to_f32(h[i * D + j]);
        } else {
            float a = alpha[i] * r[i];
            for (int j = 0; j < D; j++) {
                float A = a * c[j];
                S_out[i * D + j] = A * (float)z[i * D + j];
            }
        }
    }
    for (int j = 0; j < D; j++) {
        float u = sq_band_dot(D, k, 1, S_out + j, D);
        float d = v[j] - u;
        w[j] = beta * d;
        if (u_out) u_out[j] = u;
        if (w_out) w_out[j] = w[j];
    }
    for (int i = 0; i < D; i++)
        for (int j = 0; j < D; j++)
            S_out[i * D + j] = fmaf(k[i], w[j], S_out[i * D + j]);
    for (int j = 0; j < D; j++) o_out[j] = sq_band_dot(D, q, 1, S_out + j, D);
    free(w);
}

/* ------------------------------------------------------------------------ */
/* Plain FP32-state recurrence (the unquantized state the pages compare      */
/* against, "FP32-state").  Same update and the same band-order sums as the  */
/* packed step: S'_ij = fl(alpha_i S_ij), u_j = band(k, S'_.j),              */
/* w_j = fl(beta fl(v_j - u_j)), S_ij = fma(k_i, w_j, S'_ij),                */
/* o_j = band(q, S_.j).                                                      */
/* ------------------------------------------------------------------------ */

void sq_step_fp32(int D, float *S, const float *q, const float *k, const float *v,
                  const float *alpha, float beta, float *o_out)
{
    float *w = (float *)malloc(sizeof(float) * D);
    for (int i = 0; i < D; i++)
        for (int j = 0; j < D; j++) S[i * D + j] = alpha[i] * S[i * D + j];
    for (int j = 0; j < D; j++) {
        float u = sq_band_dot(D, k, 1, S + j, D);
        float d = v[j] - u;
        w[j] = beta * d;
    }
    for (int i = 0; i < D; i++)
        for (int j = 0; j < D; j++) S[i * D + j] = fmaf(k[i], w[j], S[i * D + j]);
    for (int j = 0; j < D; j++) o_out[j] = sq_band_dot(D, q, 1, S + j, D);
    free(w);
}

/* The same recurrence in fp64 (used for the invariants and the drift study). */
void sq_step_fp64(int D, double *S, const double *q, const double *k, const double *v,
                  const double *alpha, double beta, double *o_out)
{
    double *w = (double *)malloc(sizeof(double) * D);
    for (int i = 0; i < D; i++)
        for (int j = 0; j < D; j++) S[i * D + j] = alpha[i] * S[i * D + j];
    for (int j = 0; j < D; j++) {
        double u = 0.0;
        for (int i = 0; i < D; i++) u += k[i] * S[i * D + j];
        w[j] = beta * (v[j] - u);
    }
    for (int i = 0; i < D; i++)
        for (int j = 0; j < D; j++) S[i * D + j] = S[i * D + j] + k[i] * w[j];
    for (int j = 0; j < D; j++) {
        double o = 0.0;
        for (int i = 0; i < D; i++) o += q[i] * S[i * D + j];
        o_out[j] = o;
    }
    free(w);
}

/* ------------------------------------------------------------------------ */
/* Calibration statistics (sections 方法-1 and 方法-2).                        */
/*   g_t = A_t^T q_t with A_t = (I - beta k k^T) Diag(alpha):                 */
/*   g = alpha (.) (q - beta k (k^T q)); omega_i accumulates g_i^2.           */
/*   lsum accumulates log(alpha_i) (mean log retention gate).                 */
/* ------------------------------------------------------------------------ */

void sq_calib_accumulate(int D, const float *q, const float *k, const float *alpha,
                         float beta, double *omega_acc, double *lsum_acc)
{
    double kq = 0.0;
    for (int i = 0; i < D; i++) kq += (double)k[i] * (double)q[i];
    for (int i = 0; i < D; i++) {
        double g = (double)alpha[i] * ((double)q[i] - (double)beta * (double)k[i] * kq);
        omega_acc[i] += g * g;
        lsum_acc[i] += log((double)alpha[i]);
    }
}

/* Squared Frobenius reconstruction error of each row when the whole head is
 * quantized at uniform width b (distortion d_u(b), section 方法-1).  rho and
 * wbar are the plan's row weights.  err_rows receives D values. */
void sq_distortion_rows(int D, int b, const float *rho, const float *wbar,
                        const float *S, double *err_rows)
{
    int *widths = (int *)malloc(sizeof(int) * D);
    int32_t *z = (int32_t *)malloc(sizeof(int32_t) * D * D);
    uint16_t *h = (uint16_t *)malloc(sizeof(uint16_t) * D * D);
    float *r = (float *)malloc(sizeof(float) * D);
    float *c = (float *)malloc(sizeof(float) * D);
    float *Sh = (float *)malloc(sizeof(float) * D * D);
    for (int i = 0; i < D; i++) widths[i] = b;
    sq_quantize(D, widths, rho, wbar, S, z, h, r, c, NULL, NULL);
    sq_reconstruct(D, widths, z, h, r, c, Sh);
    for (int i = 0; i < D; i++) {
        double e = 0.0;
        for (int j = 0; j < D; j++) {
            double d = (double)Sh[i * D + j] - (double)S[i * D + j];
            e += d * d;
        }
        err_rows[i] = e;
    }
    free(widths); free(z); free(h); free(r); free(c); free(Sh);
}

/* Lifetime weight L_u = sum_{j=0}^{H-1} exp(2 j l_u) (section 方法-1),
 * summed term by term. */
double sq_lifetime_weight(double l, long H)
{
    double s = 0.0;
    for (long j = 0; j < H; j++) s += exp(2.0 * (double)j * l);
    return s;
}
