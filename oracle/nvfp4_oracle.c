/*
 * nvfp4_oracle.c -- plain, slow CPU oracle for the NVFP4 W4A4 linear layer and
 * the NVFP4 KV-cache store.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call
 * this file: only the tests, the package's smoke check and the bench's
 * cpu_baseline / reference leg do.  It shares no code, header, table or helper
 * with the CUDA library; it is written from the format definition alone.
 *
 * Sources (page title + section):
 *  [RN]  "LongLive-2.0：用 NVFP4 并行底座做长视频生成" (yingwang.github.io reading
 *        note), section 二 方法 / "NVFP4 量化格式": E2M1 element codes
 *        (1 sign, 2 exponent, 1 mantissa bit), three-level scaling (one FP32
 *        tensor factor, one FP8 E4M3 factor per 16-element block, the FP4
 *        element) and the Dequant equation X^FP4 * a^FP8 * a^FP32.
 *  [RN-T] same note, "NVFP4 训练的工程细节": W4A4 linears, 1D block scaling
 *        along K for activations.
 *  [RN-I] same note, section 二 "推理底座" (second item, KV quantization): each
 *        frame-chunk's K and V are quantized separately; storage goes from
 *        4*T_c*H*d to 9/8*T_c*H*d bytes.
 *
 * Readings where the pages are silent:
 *  R1  tensor scale  a32 = fl32(amax / 2688), 2688 = 6 * 448 (E2M1 max times
 *      E4M3 max), so the tensor's largest block gets the largest block scale.
 *  R2  a32 == 0 (all-zero tensor): every scale code and element code is 0.
 *  R3  block scale code = E4M3 round-to-nearest-even, saturating to 448, of
 *      r = fl32(amax_b / fl32(6 * a32)); subnormal E4M3 kept.
 *  R4  a block whose decoded scale is 0 is flushed: its 16 codes are +0.
 *  R5  element ratio y = fl32(x * fl32(1 / fl32(s * a32))) (multiply by a
 *      reciprocal, not a division).
 *  R6  element code = E2M1 round-to-nearest-even, saturating to 6.
 *  R7  the code's sign bit is the sign bit of y, so a negative y that rounds
 *      to zero gives code 0x8 (-0).
 *  R8  two codes per byte, element 2i in bits 3:0, element 2i+1 in bits 7:4.
 *  R9  GEMM scale layout: 128x4 tiles of 512 bytes (the block-scaled MMA's
 *      scale-factor tile), see orc_swizzle_scales.
 *  R10 dequant to bf16: fl32(fl32(e2m1 * s) * a32), then bf16 round-to-nearest-
 *      even (two roundings, in that order).
 *  R11 GELU is the tanh form.
 *  R15 KV: one a32 per (slot, K or V) over the whole chunk.
 *  R18 adaptive scale search over the targets {4, 6} (optional mode): per
 *      block, besides the standard encoding (block max aimed at 6: R3..R7),
 *      encode with the block max aimed at 4 (r = fl32(amax_b / fl32(4 * a32)),
 *      same rounding rules), and keep the one whose squared error is smaller;
 *      a tie keeps the standard one.  The error is taken in binary32, in this
 *      order: d = fl32(fl32(e2m1 * s) * a32) (R10's dequant product),
 *      e = fl32(x - d), sum = fl32(sum + fl32(e * e)) over elements 0..15.
 *      The tensor scale stays R1's.
 *  R19 LayerNorm + adaLN modulate before the quantize (optional path): row
 *      statistics by their definition (binary64, rounded once to binary32),
 *      then the modulation in binary32 steps; see orc_ln_stats.
 *  R16 KV slot = NVFP4 matrix of T*H rows x d columns, blocks along d, scales
 *      row-major (not swizzled).
 *  R20 K-smoothing of a KV chunk (optional, per tensor): subtract each
 *      channel's mean over the chunk's tokens (binary64, rounded once to
 *      binary32) before the quantize and add it back in the dequant; see
 *      orc_channel_mean.
 *  R21 2D block scaling of weights [RN-T]: one E4M3 scale per 16 x 16 block
 *      from the block's amax; see orc_quantize_2d_f32.
 *  R22 Random Hadamard Transform ahead of the weight-gradient quantize
 *      [RN-T]: 16-point, normalised, Sylvester order, one sign vector; see
 *      rht16.
 *  R24 rotary position embedding of a KV chunk's keys ahead of their
 *      quantize (optional; the fused RoPE ahead of the in-place KV update of
 *      the anzhuoshouzhuan.com article, "NVFP4 量化"): the interleaved pairs
 *      (2p, 2p+1) of every head turn by the angle of (token, p), given as a
 *      binary32 cos / sin table; see orc_rope for the order.  Values are never
 *      rounded to bf16 between the rotation and the quantize.
 *
 * Every floating-point step that the GPU must reproduce bit for bit is done in
 * IEEE binary32 (compile with -ffp-contract=off so nothing fuses); the GEMM
 * reference accumulates in binary64.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>
#include <fenv.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_API __attribute__((visibility("default")))

/* ------------------------------------------------------------------------ */
/* threads                                                                   */
/* ------------------------------------------------------------------------ */
static int g_threads = 0; /* 0 = OpenMP default */

ORC_API void orc_set_threads(int n) { g_threads = n; }

ORC_API int orc_get_threads(void)
{
#ifdef _OPENMP
    return g_threads > 0 ? g_threads : omp_get_max_threads();
#else
    return 1;
#endif
}

static int nthreads(void) { return orc_get_threads(); }

/* ------------------------------------------------------------------------ */
/* bf16 <-> binary32 / binary64                                              */
/* ------------------------------------------------------------------------ */
ORC_API float orc_bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* binary64 -> bf16, one correctly rounded step (nearest, ties to even).
 * bf16 keeps 8 significant bits; below 2^-126 its spacing is 2^-133. */
ORC_API uint16_t orc_f64_to_bf16(double x)
{
    if (isnan(x)) return 0x7FC0;
    int neg = signbit(x) ? 1 : 0;
    double a = fabs(x);
    double r;
    if (a == 0.0) {
        r = 0.0;
    } else if (isinf(a)) {
        r = INFINITY;
    } else {
        int e;
        frexp(a, &e);           /* a = f * 2^e, f in [0.5, 1) */
        int q = e - 8;          /* spacing of 8-bit significands in [2^(e-1), 2^e) */
        if (q < -133) q = -133; /* subnormal bf16 spacing */
        r = ldexp(nearbyint(ldexp(a, -q)), q);
        if (r >= ldexp(1.0, 128)) r = INFINITY;
    }
    float f = (float)r; /* exact: r has at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, 4);
    uint16_t h = (uint16_t)(u >> 16);
    return (uint16_t)(h | (neg ? 0x8000u : 0u));
}

ORC_API uint16_t orc_f32_to_bf16(float x) { return orc_f64_to_bf16((double)x); }

/* ------------------------------------------------------------------------ */
/* E2M1 (element code) and E4M3 (block scale)                                */
/* ------------------------------------------------------------------------ */
/* E2M1: bit 3 sign, bits 2:1 exponent (bias 1), bit 0 mantissa.
 * Exponent 0 is subnormal: m * 0.5.  Otherwise (1 + m/2) * 2^(e-1). [RN] */
ORC_API double orc_e2m1_value(unsigned code)
{
    unsigned s = (code >> 3) & 1u, e = (code >> 1) & 3u, m = code & 1u;
    double mag = (e == 0) ? 0.5 * (double)m : (1.0 + 0.5 * (double)m) * ldexp(1.0, (int)e - 1);
    return s ? -mag : mag;
}

/* E4M3: bit 7 sign, bits 6:3 exponent (bias 7), bits 2:0 mantissa.
 * Exponent 0 is subnormal: m/8 * 2^-6.  S.1111.111 is NaN; no infinity. */
ORC_API double orc_e4m3_value(unsigned code)
{
    unsigned s = (code >> 7) & 1u, e = (code >> 3) & 15u, m = code & 7u;
    if (e == 15 && m == 7) return NAN;
    double mag = (e == 0) ? ((double)m / 8.0) * ldexp(1.0, -6)
                          : (1.0 + (double)m / 8.0) * ldexp(1.0, (int)e - 7);
    return s ? -mag : mag;
}

/* Round |v| to the nearest entry of an ascending table of n non-negative
 * values whose index is the code; ties go to the even index; |v| beyond the
 * last entry saturates to it.  All comparisons are exact in binary64 (the
 * table entries and their midpoints are short dyadic numbers and v is a
 * binary32 value). */
static unsigned nearest_even(const double* tab, unsigned n, double v)
{
    if (v >= tab[n - 1]) return n - 1;
    unsigned i = 0;
    while (!(v >= tab[i] && v <= tab[i + 1])) i++;
    double lo = tab[i], hi = tab[i + 1], mid = 0.5 * (lo + hi);
    if (v < mid) return i;
    if (v > mid) return i + 1;
    return (i % 2 == 0) ? i : i + 1;
}

static double g_e2m1_tab[8];
static double g_e4m3_tab[127]; /* codes 0x00..0x7E, ascending */
static int g_tabs_ready = 0;

static void init_tabs(void)
{
    if (g_tabs_ready) return;
    for (unsigned c = 0; c < 8; c++) g_e2m1_tab[c] = orc_e2m1_value(c);
    for (unsigned c = 0; c < 127; c++) g_e4m3_tab[c] = orc_e4m3_value(c);
    g_tabs_ready = 1;
}

/* R6, R7: nearest-even on the E2M1 grid, saturating at 6, sign from y. */
ORC_API unsigned orc_e2m1_encode(float y)
{
    init_tabs();
    unsigned mag = nearest_even(g_e2m1_tab, 8, fabs((double)y));
    return mag | (signbit(y) ? 8u : 0u);
}

/* R3: nearest-even on the non-negative E4M3 values, saturating at 448.
 * Only non-negative finite r reach this (block amax over a positive d6). */
ORC_API unsigned orc_e4m3_encode(float r)
{
    init_tabs();
    return nearest_even(g_e4m3_tab, 127, fabs((double)r));
}

/* ------------------------------------------------------------------------ */
/* Quantize [RN] three-level scaling, [RN-T] 1D blocks of 16 along a row     */
/* ------------------------------------------------------------------------ */
#define ORC_MODE_COMPUTE 0
#define ORC_MODE_GIVEN 1
#define ORC_MODE_SEARCH46 4 /* OR-ed into the mode: R18 */

/* One candidate encoding of a 16-element block with the block max aimed at
 * `target` (6: R3..R7; 4: R18): scale code and element codes. */
static void encode_block(const float* xb, float amax_b, float a32, float target, uint8_t* sc, uint8_t* q)
{
    memset(q, 0, 16);
    float d = target * a32;
    float rb = amax_b / d;
    *sc = (uint8_t)orc_e4m3_encode(rb); /* R3 */
    float s = (float)orc_e4m3_value(*sc);
    if (s != 0.0f) { /* R4 */
        float denom = s * a32;
        float inv = 1.0f / denom; /* R5 */
        for (int i = 0; i < 16; i++) {
            float y = xb[i] * inv;
            q[i] = (uint8_t)orc_e2m1_encode(y); /* R6, R7 */
        }
    }
}

/* R18: binary32 squared error of a candidate, in the stated order. */
static float block_sq_error(const float* xb, uint8_t sc, const uint8_t* q, float a32)
{
    float s = (float)orc_e4m3_value(sc);
    float sum = 0.0f;
    for (int i = 0; i < 16; i++) {
        float e2 = (float)orc_e2m1_value(q[i]);
        float dq = (e2 * s) * a32;
        float e = xb[i] - dq;
        float ee = e * e;
        sum = sum + ee;
    }
    return sum;
}

/* x: binary32 [rows x cols], row stride ld elements.  cols % 16 == 0.
 * codes: [rows x cols/2] bytes (R8).  scales: logical [rows x cols/16] E4M3
 * codes, row-major.  *alpha is written (COMPUTE) or read (GIVEN). */
ORC_API int orc_quantize_f32(const float* x, int64_t rows, int64_t cols, int64_t ld, int mode,
                             float* alpha, uint8_t* codes, uint8_t* scales)
{
    if (cols % 16 != 0 || ld < cols) return 1;
    init_tabs();
    float a32;
    const int search = (mode & ORC_MODE_SEARCH46) != 0;
    mode &= ~ORC_MODE_SEARCH46;
    if (mode == ORC_MODE_COMPUTE) {
        float amax = 0.0f;
        for (int64_t r = 0; r < rows; r++)
            for (int64_t c = 0; c < cols; c++) {
                float v = fabsf(x[r * ld + c]);
                if (v > amax) amax = v;
            }
        a32 = amax / 2688.0f; /* R1 */
        *alpha = a32;
    } else {
        a32 = *alpha;
    }
    const int64_t nb = cols / 16;
#pragma omp parallel for schedule(static) num_threads(nthreads())
    for (int64_t r = 0; r < rows; r++) {
        for (int64_t b = 0; b < nb; b++) {
            const float* xb = x + r * ld + b * 16;
            uint8_t sc = 0;
            uint8_t q[16];
            memset(q, 0, sizeof q);
            if (a32 != 0.0f) { /* R2 */
                float amax_b = 0.0f;
                for (int i = 0; i < 16; i++)
                    if (fabsf(xb[i]) > amax_b) amax_b = fabsf(xb[i]);
                encode_block(xb, amax_b, a32, 6.0f, &sc, q);
                if (search) {
                    uint8_t sc4, q4[16];
                    encode_block(xb, amax_b, a32, 4.0f, &sc4, q4);
                    if (block_sq_error(xb, sc4, q4, a32) < block_sq_error(xb, sc, q, a32)) {
                        sc = sc4;
                        memcpy(q, q4, 16);
                    }
                }
            }
            scales[r * nb + b] = sc;
            uint8_t* cb = codes + r * (cols / 2) + b * 8;
            for (int i = 0; i < 8; i++) cb[i] = (uint8_t)(q[2 * i] | (q[2 * i + 1] << 4)); /* R8 */
        }
    }
    return 0;
}

/* bf16 input: widen each element exactly to binary32, then quantize. */
ORC_API int orc_quantize_bf16(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, int mode,
                              float* alpha, uint8_t* codes, uint8_t* scales)
{
    if (cols % 16 != 0 || ld < cols) return 1;
    float* xf = (float*)malloc((size_t)(rows * cols) * sizeof(float) + 1);
    if (!xf) return 2;
    for (int64_t r = 0; r < rows; r++)
        for (int64_t c = 0; c < cols; c++) xf[r * cols + c] = orc_bf16_to_f32(x[r * ld + c]);
    int rc = orc_quantize_f32(xf, rows, cols, cols, mode, alpha, codes, scales);
    free(xf);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* R9 scale-factor tile layout of the block-scaled MMA                       */
/* ------------------------------------------------------------------------ */
/* Logical scales [rows x sc] (sc = cols/16).  Padded to ceil(rows/128)*128
 * rows and ceil(sc/4)*4 columns; tile (i, j) = rows 128i.., columns 4j.. is
 * 512 contiguous bytes at (i * ceil(sc/4) + j) * 512, and element (r, c) of
 * the tile sits at (r % 32) * 16 + (r / 32) * 4 + c.  Padding is zero. */
ORC_API int64_t orc_swizzled_bytes(int64_t rows, int64_t sc)
{
    return ((rows + 127) / 128) * 128 * ((sc + 3) / 4) * 4;
}

ORC_API int64_t orc_swizzle_offset(int64_t r, int64_t c, int64_t sc)
{
    int64_t tiles_c = (sc + 3) / 4;
    int64_t i = r / 128, j = c / 4, rr = r % 128, cc = c % 4;
    return (i * tiles_c + j) * 512 + (rr % 32) * 16 + (rr / 32) * 4 + cc;
}

ORC_API void orc_swizzle_scales(const uint8_t* logical, int64_t rows, int64_t sc, uint8_t* out)
{
    memset(out, 0, (size_t)orc_swizzled_bytes(rows, sc));
    for (int64_t r = 0; r < rows; r++)
        for (int64_t c = 0; c < sc; c++) out[orc_swizzle_offset(r, c, sc)] = logical[r * sc + c];
}

ORC_API void orc_unswizzle_scales(const uint8_t* swz, int64_t rows, int64_t sc, uint8_t* logical)
{
    for (int64_t r = 0; r < rows; r++)
        for (int64_t c = 0; c < sc; c++) logical[r * sc + c] = swz[orc_swizzle_offset(r, c, sc)];
}

/* ------------------------------------------------------------------------ */
/* Dequant [RN] Dequant(X) = X^FP4 * a^FP8 * a^FP32                          */
/* ------------------------------------------------------------------------ */
static double code_at(const uint8_t* codes, int64_t cols, int64_t r, int64_t c)
{
    uint8_t byte = codes[r * (cols / 2) + c / 2];
    return orc_e2m1_value((c % 2 == 0) ? (byte & 15u) : (byte >> 4));
}

/* out[r, c] = fl32(fl32(e2m1 * s) * a32)  (the inner product is exact). */
ORC_API void orc_dequant_f32(const uint8_t* codes, const uint8_t* scales, float alpha, int64_t rows,
                             int64_t cols, float* out)
{
    const int64_t nb = cols / 16;
#pragma omp parallel for schedule(static) num_threads(nthreads())
    for (int64_t r = 0; r < rows; r++)
        for (int64_t c = 0; c < cols; c++) {
            float qs = (float)(code_at(codes, cols, r, c) * orc_e4m3_value(scales[r * nb + c / 16]));
            out[r * cols + c] = qs * alpha;
        }
}

/* R10: the binary32 dequant value, then bf16 nearest-even. */
ORC_API void orc_dequant_bf16(const uint8_t* codes, const uint8_t* scales, float alpha, int64_t rows,
                              int64_t cols, uint16_t* out)
{
    const int64_t nb = cols / 16;
#pragma omp parallel for schedule(static) num_threads(nthreads())
    for (int64_t r = 0; r < rows; r++)
        for (int64_t c = 0; c < cols; c++) {
            float qs = (float)(code_at(codes, cols, r, c) * orc_e4m3_value(scales[r * nb + c / 16]));
            float v = qs * alpha;
            out[r * cols + c] = orc_f32_to_bf16(v);
        }
}

/* ------------------------------------------------------------------------ */
/* GEMM: C = aA * aB * (A_q . S_A)(B_q . S_B)^T, then the epilogue, in fp64   */
/* ------------------------------------------------------------------------ */
typedef struct {
    const uint16_t* bias;      /* bf16 [N] or NULL */
    const uint16_t* mod_scale; /* bf16 [N] or NULL: y * (1 + mod_scale) + mod_shift */
    const uint16_t* mod_shift; /* bf16 [N] or NULL */
    const uint16_t* gate;      /* bf16 [N] or NULL: residual + gate * y */
    const uint16_t* residual;  /* bf16 [M x N] (row stride ld_res) or NULL */
    int64_t ld_res;
    int act;                   /* 0 none, 1 gelu (tanh form, R11) */
} orc_epilogue;

static double bfv(const uint16_t* p, int64_t i) { return (double)orc_bf16_to_f32(p[i]); }

static double gelu_tanh(double y)
{
    const double k = sqrt(2.0 / M_PI);
    return 0.5 * y * (1.0 + tanh(k * (y + 0.044715 * y * y * y)));
}

/* A: codes [M x K/2], logical scales [M x K/16]; B: codes [N x K/2], logical
 * scales [N x K/16].  rows: optional list of n_rows row indices of C to
 * compute (NULL = all M rows, in order).  y: fp64 [n_rows x N] results after
 * the epilogue (may be NULL); out_bf16: bf16 [n_rows x N] (may be NULL). */
ORC_API int orc_gemm(const uint8_t* a_codes, const uint8_t* a_scales, float a_alpha,
                     const uint8_t* b_codes, const uint8_t* b_scales, float b_alpha, int64_t M, int64_t N,
                     int64_t K, const orc_epilogue* ep, const int64_t* rows, int64_t n_rows, double* y,
                     uint16_t* out_bf16)
{
    if (K % 16 != 0) return 1;
    const int64_t nb = K / 16;
    const int64_t R = rows ? n_rows : M;
    /* dequantized B (without its tensor scale), fp64, exact */
    double* bd = (double*)malloc((size_t)(N * K) * sizeof(double) + 8);
    if (!bd) return 2;
#pragma omp parallel for schedule(static) num_threads(nthreads())
    for (int64_t n = 0; n < N; n++)
        for (int64_t k = 0; k < K; k++) bd[n * K + k] = code_at(b_codes, K, n, k) * orc_e4m3_value(b_scales[n * nb + k / 16]);
    const double alpha = (double)a_alpha * (double)b_alpha;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads())
    for (int64_t i = 0; i < R; i++) {
        int64_t m = rows ? rows[i] : i;
        if (m < 0 || m >= M) { err = 3; continue; }
        double* ad = (double*)malloc((size_t)K * sizeof(double) + 8);
        for (int64_t k = 0; k < K; k++) ad[k] = code_at(a_codes, K, m, k) * orc_e4m3_value(a_scales[m * nb + k / 16]);
        for (int64_t n = 0; n < N; n++) {
            double acc = 0.0;
            const double* br = bd + n * K;
            for (int64_t k = 0; k < K; k++) acc += ad[k] * br[k];
            double v = alpha * acc;
            if (ep) {
                if (ep->bias) v += bfv(ep->bias, n);
                if (ep->act == 1) v = gelu_tanh(v);
                if (ep->mod_scale || ep->mod_shift) {
                    double sc = ep->mod_scale ? bfv(ep->mod_scale, n) : 0.0;
                    double sh = ep->mod_shift ? bfv(ep->mod_shift, n) : 0.0;
                    v = v * (1.0 + sc) + sh;
                }
                if (ep->gate) v = bfv(ep->gate, n) * v;
                if (ep->residual) v = bfv(ep->residual, m * ep->ld_res + n) + v;
            }
            if (y) y[i * N + n] = v;
            if (out_bf16) out_bf16[i * N + n] = orc_f64_to_bf16(v);
        }
        free(ad);
    }
    free(bd);
    return err;
}

/* ------------------------------------------------------------------------ */
/* Exact GEMM for tiny inputs (pins orc_gemm): every decoded code times its  */
/* block scale is an integer multiple of 2^-10, so a product of two is a     */
/* multiple of 2^-20 and the sum over K is an exact integer.  With the two   */
/* binary32 tensor scales as integer * 2^e, the whole result is an integer   */
/* times a power of two, rounded once to bf16 here.                          */
/* ------------------------------------------------------------------------ */
typedef __int128 i128;

static int64_t scaled_int(double v) /* v * 2^10, exact integer */
{
    return (int64_t)ldexp(v, 10);
}

static void f32_parts(float f, int64_t* mant, int* ex) /* f = mant * 2^ex, mant integer */
{
    if (f == 0.0f) { *mant = 0; *ex = 0; return; }
    int e;
    double fr = frexp((double)f, &e); /* f = fr * 2^e, |fr| in [0.5,1) */
    *mant = (int64_t)ldexp(fr, 24);
    *ex = e - 24;
}

/* bf16 nearest-even of P * 2^E, P an exact integer */
static uint16_t bf16_of_scaled(i128 P, int E)
{
    if (P == 0) return 0;
    int neg = P < 0;
    unsigned __int128 u = neg ? (unsigned __int128)(-P) : (unsigned __int128)P;
    int top = 127;
    while (!((u >> top) & 1)) top--;
    /* value = u * 2^E, leading bit weight 2^(top+E) */
    int lead = top + E;
    int q = lead - 7; /* spacing exponent for 8 significant bits */
    if (q < -133) q = -133;
    int shift = q - E; /* number of low bits of u to drop */
    unsigned __int128 kept;
    if (shift <= 0) {
        kept = u << (-shift);
    } else if (shift >= 128) {
        kept = 0;
    } else {
        kept = u >> shift;
        unsigned __int128 rem = u - (kept << shift);
        unsigned __int128 half = (unsigned __int128)1 << (shift - 1);
        if (rem > half || (rem == half && (kept & 1))) kept += 1;
    }
    double r = ldexp((double)kept, q);
    if (neg) r = -r;
    return orc_f64_to_bf16(r); /* exact: r already has <= 8 significant bits */
}

ORC_API int orc_gemm_exact_bf16(const uint8_t* a_codes, const uint8_t* a_scales, float a_alpha,
                                const uint8_t* b_codes, const uint8_t* b_scales, float b_alpha, int64_t M,
                                int64_t N, int64_t K, uint16_t* out)
{
    if (K % 16 != 0 || K > 65536) return 1;
    const int64_t nb = K / 16;
    int64_t ma, mb;
    int ea, eb;
    f32_parts(a_alpha, &ma, &ea);
    f32_parts(b_alpha, &mb, &eb);
    for (int64_t m = 0; m < M; m++)
        for (int64_t n = 0; n < N; n++) {
            i128 S = 0;
            for (int64_t k = 0; k < K; k++) {
                int64_t av = scaled_int(code_at(a_codes, K, m, k) * orc_e4m3_value(a_scales[m * nb + k / 16]));
                int64_t bv = scaled_int(code_at(b_codes, K, n, k) * orc_e4m3_value(b_scales[n * nb + k / 16]));
                S += (i128)av * (i128)bv;
            }
            i128 P = S * (i128)ma * (i128)mb; /* |S| < 2^58, |ma|,|mb| < 2^24 */
            out[m * N + n] = bf16_of_scaled(P, ea + eb - 20);
        }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* KV cache [RN-I]: per (slot, K or V) quantization of a [T*H x d] chunk       */
/* ------------------------------------------------------------------------ */
/* Slot layout (R16): codes [T*H x d/2], scales row-major [T*H x d/16].
 * Bytes per slot per tensor: T*H*d*(1/2 + 1/16) = 9/16 * T*H*d, so K+V take
 * 9/8 * T*H*d bytes against 4 * T*H*d in bf16. */
ORC_API int64_t orc_kv_slot_bytes(int64_t T, int64_t H, int64_t d)
{
    int64_t rows = T * H;
    return rows * (d / 2) + rows * (d / 16);
}

/* x: bf16 chunk, token-major [T][H][d] (row r = t*H + h), row stride ld. */
ORC_API int orc_kv_append(const uint16_t* x, int64_t T, int64_t H, int64_t d, int64_t ld, uint8_t* codes,
                          uint8_t* scales, float* alpha)
{
    return orc_quantize_bf16(x, T * H, d, ld, ORC_MODE_COMPUTE, alpha, codes, scales);
}

/* As orc_kv_append with the R18 scale search. */
ORC_API int orc_kv_append_search46(const uint16_t* x, int64_t T, int64_t H, int64_t d, int64_t ld, uint8_t* codes,
                                   uint8_t* scales, float* alpha)
{
    return orc_quantize_bf16(x, T * H, d, ld, ORC_MODE_COMPUTE | ORC_MODE_SEARCH46, alpha, codes, scales);
}

ORC_API void orc_kv_dequant(const uint8_t* codes, const uint8_t* scales, float alpha, int64_t T, int64_t H,
                            int64_t d, uint16_t* out)
{
    orc_dequant_bf16(codes, scales, alpha, T * H, d, out);
}

/* ------------------------------------------------------------------------ */
/* LayerNorm + adaLN modulate + quantize (the step before the linear layer)  */
/* ------------------------------------------------------------------------ */
/* R19: per row r of x (bf16 [rows x cols], cols % 16 == 0), LayerNorm without
 * affine parameters, population variance, eps inside the square root:
 *   mu = (1/cols) sum_c x[c],  var = (1/cols) sum_c (x[c] - mu)^2,
 *   mean = fl32(mu),  rstd = fl32(1 / sqrt(var + eps)),
 * the sums, mu, var and the root taken in binary64 and each statistic rounded
 * once to binary32 (the definition, with no summation order of its own: a
 * binary64 sum of bf16 values is exact unless the row spans more than ~2^40 in
 * magnitude, and otherwise off by far less than a binary32 unit).  Then, with
 * (mean, rstd) as binary32 inputs, every element in binary32:
 *   m = fl32(fl32(fl32(fl32(x - mean) * rstd) * fl32(1 + scale[c])) + shift[c])
 *   (scale, shift bf16 [cols] or absent: 0),
 * and m is quantized as a binary32 tensor (R1..R8).  The statistics are an
 * input of the second part (orc_ln_modulate_given), so a kernel whose binary32
 * reductions land on slightly different statistics can be checked twice: its
 * statistics against orc_ln_stats within a summation bound, and its codes bit
 * for bit against the quantize of m built from its own statistics. */
ORC_API int orc_ln_stats(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, float eps, float* stats)
{
    if (cols <= 0 || ld < cols) return 1;
#pragma omp parallel for schedule(static) num_threads(nthreads())
    for (int64_t r = 0; r < rows; r++) {
        double s1 = 0.0;
        for (int64_t c = 0; c < cols; c++) s1 += (double)orc_bf16_to_f32(x[r * ld + c]);
        const double mu = s1 / (double)cols;
        double s2 = 0.0;
        for (int64_t c = 0; c < cols; c++) {
            const double d = (double)orc_bf16_to_f32(x[r * ld + c]) - mu;
            s2 += d * d;
        }
        const double var = s2 / (double)cols;
        stats[2 * r] = (float)mu;
        stats[2 * r + 1] = (float)(1.0 / sqrt(var + (double)eps));
    }
    return 0;
}

ORC_API int orc_ln_modulate_given(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, const float* stats,
                                  const uint16_t* scale, const uint16_t* shift, float* m)
{
    if (cols % 16 != 0 || ld < cols) return 1;
#pragma omp parallel for schedule(static) num_threads(nthreads())
    for (int64_t r = 0; r < rows; r++) {
        const float mean = stats[2 * r], rstd = stats[2 * r + 1];
        for (int64_t c = 0; c < cols; c++) {
            float h = (orc_bf16_to_f32(x[r * ld + c]) - mean) * rstd;
            float g = 1.0f + (scale ? orc_bf16_to_f32(scale[c]) : 0.0f);
            float t = h * g;
            m[r * cols + c] = t + (shift ? orc_bf16_to_f32(shift[c]) : 0.0f);
        }
    }
    return 0;
}

ORC_API int orc_ln_modulate(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, const uint16_t* scale,
                            const uint16_t* shift, float eps, float* m)
{
    if (cols % 16 != 0 || ld < cols) return 1;
    float* st = (float*)malloc((size_t)(rows > 0 ? rows : 1) * 2 * sizeof(float));
    if (!st) return 2;
    int rc = orc_ln_stats(x, rows, cols, ld, eps, st);
    if (rc == 0) rc = orc_ln_modulate_given(x, rows, cols, ld, st, scale, shift, m);
    free(st);
    return rc;
}

/* stats: binary32 (mean, rstd) per row to use, or NULL for orc_ln_stats' */
ORC_API int orc_ln_modulate_quantize(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld,
                                     const uint16_t* scale, const uint16_t* shift, float eps, const float* stats,
                                     int mode, float* alpha, uint8_t* codes, uint8_t* scales)
{
    float* m = (float*)malloc((size_t)(rows * cols) * sizeof(float) + 1);
    if (!m) return 2;
    int rc = stats ? orc_ln_modulate_given(x, rows, cols, ld, stats, scale, shift, m)
                   : orc_ln_modulate(x, rows, cols, ld, scale, shift, eps, m);
    if (rc == 0) rc = orc_quantize_f32(m, rows, cols, cols, mode, alpha, codes, scales);
    free(m);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* KV K-smoothing [RN-I] (R20): per chunk and tensor, each channel's mean     */
/* over the tokens is taken out before the quantize and put back at dequant  */
/* ------------------------------------------------------------------------ */
/* x: bf16 [T][C] (C = H*d channels, token t at x + t*C).  R20:
 * mean[c] = fl32((1/T) sum_t x[t][c]), the sum and the quotient in binary64
 * and rounded once to binary32 (the definition; a binary64 sum of bf16 values
 * is exact for any chunk of realistic range). */
ORC_API void orc_channel_mean(const uint16_t* x, int64_t T, int64_t C, float* mean)
{
#pragma omp parallel for schedule(static) num_threads(nthreads())
    for (int64_t c = 0; c < C; c++) {
        double s = 0.0;
        for (int64_t t = 0; t < T; t++) s += (double)orc_bf16_to_f32(x[t * C + c]);
        mean[c] = (float)(s / (double)T);
    }
}

/* x: bf16 chunk [T][H][d] (contiguous).  mean [H*d]: with mean_given == 0
 * written here (orc_channel_mean), else read as given (the means a kernel
 * stored, so its codes can be checked bit for bit against them); then
 * quantizes v = fl32(x - mean[h*d + j]) as orc_kv_append does (R15, R16; mode
 * may carry ORC_MODE_SEARCH46). */
ORC_API int orc_kv_append_smooth(const uint16_t* x, int64_t T, int64_t H, int64_t d, int mode, uint8_t* codes,
                                 uint8_t* scales, float* alpha, float* mean, int mean_given)
{
    const int64_t C = H * d;
    if (d % 16 != 0) return 1;
    if (!mean_given) orc_channel_mean(x, T, C, mean);
    float* v = (float*)malloc((size_t)(T * C) * sizeof(float) + 1);
    if (!v) return 2;
    for (int64_t t = 0; t < T; t++)
        for (int64_t c = 0; c < C; c++) v[t * C + c] = orc_bf16_to_f32(x[t * C + c]) - mean[c];
    int rc = orc_quantize_f32(v, T * H, d, d, ORC_MODE_COMPUTE | (mode & ORC_MODE_SEARCH46), alpha, codes, scales);
    free(v);
    return rc;
}

/* R20 dequant: x^ = bf16_rne(fl32(fl32(fl32(e2m1 * s) * a32) + mean[h*d + j]))
 * for row r = t*H + h, column j. */
ORC_API void orc_kv_dequant_smooth(const uint8_t* codes, const uint8_t* scales, float alpha, const float* mean,
                                   int64_t T, int64_t H, int64_t d, uint16_t* out)
{
    const int64_t rows = T * H, nb = d / 16;
#pragma omp parallel for schedule(static) num_threads(nthreads())
    for (int64_t r = 0; r < rows; r++)
        for (int64_t c = 0; c < d; c++) {
            float qs = (float)(code_at(codes, d, r, c) * orc_e4m3_value(scales[r * nb + c / 16]));
            float v = qs * alpha;
            float y = v + mean[(r % H) * d + c];
            out[r * d + c] = orc_f32_to_bf16(y);
        }
}

/* ------------------------------------------------------------------------ */
/* R24: rotary position embedding of a chunk's keys before the quantize       */
/* ------------------------------------------------------------------------ */
/* x: bf16 [T][H][d] (d even); cs, sn: binary32 [T][d/2], the cosine and sine
 * of the angle of token t's pair p.  For every token t, head h and pair p
 * (channels 2p and 2p+1 of the head), with c = cs[t][p], s = sn[t][p]:
 *   y[2p]   = fl32(fl32(x[2p] * c) - fl32(x[2p+1] * s))
 *   y[2p+1] = fl32(fl32(x[2p] * s) + fl32(x[2p+1] * c))
 * i.e. the complex product (x[2p] + i x[2p+1]) (c + i s), each product and
 * the sum rounded once in binary32. */
ORC_API void orc_rope(const uint16_t* x, int64_t T, int64_t H, int64_t d, const float* cs, const float* sn, float* y)
{
#pragma omp parallel for schedule(static) num_threads(nthreads())
    for (int64_t t = 0; t < T; t++)
        for (int64_t h = 0; h < H; h++) {
            const int64_t base = (t * H + h) * d;
            for (int64_t p = 0; p < d / 2; p++) {
                const float x0 = orc_bf16_to_f32(x[base + 2 * p]);
                const float x1 = orc_bf16_to_f32(x[base + 2 * p + 1]);
                const float c = cs[t * (d / 2) + p], s = sn[t * (d / 2) + p];
                const float a = x0 * c, b = x1 * s, e = x0 * s, f = x1 * c;
                y[base + 2 * p] = a - b;
                y[base + 2 * p + 1] = e + f;
            }
        }
}

/* R20's channel mean of binary32 values v [T][C]: fl32 of the binary64
 * mean, as orc_channel_mean. */
ORC_API void orc_channel_mean_f32(const float* v, int64_t T, int64_t C, float* mean)
{
#pragma omp parallel for schedule(static) num_threads(nthreads())
    for (int64_t c = 0; c < C; c++) {
        double s = 0.0;
        for (int64_t t = 0; t < T; t++) s += (double)v[t * C + c];
        mean[c] = (float)(s / (double)T);
    }
}

/* The keys' append with R24: y = orc_rope(x); with K-smoothing (mean != NULL)
 * the channel means of y (R20; computed here, or read as given when
 * mean_given != 0) and the quantize of fl32(y - mean), else the quantize of
 * y; a32 from the quantized values (R1), blocks and layout as orc_kv_append
 * (R15, R16; mode may carry ORC_MODE_SEARCH46). */
ORC_API int orc_kv_append_rope(const uint16_t* x, int64_t T, int64_t H, int64_t d, const float* cs,
                               const float* sn, int mode, uint8_t* codes, uint8_t* scales, float* alpha,
                               float* mean, int mean_given)
{
    const int64_t C = H * d;
    if (d % 16 != 0) return 1;
    float* y = (float*)malloc((size_t)(T * C) * sizeof(float) + 1);
    if (!y) return 2;
    orc_rope(x, T, H, d, cs, sn, y);
    if (mean) {
        if (!mean_given) orc_channel_mean_f32(y, T, C, mean);
        for (int64_t t = 0; t < T; t++)
            for (int64_t c = 0; c < C; c++) y[t * C + c] = y[t * C + c] - mean[c];
    }
    int rc = orc_quantize_f32(y, T * H, d, d, ORC_MODE_COMPUTE | (mode & ORC_MODE_SEARCH46), alpha, codes, scales);
    free(y);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Training-side NVFP4 [RN-T]: 2D block scaling of weights (R21), and the     */
/* transposed quantize with the Random Hadamard Transform (R22) for the      */
/* weight-gradient GEMM                                                      */
/* ------------------------------------------------------------------------ */
/* R21: x binary32 [rows x cols], rows and cols multiples of 16.  One E4M3
 * scale per 16 x 16 block: amax_b over its 256 elements, s = R3 of
 * fl32(amax_b / fl32(6 a32)), every element encoded with it (R4..R8); a32 from
 * the tensor amax (R1, mode COMPUTE) or given.  Outputs, either pair may be
 * NULL: codes [rows x cols/2] with logical scales [rows x cols/16] (row r,
 * column block j holds the scale of block (r/16, j): the per-row view the
 * block-scaled GEMM reads), and the transposed operand codes_t [cols x rows/2]
 * with scales_t [cols x rows/16] (the same codes and scales, transposed). */
ORC_API int orc_quantize_2d_f32(const float* x, int64_t rows, int64_t cols, int mode, float* alpha, uint8_t* codes,
                                uint8_t* scales, uint8_t* codes_t, uint8_t* scales_t)
{
    if (rows % 16 != 0 || cols % 16 != 0) return 1;
    init_tabs();
    float a32;
    if ((mode & ~ORC_MODE_SEARCH46) == ORC_MODE_COMPUTE) {
        float amax = 0.0f;
        for (int64_t i = 0; i < rows * cols; i++)
            if (fabsf(x[i]) > amax) amax = fabsf(x[i]);
        a32 = amax / 2688.0f; /* R1 */
        *alpha = a32;
    } else {
        a32 = *alpha;
    }
    const int64_t br = rows / 16, bc = cols / 16;
#pragma omp parallel for schedule(static) num_threads(nthreads())
    for (int64_t bi = 0; bi < br; bi++) {
        for (int64_t bj = 0; bj < bc; bj++) {
            float amax_b = 0.0f;
            for (int i = 0; i < 16; i++)
                for (int j = 0; j < 16; j++) {
                    float v = fabsf(x[(bi * 16 + i) * cols + bj * 16 + j]);
                    if (v > amax_b) amax_b = v;
                }
            uint8_t sc = 0, q[16][16];
            memset(q, 0, sizeof q);
            if (a32 != 0.0f) /* R2 */
                for (int i = 0; i < 16; i++) encode_block(x + (bi * 16 + i) * cols + bj * 16, amax_b, a32, 6.0f, &sc, q[i]);
            for (int i = 0; i < 16; i++) {
                const int64_t r = bi * 16 + i, c = bj * 16 + i;
                if (codes) {
                    for (int j = 0; j < 8; j++)
                        codes[r * (cols / 2) + bj * 8 + j] = (uint8_t)(q[i][2 * j] | (q[i][2 * j + 1] << 4));
                    scales[r * bc + bj] = sc;
                }
                if (codes_t) { /* row c of x^T: column bj*16 + i of x, its 16 rows bi*16 .. */
                    for (int j = 0; j < 8; j++)
                        codes_t[c * (rows / 2) + bi * 8 + j] = (uint8_t)(q[2 * j][i] | (q[2 * j + 1][i] << 4));
                    scales_t[c * br + bi] = sc;
                }
            }
        }
    }
    return 0;
}

ORC_API int orc_quantize_2d_bf16(const uint16_t* x, int64_t rows, int64_t cols, int mode, float* alpha,
                                 uint8_t* codes, uint8_t* scales, uint8_t* codes_t, uint8_t* scales_t)
{
    float* xf = (float*)malloc((size_t)(rows * cols) * sizeof(float) + 1);
    if (!xf) return 2;
    for (int64_t i = 0; i < rows * cols; i++) xf[i] = orc_bf16_to_f32(x[i]);
    int rc = orc_quantize_2d_f32(xf, rows, cols, mode, alpha, codes, scales, codes_t, scales_t);
    free(xf);
    return rc;
}

/* R22: the 16-point Random Hadamard Transform of one block, in binary32:
 * v_i = v_i * sign_i (sign_i = +1 or -1: exact), then the Walsh-Hadamard
 * butterflies for h = 1, 2, 4, 8: for every i with (i & h) == 0,
 * (v_i, v_{i+h}) <- (fl32(v_i + v_{i+h}), fl32(v_i - v_{i+h})), then
 * v_i = fl32(v_i * 0.25).  In exact arithmetic y = (1/4) H diag(sign) v with H
 * the 16 x 16 Sylvester Hadamard matrix (H_ij = (-1)^popcount(i & j)), an
 * orthogonal map. */
static void rht16(float* v, const int8_t* sign)
{
    for (int i = 0; i < 16; i++) v[i] = sign[i] < 0 ? -v[i] : v[i];
    for (int h = 1; h < 16; h <<= 1)
        for (int i = 0; i < 16; i++)
            if ((i & h) == 0) {
                float a = v[i], b = v[i + h];
                v[i] = a + b;
                v[i + h] = a - b;
            }
    for (int i = 0; i < 16; i++) v[i] = v[i] * 0.25f;
}

ORC_API void orc_rht16_f32(const float* in, int64_t n_blocks, const int8_t* sign, float* out)
{
    for (int64_t b = 0; b < n_blocks; b++) {
        float v[16];
        memcpy(v, in + b * 16, sizeof v);
        rht16(v, sign);
        memcpy(out + b * 16, v, sizeof v);
    }
}

/* x bf16 [rows x cols] (rows % 16 == 0, row stride ld): the operand of a GEMM
 * that contracts over x's rows (the weight-gradient GEMM contracts over the
 * tokens).  x^T [cols x rows] is quantized with 1D blocks of 16 along the rows
 * of x (R1..R8); with sign != NULL each block first goes through rht16 (R22),
 * and the tensor scale comes from the transformed values.  Codes
 * [cols x rows/2], logical scales [cols x rows/16]. */
ORC_API int orc_quantize_t_bf16(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, const int8_t* sign, int mode,
                                float* alpha, uint8_t* codes_t, uint8_t* scales_t)
{
    if (rows % 16 != 0 || ld < cols) return 1;
    float* xt = (float*)malloc((size_t)(rows * cols) * sizeof(float) + 1);
    if (!xt) return 2;
    for (int64_t r = 0; r < rows; r++)
        for (int64_t c = 0; c < cols; c++) xt[c * rows + r] = orc_bf16_to_f32(x[r * ld + c]);
    if (sign)
        for (int64_t c = 0; c < cols; c++)
            for (int64_t b = 0; b < rows / 16; b++) rht16(xt + c * rows + b * 16, sign);
    int rc = orc_quantize_f32(xt, cols, rows, rows, mode, alpha, codes_t, scales_t);
    free(xt);
    return rc;
}
