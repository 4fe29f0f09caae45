/*
 * nvfp4_oracle.c -- plain, slow CPU reference of the NVFP4 W4A4 / NVFP4 KV-cache path.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the library links, includes or calls this file; only the
 * tests, the smoke check and the bench's CPU-baseline leg load it (through oracle/oracle.py).
 * It shares no code, header, table or constant generator with the CUDA path.
 *
 * What it follows.  "LongLive-2.0: An NVFP4 Parallel Infrastructure for Long Video Generation"
 * (arXiv 2605.18739; abstract as mirrored on fugumt.com, and the d9249.github.io review,
 * section "핵심 아이디어 / 구조 / 동작 방식") names the method: W4A4 NVFP4 linear layers and an
 * NVFP4 KV cache restored by a parallel dequantization kernel.  The pages never define NVFP4
 * numerically (landx.limxdynamics.com, section "什么是 NVFP4?", only says it is a 4-bit float
 * native to Blackwell).  The numeric reading used here is the NVFP4 format as published by the
 * OCP Microscaling / FP8 specifications:
 *   - element code E2M1: 1 sign, 2 exponent bits (bias 1), 1 mantissa bit, no inf/NaN;
 *   - block scale E4M3 "FN": 1 sign, 4 exponent bits (bias 7), 3 mantissa bits, no inf,
 *     S.1111.111 is NaN, max finite 448;
 *   - one scale per 16 consecutive elements, one FP32 per-tensor decode scale g;
 *   - round to nearest, ties to even, saturating to the largest finite value.
 * The op order of the quantizer (all FP32, IEEE round-to-nearest, no fused multiply-add):
 *   amax = max|x|;  g = amax/2688 (1 if amax == 0);  den = g*6;
 *   per 16-block:  b = max|x_i|;  sf = E4M3(b/den) (0 if b == 0);  d = sf*g;
 *                  if d == 0 all codes are 0, else r = 1/d and code_i = E2M1(x_i*r).
 * Dequantization: y = BF16(FP32(E2M1(c)*sf) * g).  GEMM reference: fp64 sum of products of the
 * fp64-exact dequantized operands, plus the optional bias or residual.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fPIC -shared (x86-64 SSE math).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_NONFINITE 3

/* ---------------------------------------------------------------- number formats ---------- */

/* E2M1 code -> value (exact).  Sign bit is bit 3. */
double orc_e2m1_value(int code)
{
    int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    double mag = (e == 0) ? 0.5 * (double)m : ldexp(1.0 + 0.5 * (double)m, e - 1);
    return s ? -mag : mag;
}

/* E4M3 (FN) byte -> value (exact); NaN for S.1111.111. */
double orc_e4m3_value(int byte)
{
    int s = (byte >> 7) & 1, e = (byte >> 3) & 15, m = byte & 7;
    double mag;
    if (e == 15 && m == 7) return NAN;
    mag = (e == 0) ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -mag : mag;
}

/* Nearest of the ascending magnitudes value(code_lo..code_hi), exact ties to the even code. */
static int nearest_code(double a, double (*value)(int), int code_lo, int code_hi)
{
    int best = code_lo, c;
    double bestd = fabs(a - value(code_lo));
    for (c = code_lo + 1; c <= code_hi; ++c) {
        double d = fabs(a - value(c));
        if (d < bestd || (d == bestd && (c & 1) == 0)) {
            best = c;
            bestd = d;
        }
    }
    return best;
}

/* FP32 -> E2M1 code, round to nearest even, saturating to +-6.  NaN -> 0x0. */
uint8_t orc_e2m1_encode(float q)
{
    int neg = signbit(q) ? 1 : 0;
    int mag;
    if (isnan(q)) return 0;
    /* at and beyond the largest magnitude the result saturates; checking this first also keeps
     * the fp64 distances below exact (for huge |q| they would round to equal values) */
    if (fabs((double)q) >= 6.0) mag = 7;
    else mag = nearest_code(fabs((double)q), orc_e2m1_value, 0, 7);
    return (uint8_t)((neg << 3) | mag);
}

/* FP32 -> E4M3 byte, round to nearest even, saturating to +-448.  NaN -> 0x7F. */
uint8_t orc_e4m3_encode(float v)
{
    int neg = signbit(v) ? 1 : 0;
    int mag;
    if (isnan(v)) return 0x7F;
    if (fabs((double)v) >= 448.0) mag = 0x7E;  /* saturate (see orc_e2m1_encode) */
    else mag = nearest_code(fabs((double)v), orc_e4m3_value, 0, 0x7E);
    return (uint8_t)((neg << 7) | mag);
}

float orc_bf16_to_float(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* FP32 -> BF16, round to nearest even (chosen between the two neighbouring BF16 values). */
uint16_t orc_bf16_from_float(float f)
{
    uint32_t u, lo_bits, hi_bits;
    float lo, hi;
    double dlo, dhi;
    memcpy(&u, &f, 4);
    if (isnan(f)) return (uint16_t)((u >> 16) | 0x0040);
    lo_bits = u & 0xFFFF0000u;                 /* toward zero */
    if (lo_bits == u) return (uint16_t)(u >> 16);
    hi_bits = lo_bits + 0x00010000u;           /* next BF16 away from zero (may be inf) */
    memcpy(&lo, &lo_bits, 4);
    memcpy(&hi, &hi_bits, 4);
    dlo = fabs((double)f - (double)lo);
    /* past the largest finite BF16 the upper neighbour is inf, which sits where 2^128 would */
    dhi = isinf(hi) ? ldexp(1.0, 128) - fabs((double)f) : fabs((double)hi - (double)f);
    if (dlo < dhi) return (uint16_t)(lo_bits >> 16);
    if (dhi < dlo) return (uint16_t)(hi_bits >> 16);
    return (uint16_t)((((lo_bits >> 16) & 1u) == 0) ? (lo_bits >> 16) : (hi_bits >> 16));
}

/* ---------------------------------------------------------------- layouts ----------------- */

/* Bytes of one packed code row: 2 codes per byte, padded to a multiple of 16 bytes. */
int64_t orc_codes_pitch(int64_t cols) { return 16 * ((cols + 31) / 32); }

/* Bytes of one linear scale row: one E4M3 per 16-element block. */
int64_t orc_sf_pitch(int64_t cols) { return (cols + 15) / 16; }

/* Size of the tensor-core scale layout: rows padded to 128, scale columns padded to 4. */
int64_t orc_sf_mma_bytes(int64_t rows, int64_t cols)
{
    int64_t r = 128 * ((rows + 127) / 128);
    int64_t c = 4 * ((orc_sf_pitch(cols) + 3) / 4);
    return r * c;
}

/* Offset of scale (row i, block b) in the tensor-core scale layout: 128-row x 4-block atoms of
 * 512 bytes, atoms ordered block-column fastest; inside an atom row i sits at
 * (i%32)*16 + ((i%128)/32)*4 and block b at b%4.  (PTX ISA, tcgen05 "block scaling" scale-factor
 * layout; the same layout cuBLASLt documents for VEC16_UE4M3 scales.) */
int64_t orc_sf_mma_offset(int64_t i, int64_t b, int64_t cols)
{
    int64_t atoms_per_row = (orc_sf_pitch(cols) + 3) / 4;
    return ((i / 128) * atoms_per_row + b / 4) * 512 + (i % 32) * 16 + ((i % 128) / 32) * 4 + (b % 4);
}

void orc_sf_linear_to_mma(const uint8_t *sf, int64_t rows, int64_t cols, uint8_t *out)
{
    int64_t i, b, nb = orc_sf_pitch(cols);
    memset(out, 0, (size_t)orc_sf_mma_bytes(rows, cols));
    for (i = 0; i < rows; ++i)
        for (b = 0; b < nb; ++b) out[orc_sf_mma_offset(i, b, cols)] = sf[i * nb + b];
}

/* ---------------------------------------------------------------- quantizer --------------- */

/* amax over a BF16 [rows, cols] matrix with row stride ld (elements). */
int orc_amax(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld, float *amax)
{
    int64_t i, j;
    float m = 0.0f;
    for (i = 0; i < rows; ++i)
        for (j = 0; j < cols; ++j) {
            float v = fabsf(orc_bf16_to_float(x[i * ld + j]));
            if (!isfinite(v)) return ORC_NONFINITE;
            if (v > m) m = v;
        }
    *amax = m;
    return ORC_OK;
}

/* Per-tensor decode scale g from amax. */
float orc_global_scale(float amax)
{
    if (amax == 0.0f) return 1.0f;
    return amax / 2688.0f;                      /* 2688 = 6 (E2M1 max) * 448 (E4M3 max) */
}

/*
 * Row-wise NVFP4 quantization of BF16 x[rows, cols] (row stride ld) with 16-element blocks
 * along each row.  codes: [rows][orc_codes_pitch(cols)], low nibble = even column, padding 0.
 * sf: linear [rows][orc_sf_pitch(cols)].  A trailing partial block is zero-padded.
 * amax_in (nullable) replaces the amax pass.  Returns ORC_NONFINITE on inf/NaN input.
 */
int orc_quantize_rows(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                      const float *amax_in, uint8_t *codes, uint8_t *sf, float *g_out)
{
    int64_t pitch = orc_codes_pitch(cols), nb = orc_sf_pitch(cols), i, blk;
    float amax, g, den;
    if (amax_in) {
        amax = *amax_in;
        if (!isfinite(amax)) return ORC_NONFINITE;
    } else if (orc_amax(x, rows, cols, ld, &amax) != ORC_OK) {
        return ORC_NONFINITE;
    }
    g = orc_global_scale(amax);
    den = g * 6.0f;
    *g_out = g;
    memset(codes, 0, (size_t)(rows * pitch));
    for (i = 0; i < rows; ++i) {
        for (blk = 0; blk < nb; ++blk) {
            float v[16], b = 0.0f, d, r;
            uint8_t s;
            int k;
            for (k = 0; k < 16; ++k) {
                int64_t j = blk * 16 + k;
                v[k] = (j < cols) ? orc_bf16_to_float(x[i * ld + j]) : 0.0f;
                if (fabsf(v[k]) > b) b = fabsf(v[k]);
            }
            s = (b == 0.0f) ? 0 : orc_e4m3_encode(b / den);
            sf[i * nb + blk] = s;
            d = (float)orc_e4m3_value(s) * g;
            if (d == 0.0f) continue;            /* whole block encodes as +0 */
            r = 1.0f / d;
            for (k = 0; k < 16; ++k) {
                int64_t j = blk * 16 + k;
                uint8_t c;
                if (j >= cols) break;
                c = orc_e2m1_encode(v[k] * r);
                codes[i * pitch + j / 2] |= (uint8_t)((j & 1) ? (c << 4) : c);
            }
        }
    }
    return ORC_OK;
}

/* Column-wise quantization = row-wise quantization of the transpose: 16-blocks run along the
 * rows of x.  Output rows = cols of x, output cols = rows of x.  Same g as row-wise. */
int orc_quantize_cols(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                      const float *amax_in, uint8_t *codes, uint8_t *sf, float *g_out)
{
    int64_t i, j;
    int st;
    uint16_t *xt = (uint16_t *)malloc((size_t)(rows * cols) * sizeof(uint16_t));
    if (!xt) return -1;
    for (i = 0; i < rows; ++i)
        for (j = 0; j < cols; ++j) xt[j * rows + i] = x[i * ld + j];
    st = orc_quantize_rows(xt, cols, rows, rows, amax_in, codes, sf, g_out);
    free(xt);
    return st;
}

/* ---------------------------------------------------------------- dequantizer ------------- */

/* y[rows][cols] (BF16, row stride ldy) = BF16(FP32(E2M1*sf) * g). */
void orc_dequant(const uint8_t *codes, const uint8_t *sf, float g, int64_t rows, int64_t cols,
                 uint16_t *y, int64_t ldy)
{
    int64_t pitch = orc_codes_pitch(cols), nb = orc_sf_pitch(cols), i, j;
    for (i = 0; i < rows; ++i)
        for (j = 0; j < cols; ++j) {
            uint8_t byte = codes[i * pitch + j / 2];
            int c = (j & 1) ? (byte >> 4) : (byte & 15);
            float prod = (float)(orc_e2m1_value(c) * orc_e4m3_value(sf[i * nb + j / 16]));
            y[i * ldy + j] = orc_bf16_from_float(prod * g);
        }
}

/* fp64 dequantized row: e2m1 * sf * g, exact in double. */
static void deq_row_f64(const uint8_t *codes, const uint8_t *sf, double g, int64_t cols,
                        double *out)
{
    int64_t j;
    for (j = 0; j < cols; ++j) {
        uint8_t byte = codes[j / 2];
        int c = (j & 1) ? (byte >> 4) : (byte & 15);
        out[j] = orc_e2m1_value(c) * orc_e4m3_value(sf[j / 16]) * g;
    }
}

/* fp64 dequantized matrix [rows][cols] (used for B operands and tests). */
void orc_dequant_f64(const uint8_t *codes, const uint8_t *sf, float g, int64_t rows, int64_t cols,
                     double *out)
{
    int64_t i, pitch = orc_codes_pitch(cols), nb = orc_sf_pitch(cols);
    for (i = 0; i < rows; ++i) deq_row_f64(codes + i * pitch, sf + i * nb, g, cols, out + i * cols);
}

/* ---------------------------------------------------------------- GEMM reference ---------- */

/*
 * y[r][n] = sum_k Adeq[m_r,k] * Bdeq[n,k]  (+ bias[n] | + resid[m_r*ldr + n]), in fp64, for the
 * listed rows m_r of A (row_list, nrows).  bdeq is B already dequantized to fp64 [N][K].
 * A uses linear scales.  alpha = gA*gB is inside the dequantized operands.
 */
void orc_gemm_rows(const uint8_t *a_codes, const uint8_t *a_sf, float ga, const double *bdeq,
                   int64_t N, int64_t K, const uint16_t *bias, const uint16_t *resid, int64_t ldr,
                   const int64_t *row_list, int64_t nrows, double *y)
{
    int64_t r, n, k, pitch = orc_codes_pitch(K), nb = orc_sf_pitch(K);
    double *arow = (double *)malloc((size_t)K * sizeof(double));
    if (!arow) return;
    for (r = 0; r < nrows; ++r) {
        int64_t m = row_list[r];
        deq_row_f64(a_codes + m * pitch, a_sf + m * nb, (double)ga, K, arow);
        for (n = 0; n < N; ++n) {
            const double *brow = bdeq + n * K;
            double acc = 0.0;
            for (k = 0; k < K; ++k) acc += arow[k] * brow[k];
            if (bias) acc += (double)orc_bf16_to_float(bias[n]);
            if (resid) acc += (double)orc_bf16_to_float(resid[m * ldr + n]);
            y[r * N + n] = acc;
        }
    }
    free(arow);
}

/* ---------------------------------------------------------------- array helpers (tests) --- */

void orc_e2m1_encode_n(const float *q, int64_t n, uint8_t *out)
{
    int64_t i;
    for (i = 0; i < n; ++i) out[i] = orc_e2m1_encode(q[i]);
}

void orc_e4m3_encode_n(const float *v, int64_t n, uint8_t *out)
{
    int64_t i;
    for (i = 0; i < n; ++i) out[i] = orc_e4m3_encode(v[i]);
}

void orc_bf16_from_float_n(const float *f, int64_t n, uint16_t *out)
{
    int64_t i;
    for (i = 0; i < n; ++i) out[i] = orc_bf16_from_float(f[i]);
}
