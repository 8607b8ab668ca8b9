/*
 * pact_oracle.c -- plain, slow, FP64 CPU oracle for the PACT NVFP4 data flow.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and bench.py's
 * cpu_baseline / reference arm may load this library.  It shares no code, header,
 * table or constant with the CUDA library under nvfp4_gemm_b200/ and neither side
 * includes the other.
 *
 * Sources (by page and section):
 *   [FAQ]    PACT blog summary (simolm.com), section "相关问题" (FAQ), answer "NVFP4
 *            量化是什么": 16 E2M1 elements share one E4M3 block scale, ~4.5 bit/element.
 *   [METHOD] same page, section "方法" (method): NVFP4 GEMM with FP32 accumulation and
 *            BF16 output for the forward and input-gradient GEMMs of the 7 frozen
 *            projections; RMSNorm output quantized and reused for backward; SiLU-multiply
 *            keeps BF16 in forward and saves NVFP4 copies of gate/up for backward;
 *            weight layouts for forward and backward rebuilt, transposed, re-quantized.
 *   [ABS]    PACT abstract (arxiv.science page), same data flow in English.
 *   [LORA]   PEFT explainer page (kongchang.com), section "LoRA", the low-rank
 *            update h = W0 x + B A x.
 * Readings of points the pages leave open: element codes round to nearest, ties to
 * the even code, onto {0, 0.5, 1, 1.5, 2, 3, 4, 6} and saturate at 6; the block scale
 * is E4M3_RNE(amax / 6), saturating at 448; there is no second-level per-tensor scale
 * (4 + 8/16 = 4.5 bit/element leaves no room for one); a value that rounds to zero
 * keeps its sign bit; a zero scale gives zero magnitudes.
 *
 * Every function is written from the definition, element by element, in the order
 * the definition states.  No blocking, no fusion, no reordering.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int orc_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ---------------------------------------------------------------- number formats */

/* BF16 bit pattern -> value (exact). */
double orc_bf16_value(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Round a double to BF16 (8 significant bits, 8 exponent bits) with a single
 * round-to-nearest-even step.  Finite inputs only. */
uint16_t orc_bf16_rne(double v) {
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (a == 0.0) return sign;
    int e;
    frexp(a, &e);             /* a = f * 2^e, f in [0.5, 1): 2^(e-1) <= a < 2^e */
    int E = e - 1;            /* binade exponent */
    if (E < -126) E = -126;   /* BF16 subnormal range has the quantum of the min normal binade */
    double quantum = ldexp(1.0, E - 7);
    double r = rint(a / quantum) * quantum;   /* a/quantum is exact (power of two) */
    if (r >= ldexp(1.0, 128)) return sign | 0x7F80;  /* overflow -> inf */
    float f = (float)r;       /* exact: r has <= 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, 4);
    return sign | (uint16_t)(u >> 16);
}

/* E4M3 (bias 7, no infinities, 0x7F/0xFF NaN) byte -> value, for bytes 0..0x7E. */
double orc_e4m3_value(uint8_t b) {
    int e = (b >> 3) & 0xF, m = b & 7;
    double v = (e == 0) ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
    return (b & 0x80) ? -v : v;
}

/* Nearest non-negative E4M3 value to v >= 0, ties to the even byte, values beyond the
 * largest finite value (448) saturate to 448.  Written as a search over all 127
 * non-negative finite bytes so that it is obviously the definition. */
uint8_t orc_e4m3_rne_sat(double v) {
    if (v >= 448.0) return 0x7E;
    int best = 0;
    double bestd = fabs(v - orc_e4m3_value(0));
    for (int b = 1; b <= 0x7E; ++b) {
        double d = fabs(v - orc_e4m3_value((uint8_t)b));
        if (d < bestd || (d == bestd && (b & 1) == 0 && (best & 1) == 1)) {
            best = b;
            bestd = d;
        }
    }
    return (uint8_t)best;
}

/* E2M1 magnitudes of codes 0..7. */
static const double E2M1_GRID[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double orc_e2m1_value(uint8_t c) {
    double v = E2M1_GRID[c & 7];
    return (c & 8) ? -v : v;
}

/* Nearest E2M1 magnitude code to q >= 0, ties to the even code, saturating at 6. */
uint8_t orc_e2m1_rne_mag(double q) {
    if (q >= 6.0) return 7;
    int best = 0;
    double bestd = fabs(q - E2M1_GRID[0]);
    for (int c = 1; c < 8; ++c) {
        double d = fabs(q - E2M1_GRID[c]);
        if (d < bestd || (d == bestd && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            bestd = d;
        }
    }
    return (uint8_t)best;
}

/* Element codes of real (double) values against given block scale bytes, as the
 * GPTQ calibration needs them (its working weights are not BF16):
 *   code_i = signbit(x_i) << 3 | E2M1_RNE_sat(|x_i| / E4M3(s_i)), magnitude 0 if s_i == 0. */
void orc_e2m1_codes_f64(const double *x, const uint8_t *sbytes, int64_t n, uint8_t *codes) {
    for (int64_t i = 0; i < n; ++i) {
        double s = orc_e4m3_value(sbytes[i]);
        uint8_t sign = signbit(x[i]) ? 8 : 0;
        uint8_t mag = (s == 0.0) ? 0 : orc_e2m1_rne_mag(fabs(x[i]) / s);
        codes[i] = sign | mag;
    }
}

/* Scale bytes of block maxima: E4M3_RNE_sat(amax_i / 6). */
void orc_e4m3_scales_f64(const double *amax, int64_t n, uint8_t *out) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_rne_sat(amax[i] / 6.0);
}

/* ------------------------------------------------------------ NVFP4 block quantizer */

/* Quantize one block of 16 BF16 values [FAQ]:
 *   amax = max |x_i|;  scale byte s = E4M3_RNE_sat(amax / 6);
 *   code_i = sign(x_i) << 3 | E2M1_RNE_sat(|x_i| / s)   (magnitude 0 when s == 0).
 * The division amax/6 and |x|/s are taken in double; at every rounding decision point
 * the exact quotient is representable, so the double quotient decides exactly. */
static void quantize_block(const uint16_t *x, uint8_t *codes16, uint8_t *scale) {
    double amax = 0.0;
    for (int i = 0; i < 16; ++i) {
        double a = fabs(orc_bf16_value(x[i]));
        if (a > amax) amax = a;
    }
    uint8_t sb = orc_e4m3_rne_sat(amax / 6.0);
    double s = orc_e4m3_value(sb);
    for (int i = 0; i < 16; ++i) {
        uint8_t sign = (x[i] & 0x8000) ? 8 : 0;
        uint8_t mag = (s == 0.0) ? 0 : orc_e2m1_rne_mag(fabs(orc_bf16_value(x[i])) / s);
        codes16[i] = sign | mag;
    }
    *scale = sb;
}

/* Quantize rows x cols BF16 (row stride ld elements) along the columns.
 * codes: rows x cols/2 bytes, element 2j in the low nibble, 2j+1 in the high nibble.
 * scales: rows x cols/16 bytes, plain row-major (use orc_pack_scales for the
 * device layout).  cols must be a multiple of 16. */
void orc_quantize(const uint16_t *x, int64_t ld, int64_t rows, int64_t cols,
                  uint8_t *codes, uint8_t *scales) {
    int64_t nb = cols / 16;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < nb; ++b) {
            uint8_t c16[16];
            quantize_block(x + r * ld + b * 16, c16, &scales[r * nb + b]);
            for (int j = 0; j < 8; ++j)
                codes[r * (cols / 2) + b * 8 + j] = (uint8_t)(c16[2 * j] | (c16[2 * j + 1] << 4));
        }
    }
}

/* value = E2M1(code) * E4M3(scale), exactly, into a rows x cols double matrix. */
void orc_dequantize(const uint8_t *codes, const uint8_t *scales, int64_t rows, int64_t cols,
                    double *out) {
    int64_t nb = cols / 16;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t c = 0; c < cols; ++c) {
            uint8_t byte = codes[r * (cols / 2) + c / 2];
            uint8_t code = (c & 1) ? (byte >> 4) : (byte & 15);
            out[r * cols + c] = orc_e2m1_value(code) * orc_e4m3_value(scales[r * nb + c / 16]);
        }
    }
}

/* ------------------------------------------------------------------- scale layout */
/* Device layout of the block scales: 512-byte tiles of 128 rows x 4 blocks.  Tiles
 * are ordered row-tile-major (all column tiles of rows 0..127 first).  Inside a
 * tile, (row r, block c) sits at (r % 32) * 16 + ((r % 128) / 32) * 4 + (c % 4).
 * Rows are padded to a multiple of 128 and blocks to a multiple of 4; padding is 0. */
int64_t orc_scale_bytes(int64_t rows, int64_t cols) {
    int64_t rp = (rows + 127) / 128 * 128;
    int64_t bp = (cols / 16 + 3) / 4 * 4;
    return rp * bp;
}

int64_t orc_scale_offset(int64_t r, int64_t c, int64_t cols) {
    int64_t tiles_per_row = (cols / 16 + 3) / 4;
    int64_t tile = (r / 128) * tiles_per_row + c / 4;
    return tile * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + (c % 4);
}

void orc_pack_scales(const uint8_t *plain, int64_t rows, int64_t cols, uint8_t *packed) {
    memset(packed, 0, (size_t)orc_scale_bytes(rows, cols));
    int64_t nb = cols / 16;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < nb; ++c)
            packed[orc_scale_offset(r, c, cols)] = plain[r * nb + c];
}

void orc_unpack_scales(const uint8_t *packed, int64_t rows, int64_t cols, uint8_t *plain) {
    int64_t nb = cols / 16;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < nb; ++c)
            plain[r * nb + c] = packed[orc_scale_offset(r, c, cols)];
}

/* ------------------------------------------------------------------------- GEMM */
/* C[m][n] = sum_k A[m][k] * B[n][k] in double, k ascending.  [METHOD] fixes FP32
 * accumulation on the device; the oracle accumulates exactly enough (double) that
 * its own rounding is far below the parity tolerance. */
void orc_gemm_nt(const double *A, const double *B, int64_t M, int64_t N, int64_t K, double *C) {
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) acc += A[m * K + k] * B[n * K + k];
            C[m * N + n] = acc;
        }
    }
}

/* ----------------------------------------------------------------------- RMSNorm */
/* [METHOD] RMSNorm whose BF16 output is then quantized (the quantization itself is
 * orc_quantize applied to y):  ms = sum x^2 / H;  rstd = 1 / sqrt(ms + eps);
 * y = BF16_RNE((x * rstd) * gamma), one rounding from double. */
void orc_rmsnorm(const uint16_t *x, const uint16_t *gamma, double eps, int64_t M, int64_t H,
                 uint16_t *y, double *rstd) {
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        double ss = 0.0;
        for (int64_t h = 0; h < H; ++h) {
            double v = orc_bf16_value(x[m * H + h]);
            ss += v * v;
        }
        double r = 1.0 / sqrt(ss / (double)H + eps);
        rstd[m] = r;
        for (int64_t h = 0; h < H; ++h)
            y[m * H + h] = orc_bf16_rne((orc_bf16_value(x[m * H + h]) * r) * orc_bf16_value(gamma[h]));
    }
}

/* [METHOD] SiLU-multiply from the BF16 gate/up values:
 * m = BF16_RNE((g / (1 + exp(-g))) * u). */
void orc_silu_mul(const uint16_t *g, const uint16_t *u, int64_t n, uint16_t *m) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        double gv = orc_bf16_value(g[i]), uv = orc_bf16_value(u[i]);
        m[i] = orc_bf16_rne((gv / (1.0 + exp(-gv))) * uv);
    }
}

/* Backward of m = silu(g) * u evaluated at the dequantized saved copies g^, u^
 * ([METHOD]: the NVFP4 copies of gate/up are what backward reads):
 *   s = sigmoid(g^);  dg = dm * u^ * s * (1 + g^ (1 - s));  du = dm * g^ * s. */
void orc_silu_mul_bwd(const double *dm, const double *gh, const double *uh, int64_t n,
                      double *dg, double *du) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        double s = 1.0 / (1.0 + exp(-gh[i]));
        dg[i] = dm[i] * uh[i] * s * (1.0 + gh[i] * (1.0 - s));
        du[i] = dm[i] * gh[i] * s;
    }
}

/* Backward of y = x * rstd * gamma (gamma frozen) from the dequantized saved output
 * y^ ([METHOD]: the quantized RMSNorm output is reused for backward):
 *   xn = y^ / gamma;  g = gamma * dy;  dx = rstd * (g - xn * mean(g * xn)). */
void orc_rmsnorm_bwd(const double *dy, const double *yh, const double *rstd,
                     const uint16_t *gamma, int64_t M, int64_t H, double *dx) {
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        double dot = 0.0;
        for (int64_t h = 0; h < H; ++h) {
            double gm = orc_bf16_value(gamma[h]);
            dot += (gm * dy[m * H + h]) * (yh[m * H + h] / gm);
        }
        double mean = dot / (double)H;
        for (int64_t h = 0; h < H; ++h) {
            double gm = orc_bf16_value(gamma[h]);
            dx[m * H + h] = rstd[m] * (gm * dy[m * H + h] - (yh[m * H + h] / gm) * mean);
        }
    }
}

/* Element-wise orc_bf16_rne over an array (the stage outputs the data flow stores
 * as BF16: GEMM outputs, gradients). */
void orc_bf16_rne_array(const double *v, int64_t n, uint16_t *out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = orc_bf16_rne(v[i]);
}
