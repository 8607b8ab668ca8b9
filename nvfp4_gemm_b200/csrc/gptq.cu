// gptq.cu -- NVFP4-adapted GPTQ calibration of a frozen weight on the GPU.
//
// [METHOD] (PACT blog summary, section "方法", bullet 3; PACT abstract): the frozen
// weights are calibrated offline with GPTQ adapted to NVFP4, the statistics taken
// from the reconstructed NVFP4 inputs.  GPTQ is the published algorithm of Frantar
// et al. (2022): with H = 2 X~^T X~ / n the Hessian of the layer-wise loss, the
// columns of W are quantized in order and each column's error is pushed onto the
// columns not yet quantized through the upper Cholesky factor U of H^-1:
//     err = (w_j - q_j) / U[j, j],   W[:, j+1:] -= err U[j, j+1:].
// Readings: X~ = deq(q(X)) along K; a 16-column block's E4M3 scale is chosen when
// the pass reaches its first column, from the block's current (error-compensated)
// weights, by the quantizer's rule E4M3_RNE(amax / 6); dampening adds
// damp * mean(diag H) to the diagonal; a column no input reaches (H[i, i] = 0) gets
// H[i, i] = 1 and zero weights.
//
// Everything is FP64, so every discrete decision (scale byte, element code) is taken
// in the precision of the definition.  The pass is organised for the GPU:
//   X~ (FP64) <- the NVFP4 copy of X;  H = 2/n X~^T X~ (tiled FP64 product);
//   U = J L^-1 J with L the lower Cholesky factor of J H J (J reverses the index
//   order): J H J = L L^T gives H = (J L J)(J L J)^T with J L J upper, so
//   H^-1 = (J L^-1 J)^T (J L^-1 J) and J L^-1 J is the upper factor of H^-1;
//   columns are taken in blocks of 64: one thread per row quantizes the block's
//   columns in order, applying each column's update to the rest of the block, and a
//   tiled kernel then applies the block's updates to the remaining columns.  Both
//   updates subtract err * U[j, c] one column j at a time, in order, without fused
//   multiply-adds: each weight goes through the same operations, in the same order,
//   as in the column-by-column statement above.
#include <cmath>

#include "quant.cuh"

namespace pact {
namespace gptq {

constexpr int NB = 32;          // Cholesky / inverse block
constexpr int CB = 64;          // columns per quantization block
constexpr int ROWS = 128;       // rows (threads) per CTA of the column kernel

// ----------------------------------------------------------------- scalar rules
// E4M3_RNE_sat of v >= 0 (FP64): nearest E4M3 value, ties to the even byte,
// saturating at 448 (0x7E).  Subnormals are multiples of 2^-9 below 2^-6; a normal
// value with exponent e has 8 mantissa steps of 2^(e-3).
__device__ __forceinline__ uint32_t e4m3_rne_sat_f64(double v) {
    if (!(v < 448.0)) return 0x7Eu;
    if (v < 0.015625) {                                     // below 2^-6: step 2^-9
        const double m = rint(v * 512.0);                   // exact scaling; ties to even
        return (uint32_t)m;                                 // m = 8 is 2^-6 (byte 0x08)
    }
    int ex;
    const double f = frexp(v, &ex);                         // v = f 2^ex, f in [0.5, 1)
    const int e = ex - 1;                                   // v in [2^e, 2^(e+1))
    const double t = rint((ldexp(f, 1) - 1.0) * 8.0);       // mantissa steps, ties to even
    int m = (int)t, ee = e;
    if (m == 8) { m = 0; ++ee; }
    const uint32_t b = (uint32_t)(((ee + 7) << 3) | m);
    return b > 0x7Eu ? 0x7Eu : b;
}

__device__ __forceinline__ double e4m3_value_f64(uint32_t b) {
    const uint32_t e = (b >> 3) & 15u, m = b & 7u;
    return e ? ldexp(1.0 + m / 8.0, (int)e - 7) : ldexp((double)m, -9);
}

// E2M1 magnitude code of q >= 0: nearest of {0, .5, 1, 1.5, 2, 3, 4, 6}, ties to the
// even code, saturating at 6.  The midpoints 0.25 .. 5 count the codes passed; at a
// midpoint the comparison is strict when the lower code is even.
__device__ __forceinline__ uint32_t e2m1_mag_f64(double q) {
    return (uint32_t)(q > 0.25) + (q >= 0.75) + (q > 1.25) + (q >= 1.75) + (q > 2.5) + (q >= 3.5) + (q > 5.0);
}

__device__ __constant__ double kE2M1[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

// ----------------------------------------------------------------- kernels
// NVFP4 [rows x cols] -> FP64 (exact).
__global__ void k_dequant_f64(pact_nvfp4_t t, double *__restrict__ out) {
    pdl_wait();
    const int64_t per_row = t.cols / 8, n8 = t.rows * per_row;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / per_row, c = (i % per_row) * 8;
        float v[8];
        load8_nvfp4(t, r, c, v);
#pragma unroll
        for (int j = 0; j < 8; ++j) out[r * t.cols + c + j] = (double)v[j];
    }
}

// BF16 [rows x cols] (row stride ld) -> FP64 [rows x cols], zeroing the columns
// flagged dead.
__global__ void k_bf16_to_f64(const pact_bf16 *__restrict__ w, int64_t ld, int64_t rows, int64_t cols,
                              const int *__restrict__ dead, double *__restrict__ out) {
    pdl_wait();
    const int64_t n = rows * cols;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / cols, c = i % cols;
        out[i] = dead[c] ? 0.0 : (double)__uint_as_float((uint32_t)w[r * ld + c] << 16);
    }
}

// C[i, j] = alpha * sum_k A(i, k) B(k, j) + beta * C[i, j] with A(i, k) = A[i sai + k sak]
// and B(k, j) = B[k sbk + j sbj]: 64 x 64 tiles, 16-deep steps, 256 threads with 4 x 4
// outputs each.  lower: only tiles that touch the lower triangle (i >= j).
__global__ void __launch_bounds__(256) k_gemm_f64(int M, int N, int K, const double *__restrict__ A, int64_t sai,
                                                  int64_t sak, const double *__restrict__ B, int64_t sbk,
                                                  int64_t sbj, double *__restrict__ C, int64_t ldc, double alpha,
                                                  double beta, int lower) {
    pdl_wait();
    const int i0 = blockIdx.y * 64, j0 = blockIdx.x * 64;
    if (lower && j0 > i0 + 63) return;
    __shared__ double As[16][65], Bs[16][65];
    const int t = threadIdx.x, ti = (t / 16) * 4, tj = (t % 16) * 4;
    double acc[4][4] = {};
    const bool a_k_fast = sak == 1, b_k_fast = sbk == 1;
    for (int k0 = 0; k0 < K; k0 += 16) {
        for (int e = t; e < 1024; e += 256) {
            // coalesce along the unit-stride dimension
            const int kk = a_k_fast ? e % 16 : e / 64, ii = a_k_fast ? e / 16 : e % 64;
            const int gi = i0 + ii, gk = k0 + kk;
            As[kk][ii] = (gi < M && gk < K) ? A[gi * sai + gk * sak] : 0.0;
            const int kb = b_k_fast ? e % 16 : e / 64, jj = b_k_fast ? e / 16 : e % 64;
            const int gj = j0 + jj, gkb = k0 + kb;
            Bs[kb][jj] = (gj < N && gkb < K) ? B[gkb * sbk + gj * sbj] : 0.0;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
            double a[4], b[4];
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                a[x] = As[kk][ti + x];
                b[x] = Bs[kk][tj + x];
            }
#pragma unroll
            for (int x = 0; x < 4; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) acc[x][y] = fma(a[x], b[y], acc[x][y]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) {
            const int gi = i0 + ti + x, gj = j0 + tj + y;
            if (gi < M && gj < N) {
                double *c = C + (int64_t)gi * ldc + gj;
                *c = alpha * acc[x][y] + (beta != 0.0 ? beta * *c : 0.0);
            }
        }
}

// Dead columns (H[i, i] = 0): flag, and set H[i, i] = 1.
__global__ void k_dead_columns(double *H, int K, int *dead) {
    pdl_wait();
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < K; i += gridDim.x * blockDim.x) {
        const bool d = H[(int64_t)i * K + i] == 0.0;
        dead[i] = d;
        if (d) H[(int64_t)i * K + i] = 1.0;
    }
}

// Dampening, then the reversed copy R = J H J (one CTA computes the mean of the
// diagonal; every CTA adds it while copying).
__global__ void __launch_bounds__(256) k_damp_reverse(const double *__restrict__ H, int K, double damp,
                                                      double *__restrict__ R) {
    pdl_wait();
    __shared__ double red[256];
    double s = 0.0;
    for (int i = threadIdx.x; i < K; i += 256) s += H[(int64_t)i * K + i];
    red[threadIdx.x] = s;
    __syncthreads();
    for (int o = 128; o; o >>= 1) {
        if (threadIdx.x < o) red[threadIdx.x] += red[threadIdx.x + o];
        __syncthreads();
    }
    const double lambda = damp * (red[0] / K);
    const int64_t n = (int64_t)K * K;
    for (int64_t e = (int64_t)blockIdx.x * 256 + threadIdx.x; e < n; e += (int64_t)gridDim.x * 256) {
        const int64_t i = e / K, j = e % K;
        const double h = H[(K - 1 - i) * K + (K - 1 - j)];
        R[e] = i == j ? h + lambda : h;
    }
}

// Cholesky step for block column jb of the lower factor (in place in A, row-major
// K x K, trailing part already updated): every CTA factors the diagonal block in
// shared memory; CTA 0 writes it, CTA b > 0 solves row block jb + b:
// L[ib, jb] = A[ib, jb] L[jb, jb]^-T.  A pivot that is not positive sets *bad.
__global__ void __launch_bounds__(NB * NB / 4) k_chol_panel(double *A, int K, int jb, int *bad) {
    pdl_wait();
    __shared__ double D[NB][NB + 1];
    const int t = threadIdx.x, j0 = jb * NB;
    for (int e = t; e < NB * NB; e += blockDim.x) D[e / NB][e % NB] = A[(int64_t)(j0 + e / NB) * K + j0 + e % NB];
    __syncthreads();
    for (int k = 0; k < NB; ++k) {
        if (t == 0) {
            const double p = D[k][k];
            if (!(p > 0.0)) atomicExch(bad, 1);
            D[k][k] = sqrt(p > 0.0 ? p : 1.0);
        }
        __syncthreads();
        for (int i = k + 1 + t; i < NB; i += blockDim.x) D[i][k] /= D[k][k];
        __syncthreads();
        for (int e = t; e < NB * NB; e += blockDim.x) {
            const int i = e / NB, j = e % NB;
            if (j > k && i >= j) D[i][j] -= D[i][k] * D[j][k];
        }
        __syncthreads();
    }
    if (blockIdx.x == 0) {
        for (int e = t; e < NB * NB; e += blockDim.x) {
            const int i = e / NB, j = e % NB;
            A[(int64_t)(j0 + i) * K + j0 + j] = j <= i ? D[i][j] : 0.0;
        }
        return;
    }
    // row block ib: forward substitution x L^T = a, one thread per row (rows staged in
    // shared memory)
    __shared__ double Xr[NB][NB + 1];
    const int r0 = (jb + blockIdx.x) * NB;
    for (int e = t; e < NB * NB; e += blockDim.x) Xr[e / NB][e % NB] = A[(int64_t)(r0 + e / NB) * K + j0 + e % NB];
    __syncthreads();
    if (t < NB) {
        for (int j = 0; j < NB; ++j) {
            double v = Xr[t][j];
            for (int k = 0; k < j; ++k) v -= Xr[t][k] * D[j][k];
            Xr[t][j] = v / D[j][j];
        }
    }
    __syncthreads();
    for (int e = t; e < NB * NB; e += blockDim.x) A[(int64_t)(r0 + e / NB) * K + j0 + e % NB] = Xr[e / NB][e % NB];
}

// Inverse of the lower factor L, row block ib of X = L^-1 (rows ib NB .. + NB - 1,
// columns 0 .. (ib + 1) NB - 1): X[ib, :] = L[ib, ib]^-1 (E[ib, :] - T) with
// T = L[ib, 0:ib] X[0:ib, :] already in X[ib, 0 : ib NB] (from k_gemm_f64), E the
// identity's rows.  One CTA per 64 columns; each thread solves one column.
__global__ void __launch_bounds__(64) k_trtri_rows(const double *__restrict__ L, double *X, int K, int ib) {
    pdl_wait();
    __shared__ double D[NB][NB + 1];
    const int r0 = ib * NB;
    for (int e = threadIdx.x; e < NB * NB; e += 64) D[e / NB][e % NB] = L[(int64_t)(r0 + e / NB) * K + r0 + e % NB];
    __syncthreads();
    const int c = blockIdx.x * 64 + threadIdx.x;
    if (c >= r0 + NB) return;
    double x[NB];
#pragma unroll
    for (int i = 0; i < NB; ++i) {
        // right-hand side: -T (columns left of the block) or the identity
        double v = c < r0 ? -X[(int64_t)(r0 + i) * K + c] : (c - r0 == i ? 1.0 : 0.0);
        for (int k = 0; k < i; ++k) v -= D[i][k] * x[k];
        x[i] = v / D[i][i];
    }
#pragma unroll
    for (int i = 0; i < NB; ++i) X[(int64_t)(r0 + i) * K + c] = x[i];
}

// U = J X J (X = L^-1 lower, U upper), zero below the diagonal.
__global__ void k_reverse_upper(const double *__restrict__ X, int K, double *__restrict__ U) {
    pdl_wait();
    const int64_t n = (int64_t)K * K;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t i = e / K, j = e % K;
        U[e] = j >= i ? X[(K - 1 - i) * K + (K - 1 - j)] : 0.0;
    }
}

// Quantize columns c0 .. c0 + CB - 1 of W (FP64, N x K) in order, one thread per row.
// The row's CB weights sit in shared memory (thread-major); for column j: at a block
// start, the block's scale from the current weights; the code; the error
// e = (w_j - q_j) / U[j, j], recorded in E[row, j - c0]; and w_c -= e U[j, c] for the
// block's later columns.  Codes go to the NVFP4 codes (element 2j in the low nibble),
// scales to the tiled scale layout.
__global__ void __launch_bounds__(ROWS) k_gptq_cols(double *__restrict__ W, int N, int K, const double *__restrict__ U,
                                                    int c0, double *__restrict__ E, pact_nvfp4_t out) {
    pdl_wait();
    extern __shared__ double sm[];
    double *w = sm;                       // [CB][ROWS]
    double *u = sm + CB * ROWS;           // [CB][CB]: U[c0 + a, c0 + b]
    const int t = threadIdx.x, row = blockIdx.x * ROWS + t;
    for (int e = t; e < CB * CB; e += ROWS) u[e] = U[(int64_t)(c0 + e / CB) * K + c0 + e % CB];
    if (row < N)
        for (int j = 0; j < CB; ++j) w[j * ROWS + t] = W[(int64_t)row * K + c0 + j];
    __syncthreads();
    if (row >= N) return;
    double s = 0.0;
    uint32_t sbyte = 0, pair = 0;
    for (int j = 0; j < CB; ++j) {
        if (j % 16 == 0) {
            double amax = 0.0;
            for (int i = 0; i < 16; ++i) amax = fmax(amax, fabs(w[(j + i) * ROWS + t]));
            sbyte = e4m3_rne_sat_f64(__ddiv_rn(amax, 6.0));
            s = e4m3_value_f64(sbyte);
            static_cast<uint8_t *>(out.scales)[scale_offset(row, (c0 + j) / 16, K)] = (uint8_t)sbyte;
        }
        const double wj = w[j * ROWS + t];
        const uint32_t mag = s == 0.0 ? 0u : e2m1_mag_f64(__ddiv_rn(fabs(wj), s));
        const uint32_t code = (signbit(wj) ? 8u : 0u) | mag;
        const double q = (signbit(wj) ? -kE2M1[mag] : kE2M1[mag]) * s;
        const double err = __ddiv_rn(__dsub_rn(wj, q), u[j * CB + j]);
        E[(int64_t)row * CB + j] = err;
        for (int c = j + 1; c < CB; ++c) w[c * ROWS + t] = __dsub_rn(w[c * ROWS + t], __dmul_rn(err, u[j * CB + c]));
        if (j & 1) {
            static_cast<uint8_t *>(out.codes)[(int64_t)row * (K / 2) + (c0 + j) / 2] = (uint8_t)(pair | (code << 4));
        } else {
            pair = code;
        }
    }
}

// W[:, c] for c >= c0 + CB: w -= E[row, j] U[c0 + j, c], j = 0 .. CB - 1 in order, one
// multiply and one subtraction each (no fused multiply-add).  64 x 64 tiles.
__global__ void __launch_bounds__(256) k_gptq_trailing(double *__restrict__ W, int N, int K, const double *__restrict__ E,
                                                       const double *__restrict__ U, int c0) {
    pdl_wait();
    constexpr int JH = CB / 2;   // the block's columns in two halves (shared memory)
    __shared__ double Es[64][JH + 1], Us[JH][65];
    const int i0 = blockIdx.y * 64, cs = c0 + CB, j0 = cs + blockIdx.x * 64;
    const int t = threadIdx.x;
    const int ti = (t / 16) * 4, tj = (t % 16) * 4;
    double v[4][4];
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) {
            const int gi = i0 + ti + x, gj = j0 + tj + y;
            v[x][y] = (gi < N && gj < K) ? W[(int64_t)gi * K + gj] : 0.0;
        }
    for (int h = 0; h < 2; ++h) {
        __syncthreads();
        for (int e = t; e < 64 * JH; e += 256) {
            const int i = e / JH, j = e % JH;
            Es[i][j] = i0 + i < N ? E[(int64_t)(i0 + i) * CB + h * JH + j] : 0.0;
            const int a = e / 64, b = e % 64;
            Us[a][b] = j0 + b < K ? U[(int64_t)(c0 + h * JH + a) * K + j0 + b] : 0.0;
        }
        __syncthreads();
        for (int j = 0; j < JH; ++j) {
#pragma unroll
            for (int x = 0; x < 4; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) v[x][y] = __dsub_rn(v[x][y], __dmul_rn(Es[ti + x][j], Us[j][tj + y]));
        }
    }
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) {
            const int gi = i0 + ti + x, gj = j0 + tj + y;
            if (gi < N && gj < K) W[(int64_t)gi * K + gj] = v[x][y];
        }
}

// ----------------------------------------------------------------- host side
static size_t up256(size_t b) { return (b + 255) & ~(size_t)255; }

struct Layout {
    size_t xc, xs, xd, h, r, x, u, w, e, flags, total;
};

static Layout layout(int64_t N, int64_t K, int64_t n) {
    Layout l;
    size_t o = 0;
    auto take = [&](size_t b) { const size_t at = o; o += up256(b); return at; };
    l.xc = take(pact_nvfp4_code_bytes(n, K));
    l.xs = take(pact_scale_bytes(n, K));
    l.xd = take((size_t)(n * K) * 8);          // X~ in FP64
    l.h = take((size_t)(K * K) * 8);           // H
    l.r = take((size_t)(K * K) * 8);           // J H J, factored in place into L
    l.x = take((size_t)(K * K) * 8);           // L^-1
    l.u = take((size_t)(K * K) * 8);           // U
    l.w = take((size_t)(N * K) * 8);           // working weights
    l.e = take((size_t)(N * CB) * 8);          // one block's errors
    l.flags = take((size_t)(K + 1) * 4);       // dead columns, bad-pivot flag
    l.total = o;
    return l;
}

}  // namespace gptq
}  // namespace pact

using namespace pact;

extern "C" {

size_t pact_gptq_workspace_bytes(int64_t N, int64_t K, int64_t n) { return gptq::layout(N, K, n).total; }

pact_status pact_gptq_nvfp4(const pact_bf16 *W, int64_t ldw, int64_t N, int64_t K, const pact_bf16 *X, int64_t ldx,
                            int64_t n, double damp, void *workspace, size_t ws_bytes, const pact_nvfp4_t *out,
                            int *pivot_error, pact_stream_t stream) {
    using namespace gptq;
    PACT_CHECK(W && X && workspace && out, PACT_ERR_INVALID_ARG, "pact_gptq_nvfp4: NULL argument");
    PACT_CHECK(N >= 1 && N <= (1 << 20) && K >= 64 && K % 64 == 0 && K <= 32768 && n >= 1 && n <= (1 << 24),
               PACT_ERR_SHAPE, "pact_gptq_nvfp4: need 1 <= N <= 2^20, K a multiple of 64 in [64, 32768], 1 <= n <= 2^24");
    PACT_CHECK(damp >= 0.0 && std::isfinite(damp), PACT_ERR_INVALID_ARG, "pact_gptq_nvfp4: damp must be finite and >= 0");
    PACT_CHECK(ldw >= K && ldw % 8 == 0 && ldx >= K && ldx % 8 == 0 && aligned16(W) && aligned16(X) &&
                   ((uintptr_t)workspace & 255) == 0 && ((uintptr_t)pivot_error & 3) == 0,
               PACT_ERR_ALIGN, "pact_gptq_nvfp4: W, X 16-byte aligned with leading dims %% 8 == 0, workspace 256-byte "
               "aligned, pivot_error 4-byte aligned");
    PACT_CHECK(ws_bytes >= pact_gptq_workspace_bytes(N, K, n), PACT_ERR_INVALID_ARG,
               "pact_gptq_nvfp4: workspace too small (%zu < %zu)", ws_bytes, pact_gptq_workspace_bytes(N, K, n));
    pact_status s = check_nvfp4(out, N, K, "out");
    if (s != PACT_OK) return s;
    cudaStream_t st = (cudaStream_t)stream;
    const char *what = "pact_gptq_nvfp4";
    const Layout l = layout(N, K, n);
    uint8_t *base = static_cast<uint8_t *>(workspace);
    pact_nvfp4_t xq = {base + l.xc, base + l.xs, n, K};
    double *xd = reinterpret_cast<double *>(base + l.xd), *H = reinterpret_cast<double *>(base + l.h);
    double *R = reinterpret_cast<double *>(base + l.r), *Xi = reinterpret_cast<double *>(base + l.x);
    double *U = reinterpret_cast<double *>(base + l.u), *Wd = reinterpret_cast<double *>(base + l.w);
    double *E = reinterpret_cast<double *>(base + l.e);
    int *dead = reinterpret_cast<int *>(base + l.flags), *bad = dead + K;
    const int Ki = (int)K, Ni = (int)N;
    auto grid1 = [&](int64_t items) {
        int64_t g = (items + 255) / 256;
        const int64_t cap = (int64_t)sm_count() * 16;
        return (unsigned)(g < 1 ? 1 : (g > cap ? cap : g));
    };
    // X~ = deq(q(X)) in FP64
    s = pact_quantize_nvfp4(X, ldx, n, K, &xq, stream);
    if (s == PACT_OK) s = launch_dep(k_dequant_f64, dim3(grid1(n * K / 8)), dim3(256), 0, st, what, xq, xd);
    // H = 2/n X~^T X~ (lower triangle tiles are enough for the factorisation, but the
    // reversed copy reads all of H: compute it whole)
    if (s == PACT_OK)
        s = launch_dep(k_gemm_f64, dim3((unsigned)((K + 63) / 64), (unsigned)((K + 63) / 64)), dim3(256), 0, st, what,
                       Ki, Ki, (int)n, (const double *)xd, (int64_t)1, (int64_t)K, (const double *)xd, (int64_t)K,
                       (int64_t)1, H, (int64_t)K, 2.0 / (double)n, 0.0, 0);
    if (s == PACT_OK) s = launch_dep(k_dead_columns, dim3(grid1(K)), dim3(256), 0, st, what, H, Ki, dead);
    if (s == PACT_OK) {
        const cudaError_t e = cudaMemsetAsync(bad, 0, sizeof(int), st);
        if (e != cudaSuccess) return fail(PACT_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    }
    if (s == PACT_OK) s = launch_dep(k_damp_reverse, dim3(grid1(K * K)), dim3(256), 0, st, what, (const double *)H, Ki, damp, R);
    // lower Cholesky factor of J H J, in place
    const int nb = Ki / NB;
    for (int jb = 0; s == PACT_OK && jb < nb; ++jb) {
        s = launch_dep(k_chol_panel, dim3((unsigned)(nb - jb)), dim3(NB * NB / 4), 0, st, what, R, Ki, jb, bad);
        const int rest = Ki - (jb + 1) * NB;
        if (s == PACT_OK && rest > 0) {
            const double *Lp = R + (int64_t)(jb + 1) * NB * K + jb * NB;   // L[jb+1.., jb]
            double *Ap = R + (int64_t)(jb + 1) * NB * K + (jb + 1) * NB;
            s = launch_dep(k_gemm_f64, dim3((unsigned)((rest + 63) / 64), (unsigned)((rest + 63) / 64)), dim3(256), 0, st,
                           what, rest, rest, NB, Lp, (int64_t)K, (int64_t)1, Lp, (int64_t)1, (int64_t)K, Ap, (int64_t)K,
                           -1.0, 1.0, 1);
        }
    }
    // X = L^-1, one row block at a time (X starts at zero: its upper part stays zero)
    if (s == PACT_OK) {
        const cudaError_t e = cudaMemsetAsync(Xi, 0, (size_t)(K * K) * 8, st);
        if (e != cudaSuccess) return fail(PACT_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    }
    for (int ib = 0; s == PACT_OK && ib < nb; ++ib) {
        const int r0 = ib * NB;
        if (r0 > 0)   // T = L[ib, 0:r0] X[0:r0, 0:r0] into X[ib, 0:r0]
            s = launch_dep(k_gemm_f64, dim3((unsigned)((r0 + 63) / 64), 1), dim3(256), 0, st, what, NB, r0, r0,
                           (const double *)(R + (int64_t)r0 * K), (int64_t)K, (int64_t)1, (const double *)Xi, (int64_t)K,
                           (int64_t)1, Xi + (int64_t)r0 * K, (int64_t)K, 1.0, 0.0, 0);
        if (s == PACT_OK)
            s = launch_dep(k_trtri_rows, dim3((unsigned)((r0 + NB + 63) / 64)), dim3(64), 0, st, what, (const double *)R,
                           Xi, Ki, ib);
    }
    if (s == PACT_OK) s = launch_dep(k_reverse_upper, dim3(grid1(K * K)), dim3(256), 0, st, what, (const double *)Xi, Ki, U);
    // working weights (dead columns zeroed), then the column pass
    if (s == PACT_OK)
        s = launch_dep(k_bf16_to_f64, dim3(grid1(N * K)), dim3(256), 0, st, what, W, ldw, N, K, (const int *)dead, Wd);
    const size_t smem = (size_t)(CB * ROWS + CB * CB) * 8;
    if (s == PACT_OK) {
        const cudaError_t e = cudaFuncSetAttribute(k_gptq_cols, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return fail(PACT_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    }
    for (int c0 = 0; s == PACT_OK && c0 < Ki; c0 += CB) {
        s = launch_dep(k_gptq_cols, dim3((unsigned)((N + ROWS - 1) / ROWS)), dim3(ROWS), smem, st, what, Wd, Ni, Ki,
                       (const double *)U, c0, E, *out);
        if (s == PACT_OK && c0 + CB < Ki)
            s = launch_dep(k_gptq_trailing, dim3((unsigned)((Ki - c0 - CB + 63) / 64), (unsigned)((N + 63) / 64)),
                           dim3(256), 0, st, what, Wd, Ni, Ki, (const double *)E, (const double *)U, c0);
    }
    if (s == PACT_OK && N % 128) s = launch_dep(k_zero_scale_pad, dim3(64), dim3(256), 0, st, what, *out);
    if (s == PACT_OK && pivot_error) {
        const cudaError_t e = cudaMemcpyAsync(pivot_error, bad, sizeof(int), cudaMemcpyDeviceToDevice, st);
        if (e != cudaSuccess) return fail(PACT_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    }
    return s;
}

pact_status pact_weight_layout_cache_from_nvfp4(const pact_nvfp4_t *wf, int gexp, void *buf, size_t bytes,
                                                pact_weight_cache_t *out, pact_stream_t stream) {
    PACT_CHECK(wf && buf && out, PACT_ERR_INVALID_ARG, "pact_weight_layout_cache_from_nvfp4: NULL argument");
    const int64_t N = wf->rows, K = wf->cols;
    PACT_CHECK(N >= 64 && N % 64 == 0 && K >= 64 && K % 64 == 0, PACT_ERR_SHAPE,
               "pact_weight_layout_cache_from_nvfp4: N and K must be positive multiples of 64");
    PACT_CHECK(gexp >= -100 && gexp <= 100, PACT_ERR_INVALID_ARG, "pact_weight_layout_cache_from_nvfp4: |gexp| <= 100");
    pact_status s = check_nvfp4(wf, N, K, "wf");
    if (s != PACT_OK) return s;
    PACT_CHECK(bytes >= pact_weight_cache_bytes(N, K) && ((uintptr_t)buf & 255) == 0, PACT_ERR_INVALID_ARG,
               "pact_weight_layout_cache_from_nvfp4: buffer too small or not 256-byte aligned");
    cudaStream_t st = (cudaStream_t)stream;
    uint8_t *p = static_cast<uint8_t *>(buf);
    pact_weight_cache_t c;
    c.fwd.rows = N; c.fwd.cols = K;
    c.fwd.codes = p; p += gptq::up256(pact_nvfp4_code_bytes(N, K));
    c.fwd.scales = p; p += gptq::up256(pact_scale_bytes(N, K));
    c.bwd.rows = K; c.bwd.cols = N;
    c.bwd.codes = p; p += gptq::up256(pact_nvfp4_code_bytes(K, N));
    c.bwd.scales = p;
    c.gexp = gexp;
    cudaError_t e = cudaMemcpyAsync(c.fwd.codes, wf->codes, pact_nvfp4_code_bytes(N, K), cudaMemcpyDeviceToDevice, st);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(c.fwd.scales, wf->scales, pact_scale_bytes(N, K), cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return fail(PACT_ERR_CUDA, "pact_weight_layout_cache_from_nvfp4: %s", cudaGetErrorString(e));
    s = launch_dep(k_weight_bwd_layout, dim3((unsigned)(K / 64), (unsigned)(N / 64)), dim3(256), 0, st,
                   "pact_weight_layout_cache_from_nvfp4", c.fwd, c.bwd);
    if (s != PACT_OK) return s;
    if (K % 128) {
        s = launch_dep(k_zero_scale_pad, dim3(64), dim3(256), 0, st, "pact_weight_layout_cache_from_nvfp4", c.bwd);
        if (s != PACT_OK) return s;
    }
    *out = c;
    return PACT_OK;
}

}  // extern "C"
