/*
 * pact.h -- C ABI of libpact: the NVFP4 data flow through the seven frozen
 * projections of a LoRA decoder layer (PACT), for NVIDIA B200 (sm_100a).
 *
 * What each call computes is defined by the PACT pages:
 *   [FAQ]    PACT blog summary (simolm.com), section "相关问题" (FAQ), answer on
 *            NVFP4: 16 E2M1 values share one E4M3 block scale, ~4.5 bit/element.
 *   [METHOD] same page, section "方法" (method): bullet 1, NVFP4 GEMMs with FP32
 *            accumulation and BF16 output for the forward and the input gradient of
 *            the 7 frozen projections; bullet 2, the quantized RMSNorm output is
 *            reused for backward and SiLU-multiply keeps BF16 in forward while
 *            saving NVFP4 copies of gate/up; bullet 4, quantization fused into
 *            RMSNorm and SiLU-multiply, forward and backward weight layouts rebuilt,
 *            transposed, re-quantized and cached; the paragraph after the bullets,
 *            LoRA A and B stay BF16.
 *   [ABS]    PACT abstract (arxiv.science page): the same data flow.
 *   [LORA]   PEFT explainer (kongchang.com), section "LoRA": h = W0 x + B A x.
 *
 * Conventions shared by every call
 * --------------------------------
 * Numbers.  NVFP4 quantization of a block of 16 BF16 values x_i:
 *   scale byte  s = E4M3_RNE(amax / 6), saturating at 448 (never the NaN byte);
 *   element     c_i = sign(x_i) << 3 | E2M1_RNE(|x_i| / s), saturating at 6, ties to
 *               the even code, magnitude 0 when s == 0; the sign bit is kept even
 *               when the magnitude rounds to 0.
 *   value       E2M1(c_i) * E4M3(s), exact in FP32 and BF16.
 * Storage (pact_nvfp4_t).  Blocks run along the last dimension ("cols").  codes:
 *   rows x cols/2 bytes, row-major, element 2j in the low nibble of byte j.
 *   scales: pact_scale_bytes(rows, cols) bytes in 512-byte tiles of 128 rows x 4
 *   blocks; tiles are row-tile-major; inside a tile (row r, block c) is at byte
 *   (r % 32) * 16 + ((r % 128) / 32) * 4 + (c % 4).  Rows pad to 128 with zero bytes.
 *   The activations carry no per-tensor second-level scale (4 bits + 8/16 bits =
 *   4.5 bit/element).  Frozen weights may optionally carry one power of two per
 *   tensor (the two-level variant, pact_weight_layout_cache_scaled): a variant
 *   beyond the pages, for weights whose block scales would be subnormal E4M3.
 * Shapes.  cols of every NVFP4 tensor is a multiple of 64; rows >= 1 is free.
 *   Frozen weights are [N x K] (PyTorch [out, in]); N and K are multiples of 64.
 * Pointers.  Every pointer argument is DEVICE memory unless stated, 16-byte
 *   aligned; leading dimensions (ld*) are in elements and make each row start
 *   16-byte aligned.  The caller owns every buffer; libpact never allocates,
 *   frees or synchronises (except pact_get_device_status, which says so).
 * Streams.  Every call enqueues asynchronously on `stream` (a cudaStream_t; NULL
 *   is the legacy default stream) and returns once the work is enqueued.
 * Errors.  Arguments are checked on the host before anything is enqueued: a bad
 *   shape returns PACT_ERR_SHAPE, a misaligned pointer or leading dimension
 *   PACT_ERR_ALIGN, a NULL required pointer PACT_ERR_INVALID_ARG; nothing is
 *   launched then.  A failed launch returns PACT_ERR_CUDA.  Kernels bound every
 *   wait; a wait that runs out records PACT_ERR_TIMEOUT in a per-device status
 *   word read by pact_get_device_status.  pact_last_error() gives the message of
 *   the last failing call on the calling thread.
 */
#ifndef PACT_H
#define PACT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define PACT_ABI_VERSION 3

#if defined(__GNUC__)
#define PACT_API __attribute__((visibility("default")))
#else
#define PACT_API
#endif

typedef struct CUstream_st *pact_stream_t; /* cudaStream_t */
typedef uint16_t pact_bf16;                /* BF16 bit pattern */

typedef enum {
    PACT_OK = 0,
    PACT_ERR_INVALID_ARG = 1,
    PACT_ERR_SHAPE = 2,
    PACT_ERR_ALIGN = 3,
    PACT_ERR_CUDA = 4,
    PACT_ERR_TIMEOUT = 5,
    PACT_ERR_UNSUPPORTED = 6
} pact_status;

/* An NVFP4 tensor [rows x cols], blocks of 16 along cols (layout above).  The
 * struct itself is host memory; codes and scales point to device memory. */
typedef struct {
    void *codes;
    void *scales;
    int64_t rows, cols;
} pact_nvfp4_t;

/* The two cached layouts of one frozen weight W [N x K] ([METHOD] bullet 4):
 * fwd = q(W * 2^-gexp) [N x K] along K; bwd = q(deq(fwd)^T) [K x N] along N.
 * The weight the GEMMs use is 2^gexp * deq(layout); gexp is 0 for the plain
 * (one-level) layouts and a tensor exponent for the two-level variant. */
typedef struct {
    pact_nvfp4_t fwd;
    pact_nvfp4_t bwd;
    int32_t gexp;
} pact_weight_cache_t;

/* The LoRA branch fused into a frozen GEMM ([LORA]; [METHOD]: A, B in BF16).
 * Several projections that share an input can be concatenated along N (q|k|v,
 * gate|up): segment i covers output columns [seg_end[i-1], seg_end[i]) and has
 * its own rank-r adapter.
 * With R = nseg*r, the activations act are [M x 2R]: an FP32-accurate value held as
 * the unevaluated sum of two BF16 matrices, hi in columns 0..R-1 and lo in columns
 * R..2R-1 (lo = BF16(v - hi)), so the BF16 rounding of the small intermediate does
 * not reach the output.
 *   Forward  (pact_frozen_gemm_fwd):   act = T, T = scale * X A^T as written by
 *     pact_lora_fwd (segment i uses columns i*r .. i*r+r-1 of each half);
 *     weight = B [N x r] (segments' B stacked along rows); adds T_i . B_i^T.
 *   Dgrad    (pact_frozen_gemm_dgrad): act = U, U = scale * dY B as written by
 *     pact_lora_bwd_u; weight = A [R x K] (segments' A stacked along rows); adds
 *     U . A (one contraction over R).
 * r is 16, 32 or 48; nseg <= 3 and R <= 48; every internal boundary
 * seg_end[0..nseg-2] is a multiple of 256 and seg_end[nseg-1] == N.  act and
 * weight are row-major with leading dimension ld_act (>= 2R) / ld_weight. */
typedef struct {
    const pact_bf16 *act;
    int64_t ld_act;
    const pact_bf16 *weight;
    int64_t ld_weight;
    int r;
    int nseg;
    int64_t seg_end[4];
} pact_lora_t;

/* ---------------------------------------------------------------- sizes */
/* Bytes of the codes of an NVFP4 [rows x cols] tensor: rows * cols / 2. */
PACT_API size_t pact_nvfp4_code_bytes(int64_t rows, int64_t cols);
/* Bytes of its scales: round_up(rows, 128) * round_up(cols / 16, 4). */
PACT_API size_t pact_scale_bytes(int64_t rows, int64_t cols);
/* Bytes of the buffer pact_weight_layout_cache fills for W [N x K]: both
 * layouts, each part 256-byte aligned. */
PACT_API size_t pact_weight_cache_bytes(int64_t N, int64_t K);

/* ------------------------------------------------------- A2: quantize */
/* NVFP4 quantization of x [rows x cols] BF16 (row stride ldx) along cols
 * ([FAQ]; [METHOD] bullet 4: used for the attention output feeding o and for
 * every upstream gradient before its dgrad).  out->rows/cols must equal
 * rows/cols; out->codes/scales are written (scale padding included). */
PACT_API pact_status pact_quantize_nvfp4(const pact_bf16 *x, int64_t ldx, int64_t rows, int64_t cols,
                                const pact_nvfp4_t *out, pact_stream_t stream);

/* --------------------------------------------- A3: fused RMSNorm + quantize */
/* [METHOD] bullets 2 and 4.  For each row of x [M x H] (row stride ldx):
 *   rstd = 1 / sqrt(sum(x^2) / H + eps)            (double)
 *   y    = BF16_RNE((x * rstd) * gamma)            (exactly rounded)
 *   yq   = NVFP4(y)                                (the saved copy for backward)
 * y (the LoRA input of the forward, [M x H] row stride H) and rstd ([M] FP32)
 * may be NULL.  H is a multiple of 64 and at most 16384. */
PACT_API pact_status pact_rmsnorm_quant(const pact_bf16 *x, int64_t ldx, const pact_bf16 *gamma, float eps,
                               int64_t M, int64_t H, const pact_nvfp4_t *yq, pact_bf16 *y,
                               float *rstd, pact_stream_t stream);

/* ----------------------------------------- A4: fused SiLU-multiply + quantize */
/* [METHOD] bullet 2.  From BF16 gate g and up u ([M x I], shared row stride
 * ld_gu; e.g. the two halves of the gate|up GEMM output):
 *   m  = BF16_RNE(silu(g) * u)   -> m [M x I] (row stride I), the LoRA input of down
 *   mq = NVFP4(m)                -> the down GEMM operand
 *   gq = NVFP4(g), uq = NVFP4(u) -> the copies saved for backward (may be NULL)
 * m may be NULL.  I is a multiple of 64. */
PACT_API pact_status pact_silu_mul_quant(const pact_bf16 *g, const pact_bf16 *u, int64_t ld_gu, int64_t M,
                                int64_t I, pact_bf16 *m, const pact_nvfp4_t *mq,
                                const pact_nvfp4_t *gq, const pact_nvfp4_t *uq,
                                pact_stream_t stream);

/* ----------------------------------------------- A1: weight layout cache */
/* [METHOD] bullet 4.  Quantizes W [N x K] (BF16, row stride ldw) along K into the
 * forward layout and builds the backward layout q(deq(fwd)^T) [K x N] along N.
 * buf (device, >= pact_weight_cache_bytes(N, K) bytes, 256-byte aligned) receives
 * both; *out (host struct) is filled with pointers into buf.  Run once per frozen
 * weight; the result stays valid while buf lives. */
PACT_API pact_status pact_weight_layout_cache(const pact_bf16 *W, int64_t ldw, int64_t N, int64_t K,
                                     void *buf, size_t bytes, pact_weight_cache_t *out,
                                     pact_stream_t stream);

/* Two-level variant (beyond the pages: they give one E4M3 scale per block, [FAQ]).
 * Weights like N(0, 0.02^2) have block amax / 6 below E4M3's smallest normal
 * value 2^-6, so one-level block scales are subnormal with 2-3 significant bits.
 * Here a per-tensor power of two 2^gexp stands in front of the block scales:
 *   pact_absmax_bf16        *amax = max |x| over x [rows x cols] (row stride ldx),
 *                           written to device memory (amax: one float); finite x.
 *   pact_two_level_exponent (host, no GPU) the smallest integer e with
 *                           amax <= 6 * 448 * 2^e (0 for amax <= 0 or not finite),
 *                           so the largest block scale of W * 2^-e does not saturate.
 *   pact_weight_layout_cache_scaled  as pact_weight_layout_cache for W * 2^-gexp
 *                           (each product formed exactly in FP32; |gexp| <= 100,
 *                           else PACT_ERR_INVALID_ARG); out->gexp = gexp.
 * The caller reads *amax back to the host (libpact does not synchronise) and passes
 * the exponent on.  Products with a cache of exponent g are scaled by 2^g in the
 * GEMM epilogues (see pact_frozen_gemm_fwd); a power of two keeps that exact. */
PACT_API pact_status pact_absmax_bf16(const pact_bf16 *x, int64_t ldx, int64_t rows, int64_t cols, float *amax,
                                      pact_stream_t stream);
PACT_API int pact_two_level_exponent(float amax);
PACT_API pact_status pact_weight_layout_cache_scaled(const pact_bf16 *W, int64_t ldw, int64_t N, int64_t K,
                                                     int gexp, void *buf, size_t bytes, pact_weight_cache_t *out,
                                                     pact_stream_t stream);

/* ---------------------------------------------------- A5: forward GEMM */
/* [METHOD] bullet 1 with [LORA]:
 *   y[M x N] = BF16_RNE( residual + 2^g (deq(xq) . deq(w->fwd)^T + sum_i T_i . B_i^T) )
 * with g = w->gexp (0 for one-level layouts).  FP32 accumulation in tensor memory;
 * the LoRA term shares the accumulator, so for g != 0 the caller passes T computed
 * with scale * 2^-g (pact_lora_fwd's scale argument), which keeps it exact.  xq is
 * [M x K], w->fwd [N x K]; y has row stride ldy.  lora may be NULL (frozen GEMM
 * only); residual (BF16 [M x N], row stride ldr, e.g. the residual stream) may be
 * NULL and may equal y (in place). */
PACT_API pact_status pact_frozen_gemm_fwd(const pact_nvfp4_t *xq, const pact_weight_cache_t *w,
                                          const pact_lora_t *lora, const pact_bf16 *residual, int64_t ldr,
                                          pact_bf16 *y, int64_t ldy, pact_stream_t stream);

/* pact_frozen_gemm_fwd that also writes the NVFP4 copy of its output: y as above,
 * and q(y) of the BF16-rounded y, split along the columns into nq (1 or 2) NVFP4
 * tensors yq[0] (columns 0 .. yq[0].cols - 1) and yq[1] (the rest), each [M x cols_i],
 * cols_i multiples of 64 adding up to N.  [METHOD] bullet 2: the gate and up
 * projections' NVFP4 copies are what the backward keeps; quantizing them in the
 * GEMM epilogue, where the output rows are in registers, saves the SiLU-multiply
 * kernel two of its three quantizations. */
PACT_API pact_status pact_frozen_gemm_fwd_quant(const pact_nvfp4_t *xq, const pact_weight_cache_t *w,
                                                const pact_lora_t *lora, const pact_bf16 *residual, int64_t ldr,
                                                pact_bf16 *y, int64_t ldy, const pact_nvfp4_t *yq, int nq,
                                                pact_stream_t stream);

/* The gate|up GEMM fused with the SiLU-multiply ([METHOD] bullet 2): for the
 * concatenated gate|up weight (w->fwd [2I x K], gate rows first, I a multiple of
 * 256) it computes g|u = BF16_RNE(2^g (deq(xq) . deq(w->fwd)^T + LoRA)) exactly as
 * pact_frozen_gemm_fwd would, but writes, instead of g and u,
 *   m = BF16_RNE(silu(g) u)   [M x I], row stride ldm (>= I, multiple of 8)
 *   mq = q(m), gq = q(g), uq = q(u)   NVFP4 [M x I] each
 * with the same values as pact_silu_mul_quant on those g, u.  The tiles of gate and
 * up columns [256 j, 256 j + 256) run back to back on one CTA pair, so the gate block
 * waits in shared memory for its up block.  No residual; lora may be NULL. */
PACT_API pact_status pact_frozen_gemm_fwd_silu(const pact_nvfp4_t *xq, const pact_weight_cache_t *w,
                                               const pact_lora_t *lora, pact_bf16 *m, int64_t ldm,
                                               const pact_nvfp4_t *mq, const pact_nvfp4_t *gq,
                                               const pact_nvfp4_t *uq, pact_stream_t stream);

/* ------------------------------------------------------ A6: dgrad GEMM */
/* [METHOD] bullet 1 (input gradient) with [LORA]:
 *   dx[M x K] = BF16_RNE( residual + 2^g (deq(dyq) . deq(w->bwd)^T + U . A) )
 * with g = w->gexp; for g != 0, U comes from pact_lora_bwd_u with scale * 2^-g
 * (and pact_lora_bwd then takes u_gexp = g).  dyq is the NVFP4 upstream gradient
 * [M x N] (pact_quantize_nvfp4), w->bwd [K x N].  lora and residual may be NULL;
 * residual may equal dx (accumulate in place). */
PACT_API pact_status pact_frozen_gemm_dgrad(const pact_nvfp4_t *dyq, const pact_weight_cache_t *w,
                                            const pact_lora_t *lora, const pact_bf16 *residual, int64_t ldr,
                                            pact_bf16 *dx, int64_t lddx, pact_stream_t stream);

/* ------------------------------------------------------ A7: LoRA forward */
/* [LORA]: T = scale * X . A^T for X [M x K] (row stride ldx) and A [R x K] (row
 * stride K; R = nseg*r stacked adapters sharing X), FP32-accumulated and written
 * as hi + lo BF16 halves: T [M x 2R] (row stride ldt >= 2R), hi = BF16_RNE(t) in
 * columns 0..R-1, lo = BF16_RNE(t - hi) in columns R..2R-1.  R is 16, 32, 48 or 64;
 * the LoRA term fused into pact_frozen_gemm_fwd takes at most 48 columns (nseg*r <=
 * 48), so a T with R = 64 serves callers that use it outside that GEMM.
 * workspace (device, 16-byte aligned, >= pact_lora_fwd_workspace_bytes(M, K, R))
 * is caller-owned scratch for FP32 partial sums; its contents on entry do not
 * matter and calls that share it must not overlap on the GPU. */
PACT_API size_t pact_lora_fwd_workspace_bytes(int64_t M, int64_t K, int R);
PACT_API pact_status pact_lora_fwd(const pact_bf16 *x, int64_t ldx, int64_t M, int64_t K,
                                   const pact_bf16 *A, int R, float scale, pact_bf16 *T, int64_t ldt,
                                   void *workspace, size_t ws_bytes, pact_stream_t stream);

/* pact_lora_fwd that also writes xq = q(x) ([M x K], the NVFP4 copy of x exactly as
 * pact_quantize_nvfp4 writes it, padding rows' scales zeroed): the input of the
 * frozen GEMM that follows.  The kernel quantizes the tiles of x it streams for the
 * LoRA product, so x is read once for both.  xq must not overlap x, T or workspace. */
PACT_API pact_status pact_lora_fwd_quant(const pact_bf16 *x, int64_t ldx, int64_t M, int64_t K,
                                         const pact_bf16 *A, int R, float scale, pact_bf16 *T,
                                         int64_t ldt, const pact_nvfp4_t *xq, void *workspace,
                                         size_t ws_bytes, pact_stream_t stream);

/* [METHOD] + [LORA]: the down projection's LoRA input from the gate|up output, in
 * one kernel: m = BF16_RNE(silu(g) * u) exactly as pact_silu_mul_quant rounds it, its
 * NVFP4 copy mq = q(m) ([M x I], padding rows' scales zeroed), and T = scale * m .
 * A^T (hi + lo halves as pact_lora_fwd, R as there).  g and u are [M x I] with one row
 * stride ld_gu (the halves of the gate|up output).  m itself is written only when m
 * is not NULL (row stride ldm): the data flow needs mq and T, and skipping m saves
 * its write and its read by the LoRA product.  workspace as for pact_lora_fwd(M, I,
 * R).  Outputs must not overlap the inputs or the workspace.  PACT_ERR_SHAPE unless
 * M >= 1, I is a multiple of 64 and R is 16, 32, 48 or 64; PACT_ERR_ALIGN unless the
 * pointers are 16-byte aligned and the row strides multiples of 8 elements. */
PACT_API pact_status pact_lora_fwd_silu(const pact_bf16 *g, const pact_bf16 *u, int64_t ld_gu, int64_t M,
                                        int64_t I, const pact_bf16 *A, int R, float scale, pact_bf16 *T,
                                        int64_t ldt, const pact_nvfp4_t *mq, pact_bf16 *m, int64_t ldm,
                                        void *workspace, size_t ws_bytes, pact_stream_t stream);

/* Kernels one pact_lora_fwd (or _quant, or _silu with K = I) call launches for these sizes: 1 when the
 * product runs unsplit (its kernel writes T itself), 2 when a finalize kernel sums
 * the split contraction's partials. */
PACT_API int pact_lora_fwd_launches(int64_t M, int64_t K, int R);

/* pact_lora_fwd without a workspace argument.  The pages have no counterpart of
 * this call: it exists for callers that cannot allocate device memory where they
 * call the library (plain C callers without a device allocator, code that must not
 * call cudaMalloc because it may synchronise the device or because the device
 * memory budget is fixed at start-up).  Same arguments and results as
 * pact_lora_fwd; the scratch is an 8 MiB array inside the library's device code
 * that every GPU loading the library holds until the process exits.  Shapes whose
 * scratch (pact_lora_fwd_workspace_bytes) exceeds 8 MiB return PACT_ERR_SHAPE.
 * The first call on a device looks up the array's device address (a CUDA runtime
 * query, once per device, under a lock, so first calls from several host threads
 * are safe); make that first call before any stream capture.  The address is kept
 * for the life of the process: after cudaDeviceReset on a device this call must not
 * be used there again.  All calls on a device share the array, so calls that
 * overlap on the GPU (different streams) race.  A call whose kernel gave up a
 * bounded wait leaves NaN in T (never a previous call's values); as after every
 * call, pact_get_device_status reports it.  It allocates nothing. */
PACT_API pact_status pact_lora_fwd_noalloc(const pact_bf16 *x, int64_t ldx, int64_t M, int64_t K,
                                           const pact_bf16 *A, int R, float scale, pact_bf16 *T,
                                           int64_t ldt, pact_stream_t stream);

/* --------------------------------------------------- A8: LoRA backward */
/* [LORA] gradients, BF16 throughout ([METHOD]: adapters stay BF16).
 * pact_lora_bwd_u: U[:, i*r .. i*r+r-1] = scale * dY[:, seg_i] . B[seg_i, :] for dY
 *   [M x N] (row stride lddy), B [N x r]; written like T as hi + lo BF16 halves,
 *   U [M x 2*nseg*r] (row stride ldu).  U feeds pact_frozen_gemm_dgrad and
 *   pact_lora_bwd.  Segment ends are multiples of 64, the last equals N; r is 16,
 *   32, 48 or 64, nseg <= 3, nseg*r <= 64.  workspace as for pact_lora_fwd, at
 *   least pact_lora_bwd_u_workspace_bytes(M, N, r, nseg) bytes. */
PACT_API size_t pact_lora_bwd_u_workspace_bytes(int64_t M, int64_t N, int r, int nseg);
PACT_API pact_status pact_lora_bwd_u(const pact_bf16 *dy, int64_t lddy, int64_t M, int64_t N,
                                     const pact_bf16 *B, int r, int nseg, const int64_t *seg_end,
                                     float scale, pact_bf16 *U, int64_t ldu, void *workspace,
                                     size_t ws_bytes, pact_stream_t stream);

/* pact_lora_bwd_u that also writes dyq = q(dY) ([M x N], as pact_quantize_nvfp4
 * writes it): the input of the dgrad GEMM that follows, from the tiles of dY the
 * kernel streams for U.  dyq must not overlap dy, U or workspace. */
PACT_API pact_status pact_lora_bwd_u_quant(const pact_bf16 *dy, int64_t lddy, int64_t M, int64_t N,
                                           const pact_bf16 *B, int r, int nseg, const int64_t *seg_end,
                                           float scale, pact_bf16 *U, int64_t ldu, const pact_nvfp4_t *dyq,
                                           void *workspace, size_t ws_bytes, pact_stream_t stream);

/* Kernels one pact_lora_bwd_u (or _quant) call launches for these sizes (1 or 2, as
 * pact_lora_fwd_launches). */
PACT_API int pact_lora_bwd_u_launches(int64_t M, int64_t N, int r, int nseg, const int64_t *seg_end);

/* Kernels one pact_lora_bwd call launches for these sizes (X~ [M x K], R = nseg*r;
 * nvfp4_x non-zero when X~ is given as the saved NVFP4 copy): 4 or 5. */
PACT_API int pact_lora_bwd_launches(int64_t M, int64_t K, int R, int nvfp4_x);

/* The input X~ the adapter saw, as backward holds it: BF16 x, or the saved NVFP4
 * copy xq (dequantized on the fly); exactly one is non-NULL. */
typedef struct {
    int64_t M, N, K;
    const pact_bf16 *dy;      /* [M x N] BF16 upstream gradient, row stride lddy */
    int64_t lddy;
    const pact_bf16 *x;       /* [M x K] BF16, row stride ldx, or NULL */
    int64_t ldx;
    const pact_nvfp4_t *xq;   /* [M x K] NVFP4, or NULL */
    const pact_bf16 *A;       /* [nseg*r x K] */
    const pact_bf16 *U;       /* [M x 2*nseg*r] (hi + lo) from pact_lora_bwd_u, row stride ldu */
    int64_t ldu;
    int r, nseg;
    int64_t seg_end[4];
    float scale;
    int u_gexp;               /* U holds 2^-u_gexp times the gradient factor (0 usually) */
    void *dA;                 /* out [nseg*r x K]:  2^u_gexp (U_hi + U_lo)^T . X~ */
    void *dB;                 /* out [N x r]: rows seg_i = scale * dY[:, seg_i]^T . (X~ . A_i^T) */
    int grads_fp32;           /* 0: dA, dB are BF16 (pact_bf16 *); 1: FP32 (float *), unrounded,
                                 e.g. to be summed over data-parallel replicas before one
                                 rounding (pact_round_bf16) */
} pact_lora_bwd_t;

/* Scratch bytes pact_lora_bwd needs (T~ = X~ A^T and FP32 partial sums; an NVFP4
 * X~ is decoded inside the MMA kernel, no BF16 copy of it is made). */
PACT_API size_t pact_lora_bwd_workspace_bytes(int64_t M, int64_t N, int64_t K, int r, int nseg);
/* dA and dB of the adapters; workspace (device, 256-byte aligned, >=
 * pact_lora_bwd_workspace_bytes) is scratch owned by the caller; its contents on
 * entry do not matter and calls that share it must not overlap on the GPU. */
PACT_API pact_status pact_lora_bwd(const pact_lora_bwd_t *args, void *workspace, size_t ws_bytes,
                          pact_stream_t stream);

/* -------------------------------------- N1: NVFP4-adapted GPTQ calibration */
/* [METHOD] bullet 3 and the abstract: the frozen weights are calibrated offline with
 * GPTQ adapted to NVFP4, the statistics taken from the reconstructed NVFP4 inputs.
 * For W [N x K] (BF16, row stride ldw) and calibration inputs X [n x K] (BF16, row
 * stride ldx), with X~ = deq(q(X)) and H = 2 X~^T X~ / n:
 *   a column of H with H[i, i] = 0 gets H[i, i] = 1 and zero weights;
 *   H += damp * mean(diag H) * I;  U = the upper Cholesky factor of H^-1;
 *   for j = 0 .. K-1: at a 16-column block start, the block's scale byte is
 *   E4M3_RNE_sat(max |w| / 6) of its current weights; code_j = RNE onto the E2M1
 *   grid of w_j / scale (sign kept); err = (w_j - q_j) / U[j, j];
 *   W[:, j+1:] -= err U[j, j+1:].
 * All of it in FP64 (GPTQ: Frantar et al., 2022).  The codes and scales go to `out`
 * (NVFP4 [N x K], the forward weight layout); pact_weight_layout_cache_from_nvfp4
 * turns it into a weight cache.  N <= 2^20, K a multiple of 64 up to 32768, n <= 2^24.
 * workspace: device, 256-byte aligned, >= pact_gptq_workspace_bytes(N, K, n) bytes
 * (about 8 (n K + 4 K^2 + N K) bytes).  pivot_error (device int, may be NULL) gets 1
 * if the damped H was not positive definite (the result is then meaningless), else 0. */
PACT_API size_t pact_gptq_workspace_bytes(int64_t N, int64_t K, int64_t n);
PACT_API pact_status pact_gptq_nvfp4(const pact_bf16 *W, int64_t ldw, int64_t N, int64_t K,
                                     const pact_bf16 *X, int64_t ldx, int64_t n, double damp,
                                     void *workspace, size_t ws_bytes, const pact_nvfp4_t *out,
                                     int *pivot_error, pact_stream_t stream);
/* A1 from a given forward layout (e.g. a calibrated one): copies wf [N x K] into the
 * cache's forward part and builds the backward part q(deq(wf)^T); gexp as for
 * pact_weight_layout_cache_scaled (0 for one-level layouts).  buf as for
 * pact_weight_layout_cache. */
PACT_API pact_status pact_weight_layout_cache_from_nvfp4(const pact_nvfp4_t *wf, int gexp, void *buf,
                                                         size_t bytes, pact_weight_cache_t *out,
                                                         pact_stream_t stream);

/* y[i] = BF16_RNE(x[i]) for n FP32 values (device, 16-byte aligned): the one rounding of
 * gradients kept in FP32 (pact_lora_bwd with grads_fp32) after they were summed. */
PACT_API pact_status pact_round_bf16(const float *x, pact_bf16 *y, int64_t n, pact_stream_t stream);

/* ------------------------------------- A9: SiLU-multiply backward + quantize */
/* [METHOD] bullet 2 (backward reads the NVFP4 gate/up copies).  With
 * g^ = deq(gq), u^ = deq(uq), s = sigmoid(g^) and dm [M x I] (row stride lddm):
 *   dg = dm * u^ * s * (1 + g^ (1 - s)),  du = dm * g^ * s
 * written as BF16 into dgu [M x 2I] (dg in columns 0..I-1, du in I..2I-1, row
 * stride lddgu) and NVFP4-quantized (of the BF16 values) into dguq [M x 2I], the
 * operand of the gate|up dgrad.  m_re (nullable, [M x I], row stride I) receives
 * BF16_RNE(silu(g^) * u^), the down projection's LoRA input in backward. */
PACT_API pact_status pact_silu_mul_bwd_quant(const pact_bf16 *dm, int64_t lddm, const pact_nvfp4_t *gq,
                                    const pact_nvfp4_t *uq, int64_t M, int64_t I, pact_bf16 *dgu,
                                    int64_t lddgu, const pact_nvfp4_t *dguq, pact_bf16 *m_re,
                                    pact_stream_t stream);

/* ------------------------------------------------- A10: RMSNorm backward */
/* [METHOD] bullet 2 (backward reuses the quantized RMSNorm output).  With
 * y^ = deq(yq), xn = y^ / gamma, g = gamma * dy (dy [M x H], row stride lddy):
 *   dx = rstd * (g - xn * mean(g * xn))  (+ dres when dres != NULL, the residual
 *   stream's gradient), written as BF16 to dx [M x H] (row stride H) and, when
 *   dxq != NULL, NVFP4-quantized (of the BF16 values) into dxq.
 * H is a multiple of 64 and at most 16384. */
PACT_API pact_status pact_rmsnorm_bwd(const pact_bf16 *dy, int64_t lddy, const pact_nvfp4_t *yq,
                             const float *rstd, const pact_bf16 *gamma, int64_t M, int64_t H,
                             const pact_bf16 *dres, pact_bf16 *dx, const pact_nvfp4_t *dxq,
                             pact_stream_t stream);

/* ------------------------------------------------------------ status */
/* Message of the last failing call on this thread ("" if none). */
PACT_API const char *pact_last_error(void);
/* Name of a status code. */
PACT_API const char *pact_status_string(pact_status s);
/* Synchronises `stream`, then reads and clears the status word of the current
 * device: PACT_OK, or PACT_ERR_TIMEOUT if a kernel gave up a bounded wait. */
PACT_API pact_status pact_get_device_status(pact_stream_t stream);
/* PACT_ABI_VERSION of the loaded library. */
PACT_API int pact_abi_version(void);
/* Self-test of the failure path (the pages have no counterpart; it tests the
 * library's bounded waits): one kernel thread waits on an mbarrier that nothing
 * completes, through the same bounded wait every libpact kernel uses, with a limit
 * of limit_cycles SM clock cycles (1e3 .. 4e9).  The wait runs out, the kernel
 * records PACT_ERR_TIMEOUT in the device status word (read and cleared by
 * pact_get_device_status) and returns; nothing asynchronous is left in flight and
 * the context stays usable.  waited_cycles (device, 8-byte aligned, may be NULL)
 * receives the cycles the wait took. */
PACT_API pact_status pact_selftest_wait_timeout(int64_t limit_cycles, unsigned long long *waited_cycles,
                                                pact_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* PACT_H */
