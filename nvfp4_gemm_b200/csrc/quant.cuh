// quant.cuh -- the NVFP4 block quantizer as used inside libpact's kernels.
//
// NVFP4 ([FAQ]: PACT blog summary, section "相关问题", answer on NVFP4): 16 E2M1
// values share one E4M3 block scale.  Rounding, scale rule and saturation:
//   s = E4M3_RNE_sat(amax / 6);  c = sign << 3 | E2M1_RNE_sat(|x| / s).
// Work split: a warp owns 256 consecutive columns of one row; lane j holds the 8
// values [8j, 8j+8) of that chunk, so the 16-value block b lives in lanes 2b, 2b+1.
#pragma once
#include <cuda_fp16.h>

#include "common.cuh"

namespace pact {

// Have the L2 prefetch `bytes` of global memory (source 16-byte aligned, bytes a
// multiple of 16); no completion to wait for.
__device__ __forceinline__ void bulk_prefetch_l2(const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// Byte offset of the scale of (row r, block c) in the tiled scale layout of a
// tensor with `cols` columns (cols a multiple of 64).
__host__ __device__ __forceinline__ int64_t scale_offset(int64_t r, int64_t c, int64_t cols) {
    return ((r >> 7) * (cols >> 6) + (c >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (c & 3);
}

// E4M3 byte (sign clear, never 0x7F) -> float, exact.
__device__ __forceinline__ float e4m3_to_float(uint32_t b) {
    uint32_t e = (b >> 3) & 15u, m = b & 7u;
    return e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : (float)m * 0.001953125f;
}

// One byte of two E2M1 codes (element 0 in the low nibble) -> two FP16 values
// (element 0 in the low half), exact: hardware conversion.
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte) {
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\t.reg .b16 w;\n\tcvt.u16.u32 w, %1;\n\tcvt.u8.u16 t, w;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
        : "=r"(r)
        : "r"(byte));
    return r;
}

// x / s as the correctly rounded FP32 quotient would decide it (for either sign of
// x: every step is symmetric in sign), from the correctly rounded reciprocal r = 1/s: one product and one residual correction (Markstein,
// "Computation of elementary functions on the IBM RISC System/6000 processor",
// IBM J. Res. Dev. 34(1), 1990).  For BF16 |x| and E4M3 s this reproduces every
// rounding decision of the exact quotient (checked over all pairs by the tests).
__device__ __forceinline__ float quotient(float a, float s, float r) {
    float q0 = __fmul_rn(a, r);
    float e = __fmaf_rn(-q0, s, a);
    return __fmaf_rn(e, r, q0);
}

// The negated quotients -(a/s) of a pair of values at once (packed FP32), with
// s2 = (s, s) and nr2 = (-r, -r).  Round-to-nearest is symmetric in sign, so each
// step is the negation of the corresponding step above: t = RN(a (-r)) = -RN(a r),
// e = RN(a + t s) is the same residual, and RN(t + e (-r)) = -quotient(a, s, r).
// Zeros come out with the sign opposite to a's (a = -0 gives +0, a = +0 gives -0),
// so flipping the sign bit of every code afterwards yields the codes of a / s with
// a's sign, -0 included, without a per-value sign copy.
__device__ __forceinline__ void neg_quotient2(float a0, float a1, uint64_t s2, uint64_t nr2, float &q0, float &q1) {
    const uint64_t a = f2_pack(a0, a1);
    const uint64_t t = f2_mul(a, nr2);
    const uint64_t e = f2_fma(t, s2, a);
    f2_unpack(f2_fma(e, nr2, t), q0, q1);
}
constexpr uint32_t CODE_SIGNS = 0x88888888u;   // the sign bit of all 8 codes of a word

// amax -> E4M3 scale byte: RNE(amax / 6) with saturation.  The product with the
// correctly rounded FP32 value of 1/6 takes the same decision as the exact quotient
// for every BF16 amax (checked over all of them by the tests).
__device__ __forceinline__ uint32_t scale_byte(float amax) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(__fmul_rn(amax, 1.0f / 6.0f)));
    return r & 0xFFu;
}

// max(|a|, |b|) of each BF16 half of two packed words (the sign bits come out as their
// XOR; a NaN half yields the other operand's half, as fmaxf does).
__device__ __forceinline__ uint32_t bf16x2_absmax(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// The E2M1 codes of 8 quotients (RNE, saturating, signs kept) as one word: element 0
// in the low nibble.
__device__ __forceinline__ uint32_t e2m1_word(const float *q) {
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out)
        : "f"(q[0]), "f"(q[1]), "f"(q[2]), "f"(q[3]), "f"(q[4]), "f"(q[5]), "f"(q[6]), "f"(q[7]));
    return out;
}

// Quantize the 8 values of this lane (v[0] is the lowest column); the partner lane
// (lane ^ 1) holds the other half of the block.  All 32 lanes must call this.
// Returns the 4 code bytes (element 0 in the low nibble of byte 0); *sb gets the
// block's scale byte (identical in both lanes of the pair).  The quotients keep the
// sign of x (a -0 input included: see neg_quotient2), and the hardware conversion
// rounds the magnitude and keeps the sign bit.
__device__ __forceinline__ uint32_t quant8(const float (&v)[8], uint32_t *sb) {
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
    amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
    const uint32_t b = scale_byte(amax);
    const float s = e4m3_to_float(b);
    const float nr = b ? -__frcp_rn(s) : -0.0f;
    const uint64_t nr2 = f2_pack(nr, nr), s2 = f2_pack(s, s);
    float q[8];
#pragma unroll
    for (int i = 0; i < 8; i += 2) neg_quotient2(v[i], v[i + 1], s2, nr2, q[i], q[i + 1]);
    *sb = b;
    return e2m1_word(q) ^ CODE_SIGNS;
}

// Codes and scale byte of a block whose magnitude maximum is amax, from the 16 values
// as 8 pairs (element 2j, 2j+1 in pair j).
template <typename Pair>
__device__ __forceinline__ void quant16_from(float amax, Pair pair, uint32_t *lo, uint32_t *hi, uint32_t *sb) {
    const uint32_t b = scale_byte(amax);
    const float s = e4m3_to_float(b);
    const float nr = b ? -__frcp_rn(s) : -0.0f;
    const uint64_t nr2 = f2_pack(nr, nr), s2 = f2_pack(s, s);
    float q[16];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        float a0, a1;
        pair(j, a0, a1);
        neg_quotient2(a0, a1, s2, nr2, q[2 * j], q[2 * j + 1]);
    }
    *lo = e2m1_word(q) ^ CODE_SIGNS;
    *hi = e2m1_word(q + 8) ^ CODE_SIGNS;
    *sb = b;
}

// Quantize one NVFP4 block of 16 BF16 values held by one thread as 8 packed words
// (values 2j, 2j+1 in the low and high half of word j of wa, wb): the 8 code bytes go to *lo
// (elements 0..7, element 0 in the low nibble) and *hi (8..15), the scale byte to
// *sb.  Same arithmetic as quant8, without the shuffle; the block maximum is taken on
// the packed words.
__device__ __forceinline__ void quant16_bf16(const uint4 wa, const uint4 wb, uint32_t *lo, uint32_t *hi, uint32_t *sb) {
    const uint32_t w[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
    const uint32_t m = bf16x2_absmax(bf16x2_absmax(bf16x2_absmax(w[0], w[1]), bf16x2_absmax(w[2], w[3])),
                                     bf16x2_absmax(bf16x2_absmax(w[4], w[5]), bf16x2_absmax(w[6], w[7])));
    // fmaxf with 0 first: a block of NaN only has amax 0, as a running fmaxf from 0 gives
    const float amax = fmaxf(0.0f, fmaxf(fabsf(bf16lo(m)), fabsf(bf16hi(m))));
    quant16_from(amax, [&](int j, float &a0, float &a1) { a0 = bf16lo(w[j]); a1 = bf16hi(w[j]); }, lo, hi, sb);
}

// quant16_bf16 for 16 FP32 values (the same decisions for values that are BF16).
__device__ __forceinline__ void quant16_f32(const float (&v)[16], uint32_t *lo, uint32_t *hi, uint32_t *sb) {
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < 16; ++j) amax = fmaxf(amax, fabsf(v[j]));
    quant16_from(amax, [&](int j, float &a0, float &a1) { a0 = v[2 * j]; a1 = v[2 * j + 1]; }, lo, hi, sb);
}

// Gather the scales of blocks 4q..4q+3 (lanes 8q, 8q+2, 8q+4, 8q+6) into lane 8q
// as one little-endian word; meaningful in lanes with lane % 8 == 0.
__device__ __forceinline__ uint32_t gather_scales4(uint32_t sb) {
    const uint32_t s1 = __shfl_down_sync(0xFFFFFFFFu, sb, 2);
    const uint32_t s2 = __shfl_down_sync(0xFFFFFFFFu, sb, 4);
    const uint32_t s3 = __shfl_down_sync(0xFFFFFFFFu, sb, 6);
    return sb | (s1 << 8) | (s2 << 16) | (s3 << 24);
}

// Store this lane's 4 code bytes and (from lanes 8q) the packed scales of a 256-column
// chunk starting at column c0 of row `row`.  `valid` is false for lanes whose 8
// columns lie past the end of the row (cols is a multiple of 64, so validity is
// uniform over each group of 8 lanes).
// Byte offsets of this lane's 4 code bytes and (lanes 8q) of its scale word inside
// a tensor with `cols` columns; tensors of one shape share them.
struct ChunkAt {
    int64_t code_off, scale_off;
};
__device__ __forceinline__ ChunkAt chunk_at(int64_t row, int64_t c0, int64_t cols) {
    const int lane = threadIdx.x & 31;
    return {row * (cols >> 1) + ((c0 + 8 * lane) >> 1), scale_offset(row, (c0 >> 4) + (lane >> 1), cols)};
}
__device__ __forceinline__ void store_chunk_at(const pact_nvfp4_t &t, const ChunkAt &at, uint32_t codes, uint32_t sb,
                                               bool valid) {
    const int lane = threadIdx.x & 31;
    const uint32_t packed = gather_scales4(sb);
    if (valid) {
        *reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(t.codes) + at.code_off) = codes;
        if ((lane & 7) == 0) *reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(t.scales) + at.scale_off) = packed;
    }
}
__device__ __forceinline__ void store_chunk(const pact_nvfp4_t &t, int64_t row, int64_t c0, uint32_t codes,
                                            uint32_t sb, bool valid) {
    store_chunk_at(t, chunk_at(row, c0, t.cols), codes, sb, valid);
}

// Load 8 BF16 values (16 bytes) as floats.
__device__ __forceinline__ void load8_bf16(const pact_bf16 *p, float (&v)[8]) {
    const uint4 u = *reinterpret_cast<const uint4 *>(p);
    v[0] = bf16lo(u.x); v[1] = bf16hi(u.x); v[2] = bf16lo(u.y); v[3] = bf16hi(u.y);
    v[4] = bf16lo(u.z); v[5] = bf16hi(u.z); v[6] = bf16lo(u.w); v[7] = bf16hi(u.w);
}
__device__ __forceinline__ void store8_bf16(pact_bf16 *p, const float (&v)[8]) {
    uint4 u;
    u.x = pack_bf16x2(v[0], v[1]); u.y = pack_bf16x2(v[2], v[3]);
    u.z = pack_bf16x2(v[4], v[5]); u.w = pack_bf16x2(v[6], v[7]);
    *reinterpret_cast<uint4 *>(p) = u;
}

// Dequantize 8 NVFP4 values: 4 code bytes (element 0 in the low nibble of byte 0)
// and their block's scale byte.  Exact: E2M1 pairs convert to FP16 in hardware, the
// product with the E4M3 scale has at most 6 significant bits and lies in
// [2^-10, 2688], so it is exact in FP16, and FP16 widens to FP32 exactly.
__device__ __forceinline__ void dequant8(uint32_t codes, uint32_t sbyte, float (&v)[8]) {
    const __half sh = __float2half_rn(e4m3_to_float(sbyte));  // exact: E4M3 values are FP16 values
    const __half2 s2 = __half2half2(sh);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t h = e2m1x2_to_f16x2((codes >> (8 * i)) & 0xFFu);
        const __half2 p = __hmul2(*reinterpret_cast<const __half2 *>(&h), s2);
        const float2 f = __half22float2(p);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}

// Dequantize the 8 values [c, c+8) of row `row` (c a multiple of 8).
__device__ __forceinline__ void load8_nvfp4(const pact_nvfp4_t &t, int64_t row, int64_t c, float (&v)[8]) {
    const uint32_t codes =
        *reinterpret_cast<const uint32_t *>(static_cast<const uint8_t *>(t.codes) + row * (t.cols >> 1) + (c >> 1));
    dequant8(codes, static_cast<const uint8_t *>(t.scales)[scale_offset(row, c >> 4, t.cols)], v);
}

// m = BF16_RNE(silu(g) * u), exactly rounded.  The FP32 evaluation with the fast
// exponential and division has a relative error of at most (5 + 1.16 |g|) FP32 ulps
// (CUDA's documented bounds for __expf and __fdividef plus three roundings), i.e. at
// most 2 (5 + 1.16 |g|) = 10 + 2.32 |g| ulps of the result: under 47.2 for |g| <= 16.
// It decides unless it lies within 48 ulps of a BF16 midpoint, and the double
// expression decides otherwise and for |g| > 16 (Ziv's method, as above).  One margin
// for every |g| keeps the test at three integer operations; the double path stays
// rare (about 0.15 % of values).
__device__ __forceinline__ float sigmoid_fast(float g) { return __fdividef(1.0f, 1.0f + __expf(-g)); }

// True when m = (g s) u (FP32, s = sigmoid_fast(g)) does not decide BF16_RNE(silu(g) u):
// m within 48 ulps of a BF16 midpoint, |g| > 16 or NaN, or (unless BOUNDED: u is known
// to be finite, so a finite g of at most 16 gives a finite m) m not finite.
template <bool BOUNDED>
__device__ __forceinline__ bool silu_undecided(float g, float m) {
    return ((__float_as_uint(m) + 0x8030u) & 0xFFFFu) <= 0x60u || !(fabsf(g) <= 16.0f) ||
           (!BOUNDED && !isfinite(m));
}
// BF16_RNE(silu(g) u) from the double expression (a BF16 value, returned as a float).
__device__ __forceinline__ float silu_exact(float g, float u) {
    const double gd = (double)g;
    return __bfloat162float(__double2bfloat16((gd / (1.0 + exp(-gd))) * (double)u));
}

// The value whose round-to-nearest BF16 conversion is BF16_RNE(silu(g) u): the FP32
// product where it decides, else the exactly rounded value itself.
template <bool BOUNDED = false>
__device__ __forceinline__ float silu_mul_value(float g, float u, float s) {
    const float m = __fmul_rn(__fmul_rn(g, s), u);
    return silu_undecided<BOUNDED>(g, m) ? silu_exact(g, u) : m;
}
__device__ __forceinline__ float silu_mul_out(float g, float u) { return silu_mul_value(g, u, sigmoid_fast(g)); }

// silu_mul_value for 8 values, the products two at a time (packed FP32, the same
// roundings) and the rounding test once for all 8: into mv.  The FP64 path stays
// inline: moved out of line (a call per undecided group) the kernels got 10 % slower.
template <bool BOUNDED>
__device__ __forceinline__ void silu_mul8(const float (&g)[8], const float (&u)[8], const float (&s)[8],
                                          float (&mv)[8]) {
    bool slow = false;
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
        f2_unpack(f2_mul(f2_mul(f2_pack(g[i], g[i + 1]), f2_pack(s[i], s[i + 1])), f2_pack(u[i], u[i + 1])),
                  mv[i], mv[i + 1]);
        slow |= silu_undecided<BOUNDED>(g[i], mv[i]) | silu_undecided<BOUNDED>(g[i + 1], mv[i + 1]);
    }
    if (slow) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if (silu_undecided<BOUNDED>(g[i], mv[i])) mv[i] = silu_exact(g[i], u[i]);
    }
}

// 8 packed BF16 values -> floats (element 0 in the low half of .x).
__device__ __forceinline__ void unpack8_bf16(const uint4 &u, float (&v)[8]) {
    v[0] = bf16lo(u.x); v[1] = bf16hi(u.x); v[2] = bf16lo(u.y); v[3] = bf16hi(u.y);
    v[4] = bf16lo(u.z); v[5] = bf16hi(u.z); v[6] = bf16lo(u.w); v[7] = bf16hi(u.w);
}
// Round 8 values to BF16 (round to nearest even, two per conversion): the packed
// words w (values 2j, 2j+1 in word j) and the rounded values as floats in r.
__device__ __forceinline__ void round8_bf16(const float (&v)[8], uint4 &w, float (&r)[8]) {
    w.x = pack_bf16x2(v[0], v[1]); w.y = pack_bf16x2(v[2], v[3]);
    w.z = pack_bf16x2(v[4], v[5]); w.w = pack_bf16x2(v[6], v[7]);
    unpack8_bf16(w, r);
}

// Row-major (row, 256-column chunk) tasks visited by a grid-stride loop without a
// division per task: the stride is split once into whole rows and a chunk remainder.
struct TaskIter {
    int64_t row;
    int64_t chunk, nchunk, drow, dchunk;
    __device__ __forceinline__ TaskIter(int64_t start, int64_t nchunk_, int64_t stride)
        : row(start / nchunk_), chunk(start % nchunk_), nchunk(nchunk_), drow(stride / nchunk_),
          dchunk(stride % nchunk_) {}
    __device__ __forceinline__ void next() {
        row += drow;
        chunk += dchunk;
        if (chunk >= nchunk) {
            chunk -= nchunk;
            ++row;
        }
    }
};

}  // namespace pact
