// quant.cuh -- the NVFP4 block quantizer as used inside libpact's kernels.
//
// NVFP4 ([FAQ]: PACT blog summary, section "相关问题", answer on NVFP4): 16 E2M1
// values share one E4M3 block scale.  Rounding, scale rule and saturation:
//   s = E4M3_RNE_sat(amax / 6);  c = sign << 3 | E2M1_RNE_sat(|x| / s).
// Work split: a warp owns 256 consecutive columns of one row; lane j holds the 8
// values [8j, 8j+8) of that chunk, so the 16-value block b lives in lanes 2b, 2b+1.
#pragma once
#include "common.cuh"

namespace pact {

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

// E2M1 code (4 bits incl. sign) -> float, exact.
__device__ __forceinline__ float e2m1_to_float(uint32_t c) {
    // magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6 as float bit patterns
    const uint32_t e = c & 7u;
    const uint32_t bits = (e == 0) ? 0u : (e == 1) ? 0x3F000000u : (e == 2) ? 0x3F800000u : (e == 3) ? 0x3FC00000u
                        : (e == 4) ? 0x40000000u : (e == 5) ? 0x40400000u : (e == 6) ? 0x40800000u : 0x40C00000u;
    return __uint_as_float(bits | ((c & 8u) << 28));
}

// |x| / s as the correctly rounded FP32 quotient would decide it, from the correctly
// rounded reciprocal r = 1/s: one product and one residual correction (Markstein,
// "Computation of elementary functions on the IBM RISC System/6000 processor",
// IBM J. Res. Dev. 34(1), 1990).  For BF16 |x| and E4M3 s this reproduces every
// rounding decision of the exact quotient (checked over all pairs by the tests).
__device__ __forceinline__ float quotient(float a, float s, float r) {
    float q0 = __fmul_rn(a, r);
    float e = __fmaf_rn(-q0, s, a);
    return __fmaf_rn(e, r, q0);
}

// Two non-negative values -> one byte of two E2M1 magnitude codes (lo in bits 0..3).
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi) {
    uint16_t r;
    asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u16.u8 %0, t;\n\t}"
        : "=h"(r)
        : "f"(hi), "f"(lo));
    return r & 0xFFu;
}

// amax -> E4M3 scale byte: RNE(amax / 6) with saturation.  The product with the
// correctly rounded FP32 value of 1/6 takes the same decision as the exact quotient
// for every BF16 amax (checked over all of them by the tests).
__device__ __forceinline__ uint32_t scale_byte(float amax) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(__fmul_rn(amax, 1.0f / 6.0f)));
    return r & 0xFFu;
}

// Quantize the 8 values of this lane (v[0] is the lowest column); the partner lane
// (lane ^ 1) holds the other half of the block.  All 32 lanes must call this.
// Returns the 4 code bytes (element 0 in the low nibble of byte 0); *sb gets the
// block's scale byte (identical in both lanes of the pair).
__device__ __forceinline__ uint32_t quant8(const float (&v)[8], uint32_t *sb) {
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
    amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
    const uint32_t b = scale_byte(amax);
    const float s = e4m3_to_float(b);
    const float r = b ? __frcp_rn(s) : 0.0f;
    uint32_t out = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float x0 = v[2 * i], x1 = v[2 * i + 1];
        uint32_t byte = e2m1x2(quotient(fabsf(x0), s, r), quotient(fabsf(x1), s, r));
        byte |= ((__float_as_uint(x0) >> 31) << 3) | ((__float_as_uint(x1) >> 31) << 7);
        out |= byte << (8 * i);
    }
    *sb = b;
    return out;
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
__device__ __forceinline__ void store_chunk(const pact_nvfp4_t &t, int64_t row, int64_t c0, uint32_t codes,
                                            uint32_t sb, bool valid) {
    const int lane = threadIdx.x & 31;
    const uint32_t packed = gather_scales4(sb);
    if (valid) {
        uint8_t *cp = static_cast<uint8_t *>(t.codes) + row * (t.cols >> 1) + ((c0 + 8 * lane) >> 1);
        *reinterpret_cast<uint32_t *>(cp) = codes;
        if ((lane & 7) == 0) {
            const int64_t blk = (c0 >> 4) + (lane >> 1);
            *reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(t.scales) + scale_offset(row, blk, t.cols)) = packed;
        }
    }
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

// Dequantize the 8 values [c, c+8) of row `row` (c a multiple of 8).
__device__ __forceinline__ void load8_nvfp4(const pact_nvfp4_t &t, int64_t row, int64_t c, float (&v)[8]) {
    const uint32_t codes =
        *reinterpret_cast<const uint32_t *>(static_cast<const uint8_t *>(t.codes) + row * (t.cols >> 1) + (c >> 1));
    const float s = e4m3_to_float(static_cast<const uint8_t *>(t.scales)[scale_offset(row, c >> 4, t.cols)]);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = e2m1_to_float((codes >> (4 * i)) & 15u) * s;
}

}  // namespace pact
