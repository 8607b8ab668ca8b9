// quant.cu -- HBM-bound kernels of the PACT data flow: NVFP4 quantize, the fused
// RMSNorm / SiLU-multiply quantizers, their backward kernels and the weight layout
// cache.  All of them stream BF16 with 16-byte vector accesses (a warp moves 512
// contiguous bytes per instruction) and quantize with warp-shuffle block maxima.
#include <math.h>

#include <cmath>

#include "quant.cuh"

namespace pact {

constexpr int CHUNK = 256;  // columns per warp task

// Rows padded to 128 for the scale layout; padding rows get zero scales.
__device__ __forceinline__ void zero_pad_scales(const pact_nvfp4_t &t, int64_t row, int64_t c0) {
    const int lane = threadIdx.x & 31;
    if ((lane & 7) == 0 && c0 + 8 * lane < t.cols) {
        const int64_t blk = (c0 >> 4) + (lane >> 1);
        *reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(t.scales) + scale_offset(row, blk, t.cols)) = 0u;
    }
}

// ------------------------------------------------------------------ A2: quantize
// A warp task is 512 columns of a row: lane j quantizes the 16-value block j on its
// own (no block-maximum shuffle, one scale computation per block), writes its 8 code
// bytes and its scale byte.  prescale: a power of two the values are multiplied by
// first (exact in FP32); 1 for every quantization on the step path, 2^-gexp for
// two-level weight layouts.
constexpr int QCHUNK = 512;
__global__ void __launch_bounds__(256) k_quantize(const pact_bf16 *__restrict__ x, int64_t ldx, int64_t rows,
                                                  pact_nvfp4_t out, float prescale) {
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int64_t nchunk = (out.cols + QCHUNK - 1) / QCHUNK;
    const int64_t rows_pad = (rows + 127) & ~int64_t(127);
    const int64_t warp0 = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    uint8_t *codes = static_cast<uint8_t *>(out.codes), *scales = static_cast<uint8_t *>(out.scales);
    auto load = [&](const TaskIter &t, uint4 &a, uint4 &b) {
        const int64_t c = t.chunk * QCHUNK + 16 * lane;
        a = b = make_uint4(0, 0, 0, 0);
        if (t.row < rows && c < out.cols) {
            const uint4 *p = reinterpret_cast<const uint4 *>(x + t.row * ldx + c);
            a = p[0];
            b = p[1];
        }
    };
    TaskIter it(warp0, nchunk, nwarps);
    uint4 ca, cb;
    if (it.row < rows_pad) load(it, ca, cb);
    while (it.row < rows_pad) {    // software-pipelined: the next task's loads are in flight
        TaskIter nx = it;
        nx.next();
        uint4 na = make_uint4(0, 0, 0, 0), nb = make_uint4(0, 0, 0, 0);
        if (nx.row < rows_pad) load(nx, na, nb);
        const int64_t row = it.row;
        const int64_t c = it.chunk * QCHUNK + 16 * lane;
        if (c < out.cols) {
            uint8_t *sp = scales + scale_offset(row, c >> 4, out.cols);
            if (row >= rows) {
                *sp = 0;   // a padding row of the scale layout
            } else {
                uint32_t lo, hi, sb;
                if (prescale != 1.0f) {   // uniform over the launch; the FP32 products are exact
                    float v[16];
                    unpack8_bf16(ca, *reinterpret_cast<float(*)[8]>(v));
                    unpack8_bf16(cb, *reinterpret_cast<float(*)[8]>(v + 8));
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] *= prescale;
                    quant16_f32(v, &lo, &hi, &sb);
                } else {
                    quant16_bf16(ca, cb, &lo, &hi, &sb);
                }
                *reinterpret_cast<uint2 *>(codes + row * (out.cols >> 1) + (c >> 1)) = make_uint2(lo, hi);
                *sp = (uint8_t)sb;
            }
        }
        it = nx;
        ca = na;
        cb = nb;
    }
}

// max |x| over a [rows x cols] BF16 tensor into *amax (zeroed before the launch).
// Non-negative floats order like their bit patterns, so an unsigned atomicMax of
// the bits is a float max.
__global__ void __launch_bounds__(256) k_absmax_bf16(const pact_bf16 *__restrict__ x, int64_t ldx, int64_t rows,
                                                     int64_t cols, unsigned *__restrict__ amax) {
    pdl_wait();
    const int64_t per_row = cols / 8;
    const int64_t n8 = rows * per_row;
    float m = 0.0f;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / per_row, c = (i % per_row) * 8;
        float v[8];
        unpack8_bf16(*reinterpret_cast<const uint4 *>(x + r * ldx + c), v);
#pragma unroll
        for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(v[j]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if ((threadIdx.x & 31) == 0) atomicMax(amax, __float_as_uint(m));
}

static int grid_for(int64_t warp_tasks, int threads, int per_sm = 8) {
    const int sms = sm_count();
    const int64_t per_block = threads / 32;
    int64_t blocks = (warp_tasks + per_block - 1) / per_block;
    const int64_t cap = (int64_t)sms * per_sm;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    return (int)blocks;
}

// Blocks of `kernel` (256 threads, no dynamic shared memory) resident on one SM: the
// grid-stride kernels launch one wave of them, so no block waits behind another.
template <typename K>
static int resident_per_sm(K kernel) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, 256, 0) != cudaSuccess || n < 1) n = 1;
    return n;
}

// ------------------------------------------------------- A3: RMSNorm + quantize
// A CTA of 4 warps works through rows blockIdx.x, blockIdx.x + gridDim.x, ... (and
// the padding rows of the scale layout).  Whole rows stream into a ring of shared-
// memory slots by bulk copies issued `stages` rows ahead, so the next rows are in
// flight while the current one is reduced and written: the row's sum of squares
// (warp w takes 256-column chunks w, w + 4, ...; FP64 partial sums, reduced across the
// CTA), then y = BF16(x * rstd * gamma) and its NVFP4 copy, read again from shared
// memory.
// |x| for the BF16 value whose exponent and mantissa bits sit at bits 20..27 and
// 13..19 of `field` (FP64's exponent and top mantissa positions): the exponent is
// rebiased from 127 to 1023, so a normal value comes out exact without a conversion
// instruction.  Zeros and subnormals come out below 2^-126: their squares (under
// 2^-252, at most 2^-238 for a whole row) are below half an ulp of any sum from
// 2^-180 on, so the callers recompute a sum below that (and one that met exponent
// 255, infinities and NaN) from plain conversions.
__device__ __forceinline__ double f64_of_bf16(uint32_t field) {
    return __hiloint2double((int)(field + 0x38000000u), 0);
}

constexpr int RING_THREADS = 128;
constexpr int RING_WARPS = RING_THREADS / 32;
constexpr int RMS_MAX_H = 16384;

// BF16 rounding of y = (x * rstd) * gamma with one correct rounding of the double
// expression: the FP32 evaluation decides unless it lies within 64 FP32 ulps of a
// BF16 midpoint (its error is below 4 ulps), in which case the double expression
// is rounded directly (Ziv, "Fast evaluation of elementary mathematical functions
// with correctly rounded last bit", ACM TOMS 17(3), 1991).
// Returns the value whose round-to-nearest BF16 conversion is the result: the FP32
// product where it decides, else the correctly rounded value itself.
__device__ __forceinline__ float rms_out(float x, float g, float r32, double rstd) {
    const float y = __fmul_rn(__fmul_rn(x, r32), g);
    const uint32_t lo = __float_as_uint(y) & 0xFFFFu;
    if (lo - 0x7FC0u <= 0x80u) {
        const double yd = ((double)x * rstd) * (double)g;
        return __bfloat162float(__double2bfloat16(yd));
    }
    return y;
}
// The same value from the double expression alone: for a row whose rstd lies beyond
// FP32's range, which needs eps = 0 and a row of zeros and subnormals only.
__device__ __forceinline__ float rms_exact(float x, float g, double rstd) {
    return __bfloat162float(__double2bfloat16(((double)x * rstd) * (double)g));
}

// Ring geometry: slots of `slot_bytes`, as many (2 .. 4) as fit in ~48 KiB, then the
// slot barriers and `extra` bytes (a shared copy of gamma); as many CTAs per SM (up to
// 8) as fit in 200 KiB.
struct Ring {
    int stages;
    size_t slot_bytes, smem;
    int grid;
};
static Ring ring_for(int64_t rows, size_t slot_bytes, size_t extra) {
    Ring r;
    r.slot_bytes = (slot_bytes + 127) & ~(size_t)127;
    r.stages = (int)(49152 / r.slot_bytes);
    r.stages = r.stages < 2 ? 2 : (r.stages > 4 ? 4 : r.stages);
    r.smem = r.stages * r.slot_bytes + 64 + extra;   // + the barriers, + a copy of gamma
    int per_sm = (int)(200 * 1024 / r.smem);
    per_sm = per_sm < 1 ? 1 : (per_sm > 8 ? 8 : per_sm);
    const int64_t g = (int64_t)sm_count() * per_sm;
    r.grid = (int)(rows < g ? rows : g);
    return r;
}

// EPS0: the instance for eps = 0, where a row of zeros and subnormals can have an rstd
// beyond FP32's range (rounded by rms_exact throughout) and a sum of squares small
// enough for the widened zeros and subnormals of f64_of_bf16 to count (summed again
// from plain conversions).  With eps > 0 neither can change a result: rstd is at most
// 2^74.5, and eps hides the widened values' 2^-238 at most.
template <bool EPS0>
__global__ void __launch_bounds__(RING_THREADS) k_rmsnorm_quant(const pact_bf16 *__restrict__ x, int64_t ldx,
                                                               const pact_bf16 *__restrict__ gamma, float eps,
                                                               int64_t M, int64_t H, pact_nvfp4_t yq,
                                                               pact_bf16 *__restrict__ y, float *__restrict__ rstd_out,
                                                               int stages, int slot_bytes) {
    extern __shared__ __align__(128) uint8_t ring[];
    uint64_t *full = reinterpret_cast<uint64_t *>(ring + stages * slot_bytes);
    pact_bf16 *gs = reinterpret_cast<pact_bf16 *>(ring + stages * slot_bytes + 64);   // gamma [H]
    __shared__ double red[RING_WARPS];
    __shared__ double rstd_s;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t rows_pad = (M + 127) & ~int64_t(127);
    const int nchunk = (int)((H + CHUNK - 1) / CHUNK);
    const uint32_t row_bytes = (uint32_t)(H * 2);
    if (threadIdx.x == 0) {
        for (int i = 0; i < stages; ++i) mbar_init(&full[i], 1);
        fence_barrier_init();
    }
    pdl_wait();
    for (int c = 8 * threadIdx.x; c < H; c += 8 * RING_THREADS)
        *reinterpret_cast<uint4 *>(gs + c) = *reinterpret_cast<const uint4 *>(gamma + c);
    __syncthreads();
    auto issue = [&](int i) {   // thread 0: row i of this CTA into its slot
        const int64_t r = blockIdx.x + (int64_t)i * gridDim.x;
        if (r < M) {
            mbar_arrive_expect_tx(&full[i % stages], row_bytes);
            bulk_load(ring + (i % stages) * slot_bytes, x + r * ldx, row_bytes, &full[i % stages]);
        }
    };
    if (threadIdx.x == 0)
        for (int i = 0; i < stages; ++i) issue(i);
    bool ok = true;
    int i = 0;
    for (int64_t row = blockIdx.x; row < rows_pad; row += gridDim.x, ++i) {
        const int slot = i % stages;
        if (row >= M) {   // a padding row of the scale layout: zero scales (block-uniform)
            for (int k = warp; k < nchunk; k += RING_WARPS) zero_pad_scales(yq, row, (int64_t)k * CHUNK);
            continue;
        }
        ok = __syncthreads_and(ok && mbar_wait(&full[slot], (uint32_t)(i / stages) & 1u));
        if (!ok) break;
        const uint8_t *rs = ring + slot * slot_bytes;
        // sum of squares in FP64 from values widened by integer operations (f64_of_bf16)
        double s0 = 0.0, s1 = 0.0, s2 = 0.0, s3 = 0.0;
        uint32_t top = 0;   // the largest exponent|mantissa pattern of either half
        for (int k = warp; k < nchunk; k += RING_WARPS) {
            const int c = k * CHUNK + 8 * lane;
            if (c < H) {
                const uint4 u = *reinterpret_cast<const uint4 *>(rs + 2 * c);
                const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t lo = (w[j] << 13) & 0x0FFFE000u, hi = (w[j] >> 3) & 0x0FFFE000u;
                    top = max(top, max(lo, hi));
                    const double a = f64_of_bf16(lo), b = f64_of_bf16(hi);
                    if (j & 1) {
                        s2 = fma(a, a, s2);
                        s3 = fma(b, b, s3);
                    } else {
                        s0 = fma(a, a, s0);
                        s1 = fma(b, b, s1);
                    }
                }
            }
        }
        bool plain = __any_sync(0xFFFFFFFFu, top >= (0xFFu << 20));   // an infinity or NaN
        if constexpr (EPS0) {   // or a warp sum below 2^-180
            double t = (s0 + s1) + (s2 + s3);
#pragma unroll
            for (int o = 16; o; o >>= 1) t += __shfl_xor_sync(0xFFFFFFFFu, t, o);
            plain |= !(t >= 0x1p-180);
        }
        if (plain) {
            // the sum as plain conversions give it
            s0 = s1 = s2 = s3 = 0.0;
            for (int k = warp; k < nchunk; k += RING_WARPS) {
                const int c = k * CHUNK + 8 * lane;
                if (c < H) {
                    float v[8];
                    load8_bf16(reinterpret_cast<const pact_bf16 *>(rs) + c, v);
#pragma unroll
                    for (int j = 0; j < 8; ++j) s0 = fma((double)v[j], (double)v[j], s0);
                }
            }
        }
        double ss = (s0 + s1) + (s2 + s3);
#pragma unroll
        for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
        if (lane == 0) red[warp] = ss;
        __syncthreads();
        if (threadIdx.x == 0) {   // one thread evaluates rstd; the others read it
            const double q = ((red[0] + red[1]) + (red[2] + red[3])) / (double)H + (double)eps;
            rstd_s = 1.0 / sqrt(q);
            if (rstd_out) rstd_out[row] = (float)rstd_s;
        }
        __syncthreads();
        const double rstd = rstd_s;
        const float r32 = (float)rstd;
        const bool wide = EPS0 && isinf(r32);
        const uint64_t r2 = f2_pack(r32, r32);
        for (int k = warp; k < nchunk; k += RING_WARPS) {
            const int64_t c0 = (int64_t)k * CHUNK;
            const int64_t c = c0 + 8 * lane;
            const bool valid = c < H;
            float v[8] = {0, 0, 0, 0, 0, 0, 0, 0}, g[8] = {0, 0, 0, 0, 0, 0, 0, 0}, o[8];
            if (valid) {
                load8_bf16(reinterpret_cast<const pact_bf16 *>(rs) + c, v);
                load8_bf16(gs + c, g);
            }
            if constexpr (EPS0) {
                if (wide) {
#pragma unroll
                    for (int j = 0; j < 8; ++j) o[j] = rms_exact(v[j], g[j], rstd);
                } else {
#pragma unroll
                    for (int j = 0; j < 8; ++j) o[j] = rms_out(v[j], g[j], r32, rstd);   // zeros past the row end
                }
            } else {
                // the FP32 products two at a time (the roundings of rms_out), the midpoint
                // test once for the 8 values, the FP64 expression behind one branch
                bool near = false;
#pragma unroll
                for (int j = 0; j < 8; j += 2) {
                    f2_unpack(f2_mul(f2_mul(f2_pack(v[j], v[j + 1]), r2), f2_pack(g[j], g[j + 1])), o[j], o[j + 1]);
                    near |= ((__float_as_uint(o[j]) & 0xFFFFu) - 0x7FC0u <= 0x80u) |
                            ((__float_as_uint(o[j + 1]) & 0xFFFFu) - 0x7FC0u <= 0x80u);
                }
                if (near) {
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        if ((__float_as_uint(o[j]) & 0xFFFFu) - 0x7FC0u <= 0x80u) o[j] = rms_exact(v[j], g[j], rstd);
                }
            }
            uint4 ow;
            round8_bf16(o, ow, o);
            if (valid && y) *reinterpret_cast<uint4 *>(y + row * H + c) = ow;
            uint32_t sb;
            const uint32_t codes = quant8(o, &sb);
            store_chunk(yq, row, c0, codes, sb, valid);
        }
        __syncthreads();                      // every thread is done with the slot and with red
        if (threadIdx.x == 0) issue(i + stages);
    }
    // copies still in flight land before the CTA leaves (bounded waits)
    if (threadIdx.x == 0) {
        for (int j = i; j < i + stages; ++j) {
            const int64_t r = blockIdx.x + (int64_t)j * gridDim.x;
            if (r < M) mbar_wait(&full[j % stages], (uint32_t)(j / stages) & 1u);
        }
    }
}

// Register-resident RMSNorm backward (below): a warp per row, 128-thread CTAs.
constexpr int ROWS_THREADS = 128;
constexpr int ROWS_WARPS = ROWS_THREADS / 32;

// Stage gamma [H] (NB 512-column chunks, zero past H) in shared memory, per 512-column
// chunk the first halves of its 32 blocks and then the second halves: a lane's two
// 16-byte reads of its block then hit distinct banks across the warp.
template <int NB>
__device__ __forceinline__ void stage_gamma(uint4 *gs, const pact_bf16 *__restrict__ gamma, int64_t H) {
    for (int i = threadIdx.x; i < NB * 64; i += blockDim.x) {
        const int c = 512 * (i >> 6) + 16 * (i & 31) + 8 * ((i >> 5) & 1);
        gs[i] = c < H ? *reinterpret_cast<const uint4 *>(gamma + c) : make_uint4(0u, 0u, 0u, 0u);
    }
}

// --------------------------------------------------- A4: SiLU-multiply + quantize


// The task loops below are software-pipelined: a warp loads the next task's inputs
// before it computes the current one, so two tasks' loads are in flight per warp.
// A task is 512 columns of a row; lane j owns the 16-value block j of every tensor
// (one scale computation per block, no block-maximum shuffle).  GU: the instance that
// also quantizes g and u (the layer's gate|up GEMM writes those copies itself, so its
// instance carries neither, and fits three CTAs per SM).
template <bool GU>
__global__ void __launch_bounds__(256, GU ? 2 : 3) k_silu_mul_quant(const pact_bf16 *__restrict__ g, const pact_bf16 *__restrict__ u,
                                                        int64_t ld_gu, int64_t M, int64_t I,
                                                        pact_bf16 *__restrict__ m, pact_nvfp4_t mq, pact_nvfp4_t gq,
                                                        pact_nvfp4_t uq, int has_gq, int has_uq) {
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int64_t nchunk = (I + QCHUNK - 1) / QCHUNK;
    const int64_t rows_pad = (M + 127) & ~int64_t(127);
    const int64_t warp0 = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    struct In {
        uint4 g0, g1, u0, u1;
    };
    auto load = [&](const TaskIter &t, In &v) {
        const int64_t c = t.chunk * QCHUNK + 16 * lane;
        v.g0 = v.g1 = v.u0 = v.u1 = make_uint4(0, 0, 0, 0);
        if (t.row < M && c < I) {
            const uint4 *gp = reinterpret_cast<const uint4 *>(g + t.row * ld_gu + c);
            const uint4 *up = reinterpret_cast<const uint4 *>(u + t.row * ld_gu + c);
            v.g0 = gp[0]; v.g1 = gp[1]; v.u0 = up[0]; v.u1 = up[1];
        }
    };
    // m for 8 values (one 16-byte piece of g and of u) as BF16 words
    auto silu8 = [&](const uint4 &gw, const uint4 &uw) {
        float gv[8], uv[8], sv[8], mv[8];
        unpack8_bf16(gw, gv);
        unpack8_bf16(uw, uv);
#pragma unroll
        for (int i = 0; i < 8; ++i) sv[i] = sigmoid_fast(gv[i]);
        silu_mul8<false>(gv, uv, sv, mv);
        uint4 mw;
        mw.x = pack_bf16x2(mv[0], mv[1]); mw.y = pack_bf16x2(mv[2], mv[3]);
        mw.z = pack_bf16x2(mv[4], mv[5]); mw.w = pack_bf16x2(mv[6], mv[7]);
        return mw;
    };
    TaskIter it(warp0, nchunk, nwarps);
    In cur;
    if (it.row < rows_pad) load(it, cur);
    while (it.row < rows_pad) {
        TaskIter nx = it;
        nx.next();
        In nxt;
        if (nx.row < rows_pad) load(nx, nxt);
        else nxt.g0 = nxt.g1 = nxt.u0 = nxt.u1 = make_uint4(0, 0, 0, 0);
        const int64_t row = it.row;
        const int64_t c = it.chunk * QCHUNK + 16 * lane;
        if (c < I) {
            // mq, gq and uq share their shape: one code offset, one scale offset
            const int64_t so = scale_offset(row, c >> 4, I), co = row * (I >> 1) + (c >> 1);
            if (row >= M) {   // a padding row of the scale layout
                static_cast<uint8_t *>(mq.scales)[so] = 0;
                if (GU && has_gq) static_cast<uint8_t *>(gq.scales)[so] = 0;
                if (GU && has_uq) static_cast<uint8_t *>(uq.scales)[so] = 0;
            } else {
                const uint4 m0 = silu8(cur.g0, cur.u0), m1 = silu8(cur.g1, cur.u1);
                if (m) {
                    uint4 *mp = reinterpret_cast<uint4 *>(m + row * I + c);
                    mp[0] = m0;
                    mp[1] = m1;
                }
                uint32_t lo, hi, sb;
                quant16_bf16(m0, m1, &lo, &hi, &sb);
                *reinterpret_cast<uint2 *>(static_cast<uint8_t *>(mq.codes) + co) = make_uint2(lo, hi);
                static_cast<uint8_t *>(mq.scales)[so] = (uint8_t)sb;
                if (GU && has_gq) {
                    quant16_bf16(cur.g0, cur.g1, &lo, &hi, &sb);
                    *reinterpret_cast<uint2 *>(static_cast<uint8_t *>(gq.codes) + co) = make_uint2(lo, hi);
                    static_cast<uint8_t *>(gq.scales)[so] = (uint8_t)sb;
                }
                if (GU && has_uq) {
                    quant16_bf16(cur.u0, cur.u1, &lo, &hi, &sb);
                    *reinterpret_cast<uint2 *>(static_cast<uint8_t *>(uq.codes) + co) = make_uint2(lo, hi);
                    static_cast<uint8_t *>(uq.scales)[so] = (uint8_t)sb;
                }
            }
        }
        it = nx;
        cur = nxt;
    }
}

// ---------------------------------------------- A9: SiLU-multiply backward + quantize
// A task is 512 columns of a row; lane j owns the 16-value block j: one scale byte of
// g^ and of u^ to read, one block each of dg and du to quantize.
__global__ void __launch_bounds__(256) k_silu_mul_bwd_quant(const pact_bf16 *__restrict__ dm, int64_t lddm,
                                                            pact_nvfp4_t gq, pact_nvfp4_t uq, int64_t M, int64_t I,
                                                            pact_bf16 *__restrict__ dgu, int64_t lddgu,
                                                            pact_nvfp4_t dguq, pact_bf16 *__restrict__ m_re) {
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int64_t nchunk = (I + QCHUNK - 1) / QCHUNK;
    const int64_t rows_pad = (M + 127) & ~int64_t(127);
    const int64_t warp0 = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    struct In {
        uint4 d0, d1;
        uint2 gc, uc;
        uint32_t gs, us;
    };
    auto load = [&](const TaskIter &t, In &v) {
        const int64_t c = t.chunk * QCHUNK + 16 * lane;
        v.d0 = v.d1 = make_uint4(0, 0, 0, 0);
        v.gc = v.uc = make_uint2(0, 0);
        v.gs = v.us = 0;
        if (t.row < M && c < I) {
            const uint4 *dp = reinterpret_cast<const uint4 *>(dm + t.row * lddm + c);
            v.d0 = dp[0];
            v.d1 = dp[1];
            // gq and uq share their shape: one code offset, one scale offset
            const int64_t co = t.row * (I >> 1) + (c >> 1), so = scale_offset(t.row, c >> 4, I);
            v.gc = *reinterpret_cast<const uint2 *>(static_cast<const uint8_t *>(gq.codes) + co);
            v.uc = *reinterpret_cast<const uint2 *>(static_cast<const uint8_t *>(uq.codes) + co);
            v.gs = static_cast<const uint8_t *>(gq.scales)[so];
            v.us = static_cast<const uint8_t *>(uq.scales)[so];
        }
    };
    // dg = dm u sigma(g) (1 + g (1 - sigma(g))), du = dm g sigma(g), two values per packed
    // FP32 operation, and m~ = BF16_RNE(silu(g^) u^) exactly, for 8 values: rounded to
    // BF16 words (wg, wu, wm)
    const uint64_t one2 = f2_pack(1.0f, 1.0f), neg2 = f2_pack(-1.0f, -1.0f);
    auto half8 = [&](const uint4 &dw, uint32_t gc, uint32_t gsb, uint32_t uc, uint32_t usb, uint4 &wg, uint4 &wu,
                     uint4 &wm) {
        float d[8], gh[8], uh[8], dg[8], du[8], mr[8];
        unpack8_bf16(dw, d);
        dequant8(gc, gsb, gh);
        dequant8(uc, usb, uh);
        float sg[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) sg[i] = sigmoid_fast(gh[i]);
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
            const uint64_t g2 = f2_pack(gh[i], gh[i + 1]), sg2 = f2_pack(sg[i], sg[i + 1]);
            const uint64_t ds = f2_mul(f2_pack(d[i], d[i + 1]), sg2);
            const uint64_t w = f2_fma(g2, f2_fma(sg2, neg2, one2), one2);
            f2_unpack(f2_mul(f2_mul(ds, f2_pack(uh[i], uh[i + 1])), w), dg[i], dg[i + 1]);
            f2_unpack(f2_mul(ds, g2), du[i], du[i + 1]);
        }
        silu_mul8<true>(gh, uh, sg, mr);
        wg.x = pack_bf16x2(dg[0], dg[1]); wg.y = pack_bf16x2(dg[2], dg[3]);
        wg.z = pack_bf16x2(dg[4], dg[5]); wg.w = pack_bf16x2(dg[6], dg[7]);
        wu.x = pack_bf16x2(du[0], du[1]); wu.y = pack_bf16x2(du[2], du[3]);
        wu.z = pack_bf16x2(du[4], du[5]); wu.w = pack_bf16x2(du[6], du[7]);
        wm.x = pack_bf16x2(mr[0], mr[1]); wm.y = pack_bf16x2(mr[2], mr[3]);
        wm.z = pack_bf16x2(mr[4], mr[5]); wm.w = pack_bf16x2(mr[6], mr[7]);
    };
    TaskIter it(warp0, nchunk, nwarps);
    In cur;
    if (it.row < rows_pad) load(it, cur);
    while (it.row < rows_pad) {
        TaskIter nx = it;
        nx.next();
        In nxt;
        if (nx.row < rows_pad) {
            load(nx, nxt);
        } else {
            nxt.d0 = nxt.d1 = make_uint4(0, 0, 0, 0);
            nxt.gc = nxt.uc = make_uint2(0, 0);
            nxt.gs = nxt.us = 0;
        }
        const int64_t row = it.row;
        const int64_t c = it.chunk * QCHUNK + 16 * lane;
        if (c < I) {
            // dg's block is block c / 16 of the [M x 2I] copy; du's lies I columns right
            uint8_t *codes = static_cast<uint8_t *>(dguq.codes) + row * I + (c >> 1);
            uint8_t *sg = static_cast<uint8_t *>(dguq.scales) + scale_offset(row, c >> 4, 2 * I);
            uint8_t *su = static_cast<uint8_t *>(dguq.scales) + scale_offset(row, (I + c) >> 4, 2 * I);
            if (row >= M) {   // a padding row of the scale layout
                *sg = 0;
                *su = 0;
            } else {
                uint4 wg0, wu0, wm0, wg1, wu1, wm1;
                half8(cur.d0, cur.gc.x, cur.gs, cur.uc.x, cur.us, wg0, wu0, wm0);
                half8(cur.d1, cur.gc.y, cur.gs, cur.uc.y, cur.us, wg1, wu1, wm1);
                uint4 *gp = reinterpret_cast<uint4 *>(dgu + row * lddgu + c);
                uint4 *upp = reinterpret_cast<uint4 *>(dgu + row * lddgu + I + c);
                gp[0] = wg0; gp[1] = wg1;
                upp[0] = wu0; upp[1] = wu1;
                if (m_re) {
                    uint4 *mp = reinterpret_cast<uint4 *>(m_re + row * I + c);
                    mp[0] = wm0; mp[1] = wm1;
                }
                uint32_t lo, hi, sb;
                quant16_bf16(wg0, wg1, &lo, &hi, &sb);
                *reinterpret_cast<uint2 *>(codes) = make_uint2(lo, hi);
                *sg = (uint8_t)sb;
                quant16_bf16(wu0, wu1, &lo, &hi, &sb);
                *reinterpret_cast<uint2 *>(codes + (I >> 1)) = make_uint2(lo, hi);
                *su = (uint8_t)sb;
            }
        }
        it = nx;
        cur = nxt;
    }
}

// ------------------------------------------------------- A10: RMSNorm backward
// The ring of the forward kernel, with a slot holding a row of dy, the row's NVFP4
// codes of y^ and (when given) a row of the residual gradient dres.  Pass 1 forms
// sum(dy * y^) (the row's scale bytes come from global memory, L1-resident after the
// first pass); pass 2 writes dx and, when asked, its NVFP4 copy.
struct BwdSlot {
    int codes_off, dres_off;
};
__host__ __device__ inline BwdSlot bwd_slot(int64_t H) {
    const int dy_bytes = (int)(H * 2), code_bytes = (int)(H / 2);
    BwdSlot b;
    b.codes_off = (dy_bytes + 127) & ~127;
    b.dres_off = (b.codes_off + code_bytes + 127) & ~127;
    return b;
}

__global__ void __launch_bounds__(RING_THREADS) k_rmsnorm_bwd(const pact_bf16 *__restrict__ dy, int64_t lddy,
                                                             pact_nvfp4_t yq, const float *__restrict__ rstd,
                                                             const pact_bf16 *__restrict__ gamma, int64_t M, int64_t H,
                                                             const pact_bf16 *__restrict__ dres,
                                                             pact_bf16 *__restrict__ dx, pact_nvfp4_t dxq, int has_dxq,
                                                             int stages, int slot_bytes) {
    extern __shared__ __align__(128) uint8_t ring[];
    uint64_t *full = reinterpret_cast<uint64_t *>(ring + stages * slot_bytes);
    pact_bf16 *gs = reinterpret_cast<pact_bf16 *>(ring + stages * slot_bytes + 64);   // gamma [H]
    __shared__ float red[RING_WARPS];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t rows = has_dxq ? (M + 127) & ~int64_t(127) : M;
    const int nchunk = (int)((H + CHUNK - 1) / CHUNK);
    const BwdSlot sl = bwd_slot(H);
    const uint32_t dy_bytes = (uint32_t)(H * 2), code_bytes = (uint32_t)(H / 2);
    if (threadIdx.x == 0) {
        for (int i = 0; i < stages; ++i) mbar_init(&full[i], 1);
        fence_barrier_init();
    }
    pdl_wait();
    for (int c = 8 * threadIdx.x; c < H; c += 8 * RING_THREADS)
        *reinterpret_cast<uint4 *>(gs + c) = *reinterpret_cast<const uint4 *>(gamma + c);
    __syncthreads();
    auto issue = [&](int i) {   // thread 0: row i of this CTA into its slot
        const int64_t r = blockIdx.x + (int64_t)i * gridDim.x;
        if (r < M) {
            uint8_t *slot = ring + (i % stages) * slot_bytes;
            uint64_t *bar = &full[i % stages];
            mbar_arrive_expect_tx(bar, dy_bytes + code_bytes + (dres ? dy_bytes : 0u));
            bulk_load(slot, dy + r * lddy, dy_bytes, bar);
            bulk_load(slot + sl.codes_off, static_cast<const uint8_t *>(yq.codes) + r * (H / 2), code_bytes, bar);
            if (dres) bulk_load(slot + sl.dres_off, dres + r * H, dy_bytes, bar);
        }
    };
    if (threadIdx.x == 0)
        for (int i = 0; i < stages; ++i) issue(i);
    bool ok = true;
    int i = 0;
    for (int64_t row = blockIdx.x; row < rows; row += gridDim.x, ++i) {
        const int slot = i % stages;
        if (row >= M) {   // padding row of dxq's scale layout (block-uniform)
            for (int k = warp; k < nchunk; k += RING_WARPS) zero_pad_scales(dxq, row, (int64_t)k * CHUNK);
            continue;
        }
        // the row's scale bytes of y^ (scattered over the tiled layout) and its rstd come
        // from global memory: loaded before the wait, so their latency overlaps it
        const uint8_t *ysc = static_cast<const uint8_t *>(yq.scales);
        uint32_t sc[4];
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            const int c = (warp + kk * RING_WARPS) * CHUNK + 8 * lane;
            sc[kk] = c < H ? ysc[scale_offset(row, c >> 4, H)] : 0u;
        }
        const float r = rstd[row];
        ok = __syncthreads_and(ok && mbar_wait(&full[slot], (uint32_t)(i / stages) & 1u));
        if (!ok) break;
        const uint8_t *rs = ring + slot * slot_bytes;
        const pact_bf16 *dys = reinterpret_cast<const pact_bf16 *>(rs);
        const uint8_t *cs = rs + sl.codes_off;
        const pact_bf16 *rrs = reinterpret_cast<const pact_bf16 *>(rs + sl.dres_off);
        auto scale_of = [&](int k, int c) -> uint32_t {   // k = warp + kk * RING_WARPS; selects, not an index
            const int kk = (k - warp) / RING_WARPS;
            return kk == 0 ? sc[0] : kk == 1 ? sc[1] : kk == 2 ? sc[2] : kk == 3 ? sc[3]
                                                                        : ysc[scale_offset(row, c >> 4, H)];
        };
        float dot = 0.0f;
        for (int k = warp; k < nchunk; k += RING_WARPS) {
            const int c = k * CHUNK + 8 * lane;
            if (c < H) {
                float d[8], yv[8];
                load8_bf16(dys + c, d);
                dequant8(*reinterpret_cast<const uint32_t *>(cs + c / 2), scale_of(k, c), yv);
                // (gamma * dy) * (y^ / gamma) == dy * y^
#pragma unroll
                for (int j = 0; j < 8; ++j) dot = fmaf(d[j], yv[j], dot);
            }
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) dot += __shfl_xor_sync(0xFFFFFFFFu, dot, o);
        if (lane == 0) red[warp] = dot;
        __syncthreads();
        const float mean = ((red[0] + red[1]) + (red[2] + red[3])) / (float)H;
        for (int k = warp; k < nchunk; k += RING_WARPS) {
            const int64_t c0 = (int64_t)k * CHUNK;
            const int64_t c = c0 + 8 * lane;
            const bool valid = c < H;
            float d[8] = {0, 0, 0, 0, 0, 0, 0, 0}, yv[8] = {0, 0, 0, 0, 0, 0, 0, 0};
            float g[8] = {1, 1, 1, 1, 1, 1, 1, 1}, res[8] = {0, 0, 0, 0, 0, 0, 0, 0}, o[8];
            if (valid) {
                load8_bf16(dys + c, d);
                dequant8(*reinterpret_cast<const uint32_t *>(cs + c / 2), scale_of(k, (int)c), yv);
                load8_bf16(gs + c, g);
                if (dres) load8_bf16(rrs + c, res);
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) o[j] = r * (g[j] * d[j] - __fdividef(yv[j], g[j]) * mean) + res[j];
            uint4 ow;
            round8_bf16(o, ow, o);   // zeros past the row end
            if (valid) *reinterpret_cast<uint4 *>(dx + row * H + c) = ow;
            if (has_dxq) {
                uint32_t sb;
                const uint32_t codes = quant8(o, &sb);
                store_chunk(dxq, row, c0, codes, sb, valid);
            }
        }
        __syncthreads();
        if (threadIdx.x == 0) issue(i + stages);
    }
    if (threadIdx.x == 0) {
        for (int j = i; j < i + stages; ++j) {
            const int64_t r = blockIdx.x + (int64_t)j * gridDim.x;
            if (r < M) mbar_wait(&full[j % stages], (uint32_t)(j / stages) & 1u);
        }
    }
}

// ---------------------------------------- A10: RMSNorm backward, rows of up to 4096 columns
// The layout of k_rmsnorm_quant_rows: a warp per row, lane l owning the blocks at
// columns 512 j + 16 l.  When a warp starts a row it has the L2 prefetch the next
// row's dy, codes and dres (one bulk prefetch each).  Pass 1 loads the row's dy and the
// codes and scale bytes of y^ into registers and forms sum(dy * y^) as, per block, the
// scale times the sum of dy times the E2M1 values; pass 2, a loop over the lane's
// blocks, reads each block again (from L1) with its dres and writes
//   dx = rstd (gamma dy - (y^ / gamma) mean) + dres
// with 1/gamma from a table staged in shared memory (correctly rounded FP32), and,
// when asked, the NVFP4 copy of dx.
constexpr int ROWS_MAX_NB_BWD = 8;

// The 16 values of one E2M1 block (8 code bytes, element 0 in the low nibble of the
// first byte) as 8 packed FP32 pairs, exactly.
__device__ __forceinline__ void e2m1_block_f32(uint32_t lo, uint32_t hi, uint64_t (&p)[8]) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const uint32_t h = e2m1x2_to_f16x2(((k < 4 ? lo : hi) >> (8 * (k & 3))) & 0xFFu);
        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&h));
        p[k] = f2_pack(f.x, f.y);
    }
}

template <int NB>
__global__ void __launch_bounds__(ROWS_THREADS) k_rmsnorm_bwd_rows(const pact_bf16 *__restrict__ dy, int64_t lddy,
                                                                  pact_nvfp4_t yq, const float *__restrict__ rstd,
                                                                  const pact_bf16 *__restrict__ gamma, int64_t M,
                                                                  int64_t H, const pact_bf16 *__restrict__ dres,
                                                                  pact_bf16 *__restrict__ dx, pact_nvfp4_t dxq,
                                                                  int has_dxq) {
    __shared__ uint4 gs[NB * 64];          // gamma, in the order of stage_gamma
    __shared__ float4 igs[NB * 128];       // 1 / gamma: per chunk, quarter k of lane l's block at 32 k + l
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t rows = has_dxq ? (M + 127) & ~int64_t(127) : M;
    const int64_t nw = (int64_t)gridDim.x * ROWS_WARPS;
    const uint8_t *ycodes = static_cast<const uint8_t *>(yq.codes), *yscales = static_cast<const uint8_t *>(yq.scales);
    uint8_t *codes = static_cast<uint8_t *>(dxq.codes), *scales = static_cast<uint8_t *>(dxq.scales);
    pdl_wait();
    stage_gamma<NB>(gs, gamma, H);
    for (int i = threadIdx.x; i < NB * 128; i += blockDim.x) {
        // float4 i: chunk j = i / 128, quarter k = (i / 32) % 4 of the block of lane l = i % 32
        const int c = 512 * (i >> 7) + 16 * (i & 31) + 4 * ((i >> 5) & 3);
        float4 f = make_float4(1.0f, 1.0f, 1.0f, 1.0f);
        if (c < H) {
            const uint2 g = *reinterpret_cast<const uint2 *>(gamma + c);
            f = make_float4(1.0f / bf16lo(g.x), 1.0f / bf16hi(g.x), 1.0f / bf16lo(g.y), 1.0f / bf16hi(g.y));
        }
        igs[i] = f;
    }
    __syncthreads();
    for (int64_t row = (int64_t)warp * gridDim.x + blockIdx.x; row < rows; row += nw) {   // as the forward
        if (row >= M) {   // a padding row of dxq's scale layout: zero scales
#pragma unroll 1
            for (int c = 16 * lane; c < H; c += 512) scales[scale_offset(row, c >> 4, H)] = 0;
            continue;
        }
        if (lane == 0 && row + nw < M) {
            const int64_t n = row + nw;
            bulk_prefetch_l2(dy + n * lddy, (uint32_t)(H * 2));
            bulk_prefetch_l2(ycodes + n * (H >> 1), (uint32_t)(H >> 1));
            if (dres) bulk_prefetch_l2(dres + n * H, (uint32_t)(H * 2));
        }
        const pact_bf16 *dyr = dy + row * lddy;
        const uint8_t *ycr = ycodes + row * (H >> 1);
        // pass 1: sum(dy * y^); lanes whose block lies past the row end hold zeros
        uint4 d[2 * NB];
        uint2 q[NB];
        uint32_t sq[NB];
#pragma unroll
        for (int j = 0; j < NB; ++j) {
            const int c = 512 * j + 16 * lane;
            d[2 * j] = d[2 * j + 1] = make_uint4(0u, 0u, 0u, 0u);
            q[j] = make_uint2(0u, 0u);
            sq[j] = 0u;
            if (c < H) {
                const uint4 *p = reinterpret_cast<const uint4 *>(dyr + c);
                d[2 * j] = p[0];
                d[2 * j + 1] = p[1];
                q[j] = *reinterpret_cast<const uint2 *>(ycr + (c >> 1));
                sq[j] = yscales[scale_offset(row, c >> 4, H)];
            }
        }
        const float r = rstd[row];
        float dot = 0.0f;
#pragma unroll
        for (int j = 0; j < NB; ++j) {
            const uint32_t dw[8] = {d[2 * j].x, d[2 * j].y, d[2 * j].z, d[2 * j].w,
                                    d[2 * j + 1].x, d[2 * j + 1].y, d[2 * j + 1].z, d[2 * j + 1].w};
            uint64_t e[8];
            e2m1_block_f32(q[j].x, q[j].y, e);
            uint64_t acc = f2_pack(0.0f, 0.0f);
#pragma unroll
            for (int k = 0; k < 8; ++k) acc = f2_fma(f2_pack(bf16lo(dw[k]), bf16hi(dw[k])), e[k], acc);
            float a0, a1;
            f2_unpack(acc, a0, a1);
            dot = fmaf(e4m3_to_float(sq[j]), a0 + a1, dot);
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) dot += __shfl_xor_sync(0xFFFFFFFFu, dot, o);
        const float mean = dot / (float)H;
        const uint64_t r2 = f2_pack(r, r), nm2 = f2_pack(-mean, -mean);
        // pass 2
#pragma unroll 1
        for (int c = 16 * lane; c < H; c += 512) {
            const uint4 *p = reinterpret_cast<const uint4 *>(dyr + c);
            const uint4 da = p[0], db = p[1];
            uint4 ra = make_uint4(0u, 0u, 0u, 0u), rb = ra;
            if (dres) {
                const uint4 *pr = reinterpret_cast<const uint4 *>(dres + row * H + c);
                ra = pr[0];
                rb = pr[1];
            }
            const uint2 qc = *reinterpret_cast<const uint2 *>(ycr + (c >> 1));
            const float sc = e4m3_to_float(yscales[scale_offset(row, c >> 4, H)]);
            const uint32_t dw[8] = {da.x, da.y, da.z, da.w, db.x, db.y, db.z, db.w};
            const uint32_t rw[8] = {ra.x, ra.y, ra.z, ra.w, rb.x, rb.y, rb.z, rb.w};
            const int gi = (c >> 9) * 64 + lane;
            const uint4 ga = gs[gi], gb = gs[gi + 32];
            const uint32_t gw[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
            const float4 *ig = &igs[(c >> 9) * 128 + lane];
            const uint64_t sc2 = f2_pack(sc, sc);
            uint64_t e[8];
            e2m1_block_f32(qc.x, qc.y, e);
            uint32_t ow[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const float4 i4 = ig[32 * (k >> 1)];
                const uint64_t ig2 = (k & 1) ? f2_pack(i4.z, i4.w) : f2_pack(i4.x, i4.y);
                const uint64_t yh = f2_mul(e[k], sc2);                                   // y^ (exact)
                const uint64_t t = f2_mul(f2_pack(bf16lo(gw[k]), bf16hi(gw[k])),
                                          f2_pack(bf16lo(dw[k]), bf16hi(dw[k])));       // gamma dy
                const uint64_t u = f2_fma(f2_mul(yh, ig2), nm2, t);                       // - (y^ / gamma) mean
                float o0, o1;
                f2_unpack(f2_fma(r2, u, f2_pack(bf16lo(rw[k]), bf16hi(rw[k]))), o0, o1);
                ow[k] = pack_bf16x2(o0, o1);
            }
            const uint4 xa = make_uint4(ow[0], ow[1], ow[2], ow[3]), xb = make_uint4(ow[4], ow[5], ow[6], ow[7]);
            uint4 *xp = reinterpret_cast<uint4 *>(dx + row * H + c);
            xp[0] = xa;
            xp[1] = xb;
            if (has_dxq) {
                uint32_t lo, hi, sb;
                quant16_bf16(xa, xb, &lo, &hi, &sb);
                *reinterpret_cast<uint2 *>(codes + row * (H >> 1) + (c >> 1)) = make_uint2(lo, hi);
                scales[scale_offset(row, c >> 4, H)] = (uint8_t)sb;
            }
        }
    }
}

// ------------------------------------------------------- A1: backward weight layout
// Wb = q(deq(Wf)^T): a CTA turns a 64 (n) x 64 (k) tile of the forward layout into
// 64 rows (k) x 4 blocks (n) of the backward layout.  Runs once per frozen weight.
__global__ void __launch_bounds__(256) k_weight_bwd_layout(pact_nvfp4_t wf, pact_nvfp4_t wb) {
    pdl_wait();
    __shared__ float tile[64][65];
    const int64_t n0 = (int64_t)blockIdx.y * 64, k0 = (int64_t)blockIdx.x * 64;
    const int t = threadIdx.x;
    // dequantize: thread t -> row n0 + t/4, columns k0 + 16*(t%4) .. +16
    {
        const int rn = t >> 2, cb = (t & 3) * 16;
        const int64_t n = n0 + rn;
        if (n < wf.rows) {
            float a[8], b[8];
            load8_nvfp4(wf, n, k0 + cb, a);
            load8_nvfp4(wf, n, k0 + cb + 8, b);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                tile[rn][cb + i] = a[i];
                tile[rn][cb + 8 + i] = b[i];
            }
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) tile[rn][cb + i] = 0.0f;
        }
    }
    __syncthreads();
    // quantize along n: warp w handles rows k0 + 8w .. 8w+7; per row 64 columns = 8
    // lanes x 8 values, so one warp instruction covers 4 rows.
    const int lane = t & 31, warp = t >> 5;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int rk = warp * 8 + h * 4 + (lane >> 3);
        const int cn = (lane & 7) * 8;
        float v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = tile[cn + i][rk];
        uint32_t sb;
        const uint32_t codes = quant8(v, &sb);
        const uint32_t packed = gather_scales4(sb);
        const int64_t k = k0 + rk, n = n0 + cn;
        if (k < wb.rows && n < wb.cols) {
            *reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(wb.codes) + k * (wb.cols >> 1) + (n >> 1)) = codes;
            if ((lane & 7) == 0)
                *reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(wb.scales) + scale_offset(k, n >> 4, wb.cols)) =
                    packed;
        }
    }
}

// y = BF16_RNE(x), elementwise.
__global__ void __launch_bounds__(256) k_round_bf16(const float *__restrict__ x, pact_bf16 *__restrict__ y, int64_t n) {
    pdl_wait();
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        y[i] = __bfloat16_as_ushort(__float2bfloat16_rn(x[i]));
}

// Zero scale rows [rows, round_up(rows, 128)) of a tensor (the layout's padding).
__global__ void k_zero_scale_pad(pact_nvfp4_t t) {
    pdl_wait();
    const int64_t rows_pad = (t.rows + 127) & ~int64_t(127);
    const int64_t nblk = t.cols >> 4;
    const int64_t n = (rows_pad - t.rows) * nblk;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = t.rows + i / nblk, c = i % nblk;
        static_cast<uint8_t *>(t.scales)[scale_offset(r, c, t.cols)] = 0;
    }
}

// Register-resident RMSNorm backward: one instance per number of 512-column chunks.
using RmsRowsBwd = void (*)(const pact_bf16 *, int64_t, pact_nvfp4_t, const float *, const pact_bf16 *, int64_t,
                            int64_t, const pact_bf16 *, pact_bf16 *, pact_nvfp4_t, int);
static const RmsRowsBwd kRmsRowsBwd[ROWS_MAX_NB_BWD] = {
    k_rmsnorm_bwd_rows<1>, k_rmsnorm_bwd_rows<2>, k_rmsnorm_bwd_rows<3>, k_rmsnorm_bwd_rows<4>,
    k_rmsnorm_bwd_rows<5>, k_rmsnorm_bwd_rows<6>, k_rmsnorm_bwd_rows<7>, k_rmsnorm_bwd_rows<8>};

// Grid of a register-resident kernel: one resident wave of CTAs (they are issue-bound:
// every SM gets the same number of CTAs), or fewer when the rows do not need them all.
// `per_sm` caches the kernel's residency (0 until the first call).
template <typename K>
static int rows_grid(K kernel, int &per_sm, int64_t rows, size_t smem = 0) {
    if (per_sm == 0) {
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, ROWS_THREADS, smem) != cudaSuccess || n < 1)
            n = 1;
        per_sm = n;
    }
    const int64_t need = (rows + ROWS_WARPS - 1) / ROWS_WARPS, cap = (int64_t)sm_count() * per_sm;
    return (int)(need < cap ? need : cap);
}

}  // namespace pact

using namespace pact;

extern "C" {

size_t pact_nvfp4_code_bytes(int64_t rows, int64_t cols) { return (size_t)(rows * (cols / 2)); }

size_t pact_scale_bytes(int64_t rows, int64_t cols) {
    return (size_t)(((rows + 127) / 128 * 128) * ((cols / 16 + 3) / 4 * 4));
}

static size_t up256(size_t b) { return (b + 255) & ~(size_t)255; }

size_t pact_weight_cache_bytes(int64_t N, int64_t K) {
    return up256(pact_nvfp4_code_bytes(N, K)) + up256(pact_scale_bytes(N, K)) + up256(pact_nvfp4_code_bytes(K, N)) +
           up256(pact_scale_bytes(K, N));
}

pact_status pact_round_bf16(const float *x, pact_bf16 *y, int64_t n, pact_stream_t stream) {
    PACT_CHECK(x && y, PACT_ERR_INVALID_ARG, "pact_round_bf16: NULL argument");
    PACT_CHECK(n >= 1, PACT_ERR_SHAPE, "pact_round_bf16: n >= 1 required");
    PACT_CHECK(aligned16(x) && aligned16(y), PACT_ERR_ALIGN, "pact_round_bf16: pointers must be 16-byte aligned");
    return launch_dep(k_round_bf16, dim3(grid_for((n + 31) / 32, 256)), dim3(256), 0, (cudaStream_t)stream,
                      "pact_round_bf16", x, y, n);
}

pact_status pact_quantize_nvfp4(const pact_bf16 *x, int64_t ldx, int64_t rows, int64_t cols, const pact_nvfp4_t *out,
                                pact_stream_t stream) {
    PACT_CHECK(x && out, PACT_ERR_INVALID_ARG, "pact_quantize_nvfp4: NULL argument");
    PACT_CHECK(rows >= 1 && cols >= 64 && cols % 64 == 0, PACT_ERR_SHAPE,
               "pact_quantize_nvfp4: rows >= 1 and cols a positive multiple of 64 required (rows=%lld cols=%lld)",
               (long long)rows, (long long)cols);
    PACT_CHECK(ldx >= cols && ldx % 8 == 0 && aligned16(x), PACT_ERR_ALIGN,
               "pact_quantize_nvfp4: x must be 16-byte aligned with ldx >= cols, ldx %% 8 == 0");
    pact_status s = check_nvfp4(out, rows, cols, "out");
    if (s != PACT_OK) return s;
    const int64_t tasks = ((rows + 127) / 128 * 128) * ((cols + QCHUNK - 1) / QCHUNK);
    return launch_dep(k_quantize, dim3(grid_for(tasks, 256)), dim3(256), 0, (cudaStream_t)stream, "pact_quantize_nvfp4",
                      x, ldx, rows, *out, 1.0f);
}

pact_status pact_absmax_bf16(const pact_bf16 *x, int64_t ldx, int64_t rows, int64_t cols, float *amax,
                             pact_stream_t stream) {
    PACT_CHECK(x && amax, PACT_ERR_INVALID_ARG, "pact_absmax_bf16: NULL argument");
    PACT_CHECK(rows >= 1 && cols >= 8 && cols % 8 == 0, PACT_ERR_SHAPE,
               "pact_absmax_bf16: rows >= 1 and cols a positive multiple of 8 required (rows=%lld cols=%lld)",
               (long long)rows, (long long)cols);
    PACT_CHECK(ldx >= cols && ldx % 8 == 0 && aligned16(x) && ((uintptr_t)amax & 3) == 0, PACT_ERR_ALIGN,
               "pact_absmax_bf16: x 16-byte aligned with ldx >= cols, ldx %% 8 == 0; amax 4-byte aligned");
    const cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(float), (cudaStream_t)stream);
    PACT_CHECK(e == cudaSuccess, PACT_ERR_CUDA, "pact_absmax_bf16: %s", cudaGetErrorString(e));
    const int64_t threads = rows * (cols / 8);
    return launch_dep(k_absmax_bf16, dim3(grid_for((threads + 31) / 32, 256)), dim3(256), 0, (cudaStream_t)stream,
                      "pact_absmax_bf16", x, ldx, rows, cols, reinterpret_cast<unsigned *>(amax));
}

int pact_two_level_exponent(float amax) {
    // smallest e with amax <= 2688 * 2^e; 2688 * 2^e is exact in double for every e
    // reached here (|e| < 200), so each comparison is exact
    if (!(amax > 0.0f) || !std::isfinite(amax)) return 0;
    const double a = (double)amax;
    int e = std::ilogb(a) - std::ilogb(2688.0);
    while (a > std::ldexp(2688.0, e)) ++e;
    while (a <= std::ldexp(2688.0, e - 1)) --e;
    return e;
}

pact_status pact_rmsnorm_quant(const pact_bf16 *x, int64_t ldx, const pact_bf16 *gamma, float eps, int64_t M,
                               int64_t H, const pact_nvfp4_t *yq, pact_bf16 *y, float *rstd, pact_stream_t stream) {
    PACT_CHECK(x && gamma && yq, PACT_ERR_INVALID_ARG, "pact_rmsnorm_quant: NULL argument");
    PACT_CHECK(M >= 1 && H >= 64 && H % 64 == 0 && H <= RMS_MAX_H, PACT_ERR_SHAPE,
               "pact_rmsnorm_quant: M >= 1, H a multiple of 64 in [64, 16384] required (M=%lld H=%lld)",
               (long long)M, (long long)H);
    PACT_CHECK(!(eps < 0.0f) && isfinite(eps), PACT_ERR_INVALID_ARG, "pact_rmsnorm_quant: eps must be finite and >= 0");
    PACT_CHECK(ldx >= H && ldx % 8 == 0 && aligned16(x) && aligned16(gamma) && aligned16(y) && aligned16(rstd),
               PACT_ERR_ALIGN, "pact_rmsnorm_quant: pointers must be 16-byte aligned, ldx >= H, ldx %% 8 == 0");
    pact_status s = check_nvfp4(yq, M, H, "yq");
    if (s != PACT_OK) return s;
    const int64_t rows_pad = (M + 127) / 128 * 128;
    PACT_CHECK(rows_pad <= 0x7FFFFFFF, PACT_ERR_SHAPE, "pact_rmsnorm_quant: M too large");
    const Ring r = ring_for(rows_pad, (size_t)H * 2, (size_t)H * 2);
    static std::atomic<bool> attr_done[64];   // per device; setting the attribute twice is harmless
    const int d = current_device();
    if (d >= 0 && d < 64 && !attr_done[d].load(std::memory_order_acquire)) {
        cudaError_t e = cudaFuncSetAttribute(k_rmsnorm_quant<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(k_rmsnorm_quant<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
        if (e != cudaSuccess) return fail(PACT_ERR_CUDA, "pact_rmsnorm_quant: %s", cudaGetErrorString(e));
        attr_done[d].store(true, std::memory_order_release);
    }
    return launch_dep(eps == 0.0f ? k_rmsnorm_quant<true> : k_rmsnorm_quant<false>, dim3(r.grid), dim3(RING_THREADS),
                      r.smem, (cudaStream_t)stream,
                      "pact_rmsnorm_quant", x, ldx, gamma, eps, M, H, *yq, y, rstd, r.stages, (int)r.slot_bytes);
}

pact_status pact_silu_mul_quant(const pact_bf16 *g, const pact_bf16 *u, int64_t ld_gu, int64_t M, int64_t I,
                                pact_bf16 *m, const pact_nvfp4_t *mq, const pact_nvfp4_t *gq, const pact_nvfp4_t *uq,
                                pact_stream_t stream) {
    PACT_CHECK(g && u && mq, PACT_ERR_INVALID_ARG, "pact_silu_mul_quant: NULL argument");
    PACT_CHECK(M >= 1 && I >= 64 && I % 64 == 0, PACT_ERR_SHAPE,
               "pact_silu_mul_quant: M >= 1 and I a positive multiple of 64 required");
    PACT_CHECK(ld_gu >= I && ld_gu % 8 == 0 && aligned16(g) && aligned16(u) && aligned16(m), PACT_ERR_ALIGN,
               "pact_silu_mul_quant: pointers must be 16-byte aligned, ld_gu >= I, ld_gu %% 8 == 0");
    pact_status s = check_nvfp4(mq, M, I, "mq");
    if (s == PACT_OK && gq) s = check_nvfp4(gq, M, I, "gq");
    if (s == PACT_OK && uq) s = check_nvfp4(uq, M, I, "uq");
    if (s != PACT_OK) return s;
    pact_nvfp4_t none = {nullptr, nullptr, M, I};
    const int64_t tasks = ((M + 127) / 128 * 128) * ((I + QCHUNK - 1) / QCHUNK);
    if (gq || uq) {
        static const int per_sm = resident_per_sm(k_silu_mul_quant<true>);
        return launch_dep(k_silu_mul_quant<true>, dim3(grid_for(tasks, 256, per_sm)), dim3(256), 0,
                          (cudaStream_t)stream, "pact_silu_mul_quant", g, u, ld_gu, M, I, m, *mq, gq ? *gq : none,
                          uq ? *uq : none, (int)(gq != nullptr), (int)(uq != nullptr));
    }
    static const int per_sm = resident_per_sm(k_silu_mul_quant<false>);
    return launch_dep(k_silu_mul_quant<false>, dim3(grid_for(tasks, 256, per_sm)), dim3(256), 0, (cudaStream_t)stream,
                      "pact_silu_mul_quant", g, u, ld_gu, M, I, m, *mq, none, none, 0, 0);
}

pact_status pact_silu_mul_bwd_quant(const pact_bf16 *dm, int64_t lddm, const pact_nvfp4_t *gq, const pact_nvfp4_t *uq,
                                    int64_t M, int64_t I, pact_bf16 *dgu, int64_t lddgu, const pact_nvfp4_t *dguq,
                                    pact_bf16 *m_re, pact_stream_t stream) {
    PACT_CHECK(dm && gq && uq && dgu && dguq, PACT_ERR_INVALID_ARG, "pact_silu_mul_bwd_quant: NULL argument");
    PACT_CHECK(M >= 1 && I >= 64 && I % 64 == 0, PACT_ERR_SHAPE,
               "pact_silu_mul_bwd_quant: M >= 1 and I a positive multiple of 64 required");
    PACT_CHECK(lddm >= I && lddm % 8 == 0 && lddgu >= 2 * I && lddgu % 8 == 0 && aligned16(dm) && aligned16(dgu) &&
                   aligned16(m_re),
               PACT_ERR_ALIGN, "pact_silu_mul_bwd_quant: pointers must be 16-byte aligned, leading dims %% 8 == 0");
    pact_status s = check_nvfp4(gq, M, I, "gq");
    if (s == PACT_OK) s = check_nvfp4(uq, M, I, "uq");
    if (s == PACT_OK) s = check_nvfp4(dguq, M, 2 * I, "dguq");
    if (s != PACT_OK) return s;
    const int64_t tasks = ((M + 127) / 128 * 128) * ((I + QCHUNK - 1) / QCHUNK);
    static const int per_sm = resident_per_sm(k_silu_mul_bwd_quant);
    return launch_dep(k_silu_mul_bwd_quant, dim3(grid_for(tasks, 256, per_sm)), dim3(256), 0, (cudaStream_t)stream,
                      "pact_silu_mul_bwd_quant", dm, lddm, *gq, *uq, M, I, dgu, lddgu, *dguq, m_re);
}

pact_status pact_rmsnorm_bwd(const pact_bf16 *dy, int64_t lddy, const pact_nvfp4_t *yq, const float *rstd,
                             const pact_bf16 *gamma, int64_t M, int64_t H, const pact_bf16 *dres, pact_bf16 *dx,
                             const pact_nvfp4_t *dxq, pact_stream_t stream) {
    PACT_CHECK(dy && yq && rstd && gamma && dx, PACT_ERR_INVALID_ARG, "pact_rmsnorm_bwd: NULL argument");
    PACT_CHECK(M >= 1 && H >= 64 && H % 64 == 0 && H <= RMS_MAX_H, PACT_ERR_SHAPE,
               "pact_rmsnorm_bwd: M >= 1, H a multiple of 64 in [64, 16384] required");
    PACT_CHECK(lddy >= H && lddy % 8 == 0 && aligned16(dy) && aligned16(gamma) && aligned16(dx) && aligned16(dres),
               PACT_ERR_ALIGN, "pact_rmsnorm_bwd: pointers must be 16-byte aligned, lddy %% 8 == 0");
    pact_status s = check_nvfp4(yq, M, H, "yq");
    if (s == PACT_OK && dxq) s = check_nvfp4(dxq, M, H, "dxq");
    if (s != PACT_OK) return s;
    pact_nvfp4_t none = {nullptr, nullptr, M, H};
    const int64_t rows = dxq ? (M + 127) / 128 * 128 : M;
    PACT_CHECK(rows <= 0x7FFFFFFF, PACT_ERR_SHAPE, "pact_rmsnorm_bwd: M too large");
    if (H <= 512 * ROWS_MAX_NB_BWD) {
        static int per_sm[ROWS_MAX_NB_BWD] = {0};
        const int nb = (int)((H + 511) / 512);
        const int grid = rows_grid(kRmsRowsBwd[nb - 1], per_sm[nb - 1], rows);
        return launch_dep(kRmsRowsBwd[nb - 1], dim3(grid), dim3(ROWS_THREADS), 0, (cudaStream_t)stream,
                          "pact_rmsnorm_bwd", dy, lddy, *yq, rstd, gamma, M, H, dres, dx, dxq ? *dxq : none,
                          (int)(dxq != nullptr));
    }
    const BwdSlot sl = bwd_slot(H);
    const Ring r = ring_for(rows, (size_t)(dres ? sl.dres_off + H * 2 : sl.codes_off + H / 2), (size_t)H * 2);
    static std::atomic<bool> attr_done[64];   // per device; setting the attribute twice is harmless
    const int d = current_device();
    if (d >= 0 && d < 64 && !attr_done[d].load(std::memory_order_acquire)) {
        const cudaError_t e = cudaFuncSetAttribute(k_rmsnorm_bwd, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
        if (e != cudaSuccess) return fail(PACT_ERR_CUDA, "pact_rmsnorm_bwd: %s", cudaGetErrorString(e));
        attr_done[d].store(true, std::memory_order_release);
    }
    return launch_dep(k_rmsnorm_bwd, dim3(r.grid), dim3(RING_THREADS), r.smem, (cudaStream_t)stream, "pact_rmsnorm_bwd",
                      dy, lddy, *yq, rstd, gamma, M, H, dres, dx, dxq ? *dxq : none, (int)(dxq != nullptr), r.stages,
                      (int)r.slot_bytes);
}

pact_status pact_weight_layout_cache(const pact_bf16 *W, int64_t ldw, int64_t N, int64_t K, void *buf, size_t bytes,
                                     pact_weight_cache_t *out, pact_stream_t stream) {
    return pact_weight_layout_cache_scaled(W, ldw, N, K, 0, buf, bytes, out, stream);
}

pact_status pact_weight_layout_cache_scaled(const pact_bf16 *W, int64_t ldw, int64_t N, int64_t K, int gexp,
                                            void *buf, size_t bytes, pact_weight_cache_t *out,
                                            pact_stream_t stream) {
    PACT_CHECK(W && buf && out, PACT_ERR_INVALID_ARG, "pact_weight_layout_cache: NULL argument");
    PACT_CHECK(gexp >= -100 && gexp <= 100, PACT_ERR_INVALID_ARG,
               "pact_weight_layout_cache_scaled: |gexp| <= 100 required (gexp=%d)", gexp);
    PACT_CHECK(N >= 64 && K >= 64 && N % 64 == 0 && K % 64 == 0, PACT_ERR_SHAPE,
               "pact_weight_layout_cache: N and K must be positive multiples of 64 (N=%lld K=%lld)", (long long)N,
               (long long)K);
    PACT_CHECK(bytes >= pact_weight_cache_bytes(N, K), PACT_ERR_INVALID_ARG,
               "pact_weight_layout_cache: buffer too small (%zu < %zu)", bytes, pact_weight_cache_bytes(N, K));
    PACT_CHECK(((uintptr_t)buf & 255) == 0 && aligned16(W) && ldw >= K && ldw % 8 == 0, PACT_ERR_ALIGN,
               "pact_weight_layout_cache: buf must be 256-byte aligned, W 16-byte aligned with ldw %% 8 == 0");
    uint8_t *p = static_cast<uint8_t *>(buf);
    pact_weight_cache_t c;
    c.fwd.rows = N; c.fwd.cols = K;
    c.fwd.codes = p; p += up256(pact_nvfp4_code_bytes(N, K));
    c.fwd.scales = p; p += up256(pact_scale_bytes(N, K));
    c.bwd.rows = K; c.bwd.cols = N;
    c.bwd.codes = p; p += up256(pact_nvfp4_code_bytes(K, N));
    c.bwd.scales = p;
    c.gexp = gexp;
    const int64_t tasks = ((N + 127) / 128 * 128) * ((K + QCHUNK - 1) / QCHUNK);
    pact_status s = launch_dep(k_quantize, dim3(grid_for(tasks, 256)), dim3(256), 0, (cudaStream_t)stream,
                               "pact_weight_layout_cache", W, ldw, N, c.fwd, std::ldexp(1.0f, -gexp));
    if (s != PACT_OK) return s;
    dim3 grid((unsigned)(K / 64), (unsigned)(N / 64));
    s = launch_dep(k_weight_bwd_layout, grid, dim3(256), 0, (cudaStream_t)stream, "pact_weight_layout_cache", c.fwd,
                   c.bwd);
    if (s != PACT_OK) return s;
    if (K % 128) {
        s = launch_dep(k_zero_scale_pad, dim3(64), dim3(256), 0, (cudaStream_t)stream, "pact_weight_layout_cache", c.bwd);
        if (s != PACT_OK) return s;
    }
    *out = c;
    return PACT_OK;
}

}  // extern "C"
