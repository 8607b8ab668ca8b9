// lora.cu -- the BF16 LoRA branch of each frozen projection ([LORA]: PEFT explainer,
// section "LoRA": h = W0 x + B A x; [METHOD]: PACT blog summary, section "方法",
// paragraph after the bullets: A and B stay BF16 and are never quantized).
//
// The products are skinny (rank 16 per adapter) and bound by HBM:
//   T    = X . A^T           [M x R]   contraction over features   (forward)
//   U_i  = dY_i . B_i        [M x r]   contraction over segment i's outputs
//   dB_i = dY_i^T . T~_i     [N_i x r] contraction over tokens
//   dA^T = X~^T . U          [K x R]   contraction over tokens
// One tcgen05 kernel runs them all: a 128-row output tile times up to 64 columns,
// BF16 x BF16 -> FP32 in tensor memory (kind::f16), operands staged by TMA with the
// 128-byte swizzle either K-major or MN-major (the transposed products read the
// activations in place).  The contraction is split over CTAs so that enough SMs
// stream the activations; each split writes its FP32 partial tile to caller scratch
// and a finalize kernel sums the partials in a fixed order (deterministic), scales
// and rounds.
#include <cmath>
#include <mutex>

#include "quant.cuh"

namespace pact {
namespace lmma {

constexpr int BM = 128;        // output rows per CTA (MMA M)
constexpr int BK = 64;         // contraction elements per stage (128 bytes of BF16)
constexpr int MAX_STAGES = 6;  // ring depth: 6, or 3 where two CTAs should share an SM
constexpr int THREADS = 192;
// SiLU A operand (A_SILU): per stage the g and u tiles (BF16, 128 x 64 each, the
// 128-byte swizzle) land in a staging area, and 16 warps compute m = silu(g) u into
// the operand buffer (writing q(m) on the way) before the MMA reads it.
constexpr int SILU_WARPS = 16;
__host__ __device__ constexpr int threads_of(bool silu) { return silu ? 64 + 32 * SILU_WARPS : THREADS; }
// K-major BF16 A with its NVFP4 copy written (Params::aq): eight quantizing warps
// (2-9), two of each operand row's four 16-value blocks per thread
constexpr int QUANT_WARPS = 8;
constexpr int QUANT_THREADS = 64 + 32 * QUANT_WARPS;
__host__ __device__ constexpr int max_threads_of(bool silu) { return silu ? threads_of(true) : QUANT_THREADS; }
constexpr int A_BYTES = BM * BK * 2;     // 16384
constexpr int B_BYTES = 64 * BK * 2;     // 8192 per B part
// NVFP4 A operand: per stage, the codes of the A tile (128 x 64 values, 4 KiB) and
// up to two 512-byte scale chunks land in a staging area, and the four epilogue
// warps decode them into the BF16 operand buffer before the MMA reads it
constexpr int RAW_CODE_BYTES = BM * BK / 2;                      // 4096
constexpr int RAW_BYTES = RAW_CODE_BYTES + 1024;
// A stage holds the A tile, one or two B parts (the hi and lo halves of T or U) and,
// for an NVFP4 A, its staging area; all multiples of 1024 bytes.
__host__ __device__ constexpr int oper_bytes(int nparts) { return A_BYTES + nparts * B_BYTES; }
__host__ __device__ constexpr int stage_bytes(int nparts, bool fp4, bool silu = false) {
    return oper_bytes(nparts) + (fp4 ? RAW_BYTES : 0) + (silu ? 2 * A_BYTES : 0);
}
__host__ __device__ constexpr int smem_bytes(int nparts, bool fp4, int stages, bool silu = false) {
    return 1024 + stages * stage_bytes(nparts, fp4, silu) + 256;
}
constexpr int SM_SMEM = 233472;   // shared memory per SM (228 KiB), 1 KiB of it reserved per CTA
__host__ __device__ constexpr int ctas_per_sm(int nparts, bool fp4, int stages) {
    return SM_SMEM / (smem_bytes(nparts, fp4, stages) + 1024);
}
// Ring depth per product: the weight-gradient products (contraction over the tokens,
// two B parts) run 3 stages so that two CTAs share an SM; the forward and U products
// (contraction over the features) run one CTA per SM with 6 stages in flight, where
// more splits would cost more in FP32 partial-sum traffic than they gain.  A product
// whose A operand is decoded from NVFP4 in the kernel is bound by the decoding warps,
// so it runs 3 stages and two CTAs per SM (twice the decoders).
__host__ __device__ constexpr int stages_for(int nparts, bool fp4, bool silu = false) {
    return nparts == 2 || fp4 || silu ? 3 : 6;
}
constexpr int FWD_PER_SM = 1;   // split residency of the one-part products
constexpr uint32_t TMEM_COLS = 64;

// One output block: rows [row_begin, row_end) of the output, contraction
// [k_begin, k_end); b_coord positions the B operand (its row for a K-major B, its
// column for an MN-major B); out_col is the column of the block in the output.
struct Prob {
    int row_begin, row_end, k_begin, k_end, b_coord, out_col;
};

struct Params {
    int n_mma;          // MMA N (16..64, multiple of 16)
    int n_valid;        // output columns per block
    int nprob;
    Prob prob[3];
    int splits, k_per_split;
    int b_split;        // B holds hi + lo halves: second tile at column b_coord + b_lo_off
    int b_lo_off;
    float *ws;          // partials [split][row][ws_ld]
    int64_t ws_ld, ws_split_stride;
    // NVFP4 A operand (A_FP4): scale bytes of the tensor, its rows and columns
    // (K-major A: the tensor is [output rows x contraction]; MN-major: [contraction x
    // output rows])
    const uint8_t *a_scales;
    int64_t a_rows, a_cols;
    // With one split, the epilogue writes out_scale * acc itself as hi + lo BF16 halves
    // (hi at out[row * out_ld + col], lo at col + out_lo_off; k_finalize's mode 0) and no
    // finalize runs; null otherwise.
    pact_bf16 *out;
    int64_t out_ld, out_lo_off;
    float out_scale;
    // K-major BF16 A only: with aq.codes set, the epilogue warps (idle during the main
    // loop) also quantize each stage's A tile as it passes through shared memory and
    // write the NVFP4 copy aq of A ([rows x contraction]), padding rows' scales zeroed.
    // A_SILU: aq receives q(m) (always), m_out the BF16 m when not null.
    pact_nvfp4_t aq;
    pact_bf16 *m_out;
    int64_t m_ld;
};

// 8 E2M1 codes (element 0 in the low nibble) times their E4M3 block scale, as 8
// BF16 values (element 0 in the low half of .x).  Exact: E2M1 pairs convert to
// FP16 in hardware, the product with the scale has at most 6 significant bits in
// [2^-10, 2688] (exact in FP16 and in BF16), and FP16 -> FP32 -> BF16 is exact.
__device__ __forceinline__ uint4 decode8_bf16(uint32_t codes, uint32_t sbyte) {
    const __half2 s2 = __half2half2(__float2half_rn(e4m3_to_float(sbyte)));
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t h = e2m1x2_to_f16x2((codes >> (8 * i)) & 0xFFu);
        const float2 f = __half22float2(__hmul2(*reinterpret_cast<const __half2 *>(&h), s2));
        o[i] = pack_bf16x2(f.x, f.y);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// Decode one stage's NVFP4 A tile from the staging area into the BF16 operand
// buffer, laid out exactly as the TMA load of the BF16 tile with the 128-byte swizzle
// would lay it out (row q of 64 values at q * 128 bytes, its 16-byte chunk c at
// position c ^ (q % 8)).  128 threads, one 64-value row each.
//  K-major (A_MN = false): operand rows are the tensor's rows row0 .. row0 + 127,
//    the 64 values are columns k .. k + 63; codes staged as [128 rows x 32 bytes],
//    one scale chunk (rows of group row0 / 128, blocks k / 16 .. + 3).
//  MN-major (A_MN = true): operand rows are the tensor's columns row0 .. row0 + 127
//    (two 64-wide halves), the contraction runs over its rows k .. k + 63; codes
//    staged as [64 rows x 64 bytes], two scale chunks (one per half).
template <bool A_MN>
__device__ __forceinline__ void decode_stage(const uint8_t *raw, uint8_t *oper, const Params &p, int row0, int k,
                                             int tid) {
    int q, half;            // operand row within its 64-value-wide (half) tile, half index
    const uint8_t *codes;
    uint32_t sc;
    bool valid;
    if (!A_MN) {
        q = tid;
        half = 0;
        codes = raw + q * 32;
        sc = *reinterpret_cast<const uint32_t *>(raw + RAW_CODE_BYTES + (q & 31) * 16 + (q >> 5) * 4);
        valid = row0 + q < p.a_rows;
    } else {
        q = tid & 63;
        half = tid >> 6;
        codes = raw + q * 64 + half * 32;
        const int rr = (k & 127) + q;   // row within the scale group
        sc = *reinterpret_cast<const uint32_t *>(raw + RAW_CODE_BYTES + half * 512 + (rr & 31) * 16 +
                                                 ((rr >> 5) & 3) * 4);
        valid = (k + q < p.a_rows) && (row0 + 64 * half < p.a_cols);
    }
    const uint4 c0 = *reinterpret_cast<const uint4 *>(codes);
    const uint4 c1 = *reinterpret_cast<const uint4 *>(codes + 16);
    const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
    const uint32_t base = smem_u32(oper) + half * (A_BYTES / 2) + q * 128;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const uint4 v = valid ? decode8_bf16(w[c], (sc >> (8 * (c >> 1))) & 0xFFu) : make_uint4(0, 0, 0, 0);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(base + ((c ^ (q & 7)) << 4)), "r"(v.x),
                     "r"(v.y), "r"(v.z), "r"(v.w)
                     : "memory");
    }
}

template <bool A_MN, bool B_MN, bool A_FP4, bool A_SILU = false>
__global__ void __launch_bounds__(max_threads_of(A_SILU), 1)
k_lora_mma(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
           const __grid_constant__ CUtensorMap tmU, const Params p) {
    // tmU: the u tiles of an A_SILU kernel (tmA then maps g); unused otherwise
    const int nparts = p.b_split ? 2 : 1;
    const int STAGE_BYTES = stage_bytes(nparts, A_FP4, A_SILU), OPER_BYTES = oper_bytes(nparts);
    const Prob pr = p.prob[blockIdx.z];
    const int row0 = pr.row_begin + blockIdx.x * BM;
    if (row0 >= pr.row_end) return;  // block-uniform, before any shared state
    const int kb = pr.k_begin + blockIdx.y * p.k_per_split;
    const int ke = min(pr.k_end, kb + p.k_per_split);
    const int ktiles = ke > kb ? (ke - kb + BK - 1) / BK : 0;
    float *part = p.ws + (size_t)blockIdx.y * p.ws_split_stride;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool quantize_a = !A_MN && !A_FP4 && !A_SILU && p.aq.codes != nullptr;

    if (ktiles == 0) {  // empty split: its partial is zero
        pdl_wait();
        for (int i = threadIdx.x; i < BM * p.n_valid; i += blockDim.x) {
            const int r = row0 + i / p.n_valid;
            if (r < pr.row_end) part[(size_t)r * p.ws_ld + pr.out_col + i % p.n_valid] = 0.0f;
        }
        return;
    }

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + (((raw + 1023) & ~1023u) - raw);
    const int STAGES = stages_for(nparts, A_FP4, A_SILU);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE_BYTES);
    uint64_t *full = bars, *empty = bars + MAX_STAGES, *acc_full = bars + 2 * MAX_STAGES;
    uint64_t *raw_full = bars + 2 * MAX_STAGES + 1;   // [stages], A_FP4 only
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 3 * MAX_STAGES + 1);
    __shared__ uint32_t aborted;   // a bounded wait gave up somewhere in the CTA

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            // A_FP4: the producer's arrival (B bytes) and the four decoding warps'
            mbar_init(&full[s], A_SILU ? 1 + SILU_WARPS : A_FP4 ? 5 : 1);
            // the MMA warp's commit and, when they quantize A, the four epilogue warps'
            mbar_init(&empty[s], quantize_a ? 1 + QUANT_WARPS : 1);
            mbar_init(&raw_full[s], 1);
        }
        mbar_init(acc_full, 1);
        aborted = 0;
        fence_barrier_init();
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
        if (A_SILU) prefetch_tensormap(&tmU);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    pdl_wait();   // inputs of the previous kernel are complete from here on
    const uint32_t tmem = *tmem_slot;
    const uint32_t b_bytes = B_MN ? (uint32_t)B_BYTES : (uint32_t)p.n_mma * BK * 2;

    if (warp == 0) {
        if (lane == 0) {
            uint32_t stage = 0, phase = 0, pending = 0, pending_parity = 0, raw_pending = 0;
            for (int kt = 0; kt < ktiles; ++kt) {
                if (!mbar_wait(&empty[stage], phase ^ 1)) {
                    aborted = 1;
                    break;
                }
                uint8_t *st = smem + stage * STAGE_BYTES;
                const int k = kb + kt * BK;
                if (A_SILU) {
                    // the g and u tiles into the staging area; the SiLU warps fill the operand
                    uint8_t *rw = st + OPER_BYTES;
                    mbar_arrive_expect_tx(&raw_full[stage], 2 * A_BYTES);
                    tma_load_2d(rw, &tmA, &raw_full[stage], k, row0);
                    tma_load_2d(rw + A_BYTES, &tmU, &raw_full[stage], k, row0);
                    raw_pending |= 1u << stage;
                    mbar_arrive_expect_tx(&full[stage], nparts * b_bytes);
                } else if (A_FP4) {
                    // codes box and the scale chunk(s) of this stage's A tile
                    uint8_t *rw = st + OPER_BYTES;
                    const int64_t chunks_per_group = p.a_cols / 64;
                    if (!A_MN) {
                        mbar_arrive_expect_tx(&raw_full[stage], RAW_CODE_BYTES + 512);
                        tma_load_2d(rw, &tmA, &raw_full[stage], k / 2, row0);
                        bulk_load(rw + RAW_CODE_BYTES,
                                  p.a_scales + ((int64_t)(row0 / 128) * chunks_per_group + k / 64) * 512, 512,
                                  &raw_full[stage]);
                    } else {
                        // the second half's chunk exists only while its columns do
                        const uint32_t sbytes = (row0 / 64 + 1 < chunks_per_group) ? 1024u : 512u;
                        mbar_arrive_expect_tx(&raw_full[stage], RAW_CODE_BYTES + sbytes);
                        tma_load_2d(rw, &tmA, &raw_full[stage], row0 / 2, k);
                        bulk_load(rw + RAW_CODE_BYTES,
                                  p.a_scales + ((int64_t)(k / 128) * chunks_per_group + row0 / 64) * 512, sbytes,
                                  &raw_full[stage]);
                    }
                    raw_pending |= 1u << stage;
                    mbar_arrive_expect_tx(&full[stage], nparts * b_bytes);
                } else {
                    mbar_arrive_expect_tx(&full[stage], A_BYTES + nparts * b_bytes);
                    if (A_MN) {
                        tma_load_2d(st, &tmA, &full[stage], row0, k);
                        tma_load_2d(st + A_BYTES / 2, &tmA, &full[stage], row0 + 64, k);
                    } else {
                        tma_load_2d(st, &tmA, &full[stage], k, row0);
                    }
                }
                for (int h = 0; h < nparts; ++h) {
                    uint8_t *bd = st + A_BYTES + h * B_BYTES;
                    if (B_MN) tma_load_2d(bd, &tmB, &full[stage], pr.b_coord + h * p.b_lo_off, k);
                    else tma_load_2d(bd, &tmB, &full[stage], k, pr.b_coord);
                }
                pending |= 1u << stage;
                pending_parity = (pending_parity & ~(1u << stage)) | (phase << stage);
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
            }
            // copies land before the CTA may leave: the operand copies of the last use
            // of each stage complete `full` (with the decoders' arrivals), the staged
            // NVFP4 copies complete `raw_full`
            for (int s = 0; s < STAGES; ++s) {
                if (!(pending & (1u << s))) continue;
                const uint32_t par = (pending_parity >> s) & 1u;
                if ((A_FP4 || A_SILU) && (raw_pending & (1u << s))) mbar_wait(&raw_full[s], par);
                mbar_wait(&full[s], par);
            }
        }
    } else if (warp == 1) {
        const uint32_t idesc = idesc_bf16(BM, p.n_mma, A_MN, B_MN);
        uint32_t stage = 0, phase = 0, accum = 0;
        // the whole warp runs the loop converged; lane 0 alone issues (the _w forms)
        for (int kt = 0; kt < ktiles; ++kt) {
            const bool ok = warp_all(mbar_wait(&full[stage], phase));
            tc_fence_after();
            if (!ok) {
                aborted = 1;
                break;
            }
            const uint32_t st = smem_u32(smem + stage * STAGE_BYTES);
            for (int s = 0; s < BK / 16; ++s) {
                const uint64_t ad = A_MN ? smem_desc(st + s * 2048, A_BYTES / 2, 1024, SW_128)
                                         : smem_desc(st + s * 32, 16, 1024, SW_128);
                for (int h = 0; h < nparts; ++h) {
                    const uint32_t b0 = st + A_BYTES + h * B_BYTES;
                    const uint64_t bd = B_MN ? smem_desc(b0 + s * 2048, B_BYTES, 1024, SW_128)
                                             : smem_desc(b0 + s * 32, 16, 1024, SW_128);
                    mma_bf16_w(tmem, ad, bd, idesc, accum);
                    accum = 1;
                }
            }
            tc_commit_w(&empty[stage]);
            if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        // the epilogue waits for this; it also orders every MMA before the dealloc
        tc_commit_w(acc_full);
        __syncwarp();
    } else {
        bool ok = true;
        if (A_FP4) {
            // decode each stage's NVFP4 A tile into the BF16 operand buffer, then
            // announce it on the stage's `full` barrier (after a proxy fence: the
            // tensor core reads shared memory through the async proxy)
            // (one consumer per barrier: a parity wait may run at most one phase ahead)
            const int tid = threadIdx.x - 64;
            uint32_t stage = 0, phase = 0;
            for (int kt = 0; kt < ktiles; ++kt) {
                if (!(ok = warp_all(mbar_wait(&raw_full[stage], phase)))) {
                    aborted = 1;
                    break;
                }
                uint8_t *st = smem + stage * STAGE_BYTES;
                decode_stage<A_MN>(st + OPER_BYTES, st, p, row0, kb + kt * BK, tid);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&full[stage]);
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
            }
        } else if (A_SILU) {
            // m = BF16_RNE(silu(g) u) for the stage's A tile: thread t computes the
            // 16-value block b = t / 128 (columns 16 b .. 16 b + 15) of operand row q =
            // t % 128 from the staged g and u tiles (16-byte chunk c of row q at
            // (c ^ (q % 8)) * 16, as TMA's 128-byte swizzle lays them out), writes it to
            // the operand buffer in the same layout and its NVFP4 block to aq (and m to
            // m_out when set), then announces the stage (after a proxy fence: the tensor
            // core reads shared memory through the async proxy)
            const int t = threadIdx.x - 64, q = t & 127, b = t >> 7;
            const int64_t row = row0 + q, rows_pad = ((int64_t)pr.row_end + 127) & ~int64_t(127);
            const int64_t cols = p.aq.cols;
            uint8_t *qcodes = static_cast<uint8_t *>(p.aq.codes), *qscales = static_cast<uint8_t *>(p.aq.scales);
            auto silu8 = [](const uint4 &gw, const uint4 &uw) {
                float gv[8], uv[8], sv[8], mv[8];
                unpack8_bf16(gw, gv);
                unpack8_bf16(uw, uv);
#pragma unroll
                for (int i = 0; i < 8; ++i) sv[i] = sigmoid_fast(gv[i]);
                silu_mul8<false>(gv, uv, sv, mv);
                return make_uint4(pack_bf16x2(mv[0], mv[1]), pack_bf16x2(mv[2], mv[3]), pack_bf16x2(mv[4], mv[5]),
                                  pack_bf16x2(mv[6], mv[7]));
            };
            const uint32_t c0 = ((2 * b) ^ (q & 7)) << 4, c1 = ((2 * b + 1) ^ (q & 7)) << 4;
            uint32_t stage = 0, phase = 0;
            for (int kt = 0; kt < ktiles; ++kt) {
                if (!(ok = warp_all(mbar_wait(&raw_full[stage], phase)))) {
                    aborted = 1;
                    break;
                }
                const int k = kb + kt * BK;
                uint8_t *st = smem + stage * STAGE_BYTES;
                const uint32_t ga = smem_u32(st + OPER_BYTES) + q * 128, ua = ga + A_BYTES, oa = smem_u32(st) + q * 128;
                // the two 8-value halves through one copy of the SiLU code (the kernel's
                // roles compete for the instruction cache), then the block back from the
                // operand buffer for its quantization
#pragma unroll 1
                for (int h = 0; h < 2; ++h) {
                    const uint32_t c = h ? c1 : c0;
                    uint4 gw, uw;
                    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(gw.x), "=r"(gw.y), "=r"(gw.z), "=r"(gw.w) : "r"(ga + c));
                    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(uw.x), "=r"(uw.y), "=r"(uw.z), "=r"(uw.w) : "r"(ua + c));
                    const uint4 mw = silu8(gw, uw);   // rows past the end: 0 (zero-filled g, u)
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(oa + c), "r"(mw.x), "r"(mw.y),
                                 "r"(mw.z), "r"(mw.w)
                                 : "memory");
                }
                uint4 m0, m1;
                asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                             : "=r"(m0.x), "=r"(m0.y), "=r"(m0.z), "=r"(m0.w) : "r"(oa + c0) : "memory");
                asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                             : "=r"(m1.x), "=r"(m1.y), "=r"(m1.z), "=r"(m1.w) : "r"(oa + c1) : "memory");
                const int64_t c = k + 16 * b;
                if (row < pr.row_end) {
                    uint32_t lo, hi, sb;
                    quant16_bf16(m0, m1, &lo, &hi, &sb);
                    *reinterpret_cast<uint2 *>(qcodes + row * (cols >> 1) + (c >> 1)) = make_uint2(lo, hi);
                    qscales[scale_offset(row, c >> 4, cols)] = (uint8_t)sb;
                    if (p.m_out) {
                        uint4 *mp = reinterpret_cast<uint4 *>(p.m_out + row * p.m_ld + c);
                        mp[0] = m0;
                        mp[1] = m1;
                    }
                } else if (row < rows_pad) {
                    qscales[scale_offset(row, c >> 4, cols)] = 0;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&full[stage]);
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
            }
        } else if (quantize_a && warp < 2 + QUANT_WARPS) {
            // the NVFP4 copy of A: thread t quantizes blocks 2h, 2h + 1 (h = t / 128) of
            // operand row q = t % 128 of each stage (32 of its 64 values) from the
            // swizzled tile (16-byte chunk c of row q at (c ^ (q % 8)) * 16), then releases
            // the stage with the MMA's commit
            const int t = threadIdx.x - 64, q = t & 127, h = t >> 7;
            const int64_t row = row0 + q, rows_pad = ((int64_t)pr.row_end + 127) & ~int64_t(127);
            const int64_t cols = p.aq.cols;
            uint8_t *qcodes = static_cast<uint8_t *>(p.aq.codes), *qscales = static_cast<uint8_t *>(p.aq.scales);
            uint32_t stage = 0, phase = 0;
            for (int kt = 0; kt < ktiles; ++kt) {
                if (!(ok = warp_all(mbar_wait(&full[stage], phase)))) {
                    aborted = 1;
                    break;
                }
                const int k = kb + kt * BK;
                const uint32_t a = smem_u32(smem + stage * STAGE_BYTES) + q * 128;
                // blocks k/16 .. k/16 + 3 (k a multiple of 64) are one word of the scale
                // layout: this thread's two are its half h
                uint16_t *sp = reinterpret_cast<uint16_t *>(qscales + scale_offset(row, k >> 4, cols)) + h;
                if (row < pr.row_end) {
                    uint32_t cw[4], sw = 0;
#pragma unroll
                    for (int bb = 0; bb < 2; ++bb) {
                        const int b = 2 * h + bb;
                        uint4 wa, wb;
                        asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                                     : "=r"(wa.x), "=r"(wa.y), "=r"(wa.z), "=r"(wa.w)
                                     : "r"(a + (((2 * b) ^ (q & 7)) << 4)));
                        asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                                     : "=r"(wb.x), "=r"(wb.y), "=r"(wb.z), "=r"(wb.w)
                                     : "r"(a + (((2 * b + 1) ^ (q & 7)) << 4)));
                        uint32_t sb;
                        quant16_bf16(wa, wb, &cw[2 * bb], &cw[2 * bb + 1], &sb);
                        sw |= sb << (8 * bb);
                    }
                    *reinterpret_cast<uint4 *>(qcodes + row * (cols >> 1) + (k >> 1) + 16 * h) =
                        make_uint4(cw[0], cw[1], cw[2], cw[3]);
                    *sp = (uint16_t)sw;
                } else if (row < rows_pad) {
                    *sp = 0;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[stage]);
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
            }
        }
    }
    if (warp >= 2 && warp < 6) {
        // the epilogue: warps 2-5, one tensor-memory sub-partition each
        bool ok = true;
        const int sub = warp & 3;
        ok = mbar_wait(acc_full, 0) && ok;
        tc_fence_after();
        const int r = row0 + sub * 32 + lane;
        for (int c = 0; c < p.n_mma / 16; ++c) {
            uint32_t v[16];
            tmem_ld_32x32b_x16(tmem + ((uint32_t)(sub * 32) << 16) + c * 16, v);
            tmem_ld_wait();
            if (r < pr.row_end && p.out) {
                if (c * 16 < p.n_valid) {   // whole 16-column chunks (n_valid is a multiple of 16)
                    uint32_t hi[8], lo[8];
#pragma unroll
                    for (int j = 0; j < 16; j += 2) {
                        // k_finalize's arithmetic for one split: (0 + acc) * scale, then hi, lo
                        const float a0 = ok ? (0.0f + __uint_as_float(v[j])) * p.out_scale : __int_as_float(0x7fc00000);
                        const float a1 =
                            ok ? (0.0f + __uint_as_float(v[j + 1])) * p.out_scale : __int_as_float(0x7fc00000);
                        hi[j / 2] = pack_bf16x2(a0, a1);
                        lo[j / 2] = pack_bf16x2(a0 - bf16lo(hi[j / 2]), a1 - bf16hi(hi[j / 2]));
                    }
                    uint4 *oh = reinterpret_cast<uint4 *>(p.out + (size_t)r * p.out_ld + pr.out_col + c * 16);
                    uint4 *ol = reinterpret_cast<uint4 *>(p.out + (size_t)r * p.out_ld + pr.out_col + c * 16 + p.out_lo_off);
                    oh[0] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                    oh[1] = make_uint4(hi[4], hi[5], hi[6], hi[7]);
                    ol[0] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                    ol[1] = make_uint4(lo[4], lo[5], lo[6], lo[7]);
                }
            } else if (r < pr.row_end) {
                // a wait that gave up leaves NaN partials, so the result is NaN rather
                // than whatever the scratch held before
                float *dst = part + (size_t)r * p.ws_ld + pr.out_col + c * 16;
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    if (c * 16 + j < p.n_valid) dst[j] = ok ? __uint_as_float(v[j]) : __int_as_float(0x7fc00000);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
    if (aborted && warp >= 2 && warp < 6) {
        // some role of this CTA gave up a wait: its partial tile is NaN, whatever the
        // accumulator held
        const int r = row0 + (warp & 3) * 32 + lane;
        if (r < pr.row_end && p.out) {
            for (int c = 0; c < p.n_valid; ++c) {
                p.out[(size_t)r * p.out_ld + pr.out_col + c] = 0x7FC0u;   // BF16 NaN
                p.out[(size_t)r * p.out_ld + pr.out_col + c + p.out_lo_off] = 0x7FC0u;
            }
        } else if (r < pr.row_end) {
            for (int c = 0; c < p.n_valid; ++c) part[(size_t)r * p.ws_ld + pr.out_col + c] = __int_as_float(0x7fc00000);
        }
    }
}

// out = scale * sum_s ws[s][row][col] for rows x cols, written as
//   mode 0: hi + lo BF16 halves (hi at out[row * ldo + col], lo at col + lo_off)
//   mode 1: BF16
//   mode 2: BF16 transposed (out[col * ldo + row])
//   mode 3, 4: as modes 1, 2 in FP32 (out32)
// The partials are summed in split order (deterministic).  One launch serves one or
// two such jobs (the index space of the second follows the first's).  A job with
// `vec` set (modes 0, 1, 3; every stride a multiple of 4 elements, the pointers
// aligned for it) takes 4 consecutive columns per thread: one 16-byte load per
// partial, one 8-byte (BF16) or 16-byte (FP32) store per output; the sums are the
// same, element by element.
struct FinJob {
    const float *ws;
    int splits;
    int64_t split_stride, ws_ld, rows, cols;
    float scale;
    int mode;
    pact_bf16 *out;
    int64_t ldo, lo_off;
    float *out32;
    int vec;
};

__device__ __forceinline__ int64_t fin_items(const FinJob &j) { return j.rows * (j.vec ? j.cols / 4 : j.cols); }

__global__ void k_finalize(const FinJob j0, const FinJob j1, int njobs) {
    pdl_wait();
    const int64_t n0 = fin_items(j0);
    const int64_t n = n0 + (njobs > 1 ? fin_items(j1) : 0);
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const bool second = i >= n0;
        const FinJob &j = second ? j1 : j0;
        const int64_t ii = second ? i - n0 : i;
        if (j.vec) {
            const int64_t c4 = j.cols / 4, r = ii / c4, c = (ii % c4) * 4;
            float a[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            for (int s = 0; s < j.splits; ++s) {
                const float4 v = *reinterpret_cast<const float4 *>(j.ws + s * j.split_stride + r * j.ws_ld + c);
                a[0] += v.x;
                a[1] += v.y;
                a[2] += v.z;
                a[3] += v.w;
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) a[e] *= j.scale;
            if (j.mode == 3) {
                *reinterpret_cast<float4 *>(j.out32 + r * j.ldo + c) = make_float4(a[0], a[1], a[2], a[3]);
                continue;
            }
            const uint32_t h0 = pack_bf16x2(a[0], a[1]), h1 = pack_bf16x2(a[2], a[3]);
            *reinterpret_cast<uint2 *>(j.out + r * j.ldo + c) = make_uint2(h0, h1);
            if (j.mode == 0) {
                const uint32_t l0 = pack_bf16x2(a[0] - bf16lo(h0), a[1] - bf16hi(h0));
                const uint32_t l1 = pack_bf16x2(a[2] - bf16lo(h1), a[3] - bf16hi(h1));
                *reinterpret_cast<uint2 *>(j.out + r * j.ldo + c + j.lo_off) = make_uint2(l0, l1);
            }
            continue;
        }
        const bool tr = j.mode == 2 || j.mode == 4;
        const int64_t r = tr ? ii % j.rows : ii / j.cols, c = tr ? ii / j.rows : ii % j.cols;
        float acc = 0.0f;
        for (int s = 0; s < j.splits; ++s) acc += j.ws[s * j.split_stride + r * j.ws_ld + c];
        acc *= j.scale;
        if (j.mode >= 3) {
            j.out32[tr ? c * j.ldo + r : r * j.ldo + c] = acc;
            continue;
        }
        const __nv_bfloat16 hi = __float2bfloat16_rn(acc);
        if (j.mode == 2) {
            j.out[c * j.ldo + r] = __bfloat16_as_ushort(hi);
        } else {
            j.out[r * j.ldo + c] = __bfloat16_as_ushort(hi);
            if (j.mode == 0)
                j.out[r * j.ldo + c + j.lo_off] = __bfloat16_as_ushort(__float2bfloat16_rn(acc - __bfloat162float(hi)));
        }
    }
}

// ---------------------------------------------------------------- host side
static int finalize_grid(int64_t n);

typedef CUresult (*EncodeTiled)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// 2-D tiled map over a row-major matrix of `esize`-byte elements: `inner` elements
// per row (row stride `ld` elements), `outer` rows.
static pact_status map_2d(CUtensorMap *m, CUtensorMapDataType dt, int esize, CUtensorMapSwizzle sw, const void *base,
                          uint64_t inner, uint64_t outer, uint64_t ld, uint32_t box_inner, uint32_t box_outer,
                          const char *what) {
    // looked up once (a function-local static's initialisation is thread-safe)
    static const EncodeTiled enc = [] {
        void *fp = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fp, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<EncodeTiled>(fp);
        return static_cast<EncodeTiled>(nullptr);
    }();
    if (!enc) return fail(PACT_ERR_CUDA, "%s: cuTensorMapEncodeTiled unavailable", what);
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {ld * (uint64_t)esize};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t es[2] = {1, 1};
    CUresult r = enc(m, dt, 2, const_cast<void *>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PACT_ERR_CUDA, "%s: cuTensorMapEncodeTiled failed (%d)", what, (int)r);
    return PACT_OK;
}

// BF16 row-major matrix, 128-byte swizzle (the MMA operand layout).
static pact_status map_bf16(CUtensorMap *m, const void *base, uint64_t inner, uint64_t outer, uint64_t ld,
                            uint32_t box_inner, uint32_t box_outer, const char *what) {
    return map_2d(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, CU_TENSOR_MAP_SWIZZLE_128B, base, inner, outer, ld,
                  box_inner, box_outer, what);
}

// The code bytes of an NVFP4 tensor ([rows x cols / 2] bytes), unswizzled boxes of
// box_bytes x box_rows: the staging copies of an NVFP4 A operand.
static pact_status map_codes(CUtensorMap *m, const pact_nvfp4_t &t, uint32_t box_bytes, uint32_t box_rows,
                             const char *what) {
    return map_2d(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, CU_TENSOR_MAP_SWIZZLE_NONE, t.codes, (uint64_t)t.cols / 2,
                  (uint64_t)t.rows, (uint64_t)t.cols / 2, box_bytes, box_rows, what);
}

// Params of an NVFP4 A operand.
static void set_fp4_a(Params &p, const pact_nvfp4_t &t) {
    p.a_scales = static_cast<const uint8_t *>(t.scales);
    p.a_rows = t.rows;
    p.a_cols = t.cols;
}

template <bool A_MN, bool B_MN, bool A_FP4 = false, bool A_SILU = false>
static pact_status launch_mma(const CUtensorMap &ta, const CUtensorMap &tb, const Params &p, int row_tiles,
                              cudaStream_t st, const char *what, const CUtensorMap *tu = nullptr) {
    static std::atomic<bool> done[64];   // per device; setting the attribute twice is harmless
    const int d = current_device();
    const int np = p.b_split ? 2 : 1;
    const int smem = smem_bytes(np, A_FP4, stages_for(np, A_FP4, A_SILU), A_SILU);
    if (d >= 0 && d < 64 && !done[d].load(std::memory_order_acquire)) {
        int mx = 0;
        for (int n = 1; n <= 2; ++n) {
            const int b = smem_bytes(n, A_FP4, stages_for(n, A_FP4, A_SILU), A_SILU);
            mx = mx > b ? mx : b;
        }
        cudaError_t e = cudaFuncSetAttribute(k_lora_mma<A_MN, B_MN, A_FP4, A_SILU>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, mx);
        if (e != cudaSuccess) return fail(PACT_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
        done[d].store(true, std::memory_order_release);
    }
    dim3 grid((unsigned)row_tiles, (unsigned)p.splits, (unsigned)p.nprob);
    const bool quant = !A_MN && !A_FP4 && !A_SILU && p.aq.codes != nullptr;   // the kernel's quantize_a
    return launch_dep(k_lora_mma<A_MN, B_MN, A_FP4, A_SILU>, grid, dim3(quant ? QUANT_THREADS : threads_of(A_SILU)), smem,
                      st, what, ta, tb,
                      tu ? *tu : ta, p);
}

static FinJob fin_job(const float *ws, const Params &p, int64_t rows, int64_t cols, float scale, int mode,
                      void *out, int64_t ldo, int64_t lo_off) {
    // 4 columns per thread where every stride is a multiple of 4 elements and the
    // pointers are aligned for 16-byte partial loads and 8-byte (BF16) or 16-byte
    // (FP32) output stores
    const uintptr_t oa = reinterpret_cast<uintptr_t>(out);
    const int vec = (mode == 0 || mode == 1 || mode == 3) && cols % 4 == 0 && p.ws_ld % 4 == 0 &&
                    p.ws_split_stride % 4 == 0 && ldo % 4 == 0 && lo_off % 4 == 0 &&
                    (reinterpret_cast<uintptr_t>(ws) & 15) == 0 && (oa & (mode == 3 ? 15 : 7)) == 0;
    return FinJob{ws, p.splits, p.ws_split_stride, p.ws_ld, rows, cols, scale, mode,
                  mode >= 3 ? nullptr : static_cast<pact_bf16 *>(out), ldo, lo_off,
                  mode >= 3 ? static_cast<float *>(out) : nullptr, vec};
}

// A product with one split writes its hi + lo output from the epilogue (mode 0 of
// k_finalize, with the same arithmetic) instead of partials and a finalize launch.
static void set_direct_out(Params &p, pact_bf16 *out, int64_t ldo, int64_t lo_off, float scale) {
    if (p.splits != 1) return;
    p.out = out;
    p.out_ld = ldo;
    p.out_lo_off = lo_off;
    p.out_scale = scale;
}

static pact_status finalize(const FinJob &j0, const FinJob *j1, cudaStream_t st, const char *what) {
    auto items = [](const FinJob &j) { return j.rows * (j.vec ? j.cols / 4 : j.cols); };   // as fin_items
    const int64_t n = items(j0) + (j1 ? items(*j1) : 0);
    return launch_dep(k_finalize, dim3(finalize_grid(n)), dim3(256), 0, st, what, j0, j1 ? *j1 : j0, j1 ? 2 : 1);
}

// Splits of a contraction of length `len` so that `blocks` output blocks x splits
// CTAs fill the SMs in ONE wave (`per_sm` CTAs of this kind fit on an SM), each split
// at least 4 stages long.  Rounding the split count up instead left a nearly empty
// second wave.
static void choose_split(int64_t len, int64_t blocks, int per_sm, int *splits, int *kps) {
    int64_t s = (int64_t)sm_count() * per_sm / (blocks > 0 ? blocks : 1);
    const int64_t max_s = (len + 4 * BK - 1) / (4 * BK);
    if (s > max_s) s = max_s;
    if (s < 1) s = 1;
    int64_t k = (len + s - 1) / s;
    k = (k + BK - 1) / BK * BK;
    *splits = (int)((len + k - 1) / k);
    *kps = (int)k;
}

static int finalize_grid(int64_t n) {
    const int64_t g = (n + 255) / 256;
    const int64_t cap = (int64_t)sm_count() * 8;
    return (int)(g < 1 ? 1 : (g > cap ? cap : g));
}

static size_t round256(size_t b) { return (b + 255) & ~(size_t)255; }

// Bytes of FP32 partials for rows x cols outputs split `splits` ways.
static size_t partial_bytes(int64_t rows, int64_t cols, int splits) {
    return round256((size_t)(rows * cols * 4) * (size_t)splits);
}

// scale * X . A^T for X [M x K] (map tx: BF16 rows, or the codes of the NVFP4 X when
// xq is given) and A [R x K], written hi/lo into out (row stride ldo, lo at column R);
// ws holds the partials.
static pact_status rows_times_a(const CUtensorMap &tx, const pact_nvfp4_t *xq, int64_t M, int64_t K,
                                const pact_bf16 *A, int R, float scale, pact_bf16 *out, int64_t ldo, float *ws,
                                cudaStream_t st, const char *what, const pact_nvfp4_t *aq = nullptr) {
    CUtensorMap tb;
    pact_status s = map_bf16(&tb, A, K, R, K, 64, R, what);
    if (s != PACT_OK) return s;
    Params p = {};
    p.n_mma = R;
    p.n_valid = R;
    p.nprob = 1;
    p.prob[0] = Prob{0, (int)M, 0, (int)K, 0, 0};
    const int tiles = (int)((M + BM - 1) / BM);
    choose_split(K, tiles, xq ? ctas_per_sm(1, true, stages_for(1, true)) : FWD_PER_SM, &p.splits, &p.k_per_split);
    p.ws = ws;
    p.ws_ld = R;
    p.ws_split_stride = M * R;
    set_direct_out(p, out, ldo, R, scale);
    if (aq) p.aq = *aq;   // BF16 x only (the kernel quantizes K-major BF16 A tiles)
    if (xq) {
        set_fp4_a(p, *xq);
        s = launch_mma<false, false, true>(tx, tb, p, tiles, st, what);
    } else {
        s = launch_mma<false, false>(tx, tb, p, tiles, st, what);
    }
    if (s != PACT_OK || p.out) return s;
    return finalize(fin_job(ws, p, M, R, scale, 0, out, ldo, R), nullptr, st, what);
}

static pact_status check_segments(int64_t N, int nseg, const int64_t *seg_end, const char *what) {
    int64_t prev = 0;
    for (int i = 0; i < nseg; ++i) {
        PACT_CHECK(seg_end[i] > prev && seg_end[i] % 64 == 0 && (i + 1 < nseg || seg_end[i] == N), PACT_ERR_SHAPE,
                   "%s: segment ends must increase by multiples of 64 and end at N", what);
        prev = seg_end[i];
    }
    return PACT_OK;
}

}  // namespace lmma
}  // namespace pact

using namespace pact;
using namespace pact::lmma;

extern "C" {

static int splits_of(int64_t len, int64_t blocks, int per_sm) {
    int s, k;
    choose_split(len, blocks, per_sm, &s, &k);
    return s;
}

// Workspace bounds cover both the BF16 and the NVFP4 form of X~ (more CTAs per SM
// give at least as many splits).
// residency of the T~ product: the NVFP4-decoding form fits more CTAs per SM (splits
// and workspace are sized for the larger of the two)
constexpr int T_PER_SM = ctas_per_sm(1, true, stages_for(1, true)) > FWD_PER_SM ? ctas_per_sm(1, true, stages_for(1, true))
                                                                                 : FWD_PER_SM;
constexpr int DA_PER_SM = ctas_per_sm(2, false, stages_for(2, false)) > ctas_per_sm(2, true, stages_for(2, true))
                              ? ctas_per_sm(2, false, stages_for(2, false))
                              : ctas_per_sm(2, true, stages_for(2, true));

size_t pact_lora_fwd_workspace_bytes(int64_t M, int64_t K, int R) {
    return partial_bytes(M, R, splits_of(K, (M + BM - 1) / BM, FWD_PER_SM));
}

static pact_status lora_fwd(const pact_bf16 *x, int64_t ldx, int64_t M, int64_t K, const pact_bf16 *A, int R,
                            float scale, pact_bf16 *T, int64_t ldt, const pact_nvfp4_t *xq, void *workspace,
                            size_t ws_bytes, pact_stream_t stream, const char *what) {
    PACT_CHECK(x && A && T && workspace, PACT_ERR_INVALID_ARG, "%s: NULL argument", what);
    PACT_CHECK(M >= 1 && M <= 0x7FFFFFFF && K >= 64 && K % 64 == 0 && K <= 0x7FFFFFFF && R >= 16 && R <= 64 &&
                   R % 16 == 0,
               PACT_ERR_SHAPE, "%s: need M >= 1, K a multiple of 64, R in {16, 32, 48, 64}", what);
    PACT_CHECK(ldx >= K && ldx % 8 == 0 && ldt >= 2 * R && ldt % 8 == 0 && aligned16(x) && aligned16(A) &&
                   aligned16(T) && aligned16(workspace),
               PACT_ERR_ALIGN, "%s: pointers 16-byte aligned, leading dims %% 8 == 0", what);
    PACT_CHECK(ws_bytes >= pact_lora_fwd_workspace_bytes(M, K, R), PACT_ERR_INVALID_ARG,
               "%s: workspace too small (%zu < %zu)", what, ws_bytes, pact_lora_fwd_workspace_bytes(M, K, R));
    pact_status s = xq ? check_nvfp4(xq, M, K, "xq") : PACT_OK;
    if (s != PACT_OK) return s;
    CUtensorMap tx;
    s = map_bf16(&tx, x, K, M, ldx, 64, BM, what);
    if (s != PACT_OK) return s;
    return rows_times_a(tx, nullptr, M, K, A, R, scale, T, ldt, static_cast<float *>(workspace), (cudaStream_t)stream,
                        what, xq);
}

pact_status pact_lora_fwd(const pact_bf16 *x, int64_t ldx, int64_t M, int64_t K, const pact_bf16 *A, int R,
                          float scale, pact_bf16 *T, int64_t ldt, void *workspace, size_t ws_bytes,
                          pact_stream_t stream) {
    return lora_fwd(x, ldx, M, K, A, R, scale, T, ldt, nullptr, workspace, ws_bytes, stream, "pact_lora_fwd");
}

pact_status pact_lora_fwd_quant(const pact_bf16 *x, int64_t ldx, int64_t M, int64_t K, const pact_bf16 *A, int R,
                                float scale, pact_bf16 *T, int64_t ldt, const pact_nvfp4_t *xq, void *workspace,
                                size_t ws_bytes, pact_stream_t stream) {
    PACT_CHECK(xq, PACT_ERR_INVALID_ARG, "pact_lora_fwd_quant: NULL argument");
    return lora_fwd(x, ldx, M, K, A, R, scale, T, ldt, xq, workspace, ws_bytes, stream, "pact_lora_fwd_quant");
}

pact_status pact_lora_fwd_silu(const pact_bf16 *g, const pact_bf16 *u, int64_t ld_gu, int64_t M, int64_t I,
                               const pact_bf16 *A, int R, float scale, pact_bf16 *T, int64_t ldt,
                               const pact_nvfp4_t *mq, pact_bf16 *m, int64_t ldm, void *workspace, size_t ws_bytes,
                               pact_stream_t stream) {
    const char *what = "pact_lora_fwd_silu";
    PACT_CHECK(g && u && A && T && mq && workspace, PACT_ERR_INVALID_ARG, "%s: NULL argument", what);
    PACT_CHECK(M >= 1 && M <= 0x7FFFFFFF && I >= 64 && I % 64 == 0 && I <= 0x7FFFFFFF && R >= 16 && R <= 64 &&
                   R % 16 == 0,
               PACT_ERR_SHAPE, "%s: need M >= 1, I a multiple of 64, R in {16, 32, 48, 64}", what);
    PACT_CHECK(ld_gu >= I && ld_gu % 8 == 0 && ldt >= 2 * R && ldt % 8 == 0 && (!m || (ldm >= I && ldm % 8 == 0)) &&
                   aligned16(g) && aligned16(u) && aligned16(A) && aligned16(T) && aligned16(m) && aligned16(workspace),
               PACT_ERR_ALIGN, "%s: pointers 16-byte aligned, leading dims %% 8 == 0", what);
    PACT_CHECK(ws_bytes >= pact_lora_fwd_workspace_bytes(M, I, R), PACT_ERR_INVALID_ARG,
               "%s: workspace too small (%zu < %zu)", what, ws_bytes, pact_lora_fwd_workspace_bytes(M, I, R));
    pact_status s = check_nvfp4(mq, M, I, "mq");
    if (s != PACT_OK) return s;
    CUtensorMap tg, tu, tb;
    s = map_bf16(&tg, g, I, M, ld_gu, 64, BM, what);
    if (s == PACT_OK) s = map_bf16(&tu, u, I, M, ld_gu, 64, BM, what);
    if (s == PACT_OK) s = map_bf16(&tb, A, I, R, I, 64, R, what);
    if (s != PACT_OK) return s;
    Params p = {};
    p.n_mma = R;
    p.n_valid = R;
    p.nprob = 1;
    p.prob[0] = Prob{0, (int)M, 0, (int)I, 0, 0};
    const int tiles = (int)((M + BM - 1) / BM);
    choose_split(I, tiles, FWD_PER_SM, &p.splits, &p.k_per_split);
    float *ws = static_cast<float *>(workspace);
    p.ws = ws;
    p.ws_ld = R;
    p.ws_split_stride = M * R;
    set_direct_out(p, T, ldt, R, scale);
    p.aq = *mq;
    p.m_out = m;
    p.m_ld = ldm;
    cudaStream_t st = (cudaStream_t)stream;
    s = launch_mma<false, false, false, true>(tg, tb, p, tiles, st, what, &tu);
    if (s != PACT_OK || p.out) return s;
    return finalize(fin_job(ws, p, M, R, scale, 0, T, ldt, R), nullptr, st, what);
}

int pact_lora_fwd_launches(int64_t M, int64_t K, int R) {
    (void)R;
    return splits_of(K, (M + BM - 1) / BM, FWD_PER_SM) == 1 ? 1 : 2;
}

// Upper bound over segmentations: one segment may span all N outputs.
size_t pact_lora_bwd_u_workspace_bytes(int64_t M, int64_t N, int r, int nseg) {
    return partial_bytes(M, (int64_t)r * nseg, splits_of(N, (M + BM - 1) / BM, FWD_PER_SM));
}

static pact_status lora_bwd_u(const pact_bf16 *dy, int64_t lddy, int64_t M, int64_t N, const pact_bf16 *B, int r,
                              int nseg, const int64_t *seg_end, float scale, pact_bf16 *U, int64_t ldu,
                              const pact_nvfp4_t *dyq, void *workspace, size_t ws_bytes, pact_stream_t stream) {
    PACT_CHECK(dy && B && U && seg_end && workspace, PACT_ERR_INVALID_ARG, "pact_lora_bwd_u: NULL argument");
    PACT_CHECK(M >= 1 && M <= 0x7FFFFFFF && N >= 64 && N % 64 == 0 && N <= 0x7FFFFFFF &&
                   (r == 16 || r == 32 || r == 48 || r == 64) && nseg >= 1 && nseg <= 3 && nseg * r <= 64,
               PACT_ERR_SHAPE, "pact_lora_bwd_u: bad shape (r in {16,32,48,64}, nseg <= 3, nseg*r <= 64)");
    pact_status s = check_segments(N, nseg, seg_end, "pact_lora_bwd_u");
    if (s != PACT_OK) return s;
    const int R = nseg * r;
    PACT_CHECK(lddy >= N && lddy % 8 == 0 && ldu >= 2 * R && ldu % 8 == 0 && aligned16(dy) && aligned16(B) &&
                   aligned16(U) && aligned16(workspace),
               PACT_ERR_ALIGN, "pact_lora_bwd_u: pointers 16-byte aligned, leading dims %% 8 == 0");
    PACT_CHECK(ws_bytes >= pact_lora_bwd_u_workspace_bytes(M, N, r, nseg), PACT_ERR_INVALID_ARG,
               "pact_lora_bwd_u: workspace too small");
    if (dyq) {
        s = check_nvfp4(dyq, M, N, "dyq");
        if (s != PACT_OK) return s;
    }
    cudaStream_t st = (cudaStream_t)stream;
    CUtensorMap ta, tb;
    s = map_bf16(&ta, dy, N, M, lddy, 64, BM, "pact_lora_bwd_u");
    if (s == PACT_OK) s = map_bf16(&tb, B, r, N, r, 64, 64, "pact_lora_bwd_u");  // B^T, MN-major
    if (s != PACT_OK) return s;
    Params p = {};
    p.n_mma = 64;
    p.n_valid = r;
    p.nprob = nseg;
    int64_t longest = 0, prev = 0;
    for (int i = 0; i < nseg; ++i) {
        p.prob[i] = Prob{0, (int)M, (int)prev, (int)seg_end[i], 0, i * r};
        if (seg_end[i] - prev > longest) longest = seg_end[i] - prev;
        prev = seg_end[i];
    }
    const int tiles = (int)((M + BM - 1) / BM);
    choose_split(longest, (int64_t)tiles * nseg, FWD_PER_SM, &p.splits, &p.k_per_split);
    float *ws = static_cast<float *>(workspace);
    p.ws = ws;
    p.ws_ld = R;
    p.ws_split_stride = M * R;
    set_direct_out(p, U, ldu, R, scale);
    if (dyq) p.aq = *dyq;
    s = launch_mma<false, true>(ta, tb, p, tiles, st, "pact_lora_bwd_u");
    if (s != PACT_OK || p.out) return s;
    return finalize(fin_job(ws, p, M, R, scale, 0, U, ldu, R), nullptr, st, "pact_lora_bwd_u");
}

pact_status pact_lora_bwd_u(const pact_bf16 *dy, int64_t lddy, int64_t M, int64_t N, const pact_bf16 *B, int r,
                            int nseg, const int64_t *seg_end, float scale, pact_bf16 *U, int64_t ldu,
                            void *workspace, size_t ws_bytes, pact_stream_t stream) {
    return lora_bwd_u(dy, lddy, M, N, B, r, nseg, seg_end, scale, U, ldu, nullptr, workspace, ws_bytes, stream);
}

pact_status pact_lora_bwd_u_quant(const pact_bf16 *dy, int64_t lddy, int64_t M, int64_t N, const pact_bf16 *B,
                                  int r, int nseg, const int64_t *seg_end, float scale, pact_bf16 *U, int64_t ldu,
                                  const pact_nvfp4_t *dyq, void *workspace, size_t ws_bytes, pact_stream_t stream) {
    PACT_CHECK(dyq, PACT_ERR_INVALID_ARG, "pact_lora_bwd_u_quant: NULL argument");
    return lora_bwd_u(dy, lddy, M, N, B, r, nseg, seg_end, scale, U, ldu, dyq, workspace, ws_bytes, stream);
}

int pact_lora_bwd_launches(int64_t M, int64_t K, int R, int nvfp4_x) {
    (void)R;
    // T~ (a finalize unless unsplit), the dB and dA products, one finalize for both
    const int t_splits = splits_of(K, (M + BM - 1) / BM, nvfp4_x ? ctas_per_sm(1, true, stages_for(1, true)) : FWD_PER_SM);
    return (t_splits == 1 ? 1 : 2) + 3;
}

int pact_lora_bwd_u_launches(int64_t M, int64_t N, int r, int nseg, const int64_t *seg_end) {
    (void)r;
    int64_t longest = 0, prev = 0;
    for (int i = 0; i < nseg; ++i) {
        if (seg_end[i] - prev > longest) longest = seg_end[i] - prev;
        prev = seg_end[i];
    }
    return splits_of(longest, ((M + BM - 1) / BM) * nseg, FWD_PER_SM) == 1 ? 1 : 2;
}

// Upper bound over segmentations: the dB output blocks number at least N / 128.
size_t pact_lora_bwd_workspace_bytes(int64_t M, int64_t N, int64_t K, int r, int nseg) {
    const int64_t R = (int64_t)r * nseg;
    return partial_bytes(M, R, splits_of(K, (M + BM - 1) / BM, T_PER_SM))      /* T~ partials */
           + round256((size_t)(M * 2 * R * 2))                                  /* T~ hi/lo */
           + partial_bytes(N, r, splits_of(M, (N + BM - 1) / BM, ctas_per_sm(2, false, stages_for(2, false))))  /* dB partials */
           + partial_bytes(K, R, splits_of(M, (K + BM - 1) / BM, DA_PER_SM));  /* dA^T partials */
}

pact_status pact_lora_bwd(const pact_lora_bwd_t *g, void *workspace, size_t ws_bytes, pact_stream_t stream) {
    PACT_CHECK(g && workspace, PACT_ERR_INVALID_ARG, "pact_lora_bwd: NULL argument");
    PACT_CHECK(g->dy && g->A && g->U && g->dA && g->dB && ((g->x != nullptr) != (g->xq != nullptr)),
               PACT_ERR_INVALID_ARG, "pact_lora_bwd: dy, A, U, dA, dB and exactly one of x / xq are required");
    const int64_t M = g->M, N = g->N, K = g->K;
    const int r = g->r, nseg = g->nseg;
    PACT_CHECK(M >= 1 && M <= 0x7FFFFFFF && N >= 64 && N % 64 == 0 && N <= 0x7FFFFFFF && K >= 64 && K % 64 == 0 &&
                   K <= 0x7FFFFFFF && (r == 16 || r == 32 || r == 48 || r == 64) && nseg >= 1 && nseg <= 3 &&
                   nseg * r <= 64,
               PACT_ERR_SHAPE, "pact_lora_bwd: bad shape");
    PACT_CHECK(g->u_gexp >= -100 && g->u_gexp <= 100, PACT_ERR_INVALID_ARG, "pact_lora_bwd: |u_gexp| <= 100 required");
    PACT_CHECK(g->grads_fp32 == 0 || g->grads_fp32 == 1, PACT_ERR_INVALID_ARG, "pact_lora_bwd: grads_fp32 is 0 or 1");
    pact_status s = check_segments(N, nseg, g->seg_end, "pact_lora_bwd");
    if (s != PACT_OK) return s;
    const int R = nseg * r;
    PACT_CHECK(ws_bytes >= pact_lora_bwd_workspace_bytes(M, N, K, r, nseg), PACT_ERR_INVALID_ARG,
               "pact_lora_bwd: workspace too small");
    PACT_CHECK(g->lddy >= N && g->lddy % 8 == 0 && g->ldu >= 2 * R && g->ldu % 8 == 0 && aligned16(g->dy) &&
                   aligned16(g->A) && aligned16(g->U) && aligned16(g->dA) && aligned16(g->dB) &&
                   ((uintptr_t)workspace & 255) == 0 && (!g->x || (g->ldx >= K && g->ldx % 8 == 0 && aligned16(g->x))),
               PACT_ERR_ALIGN, "pact_lora_bwd: pointers 16-byte aligned (workspace 256), leading dims %% 8 == 0");
    if (g->xq) {
        s = check_nvfp4(g->xq, M, K, "xq");
        if (s != PACT_OK) return s;
    }
    cudaStream_t st = (cudaStream_t)stream;
    uint8_t *w8 = static_cast<uint8_t *>(workspace);
    float *ws_t = reinterpret_cast<float *>(w8);
    w8 += partial_bytes(M, R, splits_of(K, (M + BM - 1) / BM, T_PER_SM));
    pact_bf16 *tt = reinterpret_cast<pact_bf16 *>(w8);
    w8 += round256((size_t)(M * 2 * R * 2));
    float *ws_db = reinterpret_cast<float *>(w8);
    w8 += partial_bytes(N, r, splits_of(M, (N + BM - 1) / BM, ctas_per_sm(2, false, stages_for(2, false))));
    float *ws_da = reinterpret_cast<float *>(w8);

    // X~ is read where it lies: BF16 rows, or the saved NVFP4 copy decoded in shared
    // memory by the MMA kernel (no BF16 copy of it is written)
    // T~ = X~ . A^T (unscaled), hi/lo
    CUtensorMap tx;
    s = g->xq ? map_codes(&tx, *g->xq, BK / 2, BM, "pact_lora_bwd")
              : map_bf16(&tx, g->x, K, M, g->ldx, 64, BM, "pact_lora_bwd");
    if (s == PACT_OK) s = rows_times_a(tx, g->xq, M, K, g->A, R, 1.0f, tt, 2 * R, ws_t, st, "pact_lora_bwd");
    if (s != PACT_OK) return s;
    // dB_i = scale * dY_i^T . T~_i: output rows are the outputs n of segment i,
    // contraction over the tokens
    Params pb = {};
    {
        CUtensorMap ta, tb;
        s = map_bf16(&ta, g->dy, N, M, g->lddy, 64, 64, "pact_lora_bwd");                // dY^T, MN-major
        if (s == PACT_OK) s = map_bf16(&tb, tt, 2 * R, M, 2 * R, 64, 64, "pact_lora_bwd");  // T~^T, MN-major
        if (s != PACT_OK) return s;
        pb.n_mma = 64;
        pb.n_valid = r;
        pb.nprob = nseg;
        int64_t widest = 0, blocks = 0, prev = 0;
        for (int i = 0; i < nseg; ++i) {
            pb.prob[i] = Prob{(int)prev, (int)g->seg_end[i], 0, (int)M, i * r, 0};
            const int64_t w = g->seg_end[i] - prev;
            if (w > widest) widest = w;
            blocks += (w + BM - 1) / BM;
            prev = g->seg_end[i];
        }
        pb.b_split = 1;
        pb.b_lo_off = R;
        choose_split(M, blocks, ctas_per_sm(2, false, stages_for(2, false)), &pb.splits, &pb.k_per_split);
        pb.ws = ws_db;
        pb.ws_ld = r;
        pb.ws_split_stride = N * r;
        s = launch_mma<true, true>(ta, tb, pb, (int)((widest + BM - 1) / BM), st, "pact_lora_bwd");
        if (s != PACT_OK) return s;
    }
    // dA^T = X~^T . U  [K x R], U = hi + lo
    CUtensorMap ta, tb;
    s = g->xq ? map_codes(&ta, *g->xq, BM / 2, BK, "pact_lora_bwd")
              : map_bf16(&ta, g->x, K, M, g->ldx, 64, 64, "pact_lora_bwd");             // X~^T, MN-major
    if (s == PACT_OK) s = map_bf16(&tb, g->U, 2 * R, M, g->ldu, 64, 64, "pact_lora_bwd");  // U^T, MN-major
    if (s != PACT_OK) return s;
    Params p = {};
    p.n_mma = 64;
    p.n_valid = R;
    p.nprob = 1;
    p.prob[0] = Prob{0, (int)K, 0, (int)M, 0, 0};
    p.b_split = 1;
    p.b_lo_off = R;
    const int tiles = (int)((K + BM - 1) / BM);
    choose_split(M, tiles, ctas_per_sm(2, g->xq != nullptr, stages_for(2, g->xq != nullptr)), &p.splits, &p.k_per_split);
    p.ws = ws_da;
    p.ws_ld = R;
    p.ws_split_stride = K * R;
    if (g->xq) {
        set_fp4_a(p, *g->xq);
        s = launch_mma<true, true, true>(ta, tb, p, tiles, st, "pact_lora_bwd");
    } else {
        s = launch_mma<true, true>(ta, tb, p, tiles, st, "pact_lora_bwd");
    }
    if (s != PACT_OK) return s;
    // one pass finalizes both gradients (BF16, or FP32 for a later reduction)
    const int f32 = g->grads_fp32 ? 2 : 0;
    const FinJob jb = fin_job(ws_db, pb, N, r, g->scale, 1 + f32, g->dB, r, 0);
    const FinJob ja = fin_job(ws_da, p, K, R, std::ldexp(1.0f, g->u_gexp), 2 + f32, g->dA, K, 0);
    return finalize(jb, &ja, st, "pact_lora_bwd");
}

}  // extern "C"

// ----------------------------------------------------------------------------
// Allocation-free LoRA forward.
//
// Some callers cannot hand this library a workspace: plain C programs that have no
// device allocator of their own, and code that must not call cudaMalloc at the
// point of use (cudaMalloc may synchronise the device, and services that fix
// their device-memory budget at start-up forbid allocation afterwards).  For them,
// pact_lora_fwd_noalloc runs the same kernels as pact_lora_fwd with its scratch
// (the FP32 partial sums) in a fixed array that lives in this library's device
// code.  Every GPU that loads the library holds the array until the process
// exits.  All calls on a device share it and it keeps the last call's contents
// (each call overwrites every partial it reads, so nothing needs clearing), so two
// calls that overlap on the GPU (different streams) race on it.
// ----------------------------------------------------------------------------
namespace pact {
namespace lmma {

constexpr size_t NOALLOC_SCRATCH_BYTES = 8u << 20;  // 8 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch for the current device.  The symbol's host
// name is only a stand-in, so the address is looked up once per device (with that
// device current) and kept; a mutex makes concurrent first calls from several host
// threads safe, and a failed lookup is retried on the next call.
static pact_status noalloc_scratch(void **out) {
    static std::mutex lock;
    static void *addr[64] = {nullptr};
    const int d = current_device();
    if (d < 0 || d >= 64) return fail(PACT_ERR_UNSUPPORTED, "pact_lora_fwd_noalloc: device index %d unsupported", d);
    std::lock_guard<std::mutex> guard(lock);
    if (!addr[d]) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p)
            return fail(PACT_ERR_CUDA, "pact_lora_fwd_noalloc: cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
        addr[d] = p;
    }
    *out = addr[d];
    return PACT_OK;
}

}  // namespace lmma
}  // namespace pact

extern "C" pact_status pact_lora_fwd_noalloc(const pact_bf16 *x, int64_t ldx, int64_t M, int64_t K,
                                             const pact_bf16 *A, int R, float scale, pact_bf16 *T, int64_t ldt,
                                             pact_stream_t stream) {
    PACT_CHECK(x && A && T, PACT_ERR_INVALID_ARG, "pact_lora_fwd_noalloc: NULL argument");
    PACT_CHECK(M >= 1 && M <= 0x7FFFFFFF && K >= 64 && K % 64 == 0 && K <= 0x7FFFFFFF && R >= 16 && R <= 64 &&
                   R % 16 == 0,
               PACT_ERR_SHAPE, "pact_lora_fwd_noalloc: need M >= 1, K a multiple of 64, R in {16, 32, 48, 64}");
    PACT_CHECK(ldx >= K && ldx % 8 == 0 && ldt >= 2 * R && ldt % 8 == 0 && aligned16(x) && aligned16(A) && aligned16(T),
               PACT_ERR_ALIGN, "pact_lora_fwd_noalloc: pointers 16-byte aligned, leading dims %% 8 == 0");
    const size_t need = pact_lora_fwd_workspace_bytes(M, K, R);
    PACT_CHECK(need <= NOALLOC_SCRATCH_BYTES, PACT_ERR_SHAPE,
               "pact_lora_fwd_noalloc: this shape needs %zu bytes of scratch, more than the built-in %zu bytes; "
               "use pact_lora_fwd with a workspace",
               need, (size_t)NOALLOC_SCRATCH_BYTES);
    void *scratch = nullptr;
    pact_status s = noalloc_scratch(&scratch);
    if (s != PACT_OK) return s;
    CUtensorMap tx;
    s = map_bf16(&tx, x, K, M, ldx, 64, BM, "pact_lora_fwd_noalloc");
    if (s != PACT_OK) return s;
    return rows_times_a(tx, nullptr, M, K, A, R, scale, T, ldt, static_cast<float *>(scratch), (cudaStream_t)stream,
                        "pact_lora_fwd_noalloc");
}
