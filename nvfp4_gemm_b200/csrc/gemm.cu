// gemm.cu -- the frozen-projection NVFP4 GEMM of PACT on 5th-generation tensor cores.
//
// [METHOD] (PACT blog summary, section "方法", bullet 1): the forward and the input
// gradient of the 7 frozen projections are NVFP4 GEMMs with FP32 accumulation and
// BF16 output.  [LORA] (PEFT explainer, section "LoRA"): h = W0 x + B A x; the BF16
// low-rank term is accumulated into the same FP32 accumulator.
//
// One kernel serves both directions: D[M x N] = deq(A)[M x K] . deq(B)[N x K]^T with
// A, B NVFP4 and K-major (forward: A = q(x), B = W_fwd; dgrad: A = q(dY), B = W_bwd).
//
// Design (sm_100a):
//  * persistent CTAs, one per SM, 128 x 256 output tiles, static round-robin schedule;
//  * warp 0 issues TMA (operand tiles, 128-byte swizzle) and bulk copies (scale
//    tiles, already in the 512-byte layout the tensor core reads) into a 4-stage
//    shared-memory ring guarded by mbarriers;
//  * warp 1 moves each stage's scales shared -> tensor memory (tcgen05.cp) and issues
//    tcgen05.mma kind::mxf4nvf4 (E2M1 x E2M1, UE4M3 scale per 16) into a 128 x 256
//    FP32 accumulator in tensor memory; the LoRA term is one or more kind::f16 MMAs
//    into the same accumulator before the NVFP4 K loop;
//  * warps 2-5 drain the accumulator (tcgen05.ld), round to BF16 and store.
#include "common.cuh"

namespace pact {
namespace gemm {

constexpr int BM = 128;             // rows per tile (MMA M)
constexpr int BN = 256;             // columns per tile (MMA N)
constexpr int BK = 256;             // FP4 elements per stage = 128 bytes per row
constexpr int KSTEP = 64;           // FP4 elements per MMA
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK / 2;        // 16384
constexpr int B_BYTES = BN * BK / 2;        // 32768
constexpr int SFA_BYTES = BM * BK / 16;     // 2048: 4 chunks of 512
constexpr int SFB_BYTES = BN * BK / 16;     // 4096: 2 row groups x 4 chunks
constexpr int OFF_B = A_BYTES;
constexpr int OFF_SFA = OFF_B + B_BYTES;
constexpr int OFF_SFB = OFF_SFA + SFA_BYTES;
constexpr int STAGE_BYTES = OFF_SFB + SFB_BYTES;  // 55296, a multiple of 1024
// A LoRA stage holds up to 6 activation chunks (4 KB) and then the weight tile.
constexpr int OFF_LW = 6 * BM * 32;               // 24576
static_assert(OFF_LW + 3 * BN * 32 <= STAGE_BYTES && OFF_LW + 4 * 48 * 128 <= STAGE_BYTES, "LoRA stage");
constexpr int BAR_BYTES = 256;
constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + BAR_BYTES;
constexpr int THREADS = 192;

// tensor memory columns
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t COL_ACC = 0;     // 256 FP32 columns
constexpr uint32_t COL_SFA = 256;   // 4 columns per MMA x 4 MMAs
constexpr uint32_t COL_SFB = 272;   // 8 columns per MMA x 4 MMAs

enum LoraMode : int { LORA_NONE = 0, LORA_FWD = 1, LORA_DGRAD = 2 };

struct Params {
    int M, N, K;
    const uint8_t *sfa;   // scales of A (rows M, cols K)
    const uint8_t *sfb;   // scales of B (rows N, cols K)
    __nv_bfloat16 *out;
    int64_t ldo;
    const __nv_bfloat16 *res;   // optional residual added in the epilogue (may alias out)
    int64_t ldr;
    int lora_mode;
    int lora_steps;       // weight chunks of K = 16 per tile (two MMAs each: hi and lo activations)
    int lora_r;
    int lora_nseg;
    int64_t seg_end[4];
};

struct Tile {
    int mt, nt;
};

__device__ __forceinline__ Tile tile_of(int t, int mtiles) { return Tile{t % mtiles, t / mtiles}; }

__device__ __forceinline__ int lora_segment(const Params &p, int n0) {
    int s = 0;
    for (int i = 0; i + 1 < p.lora_nseg; ++i) s += (n0 >= p.seg_end[i]) ? 1 : 0;
    return s;
}

__global__ void __launch_bounds__(THREADS, 1)
k_nvfp4_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
             const __grid_constant__ CUtensorMap tmLa, const __grid_constant__ CUtensorMap tmLb, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + (((raw + 1023) & ~1023u) - raw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE_BYTES);
    uint64_t *full = bars;                     // [STAGES]
    uint64_t *empty = bars + STAGES;           // [STAGES]
    uint64_t *acc_full = bars + 2 * STAGES;    // MMA -> epilogue
    uint64_t *acc_empty = bars + 2 * STAGES + 1;  // epilogue -> MMA
    uint64_t *drained = bars + 2 * STAGES + 2;    // MMA warp: all its tcgen05 work done
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * STAGES + 3);
    volatile uint32_t *abort_flag = tmem_slot + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int mtiles = (p.M + BM - 1) / BM, ntiles = (p.N + BN - 1) / BN;
    const int ntile_total = mtiles * ntiles;
    const int ktiles = (p.K + BK - 1) / BK;
    const int kgroups = p.K / 64;  // scale chunks per 128-row group

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 4);
        mbar_init(drained, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
        if (p.lora_mode != LORA_NONE) {
            prefetch_tensormap(&tmLa);
            prefetch_tensormap(&tmLb);
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            uint32_t stage = 0, phase = 0;
            uint32_t pending = 0;          // stages with a load issued
            uint32_t pending_parity = 0;   // full-barrier parity of each stage's last load
            for (int t = blockIdx.x; t < ntile_total && !*abort_flag; t += gridDim.x) {
                const Tile tl = tile_of(t, mtiles);
                const int m0 = tl.mt * BM, n0 = tl.nt * BN;
                if (p.lora_mode != LORA_NONE) {
                    if (!mbar_wait(&empty[stage], phase ^ 1)) { *abort_flag = 1; break; }
                    uint8_t *st = smem + stage * STAGE_BYTES;
                    // LoRA stage: 2 * steps activation chunks (hi parts, then lo parts; 128
                    // rows x 16 BF16 each) and the weight chunks at OFF_LW.
                    const int R = p.lora_nseg * p.lora_r;
                    if (p.lora_mode == LORA_FWD) {
                        const int xs = lora_segment(p, n0) * p.lora_r;
                        mbar_arrive_expect_tx(&full[stage], p.lora_steps * (2 * BM * 32 + BN * 32));
                        for (int c = 0; c < p.lora_steps; ++c) {
                            tma_load_2d(st + c * BM * 32, &tmLa, &full[stage], xs + 16 * c, m0);
                            tma_load_2d(st + (p.lora_steps + c) * BM * 32, &tmLa, &full[stage], R + xs + 16 * c, m0);
                            tma_load_2d(st + OFF_LW + c * BN * 32, &tmLb, &full[stage], 16 * c, n0);
                        }
                    } else {
                        mbar_arrive_expect_tx(&full[stage], p.lora_steps * 2 * BM * 32 + 4 * R * 128);
                        for (int c = 0; c < p.lora_steps; ++c) {
                            tma_load_2d(st + c * BM * 32, &tmLa, &full[stage], 16 * c, m0);
                            tma_load_2d(st + (p.lora_steps + c) * BM * 32, &tmLa, &full[stage], R + 16 * c, m0);
                        }
                        for (int q = 0; q < 4; ++q)
                            tma_load_2d(st + OFF_LW + q * R * 128, &tmLb, &full[stage], n0 + 64 * q, 0);
                    }
                    pending |= 1u << stage;
                    pending_parity = (pending_parity & ~(1u << stage)) | (phase << stage);
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
                const int g0 = n0 / 128;                           // first 128-row group of B
                const int ngroups = (p.N - n0) > 128 ? 2 : 1;      // groups of B inside the padded rows
                for (int kt = 0; kt < ktiles; ++kt) {
                    if (!mbar_wait(&empty[stage], phase ^ 1)) { *abort_flag = 1; break; }
                    uint8_t *st = smem + stage * STAGE_BYTES;
                    const int nk = min(BK / KSTEP, (p.K - kt * BK) / KSTEP);
                    mbar_arrive_expect_tx(&full[stage], A_BYTES + B_BYTES + nk * 512 * (1 + ngroups));
                    tma_load_2d(st, &tmA, &full[stage], kt * (BK / 2), m0);
                    tma_load_2d(st + OFF_B, &tmB, &full[stage], kt * (BK / 2), n0);
                    bulk_load(st + OFF_SFA, p.sfa + ((size_t)tl.mt * kgroups + kt * 4) * 512, nk * 512, &full[stage]);
                    for (int g = 0; g < ngroups; ++g)
                        bulk_load(st + OFF_SFB + g * 2048, p.sfb + ((size_t)(g0 + g) * kgroups + kt * 4) * 512,
                                  nk * 512, &full[stage]);
                    pending |= 1u << stage;
                    pending_parity = (pending_parity & ~(1u << stage)) | (phase << stage);
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
            }
            // Every issued copy must land before the CTA may leave (its shared memory is
            // the destination).  In a normal run they all have; after an abort, wait for
            // them (bounded).
            for (int s = 0; s < STAGES; ++s)
                if (pending & (1u << s)) mbar_wait(&full[s], (pending_parity >> s) & 1u);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        const uint32_t idesc = idesc_nvf4(BM, BN);
        const uint32_t idesc_lora = idesc_bf16(BM, BN, false, p.lora_mode == LORA_DGRAD);
        uint32_t stage = 0, phase = 0, acc_phase = 0;
        for (int t = blockIdx.x; t < ntile_total; t += gridDim.x) {
            bool ok = mbar_wait(acc_empty, acc_phase ^ 1);
            tc_fence_after();
            uint32_t accum = 0;
            if (ok && p.lora_mode != LORA_NONE) {
                ok = mbar_wait(&full[stage], phase);
                tc_fence_after();
                if (ok && lane == 0) {
                    const uint32_t st = smem_u32(smem + stage * STAGE_BYTES);
                    const int R = p.lora_nseg * p.lora_r;
                    for (int c = 0; c < p.lora_steps; ++c) {
                        const uint64_t bd = (p.lora_mode == LORA_FWD)
                                                ? smem_desc(st + OFF_LW + c * BN * 32, 16, 256, SW_32)
                                                : smem_desc(st + OFF_LW + c * 2048, R * 128, 1024, SW_128);
                        for (int h = 0; h < 2; ++h) {  // hi part, then lo part
                            const uint64_t ad = smem_desc(st + (h * p.lora_steps + c) * BM * 32, 16, 256, SW_32);
                            mma_bf16(tmem + COL_ACC, ad, bd, idesc_lora, accum);
                            accum = 1;
                        }
                    }
                    tc_commit(&empty[stage]);
                }
                accum = 1;
                __syncwarp();
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
            }
            for (int kt = 0; ok && kt < ktiles; ++kt) {
                ok = mbar_wait(&full[stage], phase);
                tc_fence_after();
                if (ok && lane == 0) {
                    const int nk = min(BK / KSTEP, (p.K - kt * BK) / KSTEP);
                    const int n0 = (t / mtiles) * BN;
                    const int ngroups = (p.N - n0) > 128 ? 2 : 1;
                    const uint32_t st = smem_u32(smem + stage * STAGE_BYTES);
                    for (int s = 0; s < nk; ++s) {
                        tmem_cp_32x128b_x4(tmem + COL_SFA + 4 * s, smem_desc(st + OFF_SFA + s * 512, 0, 128, SW_NONE));
                        for (int g = 0; g < ngroups; ++g)
                            tmem_cp_32x128b_x4(tmem + COL_SFB + 8 * s + 4 * g,
                                               smem_desc(st + OFF_SFB + g * 2048 + s * 512, 0, 128, SW_NONE));
                    }
                    for (int s = 0; s < nk; ++s) {
                        const uint64_t ad = smem_desc(st + s * 32, 16, 1024, SW_128);
                        const uint64_t bd = smem_desc(st + OFF_B + s * 32, 16, 1024, SW_128);
                        mma_nvf4(tmem + COL_ACC, ad, bd, idesc, tmem + COL_SFA + 4 * s, tmem + COL_SFB + 8 * s, accum);
                        accum = 1;
                    }
                    tc_commit(&empty[stage]);
                }
                accum = 1;
                __syncwarp();
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
            }
            if (!ok) { *abort_flag = 1; break; }
            if (lane == 0) tc_commit(acc_full);
            __syncwarp();
            acc_phase ^= 1;
        }
        // tensor memory is released below only after every MMA and copy issued here
        // has completed
        if (lane == 0) tc_commit(drained);
        mbar_wait(drained, 0);
    } else {
        // ------------------------------------------------------------ epilogue
        const int sub = warp & 3;  // tensor-memory sub-partition this warp may read
        uint32_t acc_phase = 0;
        for (int t = blockIdx.x; t < ntile_total; t += gridDim.x) {
            const Tile tl = tile_of(t, mtiles);
            if (!mbar_wait(acc_full, acc_phase)) { *abort_flag = 1; break; }
            tc_fence_after();
            const int row = tl.mt * BM + sub * 32 + lane;
            for (int c = 0; c < BN / 32; ++c) {
                const int n = tl.nt * BN + c * 32;
                if (n >= p.N) break;
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem + ((uint32_t)(sub * 32) << 16) + COL_ACC + c * 32, r);
                tmem_ld_wait();
                if (row < p.M) {
                    __nv_bfloat16 *dst = p.out + (size_t)row * p.ldo + n;
                    uint4 *d4 = reinterpret_cast<uint4 *>(dst);
                    const uint4 *r4 = p.res ? reinterpret_cast<const uint4 *>(p.res + (size_t)row * p.ldr + n) : nullptr;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        float f[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) f[i] = __uint_as_float(r[8 * q + i]);
                        if (r4) {
                            const uint4 old = r4[q];
                            f[0] += bf16lo(old.x); f[1] += bf16hi(old.x); f[2] += bf16lo(old.y); f[3] += bf16hi(old.y);
                            f[4] += bf16lo(old.z); f[5] += bf16hi(old.z); f[6] += bf16lo(old.w); f[7] += bf16hi(old.w);
                        }
                        uint4 v;
                        v.x = pack_bf16x2(f[0], f[1]); v.y = pack_bf16x2(f[2], f[3]);
                        v.z = pack_bf16x2(f[4], f[5]); v.w = pack_bf16x2(f[6], f[7]);
                        d4[q] = v;
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acc_empty);
            acc_phase ^= 1;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}


// ---------------------------------------------------------------------------------
// CTA-pair variant: a cluster of 2 CTAs computes a 256 x 256 tile with 2-SM MMAs
// (tcgen05 cta_group::2).  CTA r of the pair holds rows 128r..128r+127 of A and of
// the accumulator, and rows 128r..128r+127 of the B tile; the MMA reads both halves
// of A and B across the pair, so each SM streams half as much B per unit of work
// as the single-CTA kernel.  Every scale tile arrives by TMA; the leader (rank 0)
// arms its full barrier for both CTAs' bytes, the peer's loads complete on it, and
// the leader issues the scale copies and MMAs for the pair and multicasts its
// commits to both CTAs' barriers.
// ---------------------------------------------------------------------------------
namespace pair {

constexpr int BM = 128;               // rows per CTA; the pair tile has 256
constexpr int BN = 256;               // columns of the pair tile; each CTA loads 128 rows of B
constexpr int BK = 256;
constexpr int KSTEP = 64;
constexpr int STAGES = 5;
constexpr int A_BYTES = BM * BK / 2;          // 16384
constexpr int B_BYTES = (BN / 2) * BK / 2;    // 16384
constexpr int OFF_B = A_BYTES;
constexpr int OFF_SFA = OFF_B + B_BYTES;      // 4 chunks of 512 (this CTA's rows)
constexpr int OFF_SFB = OFF_SFA + 2048;       // 2 row groups x 4 chunks (all 256 columns)
constexpr int STAGE_BYTES = OFF_SFB + 4096;   // 38912 = 38 KiB
constexpr int LOAD_BYTES = STAGE_BYTES;       // bytes one CTA's loads deliver per k stage
constexpr int OFF_LW = 6 * BM * 32;           // LoRA weight chunks follow 6 activation chunks
constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + 256;
constexpr int THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t COL_ACC = 0, COL_SFA = 256, COL_SFB = 272;
static_assert(OFF_LW + 3 * BM * 32 <= STAGE_BYTES && OFF_LW + 2 * 48 * 128 <= STAGE_BYTES, "LoRA stage");

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
k_nvfp4_gemm_pair(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                  const __grid_constant__ CUtensorMap tmSFA, const __grid_constant__ CUtensorMap tmSFB,
                  const __grid_constant__ CUtensorMap tmLa, const __grid_constant__ CUtensorMap tmLb,
                  const Params p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + (((raw + 1023) & ~1023u) - raw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE_BYTES);
    uint64_t *full = bars;                       // [STAGES], used in the leader
    uint64_t *empty = bars + STAGES;             // [STAGES]
    uint64_t *acc_full = bars + 2 * STAGES;      // leader MMA -> both epilogues
    uint64_t *acc_empty = bars + 2 * STAGES + 1; // both epilogues -> leader MMA
    uint64_t *drained = bars + 2 * STAGES + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * STAGES + 3);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int mpairs = (p.M + 2 * BM - 1) / (2 * BM), ntiles = (p.N + BN - 1) / BN;
    const int total = mpairs * ntiles;
    const int cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;
    const int ktiles = (p.K + BK - 1) / BK;
    const int kgroups = p.K / 64;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 8);
        mbar_init(drained, 1);
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
        prefetch_tensormap(&tmSFA);
        prefetch_tensormap(&tmSFB);
        if (p.lora_mode != LORA_NONE) {
            prefetch_tensormap(&tmLa);
            prefetch_tensormap(&tmLb);
        }
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // the peer's barriers exist before anything addresses them
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t full_leader = mapa_shared(smem_u32(full), 0);
    const uint32_t acc_empty_leader = mapa_shared(smem_u32(acc_empty), 0);

    if (warp == 0) {
        // ------------------------------------------------------------ producer (both CTAs)
        if (lane == 0) {
            uint32_t stage = 0, phase = 0;
            bool ok = true;
            for (int t = cluster; ok && t < total; t += nclusters) {
                const int mp = t % mpairs, nt = t / mpairs;
                const int m0 = mp * 2 * BM + (int)rank * BM;     // this CTA's rows
                const int n0 = nt * BN, nb = n0 + (int)rank * (BN / 2);
                if (p.lora_mode != LORA_NONE) {
                    if (!(ok = mbar_wait(&empty[stage], phase ^ 1))) break;
                    const uint32_t st = smem_u32(smem + stage * STAGE_BYTES);
                    const uint32_t fb = full_leader + 8 * stage;
                    const int R = p.lora_nseg * p.lora_r;
                    if (p.lora_mode == LORA_FWD) {
                        if (leader) mbar_arrive_expect_tx(&full[stage], 2 * p.lora_steps * (2 * BM * 32 + BM * 32));
                        const int xs = lora_segment(p, n0) * p.lora_r;
                        for (int c = 0; c < p.lora_steps; ++c) {
                            tma_load_2d_pair(st + c * BM * 32, &tmLa, fb, xs + 16 * c, m0);
                            tma_load_2d_pair(st + (p.lora_steps + c) * BM * 32, &tmLa, fb, R + xs + 16 * c, m0);
                            tma_load_2d_pair(st + OFF_LW + c * BM * 32, &tmLb, fb, 16 * c, nb);
                        }
                    } else {
                        if (leader) mbar_arrive_expect_tx(&full[stage], 2 * (p.lora_steps * 2 * BM * 32 + 2 * R * 128));
                        for (int c = 0; c < p.lora_steps; ++c) {
                            tma_load_2d_pair(st + c * BM * 32, &tmLa, fb, 16 * c, m0);
                            tma_load_2d_pair(st + (p.lora_steps + c) * BM * 32, &tmLa, fb, R + 16 * c, m0);
                        }
                        for (int q = 0; q < 2; ++q) tma_load_2d_pair(st + OFF_LW + q * R * 128, &tmLb, fb, nb + 64 * q, 0);
                    }
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
                const int ga = m0 / 128, gb = n0 / 128;
                for (int kt = 0; kt < ktiles; ++kt) {
                    if (!(ok = mbar_wait(&empty[stage], phase ^ 1))) break;
                    const uint32_t st = smem_u32(smem + stage * STAGE_BYTES);
                    const uint32_t fb = full_leader + 8 * stage;
                    if (leader) mbar_arrive_expect_tx(&full[stage], 2 * LOAD_BYTES);
                    tma_load_2d_pair(st, &tmA, fb, kt * (BK / 2), m0);
                    tma_load_2d_pair(st + OFF_B, &tmB, fb, kt * (BK / 2), nb);
                    // scale chunks: 512 bytes = two 256-byte rows of the scale map
                    tma_load_2d_pair(st + OFF_SFA, &tmSFA, fb, 0, 2 * (ga * kgroups + kt * 4));
                    tma_load_2d_pair(st + OFF_SFB, &tmSFB, fb, 0, 2 * (gb * kgroups + kt * 4));
                    tma_load_2d_pair(st + OFF_SFB + 2048, &tmSFB, fb, 0, 2 * ((gb + 1) * kgroups + kt * 4));
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (leader)
        if (leader) {
            const uint32_t idesc = idesc_nvf4(2 * BM, BN);
            const uint32_t idesc_lora = idesc_bf16(2 * BM, BN, false, p.lora_mode == LORA_DGRAD);
            uint32_t stage = 0, phase = 0, acc_phase = 0;
            for (int t = cluster; t < total; t += nclusters) {
                bool ok = mbar_wait(acc_empty, acc_phase ^ 1);
                tc_fence_after();
                uint32_t accum = 0;
                if (ok && p.lora_mode != LORA_NONE) {
                    ok = mbar_wait(&full[stage], phase);
                    tc_fence_after();
                    if (ok && lane == 0) {
                        const uint32_t st = smem_u32(smem + stage * STAGE_BYTES);
                        const int R = p.lora_nseg * p.lora_r;
                        for (int c = 0; c < p.lora_steps; ++c) {
                            const uint64_t bd = (p.lora_mode == LORA_FWD)
                                                    ? smem_desc(st + OFF_LW + c * BM * 32, 16, 256, SW_32)
                                                    : smem_desc(st + OFF_LW + c * 2048, R * 128, 1024, SW_128);
                            for (int h = 0; h < 2; ++h) {
                                const uint64_t ad = smem_desc(st + (h * p.lora_steps + c) * BM * 32, 16, 256, SW_32);
                                mma_bf16_pair(tmem + COL_ACC, ad, bd, idesc_lora, accum);
                                accum = 1;
                            }
                        }
                        tc_commit_pair(&empty[stage], 3);
                    }
                    accum = 1;
                    __syncwarp();
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
                for (int kt = 0; ok && kt < ktiles; ++kt) {
                    ok = mbar_wait(&full[stage], phase);
                    tc_fence_after();
                    if (ok && lane == 0) {
                        const int nk = min(BK / KSTEP, (p.K - kt * BK) / KSTEP);
                        const uint32_t st = smem_u32(smem + stage * STAGE_BYTES);
                        for (int s = 0; s < nk; ++s) {
                            tmem_cp_pair_32x128b_x4(tmem + COL_SFA + 4 * s,
                                                    smem_desc(st + OFF_SFA + s * 512, 0, 128, SW_NONE));
                            for (int g = 0; g < 2; ++g)
                                tmem_cp_pair_32x128b_x4(tmem + COL_SFB + 8 * s + 4 * g,
                                                        smem_desc(st + OFF_SFB + g * 2048 + s * 512, 0, 128, SW_NONE));
                        }
                        for (int s = 0; s < nk; ++s) {
                            const uint64_t ad = smem_desc(st + s * 32, 16, 1024, SW_128);
                            const uint64_t bd = smem_desc(st + OFF_B + s * 32, 16, 1024, SW_128);
                            mma_nvf4_pair(tmem + COL_ACC, ad, bd, idesc, tmem + COL_SFA + 4 * s, tmem + COL_SFB + 8 * s,
                                          accum);
                            accum = 1;
                        }
                        tc_commit_pair(&empty[stage], 3);
                    }
                    accum = 1;
                    __syncwarp();
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                if (lane == 0) tc_commit_pair(acc_full, 3);
                __syncwarp();
                acc_phase ^= 1;
            }
            if (lane == 0) tc_commit_pair(drained, 1);
            mbar_wait(drained, 0);
        }
    } else {
        // ------------------------------------------------------------ epilogue (both CTAs)
        const int sub = warp & 3;
        uint32_t acc_phase = 0;
        for (int t = cluster; t < total; t += nclusters) {
            const int mp = t % mpairs, nt = t / mpairs;
            if (!mbar_wait(acc_full, acc_phase)) break;
            tc_fence_after();
            const int row = mp * 2 * BM + (int)rank * BM + sub * 32 + lane;
            for (int c = 0; c < BN / 32; ++c) {
                const int n = nt * BN + c * 32;
                if (n >= p.N) break;
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem + ((uint32_t)(sub * 32) << 16) + COL_ACC + c * 32, r);
                tmem_ld_wait();
                if (row < p.M) {
                    uint4 *d4 = reinterpret_cast<uint4 *>(p.out + (size_t)row * p.ldo + n);
                    const uint4 *r4 = p.res ? reinterpret_cast<const uint4 *>(p.res + (size_t)row * p.ldr + n) : nullptr;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        float f[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) f[i] = __uint_as_float(r[8 * q + i]);
                        if (r4) {
                            const uint4 old = r4[q];
                            f[0] += bf16lo(old.x); f[1] += bf16hi(old.x); f[2] += bf16lo(old.y); f[3] += bf16hi(old.y);
                            f[4] += bf16lo(old.z); f[5] += bf16hi(old.z); f[6] += bf16lo(old.w); f[7] += bf16hi(old.w);
                        }
                        uint4 v;
                        v.x = pack_bf16x2(f[0], f[1]); v.y = pack_bf16x2(f[2], f[3]);
                        v.z = pack_bf16x2(f[4], f[5]); v.w = pack_bf16x2(f[6], f[7]);
                        d4[q] = v;
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(acc_empty_leader);
            acc_phase ^= 1;
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();  // every MMA of the pair has completed and both epilogues are done
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, TMEM_COLS);
    }
    cluster_sync();
}

}  // namespace pair

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiled)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiled encode_fn() {
    static EncodeTiled fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiled>(p);
    }
    return fn;
}

// 2-D tiled map over a row-major matrix: `inner` elements per row, `outer` rows,
// rows `row_bytes` apart.
static pact_status make_map(CUtensorMap *m, CUtensorMapDataType dt, const void *base, uint64_t inner, uint64_t outer,
                            uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw,
                            const char *what) {
    EncodeTiled enc = encode_fn();
    if (!enc) return fail(PACT_ERR_CUDA, "%s: cuTensorMapEncodeTiled unavailable", what);
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PACT_ERR_CUDA, "%s: cuTensorMapEncodeTiled failed (%d)", what, (int)r);
    return PACT_OK;
}

static pact_status ensure_attrs() {
    static bool done[64] = {false};
    const int d = current_device();
    if (d >= 0 && d < 64 && done[d]) return PACT_OK;
    cudaError_t e =
        cudaFuncSetAttribute(pair::k_nvfp4_gemm_pair, cudaFuncAttributeMaxDynamicSharedMemorySize, pair::SMEM_BYTES);
    if (e != cudaSuccess) return fail(PACT_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    if (d >= 0 && d < 64) done[d] = true;
    return PACT_OK;
}

static pact_status check_lora(const pact_lora_t *l, int64_t M, int64_t N, int64_t Kout, bool dgrad, const char *what) {
    PACT_CHECK(l->act && l->weight, PACT_ERR_INVALID_ARG, "%s: LoRA act/weight NULL", what);
    PACT_CHECK(l->r == 16 || l->r == 32 || l->r == 48, PACT_ERR_SHAPE, "%s: LoRA r must be 16, 32 or 48", what);
    PACT_CHECK(l->nseg >= 1 && l->nseg <= 3 && l->nseg * l->r <= 48, PACT_ERR_SHAPE,
               "%s: LoRA needs 1 <= nseg <= 3 and nseg * r <= 48", what);
    const int R = l->nseg * l->r;
    if (!dgrad) {
        int64_t prev = 0;
        for (int i = 0; i < l->nseg; ++i) {
            const int64_t e = l->seg_end[i];
            PACT_CHECK(e > prev && (i + 1 == l->nseg ? e == N : e % 256 == 0), PACT_ERR_SHAPE,
                       "%s: LoRA segment ends must increase, be multiples of 256 and end at N", what);
            prev = e;
        }
        PACT_CHECK(l->ld_act >= 2 * R && l->ld_weight >= l->r, PACT_ERR_SHAPE,
                   "%s: LoRA leading dimensions too small", what);
    } else {
        PACT_CHECK(l->ld_act >= 2 * R && l->ld_weight >= Kout, PACT_ERR_SHAPE,
                   "%s: LoRA leading dimensions too small", what);
    }
    PACT_CHECK(aligned16(l->act) && aligned16(l->weight) && l->ld_act % 8 == 0 && l->ld_weight % 8 == 0,
               PACT_ERR_ALIGN, "%s: LoRA pointers must be 16-byte aligned with leading dims %% 8 == 0", what);
    (void)M;
    return PACT_OK;
}

// D[M x N] = deq(a) . deq(b)^T (+ LoRA); a [M x K], b [N x K].
static pact_status run(const pact_nvfp4_t *a, const pact_nvfp4_t *b, const pact_lora_t *lora, bool dgrad,
                       const pact_bf16 *res, int64_t ldr, pact_bf16 *out, int64_t ldo, cudaStream_t stream,
                       const char *what) {
    const int64_t M = a->rows, K = a->cols, N = b->rows;
    PACT_CHECK(M <= 0x7FFFFFFF && N <= 0x7FFFFFFF && K <= 0x7FFFFFFF, PACT_ERR_SHAPE, "%s: dimension too large", what);
    PACT_CHECK(out, PACT_ERR_INVALID_ARG, "%s: output NULL", what);
    PACT_CHECK(ldo >= N && ldo % 8 == 0 && aligned16(out), PACT_ERR_ALIGN,
               "%s: output must be 16-byte aligned with ld >= %lld and ld %% 8 == 0", what, (long long)N);
    PACT_CHECK(!res || (ldr >= N && ldr % 8 == 0 && aligned16(res)), PACT_ERR_ALIGN,
               "%s: residual must be 16-byte aligned with ld >= %lld and ld %% 8 == 0", what, (long long)N);
    pact_status s = lora ? check_lora(lora, M, N, N, dgrad, what) : PACT_OK;
    if (s != PACT_OK) return s;
    s = ensure_attrs();
    if (s != PACT_OK) return s;
    CUtensorMap tmA, tmB, tmSFA, tmSFB, tmLa, tmLb;
    // operand tiles: 128 rows x 128 bytes (256 FP4 values), 128-byte swizzle
    s = make_map(&tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, a->codes, K / 2, M, K / 2, 128, 128,
                 CU_TENSOR_MAP_SWIZZLE_128B, what);
    if (s == PACT_OK)
        s = make_map(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, b->codes, K / 2, N, K / 2, 128, 128,
                     CU_TENSOR_MAP_SWIZZLE_128B, what);
    // scale tiles: each 512-byte chunk (128 rows x 4 blocks) is two 256-byte rows of
    // a [2 * chunks x 256] byte matrix; one box is 4 chunks
    const uint64_t chunks_a = (uint64_t)((M + 127) / 128) * (K / 64), chunks_b = (uint64_t)((N + 127) / 128) * (K / 64);
    if (s == PACT_OK)
        s = make_map(&tmSFA, CU_TENSOR_MAP_DATA_TYPE_UINT8, a->scales, 256, 2 * chunks_a, 256, 256, 8,
                     CU_TENSOR_MAP_SWIZZLE_NONE, what);
    if (s == PACT_OK)
        s = make_map(&tmSFB, CU_TENSOR_MAP_DATA_TYPE_UINT8, b->scales, 256, 2 * chunks_b, 256, 256, 8,
                     CU_TENSOR_MAP_SWIZZLE_NONE, what);
    if (s != PACT_OK) return s;
    Params p;
    p.M = (int)M; p.N = (int)N; p.K = (int)K;
    p.sfa = static_cast<const uint8_t *>(a->scales);
    p.sfb = static_cast<const uint8_t *>(b->scales);
    p.out = reinterpret_cast<__nv_bfloat16 *>(out);
    p.ldo = ldo;
    p.res = reinterpret_cast<const __nv_bfloat16 *>(res);
    p.ldr = ldr;
    p.lora_mode = LORA_NONE;
    p.lora_steps = 0; p.lora_r = 0; p.lora_nseg = 1;
    for (int i = 0; i < 4; ++i) p.seg_end[i] = N;
    tmLa = tmA;
    tmLb = tmB;
    if (lora) {
        const int R = lora->nseg * lora->r;
        p.lora_r = lora->r;
        p.lora_nseg = lora->nseg;
        for (int i = 0; i < 4; ++i) p.seg_end[i] = i < lora->nseg ? lora->seg_end[i] : N;
        s = make_map(&tmLa, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, lora->act, 2 * R, M, lora->ld_act * 2, 16, 128,
                     CU_TENSOR_MAP_SWIZZLE_32B, what);
        if (s != PACT_OK) return s;
        if (!dgrad) {
            p.lora_mode = LORA_FWD;
            p.lora_steps = lora->r / 16;
            s = make_map(&tmLb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, lora->weight, lora->r, N, lora->ld_weight * 2, 16,
                         128, CU_TENSOR_MAP_SWIZZLE_32B, what);
        } else {
            p.lora_mode = LORA_DGRAD;
            p.lora_steps = R / 16;
            s = make_map(&tmLb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, lora->weight, N, R, lora->ld_weight * 2, 64, R,
                         CU_TENSOR_MAP_SWIZZLE_128B, what);
        }
        if (s != PACT_OK) return s;
    }
    const int pairs = (int)(((M + 255) / 256) * ((N + 255) / 256));
    const int clusters = pairs < sm_count() / 2 ? pairs : sm_count() / 2;
    pair::k_nvfp4_gemm_pair<<<2 * clusters, pair::THREADS, pair::SMEM_BYTES, stream>>>(tmA, tmB, tmSFA, tmSFB, tmLa,
                                                                                        tmLb, p);
    return launch_status(what);
}

}  // namespace gemm
}  // namespace pact

using namespace pact;

extern "C" {

pact_status pact_frozen_gemm_fwd(const pact_nvfp4_t *xq, const pact_weight_cache_t *w, const pact_lora_t *lora,
                                 const pact_bf16 *residual, int64_t ldr, pact_bf16 *y, int64_t ldy,
                                 pact_stream_t stream) {
    PACT_CHECK(xq && w, PACT_ERR_INVALID_ARG, "pact_frozen_gemm_fwd: NULL argument");
    const int64_t N = w->fwd.rows, K = w->fwd.cols;
    pact_status s = check_nvfp4(&w->fwd, N, K, "w->fwd");
    if (s == PACT_OK) s = check_nvfp4(xq, xq->rows, K, "xq");
    if (s != PACT_OK) return s;
    PACT_CHECK(xq->rows >= 1 && N % 64 == 0 && K % 64 == 0, PACT_ERR_SHAPE, "pact_frozen_gemm_fwd: bad shape");
    return gemm::run(xq, &w->fwd, lora, false, residual, ldr, y, ldy, (cudaStream_t)stream, "pact_frozen_gemm_fwd");
}

pact_status pact_frozen_gemm_dgrad(const pact_nvfp4_t *dyq, const pact_weight_cache_t *w, const pact_lora_t *lora,
                                   const pact_bf16 *residual, int64_t ldr, pact_bf16 *dx, int64_t lddx,
                                   pact_stream_t stream) {
    PACT_CHECK(dyq && w, PACT_ERR_INVALID_ARG, "pact_frozen_gemm_dgrad: NULL argument");
    const int64_t K = w->bwd.rows, N = w->bwd.cols;
    pact_status s = check_nvfp4(&w->bwd, K, N, "w->bwd");
    if (s == PACT_OK) s = check_nvfp4(dyq, dyq->rows, N, "dyq");
    if (s != PACT_OK) return s;
    PACT_CHECK(dyq->rows >= 1 && N % 64 == 0 && K % 64 == 0, PACT_ERR_SHAPE, "pact_frozen_gemm_dgrad: bad shape");
    return gemm::run(dyq, &w->bwd, lora, true, residual, ldr, dx, lddx, (cudaStream_t)stream,
                     "pact_frozen_gemm_dgrad");
}

}  // extern "C"
