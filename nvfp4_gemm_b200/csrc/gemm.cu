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
// Design (sm_100a), one cluster of 2 CTAs (a CTA pair on two SMs) per 256 x 256
// output tile, persistent over tiles:
//  * 2-SM MMAs (tcgen05 cta_group::2, kind::mxf4nvf4, scale_vec::4X, K = 64 per
//    instruction): CTA r of the pair holds rows 128r..128r+127 of A, of the B tile
//    and of the FP32 accumulator (128 lanes x 256 columns of its tensor memory); the
//    leader (rank 0) issues every MMA for the pair.  Each SM streams 38 KiB per
//    K = 256 stage, 30% less than a single-CTA 128 x 256 tile needs, which keeps
//    the L2 -> shared-memory stream below what the tensor core consumes.
//  * warp 0 (both CTAs): TMA producer into a 4-stage ring: per stage the operand
//    tiles and the stage's scale tiles, all completing on the leader's `full`
//    barrier (armed by the leader for both CTAs' bytes).
//  * warp 1 (leader; the whole warp runs the loop, lane 0 issues): barrier waits in
//    batches, then per stage the LoRA MMAs (kind::f16), or per K = 64 step the three
//    tcgen05.cp copies of that step's scale chunks from shared memory into the
//    stage's tensor-memory scale slot (32 rows x 16 bytes each, replicated into the
//    four sub-partitions) followed by the NVFP4 MMA; the stage is committed to both
//    CTAs' `empty` barriers.  Copies and MMAs of one thread execute in issue order,
//    so the scales need no synchronisation of their own.
//  * warps 2-17 (both CTAs): epilogue, four warps per tensor-memory sub-partition,
//    64 columns each.  A warp loads its 32 x 64 block of the accumulator into
//    registers and releases the accumulator at once, so the pair's next tile starts
//    while the warp adds the residual (prefetched by TMA into the warp's 4 KiB
//    shared-memory slab), rounds to BF16 into the slab and writes it with one TMA
//    store, which also clips the ragged edges of the output.
#include <cmath>
#include "quant.cuh"

namespace pact {
namespace gemm {

constexpr int BM = 128;               // rows per CTA; the pair tile has 256
constexpr int BN = 256;               // columns of the pair tile; each CTA loads 128 rows of B
constexpr int BK = 256;               // FP4 elements per stage = 128 bytes per row
constexpr int KSTEP = 64;             // FP4 elements per MMA
constexpr int A_BYTES = BM * BK / 2;          // 16384
constexpr int B_BYTES = (BN / 2) * BK / 2;    // 16384
constexpr int OFF_B = A_BYTES;
constexpr int OFF_SFA = OFF_B + B_BYTES;      // 4 chunks of 512 (this CTA's rows)
constexpr int OFF_SFB = OFF_SFA + 2048;       // 2 row groups x 4 chunks (all 256 columns)
constexpr int SF_BYTES = 2048 + 4096;
constexpr int STAGE_BYTES = OFF_SFB + 4096;   // 38912 = 38 KiB
constexpr int OFF_LW = 6 * BM * 32;           // LoRA weight chunks follow 6 activation chunks
static_assert(OFF_LW + 3 * BM * 32 <= STAGE_BYTES && OFF_LW + 2 * 48 * 128 <= STAGE_BYTES, "LoRA stage");
constexpr int EPI_WARPS = 16;
constexpr int THREADS = 32 * (2 + EPI_WARPS);                 // 576
// Shared memory: the ring, then one slab per epilogue warp, then the barriers.  The
// plain GEMM writes a warp's 32 x 64 block through a 32 x 32 slab (two TMA stores,
// 64-byte swizzle), which leaves room for a fifth ring stage; the gate|up mode keeps a
// whole 32 x 64 gate block (128-byte swizzle) in the slab until the up block of the
// same columns, so it runs four stages.
template <bool SILU>
struct Layout {
    static constexpr int STAGES = SILU ? 4 : 5;
    static constexpr int SLAB_COLS = SILU ? 64 : 32;
    static constexpr int SLAB_BYTES = 32 * SLAB_COLS * 2;
    static constexpr int OFF_SLABS = STAGES * STAGE_BYTES;
    static constexpr int OFF_BARS = OFF_SLABS + EPI_WARPS * SLAB_BYTES;
    static constexpr int SMEM_BYTES = 1024 + OFF_BARS + 512;
    static_assert(SMEM_BYTES <= 232448, "shared memory");
};
constexpr int MAX_STAGES = Layout<false>::STAGES > Layout<true>::STAGES ? Layout<false>::STAGES : Layout<true>::STAGES;

// tensor memory columns
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t COL_ACC = 0;        // 256 FP32 columns
constexpr uint32_t COL_SF = 256;       // per stage: 16 columns of A scales, then 32 of B scales
constexpr uint32_t SF_COLS = 48;
static_assert(COL_SF + MAX_STAGES * SF_COLS <= TMEM_COLS, "tensor memory");

enum LoraMode : int { LORA_NONE = 0, LORA_FWD = 1, LORA_DGRAD = 2 };

struct Params {
    int M, N, K;
    int has_res;          // add the residual (map tmR; may alias the output) in the epilogue
    int lora_mode;
    int lora_steps;       // weight chunks of K = 16 per tile (two MMAs each: hi and lo activations)
    int lora_r;
    int lora_nseg;
    int64_t seg_end[4];
    float out_scale;      // 2^gexp of the weight cache: scales the accumulator (exact)
    const pact_bf16 *res; // the residual (its second 32-column half of a block is read directly)
    int64_t ldr;
    int n_fast;           // tile order: 1 = N tiles fastest (A streamed once), 0 = M tiles fastest
    // optional NVFP4 copy of the BF16 output, split along N into nq (1 or 2) tensors:
    // columns [0, q_split) into q[0], [q_split, N) into q[1]
    int nq;
    int q_split;
    uint8_t *q_codes[2];
    uint8_t *q_scales[2];
    // gate|up mode: N = 2 I with the gate rows first; the tiles of gate columns
    // [256 j, 256 j + 256) and up columns [I + 256 j, ...) run back to back on one CTA
    // pair, and the epilogue writes m = BF16(silu(g) u) (map tmD over m [M x I]) and its
    // NVFP4 copy instead of g and u
    int silu;
    int half_tiles;       // I / 256
    uint8_t *m_codes;
    uint8_t *m_scales;
};

// Pair-tile coordinates of persistent tile index t.  Consecutive indices run at the
// same time on neighbouring clusters, so the operand whose tile they share stays in
// L2 while the other one streams: with N fastest each row block of A is read once
// and shared by the clusters working across N; with M fastest the same holds for B.
__device__ __forceinline__ void tile_coords(const Params &p, int t, int mpairs, int ntiles, int &mp, int &nt) {
    if (p.silu) {   // t = 2 u + which: pair u of (gate, up) tiles
        const int u = t >> 1, h = p.half_tiles;
        int jn;
        if (p.n_fast) {
            jn = u % h;
            mp = u / h;
        } else {
            mp = u % mpairs;
            jn = u / mpairs;
        }
        nt = jn + (t & 1) * h;
    } else if (p.n_fast) {
        nt = t % ntiles;
        mp = t / ntiles;
    } else {
        mp = t % mpairs;
        nt = t / mpairs;
    }
}
// The persistent tile sequence of a cluster (every role walks the same one): tiles
// cluster, cluster + nclusters, ...; in gate|up mode the two tiles of each pair
// 2 u, 2 u + 1 for u = cluster, cluster + nclusters, ...
__device__ __forceinline__ int first_tile(const Params &p, int cluster) { return p.silu ? 2 * cluster : cluster; }
__device__ __forceinline__ int next_tile(const Params &p, int t, int nclusters) {
    return p.silu ? ((t & 1) ? t + 2 * nclusters - 1 : t + 1) : t + nclusters;
}

__device__ __forceinline__ int lora_segment(const Params &p, int n0) {
    int s = 0;
#pragma unroll
    for (int i = 0; i < 3; ++i) s += (i + 1 < p.lora_nseg && n0 >= p.seg_end[i]) ? 1 : 0;
    return s;
}

// NVFP4 copy of one row's 64 output columns (the BF16-rounded values, 32 packed
// words: columns 2j, 2j+1 in word j): four 16-value blocks quantized in this thread,
// 32 code bytes and 4 scale bytes stored; rows past M in the 128-row padding of the
// scale layout get zero scales.
// Where a row's NVFP4 copy of 64 output columns goes: its codes (nullptr for rows
// that get none) and its 4 scale bytes (nullptr past the 128-row padding).
struct QDest {
    uint8_t *codes, *scales;
};
// The same for m's NVFP4 copy in gate|up mode (col: the up block's column, I + c).
__device__ __forceinline__ QDest mdest(const Params &p, int row, int col) {
    QDest d = {nullptr, nullptr};
    if (row >= ((p.M + 127) & ~127)) return d;
    const int I = p.half_tiles * BN, lc = col - I;
    d.scales = p.m_scales + scale_offset(row, lc >> 4, I);
    if (row < p.M) d.codes = p.m_codes + (int64_t)row * (I >> 1) + (lc >> 1);
    return d;
}
__device__ __forceinline__ QDest qdest(const Params &p, int row, int col) {
    QDest d = {nullptr, nullptr};
    if (!p.nq || row >= ((p.M + 127) & ~127)) return d;
    const int seg = (p.nq > 1 && col >= p.q_split) ? 1 : 0;
    const int lc = col - (seg ? p.q_split : 0);
    const int cols = seg ? p.N - p.q_split : (p.nq > 1 ? p.q_split : p.N);
    // select, not index: a runtime index into the parameter arrays would copy them to local memory
    d.scales = (seg ? p.q_scales[1] : p.q_scales[0]) + scale_offset(row, lc >> 4, cols);
    if (row < p.M) d.codes = (seg ? p.q_codes[1] : p.q_codes[0]) + (int64_t)row * (cols >> 1) + (lc >> 1);
    return d;
}

// Every stage of the ring is used in the same order by all roles: per tile, one LoRA
// stage (when the GEMM carries a LoRA term) and then ktiles K stages.
template <int STAGES>
struct Ring {
    uint32_t stage = 0, phase = 0;
    __device__ __forceinline__ void next() {
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
    }
};

// SILU: gate|up mode (p.silu set), instantiated apart so that the plain GEMM's
// epilogue keeps its registers.
template <bool SILU>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
k_nvfp4_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
             const __grid_constant__ CUtensorMap tmSFA, const __grid_constant__ CUtensorMap tmSFB,
             const __grid_constant__ CUtensorMap tmLa, const __grid_constant__ CUtensorMap tmLb,
             const __grid_constant__ CUtensorMap tmD, const __grid_constant__ CUtensorMap tmR, const Params p) {
    using L = Layout<SILU>;
    constexpr int STAGES = L::STAGES;
    using Ring = pact::gemm::Ring<STAGES>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + (((raw + 1023) & ~1023u) - raw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::OFF_BARS);
    uint64_t *full = bars;                        // [STAGES] leader: operands and scales of both CTAs
    uint64_t *empty = bars + STAGES;              // [STAGES] local: the pair's MMAs are done with the stage
    uint64_t *acc_full = bars + 2 * STAGES;       // local: accumulator complete
    uint64_t *acc_empty = acc_full + 1;           // leader: all epilogue warps of both CTAs have read it
    uint64_t *drained = acc_full + 2;             // leader: every tcgen05 operation has completed
    uint64_t *res_full = acc_full + 3;            // [EPI_WARPS] local: residual block in the warp's slab
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(res_full + EPI_WARPS);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int mpairs = (p.M + 2 * BM - 1) / (2 * BM), ntiles = (p.N + BN - 1) / BN;
    const int total = mpairs * ntiles;
    const int cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;
    const int ktiles = (p.K + BK - 1) / BK;
    const int kgroups = p.K / 64;
    const bool lora = p.lora_mode != LORA_NONE;
    const int nsteps = ktiles + (lora ? 1 : 0);   // ring stages per tile

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 2 * EPI_WARPS);
        mbar_init(drained, 1);
        for (int w = 0; w < EPI_WARPS; ++w) mbar_init(&res_full[w], 1);
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
        prefetch_tensormap(&tmSFA);
        prefetch_tensormap(&tmSFB);
        prefetch_tensormap(&tmD);
        if (p.has_res) prefetch_tensormap(&tmR);
        if (lora) {
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
    pdl_wait();      // inputs of the previous kernel are complete from here on
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ producer (both CTAs)
        if (lane == 0) {
            const uint32_t full_leader = mapa_shared(smem_u32(full), 0);
            Ring rg;
            bool ok = true;
            for (int t = first_tile(p, cluster); ok && t < total; t = next_tile(p, t, nclusters)) {
                int mp, nt;
                tile_coords(p, t, mpairs, ntiles, mp, nt);
                const int m0 = mp * 2 * BM + (int)rank * BM;     // this CTA's rows
                const int n0 = nt * BN, nb = n0 + (int)rank * (BN / 2);
                if (lora) {
                    if (!(ok = mbar_wait(&empty[rg.stage], rg.phase ^ 1))) break;
                    const uint32_t st = smem_u32(smem + rg.stage * STAGE_BYTES);
                    const uint32_t fb = full_leader + 8 * rg.stage;
                    const int R = p.lora_nseg * p.lora_r;
                    if (p.lora_mode == LORA_FWD) {
                        if (leader) mbar_arrive_expect_tx(&full[rg.stage], 2 * p.lora_steps * (2 * BM * 32 + BM * 32));
                        const int xs = lora_segment(p, n0) * p.lora_r;
                        for (int c = 0; c < p.lora_steps; ++c) {
                            tma_load_2d_pair(st + c * BM * 32, &tmLa, fb, xs + 16 * c, m0);
                            tma_load_2d_pair(st + (p.lora_steps + c) * BM * 32, &tmLa, fb, R + xs + 16 * c, m0);
                            tma_load_2d_pair(st + OFF_LW + c * BM * 32, &tmLb, fb, 16 * c, nb);
                        }
                    } else {
                        if (leader) mbar_arrive_expect_tx(&full[rg.stage], 2 * (p.lora_steps * 2 * BM * 32 + 2 * R * 128));
                        for (int c = 0; c < p.lora_steps; ++c) {
                            tma_load_2d_pair(st + c * BM * 32, &tmLa, fb, 16 * c, m0);
                            tma_load_2d_pair(st + (p.lora_steps + c) * BM * 32, &tmLa, fb, R + 16 * c, m0);
                        }
                        for (int q = 0; q < 2; ++q) tma_load_2d_pair(st + OFF_LW + q * R * 128, &tmLb, fb, nb + 64 * q, 0);
                    }
                    rg.next();
                }
                // scale map rows: 2 per 512-byte chunk; this CTA's 128-row group of A,
                // both 128-row groups of the B tile
                const int ga = m0 / 128, gb = n0 / 128;
                for (int kt = 0; kt < ktiles; ++kt) {
                    if (!(ok = mbar_wait(&empty[rg.stage], rg.phase ^ 1))) break;
                    const uint32_t st = smem_u32(smem + rg.stage * STAGE_BYTES);
                    const uint32_t fb = full_leader + 8 * rg.stage;
                    if (leader) mbar_arrive_expect_tx(&full[rg.stage], 2 * (A_BYTES + B_BYTES + SF_BYTES));
                    tma_load_2d_pair(st, &tmA, fb, kt * (BK / 2), m0);
                    tma_load_2d_pair(st + OFF_B, &tmB, fb, kt * (BK / 2), nb);
                    // the stage's scale chunks (one box = the 4 chunks of this K stage)
                    tma_load_2d_pair(st + OFF_SFA, &tmSFA, fb, 0, 2 * (ga * kgroups + kt * 4));
                    tma_load_2d_pair(st + OFF_SFB, &tmSFB, fb, 0, 2 * (gb * kgroups + kt * 4));
                    tma_load_2d_pair(st + OFF_SFB + 2048, &tmSFB, fb, 0, 2 * ((gb + 1) * kgroups + kt * 4));
                    rg.next();
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (leader)
        // The whole warp runs this loop converged (waits, ring position, descriptors are
        // warp-uniform); lane 0 alone issues the MMAs and commits (the _w forms).
        if (leader) {
            const uint32_t idesc = idesc_nvf4(2 * BM, BN);
            const uint32_t idesc_lora = idesc_bf16(2 * BM, BN, false, p.lora_mode == LORA_DGRAD);
            // operand descriptors of stage 0, K step 0; a stage / K step adds its byte
            // offset / 16 to the start-address field (addresses stay below 256 KiB)
            const uint64_t adesc0 = smem_desc(smem_u32(smem), 16, 1024, SW_128);
            const uint64_t bdesc0 = smem_desc(smem_u32(smem) + OFF_B, 16, 1024, SW_128);
            Ring rg;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int t = first_tile(p, cluster); ok && t < total; t = next_tile(p, t, nclusters)) {
                ok = warp_all(mbar_wait(acc_empty, acc_phase ^ 1));
                tc_fence_after();
                uint32_t accum = 0;
                // Per stage: its MMAs and the commit that frees the stage once they are
                // done.  Stage barriers are observed in batches: when no observed stage is
                // left, the thread waits for the next one and tests the two after it
                // without blocking (the producers run stages ahead); one fence covers the
                // batch, whose MMAs are then issued back to back.  The ring position lives
                // in registers here.
                uint32_t stage = rg.stage, phase = rg.phase;
                int known = 0;   // observed, fenced stages from step i on
                for (int i = 0; i < nsteps; ++i) {
                    if (known == 0) {
                        if (!(ok = warp_all(mbar_wait(&full[stage], phase)))) break;
                        const uint32_t s1 = stage + 1 == STAGES ? 0 : stage + 1;
                        const uint32_t p1 = stage + 1 == STAGES ? phase ^ 1 : phase;
                        const uint32_t s2 = s1 + 1 == STAGES ? 0 : s1 + 1;
                        const uint32_t p2 = s1 + 1 == STAGES ? p1 ^ 1 : p1;
                        const bool r1 = i + 1 < nsteps && warp_all(mbar_test_wait(&full[s1], p1));
                        const bool r2 = r1 && i + 2 < nsteps && warp_all(mbar_test_wait(&full[s2], p2));
                        known = 1 + (r1 ? 1 + (r2 ? 1 : 0) : 0);
                        tc_fence_after();
                    }
                    const uint32_t st = smem_u32(smem) + stage * STAGE_BYTES;
                    if (lora && i == 0) {
                        const int R = p.lora_nseg * p.lora_r;
                        for (int c = 0; c < p.lora_steps; ++c) {
                            const uint64_t bd = (p.lora_mode == LORA_FWD)
                                                    ? smem_desc(st + OFF_LW + c * BM * 32, 16, 256, SW_32)
                                                    : smem_desc(st + OFF_LW + c * 2048, R * 128, 1024, SW_128);
                            for (int h = 0; h < 2; ++h) {  // hi part, then lo part
                                const uint64_t ad = smem_desc(st + (h * p.lora_steps + c) * BM * 32, 16, 256, SW_32);
                                mma_bf16_pair_w(tmem + COL_ACC, ad, bd, idesc_lora, accum);
                                accum = 1;
                            }
                        }
                    } else {
                        const int kt = i - (lora ? 1 : 0);
                        const int nk = min(BK / KSTEP, (p.K - kt * BK) / KSTEP);
                        const uint32_t sf = tmem + COL_SF + stage * SF_COLS;
                        const uint64_t ad = adesc0 + (uint64_t)((stage * STAGE_BYTES) >> 4);
                        const uint64_t bd = bdesc0 + (uint64_t)((stage * STAGE_BYTES) >> 4);
                        // K step s: scale chunks s of A (columns 4s..4s+3 of the slot) and of
                        // the two 128-row groups of B (16 + 8s + 4g), then its MMA
                        const uint32_t sc = st + OFF_SFA;
                        auto copy_scales = [&](int s) {
                            tmem_cp_pair_32x128b_x4_w(sf + 4 * s, smem_desc(sc + s * 512, 0, 128, SW_NONE));
                            tmem_cp_pair_32x128b_x4_w(sf + 16 + 8 * s, smem_desc(sc + 2048 + s * 512, 0, 128, SW_NONE));
                            tmem_cp_pair_32x128b_x4_w(sf + 20 + 8 * s, smem_desc(sc + 4096 + s * 512, 0, 128, SW_NONE));
                        };
                        if (nk == BK / KSTEP) {
#pragma unroll
                            for (int s = 0; s < BK / KSTEP; ++s) {
                                copy_scales(s);
                                mma_nvf4_pair_w(tmem + COL_ACC, ad + 2 * s, bd + 2 * s, idesc, sf + 4 * s, sf + 16 + 8 * s,
                                              accum);
                                accum = 1;
                            }
                        } else {
                            for (int s = 0; s < nk; ++s) {
                                copy_scales(s);
                                mma_nvf4_pair_w(tmem + COL_ACC, ad + 2 * s, bd + 2 * s, idesc, sf + 4 * s, sf + 16 + 8 * s,
                                              accum);
                                accum = 1;
                            }
                        }
                    }
                    tc_commit_pair_w(&empty[stage], 3);
                    --known;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                rg.stage = stage;
                rg.phase = phase;
                if (!ok) break;
                tc_commit_pair_w(acc_full, 3);
                acc_phase ^= 1;
            }
            // tensor memory is released below only after every MMA issued here has completed
            tc_commit_pair_w(drained, 1);
            warp_all(mbar_wait(drained, 0));
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue (both CTAs)
        const int ew = warp - 2;                 // 0..15
        const int sub = warp & 3;                // tensor-memory sub-partition this warp may read
        const int quarter = ew >> 2;             // columns 64*quarter .. 64*quarter+63 of the tile
        const uint32_t acc_empty_leader = mapa_shared(smem_u32(acc_empty), 0);
        const uint32_t taddr = tmem + ((uint32_t)(sub * 32) << 16) + COL_ACC + quarter * 64;
        uint8_t *slab_p = smem + L::OFF_SLABS + ew * L::SLAB_BYTES;
        const uint32_t slab = smem_u32(slab_p);
        // this warp's 32 x 64 block of tile t: first row and column
        auto block_y = [&](int t) {
            int mp, nt;
            tile_coords(p, t, mpairs, ntiles, mp, nt);
            return mp * 2 * BM + (int)rank * BM + sub * 32;
        };
        auto block_x = [&](int t) {
            int mp, nt;
            tile_coords(p, t, mpairs, ntiles, mp, nt);
            return nt * BN + quarter * 64;
        };
        auto inside = [&](int t) { return block_y(t) < p.M && block_x(t) < p.N; };
        auto load_residual = [&](int t) {  // lane 0; the slab is free
            mbar_arrive_expect_tx(&res_full[ew], L::SLAB_BYTES);
            tma_load_2d(slab_p, &tmR, &res_full[ew], block_x(t), block_y(t));
        };
        uint32_t acc_phase = 0, res_phase = 0;
        if (p.has_res && lane == 0 && first_tile(p, cluster) < total && inside(first_tile(p, cluster)))
            load_residual(first_tile(p, cluster));
        bool ok = true;
        for (int t = first_tile(p, cluster); ok && t < total; t = next_tile(p, t, nclusters)) {
            bool got = false;
            if (lane == 0) got = mbar_wait(acc_full, acc_phase);
            if (!(ok = __shfl_sync(0xffffffffu, got, 0))) break;
            tc_fence_after();
            uint32_t r[64];
            tmem_ld_32x32b_x32(taddr, *reinterpret_cast<uint32_t(*)[32]>(r));
            tmem_ld_32x32b_x32(taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(r + 32));
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote_relaxed(acc_empty_leader);  // the pair may reuse the accumulator
            acc_phase ^= 1;
            if (p.nq && !inside(t) && block_x(t) < p.N) {
                // a 32-row block wholly in the scale layout's padding rows: zero scales only
                const QDest qd = qdest(p, block_y(t) + lane, block_x(t));
                if (qd.scales) *reinterpret_cast<uint32_t *>(qd.scales) = 0u;
                if (SILU && (t & 1)) {
                    const QDest md = mdest(p, block_y(t) + lane, block_x(t));
                    if (md.scales) *reinterpret_cast<uint32_t *>(md.scales) = 0u;
                }
            }
            if (inside(t)) {
                if constexpr (SILU) {
                    if (p.has_res) {
                        if (lane == 0) got = mbar_wait_sleep(&res_full[ew], res_phase);
                        if (!(ok = __shfl_sync(0xffffffffu, got, 0))) break;
                        res_phase ^= 1;
                    } else {
                        if (lane == 0) bulk_wait_read_all();  // the previous block's store has read the slab
                        __syncwarp();
                    }
                    // the NVFP4 copy of the block's rounded values: block b of this lane's row is
                    // quantized once its two 8-value pieces are rounded
                    const QDest qd = qdest(p, block_y(t) + lane, block_x(t));
                    // gate|up mode: the gate block stays in the slab for the up block that follows
                    const bool up = SILU && (t & 1);
                    uint32_t sbs = 0;
                    // row `lane` of the block: 8 pieces of 16 bytes, 128-byte swizzle
    #pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const uint32_t a = slab + lane * 128 + ((q ^ (lane & 7)) << 4);
                        float f[8];
    #pragma unroll
                        for (int i = 0; i < 8; ++i) f[i] = __uint_as_float(r[8 * q + i]) * p.out_scale;
                        if (p.has_res) {
                            uint32_t o0, o1, o2, o3;
                            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                                         : "=r"(o0), "=r"(o1), "=r"(o2), "=r"(o3)
                                         : "r"(a));
                            f[0] += bf16lo(o0); f[1] += bf16hi(o0); f[2] += bf16lo(o1); f[3] += bf16hi(o1);
                            f[4] += bf16lo(o2); f[5] += bf16hi(o2); f[6] += bf16lo(o3); f[7] += bf16hi(o3);
                        }
                        const uint32_t w0 = pack_bf16x2(f[0], f[1]), w1 = pack_bf16x2(f[2], f[3]);
                        const uint32_t w2 = pack_bf16x2(f[4], f[5]), w3 = pack_bf16x2(f[6], f[7]);
                        if (!up)
                            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(w0), "r"(w1), "r"(w2),
                                         "r"(w3)
                                         : "memory");
                        // the rounded values, kept for the NVFP4 copy (r[] is free again)
                        r[4 * q] = w0; r[4 * q + 1] = w1; r[4 * q + 2] = w2; r[4 * q + 3] = w3;
                        if ((q & 1) && qd.codes) {
                            uint32_t lo, hi, sb;
                            quant16_bf16(make_uint4(r[4 * q - 4], r[4 * q - 3], r[4 * q - 2], r[4 * q - 1]),
                                         make_uint4(w0, w1, w2, w3), &lo, &hi, &sb);
                            *reinterpret_cast<uint2 *>(qd.codes + 4 * (q - 1)) = make_uint2(lo, hi);
                            sbs |= sb << (4 * (q - 1));
                        }
                    }
                    if (qd.scales) *reinterpret_cast<uint32_t *>(qd.scales) = sbs;
                    if (up) {
                        // m = BF16(silu(g) u) for the 64 columns of this row: g from the slab (the
                        // gate block, same rows and columns), u from the packed words in r[0..31];
                        // m replaces g in the slab and is quantized block by block
                        const QDest md = mdest(p, block_y(t) + lane, block_x(t));
                        uint32_t msbs = 0, n0 = 0, n1 = 0, n2 = 0, n3 = 0;
    #pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const uint32_t a = slab + lane * 128 + ((q ^ (lane & 7)) << 4);
                            uint32_t g4[4], mw[4];
                            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                                         : "=r"(g4[0]), "=r"(g4[1]), "=r"(g4[2]), "=r"(g4[3])
                                         : "r"(a));
    #pragma unroll
                            for (int j = 0; j < 4; ++j)
                                mw[j] = pack_bf16x2(silu_mul_out(bf16lo(g4[j]), bf16lo(r[4 * q + j])),
                                                    silu_mul_out(bf16hi(g4[j]), bf16hi(r[4 * q + j])));
                            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(mw[0]), "r"(mw[1]),
                                         "r"(mw[2]), "r"(mw[3])
                                         : "memory");
                            if ((q & 1) && md.codes) {
                                uint32_t lo, hi, sb;
                                quant16_bf16(make_uint4(n0, n1, n2, n3), make_uint4(mw[0], mw[1], mw[2], mw[3]), &lo, &hi,
                                             &sb);
                                *reinterpret_cast<uint2 *>(md.codes + 4 * (q - 1)) = make_uint2(lo, hi);
                                msbs |= sb << (4 * (q - 1));
                            }
                            n0 = mw[0]; n1 = mw[1]; n2 = mw[2]; n3 = mw[3];
                        }
                        if (md.scales) *reinterpret_cast<uint32_t *>(md.scales) = msbs;
                    }
                    if (!SILU || up) {   // a gate block is not stored: its m follows with the up block
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(&tmD, slab, up ? block_x(t) - p.half_tiles * BN : block_x(t), block_y(t));
                            bulk_commit_group();
                        }
                    }
                } else {
                    // two 32-column halves through the 32 x 32 slab (64-byte swizzle): the
                    // first half's residual was prefetched into the slab by TMA, the second
                    // half's is read directly while the first half is written
                    const QDest qd = qdest(p, block_y(t) + lane, block_x(t));
                    uint4 rh[4];
                    if (p.has_res) {
                        const int row = block_y(t) + lane, c1 = block_x(t) + 32;
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            rh[j] = (row < p.M && c1 + 8 * j < p.N)
                                        ? *reinterpret_cast<const uint4 *>(p.res + (int64_t)row * p.ldr + c1 + 8 * j)
                                        : make_uint4(0, 0, 0, 0);
                        if (lane == 0) got = mbar_wait_sleep(&res_full[ew], res_phase);
                        if (!(ok = __shfl_sync(0xffffffffu, got, 0))) break;
                        res_phase ^= 1;
                    } else {
                        if (lane == 0) bulk_wait_read_all();  // the previous block's stores have read the slab
                        __syncwarp();
                    }
                    uint32_t sbs = 0;
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        if (q == 4) {   // the first half is in the slab: store it, then reuse the slab
                            fence_proxy_async_smem();
                            __syncwarp();
                            if (lane == 0) {
                                tma_store_2d(&tmD, slab, block_x(t), block_y(t));
                                bulk_commit_group();
                                bulk_wait_read_all();
                            }
                            __syncwarp();
                        }
                        const uint32_t a = slab + lane * 64 + (((q & 3) ^ ((lane >> 1) & 3)) << 4);
                        float f[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) f[i] = __uint_as_float(r[8 * q + i]) * p.out_scale;
                        if (p.has_res) {
                            uint32_t o0, o1, o2, o3;
                            if (q < 4) {
                                asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                                             : "=r"(o0), "=r"(o1), "=r"(o2), "=r"(o3)
                                             : "r"(a));
                            } else {
                                o0 = rh[q - 4].x; o1 = rh[q - 4].y; o2 = rh[q - 4].z; o3 = rh[q - 4].w;
                            }
                            f[0] += bf16lo(o0); f[1] += bf16hi(o0); f[2] += bf16lo(o1); f[3] += bf16hi(o1);
                            f[4] += bf16lo(o2); f[5] += bf16hi(o2); f[6] += bf16lo(o3); f[7] += bf16hi(o3);
                        }
                        const uint32_t w0 = pack_bf16x2(f[0], f[1]), w1 = pack_bf16x2(f[2], f[3]);
                        const uint32_t w2 = pack_bf16x2(f[4], f[5]), w3 = pack_bf16x2(f[6], f[7]);
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(w0), "r"(w1), "r"(w2),
                                     "r"(w3)
                                     : "memory");
                        // the rounded values, kept for the NVFP4 copy (r[] is free again)
                        r[4 * q] = w0; r[4 * q + 1] = w1; r[4 * q + 2] = w2; r[4 * q + 3] = w3;
                        if ((q & 1) && qd.codes) {
                            uint32_t lo, hi, sb;
                            quant16_bf16(make_uint4(r[4 * q - 4], r[4 * q - 3], r[4 * q - 2], r[4 * q - 1]),
                                         make_uint4(w0, w1, w2, w3), &lo, &hi, &sb);
                            *reinterpret_cast<uint2 *>(qd.codes + 4 * (q - 1)) = make_uint2(lo, hi);
                            sbs |= sb << (4 * (q - 1));
                        }
                    }
                    if (qd.scales) *reinterpret_cast<uint32_t *>(qd.scales) = sbs;
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&tmD, slab, block_x(t) + 32, block_y(t));
                        bulk_commit_group();
                    }
                }
            }
            if (lane == 0 && p.has_res && next_tile(p, t, nclusters) < total && inside(next_tile(p, t, nclusters))) {
                bulk_wait_read_all();
                load_residual(next_tile(p, t, nclusters));
            }
            __syncwarp();
        }
        if (lane == 0) bulk_wait_all();
        __syncwarp();
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

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiled)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiled encode_fn() {
    // looked up once (a function-local static's initialisation is thread-safe)
    static const EncodeTiled fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<EncodeTiled>(p);
        return static_cast<EncodeTiled>(nullptr);
    }();
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
    static std::atomic<bool> done[64];   // per device; setting the attribute twice is harmless
    const int d = current_device();
    if (d >= 0 && d < 64 && done[d].load(std::memory_order_acquire)) return PACT_OK;
    cudaError_t e =
        cudaFuncSetAttribute(k_nvfp4_gemm<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, Layout<false>::SMEM_BYTES);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(k_nvfp4_gemm<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, Layout<true>::SMEM_BYTES);
    if (e != cudaSuccess) return fail(PACT_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    if (d >= 0 && d < 64) done[d].store(true, std::memory_order_release);
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
// Gate|up mode outputs: m [M x I] (BF16, row stride ldm) and the NVFP4 copies mq, gq, uq.
struct SiluOut {
    pact_bf16 *m;
    int64_t ldm;
    const pact_nvfp4_t *mq;
};

// D[M x N] = deq(a) . deq(b)^T (+ LoRA); a [M x K], b [N x K].  With so, gate|up mode:
// D is not written; m, mq (and through yq, gq and uq) are.
static pact_status run(const pact_nvfp4_t *a, const pact_nvfp4_t *b, int gexp, const pact_lora_t *lora, bool dgrad,
                       const pact_bf16 *res, int64_t ldr, pact_bf16 *out, int64_t ldo, const pact_nvfp4_t *yq, int nq,
                       cudaStream_t stream, const char *what, const SiluOut *so = nullptr) {
    const int64_t M = a->rows, K = a->cols, N = b->rows;
    PACT_CHECK(gexp >= -100 && gexp <= 100, PACT_ERR_INVALID_ARG, "%s: w->gexp out of range (%d)", what, gexp);
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
    CUtensorMap tmA, tmB, tmSFA, tmSFB, tmLa, tmLb, tmD, tmR;
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
    // output (and residual) blocks: 32 rows x 64 BF16 columns, 128-byte swizzle; in
    // gate|up mode the output is m [M x N / 2]
    if (s == PACT_OK)
        s = so ? make_map(&tmD, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, so->m, N / 2, M, so->ldm * 2, 64, 32,
                          CU_TENSOR_MAP_SWIZZLE_128B, what)
               : make_map(&tmD, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, out, N, M, ldo * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B,
                          what);
    tmR = tmD;
    if (s == PACT_OK && res)   // the plain GEMM's residual: the first half of each 32 x 64 block
        s = make_map(&tmR, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, res, N, M, ldr * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B,
                     what);
    if (s != PACT_OK) return s;
    Params p;
    p.M = (int)M; p.N = (int)N; p.K = (int)K;
    p.has_res = res != nullptr;
    p.out_scale = std::ldexp(1.0f, gexp);
    p.res = res;
    p.ldr = ldr;
    // stream the larger operand once: A (M x K) when M > N, else B (N x K)
    p.n_fast = M > N ? 1 : 0;
    p.nq = nq;
    p.q_split = (int)N;
    for (int i = 0; i < 2; ++i) {
        p.q_codes[i] = i < nq ? static_cast<uint8_t *>(yq[i].codes) : nullptr;
        p.q_scales[i] = i < nq ? static_cast<uint8_t *>(yq[i].scales) : nullptr;
    }
    if (nq == 2) p.q_split = (int)yq[0].cols;
    p.silu = so ? 1 : 0;
    p.half_tiles = so ? (int)(N / 2 / BN) : 0;
    p.m_codes = so ? static_cast<uint8_t *>(so->mq->codes) : nullptr;
    p.m_scales = so ? static_cast<uint8_t *>(so->mq->scales) : nullptr;
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
    // work units: output tiles, or (gate, up) tile pairs in gate|up mode
    // As few pairs as finish the tiles in the same number of rounds as all of them
    // would: the grid's last round is then full, and the pairs left over are free for
    // kernels on other streams (384 tiles on 148 SMs: 6 rounds on 64 pairs, not 5.2 on 74).
    const int units = (int)(((M + 255) / 256) * ((N + 255) / 256)) / (so ? 2 : 1);
    const int max_clusters = sm_count() / 2;
    const int rounds = (units + max_clusters - 1) / max_clusters;
    const int clusters = (units + rounds - 1) / rounds;
    return launch_dep(so ? k_nvfp4_gemm<true> : k_nvfp4_gemm<false>, dim3(2 * clusters), dim3(THREADS),
                      so ? Layout<true>::SMEM_BYTES : Layout<false>::SMEM_BYTES,
                      stream, what, tmA, tmB, tmSFA, tmSFB, tmLa, tmLb, tmD, tmR, p);
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
    return gemm::run(xq, &w->fwd, w->gexp, lora, false, residual, ldr, y, ldy, nullptr, 0, (cudaStream_t)stream,
                     "pact_frozen_gemm_fwd");
}

pact_status pact_frozen_gemm_fwd_quant(const pact_nvfp4_t *xq, const pact_weight_cache_t *w, const pact_lora_t *lora,
                                       const pact_bf16 *residual, int64_t ldr, pact_bf16 *y, int64_t ldy,
                                       const pact_nvfp4_t *yq, int nq, pact_stream_t stream) {
    const char *what = "pact_frozen_gemm_fwd_quant";
    PACT_CHECK(xq && w && yq, PACT_ERR_INVALID_ARG, "%s: NULL argument", what);
    PACT_CHECK(nq == 1 || nq == 2, PACT_ERR_INVALID_ARG, "%s: nq must be 1 or 2", what);
    const int64_t N = w->fwd.rows, K = w->fwd.cols;
    pact_status s = check_nvfp4(&w->fwd, N, K, "w->fwd");
    if (s == PACT_OK) s = check_nvfp4(xq, xq->rows, K, "xq");
    if (s != PACT_OK) return s;
    PACT_CHECK(xq->rows >= 1 && N % 64 == 0 && K % 64 == 0, PACT_ERR_SHAPE, "%s: bad shape", what);
    int64_t covered = 0;
    for (int i = 0; i < nq; ++i) {
        PACT_CHECK(yq[i].cols >= 64 && yq[i].cols % 64 == 0, PACT_ERR_SHAPE, "%s: yq[%d].cols must be a multiple of 64", what, i);
        s = check_nvfp4(&yq[i], xq->rows, yq[i].cols, "yq");
        if (s != PACT_OK) return s;
        PACT_CHECK(aligned16(yq[i].codes) && aligned16(yq[i].scales), PACT_ERR_ALIGN, "%s: yq 16-byte aligned", what);
        covered += yq[i].cols;
    }
    PACT_CHECK(covered == N, PACT_ERR_SHAPE, "%s: the yq tensors' columns must add up to N = %lld", what, (long long)N);
    return gemm::run(xq, &w->fwd, w->gexp, lora, false, residual, ldr, y, ldy, yq, nq, (cudaStream_t)stream, what);
}

pact_status pact_frozen_gemm_fwd_silu(const pact_nvfp4_t *xq, const pact_weight_cache_t *w, const pact_lora_t *lora,
                                      pact_bf16 *m, int64_t ldm, const pact_nvfp4_t *mq, const pact_nvfp4_t *gq,
                                      const pact_nvfp4_t *uq, pact_stream_t stream) {
    const char *what = "pact_frozen_gemm_fwd_silu";
    PACT_CHECK(xq && w && m && mq && gq && uq, PACT_ERR_INVALID_ARG, "%s: NULL argument", what);
    const int64_t N = w->fwd.rows, K = w->fwd.cols, I = N / 2, M = xq->rows;
    pact_status s = check_nvfp4(&w->fwd, N, K, "w->fwd");
    if (s == PACT_OK) s = check_nvfp4(xq, M, K, "xq");
    if (s != PACT_OK) return s;
    PACT_CHECK(M >= 1 && N % 512 == 0 && K % 64 == 0, PACT_ERR_SHAPE,
               "%s: the gate|up weight needs I = N / 2 a multiple of 256 (N = %lld)", what, (long long)N);
    PACT_CHECK(ldm >= I && ldm % 8 == 0 && aligned16(m), PACT_ERR_ALIGN, "%s: m 16-byte aligned with ldm >= I, %% 8 == 0",
               what);
    s = check_nvfp4(mq, M, I, "mq");
    if (s == PACT_OK) s = check_nvfp4(gq, M, I, "gq");
    if (s == PACT_OK) s = check_nvfp4(uq, M, I, "uq");
    if (s != PACT_OK) return s;
    const pact_nvfp4_t yq[2] = {*gq, *uq};
    const gemm::SiluOut so = {m, ldm, mq};
    // D itself is not written in this mode; out only has to satisfy the argument checks
    return gemm::run(xq, &w->fwd, w->gexp, lora, false, nullptr, 0, m, N, yq, 2, (cudaStream_t)stream, what, &so);
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
    return gemm::run(dyq, &w->bwd, w->gexp, lora, true, residual, ldr, dx, lddx, nullptr, 0, (cudaStream_t)stream,
                     "pact_frozen_gemm_dgrad");
}

}  // extern "C"
