// lora.cu -- the BF16 LoRA branch of each frozen projection ([LORA]: PEFT explainer,
// section "LoRA": h = W0 x + B A x; [METHOD]: PACT blog summary, section "方法",
// paragraph after the bullets: A and B stay BF16 and are never quantized).
//
// The products are skinny (rank 16 per adapter): X . A^T, dY . B (contraction over the
// feature dimension, R <= 64 outputs per row) and U^T . X, dY^T . T (contraction over
// the tokens).  These kernels run them on the CUDA cores with FP32 accumulation and
// shared-memory tiles; the token contractions are split over token chunks and reduced
// with FP32 atomics into caller-provided scratch.
#include "quant.cuh"

namespace pact {
namespace lora {

// ------------------------------------------------------------ row products
// out[m, j] = scale * sum_k X[m, k] * W(j, k) for j < R, where W(j, k) is
//   Wt = false: W[j * ldw + k]       (A [R x K] row-major)
//   Wt = true : W[k * ldw + j_src]   (B [N x r] row-major, used transposed) with
//               segment-wise contraction: column j belongs to segment j / r and sums
//               k over that segment's feature range only.
// X is BF16 (row stride ldx) or NVFP4 (xq, dequantized on load).
constexpr int RT = 32;   // rows per CTA
constexpr int KC = 64;   // contraction chunk

struct RowArgs {
    const pact_bf16 *x;
    int64_t ldx;
    pact_nvfp4_t xq;
    int use_xq;
    int64_t M, K;
    const pact_bf16 *w;
    int64_t ldw;
    int wt;       // W used transposed (B)
    int R, r, nseg;
    int64_t seg_end[4];
    float scale;
    pact_bf16 *out_bf16;  // one of these two; BF16 output is hi (columns 0..R-1) + lo (R..2R-1)
    float *out_f32;
    int64_t ldo;
};

__global__ void __launch_bounds__(256) k_rows(const RowArgs a) {
    __shared__ float xs[RT][KC + 1];
    __shared__ float ws[64][KC + 1];
    const int t = threadIdx.x;
    const int64_t m0 = (int64_t)blockIdx.x * RT;
    const int row = t >> 3;          // 0..31
    const int jl = t & 7;            // j = jl + 8 i
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    // With Wt, the contraction of segment s runs over [seg_begin(s), seg_end[s]);
    // chunk loop covers [0, K) and masks per output column.
    for (int64_t k0 = 0; k0 < a.K; k0 += KC) {
        // X chunk: 32 rows x 64 columns; thread t loads 8 values of row t/8
        {
            const int rr = t >> 3, cc = (t & 7) * 8;
            const int64_t m = m0 + rr, k = k0 + cc;
            float v[8] = {0, 0, 0, 0, 0, 0, 0, 0};
            if (m < a.M && k < a.K) {
                if (a.use_xq) load8_nvfp4(a.xq, m, k, v);
                else load8_bf16(a.x + m * a.ldx + k, v);
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) xs[rr][cc + i] = v[i];
        }
        // W chunk: R rows x 64 columns
        for (int idx = t; idx < a.R * (KC / 8); idx += 256) {
            const int j = idx / (KC / 8), cc = (idx % (KC / 8)) * 8;
            const int64_t k = k0 + cc;
            float v[8] = {0, 0, 0, 0, 0, 0, 0, 0};
            if (k < a.K) {
                if (!a.wt) {
                    load8_bf16(a.w + (int64_t)j * a.ldw + k, v);
                } else {
                    const int s = j / a.r, js = j % a.r;
                    const int64_t lo = s ? a.seg_end[s - 1] : 0, hi = a.seg_end[s];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int64_t kk = k + i;
                        v[i] = (kk >= lo && kk < hi) ? bf16lo(a.w[kk * a.ldw + js]) : 0.0f;
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) ws[j][cc + i] = v[i];
        }
        __syncthreads();
#pragma unroll 8
        for (int k = 0; k < KC; ++k) {
            const float xv = xs[row][k];
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (jl + 8 * i < a.R) acc[i] = fmaf(xv, ws[jl + 8 * i][k], acc[i]);
        }
        __syncthreads();
    }
    const int64_t m = m0 + row;
    if (m < a.M) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int j = jl + 8 * i;
            if (j < a.R) {
                const float v = acc[i] * a.scale;
                if (a.out_f32) {
                    a.out_f32[m * a.ldo + j] = v;
                } else {  // v as the unevaluated sum hi + lo of two BF16 values
                    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
                    a.out_bf16[m * a.ldo + j] = __bfloat16_as_ushort(hi);
                    a.out_bf16[m * a.ldo + a.R + j] =
                        __bfloat16_as_ushort(__float2bfloat16_rn(v - __bfloat162float(hi)));
                }
            }
        }
    }
}

// ------------------------------------------------------------ token contractions
// ws[a, b] += sum_{m in chunk} P[m, a] * Q[m, qcol(a) + b], a < A, b < Bn.
//   P: BF16 [M x A] (row stride ldp).
//   Q: BF16 (ldq) or NVFP4 (qq) or FP32 (qf, ldq); qcol(a) = seg(a) * r when
//      segmented (dB), else 0.
constexpr int TA = 64, TB = 64, MC = 32, MCHUNK = 256;

struct OuterArgs {
    const pact_bf16 *p;
    int64_t ldp;
    int p_split;  // P holds hi (columns 0..A-1) + lo (A..2A-1)
    const pact_bf16 *q;
    const float *qf;
    pact_nvfp4_t qq;
    int q_kind;  // 0 bf16, 1 nvfp4, 2 fp32
    int64_t ldq;
    int64_t M, A, Bn;
    int segmented, r, nseg;
    int64_t seg_end[4];
    float *ws;
    int64_t ldws;
};

__global__ void __launch_bounds__(256) k_outer(const OuterArgs o) {
    __shared__ float ps[MC][TA + 1];
    __shared__ float qs[MC][TB + 1];
    const int t = threadIdx.x;
    const int64_t a0 = (int64_t)blockIdx.x * TA, b0 = (int64_t)blockIdx.y * TB;
    const int64_t mbeg = (int64_t)blockIdx.z * MCHUNK;
    const int64_t mend = min(o.M, mbeg + MCHUNK);
    int64_t qoff = 0;
    if (o.segmented) {
        int s = 0;
        for (int i = 0; i + 1 < o.nseg; ++i) s += (a0 >= o.seg_end[i]) ? 1 : 0;
        qoff = (int64_t)s * o.r;
    }
    const int ta = (t >> 4) * 4, tb = (t & 15) * 4;  // 4 x 4 outputs per thread
    float acc[4][4] = {};
    for (int64_t m0 = mbeg; m0 < mend; m0 += MC) {
        // P tile: MC rows x TA columns (8 per thread load)
        {
            const int rr = t >> 3, cc = (t & 7) * 8;
            const int64_t m = m0 + rr, a = a0 + cc;
            float v[8] = {0, 0, 0, 0, 0, 0, 0, 0};
            if (m < mend && a < o.A) {
                load8_bf16(o.p + m * o.ldp + a, v);
                if (o.p_split) {
                    float lo[8];
                    load8_bf16(o.p + m * o.ldp + o.A + a, lo);
#pragma unroll
                    for (int i = 0; i < 8; ++i) v[i] += lo[i];
                }
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) ps[rr][cc + i] = v[i];
        }
        {
            const int rr = t >> 3, cc = (t & 7) * 8;
            const int64_t m = m0 + rr, b = b0 + cc;
            float v[8] = {0, 0, 0, 0, 0, 0, 0, 0};
            if (m < mend && b < o.Bn) {
                if (o.q_kind == 0) load8_bf16(o.q + m * o.ldq + qoff + b, v);
                else if (o.q_kind == 1) load8_nvfp4(o.qq, m, qoff + b, v);
                else {
                    const float4 *s4 = reinterpret_cast<const float4 *>(o.qf + m * o.ldq + qoff + b);
                    const float4 x0 = s4[0], x1 = s4[1];
                    v[0] = x0.x; v[1] = x0.y; v[2] = x0.z; v[3] = x0.w;
                    v[4] = x1.x; v[5] = x1.y; v[6] = x1.z; v[7] = x1.w;
                }
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) qs[rr][cc + i] = v[i];
        }
        __syncthreads();
#pragma unroll 4
        for (int mm = 0; mm < MC; ++mm) {
            float pv[4], qv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                pv[i] = ps[mm][ta + i];
                qv[i] = qs[mm][tb + i];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(pv[i], qv[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int64_t a = a0 + ta + i;
        if (a >= o.A) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t b = b0 + tb + j;
            if (b < o.Bn) atomicAdd(&o.ws[a * o.ldws + b], acc[i][j]);
        }
    }
}

// dst (row stride ldd) = BF16(scale * src), src FP32 [rows x cols] row-major.
__global__ void k_finalize(const float *__restrict__ src, int64_t rows, int64_t cols, float scale,
                           pact_bf16 *__restrict__ dst, int64_t ldd) {
    const int64_t n = rows * cols;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / cols, c = i % cols;
        dst[r * ldd + c] = __bfloat16_as_ushort(__float2bfloat16_rn(src[i] * scale));
    }
}

}  // namespace lora
}  // namespace pact

using namespace pact;
using namespace pact::lora;

static size_t lora_up256(size_t b) { return (b + 255) & ~(size_t)255; }

extern "C" {

pact_status pact_lora_fwd(const pact_bf16 *x, int64_t ldx, int64_t M, int64_t K, const pact_bf16 *A, int R,
                          float scale, pact_bf16 *T, int64_t ldt, pact_stream_t stream) {
    PACT_CHECK(x && A && T, PACT_ERR_INVALID_ARG, "pact_lora_fwd: NULL argument");
    PACT_CHECK(M >= 1 && K >= 64 && K % 64 == 0 && R >= 16 && R <= 64 && R % 16 == 0, PACT_ERR_SHAPE,
               "pact_lora_fwd: need M >= 1, K a multiple of 64, R in {16, 32, 48, 64}");
    PACT_CHECK(ldx >= K && ldx % 8 == 0 && ldt >= 2 * R && ldt % 8 == 0 && aligned16(x) && aligned16(A) && aligned16(T),
               PACT_ERR_ALIGN, "pact_lora_fwd: pointers 16-byte aligned, leading dims %% 8 == 0");
    RowArgs a = {};
    a.x = x; a.ldx = ldx; a.use_xq = 0; a.M = M; a.K = K;
    a.w = A; a.ldw = K; a.wt = 0; a.R = R; a.r = R; a.nseg = 1; a.seg_end[0] = K;
    a.scale = scale; a.out_bf16 = T; a.out_f32 = nullptr; a.ldo = ldt;
    k_rows<<<(unsigned)((M + RT - 1) / RT), 256, 0, (cudaStream_t)stream>>>(a);
    return launch_status("pact_lora_fwd");
}

pact_status pact_lora_bwd_u(const pact_bf16 *dy, int64_t lddy, int64_t M, int64_t N, const pact_bf16 *B, int r,
                            int nseg, const int64_t *seg_end, float scale, pact_bf16 *U, int64_t ldu,
                            pact_stream_t stream) {
    PACT_CHECK(dy && B && U && seg_end, PACT_ERR_INVALID_ARG, "pact_lora_bwd_u: NULL argument");
    PACT_CHECK(M >= 1 && N >= 64 && N % 64 == 0 && (r == 16 || r == 32 || r == 48 || r == 64) && nseg >= 1 &&
                   nseg <= 4 && nseg * r <= 64,
               PACT_ERR_SHAPE, "pact_lora_bwd_u: bad shape");
    int64_t prev = 0;
    for (int i = 0; i < nseg; ++i) {
        PACT_CHECK(seg_end[i] > prev && seg_end[i] % 64 == 0 && (i + 1 < nseg || seg_end[i] == N), PACT_ERR_SHAPE,
                   "pact_lora_bwd_u: segment ends must increase by multiples of 64 and end at N");
        prev = seg_end[i];
    }
    PACT_CHECK(lddy >= N && lddy % 8 == 0 && ldu >= 2 * nseg * r && ldu % 8 == 0 && aligned16(dy) && aligned16(B) &&
                   aligned16(U),
               PACT_ERR_ALIGN, "pact_lora_bwd_u: pointers 16-byte aligned, leading dims %% 8 == 0");
    RowArgs a = {};
    a.x = dy; a.ldx = lddy; a.use_xq = 0; a.M = M; a.K = N;
    a.w = B; a.ldw = r; a.wt = 1; a.R = nseg * r; a.r = r; a.nseg = nseg;
    for (int i = 0; i < 4; ++i) a.seg_end[i] = i < nseg ? seg_end[i] : N;
    a.scale = scale; a.out_bf16 = U; a.out_f32 = nullptr; a.ldo = ldu;
    k_rows<<<(unsigned)((M + RT - 1) / RT), 256, 0, (cudaStream_t)stream>>>(a);
    return launch_status("pact_lora_bwd_u");
}

size_t pact_lora_bwd_workspace_bytes(int64_t M, int64_t N, int64_t K, int r, int nseg) {
    const int64_t R = (int64_t)r * nseg;
    return lora_up256((size_t)(M * R * 4)) + lora_up256((size_t)(R * K * 4)) + lora_up256((size_t)(N * r * 4));
}

pact_status pact_lora_bwd(const pact_lora_bwd_t *g, void *workspace, size_t ws_bytes, pact_stream_t stream) {
    PACT_CHECK(g && workspace, PACT_ERR_INVALID_ARG, "pact_lora_bwd: NULL argument");
    PACT_CHECK(g->dy && g->A && g->U && g->dA && g->dB && ((g->x != nullptr) != (g->xq != nullptr)),
               PACT_ERR_INVALID_ARG, "pact_lora_bwd: dy, A, U, dA, dB and exactly one of x / xq are required");
    const int64_t M = g->M, N = g->N, K = g->K;
    const int r = g->r, nseg = g->nseg;
    PACT_CHECK(M >= 1 && N >= 64 && N % 64 == 0 && K >= 64 && K % 64 == 0 &&
                   (r == 16 || r == 32 || r == 48 || r == 64) && nseg >= 1 && nseg <= 4 && nseg * r <= 64,
               PACT_ERR_SHAPE, "pact_lora_bwd: bad shape");
    int64_t prev = 0;
    for (int i = 0; i < nseg; ++i) {
        PACT_CHECK(g->seg_end[i] > prev && g->seg_end[i] % 64 == 0 && (i + 1 < nseg || g->seg_end[i] == N),
                   PACT_ERR_SHAPE, "pact_lora_bwd: segment ends must increase by multiples of 64 and end at N");
        prev = g->seg_end[i];
    }
    const int R = nseg * r;
    PACT_CHECK(ws_bytes >= pact_lora_bwd_workspace_bytes(M, N, K, r, nseg), PACT_ERR_INVALID_ARG,
               "pact_lora_bwd: workspace too small");
    PACT_CHECK(g->lddy >= N && g->lddy % 8 == 0 && g->ldu >= 2 * R && g->ldu % 8 == 0 && aligned16(g->dy) &&
                   aligned16(g->A) && aligned16(g->U) && aligned16(g->dA) && aligned16(g->dB) && aligned16(workspace) &&
                   (!g->x || (g->ldx >= K && g->ldx % 8 == 0 && aligned16(g->x))),
               PACT_ERR_ALIGN, "pact_lora_bwd: pointers 16-byte aligned, leading dims %% 8 == 0");
    if (g->xq) {
        pact_status s = check_nvfp4(g->xq, M, K, "xq");
        if (s != PACT_OK) return s;
    }
    cudaStream_t st = (cudaStream_t)stream;
    uint8_t *w8 = static_cast<uint8_t *>(workspace);
    float *tt = reinterpret_cast<float *>(w8);
    float *wda = reinterpret_cast<float *>(w8 + lora_up256((size_t)(M * R * 4)));
    float *wdb = reinterpret_cast<float *>(w8 + lora_up256((size_t)(M * R * 4)) + lora_up256((size_t)(R * K * 4)));
    pact_nvfp4_t none = {nullptr, nullptr, M, K};

    // T~ = X~ . A^T (FP32, unscaled)
    RowArgs a = {};
    a.x = g->x; a.ldx = g->ldx; a.xq = g->xq ? *g->xq : none; a.use_xq = g->xq != nullptr;
    a.M = M; a.K = K; a.w = g->A; a.ldw = K; a.wt = 0; a.R = R; a.r = R; a.nseg = 1; a.seg_end[0] = K;
    a.scale = 1.0f; a.out_bf16 = nullptr; a.out_f32 = tt; a.ldo = R;
    k_rows<<<(unsigned)((M + RT - 1) / RT), 256, 0, st>>>(a);
    pact_status s = launch_status("pact_lora_bwd");
    if (s != PACT_OK) return s;
    if (cudaMemsetAsync(wda, 0, (size_t)(R * K * 4) , st) != cudaSuccess ||
        cudaMemsetAsync(wdb, 0, (size_t)(N * r * 4), st) != cudaSuccess)
        return fail(PACT_ERR_CUDA, "pact_lora_bwd: memset failed");
    const unsigned mchunks = (unsigned)((M + MCHUNK - 1) / MCHUNK);
    // dA = U^T . X~   [R x K]
    OuterArgs o = {};
    o.p = g->U; o.ldp = g->ldu; o.p_split = 1; o.q = g->x; o.qq = g->xq ? *g->xq : none; o.q_kind = g->xq ? 1 : 0; o.ldq = g->ldx;
    o.M = M; o.A = R; o.Bn = K; o.segmented = 0; o.ws = wda; o.ldws = K;
    k_outer<<<dim3((unsigned)((R + TA - 1) / TA), (unsigned)((K + TB - 1) / TB), mchunks), 256, 0, st>>>(o);
    // dB = dY^T . T~ (segment-wise)   [N x r]
    OuterArgs b = {};
    b.p = g->dy; b.ldp = g->lddy; b.qf = tt; b.q_kind = 2; b.ldq = R;
    b.M = M; b.A = N; b.Bn = r; b.segmented = 1; b.r = r; b.nseg = nseg;
    for (int i = 0; i < 4; ++i) b.seg_end[i] = i < nseg ? g->seg_end[i] : N;
    b.ws = wdb; b.ldws = r;
    k_outer<<<dim3((unsigned)((N + TA - 1) / TA), (unsigned)((r + TB - 1) / TB), mchunks), 256, 0, st>>>(b);
    k_finalize<<<256, 256, 0, st>>>(wda, R, K, 1.0f, g->dA, K);
    k_finalize<<<256, 256, 0, st>>>(wdb, N, r, g->scale, g->dB, r);
    return launch_status("pact_lora_bwd");
}

}  // extern "C"
