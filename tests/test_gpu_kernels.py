"""Parity of every libpact kernel with the CPU oracle (needs a B200).

Integer outputs (NVFP4 codes and scales, padding included) must match bit for bit;
floating-point outputs must satisfy |gpu - oracle| <= 8e-3 |oracle| + 1e-3 rms(oracle).
Stages are teacher-forced: each kernel is compared with the oracle run on the GPU
kernel's own inputs.  Sizes span several tiles and ragged tails.
"""
import numpy as np
import pytest
import torch

import synth
from tests.util import assert_close, assert_nvfp4_equal, nvfp4_host, to_bits, to_dev, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def P():
    import nvfp4_gemm_b200 as p
    return p


def sync():
    torch.cuda.synchronize()


def status_ok(P):
    assert P.pact_get_device_status() == 0, P.pact_last_error()


# --------------------------------------------------------------------- quantize
def _positive_bf16():
    bits = np.arange(1, 0x7F80, dtype=np.uint16)
    return bits, synth.bf16_bits_to_f64(bits)


def test_quantize_all_scales(P, orc):
    """Every finite positive BF16 amax, as a block [amax, 0, ...]: scale and codes
    bit-exact (pins the E4M3 decision of the device path exhaustively)."""
    bits, _ = _positive_bf16()
    blocks = np.zeros((bits.size, 64), dtype=np.uint16)
    blocks[:, 0] = bits
    blocks[:, 17] = bits | 0x8000
    dev = P.pact_quantize_nvfp4(to_dev(blocks))
    sync()
    assert_nvfp4_equal(dev, orc.quantize(blocks), orc, "all scales")


def test_quantize_all_elements(P, orc):
    """Every E4M3 scale s and every BF16 |x| <= 6s, both signs, in blocks that force
    the scale to s: codes bit-exact, every tie included."""
    bits, vals = _positive_bf16()
    rows = []
    for sb in range(0, 0x7F):
        s = orc.e4m3_value(sb)
        head = synth.f64_to_bf16_bits(np.array([6.0 * s]))[0] if sb else np.uint16(0)
        sel = vals <= 6.0 * s if sb else vals < 6 * 2.0 ** -10
        xb = np.concatenate([bits[sel], bits[sel] | np.uint16(0x8000), [0x8000]])
        xb = np.concatenate([xb, np.zeros((-xb.size) % 15, dtype=np.uint16)])
        blk = np.empty((xb.size // 15, 16), dtype=np.uint16)
        blk[:, 0] = head
        blk[:, 1:] = xb.reshape(-1, 15)
        rows.append(blk)
    blocks = np.concatenate(rows)
    blocks = np.concatenate([blocks, np.zeros(((-blocks.shape[0]) % 4, 16), dtype=np.uint16)])
    x = blocks.reshape(-1, 64)
    dev = P.pact_quantize_nvfp4(to_dev(x))
    sync()
    assert_nvfp4_equal(dev, orc.quantize(x), orc, "all elements")


@pytest.mark.parametrize("rows,cols,ld", [(1, 64, 64), (200, 320, 320), (300, 1024, 1088), (128, 256, 256),
                                          (2048, 2048, 2048)])
def test_quantize_shapes(P, orc, guards, rows, cols, ld):
    x = synth.gaussian_bf16(1, (rows, ld), std=2.0)
    xd = to_dev(x)[:, :cols]
    dev = P.pact_quantize_nvfp4(xd, out=guards.nvfp4(rows, cols))
    sync()
    assert_nvfp4_equal(dev, orc.quantize(x[:, :cols]), orc, f"quantize {rows}x{cols}")


# ------------------------------------------------------------------ weight cache
@pytest.mark.parametrize("N,K", [(64, 64), (512, 512), (448, 320), (2048, 512), (384, 2048)])
def test_weight_layout_cache(P, orc, N, K):
    w = synth.weight_bf16(0, (N, K), outliers=True)
    wc = P.pact_weight_layout_cache(to_dev(w))
    sync()
    wf, wb = orc.weight_cache(w)
    assert_nvfp4_equal(wc.fwd, wf, orc, "fwd layout")
    assert_nvfp4_equal(wc.bwd, wb, orc, "bwd layout")


# ------------------------------------------------------------------------- GEMM
def _nvfp4_from_oracle(P, t, orc):
    """Upload an oracle NVFP4 tensor (codes + packed scales) to the device."""
    d = P.NVFP4Tensor.empty(t.rows, t.cols)
    d.codes.copy_(torch.from_numpy(t.codes))
    d.scales.copy_(torch.from_numpy(orc.pack_scales(t.scales, t.rows, t.cols)))
    return d


@pytest.mark.parametrize("N,K", [(512, 512), (448, 576), (2048, 1024)])
def test_gemm_one_hot(P, orc, N, K):
    """X rows 6 e_i (scale 1, code 7): Y row = 6 deq(W_fwd)[:, i] exactly in BF16; the
    same for dgrad with the backward layout.  Pins indexing, nibble order and the
    scale layout as the tensor core reads it."""
    w = synth.weight_bf16(1, (N, K))
    wc = P.pact_weight_layout_cache(to_dev(w))
    wf, wb = orc.weight_cache(w)
    rng = np.random.default_rng(0)
    M = 256
    for lay, (rows, cols) in ((wf, (N, K)), (wb, (K, N))):
        idx = rng.integers(0, cols, size=M)
        x = np.zeros((M, cols), dtype=np.uint16)
        x[np.arange(M), idx] = synth.f64_to_bf16_bits(np.array([6.0]))[0]
        xq = P.pact_quantize_nvfp4(to_dev(x))
        if lay is wf:
            y = P.pact_frozen_gemm_fwd(xq, wc)
        else:
            y = P.pact_frozen_gemm_dgrad(xq, wc)
        sync()
        want = 6.0 * orc.dequantize(lay)[:, idx].T
        assert np.array_equal(to_f64(y), want)


GEMM_SHAPES = [(256, 512, 512), (300, 640, 576), (128, 256, 64), (1, 320, 448), (513, 1024, 2048)]


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_gemm_fwd(P, orc, guards, M, N, K):
    x = synth.gaussian_bf16(1, (M, K))
    w = synth.weight_bf16(0, (N, K))
    wc = P.pact_weight_layout_cache(to_dev(w))
    xq = P.pact_quantize_nvfp4(to_dev(x))
    y = P.pact_frozen_gemm_fwd(xq, wc, y=guards.matrix(M, N, pad_cols=8))
    sync()
    status_ok(P)
    wf, _ = orc.weight_cache(w)
    assert_close(to_f64(y), orc.nvfp4_gemm(orc.quantize(x), wf), "fwd")


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_gemm_dgrad(P, orc, guards, M, N, K):
    dy = synth.gaussian_bf16(50, (M, N))
    w = synth.weight_bf16(0, (N, K))
    wc = P.pact_weight_layout_cache(to_dev(w))
    dyq = P.pact_quantize_nvfp4(to_dev(dy))
    dx = P.pact_frozen_gemm_dgrad(dyq, wc, dx=guards.matrix(M, K, pad_cols=16))
    sync()
    _, wb = orc.weight_cache(w)
    assert_close(to_f64(dx), orc.frozen_dgrad(dy, wb), "dgrad")


def test_gemm_fwd_residual(P, orc, guards):
    M, N, K = 300, 768, 512
    x = synth.gaussian_bf16(1, (M, K))
    res = synth.gaussian_bf16(2, (M, N))
    w = synth.weight_bf16(0, (N, K))
    wc = P.pact_weight_layout_cache(to_dev(w))
    y = P.pact_frozen_gemm_fwd(P.pact_quantize_nvfp4(to_dev(x)), wc, residual=to_dev(res),
                               y=guards.matrix(M, N, pad_cols=64))
    sync()
    wf, _ = orc.weight_cache(w)
    assert_close(to_f64(y), orc.nvfp4_gemm(orc.quantize(x), wf) + synth.bf16_bits_to_f64(res), "fwd + residual")


def test_gemm_dgrad_accumulate(P, orc):
    M, N, K = 256, 512, 768
    dy = synth.gaussian_bf16(50, (M, N))
    base = synth.gaussian_bf16(2, (M, K))
    w = synth.weight_bf16(0, (N, K))
    wc = P.pact_weight_layout_cache(to_dev(w))
    dx = to_dev(base)
    P.pact_frozen_gemm_dgrad(P.pact_quantize_nvfp4(to_dev(dy)), wc, residual=dx, dx=dx)
    sync()
    _, wb = orc.weight_cache(w)
    assert_close(to_f64(dx), orc.frozen_dgrad(dy, wb) + synth.bf16_bits_to_f64(base), "dgrad accumulate")


def _segments(N, parts):
    ends, acc = [], 0
    for p_ in parts:
        acc += p_
        ends.append(acc)
    assert acc == N
    return ends


@pytest.mark.parametrize("M,parts,K,r", [(256, [512], 512, 16), (300, [512, 256, 256], 576, 16),
                                         (200, [256, 320], 256, 16), (130, [768], 320, 48)])
def test_gemm_fwd_lora(P, orc, M, parts, K, r):
    N = sum(parts)
    seg_end = _segments(N, parts)
    x = synth.gaussian_bf16(1, (M, K))
    w = synth.weight_bf16(0, (N, K))
    nseg = len(parts)
    a = synth.gaussian_bf16(20, (nseg * r, K), std=0.02)
    b = synth.gaussian_bf16(30, (N, r), std=0.02)
    s = 2.0
    wc = P.pact_weight_layout_cache(to_dev(w))
    xd = to_dev(x)
    xq = P.pact_quantize_nvfp4(xd)
    T = P.pact_lora_fwd(xd, to_dev(a), s)
    bd = to_dev(b)
    y = P.pact_frozen_gemm_fwd(xq, wc, lora=P.lora_struct(T, bd, r, seg_end))
    sync()
    # oracle, teacher-forced on the device's T (T = hi + lo)
    wf, _ = orc.weight_cache(w)
    ref = orc.nvfp4_gemm(orc.quantize(x), wf)
    R = nseg * r
    t_dev = to_f64(T[:, :R]) + to_f64(T[:, R:])
    bb = synth.bf16_bits_to_f64(b)
    lo = 0
    for i, hi in enumerate(seg_end):
        ref[:, lo:hi] += orc.gemm_nt(t_dev[:, i * r:(i + 1) * r], bb[lo:hi])
        lo = hi
    assert_close(to_f64(y), ref, "fwd + LoRA")
    # and T itself against the oracle's scale * X A^T
    assert_close(t_dev, s * orc.lora_t(synth.bf16_bits_to_f64(x), a), "T")


@pytest.mark.parametrize("M,N,K,R", [(256, 512, 512, 16), (300, 640, 576, 48), (130, 256, 320, 32)])
def test_gemm_dgrad_lora(P, orc, M, N, K, R):
    dy = synth.gaussian_bf16(50, (M, N))
    w = synth.weight_bf16(0, (N, K))
    a = synth.gaussian_bf16(20, (R, K), std=0.02)
    u = np.concatenate([synth.gaussian_bf16(31, (M, R), std=0.5), synth.gaussian_bf16(32, (M, R), std=1e-3)], 1)
    wc = P.pact_weight_layout_cache(to_dev(w))
    dyq = P.pact_quantize_nvfp4(to_dev(dy))
    ud, ad = to_dev(u), to_dev(a)
    dx = P.pact_frozen_gemm_dgrad(dyq, wc, lora=P.lora_struct(ud, ad, R, [K]))
    sync()
    _, wb = orc.weight_cache(w)
    uf = synth.bf16_bits_to_f64(u)
    ref = orc.frozen_dgrad(dy, wb) + orc.gemm_nt(uf[:, :R] + uf[:, R:], synth.bf16_bits_to_f64(a).T)
    assert_close(to_f64(dx), ref, "dgrad + LoRA")


@pytest.mark.parametrize("M,parts,K,lora", [(300, [512, 256], 512, False), (130, [768], 320, True),
                                             (2048, [1024, 1024], 256, True), (64, [256, 1280], 192, False)])
def test_gemm_fwd_quant(P, orc, guards, M, parts, K, lora):
    """The forward GEMM that also writes the NVFP4 copy of its BF16 output, split along
    the columns: the copy equals the quantizer's on the device's own y (bit-exact,
    padding scales included), y is as pact_frozen_gemm_fwd's."""
    N = sum(parts)
    x = synth.gaussian_bf16(1, (M, K))
    w = synth.weight_bf16(0, (N, K), outliers=True)
    wc = P.pact_weight_layout_cache(to_dev(w))
    xq = P.pact_quantize_nvfp4(to_dev(x))
    lo = None
    if lora:
        r = 16
        a = synth.gaussian_bf16(20, (len(parts) * r, K), std=0.02)
        b = synth.gaussian_bf16(30, (N, r), std=0.02)
        T = P.pact_lora_fwd(to_dev(x), to_dev(a), 2.0)
        lo = P.lora_struct(T, to_dev(b), r, _segments(N, parts))
    yq = [guards.nvfp4(M, c) for c in parts]
    y = P.pact_frozen_gemm_fwd_quant(xq, wc, yq, lora=lo, y=guards.matrix(M, N, pad_cols=8))
    y_ref = P.pact_frozen_gemm_fwd(xq, wc, lora=lo)
    sync()
    status_ok(P)
    assert torch.equal(y.contiguous().view(torch.int16), y_ref.view(torch.int16))
    yb = to_bits(y)
    c0 = 0
    for t, c in zip(yq, parts):
        assert_nvfp4_equal(t, orc.quantize(yb[:, c0:c0 + c]), orc, f"q(y) columns {c0}..{c0 + c}")
        c0 += c
    if not lora:
        wf, _ = orc.weight_cache(w)
        assert_close(to_f64(y), orc.nvfp4_gemm(orc.quantize(x), wf), "fwd")


@pytest.mark.parametrize("M,I,K,lora,two_level", [(300, 256, 512, False, False), (130, 512, 320, True, False),
                                                   (2048, 768, 256, True, True), (1, 256, 192, False, False),
                                                   (4096, 1280, 640, True, False)])
def test_gemm_fwd_silu(P, orc, guards, M, I, K, lora, two_level):
    """The gate|up GEMM with the SiLU-multiply in its epilogue: m, mq, gq, uq equal the
    oracle's SiLU-multiply of the plain GEMM's g|u (which the fused kernel computes with
    the same instructions) bit for bit, padding scales included; nothing past m's row
    ends or past the copies' buffers is written."""
    N = 2 * I
    x = synth.gaussian_bf16(1, (M, K))
    w = synth.weight_bf16(0, (N, K), outliers=True)
    wc = P.pact_weight_layout_cache(to_dev(w), two_level=two_level)
    xq = P.pact_quantize_nvfp4(to_dev(x))
    lo = None
    if lora:
        r = 16
        a = synth.gaussian_bf16(20, (2 * r, K), std=0.02)
        b = synth.gaussian_bf16(30, (N, r), std=0.02)
        T = P.pact_lora_fwd(to_dev(x), to_dev(a), 2.0 * 2.0 ** -wc.gexp)
        lo = P.lora_struct(T, to_dev(b), r, [I, N])
    m = guards.matrix(M, I, pad_cols=8)
    mq, gq, uq = guards.nvfp4(M, I), guards.nvfp4(M, I), guards.nvfp4(M, I)
    P.pact_frozen_gemm_fwd_silu(xq, wc, m, mq, gq, uq, lora=lo)
    gu = P.pact_frozen_gemm_fwd(xq, wc, lora=lo)
    sync()
    status_ok(P)
    gub = to_bits(gu)
    m_ref, mq_ref, gq_ref, uq_ref = orc.silu_mul_quant(gub[:, :I], gub[:, I:])
    assert np.array_equal(to_bits(m), m_ref), "m"
    assert_nvfp4_equal(mq, mq_ref, orc, "mq")
    assert_nvfp4_equal(gq, gq_ref, orc, "gq")
    assert_nvfp4_equal(uq, uq_ref, orc, "uq")
    if not lora and not two_level:
        wf, _ = orc.weight_cache(w)
        assert_close(to_f64(gu), orc.nvfp4_gemm(orc.quantize(x), wf), "g|u")


def test_gemm_fwd_silu_rejects_bad_shapes(P):
    """I must be a multiple of 256 (the gate and up tiles pair up); the copies must
    be [M x I]."""
    x = torch.zeros((64, 128), dtype=torch.bfloat16, device="cuda")
    xq = P.pact_quantize_nvfp4(x)
    wc = P.pact_weight_layout_cache(torch.zeros((2 * 320, 128), dtype=torch.bfloat16, device="cuda"))
    m = torch.empty((64, 320), dtype=torch.bfloat16, device="cuda")
    q = [P.NVFP4Tensor.empty(64, 320, torch.device("cuda")) for _ in range(3)]
    with pytest.raises(P.PactError):
        P.pact_frozen_gemm_fwd_silu(xq, wc, m, *q)
    wc = P.pact_weight_layout_cache(torch.zeros((512, 128), dtype=torch.bfloat16, device="cuda"))
    q = [P.NVFP4Tensor.empty(64, 128, torch.device("cuda")) for _ in range(3)]
    with pytest.raises(P.PactError):
        P.pact_frozen_gemm_fwd_silu(xq, wc, torch.empty((64, 256), dtype=torch.bfloat16, device="cuda"), *q)
    sync()
    status_ok(P)


# ------------------------------------------------------------------------- LoRA
def test_lora_products_with_one_split(P, orc, guards):
    """T = s X A^T and U = s dY B with enough 128-row output blocks (150 >= the SM
    count) that the contraction is not split: the MMA kernel then writes the hi + lo
    output itself (no finalize launch).  Compared with the oracle through hi + lo."""
    r, s = 16, 2.0
    M, K, R = 19200, 128, 48
    x = synth.gaussian_bf16(1, (M, K))
    a = synth.gaussian_bf16(20, (R, K), std=0.02)
    T = P.pact_lora_fwd(to_dev(x), to_dev(a), s, T=guards.matrix(M, 2 * R, pad_cols=8))
    Mu, parts = 6400, [256, 256, 512]
    N = sum(parts)
    seg_end = _segments(N, parts)
    dy = synth.gaussian_bf16(50, (Mu, N))
    b = synth.gaussian_bf16(30, (N, r), std=0.02)
    U = P.pact_lora_bwd_u(to_dev(dy), to_dev(b), r, seg_end, s, U=guards.matrix(Mu, 2 * 3 * r, pad_cols=8))
    sync()
    t_dev = to_f64(T[:, :R]) + to_f64(T[:, R:])
    assert_close(t_dev, s * orc.gemm_nt(synth.bf16_bits_to_f64(x), synth.bf16_bits_to_f64(a)), "T")
    dyf, bf = synth.bf16_bits_to_f64(dy), synth.bf16_bits_to_f64(b)
    u_ref = np.zeros((Mu, 3 * r))
    lo = 0
    for i, hi in enumerate(seg_end):
        u_ref[:, i * r:(i + 1) * r] = s * orc.gemm_nt(dyf[:, lo:hi], bf[lo:hi].T)
        lo = hi
    assert_close(to_f64(U[:, :3 * r]) + to_f64(U[:, 3 * r:]), u_ref, "U")


# the LoRA products that also write the NVFP4 copy of their streamed input: split
# contractions (small M) and unsplit ones (M with >= 148 row blocks), ragged rows
@pytest.mark.parametrize("M,K,R", [(300, 576, 48), (129, 128, 16), (19200, 192, 32)])
def test_lora_fwd_quant(P, orc, guards, M, K, R):
    x = synth.gaussian_bf16(1, (M, K))
    a = synth.gaussian_bf16(20, (R, K), std=0.02)
    xd, ad = to_dev(x), to_dev(a)
    xq = guards.nvfp4(M, K)
    T = P.pact_lora_fwd(xd, ad, 2.0, T=guards.matrix(M, 2 * R, pad_cols=8), xq=xq)
    T_ref = P.pact_lora_fwd(xd, ad, 2.0)
    sync()
    assert torch.equal(T.contiguous().view(torch.int16), T_ref.view(torch.int16))
    assert_nvfp4_equal(xq, orc.quantize(x), orc, "q(x)")


@pytest.mark.parametrize("M,parts,r", [(300, [512, 256, 256], 16), (130, [320], 32), (6400, [256, 256, 512], 16)])
def test_lora_bwd_u_quant(P, orc, guards, M, parts, r):
    N = sum(parts)
    seg_end = _segments(N, parts)
    dy = synth.gaussian_bf16(50, (M, N))
    b = synth.gaussian_bf16(30, (N, r), std=0.02)
    dyd, bd = to_dev(dy), to_dev(b)
    dyq = guards.nvfp4(M, N)
    U = P.pact_lora_bwd_u(dyd, bd, r, seg_end, 2.0, U=guards.matrix(M, 2 * len(parts) * r, pad_cols=8), dyq=dyq)
    U_ref = P.pact_lora_bwd_u(dyd, bd, r, seg_end, 2.0)
    sync()
    assert torch.equal(U.contiguous().view(torch.int16), U_ref.view(torch.int16))
    assert_nvfp4_equal(dyq, orc.quantize(dy), orc, "q(dY)")


@pytest.mark.parametrize("M,parts,r,K", [(256, [512], 16, 384), (300, [512, 256, 256], 16, 576),
                                         (130, [256, 320], 32, 320), (2048, [1024], 16, 2112)])
def test_lora_bwd(P, orc, guards, M, parts, r, K):
    """dA and dB from BF16 X and from the NVFP4 copy of X (decoded inside the MMA
    kernel); K values that end mid-way through a 128-feature tile and token counts
    that end mid-way through a 128-token scale group cover the ragged edges."""
    N = sum(parts)
    seg_end = _segments(N, parts)
    nseg = len(parts)
    dy = synth.gaussian_bf16(50, (M, N))
    x = synth.gaussian_bf16(1, (M, K))
    a = synth.gaussian_bf16(20, (nseg * r, K), std=0.02)
    b = synth.gaussian_bf16(30, (N, r), std=0.02)
    s = 2.0
    dyd, xd, ad, bd = to_dev(dy), to_dev(x), to_dev(a), to_dev(b)
    U = P.pact_lora_bwd_u(dyd, bd, r, seg_end, s, U=guards.matrix(M, 2 * nseg * r, pad_cols=8))
    dA, dB = P.pact_lora_bwd(dyd, ad, U, r, seg_end, s, x=xd, dA=guards.matrix(nseg * r, K), dB=guards.matrix(N, r))
    xq = P.pact_quantize_nvfp4(xd)
    dA2, dB2 = P.pact_lora_bwd(dyd, ad, U, r, seg_end, s, xq=xq, dA=guards.matrix(nseg * r, K),
                               dB=guards.matrix(N, r))
    # FP32 gradients (for a sum over replicas) round to the BF16 ones bit for bit
    dA3, dB3 = P.pact_lora_bwd(dyd, ad, U, r, seg_end, s, xq=xq, grads_fp32=True)
    sync()
    assert dA3.dtype == torch.float32 and dB3.dtype == torch.float32
    for g32, g16 in ((dA3, dA2), (dB3, dB2)):
        assert torch.equal(P.pact_round_bf16(g32.contiguous()).view(torch.int16), g16.view(torch.int16))
    dyf, xf = synth.bf16_bits_to_f64(dy), synth.bf16_bits_to_f64(x)
    af, bf = synth.bf16_bits_to_f64(a), synth.bf16_bits_to_f64(b)
    R = nseg * r
    u_dev = to_f64(U[:, :R]) + to_f64(U[:, R:])
    lo = 0
    u_ref = np.zeros((M, nseg * r))
    for i, hi in enumerate(seg_end):
        u_ref[:, i * r:(i + 1) * r] = s * orc.gemm_nt(dyf[:, lo:hi], bf[lo:hi].T)
        lo = hi
    assert_close(u_dev, u_ref, "U")
    for xt, gA, gB, what in ((xf, dA, dB, "bf16 x"), (orc.dequantize(orc.quantize(x)), dA2, dB2, "nvfp4 x")):
        # dA from the device's U (teacher-forced), dB per segment
        assert_close(to_f64(gA), orc.gemm_nt(u_dev.T, xt.T), f"dA ({what})")
        db_ref = np.zeros((N, r))
        lo = 0
        for i, hi in enumerate(seg_end):
            _, db_i, _ = orc.lora_bwd_at(dyf[:, lo:hi], xt, af[i * r:(i + 1) * r], bf[lo:hi], s)
            db_ref[lo:hi] = db_i
            lo = hi
        assert_close(to_f64(gB), db_ref, f"dB ({what})")


# --------------------------------------------------------------- fused producers
# several rows per CTA ring (one row slot per row in flight), ragged row counts; 16384
# is the widest row the entry point accepts
@pytest.mark.parametrize("M,H", [(64, 512), (257, 2048), (96, 3072), (33, 1536), (40, 4096), (24, 8192),
                                 (9, 16384)])
def test_rmsnorm_quant(P, orc, guards, M, H):
    x = synth.gaussian_bf16(1, (M, H))
    g = synth.gaussian_bf16(40, (H,), std=0.02, mean=1.0)
    yq, y, rstd = P.pact_rmsnorm_quant(to_dev(x), to_dev(g), 1e-5, yq=guards.nvfp4(M, H), y=guards.matrix(M, H),
                                       rstd=guards.matrix(1, M, torch.float32)[0])
    sync()
    y_ref, yq_ref, rstd_ref = orc.rmsnorm_quant(x, g, 1e-5)
    yb = to_bits(y)
    assert np.array_equal(yb, y_ref), f"y differs at {np.argwhere(yb != y_ref)[:3].tolist()}"
    assert_nvfp4_equal(yq, yq_ref, orc, "yq")
    np.testing.assert_allclose(rstd.cpu().numpy(), rstd_ref, rtol=1e-7)


def _special_rows(H, eps):
    """BF16 rows at the edges of RMSNorm's arithmetic: all zeros (eps > 0 only: with eps
    = 0 the result is 0 * inf), subnormals only (with eps = 0 the rstd of the second
    such row lies beyond FP32's range), tiny and huge normal values, a single non-zero
    value, subnormals with one normal value, and two ordinary rows."""
    g = synth.gaussian_bf16(3, (8, H)).astype(np.uint16)
    u = synth.uniform(77, 2 * H)
    sign = np.where(u[H:] < 0.5, 0x8000, 0)
    sub = ((1 + np.floor(u[:H] * 127)).astype(np.uint16) | sign).astype(np.uint16)
    sub_small = ((1 + np.floor(u[:H] * 7)).astype(np.uint16) | sign).astype(np.uint16)
    f32 = lambda a: synth.f64_to_bf16_bits(np.asarray(a, dtype=np.float64))
    rows = [np.zeros(H, np.uint16) if eps > 0 else g[0],
            sub,
            f32(synth.bf16_bits_to_f64(g[1]) * 2.0 ** -100),
            f32(synth.bf16_bits_to_f64(g[2]) * 2.0 ** 60),
            np.where(np.arange(H) == H // 3, g[3], 0).astype(np.uint16),
            np.where(np.arange(H) == 5, g[4], sub).astype(np.uint16),
            g[5], g[6], sub_small]
    return np.stack(rows)


@pytest.mark.parametrize("H", [3072, 8192])
@pytest.mark.parametrize("eps", [1e-5, 0.0])
def test_rmsnorm_quant_special_rows(P, orc, guards, H, eps):
    x = _special_rows(H, eps)
    M = x.shape[0]
    g = synth.gaussian_bf16(40, (H,), std=0.02, mean=1.0)
    yq, y, rstd = P.pact_rmsnorm_quant(to_dev(x), to_dev(g), eps, yq=guards.nvfp4(M, H), y=guards.matrix(M, H),
                                       rstd=guards.matrix(1, M, torch.float32)[0])
    sync()
    # the entry point takes eps as FP32: the oracle gets that value (rows of zeros and
    # subnormals have rstd = 1/sqrt(eps), which tells 1e-5 from FP32(1e-5))
    y_ref, yq_ref, rstd_ref = orc.rmsnorm_quant(x, g, float(np.float32(eps)))
    yb = to_bits(y)
    assert np.array_equal(yb, y_ref), f"y differs at {np.argwhere(yb != y_ref)[:3].tolist()}"
    assert_nvfp4_equal(yq, yq_ref, orc, "yq")
    with np.errstate(over="ignore"):   # the kernel writes rstd as FP32: beyond its range, inf
        np.testing.assert_array_equal(rstd.cpu().numpy(), rstd_ref.astype(np.float32))


@pytest.mark.parametrize("H", [3072, 8192])
def test_rmsnorm_quant_nonfinite_rows(P, orc, H):
    """An infinity or a NaN in a row makes rstd 0 or NaN: y is then 0 where x is finite
    and NaN elsewhere (compared as NaN, whatever its payload)."""
    x = synth.gaussian_bf16(5, (4, H)).astype(np.uint16)
    x[0, 7] = 0x7F80        # +inf
    x[1, H - 1] = 0xFF80    # -inf
    x[2, 100] = 0x7FC1      # NaN
    g = synth.gaussian_bf16(40, (H,), std=0.02, mean=1.0)
    _, y, rstd = P.pact_rmsnorm_quant(to_dev(x), to_dev(g), 1e-5)
    sync()
    y_ref, _, rstd_ref = orc.rmsnorm_quant(x, g, float(np.float32(1e-5)))
    got, want = synth.bf16_bits_to_f64(to_bits(y)), synth.bf16_bits_to_f64(y_ref)
    assert np.array_equal(np.isnan(got), np.isnan(want))
    ok = ~np.isnan(want)
    assert np.array_equal(to_bits(y)[ok], y_ref[ok])
    np.testing.assert_array_equal(rstd.cpu().numpy(), rstd_ref.astype(np.float32))


@pytest.mark.parametrize("M,I,std", [(64, 512, 2.0), (130, 8960, 2.0), (257, 2048, 2.0), (96, 2048, 9.0)])
def test_silu_mul_quant(P, orc, guards, M, I, std):
    # std 2 reaches both margins of the rounding check; std 9 also |g| > 16 (FP64 path)
    gu = synth.gaussian_bf16(4, (M, 2 * I), std=std)
    gud = to_dev(gu)
    m, mq, gq, uq = P.pact_silu_mul_quant(gud[:, :I], gud[:, I:], m=guards.matrix(M, I), mq=guards.nvfp4(M, I),
                                          gq=guards.nvfp4(M, I), uq=guards.nvfp4(M, I))
    sync()
    m_ref, mq_ref, gq_ref, uq_ref = orc.silu_mul_quant(gu[:, :I], gu[:, I:])
    mb = to_bits(m)
    assert np.array_equal(mb, m_ref), f"m differs at {np.argwhere(mb != m_ref)[:3].tolist()}"
    assert_nvfp4_equal(mq, mq_ref, orc, "mq")
    assert_nvfp4_equal(gq, gq_ref, orc, "gq")
    assert_nvfp4_equal(uq, uq_ref, orc, "uq")


# m = silu(g) u formed inside the down projection's LoRA kernel: m (when asked), q(m) and
# T = s m A^T, split (small M) and unsplit (>= 148 row blocks), |g| > 16 included (std 9)
@pytest.mark.parametrize("M,I,R,std", [(130, 512, 16, 2.0), (257, 1024, 32, 9.0), (19000, 128, 16, 2.0)])
def test_lora_fwd_silu(P, orc, guards, M, I, R, std):
    gu = synth.gaussian_bf16(4, (M, 2 * I), std=std)
    a = synth.gaussian_bf16(20, (R, I), std=0.02)
    gud, ad = to_dev(gu), to_dev(a)
    mq, m = guards.nvfp4(M, I), guards.matrix(M, I)
    T = P.pact_lora_fwd_silu(gud[:, :I], gud[:, I:], ad, 2.0, mq, T=guards.matrix(M, 2 * R, pad_cols=8), m=m)
    mq2 = P.NVFP4Tensor.empty(M, I)
    T2 = P.pact_lora_fwd_silu(gud[:, :I], gud[:, I:], ad, 2.0, mq2)   # without m: the same mq and T
    sync()
    m_ref, mq_ref, _, _ = orc.silu_mul_quant(gu[:, :I], gu[:, I:])
    mb = to_bits(m)
    assert np.array_equal(mb, m_ref), f"m differs at {np.argwhere(mb != m_ref)[:3].tolist()}"
    assert_nvfp4_equal(mq, mq_ref, orc, "mq")
    assert_nvfp4_equal(mq2, mq_ref, orc, "mq (no m)")
    assert torch.equal(T.contiguous().view(torch.int16), T2.view(torch.int16))
    t_dev = to_f64(T[:, :R]) + to_f64(T[:, R:])
    assert_close(t_dev, 2.0 * orc.gemm_nt(synth.bf16_bits_to_f64(m_ref), synth.bf16_bits_to_f64(a)), "T")


@pytest.mark.parametrize("M,I,std", [(64, 512, 2.0), (130, 2048, 2.0), (96, 1024, 9.0)])
def test_silu_mul_bwd_quant(P, orc, guards, M, I, std):
    gu = synth.gaussian_bf16(4, (M, 2 * I), std=std)
    dm = synth.gaussian_bf16(56, (M, I))
    _, _, gq, uq = orc.silu_mul_quant(gu[:, :I], gu[:, I:])
    gqd, uqd = _nvfp4_from_oracle(P, gq, orc), _nvfp4_from_oracle(P, uq, orc)
    dgu, dguq, m_re = P.pact_silu_mul_bwd_quant(to_dev(dm), gqd, uqd, dgu=guards.matrix(M, 2 * I, pad_cols=64),
                                                dguq=guards.nvfp4(M, 2 * I), m_re=guards.matrix(M, I))
    sync()
    dg_ref, du_ref = orc.silu_mul_bwd(synth.bf16_bits_to_f64(dm), gq, uq)
    dgu_dev = to_f64(dgu)
    assert_close(dgu_dev[:, :I], dg_ref, "dg")
    assert_close(dgu_dev[:, I:], du_ref, "du")
    assert_nvfp4_equal(dguq, orc.quantize(to_bits(dgu)), orc, "q(dg|du)")
    mr = to_bits(m_re)
    want = orc.silu_mul_recompute(gq, uq)
    assert np.array_equal(mr, want), f"m~ differs at {np.argwhere(mr != want)[:3].tolist()}"


# rows of up to 4096 columns take the register-resident kernel, wider ones the ring
@pytest.mark.parametrize("M,H,with_res", [(64, 512, False), (130, 2048, True), (33, 3072, True), (40, 1536, False),
                                          (24, 4096, True), (9, 8192, False)])
def test_rmsnorm_bwd(P, orc, guards, M, H, with_res):
    x = synth.gaussian_bf16(1, (M, H))
    g = synth.gaussian_bf16(40, (H,), std=0.02, mean=1.0)
    dy = synth.gaussian_bf16(57, (M, H))
    res = synth.gaussian_bf16(58, (M, H))
    yq, _, rstd = P.pact_rmsnorm_quant(to_dev(x), to_dev(g), 1e-5)
    dx, dxq = P.pact_rmsnorm_bwd(to_dev(dy), yq, rstd, to_dev(g), dres=to_dev(res) if with_res else None,
                                 dx=guards.matrix(M, H), dxq=guards.nvfp4(M, H))
    sync()
    _, yq_ref, _ = orc.rmsnorm_quant(x, g, 1e-5)
    ref = orc.rmsnorm_bwd(synth.bf16_bits_to_f64(dy), yq_ref, rstd.cpu().numpy().astype(np.float64), g)
    if with_res:
        ref = ref + synth.bf16_bits_to_f64(res)
    assert_close(to_f64(dx), ref, "dx")
    assert_nvfp4_equal(dxq, orc.quantize(to_bits(dx)), orc, "q(dx)")


# ------------------------------------------------------------- host-side errors
def test_errors_leave_nothing_enqueued(P):
    x = torch.zeros((128, 100), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(P.PactError) as e:
        P.pact_quantize_nvfp4(x)
    assert e.value.status == 2
    status_ok(P)


# ------------------------------------------------- one projection, not teacher-forced
@pytest.mark.parametrize("M,N,K", [(256, 512, 512), (300, 768, 320)])
def test_projection_end_to_end(P, orc, M, N, K):
    """Forward, dgrad and dA/dB of one projection with its LoRA branch against the
    fully independent oracle (no device intermediate fed back)."""
    r, s = 16, 2.0
    x = synth.gaussian_bf16(1, (M, K))
    w = synth.weight_bf16(0, (N, K))
    a = synth.gaussian_bf16(20, (r, K), std=0.02)
    b = synth.gaussian_bf16(30, (N, r), std=0.02)
    dy = synth.gaussian_bf16(50, (M, N))
    xd, ad, bd, dyd = to_dev(x), to_dev(a), to_dev(b), to_dev(dy)
    wc = P.pact_weight_layout_cache(to_dev(w))
    T = P.pact_lora_fwd(xd, ad, s)
    y = P.pact_frozen_gemm_fwd(P.pact_quantize_nvfp4(xd), wc, lora=P.lora_struct(T, bd, r, [N]))
    U = P.pact_lora_bwd_u(dyd, bd, r, [N], s)
    dx = P.pact_frozen_gemm_dgrad(P.pact_quantize_nvfp4(dyd), wc, lora=P.lora_struct(U, ad, r, [K]))
    dA, dB = P.pact_lora_bwd(dyd, ad, U, r, [N], s, x=xd)
    sync()
    wf, wb = orc.weight_cache(w)
    assert_close(to_f64(y), orc.frozen_fwd(orc.quantize(x), wf, x, a, b, s), "y")
    assert_close(to_f64(dx), orc.frozen_dgrad(dy, wb, a, b, s), "dx")
    da, db, _ = orc.lora_bwd(dy, synth.bf16_bits_to_f64(x), a, b, s)
    assert_close(to_f64(dA), da, "dA")
    assert_close(to_f64(dB), db, "dB")
