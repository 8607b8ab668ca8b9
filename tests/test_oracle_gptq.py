"""Pins of the oracle's NVFP4-adapted GPTQ calibration (CPU): the reduction to plain
round-to-nearest quantization under a diagonal Hessian, agreement with the textbook
optimal-brain-surgeon form of the sequential update (explicit inverses of the
Hessian restricted to the columns not yet quantized, instead of the Cholesky
factor), a lower layer loss than round-to-nearest, and GPTQ's dead-column rule."""
import numpy as np

import synth
from oracle import gptq


def _unpack(q):
    c = np.empty((q.rows, q.cols), dtype=np.uint8)
    c[:, 0::2] = q.codes & 0xF
    c[:, 1::2] = q.codes >> 4
    return c


def test_diagonal_hessian_is_round_to_nearest(orc):
    """One-hot calibration rows make X~^T X~ diagonal, so no error is pushed to other
    columns and GPTQ's codes and scales are the plain quantizer's."""
    K = 64
    x = np.zeros((K, K))
    for i in range(K):
        x[i, i] = 1.0 + (i % 5) * 0.25
    xb = synth.f64_to_bf16_bits(x)
    w = synth.weight_bf16(42, (24, K))
    q, _ = gptq.gptq_nvfp4(w, xb)
    ref = orc.quantize(w)
    assert np.array_equal(q.codes, ref.codes) and np.array_equal(q.scales, ref.scales)


def _obs_reference(orc, w_bits, x_bits, damp=0.01):
    """Sequential quantization with the optimal-brain-surgeon update written with an
    explicit inverse of the Hessian restricted to the remaining columns F = j..K-1:
    W[:, F] -= (w_j - q_j) / Hinv_F[0, 0] * Hinv_F[0, :]."""
    W = synth.bf16_bits_to_f64(w_bits).copy()
    N, K = W.shape
    xt = orc.dequantize(orc.quantize(x_bits))
    H = 2.0 * (xt.T @ xt) / xt.shape[0]
    H = H + damp * np.mean(np.diag(H)) * np.eye(K)
    codes = np.zeros((N, K), dtype=np.uint8)
    scales = np.zeros((N, K // 16), dtype=np.uint8)
    grid = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    for j in range(K):
        if j % 16 == 0:
            for n in range(N):
                scales[n, j // 16] = orc.e4m3_rne_sat(float(np.max(np.abs(W[n, j:j + 16]))) / 6.0)
        q = np.zeros(N)
        for n in range(N):
            s = orc.e4m3_value(int(scales[n, j // 16]))
            mag = 0 if s == 0.0 else orc.e2m1_rne_mag(abs(W[n, j]) / s)
            codes[n, j] = (8 if np.signbit(W[n, j]) else 0) | mag
            q[n] = (-grid[mag] if np.signbit(W[n, j]) else grid[mag]) * s
        Hinv_F = np.linalg.inv(H[j:, j:])
        W[:, j:] -= np.outer((W[:, j] - q) / Hinv_F[0, 0], Hinv_F[0, :])
    return codes, scales


def test_matches_the_explicit_inverse_form(orc):
    for seed in (43, 44):
        w = synth.weight_bf16(seed, (6, 48))
        x = synth.gaussian_bf16(seed + 100, (96, 48))
        q, _ = gptq.gptq_nvfp4(w, x)
        codes, scales = _obs_reference(orc, w, x)
        assert np.array_equal(_unpack(q), codes)
        assert np.array_equal(q.scales, scales)


def test_lower_layer_loss_than_round_to_nearest(orc):
    for seed in (45, 46, 47):
        w = synth.weight_bf16(seed, (32, 128), outliers=(seed == 47))
        x = synth.gaussian_bf16(seed + 100, (256, 128))
        q, _ = gptq.gptq_nvfp4(w, x)
        assert gptq.layer_loss(w, q, x) < 0.9 * gptq.layer_loss(w, orc.quantize(w), x)


def test_dead_columns_are_zeroed(orc):
    K = 32
    x = synth.gaussian_bf16(48, (64, K))
    x[:, 5] = 0                       # BF16 +0: no calibration input reaches column 5
    w = synth.weight_bf16(49, (8, K))
    q, W = gptq.gptq_nvfp4(w, x)
    assert np.all(W[:, 5] == 0.0)
    assert np.all(_unpack(q)[:, 5] == 0)


def test_hessian_of_exact_inputs(orc):
    """Inputs already on the NVFP4 grid reconstruct exactly, so H = 2 X^T X / n."""
    x = np.where(np.random.default_rng(50).random((40, 32)) < 0.5, -6.0, 6.0)
    xb = synth.f64_to_bf16_bits(x)
    H = gptq.reconstructed_hessian(xb)
    np.testing.assert_allclose(H, 2.0 * (x.T @ x) / 40, rtol=0, atol=0)
