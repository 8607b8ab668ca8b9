"""NVFP4-adapted GPTQ calibration of a frozen weight (test infrastructure only).

PACT calibrates the frozen weights offline with GPTQ adapted to NVFP4 (PACT blog
summary, section "方法" (method), bullet 3; PACT abstract): the statistics come from
the reconstructed NVFP4 inputs, so that the calibration objective matches the
activations the frozen GEMM sees in training, and the weights are quantized into
NVFP4 blocks (16 values along K, one E4M3 scale each).

GPTQ itself is the published algorithm of Frantar et al., "GPTQ: Accurate
Post-Training Quantization for Generative Pre-trained Transformers" (2022): with
H = 2 X^T X / n the layer-wise Hessian of ||X W^T - X Q^T||^2, the columns of W are
quantized one at a time in order, and each column's quantization error is pushed
onto the columns not yet quantized through the upper Cholesky factor U of H^-1
(H^-1 = U^T U): err = (w_j - q_j) / U[j, j];  W[:, j+1:] -= err U[j, j+1:].

Readings (the pages name the method only):
- X~ = deq(q(X)) along K is the "reconstructed NVFP4 input";
- a block's scale is chosen when GPTQ reaches the block's first column, from the
  block's current (error-compensated) weights: E4M3_RNE(amax / 6), the same rule as
  the quantizer's;
- dampening: lambda = 0.01 of the mean diagonal of H is added to the diagonal; a
  column no calibration input touches (H[i, i] = 0) gets H[i, i] = 1 and a zero
  weight, as GPTQ does.
The result is an NVFP4 tensor [N x K] in the layout of weight_cache's forward part.
Everything is float64; numpy's Cholesky factorisation and inverse are library steps.
"""
from __future__ import annotations

import numpy as np

from . import NVFP4, _c, _load, _p, bf16_to_f64, dequantize, e4m3_value, quantize


def _scales(amax: np.ndarray) -> np.ndarray:
    a = _c(amax, np.float64)
    out = np.empty(a.size, dtype=np.uint8)
    if a.size:
        _load().orc_e4m3_scales_f64(_p(a), a.size, _p(out))
    return out


def _codes(x: np.ndarray, sbytes: np.ndarray) -> np.ndarray:
    xv = _c(x, np.float64)
    sb = _c(sbytes, np.uint8)
    out = np.empty(xv.size, dtype=np.uint8)
    if xv.size:
        _load().orc_e2m1_codes_f64(_p(xv), _p(sb), xv.size, _p(out))
    return out


_E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _values(codes: np.ndarray, sbytes: np.ndarray) -> np.ndarray:
    mag = _E2M1[codes & 7]
    s = np.array([e4m3_value(int(b)) for b in sbytes])
    return np.where(codes & 8, -mag, mag) * s


def reconstructed_hessian(x_bits: np.ndarray) -> np.ndarray:
    """H = 2 X~^T X~ / n with X~ = deq(q(X)), X [n x K] BF16 calibration inputs."""
    xt = dequantize(quantize(x_bits))
    return 2.0 * (xt.T @ xt) / xt.shape[0]


def gptq_nvfp4(w_bits: np.ndarray, x_bits: np.ndarray, damp: float = 0.01):
    """Calibrated NVFP4 codes and scales of W [N x K] (BF16) for calibration inputs
    X [n x K] (BF16).  Returns (NVFP4 tensor, the error-compensated float64 weights
    at the end of the pass)."""
    W = bf16_to_f64(w_bits).copy()
    N, K = W.shape
    assert K % 16 == 0
    H = reconstructed_hessian(x_bits)
    dead = np.diag(H) == 0.0
    H[dead, dead] = 1.0
    W[:, dead] = 0.0
    H = H + damp * np.mean(np.diag(H)) * np.eye(K)
    U = np.linalg.cholesky(np.linalg.inv(H)).T          # upper: H^-1 = U^T U
    codes = np.zeros((N, K), dtype=np.uint8)
    scales = np.zeros((N, K // 16), dtype=np.uint8)
    for j in range(K):
        b = j // 16
        if j % 16 == 0:
            scales[:, b] = _scales(np.max(np.abs(W[:, j:j + 16]), axis=1))
        codes[:, j] = _codes(W[:, j], scales[:, b])
        q = _values(codes[:, j], scales[:, b])
        err = (W[:, j] - q) / U[j, j]
        W[:, j + 1:] -= np.outer(err, U[j, j + 1:])
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return NVFP4(packed, scales, N, K), W


def layer_loss(w_bits: np.ndarray, q: NVFP4, x_bits: np.ndarray) -> float:
    """||X~ W^T - X~ deq(Q)^T||_F^2 / n: the objective GPTQ lowers, on the
    reconstructed inputs."""
    xt = dequantize(quantize(x_bits))
    d = xt @ (bf16_to_f64(w_bits) - dequantize(q)).T
    return float(np.sum(d * d) / xt.shape[0])
