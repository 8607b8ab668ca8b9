"""The GEMM shape sweep (six N x K weight shapes, forward and dgrad) against the
oracle at full size, on sampled rows the oracle computes one by one.

Quantization is row-local (blocks of 16 along the contraction), so the oracle
quantizes only the sampled rows of X (or dY) and multiplies them by its dequantized
weight layouts; the GPU runs the whole GEMM through the C ABI in the launch
configuration bench.py --sweep times.  M = 512 and M = 8192 cover a partial wave and
several waves of 256 x 256 pair tiles."""
import numpy as np
import pytest
import torch

import synth
from tests.util import assert_close, to_dev, to_f64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("N,K", synth.SWEEP_NK)
def test_sweep_shape_sampled_rows(orc, N, K):
    import nvfp4_gemm_b200 as P
    w = synth.weight_bf16(0, (N, K))
    wc = P.pact_weight_layout_cache(to_dev(w))
    wf, wb = orc.weight_cache(w)
    rng = np.random.default_rng(N * 7 + K)
    for M in (512, 8192):
        x = synth.gaussian_bf16(1, (M, K))
        dy = synth.gaussian_bf16(50, (M, N))
        y = P.pact_frozen_gemm_fwd(P.pact_quantize_nvfp4(to_dev(x)), wc)
        dx = P.pact_frozen_gemm_dgrad(P.pact_quantize_nvfp4(to_dev(dy)), wc)
        torch.cuda.synchronize()
        assert P.pact_get_device_status() == 0, P.pact_last_error()
        rows = np.sort(rng.choice(M, size=24, replace=False))
        rows[-1] = M - 1
        assert_close(to_f64(y)[rows], orc.nvfp4_gemm(orc.quantize(x[rows]), wf), f"fwd N{N} K{K} M{M}")
        assert_close(to_f64(dx)[rows], orc.nvfp4_gemm(orc.quantize(dy[rows]), wb), f"dgrad N{N} K{K} M{M}")
