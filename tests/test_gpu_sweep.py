"""The GEMM shape sweep (six N x K weight shapes x M in {512, 2048, 8192, 32768},
forward and dgrad) against the oracle at full size, on sampled rows the oracle
computes one by one.

Quantization is row-local (blocks of 16 along the contraction), so the oracle
quantizes only the sampled rows of X (or dY) and multiplies them by its dequantized
weight layouts; the GPU runs the whole GEMM through the C ABI in the launch
configuration bench.py --sweep times.  The four token counts cover a partial wave,
about one wave and many waves of 256 x 256 pair tiles.  The inputs of a smaller M
are the leading rows of the M = 32768 inputs (the generator is counter-based and
row-major), so each shape generates its inputs once."""
import functools

import numpy as np
import pytest
import torch

import synth
from tests.util import assert_close, to_dev, to_f64

pytestmark = pytest.mark.gpu

M_MAX = max(synth.SWEEP_M)


@functools.lru_cache(maxsize=4)
def _host(tensor_id, cols):
    return synth.gaussian_bf16(tensor_id, (M_MAX, cols))


@pytest.mark.parametrize("N,K", synth.SWEEP_NK)
def test_sweep_shape_sampled_rows(orc, N, K):
    import nvfp4_gemm_b200 as P
    w = synth.weight_bf16(0, (N, K))
    wc = P.pact_weight_layout_cache(to_dev(w))
    wf, wb = orc.weight_cache(w)
    rng = np.random.default_rng(N * 7 + K)
    x_all, dy_all = _host(1, K), _host(50, N)
    x_dev, dy_dev = to_dev(x_all), to_dev(dy_all)
    for M in synth.SWEEP_M:
        y = P.pact_frozen_gemm_fwd(P.pact_quantize_nvfp4(x_dev[:M]), wc)
        dx = P.pact_frozen_gemm_dgrad(P.pact_quantize_nvfp4(dy_dev[:M]), wc)
        torch.cuda.synchronize()
        assert P.pact_get_device_status() == 0, P.pact_last_error()
        rows = np.sort(rng.choice(M, size=24, replace=False))
        rows[-1] = M - 1
        assert_close(to_f64(y)[rows], orc.nvfp4_gemm(orc.quantize(x_all[rows]), wf), f"fwd N{N} K{K} M{M}")
        assert_close(to_f64(dx)[rows], orc.nvfp4_gemm(orc.quantize(dy_all[rows]), wb), f"dgrad N{N} K{K} M{M}")
        del y, dx
    del x_dev, dy_dev
    torch.cuda.empty_cache()
