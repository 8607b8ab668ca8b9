"""NVFP4-adapted GPTQ calibration on the GPU (pact_gptq_nvfp4) against the oracle
(oracle/gptq.py): codes and scales bit-exact.  Both sides take every decision (block
scale bytes, element codes) in FP64; the GPU computes the Cholesky factor of H^-1
by its own route (a blocked factorisation of the index-reversed H and a triangular
inverse), so the working weights agree to rounding and the discrete decisions agree
exactly unless a value falls within rounding of a decision boundary.

GPTQ's rows are independent once H is fixed (H depends on the calibration inputs
only), so full-size weights are checked on sampled rows that the oracle calibrates
on their own.  Also: a diagonal Hessian (one-hot calibration rows) reduces GPTQ to
the plain quantizer, dead columns are zeroed, and a calibrated layout drives the
frozen GEMM through pact_weight_layout_cache_from_nvfp4."""
import numpy as np
import pytest
import torch

import synth
from oracle import gptq
from tests.util import assert_close, assert_nvfp4_equal, to_dev, to_f64

pytestmark = pytest.mark.gpu


def _run(P, w_bits, x_bits, damp=0.01):
    err = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    q = P.pact_gptq_nvfp4(to_dev(w_bits), to_dev(x_bits), damp, pivot_error=err)
    torch.cuda.synchronize()
    assert P.pact_get_device_status() == 0, P.pact_last_error()
    assert int(err.item()) == 0
    return q


@pytest.mark.parametrize("N,K,n,dead", [(200, 576, 300, False), (64, 128, 96, True), (130, 1024, 1000, False)])
def test_gptq_matches_the_oracle(orc, N, K, n, dead):
    import nvfp4_gemm_b200 as P
    w = synth.weight_bf16(3, (N, K))
    x = synth.gaussian_bf16(90, (n, K))
    if dead:
        x[:, [5, 77]] = 0                       # no calibration input reaches columns 5 and 77
    q = _run(P, w, x)
    ref, _ = gptq.gptq_nvfp4(w, x)
    assert_nvfp4_equal(q, ref, orc, f"GPTQ N{N} K{K} n{n}")
    if dead:
        codes = q.codes.cpu().numpy()
        assert np.all((codes[:, 2] & 0xF0) == 0) and np.all((codes[:, 38] & 0xF0) == 0)


@pytest.mark.parametrize("name,group", [("llama-3.2-1b", ("q", "k", "v")), ("llama-3.2-3b", ("gate", "up")),
                                        ("qwen2.5-1.5b", ("down",))])
def test_gptq_full_size_sampled_rows(orc, name, group):
    """A layer's concatenated weight group at full size, 512 calibration tokens; the
    oracle calibrates 24 sampled rows (the last row included) with the same inputs."""
    import nvfp4_gemm_b200 as P
    shp = synth.layer_shapes(name)
    c = synth.LAYERS[name]
    w = np.concatenate([synth.weight_bf16(synth.PROJ.index(p), shp[p], outliers=c["outliers"]) for p in group], 0)
    N, K = w.shape
    x = synth.gaussian_bf16(91, (512, K))
    q = _run(P, w, x)
    rng = np.random.default_rng(N + K)
    rows = np.sort(rng.choice(N, size=24, replace=False))
    rows[-1] = N - 1
    ref, _ = gptq.gptq_nvfp4(w[rows], x)
    codes = q.codes.cpu().numpy()[rows]
    assert np.array_equal(codes, ref.codes), f"{name} {group}: {int((codes != ref.codes).sum())} code bytes differ"
    got_scales = orc.unpack_scales(q.scales.cpu().numpy(), N, K)[rows]
    assert np.array_equal(got_scales, ref.scales)


def test_diagonal_hessian_gives_the_plain_quantizer(orc):
    """One-hot calibration rows make H diagonal: no error moves to other columns, so
    the calibrated layout is the plain quantizer's (pact_quantize_nvfp4)."""
    import nvfp4_gemm_b200 as P
    K = 256
    x = np.zeros((K, K))
    for i in range(K):
        x[i, i] = 1.0 + (i % 7) * 0.25
    w = synth.weight_bf16(5, (192, K), outliers=True)
    q = _run(P, w, synth.f64_to_bf16_bits(x))
    assert_nvfp4_equal(q, orc.quantize(w), orc, "GPTQ with a diagonal Hessian")


def test_calibrated_layout_drives_the_gemm(orc):
    """The calibrated forward layout, cached with its re-quantized backward layout,
    in the forward and dgrad GEMMs."""
    import nvfp4_gemm_b200 as P
    N, K, M = 384, 512, 300
    w = synth.weight_bf16(6, (N, K))
    xc = synth.gaussian_bf16(92, (256, K))
    q = _run(P, w, xc)
    wc = P.pact_weight_layout_cache_from_nvfp4(q)
    x = synth.gaussian_bf16(1, (M, K))
    dy = synth.gaussian_bf16(50, (M, N))
    y = P.pact_frozen_gemm_fwd(P.pact_quantize_nvfp4(to_dev(x)), wc)
    dx = P.pact_frozen_gemm_dgrad(P.pact_quantize_nvfp4(to_dev(dy)), wc)
    torch.cuda.synchronize()
    assert P.pact_get_device_status() == 0, P.pact_last_error()
    ref, _ = gptq.gptq_nvfp4(w, xc)
    wb = orc.quantize(orc.f64_to_bf16_exact(orc.dequantize(ref).T))
    assert_nvfp4_equal(wc.fwd, ref, orc, "cached forward layout")
    assert_nvfp4_equal(wc.bwd, wb, orc, "cached backward layout")
    assert_close(to_f64(y), orc.nvfp4_gemm(orc.quantize(x), ref), "fwd with the calibrated weight")
    assert_close(to_f64(dx), orc.nvfp4_gemm(orc.quantize(dy), wb), "dgrad with the calibrated weight")
