"""The two-level weight layouts on the GPU against the oracle (needs a B200): the
absolute maximum and the tensor exponent, the cached codes and scales bit for bit,
and the forward / input-gradient GEMMs with the LoRA branch, whose activations
enter divided by 2^g and whose dA is scaled back, within
|gpu - oracle| <= 8e-3 |oracle| + 1e-3 rms(oracle)."""
import numpy as np
import pytest
import torch

import synth
from tests.util import assert_close, assert_nvfp4_equal, to_dev, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def P():
    import nvfp4_gemm_b200 as p
    return p


def _segments(parts):
    out, acc = [], 0
    for p in parts:
        acc += p
        out.append(acc)
    return out


@pytest.mark.parametrize("N,K,outliers", [(512, 512, False), (448, 320, True), (2048, 512, False),
                                          (384, 2048, True)])
def test_two_level_cache(P, orc, N, K, outliers):
    w = synth.weight_bf16(0, (N, K), outliers=outliers)
    wd = to_dev(w)
    amax = P.pact_absmax_bf16(wd)
    torch.cuda.synchronize()
    assert float(amax.cpu()) == np.max(np.abs(synth.bf16_bits_to_f64(w)))
    wc = P.pact_weight_layout_cache(wd, two_level=True)
    torch.cuda.synchronize()
    e, wf, wb = orc.weight_cache_two_level(w)
    assert wc.gexp == e < 0
    assert_nvfp4_equal(wc.fwd, wf, orc, "two-level fwd layout")
    assert_nvfp4_equal(wc.bwd, wb, orc, "two-level bwd layout")
    assert P.pact_get_device_status() == 0, P.pact_last_error()


@pytest.mark.parametrize("M,parts,K,r", [(256, [512], 512, 16), (300, [512, 256, 256], 576, 16),
                                         (130, [768], 320, 48)])
def test_two_level_gemms_with_lora(P, orc, M, parts, K, r):
    N = sum(parts)
    seg_end = _segments(parts)
    nseg, R = len(parts), len(parts) * r
    x = synth.gaussian_bf16(1, (M, K))
    w = synth.weight_bf16(0, (N, K), outliers=True)
    a = synth.gaussian_bf16(20, (R, K), std=0.02)
    b = synth.gaussian_bf16(30, (N, r), std=0.02)
    res = synth.gaussian_bf16(40, (M, N))
    dy = synth.gaussian_bf16(50, (M, N))
    s = 2.0
    xd, ad, bd, resd, dyd = to_dev(x), to_dev(a), to_dev(b), to_dev(res), to_dev(dy)
    wc = P.pact_weight_layout_cache(to_dev(w), two_level=True)
    g = wc.gexp
    sc = s * 2.0 ** -g
    # forward: T with s 2^-g, the GEMM scales its whole accumulator by 2^g
    xq = P.pact_quantize_nvfp4(xd)
    T = P.pact_lora_fwd(xd, ad, sc)
    y = P.pact_frozen_gemm_fwd(xq, wc, lora=P.lora_struct(T, bd, r, seg_end), residual=resd)
    # input gradient: U with s 2^-g; dA from U scaled back by 2^g
    dyq = P.pact_quantize_nvfp4(dyd)
    U = P.pact_lora_bwd_u(dyd, bd, r, seg_end, sc)
    dx = P.pact_frozen_gemm_dgrad(dyq, wc, lora=P.lora_struct(U, ad, R, [K]))
    dA, dB = P.pact_lora_bwd(dyd, ad, U, r, seg_end, s, x=xd, u_gexp=g)
    torch.cuda.synchronize()
    assert P.pact_get_device_status() == 0, P.pact_last_error()

    e, wf, wb = orc.weight_cache_two_level(w)
    assert e == g
    f = synth.bf16_bits_to_f64
    xf, af, bf, dyf = f(x), f(a), f(b), f(dy)
    t_dev = to_f64(T[:, :R]) + to_f64(T[:, R:])
    u_dev = to_f64(U[:, :R]) + to_f64(U[:, R:])
    # the activations are s 2^-g times the oracle's
    t_ref = np.concatenate([sc * orc.gemm_nt(xf, af[i * r:(i + 1) * r]) for i in range(nseg)], 1)
    assert_close(t_dev, t_ref, "T")
    lo, u_ref = 0, np.zeros((M, R))
    for i, hi in enumerate(seg_end):
        u_ref[:, i * r:(i + 1) * r] = sc * orc.gemm_nt(dyf[:, lo:hi], bf[lo:hi].T)
        lo = hi
    assert_close(u_dev, u_ref, "U")
    # the GEMMs, teacher-forced on the device's activations
    ref = orc.nvfp4_gemm(orc.quantize(x), wf)
    lo = 0
    for i, hi in enumerate(seg_end):
        ref[:, lo:hi] += orc.gemm_nt(t_dev[:, i * r:(i + 1) * r], bf[lo:hi])
        lo = hi
    assert_close(to_f64(y), f(res) + 2.0 ** g * ref, "fwd + LoRA + residual")
    ref_d = 2.0 ** g * (orc.nvfp4_gemm(orc.quantize(dy), wb) + orc.gemm_nt(u_dev, af.T))
    assert_close(to_f64(dx), ref_d, "dgrad + LoRA")
    # end to end against the oracle's projection semantics (its own LoRA terms)
    if nseg == 1:
        assert_close(to_f64(y), f(res) + orc.frozen_fwd(orc.quantize(x), wf, x, a, b, s, gexp=g), "fwd (oracle)")
        assert_close(to_f64(dx), orc.frozen_dgrad(dy, wb, a, b, s, gexp=g), "dgrad (oracle)")
    # LoRA weight gradients: dA = s (dY B)^T X, dB = s dY^T (X A^T)
    assert_close(to_f64(dA), 2.0 ** g * orc.gemm_nt(u_dev.T, xf.T), "dA (teacher-forced)")
    db_ref, lo = np.zeros((N, r)), 0
    for i, hi in enumerate(seg_end):
        db_ref[lo:hi] = s * orc.gemm_nt(dyf[:, lo:hi].T, orc.gemm_nt(xf, af[i * r:(i + 1) * r]).T)
        lo = hi
    assert_close(to_f64(dB), db_ref, "dB")
