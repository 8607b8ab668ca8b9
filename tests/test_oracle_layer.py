"""Pins for the oracle's decoder-layer step (oracle/layer.py), which the CPU baseline
times and which nothing else would check: every output of OracleLayer.step is
compared with facts that do not go through its own wiring.

1. A composition written here from the data flow (PACT blog summary, section "方法"
   (method), bullets 1, 2 and 4 and the paragraph after them; PEFT explainer,
   section "LoRA"), one projection at a time with per-projection weight caches and
   the single-projection oracle functions (frozen_fwd, frozen_dgrad, lora_bwd_at),
   each pinned on its own in test_oracle_pins.py.  OracleLayer concatenates q|k|v
   and gate|up; this side never does, so a slip in the concatenation, in the segment
   bounds, in which saved copy feeds which gradient, or in a residual shows up.
2. Zero-adapter reductions: with every B = 0 the forward outputs are the frozen
   products alone (plus the residuals) and every dA is 0; with every A = 0 every dB
   is 0 and the dgrads are the frozen products alone.
3. The saved copies are distinct enough for check 1 to tell them apart: dA/dB of
   gate|up computed on the first RMSNorm's copy instead of the second's differ.

A tiny layer (H 64, I 128, k/v 32, 40 tokens, r 16) keeps everything below a second."""
import numpy as np
import pytest

import synth

H, I, KV, M, R = 64, 128, 32, 40, 16
ALPHA, EPS = 32.0, 1e-5


def _inputs(zero_a=False, zero_b=False):
    shp = {"q": (H, H), "k": (KV, H), "v": (KV, H), "o": (H, H), "gate": (I, H), "up": (I, H), "down": (H, I)}
    w, a, b = {}, {}, {}
    for p, proj in enumerate(synth.PROJ):
        N, K = shp[proj]
        w[proj] = synth.weight_bf16(p, (N, K))
        a[proj] = synth.gaussian_bf16(20 + p, (R, K), std=0.02)
        b[proj] = synth.gaussian_bf16(30 + p, (N, R), std=0.02)
        if zero_a:
            a[proj] = np.zeros_like(a[proj])
        if zero_b:
            b[proj] = np.zeros_like(b[proj])
    return {
        "w": w, "a": a, "b": b,
        "g1": synth.gaussian_bf16(40, (H,), std=0.02, mean=1.0),
        "g2": synth.gaussian_bf16(41, (H,), std=0.02, mean=1.0),
        "h": synth.gaussian_bf16(1, (M, H)), "attn": synth.gaussian_bf16(60, (M, H)),
        "d_out": synth.gaussian_bf16(56, (M, H)),
        "d_qkv": np.concatenate([synth.gaussian_bf16(61, (M, H)), synth.gaussian_bf16(62, (M, KV)),
                                 synth.gaussian_bf16(63, (M, KV))], axis=1),
    }


def _run(inp):
    from oracle.layer import OracleLayer
    L = OracleLayer(H, I, KV, R, ALPHA, EPS, inp["w"], inp["a"], inp["b"], inp["g1"], inp["g2"])
    return L.step(inp["h"], inp["attn"], inp["d_out"], inp["d_qkv"])


def _compose(orc, inp):
    """The layer step, one projection at a time (see the module docstring)."""
    f, q = orc.bf16_to_f64, orc.f64_to_bf16
    s = ALPHA / R
    w, a, b = inp["w"], inp["a"], inp["b"]
    cache = {p: orc.weight_cache(w[p]) for p in synth.PROJ}          # (Wf, Wb) per projection
    fwd = lambda xq, x, p: orc.frozen_fwd(xq, cache[p][0], x, a[p], b[p], s)
    dgr = lambda dy, p: orc.frozen_dgrad(dy, cache[p][1], a[p], b[p], s)
    grads = lambda dy, xt, p: orc.lora_bwd_at(f(dy), xt, f(a[p]), f(b[p]), s)[:2]
    o = {}
    # forward
    y1, xq1, rstd1 = orc.rmsnorm_quant(inp["h"], inp["g1"], EPS)
    o["qkv"] = q(np.concatenate([fwd(xq1, y1, p) for p in ("q", "k", "v")], 1))
    attn = inp["attn"]
    o["h2"] = h2 = q(f(inp["h"]) + fwd(orc.quantize(attn), attn, "o"))
    y2, xq2, rstd2 = orc.rmsnorm_quant(h2, inp["g2"], EPS)
    gate, up = q(fwd(xq2, y2, "gate")), q(fwd(xq2, y2, "up"))
    o["gu"] = np.concatenate([gate, up], 1)
    m, mq, gq, uq = orc.silu_mul_quant(gate, up)
    o["out"] = q(f(h2) + fwd(mq, m, "down"))
    # backward: down
    d_out = inp["d_out"]
    o["dm"] = dm = q(dgr(d_out, "down"))
    dg, du = orc.silu_mul_bwd(f(dm), gq, uq)
    dgate, dup = q(dg), q(du)
    o["dgu"] = np.concatenate([dgate, dup], 1)
    o["dA_d"], o["dB_d"] = grads(d_out, f(orc.silu_mul_recompute(gq, uq)), "down")
    # gate, up: the two dgrads add up; the gradients read the second RMSNorm's copy
    o["dx2"] = dx2 = q(dgr(dgate, "gate") + dgr(dup, "up"))
    x2t = xq2.dequantize()
    ga, gb = grads(dgate, x2t, "gate")
    ua, ub = grads(dup, x2t, "up")
    o["dA_gu"], o["dB_gu"] = np.concatenate([ga, ua], 0), np.concatenate([gb, ub], 0)
    o["dh2"] = dh2 = q(orc.rmsnorm_bwd(f(dx2), xq2, rstd2, inp["g2"]) + f(d_out))
    # o: its output joined the residual stream h2; its gradients read attn
    o["dattn"] = q(dgr(dh2, "o"))
    o["dA_o"], o["dB_o"] = grads(dh2, f(attn), "o")
    # q, k, v: d_qkv splits into the three projections' upstream gradients
    parts = {"q": inp["d_qkv"][:, :H], "k": inp["d_qkv"][:, H:H + KV], "v": inp["d_qkv"][:, H + KV:]}
    o["dx1"] = dx1 = q(sum(dgr(parts[p], p) for p in ("q", "k", "v")))
    x1t = xq1.dequantize()
    g = {p: grads(parts[p], x1t, p) for p in ("q", "k", "v")}
    o["dA_qkv"] = np.concatenate([g[p][0] for p in ("q", "k", "v")], 0)
    o["dB_qkv"] = np.concatenate([g[p][1] for p in ("q", "k", "v")], 0)
    o["dh"] = q(orc.rmsnorm_bwd(f(dx1), xq1, rstd1, inp["g1"]) + f(dh2))
    return o


BF16_OUT = ("qkv", "h2", "gu", "out", "dm", "dgu", "dx2", "dh2", "dattn", "dx1", "dh")
F64_OUT = ("dA_d", "dB_d", "dA_gu", "dB_gu", "dA_o", "dB_o", "dA_qkv", "dB_qkv")


def _bf16_equal_or_adjacent(orc, got, want, what):
    """BF16 outputs: the two sides sum in a different order (one GEMM over q|k|v
    against three), so a value on a rounding boundary may land one ulp apart;
    anything further is a wiring difference."""
    g = got.astype(np.int32)
    wv = want.astype(np.int32)
    same_sign = (g ^ wv) & 0x8000 == 0
    ulps = np.where(same_sign, np.abs(g - wv), np.abs((g & 0x7FFF) + (wv & 0x7FFF)))
    assert got.shape == want.shape, what
    assert int(ulps.max()) <= 1, f"{what}: {int((ulps > 1).sum())} values differ by more than one BF16 ulp"
    assert np.mean(ulps == 0) > 0.99, f"{what}: {int((ulps != 0).sum())} values off by one ulp"


def test_step_equals_per_projection_composition(orc):
    inp = _inputs()
    got, want = _run(inp), _compose(orc, inp)
    assert set(got) == set(BF16_OUT) | set(F64_OUT)
    for k in BF16_OUT:
        _bf16_equal_or_adjacent(orc, got[k], want[k], k)
    for k in F64_OUT:
        np.testing.assert_allclose(got[k], want[k], rtol=1e-12, atol=1e-14 * np.abs(want[k]).max(), err_msg=k)


def test_zero_B_forward_is_frozen_only_and_dA_vanishes(orc):
    inp = _inputs(zero_b=True)
    got = _run(inp)
    f, q = orc.bf16_to_f64, orc.f64_to_bf16
    cat = lambda names: np.concatenate([inp["w"][n] for n in names], 0)
    y1, xq1, _ = orc.rmsnorm_quant(inp["h"], inp["g1"], EPS)
    assert np.array_equal(got["qkv"], q(orc.nvfp4_gemm(xq1, orc.weight_cache(cat("qkv"))[0])))
    wf_o = orc.weight_cache(inp["w"]["o"])[0]
    h2 = q(f(inp["h"]) + orc.nvfp4_gemm(orc.quantize(inp["attn"]), wf_o))
    assert np.array_equal(got["h2"], h2)
    _, xq2, _ = orc.rmsnorm_quant(h2, inp["g2"], EPS)
    gu = q(orc.nvfp4_gemm(xq2, orc.weight_cache(cat(("gate", "up")))[0]))
    assert np.array_equal(got["gu"], gu)
    _, mq, _, _ = orc.silu_mul_quant(gu[:, :I], gu[:, I:])
    assert np.array_equal(got["out"], q(f(h2) + orc.nvfp4_gemm(mq, orc.weight_cache(inp["w"]["down"])[0])))
    for k in ("dA_d", "dA_gu", "dA_o", "dA_qkv"):
        assert not np.any(got[k]), k
    # the input gradients reduce to the frozen dgrads: dm = q(q(d_out) . deq(Wb_down)^T)
    wb_d = orc.weight_cache(inp["w"]["down"])[1]
    assert np.array_equal(got["dm"], q(orc.nvfp4_gemm(orc.quantize(inp["d_out"]), wb_d)))


def test_zero_A_makes_dB_vanish(orc):
    inp = _inputs(zero_a=True)
    got = _run(inp)
    for k in ("dB_d", "dB_gu", "dB_o", "dB_qkv"):
        assert not np.any(got[k]), k
    for k in ("dA_d", "dA_gu", "dA_o", "dA_qkv"):
        assert np.any(got[k]), k


def test_the_saved_copies_are_told_apart(orc):
    """If gate|up's gradients read the first RMSNorm's copy instead of the second's,
    they change by far more than the composition test's tolerance."""
    inp = _inputs()
    got = _run(inp)
    f = orc.bf16_to_f64
    _, xq1, _ = orc.rmsnorm_quant(inp["h"], inp["g1"], EPS)
    wrong = orc.lora_bwd_at(f(got["dgu"][:, :I]), xq1.dequantize(), f(inp["a"]["gate"]), f(inp["b"]["gate"]),
                            ALPHA / R)[0]
    assert np.max(np.abs(wrong - got["dA_gu"][:R])) > 1e-3 * np.max(np.abs(got["dA_gu"][:R]))
