"""The oracle's decoder-layer step (test infrastructure only).

Composes the element-level oracle functions in the order of PACT's data flow (PACT
blog summary, section "方法" (method); PACT abstract): RMSNorm + NVFP4 quantization
of its BF16 output, NVFP4 GEMMs of the seven frozen projections (q|k|v and gate|up
sharing an input) with the BF16 LoRA branch, SiLU-multiply from BF16 gate/up with
NVFP4 copies saved, and the backward pass reading those copies and the cached
transposed, re-quantized weight layouts.  Everything is float64; values are rounded
to BF16 exactly where the data flow stores BF16 (stage outputs, gradients).  The
attention core is not on this path: a BF16 `attn` tensor stands in for its output
and `d_qkv` for its input gradient.  The LoRA update is h = W0 x + scale B A x
(PEFT explainer, section "LoRA").
"""
from __future__ import annotations

import numpy as np

from . import (bf16_to_f64, f64_to_bf16, frozen_dgrad, frozen_fwd, gemm_nt, lora_bwd, nvfp4_gemm, quantize,
               rmsnorm_bwd, rmsnorm_quant, silu_mul_bwd, silu_mul_quant, silu_mul_recompute, weight_cache,
               weight_cache_two_level)


def _segments(seg_end):
    lo = 0
    for i, hi in enumerate(seg_end):
        yield i, lo, hi
        lo = hi


def lora_fwd_term(x, a, b, r, seg_end, scale):
    """scale * (X A_i^T) B_i^T for the columns of each segment i; float64."""
    out = np.zeros((x.shape[0], seg_end[-1]))
    for i, lo, hi in _segments(seg_end):
        out[:, lo:hi] = scale * gemm_nt(gemm_nt(x, a[i * r:(i + 1) * r]), b[lo:hi])
    return out


def lora_dgrad_term(dy, a, b, r, seg_end, scale):
    """sum_i scale * (dY[:, seg_i] B_i) A_i; float64."""
    out = np.zeros((dy.shape[0], a.shape[1]))
    for i, lo, hi in _segments(seg_end):
        u = gemm_nt(dy[:, lo:hi], b[lo:hi].T)
        out += scale * gemm_nt(u, a[i * r:(i + 1) * r].T)
    return out


def lora_grads(dy, xt, a, b, r, seg_end, scale):
    """dA_i = scale (dY_i B_i)^T X~, dB_i = scale dY_i^T (X~ A_i^T), stacked like A, B."""
    da = np.zeros_like(a)
    db = np.zeros_like(b)
    for i, lo, hi in _segments(seg_end):
        ai = a[i * r:(i + 1) * r]
        u = gemm_nt(dy[:, lo:hi], b[lo:hi].T)
        da[i * r:(i + 1) * r] = scale * gemm_nt(u.T, xt.T)
        db[lo:hi] = scale * gemm_nt(dy[:, lo:hi].T, gemm_nt(xt, ai).T)
    return da, db


class OracleProjection:
    """One frozen projection with its LoRA branch (w [N x K], A [r x K], B [N x r],
    BF16 bits), forward and backward on X and dY:
      Y = deq(q(X)) deq(Wf)^T + s (X A^T) B^T,  dX = deq(q(dY)) deq(Wb)^T + s (dY B) A,
      dA = s (dY B)^T X~,  dB = s dY^T (X~ A^T),  X~ = deq(q(X)) the saved NVFP4 copy."""

    input_keys = ("x", "dy")

    def __init__(self, w, a, b, r, alpha):
        self.wf, self.wb = weight_cache(w)
        self.a, self.b, self.r, self.scale = a, b, r, alpha / r

    def step(self, x, dy):
        xq = quantize(x)
        da, db, _ = lora_bwd(dy, xq.dequantize(), self.a, self.b, self.scale)
        return {"y": f64_to_bf16(frozen_fwd(xq, self.wf, x, self.a, self.b, self.scale)),
                "dx": f64_to_bf16(frozen_dgrad(dy, self.wb, self.a, self.b, self.scale)), "dA": da, "dB": db}


class OracleLayer:
    """w, lora_a, lora_b: dicts of BF16 bit arrays keyed q, k, v, o, gate, up, down
    (PyTorch [out, in] layout); gamma1, gamma2: BF16 bits [H].  two_level: cache the
    weights in the two-level variant (weight_cache_two_level), one exponent per
    concatenated group."""

    input_keys = ("h", "attn", "d_out", "d_qkv")

    def __init__(self, H, I, KV, r, alpha, eps, w, lora_a, lora_b, gamma1, gamma2, two_level=False):
        self.H, self.I, self.KV, self.r, self.eps = H, I, KV, r, eps
        self.scale = alpha / r
        cat = lambda names, d: np.concatenate([d[n] for n in names], 0)
        self.wf, self.wb, self.gexp = {}, {}, {}
        for key, names in (("qkv", ("q", "k", "v")), ("o", ("o",)), ("gu", ("gate", "up")), ("d", ("down",))):
            if two_level:
                self.gexp[key], self.wf[key], self.wb[key] = weight_cache_two_level(cat(names, w))
            else:
                self.gexp[key] = 0
                self.wf[key], self.wb[key] = weight_cache(cat(names, w))
            self.wf[key].dequantize()
            self.wb[key].dequantize()
        f = bf16_to_f64
        self.a = {"qkv": f(cat(("q", "k", "v"), lora_a)), "o": f(lora_a["o"]), "gu": f(cat(("gate", "up"), lora_a)),
                  "d": f(lora_a["down"])}
        self.b = {"qkv": f(cat(("q", "k", "v"), lora_b)), "o": f(lora_b["o"]), "gu": f(cat(("gate", "up"), lora_b)),
                  "d": f(lora_b["down"])}
        self.seg = {"qkv": [H, H + KV, H + 2 * KV], "o": [H], "gu": [I, 2 * I], "d": [H]}
        self.g1, self.g2 = gamma1, gamma2

    def _g(self, key, aq, cache):
        """The frozen product with group `key`'s cached layout, times its 2^e."""
        return 2.0 ** self.gexp[key] * nvfp4_gemm(aq, cache[key])

    def step(self, h, attn, d_out, d_qkv):
        """One forward + backward over the given tokens (BF16 bit arrays).  Returns the
        stage outputs (BF16 bits or float64 where the path keeps higher precision)."""
        H, I, r, s = self.H, self.I, self.r, self.scale
        f, q = bf16_to_f64, f64_to_bf16
        o = {}
        # ---------------- forward
        y1, xq1, rstd1 = rmsnorm_quant(h, self.g1, self.eps)
        qkv = self._g("qkv", xq1, self.wf) + lora_fwd_term(f(y1), self.a["qkv"], self.b["qkv"], r,
                                                                self.seg["qkv"], s)
        o["qkv"] = q(qkv)
        aq = quantize(attn)
        o["h2"] = h2 = q(f(h) + self._g("o", aq, self.wf) + lora_fwd_term(f(attn), self.a["o"], self.b["o"], r,
                                                                             self.seg["o"], s))
        y2, xq2, rstd2 = rmsnorm_quant(h2, self.g2, self.eps)
        o["gu"] = gu = q(self._g("gu", xq2, self.wf) + lora_fwd_term(f(y2), self.a["gu"], self.b["gu"], r,
                                                                         self.seg["gu"], s))
        m, mq, gq, uq = silu_mul_quant(gu[:, :I], gu[:, I:])
        o["out"] = q(f(h2) + self._g("d", mq, self.wf) + lora_fwd_term(f(m), self.a["d"], self.b["d"], r,
                                                                           self.seg["d"], s))
        # ---------------- backward
        dof = f(d_out)
        o["dm"] = dm = q(self._g("d", quantize(d_out), self.wb) +
                         lora_dgrad_term(dof, self.a["d"], self.b["d"], r, self.seg["d"], s))
        dg, du = silu_mul_bwd(f(dm), gq, uq)
        o["dgu"] = dgu = q(np.concatenate([dg, du], 1))
        m_re = silu_mul_recompute(gq, uq)
        o["dA_d"], o["dB_d"] = lora_grads(dof, f(m_re), self.a["d"], self.b["d"], r, self.seg["d"], s)
        o["dx2"] = dx2 = q(self._g("gu", quantize(dgu), self.wb) +
                           lora_dgrad_term(f(dgu), self.a["gu"], self.b["gu"], r, self.seg["gu"], s))
        o["dA_gu"], o["dB_gu"] = lora_grads(f(dgu), xq2.dequantize(), self.a["gu"], self.b["gu"], r,
                                            self.seg["gu"], s)
        o["dh2"] = dh2 = q(rmsnorm_bwd(f(dx2), xq2, rstd2, self.g2) + dof)
        o["dattn"] = q(self._g("o", quantize(dh2), self.wb) +
                       lora_dgrad_term(f(dh2), self.a["o"], self.b["o"], r, self.seg["o"], s))
        o["dA_o"], o["dB_o"] = lora_grads(f(dh2), f(attn), self.a["o"], self.b["o"], r, self.seg["o"], s)
        o["dx1"] = dx1 = q(self._g("qkv", quantize(d_qkv), self.wb) +
                           lora_dgrad_term(f(d_qkv), self.a["qkv"], self.b["qkv"], r, self.seg["qkv"], s))
        o["dA_qkv"], o["dB_qkv"] = lora_grads(f(d_qkv), xq1.dequantize(), self.a["qkv"], self.b["qkv"], r,
                                              self.seg["qkv"], s)
        o["dh"] = q(rmsnorm_bwd(f(dx1), xq1, rstd1, self.g1) + f(dh2))
        return o
