"""One PACT LoRA decoder layer: the NVFP4 data flow through its seven frozen
projections, forward and backward, composed from libpact calls.

Data flow (PACT blog summary, section "方法" (method); PACT abstract):
  forward   xq1, x1, rstd1 = RMSNorm+quantize(h)            x1 BF16 feeds LoRA only
            qkv  = NVFP4 GEMM(xq1, W_qkv) + LoRA(x1)          q|k|v concatenated along N
            [attention core: not on the NVFP4 path; a synthetic BF16 `attn` stands in]
            h2   = h + NVFP4 GEMM(q(attn), W_o) + LoRA(attn)  residual fused in the epilogue
            xq2, x2, rstd2 = RMSNorm+quantize(h2)
            gu   = NVFP4 GEMM(xq2, W_gu) + LoRA(x2)           gate|up concatenated along N
            m, mq = SiLU-multiply+quantize(gate, up)           gq, uq (NVFP4 copies of gate, up,
                                                                written by the GEMM) saved for backward
            out  = h2 + NVFP4 GEMM(mq, W_down) + LoRA(m)
  saved for backward: xq1, rstd1, xq2, rstd2, gq, uq (NVFP4) and attn.
  backward  the input gradients run the NVFP4 dgrad GEMMs on the cached transposed,
            re-quantized weight layouts; the LoRA weight gradients read the saved
            NVFP4 copies (q/k/v, gate/up: xq; down: m~ recomputed from gq, uq) or
            attn (o).  The attention backward is replaced by a synthetic d(qkv).

Every op writes into buffers allocated once here, so a whole step can be captured
into CUDA graphs.  Nothing below computes on the host or in PyTorch kernels.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Callable, Dict, List

import torch

from . import pact as P


@dataclass
class Op:
    name: str
    fn: Callable[[], None]
    kind: str = "other"        # "gemm" for the NVFP4 frozen GEMMs
    flops: float = 0.0         # algorithmic FLOPs of a GEMM op
    kernels: int = 1           # libpact kernels one call launches
    bytes: float = 0.0         # algorithmic HBM bytes of one call (each input read once, each output written once)
    side: bool = False         # a leaf (LoRA weight gradients): may run beside the rest of the step


@dataclass
class LayerShape:
    M: int
    H: int
    I: int
    KV: int
    r: int = 16
    alpha: float = 32.0
    eps: float = 1e-5

    @property
    def scale(self) -> float:
        return self.alpha / self.r

    @property
    def n_qkv(self) -> int:
        return self.H + 2 * self.KV

    def nv(self, rows: int, cols: int) -> float:
        """Bytes of an NVFP4 tensor: codes plus one scale byte per 16 values."""
        return rows * cols / 2 + rows * cols / 16

    def frozen_flops(self) -> float:
        """2 M N K for the forward and the dgrad of the seven frozen projections."""
        nk = self.n_qkv * self.H + self.H * self.H + 2 * self.I * self.H + self.H * self.I
        return 2.0 * 2.0 * self.M * nk


class PactLayer:
    """Weights are BF16 device tensors in PyTorch [out, in] layout:
    w = {q, k, v, o, gate, up, down}; lora_a = {p: [r, in]}, lora_b = {p: [out, r]};
    gamma1, gamma2: [H].  Frozen weights are cached as NVFP4 forward/backward layouts
    at construction (once); two_level selects the variant with a power of two per
    cached group (pact_weight_layout_cache_scaled).  grad_fp32: the LoRA weight
    gradients are written unrounded in FP32 into one flat buffer (grad_bucket, views
    in grads32), to be summed over data-parallel replicas in one collective and then
    rounded once to BF16 by round_grads() into `grads`."""

    input_keys = ("h", "attn", "d_out", "d_qkv")

    def __init__(self, shape: LayerShape, w: Dict[str, torch.Tensor], lora_a: Dict[str, torch.Tensor],
                 lora_b: Dict[str, torch.Tensor], gamma1: torch.Tensor, gamma2: torch.Tensor,
                 two_level: bool = False, grad_fp32: bool = False, fuse_silu: bool = False):
        self.s = shape
        self.two_level = two_level
        self.grad_fp32 = grad_fp32
        # fuse_silu: the SiLU-multiply in the gate|up GEMM's epilogue (needs I a multiple
        # of 256).  Off by default: at K = H = 3072 the 16 epilogue warps, not the tensor
        # pipe, bound that kernel, and it takes longer than the GEMM that writes g|u
        # plus the separate SiLU kernel that reads it back.
        self.fuse_silu = fuse_silu and shape.I % 256 == 0
        S = shape
        dev = gamma1.device
        cat = lambda names, d: torch.cat([d[n] for n in names], 0).contiguous()
        # frozen weights: concatenated where projections share an input, then cached
        cache = lambda t: P.pact_weight_layout_cache(t, two_level=two_level)
        self.c_qkv = cache(cat(("q", "k", "v"), w))
        self.c_o = cache(w["o"].contiguous())
        self.c_gu = cache(cat(("gate", "up"), w))
        self.c_d = cache(w["down"].contiguous())
        # a group cached with exponent g scales its whole GEMM accumulator by 2^g, so
        # its LoRA activations (T, U) are computed with scale * 2^-g (exact) and the
        # dA contraction over U is scaled back by 2^g
        self.gexp = {"qkv": self.c_qkv.gexp, "o": self.c_o.gexp, "gu": self.c_gu.gexp, "d": self.c_d.gexp}
        self.sc = {k: shape.scale * 2.0 ** -g for k, g in self.gexp.items()}
        # adapters, stacked like the weights
        self.a_qkv, self.b_qkv = cat(("q", "k", "v"), lora_a), cat(("q", "k", "v"), lora_b)
        self.a_o, self.b_o = lora_a["o"].contiguous(), lora_b["o"].contiguous()
        self.a_gu, self.b_gu = cat(("gate", "up"), lora_a), cat(("gate", "up"), lora_b)
        self.a_d, self.b_d = lora_a["down"].contiguous(), lora_b["down"].contiguous()
        self.seg_qkv = [S.H, S.H + S.KV, S.H + 2 * S.KV]
        self.seg_gu = [S.I, 2 * S.I]
        self.g1, self.g2 = gamma1, gamma2
        M, H, I, r = S.M, S.H, S.I, S.r
        bf = lambda *sh: torch.empty(sh, dtype=torch.bfloat16, device=dev)
        nv = lambda rows, cols: P.NVFP4Tensor.empty(rows, cols, dev)
        # forward activations
        self.xq1, self.x1, self.rstd1 = nv(M, H), bf(M, H), torch.empty(M, dtype=torch.float32, device=dev)
        self.t_qkv, self.qkv = bf(M, 2 * 3 * r), bf(M, S.n_qkv)
        self.aq, self.t_o, self.h2 = nv(M, H), bf(M, 2 * r), bf(M, H)
        self.xq2, self.x2, self.rstd2 = nv(M, H), bf(M, H), torch.empty(M, dtype=torch.float32, device=dev)
        self.t_gu = bf(M, 2 * 2 * r)
        self.gu = None if self.fuse_silu else bf(M, 2 * I)
        # m itself (BF16) exists only with the fused SiLU GEMM; the default path takes
        # mq and the down projection's T straight from gate|up (pact_lora_fwd_silu)
        self.m = bf(M, I) if self.fuse_silu else None
        self.mq, self.gq, self.uq = nv(M, I), nv(M, I), nv(M, I)
        self.t_d, self.out = bf(M, 2 * r), bf(M, H)
        # backward
        self.u_d, self.doq, self.dm = bf(M, 2 * r), nv(M, H), bf(M, I)
        self.dgu, self.dguq, self.m_re = bf(M, 2 * I), nv(M, 2 * I), bf(M, I)
        self.u_gu, self.dx2 = bf(M, 2 * 2 * r), bf(M, H)
        self.dh2, self.dh2q = bf(M, H), nv(M, H)
        self.u_o, self.dattn = bf(M, 2 * r), bf(M, H)
        self.u_qkv, self.dqkvq, self.dx1, self.dh = bf(M, 2 * 3 * r), nv(M, S.n_qkv), bf(M, H), bf(M, H)
        # LoRA weight gradients (BF16, same stacking as the adapters), views of one flat
        # buffer; with grad_fp32 also an FP32 flat buffer the backward writes
        shapes = {"a_qkv": self.a_qkv.shape, "b_qkv": self.b_qkv.shape, "a_o": self.a_o.shape,
                  "b_o": self.b_o.shape, "a_gu": self.a_gu.shape, "b_gu": self.b_gu.shape,
                  "a_d": self.a_d.shape, "b_d": self.b_d.shape}
        self.grad_bucket_bf16, self.grads = flat_views(shapes, torch.bfloat16, dev)
        self.grad_bucket, self.grads32 = (flat_views(shapes, torch.float32, dev) if grad_fp32 else (None, None))
        # one scratch buffer shared by the LoRA calls (they run in order on one stream)
        ws = max(P.pact_lora_bwd_workspace_bytes(M, S.n_qkv, H, r, 3),
                 P.pact_lora_bwd_workspace_bytes(M, 2 * I, H, r, 2),
                 P.pact_lora_bwd_workspace_bytes(M, H, I, r, 1),
                 P.pact_lora_bwd_workspace_bytes(M, H, H, r, 1),
                 P.pact_lora_fwd_workspace_bytes(M, I, 3 * r),
                 P.pact_lora_fwd_workspace_bytes(M, H, 3 * r),
                 P.pact_lora_bwd_u_workspace_bytes(M, 2 * I, r, 2),
                 P.pact_lora_bwd_u_workspace_bytes(M, S.n_qkv, r, 3))
        self.ws = self._scratch(ws, dev)
        # the LoRA weight-gradient calls are leaves of the step and may run on a second
        # stream beside the rest of it: each gets scratch of its own
        self.ws_leaf = {
            "down": self._scratch(P.pact_lora_bwd_workspace_bytes(M, H, I, r, 1), dev),
            "gu": self._scratch(P.pact_lora_bwd_workspace_bytes(M, 2 * I, H, r, 2), dev),
            "o": self._scratch(P.pact_lora_bwd_workspace_bytes(M, H, H, r, 1), dev),
            "qkv": self._scratch(P.pact_lora_bwd_workspace_bytes(M, S.n_qkv, H, r, 3), dev),
        }
        # LoRA descriptors for the fused GEMM epilogue
        self.l_qkv_f = P.lora_struct(self.t_qkv, self.b_qkv, r, self.seg_qkv)
        self.l_o_f = P.lora_struct(self.t_o, self.b_o, r, [H])
        self.l_gu_f = P.lora_struct(self.t_gu, self.b_gu, r, self.seg_gu)
        self.l_d_f = P.lora_struct(self.t_d, self.b_d, r, [H])
        self.l_d_b = P.lora_struct(self.u_d, self.a_d, 1 * r, [I])
        self.l_gu_b = P.lora_struct(self.u_gu, self.a_gu, 2 * r, [H])
        self.l_o_b = P.lora_struct(self.u_o, self.a_o, r, [H])
        self.l_qkv_b = P.lora_struct(self.u_qkv, self.a_qkv, 3 * r, [H])
        self.inputs = None

    @staticmethod
    def _scratch(nbytes: int, dev) -> torch.Tensor:
        raw = torch.empty(nbytes + 256, dtype=torch.uint8, device=dev)
        off = (-raw.data_ptr()) % 256
        return raw[off:off + nbytes]

    # ------------------------------------------------------------------ op lists
    def bind(self, h: torch.Tensor, attn: torch.Tensor, d_out: torch.Tensor, d_qkv: torch.Tensor):
        """Attach the step's inputs: layer input h [M, H], the attention-output stand-in
        attn [M, H], the upstream gradient d_out [M, H] and the attention-backward
        stand-in d_qkv [M, H + 2 KV].  The op lists read these tensors in place."""
        self.inputs = (h, attn, d_out, d_qkv)

    def forward_ops(self) -> List[Op]:
        S, s = self.s, self.s.scale
        h, attn, _, _ = self.inputs
        M, H, I, r = S.M, S.H, S.I, S.r
        gemm = lambda M, N, K: 2.0 * M * N * K
        # NVFP4 GEMM: activation codes + weight codes in, BF16 output and the LoRA term's
        # hi|lo activations [M x 2R] and B chunk [N x R] in (residual added by the caller)
        gbytes = lambda N, K, R: S.nv(M, K) + S.nv(N, K) + 2 * M * N + 2 * M * 2 * R + 2 * N * R
        # LoRA forward T = s x A^T as hi|lo: x [M x K] and A [R x K] in, T [M x 2R] out
        lora_fwd = lambda K, R: 2 * M * K + 2 * R * K + 2 * M * 2 * R
        nk = lambda K, R: P.pact_lora_fwd_launches(M, K, R)   # 1 unsplit, 2 with a finalize
        return [
            Op("rmsnorm_quant_1", lambda: P.pact_rmsnorm_quant(h, self.g1, S.eps, self.xq1, self.x1, self.rstd1),
               bytes=2 * M * H + 2 * H + S.nv(M, H) + 2 * M * H + 4 * M),
            Op("lora_fwd_qkv", lambda: P.pact_lora_fwd(self.x1, self.a_qkv, self.sc["qkv"], self.t_qkv, self.ws),
               kernels=nk(H, 3 * r), bytes=lora_fwd(H, 3 * r)),
            Op("gemm_fwd_qkv", lambda: P.pact_frozen_gemm_fwd(self.xq1, self.c_qkv, self.l_qkv_f, y=self.qkv),
               "gemm", gemm(S.M, S.n_qkv, S.H), bytes=gbytes(S.n_qkv, H, 3 * r)),
            # the LoRA product streams attn and writes its NVFP4 copy aq (the GEMM's input)
            Op("lora_fwd_o+q(attn)", lambda: P.pact_lora_fwd(attn, self.a_o, self.sc["o"], self.t_o, self.ws,
                                                             xq=self.aq),
               kernels=nk(H, r), bytes=lora_fwd(H, r) + S.nv(M, H)),
            Op("gemm_fwd_o", lambda: P.pact_frozen_gemm_fwd(self.aq, self.c_o, self.l_o_f, residual=h, y=self.h2),
               "gemm", gemm(S.M, S.H, S.H), bytes=gbytes(H, H, r) + 2 * M * H),
            Op("rmsnorm_quant_2", lambda: P.pact_rmsnorm_quant(self.h2, self.g2, S.eps, self.xq2, self.x2,
                                                               self.rstd2),
               bytes=2 * M * H + 2 * H + S.nv(M, H) + 2 * M * H + 4 * M),
            Op("lora_fwd_gu", lambda: P.pact_lora_fwd(self.x2, self.a_gu, self.sc["gu"], self.t_gu, self.ws),
               kernels=nk(H, 2 * r), bytes=lora_fwd(H, 2 * r)),
            *self._gate_up_ops(gemm, gbytes, nk),
            Op("gemm_fwd_down", lambda: P.pact_frozen_gemm_fwd(self.mq, self.c_d, self.l_d_f, residual=self.h2,
                                                               y=self.out),
               "gemm", gemm(S.M, S.H, I), bytes=gbytes(H, I, r) + 2 * M * H),
        ]

    def _gate_up_ops(self, gemm, gbytes, nk) -> List[Op]:
        S, M, H, I, r = self.s, self.s.M, self.s.H, self.s.I, self.s.r
        lora_fwd_d = 2 * r * I + 2 * M * 2 * r   # A_down in, T_down (hi|lo) out
        if self.fuse_silu:
            # one kernel: g|u stays on chip; m, mq and the saved copies gq, uq are written
            return [Op("gemm_fwd_silu", lambda: P.pact_frozen_gemm_fwd_silu(self.xq2, self.c_gu, self.m, self.mq,
                                                                            self.gq, self.uq, self.l_gu_f),
                       "gemm", gemm(S.M, 2 * I, S.H),
                       bytes=gbytes(2 * I, H, 2 * r) - 2 * M * 2 * I + 2 * M * I + 3 * S.nv(M, I)),
                    Op("lora_fwd_down", lambda: P.pact_lora_fwd(self.m, self.a_d, self.sc["d"], self.t_d, self.ws),
                       kernels=nk(I, r), bytes=2 * M * I + lora_fwd_d)]
        # the gate|up GEMM also writes the NVFP4 copies gq, uq kept for the backward; one
        # kernel then forms m = silu(g) u from gate|up, writes mq and the down
        # projection's T (m itself never goes to memory)
        return [Op("gemm_fwd_gu", lambda: P.pact_frozen_gemm_fwd_quant(self.xq2, self.c_gu, [self.gq, self.uq],
                                                                       self.l_gu_f, y=self.gu),
                   "gemm", gemm(S.M, 2 * I, S.H), bytes=gbytes(2 * I, H, 2 * r) + 2 * S.nv(M, I)),
                Op("silu_mul_quant+lora_fwd_down", lambda: P.pact_lora_fwd_silu(self.gu[:, :I], self.gu[:, I:], self.a_d,
                                                                                self.sc["d"], self.mq, self.t_d,
                                                                                workspace=self.ws),
                   kernels=nk(I, r), bytes=4 * M * I + S.nv(M, I) + lora_fwd_d)]

    def backward_ops(self) -> List[Op]:
        S, s, r = self.s, self.s.scale, self.s.r
        H, I = S.H, S.I
        _, attn, d_out, d_qkv = self.inputs
        g = self.grads32 if self.grad_fp32 else self.grads
        f32 = self.grad_fp32
        M = S.M
        gemm = lambda M, N, K: 2.0 * M * N * K
        gbytes = lambda N, K, R: S.nv(M, K) + S.nv(N, K) + 2 * M * N + 2 * M * 2 * R + 2 * K * R
        # U = s dY B as hi|lo: dY [M x N] and B [N x R] in, U [M x 2R] out
        lora_u = lambda N, R: 2 * M * N + 2 * N * R + 2 * M * 2 * R
        nku = lambda N, seg: P.pact_lora_bwd_u_launches(M, N, r, seg)   # 1 unsplit, 2 with a finalize
        # dA, dB: dY [M x N], the saved input (x_bytes), U [M x 2R] and A [R x K] in; dA, dB out
        lora_bwd = lambda N, x_bytes, K, R: 2 * M * N + x_bytes + 2 * M * 2 * R + 2 * R * K + 2 * R * K + 2 * N * R
        LB = lambda K, R, nv: P.pact_lora_bwd_launches(M, K, R, nv)  # kernels of one pact_lora_bwd call
        return [
            # down projection
            # U streams d_out and writes its NVFP4 copy doq (the dgrad GEMM's input)
            Op("lora_bwd_u_down+q(dout)", lambda: P.pact_lora_bwd_u(d_out, self.b_d, r, [H], self.sc["d"], self.u_d,
                                                                    self.ws, dyq=self.doq),
               kernels=nku(H, [H]), bytes=lora_u(H, r) + S.nv(M, H)),
            Op("gemm_dgrad_down", lambda: P.pact_frozen_gemm_dgrad(self.doq, self.c_d, self.l_d_b, dx=self.dm),
               "gemm", gemm(S.M, I, H), bytes=gbytes(I, H, r)),
            Op("silu_mul_bwd_quant", lambda: P.pact_silu_mul_bwd_quant(self.dm, self.gq, self.uq, self.dgu,
                                                                       self.dguq, self.m_re),
               bytes=2 * M * I + 2 * S.nv(M, I) + 4 * M * I + S.nv(M, 2 * I) + 2 * M * I),
            Op("lora_bwd_down", lambda: P.pact_lora_bwd(d_out, self.a_d, self.u_d, r, [H], s, x=self.m_re,
                                                        dA=g["a_d"], dB=g["b_d"], workspace=self.ws_leaf["down"],
                                                        u_gexp=self.gexp["d"], grads_fp32=f32),
               kernels=LB(I, r, False), side=True,
               bytes=lora_bwd(H, 2 * M * I, I, r)),
            # gate|up
            Op("lora_bwd_u_gu", lambda: P.pact_lora_bwd_u(self.dgu, self.b_gu, r, self.seg_gu, self.sc["gu"], self.u_gu,
                                                          self.ws),
               kernels=nku(2 * I, self.seg_gu), bytes=lora_u(2 * I, 2 * r)),
            Op("gemm_dgrad_gu", lambda: P.pact_frozen_gemm_dgrad(self.dguq, self.c_gu, self.l_gu_b, dx=self.dx2),
               "gemm", gemm(S.M, H, 2 * I), bytes=gbytes(H, 2 * I, 2 * r)),
            Op("lora_bwd_gu", lambda: P.pact_lora_bwd(self.dgu, self.a_gu, self.u_gu, r, self.seg_gu, s,
                                                      xq=self.xq2, dA=g["a_gu"], dB=g["b_gu"],
                                                      workspace=self.ws_leaf["gu"], u_gexp=self.gexp["gu"], grads_fp32=f32),
               kernels=LB(H, 2 * r, True), side=True, bytes=lora_bwd(2 * I, S.nv(M, H), H, 2 * r)),
            Op("rmsnorm_bwd_2", lambda: P.pact_rmsnorm_bwd(self.dx2, self.xq2, self.rstd2, self.g2, dres=d_out,
                                                           dx=self.dh2, dxq=self.dh2q),
               bytes=2 * M * H + S.nv(M, H) + 4 * M + 2 * H + 2 * M * H + 2 * M * H + S.nv(M, H)),
            # o projection (its output joined the residual stream h2)
            Op("lora_bwd_u_o", lambda: P.pact_lora_bwd_u(self.dh2, self.b_o, r, [H], self.sc["o"], self.u_o, self.ws),
               kernels=nku(H, [H]), bytes=lora_u(H, r)),
            Op("gemm_dgrad_o", lambda: P.pact_frozen_gemm_dgrad(self.dh2q, self.c_o, self.l_o_b, dx=self.dattn),
               "gemm", gemm(S.M, H, H), bytes=gbytes(H, H, r)),
            Op("lora_bwd_o", lambda: P.pact_lora_bwd(self.dh2, self.a_o, self.u_o, r, [H], s, x=attn,
                                                     dA=g["a_o"], dB=g["b_o"], workspace=self.ws_leaf["o"],
                                                     u_gexp=self.gexp["o"], grads_fp32=f32),
               kernels=LB(H, r, False), side=True,
               bytes=lora_bwd(H, 2 * M * H, H, r)),
            # q|k|v (d_qkv stands in for the attention backward)
            # U streams d_qkv and writes its NVFP4 copy dqkvq (the dgrad GEMM's input)
            Op("lora_bwd_u_qkv+q(dqkv)", lambda: P.pact_lora_bwd_u(d_qkv, self.b_qkv, r, self.seg_qkv, self.sc["qkv"],
                                                                   self.u_qkv, self.ws, dyq=self.dqkvq),
               kernels=nku(S.n_qkv, self.seg_qkv), bytes=lora_u(S.n_qkv, 3 * r) + S.nv(M, S.n_qkv)),
            Op("gemm_dgrad_qkv", lambda: P.pact_frozen_gemm_dgrad(self.dqkvq, self.c_qkv, self.l_qkv_b, dx=self.dx1),
               "gemm", gemm(S.M, H, S.n_qkv), bytes=gbytes(H, S.n_qkv, 3 * r)),
            Op("lora_bwd_qkv", lambda: P.pact_lora_bwd(d_qkv, self.a_qkv, self.u_qkv, r, self.seg_qkv, s,
                                                       xq=self.xq1, dA=g["a_qkv"], dB=g["b_qkv"],
                                                       workspace=self.ws_leaf["qkv"], u_gexp=self.gexp["qkv"], grads_fp32=f32),
               kernels=LB(H, 3 * r, True), side=True,
               bytes=lora_bwd(S.n_qkv, S.nv(M, H), H, 3 * r)),
            Op("rmsnorm_bwd_1", lambda: P.pact_rmsnorm_bwd(self.dx1, self.xq1, self.rstd1, self.g1, dres=self.dh2,
                                                           dx=self.dh),
               bytes=2 * M * H + S.nv(M, H) + 4 * M + 2 * H + 2 * M * H + 2 * M * H),
        ]

    def round_grads(self):
        """grads = BF16_RNE(grads32), one rounding of the (possibly summed) FP32 gradients."""
        P.pact_round_bf16(self.grad_bucket, self.grad_bucket_bf16)

    def saved_for_backward(self) -> Dict[str, torch.Tensor]:
        """The device tensors the forward leaves for the backward, i.e. the activation
        memory a layer holds between its forward and its backward: the NVFP4 copies
        (codes and padded scales) of both RMSNorm outputs and of gate and up, the two
        rstd vectors, and the attention output the o adapter's gradient reads.  The
        BF16 RMSNorm outputs, m and T are dead once the forward has used them."""
        _, attn, _, _ = self.inputs
        out = {"rstd1": self.rstd1, "rstd2": self.rstd2, "attn": attn}
        for name in ("xq1", "xq2", "gq", "uq"):
            t = getattr(self, name)
            out[name + ".codes"], out[name + ".scales"] = t.codes, t.scales
        return out

    def saved_bytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in self.saved_for_backward().values())

    def weight_cache_bytes(self) -> int:
        """Device bytes of the four cached weight groups (both layouts each)."""
        return sum(c.buf.numel() for c in (self.c_qkv, self.c_o, self.c_gu, self.c_d))

    def bf16_weight_bytes(self) -> int:
        """Bytes of the seven frozen weights in BF16."""
        return 2 * int(self.s.frozen_flops() / (4.0 * self.s.M))

    def step_ops(self) -> List[Op]:
        return self.forward_ops() + self.backward_ops()

    def step(self):
        for op in self.step_ops():
            op.fn()

    def step_concurrent(self, side: torch.cuda.Stream):
        """The step with its leaf ops (LoRA weight gradients) on the stream `side`, each
        ordered after everything issued before it on the current stream; the current
        stream waits for `side` at the end.  Same results as step(); under CUDA graph
        capture the leaves become a parallel branch of the graph."""
        run_concurrent(self.step_ops(), side)


def flat_views(shapes: Dict[str, tuple], dtype, dev):
    """One flat device buffer and a view of each requested shape in it, every view
    starting 16-byte aligned."""
    esz = torch.empty(0, dtype=dtype).element_size()
    step = 16 // esz
    offs, n = {}, 0
    for k, shp in shapes.items():
        offs[k] = n
        cnt = 1
        for d in shp:
            cnt *= d
        n += (cnt + step - 1) // step * step
    buf = torch.zeros(n, dtype=dtype, device=dev)
    views = {}
    for k, shp in shapes.items():
        cnt = 1
        for d in shp:
            cnt *= d
        views[k] = buf[offs[k]:offs[k] + cnt].view(shp)
    return buf, views


def run_concurrent(ops: List[Op], side: torch.cuda.Stream):
    """Run `ops` in order on the current stream, except the leaves (op.side), which
    run on `side` after everything issued before them; the current stream waits for
    `side` at the end."""
    main = torch.cuda.current_stream()
    for op in ops:
        if op.side:
            ready = torch.cuda.Event()
            ready.record(main)
            side.wait_event(ready)
            with torch.cuda.stream(side):
                op.fn()
        else:
            op.fn()
    done = torch.cuda.Event()
    done.record(side)
    main.wait_event(done)


class PactProjection:
    """One frozen projection with its BF16 LoRA branch, forward and backward: the
    single-projection workload (X[M x K], W[N x K], LoRA r, alpha).

      forward   xq = q(X);  T = s X A^T;  Y = deq(xq) deq(Wf)^T + T B^T
      backward  U = s dY B;  dX = deq(q(dY)) deq(Wb)^T + U A
                dA = U^T X~,  dB = s dY^T (X~ A^T)   with X~ = deq(xq), the saved copy

    (PACT blog summary, section "方法", bullets 1, 2 and 4 and the paragraph after
    them; PEFT explainer, section "LoRA").  Same interface as PactLayer: bind() the
    step's inputs, then step() / step_ops() / step_concurrent()."""

    input_keys = ("x", "dy")

    def __init__(self, W: torch.Tensor, A: torch.Tensor, B: torch.Tensor, M: int, r: int = 16,
                 alpha: float = 32.0):
        N, K = W.shape
        self.M, self.N, self.K, self.r = M, N, K, r
        self.scale = alpha / r
        dev = W.device
        self.c_w = P.pact_weight_layout_cache(W)
        self.A, self.B = A.contiguous(), B.contiguous()
        bf = lambda *sh: torch.empty(sh, dtype=torch.bfloat16, device=dev)
        self.xq, self.t, self.y = P.NVFP4Tensor.empty(M, K, dev), bf(M, 2 * r), bf(M, N)
        self.u, self.dyq, self.dx = bf(M, 2 * r), P.NVFP4Tensor.empty(M, N, dev), bf(M, K)
        self.grads = {"a": torch.empty_like(self.A), "b": torch.empty_like(self.B)}
        ws = max(P.pact_lora_fwd_workspace_bytes(M, K, r), P.pact_lora_bwd_u_workspace_bytes(M, N, r, 1))
        self.ws = PactLayer._scratch(ws, dev)
        self.ws_leaf = PactLayer._scratch(P.pact_lora_bwd_workspace_bytes(M, N, K, r, 1), dev)
        self.l_f = P.lora_struct(self.t, self.B, r, [N])
        self.l_b = P.lora_struct(self.u, self.A, r, [K])
        self.inputs = None

    def bind(self, x: torch.Tensor, dy: torch.Tensor):
        self.inputs = (x, dy)

    def forward_ops(self) -> List[Op]:
        M, N, K, r = self.M, self.N, self.K, self.r
        x, _ = self.inputs
        nv = lambda rows, cols: rows * cols / 2 + rows * cols / 16
        return [
            # the LoRA product streams x and writes its NVFP4 copy xq (the GEMM's input)
            Op("lora_fwd+q(x)", lambda: P.pact_lora_fwd(x, self.A, self.scale, self.t, self.ws, xq=self.xq),
               kernels=P.pact_lora_fwd_launches(M, K, r), bytes=2 * M * K + 2 * r * K + 2 * M * 2 * r + nv(M, K)),
            Op("gemm_fwd", lambda: P.pact_frozen_gemm_fwd(self.xq, self.c_w, self.l_f, y=self.y), "gemm",
               2.0 * M * N * K, bytes=nv(M, K) + nv(N, K) + 2 * M * N + 2 * M * 2 * r + 2 * N * r),
        ]

    def backward_ops(self) -> List[Op]:
        M, N, K, r = self.M, self.N, self.K, self.r
        _, dy = self.inputs
        g = self.grads
        nv = lambda rows, cols: rows * cols / 2 + rows * cols / 16
        return [
            # U streams dy and writes its NVFP4 copy dyq (the dgrad GEMM's input)
            Op("lora_bwd_u+q(dy)", lambda: P.pact_lora_bwd_u(dy, self.B, r, [N], self.scale, self.u, self.ws,
                                                             dyq=self.dyq),
               kernels=P.pact_lora_bwd_u_launches(M, N, r, [N]), bytes=2 * M * N + 2 * N * r + 2 * M * 2 * r + nv(M, N)),
            Op("gemm_dgrad", lambda: P.pact_frozen_gemm_dgrad(self.dyq, self.c_w, self.l_b, dx=self.dx), "gemm",
               2.0 * M * N * K, bytes=nv(M, N) + nv(N, K) + 2 * M * K + 2 * M * 2 * r + 2 * K * r),
            Op("lora_bwd", lambda: P.pact_lora_bwd(dy, self.A, self.u, r, [N], self.scale, xq=self.xq, dA=g["a"],
                                                   dB=g["b"], workspace=self.ws_leaf),
               kernels=P.pact_lora_bwd_launches(M, K, r, True), side=True,
               bytes=2 * M * N + nv(M, K) + 2 * M * 2 * r + 4 * r * K + 2 * N * r),
        ]

    def step_ops(self) -> List[Op]:
        return self.forward_ops() + self.backward_ops()

    def step(self):
        for op in self.step_ops():
            op.fn()

    def step_concurrent(self, side: torch.cuda.Stream):
        run_concurrent(self.step_ops(), side)

    def saved_bytes(self) -> int:
        """The forward leaves the NVFP4 copy of X (codes and padded scales) for the
        backward."""
        return self.xq.codes.numel() + self.xq.scales.numel()

    def weight_cache_bytes(self) -> int:
        return self.c_w.buf.numel()

    def bf16_weight_bytes(self) -> int:
        return 2 * self.N * self.K
