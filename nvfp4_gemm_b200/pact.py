"""Thin Python binding of libpact (include/pact.h): argument marshalling only.

Every function here has the name of the C entry point it calls.  Outputs the caller
does not pass are allocated with PyTorch (device memory is PyTorch's job); the
computation itself always runs in libpact's CUDA kernels.  There is no fallback:
if libpact.so cannot be loaded, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpact.so")

PACT_OK = 0
STATUS_NAMES = {0: "PACT_OK", 1: "PACT_ERR_INVALID_ARG", 2: "PACT_ERR_SHAPE", 3: "PACT_ERR_ALIGN",
                4: "PACT_ERR_CUDA", 5: "PACT_ERR_TIMEOUT", 6: "PACT_ERR_UNSUPPORTED"}


class PactError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class c_nvfp4(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("rows", ctypes.c_int64), ("cols", ctypes.c_int64)]


class c_weight_cache(ctypes.Structure):
    _fields_ = [("fwd", c_nvfp4), ("bwd", c_nvfp4), ("gexp", ctypes.c_int32)]


class c_lora(ctypes.Structure):
    _fields_ = [("act", ctypes.c_void_p), ("ld_act", ctypes.c_int64), ("weight", ctypes.c_void_p),
                ("ld_weight", ctypes.c_int64), ("r", ctypes.c_int), ("nseg", ctypes.c_int),
                ("seg_end", ctypes.c_int64 * 4)]


class c_lora_bwd(ctypes.Structure):
    _fields_ = [("M", ctypes.c_int64), ("N", ctypes.c_int64), ("K", ctypes.c_int64),
                ("dy", ctypes.c_void_p), ("lddy", ctypes.c_int64),
                ("x", ctypes.c_void_p), ("ldx", ctypes.c_int64),
                ("xq", ctypes.POINTER(c_nvfp4)),
                ("A", ctypes.c_void_p), ("U", ctypes.c_void_p), ("ldu", ctypes.c_int64),
                ("r", ctypes.c_int), ("nseg", ctypes.c_int), ("seg_end", ctypes.c_int64 * 4),
                ("scale", ctypes.c_float), ("u_gexp", ctypes.c_int), ("dA", ctypes.c_void_p),
                ("dB", ctypes.c_void_p), ("grads_fp32", ctypes.c_int)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libpact.so is not built ({LIB_PATH}); run nvfp4_gemm_b200/build.py")
    lib = ctypes.CDLL(LIB_PATH)
    P, I64, I, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
    S = ctypes.c_int
    NV = ctypes.POINTER(c_nvfp4)
    sig = {
        "pact_nvfp4_code_bytes": (ctypes.c_size_t, [I64, I64]),
        "pact_scale_bytes": (ctypes.c_size_t, [I64, I64]),
        "pact_weight_cache_bytes": (ctypes.c_size_t, [I64, I64]),
        "pact_quantize_nvfp4": (S, [P, I64, I64, I64, NV, P]),
        "pact_rmsnorm_quant": (S, [P, I64, P, F, I64, I64, NV, P, P, P]),
        "pact_silu_mul_quant": (S, [P, P, I64, I64, I64, P, NV, NV, NV, P]),
        "pact_weight_layout_cache": (S, [P, I64, I64, I64, P, ctypes.c_size_t, ctypes.POINTER(c_weight_cache), P]),
        "pact_weight_layout_cache_scaled": (S, [P, I64, I64, I64, I, P, ctypes.c_size_t,
                                                ctypes.POINTER(c_weight_cache), P]),
        "pact_absmax_bf16": (S, [P, I64, I64, I64, P, P]),
        "pact_two_level_exponent": (I, [F]),
        "pact_frozen_gemm_fwd": (S, [NV, ctypes.POINTER(c_weight_cache), ctypes.POINTER(c_lora), P, I64, P, I64, P]),
        "pact_frozen_gemm_dgrad": (S, [NV, ctypes.POINTER(c_weight_cache), ctypes.POINTER(c_lora), P, I64, P, I64,
                                       P]),
        "pact_frozen_gemm_fwd_quant": (S, [NV, ctypes.POINTER(c_weight_cache), ctypes.POINTER(c_lora), P, I64, P,
                                           I64, NV, I, P]),
        "pact_frozen_gemm_fwd_silu": (S, [NV, ctypes.POINTER(c_weight_cache), ctypes.POINTER(c_lora), P, I64, NV,
                                          NV, NV, P]),
        "pact_lora_fwd_workspace_bytes": (ctypes.c_size_t, [I64, I64, I]),
        "pact_lora_fwd": (S, [P, I64, I64, I64, P, I, F, P, I64, P, ctypes.c_size_t, P]),
        "pact_lora_fwd_quant": (S, [P, I64, I64, I64, P, I, F, P, I64, NV, P, ctypes.c_size_t, P]),
        "pact_lora_fwd_launches": (I, [I64, I64, I]),
        "pact_lora_fwd_silu": (S, [P, P, I64, I64, I64, P, I, F, P, I64, NV, P, I64, P, ctypes.c_size_t, P]),
        "pact_lora_fwd_noalloc": (S, [P, I64, I64, I64, P, I, F, P, I64, P]),
        "pact_lora_bwd_u_workspace_bytes": (ctypes.c_size_t, [I64, I64, I, I]),
        "pact_lora_bwd_u": (S, [P, I64, I64, I64, P, I, I, ctypes.POINTER(I64), F, P, I64, P, ctypes.c_size_t, P]),
        "pact_lora_bwd_u_quant": (S, [P, I64, I64, I64, P, I, I, ctypes.POINTER(I64), F, P, I64, NV, P,
                                      ctypes.c_size_t, P]),
        "pact_lora_bwd_u_launches": (I, [I64, I64, I, I, ctypes.POINTER(I64)]),
        "pact_lora_bwd_launches": (I, [I64, I64, I, I]),
        "pact_lora_bwd_workspace_bytes": (ctypes.c_size_t, [I64, I64, I64, I, I]),
        "pact_lora_bwd": (S, [ctypes.POINTER(c_lora_bwd), P, ctypes.c_size_t, P]),
        "pact_silu_mul_bwd_quant": (S, [P, I64, NV, NV, I64, I64, P, I64, NV, P, P]),
        "pact_rmsnorm_bwd": (S, [P, I64, NV, P, P, I64, I64, P, P, NV, P]),
        "pact_last_error": (ctypes.c_char_p, []),
        "pact_status_string": (ctypes.c_char_p, [S]),
        "pact_get_device_status": (S, [P]),
        "pact_abi_version": (I, []),
        "pact_selftest_wait_timeout": (S, [I64, P, P]),
        "pact_round_bf16": (S, [P, P, I64, P]),
        "pact_gptq_workspace_bytes": (ctypes.c_size_t, [I64, I64, I64]),
        "pact_gptq_nvfp4": (S, [P, I64, I64, I64, P, I64, I64, ctypes.c_double, P, ctypes.c_size_t, NV, P, P]),
        "pact_weight_layout_cache_from_nvfp4": (S, [NV, I, P, ctypes.c_size_t, ctypes.POINTER(c_weight_cache), P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()
lib = _lib


def _check(status: int):
    if status != PACT_OK:
        raise PactError(status, _lib.pact_last_error().decode())


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _bf16(t: torch.Tensor, name: str) -> torch.Tensor:
    if t.dtype != torch.bfloat16 or not t.is_cuda:
        raise TypeError(f"{name}: expected a CUDA bfloat16 tensor")
    if t.dim() == 2 and t.stride(1) != 1:
        raise ValueError(f"{name}: rows must be contiguous")
    return t


def _ld(t: torch.Tensor) -> int:
    return t.stride(0) if t.dim() == 2 else t.shape[-1]


# ------------------------------------------------------------------- tensor types
@dataclass
class NVFP4Tensor:
    """NVFP4 tensor [rows x cols]: codes (uint8, rows x cols/2) and scales (uint8,
    tiled layout of pact_scale_bytes(rows, cols) bytes), both on the device."""
    codes: torch.Tensor
    scales: torch.Tensor
    rows: int
    cols: int

    @staticmethod
    def empty(rows: int, cols: int, device="cuda") -> "NVFP4Tensor":
        codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=device)
        scales = torch.empty(int(_lib.pact_scale_bytes(rows, cols)), dtype=torch.uint8, device=device)
        return NVFP4Tensor(codes, scales, rows, cols)

    def c(self) -> c_nvfp4:
        return c_nvfp4(self.codes.data_ptr(), self.scales.data_ptr(), self.rows, self.cols)


@dataclass
class WeightCache:
    """The cached forward [N x K] and backward [K x N] NVFP4 layouts of one frozen weight."""
    buf: torch.Tensor
    cstruct: c_weight_cache
    N: int
    K: int

    @property
    def gexp(self) -> int:
        """The tensor exponent of a two-level cache (0 for the one-level layouts)."""
        return int(self.cstruct.gexp)

    @property
    def fwd(self) -> NVFP4Tensor:
        return self._view(self.cstruct.fwd)

    @property
    def bwd(self) -> NVFP4Tensor:
        return self._view(self.cstruct.bwd)

    def _view(self, s: c_nvfp4) -> NVFP4Tensor:
        base = self.buf.data_ptr()
        co = s.codes - base
        so = s.scales - base
        nc = int(_lib.pact_nvfp4_code_bytes(s.rows, s.cols))
        ns = int(_lib.pact_scale_bytes(s.rows, s.cols))
        return NVFP4Tensor(self.buf[co:co + nc].view(s.rows, s.cols // 2), self.buf[so:so + ns], s.rows, s.cols)


def lora_struct(act: torch.Tensor, weight: torch.Tensor, r: int, seg_end: Sequence[int]) -> c_lora:
    """The pact_lora_t of (act, weight).  The struct holds the two tensors, so their
    memory stays allocated for as long as the struct can reach a launch."""
    se = (ctypes.c_int64 * 4)(*(list(seg_end) + [0] * (4 - len(seg_end))))
    c = c_lora(act.data_ptr(), _ld(act), weight.data_ptr(), _ld(weight), r, len(seg_end), se)
    c._tensors = (act, weight)
    return c


# ------------------------------------------------------------------- entry points
def pact_nvfp4_code_bytes(rows: int, cols: int) -> int:
    return int(_lib.pact_nvfp4_code_bytes(rows, cols))


def pact_scale_bytes(rows: int, cols: int) -> int:
    return int(_lib.pact_scale_bytes(rows, cols))


def pact_weight_cache_bytes(N: int, K: int) -> int:
    return int(_lib.pact_weight_cache_bytes(N, K))


def pact_quantize_nvfp4(x: torch.Tensor, out: Optional[NVFP4Tensor] = None, stream=None) -> NVFP4Tensor:
    _bf16(x, "x")
    rows, cols = x.shape
    out = out or NVFP4Tensor.empty(rows, cols, x.device)
    s = out.c()
    _check(_lib.pact_quantize_nvfp4(x.data_ptr(), _ld(x), rows, cols, ctypes.byref(s), _stream(stream)))
    return out


def pact_rmsnorm_quant(x: torch.Tensor, gamma: torch.Tensor, eps: float, yq: Optional[NVFP4Tensor] = None,
                       y: Optional[torch.Tensor] = None, rstd: Optional[torch.Tensor] = None,
                       want_y: bool = True, want_rstd: bool = True, stream=None):
    _bf16(x, "x")
    M, H = x.shape
    yq = yq or NVFP4Tensor.empty(M, H, x.device)
    if y is None and want_y:
        y = torch.empty((M, H), dtype=torch.bfloat16, device=x.device)
    if rstd is None and want_rstd:
        rstd = torch.empty(M, dtype=torch.float32, device=x.device)
    s = yq.c()
    _check(_lib.pact_rmsnorm_quant(x.data_ptr(), _ld(x), gamma.data_ptr(), float(eps), M, H, ctypes.byref(s),
                                   _ptr(y), _ptr(rstd), _stream(stream)))
    return yq, y, rstd


def pact_silu_mul_quant(g: torch.Tensor, u: torch.Tensor, m: Optional[torch.Tensor] = None,
                        mq: Optional[NVFP4Tensor] = None, gq: Optional[NVFP4Tensor] = None,
                        uq: Optional[NVFP4Tensor] = None, want_m: bool = True, want_copies: bool = True,
                        stream=None):
    _bf16(g, "g")
    _bf16(u, "u")
    if _ld(g) != _ld(u):
        raise ValueError("g and u must share a row stride")
    M, I = g.shape
    if m is None and want_m:
        m = torch.empty((M, I), dtype=torch.bfloat16, device=g.device)
    mq = mq or NVFP4Tensor.empty(M, I, g.device)
    if want_copies:
        gq = gq or NVFP4Tensor.empty(M, I, g.device)
        uq = uq or NVFP4Tensor.empty(M, I, g.device)
    smq, sgq, suq = mq.c(), gq.c() if gq else None, uq.c() if uq else None
    _check(_lib.pact_silu_mul_quant(g.data_ptr(), u.data_ptr(), _ld(g), M, I, _ptr(m), ctypes.byref(smq),
                                    ctypes.byref(sgq) if sgq else None, ctypes.byref(suq) if suq else None,
                                    _stream(stream)))
    return m, mq, gq, uq


def pact_absmax_bf16(x: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """max |x| of a 2-D BF16 tensor, as a one-element FP32 device tensor."""
    _bf16(x, "x")
    if out is None:
        out = torch.empty(1, dtype=torch.float32, device=x.device)
    _check(_lib.pact_absmax_bf16(x.data_ptr(), _ld(x), x.shape[0], x.shape[1], out.data_ptr(), _stream(stream)))
    return out


def pact_two_level_exponent(amax: float) -> int:
    return int(_lib.pact_two_level_exponent(ctypes.c_float(amax)))


def pact_weight_layout_cache(W: torch.Tensor, stream=None, two_level: bool = False) -> WeightCache:
    """The cached layouts of W.  two_level: the variant with a per-tensor power of two
    (its exponent comes from pact_absmax_bf16 on the device; reading that one float
    back makes this call wait for the stream, once per frozen weight)."""
    _bf16(W, "W")
    N, K = W.shape
    nbytes = pact_weight_cache_bytes(N, K)
    buf = torch.empty(nbytes + 256, dtype=torch.uint8, device=W.device)
    off = (-buf.data_ptr()) % 256
    buf = buf[off:off + nbytes]
    c = c_weight_cache()
    if two_level:
        amax = pact_absmax_bf16(W, stream=stream)
        torch.cuda.synchronize(W.device)       # the kernel may run on a caller's stream
        gexp = pact_two_level_exponent(float(amax.cpu()))
        _check(_lib.pact_weight_layout_cache_scaled(W.data_ptr(), _ld(W), N, K, gexp, buf.data_ptr(), nbytes,
                                                    ctypes.byref(c), _stream(stream)))
    else:
        _check(_lib.pact_weight_layout_cache(W.data_ptr(), _ld(W), N, K, buf.data_ptr(), nbytes, ctypes.byref(c),
                                             _stream(stream)))
    return WeightCache(buf, c, N, K)


def pact_gptq_workspace_bytes(N: int, K: int, n: int) -> int:
    return int(_lib.pact_gptq_workspace_bytes(N, K, n))


def pact_gptq_nvfp4(W: torch.Tensor, X: torch.Tensor, damp: float = 0.01, out: Optional[NVFP4Tensor] = None,
                    workspace: Optional[torch.Tensor] = None, pivot_error: Optional[torch.Tensor] = None,
                    stream=None) -> NVFP4Tensor:
    """NVFP4-adapted GPTQ calibration of W [N x K] on calibration inputs X [n x K]:
    the calibrated forward NVFP4 layout of W."""
    _bf16(W, "W")
    _bf16(X, "X")
    N, K = W.shape
    n = X.shape[0]
    out = out or NVFP4Tensor.empty(N, K, W.device)
    need = pact_gptq_workspace_bytes(N, K, n)
    if workspace is None:
        raw = torch.empty(need + 256, dtype=torch.uint8, device=W.device)
        off = (-raw.data_ptr()) % 256
        workspace = raw[off:off + need]
    s = out.c()
    _check(_lib.pact_gptq_nvfp4(W.data_ptr(), _ld(W), N, K, X.data_ptr(), _ld(X), n, float(damp),
                                workspace.data_ptr(), workspace.numel(), ctypes.byref(s), _ptr(pivot_error),
                                _stream(stream)))
    return out


def pact_weight_layout_cache_from_nvfp4(wf: NVFP4Tensor, gexp: int = 0, stream=None) -> WeightCache:
    """The cached layouts of a weight given by its forward NVFP4 layout (e.g. a
    GPTQ-calibrated one)."""
    N, K = wf.rows, wf.cols
    nbytes = pact_weight_cache_bytes(N, K)
    buf = torch.empty(nbytes + 256, dtype=torch.uint8, device=wf.codes.device)
    off = (-buf.data_ptr()) % 256
    buf = buf[off:off + nbytes]
    c = c_weight_cache()
    s = wf.c()
    _check(_lib.pact_weight_layout_cache_from_nvfp4(ctypes.byref(s), int(gexp), buf.data_ptr(), nbytes,
                                                    ctypes.byref(c), _stream(stream)))
    return WeightCache(buf, c, N, K)


def pact_frozen_gemm_fwd(xq: NVFP4Tensor, w: WeightCache, lora: Optional[c_lora] = None,
                         residual: Optional[torch.Tensor] = None, y: Optional[torch.Tensor] = None,
                         stream=None) -> torch.Tensor:
    if y is None:
        y = torch.empty((xq.rows, w.N), dtype=torch.bfloat16, device=xq.codes.device)
    s = xq.c()
    _check(_lib.pact_frozen_gemm_fwd(ctypes.byref(s), ctypes.byref(w.cstruct),
                                     ctypes.byref(lora) if lora is not None else None,
                                     _ptr(residual), _ld(residual) if residual is not None else 0,
                                     y.data_ptr(), _ld(y), _stream(stream)))
    return y


def pact_frozen_gemm_fwd_quant(xq: NVFP4Tensor, w: WeightCache, yq: Sequence[NVFP4Tensor],
                               lora: Optional[c_lora] = None, residual: Optional[torch.Tensor] = None,
                               y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """pact_frozen_gemm_fwd that also writes the NVFP4 copy of y, split along the
    columns into the tensors of yq (1 or 2, in column order)."""
    if y is None:
        y = torch.empty((xq.rows, w.N), dtype=torch.bfloat16, device=xq.codes.device)
    s = xq.c()
    arr = (c_nvfp4 * len(yq))(*[t.c() for t in yq])
    _check(_lib.pact_frozen_gemm_fwd_quant(ctypes.byref(s), ctypes.byref(w.cstruct),
                                           ctypes.byref(lora) if lora is not None else None,
                                           _ptr(residual), _ld(residual) if residual is not None else 0,
                                           y.data_ptr(), _ld(y), arr, len(yq), _stream(stream)))
    return y


def pact_frozen_gemm_fwd_silu(xq: NVFP4Tensor, w: WeightCache, m: torch.Tensor, mq: NVFP4Tensor, gq: NVFP4Tensor,
                              uq: NVFP4Tensor, lora: Optional[c_lora] = None, stream=None) -> torch.Tensor:
    """The gate|up GEMM with the SiLU-multiply in its epilogue: m = BF16(silu(g) u)
    and the NVFP4 copies mq, gq, uq; g and u themselves are not written."""
    s, a, b, c = xq.c(), mq.c(), gq.c(), uq.c()
    _check(_lib.pact_frozen_gemm_fwd_silu(ctypes.byref(s), ctypes.byref(w.cstruct),
                                          ctypes.byref(lora) if lora is not None else None, m.data_ptr(), _ld(m),
                                          ctypes.byref(a), ctypes.byref(b), ctypes.byref(c), _stream(stream)))
    return m


def pact_frozen_gemm_dgrad(dyq: NVFP4Tensor, w: WeightCache, lora: Optional[c_lora] = None,
                           residual: Optional[torch.Tensor] = None, dx: Optional[torch.Tensor] = None,
                           stream=None) -> torch.Tensor:
    if dx is None:
        dx = torch.empty((dyq.rows, w.K), dtype=torch.bfloat16, device=dyq.codes.device)
    s = dyq.c()
    _check(_lib.pact_frozen_gemm_dgrad(ctypes.byref(s), ctypes.byref(w.cstruct),
                                       ctypes.byref(lora) if lora is not None else None,
                                       _ptr(residual), _ld(residual) if residual is not None else 0,
                                       dx.data_ptr(), _ld(dx), _stream(stream)))
    return dx


def _workspace(ws: Optional[torch.Tensor], need: int, device) -> torch.Tensor:
    if ws is None:
        ws = torch.empty(need, dtype=torch.uint8, device=device)
    return ws


def pact_lora_fwd_workspace_bytes(M: int, K: int, R: int) -> int:
    return int(_lib.pact_lora_fwd_workspace_bytes(M, K, R))


def pact_lora_fwd(x: torch.Tensor, A: torch.Tensor, scale: float, T: Optional[torch.Tensor] = None,
                  workspace: Optional[torch.Tensor] = None, xq: Optional[NVFP4Tensor] = None,
                  stream=None) -> torch.Tensor:
    """T = scale x A^T as hi|lo BF16; with xq given (pact_lora_fwd_quant) the kernel
    also writes the NVFP4 copy of x into it."""
    _bf16(x, "x")
    _bf16(A, "A")
    M, K = x.shape
    R = A.shape[0]
    if T is None:
        T = torch.empty((M, 2 * R), dtype=torch.bfloat16, device=x.device)
    ws = _workspace(workspace, pact_lora_fwd_workspace_bytes(M, K, R), x.device)
    if xq is None:
        _check(_lib.pact_lora_fwd(x.data_ptr(), _ld(x), M, K, A.data_ptr(), R, float(scale), T.data_ptr(), _ld(T),
                                  ws.data_ptr(), ws.numel(), _stream(stream)))
    else:
        sq = xq.c()
        _check(_lib.pact_lora_fwd_quant(x.data_ptr(), _ld(x), M, K, A.data_ptr(), R, float(scale), T.data_ptr(),
                                        _ld(T), ctypes.byref(sq), ws.data_ptr(), ws.numel(), _stream(stream)))
    return T


def pact_lora_fwd_silu(g: torch.Tensor, u: torch.Tensor, A: torch.Tensor, scale: float, mq: NVFP4Tensor,
                       T: Optional[torch.Tensor] = None, m: Optional[torch.Tensor] = None,
                       workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """T = scale m A^T and mq = q(m) for m = silu(g) u, in one kernel; m itself is
    written only into a given `m`."""
    _bf16(g, "g")
    _bf16(u, "u")
    _bf16(A, "A")
    if _ld(g) != _ld(u):
        raise ValueError("g and u must share a row stride")
    M, I = g.shape
    R = A.shape[0]
    if T is None:
        T = torch.empty((M, 2 * R), dtype=torch.bfloat16, device=g.device)
    ws = _workspace(workspace, pact_lora_fwd_workspace_bytes(M, I, R), g.device)
    sq = mq.c()
    _check(_lib.pact_lora_fwd_silu(g.data_ptr(), u.data_ptr(), _ld(g), M, I, A.data_ptr(), R, float(scale),
                                   T.data_ptr(), _ld(T), ctypes.byref(sq), _ptr(m), _ld(m) if m is not None else 0,
                                   ws.data_ptr(), ws.numel(), _stream(stream)))
    return T


def pact_lora_fwd_launches(M: int, K: int, R: int) -> int:
    """Kernels one pact_lora_fwd call launches for these sizes (1 or 2)."""
    return int(_lib.pact_lora_fwd_launches(M, K, R))


def pact_lora_fwd_noalloc(x: torch.Tensor, A: torch.Tensor, scale: float, T: Optional[torch.Tensor] = None,
                          stream=None) -> torch.Tensor:
    """pact_lora_fwd without a workspace: the library's built-in device scratch is used."""
    _bf16(x, "x")
    _bf16(A, "A")
    M, K = x.shape
    R = A.shape[0]
    if T is None:
        T = torch.empty((M, 2 * R), dtype=torch.bfloat16, device=x.device)
    _check(_lib.pact_lora_fwd_noalloc(x.data_ptr(), _ld(x), M, K, A.data_ptr(), R, float(scale), T.data_ptr(), _ld(T),
                                      _stream(stream)))
    return T


def pact_lora_bwd_u_workspace_bytes(M: int, N: int, r: int, nseg: int) -> int:
    return int(_lib.pact_lora_bwd_u_workspace_bytes(M, N, r, nseg))


def pact_lora_bwd_u(dy: torch.Tensor, B: torch.Tensor, r: int, seg_end: Sequence[int], scale: float,
                    U: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                    dyq: Optional[NVFP4Tensor] = None, stream=None) -> torch.Tensor:
    """U = scale dY B per segment as hi|lo BF16; with dyq given (pact_lora_bwd_u_quant)
    the kernel also writes the NVFP4 copy of dY into it."""
    _bf16(dy, "dy")
    M, N = dy.shape
    if U is None:
        U = torch.empty((M, 2 * r * len(seg_end)), dtype=torch.bfloat16, device=dy.device)
    se = (ctypes.c_int64 * 4)(*(list(seg_end) + [0] * (4 - len(seg_end))))
    ws = _workspace(workspace, pact_lora_bwd_u_workspace_bytes(M, N, r, len(seg_end)), dy.device)
    if dyq is None:
        _check(_lib.pact_lora_bwd_u(dy.data_ptr(), _ld(dy), M, N, B.data_ptr(), r, len(seg_end), se, float(scale),
                                    U.data_ptr(), _ld(U), ws.data_ptr(), ws.numel(), _stream(stream)))
    else:
        sq = dyq.c()
        _check(_lib.pact_lora_bwd_u_quant(dy.data_ptr(), _ld(dy), M, N, B.data_ptr(), r, len(seg_end), se,
                                          float(scale), U.data_ptr(), _ld(U), ctypes.byref(sq), ws.data_ptr(),
                                          ws.numel(), _stream(stream)))
    return U


def pact_lora_bwd_launches(M: int, K: int, R: int, nvfp4_x: bool) -> int:
    """Kernels one pact_lora_bwd call launches for these sizes (4 or 5)."""
    return int(_lib.pact_lora_bwd_launches(M, K, R, int(bool(nvfp4_x))))


def pact_lora_bwd_u_launches(M: int, N: int, r: int, seg_end: Sequence[int]) -> int:
    """Kernels one pact_lora_bwd_u call launches for these sizes (1 or 2)."""
    se = (ctypes.c_int64 * 4)(*(list(seg_end) + [0] * (4 - len(seg_end))))
    return int(_lib.pact_lora_bwd_u_launches(M, N, r, len(seg_end), se))


def pact_lora_bwd_workspace_bytes(M: int, N: int, K: int, r: int, nseg: int) -> int:
    return int(_lib.pact_lora_bwd_workspace_bytes(M, N, K, r, nseg))


def pact_lora_bwd(dy: torch.Tensor, A: torch.Tensor, U: torch.Tensor, r: int, seg_end: Sequence[int], scale: float,
                  x: Optional[torch.Tensor] = None, xq: Optional[NVFP4Tensor] = None,
                  dA: Optional[torch.Tensor] = None, dB: Optional[torch.Tensor] = None,
                  workspace: Optional[torch.Tensor] = None, stream=None, u_gexp: int = 0, grads_fp32: bool = False):
    """dA, dB (BF16, or FP32 when grads_fp32: unrounded, for a later sum over replicas)."""
    _bf16(dy, "dy")
    M, N = dy.shape
    K = A.shape[1]
    nseg = len(seg_end)
    gdt = torch.float32 if grads_fp32 else torch.bfloat16
    if dA is None:
        dA = torch.empty((nseg * r, K), dtype=gdt, device=dy.device)
    if dB is None:
        dB = torch.empty((N, r), dtype=gdt, device=dy.device)
    if dA.dtype != gdt or dB.dtype != gdt:
        raise TypeError(f"dA and dB must be {gdt}")
    need = pact_lora_bwd_workspace_bytes(M, N, K, r, nseg)
    if workspace is None:
        workspace = torch.empty(need + 256, dtype=torch.uint8, device=dy.device)
        off = (-workspace.data_ptr()) % 256
        workspace = workspace[off:off + need]
    xq_s = xq.c() if xq is not None else None
    args = c_lora_bwd()
    args.M, args.N, args.K = M, N, K
    args.dy, args.lddy = dy.data_ptr(), _ld(dy)
    args.x, args.ldx = (x.data_ptr(), _ld(x)) if x is not None else (None, 0)
    args.xq = ctypes.pointer(xq_s) if xq_s is not None else None
    args.A, args.U, args.ldu = A.data_ptr(), U.data_ptr(), _ld(U)
    args.r, args.nseg = r, nseg
    for i in range(4):
        args.seg_end[i] = seg_end[i] if i < nseg else 0
    args.scale = float(scale)
    args.u_gexp = int(u_gexp)
    args.dA, args.dB = dA.data_ptr(), dB.data_ptr()
    args.grads_fp32 = int(bool(grads_fp32))
    _check(_lib.pact_lora_bwd(ctypes.byref(args), workspace.data_ptr(), workspace.numel(), _stream(stream)))
    return dA, dB


def pact_round_bf16(x: torch.Tensor, y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """BF16 rounding of a contiguous FP32 device tensor (same shape)."""
    if x.dtype != torch.float32 or not x.is_contiguous():
        raise TypeError("x: expected a contiguous float32 tensor")
    if y is None:
        y = torch.empty(x.shape, dtype=torch.bfloat16, device=x.device)
    _check(_lib.pact_round_bf16(x.data_ptr(), y.data_ptr(), x.numel(), _stream(stream)))
    return y


def pact_silu_mul_bwd_quant(dm: torch.Tensor, gq: NVFP4Tensor, uq: NVFP4Tensor, dgu: Optional[torch.Tensor] = None,
                            dguq: Optional[NVFP4Tensor] = None, m_re: Optional[torch.Tensor] = None,
                            want_m: bool = False, stream=None):
    _bf16(dm, "dm")
    M, I = dm.shape
    if dgu is None:
        dgu = torch.empty((M, 2 * I), dtype=torch.bfloat16, device=dm.device)
    dguq = dguq or NVFP4Tensor.empty(M, 2 * I, dm.device)
    if m_re is None and want_m:
        m_re = torch.empty((M, I), dtype=torch.bfloat16, device=dm.device)
    sg, su, sd = gq.c(), uq.c(), dguq.c()
    _check(_lib.pact_silu_mul_bwd_quant(dm.data_ptr(), _ld(dm), ctypes.byref(sg), ctypes.byref(su), M, I,
                                        dgu.data_ptr(), _ld(dgu), ctypes.byref(sd), _ptr(m_re), _stream(stream)))
    return dgu, dguq, m_re


def pact_rmsnorm_bwd(dy: torch.Tensor, yq: NVFP4Tensor, rstd: torch.Tensor, gamma: torch.Tensor,
                     dres: Optional[torch.Tensor] = None, dx: Optional[torch.Tensor] = None,
                     dxq: Optional[NVFP4Tensor] = None, want_q: bool = False, stream=None):
    _bf16(dy, "dy")
    M, H = dy.shape
    if dx is None:
        dx = torch.empty((M, H), dtype=torch.bfloat16, device=dy.device)
    if dxq is None and want_q:
        dxq = NVFP4Tensor.empty(M, H, dy.device)
    sy = yq.c()
    sq = dxq.c() if dxq is not None else None
    _check(_lib.pact_rmsnorm_bwd(dy.data_ptr(), _ld(dy), ctypes.byref(sy), rstd.data_ptr(), gamma.data_ptr(), M, H,
                                 _ptr(dres), dx.data_ptr(), ctypes.byref(sq) if sq else None, _stream(stream)))
    return dx, dxq


def pact_get_device_status(stream=None) -> int:
    return int(_lib.pact_get_device_status(_stream(stream)))


def pact_last_error() -> str:
    return _lib.pact_last_error().decode()


def pact_abi_version() -> int:
    return int(_lib.pact_abi_version())


def pact_selftest_wait_timeout(limit_cycles: int, waited: Optional[torch.Tensor] = None, stream=None) -> None:
    """Make one bounded device wait run out (see include/pact.h); `waited`, a one-element
    int64 device tensor, receives the cycles the wait took."""
    _check(_lib.pact_selftest_wait_timeout(int(limit_cycles), _ptr(waited), _stream(stream)))
