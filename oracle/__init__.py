"""FP64 CPU oracle for the PACT NVFP4 data flow (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its cpu_baseline and
``--impl reference`` legs) may import this package.  It shares no code with the CUDA
library in ``nvfp4_gemm_b200``; both sides only share the seeded input generator
in ``synth``.  The element-level definitions live in ``pact_oracle.c`` (compiled
with gcc, called through ctypes); this module composes them exactly as the data
flow on the PACT pages states it, with no blocking, fusion or reordering.

Citations (page and section):
  [FAQ]    PACT blog summary, section "相关问题" (FAQ), answer on NVFP4: 16 E2M1
           values share one E4M3 block scale, ~4.5 bit/element.
  [METHOD] same page, section "方法" (method), bullets 1, 2 and 4: NVFP4 GEMMs
           (FP32 accumulate, BF16 out) for the forward and the input gradient of the
           7 frozen projections; quantized RMSNorm output reused for backward;
           SiLU-multiply keeps BF16 forward inputs and saves NVFP4 gate/up copies;
           forward/backward weight layouts rebuilt, transposed, re-quantized, cached.
           The paragraph after the bullets: LoRA A, B stay BF16.
  [ABS]    PACT abstract (arxiv.science page): the same data flow.
  [LORA]   PEFT explainer (kongchang.com), section "LoRA": h = W0 x + B A x, with
           the alpha/r scaling of the LoRA update.

Parity pins: every function here is checked in tests/test_oracle_pins.py against
closed forms, exhaustive exact-rational enumeration, brute force and library
routines it does not use itself.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pact_oracle.c")
_LIB = os.path.join(_HERE, "_build", "libpact_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile pact_oracle.c with gcc (-O2, OpenMP, strict IEEE: no -ffast-math)."""
    os.makedirs(os.path.dirname(_LIB), exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-ffp-contract=off", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            I = ctypes.c_int64
            D = ctypes.c_double
            lib.orc_bf16_value.argtypes = [ctypes.c_uint16]
            lib.orc_bf16_value.restype = D
            lib.orc_bf16_rne.argtypes = [D]
            lib.orc_bf16_rne.restype = ctypes.c_uint16
            lib.orc_e4m3_value.argtypes = [ctypes.c_uint8]
            lib.orc_e4m3_value.restype = D
            lib.orc_e4m3_rne_sat.argtypes = [D]
            lib.orc_e4m3_rne_sat.restype = ctypes.c_uint8
            lib.orc_e2m1_value.argtypes = [ctypes.c_uint8]
            lib.orc_e2m1_value.restype = D
            lib.orc_e2m1_rne_mag.argtypes = [D]
            lib.orc_e2m1_rne_mag.restype = ctypes.c_uint8
            lib.orc_quantize.argtypes = [P, I, I, I, P, P]
            lib.orc_e2m1_codes_f64.argtypes = [P, P, I, P]
            lib.orc_e4m3_scales_f64.argtypes = [P, I, P]
            lib.orc_dequantize.argtypes = [P, P, I, I, P]
            lib.orc_scale_bytes.argtypes = [I, I]
            lib.orc_scale_bytes.restype = I
            lib.orc_scale_offset.argtypes = [I, I, I]
            lib.orc_scale_offset.restype = I
            lib.orc_pack_scales.argtypes = [P, I, I, P]
            lib.orc_unpack_scales.argtypes = [P, I, I, P]
            lib.orc_gemm_nt.argtypes = [P, P, I, I, I, P]
            lib.orc_rmsnorm.argtypes = [P, P, D, I, I, P, P]
            lib.orc_silu_mul.argtypes = [P, P, I, P]
            lib.orc_silu_mul_bwd.argtypes = [P, P, P, I, P, P]
            lib.orc_rmsnorm_bwd.argtypes = [P, P, P, P, I, I, P]
            lib.orc_num_threads.restype = ctypes.c_int
            lib.orc_bf16_rne_array.argtypes = [P, I, P]
            _lib = lib
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return int(_load().orc_num_threads())


# ------------------------------------------------------------------ scalar formats
def bf16_value(bits: int) -> float:
    return _load().orc_bf16_value(bits)


def bf16_rne(v: float) -> int:
    return _load().orc_bf16_rne(v)


def e4m3_value(b: int) -> float:
    return _load().orc_e4m3_value(b)


def e4m3_rne_sat(v: float) -> int:
    return _load().orc_e4m3_rne_sat(v)


def e2m1_value(c: int) -> float:
    return _load().orc_e2m1_value(c)


def e2m1_rne_mag(q: float) -> int:
    return _load().orc_e2m1_rne_mag(q)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact BF16 -> float64 (a widening of the bit pattern)."""
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f64_to_bf16(v: np.ndarray) -> np.ndarray:
    """Single-rounding RNE float64 -> BF16 bits, element by element (orc_bf16_rne)."""
    flat = _c(np.asarray(v, dtype=np.float64).ravel(), np.float64)
    out = np.empty(flat.size, dtype=np.uint16)
    if flat.size:
        _load().orc_bf16_rne_array(_p(flat), flat.size, _p(out))
    return out.reshape(np.shape(v))


# --------------------------------------------------------------------- NVFP4 tensors
class NVFP4:
    """An NVFP4 tensor as the oracle holds it: codes [rows x cols/2] (low nibble =
    even element), plain row-major scales [rows x cols/16] (E4M3 bytes)."""

    def __init__(self, codes: np.ndarray, scales: np.ndarray, rows: int, cols: int):
        self.codes, self.scales, self.rows, self.cols = codes, scales, rows, cols
        self._deq = None

    def dequantize(self) -> np.ndarray:
        """Dequantized values (computed once per tensor; the tensor is immutable)."""
        if self._deq is None:
            self._deq = dequantize(self)
            self._deq.flags.writeable = False
        return self._deq

    def rows_slice(self, rows) -> "NVFP4":
        """The NVFP4 tensor made of the given rows (blocks run along rows, so a row
        subset is itself a valid NVFP4 tensor)."""
        idx = np.asarray(rows)
        return NVFP4(self.codes[idx], self.scales[idx], len(idx), self.cols)

    def packed_scales(self) -> np.ndarray:
        return pack_scales(self.scales, self.rows, self.cols)


def quantize(x_bits: np.ndarray) -> NVFP4:
    """NVFP4 quantization of a 2-D BF16 array along its last dimension ([FAQ])."""
    x = _c(x_bits, np.uint16)
    rows, cols = x.shape
    assert cols % 16 == 0
    codes = np.empty((rows, cols // 2), dtype=np.uint8)
    scales = np.empty((rows, cols // 16), dtype=np.uint8)
    if rows:
        _load().orc_quantize(_p(x), cols, rows, cols, _p(codes), _p(scales))
    return NVFP4(codes, scales, rows, cols)


def dequantize(t: NVFP4) -> np.ndarray:
    out = np.empty((t.rows, t.cols), dtype=np.float64)
    if t.rows:
        _load().orc_dequantize(_p(_c(t.codes, np.uint8)), _p(_c(t.scales, np.uint8)),
                               t.rows, t.cols, _p(out))
    return out


def scale_bytes(rows: int, cols: int) -> int:
    return int(_load().orc_scale_bytes(rows, cols))


def scale_offset(r: int, c: int, cols: int) -> int:
    return int(_load().orc_scale_offset(r, c, cols))


def pack_scales(plain: np.ndarray, rows: int, cols: int) -> np.ndarray:
    out = np.empty(scale_bytes(rows, cols), dtype=np.uint8)
    _load().orc_pack_scales(_p(_c(plain, np.uint8)), rows, cols, _p(out))
    return out


def unpack_scales(packed: np.ndarray, rows: int, cols: int) -> np.ndarray:
    out = np.empty((rows, cols // 16), dtype=np.uint8)
    _load().orc_unpack_scales(_p(_c(packed, np.uint8)), rows, cols, _p(out))
    return out


# ------------------------------------------------------------------------------ GEMM
def gemm_nt(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """C = A . B^T in float64, k ascending (plain triple loop in C)."""
    a = _c(a, np.float64)
    b = _c(b, np.float64)
    M, K = a.shape
    N, K2 = b.shape
    assert K == K2
    out = np.empty((M, N), dtype=np.float64)
    if M and N:
        _load().orc_gemm_nt(_p(a), _p(b), M, N, K, _p(out))
    return out


def nvfp4_gemm(aq: NVFP4, bq: NVFP4) -> np.ndarray:
    """[METHOD] NVFP4 GEMM: deq(A) . deq(B)^T, accumulated without rounding."""
    return gemm_nt(aq.dequantize(), bq.dequantize())


def weight_cache(w_bits: np.ndarray):
    """[METHOD] cached weight layouts.  Forward: Wf = q(W) along K (W is [N x K]).
    Backward: the forward layout is rebuilt (dequantized, exact in BF16), transposed
    to [K x N] and re-quantized along N: Wb = q(deq(Wf)^T)."""
    wf = quantize(w_bits)
    wd = wf.dequantize()
    wd_bits = f64_to_bf16_exact(wd.T)
    wb = quantize(wd_bits)
    return wf, wb


# Two-level variant of the weight layouts (a reading; the pages give a single E4M3
# block scale, [FAQ]).  Weights drawn like N(0, 0.02^2) have block amax / 6 below
# E4M3's smallest normal (2^-6), so their block scales are subnormal and carry two or
# three significant bits.  The variant puts a per-tensor power of two 2^e in front:
# the cached codes and scales are those of W * 2^-e, with e the smallest integer
# for which the largest block scale does not saturate, and every product with the
# cached weight is multiplied back by 2^e.  A power of two keeps the scaling exact.
E2M1_MAX = 6.0
E4M3_MAX = 448.0


def two_level_exponent(amax: float) -> int:
    """The smallest integer e with amax <= 6 * 448 * 2^e (0 when amax is 0), by
    stepping e one at a time against exact powers of two."""
    top = E2M1_MAX * E4M3_MAX
    if not amax > 0.0:
        return 0
    e = 0
    while amax > top * 2.0 ** e:
        e += 1
    while amax <= top * 2.0 ** (e - 1):
        e -= 1
    return e


def weight_cache_two_level(w_bits: np.ndarray):
    """(e, Wf, Wb): e = two_level_exponent(max |W|); Wf, Wb = weight_cache(W * 2^-e).
    The scaled values are exact in BF16 wherever they can matter: a value scaled
    below BF16's normal range sits in a block whose codes it cannot change (its
    quotient by the block scale rounds to a signed zero, or the block scale itself is
    zero), and rounding keeps its sign."""
    w = bf16_to_f64(w_bits)
    e = two_level_exponent(float(np.max(np.abs(w))) if w.size else 0.0)
    wf, wb = weight_cache(f64_to_bf16(w * 2.0 ** -e))
    return e, wf, wb


def f64_to_bf16_exact(v: np.ndarray) -> np.ndarray:
    """Bits of float64 values that are exactly representable in BF16 (asserted)."""
    f = np.ascontiguousarray(v, dtype=np.float32)
    assert np.array_equal(f.astype(np.float64), np.asarray(v)), "value not exact in BF16"
    u = f.view(np.uint32)
    assert not np.any(u & 0xFFFF), "value not exact in BF16"
    return (u >> 16).astype(np.uint16)


# ---------------------------------------------------------------- fused producers
def rmsnorm_quant(x_bits: np.ndarray, gamma_bits: np.ndarray, eps: float):
    """[METHOD] RMSNorm + NVFP4 quantization of its BF16 output.
    Returns (y BF16 bits, q(y), rstd float64)."""
    x = _c(x_bits, np.uint16)
    g = _c(gamma_bits, np.uint16)
    M, H = x.shape
    y = np.empty((M, H), dtype=np.uint16)
    rstd = np.empty(M, dtype=np.float64)
    if M:
        _load().orc_rmsnorm(_p(x), _p(g), eps, M, H, _p(y), _p(rstd))
    return y, quantize(y), rstd


def silu_mul_quant(g_bits: np.ndarray, u_bits: np.ndarray):
    """[METHOD] SiLU-multiply from BF16 gate/up; returns (m BF16 bits, q(m), q(g), q(u))."""
    g = _c(g_bits, np.uint16)
    u = _c(u_bits, np.uint16)
    m = np.empty_like(g)
    if g.size:
        _load().orc_silu_mul(_p(g), _p(u), g.size, _p(m))
    return m, quantize(m), quantize(g), quantize(u)


def silu_mul_bwd(dm: np.ndarray, gq: NVFP4, uq: NVFP4):
    """Backward of m = silu(g) u at the dequantized saved NVFP4 copies; float64 (dg, du)."""
    return silu_mul_bwd_at(dm, dequantize(gq), dequantize(uq))


def silu_mul_bwd_at(dm: np.ndarray, gh: np.ndarray, uh: np.ndarray):
    """The same backward formula evaluated at given float64 g^, u^."""
    dm = _c(dm, np.float64)
    gh = _c(gh, np.float64)
    uh = _c(uh, np.float64)
    dg = np.empty_like(dm)
    du = np.empty_like(dm)
    if dm.size:
        _load().orc_silu_mul_bwd(_p(dm), _p(gh), _p(uh), dm.size, _p(dg), _p(du))
    return dg, du


def silu_mul_recompute(gq: NVFP4, uq: NVFP4) -> np.ndarray:
    """BF16 bits of m~ = BF16_RNE(silu(g^) u^) from the saved copies (the down
    projection's LoRA input in backward)."""
    gb = f64_to_bf16_exact(dequantize(gq))
    ub = f64_to_bf16_exact(dequantize(uq))
    m = np.empty_like(gb)
    if gb.size:
        _load().orc_silu_mul(_p(gb), _p(ub), gb.size, _p(m))
    return m


def rmsnorm_bwd(dy: np.ndarray, yq: NVFP4, rstd: np.ndarray, gamma_bits: np.ndarray) -> np.ndarray:
    """Backward of RMSNorm from the dequantized saved output; float64 dx."""
    return rmsnorm_bwd_at(dy, dequantize(yq), rstd, gamma_bits)


def rmsnorm_bwd_at(dy: np.ndarray, yh: np.ndarray, rstd: np.ndarray, gamma_bits: np.ndarray) -> np.ndarray:
    """The same backward formula evaluated at a given float64 output y^."""
    dy = _c(dy, np.float64)
    yh = _c(yh, np.float64)
    M, H = dy.shape
    dx = np.empty_like(dy)
    if M:
        _load().orc_rmsnorm_bwd(_p(dy), _p(yh), _p(_c(rstd, np.float64)),
                                _p(_c(gamma_bits, np.uint16)), M, H, _p(dx))
    return dx


# ---------------------------------------------------------------------------- LoRA
def lora_t(x: np.ndarray, a_bits: np.ndarray) -> np.ndarray:
    """T = X . A^T for float64 X [M x K] and BF16 A [r x K] ([LORA]: A x)."""
    return gemm_nt(x, bf16_to_f64(a_bits))


def frozen_fwd(xq: NVFP4, wf: NVFP4, x_bits=None, a_bits=None, b_bits=None, scale=0.0, gexp=0):
    """[METHOD]+[LORA] forward of one frozen projection with its LoRA branch:
    Y = 2^gexp deq(Xq) . deq(Wf)^T + scale * (X . A^T) . B^T, with BF16 X, A, B;
    float64 (gexp: the exponent of a two-level weight cache, else 0)."""
    y = 2.0 ** gexp * nvfp4_gemm(xq, wf)
    if a_bits is not None:
        t = lora_t(bf16_to_f64(x_bits), a_bits)
        y = y + scale * gemm_nt(t, bf16_to_f64(b_bits))
    return y


def frozen_dgrad(dy_bits: np.ndarray, wb: NVFP4, a_bits=None, b_bits=None, scale=0.0, gexp=0):
    """[METHOD]+[LORA] input gradient of one projection:
    dX = 2^gexp deq(q(dY)) . deq(Wb)^T + scale * (dY . B) . A, dY BF16; float64."""
    dx = 2.0 ** gexp * nvfp4_gemm(quantize(dy_bits), wb)
    if a_bits is not None:
        dy = bf16_to_f64(dy_bits)
        u = gemm_nt(dy, bf16_to_f64(b_bits).T)          # dY . B        [M x r]
        dx = dx + scale * gemm_nt(u, bf16_to_f64(a_bits).T)  # (dY B) . A  [M x K]
    return dx


def lora_bwd(dy_bits: np.ndarray, xt: np.ndarray, a_bits: np.ndarray, b_bits: np.ndarray, scale: float):
    """[LORA] weight gradients of h = scale * B A x for upstream dY (BF16) and the
    backward's view X~ of the input (float64):
      U  = dY . B                       [M x r]
      dB = scale * dY^T . (X~ . A^T)    [N x r]
      dA = scale * U^T . X~             [r x K]
    Returns (dA, dB, scale * U) in float64."""
    return lora_bwd_at(bf16_to_f64(dy_bits), xt, bf16_to_f64(a_bits), bf16_to_f64(b_bits), scale)


def lora_bwd_at(dy: np.ndarray, xt: np.ndarray, a: np.ndarray, b: np.ndarray, scale: float):
    """The same LoRA gradients for float64 dY, X~, A, B."""
    u = gemm_nt(dy, b.T)
    t = gemm_nt(xt, a)
    db = scale * gemm_nt(dy.T, t.T)
    da = scale * gemm_nt(u.T, xt.T)
    return da, db, scale * u


# ------------------------------------------------------------- saved activations
def saved_bytes_pact(M: int, H: int, I: int) -> int:
    """Bytes a PACT layer of M tokens holds from its forward for its backward
    ([METHOD] bullet 2: the quantized RMSNorm outputs are reused, gate and up are kept
    as NVFP4 copies; the o adapter reads the BF16 attention output): NVFP4 [M x H]
    twice and [M x I] twice (codes plus padded scales), two FP32 rstd vectors of M,
    and the BF16 attention output [M x H]."""
    nv = lambda rows, cols: rows * cols // 2 + scale_bytes(rows, cols)
    return 2 * nv(M, H) + 2 * nv(M, I) + 2 * 4 * M + 2 * M * H
