"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the CPU oracle.

This module holds no arithmetic of the method itself (no quantization, no
normalisation, no GEMM): it only draws tensors.  Every tensor is defined by a
tensor id; its seed is ``0x50414354 + id``.  Numbers come from a counter-based
splitmix64 stream (Steele, Lea & Flood, "Fast splittable pseudorandom number
generators", OOPSLA 2014) turned into normals by the Box-Muller transform, in
float64, then rounded to BF16 (round-to-nearest-even from the float32 value).

Tensor ids (one per role in a decoder layer; projection index p is
q=0, k=1, v=2, o=3, gate=4, up=5, down=6):
  X (layer input h) = 1, second RMSNorm input h2 = 2, W_p = 10+p, A_p = 20+p,
  B_p = 30+p, RMSNorm weights gamma_i = 40+i, upstream gradient of projection
  p = 50+p, attention output stand-in = 60, attention-backward stand-ins
  dq/dk/dv = 61..63, outlier mask of W_p = 70+p.

The workload shapes follow the models the PACT pages evaluate (Llama-3.2-1B/3B,
Qwen2.5-1.5B; PACT blog summary, section "实验数据" (results)).
"""
from __future__ import annotations

import numpy as np

SEED_BASE = 0x50414354
_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

PROJ = ("q", "k", "v", "o", "gate", "up", "down")


def _splitmix64(seed: int, n: int, offset: int = 0) -> np.ndarray:
    """Outputs offset+1 .. offset+n of splitmix64 started at state ``seed`` (counter
    form: output i is the finaliser of seed + i * golden)."""
    with np.errstate(over="ignore"):
        i = np.arange(offset + 1, offset + n + 1, dtype=np.uint64)
        z = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + i * _GOLDEN
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        z = z ^ (z >> np.uint64(31))
    return z


def uniform(tensor_id: int, n: int, offset: int = 0) -> np.ndarray:
    """Uniforms offset .. offset+n-1 in (0, 1) of the stream of ``tensor_id`` (float64)."""
    z = _splitmix64(SEED_BASE + tensor_id, n, offset)
    return ((z >> np.uint64(11)).astype(np.float64) + 0.5) * (2.0 ** -53)


def normal(tensor_id: int, n: int, offset: int = 0) -> np.ndarray:
    """Standard normals offset .. offset+n-1 of the stream of ``tensor_id`` (float64;
    Box-Muller over consecutive uniform pairs, normal 2j and 2j+1 from uniforms 2j
    and 2j+1; ``offset`` must be even)."""
    assert offset % 2 == 0
    m = (n + 1) // 2
    u = uniform(tensor_id, 2 * m, offset)
    r = np.sqrt(-2.0 * np.log(u[0::2]))
    t = 2.0 * np.pi * u[1::2]
    out = np.empty(2 * m, dtype=np.float64)
    out[0::2] = r * np.cos(t)
    out[1::2] = r * np.sin(t)
    return out[:n]


def f64_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """Round float64 -> float32 -> BF16 (RNE at each step); returns uint16 bits."""
    f = np.ascontiguousarray(v, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = (u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    return r.astype(np.uint16).reshape(np.shape(v))


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


_CHUNK = 1 << 22   # elements generated at a time (bounds the float64 temporaries)


def gaussian_bf16(tensor_id: int, shape, std: float = 1.0, mean: float = 0.0) -> np.ndarray:
    """BF16 bit pattern (uint16 array of ``shape``) of mean + std * N(0, 1)."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)

    def fill(o):
        k = min(_CHUNK, n - o)
        out[o:o + k] = f64_to_bf16_bits(mean + std * normal(tensor_id, k, o))

    starts = range(0, n, _CHUNK)
    if len(starts) > 1:   # chunks are independent (counter-based stream): numpy releases the GIL
        from concurrent.futures import ThreadPoolExecutor
        import os
        with ThreadPoolExecutor(max_workers=min(len(starts), os.cpu_count() or 1, 16)) as ex:
            list(ex.map(fill, starts))
    else:
        for o in starts:
            fill(o)
    return out.reshape(shape)


def weight_bf16(p: int, shape, outliers: bool = False) -> np.ndarray:
    """Frozen weight W_p ~ N(0, 0.02^2); with ``outliers`` a seeded Bernoulli(0.01)
    mask (tensor id 70+p) multiplies the chosen entries by 20."""
    n = int(np.prod(shape))
    w = 0.02 * normal(10 + p, n)
    if outliers:
        w = np.where(uniform(70 + p, n) < 0.01, 20.0 * w, w)
    return f64_to_bf16_bits(w).reshape(shape)


# --------------------------------------------------------------------------------------
# Workloads.  Decoder-layer shapes of the models in the PACT evaluation; token count
# M = batch x sequence.  LoRA rank 16, alpha 32 on all seven projections.
# --------------------------------------------------------------------------------------
LAYERS = {
    "llama-3.2-1b": dict(H=2048, I=8192, KV=512, batch=4, seq=512, outliers=False),
    "qwen2.5-1.5b": dict(H=1536, I=8960, KV=256, batch=1, seq=2048, outliers=False),
    "llama-3.2-3b": dict(H=3072, I=8192, KV=1024, batch=4, seq=2048, outliers=True),
}
LORA_R = 16
LORA_ALPHA = 32
RMS_EPS = 1e-5

# single projection + LoRA: X[256x512], W[512x512]
SINGLE = dict(M=256, N=512, K=512)


def single_inputs(r: int = LORA_R) -> dict:
    """BF16 bit arrays of the single-projection workload: X [M x K] ~ N(0, 1) (tensor
    id 1), W [N x K] ~ N(0, 0.02^2) (the q weight's stream, id 10), LoRA A [r x K] and
    B [N x r] ~ N(0, 0.02^2) (ids 20, 30), upstream gradient dY [M x N] ~ N(0, 1)
    (id 50)."""
    M, N, K = SINGLE["M"], SINGLE["N"], SINGLE["K"]
    return {"w": weight_bf16(0, (N, K)), "lora_a": gaussian_bf16(20, (r, K), std=0.02),
            "lora_b": gaussian_bf16(30, (N, r), std=0.02), "x": gaussian_bf16(1, (M, K)),
            "dy": gaussian_bf16(50, (M, N))}

# NVFP4 GEMM sweep: (N, K) x M
SWEEP_NK = [(2048, 2048), (512, 2048), (8192, 2048), (2048, 8192), (8960, 1536), (8192, 3072)]
SWEEP_M = [512, 2048, 8192, 32768]


def layer_shapes(name: str) -> dict:
    """Projection shapes (N, K) of one decoder layer, in PyTorch [out, in] order."""
    c = LAYERS[name]
    H, I, KV = c["H"], c["I"], c["KV"]
    return {
        "q": (H, H), "k": (KV, H), "v": (KV, H), "o": (H, H),
        "gate": (I, H), "up": (I, H), "down": (H, I),
    }


def tokens(name: str) -> int:
    c = LAYERS[name]
    return c["batch"] * c["seq"]


def layer_inputs(name: str, M: int = None, r: int = LORA_R) -> dict:
    """BF16 bit arrays of one decoder layer's weights and one step's inputs:
    frozen weights W_p ~ N(0, 0.02^2) (with the outlier mask when the workload has
    one), LoRA A_p [r, in] and B_p [out, r] ~ N(0, 0.02^2), RMSNorm weights
    gamma_i = 1 + N(0, 0.02^2), layer input h, attention-output stand-in attn,
    upstream gradient d_out and attention-backward stand-in d_qkv ~ N(0, 1)."""
    c = LAYERS[name]
    M = M or tokens(name)
    shp = layer_shapes(name)
    w, a, b = {}, {}, {}
    for p, proj in enumerate(PROJ):
        N, K = shp[proj]
        w[proj] = weight_bf16(p, (N, K), outliers=c["outliers"])
        a[proj] = gaussian_bf16(20 + p, (r, K), std=0.02)
        b[proj] = gaussian_bf16(30 + p, (N, r), std=0.02)
    H, KV = c["H"], c["KV"]
    return {
        "w": w, "lora_a": a, "lora_b": b,
        "gamma1": gaussian_bf16(40, (H,), std=0.02, mean=1.0),
        "gamma2": gaussian_bf16(41, (H,), std=0.02, mean=1.0),
        "h": gaussian_bf16(1, (M, H)),
        "attn": gaussian_bf16(60, (M, H)),
        "d_out": gaussian_bf16(56, (M, H)),
        "d_qkv": np.concatenate([gaussian_bf16(61, (M, H)), gaussian_bf16(62, (M, KV)),
                                 gaussian_bf16(63, (M, KV))], axis=1),
    }
