#!/usr/bin/env python
"""Benchmark of one PACT LoRA decoder layer step on B200.

A step is the forward and backward pass of the NVFP4 data flow through a decoder
layer's seven frozen projections (fused RMSNorm / SiLU-multiply quantizers, NVFP4
GEMMs with the fused BF16 LoRA branch, NVFP4 dgrad GEMMs on the cached transposed
weight layouts, LoRA weight gradients, the backward elementwise kernels), all in
libpact.  Inputs are seeded synthetic tensors shaped like a Llama-3.2-3B layer
(H 3072, I 8192, k/v 1024, batch 4 x seq 2048 = 8192 tokens, weights with 1% outliers
x20), LoRA r 16, alpha 32; --workload picks the Llama-3.2-1B or Qwen2.5-1.5B layer, or
`single` (one 512 x 512 projection with LoRA on X[256 x 512]).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl pact|reference] [--workload W]

prints one JSON line.  --impl reference times the CPU oracle (the plain FP64
reference implementation) on the host cores on a bounded token sample of the
same workload, for exactly --steps steps.  Multi-GPU runs (torchrun) are data-parallel replicas: each rank
runs its own layer step on its own tokens and the LoRA gradients are all-reduced
over NCCL.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "NVFP4 frozen-proj fwd+dgrad TFLOPS & layer tokens/s; % of FP4 tensor peak"
WORKLOAD = "llama-3.2-3b"
# nominal dense FP4 / BF16 tensor throughput ratio on B200 (9 / 2.25 PFLOP/s)
FP4_PER_BF16 = 4.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("pact", "reference"), default="pact")
    ap.add_argument("--workload", default=WORKLOAD, choices=("llama-3.2-3b", "llama-3.2-1b", "qwen2.5-1.5b", "single"))
    ap.add_argument("--cpu-tokens", type=int, default=64, help="token sample of the CPU oracle baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sweep", action="store_true",
                    help="NVFP4 GEMM shape sweep (N x K x M, forward and dgrad): one JSON line per shape")
    ap.add_argument("--gemm", type=int, nargs=3, metavar=("N", "K", "M"),
                    help="time one NVFP4 GEMM shape (forward and dgrad) instead of the layer step")
    ap.add_argument("--ops", action="store_true",
                    help="time each op of the layer step alone: one JSON line per op with its roofline")
    ap.add_argument("--only", default=None, help="with --ops: time only the ops whose name contains this")
    ap.add_argument("--gptq", action="store_true",
                    help="time the NVFP4-adapted GPTQ calibration of each weight group of the layer (one JSON line "
                         "per group)")
    ap.add_argument("--calib-tokens", type=int, default=512, help="calibration tokens for --gptq")
    ap.add_argument("--two-level", action="store_true",
                    help="cache the frozen weights in the two-level variant (a power of two per tensor)")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16": float(d["bf16_tflops"]),
                "bf16_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "src": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "src": "fallback"}


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples (every 200 ms) while the timed region runs."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=2)

    def summary(self):
        sm, mx, reasons = [], 0.0, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[0]))
                mx = max(mx, float(f[1]))
            except ValueError:
                continue
            for n, v in zip(names, f[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx or None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ data-parallel replicas
class Replicas:
    """The host side of a multi-GPU run: one process per GPU (torchrun's RANK,
    WORLD_SIZE, LOCAL_RANK), each a full replica of the layer step on its own
    tokens.  The only exchange is the sum of the LoRA weight gradients: each rank's
    backward writes them unrounded in FP32 into one flat buffer, one all-reduce sums
    the buffer, and the sum is rounded to BF16 once.  Timings are reduced to their
    maximum over ranks; rank 0 alone prints.  `backend` is "nccl" on GPUs ("gloo"
    runs the same logic on CPU tensors)."""

    def __init__(self, backend: str = "nccl", device=None, timeout_s: float = 120.0):
        import datetime
        import torch.distributed as dist
        self.dist = dist
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.device = device
        if self.world > 1 and not dist.is_initialized():
            kw = {"device_id": device} if backend == "nccl" and device is not None else {}
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)

    def allreduce_bucket(self, bucket):
        """Sum one flat FP32 gradient buffer over the ranks, in place, in one collective
        (every rank calls it at the same point of every step)."""
        import torch
        if bucket.dtype != torch.float32 or not bucket.is_contiguous() or bucket.dim() != 1:
            raise TypeError("the gradient bucket is one flat contiguous float32 tensor")
        if self.world > 1:
            self.dist.all_reduce(bucket)

    def max_over_ranks(self, value: float) -> float:
        if self.world == 1:
            return value
        import torch
        t = torch.tensor([value], dtype=torch.float64, device=self.device if self.device is not None else "cpu")
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def barrier(self):
        if self.world > 1:
            self.dist.barrier()

    def emit(self, line: dict):
        """Print the JSON line on rank 0 only."""
        if self.rank == 0:
            print(json.dumps(line), flush=True)

    def close(self):
        if self.world > 1 and self.dist.is_initialized():
            self.dist.destroy_process_group()


# ------------------------------------------------------------------ CPU oracle
# DRAM bytes (read + write) per k_nvfp4_gemm launch, mean over the GEMMs of one layer
# step, from one ncu capture of the step's first eager pass (cold L2), per workload.
# Valid only for the GEMM source it was taken on: reported as null once csrc/gemm.cu,
# csrc/common.cuh or csrc/quant.cuh (the epilogue's quantizer) differ from the
# recorded hashes.
GEMM_TRAFFIC = {
    "llama-3.2-3b": {"bytes_per_launch": 117337376,
                     "sha256_16": {"gemm.cu": "6416243381f4c318", "common.cuh": "0f3b4168a8204ce6",
                                   "quant.cuh": "fc9734f97b40c05b"}},
}


def gemm_traffic(workload):
    import hashlib
    rec = GEMM_TRAFFIC.get(workload)
    if rec is None:
        return None
    csrc = os.path.join(os.path.dirname(os.path.abspath(__file__)), "nvfp4_gemm_b200", "csrc")
    for name, h in rec["sha256_16"].items():
        with open(os.path.join(csrc, name), "rb") as f:
            if hashlib.sha256(f.read()).hexdigest()[:16] != h:
                return None
    return rec["bytes_per_launch"]


def gpu_local_cpus(dev):
    """The CPUs NVML lists as local to the GPU (its NUMA node), within this process's
    allowed set; empty when NVML cannot tell."""
    import torch
    try:
        import pynvml
        props = torch.cuda.get_device_properties(dev)
        pynvml.nvmlInit()
        try:
            h = pynvml.nvmlDeviceGetHandleByPciBusId(
                f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0")
            words = pynvml.nvmlDeviceGetCpuAffinity(h, (os.cpu_count() + 63) // 64)
        finally:
            pynvml.nvmlShutdown()
        cpus = {64 * i + b for i, w in enumerate(words) for b in range(64) if (int(w) >> b) & 1}
        return cpus & os.sched_getaffinity(0)
    except Exception:
        return set()


def bf16_lora_saved_bytes(M, H, I, r):
    """Activation bytes a plain BF16 LoRA layer of the same scope (attention core
    excluded) keeps for its backward under autograd: the RMSNorm inputs h and h2 (BF16)
    and their rstd (FP32); the adapters' inputs x_norm1 (shared by q, k, v), attn,
    x_norm2 (shared by gate, up) and m; gate and up for the SiLU-multiply backward;
    the rank-r intermediates A x of the seven adapters (BF16)."""
    return 2 * 2 * M * H + 2 * 4 * M + 3 * 2 * M * H + 2 * M * I + 2 * 2 * M * I + 7 * 2 * M * r


def bf16_lora_saved_bytes_measured(name, dev, M=None):
    """Bytes PyTorch autograd actually keeps for the backward of a plain BF16 LoRA
    decoder layer of the same scope as the PACT layer (RMSNorm, the seven projections
    with frozen BF16 weights and trainable BF16 adapters, SiLU-multiply, both
    residuals; the attention core excluded, its output a given BF16 tensor), counted
    with saved-tensor hooks during the forward: every saved activation storage once,
    the weights and adapters (parameters, not activations) excluded.  A comparison
    model in PyTorch ops, not part of the PACT path."""
    import torch
    import torch.nn.functional as F
    import synth
    c = synth.LAYERS[name]
    M = M or synth.tokens(name)
    H, I, r = c["H"], c["I"], synth.LORA_R
    s = synth.LORA_ALPHA / r
    gen = torch.Generator(device=dev).manual_seed(0)
    rnd = lambda *sh, std=1.0: (torch.randn(sh, device=dev, generator=gen) * std).to(torch.bfloat16)
    shapes = synth.layer_shapes(name)
    W = {p: rnd(*shapes[p], std=0.02) for p in synth.PROJ}
    A = {p: rnd(r, shapes[p][1], std=0.02).requires_grad_() for p in synth.PROJ}
    B = {p: rnd(shapes[p][0], r, std=0.02).requires_grad_() for p in synth.PROJ}
    g1, g2 = (1 + rnd(H, std=0.02)), (1 + rnd(H, std=0.02))
    params = {t.untyped_storage().data_ptr() for d in (W, A, B) for t in d.values()} | {
        g1.untyped_storage().data_ptr(), g2.untyped_storage().data_ptr()}
    seen = {}

    def pack(t):
        st = t.untyped_storage()
        if st.data_ptr() not in params:
            seen[st.data_ptr()] = st.nbytes()
        return t

    h, attn = rnd(M, H).requires_grad_(), rnd(M, H).requires_grad_()
    lin = lambda x, p: F.linear(x, W[p]) + s * F.linear(F.linear(x, A[p]), B[p])
    with torch.autograd.graph.saved_tensors_hooks(pack, lambda t: t):
        x1 = F.rms_norm(h, (H,), g1, synth.RMS_EPS)
        q, k, v = lin(x1, "q"), lin(x1, "k"), lin(x1, "v")
        h2 = h + lin(attn, "o")
        x2 = F.rms_norm(h2, (H,), g2, synth.RMS_EPS)
        m = F.silu(lin(x2, "gate")) * lin(x2, "up")
        out = h2 + lin(m, "down")
    del q, k, v, out
    return int(sum(seen.values()))


def oracle_layer(name, inputs, two_level=False):
    import oracle
    from oracle.layer import OracleLayer, OracleProjection
    import synth
    oracle.build()
    if name == "single":
        return OracleProjection(inputs["w"], inputs["lora_a"], inputs["lora_b"], synth.LORA_R, synth.LORA_ALPHA)
    c = synth.LAYERS[name]
    return OracleLayer(c["H"], c["I"], c["KV"], synth.LORA_R, synth.LORA_ALPHA, synth.RMS_EPS, inputs["w"],
                       inputs["lora_a"], inputs["lora_b"], inputs["gamma1"], inputs["gamma2"], two_level=two_level)


def oracle_rate(layer, inputs, tokens, min_seconds=10.0, max_steps=20, exact_steps=None):
    """Tokens/s of the oracle's step on the first `tokens` tokens: steps until
    `min_seconds` have passed or `max_steps` ran, or exactly `exact_steps` steps."""
    import oracle
    sl = slice(0, tokens)
    args = tuple(inputs[k][sl] for k in layer.input_keys)
    t0 = time.perf_counter()
    n = 0
    while True:
        layer.step(*args)
        n += 1
        el = time.perf_counter() - t0
        if exact_steps is not None:
            if n >= exact_steps:
                break
        elif el >= min_seconds or n >= max_steps:
            break
    return n * tokens / el, n, el, oracle.num_threads()


def cpu_sample_tokens(a, M):
    """Tokens per oracle step: the whole single-projection workload (256 tokens, well
    under a second), else a sample of --cpu-tokens of the layer's tokens."""
    return M if a.workload == "single" else max(8, min(a.cpu_tokens, M))


def reference_arm(a):
    """--impl reference: the CPU oracle timed on the host cores (rank 0 only)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import synth
    M = workload_tokens(a.workload)
    inputs = workload_inputs(a.workload)
    layer = oracle_layer(a.workload, inputs, a.two_level)
    for _ in range(a.warmup):      # small untimed passes
        layer.step(*(inputs[k][:8] for k in layer.input_keys))
    tok = cpu_sample_tokens(a, M)
    rate, n, el, cores = oracle_rate(layer, inputs, tok, exact_steps=max(1, a.steps))
    sample = (f"{tok} of {M} tokens per step ({n} steps, {el:.1f} s), one "
              f"{'projection' if a.workload == 'single' else 'layer'} fwd+bwd; weight layouts cached before timing")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": rate, "unit": "tokens/s", "n_gpus": a.gpus,
        "steps": n, "warmup": a.warmup, "ms_per_step": 1000.0 * el / n, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_block(a.workload, M),
        "cpu_baseline": {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": rate, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def workload_tokens(name):
    import synth
    return synth.SINGLE["M"] if name == "single" else synth.tokens(name)


def workload_inputs(name):
    import synth
    return synth.single_inputs() if name == "single" else synth.layer_inputs(name)


def config_block(name, M):
    import synth
    if name == "single":
        c = synth.SINGLE
        return {"workload": "single frozen projection + LoRA fwd+bwd (X[256x512], W[512x512], r 16, alpha 32)",
                "M": c["M"], "N": c["N"], "K": c["K"], "tokens": M, "lora_r": synth.LORA_R,
                "lora_alpha": synth.LORA_ALPHA, "l2": "flushed between timed steps (256 MiB write)",
                "launch": "one CUDA graph per step (LoRA weight gradients on a parallel branch)"}
    c = synth.LAYERS[name]
    return {"workload": f"{name} decoder layer fwd+bwd: 7 NVFP4 frozen projections + LoRA",
            "H": c["H"], "I": c["I"], "kv": c["KV"], "tokens": M, "batch": c["batch"], "seq": c["seq"],
            "lora_r": synth.LORA_R, "lora_alpha": synth.LORA_ALPHA,
            "l2": "flushed between timed steps (256 MiB write)", "launch": "one CUDA graph per step (LoRA weight gradients on a parallel branch)"}


# ------------------------------------------------------------------ GPU arm
def make_layer(name, dev, two_level=False, grad_fp32=False):
    """The layer (or the single projection) of workload `name` on device `dev` with its
    seeded synthetic inputs bound."""
    import torch
    import synth
    from nvfp4_gemm_b200.layer import LayerShape, PactLayer, PactProjection
    d = lambda bits: torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)
    if name == "single":
        inputs = synth.single_inputs()
        layer = PactProjection(d(inputs["w"]), d(inputs["lora_a"]), d(inputs["lora_b"]), synth.SINGLE["M"],
                               synth.LORA_R, synth.LORA_ALPHA)
        x_in = {k: d(inputs[k]) for k in layer.input_keys}
        layer.bind(*(x_in[k] for k in layer.input_keys))
        return inputs, layer, x_in
    c = synth.LAYERS[name]
    M = synth.tokens(name)
    inputs = synth.layer_inputs(name)
    shape = LayerShape(M=M, H=c["H"], I=c["I"], KV=c["KV"], r=synth.LORA_R, alpha=synth.LORA_ALPHA,
                       eps=synth.RMS_EPS)
    layer = PactLayer(shape, {k: d(v) for k, v in inputs["w"].items()},
                      {k: d(v) for k, v in inputs["lora_a"].items()},
                      {k: d(v) for k, v in inputs["lora_b"].items()}, d(inputs["gamma1"]), d(inputs["gamma2"]),
                      two_level=two_level, grad_fp32=grad_fp32)
    x_in = {k: d(inputs[k]) for k in layer.input_keys}
    layer.bind(*(x_in[k] for k in layer.input_keys))
    return inputs, layer, x_in


def device_ms(fn, stream, flush, reps=8, samples=5):
    """Device time of one call of `fn` with a cold L2 and without launch overhead:
    (graph of reps x [flush, fn] - graph of reps x [flush]) / reps, each graph timed
    `samples` times with CUDA events on `stream`."""
    import torch
    graphs = []
    for with_op in (True, False):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for _ in range(reps):
                flush.zero_()
                if with_op:
                    fn()
        graphs.append(g)
    out = []
    with torch.cuda.stream(stream):
        for g in graphs:
            g.replay()
            tt = []
            for _ in range(samples):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                g.replay()
                e1.record(stream)
                tt.append((e0, e1))
            torch.cuda.synchronize()
            out.append(sum(x.elapsed_time(y) for x, y in tt) / samples)
    return max(out[0] - out[1], 1e-6) / reps


def op_table(a, layer, dev):
    """Each op of the step alone (device time per call, cold L2, no launch overhead),
    its algorithmic bytes / FLOPs and the fraction of the measured peak."""
    import torch
    import nvfp4_gemm_b200 as P
    pk = peaks()
    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        layer.step()          # every op once: per-device attributes, lazy init
    torch.cuda.synchronize()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for op in layer.step_ops():
        if a.only and a.only not in op.name:
            continue
        ms = device_ms(op.fn, stream, flush, reps=8, samples=max(3, a.steps))
        row = {"op": op.name, "kind": op.kind, "kernels": op.kernels, "us": round(ms * 1e3, 2),
               "bytes": op.bytes, "GBps": round(op.bytes / (ms / 1e3) / 1e9, 1),
               "frac_hbm": round(op.bytes / (ms / 1e3) / 1e9 / pk["hbm_gbs"], 3)}
        if op.kind == "gemm":
            tf = op.flops / (ms / 1e3) / 1e12
            row.update({"tflops": round(tf, 1), "frac_fp4_peak": round(tf / (FP4_PER_BF16 * pk["bf16"]), 3)})
        print(json.dumps(row), flush=True)
    if P.pact_get_device_status() != 0:
        raise RuntimeError(P.pact_last_error())


def gemm_sweep(a, shapes):
    """Time NVFP4 frozen GEMMs (forward Y = X W^T and dgrad dX = dY W) per shape;
    inputs X, dY ~ N(0, 1), W ~ N(0, 0.02^2); device time per launch with a cold L2
    and without launch overhead."""
    import torch
    import synth
    import nvfp4_gemm_b200 as P
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    d = lambda bits: torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)
    pk = peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)
    for N, K, M in shapes:
        w = d(synth.weight_bf16(0, (N, K)))
        wc = P.pact_weight_layout_cache(w)
        xq = P.pact_quantize_nvfp4(d(synth.gaussian_bf16(1, (M, K))))
        dyq = P.pact_quantize_nvfp4(d(synth.gaussian_bf16(50, (M, N))))
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        dx = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
        res = {}
        for kind, fn in (("fwd", lambda: P.pact_frozen_gemm_fwd(xq, wc, y=y)),
                         ("dgrad", lambda: P.pact_frozen_gemm_dgrad(dyq, wc, dx=dx))):
            for _ in range(max(3, a.warmup)):
                fn()
            med = device_ms(fn, stream, flush, reps=8, samples=max(3, a.steps))
            tf = 2.0 * M * N * K / (med / 1e3) / 1e12
            res[kind] = {"ms": med, "tflops": tf, "frac_fp4_peak": tf / (FP4_PER_BF16 * pk["bf16"])}
        if P.pact_get_device_status() != 0:
            raise RuntimeError(P.pact_last_error())
        print(json.dumps({"gemm": {"N": N, "K": K, "M": M}, **res,
                          "peak_note": f"{pk['src']} burst BF16 {pk['bf16']} TF/s x {FP4_PER_BF16}"}), flush=True)
        del w, wc, xq, dyq, y, dx
        torch.cuda.empty_cache()


def saved_block(name, layer, dev, M):
    """Activation bytes held from forward to backward: the PACT path's, against what
    autograd keeps for a plain BF16 LoRA layer of the same scope (measured with
    saved-tensor hooks) and the hand count of the same tensors."""
    if name == "single":
        return {"pact": layer.saved_bytes(), "note": "the NVFP4 copy of X"}
    import torch
    out = {"pact": layer.saved_bytes(),
           "bf16_lora_autograd": bf16_lora_saved_bytes_measured(name, dev, M),
           "bf16_lora_model": bf16_lora_saved_bytes(M, layer.s.H, layer.s.I, layer.s.r),
           "note": "bytes held from forward to backward per layer (PACT: the NVFP4 copies, rstd, attn) against "
                   "PyTorch autograd's saved tensors for a BF16 LoRA layer of the same scope (measured) and a hand "
                   "count of the tensors that layer needs"}
    torch.cuda.empty_cache()
    return out


def gptq_bench(a):
    """NVFP4-adapted GPTQ calibration of the workload's four weight groups (q|k|v, o,
    gate|up, down) on seeded synthetic calibration activations ~N(0, 1): device time
    per group (CUDA events on the launching stream), the FP64 work it implies, and
    the oracle on a sample of rows (GPTQ's rows are independent once H is fixed),
    scaled to the group."""
    import torch
    import synth
    import nvfp4_gemm_b200 as P
    from oracle import gptq as ogptq
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    c = synth.LAYERS[a.workload]
    shp = synth.layer_shapes(a.workload)
    d = lambda bits: torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)
    stream = torch.cuda.Stream(device=dev)
    for key, group in (("qkv", ("q", "k", "v")), ("o", ("o",)), ("gu", ("gate", "up")), ("d", ("down",))):
        w = np.concatenate([synth.weight_bf16(synth.PROJ.index(p), shp[p], outliers=c["outliers"]) for p in group], 0)
        N, K = w.shape
        x = synth.gaussian_bf16(91, (a.calib_tokens, K))
        wd, xd = d(w), d(x)
        out = P.NVFP4Tensor.empty(N, K, dev)
        need = P.pact_gptq_workspace_bytes(N, K, a.calib_tokens)
        raw = torch.empty(need + 256, dtype=torch.uint8, device=dev)
        off = (-raw.data_ptr()) % 256
        ws = raw[off:off + need]
        with torch.cuda.stream(stream):
            P.pact_gptq_nvfp4(wd, xd, 0.01, out=out, workspace=ws, stream=stream)   # warm-up
            torch.cuda.synchronize()
            times = []
            for _ in range(max(1, a.steps)):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                P.pact_gptq_nvfp4(wd, xd, 0.01, out=out, workspace=ws, stream=stream)
                e1.record(stream)
                torch.cuda.synchronize()
                times.append(e0.elapsed_time(e1))
        if P.pact_get_device_status() != 0:
            raise RuntimeError(P.pact_last_error())
        ms = statistics.median(times)
        n = a.calib_tokens
        flop = 2.0 * n * K * K + 2.0 * K ** 3 / 3.0 + 1.0 * N * K * K
        rows = 8
        t0 = time.perf_counter()
        ogptq.gptq_nvfp4(w[:rows], x)
        cpu_s = time.perf_counter() - t0
        print(json.dumps({"gptq": {"workload": a.workload, "group": key, "N": N, "K": K, "calib_tokens": n},
                          "ms": ms, "fp64_flop": flop, "fp64_tflops": flop / (ms / 1e3) / 1e12,
                          "oracle_s_for_8_rows": cpu_s,
                          "note": "FP64 work: H (2 n K^2), the factorisation and triangular inverse (2 K^3 / 3), "
                                  "the column pass (N K^2 / 2 multiply-subtract pairs)"}), flush=True)
        del wd, xd, out, raw, ws
        torch.cuda.empty_cache()


def main():
    a = parse()
    if a.impl == "reference":
        return reference_arm(a)
    if a.gptq:
        return gptq_bench(a)
    if a.gemm:
        return gemm_sweep(a, [tuple(a.gemm)])
    if a.sweep:
        import synth
        return gemm_sweep(a, [(n, k, m) for (n, k) in synth.SWEEP_NK for m in synth.SWEEP_M])

    import torch

    import synth
    import nvfp4_gemm_b200 as P

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    rep = Replicas("nccl", dev)
    world, rank = rep.world, rep.rank

    M = workload_tokens(a.workload)
    inputs, layer, x_in = make_layer(a.workload, dev, a.two_level, grad_fp32=world > 1)
    if a.ops:
        return op_table(a, layer, dev)
    ops = layer.step_ops()
    launches_per_step = sum(op.kernels for op in ops)

    # segments: each NVFP4 GEMM alone, consecutive other ops together
    segs = []
    for op in ops:
        if op.kind == "gemm" or not segs or segs[-1]["kind"] == "gemm":
            segs.append({"kind": op.kind, "ops": [op], "flops": op.flops})
        else:
            segs[-1]["ops"].append(op)
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for _ in range(2):           # eager passes: per-device attributes, lazy init
            layer.step()
    torch.cuda.synchronize()
    if P.pact_get_device_status() != 0:
        raise RuntimeError(P.pact_last_error())
    # the timed step: every op of the step in one CUDA graph (kernels back to back);
    # per-segment graphs give the breakdown in a separate pass after the timed region
    side = torch.cuda.Stream(device=dev)
    step_graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(step_graph, stream=stream):
        layer.step_concurrent(side)   # LoRA weight-gradient leaves on a parallel branch
    for sg in segs:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for op in sg["ops"]:
                op.fn()
        sg["graph"] = g
    torch.cuda.synchronize()

    def run_step():
        step_graph.replay()

    grads = list(layer.grads.values())

    def allreduce_grads():
        """Replicas: sum the FP32 gradient buffer over the ranks, then round it once."""
        if world > 1:
            rep.allreduce_bucket(layer.grad_bucket)
            layer.round_grads()

    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    with torch.cuda.stream(stream):
        for _ in range(a.warmup):
            flush.zero_()
            run_step()
            allreduce_grads()
    torch.cuda.synchronize()

    K = a.steps
    ev = lambda: torch.cuda.Event(enable_timing=True)
    st_ev = [(ev(), ev()) for _ in range(K)]
    rep.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        time.sleep(0.25)
        with torch.cuda.stream(stream):
            for k in range(K):
                flush.zero_()
                st_ev[k][0].record(stream)
                run_step()
                allreduce_grads()
                st_ev[k][1].record(stream)
        torch.cuda.synchronize()
        time.sleep(0.25)
    rep.barrier()
    step_ms = [s.elapsed_time(e) for s, e in st_ev]
    total_ms = sum(step_ms)
    # breakdown (not the timed number): each segment's graph alone, after a flush
    seg_ev = [[(ev(), ev()) for _ in segs] for _ in range(K)]
    with torch.cuda.stream(stream):
        for k in range(K):
            for i, sg in enumerate(segs):
                flush.zero_()
                seg_ev[k][i][0].record(stream)
                sg["graph"].replay()
                seg_ev[k][i][1].record(stream)
    torch.cuda.synchronize()
    seg_ms = [sum(seg_ev[k][i][0].elapsed_time(seg_ev[k][i][1]) for k in range(K)) / K for i in range(len(segs))]
    total_ms = rep.max_over_ranks(total_ms)
    ms_per_step = total_ms / K
    tokens_per_s = M * K * world / (total_ms / 1e3)

    # the dominant kernel (the NVFP4 GEMM): device time per launch, cold L2, no launch overhead
    gemm_ops = [op for op in ops if op.kind == "gemm"]
    gemm_flops = sum(op.flops for op in gemm_ops)
    gemm_ms = sum(device_ms(op.fn, stream, flush) for op in gemm_ops)
    gemm_launch_ms = gemm_ms / len(gemm_ops)
    tflops = gemm_flops / (gemm_ms / 1e3) / 1e12
    pk = peaks()
    fp4_peak = FP4_PER_BF16 * pk["bf16"]   # the GEMM is timed alone: burst peak

    # end to end, as a training loop runs it: every step's inputs come from pinned host
    # memory and the LoRA gradients go back to pinned host memory.  The inputs of a
    # step sit in one pinned buffer and travel as one copy (one DMA stream at full
    # PCIe rate); the copy of step k+1 runs on a copy stream while step k computes
    # (two device input sets, one captured step graph each).  The timed region spans
    # all K steps, from the first copy to the last gradient read-back.
    keys = layer.input_keys
    sizes = [x_in[k].numel() for k in keys]          # multiples of 8: every view is 16-byte aligned
    # pinned buffers on the GPU's NUMA node: allocated and first touched by this thread
    # while it runs on the GPU's local CPUs (the previous CPU set comes back after)
    allowed, local_cpus = os.sched_getaffinity(0), gpu_local_cpus(dev)
    if local_cpus:
        os.sched_setaffinity(0, local_cpus)
    try:
        host_flat = torch.empty(sum(sizes), dtype=torch.bfloat16, pin_memory=True)
        host_out = [torch.empty(gt.shape, dtype=gt.dtype, pin_memory=True) for gt in grads]
    finally:
        os.sched_setaffinity(0, allowed)
    dev_flat = [torch.empty(sum(sizes), dtype=torch.bfloat16, device=dev) for _ in range(2)]

    def views(flat):
        out, off = {}, 0
        for k, n in zip(keys, sizes):
            out[k] = flat[off:off + n].view(x_in[k].shape)
            off += n
        return out

    for k, v in views(host_flat).items():
        v.copy_(x_in[k].cpu())
    h2d = host_flat.numel() * host_flat.element_size()
    d2h = sum(t.numel() * t.element_size() for t in host_out)
    graphs = []
    for flat in dev_flat:
        sv = views(flat)
        layer.bind(*(sv[k] for k in keys))
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            layer.step_concurrent(side)
        graphs.append(g)
    layer.bind(*(x_in[k] for k in keys))
    copier = torch.cuda.Stream(device=dev)
    loaded = [torch.cuda.Event() for _ in range(K)]
    consumed = [torch.cuda.Event() for _ in range(K)]
    e_start, e_end = ev(), ev()
    torch.cuda.synchronize()
    e_start.record(stream)
    copier.wait_stream(stream)
    for k in range(K):
        slot = k % 2
        with torch.cuda.stream(copier):
            if k >= 2:
                copier.wait_event(consumed[k - 2])   # the step that read this input set is done
            dev_flat[slot].copy_(host_flat, non_blocking=True)
            loaded[k].record(copier)
        stream.wait_event(loaded[k])
        with torch.cuda.stream(stream):
            graphs[slot].replay()
            consumed[k].record(stream)
            allreduce_grads()
            for ho, gt in zip(host_out, grads):
                ho.copy_(gt, non_blocking=True)
    e_end.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e_start.elapsed_time(e_end)
    e2e_ms = rep.max_over_ranks(e2e_ms)
    if P.pact_get_device_status() != 0:
        raise RuntimeError(P.pact_last_error())

    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        ol = oracle_layer(a.workload, inputs, a.two_level)
        tok = cpu_sample_tokens(a, M)
        rate, n, el, cores = oracle_rate(ol, inputs, tok)
        cpu = {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": f"{tok} of {M} tokens per step ({n} steps, {el:.1f} s), one "
                         f"{'projection' if a.workload == 'single' else 'layer'} fwd+bwd on the FP64 CPU oracle; "
                         f"weight layouts cached before timing"}

    out = {
        "metric": METRIC, "value": tokens_per_s, "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": a.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "nvfp4", "data": "synthetic",
        "config": {**config_block(a.workload, M), "parallelism": f"dp{world}" if world > 1 else "single",
                   **({"weights": "two-level layouts (a power of two per cached tensor)"} if a.two_level else {})},
        "frozen_proj_tflops": tflops,
        "frac_fp4_peak": tflops / fp4_peak,
        "roofline": {"bound": "tensor", "kernel": "k_nvfp4_gemm (frozen fwd + dgrad GEMMs)",
                     "achieved": tflops, "peak": fp4_peak, "unit": "TFLOP/s", "frac": tflops / fp4_peak,
                     "traffic": gemm_traffic(a.workload),
                     "traffic_note": "DRAM read+write bytes per launch, mean over the 8 layer GEMMs, one ncu "
                                     "capture with cold L2 (outputs stay in L2); null when the GEMM source changed",
                     "peak_note": f"{pk['src']} burst BF16 {pk['bf16']} TF/s x {FP4_PER_BF16} "
                                  f"(nominal FP4/BF16 ratio); GEMM launches timed alone, cold L2",
                     "flops_per_step": gemm_flops, "avg_launch_ms": gemm_launch_ms},
        "cpu_baseline": cpu,
        "e2e": {"value": M * K * world / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "note": "inputs copied from pinned host memory every step, the next step's copy overlapping the "
                        "current step; LoRA gradients read back every step",
                "host_buffers": (f"pinned on the GPU's NUMA node ({len(local_cpus)} local CPUs)" if local_cpus
                                 else "pinned; the GPU's NUMA node unknown")},
        "saved_activation_bytes": saved_block(a.workload, layer, dev, M),
        "weight_bytes": {"pact_cached_layouts": layer.weight_cache_bytes(), "bf16": layer.bf16_weight_bytes()},
        "gpu_launches": launches_per_step * K,
        "clocks": clk.summary(),
        "segments_ms": {"+".join(op.name for op in sg["ops"]): round(t, 4) for sg, t in zip(segs, seg_ms)},
    }
    rep.emit(out)
    for sg in segs:
        sg["graph"] = None
    step_graph = graphs = None   # release every graph before the process group
    rep.close()


if __name__ == "__main__":
    main()
