"""Host-side helpers of bench.py without a GPU: the guard that drops the recorded
DRAM traffic once the GEMM source changes, the BF16-LoRA saved-activation count,
and the NUMA lookup's fallback."""
import hashlib
import os

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_gemm_traffic_follows_the_source_hash():
    csrc = os.path.join(ROOT, "nvfp4_gemm_b200", "csrc")
    for workload, rec in bench.GEMM_TRAFFIC.items():
        same = all(hashlib.sha256(open(os.path.join(csrc, n), "rb").read()).hexdigest()[:16] == h
                   for n, h in rec["sha256_16"].items())
        assert bench.gemm_traffic(workload) == (rec["bytes_per_launch"] if same else None)
    assert bench.gemm_traffic("no-such-workload") is None


def test_bf16_lora_saved_bytes_hand_count():
    # M 10, H 64, I 128, r 16: h, h2 (2 * 2 * 640) + rstd (2 * 4 * 10) + x_norm1, attn,
    # x_norm2 (3 * 2 * 640) + m (2 * 1280) + gate, up (2 * 2 * 1280) + 7 * A x (7 * 2 * 160)
    want = 2560 + 80 + 3840 + 2560 + 5120 + 2240
    assert bench.bf16_lora_saved_bytes(10, 64, 128, 16) == want


def test_gpu_local_cpus_without_a_gpu_is_empty():
    import torch
    if torch.cuda.is_available():
        return
    assert bench.gpu_local_cpus(torch.device("cuda", 0)) == set()
