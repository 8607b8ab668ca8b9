"""First library calls from several host threads at once.

The library keeps small per-device host caches: the SM count, whether each kernel's
shared-memory attribute has been set, the driver's tensor-map encoder.  Here four
threads of a fresh Python process make their first libpact calls together (weight
layouts, quantization, the frozen GEMM, the LoRA product, each on a stream of its
own), so those caches fill concurrently.  Every thread's outputs must equal, bit for
bit, those of the same calls made afterwards from one thread, and the device status
word must stay clear."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_CHILD = r"""
import sys, threading
sys.path.insert(0, {root!r})
import numpy as np, torch
import synth
import nvfp4_gemm_b200 as P

dev = torch.device("cuda:0")
def d(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)
M, N, K, r = 300, 512, 512, 16
x = d(synth.gaussian_bf16(1, (M, K)))
w = d(synth.weight_bf16(0, (N, K), outliers=True))
a = d(synth.gaussian_bf16(20, (r, K), std=0.02))
torch.cuda.synchronize()

def work():
    s = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(s):
        wc = P.pact_weight_layout_cache(w)
        xq = P.pact_quantize_nvfp4(x)
        y = P.pact_frozen_gemm_fwd(xq, wc)
        t = P.pact_lora_fwd(x, a, 2.0)
    s.synchronize()
    return [xq.codes, xq.scales, y, t]

out, errs = [None] * 4, []
def run(i):
    try:
        out[i] = work()
    except Exception as e:
        errs.append(repr(e))
ts = [threading.Thread(target=run, args=(i,)) for i in range(4)]
for t in ts:
    t.start()
for t in ts:
    t.join()
assert not errs, errs
ref = work()
same = [all(torch.equal(u.view(torch.uint8), v.view(torch.uint8)) for u, v in zip(o, ref)) for o in out]
print("THREADS", same, P.pact_get_device_status())
"""


def test_first_calls_from_several_host_threads():
    r = subprocess.run([sys.executable, "-c", _CHILD.format(root=ROOT)], capture_output=True, text=True, timeout=600,
                       cwd=ROOT)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
    assert "THREADS [True, True, True, True] 0" in r.stdout, r.stdout[-2000:]
