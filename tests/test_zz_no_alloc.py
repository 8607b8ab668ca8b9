"""The allocation-free LoRA forward (pact_lora_fwd_noalloc) against the workspace
version (pact_lora_fwd) and the oracle, through the C ABI.

pact_lora_fwd_noalloc serves callers that cannot allocate device memory where they
call the library; it keeps its scratch in an array inside the library's device
code, shared by every call and holding the last call's contents.  Two calls in a
row on different inputs check that stale contents from the first call do not leak
into the second.  The file's name makes pytest collect it after every other test
file, so a run that stops at the first failure has run everything else first; one
test repeats the check in a fresh Python process whose first libpact call is this
one (the device-address lookup then happens on that call)."""
import ctypes
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import synth
from tests.util import assert_close, to_dev, to_f64

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CASES = [(2048, 2048, 48, 1), (300, 8192, 16, 2)]   # two calls in a row, different inputs


def _noalloc(lib, x, a, M, K, R, scale):
    stream = torch.cuda.current_stream().cuda_stream
    t = torch.full((M, 2 * R), float("nan"), dtype=torch.bfloat16, device="cuda")
    st = lib.pact_lora_fwd_noalloc(x.data_ptr(), K, M, K, a.data_ptr(), R, ctypes.c_float(scale), t.data_ptr(),
                                   2 * R, ctypes.c_void_p(stream))
    return st, t


def test_lora_fwd_noalloc_matches_workspace_version_and_oracle(orc):
    import nvfp4_gemm_b200 as P
    lib = P.pact.lib
    torch.cuda.set_device(0)
    for M, K, R, seed in CASES:
        xb = synth.gaussian_bf16(100 + seed, (M, K))
        ab = synth.gaussian_bf16(110 + seed, (R, K), std=0.02)
        x, a = to_dev(xb), to_dev(ab)
        t_ref = P.pact_lora_fwd(x, a, 2.0)
        st, t = _noalloc(lib, x, a, M, K, R, 2.0)
        assert st == 0, P.pact_last_error()
        torch.cuda.synchronize()
        got = to_f64(t[:, :R]) + to_f64(t[:, R:])
        assert_close(got, 2.0 * orc.lora_t(synth.bf16_bits_to_f64(xb), ab), f"noalloc vs oracle, M={M} K={K} R={R}")
        assert np.array_equal(to_f64(t), to_f64(t_ref)), "noalloc and workspace versions differ"
    assert P.pact_get_device_status() == 0, P.pact_last_error()


def test_lora_fwd_noalloc_rejects_oversize():
    import nvfp4_gemm_b200 as P
    lib = P.pact.lib
    M, K, R = 1 << 17, 64, 64   # scratch need beyond the built-in 8 MiB
    x = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    a = torch.empty((R, K), dtype=torch.bfloat16, device="cuda")
    t = torch.empty((M, 2 * R), dtype=torch.bfloat16, device="cuda")
    st = lib.pact_lora_fwd_noalloc(x.data_ptr(), K, M, K, a.data_ptr(), R, ctypes.c_float(1.0), t.data_ptr(), 2 * R,
                                   None)
    assert st == 2 and "scratch" in P.pact_last_error()


_FRESH = r"""
import ctypes, sys
import numpy as np
import torch
sys.path.insert(0, {root!r})
import synth
import nvfp4_gemm_b200 as P
torch.cuda.set_device(0)
out = []
for M, K, R, seed in {cases!r}:
    x = torch.from_numpy(synth.gaussian_bf16(100 + seed, (M, K)).view(np.int16)).view(torch.bfloat16).cuda()
    a = torch.from_numpy(synth.gaussian_bf16(110 + seed, (R, K), std=0.02).view(np.int16)).view(torch.bfloat16).cuda()
    t = torch.full((M, 2 * R), float("nan"), dtype=torch.bfloat16, device="cuda")
    st = P.pact.lib.pact_lora_fwd_noalloc(x.data_ptr(), K, M, K, a.data_ptr(), R, ctypes.c_float(2.0), t.data_ptr(),
                                          2 * R, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, P.pact_last_error()
    ref = P.pact_lora_fwd(x, a, 2.0)
    torch.cuda.synchronize()
    out.append(bool(torch.equal(t.view(torch.int16), ref.view(torch.int16))))
assert P.pact_get_device_status() == 0, P.pact_last_error()
print("FRESH", out)
"""


def test_lora_fwd_noalloc_first_call_in_a_fresh_process():
    code = _FRESH.format(root=ROOT, cases=CASES)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
    assert "FRESH [True, True]" in r.stdout, r.stdout[-2000:]
