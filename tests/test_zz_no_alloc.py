"""The allocation-free LoRA forward (pact_lora_fwd_noalloc) against the workspace
version (pact_lora_fwd), through the C ABI.

pact_lora_fwd_noalloc serves callers that cannot allocate device memory where they
call the library; it keeps its scratch in an array inside the library's device
code, shared by every call and holding the last call's contents.  Two calls in a
row on different inputs check that stale contents from the first call do not leak
into the second.  This file is collected last on purpose: it runs alone in a fresh
process as well as after the other tests."""
import ctypes

import numpy as np
import pytest
import torch

import synth
from tests.util import assert_close, to_dev, to_f64

pytestmark = pytest.mark.gpu


def test_lora_fwd_noalloc_matches_workspace_version():
    import nvfp4_gemm_b200 as P
    lib = P.pact.lib
    torch.cuda.set_device(0)
    stream = torch.cuda.current_stream().cuda_stream
    cases = [(2048, 2048, 48, 1), (300, 8192, 16, 2)]   # two calls in a row, different inputs
    for M, K, R, seed in cases:
        x = to_dev(synth.gaussian_bf16(100 + seed, (M, K)))
        a = to_dev(synth.gaussian_bf16(110 + seed, (R, K), std=0.02))
        t_ref = P.pact_lora_fwd(x, a, 2.0)
        t = torch.full((M, 2 * R), float("nan"), dtype=torch.bfloat16, device="cuda")
        st = lib.pact_lora_fwd_noalloc(x.data_ptr(), K, M, K, a.data_ptr(), R, ctypes.c_float(2.0), t.data_ptr(),
                                       2 * R, ctypes.c_void_p(stream))
        assert st == 0, P.pact_last_error()
        torch.cuda.synchronize()
        got = to_f64(t[:, :R]) + to_f64(t[:, R:])
        ref = to_f64(t_ref[:, :R]) + to_f64(t_ref[:, R:])
        assert_close(got, ref, f"noalloc vs workspace, M={M} K={K} R={R}")
        assert np.array_equal(to_f64(t), to_f64(t_ref))
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
