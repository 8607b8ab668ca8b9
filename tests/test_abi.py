"""The C ABI without a GPU: libpact.so loads, exports every function include/pact.h
declares, its size queries agree with the layout definition, and host-side argument
checks reject bad calls with the documented status before anything is enqueued."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "pact.h")).read()
    return sorted(set(re.findall(r"PACT_API\s+[\w\s\*]+?\b(pact_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def P():
    # the build script is loaded by path so that a stale library is not loaded first
    import importlib.util
    spec = importlib.util.spec_from_file_location("_pact_build", os.path.join(ROOT, "nvfp4_gemm_b200", "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    b.build()
    import nvfp4_gemm_b200 as p
    return p


def test_every_declared_symbol_is_exported(P):
    names = declared_functions()
    assert len(names) >= 18
    lib = ctypes.CDLL(P.pact.LIB_PATH)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing


def test_abi_version_and_status_names(P):
    assert P.pact_abi_version() == 3
    lib = P.pact.lib
    assert lib.pact_status_string(0) == b"PACT_OK"
    assert lib.pact_status_string(5) == b"PACT_ERR_TIMEOUT"


def test_sizes_match_the_layout(P, orc):
    for rows, cols in [(1, 64), (128, 64), (300, 320), (2048, 8960), (129, 1536)]:
        assert P.pact_scale_bytes(rows, cols) == orc.scale_bytes(rows, cols)
        assert P.pact_nvfp4_code_bytes(rows, cols) == rows * cols // 2
    up = lambda b: (b + 255) // 256 * 256
    N, K = 448, 320
    assert P.pact_weight_cache_bytes(N, K) == (up(N * K // 2) + up(orc.scale_bytes(N, K)) + up(K * N // 2)
                                               + up(orc.scale_bytes(K, N)))


def _nv(rows, cols, codes=0x1000, scales=0x2000):
    return P_mod().c_nvfp4(codes, scales, rows, cols)


def P_mod():
    import nvfp4_gemm_b200.pact as pm
    return pm


def test_host_checks_reject_bad_arguments(P):
    lib = P.pact.lib
    pm = P_mod()
    good = pm.c_nvfp4(0x1000, 0x2000, 128, 128)
    # NULL input
    assert lib.pact_quantize_nvfp4(None, 128, 128, 128, ctypes.byref(good), None) == 1
    # cols not a multiple of 64
    bad = pm.c_nvfp4(0x1000, 0x2000, 128, 100)
    assert lib.pact_quantize_nvfp4(0x3000, 100, 128, 100, ctypes.byref(bad), None) == 2
    # misaligned input pointer
    assert lib.pact_quantize_nvfp4(0x3008, 128, 128, 128, ctypes.byref(good), None) == 3
    # output descriptor of the wrong shape
    other = pm.c_nvfp4(0x1000, 0x2000, 64, 128)
    assert lib.pact_quantize_nvfp4(0x3000, 128, 128, 128, ctypes.byref(other), None) == 2
    assert "shape" in P.pact_last_error()
    # RMSNorm: H beyond the supported maximum
    big = pm.c_nvfp4(0x1000, 0x2000, 4, 32768)
    assert lib.pact_rmsnorm_quant(0x3000, 32768, 0x4000, ctypes.c_float(1e-5), 4, 32768, ctypes.byref(big),
                                  None, None, None) == 2
    # weight cache: buffer too small / misaligned
    wc = pm.c_weight_cache()
    assert lib.pact_weight_layout_cache(0x3000, 512, 512, 512, 0x10000, 16, ctypes.byref(wc), None) == 1
    n = P.pact_weight_cache_bytes(512, 512)
    assert lib.pact_weight_layout_cache(0x3000, 512, 512, 512, 0x10010, n, ctypes.byref(wc), None) == 3
    # GEMM: output leading dimension not a multiple of 8
    wcache = pm.c_weight_cache(pm.c_nvfp4(0x1000, 0x2000, 512, 512), pm.c_nvfp4(0x3000, 0x4000, 512, 512))
    xq = pm.c_nvfp4(0x5000, 0x6000, 256, 512)
    assert lib.pact_frozen_gemm_fwd(ctypes.byref(xq), ctypes.byref(wcache), None, None, 0, 0x7000, 516, None) == 3
    # GEMM: activation K does not match the weight
    xq2 = pm.c_nvfp4(0x5000, 0x6000, 256, 448)
    assert lib.pact_frozen_gemm_fwd(ctypes.byref(xq2), ctypes.byref(wcache), None, None, 0, 0x7000, 512, None) == 2
    # LoRA: internal segment boundary not a multiple of 256
    se = (ctypes.c_int64 * 4)(320, 512, 0, 0)
    lo = pm.c_lora(0x8000, 32, 0x9000, 16, 16, 2, se)
    assert lib.pact_frozen_gemm_fwd(ctypes.byref(xq), ctypes.byref(wcache), ctypes.byref(lo), None, 0, 0x7000,
                                    512, None) == 2
    # LoRA rank not supported
    lo2 = pm.c_lora(0x8000, 32, 0x9000, 16, 8, 1, (ctypes.c_int64 * 4)(512, 0, 0, 0))
    assert lib.pact_frozen_gemm_fwd(ctypes.byref(xq), ctypes.byref(wcache), ctypes.byref(lo2), None, 0,
                                    0x7000, 512, None) == 2
    # LoRA backward: workspace too small
    args = pm.c_lora_bwd()
    args.M, args.N, args.K = 256, 512, 512
    args.dy, args.lddy, args.x, args.ldx = 0x1000, 512, 0x2000, 512
    args.A, args.U, args.ldu, args.r, args.nseg = 0x3000, 0x4000, 16, 16, 1
    args.seg_end[0] = 512
    args.dA, args.dB, args.scale = 0x5000, 0x6000, 2.0
    assert lib.pact_lora_bwd(ctypes.byref(args), 0x10000, 64, None) == 1
    # both x and xq given
    xq3 = pm.c_nvfp4(0x5000, 0x6000, 256, 512)
    args.xq = ctypes.pointer(xq3)
    need = P.pact_lora_bwd_workspace_bytes(256, 512, 512, 16, 1)
    assert lib.pact_lora_bwd(ctypes.byref(args), 0x10000, need, None) == 1


def test_two_level_exponent_host_function(P, orc):
    """pact_two_level_exponent (host code, no GPU) against the oracle's definition."""
    import numpy as np
    rng = np.random.default_rng(31)
    vals = [0.0, -1.0, float("inf"), float("nan"), 2688.0, 1344.0, 6.0, 0.1, 2.0 ** -140, 3.0e38]
    vals += [float(np.float32(v)) for v in np.exp(rng.uniform(-90, 88, 300))]
    for v in vals:
        want = orc.two_level_exponent(v) if np.isfinite(v) else 0
        assert P.pact_two_level_exponent(v) == want, v


def test_two_level_host_checks(P):
    lib = P.pact.lib
    pm = P_mod()
    wc = pm.c_weight_cache()
    n = P.pact_weight_cache_bytes(512, 512)
    assert lib.pact_weight_layout_cache_scaled(0x3000, 512, 512, 512, 101, 0x10000, n, ctypes.byref(wc), None) == 1
    assert lib.pact_absmax_bf16(None, 512, 512, 512, 0x2000, None) == 1
    assert lib.pact_absmax_bf16(0x3000, 512, 512, 100, 0x2000, None) == 2
    assert lib.pact_absmax_bf16(0x3008, 512, 512, 512, 0x2000, None) == 3
    # GEMM with a cache exponent out of range
    wcache = pm.c_weight_cache(pm.c_nvfp4(0x1000, 0x2000, 512, 512), pm.c_nvfp4(0x3000, 0x4000, 512, 512), 200)
    xq = pm.c_nvfp4(0x5000, 0x6000, 256, 512)
    assert lib.pact_frozen_gemm_fwd(ctypes.byref(xq), ctypes.byref(wcache), None, None, 0, 0x7000, 512, None) == 1


def test_wait_selftest_limit_is_checked_on_the_host(P):
    lib = P.pact.lib
    for bad in (0, 10, 5_000_000_000):
        assert lib.pact_selftest_wait_timeout(bad, None, None) == 1
    assert lib.pact_selftest_wait_timeout(10_000, 0x1004, None) == 3      # misaligned output


def test_plain_c_program_links_and_calls_the_host_functions(P, tmp_path):
    """A C99 program includes pact.h, links libpact.so and calls the calls that need no
    GPU: the ABI version, the size queries, the two-level exponent and a rejected
    argument check."""
    import subprocess
    src = tmp_path / "abi.c"
    src.write_text(r'''
#include <stdio.h>
#include "pact.h"
int main(void) {
    pact_nvfp4_t t = {0, 0, 128, 100};
    if (pact_abi_version() != PACT_ABI_VERSION) return 1;
    if (pact_nvfp4_code_bytes(128, 64) != 4096) return 2;
    if (pact_scale_bytes(200, 64) != 1024) return 3;
    if (pact_two_level_exponent(2688.0f) != 0 || pact_two_level_exponent(0.1f) != -14) return 4;
    if (pact_quantize_nvfp4((const pact_bf16 *)0x3000, 100, 128, 100, &t, 0) != PACT_ERR_SHAPE) return 5;
    printf("ok\n");
    return 0;
}
''')
    exe = tmp_path / "abi"
    lib_dir = os.path.dirname(P.pact.LIB_PATH)
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
                           "-L", lib_dir, "-lpact", f"-Wl,-rpath,{lib_dir}", "-o", str(exe)])
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0 and out.stdout.strip() == "ok", (out.returncode, out.stdout, out.stderr)


def test_lora_struct_keeps_its_tensors_alive(P):
    """The descriptor carries raw device pointers; the tensors behind them must live as
    long as the descriptor, or a later allocation could reuse their memory while a
    GEMM still reads it."""
    import gc
    import weakref

    import torch
    act, w = torch.zeros(64, 32, dtype=torch.bfloat16), torch.zeros(256, 16, dtype=torch.bfloat16)
    refs = weakref.ref(act), weakref.ref(w)
    lo = P.lora_struct(act, w, 16, [256])
    del act, w
    gc.collect()
    assert all(r() is not None for r in refs)
    assert lo.act == refs[0]().data_ptr() and lo.weight == refs[1]().data_ptr()
    del lo
    gc.collect()
    assert all(r() is None for r in refs)
