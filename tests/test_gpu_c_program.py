"""The C ABI from C on the GPU: a C99 program that includes pact.h, allocates device
buffers with cudaMalloc, quantizes X and W's forward layout, runs the frozen GEMM
and reads the output back, with no Python or PyTorch in the process.  The test
writes the seeded inputs to files, the program writes its outputs, and the outputs
are compared with the oracle (codes and scales bit-exact, the GEMM within the
tolerance)."""
import os
import subprocess

import numpy as np
import pytest

import synth
from tests.util import assert_close

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")

PROGRAM = r'''
#include <stdio.h>
#include <stdlib.h>
#include <cuda_runtime.h>
#include "pact.h"

static void *load(const char *path, size_t n) {
    void *h = malloc(n);
    FILE *f = fopen(path, "rb");
    if (!f || fread(h, 1, n, f) != n) { fprintf(stderr, "read %s\n", path); exit(10); }
    fclose(f);
    return h;
}
static void save(const char *path, const void *h, size_t n) {
    FILE *f = fopen(path, "wb");
    if (!f || fwrite(h, 1, n, f) != n) { fprintf(stderr, "write %s\n", path); exit(11); }
    fclose(f);
}
#define CK(x) do { cudaError_t e_ = (x); if (e_ != cudaSuccess) { fprintf(stderr, "%s\n", cudaGetErrorString(e_)); return 20; } } while (0)
#define PK(x) do { pact_status s_ = (x); if (s_ != PACT_OK) { fprintf(stderr, "%s: %s\n", #x, pact_last_error()); return 30; } } while (0)

int main(int argc, char **argv) {
    const int64_t M = atoll(argv[2]), N = atoll(argv[3]), K = atoll(argv[4]);
    char p[4096];
    snprintf(p, sizeof p, "%s/x.bin", argv[1]);
    void *hx = load(p, (size_t)(M * K * 2));
    snprintf(p, sizeof p, "%s/w.bin", argv[1]);
    void *hw = load(p, (size_t)(N * K * 2));
    void *x, *w, *xc, *xs, *cache, *y;
    const size_t xsb = pact_scale_bytes(M, K), cb = pact_weight_cache_bytes(N, K);
    CK(cudaMalloc(&x, M * K * 2));
    CK(cudaMalloc(&w, N * K * 2));
    CK(cudaMalloc(&xc, pact_nvfp4_code_bytes(M, K)));
    CK(cudaMalloc(&xs, xsb));
    CK(cudaMalloc(&cache, cb));
    CK(cudaMalloc(&y, M * N * 2));
    CK(cudaMemcpy(x, hx, M * K * 2, cudaMemcpyHostToDevice));
    CK(cudaMemcpy(w, hw, N * K * 2, cudaMemcpyHostToDevice));
    cudaStream_t st;
    CK(cudaStreamCreate(&st));
    pact_nvfp4_t xq = {xc, xs, M, K};
    pact_weight_cache_t wc;
    PK(pact_weight_layout_cache((const pact_bf16 *)w, K, N, K, cache, cb, &wc, (pact_stream_t)st));
    PK(pact_quantize_nvfp4((const pact_bf16 *)x, K, M, K, &xq, (pact_stream_t)st));
    PK(pact_frozen_gemm_fwd(&xq, &wc, NULL, NULL, 0, (pact_bf16 *)y, N, (pact_stream_t)st));
    PK(pact_get_device_status((pact_stream_t)st));
    void *hc = malloc(pact_nvfp4_code_bytes(M, K)), *hs = malloc(xsb), *hy = malloc(M * N * 2);
    CK(cudaMemcpy(hc, xc, pact_nvfp4_code_bytes(M, K), cudaMemcpyDeviceToHost));
    CK(cudaMemcpy(hs, xs, xsb, cudaMemcpyDeviceToHost));
    CK(cudaMemcpy(hy, y, M * N * 2, cudaMemcpyDeviceToHost));
    snprintf(p, sizeof p, "%s/xq_codes.bin", argv[1]); save(p, hc, pact_nvfp4_code_bytes(M, K));
    snprintf(p, sizeof p, "%s/xq_scales.bin", argv[1]); save(p, hs, xsb);
    snprintf(p, sizeof p, "%s/y.bin", argv[1]); save(p, hy, M * N * 2);
    cudaFree(x); cudaFree(w); cudaFree(xc); cudaFree(xs); cudaFree(cache); cudaFree(y);
    cudaStreamDestroy(st);
    printf("ok\n");
    return 0;
}
'''


def test_c_program_quantizes_and_runs_the_gemm(orc, tmp_path):
    import nvfp4_gemm_b200 as P
    M, N, K = 300, 640, 576                      # ragged in M against 128-row tiles
    x = synth.gaussian_bf16(1, (M, K))
    w = synth.weight_bf16(0, (N, K))
    x.tofile(tmp_path / "x.bin")
    w.tofile(tmp_path / "w.bin")
    src = tmp_path / "prog.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "prog"
    lib_dir = os.path.dirname(P.pact.LIB_PATH)
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                           "-I", os.path.join(CUDA, "include"), str(src), "-L", lib_dir, "-lpact",
                           "-L", os.path.join(CUDA, "lib64"), "-lcudart", f"-Wl,-rpath,{lib_dir}",
                           f"-Wl,-rpath,{os.path.join(CUDA, 'lib64')}", "-o", str(exe)])
    out = subprocess.run([str(exe), str(tmp_path), str(M), str(N), str(K)], capture_output=True, text=True,
                         timeout=300)
    assert out.returncode == 0 and out.stdout.strip() == "ok", (out.returncode, out.stdout, out.stderr)
    ref = orc.quantize(x)
    codes = np.fromfile(tmp_path / "xq_codes.bin", dtype=np.uint8).reshape(M, K // 2)
    scales = np.fromfile(tmp_path / "xq_scales.bin", dtype=np.uint8)
    assert np.array_equal(codes, ref.codes)
    assert np.array_equal(scales, orc.pack_scales(ref.scales, M, K))
    y = synth.bf16_bits_to_f64(np.fromfile(tmp_path / "y.bin", dtype=np.uint16).reshape(M, N))
    wf, _ = orc.weight_cache(w)
    assert_close(y, orc.nvfp4_gemm(ref, wf), "C program GEMM")
