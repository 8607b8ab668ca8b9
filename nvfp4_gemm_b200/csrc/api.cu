// api.cu -- status codes, error messages and argument validation of libpact.
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include "common.cuh"

namespace pact {

static thread_local char t_error[512] = "";

void set_error(const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(t_error, sizeof(t_error), fmt, ap);
    va_end(ap);
}

pact_status fail(pact_status s, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(t_error, sizeof(t_error), fmt, ap);
    va_end(ap);
    return s;
}

pact_status launch_status(const char *what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(PACT_ERR_CUDA, "%s: launch failed: %s", what, cudaGetErrorString(e));
    return PACT_OK;
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }  // NULL counts as aligned

int current_device() {
    int d = 0;
    cudaGetDevice(&d);
    return d;
}

int sm_count() {
    static std::atomic<int> cache[64];   // 0: not looked up yet (host threads may race to fill it)
    const int d = current_device();
    if (d < 0 || d >= 64) return 148;
    int n = cache[d].load(std::memory_order_relaxed);
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d) != cudaSuccess || n <= 0) n = 148;
        cache[d].store(n, std::memory_order_relaxed);
    }
    return n;
}

pact_status check_nvfp4(const pact_nvfp4_t *t, int64_t rows, int64_t cols, const char *name) {
    if (!t || !t->codes || !t->scales) return fail(PACT_ERR_INVALID_ARG, "NVFP4 tensor %s: NULL pointer", name);
    if (t->rows != rows || t->cols != cols)
        return fail(PACT_ERR_SHAPE, "NVFP4 tensor %s: shape [%lld x %lld], expected [%lld x %lld]", name,
                    (long long)t->rows, (long long)t->cols, (long long)rows, (long long)cols);
    if (cols % 64 != 0) return fail(PACT_ERR_SHAPE, "NVFP4 tensor %s: cols must be a multiple of 64", name);
    if (!aligned16(t->codes) || !aligned16(t->scales))
        return fail(PACT_ERR_ALIGN, "NVFP4 tensor %s: codes and scales must be 16-byte aligned", name);
    return PACT_OK;
}

// Self-test of the failure path: one thread waits, with the given limit, on an
// mbarrier that nothing arrives on, through the same bounded wait every kernel uses.
// The wait runs out, records the timeout in the status word and the kernel returns;
// nothing asynchronous (no copy, no tensor-core operation) is outstanding.
__global__ void k_wait_selftest(long long limit_cycles, unsigned long long *waited_cycles) {
    __shared__ uint64_t bar;
    pdl_wait();
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    fence_barrier_init();
    const long long t0 = clock64();
    const bool ok = mbar_wait(&bar, 0, limit_cycles);
    if (waited_cycles) *waited_cycles = ok ? 0ull : (unsigned long long)(clock64() - t0);
}

}  // namespace pact

extern "C" {

pact_status pact_selftest_wait_timeout(int64_t limit_cycles, unsigned long long *waited_cycles,
                                       pact_stream_t stream) {
    PACT_CHECK(limit_cycles >= 1000 && limit_cycles <= 4000000000ll, PACT_ERR_INVALID_ARG,
               "pact_selftest_wait_timeout: limit must be in [1e3, 4e9] cycles (got %lld)", (long long)limit_cycles);
    PACT_CHECK(((uintptr_t)waited_cycles & 7) == 0, PACT_ERR_ALIGN, "pact_selftest_wait_timeout: waited_cycles 8-byte aligned");
    return pact::launch_dep(pact::k_wait_selftest, dim3(1), dim3(32), 0, (cudaStream_t)stream,
                            "pact_selftest_wait_timeout", (long long)limit_cycles, waited_cycles);
}

const char *pact_last_error(void) { return pact::t_error; }

const char *pact_status_string(pact_status s) {
    switch (s) {
        case PACT_OK: return "PACT_OK";
        case PACT_ERR_INVALID_ARG: return "PACT_ERR_INVALID_ARG";
        case PACT_ERR_SHAPE: return "PACT_ERR_SHAPE";
        case PACT_ERR_ALIGN: return "PACT_ERR_ALIGN";
        case PACT_ERR_CUDA: return "PACT_ERR_CUDA";
        case PACT_ERR_TIMEOUT: return "PACT_ERR_TIMEOUT";
        case PACT_ERR_UNSUPPORTED: return "PACT_ERR_UNSUPPORTED";
    }
    return "PACT_ERR_UNKNOWN";
}

pact_status pact_get_device_status(pact_stream_t stream) {
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return pact::fail(PACT_ERR_CUDA, "pact_get_device_status: %s", cudaGetErrorString(e));
    uint32_t word = 0, zero = 0;
    e = cudaMemcpyFromSymbol(&word, pact::g_status, sizeof(word));
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(pact::g_status, &zero, sizeof(zero));
    if (e != cudaSuccess) return pact::fail(PACT_ERR_CUDA, "pact_get_device_status: %s", cudaGetErrorString(e));
    if (word & pact::STATUS_TIMEOUT)
        return pact::fail(PACT_ERR_TIMEOUT, "a libpact kernel gave up a bounded wait (status word 0x%x)", word);
    return PACT_OK;
}

int pact_abi_version(void) { return PACT_ABI_VERSION; }

}  // extern "C"
