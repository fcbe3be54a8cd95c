// Test stand-ins for the two device-facing calls of quantized_moe_router_b200/csrc/moe_cache.cu, so
// that the cache's host logic runs on a machine without a GPU: the copy becomes a memcpy into host
// memory that plays the device pool (optionally failing after a given number of copies), and the
// device check returns a status the test sets. Compiled with that source file into a test library
// by tests/test_cache.py; the product library never contains this file.
#include <cstring>
#include <cuda_runtime_api.h>

#include "moe.h"

namespace {
int g_fail_after = -1;   // copies left before one fails; -1: never
long g_copies = 0;
moe_status_t g_device = MOE_OK;
}  // namespace

extern "C" cudaError_t cudaMemcpyAsync(void *dst, const void *src, size_t n, cudaMemcpyKind kind, cudaStream_t) {
    if (kind != cudaMemcpyHostToDevice) return cudaErrorInvalidValue;
    if (g_fail_after == 0) return cudaErrorLaunchFailure;
    if (g_fail_after > 0) --g_fail_after;
    std::memcpy(dst, src, n);
    ++g_copies;
    return cudaSuccess;
}

namespace moe {
moe_status_t require_sm100() { return g_device; }
}  // namespace moe

extern "C" {
void shim_fail_after(int n) { g_fail_after = n; }
long shim_copies(void) { return g_copies; }
void shim_set_device_status(int s) { g_device = (moe_status_t)s; }
}
