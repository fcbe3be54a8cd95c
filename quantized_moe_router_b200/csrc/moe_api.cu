// moe_api.cu -- the extern "C" entry points of include/moe.h: argument validation, workspace
// sizing and dispatch to the kernels. Nothing here allocates device memory.
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>

#include "moe_internal.cuh"

namespace moe {

moe_status_t launch_decode(const uint16_t *x, const float *wr, const float *bias, const void *packed, int T, int H,
                           int I, int E, int k, uint16_t *out, int32_t *idx_out, float *w_out, void *ws,
                           cudaStream_t st);
moe_status_t launch_prefill(const uint16_t *x, const float *wr, const float *bias, const void *packed, int T, int H,
                            int I, int E, int k, uint16_t *out, int32_t *idx_out, float *w_out, void *ws,
                            cudaStream_t st);
moe_status_t launch_route(const uint16_t *x, const float *wr, const float *bias, int T, int H, int E, int k,
                          int32_t *idx_out, float *w_out, cudaStream_t st);
moe_status_t launch_prefill_route(const uint16_t *x, const float *wr, const float *bias, int T, int H, int I, int E,
                                  int k, int32_t *idx_out, float *w_out, void *ws, cudaStream_t st);
moe_status_t launch_prefill_experts(const uint16_t *x, const void *packed, int T, int H, int I, int E, int k,
                                    uint16_t *out, void *ws, cudaStream_t st);
moe_status_t launch_pack(const moe_expert_src_t *src, int E, int H, int I, void *packed, cudaStream_t st);
moe_status_t launch_quantize_hqq(const uint16_t *w, int rows, int cols, int bits, double p, double beta,
                                 double kappa, int iters, void *codes, uint16_t *scale, uint16_t *zero,
                                 int32_t *iters_used, cudaStream_t st);
size_t packed_layer_bytes(int E, int H, int I, const int32_t *bits);

moe_status_t require_sm100() {
    const DeviceInfo *d = device_info();
    if (!d) return MOE_ERR_CUDA;
    if (d->cc_major != 10 || d->cc_minor != 0) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

static std::atomic<uint64_t> g_wait_ns{2000000000ull};
uint64_t wait_limit_ns() { return g_wait_ns.load(); }

const DeviceInfo *device_info() {
    static DeviceInfo info[64];
    static bool have[64] = {false};
    static std::mutex mu;
    int d = 0;
    if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!have[d]) {
        cudaDeviceProp p;
        if (cudaGetDeviceProperties(&p, d) != cudaSuccess) return nullptr;
        info[d].sms = p.multiProcessorCount;
        info[d].cc_major = p.major;
        info[d].cc_minor = p.minor;
        info[d].max_smem_optin = (int)p.sharedMemPerBlockOptin;
        have[d] = true;
    }
    return &info[d];
}

}  // namespace moe

using namespace moe;

namespace {

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

moe_status_t check_device() { return require_sm100(); }

bool shape_ok(int T, int H, int I, int E, int k) {
    return T >= 1 && H >= 64 && H % kGroup == 0 && I >= 64 && I % kGroup == 0 && E >= 1 && E <= kMaxE &&
           k >= 1 && k <= kMaxK && k <= E && (long long)T * k < (1ll << 31) && (long long)T * H < (1ll << 31);
}

bool packed_ok(const void *packed) { return packed && aligned(packed, 256); }

// Host-side checks shared by the forward entry points (everything but the workspace).
moe_status_t block_args_ok(const uint16_t *x, const float *w_router, const float *bias, const void *packed, int T,
                           int H, int I, int E, int k, uint16_t *out, int32_t *idx_out, float *w_out) {
    if (!shape_ok(T, H, I, E, k)) return MOE_ERR_INVALID_ARG;
    if (!x || !w_router || !out || !packed_ok(packed)) return MOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(w_router, 16) || !aligned(out, 16)) return MOE_ERR_INVALID_ARG;
    if (bias && !aligned(bias, 4)) return MOE_ERR_INVALID_ARG;
    if ((idx_out && !aligned(idx_out, 4)) || (w_out && !aligned(w_out, 4))) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

moe_status_t forward_common(const uint16_t *x, const float *w_router, const float *bias, const void *packed, int T,
                            int H, int I, int E, int k, uint16_t *out, int32_t *idx_out, float *w_out, void *ws,
                            size_t ws_bytes, int mode) {
    const moe_status_t s = block_args_ok(x, w_router, bias, packed, T, H, I, E, k, out, idx_out, w_out);
    if (s != MOE_OK) return s;
    if (!ws || !aligned(ws, 256)) return MOE_ERR_INVALID_ARG;
    if (ws_bytes < moe_workspace_bytes(T, H, I, E, k, mode)) return MOE_ERR_INVALID_ARG;
    return check_device();
}

bool decode_shape_supported(int T, int H, int k) { return T <= kMaxT && (long long)T * k <= kDecodeMaxP && H <= kDecodeMaxH; }

// Scratch of moe_expert_forward_decode_noalloc: a fixed array in the library's own device memory,
// zero-initialised when the library is loaded on a device and kept (with the last call's
// contents) until the process exits. Host code may not use the array's name as an address; the
// device address is resolved once per device, with that device current, by cudaGetSymbolAddress.
constexpr size_t kNoAllocScratchBytes = 2u << 20;   // 2 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
std::mutex g_noalloc_mu;
void *g_noalloc_addr[64] = {nullptr};

// The array's device address on the current device (the set-up of the first call per device).
moe_status_t noalloc_scratch(void **addr) {
    int d = 0;
    if (cudaGetDevice(&d) != cudaSuccess) return MOE_ERR_CUDA;
    if (d < 0 || d >= 64) return MOE_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_addr[d]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return MOE_ERR_CUDA;
        g_noalloc_addr[d] = p;
    }
    *addr = g_noalloc_addr[d];
    return MOE_OK;
}

}  // namespace

extern "C" {

const char *moe_status_str(moe_status_t s) {
    switch (s) {
        case MOE_OK: return "MOE_OK";
        case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
        case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
        case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
        case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
        case MOE_ERR_DEVICE_CHECK: return "MOE_ERR_DEVICE_CHECK";
    }
    return "MOE_ERR_UNKNOWN";
}

int moe_abi_version(void) { return 1; }

void moe_set_wait_limit_ns(uint64_t ns) {
    const uint64_t cap = 60000000000ull;
    g_wait_ns.store(ns > cap ? cap : ns);
}

size_t moe_packed_layer_bytes(int E, int H, int I, const int32_t *bits) {
    if (!bits || E < 1 || E > kMaxE || H < 64 || H % kGroup || I < 64 || I % kGroup) return 0;
    for (int e = 0; e < E; ++e)
        if (bits[e] != 4 && bits[e] != 6 && bits[e] != 8) return 0;
    return packed_layer_bytes(E, H, I, bits);
}

moe_status_t moe_pack_layer(const moe_expert_src_t *src, int E, int H, int I, void *packed, size_t packed_bytes,
                            moe_stream_t stream) {
    if (!src || E < 1 || E > kMaxE || H < 64 || H % kGroup || I < 64 || I % kGroup) return MOE_ERR_INVALID_ARG;
    if (!packed_ok(packed)) return MOE_ERR_INVALID_ARG;
    int32_t bits[kMaxE];
    for (int e = 0; e < E; ++e) {
        bits[e] = src[e].bits;
        if (bits[e] != 4 && bits[e] != 6 && bits[e] != 8) return MOE_ERR_INVALID_ARG;
        for (int m = 0; m < 3; ++m) {
            if (!src[e].codes[m] || !src[e].scale[m] || !src[e].zero[m]) return MOE_ERR_INVALID_ARG;
            if (!aligned(src[e].codes[m], 16) || !aligned(src[e].scale[m], 2) || !aligned(src[e].zero[m], 2))
                return MOE_ERR_INVALID_ARG;
        }
    }
    if (packed_bytes < packed_layer_bytes(E, H, I, bits)) return MOE_ERR_INVALID_ARG;
    const moe_status_t d = check_device();
    if (d != MOE_OK) return d;
    return launch_pack(src, E, H, I, packed, (cudaStream_t)stream);
}

moe_status_t moe_quantize_hqq(const uint16_t *w, int rows, int cols, int bits, const moe_hqq_params_t *params,
                              void *codes, uint16_t *scale, uint16_t *zero, int32_t *iters_used,
                              moe_stream_t stream) {
    if (rows < 0 || cols < kGroup || cols % kGroup || (bits != 4 && bits != 6 && bits != 8))
        return MOE_ERR_INVALID_ARG;
    const moe_hqq_params_t p = params ? *params : moe_hqq_params_t{0.7, 10.0, 1.01, 20};
    if (!(p.lp_norm > 0.0 && p.lp_norm <= 1.0) || !(p.beta > 0.0 && p.beta < HUGE_VAL) ||
        !(p.kappa >= 1.0 && p.kappa < HUGE_VAL) || p.iters < 0 || p.iters > 1000)
        return MOE_ERR_INVALID_ARG;
    if (rows == 0) return MOE_OK;
    if (!w || !codes || !scale || !zero) return MOE_ERR_INVALID_ARG;
    if (!aligned(w, 16) || !aligned(codes, 4) || !aligned(scale, 2) || !aligned(zero, 2) ||
        (iters_used && !aligned(iters_used, 4)))
        return MOE_ERR_INVALID_ARG;
    const moe_status_t d = check_device();
    if (d != MOE_OK) return d;
    return launch_quantize_hqq(w, rows, cols, bits, p.lp_norm, p.beta, p.kappa, p.iters, codes, scale, zero,
                               iters_used, (cudaStream_t)stream);
}

moe_status_t moe_route_topk(const uint16_t *x, const float *w_router, const float *bias, int T, int H, int E, int k,
                            int32_t *idx_out, float *w_out, moe_stream_t stream) {
    if (!shape_ok(T, H, 64, E, k)) return MOE_ERR_INVALID_ARG;
    if (!x || !w_router || !idx_out || !w_out) return MOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(w_router, 16) || (bias && !aligned(bias, 4)) || !aligned(idx_out, 4) ||
        !aligned(w_out, 4))
        return MOE_ERR_INVALID_ARG;
    const moe_status_t d = check_device();
    if (d != MOE_OK) return d;
    return launch_route(x, w_router, bias, T, H, E, k, idx_out, w_out, (cudaStream_t)stream);
}

size_t moe_workspace_bytes(int T, int H, int I, int E, int k, int mode) {
    if (!shape_ok(T, H, I, E, k)) return 0;
    if (mode == MOE_MODE_DECODE) return decode_ws_layout(T, H, I, E, k).total;
    if (mode == MOE_MODE_PREFILL) return prefill_ws_layout(T, H, I, E, k).total;
    return 0;
}

moe_status_t moe_workspace_init(void *ws, size_t ws_bytes, moe_stream_t stream) {
    if (!ws || !aligned(ws, 256) || ws_bytes < sizeof(Control)) return MOE_ERR_INVALID_ARG;
    return cudaMemsetAsync(ws, 0, ws_bytes, (cudaStream_t)stream) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status_t moe_expert_forward_decode(const uint16_t *x, const float *w_router, const float *bias,
                                       const void *packed, int T, int H, int I, int E, int k, uint16_t *out,
                                       int32_t *idx_out, float *w_out, void *ws, size_t ws_bytes,
                                       moe_stream_t stream) {
    moe_status_t s = forward_common(x, w_router, bias, packed, T, H, I, E, k, out, idx_out, w_out, ws, ws_bytes,
                                    MOE_MODE_DECODE);
    if (s != MOE_OK) return s;
    if (!decode_shape_supported(T, H, k)) return MOE_ERR_UNSUPPORTED;
    return launch_decode(x, w_router, bias, packed, T, H, I, E, k, out, idx_out, w_out, ws, (cudaStream_t)stream);
}

moe_status_t moe_expert_forward_decode_noalloc(const uint16_t *x, const float *w_router, const float *bias,
                                               const void *packed, int T, int H, int I, int E, int k, uint16_t *out,
                                               int32_t *idx_out, float *w_out, moe_stream_t stream) {
    // the same host-side checks as moe_expert_forward_decode, before the device is touched
    moe_status_t s = block_args_ok(x, w_router, bias, packed, T, H, I, E, k, out, idx_out, w_out);
    if (s != MOE_OK) return s;
    if (!decode_shape_supported(T, H, k)) return MOE_ERR_UNSUPPORTED;
    if (moe_workspace_bytes(T, H, I, E, k, MOE_MODE_DECODE) > kNoAllocScratchBytes) return MOE_ERR_UNSUPPORTED;
    s = check_device();
    if (s != MOE_OK) return s;
    void *scratch = nullptr;
    s = noalloc_scratch(&scratch);
    if (s != MOE_OK) return s;
    return moe_expert_forward_decode(x, w_router, bias, packed, T, H, I, E, k, out, idx_out, w_out, scratch,
                                     kNoAllocScratchBytes, stream);
}

moe_status_t moe_noalloc_get_device_status(moe_stream_t stream) {
    moe_status_t s = check_device();
    if (s != MOE_OK) return s;
    void *scratch = nullptr;
    s = noalloc_scratch(&scratch);
    if (s != MOE_OK) return s;
    return moe_get_device_status(scratch, stream);
}

moe_status_t moe_expert_forward_prefill(const uint16_t *x, const float *w_router, const float *bias,
                                        const void *packed, int T, int H, int I, int E, int k, uint16_t *out,
                                        int32_t *idx_out, float *w_out, void *ws, size_t ws_bytes,
                                        moe_stream_t stream) {
    moe_status_t s = forward_common(x, w_router, bias, packed, T, H, I, E, k, out, idx_out, w_out, ws, ws_bytes,
                                    MOE_MODE_PREFILL);
    if (s != MOE_OK) return s;
    return launch_prefill(x, w_router, bias, packed, T, H, I, E, k, out, idx_out, w_out, ws, (cudaStream_t)stream);
}

moe_status_t moe_prefill_route(const uint16_t *x, const float *w_router, const float *bias, int T, int H, int I,
                               int E, int k, int32_t *idx_out, float *w_out, void *ws, size_t ws_bytes,
                               moe_stream_t stream) {
    if (!shape_ok(T, H, I, E, k)) return MOE_ERR_INVALID_ARG;
    if (!x || !w_router || !ws) return MOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(w_router, 16) || !aligned(ws, 256)) return MOE_ERR_INVALID_ARG;
    if (bias && !aligned(bias, 4)) return MOE_ERR_INVALID_ARG;
    if ((idx_out && !aligned(idx_out, 4)) || (w_out && !aligned(w_out, 4))) return MOE_ERR_INVALID_ARG;
    if (ws_bytes < moe_workspace_bytes(T, H, I, E, k, MOE_MODE_PREFILL)) return MOE_ERR_INVALID_ARG;
    const moe_status_t d = check_device();
    if (d != MOE_OK) return d;
    return launch_prefill_route(x, w_router, bias, T, H, I, E, k, idx_out, w_out, ws, (cudaStream_t)stream);
}

moe_status_t moe_prefill_experts(const uint16_t *x, const void *packed, int T, int H, int I, int E, int k,
                                 uint16_t *out, void *ws, size_t ws_bytes, moe_stream_t stream) {
    if (!shape_ok(T, H, I, E, k)) return MOE_ERR_INVALID_ARG;
    if (!x || !out || !ws || !packed_ok(packed)) return MOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(ws, 256) || !aligned(out, 16)) return MOE_ERR_INVALID_ARG;
    if (ws_bytes < moe_workspace_bytes(T, H, I, E, k, MOE_MODE_PREFILL)) return MOE_ERR_INVALID_ARG;
    const moe_status_t d = check_device();
    if (d != MOE_OK) return d;
    return launch_prefill_experts(x, packed, T, H, I, E, k, out, ws, (cudaStream_t)stream);
}

moe_status_t moe_get_device_status(void *ws, moe_stream_t stream) {
    if (!ws || !aligned(ws, 256)) return MOE_ERR_INVALID_ARG;
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return MOE_ERR_CUDA;
    Control *ctl = static_cast<Control *>(ws);
    uint32_t st = 0;
    if (cudaMemcpy(&st, &ctl->status, sizeof st, cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
    if (st) {
        // every CTA of the failed call has exited (its waits are bounded and the stream is idle);
        // only the status word is cleared: the completion count must keep growing so that no
        // later call can take a stale logit entry for its own
        if (cudaMemset(&ctl->status, 0, sizeof st) != cudaSuccess) return MOE_ERR_CUDA;
    }
    if (st & kStatusTimeout) return MOE_ERR_TIMEOUT;
    if (st & kStatusCheck) return MOE_ERR_DEVICE_CHECK;
    return MOE_OK;
}

}  // extern "C"
