/*
 * moe.h -- C ABI of the B200 (sm_100a) quantized Mixture-of-Experts expert block.
 *
 * Per layer the library computes, for every token t of the hidden states x [T x H]:
 *   logits l = W_r x (+ bias); the k experts with the largest logits (ties -> lower index);
 *   routing weights = softmax over those k logits; for each selected expert e the FFN
 *   y_e = Wd_e (silu(Wg_e x) * (Wu_e x)) with group-affine low-bit weights
 *   W[r,c] = (q[r,c] - z[r,c/64]) * s[r,c/64]; and out[t] = sum_i w_i y_{e_i}.
 * This is the MoE expert block that the pages "Krasis update" (HQQ 4/6/8-bit experts),
 * "--moe-direct-io" / "Qwen-tin" (512 experts, top-10 routing) and "Raon-1-mini on an
 * RTX 5070 Ti" (table rows "MoE megakernel" and "Pipelined megakernel": one persistent kernel
 * per layer's expert block, next expert loaded while the current one computes) run in their
 * decode and prefill loops; the pages print no formula, so the steps above are the plain
 * reading of router top-k + softmax renormalisation, affine group dequantisation, gate/up,
 * SiLU-GLU, down and a routing-weighted combine.
 *
 * Conventions for every entry point:
 *  - Pointers marked (device) are CUDA device pointers owned by the caller; the library never
 *    frees or retains them. Pointers marked (host) are read during the call only.
 *  - bf16 and fp16 values are passed as their 16-bit patterns (uint16_t).
 *  - All arguments are validated on the host before anything is launched; a bad argument
 *    returns MOE_ERR_INVALID_ARG (or MOE_ERR_UNSUPPORTED for a valid but unsupported shape)
 *    and launches nothing. A failed launch returns MOE_ERR_CUDA.
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default stream) and the call
 *    returns without synchronising, except moe_get_device_status.
 *  - No entry point allocates device memory: scratch space is the caller's workspace.
 *  - Two calls that share a workspace must be ordered (same stream, or events); calls with
 *    distinct workspaces may run concurrently.
 *  - The library supports sm_100a (B200) only; on any other device calls return
 *    MOE_ERR_UNSUPPORTED.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t (a pointer to the runtime's opaque stream struct). */
typedef struct CUstream_st *moe_stream_t;

typedef enum moe_status {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size, workspace too small */
    MOE_ERR_UNSUPPORTED = 2,   /* shape or device outside what the kernels implement */
    MOE_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed */
    MOE_ERR_TIMEOUT = 4,       /* a bounded device-side wait expired (see moe_get_device_status) */
    MOE_ERR_DEVICE_CHECK = 5   /* a device-side consistency check failed */
} moe_status_t;

/* Human-readable name of a status (static string, never NULL). */
const char *moe_status_str(moe_status_t s);

/* ABI version of this header: 1. */
int moe_abi_version(void);

/* ---------------------------------------------------------------------------------------
 * Expert weights.
 *
 * Canonical (input) format of one expert, the format a quantiser hands over. Matrix m is
 * 0 = gate [I x H], 1 = up [I x H], 2 = down [H x I] (rows x cols; the input dimension is
 * the column dimension). For each matrix (all pointers device, 16-byte aligned):
 *   codes[m]: rows x (cols*bits/8) bytes, row-major. Group g of a row (columns 64g..64g+63)
 *             is a block of 8*bits bytes; code j of the group occupies bits
 *             [j*bits, (j+1)*bits) of that block read as one little-endian bit string.
 *   scale[m], zero[m]: fp16 [rows x cols/64], row-major; W[r,c] = (q - zero) * scale.
 * bits is 4, 6 or 8 and may differ between the experts of one layer.
 * ------------------------------------------------------------------------------------- */
typedef struct moe_expert_src {
    const void *codes[3];
    const uint16_t *scale[3];
    const uint16_t *zero[3];
    int32_t bits;
} moe_expert_src_t;

/* Bytes of the packed form of one layer of E experts with per-expert widths bits[E] (host).
 * Returns 0 if an argument is invalid (H or I not a multiple of 64, E < 1, bits not in
 * {4,6,8}). */
size_t moe_packed_layer_bytes(int E, int H, int I, const int32_t *bits);

/* Converts one layer's experts from the canonical format (src: host array of E descriptors
 * whose pointers are device pointers) into the packed form the forward kernels read, written
 * to `packed` (device, 256-byte aligned, packed_bytes >= moe_packed_layer_bytes). The packed
 * form is self-describing (it records E, H, I and each expert's width). The conversion is a
 * byte permutation: no value is rounded. Asynchronous on `stream`; the canonical buffers
 * must stay valid until it completes. */
moe_status_t moe_pack_layer(const moe_expert_src_t *src, int E, int H, int I, void *packed,
                            size_t packed_bytes, moe_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * Expert cache: packed layers kept in host memory, the experts a call needs streamed into a
 * fixed pool of device slots.
 *
 * The pages run models whose experts do not fit in GPU memory: "Krasis update" (overview)
 * streams the model from system RAM to VRAM; "RTX 3060 12GB ... --moe-direct-io" loads the
 * selected experts on demand into a fixed number of slots per layer (72), without dropping
 * experts and with output bit-identical to the stock engine; the Qwen-tin news page (memory
 * placement and performance) keeps the expert weights on SSD and caches part of them in RAM
 * and VRAM, about 96% of a token's expert bytes being resident already. Here each layer's
 * packed form (as written by moe_pack_layer) stays in host memory, ideally page-locked, and a
 * device pool holds one header per layer and `slots` expert-sized slots shared by all layers
 * (a per-layer limit is one cache per layer). The forward calls read the same packed bytes
 * either way, so a call through the cache computes what the resident call computes; the
 * forward kernels add partial sums in arrival order, so either may differ from a repeat of
 * itself in the last bit of an output.
 *   [header of layer 0] ... [header of layer L-1] [slot 0] ... [slot slots-1]
 * A layer's header has the packed format's layout; its entries point into the slots, so the
 * header's address is a packed layer that the forward calls accept unchanged, as long as every
 * expert the call selects is resident. Entries of experts that are not resident still point
 * inside the pool (they read another expert's bytes, never memory outside it).
 *
 * Use per layer call: route (moe_route_topk, or the caller's own prediction), read the selected
 * experts on the host, moe_cache_request (which experts are missing and where they go: host work
 * only), moe_cache_commit (the copies and the header rewrite, on `stream`), then the forward
 * call with the returned header. The forward call's idx_out shows which experts it used; a
 * selection outside the request (possible only at a near-tie between the two routings) is
 * requested and the call repeated.
 *
 * Eviction: a missing expert takes a free slot, else the slot of the least recently requested
 * expert that none of the last `keep_recent` requests (this one included) named. keep_recent = 2
 * lets the copies of one layer run while the previous layer's call still reads its experts,
 * provided the caller orders the copies after the previous request's commit. A cache object is
 * not thread-safe. Calls that read the pool must be ordered with the commits that overwrite it
 * (one stream, or events).
 * ------------------------------------------------------------------------------------- */
typedef struct moe_expert_cache moe_expert_cache_t;

/* Device bytes of the pool for L host layers (host_layers[l]: host pointer to layer l's packed
 * form; all layers with the same E, H, I) and `slots` slots; 0 if an argument is invalid. */
size_t moe_cache_pool_bytes(int L, const void *const *host_layers, const size_t *host_bytes,
                            int slots);

/* Creates the cache: host_layers / host_bytes (host arrays [L]) give each layer's packed form in
 * host memory and its size, checked against the headers; pool (device, 256-byte aligned) holds
 * pool_bytes >= moe_cache_pool_bytes. 1 <= slots, 1 <= keep_recent <= 8. The host layers must
 * stay valid and unchanged while the cache exists. Host work only: no device memory is touched
 * until the first commit. */
moe_status_t moe_cache_create(int L, const void *const *host_layers, const size_t *host_bytes,
                              int slots, int keep_recent, void *pool, size_t pool_bytes,
                              moe_expert_cache_t **cache);

void moe_cache_destroy(moe_expert_cache_t *cache);

/* Makes experts[0..n) of `layer` (host array; duplicates allowed) the current request: counts
 * hits and misses, gives every missing expert a slot (evicting as described above) and writes
 * the missing experts and their slots to load_experts / load_slots (host arrays of at least n
 * entries; either may be NULL) and their number to *n_load. Host work only. Fails with
 * MOE_ERR_UNSUPPORTED, changing nothing, if the slots that may be evicted are too few. A
 * request replaces an earlier request that was not committed. */
moe_status_t moe_cache_request(moe_expert_cache_t *cache, int layer, const int32_t *experts,
                               int n, int32_t *load_experts, int32_t *load_slots, int *n_load);

/* Enqueues on `stream` the host -> device copies of the current request's missing experts and
 * the rewrite of its layer's header (a copy from pageable host memory, so the call returns once
 * the stream has drained up to it), and returns in *packed the device address of that layer's
 * packed header. If a copy cannot be enqueued the missing experts are marked absent again and
 * MOE_ERR_CUDA is returned. */
moe_status_t moe_cache_commit(moe_expert_cache_t *cache, moe_stream_t stream, const void **packed);

/* Slot that holds (layer, expert), or -1 (also for invalid arguments). */
int moe_cache_slot_of(const moe_expert_cache_t *cache, int layer, int expert);

/* Counters since creation: experts requested that were resident (hits), that had to be loaded
 * (misses), and resident experts that lost their slot (evictions). */
moe_status_t moe_cache_stats(const moe_expert_cache_t *cache, uint64_t *hits, uint64_t *misses,
                             uint64_t *evictions);

/* ---------------------------------------------------------------------------------------
 * Quantiser: bf16 weights -> the canonical format above.
 *
 * HQQ-style group quantisation (Half-Quadratic Quantization, H. Badri and A. Shaji, 2023; the
 * page "Krasis update", list of the v1.0 results, names it at 4, 6 and 8 bits, built from the
 * weights alone). For each 64-wide group of a row, Q = 2^bits - 1:
 *   1. s = fp16((max - min) / Q), kept within [least positive fp16, 65504]; z = -min / s.
 *      A constant group c is quantised over [min(c, 0), max(c, 0)], an all-zero group with
 *      scale 1.
 *   2. Up to `iters` half-quadratic steps on the zero point: with q = clamp(rint(w/s + z), 0, Q)
 *      and r = (q - z) * s, stop if sum |w - r| did not fall below (1 - 2^-40) times the best
 *      so far (which keeps its zero; the margin exceeds the sum's rounding, so ties on the flat
 *      stretches of the L1 error stop as in exact arithmetic); otherwise e = shrink(w - r) with
 *      shrink(x) = sign(x) * max(|x| - |x|^(lp_norm - 1) / beta, 0), z = mean(q - (w - e)/s),
 *      beta = beta * kappa.
 *   3. zero = fp16(best z), clamped to +-65504; codes = the nearest points of the stored fp16
 *      grid, clamp(rint(w/scale + zero), 0, Q).
 * Arithmetic is IEEE fp64, each operation correctly rounded and unfused, and the two sums over
 * a group run in index order, so results are those of the definition evaluated in that order
 * (the power function of the shrink, accurate to a few units in the last place, aside).
 *   w (device, 16-byte aligned) bf16 [rows x cols], row-major, cols % 64 == 0, rows >= 0.
 *   params (host) or NULL for the published defaults {0.7, 10.0, 1.01, 20}; required:
 *     0 < lp_norm <= 1, beta > 0 and finite, kappa >= 1 and finite, 0 <= iters <= 1000
 *     (iters = 0 is plain min-max rounding).
 *   codes (device, 4-byte aligned): rows x (cols*bits/8) bytes in the canonical layout.
 *   scale, zero (device, 2-byte aligned): fp16 [rows x cols/64].
 *   iters_used (device, 4-byte aligned) int32 [rows x cols/64] or NULL: steps run per group,
 *     counting the one that stopped.
 * rows == 0 launches nothing. Asynchronous on `stream`.
 * ------------------------------------------------------------------------------------- */
typedef struct moe_hqq_params {
    double lp_norm;
    double beta;
    double kappa;
    int32_t iters;
} moe_hqq_params_t;

moe_status_t moe_quantize_hqq(const uint16_t *w, int rows, int cols, int bits,
                              const moe_hqq_params_t *params, void *codes, uint16_t *scale,
                              uint16_t *zero, int32_t *iters_used, moe_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * Routing alone.
 *
 * x (device) bf16 [T x H]; w_router (device) fp32 [E x H]; bias (device) fp32 [E] or NULL.
 * Writes idx_out (device) int32 [T x k], experts in descending logit order (ties -> lower
 * index), and w_out (device) fp32 [T x k], the softmax of those k logits. Logits are fp32
 * dot products of the bf16 x with the fp32 router rows.
 * Limits: 1 <= T, H % 64 == 0, 1 <= k <= min(E, 32), E <= 1024. No workspace.
 * ------------------------------------------------------------------------------------- */
moe_status_t moe_route_topk(const uint16_t *x, const float *w_router, const float *bias, int T,
                            int H, int E, int k, int32_t *idx_out, float *w_out,
                            moe_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * Whole expert block.
 * ------------------------------------------------------------------------------------- */
enum { MOE_MODE_DECODE = 0, MOE_MODE_PREFILL = 1 };

/* Workspace bytes needed by a forward call of the given mode and shape (0 if invalid). */
size_t moe_workspace_bytes(int T, int H, int I, int E, int k, int mode);

/* Prepares a workspace (device, 256-byte aligned) for first use: clears all ws_bytes of it
 * (asynchronously on `stream`). Needed once after allocation; the forward calls keep it
 * consistent afterwards. */
moe_status_t moe_workspace_init(void *workspace, size_t ws_bytes, moe_stream_t stream);

/* Decode path, 1 <= T <= 32: one persistent kernel per call (routing, gate/up, SiLU-GLU,
 * down and combine fused; intermediates stay on chip or in L2). Launched with programmatic
 * dependent launch so that consecutive layer calls overlap their start-up.
 *   x (device, 16-byte aligned) bf16 [T x H]; w_router (device, 16-byte aligned) fp32 [E x H];
 *   bias (device) fp32 [E] or NULL; packed (device, 256-byte aligned) one layer in moe_pack_layer form with the same E, H, I;
 *   out (device, 16-byte aligned) bf16 [T x H]; idx_out (device) int32 [T x k] or NULL; w_out (device) fp32
 *   [T x k] or NULL; workspace (device) of ws_bytes >= moe_workspace_bytes(..., DECODE),
 *   prepared by moe_workspace_init.
 * Limits: H % 64 == 0, I % 64 == 0, 1 <= k <= min(E, 32), E <= 1024.
 * A bounded device-side wait that expires leaves `out` undefined and sets the workspace's
 * status word (read it with moe_get_device_status). */
moe_status_t moe_expert_forward_decode(const uint16_t *x, const float *w_router,
                                       const float *bias, const void *packed, int T, int H,
                                       int I, int E, int k, uint16_t *out, int32_t *idx_out,
                                       float *w_out, void *workspace, size_t ws_bytes,
                                       moe_stream_t stream);

/* Decode path without a caller workspace. Same computation, arguments, limits and results as
 * moe_expert_forward_decode, but the scratch memory lives in a fixed 2 MiB array inside this
 * library's device memory, so the caller passes only inputs and outputs and nothing is
 * allocated. The pages describe no such entry point; it exists for callers that cannot call
 * cudaMalloc: for example an operator plugin that a host runtime hands only its input and
 * output buffers, or a process whose device memory is owned by another allocator.
 *  - Arguments are checked on the host exactly as for moe_expert_forward_decode, before the
 *    device is touched; shapes whose decode workspace (moe_workspace_bytes(..., MOE_MODE_DECODE))
 *    would exceed 2 MiB are rejected with MOE_ERR_UNSUPPORTED before anything is launched (the
 *    decode workspace has fixed regions, so every supported decode shape fits today).
 *  - The first call on a device looks up the array's device address (once per device, with
 *    that device current); make that first call before any stream capture.
 *  - Every call on a device shares the one array, which keeps the previous call's contents
 *    (the kernel clears what must start at zero itself). Calls whose executions overlap on the
 *    GPU (other streams, other host threads) race on it: order them.
 *  - Every GPU that loads the library holds the 2 MiB until the process exits.
 *  - A device-side wait that expires leaves `out` undefined and sets the array's status word;
 *    read (and clear) it with moe_noalloc_get_device_status. */
moe_status_t moe_expert_forward_decode_noalloc(const uint16_t *x, const float *w_router,
                                               const float *bias, const void *packed, int T,
                                               int H, int I, int E, int k, uint16_t *out,
                                               int32_t *idx_out, float *w_out,
                                               moe_stream_t stream);

/* moe_get_device_status for the fixed array of moe_expert_forward_decode_noalloc on the current
 * device: synchronises `stream`, returns MOE_OK, MOE_ERR_TIMEOUT or MOE_ERR_DEVICE_CHECK and
 * clears a non-zero status word. Allocates nothing. */
moe_status_t moe_noalloc_get_device_status(moe_stream_t stream);

/* Prefill path, any T >= 1: routing, bucketing of the T*k (token, expert) pairs per expert
 * (stable: ascending token within an expert), a grouped gate/up GEMM with a SiLU-GLU
 * epilogue and a grouped down GEMM whose epilogue adds the routing-weighted rows into the
 * output. Arguments as for moe_expert_forward_decode, with the PREFILL workspace size. */
moe_status_t moe_expert_forward_prefill(const uint16_t *x, const float *w_router,
                                        const float *bias, const void *packed, int T, int H,
                                        int I, int E, int k, uint16_t *out, int32_t *idx_out,
                                        float *w_out, void *workspace, size_t ws_bytes,
                                        moe_stream_t stream);

/* The two halves of moe_expert_forward_prefill, for callers that schedule them separately (for
 * example to overlap the routing of one layer with other work, or to time the expert GEMMs).
 * moe_prefill_route: routing (as moe_route_topk) and the bucketing of the T*k pairs per expert
 * into the PREFILL workspace; idx_out / w_out (device) may be NULL. moe_prefill_experts: the
 * grouped gate/up and down GEMMs and the combine over the buckets that the last
 * moe_prefill_route left in the same workspace (same T, H, I, E, k), writing out (device)
 * bf16 [T x H]; x must be the same hidden states. Arguments and limits as for
 * moe_expert_forward_prefill. */
moe_status_t moe_prefill_route(const uint16_t *x, const float *w_router, const float *bias, int T,
                               int H, int I, int E, int k, int32_t *idx_out, float *w_out,
                               void *workspace, size_t ws_bytes, moe_stream_t stream);
moe_status_t moe_prefill_experts(const uint16_t *x, const void *packed, int T, int H, int I,
                                 int E, int k, uint16_t *out, void *workspace, size_t ws_bytes,
                                 moe_stream_t stream);

/* Synchronises `stream`, reads the workspace's device status word and maps it to a status:
 * MOE_OK, MOE_ERR_TIMEOUT (a bounded wait expired) or MOE_ERR_DEVICE_CHECK. A non-zero word
 * is cleared; the kernels leave the rest of the workspace ready for the next call even after
 * an expired wait. */
moe_status_t moe_get_device_status(void *workspace, moe_stream_t stream);

/* Upper bound, in nanoseconds, of every device-side wait (exchanges between CTAs, copy
 * completion).
 * Default 2e9 (2 s). Values are clamped to [0, 6e10]; 0 makes every wait that is not
 * already satisfied expire at once, which tests use to exercise the timeout path. */
void moe_set_wait_limit_ns(uint64_t ns);

#ifdef __cplusplus
}
#endif
#endif /* MOE_H_ */
