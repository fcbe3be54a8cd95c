// moe_quant.cu -- HQQ-style group quantiser: bf16 weights -> the canonical expert format
// (b-bit codes, fp16 scale and zero per 64-wide group along a row).
//
// Method (Half-Quadratic Quantization, H. Badri and A. Shaji, 2023; the page "Krasis update",
// list of the v1.0 results, names it at 4, 6 and 8 bits, built from the weights alone): the
// min-max scale of a group is kept and only the zero point is optimised, by half-quadratic
// splitting of an l_p (p <= 1) reconstruction error. Per group, Q = 2^b - 1:
//   s = fp16((max - min) / Q), z = -min / s;
//   repeat: q = clamp(rint(w/s + z), 0, Q), r = (q - z) s, err = sum |w - r| -- stop when err
//   does not fall below (1 - 2^-40) best (the best zero is kept) -- e = shrink_p(w - r, beta),
//   z = mean(q - (w - e)/s), beta *= kappa;
//   store fp16(best z) and the nearest codes of the stored grid.
// shrink_p(x, beta) = sign(x) max(|x| - |x|^(p-1)/beta, 0), the generalised soft threshold.
// The 2^-40 margin makes the stop test the one exact arithmetic takes: near its optimum the L1
// error is flat in the zero, successive iterates often have equal error, and the rounding of a
// 64-term sum (below 2^-46 of it in any order) would otherwise decide those ties.
//
// Work split: one thread per group, so that both sums over a group (the error and the new
// zero) run in index order, the order in which the method's definition writes them; with every
// other step an unfused, correctly rounded IEEE fp64 operation, a thread computes the same bits
// as that definition. (A warp per group with butterfly sums was measured, in a CPU model of its
// arithmetic, to change 1 group in 10,000: the zero moves in steps of exactly 1/64 and bf16
// weights sit on coarse grids, so real-arithmetic ties in the codes are common and the
// summation order decides them.) Only the power function of the shrink is not correctly
// rounded, which matters only where the shrink is active.
// Groups stop after different numbers of steps, so each thread runs a flat loop of steps and
// moves to its next group when the current one stops; a warp runs in lockstep only within a
// step. The group's 64 weights sit in shared memory, element-major across the block's threads
// (conflict-free), loaded with eight 16-byte reads per thread.
// The kernel is bound by the fp64 pipe, not by memory: 2 bytes read and b/8 + 1/16 bytes written
// per weight, against roughly 40 fp64 operations and three divisions per weight and step, plus
// the power function of the shrink for the weights outside its dead zone.
#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kQuantThreads = 128;
constexpr double kFall = 1.0 - 0x1p-40;   // an error must fall below kFall * best to count

struct QuantArgs {
    double p, beta, kappa;
    int iters;
};

// nearest code of w on the grid (q - z) * s, q in 0..qmax
__device__ __forceinline__ double grid_code(double w, double s, double z, double qmax) {
    const double q = rint(__dadd_rn(__ddiv_rn(w, s), z));
    return fmin(fmax(q, 0.0), qmax);
}

// The shrink is 0 on its dead zone |x| <= beta^(-1/(2-p)). `dead` is that bound lowered by a
// relative 2^-20: below it the exact |x| - |x|^(p-1)/beta is negative by more than 2^-20 of |x|,
// a million times the error of the power function and the division, so the formula evaluated in
// fp64 is negative too and the result is the same 0 -- without the power function, which is
// most of the step's cost when the shrink is inactive (as for LLM-like weights at the published
// defaults).
__device__ __forceinline__ double dead_zone(double beta, double p) {
    return p < 1.0 ? __dmul_rn(pow(beta, -1.0 / (2.0 - p)), 1.0 - 0x1p-20) : 0.0;
}

__device__ __forceinline__ double shrink_lp(double x, double beta, double p, double dead) {
    if (x == 0.0) return 0.0;
    const double a = fabs(x);
    if (a < dead) return 0.0;
    const double pw = p == 1.0 ? 1.0 : pow(a, p - 1.0);   // pow(a, 0) is exactly 1
    const double t = __dsub_rn(a, __ddiv_rn(pw, beta));
    return t > 0.0 ? copysign(t, x) : 0.0;
}

__device__ __forceinline__ uint16_t f64_to_f16_bits(double v) {
    return __half_as_ushort(__double2half(v));   // round to nearest even
}

__device__ __forceinline__ double f16_bits_to_f64(uint16_t h) {
    return (double)__half2float(__ushort_as_half(h));
}

// weight j of this thread's group (element-major shared layout: [j][thread])
__device__ __forceinline__ double wt(const uint16_t *sw, int j) {
    return (double)__uint_as_float((uint32_t)sw[j * kQuantThreads] << 16);
}

__global__ void __launch_bounds__(kQuantThreads)
    hqq_quantize_kernel(const uint4 *__restrict__ w, long long ngroups, int bits, const QuantArgs a,
                        uint32_t *__restrict__ codes, uint16_t *__restrict__ scale, uint16_t *__restrict__ zero,
                        int32_t *__restrict__ iters_used) {
    __shared__ uint16_t smem_w[kGroup * kQuantThreads];
    uint16_t *sw = smem_w + threadIdx.x;
    const double qmax = (double)((1 << bits) - 1);
    const int words = 2 * bits;   // 32-bit words in a group's 8*bits-byte code block
    const long long stride = (long long)gridDim.x * kQuantThreads;

    long long g = (long long)blockIdx.x * kQuantThreads + threadIdx.x;
    double s = 1.0, z = 0.0, zbest = 0.0, best = 0.0, beta = 0.0;
    uint16_t sb = 0;
    int step = 0;
    bool start = true;   // the thread has to set up group g
    while (g < ngroups) {
        if (start) {
            // load: the group's 128 bytes, eight 16-byte reads, stored element-major
            const uint4 *src = w + g * (kGroup / 8);
#pragma unroll
            for (int k = 0; k < kGroup / 8; ++k) {
                const uint4 v = __ldg(src + k);
                const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    sw[(8 * k + 2 * m) * kQuantThreads] = (uint16_t)(u[m] & 0xffffu);
                    sw[(8 * k + 2 * m + 1) * kQuantThreads] = (uint16_t)(u[m] >> 16);
                }
            }
            // min-max scale and the starting zero
            double lo = wt(sw, 0), hi = lo;
            for (int j = 1; j < kGroup; ++j) {
                const double v = wt(sw, j);
                lo = v < lo ? v : lo;
                hi = v > hi ? v : hi;
            }
            if (lo == hi) {   // constant group: quantise over [min(c, 0), max(c, 0)]; all zero: scale 1
                if (lo == 0.0) {
                    hi = qmax;
                } else {
                    lo = fmin(lo, 0.0);
                    hi = fmax(hi, 0.0);
                }
            }
            sb = f64_to_f16_bits(fmin(__ddiv_rn(__dsub_rn(hi, lo), qmax), 65504.0));
            if (sb == 0) sb = 1;   // least positive fp16
            s = f16_bits_to_f64(sb);
            z = __ddiv_rn(-lo, s);
            zbest = z;
            best = __longlong_as_double(0x7ff0000000000000ll);   // +inf
            beta = a.beta;
            step = 0;
            start = false;
        }

        bool done = step >= a.iters;
        if (!done) {
            // one half-quadratic step: the error at z, then (if it fell) the shrink and the new zero
            double err = 0.0;
            for (int j = 0; j < kGroup; ++j) {
                const double v = wt(sw, j);
                const double d = __dsub_rn(v, __dmul_rn(__dsub_rn(grid_code(v, s, z, qmax), z), s));
                err = __dadd_rn(err, fabs(d));
            }
            ++step;
            if (!(err < __dmul_rn(best, kFall))) {
                done = true;
            } else {
                best = err;
                zbest = z;
                const double dead = dead_zone(beta, a.p);
                double acc = 0.0;
                for (int j = 0; j < kGroup; ++j) {
                    const double v = wt(sw, j);
                    const double q = grid_code(v, s, z, qmax);
                    const double e = shrink_lp(__dsub_rn(v, __dmul_rn(__dsub_rn(q, z), s)), beta, a.p, dead);
                    acc = __dadd_rn(acc, __dsub_rn(q, __ddiv_rn(__dsub_rn(v, e), s)));
                }
                z = __ddiv_rn(acc, (double)kGroup);
                beta = __dmul_rn(beta, a.kappa);
                done = step >= a.iters;
            }
        }

        if (done) {
            // store: fp16 zero of the best step and the nearest codes of the stored grid, packed
            // into the canonical bit string (code j at bits [j*bits, (j+1)*bits))
            const uint16_t zb = f64_to_f16_bits(fmin(fmax(zbest, -65504.0), 65504.0));
            const double zs = f16_bits_to_f64(zb);
            uint32_t *dst = codes + g * words;
            uint64_t acc = 0;
            int nb = 0, wi = 0;
            for (int j = 0; j < kGroup; ++j) {
                acc |= (uint64_t)grid_code(wt(sw, j), s, zs, qmax) << nb;
                nb += bits;
                if (nb >= 32) {
                    dst[wi++] = (uint32_t)acc;
                    acc >>= 32;
                    nb -= 32;
                }
            }
            scale[g] = sb;
            zero[g] = zb;
            if (iters_used) iters_used[g] = step;
            g += stride;
            start = true;
        }
    }
}

}  // namespace

moe_status_t launch_quantize_hqq(const uint16_t *w, int rows, int cols, int bits, double p, double beta,
                                 double kappa, int iters, void *codes, uint16_t *scale, uint16_t *zero,
                                 int32_t *iters_used, cudaStream_t st) {
    const long long groups = (long long)rows * (cols / kGroup);
    if (groups == 0) return MOE_OK;
    const DeviceInfo *d = device_info();
    if (!d) return MOE_ERR_CUDA;
    // one wave of resident blocks; the threads stride over the groups
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, hqq_quantize_kernel, kQuantThreads, 0) !=
            cudaSuccess ||
        per_sm < 1)
        return MOE_ERR_CUDA;
    long long blocks = (groups + kQuantThreads - 1) / kQuantThreads;
    const long long cap = (long long)d->sms * per_sm;
    if (blocks > cap) blocks = cap;
    const QuantArgs a{p, beta, kappa, iters};
    hqq_quantize_kernel<<<(unsigned)blocks, kQuantThreads, 0, st>>>(
        reinterpret_cast<const uint4 *>(w), groups, bits, a, static_cast<uint32_t *>(codes), scale, zero,
        iters_used);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
