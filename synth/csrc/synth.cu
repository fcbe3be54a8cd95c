// synth.cu -- device-side copy of the seeded input generator in synth/__init__.py.
//
// Input plumbing only (no step of the expert block's arithmetic). Every element is a pure
// function of (key, index): SplitMix64 draws (Steele, Lea & Flood 2014) used counter-style,
// Box-Muller normals (cosine branch) with the logarithm from the artanh series (Abramowitz &
// Stegun 4.1.27) and the cosine from its Taylor series after an exact turn reduction. All
// double arithmetic goes through __dadd_rn/__dmul_rn/__ddiv_rn/__dsqrt_rn so that no
// multiply-add is fused and the host (numpy) and device produce identical bits.
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace {

constexpr unsigned long long kGamma = 0x9E3779B97F4A7C15ull;

__device__ __forceinline__ unsigned long long mix64(unsigned long long z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}
__device__ __forceinline__ unsigned long long draw(unsigned long long key, unsigned long long i) {
    return mix64(key + (i + 1ull) * kGamma);
}
__device__ __forceinline__ double uniform_open(unsigned long long d) {
    return __dmul_rn(__dadd_rn(__dmul_rn((double)(d >> 12), 2.0), 1.0), 0x1.0p-53);
}

__constant__ double kAtanh[12] = {0x1.0000000000000p+0, 0x1.5555555555555p-2, 0x1.999999999999ap-3,
                                  0x1.2492492492492p-3, 0x1.c71c71c71c71cp-4, 0x1.745d1745d1746p-4,
                                  0x1.3b13b13b13b14p-4, 0x1.1111111111111p-4, 0x1.e1e1e1e1e1e1ep-5,
                                  0x1.af286bca1af28p-5, 0x1.8618618618618p-5, 0x1.642c8590b2164p-5};
__constant__ double kCos[11] = {0x1.0000000000000p+0,  -0x1.0000000000000p-1, 0x1.5555555555555p-5,
                                -0x1.6c16c16c16c17p-10, 0x1.a01a01a01a01ap-16, -0x1.27e4fb7789f5cp-22,
                                0x1.1eed8eff8d898p-29,  -0x1.93974a8c07c9dp-37, 0x1.ae7f3e733b81fp-45,
                                -0x1.6827863b97d97p-53, 0x1.e542ba4020225p-62};
__constant__ double kSin[11] = {0x1.0000000000000p+0,  -0x1.5555555555555p-3, 0x1.1111111111111p-7,
                                -0x1.a01a01a01a01ap-13, 0x1.71de3a556c734p-19, -0x1.ae64567f544e4p-26,
                                0x1.6124613a86d09p-33,  -0x1.ae7f3e733b81fp-41, 0x1.952c77030ad4ap-49,
                                -0x1.2f49b46814157p-57, 0x1.71b8ef6dcf572p-66};
constexpr double kLn2 = 0x1.62e42fefa39efp-1;
constexpr double kTwoPi = 0x1.921fb54442d18p+2;
constexpr double kSqrt2 = 0x1.6a09e667f3bcdp+0;

__device__ double ln_series(double u) {
    const unsigned long long bits = (unsigned long long)__double_as_longlong(u);
    long long e = (long long)((bits >> 52) & 0x7FFull) - 1023;
    double m = __longlong_as_double((long long)((bits & 0x000FFFFFFFFFFFFFull) | 0x3FF0000000000000ull));
    if (m > kSqrt2) {
        m = __dmul_rn(m, 0.5);
        e += 1;
    }
    const double t = __ddiv_rn(__dadd_rn(m, -1.0), __dadd_rn(m, 1.0));
    const double t2 = __dmul_rn(t, t);
    double p = kAtanh[11];
    for (int n = 10; n >= 0; --n) p = __dadd_rn(__dmul_rn(p, t2), kAtanh[n]);
    const double ln_m = __dmul_rn(2.0, __dmul_rn(t, p));
    return __dadd_rn(__dmul_rn((double)e, kLn2), ln_m);
}

__device__ double cos_turns(double v) {
    if (v > 0.5) v = __dadd_rn(1.0, -v);
    const bool neg = v > 0.25;
    if (neg) v = __dadd_rn(0.5, -v);
    const bool use_cos = v <= 0.125;
    const double a = __dmul_rn(kTwoPi, use_cos ? v : __dadd_rn(0.25, -v));
    const double a2 = __dmul_rn(a, a);
    double r;
    if (use_cos) {
        double p = kCos[10];
        for (int n = 9; n >= 0; --n) p = __dadd_rn(__dmul_rn(p, a2), kCos[n]);
        r = p;
    } else {
        double p = kSin[10];
        for (int n = 9; n >= 0; --n) p = __dadd_rn(__dmul_rn(p, a2), kSin[n]);
        r = __dmul_rn(a, p);
    }
    return neg ? -r : r;
}

__device__ double normal_at(unsigned long long key, unsigned long long i) {
    const double u1 = uniform_open(draw(key, 2ull * i));
    const double u2 = uniform_open(draw(key, 2ull * i + 1ull));
    return __dmul_rn(__dsqrt_rn(__dmul_rn(-2.0, ln_series(u1))), cos_turns(u2));
}

__device__ __forceinline__ uint16_t to_bf16(double v) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(__double2float_rn(v)));
}
__device__ __forceinline__ uint16_t to_f16(double v) {
    return __half_as_ushort(__float2half_rn(__double2float_rn(v)));
}

// kind 0: bf16(normal); 1: fp32(normal / sqrt(H)) (param = H); 2: fp16(|normal| * sqrt(0.02) + 1e-3) * mult
// (param = bits); 3: fp16(uniform * (2^bits - 1)) (param = bits).
__global__ void fill_kernel(void *out, unsigned long long key, unsigned long long start, unsigned long long n,
                            int kind, int param) {
    for (unsigned long long i = blockIdx.x * (unsigned long long)blockDim.x + threadIdx.x; i < n;
         i += (unsigned long long)gridDim.x * blockDim.x) {
        const unsigned long long j = start + i;
        if (kind == 0) {
            static_cast<uint16_t *>(out)[i] = to_bf16(normal_at(key, j));
        } else if (kind == 1) {
            static_cast<float *>(out)[i] = __double2float_rn(__ddiv_rn(normal_at(key, j), __dsqrt_rn((double)param)));
        } else if (kind == 2) {
            const double z = normal_at(key, j);
            const double mult = __ddiv_rn(15.0, (double)((1 << param) - 1));
            const double s = __dmul_rn(__dadd_rn(__dmul_rn(fabs(z), 0x1.21a1851ff630ap-3), 1e-3), mult);
            static_cast<uint16_t *>(out)[i] = to_f16(s);
        } else {
            const double u = uniform_open(draw(key, j));
            static_cast<uint16_t *>(out)[i] = to_f16(__dmul_rn(u, (double)((1 << param) - 1)));
        }
    }
}

__global__ void bytes_kernel(uint8_t *out, unsigned long long key, unsigned long long start_byte,
                             unsigned long long nbytes) {
    for (unsigned long long i = blockIdx.x * (unsigned long long)blockDim.x + threadIdx.x; i < nbytes;
         i += (unsigned long long)gridDim.x * blockDim.x) {
        const unsigned long long b = start_byte + i;
        out[i] = (uint8_t)(draw(key, b >> 3) >> (8 * (b & 7)));
    }
}

unsigned grid_for(unsigned long long n) {
    unsigned long long b = (n + 255) / 256;
    return (unsigned)(b < 65536 ? (b ? b : 1) : 65536);
}

}  // namespace

extern "C" {
// Fills `out` (device) with elements start..start+n-1 of the stream `key`; see fill_kernel.
int synth_fill(void *out, unsigned long long key, unsigned long long start, unsigned long long n, int kind,
               int param, void *stream) {
    if (n == 0) return 0;
    fill_kernel<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(out, key, start, n, kind, param);
    return (int)cudaGetLastError();
}
int synth_bytes(void *out, unsigned long long key, unsigned long long start_byte, unsigned long long nbytes,
                void *stream) {
    if (nbytes == 0) return 0;
    bytes_kernel<<<grid_for(nbytes), 256, 0, (cudaStream_t)stream>>>(static_cast<uint8_t *>(out), key, start_byte,
                                                                      nbytes);
    return (int)cudaGetLastError();
}
}
