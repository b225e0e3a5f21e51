// synth.cu -- seeded synthetic LLM-like weights on the device.
//
// Input generator only: it holds none of the quantization method's arithmetic
// and is shared by the tests, the benchmark and the smoke check.
//
// Distribution: Student-t with nu = 4 degrees of freedom, scaled to a target
// standard deviation (t(4) has variance 2), then an independent fraction of
// entries multiplied by an outlier factor, then rounded to fp16.
//   Z     = sqrt(-2 ln U1) cos(2 pi U2)          (Box-Muller)
//   chi2  = -2 ln(U3 U4)                          (chi-square, 4 d.o.f.)
//   t     = Z / sqrt(chi2 / 4)
// Uniforms come from the counter-based generator Philox4x32-10 (J. Salmon,
// M. Moraes, R. Dror, D. Shaw, "Parallel random numbers: as easy as 1, 2, 3",
// SC'11): counter = (element index lo, hi, draw, 0), key = (seed, stream).
#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace {

struct u4 { uint32_t x, y, z, w; };

__device__ __forceinline__ u4 philox4x32_10(u4 c, uint32_t k0, uint32_t k1) {
    const uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;
    const uint32_t W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        const uint32_t hi0 = __umulhi(M0, c.x), lo0 = M0 * c.x;
        const uint32_t hi1 = __umulhi(M1, c.z), lo1 = M1 * c.z;
        c = u4{hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0};
        k0 += W0;
        k1 += W1;
    }
    return c;
}

__device__ __forceinline__ float unit_open(uint32_t x) {  // (0, 1)
    return ((float)(x >> 8) + 0.5f) * (1.0f / 16777216.0f);
}

__global__ void student_t_kernel(__half* __restrict__ out, int64_t n, uint32_t seed,
                                 uint32_t stream, float scale, uint32_t outlier_thresh,
                                 float outlier_mult) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
        const uint32_t lo = (uint32_t)i, hi = (uint32_t)((uint64_t)i >> 32);
        const u4 a = philox4x32_10(u4{lo, hi, 0u, 0u}, seed, stream);
        const u4 b = philox4x32_10(u4{lo, hi, 1u, 0u}, seed, stream);
        const float zn = sqrtf(-2.0f * logf(unit_open(a.x))) * cospif(2.0f * unit_open(a.y));
        const float chi2 = -2.0f * (logf(unit_open(a.z)) + logf(unit_open(a.w)));
        float v = zn * rsqrtf(chi2 * 0.25f) * scale;
        if (b.x < outlier_thresh) v *= outlier_mult;
        out[i] = __float2half_rn(v);
    }
}

}  // namespace

extern "C" int synth_student_t_fp16(void* out, int64_t n, uint32_t seed, uint32_t stream,
                                    float std_target, double outlier_frac,
                                    float outlier_mult, void* cuda_stream) {
    if (n <= 0) return 0;
    if (out == nullptr) return 1;
    const float scale = std_target * 0.70710678118654752f;  // t(4) has std sqrt(2)
    double th = outlier_frac * 4294967296.0;
    if (th < 0) th = 0;
    if (th > 4294967295.0) th = 4294967295.0;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t blocks = (n + 255) / 256;
    if (blocks > (int64_t)sms * 32) blocks = (int64_t)sms * 32;
    student_t_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)cuda_stream>>>(
        (__half*)out, n, seed, stream, scale, (uint32_t)th, outlier_mult);
    return cudaGetLastError() == cudaSuccess ? 0 : 6;
}
