// hqq_dequantize.cu -- Q^-1 of "Half-Quadratic Quantization of Large Machine
// Learning Models", section 2: W_hat = s (Wq - z), as fp16((code - z) * s) in
// binary32 from the stored fp16 scale and zero.
//
// Streaming kernel: the unit of work is 8 consecutive weights (one 16-byte
// store), which always lie in one group (8 divides every group size).  Lane l
// of a warp takes unit base + l, so each warp instruction reads a contiguous
// run of packed codes and writes 512 contiguous bytes.
#include "hqq_common.cuh"

namespace hqq {

constexpr int kDqThreads = 256;
constexpr int kDqUnroll = 4;

__device__ __forceinline__ float code_to_float(uint32_t c) {
    return __fsub_rn(__uint_as_float(0x4B000000u | c), 8388608.0f);   // exact for c < 2^23
}

template <int NBITS>
__device__ __forceinline__ void unit_codes(const uint8_t* __restrict__ packed, int64_t u,
                                           uint32_t (&c)[8]) {
    if constexpr (NBITS == 4) {
        const uint32_t wd = __ldg(reinterpret_cast<const uint32_t*>(packed) + u);
#pragma unroll
        for (int i = 0; i < 8; ++i) c[i] = (wd >> (4 * i)) & 15u;
    } else if constexpr (NBITS == 2) {
        const uint32_t h = __ldg(reinterpret_cast<const uint16_t*>(packed) + u);
#pragma unroll
        for (int i = 0; i < 8; ++i) c[i] = (h >> (2 * i)) & 3u;
    } else {
        const int64_t e0 = u * 8;
        const int64_t w0 = e0 / 10;
        const uint32_t k0 = (uint32_t)(e0 - w0 * 10);       // 0, 2, 4, 6 or 8
        const uint32_t* p32 = reinterpret_cast<const uint32_t*>(packed);
        const uint64_t lo = __ldg(p32 + w0);
        // codes k0..k0+7 reach into the next word when k0 > 2 (that word exists:
        // it holds the unit's own last code)
        const uint64_t hi = k0 > 2 ? (uint64_t)__ldg(p32 + w0 + 1) : 0ull;
        const uint64_t v = (lo | (hi << 30)) >> (3 * k0);
#pragma unroll
        for (int i = 0; i < 8; ++i) c[i] = (uint32_t)(v >> (3 * i)) & 7u;
    }
}

template <int NBITS>
__global__ void __launch_bounds__(kDqThreads)
dequantize_kernel(const __grid_constant__ DequantParams prm, int log2_group) {
    const int64_t per_block = (int64_t)kDqThreads * kDqUnroll;
    for (int64_t base = (int64_t)blockIdx.x * per_block; base < prm.n_units;
         base += (int64_t)gridDim.x * per_block) {
        // all loads of the kDqUnroll units first, so they are in flight together
        uint32_t c[kDqUnroll][8];
        float sf[kDqUnroll], zf[kDqUnroll];
        bool ok[kDqUnroll];
#pragma unroll
        for (int r = 0; r < kDqUnroll; ++r) {
            const int64_t u = base + r * kDqThreads + threadIdx.x;
            ok[r] = u < prm.n_units;
            const int64_t uu = ok[r] ? u : 0;
            const int64_t g = (uu * 8) >> log2_group;
            sf[r] = __half2float(__ldg(prm.scale + g));
            zf[r] = __half2float(__ldg(prm.zero + g));
            unit_codes<NBITS>(prm.packed, uu, c[r]);
        }
#pragma unroll
        for (int r = 0; r < kDqUnroll; ++r) {
            uint32_t o[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float a = __fmul_rn(__fsub_rn(code_to_float(c[r][2 * k]), zf[r]), sf[r]);
                const float b = __fmul_rn(__fsub_rn(code_to_float(c[r][2 * k + 1]), zf[r]), sf[r]);
                const __half2 h = __floats2half2_rn(a, b);
                o[k] = *reinterpret_cast<const uint32_t*>(&h);
            }
            if (ok[r]) {
                const int64_t u = base + r * kDqThreads + threadIdx.x;
                reinterpret_cast<uint4*>(prm.out)[u] = make_uint4(o[0], o[1], o[2], o[3]);
            }
        }
    }
}

cudaError_t launch_dequantize(const DequantParams& prm, int nbits, int log2_group,
                              cudaStream_t stream) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t per_block = (int64_t)kDqThreads * kDqUnroll;
    int64_t blocks = (prm.n_units + per_block - 1) / per_block;
    const int64_t cap = (int64_t)sms * 32;
    if (blocks > cap) blocks = cap;
    switch (nbits) {
        case 2: dequantize_kernel<2><<<(unsigned)blocks, kDqThreads, 0, stream>>>(prm, log2_group); break;
        case 3: dequantize_kernel<3><<<(unsigned)blocks, kDqThreads, 0, stream>>>(prm, log2_group); break;
        case 4: dequantize_kernel<4><<<(unsigned)blocks, kDqThreads, 0, stream>>>(prm, log2_group); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace hqq
