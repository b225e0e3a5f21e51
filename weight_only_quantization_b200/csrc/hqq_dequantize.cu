// hqq_dequantize.cu -- Q^-1 of "Half-Quadratic Quantization of Large Machine
// Learning Models", section 2: W_hat = s (Wq - z), as fp16((code - z) * s) in
// binary32 from the stored fp16 scale and zero.
//
// Streaming kernel (HBM-bound).  The unit of work is 8 consecutive weights:
// one 16-byte output, always inside one group (8 divides every group size).
// Lane l of a block takes units base + r*256 + l, so every warp load is a
// contiguous run of packed codes and every warp store writes 512 contiguous
// bytes; all loads of a thread's units are issued before any store.  No shared
// memory, so occupancy is limited only by registers (staging the output tile
// in shared memory for TMA bulk stores measured slower: it cost occupancy).
//
// A code c at bit offset k of a field becomes an exact binary32 value without
// a shift per code: OR-ing the masked field into the mantissa of 2^23 gives
// 2^23 + c 2^k, and fma(x, 2^-k, -2^(23-k)) = c exactly (exact while
// c 2^k < 2^23).  Two codes go through each f32x2 operation; (c - z) is exact
// for fp16 z, so the only roundings are the product with s and the conversion
// to fp16, as the definition requires.
#include "hqq_common.cuh"

namespace hqq {

constexpr int kDqThreads = 256;
constexpr int kDqUnits = 4;                          // units per thread per pass
constexpr int kDqTile = kDqThreads * kDqUnits;

// Exact codes of the fields (mask0) of x0 and (mask1) of x1, as a pair.
__device__ __forceinline__ float2 codes2(uint32_t x0, uint32_t mask0, float inv0, float off0,
                                         uint32_t x1, uint32_t mask1, float inv1, float off1) {
    const float2 f = make_float2(__uint_as_float((x0 & mask0) | 0x4B000000u),
                                 __uint_as_float((x1 & mask1) | 0x4B000000u));
    return __ffma2_rn(f, make_float2(inv0, inv1), make_float2(off0, off1));
}

// fp16((c - z) * s) of a pair of codes, packed into one 32-bit word.
__device__ __forceinline__ uint32_t dq2(float2 c, float z, float s) {
    const float2 v = __fmul2_rn(__fadd2_rn(c, make_float2(-z, -z)), make_float2(s, s));
    const __half2 h = __floats2half2_rn(v.x, v.y);
    return *reinterpret_cast<const uint32_t*>(&h);
}

// Eight codes of bit width B stored LSB-first in the low 8*B bits of `x`.
template <int B>
__device__ __forceinline__ uint4 unit8(uint32_t x, float z, float s) {
    constexpr uint32_t M = (1u << B) - 1u;
    const uint32_t lo = x, hi = x >> (4 * B);        // fields 0..3 and 4..7, each < 2^16
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const int k0 = 2 * j * B, k1 = (2 * j + 1) * B;
        const float2 a = codes2(lo, M << k0, 1.0f / (float)(1u << k0), -(float)(1u << (23 - k0)),
                                lo, M << k1, 1.0f / (float)(1u << k1), -(float)(1u << (23 - k1)));
        const float2 b = codes2(hi, M << k0, 1.0f / (float)(1u << k0), -(float)(1u << (23 - k0)),
                                hi, M << k1, 1.0f / (float)(1u << k1), -(float)(1u << (23 - k1)));
        o[j] = dq2(a, z, s);
        o[j + 2] = dq2(b, z, s);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// The 8*NBITS code bits of unit u, LSB-first.  4/2 bit: one aligned field.
// 3 bit: codes 8u..8u+7 start at slot k0 = 8u mod 10 of word w0 = floor(8u/10)
// and reach into word w0 + 1 when k0 > 2 (that word exists: it holds the
// unit's own last code); words hold 10 codes in bits 0..29.  SMALL: 4u fits
// in 32 bits, so w0 = floor(4u/5) is one multiply-high.
template <int NBITS, bool SMALL>
__device__ __forceinline__ uint32_t unit_bits(const uint8_t* __restrict__ packed, int64_t u) {
    if constexpr (NBITS == 4) {
        return __ldg(reinterpret_cast<const uint32_t*>(packed) + u);
    } else if constexpr (NBITS == 2) {
        return __ldg(reinterpret_cast<const uint16_t*>(packed) + u);
    } else {
        int64_t w0;
        uint32_t k0;
        if (SMALL) {
            const uint32_t u4 = 4u * (uint32_t)u;
            const uint32_t q = __umulhi(u4, 0xCCCCCCCDu) >> 2;      // floor(u4 / 5)
            w0 = q;
            k0 = 2u * (u4 - 5u * q);                                 // 8u mod 10
        } else {
            w0 = (4 * u) / 5;
            k0 = (uint32_t)(8 * u - 10 * w0);
        }
        const uint32_t* p32 = reinterpret_cast<const uint32_t*>(packed);
        const uint64_t lo = __ldg(p32 + w0);
        const uint64_t hi = k0 > 2 ? (uint64_t)__ldg(p32 + w0 + 1) : 0ull;
        return (uint32_t)((lo | (hi << 30)) >> (3 * k0));
    }
}

// Zero point or scale of group g restored from its 8-bit form (method section
// 4.1's 8-bit meta data): fp16((c - z2) s2) with the second-level fp16 s2, z2.
__device__ __forceinline__ float restore_meta(const Meta8& m, int64_t g) {
    const int64_t k = g >> m.shift;
    const float c = (float)__ldg(m.codes + g);
    const float v = __fmul_rn(__fsub_rn(c, __half2float(__ldg(m.zero + k))),
                              __half2float(__ldg(m.scale + k)));
    return __half2float(__float2half_rn(v));
}

// META bit 0: zero points in 8-bit form; bit 1: scales in 8-bit form.
template <int NBITS, bool SMALL, int META>
__global__ void __launch_bounds__(kDqThreads)
dequantize_kernel(const __grid_constant__ DequantParams prm, int log2_group) {
    for (int64_t base = (int64_t)blockIdx.x * kDqTile; base < prm.n_units;
         base += (int64_t)gridDim.x * kDqTile) {
        uint32_t x[kDqUnits];
        float sf[kDqUnits], zf[kDqUnits];
#pragma unroll
        for (int r = 0; r < kDqUnits; ++r) {        // all loads first
            int64_t u = base + r * kDqThreads + threadIdx.x;
            if (u >= prm.n_units) u = 0;
            const int64_t g = (u * 8) >> log2_group;
            sf[r] = (META & 2) ? restore_meta(prm.sq, g) : __half2float(__ldg(prm.scale + g));
            zf[r] = (META & 1) ? restore_meta(prm.zq, g) : __half2float(__ldg(prm.zero + g));
            x[r] = unit_bits<NBITS, SMALL>(prm.packed, u);
        }
#pragma unroll
        for (int r = 0; r < kDqUnits; ++r) {
            const int64_t u = base + r * kDqThreads + threadIdx.x;
            const uint4 o = unit8<NBITS>(x[r], zf[r], sf[r]);
            if (u < prm.n_units) reinterpret_cast<uint4*>(prm.out)[u] = o;
        }
    }
}

template <int NBITS, bool SMALL>
static void launch_dq(const DequantParams& prm, int log2_group, unsigned grid, cudaStream_t stream) {
    const int meta = (prm.zq.codes ? 1 : 0) | (prm.sq.codes ? 2 : 0);
    switch (meta) {
        case 0: dequantize_kernel<NBITS, SMALL, 0><<<grid, kDqThreads, 0, stream>>>(prm, log2_group); break;
        case 1: dequantize_kernel<NBITS, SMALL, 1><<<grid, kDqThreads, 0, stream>>>(prm, log2_group); break;
        case 2: dequantize_kernel<NBITS, SMALL, 2><<<grid, kDqThreads, 0, stream>>>(prm, log2_group); break;
        default: dequantize_kernel<NBITS, SMALL, 3><<<grid, kDqThreads, 0, stream>>>(prm, log2_group); break;
    }
}

cudaError_t launch_dequantize(const DequantParams& prm, int nbits, int log2_group,
                              cudaStream_t stream) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t blocks = (prm.n_units + kDqTile - 1) / kDqTile;
    const int64_t cap = (int64_t)sms * 32;
    if (blocks > cap) blocks = cap;
    const bool small = prm.n_units < ((int64_t)1 << 30);
    const unsigned g = (unsigned)blocks;
    switch (nbits) {
        case 2: launch_dq<2, true>(prm, log2_group, g, stream); break;
        case 4: launch_dq<4, true>(prm, log2_group, g, stream); break;
        case 3:
            if (small) launch_dq<3, true>(prm, log2_group, g, stream);
            else launch_dq<3, false>(prm, log2_group, g, stream);
            break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace hqq
