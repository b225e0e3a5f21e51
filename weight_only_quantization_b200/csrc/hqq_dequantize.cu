// hqq_dequantize.cu -- Q^-1 of "Half-Quadratic Quantization of Large Machine
// Learning Models", section 2: W_hat = s (Wq - z), as fp16((code - z) * s) in
// binary32 from the stored fp16 scale and zero.
//
// Streaming kernel (HBM-bound).  The unit of work is 8 consecutive weights:
// one 16-byte output, always inside one group (8 divides every group size).
// Lane l of a block takes units base + r*256 + l, so every warp load is a
// contiguous run of packed codes and every warp store writes 512 contiguous
// bytes (streaming stores: the output is written once and not re-read by this
// kernel); all loads of a thread's units are issued before any store.  No shared
// memory, so occupancy is limited only by registers (staging the output tile
// in shared memory for TMA bulk stores measured slower: it cost occupancy).
// The code-to-weight arithmetic is in hqq_unpack.cuh.
#include "hqq_unpack.cuh"

namespace hqq {

constexpr int kDqThreads = 256;
constexpr int kDqUnits = 4;                          // units per thread per pass
constexpr int kDqTile = kDqThreads * kDqUnits;

// META bit 0: zero points in 8-bit form; bit 1: scales in 8-bit form.
template <int NBITS, bool SMALL, int META>
__global__ void __launch_bounds__(kDqThreads)
dequantize_kernel(const __grid_constant__ DequantParams prm, int log2_group) {
    for (int64_t base = (int64_t)blockIdx.x * kDqTile; base < prm.n_units;
         base += (int64_t)gridDim.x * kDqTile) {
        // 8-bit units are 64 bits (fetched raw); narrower ones one word; 3 bits
        // (word indices < 2^32): the warp's 32 consecutive units span at most
        // 27 words, so lane l loads word l of the span and each unit takes its
        // two words from their lanes by shuffle
        constexpr bool kWarp3 = NBITS == 3 && SMALL;
        uint32_t x[kDqUnits];
        UnitRaw x8[NBITS == 8 ? kDqUnits : 1];
        float sf[kDqUnits], zf[kDqUnits];
#pragma unroll
        for (int r = 0; r < kDqUnits; ++r) {        // all loads first
            int64_t u = base + r * kDqThreads + threadIdx.x;
            if (u >= prm.n_units) u = 0;
            const int64_t g = (u * 8) >> log2_group;
            sf[r] = (META & 2) ? restore_meta(prm.sq, g) : __half2float(__ldg(prm.scale + g));
            zf[r] = (META & 1) ? restore_meta(prm.zq, g) : __half2float(__ldg(prm.zero + g));
            if constexpr (NBITS == 8) {
                x8[r] = unit_fetch<8, SMALL>(prm.packed, u);
            } else if constexpr (kWarp3) {
                const uint32_t u0 = (uint32_t)(base + r * kDqThreads + (threadIdx.x & ~31u));
                const uint32_t wfirst = __umulhi(4u * u0, 0xCCCCCCCDu) >> 2;   // floor(8 u0 / 10)
                const uint32_t wi = wfirst + (threadIdx.x & 31u);
                x[r] = wi < prm.n_words ? __ldg(reinterpret_cast<const uint32_t*>(prm.packed) + wi)
                                        : 0u;
            } else {
                x[r] = unit_bits<NBITS, SMALL>(prm.packed, u);
            }
        }
#pragma unroll
        for (int r = 0; r < kDqUnits; ++r) {
            const int64_t u = base + r * kDqThreads + threadIdx.x;
            uint4 o;
            if constexpr (NBITS == 8) {
                o = unit8_raw<8>(x8[r], zf[r], sf[r]);
            } else if constexpr (kWarp3) {
                const uint32_t u0 = (uint32_t)(base + r * kDqThreads + (threadIdx.x & ~31u));
                const uint32_t wfirst = __umulhi(4u * u0, 0xCCCCCCCDu) >> 2;
                const uint32_t u4 = 4u * (u0 + (threadIdx.x & 31u));
                const uint32_t a = __umulhi(u4, 0xCCCCCCCDu) >> 2;             // floor(8u / 10)
                const uint32_t k0 = 2u * (u4 - 5u * a);                         // 8u mod 10
                const uint32_t lo = __shfl_sync(0xffffffffu, x[r], (int)(a - wfirst));
                const uint32_t hi = __shfl_sync(0xffffffffu, x[r], (int)(a - wfirst + 1u));
                const uint32_t bits = (uint32_t)(((uint64_t)lo | ((uint64_t)hi << 30)) >> (3u * k0));
                o = unit8<3>(bits, zf[r], sf[r]);
            } else {
                o = unit8<NBITS>(x[r], zf[r], sf[r]);
            }
            if (u < prm.n_units) __stcs(reinterpret_cast<uint4*>(prm.out) + u, o);   // written once: evict first
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
        case 1: launch_dq<1, true>(prm, log2_group, g, stream); break;
        case 2: launch_dq<2, true>(prm, log2_group, g, stream); break;
        case 4: launch_dq<4, true>(prm, log2_group, g, stream); break;
        case 8: launch_dq<8, true>(prm, log2_group, g, stream); break;
        case 3:
            if (small) launch_dq<3, true>(prm, log2_group, g, stream);
            else launch_dq<3, false>(prm, log2_group, g, stream);
            break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace hqq
