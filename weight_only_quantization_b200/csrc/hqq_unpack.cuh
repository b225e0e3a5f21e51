// hqq_unpack.cuh -- packed codes to fp16 weights, shared by the dequantize
// kernel and the producers of the weight-only linear layer, so that both form
// exactly W_hat = fp16((code - z) * s) of "Half-Quadratic Quantization of Large
// Machine Learning Models", section 2 (Q^-1), in binary32.
//
// A unit is 8 consecutive codes of the flat row-major index (one 16-byte fp16
// output); 8 divides every group size, so a unit never straddles groups.
//
// A code c at bit offset k of a field becomes an exact binary32 value without
// a shift per code: OR-ing the masked field into the mantissa of 2^23 gives
// 2^23 + c 2^k, and fma(x, 2^-k, -2^(23-k)) = c exactly (exact while
// c 2^k < 2^23).  Two codes go through each f32x2 operation; (c - z) is exact
// for fp16 z, so the only roundings are the product with s and the conversion
// to fp16, as the definition requires.
#pragma once
#include "hqq_params.cuh"

namespace hqq {

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
// unit_bits in two steps, so that a caller can keep loads in flight: the raw
// words of unit u (w0 and, for 3 bits, w1 and the bit shift) and their merge.
struct UnitRaw {
    uint32_t w0, w1, shift;
};

template <int NBITS, bool SMALL>
__device__ __forceinline__ UnitRaw unit_fetch(const uint8_t* __restrict__ packed, int64_t u) {
    UnitRaw r;
    r.w1 = 0u;
    r.shift = 0u;
    if constexpr (NBITS == 8) {                       // 8 bytes: w0 codes 0..3, w1 codes 4..7
        const uint2 v = __ldg(reinterpret_cast<const uint2*>(packed) + u);
        r.w0 = v.x;
        r.w1 = v.y;
    } else if constexpr (NBITS == 1) {
        r.w0 = __ldg(packed + u);
    } else if constexpr (NBITS == 4) {
        r.w0 = __ldg(reinterpret_cast<const uint32_t*>(packed) + u);
    } else if constexpr (NBITS == 2) {
        r.w0 = __ldg(reinterpret_cast<const uint16_t*>(packed) + u);
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
        r.w0 = __ldg(p32 + w0);
        r.w1 = k0 > 2 ? __ldg(p32 + w0 + 1) : 0u;
        r.shift = 3u * k0;
    }
    return r;
}

template <int NBITS>
__device__ __forceinline__ uint32_t unit_merge(const UnitRaw& r) {
    if constexpr (NBITS == 3)
        return (uint32_t)(((uint64_t)r.w0 | ((uint64_t)r.w1 << 30)) >> r.shift);
    else
        return r.w0;
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

__device__ __forceinline__ __half restore_meta_h(const Meta8& m, int64_t g) {
    const int64_t k = g >> m.shift;
    const float c = (float)__ldg(m.codes + g);
    return __float2half_rn(__fmul_rn(__fsub_rn(c, __half2float(__ldg(m.zero + k))),
                                     __half2float(__ldg(m.scale + k))));
}

// Eight 8-bit codes (bytes of w0 then w1) -> fp16((c - z) s).  Byte i becomes
// the mantissa of 2^23 by one byte permute; subtracting 2^23 is exact.
__device__ __forceinline__ uint4 unit8_bytes(uint32_t w0, uint32_t w1, float z, float s) {
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t w = j < 2 ? w0 : w1;
        const int b0 = 2 * (j & 1), b1 = b0 + 1;
        // result bytes: (code, 0x00, 0x00, 0x4B) from (w, 0x4B000000)
        const float2 f = make_float2(
            __uint_as_float(__byte_perm(w, 0x4B000000u, (uint32_t)b0 | 0x7440u)),
            __uint_as_float(__byte_perm(w, 0x4B000000u, (uint32_t)b1 | 0x7440u)));
        const float2 c = __fadd2_rn(f, make_float2(-8388608.0f, -8388608.0f));
        o[j] = dq2(c, z, s);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// The eight weights of a fetched unit, for every width.
template <int NBITS>
__device__ __forceinline__ uint4 unit8_raw(const UnitRaw& r, float z, float s) {
    if constexpr (NBITS == 8)
        return unit8_bytes(r.w0, r.w1, z, s);
    else
        return unit8<NBITS>(unit_merge<NBITS>(r), z, s);
}

template <int NBITS, bool SMALL>
__device__ __forceinline__ uint32_t unit_bits(const uint8_t* __restrict__ packed, int64_t u) {
    static_assert(NBITS != 8, "8-bit units are 64 bits: use unit_fetch and unit8_raw");
    if constexpr (NBITS == 1) {
        return __ldg(packed + u);
    } else if constexpr (NBITS == 4) {
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

// A quad: 4 consecutive units (32 codes) of one row, the work item of the
// linear-layer kernels.  Its codes are one vector load (VEC, when rows start
// on a quad: 4, 8, 16 or 32 bytes at 1, 2, 4 or 8 bits; four 32-bit words at
// 3 bits) and its group data one (scale, zero) pair (two for groups of 16).
template <int NBITS>
struct QuadCodes {
    static constexpr int NW = NBITS == 3 ? 4 : NBITS;     // 32-bit words of codes
    uint32_t w[NW];
    __half2 sz[2];                                     // (s, z) of units 0-1 and 2-3
    uint32_t off;                                      // 3 bits: slot of code 0 in w[0]
    uint32_t present;                                  // bit t: unit t inside the matrix
                                                       // (absent units decode to 0)
};

// (s, z) of group g: the stored fp16 values, or restored from their 8-bit
// form when the layer was given one (a launch-uniform branch).
__device__ __forceinline__ __half2 group_sz(const LinearParams& p, int64_t g) {
    const __half s = p.sq.codes ? restore_meta_h(p.sq, g) : __ldg(p.scale + g);
    const __half z = p.zq.codes ? restore_meta_h(p.zq, g) : __ldg(p.zero + g);
    return __halves2half2(s, z);
}

template <int NBITS, bool SMALL, bool VEC>
__device__ __forceinline__ void load_quad(const LinearParams& p, int64_t fbase, bool row_ok,
                                          int64_t kq, QuadCodes<NBITS>& c) {
    // fbase: flat index of the row's first code; kq: k of the quad's first code
    c.present = 0u;
    c.off = 0u;
#pragma unroll
    for (int i = 0; i < QuadCodes<NBITS>::NW; ++i) c.w[i] = 0u;
    c.sz[0] = c.sz[1] = __float2half2_rn(0.0f);
    if (!row_ok || kq >= p.K) return;
    const int64_t f = fbase + kq;
#pragma unroll
    for (int t = 0; t < 4; ++t)
        if (kq + 8 * t < p.K) c.present |= 1u << t;
    if constexpr (NBITS == 3) {
        const int64_t u = f >> 3;
        int64_t w0;
        if (SMALL) {
            const uint32_t u4 = 4u * (uint32_t)u;
            w0 = __umulhi(u4, 0xCCCCCCCDu) >> 2;         // floor(f / 10)
        } else {
            w0 = (4 * u) / 5;
        }
        c.off = (uint32_t)(f - 10 * w0);
        // slots off .. off + 8 * (present units) - 1 (< 40): only the words they
        // touch are read, so a partial quad at the end stays inside the buffer
        const uint32_t slots = c.off + 8u * (uint32_t)__popc(c.present);
        const uint32_t* p32 = reinterpret_cast<const uint32_t*>(p.packed) + w0;
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if (10u * i < slots) c.w[i] = __ldg(p32 + i);
    } else if constexpr (VEC) {
        const uint8_t* src = p.packed + (f >> 5) * (4 * NBITS);
        if constexpr (NBITS == 8) {
            const uint4 a = __ldg(reinterpret_cast<const uint4*>(src));
            const uint4 b = __ldg(reinterpret_cast<const uint4*>(src) + 1);
            c.w[0] = a.x; c.w[1] = a.y; c.w[2] = a.z; c.w[3] = a.w;
            c.w[4] = b.x; c.w[5] = b.y; c.w[6] = b.z; c.w[7] = b.w;
        } else if constexpr (NBITS == 4) {
            const uint4 a = __ldg(reinterpret_cast<const uint4*>(src));
            c.w[0] = a.x; c.w[1] = a.y; c.w[2] = a.z; c.w[3] = a.w;
        } else if constexpr (NBITS == 2) {
            const uint2 a = __ldg(reinterpret_cast<const uint2*>(src));
            c.w[0] = a.x; c.w[1] = a.y;
        } else {
            c.w[0] = __ldg(reinterpret_cast<const uint32_t*>(src));
        }
    } else {                                           // unit by unit (any k alignment)
        const int64_t u = f >> 3;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            if (!(c.present & (1u << t))) continue;
            const UnitRaw r = unit_fetch<NBITS, SMALL>(p.packed, u + t);
            if constexpr (NBITS == 8) {
                c.w[2 * t] = r.w0;
                c.w[2 * t + 1] = r.w1;
            } else if constexpr (NBITS == 4) {
                c.w[t] = r.w0;
            } else if constexpr (NBITS == 2) {
                c.w[t >> 1] |= r.w0 << (16 * (t & 1));
            } else {
                c.w[0] |= r.w0 << (8 * t);
            }
        }
    }
    const int64_t g = f >> p.log2_group;
    c.sz[0] = group_sz(p, g);
    c.sz[1] = c.sz[0];
    if (p.log2_group == 4 && (c.present & 4u)) c.sz[1] = group_sz(p, g + 1);
    // K is a multiple of 16: units 0-1 are both present, and so are 2-3 or
    // neither; absent units get s = z = 0, so their weights are exactly 0
    if (!(c.present & 4u)) c.sz[1] = __float2half2_rn(0.0f);
}

// Weights of unit t (0..3) of a loaded quad.
template <int NBITS>
__device__ __forceinline__ uint4 quad_unit(const QuadCodes<NBITS>& c, int t) {
    const __half2 sz = c.sz[t >> 1];
    const float s = __low2float(sz), z = __high2float(sz);
    if constexpr (NBITS == 8) {
        return unit8_bytes(c.w[2 * t], c.w[2 * t + 1], z, s);
    } else if constexpr (NBITS == 4) {
        return unit8<4>(c.w[t], z, s);
    } else if constexpr (NBITS == 2) {
        return unit8<2>((c.w[t >> 1] >> (16 * (t & 1))) & 0xFFFFu, z, s);
    } else if constexpr (NBITS == 1) {
        return unit8<1>((c.w[0] >> (8 * t)) & 0xFFu, z, s);
    } else {
        // the 30-bit fields of the four words as two 60-bit runs
        const uint64_t A = (uint64_t)c.w[0] | ((uint64_t)c.w[1] << 30);
        const uint64_t B = (uint64_t)c.w[2] | ((uint64_t)c.w[3] << 30);
        const uint32_t pos = 3u * (c.off + 8u * (uint32_t)t);   // bit of code 8t
        uint64_t v;
        if (pos + 24u <= 60u) v = A >> pos;
        else if (pos >= 60u) v = B >> (pos - 60u);
        else v = (A >> pos) | (B << (60u - pos));
        return unit8<3>((uint32_t)v & 0xFFFFFFu, z, s);
    }
}

}  // namespace hqq
