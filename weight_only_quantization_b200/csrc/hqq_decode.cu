// hqq_decode.cu -- the weight-only linear layer for few tokens (the decode
// shape: up to 16 at 3 bits, 8 otherwise; decode_max_tokens in hqq_params.cuh):
// Y[m, n] = sum_k X[m, k] * W_hat[n, k] with W_hat =
// fp16((code - z) * s) (section 2's Q^-1 of "Half-Quadratic Quantization of
// Large Machine Learning Models"), the same product as hqq_linear.cu.
//
// With so few tokens the product is bound by reading the packed weights and by
// the instructions that turn codes into fp16 weights, not by multiply-adds.  A
// warp owns 16 output features and feeds the A operand of m16n8k16 warp MMAs
// straight from registers: lane (r, j) = (lane / 4, lane % 4) decodes a run of
// S consecutive codes (inside one quantization group) of features r and r + 8
// and supplies four codes of each per MMA, in the k slots 2j, 2j+1, 2j+8, 2j+9.
// The B operand holds X in the same k order (column m = token m of an 8-token
// block; columns past M repeat the last token and are not stored), so the fp32
// accumulation runs in the tensor core and each weight costs its decode (a
// mask, then four fp32 pair operations for exact fp16 W_hat) and nothing else.
// The 4 lanes of a feature cover 4 consecutive runs (a chunk); a CTA's 8 warps
// take interleaved chunks of the same 16 features, staged through per-warp
// cp.async rings; a cluster of up to 8 CTAs splits the chunks further when the
// matrix has few features or long rows, and the partial tiles meet in shared
// memory and distributed shared memory.
#include <cooperative_groups.h>

#include "hqq_unpack.cuh"

namespace cg = cooperative_groups;

namespace hqq {

namespace {

constexpr int kDcWarps = 8;
constexpr int kDcThreads = kDcWarps * 32;
constexpr int kDcMaxSplit = 8;

// D (16x8 fp32) += A (16x16 fp16, row) * B (16x8 fp16, col).
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Codes at bits b and b + B of x as exact floats: both fields must lie in the
// 23 mantissa bits (b + 2B <= 23).
template <int B>
__device__ __forceinline__ float2 field_pair(uint32_t x, int b) {
    constexpr uint32_t M = (1u << B) - 1u;
    return codes2(x, M << b, 1.0f / (float)(1u << b), -(float)(1u << (23 - b)),
                  x, M << (b + B), 1.0f / (float)(1u << (b + B)), -(float)(1u << (23 - b - B)));
}

// A run of S codes of one feature: load(packed, f, ok) with f the flat index of
// its first code; pair(pp) = codes 2pp and 2pp + 1 as exact floats (pp a
// compile-time constant after unrolling); dq(pp, z, s) = their fp16 weights
// packed in one word.  ok == false leaves every code 0.
template <int NBITS, int S, bool VEC>
struct Run;

// 3 bits: words hold 10 codes in bits 0..29.  The run starts at slot o (even)
// of word w0; re-based word i holds slots o + 10i .. o + 10i + 9 in bits 0..29,
// one funnel shift of the 60-bit payload of words i and i + 1.
template <int S, bool VEC>
struct Run<3, S, VEC> {
    static constexpr int NR = (S + 9) / 10;
    uint32_t r[NR];
    __device__ __forceinline__ void load(const uint8_t* __restrict__ packed, int64_t f, bool ok) {
        const int64_t w0 = f / 10;
        const uint32_t o = (uint32_t)(f - 10 * w0);
        const uint32_t* src = reinterpret_cast<const uint32_t*>(packed) + w0;
        uint32_t p[NR + 1];
#pragma unroll
        for (int i = 0; i <= NR; ++i)                  // only words holding slots o .. o+S-1
            p[i] = (ok && 10u * i < o + S) ? __ldg(src + i) : 0u;
#pragma unroll
        for (int i = 0; i < NR; ++i) r[i] = __funnelshift_r(p[i] << 2, p[i + 1], 2u + 3u * o);
    }
    // from a staged copy: words at w[0..NR], the run starting at slot o of w[0]
    __device__ __forceinline__ void read(const uint32_t* w, uint32_t o) {
        uint32_t p[NR + 1];
#pragma unroll
        for (int i = 0; i <= NR; ++i) p[i] = w[i];
#pragma unroll
        for (int i = 0; i < NR; ++i) r[i] = __funnelshift_r(p[i] << 2, p[i + 1], 2u + 3u * o);
    }
    // Constants the caller sets once per kernel, opaque to the compiler so that
    // they stay in registers: the bits of 2^23 (one logic operation per code,
    // (field & mask) | magic, with the mask as the immediate) and the
    // multipliers 2^20 and 2^8 (a right shift by 12 or 24 as a multiply-high,
    // kept off the logic pipe).
    uint32_t mg, k20, k8;
    // codes at bits b, b + 3 of x (b = 0, or 6 when B6) as exact floats
    template <int B6>
    __device__ __forceinline__ float2 pair3(uint32_t x) const {
        constexpr uint32_t m0 = 7u << (B6 ? 6 : 0), m1 = m0 << 3;
        uint32_t f0, f1;
        asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(f0) : "r"(x), "n"(m0), "r"(mg));
        asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(f1) : "r"(x), "n"(m1), "r"(mg));
        constexpr float i0 = B6 ? 1.0f / 64 : 1.0f, i1 = B6 ? 1.0f / 512 : 1.0f / 8;
        constexpr float o0 = B6 ? -131072.0f : -8388608.0f, o1 = B6 ? -16384.0f : -1048576.0f;
        return __ffma2_rn(make_float2(__uint_as_float(f0), __uint_as_float(f1)), make_float2(i0, i1),
                          make_float2(o0, o1));
    }
    // slots 0-1, 2-3 from x; 4-5, 6-7 from x >> 12; 8-9 from x >> 24: two
    // constant sets for the five pairs of a word
    __device__ __forceinline__ float2 pair(int pp) const {
        const int m = 2 * pp, sl = m % 10;
        const uint32_t x = r[m / 10];
        if (sl == 0) return pair3<0>(x);
        if (sl == 2) return pair3<1>(x);
        if (sl == 4) return pair3<0>(__umulhi(x, k20));
        if (sl == 6) return pair3<1>(__umulhi(x, k20));
        return pair3<0>(__umulhi(x, k8));
    }
    __device__ __forceinline__ uint32_t dq(int pp, float z, float s) const { return dq2(pair(pp), z, s); }
};

template <int S, bool VEC>
struct Run<4, S, VEC> {
    static constexpr int NW = S / 8;
    uint32_t w[NW];
    __device__ __forceinline__ void load(const uint8_t* __restrict__ packed, int64_t f, bool ok) {
        const uint32_t* src = reinterpret_cast<const uint32_t*>(packed) + (f >> 3);
        if constexpr (VEC) {                           // f % 16 == 0: 8-byte aligned pairs
#pragma unroll
            for (int i = 0; i < NW; i += 2) {
                const uint2 v = ok ? __ldg(reinterpret_cast<const uint2*>(src + i)) : make_uint2(0u, 0u);
                w[i] = v.x;
                w[i + 1] = v.y;
            }
        } else {
#pragma unroll
            for (int i = 0; i < NW; ++i) w[i] = ok ? __ldg(src + i) : 0u;
        }
    }
    __device__ __forceinline__ void read(const uint32_t* src, uint32_t) {   // src 8-byte aligned
#pragma unroll
        for (int i = 0; i < NW; i += 2) {
            const uint2 v = *reinterpret_cast<const uint2*>(src + i);
            w[i] = v.x;
            w[i + 1] = v.y;
        }
    }
    __device__ __forceinline__ float2 pair(int pp) const {
        const int m = 2 * pp, sl = m % 8;
        return sl < 4 ? field_pair<4>(w[m / 8], 4 * sl) : field_pair<4>(w[m / 8] >> 16, 4 * sl - 16);
    }
    // Two codes per mask: nibbles i and i + 4 of a word sit 16 bits apart, so
    // (x & 0x000F000F) | 0x64006400 is the half2 (1024 + c_i, 1024 + c_i+4);
    // an exact fp16 subtraction (or, for the odd nibbles shifted by 4, an
    // exact fp16 fma by 1/16 and -64) leaves the codes, and one mixed-precision
    // add per code gives fl32(c - z) from the fp16 code and the fp32 -z, the
    // same value as the f32 path; the product by s and the fp16 pack follow.
    __device__ __forceinline__ uint32_t dq(int pp, float z, float s) const { return dq2(pair(pp), z, s); }
    // (measured faster for one token only; chosen at launch)
    __device__ __forceinline__ uint32_t dq_mx(int pp, float z, float s) const {
        const int m = 2 * pp, sl = m % 8;
        const uint32_t x = (sl & 2) ? (w[m / 8] >> 8) : w[m / 8];   // nibbles 2,3,6,7 shifted down
        const uint32_t lo = (x & 0x000F000Fu) | 0x64006400u;          // codes i, i + 4 (i even)
        const uint32_t hi = (x & 0x00F000F0u) | 0x64006400u;          // codes i + 1, i + 5, times 16
        const __half2 e0 = __hsub2(*reinterpret_cast<const __half2*>(&lo), __float2half2_rn(1024.0f));
        const __half2 e1 = __hfma2(*reinterpret_cast<const __half2*>(&hi), __float2half2_rn(0.0625f),
                                   __float2half2_rn(-64.0f));
        const bool up = sl >= 4;                                     // codes 4..7: high halves
        const __half c0 = up ? __high2half(e0) : __low2half(e0);
        const __half c1 = up ? __high2half(e1) : __low2half(e1);
        float d0, d1;
        asm("add.rn.f32.f16 %0, %1, %2;" : "=f"(d0) : "h"(__half_as_ushort(c0)), "f"(-z));
        asm("add.rn.f32.f16 %0, %1, %2;" : "=f"(d1) : "h"(__half_as_ushort(c1)), "f"(-z));
        const float2 v = __fmul2_rn(make_float2(d0, d1), make_float2(s, s));
        const __half2 h = __floats2half2_rn(v.x, v.y);
        return *reinterpret_cast<const uint32_t*>(&h);
    }
};

template <int S, bool VEC>
struct Run<2, S, VEC> {
    static constexpr int NW = S / 16;
    uint32_t w[NW];
    __device__ __forceinline__ void load(const uint8_t* __restrict__ packed, int64_t f, bool ok) {
        const uint32_t* src = reinterpret_cast<const uint32_t*>(packed) + (f >> 4);
#pragma unroll
        for (int i = 0; i < NW; ++i) w[i] = ok ? __ldg(src + i) : 0u;
    }
    __device__ __forceinline__ void read(const uint32_t* src, uint32_t) {
#pragma unroll
        for (int i = 0; i < NW; ++i) w[i] = src[i];
    }
    __device__ __forceinline__ float2 pair(int pp) const {
        const int m = 2 * pp, sl = m % 16;
        return sl < 10 ? field_pair<2>(w[m / 16], 2 * sl)
                       : field_pair<2>(w[m / 16] >> 12, 2 * sl - 12);
    }
    __device__ __forceinline__ uint32_t dq(int pp, float z, float s) const { return dq2(pair(pp), z, s); }
};

// 1 bit: a row starts on a 16-code boundary, so the run loads as 16-bit halves.
template <int S, bool VEC>
struct Run<1, S, VEC> {
    static constexpr int NH = S / 16;
    uint32_t h[NH];
    __device__ __forceinline__ void load(const uint8_t* __restrict__ packed, int64_t f, bool ok) {
        const uint16_t* src = reinterpret_cast<const uint16_t*>(packed) + (f >> 4);
#pragma unroll
        for (int i = 0; i < NH; ++i) h[i] = ok ? (uint32_t)__ldg(src + i) : 0u;
    }
    __device__ __forceinline__ void read(const uint16_t* src, uint32_t) {
#pragma unroll
        for (int i = 0; i < NH; ++i) h[i] = src[i];
    }
    __device__ __forceinline__ float2 pair(int pp) const {
        const int m = 2 * pp;
        return field_pair<1>(h[m / 16], m % 16);
    }
    __device__ __forceinline__ uint32_t dq(int pp, float z, float s) const { return dq2(pair(pp), z, s); }
};

// 8 bits: byte i becomes the mantissa of 2^23 by one byte permute.
template <int S, bool VEC>
struct Run<8, S, VEC> {
    static constexpr int NW = S / 4;
    uint32_t w[NW];
    __device__ __forceinline__ void load(const uint8_t* __restrict__ packed, int64_t f, bool ok) {
        const uint2* src = reinterpret_cast<const uint2*>(packed + f);
#pragma unroll
        for (int i = 0; i < NW; i += 2) {
            const uint2 v = ok ? __ldg(src + i / 2) : make_uint2(0u, 0u);
            w[i] = v.x;
            w[i + 1] = v.y;
        }
    }
    __device__ __forceinline__ void read(const uint32_t* src, uint32_t) {   // src 16-byte aligned
#pragma unroll
        for (int i = 0; i < NW; i += 4) {
            const uint4 v = *reinterpret_cast<const uint4*>(src + i);
            w[i] = v.x;
            w[i + 1] = v.y;
            w[i + 2] = v.z;
            w[i + 3] = v.w;
        }
    }
    __device__ __forceinline__ float2 pair(int pp) const {
        const int m = 2 * pp, b = m % 4;
        const uint32_t x = w[m / 4];
        const float2 f = make_float2(__uint_as_float(__byte_perm(x, 0x4B000000u, (uint32_t)b | 0x7440u)),
                                     __uint_as_float(__byte_perm(x, 0x4B000000u, (uint32_t)(b + 1) | 0x7440u)));
        return __fadd2_rn(f, make_float2(-8388608.0f, -8388608.0f));
    }
    __device__ __forceinline__ uint32_t dq(int pp, float z, float s) const { return dq2(pair(pp), z, s); }
};

// Staging geometry of one chunk (4 runs = 4S codes) of one feature: its bytes
// lie in GR 16-byte granules from granule g of the packed buffer (3 bits: up to
// one word past the last code, read but unused by the re-basing); a warp's
// stage holds the chunk of its 16 features, RS words apart (RS % 32 != 0, so
// the 8 features of one load fall into different banks).
template <int NBITS, int S>
struct Geo {
    static constexpr int BYTES = NBITS == 3 ? 4 * ((4 * S + 9) / 10 + 1) : 4 * S * NBITS / 8;
    static constexpr int GR = (BYTES + 16 + 15) / 16;
    static constexpr int RS = GR % 2 == 0 ? 4 * GR + 4 : 4 * GR;
    static constexpr int STAGE = 16 * RS + 8;             // words
    static constexpr int GPL = (GR + 3) / 4;              // granules per lane and feature
};

constexpr int kDcStages = 3;

// Dynamic shared memory: the warps' rings (staged), reused after the main loop
// for the warps' partial tiles and the cluster's.
template <int NBITS, int S, bool STAGED, int NT>
constexpr size_t decode_smem() {
    const size_t ring = STAGED ? (size_t)kDcWarps * kDcStages * Geo<NBITS, S>::STAGE * 4 : 0;
    const size_t red = (size_t)(kDcWarps * 4 * NT * 32 + (kDcMaxSplit - 1) * 128 * NT) * 4;
    return ring > red ? ring : red;
}

// Where the chunk at k = kc of feature n starts: granule g and, for run j of
// the lane, the offset of its first word (16-bit half at 1 bit) from granule g
// and its first code's slot (3 bits).  b0 / b1: per-feature constants (3 bits:
// n*K = 10 b0 + b1; otherwise the word, or half, index of n*K).
template <int NBITS, int S>
struct Loc {
    int64_t g;
    uint32_t off, o;
    __device__ __forceinline__ Loc(int64_t b0, uint32_t b1, uint32_t kc, int j) {
        if constexpr (NBITS == 3) {
            const uint32_t t = b1 + kc, tj = t + (uint32_t)(S * j);
            const uint32_t qa = t / 10u, qj = tj / 10u;
            const int64_t wa = b0 + qa;
            g = wa >> 2;
            off = (uint32_t)(wa & 3) + (qj - qa);
            o = tj - 10u * qj;
        } else if constexpr (NBITS == 1) {
            const int64_t ha = b0 + (kc >> 4);
            g = ha >> 3;
            off = (uint32_t)(ha & 7) + (uint32_t)(j * S / 16);
            o = 0;
        } else {
            const int64_t wa = b0 + (kc * NBITS >> 5);
            g = wa >> 2;
            off = (uint32_t)(wa & 3) + (uint32_t)(j * S * NBITS / 32);
            o = 0;
        }
    }
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// S/4 MMAs per 8-token block of one chunk: codes 4i..4i+3 of the lane's runs of
// features r and r + 8 against X[m, k + 4i .. k + 4i + 3]; xo[c] = row offset
// of token 8c + r in X (the last token for rows past M).
template <int NBITS, int S, bool VEC, int NT, bool MX, typename XF>
__device__ __forceinline__ void chunk_mma_x(float (&acc)[NT][4], const Run<NBITS, S, VEC>& a,
                                            const Run<NBITS, S, VEC>& b, __half2 sz0, __half2 sz1,
                                            XF xfrag) {
    const float s0 = __low2float(sz0), z0 = __high2float(sz0);
    const float s1 = __low2float(sz1), z1 = __high2float(sz1);
    auto dq = [&](const Run<NBITS, S, VEC>& run, int pp, float z, float s) {
        if constexpr (MX) return run.dq_mx(pp, z, s);
        else return run.dq(pp, z, s);
    };
#pragma unroll
    for (int i = 0; i < S / 4; i += 2) {
        const uint32_t a0 = dq(a, 2 * i, z0, s0), a1 = dq(b, 2 * i, z1, s1);
        const uint32_t a2 = dq(a, 2 * i + 1, z0, s0), a3 = dq(b, 2 * i + 1, z1, s1);
        const uint32_t a4 = dq(a, 2 * i + 2, z0, s0), a5 = dq(b, 2 * i + 2, z1, s1);
        const uint32_t a6 = dq(a, 2 * i + 3, z0, s0), a7 = dq(b, 2 * i + 3, z1, s1);
#pragma unroll
        for (int c = 0; c < NT; ++c) {
            const uint4 x = xfrag(c, i / 2);
            mma16816(acc[c], a0, a1, a2, a3, x.x, x.y);
            mma16816(acc[c], a4, a5, a6, a7, x.z, x.w);
        }
    }
}

// X fragments straight from global memory: eight halves of token row xo[c]
// from k + 8 u.
template <int NBITS, int S, bool VEC, int NT, bool MX>
__device__ __forceinline__ void chunk_mma(float (&acc)[NT][4], const Run<NBITS, S, VEC>& a,
                                          const Run<NBITS, S, VEC>& b, __half2 sz0, __half2 sz1,
                                          const __half* __restrict__ X, const int64_t (&xo)[NT],
                                          int64_t k) {
    chunk_mma_x<NBITS, S, VEC, NT, MX>(acc, a, b, sz0, sz1, [&](int c, int u) {
        return __ldg(reinterpret_cast<const uint4*>(X + xo[c] + k) + u);
    });
}

// Grid: ceil(N / 16) feature tiles x `split` CTAs (a (split, 1, 1) cluster when
// split > 1; rank = blockIdx.x % split).  Chunk ch = 4 runs of S codes; CTA
// rank c, warp w takes chunks c * 8 + w, then every 8 * split.  NT (1 or 2)
// blocks of 8 tokens share every decoded weight.
// STAGED (packed 16-byte aligned, K < 2^30): each warp copies its chunks'
// granules into a kDcStages-deep ring of its own with cp.async (lane (r, j)
// copies granules j, j+4, .. of features r and r + 8; past the buffer's end
// the copy is zero-filled), so two chunks are in flight while one is decoded;
// otherwise the lanes load their runs from global memory directly.
template <int NBITS, int S, bool VEC, bool STAGED, int NT, bool MX>
__global__ void __launch_bounds__(kDcThreads, NT == 2 ? 2 : NBITS == 3 ? 4 : 3)
decode_kernel(const __half* __restrict__ X, const __grid_constant__ LinearParams p, int split,
              int64_t packed_bytes) {
    extern __shared__ __align__(16) uint32_t dc_smem[];
    using G = Geo<NBITS, S>;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = lane >> 2, j = lane & 3;
    const int rank = (int)(blockIdx.x % (unsigned)split);
    const int64_t tile = blockIdx.x / (unsigned)split;

    uint32_t mg = 0x4B000000u, k20 = 1u << 20, k8 = 1u << 8;
    asm volatile("" : "+r"(mg), "+r"(k20), "+r"(k8));
    const int64_t n0 = tile * 16 + r, n1 = n0 + 8;
    const bool ok0 = n0 < p.N, ok1 = n1 < p.N;
    const int64_t runs = p.K / S;                         // runs per feature
    const int64_t nchunk = (runs + 3) >> 2;
    const int64_t step = (int64_t)split * kDcWarps;
    int64_t xo[NT];
#pragma unroll
    for (int c = 0; c < NT; ++c) xo[c] = (8 * c + r < p.M ? (int64_t)(8 * c + r) : p.M - 1) * p.K;
    float acc[NT][4];
#pragma unroll
    for (int c = 0; c < NT; ++c) acc[c][0] = acc[c][1] = acc[c][2] = acc[c][3] = 0.0f;
    int64_t ch = (int64_t)rank * kDcWarps + warp;
    // groups of the lane's runs: they advance by a whole number of groups per step
    const int64_t gstep = (4 * S * step) >> p.log2_group;
    int64_t g0 = (n0 * p.K + (4 * ch + j) * S) >> p.log2_group;
    int64_t g1 = g0 + ((8 * p.K) >> p.log2_group);
    auto group_of = [&](int64_t c, int64_t g, bool ok) {
        return (ok && 4 * c + j < runs) ? group_sz(p, g) : __float2half2_rn(0.0f);
    };

    if constexpr (STAGED) {
        uint32_t* ring = dc_smem + (size_t)warp * kDcStages * G::STAGE;
        const uint32_t ring_s = (uint32_t)__cvta_generic_to_shared(ring);
        // per-feature constants of the chunk locations
        int64_t b00, b10;
        uint32_t b01 = 0, b11 = 0;
        if constexpr (NBITS == 3) {
            b00 = n0 * p.K / 10;
            b01 = (uint32_t)(n0 * p.K - 10 * b00);
            b10 = n1 * p.K / 10;
            b11 = (uint32_t)(n1 * p.K - 10 * b10);
        } else if constexpr (NBITS == 1) {
            b00 = n0 * p.K >> 4;
            b10 = n1 * p.K >> 4;
        } else {
            b00 = n0 * p.K * NBITS >> 5;
            b10 = n1 * p.K * NBITS >> 5;
        }
        // copy the chunk's granules of features r and r + 8: whole 16-byte
        // copies while a feature's slot lies inside the buffer, else clamped
        // (zero-filled) ones
        auto fill = [&](int64_t c, int stage) {
            if (c < nchunk) {
                const uint32_t kc = (uint32_t)(4 * S * c);
                const Loc<NBITS, S> l0(b00, b01, kc, 0), l1(b10, b11, kc, 0);
                const uint32_t d0 = ring_s + 4u * (uint32_t)(stage * G::STAGE + r * G::RS) + 16u * j;
                const uint32_t d1 = d0 + 4u * 8u * G::RS;
                const uint8_t* src0 = p.packed + 16 * (l0.g + j);
                const uint8_t* src1 = p.packed + 16 * (l1.g + j);
                // (feature r + 8 valid and inside the buffer: so is feature r)
                if (ok1 && 16 * (l1.g + G::GR) <= packed_bytes) {
#pragma unroll
                    for (int t = 0; t < G::GPL; ++t)
                        if (j + 4 * t < G::GR) {
                            cp_async16(d0 + 64u * t, src0 + 64 * t);
                            cp_async16(d1 + 64u * t, src1 + 64 * t);
                        }
                } else {
#pragma unroll
                    for (int t = 0; t < G::GPL; ++t) {
                        const int gi = j + 4 * t;
                        if (gi < G::GR) {
                            const int64_t s0 = 16 * (l0.g + gi), s1 = 16 * (l1.g + gi);
                            const int64_t r0 = ok0 ? packed_bytes - s0 : 0, r1 = ok1 ? packed_bytes - s1 : 0;
                            const uint32_t c0 = r0 <= 0 ? 0u : r0 >= 16 ? 16u : (uint32_t)r0;
                            const uint32_t c1 = r1 <= 0 ? 0u : r1 >= 16 ? 16u : (uint32_t)r1;
                            cp_async16(d0 + 64u * t, p.packed + (c0 ? s0 : 0), c0);
                            cp_async16(d1 + 64u * t, p.packed + (c1 ? s1 : 0), c1);
                        }
                    }
                }
            }
            cp_commit();
        };
#pragma unroll
        for (int s = 0; s < kDcStages - 1; ++s) fill(ch + s * step, s);
        // (s, z) of the current chunk's runs, loaded one chunk ahead
        __half2 sz0 = group_of(ch, g0, ok0), sz1 = group_of(ch, g1, ok1);
        for (int it = 0; ch < nchunk; ++it, ch += step) {
            g0 += gstep;
            g1 += gstep;
            const __half2 nz0 = group_of(ch + step, g0, ok0), nz1 = group_of(ch + step, g1, ok1);
            cp_wait<kDcStages - 2>();
            __syncwarp();
            fill(ch + (kDcStages - 1) * step, (it + kDcStages - 1) % kDcStages);
            const int stage = it % kDcStages;
            const uint32_t kc = (uint32_t)(4 * S * ch);
            const Loc<NBITS, S> l0(b00, b01, kc, j), l1(b10, b11, kc, j);
            const uint32_t* s0 = ring + stage * G::STAGE + r * G::RS;
            const uint32_t* s1 = s0 + 8 * G::RS;
            Run<NBITS, S, VEC> a, b;
            if constexpr (NBITS == 3) {
                a.mg = b.mg = mg;
                a.k20 = b.k20 = k20;
                a.k8 = b.k8 = k8;
            }
            if constexpr (NBITS == 1) {
                a.read(reinterpret_cast<const uint16_t*>(s0) + l0.off, 0u);
                b.read(reinterpret_cast<const uint16_t*>(s1) + l1.off, 0u);
            } else {
                a.read(s0 + l0.off, l0.o);
                b.read(s1 + l1.off, l1.o);
            }
            const int64_t q = 4 * ch + j;
            chunk_mma<NBITS, S, VEC, NT, MX>(acc, a, b, sz0, sz1, X, xo, q < runs ? q * S : 0);
            sz0 = nz0;
            sz1 = nz1;
        }
        cp_wait<0>();
    } else {
        for (; ch < nchunk; ch += step, g0 += gstep, g1 += gstep) {
            const int64_t q = 4 * ch + j;
            const bool qok = q < runs;
            const int64_t k = qok ? q * S : 0;
            const bool v0 = ok0 && qok, v1 = ok1 && qok;
            const int64_t f0 = n0 * p.K + k, f1 = f0 + 8 * p.K;
            Run<NBITS, S, VEC> a, b;
            if constexpr (NBITS == 3) {
                a.mg = b.mg = mg;
                a.k20 = b.k20 = k20;
                a.k8 = b.k8 = k8;
            }
            a.load(p.packed, f0, v0);
            b.load(p.packed, f1, v1);
            chunk_mma<NBITS, S, VEC, NT, MX>(acc, a, b, group_of(ch, g0, ok0), group_of(ch, g1, ok1),
                                             X, xo, k);
        }
    }

    // the warps' tiles, then the cluster's (in the then idle ring memory):
    // element e of block c in lane l is feature tile*16 + l/4 + 8*(e/2), token
    // 8c + 2*(l%4) + e%2
    constexpr int TW = 4 * NT * 32;                       // floats per warp
    float* red = reinterpret_cast<float*>(dc_smem);
    float* cred = red + kDcWarps * TW;
    __syncthreads();
#pragma unroll
    for (int c = 0; c < NT; ++c)
#pragma unroll
        for (int e = 0; e < 4; ++e) red[warp * TW + (4 * c + e) * 32 + lane] = acc[c][e];
    __syncthreads();
    const int t = threadIdx.x;
    float v[TW / kDcThreads + 1];
#pragma unroll
    for (int u = 0; u * kDcThreads < TW; ++u) {
        v[u] = 0.0f;
        if (u * kDcThreads + t < TW)
#pragma unroll
            for (int w = 0; w < kDcWarps; ++w) v[u] += red[w * TW + u * kDcThreads + t];
    }
    if (split > 1) {
        // every CTA of the cluster is past its main loop: rank 0's memory is free
        asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
                     "barrier.cluster.wait.acquire.aligned;" ::: "memory");
        if (rank != 0) {
            float* dst = cg::this_cluster().map_shared_rank(cred, 0) + (rank - 1) * TW;
#pragma unroll
            for (int u = 0; u * kDcThreads < TW; ++u)
                if (u * kDcThreads + t < TW) dst[u * kDcThreads + t] = v[u];
        }
        asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
                     "barrier.cluster.wait.acquire.aligned;" ::: "memory");
        if (rank == 0)
#pragma unroll
            for (int u = 0; u * kDcThreads < TW; ++u)
                if (u * kDcThreads + t < TW)
                    for (int c = 1; c < split; ++c) v[u] += cred[(c - 1) * TW + u * kDcThreads + t];
    }
    if (rank == 0) {
#pragma unroll
        for (int u = 0; u * kDcThreads < TW; ++u) {
            const int i = u * kDcThreads + t;
            if (i < TW) {
                const int c = i >> 7, e = (i >> 5) & 3, l = i & 31;
                const int64_t n = tile * 16 + (l >> 2) + 8 * (e >> 1);
                const int64_t m = 8 * c + 2 * (l & 3) + (e & 1);
                if (n < p.N && m < p.M) p.Y[m * p.N + n] = __float2half_rn(v[u]);
            }
        }
    }
}

// Halves per run row of the shared X stage (a run's S values + 8 of padding,
// so that the eight lanes of each quarter-warp read distinct banks) and per
// stage (16 token rows x 4 runs).
template <int S, int NT>
struct XGeo {
    static constexpr int XR = S + 8;
    static constexpr int STAGE = 8 * NT * 4 * XR;
};

template <int NBITS, int S, int NT>
constexpr size_t decode_sx_smem() {
    const size_t ring = (size_t)kDcWarps * kDcStages * Geo<NBITS, S>::STAGE * 4 +
                        (size_t)kDcStages * XGeo<S, NT>::STAGE * 2;
    const size_t red = (size_t)(kDcMaxSplit - 1) * kDcWarps * 4 * NT * 32 * 4;
    return ring > red ? ring : red;
}

// NT 8-token blocks (2 to 16 tokens): the 8 warps of a CTA own 8 consecutive
// 16-feature tiles and walk the same chunks, so one copy of X per chunk (8 NT
// token rows x 4S columns, zero past M and past K) serves them all: the CTA's
// threads stage it with cp.async next to each warp's code ring, and a CTA
// barrier per chunk publishes it.  Grid: ceil(N / 128) CTA tiles x `split`
// (a (split, 1, 1) cluster when split > 1; rank = blockIdx.x % split takes
// chunks rank, rank + split, ..); partial tiles meet in rank 0's shared memory.
// Needs X 16-byte aligned and K < 2^30.  STAGED (packed 16-byte aligned): each
// warp's codes come through its cp.async ring as in decode_kernel; otherwise
// the lanes load their runs from global memory (same products, same order).
template <int NBITS, int S, int NT, bool STAGED>
__global__ void __launch_bounds__(kDcThreads, NT == 2 ? 2 : 3)
decode_sx_kernel(const __half* __restrict__ X, const __grid_constant__ LinearParams p, int split,
                 int64_t packed_bytes) {
    extern __shared__ __align__(16) uint32_t dc_smem[];
    using G = Geo<NBITS, S>;
    using XG = XGeo<S, NT>;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = lane >> 2, j = lane & 3;
    const int rank = (int)(blockIdx.x % (unsigned)split);
    const int64_t tile = (int64_t)(blockIdx.x / (unsigned)split) * kDcWarps + warp;
    uint32_t mg = 0x4B000000u, k20 = 1u << 20, k8 = 1u << 8;
    asm volatile("" : "+r"(mg), "+r"(k20), "+r"(k8));

    const int64_t n0 = tile * 16 + r, n1 = n0 + 8;
    const bool ok0 = n0 < p.N, ok1 = n1 < p.N;
    const int64_t runs = p.K / S;
    const int64_t nchunk = (runs + 3) >> 2;
    float acc[NT][4];
#pragma unroll
    for (int c = 0; c < NT; ++c) acc[c][0] = acc[c][1] = acc[c][2] = acc[c][3] = 0.0f;
    int64_t ch = rank;
    const int64_t gstep = (4 * S * (int64_t)split) >> p.log2_group;
    int64_t g0 = (n0 * p.K + (4 * ch + j) * S) >> p.log2_group;
    int64_t g1 = g0 + ((8 * p.K) >> p.log2_group);
    auto group_of = [&](int64_t c, int64_t g, bool ok) {
        return (ok && c < nchunk && 4 * c + j < runs) ? group_sz(p, g) : __float2half2_rn(0.0f);
    };

    uint32_t* ring = dc_smem + (size_t)warp * kDcStages * G::STAGE;
    const uint32_t ring_s = (uint32_t)__cvta_generic_to_shared(ring);
    const __half* xring = reinterpret_cast<const __half*>(dc_smem + (size_t)kDcWarps * kDcStages * G::STAGE);
    const uint32_t xring_s = (uint32_t)__cvta_generic_to_shared(xring);
    const int64_t b00 = NBITS == 3 ? n0 * p.K / 10 : n0 * p.K * NBITS >> 5;
    const int64_t b10 = NBITS == 3 ? n1 * p.K / 10 : n1 * p.K * NBITS >> 5;
    const uint32_t b01 = NBITS == 3 ? (uint32_t)(n0 * p.K - 10 * b00) : 0u;
    const uint32_t b11 = NBITS == 3 ? (uint32_t)(n1 * p.K - 10 * b10) : 0u;
    // this warp's code granules of chunk c (as in decode_kernel), and this
    // thread's share of the chunk's X granules: granule q of the stage is
    // token m = q / (S / 2), run jj, 16-byte piece u of that run
    auto fill = [&](int64_t c, int stage) {
        if (c < nchunk) {
            const uint32_t kc = (uint32_t)(4 * S * c);
            const Loc<NBITS, S> l0(b00, b01, kc, 0), l1(b10, b11, kc, 0);
            if constexpr (STAGED) {
            const uint32_t d0 = ring_s + 4u * (uint32_t)(stage * G::STAGE + r * G::RS) + 16u * j;
            const uint32_t d1 = d0 + 4u * 8u * G::RS;
#pragma unroll
            for (int t = 0; t < G::GPL; ++t) {
                const int gi = j + 4 * t;
                if (gi < G::GR) {
                    const int64_t s0 = 16 * (l0.g + gi), s1 = 16 * (l1.g + gi);
                    const int64_t r0 = ok0 ? packed_bytes - s0 : 0, r1 = ok1 ? packed_bytes - s1 : 0;
                    const uint32_t c0 = r0 <= 0 ? 0u : r0 >= 16 ? 16u : (uint32_t)r0;
                    const uint32_t c1 = r1 <= 0 ? 0u : r1 >= 16 ? 16u : (uint32_t)r1;
                    cp_async16(d0 + 64u * t, p.packed + (c0 ? s0 : 0), c0);
                    cp_async16(d1 + 64u * t, p.packed + (c1 ? s1 : 0), c1);
                }
            }
            }
            constexpr int XQ = 8 * NT * 4 * S / 8;           // 16-byte granules per X stage
            for (int q = threadIdx.x; q < XQ; q += kDcThreads) {
                const int m = q / (S / 2), o = q % (S / 2), jj = o / (S / 8), u = o % (S / 8);
                const int64_t k = 4 * S * c + (int64_t)jj * S + 8 * u;
                const bool in = m < p.M && k < p.K;
                cp_async16(xring_s + 2u * (uint32_t)(stage * XG::STAGE + (m * 4 + jj) * XG::XR + 8 * u),
                           in ? X + m * p.K + k : X, in ? 16u : 0u);
            }
        }
        cp_commit();
    };
#pragma unroll
    for (int st = 0; st < kDcStages - 1; ++st) fill(ch + st * (int64_t)split, st);
    __half2 sz0 = group_of(ch, g0, ok0), sz1 = group_of(ch, g1, ok1);
    for (int it = 0; ch < nchunk; ++it, ch += split) {
        g0 += gstep;
        g1 += gstep;
        const __half2 nz0 = group_of(ch + split, g0, ok0), nz1 = group_of(ch + split, g1, ok1);
        cp_wait<kDcStages - 2>();
        __syncthreads();                       // every thread's copies of this chunk landed
        fill(ch + (kDcStages - 1) * (int64_t)split, (it + kDcStages - 1) % kDcStages);
        const int stage = it % kDcStages;
        Run<NBITS, S, false> a, b;
        if constexpr (NBITS == 3) {
            a.mg = b.mg = mg;
            a.k20 = b.k20 = k20;
            a.k8 = b.k8 = k8;
        }
        if constexpr (STAGED) {
            const uint32_t kc = (uint32_t)(4 * S * ch);
            const Loc<NBITS, S> l0(b00, b01, kc, j), l1(b10, b11, kc, j);
            const uint32_t* s0 = ring + stage * G::STAGE + r * G::RS;
            const uint32_t* s1 = s0 + 8 * G::RS;
            a.read(s0 + l0.off, l0.o);
            b.read(s1 + l1.off, l1.o);
        } else {
            const int64_t q = 4 * ch + j;
            const bool qok = q < runs;
            const int64_t f0 = n0 * p.K + (qok ? q * S : 0), f1 = f0 + 8 * p.K;
            a.load(p.packed, f0, ok0 && qok);
            b.load(p.packed, f1, ok1 && qok);
        }
        const __half* xs = xring + stage * XG::STAGE + j * XG::XR;
        chunk_mma_x<NBITS, S, false, NT, false>(acc, a, b, sz0, sz1, [&](int c, int u) {
            return *reinterpret_cast<const uint4*>(xs + (8 * c + r) * 4 * XG::XR + 8 * u);
        });
        sz0 = nz0;
        sz1 = nz1;
    }
    cp_wait<0>();
    __syncthreads();

    // element e of block c in lane l: feature tile*16 + l/4 + 8*(e/2), token
    // 8c + 2*(l%4) + e%2
    constexpr int TW = 4 * NT * 32;                       // floats per warp
    float* cred = reinterpret_cast<float*>(dc_smem);
    if (split > 1) {
        // every CTA of the cluster is past its main loop: rank 0's memory is free
        asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
                     "barrier.cluster.wait.acquire.aligned;" ::: "memory");
        if (rank != 0) {
            float* dst = cg::this_cluster().map_shared_rank(cred, 0) + ((rank - 1) * kDcWarps + warp) * TW;
#pragma unroll
            for (int c = 0; c < NT; ++c)
#pragma unroll
                for (int e = 0; e < 4; ++e) dst[(4 * c + e) * 32 + lane] = acc[c][e];
        }
        asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
                     "barrier.cluster.wait.acquire.aligned;" ::: "memory");
        if (rank == 0)
            for (int q = 1; q < split; ++q)
#pragma unroll
                for (int c = 0; c < NT; ++c)
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        acc[c][e] += cred[((q - 1) * kDcWarps + warp) * TW + (4 * c + e) * 32 + lane];
    }
    if (rank == 0) {
#pragma unroll
        for (int c = 0; c < NT; ++c)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int64_t n = tile * 16 + r + 8 * (e >> 1);
                const int64_t m = 8 * c + 2 * j + (e & 1);
                if (n < p.N && m < p.M) p.Y[m * p.N + n] = __float2half_rn(acc[c][e]);
            }
    }
}

template <int NBITS, int S, int NT, bool STAGED>
cudaError_t launch_sx(const LinearParams& p, const void* X, int64_t packed_bytes, cudaStream_t stream) {
    auto kern = decode_sx_kernel<NBITS, S, NT, STAGED>;
    constexpr size_t smem = decode_sx_smem<NBITS, S, NT>();
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // split the chunks over a cluster while the grid is short of two CTAs per
    // SM and every CTA keeps at least two chunks
    const int64_t ctiles = (p.N + 16 * kDcWarps - 1) / (16 * kDcWarps);
    const int64_t nchunk = (p.K / S + 3) / 4;
    int split = 1;
    while (split < kDcMaxSplit && ctiles * split < 2 * sms && nchunk >= 4 * split) split *= 2;
    const __half* xp = static_cast<const __half*>(X);
    if (split == 1) {
        kern<<<(unsigned)ctiles, kDcThreads, smem, stream>>>(xp, p, 1, packed_bytes);
        return cudaGetLastError();
    }
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = (unsigned)split;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.gridDim = dim3((unsigned)(ctiles * split));
    cfg.blockDim = dim3(kDcThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, xp, p, split, packed_bytes);
}

template <int NBITS, int S, bool VEC, bool STAGED, int NT, bool MX>
cudaError_t launch_s(const LinearParams& p, const void* X, int64_t packed_bytes,
                     cudaStream_t stream) {
    auto kern = decode_kernel<NBITS, S, VEC, STAGED, NT, MX>;
    constexpr size_t smem = decode_smem<NBITS, S, STAGED, NT>();
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // split the chunks of a tile over a cluster while the grid is short of two
    // CTAs per SM (measured: finer splits for wave balance cost more than they
    // gain, as each warp then sees too few chunks to fill its copy ring)
    const int64_t tiles = (p.N + 15) / 16;
    const int64_t nchunk = (p.K / S + 3) / 4;
    int split = 1;
    while (split < kDcMaxSplit && tiles * split < 2 * sms && nchunk >= 2 * split * kDcWarps)
        split *= 2;
    // long rows: halve the chunks per CTA while each warp keeps >= 6 of them
    // and the tiles fill the last round of resident CTAs badly
    int per_sm = 1;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kDcThreads, smem);
    const int64_t slots = (int64_t)sms * (per_sm > 0 ? per_sm : 1);
    auto fill_frac = [&](int64_t units) {
        return (double)units / (double)(((units + slots - 1) / slots) * slots);
    };
    while (split < kDcMaxSplit && nchunk >= (int64_t)12 * split * kDcWarps &&
           fill_frac(tiles * split * 2) > fill_frac(tiles * split) + 0.1)
        split *= 2;
    const __half* xp = static_cast<const __half*>(X);
    if (split == 1) {
        kern<<<(unsigned)tiles, kDcThreads, smem, stream>>>(xp, p, 1, packed_bytes);
        return cudaGetLastError();
    }
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = (unsigned)split;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.gridDim = dim3((unsigned)(tiles * split));
    cfg.blockDim = dim3(kDcThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, xp, p, split, packed_bytes);
}

// S = min(group, 64) codes per run (32 at 8 bits), so a run never leaves its group.
template <int NBITS, bool VEC, bool STAGED, int NT, bool MX>
cudaError_t launch_g(const LinearParams& p, const void* X, int64_t pb, cudaStream_t stream) {
    constexpr int SMAX = NBITS == 8 ? 32 : 64;
    if (p.log2_group == 4) return launch_s<NBITS, 16, VEC, STAGED, NT, MX>(p, X, pb, stream);
    if (p.log2_group == 5 || SMAX == 32)
        return launch_s<NBITS, 32, VEC, STAGED, NT, MX>(p, X, pb, stream);
    return launch_s<NBITS, SMAX, VEC, STAGED, NT, MX>(p, X, pb, stream);
}

template <int NBITS, bool VEC, int NT, bool MX>
cudaError_t launch_st(const LinearParams& p, const void* X, int64_t pb, cudaStream_t stream) {
    const bool staged = (reinterpret_cast<uintptr_t>(p.packed) & 15u) == 0 && p.K < ((int64_t)1 << 30);
    // 3 bits, 6 to 16 tokens: CTAs that share one staged copy of X (measured
    // on the 70B gate and down shapes: 102-111 -> 103 us at 6 tokens, 123-144
    // -> 103-105 us at 8, 168 -> 114-120 us at 16; slower than the per-warp
    // form below 6)
    if constexpr (NBITS == 3) {
        if (p.M >= 6 && p.K < ((int64_t)1 << 30) && (reinterpret_cast<uintptr_t>(X) & 15u) == 0) {
            if (staged) {
                if (p.log2_group == 4) return launch_sx<3, 16, NT, true>(p, X, pb, stream);
                if (p.log2_group == 5) return launch_sx<3, 32, NT, true>(p, X, pb, stream);
                return launch_sx<3, 64, NT, true>(p, X, pb, stream);
            }
            if (p.log2_group == 4) return launch_sx<3, 16, NT, false>(p, X, pb, stream);
            if (p.log2_group == 5) return launch_sx<3, 32, NT, false>(p, X, pb, stream);
            return launch_sx<3, 64, NT, false>(p, X, pb, stream);
        }
    }
    return staged ? launch_g<NBITS, VEC, true, NT, MX>(p, X, pb, stream)
                  : launch_g<NBITS, VEC, false, NT, MX>(p, X, pb, stream);
}

template <int NBITS, bool VEC>
cudaError_t launch_nt(const LinearParams& p, const void* X, int64_t pb, cudaStream_t stream) {
    // 4 bits, one token: codes in pairs through half-precision magic numbers
    // (measured on 8192 x 8192: 25.0 -> 22.4 us; slower from 2 tokens)
    if constexpr (NBITS == 4)
        if (p.M == 1) return launch_st<NBITS, VEC, 1, true>(p, X, pb, stream);
    if (p.M <= 8) return launch_st<NBITS, VEC, 1, false>(p, X, pb, stream);
    return launch_st<NBITS, VEC, 2, false>(p, X, pb, stream);
}

}  // namespace

// Few-token form of the linear layer (1 <= M <= decode_max_tokens(nbits));
// packed_bytes is the size of the packed buffer (hqq_packed_bytes).
cudaError_t launch_decode(const LinearParams& p, const void* X, int nbits, int64_t packed_bytes,
                          cudaStream_t stream) {
    const bool vec8 = (reinterpret_cast<uintptr_t>(p.packed) & 7u) == 0;
    switch (nbits) {
        case 1: return launch_nt<1, false>(p, X, packed_bytes, stream);
        case 2: return launch_nt<2, false>(p, X, packed_bytes, stream);
        case 3: return launch_nt<3, false>(p, X, packed_bytes, stream);
        case 4:
            return vec8 ? launch_nt<4, true>(p, X, packed_bytes, stream)
                        : launch_nt<4, false>(p, X, packed_bytes, stream);
        case 8: return launch_nt<8, true>(p, X, packed_bytes, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace hqq
