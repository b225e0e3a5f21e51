// hqq_common.cuh -- the quantize kernel's types and device helpers, and the
// arithmetic contract every libhqq kernel follows.
//
// Arithmetic contract of the solver (binary32, round-to-nearest-even, every
// rounding explicit): products and sums that the method writes separately are
// issued as __fmul_rn / __fadd_rn or their packed f32x2 forms (__fmul2_rn,
// __fadd2_rn: two independent binary32 operations, each rounded to nearest),
// never contracted, and the places defined as one fused multiply-add use
// __fmaf_rn / __ffma2_rn.  The library is also compiled with -fmad=false.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace hqq {

// |x|^p by table-driven evaluation (after P. T. P. Tang, "Table-driven
// implementation of the exponential function", ACM TOMS 15(2), 1989):
//   x = 2^k m, m in [1,2); c_j = 1 + (2j+1)/64 is the centre of the 1/32-wide
//   cell of m picked by its top five mantissa bits; r = fma(m, fl(1/c_j), -1),
//   |r| <= 1/64, and (1+r)^p = 1 + r(a1 + r(a2 + r a3)) (binomial series).
//   |x|^p = (2^(p k) * c_j^p) * (1+r)^p.
// two_pk[e] for the biased exponent e (e = 0: +0 and subnormals -> 0, +inf or 1
// for p >0, <0, =0); cj_p and inv_cj per cell.  Built on the host per call.
struct PowTable {
    float two_pk[256];
    float cj_p[32];
    float inv_cj[32];
    float a1, a2, a3;
};

constexpr int kMaxIters = 255;

struct QuantParams {
    const __half* W;
    uint8_t* packed;
    __half* scale;
    __half* zero;
    float* zero_f32;       // nullable
    float* err_out;        // nullable
    uint8_t* iters_out;    // nullable
    uint8_t* half_out;     // nullable: 1 where a group was solved in half precision
    int64_t n_groups;
    int64_t n_elems;
    int iters;
    float beta;
    float kappa;
    PowTable tp;           // exponent p     (l_p error)
    PowTable tq;           // exponent p - 1 (generalised shrink)
    float shrink_thr[kMaxIters];  // |r| <= thr[t] guarantees W_e == 0 at step t
    float shrink_thr16[kMaxIters];  // the same for the half-precision shrink
};

// Shared-memory image of one PowTable (separate arrays, so that the two values
// of an f32x2 pair are loaded straight into the two halves of a register pair).
struct PowSmem {
    float te[256];   // 2^(p k) by biased exponent
    float tc[32];    // c_j^p
    float ic[32];    // fl(1 / c_j)
};

__device__ __forceinline__ void load_pow_smem(PowSmem& dst, const PowTable& t) {
    for (int i = threadIdx.x; i < 256; i += blockDim.x) dst.te[i] = t.two_pk[i];
    for (int i = threadIdx.x; i < 32; i += blockDim.x) {
        dst.tc[i] = t.cj_p[i];
        dst.ic[i] = t.inv_cj[i];
    }
}

// Word at byte offset `off` of a shared-memory table.
__device__ __forceinline__ float tab_at(const float* t, uint32_t off) {
    return *reinterpret_cast<const float*>(reinterpret_cast<const char*>(t) + off);
}

// |x|^p of two values (any sign) with the table in shared memory.  The table
// offsets are taken straight from the bit pattern: bits 23..30 (exponent of
// |x|) times 4 and bits 18..22 (mantissa cell) times 4.
__device__ __forceinline__ float2 powp2(const PowSmem& T, float2 a1, float2 a2, float2 a3,
                                        float2 x) {
    const uint32_t bx = __float_as_uint(x.x), by = __float_as_uint(x.y);
    const uint32_t ex = (bx >> 21) & 0x3FCu, ey = (by >> 21) & 0x3FCu;
    const uint32_t jx = (bx >> 16) & 0x7Cu, jy = (by >> 16) & 0x7Cu;
    const float2 m = make_float2(__uint_as_float((bx & 0x007FFFFFu) | 0x3F800000u),
                                 __uint_as_float((by & 0x007FFFFFu) | 0x3F800000u));
    const float2 r = __ffma2_rn(m, make_float2(tab_at(T.ic, jx), tab_at(T.ic, jy)),
                                make_float2(-1.0f, -1.0f));
    float2 poly = __ffma2_rn(r, a3, a2);
    poly = __ffma2_rn(poly, r, a1);
    poly = __ffma2_rn(poly, r, make_float2(1.0f, 1.0f));
    const float2 tt = __fmul2_rn(make_float2(tab_at(T.te, ex), tab_at(T.te, ey)),
                                 make_float2(tab_at(T.tc, jx), tab_at(T.tc, jy)));
    return __fmul2_rn(tt, poly);
}

// Combined table for the hot |x|^p: t2[e*32 + j] = fl(2^(p(e-127)) * c_j^p),
// exactly the product the method's power forms first, so one lookup replaces
// two and a multiplication.  Its byte offset comes straight from bits 18..30 of
// x ((x >> 16) & 0x7FFC); the cell's 1/c_j from bits 18..22 ((x >> 16) & 0x7C).
struct PowSmem2 {
    float t2[256 * 32];
    float ic[32];
};

// Lane l fills cell l of every exponent row; the row's 2^(pk) is warp-uniform,
// so each warp reads kernel parameters without per-lane serialisation.
__device__ __forceinline__ void load_pow_smem2(PowSmem2& dst, const PowTable& t) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const float cj = t.cj_p[lane];
    for (int e = warp; e < 256; e += nw) dst.t2[e * 32 + lane] = __fmul_rn(t.two_pk[e], cj);
    if (threadIdx.x < 32) dst.ic[threadIdx.x] = t.inv_cj[threadIdx.x];
}

// |x|^p of two values (any sign) with the combined table.
__device__ __forceinline__ float2 powp2c(const PowSmem2& T, float2 a1, float2 a2, float2 a3,
                                         float2 x) {
    const uint32_t ux = __float_as_uint(x.x), uy = __float_as_uint(x.y);
    const uint32_t hx = ux >> 16, hy = uy >> 16;
    const float2 m = make_float2(__uint_as_float((ux & 0x007FFFFFu) | 0x3F800000u),
                                 __uint_as_float((uy & 0x007FFFFFu) | 0x3F800000u));
    const float2 r = __ffma2_rn(m, make_float2(tab_at(T.ic, hx & 0x7Cu), tab_at(T.ic, hy & 0x7Cu)),
                                make_float2(-1.0f, -1.0f));
    float2 poly = __ffma2_rn(r, a3, a2);
    poly = __ffma2_rn(poly, r, a1);
    poly = __ffma2_rn(poly, r, make_float2(1.0f, 1.0f));
    return __fmul2_rn(make_float2(tab_at(T.t2, hx & 0x7FFCu), tab_at(T.t2, hy & 0x7FFCu)), poly);
}

// The hot power for either table layout.
__device__ __forceinline__ float2 powp_hot(const PowSmem2& T, float2 a1, float2 a2, float2 a3,
                                           float2 x) {
    return powp2c(T, a1, a2, a3, x);
}
__device__ __forceinline__ float2 powp_hot(const PowSmem& T, float2 a1, float2 a2, float2 a3,
                                           float2 x) {
    return powp2(T, a1, a2, a3, x);
}
__device__ __forceinline__ void load_pow_hot(PowSmem2& dst, const PowTable& t) {
    load_pow_smem2(dst, t);
}
__device__ __forceinline__ void load_pow_hot(PowSmem& dst, const PowTable& t) {
    load_pow_smem(dst, t);
}

// Scalar form (same operations) for the shrink's |x|^(p-1), x >= +0.
__device__ __forceinline__ float powp1(const PowSmem& T, float a1, float a2, float a3, float x) {
    const uint32_t b = __float_as_uint(x);
    const uint32_t j = (b >> 18) & 31u;
    const float m = __uint_as_float((b & 0x007FFFFFu) | 0x3F800000u);
    const float r = __fmaf_rn(m, T.ic[j], -1.0f);
    const float poly = __fmaf_rn(__fmaf_rn(__fmaf_rn(r, a3, a2), r, a1), r, 1.0f);
    return __fmul_rn(__fmul_rn(T.te[(b >> 23) & 0xFFu], T.tc[j]), poly);
}

// Round-half-even of v in [0, 2^22) by the 1.5*2^23 shift: the sum's last
// mantissa bit is worth 1, so the addition itself rounds; the low bits of the
// sum then hold the integer.
constexpr float kRoundShift = 12582912.0f;   // 1.5 * 2^23, bits 0x4B400000

}  // namespace hqq
