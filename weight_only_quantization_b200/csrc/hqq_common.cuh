// hqq_common.cuh -- types and device helpers shared by libhqq's kernels.
//
// Arithmetic contract of the solver (binary32, round-to-nearest-even, every
// rounding explicit): products and sums that the method writes separately are
// issued as __fmul_rn / __fadd_rn / __fsub_rn (never contracted), and the three
// places that are defined as one fused multiply-add use __fmaf_rn.  The library
// is also compiled with -fmad=false.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace hqq {

// |x|^p by table-driven evaluation (after P. T. P. Tang, "Table-driven
// implementation of the exponential function", ACM TOMS 15(2), 1989):
//   x = 2^k m, m in [1,2); c_j = 1 + (2j+1)/64 is the centre of the 1/32-wide
//   cell of m picked by its top five mantissa bits; r = (m - c_j) * (1/c_j),
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

constexpr int kTabFloats = 256 + 32 + 32;   // the part copied to shared memory
constexpr int kMaxIters = 255;

struct QuantParams {
    const __half* W;
    uint8_t* packed;
    __half* scale;
    __half* zero;
    float* zero_f32;       // nullable
    uint8_t* iters_out;    // nullable
    int64_t n_groups;
    int64_t n_elems;
    int iters;
    float beta;
    float kappa;
    PowTable tp;           // exponent p     (l_p error)
    PowTable tq;           // exponent p - 1 (generalised shrink)
    float shrink_thr[kMaxIters];  // |r| <= thr[t] guarantees W_e == 0 at step t
};

struct DequantParams {
    const uint8_t* packed;
    const __half* scale;
    const __half* zero;
    __half* out;
    int64_t n_units;       // n_elems / 8
    int group;
};

// Table-driven |x|^p for x >= +0 (sign bit clear).  `tab` points at the
// kTabFloats-long shared-memory copy of two_pk, cj_p, inv_cj.
__device__ __forceinline__ float powp(const float* __restrict__ tab, float a1, float a2,
                                      float a3, float x) {
    const uint32_t b = __float_as_uint(x);
    const uint32_t e = b >> 23;
    const uint32_t j = (b >> 18) & 31u;
    const float m = __uint_as_float((b & 0x007FFFFFu) | 0x3F800000u);
    const float c = __uint_as_float((b & 0x007C0000u) | 0x3F820000u);
    const float r = __fmul_rn(__fsub_rn(m, c), tab[288 + j]);   // m - c is exact
    const float poly = __fmaf_rn(__fmaf_rn(__fmaf_rn(r, a3, a2), r, a1), r, 1.0f);
    return __fmul_rn(__fmul_rn(tab[e], tab[256 + j]), poly);
}

// Round-half-even of v in [0, 2^22) by the 1.5*2^23 shift: the sum's last
// mantissa bit is worth 1, so the addition itself rounds; the low bits of the
// sum then hold the integer.
constexpr float kRoundShift = 12582912.0f;   // 1.5 * 2^23, bits 0x4B400000

}  // namespace hqq
