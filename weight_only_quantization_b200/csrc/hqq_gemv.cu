// hqq_gemv.cu -- the weight-only linear layer for a few tokens (M <= 8): the
// same product as hqq_linear.cu, Y[m, n] = sum_k X[m, k] * W_hat[n, k] with
// W_hat = fp16((code - z) * s) (section 2's Q^-1 of "Half-Quadratic
// Quantization of Large Machine Learning Models"), but as a streaming kernel
// on the CUDA cores.  With so few tokens the product is bound by reading the
// packed weights (0.3 .. 1 byte per weight), not by arithmetic, so it gets no
// tensor-core pipeline: a CTA owns R consecutive output features, its 8 warps
// split the input dimension, and every lane streams consecutive 8-weight
// units (one warp load = 32 consecutive units of one row).  Each unit is
// dequantized exactly as hqq_dequantize does (fp16 W_hat), widened to fp32 and
// multiplied into fp32 accumulators; the warps' partial sums meet in shared
// memory and the result is rounded to fp16 once.
#include "hqq_unpack.cuh"

namespace hqq {

namespace {

constexpr int kGvWarps = 8;
constexpr int kGvThreads = kGvWarps * 32;

// R rows per CTA (2 up to 4 tokens, else 1: measured best for one token, and
// it bounds the R * M accumulator pairs and the M token vectors of a unit kept
// in registers); U units per lane and row are loaded ahead.
template <int NBITS, bool SMALL, int M, int R>
__global__ void __launch_bounds__(kGvThreads)
gemv_kernel(const __half* __restrict__ X, const __grid_constant__ LinearParams p) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t n0 = (int64_t)blockIdx.x * R;
    const int64_t ku = p.K >> 3;                                  // units per row
    // this warp's slice of the units of a row
    const int64_t per = (ku + kGvWarps - 1) / kGvWarps;
    const int64_t u_begin = per * warp;
    const int64_t u_end = min(ku, u_begin + per);

    float2 acc[R][M];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int m = 0; m < M; ++m) acc[r][m] = make_float2(0.0f, 0.0f);

    constexpr int kGvUnroll = R >= 8 ? 2 : 4;
    for (int64_t ub = u_begin; ub < u_end; ub += 32 * kGvUnroll) {
        // all loads of the step first: codes and group data of R rows
        uint32_t bits[kGvUnroll][R];
        UnitRaw raw8[NBITS == 8 ? kGvUnroll : 1][NBITS == 8 ? R : 1];
        __half2 sz[kGvUnroll][R];
#pragma unroll
        for (int i = 0; i < kGvUnroll; ++i) {
            const int64_t u = ub + 32 * i + lane;
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const int64_t n = n0 + r;
                if (u < u_end && n < p.N) {
                    const int64_t unit = n * ku + u;
                    const int64_t g = (unit << 3) >> p.log2_group;
                    if constexpr (NBITS == 8)
                        raw8[i][r] = unit_fetch<8, SMALL>(p.packed, unit);
                    else
                        bits[i][r] = unit_bits<NBITS, SMALL>(p.packed, unit);
                    sz[i][r] = __halves2half2(__ldg(p.scale + g), __ldg(p.zero + g));
                } else {
                    if constexpr (NBITS == 8) raw8[i][r].w0 = raw8[i][r].w1 = 0u;
                    else bits[i][r] = 0u;
                    sz[i][r] = __float2half2_rn(0.0f);           // s = 0: W_hat = 0
                }
            }
        }
#pragma unroll
        for (int i = 0; i < kGvUnroll; ++i) {
            const int64_t u = ub + 32 * i + lane;
            if (u >= u_end) continue;
            float2 x[M][4];                                       // X[m, 8u .. 8u+7]
#pragma unroll
            for (int m = 0; m < M; ++m) {
                const uint4 xv = __ldg(reinterpret_cast<const uint4*>(X + m * p.K) + u);
                x[m][0] = __half22float2(*reinterpret_cast<const __half2*>(&xv.x));
                x[m][1] = __half22float2(*reinterpret_cast<const __half2*>(&xv.y));
                x[m][2] = __half22float2(*reinterpret_cast<const __half2*>(&xv.z));
                x[m][3] = __half22float2(*reinterpret_cast<const __half2*>(&xv.w));
            }
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const float s = __low2float(sz[i][r]), z = __high2float(sz[i][r]);
                uint4 wv;
                if constexpr (NBITS == 8)
                    wv = unit8_raw<8>(raw8[i][r], z, s);
                else
                    wv = unit8<NBITS>(bits[i][r], z, s);
                const float2 w0 = __half22float2(*reinterpret_cast<const __half2*>(&wv.x));
                const float2 w1 = __half22float2(*reinterpret_cast<const __half2*>(&wv.y));
                const float2 w2 = __half22float2(*reinterpret_cast<const __half2*>(&wv.z));
                const float2 w3 = __half22float2(*reinterpret_cast<const __half2*>(&wv.w));
#pragma unroll
                for (int m = 0; m < M; ++m) {
                    float2 a = acc[r][m];
                    a = __ffma2_rn(w0, x[m][0], a);
                    a = __ffma2_rn(w1, x[m][1], a);
                    a = __ffma2_rn(w2, x[m][2], a);
                    a = __ffma2_rn(w3, x[m][3], a);
                    acc[r][m] = a;
                }
            }
        }
    }

    // warp sums, then the warps' partials in shared memory
    __shared__ float part[kGvWarps][R * M];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int m = 0; m < M; ++m) {
            float v = __fadd_rn(acc[r][m].x, acc[r][m].y);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
            if (lane == 0) part[warp][r * M + m] = v;
        }
    __syncthreads();
    if (threadIdx.x < R * M) {
        const int r = threadIdx.x / M, m = threadIdx.x % M;
        float v = 0.0f;
#pragma unroll
        for (int w = 0; w < kGvWarps; ++w) v = __fadd_rn(v, part[w][threadIdx.x]);
        const int64_t n = n0 + r;
        if (n < p.N) p.Y[(int64_t)m * p.N + n] = __float2half_rn(v);
    }
}

template <int NBITS, bool SMALL, int M>
cudaError_t launch_m(const LinearParams& p, const void* X, cudaStream_t stream) {
    constexpr int R = M <= 4 ? 2 : 1;
    const int64_t blocks = (p.N + R - 1) / R;
    gemv_kernel<NBITS, SMALL, M, R><<<(unsigned)blocks, kGvThreads, 0, stream>>>(
        static_cast<const __half*>(X), p);
    return cudaGetLastError();
}

template <int NBITS, bool SMALL>
cudaError_t launch_gv(const LinearParams& p, const void* X, cudaStream_t stream) {
    switch (p.M) {
        case 1: return launch_m<NBITS, SMALL, 1>(p, X, stream);
        case 2: return launch_m<NBITS, SMALL, 2>(p, X, stream);
        case 3: return launch_m<NBITS, SMALL, 3>(p, X, stream);
        case 4: return launch_m<NBITS, SMALL, 4>(p, X, stream);
        case 5: return launch_m<NBITS, SMALL, 5>(p, X, stream);
        case 6: return launch_m<NBITS, SMALL, 6>(p, X, stream);
        case 7: return launch_m<NBITS, SMALL, 7>(p, X, stream);
        default: return launch_m<NBITS, SMALL, 8>(p, X, stream);
    }
}

}  // namespace

// Few-token form of the linear layer (1 <= M <= 8).
cudaError_t launch_gemv(const LinearParams& p, const void* X, int nbits, cudaStream_t stream) {
    const bool small = p.N * p.K / 8 < ((int64_t)1 << 30);
    switch (nbits) {
        case 1: return launch_gv<1, true>(p, X, stream);
        case 2: return launch_gv<2, true>(p, X, stream);
        case 4: return launch_gv<4, true>(p, X, stream);
        case 8: return launch_gv<8, true>(p, X, stream);
        case 3: return small ? launch_gv<3, true>(p, X, stream) : launch_gv<3, false>(p, X, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace hqq
