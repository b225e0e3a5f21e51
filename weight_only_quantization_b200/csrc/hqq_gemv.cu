// hqq_gemv.cu -- the weight-only linear layer for one or two tokens: the
// same product as hqq_linear.cu, Y[m, n] = sum_k X[m, k] * W_hat[n, k] with
// W_hat = fp16((code - z) * s) (section 2's Q^-1 of "Half-Quadratic
// Quantization of Large Machine Learning Models"), but as a streaming kernel
// on the CUDA cores.  With so few tokens the product is bound by reading the
// packed weights (0.3 .. 1 byte per weight), not by arithmetic, so it gets no
// tensor-core pipeline: a CTA owns R consecutive output features, its 8 warps
// split the input dimension, and every lane streams quads of 32 consecutive
// codes (a warp load covers 1024 codes of one row).  Each unit is dequantized
// exactly as hqq_dequantize does (fp16 W_hat), widened to fp32 and multiplied
// into fp32 accumulators; the warps' partial sums meet in shared memory and
// the result is rounded to fp16 once.
#include "hqq_unpack.cuh"

namespace hqq {

namespace {

constexpr int kGvWarps = 8;
constexpr int kGvThreads = kGvWarps * 32;
constexpr int kGvUnroll = 2;               // quads per lane and row loaded ahead

// MT >= M token rows (rows past M read as zero and are not stored).  A CTA owns
// R output features; its 8 warps split the quads (32 codes) of a row, and each
// lane takes one quad of each of the R rows per step: one vector load of codes
// and one (scale, zero) pair per quad and row, four 16-byte token loads per
// quad shared by the R rows.
template <int NBITS, bool SMALL, bool VEC, int MT, int R>
__global__ void __launch_bounds__(kGvThreads)
gemv_kernel(const __half* __restrict__ X, const __grid_constant__ LinearParams p) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t n0 = (int64_t)blockIdx.x * R;
    const int64_t nq = (p.K + 31) >> 5;                             // quads per row
    const int64_t per = (nq + kGvWarps - 1) / kGvWarps;
    const int64_t q_begin = per * warp;
    const int64_t q_end = min(nq, q_begin + per);

    float2 acc[R][MT];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[r][m] = make_float2(0.0f, 0.0f);

    for (int64_t qb = q_begin; qb < q_end; qb += 32 * kGvUnroll) {
        QuadCodes<NBITS> qc[kGvUnroll][R];                          // all loads first
#pragma unroll
        for (int i = 0; i < kGvUnroll; ++i) {
            const int64_t q = qb + 32 * i + lane;
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const int64_t n = n0 + r;
                load_quad<NBITS, SMALL, VEC>(p, n * p.K, n < p.N && q < q_end, q * 32, qc[i][r]);
            }
        }
#pragma unroll
        for (int i = 0; i < kGvUnroll; ++i) {
            const int64_t q = qb + 32 * i + lane;
            if (q >= q_end) continue;
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const int64_t k = q * 32 + 8 * t;
                if (k >= p.K) break;
                float2 x[MT][4];                                     // X[m, k .. k+7]
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    if (m < p.M) {
                        const uint4 xv = __ldg(reinterpret_cast<const uint4*>(X + m * p.K + k));
                        x[m][0] = __half22float2(*reinterpret_cast<const __half2*>(&xv.x));
                        x[m][1] = __half22float2(*reinterpret_cast<const __half2*>(&xv.y));
                        x[m][2] = __half22float2(*reinterpret_cast<const __half2*>(&xv.z));
                        x[m][3] = __half22float2(*reinterpret_cast<const __half2*>(&xv.w));
                    } else {
#pragma unroll
                        for (int e = 0; e < 4; ++e) x[m][e] = make_float2(0.0f, 0.0f);
                    }
                }
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    if (!(qc[i][r].present & (1u << t))) continue;
                    const uint4 wv = quad_unit<NBITS>(qc[i][r], t);
                    const float2 w0 = __half22float2(*reinterpret_cast<const __half2*>(&wv.x));
                    const float2 w1 = __half22float2(*reinterpret_cast<const __half2*>(&wv.y));
                    const float2 w2 = __half22float2(*reinterpret_cast<const __half2*>(&wv.z));
                    const float2 w3 = __half22float2(*reinterpret_cast<const __half2*>(&wv.w));
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
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
    }

    // warp sums, then the warps' partials in shared memory
    __shared__ float part[kGvWarps][R * MT];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            float v = __fadd_rn(acc[r][m].x, acc[r][m].y);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
            if (lane == 0) part[warp][r * MT + m] = v;
        }
    __syncthreads();
    if (threadIdx.x < R * MT) {
        const int r = threadIdx.x / MT, m = threadIdx.x % MT;
        float v = 0.0f;
#pragma unroll
        for (int w = 0; w < kGvWarps; ++w) v = __fadd_rn(v, part[w][threadIdx.x]);
        const int64_t n = n0 + r;
        if (n < p.N && m < p.M) p.Y[(int64_t)m * p.N + n] = __float2half_rn(v);
    }
}

// Persistent form: X staged once per CTA in shared memory (fp16), each warp
// owns whole output features (rows), its lanes take quads l, l+32, ... of the
// row with kPvUnroll quads' loads issued before any use, and a warp shuffle
// sums the row.  No cross-warp reduction, no token reloads per row.
constexpr int kPvUnroll = 4;

template <int NBITS, bool SMALL, bool VEC, int MT>
__global__ void __launch_bounds__(kGvThreads)
gemv_rows_kernel(const __half* __restrict__ X, const __grid_constant__ LinearParams p) {
    extern __shared__ __align__(16) uint8_t gv_smem[];
    __half* xs = reinterpret_cast<__half*>(gv_smem);            // [MT][K], rows past M zero
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    {
        const int64_t nv = (int64_t)MT * p.K / 8;                  // 16-byte vectors
        for (int64_t v = threadIdx.x; v < nv; v += kGvThreads) {
            const int64_t m = v * 8 / p.K;
            uint4 val = make_uint4(0u, 0u, 0u, 0u);
            if (m < p.M) val = __ldg(reinterpret_cast<const uint4*>(X) + v);
            reinterpret_cast<uint4*>(xs)[v] = val;
        }
    }
    __syncthreads();
    const int64_t nq = (p.K + 31) >> 5;
    for (int64_t n = (int64_t)blockIdx.x * kGvWarps + warp; n < p.N;
         n += (int64_t)gridDim.x * kGvWarps) {
        float2 acc[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[m] = make_float2(0.0f, 0.0f);
        for (int64_t qb = 0; qb < nq; qb += 32 * kPvUnroll) {
            QuadCodes<NBITS> qc[kPvUnroll];
#pragma unroll
            for (int i = 0; i < kPvUnroll; ++i) {
                const int64_t q = qb + 32 * i + lane;
                load_quad<NBITS, SMALL, VEC>(p, n * p.K, q < nq, q * 32, qc[i]);
            }
#pragma unroll
            for (int i = 0; i < kPvUnroll; ++i) {
                const int64_t q = qb + 32 * i + lane;
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    if (!(qc[i].present & (1u << t))) continue;
                    const uint4 wv = quad_unit<NBITS>(qc[i], t);
                    const float2 w0 = __half22float2(*reinterpret_cast<const __half2*>(&wv.x));
                    const float2 w1 = __half22float2(*reinterpret_cast<const __half2*>(&wv.y));
                    const float2 w2 = __half22float2(*reinterpret_cast<const __half2*>(&wv.z));
                    const float2 w3 = __half22float2(*reinterpret_cast<const __half2*>(&wv.w));
                    const int64_t k = q * 32 + 8 * t;
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        const uint4 xv = *reinterpret_cast<const uint4*>(xs + m * p.K + k);
                        float2 a = acc[m];
                        a = __ffma2_rn(w0, __half22float2(*reinterpret_cast<const __half2*>(&xv.x)), a);
                        a = __ffma2_rn(w1, __half22float2(*reinterpret_cast<const __half2*>(&xv.y)), a);
                        a = __ffma2_rn(w2, __half22float2(*reinterpret_cast<const __half2*>(&xv.z)), a);
                        a = __ffma2_rn(w3, __half22float2(*reinterpret_cast<const __half2*>(&xv.w)), a);
                        acc[m] = a;
                    }
                }
            }
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            float v = __fadd_rn(acc[m].x, acc[m].y);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
            if (lane == 0 && m < p.M) p.Y[(int64_t)m * p.N + n] = __float2half_rn(v);
        }
    }
}

// Shared memory of the persistent form: the token rows in fp16.
constexpr int64_t kPvMaxSmem = 160 * 1024;

template <int NBITS, bool SMALL, bool VEC, int MT>
cudaError_t launch_rows(const LinearParams& p, const void* X, cudaStream_t stream) {
    auto kern = gemv_rows_kernel<NBITS, SMALL, VEC, MT>;
    const size_t smem = (size_t)MT * p.K * 2;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148, per_sm = 1;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kGvThreads, smem);
    if (per_sm < 1) per_sm = 1;
    int64_t blocks = (int64_t)sms * per_sm;
    const int64_t need = (p.N + kGvWarps - 1) / kGvWarps;
    if (blocks > need) blocks = need;
    kern<<<(unsigned)blocks, kGvThreads, smem, stream>>>(static_cast<const __half*>(X), p);
    return cudaGetLastError();
}

template <int NBITS, bool SMALL, bool VEC, int MT>
cudaError_t launch_m(const LinearParams& p, const void* X, cudaStream_t stream) {
    // measured: the persistent form is faster at 3 bits (gate 28672x8192: 0.129
    // vs 0.141 ms for one token), slower at 4 bits (8192^2: 0.053 vs 0.041 ms)
    if (NBITS == 3 && (int64_t)MT * p.K * 2 <= kPvMaxSmem)
        return launch_rows<NBITS, SMALL, VEC, MT>(p, X, stream);
    constexpr int R = MT <= 2 ? 2 : 1;
    const int64_t blocks = (p.N + R - 1) / R;
    gemv_kernel<NBITS, SMALL, VEC, MT, R><<<(unsigned)blocks, kGvThreads, 0, stream>>>(
        static_cast<const __half*>(X), p);
    return cudaGetLastError();
}

template <int NBITS, bool SMALL, bool VEC>
cudaError_t launch_gv(const LinearParams& p, const void* X, cudaStream_t stream) {
    if (p.M <= 1) return launch_m<NBITS, SMALL, VEC, 1>(p, X, stream);
    return launch_m<NBITS, SMALL, VEC, 2>(p, X, stream);
}

template <int NBITS>
cudaError_t launch_gvec(const LinearParams& p, const void* X, cudaStream_t stream) {
    const bool vec = p.K % 32 == 0 && (reinterpret_cast<uintptr_t>(p.packed) & 15u) == 0;
    return vec ? launch_gv<NBITS, true, true>(p, X, stream)
               : launch_gv<NBITS, true, false>(p, X, stream);
}

}  // namespace

// Few-token form of the linear layer (1 <= M <= kGemvMaxTokens).
cudaError_t launch_gemv(const LinearParams& p, const void* X, int nbits, cudaStream_t stream) {
    const bool small = p.N * p.K / 8 < ((int64_t)1 << 30);
    switch (nbits) {
        case 1: return launch_gvec<1>(p, X, stream);
        case 2: return launch_gvec<2>(p, X, stream);
        case 4: return launch_gvec<4>(p, X, stream);
        case 8: return launch_gvec<8>(p, X, stream);
        case 3:
            return small ? launch_gv<3, true, false>(p, X, stream)
                         : launch_gv<3, false, false>(p, X, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace hqq
