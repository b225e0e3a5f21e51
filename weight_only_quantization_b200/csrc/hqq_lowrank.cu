// hqq_lowrank.cu -- rank-r residual of the quantization error: Delta W =
// W - W_hat ~ B A with B = U_r Sigma_r, A = V_r^T, the plain-SVD compensation
// of "Boost 2-bit LLM accuracy with EoRA" (section on finding adapters in the
// feature space).  Delta W is never stored: every product forms it tile by
// tile from the fp16 W and the packed codes (W_hat exactly as hqq_dequantize
// restores it, the difference in fp32).
//
// The truncated SVD is computed by randomized subspace iteration (Halko,
// Martinsson and Tropp, "Finding structure with randomness", SIAM Review 2011:
// Algorithm 4.4 for the range, Algorithm 5.1 for the factorization) with a
// sketch of l = 16, 32 or 64 columns and a Gaussian test matrix given by the
// caller:
//   Y = orth(dW Omega); q times { Z = orth(dW^T Y); Y = orth(dW Z) };
//   Z = dW^T Y (so Z^T = Q^T dW, l x K); Z^T Z = U_s Lambda U_s^T (Jacobi);
//   sigma = sqrt(Lambda); B = Y U_s,r Sigma_r; A = (Z U_s,r Sigma_r^-1)^T.
// orth() is shifted CholeskyQR3 (Fukaya, Kannan, Nakatsukasa, Yamamoto and
// Yanagisawa, SIAM J. Sci. Comput. 2020): three passes of Gram matrix (fp64),
// Cholesky factor R and X <- X R^-1, the first with a small diagonal shift.
// The l x l eigenproblem is solved by cyclic Jacobi in fp64 (Golub and Van
// Loan, "Matrix Computations", the symmetric Schur rotation), L/2 disjoint
// rotations at a time in round-robin order.
#include <cuda.h>
#include <mutex>
#include <utility>

#include "hqq_unpack.cuh"

namespace hqq {

namespace {

constexpr int kLrThreads = 256;

struct LrParams {
    const __half* W;
    const uint8_t* packed;
    const __half* scale;
    const __half* zero;
    int64_t N, K;
    int log2_group;
};

// One unit (8 consecutive weights of a row, flat index f, f % 8 == 0) in
// flight: its fp16 weights, raw code words and group constants, so that the
// loads of the next tile overlap the current tile's FMAs.
struct UnitLoad {
    uint4 w;
    UnitRaw r;
    __half s, z;
};

template <int NBITS>
__device__ __forceinline__ UnitLoad unit_load(const LrParams& p, int64_t f, bool ok) {
    UnitLoad u;
    if (ok) {
        u.w = __ldg(reinterpret_cast<const uint4*>(p.W + f));
        u.r = unit_fetch<NBITS, false>(p.packed, f >> 3);
        const int64_t g = f >> p.log2_group;
        u.s = __ldg(p.scale + g);
        u.z = __ldg(p.zero + g);
    } else {                                   // W = W_hat = 0: Delta W = 0
        u.w = make_uint4(0u, 0u, 0u, 0u);
        u.r.w0 = u.r.w1 = u.r.shift = 0u;
        u.s = u.z = __float2half(0.0f);
    }
    return u;
}

// Delta W = W - W_hat of the unit in fp32 (W_hat exactly as hqq_dequantize).
template <int NBITS>
__device__ __forceinline__ void unit_delta(const UnitLoad& u, float (&d)[8]) {
    const uint4 hv = unit8_raw<NBITS>(u.r, __half2float(u.z), __half2float(u.s));
    const __half2* w2 = reinterpret_cast<const __half2*>(&u.w);
    const __half2* h2 = reinterpret_cast<const __half2*>(&hv);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 a = __half22float2(w2[i]), b = __half22float2(h2[i]);
        d[2 * i] = __fsub_rn(a.x, b.x);
        d[2 * i + 1] = __fsub_rn(a.y, b.y);
    }
}

// Both products run on the tensor cores: mma.sync m16n8k8 with tf32 operands
// and fp32 accumulation, each fp32 operand split into a tf32 high part and a
// tf32 remainder, a b ~ ah bh + ah bl + al bh (the dropped al bl is below
// 2^-22 of the product), so the products keep fp32 accuracy.  A CTA's 8 warps
// take a 16-row block each and half of the L columns (L/16 blocks of 8).
// Fragments of m16n8k8 (g = lane / 4, q = lane % 4): A (row-major 16 x 8)
// a0 = (g, q), a1 = (g + 8, q), a2 = (g, q + 4), a3 = (g + 8, q + 4);
// B (8 x 8) b0 = (k q, column g), b1 = (k q + 4, column g); D c0 = (g, 2q),
// c1 = (g, 2q + 1), c2 = (g + 8, 2q), c3 = (g + 8, 2q + 1).
// x rounded to tf32 (10 mantissa bits), half-way cases away from zero, as bit
// operations on the magnitude: a carry out of the mantissa moves to the next
// binade, as it should (finite inputs only; the products' operands are).
__device__ __forceinline__ uint32_t tf32_of(float x) {
    return (__float_as_uint(x) + 0x1000u) & 0xFFFFE000u;
}

// x = hi + lo with hi = tf32(x) and lo = tf32(x - hi) (x - hi is exact in fp32).
__device__ __forceinline__ void split_tf32(float x, uint32_t& hi, uint32_t& lo) {
    hi = tf32_of(x);
    lo = tf32_of(__fsub_rn(x, __uint_as_float(hi)));
}

__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// d += A B in split tf32 for one 16 x 8 block: A given as its four fp32
// fragment values, B as the high and low tf32 parts of its two.
__device__ __forceinline__ void mma3(float (&d)[4], const uint32_t (&ah)[4],
                                     const uint32_t (&al)[4], uint32_t bh0, uint32_t bh1,
                                     uint32_t bl0, uint32_t bl1) {
    mma_tf32(d, al, bh0, bh1);
    mma_tf32(d, ah, bl0, bl1);
    mma_tf32(d, ah, bh0, bh1);
}

// Store 4 consecutive values of an operand tile as high and low tf32 parts.
__device__ __forceinline__ void store_split4(uint32_t* hi, uint32_t* lo, float4 v) {
    uint4 h, l;
    split_tf32(v.x, h.x, l.x);
    split_tf32(v.y, h.y, l.y);
    split_tf32(v.z, h.z, l.z);
    split_tf32(v.w, h.w, l.w);
    *reinterpret_cast<uint4*>(hi) = h;
    *reinterpret_cast<uint4*>(lo) = l;
}

// Shared memory of one product CTA: the dW tile (64 x 64, row stride AS) and
// the other operand's tile split into high and low tf32 parts (64 x L, row
// stride L + 8).
constexpr int kLrTile = 64;                               // k (right) or rows (left) per step
template <int L, int AS>
constexpr int prod_smem() {
    return (64 * AS + 2 * kLrTile * (L + 8)) * 4;
}

// Y[N, L] = dW[N, K] M[K, L] over the k-tiles of split blockIdx.y (out: Y, or
// the split's partial block when gridDim.y > 1).  CTA: 64 rows x L, k-tiles
// of 64.  Thread t forms units u = t and t + 256 (row u/8, k 8(u%8)) into
// As[row][k] (row stride 68 words: the fragment loads of a warp hit 32
// distinct banks; lanes 4..7 of each 8 store their upper half first, so each
// quarter-warp store covers 8 distinct 16-byte bank groups); the M tile is
// stored split, [k][column].  Warp w: rows 16 (w / 2) .. +15, column blocks
// (w % 2) L/16 .. +L/16 - 1.  The next tile's loads are issued before the
// current tile's MMAs.
template <int NBITS, int L>
__global__ void __launch_bounds__(kLrThreads)
lr_right_kernel(const __grid_constant__ LrParams p, const float* __restrict__ M,
                float* __restrict__ out, int64_t tiles_per_split) {
    constexpr int NBW = L / 16, LP = L + 8, CG = L / 4, AS = 68;
    constexpr int MV = kLrTile * L / 4, MVT = (MV + kLrThreads - 1) / kLrThreads;
    extern __shared__ __align__(16) float lr_psm[];
    auto As = reinterpret_cast<float(*)[AS]>(lr_psm);
    auto Bh = reinterpret_cast<uint32_t(*)[LP]>(lr_psm + 64 * AS);
    auto Bl = reinterpret_cast<uint32_t(*)[LP]>(lr_psm + 64 * AS + kLrTile * LP);
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31, g = lane >> 2, q = lane & 3;
    const int rb = 16 * (warp >> 1), cb = (warp & 1) * NBW;
    const int64_t n0 = (int64_t)blockIdx.x * 64;
    const int64_t kt0 = (int64_t)blockIdx.y * tiles_per_split;
    const int64_t ktiles = (p.K + kLrTile - 1) / kLrTile;
    const int64_t kt1 = kt0 + tiles_per_split < ktiles ? kt0 + tiles_per_split : ktiles;
    const int ur[2] = {t >> 3, (t >> 3) + 32}, uk = 8 * (t & 7);
    const int hs = (t & 4) ? 4 : 0;                         // half stored first
    float acc[NBW][4];
#pragma unroll
    for (int i = 0; i < NBW; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.0f;
    auto load = [&](int64_t kt, UnitLoad (&u)[2], float4 (&mv)[MVT]) {
        const int64_t k = kt * kLrTile + uk;
#pragma unroll
        for (int h = 0; h < 2; ++h)
            u[h] = unit_load<NBITS>(p, (n0 + ur[h]) * p.K + k, n0 + ur[h] < p.N && k < p.K);
#pragma unroll
        for (int v = 0; v < MVT; ++v) {
            const int idx = t + v * kLrThreads;
            const int kk = idx / CG, c4 = idx % CG;
            mv[v] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (idx < MV && kt * kLrTile + kk < p.K)
                mv[v] = __ldg(reinterpret_cast<const float4*>(M + (kt * kLrTile + kk) * L) + c4);
        }
    };
    UnitLoad u[2];
    float4 mv[MVT];
    if (kt0 < kt1) load(kt0, u, mv);
    for (int64_t kt = kt0; kt < kt1; ++kt) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float d[8];
            unit_delta<NBITS>(u[h], d);
            const float4 lo = make_float4(d[0], d[1], d[2], d[3]), hi = make_float4(d[4], d[5], d[6], d[7]);
            *reinterpret_cast<float4*>(&As[ur[h]][uk + hs]) = hs ? hi : lo;
            *reinterpret_cast<float4*>(&As[ur[h]][uk + 4 - hs]) = hs ? lo : hi;
        }
#pragma unroll
        for (int v = 0; v < MVT; ++v) {
            const int idx = t + v * kLrThreads;
            if (idx < MV) store_split4(&Bh[idx / CG][4 * (idx % CG)], &Bl[idx / CG][4 * (idx % CG)], mv[v]);
        }
        __syncthreads();
        if (kt + 1 < kt1) load(kt + 1, u, mv);
#pragma unroll 4
        for (int k8 = 0; k8 < kLrTile; k8 += 8) {
            uint32_t ah[4], al[4];
            split_tf32(As[rb + g][k8 + q], ah[0], al[0]);
            split_tf32(As[rb + g + 8][k8 + q], ah[1], al[1]);
            split_tf32(As[rb + g][k8 + q + 4], ah[2], al[2]);
            split_tf32(As[rb + g + 8][k8 + q + 4], ah[3], al[3]);
#pragma unroll
            for (int i = 0; i < NBW; ++i) {
                const int c = 8 * (cb + i) + g;
                mma3(acc[i], ah, al, Bh[k8 + q][c], Bh[k8 + q + 4][c], Bl[k8 + q][c],
                     Bl[k8 + q + 4][c]);
            }
        }
        __syncthreads();
    }
    float* o = out + (int64_t)blockIdx.y * p.N * L;
#pragma unroll
    for (int i = 0; i < NBW; ++i) {
        const int c = 8 * (cb + i) + 2 * q;
        const int64_t r0 = n0 + rb + g, r1 = r0 + 8;
        if (r0 < p.N) *reinterpret_cast<float2*>(o + r0 * L + c) = make_float2(acc[i][0], acc[i][1]);
        if (r1 < p.N) *reinterpret_cast<float2*>(o + r1 * L + c) = make_float2(acc[i][2], acc[i][3]);
    }
}

// Z[K, L] = dW^T Y over the rows of split blockIdx.y (out: Z, or the split's
// partial block).  CTA: 64 columns k x L, rows in tiles of 64.  Thread t forms
// units u = t and t + 256 (row u/8, k 8(u%8)) into As[row][k] (stride 72
// words, upper half first on lanes 4..7 as above); the Y tile is stored split,
// [row][column].  Warp w: k 16 (w / 2) .. +15 (the rows of dW^T), column
// blocks as above.
template <int NBITS, int L>
__global__ void __launch_bounds__(kLrThreads)
lr_left_kernel(const __grid_constant__ LrParams p, const float* __restrict__ Y,
               float* __restrict__ out, int64_t rows_per_split) {
    constexpr int NBW = L / 16, LP = L + 8, CG = L / 4, AS = 72;
    constexpr int YV = kLrTile * L / 4, YVT = (YV + kLrThreads - 1) / kLrThreads;
    extern __shared__ __align__(16) float lr_psm[];
    auto As = reinterpret_cast<float(*)[AS]>(lr_psm);
    auto Bh = reinterpret_cast<uint32_t(*)[LP]>(lr_psm + 64 * AS);
    auto Bl = reinterpret_cast<uint32_t(*)[LP]>(lr_psm + 64 * AS + kLrTile * LP);
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31, g = lane >> 2, q = lane & 3;
    const int kb = 16 * (warp >> 1), cb = (warp & 1) * NBW;
    const int64_t k0 = (int64_t)blockIdx.x * 64;
    const int64_t rb = (int64_t)blockIdx.y * rows_per_split;
    const int64_t re = rb + rows_per_split < p.N ? rb + rows_per_split : p.N;
    const int ur[2] = {t >> 3, (t >> 3) + 32}, uk = 8 * (t & 7);
    const int hs = (t & 4) ? 4 : 0;
    const bool col_ok = k0 + uk < p.K;
    float acc[NBW][4];
#pragma unroll
    for (int i = 0; i < NBW; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.0f;
    auto load = [&](int64_t r0, UnitLoad (&u)[2], float4 (&yv)[YVT]) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int64_t n = r0 + ur[h];
            u[h] = unit_load<NBITS>(p, n * p.K + k0 + uk, col_ok && n < re);
        }
#pragma unroll
        for (int v = 0; v < YVT; ++v) {
            const int idx = t + v * kLrThreads;
            const int r = idx / CG, c4 = idx % CG;
            yv[v] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (idx < YV && r0 + r < re)
                yv[v] = __ldg(reinterpret_cast<const float4*>(Y + (r0 + r) * L) + c4);
        }
    };
    UnitLoad u[2];
    float4 yv[YVT];
    if (rb < re) load(rb, u, yv);
    for (int64_t r0 = rb; r0 < re; r0 += kLrTile) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float d[8];
            unit_delta<NBITS>(u[h], d);
            const float4 lo = make_float4(d[0], d[1], d[2], d[3]), hi = make_float4(d[4], d[5], d[6], d[7]);
            *reinterpret_cast<float4*>(&As[ur[h]][uk + hs]) = hs ? hi : lo;
            *reinterpret_cast<float4*>(&As[ur[h]][uk + 4 - hs]) = hs ? lo : hi;
        }
#pragma unroll
        for (int v = 0; v < YVT; ++v) {
            const int idx = t + v * kLrThreads;
            if (idx < YV) store_split4(&Bh[idx / CG][4 * (idx % CG)], &Bl[idx / CG][4 * (idx % CG)], yv[v]);
        }
        __syncthreads();
        if (r0 + kLrTile < re) load(r0 + kLrTile, u, yv);
#pragma unroll 4
        for (int n8 = 0; n8 < kLrTile; n8 += 8) {
            uint32_t ah[4], al[4];                 // dW^T fragment: (k, n) = As[n][k]
            split_tf32(As[n8 + q][kb + g], ah[0], al[0]);
            split_tf32(As[n8 + q][kb + g + 8], ah[1], al[1]);
            split_tf32(As[n8 + q + 4][kb + g], ah[2], al[2]);
            split_tf32(As[n8 + q + 4][kb + g + 8], ah[3], al[3]);
#pragma unroll
            for (int i = 0; i < NBW; ++i) {
                const int c = 8 * (cb + i) + g;
                mma3(acc[i], ah, al, Bh[n8 + q][c], Bh[n8 + q + 4][c], Bl[n8 + q][c],
                     Bl[n8 + q + 4][c]);
            }
        }
        __syncthreads();
    }
    float* o = out + (int64_t)blockIdx.y * p.K * L;
#pragma unroll
    for (int i = 0; i < NBW; ++i) {
        const int c = 8 * (cb + i) + 2 * q;
        const int64_t r0 = k0 + kb + g, r1 = r0 + 8;
        if (r0 < p.K) *reinterpret_cast<float2*>(o + r0 * L + c) = make_float2(acc[i][0], acc[i][1]);
        if (r1 < p.K) *reinterpret_cast<float2*>(o + r1 * L + c) = make_float2(acc[i][2], acc[i][3]);
    }
}

// Z[i] = sum_s Zp[s * n + i].
__global__ void __launch_bounds__(kLrThreads)
lr_reduce_kernel(const float* __restrict__ Zp, int splits, int64_t n, float* __restrict__ Z) {
    for (int64_t i = (int64_t)blockIdx.x * kLrThreads + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * kLrThreads) {
        float s = Zp[i];
        for (int k = 1; k < splits; ++k) s = __fadd_rn(s, Zp[k * n + i]);
        Z[i] = s;
    }
}

// GP[block] = X[rows of the block]^T X[rows of the block] in fp64 (L x L).
template <int L>
__global__ void __launch_bounds__(kLrThreads)
lr_gram_kernel(const float* __restrict__ X, int64_t n, int64_t rpb, double* __restrict__ GP) {
    constexpr int EPT = L * L / kLrThreads;
    __shared__ float Xs[32][L + 1];
    const int t = threadIdx.x;
    const int e0 = t * EPT, i = e0 / L, j0 = e0 % L;
    double acc[EPT];
#pragma unroll
    for (int e = 0; e < EPT; ++e) acc[e] = 0.0;
    const int64_t rb = (int64_t)blockIdx.x * rpb;
    const int64_t re = rb + rpb < n ? rb + rpb : n;
    constexpr int LPT = 32 * L / kLrThreads;              // tile values per thread
    float nx[LPT];                                        // the next tile, loaded ahead
    auto fetch = [&](int64_t r0) {
#pragma unroll
        for (int u = 0; u < LPT; ++u) {
            const int idx = t + u * kLrThreads, r = idx / L, c = idx % L;
            nx[u] = r0 + r < re ? __ldg(X + (r0 + r) * L + c) : 0.0f;
        }
    };
    if (rb < re) fetch(rb);
    for (int64_t r0 = rb; r0 < re; r0 += 32) {
#pragma unroll
        for (int u = 0; u < LPT; ++u) {
            const int idx = t + u * kLrThreads;
            Xs[idx / L][idx % L] = nx[u];
        }
        __syncthreads();
        if (r0 + 32 < re) fetch(r0 + 32);
        for (int r = 0; r < 32; ++r) {
            const double a = (double)Xs[r][i];
#pragma unroll
            for (int e = 0; e < EPT; ++e) acc[e] = fma(a, (double)Xs[r][j0 + e], acc[e]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int e = 0; e < EPT; ++e) GP[(int64_t)blockIdx.x * L * L + e0 + e] = acc[e];
}

// Block 0 of GP <- the sum of the nparts Gram blocks (L x L doubles each), in a
// fixed order: CTA b owns elements 32b .. 32b + 31 (L * L is a multiple of 32);
// warp s of 8 sums blocks s, s + 8, .. (four running sums), then the eight
// warp sums are added in order.  Each element is read and written by its own
// CTA only, and block 0's element is written after every read of it.
template <int L>
__global__ void __launch_bounds__(kLrThreads)
lr_gsum_kernel(double* GP, int nparts) {
    __shared__ double red[8][32];
    constexpr int64_t LL = (int64_t)L * L;
    const int el = threadIdx.x & 31, s = threadIdx.x >> 5;
    const int64_t e = (int64_t)blockIdx.x * 32 + el;
    double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
    int q = s;
    for (; q + 24 < nparts; q += 32) {
        a0 += __ldg(GP + q * LL + e);
        a1 += __ldg(GP + (q + 8) * LL + e);
        a2 += __ldg(GP + (q + 16) * LL + e);
        a3 += __ldg(GP + (q + 24) * LL + e);
    }
    for (; q < nparts; q += 8) a0 += __ldg(GP + q * LL + e);
    red[s][el] = (a0 + a1) + (a2 + a3);
    __syncthreads();
    if (s == 0) {
        double t = red[0][el];
#pragma unroll
        for (int i = 1; i < 8; ++i) t += red[i][el];
        GP[e] = t;
    }
}

// Sum over the nparts Gram blocks of element e: eight independent partial
// sums (loads in flight), then added in a fixed order.
template <int L>
__device__ __forceinline__ double sum_parts(const double* __restrict__ GP, int nparts, int e) {
    double a[8] = {0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
    int q = 0;
    for (; q + 8 <= nparts; q += 8)
#pragma unroll
        for (int i = 0; i < 8; ++i) a[i] += __ldg(GP + (int64_t)(q + i) * L * L + e);
    for (; q < nparts; ++q) a[q & 7] += __ldg(GP + (int64_t)q * L * L + e);
    return ((a[0] + a[1]) + (a[2] + a[3])) + ((a[4] + a[5]) + (a[6] + a[7]));
}

// One warp: G = the Gram matrix in block 0 of GP (+ shift * trace / L on the
// diagonal when shift > 0), G = R^T R (upper R, row by row: R[k][j] = (G[k][j]
// - sum_{i<k} R[i][k] R[i][j]) / R[k][k]), Rinv = R^-1 (fp32 out).  Lane l
// owns columns l, l + 32, ..  A pivot at most 1e-20 of G's largest diagonal (a
// column with no norm left) becomes 1 with a zero row of R: that column of
// X R^-1 stays as it is (near zero) instead of being blown up.
template <int L>
__global__ void __launch_bounds__(32)
lr_chol_kernel(const double* __restrict__ GP, double shift, float* __restrict__ Rinv) {
    constexpr int CPL = (L + 31) / 32;                    // columns per lane
    extern __shared__ double lr_dsm[];                    // G, R, Ri: L x (L + 1) each
    auto G = reinterpret_cast<double(*)[L + 1]>(lr_dsm);
    auto R = reinterpret_cast<double(*)[L + 1]>(lr_dsm + L * (L + 1));
    auto Ri = reinterpret_cast<double(*)[L + 1]>(lr_dsm + 2 * L * (L + 1));
    __shared__ double ir[L];                              // 1 / R[k][k]
    const int lane = threadIdx.x;
#pragma unroll 16
    for (int e = lane; e < L * L; e += 32) {              // loads kept in flight
        G[e / L][e % L] = __ldg(GP + e);
        R[e / L][e % L] = 0.0;
    }
    __syncwarp();
    double tr = 0.0, dmax = 0.0;
    for (int i = lane; i < L; i += 32) {
        tr += G[i][i];
        dmax = G[i][i] > dmax ? G[i][i] : dmax;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        tr += __shfl_xor_sync(0xffffffffu, tr, o);
        dmax = fmax(dmax, __shfl_xor_sync(0xffffffffu, dmax, o));
    }
    const double sh = shift * tr / L, thr = 1e-20 * dmax + 1e-300;
    for (int k = 0; k < L; ++k) {
        double sv[CPL];
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            const int j = lane + 32 * c;
            double s0 = 0.0, s1 = 0.0, s2 = 0.0, s3 = 0.0;
            if (j < L && j >= k) {
                int i = 0;
                for (; i + 4 <= k; i += 4) {
                    s0 = fma(R[i][k], R[i][j], s0);
                    s1 = fma(R[i + 1][k], R[i + 1][j], s1);
                    s2 = fma(R[i + 2][k], R[i + 2][j], s2);
                    s3 = fma(R[i + 3][k], R[i + 3][j], s3);
                }
                for (; i < k; ++i) s0 = fma(R[i][k], R[i][j], s0);
            }
            sv[c] = (j < L ? G[k][j] + (j == k ? sh : 0.0) : 0.0) - ((s0 + s1) + (s2 + s3));
        }
        double d = sv[0];
#pragma unroll
        for (int c = 1; c < CPL; ++c)
            if ((k >> 5) == c) d = sv[c];
        d = __shfl_sync(0xffffffffu, d, k & 31);
        const bool live = d > thr;
        const double inv = live ? rsqrt(d) : 1.0, rkk = live ? d * inv : 1.0;
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            const int j = lane + 32 * c;
            if (j < L && j > k) R[k][j] = live ? sv[c] * inv : 0.0;
        }
        if (lane == 0) {
            R[k][k] = rkk;
            ir[k] = inv;
        }
        __syncwarp();
    }
#pragma unroll
    for (int c = 0; c < CPL; ++c) {                       // column j of the upper inverse
        const int j = lane + 32 * c;
        if (j < L) {
            for (int i = L - 1; i > j; --i) Ri[i][j] = 0.0;
            Ri[j][j] = ir[j];
            for (int i = j - 1; i >= 0; --i) {
                double s0 = 0.0, s1 = 0.0;
                int k = i + 1;
                for (; k + 2 <= j + 1; k += 2) {
                    s0 = fma(R[i][k], Ri[k][j], s0);
                    s1 = fma(R[i][k + 1], Ri[k + 1][j], s1);
                }
                if (k <= j) s0 = fma(R[i][k], Ri[k][j], s0);
                Ri[i][j] = -(s0 + s1) * ir[i];
            }
        }
    }
    __syncwarp();
    for (int e = lane; e < L * L; e += 32) Rinv[e] = (float)Ri[e / L][e % L];
}

// out = X[n, L] Rm[L, L] restricted to the first ncols columns; one row per
// thread (in place when out == X: the row is read before it is written).
// trans: out[j * ostride + row], else out[row * ostride + j].
template <int L>
__global__ void __launch_bounds__(kLrThreads)
lr_apply_kernel(const float* X, int64_t n, const float* __restrict__ Rm, int ncols, float* out,
                int64_t ostride, int trans) {
    __shared__ float Rs[L][L];
    for (int e = threadIdx.x; e < L * L; e += kLrThreads) Rs[e / L][e % L] = Rm[e];
    __syncthreads();
    const int64_t row = (int64_t)blockIdx.x * kLrThreads + threadIdx.x;
    if (row >= n) return;
    float x[L];
#pragma unroll
    for (int c = 0; c < L; c += 4) {
        const float4 v = *reinterpret_cast<const float4*>(X + row * L + c);
        x[c] = v.x;
        x[c + 1] = v.y;
        x[c + 2] = v.z;
        x[c + 3] = v.w;
    }
    constexpr int JB = L < 16 ? L : 16;
    // row-major output in whole 16-byte pieces when the rows allow it
    const bool vec = !trans && (ostride & 3) == 0 && (reinterpret_cast<uintptr_t>(out) & 15) == 0;
    for (int j0 = 0; j0 < ncols; j0 += JB) {
        float o[JB];
#pragma unroll
        for (int jj = 0; jj < JB; ++jj) o[jj] = 0.0f;
#pragma unroll
        for (int c = 0; c < L; ++c)
#pragma unroll
            for (int jj = 0; jj < JB; ++jj)
                if (j0 + jj < L) o[jj] = __fmaf_rn(x[c], Rs[c][j0 + jj], o[jj]);
        if (vec && j0 + JB <= ncols) {
#pragma unroll
            for (int jj = 0; jj < JB; jj += 4)
                *reinterpret_cast<float4*>(out + row * ostride + j0 + jj) =
                    make_float4(o[jj], o[jj + 1], o[jj + 2], o[jj + 3]);
        } else {
#pragma unroll
            for (int jj = 0; jj < JB; ++jj) {
                const int j = j0 + jj;
                if (j < ncols) {
                    if (trans) out[(int64_t)j * ostride + row] = o[jj];
                    else out[row * ostride + j] = o[jj];
                }
            }
        }
    }
}

// One CTA: S = sum of the Gram blocks (symmetric L x L), cyclic Jacobi until
// the off-diagonal mass is below 1e-28 of the total (at most 40 sweeps);
// eigenvalues sorted decreasing, sigma = sqrt(max(lambda, 0)).  Writes
// Mr = U_s,r Sigma_r and Mi = U_s,r Sigma_r^-1 (L x L, columns >= rank zero;
// a column whose sigma is at most 1e-7 sigma_1 is zero in Mi) and sigma[rank].
template <int L>
__global__ void __launch_bounds__(kLrThreads)
lr_jacobi_kernel(const double* __restrict__ GP, int nparts, int rank, float* __restrict__ Mr,
                 float* __restrict__ Mi, float* __restrict__ sigma) {
    extern __shared__ double lr_dsm[];                    // A, V: L x (L + 1) each
    auto A = reinterpret_cast<double(*)[L + 1]>(lr_dsm);
    auto V = reinterpret_cast<double(*)[L + 1]>(lr_dsm + L * (L + 1));
    __shared__ double rc[L / 2], rs[L / 2];
    __shared__ int rp[L / 2], rq[L / 2];
    __shared__ double off_rel;
    __shared__ double wsum[kLrThreads / 32][2];
    __shared__ int perm[L];
    __shared__ double sg[L];
    const int t = threadIdx.x;
    for (int e = t; e < L * L; e += kLrThreads) {
        double s = 0.0;
        s = sum_parts<L>(GP, nparts, e);
        A[e / L][e % L] = s;
        V[e / L][e % L] = (e / L == e % L) ? 1.0 : 0.0;
    }
    __syncthreads();
    for (int sweep = 0; sweep < 40; ++sweep) {
        {
            double off = 0.0, tot = 0.0;
            for (int e = t; e < L * L; e += kLrThreads) {
                const int i = e / L, j = e % L;
                const double a2 = A[i][j] * A[i][j];
                tot += a2;
                if (i != j) off += a2;
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                off += __shfl_xor_sync(0xffffffffu, off, o);
                tot += __shfl_xor_sync(0xffffffffu, tot, o);
            }
            if ((t & 31) == 0) {
                wsum[t >> 5][0] = off;
                wsum[t >> 5][1] = tot;
            }
            __syncthreads();
            if (t == 0) {
                double fo = 0.0, ft = 0.0;
                for (int w = 0; w < kLrThreads / 32; ++w) {
                    fo += wsum[w][0];
                    ft += wsum[w][1];
                }
                off_rel = ft > 0.0 ? fo / ft : 0.0;
            }
        }
        __syncthreads();
        if (off_rel < 1e-28) break;
        for (int step = 0; step < L - 1; ++step) {
            if (t < L / 2) {                       // round-robin pairs (circle method)
                const int p = t == 0 ? 0 : ((t - 1 + step) % (L - 1)) + 1;
                const int q = ((L - 2 - t + step) % (L - 1)) + 1;
                const double apq = A[p][q];
                double c = 1.0, s = 0.0;
                if (fabs(apq) > 1e-300) {
                    // t = tan of the rotation angle, the smaller root of
                    // t^2 + 2 tau t - 1 = 0 with tau = (a_qq - a_pp) / (2 a_pq),
                    // written as 2 a_pq sign(dq) / (|dq| + sqrt(dq^2 + 4 a_pq^2))
                    const double dq = A[q][q] - A[p][p];
                    const double tt = (dq >= 0.0 ? 2.0 * apq : -2.0 * apq) /
                                      (fabs(dq) + sqrt(dq * dq + 4.0 * apq * apq));
                    c = rsqrt(1.0 + tt * tt);
                    s = tt * c;
                }
                rp[t] = p;
                rq[t] = q;
                rc[t] = c;
                rs[t] = s;
            }
            __syncthreads();
            for (int e = t; e < (L / 2) * L; e += kLrThreads) {      // rows: A <- J^T A
                const int k = e / L, j = e % L, p = rp[k], q = rq[k];
                const double ap = A[p][j], aq = A[q][j];
                A[p][j] = rc[k] * ap - rs[k] * aq;
                A[q][j] = rs[k] * ap + rc[k] * aq;
            }
            __syncthreads();
            for (int e = t; e < (L / 2) * L; e += kLrThreads) {      // columns: A <- A J, V <- V J
                const int k = e / L, j = e % L, p = rp[k], q = rq[k];
                const double ap = A[j][p], aq = A[j][q];
                A[j][p] = rc[k] * ap - rs[k] * aq;
                A[j][q] = rs[k] * ap + rc[k] * aq;
                const double vp = V[j][p], vq = V[j][q];
                V[j][p] = rc[k] * vp - rs[k] * vq;
                V[j][q] = rs[k] * vp + rc[k] * vq;
            }
            __syncthreads();
        }
    }
    if (t == 0) {
        for (int i = 0; i < L; ++i) perm[i] = i;
        for (int i = 0; i < L; ++i) {              // selection sort, decreasing eigenvalue
            int b = i;
            for (int j = i + 1; j < L; ++j)
                if (A[perm[j]][perm[j]] > A[perm[b]][perm[b]]) b = j;
            const int tmp = perm[i];
            perm[i] = perm[b];
            perm[b] = tmp;
        }
        for (int i = 0; i < L; ++i) {
            const double lam = A[perm[i]][perm[i]];
            sg[i] = lam > 0.0 ? sqrt(lam) : 0.0;
        }
    }
    __syncthreads();
    const double floor_sg = 1e-7 * sg[0];
    for (int e = t; e < L * L; e += kLrThreads) {
        const int c = e / L, j = e % L;
        const bool live = j < rank;
        const double u = V[c][perm[j]];
        Mr[e] = live ? (float)(u * sg[j]) : 0.0f;
        Mi[e] = live && sg[j] > floor_sg && sg[j] > 0.0 ? (float)(u / sg[j]) : 0.0f;
    }
    if (t < rank) sigma[t] = (float)sg[t];
}

constexpr int64_t kGramRows = 128;                 // rows per Gram block

int64_t align256(int64_t b) { return (b + 255) & ~(int64_t)255; }

// Splits of a product's reduction dimension: enough CTAs for about two per SM
// of a 148-SM part (a fixed rule, so that the workspace size does not depend
// on the device).
int64_t splits_for(int64_t tiles) {
    int64_t s = (296 + tiles - 1) / tiles;
    return s < 1 ? 1 : s > 16 ? 16 : s;
}
int64_t right_splits(int64_t N) { return splits_for((N + 63) / 64); }
int64_t left_splits(int64_t K) { return splits_for((K + 63) / 64); }

struct LrWorkspace {
    float *Y, *Z, *P, *R, *Mr, *Mi;            // P: split partials of either product
    double* GP;
};

int64_t partial_floats(int64_t N, int64_t K, int L) {
    const int64_t sr = right_splits(N), sl = left_splits(K);
    const int64_t a = sr > 1 ? sr * N * L : 0, b = sl > 1 ? sl * K * L : 0;
    return a > b ? a : b;
}

LrWorkspace carve(void* ws, int64_t N, int64_t K, int L) {
    uint8_t* b = static_cast<uint8_t*>(ws);
    LrWorkspace w;
    w.Y = reinterpret_cast<float*>(b);
    b += align256(N * L * 4);
    w.Z = reinterpret_cast<float*>(b);
    b += align256(K * L * 4);
    w.P = reinterpret_cast<float*>(b);
    b += align256(partial_floats(N, K, L) * 4);
    w.GP = reinterpret_cast<double*>(b);
    const int64_t parts = ((N > K ? N : K) + kGramRows - 1) / kGramRows;
    b += align256(parts * (int64_t)L * L * 8);
    w.R = reinterpret_cast<float*>(b);
    b += align256((int64_t)L * L * 4);
    w.Mr = reinterpret_cast<float*>(b);
    b += align256((int64_t)L * L * 4);
    w.Mi = reinterpret_cast<float*>(b);
    return w;
}

template <int NBITS, int L>
cudaError_t run(const LrParams& p, int rank, int power_iters, const float* omega, float* B,
                float* A, float* sigma, void* ws, cudaStream_t st) {
    const LrWorkspace w = carve(ws, p.N, p.K, L);
    constexpr int kCholSmem = 3 * L * (L + 1) * 8, kJacobiSmem = 2 * L * (L + 1) * 8;
    cudaError_t e = cudaFuncSetAttribute(lr_chol_kernel<L>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kCholSmem);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(lr_jacobi_kernel<L>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kJacobiSmem);
    if (e != cudaSuccess) return e;
    constexpr int kRightSmem = prod_smem<L, 68>(), kLeftSmem = prod_smem<L, 72>();
    e = cudaFuncSetAttribute(lr_right_kernel<NBITS, L>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, kRightSmem);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(lr_left_kernel<NBITS, L>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, kLeftSmem);
    if (e != cudaSuccess) return e;
    const int64_t SR = right_splits(p.N), SL = left_splits(p.K);
    const int64_t ktiles = (p.K + kLrTile - 1) / kLrTile;
    const int64_t tps = (ktiles + SR - 1) / SR;                 // k-tiles per right split
    const int64_t rps = ((p.N + SL - 1) / SL + kLrTile - 1) / kLrTile * kLrTile;   // rows per left split
    auto right = [&](const float* M) {
        lr_right_kernel<NBITS, L><<<dim3((unsigned)((p.N + 63) / 64), (unsigned)SR), kLrThreads,
                                    kRightSmem, st>>>(p, M, SR > 1 ? w.P : w.Y, tps);
        if (SR > 1) lr_reduce_kernel<<<592, kLrThreads, 0, st>>>(w.P, (int)SR, p.N * L, w.Y);
    };
    auto left = [&]() {
        lr_left_kernel<NBITS, L><<<dim3((unsigned)((p.K + 63) / 64), (unsigned)SL), kLrThreads,
                                   kLeftSmem, st>>>(p, w.Y, SL > 1 ? w.P : w.Z, rps);
        if (SL > 1) lr_reduce_kernel<<<592, kLrThreads, 0, st>>>(w.P, (int)SL, p.K * L, w.Z);
    };
    // X^T X into block 0 of w.GP: Gram blocks of at least kGramRows rows, about
    // one per SM of a 148-SM part (never more blocks than the workspace holds),
    // then their fixed-order sum
    auto gram = [&](const float* X, int64_t n) {
        int64_t rpb = ((n + 147) / 148 + 31) / 32 * 32;
        rpb = rpb < kGramRows ? kGramRows : rpb;
        const int64_t parts = (n + rpb - 1) / rpb;
        lr_gram_kernel<L><<<(unsigned)parts, kLrThreads, 0, st>>>(X, n, rpb, w.GP);
        if (parts > 1) lr_gsum_kernel<L><<<L * L / 32, kLrThreads, 0, st>>>(w.GP, (int)parts);
    };
    auto orth = [&](float* X, int64_t n) {
        for (int pass = 0; pass < 3; ++pass) {
            gram(X, n);
            lr_chol_kernel<L><<<1, 32, kCholSmem, st>>>(w.GP, pass == 0 ? 1e-9 : 0.0, w.R);
            lr_apply_kernel<L><<<(unsigned)((n + kLrThreads - 1) / kLrThreads), kLrThreads, 0, st>>>(
                X, n, w.R, L, X, L, 0);
        }
    };
    right(omega);
    orth(w.Y, p.N);
    for (int it = 0; it < power_iters; ++it) {
        left();
        orth(w.Z, p.K);
        right(w.Z);
        orth(w.Y, p.N);
    }
    left();
    gram(w.Z, p.K);
    lr_jacobi_kernel<L><<<1, kLrThreads, kJacobiSmem, st>>>(w.GP, 1, rank, w.Mr, w.Mi, sigma);
    lr_apply_kernel<L><<<(unsigned)((p.N + kLrThreads - 1) / kLrThreads), kLrThreads, 0, st>>>(
        w.Y, p.N, w.Mr, rank, B, rank, 0);
    lr_apply_kernel<L><<<(unsigned)((p.K + kLrThreads - 1) / kLrThreads), kLrThreads, 0, st>>>(
        w.Z, p.K, w.Mi, rank, A, p.K, 1);
    return cudaGetLastError();
}

template <int NBITS>
cudaError_t run_l(const LrParams& p, int rank, int sketch, int power_iters, const float* omega,
                  float* B, float* A, float* sigma, void* ws, cudaStream_t st) {
    switch (sketch) {
        case 16: return run<NBITS, 16>(p, rank, power_iters, omega, B, A, sigma, ws, st);
        case 32: return run<NBITS, 32>(p, rank, power_iters, omega, B, A, sigma, ws, st);
        case 64: return run<NBITS, 64>(p, rank, power_iters, omega, B, A, sigma, ws, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

// Bytes of workspace the low-rank residual needs for an N x K matrix and a
// sketch of l columns (the last 256 bytes hold sigma when the caller gives none).
int64_t lowrank_workspace_bytes(int64_t N, int64_t K, int sketch) {
    const int64_t L = sketch;
    const int64_t parts = ((N > K ? N : K) + kGramRows - 1) / kGramRows;
    return align256(N * L * 4) + align256(K * L * 4) + align256(partial_floats(N, K, sketch) * 4) +
           align256(parts * L * L * 8) + 3 * align256(L * L * 4) + 256;   // + sigma slot
}

cudaError_t launch_lowrank(const void* W, const uint8_t* packed, const __half* scale,
                           const __half* zero, int64_t N, int64_t K, int nbits, int log2_group,
                           int rank, int sketch, int power_iters, const float* omega, float* B,
                           float* A, float* sigma, void* ws, cudaStream_t st) {
    LrParams p;
    p.W = static_cast<const __half*>(W);
    p.packed = packed;
    p.scale = scale;
    p.zero = zero;
    p.N = N;
    p.K = K;
    p.log2_group = log2_group;
    switch (nbits) {
        case 1: return run_l<1>(p, rank, sketch, power_iters, omega, B, A, sigma, ws, st);
        case 2: return run_l<2>(p, rank, sketch, power_iters, omega, B, A, sigma, ws, st);
        case 3: return run_l<3>(p, rank, sketch, power_iters, omega, B, A, sigma, ws, st);
        case 4: return run_l<4>(p, rank, sketch, power_iters, omega, B, A, sigma, ws, st);
        case 8: return run_l<8>(p, rank, sketch, power_iters, omega, B, A, sigma, ws, st);
        default: return cudaErrorInvalidValue;
    }
}

// Fixed device scratch for callers that cannot allocate device memory (see
// hqq_lowrank_noalloc in hqq.h): 16 MiB in every GPU's copy of this module,
// held until the process exits.  Nothing in it needs to start at zero (every
// part is written before it is read), and every call shares it.
constexpr int64_t kLowrankScratchBytes = (int64_t)16 << 20;
static __device__ __align__(256) uint8_t g_lowrank_scratch[kLowrankScratchBytes];

int64_t lowrank_scratch_bytes() { return kLowrankScratchBytes; }

// Id of the calling thread's current CUDA context (the driver's cuCtxGetId:
// unique for the life of the process, so a context created after a
// cudaDeviceReset, or a second context on the same device, has a new one).
// The two driver calls are looked up once through the runtime.
static bool current_context_id(unsigned long long* id) {
    using GetCurrentFn = CUresult (*)(CUcontext*);
    using GetIdFn = CUresult (*)(CUcontext, unsigned long long*);
    static const auto fns = [] {
        void* a = nullptr;
        void* b = nullptr;
        cudaDriverEntryPointQueryResult qa, qb;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) != cudaSuccess ||
            qa != cudaDriverEntryPointSuccess)
            a = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) != cudaSuccess ||
            qb != cudaDriverEntryPointSuccess)
            b = nullptr;
        cudaGetLastError();                    // a failed lookup leaves no error behind
        return std::make_pair(reinterpret_cast<GetCurrentFn>(a), reinterpret_cast<GetIdFn>(b));
    }();
    if (!fns.first || !fns.second) return false;
    CUcontext ctx = nullptr;
    if (fns.first(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
    return fns.second(ctx, id) == CUDA_SUCCESS;
}

// The device address of the scratch array in the current context, looked up
// (with that context current) on the first call and whenever the current
// context differs from the one the cached address belongs to; host code can
// only name the array's host-side stand-in, which is not a device address.
// Without the driver's context id the address is looked up on every call.
cudaError_t lowrank_scratch(void** ptr) {
    constexpr int kMaxDevices = 64;
    struct Entry {
        unsigned long long ctx;
        void* addr;
    };
    static std::mutex mu;
    static Entry cached[kMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    unsigned long long ctx = 0;
    const bool have_id = current_context_id(&ctx);
    std::lock_guard<std::mutex> lock(mu);
    if (have_id && cached[dev].addr && cached[dev].ctx == ctx) {
        *ptr = cached[dev].addr;
        return cudaSuccess;
    }
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_lowrank_scratch);   // makes the runtime's context current
    if (e != cudaSuccess) return e;
    unsigned long long now = 0;
    cached[dev] = current_context_id(&now) ? Entry{now, p} : Entry{0ull, nullptr};
    *ptr = p;
    return cudaSuccess;
}

}  // namespace hqq
