// hqq_quantize.cu -- fused HQQ solver + code packing kernel (sm_100a).
//
// "Half-Quadratic Quantization of Large Machine Learning Models", section 2
// (Q, Q^-1, l_p error, sp1 shrink, sp2 mean, beta <- kappa beta, 1/s held) and
// section 4.1 (solver parameters, early exit when the error stops improving).
//
// Layout: a group of G weights is held by a sub-warp of K = G/8 lanes, each
// lane owning 8 consecutive weights loaded with one 128-bit load, so a warp
// holds 256 consecutive weights (32/K groups) and a CTA of 10 warps a tile of
// 2560 weights -- five whole groups of any size at the 3-bit layout's 10 codes
// per word, so every packed word of a tile is written by exactly one thread.
// All solver state lives in registers; group sums are the pairwise sum over
// contiguous halves (8 in-lane, then xor-shuffles 1, 2, .. K/2).  Every
// sub-warp stops on its own; the warp iterates while any of its groups runs.
#include "hqq_common.cuh"

namespace hqq {

constexpr int kQuantThreads = 320;
constexpr int kTileElems = kQuantThreads * 8;   // 2560
constexpr unsigned kFull = 0xFFFFFFFFu;

template <int K>
__device__ __forceinline__ float group_sum(float v) {
#pragma unroll
    for (int o = 1; o < K; o <<= 1) v = __fadd_rn(v, __shfl_xor_sync(kFull, v, o));
    return v;
}

template <int K>
__device__ __forceinline__ float group_min(float v) {
#pragma unroll
    for (int o = 1; o < K; o <<= 1) v = fminf(v, __shfl_xor_sync(kFull, v, o));
    return v;
}

template <int K>
__device__ __forceinline__ float group_max(float v) {
#pragma unroll
    for (int o = 1; o < K; o <<= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
    return v;
}

__device__ __forceinline__ float sum8(const float (&x)[8]) {
    return __fadd_rn(__fadd_rn(__fadd_rn(x[0], x[1]), __fadd_rn(x[2], x[3])),
                     __fadd_rn(__fadd_rn(x[4], x[5]), __fadd_rn(x[6], x[7])));
}

// clamp(round(v), 0, L) with round half to even; returns the code as a float
// and its integer value.
template <int L>
__device__ __forceinline__ float code_of(float v, uint32_t& ci) {
    v = fminf(fmaxf(v, 0.0f), (float)L);
    const float t = __fadd_rn(v, kRoundShift);
    ci = __float_as_uint(t) & 0xFFu;
    return __fsub_rn(t, kRoundShift);
}

__device__ __forceinline__ void load_table(float* dst, const PowTable& t) {
    for (int i = threadIdx.x; i < kTabFloats; i += blockDim.x)
        dst[i] = i < 256 ? t.two_pk[i] : (i < 288 ? t.cj_p[i - 256] : t.inv_cj[i - 288]);
}

template <int NBITS, int G>
__global__ void __launch_bounds__(kQuantThreads, 2)
quantize_kernel(const __grid_constant__ QuantParams prm) {
    constexpr int K = G / 8;              // lanes per group
    constexpr int GPW = 32 / K;           // groups per warp
    constexpr int GPC = GPW * (kQuantThreads / 32);
    constexpr int L = (1 << NBITS) - 1;
    constexpr float kInvG = 1.0f / (float)G;

    __shared__ float s_tp[kTabFloats];
    __shared__ float s_tq[kTabFloats];
    __shared__ float s_thr[kMaxIters];
    __shared__ __align__(16) uint8_t s_codes[NBITS == 3 ? kTileElems : 16];

    load_table(s_tp, prm.tp);
    load_table(s_tq, prm.tq);
    for (int i = threadIdx.x; i < prm.iters; i += blockDim.x) s_thr[i] = prm.shrink_thr[i];
    __syncthreads();

    const float pa1 = prm.tp.a1, pa2 = prm.tp.a2, pa3 = prm.tp.a3;
    const float qa1 = prm.tq.a1, qa2 = prm.tq.a2, qa3 = prm.tq.a3;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int kl = lane % K;
    const int64_t n_tiles = (prm.n_groups + GPC - 1) / GPC;

    for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
        const int64_t g = tile * GPC + warp * GPW + lane / K;
        const bool valid = g < prm.n_groups;

        // ---- load 8 fp16 weights (one 128-bit load) ------------------------------
        float w[8];
        {
            uint4 raw = make_uint4(0u, 0u, 0u, 0u);
            if (valid) raw = __ldg(reinterpret_cast<const uint4*>(prm.W + g * G + kl * 8));
            const uint32_t r4[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&r4[k]));
                w[2 * k] = f.x;
                w[2 * k + 1] = f.y;
            }
        }

        // ---- min-max initialisation ---------------------------------------------
        float mn = w[0], mx = w[0];
#pragma unroll
        for (int i = 1; i < 8; ++i) {
            mn = fminf(mn, w[i]);
            mx = fmaxf(mx, w[i]);
        }
        mn = group_min<K>(mn);
        mx = group_max<K>(mx);
        const float rng = __fsub_rn(mx, mn);
        float s = 1.0f, inv = 1.0f;
        if (rng != 0.0f) {
            s = __fdiv_rn(rng, (float)L);
            inv = __fdiv_rn(1.0f, s);
        }
        float z = -__fmul_rn(mn, inv);
        float zb = z, eb = __int_as_float(0x7F800000);   // +inf
        float bt = prm.beta;
        int accepted = 0;
        bool active = valid;

        // ---- half-quadratic iterations -------------------------------------------
        for (int t = 0; t < prm.iters; ++t) {
            if (!__any_sync(kFull, active)) break;
            float q[8], d[8], pw[8], tm[8];
            float amax = 0.0f;
            uint32_t ci;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                q[i] = code_of<L>(__fmaf_rn(w[i], inv, z), ci);
                d[i] = __fmaf_rn(__fsub_rn(z, q[i]), s, w[i]);
                const float a = fabsf(d[i]);
                amax = fmaxf(amax, a);
                pw[i] = powp(s_tp, pa1, pa2, pa3, a);
                tm[i] = __fmaf_rn(-w[i], inv, q[i]);     // sp2 term when W_e == 0
            }
            const float e = group_sum<K>(sum8(pw));
            const bool acc = active && (e < eb);
            if (acc) {
                eb = e;
                zb = z;
                ++accepted;
            }
            active = acc;
            // sp1: W_e is exactly zero unless some |r| exceeds the threshold
            if (__any_sync(kFull, active && amax > s_thr[t])) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float a = fabsf(d[i]);
                    const float y = __fsub_rn(a, __fdiv_rn(powp(s_tq, qa1, qa2, qa3, a), bt));
                    const float we = copysignf(fmaxf(y, 0.0f), d[i]);
                    tm[i] = __fmaf_rn(-__fsub_rn(w[i], we), inv, q[i]);
                }
            }
            const float zs = group_sum<K>(sum8(tm));
            if (active) z = __fmul_rn(zs, kInvG);
            bt = __fmul_rn(bt, prm.kappa);
        }

        // ---- final codes, packing and stores ---------------------------------------
        uint32_t c[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) code_of<L>(__fmaf_rn(w[i], inv, zb), c[i]);

        const int64_t chunk = tile * (kTileElems / 8) + threadIdx.x;   // 8-weight chunk id
        if constexpr (NBITS == 4) {
            uint32_t word = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) word |= c[i] << (4 * i);
            if (valid) reinterpret_cast<uint32_t*>(prm.packed)[chunk] = word;
        } else if constexpr (NBITS == 2) {
            uint32_t h = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) h |= c[i] << (2 * i);
            if (valid) reinterpret_cast<uint16_t*>(prm.packed)[chunk] = (uint16_t)h;
        } else {
            uint2 b;
            b.x = c[0] | (c[1] << 8) | (c[2] << 16) | (c[3] << 24);
            b.y = c[4] | (c[5] << 8) | (c[6] << 16) | (c[7] << 24);
            reinterpret_cast<uint2*>(s_codes)[threadIdx.x] = b;   // zeros when !valid
            __syncthreads();
            if (threadIdx.x < kTileElems / 10) {
                const int64_t word_id = tile * (kTileElems / 10) + threadIdx.x;
                const int64_t n_words = (prm.n_elems + 9) / 10;
                const uint16_t* src = reinterpret_cast<const uint16_t*>(s_codes) + threadIdx.x * 5;
                uint32_t word = 0;
#pragma unroll
                for (int k = 0; k < 5; ++k) {
                    const uint32_t two = src[k];
                    word |= ((two & 0xFFu) | ((two >> 8) << 3)) << (6 * k);
                }
                if (word_id < n_words) reinterpret_cast<uint32_t*>(prm.packed)[word_id] = word;
            }
            __syncthreads();
        }
        if (valid && kl == 0) {
            prm.scale[g] = __float2half_rn(s);
            prm.zero[g] = __float2half_rn(zb);
            if (prm.zero_f32) prm.zero_f32[g] = zb;
            if (prm.iters_out) prm.iters_out[g] = (uint8_t)accepted;
        }
    }
}

template <int NBITS, int G>
static cudaError_t launch_quantize_g(const QuantParams& prm, cudaStream_t stream) {
    constexpr int GPC = (32 / (G / 8)) * (kQuantThreads / 32);
    const int64_t tiles = (prm.n_groups + GPC - 1) / GPC;
    const unsigned grid = (unsigned)(tiles < (1 << 30) ? tiles : (1 << 30));
    quantize_kernel<NBITS, G><<<grid, kQuantThreads, 0, stream>>>(prm);
    return cudaGetLastError();
}

template <int NBITS>
static cudaError_t launch_quantize_b(const QuantParams& prm, int group, cudaStream_t stream) {
    switch (group) {
        case 16: return launch_quantize_g<NBITS, 16>(prm, stream);
        case 32: return launch_quantize_g<NBITS, 32>(prm, stream);
        case 64: return launch_quantize_g<NBITS, 64>(prm, stream);
        case 128: return launch_quantize_g<NBITS, 128>(prm, stream);
        case 256: return launch_quantize_g<NBITS, 256>(prm, stream);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_quantize(const QuantParams& prm, int nbits, int group, cudaStream_t stream) {
    switch (nbits) {
        case 2: return launch_quantize_b<2>(prm, group, stream);
        case 3: return launch_quantize_b<3>(prm, group, stream);
        case 4: return launch_quantize_b<4>(prm, group, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace hqq
