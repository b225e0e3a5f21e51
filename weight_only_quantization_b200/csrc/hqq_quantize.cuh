// hqq_quantize.cuh -- fused HQQ solver + code packing kernel (sm_100a),
// instantiated in single precision by hqq_quantize.cu and in half precision by
// hqq_quantize_half.cu.
//
// "Half-Quadratic Quantization of Large Machine Learning Models", section 2
// (Q, Q^-1, l_p error, sp1 shrink, sp2 mean, beta <- kappa beta, 1/s held) and
// section 4.1 (solver parameters, early exit when the error stops improving).
//
// Work decomposition (persistent warps):
//  * A group of G weights is held by a sub-warp of K = G/(8 NB) lanes, each lane
//    owning NB blocks of 8 consecutive weights.  Within a block the weights sit
//    in f32x2 register pairs (x_k, x_k+4), k = 0..3, for the packed element-wise
//    arithmetic; the pairwise sum over contiguous halves then reads the halves
//    with scalar adds, and lane sums are combined by xor-shuffles 1, 2, .., K/2
//    (same pairwise order).
//  * Each warp owns chunks of 2560 consecutive weights (five groups of any size
//    fill whole 3-bit words), staged once into the warp's shared memory.
//  * Phase A: every group of the chunk is initialised and runs its first two
//    error evaluations in lock-step -- every group needs at least two, so no
//    lane idles.  Groups that stop are finalised; the others are queued with
//    their state in shared memory.
//  * Phase B: each sub-warp pulls queued groups, iterates until its group stops,
//    finalises it and pulls the next, so the early-stop divergence costs almost
//    nothing.  No block-wide barrier is ever taken after start-up.
//  * Two exact shortcuts, both tested per group and per step: when
//    fma(min, 1/s, z) >= -1/2 and fma(max, 1/s, z) < L + 1/2 no code can leave
//    [0, L] (fma is monotone in the weight), so the clamp is skipped; when a
//    bound on |W - Q^-1(Q(W))| lies below the shrink threshold, W_e is exactly
//    zero, so sp1 reduces to W - W_e = W.
#pragma once
#include <cmath>
#include <type_traits>

#include "hqq_common.cuh"

namespace hqq {

// Warps per CTA (they share the power tables): 8 in each of two CTAs per SM
// (up to 128 registers per thread), or 20 in one CTA per SM at 96 registers
// (no spills in single precision, a few bytes in half precision).  3-bit
// 28672 x 8192, single precision: 20 warps 0.90 ms, 2 x 8 warps 0.98 ms,
// 1 x 16 warps 0.94 ms, 2 x 10 warps 0.94 ms, 22 warps (88 registers)
// 1.01 ms, 24 warps (80 registers) 0.92 ms; half precision: 20 warps
// 1.21 ms, 2 x 8 warps 1.42 ms.
constexpr int kWideWarps = 20;
constexpr int kChunk = 2560;               // weights per warp chunk
constexpr unsigned kFull = 0xFFFFFFFFu;

template <int NBITS, int G, int NB>
struct QCfg {
    static constexpr int EPL = 8 * NB;           // weights per lane
    static constexpr int K = G / EPL;            // lanes per group
    static constexpr int GPW = 32 / K;           // groups per warp round
    static constexpr int ROUND = 32 * EPL;       // weights per warp round
    static constexpr int ROUNDS = kChunk / ROUND;
    static constexpr int CG = kChunk / G;        // groups per chunk
    static constexpr int L = (1 << NBITS) - 1;
    static constexpr int W_BYTES = kChunk * 2;
    static constexpr int ST_BYTES = CG * 16;     // (z, zb, eb, s) per group
    static constexpr int ST2_BYTES = CG * 16;    // (1/s, min, max, t << 16 | accepted)
    static constexpr int Q_BYTES = (CG + 15) / 16 * 16;
    static constexpr int SLOTS = GPW;            // phase-B slots per warp (this layout)
    static constexpr int POOL_W_BYTES = SLOTS * G * 2;
    static constexpr int POOL_ST_BYTES = SLOTS * 32;
    static constexpr int POOL_GI_BYTES = (SLOTS * 8 + 15) / 16 * 16;
    static constexpr int CHUNK_BYTES = W_BYTES + ST_BYTES + ST2_BYTES + Q_BYTES;
    static constexpr int POOL_BYTES = POOL_W_BYTES + POOL_ST_BYTES + POOL_GI_BYTES;
    // every region starts on a 16-byte boundary (128-bit shared-memory accesses)
    static_assert(W_BYTES % 16 == 0 && ST_BYTES % 16 == 0 && ST2_BYTES % 16 == 0 &&
                  Q_BYTES % 16 == 0 && POOL_W_BYTES % 16 == 0 && POOL_ST_BYTES % 16 == 0 &&
                  POOL_GI_BYTES % 16 == 0, "shared-memory regions must be 16-byte multiples");
    static_assert(K >= 1 && K <= 32 && kChunk % ROUND == 0, "bad layout");
};

// TAB2: the hot |x|^p uses the combined 32 KiB exponent x cell table (one
// lookup fewer); otherwise the separate small tables (less shared memory).
template <bool TAB2, bool HALF>
struct QuantSmem {
    std::conditional_t<TAB2, PowSmem2, PowSmem> tp;   // |x|^p
    PowSmem tq;                 // |x|^(p-1)
    float beta[kMaxIters + 1];  // beta_t = beta * kappa^t by repeated binary32 products
    float thr[kMaxIters + 1];   // shrink thresholds
    float thr16[HALF ? kMaxIters + 1 : 1];   // the same for the half-precision shrink
};

template <int K>
__device__ __forceinline__ float2 group_sum2(float2 v) {
#pragma unroll
    for (int o = 1; o < K; o <<= 1) {
        const float ux = __shfl_xor_sync(kFull, v.x, o), uy = __shfl_xor_sync(kFull, v.y, o);
        v = make_float2(__fadd_rn(v.x, ux), __fadd_rn(v.y, uy));
    }
    return v;
}

template <int K>
__device__ __forceinline__ void group_minmax(float& mn, float& mx) {
#pragma unroll
    for (int o = 1; o < K; o <<= 1) {
        mn = fminf(mn, __shfl_xor_sync(kFull, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, o));
    }
}

// NB blocks of 8 fp16 weights -> pairs (x_k, x_k+4) of each block.
template <int NB>
__device__ __forceinline__ void load_lane(const __half* src, float2 (&w)[NB][4]) {
#pragma unroll
    for (int b = 0; b < NB; ++b) {
        const uint4 raw = reinterpret_cast<const uint4*>(src)[b];
        const __half2 h01 = *reinterpret_cast<const __half2*>(&raw.x);
        const __half2 h23 = *reinterpret_cast<const __half2*>(&raw.y);
        const __half2 h45 = *reinterpret_cast<const __half2*>(&raw.z);
        const __half2 h67 = *reinterpret_cast<const __half2*>(&raw.w);
        w[b][0] = make_float2(__low2float(h01), __low2float(h45));
        w[b][1] = make_float2(__high2float(h01), __high2float(h45));
        w[b][2] = make_float2(__low2float(h23), __low2float(h67));
        w[b][3] = make_float2(__high2float(h23), __high2float(h67));
    }
}

// load_lane plus the lane's min and max, taken on the packed fp16 values
// (exact: the conversion to binary32 is exact and monotone).
template <int NB>
__device__ __forceinline__ void load_lane_minmax(const __half* src, float2 (&w)[NB][4],
                                                 float& mn, float& mx) {
    __half2 hmn, hmx;
#pragma unroll
    for (int b = 0; b < NB; ++b) {
        const uint4 raw = reinterpret_cast<const uint4*>(src)[b];
        const __half2 h01 = *reinterpret_cast<const __half2*>(&raw.x);
        const __half2 h23 = *reinterpret_cast<const __half2*>(&raw.y);
        const __half2 h45 = *reinterpret_cast<const __half2*>(&raw.z);
        const __half2 h67 = *reinterpret_cast<const __half2*>(&raw.w);
        const __half2 bmn = __hmin2(__hmin2(h01, h23), __hmin2(h45, h67));
        const __half2 bmx = __hmax2(__hmax2(h01, h23), __hmax2(h45, h67));
        hmn = b == 0 ? bmn : __hmin2(hmn, bmn);
        hmx = b == 0 ? bmx : __hmax2(hmx, bmx);
        w[b][0] = make_float2(__low2float(h01), __low2float(h45));
        w[b][1] = make_float2(__high2float(h01), __high2float(h45));
        w[b][2] = make_float2(__low2float(h23), __low2float(h67));
        w[b][3] = make_float2(__high2float(h23), __high2float(h67));
    }
    mn = fminf(__low2float(hmn), __high2float(hmn));
    mx = fmaxf(__low2float(hmx), __high2float(hmx));
}

// Pairwise sum ((x0+x1)+(x2+x3)) + ((x4+x5)+(x6+x7)) of one block of 8 values
// held as pairs (x_k, x_k+4).  The pair halves are read one by one with scalar
// adds: packed f32x2 adds of these pairs were found, twice, to give error sums
// one unit off the canonical order in some groups on this toolchain, so no
// packed add is used for a reduction.
__device__ __forceinline__ float block_sum8(const float2 (&v)[4]) {
    return __fadd_rn(__fadd_rn(__fadd_rn(v[0].x, v[1].x), __fadd_rn(v[2].x, v[3].x)),
                     __fadd_rn(__fadd_rn(v[0].y, v[1].y), __fadd_rn(v[2].y, v[3].y)));
}

// Per-group constants of one evaluation, as f32x2 pairs.
struct EvalConst {
    float2 z, nz, ns, inv, ninv;
    float s, invs;
};

// One error evaluation of the lane's weights at zero-point z.  Returns the
// lane's pairwise sums of (|r|^p, sp2 term) where r = W - s(Wq - z) and the sp2
// term is Wq - (W - W_e)/s.  CLAMP: codes may leave [0, L].  SHRINK: W_e is
// evaluated exactly; otherwise W_e is known to be zero.
template <int L, int NB, bool CLAMP, bool SHRINK, class SM>
__device__ __forceinline__ float2 eval_lane(const SM& S, const float2 (&w)[NB][4],
                                            const EvalConst& c, float2 pa1, float2 pa2,
                                            float2 pa3, float qa1, float qa2, float qa3,
                                            float beta) {
    const float2 sh = make_float2(kRoundShift, kRoundShift);
    const float2 nsh = make_float2(-kRoundShift, -kRoundShift);
    float pe = 0.0f, pt = 0.0f;
#pragma unroll
    for (int b = 0; b < NB; ++b) {
        float2 P[4], T[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            float2 v = __ffma2_rn(w[b][k], c.inv, c.z);                // W/s + z
            if (CLAMP) {
                v.x = fminf(fmaxf(v.x, 0.0f), (float)L);
                v.y = fminf(fmaxf(v.y, 0.0f), (float)L);
            }
            const float2 q = __fadd2_rn(__fadd2_rn(v, sh), nsh);      // round half even
            const float2 qz = __fadd2_rn(q, c.nz);                     // Wq - z
            const float2 d = __ffma2_rn(qz, c.ns, w[b][k]);            // W - s(Wq - z)
            P[k] = powp_hot(S.tp, pa1, pa2, pa3, d);
            if (SHRINK) {
                float we[2];
                const float dd[2] = {d.x, d.y};
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const float a = fabsf(dd[e]);
                    const float y = __fsub_rn(a, __fdiv_rn(powp1(S.tq, qa1, qa2, qa3, a), beta));
                    we[e] = copysignf(fmaxf(y, 0.0f), dd[e]);
                }
                T[k].x = __fmaf_rn(-__fsub_rn(w[b][k].x, we[0]), c.invs, q.x);
                T[k].y = __fmaf_rn(-__fsub_rn(w[b][k].y, we[1]), c.invs, q.y);
            } else {
                T[k] = __ffma2_rn(w[b][k], c.ninv, q);                 // Wq - W/s
            }
        }
        const float bp = block_sum8(P), bt = block_sum8(T);
        if (b == 0) {
            pe = bp;
            pt = bt;
        } else {
            pe = __fadd_rn(pe, bp);
            pt = __fadd_rn(pt, bt);
        }
    }
    return make_float2(pe, pt);
}

struct GroupState {
    float z, zb, eb, s, inv, mn, mx;
    int t;    // evaluations done
    int na;   // evaluations accepted
    bool h;   // solved in half precision (s, 1/s, z, errors are fp16 values)
};

// fp16 rounding (nearest even) of a binary32 value, returned as binary32.  For
// a +, -, * or / of fp16 operands formed in binary32, this is the correctly
// rounded fp16 result (24 >= 2 * 11 + 2 bits).
__device__ __forceinline__ float r16(float x) { return __half2float(__float2half_rn(x)); }

// Starting point of a group (section 2 with the min-max start): s, 1/s and z.
// Single precision: s = (max - min)/L, 1/s correctly rounded, z = -min (1/s).
// Half precision (HALF): the same steps, each rounded to fp16, for groups
// inside the fp16 bounds -- max|W| <= 8192, s not rounded to zero and
// max|W| (1/s) <= 2^14 (binary32 product); other groups start (and are
// solved) in single precision.  A constant group has s = 1/s = 1, z = -min.
template <int L, bool HALF>
__device__ __forceinline__ void init_group(GroupState& g, float mn, float mx) {
    g.h = false;
    if constexpr (HALF) {
        const float rng = r16(__fsub_rn(mx, mn));
        if (rng == 0.0f) {
            g.s = 1.0f;
            g.inv = 1.0f;
            g.z = -mn;
            g.h = true;
        } else {
            const float s = r16(__fdiv_rn(rng, (float)L));
            const float inv = r16(__frcp_rn(s));
            const float m = fmaxf(fabsf(mn), fabsf(mx));
            if (m <= 8192.0f && s > 0.0f && __fmul_rn(m, inv) <= 16384.0f) {
                g.s = s;
                g.inv = inv;
                g.z = -r16(__fmul_rn(mn, inv));
                g.h = true;
            }
        }
    }
    if (!g.h) {
        const float rng = __fsub_rn(mx, mn);
        g.s = 1.0f;
        g.inv = 1.0f;
        if (rng != 0.0f) {
            g.s = __fdiv_rn(rng, (float)L);
            g.inv = __frcp_rn(g.s);             // correctly rounded 1/s
        }
        g.z = -__fmul_rn(mn, g.inv);
    }
    g.mn = mn;
    g.mx = mx;
    g.zb = g.z;
    g.eb = __int_as_float(0x7F800000);
    g.t = 0;
    g.na = 0;
}

// Per-group constants of one half-precision evaluation (fp16 pairs).
struct EvalConst16 {
    __half2 z, s, inv;
    float zf, invf;
};

// One error evaluation in half precision: every element-wise step on fp16
// pairs (__hmul2_rn etc.: correctly rounded fp16, never contracted), |d|^p as
// the binary32 table power of the fp16 residual rounded to fp16, and the sums
// in binary32 with the single-precision evaluation's pairwise order.  Returns
// (sum of |d|^p, sum of sp2 terms).  Without SHRINK the sp2 term is
// Wq - fp16(W (1/s)), valid while every |d| <= thr16 (then the exact shrink
// is zero); `above` reports a residual beyond that bound.
template <int L, int NB, bool CLAMP, bool SHRINK, class SM>
__device__ __forceinline__ float2 eval_lane16(const SM& S, const float2 (&w)[NB][4],
                                              const EvalConst16& c, float2 pa1, float2 pa2,
                                              float2 pa3, float qa1, float qa2, float qa3,
                                              float beta, float thr16, bool& above) {
    const __half2 lo = __float2half2_rn(0.0f), hi = __float2half2_rn((float)L);
    float pe = 0.0f, pt = 0.0f;
    bool ab = false;
#pragma unroll
    for (int b = 0; b < NB; ++b) {
        float2 P[4], T[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const __half2 w16 = __floats2half2_rn(w[b][k].x, w[b][k].y);   // exact
            const __half2 u = __hmul2_rn(w16, c.inv);                       // W / s
            __half2 v = __hadd2_rn(u, c.z);
            if (CLAMP) v = __hmin2(__hmax2(v, lo), hi);
            const __half2 q = h2rint(v);                                    // half to even
            const __half2 d = __hsub2_rn(w16, __hmul2_rn(c.s, __hsub2_rn(q, c.z)));
            const float2 d32 = __half22float2(d);
            P[k] = __half22float2(__float22half2_rn(powp_hot(S.tp, pa1, pa2, pa3, d32)));
            if (SHRINK) {
                const float2 q32 = __half22float2(q);
                const float dd[2] = {d32.x, d32.y}, qq[2] = {q32.x, q32.y};
                const float ww[2] = {w[b][k].x, w[b][k].y};
                float tt[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const float a = fabsf(dd[e]);
                    const float r = r16(__fdiv_rn(r16(powp1(S.tq, qa1, qa2, qa3, a)), beta));
                    const float we = copysignf(fmaxf(r16(__fsub_rn(a, r)), 0.0f), dd[e]);
                    tt[e] = r16(__fsub_rn(qq[e], r16(__fmul_rn(r16(__fsub_rn(ww[e], we)), c.invf))));
                }
                T[k] = make_float2(tt[0], tt[1]);
            } else {
                T[k] = __half22float2(__hsub2_rn(q, u));
                ab = ab || fabsf(d32.x) > thr16 || fabsf(d32.y) > thr16;
            }
        }
        const float bp = block_sum8(P), bt = block_sum8(T);
        if (b == 0) {
            pe = bp;
            pt = bt;
        } else {
            pe = __fadd_rn(pe, bp);
            pt = __fadd_rn(pt, bt);
        }
    }
    above = ab;
    return make_float2(pe, pt);
}

// One solver iteration (error evaluation, early-stop test, sp1 + sp2) for the
// sub-warp's group; `live` lanes only change state.  Returns true when the
// group has finished (stopped, or used its iterations).  With HALF, groups
// marked g.h take the half-precision evaluation (error and z as fp16 group
// means), the others the single-precision one.
template <int NBITS, int G, int NB, bool HALF, class SM>
__device__ __forceinline__ bool solver_step(const SM& S, const QuantParams& prm,
                                            const float2 (&w)[NB][4], GroupState& g, bool live,
                                            float2 pa1, float2 pa2, float2 pa3,
                                            float qa1, float qa2, float qa3) {
    using C = QCfg<NBITS, G, NB>;
    constexpr float L = (float)C::L;
    const int t = live ? g.t : 0;
    const float beta = S.beta[t];
    float2 r = make_float2(0.0f, 0.0f);
    if (!HALF || __any_sync(kFull, live && !g.h)) {
        const float vmin = __fmaf_rn(g.mn, g.inv, g.z);
        const float vmax = __fmaf_rn(g.mx, g.inv, g.z);
        const bool inside = vmin >= -0.5f && vmax < L + 0.5f;
        const float reach = fmaxf(0.5f, fmaxf(-vmin, vmax - L)) + 1e-3f * (1.0f + fabsf(g.z));
        const bool shrink = 2.0f * g.s * reach > S.thr[t];
        const bool mine = live && !(HALF && g.h);
        EvalConst c;
        c.z = make_float2(g.z, g.z);
        c.nz = make_float2(-g.z, -g.z);
        c.ns = make_float2(-g.s, -g.s);
        c.inv = make_float2(g.inv, g.inv);
        c.ninv = make_float2(-g.inv, -g.inv);
        c.s = g.s;
        c.invs = g.inv;
        if (__any_sync(kFull, mine && shrink))
            r = eval_lane<C::L, NB, true, true>(S, w, c, pa1, pa2, pa3, qa1, qa2, qa3, beta);
        else if (__all_sync(kFull, !mine || inside))
            r = eval_lane<C::L, NB, false, false>(S, w, c, pa1, pa2, pa3, qa1, qa2, qa3, beta);
        else
            r = eval_lane<C::L, NB, true, false>(S, w, c, pa1, pa2, pa3, qa1, qa2, qa3, beta);
    }
    if constexpr (HALF) {
        if (__any_sync(kFull, live && g.h)) {
            const bool mine = live && g.h;
            // fp16 Q is monotone in W: the group's extreme codes bound all others
            const float vmin = r16(__fadd_rn(r16(__fmul_rn(g.mn, g.inv)), g.z));
            const float vmax = r16(__fadd_rn(r16(__fmul_rn(g.mx, g.inv)), g.z));
            const bool inside = vmin >= -0.5f && vmax < L + 0.5f;
            EvalConst16 c;
            c.z = __float2half2_rn(g.z);
            c.s = __float2half2_rn(g.s);
            c.inv = __float2half2_rn(g.inv);
            c.zf = g.z;
            c.invf = g.inv;
            const float thr = S.thr16[t];
            bool above = false;
            float2 r16v;
            if (__all_sync(kFull, !mine || inside))
                r16v = eval_lane16<C::L, NB, false, false>(S, w, c, pa1, pa2, pa3, qa1, qa2, qa3,
                                                           beta, thr, above);
            else
                r16v = eval_lane16<C::L, NB, true, false>(S, w, c, pa1, pa2, pa3, qa1, qa2, qa3,
                                                          beta, thr, above);
            if (__any_sync(kFull, mine && above))
                r16v = eval_lane16<C::L, NB, true, true>(S, w, c, pa1, pa2, pa3, qa1, qa2, qa3,
                                                         beta, thr, above);
            if (g.h) r = r16v;
        }
    }
    r = group_sum2<C::K>(r);                       // (error, sp2 sum) of the whole group
    float e = r.x, zn = __fmul_rn(r.y, 1.0f / (float)G);
    if (HALF && g.h) {                             // fp16 group means
        e = r16(__fmul_rn(r.x, 1.0f / (float)G));
        zn = r16(zn);
    }
    const bool acc = live && e < g.eb;
    bool repeat = false;
    if (acc) {
        // the update reproduced the z just evaluated: the next evaluation would
        // repeat this one exactly, its error would not fall, and the group would
        // stop with the same best z -- so it stops now (identical outputs)
        repeat = zn == g.z;
        g.eb = e;
        g.zb = g.z;
        g.z = zn;
        ++g.na;
    }
    if (live) ++g.t;
    return live && (!acc || repeat || g.t == prm.iters);
}

// Group state kept in the chunk's shared memory between phases.
constexpr int kHalfBit = 1 << 29;   // flag in the packed (t, accepted) word

__device__ __forceinline__ void save_state(float4* st, float4* st2, int gl, const GroupState& g) {
    st[gl] = make_float4(g.z, g.zb, g.eb, g.s);
    st2[gl] = make_float4(g.inv, g.mn, g.mx,
                          __int_as_float((g.t << 16) | g.na | (g.h ? kHalfBit : 0)));
}

__device__ __forceinline__ void load_state(const float4* st, const float4* st2, int gl,
                                           GroupState& g) {
    const float4 a = st[gl];
    const float4 b = st2[gl];
    g.z = a.x;
    g.zb = a.y;
    g.eb = a.z;
    g.s = a.w;
    g.inv = b.x;
    g.mn = b.y;
    g.mx = b.z;
    const int tn = __float_as_int(b.w);
    g.t = (tn >> 16) & 0xFF;
    g.na = tn & 0xFFFF;
    g.h = (tn & kHalfBit) != 0;
}

constexpr int kCarried = 1 << 30;   // flag in the packed (t, accepted) word
constexpr int kPoolTag = 256;       // queue handles >= kPoolTag name pool entries

// Pack the lane's weights back to fp16 in memory order (exact: they came from fp16).
template <int NB>
__device__ __forceinline__ void store_lane(__half* dst, const float2 (&w)[NB][4]) {
#pragma unroll
    for (int b = 0; b < NB; ++b) {
        const __half2 h01 = __floats2half2_rn(w[b][0].x, w[b][1].x);
        const __half2 h23 = __floats2half2_rn(w[b][2].x, w[b][3].x);
        const __half2 h45 = __floats2half2_rn(w[b][0].y, w[b][1].y);
        const __half2 h67 = __floats2half2_rn(w[b][2].y, w[b][3].y);
        uint4 raw;
        raw.x = *reinterpret_cast<const uint32_t*>(&h01);
        raw.y = *reinterpret_cast<const uint32_t*>(&h23);
        raw.z = *reinterpret_cast<const uint32_t*>(&h45);
        raw.w = *reinterpret_cast<const uint32_t*>(&h67);
        reinterpret_cast<uint4*>(dst)[b] = raw;
    }
}

// W (1/s) + z_best of one pair, in the precision the group was solved in
// (HALF && h: fp16 product and sum, as in the half-precision evaluation).
template <bool HALF>
__device__ __forceinline__ float2 final_v(float2 w, float2 inv2, float2 zb2, bool h) {
    if constexpr (HALF) {
        if (h) {
            const __half2 u = __hmul2_rn(__floats2half2_rn(w.x, w.y),
                                         __floats2half2_rn(inv2.x, inv2.y));
            return __half22float2(__hadd2_rn(u, __floats2half2_rn(zb2.x, zb2.y)));
        }
    }
    return __ffma2_rn(w, inv2, zb2);
}

// Final codes of one group finished after its chunk was written (a group
// carried over to a later chunk): codes go straight to HBM; 3 bit codes are
// OR-ed into the words, whose bits for this group were written as zero.
template <int NBITS, int G, int NB, bool HALF>
__device__ __forceinline__ void finalize_direct(const QuantParams& prm, const float2 (&w)[NB][4],
                                                const GroupState& g, int64_t gi, int kl) {
    constexpr float L = (float)((1 << NBITS) - 1);
    const float2 inv2 = make_float2(g.inv, g.inv), zb2 = make_float2(g.zb, g.zb);
    uint32_t c[NB][8];
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            float2 v = final_v<HALF>(w[b][k], inv2, zb2, g.h);
            v.x = fminf(fmaxf(v.x, 0.0f), L);
            v.y = fminf(fmaxf(v.y, 0.0f), L);
            const float2 t = __fadd2_rn(v, make_float2(kRoundShift, kRoundShift));
            c[b][k] = __float_as_uint(t.x) & 0xFFu;
            c[b][k + 4] = __float_as_uint(t.y) & 0xFFu;
        }
    if constexpr (NBITS == 3) {
        const int64_t e0 = gi * G + (int64_t)kl * 8 * NB;    // first element of the lane
        const int64_t w0 = e0 / 10;
        uint32_t acc[3] = {0u, 0u, 0u};                       // 8 NB <= 16 codes span <= 3 words
        int off = (int)(e0 - w0 * 10);
#pragma unroll
        for (int b = 0; b < NB; ++b)
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int pos = off + 8 * b + i;
                const int wi = pos / 10;
                const uint32_t bits = c[b][i] << (3 * (pos - 10 * wi));
                if (wi == 0) acc[0] |= bits;
                else if (wi == 1) acc[1] |= bits;
                else acc[2] |= bits;
            }
        uint32_t* p32 = reinterpret_cast<uint32_t*>(prm.packed);
#pragma unroll
        for (int k = 0; k < 3; ++k)
            if (acc[k]) atomicOr(p32 + w0 + k, acc[k]);
    } else {
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            const int64_t unit = gi * (G / 8) + kl * NB + b;
            uint32_t word = 0;
            if constexpr (NBITS == 8) {
                uint2 bb;
                bb.x = c[b][0] | (c[b][1] << 8) | (c[b][2] << 16) | (c[b][3] << 24);
                bb.y = c[b][4] | (c[b][5] << 8) | (c[b][6] << 16) | (c[b][7] << 24);
                reinterpret_cast<uint2*>(prm.packed)[unit] = bb;
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) word |= c[b][i] << (NBITS * i);
                if constexpr (NBITS == 4)
                    reinterpret_cast<uint32_t*>(prm.packed)[unit] = word;
                else if constexpr (NBITS == 2)
                    reinterpret_cast<uint16_t*>(prm.packed)[unit] = (uint16_t)word;
                else
                    prm.packed[unit] = (uint8_t)word;
            }
        }
    }
    if (kl == 0) {
        prm.scale[gi] = __float2half_rn(g.s);
        prm.zero[gi] = __float2half_rn(g.zb);
        if (prm.zero_f32) prm.zero_f32[gi] = g.zb;
        if (prm.err_out) prm.err_out[gi] = g.eb;
        if (prm.iters_out) prm.iters_out[gi] = (uint8_t)g.na;
        if (HALF && prm.half_out) prm.half_out[gi] = g.h ? 1 : 0;
    }
}

// Codes of one round of the final pass (the lane's NB blocks): 8, 4, 2 and 1
// bit codes to HBM, 3 bit code bytes to the chunk's code buffer (zero for a
// carried group, whose codes are OR-ed in later).  CLAMP: codes may leave
// [0, L].  A code is the low byte of W/s + z_best + 1.5 * 2^23.
template <int NBITS, int G, int NB, bool HALF, bool CLAMP>
__device__ __forceinline__ void final_codes(const QuantParams& prm, uint8_t* codes,
                                            const float2 (&w)[NB][4], const GroupState& g,
                                            int64_t chunk, int gl, int kl, bool valid, bool mine) {
    constexpr float L = (float)((1 << NBITS) - 1);
    const float2 inv2 = make_float2(g.inv, g.inv), zb2 = make_float2(g.zb, g.zb);
#pragma unroll
    for (int b = 0; b < NB; ++b) {
        uint32_t t[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            float2 v = final_v<HALF>(w[b][k], inv2, zb2, g.h);
            if (CLAMP) {
                v.x = fminf(fmaxf(v.x, 0.0f), L);
                v.y = fminf(fmaxf(v.y, 0.0f), L);
            }
            const float2 r = __fadd2_rn(v, make_float2(kRoundShift, kRoundShift));
            t[k] = __float_as_uint(r.x);
            t[k + 4] = __float_as_uint(r.y);
        }
        if (!valid || (!mine && NBITS != 3)) continue;
        const int64_t unit = chunk * (kChunk / 8) + (int64_t)gl * (G / 8) + kl * NB + b;
        if constexpr (NBITS == 8 || NBITS == 3) {
            // the eight low bytes in order, two byte permutes per word
            uint2 bb;
            bb.x = __byte_perm(__byte_perm(t[0], t[1], 0x0040), __byte_perm(t[2], t[3], 0x0040),
                               0x5410);
            bb.y = __byte_perm(__byte_perm(t[4], t[5], 0x0040), __byte_perm(t[6], t[7], 0x0040),
                               0x5410);
            if (NBITS == 3 && !mine) bb = make_uint2(0u, 0u);
            if constexpr (NBITS == 8)
                reinterpret_cast<uint2*>(prm.packed)[unit] = bb;
            else
                *reinterpret_cast<uint2*>(codes + gl * G + (kl * NB + b) * 8) = bb;
        } else {
            uint32_t word = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) word |= (t[i] & 0xFFu) << (NBITS * i);
            if constexpr (NBITS == 4)
                reinterpret_cast<uint32_t*>(prm.packed)[unit] = word;
            else if constexpr (NBITS == 2)
                reinterpret_cast<uint16_t*>(prm.packed)[unit] = (uint16_t)word;
            else
                prm.packed[unit] = (uint8_t)word;
        }
    }
}

// Final codes of every group of a chunk (one uniform pass, phase-A layout),
// from the staged weights and each group's (z_best, 1/s); 8, 4, 2 and 1 bit
// codes are stored straight to HBM, 3 bit code bytes overwrite the front of the
// chunk's weight buffer (round r writes bytes [512r, 512r+512), never ahead of
// the weights still to be read) for word packing.  Scale, zero and the
// diagnostics are written by each group's first lane.
template <int NBITS, int G, int NB, bool HALF>
__device__ __forceinline__ void final_pass(const QuantParams& prm, __half* s_w, const float4* st,
                                           const float4* st2, int64_t chunk, int cg, int lane) {
    using C = QCfg<NBITS, G, NB>;
    constexpr float L = (float)C::L;
    const int sub = lane / C::K, kl = lane % C::K;
    uint8_t* codes = reinterpret_cast<uint8_t*>(s_w);
    for (int r = 0; r < C::ROUNDS; ++r) {
        if (r * C::GPW >= cg) break;
        const int gl = r * C::GPW + sub;
        const bool valid = gl < cg;
        float2 w[NB][4];
        GroupState g;
        bool mine = valid;                          // false: carried over, finalised later
        if (valid) {
            load_lane<NB>(s_w + gl * G + kl * C::EPL, w);
            load_state(st, st2, gl, g);
            mine = (__float_as_int(st2[gl].w) & kCarried) == 0;
        } else {
#pragma unroll
            for (int b = 0; b < NB; ++b)
#pragma unroll
                for (int k = 0; k < 4; ++k) w[b][k] = make_float2(0.0f, 0.0f);
            g.zb = 0.0f;
            g.inv = 1.0f;
            g.h = false;
        }
        if constexpr (NBITS == 3) __syncwarp();     // all reads of the round before any write
        // codes need no clamp when every group of the warp has its extreme
        // weights (hence, by monotonicity, all weights) inside [-1/2, L + 1/2)
        bool inside = true;
        if (valid && mine) {
            float vmin, vmax;
            if (HALF && g.h) {
                vmin = r16(__fadd_rn(r16(__fmul_rn(g.mn, g.inv)), g.zb));
                vmax = r16(__fadd_rn(r16(__fmul_rn(g.mx, g.inv)), g.zb));
            } else {
                vmin = __fmaf_rn(g.mn, g.inv, g.zb);
                vmax = __fmaf_rn(g.mx, g.inv, g.zb);
            }
            inside = vmin >= -0.5f && vmax < L + 0.5f;
        }
        if (__all_sync(kFull, inside))
            final_codes<NBITS, G, NB, HALF, false>(prm, codes, w, g, chunk, gl, kl, valid, mine);
        else
            final_codes<NBITS, G, NB, HALF, true>(prm, codes, w, g, chunk, gl, kl, valid, mine);
        if (mine && kl == 0) {
            const int64_t gi = chunk * C::CG + gl;
            prm.scale[gi] = __float2half_rn(g.s);
            prm.zero[gi] = __float2half_rn(g.zb);
            if (prm.zero_f32) prm.zero_f32[gi] = g.zb;
            if (prm.err_out) prm.err_out[gi] = g.eb;
            if (prm.iters_out) prm.iters_out[gi] = (uint8_t)g.na;
            if (HALF && prm.half_out) prm.half_out[gi] = g.h ? 1 : 0;
        }
    }
}

// NB / NBB: 8-weight blocks per lane in phase A / phase B.  CARRY: park the
// last busy groups of a chunk and resume them with the next chunk, parking
// once at most PARK/4 of the phase-B slots are busy.  TAB2: combined power
// table (off for G = 16, whose per-group state already fills the shared memory
// that two resident CTAs per SM can have).
template <int NBITS, int G, int NB, int NBB, bool CARRY, int PARK, bool TAB2, bool HALF,
          int WARPS>
__global__ void __launch_bounds__(WARPS * 32, WARPS > 8 ? 1 : 2)
quantize_kernel(const __grid_constant__ QuantParams prm) {
    using C = QCfg<NBITS, G, NB>;      // phase A layout (and the chunk's shared memory)
    using CB = QCfg<NBITS, G, NBB>;    // phase B layout
    __shared__ QuantSmem<TAB2, HALF> S;
    extern __shared__ __align__(16) uint8_t dyn[];

    load_pow_hot(S.tp, prm.tp);
    load_pow_smem(S.tq, prm.tq);
    for (int i = threadIdx.x; i < prm.iters; i += blockDim.x) S.thr[i] = prm.shrink_thr[i];
    if constexpr (HALF)
        for (int i = threadIdx.x; i < prm.iters; i += blockDim.x) S.thr16[i] = prm.shrink_thr16[i];
    if (threadIdx.x == 0) {
        float b = prm.beta;
        for (int t = 0; t < prm.iters; ++t) {
            S.beta[t] = b;
            b = __fmul_rn(b, prm.kappa);
        }
        S.beta[prm.iters] = b;
        S.thr[prm.iters] = 0.0f;
        if constexpr (HALF) S.thr16[prm.iters] = 0.0f;
    }
    __syncthreads();

    const float2 pa1 = make_float2(prm.tp.a1, prm.tp.a1);
    const float2 pa2 = make_float2(prm.tp.a2, prm.tp.a2);
    const float2 pa3 = make_float2(prm.tp.a3, prm.tp.a3);
    const float qa1 = prm.tq.a1, qa2 = prm.tq.a2, qa3 = prm.tq.a3;

    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int sub = lane / C::K;
    const int kl = lane % C::K;
    const bool leader = kl == 0;
    constexpr int WARP_BYTES = C::CHUNK_BYTES + (CARRY ? CB::POOL_BYTES : 0);
    uint8_t* wb = dyn + warp * WARP_BYTES;
    __half* s_w = reinterpret_cast<__half*>(wb);
    float4* s_st = reinterpret_cast<float4*>(wb + C::W_BYTES);
    float4* s_st2 = reinterpret_cast<float4*>(wb + C::W_BYTES + C::ST_BYTES);
    uint8_t* s_q = wb + C::W_BYTES + C::ST_BYTES + C::ST2_BYTES;
    __half* pool_w = reinterpret_cast<__half*>(s_q + C::Q_BYTES);
    float4* pool_st = reinterpret_cast<float4*>(s_q + C::Q_BYTES + CB::POOL_W_BYTES);
    int64_t* pool_gi = reinterpret_cast<int64_t*>(s_q + C::Q_BYTES + CB::POOL_W_BYTES +
                                                  CB::POOL_ST_BYTES);
    int np = 0;                        // groups parked in the pool by the last yield

    const int64_t n_chunks = (prm.n_elems + kChunk - 1) / kChunk;
    for (int64_t chunk = (int64_t)blockIdx.x * WARPS + warp; chunk < n_chunks;
         chunk += (int64_t)gridDim.x * WARPS) {
        const int64_t e0 = chunk * kChunk;
        const int64_t left = prm.n_elems - e0;
        const int n_here = left < kChunk ? (int)left : kChunk;
        const int cg = n_here / G;

        // ---- stage the chunk's weights (one pass over HBM) ---------------------
        {
            const uint4* src = reinterpret_cast<const uint4*>(prm.W + e0);
            uint4* dst = reinterpret_cast<uint4*>(s_w);
            for (int u = lane; u < n_here / 8; u += 32) dst[u] = __ldg(src + u);
        }
        __syncwarp();

        // ---- phase A: initialise + first two iterations, all groups in step ---
        int qn = 0;
        for (int r = 0; r < C::ROUNDS; ++r) {
            if (r * C::GPW >= cg) break;
            const int gl = r * C::GPW + sub;
            const bool valid = gl < cg;
            float2 w[NB][4];
            float mn, mx;
            if (valid) {
                load_lane_minmax<NB>(s_w + gl * G + kl * C::EPL, w, mn, mx);
            } else {
#pragma unroll
                for (int b = 0; b < NB; ++b)
#pragma unroll
                    for (int k = 0; k < 4; ++k) w[b][k] = make_float2(0.0f, 0.0f);
                mn = mx = 0.0f;
            }
            GroupState g;
            group_minmax<C::K>(mn, mx);
            init_group<C::L, HALF>(g, mn, mx);
            bool live = valid && prm.iters > 0;
            bool done = valid && prm.iters == 0;
            const int ta = prm.iters < 2 ? prm.iters : 2;
            for (int tt = 0; tt < ta; ++tt) {
                const bool fin = solver_step<NBITS, G, NB, HALF>(S, prm, w, g, live, pa1, pa2,
                                                                 pa3, qa1, qa2, qa3);
                done = done || fin;
                live = live && !fin;
            }
            if ((done || live) && leader) save_state(s_st, s_st2, gl, g);
            const unsigned pmask = __ballot_sync(kFull, live && leader);
            if (live && leader) s_q[qn + __popc(pmask & ((1u << lane) - 1u))] = (uint8_t)gl;
            qn += __popc(pmask);
        }
        __syncwarp();

        // ---- phase B: queued groups, refilled as each sub-warp finishes -------
        // The queue holds the groups parked by the previous chunk (pool entries
        // 0..np-1) and then this chunk's continuing groups.  Once the queue is
        // empty and at most half the slots are busy, the warp parks the busy
        // groups in the pool and moves on (unless this is its last chunk), so the
        // longest groups never leave the other slots idle.
        {
            const int subb = lane / CB::K;
            const int klb = lane % CB::K;
            const bool leadb = klb == 0;
            const bool more = CARRY && chunk + (int64_t)gridDim.x * WARPS < n_chunks;
            const int nq = np + qn;
            int head = 0;
            bool live = false;
            int hnd = 0;                   // < kPoolTag: chunk group gl; else pool entry
            int64_t gi = 0;
            GroupState g;
            g.z = g.zb = g.eb = g.s = g.inv = g.mn = g.mx = 0.0f;
            g.t = 0;
            g.na = 0;
            g.h = false;
            float2 w[NBB][4];
#pragma unroll
            for (int b = 0; b < NBB; ++b)
#pragma unroll
                for (int k = 0; k < 4; ++k) w[b][k] = make_float2(0.0f, 0.0f);
            int parked = 0;
            while (true) {
                const unsigned want = __ballot_sync(kFull, !live && leadb);
                if (head < nq && want) {
                    const int slot = head + __popc(want & ((1u << (subb * CB::K)) - 1u));
                    if (!live && slot < nq) {
                        if (CARRY && slot < np) {
                            hnd = kPoolTag + slot;
                            load_lane<NBB>(pool_w + slot * G + klb * CB::EPL, w);
                            load_state(pool_st, pool_st + CB::SLOTS, slot, g);
                            gi = pool_gi[slot];
                        } else {
                            hnd = s_q[slot - np];
                            load_lane<NBB>(s_w + hnd * G + klb * CB::EPL, w);
                            load_state(s_st, s_st2, hnd, g);
                            gi = chunk * C::CG + hnd;
                        }
                        live = true;
                    }
                    head = min(nq, head + __popc(want));
                }
                const unsigned lmask = __ballot_sync(kFull, live && leadb);
                if (lmask == 0) break;
                if (more && head >= nq && 4 * __popc(lmask) <= PARK * CB::SLOTS) {
                    // park the busy groups (the pool's old entries are all taken)
                    __syncwarp();
                    if (live) {
                        const int j = __popc(lmask & ((1u << (subb * CB::K)) - 1u));
                        store_lane<NBB>(pool_w + j * G + klb * CB::EPL, w);
                        if (leadb) {
                            save_state(pool_st, pool_st + CB::SLOTS, j, g);
                            pool_gi[j] = gi;
                            if (hnd < kPoolTag)          // exclude it from the chunk pass
                                s_st2[hnd].w = __int_as_float(__float_as_int(s_st2[hnd].w) |
                                                              kCarried);
                        }
                    }
                    parked = __popc(lmask);
                    break;
                }
                const bool fin = solver_step<NBITS, G, NBB, HALF>(S, prm, w, g, live, pa1, pa2,
                                                                  pa3, qa1, qa2, qa3);
                if (fin) {
                    if (!CARRY || hnd < kPoolTag) {
                        if (leadb) save_state(s_st, s_st2, hnd, g);
                    } else {
                        finalize_direct<NBITS, G, NBB, HALF>(prm, w, g, gi, klb);
                    }
                }
                live = live && !fin;
            }
            np = parked;
        }

        // ---- final codes of the whole chunk, then 3-bit words -------------------
        __syncwarp();
        final_pass<NBITS, G, NB, HALF>(prm, s_w, s_st, s_st2, chunk, cg, lane);
        if constexpr (NBITS == 3) {
            uint8_t* s_codes = reinterpret_cast<uint8_t*>(s_w);
            __syncwarp();
            const int n_words = (n_here + 9) / 10;
            if (lane < n_words * 10 - n_here) s_codes[n_here + lane] = 0;   // zero padding
            __syncwarp();
            const int64_t total_words = (prm.n_elems + 9) / 10;
            for (int k = lane; k < n_words; k += 32) {
                const uint16_t* src = reinterpret_cast<const uint16_t*>(s_codes) + k * 5;
                uint32_t word = 0;
#pragma unroll
                for (int i = 0; i < 5; ++i) {
                    const uint32_t two = src[i];
                    word |= ((two & 0xFFu) | ((two >> 8) << 3)) << (6 * i);
                }
                const int64_t wi = chunk * (kChunk / 10) + k;
                if (wi < total_words) reinterpret_cast<uint32_t*>(prm.packed)[wi] = word;
            }
        }
        __syncwarp();
    }
}

// A kernel instance with its dynamic shared memory set, and the warps it keeps
// resident per SM.
template <int NBITS, int G, int NB, int NBB, bool CARRY, int PARK, bool HALF, bool TAB2,
          int WARPS>
struct QuantLaunch {
    using C = QCfg<NBITS, G, NB>;
    using CB = QCfg<NBITS, G, NBB>;
    static constexpr int SMEM = WARPS * (C::CHUNK_BYTES + (CARRY ? CB::POOL_BYTES : 0));
    static_assert(SMEM + sizeof(QuantSmem<TAB2, HALF>) <= 227 * 1024, "shared memory per CTA");
    static constexpr auto kern = quantize_kernel<NBITS, G, NB, NBB, CARRY, PARK, TAB2, HALF, WARPS>;
    int per_sm = 1;
    cudaError_t prepare() {
        cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               SMEM);
        if (err != cudaSuccess) return err;
        err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, WARPS * 32, SMEM);
        if (per_sm < 1) per_sm = 1;
        return err;
    }
    // resident warps per SM x (chunks per warp / rounds of chunks): the share
    // of the warp-slots that the chunks fill
    double fill(int64_t n_chunks, int sms) const {
        const double rounds = (double)n_chunks / ((double)sms * per_sm * WARPS);
        return rounds / std::ceil(rounds);
    }
    cudaError_t launch(const QuantParams& prm, int64_t n_chunks, int sms, cudaStream_t stream) {
        const int64_t want = (n_chunks + WARPS - 1) / WARPS;
        const int64_t cap = (int64_t)sms * per_sm;
        const unsigned grid = (unsigned)(want < cap ? want : cap);
        kern<<<grid, WARPS * 32, SMEM, stream>>>(prm);
        return cudaGetLastError();
    }
};

// The kernels come in two shapes where the shared memory allows: 20 warps in
// one CTA per SM (more warps to hide latency: 9% faster per SM on large
// matrices in single precision, 15% in half precision) and 8 warps in each
// of two CTAs per SM.  Chunks are dealt to
// warps round-robin, so a matrix of few chunks leaves part of its last round
// of warps idle; the launch takes the shape whose filled share of warp-slots,
// weighted by that per-SM speed, is larger (the 70B q/o/gate/up/down shapes
// take 20 warps, 4096 x 4096 and the 1024-row k/v take 8).
template <int NBITS, int G, int NB, int NBB, bool CARRY, int PARK, bool HALF,
          bool TAB2 = (G > 16)>
static cudaError_t launch_quantize_g(const QuantParams& prm, cudaStream_t stream) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t n_chunks = (prm.n_elems + kChunk - 1) / kChunk;
    QuantLaunch<NBITS, G, NB, NBB, CARRY, PARK, HALF, TAB2, 8> l8;
    cudaError_t err = l8.prepare();
    if (err != cudaSuccess) return err;
    using C = QCfg<NBITS, G, NB>;
    using CB = QCfg<NBITS, G, NBB>;
    constexpr int kWarpBytes = C::CHUNK_BYTES + (CARRY ? CB::POOL_BYTES : 0);
    constexpr bool kWide =
        kWideWarps * kWarpBytes + (int)sizeof(QuantSmem<TAB2, HALF>) <= 227 * 1024;
    if constexpr (kWide) {
        QuantLaunch<NBITS, G, NB, NBB, CARRY, PARK, HALF, TAB2, kWideWarps> lw;
        err = lw.prepare();
        if (err != cudaSuccess) return err;
        if (1.09 * lw.fill(n_chunks, sms) > l8.fill(n_chunks, sms))
            return lw.launch(prm, n_chunks, sms, stream);
    }
    return l8.launch(prm, n_chunks, sms, stream);
}

// 16 weights per lane in both phases.  4 bit: park the last busy groups of a
// chunk once at most half the slots are busy (measured faster); 3 and 2 bit:
// drain each chunk (measured faster: their carried groups cost more to
// finalise one by one than the idle slots they save).
template <int NBITS, bool HALF>
static cudaError_t launch_quantize_b(const QuantParams& prm, int group, cudaStream_t stream) {
    constexpr bool carry = NBITS == 4;
    switch (group) {
        case 16: return launch_quantize_g<NBITS, 16, 2, 2, carry, 2, HALF>(prm, stream);
        case 32: return launch_quantize_g<NBITS, 32, 2, 2, carry, 2, HALF>(prm, stream);
        case 64: return launch_quantize_g<NBITS, 64, 2, 2, carry, 2, HALF>(prm, stream);
        case 128: return launch_quantize_g<NBITS, 128, 2, 2, carry, 2, HALF>(prm, stream);
        case 256: return launch_quantize_g<NBITS, 256, 2, 2, carry, 2, HALF>(prm, stream);
        default: return cudaErrorInvalidValue;
    }
}

template <bool HALF>
static cudaError_t launch_quantize_nb(const QuantParams& prm, int nbits, int group,
                                      cudaStream_t stream) {
    switch (nbits) {
        case 1: return launch_quantize_b<1, HALF>(prm, group, stream);
        case 2: return launch_quantize_b<2, HALF>(prm, group, stream);
        case 3: return launch_quantize_b<3, HALF>(prm, group, stream);
        case 4: return launch_quantize_b<4, HALF>(prm, group, stream);
        case 8: return launch_quantize_b<8, HALF>(prm, group, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace hqq
