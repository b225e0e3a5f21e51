// hqq_linear.cu -- weight-only linear layer on a quantized matrix, the consumer
// of the stored format of "Half-Quadratic Quantization of Large Machine Learning
// Models" (section 2's Q^-1 fused into the matrix product):
//
//   Y[m, n] = sum_k X[m, k] * W_hat[n, k],   W_hat = fp16((code - z) * s),
//
// with X fp16 [M, K] (tokens x input features), W_hat never written to HBM,
// products and sums in the tensor cores' fp32 accumulator, Y rounded to fp16.
//
// One CTA computes a 128-feature x BN-token tile of Y^T on the 5th-generation
// tensor cores (tcgen05.mma, kind::f16, accumulator in tensor memory):
//   A = W_hat tile [128 features x 64 k], K-major, 128-byte swizzle, written to
//       shared memory by 8 producer warps that unpack and dequantize the codes
//       (four 16-byte units per thread and k-tile; the 8 lanes of a row read
//       its codes as one contiguous run);
//   B = X tile [BN tokens x 64 k], K-major, 128-byte swizzle, loaded by TMA
//       (rows past M and columns past K read as zeros);
//   D = [128 x BN] fp32 in tensor memory, read back by the producer warps with
//       tcgen05.ld after the last k-tile and stored as fp16.
// Warp 0 issues the TMA loads, warp 1 owns the tensor memory and issues the
// MMAs (one elected thread), warps 2..9 produce A and run the epilogue.  For
// few tokens (BN <= 32) and a grid short of two CTAs per SM, a cluster of 2 or
// 4 CTAs splits the k-tiles of one output tile and reduces the partial sums
// through distributed shared memory.  A
// STAGES-deep ring of (A, B) stages is handed over with mbarriers: full_a (128
// producer arrivals), full_b (TMA transaction bytes), empty (tcgen05.commit of
// the MMAs that read the stage).
//
// Every mbarrier wait is bounded in time (globaltimer).  A wait that runs out
// records a status, makes every later wait of the CTA return at once, and the
// CTA still drains its own TMA loads and MMAs (again with a bound) before it
// frees its tensor memory and exits; the result is then unspecified.
#include <cooperative_groups.h>
#include <cuda.h>

#include "hqq_unpack.cuh"

namespace hqq {

namespace cg = cooperative_groups;

namespace {

constexpr int kBM = 128;                 // features per CTA (MMA M)
constexpr int kBK = 64;                  // k per stage: one 128-byte swizzle row
constexpr int kStages = 4;

// Stage count: 4, except 2 for 512-token tiles (80 KiB per stage).
__host__ __device__ constexpr int stages_of(int bn) { return bn > 256 ? 2 : kStages; }
constexpr int kThreads = 320;            // 10 warps
constexpr uint32_t kABytes = kBM * kBK * 2;
constexpr uint64_t kWaitNs = 1000000000ull;   // 1 s per wait

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// One test of the phase; the waiting thread may be suspended in hardware for
// up to about 0.1 ms (the suspend-time hint) before the test fails, so that
// waiting warps take no issue slots from the warps doing work.
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "n"(100000)
        : "memory");
    return ok != 0;
}

// Bounded wait for the phase of `parity` to complete.  `abort` (shared) makes
// waits return false at once after any wait of the CTA has run out; `drain`
// waits ignore it (used to let the CTA's own copies and MMAs land).
__device__ __noinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort,
                                       int* status, bool drain) {
    if (mbar_try(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (!mbar_try(bar, parity)) {
        if (!drain && *abort) return false;
        if (global_ns() - t0 > kWaitNs) {
            *abort = 1;
            if (status) atomicExch(status, 1);
            return false;
        }
    }
    return true;
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

// 2-D tiled TMA load (no multicast) of box {64 k, BN rows} at (k, row).
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int k, int row) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(k), "r"(row), "r"(bar)
        : "memory");
}

// Shared-memory matrix descriptor of a K-major operand with the 128-byte
// swizzle: rows of 128 bytes, 8-row core-matrix groups 1024 bytes apart.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t addr) {
    return (uint64_t)((addr & 0x3FFFFu) >> 4)   // start address / 16
           | ((uint64_t)1 << 16)                 // leading byte offset (unused with swizzle)
           | ((uint64_t)(1024 >> 4) << 32)       // stride byte offset: 1024 B
           | ((uint64_t)1 << 46)                 // descriptor version of sm_100
           | ((uint64_t)2 << 61);                // 128-byte swizzle
}

// Instruction descriptor of kind::f16: fp16 A and B, fp32 D, both K-major.
template <int BN>
__device__ __forceinline__ uint32_t f16_idesc() {
    return (1u << 4)                             // D format: f32
           | ((uint32_t)(BN >> 3) << 17)         // N / 8
           | ((uint32_t)(kBM >> 4) << 24);       // M / 16
}

__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                        uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
        : "memory");
}

__device__ __forceinline__ void fence_before_sync() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void fence_after_sync() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

}  // namespace


namespace {

constexpr int kProducerWarps = 8;                     // warps 2..9
constexpr int kProducers = kProducerWarps * 32;
constexpr int kUnitsPerThread = kBM * (kBK / 8) / kProducers;   // 4: one quad
static_assert(kUnitsPerThread == 4, "one quad of units per producer thread and k-tile");
constexpr int kMaxSplit = 4;                          // k-slices per cluster (decode shapes)
// From this many tokens a CTA takes 512 (both 256-column halves of tensor
// memory): each dequantized weight tile then serves twice the tokens.
constexpr int64_t kLargeTileTokens = 1024;

// The units one producer thread writes per k-tile: a quad of 4 consecutive
// units (32 codes) of one row, units 4 (lane % 2) .. +3 of tile row
// pw*16 + lane/2 (QuadCodes, load_quad and quad_unit in hqq_unpack.cuh).

// 8 consecutive fp32 columns of this warp's 32 tensor-memory lanes.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
    uint32_t r[8];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

// k-tiles of codes in flight per producer thread: 2 keeps two CTAs per SM for
// small token tiles (3 and 4 measured slower there); from 256 tokens a CTA has
// an SM to itself and takes a deeper ring.
__host__ __device__ constexpr int prefetch_of(int bn) { return bn >= 256 ? 4 : 2; }

// The 32 codes of a 3-bit quad as four re-based words: word i holds codes
// 10i .. 10i + 9 in bits 0..29 (one funnel shift of the 60-bit payload of the
// stored words i and i + 1 from the quad's first slot, which is even).
__device__ __forceinline__ void rebase3(const QuadCodes<3>& c, uint32_t (&r)[4]) {
    const uint32_t sh = 2u + 3u * c.off;
#pragma unroll
    for (int i = 0; i < 4; ++i) r[i] = __funnelshift_r(c.w[i] << 2, i < 3 ? c.w[i + 1] : 0u, sh);
}

// Codes at bits b, b + 3 of x (b = 0, or 6 when B6) as exact floats: one
// logic operation per code, (x & mask) | magic with the mask as the immediate
// and the bits of 2^23 in a register (mg), then one fma pair.
// Constants of the 3-bit decode, made opaque once per thread so that they
// stay in registers (packed f32x2 operations take register pairs only):
// mg = the bits of 2^23, k20 = 2^20, k8 = 2^8, and per field pair (b, b + 3)
// with b = 0 or 6 the multipliers (2^-b, 2^-(b+3)) and offsets
// (-2^(23-b), -2^(20-b)) that turn 2^23 + c 2^b into c.
struct Dec3 {
    uint32_t mg, k20, k8;
    uint64_t i0, o0, i6, o6;                  // f32x2 pairs, low word first
    __device__ __forceinline__ void init() {
        mg = 0x4B000000u;
        k20 = 1u << 20;
        k8 = 1u << 8;
        auto pack = [](float lo, float hi) {
            return (uint64_t)__float_as_uint(lo) | ((uint64_t)__float_as_uint(hi) << 32);
        };
        i0 = pack(1.0f, 0.125f);
        o0 = pack(-8388608.0f, -1048576.0f);
        i6 = pack(0.015625f, 0.001953125f);
        o6 = pack(-131072.0f, -16384.0f);
        asm volatile("" : "+r"(mg), "+r"(k20), "+r"(k8));
        asm volatile("" : "+l"(i0), "+l"(o0), "+l"(i6), "+l"(o6));
    }
};

// fp16((c - z) s) of the codes at bits b, b + 3 of x (b = 0, or 6 when B6),
// packed in one word, as one block: the two fields into the mantissa of 2^23
// (one logic operation each), the exact codes (one f32x2 fma), fl32(c - z) and
// fl32(. s) (one f32x2 add and multiply, nz = (-z, -z), ss = (s, s)), the fp16
// pair.
template <int B6>
__device__ __forceinline__ uint32_t pair3_dq(uint32_t x, const Dec3& d, uint64_t nz, uint64_t ss) {
    constexpr uint32_t m0 = 7u << (B6 ? 6 : 0), m1 = m0 << 3;
    uint32_t h;
    asm("{\n\t.reg .b32 a, b, lo, hi;\n\t.reg .b64 ab, c;\n\t"
        "lop3.b32 a, %1, %2, %4, 0xEA;\n\t"
        "lop3.b32 b, %1, %3, %4, 0xEA;\n\t"
        "mov.b64 ab, {a, b};\n\t"
        "fma.rn.f32x2 c, ab, %5, %6;\n\t"
        "add.rn.f32x2 c, c, %7;\n\t"
        "mul.rn.f32x2 c, c, %8;\n\t"
        "mov.b64 {lo, hi}, c;\n\t"
        "cvt.rn.f16x2.f32 %0, hi, lo;\n\t}"
        : "=r"(h)
        : "r"(x), "n"(m0), "n"(m1), "r"(d.mg), "l"(B6 ? d.i6 : d.i0), "l"(B6 ? d.o6 : d.o0),
          "l"(nz), "l"(ss));
    return h;
}

// Unit t (codes 8t .. 8t + 7) of a re-based 3-bit quad as fp16 weights: pair
// (2m, 2m + 1) sits at slot 2m % 10 of word 2m / 10; slots 0-3 are read from
// the word, 4-7 from the word shifted right by 12 and 8-9 by 24 (multiply-high
// by the opaque k20 = 2^20 and k8 = 2^8), so two constant sets serve all.
__device__ __forceinline__ uint4 quad_unit3(const QuadCodes<3>& c, const uint32_t (&r)[4], int t,
                                            const Dec3& d) {
    const __half2 sz = c.sz[t >> 1];
    const float s = __low2float(sz), z = __high2float(sz);
    uint64_t ss, nz;
    asm("mov.b64 %0, {%1, %1};" : "=l"(ss) : "f"(s));
    asm("mov.b64 %0, {%1, %1};" : "=l"(nz) : "f"(-z));
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int m = 2 * (4 * t + q), sl = m % 10;
        const uint32_t x = r[m / 10];
        if (sl == 0) o[q] = pair3_dq<0>(x, d, nz, ss);
        else if (sl == 2) o[q] = pair3_dq<1>(x, d, nz, ss);
        else if (sl == 4) o[q] = pair3_dq<0>(__umulhi(x, d.k20), d, nz, ss);
        else if (sl == 6) o[q] = pair3_dq<1>(__umulhi(x, d.k20), d, nz, ss);
        else o[q] = pair3_dq<0>(__umulhi(x, d.k8), d, nz, ss);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// gridDim.z > 1: the CTAs of a (1, 1, gridDim.z) cluster split the k-tiles of
// one output tile; each keeps its partial sums in its own tensor memory, the
// others write theirs into rank 0's (then idle) stage buffers through
// distributed shared memory, and rank 0 adds them and stores Y.
template <int NBITS, bool SMALL, bool VEC, int BN>
__global__ void __launch_bounds__(kThreads, 1)
linear_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ LinearParams prm) {
    constexpr int S = stages_of(BN);
    constexpr uint32_t kBBytes = BN * kBK * 2;
    constexpr int kTmemCols = BN < 32 ? 32 : BN;
    constexpr int kMmaN = BN > 256 ? 256 : BN;             // N of one MMA (and TMA box rows)
    constexpr int kParts = BN / kMmaN;                     // accumulators side by side
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* a_st = smem;                                  // S x 16 KB
    uint8_t* b_st = smem + S * kABytes;              // S x BN*128 B
    uint64_t* bars = reinterpret_cast<uint64_t*>(b_st + S * kBBytes);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 3 * S + 1);
    float* red = reinterpret_cast<float*>(smem);           // split-k partials (rank 0)
    __shared__ int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // token tiles of one feature tile are adjacent in the grid (x), so a
    // feature tile's codes come from HBM once and from L2 for the others
    const int64_t n0 = (int64_t)blockIdx.y * kBM;
    const int64_t m0 = (int64_t)blockIdx.x * BN;
    const int ks = (int)gridDim.z, rank = (int)blockIdx.z;
    const int KT = (int)((prm.K + kBK - 1) / kBK);
    const int kt0 = (int)((int64_t)KT * rank / ks);
    const int nkt = (int)((int64_t)KT * (rank + 1) / ks) - kt0;
    const uint32_t bar0 = smem_u32(bars);
    // full_a[s] = bar0 + 8s, full_b[s] = bar0 + 8(S+s), empty[s] = bar0 + 8(2S+s), done
    auto full_a = [&](int s) { return bar0 + 8u * s; };
    auto full_b = [&](int s) { return bar0 + 8u * (S + s); };
    auto empty = [&](int s) { return bar0 + 8u * (2 * S + s); };
    const uint32_t done = bar0 + 8u * (3 * S);

    if (threadIdx.x == 0) {
        abort_flag = 0;
        for (int s = 0; s < S; ++s) {
            mbar_init(full_a(s), kProducers);
            mbar_init(full_b(s), 1);
            mbar_init(empty(s), 1);
        }
        mbar_init(done, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&xmap))
                     : "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_holder)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tmem_holder;
    volatile int* abrt = &abort_flag;

    if (warp == 0) {
        if (lane == 0) {                                    // X tiles by TMA
            for (int kt = 0; kt < nkt; ++kt) {
                const int s = kt % S;
                const uint32_t ph = (uint32_t)(kt / S) & 1u;
                mbar_wait(empty(s), ph ^ 1u, abrt, prm.status, false);
                mbar_expect_tx(full_b(s), kBBytes);
#pragma unroll
                for (int h = 0; h < kParts; ++h)
                    tma_load_2d(smem_u32(b_st + s * kBBytes + h * kMmaN * kBK * 2), &xmap,
                                full_b(s), (kt0 + kt) * kBK, (int)m0 + h * kMmaN);
            }
            for (int kt = nkt > S ? nkt - S : 0; kt < nkt; ++kt)  // own loads landed
                mbar_wait(full_b(kt % S), (uint32_t)(kt / S) & 1u, abrt, prm.status,
                          true);
        }
    } else if (warp == 1) {
        if (lane == 0) {                                    // MMA issue
            const uint32_t idesc = f16_idesc<kMmaN>();
            for (int kt = 0; kt < nkt; ++kt) {
                const int s = kt % S;
                const uint32_t ph = (uint32_t)(kt / S) & 1u;
                mbar_wait(full_b(s), ph, abrt, prm.status, false);
                mbar_wait(full_a(s), ph, abrt, prm.status, false);
                fence_after_sync();
                const uint32_t a0 = smem_u32(a_st + s * kABytes);
                const uint32_t b0 = smem_u32(b_st + s * kBBytes);
#pragma unroll
                for (int h = 0; h < kParts; ++h)            // columns [h kMmaN, (h+1) kMmaN)
#pragma unroll
                    for (int k4 = 0; k4 < kBK / 16; ++k4)
                        mma_f16(tmem + (uint32_t)(h * kMmaN), sw128_desc(a0 + 32u * k4),
                                sw128_desc(b0 + (uint32_t)(h * kMmaN * kBK * 2) + 32u * k4),
                                idesc, (kt | k4) != 0 ? 1u : 0u);
                mma_commit(empty(s));                       // stage free once these MMAs end
            }
            mma_commit(done);
        }
    } else {
        // ---- producers of W_hat: quads of 4 units, a ring of kPrefetch k-tiles
        constexpr int kPrefetch = prefetch_of(BN);
        Dec3 dec;
        if constexpr (NBITS == 3) dec.init();
        // of codes in registers (indices fixed by unrolling)
        const int pw = warp - 2, j4 = lane & 1;
        const int r = pw * 16 + (lane >> 1);
        const int64_t n = n0 + r;
        const bool row_ok = n < prm.N;
        const int64_t fbase = n * prm.K;
        QuadCodes<NBITS> ring[kPrefetch];
#pragma unroll
        for (int u = 0; u < kPrefetch - 1; ++u)
            if (u < nkt)
                load_quad<NBITS, SMALL, VEC>(prm, fbase, row_ok,
                                             (int64_t)(kt0 + u) * kBK + 32 * j4, ring[u]);
        for (int kb = 0; kb < nkt; kb += kPrefetch) {
#pragma unroll
            for (int u = 0; u < kPrefetch; ++u) {
                const int kt = kb + u;
                if (kt < nkt) {
                    if (kt + kPrefetch - 1 < nkt)
                        load_quad<NBITS, SMALL, VEC>(
                            prm, fbase, row_ok,
                            (int64_t)(kt0 + kt + kPrefetch - 1) * kBK + 32 * j4,
                            ring[(u + kPrefetch - 1) % kPrefetch]);
                    const int s = kt % S;
                    const uint32_t ph = (uint32_t)(kt / S) & 1u;
                    mbar_wait(empty(s), ph ^ 1u, abrt, prm.status, false);
                    uint8_t* arow = a_st + s * kABytes + r * 128;
                    const QuadCodes<NBITS>& cur = ring[u];
                    if constexpr (NBITS == 3) {
                        uint32_t rb[4];
                        rebase3(cur, rb);
#pragma unroll
                        for (int t = 0; t < 4; ++t) {                // absent units: s = z = 0
                            const int j = 4 * j4 + t;
                            *reinterpret_cast<uint4*>(arow + ((j ^ (r & 7)) << 4)) =
                                quad_unit3(cur, rb, t, dec);
                        }
                    } else {
#pragma unroll
                        for (int t = 0; t < 4; ++t) {                // absent units: s = z = 0
                            const int j = 4 * j4 + t;
                            *reinterpret_cast<uint4*>(arow + ((j ^ (r & 7)) << 4)) =
                                quad_unit<NBITS>(cur, t);
                        }
                    }
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    mbar_arrive(full_a(s));
                }
            }
        }
        mbar_wait(done, 0u, abrt, prm.status, true);        // every MMA of this CTA ended
        fence_after_sync();
    }

    // ---- epilogue: D[feature][token] -> Y[token][feature] in fp16.  Producer
    // warp w reads tensor-memory lanes 32 (w % 4) .. +31 (its quarter); warps
    // 2..5 take the first half of the BN columns, warps 6..9 the second.
    const bool epi = warp >= 2;
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    const int f = 32 * q + lane;                            // feature row within the tile
    const int64_t nf = n0 + f;
    constexpr int kHalf = BN / 2;
    const uint32_t trow = tmem + ((uint32_t)(32 * q) << 16);
    if (ks > 1) {
        cg::cluster_group cluster = cg::this_cluster();
        __syncwarp();
        cluster.sync();                                     // rank 0's stages are free
        if (epi && rank != 0) {
            float* dst = cluster.map_shared_rank(red, 0) + (size_t)(rank - 1) * BN * kBM;
#pragma unroll 1
            for (int c0 = half * kHalf; c0 < (half + 1) * kHalf; c0 += 8) {
                float v[8];
                tmem_ld8(trow + (uint32_t)c0, v);
#pragma unroll
                for (int i = 0; i < 8; ++i) dst[(c0 + i) * kBM + f] = v[i];
            }
        }
        __syncwarp();
        cluster.sync();                                     // every partial has arrived
    }
    if (epi && rank == 0) {
#pragma unroll 1
        for (int c0 = half * kHalf; c0 < (half + 1) * kHalf; c0 += 8) {
            float v[8];
            tmem_ld8(trow + (uint32_t)c0, v);
            for (int r = 1; r < ks; ++r) {
                const float* src = red + (size_t)(r - 1) * BN * kBM;
#pragma unroll
                for (int i = 0; i < 8; ++i) v[i] += src[(c0 + i) * kBM + f];
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int64_t m = m0 + c0 + i;
                if (m < prm.M && nf < prm.N) prm.Y[m * prm.N + nf] = __float2half_rn(v[i]);
            }
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        fence_after_sync();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(kTmemCols)
                     : "memory");
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn lookup_encode_fn() {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    EncodeTiledFn fn = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
        fn = reinterpret_cast<EncodeTiledFn>(p);
    cudaGetLastError();                               // a failed lookup leaves no error behind
    return fn;
}

// The driver's tensor-map encoder, looked up once (a function-local static is
// initialised exactly once even when several host threads call at once).
EncodeTiledFn encode_fn() {
    static const EncodeTiledFn fn = lookup_encode_fn();
    return fn;
}

template <int BN>
constexpr size_t linear_smem() {
    return 1024 + (size_t)stages_of(BN) * (kABytes + BN * kBK * 2) + (3 * stages_of(BN) + 1) * 8 +
           16;
}

template <int NBITS, bool SMALL, bool VEC, int BN>
cudaError_t launch_bn(const LinearParams& prm, const void* X, cudaStream_t stream) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    CUtensorMap map;
    const cuuint64_t dims[2] = {(cuuint64_t)prm.K, (cuuint64_t)prm.M};
    const cuuint64_t strides[1] = {(cuuint64_t)prm.K * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)(BN > 256 ? 256 : BN)};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(X), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    auto kern = linear_kernel<NBITS, SMALL, VEC, BN>;
    constexpr size_t smem = linear_smem<BN>();
    // split-k partials of up to kMaxSplit - 1 ranks fit in rank 0's stage buffers
    static_assert(BN > 32 || (size_t)(kMaxSplit - 1) * BN * kBM * 4 <= (size_t)kStages * kABytes,
                  "split-k buffer");
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t tiles_n = (prm.N + kBM - 1) / kBM, tiles_m = (prm.M + BN - 1) / BN;
    const int KT = (int)((prm.K + kBK - 1) / kBK);
    int ks = 1;                               // split k while the grid is short of 2 CTAs/SM
    while (BN <= 32 && ks < kMaxSplit && tiles_n * tiles_m * ks < 2 * sms && KT >= 4 * ks)
        ks *= 2;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 1;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = (unsigned)ks;
    cfg.gridDim = dim3((unsigned)tiles_m, (unsigned)tiles_n, (unsigned)ks);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, map, prm);
}

template <int NBITS, bool SMALL, bool VEC>
cudaError_t launch_nb(const LinearParams& prm, const void* X, cudaStream_t stream) {
    if (prm.M <= 16) return launch_bn<NBITS, SMALL, VEC, 16>(prm, X, stream);
    if (prm.M <= 32) return launch_bn<NBITS, SMALL, VEC, 32>(prm, X, stream);
    if (prm.M <= 64) return launch_bn<NBITS, SMALL, VEC, 64>(prm, X, stream);
    if (prm.M <= 128) return launch_bn<NBITS, SMALL, VEC, 128>(prm, X, stream);
    if (prm.M < kLargeTileTokens) return launch_bn<NBITS, SMALL, VEC, 256>(prm, X, stream);
    return launch_bn<NBITS, SMALL, VEC, 512>(prm, X, stream);
}

// Quads of codes load as one vector when every row starts on a quad (K % 32)
// and the packed buffer is 16-byte aligned.
template <int NBITS>
cudaError_t launch_vec(const LinearParams& prm, const void* X, cudaStream_t stream) {
    const bool vec = prm.K % 32 == 0 && (reinterpret_cast<uintptr_t>(prm.packed) & 15u) == 0;
    return vec ? launch_nb<NBITS, true, true>(prm, X, stream)
               : launch_nb<NBITS, true, false>(prm, X, stream);
}

}  // namespace

cudaError_t launch_linear(const LinearParams& prm, const void* X, int nbits, cudaStream_t stream) {
    const bool small = prm.N * prm.K / 8 < ((int64_t)1 << 30);
    switch (nbits) {
        case 1: return launch_vec<1>(prm, X, stream);
        case 2: return launch_vec<2>(prm, X, stream);
        case 4: return launch_vec<4>(prm, X, stream);
        case 8: return launch_vec<8>(prm, X, stream);
        case 3:
            return small ? launch_nb<3, true, false>(prm, X, stream)
                         : launch_nb<3, false, false>(prm, X, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace hqq
