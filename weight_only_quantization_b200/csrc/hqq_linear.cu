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
//       shared memory by 4 producer warps that unpack and dequantize the codes
//       (one feature row per thread, eight 16-byte units per k-tile);
//   B = X tile [BN tokens x 64 k], K-major, 128-byte swizzle, loaded by TMA
//       (rows past M and columns past K read as zeros);
//   D = [128 x BN] fp32 in tensor memory, read back by the producer warps with
//       tcgen05.ld after the last k-tile and stored as fp16.
// Warp 0 issues the TMA loads, warp 1 owns the tensor memory and issues the
// MMAs (one elected thread), warps 2..5 produce A and run the epilogue.  A
// STAGES-deep ring of (A, B) stages is handed over with mbarriers: full_a (128
// producer arrivals), full_b (TMA transaction bytes), empty (tcgen05.commit of
// the MMAs that read the stage).
//
// Every mbarrier wait is bounded in time (globaltimer).  A wait that runs out
// records a status, makes every later wait of the CTA return at once, and the
// CTA still drains its own TMA loads and MMAs (again with a bound) before it
// frees its tensor memory and exits; the result is then unspecified.
#include <cuda.h>

#include "hqq_unpack.cuh"

namespace hqq {

namespace {

constexpr int kBM = 128;                 // features per CTA (MMA M)
constexpr int kBK = 64;                  // k per stage: one 128-byte swizzle row
constexpr int kStages = 4;
constexpr int kThreads = 192;            // 6 warps
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

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
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

// 16 consecutive fp32 columns of this warp's 32 tensor-memory lanes.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

}  // namespace

struct LinearParams {
    const uint8_t* packed;
    const __half* scale;
    const __half* zero;
    __half* Y;
    int* status;             // optional: set to 1 if a wait ran out
    int64_t M, N, K;
    int log2_group;
};

namespace {

template <int NBITS, bool SMALL>
struct KTileCodes {          // one feature row's codes and group data for one k-tile
    uint32_t bits[8];
    float s[8], z[8];
    uint32_t present;        // bit j: unit j lies inside the matrix
};

template <int NBITS, bool SMALL>
__device__ __forceinline__ void load_ktile(const LinearParams& p, int64_t n, int kt,
                                           KTileCodes<NBITS, SMALL>& c) {
    c.present = 0u;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int64_t kk = (int64_t)kt * kBK + 8 * j;
        if (n < p.N && kk < p.K) {
            const int64_t flat = n * p.K + kk;
            const int64_t g = flat >> p.log2_group;
            c.bits[j] = unit_bits<NBITS, SMALL>(p.packed, flat >> 3);
            c.s[j] = __half2float(__ldg(p.scale + g));
            c.z[j] = __half2float(__ldg(p.zero + g));
            c.present |= 1u << j;
        } else {
            c.bits[j] = 0u;
            c.s[j] = 0.0f;
            c.z[j] = 0.0f;
        }
    }
}

template <int NBITS, bool SMALL, int BN>
__global__ void __launch_bounds__(kThreads, 1)
linear_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ LinearParams prm) {
    constexpr uint32_t kBBytes = BN * kBK * 2;
    constexpr int kTmemCols = BN < 32 ? 32 : BN;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* a_st = smem;                                  // kStages x 16 KB
    uint8_t* b_st = smem + kStages * kABytes;              // kStages x BN*128 B
    uint64_t* bars = reinterpret_cast<uint64_t*>(b_st + kStages * kBBytes);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 3 * kStages + 1);
    __shared__ int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t n0 = (int64_t)blockIdx.x * kBM;
    const int64_t m0 = (int64_t)blockIdx.y * BN;
    const int KT = (int)((prm.K + kBK - 1) / kBK);
    const uint32_t bar0 = smem_u32(bars);
    // full_a[s] = bar0 + 8s, full_b[s] = bar0 + 8(S+s), empty[s] = bar0 + 8(2S+s), done
    auto full_a = [&](int s) { return bar0 + 8u * s; };
    auto full_b = [&](int s) { return bar0 + 8u * (kStages + s); };
    auto empty = [&](int s) { return bar0 + 8u * (2 * kStages + s); };
    const uint32_t done = bar0 + 8u * (3 * kStages);

    if (threadIdx.x == 0) {
        abort_flag = 0;
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full_a(s), kBM);
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
            for (int kt = 0; kt < KT; ++kt) {
                const int s = kt % kStages;
                const uint32_t ph = (uint32_t)(kt / kStages) & 1u;
                mbar_wait(empty(s), ph ^ 1u, abrt, prm.status, false);
                mbar_expect_tx(full_b(s), kBBytes);
                tma_load_2d(smem_u32(b_st + s * kBBytes), &xmap, full_b(s), kt * kBK, (int)m0);
            }
            for (int kt = KT > kStages ? KT - kStages : 0; kt < KT; ++kt)   // own loads landed
                mbar_wait(full_b(kt % kStages), (uint32_t)(kt / kStages) & 1u, abrt, prm.status,
                          true);
        }
    } else if (warp == 1) {
        if (lane == 0) {                                    // MMA issue
            const uint32_t idesc = f16_idesc<BN>();
            for (int kt = 0; kt < KT; ++kt) {
                const int s = kt % kStages;
                const uint32_t ph = (uint32_t)(kt / kStages) & 1u;
                mbar_wait(full_b(s), ph, abrt, prm.status, false);
                mbar_wait(full_a(s), ph, abrt, prm.status, false);
                fence_after_sync();
                const uint32_t a0 = smem_u32(a_st + s * kABytes);
                const uint32_t b0 = smem_u32(b_st + s * kBBytes);
#pragma unroll
                for (int k4 = 0; k4 < kBK / 16; ++k4)
                    mma_f16(tmem, sw128_desc(a0 + 32u * k4), sw128_desc(b0 + 32u * k4), idesc,
                            (kt | k4) != 0 ? 1u : 0u);
                mma_commit(empty(s));                       // stage free once these MMAs end
            }
            mma_commit(done);
        }
    } else {
        // ---- producers of W_hat: thread r writes feature row n0 + r of every stage
        const int r = threadIdx.x - 64;
        const int64_t n = n0 + r;
        KTileCodes<NBITS, SMALL> cur, nxt;
        load_ktile<NBITS, SMALL>(prm, n, 0, cur);
        for (int kt = 0; kt < KT; ++kt) {
            const int s = kt % kStages;
            const uint32_t ph = (uint32_t)(kt / kStages) & 1u;
            if (kt + 1 < KT) load_ktile<NBITS, SMALL>(prm, n, kt + 1, nxt);
            mbar_wait(empty(s), ph ^ 1u, abrt, prm.status, false);
            uint8_t* row = a_st + s * kABytes + r * 128;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (cur.present & (1u << j)) v = unit8<NBITS>(cur.bits[j], cur.z[j], cur.s[j]);
                *reinterpret_cast<uint4*>(row + ((j ^ (r & 7)) << 4)) = v;
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            mbar_arrive(full_a(s));
            cur = nxt;
        }
        // ---- epilogue: D[feature][token] -> Y[token][feature] in fp16
        mbar_wait(done, 0u, abrt, prm.status, true);
        fence_after_sync();
        const int q = warp & 3;                             // tensor-memory lane quarter
        const int64_t nf = n0 + 32 * q + lane;
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 16) {
            float v[16];
            tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)c0, v);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
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

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        cudaGetLastError();
    }
    return fn;
}

template <int BN>
constexpr size_t linear_smem() {
    return 1024 + (size_t)kStages * (kABytes + BN * kBK * 2) + (3 * kStages + 1) * 8 + 16;
}

template <int NBITS, bool SMALL, int BN>
cudaError_t launch_bn(const LinearParams& prm, const void* X, cudaStream_t stream) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    CUtensorMap map;
    const cuuint64_t dims[2] = {(cuuint64_t)prm.K, (cuuint64_t)prm.M};
    const cuuint64_t strides[1] = {(cuuint64_t)prm.K * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)BN};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(X), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    auto kern = linear_kernel<NBITS, SMALL, BN>;
    constexpr size_t smem = linear_smem<BN>();
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)((prm.N + kBM - 1) / kBM), (unsigned)((prm.M + BN - 1) / BN));
    kern<<<grid, kThreads, smem, stream>>>(map, prm);
    return cudaGetLastError();
}

template <int NBITS, bool SMALL>
cudaError_t launch_nb(const LinearParams& prm, const void* X, cudaStream_t stream) {
    if (prm.M <= 16) return launch_bn<NBITS, SMALL, 16>(prm, X, stream);
    if (prm.M <= 32) return launch_bn<NBITS, SMALL, 32>(prm, X, stream);
    if (prm.M <= 64) return launch_bn<NBITS, SMALL, 64>(prm, X, stream);
    if (prm.M <= 128) return launch_bn<NBITS, SMALL, 128>(prm, X, stream);
    return launch_bn<NBITS, SMALL, 256>(prm, X, stream);
}

}  // namespace

cudaError_t launch_linear(const LinearParams& prm, const void* X, int nbits, cudaStream_t stream) {
    const bool small = prm.N * prm.K / 8 < ((int64_t)1 << 30);
    switch (nbits) {
        case 2: return launch_nb<2, true>(prm, X, stream);
        case 4: return launch_nb<4, true>(prm, X, stream);
        case 3:
            return small ? launch_nb<3, true>(prm, X, stream) : launch_nb<3, false>(prm, X, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace hqq
