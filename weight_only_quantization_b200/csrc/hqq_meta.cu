// hqq_meta.cu -- 8-bit storage of the per-group zero points and scales, from
// the settings of section 4.1 of "Half-Quadratic Quantization of Large Machine
// Learning Models": the zero points are kept in 8 bits with neither grouping
// nor optimisation, and the starred row of the section's table also keeps the
// scales in 8 bits, in groups of 128.  "Without optimisation" is section 2's Q
// with its min-max start and no solver iterations, applied to the stored fp16
// meta tensor with 255 levels:
//   s = (max - min)/255 and 1/s (1 and 1 for a constant group), z = -min (1/s),
//   c = clamp(rint(fma(x, 1/s, z)), 0, 255), s and z stored in fp16;
// restored as fp16((c - z) s) from the stored fp16 s and z.
//
// Kernels
//  - meta_group_kernel / meta_group_vec_kernel: groups of 2^k values; a
//    segment of lanes per group (one value, or for 2^k >= 8 one 16-byte vector
//    of 8 values, per lane and step), exact min/max by shuffles, then the
//    codes.  Meta tensors are 1/16..1/256 of the weights: a small
//    memory-bound pass.
//  - meta_whole_kernel: one group over the whole tensor ("no grouping").  One
//    thread-block cluster reduces the tensor: every CTA takes an interleaved
//    share of 16-byte vectors, the CTAs exchange their min/max through
//    distributed shared memory, and each quantizes its share on a second read
//    (from L2 for one matrix's meta tensor).  One launch, no global scratch.
//  - meta_dequant_kernel: 8 codes (one 8-byte load) -> one 16-byte store.
#include <cooperative_groups.h>

#include "hqq_params.cuh"

namespace hqq {

namespace cg = cooperative_groups;

namespace {

constexpr float kMetaL = 255.0f;

struct MetaAffine {
    float s, inv, z;
};

// Binary32 start of min-max round-to-nearest with 255 levels.
__device__ __forceinline__ MetaAffine meta_affine(float mn, float mx) {
    const float rng = __fsub_rn(mx, mn);
    MetaAffine a;
    if (rng == 0.0f) {
        a.s = 1.0f;
        a.inv = 1.0f;
    } else {
        a.s = __fdiv_rn(rng, kMetaL);
        a.inv = __frcp_rn(a.s);
    }
    a.z = -__fmul_rn(mn, a.inv);
    return a;
}

// clamp(round(x (1/s) + z), 0, 255), half to even: clamping to the integers 0
// and 255 first gives the same code, and adding 1.5 * 2^23 then rounds to an
// integer held in the low mantissa bits (no conversion instructions).
constexpr float kMetaShift = 12582912.0f;   // 1.5 * 2^23

__device__ __forceinline__ uint32_t meta_code(float x, const MetaAffine& a) {
    const float v = fminf(fmaxf(__fmaf_rn(x, a.inv, a.z), 0.0f), kMetaL);
    return __float_as_uint(__fadd_rn(v, kMetaShift)) & 0xFFu;
}

// Eight consecutive values -> eight codes, first code in the low byte.
__device__ __forceinline__ uint2 meta_codes8(uint4 v, const MetaAffine& a) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    const float2 inv2 = make_float2(a.inv, a.inv), z2 = make_float2(a.z, a.z);
    const float2 sh2 = make_float2(kMetaShift, kMetaShift);
    uint32_t t[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float2 f = __ffma2_rn(__half22float2(*reinterpret_cast<const __half2*>(&w[j])), inv2, z2);
        f.x = fminf(fmaxf(f.x, 0.0f), kMetaL);
        f.y = fminf(fmaxf(f.y, 0.0f), kMetaL);
        f = __fadd2_rn(f, sh2);
        t[2 * j] = __float_as_uint(f.x);
        t[2 * j + 1] = __float_as_uint(f.y);
    }
    // the low byte of each sum, in order
    return make_uint2(
        __byte_perm(__byte_perm(t[0], t[1], 0x0040), __byte_perm(t[2], t[3], 0x0040), 0x5410),
        __byte_perm(__byte_perm(t[4], t[5], 0x0040), __byte_perm(t[6], t[7], 0x0040), 0x5410));
}

__device__ __forceinline__ void minmax8(uint4 v, __half2& mn, __half2& mx) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const __half2 h = *reinterpret_cast<const __half2*>(&w[j]);
        mn = __hmin2(mn, h);
        mx = __hmax2(mx, h);
    }
}

constexpr int kGroupThreads = 256;
constexpr int kMetaBatchMax = 128;                    // jobs per batched launch

// Groups of 2^k values, one value per lane and step; `block` of `nblocks`
// blocks working on this tensor.
__device__ __forceinline__ void meta_group_body(const __half* __restrict__ x, int64_t n,
                                                int log2g, int64_t ngroups,
                                                uint8_t* __restrict__ codes,
                                                __half* __restrict__ scale,
                                                __half* __restrict__ zero, int64_t block,
                                                int64_t nblocks) {
    const int lane = threadIdx.x & 31;
    const int lseg = log2g < 5 ? log2g : 5;          // log2(lanes per group)
    const int seg = 1 << lseg;
    const int per_warp = 32 >> lseg;                  // groups per warp step
    const int64_t gs = (int64_t)1 << log2g;
    const int64_t warp = (block * kGroupThreads + threadIdx.x) >> 5;
    const int64_t nwarps = (nblocks * kGroupThreads) >> 5;
    const int k0 = lane & (seg - 1);
    for (int64_t gb = warp * per_warp; gb < ngroups; gb += nwarps * per_warp) {
        const int64_t gi = gb + (lane >> lseg);
        const bool valid = gi < ngroups;
        const int64_t g0 = gi << log2g;
        const int64_t m = valid ? (n - g0 < gs ? n - g0 : gs) : 0;
        float mn = INFINITY, mx = -INFINITY;
        for (int64_t k = k0; k < m; k += seg) {
            const float v = __half2float(x[g0 + k]);
            mn = fminf(mn, v);
            mx = fmaxf(mx, v);
        }
        for (int o = seg >> 1; o > 0; o >>= 1) {
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        }
        if (valid) {
            const MetaAffine a = meta_affine(mn, mx);
            for (int64_t k = k0; k < m; k += seg)
                codes[g0 + k] = (uint8_t)meta_code(__half2float(x[g0 + k]), a);
            if (k0 == 0) {
                scale[gi] = __float2half_rn(a.s);
                zero[gi] = __float2half_rn(a.z);
            }
        }
    }
}

// Groups of 2^k >= 8 values: each lane takes 16-byte vectors (8 values), a
// segment of min(2^k/8, 32) lanes per group.  The vector that holds the end of
// a ragged last group is read value by value.
__device__ __forceinline__ void meta_group_vec_body(const __half* __restrict__ x, int64_t n,
                                                    int log2g, int64_t ngroups,
                                                    uint8_t* __restrict__ codes,
                                                    __half* __restrict__ scale,
                                                    __half* __restrict__ zero, int64_t block,
                                                    int64_t nblocks) {
    const int lane = threadIdx.x & 31;
    const int lv = log2g - 3;                         // log2(vectors per group)
    const int lseg = lv < 5 ? lv : 5;
    const int seg = 1 << lseg;
    const int per_warp = 32 >> lseg;
    const int64_t warp = (block * kGroupThreads + threadIdx.x) >> 5;
    const int64_t nwarps = (nblocks * kGroupThreads) >> 5;
    const int k0 = lane & (seg - 1);
    const uint4* xv = reinterpret_cast<const uint4*>(x);
    const int64_t nfull = n >> 3;                     // vectors entirely inside x
    for (int64_t gb = warp * per_warp; gb < ngroups; gb += nwarps * per_warp) {
        const int64_t gi = gb + (lane >> lseg);
        const bool valid = gi < ngroups;
        const int64_t v0 = gi << lv;                  // first vector of the group
        const int64_t vend = valid ? min(v0 + ((int64_t)1 << lv), (n + 7) >> 3) : v0;
        __half2 hmn = __float2half2_rn(INFINITY), hmx = __float2half2_rn(-INFINITY);
        float mn = INFINITY, mx = -INFINITY;
        for (int64_t v = v0 + k0; v < vend; v += seg) {
            if (v < nfull) {
                minmax8(__ldg(xv + v), hmn, hmx);
            } else {
                for (int64_t i = v << 3; i < n; ++i) {
                    const float f = __half2float(x[i]);
                    mn = fminf(mn, f);
                    mx = fmaxf(mx, f);
                }
            }
        }
        mn = fminf(mn, fminf(__low2float(hmn), __high2float(hmn)));
        mx = fmaxf(mx, fmaxf(__low2float(hmx), __high2float(hmx)));
        for (int o = seg >> 1; o > 0; o >>= 1) {
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        }
        if (valid) {
            const MetaAffine a = meta_affine(mn, mx);
            for (int64_t v = v0 + k0; v < vend; v += seg) {
                if (v < nfull) {
                    reinterpret_cast<uint2*>(codes)[v] = meta_codes8(__ldg(xv + v), a);
                } else {
                    for (int64_t i = v << 3; i < n; ++i)
                        codes[i] = (uint8_t)meta_code(__half2float(x[i]), a);
                }
            }
            if (k0 == 0) {
                scale[gi] = __float2half_rn(a.s);
                zero[gi] = __float2half_rn(a.z);
            }
        }
    }
}

__global__ void __launch_bounds__(kGroupThreads)
meta_group_kernel(const __half* __restrict__ x, int64_t n, int log2g, int64_t ngroups,
                  uint8_t* __restrict__ codes, __half* __restrict__ scale,
                  __half* __restrict__ zero) {
    meta_group_body(x, n, log2g, ngroups, codes, scale, zero, blockIdx.x, gridDim.x);
}

__global__ void __launch_bounds__(kGroupThreads)
meta_group_vec_kernel(const __half* __restrict__ x, int64_t n, int log2g, int64_t ngroups,
                      uint8_t* __restrict__ codes, __half* __restrict__ scale,
                      __half* __restrict__ zero) {
    meta_group_vec_body(x, n, log2g, ngroups, codes, scale, zero, blockIdx.x, gridDim.x);
}

constexpr int kWholeThreads = 512;
constexpr int kWholeBatch = 8;                        // 16-byte loads in flight per thread

// One tensor reduced and quantized by the calling thread-block cluster.
__device__ __forceinline__ void meta_whole_body(const __half* __restrict__ x, int64_t n,
                                                uint8_t* __restrict__ codes,
                                                __half* __restrict__ scale,
                                                __half* __restrict__ zero) {
    cg::cluster_group cluster = cg::this_cluster();
    const int64_t rank = cluster.block_rank();
    const int64_t ncta = cluster.num_blocks();
    __shared__ float warp_mn[32], warp_mx[32];
    __shared__ float cta_mm[2];

    const uint4* xv = reinterpret_cast<const uint4*>(x);
    const int64_t nvec = n >> 3;
    const int64_t first = rank * kWholeThreads + threadIdx.x;
    const int64_t stride = ncta * kWholeThreads;

    const __half2 pinf = __float2half2_rn(INFINITY), ninf = __float2half2_rn(-INFINITY);
    __half2 hmn = pinf, hmx = ninf;
    for (int64_t v0 = first; v0 < nvec; v0 += kWholeBatch * stride) {
        uint4 r[kWholeBatch];
#pragma unroll
        for (int b = 0; b < kWholeBatch; ++b) {
            const int64_t v = v0 + b * stride;
            r[b] = v < nvec ? __ldg(xv + v) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int b = 0; b < kWholeBatch; ++b)
            if (v0 + b * stride < nvec) minmax8(r[b], hmn, hmx);
    }
    float mn = fminf(__low2float(hmn), __high2float(hmn));
    float mx = fmaxf(__low2float(hmx), __high2float(hmx));
    const int64_t tail0 = nvec << 3;                  // the last n % 8 values
    if (rank == 0 && threadIdx.x < n - tail0) {
        const float v = __half2float(x[tail0 + threadIdx.x]);
        mn = fminf(mn, v);
        mx = fmaxf(mx, v);
    }
    for (int o = 16; o > 0; o >>= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) {
        warp_mn[warp] = mn;
        warp_mx[warp] = mx;
    }
    __syncthreads();
    if (warp == 0) {
        constexpr int kWarps = kWholeThreads / 32;
        mn = lane < kWarps ? warp_mn[lane] : INFINITY;
        mx = lane < kWarps ? warp_mx[lane] : -INFINITY;
        for (int o = 16; o > 0; o >>= 1) {
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        }
        if (lane == 0) {
            cta_mm[0] = mn;
            cta_mm[1] = mx;
        }
    }
    cluster.sync();                                   // every CTA's min/max is visible
    mn = INFINITY;
    mx = -INFINITY;
    for (int r = 0; r < (int)ncta; ++r) {
        const float* peer = cluster.map_shared_rank(cta_mm, r);
        mn = fminf(mn, peer[0]);
        mx = fmaxf(mx, peer[1]);
    }
    cluster.sync();                                   // no CTA exits while read remotely

    const MetaAffine a = meta_affine(mn, mx);
    uint2* cv = reinterpret_cast<uint2*>(codes);
    for (int64_t v0 = first; v0 < nvec; v0 += kWholeBatch * stride) {
        uint4 r[kWholeBatch];
#pragma unroll
        for (int b = 0; b < kWholeBatch; ++b) {
            const int64_t v = v0 + b * stride;
            r[b] = v < nvec ? __ldg(xv + v) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int b = 0; b < kWholeBatch; ++b) {
            const int64_t v = v0 + b * stride;
            if (v < nvec) cv[v] = meta_codes8(r[b], a);
        }
    }
    if (rank == 0) {
        if (threadIdx.x < n - tail0)
            codes[tail0 + threadIdx.x] = (uint8_t)meta_code(__half2float(x[tail0 + threadIdx.x]), a);
        if (threadIdx.x == 0) {
            scale[0] = __float2half_rn(a.s);
            zero[0] = __float2half_rn(a.z);
        }
    }
}

__global__ void __launch_bounds__(kWholeThreads, 2)
meta_whole_kernel(const __half* __restrict__ x, int64_t n, uint8_t* __restrict__ codes,
                  __half* __restrict__ scale, __half* __restrict__ zero) {
    meta_whole_body(x, n, codes, scale, zero);
}

// ---- batches: many meta tensors per launch ----------------------------------
// Whole-tensor jobs: cluster c of the grid takes job c.  Grouped jobs: job j owns
// blocks [first[j], first[j+1]) of the grid.
struct MetaJob {
    const __half* x;
    int64_t n;
    uint8_t* codes;
    __half* scale;
    __half* zero;
    int64_t ngroups;
    int log2g;
};

struct MetaBatch {
    int count;
    int first[kMetaBatchMax + 1];
    MetaJob job[kMetaBatchMax];
};

__global__ void __launch_bounds__(kWholeThreads, 2)
meta_whole_batch_kernel(const __grid_constant__ MetaBatch b) {
    const MetaJob& j = b.job[blockIdx.x / cg::this_cluster().num_blocks()];
    meta_whole_body(j.x, j.n, j.codes, j.scale, j.zero);
}

__global__ void __launch_bounds__(kGroupThreads)
meta_group_batch_kernel(const __grid_constant__ MetaBatch b) {
    int lo = 0, hi = b.count - 1;                     // the job whose block range holds us
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (b.first[mid] <= (int)blockIdx.x) lo = mid; else hi = mid - 1;
    }
    const MetaJob& j = b.job[lo];
    const int64_t block = (int64_t)blockIdx.x - b.first[lo];
    const int64_t nblocks = b.first[lo + 1] - b.first[lo];
    if (j.log2g >= 3)
        meta_group_vec_body(j.x, j.n, j.log2g, j.ngroups, j.codes, j.scale, j.zero, block,
                            nblocks);
    else
        meta_group_body(j.x, j.n, j.log2g, j.ngroups, j.codes, j.scale, j.zero, block, nblocks);
}

constexpr int kMdqThreads = 256;

__device__ __forceinline__ uint32_t restore2(uint32_t c01, float z0, float s0, float z1, float s1) {
    const float a = __fmul_rn(__fsub_rn((float)(c01 & 0xFFu), z0), s0);
    const float b = __fmul_rn(__fsub_rn((float)((c01 >> 8) & 0xFFu), z1), s1);
    const __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&h);
}

// shift: log2 of the second-level group, or 62 for one group over everything.
__global__ void __launch_bounds__(kMdqThreads)
meta_dequant_kernel(const uint8_t* __restrict__ codes, const __half* __restrict__ scale,
                    const __half* __restrict__ zero, int64_t n, int shift,
                    __half* __restrict__ out) {
    const int64_t nvec = n >> 3;
    const int64_t stride = (int64_t)gridDim.x * kMdqThreads;
    for (int64_t v = (int64_t)blockIdx.x * kMdqThreads + threadIdx.x; v < nvec; v += stride) {
        const uint2 c = __ldg(reinterpret_cast<const uint2*>(codes) + v);
        const uint32_t cw[2] = {c.x, c.y};
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t i = (v << 3) + 2 * j;
            const int64_t g0 = i >> shift, g1 = (i + 1) >> shift;
            o[j] = restore2(cw[j >> 1] >> (16 * (j & 1)),
                            __half2float(__ldg(zero + g0)), __half2float(__ldg(scale + g0)),
                            __half2float(__ldg(zero + g1)), __half2float(__ldg(scale + g1)));
        }
        reinterpret_cast<uint4*>(out)[v] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    const int64_t tail0 = nvec << 3;
    if (blockIdx.x == 0 && threadIdx.x < n - tail0) {
        const int64_t i = tail0 + threadIdx.x;
        const int64_t g = i >> shift;
        const float r = __fmul_rn(__fsub_rn((float)codes[i], __half2float(zero[g])),
                                  __half2float(scale[g]));
        out[i] = __float2half_rn(r);
    }
}

int sm_count() {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

// Cluster size of the whole-tensor kernel: 16 CTAs where the device can place
// such a cluster (non-portable size), else the portable 8.
template <class Kern>
int whole_cluster_size(Kern kern) {
    static thread_local int cached = 0;
    if (cached) return cached;
    int best = 8;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed,
                             1) == cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr;
        attr.id = cudaLaunchAttributeClusterDimension;
        attr.val.clusterDim.x = 16;
        attr.val.clusterDim.y = 1;
        attr.val.clusterDim.z = 1;
        cfg.gridDim = dim3(16);
        cfg.blockDim = dim3(kWholeThreads);
        cfg.attrs = &attr;
        cfg.numAttrs = 1;
        int clusters = 0;
        if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) == cudaSuccess &&
            clusters > 0)
            best = 16;
    }
    cudaGetLastError();                               // a refused query leaves no error behind
    cached = best;
    return best;
}

}  // namespace

cudaError_t launch_meta_quantize(const __half* x, int64_t n, int log2g, uint8_t* codes,
                                 __half* scale, __half* zero, cudaStream_t stream) {
    // log2g < 0: one group over all n values (as is any single group)
    int lg = log2g;
    const int64_t ngroups = lg < 0 ? 1 : (n + ((int64_t)1 << lg) - 1) >> lg;
    if (ngroups == 1 && n > 4096) {
        const int cl = whole_cluster_size(meta_whole_kernel);
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr;
        attr.id = cudaLaunchAttributeClusterDimension;
        attr.val.clusterDim.x = cl;
        attr.val.clusterDim.y = 1;
        attr.val.clusterDim.z = 1;
        cfg.gridDim = dim3(cl);
        cfg.blockDim = dim3(kWholeThreads);
        cfg.dynamicSmemBytes = 0;
        cfg.stream = stream;
        cfg.attrs = &attr;
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, meta_whole_kernel, x, n, codes, scale, zero);
    }
    if (ngroups == 1) {                               // small tensor: one warp-wide group
        lg = 0;
        while (((int64_t)1 << lg) < n) ++lg;
    }
    const bool vec = lg >= 3;                         // 16-byte vectors never straddle groups
    const int lanes_log = vec ? lg - 3 : lg;
    const int lseg = lanes_log < 5 ? lanes_log : 5;
    const int64_t warps = (ngroups + (32 >> lseg) - 1) / (32 >> lseg);
    int64_t blocks = (warps + kGroupThreads / 32 - 1) / (kGroupThreads / 32);
    const int64_t cap = (int64_t)sm_count() * 16;
    if (blocks > cap) blocks = cap;
    if (vec)
        meta_group_vec_kernel<<<(unsigned)blocks, kGroupThreads, 0, stream>>>(
            x, n, lg, ngroups, codes, scale, zero);
    else
        meta_group_kernel<<<(unsigned)blocks, kGroupThreads, 0, stream>>>(x, n, lg, ngroups,
                                                                          codes, scale, zero);
    return cudaGetLastError();
}

// Many meta tensors: whole-tensor jobs (one group) as one cluster each, grouped
// jobs as block ranges of one grid, at most kMetaBatchMax jobs per launch.
cudaError_t launch_meta_quantize_batch(const MetaJobIn* jobs, int64_t count,
                                       cudaStream_t stream) {
    const int64_t cap = (int64_t)sm_count() * 16;
    MetaBatch whole, grouped;
    whole.count = grouped.count = 0;
    whole.first[0] = grouped.first[0] = 0;
    auto flush_whole = [&]() -> cudaError_t {
        if (whole.count == 0) return cudaSuccess;
        const int cl = whole_cluster_size(meta_whole_batch_kernel);
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr;
        attr.id = cudaLaunchAttributeClusterDimension;
        attr.val.clusterDim.x = cl;
        attr.val.clusterDim.y = 1;
        attr.val.clusterDim.z = 1;
        cfg.gridDim = dim3((unsigned)(whole.count * cl));
        cfg.blockDim = dim3(kWholeThreads);
        cfg.stream = stream;
        cfg.attrs = &attr;
        cfg.numAttrs = 1;
        const cudaError_t e = cudaLaunchKernelEx(&cfg, meta_whole_batch_kernel, whole);
        whole.count = 0;
        return e;
    };
    auto flush_grouped = [&]() -> cudaError_t {
        if (grouped.count == 0) return cudaSuccess;
        meta_group_batch_kernel<<<(unsigned)grouped.first[grouped.count], kGroupThreads, 0,
                                  stream>>>(grouped);
        grouped.count = 0;
        grouped.first[0] = 0;
        return cudaGetLastError();
    };
    for (int64_t i = 0; i < count; ++i) {
        const MetaJobIn& in = jobs[i];
        if (in.n == 0) continue;
        int lg = in.log2g;
        const int64_t ngroups = lg < 0 ? 1 : (in.n + ((int64_t)1 << lg) - 1) >> lg;
        MetaJob j;
        j.x = in.x;
        j.n = in.n;
        j.codes = in.codes;
        j.scale = in.scale;
        j.zero = in.zero;
        j.ngroups = ngroups;
        j.log2g = lg;
        if (ngroups == 1) {
            whole.job[whole.count++] = j;
            if (whole.count == kMetaBatchMax) {
                const cudaError_t e = flush_whole();
                if (e != cudaSuccess) return e;
            }
            continue;
        }
        const bool vec = lg >= 3;
        const int lanes_log = vec ? lg - 3 : lg;
        const int lseg = lanes_log < 5 ? lanes_log : 5;
        const int64_t warps = (ngroups + (32 >> lseg) - 1) / (32 >> lseg);
        int64_t blocks = (warps + kGroupThreads / 32 - 1) / (kGroupThreads / 32);
        if (blocks > cap) blocks = cap;
        if ((int64_t)grouped.first[grouped.count] + blocks > ((int64_t)1 << 30)) {
            const cudaError_t e = flush_grouped();
            if (e != cudaSuccess) return e;
        }
        grouped.job[grouped.count] = j;
        grouped.first[grouped.count + 1] = grouped.first[grouped.count] + (int)blocks;
        ++grouped.count;
        if (grouped.count == kMetaBatchMax) {
            const cudaError_t e = flush_grouped();
            if (e != cudaSuccess) return e;
        }
    }
    cudaError_t e = flush_whole();
    if (e != cudaSuccess) return e;
    return flush_grouped();
}

cudaError_t launch_meta_dequantize(const uint8_t* codes, const __half* scale, const __half* zero,
                                   int64_t n, int log2g, __half* out, cudaStream_t stream) {
    const int shift = log2g < 0 ? 62 : log2g;
    int64_t blocks = ((n >> 3) + kMdqThreads - 1) / kMdqThreads;
    if (blocks < 1) blocks = 1;
    const int64_t cap = (int64_t)sm_count() * 16;
    if (blocks > cap) blocks = cap;
    meta_dequant_kernel<<<(unsigned)blocks, kMdqThreads, 0, stream>>>(codes, scale, zero, n, shift,
                                                                      out);
    return cudaGetLastError();
}

}  // namespace hqq
