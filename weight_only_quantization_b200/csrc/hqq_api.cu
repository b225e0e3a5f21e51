// hqq_api.cu -- the extern "C" boundary of libhqq (declared in include/hqq.h):
// host-side validation, the per-call power tables and shrink thresholds, and
// kernel dispatch.  Nothing is launched unless every check passes.
#include <cmath>
#include <cstring>
#include <vector>

#include "../../include/hqq.h"
#include "hqq_params.cuh"

namespace hqq {
cudaError_t launch_quantize(const QuantParams& prm, int nbits, int group, cudaStream_t stream);
cudaError_t launch_quantize_half(const QuantParams& prm, int nbits, int group,
                                 cudaStream_t stream);
struct RtnParams {
    const __half* W;
    uint8_t* packed;
    __half* scale;
    __half* zero;
    float* zero_f32;
    float* err_out;
    uint8_t* iters_out;
    int64_t n_elems;
};
cudaError_t launch_rtn(const RtnParams& p, int nbits, int group, cudaStream_t stream);
cudaError_t launch_dequantize(const DequantParams& prm, int nbits, int log2_group,
                              cudaStream_t stream);
cudaError_t launch_linear(const LinearParams& prm, const void* X, int nbits, cudaStream_t stream);
cudaError_t launch_decode(const LinearParams& prm, const void* X, int nbits, int64_t packed_bytes,
                          cudaStream_t stream);
int64_t lowrank_workspace_bytes(int64_t N, int64_t K, int sketch);
int64_t lowrank_scratch_bytes();
cudaError_t lowrank_scratch(void** ptr);
cudaError_t launch_lowrank(const void* W, const uint8_t* packed, const __half* scale,
                           const __half* zero, int64_t N, int64_t K, int nbits, int log2_group,
                           int rank, int sketch, int power_iters, const float* omega, float* B,
                           float* A, float* sigma, void* ws, cudaStream_t st);
cudaError_t launch_meta_quantize(const __half* x, int64_t n, int log2g, uint8_t* codes,
                                 __half* scale, __half* zero, cudaStream_t stream);
cudaError_t launch_meta_dequantize(const uint8_t* codes, const __half* scale, const __half* zero,
                                   int64_t n, int log2g, __half* out, cudaStream_t stream);
cudaError_t launch_meta_quantize_batch(const MetaJobIn* jobs, int64_t count, cudaStream_t stream);

namespace {

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int log2_of_group(int group) {
    switch (group) {
        case 16: return 4;
        case 32: return 5;
        case 64: return 6;
        case 128: return 7;
        case 256: return 8;
        default: return -1;
    }
}

// Table of |x|^p for one exponent p (see PowTable).  Each entry is the double
// library value rounded once to binary32.
void build_pow_table(PowTable& t, float p) {
    const double pd = (double)p;
    for (int e = 0; e < 256; ++e) {
        if (e == 0)
            t.two_pk[e] = p > 0.0f ? 0.0f : (p < 0.0f ? INFINITY : 1.0f);
        else if (e == 255)
            t.two_pk[e] = p > 0.0f ? INFINITY : (p < 0.0f ? 0.0f : 1.0f);
        else
            t.two_pk[e] = (float)std::exp2(pd * (double)(e - 127));
    }
    for (int j = 0; j < 32; ++j) {
        const double c = 1.0 + (double)(2 * j + 1) / 64.0;
        t.cj_p[j] = (float)std::pow(c, pd);
        const float cf = (float)c;
        t.inv_cj[j] = 1.0f / cf;
    }
    t.a1 = p;
    t.a2 = (float)(pd * (pd - 1.0) / 2.0);
    t.a3 = (float)(pd * (pd - 1.0) * (pd - 2.0) / 6.0);
}

// Tables depend on p only; reuse them across calls made by the same host thread.
struct TableCache {
    bool valid = false;
    uint32_t p_bits = 0;
    PowTable tp, tq;
};
thread_local TableCache g_cache;

// Alignment of the packed codes: the kernels move 8-bit units as 8-byte words,
// the other widths in units of at most 4 bytes.
uintptr_t packed_align(int nbits) { return nbits == 8 ? 8 : 4; }

// log2 of a second-level (meta) group: -1 for 0 (one group over everything),
// -2 when the size is not a power of two up to 2^30.
int meta_log2(int64_t mgroup) {
    if (mgroup == 0) return -1;
    for (int k = 0; k <= 30; ++k)
        if (mgroup == ((int64_t)1 << k)) return k;
    return -2;
}

int validate_common(int64_t rows, int64_t cols, int nbits, int group) {
    if (rows < 0 || cols < 0) return HQQ_ERR_SHAPE;
    if (nbits != 1 && nbits != 2 && nbits != 3 && nbits != 4 && nbits != 8)
        return HQQ_ERR_UNSUPPORTED;
    if (log2_of_group(group) < 0) return HQQ_ERR_UNSUPPORTED;
    if (cols % group != 0) return HQQ_ERR_SHAPE;
    if (rows > 0 && cols > ((int64_t)1 << 46) / rows) return HQQ_ERR_SHAPE;
    return HQQ_OK;
}

}  // namespace
}  // namespace hqq

using namespace hqq;

extern "C" int64_t hqq_packed_bytes(int64_t rows, int64_t cols, int nbits) {
    if (rows < 0 || cols < 0) return -1;
    if (rows > 0 && cols > ((int64_t)1 << 46) / rows) return -1;
    const int64_t n = rows * cols;
    switch (nbits) {
        case 8: return n;
        case 4: return (n + 1) / 2;
        case 2: return (n + 3) / 4;
        case 1: return (n + 7) / 8;
        case 3: return 4 * ((n + 9) / 10);
        default: return -1;
    }
}

extern "C" const char* hqq_status_string(int status) {
    switch (status) {
        case HQQ_OK: return "HQQ_OK";
        case HQQ_ERR_NULL: return "HQQ_ERR_NULL: a required pointer is NULL";
        case HQQ_ERR_SHAPE: return "HQQ_ERR_SHAPE: bad rows/cols or cols not a multiple of group";
        case HQQ_ERR_UNSUPPORTED: return "HQQ_ERR_UNSUPPORTED: nbits must be 1/2/3/4/8, group 16..256 (power of two), meta group 0 or a power of two up to 2^30";
        case HQQ_ERR_PARAM: return "HQQ_ERR_PARAM: need 0<p<=1, beta>0, kappa>0 (finite), 0<=iters<=255";
        case HQQ_ERR_ALIGN: return "HQQ_ERR_ALIGN: W/W_out/X/meta x/meta out need 16-byte, meta codes and 8-bit packed 8-byte, packed/zero_f32 4-byte, scale/zero 2-byte alignment";
        case HQQ_ERR_CUDA: return "HQQ_ERR_CUDA: kernel launch failed (see cudaGetLastError)";
        case HQQ_ERR_SCRATCH: return "HQQ_ERR_SCRATCH: the problem needs more scratch than the fixed array of hqq_lowrank_noalloc holds (hqq_lowrank_noalloc_max_bytes)";
        default: return "HQQ: unknown status";
    }
}

namespace {

// Shared body of hqq_quantize_ex (binary32 solver) and hqq_quantize_half.
int quantize_common(const void* W, int64_t rows, int64_t cols, int nbits, int group, float p,
                    float beta, float kappa, int iters, void* packed, void* scale, void* zero,
                    float* zero_f32, float* err_out, uint8_t* iters_out, bool half,
                    uint8_t* half_out, void* stream) {
    int st = validate_common(rows, cols, nbits, group);
    if (st != HQQ_OK) return st;
    if (!(p > 0.0f && p <= 1.0f)) return HQQ_ERR_PARAM;
    if (!(beta > 0.0f) || !std::isfinite(beta)) return HQQ_ERR_PARAM;
    if (!(kappa > 0.0f) || !std::isfinite(kappa)) return HQQ_ERR_PARAM;
    if (iters < 0 || iters > kMaxIters) return HQQ_ERR_PARAM;
    const int64_t n = rows * cols;
    if (n == 0) return HQQ_OK;
    if (!W || !packed || !scale || !zero) return HQQ_ERR_NULL;
    if (!aligned(W, 16) || !aligned(packed, packed_align(nbits)) || !aligned(scale, 2) ||
        !aligned(zero, 2) || (zero_f32 && !aligned(zero_f32, 4)) ||
        (err_out && !aligned(err_out, 4)))
        return HQQ_ERR_ALIGN;

    if (iters == 0 && !half) {         // min-max round-to-nearest: the streaming kernel
        RtnParams rp;
        rp.W = static_cast<const __half*>(W);
        rp.packed = static_cast<uint8_t*>(packed);
        rp.scale = static_cast<__half*>(scale);
        rp.zero = static_cast<__half*>(zero);
        rp.zero_f32 = zero_f32;
        rp.err_out = err_out;
        rp.iters_out = iters_out;
        rp.n_elems = n;
        const cudaError_t err = launch_rtn(rp, nbits, group, static_cast<cudaStream_t>(stream));
        return err == cudaSuccess ? HQQ_OK : HQQ_ERR_CUDA;
    }

    QuantParams prm;
    std::memset(&prm, 0, sizeof prm);
    prm.W = static_cast<const __half*>(W);
    prm.packed = static_cast<uint8_t*>(packed);
    prm.scale = static_cast<__half*>(scale);
    prm.zero = static_cast<__half*>(zero);
    prm.zero_f32 = zero_f32;
    prm.err_out = err_out;
    prm.iters_out = iters_out;
    prm.half_out = half_out;
    prm.n_groups = n / group;
    prm.n_elems = n;
    prm.iters = iters;
    prm.beta = beta;
    prm.kappa = kappa;

    uint32_t pbits;
    std::memcpy(&pbits, &p, 4);
    if (!g_cache.valid || g_cache.p_bits != pbits) {
        build_pow_table(g_cache.tp, p);
        build_pow_table(g_cache.tq, p - 1.0f);
        g_cache.p_bits = pbits;
        g_cache.valid = true;
    }
    prm.tp = g_cache.tp;
    prm.tq = g_cache.tq;

    // Shrink shortcut: |r| - |r|^(p-1)/beta > 0  <=>  |r| > T = beta^(-1/(2-p)).
    // Below T lowered by a 1e-4 relative margin (far above the rounding error
    // of the binary32 table power), W_e is exactly zero, so the kernel may skip
    // it.  The half-precision shrink rounds the power and its quotient by beta
    // to fp16 (2^-11 each); below T (1 - 1e-2) the computed |r|^(p-1)/beta still
    // exceeds |r| by at least (1 + (2-p) 1e-2)(1 - 2^-10) > 1, so its W_e is
    // exactly zero too.
    float bt = beta;
    for (int t = 0; t < iters; ++t) {
        const double T = std::pow((double)bt, -1.0 / (2.0 - (double)p));
        prm.shrink_thr[t] = (float)(T * (1.0 - 1e-4));
        prm.shrink_thr16[t] = (float)(T * (1.0 - 1e-2));
        bt = bt * kappa;
    }

    const cudaStream_t cs = static_cast<cudaStream_t>(stream);
    const cudaError_t err = half ? launch_quantize_half(prm, nbits, group, cs)
                                 : launch_quantize(prm, nbits, group, cs);
    return err == cudaSuccess ? HQQ_OK : HQQ_ERR_CUDA;
}

}  // namespace

extern "C" int hqq_quantize_ex(const void* W, int64_t rows, int64_t cols, int nbits, int group,
                               float p, float beta, float kappa, int iters, void* packed,
                               void* scale, void* zero, float* zero_f32, float* err_out,
                               uint8_t* iters_out, void* stream) {
    return quantize_common(W, rows, cols, nbits, group, p, beta, kappa, iters, packed, scale,
                           zero, zero_f32, err_out, iters_out, false, nullptr, stream);
}

extern "C" int hqq_quantize_half(const void* W, int64_t rows, int64_t cols, int nbits,
                                 int group, float p, float beta, float kappa, int iters,
                                 void* packed, void* scale, void* zero, float* zero_f32,
                                 float* err_out, uint8_t* iters_out, uint8_t* half_out,
                                 void* stream) {
    return quantize_common(W, rows, cols, nbits, group, p, beta, kappa, iters, packed, scale,
                           zero, zero_f32, err_out, iters_out, true, half_out, stream);
}

extern "C" int hqq_quantize(const void* W, int64_t rows, int64_t cols, int nbits, int group,
                            float p, float beta, float kappa, int iters, void* packed,
                            void* scale, void* zero, void* stream) {
    return hqq_quantize_ex(W, rows, cols, nbits, group, p, beta, kappa, iters, packed, scale,
                           zero, nullptr, nullptr, nullptr, stream);
}

extern "C" int hqq_dequantize(const void* packed, const void* scale, const void* zero,
                              int64_t rows, int64_t cols, int nbits, int group, void* W_out,
                              void* stream) {
    int st = validate_common(rows, cols, nbits, group);
    if (st != HQQ_OK) return st;
    const int64_t n = rows * cols;
    if (n == 0) return HQQ_OK;
    if (!packed || !scale || !zero || !W_out) return HQQ_ERR_NULL;
    if (!aligned(packed, packed_align(nbits)) || !aligned(scale, 2) || !aligned(zero, 2) ||
        !aligned(W_out, 16))
        return HQQ_ERR_ALIGN;
    DequantParams prm;
    std::memset(&prm, 0, sizeof prm);
    prm.packed = static_cast<const uint8_t*>(packed);
    prm.scale = static_cast<const __half*>(scale);
    prm.zero = static_cast<const __half*>(zero);
    prm.out = static_cast<__half*>(W_out);
    prm.n_units = n / 8;
    prm.n_words = (uint32_t)((n + 9) / 10 < ((int64_t)1 << 32) ? (n + 9) / 10 : 0);
    prm.group = group;
    const cudaError_t err = launch_dequantize(prm, nbits, log2_of_group(group),
                                              static_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? HQQ_OK : HQQ_ERR_CUDA;
}

extern "C" int64_t hqq_meta_groups(int64_t n, int64_t mgroup) {
    if (n < 0 || mgroup < 0) return -1;
    if (n == 0) return 0;
    if (mgroup == 0) return 1;
    return (n + mgroup - 1) / mgroup;
}

extern "C" int hqq_meta_quantize(const void* x, int64_t n, int64_t mgroup, uint8_t* codes,
                                 void* scale, void* zero, void* stream) {
    if (n < 0 || mgroup < 0 || n > ((int64_t)1 << 40)) return HQQ_ERR_SHAPE;
    const int lg = meta_log2(mgroup);
    if (lg == -2) return HQQ_ERR_UNSUPPORTED;
    if (n == 0) return HQQ_OK;
    if (!x || !codes || !scale || !zero) return HQQ_ERR_NULL;
    if (!aligned(x, 16) || !aligned(codes, 8) || !aligned(scale, 2) || !aligned(zero, 2))
        return HQQ_ERR_ALIGN;
    const cudaError_t err = launch_meta_quantize(
        static_cast<const __half*>(x), n, lg, codes, static_cast<__half*>(scale),
        static_cast<__half*>(zero), static_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? HQQ_OK : HQQ_ERR_CUDA;
}

extern "C" int hqq_meta_quantize_batch(const hqq_meta_job* jobs, int64_t count, void* stream) {
    if (count < 0) return HQQ_ERR_SHAPE;
    if (count == 0) return HQQ_OK;
    if (!jobs) return HQQ_ERR_NULL;
    for (int64_t i = 0; i < count; ++i) {          // every job checked before any launch
        const hqq_meta_job& j = jobs[i];
        if (j.n < 0 || j.mgroup < 0 || j.n > ((int64_t)1 << 40)) return HQQ_ERR_SHAPE;
        if (meta_log2(j.mgroup) == -2) return HQQ_ERR_UNSUPPORTED;
        if (j.n == 0) continue;
        if (!j.x || !j.codes || !j.scale || !j.zero) return HQQ_ERR_NULL;
        if (!aligned(j.x, 16) || !aligned(j.codes, 8) || !aligned(j.scale, 2) ||
            !aligned(j.zero, 2))
            return HQQ_ERR_ALIGN;
    }
    std::vector<MetaJobIn> in((size_t)count);
    for (int64_t i = 0; i < count; ++i) {
        in[i].x = static_cast<const __half*>(jobs[i].x);
        in[i].n = jobs[i].n;
        in[i].log2g = meta_log2(jobs[i].mgroup);
        in[i].codes = jobs[i].codes;
        in[i].scale = static_cast<__half*>(jobs[i].scale);
        in[i].zero = static_cast<__half*>(jobs[i].zero);
    }
    const cudaError_t err =
        launch_meta_quantize_batch(in.data(), count, static_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? HQQ_OK : HQQ_ERR_CUDA;
}

extern "C" int hqq_meta_dequantize(const uint8_t* codes, const void* scale, const void* zero,
                                   int64_t n, int64_t mgroup, void* out, void* stream) {
    if (n < 0 || mgroup < 0 || n > ((int64_t)1 << 40)) return HQQ_ERR_SHAPE;
    const int lg = meta_log2(mgroup);
    if (lg == -2) return HQQ_ERR_UNSUPPORTED;
    if (n == 0) return HQQ_OK;
    if (!codes || !scale || !zero || !out) return HQQ_ERR_NULL;
    if (!aligned(codes, 8) || !aligned(scale, 2) || !aligned(zero, 2) || !aligned(out, 16))
        return HQQ_ERR_ALIGN;
    const cudaError_t err = launch_meta_dequantize(
        codes, static_cast<const __half*>(scale), static_cast<const __half*>(zero), n, lg,
        static_cast<__half*>(out), static_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? HQQ_OK : HQQ_ERR_CUDA;
}

namespace {
// Checks one 8-bit meta form and fills its kernel image; HQQ_OK or an error.
int meta8_image(const hqq_meta8* m, Meta8& out) {
    if (!m->codes || !m->scale || !m->zero) return HQQ_ERR_NULL;
    if (m->group < 0) return HQQ_ERR_SHAPE;
    const int lg = meta_log2(m->group);
    if (lg == -2) return HQQ_ERR_UNSUPPORTED;
    if (!aligned(m->scale, 2) || !aligned(m->zero, 2)) return HQQ_ERR_ALIGN;
    out.codes = m->codes;
    out.scale = static_cast<const __half*>(m->scale);
    out.zero = static_cast<const __half*>(m->zero);
    out.shift = lg < 0 ? 62 : lg;
    return HQQ_OK;
}
}  // namespace

extern "C" int hqq_dequantize_meta(const void* packed, const hqq_meta8* zero_q, const void* scale,
                                   const hqq_meta8* scale_q, int64_t rows, int64_t cols,
                                   int nbits, int group, void* W_out, void* stream) {
    int st = validate_common(rows, cols, nbits, group);
    if (st != HQQ_OK) return st;
    if (scale && scale_q) return HQQ_ERR_PARAM;
    const int64_t n = rows * cols;
    if (n == 0) return HQQ_OK;
    if (!packed || !zero_q || !W_out || (!scale && !scale_q)) return HQQ_ERR_NULL;
    DequantParams prm;
    std::memset(&prm, 0, sizeof prm);
    if ((st = meta8_image(zero_q, prm.zq)) != HQQ_OK) return st;
    if (scale_q && (st = meta8_image(scale_q, prm.sq)) != HQQ_OK) return st;
    if (!aligned(packed, packed_align(nbits)) || !aligned(W_out, 16) ||
        (scale && !aligned(scale, 2)))
        return HQQ_ERR_ALIGN;
    prm.packed = static_cast<const uint8_t*>(packed);
    prm.scale = static_cast<const __half*>(scale);
    prm.out = static_cast<__half*>(W_out);
    prm.n_units = n / 8;
    prm.n_words = (uint32_t)((n + 9) / 10 < ((int64_t)1 << 32) ? (n + 9) / 10 : 0);
    prm.group = group;
    const cudaError_t err = launch_dequantize(prm, nbits, log2_of_group(group),
                                              static_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? HQQ_OK : HQQ_ERR_CUDA;
}

namespace {
// Shared body of hqq_linear and hqq_linear_meta: zero_q / scale_q (host
// structs, nullable) replace zero / scale by their 8-bit forms.
int linear_common(const void* X, int64_t M, const void* packed, const void* scale,
                  const void* zero, const hqq_meta8* zero_q, const hqq_meta8* scale_q,
                  int64_t rows, int64_t cols, int nbits, int group, void* Y, int* status,
                  void* stream) {
    int st = validate_common(rows, cols, nbits, group);
    if (st != HQQ_OK) return st;
    // the grid holds 65535 feature tiles of 128; token coordinates of the
    // 512-token tiles stay below 2^31
    if (M < 0 || M > (((int64_t)1 << 31) - 1024)) return HQQ_ERR_SHAPE;
    if (rows > (int64_t)65535 * 128) return HQQ_ERR_SHAPE;
    if (M == 0 || rows == 0 || cols == 0) return HQQ_OK;
    if (!X || !packed || !Y || (!scale && !scale_q) || (!zero && !zero_q)) return HQQ_ERR_NULL;
    LinearParams prm;
    std::memset(&prm, 0, sizeof prm);
    if (zero_q && (st = meta8_image(zero_q, prm.zq)) != HQQ_OK) return st;
    if (scale_q && (st = meta8_image(scale_q, prm.sq)) != HQQ_OK) return st;
    if (!aligned(X, 16) || !aligned(packed, packed_align(nbits)) ||
        (scale && !aligned(scale, 2)) || (zero && !aligned(zero, 2)) || !aligned(Y, 2) ||
        (status && !aligned(status, 4)))
        return HQQ_ERR_ALIGN;
    prm.packed = static_cast<const uint8_t*>(packed);
    prm.scale = static_cast<const __half*>(scale);
    prm.zero = static_cast<const __half*>(zero);
    prm.Y = static_cast<__half*>(Y);
    prm.status = status;
    prm.M = M;
    prm.N = rows;
    prm.K = cols;
    prm.log2_group = log2_of_group(group);
    // few tokens: warp-level MMAs fed from registers; more: tensor-memory tiles
    const cudaError_t err = M <= decode_max_tokens(nbits)
        ? launch_decode(prm, X, nbits, hqq_packed_bytes(rows, cols, nbits),
                        static_cast<cudaStream_t>(stream))
        : launch_linear(prm, X, nbits, static_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? HQQ_OK : HQQ_ERR_CUDA;
}
}  // namespace

extern "C" int hqq_linear(const void* X, int64_t M, const void* packed, const void* scale,
                          const void* zero, int64_t rows, int64_t cols, int nbits, int group,
                          void* Y, int* status, void* stream) {
    if (M > 0 && rows > 0 && cols > 0 && (!scale || !zero)) {
        const int st = validate_common(rows, cols, nbits, group);
        return st != HQQ_OK ? st : HQQ_ERR_NULL;
    }
    return linear_common(X, M, packed, scale, zero, nullptr, nullptr, rows, cols, nbits, group, Y,
                         status, stream);
}

extern "C" int hqq_linear_meta(const void* X, int64_t M, const void* packed,
                               const hqq_meta8* zero_q, const void* scale,
                               const hqq_meta8* scale_q, int64_t rows, int64_t cols, int nbits,
                               int group, void* Y, int* status, void* stream) {
    if (scale && scale_q) return HQQ_ERR_PARAM;
    if (M > 0 && rows > 0 && cols > 0 && !zero_q) return HQQ_ERR_NULL;
    return linear_common(X, M, packed, scale, nullptr, zero_q, scale_q, rows, cols, nbits, group,
                         Y, status, stream);
}

extern "C" int64_t hqq_lowrank_workspace_bytes(int64_t rows, int64_t cols, int sketch) {
    if (rows < 0 || cols < 0 || (sketch != 16 && sketch != 32 && sketch != 64)) return -1;
    return lowrank_workspace_bytes(rows, cols, sketch);
}

extern "C" int hqq_lowrank(const void* W, const void* packed, const void* scale, const void* zero,
                           int64_t rows, int64_t cols, int nbits, int group, int rank, int sketch,
                           int power_iters, const float* omega, float* B, float* A, float* sigma,
                           void* workspace, int64_t workspace_bytes, void* stream) {
    int st = validate_common(rows, cols, nbits, group);
    if (st != HQQ_OK) return st;
    if (sketch != 16 && sketch != 32 && sketch != 64) return HQQ_ERR_UNSUPPORTED;
    if (rank < 1 || rank > sketch || power_iters < 0 || power_iters > 16) return HQQ_ERR_PARAM;
    if (rows < sketch || cols < sketch || cols >= ((int64_t)1 << 30)) return HQQ_ERR_SHAPE;
    if (!W || !packed || !scale || !zero || !omega || !B || !A || !workspace) return HQQ_ERR_NULL;
    if (workspace_bytes < lowrank_workspace_bytes(rows, cols, sketch)) return HQQ_ERR_PARAM;
    if (!aligned(W, 16) || !aligned(packed, packed_align(nbits)) || !aligned(scale, 2) ||
        !aligned(zero, 2) || !aligned(omega, 16) || !aligned(B, 4) || !aligned(A, 4) ||
        (sigma && !aligned(sigma, 4)) || !aligned(workspace, 256))
        return HQQ_ERR_ALIGN;
    float* sg = sigma;
    float* scratch_sigma = nullptr;
    if (!sg) {                          // the solver always writes sigma: use workspace slack
        scratch_sigma = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                                 lowrank_workspace_bytes(rows, cols, sketch) - 256);
        sg = scratch_sigma;
    }
    const cudaError_t err = launch_lowrank(
        W, static_cast<const uint8_t*>(packed), static_cast<const __half*>(scale),
        static_cast<const __half*>(zero), rows, cols, nbits, log2_of_group(group), rank, sketch,
        power_iters, omega, B, A, sg, workspace, static_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? HQQ_OK : HQQ_ERR_CUDA;
}

extern "C" int64_t hqq_lowrank_noalloc_max_bytes(void) { return lowrank_scratch_bytes(); }

extern "C" int hqq_lowrank_noalloc(const void* W, const void* packed, const void* scale,
                                   const void* zero, int64_t rows, int64_t cols, int nbits,
                                   int group, int rank, int sketch, int power_iters,
                                   const float* omega, float* B, float* A, float* sigma,
                                   void* stream) {
    // the argument checks of hqq_lowrank that come before its workspace, so
    // that a bad call is reported as such before any device lookup
    const int st = validate_common(rows, cols, nbits, group);
    if (st != HQQ_OK) return st;
    if (sketch != 16 && sketch != 32 && sketch != 64) return HQQ_ERR_UNSUPPORTED;
    if (rank < 1 || rank > sketch || power_iters < 0 || power_iters > 16) return HQQ_ERR_PARAM;
    if (rows < sketch || cols < sketch || cols >= ((int64_t)1 << 30)) return HQQ_ERR_SHAPE;
    if (lowrank_workspace_bytes(rows, cols, sketch) > lowrank_scratch_bytes())
        return HQQ_ERR_SCRATCH;
    if (!W || !packed || !scale || !zero || !omega || !B || !A) return HQQ_ERR_NULL;
    void* scratch = nullptr;
    if (lowrank_scratch(&scratch) != cudaSuccess) return HQQ_ERR_CUDA;
    return hqq_lowrank(W, packed, scale, zero, rows, cols, nbits, group, rank, sketch,
                       power_iters, omega, B, A, sigma, scratch, lowrank_scratch_bytes(), stream);
}
