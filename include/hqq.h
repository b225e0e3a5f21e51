/*
 * hqq.h -- C ABI of libhqq: group-wise weight-only quantization of fp16 weight
 * matrices with the Half-Quadratic Quantization (HQQ) zero-point solver, bit
 * packing of the codes, and the matching dequantization, on NVIDIA B200 (sm_100a).
 *
 * Method: "Half-Quadratic Quantization of Large Machine Learning Models"
 * (Dropbox tech blog), section 2 (operators Q and Q^-1, l_p objective,
 * half-quadratic split with s fixed, sp1 generalised soft-threshold, sp2 mean
 * along the group axis, 1/s held instead of s) and section 4.1 (p = 0.7,
 * beta = 1, kappa = 1.01, 20 iterations, early exit when the error stops
 * improving, group-wise buffers).
 *
 * Conventions shared by every entry point
 *  - All buffer pointers are DEVICE pointers owned by the caller.  The library
 *    allocates nothing, keeps no per-call state and never synchronises: work is
 *    enqueued on `stream` (a cudaStream_t passed as void*, NULL = legacy default
 *    stream) and the call returns at once.
 *  - Arguments are validated on the host before anything is enqueued.  On any
 *    error nothing is launched and no output is touched.  HQQ_ERR_CUDA means the
 *    launch itself failed; the CUDA error is then readable with cudaGetLastError.
 *  - W is row-major [rows, cols]; a group is `group` consecutive weights along
 *    a row (the input axis), so cols must be a multiple of group and group g
 *    (0 <= g < rows*cols/group) covers flat elements [g*group, (g+1)*group).
 *  - Inputs must be finite.  Inputs and outputs must not overlap.
 *  - Thread safety: calls may be made concurrently from several host threads.
 */
#ifndef HQQ_H
#define HQQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes of every entry point. */
typedef enum hqq_status {
    HQQ_OK = 0,
    HQQ_ERR_NULL = 1,        /* a required pointer is NULL                       */
    HQQ_ERR_SHAPE = 2,       /* rows/cols negative, cols % group != 0, too large */
    HQQ_ERR_UNSUPPORTED = 3, /* nbits not in {2,3,4}, group not in {16..256, 2^k} */
    HQQ_ERR_PARAM = 4,       /* p not in (0,1], beta/kappa not > 0 and finite,
                                iters not in [0,255]                             */
    HQQ_ERR_ALIGN = 5,       /* W / W_out not 16-byte aligned; packed, zero_f32
                                or err_out not 4-byte; scale/zero not 2-byte     */
    HQQ_ERR_CUDA = 6         /* the kernel launch failed                         */
} hqq_status;

/* Solver defaults of the method's section 4.1. */
#define HQQ_DEFAULT_P 0.7f
#define HQQ_DEFAULT_BETA 1.0f
#define HQQ_DEFAULT_KAPPA 1.01f
#define HQQ_DEFAULT_ITERS 20

/*
 * Packed code layout (over the flat row-major element index i):
 *   nbits 4: byte  i/2  holds code i in bits 4*(i%2)   (even index = low nibble)
 *   nbits 2: byte  i/4  holds code i in bits 2*(i%4)   (first code = lowest bits)
 *   nbits 3: little-endian uint32 word i/10 holds code i in bits 3*(i%10);
 *            bits 30..31 and the slots past the last code are zero.
 * Returns the byte size of the packed buffer for rows*cols codes
 * (4 bit: N/2, 2 bit: N/4, 3 bit: 4*ceil(N/10)), or -1 for bad arguments.
 */
int64_t hqq_packed_bytes(int64_t rows, int64_t cols, int nbits);

/*
 * hqq_quantize -- HQQ quantization of one fp16 weight matrix (method section 2,
 * parameters of section 4.1), fused with code packing.
 *
 * Per group, in binary32 with round-to-nearest-even:
 *   1. s = (max - min) / (2^nbits - 1) and 1/s (s = 1/s = 1 when max == min);
 *      z = -min * (1/s).
 *   2. For t < iters: Wq = clamp(round(W*(1/s) + z), 0, 2^nbits - 1) (round
 *      half to even); e = sum over the group of |W - s(Wq - z)|^p.  If e is not
 *      strictly below the best error so far the group stops; otherwise z is
 *      recorded as the best z, W_e = sign(r) max(|r| - |r|^(p-1)/beta, 0) with
 *      r = W - s(Wq - z) (sp1), z = mean(Wq - (W - W_e)*(1/s)) (sp2), and
 *      beta = beta * kappa.
 *   3. codes = clamp(round(W*(1/s) + z_best), 0, 2^nbits - 1), packed as above.
 *
 *   W        [in]  fp16 [rows, cols] row-major, 16-byte aligned.
 *   rows     [in]  output features (>= 0).  cols: input features (>= 0).
 *   nbits    [in]  2, 3 or 4.
 *   group    [in]  16, 32, 64, 128 or 256; cols % group == 0.
 *   p, beta, kappa, iters [in]  solver parameters (0 < p <= 1, beta > 0,
 *                  kappa > 0, 0 <= iters <= 255; iters = 0 gives min-max
 *                  round-to-nearest).
 *   packed   [out] hqq_packed_bytes(rows, cols, nbits) bytes, 4-byte aligned.
 *   scale    [out] fp16 [rows, cols/group]: s of each group (multiply to
 *                  dequantize), 2-byte aligned.
 *   zero     [out] fp16 [rows, cols/group]: z_best of each group.
 *   stream   [in]  cudaStream_t (NULL = legacy default stream).
 * rows == 0 or cols == 0 is a valid no-op.
 */
int hqq_quantize(const void* W, int64_t rows, int64_t cols, int nbits, int group,
                 float p, float beta, float kappa, int iters,
                 void* packed, void* scale, void* zero, void* stream);

/*
 * hqq_quantize_ex -- hqq_quantize plus three optional per-group diagnostics
 * (any may be NULL; the float arrays must be 4-byte aligned):
 *   zero_f32  [out] float [rows, cols/group]: z_best before fp16 rounding.
 *   err_out   [out] float [rows, cols/group]: the solver's binary32 error sum
 *                   over the group of |W - s(Wq - z_best)|^p (the accepted
 *                   minimum); +inf when iters = 0 (no evaluation is made).
 *   iters_out [out] uint8 [rows, cols/group]: accepted iterations (0..iters);
 *                   a group evaluated its error iters_out+1 times, or iters
 *                   times when it never stopped early.
 */
int hqq_quantize_ex(const void* W, int64_t rows, int64_t cols, int nbits, int group,
                    float p, float beta, float kappa, int iters,
                    void* packed, void* scale, void* zero,
                    float* zero_f32, float* err_out, uint8_t* iters_out, void* stream);

/*
 * hqq_dequantize -- Q^-1 of the method's section 2: W_hat = s (Wq - z), computed
 * as fp16( (code - z) * s ) in binary32 from the stored fp16 s and z.
 *
 *   packed [in]  codes in the layout above, 4-byte aligned.
 *   scale, zero [in] fp16 [rows, cols/group], 2-byte aligned.
 *   rows, cols, nbits, group [in] as for hqq_quantize.
 *   W_out  [out] fp16 [rows, cols] row-major, 16-byte aligned.
 *   stream [in]  cudaStream_t (NULL = legacy default stream).
 */
int hqq_dequantize(const void* packed, const void* scale, const void* zero,
                   int64_t rows, int64_t cols, int nbits, int group,
                   void* W_out, void* stream);

/* Human-readable name of a status code (static string, never NULL). */
const char* hqq_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* HQQ_H */
