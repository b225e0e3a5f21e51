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
    HQQ_ERR_UNSUPPORTED = 3, /* nbits not in {1,2,3,4,8}, group not in {16..256,
                                2^k}, meta group not 0 or 2^k                    */
    HQQ_ERR_PARAM = 4,       /* p not in (0,1], beta/kappa not > 0 and finite,
                                iters not in [0,255]                             */
    HQQ_ERR_ALIGN = 5,       /* W / W_out / X not 16-byte aligned; packed not
                                4-byte (8-byte at 8 bits); zero_f32 or err_out
                                not 4-byte; scale/zero not 2-byte                */
    HQQ_ERR_CUDA = 6,        /* the kernel launch failed                         */
    HQQ_ERR_SCRATCH = 7      /* hqq_lowrank_noalloc: the problem's workspace is
                                larger than its fixed scratch array              */
} hqq_status;

/* Solver defaults of the method's section 4.1. */
#define HQQ_DEFAULT_P 0.7f
#define HQQ_DEFAULT_BETA 1.0f
#define HQQ_DEFAULT_KAPPA 1.01f
#define HQQ_DEFAULT_ITERS 20

/*
 * Packed code layout (over the flat row-major element index i):
 *   nbits 8: byte  i    holds code i
 *   nbits 4: byte  i/2  holds code i in bits 4*(i%2)   (even index = low nibble)
 *   nbits 2: byte  i/4  holds code i in bits 2*(i%4)   (first code = lowest bits)
 *   nbits 1: byte  i/8  holds code i in bit  i%8       (first code = lowest bit)
 *   nbits 3: little-endian uint32 word i/10 holds code i in bits 3*(i%10);
 *            bits 30..31 and the slots past the last code are zero.
 * Returns the byte size of the packed buffer for rows*cols codes
 * (8 bit: N, 4 bit: ceil(N/2), 2 bit: ceil(N/4), 1 bit: ceil(N/8),
 * 3 bit: 4*ceil(N/10)), or -1 for bad arguments.
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
 *   nbits    [in]  1, 2, 3, 4 or 8 (section 4.1's table has 8/4/3/2; 1 bit
 *                  is the same operator with two levels).
 *   group    [in]  16, 32, 64, 128 or 256; cols % group == 0.
 *   p, beta, kappa, iters [in]  solver parameters (0 < p <= 1, beta > 0,
 *                  kappa > 0, 0 <= iters <= 255; iters = 0 gives min-max
 *                  round-to-nearest).
 *   packed   [out] hqq_packed_bytes(rows, cols, nbits) bytes, 4-byte aligned
 *                  (8-byte aligned at 8 bits).
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
 * hqq_quantize_half -- hqq_quantize_ex with the solver in half precision, the
 * way the method runs it: section 2.2 holds 1/s because it "is more stable in
 * half precision", and section 3 runs the whole solve on the GPU in half
 * precision.  The page fixes no rounding step; this library takes:
 *   - every element-wise step (W*(1/s), + z, Wq - z, s*(.), W - ., the shrink's
 *     power, quotient and difference, the sp2 terms) rounded once to fp16,
 *     round to nearest even, never fused;
 *   - |x|^p and |x|^(p-1) as the binary32 table power rounded to fp16;
 *   - the group reductions accumulated in binary32 (pairwise over contiguous
 *     halves) and rounded once to fp16: the error is the group MEAN of |r|^p
 *     (compared in fp16), z the group mean of the sp2 terms;
 *   - p, beta, kappa and beta_t as in hqq_quantize (binary32 scalars);
 *   - s = fp16(fp16(max - min)/L), 1/s = fp16(1/s), z = -fp16(min*(1/s))
 *     (s = 1/s = 1, z = -min for a constant group).
 * fp16 cannot hold every group's intermediates: a group whose largest |W|
 * exceeds 8192, whose s rounds to zero, or whose max|W|*(1/s) (binary32
 * product) exceeds 2^14 is solved in single precision exactly as
 * hqq_quantize_ex solves it.  iters = 0 gives min-max round-to-nearest with
 * these fp16 steps.
 *   Arguments as for hqq_quantize_ex, except:
 *   err_out   [out] float [rows, cols/group] or NULL: the accepted minimum of
 *                   the group's error -- its fp16 mean for a group solved in
 *                   half precision, the binary32 sum otherwise; +inf when
 *                   iters = 0.
 *   half_out  [out] uint8 [rows, cols/group] or NULL: 1 where the group was
 *                   solved in half precision, 0 where in single precision.
 * Errors as for hqq_quantize.
 */
int hqq_quantize_half(const void* W, int64_t rows, int64_t cols, int nbits, int group,
                      float p, float beta, float kappa, int iters,
                      void* packed, void* scale, void* zero,
                      float* zero_f32, float* err_out, uint8_t* iters_out, uint8_t* half_out,
                      void* stream);

/*
 * hqq_dequantize -- Q^-1 of the method's section 2: W_hat = s (Wq - z), computed
 * as fp16( (code - z) * s ) in binary32 from the stored fp16 s and z.
 *
 *   packed [in]  codes in the layout above, 4-byte aligned (8 at 8 bits).
 *   scale, zero [in] fp16 [rows, cols/group], 2-byte aligned.
 *   rows, cols, nbits, group [in] as for hqq_quantize.
 *   W_out  [out] fp16 [rows, cols] row-major, 16-byte aligned.
 *   stream [in]  cudaStream_t (NULL = legacy default stream).
 */
int hqq_dequantize(const void* packed, const void* scale, const void* zero,
                   int64_t rows, int64_t cols, int nbits, int group,
                   void* W_out, void* stream);

/*
 * 8-bit storage of the per-group zero points and scales (the method's section
 * 4.1: its settings keep the zero points in 8 bits, with neither grouping nor
 * optimisation; the starred row of its table also keeps the scales in 8 bits,
 * in groups of 128).
 *
 * A meta tensor is an fp16 vector x of n values -- a matrix's zero or scale
 * output of hqq_quantize, in flat row-major order.  It is cut into groups of
 * `mgroup` consecutive values (the last group may be shorter); mgroup = 0 means
 * one group over all n values.  mgroup is 0 or a power of two 1 .. 2^30.  Each
 * group is min-max round-to-nearest quantized with 255 levels, in binary32:
 *   s = (max - min) / 255 and 1/s (s = 1/s = 1 when max == min);
 *   z = -min * (1/s);  c = clamp(round(x * (1/s) + z), 0, 255), half to even;
 * and its s and z are stored in fp16.  The inverse restores
 *   x' = fp16( (c - z) * s )  with the group's stored fp16 s and z.
 */

/* Second-level groups of an n-value meta tensor: 0 when n == 0, 1 when
   mgroup == 0, else ceil(n / mgroup); -1 for negative arguments. */
int64_t hqq_meta_groups(int64_t n, int64_t mgroup);

/*
 * hqq_meta_quantize -- 8-bit codes of a meta tensor.
 *   x      [in]  fp16 [n], 16-byte aligned.
 *   n      [in]  number of values (>= 0; n == 0 is a valid no-op).
 *   mgroup [in]  0 or a power of two up to 2^30 (else HQQ_ERR_UNSUPPORTED).
 *   codes  [out] uint8 [n], 8-byte aligned.
 *   scale, zero [out] fp16 [hqq_meta_groups(n, mgroup)], 2-byte aligned.
 *   stream [in]  cudaStream_t (NULL = legacy default stream).
 * With mgroup = 0 (or one group covering all n values) the whole tensor is
 * reduced by one cluster of thread blocks; that form is meant for the meta
 * tensor of one matrix (millions of values), not for billions.
 */
int hqq_meta_quantize(const void* x, int64_t n, int64_t mgroup, uint8_t* codes,
                      void* scale, void* zero, void* stream);

/* One meta tensor of a batch: the arguments of hqq_meta_quantize. */
typedef struct hqq_meta_job {
    const void* x;          /* fp16 [n], 16-byte aligned                    */
    int64_t n;              /* values (>= 0; 0 is skipped)                  */
    int64_t mgroup;         /* 0 or a power of two up to 2^30               */
    uint8_t* codes;         /* uint8 [n], 8-byte aligned                    */
    void* scale;            /* fp16 [hqq_meta_groups(n, mgroup)]            */
    void* zero;             /* fp16 [hqq_meta_groups(n, mgroup)]            */
} hqq_meta_job;

/*
 * hqq_meta_quantize_batch -- hqq_meta_quantize of `count` meta tensors at once
 * (say every zero-point and scale tensor of a layer or of a whole model),
 * with the same results, bit for bit, as one call per tensor.  The tensors
 * share launches: each one-group tensor is reduced by a cluster of thread
 * blocks of its own and the grouped tensors split one grid, up to 128 tensors
 * per launch, so that a batch of small tensors occupies the whole GPU.
 *   jobs   [in] HOST array of `count` descriptors (device pointers inside);
 *              it may be freed when the call returns.
 *   count  [in] >= 0 (0: no-op).
 * Every descriptor is validated first (errors as for hqq_meta_quantize); on
 * any error nothing is launched.  Tensors of one batch must not overlap each
 * other's outputs.
 */
int hqq_meta_quantize_batch(const hqq_meta_job* jobs, int64_t count, void* stream);

/*
 * hqq_meta_dequantize -- the inverse: out = fp16((c - z) * s) per value.
 *   codes [in] uint8 [n], 8-byte aligned.   scale, zero [in] fp16, 2-byte aligned.
 *   n, mgroup [in] as for hqq_meta_quantize.   out [out] fp16 [n], 16-byte aligned.
 */
int hqq_meta_dequantize(const uint8_t* codes, const void* scale, const void* zero,
                        int64_t n, int64_t mgroup, void* out, void* stream);

/* The 8-bit form of one meta tensor, as hqq_meta_quantize writes it (device
   pointers; the struct itself lives in host memory). */
typedef struct hqq_meta8 {
    const uint8_t* codes;   /* uint8 [n]                                   */
    const void* scale;      /* fp16 [hqq_meta_groups(n, group)]            */
    const void* zero;       /* fp16 [hqq_meta_groups(n, group)]            */
    int64_t group;          /* 0 or a power of two, as mgroup above         */
} hqq_meta8;

/*
 * hqq_dequantize_meta -- hqq_dequantize for a matrix whose zero points (and,
 * optionally, scales) are kept in their 8-bit form: each group's zero point is
 * restored first, z' = fp16((c_z - z_z) * s_z), the scale likewise when scale_q
 * is given, and then W_hat = fp16((code - z') * s') exactly as hqq_dequantize
 * does.  The result equals hqq_meta_dequantize of the zero points (and scales)
 * followed by hqq_dequantize, bit for bit, in one pass.
 *   packed  [in]  codes, as for hqq_dequantize.
 *   zero_q  [in]  HOST pointer to the zero points' 8-bit form (required; its
 *                 codes hold rows*cols/group values).
 *   scale   [in]  fp16 [rows, cols/group] scales, or NULL when scale_q is given.
 *   scale_q [in]  HOST pointer to the scales' 8-bit form, or NULL.
 *                 Exactly one of scale and scale_q must be non-NULL.
 *   rows, cols, nbits, group, W_out, stream [in/out] as for hqq_dequantize.
 * Alignment: packed 4 bytes, zero_q/scale_q codes 1, their fp16 arrays and
 * scale 2, W_out 16.
 */
int hqq_dequantize_meta(const void* packed, const hqq_meta8* zero_q, const void* scale,
                        const hqq_meta8* scale_q, int64_t rows, int64_t cols, int nbits,
                        int group, void* W_out, void* stream);

/*
 * hqq_linear -- weight-only linear layer on a quantized matrix: the matrix
 * product with section 2's Q^-1 fused in,
 *   Y[m, n] = sum over k of X[m, k] * W_hat[n, k],
 *   W_hat   = fp16((code - z) * s), exactly the values hqq_dequantize writes,
 * without W_hat ever being stored.  Products and sums are formed in the
 * tensor cores' fp32 accumulator (summation order unspecified) and Y is
 * rounded to fp16 once.
 *
 *   X      [in]  fp16 [M, cols] row-major (tokens x input features),
 *                16-byte aligned.
 *   M      [in]  number of tokens, 0 <= M <= 2^31 - 1024 (M == 0: no-op);
 *                rows at most 65535*128.
 *   packed, scale, zero, rows, cols, nbits, group [in]  the quantized
 *                [rows, cols] matrix as hqq_quantize writes it (alignment as
 *                for hqq_dequantize).
 *   Y      [out] fp16 [M, rows] row-major (tokens x output features), 2-byte
 *                aligned.
 *   status [out] optional device int (NULL allowed), 4-byte aligned.  The
 *                kernel stores 1 there when one of its internal waits ran
 *                out (a device fault, never a consequence of valid arguments;
 *                Y is then unspecified).  It never stores 0: clear it first.
 *   stream [in]  cudaStream_t (NULL = legacy default stream).
 * HQQ_ERR_CUDA also covers a driver without the tensor-map entry point.
 */
int hqq_linear(const void* X, int64_t M, const void* packed, const void* scale,
               const void* zero, int64_t rows, int64_t cols, int nbits, int group,
               void* Y, int* status, void* stream);

/*
 * hqq_linear_meta -- hqq_linear for a matrix whose zero points (and,
 * optionally, scales) are kept in their 8-bit form (hqq_meta_quantize): each
 * group's z' = fp16((c_z - z_z) * s_z) (and s' likewise) is restored inside the
 * kernel, then Y = X W_hat^T with W_hat = fp16((code - z') * s').  The result is
 * that of hqq_meta_dequantize followed by hqq_linear (same tolerance).
 *   zero_q  [in]  HOST pointer to the zero points' 8-bit form (required).
 *   scale   [in]  fp16 scales, or NULL when scale_q is given.
 *   scale_q [in]  HOST pointer to the scales' 8-bit form, or NULL.
 *                 Exactly one of scale and scale_q must be non-NULL.
 *   other arguments as for hqq_linear.
 */
int hqq_linear_meta(const void* X, int64_t M, const void* packed, const hqq_meta8* zero_q,
                    const void* scale, const hqq_meta8* scale_q, int64_t rows, int64_t cols,
                    int nbits, int group, void* Y, int* status, void* stream);

/* Human-readable name of a status code (static string, never NULL). */
const char* hqq_status_string(int status);

/*
 * Low-rank residual of the quantization error ("Boost 2-bit LLM accuracy with
 * EoRA", the section on finding adapters in the feature space: Delta W =
 * W - W_hat = U Sigma V^T, B = U_r Sigma_r, A = V_r^T, the best rank-r
 * approximation in the Frobenius norm).  Computed on the GPU by randomized
 * subspace iteration (Halko, Martinsson and Tropp 2011, Algorithms 4.4 and
 * 5.1) with shifted CholeskyQR3 orthonormalization and a Jacobi eigensolver
 * for the sketch-sized problem; Delta W is formed inside every product from W
 * and the packed codes and is never stored.  The result approximates the
 * truncated SVD: the closer sigma_r / sigma_{r+1} is to 1, the more power
 * iterations it needs; with a clear gap it matches the SVD to fp32 accuracy.
 *
 * hqq_lowrank_workspace_bytes -- device workspace bytes hqq_lowrank needs for
 * a rows x cols matrix and a sketch of 16, 32 or 64 columns; -1 for a bad
 * argument.
 */
int64_t hqq_lowrank_workspace_bytes(int64_t rows, int64_t cols, int sketch);

/*
 * hqq_lowrank -- B and A of the rank-`rank` residual and its singular values.
 *   W        [in]  fp16 [rows, cols] row-major, 16-byte aligned: the weights
 *                  that packed/scale/zero quantize.
 *   packed, scale, zero, rows, cols, nbits, group [in]  as for hqq_dequantize.
 *   rank     [in]  1 <= rank <= sketch.
 *   sketch   [in]  16, 32 or 64 columns of the random sketch; rows and cols
 *                  must be at least sketch, cols below 2^30.
 *   power_iters [in] 0..16 subspace iterations (each adds two products with
 *                  Delta W; 2 suits the nearly flat spectra of quantization
 *                  errors).
 *   omega    [in]  fp32 [cols, sketch] row-major, 16-byte aligned: the
 *                  Gaussian test matrix, drawn by the caller (any seeded
 *                  standard normal source).
 *   B        [out] fp32 [rows, rank] row-major; A [out] fp32 [rank, cols].
 *   sigma    [out] fp32 [rank] decreasing, or NULL.  A singular value below
 *                  1e-7 sigma_1 gives a zero row of A (and its B column is
 *                  sigma times the basis vector, i.e. near zero).
 *   workspace [in] device memory, 256-byte aligned, at least
 *                  hqq_lowrank_workspace_bytes() bytes (workspace_bytes); its
 *                  contents on return are unspecified.
 *   stream   [in]  cudaStream_t or NULL; asynchronous.
 * Errors: HQQ_ERR_UNSUPPORTED (sketch), HQQ_ERR_PARAM (rank, power_iters,
 * workspace too small), HQQ_ERR_SHAPE (rows or cols below sketch),
 * HQQ_ERR_NULL, HQQ_ERR_ALIGN, plus those of hqq_dequantize.
 */
int hqq_lowrank(const void* W, const void* packed, const void* scale, const void* zero,
                int64_t rows, int64_t cols, int nbits, int group, int rank, int sketch,
                int power_iters, const float* omega, float* B, float* A, float* sigma,
                void* workspace, int64_t workspace_bytes, void* stream);

/*
 * hqq_lowrank_noalloc -- hqq_lowrank for callers that cannot allocate device
 * memory: code that runs where cudaMalloc is not available or not allowed
 * (a host whose allocator is owned by another framework, a plugin loaded into
 * a process that forbids extra allocations after start-up, a real-time loop
 * that must not allocate).  The paper has no counterpart of this entry point;
 * it is a service of this library.
 *
 * Same arguments and results as hqq_lowrank without workspace and
 * workspace_bytes: the workspace is a fixed scratch array inside the library
 * (hqq_lowrank_noalloc_max_bytes() bytes, 16 MiB, present on every GPU that
 * loads the library until the process exits).  A matrix whose
 * hqq_lowrank_workspace_bytes() exceeds it returns HQQ_ERR_SCRATCH (at a
 * 32-column sketch every Llama-2-70B matrix fits).  No call allocates device
 * or host memory.
 * The first call in each CUDA context looks up the array's device address
 * (with that context current) and keeps it for that context; a call made
 * under another context -- a second context on the device, or the new one
 * after cudaDeviceReset -- looks it up again.  Make the first call in a
 * context before any stream capture.  All calls share the one array: calls whose work overlaps on the
 * GPU (other streams, other host threads) race and give wrong results, so the
 * caller orders them.  Nothing in the array needs to start at zero.
 */
int hqq_lowrank_noalloc(const void* W, const void* packed, const void* scale, const void* zero,
                        int64_t rows, int64_t cols, int nbits, int group, int rank, int sketch,
                        int power_iters, const float* omega, float* B, float* A, float* sigma,
                        void* stream);

/* Bytes of the fixed scratch array of hqq_lowrank_noalloc. */
int64_t hqq_lowrank_noalloc_max_bytes(void);

#ifdef __cplusplus
}
#endif

#endif /* HQQ_H */
