// hqq_params.cuh -- launch parameters of the dequantize, 8-bit meta-data and
// linear-layer kernels (the quantize kernel's own types are in hqq_common.cuh).
#pragma once
#include "hqq_common.cuh"

namespace hqq {

// 8-bit form of a meta tensor (zero points or scales): codes, the fp16 s and z
// of each second-level group, and log2 of that group (62: one group).
struct Meta8 {
    const uint8_t* codes;
    const __half* scale;
    const __half* zero;
    int shift;
};

// Token counts up to which the linear layer runs as warp-level MMAs fed from
// registers (one or two 8-token m16n8k16 column blocks share each decoded
// weight); above it, the tensor-memory kernel.  Measured on the 28672 x 8192
// and 8192 x 28672 3-bit and 8192 x 8192 4-bit shapes: the second block pays
// at 3 bits (16 tokens: 0.17 vs 0.23 ms), not at 4 bits.
__host__ __device__ constexpr int64_t decode_max_tokens(int nbits) { return nbits == 3 ? 16 : 8; }

// Weight-only linear layer Y = X W_hat^T on a quantized [N, K] matrix.
struct LinearParams {
    const uint8_t* packed;
    const __half* scale;
    const __half* zero;
    __half* Y;
    int* status;             // optional: set to 1 if a wait inside a kernel ran out
    int64_t M, N, K;         // tokens, output features, input features
    int log2_group;
    Meta8 zq, sq;            // 8-bit zero points / scales (codes NULL: use zero / scale)
};

// One meta tensor of a batch (validated on the host): log2g < 0 for one group.
struct MetaJobIn {
    const __half* x;
    int64_t n;
    int log2g;
    uint8_t* codes;
    __half* scale;
    __half* zero;
};

struct DequantParams {
    const uint8_t* packed;
    const __half* scale;   // fp16 scales, unless given in 8-bit form (sq)
    const __half* zero;    // fp16 zero points, unless given in 8-bit form (zq)
    __half* out;
    int64_t n_units;       // n_elems / 8
    uint32_t n_words;      // 3 bits: 32-bit words of packed codes (when < 2^32)
    int group;
    Meta8 zq, sq;
};

}  // namespace hqq
