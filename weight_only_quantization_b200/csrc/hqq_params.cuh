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

// Token counts up to which the linear layer runs on the CUDA cores (measured:
// from 3 tokens on, the tensor-core kernel is faster on the 8192 x 8192 and
// 28672 x 8192 shapes).
constexpr int64_t kGemvMaxTokens = 2;

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
