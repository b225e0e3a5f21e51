// hqq_quantize.cu -- the single-precision instantiations of the fused HQQ
// solver + packing kernel (hqq_quantize.cuh): every step of section 2 of "Half-
// Quadratic Quantization of Large Machine Learning Models" in binary32.
#include "hqq_quantize.cuh"

namespace hqq {

cudaError_t launch_quantize(const QuantParams& prm, int nbits, int group, cudaStream_t stream) {
    return launch_quantize_nb<false>(prm, nbits, group, stream);
}

}  // namespace hqq
