// hqq_quantize_half.cu -- the half-precision instantiations of the fused HQQ
// solver + packing kernel (hqq_quantize.cuh).  "Half-Quadratic Quantization of
// Large Machine Learning Models", section 2.2 (1/s is held because it is more
// stable in half precision) and section 3 (the whole solve runs on the GPU in
// half precision): each element-wise step is rounded to fp16, the group means
// are accumulated in binary32 and rounded to fp16, and groups outside the fp16
// bounds are solved in single precision (see init_group).
#include "hqq_quantize.cuh"

namespace hqq {

cudaError_t launch_quantize_half(const QuantParams& prm, int nbits, int group,
                                 cudaStream_t stream) {
    return launch_quantize_nb<true>(prm, nbits, group, stream);
}

}  // namespace hqq
