// decode_sparse.cu -- the tensor-core decode kernel's instances for dense-and-sparse
// keys (each token's outliers add their q_c x_c to its logit); see decode_kernels.cuh.
#include "decode_kernels.cuh"

namespace kvq {

cudaError_t launch_decode_sparse(const DecodeArgs &a, cudaStream_t s) {
    return launch_decode_variant<false, true>(a, s);
}

int decode_ctas_per_sm_sparse(const DecodeArgs &a) { return ctas_per_sm_variant<false, true>(a); }

}  // namespace kvq
