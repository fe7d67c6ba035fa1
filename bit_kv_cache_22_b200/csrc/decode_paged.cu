// decode_paged.cu -- the decode kernels' instances for paged, ragged caches (a page
// table per sequence and a token count per sequence); see decode_kernels.cuh.
#include "decode_kernels.cuh"

namespace kvq {

cudaError_t launch_decode_paged(const DecodeArgs &a, cudaStream_t s) { return launch_decode_variant<true>(a, s); }

int decode_ctas_per_sm_paged(const DecodeArgs &a) { return ctas_per_sm_variant<true>(a); }

}  // namespace kvq
