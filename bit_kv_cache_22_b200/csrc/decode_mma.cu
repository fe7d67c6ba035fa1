// decode_mma.cu -- the instances of decode_mma_kernel (contiguous caches, 1, 2 or 4 query
// heads per kv head, key groups of >= 32 tokens) and their launch; see decode_mma.cuh.
#include "decode_mma.cuh"

namespace kvq {

cudaError_t launch_decode_mma(const DecodeArgs &a, cudaStream_t s) { return launch_mma_any(a, s, false, nullptr); }

int decode_ctas_per_sm_mma(const DecodeArgs &a) {
    int n = 1;
    if (launch_mma_any(a, nullptr, true, &n) != cudaSuccess || n < 1) n = 1;
    return n;
}

}  // namespace kvq
