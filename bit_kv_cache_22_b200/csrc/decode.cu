// decode.cu -- decode attention over contiguous caches, the merge of token-split
// partials, and the dispatch between contiguous, paged and dense-and-sparse caches.
// The kernels are in decode_kernels.cuh and decode_mma.cuh; decode_paged.cu,
// decode_sparse.cu and decode_mma.cu hold their other instances.
#include "decode_kernels.cuh"

namespace kvq {
namespace {

// Token-split decode: t_O row = sum_k o_k 2^(m_k - M) / sum_k l_k 2^(m_k - M), M = max_k m_k,
// over n partials of caches holding disjoint tokens (o_all [n][rows][d], m_all and l_all
// [n][rows]); a partial with m = -inf (no tokens) has weight 0.  One CTA per row.
__global__ void merge_partials_kernel(const float *o_all, const float *m_all, const float *l_all, int n,
                                      int64_t rows, int d, float *out) {
    const int64_t row = blockIdx.x;
    float M = -INFINITY;
    for (int k = 0; k < n; ++k) M = fmaxf(M, m_all[k * rows + row]);
    float L = 0.f;
    for (int k = 0; k < n; ++k) {
        const float mk = m_all[k * rows + row];
        if (mk != -INFINITY) L = fmaf(l_all[k * rows + row], exp2f(mk - M), L);
    }
    for (int c = threadIdx.x; c < d; c += blockDim.x) {
        float o = 0.f;
        for (int k = 0; k < n; ++k) {
            const float mk = m_all[k * rows + row];
            if (mk != -INFINITY) o = fmaf(o_all[(k * rows + row) * d + c], exp2f(mk - M), o);
        }
        out[row * d + c] = o / L;
    }
}

}  // namespace

cudaError_t launch_merge_partials(const float *o_all, const float *m_all, const float *l_all, int n,
                                  int64_t rows, int d, float *out, cudaStream_t s) {
    if (rows == 0) return cudaSuccess;
    merge_partials_kernel<<<static_cast<unsigned>(rows), 128, 0, s>>>(o_all, m_all, l_all, n, rows, d, out);
    count_launches(1);
    return cudaGetLastError();
}

int binary_version() {
    cudaFuncAttributes at{};
    if (cudaFuncGetAttributes(&at, merge_partials_kernel) != cudaSuccess) return -1;
    return at.binaryVersion;
}

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t s) {
    if (a.page_table) return launch_decode_paged(a, s);
    if (a.k_out) return launch_decode_sparse(a, s);
    if (a.path == kPathMma) return launch_decode_mma(a, s);
    return launch_decode_variant<false>(a, s);
}

int decode_ctas_per_sm(const DecodeArgs &a) {
    if (a.page_table) return decode_ctas_per_sm_paged(a);
    if (a.k_out) return decode_ctas_per_sm_sparse(a);
    if (a.path == kPathMma) return decode_ctas_per_sm_mma(a);
    return ctas_per_sm_variant<false>(a);
}

}  // namespace kvq
