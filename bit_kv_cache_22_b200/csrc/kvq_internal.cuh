// kvq_internal.cuh -- declarations shared by the libkvq translation units.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace kvq {

constexpr int kTile = 16;          // tokens per code tile (and channels per chunk)

// Words of one 16-token tile of one (batch, kv-head) slice: 16*d*n/32.
__host__ __device__ constexpr int tile_words(int d, int n) { return d * n / 2; }
// Words owned by each of the 32 lanes inside a tile.
__host__ __device__ constexpr int lane_words(int d, int n) { return d * n / 64; }

// fp16 / bf16 bit pattern -> float (exact).
__device__ __forceinline__ float widen(uint16_t h, bool bf16) {
    if (bf16) return __uint_as_float(static_cast<uint32_t>(h) << 16);
    __half_raw r;
    r.x = h;
    return __half2float(__half(r));
}

// Bounds-check builds (-DKVQ_CHECK: libkvq_check.so).  Kernels that index through a list
// made on the host or by the caller check every index against its buffer; a bad one raises
// status bit 3 (value 8) and is replaced by row 0 (reads) or skipped (writes).  The product
// build compiles these checks out.
#ifdef KVQ_CHECK
constexpr bool kCheck = true;
#else
constexpr bool kCheck = false;
#endif

// Record n kernel launches (reported by kvq_kernel_launches()).
void count_launches(int n);

// ---------------------------------------------------------------------------
// launch helpers (implemented in quantize.cu / decode.cu); all return the
// cudaError_t of the launch.
// ---------------------------------------------------------------------------

struct QuantizeArgs {
    const uint16_t *xk, *xv;     // e [BH][*][d]; slice stride in elements below
    int64_t in_bh_stride;        // elements between consecutive (b,h) slices
    int64_t in_tok0;             // first input token
    const int32_t *in_rows;      // or, when non-NULL: input row of token i (device [n_groups * G]);
                                 // in_tok0 is then unused
    int64_t in_rows_limit;       // rows of each input slice the list may name (bounds-check builds)
    int64_t n_groups;            // key groups to quantize per slice
    int64_t BH;
    int d, G, Gv, bits;
    bool sym, bf16;
    uint32_t *kc, *vc;           // packed codes, [BH][cap*d*n/32]
    float *ks, *vs;              // [BH][cap/G][d], [BH][cap][d/Gv]
    int16_t *kz, *vz;            // same shapes (unused when sym)
    int64_t cap;                 // token capacity per slice
    int64_t out_tok0;            // first output token (multiple of G)
    // paged pool (page_table non-NULL): slice (page, kv head) of cap = P tokens; the
    // slice of output token t of sequence b is page_table[b][t / P] * Hkv + kv head
    const int32_t *page_table;   // [B][max_pages]
    int max_pages, num_pages, Hkv;
    int seq0;                    // first sequence of the launch: CTA y = (seq - seq0) * Hkv + head
    const int32_t *seq_len;      // flush: tokens of each sequence after the append; only those
                                 // at a multiple of R flush, to tokens [len - R, len)
    unsigned int *status;        // the cache's status word: bit 2 raised for a page number outside
                                 // the pool, bit 4 for a scale above the decode kernels' range
    // dense-and-sparse keys (k_out non-NULL): each token's n_out largest-magnitude key
    // entries leave the dense part (set to +0 before quantizing) and are written as words
    // (channel << 16) | element bits to k_out [slice][cap][n_out], largest first
    uint32_t *k_out;
    int n_out;
    int gpc;                     // key groups per CTA (1, or 2 for short groups: set by the launch)
};
cudaError_t launch_quantize(const QuantizeArgs &a, cudaStream_t s);

// For both (src, dst) pairs: dst[bh][dst_row0 + i][:] = src[bh][src_row0 + i][:],
// i < rows (e elements); one launch.
cudaError_t launch_copy_rows(const uint16_t *src0, const uint16_t *src1, int64_t src_bh_stride,
                             int64_t src_row0, uint16_t *dst0, uint16_t *dst1,
                             int64_t dst_bh_stride, int64_t dst_row0, int64_t rows, int64_t BH,
                             int d, cudaStream_t s);

// The decode kernel that serves a configuration:
//  kPathMma   contiguous caches with 1, 2 or 4 query heads per kv head and key groups of
//             >= 32 tokens: decode_mma_kernel (tensor cores, bf16 MMA for keys and values),
//             one CTA per (batch, kv head, split) serving those heads;
//  kPathTc    the same geometries for paged caches and dense-and-sparse keys:
//             decode_tc_kernel (tensor cores, integer MMA for keys);
//  kPathSplit any other grouping, or 16-token key groups: CUDA cores, one CTA per
//             (batch, query head, split).
enum DecodePath : int { kPathSplit = 0, kPathTc = 1, kPathMma = 2 };
// Most splits of one decode: up to 128 over the quantized tiles and 16 residual ones.
constexpr int kMaxDecodeSplits = 144;

inline int decode_path(int q_heads, int kv_heads, int group_k, bool plain = true) {
    const int g = q_heads / kv_heads;
    if (!((g == 1 || g == 2 || g == 4) && group_k >= 32)) return kPathSplit;
    return plain ? kPathMma : kPathTc;
}
// Split boundaries must fall on multiples of this many tiles (the tensor-core
// kernels stream items of 4 or 2 tiles).
inline int split_tile_align(int path) { return path == kPathTc ? 4 : path == kPathMma ? 2 : 1; }
// Paths whose CTAs serve every query head of one kv head.
inline bool path_per_kv_head(int path) { return path == kPathTc || path == kPathMma; }

struct DecodeArgs {
    const uint32_t *kc, *vc;
    const float *ks, *vs;
    const int16_t *kz, *vz;
    uint16_t *kr, *vr;           // residual [BH][R][d]
    const uint16_t *new_k, *new_v;   // fused append: the new token [BH][d] (row new_row), else NULL
    int new_row;
    const uint16_t *q;           // [B][Hq][d]
    float *o_part, *m_part, *l_part;   // [B*Hq][S][d], [B*Hq][S], [B*Hq][S]
    float *out;                  // [B][Hq][d]
    float *po, *pm, *pl;         // instead of out (token-split decode): o [B][Hq][d] and m, l [B][Hq]
                                 // of the whole cache, o and l relative to m (log2 units); else NULL
    unsigned int *arrivals;      // [B*Hq] split-arrival counters, zero between calls
    unsigned int *status;        // nonzero once a bounded wait inside a decode kernel gave up
    int64_t cap;
    int B, Hq, Hkv, d, G, Gv, R, bits;
    int gshift;                  // log2(G / 16): key groups are 2^gshift tiles
    bool sym, bf16;
    int path;                    // DecodePath
    int n_qtiles;                // Tq / 16
    int r;                       // residual rows
    int tiles_per_split;         // quantized tiles per split
    int n_qsplits;               // splits over the quantized tiles
    int S;                       // n_qsplits + (r > 0)
    float qscale;                // log2(e) / sqrt(d)
    // paged, ragged cache (page_table non-NULL): the pool is cut into pages of P tokens per
    // (page, kv head) slice, laid out like a contiguous cache of capacity P whose batch is
    // the page; sequence b's tokens [jP, (j+1)P) are in page page_table[b][j], and its token
    // count is seq_len[b] (Tq = floor(len / R) R, r = len mod R; len < 0: an inactive slot,
    // treated as empty).  n_qtiles / r above are unused then.
    const int32_t *page_table;   // [B][max_pages]
    const int32_t *seq_len;      // [B]
    int page_tiles;              // P / 16
    int max_pages, num_pages;
    // dense-and-sparse keys (contiguous caches, tensor-core path): outlier words
    // [BH][cap][n_out] as written by the quantizer, or NULL
    const uint32_t *k_out;
    int n_out;
    // bounds-check builds: warp 0 of CTA (0, 0, 0) of the bf16-MMA kernel first waits on a
    // barrier nothing arrives at, bounded by this many polls, and gives up (0: no wait)
    int stall_polls;
};
cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t s);
cudaError_t launch_decode_paged(const DecodeArgs &a, cudaStream_t s);
int decode_ctas_per_sm_paged(const DecodeArgs &a);
cudaError_t launch_decode_sparse(const DecodeArgs &a, cudaStream_t s);
int decode_ctas_per_sm_sparse(const DecodeArgs &a);
cudaError_t launch_decode_mma(const DecodeArgs &a, cudaStream_t s);
int decode_ctas_per_sm_mma(const DecodeArgs &a);
// LogQuant retention event: in every (b, h) slice of the full-precision store (rows
// [0, 3W) of `rows` rows each, ascending positions), rows 2i (i < W) move to row i and rows
// 2W + j (j < W) to row W + j, for K and V.  One launch.
cudaError_t launch_lq_compact(uint16_t *kr, uint16_t *vr, int64_t BH, int rows, int W, int d, unsigned int *status,
                              cudaStream_t s);
// dst[bh][i] = src[bh][idx[i]] for i < n, K and V (idx device [n]).  One launch.
cudaError_t launch_gather_rows(const uint16_t *srck, const uint16_t *srcv, int64_t src_bh_stride,
                               int64_t src_rows, const int32_t *idx, int n, uint16_t *dstk, uint16_t *dstv,
                               int64_t dst_bh_stride, int64_t BH, int d, unsigned int *status, cudaStream_t s);

// Paged append: for each sequence slot b with seq_len[b] >= 0, rows t_K[b], t_V[b] ([Hkv][d])
// become residual row seq_len[b] mod R and seq_len[b] grows by one.  One launch.
cudaError_t launch_paged_append(const uint16_t *tk, const uint16_t *tv, uint16_t *kr, uint16_t *vr,
                                int32_t *seq_len, int B, int Hkv, int R, int d, cudaStream_t s);
// Sets seq_len[seq] = value and copies rows [row0, row0 + rows) of X_K / X_V ([Hkv][T][d])
// to residual rows 0 .. rows-1 of sequence seq.  One launch.
cudaError_t launch_paged_residual(const uint16_t *xk, const uint16_t *xv, int64_t T, int64_t row0,
                                  int64_t rows, uint16_t *kr, uint16_t *vr, int32_t *seq_len, int seq,
                                  int32_t value, int Hkv, int R, int d, cudaStream_t s);
// t_O [rows][d] from n partials o_all [n][rows][d], m_all / l_all [n][rows] (log2 units).
cudaError_t launch_merge_partials(const float *o_all, const float *m_all, const float *l_all, int n,
                                  int64_t rows, int d, float *out, cudaStream_t s);
// The compute capability the library's kernels were compiled for (major * 10 + minor, as
// the CUDA runtime reports it for a loaded kernel), or -1 when it cannot be read.
int binary_version();
// CTAs of the split kernel that fit on one SM for this configuration.
int decode_ctas_per_sm(const DecodeArgs &a);

}  // namespace kvq
