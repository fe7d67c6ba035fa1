/*
 * kvq.h -- C ABI of libkvq: decode-phase attention over a KIVI-style low-bit
 * quantized KV cache on NVIDIA B200 (sm_100a).
 *
 * What is computed (web pages the operations follow):
 *  - "LLM系列：KVCache量化1 KIVI: A Tuning-Free Asymmetric 2bit Quantization
 *    for KV Cache", section 1: keys are quantized per channel in groups of G
 *    tokens, values per token; the newest tokens stay in a full-precision
 *    residual X_Kr that is quantized and appended when it holds R tokens;
 *    A = Concat(A_g, A_r), t_O = A X_V.
 *  - "Atom: Low-bit Quantization for Efficient and Accurate LLM Serving",
 *    section 核心公式 / 量化基础: asymmetric s = (max-min)/(2^n-1),
 *    z = round(-min/s), code = clamp(round(x/s) + z, 0, 2^n-1); symmetric
 *    s = 2 max|x| / (2^n-1), code = clamp(round(x/s), -2^(n-1), 2^(n-1)-1).
 *  - "KV Cache的Int4量化…", section 2 (x' = (q - z) s) and section 3
 *    (softmax(Q K^T / sqrt(d_k)) V).
 * Rounding is half-to-even in IEEE fp32; a constant group uses s = |min|
 * (1 when min = 0) so that it reconstructs exactly; the symmetric variant
 * stores u = q + 2^(n-1) and has no zero-point tensors.
 *
 * Conventions for every call:
 *  - All device memory (cache buffers, inputs, outputs, workspace and the
 *    cache's state buffer) is owned and allocated by the caller; the library
 *    allocates none.  The state buffer (kvq_sizes.state bytes) holds a 4-byte
 *    split-arrival counter per (batch, query head), through which the last
 *    split of a decode merges the others, and a status word (a LogQuant cache
 *    adds its row lists, a paged cache its slots' lengths).  kvq_create
 *    initialises it; every decode leaves the counters at zero, so decode calls
 *    on one cache must be ordered (one stream, or synchronised).  The
 *    host-side handle keeps the cache geometry and the two counters Tq
 *    (quantized tokens) and r (residual tokens).
 *  - Work is enqueued asynchronously on the caller's CUDA stream (`stream`
 *    is a cudaStream_t, NULL for the legacy default stream).  Host counters
 *    advance when a call is enqueued, so a sequence of calls needs no
 *    device-to-host synchronisation.
 *  - A call that returns an error has launched nothing and changed no state;
 *    kvq_last_error() then describes the cause (thread-local string).
 *  - Device pointers must be 16-byte aligned; tensors are dense and
 *    row-major in the shapes given below.  Element type `e` is fp16 or bf16
 *    (kvq_config.dtype) and is passed as raw 16-bit patterns.
 *  - Query head i reads kv head i / (Hq / Hkv).
 *  - No C++ exception crosses this interface.
 *
 * Storage format of the cache (this library's own; the pages fix none):
 *  - k_codes, v_codes: uint32 [B][Hkv][capacity * d * n / 32].  Tokens are cut
 *    into tiles of 16 and channels into chunks of 16.  A tile occupies
 *    d*n/2 consecutive words; inside it 32 lanes own W = d*n/64 words each.
 *    In chunk j, a 16x16 block indexed (row, col) -- keys (token%16,
 *    channel%16), values (channel%16, token%16) -- places element (row, col)
 *    in lane 4*(row%8) + col/4, byte col%4, half row/8.  A lane's word holds
 *    B = 4/n blocks: block j in word j/B, element at bit
 *    8*byte + n*(2*(j%B) + half).  Keeping the low n bits of every byte of
 *    (word >> n*slot) gives four codes of one row, one per byte: the operand
 *    of a 4-way byte dot product and the A fragment of an 8-bit 16x8x32
 *    tensor-core MMA.
 *  - k_scales float / k_zeros int16: [B][Hkv][capacity/G][d]   (group, channel)
 *  - v_scales float / v_zeros int16: [B][Hkv][capacity][d/Gv]  (token, group)
 *  - k_residual, v_residual: e [B][Hkv][R][d]  (rows 0..r-1 valid)
 *  Symmetric caches have no zero tensors (pass NULL).
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KVQ_API __attribute__((visibility("default")))
#else
#define KVQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KVQ_OK = 0,
    KVQ_ERR_INVALID_ARG = 1,   /* bad pointer, alignment, shape or parameter   */
    KVQ_ERR_UNSUPPORTED = 2,   /* valid but not built (e.g. head_dim 96)        */
    KVQ_ERR_CAPACITY = 3,      /* the call would exceed the token capacity      */
    KVQ_ERR_STATE = 4,         /* call out of order (prefill twice, empty cache) */
    KVQ_ERR_CUDA = 5,          /* a CUDA runtime call or launch failed          */
    KVQ_ERR_DEVICE_CHECK = 6   /* a check inside a kernel failed (see kvq_check_device) */
} kvq_status;

typedef enum { KVQ_FP16 = 0, KVQ_BF16 = 1 } kvq_dtype;

/* Cache geometry and quantiser settings. */
typedef struct {
    int32_t batch;       /* B                                                   */
    int32_t q_heads;     /* Hq                                                  */
    int32_t kv_heads;    /* Hkv, divides Hq                                     */
    int32_t head_dim;    /* d: 64 or 128                                        */
    int32_t group_k;     /* G: tokens per key group: 16, 32, 64, 128 or 256,
                            G * d <= 32768                                      */
    int32_t group_v;     /* Gv: channels per value group: 16, 32, 64 or 128, <= d */
    int32_t residual;    /* R: residual capacity, multiple of G                 */
    int32_t bits;        /* n: 2 or 4                                           */
    int32_t symmetric;   /* 0 asymmetric min-max, 1 symmetric (offset codes)    */
    int32_t dtype;       /* kvq_dtype of every e tensor                         */
    int64_t capacity;    /* quantized-token capacity per sequence, multiple of R */
} kvq_config;

/* Byte sizes of the caller-allocated device buffers. */
typedef struct {
    size_t k_codes, k_scales, k_zeros;
    size_t v_codes, v_scales, v_zeros;
    size_t k_residual, v_residual;
    size_t workspace;    /* scratch needed by kvq_decode_attention              */
    size_t state;        /* the cache's state buffer (kvq_buffers.state)        */
} kvq_sizes;

/* Caller-owned device buffers of one cache (layout above). */
typedef struct {
    void *k_codes;
    float *k_scales;
    int16_t *k_zeros;    /* NULL when symmetric                                 */
    void *v_codes;
    float *v_scales;
    int16_t *v_zeros;    /* NULL when symmetric                                 */
    void *k_residual;
    void *v_residual;
    void *state;         /* kvq_sizes.state bytes; initialised by the create call,
                            then the library's for the life of the handle       */
} kvq_buffers;

typedef struct kvq_cache kvq_cache;   /* opaque host-side handle */

/* Validates `cfg` and fills `out` with the buffer sizes.  No device needed. */
KVQ_API kvq_status kvq_get_sizes(const kvq_config *cfg, kvq_sizes *out);

/*
 * Creates a handle over caller-owned buffers (not copied, not freed).  The
 * cache starts empty (Tq = 0, r = 0).  Reads device properties of the current
 * device and zero-fills the state buffer there (synchronously); allocates no
 * device memory.  All later calls must run with that device current.
 * KVQ_ERR_INVALID_ARG for a NULL or misaligned buffer; KVQ_ERR_CUDA if the fill
 * fails.
 */
KVQ_API kvq_status kvq_create(const kvq_config *cfg, const kvq_buffers *bufs, kvq_cache **out);

/* Frees the host-side handle (no device memory is the library's).  NULL is ignored. */
KVQ_API void kvq_destroy(kvq_cache *cache);

/* Empties the cache (Tq = r = 0) without touching device memory. */
KVQ_API kvq_status kvq_reset(kvq_cache *cache);

/*
 * Prefill (KIVI section 1, prefill phase): X_K, X_V are e [B][Hkv][T][d]
 * device tensors of the prompt's keys and values.  The first
 * Tq = floor(T/R)*R tokens are quantized (keys per channel over G tokens,
 * values per token over Gv channels) and packed; the remaining T - Tq
 * tokens are copied into the residual.  Only allowed on an empty cache
 * (KVQ_ERR_STATE otherwise); Tq > capacity gives KVQ_ERR_CAPACITY.
 * T = 0 is accepted and does nothing.
 * Range: the decode kernels serve key and value scales s <= 2^31 (values of
 * magnitude up to about 2^31 (2^n - 1)) and queries |q| <= 2^30.  A group whose
 * scale exceeds 2^31 is still quantized exactly, but raises status bit 2 of the
 * state buffer, which the next kvq_check_device reports as KVQ_ERR_DEVICE_CHECK
 * (the same holds for the quantization done by kvq_append's flush).  Scales
 * near 0 need no check: tokens that small only lose contributions below fp32's
 * normal range.
 */
KVQ_API kvq_status kvq_prefill_quantize(kvq_cache *cache, const void *X_K, const void *X_V,
                                int64_t T, void *stream);

/*
 * Decode-phase append (KIVI section 1): t_K, t_V are e [B][Hkv][d] device
 * tensors of one new token per sequence.  They are written to residual row
 * r and r is incremented; when r reaches R the R residual rows are quantized
 * into tokens [Tq, Tq+R) of the quantized cache, Tq += R and r = 0.  A flush
 * that would exceed the capacity gives KVQ_ERR_CAPACITY (nothing written).
 */
KVQ_API kvq_status kvq_append(kvq_cache *cache, const void *t_K, const void *t_V, void *stream);

/*
 * Decode attention (KIVI section 1: A = Concat(A_g, A_r), t_O = A X_V with
 * the 1/sqrt(d) scaling): t_Q is e [B][Hq][d]; t_O receives float
 * [B][Hq][d] = softmax(t_Q [deq(K_g); K_r]^T / sqrt(d)) [deq(V_g); V_r].
 * `workspace` is device scratch of at least kvq_sizes.workspace bytes
 * (holds per-split partial results; contents on entry are ignored).
 * An empty cache gives KVQ_ERR_STATE.
 */
KVQ_API kvq_status kvq_decode_attention(kvq_cache *cache, const void *t_Q, float *t_O,
                                void *workspace, size_t workspace_bytes, void *stream);

/*
 * kvq_append(t_K, t_V) followed by kvq_decode_attention(t_Q -> t_O), in one call
 * (KIVI section 1: each decode step appends its token, then attends over
 * [deq(K_g); K_r] including it).  Same arguments, state change and result as the
 * two calls.  On the tensor-core path (1, 2 or 4 query heads per kv head, key
 * groups of >= 32 tokens), when the append does not flush, it is one kernel
 * launch: the decode reads the new token straight from t_K / t_V as residual
 * row r and stores it there for later steps.  Otherwise it makes the two calls'
 * launches.  Errors as for the two calls; arguments are checked before
 * anything is launched or changed.
 */
KVQ_API kvq_status kvq_append_decode_attention(kvq_cache *cache, const void *t_K, const void *t_V,
                                               const void *t_Q, float *t_O, void *workspace,
                                               size_t workspace_bytes, void *stream);

/*
 * Token-split decode (several caches holding disjoint tokens of the same
 * sequences, e.g. one per GPU; the order of a concatenation does not matter,
 * "Resumo Técnico: LogQuant", section 4).  Like kvq_decode_attention, but
 * instead of t_O it writes this cache's unnormalised partial:
 *   m_part [B][Hq]     = max_t y_t over this cache's tokens,
 *   l_part [B][Hq]     = sum_t 2^(y_t - m),
 *   o_part [B][Hq][d]  = sum_t 2^(y_t - m) v_t,
 * with y_t = log2(e) q.k_t / sqrt(d) (base-2 logits).  All float, 16-byte
 * aligned, caller-owned.  An empty cache gives KVQ_ERR_STATE (its partial would
 * be m = -inf, l = 0, o = 0).  The pages have no counterpart for the split.
 */
KVQ_API kvq_status kvq_decode_attention_partial(kvq_cache *cache, const void *t_Q, float *o_part,
                                                float *m_part, float *l_part, void *workspace,
                                                size_t workspace_bytes, void *stream);

/*
 * Merges n partials of kvq_decode_attention_partial (from caches holding
 * disjoint tokens of the same rows): o_parts [n][rows][d], m_parts and l_parts
 * [n][rows], device, contiguous -> t_O [rows][d] =
 * sum_k 2^(m_k - M) o_k / sum_k 2^(m_k - M) l_k with M = max_k m_k (partials
 * with m = -inf count for nothing).  rows = B * Hq.  One kernel launch.
 */
KVQ_API kvq_status kvq_merge_partials(const float *o_parts, const float *m_parts, const float *l_parts,
                                      int32_t n, int64_t rows, int32_t d, float *t_O, void *stream);

/*
 * Decode attention that allocates nothing and takes no workspace (the pages
 * have no counterpart: this is an interface for callers that cannot allocate
 * device memory -- for instance code that runs while another framework owns
 * every allocation on the device, a plugin host that forbids cudaMalloc, or a
 * latency-bound loop that must not hit the allocator).  Same inputs, outputs
 * and result as kvq_decode_attention; the per-split partial results go to a
 * fixed 4 MiB device array inside the library (allocated once per device that
 * loads the library and held until the process exits).
 *  - Calls whose partials would exceed 4 MiB (B * Hq * splits * (d + 2) * 4
 *    bytes, splits as reported by kvq_decode_splits) return KVQ_ERR_CAPACITY
 *    and launch nothing.
 *  - All calls on a device share that array: calls whose kernels may overlap
 *    on the GPU (different streams without ordering) race and give undefined
 *    results.  Nothing in it needs to start at zero; every call writes the
 *    partials it reads.
 *  - Every call looks up the array's device address in the calling thread's
 *    current context, so a context made after a device reset, or another
 *    context on the device, is served correctly.  The first call in a context
 *    may load the library's device code: make it before any stream capture.
 */
KVQ_API kvq_status kvq_decode_attention_noalloc(kvq_cache *cache, const void *t_Q, float *t_O,
                                                void *stream);

/* Current counters: quantized tokens Tq and residual tokens r. */
KVQ_API kvq_status kvq_cache_state(const kvq_cache *cache, int64_t *quantized_tokens,
                           int32_t *residual_tokens);

/*
 * Upper bound on the splits kvq_decode_attention cuts the quantized tokens into
 * (1 .. 128; 0 restores the default of 128).  With one query head per kv head
 * the residual tokens are shared out among those splits; otherwise they form
 * 1 to 16 more splits of their own when there are any (more of them for a
 * longer full-precision part, such as a LogQuant store).  Fewer splits mean fewer
 * partial results to merge, more splits more parallelism for short batches;
 * the result is the same up to fp32 rounding.
 */
KVQ_API kvq_status kvq_set_split_limit(kvq_cache *cache, int32_t max_splits);

/*
 * The decode kernel a cache's decode calls launch (all read the same layout and give the
 * same result up to fp32 rounding, so this only trades speed; for measurement and A/B
 * checks):
 *   KVQ_DECODE_AUTO        the library's choice (the default): KVQ_DECODE_BF16_MMA where it
 *                          applies, else KVQ_DECODE_INT8_MMA with key outliers, else
 *                          KVQ_DECODE_CUDA_CORES;
 *   KVQ_DECODE_CUDA_CORES  decode_split_kernel, CUDA cores only (any geometry);
 *   KVQ_DECODE_INT8_MMA    decode_tc_kernel: keys on integer mma.sync against fixed-point
 *                          query digits, values on bf16 mma.sync;
 *   KVQ_DECODE_BF16_MMA    decode_mma_kernel: keys and values on bf16 mma.sync.
 * The MMA kernels need 1, 2 or 4 query heads per kv head and key groups of >= 32 tokens;
 * KVQ_DECODE_BF16_MMA also needs a cache without key outliers (kvq_set_key_outliers),
 * which serves KVQ_DECODE_AUTO and KVQ_DECODE_INT8_MMA only.  Otherwise
 * KVQ_ERR_UNSUPPORTED and the cache keeps its kernel.  Host only; takes effect at the next
 * decode call.
 */
enum {
    KVQ_DECODE_AUTO = 0,
    KVQ_DECODE_CUDA_CORES = 1,
    KVQ_DECODE_INT8_MMA = 2,
    KVQ_DECODE_BF16_MMA = 3
};
KVQ_API kvq_status kvq_set_decode_kernel(kvq_cache *cache, int32_t kernel);

/*
 * The split plan of a decode over cfg->batch sequences of lengths[b] tokens each
 * (host int64; Tq = floor(len/R) R quantized, r = len mod R residual; a length
 * < 0 counts as empty), on a GPU of num_sms SMs holding ctas_per_sm decode CTAs
 * each.  Writes the splits over the quantized tokens, the 16-token tiles per
 * split and the total splits including the residual ones (>= 1): what the
 * decode calls choose for those lengths (kvq_decode_splits reports a cache's
 * total on its device).  Host only, no device needed; KVQ_ERR_CAPACITY if a
 * sequence's Tq exceeds cfg->capacity.
 */
KVQ_API kvq_status kvq_plan_decode(const kvq_config *cfg, const int64_t *lengths, int32_t num_sms,
                                   int32_t ctas_per_sm, int32_t *n_qsplits, int32_t *tiles_per_split,
                                   int32_t *splits);

/* Number of token splits the next kvq_decode_attention would use (>= 1). */
KVQ_API int32_t kvq_decode_splits(const kvq_cache *cache);

/*
 * Reads, waiting for the device to finish its queued work, the status word in
 * this cache's state buffer, which its kernels raise when a check fails: a
 * decode kernel's bounded wait for a copy into shared memory gave up (bit 0; a
 * condition working hardware never reaches -- the wait is bounded so that a
 * fault cannot hang the GPU), or a quantizer met a scale outside the range the
 * decode kernels serve (bit 2; see kvq_prefill_quantize), or -- in the
 * bounds-check build only (include/kvq_check.h) -- a kernel met a list index
 * outside its buffer (bit 3).  KVQ_OK when the word
 * is clear; KVQ_ERR_DEVICE_CHECK when it was raised -- the outputs of the calls
 * since the last check are then unreliable, kvq_last_error() names the checks,
 * and the word is cleared -- or KVQ_ERR_CUDA when the read fails.  The pages
 * have no counterpart.
 */
KVQ_API kvq_status kvq_check_device(kvq_cache *cache);

/*
 * ---------------------------------------------------------------------------
 * Paged, ragged cache: sequence slots of different lengths whose quantized tokens
 * live in pages of one shared pool, each sequence with its own page table (the
 * way serving systems hold KV caches: "Atom: Low-bit Quantization ...", section
 * 六 (related work: vLLM's page tables) and Figure 3 (PageAttention)).  Every
 * sequence is a KIVI cache of its own, with the same quantiser, residual and
 * flush as above; only the storage is shared.
 *
 * Storage:
 *  - A page holds P = page_tokens tokens of one sequence for every kv head.  The
 *    pool's six arrays are laid out exactly like a contiguous cache whose batch is
 *    the page number and whose capacity is P: k_codes [num_pages][Hkv][P*d*n/32],
 *    k_scales / k_zeros [num_pages][Hkv][P/G][d], v_codes likewise, v_scales /
 *    v_zeros [num_pages][Hkv][P][d/Gv].
 *  - k_residual, v_residual: e [B][Hkv][R][d], one residual per slot.
 *  - page_table: int32 [B][capacity / P], caller-owned device memory.  Entry
 *    [b][j] is the pool page holding tokens [jP, (j+1)P) of slot b.  The library
 *    reads it at run time and never writes it.  The caller fills entry j of slot
 *    b, in stream order, before the first call that writes or reads one of those
 *    tokens: a prefill (entries 0 .. ceil(Tq/P) - 1), an append whose flush
 *    reaches a new page (entry Tq/P before the flush), every later decode.  Pages
 *    of live slots must be distinct.  A kernel that meets an entry outside
 *    [0, num_pages) touches page 0 instead (reads) or writes nothing (flushes)
 *    and raises a status bit that kvq_paged_check_device reports.
 * State: each slot is inactive (after create and release) or active with a length
 * of len tokens (Tq = floor(len / R) R quantized, r = len mod R residual), kept
 * on the host for planning and on the device (in the state buffer) for the kernels.
 * ---------------------------------------------------------------------------
 */
typedef struct {
    kvq_config geom;      /* batch = sequence slots B; capacity = quantized tokens one
                             sequence may hold, a multiple of page_tokens           */
    int32_t page_tokens;  /* P: a multiple of residual (R) and of 64                */
    int32_t num_pages;    /* pages in the pool, >= 1                                */
} kvq_paged_config;

typedef struct {
    size_t k_codes, k_scales, k_zeros;   /* the pool of num_pages pages             */
    size_t v_codes, v_scales, v_zeros;
    size_t k_residual, v_residual;       /* [B][Hkv][R][d] e                        */
    size_t page_table;                   /* int32 [B][capacity / P]                 */
    size_t workspace;                    /* scratch of kvq_paged_decode_attention   */
    size_t state;                        /* kvq_buffers.state of the paged cache    */
} kvq_paged_sizes;

typedef struct kvq_paged kvq_paged;   /* opaque host-side handle */

/* Validates `cfg` and fills `out` with the buffer sizes.  No device needed. */
KVQ_API kvq_status kvq_paged_get_sizes(const kvq_paged_config *cfg, kvq_paged_sizes *out);

/*
 * Creates a handle over the caller's pool, residual, state and page-table
 * buffers (not copied, not freed); every slot starts inactive.  Like kvq_create,
 * initialises the state buffer (synchronously): split-arrival counters, the
 * status word and the slots' lengths.  Allocates no device memory.
 */
KVQ_API kvq_status kvq_paged_create(const kvq_paged_config *cfg, const kvq_buffers *bufs,
                                    const int32_t *page_table, kvq_paged **out);

/* Frees the handle and the library's array.  NULL is ignored. */
KVQ_API void kvq_paged_destroy(kvq_paged *cache);

/*
 * Prefill of slot `seq` (inactive; KVQ_ERR_STATE otherwise) with the prompt
 * X_K, X_V: e [Hkv][T][d] device tensors.  As kvq_prefill_quantize for one
 * sequence: its first Tq = floor(T/R) R tokens are quantized into the pages of
 * its page table, the rest copied into its residual; the slot becomes active
 * with len = T (T = 0 allowed).  Tq > capacity gives KVQ_ERR_CAPACITY.
 */
KVQ_API kvq_status kvq_paged_prefill(kvq_paged *cache, int32_t seq, const void *X_K, const void *X_V,
                                     int64_t T, void *stream);

/*
 * Decode-phase append to every active slot: t_K, t_V are e [B][Hkv][d] (rows of
 * inactive slots are ignored).  Each active slot's row goes to its residual row r
 * and its len grows by one; the slots whose residual becomes full (r = R) are
 * flushed (quantized into tokens [Tq, Tq + R) of their pages).  KVQ_ERR_CAPACITY
 * (nothing launched) if a flush would pass capacity.  One launch, plus one when
 * any slot flushes.
 */
KVQ_API kvq_status kvq_paged_append(kvq_paged *cache, const void *t_K, const void *t_V, void *stream);

/*
 * Decode attention of every slot: t_Q e [B][Hq][d] -> t_O float [B][Hq][d] as
 * kvq_decode_attention, each slot over its own tokens; an inactive or empty slot
 * gives zeros.  `workspace`: at least kvq_paged_sizes.workspace bytes.  One
 * launch.
 */
KVQ_API kvq_status kvq_paged_decode_attention(kvq_paged *cache, const void *t_Q, float *t_O,
                                              void *workspace, size_t workspace_bytes, void *stream);

/*
 * Makes slot `seq` inactive (its pages are the caller's to reuse once the work
 * queued before this call is done).  One launch (it sets the device length).
 */
KVQ_API kvq_status kvq_paged_release(kvq_paged *cache, int32_t seq, void *stream);

/* Length of slot `seq` (-1 when inactive). */
KVQ_API kvq_status kvq_paged_seq_len(const kvq_paged *cache, int32_t seq, int64_t *len);

/* Number of token splits the next kvq_paged_decode_attention would use (>= 1). */
KVQ_API int32_t kvq_paged_decode_splits(const kvq_paged *cache);

/*
 * As kvq_check_device, for a paged cache.  Also reports (KVQ_ERR_DEVICE_CHECK,
 * bit 1) a page-table entry outside the pool met by a kernel since the last
 * check; the outputs since then are unreliable and the word is cleared.
 */
KVQ_API kvq_status kvq_paged_check_device(kvq_paged *cache);

/*
 * ---------------------------------------------------------------------------
 * LogQuant retention ("Resumo Técnico: LogQuant", section 2, Estratégia de
 * Filtragem Baseada em Logaritmos, and section 4).  Instead of KIVI's residual of
 * the newest < R tokens, a full-precision store keeps up to 3W tokens: every new
 * token enters it; when it holds 3W, every other one of its 2W oldest tokens (the
 * 2nd, 4th, ... oldest) leaves it and those W tokens are quantized together as
 * one block (keys per channel over groups of G tokens inside the block, values
 * per token), appended to the quantized tokens in the order the blocks leave.
 * Repeated halving leaves the store log-spaced (the newest tokens dense, older
 * ones at strides 2, 4, ...; the first token stays).  Attention runs over
 * [deq(blocks); store], whose order does not matter.
 *
 * A LogQuant cache is a kvq_cache: kvq_prefill_quantize (the prompt's tokens
 * enter one by one), kvq_append, kvq_append_decode_attention, the decode calls,
 * kvq_cache_state (r = tokens in the store), kvq_reset and kvq_destroy serve it.
 * Its residual buffers hold the store: e [B][Hkv][3W][d], rows in ascending
 * token position.  The cache's capacity is rounded up to a multiple of 3W for
 * the layout (kvq_logquant_get_sizes reports the sizes).  Its prefill uploads
 * row lists from host memory with one copy (so it cannot be captured in a CUDA
 * graph); append and decode can.  Its state buffer also holds (capacity + 4W)
 * int32 row indices (kvq_logquant_get_sizes counts them in `state`).
 * ---------------------------------------------------------------------------
 */

/* Buffer sizes of a LogQuant cache with window W (W a multiple of group_k in
 * 16..4096; cfg->residual is ignored; capacity a multiple of W). */
KVQ_API kvq_status kvq_logquant_get_sizes(const kvq_config *cfg, int32_t window, kvq_sizes *out);

/* Creates a LogQuant cache over caller-owned buffers (sizes as above). */
KVQ_API kvq_status kvq_logquant_create(const kvq_config *cfg, int32_t window, const kvq_buffers *bufs,
                                       kvq_cache **out);

/*
 * Token positions of the rows of the full-precision store, in row order
 * (ascending): *count receives their number; `positions` (host, `capacity`
 * entries, or NULL to ask for the count only) receives them.  KVQ_ERR_STATE for
 * a cache that is not a LogQuant cache.
 */
KVQ_API kvq_status kvq_logquant_retained(const kvq_cache *cache, int64_t *positions, int32_t capacity,
                                         int32_t *count);

/*
 * Dense-and-sparse keys (the KV-cache quantization pages: KVQuant's per-vector
 * dense-and-sparse quantization keeps a small share of outliers, e.g. 1%, at
 * full precision in a separate sparse matrix; SqueezeLLM's W = D + S).  For each
 * token's key (d channels of one kv head) the n_out entries of largest magnitude
 * (ties: the lower channel) form the sparse part; they are set to +0 in the
 * dense part, which is quantized as usual.  The 0 quantizes to its group's zero
 * point and dequantizes to exactly 0, so the reconstruction deq(D) + S is exact
 * at the outliers; the decode adds q_c x_c of each outlier to its token's logit.
 * Values are unchanged.
 *
 * Enables this on an empty cache (KVQ_ERR_STATE otherwise) of the tensor-core
 * path: 1, 2 or 4 query heads per kv head and key groups of >= 32 tokens
 * (KVQ_ERR_UNSUPPORTED otherwise); not for paged caches.  n_out: 1 or 2 (about
 * 1% or 2% of d = 128); 0 turns it off.  k_outliers: caller-owned device memory
 * of at least `bytes` = B * Hkv * capacity * n_out * 4 bytes (capacity as in the
 * cache's sizes; a LogQuant cache's is rounded up to a multiple of 3W), holding
 * uint32 [B][Hkv][capacity][n_out]: per quantized token its outliers, largest
 * first, each (channel << 16) | element bits.  Applies to every later prefill,
 * flush (and LogQuant block) of this cache.
 */
KVQ_API kvq_status kvq_set_key_outliers(kvq_cache *cache, int32_t n_out, uint32_t *k_outliers, size_t bytes);

/* Kernels this library has launched in the process so far (all devices). */
KVQ_API uint64_t kvq_kernel_launches(void);

/* Description of the last error on the calling thread ("" if none). */
KVQ_API const char *kvq_last_error(void);

/* Version of the storage format described above (currently 2). */
KVQ_API int32_t kvq_layout_version(void);

/*
 * The GPU architecture the library's kernels were compiled for, as the CUDA
 * runtime reports it for a loaded kernel (major * 10 + minor: 100 for sm_100a),
 * or -1 when it cannot be read (no device).  Needs the device the caller uses to
 * be current.  The pages have no counterpart.
 */
KVQ_API int32_t kvq_binary_arch(void);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H */
