// kvq_api.cu -- the C ABI of include/kvq.h: validation, host-side cache state and launches.
//
// A contiguous cache's handle keeps geometry, the caller's device pointers and
// the two counters of the KIVI cache ("LLM系列：KVCache量化1 KIVI ...", section 1):
// Tq quantized tokens and r < R residual tokens; a LogQuant cache also keeps
// the positions of its full-precision store, a paged cache every slot's length.
// Every branch of the streaming logic (when to flush, where a token goes, how
// many splits) is decided here on the host from that state, so a sequence of
// calls never waits on the device.  The kernels read their own copy of the
// state only where a batch is ragged (the paged cache's slot lengths).
#include <cmath>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <mutex>
#include <new>
#include <string>
#include <vector>

#include "../../include/kvq.h"
#include "kvq_internal.cuh"

namespace {
std::atomic<uint64_t> g_launches{0};
}  // namespace

void kvq::count_launches(int n) { g_launches.fetch_add(static_cast<uint64_t>(n)); }

namespace {

thread_local std::string g_last_error;

kvq_status fail(kvq_status st, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
kvq_status fail(kvq_status st, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return st;
}

kvq_status ok() {
    g_last_error.clear();
    return KVQ_OK;
}

kvq_status cuda_fail(cudaError_t e, const char *what) {
    return fail(KVQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr int kMaxSplits = 128;
constexpr int kMaxResidualSplits = 16;
static_assert(kMaxSplits + kMaxResidualSplits == kvq::kMaxDecodeSplits, "split bound");
constexpr int kMinTilesPerSplit = 4;

kvq_status validate(const kvq_config *c) {
    if (!c) return fail(KVQ_ERR_INVALID_ARG, "config is NULL");
    if (c->batch < 1 || c->q_heads < 1 || c->kv_heads < 1)
        return fail(KVQ_ERR_INVALID_ARG, "batch, q_heads and kv_heads must be >= 1");
    if (c->q_heads % c->kv_heads != 0)
        return fail(KVQ_ERR_INVALID_ARG, "q_heads (%d) must be a multiple of kv_heads (%d)",
                    c->q_heads, c->kv_heads);
    if (static_cast<int64_t>(c->batch) * c->kv_heads > 65535 ||
        static_cast<int64_t>(c->batch) > 65535 || c->q_heads > 65535)
        return fail(KVQ_ERR_UNSUPPORTED, "batch * kv_heads must be <= 65535");
    if (c->bits != 2 && c->bits != 4)
        return fail(KVQ_ERR_UNSUPPORTED, "bits must be 2 or 4 (got %d)", c->bits);
    if (c->head_dim != 64 && c->head_dim != 128)
        return fail(KVQ_ERR_UNSUPPORTED, "head_dim must be 64 or 128 (got %d)", c->head_dim);
    if (!(c->group_k == 16 || c->group_k == 32 || c->group_k == 64 || c->group_k == 128 ||
          c->group_k == 256) ||
        c->group_k * c->head_dim > 32768)
        return fail(KVQ_ERR_INVALID_ARG,
                    "group_k must be 16, 32, 64, 128 or 256 with group_k*head_dim <= 32768");
    if (!(c->group_v == 16 || c->group_v == 32 || c->group_v == 64 || c->group_v == 128) ||
        c->group_v > c->head_dim)
        return fail(KVQ_ERR_INVALID_ARG, "group_v must be 16, 32, 64 or 128 and <= head_dim");
    if (c->residual < c->group_k || c->residual % c->group_k != 0)
        return fail(KVQ_ERR_INVALID_ARG, "residual (%d) must be a positive multiple of group_k (%d)",
                    c->residual, c->group_k);
    if (c->symmetric != 0 && c->symmetric != 1)
        return fail(KVQ_ERR_INVALID_ARG, "symmetric must be 0 or 1");
    if (c->dtype != KVQ_FP16 && c->dtype != KVQ_BF16)
        return fail(KVQ_ERR_INVALID_ARG, "dtype must be KVQ_FP16 or KVQ_BF16");
    if (c->capacity < c->residual || c->capacity % c->residual != 0)
        return fail(KVQ_ERR_INVALID_ARG, "capacity must be a positive multiple of residual");
    if (c->capacity / 16 > (int64_t{1} << 30))
        return fail(KVQ_ERR_UNSUPPORTED, "capacity too large");
    return KVQ_OK;
}

// Splits over the quantized tiles are at most kMaxSplits; the residual rows add up to
// kMaxResidualSplits.
int max_splits(const kvq_config *c) {
    const int64_t tiles = c->capacity / 16;
    return static_cast<int>(tiles < kMaxSplits ? tiles : kMaxSplits) + kMaxResidualSplits;
}

// The state buffer: split-arrival counters [B * Hq] and the status word (u32), padded to
// 16 bytes; a LogQuant cache adds its row lists, a paged cache its slots' lengths.
size_t counter_bytes(const kvq_config *c) {
    const size_t n = (static_cast<size_t>(c->batch) * c->q_heads + 1) * sizeof(unsigned int);
    return (n + 15) / 16 * 16;
}
size_t lq_list_entries(const kvq_config *g, int32_t W) {
    return static_cast<size_t>(W) + static_cast<size_t>(g->capacity) + 3 * static_cast<size_t>(W);
}

}  // namespace

struct kvq_cache {
    kvq_config cfg;
    kvq_buffers buf;
    unsigned int *arrivals = nullptr;   // device, in the caller's state buffer: B * Hq split-arrival
                                        // counters, then the status word
    int64_t Tq = 0;
    int32_t r = 0;
    int num_sms = 148;
    int ctas_per_sm = 4;
    int split_limit = kMaxSplits;
    int path = kvq::kPathSplit;         // the decode kernel (kvq::DecodePath) serving this cache
    int stall_polls = 0;                // bounds-check builds: see kvq_debug_set_stall
    // LogQuant retention (lq_window W > 0): the residual buffer is the full-precision store
    // of up to 3W rows (cfg.residual = 3W), rows in ascending token position; lq_F holds
    // those positions, lq_n the tokens seen.  lq_rows (device, in the caller's state buffer
    // after the counters): [0, W) the rows an event quantizes (1, 3, ..., 2W - 1), then room
    // for a prefill's row lists.
    int32_t lq_window = 0;
    int32_t *lq_rows = nullptr;
    // dense-and-sparse keys: n_out outlier words per token (caller-owned), or none
    uint32_t *k_out = nullptr;
    int32_t n_out = 0;
    std::vector<int64_t> lq_F;
    int64_t lq_n = 0;
};

namespace {

// Split count for a decode.  The quantized tiles of every sequence are cut into
// splits of tiles_per_split tiles (a multiple of the path's tile alignment); S
// covers the longest sequence, and a shorter one leaves its later splits empty.
// The residual rows (if any) get one split of their own, except on the tensor-core
// path with one query head per kv head, where they are dealt to the warps of the
// quantized splits.  A CTA's time is modelled as a fixed start/finish cost of
// kCtaFixedTiles tiles plus the tiles its busiest warp streams (an empty split
// costs kEmptyCtaTiles); the kernel's time as the largest of (the waves of quantized
// CTAs over the GPU's resident slots x one quantized CTA), (all CTA time spread evenly
// over the slots, plus one residual CTA) and the longest chain of CTAs on one slot; when
// every CTA is resident at once it is the longest CTA's.  The split count with the
// lowest modelled time wins (ties: fewer splits).
constexpr double kCtaFixedTiles = 6.0;
// a residual CTA starts and ends cheaper (no copy pipeline; measured: more, shorter residual
// CTAs beside a one-wave quantized grid pay on the bf16-MMA kernel)
constexpr double kResCtaFixedTiles = 2.0;
constexpr double kEmptyCtaTiles = 1.0;

// The sequences' lengths as the planner sees them: n entries of quantized tiles,
// each standing for `mult` sequences, and the most residual rows of any sequence.
struct PlanInput {
    const int64_t *tiles;
    int n;
    int64_t mult;
    int32_t max_r;
};

void plan_splits_for(const kvq_cache *h, const PlanInput &in, int *n_qsplits, int *tiles_per_split,
                     int *S_out) {
    const kvq_config &c = h->cfg;
    int64_t tiles = 0;
    for (int i = 0; i < in.n; ++i) tiles = in.tiles[i] > tiles ? in.tiles[i] : tiles;
    const int path = h->path;
    // with one query head per kv head the integer-MMA kernel deals the residual tiles to the
    // warps of the quantized splits
    const int hg = c.q_heads / c.kv_heads;
    const bool res_shared = path == kvq::kPathTc && hg == 1;
    const bool per_kv = kvq::path_per_kv_head(path);
    const int extra = (in.max_r > 0 && !res_shared) ? 1 : 0;   // residual splits (the tensor-core
                                                                // path may take more, below)
    const int64_t align = kvq::split_tile_align(path);
    // CTAs per split and sequence: one per kv head on the tensor-core path, else one per query head
    const int64_t per_seq = per_kv ? c.kv_heads : c.q_heads;
    const int64_t units = static_cast<int64_t>(c.batch) * per_seq;
    const double slots = static_cast<double>(h->num_sms) * h->ctas_per_sm;
    const int64_t nres = (in.max_r + 15) / 16;
    // residual CTA: its tiles shared by the 4 warps of each of its query heads
    const int heads_per_cta = per_kv ? hg : 1;
    const double c_res1 = kResCtaFixedTiles + static_cast<double>((nres * heads_per_cta + 3) / 4);
    // the tensor-core kernel deals the residual tiles over the warps of n_rs residual splits
    // (4 / HG warps per head in each); a residual tile on CUDA cores costs about two
    // quantized tiles.  n_rs grows until a residual warp's share costs no more than a
    // quantized CTA (a long full-precision store, e.g. LogQuant's, then spreads out).
    const int64_t wph = 4 / heads_per_cta;
    auto residual_cost = [&](int64_t n_rs) {
        return kResCtaFixedTiles + 2.0 * static_cast<double>((nres + wph * n_rs - 1) / (wph * n_rs));
    };
    int64_t best_S = 0, best_per = 1, best_rs = extra;
    if (tiles > 0) {
        int64_t cap = (tiles + kMinTilesPerSplit - 1) / kMinTilesPerSplit;
        if (cap > max_splits(&c) - kMaxResidualSplits) cap = max_splits(&c) - kMaxResidualSplits;
        if (cap > h->split_limit) cap = h->split_limit;
        if (cap < 1) cap = 1;
        double best_cost = -1.0;
        for (int64_t S = 1; S <= cap; ++S) {
            const int64_t per = ((tiles + S - 1) / S + align - 1) / align * align;
            if ((tiles + per - 1) / per != S) continue;
            const int64_t per_warp = ((per + 4 * align - 1) / (4 * align)) * align;
            // a residual tile on CUDA cores costs about two quantized tiles
            const int64_t res_warp = res_shared ? (nres + 4 * S - 1) / (4 * S) : 0;
            const double c_q = kCtaFixedTiles + static_cast<double>(per_warp + 2 * res_warp);
            int64_t busy = 0;   // non-empty quantized splits over all sequences
            for (int i = 0; i < in.n; ++i) busy += in.mult * ((in.tiles[i] + per - 1) / per);
            const double nq = static_cast<double>(per_seq * busy);
            const double n_empty = static_cast<double>(units * S) - nq;
            const double t_waves = std::ceil(nq / slots) * c_q;
            // residual splits: the tensor-core path tries 1 .. most of them (most: one tile per
            // residual warp).  Residual CTAs start after every quantized CTA (the grid's order):
            // when they do not all fit beside the quantized ones, they add to the critical path.
            int64_t most = 1;
            if (extra && per_kv) {
                most = (nres + wph - 1) / wph;
                if (most > kMaxResidualSplits) most = kMaxResidualSplits;
            }
            for (int64_t n_rs = extra; n_rs <= (extra ? most : 0); ++n_rs) {
                const double c_res = (per_kv && n_rs) ? residual_cost(n_rs) : c_res1;
                const double n_res = static_cast<double>(units * n_rs);
                const double t_spread =
                    (nq * c_q + n_empty * kEmptyCtaTiles + n_res * c_res) / slots + (n_rs ? c_res : 0.0);
                // the longest chain of CTAs on one slot: with the quantized CTAs resident in one
                // wave, the residual CTAs run in turns on the slots left beside them; else
                // they start after the quantized ones
                double t_crit = c_q;
                if (n_rs) {
                    if (nq + n_res <= slots) {
                        t_crit = c_res > c_q ? c_res : c_q;
                    } else if (nq < slots) {
                        const double turns = std::ceil(n_res / (slots - nq));
                        t_crit = c_res * turns > c_q ? c_res * turns : c_q;
                    } else {
                        t_crit = c_q + c_res;
                    }
                }
                double cost = t_waves > t_spread ? t_waves : t_spread;
                cost = cost > t_crit ? cost : t_crit;
                // every CTA resident at once (one wave): the longest CTA sets the time
                if (nq + n_res + n_empty <= slots) cost = t_crit;
                if (best_cost < 0 || cost < best_cost - 1e-9) {
                    best_cost = cost;
                    best_S = S;
                    best_per = per;
                    best_rs = n_rs;
                }
            }
        }
    }
    if (res_shared && best_S == 0) {   // residual rows only: one split whose warps share them
        best_S = 1;
        best_per = 0;
    }
    if (best_S == 0 && extra && per_kv) {   // residual rows only: spread them too
        int64_t most = (nres + wph - 1) / wph;
        if (most > kMaxResidualSplits) most = kMaxResidualSplits;
        const int64_t want = (static_cast<int64_t>(slots) + units - 1) / units;
        best_rs = want < most ? want : most;
        if (best_rs < 1) best_rs = 1;
    }
    if (best_S + best_rs == 0) {        // nothing in any sequence: one empty split writes zeros
        best_S = 1;
        best_per = align;
    }
    *n_qsplits = static_cast<int>(best_S);
    *tiles_per_split = static_cast<int>(best_per);
    *S_out = static_cast<int>(best_S + best_rs);
}

void plan_splits(const kvq_cache *h, int *n_qsplits, int *tiles_per_split, int *S_out) {
    const int64_t tiles = h->Tq / 16;
    const PlanInput in{&tiles, 1, h->cfg.batch, h->r};
    plan_splits_for(h, in, n_qsplits, tiles_per_split, S_out);
}

kvq::DecodeArgs decode_args(const kvq_cache *h) {
    const kvq_config &c = h->cfg;
    kvq::DecodeArgs a{};
    a.kc = static_cast<const uint32_t *>(h->buf.k_codes);
    a.vc = static_cast<const uint32_t *>(h->buf.v_codes);
    a.ks = h->buf.k_scales;
    a.vs = h->buf.v_scales;
    a.kz = h->buf.k_zeros;
    a.vz = h->buf.v_zeros;
    a.kr = static_cast<uint16_t *>(h->buf.k_residual);
    a.vr = static_cast<uint16_t *>(h->buf.v_residual);
    a.new_k = a.new_v = nullptr;
    a.new_row = -1;
    a.cap = c.capacity;
    a.B = c.batch;
    a.Hq = c.q_heads;
    a.Hkv = c.kv_heads;
    a.d = c.head_dim;
    a.G = c.group_k;
    a.Gv = c.group_v;
    a.R = c.residual;
    a.bits = c.bits;
    a.sym = c.symmetric != 0;
    a.bf16 = c.dtype == KVQ_BF16;
    a.path = h->path;
    a.arrivals = h->arrivals;
    a.status = h->arrivals + static_cast<int64_t>(c.batch) * c.q_heads;
    a.k_out = h->k_out;
    a.n_out = h->n_out;
    a.gshift = 0;
    while ((16 << a.gshift) < c.group_k) ++a.gshift;
    a.qscale = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(c.head_dim)));
    a.stall_polls = h->stall_polls;
    return a;
}

kvq::QuantizeArgs quantize_args(const kvq_cache *h) {
    const kvq_config &c = h->cfg;
    kvq::QuantizeArgs q{};
    q.BH = static_cast<int64_t>(c.batch) * c.kv_heads;
    q.d = c.head_dim;
    q.G = c.group_k;
    q.Gv = c.group_v;
    q.bits = c.bits;
    q.sym = c.symmetric != 0;
    q.bf16 = c.dtype == KVQ_BF16;
    q.kc = static_cast<uint32_t *>(h->buf.k_codes);
    q.vc = static_cast<uint32_t *>(h->buf.v_codes);
    q.ks = h->buf.k_scales;
    q.vs = h->buf.v_scales;
    q.kz = h->buf.k_zeros;
    q.vz = h->buf.v_zeros;
    q.cap = c.capacity;
    q.k_out = h->k_out;
    q.n_out = h->n_out;
    q.status = h->arrivals + static_cast<int64_t>(c.batch) * c.q_heads;
    return q;
}

// LogQuant host state: token lq_n enters the full-precision positions; at an event (the
// store reached 3W) every other one of the 2W oldest leaves ("Resumo Técnico: LogQuant",
// section 2; the same rule the kernels apply to the rows).
void lq_push(kvq_cache *h) {
    if (!h->lq_window) return;
    const int64_t W = h->lq_window;
    std::vector<int64_t> &F = h->lq_F;
    F.push_back(h->lq_n++);
    if (static_cast<int64_t>(F.size()) < 3 * W) return;
    for (int64_t i = 0; i < W; ++i) F[i] = F[2 * i];
    for (int64_t j = 0; j < W; ++j) F[W + j] = F[2 * W + j];
    F.resize(2 * W);
}

kvq_status lq_prefill(kvq_cache *h, const void *X_K, const void *X_V, int64_t T, void *stream);
kvq_status check_status_word(unsigned int *word);

kvq_status check_decode_args(const kvq_cache *h, const void *t_Q, const float *t_O, const void *workspace,
                             size_t workspace_bytes);
kvq_status launch_decode_call(kvq_cache *h, const void *t_Q, float *t_O, void *workspace,
                              const uint16_t *new_k, const uint16_t *new_v, void *stream,
                              float *po = nullptr, float *pm = nullptr, float *pl = nullptr);

}  // namespace

extern "C" {

kvq_status kvq_get_sizes(const kvq_config *cfg, kvq_sizes *out) {
    if (!out) return fail(KVQ_ERR_INVALID_ARG, "out is NULL");
    kvq_status st = validate(cfg);
    if (st != KVQ_OK) return st;
    const int64_t BH = static_cast<int64_t>(cfg->batch) * cfg->kv_heads;
    const int64_t cap = cfg->capacity;
    const int64_t d = cfg->head_dim;
    std::memset(out, 0, sizeof *out);
    out->k_codes = out->v_codes = static_cast<size_t>(BH * cap * d * cfg->bits / 8);
    out->k_scales = static_cast<size_t>(BH * (cap / cfg->group_k) * d * 4);
    out->k_zeros = cfg->symmetric ? 0 : static_cast<size_t>(BH * (cap / cfg->group_k) * d * 2);
    out->v_scales = static_cast<size_t>(BH * cap * (d / cfg->group_v) * 4);
    out->v_zeros = cfg->symmetric ? 0 : static_cast<size_t>(BH * cap * (d / cfg->group_v) * 2);
    out->k_residual = out->v_residual = static_cast<size_t>(BH * cfg->residual * d * 2);
    const int64_t units = static_cast<int64_t>(cfg->batch) * cfg->q_heads;
    out->workspace = static_cast<size_t>(units * max_splits(cfg) * (d + 2) * 4);
    out->state = counter_bytes(cfg);
    return ok();
}

kvq_status kvq_create(const kvq_config *cfg, const kvq_buffers *bufs, kvq_cache **out) {
    if (!out) return fail(KVQ_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    kvq_status st = validate(cfg);
    if (st != KVQ_OK) return st;
    if (!bufs) return fail(KVQ_ERR_INVALID_ARG, "buffers are NULL");
    const void *need[] = {bufs->k_codes, bufs->k_scales, bufs->v_codes, bufs->v_scales,
                          bufs->k_residual, bufs->v_residual, bufs->state};
    for (const void *p : need)
        if (!p || !aligned16(p))
            return fail(KVQ_ERR_INVALID_ARG, "cache buffers and the state buffer must be non-NULL and "
                                             "16-byte aligned");
    if (!cfg->symmetric && (!bufs->k_zeros || !bufs->v_zeros || !aligned16(bufs->k_zeros) ||
                            !aligned16(bufs->v_zeros)))
        return fail(KVQ_ERR_INVALID_ARG, "asymmetric caches need 16-byte aligned zero buffers");
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "querying the current device");
    kvq_cache *h = new (std::nothrow) kvq_cache();
    if (!h) return fail(KVQ_ERR_INVALID_ARG, "out of host memory");
    h->cfg = *cfg;
    h->buf = *bufs;
    if (cfg->symmetric) {
        h->buf.k_zeros = nullptr;
        h->buf.v_zeros = nullptr;
    }
    h->num_sms = sms > 0 ? sms : 148;
    h->path = kvq::decode_path(cfg->q_heads, cfg->kv_heads, cfg->group_k);
    h->ctas_per_sm = kvq::decode_ctas_per_sm(decode_args(h));
    // the decode kernels' split-arrival counters (zeroed once here, left at zero by every
    // decode) and, after them, their status word: the start of the caller's state buffer
    h->arrivals = static_cast<unsigned int *>(bufs->state);
    e = cudaMemset(h->arrivals, 0, counter_bytes(cfg));
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) {
        delete h;
        return cuda_fail(e, "zeroing the state buffer");
    }
    *out = h;
    return ok();
}

void kvq_destroy(kvq_cache *cache) { delete cache; }

kvq_status kvq_reset(kvq_cache *cache) {
    if (!cache) return fail(KVQ_ERR_INVALID_ARG, "cache is NULL");
    cache->Tq = 0;
    cache->r = 0;
    cache->lq_F.clear();
    cache->lq_n = 0;
    return ok();
}

kvq_status kvq_prefill_quantize(kvq_cache *h, const void *X_K, const void *X_V, int64_t T,
                                void *stream) {
    if (!h) return fail(KVQ_ERR_INVALID_ARG, "cache is NULL");
    if (T < 0) return fail(KVQ_ERR_INVALID_ARG, "T must be >= 0");
    if (h->Tq != 0 || h->r != 0) return fail(KVQ_ERR_STATE, "prefill needs an empty cache");
    if (T == 0) return ok();
    if (!X_K || !X_V || !aligned16(X_K) || !aligned16(X_V))
        return fail(KVQ_ERR_INVALID_ARG, "X_K and X_V must be non-NULL and 16-byte aligned");
    if (h->lq_window) return lq_prefill(h, X_K, X_V, T, stream);
    const kvq_config &c = h->cfg;
    const int64_t Tq = (T / c.residual) * c.residual;
    const int64_t r = T - Tq;
    if (Tq > c.capacity)
        return fail(KVQ_ERR_CAPACITY, "prefill of %lld tokens exceeds capacity %lld",
                    static_cast<long long>(Tq), static_cast<long long>(c.capacity));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    kvq::QuantizeArgs q = quantize_args(h);
    q.xk = static_cast<const uint16_t *>(X_K);
    q.xv = static_cast<const uint16_t *>(X_V);
    q.in_bh_stride = T * c.head_dim;
    q.in_tok0 = 0;
    q.n_groups = Tq / c.group_k;
    q.out_tok0 = 0;
    cudaError_t e = kvq::launch_quantize(q, s);
    if (e != cudaSuccess) return cuda_fail(e, "prefill quantize launch");
    const int64_t BH = static_cast<int64_t>(c.batch) * c.kv_heads;
    const int64_t rstride = static_cast<int64_t>(c.residual) * c.head_dim;
    e = kvq::launch_copy_rows(static_cast<const uint16_t *>(X_K), static_cast<const uint16_t *>(X_V),
                              T * c.head_dim, Tq, static_cast<uint16_t *>(h->buf.k_residual),
                              static_cast<uint16_t *>(h->buf.v_residual), rstride, 0, r, BH,
                              c.head_dim, s);
    if (e != cudaSuccess) return cuda_fail(e, "prefill residual copy launch");
    h->Tq = Tq;
    h->r = static_cast<int32_t>(r);
    return ok();
}

kvq_status kvq_append(kvq_cache *h, const void *t_K, const void *t_V, void *stream) {
    if (!h) return fail(KVQ_ERR_INVALID_ARG, "cache is NULL");
    if (!t_K || !t_V || !aligned16(t_K) || !aligned16(t_V))
        return fail(KVQ_ERR_INVALID_ARG, "t_K and t_V must be non-NULL and 16-byte aligned");
    const kvq_config &c = h->cfg;
    const bool flush = h->r + 1 == c.residual;
    const int64_t flush_tokens = h->lq_window ? h->lq_window : c.residual;
    if (flush && h->Tq + flush_tokens > c.capacity)
        return fail(KVQ_ERR_CAPACITY, "flushing the residual would exceed capacity %lld",
                    static_cast<long long>(c.capacity));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t BH = static_cast<int64_t>(c.batch) * c.kv_heads;
    const int64_t rstride = static_cast<int64_t>(c.residual) * c.head_dim;
    cudaError_t e = kvq::launch_copy_rows(
        static_cast<const uint16_t *>(t_K), static_cast<const uint16_t *>(t_V), c.head_dim, 0,
        static_cast<uint16_t *>(h->buf.k_residual), static_cast<uint16_t *>(h->buf.v_residual),
        rstride, h->r, 1, BH, c.head_dim, s);
    if (e != cudaSuccess) return cuda_fail(e, "append launch");
    if (flush && h->lq_window) {
        // LogQuant event: the W rows 1, 3, ..., 2W - 1 (every other one of the 2W oldest)
        // leave the full-precision store as one quantized block; the store is compacted
        const int W = h->lq_window;
        kvq::QuantizeArgs q = quantize_args(h);
        q.xk = static_cast<const uint16_t *>(h->buf.k_residual);
        q.xv = static_cast<const uint16_t *>(h->buf.v_residual);
        q.in_bh_stride = rstride;
        q.in_rows = h->lq_rows;
        q.in_rows_limit = c.residual;
        q.n_groups = W / c.group_k;
        q.out_tok0 = h->Tq;
        e = kvq::launch_quantize(q, s);
        if (e == cudaSuccess)
            e = kvq::launch_lq_compact(static_cast<uint16_t *>(h->buf.k_residual),
                                       static_cast<uint16_t *>(h->buf.v_residual), BH, c.residual, W,
                                       c.head_dim, q.status, s);
        if (e != cudaSuccess) return cuda_fail(e, "LogQuant event launch");
        lq_push(h);
        h->Tq += W;
        h->r = 2 * W;
    } else if (flush) {
        kvq::QuantizeArgs q = quantize_args(h);
        q.xk = static_cast<const uint16_t *>(h->buf.k_residual);
        q.xv = static_cast<const uint16_t *>(h->buf.v_residual);
        q.in_bh_stride = rstride;
        q.in_tok0 = 0;
        q.n_groups = c.residual / c.group_k;
        q.out_tok0 = h->Tq;
        e = kvq::launch_quantize(q, s);
        if (e != cudaSuccess) return cuda_fail(e, "flush quantize launch");
        h->Tq += c.residual;
        h->r = 0;
    } else {
        lq_push(h);
        h->r += 1;
    }
    return ok();
}

kvq_status kvq_set_split_limit(kvq_cache *h, int32_t max_splits) {
    if (!h) return fail(KVQ_ERR_INVALID_ARG, "cache is NULL");
    if (max_splits < 0 || max_splits > kMaxSplits)
        return fail(KVQ_ERR_INVALID_ARG, "max_splits must be in 0..%d", kMaxSplits);
    h->split_limit = max_splits == 0 ? kMaxSplits : max_splits;
    return ok();
}

kvq_status kvq_set_decode_kernel(kvq_cache *h, int32_t kernel) {
    if (!h) return fail(KVQ_ERR_INVALID_ARG, "cache is NULL");
    const kvq_config &c = h->cfg;
    const bool mma_geom = kvq::decode_path(c.q_heads, c.kv_heads, c.group_k) != kvq::kPathSplit;
    int path;
    switch (kernel) {
        case KVQ_DECODE_AUTO:
            path = h->n_out > 0 ? kvq::kPathTc : kvq::decode_path(c.q_heads, c.kv_heads, c.group_k);
            break;
        case KVQ_DECODE_CUDA_CORES:
            if (h->n_out > 0) return fail(KVQ_ERR_UNSUPPORTED, "key outliers are served by the integer-MMA kernel");
            path = kvq::kPathSplit;
            break;
        case KVQ_DECODE_INT8_MMA:
        case KVQ_DECODE_BF16_MMA:
            if (!mma_geom)
                return fail(KVQ_ERR_UNSUPPORTED, "the MMA kernels need 1, 2 or 4 query heads per kv head and "
                                                 "key groups of >= 32 tokens");
            if (kernel == KVQ_DECODE_BF16_MMA && h->n_out > 0)
                return fail(KVQ_ERR_UNSUPPORTED, "key outliers are served by the integer-MMA kernel");
            path = kernel == KVQ_DECODE_INT8_MMA ? kvq::kPathTc : kvq::kPathMma;
            break;
        default:
            return fail(KVQ_ERR_INVALID_ARG, "unknown decode kernel %d", kernel);
    }
    h->path = path;
    h->ctas_per_sm = kvq::decode_ctas_per_sm(decode_args(h));
    return ok();
}

int32_t kvq_decode_splits(const kvq_cache *h) {
    if (!h) return 0;
    int nq, per, S;
    plan_splits(h, &nq, &per, &S);
    return S;
}

kvq_status kvq_decode_attention(kvq_cache *h, const void *t_Q, float *t_O, void *workspace,
                                size_t workspace_bytes, void *stream) {
    if (!h) return fail(KVQ_ERR_INVALID_ARG, "cache is NULL");
    kvq_status st = check_decode_args(h, t_Q, t_O, workspace, workspace_bytes);
    if (st != KVQ_OK) return st;
    if (h->Tq == 0 && h->r == 0) return fail(KVQ_ERR_STATE, "the cache is empty");
    return launch_decode_call(h, t_Q, t_O, workspace, nullptr, nullptr, stream);
}

kvq_status kvq_append_decode_attention(kvq_cache *h, const void *t_K, const void *t_V, const void *t_Q,
                                       float *t_O, void *workspace, size_t workspace_bytes, void *stream) {
    if (!h) return fail(KVQ_ERR_INVALID_ARG, "cache is NULL");
    if (!t_K || !t_V || !aligned16(t_K) || !aligned16(t_V))
        return fail(KVQ_ERR_INVALID_ARG, "t_K and t_V must be non-NULL and 16-byte aligned");
    kvq_status st = check_decode_args(h, t_Q, t_O, workspace, workspace_bytes);
    if (st != KVQ_OK) return st;
    const kvq_config &c = h->cfg;
    const bool flush = h->r + 1 == c.residual;
    if (flush || !kvq::path_per_kv_head(h->path)) {
        // a flush (or the CUDA-core kernel): the append's own launches, then the decode
        st = kvq_append(h, t_K, t_V, stream);
        if (st != KVQ_OK) return st;
        return launch_decode_call(h, t_Q, t_O, workspace, nullptr, nullptr, stream);
    }
    // one kernel: the new token is read as residual row r and stored there by split 0
    h->r += 1;
    st = launch_decode_call(h, t_Q, t_O, workspace, static_cast<const uint16_t *>(t_K),
                            static_cast<const uint16_t *>(t_V), stream);
    if (st != KVQ_OK) {
        h->r -= 1;
        return st;
    }
    lq_push(h);
    return st;
}

kvq_status kvq_decode_attention_partial(kvq_cache *h, const void *t_Q, float *o_part, float *m_part,
                                        float *l_part, void *workspace, size_t workspace_bytes, void *stream) {
    if (!h) return fail(KVQ_ERR_INVALID_ARG, "cache is NULL");
    if (!m_part || !l_part || !aligned16(m_part) || !aligned16(l_part))
        return fail(KVQ_ERR_INVALID_ARG, "m_part and l_part must be non-NULL and 16-byte aligned");
    kvq_status st = check_decode_args(h, t_Q, o_part, workspace, workspace_bytes);
    if (st != KVQ_OK) return st;
    if (h->Tq == 0 && h->r == 0) return fail(KVQ_ERR_STATE, "the cache is empty");
    return launch_decode_call(h, t_Q, nullptr, workspace, nullptr, nullptr, stream, o_part, m_part, l_part);
}

kvq_status kvq_merge_partials(const float *o_parts, const float *m_parts, const float *l_parts, int32_t n,
                              int64_t rows, int32_t d, float *t_O, void *stream) {
    if (n < 1 || rows < 0 || d < 1) return fail(KVQ_ERR_INVALID_ARG, "n, rows and d must be >= 1, >= 0, >= 1");
    if (rows > 0 && (!o_parts || !m_parts || !l_parts || !t_O))
        return fail(KVQ_ERR_INVALID_ARG, "partials and t_O must be non-NULL");
    if (rows > 0x7fffffffLL) return fail(KVQ_ERR_UNSUPPORTED, "rows must be < 2^31");
    cudaError_t e = kvq::launch_merge_partials(o_parts, m_parts, l_parts, n, rows, d, t_O,
                                               static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "merge launch");
    return ok();
}

}  // extern "C"

namespace {

kvq_status check_decode_args(const kvq_cache *h, const void *t_Q, const float *t_O, const void *workspace,
                             size_t workspace_bytes) {
    if (!t_Q || !t_O || !workspace || !aligned16(t_Q) || !aligned16(t_O) || !aligned16(workspace))
        return fail(KVQ_ERR_INVALID_ARG, "t_Q, t_O and workspace must be non-NULL and 16-byte aligned");
    kvq_sizes sz;
    kvq_get_sizes(&h->cfg, &sz);
    if (workspace_bytes < sz.workspace)
        return fail(KVQ_ERR_INVALID_ARG, "workspace needs %zu bytes, got %zu", sz.workspace,
                    workspace_bytes);
    return KVQ_OK;
}

// Launches one decode over the current state; new_k / new_v (or NULL): residual row r - 1
// is that token, read from it and stored by the kernel; po / pm / pl (or NULL): write the
// cache's partial there instead of t_O.
kvq_status launch_decode_call(kvq_cache *h, const void *t_Q, float *t_O, void *workspace,
                              const uint16_t *new_k, const uint16_t *new_v, void *stream, float *po,
                              float *pm, float *pl) {
    const kvq_config &c = h->cfg;
    kvq::DecodeArgs a = decode_args(h);
    plan_splits(h, &a.n_qsplits, &a.tiles_per_split, &a.S);
    const int64_t units = static_cast<int64_t>(c.batch) * c.q_heads;
    float *ws = static_cast<float *>(workspace);
    a.o_part = ws;
    a.m_part = ws + units * a.S * c.head_dim;
    a.l_part = a.m_part + units * a.S;
    a.q = static_cast<const uint16_t *>(t_Q);
    a.out = t_O;
    a.n_qtiles = static_cast<int>(h->Tq / 16);
    a.r = h->r;
    a.new_k = new_k;
    a.new_v = new_v;
    a.new_row = new_k ? h->r - 1 : -1;
    a.po = po;
    a.pm = pm;
    a.pl = pl;
    cudaError_t e = kvq::launch_decode(a, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "decode launch");
    return ok();
}

}  // namespace

// ---------------------------------------------------------------------------
// Decode attention without a caller-provided workspace.
//
// The split partials live in one file-scope device array instead of caller
// memory.  Host code cannot use the array's name as a device address (it is a
// host-side stand-in for the symbol), so every call looks the address up with
// cudaGetSymbolAddress in the calling thread's current context: a context made
// after a device reset, or another context on the same device, gets its own
// array and never a stale address.  The first lookup in a context may load the
// library's device code.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocScratchFloats = size_t{1} << 20;   // 4 MiB per device

static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchFloats];

kvq_status noalloc_scratch(float **out) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "looking up the static decode scratch");
    *out = static_cast<float *>(p);
    return KVQ_OK;
}

}  // namespace

extern "C" {

kvq_status kvq_decode_attention_noalloc(kvq_cache *h, const void *t_Q, float *t_O, void *stream) {
    if (!h) return fail(KVQ_ERR_INVALID_ARG, "cache is NULL");
    if (!t_Q || !t_O || !aligned16(t_Q) || !aligned16(t_O))
        return fail(KVQ_ERR_INVALID_ARG, "t_Q and t_O must be non-NULL and 16-byte aligned");
    if (h->Tq == 0 && h->r == 0) return fail(KVQ_ERR_STATE, "the cache is empty");
    const kvq_config &c = h->cfg;
    kvq::DecodeArgs a = decode_args(h);
    plan_splits(h, &a.n_qsplits, &a.tiles_per_split, &a.S);
    const int64_t units = static_cast<int64_t>(c.batch) * c.q_heads;
    const size_t need = static_cast<size_t>(units) * a.S * (c.head_dim + 2);
    if (need > kNoAllocScratchFloats)
        return fail(KVQ_ERR_CAPACITY,
                    "this decode needs %zu bytes of scratch but the static scratch holds %zu; "
                    "use kvq_decode_attention with a workspace",
                    need * sizeof(float), kNoAllocScratchFloats * sizeof(float));
    float *ws = nullptr;
    kvq_status st = noalloc_scratch(&ws);
    if (st != KVQ_OK) return st;
    a.o_part = ws;
    a.m_part = ws + units * a.S * c.head_dim;
    a.l_part = a.m_part + units * a.S;
    a.q = static_cast<const uint16_t *>(t_Q);
    a.out = t_O;
    a.n_qtiles = static_cast<int>(h->Tq / 16);
    a.r = h->r;
    cudaError_t e = kvq::launch_decode(a, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "decode launch");
    return ok();
}

kvq_status kvq_cache_state(const kvq_cache *h, int64_t *quantized_tokens, int32_t *residual_tokens) {
    if (!h) return fail(KVQ_ERR_INVALID_ARG, "cache is NULL");
    if (quantized_tokens) *quantized_tokens = h->Tq;
    if (residual_tokens) *residual_tokens = h->r;
    return ok();
}

kvq_status kvq_check_device(kvq_cache *h) {
    if (!h) return fail(KVQ_ERR_INVALID_ARG, "cache is NULL");
    return check_status_word(h->arrivals + static_cast<int64_t>(h->cfg.batch) * h->cfg.q_heads);
}

uint64_t kvq_kernel_launches(void) { return g_launches.load(); }

const char *kvq_last_error(void) { return g_last_error.c_str(); }

int32_t kvq_layout_version(void) { return 2; }

int32_t kvq_binary_arch(void) { return kvq::binary_version(); }

}  // extern "C"

// ---------------------------------------------------------------------------
// Paged, ragged cache.
//
// The handle wraps a kvq_cache for the geometry, the launch properties and the
// library-owned counters; its six cache buffers are the pool.  The host keeps
// every slot's length (-1: inactive) to decide flushes and plan splits; the
// kernels read the device copy, which the paged append kernel advances in
// stream order.
// ---------------------------------------------------------------------------
struct kvq_paged {
    kvq_cache base;
    int32_t page_tokens = 0, num_pages = 0, max_pages = 0;
    const int32_t *page_table = nullptr;
    int32_t *seq_len = nullptr;   // device [B], inside base.arrivals' allocation
    int64_t *len = nullptr;       // host [B]
};

namespace {

kvq_status validate_paged(const kvq_paged_config *c) {
    if (!c) return fail(KVQ_ERR_INVALID_ARG, "config is NULL");
    kvq_status st = validate(&c->geom);
    if (st != KVQ_OK) return st;
    const int P = c->page_tokens;
    if (P < 64 || P % 64 != 0 || P % c->geom.residual != 0)
        return fail(KVQ_ERR_INVALID_ARG, "page_tokens (%d) must be a positive multiple of 64 and of residual (%d)",
                    P, c->geom.residual);
    if (c->geom.capacity % P != 0)
        return fail(KVQ_ERR_INVALID_ARG, "capacity must be a multiple of page_tokens");
    if (c->num_pages < 1) return fail(KVQ_ERR_INVALID_ARG, "num_pages must be >= 1");
    if (static_cast<int64_t>(c->num_pages) * c->geom.kv_heads * (P / 16) > (int64_t{1} << 40))
        return fail(KVQ_ERR_UNSUPPORTED, "pool too large");
    if (static_cast<int64_t>(c->geom.batch) * (c->geom.capacity / P) > (int64_t{1} << 31) - 1)
        return fail(KVQ_ERR_UNSUPPORTED, "page table too large");
    return KVQ_OK;
}

kvq::DecodeArgs paged_decode_args(const kvq_paged *h) {
    kvq::DecodeArgs a = decode_args(&h->base);
    a.cap = h->page_tokens;
    a.page_table = h->page_table;
    a.seq_len = h->seq_len;
    a.page_tiles = h->page_tokens / 16;
    a.max_pages = h->max_pages;
    a.num_pages = h->num_pages;
    a.n_qtiles = 0;
    a.r = 0;
    return a;
}

kvq::QuantizeArgs paged_quantize_args(const kvq_paged *h) {
    kvq::QuantizeArgs q = quantize_args(&h->base);
    q.cap = h->page_tokens;
    q.page_table = h->page_table;
    q.max_pages = h->max_pages;
    q.num_pages = h->num_pages;
    q.Hkv = h->base.cfg.kv_heads;
    q.status = h->base.arrivals + static_cast<int64_t>(h->base.cfg.batch) * h->base.cfg.q_heads;
    return q;
}

void paged_plan(const kvq_paged *h, int *n_qsplits, int *tiles_per_split, int *S) {
    const kvq_config &c = h->base.cfg;
    // lengths of the active slots (tiles per slot) and the most residual rows
    std::vector<int64_t> tiles(static_cast<size_t>(c.batch));
    int32_t max_r = 0;
    for (int b = 0; b < c.batch; ++b) {
        const int64_t len = h->len[b] > 0 ? h->len[b] : 0;
        tiles[b] = (len / c.residual) * c.residual / 16;
        const int32_t r = static_cast<int32_t>(len % c.residual);
        max_r = r > max_r ? r : max_r;
    }
    const PlanInput in{tiles.data(), c.batch, 1, max_r};
    plan_splits_for(&h->base, in, n_qsplits, tiles_per_split, S);
}

kvq_status check_status_word(unsigned int *word) {
    unsigned int v = 0;
    cudaError_t e = cudaMemcpy(&v, word, sizeof v, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "reading the status word");
    if (v == 0) return ok();
    e = cudaMemset(word, 0, sizeof v);
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "clearing the status word");
    std::string why;
    if (v & 1u) why += " a decode kernel gave up waiting for a copy into shared memory;";
    if (v & 2u) why += " a kernel met a page-table entry outside the pool;";
    if (v & 4u) why += " a quantizer met a scale outside the range the decode kernels serve;";
    if (v & 8u) why += " a kernel met a list index outside its buffer (bounds-check build);";
    return fail(KVQ_ERR_DEVICE_CHECK, "device check (status 0x%x):%s outputs since the last check are "
                                      "unreliable", v, why.c_str());
}

}  // namespace

extern "C" {

kvq_status kvq_paged_get_sizes(const kvq_paged_config *cfg, kvq_paged_sizes *out) {
    if (!out) return fail(KVQ_ERR_INVALID_ARG, "out is NULL");
    kvq_status st = validate_paged(cfg);
    if (st != KVQ_OK) return st;
    const kvq_config &g = cfg->geom;
    const int64_t slices = static_cast<int64_t>(cfg->num_pages) * g.kv_heads;
    const int64_t P = cfg->page_tokens, d = g.head_dim;
    std::memset(out, 0, sizeof *out);
    out->k_codes = out->v_codes = static_cast<size_t>(slices * P * d * g.bits / 8);
    out->k_scales = static_cast<size_t>(slices * (P / g.group_k) * d * 4);
    out->k_zeros = g.symmetric ? 0 : static_cast<size_t>(slices * (P / g.group_k) * d * 2);
    out->v_scales = static_cast<size_t>(slices * P * (d / g.group_v) * 4);
    out->v_zeros = g.symmetric ? 0 : static_cast<size_t>(slices * P * (d / g.group_v) * 2);
    const int64_t BH = static_cast<int64_t>(g.batch) * g.kv_heads;
    out->k_residual = out->v_residual = static_cast<size_t>(BH * g.residual * d * 2);
    out->page_table = static_cast<size_t>(static_cast<int64_t>(g.batch) * (g.capacity / P) * 4);
    const int64_t units = static_cast<int64_t>(g.batch) * g.q_heads;
    out->workspace = static_cast<size_t>(units * max_splits(&g) * (d + 2) * 4);
    out->state = counter_bytes(&g) + (static_cast<size_t>(g.batch) * 4 + 15) / 16 * 16;
    return ok();
}

kvq_status kvq_paged_create(const kvq_paged_config *cfg, const kvq_buffers *bufs, const int32_t *page_table,
                            kvq_paged **out) {
    if (!out) return fail(KVQ_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    kvq_status st = validate_paged(cfg);
    if (st != KVQ_OK) return st;
    if (!bufs) return fail(KVQ_ERR_INVALID_ARG, "buffers are NULL");
    if (!page_table || !aligned16(page_table))
        return fail(KVQ_ERR_INVALID_ARG, "page_table must be non-NULL and 16-byte aligned");
    const void *need[] = {bufs->k_codes, bufs->k_scales, bufs->v_codes, bufs->v_scales,
                          bufs->k_residual, bufs->v_residual, bufs->state};
    for (const void *p : need)
        if (!p || !aligned16(p))
            return fail(KVQ_ERR_INVALID_ARG, "cache buffers and the state buffer must be non-NULL and "
                                             "16-byte aligned");
    const kvq_config &g = cfg->geom;
    if (!g.symmetric && (!bufs->k_zeros || !bufs->v_zeros || !aligned16(bufs->k_zeros) ||
                         !aligned16(bufs->v_zeros)))
        return fail(KVQ_ERR_INVALID_ARG, "asymmetric caches need 16-byte aligned zero buffers");
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "querying the current device");
    kvq_paged *h = new (std::nothrow) kvq_paged();
    int64_t *len = new (std::nothrow) int64_t[g.batch];
    if (!h || !len) {
        delete h;
        delete[] len;
        return fail(KVQ_ERR_INVALID_ARG, "out of host memory");
    }
    for (int b = 0; b < g.batch; ++b) len[b] = -1;
    h->len = len;
    h->base.cfg = g;
    h->base.buf = *bufs;
    if (g.symmetric) {
        h->base.buf.k_zeros = nullptr;
        h->base.buf.v_zeros = nullptr;
    }
    h->page_tokens = cfg->page_tokens;
    h->num_pages = cfg->num_pages;
    h->max_pages = static_cast<int32_t>(g.capacity / cfg->page_tokens);
    h->page_table = page_table;
    h->base.num_sms = sms > 0 ? sms : 148;
    h->base.path = kvq::decode_path(g.q_heads, g.kv_heads, g.group_k, false);
    // the caller's state buffer: counters [B * Hq] and the status word (zeroed), then the
    // slots' lengths [B] (all -1: inactive)
    h->base.arrivals = static_cast<unsigned int *>(bufs->state);
    const size_t cb = counter_bytes(&g);
    e = cudaMemset(h->base.arrivals, 0, cb);
    if (e == cudaSuccess)
        e = cudaMemset(static_cast<unsigned char *>(bufs->state) + cb, 0xff, g.batch * sizeof(unsigned int));
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) {
        delete[] h->len;
        delete h;
        return cuda_fail(e, "initialising the paged cache's state buffer");
    }
    h->seq_len = reinterpret_cast<int32_t *>(static_cast<unsigned char *>(bufs->state) + cb);
    h->base.ctas_per_sm = kvq::decode_ctas_per_sm(paged_decode_args(h));
    *out = h;
    return ok();
}

void kvq_paged_destroy(kvq_paged *h) {
    if (!h) return;
    delete[] h->len;
    delete h;
}

kvq_status kvq_paged_prefill(kvq_paged *h, int32_t seq, const void *X_K, const void *X_V, int64_t T,
                             void *stream) {
    if (!h) return fail(KVQ_ERR_INVALID_ARG, "cache is NULL");
    const kvq_config &c = h->base.cfg;
    if (seq < 0 || seq >= c.batch) return fail(KVQ_ERR_INVALID_ARG, "seq must be in 0..%d", c.batch - 1);
    if (T < 0) return fail(KVQ_ERR_INVALID_ARG, "T must be >= 0");
    if (h->len[seq] >= 0) return fail(KVQ_ERR_STATE, "slot %d is active; release it first", seq);
    if (T > 0 && (!X_K || !X_V || !aligned16(X_K) || !aligned16(X_V)))
        return fail(KVQ_ERR_INVALID_ARG, "X_K and X_V must be non-NULL and 16-byte aligned");
    const int64_t Tq = (T / c.residual) * c.residual;
    if (Tq > c.capacity)
        return fail(KVQ_ERR_CAPACITY, "prefill of %lld tokens exceeds capacity %lld",
                    static_cast<long long>(Tq), static_cast<long long>(c.capacity));
    if (T > 0x7fffffffLL) return fail(KVQ_ERR_UNSUPPORTED, "T must be < 2^31");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    kvq::QuantizeArgs q = paged_quantize_args(h);
    q.xk = static_cast<const uint16_t *>(X_K);
    q.xv = static_cast<const uint16_t *>(X_V);
    q.in_bh_stride = T * c.head_dim;
    q.in_tok0 = 0;
    q.n_groups = Tq / c.group_k;
    q.out_tok0 = 0;
    q.BH = c.kv_heads;
    q.seq0 = seq;
    q.seq_len = nullptr;
    cudaError_t e = kvq::launch_quantize(q, s);
    if (e != cudaSuccess) return cuda_fail(e, "paged prefill quantize launch");
    e = kvq::launch_paged_residual(static_cast<const uint16_t *>(X_K), static_cast<const uint16_t *>(X_V), T, Tq,
                                   T - Tq, static_cast<uint16_t *>(h->base.buf.k_residual),
                                   static_cast<uint16_t *>(h->base.buf.v_residual), h->seq_len, seq,
                                   static_cast<int32_t>(T), c.kv_heads, c.residual, c.head_dim, s);
    if (e != cudaSuccess) return cuda_fail(e, "paged prefill residual launch");
    h->len[seq] = T;
    return ok();
}

kvq_status kvq_paged_append(kvq_paged *h, const void *t_K, const void *t_V, void *stream) {
    if (!h) return fail(KVQ_ERR_INVALID_ARG, "cache is NULL");
    if (!t_K || !t_V || !aligned16(t_K) || !aligned16(t_V))
        return fail(KVQ_ERR_INVALID_ARG, "t_K and t_V must be non-NULL and 16-byte aligned");
    const kvq_config &c = h->base.cfg;
    bool any_flush = false;
    for (int b = 0; b < c.batch; ++b) {
        if (h->len[b] < 0) continue;
        const int64_t n = h->len[b] + 1;
        if (n % c.residual == 0) {
            if (n > c.capacity)
                return fail(KVQ_ERR_CAPACITY, "flushing slot %d would exceed capacity %lld", b,
                            static_cast<long long>(c.capacity));
            any_flush = true;
        }
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = kvq::launch_paged_append(static_cast<const uint16_t *>(t_K), static_cast<const uint16_t *>(t_V),
                                             static_cast<uint16_t *>(h->base.buf.k_residual),
                                             static_cast<uint16_t *>(h->base.buf.v_residual), h->seq_len, c.batch,
                                             c.kv_heads, c.residual, c.head_dim, s);
    if (e != cudaSuccess) return cuda_fail(e, "paged append launch");
    if (any_flush) {
        kvq::QuantizeArgs q = paged_quantize_args(h);
        q.xk = static_cast<const uint16_t *>(h->base.buf.k_residual);
        q.xv = static_cast<const uint16_t *>(h->base.buf.v_residual);
        q.in_bh_stride = static_cast<int64_t>(c.residual) * c.head_dim;
        q.in_tok0 = 0;
        q.n_groups = c.residual / c.group_k;
        q.out_tok0 = 0;
        q.BH = static_cast<int64_t>(c.batch) * c.kv_heads;
        q.seq0 = 0;
        q.seq_len = h->seq_len;
        e = kvq::launch_quantize(q, s);
        if (e != cudaSuccess) return cuda_fail(e, "paged flush launch");
    }
    for (int b = 0; b < c.batch; ++b)
        if (h->len[b] >= 0) ++h->len[b];
    return ok();
}

kvq_status kvq_paged_decode_attention(kvq_paged *h, const void *t_Q, float *t_O, void *workspace,
                                      size_t workspace_bytes, void *stream) {
    if (!h) return fail(KVQ_ERR_INVALID_ARG, "cache is NULL");
    if (!t_Q || !t_O || !workspace || !aligned16(t_Q) || !aligned16(t_O) || !aligned16(workspace))
        return fail(KVQ_ERR_INVALID_ARG, "t_Q, t_O and workspace must be non-NULL and 16-byte aligned");
    const kvq_config &c = h->base.cfg;
    const int64_t units = static_cast<int64_t>(c.batch) * c.q_heads;
    const size_t need = static_cast<size_t>(units * max_splits(&c) * (c.head_dim + 2) * 4);
    if (workspace_bytes < need)
        return fail(KVQ_ERR_INVALID_ARG, "workspace needs %zu bytes, got %zu", need, workspace_bytes);
    kvq::DecodeArgs a = paged_decode_args(h);
    paged_plan(h, &a.n_qsplits, &a.tiles_per_split, &a.S);
    float *ws = static_cast<float *>(workspace);
    a.o_part = ws;
    a.m_part = ws + units * a.S * c.head_dim;
    a.l_part = a.m_part + units * a.S;
    a.q = static_cast<const uint16_t *>(t_Q);
    a.out = t_O;
    cudaError_t e = kvq::launch_decode(a, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "paged decode launch");
    return ok();
}

kvq_status kvq_paged_release(kvq_paged *h, int32_t seq, void *stream) {
    if (!h) return fail(KVQ_ERR_INVALID_ARG, "cache is NULL");
    const kvq_config &c = h->base.cfg;
    if (seq < 0 || seq >= c.batch) return fail(KVQ_ERR_INVALID_ARG, "seq must be in 0..%d", c.batch - 1);
    cudaError_t e = kvq::launch_paged_residual(nullptr, nullptr, 0, 0, 0, nullptr, nullptr, h->seq_len, seq, -1,
                                               c.kv_heads, c.residual, c.head_dim, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "paged release launch");
    h->len[seq] = -1;
    return ok();
}

kvq_status kvq_paged_seq_len(const kvq_paged *h, int32_t seq, int64_t *len) {
    if (!h || !len) return fail(KVQ_ERR_INVALID_ARG, "cache and len must be non-NULL");
    if (seq < 0 || seq >= h->base.cfg.batch)
        return fail(KVQ_ERR_INVALID_ARG, "seq must be in 0..%d", h->base.cfg.batch - 1);
    *len = h->len[seq];
    return ok();
}

int32_t kvq_paged_decode_splits(const kvq_paged *h) {
    if (!h) return 0;
    int nq, per, S;
    paged_plan(h, &nq, &per, &S);
    return S;
}

kvq_status kvq_paged_check_device(kvq_paged *h) {
    if (!h) return fail(KVQ_ERR_INVALID_ARG, "cache is NULL");
    return check_status_word(h->base.arrivals + static_cast<int64_t>(h->base.cfg.batch) * h->base.cfg.q_heads);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// LogQuant retention ("Resumo Técnico: LogQuant", section 2, Estratégia de
// Filtragem Baseada em Logaritmos; section 4): a cache whose full-precision
// store holds up to 3W tokens and, whenever it fills, quantizes every other one
// of its 2W oldest tokens as a block of W.  It is a kvq_cache whose residual
// buffer is that store (residual = 3W); kvq_append, kvq_append_decode_attention,
// the decode calls and kvq_cache_state (r = tokens in the store) serve it as is.
// ---------------------------------------------------------------------------
namespace {

kvq_config lq_geometry(const kvq_config *cfg, int32_t W) {
    kvq_config g = *cfg;
    const int64_t R = 3 * static_cast<int64_t>(W);
    g.residual = static_cast<int32_t>(R);
    g.capacity = (cfg->capacity + R - 1) / R * R;
    return g;
}

kvq_status validate_lq(const kvq_config *cfg, int32_t W) {
    if (!cfg) return fail(KVQ_ERR_INVALID_ARG, "config is NULL");
    if (W < 16 || W > 4096 || cfg->group_k < 1 || W % cfg->group_k != 0)
        return fail(KVQ_ERR_INVALID_ARG, "window (%d) must be a multiple of group_k in 16..4096", W);
    if (cfg->capacity < W || cfg->capacity % W != 0)
        return fail(KVQ_ERR_INVALID_ARG, "capacity must be a positive multiple of the window");
    const kvq_config g = lq_geometry(cfg, W);
    return validate(&g);
}

kvq_status lq_prefill(kvq_cache *h, const void *X_K, const void *X_V, int64_t T, void *stream) {
    const kvq_config &c = h->cfg;
    const int64_t W = h->lq_window;
    if (T > 0x7fffffffLL) return fail(KVQ_ERR_UNSUPPORTED, "T must be < 2^31");
    // the tokens enter one by one: the blocks that leave (in the order they leave) and the
    // positions that stay
    std::vector<int32_t> lists;
    std::vector<int64_t> F;
    F.reserve(3 * W);
    for (int64_t t = 0; t < T; ++t) {
        F.push_back(t);
        if (static_cast<int64_t>(F.size()) == 3 * W) {
            for (int64_t i = 0; i < W; ++i) lists.push_back(static_cast<int32_t>(F[2 * i + 1]));
            for (int64_t i = 0; i < W; ++i) F[i] = F[2 * i];
            for (int64_t j = 0; j < W; ++j) F[W + j] = F[2 * W + j];
            F.resize(2 * W);
        }
    }
    const int64_t Tq = static_cast<int64_t>(lists.size());
    if (Tq > c.capacity)
        return fail(KVQ_ERR_CAPACITY, "prefill of %lld tokens quantizes %lld, beyond capacity %lld",
                    static_cast<long long>(T), static_cast<long long>(Tq), static_cast<long long>(c.capacity));
    for (int64_t p : F) lists.push_back(static_cast<int32_t>(p));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t *dev_lists = h->lq_rows + W;
    // from pageable memory: returns once the list is staged, so the vector may go
    cudaError_t e = cudaMemcpyAsync(dev_lists, lists.data(), lists.size() * sizeof(int32_t),
                                    cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e, "uploading the prefill's row lists");
    kvq::QuantizeArgs q = quantize_args(h);
    q.xk = static_cast<const uint16_t *>(X_K);
    q.xv = static_cast<const uint16_t *>(X_V);
    q.in_bh_stride = T * c.head_dim;
    q.in_rows = dev_lists;
    q.in_rows_limit = T;
    q.n_groups = Tq / c.group_k;
    q.out_tok0 = 0;
    e = kvq::launch_quantize(q, s);
    if (e != cudaSuccess) return cuda_fail(e, "LogQuant prefill quantize launch");
    const int64_t BH = static_cast<int64_t>(c.batch) * c.kv_heads;
    e = kvq::launch_gather_rows(static_cast<const uint16_t *>(X_K), static_cast<const uint16_t *>(X_V),
                                T * c.head_dim, T, dev_lists + Tq, static_cast<int>(F.size()),
                                static_cast<uint16_t *>(h->buf.k_residual), static_cast<uint16_t *>(h->buf.v_residual),
                                static_cast<int64_t>(c.residual) * c.head_dim, BH, c.head_dim, q.status, s);
    if (e != cudaSuccess) return cuda_fail(e, "LogQuant prefill store launch");
    h->Tq = Tq;
    h->r = static_cast<int32_t>(F.size());
    h->lq_F = F;
    h->lq_n = T;
    return ok();
}

}  // namespace

extern "C" {

kvq_status kvq_logquant_get_sizes(const kvq_config *cfg, int32_t window, kvq_sizes *out) {
    if (!out) return fail(KVQ_ERR_INVALID_ARG, "out is NULL");
    kvq_status st = validate_lq(cfg, window);
    if (st != KVQ_OK) return st;
    const kvq_config g = lq_geometry(cfg, window);
    st = kvq_get_sizes(&g, out);
    if (st == KVQ_OK) out->state += lq_list_entries(&g, window) * sizeof(int32_t);
    return st;
}

kvq_status kvq_logquant_create(const kvq_config *cfg, int32_t window, const kvq_buffers *bufs, kvq_cache **out) {
    if (!out) return fail(KVQ_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    kvq_status st = validate_lq(cfg, window);
    if (st != KVQ_OK) return st;
    const kvq_config g = lq_geometry(cfg, window);
    kvq_cache *h = nullptr;
    st = kvq_create(&g, bufs, &h);
    if (st != KVQ_OK) return st;
    h->lq_window = window;
    h->lq_F.reserve(3 * static_cast<size_t>(window));
    // in the state buffer after the counters: rows 1, 3, ..., 2W - 1, then room for a
    // prefill's lists (capacity + 3W entries)
    h->lq_rows = reinterpret_cast<int32_t *>(static_cast<unsigned char *>(bufs->state) + counter_bytes(&g));
    std::vector<int32_t> odd(static_cast<size_t>(window));
    for (int32_t i = 0; i < window; ++i) odd[i] = 2 * i + 1;
    cudaError_t e = cudaMemcpy(h->lq_rows, odd.data(), odd.size() * sizeof(int32_t), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) {
        kvq_destroy(h);
        return cuda_fail(e, "writing the LogQuant row list");
    }
    *out = h;
    return ok();
}

kvq_status kvq_logquant_retained(const kvq_cache *h, int64_t *positions, int32_t capacity, int32_t *count) {
    if (!h || !count) return fail(KVQ_ERR_INVALID_ARG, "cache and count must be non-NULL");
    if (!h->lq_window) return fail(KVQ_ERR_STATE, "not a LogQuant cache");
    const int32_t n = static_cast<int32_t>(h->lq_F.size());
    *count = n;
    if (positions) {
        if (capacity < n) return fail(KVQ_ERR_INVALID_ARG, "positions holds %d entries, %d needed", capacity, n);
        for (int32_t i = 0; i < n; ++i) positions[i] = h->lq_F[i];
    }
    return ok();
}

}  // extern "C"

extern "C" {

kvq_status kvq_set_key_outliers(kvq_cache *h, int32_t n_out, uint32_t *k_outliers, size_t bytes) {
    if (!h) return fail(KVQ_ERR_INVALID_ARG, "cache is NULL");
    if (h->Tq != 0 || h->r != 0) return fail(KVQ_ERR_STATE, "key outliers are set on an empty cache");
    if (n_out < 0 || n_out > 2) return fail(KVQ_ERR_INVALID_ARG, "n_out must be 0, 1 or 2");
    const kvq_config &c = h->cfg;
    if (n_out == 0) {
        h->k_out = nullptr;
        h->n_out = 0;
        h->path = kvq::decode_path(c.q_heads, c.kv_heads, c.group_k);
        h->ctas_per_sm = kvq::decode_ctas_per_sm(decode_args(h));
        return ok();
    }
    if (kvq::decode_path(c.q_heads, c.kv_heads, c.group_k, false) != kvq::kPathTc)
        return fail(KVQ_ERR_UNSUPPORTED, "dense-and-sparse keys need 1, 2 or 4 query heads per kv head "
                                         "and key groups of >= 32 tokens");
    const size_t need = static_cast<size_t>(c.batch) * c.kv_heads * static_cast<size_t>(c.capacity) * n_out * 4;
    if (!k_outliers || !aligned16(k_outliers))
        return fail(KVQ_ERR_INVALID_ARG, "k_outliers must be non-NULL and 16-byte aligned");
    if (bytes < need) return fail(KVQ_ERR_INVALID_ARG, "k_outliers needs %zu bytes, got %zu", need, bytes);
    h->k_out = k_outliers;
    h->n_out = n_out;
    h->path = kvq::kPathTc;   // the integer-MMA kernel's dense-and-sparse instances
    h->ctas_per_sm = kvq::decode_ctas_per_sm(decode_args(h));
    return ok();
}

}  // extern "C"

// ---------------------------------------------------------------------------
// The split plan without a device: the same planner the decode calls use, for
// capacity planning and for tests of its invariants on the host.
// ---------------------------------------------------------------------------
extern "C" {

kvq_status kvq_plan_decode(const kvq_config *cfg, const int64_t *lengths, int32_t num_sms, int32_t ctas_per_sm,
                           int32_t *n_qsplits, int32_t *tiles_per_split, int32_t *splits) {
    kvq_status st = validate(cfg);
    if (st != KVQ_OK) return st;
    if (!lengths || !n_qsplits || !tiles_per_split || !splits)
        return fail(KVQ_ERR_INVALID_ARG, "lengths and the outputs must be non-NULL");
    if (num_sms < 1 || ctas_per_sm < 1) return fail(KVQ_ERR_INVALID_ARG, "num_sms and ctas_per_sm must be >= 1");
    kvq_cache h;
    h.cfg = *cfg;
    h.path = kvq::decode_path(cfg->q_heads, cfg->kv_heads, cfg->group_k);
    h.num_sms = num_sms;
    h.ctas_per_sm = ctas_per_sm;
    std::vector<int64_t> tiles(static_cast<size_t>(cfg->batch));
    int32_t max_r = 0;
    for (int b = 0; b < cfg->batch; ++b) {
        const int64_t len = lengths[b] > 0 ? lengths[b] : 0;
        const int64_t tq = (len / cfg->residual) * cfg->residual;
        if (tq > cfg->capacity)
            return fail(KVQ_ERR_CAPACITY, "sequence %d: %lld quantized tokens exceed capacity %lld", b,
                        static_cast<long long>(tq), static_cast<long long>(cfg->capacity));
        tiles[static_cast<size_t>(b)] = tq / 16;
        const int32_t r = static_cast<int32_t>(len - tq);
        max_r = r > max_r ? r : max_r;
    }
    const PlanInput in{tiles.data(), cfg->batch, 1, max_r};
    int nq = 0, per = 0, S = 0;
    plan_splits_for(&h, in, &nq, &per, &S);
    *n_qsplits = nq;
    *tiles_per_split = per;
    *splits = S;
    return ok();
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Bounds-check builds only (libkvq_check.so, include/kvq_check.h): entry points that make
// the kernels' checks fire, for tests.
// ---------------------------------------------------------------------------
#ifdef KVQ_CHECK
#include "../../include/kvq_check.h"

extern "C" {

kvq_status kvq_debug_set_stall(kvq_cache *h, int32_t polls) {
    if (!h) return fail(KVQ_ERR_INVALID_ARG, "cache is NULL");
    if (polls < 0 || polls > 4096) return fail(KVQ_ERR_INVALID_ARG, "polls must be in 0..4096");
    h->stall_polls = polls;
    return ok();
}

kvq_status kvq_debug_gather_rows(kvq_cache *h, const void *src, int64_t src_rows, const int32_t *idx, int32_t n,
                                 void *dst, void *stream) {
    if (!h || !src || !idx || !dst || !aligned16(src) || !aligned16(dst) || n < 0 || src_rows < 1)
        return fail(KVQ_ERR_INVALID_ARG, "bad arguments");
    const kvq_config &c = h->cfg;
    unsigned int *status = h->arrivals + static_cast<int64_t>(c.batch) * c.q_heads;
    const cudaError_t e = kvq::launch_gather_rows(static_cast<const uint16_t *>(src), static_cast<const uint16_t *>(src),
                                                  src_rows * c.head_dim, src_rows, idx, n, static_cast<uint16_t *>(dst),
                                                  static_cast<uint16_t *>(dst), static_cast<int64_t>(n) * c.head_dim, 1,
                                                  c.head_dim, status, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "gather launch");
    return ok();
}

}  // extern "C"
#endif  // KVQ_CHECK
