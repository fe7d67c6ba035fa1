// decode_kernels.cuh -- the decode-attention kernels and their launch dispatch, shared by
// decode.cu (contiguous caches), decode_paged.cu (paged, ragged caches) and
// decode_sparse.cu (dense-and-sparse keys).
//
// Two kernels: decode_split_kernel (CUDA cores, described first, below) and
// decode_tc_kernel (tensor cores, described above its definition).  Both compute,
// for every (batch, query head), one decode step of
//   A = softmax(q [deq(K_g); K_r]^T / sqrt(d)),   t_O = A [deq(V_g); V_r]
// ("LLM系列：KVCache量化1 KIVI ...", section 1: A = Concat(A_g, A_r), t_O = A X_V;
//  the 1/sqrt(d_k) of "KV Cache的Int4量化…" section 3), with deq(x) = (code - z) s.
//
// Split-K (flash-decoding): the quantized 16-token tiles are divided into
// contiguous splits and the residual rows, cut into 16-row tiles, form splits
// of their own (one here; up to 16 in the tensor-core kernel), so they run beside
// the others instead of lengthening one of them; a CTA owns one (batch, query
// head, split) and each of its four warps a contiguous share of the split's tiles,
// streamed through a per-warp cp.async ring of shared-memory stages.  Token order does not change the result
// (A . V = A_P . V_P, "Resumo Técnico: LogQuant", section 4), which is what
// allows the splits and the residual to be folded into one online-softmax pass.
// Each CTA merges its warps into an unnormalised partial (o, m, l); the last
// CTA of each (batch, head) to finish merges the S partials (finish_cta).
//
// Lane = 4*g8 + t4.  In a tile it holds, per 16-channel chunk j, the codes of
// rows g8 and g8+8 at columns 4*t4 .. 4*t4+3 (keys: rows = tokens, columns =
// channels; values: rows = channels, columns = tokens); (word >> n*slot) with
// the low n bits of each byte kept is four such codes, one per byte.
//   keys   : logit_t = sum_c q_c s_{g,c} (code - z_{g,c}) log2(e)/sqrt(d)
//            = 2^-e sum_c Q_c code_{t,c} - bias_g.  Once per key group the
//            multipliers q_c s_{g,c} log2(e)/sqrt(d) are rounded to 22-bit fixed
//            point Q_c = round(2^e q'_c) (e from the group's largest |q'|), split
//            into three byte digits, and the integer dot products run as
//            byte dot products (dp4a) with exact int32 accumulation;
//            bias_g = sum_c q'_c z_{g,c} in fp32.
//   values : o_c += sum_t p_t s_{t,gv} code_{t,c} - sum_t p_t s_{t,gv} z_{t,gv} in fp32:
//            (word & mask) | 0x4B000000 is the float 2^23 + code * 2^pos exactly
//            (one lop3); a packed fp32x2 add removes 2^23 and a packed fp32x2
//            FMA accumulates two codes, the 2^pos factors folded into the
//            multipliers and accumulators (exact powers of two).
#pragma once

#include <cfloat>
#include <cmath>
#include <cstdint>

#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr int kDecodeWarps = 4;
constexpr int kDecodeThreads = 32 * kDecodeWarps;
constexpr uint32_t kMagicBits = 0x4B000000u;   // 2^23
constexpr float kMagic = 8388608.0f;

__device__ __forceinline__ unsigned long long pk(float2 v) {
    unsigned long long r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(v.x), "f"(v.y));
    return r;
}
__device__ __forceinline__ float2 upk(unsigned long long r) {
    float2 v;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(v.x), "=f"(v.y) : "l"(r));
    return v;
}
// packed fp32x2 arithmetic (sm_100)
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
    unsigned long long d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(pk(a)), "l"(pk(b)), "l"(pk(c)));
    return upk(d);
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
    unsigned long long d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(pk(a)), "l"(pk(b)));
    return upk(d);
}
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
    unsigned long long d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(pk(a)), "l"(pk(b)));
    return upk(d);
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
    unsigned long long d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(pk(a)), "l"(pk(b)));
    return upk(d);
}

// (a & b) | c in one lop3.
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
    return r;
}

// byte dot products with int32 accumulation: bytes of a unsigned, of b unsigned / signed
__device__ __forceinline__ int dp4a_uu(uint32_t a, uint32_t b, int c) {
    int d;
    asm("dp4a.u32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
    int d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// 2^x (ex2.approx.ftz: relative error ~2^-22, 2^-inf = 0)
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Exact int -> float for |x| < 2^22: 1.5 * 2^23 + x as a bit pattern, minus 1.5 * 2^23.
__device__ __forceinline__ float small_int_to_float(int x) {
    return __int_as_float(0x4B400000 + x) - 12582912.0f;
}
// round(x) for |x| < 2^22, exactly (round half to even), without the XU pipe
__device__ __forceinline__ int round_small(float x) {
    return __float_as_int(x + 12582912.0f) - 0x4B400000;
}

// The lane's W words of one stage array (chunk-major, see Stage).
template <int W>
__device__ __forceinline__ void load_stage_words(const uint32_t *base, int lane, uint32_t (&w)[W]) {
    if constexpr (W % 4 == 0) {
#pragma unroll
        for (int i = 0; i < W / 4; ++i) {
            const uint4 v = reinterpret_cast<const uint4 *>(base)[32 * i + lane];
            w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
        }
    } else {
        const uint2 v = reinterpret_cast<const uint2 *>(base)[lane];
        w[0] = v.x; w[1] = v.y;
    }
}

// cp.async (global -> shared, bypassing L1) and its group bookkeeping.
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
    const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem));
}
__device__ __forceinline__ void cp_async8(void *smem, const void *gmem) {
    const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(s), "l"(gmem));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;"); }
template <int PENDING>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(PENDING));
}

// Bulk (TMA) copies global -> shared completing on an mbarrier, and the barrier
// operations (no cluster multicast anywhere).
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_inval(uint64_t *bar) {
    asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// barrier initialisations visible to the async proxy
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// earlier generic-proxy accesses to shared memory ordered before later async-proxy ones
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
// bytes: a multiple of 16; both addresses 16-byte aligned
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}
// Hint: bring [src, src + bytes) into L2 (16-byte aligned, a multiple of 16 bytes; no
// completion to wait for).
__device__ __forceinline__ void bulk_prefetch_l2(const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}
// One poll; the thread may be suspended up to kPollSuspendNs waiting for the phase, so a
// waiting warp takes (almost) no issue slots from the working ones.
constexpr uint32_t kPollSuspendNs = 200000;
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "n"(kPollSuspendNs)
        : "memory");
    return ok != 0;
}
// Waits for the phase of `parity` to complete, giving up after kSpinLimit polls
// (at most about kSpinLimit * kPollSuspendNs, a few seconds); false when it gave up.
constexpr uint32_t kSpinLimit = 1u << 14;
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity) {
    for (uint32_t i = 0; i < kSpinLimit; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

// Shared-memory stage of one 16-token tile, owned by one warp:
//   [K codes][V codes], each as (W/4 chunks) x (32 lanes) x 16 bytes, chunk-major so
//   that a warp's 16-byte loads of one chunk hit 32 consecutive 16-byte slots
//   (W = 2: 32 lanes x 8 bytes)
//   [value scales 16 x NGV f32][value zeros 16 x NGV i16]
//   [key scales D f32][key zeros D i16]   (filled only when the tile opens a key group)
template <int N, int D, int GV>
struct Stage {
    static constexpr int W = D * N / 64;
    static constexpr int NGV = D / GV;
    static constexpr int kCodes = 32 * W * 4;          // bytes of one code array
    static constexpr int kVs = 2 * kCodes;
    static constexpr int kVz = kVs + 16 * NGV * 4;
    static constexpr int kKs = kVz + 16 * NGV * 2;
    static constexpr int kKz = kKs + D * 4;
    static constexpr int kBytes = kKz + D * 2;
    static_assert(kVz % 16 == 0 && kKs % 16 == 0 && kKz % 16 == 0 && kBytes % 16 == 0, "align");
};

constexpr int kStages = 4;

// Quantized 16-token tiles and residual rows of sequence b: the call's uniform counts
// for a contiguous cache, the sequence's own count for a paged one (Tq = floor(len / R) R,
// r = len mod R; an inactive slot, len < 0, is empty).
template <bool PAGED>
__device__ __forceinline__ void seq_extent(const DecodeArgs &a, int b, int &n_qtiles, int &r) {
    if constexpr (PAGED) {
        const int len = a.seq_len[b];
        n_qtiles = len > 0 ? (len / a.R) * (a.R / 16) : 0;
        r = len > 0 ? len % a.R : 0;
    } else {
        n_qtiles = a.n_qtiles;
        r = a.r;
    }
}

// Paged cache: index of the first tile of page pi of sequence b, kv head hk, counted as if
// the sequence's tiles were contiguous (global tile of sequence tile t = result + t for t
// in that page).  A page number outside the pool raises status bit 2 and reads page 0
// instead, so that a bad page table cannot make a kernel read out of bounds.
__device__ __forceinline__ int64_t page_tile_base(const DecodeArgs &a, int page, int hk, int pi) {
    if (page < 0 || page >= a.num_pages) {
        atomicOr(a.status, 2u);
        page = 0;
    }
    return (static_cast<int64_t>(page) * a.Hkv + hk - pi) * a.page_tiles;
}

// A warp's window on 32 consecutive entries of one sequence's page table, one per lane:
// lookups inside the window are a shuffle, the rest reload it (all lanes call it).
struct PageWindow {
    int base = -64, reg = 0;
    __device__ __forceinline__ int page(const DecodeArgs &a, int b, int pi, int lane) {
        if (pi < base || pi >= base + 32) {
            base = pi;
            const int j = pi + lane;
            reg = j < a.max_pages ? __ldg(a.page_table + static_cast<int64_t>(b) * a.max_pages + j) : 0;
        }
        return __shfl_sync(0xffffffffu, reg, pi - base);
    }
};

// Floats of shared scratch finish_cta needs after the per-warp outputs (wts): the split
// weights HG (S + 1), S <= kMaxDecodeSplits, padded to 4, and the [P][C] float4 sums of
// the merge.
template <int HG, int D>
__host__ __device__ constexpr int finish_scratch_floats() {
    return (HG * (kMaxDecodeSplits + 1) + 3) / 4 * 4 + 4 * kDecodeThreads;
}

// End of every decode CTA.  o_w [warp][HG][D] and ml_w [warp][HG] = (m, l) are
// the per-warp partials of the CTA's HG query heads (unnormalised, log2
// domain; m = -inf for a warp without tokens).  They are merged into the CTA's
// partial of split `sigma`.  With one split that is the answer and is written
// out.  Otherwise the partial goes to the workspace, and the CTA that brings
// the unit's arrival counter to S merges all S partials with a log-sum-exp
// reduction, writes t_O and puts the counter back to zero for the next call
// (flash-decoding's reduction, done by the last split instead of a second
// kernel).  wts is shared scratch of HG * (S + 1) floats that may alias o_w.
template <int HG, int D>
__device__ __forceinline__ void finish_cta(const DecodeArgs &a, const float *o_w,
                                           const float (*ml_w)[HG][2], int64_t unit, int64_t bq0,
                                           int sigma, int *last, float *wts) {
    for (int i = threadIdx.x; i < HG * D; i += kDecodeThreads) {
        const int hh = i / D, c = i % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kDecodeWarps; ++w) M = fmaxf(M, ml_w[w][hh][0]);
        float o = 0.f, l = 0.f;
#pragma unroll
        for (int w = 0; w < kDecodeWarps; ++w) {
            if (ml_w[w][hh][0] == -INFINITY) continue;
            const float f = exp2f(ml_w[w][hh][0] - M);
            o = fmaf(o_w[(w * HG + hh) * D + c], f, o);
            l = fmaf(ml_w[w][hh][1], f, l);
        }
        const int64_t bq = bq0 + hh;
        if (a.S == 1) {
            if (a.po) {   // the cache's partial (token-split decode)
                a.po[bq * D + c] = o;
                if (c == 0) {
                    a.pm[bq] = M;
                    a.pl[bq] = l;
                }
            } else {
                a.out[bq * D + c] = l > 0.f ? o / l : 0.f;   // an empty sequence gives 0
            }
            continue;
        }
        a.o_part[(bq * a.S + sigma) * D + c] = o;
        if (c == 0) {
            a.m_part[bq * a.S + sigma] = M;
            a.l_part[bq * a.S + sigma] = l;
        }
    }
    if (a.S == 1) return;
    __threadfence();   // this CTA's partial is visible before its arrival is counted
    __syncthreads();
    if (threadIdx.x == 0)
        *last = atomicAdd(a.arrivals + unit, 1u) == static_cast<unsigned>(a.S - 1);
    __syncthreads();
    if (!*last) return;
    __threadfence();
    // split weights 2^(m_s - M) and 1 / sum_s l_s 2^(m_s - M), one warp per head
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int hh = warp; hh < HG; hh += kDecodeWarps) {
        const int64_t row = (bq0 + hh) * a.S;
        float M = -INFINITY;
        for (int s = lane; s < a.S; s += 32) M = fmaxf(M, __ldcg(a.m_part + row + s));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        float L = 0.f;
        for (int s = lane; s < a.S; s += 32) {
            const float ms = __ldcg(a.m_part + row + s);
            const float f = ms == -INFINITY ? 0.f : exp2f(ms - M);
            wts[hh * a.S + s] = f;
            L = fmaf(__ldcg(a.l_part + row + s), f, L);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
        if (lane == 0) wts[HG * a.S + hh] = L;
    }
    __syncthreads();
    // weighted sum of the S partials: thread t takes 4 channels (float4 column t mod C of the
    // HG x D outputs) and every P-th split from t / C, with 16 loads in flight; the P partial
    // sums of a column are then added through shared memory (finish_scratch_floats<HG, D>)
    constexpr int C = HG * D / 4;                       // float4 columns
    constexpr int P = kDecodeThreads / C;
    static_assert(kDecodeThreads % C == 0, "columns");
    float4 *red = reinterpret_cast<float4 *>(wts + ((HG * (a.S + 1) + 3) & ~3));   // [P][C]
    {
        const int col = threadIdx.x % C, part = threadIdx.x / C;
        const int hh = (4 * col) / D, c = (4 * col) % D;
        const float4 *op = reinterpret_cast<const float4 *>(a.o_part + (bq0 + hh) * a.S * D + c);
        const float *wp = wts + hh * a.S;
        float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 16
        for (int s = part; s < a.S; s += P) {
            const float4 v = __ldcg(op + static_cast<int64_t>(s) * (D / 4));
            const float wgt = wp[s];
            o.x = fmaf(v.x, wgt, o.x); o.y = fmaf(v.y, wgt, o.y);
            o.z = fmaf(v.z, wgt, o.z); o.w = fmaf(v.w, wgt, o.w);
        }
        red[part * C + col] = o;
    }
    __syncthreads();
    for (int col = threadIdx.x; col < C; col += kDecodeThreads) {
        float4 o = red[col];
#pragma unroll
        for (int q = 1; q < P; ++q) {
            const float4 v = red[q * C + col];
            o.x += v.x; o.y += v.y; o.z += v.z; o.w += v.w;
        }
        const int hh = (4 * col) / D, c = (4 * col) % D;
        if (a.po) {   // the cache's partial (token-split decode): o and l relative to M
            *reinterpret_cast<float4 *>(a.po + (bq0 + hh) * D + c) = o;
            if (c == 0) {
                float M = -INFINITY;
                for (int s = 0; s < a.S; ++s) M = fmaxf(M, __ldcg(a.m_part + (bq0 + hh) * a.S + s));
                a.pm[bq0 + hh] = M;
                a.pl[bq0 + hh] = wts[HG * a.S + hh];
            }
        } else {
            const float L = wts[HG * a.S + hh];
            *reinterpret_cast<float4 *>(a.out + (bq0 + hh) * D + c) =
                L > 0.f ? make_float4(o.x / L, o.y / L, o.z / L, o.w / L)    // an empty sequence gives 0
                        : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    if (threadIdx.x == 0) a.arrivals[unit] = 0u;
}

template <int N, int D, int GV, bool PAGED>
__global__ void __launch_bounds__(kDecodeThreads, 4) decode_split_kernel(const DecodeArgs a) {
    constexpr int W = D * N / 64;     // words per lane per tile
    constexpr int TW = D * N / 2;     // words per tile
    constexpr int NJ = D / 16;        // 16-channel chunks
    constexpr int BPW = 4 / N;        // chunks per word
    constexpr int SLOTS = 2 * BPW;    // byte groups per word
    constexpr int NGV = D / GV;       // value groups per token
    constexpr uint32_t BYTE_MASK = ((1u << N) - 1u) * 0x01010101u;
    using St = Stage<N, D, GV>;
    static_assert(finish_scratch_floats<1, D>() * 4 <= kDecodeWarps * kStages * St::kBytes, "merge scratch");

    __shared__ float q_s[D];
    __shared__ float o_s[kDecodeWarps][D];
    __shared__ float ml_s[kDecodeWarps][2];
    __shared__ int last_s;
    extern __shared__ __align__(128) unsigned char stage_mem[];

    const int qi = blockIdx.x, b = blockIdx.y, sigma = blockIdx.z;
    const int g = a.Hq / a.Hkv;
    const int64_t bh = static_cast<int64_t>(b) * a.Hkv + qi / g;
    const int64_t bq = static_cast<int64_t>(b) * a.Hq + qi;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g8 = lane >> 2, t4 = lane & 3;
    unsigned char *wmem = stage_mem + static_cast<size_t>(warp) * kStages * St::kBytes;
    const uint32_t magic = kMagicBits;

    for (int c = threadIdx.x; c < D; c += kDecodeThreads)
        q_s[c] = widen(a.q[bq * D + c], a.bf16) * a.qscale;
    __syncthreads();

    // this warp's contiguous share of the split's tiles: splits 0 .. n_qsplits-1 cut the
    // quantized tiles, the last split (when r > 0) owns the residual tiles alone
    int n_qt, r_rows;
    seq_extent<PAGED>(a, b, n_qt, r_rows);
    const int total_tiles = n_qt + (r_rows + 15) / 16;
    const int t_begin = sigma < a.n_qsplits ? min(n_qt, sigma * a.tiles_per_split) : n_qt;
    const int t_end = sigma < a.n_qsplits ? min(n_qt, t_begin + a.tiles_per_split) : total_tiles;
    const int per_w = (t_end - t_begin + kDecodeWarps - 1) / kDecodeWarps;
    const int wb = t_begin + warp * per_w;
    const int we = min(t_end, wb + per_w);
    const int qe = min(we, n_qt);
    const int zsym = 1 << (N - 1);
    const int gmask = (1 << a.gshift) - 1;   // tiles per key group - 1

    // producer: stage the tile's lane segments, value meta and (at a group start) key meta
    auto issue = [&](int ti) {
        if (ti >= qe) return;
        unsigned char *st = wmem + ((ti - wb) % kStages) * St::kBytes;
        // global tile of sequence tile ti (paged: through the page table)
        int64_t gt = bh * (a.cap / 16) + ti;
        if constexpr (PAGED) {
            const int pi = ti / a.page_tiles;
            gt = page_tile_base(a, __ldg(a.page_table + static_cast<int64_t>(b) * a.max_pages + pi), qi / g, pi) + ti;
        }
        const uint32_t *ksrc = a.kc + gt * TW + lane * W;
        const uint32_t *vsrc = a.vc + gt * TW + lane * W;
        if constexpr (W % 4 == 0) {
            uint32_t *kdst = reinterpret_cast<uint32_t *>(st) + 4 * lane;
            uint32_t *vdst = reinterpret_cast<uint32_t *>(st + St::kCodes) + 4 * lane;
#pragma unroll
            for (int i = 0; i < W / 4; ++i) {
                cp_async16(kdst + 128 * i, ksrc + 4 * i);
                cp_async16(vdst + 128 * i, vsrc + 4 * i);
            }
        } else {
            static_assert(W == 2, "lane segment of 8 bytes");
            cp_async8(reinterpret_cast<uint32_t *>(st) + lane * W, ksrc);
            cp_async8(reinterpret_cast<uint32_t *>(st + St::kCodes) + lane * W, vsrc);
        }
        const int64_t tok0 = gt * 16;
        for (int c = lane; c < NGV * 4; c += 32)
            cp_async16(st + St::kVs + 16 * c, a.vs + tok0 * NGV + 4 * c);
        if (!a.sym)
            for (int c = lane; c < NGV * 2; c += 32)
                cp_async16(st + St::kVz + 16 * c, a.vz + tok0 * NGV + 8 * c);
        if (ti == wb || (ti & gmask) == 0) {
            const int64_t gofs = (gt >> a.gshift) * D;
            for (int c = lane; c < D / 4; c += 32) cp_async16(st + St::kKs + 16 * c, a.ks + gofs + 4 * c);
            if (!a.sym)
                for (int c = lane; c < D / 8; c += 32) cp_async16(st + St::kKz + 16 * c, a.kz + gofs + 8 * c);
        }
    };

    float m = -INFINITY, lsum = 0.0f;
    float2 acc[NJ][2];       // value accumulators, channel 16j + g8 + 8h, x: tokens 4t4+{0,1}, y: +{2,3}
    float zsum[NGV];
#pragma unroll
    for (int j = 0; j < NJ; ++j) acc[j][0] = acc[j][1] = make_float2(0.f, 0.f);
#pragma unroll
    for (int v = 0; v < NGV; ++v) zsum[v] = 0.f;
    uint32_t kdig[NJ][3];    // key multiplier digits, channels 16j + 4t4 + {0..3}
    float kbias = 0.f, kinv = 0.f;

#pragma unroll
    for (int s = 0; s < kStages - 1; ++s) {
        issue(wb + s);
        cp_async_commit();
    }

    for (int ti = wb; ti < we; ++ti) {
        issue(ti + kStages - 1);
        cp_async_commit();
        cp_async_wait<kStages - 1>();
        __syncwarp();
        const unsigned char *st = wmem + ((ti - wb) % kStages) * St::kBytes;
        const bool quant = ti < n_qt;
        float lg0, lg1;   // log2-domain logits of tokens g8 and g8 + 8 of the tile
        if (quant) {
            if (ti == wb || (ti & gmask) == 0) {
                // fixed-point key multipliers and bias of the group this tile opens
                const float *ks_s = reinterpret_cast<const float *>(st + St::kKs);
                const int16_t *kz_s = reinterpret_cast<const int16_t *>(st + St::kKz);
                float qs[NJ][4];
                float kb = 0.f, mx = 0.f;
#pragma unroll
                for (int j = 0; j < NJ; ++j) {
                    const int c0 = 16 * j + 4 * t4;
                    const float4 sc = *reinterpret_cast<const float4 *>(ks_s + c0);
                    const float4 qq = *reinterpret_cast<const float4 *>(q_s + c0);
                    qs[j][0] = qq.x * sc.x; qs[j][1] = qq.y * sc.y;
                    qs[j][2] = qq.z * sc.z; qs[j][3] = qq.w * sc.w;
                    float z[4] = {static_cast<float>(zsym), static_cast<float>(zsym),
                                  static_cast<float>(zsym), static_cast<float>(zsym)};
                    if (!a.sym) {
                        const uint2 zz = *reinterpret_cast<const uint2 *>(kz_s + c0);
                        z[0] = small_int_to_float(static_cast<int16_t>(zz.x & 0xffffu));
                        z[1] = small_int_to_float(static_cast<int16_t>(zz.x >> 16));
                        z[2] = small_int_to_float(static_cast<int16_t>(zz.y & 0xffffu));
                        z[3] = small_int_to_float(static_cast<int16_t>(zz.y >> 16));
                    }
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        kb = fmaf(qs[j][i], z[i], kb);
                        mx = fmaxf(mx, fabsf(qs[j][i]));
                    }
                }
                kb += __shfl_xor_sync(0xffffffffu, kb, 1);
                kb += __shfl_xor_sync(0xffffffffu, kb, 2);
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                // 2^e with |q'| * 2^e < 2^21: exponent of mx plus one, subtracted from 21
                int e = 0;
                if (mx > 0.f) e = 21 - (static_cast<int>((__float_as_uint(mx) >> 23) & 0xff) - 126);
                e = max(-120, min(120, e));
                const float scale = __uint_as_float(static_cast<uint32_t>(127 + e) << 23);
                kinv = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
#pragma unroll
                for (int j = 0; j < NJ; ++j) {
                    const int Q0 = round_small(qs[j][0] * scale), Q1 = round_small(qs[j][1] * scale);
                    const int Q2 = round_small(qs[j][2] * scale), Q3 = round_small(qs[j][3] * scale);
#pragma unroll
                    for (int k = 0; k < 3; ++k) {
                        const uint32_t sel = static_cast<uint32_t>(k | ((k + 4) << 4));
                        const uint32_t lo = __byte_perm(Q0, Q1, sel);
                        const uint32_t hi = __byte_perm(Q2, Q3, sel);
                        kdig[j][k] = __byte_perm(lo, hi, 0x5410);
                    }
                }
                kbias = kb;
            }
            uint32_t kw[W];
            load_stage_words<W>(reinterpret_cast<const uint32_t *>(st), lane, kw);
            int ak[2][3] = {{0, 0, 0}, {0, 0, 0}};
#pragma unroll
            for (int wi = 0; wi < W; ++wi) {
#pragma unroll
                for (int sl = 0; sl < SLOTS; ++sl) {
                    const uint32_t x = (kw[wi] >> (N * sl)) & BYTE_MASK;
                    const int j = wi * BPW + (sl >> 1), h = sl & 1;
                    ak[h][0] = dp4a_uu(x, kdig[j][0], ak[h][0]);
                    ak[h][1] = dp4a_uu(x, kdig[j][1], ak[h][1]);
                    ak[h][2] = dp4a_us(x, kdig[j][2], ak[h][2]);
                }
            }
            float x0 = (small_int_to_float(ak[0][0]) + 256.f * small_int_to_float(ak[0][1]) +
                        65536.f * small_int_to_float(ak[0][2])) * kinv;
            float x1 = (small_int_to_float(ak[1][0]) + 256.f * small_int_to_float(ak[1][1]) +
                        65536.f * small_int_to_float(ak[1][2])) * kinv;
            x0 += __shfl_xor_sync(0xffffffffu, x0, 1);
            x1 += __shfl_xor_sync(0xffffffffu, x1, 1);
            x0 += __shfl_xor_sync(0xffffffffu, x0, 2);
            x1 += __shfl_xor_sync(0xffffffffu, x1, 2);
            lg0 = x0 - kbias;
            lg1 = x1 - kbias;
        } else {
            // residual rows: exact e values
            const int row0 = (ti - n_qt) * 16 + g8, row1 = row0 + 8;
            float x0 = 0.f, x1 = 0.f;
            const uint16_t *kr = a.kr + bh * a.R * D;
#pragma unroll
            for (int j = 0; j < NJ; ++j) {
                const int c0 = 16 * j + 4 * t4;
                const float4 qq = *reinterpret_cast<const float4 *>(q_s + c0);
                if (row0 < r_rows) {
                    const uint2 kk = *reinterpret_cast<const uint2 *>(kr + row0 * D + c0);
                    x0 = fmaf(qq.x, widen(kk.x & 0xffffu, a.bf16), x0);
                    x0 = fmaf(qq.y, widen(kk.x >> 16, a.bf16), x0);
                    x0 = fmaf(qq.z, widen(kk.y & 0xffffu, a.bf16), x0);
                    x0 = fmaf(qq.w, widen(kk.y >> 16, a.bf16), x0);
                }
                if (row1 < r_rows) {
                    const uint2 kk = *reinterpret_cast<const uint2 *>(kr + row1 * D + c0);
                    x1 = fmaf(qq.x, widen(kk.x & 0xffffu, a.bf16), x1);
                    x1 = fmaf(qq.y, widen(kk.x >> 16, a.bf16), x1);
                    x1 = fmaf(qq.z, widen(kk.y & 0xffffu, a.bf16), x1);
                    x1 = fmaf(qq.w, widen(kk.y >> 16, a.bf16), x1);
                }
            }
            x0 += __shfl_xor_sync(0xffffffffu, x0, 1);
            x1 += __shfl_xor_sync(0xffffffffu, x1, 1);
            x0 += __shfl_xor_sync(0xffffffffu, x0, 2);
            x1 += __shfl_xor_sync(0xffffffffu, x1, 2);
            lg0 = row0 < r_rows ? x0 : -INFINITY;
            lg1 = row1 < r_rows ? x1 : -INFINITY;
        }

        // online softmax (log2 domain); m is uniform across the warp
        float tmax = fmaxf(lg0, lg1);
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 4));
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 8));
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 16));
        if (tmax > m) {
            const float alpha = fast_exp2(m - tmax);
            lsum *= alpha;
#pragma unroll
            for (int j = 0; j < NJ; ++j) {
                acc[j][0] = mul2(acc[j][0], make_float2(alpha, alpha));
                acc[j][1] = mul2(acc[j][1], make_float2(alpha, alpha));
            }
#pragma unroll
            for (int v = 0; v < NGV; ++v) zsum[v] *= alpha;
            m = tmax;
        }
        const float p0 = fast_exp2(lg0 - m), p1 = fast_exp2(lg1 - m);
        lsum += p0 + p1;
        // probabilities of the lane's value tokens 4*t4 + i (rows g8 + 8*(t4/2))
        const float pexp = (t4 & 2) ? p1 : p0;
        float pt[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            pt[i] = __shfl_sync(0xffffffffu, pexp, 4 * ((4 * t4 + i) & 7) + 2 * (t4 >> 1));

        if (quant) {
            const float *vsp = reinterpret_cast<const float *>(st + St::kVs) + 4 * t4 * NGV;
            const int16_t *vzp = reinterpret_cast<const int16_t *>(st + St::kVz) + 4 * t4 * NGV;
            float2 pm[NGV][2];   // (tokens i, i+2) x value scale x 2^-8i
#pragma unroll
            for (int v = 0; v < NGV; ++v) {
                float ps[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    ps[i] = pt[i] * vsp[i * NGV + v];
                    const float z = a.sym ? static_cast<float>(zsym) : small_int_to_float(vzp[i * NGV + v]);
                    zsum[v] = fmaf(ps[i], z, zsum[v]);
                }
                pm[v][0] = make_float2(ps[0], ps[2]);
                pm[v][1] = make_float2(ps[1] * (1.0f / 256.0f), ps[3] * (1.0f / 256.0f));
            }
            uint32_t vw[W];
            load_stage_words<W>(reinterpret_cast<const uint32_t *>(st + St::kCodes), lane, vw);
#pragma unroll
            for (int wi = 0; wi < W; ++wi) {
                const uint32_t lo = vw[wi], hi = vw[wi] >> 16;
#pragma unroll
                for (int sl = 0; sl < SLOTS; ++sl) {
                    const int j = wi * BPW + (sl >> 1), h = sl & 1;
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        const uint32_t msk = ((1u << N) - 1u) << (8 * i + N * sl);
                        float2 v = make_float2(__uint_as_float(and_or(lo, msk, magic)),
                                               __uint_as_float(and_or(hi, msk, magic)));
                        v = add2(v, make_float2(-kMagic, -kMagic));
                        acc[j][h] = fma2(v, pm[(16 * j) / GV][i], acc[j][h]);
                    }
                }
            }
        } else {
            const int ra = (ti - n_qt) * 16 + 4 * t4;
            const uint16_t *vr = a.vr + bh * a.R * D;
#pragma unroll
            for (int j = 0; j < NJ; ++j) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int c = 16 * j + g8 + 8 * h;
                    const float f = static_cast<float>(1u << (N * (2 * (j % BPW) + h)));
                    float vv[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        vv[i] = (ra + i < r_rows) ? pt[i] * widen(vr[(ra + i) * D + c], a.bf16) : 0.f;
                    acc[j][h] = fma2(make_float2(vv[0] + vv[1], vv[2] + vv[3]), make_float2(f, f),
                                     acc[j][h]);
                }
            }
        }
        __syncwarp();   // every lane is done with this stage before it is refilled
    }
    cp_async_wait<0>();

    // ---- warp epilogue: o for channels 16j + g8 + 8h, unnormalised ----
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 4);
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 8);
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 16);
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const float f = 1.0f / static_cast<float>(1u << (N * (2 * (j % BPW) + h)));
            float val = (acc[j][h].x + acc[j][h].y) * f - zsum[(16 * j) / GV];
            val += __shfl_xor_sync(0xffffffffu, val, 1);
            val += __shfl_xor_sync(0xffffffffu, val, 2);
            if (t4 == 0) o_s[warp][16 * j + g8 + 8 * h] = val;
        }
    }
    if (lane == 0) {
        ml_s[warp][0] = m;
        ml_s[warp][1] = lsum;
    }
    __syncthreads();

    // ---- merge the four warps, finish the split ----
    finish_cta<1, D>(a, &o_s[0][0], reinterpret_cast<const float(*)[1][2]>(ml_s), bq, bq, sigma,
                     &last_s, reinterpret_cast<float *>(stage_mem));
}

// Shared-memory bytes residual_pass needs per warp: one 16-row tile of K and of V,
// rows padded by 16 bytes so that the 8 row groups of a warp hit distinct banks.
template <int D>
__host__ __device__ constexpr int residual_scratch_bytes() { return 2 * 16 * (2 * D + 16); }

// Online-softmax pass of one warp over residual tiles rt0, rt0 + stride, ... < rt1
// of one query head (16 rows each; rows >= r, the residual rows of slice bh, masked) with the exact e values on
// CUDA cores.  Each tile's K and V rows are first staged in `scratch`
// (residual_scratch_bytes<D>() bytes of this warp's shared memory) with
// coalesced cp.async; the caller must have no cp.async group of its own
// pending.  qh is the log2-scaled query in shared memory; acc[j][h] accumulates
// channel 16j + g8 + 8h, x over tokens 4*t4 + {0, 1}, y over 4*t4 + {2, 3}.
template <int D>
__device__ __forceinline__ void residual_pass(const DecodeArgs &a, int64_t bh, int r, const float *qh, int rt0,
                                              int rt1, int lane, float &m, float &lsum, float2 (&acc)[D / 16][2],
                                              unsigned char *scratch, int stride = 1) {
    const uint16_t *kr = a.kr + bh * a.R * D, *vr = a.vr + bh * a.R * D;
    // a fused append: row new_row is read from the new token itself
    const uint16_t *nk = a.new_k ? a.new_k + bh * D : nullptr, *nv = a.new_v ? a.new_v + bh * D : nullptr;
    constexpr int NJ = D / 16;
    constexpr int kRow = 2 * D + 16;          // padded row stride in bytes
    constexpr int kPieces = 2 * D / 16;       // 16-byte pieces of one row
    const int g8 = lane >> 2, t4 = lane & 3;
    unsigned char *ks = scratch, *vs = scratch + 16 * kRow;
    for (int rt = rt0; rt < rt1; rt += stride) {
        const int rows = min(16, r - 16 * rt);
        const int n = rows * kPieces;
        __syncwarp();   // the previous tile's rows have been read
        for (int c = lane; c < 2 * n; c += 32) {
            const bool isv = c >= n;
            const int cc = isv ? c - n : c, row = cc / kPieces, pc = cc % kPieces;
            const int gr = 16 * rt + row;
            const uint16_t *src = (nk && gr == a.new_row) ? (isv ? nv : nk) : (isv ? vr : kr) + static_cast<int64_t>(gr) * D;
            cp_async16((isv ? vs : ks) + row * kRow + 16 * pc, src + 8 * pc);
        }
        cp_async_commit();
        cp_async_wait<0>();
        __syncwarp();
        const int row0 = g8, row1 = g8 + 8;
        float x0 = 0.f, x1 = 0.f;
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
            const int c0 = 16 * j + 4 * t4;
            const float4 qq = *reinterpret_cast<const float4 *>(qh + c0);
            const uint2 k0 = *reinterpret_cast<const uint2 *>(ks + row0 * kRow + 2 * c0);
            const uint2 k1 = *reinterpret_cast<const uint2 *>(ks + row1 * kRow + 2 * c0);
            x0 = fmaf(qq.x, widen(k0.x & 0xffffu, a.bf16), x0);
            x0 = fmaf(qq.y, widen(k0.x >> 16, a.bf16), x0);
            x0 = fmaf(qq.z, widen(k0.y & 0xffffu, a.bf16), x0);
            x0 = fmaf(qq.w, widen(k0.y >> 16, a.bf16), x0);
            x1 = fmaf(qq.x, widen(k1.x & 0xffffu, a.bf16), x1);
            x1 = fmaf(qq.y, widen(k1.x >> 16, a.bf16), x1);
            x1 = fmaf(qq.z, widen(k1.y & 0xffffu, a.bf16), x1);
            x1 = fmaf(qq.w, widen(k1.y >> 16, a.bf16), x1);
        }
        x0 += __shfl_xor_sync(0xffffffffu, x0, 1);
        x1 += __shfl_xor_sync(0xffffffffu, x1, 1);
        x0 += __shfl_xor_sync(0xffffffffu, x0, 2);
        x1 += __shfl_xor_sync(0xffffffffu, x1, 2);
        const float lg0 = row0 < rows ? x0 : -INFINITY;
        const float lg1 = row1 < rows ? x1 : -INFINITY;
        float tmax = fmaxf(lg0, lg1);
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 4));
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 8));
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 16));
        if (tmax > m) {
            const float alpha = fast_exp2(m - tmax);
            lsum *= alpha;
#pragma unroll
            for (int j = 0; j < NJ; ++j) {
                acc[j][0] = mul2(acc[j][0], make_float2(alpha, alpha));
                acc[j][1] = mul2(acc[j][1], make_float2(alpha, alpha));
            }
            m = tmax;
        }
        const float p0 = fast_exp2(lg0 - m), p1 = fast_exp2(lg1 - m);
        lsum += p0 + p1;
        const float pexp = (t4 & 2) ? p1 : p0;
        float pt[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            pt[i] = __shfl_sync(0xffffffffu, pexp, 4 * ((4 * t4 + i) & 7) + 2 * (t4 >> 1));
        // rows >= r hold stale bytes: their p is exactly 0 but 0 * stale could be NaN
        float vv[NJ][2][4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const bool ok = 4 * t4 + i < rows;
            const uint16_t *vrow = reinterpret_cast<const uint16_t *>(vs + (4 * t4 + i) * kRow);
#pragma unroll
            for (int j = 0; j < NJ; ++j)
#pragma unroll
                for (int h = 0; h < 2; ++h)
                    vv[j][h][i] = ok ? pt[i] * widen(vrow[16 * j + g8 + 8 * h], a.bf16) : 0.f;
        }
#pragma unroll
        for (int j = 0; j < NJ; ++j)
#pragma unroll
            for (int h = 0; h < 2; ++h)
                acc[j][h] = add2(acc[j][h], make_float2(vv[j][h][0] + vv[j][h][1], vv[j][h][2] + vv[j][h][3]));
    }
    __syncwarp();
}

// ---------------------------------------------------------------------------
// Tensor-core helpers (mma.sync).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void imma_uu(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void imma_uu0(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%10,%10,%10};"
        : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "r"(0));
}
__device__ __forceinline__ void imma_us(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// d = A B (no accumulator input)
__device__ __forceinline__ void imma_us0(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%10,%10,%10};"
        : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "r"(0));
}
__device__ __forceinline__ void hmma(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                     uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// (lo, hi) floats -> bf16x2 (round to nearest)
__device__ __forceinline__ uint32_t f2bf2(float lo, float hi) {
    uint32_t d;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}

// One token's value scales and zeros (NGV of each) from a stage, with vector loads.
template <int NGV>
__device__ __forceinline__ void load_meta(const float *sp, const int16_t *zp, bool sym, int zsym,
                                          float (&s)[NGV], int16_t (&z)[NGV]) {
    if constexpr (NGV == 4) {
        const float4 v = *reinterpret_cast<const float4 *>(sp);
        s[0] = v.x; s[1] = v.y; s[2] = v.z; s[3] = v.w;
    } else if constexpr (NGV == 2) {
        const float2 v = *reinterpret_cast<const float2 *>(sp);
        s[0] = v.x; s[1] = v.y;
    } else {
#pragma unroll
        for (int i = 0; i < NGV; ++i) s[i] = sp[i];
    }
    if (sym) {
#pragma unroll
        for (int i = 0; i < NGV; ++i) z[i] = static_cast<int16_t>(zsym);
    } else if constexpr (NGV == 4) {
        const uint2 v = *reinterpret_cast<const uint2 *>(zp);
        z[0] = static_cast<int16_t>(v.x & 0xffffu); z[1] = static_cast<int16_t>(v.x >> 16);
        z[2] = static_cast<int16_t>(v.y & 0xffffu); z[3] = static_cast<int16_t>(v.y >> 16);
    } else {
#pragma unroll
        for (int i = 0; i < NGV; ++i) z[i] = zp[i];
    }
}

// ---------------------------------------------------------------------------
// Tensor-core decode for HG = 1, 2 or 4 query heads per kv head.
//
// A CTA owns one (batch, kv head, split) and serves the HG query heads that
// read that kv head, so every code is fetched and unpacked once for all of
// them.  Each warp takes a contiguous share of the split's tiles, aligned to items,
// and walks it in chunks of tc_chunk<HG>() tiles: first the chunk's keys (the
// logits of its HG heads go to shared memory, each lane keeps a running
// maximum), then, with the chunk's maxima fixed, its values.  So probabilities
// need no per-tile cross-lane maximum, key and value work form two streams
// without dependences between tiles, and accumulators are rescaled at most once
// per chunk.  Items -- 4 tiles of keys or 4 tiles of values -- stream through a
// per-warp ring of bulk-copy stages.  Lane = 4*g8 + t4.
//   keys   : int8 MMA m16n8k32, rows = tokens, k = channels.  A is a stored
//            word masked to one byte slot, without a shift: slot s arrives as
//            code * 2^(N*s); the two 16-channel chunks of one MMA come from the
//            same slot class, so the factor is constant per row of the product
//            and divided out exactly.  B holds the balanced base-256 digits
//            (each in [-128, 127]) of the 22-bit fixed-point multipliers
//            Q_c = round(2^e q_c s_{g,c} log2(e)/sqrt(d)) of each head (e per
//            head and key group), built once per key group.  Head h's digits 0
//            and 1 sit in columns 2h, 2h+1, digit 2 in column 4 + 2h (HG <= 2)
//            or in column 2h of a second n-tile (HG = 4); int32 sums are exact.
//   values : bf16 MMA m16n8k16, rows = channels, k = tokens.  A is a stored
//            word masked to one byte slot (bytes 0, 2 of the word, or 1, 3 after
//            a shift by 8).  A bf16 pattern whose bits 8..15 are zero is exactly
//            (bits 0..7) * 2^-133: subnormal, or with bit 7 set the lowest
//            normal binade, and the two join linearly.  So A = code * 2^(N*s) *
//            2^-133 with no conversion.  B = p_t s_t 2^96 split into a bf16 hi
//            part (even columns) and lo part (odd columns) of head (g8/2) mod
//            HG; products ~ p s code 2^-37 stay well inside fp32's normal range
//            for value scales in [2^-40, 2^31].
//   z-terms: bias_{g,h} = sum_c q'_c z_{g,c} and sum_t p_t s_t z_t in fp32.
// Residual rows: with HG = 1 their tiles are dealt round-robin to the warps of
// all splits, which run them first on CUDA cores (staged in shared memory) and
// start their softmax state from them; with HG > 1 they form 1 to 16 splits of
// their own, their tiles dealt round-robin over the warps of all of them.
// Instances: PAGED reads a paged pool through each sequence's page table and
// takes each sequence's own length; SPARSE adds each token's key outliers.
// ---------------------------------------------------------------------------
constexpr int kTcItem = 4;         // tiles per item (stage)
constexpr int kVScaleLog2 = 96;   // the value MMA's B operand is p s 2^96

// Tiles per key phase / value phase of a warp (the logits of a chunk take 2 KB).
template <int HG>
__host__ __device__ constexpr int tc_chunk() { return 32 / HG; }

// cp.async of one tile's code array -- lane-major in global memory, lane l's W
// words at l*W -- into the chunk-major stage layout (16-byte piece p of lane l
// at slot 32p + l).  Every instruction reads 512 contiguous bytes; the slots
// one instruction writes are distinct banks in each quarter.
template <int W>
__device__ __forceinline__ void copy_tile_codes(unsigned char *dst, const uint32_t *src, int lane) {
    if constexpr (W % 4 == 0) {
        constexpr int P = W / 4;
#pragma unroll
        for (int i = 0; i < P; ++i) {
            const int gp = 32 * i + lane;
            cp_async16(dst + 16 * ((gp % P) * 32 + gp / P), src + 4 * gp);
        }
    } else {
        static_assert(W == 2, "lane segment of 8 bytes");
        cp_async8(dst + 8 * lane, src + 2 * lane);
    }
}

// The lane's W words of one tile's code array as stored (lane-major: lane l's words at l*W).
template <int W>
__device__ __forceinline__ void load_lane_words(const unsigned char *base, int lane, uint32_t (&w)[W]) {
    if constexpr (W % 4 == 0) {
#pragma unroll
        for (int i = 0; i < W / 4; ++i) {
            const uint4 v = reinterpret_cast<const uint4 *>(base)[lane * (W / 4) + i];
            w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
        }
    } else {
        static_assert(W == 2, "lane segment of 8 bytes");
        const uint2 v = reinterpret_cast<const uint2 *>(base)[lane];
        w[0] = v.x; w[1] = v.y;
    }
}

template <int N, int D, int GV>
struct TcStage {                  // one item: kTcItem tiles of one code array and their meta
    static constexpr int W = D * N / 64;
    static constexpr int NGV = D / GV;
    static constexpr int kCodes = 32 * W * 4;            // one tile's code array, as stored (lane-major)
    static constexpr int kMeta = kTcItem * kCodes;
    // key item: scales [2][D] f32 at kMeta and zeros [2][D] i16 at kKz: slot 0 the group its
    // first tile opens, slot 1 the group its third tile opens (groups of 32 tokens); groups
    // of >= 64 tokens start on item boundaries, so they use slot 0 only
    static constexpr int kKz = kMeta + 2 * D * 4;
    // value item: scales [16 * kTcItem][NGV] f32 at kMeta, zeros [16 * kTcItem][NGV] i16 at kVz
    static constexpr int kVz = kMeta + 16 * kTcItem * NGV * 4;
    static constexpr int kEnd = (kKz + 2 * D * 2 > kVz + 16 * kTcItem * NGV * 2) ? kKz + 2 * D * 2
                                                                                : kVz + 16 * kTcItem * NGV * 2;
    static constexpr int kBytes = (kEnd + 15) / 16 * 16;
    static_assert(kMeta % 16 == 0 && kKz % 16 == 0 && kVz % 16 == 0, "align");
};

// Stages per warp ring: two (one in use, one in flight), three when items are small enough
// for four CTAs of four warps to keep them in shared memory.
template <int N, int D, int GV>
__host__ __device__ constexpr int tc_stages() { return TcStage<N, D, GV>::kBytes <= 3072 ? 3 : 2; }

template <int N, int D, int GV, int HG>
struct TcSmem {
    static constexpr int kSt = tc_stages<N, D, GV>();
    static constexpr int kKdWords = D / 4 + 4;   // one digit row (4 channels a word), padded by 4 banks
    static constexpr int kLg = kSt * TcStage<N, D, GV>::kBytes;                // logits [chunk][HG][16] f32
    static constexpr int kKd = kLg + tc_chunk<HG>() * HG * 16 * 4;             // digits [HG][3][kKdWords]
    static constexpr int kBars = kKd + HG * 3 * kKdWords * 4;                 // stage barriers [kSt]
    static constexpr int kWarpBytes = (kBars + kSt * 8 + 15) / 16 * 16;
    static_assert(kLg % 16 == 0 && kBars % 16 == 0, "align");
};

// Position of token t (0..15) of a tile in the logits buffer: tokens 4q + e and 4q + e + 2
// sit side by side, the pair one lane of the value-B build needs.
__device__ __forceinline__ int logit_pos(int t) { return 4 * (t >> 2) + 2 * (t & 1) + ((t >> 1) & 1); }

template <int D, int GV, int HG>
__host__ __device__ constexpr int tc_min_ctas() { return 4; }

template <int N, int D, int GV, int HG, bool PAGED, bool SPARSE>
__global__ void __launch_bounds__(kDecodeThreads, tc_min_ctas<D, GV, HG>()) decode_tc_kernel(const DecodeArgs a) {
    constexpr int W = D * N / 64;
    constexpr int TW = D * N / 2;
    constexpr int NJ = D / 16;
    constexpr int BPW = 4 / N;        // slot classes (chunks per word)
    constexpr int NP = W / 2;         // word pairs; the key MMAs of a tile are (pair, class)
    constexpr int NGV = D / GV;
    constexpr int NTK = HG == 4 ? 2 : 1;                  // n-tiles of the key MMA
    constexpr int LPH = 32 / HG;                          // lanes per head when building digits
    constexpr int QPL = (D / 4 + LPH - 1) / LPH;          // channel quads per lane when building digits
    constexpr int kChunk = tc_chunk<HG>();
    constexpr uint32_t BYTE_L = ((1u << N) - 1u) * 0x01010101u;
    constexpr uint32_t HALF_L = ((1u << N) - 1u) * 0x00010001u;
    using St = TcStage<N, D, GV>;
    using Sm = TcSmem<N, D, GV, HG>;
    constexpr int kSt = Sm::kSt;
    static_assert(HG == 1 || HG == 2 || HG == 4, "heads per kv head");
    static_assert(W % 2 == 0, "key MMAs take words in pairs");
    static_assert(kChunk % kTcItem == 0 && (kChunk & (kChunk - 1)) == 0, "chunk");
    static_assert(residual_scratch_bytes<D>() <= Sm::kBars, "residual staging");
    static_assert((kDecodeWarps * HG * D + finish_scratch_floats<HG, D>()) * 4 <= kDecodeWarps * Sm::kWarpBytes,
                  "epilogue");

    __shared__ __align__(16) float q_s[HG][D];
    __shared__ float ml_s[kDecodeWarps][HG][2];
    __shared__ int last_s;
    extern __shared__ __align__(128) unsigned char stage_mem[];

    const int hk = blockIdx.x, b = blockIdx.y, sigma = blockIdx.z;
    const int64_t bh = static_cast<int64_t>(b) * a.Hkv + hk;
    const int64_t bq0 = static_cast<int64_t>(b) * a.Hq + static_cast<int64_t>(hk) * HG;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g8 = lane >> 2, t4 = lane & 3;
    const int hown = t4 & (HG - 1);            // head of this lane's logits and value columns
    const int hb = (g8 >> 1) & (HG - 1);       // head of this lane's value-B column
    unsigned char *wmem = stage_mem + static_cast<size_t>(warp) * Sm::kWarpBytes;
    float *lgs = reinterpret_cast<float *>(wmem + Sm::kLg);
    uint32_t *kd = reinterpret_cast<uint32_t *>(wmem + Sm::kKd);
    uint64_t *bars = reinterpret_cast<uint64_t *>(wmem + Sm::kBars);
    const int zsym = 1 << (N - 1);
    int n_qt, r_rows;
    seq_extent<PAGED>(a, b, n_qt, r_rows);

    for (int i = threadIdx.x; i < HG * D; i += kDecodeThreads)
        q_s[i / D][i % D] = widen(a.q[bq0 * D + i], a.bf16) * a.qscale;
    // a fused append: split 0 stores the new token as residual row new_row, for later steps
    // (every CTA of this call reads that row from the new token itself)
    if (a.new_k && sigma == 0) {
        for (int i = threadIdx.x; i < 2 * D / 8; i += kDecodeThreads) {
            const bool isv = i >= D / 8;
            const int c = isv ? i - D / 8 : i;
            const uint4 val = reinterpret_cast<const uint4 *>((isv ? a.new_v : a.new_k) + bh * D)[c];
            reinterpret_cast<uint4 *>((isv ? a.vr : a.kr) + (bh * a.R + a.new_row) * D)[c] = val;
        }
    }
    __syncthreads();

    float *o_s = reinterpret_cast<float *>(stage_mem);   // epilogue: [warp][HG][D]

    if constexpr (HG > 1) {
        if (sigma >= a.n_qsplits) {
            // ---------------- residual splits: kDecodeWarps / HG warps per head in each; the
            //                  residual tiles are dealt round-robin over the warps of all of them ----
            constexpr int WPH = kDecodeWarps / HG;
            const int h = warp / WPH;
            const int rs = sigma - a.n_qsplits, nrs = a.S - a.n_qsplits;
            float m = -INFINITY, lsum = 0.f;
            float2 acc[NJ][2];
#pragma unroll
            for (int j = 0; j < NJ; ++j) acc[j][0] = acc[j][1] = make_float2(0.f, 0.f);
            residual_pass<D>(a, bh, r_rows, q_s[h], rs * WPH + warp % WPH, (r_rows + 15) / 16, lane, m, lsum, acc,
                             wmem, WPH * nrs);
            lsum += __shfl_xor_sync(0xffffffffu, lsum, 4);
            lsum += __shfl_xor_sync(0xffffffffu, lsum, 8);
            lsum += __shfl_xor_sync(0xffffffffu, lsum, 16);
            __syncthreads();   // every warp is done with its staged rows before o_s overwrites them
#pragma unroll
            for (int j = 0; j < NJ; ++j) {
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    float val = acc[j][hh].x + acc[j][hh].y;
                    val += __shfl_xor_sync(0xffffffffu, val, 1);
                    val += __shfl_xor_sync(0xffffffffu, val, 2);
                    if (t4 == 0) o_s[(warp * HG + h) * D + 16 * j + g8 + 8 * hh] = val;
                }
            }
            if (lane < HG) {
                ml_s[warp][lane][0] = lane == h ? m : -INFINITY;
                ml_s[warp][lane][1] = lane == h ? lsum : 0.f;
            }
            __syncthreads();
            finish_cta<HG, D>(a, o_s, ml_s, bh, bq0, sigma, &last_s, o_s + kDecodeWarps * HG * D);
            return;
        }
    }

    // ---------------- quantized split ----------------
    const int t_begin = min(n_qt, sigma * a.tiles_per_split);      // multiple of kTcItem
    const int t_end = min(n_qt, t_begin + a.tiles_per_split);
    const int per_w = kTcItem * ((t_end - t_begin + kTcItem * kDecodeWarps - 1) / (kTcItem * kDecodeWarps));
    const int wb = min(t_end, t_begin + warp * per_w);             // multiple of kTcItem
    const int ntiles = min(t_end, wb + per_w) - wb;
    const int nitems = 2 * ((ntiles + kTcItem - 1) / kTcItem);     // a key item and a value item per kTcItem tiles
    const int64_t tile0 = bh * (a.cap / 16) + wb;
    const int gmask = (1 << a.gshift) - 1;

    // Item cursor: chunk [cb, cb + kChunk) of the warp's tiles holds ni items of each kind;
    // items 0 .. ni-1 of a chunk are its key items, ni .. 2ni-1 its value items.
    struct Cursor {
        int cb, r, ni;
        __device__ void start(int n) { cb = 0; r = 0; ni = (min(kChunk, n) + kTcItem - 1) / kTcItem; }
        __device__ void next(int n) {
            if (++r == 2 * ni) {
                cb += kChunk;
                r = 0;
                ni = (min(kChunk, n - cb) + kTcItem - 1) / kTcItem;
            }
        }
        __device__ bool key() const { return r < ni; }
        __device__ int rel() const { return cb + kTcItem * (r < ni ? r : r - ni); }
    };

    // Producer: lane 0 loads item `issued` into stage issued % kSt with bulk copies that
    // complete on the stage's barrier: the item's codes (one contiguous copy), then a key
    // item's group scales / zeros (the groups its tiles open, consecutive in memory) or a
    // value item's scales / zeros.  Key and value items each advance through the warp's tiles
    // in order, so the sources are running pointers.
    Cursor ic;       // producer's cursor, kSt - 1 items ahead
    ic.start(ntiles);
    int issued = 0;
    const uint32_t *ksrc = a.kc + tile0 * TW, *vsrc = a.vc + tile0 * TW;
    const float *vssrc = a.vs + tile0 * 16 * NGV;
    const int16_t *vzsrc = a.sym ? nullptr : a.vz + tile0 * 16 * NGV;
    const int64_t gbase = bh * (a.cap / a.G);
    // paged cache: each kind's running pointers restart at every page its items enter
    // (pages hold whole items); kt0 is the key page's tile base (global tile = kt0 + ti)
    int64_t kt0 = 0;
    PageWindow kwin, vwin;
    auto issue_next = [&]() {
        if (issued < nitems) {
            const int rel = ic.rel();
            const int nt = min(kTcItem, ntiles - rel);
            if constexpr (PAGED) {
                const int ti = wb + rel;
                if (rel == 0 || ti % a.page_tiles == 0) {
                    const int pi = ti / a.page_tiles;
                    if (ic.key()) {
                        kt0 = page_tile_base(a, kwin.page(a, b, pi, lane), hk, pi);
                        ksrc = a.kc + (kt0 + ti) * TW;
                    } else {
                        const int64_t vt = page_tile_base(a, vwin.page(a, b, pi, lane), hk, pi) + ti;
                        vsrc = a.vc + vt * TW;
                        vssrc = a.vs + vt * 16 * NGV;
                        if (!a.sym) vzsrc = a.vz + vt * 16 * NGV;
                    }
                }
            }
            if (lane == 0) {
                unsigned char *st = wmem + (issued % kSt) * St::kBytes;
                uint64_t *bar = bars + issued % kSt;
                const uint32_t cbytes = static_cast<uint32_t>(nt * St::kCodes);
                fence_proxy_async();   // this stage's earlier reads come before the copies below
                if (ic.key()) {
                    const int ti = wb + rel;
                    const bool open0 = rel == 0 || (ti & gmask) == 0;
                    const bool open2 = nt > 2 && ((ti + 2) & gmask) == 0;   // groups of 32 tokens
                    const int ng = open0 + open2;
                    const uint32_t sb = static_cast<uint32_t>(ng * D * 4);
                    const uint32_t zb = a.sym ? 0u : static_cast<uint32_t>(ng * D * 2);
                    mbar_expect_tx(bar, cbytes + sb + zb);
                    bulk_g2s(st, ksrc, cbytes, bar);
                    if constexpr (SPARSE)   // the item's outlier words, read by every lane next to its MMAs
                        bulk_prefetch_l2(a.k_out + (bh * (a.cap / 16) + ti) * 16 * a.n_out,
                                         static_cast<uint32_t>(nt * 16 * a.n_out * 4));
                    if (ng > 0) {
                        const int tg = open0 ? ti : ti + 2;
                        const int64_t gofs = (PAGED ? (kt0 + tg) >> a.gshift : gbase + (tg >> a.gshift)) * D;
                        bulk_g2s(st + St::kMeta + (open0 ? 0 : D * 4), a.ks + gofs, sb, bar);
                        if (!a.sym) bulk_g2s(st + St::kKz + (open0 ? 0 : D * 2), a.kz + gofs, zb, bar);
                    }
                } else {
                    const uint32_t sb = static_cast<uint32_t>(nt * 16 * NGV * 4);
                    const uint32_t zb = a.sym ? 0u : sb / 2;
                    mbar_expect_tx(bar, cbytes + sb + zb);
                    bulk_g2s(st, vsrc, cbytes, bar);
                    bulk_g2s(st + St::kMeta, vssrc, sb, bar);
                    if (!a.sym) bulk_g2s(st + St::kVz, vzsrc, zb, bar);
                }
            }
            if (ic.key()) {
                ksrc += kTcItem * TW;
            } else {
                vsrc += kTcItem * TW;
                vssrc += kTcItem * 16 * NGV;
                if (!a.sym) vzsrc += kTcItem * 16 * NGV;
            }
            ic.next(ntiles);
        }
        ++issued;
    };

    float m_own = -INFINITY;   // running maximum of head hown (this lane's logits and value columns)
    float mB = -INFINITY;      // running maximum of head hb (this lane's value-B column)
    float lsum = 0.f;          // sum of p 2^96 of head hb over this lane's tokens
    float dv[NJ][4];           // value MMA accumulators: rows = channels 16j + g8 (+8), columns 2*t4, 2*t4 + 1
#pragma unroll
    for (int j = 0; j < NJ; ++j) dv[j][0] = dv[j][1] = dv[j][2] = dv[j][3] = 0.f;
    float zsum[NGV];           // sum of p s z 2^96 of head hb over this lane's tokens
#pragma unroll
    for (int v = 0; v < NGV; ++v) zsum[v] = 0.f;
    uint32_t kb[NTK][NP * BPW][2];   // key MMA B fragments of the current group
    float klane = 0.f, kinv2 = 0.f, kbias = 0.f;
    float mloc = -INFINITY;          // this lane's largest logit of the current chunk

    // Key digits of a key group (scales [D] f32, zeros [D] i16); lane l builds head
    // l / LPH, channel quads l % LPH + LPH * i.
    auto rebuild_key_digits = [&](const float *ks_s, const int16_t *kz_s) {
        const int hd = lane / LPH, li = lane % LPH;
        float qv[QPL][4];
        float kbp = 0.f, mx = 0.f;
#pragma unroll
        for (int i = 0; i < QPL; ++i) {
            const int c4 = li + LPH * i;
            const bool ok = c4 < D / 4;             // d = 64, HG = 1: lanes 16..31 repeat quads
            const int cc = ok ? c4 : c4 - D / 4;
            const float4 sc = *reinterpret_cast<const float4 *>(ks_s + 4 * cc);
            const float4 qq = *reinterpret_cast<const float4 *>(&q_s[hd][4 * cc]);
            qv[i][0] = qq.x * sc.x; qv[i][1] = qq.y * sc.y; qv[i][2] = qq.z * sc.z; qv[i][3] = qq.w * sc.w;
            float z[4] = {static_cast<float>(zsym), static_cast<float>(zsym), static_cast<float>(zsym),
                          static_cast<float>(zsym)};
            if (!a.sym) {
                const uint2 zz = *reinterpret_cast<const uint2 *>(kz_s + 4 * cc);
                z[0] = static_cast<float>(static_cast<int16_t>(zz.x & 0xffffu));
                z[1] = static_cast<float>(static_cast<int16_t>(zz.x >> 16));
                z[2] = static_cast<float>(static_cast<int16_t>(zz.y & 0xffffu));
                z[3] = static_cast<float>(static_cast<int16_t>(zz.y >> 16));
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                if (ok) kbp = fmaf(qv[i][k], z[k], kbp);
                mx = fmaxf(mx, fabsf(qv[i][k]));
            }
        }
#pragma unroll
        for (int o = 1; o < LPH; o <<= 1) {
            kbp += __shfl_xor_sync(0xffffffffu, kbp, o);
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        }
        // 2^e with |q'| 2^e < 2^21, from the exponent of the head's largest |q'|
        int e = 0;
        if (mx > 0.f) e = 21 - (static_cast<int>((__float_as_uint(mx) >> 23) & 0xff) - 126);
        e = max(-120, min(120, e));
        const float scale = __uint_as_float(static_cast<uint32_t>(127 + e) << 23);
        // base-256 digits Q = d0 + 256 d1 + 65536 d2.  HG = 4: the bytes of Q themselves,
        // d0 and d1 unsigned and d2 signed (digit 2 has an n-tile, and an MMA type, of its own);
        // HG <= 2 (all digits in one n-tile, one signed type): balanced d0, d1 in [-128, 127]
        uint32_t dw[3][QPL];
#pragma unroll
        for (int i = 0; i < QPL; ++i) {
            int dg[3][4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int Q = round_small(qv[i][k] * scale);
                if constexpr (HG == 4) {
                    dg[0][k] = Q;
                    dg[1][k] = Q >> 8;
                    dg[2][k] = Q >> 16;
                } else {
                    const int Q1 = (Q + 128) >> 8;
                    dg[0][k] = Q;
                    dg[1][k] = Q1;
                    dg[2][k] = (Q1 + 128) >> 8;
                }
            }
#pragma unroll
            for (int k = 0; k < 3; ++k)
                dw[k][i] = __byte_perm(__byte_perm(dg[k][0], dg[k][1], 0x0040),
                                       __byte_perm(dg[k][2], dg[k][3], 0x0040), 0x5410);
        }
        __syncwarp();   // the previous group's digits have been read
#pragma unroll
        for (int i = 0; i < QPL; ++i) {
            const int c4 = li + LPH * i;
            if (c4 < D / 4) {
#pragma unroll
                for (int k = 0; k < 3; ++k) kd[(hd * 3 + k) * Sm::kKdWords + c4] = dw[k][i];
            }
        }
        __syncwarp();
        // B fragments: column g8 of each n-tile
#pragma unroll
        for (int nt = 0; nt < NTK; ++nt) {
            int hh, dig;
            bool has;
            if (HG == 4) {
                hh = g8 >> 1;
                dig = nt == 0 ? (g8 & 1) : 2;
                has = nt == 0 || (g8 & 1) == 0;
            } else if (g8 < 2 * HG) {
                hh = g8 >> 1;
                dig = g8 & 1;
                has = true;
            } else {
                hh = (g8 - 4) >> 1;
                dig = 2;
                has = g8 >= 4 && (g8 & 1) == 0 && hh < HG;
            }
            const uint32_t *row = kd + ((has ? hh : 0) * 3 + dig) * Sm::kKdWords;
#pragma unroll
            for (int pm = 0; pm < NP; ++pm) {
#pragma unroll
                for (int c = 0; c < BPW; ++c) {
                    const int j1 = 2 * pm * BPW + c, j2 = j1 + BPW;
                    kb[nt][pm * BPW + c][0] = has ? row[4 * j1 + t4] : 0u;
                    kb[nt][pm * BPW + c][1] = has ? row[4 * j2 + t4] : 0u;
                }
            }
        }
        // this lane's head (hown): its exponent and bias from the head's first building lane
        const float kinv = __shfl_sync(0xffffffffu, __uint_as_float(static_cast<uint32_t>(127 - e) << 23),
                                       hown * LPH);
        kbias = __shfl_sync(0xffffffffu, kbp, hown * LPH);
        if constexpr (HG == 4) {
            klane = kinv;
            kinv2 = kinv * 65536.f;
        } else {
            klane = t4 >= 2 ? kinv * 65536.f : kinv;   // lanes t4 = 2, 3 hold digit 2
        }
    };

    // ---- HG = 1: this warp's share of the residual tiles (dealt round-robin over the
    //      warps of all splits), on CUDA cores before the stream starts; its result seeds
    //      the softmax state (lane t4 = 0 holds channels 16j + g8 (+8) in both layouts) ----
    if constexpr (HG == 1) {
        const int nres = (r_rows + 15) / 16;
        const int gw = sigma * kDecodeWarps + warp, nw = a.S * kDecodeWarps;
        if (gw < nres) {
            float lr = 0.f;
            float2 acc[NJ][2];
#pragma unroll
            for (int j = 0; j < NJ; ++j) acc[j][0] = acc[j][1] = make_float2(0.f, 0.f);
            residual_pass<D>(a, bh, r_rows, q_s[0], gw, nres, lane, m_own, lr, acc, wmem, nw);
            lr += __shfl_xor_sync(0xffffffffu, lr, 4);     // lanes hold rows g8, g8 + 8
            lr += __shfl_xor_sync(0xffffffffu, lr, 8);
            lr += __shfl_xor_sync(0xffffffffu, lr, 16);
#pragma unroll
            for (int j = 0; j < NJ; ++j) {
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    float val = acc[j][hh].x + acc[j][hh].y;
                    val += __shfl_xor_sync(0xffffffffu, val, 1);
                    val += __shfl_xor_sync(0xffffffffu, val, 2);
                    const int slot = 2 * (j % BPW) + hh;   // value-MMA units: 2^(N slot - 37)
                    dv[j][2 * hh] = t4 == 0 ? val * __uint_as_float(static_cast<uint32_t>(127 + N * slot - 37) << 23) : 0.f;
                }
            }
            lsum = lane == 0 ? lr * __uint_as_float(static_cast<uint32_t>(127 + kVScaleLog2) << 23) : 0.f;
            mB = m_own;
        }
    }

    if (lane == 0) {
#pragma unroll
        for (int s = 0; s < kSt; ++s) mbar_init(bars + s, 1);
        fence_mbar_init();
    }
    __syncwarp();
#pragma unroll
    for (int s = 0; s < kSt - 1; ++s) issue_next();

    Cursor cc;       // consumer's cursor
    cc.start(ntiles);
    int k = 0;
    const int e = g8 & 1, te = 4 * t4 + e;   // value-B lanes: token pair te, te + 2 (see below)
    for (; k < nitems; ++k) {
        issue_next();
        // wait for item k; a wait that gives up (never expected) raises the device status flag
        // and abandons the rest of this warp's items
        const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(bars + k % kSt, (k / kSt) & 1));
        if (!ok) {
            if (lane == 0) atomicOr(a.status, 1u);
            break;
        }
        const unsigned char *st = wmem + (k % kSt) * St::kBytes;
        const int rel = cc.rel();
        const int nt = min(kTcItem, ntiles - rel);
        float *lgc = lgs + (rel & (kChunk - 1)) * HG * 16;   // logits of the item's tiles: [tile][head][16]
        if (cc.key()) {
            // ---- key MMAs: log2-domain logits of tokens g8 and g8 + 8, head hown ----
            const bool open0 = rel == 0 || ((wb + rel) & gmask) == 0;
            const bool open2 = ((wb + rel + 2) & gmask) == 0;
#pragma unroll
            for (int u = 0; u < kTcItem; ++u) {
                if (u < nt) {
                    if ((u == 0 && open0) || (u == 2 && open2))
                        rebuild_key_digits(reinterpret_cast<const float *>(st + St::kMeta) + (u == 2 ? D : 0),
                                           reinterpret_cast<const int16_t *>(st + St::kKz) + (u == 2 ? D : 0));
                    uint32_t ko[2][2] = {};   // dense-and-sparse keys: outlier words of tokens g8, g8 + 8
                    if constexpr (SPARSE) {
                        const int64_t tok = (bh * (a.cap / 16) + wb + rel + u) * 16 + g8;
#pragma unroll
                        for (int o = 0; o < 2; ++o) {
                            if (o < a.n_out) {
                                ko[0][o] = __ldg(a.k_out + tok * a.n_out + o);
                                ko[1][o] = __ldg(a.k_out + (tok + 8) * a.n_out + o);
                            }
                        }
                    }
                    uint32_t kw[W];
                    load_lane_words<W>(st + u * St::kCodes, lane, kw);
                    int acc[NTK][2][BPW][4];   // two chains (even / odd word pair) per n-tile
#pragma unroll
                    for (int pm = 0; pm < NP; ++pm) {
#pragma unroll
                        for (int c = 0; c < BPW; ++c) {
                            const uint32_t mlo = BYTE_L << (N * 2 * c), mhi = BYTE_L << (N * (2 * c + 1));
                            const uint32_t af[4] = {kw[2 * pm] & mlo, kw[2 * pm] & mhi, kw[2 * pm + 1] & mlo,
                                                    kw[2 * pm + 1] & mhi};
#pragma unroll
                            for (int n = 0; n < NTK; ++n) {
                                if (HG == 4 && n == 0) {   // unsigned digits 0, 1
                                    if (pm < 2) imma_uu0(acc[n][pm][c], af, kb[n][pm * BPW + c][0], kb[n][pm * BPW + c][1]);
                                    else imma_uu(acc[n][pm & 1][c], af, kb[n][pm * BPW + c][0], kb[n][pm * BPW + c][1]);
                                } else {
                                    if (pm < 2) imma_us0(acc[n][pm][c], af, kb[n][pm * BPW + c][0], kb[n][pm * BPW + c][1]);
                                    else imma_us(acc[n][pm & 1][c], af, kb[n][pm * BPW + c][0], kb[n][pm * BPW + c][1]);
                                }
                            }
                        }
                    }
                    float x0 = 0.f, x1 = 0.f;
#pragma unroll
                    for (int c = 0; c < BPW; ++c) {   // digit sums d0 + 256 d1 (< 2^31), slot factor out
                        const float f0 = 1.0f / static_cast<float>(1u << (2 * N * c));
                        const float f1 = 1.0f / static_cast<float>(1u << (N * (2 * c + 1)));
                        float y0, y1;
                        if constexpr (HG == 4) {   // unsigned digit sums (< 2^23 each): convert apart
                            int s0 = acc[0][0][c][0], s1 = acc[0][0][c][1], s2 = acc[0][0][c][2], s3 = acc[0][0][c][3];
                            if constexpr (NP > 1) {
                                s0 += acc[0][1][c][0]; s1 += acc[0][1][c][1];
                                s2 += acc[0][1][c][2]; s3 += acc[0][1][c][3];
                            }
                            y0 = fmaf(static_cast<float>(s1), 256.f, static_cast<float>(s0)) * klane;
                            y1 = fmaf(static_cast<float>(s3), 256.f, static_cast<float>(s2)) * klane;
                        } else {
                            int r0 = acc[0][0][c][0] + acc[0][0][c][1] * 256, r1 = acc[0][0][c][2] + acc[0][0][c][3] * 256;
                            if constexpr (NP > 1) {
                                r0 += acc[0][1][c][0] + acc[0][1][c][1] * 256;
                                r1 += acc[0][1][c][2] + acc[0][1][c][3] * 256;
                            }
                            y0 = static_cast<float>(r0) * klane;
                            y1 = static_cast<float>(r1) * klane;
                        }
                        if constexpr (NTK == 2) {   // digit 2 of head t4 in the second n-tile
                            int e0 = acc[1][0][c][0], e1 = acc[1][0][c][2];
                            if constexpr (NP > 1) {
                                e0 += acc[1][1][c][0];
                                e1 += acc[1][1][c][2];
                            }
                            y0 = fmaf(static_cast<float>(e0), kinv2, y0);
                            y1 = fmaf(static_cast<float>(e1), kinv2, y1);
                        }
                        x0 = fmaf(y0, f0, x0);
                        x1 = fmaf(y1, f1, x1);
                    }
                    if constexpr (HG == 1) {   // every lane of a row group gets the logits
                        x0 += __shfl_xor_sync(0xffffffffu, x0, 1);
                        x1 += __shfl_xor_sync(0xffffffffu, x1, 1);
                    }
                    if constexpr (HG <= 2) {   // digit 2 from lane t4 ^ 2
                        x0 += __shfl_xor_sync(0xffffffffu, x0, 2);
                        x1 += __shfl_xor_sync(0xffffffffu, x1, 2);
                    }
                    float lg0 = x0 - kbias, lg1 = x1 - kbias;
                    if constexpr (SPARSE) {   // the outliers' q_c x_c (the dense part is 0 there)
#pragma unroll
                        for (int o = 0; o < 2; ++o) {
                            if (o < a.n_out) {
                                lg0 = fmaf(q_s[hown][ko[0][o] >> 16], widen(ko[0][o] & 0xffffu, a.bf16), lg0);
                                lg1 = fmaf(q_s[hown][ko[1][o] >> 16], widen(ko[1][o] & 0xffffu, a.bf16), lg1);
                            }
                        }
                    }
                    mloc = fmaxf(mloc, fmaxf(lg0, lg1));
                    if (t4 < HG) {
                        lgc[(u * HG + hown) * 16 + logit_pos(g8)] = lg0;
                        lgc[(u * HG + hown) * 16 + logit_pos(g8 + 8)] = lg1;
                    }
                }
            }
            if (cc.r == cc.ni - 1) {
                // the chunk's keys are done: fix its maxima, rescale what came before
                float cm = mloc;
                cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 4));
                cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 8));
                cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 16));
                const float mo = fmaxf(m_own, cm);
                const float ao = fast_exp2(m_own - mo);
                m_own = mo;
                const float mBn = __shfl_sync(0xffffffffu, m_own, hb);   // lane hb holds head hb
                const float aB = fast_exp2(mB - mBn);
                mB = mBn;
                if (__any_sync(0xffffffffu, ao != 1.f || aB != 1.f)) {
#pragma unroll
                    for (int j = 0; j < NJ; ++j) {
                        dv[j][0] *= ao; dv[j][1] *= ao; dv[j][2] *= ao; dv[j][3] *= ao;
                    }
                    lsum *= aB;
#pragma unroll
                    for (int v = 0; v < NGV; ++v) zsum[v] *= aB;
                }
                mloc = -INFINITY;
            }
        } else {
            // Value B of head hb: lane (g8, t4) owns tokens te = 4*t4 + e and te + 2 (e = g8 & 1),
            // the k-pair of B register e, and builds both bf16 parts of p s 2^96 for them; the
            // lane pair (e = 0, 1) then swaps halves: lane e = 0 keeps hi parts (column 2h),
            // lane e = 1 lo parts (column 2h + 1).
            const float mb = mB - static_cast<float>(kVScaleLog2);
#pragma unroll
            for (int u = 0; u < kTcItem; ++u) {
                if (u < nt) {
                    const float2 l2 = *reinterpret_cast<const float2 *>(lgc + (u * HG + hb) * 16 + 4 * t4 + 2 * e);
                    const float p0 = fast_exp2(l2.x - mb), p1 = fast_exp2(l2.y - mb);
                    lsum += p0 + p1;
                    float s0[NGV], s1[NGV];
                    int16_t z0[NGV], z1[NGV];
                    load_meta<NGV>(reinterpret_cast<const float *>(st + St::kMeta) + (16 * u + te) * NGV,
                                   reinterpret_cast<const int16_t *>(st + St::kVz) + (16 * u + te) * NGV, a.sym,
                                   zsym, s0, z0);
                    load_meta<NGV>(reinterpret_cast<const float *>(st + St::kMeta) + (16 * u + te + 2) * NGV,
                                   reinterpret_cast<const int16_t *>(st + St::kVz) + (16 * u + te + 2) * NGV, a.sym,
                                   zsym, s1, z1);
                    uint32_t B0[NGV], B1[NGV];
#pragma unroll
                    for (int v = 0; v < NGV; ++v) {
                        const float ps0 = p0 * s0[v], ps1 = p1 * s1[v];
                        zsum[v] = fmaf(ps0, static_cast<float>(z0[v]), zsum[v]);
                        zsum[v] = fmaf(ps1, static_cast<float>(z1[v]), zsum[v]);
                        const uint32_t hi = f2bf2(ps0, ps1);
                        const uint32_t lo = f2bf2(ps0 - __uint_as_float(hi << 16), ps1 - __uint_as_float(hi & 0xffff0000u));
                        const uint32_t y = __shfl_xor_sync(0xffffffffu, e ? hi : lo, 4);
                        B0[v] = e ? y : hi;
                        B1[v] = e ? lo : y;
                    }
                    // ---- value MMAs: rows = channels of chunk j, k = the tile's tokens ----
                    uint32_t vw[W];
                    load_lane_words<W>(st + u * St::kCodes, lane, vw);
#pragma unroll
                    for (int wi = 0; wi < W; ++wi) {
                        const uint32_t w02 = vw[wi], w13 = vw[wi] >> 8;   // bytes 0, 2 and 1, 3 in bits 0..7 of each half
#pragma unroll
                        for (int c = 0; c < BPW; ++c) {
                            const int j = wi * BPW + c;
                            const uint32_t m0 = HALF_L << (N * 2 * c), m1 = HALF_L << (N * (2 * c + 1));
                            hmma(dv[j], w02 & m0, w02 & m1, w13 & m0, w13 & m1, B0[(16 * j) / GV], B1[(16 * j) / GV]);
                        }
                    }
                }
            }
        }
        cc.next(ntiles);
        __syncwarp();   // stage consumed and the chunk's logits visible to every lane
    }
    // after an abandoned wait: give the copies still in flight their (bounded) time to land
    for (int j = k + 1; j < min(issued, nitems); ++j) mbar_wait_bounded(bars + j % kSt, (j / kSt) & 1);
    __syncwarp();
    if (lane == 0) {
#pragma unroll
        for (int s = 0; s < kSt; ++s) mbar_inval(bars + s);
    }

    // head sums of the value-B lanes: lanes g8 = 2h, 2h + 1 hold head h's tokens; reduce over
    // t4 and the lane pair, then the lanes of head hown read them from lane 8 * hown
#pragma unroll
    for (int o = 1; o <= 4; o <<= 1) {
        lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
#pragma unroll
        for (int v = 0; v < NGV; ++v) zsum[v] += __shfl_xor_sync(0xffffffffu, zsum[v], o);
    }
    constexpr float kUnB = 1.0f / (static_cast<float>(1ull << 48) * static_cast<float>(1ull << 48));   // 2^-96
    const float l_own = __shfl_sync(0xffffffffu, lsum, 8 * hown) * kUnB;
    float z_own[NGV];
#pragma unroll
    for (int v = 0; v < NGV; ++v) z_own[v] = __shfl_sync(0xffffffffu, zsum[v], 8 * hown) * kUnB;
    // dv sums code 2^(N slot) 2^-133 p s 2^96 = 2^(N slot - 37) p s code
    float ov[NJ][2];
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
        const int s0 = 2 * (j % BPW);
        const float f0 = __uint_as_float(static_cast<uint32_t>(127 + 37 - N * s0) << 23);
        const float f1 = __uint_as_float(static_cast<uint32_t>(127 + 37 - N * (s0 + 1)) << 23);
        ov[j][0] = (dv[j][0] + dv[j][1]) * f0 - z_own[(16 * j) / GV];
        ov[j][1] = (dv[j][2] + dv[j][3]) * f1 - z_own[(16 * j) / GV];
    }

    __syncthreads();   // stage memory is reused for the per-warp outputs
    if (t4 < HG) {
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
            o_s[(warp * HG + hown) * D + 16 * j + g8] = ov[j][0];
            o_s[(warp * HG + hown) * D + 16 * j + g8 + 8] = ov[j][1];
        }
        if (g8 == 0) {
            ml_s[warp][hown][0] = m_own;
            ml_s[warp][hown][1] = l_own;
        }
    }
    __syncthreads();
    finish_cta<HG, D>(a, o_s, ml_s, bh, bq0, sigma, &last_s, o_s + kDecodeWarps * HG * D);
}

template <int N, int D, int GV>
constexpr int split_smem() { return kDecodeWarps * kStages * Stage<N, D, GV>::kBytes; }
template <int N, int D, int GV, int HG>
constexpr int tc_smem() { return kDecodeWarps * TcSmem<N, D, GV, HG>::kWarpBytes; }

// The opt-in to more than 48 KB of dynamic shared memory is per device and per
// kernel; it is made once for each.
template <auto Kernel>
cudaError_t configure_smem(int smem) {
    static bool configured[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 64 && configured[dev]) return cudaSuccess;
    e = cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess && dev < 64) configured[dev] = true;
    return e;
}

template <auto Kernel>
cudaError_t launch_kernel(const DecodeArgs &a, dim3 grid, int smem, cudaStream_t s) {
    cudaError_t e = configure_smem<Kernel>(smem);
    if (e != cudaSuccess) return e;
    Kernel<<<grid, kDecodeThreads, smem, s>>>(a);
    count_launches(1);
    return cudaGetLastError();
}

template <auto Kernel>
int occupancy_of(int smem) {
    int n = 0;
    if (configure_smem<Kernel>(smem) != cudaSuccess) return 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, Kernel, kDecodeThreads, smem) != cudaSuccess)
        return 1;
    return n > 0 ? n : 1;
}

// Dispatch over the compiled (bits, head_dim, value-group) variants and the kernels.
// The split index is the slowest grid dimension: CTAs start in linear order, so every
// quantized split is resident before the (short) residual-split CTAs fill the slots
// that remain.
template <int N, int D, int GV, bool PAGED, bool SPARSE>
struct LaunchF {
    template <int HG>
    static cudaError_t tc(const DecodeArgs &a, cudaStream_t s) {
        return launch_kernel<decode_tc_kernel<N, D, GV, HG, PAGED, SPARSE>>(a, dim3(a.Hkv, a.B, a.S),
                                                                            tc_smem<N, D, GV, HG>(), s);
    }
    static cudaError_t run(const DecodeArgs &a, cudaStream_t s) {
        if (a.path == kPathTc) {
            switch (a.Hq / a.Hkv) {
                case 1: return tc<1>(a, s);
                case 2: return tc<2>(a, s);
                case 4: return tc<4>(a, s);
                default: return cudaErrorInvalidValue;
            }
        }
        if constexpr (SPARSE) {
            return cudaErrorInvalidValue;   // dense-and-sparse keys run on the tensor-core path only
        } else {
            return launch_kernel<decode_split_kernel<N, D, GV, PAGED>>(a, dim3(a.Hq, a.B, a.S),
                                                                       split_smem<N, D, GV>(), s);
        }
    }
    static int occ(const DecodeArgs &a) {
        if (a.path == kPathTc) {
            switch (a.Hq / a.Hkv) {
                case 1: return occupancy_of<decode_tc_kernel<N, D, GV, 1, PAGED, SPARSE>>(tc_smem<N, D, GV, 1>());
                case 2: return occupancy_of<decode_tc_kernel<N, D, GV, 2, PAGED, SPARSE>>(tc_smem<N, D, GV, 2>());
                case 4: return occupancy_of<decode_tc_kernel<N, D, GV, 4, PAGED, SPARSE>>(tc_smem<N, D, GV, 4>());
                default: return 1;
            }
        }
        if constexpr (SPARSE) return 1;
        else return occupancy_of<decode_split_kernel<N, D, GV, PAGED>>(split_smem<N, D, GV>());
    }
};

template <int N, int D, bool PAGED, bool SPARSE>
cudaError_t launch_gv(const DecodeArgs &a, cudaStream_t s) {
    switch (a.Gv) {
        case 16: return LaunchF<N, D, 16, PAGED, SPARSE>::run(a, s);
        case 32: return LaunchF<N, D, 32, PAGED, SPARSE>::run(a, s);
        case 64: return LaunchF<N, D, 64, PAGED, SPARSE>::run(a, s);
        default: if constexpr (D >= 128) { if (a.Gv == 128) return LaunchF<N, D, 128, PAGED, SPARSE>::run(a, s); }
    }
    return cudaErrorInvalidValue;
}

template <int N, int D, bool PAGED, bool SPARSE>
int occ_gv(const DecodeArgs &a) {
    switch (a.Gv) {
        case 16: return LaunchF<N, D, 16, PAGED, SPARSE>::occ(a);
        case 32: return LaunchF<N, D, 32, PAGED, SPARSE>::occ(a);
        case 64: return LaunchF<N, D, 64, PAGED, SPARSE>::occ(a);
        default: if constexpr (D >= 128) { if (a.Gv == 128) return LaunchF<N, D, 128, PAGED, SPARSE>::occ(a); }
    }
    return 1;
}

template <bool PAGED, bool SPARSE = false>
cudaError_t launch_decode_variant(const DecodeArgs &a, cudaStream_t s) {
    if (a.bits == 2 && a.d == 64) return launch_gv<2, 64, PAGED, SPARSE>(a, s);
    if (a.bits == 2 && a.d == 128) return launch_gv<2, 128, PAGED, SPARSE>(a, s);
    if (a.bits == 4 && a.d == 64) return launch_gv<4, 64, PAGED, SPARSE>(a, s);
    if (a.bits == 4 && a.d == 128) return launch_gv<4, 128, PAGED, SPARSE>(a, s);
    return cudaErrorInvalidValue;
}

template <bool PAGED, bool SPARSE = false>
int ctas_per_sm_variant(const DecodeArgs &a) {
    if (a.bits == 2 && a.d == 64) return occ_gv<2, 64, PAGED, SPARSE>(a);
    if (a.bits == 2 && a.d == 128) return occ_gv<2, 128, PAGED, SPARSE>(a);
    if (a.bits == 4 && a.d == 64) return occ_gv<4, 64, PAGED, SPARSE>(a);
    if (a.bits == 4 && a.d == 128) return occ_gv<4, 128, PAGED, SPARSE>(a);
    return 1;
}

}  // namespace
}  // namespace kvq
