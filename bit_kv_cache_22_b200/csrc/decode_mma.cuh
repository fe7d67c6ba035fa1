// decode_mma.cuh -- the decode-attention kernel for contiguous caches whose query heads
// come 1, 2 or 4 to a kv head and whose key groups hold 32 tokens or more:
// decode_mma_kernel<N, D, GV, HG>.  It computes, for every (batch, query head),
//   A = softmax(q [deq(K_g); K_r]^T / sqrt(d)),   t_O = A [deq(V_g); V_r]
// ("LLM系列：KVCache量化1 KIVI ...", section 1: A = Concat(A_g, A_r), t_O = A X_V; the
// 1/sqrt(d_k) of "KV Cache的Int4量化…" section 3), deq(x) = (code - z) s ("Atom: Low-bit
// Quantization for Efficient and Accurate LLM Serving", 核心公式 / 量化基础).
//
// Work: one CTA per (batch, kv head, split) serves the HG query heads of that kv head,
// so every code is fetched and unpacked once for all of them.  Each of its four warps
// streams a contiguous, even-aligned share of the split's 16-token tiles in items of
// two tiles (32 tokens): one bulk copy (TMA engine, no multicast) per array brings the
// item's key codes, value codes, value scales / zeros and, when the item opens a key
// group, that group's key scales / zeros into a per-warp ring of shared-memory stages
// that complete on an mbarrier.  The residual rows form splits of their own (CUDA
// cores, exact e values).  The last split of a unit to finish merges the partials
// (finish_cta).
//
// Both contractions run on the tensor cores as bf16 mma.sync.m16n8k16 with fp32
// accumulation.  A stored code word masked to one n-bit slot of bytes 0 and 2 (or of
// bytes 1 and 3 after a shift by 8) is, read as two bf16 values, exactly
// code * 2^(n slot) * 2^-133: a bf16 pattern whose bits 8..15 are clear is its bits 0..7
// times 2^-133 (subnormal, or the lowest normal binade when bit 7 is set -- the two join
// linearly).  So the A operand costs one AND per register and no conversion.  The B
// operand holds the other factor split into a high part (the top 16 bits of the fp32
// value, i.e. truncated) and a low part (the exact remainder rounded to bf16), in the
// even and odd columns of each head: 16 significant bits per factor, about 2^-17
// relative error per product, before fp32 accumulation.
//   keys   : rows = tokens, k = channels, B = q_c s_{g,c} log2(e)/sqrt(d) 2^64, with chunks
//            of slot class c (channel chunk j, c = j mod 4/n) scaled by 2^(-2nc) so that
//            every chunk of a tile adds into one accumulator (rows g8 carry 2^0, rows
//            g8 + 8 carry 2^n).  logit = 2^69 (hi + lo) - bias, bias_g = sum_c q_c s z.
//   values : rows = channels, k = tokens, B = p_t s_{t,gv} 2^80 for each value group;
//            o_c = 2^(53 - n slot) (hi + lo) - sum_t p_t s_t z_t.
// Online softmax in the log2 domain with the exact running maximum per head, updated
// once per item; accumulators are rescaled only when a maximum grows.
#pragma once

#include "decode_kernels.cuh"

namespace kvq {
namespace {

constexpr int kMmaItemTiles = 2;    // tiles per item (stage)
constexpr int kKeyScaleLog2 = 64;   // the key MMA's B operand is q' s 2^64
constexpr int kValScaleLog2 = 80;   // the value MMA's B operand is p s 2^80
constexpr float kLazyRescale = 8.0f; // log2 units the logits may pass the running maximum by

template <int N, int D, int GV, int HG, bool RR>
struct MmaLayout {
    static constexpr int W = D * N / 64;            // code words per lane per tile
    static constexpr int TW = D * N / 2;            // code words per tile
    static constexpr int NJ = D / 16;               // 16-channel chunks
    static constexpr int BPW = 4 / N;               // chunks per word (slot classes)
    static constexpr int NGV = D / GV;              // value groups per token
    static constexpr int kTok = 16 * kMmaItemTiles;
    // A stage holds what arrives for kIPS items, each array as one contiguous block:
    //   [key codes][value codes][key scales][key zeros][value scales][value zeros],
    // codes lane-major per tile, and the key scales / zeros of up to kGPS key groups.
    // RR (round robin, key groups of 2 tiles): one ring shared by the CTA whose stages hold
    // a round, the kDecodeWarps consecutive items the warps take one each.  A round is
    // 2 kDecodeWarps tiles from an even tile, so it meets at most kDecodeWarps groups.
    // Otherwise every warp has a ring of its own whose stages hold one of its items.
    static constexpr int kIPS = RR ? kDecodeWarps : 1;             // items per stage
    static constexpr int kGPS = RR ? kDecodeWarps : 1;             // key groups per stage
    static constexpr int kRings = RR ? 1 : kDecodeWarps;
    static constexpr int kItemCodes = kMmaItemTiles * TW * 4;   // bytes of one item's key (or value) codes
    static constexpr int kItemVs = kTok * NGV * 4;              // bytes of one item's value scales
    static constexpr int kRk = 0;
    static constexpr int kRv = kIPS * kItemCodes;
    static constexpr int kRks = 2 * kIPS * kItemCodes;
    static constexpr int kRkz = kRks + kGPS * D * 4;
    static constexpr int kRvs = kRkz + kGPS * D * 2;
    static constexpr int kRvz = kRvs + kIPS * kItemVs;
    static constexpr int kStage = (kRvz + kIPS * kItemVs / 2 + 127) / 128 * 128;
    static constexpr int kSt = 2;                            // ring depth: one stage in flight
    // per-warp scratch.  Key B staging [part][head][t4][2 NJ words]: rows of 24 words and a
    // part stride of 4 mod 32 words keep both the producers' 8-byte stores and the
    // consumers' 16-byte loads free of bank conflicts.  It is dead once the fragments are in
    // registers, so the value-phase buffers share its memory.
    static constexpr int RS = 24;
    static constexpr int PS = HG * 4 * RS + 4;
    // value B exchange (NGV >= 4): [part][head][t4][e][NGV words], part stride 4 mod 32 words
    static constexpr int VXS = HG * 4 * 2 * NGV + 4;
    static constexpr int kKb = 0;                                    // u32 [2 * PS]
    static constexpr int kVx = 0;                                    // u32 [2 * VXS]
    static constexpr int kUv = kVx + (NGV >= 4 ? 2 * VXS * 4 : 0);   // f32 [kTok][NGV]: s z per (token, group)
    static constexpr int kPb = kUv + kTok * NGV * 4;                 // f32 [2 tiles][HG][18]: p 2^80
    static constexpr int kValueEnd = kPb + kMmaItemTiles * HG * 18 * 4;
    static constexpr int kWarpBytes = ((2 * PS * 4 > kValueEnd ? 2 * PS * 4 : kValueEnd) + 15) / 16 * 16;
    static constexpr int kQuantBytes = kRings * kSt * kStage + kDecodeWarps * kWarpBytes;
    // (the residual splits stage one 16-row tile of K and V rows per warp in the same memory)
    static constexpr int kSmem = kQuantBytes > kDecodeWarps * residual_scratch_bytes<D>()
                                     ? kQuantBytes : kDecodeWarps * residual_scratch_bytes<D>();
    static_assert(2 * NJ <= RS, "row");
    static_assert(kItemCodes % 16 == 0 && kRv % 16 == 0 && kRks % 16 == 0 && kRkz % 16 == 0 && kRvs % 16 == 0 &&
                  kRvz % 16 == 0 && (kItemVs / 2) % 16 == 0 && kUv % 16 == 0 && kPb % 16 == 0, "align");
};

template <int N, int D, int GV, int HG, bool RR>
__host__ __device__ constexpr int mma_smem() { return MmaLayout<N, D, GV, HG, RR>::kSmem; }

// The barrier arm and the bulk copy on 32-bit shared addresses.
__device__ __forceinline__ void mbar_expect_tx_u32(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bulk_g2s_u32(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_u32(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_u32(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "n"(kPollSuspendNs)
        : "memory");
    return ok != 0;
}
// Every lane of the warp waits for the phase of `parity` of barrier `bar`: one poll when the
// data is there, else bounded polling (false when it gave up).
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity) {
    if (__all_sync(0xffffffffu, mbar_try_wait_u32(bar, parity))) return true;
    bool ok = false;
    for (uint32_t i = 0; i < kSpinLimit && !ok; ++i) ok = mbar_try_wait_u32(bar, parity);
    return __all_sync(0xffffffffu, ok);
}

// n consecutive 32-bit values from / to shared memory with the widest vector accesses
template <int n, typename T>
__device__ __forceinline__ void load_vec(const T *p, T (&v)[n]) {
    static_assert(sizeof(T) == 4, "32-bit elements");
    if constexpr (n % 4 == 0) {
#pragma unroll
        for (int i = 0; i < n; i += 4) {
            const uint4 x = *reinterpret_cast<const uint4 *>(p + i);
            memcpy(&v[i], &x, 16);
        }
    } else if constexpr (n % 2 == 0) {
#pragma unroll
        for (int i = 0; i < n; i += 2) {
            const uint2 x = *reinterpret_cast<const uint2 *>(p + i);
            memcpy(&v[i], &x, 8);
        }
    } else {
#pragma unroll
        for (int i = 0; i < n; ++i) v[i] = p[i];
    }
}
template <int n, typename T>
__device__ __forceinline__ void store_vec(T *p, const T (&v)[n]) {
    static_assert(sizeof(T) == 4, "32-bit elements");
    if constexpr (n % 4 == 0) {
#pragma unroll
        for (int i = 0; i < n; i += 4) {
            uint4 x;
            memcpy(&x, &v[i], 16);
            *reinterpret_cast<uint4 *>(p + i) = x;
        }
    } else if constexpr (n % 2 == 0) {
#pragma unroll
        for (int i = 0; i < n; i += 2) {
            uint2 x;
            memcpy(&x, &v[i], 8);
            *reinterpret_cast<uint2 *>(p + i) = x;
        }
    } else {
#pragma unroll
        for (int i = 0; i < n; ++i) p[i] = v[i];
    }
}

// float -> its top 16 bits as bf16 (truncation), two at a time: lo half from a, hi from b
__device__ __forceinline__ uint32_t bf16_trunc2(float a, float b) {
    return __byte_perm(__float_as_uint(a), __float_as_uint(b), 0x7632);
}
// exact remainders a - trunc(a), b - trunc(b) rounded to bf16: lo half from a, hi from b
__device__ __forceinline__ uint32_t bf16_rem2(float a, float b) {
    const float ra = a - __uint_as_float(__float_as_uint(a) & 0xffff0000u);
    const float rb = b - __uint_as_float(__float_as_uint(b) & 0xffff0000u);
    return f2bf2(ra, rb);
}

// Sums v[0..H) over every aligned group of G lanes (G a power of two >= H) with log2 G
// shuffles of the halving kind: while a lane holds several values it keeps half of them
// and hands the other half to its partner.  Afterwards lane l holds the group's sum of
// v[(l mod G) / (G / H)].
template <int H, int G>
__device__ __forceinline__ float transpose_reduce(const float (&v)[H], int lane) {
    if constexpr (H == 1) {
        float x = v[0];
#pragma unroll
        for (int o = G / 2; o >= 1; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
        return x;
    } else {
        constexpr int o = G / 2;
        const bool up = (lane & o) != 0;
        float w[H / 2];
#pragma unroll
        for (int i = 0; i < H / 2; ++i) {
            const float send = up ? v[i] : v[i + H / 2];
            const float keep = up ? v[i + H / 2] : v[i];
            w[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
        return transpose_reduce<H / 2, G / 2>(w, lane);
    }
}

template <int N, int D, int GV, int HG, bool RR>
__global__ void __launch_bounds__(kDecodeThreads, D / GV >= 8 ? 3 : 4) decode_mma_kernel(const DecodeArgs a) {
    using L = MmaLayout<N, D, GV, HG, RR>;
    constexpr int W = L::W, TW = L::TW, NJ = L::NJ, BPW = L::BPW, NGV = L::NGV;
    constexpr int kSt = L::kSt;
    constexpr uint32_t HALF_L = ((1u << N) - 1u) * 0x00010001u;
    // key B producers: lane l owns channel quad l mod QUADS (channels 4 quad .. 4 quad + 3)
    // for HPL heads starting at head (l / QUADS) HPL
    constexpr int QUADS = D / 4;
    constexpr int LPQ = 32 / QUADS;                       // lanes per quad (1 or 2)
    constexpr int HPL = HG / LPQ > 0 ? HG / LPQ : 1;      // heads per producer lane
    static_assert(HG == 1 || HG == 2 || HG == 4, "heads per kv head");
    static_assert(W % 2 == 0 || W == 2, "words");
    // epilogue: per-warp outputs, then finish_cta's scratch
    static_assert((kDecodeWarps * HG * D + finish_scratch_floats<HG, D>()) * 4 <= L::kSmem, "epilogue");

    __shared__ __align__(16) float q_s[HG][D];   // q log2(e) / sqrt(d)
    __shared__ __align__(16) float qm_s[HG][D];  // the key MMA's multipliers: q_s 2^64 2^(-2n class)
    __shared__ float ml_s[kDecodeWarps][HG][2];
    __shared__ int last_s;
    // full barriers (copies landed), [ring][stage]; RR: then the empty barriers (released)
    __shared__ uint64_t rbar[L::kRings * kSt + (RR ? kSt : 0)];
    extern __shared__ __align__(128) unsigned char stage_mem[];

    const int hk = blockIdx.x, b = blockIdx.y, sigma = blockIdx.z;
    const int64_t bh = static_cast<int64_t>(b) * a.Hkv + hk;
    const int64_t bq0 = static_cast<int64_t>(b) * a.Hq + static_cast<int64_t>(hk) * HG;
    // the warp index through a shuffle from lane 0: provably warp-uniform, so everything derived
    // from it (the warp's tile range, the copy sources) can live in uniform registers
    const int warp = __shfl_sync(0xffffffffu, static_cast<int>(threadIdx.x >> 5), 0);
    const int lane = threadIdx.x & 31;
    const int g8 = lane >> 2, t4 = lane & 3;
    unsigned char *wmem = stage_mem + L::kRings * kSt * L::kStage + static_cast<size_t>(warp) * L::kWarpBytes;
    const int zsym = 1 << (N - 1);

    for (int i = threadIdx.x; i < HG * D; i += kDecodeThreads) {
        const float qv = widen(a.q[bq0 * D + i], a.bf16) * a.qscale;
        const int cls = ((i % D) / 16) % BPW;   // slot class of the channel's chunk
        q_s[i / D][i % D] = qv;
        qm_s[i / D][i % D] = qv * __uint_as_float(static_cast<uint32_t>(127 + kKeyScaleLog2 - 2 * N * cls) << 23);
    }
    if (threadIdx.x == 0) {
#pragma unroll
        for (int i = 0; i < L::kRings * kSt; ++i) mbar_init(rbar + i, 1);
        if constexpr (RR) {
#pragma unroll
            for (int i = 0; i < kSt; ++i) mbar_init(rbar + kSt + i, kDecodeWarps);
        }
        fence_mbar_init();
    }
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
    int n_qt, r_rows;
    seq_extent<false>(a, b, n_qt, r_rows);

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
                         stage_mem + warp * residual_scratch_bytes<D>(), WPH * nrs);
        lsum += __shfl_xor_sync(0xffffffffu, lsum, 4);
        lsum += __shfl_xor_sync(0xffffffffu, lsum, 8);
        lsum += __shfl_xor_sync(0xffffffffu, lsum, 16);
        __syncthreads();   // every warp is done with its staged rows before o_s overwrites them
        // each warp is a partial of its own for head h (its slots of the CTA's other heads
        // stay empty); finish_cta merges them like any warps
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

    // ---------------- quantized split ----------------
    // The CTA's tiles form items of kMmaItemTiles tiles, and round r gives each warp one item.
    // RR: warp w takes item w of every kDecodeWarps consecutive items, so a round is contiguous
    // in memory and arrives in one stage of the CTA's ring with one bulk copy per array.
    // Otherwise warp w takes the w-th contiguous quarter of the items (so it builds each key
    // group's operand once) and streams them through a ring of its own.
    const int t_begin = min(n_qt, sigma * a.tiles_per_split);      // multiple of kMmaItemTiles
    const int t_end = min(n_qt, t_begin + a.tiles_per_split);
    const int n_items = (t_end - t_begin) / kMmaItemTiles;        // (Tq is a multiple of G >= 32)
    const int n_rounds = (n_items + kDecodeWarps - 1) / kDecodeWarps;
    const int my_items = RR ? n_items : min(n_rounds, n_items - warp * n_rounds);   // (may be <= 0)
    auto item_of = [&](int r) { return RR ? r * kDecodeWarps + warp : warp * n_rounds + r; };
    const int64_t unit_tile0 = bh * (a.cap / 16);                 // global tile of the unit's tile 0
    const int gmask = (1 << a.gshift) - 1;                         // tiles per key group - 1
    uint32_t *kbs = reinterpret_cast<uint32_t *>(wmem + L::kKb);
    float *pb = reinterpret_cast<float *>(wmem + L::kPb);

    // Stage r mod kSt of the ring and its full barrier; RR: the stage's empty barrier, which
    // every warp arrives at once done with the round.
    const int ring = RR ? 0 : warp;
    const uint32_t s_stage0 = smem_u32(stage_mem) + ring * kSt * L::kStage;
    const uint32_t s_full0 = smem_u32(rbar) + 8u * ring * kSt, s_empty0 = smem_u32(rbar) + 8u * L::kRings * kSt;
    const unsigned char *kc = reinterpret_cast<const unsigned char *>(a.kc);
    const unsigned char *vc = reinterpret_cast<const unsigned char *>(a.vc);
    const unsigned char *vs = reinterpret_cast<const unsigned char *>(a.vs);
    const unsigned char *vz = reinterpret_cast<const unsigned char *>(a.vz);
    const unsigned char *ks = reinterpret_cast<const unsigned char *>(a.ks);
    const unsigned char *kz = reinterpret_cast<const unsigned char *>(a.kz);
    // Producer of round r (RR: lane 0 of warp r mod kDecodeWarps, the role rotating, once every
    // warp released the stage's previous round; else lane 0 of the ring's own warp): it arms
    // the stage's full barrier with the byte count and issues the copies.  Sources,
    // destinations and sizes are warp-uniform, so the copies take their operands from
    // uniform registers.
    auto issue_round = [&](int r) {
        const uint32_t slot = static_cast<uint32_t>(r % kSt);
        const uint32_t bar = s_full0 + 8u * slot, dst = s_stage0 + slot * L::kStage;
        fence_proxy_async();   // the stage's earlier reads come before the copies below
        if constexpr (RR) {
            const int i0 = r * kDecodeWarps;
            const int ni = min(kDecodeWarps, n_items - i0);
            const int t0 = t_begin + i0 * kMmaItemTiles;               // unit-local tiles [t0, t1)
            const int t1 = t0 + ni * kMmaItemTiles;
            const int g0 = t0 >> a.gshift;
            const uint32_t ng = static_cast<uint32_t>(((t1 - 1) >> a.gshift) - g0 + 1);
            const uint32_t codes = static_cast<uint32_t>(ni) * L::kItemCodes;
            const uint32_t vsb = static_cast<uint32_t>(ni) * L::kItemVs, ksb = ng * (D * 4);
            const uint32_t tx = 2u * codes + vsb + ksb + (a.sym ? 0u : (vsb + ksb) / 2);
            if (lane == 0) {
                const int64_t gt = unit_tile0 + t0, gg = (unit_tile0 >> a.gshift) + g0;
                mbar_expect_tx_u32(bar, tx);
                bulk_g2s_u32(dst + L::kRk, kc + gt * (TW * 4), codes, bar);
                bulk_g2s_u32(dst + L::kRv, vc + gt * (TW * 4), codes, bar);
                bulk_g2s_u32(dst + L::kRvs, vs + gt * (16 * NGV * 4), vsb, bar);
                bulk_g2s_u32(dst + L::kRks, ks + gg * (D * 4), ksb, bar);
                if (!a.sym) {
                    bulk_g2s_u32(dst + L::kRvz, vz + gt * (16 * NGV * 2), vsb / 2, bar);
                    bulk_g2s_u32(dst + L::kRkz, kz + gg * (D * 2), ksb / 2, bar);
                }
            }
        } else {
            // the warp's item r; its key group's scales / zeros when it opens a group or
            // starts the warp's quarter
            const int t = t_begin + item_of(r) * kMmaItemTiles;
            const bool open = r == 0 || (t & gmask) == 0;
            const uint32_t tx = 2u * L::kItemCodes + L::kItemVs + (a.sym ? 0u : L::kItemVs / 2) +
                                (open ? static_cast<uint32_t>(D * (a.sym ? 4 : 6)) : 0u);
            if (lane == 0) {
                const int64_t gt = unit_tile0 + t;
                mbar_expect_tx_u32(bar, tx);
                bulk_g2s_u32(dst + L::kRk, kc + gt * (TW * 4), L::kItemCodes, bar);
                bulk_g2s_u32(dst + L::kRv, vc + gt * (TW * 4), L::kItemCodes, bar);
                bulk_g2s_u32(dst + L::kRvs, vs + gt * (16 * NGV * 4), L::kItemVs, bar);
                if (!a.sym) bulk_g2s_u32(dst + L::kRvz, vz + gt * (16 * NGV * 2), L::kItemVs / 2, bar);
                if (open) {
                    const int64_t gg = gt >> a.gshift;
                    bulk_g2s_u32(dst + L::kRks, ks + gg * (D * 4), D * 4, bar);
                    if (!a.sym) bulk_g2s_u32(dst + L::kRkz, kz + gg * (D * 2), D * 2, bar);
                }
            }
        }
    };

    // key B producers: lane l owns channel quad l mod QUADS for HPL heads from hp0
    const int quad = lane % QUADS, hp0 = (lane / QUADS) * HPL % HG;
    const int pcls = (quad / 4) % BPW;
    // the bias from the producers' partial sums: 2^(-64 + 2nc) undoes qm's factors
    const float pbias_f = __uint_as_float(static_cast<uint32_t>(127 - kKeyScaleLog2 + 2 * N * pcls) << 23);

    uint32_t kb[NJ][2];        // key B fragments of the current group (column g8: head (g8/2) mod HG, part g8 & 1)
    float kbias = 0.f;         // bias of head t4 mod HG, current group
    float m_own = -INFINITY;   // running maximum of head t4 mod HG (logits and value columns of this lane)
    float lsum = 0.f;          // sum of p of head t4 mod HG over this lane's tokens
    float dv[NJ][4];           // value MMA accumulators: rows = channels 16j + g8 (+8), columns 2 t4, 2 t4 + 1
#pragma unroll
    for (int j = 0; j < NJ; ++j) dv[j][0] = dv[j][1] = dv[j][2] = dv[j][3] = 0.f;
    float zsum[NGV];           // sum of p s z of head hb over this lane's value tokens
#pragma unroll
    for (int v = 0; v < NGV; ++v) zsum[v] = 0.f;
    const int hb = (g8 >> 1) % HG;             // head of this lane's value-B column
    const int e = g8 & 1;                      // part of this lane's B columns: 0 = high, 1 = low
    const int te = 4 * t4 + e;                 // value-B tokens te, te + 2 of a tile
    const int kb_row = e * L::PS + (hb * 4 + t4) * L::RS;

    // Key B operand and bias of the group whose scales / zeros sit at ksp / kzp.
    auto build_key_b = [&](const unsigned char *ksp, const unsigned char *kzp) {
        const float4 s4 = *reinterpret_cast<const float4 *>(ksp + 16 * quad);
        float2 z01 = make_float2(static_cast<float>(zsym), static_cast<float>(zsym)), z23 = z01;
        if (!a.sym) {
            const uint2 zz = *reinterpret_cast<const uint2 *>(kzp + 8 * quad);
            z01 = make_float2(static_cast<float>(static_cast<int16_t>(zz.x & 0xffffu)),
                              static_cast<float>(static_cast<int16_t>(zz.x >> 16)));
            z23 = make_float2(static_cast<float>(static_cast<int16_t>(zz.y & 0xffffu)),
                              static_cast<float>(static_cast<int16_t>(zz.y >> 16)));
        }
        // the bias scale 2^(-64 + 2nc) (exact) folded into the zeros: bp is the scaled partial
        z01 = mul2(z01, make_float2(pbias_f, pbias_f));
        z23 = mul2(z23, make_float2(pbias_f, pbias_f));
        float bp[HPL];
        __syncwarp();   // the previous group's fragments have been read
#pragma unroll
        for (int i = 0; i < HPL; ++i) {
            const float4 q4 = *reinterpret_cast<const float4 *>(&qm_s[hp0 + i][4 * quad]);
            const float2 x01 = mul2(make_float2(q4.x, q4.y), make_float2(s4.x, s4.y));
            const float2 x23 = mul2(make_float2(q4.z, q4.w), make_float2(s4.z, s4.w));
            const float2 bb = fma2(x01, z01, mul2(x23, z23));
            bp[i] = bb.x + bb.y;
            // b0 = channels (4 quad, 4 quad + 2), b1 = (4 quad + 1, 4 quad + 3); chunk quad / 4,
            // column t4 of the consumers = quad mod 4
            const float2 t01 = make_float2(__uint_as_float(__float_as_uint(x01.x) & 0xffff0000u),
                                           __uint_as_float(__float_as_uint(x01.y) & 0xffff0000u));
            const float2 t23 = make_float2(__uint_as_float(__float_as_uint(x23.x) & 0xffff0000u),
                                           __uint_as_float(__float_as_uint(x23.y) & 0xffff0000u));
            const float2 r01 = sub2(x01, t01);
            const float2 r23 = sub2(x23, t23);
            uint32_t *row = kbs + (hp0 + i) * 4 * L::RS + (quad & 3) * L::RS + 2 * (quad >> 2);
            *reinterpret_cast<uint2 *>(row) = make_uint2(bf16_trunc2(x01.x, x23.x), bf16_trunc2(x01.y, x23.y));
            *reinterpret_cast<uint2 *>(row + L::PS) = make_uint2(f2bf2(r01.x, r23.x), f2bf2(r01.y, r23.y));
        }
        __syncwarp();
        const uint32_t *src = kbs + kb_row;
#pragma unroll
        for (int i = 0; i < NJ / 2; ++i) {
            const uint4 v = *reinterpret_cast<const uint4 *>(src + 4 * i);
            kb[2 * i][0] = v.x; kb[2 * i][1] = v.y; kb[2 * i + 1][0] = v.z; kb[2 * i + 1][1] = v.w;
        }
        // bias of each head: the producers' partials summed over the QUADS lanes of its quads
        const float bsum = transpose_reduce<HPL, QUADS>(bp, lane);
        // head t4 mod HG: in the lane group of heads (h / HPL), at lane offset (h mod HPL) QUADS / HPL
        const int hh = t4 % HG;
        kbias = __shfl_sync(0xffffffffu, bsum, (hh / HPL) * QUADS + (hh % HPL) * (QUADS / HPL));
        __syncwarp();   // the staging is read before the value phase reuses its memory
    };

    bool skip = false;
    if constexpr (kCheck) {
        // bounds-check builds: a bounded wait on a barrier nothing arrives at, which gives up
        // (kvq_debug_set_stall); the warp then follows the rounds without doing their work
        __shared__ uint64_t stall_bar;
        if (a.stall_polls > 0 && hk == 0 && b == 0 && sigma == 0 && warp == 0) {
            if (lane == 0) {
                mbar_init(&stall_bar, 1);
                fence_mbar_init();
            }
            __syncwarp();
            bool done = false;
            for (int i = 0; i < a.stall_polls && !done; ++i) done = mbar_try_wait(&stall_bar, 0);
            if (!__all_sync(0xffffffffu, done)) {
                if (lane == 0) atomicOr(a.status, 1u);
                skip = true;
            }
            __syncwarp();
            if (lane == 0) mbar_inval(&stall_bar);
        }
    }

    // RR: round j is issued by warp j mod kDecodeWarps, else by the ring's warp; rounds
    // 0 .. kSt - 2 now, round r + kSt - 1 while round r is consumed
    const int n_loop = RR ? n_rounds : my_items;   // the rounds this warp takes part in
    int my_last = -1;   // the last round this warp issued
#pragma unroll
    for (int j = 0; j < kSt - 1; ++j) {
        if (j < n_loop && (!RR || j == warp)) {
            issue_round(j);
            my_last = j;
        }
    }
    int g_cur = -1;     // key group of the fragments in kb
    bool failed = false;
    int r = 0;
    for (; r < n_loop; ++r) {
        const int rn = r + kSt - 1;
        if (rn < n_loop && (!RR || rn % kDecodeWarps == warp)) {
            // RR: the stage's previous round, rn - kSt, must have been released by every warp
            if (RR && rn >= kSt &&
                !warp_wait(s_empty0 + 8u * static_cast<uint32_t>(rn % kSt), static_cast<uint32_t>(rn / kSt - 1) & 1u)) {
                failed = true;
                break;
            }
            issue_round(rn);
            my_last = rn;
        }
        const uint32_t slot = static_cast<uint32_t>(r % kSt);
        if (!warp_wait(s_full0 + 8u * slot, static_cast<uint32_t>(r / kSt) & 1u)) {
            failed = true;
            break;
        }
        const int item = item_of(r);
        if (item < n_items && !skip) {
        const unsigned char *st = stage_mem + (ring * kSt + slot) * L::kStage;
            const int ti = t_begin + item * kMmaItemTiles;   // unit-local tile of the item
            if ((ti >> a.gshift) != g_cur) {
                g_cur = ti >> a.gshift;
                // the group's slot: its place among the round's groups, or the warp's own slot
                const int gi = RR ? g_cur - ((t_begin + r * kDecodeWarps * kMmaItemTiles) >> a.gshift) : 0;
                build_key_b(st + L::kRks + gi * (D * 4), st + L::kRkz + gi * (D * 2));
            }
            const int is = RR ? warp : 0;   // the item's place in the stage
            const unsigned char *kcp = st + L::kRk + is * L::kItemCodes;
            const unsigned char *vcp = st + L::kRv + is * L::kItemCodes;
            const float *vsp = reinterpret_cast<const float *>(st + L::kRvs + is * L::kItemVs);
            const int16_t *vzp = reinterpret_cast<const int16_t *>(st + L::kRvz + is * (L::kItemVs / 2));

            // ---- keys: log2-domain logits of head t4 mod HG, tokens g8 and g8 + 8 of each tile ----
            float lg[kMmaItemTiles][2];
#pragma unroll
            for (int u = 0; u < kMmaItemTiles; ++u) {
                uint32_t kw[W];
                load_lane_words<W>(kcp + u * TW * 4, lane, kw);
                float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
                for (int wi = 0; wi < W; ++wi) {
                    const uint32_t w02 = kw[wi], w13 = kw[wi] >> 8;
#pragma unroll
                    for (int c = 0; c < BPW; ++c) {
                        const int j = wi * BPW + c;
                        const uint32_t m0 = HALF_L << (N * 2 * c), m1 = HALF_L << (N * (2 * c + 1));
                        hmma(acc[wi & 1], w02 & m0, w02 & m1, w13 & m0, w13 & m1, kb[j][0], kb[j][1]);
                    }
                }
                constexpr float f0 = static_cast<float>(1ull << 62) * 128.0f;                       // 2^69
                constexpr float f1 = static_cast<float>(1ull << 62) * static_cast<float>(128 >> N); // 2^(69 - n)
                // rows g8 (.x) and g8 + 8 (.y): (chain 0 + chain 1), column 2 t4 plus column 2 t4 + 1
                const float2 c0 = add2(make_float2(acc[0][0], acc[0][2]), make_float2(acc[1][0], acc[1][2]));
                const float2 c1 = add2(make_float2(acc[0][1], acc[0][3]), make_float2(acc[1][1], acc[1][3]));
                const float2 cs = add2(c0, c1);
                lg[u][0] = fmaf(cs.x, f0, -kbias);
                lg[u][1] = fmaf(cs.y, f1, -kbias);
            }

            // ---- online softmax of head t4 mod HG: the item's maximum, rescale, p ----
            {
                float mx = fmaxf(fmaxf(lg[0][0], lg[0][1]), fmaxf(lg[1][0], lg[1][1]));
                // lazily: only when a logit of the item passes the running maximum by more than
                // kLazyRescale (p may reach 2^kLazyRescale meanwhile), so rescales stay rare;
                // the lanes of a head (same t4) agree on m_own, so any lane's logit decides
                if (__any_sync(0xffffffffu, mx > m_own + kLazyRescale)) {
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));   // the item's maximum of the head
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                    const float mn = fmaxf(m_own, mx);
                    const float alpha = fast_exp2(m_own - mn);
                    m_own = mn;
#pragma unroll
                    for (int j = 0; j < NJ; ++j) {
                        dv[j][0] *= alpha; dv[j][1] *= alpha; dv[j][2] *= alpha; dv[j][3] *= alpha;
                    }
                    lsum *= alpha;
                    const float ab = __shfl_sync(0xffffffffu, alpha, hb);   // lane hb holds head hb
#pragma unroll
                    for (int v = 0; v < NGV; ++v) zsum[v] *= ab;
                }
            }
            // p 2^80 = 2^(logit - (m - 80)): the value MMA's scale comes with the exponential
            const float m80 = m_own - static_cast<float>(kValScaleLog2);
            if (HG == 4 || t4 < HG) {
#pragma unroll
                for (int u = 0; u < kMmaItemTiles; ++u) {
                    const float p0 = fast_exp2(lg[u][0] - m80), p1 = fast_exp2(lg[u][1] - m80);
                    lsum += p0 + p1;
                    pb[(u * HG + t4) * 18 + logit_pos(g8)] = p0;
                    pb[(u * HG + t4) * 18 + logit_pos(g8 + 8)] = p1;
                }
            }
            // value meta of the item: lane l computes s z of token l for every value group
            float *uv = reinterpret_cast<float *>(wmem + L::kUv);
            {
                float sv[NGV];
                int16_t zv[NGV];
                load_meta<NGV>(vsp + lane * NGV, vzp + lane * NGV, a.sym, zsym, sv, zv);
                float uz[NGV];
#pragma unroll
                for (int v = 0; v < NGV; ++v) uz[v] = sv[v] * static_cast<float>(zv[v]);
                store_vec<NGV>(uv + lane * NGV, uz);
            }
            __syncwarp();

            // ---- values: B = p s 2^80 of head hb; lane (g8, t4) builds both parts for tokens
            //      te, te + 2 of a tile (the k pair of B register e) and trades halves with
            //      lane g8 ^ 1 ----
#pragma unroll
            for (int u = 0; u < kMmaItemTiles; ++u) {
                const float2 pp = *reinterpret_cast<const float2 *>(pb + (u * HG + hb) * 18 + 4 * t4 + 2 * e);
                float s0[NGV], s1[NGV], u0[NGV], u1[NGV];
                const int r0 = 16 * u + te, r1 = r0 + 2;
                load_vec<NGV>(vsp + r0 * NGV, s0);
                load_vec<NGV>(vsp + r1 * NGV, s1);
                load_vec<NGV>(uv + r0 * NGV, u0);
                load_vec<NGV>(uv + r1 * NGV, u1);
                uint32_t hi[NGV], lo[NGV];
                if constexpr (NGV % 2 == 0) {
                    // packed over value-group pairs: (ps0[v], ps0[v + 1]), (ps1[v], ps1[v + 1])
#pragma unroll
                    for (int v = 0; v < NGV; v += 2) {
                        const float2 a0 = mul2(make_float2(pp.x, pp.x), make_float2(s0[v], s0[v + 1]));
                        const float2 a1 = mul2(make_float2(pp.y, pp.y), make_float2(s1[v], s1[v + 1]));
                        float2 zz = fma2(make_float2(pp.x, pp.x), make_float2(u0[v], u0[v + 1]),
                                         make_float2(zsum[v], zsum[v + 1]));
                        zz = fma2(make_float2(pp.y, pp.y), make_float2(u1[v], u1[v + 1]), zz);
                        zsum[v] = zz.x;
                        zsum[v + 1] = zz.y;
                        const float2 t0 = make_float2(__uint_as_float(__float_as_uint(a0.x) & 0xffff0000u),
                                                      __uint_as_float(__float_as_uint(a0.y) & 0xffff0000u));
                        const float2 t1 = make_float2(__uint_as_float(__float_as_uint(a1.x) & 0xffff0000u),
                                                      __uint_as_float(__float_as_uint(a1.y) & 0xffff0000u));
                        const float2 r0 = sub2(a0, t0), r1 = sub2(a1, t1);
                        hi[v] = bf16_trunc2(a0.x, a1.x);
                        hi[v + 1] = bf16_trunc2(a0.y, a1.y);
                        lo[v] = f2bf2(r0.x, r1.x);
                        lo[v + 1] = f2bf2(r0.y, r1.y);
                    }
                } else {
#pragma unroll
                    for (int v = 0; v < NGV; ++v) {
                        const float ps0 = pp.x * s0[v], ps1 = pp.y * s1[v];
                        zsum[v] = fmaf(pp.x, u0[v], fmaf(pp.y, u1[v], zsum[v]));
                        hi[v] = bf16_trunc2(ps0, ps1);
                        lo[v] = bf16_rem2(ps0, ps1);
                    }
                }
                uint32_t B0[NGV], B1[NGV];
                if constexpr (NGV >= 4) {
                    // through shared memory: [part][head][t4][e][v]; this lane's B0 is part e of
                    // tokens (4 t4, 4 t4 + 2) (e = 0 row), B1 part e of (4 t4 + 1, 4 t4 + 3)
                    uint32_t *vx = reinterpret_cast<uint32_t *>(wmem + L::kVx);
                    uint32_t *mine = vx + ((hb * 4 + t4) * 2 + e) * NGV;
                    store_vec<NGV>(mine, hi);
                    store_vec<NGV>(mine + L::VXS, lo);
                    __syncwarp();
                    const uint32_t *part = vx + e * L::VXS + (hb * 4 + t4) * 2 * NGV;
                    load_vec<NGV>(part, B0);
                    load_vec<NGV>(part + NGV, B1);
                } else {
#pragma unroll
                    for (int v = 0; v < NGV; ++v) {
                        const uint32_t y = __shfl_xor_sync(0xffffffffu, e ? hi[v] : lo[v], 4);
                        B0[v] = e ? y : hi[v];
                        B1[v] = e ? lo[v] : y;
                    }
                }
                uint32_t vw[W];
                load_lane_words<W>(vcp + u * TW * 4, lane, vw);
#pragma unroll
                for (int wi = 0; wi < W; ++wi) {
                    const uint32_t w02 = vw[wi], w13 = vw[wi] >> 8;
#pragma unroll
                    for (int c = 0; c < BPW; ++c) {
                        const int j = wi * BPW + c;
                        const uint32_t m0 = HALF_L << (N * 2 * c), m1 = HALF_L << (N * (2 * c + 1));
                        hmma(dv[j], w02 & m0, w02 & m1, w13 & m0, w13 & m1, B0[(16 * j) / GV], B1[(16 * j) / GV]);
                    }
                }
                if constexpr (NGV >= 4) __syncwarp();   // the exchange is read before the next tile writes it
            }
        }
        __syncwarp();   // the warp's reads of the stage and its scratch are done
        if (RR && lane == 0) mbar_arrive_u32(s_empty0 + 8u * slot);
    }
    if (failed) {
        // an abandoned wait: the status word says so; the copies this warp issued for rounds
        // it has not waited for get their (bounded) time to land before the CTA exits
        if (lane == 0) atomicOr(a.status, 1u);
        for (int j = r; j <= my_last; ++j)
            if (!RR || j % kDecodeWarps == warp)
                mbar_wait_bounded(rbar + ring * kSt + j % kSt, static_cast<uint32_t>(j / kSt) & 1u);
        __syncwarp();
    }

    // ---- warp epilogue (lsum and zsum carry the factor 2^80 of p) ----
    constexpr float kUnB = 1.0f / (static_cast<float>(1ull << 40) * static_cast<float>(1ull << 40));   // 2^-80
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 4);
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 8);
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 16);
    lsum *= kUnB;
#pragma unroll
    for (int o = 1; o <= 4; o <<= 1) {
#pragma unroll
        for (int v = 0; v < NGV; ++v) zsum[v] += __shfl_xor_sync(0xffffffffu, zsum[v], o);
    }
    const int hown = t4 % HG;
    float z_own[NGV];
#pragma unroll
    for (int v = 0; v < NGV; ++v) z_own[v] = __shfl_sync(0xffffffffu, zsum[v], 8 * hown) * kUnB;
    // dv sums code 2^(n slot) 2^-133 p s 2^80 = 2^(n slot - 53) p s code
    float ov[NJ][2];
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
        const int s0 = 2 * (j % BPW);
        const float f0 = __uint_as_float(static_cast<uint32_t>(127 + 53 - N * s0) << 23);
        const float f1 = __uint_as_float(static_cast<uint32_t>(127 + 53 - N * (s0 + 1)) << 23);
        ov[j][0] = (dv[j][0] + dv[j][1]) * f0 - z_own[(16 * j) / GV];
        ov[j][1] = (dv[j][2] + dv[j][3]) * f1 - z_own[(16 * j) / GV];
    }

    __syncthreads();   // stage memory is reused for the per-warp outputs
    if (t4 < HG) {
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
            o_s[(warp * HG + t4) * D + 16 * j + g8] = ov[j][0];
            o_s[(warp * HG + t4) * D + 16 * j + g8 + 8] = ov[j][1];
        }
        if (g8 == 0) {
            ml_s[warp][t4][0] = m_own;
            ml_s[warp][t4][1] = lsum;
        }
    }
    __syncthreads();
    finish_cta<HG, D>(a, o_s, ml_s, bh, bq0, sigma, &last_s, o_s + kDecodeWarps * HG * D);
}

// the round-robin instance for key groups of 2 tiles, else the per-warp rings
template <int N, int D, int GV, int HG>
cudaError_t launch_mma(const DecodeArgs &a, cudaStream_t s) {
    if (a.gshift == 1)
        return launch_kernel<decode_mma_kernel<N, D, GV, HG, true>>(a, dim3(a.Hkv, a.B, a.S),
                                                                      mma_smem<N, D, GV, HG, true>(), s);
    return launch_kernel<decode_mma_kernel<N, D, GV, HG, false>>(a, dim3(a.Hkv, a.B, a.S),
                                                                   mma_smem<N, D, GV, HG, false>(), s);
}
template <int N, int D, int GV, int HG>
int occ_mma(const DecodeArgs &a) {
    if (a.gshift == 1) return occupancy_of<decode_mma_kernel<N, D, GV, HG, true>>(mma_smem<N, D, GV, HG, true>());
    return occupancy_of<decode_mma_kernel<N, D, GV, HG, false>>(mma_smem<N, D, GV, HG, false>());
}

template <int N, int D, int GV>
cudaError_t launch_mma_hg(const DecodeArgs &a, cudaStream_t s, bool occ_only, int *occ) {
    switch (a.Hq / a.Hkv) {
        case 1: if (occ_only) { *occ = occ_mma<N, D, GV, 1>(a); return cudaSuccess; } return launch_mma<N, D, GV, 1>(a, s);
        case 2: if (occ_only) { *occ = occ_mma<N, D, GV, 2>(a); return cudaSuccess; } return launch_mma<N, D, GV, 2>(a, s);
        case 4: if (occ_only) { *occ = occ_mma<N, D, GV, 4>(a); return cudaSuccess; } return launch_mma<N, D, GV, 4>(a, s);
        default: return cudaErrorInvalidValue;
    }
}

template <int N, int D>
cudaError_t launch_mma_gv(const DecodeArgs &a, cudaStream_t s, bool occ_only, int *occ) {
    switch (a.Gv) {
        case 16: return launch_mma_hg<N, D, 16>(a, s, occ_only, occ);
        case 32: return launch_mma_hg<N, D, 32>(a, s, occ_only, occ);
        case 64: return launch_mma_hg<N, D, 64>(a, s, occ_only, occ);
        default:
            if constexpr (D >= 128) {
                if (a.Gv == 128) return launch_mma_hg<N, D, 128>(a, s, occ_only, occ);
            }
    }
    return cudaErrorInvalidValue;
}

// Launch (or, with occ_only, the CTAs per SM of) the kernel serving a's geometry.
cudaError_t launch_mma_any(const DecodeArgs &a, cudaStream_t s, bool occ_only, int *occ) {
    if (a.bits == 2 && a.d == 64) return launch_mma_gv<2, 64>(a, s, occ_only, occ);
    if (a.bits == 2 && a.d == 128) return launch_mma_gv<2, 128>(a, s, occ_only, occ);
    if (a.bits == 4 && a.d == 64) return launch_mma_gv<4, 64>(a, s, occ_only, occ);
    if (a.bits == 4 && a.d == 128) return launch_mma_gv<4, 128>(a, s, occ_only, occ);
    return cudaErrorInvalidValue;
}

}  // namespace
}  // namespace kvq
