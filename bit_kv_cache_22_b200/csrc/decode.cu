// decode.cu -- split-K decode attention over the packed low-bit cache (CUDA cores).
//
// Computes, for every (batch, query head), one decode step of
//   A = softmax(q [deq(K_g); K_r]^T / sqrt(d)),   t_O = A [deq(V_g); V_r]
// ("LLM系列：KVCache量化1 KIVI ...", section 1: A = Concat(A_g, A_r), t_O = A X_V;
//  the 1/sqrt(d_k) of "KV Cache的Int4量化…" section 3), with deq(x) = (code - z) s.
//
// Split-K (flash-decoding): the quantized 16-token tiles are divided into
// contiguous splits and the residual rows, cut into 16-row tiles, form one more
// split of their own (they are read unstaged, so they run beside the others
// instead of lengthening one of them); a CTA owns one (batch, query head,
// split) and each of its four warps a contiguous share of the split's tiles,
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
            a.out[bq * D + c] = o / l;
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
    for (int i = threadIdx.x; i < HG * D; i += kDecodeThreads) {
        const int hh = i / D, c = i % D;
        const float *op = a.o_part + (bq0 + hh) * a.S * D + c;
        const float *wp = wts + hh * a.S;
        float o = 0.f;
#pragma unroll 8
        for (int s = 0; s < a.S; ++s) o = fmaf(__ldcg(op + static_cast<int64_t>(s) * D), wp[s], o);
        a.out[(bq0 + hh) * D + c] = o / wts[HG * a.S + hh];
    }
    if (threadIdx.x == 0) a.arrivals[unit] = 0u;
}

template <int N, int D, int GV>
__global__ void __launch_bounds__(kDecodeThreads, 4) decode_split_kernel(const DecodeArgs a) {
    constexpr int W = D * N / 64;     // words per lane per tile
    constexpr int TW = D * N / 2;     // words per tile
    constexpr int NJ = D / 16;        // 16-channel chunks
    constexpr int BPW = 4 / N;        // chunks per word
    constexpr int SLOTS = 2 * BPW;    // byte groups per word
    constexpr int NGV = D / GV;       // value groups per token
    constexpr uint32_t BYTE_MASK = ((1u << N) - 1u) * 0x01010101u;
    using St = Stage<N, D, GV>;

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
    const int total_tiles = a.n_qtiles + (a.r + 15) / 16;
    const int t_begin = sigma < a.n_qsplits ? sigma * a.tiles_per_split : a.n_qtiles;
    const int t_end = sigma < a.n_qsplits ? min(a.n_qtiles, t_begin + a.tiles_per_split) : total_tiles;
    const int per_w = (t_end - t_begin + kDecodeWarps - 1) / kDecodeWarps;
    const int wb = t_begin + warp * per_w;
    const int we = min(t_end, wb + per_w);
    const int qe = min(we, a.n_qtiles);
    const int64_t groups_cap = a.cap / a.G;
    const uint32_t *kc = a.kc + bh * (a.cap / 16) * TW;
    const uint32_t *vc = a.vc + bh * (a.cap / 16) * TW;
    const float *vs_g = a.vs + bh * a.cap * NGV;
    const int16_t *vz_g = a.vz + bh * a.cap * NGV;
    const int zsym = 1 << (N - 1);
    const int gmask = (1 << a.gshift) - 1;   // tiles per key group - 1

    // producer: stage the tile's lane segments, value meta and (at a group start) key meta
    auto issue = [&](int ti) {
        if (ti >= qe) return;
        unsigned char *st = wmem + ((ti - wb) % kStages) * St::kBytes;
        const uint32_t *ksrc = kc + static_cast<int64_t>(ti) * TW + lane * W;
        const uint32_t *vsrc = vc + static_cast<int64_t>(ti) * TW + lane * W;
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
        const int64_t tok0 = static_cast<int64_t>(ti) * 16;
        for (int c = lane; c < NGV * 4; c += 32)
            cp_async16(st + St::kVs + 16 * c, vs_g + tok0 * NGV + 4 * c);
        if (!a.sym)
            for (int c = lane; c < NGV * 2; c += 32)
                cp_async16(st + St::kVz + 16 * c, vz_g + tok0 * NGV + 8 * c);
        if (ti == wb || (ti & gmask) == 0) {
            const int64_t gofs = (bh * groups_cap + (ti >> a.gshift)) * D;
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
        const bool quant = ti < a.n_qtiles;
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
            const int row0 = (ti - a.n_qtiles) * 16 + g8, row1 = row0 + 8;
            float x0 = 0.f, x1 = 0.f;
            const uint16_t *kr = a.kr + bh * a.R * D;
#pragma unroll
            for (int j = 0; j < NJ; ++j) {
                const int c0 = 16 * j + 4 * t4;
                const float4 qq = *reinterpret_cast<const float4 *>(q_s + c0);
                if (row0 < a.r) {
                    const uint2 kk = *reinterpret_cast<const uint2 *>(kr + row0 * D + c0);
                    x0 = fmaf(qq.x, widen(kk.x & 0xffffu, a.bf16), x0);
                    x0 = fmaf(qq.y, widen(kk.x >> 16, a.bf16), x0);
                    x0 = fmaf(qq.z, widen(kk.y & 0xffffu, a.bf16), x0);
                    x0 = fmaf(qq.w, widen(kk.y >> 16, a.bf16), x0);
                }
                if (row1 < a.r) {
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
            lg0 = row0 < a.r ? x0 : -INFINITY;
            lg1 = row1 < a.r ? x1 : -INFINITY;
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
            const int ra = (ti - a.n_qtiles) * 16 + 4 * t4;
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
                        vv[i] = (ra + i < a.r) ? pt[i] * widen(vr[(ra + i) * D + c], a.bf16) : 0.f;
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
// of one query head (16 rows each; rows >= r masked) with the exact e values on
// CUDA cores.  Each tile's K and V rows are first staged in `scratch`
// (residual_scratch_bytes<D>() bytes of this warp's shared memory) with
// coalesced cp.async; the caller must have no cp.async group of its own
// pending.  qh is the log2-scaled query in shared memory; acc[j][h] accumulates
// channel 16j + g8 + 8h, x over tokens 4*t4 + {0, 1}, y over 4*t4 + {2, 3}.
template <int D>
__device__ __forceinline__ void residual_pass(const DecodeArgs &a, const float *qh, const uint16_t *kr,
                                              const uint16_t *vr, int rt0, int rt1, int lane, float &m,
                                              float &lsum, float2 (&acc)[D / 16][2], unsigned char *scratch,
                                              int stride = 1) {
    constexpr int NJ = D / 16;
    constexpr int kRow = 2 * D + 16;          // padded row stride in bytes
    constexpr int kPieces = 2 * D / 16;       // 16-byte pieces of one row
    const int g8 = lane >> 2, t4 = lane & 3;
    unsigned char *ks = scratch, *vs = scratch + 16 * kRow;
    for (int rt = rt0; rt < rt1; rt += stride) {
        const int rows = min(16, a.r - 16 * rt);
        const int n = rows * kPieces;
        __syncwarp();   // the previous tile's rows have been read
        for (int c = lane; c < 2 * n; c += 32) {
            const bool isv = c >= n;
            const int cc = isv ? c - n : c, row = cc / kPieces, pc = cc % kPieces;
            cp_async16((isv ? vs : ks) + row * kRow + 16 * pc,
                       (isv ? vr : kr) + (static_cast<int64_t>(rt) * 16 + row) * D + 8 * pc);
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
// Grouped-query heads (4 query heads per kv head): tensor-core path.
//
// A CTA owns one (batch, kv head, split) and serves the 4 query heads that read
// that kv head, so every code is fetched and unpacked once for all of them.
// Lane = 4*g8 + t4; query head t4 is "owned" by the lanes with that t4.
//   keys   : int8 MMA m16n8k32.  A = the byte-masked key codes (rows = tokens,
//            k = channels) exactly as stored; B = byte digits of the 21-bit
//            fixed-point multipliers q_c s_{g,c} log2(e)/sqrt(d) (exponent per
//            key group and head), columns 2h+d (digits 0, 1 of head h) in the
//            first n-tile and 2h (signed digit 2) in the second; int32 sums,
//            exact.  The digits are built once per key group, cooperatively by
//            the warp (lane l: head l/8, 16 channels), in shared memory.
//   values : bf16 MMA m16n8k16.  A = value codes as exact bf16 (rows = channels,
//            k = tokens; bytes 0,2 and 1,3 of a word slot are bf16x2 pairs via
//            the 0x4300 exponent trick); B = p_t s_{t,gv} split into bf16 hi +
//            lo parts (columns 2h, 2h+1; bf16 keeps fp32's exponent range, so
//            the tiny probabilities of long contexts do not underflow), built
//            cooperatively per tile; fp32 accumulators, rescaled when a head's
//            running maximum grows.
//   z-terms: bias_g = sum_c q'_c z_{g,c} and sum_t p_t s_t z_t in fp32.
// Residual rows form the last split, where each warp serves one query head
// with exact e values on CUDA cores.
// ---------------------------------------------------------------------------
constexpr int kGqa = 4;

__device__ __forceinline__ void imma_uu(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
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

// Codes of one slot of a value word as two bf16x2 registers, (byte 0, byte 2)
// and (byte 1, byte 3), each element equal to 2^(7-N) * (2^N + code) exactly:
// the code is shifted to the top N mantissa bits of 0x4300 (bf16 128, unit
// mantissa steps).  The 2^N offset is small next to the code range, so it is
// kept: the value MMA accumulates sum_t b_t (2^N + code) and the z-term uses
// z + 2^N instead of z; the 2^(7-N) factor is folded into the B operand.
template <int N>
__device__ __forceinline__ void codes_bf16(uint32_t w, int slot, uint32_t magic16, uint32_t &r02,
                                           uint32_t &r13) {
    constexpr uint32_t L = (1u << N) - 1u;
    constexpr uint32_t M = (L << (7 - N)) | (L << (23 - N));
    const int up = 7 - N - N * slot;                  // byte 0/2 code: bit N*slot -> 7 - N
    const uint32_t x02 = up >= 0 ? (w << up) : (w >> -up);
    const uint32_t x13 = w >> (N * slot + N + 1);     // byte 1/3 code: bit 8 + N*slot -> 7 - N
    r02 = and_or(x02, M, magic16);
    r13 = and_or(x13, M, magic16);
}

// Shared-memory stages of the grouped-query kernel (it consumes two tiles per
// iteration, so it keeps a deeper ring when a stage is small).
template <int N>
__host__ __device__ constexpr int gqa_stages() { return N == 2 ? 6 : 4; }

template <int N, int D, int GV>
struct GqaSmem {
    static constexpr int NGV = D / GV;
    static constexpr int kStageBytes = gqa_stages<N>() * Stage<N, D, GV>::kBytes;
    static constexpr int kKdRow = D + 16;                    // padded: the 8 B-fragment rows hit distinct banks
    static constexpr int kKd = kStageBytes;                  // key digits [3][4 heads][kKdRow] bytes
    static constexpr int kVb = kKd + 3 * kGqa * kKdRow;      // value B [2 tiles][NGV][4][2][16] bf16
    // p [2 tiles][2 token halves][4 heads][8] f32, tokens of a half in (0, 2, 1, 3) order
    // within each 4-group: owners store and builders read (as pairs) without conflicts
    static constexpr int kPs = kVb + 2 * NGV * kGqa * 2 * 16 * 2;
    static constexpr int kAl = kPs + 2 * 2 * kGqa * 8 * 4;   // alpha [4], key scale [4], bias [4]
    static constexpr int kWarpBytes = kAl + 16 * 4;
    static_assert(kKd % 16 == 0 && kVb % 16 == 0 && kPs % 16 == 0 && kAl % 16 == 0, "align");
};

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

template <int N, int D, int GV>
__global__ void __launch_bounds__(kDecodeThreads, 3) decode_gqa_kernel(const DecodeArgs a) {
    constexpr int W = D * N / 64;
    constexpr int TW = D * N / 2;
    constexpr int NJ = D / 16;
    constexpr int NK = D / 32;        // k32 steps of the key MMA
    constexpr int BPW = 4 / N;
    constexpr int NGV = D / GV;
    constexpr uint32_t BYTE_MASK = ((1u << N) - 1u) * 0x01010101u;
    using St = Stage<N, D, GV>;
    using Sm = GqaSmem<N, D, GV>;
    constexpr int kGqaStages = gqa_stages<N>();

    __shared__ __align__(16) float q_s[kGqa][D];
    __shared__ float ml_s[kDecodeWarps][kGqa][2];
    __shared__ int last_s;
    extern __shared__ __align__(128) unsigned char stage_mem[];

    const int hk = blockIdx.x, b = blockIdx.y, sigma = blockIdx.z;
    const int64_t bh = static_cast<int64_t>(b) * a.Hkv + hk;
    const int64_t bq0 = static_cast<int64_t>(b) * a.Hq + hk * kGqa;   // first query head
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g8 = lane >> 2, t4 = lane & 3;
    unsigned char *wmem = stage_mem + static_cast<size_t>(warp) * Sm::kWarpBytes;
    uint8_t *kd = wmem + Sm::kKd;
    uint16_t *vb = reinterpret_cast<uint16_t *>(wmem + Sm::kVb);
    float *ps = reinterpret_cast<float *>(wmem + Sm::kPs);
    float *al = reinterpret_cast<float *>(wmem + Sm::kAl);
    const uint32_t magic = kMagicBits;
    const uint32_t magic16 = 0x43004300u;    // bf16 128 in both halves

    for (int i = threadIdx.x; i < kGqa * D; i += kDecodeThreads)
        q_s[i / D][i % D] = widen(a.q[bq0 * D + i], a.bf16) * a.qscale;
    __syncthreads();

    const int total_tiles = a.n_qtiles + (a.r + 15) / 16;
    const int zsym = 1 << (N - 1);

    if (sigma >= a.n_qsplits) {
        // ---------------- residual split: warp = query head ----------------
        const float *qh = q_s[warp];
        float m = -INFINITY, lsum = 0.f;
        float2 acc[NJ][2];
#pragma unroll
        for (int j = 0; j < NJ; ++j) acc[j][0] = acc[j][1] = make_float2(0.f, 0.f);
        residual_pass<D>(a, qh, a.kr + bh * a.R * D, a.vr + bh * a.R * D, 0, total_tiles - a.n_qtiles,
                         lane, m, lsum, acc, wmem);
        lsum += __shfl_xor_sync(0xffffffffu, lsum, 4);
        lsum += __shfl_xor_sync(0xffffffffu, lsum, 8);
        lsum += __shfl_xor_sync(0xffffffffu, lsum, 16);
        static_assert(residual_scratch_bytes<D>() <= Sm::kWarpBytes, "residual staging");
        __syncthreads();   // every warp is done with its staged rows before o_s overwrites them
        float *o_s = reinterpret_cast<float *>(stage_mem);   // [warp][head][D]; only head == warp
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float val = acc[j][h].x + acc[j][h].y;
                val += __shfl_xor_sync(0xffffffffu, val, 1);
                val += __shfl_xor_sync(0xffffffffu, val, 2);
                if (t4 == 0) o_s[(warp * kGqa + warp) * D + 16 * j + g8 + 8 * h] = val;
            }
        }
        if (lane < kGqa) {
            ml_s[warp][lane][0] = lane == warp ? m : -INFINITY;
            ml_s[warp][lane][1] = lane == warp ? lsum : 0.f;
        }
        __syncthreads();
        finish_cta<kGqa, D>(a, o_s, ml_s, bh, bq0, sigma, &last_s, o_s + kDecodeWarps * kGqa * D);
        return;
    }

    // ---------------- quantized split ----------------
    const int t_begin = sigma * a.tiles_per_split;
    const int t_end = min(a.n_qtiles, t_begin + a.tiles_per_split);
    const int per_w = (t_end - t_begin + kDecodeWarps - 1) / kDecodeWarps;
    const int wb = t_begin + warp * per_w;
    const int we = min(t_end, wb + per_w);
    const int64_t groups_cap = a.cap / a.G;
    const uint32_t *kc = a.kc + bh * (a.cap / 16) * TW;
    const uint32_t *vc = a.vc + bh * (a.cap / 16) * TW;
    const float *vs_g = a.vs + bh * a.cap * NGV;
    const int16_t *vz_g = a.vz + bh * a.cap * NGV;
    const int gmask = (1 << a.gshift) - 1;

    auto issue = [&](int ti) {
        if (ti >= we) return;
        unsigned char *st = wmem + ((ti - wb) % kGqaStages) * St::kBytes;
        const uint32_t *ksrc = kc + static_cast<int64_t>(ti) * TW + lane * W;
        const uint32_t *vsrc = vc + static_cast<int64_t>(ti) * TW + lane * W;
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
        const int64_t tok0 = static_cast<int64_t>(ti) * 16;
        for (int c = lane; c < NGV * 4; c += 32)
            cp_async16(st + St::kVs + 16 * c, vs_g + tok0 * NGV + 4 * c);
        if (!a.sym)
            for (int c = lane; c < NGV * 2; c += 32)
                cp_async16(st + St::kVz + 16 * c, vz_g + tok0 * NGV + 8 * c);
        if (ti == wb || (ti & gmask) == 0) {
            const int64_t gofs = (bh * groups_cap + (ti >> a.gshift)) * D;
            for (int c = lane; c < D / 4; c += 32) cp_async16(st + St::kKs + 16 * c, a.ks + gofs + 4 * c);
            if (!a.sym)
                for (int c = lane; c < D / 8; c += 32) cp_async16(st + St::kKz + 16 * c, a.kz + gofs + 8 * c);
        }
    };

    // owner state (query head t4)
    float m = -INFINITY, lsum = 0.f;
    float dv[NJ][4];                  // value accumulators: channel 16j + g8 (+8), head t4 hi / lo
#pragma unroll
    for (int j = 0; j < NJ; ++j) dv[j][0] = dv[j][1] = dv[j][2] = dv[j][3] = 0.f;
    float kinv = 0.f, kbias = 0.f;
    // builder state (head hb = lane / 8)
    const int hb = lane >> 3, lb = lane & 7;
    float zsum[NGV];
#pragma unroll
    for (int v = 0; v < NGV; ++v) zsum[v] = 0.f;
    // B operands of the key MMA for the current group
    uint32_t kb0[NK][2], kb1[NK][2];

    // Key digits of the group tile `st` opens: lane builds head hb, channels
    // 4*lb + 32*i4 + {0..3}, i4 < D/32 (a quarter-warp reads 128 contiguous bytes).
    auto rebuild_key_digits = [&](const unsigned char *st) {
        const float *ks_s = reinterpret_cast<const float *>(st + St::kKs);
        const int16_t *kz_s = reinterpret_cast<const int16_t *>(st + St::kKz);
        constexpr int NQ = D / 32;
        float qv[4 * NQ];
        float mx = 0.f, kbp = 0.f;
#pragma unroll
        for (int i4 = 0; i4 < NQ; ++i4) {
            const int c0 = 4 * lb + 32 * i4;
            const float4 sc = *reinterpret_cast<const float4 *>(ks_s + c0);
            const float4 qq = *reinterpret_cast<const float4 *>(&q_s[hb][c0]);
            qv[4 * i4 + 0] = qq.x * sc.x; qv[4 * i4 + 1] = qq.y * sc.y;
            qv[4 * i4 + 2] = qq.z * sc.z; qv[4 * i4 + 3] = qq.w * sc.w;
            float z[4] = {static_cast<float>(zsym), static_cast<float>(zsym),
                          static_cast<float>(zsym), static_cast<float>(zsym)};
            if (!a.sym) {
                const uint2 zz = *reinterpret_cast<const uint2 *>(kz_s + c0);
                z[0] = __int2float_rn(static_cast<int16_t>(zz.x & 0xffffu));
                z[1] = __int2float_rn(static_cast<int16_t>(zz.x >> 16));
                z[2] = __int2float_rn(static_cast<int16_t>(zz.y & 0xffffu));
                z[3] = __int2float_rn(static_cast<int16_t>(zz.y >> 16));
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                kbp = fmaf(qv[4 * i4 + i], z[i], kbp);
                mx = fmaxf(mx, fabsf(qv[4 * i4 + i]));
            }
        }
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) {
            kbp += __shfl_xor_sync(0xffffffffu, kbp, o);
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        }
        int e = 0;
        if (mx > 0.f) e = 21 - (static_cast<int>((__float_as_uint(mx) >> 23) & 0xff) - 126);
        e = max(-120, min(120, e));
        const float scale = __uint_as_float(static_cast<uint32_t>(127 + e) << 23);
        uint32_t dw[3][NQ];
#pragma unroll
        for (int i4 = 0; i4 < NQ; ++i4) {
            const int Q0 = round_small(qv[4 * i4 + 0] * scale), Q1 = round_small(qv[4 * i4 + 1] * scale);
            const int Q2 = round_small(qv[4 * i4 + 2] * scale), Q3 = round_small(qv[4 * i4 + 3] * scale);
#pragma unroll
            for (int k = 0; k < 3; ++k) {
                const uint32_t sel = static_cast<uint32_t>(k | ((k + 4) << 4));
                dw[k][i4] = __byte_perm(__byte_perm(Q0, Q1, sel), __byte_perm(Q2, Q3, sel), 0x5410);
            }
        }
        __syncwarp();   // the previous group's digits have been read into registers
#pragma unroll
        for (int k = 0; k < 3; ++k)
#pragma unroll
            for (int i4 = 0; i4 < NQ; ++i4)
                reinterpret_cast<uint32_t *>(kd + (k * kGqa + hb) * Sm::kKdRow)[lb + 8 * i4] = dw[k][i4];
        if (lb == 0) {
            al[4 + hb] = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
            al[8 + hb] = kbp;
        }
        __syncwarp();
        // B fragments: column g8 = head g8/2, digit g8%2 (first n-tile), digit 2 for even g8
        const uint32_t *kdw0 =
            reinterpret_cast<const uint32_t *>(kd + ((g8 & 1) * kGqa + (g8 >> 1)) * Sm::kKdRow);
        const uint32_t *kdw2 = reinterpret_cast<const uint32_t *>(kd + (2 * kGqa + (g8 >> 1)) * Sm::kKdRow);
#pragma unroll
        for (int mk = 0; mk < NK; ++mk) {
            kb0[mk][0] = kdw0[8 * mk + t4];
            kb0[mk][1] = kdw0[8 * mk + 4 + t4];
            kb1[mk][0] = (g8 & 1) ? 0u : kdw2[8 * mk + t4];
            kb1[mk][1] = (g8 & 1) ? 0u : kdw2[8 * mk + 4 + t4];
        }
        kinv = al[4 + t4];
        kbias = al[8 + t4];
    };

#pragma unroll
    for (int s = 0; s < kGqaStages - 2; ++s) {
        issue(wb + s);
        cp_async_commit();
    }

    // two tiles per iteration: their key MMAs, one softmax update and their value MMAs
    // are independent streams of work for the scheduler
    for (int ti = wb; ti < we; ti += 2) {
        const int nt = min(2, we - ti);
        issue(ti + kGqaStages - 2);
        cp_async_commit();
        issue(ti + kGqaStages - 1);
        cp_async_commit();
        cp_async_wait<kGqaStages - 2>();
        __syncwarp();

        // ---- key MMAs: logits of tokens g8, g8 + 8 of both tiles, query head t4 ----
        float lg[2][2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            lg[u][0] = lg[u][1] = -INFINITY;
            if (u < nt) {
                const int t = ti + u;
                const unsigned char *st = wmem + ((t - wb) % kGqaStages) * St::kBytes;
                if (t == wb || (t & gmask) == 0) rebuild_key_digits(st);
                uint32_t kw[W];
                load_stage_words<W>(reinterpret_cast<const uint32_t *>(st), lane, kw);
                int d0[4] = {0, 0, 0, 0}, d1[4] = {0, 0, 0, 0};
#pragma unroll
                for (int mk = 0; mk < NK; ++mk) {
                    uint32_t af[4];
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        const int j = 2 * mk + (r >> 1), half = r & 1;
                        af[r] = (kw[j / BPW] >> (N * (2 * (j % BPW) + half))) & BYTE_MASK;
                    }
                    imma_uu(d0, af, kb0[mk][0], kb0[mk][1]);
                    imma_us(d1, af, kb1[mk][0], kb1[mk][1]);
                }
                lg[u][0] = (small_int_to_float(d0[0]) + 256.f * small_int_to_float(d0[1]) +
                            65536.f * small_int_to_float(d1[0])) * kinv - kbias;
                lg[u][1] = (small_int_to_float(d0[2]) + 256.f * small_int_to_float(d0[3]) +
                            65536.f * small_int_to_float(d1[2])) * kinv - kbias;
            }
        }

        // ---- online softmax of head t4 over both tiles ----
        float tmax = fmaxf(fmaxf(lg[0][0], lg[0][1]), fmaxf(lg[1][0], lg[1][1]));
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 4));
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 8));
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 16));
        const bool grew = tmax > m;
        if (__any_sync(0xffffffffu, grew)) {
            const float alpha = grew ? fast_exp2(m - tmax) : 1.f;
            if (grew) m = tmax;
            lsum *= alpha;
#pragma unroll
            for (int j = 0; j < NJ; ++j) {
                dv[j][0] *= alpha; dv[j][1] *= alpha; dv[j][2] *= alpha; dv[j][3] *= alpha;
            }
            if (g8 == 0) al[t4] = alpha;
            __syncwarp();
            const float ab = al[lane & 3];     // zsum belongs to head lane % 4
#pragma unroll
            for (int v = 0; v < NGV; ++v) zsum[v] *= ab;
        }
        // position of token g8 (and g8 + 8) inside its half: 4-groups in (0, 2, 1, 3) order
        const int ppos = (g8 & 4) + ((g8 & 1) << 1) + ((g8 >> 1) & 1);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const float p0 = fast_exp2(lg[u][0] - m), p1 = fast_exp2(lg[u][1] - m);
            lsum += p0 + p1;
            ps[((u * 2 + 0) * kGqa + t4) * 8 + ppos] = p0;
            ps[((u * 2 + 1) * kGqa + t4) * 8 + ppos] = p1;
        }
        __syncwarp();

        // ---- value B of both tiles: lane l builds head l % 4 for tokens 4q + e and
        //      4q + e + 2, (q, e) = (l / 8, (l / 4) % 2): a quarter-warp covers one token pair
        //      of all four heads (broadcast meta reads, distinct p rows and plane words) ----
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            if (u < nt) {
                const unsigned char *st = wmem + ((ti + u - wb) % kGqaStages) * St::kBytes;
                constexpr float kBscale = 1.0f / static_cast<float>(1 << (7 - N));
                constexpr int kOff = 1 << N;          // code offset carried by the bf16 A operand
                const int hv = lane & 3, q4 = lane >> 3, e = (lane >> 2) & 1;
                const int ta = 4 * q4 + e, tb = ta + 2;
                // tokens ta, tb sit side by side: half q4/2, position 4*(q4%2) + 2e (+1)
                const float2 pr = *reinterpret_cast<const float2 *>(
                    ps + ((u * 2 + (q4 >> 1)) * kGqa + hv) * 8 + 4 * (q4 & 1) + 2 * e);
                const float2 pab = make_float2(pr.x * kBscale, pr.y * kBscale);
                const float *vsp = reinterpret_cast<const float *>(st + St::kVs);
                const int16_t *vzp = reinterpret_cast<const int16_t *>(st + St::kVz);
                float sa[NGV], sb[NGV];
                int16_t zza[NGV], zzb[NGV];
                load_meta<NGV>(vsp + ta * NGV, vzp + ta * NGV, a.sym, zsym, sa, zza);
                load_meta<NGV>(vsp + tb * NGV, vzp + tb * NGV, a.sym, zsym, sb, zzb);
#pragma unroll
                for (int v = 0; v < NGV; ++v) {
                    const float2 x = mul2(pab, make_float2(sa[v], sb[v]));
                    const float2 z = make_float2(__int2float_rn(zza[v] + kOff), __int2float_rn(zzb[v] + kOff));
                    zsum[v] = fmaf(x.x, z.x, fmaf(x.y, z.y, zsum[v]));
                    const uint32_t hi = f2bf2(x.x, x.y);
                    const float2 lof = add2(x, make_float2(-__uint_as_float(hi << 16),
                                                           -__uint_as_float(hi & 0xffff0000u)));
                    const uint32_t lo = f2bf2(lof.x, lof.y);
                    // planes (part p of head h) at sub-block p ^ (h >> 1): conflict-free stores and loads
                    uint32_t *dst = reinterpret_cast<uint32_t *>(vb + (((u * NGV + v) * kGqa + hv) * 2) * 16);
                    dst[((hv >> 1) << 3) + ((4 * q4 + 2 * e) >> 1)] = hi;          // part 0 plane
                    dst[((1 ^ (hv >> 1)) << 3) + ((4 * q4 + 2 * e) >> 1)] = lo;    // part 1 plane
                }
            }
        }
        __syncwarp();

        // ---- value MMAs: rows = channels of chunk j, k = a tile's tokens ----
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            if (u < nt) {
                const unsigned char *st = wmem + ((ti + u - wb) % kGqaStages) * St::kBytes;
                uint32_t vw[W];
                load_stage_words<W>(reinterpret_cast<const uint32_t *>(st + St::kCodes), lane, vw);
#pragma unroll
                for (int j = 0; j < NJ; ++j) {
                    uint32_t a02, a13, b02, b13;
                    codes_bf16<N>(vw[j / BPW], 2 * (j % BPW), magic16, a02, a13);       // channel 16j + g8
                    codes_bf16<N>(vw[j / BPW], 2 * (j % BPW) + 1, magic16, b02, b13);   // channel 16j + g8 + 8
                    const uint2 bb = *reinterpret_cast<const uint2 *>(
                        vb + ((((u * NGV + (16 * j) / GV) * kGqa + (g8 >> 1)) * 2 + ((g8 & 1) ^ (g8 >> 2))) * 16) +
                        4 * t4);
                    hmma(dv[j], a02, b02, a13, b13, bb.x, bb.y);
                }
            }
        }
        __syncwarp();
    }
    cp_async_wait<0>();
    (void)magic;

    // ---- epilogue: reduce per head, subtract the z-terms, merge warps ----
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 4);
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 8);
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 16);
#pragma unroll
    for (int v = 0; v < NGV; ++v) {      // lanes with the same lane % 4 hold one head's partials
        zsum[v] += __shfl_xor_sync(0xffffffffu, zsum[v], 4);
        zsum[v] += __shfl_xor_sync(0xffffffffu, zsum[v], 8);
        zsum[v] += __shfl_xor_sync(0xffffffffu, zsum[v], 16);
    }
    __syncthreads();   // stage memory is reused for the per-warp outputs below
    float *o_s = reinterpret_cast<float *>(stage_mem);   // [warp][head][D]
    float *zs_s = o_s + kDecodeWarps * kGqa * D;          // [warp][head][NGV]
    if (lane < kGqa)
        for (int v = 0; v < NGV; ++v) zs_s[(warp * kGqa + lane) * NGV + v] = zsum[v];
    // dv sums A * B = (2^N + code) p s; zsum sums b (2^N + z) with b = p s 2^-(7-N)
    __syncwarp();
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
        const float z = zs_s[(warp * kGqa + t4) * NGV + (16 * j) / GV];
        constexpr float kUnscale = static_cast<float>(1 << (7 - N));
        o_s[(warp * kGqa + t4) * D + 16 * j + g8] = dv[j][0] + dv[j][1] - z * kUnscale;
        o_s[(warp * kGqa + t4) * D + 16 * j + g8 + 8] = dv[j][2] + dv[j][3] - z * kUnscale;
    }
    if (g8 == 0) {
        ml_s[warp][t4][0] = m;
        ml_s[warp][t4][1] = lsum;
    }
    __syncthreads();
    finish_cta<kGqa, D>(a, o_s, ml_s, bh, bq0, sigma, &last_s, o_s + kDecodeWarps * kGqa * D);
}

// ---------------------------------------------------------------------------
// One query head per kv head: tensor-core path.
//
// A CTA owns one (batch, head, split); each warp takes an even-aligned,
// contiguous share of the split's tiles and walks it in chunks of kMhaChunk
// tiles: first the keys of the chunk (logits to shared memory, a running
// maximum per lane), then, with the chunk's maximum fixed, its values.  So the
// probabilities need no per-tile cross-lane maximum, key and value work form
// two streams without dependences between tiles, and the accumulators are
// rescaled at most once per chunk.  Items -- a key tile pair or a value tile
// pair -- stream through a per-warp ring of cp.async stages; a key pair never
// straddles a key group (groups of >= 32 tokens).
//   keys   : int8 MMA m16n8k32, rows = tokens, k = channels.  A is a stored
//            word masked to one byte slot, without a shift: slot s arrives as
//            code * 2^(N*s).  The two 16-channel chunks of one MMA are taken
//            from the same slot class (same 2^(N*s) for its first 8 rows, the
//            next slot for the other 8), so the factor is constant per row of
//            the product and is divided out of the row sum exactly.  B holds
//            the balanced base-256 digits (each in [-128, 127]) of the 22-bit
//            fixed-point multipliers Q_c = round(2^e q_c s_{g,c} log2(e)/sqrt(d)),
//            built once per key group: columns 0, 1 hold digits 0, 1 and column
//            4 digit 2, so lanes t4 = 0 and t4 = 2 of a row group hold the row's
//            three digit sums; int32 accumulation is exact (|sum| < 2^22).
//   values : bf16 MMA m16n8k16, rows = channels, k = tokens: A = the codes as
//            exact bf16 2^(7-N) (2^N + code) (codes_bf16), B = p_t s_t 2^-(7-N)
//            split into a bf16 hi part (column 0) and lo part (column 1).
//   z-terms: bias_g = sum_c q'_c z_{g,c} and sum_t p_t s_t (z_t + 2^N) in fp32.
// The residual rows get no split of their own: their 16-row tiles are dealt
// round-robin to the warps of all splits, which run them on CUDA cores (staged
// in their stage memory) before streaming and start their softmax state there.
// ---------------------------------------------------------------------------
constexpr int kMhaChunk = 32;     // tiles per key phase / value phase of a warp
constexpr int kMhaStages = 4;

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

template <int N, int D, int GV>
struct MhaStage {                 // one item: two tiles of one code array and their meta
    static constexpr int W = D * N / 64;
    static constexpr int NGV = D / GV;
    static constexpr int kCodes = 32 * W * 4;            // one tile's code array (chunk-major)
    static constexpr int kMeta = 2 * kCodes;              // key item: scales [D] f32; value item: [32][NGV] f32
    static constexpr int kKz = kMeta + D * 4;             // key zeros [D] i16
    static constexpr int kVz = kMeta + 32 * NGV * 4;      // value zeros [32][NGV] i16
    static constexpr int kEnd = (kKz + D * 2 > kVz + 32 * NGV * 2) ? kKz + D * 2 : kVz + 32 * NGV * 2;
    static constexpr int kBytes = (kEnd + 15) / 16 * 16;
    static_assert(kMeta % 16 == 0 && kKz % 16 == 0 && kVz % 16 == 0, "align");
};

template <int N, int D, int GV>
struct MhaSmem {
    static constexpr int kKdWords = D / 4 + 4;   // one digit row (4 channels a word), padded by 4 banks
    static constexpr int kLg = kMhaStages * MhaStage<N, D, GV>::kBytes;   // logits [kMhaChunk][16] f32
    static constexpr int kKd = kLg + kMhaChunk * 16 * 4;
    static constexpr int kWarpBytes = kKd + 3 * kKdWords * 4;
    static_assert(kLg % 16 == 0 && kWarpBytes % 16 == 0, "align");
};

// Value scales and zeros of the four tokens 4*t4 + i of a lane (NGV of each).
template <int NGV>
__device__ __forceinline__ void load_meta4(const float *sp, const int16_t *zp, bool sym, int zsym,
                                           float (&s)[4][NGV], int (&z)[4][NGV]) {
    if constexpr (NGV == 1) {
        const float4 v = *reinterpret_cast<const float4 *>(sp);
        s[0][0] = v.x; s[1][0] = v.y; s[2][0] = v.z; s[3][0] = v.w;
        if (sym) {
#pragma unroll
            for (int i = 0; i < 4; ++i) z[i][0] = zsym;
        } else {
            const uint2 u = *reinterpret_cast<const uint2 *>(zp);
            z[0][0] = static_cast<int16_t>(u.x & 0xffffu); z[1][0] = static_cast<int16_t>(u.x >> 16);
            z[2][0] = static_cast<int16_t>(u.y & 0xffffu); z[3][0] = static_cast<int16_t>(u.y >> 16);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            int16_t zz[NGV];
            load_meta<NGV>(sp + i * NGV, zp + i * NGV, sym, zsym, s[i], zz);
#pragma unroll
            for (int v = 0; v < NGV; ++v) z[i][v] = zz[v];
        }
    }
}

template <int N, int D, int GV>
__global__ void __launch_bounds__(kDecodeThreads, (D / GV >= 4) ? 3 : 4) decode_mha_kernel(const DecodeArgs a) {
    constexpr int W = D * N / 64;
    constexpr int TW = D * N / 2;
    constexpr int NJ = D / 16;
    constexpr int BPW = 4 / N;        // slot classes (chunks per word)
    constexpr int NP = W / 2;         // word pairs; the key MMAs of a tile are (pair, class)
    constexpr int NGV = D / GV;
    constexpr uint32_t BYTE_L = ((1u << N) - 1u) * 0x01010101u;
    constexpr int kSt = kMhaStages;
    using St = MhaStage<N, D, GV>;
    using Sm = MhaSmem<N, D, GV>;
    static_assert(W % 2 == 0, "key MMAs take words in pairs");
    static_assert(kMhaChunk % 2 == 0 && (kMhaChunk & (kMhaChunk - 1)) == 0, "chunk");

    __shared__ __align__(16) float q_s[D];
    __shared__ float ml_s[kDecodeWarps][1][2];
    __shared__ int last_s;
    extern __shared__ __align__(128) unsigned char stage_mem[];

    const int qi = blockIdx.x, b = blockIdx.y, sigma = blockIdx.z;
    const int64_t bh = static_cast<int64_t>(b) * a.Hkv + qi;
    const int64_t bq = static_cast<int64_t>(b) * a.Hq + qi;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g8 = lane >> 2, t4 = lane & 3;
    unsigned char *wmem = stage_mem + static_cast<size_t>(warp) * Sm::kWarpBytes;
    float *lgs = reinterpret_cast<float *>(wmem + Sm::kLg);
    uint32_t *kd = reinterpret_cast<uint32_t *>(wmem + Sm::kKd);
    const int zsym = 1 << (N - 1);

    for (int c = threadIdx.x; c < D; c += kDecodeThreads)
        q_s[c] = widen(a.q[bq * D + c], a.bf16) * a.qscale;
    __syncthreads();

    float m = -INFINITY, lsum = 0.f;
    float ov[NJ][2];   // channels 16j + g8 (+8), final in lanes t4 == 0

    {
        // ---------------- quantized split ----------------
        const int t_begin = sigma * a.tiles_per_split;                 // even
        const int t_end = min(a.n_qtiles, t_begin + a.tiles_per_split);
        const int per_w = 2 * ((t_end - t_begin + 2 * kDecodeWarps - 1) / (2 * kDecodeWarps));
        const int wb = min(t_end, t_begin + warp * per_w);             // even
        const int ntiles = min(t_end, wb + per_w) - wb;
        const int nitems = 2 * ((ntiles + 1) / 2);   // one key item and one value item per tile pair
        const int64_t groups_cap = a.cap / a.G;
        const int64_t tile0 = bh * (a.cap / 16) + wb;
        const uint32_t *kp = a.kc + tile0 * TW;
        const uint32_t *vp = a.vc + tile0 * TW;
        const float *vsp = a.vs + tile0 * 16 * NGV;
        const int16_t *vzp = a.sym ? nullptr : a.vz + tile0 * 16 * NGV;
        const int gmask = (1 << a.gshift) - 1;
        const int n_vs = 4 * NGV, n_meta = a.sym ? n_vs : 6 * NGV;   // 16-byte pieces per value tile

        // Item cursor: chunk [cb, cb + kMhaChunk) of the warp's tiles holds np tile pairs; items
        // 0 .. np-1 of a chunk are its key pairs, np .. 2np-1 its value pairs.
        struct Cursor {
            int cb, r, np;
            __device__ void start(int ntiles) { cb = 0; r = 0; np = (min(kMhaChunk, ntiles) + 1) / 2; }
            __device__ void next(int ntiles) {
                if (++r == 2 * np) {
                    cb += kMhaChunk;
                    r = 0;
                    np = (min(kMhaChunk, ntiles - cb) + 1) / 2;
                }
            }
            __device__ bool key() const { return r < np; }
            __device__ int rel() const { return cb + 2 * (r < np ? r : r - np); }
        };

        Cursor ic;       // producer's cursor, kSt - 1 items ahead
        ic.start(ntiles);
        int issued = 0;
        auto issue_next = [&]() {
            if (issued < nitems) {
                unsigned char *st = wmem + (issued % kSt) * St::kBytes;
                const int rel = ic.rel();
                const bool two = rel + 1 < ntiles;
                if (ic.key()) {
                    const uint32_t *src = kp + static_cast<int64_t>(rel) * TW;
                    copy_tile_codes<W>(st, src, lane);
                    if (two) copy_tile_codes<W>(st + St::kCodes, src + TW, lane);
                    const int ti = wb + rel;
                    if (rel == 0 || (ti & gmask) == 0) {
                        const int64_t gofs = (bh * groups_cap + (ti >> a.gshift)) * D;
                        for (int c = lane; c < (a.sym ? D / 4 : D / 4 + D / 8); c += 32) {
                            if (c < D / 4) cp_async16(st + St::kMeta + 16 * c, a.ks + gofs + 4 * c);
                            else cp_async16(st + St::kKz + 16 * (c - D / 4), a.kz + gofs + 8 * (c - D / 4));
                        }
                    }
                } else {
                    const uint32_t *src = vp + static_cast<int64_t>(rel) * TW;
                    copy_tile_codes<W>(st, src, lane);
                    if (two) copy_tile_codes<W>(st + St::kCodes, src + TW, lane);
                    const int64_t tok = static_cast<int64_t>(rel) * 16 * NGV;
                    const int nvs = two ? 2 * n_vs : n_vs;
                    for (int c = lane; c < (two ? 2 * n_meta : n_meta); c += 32) {
                        if (c < nvs) cp_async16(st + St::kMeta + 16 * c, vsp + tok + 4 * c);
                        else cp_async16(st + St::kVz + 16 * (c - nvs), vzp + tok + 8 * (c - nvs));
                    }
                }
                ic.next(ntiles);
            }
            cp_async_commit();
            ++issued;
        };

        float dv[NJ][4];   // value MMA accumulators: rows = channels 16j + g8 (+8), columns 2*t4, 2*t4 + 1
#pragma unroll
        for (int j = 0; j < NJ; ++j) dv[j][0] = dv[j][1] = dv[j][2] = dv[j][3] = 0.f;
        float zsum[NGV];
#pragma unroll
        for (int v = 0; v < NGV; ++v) zsum[v] = 0.f;
        uint32_t kb[NP * BPW][2];   // key MMA B fragments of the current group
        float klane = 0.f, kbias = 0.f;
        float mloc = -INFINITY;     // this lane's largest logit of the current chunk

        // Key digits of the group the stage opens: lane l builds channels 4l .. 4l+3.
        auto rebuild_key_digits = [&](const unsigned char *st) {
            const int cl = lane % (D / 4);
            const float4 sc = *reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(st + St::kMeta) + 4 * cl);
            const float4 qq = *reinterpret_cast<const float4 *>(q_s + 4 * cl);
            const float qv[4] = {qq.x * sc.x, qq.y * sc.y, qq.z * sc.z, qq.w * sc.w};
            float z[4] = {static_cast<float>(zsym), static_cast<float>(zsym), static_cast<float>(zsym),
                          static_cast<float>(zsym)};
            if (!a.sym) {
                const uint2 zz = *reinterpret_cast<const uint2 *>(reinterpret_cast<const int16_t *>(st + St::kKz) + 4 * cl);
                z[0] = small_int_to_float(static_cast<int16_t>(zz.x & 0xffffu));
                z[1] = small_int_to_float(static_cast<int16_t>(zz.x >> 16));
                z[2] = small_int_to_float(static_cast<int16_t>(zz.y & 0xffffu));
                z[3] = small_int_to_float(static_cast<int16_t>(zz.y >> 16));
            }
            float kbp = 0.f, mx = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                kbp = fmaf(qv[i], z[i], kbp);
                mx = fmaxf(mx, fabsf(qv[i]));
            }
            if (lane >= D / 4) kbp = 0.f;    // d = 64: lanes 16..31 repeat channels
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                kbp += __shfl_xor_sync(0xffffffffu, kbp, o);
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            }
            // 2^e with |q'| 2^e < 2^21, from the exponent of the largest |q'|
            int e = 0;
            if (mx > 0.f) e = 21 - (static_cast<int>((__float_as_uint(mx) >> 23) & 0xff) - 126);
            e = max(-120, min(120, e));
            const float scale = __uint_as_float(static_cast<uint32_t>(127 + e) << 23);
            // balanced base-256 digits: Q = d0 + 256 d1 + 65536 d2 with d0, d1 in [-128, 127]
            int dg[3][4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int Q = round_small(qv[i] * scale);
                const int Q1 = (Q + 128) >> 8;
                dg[0][i] = Q;
                dg[1][i] = Q1;
                dg[2][i] = (Q1 + 128) >> 8;
            }
            __syncwarp();   // the previous group's digits have been read
            if (lane < D / 4) {
#pragma unroll
                for (int k = 0; k < 3; ++k)
                    kd[k * Sm::kKdWords + cl] = __byte_perm(__byte_perm(dg[k][0], dg[k][1], 0x0040),
                                                            __byte_perm(dg[k][2], dg[k][3], 0x0040), 0x5410);
            }
            __syncwarp();
            // B fragments: column g8 holds digit 0 (g8 = 0), 1 (g8 = 1) or 2 (g8 = 4)
            const int dig = g8 == 0 ? 0 : (g8 == 1 ? 1 : 2);
            const bool has = g8 == 0 || g8 == 1 || g8 == 4;
            const uint32_t *row = kd + dig * Sm::kKdWords;
#pragma unroll
            for (int pm = 0; pm < NP; ++pm) {
#pragma unroll
                for (int c = 0; c < BPW; ++c) {
                    const int j1 = 2 * pm * BPW + c, j2 = j1 + BPW;
                    kb[pm * BPW + c][0] = has ? row[4 * j1 + t4] : 0u;
                    kb[pm * BPW + c][1] = has ? row[4 * j2 + t4] : 0u;
                }
            }
            const float kinv = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
            klane = t4 == 2 ? kinv * 65536.f : kinv;
            kbias = kbp;
        };

        // This warp's share of the residual tiles (dealt round-robin over the warps of all
        // splits), on CUDA cores in the stage memory before the stream starts.  Its result
        // seeds the softmax state: lane t4 = 0 holds channels 16j + g8 (+8) in both layouts,
        // and lsum carries the B operand's 2^-(7-N).
        static_assert(residual_scratch_bytes<D>() <= Sm::kWarpBytes, "residual staging");
        {
            const int nres = (a.r + 15) / 16;
            const int gw = sigma * kDecodeWarps + warp, nw = a.S * kDecodeWarps;
            if (gw < nres) {
                float lr = 0.f;
                float2 acc[NJ][2];
#pragma unroll
                for (int j = 0; j < NJ; ++j) acc[j][0] = acc[j][1] = make_float2(0.f, 0.f);
                residual_pass<D>(a, q_s, a.kr + bh * a.R * D, a.vr + bh * a.R * D, gw, nres, lane, m, lr,
                                 acc, wmem, nw);
                lr += __shfl_xor_sync(0xffffffffu, lr, 4);     // lanes hold rows g8, g8 + 8
                lr += __shfl_xor_sync(0xffffffffu, lr, 8);
                lr += __shfl_xor_sync(0xffffffffu, lr, 16);
#pragma unroll
                for (int j = 0; j < NJ; ++j) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        float val = acc[j][h].x + acc[j][h].y;
                        val += __shfl_xor_sync(0xffffffffu, val, 1);
                        val += __shfl_xor_sync(0xffffffffu, val, 2);
                        dv[j][2 * h] = t4 == 0 ? val : 0.f;
                    }
                }
                lsum = t4 == 0 ? lr / static_cast<float>(1 << (7 - N)) : 0.f;
            }
        }

#pragma unroll
        for (int s = 0; s < kSt - 1; ++s) issue_next();

        Cursor cc;       // consumer's cursor
        cc.start(ntiles);
        for (int k = 0; k < nitems; ++k) {
            issue_next();
            cp_async_wait<kSt - 1>();
            __syncwarp();
            const unsigned char *st = wmem + (k % kSt) * St::kBytes;
            const int rel = cc.rel();
            const int nt = rel + 1 < ntiles ? 2 : 1;
            float *lgc = lgs + (rel % kMhaChunk) * 16;   // logits of tiles rel, rel + 1
            if (cc.key()) {
                if (rel == 0 || ((wb + rel) & gmask) == 0) rebuild_key_digits(st);
                // ---- key MMAs: log2-domain logits of tokens g8 and g8 + 8 ----
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    if (u < nt) {
                        uint32_t kw[W];
                        load_stage_words<W>(reinterpret_cast<const uint32_t *>(st + u * St::kCodes), lane, kw);
                        int acc[2][BPW][4];   // two chains (even / odd word pair)
#pragma unroll
                        for (int pm = 0; pm < NP; ++pm) {
#pragma unroll
                            for (int c = 0; c < BPW; ++c) {
                                const uint32_t mlo = BYTE_L << (N * 2 * c), mhi = BYTE_L << (N * (2 * c + 1));
                                const uint32_t af[4] = {kw[2 * pm] & mlo, kw[2 * pm] & mhi, kw[2 * pm + 1] & mlo,
                                                        kw[2 * pm + 1] & mhi};
                                if (pm < 2) imma_us0(acc[pm][c], af, kb[pm * BPW + c][0], kb[pm * BPW + c][1]);
                                else imma_us(acc[pm & 1][c], af, kb[pm * BPW + c][0], kb[pm * BPW + c][1]);
                            }
                        }
                        float x0 = 0.f, x1 = 0.f;
#pragma unroll
                        for (int c = 0; c < BPW; ++c) {   // digit sums d0 + 256 d1 (< 2^31), slot factor out
                            const float f0 = 1.0f / static_cast<float>(1u << (2 * N * c));
                            const float f1 = 1.0f / static_cast<float>(1u << (N * (2 * c + 1)));
                            int r0 = acc[0][c][0] + acc[0][c][1] * 256, r1 = acc[0][c][2] + acc[0][c][3] * 256;
                            if constexpr (NP > 1) {
                                r0 += acc[1][c][0] + acc[1][c][1] * 256;
                                r1 += acc[1][c][2] + acc[1][c][3] * 256;
                            }
                            x0 = fmaf(static_cast<float>(r0), f0, x0);
                            x1 = fmaf(static_cast<float>(r1), f1, x1);
                        }
                        x0 *= klane;
                        x1 *= klane;
                        x0 += __shfl_xor_sync(0xffffffffu, x0, 1);
                        x1 += __shfl_xor_sync(0xffffffffu, x1, 1);
                        x0 += __shfl_xor_sync(0xffffffffu, x0, 2);
                        x1 += __shfl_xor_sync(0xffffffffu, x1, 2);
                        const float lg0 = x0 - kbias, lg1 = x1 - kbias;
                        mloc = fmaxf(mloc, fmaxf(lg0, lg1));
                        if (t4 == 0) {
                            lgc[16 * u + g8] = lg0;
                            lgc[16 * u + g8 + 8] = lg1;
                        }
                    }
                }
                if (cc.r == cc.np - 1) {
                    // the chunk's keys are done: fix its maximum, rescale what came before
                    float cm = mloc;
                    cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 4));
                    cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 8));
                    cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 16));
                    if (cm > m) {
                        const float alpha = fast_exp2(m - cm);
                        m = cm;
                        lsum *= alpha;
#pragma unroll
                        for (int j = 0; j < NJ; ++j) {
                            dv[j][0] *= alpha; dv[j][1] *= alpha; dv[j][2] *= alpha; dv[j][3] *= alpha;
                        }
#pragma unroll
                        for (int v = 0; v < NGV; ++v) zsum[v] *= alpha;
                    }
                    mloc = -INFINITY;
                }
            } else {
                // p 2^-(7-N) of tokens 4*t4 + i (the B scale folded into the exponent)
                const float mb = m + static_cast<float>(7 - N);
                constexpr int kOff = 1 << N;
                const bool lo_part = (g8 & 1) != 0;   // B column g8: hi part (even), lo part (odd)
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    if (u < nt) {
                        const float4 l4 = *reinterpret_cast<const float4 *>(lgc + 16 * u + 4 * t4);
                        const float pt[4] = {fast_exp2(l4.x - mb), fast_exp2(l4.y - mb), fast_exp2(l4.z - mb),
                                             fast_exp2(l4.w - mb)};
                        lsum += (pt[0] + pt[1]) + (pt[2] + pt[3]);
                        float sv[4][NGV];
                        int zv[4][NGV];
                        load_meta4<NGV>(reinterpret_cast<const float *>(st + St::kMeta) + (16 * u + 4 * t4) * NGV,
                                        reinterpret_cast<const int16_t *>(st + St::kVz) + (16 * u + 4 * t4) * NGV,
                                        a.sym, zsym, sv, zv);
                        uint32_t B0[NGV], B1[NGV];
#pragma unroll
                        for (int v = 0; v < NGV; ++v) {
                            float ps[4];
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                ps[i] = pt[i] * sv[i][v];
                                zsum[v] = fmaf(ps[i], small_int_to_float(zv[i][v] + kOff), zsum[v]);
                            }
                            // k order of the B fragment: (4t4, 4t4+2 | 4t4+1, 4t4+3), as codes_bf16 pairs
                            // bytes; columns 2..7 repeat columns 0, 1 and their sums are not read
                            const uint32_t h02 = f2bf2(ps[0], ps[2]), h13 = f2bf2(ps[1], ps[3]);
                            const uint32_t l02 = f2bf2(ps[0] - __uint_as_float(h02 << 16),
                                                       ps[2] - __uint_as_float(h02 & 0xffff0000u));
                            const uint32_t l13 = f2bf2(ps[1] - __uint_as_float(h13 << 16),
                                                       ps[3] - __uint_as_float(h13 & 0xffff0000u));
                            B0[v] = lo_part ? l02 : h02;
                            B1[v] = lo_part ? l13 : h13;
                        }
                        // ---- value MMAs: rows = channels of chunk j, k = the tile's tokens ----
                        uint32_t vw[W];
                        load_stage_words<W>(reinterpret_cast<const uint32_t *>(st + u * St::kCodes), lane, vw);
                        const uint32_t magic16 = 0x43004300u;
#pragma unroll
                        for (int j = 0; j < NJ; ++j) {
                            uint32_t a02, a13, b02, b13;
                            codes_bf16<N>(vw[j / BPW], 2 * (j % BPW), magic16, a02, a13);       // channel 16j + g8
                            codes_bf16<N>(vw[j / BPW], 2 * (j % BPW) + 1, magic16, b02, b13);   // channel 16j + g8 + 8
                            hmma(dv[j], a02, b02, a13, b13, B0[(16 * j) / GV], B1[(16 * j) / GV]);
                        }
                    }
                }
            }
            cc.next(ntiles);
            __syncwarp();   // stage consumed and the chunk's logits visible to every lane
        }
        cp_async_wait<0>();

        // lanes with the same t4 hold the same token sums: reduce over t4; lsum and zsum carry
        // the 2^-(7-N) of the B operand, dv sums (2^N + code) p s
        lsum += __shfl_xor_sync(0xffffffffu, lsum, 1);
        lsum += __shfl_xor_sync(0xffffffffu, lsum, 2);
        lsum *= static_cast<float>(1 << (7 - N));
#pragma unroll
        for (int v = 0; v < NGV; ++v) {
            zsum[v] += __shfl_xor_sync(0xffffffffu, zsum[v], 1);
            zsum[v] += __shfl_xor_sync(0xffffffffu, zsum[v], 2);
        }
        constexpr float kUnscale = static_cast<float>(1 << (7 - N));
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
            const float z = zsum[(16 * j) / GV] * kUnscale;
            ov[j][0] = dv[j][0] + dv[j][1] - z;
            ov[j][1] = dv[j][2] + dv[j][3] - z;
        }
    }

    __syncthreads();   // stage memory is reused for the per-warp outputs
    float *o_s = reinterpret_cast<float *>(stage_mem);   // [warp][D]
    if (t4 == 0) {
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
            o_s[warp * D + 16 * j + g8] = ov[j][0];
            o_s[warp * D + 16 * j + g8 + 8] = ov[j][1];
        }
    }
    if (lane == 0) {
        ml_s[warp][0][0] = m;
        ml_s[warp][0][1] = lsum;
    }
    __syncthreads();
    finish_cta<1, D>(a, o_s, ml_s, bq, bq, sigma, &last_s, o_s + kDecodeWarps * D);
}

template <int N, int D, int GV>
constexpr int split_smem() { return kDecodeWarps * kStages * Stage<N, D, GV>::kBytes; }
template <int N, int D, int GV>
constexpr int gqa_smem() { return kDecodeWarps * GqaSmem<N, D, GV>::kWarpBytes; }
template <int N, int D, int GV>
constexpr int mha_smem() { return kDecodeWarps * MhaSmem<N, D, GV>::kWarpBytes; }

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

// Dispatch over the compiled (bits, head_dim, value-group) variants and the three kernels.
// The split index is the slowest grid dimension: CTAs start in linear order, so every
// quantized split is resident before the (short) residual-split CTAs fill the slots
// that remain.
template <int N, int D, int GV>
struct LaunchF {
    static cudaError_t run(const DecodeArgs &a, cudaStream_t s) {
        switch (a.path) {
            case kPathGqa:
                return launch_kernel<decode_gqa_kernel<N, D, GV>>(a, dim3(a.Hkv, a.B, a.S),
                                                                  gqa_smem<N, D, GV>(), s);
            case kPathMha:
                return launch_kernel<decode_mha_kernel<N, D, GV>>(a, dim3(a.Hq, a.B, a.S),
                                                                  mha_smem<N, D, GV>(), s);
            default:
                return launch_kernel<decode_split_kernel<N, D, GV>>(a, dim3(a.Hq, a.B, a.S),
                                                                    split_smem<N, D, GV>(), s);
        }
    }
    static int occ(const DecodeArgs &a) {
        switch (a.path) {
            case kPathGqa: return occupancy_of<decode_gqa_kernel<N, D, GV>>(gqa_smem<N, D, GV>());
            case kPathMha: return occupancy_of<decode_mha_kernel<N, D, GV>>(mha_smem<N, D, GV>());
            default: return occupancy_of<decode_split_kernel<N, D, GV>>(split_smem<N, D, GV>());
        }
    }
};

template <int N, int D>
cudaError_t launch_gv(const DecodeArgs &a, cudaStream_t s) {
    switch (a.Gv) {
        case 16: return LaunchF<N, D, 16>::run(a, s);
        case 32: return LaunchF<N, D, 32>::run(a, s);
        case 64: return LaunchF<N, D, 64>::run(a, s);
        default: if constexpr (D >= 128) { if (a.Gv == 128) return LaunchF<N, D, 128>::run(a, s); }
    }
    return cudaErrorInvalidValue;
}

template <int N, int D>
int occ_gv(const DecodeArgs &a) {
    switch (a.Gv) {
        case 16: return LaunchF<N, D, 16>::occ(a);
        case 32: return LaunchF<N, D, 32>::occ(a);
        case 64: return LaunchF<N, D, 64>::occ(a);
        default: if constexpr (D >= 128) { if (a.Gv == 128) return LaunchF<N, D, 128>::occ(a); }
    }
    return 1;
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t s) {
    cudaError_t e = cudaErrorInvalidValue;
    if (a.bits == 2 && a.d == 64) e = launch_gv<2, 64>(a, s);
    else if (a.bits == 2 && a.d == 128) e = launch_gv<2, 128>(a, s);
    else if (a.bits == 4 && a.d == 64) e = launch_gv<4, 64>(a, s);
    else if (a.bits == 4 && a.d == 128) e = launch_gv<4, 128>(a, s);
    return e;
}

int decode_ctas_per_sm(const DecodeArgs &a) {
    if (a.bits == 2 && a.d == 64) return occ_gv<2, 64>(a);
    if (a.bits == 2 && a.d == 128) return occ_gv<2, 128>(a);
    if (a.bits == 4 && a.d == 64) return occ_gv<4, 64>(a);
    if (a.bits == 4 && a.d == 128) return occ_gv<4, 128>(a);
    return 1;
}

}  // namespace kvq
