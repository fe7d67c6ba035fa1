// decode.cu -- split-K decode attention over the packed low-bit cache.
//
// Computes, for every (batch, query head), one decode step of
//   A = softmax(q [deq(K_g); K_r]^T / sqrt(d)),   t_O = A [deq(V_g); V_r]
// ("LLM系列：KVCache量化1 KIVI ...", section 1: A = Concat(A_g, A_r), t_O = A X_V;
//  the 1/sqrt(d_k) of "KV Cache的Int4量化…" section 3), with deq(x) = (code - z) s.
//
// Split-K (flash-decoding): the token axis -- quantized 16-token tiles followed
// by the residual rows, cut into 16-row tiles -- is divided into S contiguous
// splits; a CTA owns one (batch, query head, split) and its four warps take the
// split's tiles round-robin.  Token order does not change the result
// (A . V = A_P . V_P, "Resumo Técnico: LogQuant", section 4), which is what
// allows the splits and the residual to be folded into one online-softmax pass.
// Each CTA writes an unnormalised partial (o, m, l); combine_kernel merges the
// S partials with a log-sum-exp reduction.
//
// Inner loop, per lane and tile (lane = 4*r8 + l4 owns the A-fragment slots of
// the packed layout):
//   keys   : logit_t = sum_c q_c s_{g,c} (code - z_{g,c}) / sqrt(d)
//            = sum_c M_c code_{t,c} - bias_g, with M_c = q_c s_{g,c} log2(e)/sqrt(d)
//            refreshed once per key group and bias_g = sum_c M_c z_{g,c};
//   values : o_c += sum_t p_t s_{t,gv} code_{t,c} - sum_t p_t s_{t,gv} z_{t,gv}.
// Codes are turned into floats with the exponent trick: (word & mask) | 0x4B000000
// is the float 2^23 + code * 2^pos exactly; one packed fp32x2 add removes 2^23
// and one packed fp32x2 FMA accumulates two codes, the 2^pos factors being
// folded into the multipliers (exact powers of two).
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

// Load the W words a lane owns in one tile with the widest aligned loads.
template <int W>
__device__ __forceinline__ void load_lane_words(const uint32_t *p, uint32_t (&w)[W]) {
    if constexpr (W % 4 == 0) {
#pragma unroll
        for (int i = 0; i < W / 4; ++i) {
            const uint4 v = __ldg(reinterpret_cast<const uint4 *>(p) + i);
            w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
        }
    } else if constexpr (W % 2 == 0) {
#pragma unroll
        for (int i = 0; i < W / 2; ++i) {
            const uint2 v = __ldg(reinterpret_cast<const uint2 *>(p) + i);
            w[2 * i] = v.x; w[2 * i + 1] = v.y;
        }
    } else {
#pragma unroll
        for (int i = 0; i < W; ++i) w[i] = __ldg(p + i);
    }
}

// Code pair (half 0 from the low 16 bits, half 1 from the high) at slot pi,
// as floats code * 2^(N*pi).
template <int N>
__device__ __forceinline__ float2 code_pair(uint32_t lo, uint32_t hi, int pi) {
    const uint32_t msk = ((1u << N) - 1u) << (N * pi);
    float2 v = make_float2(__uint_as_float((lo & msk) | kMagicBits),
                           __uint_as_float((hi & msk) | kMagicBits));
    return add2(v, make_float2(-kMagic, -kMagic));
}

template <int N, int D, int GV>
__global__ void __launch_bounds__(kDecodeThreads, 4) decode_split_kernel(const DecodeArgs a) {
    constexpr int P = 16 / N;         // code pairs per word
    constexpr int W = D * N / 64;     // words per lane per tile
    constexpr int TW = D * N / 2;     // words per tile
    constexpr int NJ = D / 16;        // 16-channel chunks
    constexpr int NGV = D / GV;       // value groups per token
    constexpr float kInvN = 1.0f / (1 << N);

    __shared__ float q_s[D];
    __shared__ float o_s[kDecodeWarps][D];
    __shared__ float ml_s[kDecodeWarps][2];

    const int sigma = blockIdx.x, qi = blockIdx.y, b = blockIdx.z;
    const int g = a.Hq / a.Hkv;
    const int64_t bh = static_cast<int64_t>(b) * a.Hkv + qi / g;
    const int64_t bq = static_cast<int64_t>(b) * a.Hq + qi;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r8 = lane >> 2, l4 = lane & 3;

    for (int c = threadIdx.x; c < D; c += kDecodeThreads)
        q_s[c] = widen(a.q[bq * D + c], a.bf16) * a.qscale;
    __syncthreads();

    const int total_tiles = a.n_qtiles + (a.r + 15) / 16;
    const int t_begin = sigma * a.tiles_per_split;
    const int t_end = min(total_tiles, t_begin + a.tiles_per_split);
    const int64_t groups_cap = a.cap / a.G;
    const uint32_t *kc = a.kc + bh * (a.cap / 16) * TW;
    const uint32_t *vc = a.vc + bh * (a.cap / 16) * TW;
    const int zsym = 1 << (N - 1);

    float m = -INFINITY, lsum = 0.0f;
    float2 acc[NJ][2];
    float zsum[NGV];
#pragma unroll
    for (int j = 0; j < NJ; ++j) acc[j][0] = acc[j][1] = make_float2(0.f, 0.f);
#pragma unroll
    for (int v = 0; v < NGV; ++v) zsum[v] = 0.f;
    float2 mk[NJ][2];
    float kbias = 0.f;
    int64_t cur_group = -1;

    for (int ti = t_begin + warp; ti < t_end; ti += kDecodeWarps) {
        const bool quant = ti < a.n_qtiles;
        float lg0, lg1;   // log2-domain logits of tokens r8 and r8 + 8 of the tile
        if (quant) {
            const int64_t tok0 = static_cast<int64_t>(ti) * 16;
            const int64_t grp = tok0 / a.G;
            if (grp != cur_group) {
                // key multipliers and bias of the new group
                const int64_t gofs = (bh * groups_cap + grp) * D;
                float kb = 0.f;
#pragma unroll
                for (int j = 0; j < NJ; ++j) {
#pragma unroll
                    for (int s = 0; s < 2; ++s) {
                        const int c0 = 16 * j + 2 * l4 + 8 * s;
                        const float2 sc = *reinterpret_cast<const float2 *>(a.ks + gofs + c0);
                        const float2 qs = make_float2(q_s[c0] * sc.x, q_s[c0 + 1] * sc.y);
                        float z0 = static_cast<float>(zsym), z1 = z0;
                        if (!a.sym) {
                            const uint32_t zz = *reinterpret_cast<const uint32_t *>(a.kz + gofs + c0);
                            z0 = static_cast<float>(static_cast<int16_t>(zz & 0xffffu));
                            z1 = static_cast<float>(static_cast<int16_t>(zz >> 16));
                        }
                        kb = fmaf(qs.x, z0, kb);
                        kb = fmaf(qs.y, z1, kb);
                        const int pos = (4 * j + 2 * s) % P;
                        const float f = 1.0f / static_cast<float>(1u << (N * pos));
                        mk[j][s] = make_float2(qs.x * f, qs.y * f);
                    }
                }
                kb += __shfl_xor_sync(0xffffffffu, kb, 1);
                kb += __shfl_xor_sync(0xffffffffu, kb, 2);
                kbias = kb;
                cur_group = grp;
            }
            uint32_t kw[W];
            load_lane_words<W>(kc + static_cast<int64_t>(ti) * TW + lane * W, kw);
            float2 s0 = make_float2(0.f, 0.f), s1 = s0;
#pragma unroll
            for (int wi = 0; wi < W; ++wi) {
                const uint32_t lo = kw[wi], hi = kw[wi] >> 16;
#pragma unroll
                for (int pi = 0; pi < P; ++pi) {
                    const int psi = wi * P + pi;
                    const int j = psi >> 2, k = psi & 3;
                    const float2 v = code_pair<N>(lo, hi, pi);
                    if ((k & 1) == 0)
                        s0 = fma2(v, mk[j][k >> 1], s0);
                    else
                        s1 = fma2(v, mk[j][k >> 1], s1);
                }
            }
            float x0 = s0.x + s0.y, x1 = (s1.x + s1.y) * kInvN;
            x0 += __shfl_xor_sync(0xffffffffu, x0, 1);
            x1 += __shfl_xor_sync(0xffffffffu, x1, 1);
            x0 += __shfl_xor_sync(0xffffffffu, x0, 2);
            x1 += __shfl_xor_sync(0xffffffffu, x1, 2);
            lg0 = x0 - kbias;
            lg1 = x1 - kbias;
        } else {
            // residual rows: exact e values
            const int row0 = (ti - a.n_qtiles) * 16 + r8, row1 = row0 + 8;
            float x0 = 0.f, x1 = 0.f;
            const uint16_t *kr = a.kr + bh * a.R * D;
#pragma unroll
            for (int j = 0; j < NJ; ++j) {
#pragma unroll
                for (int s = 0; s < 2; ++s) {
                    const int c0 = 16 * j + 2 * l4 + 8 * s;
                    if (row0 < a.r) {
                        const uint32_t two = *reinterpret_cast<const uint32_t *>(kr + row0 * D + c0);
                        x0 = fmaf(q_s[c0], widen(two & 0xffffu, a.bf16), x0);
                        x0 = fmaf(q_s[c0 + 1], widen(two >> 16, a.bf16), x0);
                    }
                    if (row1 < a.r) {
                        const uint32_t two = *reinterpret_cast<const uint32_t *>(kr + row1 * D + c0);
                        x1 = fmaf(q_s[c0], widen(two & 0xffffu, a.bf16), x1);
                        x1 = fmaf(q_s[c0 + 1], widen(two >> 16, a.bf16), x1);
                    }
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
            const float alpha = exp2f(m - tmax);
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
        const float p0 = exp2f(lg0 - m), p1 = exp2f(lg1 - m);
        lsum += p0 + p1;
        // probabilities of the lane's value tokens 2*l4, 2*l4+1, 2*l4+8, 2*l4+9
        const float pa = __shfl_sync(0xffffffffu, p0, 8 * l4);
        const float pb = __shfl_sync(0xffffffffu, p0, 8 * l4 + 4);
        const float pc = __shfl_sync(0xffffffffu, p1, 8 * l4);
        const float pd = __shfl_sync(0xffffffffu, p1, 8 * l4 + 4);

        if (quant) {
            const int64_t ta = static_cast<int64_t>(ti) * 16 + 2 * l4;
            const float *vsp = a.vs + (bh * a.cap + ta) * NGV;
            const int16_t *vzp = a.vz + (bh * a.cap + ta) * NGV;
            float2 pm[NGV][2];
#pragma unroll
            for (int v = 0; v < NGV; ++v) {
                const float sa = vsp[v], sb = vsp[NGV + v];
                const float sc = vsp[8 * NGV + v], sd = vsp[9 * NGV + v];
                const float2 plo = make_float2(pa * sa, pb * sb);
                const float2 phi = make_float2(pc * sc, pd * sd);
                float za, zb, zc, zd;
                if (a.sym) {
                    za = zb = zc = zd = static_cast<float>(zsym);
                } else {
                    za = vzp[v]; zb = vzp[NGV + v]; zc = vzp[8 * NGV + v]; zd = vzp[9 * NGV + v];
                }
                zsum[v] = fmaf(plo.x, za, zsum[v]);
                zsum[v] = fmaf(plo.y, zb, zsum[v]);
                zsum[v] = fmaf(phi.x, zc, zsum[v]);
                zsum[v] = fmaf(phi.y, zd, zsum[v]);
                pm[v][0] = plo;
                pm[v][1] = mul2(phi, make_float2(1.0f / (1 << (2 * N)), 1.0f / (1 << (2 * N))));
            }
            uint32_t vw[W];
            load_lane_words<W>(vc + static_cast<int64_t>(ti) * TW + lane * W, vw);
#pragma unroll
            for (int wi = 0; wi < W; ++wi) {
                const uint32_t lo = vw[wi], hi = vw[wi] >> 16;
#pragma unroll
                for (int pi = 0; pi < P; ++pi) {
                    const int psi = wi * P + pi;
                    const int j = psi >> 2, k = psi & 3;
                    const float2 v = code_pair<N>(lo, hi, pi);
                    acc[j][k & 1] = fma2(v, pm[(16 * j) / GV][k >> 1], acc[j][k & 1]);
                }
            }
        } else {
            const int ra = (ti - a.n_qtiles) * 16 + 2 * l4;
            const uint16_t *vr = a.vr + bh * a.R * D;
#pragma unroll
            for (int j = 0; j < NJ; ++j) {
                const int base = (4 * j) % P;
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int c = 16 * j + r8 + 8 * e;
                    const float f = static_cast<float>(1u << (N * (base + e)));
                    float2 add = make_float2(0.f, 0.f);
                    if (ra < a.r) add.x = fmaf(pa, widen(vr[ra * D + c], a.bf16), add.x);
                    if (ra + 1 < a.r) add.y = fmaf(pb, widen(vr[(ra + 1) * D + c], a.bf16), add.y);
                    if (ra + 8 < a.r) add.x = fmaf(pc, widen(vr[(ra + 8) * D + c], a.bf16), add.x);
                    if (ra + 9 < a.r) add.y = fmaf(pd, widen(vr[(ra + 9) * D + c], a.bf16), add.y);
                    acc[j][e] = fma2(add, make_float2(f, f), acc[j][e]);
                }
            }
        }
    }

    // ---- warp epilogue: o for channels 16j + r8 + 8e, unnormalised ----
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 4);
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 8);
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 16);
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
        const int base = (4 * j) % P;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const float f = 1.0f / static_cast<float>(1u << (N * (base + e)));
            float val = (acc[j][e].x + acc[j][e].y) * f - zsum[(16 * j) / GV];
            val += __shfl_xor_sync(0xffffffffu, val, 1);
            val += __shfl_xor_sync(0xffffffffu, val, 2);
            if (l4 == 0) o_s[warp][16 * j + r8 + 8 * e] = val;
        }
    }
    if (lane == 0) {
        ml_s[warp][0] = m;
        ml_s[warp][1] = lsum;
    }
    __syncthreads();

    // ---- merge the four warps, write this split's partial ----
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDecodeWarps; ++w) M = fmaxf(M, ml_s[w][0]);
    for (int c = threadIdx.x; c < D; c += kDecodeThreads) {
        float o = 0.f, l = 0.f;
#pragma unroll
        for (int w = 0; w < kDecodeWarps; ++w) {
            if (ml_s[w][0] == -INFINITY) continue;
            const float f = exp2f(ml_s[w][0] - M);
            o = fmaf(o_s[w][c], f, o);
            l = fmaf(ml_s[w][1], f, l);
        }
        a.o_part[(bq * a.S + sigma) * D + c] = o;
        if (c == 0) {
            a.m_part[bq * a.S + sigma] = M;
            a.l_part[bq * a.S + sigma] = l;
        }
    }
}

// Log-sum-exp merge of the S split partials of one (batch, query head).
__global__ void combine_kernel(const float *o_part, const float *m_part, const float *l_part,
                               float *out, int S, int D) {
    const int64_t bq = blockIdx.x;
    float M = -INFINITY;
    for (int s = 0; s < S; ++s) M = fmaxf(M, m_part[bq * S + s]);
    for (int c = threadIdx.x; c < D; c += blockDim.x) {
        float o = 0.f, l = 0.f;
        for (int s = 0; s < S; ++s) {
            const float ms = m_part[bq * S + s];
            if (ms == -INFINITY) continue;
            const float f = exp2f(ms - M);
            o = fmaf(o_part[(bq * S + s) * D + c], f, o);
            l = fmaf(l_part[bq * S + s], f, l);
        }
        out[bq * D + c] = o / l;
    }
}

template <int N, int D, int GV>
cudaError_t launch_split(const DecodeArgs &a, cudaStream_t s) {
    dim3 grid(a.S, a.Hq, a.B);
    decode_split_kernel<N, D, GV><<<grid, kDecodeThreads, 0, s>>>(a);
    count_launches(1);
    return cudaGetLastError();
}

template <int N, int D, int GV>
int occupancy() {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_split_kernel<N, D, GV>,
                                                      kDecodeThreads, 0) != cudaSuccess)
        return 1;
    return n > 0 ? n : 1;
}

// Dispatch over the compiled (bits, head_dim, value-group) variants.
template <int N, int D, int GV>
struct LaunchF {
    static cudaError_t run(const DecodeArgs &a, cudaStream_t s) { return launch_split<N, D, GV>(a, s); }
    static int occ() { return occupancy<N, D, GV>(); }
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
        case 16: return LaunchF<N, D, 16>::occ();
        case 32: return LaunchF<N, D, 32>::occ();
        case 64: return LaunchF<N, D, 64>::occ();
        default: if constexpr (D >= 128) { if (a.Gv == 128) return LaunchF<N, D, 128>::occ(); }
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
    if (e != cudaSuccess) return e;
    combine_kernel<<<static_cast<unsigned>(static_cast<int64_t>(a.B) * a.Hq), a.d, 0, s>>>(
        a.o_part, a.m_part, a.l_part, a.out, a.S, a.d);
    count_launches(1);
    return cudaGetLastError();
}

int decode_ctas_per_sm(const DecodeArgs &a) {
    if (a.bits == 2 && a.d == 64) return occ_gv<2, 64>(a);
    if (a.bits == 2 && a.d == 128) return occ_gv<2, 128>(a);
    if (a.bits == 4 && a.d == 64) return occ_gv<4, 64>(a);
    if (a.bits == 4 && a.d == 128) return occ_gv<4, 128>(a);
    return 1;
}

}  // namespace kvq
