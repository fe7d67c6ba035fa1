// quantize.cu -- KIVI quantize + pack (prefill, residual flush, LogQuant blocks),
// residual copies, the paged cache's append and the LogQuant store's compaction.
//
// One CTA quantizes one key group of G tokens of one (batch, kv-head) slice:
//   keys   : per channel over the G tokens ("LLM系列：KVCache量化1 KIVI ...",
//            section 1: Key per-channel), values: per token over Gv channels
//            (Value per-token);
//   params : asymmetric s = (max-min)/(2^n-1), z = round(-min/s),
//            code = clamp(round(x/s) + z, 0, 2^n-1), or symmetric
//            s = 2 max|x|/(2^n-1), u = clamp(round(x/s), -2^(n-1), 2^(n-1)-1) + 2^(n-1)
//            ("Atom: Low-bit Quantization ...", section 核心公式 / 量化基础, c = 1).
// Every fp32 operation that decides a code is a single IEEE round-to-nearest
// operation (explicit __f*_rn intrinsics, rintf = half-to-even), so codes,
// scales and zeros are bit-identical to a plain fp32 evaluation of the
// formulas.  A constant group takes s = |min| (1 if min = 0), which
// reconstructs it exactly.
//
// Packing writes the library's tile layout (see include/kvq.h): each output
// word is assembled from the 8-bit MMA A-fragment table (four codes of one
// row per byte group), so writes are fully coalesced and each thread produces
// whole words.  The group's rows come from consecutive tokens or from a row
// list (a LogQuant block); its output slice is a page of a paged pool when a
// page table is given; dense-and-sparse keys first move each token's largest
// entries out of the dense part.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cfloat>
#include <cstdint>
#include <type_traits>

#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr int kQuantThreads = 256;
// Largest scale the decode kernels serve: their tensor-core operands carry q s and p s times
// fixed powers of two in bf16 / fp32.  A larger scale still quantizes exactly, but raises
// status bit 4 (kvq_check_device reports it).
constexpr float kMaxServedScale = 2147483648.0f;   // 2^31

struct GroupParams {
    float s;
    int z;
};

__device__ __forceinline__ GroupParams asym_params(float mn, float mx, int bits) {
    const float L = static_cast<float>((1 << bits) - 1);
    float s;
    if (mx > mn)
        s = __fdiv_rn(__fsub_rn(mx, mn), L);
    else
        s = (mn != 0.0f) ? fabsf(mn) : 1.0f;
    const float zf = rintf(__fdiv_rn(-mn, s));
    return {s, static_cast<int>(zf)};
}

__device__ __forceinline__ float sym_scale(float amax, int bits) {
    const float L = static_cast<float>((1 << bits) - 1);
    return __fdiv_rn(__fmul_rn(2.0f, amax), L);
}

// packed fp32x2 arithmetic (sm_100): two IEEE round-to-nearest operations at once
__device__ __forceinline__ unsigned long long pack2(float2 v) {
    unsigned long long r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(v.x), "f"(v.y));
    return r;
}
__device__ __forceinline__ float2 unpack2(unsigned long long r) {
    float2 v;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(v.x), "=f"(v.y) : "l"(r));
    return v;
}
__device__ __forceinline__ float2 mul_x2(float2 a, float2 b) {
    unsigned long long d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(pack2(a)), "l"(pack2(b)));
    return unpack2(d);
}
__device__ __forceinline__ float2 add_x2(float2 a, float2 b) {
    unsigned long long d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(pack2(a)), "l"(pack2(b)));
    return unpack2(d);
}
__device__ __forceinline__ float2 sub_x2(float2 a, float2 b) {
    unsigned long long d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(pack2(a)), "l"(pack2(b)));
    return unpack2(d);
}

// One group's parameters for code_quad: code = clamp(round(x / s) + off, 0, L), with
// off = z (asymmetric) or 2^(n-1) (symmetric: clamp(round(x/s), -2^(n-1), 2^(n-1)-1) +
// 2^(n-1) is the same clamp).  ri = RN(1/s) (0 when s = 0, which gives code off).
// cut = 1/2 - 2^-18 qmax with qmax >= |x / s| over the group.  q = RN(x ri) is within
// |q| 2^-22 of RN(x / s), so both round to the same integer unless q lies within that
// distance of a half-integer; while |q - round(q)| < cut it is more than qmax 2^-18 away
// (an all-zero group has q = 0).  An element nearer a tie takes the IEEE division.
struct CodeParams {
    float s, ri, cut;
    int off;
};

__device__ __forceinline__ CodeParams code_params(float s, int off, float amax) {
    const float ri = s != 0.0f ? __frcp_rn(s) : 0.0f;
    const float qmax = amax * ri * 1.0001f;
    const float cut = fmaxf(0.5f - qmax * 0x1p-18f, 0.0f);   // 0: every element takes the division
    return {s, ri, cut, off};
}

// M = 1.5 2^23: RN(q + M + off) holds the integer nearest q + off in its low mantissa bits
constexpr float kRoundMagic = 12582912.0f;

// Codes of four elements, as the four bytes of a word.  For element i with
// ri = RN(1/s) and moff = M + off (M = 1.5 2^23), t = RN(RN(x ri) + moff) lies in
// [2^23, 2^24), so its low byte is the integer nearest RN(x ri) + off.  Away from a tie
// (|r| < cut for r = RN(x ri) - (t - moff), exact) that is rint(RN(x / s)) + off, as
// before; an element nearer a tie, or with a non-finite r, takes the IEEE
// division.  The code is at least 0 (x >= the group's minimum, and rint is odd) and at
// most L + 1 (s rounds to within 2^-24 of (max - min) / L), so the upper clamp alone
// remains: a byte with bit n set is L + 1.
struct QuadParams {
    float4 ri, moff;   // per element
    float cut;         // |r| < cut: the fast code stands (0: every element is divided)
};

// Codes of x.x .. x.w as the four bytes of a word; s4 / off4 (per element) serve the
// elements that take the division.
template <int N>
__device__ __forceinline__ uint32_t code_quad(const float4 &x, const QuadParams &p, const float4 &s4,
                                              const int4 &off4) {
    constexpr int L = (1 << N) - 1;
    const float2 q01 = mul_x2(make_float2(x.x, x.y), make_float2(p.ri.x, p.ri.y));
    const float2 q23 = mul_x2(make_float2(x.z, x.w), make_float2(p.ri.z, p.ri.w));
    const float2 t01 = add_x2(q01, make_float2(p.moff.x, p.moff.y));
    const float2 t23 = add_x2(q23, make_float2(p.moff.z, p.moff.w));
    const float2 r01 = add_x2(q01, sub_x2(make_float2(p.moff.x, p.moff.y), t01));   // moff - t: exact
    const float2 r23 = add_x2(q23, sub_x2(make_float2(p.moff.z, p.moff.w), t23));
    uint32_t w = __byte_perm(__byte_perm(__float_as_uint(t01.x), __float_as_uint(t01.y), 0x0040),
                             __byte_perm(__float_as_uint(t23.x), __float_as_uint(t23.y), 0x0040), 0x5410);
    const bool near = !(fabsf(r01.x) < p.cut) || !(fabsf(r01.y) < p.cut) || !(fabsf(r23.x) < p.cut) ||
                      !(fabsf(r23.y) < p.cut);
    if (near) {
        const float xs[4] = {x.x, x.y, x.z, x.w}, ss[4] = {s4.x, s4.y, s4.z, s4.w};
        const float rs[4] = {r01.x, r01.y, r23.x, r23.y};
        const int os[4] = {off4.x, off4.y, off4.z, off4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            if (!(fabsf(rs[e]) < p.cut)) {
                const int c = static_cast<int>(rintf(__fdiv_rn(xs[e], ss[e]))) + os[e];
                w = (w & ~(0xffu << (8 * e))) | (static_cast<uint32_t>(min(max(c, 0), L + 1)) << (8 * e));
            }
        }
    }
    constexpr uint32_t kOver = 0x01010101u << N;   // bit n of every byte: the code L + 1
    return w - ((w & kOver) >> N);                 // L + 1 -> L: 1 off each such byte, no borrow
}

// Assemble the packed words of `ntiles` 16-token tiles from byte codes
// codes[t * D + c] (t relative to the first tile) and store them at dst.
// Word w of a tile belongs to lane w / W; its slot s (0 .. 8/N - 1) holds, in
// byte b, the element (row = lane/4 + 8*(s%2), col = 4*(lane%4) + b) of block
// (chunk) j = (w % W) * (4/N) + s/2 at bit 8*b + N*s.  Every code is below 2^N, so a
// slot's four bytes shifted by N*s stay inside their bytes.  For keys (rows = tokens,
// columns = channels) a row's four columns are four consecutive channels: one 32-bit
// load of codes per slot.
template <int D, int N>
__device__ void pack_key_tiles(const uint8_t *codes, int ntiles, uint32_t *dst) {
    constexpr int TW = D * N / 2;        // words per tile
    constexpr int W = D * N / 64;        // words per lane
    constexpr int B = 4 / N;             // blocks per word
    const int total = ntiles * TW;
    for (int wi = threadIdx.x; wi < total; wi += blockDim.x) {
        const int tile = wi / TW;
        const int w = wi - tile * TW;
        const int lane = w / W;
        const int wl = w - lane * W;
        uint32_t word = 0;
#pragma unroll
        for (int slot = 0; slot < 2 * B; ++slot) {
            const int j = wl * B + (slot >> 1);
            const int row = (lane >> 2) + 8 * (slot & 1);
            const int col0 = 4 * (lane & 3);
            const uint32_t v = *reinterpret_cast<const uint32_t *>(codes + (tile * 16 + row) * D + 16 * j + col0);
            word |= v << (N * slot);
        }
        dst[wi] = word;
    }
}

// The same words for values (rows = channels, columns = tokens), four at a time.  The words of lanes
// q + 4k + 16h (k = 0 .. 3) at word wl share their tokens (4q .. 4q + 3) and hold, slot by
// slot, four consecutive channels c0 + k: one 32-bit load per token brings a 4 x 4 block of
// codes, and a byte transpose in registers gives the four words' bytes.  Thread (q, h) takes
// the slots from slot q on, so the loads of a warp spread over the banks.
template <int D, int N>
__device__ void pack_value_tiles(const uint8_t *codes, int ntiles, uint32_t *dst) {
    constexpr int TW = D * N / 2;        // words per tile
    constexpr int W = D * N / 64;        // words per lane
    constexpr int B = 4 / N;             // blocks per word
    constexpr int NS = 2 * B;            // slots per word
    constexpr int TPT = TW / 4;          // threads per tile: (wl, q, h)
    const int total = ntiles * TPT;
    for (int i = threadIdx.x; i < total; i += blockDim.x) {
        const int tile = i / TPT;
        const int r = i - tile * TPT;
        const int wl = r % W, q = (r / W) & 3, h = r / (4 * W);
        const uint8_t *rows = codes + (tile * 16 + 4 * q) * D;
        uint32_t word[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int step = 0; step < NS; ++step) {
            const int slot = (step + q) % NS;
            const int c0 = 16 * (wl * B + (slot >> 1)) + 8 * (slot & 1) + 4 * h;
            uint32_t in[4];
#pragma unroll
            for (int b = 0; b < 4; ++b) in[b] = *reinterpret_cast<const uint32_t *>(rows + b * D + c0);
            // out[k] byte b = in[b] byte k
            const uint32_t t0 = __byte_perm(in[0], in[1], 0x5140), t1 = __byte_perm(in[0], in[1], 0x7362);
            const uint32_t t2 = __byte_perm(in[2], in[3], 0x5140), t3 = __byte_perm(in[2], in[3], 0x7362);
            const int sh = N * slot;
            word[0] |= __byte_perm(t0, t2, 0x5410) << sh;
            word[1] |= __byte_perm(t0, t2, 0x7632) << sh;
            word[2] |= __byte_perm(t1, t3, 0x5410) << sh;
            word[3] |= __byte_perm(t1, t3, 0x7632) << sh;
        }
        uint32_t *out = dst + tile * TW + (q + 16 * h) * W + wl;
#pragma unroll
        for (int k = 0; k < 4; ++k) out[4 * k * W] = word[k];
    }
}

// Two 16-bit elements (a 32-bit word, low half first) as floats.
__device__ __forceinline__ float2 widen2(uint32_t v, bool bf16) {
    if (bf16) return make_float2(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u));
    return __half22float2(*reinterpret_cast<const __half2 *>(&v));
}

// Element-wise minimum and maximum (sym: maximum magnitude, returned in hi) of n packed
// pairs p[0], p[stride], ...: exact in the 16-bit type.
template <bool BF16>
__device__ __forceinline__ void pair_minmax(const uint32_t *p, int stride, int n, bool sym, uint32_t &lo,
                                            uint32_t &hi) {
    using T2 = typename std::conditional<BF16, __nv_bfloat162, __half2>::type;
    T2 l = *reinterpret_cast<const T2 *>(p), h = l;
    if (sym) {
        h = __habs2(h);
        for (int i = 1; i < n; ++i) h = __hmax2(h, __habs2(*reinterpret_cast<const T2 *>(p + i * stride)));
    } else {
        for (int i = 1; i < n; ++i) {
            const T2 v = *reinterpret_cast<const T2 *>(p + i * stride);
            l = __hmin2(l, v);
            h = __hmax2(h, v);
        }
    }
    lo = *reinterpret_cast<const uint32_t *>(&l);
    hi = *reinterpret_cast<const uint32_t *>(&h);
}

// n consecutive 32-bit words from shared memory in one vector load (n = 2 or 4)
template <int n>
__device__ __forceinline__ void load_words(const uint32_t *p, uint32_t (&w)[n]) {
    static_assert(n == 2 || n == 4, "words");
    if constexpr (n == 4) {
        const uint4 v = *reinterpret_cast<const uint4 *>(p);
        w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else {
        const uint2 v = *reinterpret_cast<const uint2 *>(p);
        w[0] = v.x; w[1] = v.y;
    }
}

// Copy the G rows of d 16-bit elements of one group into shared memory with 16-byte
// loads: rows tok0 .. tok0+G-1 of `slice`, or rows rows[0 .. G-1] when rows is non-NULL.
// Each thread issues up to kLoadBatch loads before it stores any, so a group arrives in
// about one memory latency instead of one per load.
constexpr int kLoadBatch = 8;

__device__ void load_group(const uint16_t *slice, int64_t tok0, const int32_t *rows, int64_t row_limit,
                           unsigned int *status, uint16_t *dst, int G, int d) {
    const int vec = d / 8, vshift = d == 64 ? 3 : 4;   // d is 64 or 128
    const int total = G * vec;
    uint4 *d4 = reinterpret_cast<uint4 *>(dst);
    for (int base = threadIdx.x; base < total; base += kLoadBatch * blockDim.x) {
        uint4 v[kLoadBatch];
#pragma unroll
        for (int k = 0; k < kLoadBatch; ++k) {
            const int i = base + k * blockDim.x;
            if (i < total) {
                const int t = i >> vshift, c = i & (vec - 1);
                int64_t row = rows ? rows[t] : tok0 + t;
                if constexpr (kCheck) {
                    if (rows && (row < 0 || row >= row_limit)) {
                        atomicOr(status, 8u);
                        row = 0;
                    }
                }
                v[k] = __ldcs(reinterpret_cast<const uint4 *>(slice + row * d) + c);   // read once: stream
            }
        }
#pragma unroll
        for (int k = 0; k < kLoadBatch; ++k) {
            const int i = base + k * blockDim.x;
            if (i < total) d4[i] = v[k];
        }
    }
}

// BATCH: the value parameters batched per warp (groups of 64 tokens or more, four or more
// token pairs per warp); else computed per token pair.  UNROLL: the value phase's token-pair
// loops unrolled by two (eight or more token pairs per warp).  BF16: the inputs are bf16, else
// fp16.
template <int D, int N, bool BATCH, bool UNROLL, bool BF16>
__global__ void __launch_bounds__(kQuantThreads, 4) quantize_pack_kernel(const QuantizeArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    constexpr int d = D, bits = N;
    const int GK = a.G;                            // key group
    const int G = a.gpc * GK;                      // tokens of the CTA: gpc key groups
    uint16_t *xs = reinterpret_cast<uint16_t *>(smem);                       // [G][d]
    uint8_t *codes = smem + static_cast<size_t>(G) * d * 2;                  // [G][d]
    float *red = reinterpret_cast<float *>(codes + static_cast<size_t>(G) * d);  // 2*256
    float *ch_s = red + 2 * kQuantThreads;                                   // [d]
    int *ch_z = reinterpret_cast<int *>(ch_s + d);                           // [d]
    float *ch_r = reinterpret_cast<float *>(ch_z + d);                       // [d] 1/s
    float *ch_c = ch_r + d;                                                  // [d] near-tie bound
    // value groups: [G][d / Gv] entries of 4 floats: (min, max), then (RN(1/s), M + off, cut, s)
    float4 *vg = reinterpret_cast<float4 *>(ch_c + d);

    const int64_t grp = blockIdx.x;
    const int64_t bh = blockIdx.y;                 // input slice
    const int64_t in_tok = a.in_tok0 + grp * G;
    int64_t out_tok = a.out_tok0 + grp * G;
    int64_t slice = bh, cap = a.cap;               // output slice and its token capacity
    if (a.page_table) {
        // paged pool: the group's page of its sequence (groups never straddle pages)
        const int64_t b = a.seq0 + bh / a.Hkv;
        if (a.seq_len) {                           // flush: only sequences whose residual just filled
            const int64_t len = a.seq_len[b], R = a.n_groups * GK;
            if (len <= 0 || len % R != 0) return;
            out_tok = len - R + grp * G;
        }
        const int64_t pi = out_tok / a.cap;
        const int page = pi < a.max_pages ? a.page_table[b * a.max_pages + pi] : -1;
        if (page < 0 || page >= a.num_pages) {    // not a page of the pool: write nothing
            if (threadIdx.x == 0) atomicOr(a.status, 2u);
            return;
        }
        slice = static_cast<int64_t>(page) * a.Hkv + bh % a.Hkv;
        out_tok -= pi * a.cap;
    }
    const int TW = tile_words(d, bits);
    const int64_t words_per_slice = cap / 16 * TW;
    const int64_t groups_cap = cap / GK;

    // ------------------------------ keys ------------------------------
    const int32_t *rows = a.in_rows ? a.in_rows + grp * G : nullptr;
    load_group(a.xk + bh * a.in_bh_stride, in_tok, rows, a.in_rows_limit, a.status, xs, G, d);
    __syncthreads();
    if (a.n_out > 0) {
        // dense-and-sparse keys: per token, the n_out entries of largest magnitude (ties: the
        // lower channel) are written as outlier words and set to +0 in the dense part
        const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
        const int per_lane = d / 32;                 // 2 or 4
        for (int t = warp; t < G; t += kQuantThreads / 32) {
            uint32_t mag[4];
            for (int e = 0; e < per_lane; ++e)
                mag[e] = __float_as_uint(fabsf(widen(xs[t * d + lane * per_lane + e], BF16)));
            unsigned picked = 0;
            for (int o = 0; o < a.n_out; ++o) {
                uint64_t best = 0;   // (|x| bits << 16) | (0xffff - channel): the larger key wins
                for (int e = 0; e < per_lane; ++e) {
                    const uint64_t key = (static_cast<uint64_t>(mag[e]) << 16) |
                                         static_cast<uint64_t>(0xffff - (lane * per_lane + e));
                    if (!((picked >> e) & 1u) && key > best) best = key;
                }
                for (int off = 16; off > 0; off >>= 1) {
                    const uint64_t other = __shfl_xor_sync(0xffffffffu, best, off);
                    best = other > best ? other : best;
                }
                const int c = 0xffff - static_cast<int>(best & 0xffffu);
                if (c / per_lane == lane) picked |= 1u << (c % per_lane);
                if (lane == 0)
                    a.k_out[(slice * cap + out_tok + t) * a.n_out + o] =
                        (static_cast<uint32_t>(c) << 16) | xs[t * d + c];
            }
            __syncwarp();    // every lane has read the chosen elements' bits
            for (int e = 0; e < per_lane; ++e)
                if ((picked >> e) & 1u) xs[t * d + lane * per_lane + e] = 0;
        }
        __syncthreads();
    }
    for (int kg = 0; kg < a.gpc; ++kg) {
        // key group kg of the CTA (rows kg GK .. kg GK + GK - 1)
        // per-channel minimum and maximum (or largest magnitude) over the GK tokens: thread
        // (channel pair cp, part) scans its part with packed 16-bit min / max, which are
        // exact; the parts meet in shared memory
        constexpr int NP = D / 2;                    // channel pairs
        constexpr int parts = kQuantThreads / NP;    // 4 (d = 128) or 8 (d = 64); G >= 16
        const int cp = threadIdx.x % NP, part = threadIdx.x / NP;
        const uint32_t *xw = reinterpret_cast<const uint32_t *>(xs) + kg * GK * NP;   // [GK][NP] pairs
        const int per = GK / parts;
        uint32_t lo, hi;
        pair_minmax<BF16>(xw + (part * per) * NP + cp, NP, per, a.sym, lo, hi);
        uint32_t *redu = reinterpret_cast<uint32_t *>(red);
        redu[threadIdx.x] = lo;
        redu[kQuantThreads + threadIdx.x] = hi;
        __syncthreads();
        if (threadIdx.x < d) {
            const int c = threadIdx.x, pc = c >> 1, sh = 16 * (c & 1);
            float mn = FLT_MAX, mx = -FLT_MAX;
            for (int p = 0; p < parts; ++p) {
                mn = fminf(mn, widen(static_cast<uint16_t>(redu[p * NP + pc] >> sh), BF16));
                mx = fmaxf(mx, widen(static_cast<uint16_t>(redu[kQuantThreads + p * NP + pc] >> sh), BF16));
            }
            float s;
            int z;
            if (a.sym) {
                s = sym_scale(mx, bits);
                z = 1 << (bits - 1);
            } else {
                const GroupParams gp = asym_params(mn, mx, bits);
                s = gp.s;
                z = gp.z;
                a.kz[(slice * groups_cap + out_tok / GK + kg) * d + c] = static_cast<int16_t>(z);
            }
            a.ks[(slice * groups_cap + out_tok / GK + kg) * d + c] = s;
            if (s > kMaxServedScale) atomicOr(a.status, 4u);
            const CodeParams cp = code_params(s, z, a.sym ? mx : fmaxf(fabsf(mn), fabsf(mx)));
            ch_s[c] = s;
            ch_z[c] = z;
            ch_r[c] = cp.ri;
            ch_c[c] = cp.cut;
        }
        __syncthreads();
        {   // codes: thread (cp, part) takes channels 2 cp, 2 cp + 1 of rows part, part + parts, ...,
            // two rows at a time (GK / parts is even)
            QuadParams qp;
            const float r0 = ch_r[2 * cp], r1 = ch_r[2 * cp + 1];
            const int z0 = ch_z[2 * cp], z1 = ch_z[2 * cp + 1];
            qp.ri = make_float4(r0, r1, r0, r1);
            qp.moff = make_float4(kRoundMagic + z0, kRoundMagic + z1, kRoundMagic + z0, kRoundMagic + z1);
            qp.cut = fminf(ch_c[2 * cp], ch_c[2 * cp + 1]);
            const float4 s4 = make_float4(ch_s[2 * cp], ch_s[2 * cp + 1], ch_s[2 * cp], ch_s[2 * cp + 1]);
            const int4 o4 = make_int4(z0, z1, z0, z1);
            uint8_t *kcodes = codes + kg * GK * d;
            for (int t = part; t < GK; t += 2 * parts) {
                const float2 x0 = widen2(xw[t * NP + cp], BF16), x1 = widen2(xw[(t + parts) * NP + cp], BF16);
                const uint32_t w = code_quad<N>(make_float4(x0.x, x0.y, x1.x, x1.y), qp, s4, o4);
                *reinterpret_cast<uint16_t *>(kcodes + t * d + 2 * cp) = static_cast<uint16_t>(w & 0xffffu);
                *reinterpret_cast<uint16_t *>(kcodes + (t + parts) * d + 2 * cp) = static_cast<uint16_t>(w >> 16);
            }
        }
        __syncthreads();
    }
    pack_key_tiles<D, N>(codes, G / 16, a.kc + slice * words_per_slice + (out_tok / 16) * TW);
    __syncthreads();

    // ------------------------------ values ----------------------------
    load_group(a.xv + bh * a.in_bh_stride, in_tok, rows, a.in_rows_limit, a.status, xs, G, d);
    __syncthreads();
    {
        // one token per half-warp (two per warp).  With four or more token pairs per warp, a warp
        // first takes the minimum and maximum of every value group of its tokens (segment
        // reductions over the lanes of a group), then computes the parameters (the IEEE
        // divisions) with one lane per (token, group), so that one pass of that code serves up
        // to 32 groups, then the codes.  With fewer, each token pair's lanes compute their
        // groups' parameters themselves.
        constexpr int per_lane = d / 16;             // contiguous channels per lane: 8 or 4
        const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
        const int half = (threadIdx.x >> 4) & 1, hl = threadIdx.x & 15;
        const int seg = a.Gv / per_lane;             // lanes per value group (power of 2, <= 16)
        const int ngv = d / a.Gv;
        const int j = hl / seg;                      // this lane's group in its token
        constexpr int kWarps = kQuantThreads / 32;
        if constexpr (BATCH) {       // four or more token pairs per warp: parameters batched
#pragma unroll(UNROLL ? 2 : 1)
            for (int tp = warp; tp < G / 2; tp += kWarps) {
                const int t = 2 * tp + half;
                uint32_t w[per_lane / 2];
                load_words<per_lane / 2>(reinterpret_cast<const uint32_t *>(xs + t * d + hl * per_lane), w);
                uint32_t lo, hi;
                pair_minmax<BF16>(w, 1, per_lane / 2, a.sym, lo, hi);
                const float2 l2 = widen2(lo, BF16), h2 = widen2(hi, BF16);
                float mn = fminf(l2.x, l2.y), mx = fmaxf(h2.x, h2.y);
                for (int off = seg >> 1; off > 0; off >>= 1) {
                    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
                }
                if (hl % seg == 0) vg[t * ngv + j] = make_float4(mn, mx, 0.f, 0.f);
            }
            __syncwarp();
            // the warp's (token, group) pairs: token pairs tp = warp + kWarps i, both tokens, every group
            const int n_pairs = ((G / 2 - warp + kWarps - 1) / kWarps) * 2 * ngv;
            for (int q = lane; q < n_pairs; q += 32) {
                const int i = q / (2 * ngv), hq = (q / ngv) % 2, jq = q % ngv;
                const int t = 2 * (warp + kWarps * i) + hq;
                const float4 e = vg[t * ngv + jq];
                const float mn = e.x, mx = e.y;
                float s;
                int z;
                if (a.sym) {
                    s = sym_scale(mx, bits);
                    z = 0;
                } else {
                    const GroupParams gp = asym_params(mn, mx, bits);
                    s = gp.s;
                    z = gp.z;
                }
                const int64_t mi = (slice * cap + out_tok + t) * ngv + jq;
                a.vs[mi] = s;
                if (!a.sym) a.vz[mi] = static_cast<int16_t>(z);
                if (s > kMaxServedScale) atomicOr(a.status, 4u);
                const CodeParams cp = code_params(s, a.sym ? (1 << (bits - 1)) : z,
                                                  a.sym ? mx : fmaxf(fabsf(mn), fabsf(mx)));
                vg[t * ngv + jq] = make_float4(cp.ri, kRoundMagic + static_cast<float>(cp.off), cp.cut, cp.s);
            }
            __syncwarp();
#pragma unroll(UNROLL ? 2 : 1)
            for (int tp = warp; tp < G / 2; tp += kWarps) {
                const int t = 2 * tp + half;
                uint32_t w[per_lane / 2];
                load_words<per_lane / 2>(reinterpret_cast<const uint32_t *>(xs + t * d + hl * per_lane), w);
                const float4 e = vg[t * ngv + j];
                QuadParams qp;
                qp.ri = make_float4(e.x, e.x, e.x, e.x);
                qp.moff = make_float4(e.y, e.y, e.y, e.y);
                qp.cut = e.z;
                const float4 s4 = make_float4(e.w, e.w, e.w, e.w);
                const int off = static_cast<int>(e.y - kRoundMagic);
                const int4 o4 = make_int4(off, off, off, off);
    #pragma unroll
                for (int k = 0; k < per_lane / 4; ++k) {
                    const float2 x0 = widen2(w[2 * k], BF16), x1 = widen2(w[2 * k + 1], BF16);
                    reinterpret_cast<uint32_t *>(codes + t * d + hl * per_lane)[k] =
                        code_quad<N>(make_float4(x0.x, x0.y, x1.x, x1.y), qp, s4, o4);
                }
            }
        } else {                     // short groups: parameters per token pair, as they come
            for (int tp = warp; tp < G / 2; tp += kQuantThreads / 32) {
                const int t = 2 * tp + half;
                float x[per_lane];
                float mn = FLT_MAX, mx = -FLT_MAX;
                uint16_t xb[per_lane];
                if constexpr (per_lane == 8) {
                    const uint4 v = *reinterpret_cast<const uint4 *>(xs + t * d + hl * per_lane);
                    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    #pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        xb[2 * k] = static_cast<uint16_t>(w[k] & 0xffffu);
                        xb[2 * k + 1] = static_cast<uint16_t>(w[k] >> 16);
                    }
                } else {
                    const uint2 v = *reinterpret_cast<const uint2 *>(xs + t * d + hl * per_lane);
                    xb[0] = static_cast<uint16_t>(v.x & 0xffffu);
                    xb[1] = static_cast<uint16_t>(v.x >> 16);
                    xb[2] = static_cast<uint16_t>(v.y & 0xffffu);
                    xb[3] = static_cast<uint16_t>(v.y >> 16);
                }
    #pragma unroll
                for (int e = 0; e < per_lane; ++e) {
                    x[e] = widen(xb[e], BF16);
                    if (a.sym) {
                        mx = fmaxf(mx, fabsf(x[e]));
                    } else {
                        mn = fminf(mn, x[e]);
                        mx = fmaxf(mx, x[e]);
                    }
                }
                for (int off = seg >> 1; off > 0; off >>= 1) {
                    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
                }
                float s;
                int z;
                if (a.sym) {
                    s = sym_scale(mx, bits);
                    z = 0;
                } else {
                    const GroupParams gp = asym_params(mn, mx, bits);
                    s = gp.s;
                    z = gp.z;
                }
                const int j = hl / seg;
                if (hl % seg == 0) {
                    const int64_t mi = (slice * cap + out_tok + t) * ngv + j;
                    a.vs[mi] = s;
                    if (!a.sym) a.vz[mi] = static_cast<int16_t>(z);
                    if (s > kMaxServedScale) atomicOr(a.status, 4u);
                }
                const CodeParams cp = code_params(s, a.sym ? (1 << (bits - 1)) : z,
                                                  a.sym ? mx : fmaxf(fabsf(mn), fabsf(mx)));
                QuadParams qp;
                qp.ri = make_float4(cp.ri, cp.ri, cp.ri, cp.ri);
                const float mo = kRoundMagic + static_cast<float>(cp.off);
                qp.moff = make_float4(mo, mo, mo, mo);
                qp.cut = cp.cut;
                const float4 s4 = make_float4(cp.s, cp.s, cp.s, cp.s);
                const int4 o4 = make_int4(cp.off, cp.off, cp.off, cp.off);
    #pragma unroll
                for (int k = 0; k < per_lane / 4; ++k)
                    reinterpret_cast<uint32_t *>(codes + t * d + hl * per_lane)[k] =
                        code_quad<N>(make_float4(x[4 * k], x[4 * k + 1], x[4 * k + 2], x[4 * k + 3]), qp, s4, o4);
            }
        }
        __syncthreads();
        pack_value_tiles<D, N>(codes, G / 16, a.vc + slice * words_per_slice + (out_tok / 16) * TW);
    }
}

__global__ void copy_rows_kernel(const uint16_t *src0, const uint16_t *src1, int64_t src_bh_stride,
                                 int64_t src_row0, uint16_t *dst0, uint16_t *dst1,
                                 int64_t dst_bh_stride, int64_t dst_row0, int64_t rows,
                                 int64_t BH, int d) {
    const int64_t vec_per_row = d / 8;
    const int64_t per_pair = BH * rows * vec_per_row;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < 2 * per_pair;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const bool second = i >= per_pair;
        const int64_t k = second ? i - per_pair : i;
        const int64_t v = k % vec_per_row;
        const int64_t row = (k / vec_per_row) % rows;
        const int64_t bh = k / (vec_per_row * rows);
        const uint16_t *src = second ? src1 : src0;
        uint16_t *dst = second ? dst1 : dst0;
        const uint4 *sp = reinterpret_cast<const uint4 *>(src + bh * src_bh_stride +
                                                          (src_row0 + row) * d) + v;
        uint4 *tp = reinterpret_cast<uint4 *>(dst + bh * dst_bh_stride + (dst_row0 + row) * d) + v;
        *tp = *sp;
    }
}

// LogQuant compaction of one (b, h) slice per CTA, in place: row 2i -> row i (i < W) and
// row 2W + j -> row W + j (j < W).  Every destination row is at or below its source, so
// moving the rows in ascending order never overwrites a row before it is read; each
// wave of rows is read whole before any of it is written.
__global__ void lq_compact_kernel(uint16_t *kr, uint16_t *vr, int rows, int W, int d, unsigned int *status) {
    const int64_t bh = blockIdx.x;
    const int vec = d / 8;
    const int per_wave = blockDim.x / vec;                 // destination rows per wave
    uint4 *k4 = reinterpret_cast<uint4 *>(kr + bh * rows * d);
    uint4 *v4 = reinterpret_cast<uint4 *>(vr + bh * rows * d);
    const int r = threadIdx.x / vec, c = threadIdx.x % vec;
    for (int base = 0; base < 2 * W; base += per_wave) {
        const int dst = base + r;
        bool on = r < per_wave && dst < 2 * W;
        const int src = dst < W ? 2 * dst : W + dst;
        if constexpr (kCheck) {
            if (on && (src >= rows || dst >= rows)) {
                atomicOr(status, 8u);
                on = false;
            }
        }
        uint4 kx = make_uint4(0, 0, 0, 0), vx = kx;
        if (on) {
            kx = k4[src * vec + c];
            vx = v4[src * vec + c];
        }
        __syncthreads();
        if (on) {
            k4[dst * vec + c] = kx;
            v4[dst * vec + c] = vx;
        }
        __syncthreads();
    }
}

__global__ void gather_rows_kernel(const uint16_t *srck, const uint16_t *srcv, int64_t src_bh_stride,
                                   int64_t src_rows, const int32_t *idx, int n, uint16_t *dstk, uint16_t *dstv,
                                   int64_t dst_bh_stride, int64_t BH, int d, unsigned int *status) {
    const int64_t vec = d / 8, per = BH * n * vec;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < 2 * per;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const bool isv = i >= per;
        const int64_t k = isv ? i - per : i;
        const int64_t v = k % vec, row = (k / vec) % n, bh = k / (vec * n);
        int64_t src = idx[row];
        if constexpr (kCheck) {
            if (src < 0 || src >= src_rows) {
                atomicOr(status, 8u);
                src = 0;
            }
        }
        const uint4 x = reinterpret_cast<const uint4 *>((isv ? srcv : srck) + bh * src_bh_stride + src * d)[v];
        reinterpret_cast<uint4 *>((isv ? dstv : dstk) + bh * dst_bh_stride + row * d)[v] = x;
    }
}

// Paged append: CTA b copies the new rows of all kv heads of sequence b (if active) into
// residual row seq_len[b] mod R, then advances seq_len[b].
__global__ void paged_append_kernel(const uint16_t *tk, const uint16_t *tv, uint16_t *kr, uint16_t *vr,
                                    int32_t *seq_len, int Hkv, int R, int d) {
    const int b = blockIdx.x;
    const int len = seq_len[b];
    if (len < 0) return;
    const int row = len % R;
    const int vec = d / 8, per_seq = Hkv * vec;
    for (int i = threadIdx.x; i < 2 * per_seq; i += blockDim.x) {
        const bool isv = i >= per_seq;
        const int k = isv ? i - per_seq : i;
        const int h = k / vec, v = k % vec;
        const int64_t bh = static_cast<int64_t>(b) * Hkv + h;
        const uint4 x = reinterpret_cast<const uint4 *>((isv ? tv : tk) + bh * d)[v];
        reinterpret_cast<uint4 *>((isv ? vr : kr) + (bh * R + row) * d)[v] = x;
    }
    __syncthreads();   // every thread has read seq_len[b]
    if (threadIdx.x == 0) seq_len[b] = len + 1;
}

// Paged prefill tail: rows [row0, row0 + rows) of X_K / X_V ([Hkv][T][d]) become residual
// rows 0 .. rows-1 of sequence seq; seq_len[seq] = value.
__global__ void paged_residual_kernel(const uint16_t *xk, const uint16_t *xv, int64_t T, int64_t row0,
                                      int64_t rows, uint16_t *kr, uint16_t *vr, int32_t *seq_len, int seq,
                                      int32_t value, int Hkv, int R, int d) {
    const int64_t vec = d / 8, per = static_cast<int64_t>(Hkv) * rows * vec;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < 2 * per;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const bool isv = i >= per;
        const int64_t k = isv ? i - per : i;
        const int64_t v = k % vec, row = (k / vec) % rows, h = k / (vec * rows);
        const uint4 x = reinterpret_cast<const uint4 *>((isv ? xv : xk) + (h * T + row0 + row) * d)[v];
        reinterpret_cast<uint4 *>((isv ? vr : kr) + ((static_cast<int64_t>(seq) * Hkv + h) * R + row) * d)[v] = x;
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) seq_len[seq] = value;
}

}  // namespace

size_t quantize_smem_bytes(int d, int G, int Gv) {
    return static_cast<size_t>(G) * d * 3 + 2 * kQuantThreads * sizeof(float) +
           static_cast<size_t>(d) * 16 + static_cast<size_t>(G) * (d / Gv) * 16;
}

using QuantizeKernel = void (*)(const QuantizeArgs);
template <int D, int N>
QuantizeKernel quantize_instance(bool batch, bool unroll, bool bf16) {
    if (bf16) {
        if (!batch) return quantize_pack_kernel<D, N, false, false, true>;
        return unroll ? quantize_pack_kernel<D, N, true, true, true> : quantize_pack_kernel<D, N, true, false, true>;
    }
    if (!batch) return quantize_pack_kernel<D, N, false, false, false>;
    return unroll ? quantize_pack_kernel<D, N, true, true, false> : quantize_pack_kernel<D, N, true, false, false>;
}

cudaError_t launch_quantize(const QuantizeArgs &a, cudaStream_t s) {
    if (a.n_groups == 0 || a.BH == 0) return cudaSuccess;
    // short key groups of a contiguous cache go two to a CTA, so a CTA streams 64 tokens and
    // the value parameters are batched (paged pools and row lists keep one group per CTA)
    QuantizeArgs b = a;
    b.gpc = (a.G / 2 < 4 * (kQuantThreads / 32) && a.n_groups % 2 == 0 && !a.page_table && !a.in_rows) ? 2 : 1;
    const int tokens = b.gpc * a.G;
    const size_t smem = quantize_smem_bytes(a.d, tokens, a.Gv);
    void (*kernel)(const QuantizeArgs) = nullptr;
    int variant = -1;
    const bool batch = tokens / 2 >= 4 * (kQuantThreads / 32);
    const bool unroll = tokens / 2 >= 8 * (kQuantThreads / 32);
    if (a.d == 64 && a.bits == 2) kernel = quantize_instance<64, 2>(batch, unroll, a.bf16), variant = 0;
    else if (a.d == 64 && a.bits == 4) kernel = quantize_instance<64, 4>(batch, unroll, a.bf16), variant = 1;
    else if (a.d == 128 && a.bits == 2) kernel = quantize_instance<128, 2>(batch, unroll, a.bf16), variant = 2;
    else if (a.d == 128 && a.bits == 4) kernel = quantize_instance<128, 4>(batch, unroll, a.bf16), variant = 3;
    if (!kernel) return cudaErrorInvalidValue;
    variant = 6 * variant + (a.bf16 ? 3 : 0) + (batch ? (unroll ? 2 : 1) : 0);
    // opt in to the largest dynamic shared memory any configuration needs, once per device and variant
    static bool configured[64][24] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 64 || !configured[dev][variant]) {
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(quantize_smem_bytes(256, 128, 16)));
        if (e != cudaSuccess) return e;
        if (dev < 64) configured[dev][variant] = true;
    }
    dim3 grid(static_cast<unsigned>(a.n_groups / b.gpc), static_cast<unsigned>(a.BH));
    kernel<<<grid, kQuantThreads, smem, s>>>(b);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_copy_rows(const uint16_t *src0, const uint16_t *src1, int64_t src_bh_stride,
                             int64_t src_row0, uint16_t *dst0, uint16_t *dst1,
                             int64_t dst_bh_stride, int64_t dst_row0, int64_t rows, int64_t BH,
                             int d, cudaStream_t s) {
    const int64_t total = 2 * BH * rows * (d / 8);
    if (total == 0) return cudaSuccess;
    const int threads = 256;
    const int64_t blocks = (total + threads - 1) / threads;
    copy_rows_kernel<<<static_cast<unsigned>(blocks < 65536 ? blocks : 65536), threads, 0, s>>>(
        src0, src1, src_bh_stride, src_row0, dst0, dst1, dst_bh_stride, dst_row0, rows, BH, d);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace kvq

namespace kvq {

cudaError_t launch_paged_append(const uint16_t *tk, const uint16_t *tv, uint16_t *kr, uint16_t *vr,
                                int32_t *seq_len, int B, int Hkv, int R, int d, cudaStream_t s) {
    if (B == 0) return cudaSuccess;
    paged_append_kernel<<<B, 128, 0, s>>>(tk, tv, kr, vr, seq_len, Hkv, R, d);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_paged_residual(const uint16_t *xk, const uint16_t *xv, int64_t T, int64_t row0,
                                  int64_t rows, uint16_t *kr, uint16_t *vr, int32_t *seq_len, int seq,
                                  int32_t value, int Hkv, int R, int d, cudaStream_t s) {
    const int64_t total = 2 * static_cast<int64_t>(Hkv) * rows * (d / 8);
    const int64_t blocks = total > 0 ? (total + 255) / 256 : 1;
    paged_residual_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(xk, xv, T, row0, rows, kr, vr, seq_len,
                                                                        seq, value, Hkv, R, d);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace kvq

namespace kvq {

cudaError_t launch_lq_compact(uint16_t *kr, uint16_t *vr, int64_t BH, int rows, int W, int d, unsigned int *status,
                              cudaStream_t s) {
    if (BH == 0) return cudaSuccess;
    lq_compact_kernel<<<static_cast<unsigned>(BH), 256, 0, s>>>(kr, vr, rows, W, d, status);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_gather_rows(const uint16_t *srck, const uint16_t *srcv, int64_t src_bh_stride,
                               int64_t src_rows, const int32_t *idx, int n, uint16_t *dstk, uint16_t *dstv,
                               int64_t dst_bh_stride, int64_t BH, int d, unsigned int *status, cudaStream_t s) {
    const int64_t total = 2 * BH * n * (d / 8);
    if (total == 0) return cudaSuccess;
    const int64_t blocks = (total + 255) / 256;
    gather_rows_kernel<<<static_cast<unsigned>(blocks < 65536 ? blocks : 65536), 256, 0, s>>>(
        srck, srcv, src_bh_stride, src_rows, idx, n, dstk, dstv, dst_bh_stride, BH, d, status);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace kvq
