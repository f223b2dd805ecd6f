// Selection helpers shared by the select and decode kernels.
//
// Activation-sparsity overview page (激活稀疏化技术：提升LLM推理效率的动态剪枝方法)
// section 2.1 / 2.2.1: keep N of every M consecutive channels by score; the
// page's snippet keeps everything >= the N-th value, which can keep more
// than N on ties.  Here exactly N are kept and equal float32 scores go to the
// lower channel index, so the result is unique.
#pragma once

#include "common.cuh"

namespace as {

// Eight consecutive channels of one token, converted to float32 (exact).
__device__ __forceinline__ void load8(const __nv_bfloat16 *p, float (&v)[8])
{
    uint4 r = *reinterpret_cast<const uint4 *>(p);
    uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

__device__ __forceinline__ void load8(const float *p, float (&v)[8])
{
    float4 a = *reinterpret_cast<const float4 *>(p);
    float4 b = *reinterpret_cast<const float4 *>(p + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

__device__ __forceinline__ void load8f(const float *p, float (&v)[8]) { load8(p, v); }

// Eight bf16 values held in a 16-byte register vector, converted to float32.
__device__ __forceinline__ void load8(const uint4 *r, float (&v)[8])
{
    const uint32_t w[4] = {r->x, r->y, r->z, r->w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

// Score of eight channels: s = fl32(|xhat| * f), xhat = fl32(x - eta) when
// shift != 0.  Explicit round-to-nearest intrinsics keep the compiler from
// contracting or reassociating (the selection decision depends on the bits).
__device__ __forceinline__ void score8(const float (&x)[8], bool shift, float eta, const float *f, int c0,
                                       float (&xh)[8], float (&s)[8])
{
    float fv[8];
    if (f) load8f(f + c0, fv);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        xh[e] = shift ? __fsub_rn(x[e], eta) : x[e];
        float a = fabsf(xh[e]);
        s[e] = f ? __fmul_rn(a, fv[e]) : a;
    }
}

// Same with the channel factors already in registers (has_f false: f = 1).
__device__ __forceinline__ void score8v(const float (&x)[8], bool shift, float eta, bool has_f, const float (&fv)[8],
                                        float (&xh)[8], float (&s)[8])
{
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        xh[e] = shift ? __fsub_rn(x[e], eta) : x[e];
        float a = fabsf(xh[e]);
        s[e] = has_f ? __fmul_rn(a, fv[e]) : a;
    }
}

// "j ranks ahead of i": higher score, or equal score and lower index.
__device__ __forceinline__ int ahead(float sj, int j, float si, int i) { return (sj > si) | ((sj == si) & (j < i)); }

// Keep bits (bit e = channel 8*lane_group + e) of exactly-N-per-M selection.
// The lane holds channels [8g, 8g+8); blocks of M > 8 span M/8 consecutive
// lanes, whose scores are exchanged with shuffles (all 32 lanes must call).
template <int M>
__device__ __forceinline__ uint32_t nm_keep(const float (&s)[8], int lane, int n)
{
    uint32_t keep = 0;
    if constexpr (M <= 8) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int b0 = (e / M) * M;
            int rank = 0;
#pragma unroll
            for (int j = 0; j < M; ++j) rank += (j + b0 != e) & ahead(s[b0 + j], b0 + j, s[e], e);
            keep |= (uint32_t)(rank < n) << e;
        }
    } else {
        constexpr int G = M / 8;
        float blk[M];
        const int base = lane & ~(G - 1);
#pragma unroll
        for (int q = 0; q < G; ++q)
#pragma unroll
            for (int e = 0; e < 8; ++e) blk[q * 8 + e] = __shfl_sync(0xffffffffu, s[e], base + q);
        const int pe0 = (lane & (G - 1)) * 8;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            int rank = 0;
#pragma unroll
            for (int j = 0; j < M; ++j) rank += (j != pe0 + e) & ahead(blk[j], j, s[e], pe0 + e);
            keep |= (uint32_t)(rank < n) << e;
        }
    }
    return keep;
}

// The same decision through the block's n-th largest score theta: keep
// every score > theta, and of the scores == theta the lowest-indexed ones
// until n are kept.  That is exactly "rank < n" for the order above (higher
// score first, equal scores by lower index).  theta comes from a bitonic
// sort of the M scores (descending) across the M/8 lanes of the block.
// Requires M >= 8; all 32 lanes must call.
template <int M>
__device__ __forceinline__ uint32_t nm_keep_sorted(const float (&s)[8], int lane, int n)
{
    constexpr int G = M / 8;  // lanes per block
    const int q = lane & (G - 1);
    float v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = s[e];
    // element k = 8 q + e; compare-exchange partners k ^ d, descending where
    // (k & size) == 0
#pragma unroll
    for (int size = 2; size <= M; size <<= 1) {
#pragma unroll
        for (int d = size >> 1; d > 0; d >>= 1) {
            if (d >= 8) {
                const int ld = d >> 3;  // partner lane distance
                const bool lower = (q & ld) == 0;
                const bool desc = ((8 * q) & size) == 0;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float p = __shfl_xor_sync(0xffffffffu, v[e], ld);
                    v[e] = (lower == desc) ? fmaxf(v[e], p) : fminf(v[e], p);
                }
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int pe = e ^ d;
                    if (pe > e) {
                        const bool desc = size >= 8 ? (((8 * q) & size) == 0) : ((e & size) == 0);
                        const float hi = fmaxf(v[e], v[pe]), lo = fminf(v[e], v[pe]);
                        v[e] = desc ? hi : lo;
                        v[pe] = desc ? lo : hi;
                    }
                }
            }
        }
    }
    // theta = sorted[n - 1]: slot (n-1) % 8 of lane (n-1) / 8 of the block
    const int slot = (n - 1) & 7;
    float th = v[0];
#pragma unroll
    for (int e = 1; e < 8; ++e) th = slot == e ? v[e] : th;
    th = __shfl_sync(0xffffffffu, th, (lane & ~(G - 1)) + ((n - 1) >> 3));
    uint32_t gt = 0, eq = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        gt |= (uint32_t)(s[e] > th) << e;
        eq |= (uint32_t)(s[e] == th) << e;
    }
    const int neq = __popc(eq);
    int ngt = __popc(gt), inc = neq;
#pragma unroll
    for (int o = 1; o < G; o <<= 1) ngt += __shfl_xor_sync(0xffffffffu, ngt, o);
#pragma unroll
    for (int o = 1; o < G; o <<= 1) {
        const int up = __shfl_up_sync(0xffffffffu, inc, o);
        if (q >= o) inc += up;
    }
    int before = inc - neq;  // equal scores in the lower lanes of the block
    const int room = n - ngt;  // equal scores that still fit
    uint32_t keep = gt;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        if ((eq >> e) & 1u) {
            keep |= (uint32_t)(before < room) << e;
            ++before;
        }
    }
    return keep;
}

// The n = M/2 -th largest score of the M-block (M = 16 or 32; the block's
// M/8 consecutive lanes hold 8 scores each), without a full sort:
//   1. each lane sorts its 8 scores (descending bitonic network);
//   2. M = 32: lanes q, q^1 merge into one sorted 16-list (half-cleaner on
//      A ++ reverse(B), then a bitonic merge in each lane; the even lane
//      holds ranks 0..7, the odd lane 8..15);
//   3. the n largest of two sorted lists A, B (n = M/2 each) are
//      {max(A[i], B[n-1-i])} (half-cleaner of a bitonic sequence), so their
//      minimum is the n-th largest of the block.
// Every lane of the block gets the same value.  All 32 lanes must call.
__device__ __forceinline__ void sort8_desc(float (&v)[8])
{
#pragma unroll
    for (int size = 2; size <= 8; size <<= 1)
#pragma unroll
        for (int d = size >> 1; d > 0; d >>= 1)
#pragma unroll
            for (int e = 0; e < 8; ++e)
                if ((e & d) == 0) {
                    const float hi = fmaxf(v[e], v[e | d]), lo = fminf(v[e], v[e | d]);
                    const bool desc = (e & size) == 0;
                    v[e] = desc ? hi : lo;
                    v[e | d] = desc ? lo : hi;
                }
}

template <int M>
__device__ __forceinline__ float theta_half(const float (&s)[8], int lane)
{
    static_assert(M == 16 || M == 32, "theta_half: M = 16 or 32");
    float v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = s[e];
    sort8_desc(v);
    if constexpr (M == 32) {
        float p[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) p[e] = __shfl_xor_sync(0xffffffffu, v[7 - e], 1);
        const bool upper = (lane & 1) == 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = upper ? fmaxf(v[e], p[e]) : fminf(v[e], p[e]);
#pragma unroll
        for (int d = 4; d > 0; d >>= 1)
#pragma unroll
            for (int e = 0; e < 8; ++e)
                if ((e & d) == 0) {
                    const float hi = fmaxf(v[e], v[e | d]), lo = fminf(v[e], v[e | d]);
                    v[e] = hi;
                    v[e | d] = lo;
                }
    }
    constexpr int partner = M == 32 ? 3 : 1;  // the lane holding the reversed ranks of the other list
    float mn = __int_as_float(0x7f800000);      // +inf
#pragma unroll
    for (int e = 0; e < 8; ++e) mn = fminf(mn, fmaxf(v[e], __shfl_xor_sync(0xffffffffu, v[7 - e], partner)));
    if constexpr (M == 32) mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 1));
    return mn;
}

// Exactly n of every M-block kept (rank < n for "higher score first, equal
// scores by lower index") from the block's n-th largest score theta: every
// score > theta, and of the scores == theta the lowest-indexed ones until n.
template <int M>
__device__ __forceinline__ uint32_t keep_from_theta(const float (&s)[8], int lane, int n, float th)
{
    constexpr int G = M / 8;  // lanes per block
    const int q = lane & (G - 1);
    uint32_t gt = 0, eq = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        gt |= (uint32_t)(s[e] > th) << e;
        eq |= (uint32_t)(s[e] == th) << e;
    }
    const int neq = __popc(eq);
    int ngt = __popc(gt), inc = neq;
#pragma unroll
    for (int o = 1; o < G; o <<= 1) ngt += __shfl_xor_sync(0xffffffffu, ngt, o);
#pragma unroll
    for (int o = 1; o < G; o <<= 1) {
        const int up = __shfl_up_sync(0xffffffffu, inc, o);
        if (q >= o) inc += up;
    }
    int before = inc - neq;  // equal scores in the lower lanes of the block
    const int room = n - ngt;  // equal scores that still fit
    uint32_t keep = gt;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        if ((eq >> e) & 1u) {
            keep |= (uint32_t)(before < room) << e;
            ++before;
        }
    }
    return keep;
}

// n = M/2 selection through theta_half (M = 16, 32).
template <int M>
__device__ __forceinline__ uint32_t nm_keep_half(const float (&s)[8], int lane, int n)
{
    return keep_from_theta<M>(s, lane, n, theta_half<M>(s, lane));
}

// 2:4 blocks inside the lane: one comparison per pair of the block decides
// for both (j ahead of i: s_j > s_i, or s_j == s_i and j < i).  S is float
// (scores) or uint32_t (bf16 magnitude bits, which order like the values).
template <typename S>
__device__ __forceinline__ uint32_t keep_2of4(const S (&s)[8])
{
    uint32_t keep = 0;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const S a = s[4 * h], b = s[4 * h + 1], c = s[4 * h + 2], d = s[4 * h + 3];  // no conversion
        const int ab = b > a, ac = c > a, ad = d > a, bc = c > b, bd = d > b, cd = d > c;
        const int ra = ab + ac + ad;
        const int rb = (1 - ab) + bc + bd;
        const int rc = (1 - ac) + (1 - bc) + cd;
        const int rd = (1 - ad) + (1 - bd) + (1 - cd);
        keep |= ((uint32_t)(ra < 2) | ((uint32_t)(rb < 2) << 1) | ((uint32_t)(rc < 2) << 2) | ((uint32_t)(rd < 2) << 3))
                << (4 * h);
    }
    return keep;
}

// Positions of the two kept channels of a 2:4 block from its 4-bit keep
// mask (exactly two bits set), without bit-scan instructions.
__device__ __forceinline__ void pos_2of4(uint32_t b, int &i0, int &i1)
{
    i0 = (b & 1u) ? 0 : ((b & 2u) ? 1 : 2);
    i1 = (b & 8u) ? 3 : ((b & 4u) ? 2 : 1);
}

// Threshold selection: keep the channels whose score is above tau.
__device__ __forceinline__ uint32_t keep_thresh(const float (&s)[8], float tau)
{
    uint32_t keep = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) keep |= (uint32_t)(s[e] > tau) << e;
    return keep;
}

__device__ __forceinline__ uint32_t nm_keep_dispatch(const float (&s)[8], int lane, int n, int m)
{
    switch (m) {
    case 1: return nm_keep<1>(s, lane, n);
    case 2: return nm_keep<2>(s, lane, n);
    case 4: return n == 2 ? keep_2of4(s) : nm_keep<4>(s, lane, n);
    case 8: return nm_keep_sorted<8>(s, lane, n);
    case 16: return n == 8 ? nm_keep_half<16>(s, lane, n) : nm_keep_sorted<16>(s, lane, n);
    default: return n == 16 ? nm_keep_half<32>(s, lane, n) : nm_keep_sorted<32>(s, lane, n);
    }
}

// Lane `lane` of a warp holds channel `lane` of a 32-channel word whose
// scores are in sc[0..31] (shared memory); keep it if it ranks among the n
// best of its M-block (blocks [jm, jm+m) inside the word).
template <int M>
__device__ __forceinline__ bool nm_rank_keep_m(const float *sc, int lane, int n)
{
    const int b0 = lane & ~(M - 1), i = lane & (M - 1);
    const float si = sc[lane];
    int rank = 0;
#pragma unroll
    for (int j = 0; j < M; ++j) rank += (j != i) & ahead(sc[b0 + j], j, si, i);
    return rank < n;
}

__device__ __forceinline__ bool nm_rank_keep(const float *sc, int lane, int n, int m)
{
    switch (m) {
    case 1: return true;
    case 2: return nm_rank_keep_m<2>(sc, lane, n);
    case 4: return nm_rank_keep_m<4>(sc, lane, n);
    case 8: return nm_rank_keep_m<8>(sc, lane, n);
    case 16: return nm_rank_keep_m<16>(sc, lane, n);
    default: return nm_rank_keep_m<32>(sc, lane, n);
    }
}

}  // namespace as
