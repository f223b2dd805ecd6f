// Decode sparse GEMV: 1..16 tokens, y = prune(x) W^T streaming only the kept
// rows of the channel-major weight Wt [K, n_out].
//
// WiSparse page (大模型推理优化：WiSparse激活稀疏化技术解析) section 3.1: the
// sparse operator fuses sparsification with the matrix multiply so no
// intermediate activation is written; activation-sparsity overview page
// (激活稀疏化技术：提升LLM推理效率的动态剪枝方法) section 1.1: dropped
// activations are not transferred, and section 3.1 (D-PTS).
//
// One kernel per call.  CTA (slice, split) owns 256 output columns and a
// range of 32-channel words of K.  It
//   1. computes the D-PTS mean of every token (float64, fixed order, the same
//      code in every CTA so every CTA gets the same float32 bits),
//   2. scores and selects its channels (exactly N per M-block, ties to the
//      lower index) or reads a precomputed bitmask (top-k),
//   3. compacts the union over tokens of the kept channels into a list with
//      the per-token kept values (zero where a token dropped the channel),
//   4. streams those rows of Wt (128-bit loads, the only large traffic),
//      accumulating in float32 registers, and
//   5. reduces row groups in shared memory and split-K partials through the
//      workspace; the last CTA of a column slice sums the partials in split
//      order (deterministic), adds eta * rowsum and writes y.
#include <type_traits>

#include "common.cuh"
#include "kernels.cuh"
#include "select_util.cuh"

namespace as {

constexpr int DEC_THREADS = 512;
constexpr int DEC_NS = 256;         // output columns per CTA
constexpr int DEC_MAX_WORDS = 32;   // 32-channel words per CTA (list <= 1024)
constexpr int DEC_TARGET_CTAS = 296; // two resident CTAs on each of 148 SMs

template <typename TW, int VEC>
struct WVec;
template <>
struct WVec<__nv_bfloat16, 8> {
    using raw = uint4;
    __device__ static void cvt(const raw &r, float (&w)[8])
    {
        uint32_t u[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            w[2 * i] = __uint_as_float(u[i] << 16);
            w[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
        }
    }
};
template <>
struct WVec<__nv_bfloat16, 4> {
    using raw = uint2;
    __device__ static void cvt(const raw &r, float (&w)[4])
    {
        w[0] = __uint_as_float(r.x << 16);
        w[1] = __uint_as_float(r.x & 0xFFFF0000u);
        w[2] = __uint_as_float(r.y << 16);
        w[3] = __uint_as_float(r.y & 0xFFFF0000u);
    }
};
template <>
struct WVec<__nv_bfloat16, 2> {
    using raw = uint32_t;
    __device__ static void cvt(const raw &r, float (&w)[2])
    {
        w[0] = __uint_as_float(r << 16);
        w[1] = __uint_as_float(r & 0xFFFF0000u);
    }
};
template <>
struct WVec<float, 4> {
    using raw = float4;
    __device__ static void cvt(const raw &r, float (&w)[4])
    {
        w[0] = r.x; w[1] = r.y; w[2] = r.z; w[3] = r.w;
    }
};
template <>
struct WVec<float, 2> {
    using raw = float2;
    __device__ static void cvt(const raw &r, float (&w)[2])
    {
        w[0] = r.x; w[1] = r.y;
    }
};

template <typename R>
__device__ __forceinline__ R ld_stream(const R *p)
{
    return __ldcs(p);
}

// Shared-memory layout (dynamic):
//   list_ch[1024] int, list_x[1024][TP] float        (phases 2-4)
//   red[RG][TP][DEC_NS] float                         (phase 5, aliases the list)
template <int TP, int VEC, typename TW>
struct DecCfg {
    static constexpr int TPR = DEC_NS / VEC;             // threads per row group
    static constexpr int RG = DEC_THREADS / TPR;          // row groups
    static constexpr int U = (TP <= 2) ? 8 : (TP <= 4 ? 4 : (TP <= 8 ? 4 : 8));
    static constexpr size_t list_bytes = (size_t)DEC_MAX_WORDS * 32 * (sizeof(int) + TP * sizeof(float));
    static constexpr size_t red_bytes = (size_t)RG * TP * DEC_NS * sizeof(float);
    static constexpr size_t smem = list_bytes > red_bytes ? list_bytes : red_bytes;
};

template <typename TW, int TP, int VEC>
__global__ void __launch_bounds__(DEC_THREADS) k_decode(DecodeArgs a, int words_per_split)
{
    using C = DecCfg<TP, VEC, TW>;
    using V = WVec<TW, VEC>;
    extern __shared__ __align__(16) unsigned char smem[];
    int *list_ch = reinterpret_cast<int *>(smem);
    float *list_x = reinterpret_cast<float *>(smem + DEC_MAX_WORDS * 32 * sizeof(int));
    float *red = reinterpret_cast<float *>(smem);

    __shared__ double s_red[DEC_THREADS / 32][TP];
    __shared__ float s_eta[TP];
    __shared__ uint32_t s_keep[TP][DEC_MAX_WORDS];
    __shared__ int s_wbase[DEC_MAX_WORDS + 1];
    __shared__ int s_last;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int slice = blockIdx.x, split = blockIdx.y;
    const int T = a.T, K = a.K, n_out = a.n_out;
    const int nwords = (K + 31) >> 5;
    const int w0 = split * words_per_split, w1 = min(nwords, w0 + words_per_split);
    const int nw = max(0, w1 - w0);
    const TW *x = static_cast<const TW *>(a.x);

    // ---- 1. D-PTS mean of every token (float64, identical in every CTA);
    // S-PTS takes the caller's table
    if (a.dpts == AS_PTS_STATIC) {
        if (tid < TP) s_eta[tid] = tid < T ? a.eta_static[tid] : 0.0f;
        __syncthreads();
        if (a.eta_out && slice == 0 && split == 0 && tid < T) a.eta_out[tid] = s_eta[tid];
    } else if (a.dpts) {
        double acc[TP];
#pragma unroll
        for (int t = 0; t < TP; ++t) acc[t] = 0.0;
        const int ng = K >> 3;
        for (int g = tid; g < ng; g += DEC_THREADS) {
#pragma unroll
            for (int t = 0; t < TP; ++t) {
                if (t < T) {
                    float v[8];
                    load8(x + (size_t)t * K + 8 * g, v);
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc[t] += (double)v[e];
                }
            }
        }
#pragma unroll
        for (int t = 0; t < TP; ++t) {
            double s = warp_sum_f64(acc[t]);
            if (lane == 0) s_red[warp][t] = s;
        }
        __syncthreads();
        if (tid < TP) {
            double s = 0.0;
            for (int w = 0; w < DEC_THREADS / 32; ++w) s += s_red[w][tid];
            s_eta[tid] = (float)(s / (double)K);
        }
        __syncthreads();
        if (a.eta_out && slice == 0 && split == 0 && tid < T) a.eta_out[tid] = s_eta[tid];
    } else if (tid < TP) {
        s_eta[tid] = 0.0f;
    }

    // ---- 2. selection of channels [32*w0, 32*w1) for every token
    {
        const int nwt = (nw + 7) >> 3;  // 256-channel warp tiles
        for (int item = warp; item < T * nwt; item += DEC_THREADS / 32) {
            const int t = item / nwt, wt = item % nwt;
            const int c0 = 32 * w0 + 256 * wt + 8 * lane;
            const bool act = (c0 < 32 * w1) && (c0 < K);
            uint32_t keep = 0;
            if (a.mask_in) {
                if (act)
                    keep = reinterpret_cast<const uint8_t *>(a.mask_in + (size_t)t * nwords)[c0 >> 3];
            } else {
                float v[8] = {0, 0, 0, 0, 0, 0, 0, 0}, f[8], xh[8], s[8];
                const float *fac = nullptr;
                if (act) {
                    load8(x + (size_t)t * K + c0, v);
                    if (a.score == AS_SCORE_WEIGHT) fac = a.g;
                }
                if (a.score == AS_SCORE_CLACT) {
                    // c_j over the T tokens of the call, float64 then rounded
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        double q = 0.0;
                        if (act)
                            for (int u = 0; u < T; ++u) {
                                double xv = (double)Elem<TW>::to_f32(x[(size_t)u * K + c0 + e]);
                                q += xv * xv;
                            }
                        f[e] = (float)sqrt(q);
                    }
                    if (act && t == 0 && slice == 0 && a.colnorm_out) {
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            if (as_in(c0 + e, K)) a.colnorm_out[c0 + e] = f[e];
                    }
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        xh[e] = a.dpts ? __fsub_rn(v[e], s_eta[t]) : v[e];
                        s[e] = __fmul_rn(fabsf(xh[e]), f[e]);
                    }
                } else {
                    score8(v, a.dpts, s_eta[t], fac, c0, xh, s);
                }
                keep = a.sel == AS_SEL_NM       ? nm_keep_dispatch(s, lane, a.n, a.m)
                       : a.sel == AS_SEL_THRESH ? keep_thresh(s, a.tau)
                                                : 0xFFu;
                if (!act) keep = 0;
            }
            // assemble 32-bit words: lanes 4j..4j+3 hold the bytes of word j
            uint32_t word = keep << (8 * (lane & 3));
            word |= __shfl_xor_sync(0xffffffffu, word, 1);
            word |= __shfl_xor_sync(0xffffffffu, word, 2);
            const int wl = 8 * wt + (lane >> 2);
            if ((lane & 3) == 0 && wl < nw) {
                s_keep[t][wl] = word;
                if (a.mask_out && slice == 0 && as_in((long long)t * nwords + w0 + wl, (long long)T * nwords))
                    a.mask_out[(size_t)t * nwords + w0 + wl] = word;
            }
        }
    }
    __syncthreads();

    // ---- 3. union list (ascending channel order) with per-token values
    if (warp == 0) {
        int cnt = 0;
        if (lane < nw) {
            uint32_t u = 0;
            for (int t = 0; t < T; ++t) u |= s_keep[t][lane];
            cnt = __popc(u);
        }
        int inc = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int v = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += v;
        }
        s_wbase[lane] = inc - cnt;
        if (lane == 31) s_wbase[DEC_MAX_WORDS] = inc;
    }
    __syncthreads();
    const int L = s_wbase[DEC_MAX_WORDS];
    for (int wl = warp; wl < nw; wl += DEC_THREADS / 32) {
        uint32_t u = 0;
        for (int t = 0; t < T; ++t) u |= s_keep[t][wl];
        if ((u >> lane) & 1u) {
            const int pos = s_wbase[wl] + __popc(u & ((1u << lane) - 1u));
            const int c = 32 * (w0 + wl) + lane;
            list_ch[pos] = c;
#pragma unroll
            for (int t = 0; t < TP; ++t) {
                float v = 0.0f;
                if (t < T && ((s_keep[t][wl] >> lane) & 1u)) {
                    float xv = Elem<TW>::to_f32(x[(size_t)t * K + c]);
                    v = a.dpts ? __fsub_rn(xv, s_eta[t]) : xv;
                }
                list_x[pos * TP + t] = v;
            }
        }
    }
    __syncthreads();

    // ---- 4. stream the kept rows of Wt
    const int rg = tid / C::TPR, tc = tid % C::TPR;
    const int col = slice * DEC_NS + tc * VEC;
    const bool col_ok = col < n_out;
    float acc[TP][VEC];
#pragma unroll
    for (int t = 0; t < TP; ++t)
#pragma unroll
        for (int v = 0; v < VEC; ++v) acc[t][v] = 0.0f;
    const TW *wt = static_cast<const TW *>(a.Wt) + col;
    for (int p0 = rg; p0 < L; p0 += C::RG * C::U) {
        typename V::raw r[C::U];
#pragma unroll
        for (int u = 0; u < C::U; ++u) {
            const int p = p0 + u * C::RG;
            if (p < L && col_ok)
                r[u] = ld_stream(reinterpret_cast<const typename V::raw *>(wt + (size_t)list_ch[p] * n_out));
        }
#pragma unroll
        for (int u = 0; u < C::U; ++u) {
            const int p = p0 + u * C::RG;
            if (p < L && col_ok) {
                float w[VEC];
                V::cvt(r[u], w);
#pragma unroll
                for (int t = 0; t < TP; ++t) {
                    const float xv = list_x[p * TP + t];
#pragma unroll
                    for (int v = 0; v < VEC; ++v) acc[t][v] = fmaf(xv, w[v], acc[t][v]);
                }
            }
        }
    }
    __syncthreads();  // list no longer needed; reuse shared memory for the reduction

    // ---- 5. reduce the row groups, then split-K
#pragma unroll
    for (int t = 0; t < TP; ++t)
#pragma unroll
        for (int v = 0; v < VEC; ++v) red[(rg * TP + t) * DEC_NS + tc * VEC + v] = acc[t][v];
    __syncthreads();

    const int k_splits = gridDim.y;
    for (int i = tid; i < TP * DEC_NS; i += DEC_THREADS) {
        const int t = i / DEC_NS, c = i % DEC_NS;
        float s = 0.0f;
        for (int g = 0; g < C::RG; ++g) s += red[(g * TP + t) * DEC_NS + c];
        red[i] = s;  // row group 0's slot for (t, c) is index i; only this thread reads/writes it
    }
    __syncthreads();

    auto emit = [&](int t, int c, float v) {
        const int o = slice * DEC_NS + c;
        if (t < T && o < n_out && as_in((long long)t * n_out + o, (long long)T * n_out)) {
            if (a.dpts) v = fmaf(s_eta[t], a.rowsum[o], v);
            if (a.out_bf16)
                static_cast<__nv_bfloat16 *>(a.y)[(size_t)t * n_out + o] = __float2bfloat16_rn(v);
            else
                static_cast<float *>(a.y)[(size_t)t * n_out + o] = v;
        }
    };

    if (k_splits == 1) {
        for (int i = tid; i < TP * DEC_NS; i += DEC_THREADS) emit(i / DEC_NS, i % DEC_NS, red[i]);
        return;
    }
    for (int i = tid; i < TP * DEC_NS; i += DEC_THREADS) {
        const int t = i / DEC_NS, c = i % DEC_NS, o = slice * DEC_NS + c;
        if (t < T && o < n_out && as_in(((long long)split * T + t) * n_out + o, (long long)k_splits * T * n_out))
            a.partial[((size_t)split * T + t) * n_out + o] = red[i];
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        const unsigned prev = atomicAdd(&a.counters[slice], 1u);
        s_last = (prev == (unsigned)(k_splits - 1));
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    for (int i = tid; i < TP * DEC_NS; i += DEC_THREADS) {
        const int t = i / DEC_NS, c = i % DEC_NS, o = slice * DEC_NS + c;
        if (t < T && o < n_out) {
            float s = 0.0f;
            for (int k = 0; k < k_splits; ++k) s += __ldcg(a.partial + ((size_t)k * T + t) * n_out + o);
            emit(t, c, s);
        }
    }
    if (tid == 0) a.counters[slice] = 0u;  // leave the workspace zeroed for the next call
}

// ============================================================================
// bf16 path: tensor-core decode kernel, D-PTS mean kernel, split-K reduction
// ============================================================================
//
// bf16 decode = up to three kernels chained by programmatic dependent launch:
//   k_select_nm_decode (select.cu, more than 2 tokens): D-PTS mean, score,
//     exact N:M selection -> keep words [T, K/32] and eta;
//   k_decode_tc: CTA (slice, split) owns NS = 512 output columns and a range
//     of up to 1024 channels.  It loads its activation chunk while the
//     selection finishes (at most 2 tokens: it computes the means and the
//     selection itself), turns the chunk in place into the dense kept values
//     xhat = keep ? x - eta : 0 (bf16 hi, plus lo = xhat - hi for float32
//     outputs), lists the union over tokens of the kept channels (ascending)
//     and streams those rows of Wt: each of the 8 warps owns 64 output
//     columns and runs its own cp.async ring over the 128-byte pieces of the
//     kept rows (no block-wide barrier in the loop).  Each staged 16-channel
//     slab goes through ldmatrix.trans into A fragments; the B fragments are
//     gathered from the dense kept values through the list; the tensor cores
//     (mma.sync m16n8k16, bf16 in, float32 accumulate) take hi (and lo).  It
//     writes y directly (one split) or its split-K partial sums;
//   k_decode_reduce: adds the partials in split order, with eta*rowsum.

constexpr int TC_WARPS = 8;
constexpr int TC_THREADS = TC_WARPS * 32;
constexpr int TC_NS = 512;                     // output columns per CTA
constexpr int TC_WCOLS = TC_NS / TC_WARPS;     // 64 columns (128 bytes) per warp
constexpr int TC_WROWP = TC_WCOLS * 2 + 16;    // 144-byte padded row piece (ldmatrix: no bank conflicts)
constexpr int TC_KS = 16;                      // rows per stage = one mma k-step
constexpr int TC_MAXW = 32;                    // 32-channel words per CTA
constexpr int TC_MAXL = TC_MAXW * 32;          // 1024 channels
constexpr int TC_XP = TC_MAXL + 24;            // kept-value row stride (bf16): rows 12 banks apart
constexpr int TC_PAD = TC_MAXL;                // list entry of padding positions: a zero kept value

template <int TP>
struct TcCfg {
    static constexpr int NS = TC_NS;
    static constexpr int MT = TC_WCOLS / 16;            // 16-output m-tiles per warp
    static constexpr int STAGES = TP <= 4 ? 4 : 8;
    static constexpr int NT = (TP + 7) / 8;             // 8-token n-tiles
    static constexpr size_t wstage = (size_t)TC_KS * TC_WROWP;
    static constexpr size_t ring = (size_t)TC_WARPS * STAGES * wstage;
    static constexpr size_t red = (size_t)TP * NS * 4;  // after the main loop; aliases the ring
    static constexpr size_t big = ring > red ? ring : red;
    static constexpr size_t xrow = (size_t)TP * TC_XP * 2;              // one dense kept-value array
    static constexpr size_t list = (size_t)(TC_MAXL + TC_KS) * 4;        // channel offsets
    static constexpr size_t smem(bool lo) { return big + (lo ? 2 : 1) * xrow + list; }
    static constexpr int MINB = TP <= 4 ? 2 : 1;
};

// Sum of the split-K partials p[0], p[stride], ... in split order, with
// every load of a batch of TC_SPLIT_BATCH issued before the first add
// (latency of one L2 round trip per batch instead of one per split).
constexpr int TC_SPLIT_BATCH = 48;

template <typename V>
__device__ __forceinline__ void add_to(V &a, const V &b);
template <>
__device__ __forceinline__ void add_to<float>(float &a, const float &b) { a += b; }
template <>
__device__ __forceinline__ void add_to<float4>(float4 &a, const float4 &b)
{
    a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
}

template <typename V, int B>
__device__ __forceinline__ V sum_splits(const V *p, size_t stride, int k_splits)
{
    V s = __ldcg(p);
    for (int k0 = 1; k0 < k_splits; k0 += B) {
        V v[B];
#pragma unroll
        for (int u = 0; u < B; ++u)
            if (k0 + u < k_splits) v[u] = __ldcg(p + (size_t)(k0 + u) * stride);
#pragma unroll
        for (int u = 0; u < B; ++u)
            if (k0 + u < k_splits) add_to(s, v[u]);
    }
    return s;
}

// y = sum of the split-K partials in split order (+ eta*rowsum).  Partials
// are [split][column][TP]; a thread owns one column and VW consecutive
// tokens (one vector load per split).
template <int TP>
struct RedVec {
    static constexpr int VW = TP >= 4 ? 4 : TP;
    using V = typename std::conditional<VW == 4, float4, typename std::conditional<VW == 2, float2, float>::type>::type;
};
template <>
__device__ __forceinline__ void add_to<float2>(float2 &a, const float2 &b)
{
    a.x += b.x; a.y += b.y;
}
template <typename V>
__device__ __forceinline__ float vget(const V &v, int k);
template <>
__device__ __forceinline__ float vget<float>(const float &v, int) { return v; }
template <>
__device__ __forceinline__ float vget<float2>(const float2 &v, int k) { return k == 0 ? v.x : v.y; }
template <>
__device__ __forceinline__ float vget<float4>(const float4 &v, int k)
{
    return k == 0 ? v.x : (k == 1 ? v.y : (k == 2 ? v.z : v.w));
}

template <int TP>
__global__ void __launch_bounds__(256) k_decode_reduce(const float *__restrict__ partial, int k_splits, int T,
                                                       int n_out, const float *__restrict__ eta,
                                                       const float *__restrict__ rowsum, void *__restrict__ y,
                                                       int out_bf16)
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");  // after the wait: see k_select_nm_decode
    using R = RedVec<TP>;
    using V = typename R::V;
    constexpr int G = TP / R::VW;  // vectors per column
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n_out * G) return;
    const int o = i / G, j = i % G;
    if (R::VW * j >= T) return;
    if (!as_in((long long)(k_splits - 1) * n_out * G + i, (long long)k_splits * n_out * G)) return;
    // one token: scalar partials, so every split's load is in flight at once
    // (T = 1 runs ~37 splits); wider vectors in batches of 24 (registers)
    constexpr int B = R::VW == 1 ? TC_SPLIT_BATCH : 24;
    const V s = sum_splits<V, B>(reinterpret_cast<const V *>(partial) + i, (size_t)n_out * G, k_splits);
    const float rs = eta ? rowsum[o] : 0.0f;
#pragma unroll
    for (int k = 0; k < R::VW; ++k) {
        const int t = R::VW * j + k;
        if (t < T && as_in((long long)t * n_out + o, (long long)T * n_out)) {
            float v = vget(s, k);
            if (eta) v = fmaf(eta[t], rs, v);
            if (out_bf16)
                static_cast<__nv_bfloat16 *>(y)[(size_t)t * n_out + o] = __float2bfloat16_rn(v);
            else
                static_cast<float *>(y)[(size_t)t * n_out + o] = v;
        }
    }
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
// FUSED (at most 2 tokens): the kernel computes the means and the selection
// itself (no select kernel before it).  Otherwise the select kernel precedes
// it.  With several splits k_decode_reduce follows it in both cases.
// LO: the kept values enter the tensor cores as bf16 hi + lo (float32 outputs);
// without it as one bf16 (bf16 outputs, whose own rounding error, up to
// 2^-9 relative, is as large as that of rounding xhat to bf16).
// DENSE (not FUSED): the CTA streams every row of its chunk, in order.  Used
// when the union over tokens of the kept channels is expected to cover
// nearly all of them; the stream then does not depend on the selection, so
// the CTA fills its ring before waiting for the select kernel.
template <int TP, bool FUSED, bool LO, bool DENSE>
__global__ void __launch_bounds__(TC_THREADS, TcCfg<TP>::MINB)
    k_decode_tc(DecodeArgs a, int words_per_split)
{
    using C = TcCfg<TP>;
    extern __shared__ __align__(16) unsigned char smem[];
    unsigned char *ring = smem;
    float *red = reinterpret_cast<float *>(smem);  // [TP][NS] after the main loop
    __nv_bfloat16 *xh = reinterpret_cast<__nv_bfloat16 *>(smem + C::big);   // [TP][TC_XP] dense kept values (hi)
    __nv_bfloat16 *xl = xh + (LO ? TP * TC_XP : 0);                           // [TP][TC_XP] lo parts (LO)
    int *list_cl = reinterpret_cast<int *>(smem + C::big + (LO ? 2 : 1) * C::xrow);  // [L padded]

    __shared__ float s_eta[TP];
    __shared__ uint32_t s_keep[TP][TC_MAXW];
    __shared__ __align__(16) float s_f[FUSED ? TC_MAXL : 4];  // channel factors (16-byte loads)
    __shared__ double s_red[TC_WARPS][TP];

    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int slice = blockIdx.x, split = blockIdx.y;
    const int T = a.T, K = a.K, n_out = a.n_out;
    const int nwords = (K + 31) >> 5;
    const int w0 = split * words_per_split, w1 = min(nwords, w0 + words_per_split);
    const int nw = max(0, w1 - w0);
    const int c_begin = 32 * w0, c_end = min(32 * w1, K);
    const int nch = max(0, c_end - c_begin);  // multiple of 8
    const int ngc = nch >> 3;                 // 8-channel groups of the chunk
    const __nv_bfloat16 *x = static_cast<const __nv_bfloat16 *>(a.x);

    // store 8 kept values (hi, and lo with LO) of token t, channels 8g..8g+7
    auto put8 = [&](int t, int g, const float (&v)[8], uint32_t keep8, float eta) {
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float e0 = 0.0f, e1 = 0.0f;
            if ((keep8 >> (2 * i)) & 1u) e0 = a.dpts ? __fsub_rn(v[2 * i], eta) : v[2 * i];
            if ((keep8 >> (2 * i + 1)) & 1u) e1 = a.dpts ? __fsub_rn(v[2 * i + 1], eta) : v[2 * i + 1];
            const __nv_bfloat162 h = __floats2bfloat162_rn(e0, e1);
            hw[i] = *reinterpret_cast<const uint32_t *>(&h);
            if constexpr (LO) {
                const __nv_bfloat162 l =
                    __floats2bfloat162_rn(e0 - __low2float(h), e1 - __high2float(h));
                lw[i] = *reinterpret_cast<const uint32_t *>(&l);
            }
        }
        *reinterpret_cast<uint4 *>(xh + t * TC_XP + 8 * g) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        if constexpr (LO) *reinterpret_cast<uint4 *>(xl + t * TC_XP + 8 * g) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    };

    // per-warp cp.async ring: stage st = list positions [16 st, 16 st + 16)
    // (DENSE: channel offsets), this warp's 64 columns of each row
    const int col0 = slice * C::NS + warp * TC_WCOLS;
    const __nv_bfloat16 *wt = static_cast<const __nv_bfloat16 *>(a.Wt) + (size_t)c_begin * n_out;
    const uint32_t wring = smem_u32(ring) + (uint32_t)(warp * C::STAGES * C::wstage);
    auto issue = [&](int st) {
        const uint32_t base = wring + (uint32_t)((st % C::STAGES) * C::wstage);
#pragma unroll
        for (int r = 0; r < (TC_KS * TC_WCOLS * 2 / 16) / 32; ++r) {
            const int id = lane + 32 * r;
            const int row = id >> 3, c16 = id & 7;
            const int pos = st * TC_KS + row;
            const int cl = DENSE ? (pos < nch ? pos : TC_PAD) : list_cl[pos];
            const int col = col0 + 8 * c16;
            bool ok = cl != TC_PAD && col < n_out;
            if (ok) ok = as_in((long long)(c_begin + cl) * n_out + col + 7, (long long)K * n_out);
            const void *src = ok ? (const void *)(wt + (size_t)cl * n_out + col) : (const void *)wt;
            cp_async16(base + row * TC_WROWP + c16 * 16, src, ok ? 16u : 0u);  // 0 bytes: zero fill
        }
    };
    auto issue_prologue = [&](int nst) {
#pragma unroll
        for (int st = 0; st < C::STAGES - 1; ++st) {
            if (st < nst) issue(st);
            cp_async_commit();
        }
    };

    if constexpr (FUSED) {
        // launched programmatically: wait for the previous kernel in the
        // stream (which may have written x) before the first load
        asm volatile("griddepcontrol.wait;" ::: "memory");
        // ---- 1. whole rows (D-PTS mean), own chunk and channel factors,
        // every load issued before any is used
        const int ng = K >> 3, gc0 = c_begin >> 3;
        uint4 rowv[TP][8];
        float4 gv = make_float4(0.f, 0.f, 0.f, 0.f);
        const bool want_g = a.score == AS_SCORE_WEIGHT && tid < (nch >> 2);
        if (want_g) gv = *reinterpret_cast<const float4 *>(a.g + c_begin + 4 * tid);
        const bool whole = a.dpts == AS_PTS_DYNAMIC;  // whole rows for the mean, else the chunk alone
#pragma unroll
        for (int t = 0; t < TP; ++t)
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const int g = tid + r * TC_THREADS;
                if (t < T && g < ng && (whole || (g >= gc0 && g < gc0 + ngc)))
                    rowv[t][r] = *reinterpret_cast<const uint4 *>(x + (size_t)t * K + 8 * g);
            }
        if (want_g) *reinterpret_cast<float4 *>(s_f + 4 * tid) = gv;
#pragma unroll
        for (int t = 0; t < TP; ++t) {
            double sum = 0.0;
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const int g = tid + r * TC_THREADS;
                if (t < T && g < ng && (whole || (g >= gc0 && g < gc0 + ngc))) {
                    if (whole) {
                        float w[8];
                        load8(&rowv[t][r], w);
#pragma unroll
                        for (int e = 0; e < 8; ++e) sum += (double)w[e];
                    }
                    if (g >= gc0 && g < gc0 + ngc) *reinterpret_cast<uint4 *>(xh + t * TC_XP + 8 * (g - gc0)) = rowv[t][r];
                } else if (t >= T && g >= gc0 && g < gc0 + ngc) {
                    *reinterpret_cast<uint4 *>(xh + t * TC_XP + 8 * (g - gc0)) = make_uint4(0, 0, 0, 0);
                }
            }
            sum = warp_sum_f64(sum);
            if (lane == 0) s_red[warp][t] = sum;
        }
        __syncthreads();
        // every thread forms the means from the warp sums (same order everywhere)
        float eta_r[TP];
#pragma unroll
        for (int t = 0; t < TP; ++t) {
            double sum = 0.0;
            for (int w = 0; w < TC_WARPS; ++w) sum += s_red[w][t];
            eta_r[t] = (a.dpts && t < T) ? (a.dpts == AS_PTS_STATIC ? a.eta_static[t] : (float)(sum / (double)K))
                                         : 0.0f;
        }
#pragma unroll
        for (int t = 0; t < TP; ++t)
            if (tid == t) {
                s_eta[t] = eta_r[t];
                if (a.dpts && slice == 0 && split == 0 && t < T) {
                    a.eta_in[t] = eta_r[t];  // for the split-K reduction kernel
                    if (a.eta_out) a.eta_out[t] = eta_r[t];
                }
            }
        if (a.score == AS_SCORE_CLACT) {
            for (int i = tid; i < nch; i += TC_THREADS) {
                double q = 0.0;
                for (int t = 0; t < T; ++t) {
                    const double v = (double)__bfloat162float(xh[t * TC_XP + i]);
                    q += v * v;
                }
                s_f[i] = (float)sqrt(q);
                if (slice == 0 && a.colnorm_out && as_in(c_begin + i, K)) a.colnorm_out[c_begin + i] = s_f[i];
            }
            __syncthreads();
        }
        // ---- 2. selection: a warp scores a (token, 32-channel word) item, one
        // channel per lane, ranks each in its M-block; its ballot is the word.
        // The lane then replaces its activation by the kept value.
        float *wsc = reinterpret_cast<float *>(ring) + warp * 32;
        for (int item = warp; item < T * nw; item += TC_WARPS) {
            const int t = item / nw, wl = item % nw;
            const int c = 32 * wl + lane;
            float eta_t = eta_r[0];  // eta_r[t] without a dynamic register index
#pragma unroll
            for (int k = 1; k < TP; ++k)
                if (t == k) eta_t = eta_r[k];
            float xv = 0.0f, sc = 0.0f;
            if (c < nch) {
                xv = __bfloat162float(xh[t * TC_XP + c]);
                const float xs = a.dpts ? __fsub_rn(xv, eta_t) : xv;
                sc = a.score != AS_SCORE_MAG ? __fmul_rn(fabsf(xs), s_f[c]) : fabsf(xs);
            }
            wsc[lane] = sc;
            __syncwarp();
            const bool keep =
                c < nch && (a.sel == AS_SEL_THRESH ? sc > a.tau : nm_rank_keep(wsc, lane, a.n, a.m));
            const uint32_t word = __ballot_sync(0xffffffffu, keep);
            if (c < nch) {
                const float e = keep ? (a.dpts ? __fsub_rn(xv, eta_t) : xv) : 0.0f;
                const __nv_bfloat16 h = __float2bfloat16_rn(e);
                xh[t * TC_XP + c] = h;
                if constexpr (LO) xl[t * TC_XP + c] = __float2bfloat16_rn(e - __bfloat162float(h));
            }
            if (lane == 0) {
                s_keep[t][wl] = word;
                if (a.mask_out && slice == 0 && as_in((long long)t * nwords + w0 + wl, (long long)T * nwords))
                    a.mask_out[(size_t)t * nwords + w0 + wl] = word;
            }
            __syncwarp();
        }
        if constexpr (LO) {  // tokens T..TP-1 of the lo array
            for (int i = tid; i < (TP - T) * ngc; i += TC_THREADS)
                *reinterpret_cast<uint4 *>(xl + (T + i / ngc) * TC_XP + 8 * (i % ngc)) = make_uint4(0, 0, 0, 0);
        }
        if (tid < TP) {
            xh[tid * TC_XP + TC_PAD] = __float2bfloat16_rn(0.0f);
            if constexpr (LO) xl[tid * TC_XP + TC_PAD] = __float2bfloat16_rn(0.0f);
        }
        __syncthreads();
    } else {
        // ---- 1. activation chunk (issued before waiting for the selection
        // kernel, which itself waited for the producer of x), then the keep
        // words and D-PTS means it wrote, then the kept values from registers
        uint4 chv[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            const int i = tid + r * TC_THREADS;
            if (i < TP * ngc) {
                const int t = i / ngc, g = i % ngc;
                chv[r] = (t < T && as_in((long long)t * K + c_begin + 8 * g + 7, (long long)T * K))
                             ? *reinterpret_cast<const uint4 *>(x + (size_t)t * K + c_begin + 8 * g)
                             : make_uint4(0, 0, 0, 0);
            }
        }
        // DENSE: the first stages of the weight stream, also before the wait
        // (this kernel starts only once the select kernel has passed its own
        // wait, so everything before that kernel in the stream is complete)
        if constexpr (DENSE) issue_prologue((nch + TC_KS - 1) / TC_KS);
        asm volatile("griddepcontrol.wait;" ::: "memory");  // selection kernel complete
        if (tid < TP) s_eta[tid] = (a.dpts && tid < T) ? a.eta_in[tid] : 0.0f;
        if (a.eta_out && a.dpts && slice == 0 && split == 0 && tid < T) a.eta_out[tid] = a.eta_in[tid];
        for (int i = tid; i < TP * nw; i += TC_THREADS) {
            const int t = i / nw, wl = i % nw;
            uint32_t word = 0u;
            if (t < T && as_in((long long)t * nwords + w0 + wl, (long long)T * nwords)) {
                word = a.mask_in[(size_t)t * nwords + w0 + wl];
                if (a.mask_out && slice == 0) a.mask_out[(size_t)t * nwords + w0 + wl] = word;
            }
            s_keep[t][wl] = word;
        }
        if (tid < TP) {
            xh[tid * TC_XP + TC_PAD] = __float2bfloat16_rn(0.0f);
            if constexpr (LO) xl[tid * TC_XP + TC_PAD] = __float2bfloat16_rn(0.0f);
        }
        __syncthreads();
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            const int i = tid + r * TC_THREADS;
            if (i < TP * ngc) {
                const int t = i / ngc, g = i % ngc;
                float v[8];
                load8(&chv[r], v);
                put8(t, g, v, (s_keep[t][g >> 2] >> ((g & 3) << 3)) & 0xFFu, s_eta[t]);
            }
        }
    }

    // ---- 3. union list (ascending channel offsets).  Every warp forms the
    // prefix over the words itself (no barrier), then lists its own words.
    // DENSE: every channel, in order (no list; the padding columns of the
    // kept values are zero).
    int L = nch;
    if constexpr (DENSE) {
        const int npad = (nch + TC_KS - 1) / TC_KS * TC_KS - nch;  // multiple of 8
        for (int i = tid; i < TP * (npad >> 3); i += TC_THREADS) {
            const int t = i / (npad >> 3), q = i % (npad >> 3);
            *reinterpret_cast<uint4 *>(xh + t * TC_XP + nch + 8 * q) = make_uint4(0, 0, 0, 0);
            if constexpr (LO) *reinterpret_cast<uint4 *>(xl + t * TC_XP + nch + 8 * q) = make_uint4(0, 0, 0, 0);
        }
    } else {
        uint32_t u = 0;
        if (lane < nw)
            for (int t = 0; t < T; ++t) u |= s_keep[t][lane];
        const int cnt = __popc(u);
        int inc = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += v;
        }
        L = __shfl_sync(0xffffffffu, inc, 31);
        for (int wl = warp; wl < nw; wl += TC_WARPS) {
            const uint32_t uw = __shfl_sync(0xffffffffu, u, wl);
            const int base = __shfl_sync(0xffffffffu, inc - cnt, wl);
            const int li = base + __popc(uw & ((1u << lane) - 1u));
            if (((uw >> lane) & 1u) && as_in(li, TC_MAXL) && as_in(32 * wl + lane, nch)) list_cl[li] = 32 * wl + lane;
        }
    }
    const int Lp = (L + TC_KS - 1) / TC_KS * TC_KS;
    if (!DENSE && tid < Lp - L) list_cl[L + tid] = TC_PAD;  // padding positions of the last k-step
    __syncthreads();

    // ---- 4. per-warp cp.async ring over this warp's 64 columns + tensor cores
    const int nst = Lp / TC_KS;
    float acc[C::MT][C::NT][4];
#pragma unroll
    for (int mt = 0; mt < C::MT; ++mt)
#pragma unroll
        for (int nt = 0; nt < C::NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[mt][nt][i] = 0.0f;
    if constexpr (!DENSE) issue_prologue(nst);
    const int g8 = lane >> 2, q4 = lane & 3;
    const int mi = lane >> 3, mr = lane & 7;  // ldmatrix: matrix index, row within it
    auto pack2 = [](const __nv_bfloat16 *row, int c0, int c1) {
        const uint32_t lo = *reinterpret_cast<const uint16_t *>(row + c0);
        const uint32_t hi = *reinterpret_cast<const uint16_t *>(row + c1);
        return lo | (hi << 16);
    };
    for (int st = 0; st < nst; ++st) {
        cp_async_wait<C::STAGES - 2>();
        __syncwarp();  // every lane's pieces of stage st have landed
        if (st + C::STAGES - 1 < nst) issue(st + C::STAGES - 1);  // into the slot read at st-1
        cp_async_commit();
        const uint32_t base = wring + (uint32_t)((st % C::STAGES) * C::wstage);
        const int pk = st * TC_KS;
        // B fragments: kept values of token nt*8+g8 at list positions
        // pk+2q4, +1 (b0) and pk+2q4+8, +9 (b1), gathered from the dense rows
        // (DENSE: the positions are the channel offsets, pairs adjacent)
        int2 ca = make_int2(pk + 2 * q4, pk + 2 * q4 + 1), cb = make_int2(pk + 2 * q4 + 8, pk + 2 * q4 + 9);
        if constexpr (!DENSE) {
            ca = *reinterpret_cast<const int2 *>(list_cl + pk + 2 * q4);
            cb = *reinterpret_cast<const int2 *>(list_cl + pk + 2 * q4 + 8);
        }
        uint32_t bh[C::NT][2], bl[C::NT][2];
#pragma unroll
        for (int nt = 0; nt < C::NT; ++nt) {
            const int t = nt * 8 + g8;
            bh[nt][0] = bh[nt][1] = bl[nt][0] = bl[nt][1] = 0u;
            if (t < TP) {
                if constexpr (DENSE) {
                    bh[nt][0] = *reinterpret_cast<const uint32_t *>(xh + t * TC_XP + ca.x);
                    bh[nt][1] = *reinterpret_cast<const uint32_t *>(xh + t * TC_XP + cb.x);
                    if constexpr (LO) {
                        bl[nt][0] = *reinterpret_cast<const uint32_t *>(xl + t * TC_XP + ca.x);
                        bl[nt][1] = *reinterpret_cast<const uint32_t *>(xl + t * TC_XP + cb.x);
                    }
                } else {
                    bh[nt][0] = pack2(xh + t * TC_XP, ca.x, ca.y);
                    bh[nt][1] = pack2(xh + t * TC_XP, cb.x, cb.y);
                    if constexpr (LO) {
                        bl[nt][0] = pack2(xl + t * TC_XP, ca.x, ca.y);
                        bl[nt][1] = pack2(xl + t * TC_XP, cb.x, cb.y);
                    }
                }
            }
        }
#pragma unroll
        for (int mt = 0; mt < C::MT; ++mt) {
            const uint32_t addr = base + (uint32_t)(((mi >> 1) * 8 + mr) * TC_WROWP + (mt * 16 + (mi & 1) * 8) * 2);
            uint32_t a0, a1, a2, a3;
            ldsm_x4_trans(addr, a0, a1, a2, a3);
#pragma unroll
            for (int nt = 0; nt < C::NT; ++nt) {
                mma_16816(acc[mt][nt], a0, a1, a2, a3, bh[nt][0], bh[nt][1]);
                if constexpr (LO) mma_16816(acc[mt][nt], a0, a1, a2, a3, bl[nt][0], bl[nt][1]);
            }
        }
    }
    cp_async_wait<0>();

    // ---- 5. split-K partial sums straight from the fragments, layout
    // [split][column][TP]: a lane holds tokens 2q4, 2q4+1 of columns o and o+8
    const int k_splits = gridDim.y;
    if (k_splits > 1) {
        float *pp = a.partial + (size_t)split * n_out * TP;
#pragma unroll
        for (int mt = 0; mt < C::MT; ++mt)
#pragma unroll
            for (int nt = 0; nt < C::NT; ++nt) {
                const int o = col0 + mt * 16 + g8;
                const int t = nt * 8 + 2 * q4;
                // (checked build) the last float this lane stores
                const long long pbase = (long long)split * n_out * TP, pn = (long long)k_splits * n_out * TP;
                const bool t_ok = o < n_out && (TP == 1 ? q4 == 0 : t < TP);
                if (t_ok && !as_in(pbase + (long long)(o + 8 < n_out ? o + 8 : o) * TP + (TP == 1 ? 0 : t + 1), pn))
                    continue;
                if constexpr (TP == 1) {
                    if (q4 == 0) {
                        if (o < n_out) pp[o] = acc[mt][nt][0];
                        if (o + 8 < n_out) pp[o + 8] = acc[mt][nt][2];
                    }
                } else if (t < TP) {
                    if (o < n_out)
                        *reinterpret_cast<float2 *>(pp + (size_t)o * TP + t) = make_float2(acc[mt][nt][0], acc[mt][nt][1]);
                    if (o + 8 < n_out)
                        *reinterpret_cast<float2 *>(pp + (size_t)(o + 8) * TP + t) =
                            make_float2(acc[mt][nt][2], acc[mt][nt][3]);
                }
            }
        return;
    }
    __syncthreads();  // every warp done with its ring: the space becomes the output staging buffer
#pragma unroll
    for (int mt = 0; mt < C::MT; ++mt)
#pragma unroll
        for (int nt = 0; nt < C::NT; ++nt) {
            const int o = warp * TC_WCOLS + mt * 16 + g8;
            const int t = nt * 8 + 2 * q4;
            if (t < TP) {
                red[t * C::NS + o] = acc[mt][nt][0];
                red[t * C::NS + o + 8] = acc[mt][nt][2];
            }
            if (t + 1 < TP) {
                red[(t + 1) * C::NS + o] = acc[mt][nt][1];
                red[(t + 1) * C::NS + o + 8] = acc[mt][nt][3];
            }
        }
    __syncthreads();
    const int ocol0 = slice * C::NS;
    for (int i = tid; i < T * C::NS; i += TC_THREADS) {
        const int t = i / C::NS, c = i % C::NS, o = ocol0 + c;
        if (o >= n_out || !as_in((long long)t * n_out + o, (long long)T * n_out)) continue;
        float v = red[t * C::NS + c];
        if (a.dpts) v = fmaf(s_eta[t], a.rowsum[o], v);
        if (a.out_bf16)
            static_cast<__nv_bfloat16 *>(a.y)[(size_t)t * n_out + o] = __float2bfloat16_rn(v);
        else
            static_cast<float *>(a.y)[(size_t)t * n_out + o] = v;
    }
}

// ============================================================================
// planning and launch
// ============================================================================
static int tpad_of(int T) { return T <= 1 ? 1 : T <= 2 ? 2 : T <= 4 ? 4 : T <= 8 ? 8 : 16; }

static int vec_of(int tp, int bf16)
{
    if (bf16) return tp <= 4 ? 8 : (tp <= 8 ? 4 : 2);
    return tp <= 8 ? 4 : 2;
}

static size_t tc_smem(int tp, bool lo)
{
    switch (tp) {
    case 1: return TcCfg<1>::smem(lo);
    case 2: return TcCfg<2>::smem(lo);
    case 4: return TcCfg<4>::smem(lo);
    case 8: return TcCfg<8>::smem(lo);
    default: return TcCfg<16>::smem(lo);
    }
}

static int tc_ns(int) { return TC_NS; }

DecodePlan decode_plan(int T, int K, int n_out, int bf16)
{
    DecodePlan p{};
    p.tpad = tpad_of(T);
    p.tc = bf16 ? 1 : 0;
    const int nwords = (K + 31) / 32;
    const int ns = p.tc ? tc_ns(p.tpad) : DEC_NS;
    const int maxw = p.tc ? TC_MAXW : DEC_MAX_WORDS;
    const int target = p.tc ? (p.tpad <= 4 ? 296 : 148) : DEC_TARGET_CTAS;
    p.n_slices = (n_out + ns - 1) / ns;
    int want = target / p.n_slices;
    if (want < 1) want = 1;
    int wps = (nwords + want - 1) / want;
    if (wps > maxw) wps = maxw;
    // at least 128 channels a CTA: narrow layers would otherwise split K so
    // finely that summing the partials costs more than streaming the rows
    if (p.tc && wps < 4) wps = 4;
    if (wps < 1) wps = 1;
    p.words_per_split = wps;
    p.k_splits = (nwords + wps - 1) / wps;
    p.partial_bytes = p.k_splits > 1 ? (size_t)p.k_splits * p.tpad * n_out * sizeof(float) : 0;
    p.counter_bytes = (size_t)p.n_slices * sizeof(unsigned);
    p.eta_bytes = (size_t)T * sizeof(float);
    if (p.tc) {
        p.smem_bytes = tc_smem(p.tpad, true);
    } else {
        const int vec = vec_of(p.tpad, bf16);
        const int tpr = DEC_NS / vec, rg = DEC_THREADS / tpr;
        size_t list = (size_t)DEC_MAX_WORDS * 32 * (sizeof(int) + p.tpad * sizeof(float));
        size_t red = (size_t)rg * p.tpad * DEC_NS * sizeof(float);
        p.smem_bytes = list > red ? list : red;
    }
    return p;
}

template <typename TW, int TP, int VEC>
static cudaError_t launch_t(const DecodeArgs &a, const DecodePlan &p, cudaStream_t st)
{
    const size_t smem = DecCfg<TP, VEC, TW>::smem;
    if (smem > 40 * 1024) {  // the 48 KB default also counts the kernel's static shared memory (< 8 KB)
        cudaError_t e = cudaFuncSetAttribute(k_decode<TW, TP, VEC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
    }
    dim3 grid(p.n_slices, p.k_splits);
    k_decode<TW, TP, VEC><<<grid, DEC_THREADS, smem, st>>>(a, p.words_per_split);
    return cudaGetLastError();
}

// whole-row loads for the mean are held in registers: K <= 8 * 256 * 8
bool decode_fused(int tpad, int sel, int K)
{
    return tpad <= 2 && (sel == AS_SEL_NM || sel == AS_SEL_THRESH) && K <= 8 * TC_THREADS * 8;
}

int decode_launch_count(const DecodeArgs &a, const DecodePlan &p)
{
    (void)a;
    if (!p.tc) return 1;
    return 1 + (p.k_splits > 1 ? 1 : 0);  // decode (+ split-K reduction); the select kernel is counted by the caller
}

// Programmatic dependent launch: the kernel may start before the previous
// kernel in the stream finishes and must wait (griddepcontrol.wait) before
// reading what that kernel writes.
static void set_pdl(cudaLaunchConfig_t &cfg, cudaLaunchAttribute *attr)
{
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
}

// The tensor-core decode follows the select kernel (which wrote the keep
// words and means) and, for several splits, is followed by the reduction;
// both links are programmatic.
// Expected share of channels kept by at least one of the T tokens, if each
// token keeps a channel with probability f independently.
static double expected_union(const DecodeArgs &a)
{
    if (a.sel == AS_SEL_THRESH) return 0.0;  // the share kept depends on the data: stream the union
    double f = 1.0;
    if (a.sel == AS_SEL_NM) f = (double)a.n / (double)a.m;
    else if (a.sel == AS_SEL_TOPK) f = a.K > 0 ? (double)a.k_keep / (double)a.K : 0.0;
    double miss = 1.0;
    for (int t = 0; t < a.T; ++t) miss *= 1.0 - f;
    return 1.0 - miss;
}

// DENSE streaming when the union is expected to reach 97 % of the channels.
static bool decode_dense(const DecodeArgs &a, int tpad) { return !decode_fused(tpad, a.sel, a.K) && expected_union(a) >= 0.97; }

template <int TP, bool FUSED, bool LO, bool DENSE>
static cudaError_t launch_tc_one(const DecodeArgs &a, const DecodePlan &p, cudaStream_t st)
{
    const size_t smem = TcCfg<TP>::smem(LO);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.n_slices, p.k_splits);
    cfg.blockDim = dim3(TC_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    set_pdl(cfg, attr);
    static int done[64];
    cudaError_t e = smem_limit_once(k_decode_tc<TP, FUSED, LO, DENSE>, smem, done);
    if (e == cudaSuccess) e = cudaLaunchKernelEx(&cfg, k_decode_tc<TP, FUSED, LO, DENSE>, a, p.words_per_split);
    return e;
}

template <int TP, bool LO>
static cudaError_t launch_tc_k(const DecodeArgs &a, const DecodePlan &p, cudaStream_t st)
{
    if constexpr (TP <= 2) {
        if (decode_fused(TP, a.sel, a.K)) return launch_tc_one<TP, true, LO, false>(a, p, st);
    }
    if (decode_dense(a, TP)) return launch_tc_one<TP, false, LO, true>(a, p, st);
    return launch_tc_one<TP, false, LO, false>(a, p, st);
}

template <int TP>
static cudaError_t launch_tc(const DecodeArgs &a, const DecodePlan &p, cudaStream_t st)
{
    cudaError_t e = a.out_bf16 ? launch_tc_k<TP, false>(a, p, st) : launch_tc_k<TP, true>(a, p, st);
    if (e != cudaSuccess || p.k_splits == 1) return e;
    cudaLaunchConfig_t rc = {};
    const int nthreads = a.n_out * (TP / RedVec<TP>::VW);
    rc.gridDim = dim3((nthreads + 255) / 256);
    rc.blockDim = dim3(256);
    rc.stream = st;
    cudaLaunchAttribute rattr[1];
    set_pdl(rc, rattr);
    return cudaLaunchKernelEx(&rc, k_decode_reduce<TP>, (const float *)a.partial, p.k_splits, a.T, a.n_out,
                              a.dpts ? (const float *)a.eta_in : (const float *)nullptr, a.rowsum, a.y, a.out_bf16);
}

bool decode_needs_select(int T, int K, int n_out, int bf16, int out_bf16, int sel)
{
    (void)n_out;
    (void)out_bf16;
    if (sel == AS_SEL_TOPK) return true;  // top-k needs the whole row's scores
    if (!bf16) return sel == AS_SEL_ALL;
    return !decode_fused(tpad_of(T), sel, K) || sel == AS_SEL_ALL;
}

cudaError_t launch_decode(const DecodeArgs &a, const DecodePlan &p, cudaStream_t st)
{
    if (a.bf16) {
        switch (p.tpad) {
        case 1: return launch_tc<1>(a, p, st);
        case 2: return launch_tc<2>(a, p, st);
        case 4: return launch_tc<4>(a, p, st);
        case 8: return launch_tc<8>(a, p, st);
        default: return launch_tc<16>(a, p, st);
        }
    }
    switch (p.tpad) {
    case 1: return launch_t<float, 1, 4>(a, p, st);
    case 2: return launch_t<float, 2, 4>(a, p, st);
    case 4: return launch_t<float, 4, 4>(a, p, st);
    case 8: return launch_t<float, 8, 4>(a, p, st);
    default: return launch_t<float, 16, 2>(a, p, st);
    }
}

}  // namespace as
