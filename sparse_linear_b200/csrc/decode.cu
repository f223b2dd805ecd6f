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

    // ---- 1. D-PTS mean of every token (float64, identical in every CTA)
    if (a.dpts) {
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
                        for (int e = 0; e < 8; ++e) a.colnorm_out[c0 + e] = f[e];
                    }
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        xh[e] = a.dpts ? __fsub_rn(v[e], s_eta[t]) : v[e];
                        s[e] = __fmul_rn(fabsf(xh[e]), f[e]);
                    }
                } else {
                    score8(v, a.dpts, s_eta[t], fac, c0, xh, s);
                }
                keep = a.sel == AS_SEL_NM ? nm_keep_dispatch(s, lane, a.n, a.m) : 0xFFu;
                if (!act) keep = 0;
            }
            // assemble 32-bit words: lanes 4j..4j+3 hold the bytes of word j
            uint32_t word = keep << (8 * (lane & 3));
            word |= __shfl_xor_sync(0xffffffffu, word, 1);
            word |= __shfl_xor_sync(0xffffffffu, word, 2);
            const int wl = 8 * wt + (lane >> 2);
            if ((lane & 3) == 0 && wl < nw) {
                s_keep[t][wl] = word;
                if (a.mask_out && slice == 0) a.mask_out[(size_t)t * nwords + w0 + wl] = word;
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
        if (t < T && o < n_out) {
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
        if (t < T && o < n_out) a.partial[((size_t)split * T + t) * n_out + o] = red[i];
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

static int tpad_of(int T) { return T <= 1 ? 1 : T <= 2 ? 2 : T <= 4 ? 4 : T <= 8 ? 8 : 16; }

static int vec_of(int tp, int bf16)
{
    if (bf16) return tp <= 4 ? 8 : (tp <= 8 ? 4 : 2);
    return tp <= 8 ? 4 : 2;
}

template <typename TW, int TP, int VEC>
static size_t smem_of()
{
    return DecCfg<TP, VEC, TW>::smem;
}

DecodePlan decode_plan(int T, int K, int n_out, int bf16)
{
    DecodePlan p{};
    p.tpad = tpad_of(T);
    const int nwords = (K + 31) / 32;
    p.n_slices = (n_out + DEC_NS - 1) / DEC_NS;
    int want = DEC_TARGET_CTAS / p.n_slices;
    if (want < 1) want = 1;
    int wps = (nwords + want - 1) / want;
    if (wps > DEC_MAX_WORDS) wps = DEC_MAX_WORDS;
    if (wps < 1) wps = 1;
    p.words_per_split = wps;
    p.k_splits = (nwords + wps - 1) / wps;
    p.partial_bytes = p.k_splits > 1 ? (size_t)p.k_splits * T * n_out * sizeof(float) : 0;
    p.counter_bytes = (size_t)p.n_slices * sizeof(unsigned);
    const int vec = vec_of(p.tpad, bf16);
    const int tpr = DEC_NS / vec, rg = DEC_THREADS / tpr;
    size_t list = (size_t)DEC_MAX_WORDS * 32 * (sizeof(int) + p.tpad * sizeof(float));
    size_t red = (size_t)rg * p.tpad * DEC_NS * sizeof(float);
    p.smem_bytes = list > red ? list : red;
    return p;
}

template <typename TW, int TP, int VEC>
static cudaError_t launch_t(const DecodeArgs &a, const DecodePlan &p, cudaStream_t st)
{
    const size_t smem = DecCfg<TP, VEC, TW>::smem;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k_decode<TW, TP, VEC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
    }
    dim3 grid(p.n_slices, p.k_splits);
    k_decode<TW, TP, VEC><<<grid, DEC_THREADS, smem, st>>>(a, p.words_per_split);
    return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeArgs &a, const DecodePlan &p, cudaStream_t st)
{
    if (a.bf16) {
        switch (p.tpad) {
        case 1: return launch_t<__nv_bfloat16, 1, 8>(a, p, st);
        case 2: return launch_t<__nv_bfloat16, 2, 8>(a, p, st);
        case 4: return launch_t<__nv_bfloat16, 4, 8>(a, p, st);
        case 8: return launch_t<__nv_bfloat16, 8, 4>(a, p, st);
        default: return launch_t<__nv_bfloat16, 16, 2>(a, p, st);
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
