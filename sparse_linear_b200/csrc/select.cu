// Per-token score, selection and compensation statistics (as_select).
//
// One CTA of 256 threads per token row.  Sources (page title, section):
//  - 激活稀疏化技术：提升LLM推理效率的动态剪枝方法 (activation-sparsity overview):
//    2.1 N:M patterns; 2.2.1 magnitude score; 2.2.3 CLACT score; 3.1 D-PTS
//    (eta = token mean, prune x - eta, add eta back); 3.2 VAR (variance ratio
//    with a running average).
//  - 大模型推理优化：WiSparse激活稀疏化技术解析: 2.1 eq. (4) weight-aware score;
//    2.2 per-layer keep fraction (exact top-k per token here).
//  - 利用2:4稀疏性与Squared-ReLU加速Transformer训练与推理: 3.3 compressed
//    layout with the kept values contiguous, plus position metadata.
//
// Row statistics accumulate in float64 (fixed order: per-thread strided sums,
// warp tree, then the eight warps in order), the score is one float32
// subtraction and one float32 multiply, and the decision compares float32
// bit patterns (scores are >= 0) with ties to the lower index.
#include <algorithm>
#include <type_traits>

#include "common.cuh"
#include "kernels.cuh"
#include "select_util.cuh"

namespace as {

// Block-wide sum of two float64 values (deterministic order).
template <int NT>
__device__ __forceinline__ void block_sum2(double &a, double &b, double (*red)[NT / 32])
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    a = warp_sum_f64(a);
    b = warp_sum_f64(b);
    if (lane == 0) { red[0][warp] = a; red[1][warp] = b; }
    __syncthreads();
    double sa = 0.0, sb = 0.0;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) { sa += red[0][w]; sb += red[1][w]; }
    a = sa;
    b = sb;
    __syncthreads();
}

// Exclusive prefix sum over the block in thread order; returns the prefix,
// `total` receives the block total.
template <int NT>
__device__ __forceinline__ int block_excl_scan(int v, int &total, int *wsum)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int u = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += u;
    }
    if (lane == 31) wsum[warp] = inc;
    __syncthreads();
    int base = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) {
        if (w < warp) base += wsum[w];
        tot += wsum[w];
    }
    __syncthreads();
    total = tot;
    return base + inc - v;
}

// 2:4 metadata byte address (see the meta24 layout in actsparse.h).
__device__ __forceinline__ uint8_t *meta_byte(uint32_t *meta, int t, int c0, int kt)
{
    const int p = t & 127, tile = (t >> 7) * kt + (c0 >> 7);
    const int j = (c0 & 127) >> 5, q = c0 & 31;
    const int lane = 16 * (p >> 4) + 8 * (q >> 4) + (p & 7);
    const int byte = 2 * ((p & 15) >> 3) + ((q & 15) >> 3);
    return reinterpret_cast<uint8_t *>(meta) + (size_t)tile * 2048 + lane * 16 + j * 4 + byte;
}

// Writes one 2:4 metadata byte (the checked build verifies that the address
// lies in the ceil(T / 128) x kt tiles of 2048 bytes).
__device__ __forceinline__ void meta_put(uint32_t *meta, int t, int c0, int kt, int T, uint8_t v)
{
    uint8_t *b = meta_byte(meta, t, c0, kt);
    if (as_in(b - reinterpret_cast<uint8_t *>(meta), (long long)((T + 127) / 128) * kt * 2048)) *b = v;
}

// v[base + i] for i in 0..3 without a dynamic register index.
__device__ __forceinline__ float pick4(const float (&v)[8], int base, int i)
{
    float r = v[base];
    r = i == 1 ? v[base + 1] : r;
    r = i == 2 ? v[base + 2] : r;
    r = i == 3 ? v[base + 3] : r;
    return r;
}

template <typename TX>
__device__ __forceinline__ void store8(TX *p, const float (&v)[8]);

template <>
__device__ __forceinline__ void store8<__nv_bfloat16>(__nv_bfloat16 *p, const float (&v)[8])
{
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        w[i] = *reinterpret_cast<uint32_t *>(&h);
    }
    *reinterpret_cast<uint4 *>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}

template <>
__device__ __forceinline__ void store8<float>(float *p, const float (&v)[8])
{
    *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
    *reinterpret_cast<float4 *>(p + 4) = make_float4(v[4], v[5], v[6], v[7]);
}

// Residuals of rounding 8 float32 values to bf16: lo = bf16(v - bf16(v)).
// hi + lo keeps v to about 2^-17 relative, which the float32-output GEMM
// needs when the kept values were shifted (D-PTS / S-PTS) and so are no
// longer bf16 numbers.
__device__ __forceinline__ void store8_lo(__nv_bfloat16 *p, const float (&v)[8])
{
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        const __nv_bfloat162 l = __floats2bfloat162_rn(v[2 * i] - __low2float(h), v[2 * i + 1] - __high2float(h));
        w[i] = *reinterpret_cast<const uint32_t *>(&l);
    }
    *reinterpret_cast<uint4 *>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}

// The same for 4 values (two 2:4 blocks of the compact operand).
__device__ __forceinline__ uint2 lo4(const float (&cv)[4])
{
    const __nv_bfloat162 h0 = __floats2bfloat162_rn(cv[0], cv[1]);
    const __nv_bfloat162 h1 = __floats2bfloat162_rn(cv[2], cv[3]);
    const __nv_bfloat162 l0 = __floats2bfloat162_rn(cv[0] - __low2float(h0), cv[1] - __high2float(h0));
    const __nv_bfloat162 l1 = __floats2bfloat162_rn(cv[2] - __low2float(h1), cv[3] - __high2float(h1));
    return make_uint2(*reinterpret_cast<const uint32_t *>(&l0), *reinterpret_cast<const uint32_t *>(&l1));
}

// NT threads per token row: 256 for prefill batches, 1024 for the few rows
// of a decode call (fewer rounds of loads per row).
template <typename TX, int NT>
__global__ void __launch_bounds__(NT) k_select(SelectArgs a)
{
    // launched programmatically: wait for the previous kernel in the stream
    // (it may have written x), then let a decode kernel chained after this
    // one start its own loads (it relies on this wait having returned)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    extern __shared__ __align__(16) uint32_t keys[];  // [K] score bits (top-k only)
    __shared__ double red[2][NT / 32];
    __shared__ int wsum[NT / 32];
    __shared__ uint32_t hist[256];
    __shared__ uint32_t s_digit, s_remaining;

    const int t = blockIdx.x, tid = threadIdx.x, lane = tid & 31;
    const int K = a.K, ngroups = K >> 3, ntiles = (ngroups + NT - 1) / NT;
    const int kt = (K + 127) >> 7;

    if (t >= a.T) {  // padding rows of the 2:4 metadata tiles
        if (a.meta24)
            for (int g = tid; g < kt * 16; g += NT) meta_put(a.meta24, t, 8 * g, kt, a.T, 0x44);
        return;
    }
    const TX *xr = static_cast<const TX *>(a.x) + (size_t)t * K;

    // ---- row statistics: sum x, sum x^2 (float64)
    constexpr int U = 1;  // tiles whose loads are in flight together (more costs occupancy)
    double sx = 0.0, sxx = 0.0;
    if (a.dpts == AS_PTS_DYNAMIC || a.var) {
        for (int g0 = tid; g0 < ngroups; g0 += U * NT) {
            float v[U][8];
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (g0 + u * NT < ngroups) load8(xr + 8 * (g0 + u * NT), v[u]);
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (g0 + u * NT < ngroups)
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        sx += (double)v[u][e];
                        sxx += (double)v[u][e] * (double)v[u][e];
                    }
        }
        block_sum2<NT>(sx, sxx, red);
    }
    const float eta = a.dpts == AS_PTS_STATIC ? a.eta_static[t] : (a.dpts ? (float)(sx / (double)K) : 0.0f);
    if (a.dpts && a.eta && tid == 0) a.eta[t] = eta;

    // ---- top-k: scores to shared memory, then an MSB-first radix select of
    // the k-th largest key and the number of equal keys to keep.
    uint32_t tau = 0;
    int need = 0;
    const bool topk = a.sel == AS_SEL_TOPK;
    const int kk = a.k_keep;
    if (topk && kk > 0 && kk < K) {
        for (int g = tid; g < ngroups; g += NT) {
            float v[8], xh[8], s[8];
            load8(xr + 8 * g, v);
            score8(v, a.dpts, eta, a.f, 8 * g, xh, s);
#pragma unroll
            for (int e = 0; e < 8; ++e) keys[8 * g + e] = __float_as_uint(s[e]);
        }
        uint32_t prefix = 0, pmask = 0, remaining = (uint32_t)kk;
        for (int shift = 24; shift >= 0; shift -= 8) {
            if (tid < 256) hist[tid] = 0;
            __syncthreads();
            for (int i = tid; i < K; i += NT) {
                uint32_t key = keys[i];
                if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
            }
            __syncthreads();
            if (tid < 32) {
                // lane l owns digits 255-8l .. 248-8l (highest first)
                uint32_t c = 0;
#pragma unroll
                for (int d = 0; d < 8; ++d) c += hist[255 - 8 * lane - d];
                uint32_t inc = c;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    uint32_t u = __shfl_up_sync(0xffffffffu, inc, o);
                    if (lane >= o) inc += u;
                }
                unsigned hit = __ballot_sync(0xffffffffu, inc >= remaining);
                int L = __ffs(hit) - 1;
                if (lane == L) {
                    uint32_t cum = inc - c;
                    for (int d = 0; d < 8; ++d) {
                        uint32_t h = hist[255 - 8 * lane - d];
                        if (cum + h >= remaining) {
                            s_digit = 255 - 8 * lane - d;
                            s_remaining = remaining - cum;
                            break;
                        }
                        cum += h;
                    }
                }
            }
            __syncthreads();
            prefix |= s_digit << shift;
            pmask |= 255u << shift;
            remaining = s_remaining;
            __syncthreads();
        }
        tau = prefix;
        need = (int)remaining;
    }

    // ---- decisions and outputs, 2048 channels (8 per thread) per tile
    const int words = (K + 31) >> 5;
    double skm = 0.0, skmm = 0.0;
    int eq_base = 0;
    // top-k decides from the keys; the activations are reread only when a
    // value output (masked copy, compact operand, VAR sums) needs them
    const bool need_vals = !topk || a.x_masked || a.x_compact || a.var;
    for (int tile0 = 0; tile0 < ntiles; tile0 += U) {
        float vv[U][8], fv[U][8];
        const bool has_f = a.f != nullptr;
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int g = (tile0 + u) * NT + tid;
#pragma unroll
            for (int e = 0; e < 8; ++e) { vv[u][e] = 0.0f; fv[u][e] = 1.0f; }
            if (g < ngroups && need_vals) {
                load8(xr + 8 * g, vv[u]);
                if (has_f) load8f(a.f + 8 * g, fv[u]);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (tile0 + u >= ntiles) break;  // uniform across the block
            const int g = (tile0 + u) * NT + tid, c0 = 8 * g;
            const bool act = g < ngroups;
            float v[8], xh[8], s[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = act ? vv[u][e] : 0.0f;
            score8v(v, a.dpts, eta, act && has_f, fv[u], xh, s);
            uint32_t keep;
            if (a.sel == AS_SEL_NM) {
                keep = nm_keep_dispatch(s, lane, a.n, a.m);
            } else if (a.sel == AS_SEL_THRESH) {
                keep = keep_thresh(s, a.tau);
            } else if (topk) {
                if (kk <= 0) keep = 0;
                else if (kk >= K) keep = 0xFF;
                else {
                    uint32_t gt = 0, eq = 0;
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        uint32_t key = act ? keys[c0 + e] : 0u;
                        gt |= (uint32_t)(act && key > tau) << e;
                        eq |= (uint32_t)(act && key == tau) << e;
                    }
                    int total;
                    int before = eq_base + block_excl_scan<NT>(__popc(eq), total, wsum);
                    eq_base += total;
                    keep = gt;
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        if ((eq >> e) & 1u) {
                            keep |= (uint32_t)(before < need) << e;
                            ++before;
                        }
                }
            } else {
                keep = 0xFF;
            }
            if (act && as_in((long long)t * K + c0 + 7, (long long)a.T * K)) {
                if (a.bitmask) {
                    uint8_t *bm = reinterpret_cast<uint8_t *>(a.bitmask + (size_t)t * words);
                    bm[g] = (uint8_t)keep;
                    if (g == ngroups - 1)
                        for (int b = ngroups; b < words * 4; ++b) bm[b] = 0;
                }
                float km[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) km[e] = ((keep >> e) & 1u) ? xh[e] : 0.0f;
                if (a.var) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        skm += (double)km[e];
                        skmm += (double)km[e] * (double)km[e];
                    }
                }
                if (a.x_masked) store8<TX>(static_cast<TX *>(a.x_masked) + (size_t)t * K + c0, km);
                if (a.x_masked_lo) store8_lo(static_cast<__nv_bfloat16 *>(a.x_masked_lo) + (size_t)t * K + c0, km);
                if (a.x_compact) {
                    // two 4-blocks per thread, two kept values each (exactly 2:4)
                    float cv[4];
                    uint32_t nib[2];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        uint32_t b = (keep >> (4 * h)) & 0xFu;
                        int i0 = __ffs(b) - 1;
                        int i1 = 31 - __clz(b);
                        cv[2 * h] = pick4(xh, 4 * h, i0);
                        cv[2 * h + 1] = pick4(xh, 4 * h, i1);
                        nib[h] = (uint32_t)i0 | ((uint32_t)i1 << 2);
                    }
                    __nv_bfloat162 p0 = __floats2bfloat162_rn(cv[0], cv[1]);
                    __nv_bfloat162 p1 = __floats2bfloat162_rn(cv[2], cv[3]);
                    uint2 pk = make_uint2(*reinterpret_cast<uint32_t *>(&p0), *reinterpret_cast<uint32_t *>(&p1));
                    *reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(a.x_compact) + (size_t)t * (K / 2) + c0 / 2) = pk;
                    if (a.x_compact_lo)
                        *reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(a.x_compact_lo) + (size_t)t * (K / 2) +
                                                   c0 / 2) = lo4(cv);
                    if (a.meta24) meta_put(a.meta24, t, c0, kt, a.T, (uint8_t)(nib[0] | (nib[1] << 4)));
                }
            }  // act
        }  // u
    }
    if (a.meta24 && tid < 16 * kt - ngroups)  // channel padding of the last 128-channel tile
        meta_put(a.meta24, t, 8 * (ngroups + tid), kt, a.T, 0x44);

    // ---- VAR: variances, running average, scale
    if (a.var) {
        block_sum2<NT>(skm, skmm, red);
        if (tid == 0) {
            const double Kd = (double)K;
            double vd = (sxx - sx * sx / Kd) / (Kd - 1.0);
            double vk = (skmm - skm * skm / Kd) / (Kd - 1.0);
            double run = a.first ? vd : (double)a.mom * (double)a.running_var[t] + (1.0 - (double)a.mom) * vd;
            a.running_var[t] = (float)run;
            if (a.var_dense) a.var_dense[t] = (float)vd;
            if (a.var_kept) a.var_kept[t] = (float)vk;
            if (a.nu) a.nu[t] = (float)sqrt(run / (vk + (double)a.eps));
        }
    }
}

// ---------------------------------------------------------------- N:M rows
// Prefill N:M (or keep-all) selection, persistent: a CTA takes rows
// blockIdx.x, blockIdx.x + gridDim.x, ...  Each row arrives in shared
// memory by 1-D bulk copies into a ring of SR_BUFS row buffers (the next
// rows are in flight while one is scored), the channel factors once per
// CTA.  Statistics, score, selection and outputs are those of k_select.
constexpr int SR_THREADS = 256;
constexpr int SR_BUFS = 4;
constexpr uint32_t SR_PIECE = 16384;  // bytes per bulk copy instruction

__device__ __forceinline__ void bulk_load_pieces(void *dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    for (uint32_t o = 0; o < bytes; o += SR_PIECE)
        bulk_load(static_cast<unsigned char *>(dst) + o, static_cast<const unsigned char *>(src) + o,
                  min(SR_PIECE, bytes - o), bar);
}

// M: block size fixed at compile time (0: from the arguments); COMPACT: the
// 2:4 outputs (compact operand + positions; no masked copy, no VAR).  FREG:
// the channel factors stay in registers (a thread scores the same channels
// of every row; at most SR_FREG_TILES tiles), freeing their shared memory for
// more CTAs per SM.
constexpr int SR_FREG_TILES = 4;

template <typename TX, int M, bool COMPACT, bool FREG>
__global__ void __launch_bounds__(SR_THREADS, FREG ? 3 : 1) k_select_rows(SelectArgs a)
{
    extern __shared__ __align__(128) unsigned char sm[];
    __shared__ double red[2][SR_THREADS / 32];
    __shared__ __align__(8) uint64_t bars[SR_BUFS + 1];
    const int K = a.K, T = a.T, tid = threadIdx.x, lane = tid & 31;
    const int ngroups = K >> 3, ntiles = (ngroups + SR_THREADS - 1) / SR_THREADS, kt = (K + 127) >> 7;
    const int Tpad = a.meta24 ? (T + 127) / 128 * 128 : T;
    const bool has_f = a.f != nullptr;
    const uint32_t fbytes = (has_f && !FREG) ? (uint32_t)K * 4u : 0u, rowbytes = (uint32_t)K * (uint32_t)sizeof(TX);
    float fr[FREG ? SR_FREG_TILES : 1][8];
    if constexpr (FREG) {
#pragma unroll
        for (int tile = 0; tile < SR_FREG_TILES; ++tile) {
            const int g = tile * SR_THREADS + tid;
#pragma unroll
            for (int e = 0; e < 8; ++e) fr[tile][e] = 1.0f;
            if (g < ngroups) load8f(a.f + 8 * g, fr[tile]);
        }
    }
    float *sf = reinterpret_cast<float *>(sm);
    TX *rows = reinterpret_cast<TX *>(sm + fbytes);
    const TX *x = static_cast<const TX *>(a.x);
    const int words = (K + 31) >> 5;

    if (tid == 0) {
        for (int b = 0; b <= SR_BUFS; ++b) mbar_init(&bars[b], 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0) {
        if (fbytes) {
            mbar_arrive_expect_tx(&bars[SR_BUFS], fbytes);
            bulk_load_pieces(sf, a.f, fbytes, &bars[SR_BUFS]);
        }
        for (int b = 0; b < SR_BUFS; ++b) {
            const int t = blockIdx.x + b * gridDim.x;
            if (t < T) {
                mbar_arrive_expect_tx(&bars[b], rowbytes);
                bulk_load_pieces(rows + (size_t)b * K, x + (size_t)t * K, rowbytes, &bars[b]);
            }
        }
    }
    if (fbytes && !mbar_wait(&bars[SR_BUFS], 0)) return;

    int it = 0;
    for (int t = blockIdx.x; t < Tpad; t += gridDim.x, ++it) {
        if (t >= T) {  // padding rows of the 2:4 metadata tiles
            for (int g = tid; g < kt * 16; g += SR_THREADS) meta_put(a.meta24, t, 8 * g, kt, a.T, 0x44);
            continue;
        }
        const int buf = it % SR_BUFS;
        if (!mbar_wait(&bars[buf], (uint32_t)(it / SR_BUFS) & 1u)) return;
        const TX *xr = rows + (size_t)buf * K;

        // ---- row statistics: sum x, sum x^2 (float64)
        double sx = 0.0, sxx = 0.0;
        if (a.dpts == AS_PTS_DYNAMIC || a.var) {
            for (int g = tid; g < ngroups; g += SR_THREADS) {
                float v[8];
                load8(xr + 8 * g, v);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    sx += (double)v[e];
                    sxx += (double)v[e] * (double)v[e];
                }
            }
            block_sum2<SR_THREADS>(sx, sxx, red);
        }
        const float eta =
            a.dpts == AS_PTS_STATIC ? a.eta_static[t] : (a.dpts ? (float)(sx / (double)K) : 0.0f);
        if (a.dpts && a.eta && tid == 0) a.eta[t] = eta;

        // ---- decisions and outputs, 8 channels per thread per tile.  The
        // thread's position-metadata byte moves by a fixed stride per tile
        // (its channel offset within a 32-channel block is the same in
        // every tile).
        uint8_t *mrow = nullptr;
        if (a.meta24) mrow = meta_byte(a.meta24, t, 8 * tid, kt);
        constexpr size_t mstride = (size_t)(8 * SR_THREADS / 128) * 2048;  // bytes per tile
        const bool plain = !a.dpts && !has_f;  // score = |x|
        if constexpr (COMPACT) {
            if (plain) {
                // score = |x|: a thread takes 16 channels (two 2:4 byte groups
                // whose metadata bytes are adjacent), compares the bf16
                // magnitude bits as integers and moves the kept values as raw
                // 16-bit halves: one 16-byte compact store per thread
                const int ng16 = K >> 4;
                uint8_t *m16 = meta_byte(a.meta24, t, 16 * tid, kt);
                constexpr size_t mst16 = (size_t)(16 * SR_THREADS / 128) * 2048;
                uint8_t *bmr = a.bitmask ? reinterpret_cast<uint8_t *>(a.bitmask + (size_t)t * words) : nullptr;
                for (int tile = 0; tile * SR_THREADS < ng16; ++tile) {
                    const int g16 = tile * SR_THREADS + tid;
                    if (g16 >= ng16) continue;
                    const int c0 = 16 * g16;
                    if (!as_in((long long)t * K + c0 + 15, (long long)T * K)) continue;
                    const uint4 r0 = *reinterpret_cast<const uint4 *>(xr + c0);
                    const uint4 r1 = *reinterpret_cast<const uint4 *>(xr + c0 + 8);
                    const uint32_t w[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
                    uint32_t out[4], keepbits = 0, metab = 0;
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        uint32_t hw[8], mk[8];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            hw[2 * i] = w[4 * q + i] & 0xFFFFu;
                            hw[2 * i + 1] = w[4 * q + i] >> 16;
                        }
#pragma unroll
                        for (int e = 0; e < 8; ++e) mk[e] = hw[e] & 0x7FFFu;
                        const uint32_t keep = keep_2of4(mk);
                        keepbits |= keep << (8 * q);
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            int i0, i1;
                            pos_2of4((keep >> (4 * h)) & 0xFu, i0, i1);
                            uint32_t v0 = hw[4 * h], v1 = hw[4 * h + 1];
                            v0 = i0 == 1 ? hw[4 * h + 1] : v0;
                            v0 = i0 == 2 ? hw[4 * h + 2] : v0;
                            v1 = i1 == 2 ? hw[4 * h + 2] : v1;
                            v1 = i1 == 3 ? hw[4 * h + 3] : v1;
                            out[2 * q + h] = v0 | (v1 << 16);
                            metab |= ((uint32_t)i0 | ((uint32_t)i1 << 2)) << (8 * q + 4 * h);
                        }
                    }
                    if (bmr) {
                        *reinterpret_cast<uint16_t *>(bmr + 2 * g16) = (uint16_t)keepbits;
                        if (g16 == ng16 - 1)
                            for (int b = 2 * ng16; b < words * 4; ++b) bmr[b] = 0;
                    }
                    *reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(a.x_compact) + (size_t)t * (K / 2) + c0 / 2) =
                        make_uint4(out[0], out[1], out[2], out[3]);
                    if (a.x_compact_lo)  // unshifted bf16 values: nothing is lost in rounding
                        *reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(a.x_compact_lo) + (size_t)t * (K / 2) +
                                                   c0 / 2) = make_uint4(0, 0, 0, 0);
                    if (as_in(m16 + tile * mst16 + 1 - reinterpret_cast<uint8_t *>(a.meta24),
                              (long long)((T + 127) / 128) * kt * 2048))
                        *reinterpret_cast<uint16_t *>(m16 + tile * mst16) = (uint16_t)metab;
                }
            }
        }
        double skm = 0.0, skmm = 0.0;
        // one tile of 8 channels per thread; fv: the tile's channel factors
        auto tile_step = [&](int tile, const float (&fvin)[8]) {
            const int g = tile * SR_THREADS + tid, c0 = 8 * g;
            const bool act = g < ngroups;
            float v[8] = {0, 0, 0, 0, 0, 0, 0, 0}, fv[8] = {1, 1, 1, 1, 1, 1, 1, 1}, xh[8], sc[8];
            if (act) {
                load8(xr + c0, v);
#pragma unroll
                for (int e = 0; e < 8; ++e) fv[e] = fvin[e];
            }
            score8v(v, a.dpts, eta, act && has_f, fv, xh, sc);
            const bool in_rows = act && as_in((long long)t * K + c0 + 7, (long long)T * K);
            uint32_t keep;
            if constexpr (COMPACT) keep = keep_2of4(sc);
            else if constexpr (M == 0)
                keep = a.sel == AS_SEL_NM       ? nm_keep_dispatch(sc, lane, a.n, a.m)
                       : a.sel == AS_SEL_THRESH ? keep_thresh(sc, a.tau)
                                                : 0xFFu;
            else if constexpr (M >= 16) keep = 2 * a.n == M ? nm_keep_half<M>(sc, lane, a.n) : nm_keep_sorted<M>(sc, lane, a.n);
            else if constexpr (M == 8) keep = nm_keep_sorted<M>(sc, lane, a.n);
            else keep = nm_keep<M>(sc, lane, a.n);
            if (act && in_rows) {
                if (a.bitmask) {
                    uint8_t *bm = reinterpret_cast<uint8_t *>(a.bitmask + (size_t)t * words);
                    bm[g] = (uint8_t)keep;
                    if (g == ngroups - 1)
                        for (int b = ngroups; b < words * 4; ++b) bm[b] = 0;
                }
                if constexpr (!COMPACT) {
                    float km[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) km[e] = ((keep >> e) & 1u) ? xh[e] : 0.0f;
                    if (a.var) {
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            skm += (double)km[e];
                            skmm += (double)km[e] * (double)km[e];
                        }
                    }
                    if (a.x_masked) store8<TX>(static_cast<TX *>(a.x_masked) + (size_t)t * K + c0, km);
                    if (a.x_masked_lo)
                        store8_lo(static_cast<__nv_bfloat16 *>(a.x_masked_lo) + (size_t)t * K + c0, km);
                    if (a.bitmask24) {
                        // the 2:4 part of the N:M selection: per 4-block the two channels
                        // ranked first by (kept, higher score, lower index); dropped
                        // channels rank below every kept one (score -1)
                        float s2[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) s2[e] = ((keep >> e) & 1u) ? sc[e] : -1.0f;
                        const uint32_t pos = keep_2of4(s2);
                        float cv[4];
                        uint32_t nib[2];
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            int i0, i1;
                            pos_2of4((pos >> (4 * h)) & 0xFu, i0, i1);
                            cv[2 * h] = pick4(km, 4 * h, i0);
                            cv[2 * h + 1] = pick4(km, 4 * h, i1);
                            nib[h] = (uint32_t)i0 | ((uint32_t)i1 << 2);
                        }
                        const __nv_bfloat162 p0 = __floats2bfloat162_rn(cv[0], cv[1]);
                        const __nv_bfloat162 p1 = __floats2bfloat162_rn(cv[2], cv[3]);
                        *reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(a.x_compact) + (size_t)t * (K / 2) +
                                                   c0 / 2) =
                            make_uint2(*reinterpret_cast<const uint32_t *>(&p0), *reinterpret_cast<const uint32_t *>(&p1));
                        if (a.x_compact_lo)
                            *reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(a.x_compact_lo) + (size_t)t * (K / 2) +
                                                       c0 / 2) = lo4(cv);
                        if (as_in(mrow + tile * mstride - reinterpret_cast<uint8_t *>(a.meta24), (long long)((T + 127) / 128) * kt * 2048))
                        mrow[tile * mstride] = (uint8_t)(nib[0] | (nib[1] << 4));
                        uint8_t *b24 = reinterpret_cast<uint8_t *>(a.bitmask24 + (size_t)t * words);
                        b24[g] = (uint8_t)(pos & keep);
                        if (g == ngroups - 1)
                            for (int b = ngroups; b < words * 4; ++b) b24[b] = 0;
                    }
                }
                if constexpr (COMPACT) {
                    float cv[4];
                    uint32_t nib[2];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        int i0, i1;
                        pos_2of4((keep >> (4 * h)) & 0xFu, i0, i1);
                        cv[2 * h] = pick4(xh, 4 * h, i0);
                        cv[2 * h + 1] = pick4(xh, 4 * h, i1);
                        nib[h] = (uint32_t)i0 | ((uint32_t)i1 << 2);
                    }
                    const __nv_bfloat162 p0 = __floats2bfloat162_rn(cv[0], cv[1]);
                    const __nv_bfloat162 p1 = __floats2bfloat162_rn(cv[2], cv[3]);
                    *reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(a.x_compact) + (size_t)t * (K / 2) + c0 / 2) =
                        make_uint2(*reinterpret_cast<const uint32_t *>(&p0), *reinterpret_cast<const uint32_t *>(&p1));
                    if (a.x_compact_lo)
                        *reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(a.x_compact_lo) + (size_t)t * (K / 2) +
                                                   c0 / 2) = lo4(cv);
                    if (as_in(mrow + tile * mstride - reinterpret_cast<uint8_t *>(a.meta24), (long long)((T + 127) / 128) * kt * 2048))
                        mrow[tile * mstride] = (uint8_t)(nib[0] | (nib[1] << 4));
                }
            }
        };
        if constexpr (FREG) {
#pragma unroll
            for (int tile = 0; tile < SR_FREG_TILES; ++tile)
                if (tile < ntiles) tile_step(tile, fr[tile]);  // compile-time index: fr stays in registers
        } else if (!(COMPACT && plain)) {  // the plain 2:4 case was done by the 16-channel loop above
            for (int tile = 0; tile < ntiles; ++tile) {
                float fv[8] = {1, 1, 1, 1, 1, 1, 1, 1};
                if (has_f && tile * SR_THREADS + tid < ngroups) load8f(sf + 8 * (tile * SR_THREADS + tid), fv);
                tile_step(tile, fv);
            }
        }
        if (a.meta24 && tid < 16 * kt - ngroups)  // channel padding of the last 128-channel tile
            meta_put(a.meta24, t, 8 * (ngroups + tid), kt, a.T, 0x44);

        // ---- VAR: variances, running average, scale
        if (!COMPACT && a.var) {
            block_sum2<SR_THREADS>(skm, skmm, red);
            if (tid == 0) {
                const double Kd = (double)K;
                const double vd = (sxx - sx * sx / Kd) / (Kd - 1.0);
                const double vk = (skmm - skm * skm / Kd) / (Kd - 1.0);
                const double run =
                    a.first ? vd : (double)a.mom * (double)a.running_var[t] + (1.0 - (double)a.mom) * vd;
                a.running_var[t] = (float)run;
                if (a.var_dense) a.var_dense[t] = (float)vd;
                if (a.var_kept) a.var_kept[t] = (float)vk;
                if (a.nu) a.nu[t] = (float)sqrt(run / (vk + (double)a.eps));
            }
        }
        // ---- the buffer is free: the row SR_BUFS iterations ahead goes into it
        __syncthreads();
        if (tid == 0) {
            const int tn = t + SR_BUFS * gridDim.x;
            if (tn < T) {
                mbar_arrive_expect_tx(&bars[buf], rowbytes);
                bulk_load_pieces(rows + (size_t)buf * K, x + (size_t)tn * K, rowbytes, &bars[buf]);
            }
        }
    }
}

// ---------------------------------------------------------------- CLACT
// Column energy c_j = sqrt(sum_t x_tj^2) over the T rows.
// k_colsq_ring: persistent, one CTA per SM; CTA b takes rows b, b + G, ...
// of a window of up to CN_WIN channels.  Whole rows of the window arrive in
// shared memory by 1-D bulk copies (a ring of CN_BUFS rows, 192 KB, the next
// rows in flight while one is summed); thread i keeps the float64 sums of channels
// 8i .. 8i+7, 8i+2048 .. and so on in registers and writes them as the CTA's
// partial [b][K] at the end.  k_colnorm_final sums the G partials of a
// channel in a fixed order (8 threads per channel, then a fixed shuffle
// tree), so c is deterministic.
constexpr int CN_THREADS = 256;
constexpr int CN_WIN = 8 * 4 * CN_THREADS;  // 8192 channels: 4 groups of 8 per thread
constexpr int CN_BUFS_BF16 = 12;  // 192 KB of 16 KB rows in flight per SM
constexpr int CN_BUFS_F32 = 6;    // 192 KB of 32 KB rows

template <typename TX, int CN_BUFS>
__global__ void __launch_bounds__(CN_THREADS) k_colsq_ring(const TX *__restrict__ x, int T, int K,
                                                           double *__restrict__ part)
{
    extern __shared__ __align__(128) unsigned char sm[];
    __shared__ __align__(8) uint64_t bars[CN_BUFS];
    const int tid = threadIdx.x;
    const int c_lo = blockIdx.y * CN_WIN, nwin = min(CN_WIN, K - c_lo);  // nwin % 8 == 0
    const uint32_t rowbytes = (uint32_t)nwin * (uint32_t)sizeof(TX);
    TX *rows = reinterpret_cast<TX *>(sm);
    if (tid == 0) {
        for (int b = 0; b < CN_BUFS; ++b) mbar_init(&bars[b], 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0)
        for (int b = 0; b < CN_BUFS; ++b) {
            const int t = blockIdx.x + b * gridDim.x;
            if (t < T) {
                mbar_arrive_expect_tx(&bars[b], rowbytes);
                bulk_load_pieces(rows + (size_t)b * CN_WIN, x + (size_t)t * K + c_lo, rowbytes, &bars[b]);
            }
        }
    double acc[4][8];
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[q][e] = 0.0;
    int it = 0;
    for (int t = blockIdx.x; t < T; t += gridDim.x, ++it) {
        const int buf = it % CN_BUFS;
        if (!mbar_wait(&bars[buf], (uint32_t)(it / CN_BUFS) & 1u)) break;
        const TX *xr = rows + (size_t)buf * CN_WIN;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int c0 = 8 * (tid + q * CN_THREADS);
            if (c0 < nwin) {
                float v[8];
                load8(xr + c0, v);
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[q][e] += (double)v[e] * (double)v[e];
            }
        }
        __syncthreads();  // every thread is done with the buffer: the row CN_BUFS ahead goes into it
        if (tid == 0) {
            const int tn = t + CN_BUFS * gridDim.x;
            if (tn < T) {
                mbar_arrive_expect_tx(&bars[buf], rowbytes);
                bulk_load_pieces(rows + (size_t)buf * CN_WIN, x + (size_t)tn * K + c_lo, rowbytes, &bars[buf]);
            }
        }
    }
    double *pr = part + (size_t)blockIdx.x * K + c_lo;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int c0 = 8 * (tid + q * CN_THREADS);
        if (c0 < nwin)
#pragma unroll
            for (int e = 0; e < 8; ++e) pr[c0 + e] = acc[q][e];
    }
}

// c[i] = sqrt(sum over the G partials), 8 threads per channel: thread k of
// a channel sums partials k, k + 8, ... in order, then a fixed shuffle tree.
__global__ void k_colnorm_final(const double *__restrict__ part, int G, int K, float *__restrict__ c)
{
    const int gi = blockIdx.x * blockDim.x + threadIdx.x;
    const int i = gi >> 3, k = gi & 7;
    double s = 0.0;
    if (i < K)
        for (int j = k; j < G; j += 8) s += part[(size_t)j * K + i];
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    s += __shfl_xor_sync(0xffffffffu, s, 4);
    if (i < K && k == 0) c[i] = (float)sqrt(s);
}

static int colnorm_ctas(int T)
{
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
    return T < sms ? (T > 0 ? T : 1) : sms;
}

size_t colnorm_workspace(int T, int K)
{
    return (size_t)colnorm_ctas(T) * (size_t)K * sizeof(double) + (size_t)K * sizeof(float);
}

cudaError_t launch_colnorm(const void *x, int bf16, int T, int K, float *c, void *ws, cudaStream_t st)
{
    const int G = colnorm_ctas(T);
    double *part = static_cast<double *>(ws);
    dim3 grid(G, (K + CN_WIN - 1) / CN_WIN);  // K % 8 == 0
    cudaError_t e;
    if (bf16) {
        const size_t smem = (size_t)CN_BUFS_BF16 * CN_WIN * 2;
        static int done[64];
        e = smem_limit_once(k_colsq_ring<__nv_bfloat16, CN_BUFS_BF16>, smem, done);
        if (e == cudaSuccess)
            k_colsq_ring<__nv_bfloat16, CN_BUFS_BF16><<<grid, CN_THREADS, smem, st>>>(
                static_cast<const __nv_bfloat16 *>(x), T, K, part);
    } else {
        const size_t smem = (size_t)CN_BUFS_F32 * CN_WIN * 4;
        static int done[64];
        e = smem_limit_once(k_colsq_ring<float, CN_BUFS_F32>, smem, done);
        if (e == cudaSuccess)
            k_colsq_ring<float, CN_BUFS_F32><<<grid, CN_THREADS, smem, st>>>(static_cast<const float *>(x), T, K, part);
    }
    if (e != cudaSuccess) return e;
    const long long threads = (long long)K * 8;
    k_colnorm_final<<<(unsigned)((threads + 255) / 256), 256, 0, st>>>(part, G, K, c);
    return cudaGetLastError();
}

template <typename TX, int NT>
static cudaError_t launch_select_t(const SelectArgs &a, size_t smem, int grid, cudaStream_t st)
{
    if (smem > 40 * 1024) {  // the 48 KB default also counts the kernel's static shared memory
        static int done[64];
        cudaError_t e = smem_limit_once(k_select<TX, NT>, smem, done);
        if (e != cudaSuccess) return e;
    }
    // programmatic launch: the CTAs become resident while the previous
    // kernel finishes and wait for it before their first load
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(NT);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_select<TX, NT>, a);
}

template <typename TX, int M, bool COMPACT, bool FREG>
static cudaError_t launch_select_rows_f(const SelectArgs &a, cudaStream_t st)
{
    const size_t smem = ((a.f && !FREG) ? (size_t)a.K * 4 : 0) + (size_t)SR_BUFS * a.K * sizeof(TX);
    static int done[64];
    cudaError_t e = smem_limit_once(k_select_rows<TX, M, COMPACT, FREG>, smem, done);
    if (e != cudaSuccess) return e;
    int per_sm = 0, dev = 0, sms = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_select_rows<TX, M, COMPACT, FREG>, SR_THREADS, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int rows = a.meta24 ? (a.T + 127) / 128 * 128 : a.T;
    const int grid = std::min(rows, per_sm * sms);
    k_select_rows<TX, M, COMPACT, FREG><<<grid, SR_THREADS, smem, st>>>(a);
    return cudaGetLastError();
}

// Channel factors in registers when every thread scores at most
// SR_FREG_TILES tiles of 8 channels (K <= 8192).
template <typename TX, int M, bool COMPACT>
static cudaError_t launch_select_rows_t(const SelectArgs &a, cudaStream_t st)
{
    const int ntiles = (a.K / 8 + SR_THREADS - 1) / SR_THREADS;
    if (!COMPACT && a.f && ntiles <= SR_FREG_TILES) return launch_select_rows_f<TX, M, COMPACT, true>(a, st);
    return launch_select_rows_f<TX, M, COMPACT, false>(a, st);
}

template <typename TX>
static cudaError_t launch_select_rows(const SelectArgs &a, cudaStream_t st)
{
    if (a.sel == AS_SEL_NM) {
        if (a.x_compact && !a.bitmask24) {  // a 2:4 selection (bitmask24: the 2:4 part of an N:M one)
            if constexpr (std::is_same<TX, __nv_bfloat16>::value) return launch_select_rows_t<TX, 4, true>(a, st);
        }
        switch (a.m) {
        case 8: return launch_select_rows_t<TX, 8, false>(a, st);
        case 16: return launch_select_rows_t<TX, 16, false>(a, st);
        case 32: return launch_select_rows_t<TX, 32, false>(a, st);
        default: break;
        }
    }
    return launch_select_rows_t<TX, 0, false>(a, st);
}

// Shared memory the row kernel needs (channel factors + row ring); the
// per-token kernel takes over beyond it.
static bool select_rows_fits(const SelectArgs &a)
{
    const size_t elem = a.bf16 ? 2 : 4;
    return (a.f ? (size_t)a.K * 4 : 0) + (size_t)SR_BUFS * a.K * elem <= 200 * 1024;
}

bool select_rows_kernel(const SelectArgs &a) { return a.sel != AS_SEL_TOPK && select_rows_fits(a); }

cudaError_t launch_select(const SelectArgs &a, cudaStream_t st, int wide)
{
    if (!wide && select_rows_kernel(a))
        return a.bf16 ? launch_select_rows<__nv_bfloat16>(a, st) : launch_select_rows<float>(a, st);
    const bool topk = a.sel == AS_SEL_TOPK && a.k_keep > 0 && a.k_keep < a.K;
    const size_t smem = topk ? (size_t)a.K * sizeof(uint32_t) : 0;
    const int grid = a.meta24 ? ((a.T + 127) / 128) * 128 : a.T;
    if (a.bf16)
        return wide ? launch_select_t<__nv_bfloat16, 1024>(a, smem, grid, st)
                    : launch_select_t<__nv_bfloat16, 256>(a, smem, grid, st);
    return wide ? launch_select_t<float, 1024>(a, smem, grid, st) : launch_select_t<float, 256>(a, smem, grid, st);
}

// ---------------------------------------------------------------- decode N:M
// Selection for a decode call (few tokens): grid (token, 2048-channel chunk),
// 256 threads.  Every CTA of a token computes the token mean from the whole
// row with the same code and order (identical float32 bits in all of them);
// all loads of a thread are issued before any is used.  Output: the keep
// words of its chunk and, from chunk 0, eta.
constexpr int SELD_THREADS = 256;
constexpr int SELD_CHUNK = 2048;             // channels per CTA: one 256-channel tile per warp
constexpr int SELD_ROWREG = 8;               // row loads held in registers per thread (K <= 16384)

__global__ void __launch_bounds__(SELD_THREADS) k_select_nm_decode(SelectArgs a)
{
    using TX = __nv_bfloat16;  // 16-byte row loads hold 8 channels
    // launched programmatically: the previous kernel in the stream may have
    // written x.  The decode kernel after this one loads x before its own
    // wait, so this kernel lets it start only once that wait has returned.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    __shared__ double red[SELD_THREADS / 32];
    const int t = blockIdx.x, chunk = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int K = a.K, ng = K >> 3, words = (K + 31) >> 5;
    const TX *xr = static_cast<const TX *>(a.x) + (size_t)t * K;
    const int c0 = chunk * SELD_CHUNK + warp * 256 + 8 * lane;  // this lane's 8 channels
    const bool act = c0 < K;

    // issue: own channels, their factors, and (D-PTS) the whole row
    float v[8] = {0, 0, 0, 0, 0, 0, 0, 0}, f[8];
    if (act) load8(xr + c0, v);
    const bool has_f = a.f != nullptr && act;
    if (has_f) load8f(a.f + c0, f);
    float eta = a.dpts == AS_PTS_STATIC ? a.eta_static[t] : 0.0f;
    if (a.dpts == AS_PTS_STATIC && chunk == 0 && tid == 0 && a.eta) a.eta[t] = eta;
    if (a.dpts == AS_PTS_DYNAMIC) {
        uint4 raw[SELD_ROWREG];
#pragma unroll
        for (int r = 0; r < SELD_ROWREG; ++r) {
            const int g = tid + r * SELD_THREADS;
            if (g < ng) raw[r] = *reinterpret_cast<const uint4 *>(xr + 8 * g);
        }
        double sum = 0.0;
#pragma unroll
        for (int r = 0; r < SELD_ROWREG; ++r) {
            const int g = tid + r * SELD_THREADS;
            if (g < ng) {
                float w[8];
                load8(&raw[r], w);
#pragma unroll
                for (int e = 0; e < 8; ++e) sum += (double)w[e];
            }
        }
        for (int g = tid + SELD_ROWREG * SELD_THREADS; g < ng; g += SELD_THREADS) {  // K > 16384
            float w[8];
            load8(xr + 8 * g, w);
#pragma unroll
            for (int e = 0; e < 8; ++e) sum += (double)w[e];
        }
        sum = warp_sum_f64(sum);
        if (lane == 0) red[warp] = sum;
        __syncthreads();
        double tot = 0.0;
#pragma unroll
        for (int w = 0; w < SELD_THREADS / 32; ++w) tot += red[w];
        eta = (float)(tot / (double)K);
        if (chunk == 0 && tid == 0 && a.eta) a.eta[t] = eta;
    }
    float xh[8], sc[8];
    score8(v, a.dpts, eta, has_f ? f : nullptr, 0, xh, sc);
    uint32_t keep = a.sel == AS_SEL_THRESH ? keep_thresh(sc, a.tau) : nm_keep_dispatch(sc, lane, a.n, a.m);
    if (!act) keep = 0;
    uint32_t word = keep << (8 * (lane & 3));
    word |= __shfl_xor_sync(0xffffffffu, word, 1);
    word |= __shfl_xor_sync(0xffffffffu, word, 2);
    const int wi = c0 >> 5;
    if ((lane & 3) == 0 && act && as_in((long long)t * words + wi, (long long)a.T * words))
        a.bitmask[(size_t)t * words + wi] = word;
}

cudaError_t launch_select_nm_decode(const SelectArgs &a, cudaStream_t st)
{
    dim3 grid(a.T, (a.K + SELD_CHUNK - 1) / SELD_CHUNK);
    if (!a.bf16) return cudaErrorInvalidValue;  // the float32 decode selects inside its kernel
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(SELD_THREADS);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_select_nm_decode, a);
}

// ---------------------------------------------------------------- statistics
// Per-token kept count and natural nonzeros dropped by a selection: one CTA
// per token (grid-strided), 8 channels per thread per step, exact integer
// counts reduced over the block.
template <typename TX>
__global__ void __launch_bounds__(256) k_select_stats(const TX *__restrict__ x, const uint32_t *__restrict__ bitmask,
                                                      int T, int K, int32_t *kept, int32_t *nz_dropped)
{
    __shared__ int red[2][8];
    const int words = (K + 31) >> 5, ng = K >> 3;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int t = blockIdx.x; t < T; t += gridDim.x) {
        const TX *xr = x + (size_t)t * K;
        const uint8_t *bm = reinterpret_cast<const uint8_t *>(bitmask + (size_t)t * words);
        int nk = 0, nd = 0;
        for (int g = threadIdx.x; g < ng; g += blockDim.x) {
            float v[8];
            load8(xr + 8 * g, v);
            uint32_t nz = 0;
#pragma unroll
            for (int e = 0; e < 8; ++e) nz |= (uint32_t)(v[e] != 0.0f) << e;
            const uint32_t keep = as_in((long long)t * words * 4 + g, (long long)T * words * 4) ? bm[g] : 0u;
            nk += __popc(keep);
            nd += __popc(nz & ~keep);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            nk += __shfl_xor_sync(0xffffffffu, nk, o);
            nd += __shfl_xor_sync(0xffffffffu, nd, o);
        }
        if (lane == 0) {
            red[0][warp] = nk;
            red[1][warp] = nd;
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            int a = 0, b = 0;
            for (int w = 0; w < 8; ++w) {
                a += red[0][w];
                b += red[1][w];
            }
            if (kept) kept[t] = a;
            if (nz_dropped) nz_dropped[t] = b;
        }
        __syncthreads();
    }
}

cudaError_t launch_select_stats(const void *x, int bf16, const uint32_t *bitmask, int T, int K, int32_t *kept,
                                int32_t *nz_dropped, cudaStream_t st)
{
    const int grid = T < 4096 ? T : 4096;
    if (bf16)
        k_select_stats<__nv_bfloat16><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16 *>(x), bitmask, T, K,
                                                             kept, nz_dropped);
    else
        k_select_stats<float><<<grid, 256, 0, st>>>(static_cast<const float *>(x), bitmask, T, K, kept, nz_dropped);
    return cudaGetLastError();
}

}  // namespace as
