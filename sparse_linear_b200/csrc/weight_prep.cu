// Weight preparation, once per layer.
//
// WiSparse page (大模型推理优化：WiSparse激活稀疏化技术解析) section 2.1, eq. (4):
// the weight-aware score uses g_i = ||W[:,i]||_2^alpha, "precomputed, almost
// no runtime cost".  Activation-sparsity overview page section 3.1 (D-PTS):
// y = (x_sparse + eta) W^T needs rowsum_o = sum_i W[o,i].  The decode path
// streams the channel-major copy Wt = W^T so every kept channel is one
// contiguous row.
//
// Reductions accumulate in float64 in a fixed order (two-phase column sums:
// per row-slab partials, then an ordered sum), so results are deterministic.
#include "common.cuh"
#include "kernels.cuh"

namespace as {

// partial[s][i] = sum over rows [s*rows_per, (s+1)*rows_per) of W[o,i]^2.
template <typename TW>
__global__ void k_colsq_partial(const TW *__restrict__ W, int n_out, int k, int rows_per, double *__restrict__ partial)
{
    int i = blockIdx.x * blockDim.x + threadIdx.x;
    int s = blockIdx.y;
    if (i >= k) return;
    int o0 = s * rows_per, o1 = min(n_out, o0 + rows_per);
    double acc = 0.0;
    for (int o = o0; o < o1; ++o) {
        double w = (double)Elem<TW>::to_f32(W[(size_t)o * k + i]);
        acc += w * w;
    }
    partial[(size_t)s * k + i] = acc;
}

__global__ void k_colsq_final(const double *__restrict__ partial, int slabs, int k, double alpha,
                              float *__restrict__ g)
{
    int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= k) return;
    double s = 0.0;
    for (int j = 0; j < slabs; ++j) s += partial[(size_t)j * k + i];
    g[i] = (float)pow(sqrt(s), alpha);
}

// One warp per output row: rowsum_o = sum_i W[o,i] (float64, fixed order).
template <typename TW>
__global__ void k_rowsum(const TW *__restrict__ W, int n_out, int k, float *__restrict__ rowsum)
{
    int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    int lane = threadIdx.x & 31;
    if (warp >= n_out) return;
    const TW *row = W + (size_t)warp * k;
    double acc = 0.0;
    for (int i = lane; i < k; i += 32) acc += (double)Elem<TW>::to_f32(row[i]);
    acc = warp_sum_f64(acc);
    if (lane == 0) rowsum[warp] = (float)acc;
}

// 32x32 tiled transpose W [n_out, k] -> Wt [k, n_out].
template <typename TW>
__global__ void k_transpose(const TW *__restrict__ W, int n_out, int k, TW *__restrict__ Wt)
{
    __shared__ TW tile[32][33];
    int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
    int tx = threadIdx.x, ty = threadIdx.y;  // 32 x 8
    for (int j = ty; j < 32; j += 8) {
        int r = r0 + j, c = c0 + tx;
        if (r < n_out && c < k) tile[j][tx] = W[(size_t)r * k + c];
    }
    __syncthreads();
    for (int j = ty; j < 32; j += 8) {
        int c = c0 + j, r = r0 + tx;  // output row c (channel), column r (output)
        if (c < k && r < n_out) Wt[(size_t)c * n_out + r] = tile[tx][j];
    }
}

static int colsq_slabs(int n_out) { return (n_out + 255) / 256; }

size_t weight_prep_workspace(int n_out, int k) { return (size_t)colsq_slabs(n_out) * (size_t)k * sizeof(double); }

template <typename TW>
static cudaError_t launch_weight_prep_t(const TW *W, int n_out, int k, float alpha, TW *Wt, float *g, float *rowsum,
                                        void *ws, cudaStream_t st)
{
    if (g) {
        int slabs = colsq_slabs(n_out);
        double *part = static_cast<double *>(ws);
        dim3 grid((k + 255) / 256, slabs);
        k_colsq_partial<TW><<<grid, 256, 0, st>>>(W, n_out, k, 256, part);
        k_colsq_final<<<(k + 255) / 256, 256, 0, st>>>(part, slabs, k, (double)alpha, g);
    }
    if (rowsum) k_rowsum<TW><<<(n_out + 7) / 8, 256, 0, st>>>(W, n_out, k, rowsum);
    if (Wt) {
        dim3 grid((k + 31) / 32, (n_out + 31) / 32);
        k_transpose<TW><<<grid, dim3(32, 8), 0, st>>>(W, n_out, k, Wt);
    }
    return cudaGetLastError();
}

cudaError_t launch_weight_prep(const void *W, int bf16, int n_out, int k, float alpha, void *Wt, float *g,
                               float *rowsum, void *ws, cudaStream_t st)
{
    if (bf16)
        return launch_weight_prep_t<__nv_bfloat16>(static_cast<const __nv_bfloat16 *>(W), n_out, k, alpha,
                                                   static_cast<__nv_bfloat16 *>(Wt), g, rowsum, ws, st);
    return launch_weight_prep_t<float>(static_cast<const float *>(W), n_out, k, alpha, static_cast<float *>(Wt), g,
                                       rowsum, ws, st);
}

// ---------------------------------------------------------------- Amber-Pruner
// Activation-sparsity overview page section 2.2.2 (Amber-Pruner): drop the
// weights outside the [lo, hi] percentiles, standardise the remaining ones
// (z-score), and take each input channel's l2 norm as its importance.
// Percentiles are order statistics of all n_out*K values: the value of
// ascending rank floor(q (N-1)), q = pct/100, found exactly by an MSB-first
// radix select on order-preserving 32-bit keys (-0 and +0 share one key, as
// they compare equal).  The weights are finite.
// Moments are float64 in a fixed order; the variance is the population one.

struct AmberState {
    uint32_t prefix[2], pmask[2], remaining[2];  // radix select of the two ranks
    double count, mean, var;                     // kept weights
};

constexpr int AMB_THREADS = 256;
constexpr int AMB_GRID = 296;

__device__ __forceinline__ uint32_t fkey(float v)
{
    uint32_t b = __float_as_uint(v);
    if (b == 0x80000000u) b = 0u;
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

template <typename TW>
__global__ void __launch_bounds__(AMB_THREADS) k_amber_hist(const TW *__restrict__ W, size_t N, const AmberState *st,
                                                            int shift, uint32_t *__restrict__ hist)
{
    __shared__ uint32_t sh[2][256];
    for (int i = threadIdx.x; i < 512; i += AMB_THREADS) (&sh[0][0])[i] = 0;
    __syncthreads();
    const uint32_t p0 = st->prefix[0], m0 = st->pmask[0], p1 = st->prefix[1], m1 = st->pmask[1];
    for (size_t i = (size_t)blockIdx.x * AMB_THREADS + threadIdx.x; i < N; i += (size_t)gridDim.x * AMB_THREADS) {
        const uint32_t k = fkey(Elem<TW>::to_f32(W[i]));
        const uint32_t d = (k >> shift) & 255u;
        if ((k & m0) == p0) atomicAdd(&sh[0][d], 1u);
        if ((k & m1) == p1) atomicAdd(&sh[1][d], 1u);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < 512; i += AMB_THREADS) {
        const uint32_t v = (&sh[0][0])[i];
        if (v) atomicAdd(&hist[i], v);
    }
}

__global__ void k_amber_init(AmberState *st, uint32_t rank_lo, uint32_t rank_hi, uint32_t *hist)
{
    for (int i = threadIdx.x; i < 512; i += blockDim.x) hist[i] = 0;
    if (threadIdx.x == 0) {
        AmberState s{};
        s.remaining[0] = rank_lo;
        s.remaining[1] = rank_hi;
        *st = s;
    }
}

// One thread: the digit of each rank at this shift, then clears the histogram.
__global__ void k_amber_digit(AmberState *st, int shift, uint32_t *hist)
{
    if (threadIdx.x != 0) return;
    for (int s = 0; s < 2; ++s) {
        uint32_t cum = 0;
        for (int d = 0; d < 256; ++d) {
            const uint32_t h = hist[256 * s + d];
            if (cum + h > st->remaining[s]) {
                st->remaining[s] -= cum;
                st->prefix[s] |= (uint32_t)d << shift;
                st->pmask[s] |= 255u << shift;
                break;
            }
            cum += h;
        }
    }
    for (int i = 0; i < 512; ++i) hist[i] = 0;
}

// Per-block count and sum of the kept weights (float64, fixed order).
template <typename TW>
__global__ void __launch_bounds__(AMB_THREADS) k_amber_sum(const TW *__restrict__ W, size_t N, const AmberState *st,
                                                           double *__restrict__ part)
{
    __shared__ double red[2][AMB_THREADS / 32];
    const uint32_t klo = st->prefix[0], khi = st->prefix[1];
    double c = 0.0, sum = 0.0;
    for (size_t i = (size_t)blockIdx.x * AMB_THREADS + threadIdx.x; i < N; i += (size_t)gridDim.x * AMB_THREADS) {
        const float w = Elem<TW>::to_f32(W[i]);
        const uint32_t k = fkey(w);
        if (k >= klo && k <= khi) {
            c += 1.0;
            sum += (double)w;
        }
    }
    c = warp_sum_f64(c);
    sum = warp_sum_f64(sum);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) { red[0][warp] = c; red[1][warp] = sum; }
    __syncthreads();
    if (threadIdx.x == 0) {
        double a = 0.0, b = 0.0;
        for (int w = 0; w < AMB_THREADS / 32; ++w) { a += red[0][w]; b += red[1][w]; }
        part[2 * blockIdx.x] = a;
        part[2 * blockIdx.x + 1] = b;
    }
}

__device__ __forceinline__ float fkey_value(uint32_t key)
{
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

// Count and mean of the kept weights; the two clip values to `bounds`.
__global__ void k_amber_mean(const double *__restrict__ part, int blocks, AmberState *st, float *bounds)
{
    if (threadIdx.x != 0) return;
    double c = 0.0, sum = 0.0;
    for (int b = 0; b < blocks; ++b) { c += part[2 * b]; sum += part[2 * b + 1]; }
    st->count = c;
    st->mean = c > 0.0 ? sum / c : 0.0;
    if (bounds) {
        bounds[0] = fkey_value(st->prefix[0]);
        bounds[1] = fkey_value(st->prefix[1]);
    }
}

// partial[s][i] = sum over the kept weights of rows [s*rows_per, ...) of
// column i of (w - mean)^2.
template <typename TW>
__global__ void k_amber_colsq(const TW *__restrict__ W, int n_out, int k, int rows_per, const AmberState *st,
                              double *__restrict__ partial)
{
    const int i = blockIdx.x * blockDim.x + threadIdx.x, s = blockIdx.y;
    if (i >= k) return;
    const uint32_t klo = st->prefix[0], khi = st->prefix[1];
    const double mu = st->mean;
    const int o0 = s * rows_per, o1 = min(n_out, o0 + rows_per);
    double acc = 0.0;
    for (int o = o0; o < o1; ++o) {
        const float w = Elem<TW>::to_f32(W[(size_t)o * k + i]);
        const uint32_t key = fkey(w);
        if (key >= klo && key <= khi) {
            const double d = (double)w - mu;
            acc += d * d;
        }
    }
    partial[(size_t)s * k + i] = acc;
}

// Column sums S_i (in place in slab 0), then the population variance.
__global__ void k_amber_colsum(double *__restrict__ partial, int slabs, int k)
{
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= k) return;
    double s = 0.0;
    for (int j = 0; j < slabs; ++j) s += partial[(size_t)j * k + i];
    partial[i] = s;
}

__global__ void k_amber_var(const double *__restrict__ colsum, int k, AmberState *st)
{
    if (threadIdx.x != 0) return;
    double s = 0.0;
    for (int i = 0; i < k; ++i) s += colsum[i];
    st->var = st->count > 0.0 ? s / st->count : 0.0;
}

__global__ void k_amber_final(const double *__restrict__ colsum, int k, double alpha, const AmberState *st,
                              float *__restrict__ g)
{
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= k) return;
    const double v = st->var;
    const double z2 = v > 0.0 ? colsum[i] / v : 0.0;  // sum over o of z_oi^2
    g[i] = (float)pow(sqrt(z2), alpha);
}

size_t amber_workspace(int n_out, int k)
{
    return 4096 /* state + histogram */ + (size_t)AMB_GRID * 2 * sizeof(double) +
           (size_t)colsq_slabs(n_out) * (size_t)k * sizeof(double);
}

template <typename TW>
static cudaError_t launch_amber_t(const TW *W, int n_out, int k, float alpha, uint32_t rank_lo, uint32_t rank_hi,
                                  float *g, float *bounds, void *ws, cudaStream_t st)
{
    unsigned char *base = static_cast<unsigned char *>(ws);
    AmberState *state = reinterpret_cast<AmberState *>(base);
    uint32_t *hist = reinterpret_cast<uint32_t *>(base + 2048);
    double *sums = reinterpret_cast<double *>(base + 4096);
    double *cols = sums + (size_t)AMB_GRID * 2;
    const size_t N = (size_t)n_out * k;
    k_amber_init<<<1, 256, 0, st>>>(state, rank_lo, rank_hi, hist);
    for (int shift = 24; shift >= 0; shift -= 8) {
        k_amber_hist<TW><<<AMB_GRID, AMB_THREADS, 0, st>>>(W, N, state, shift, hist);
        k_amber_digit<<<1, 32, 0, st>>>(state, shift, hist);
    }
    k_amber_sum<TW><<<AMB_GRID, AMB_THREADS, 0, st>>>(W, N, state, sums);
    k_amber_mean<<<1, 32, 0, st>>>(sums, AMB_GRID, state, bounds);
    const int slabs = colsq_slabs(n_out);
    dim3 grid((k + 255) / 256, slabs);
    k_amber_colsq<TW><<<grid, 256, 0, st>>>(W, n_out, k, 256, state, cols);
    k_amber_colsum<<<(k + 255) / 256, 256, 0, st>>>(cols, slabs, k);
    k_amber_var<<<1, 32, 0, st>>>(cols, k, state);
    k_amber_final<<<(k + 255) / 256, 256, 0, st>>>(cols, k, (double)alpha, state, g);
    return cudaGetLastError();
}

cudaError_t launch_amber(const void *W, int bf16, int n_out, int k, float alpha, uint32_t rank_lo, uint32_t rank_hi,
                         float *g, float *bounds, void *ws, cudaStream_t st)
{
    if (bf16)
        return launch_amber_t<__nv_bfloat16>(static_cast<const __nv_bfloat16 *>(W), n_out, k, alpha, rank_lo,
                                             rank_hi, g, bounds, ws, st);
    return launch_amber_t<float>(static_cast<const float *>(W), n_out, k, alpha, rank_lo, rank_hi, g, bounds, ws, st);
}

}  // namespace as
