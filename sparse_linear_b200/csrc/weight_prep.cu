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

}  // namespace as
