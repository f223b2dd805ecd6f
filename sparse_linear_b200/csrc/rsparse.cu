// R-Sparse low-rank compensation for decode (activation-sparsity overview
// page, 激活稀疏化技术：提升LLM推理效率的动态剪枝方法, section 3.3): with
// W ~ W_sparse + A_r B_r^T from a truncated SVD (A_r = U_r S_r [n_out, r],
// B_r = V_r [K, r]), the dropped channels contribute through the rank-r
// factors:
//   u[t, j]  = sum over the dropped channels i of token t of xhat[t, i] B[i, j]
//   y[t, o] += sum_j u[t, j] A[o, j]
// xhat = fl32(x - eta) with the call's token shift, else x.
//
// k_rs_u      grid = 128-channel chunks, 8 warps of 16 channels each; a lane
//             owns r/32 rank columns, issues the B loads of all 16 channels
//             at once and keeps T x r/32 partial sums; the 8 warps are
//             summed in shared memory in warp order and written as the
//             chunk's partial [chunk][T][r].
// Both are programmatic dependents: the constant factors (B, A) are read
// before griddepcontrol.wait, everything the decode call wrote after it.
// k_rs_apply  grid = 256-column block x token: the CTA first forms u[t, :]
//             from the chunk partials (each warp takes r/8 adjacent columns;
//             lanes stride over the chunks, then a fixed shuffle tree), then
//             one thread per output column adds u A^T.
// Deterministic (every sum has a fixed order); float32 accumulation.
#include "common.cuh"
#include "kernels.cuh"

namespace as {

constexpr int RS_THREADS = 256;
constexpr int RS_WARPS = RS_THREADS / 32;
constexpr int RS_WCH = 16;                    // channels per warp
constexpr int RS_CHUNK = RS_WARPS * RS_WCH;   // 128 channels per k_rs_u CTA

template <typename TW, int TP, int RL>
__global__ void __launch_bounds__(RS_THREADS) k_rs_u(const TW *__restrict__ x, const uint32_t *__restrict__ mask,
                                                     const float *__restrict__ eta,
                                                     const __nv_bfloat16 *__restrict__ B, int T, int K,
                                                     float *__restrict__ part)
{
    constexpr int R = 32 * RL;                 // rank
    __shared__ float s_x[TP][RS_CHUNK];        // xhat of the dropped channels, 0 for kept ones
    extern __shared__ float s_red[];           // [RS_WARPS][TP][R]
    // k_rs_apply reads only the constant factor A before its own wait
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int c0 = blockIdx.x * RS_CHUNK;
    const int nc = min(RS_CHUNK, K - c0);
    const int words = (K + 31) / 32;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    // B rows of this warp's channels cw .. cw + 15 (lane's rank columns
    // RL*lane .. +RL): constant weights, loaded before the wait
    const int cw = warp * RS_WCH;
    float b[RS_WCH][RL];
#pragma unroll
    for (int k = 0; k < RS_WCH; ++k) {
        const bool in = cw + k < nc;
        const __nv_bfloat16 *row = B + (size_t)(c0 + cw + k) * R + RL * lane;
#pragma unroll
        for (int e = 0; e < RL; ++e) b[k][e] = in ? __bfloat162float(row[e]) : 0.0f;
    }
    // the mask and eta come from the decode call before this kernel
    asm volatile("griddepcontrol.wait;" ::: "memory");
#pragma unroll
    for (int r = 0; r < (TP * RS_CHUNK + RS_THREADS - 1) / RS_THREADS; ++r) {
        const int i = tid + r * RS_THREADS;
        if (i >= TP * RS_CHUNK) break;
        const int t = i / RS_CHUNK, c = i % RS_CHUNK;
        float v = 0.0f;
        if (t < T && c < nc) {
            const int ch = c0 + c;
            if (!((mask[(size_t)t * words + (ch >> 5)] >> (ch & 31)) & 1u)) {
                v = Elem<TW>::to_f32(x[(size_t)t * K + ch]);
                if (eta) v = __fsub_rn(v, eta[t]);
            }
        }
        s_x[t][c] = v;
    }
    __syncthreads();

    float acc[TP][RL];
#pragma unroll
    for (int t = 0; t < TP; ++t)
#pragma unroll
        for (int e = 0; e < RL; ++e) acc[t][e] = 0.0f;
#pragma unroll
    for (int k = 0; k < RS_WCH; ++k)
#pragma unroll
        for (int t = 0; t < TP; ++t) {
            const float xv = s_x[t][cw + k];
#pragma unroll
            for (int e = 0; e < RL; ++e) acc[t][e] = fmaf(xv, b[k][e], acc[t][e]);
        }
#pragma unroll
    for (int t = 0; t < TP; ++t)
#pragma unroll
        for (int e = 0; e < RL; ++e) s_red[((size_t)warp * TP + t) * R + RL * lane + e] = acc[t][e];
    __syncthreads();
    for (int i = tid; i < T * R; i += RS_THREADS) {
        const int t = i / R, j = i % R;
        float s = 0.0f;
#pragma unroll
        for (int w = 0; w < RS_WARPS; ++w) s += s_red[((size_t)w * TP + t) * R + j];
        if (as_in(((long long)blockIdx.x * T + t) * R + j, (long long)gridDim.x * T * R))
            part[((size_t)blockIdx.x * T + t) * R + j] = s;
    }
}

template <int RL>
__global__ void __launch_bounds__(RS_THREADS) k_rs_apply(const float *__restrict__ part, int chunks,
                                                         const __nv_bfloat16 *__restrict__ A, int T, int n_out,
                                                         float *__restrict__ y)
{
    constexpr int R = 32 * RL;
    __shared__ float s_u[R];
    const int t = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int o = blockIdx.x * RS_THREADS + tid;
    // this column's row of the constant factor A, before the wait
    uint4 w[R / 8];
    if (o < n_out) {
        const __nv_bfloat16 *ar = A + (size_t)o * R;
#pragma unroll
        for (int q = 0; q < R / 8; ++q) w[q] = *reinterpret_cast<const uint4 *>(ar + 8 * q);
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");  // the partials and the call's y are complete
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // u[t, j] for the JW columns of this warp: lanes stride over the chunks
    // in a fixed pattern, then a fixed shuffle tree
    constexpr int JW = R / RS_WARPS;
    float s[JW];
#pragma unroll
    for (int q = 0; q < JW; ++q) s[q] = 0.0f;
    for (int c = lane; c < chunks; c += 32) {
        const float *pc = part + ((size_t)c * T + t) * R + warp * JW;
#pragma unroll
        for (int q = 0; q < JW; ++q) s[q] += pc[q];
    }
#pragma unroll
    for (int q = 0; q < JW; ++q) {
#pragma unroll
        for (int o = 16; o; o >>= 1) s[q] += __shfl_xor_sync(0xffffffffu, s[q], o);
    }
    if (lane == 0)
#pragma unroll
        for (int q = 0; q < JW; ++q) s_u[warp * JW + q] = s[q];
    __syncthreads();
    if (o >= n_out) return;
    float acc = 0.0f;
#pragma unroll
    for (int q = 0; q < R / 8; ++q) {
        const uint32_t ws[4] = {w[q].x, w[q].y, w[q].z, w[q].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            acc = fmaf(s_u[8 * q + 2 * e], __uint_as_float(ws[e] << 16), acc);
            acc = fmaf(s_u[8 * q + 2 * e + 1], __uint_as_float(ws[e] & 0xffff0000u), acc);
        }
    }
    if (as_in((long long)t * n_out + o, (long long)T * n_out)) y[(size_t)t * n_out + o] += acc;
}

size_t rsparse_workspace(int T, int K, int r) { return (size_t)((K + RS_CHUNK - 1) / RS_CHUNK) * T * r * 4; }

template <typename TW, int TP, int RL>
static cudaError_t launch_rs_t(const RsparseArgs &a, cudaStream_t st)
{
    const int chunks = (a.K + RS_CHUNK - 1) / RS_CHUNK;
    float *part = static_cast<float *>(a.workspace);
    const size_t red = (size_t)RS_WARPS * TP * 32 * RL * sizeof(float);
    if (red > 48 * 1024) {
        static int done[64];
        const cudaError_t e = smem_limit_once(k_rs_u<TW, TP, RL>, red, done);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cu = {};
    cu.gridDim = dim3(chunks);
    cu.blockDim = dim3(RS_THREADS);
    cu.dynamicSmemBytes = red;
    cu.stream = st;
    cu.attrs = attr;
    cu.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cu, k_rs_u<TW, TP, RL>, static_cast<const TW *>(a.x), a.mask, a.eta,
                                       static_cast<const __nv_bfloat16 *>(a.B), a.T, a.K, part);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t ca = cu;
    ca.gridDim = dim3((a.n_out + RS_THREADS - 1) / RS_THREADS, a.T);
    ca.dynamicSmemBytes = 0;
    return cudaLaunchKernelEx(&ca, k_rs_apply<RL>, (const float *)part, chunks,
                              static_cast<const __nv_bfloat16 *>(a.A), a.T, a.n_out, a.y);
}

template <typename TW, int RL>
static cudaError_t launch_rs_r(const RsparseArgs &a, cudaStream_t st)
{
    if (a.T <= 1) return launch_rs_t<TW, 1, RL>(a, st);
    if (a.T <= 2) return launch_rs_t<TW, 2, RL>(a, st);
    if (a.T <= 4) return launch_rs_t<TW, 4, RL>(a, st);
    if (a.T <= 8) return launch_rs_t<TW, 8, RL>(a, st);
    return launch_rs_t<TW, 16, RL>(a, st);
}

template <typename TW>
static cudaError_t launch_rs_dt(const RsparseArgs &a, cudaStream_t st)
{
    switch (a.r) {
    case 32: return launch_rs_r<TW, 1>(a, st);
    case 64: return launch_rs_r<TW, 2>(a, st);
    default: return launch_rs_r<TW, 4>(a, st);
    }
}

cudaError_t launch_rsparse(const RsparseArgs &a, cudaStream_t st)
{
    return a.bf16 ? launch_rs_dt<__nv_bfloat16>(a, st) : launch_rs_dt<float>(a, st);
}

}  // namespace as
