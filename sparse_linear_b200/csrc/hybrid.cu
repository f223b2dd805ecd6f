// Hybrid 2:4 prefill (2:4 + Squared-ReLU page, 利用2:4稀疏性与Squared-ReLU
// 加速Transformer训练与推理, sections 3.2 and 3.3): the densest features are
// computed densely and the rest with 2:4, and the layer's measured sparsity
// picks the mode.  Features are taken in 4-channel blocks so the 2:4 part
// stays block-aligned; the dense set D is the n_dense blocks with the most
// nonzeros over the batch (ties to the lower block index).
//
// The split needs no second selection: the 2:4 GEMM already multiplies the
// kept values of every block, so the dense GEMM takes only what 2:4 dropped
// in the dense blocks, x * (1 - m) on D, and its float32 result is added in
// the 2:4 GEMM's epilogue:
//   y = (x (.) m) W^T + (x (.) (1 - m))[:, D] W[:, D]^T
//
// k_block_nnz     nonzeros per 4-channel block over the tokens (integer
//                 atomics: exact in any order) and the total
// k_pick_dense    one CTA: radix select of the n_dense-th largest count,
//                 ties by a prefix count in index order, the taken blocks
//                 compacted in ascending order; also the sparsity
//                 1 - total / (T K)
// k_gather_dense  the dropped values of the dense blocks [T, 4 n_dense] and
//                 the matching weight columns [n_out, 4 n_dense]
#include "common.cuh"
#include "kernels.cuh"

namespace as {

constexpr int HY_THREADS = 256;
constexpr int HY_TOK = 64;          // tokens per k_block_nnz CTA
constexpr int HY_PICK_THREADS = 1024;

__global__ void __launch_bounds__(HY_THREADS) k_block_nnz(const __nv_bfloat16 *__restrict__ x, int T, int K,
                                                          unsigned *__restrict__ nnz,
                                                          unsigned long long *__restrict__ total)
{
    __shared__ unsigned s_tot[HY_THREADS / 32];
    const int c = blockIdx.x * HY_THREADS + threadIdx.x;  // 8-channel chunk
    const int t0 = blockIdx.y * HY_TOK;
    unsigned n0 = 0, n1 = 0;
    if (c < K / 8) {
        const int t1 = min(T, t0 + HY_TOK);
        for (int tb = t0; tb < t1; tb += 8) {
            uint4 u[8];
#pragma unroll
            for (int r = 0; r < 8; ++r)  // eight rows in flight
                u[r] = tb + r < t1 ? *reinterpret_cast<const uint4 *>(x + (size_t)(tb + r) * K + 8 * c)
                                   : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const uint32_t w[4] = {u[r].x, u[r].y, u[r].z, u[r].w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const unsigned nz = ((w[i] & 0x7fffu) != 0) + ((w[i] & 0x7fff0000u) != 0);
                    if (i < 2) n0 += nz; else n1 += nz;
                }
            }
        }
        if (n0) atomicAdd(&nnz[2 * c], n0);
        if (n1) atomicAdd(&nnz[2 * c + 1], n1);
    }
    unsigned s = n0 + n1;
#pragma unroll
    for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if ((threadIdx.x & 31) == 0) s_tot[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned long long b = 0;
        for (int w = 0; w < HY_THREADS / 32; ++w) b += s_tot[w];
        if (b) atomicAdd(total, b);
    }
}

// Exclusive prefix over the blocks of per-thread counts (each thread owns a
// contiguous run of blocks); returns this thread's start and writes the
// grand total to *sum (all threads call it).
__device__ __forceinline__ int run_scan(int cnt, int *s_warp, int *sum)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    int base = 0, tot = 0;
    for (int w = 0; w < HY_PICK_THREADS / 32; ++w) {
        if (w < warp) base += s_warp[w];
        tot += s_warp[w];
    }
    __syncthreads();
    *sum = tot;
    return base + incl - cnt;
}

// One CTA.  theta = the n_dense-th largest count, by an MSB-first radix
// select over three 8-bit digits (counts < 2^24); taken = count > theta, or
// count == theta among the lowest-indexed (by a prefix count of the equal
// ones) until n_dense; then the taken blocks in ascending order.  A thread
// holds its (at most HY_PICK_PER) consecutive counts in registers; warp 0
// finds each digit with a shuffle scan over the 256 bins.
constexpr int HY_PICK_PER = 8;  // K <= 32768: at most 8192 blocks over 1024 threads

__global__ void __launch_bounds__(HY_PICK_THREADS) k_pick_dense(const unsigned *__restrict__ nnz, int nb, int n_dense,
                                                                const unsigned long long *__restrict__ total,
                                                                double elems, int *__restrict__ idx,
                                                                float *__restrict__ sparsity)
{
    __shared__ unsigned s_hist[256];
    __shared__ unsigned s_prefix, s_rem;
    __shared__ int s_warp[HY_PICK_THREADS / 32];
    const int tid = threadIdx.x, lane = tid & 31;
    if (tid == 0) *sparsity = (float)(1.0 - (double)*total / elems);
    if (n_dense <= 0) return;
    const int per = (nb + HY_PICK_THREADS - 1) / HY_PICK_THREADS;
    const int b0 = min(nb, tid * per), b1 = min(nb, b0 + per);
    unsigned v[HY_PICK_PER];
#pragma unroll
    for (int k = 0; k < HY_PICK_PER; ++k) v[k] = (k < per && b0 + k < b1) ? nnz[b0 + k] : 0u;
    if (tid == 0) {
        s_prefix = 0;
        s_rem = (unsigned)n_dense;  // rank (1-based, from the top) still to find
    }
    for (int shift = 16; shift >= 0; shift -= 8) {
        for (int i = tid; i < 256; i += HY_PICK_THREADS) s_hist[i] = 0;
        __syncthreads();
        const unsigned hi_mask = shift == 16 ? 0u : (0xffffffu << (shift + 8)) & 0xffffffu;
        const unsigned prefix = s_prefix;
#pragma unroll
        for (int k = 0; k < HY_PICK_PER; ++k)
            if (b0 + k < b1 && (v[k] & hi_mask) == prefix) atomicAdd(&s_hist[(v[k] >> shift) & 255u], 1u);
        __syncthreads();
        if (tid < 32) {
            // lane l owns digits 255-8l .. 248-8l (highest first)
            unsigned c = 0;
#pragma unroll
            for (int d = 0; d < 8; ++d) c += s_hist[255 - 8 * lane - d];
            unsigned inc = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned u = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += u;
            }
            const unsigned rem = s_rem;
            const unsigned hit = __ballot_sync(0xffffffffu, inc >= rem);
            const int L = __ffs(hit) - 1;
            if (lane == L) {
                unsigned cum = inc - c;
                for (int d = 0; d < 8; ++d) {
                    const unsigned h = s_hist[255 - 8 * lane - d];
                    if (cum + h >= rem) {
                        s_prefix = prefix | ((unsigned)(255 - 8 * lane - d) << shift);
                        s_rem = rem - cum;
                        break;
                    }
                    cum += h;
                }
            }
        }
        __syncthreads();
    }
    const unsigned theta = s_prefix;
    // blocks above theta, and the equal ones in index order
    int gt = 0, eq = 0;
#pragma unroll
    for (int k = 0; k < HY_PICK_PER; ++k)
        if (b0 + k < b1) {
            gt += v[k] > theta;
            eq += v[k] == theta;
        }
    int n_gt;
    run_scan(gt, s_warp, &n_gt);
    int n_eq;
    const int eq_rank = run_scan(eq, s_warp, &n_eq);
    const int need = n_dense - n_gt;  // equal blocks to take, lowest indices first
    int take = 0;
    {
        int r = eq_rank;
#pragma unroll
        for (int k = 0; k < HY_PICK_PER; ++k)
            if (b0 + k < b1) {
                if (v[k] > theta) ++take;
                else if (v[k] == theta) take += r++ < need;
            }
    }
    int n_take;
    int pos = run_scan(take, s_warp, &n_take);
    int r = eq_rank;
#pragma unroll
    for (int k = 0; k < HY_PICK_PER; ++k)
        if (b0 + k < b1) {
            const bool t = v[k] > theta || (v[k] == theta && r++ < need);
            if (t && as_in(pos, n_dense)) idx[pos++] = b0 + k;
        }
}

// Rows 0..T-1: the dropped values of the dense blocks; rows T..T+n_out-1:
// the weight columns of the dense blocks.  A CTA takes HY_GROWS rows and its
// threads run over their (row, block) items, several loads in flight each.
constexpr int HY_GROWS = 16;

__global__ void __launch_bounds__(HY_THREADS) k_gather_dense(const __nv_bfloat16 *__restrict__ x,
                                                             const uint32_t *__restrict__ bitmask,
                                                             const __nv_bfloat16 *__restrict__ W, int T, int K,
                                                             int n_out, const int *__restrict__ idx, int n_dense,
                                                             __nv_bfloat16 *__restrict__ xr,
                                                             __nv_bfloat16 *__restrict__ wd)
{
    const long long rows = (long long)T + n_out;
    const long long r0 = (long long)blockIdx.x * HY_GROWS;
    const int items = HY_GROWS * n_dense;
#pragma unroll 4
    for (int i = threadIdx.x; i < items; i += HY_THREADS) {
        const long long r = r0 + i / n_dense;
        const int q = i % n_dense;
        if (r >= rows) continue;
        const int b = idx[q];
        if (!as_in(b, K / 4)) continue;  // a dense block index outside the row
        if (r < T) {
            uint2 v = *reinterpret_cast<const uint2 *>(x + (size_t)r * K + 4 * b);
            const uint32_t m = (bitmask[(size_t)r * ((K + 31) / 32) + (b >> 3)] >> (4 * (b & 7))) & 15u;
            // keep the dropped values (mask bit clear), zero the kept ones
            if (m & 1u) v.x &= 0xffff0000u;
            if (m & 2u) v.x &= 0x0000ffffu;
            if (m & 4u) v.y &= 0xffff0000u;
            if (m & 8u) v.y &= 0x0000ffffu;
            *reinterpret_cast<uint2 *>(xr + (size_t)r * (4 * n_dense) + 4 * q) = v;
        } else {
            const size_t o = (size_t)(r - T);
            *reinterpret_cast<uint2 *>(wd + o * (4 * n_dense) + 4 * q) =
                *reinterpret_cast<const uint2 *>(W + o * K + 4 * b);
        }
    }
}

HybridLayout hybrid_layout(int T, int K, int n_out, int n_dense)
{
    HybridLayout L{};
    auto up = [](size_t v) { return (v + 255) / 256 * 256; };
    size_t off = 0;
    L.nnz = off;    off += up((size_t)(K / 4) * 4);
    L.total = off;  off += 256;
    L.idx = off;    off += up((size_t)(n_dense > 0 ? n_dense : 1) * 4);
    L.xr = off;     off += up((size_t)T * 4 * n_dense * 2);
    L.wd = off;     off += up((size_t)n_out * 4 * n_dense * 2);
    L.bytes = off;
    return L;
}

cudaError_t launch_block_sparsity(const void *x, int T, int K, int n_dense, int *idx, float *sparsity, void *ws,
                                  cudaStream_t st)
{
    const HybridLayout L = hybrid_layout(T, K, 0, 0);
    unsigned char *base = static_cast<unsigned char *>(ws);
    unsigned *nnz = reinterpret_cast<unsigned *>(base + L.nnz);
    unsigned long long *total = reinterpret_cast<unsigned long long *>(base + L.total);
    cudaError_t e = cudaMemsetAsync(base, 0, L.idx, st);  // counts and total
    if (e != cudaSuccess) return e;
    dim3 g((K / 8 + HY_THREADS - 1) / HY_THREADS, (T + HY_TOK - 1) / HY_TOK);
    k_block_nnz<<<g, HY_THREADS, 0, st>>>(static_cast<const __nv_bfloat16 *>(x), T, K, nnz, total);
    k_pick_dense<<<1, HY_PICK_THREADS, 0, st>>>(nnz, K / 4, n_dense, total, (double)T * K, idx, sparsity);
    return cudaGetLastError();
}

cudaError_t launch_hybrid(const HybridArgs &a, cudaStream_t st)
{
    const HybridLayout L = hybrid_layout(a.T, a.K, a.n_out, a.n_dense);
    unsigned char *base = static_cast<unsigned char *>(a.workspace);
    int *idx = a.idx_out ? a.idx_out : reinterpret_cast<int *>(base + L.idx);
    float *sp = a.sparsity_out ? a.sparsity_out : reinterpret_cast<float *>(base + L.total + 16);
    cudaError_t e = launch_block_sparsity(a.x, a.T, a.K, a.n_dense, idx, sp, a.workspace, st);
    if (e != cudaSuccess) return e;
    GemmArgs s{};
    if (a.n_dense > 0) {
        __nv_bfloat16 *xr = reinterpret_cast<__nv_bfloat16 *>(base + L.xr);
        __nv_bfloat16 *wd = reinterpret_cast<__nv_bfloat16 *>(base + L.wd);
        const long long rows = (long long)a.T + a.n_out;
        k_gather_dense<<<(unsigned)((rows + HY_GROWS - 1) / HY_GROWS), HY_THREADS, 0, st>>>(static_cast<const __nv_bfloat16 *>(a.x), a.bitmask,
                                                 static_cast<const __nv_bfloat16 *>(a.W), a.T, a.K, a.n_out, idx,
                                                 a.n_dense, xr, wd);
        // the gathered remainder against the dense blocks' W columns: extra
        // dense K blocks of the 2:4 GEMM, into the same accumulator
        s.U2 = xr;
        s.Ar = wd;
        s.r = 4 * a.n_dense;
        s.u_parts = 1;
    }
    s.A = a.x_compact;
    s.meta = a.meta24;
    s.W = a.W;
    s.T = a.T;
    s.K = a.K;
    s.n_out = a.n_out;
    s.sparse = 1;
    s.y = a.y;
    s.out_bf16 = a.out_bf16;
    s.rowsum = a.rowsum;
    s.eta = a.eta;
    s.nu = a.nu;
    return launch_gemm(s, st);
}

}  // namespace as
