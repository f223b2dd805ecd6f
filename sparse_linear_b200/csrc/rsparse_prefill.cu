// R-Sparse low-rank compensation for prefill (activation-sparsity overview
// page, 激活稀疏化技术：提升LLM推理效率的动态剪枝方法, section 3.3): with
// W ~ W_sparse + A_r B_r^T (A_r = U_r S_r [n_out, r], B_r = V_r [K, r]), the
// channels the selection dropped contribute through the rank-r factors:
//   U = (xhat (.) (1 - m)) B_r          [T, r]
//   y = (xhat (.) m) W^T + U A_r^T      (+ eta rowsum_o with a token shift)
// The second product is r more columns of K in the prefill GEMM: the GEMM
// runs extra K blocks whose A operand is U (bf16 hi and lo parts) and whose
// B operand is A_r, accumulating into the same tensor-memory tile, so the
// compensation needs no pass over y.
//
// k_rsp_u    grid (128-token tiles, K splits), 8 warps: each 64-channel
//            block of x is loaded (registers, one block ahead), shifted and
//            masked to the dropped values, split into bf16 hi + lo and
//            stored in shared memory next to the block of B_r; warp w
//            multiplies tokens 16w..16w+15 by all r columns (mma.sync
//            m16n8k16, float32 accumulation).  Partial sums per split.
// k_rsp_fin  sums the splits in split order and writes U as bf16 hi (rows
//            0..T-1) and lo (rows T..2T-1) of one [2T, r] operand.
// Deterministic; xhat = fl32(x - eta) with a token shift, else x.
#include "common.cuh"
#include "kernels.cuh"
#include "select_util.cuh"

namespace as {

constexpr int RSP_THREADS = 256;
constexpr int RSP_TM = 128;       // tokens per CTA
constexpr int RSP_KB = 64;        // channels per block
constexpr int RSP_XP = RSP_KB + 8;  // padded row of a staged x block (144 bytes: ldmatrix without conflicts)

template <int R>
__global__ void __launch_bounds__(RSP_THREADS) k_rsp_u(const __nv_bfloat16 *__restrict__ x,
                                                       const uint32_t *__restrict__ mask,
                                                       const float *__restrict__ eta,
                                                       const __nv_bfloat16 *__restrict__ B, int T, int K,
                                                       int blocks_per_split, float *__restrict__ part)
{
    constexpr int BP = R + 8;  // padded row of a staged B block
    constexpr int NTN = R / 8;  // 8-column n-tiles
    // two buffers each of: the x block as bf16 hi and lo, the B_r block
    extern __shared__ __align__(16) unsigned char smem[];
    __nv_bfloat16 (*s_hi)[RSP_TM * RSP_XP] = reinterpret_cast<__nv_bfloat16 (*)[RSP_TM * RSP_XP]>(smem);
    __nv_bfloat16 (*s_lo)[RSP_TM * RSP_XP] =
        reinterpret_cast<__nv_bfloat16 (*)[RSP_TM * RSP_XP]>(smem + 2 * RSP_TM * RSP_XP * 2);
    __nv_bfloat16 (*s_b)[RSP_KB * BP] = reinterpret_cast<__nv_bfloat16 (*)[RSP_KB * BP]>(smem + 4 * RSP_TM * RSP_XP * 2);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int t0 = blockIdx.x * RSP_TM;
    const int nkb = (K + RSP_KB - 1) / RSP_KB;
    const int kb0 = blockIdx.y * blocks_per_split, kb1 = min(nkb, kb0 + blocks_per_split);
    const int words = (K + 31) / 32;

    // thread -> (row, 16-byte piece) of the x block: 128 rows x 8 pieces, 4 per thread
    uint4 xv[4];
    uint32_t mw[4];
    float ev[4];
    uint4 bv[R / 32];  // the B block: 64 rows x R/8 pieces, R/32 per thread
    auto load = [&](int kb) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int i = tid + q * RSP_THREADS, row = i >> 3, pc = i & 7;
            const int t = t0 + row, c = kb * RSP_KB + 8 * pc;
            const bool in = t < T && c < K;
            xv[q] = in ? *reinterpret_cast<const uint4 *>(x + (size_t)t * K + c) : make_uint4(0, 0, 0, 0);
            mw[q] = in ? mask[(size_t)t * words + (c >> 5)] >> (c & 31) : 0xFFu;  // out of range: "kept" (dropped = 0)
            ev[q] = (in && eta) ? eta[t] : 0.0f;
        }
#pragma unroll
        for (int q = 0; q < R / 32; ++q) {
            const int i = tid + q * RSP_THREADS, row = i / (R / 8), pc = i % (R / 8);
            const int c = kb * RSP_KB + row;
            bv[q] = c < K ? *reinterpret_cast<const uint4 *>(B + (size_t)c * R + 8 * pc) : make_uint4(0, 0, 0, 0);
        }
    };
    auto stage = [&](int buf) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int i = tid + q * RSP_THREADS, row = i >> 3, pc = i & 7;
            float v[8];
            load8(&xv[q], v);
            uint32_t hw[4], lw[4];
#pragma unroll
            for (int e2 = 0; e2 < 4; ++e2) {
                float d[2];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int e = 2 * e2 + h;
                    const bool dropped = !((mw[q] >> e) & 1u);
                    d[h] = dropped ? (eta ? __fsub_rn(v[e], ev[q]) : v[e]) : 0.0f;
                }
                const __nv_bfloat162 hh = __floats2bfloat162_rn(d[0], d[1]);
                const __nv_bfloat162 ll = __floats2bfloat162_rn(d[0] - __low2float(hh), d[1] - __high2float(hh));
                hw[e2] = *reinterpret_cast<const uint32_t *>(&hh);
                lw[e2] = *reinterpret_cast<const uint32_t *>(&ll);
            }
            *reinterpret_cast<uint4 *>(&s_hi[buf][row * RSP_XP + 8 * pc]) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
            *reinterpret_cast<uint4 *>(&s_lo[buf][row * RSP_XP + 8 * pc]) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
        }
#pragma unroll
        for (int q = 0; q < R / 32; ++q) {
            const int i = tid + q * RSP_THREADS, row = i / (R / 8), pc = i % (R / 8);
            *reinterpret_cast<uint4 *>(&s_b[buf][row * BP + 8 * pc]) = bv[q];
        }
    };

    float acc[NTN][4];
#pragma unroll
    for (int n = 0; n < NTN; ++n)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[n][i] = 0.0f;
    const int g8 = lane >> 2, q4 = lane & 3, mi = lane >> 3, mr = lane & 7;
    if (kb0 < kb1) load(kb0);
    for (int kb = kb0; kb < kb1; ++kb) {
        const int buf = (kb - kb0) & 1;
        stage(buf);
        __syncthreads();
        if (kb + 1 < kb1) load(kb + 1);  // next block in flight during the multiplies
        const uint32_t hbase = smem_u32(&s_hi[buf][0]), lbase = smem_u32(&s_lo[buf][0]), bbase = smem_u32(&s_b[buf][0]);
#pragma unroll
        for (int ks = 0; ks < RSP_KB / 16; ++ks) {
            // A: tokens 16 warp .. +15, channels 16 ks .. +15 (row-major, non-transposed)
            const uint32_t aoff = (uint32_t)(((warp * 16 + (mi & 1) * 8 + mr) * RSP_XP + ks * 16 + (mi >> 1) * 8) * 2);
            uint32_t h0, h1, h2, h3, l0, l1, l2, l3;
            asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                         : "=r"(h0), "=r"(h1), "=r"(h2), "=r"(h3) : "r"(hbase + aoff));
            asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                         : "=r"(l0), "=r"(l1), "=r"(l2), "=r"(l3) : "r"(lbase + aoff));
#pragma unroll
            for (int n = 0; n < NTN; n += 2) {
                // B: channels 16 ks .. +15 (rows of the staged block), columns 8n .. 8n+15
                const uint32_t boff = (uint32_t)(((ks * 16 + (mi & 1) * 8 + mr) * BP + n * 8 + (mi >> 1) * 8) * 2);
                uint32_t b0, b1, b2, b3;
                asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                             : "=r"(b0), "=r"(b1), "=r"(b2), "=r"(b3) : "r"(bbase + boff));
                mma_16816(acc[n], h0, h1, h2, h3, b0, b1);
                mma_16816(acc[n], l0, l1, l2, l3, b0, b1);
                mma_16816(acc[n + 1], h0, h1, h2, h3, b2, b3);
                mma_16816(acc[n + 1], l0, l1, l2, l3, b2, b3);
            }
        }
    }
    // partial sums of this split: rows g8, g8 + 8 of the warp's tokens, columns 2 q4, +1
    float *ps = part + (size_t)blockIdx.y * T * R;
#pragma unroll
    for (int n = 0; n < NTN; ++n)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int t = t0 + warp * 16 + g8 + 8 * h;
            if (t < T)
                *reinterpret_cast<float2 *>(ps + (size_t)t * R + 8 * n + 2 * q4) =
                    make_float2(acc[n][2 * h], acc[n][2 * h + 1]);
        }
}

// U = sum of the split partials in split order, as bf16 hi (rows 0..T-1)
// and lo (rows T..2T-1).
__global__ void k_rsp_fin(const float *__restrict__ part, int splits, int T, int R, __nv_bfloat16 *__restrict__ U)
{
    const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const size_t n = (size_t)T * R;
    if (i >= n) return;
    float s = 0.0f;
    for (int k = 0; k < splits; ++k) s += part[(size_t)k * n + i];
    const __nv_bfloat16 h = __float2bfloat16_rn(s);
    U[i] = h;
    U[n + i] = __float2bfloat16_rn(s - __bfloat162float(h));
}

static int rsp_splits(int T, int K)
{
    const int mt = (T + RSP_TM - 1) / RSP_TM, nkb = (K + RSP_KB - 1) / RSP_KB;
    int s = (296 + mt - 1) / mt;  // about two CTAs per SM
    if (s > nkb) s = nkb;
    if (s < 1) s = 1;
    const int per = (nkb + s - 1) / s;
    return (nkb + per - 1) / per;
}

RspLayout rsp_layout(int T, int K, int r)
{
    RspLayout L{};
    L.splits = rsp_splits(T, K);
    const int nkb = (K + RSP_KB - 1) / RSP_KB;
    L.blocks_per_split = (nkb + L.splits - 1) / L.splits;
    auto up = [](size_t v) { return (v + 255) / 256 * 256; };
    L.part = 0;
    L.u = up((size_t)L.splits * T * r * 4);
    L.bytes = L.u + up((size_t)2 * T * r * 2);
    return L;
}

cudaError_t launch_rsp_u(const void *x, const uint32_t *mask, const float *eta, const void *B, int T, int K, int r,
                         void *ws, cudaStream_t st)
{
    const RspLayout L = rsp_layout(T, K, r);
    unsigned char *base = static_cast<unsigned char *>(ws);
    float *part = reinterpret_cast<float *>(base + L.part);
    __nv_bfloat16 *U = reinterpret_cast<__nv_bfloat16 *>(base + L.u);
    dim3 grid((T + RSP_TM - 1) / RSP_TM, L.splits);
    const __nv_bfloat16 *xb = static_cast<const __nv_bfloat16 *>(x), *Bb = static_cast<const __nv_bfloat16 *>(B);
    const size_t smem = (size_t)4 * RSP_TM * RSP_XP * 2 + (size_t)2 * RSP_KB * (r + 8) * 2;
    cudaError_t e;
    if (r == 64) {
        static int done[64];
        e = smem_limit_once(k_rsp_u<64>, smem, done);
        if (e == cudaSuccess)
            k_rsp_u<64><<<grid, RSP_THREADS, smem, st>>>(xb, mask, eta, Bb, T, K, L.blocks_per_split, part);
    } else {
        static int done[64];
        e = smem_limit_once(k_rsp_u<128>, smem, done);
        if (e == cudaSuccess)
            k_rsp_u<128><<<grid, RSP_THREADS, smem, st>>>(xb, mask, eta, Bb, T, K, L.blocks_per_split, part);
    }
    if (e != cudaSuccess) return e;
    const size_t n = (size_t)T * r;
    k_rsp_fin<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(part, L.splits, T, r, U);
    return cudaGetLastError();
}

}  // namespace as
