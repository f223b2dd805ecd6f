// Prefill contraction y = A W^T on the 5th-generation tensor cores.
//
// Dense variant (masked activations, any N:M or top-k selection):
//   tcgen05.mma kind::f16, M=128, N=256, K=16 per instruction.
// Sparse variant (2:4 selection): the 2:4 + Squared-ReLU page
// (利用2:4稀疏性与Squared-ReLU加速Transformer训练与推理) section 2.1: when A
// holds two nonzeros in every four consecutive K elements, the tensor core
// skips half of the multiply-adds.  A is the compacted half (x_compact) and
// the positions live in tensor memory; tcgen05.mma.sp kind::f16, M=128,
// N=128, K=32 (logical) per instruction.
//
// Persistent, warp-specialised CTA (one per SM, 192 threads):
//   warp 0   TMA producer: A and W tiles (128-byte swizzle, K-major) and the
//            2:4 metadata tile into a STAGES-deep shared-memory ring.
//   warp 1   allocates tensor memory; one thread issues the MMAs (and, for
//            the sparse variant, copies each metadata tile into TMEM first).
//   warps 2-5 epilogue: TMEM -> registers (tcgen05.ld), eta*rowsum or nu
//            scaling, rounding, stores.  Two accumulator buffers let the
//            epilogue of one tile overlap the main loop of the next.
// No load uses cluster multicast.  Every mbarrier wait is bounded.
#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"

namespace as {

constexpr int GEMM_THREADS = 192;
constexpr int GEMM_BM = 128;
constexpr int GEMM_GROUP_M = 16;  // tile raster: 16 row tiles share each weight tile

template <bool SPARSE>
struct GemmCfg;
template <>
struct GemmCfg<false> {
    static constexpr int BN = 256;
    static constexpr int STAGES = 4;
    static constexpr int KB = 64;                         // logical K per stage
    static constexpr int A_BYTES = GEMM_BM * 64 * 2;      // 128 rows x 128 B
    static constexpr int B_BYTES = BN * 64 * 2;           // 256 rows x 128 B
    static constexpr int M_BYTES = 0;
    static constexpr int MMAS = 4;                        // K = 16 each
    static constexpr int NACC = 2;
};
template <>
struct GemmCfg<true> {
    static constexpr int BN = 128;
    static constexpr int STAGES = 4;
    static constexpr int KB = 128;                        // logical K per stage (64 kept)
    static constexpr int A_BYTES = GEMM_BM * 64 * 2;      // compact half: 128 rows x 128 B
    static constexpr int B_BYTES = BN * 128 * 2;          // two 128-byte-wide K sub-tiles
    static constexpr int M_BYTES = 2048;                  // 128 lanes x 16 B of positions
    static constexpr int MMAS = 4;                        // K = 32 (logical) each
    static constexpr int NACC = 2;
};

template <bool SPARSE>
constexpr size_t gemm_smem_bytes()
{
    using C = GemmCfg<SPARSE>;
    return 1024 /* alignment slack */ + (size_t)C::STAGES * (C::A_BYTES + C::B_BYTES + C::M_BYTES) + 256;
}

struct GemmParams {
    const uint32_t *meta;
    const float *rowsum, *eta, *nu;
    const float *xscale, *wscale;  // FP8 row scales (tokens, output rows)
    void *y;
    int T, K, n_out, out_bf16;
    int m_tiles, n_tiles, k_blocks, meta_kt;
    int kb_pass;  // K blocks of one pass over K
    int kb_main;  // kb_pass, or 2 kb_pass when a residual A operand follows
    int rblk;     // extra dense blocks: 64-wide blocks of r (k_blocks = kb_main + u_parts rblk)
};

// Extra K block e (0 .. u_parts rblk - 1): which part of U (R-Sparse: 0 hi,
// 1 lo) and which 64-wide block of r it covers.
__device__ __forceinline__ void extra_block(int e, int rblk, int &part, int &j)
{
    part = e / rblk;
    j = e - part * rblk;
}

__device__ __forceinline__ void tile_coords(int tile, int m_tiles, int n_tiles, int &mt, int &nt)
{
    const int per_group = GEMM_GROUP_M * n_tiles;
    const int group = tile / per_group, rem = tile % per_group;
    const int gm = min(GEMM_GROUP_M, m_tiles - group * GEMM_GROUP_M);
    mt = group * GEMM_GROUP_M + rem % gm;
    nt = rem / gm;
}

template <bool SPARSE>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    k_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
           const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmU,
           const __grid_constant__ CUtensorMap tmR, GemmParams p)
{
    using C = GemmCfg<SPARSE>;
    constexpr int BN = C::BN, S = C::STAGES;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                            ~uintptr_t(1023));
    unsigned char *sA = smem;
    unsigned char *sB = sA + S * C::A_BYTES;
    unsigned char *sM = sB + S * C::B_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sM + S * C::M_BYTES);
    uint64_t *full = bars, *empty = bars + S, *acc_full = bars + 2 * S, *acc_empty = bars + 2 * S + 2;
    uint64_t *drain = bars + 2 * S + 4;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * S + 5);
    int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_tiles = p.m_tiles * p.n_tiles;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], 4);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
        prefetch_tensormap(&tmA2);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            for (int tile = blockIdx.x; tile < num_tiles && !*(volatile int *)abort_flag; tile += gridDim.x) {
                int mt, nt;
                tile_coords(tile, p.m_tiles, p.n_tiles, mt, nt);
                for (int kb = 0; kb < p.k_blocks; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1)) { *(volatile int *)abort_flag = 1; break; }
                    if (kb >= p.kb_main) {  // R-Sparse: U (dense) against A_r, first B sub-tile only
                        int part, j;
                        extra_block(kb - p.kb_main, p.rblk, part, j);
                        mbar_arrive_expect_tx(&full[stage], C::A_BYTES + (SPARSE ? C::B_BYTES / 2 : C::B_BYTES));
                        tma_load_2d(sA + stage * C::A_BYTES, &tmU, &full[stage], j * 64, mt * GEMM_BM + part * p.T);
                        tma_load_2d(sB + stage * C::B_BYTES, &tmR, &full[stage], j * 64, nt * BN);
                        if (++stage == S) { stage = 0; phase ^= 1; }
                        continue;
                    }
                    mbar_arrive_expect_tx(&full[stage], C::A_BYTES + C::B_BYTES + C::M_BYTES);
                    // second pass over K: the residual operand against the same W blocks
                    const bool lo = kb >= p.kb_pass;
                    const int kk = lo ? kb - p.kb_pass : kb;
                    unsigned char *a_dst = sA + stage * C::A_BYTES;
                    unsigned char *b_dst = sB + stage * C::B_BYTES;
                    tma_load_2d(a_dst, lo ? &tmA2 : &tmA, &full[stage], kk * 64, mt * GEMM_BM);
                    if constexpr (SPARSE) {
                        tma_load_2d(b_dst, &tmB, &full[stage], kk * 128, nt * BN);
                        tma_load_2d(b_dst + BN * 128, &tmB, &full[stage], kk * 128 + 64, nt * BN);
                        const uint32_t *src = p.meta + ((size_t)mt * p.meta_kt + kk) * 512;
                        bulk_load(sM + stage * C::M_BYTES, src, C::M_BYTES, &full[stage]);
                    } else {
                        tma_load_2d(b_dst, &tmB, &full[stage], kk * 64, nt * BN);
                    }
                    if (++stage == S) { stage = 0; phase ^= 1; }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16(GEMM_BM, BN, SPARSE);
            const uint32_t meta_tmem = tmem + C::NACC * BN;
            int stage = 0;
            uint32_t phase = 0;
            int it = 0;
            for (int tile = blockIdx.x; tile < num_tiles && !*(volatile int *)abort_flag; tile += gridDim.x, ++it) {
                const int acc = it & 1;
                const uint32_t acc_phase = (it >> 1) & 1;
                if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1)) { *(volatile int *)abort_flag = 1; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem + acc * BN;
                bool ok = true;
                for (int kb = 0; kb < p.k_blocks; ++kb) {
                    if (!mbar_wait(&full[stage], phase)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(sA + stage * C::A_BYTES);
                    const uint32_t b_addr = smem_u32(sB + stage * C::B_BYTES);
                    const uint64_t a_desc = sdesc_kmajor_sw128(a_addr);
                    if (SPARSE && kb >= p.kb_main) {  // R-Sparse block: dense MMAs into the same accumulator
                        const uint64_t b_desc = sdesc_kmajor_sw128(b_addr);
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            mma_bf16(d_tmem, a_desc + (uint64_t)((32 * j) >> 4), b_desc + (uint64_t)((32 * j) >> 4),
                                     idesc_bf16(GEMM_BM, BN, false), 1u);
                    } else if constexpr (SPARSE) {
                        const uint32_t e_tmem = meta_tmem + stage * 4;
                        tmem_cp_128x128b(e_tmem, sdesc_rows16(smem_u32(sM + stage * C::M_BYTES)));
#pragma unroll
                        for (int j = 0; j < C::MMAS; ++j) {
                            // step j: kept K elements [16j, 16j+16) of A (32 bytes in),
                            // logical K [32j, 32j+32) of W: sub-tile j/2, 64 bytes in
                            const uint64_t a_j = a_desc + (uint64_t)((32 * j) >> 4);
                            const uint64_t b_j =
                                sdesc_kmajor_sw128(b_addr + (j >> 1) * (BN * 128) + (j & 1) * 64);
                            // metadata column e_tmem + j, addressed as the even column
                            // plus the selector (bit 0 of the instruction descriptor)
                            mma_sp_bf16(d_tmem, a_j, b_j, idesc | (uint32_t)(j & 1), e_tmem + (j & ~1),
                                        (kb | j) != 0);
                        }
                    } else {
                        const uint64_t b_desc = sdesc_kmajor_sw128(b_addr);
#pragma unroll
                        for (int j = 0; j < C::MMAS; ++j)
                            mma_bf16(d_tmem, a_desc + (uint64_t)((32 * j) >> 4), b_desc + (uint64_t)((32 * j) >> 4),
                                     idesc, (kb | j) != 0);
                    }
                    tc_commit(&empty[stage]);  // frees the stage when these MMAs finish
                    if (++stage == S) { stage = 0; phase ^= 1; }
                }
                if (!ok) { *(volatile int *)abort_flag = 1; break; }
                tc_commit(&acc_full[acc]);
            }
            // drain: wait until every MMA issued above has completed
            tc_commit(drain);
            mbar_wait(drain, 0);
        }
    } else {
        // ------------------------------------------------ epilogue (warps 2..5)
        const int q = warp & 3;  // TMEM lanes 32q..32q+31
        int it = 0;
        for (int tile = blockIdx.x; tile < num_tiles && !*(volatile int *)abort_flag; tile += gridDim.x, ++it) {
            const int acc = it & 1;
            const uint32_t acc_phase = (it >> 1) & 1;
            int mt, nt;
            tile_coords(tile, p.m_tiles, p.n_tiles, mt, nt);
            if (!mbar_wait(&acc_full[acc], acc_phase)) { *(volatile int *)abort_flag = 1; break; }
            tc_fence_after();
            const int row = mt * GEMM_BM + 32 * q + lane;
            const bool row_ok = row < p.T;
            float rscale = 1.0f, reta = 0.0f;
            if (row_ok) {
                if (p.nu) rscale = p.nu[row];
                if (p.eta) reta = p.eta[row];
            }
#pragma unroll 1
            for (int ch = 0; ch < BN / 32; ++ch) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * q) << 16) + acc * BN + ch * 32, r);
                tmem_ld_wait();
                const int col0 = nt * BN + ch * 32;
                if (!row_ok || col0 >= p.n_out) continue;
                if (!as_in((long long)row * p.n_out + min(col0 + 31, p.n_out - 1), (long long)p.T * p.n_out)) continue;
                float v[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    float f = __uint_as_float(r[i]);
                    if (p.nu) f *= rscale;
                    if (p.eta) {
                        const int c = min(col0 + i, p.n_out - 1);
                        f = fmaf(reta, p.rowsum[c], f);
                    }
                    v[i] = f;
                }
                if (p.out_bf16) {
                    __nv_bfloat16 *yr = static_cast<__nv_bfloat16 *>(p.y) + (size_t)row * p.n_out + col0;
#pragma unroll
                    for (int c8 = 0; c8 < 4; ++c8) {
                        if (col0 + 8 * c8 < p.n_out) {
                            uint32_t w[4];
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                __nv_bfloat162 h = __floats2bfloat162_rn(v[8 * c8 + 2 * i], v[8 * c8 + 2 * i + 1]);
                                w[i] = *reinterpret_cast<uint32_t *>(&h);
                            }
                            *reinterpret_cast<uint4 *>(yr + 8 * c8) = make_uint4(w[0], w[1], w[2], w[3]);
                        }
                    }
                } else {
                    float *yr = static_cast<float *>(p.y) + (size_t)row * p.n_out + col0;
#pragma unroll
                    for (int c4 = 0; c4 < 8; ++c4)
                        if (col0 + 4 * c4 < p.n_out)
                            *reinterpret_cast<float4 *>(yr + 4 * c4) =
                                make_float4(v[4 * c4], v[4 * c4 + 1], v[4 * c4 + 2], v[4 * c4 + 3]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[acc]);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------- sparse, CTA pair (2 SMs)
// The same 2:4 contraction with two SMs of a cluster working as one
// 256 x 256 tile (tcgen05.mma.sp.cta_group::2, M = 256, N = 256, K = 32
// logical per instruction).  Each CTA stages its own 128 rows of A, its own
// 2:4 positions and half (128 rows) of the weight tile; the leader CTA
// issues the MMAs, which read both CTAs' shared memory and write each CTA's
// tensor memory (its 128 rows x 256 columns).  Per SM this halves the
// weight bytes fetched per multiply-add compared with the 1-SM 128 x 128
// tile, which is what bounds that kernel (L2 -> SM bandwidth).
//   warp 0      TMA producer (both CTAs); the leader's full barrier counts
//               the bytes of both CTAs.
//   warp 1      tensor-memory allocation (both CTAs, cta_group::2); lane 0
//               of the leader issues metadata copies and MMAs.
//   warps 2-9   epilogue: (lane quarter, column half) per warp; the whole
//               accumulator slice is read into registers and released
//               before the scaling and the stores, so the next tile's MMAs
//               overlap the stores.
// Loads carry no multicast; only tcgen05.commit signals both CTAs.
//
// FP8 variant (2:4 + Squared-ReLU page section 3.1, FP8 row-scaled 2:4 GEMM):
// tcgen05.mma.sp kind::f8f6f4 with E4M3 A and B, K = 64 (logical) per
// instruction.  A stage holds the same bytes (128 compact codes per row =
// 256 logical K; B two 128-byte sub-tiles) and twice the positions: each
// instruction reads 64 position bits per row from two TMEM columns (row =
// lane).  The epilogue multiplies by the token's and the output row's scale.
constexpr int PAIR_THREADS = 320;
constexpr int PAIR_BM = 256;  // rows per CTA pair (128 per CTA)
constexpr int PAIR_BN = 256;  // weight rows per CTA pair (128 per CTA)
constexpr int PAIR_STAGES = 4;
constexpr int PAIR_A_BYTES = 128 * 128;      // kept half of 128 rows: 128 bytes per row
constexpr int PAIR_B_BYTES = 128 * 256;      // 128 weight rows x 256 bytes, two sub-tiles

template <bool FP8>
struct PairCfg {
    static constexpr int M_BYTES = FP8 ? 4096 : 2048;  // positions of 128 rows x one K block
    static constexpr int STAGE_BYTES = PAIR_A_BYTES + PAIR_B_BYTES + M_BYTES;
    static constexpr int KB = FP8 ? 256 : 128;         // logical K per stage
    static constexpr int KA = KB / 2;                  // compact A elements per stage
    static constexpr int BSUB = FP8 ? 128 : 64;        // B elements per 128-byte sub-tile
    static constexpr int META_COLS = FP8 ? 8 : 4;      // TMEM columns of positions per stage
};

template <bool FP8>
constexpr size_t pair_smem_bytes() { return 1024 + (size_t)PAIR_STAGES * PairCfg<FP8>::STAGE_BYTES + 256; }

template <bool FP8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PAIR_THREADS, 1)
    k_gemm_sp_pair(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmE, const __grid_constant__ CUtensorMap tmA2,
                   const __grid_constant__ CUtensorMap tmU, const __grid_constant__ CUtensorMap tmR, GemmParams p)
{
    using C = PairCfg<FP8>;
    constexpr int S = PAIR_STAGES;
    constexpr int PAIR_M_BYTES = C::M_BYTES;
    constexpr int PAIR_STAGE_BYTES = C::STAGE_BYTES;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                            ~uintptr_t(1023));
    unsigned char *sA = smem;
    unsigned char *sB = sA + S * PAIR_A_BYTES;
    unsigned char *sM = sB + S * PAIR_B_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sM + S * PAIR_M_BYTES);
    uint64_t *full = bars, *empty = bars + S, *acc_full = bars + 2 * S, *acc_empty = bars + 2 * S + 1;
    uint64_t *drain = bars + 2 * S + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * S + 3);
    int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const int num_tiles = p.m_tiles * p.n_tiles;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);   // the leader's expect_tx arrival (+ both CTAs' bytes)
            mbar_init(&empty[s], 1);  // one commit from the leader's MMA thread
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 16);  // 8 epilogue warps in each CTA (leader's copy is the one used)
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
        prefetch_tensormap(&tmE);
        prefetch_tensormap(&tmA2);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, 512);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync_all();  // barriers of both CTAs initialised before either uses the other's
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            for (int tile = pair; tile < num_tiles && !*(volatile int *)abort_flag; tile += npairs) {
                int mt, nt;
                tile_coords(tile, p.m_tiles, p.n_tiles, mt, nt);
                const int arow = mt * PAIR_BM + 128 * (int)rank;
                const int brow = nt * PAIR_BN + 128 * (int)rank;
                const int echunk = (2 * mt + (int)rank) * p.meta_kt;
                for (int kb = 0; kb < p.k_blocks; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1)) { *(volatile int *)abort_flag = 1; break; }
                    if (!FP8 && kb >= p.kb_main) {  // R-Sparse: U (dense) against A_r, first B sub-tile only
                        int part, j;
                        extra_block(kb - p.kb_main, p.rblk, part, j);
                        if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * (PAIR_A_BYTES + 128 * 128));
                        const uint32_t bar = mapa_u32(smem_u32(&full[stage]), 0);
                        tma_load_2d_pair(sA + stage * PAIR_A_BYTES, &tmU, bar, j * 64, arow + part * p.T);
                        tma_load_2d_pair(sB + stage * PAIR_B_BYTES, &tmR, bar, j * 64, brow);
                        if (++stage == S) { stage = 0; phase ^= 1; }
                        continue;
                    }
                    if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * PAIR_STAGE_BYTES);
                    const uint32_t bar = mapa_u32(smem_u32(&full[stage]), 0);
                    // second pass over K: the residual operand, same positions and W blocks
                    const bool lo = kb >= p.kb_pass;
                    const int kk = lo ? kb - p.kb_pass : kb;
                    unsigned char *b_dst = sB + stage * PAIR_B_BYTES;
                    tma_load_2d_pair(sA + stage * PAIR_A_BYTES, lo ? &tmA2 : &tmA, bar, kk * C::KA, arow);
                    tma_load_2d_pair(b_dst, &tmB, bar, kk * C::KB, brow);
                    tma_load_2d_pair(b_dst + 128 * 128, &tmB, bar, kk * C::KB + C::BSUB, brow);
                    tma_load_2d_pair(sM + stage * PAIR_M_BYTES, &tmE, bar, 0, (echunk + kk) * (PAIR_M_BYTES / 256));
                    if constexpr (FP8)
                        tma_load_2d_pair(sM + stage * PAIR_M_BYTES + 2048, &tmE, bar, 0,
                                         (echunk + kk) * (PAIR_M_BYTES / 256) + 8);
                    if (++stage == S) { stage = 0; phase ^= 1; }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (leader only)
        if (rank == 0 && lane == 0) {
            constexpr uint32_t idesc = FP8 ? idesc_e4m3(PAIR_BM, PAIR_BN, true) : idesc_bf16(PAIR_BM, PAIR_BN, true);
            const uint32_t meta_tmem = tmem + PAIR_BN;
            int stage = 0;
            uint32_t phase = 0;
            int it = 0;
            for (int tile = pair; tile < num_tiles && !*(volatile int *)abort_flag; tile += npairs, ++it) {
                if (!mbar_wait(acc_empty, (it & 1) ^ 1)) { *(volatile int *)abort_flag = 1; break; }
                tc_fence_after();
                bool ok = true;
                for (int kb = 0; kb < p.k_blocks; ++kb) {
                    if (!mbar_wait(&full[stage], phase)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t b_addr = smem_u32(sB + stage * PAIR_B_BYTES);
                    const uint64_t a_desc = sdesc_kmajor_sw128(smem_u32(sA + stage * PAIR_A_BYTES));
                    if (!FP8 && kb >= p.kb_main) {  // R-Sparse block: dense MMAs into the same accumulator
                        const uint64_t b_desc = sdesc_kmajor_sw128(b_addr);
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            mma_bf16_pair(tmem, a_desc + (uint64_t)((32 * j) >> 4), b_desc + (uint64_t)((32 * j) >> 4),
                                          idesc_bf16(PAIR_BM, PAIR_BN, false), 1u);
                        tc_commit_pair_mc(&empty[stage], 0x3);
                        if (++stage == S) { stage = 0; phase ^= 1; }
                        continue;
                    }
                    const uint32_t e_tmem = meta_tmem + stage * C::META_COLS;
                    tmem_cp_128x128b_pair(e_tmem, sdesc_rows16(smem_u32(sM + stage * PAIR_M_BYTES)));
                    if constexpr (FP8)
                        tmem_cp_128x128b_pair(e_tmem + 4, sdesc_rows16(smem_u32(sM + stage * PAIR_M_BYTES + 2048)));
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint64_t a_j = a_desc + (uint64_t)((32 * j) >> 4);
                        const uint64_t b_j = sdesc_kmajor_sw128(b_addr + (j >> 1) * (128 * 128) + (j & 1) * 64);
                        if constexpr (FP8)
                            mma_sp_e4m3_pair(tmem, a_j, b_j, idesc, e_tmem + 2 * j, (kb | j) != 0);
                        else
                            mma_sp_bf16_pair(tmem, a_j, b_j, idesc | (uint32_t)(j & 1), e_tmem + (j & ~1),
                                             (kb | j) != 0);
                    }
                    tc_commit_pair_mc(&empty[stage], 0x3);  // frees the stage in both CTAs
                    if (++stage == S) { stage = 0; phase ^= 1; }
                }
                if (!ok) { *(volatile int *)abort_flag = 1; break; }
                tc_commit_pair_mc(acc_full, 0x3);
            }
            tc_commit_pair(drain);
            mbar_wait(drain, 0);
        }
    } else {
        // ------------------------------------------------ epilogue (warps 2..9)
        const int q = warp & 3;           // TMEM lanes 32q..32q+31
        const int h = (warp - 2) >> 2;    // accumulator columns [128h, 128h+128)
        const uint32_t acc_empty_leader = mapa_u32(smem_u32(acc_empty), 0);
        int it = 0;
        for (int tile = pair; tile < num_tiles && !*(volatile int *)abort_flag; tile += npairs, ++it) {
            int mt, nt;
            tile_coords(tile, p.m_tiles, p.n_tiles, mt, nt);
            if (!mbar_wait(acc_full, it & 1)) { *(volatile int *)abort_flag = 1; break; }
            tc_fence_after();
            uint32_t r[4][32];
#pragma unroll
            for (int ch = 0; ch < 4; ++ch)
                tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * q) << 16) + 128 * h + 32 * ch, r[ch]);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(acc_empty_leader);

            const int row = mt * PAIR_BM + 128 * (int)rank + 32 * q + lane;
            if (row >= p.T) continue;
            float rscale = 1.0f, reta = 0.0f, xs = 1.0f;
            if (p.nu) rscale = p.nu[row];
            if (p.eta) reta = p.eta[row];
            if (FP8) xs = p.xscale[row];
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                const int col0 = nt * PAIR_BN + 128 * h + 32 * ch;
                if (col0 >= p.n_out) continue;
                if (!as_in((long long)row * p.n_out + min(col0 + 31, p.n_out - 1), (long long)p.T * p.n_out)) continue;
                if constexpr (FP8) {
                    // n_out % 8 == 0: every 4-column group past col0 starts in range
                    // or is clamped to the last one (its values are not stored)
#pragma unroll
                    for (int c4 = 0; c4 < 8; ++c4) {
                        const int c = min(col0 + 4 * c4, p.n_out - 4);
                        const float4 w4 = *reinterpret_cast<const float4 *>(p.wscale + c);
                        const float ws[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            r[ch][4 * c4 + i] = __float_as_uint((__uint_as_float(r[ch][4 * c4 + i]) * xs) * ws[i]);
                    }
                }
                float v[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    float f = __uint_as_float(r[ch][i]);
                    if (p.nu) f *= rscale;
                    if (p.eta) {
                        const int c = min(col0 + i, p.n_out - 1);
                        f = fmaf(reta, p.rowsum[c], f);
                    }
                    v[i] = f;
                }
                if (p.out_bf16) {
                    __nv_bfloat16 *yr = static_cast<__nv_bfloat16 *>(p.y) + (size_t)row * p.n_out + col0;
#pragma unroll
                    for (int c8 = 0; c8 < 4; ++c8) {
                        if (col0 + 8 * c8 < p.n_out) {
                            uint32_t w[4];
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                __nv_bfloat162 hh = __floats2bfloat162_rn(v[8 * c8 + 2 * i], v[8 * c8 + 2 * i + 1]);
                                w[i] = *reinterpret_cast<uint32_t *>(&hh);
                            }
                            *reinterpret_cast<uint4 *>(yr + 8 * c8) = make_uint4(w[0], w[1], w[2], w[3]);
                        }
                    }
                } else {
                    float *yr = static_cast<float *>(p.y) + (size_t)row * p.n_out + col0;
#pragma unroll
                    for (int c4 = 0; c4 < 8; ++c4)
                        if (col0 + 4 * c4 < p.n_out)
                            *reinterpret_cast<float4 *>(yr + 4 * c4) =
                                make_float4(v[4 * c4], v[4 * c4 + 1], v[4 * c4 + 2], v[4 * c4 + 3]);
                }
            }
        }
    }

    // Both CTAs' tensor memory stays allocated until the leader's last MMA
    // has completed and both epilogues have read their accumulators.
    tc_fence_before();
    cluster_sync_all();
    tc_fence_after();
    if (warp == 1) tmem_dealloc_pair(tmem, 512);
}

// -------------------------------------------------- dense, CTA pair (2 SMs)
// The masked dense contraction on a CTA pair: 256 x 256 output tile per pair
// (tcgen05.mma.cta_group::2.kind::f16, M = 256, N = 256, K = 16 per
// instruction).  Each CTA stages its own 128 rows of A and half (128 rows) of
// the weight tile per 64-wide K block; the leader issues the MMAs.  Without
// 2:4 positions two 256-column accumulators fit in tensor memory, so the
// epilogue of one tile overlaps the main loop of the next.
constexpr int DP_STAGES = 6;
constexpr int DP_A_BYTES = 128 * 64 * 2;
constexpr int DP_B_BYTES = 128 * 64 * 2;
constexpr int DP_STAGE_BYTES = DP_A_BYTES + DP_B_BYTES;

constexpr size_t dense_pair_smem_bytes() { return 1024 + (size_t)DP_STAGES * DP_STAGE_BYTES + 256; }

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PAIR_THREADS, 1)
    k_gemm_dense_pair(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmU,
                      const __grid_constant__ CUtensorMap tmR, GemmParams p)
{
    constexpr int S = DP_STAGES;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                            ~uintptr_t(1023));
    unsigned char *sA = smem;
    unsigned char *sB = sA + S * DP_A_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sB + S * DP_B_BYTES);
    uint64_t *full = bars, *empty = bars + S, *acc_full = bars + 2 * S, *acc_empty = bars + 2 * S + 2;
    uint64_t *drain = bars + 2 * S + 4;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * S + 5);
    int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const int num_tiles = p.m_tiles * p.n_tiles;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);   // the leader's expect_tx arrival (+ both CTAs' bytes)
            mbar_init(&empty[s], 1);  // one commit from the leader's MMA thread
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], 16);  // 8 epilogue warps in each CTA (the leader's copy is used)
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
        prefetch_tensormap(&tmA2);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, 512);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync_all();  // barriers of both CTAs initialised before either uses the other's
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            for (int tile = pair; tile < num_tiles && !*(volatile int *)abort_flag; tile += npairs) {
                int mt, nt;
                tile_coords(tile, p.m_tiles, p.n_tiles, mt, nt);
                const int arow = mt * PAIR_BM + 128 * (int)rank;
                const int brow = nt * PAIR_BN + 128 * (int)rank;
                for (int kb = 0; kb < p.k_blocks; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1)) { *(volatile int *)abort_flag = 1; break; }
                    if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * DP_STAGE_BYTES);
                    const uint32_t bar = mapa_u32(smem_u32(&full[stage]), 0);
                    if (kb >= p.kb_main) {  // R-Sparse: U against A_r
                        int part, j;
                        extra_block(kb - p.kb_main, p.rblk, part, j);
                        tma_load_2d_pair(sA + stage * DP_A_BYTES, &tmU, bar, j * 64, arow + part * p.T);
                        tma_load_2d_pair(sB + stage * DP_B_BYTES, &tmR, bar, j * 64, brow);
                        if (++stage == S) { stage = 0; phase ^= 1; }
                        continue;
                    }
                    // second pass over K: the residual operand against the same W blocks
                    const bool lo = kb >= p.kb_pass;
                    const int kk = lo ? kb - p.kb_pass : kb;
                    tma_load_2d_pair(sA + stage * DP_A_BYTES, lo ? &tmA2 : &tmA, bar, kk * 64, arow);
                    tma_load_2d_pair(sB + stage * DP_B_BYTES, &tmB, bar, kk * 64, brow);
                    if (++stage == S) { stage = 0; phase ^= 1; }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (leader only)
        if (rank == 0 && lane == 0) {
            constexpr uint32_t idesc = idesc_bf16(PAIR_BM, PAIR_BN, false);
            int stage = 0;
            uint32_t phase = 0;
            int it = 0;
            for (int tile = pair; tile < num_tiles && !*(volatile int *)abort_flag; tile += npairs, ++it) {
                const int acc = it & 1;
                const uint32_t acc_phase = (it >> 1) & 1;
                if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1)) { *(volatile int *)abort_flag = 1; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem + acc * PAIR_BN;
                bool ok = true;
                for (int kb = 0; kb < p.k_blocks; ++kb) {
                    if (!mbar_wait(&full[stage], phase)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t a_desc = sdesc_kmajor_sw128(smem_u32(sA + stage * DP_A_BYTES));
                    const uint64_t b_desc = sdesc_kmajor_sw128(smem_u32(sB + stage * DP_B_BYTES));
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        mma_bf16_pair(d_tmem, a_desc + (uint64_t)((32 * j) >> 4), b_desc + (uint64_t)((32 * j) >> 4),
                                      idesc, (kb | j) != 0);
                    tc_commit_pair_mc(&empty[stage], 0x3);  // frees the stage in both CTAs
                    if (++stage == S) { stage = 0; phase ^= 1; }
                }
                if (!ok) { *(volatile int *)abort_flag = 1; break; }
                tc_commit_pair_mc(&acc_full[acc], 0x3);
            }
            tc_commit_pair(drain);
            mbar_wait(drain, 0);
        }
    } else {
        // ------------------------------------------------ epilogue (warps 2..9)
        const int q = warp & 3;           // TMEM lanes 32q..32q+31
        const int h = (warp - 2) >> 2;    // accumulator columns [128h, 128h+128)
        const uint32_t leader_empty0 = mapa_u32(smem_u32(&acc_empty[0]), 0);
        int it = 0;
        for (int tile = pair; tile < num_tiles && !*(volatile int *)abort_flag; tile += npairs, ++it) {
            const int acc = it & 1;
            const uint32_t acc_phase = (it >> 1) & 1;
            int mt, nt;
            tile_coords(tile, p.m_tiles, p.n_tiles, mt, nt);
            if (!mbar_wait(&acc_full[acc], acc_phase)) { *(volatile int *)abort_flag = 1; break; }
            tc_fence_after();
            uint32_t r[4][32];
#pragma unroll
            for (int ch = 0; ch < 4; ++ch)
                tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * q) << 16) + acc * PAIR_BN + 128 * h + 32 * ch, r[ch]);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(leader_empty0 + 8u * (uint32_t)acc);

            const int row = mt * PAIR_BM + 128 * (int)rank + 32 * q + lane;
            if (row >= p.T) continue;
            float rscale = 1.0f, reta = 0.0f;
            if (p.nu) rscale = p.nu[row];
            if (p.eta) reta = p.eta[row];
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                const int col0 = nt * PAIR_BN + 128 * h + 32 * ch;
                if (col0 >= p.n_out) continue;
                if (!as_in((long long)row * p.n_out + min(col0 + 31, p.n_out - 1), (long long)p.T * p.n_out)) continue;
                float v[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    float f = __uint_as_float(r[ch][i]);
                    if (p.nu) f *= rscale;
                    if (p.eta) {
                        const int c = min(col0 + i, p.n_out - 1);
                        f = fmaf(reta, p.rowsum[c], f);
                    }
                    v[i] = f;
                }
                if (p.out_bf16) {
                    __nv_bfloat16 *yr = static_cast<__nv_bfloat16 *>(p.y) + (size_t)row * p.n_out + col0;
#pragma unroll
                    for (int c8 = 0; c8 < 4; ++c8) {
                        if (col0 + 8 * c8 < p.n_out) {
                            uint32_t w[4];
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                __nv_bfloat162 hh = __floats2bfloat162_rn(v[8 * c8 + 2 * i], v[8 * c8 + 2 * i + 1]);
                                w[i] = *reinterpret_cast<uint32_t *>(&hh);
                            }
                            *reinterpret_cast<uint4 *>(yr + 8 * c8) = make_uint4(w[0], w[1], w[2], w[3]);
                        }
                    }
                } else {
                    float *yr = static_cast<float *>(p.y) + (size_t)row * p.n_out + col0;
#pragma unroll
                    for (int c4 = 0; c4 < 8; ++c4)
                        if (col0 + 4 * c4 < p.n_out)
                            *reinterpret_cast<float4 *>(yr + 4 * c4) =
                                make_float4(v[4 * c4], v[4 * c4 + 1], v[4 * c4 + 2], v[4 * c4 + 3]);
                }
            }
        }
    }

    // Both CTAs' tensor memory stays allocated until the leader's last MMA
    // has completed and both epilogues have read their accumulators.
    tc_fence_before();
    cluster_sync_all();
    tc_fence_after();
    if (warp == 1) tmem_dealloc_pair(tmem, 512);
}

// ---------------------------------------------------------------- host side
typedef CUresult (*PFN_encodeTiled_t)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                      const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                      CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                      CUtensorMapFloatOOBfill);

static PFN_encodeTiled_t encode_fn()
{
    static PFN_encodeTiled_t fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_encodeTiled_t>(ptr);
    }
    return fn;
}

// 2-D bf16 tensor [rows, cols] (cols contiguous), box {64 cols, box_rows}.
static bool make_map(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows)
{
    PFN_encodeTiled_t enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2:4 positions as a 2-D uint32 tensor of 256-byte rows: one 2 KB chunk
// (128 rows x 128 K of A) is 8 rows, box {64, 8}, no swizzle.
static bool make_map_meta(CUtensorMap *m, const void *base, uint64_t chunks)
{
    PFN_encodeTiled_t enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {64, chunks * 8};
    cuuint64_t strides[1] = {256};
    cuuint32_t box[2] = {64, 8};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// E4M3 codes as a 2-D uint8 tensor, 128-byte (128-element) boxes, 128-byte swizzle.
static bool make_map_u8(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows)
{
    PFN_encodeTiled_t enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols};
    cuuint32_t box[2] = {128, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static int sm_count()
{
    static int n = 0;
    if (!n) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 148;
    }
    return n;
}

template <bool SPARSE>
static cudaError_t launch_gemm_t(const GemmArgs &a, cudaStream_t st)
{
    using C = GemmCfg<SPARSE>;
    CUtensorMap mA, mB, mA2;
    const uint64_t ka = SPARSE ? (uint64_t)a.K / 2 : (uint64_t)a.K;
    if (!make_map(&mA, a.A, (uint64_t)a.T, ka, GEMM_BM)) return cudaErrorInvalidValue;
    if (!make_map(&mB, a.W, (uint64_t)a.n_out, (uint64_t)a.K, C::BN)) return cudaErrorInvalidValue;
    if (!make_map(&mA2, a.A_lo ? a.A_lo : a.A, (uint64_t)a.T, ka, GEMM_BM)) return cudaErrorInvalidValue;
    CUtensorMap mU = mA, mR = mB;
    if (a.r > 0 && (!make_map(&mU, a.U2, (uint64_t)a.u_parts * a.T, (uint64_t)a.r, GEMM_BM) ||
                    !make_map(&mR, a.Ar, (uint64_t)a.n_out, (uint64_t)a.r, C::BN)))
        return cudaErrorInvalidValue;
    GemmParams p{};
    p.meta = a.meta;
    p.rowsum = a.rowsum;
    p.eta = a.eta;
    p.nu = a.nu;
    p.y = a.y;
    p.T = a.T;
    p.K = a.K;
    p.n_out = a.n_out;
    p.out_bf16 = a.out_bf16;
    p.m_tiles = (a.T + GEMM_BM - 1) / GEMM_BM;
    p.n_tiles = (a.n_out + C::BN - 1) / C::BN;
    p.kb_pass = (a.K + C::KB - 1) / C::KB;
    p.kb_main = p.kb_pass * (a.A_lo ? 2 : 1);
    p.rblk = a.r / 64;
    p.k_blocks = p.kb_main + a.u_parts * p.rblk;
    p.meta_kt = (a.K + 127) / 128;
    const size_t smem = gemm_smem_bytes<SPARSE>();
    cudaError_t e = cudaFuncSetAttribute(k_gemm<SPARSE>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int tiles = p.m_tiles * p.n_tiles;
    const int grid = std::min(tiles, sm_count());
    k_gemm<SPARSE><<<grid, GEMM_THREADS, smem, st>>>(mA, mB, mA2, mU, mR, p);
    return cudaGetLastError();
}

// Number of 2-CTA clusters of k_gemm_sp_pair that fit on the device at once
// (0 if the query fails).
template <typename KernelT>
static int pair_clusters_of(KernelT kernel, size_t smem, int &cached)
{
    if (cached >= 0) return cached;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(2 * 74, 1, 1);
    cfg.blockDim = dim3(PAIR_THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess ||
        cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess) {
        cudaGetLastError();
        n = 0;
    }
    cached = n;
    return n;
}

static int pair_clusters(size_t smem)
{
    static int cached = -1;
    return pair_clusters_of(k_gemm_sp_pair<false>, smem, cached);
}

static int pair_clusters_fp8(size_t smem)
{
    static int cached = -1;
    return pair_clusters_of(k_gemm_sp_pair<true>, smem, cached);
}

static int dense_pair_clusters(size_t smem)
{
    static int cached = -1;
    return pair_clusters_of(k_gemm_dense_pair, smem, cached);
}

// The pair kernel needs every CTA's 128-row box to hold at least one real
// row (an even number of 128-row tiles) and a 16-byte-aligned position
// buffer for its tensor map.
static bool use_pair(const GemmArgs &a)
{
    const int mt128 = (a.T + GEMM_BM - 1) / GEMM_BM;
    if ((mt128 % 2) != 0) return false;
    return !a.sparse || (reinterpret_cast<uintptr_t>(a.meta) & 15) == 0;
}

static cudaError_t launch_gemm_pair(const GemmArgs &a, cudaStream_t st)
{
    CUtensorMap mA, mB, mE, mA2;
    const int mt128 = (a.T + GEMM_BM - 1) / GEMM_BM;
    GemmParams p{};
    p.meta = a.meta;
    p.rowsum = a.rowsum;
    p.eta = a.eta;
    p.nu = a.nu;
    p.y = a.y;
    p.T = a.T;
    p.K = a.K;
    p.n_out = a.n_out;
    p.out_bf16 = a.out_bf16;
    p.m_tiles = mt128 / 2;
    p.n_tiles = (a.n_out + PAIR_BN - 1) / PAIR_BN;
    p.kb_pass = (a.K + 127) / 128;
    p.kb_main = p.kb_pass * (a.A_lo ? 2 : 1);
    p.rblk = a.r / 64;
    p.k_blocks = p.kb_main + a.u_parts * p.rblk;
    p.meta_kt = (a.K + 127) / 128;
    if (!make_map(&mA, a.A, (uint64_t)a.T, (uint64_t)a.K / 2, 128)) return cudaErrorInvalidValue;
    if (!make_map(&mA2, a.A_lo ? a.A_lo : a.A, (uint64_t)a.T, (uint64_t)a.K / 2, 128)) return cudaErrorInvalidValue;
    if (!make_map(&mB, a.W, (uint64_t)a.n_out, (uint64_t)a.K, 128)) return cudaErrorInvalidValue;
    if (!make_map_meta(&mE, a.meta, (uint64_t)mt128 * p.meta_kt)) return cudaErrorInvalidValue;
    CUtensorMap mU = mA, mR = mB;
    if (a.r > 0 && (!make_map(&mU, a.U2, (uint64_t)a.u_parts * a.T, (uint64_t)a.r, 128) ||
                    !make_map(&mR, a.Ar, (uint64_t)a.n_out, (uint64_t)a.r, 128)))
        return cudaErrorInvalidValue;
    const size_t smem = pair_smem_bytes<false>();
    cudaError_t e = cudaFuncSetAttribute(k_gemm_sp_pair<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int clusters = pair_clusters(smem);
    if (clusters <= 0) return cudaErrorNotSupported;
    const int tiles = p.m_tiles * p.n_tiles;
    const int grid = 2 * std::min(tiles, clusters);
    k_gemm_sp_pair<false><<<grid, PAIR_THREADS, smem, st>>>(mA, mB, mE, mA2, mU, mR, p);
    return cudaGetLastError();
}

static cudaError_t launch_gemm_dense_pair(const GemmArgs &a, cudaStream_t st)
{
    CUtensorMap mA, mB, mA2;
    const int mt128 = (a.T + GEMM_BM - 1) / GEMM_BM;
    GemmParams p{};
    p.rowsum = a.rowsum;
    p.eta = a.eta;
    p.nu = a.nu;
    p.y = a.y;
    p.T = a.T;
    p.K = a.K;
    p.n_out = a.n_out;
    p.out_bf16 = a.out_bf16;
    p.m_tiles = mt128 / 2;
    p.n_tiles = (a.n_out + PAIR_BN - 1) / PAIR_BN;
    p.kb_pass = (a.K + 63) / 64;
    p.kb_main = p.kb_pass * (a.A_lo ? 2 : 1);
    p.rblk = a.r / 64;
    p.k_blocks = p.kb_main + a.u_parts * p.rblk;
    if (!make_map(&mA, a.A, (uint64_t)a.T, (uint64_t)a.K, 128)) return cudaErrorInvalidValue;
    if (!make_map(&mB, a.W, (uint64_t)a.n_out, (uint64_t)a.K, 128)) return cudaErrorInvalidValue;
    if (!make_map(&mA2, a.A_lo ? a.A_lo : a.A, (uint64_t)a.T, (uint64_t)a.K, 128)) return cudaErrorInvalidValue;
    CUtensorMap mU = mA, mR = mB;
    if (a.r > 0 && (!make_map(&mU, a.U2, (uint64_t)a.u_parts * a.T, (uint64_t)a.r, 128) ||
                    !make_map(&mR, a.Ar, (uint64_t)a.n_out, (uint64_t)a.r, 128)))
        return cudaErrorInvalidValue;
    const size_t smem = dense_pair_smem_bytes();
    const int clusters = dense_pair_clusters(smem);
    if (clusters <= 0) return cudaErrorNotSupported;
    const int tiles = p.m_tiles * p.n_tiles;
    const int grid = 2 * std::min(tiles, clusters);
    k_gemm_dense_pair<<<grid, PAIR_THREADS, smem, st>>>(mA, mB, mA2, mU, mR, p);
    return cudaGetLastError();
}

// FP8 2:4 GEMM on CTA pairs.  The metadata buffer covers an even number of
// 128-row tiles (meta8_words), so an odd tile count runs its last pair with
// a second CTA whose rows all lie past T (zero-filled by TMA, not stored).
cudaError_t launch_gemm_fp8(const Fp8GemmArgs &a, cudaStream_t st)
{
    CUtensorMap mA, mB, mE;
    const int mt128 = (a.T + GEMM_BM - 1) / GEMM_BM;
    GemmParams p{};
    p.xscale = a.x_scale;
    p.wscale = a.w_scale;
    p.y = a.y;
    p.T = a.T;
    p.K = a.K;
    p.n_out = a.n_out;
    p.out_bf16 = a.out_bf16;
    p.m_tiles = (mt128 + 1) / 2;
    p.n_tiles = (a.n_out + PAIR_BN - 1) / PAIR_BN;
    p.k_blocks = (a.K + 255) / 256;
    p.kb_pass = p.k_blocks;
    p.kb_main = p.k_blocks;
    p.rblk = 0;
    p.meta_kt = p.k_blocks;
    if (!make_map_u8(&mA, a.x8, (uint64_t)a.T, (uint64_t)a.K / 2, 128)) return cudaErrorInvalidValue;
    if (!make_map_u8(&mB, a.Wq, (uint64_t)a.n_out, (uint64_t)a.K, 128)) return cudaErrorInvalidValue;
    if (!make_map_meta(&mE, a.meta8, (uint64_t)p.m_tiles * 2 * p.meta_kt * 2)) return cudaErrorInvalidValue;
    const size_t smem = pair_smem_bytes<true>();
    cudaError_t e = cudaFuncSetAttribute(k_gemm_sp_pair<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int clusters = pair_clusters_fp8(smem);
    if (clusters <= 0) return cudaErrorNotSupported;
    const int tiles = p.m_tiles * p.n_tiles;
    const int grid = 2 * std::min(tiles, clusters);
    k_gemm_sp_pair<true><<<grid, PAIR_THREADS, smem, st>>>(mA, mB, mE, mA, mA, mB, p);
    return cudaGetLastError();
}

cudaError_t launch_gemm(const GemmArgs &a, cudaStream_t st)
{
    if (use_pair(a)) {
        if (a.sparse) {
            const size_t smem = pair_smem_bytes<false>();
            if (cudaFuncSetAttribute(k_gemm_sp_pair<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) ==
                    cudaSuccess &&
                pair_clusters(smem) > 0)
                return launch_gemm_pair(a, st);
        } else if (dense_pair_clusters(dense_pair_smem_bytes()) > 0) {
            return launch_gemm_dense_pair(a, st);
        }
        cudaGetLastError();
    }
    return a.sparse ? launch_gemm_t<true>(a, st) : launch_gemm_t<false>(a, st);
}

}  // namespace as
