// Host-side launchers of the kernels (internal to libactsparse).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace as {

// ------------------------------------------------------------ weight prep
size_t weight_prep_workspace(int n_out, int k);
cudaError_t launch_weight_prep(const void *W, int bf16, int n_out, int k, float alpha, void *Wt, float *g,
                               float *rowsum, void *ws, cudaStream_t st);
// Amber-Pruner importance: ranks of the two percentile weights (ascending).
size_t amber_workspace(int n_out, int k);
cudaError_t launch_amber(const void *W, int bf16, int n_out, int k, float alpha, uint32_t rank_lo, uint32_t rank_hi,
                         float *g, float *bounds, void *ws, cudaStream_t st);

// ------------------------------------------------------------ select
struct SelectArgs {
    const void *x;
    int bf16;
    int T, K;
    int score, sel, n, m, k_keep, dpts, var, first;
    float mom, eps;
    float tau;                 // AS_SEL_THRESH
    const float *eta_static;   // S-PTS table [T], or nullptr
    const float *f;  // channel factor (g or c) or nullptr
    float *running_var;
    uint32_t *bitmask;
    float *eta, *var_dense, *var_kept, *nu;
    void *x_masked;
    void *x_compact;
    uint32_t *meta24;
    void *x_masked_lo;   // bf16 residuals of x_masked (float32-output GEMM operand), or nullptr
    void *x_compact_lo;  // bf16 residuals of x_compact, or nullptr
    uint32_t *bitmask24; // N:M selection: kept channels of its 2:4 part (x_compact/meta24 hold the part)
};
// CLACT column energy c_j = sqrt(sum_t x_tj^2), float64 partials in ws.
size_t colnorm_workspace(int T, int K);
cudaError_t launch_colnorm(const void *x, int bf16, int T, int K, float *c, void *ws, cudaStream_t st);
cudaError_t launch_select(const SelectArgs &a, cudaStream_t st, int wide = 0);
// Whether launch_select (not wide) runs the row kernel for these arguments.
bool select_rows_kernel(const SelectArgs &a);
// N:M selection of a decode call: keep words and eta only (grid token x chunk).
cudaError_t launch_select_nm_decode(const SelectArgs &a, cudaStream_t st);
// Kept count and natural nonzeros dropped per token (as_select_stats).
cudaError_t launch_select_stats(const void *x, int bf16, const uint32_t *bitmask, int T, int K, int32_t *kept,
                                int32_t *nz_dropped, cudaStream_t st);

// ------------------------------------------------------------ decode
struct DecodeArgs {
    const void *x;
    const void *Wt;
    int bf16;
    int T, K, n_out;
    int score, sel, n, m, k_keep, dpts;
    float tau;                 // AS_SEL_THRESH
    const float *eta_static;   // S-PTS table [T], or nullptr
    const float *g;
    const float *rowsum;
    const uint32_t *mask_in;  // precomputed selection (top-k / all), or nullptr for fused N:M
    void *y;
    int out_bf16;
    uint32_t *mask_out;
    float *eta_out;
    float *colnorm_out;
    float *partial;     // split-K partial sums
    unsigned *counters; // one per N-slice, zero between calls
    float *eta_in;      // D-PTS means written by the select kernel (bf16 path)
};
struct DecodePlan {
    int n_slices, k_splits, words_per_split, tpad, tc;
    size_t partial_bytes, counter_bytes, eta_bytes, smem_bytes;
};
DecodePlan decode_plan(int T, int K, int n_out, int bf16);
// Whether a decode call runs a separate selection kernel first.
bool decode_needs_select(int T, int K, int n_out, int bf16, int out_bf16, int sel);
int decode_launch_count(const DecodeArgs &a, const DecodePlan &p);
// True when a bf16 decode of this token pad and selection is one fused launch.
bool decode_fused(int tpad, int sel, int K);
cudaError_t launch_decode(const DecodeArgs &a, const DecodePlan &p, cudaStream_t st);

// ------------------------------------------------------------ prefill GEMM
struct GemmArgs {
    const void *A;        // bf16 [T, Ka] K-major (x_masked, x or x_compact)
    const void *A_lo = nullptr;  // bf16 residual of A (same layout): a second pass over K adds A_lo W^T
    const uint32_t *meta; // 2:4 metadata (sparse only)
    const void *W;        // bf16 [n_out, K] K-major
    int T, K, n_out;
    int sparse;
    const float *rowsum, *eta, *nu;  // epilogue terms (optional)
    void *y;
    int out_bf16;
    // Extra dense K blocks after the main ones: U2 bf16 [u_parts T, r] against
    // Ar bf16 [n_out, r], u_parts r/64 blocks of 64 into the same accumulator.
    // R-Sparse: u_parts 2 (U hi rows, then U lo rows), Ar = A_r.  Hybrid
    // split: u_parts 1, the gathered remainder of the dense blocks against
    // their W columns.
    const void *U2 = nullptr;
    const void *Ar = nullptr;
    int r = 0;
    int u_parts = 2;
};
// R-Sparse prefill U = (xhat (.) (1 - m)) B_r (rsparse_prefill.cu)
struct RspLayout {
    int splits, blocks_per_split;
    size_t part, u, bytes;
};
RspLayout rsp_layout(int T, int K, int r);
cudaError_t launch_rsp_u(const void *x, const uint32_t *mask, const float *eta, const void *B, int T, int K, int r,
                         void *ws, cudaStream_t st);
cudaError_t launch_gemm(const GemmArgs &a, cudaStream_t st);

// FP8 2:4 prefill (fp8.cu, gemm.cu).
struct Fp8GemmArgs {
    const uint8_t *x8;       // E4M3 codes of the kept values [T, K/2]
    const uint32_t *meta8;   // positions, meta8_words(T, K) words
    const float *x_scale;    // [T]
    const uint8_t *Wq;       // E4M3 [n_out, K]
    const float *w_scale;    // [n_out]
    int T, K, n_out;
    void *y;
    int out_bf16;
};
cudaError_t launch_gemm_fp8(const Fp8GemmArgs &a, cudaStream_t st);

// R-Sparse decode compensation (rsparse.cu).
struct RsparseArgs {
    const void *x;          // [T, K] in the call's dtype
    int bf16;
    const uint32_t *mask;   // [T, ceil(K/32)], bit set = kept
    const float *eta;       // [T] or NULL
    const void *B, *A;      // bf16 [K, r], [n_out, r]
    int T, K, n_out, r;
    float *y;               // [T, n_out], in/out
    void *workspace;
};
// Hybrid 2:4 prefill (hybrid.cu).
struct HybridArgs {
    const void *x;            // bf16 [T, K]
    const uint32_t *bitmask;  // 2:4 selection of x, [T, ceil(K/32)]
    const void *x_compact;    // its kept values
    const uint32_t *meta24;   // and positions
    const void *W;            // bf16 [n_out, K]
    int T, K, n_out, n_dense;
    void *y;
    int out_bf16;
    int *idx_out;             // [n_dense] or NULL
    float *sparsity_out;      // [1] or NULL
    void *workspace;
    const float *rowsum = nullptr, *eta = nullptr, *nu = nullptr;  // epilogue terms of the 2:4 GEMM
};
struct HybridLayout {
    size_t nnz, total, idx, xr, wd, bytes;
};
HybridLayout hybrid_layout(int T, int K, int n_out, int n_dense);
cudaError_t launch_block_sparsity(const void *x, int T, int K, int n_dense, int *idx, float *sparsity, void *ws,
                                  cudaStream_t st);
cudaError_t launch_hybrid(const HybridArgs &a, cudaStream_t st);
size_t rsparse_workspace(int T, int K, int r);
cudaError_t launch_rsparse(const RsparseArgs &a, cudaStream_t st);
int meta8_kt(int K);
size_t meta8_words(int T, int K);
cudaError_t launch_sqrelu24_fp8(const void *z, int T, int K, uint8_t *x8, uint32_t *meta8, float *x_scale,
                                uint32_t *bitmask, cudaStream_t st);
cudaError_t launch_quant_rows_fp8(const void *W, int bf16, int n_out, int K, uint8_t *Wq, float *w_scale,
                                  cudaStream_t st);

}  // namespace as
