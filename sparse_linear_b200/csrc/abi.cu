// extern "C" entry points of libactsparse (declared in include/actsparse.h).
//
// Every entry point validates its arguments on the host and launches nothing
// when they are invalid; CUDA launch errors are mapped to AS_ERR_CUDA.  No
// entry point allocates device memory: scratch space is the caller's
// workspace, sized by as_workspace_size().
#include <string.h>

#include "common.cuh"
#include "kernels.cuh"

using namespace as;

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

bool valid_m(int m) { return m == 1 || m == 2 || m == 4 || m == 8 || m == 16 || m == 32; }

as_status check_cfg(const as_config *cfg, int K)
{
    if (!cfg) return AS_ERR_INVALID_ARG;
    if (cfg->score < AS_SCORE_MAG || cfg->score > AS_SCORE_CLACT) return AS_ERR_INVALID_ARG;
    if (cfg->sel < AS_SEL_NM || cfg->sel > AS_SEL_THRESH) return AS_ERR_INVALID_ARG;
    if (cfg->dpts < AS_PTS_OFF || cfg->dpts > AS_PTS_STATIC) return AS_ERR_INVALID_ARG;
    if (cfg->dpts == AS_PTS_STATIC && (!cfg->eta_static || !aligned16(cfg->eta_static))) return AS_ERR_INVALID_ARG;
    if (cfg->sel == AS_SEL_THRESH && !(cfg->tau == cfg->tau)) return AS_ERR_INVALID_ARG;  // NaN
    if (cfg->out_dtype != AS_F32 && cfg->out_dtype != AS_BF16) return AS_ERR_DTYPE;
    if (cfg->sel == AS_SEL_NM) {
        if (!valid_m(cfg->m)) return AS_ERR_SHAPE;
        if (cfg->n < 1 || cfg->n > cfg->m) return AS_ERR_SHAPE;
        if (K % cfg->m != 0) return AS_ERR_SHAPE;
    }
    if (cfg->sel == AS_SEL_TOPK && (cfg->k_keep < 0 || cfg->k_keep > K)) return AS_ERR_SHAPE;
    if (cfg->dpts && cfg->var) return AS_ERR_UNSUPPORTED;
    if (cfg->var && !(cfg->var_eps >= 0.0f && cfg->var_momentum >= 0.0f && cfg->var_momentum <= 1.0f))
        return AS_ERR_INVALID_ARG;
    return AS_OK;
}

bool is24(const as_config *cfg) { return cfg->sel == AS_SEL_NM && cfg->n == 2 && cfg->m == 4; }

as_status cuda_status(cudaError_t e) { return e == cudaSuccess ? AS_OK : AS_ERR_CUDA; }

size_t decode_ws(int T, int K, int n_out, const as_config *cfg, int bf16)
{
    DecodePlan p = decode_plan(T, K, n_out, bf16);
    size_t bytes = round_up(p.counter_bytes, 256) + round_up(p.partial_bytes, 256) + round_up(p.eta_bytes, 256);
    // a separate selection kernel (top-k; the non-cluster bf16 path beyond 2 tokens; keep-all)
    const bool sel_kernel = decode_needs_select(T, K, n_out, bf16, cfg->out_dtype == AS_BF16, cfg->sel);
    if (sel_kernel) bytes += round_up((size_t)T * ((K + 31) / 32) * sizeof(uint32_t), 256);
    if (sel_kernel && cfg->score == AS_SCORE_CLACT) bytes += round_up(colnorm_workspace(T, K), 256);
    return bytes;
}

size_t select_ws(int T, int K, const as_config *cfg)
{
    return cfg->score == AS_SCORE_CLACT ? round_up(colnorm_workspace(T, K), 256) : 0;
}

}  // namespace

extern "C" {

int as_abi_version(void) { return AS_ABI_VERSION; }

const char *as_status_string(as_status s)
{
    switch (s) {
    case AS_OK: return "AS_OK";
    case AS_ERR_INVALID_ARG: return "AS_ERR_INVALID_ARG: missing buffer or bad enum";
    case AS_ERR_SHAPE: return "AS_ERR_SHAPE: shape not supported (K % M, N > M, k_keep, T range)";
    case AS_ERR_DTYPE: return "AS_ERR_DTYPE: dtype not supported by this operation";
    case AS_ERR_ALIGN: return "AS_ERR_ALIGN: pointer or row stride not 16-byte aligned";
    case AS_ERR_UNSUPPORTED: return "AS_ERR_UNSUPPORTED: combination not supported";
    case AS_ERR_WORKSPACE: return "AS_ERR_WORKSPACE: workspace missing or too small";
    case AS_ERR_CUDA: return "AS_ERR_CUDA: a CUDA call failed";
    case AS_ERR_TIMEOUT: return "AS_ERR_TIMEOUT: a device-side bounded wait gave up";
    case AS_ERR_BOUNDS: return "AS_ERR_BOUNDS: a checked build found an index outside its buffer";
    }
    return "unknown as_status";
}

size_t as_meta24_words(int T, int K)
{
    if (T <= 0 || K <= 0) return 0;
    return (size_t)((T + 127) / 128) * (size_t)((K + 127) / 128) * 512;
}

size_t as_workspace_size(int op, int T, int K, int n_out, const as_config *cfg)
{
    if (K <= 0) return (size_t)-1;
    switch (op) {
    case AS_OP_WEIGHT_PREP:
        if (n_out <= 0) return (size_t)-1;
        return weight_prep_workspace(n_out, K);
    case AS_OP_SELECT:
        if (T <= 0 || check_cfg(cfg, K) != AS_OK) return (size_t)-1;
        return select_ws(T, K, cfg);
    case AS_OP_DECODE:
        if (T < 1 || T > AS_MAX_DECODE_T || n_out <= 0 || check_cfg(cfg, K) != AS_OK) return (size_t)-1;
        return decode_ws(T, K, n_out, cfg, 1) > decode_ws(T, K, n_out, cfg, 0) ? decode_ws(T, K, n_out, cfg, 1)
                                                                                : decode_ws(T, K, n_out, cfg, 0);
    case AS_OP_PREFILL:
        if (T <= 0 || n_out <= 0 || check_cfg(cfg, K) != AS_OK) return (size_t)-1;
        return 0;
    case AS_OP_AMBER:
        if (n_out <= 0) return (size_t)-1;
        return amber_workspace(n_out, K);
    }
    return (size_t)-1;
}

as_status as_weight_prep(const void *W, as_dtype dt, int n_out, int K, float alpha, void *Wt, float *g,
                         float *rowsum, void *workspace, size_t ws_bytes, cudaStream_t stream)
{
    if (!W || n_out <= 0 || K <= 0) return AS_ERR_INVALID_ARG;
    if (dt != AS_F32 && dt != AS_BF16) return AS_ERR_DTYPE;
    if (!aligned16(W) || !aligned16(Wt) || !aligned16(g) || !aligned16(rowsum)) return AS_ERR_ALIGN;
    if (g) {
        if (!workspace || ws_bytes < weight_prep_workspace(n_out, K)) return AS_ERR_WORKSPACE;
        if (!aligned16(workspace)) return AS_ERR_ALIGN;
    }
    return cuda_status(launch_weight_prep(W, dt == AS_BF16, n_out, K, alpha, Wt, g, rowsum, workspace, stream));
}

as_status as_weight_prep_amber(const void *W, as_dtype dt, int n_out, int K, float alpha, double lo_pct,
                               double hi_pct, float *g, float *bounds, void *workspace, size_t ws_bytes,
                               cudaStream_t stream)
{
    if (!W || !g || n_out <= 0 || K <= 0) return AS_ERR_INVALID_ARG;
    if (!(lo_pct >= 0.0 && lo_pct <= hi_pct && hi_pct <= 100.0)) return AS_ERR_INVALID_ARG;
    if (dt != AS_F32 && dt != AS_BF16) return AS_ERR_DTYPE;
    const uint64_t N = (uint64_t)n_out * (uint64_t)K;
    if (N >= (1ull << 32)) return AS_ERR_SHAPE;
    if (!aligned16(W) || !aligned16(g) || !aligned16(bounds)) return AS_ERR_ALIGN;
    if (!workspace || ws_bytes < amber_workspace(n_out, K)) return AS_ERR_WORKSPACE;
    if (!aligned16(workspace)) return AS_ERR_ALIGN;
    // Ascending ranks of the two percentile values among the N weights.
    const uint32_t r_lo = (uint32_t)floor(lo_pct / 100.0 * (double)(N - 1));
    const uint32_t r_hi = (uint32_t)floor(hi_pct / 100.0 * (double)(N - 1));
    return cuda_status(launch_amber(W, dt == AS_BF16, n_out, K, alpha, r_lo, r_hi, g, bounds, workspace, stream));
}

static as_status hybrid_shape(int T, int K, int n_out, int n_dense)
{
    if (T <= 0 || K <= 0 || n_out < 0) return AS_ERR_INVALID_ARG;
    if (K % 64 != 0 || K > 32768 || n_out % 8 != 0) return AS_ERR_SHAPE;
    if (T >= (1 << 22)) return AS_ERR_SHAPE;  // a block's count (<= 4 T) must stay below 2^24
    if (n_dense < 0 || n_dense > K / 4 || n_dense % 16 != 0) return AS_ERR_SHAPE;
    return AS_OK;
}

size_t as_hybrid_workspace(int T, int K, int n_out, int n_dense)
{
    if (hybrid_shape(T, K, n_out, n_dense) != AS_OK) return (size_t)-1;
    return hybrid_layout(T, K, n_out, n_dense).bytes;
}

as_status as_block_sparsity(const void *x, int T, int K, int n_dense, int32_t *dense_idx, float *sparsity,
                            void *workspace, size_t ws_bytes, cudaStream_t stream)
{
    if (!x || !sparsity || (n_dense > 0 && !dense_idx)) return AS_ERR_INVALID_ARG;
    as_status st = hybrid_shape(T, K, 0, n_dense);
    if (st != AS_OK) return st;
    if (!aligned16(x) || !aligned16(workspace)) return AS_ERR_ALIGN;
    if (!workspace || ws_bytes < hybrid_layout(T, K, 0, 0).bytes) return AS_ERR_WORKSPACE;
    return cuda_status(launch_block_sparsity(x, T, K, n_dense, dense_idx, sparsity, workspace, stream));
}

as_status as_select_stats(const void *x, as_dtype dt, const uint32_t *bitmask, int T, int K, int32_t *kept,
                          int32_t *nz_dropped, cudaStream_t stream)
{
    if (!x || !bitmask) return AS_ERR_INVALID_ARG;
    if (dt != AS_F32 && dt != AS_BF16) return AS_ERR_DTYPE;
    if (T <= 0 || K <= 0 || K % 8 != 0) return AS_ERR_SHAPE;
    for (const void *q : {x, (const void *)bitmask, (const void *)kept, (const void *)nz_dropped})
        if (!aligned16(q)) return AS_ERR_ALIGN;
    if (!kept && !nz_dropped) return AS_OK;
    return cuda_status(launch_select_stats(x, dt == AS_BF16, bitmask, T, K, kept, nz_dropped, stream));
}

as_status as_linear_prefill_hybrid(const as_select_out *sel, const void *x, int T, int K, const void *W, int n_out,
                                   int n_dense, as_dtype out_dtype, void *y, int32_t *dense_idx, float *sparsity,
                                   void *workspace, size_t ws_bytes, cudaStream_t stream)
{
    if (!sel || !x || !W || !y || !sel->bitmask || !sel->x_compact || !sel->meta24) return AS_ERR_INVALID_ARG;
    if (n_out <= 0) return AS_ERR_INVALID_ARG;
    as_status st = hybrid_shape(T, K, n_out, n_dense);
    if (st != AS_OK) return st;
    if (out_dtype != AS_F32 && out_dtype != AS_BF16) return AS_ERR_DTYPE;
    for (const void *q : {x, W, (const void *)y, (const void *)sel->bitmask, (const void *)sel->x_compact,
                          (const void *)sel->meta24, (const void *)workspace})
        if (!aligned16(q)) return AS_ERR_ALIGN;
    if (!workspace || ws_bytes < hybrid_layout(T, K, n_out, n_dense).bytes) return AS_ERR_WORKSPACE;
    HybridArgs a{};
    a.x = x;
    a.bitmask = sel->bitmask;
    a.x_compact = sel->x_compact;
    a.meta24 = sel->meta24;
    a.W = W;
    a.T = T;
    a.K = K;
    a.n_out = n_out;
    a.n_dense = n_dense;
    a.y = y;
    a.out_bf16 = out_dtype == AS_BF16;
    a.idx_out = dense_idx;
    a.sparsity_out = sparsity;
    a.workspace = workspace;
    return cuda_status(launch_hybrid(a, stream));
}

int as_prefill_mode(double sparsity)
{
    if (sparsity > 0.95) return AS_MODE_24;
    if (sparsity >= 0.90) return AS_MODE_SPLIT;
    return AS_MODE_DENSE;  // also NaN
}

int as_hybrid_dense_blocks(int K, double dense_frac)
{
    if (K <= 0 || K % 64 != 0 || !(dense_frac >= 0.0 && dense_frac <= 1.0)) return -1;
    const int nb = K / 4;
    const int n = (int)ceil(dense_frac * (double)nb / 16.0) * 16;
    const int hi = nb / 16 * 16;
    return n < 16 ? 16 : (n > hi ? hi : n);
}

as_status as_linear_prefill_nm_split(const as_select_out *sel, int T, int K, const void *W, int n_out, int n_dense,
                                     const as_config *cfg, const float *rowsum, const float *eta, const float *nu,
                                     void *y, int32_t *dense_idx, float *sparsity, void *workspace, size_t ws_bytes,
                                     cudaStream_t stream)
{
    if (!sel || !W || !y || !sel->x_masked || !sel->x_compact || !sel->meta24 || !sel->bitmask24)
        return AS_ERR_INVALID_ARG;
    if (n_out <= 0) return AS_ERR_INVALID_ARG;
    as_status st = check_cfg(cfg, K);
    if (st != AS_OK) return st;
    if (cfg->sel != AS_SEL_NM || cfg->m < 8 || cfg->m % 4 != 0) return AS_ERR_UNSUPPORTED;
    st = hybrid_shape(T, K, n_out, n_dense);
    if (st != AS_OK) return st;
    if (cfg->dpts && (!rowsum || !eta)) return AS_ERR_INVALID_ARG;
    if (cfg->var && !nu) return AS_ERR_INVALID_ARG;
    const void *ptrs[] = {W, y, sel->x_masked, sel->x_compact, sel->meta24, sel->bitmask24, workspace, rowsum,
                          eta, nu};
    for (const void *q : ptrs)
        if (!aligned16(q)) return AS_ERR_ALIGN;
    if (!workspace || ws_bytes < hybrid_layout(T, K, n_out, n_dense).bytes) return AS_ERR_WORKSPACE;
    HybridArgs a{};
    a.x = sel->x_masked;  // the masked activation: its nonzeros pick D, its overflow is the dense remainder
    a.bitmask = sel->bitmask24;
    a.x_compact = sel->x_compact;
    a.meta24 = sel->meta24;
    a.W = W;
    a.T = T;
    a.K = K;
    a.n_out = n_out;
    a.n_dense = n_dense;
    a.y = y;
    a.out_bf16 = cfg->out_dtype == AS_BF16;
    a.idx_out = dense_idx;
    a.sparsity_out = sparsity;
    a.workspace = workspace;
    a.rowsum = cfg->dpts ? rowsum : nullptr;
    a.eta = cfg->dpts ? eta : nullptr;
    a.nu = cfg->var ? nu : nullptr;
    return cuda_status(launch_hybrid(a, stream));
}

static bool rsparse_rank_ok(int r) { return r == 32 || r == 64 || r == 128; }

size_t as_rsparse_workspace(int T, int K, int r)
{
    if (T < 1 || T > AS_MAX_DECODE_T || K <= 0 || !rsparse_rank_ok(r)) return (size_t)-1;
    return rsparse_workspace(T, K, r);
}

as_status as_rsparse_decode(const void *x, as_dtype dt, int T, int K, int n_out, int r, const uint32_t *mask,
                            const float *eta, const void *B, const void *A, float *y, void *workspace,
                            size_t ws_bytes, cudaStream_t stream)
{
    if (!x || !mask || !B || !A || !y || K <= 0 || n_out <= 0) return AS_ERR_INVALID_ARG;
    if (dt != AS_F32 && dt != AS_BF16) return AS_ERR_DTYPE;
    if (T < 1 || T > AS_MAX_DECODE_T || !rsparse_rank_ok(r)) return AS_ERR_SHAPE;
    if (!aligned16(A) || !aligned16(B) || !aligned16(workspace)) return AS_ERR_ALIGN;
    if (!workspace || ws_bytes < rsparse_workspace(T, K, r)) return AS_ERR_WORKSPACE;
    RsparseArgs a{};
    a.x = x;
    a.bf16 = dt == AS_BF16;
    a.mask = mask;
    a.eta = eta;
    a.B = B;
    a.A = A;
    a.T = T;
    a.K = K;
    a.n_out = n_out;
    a.r = r;
    a.y = y;
    a.workspace = workspace;
    return cuda_status(launch_rsparse(a, stream));
}

size_t as_meta8_words(int T, int K)
{
    if (T <= 0 || K <= 0) return 0;
    return meta8_words(T, K);
}

as_status as_weight_quant_fp8(const void *W, as_dtype dt, int n_out, int K, uint8_t *Wq, float *w_scale,
                              cudaStream_t stream)
{
    if (!W || !Wq || !w_scale || n_out <= 0 || K <= 0) return AS_ERR_INVALID_ARG;
    if (dt != AS_F32 && dt != AS_BF16) return AS_ERR_DTYPE;
    if (K % 16 != 0) return AS_ERR_SHAPE;
    if (!aligned16(W) || !aligned16(Wq) || !aligned16(w_scale)) return AS_ERR_ALIGN;
    return cuda_status(launch_quant_rows_fp8(W, dt == AS_BF16, n_out, K, Wq, w_scale, stream));
}

as_status as_select_sqrelu24_fp8(const void *z, int T, int K, uint8_t *x8, uint32_t *meta8, float *x_scale,
                                 uint32_t *bitmask, cudaStream_t stream)
{
    if (!z || !x8 || !meta8 || !x_scale || T <= 0 || K <= 0) return AS_ERR_INVALID_ARG;
    if (K % 64 != 0) return AS_ERR_SHAPE;
    if (!aligned16(z) || !aligned16(x8) || !aligned16(meta8) || !aligned16(x_scale) || !aligned16(bitmask))
        return AS_ERR_ALIGN;
    return cuda_status(launch_sqrelu24_fp8(z, T, K, x8, meta8, x_scale, bitmask, stream));
}

as_status as_linear_prefill_fp8(const uint8_t *x8, const uint32_t *meta8, const float *x_scale, int T, int K,
                                int n_out, const uint8_t *Wq, const float *w_scale, as_dtype out_dtype, void *y,
                                cudaStream_t stream)
{
    if (!x8 || !meta8 || !x_scale || !Wq || !w_scale || !y || T <= 0 || K <= 0 || n_out <= 0)
        return AS_ERR_INVALID_ARG;
    if (out_dtype != AS_F32 && out_dtype != AS_BF16) return AS_ERR_DTYPE;
    if (K % 64 != 0 || n_out % 8 != 0) return AS_ERR_SHAPE;
    for (const void *q : {(const void *)x8, (const void *)meta8, (const void *)x_scale, (const void *)Wq,
                          (const void *)w_scale, (const void *)y})
        if (!aligned16(q)) return AS_ERR_ALIGN;
    Fp8GemmArgs a{};
    a.x8 = x8;
    a.meta8 = meta8;
    a.x_scale = x_scale;
    a.Wq = Wq;
    a.w_scale = w_scale;
    a.T = T;
    a.K = K;
    a.n_out = n_out;
    a.y = y;
    a.out_bf16 = out_dtype == AS_BF16;
    const cudaError_t e = launch_gemm_fp8(a, stream);
    return e == cudaErrorNotSupported ? AS_ERR_UNSUPPORTED : cuda_status(e);
}

as_status as_select(const void *x, as_dtype dt, int T, int K, const as_config *cfg, const float *chan_factor,
                    float *running_var, int var_first_batch, const as_select_out *out, void *workspace,
                    size_t ws_bytes, cudaStream_t stream)
{
    if (!x || !out || T <= 0 || K <= 0) return AS_ERR_INVALID_ARG;
    if (dt != AS_F32 && dt != AS_BF16) return AS_ERR_DTYPE;
    as_status st = check_cfg(cfg, K);
    if (st != AS_OK) return st;
    if (K % 8 != 0) return AS_ERR_SHAPE;
    if (cfg->score == AS_SCORE_WEIGHT && !chan_factor) return AS_ERR_INVALID_ARG;
    if (cfg->var && !running_var) return AS_ERR_INVALID_ARG;
    // the 2:4 part of an N:M selection (bitmask24 with x_compact, meta24 and x_masked)
    const bool part24 = out->bitmask24 != nullptr;
    if (part24) {
        if (cfg->sel != AS_SEL_NM || cfg->m < 8 || cfg->m % 4 != 0) return AS_ERR_UNSUPPORTED;
        if (!out->x_compact || !out->meta24 || !out->x_masked) return AS_ERR_INVALID_ARG;
    }
    if ((out->x_compact || out->meta24) && ((!is24(cfg) && !part24) || dt != AS_BF16 || K % 16 != 0))
        return AS_ERR_UNSUPPORTED;
    if ((out->x_compact == nullptr) != (out->meta24 == nullptr)) return AS_ERR_INVALID_ARG;
    if ((out->x_masked_lo && (!out->x_masked || dt != AS_BF16)) || (out->x_compact_lo && !out->x_compact))
        return AS_ERR_INVALID_ARG;
    const void *ptrs[] = {x, chan_factor, running_var, out->bitmask, out->eta, out->colnorm, out->var_dense,
                          out->var_kept, out->nu, out->x_masked, out->x_compact, out->meta24, workspace,
                          out->x_masked_lo, out->x_compact_lo, out->bitmask24};
    for (const void *p : ptrs)
        if (!aligned16(p)) return AS_ERR_ALIGN;
    if (cfg->sel == AS_SEL_TOPK && cfg->k_keep > 0 && cfg->k_keep < K && (size_t)K * 4 > 200 * 1024)
        return AS_ERR_SHAPE;  // top-k keeps the row's scores in shared memory
    const size_t need = select_ws(T, K, cfg);
    if (need && (!workspace || ws_bytes < need)) return AS_ERR_WORKSPACE;

    const float *f = cfg->score == AS_SCORE_WEIGHT ? chan_factor : nullptr;
    if (cfg->score == AS_SCORE_CLACT) {
        float *c = out->colnorm;
        if (!c) c = reinterpret_cast<float *>(static_cast<char *>(workspace) + colnorm_workspace(T, K) -
                                              (size_t)K * sizeof(float));
        cudaError_t e = launch_colnorm(x, dt == AS_BF16, T, K, c, workspace, stream);
        if (e != cudaSuccess) return AS_ERR_CUDA;
        f = c;
    }
    SelectArgs a{};
    a.x = x;
    a.bf16 = dt == AS_BF16;
    a.T = T;
    a.K = K;
    a.score = cfg->score;
    a.sel = cfg->sel;
    a.n = cfg->n;
    a.m = cfg->m;
    a.k_keep = cfg->k_keep;
    a.dpts = cfg->dpts;
    a.tau = cfg->tau;
    a.eta_static = cfg->dpts == AS_PTS_STATIC ? cfg->eta_static : nullptr;
    a.var = cfg->var;
    a.first = var_first_batch;
    a.mom = cfg->var_momentum;
    a.eps = cfg->var_eps;
    a.f = f;
    a.running_var = running_var;
    a.bitmask = out->bitmask;
    a.eta = out->eta;
    a.var_dense = out->var_dense;
    a.var_kept = out->var_kept;
    a.nu = out->nu;
    a.x_masked = out->x_masked;
    a.x_compact = out->x_compact;
    a.meta24 = out->meta24;
    a.x_masked_lo = out->x_masked_lo;
    a.x_compact_lo = out->x_compact_lo;
    a.bitmask24 = out->bitmask24;
    if (part24 && !select_rows_kernel(a)) return AS_ERR_UNSUPPORTED;  // written by the row kernel only
    return cuda_status(launch_select(a, stream));
}

}  // extern "C"

// Every check of a decode call except the workspace's (shared with the
// entry point that takes no workspace, which must refuse a bad call before
// it touches its scratch).
as_status decode_check_args(const void *x, as_dtype dt, int T, int K, int n_out, const void *Wt, const float *g,
                            const float *rowsum, const as_config *cfg, const void *y, const uint32_t *mask_out,
                            const float *eta_out, const float *colnorm_out)
{
    if (!x || !Wt || !y) return AS_ERR_INVALID_ARG;
    if (dt != AS_F32 && dt != AS_BF16) return AS_ERR_DTYPE;
    if (T < 1 || T > AS_MAX_DECODE_T || K <= 0 || n_out <= 0) return AS_ERR_SHAPE;
    as_status st = check_cfg(cfg, K);
    if (st != AS_OK) return st;
    if (cfg->var) return AS_ERR_UNSUPPORTED;
    if (K % 8 != 0 || n_out % 8 != 0) return AS_ERR_SHAPE;
    if (cfg->score == AS_SCORE_WEIGHT && !g) return AS_ERR_INVALID_ARG;
    if (cfg->dpts && !rowsum) return AS_ERR_INVALID_ARG;
    if (cfg->sel == AS_SEL_TOPK && (size_t)K * 4 > 200 * 1024 && cfg->k_keep > 0 && cfg->k_keep < K)
        return AS_ERR_SHAPE;  // top-k keeps the row's scores in shared memory
    const void *ptrs[] = {x, Wt, g, rowsum, y, mask_out, eta_out, colnorm_out};
    for (const void *p : ptrs)
        if (!aligned16(p)) return AS_ERR_ALIGN;
    return AS_OK;
}

extern "C" {

as_status as_linear_decode(const void *x, as_dtype dt, int T, int K, int n_out, const void *Wt, const float *g,
                           const float *rowsum, const as_config *cfg, void *y, uint32_t *mask_out, float *eta_out,
                           float *colnorm_out, void *workspace, size_t ws_bytes, cudaStream_t stream)
{
    as_status st = decode_check_args(x, dt, T, K, n_out, Wt, g, rowsum, cfg, y, mask_out, eta_out, colnorm_out);
    if (st != AS_OK) return st;
    if (!aligned16(workspace)) return AS_ERR_ALIGN;
    const int bf16 = dt == AS_BF16;
    const size_t need = decode_ws(T, K, n_out, cfg, bf16);
    if (!workspace || ws_bytes < need) return AS_ERR_WORKSPACE;

    DecodePlan plan = decode_plan(T, K, n_out, bf16);
    char *ws = static_cast<char *>(workspace);
    unsigned *counters = reinterpret_cast<unsigned *>(ws);
    ws += round_up(plan.counter_bytes, 256);
    float *partial = reinterpret_cast<float *>(ws);
    ws += round_up(plan.partial_bytes, 256);
    float *eta_ws = reinterpret_cast<float *>(ws);
    ws += round_up(plan.eta_bytes, 256);

    const uint32_t *mask_in = nullptr;
    if (decode_needs_select(T, K, n_out, bf16, cfg->out_dtype == AS_BF16, cfg->sel)) {
        // per-token selection kernel first (bf16: always; float32: top-k needs the whole row)
        uint32_t *bm = reinterpret_cast<uint32_t *>(ws);
        ws += round_up((size_t)T * ((K + 31) / 32) * sizeof(uint32_t), 256);
        const float *f = cfg->score == AS_SCORE_WEIGHT ? g : nullptr;
        if (cfg->score == AS_SCORE_CLACT) {
            float *c = colnorm_out;
            if (!c) c = reinterpret_cast<float *>(ws + colnorm_workspace(T, K) - (size_t)K * sizeof(float));
            if (launch_colnorm(x, bf16, T, K, c, ws, stream) != cudaSuccess) return AS_ERR_CUDA;
            f = c;
        }
        SelectArgs s{};
        s.x = x;
        s.bf16 = bf16;
        s.T = T;
        s.K = K;
        s.score = cfg->score;
        s.sel = cfg->sel;
        s.n = cfg->n;
        s.m = cfg->m;
        s.k_keep = cfg->k_keep;
        s.dpts = cfg->dpts;
        s.tau = cfg->tau;
        s.eta_static = cfg->dpts == AS_PTS_STATIC ? cfg->eta_static : nullptr;
        s.f = f;
        s.bitmask = bm;
        s.eta = cfg->dpts ? eta_ws : nullptr;  // the decode kernel reuses the means the selection used
        const cudaError_t se = (cfg->sel == AS_SEL_NM) ? launch_select_nm_decode(s, stream)
                                                       : launch_select(s, stream, /*wide=*/1);
        if (se != cudaSuccess) return AS_ERR_CUDA;
        mask_in = bm;
    }
    DecodeArgs a{};
    a.x = x;
    a.Wt = Wt;
    a.bf16 = bf16;
    a.T = T;
    a.K = K;
    a.n_out = n_out;
    a.score = mask_in ? AS_SCORE_MAG : cfg->score;
    a.sel = cfg->sel;
    a.n = cfg->n;
    a.m = cfg->m;
    a.k_keep = cfg->k_keep;
    a.dpts = cfg->dpts;
    a.tau = cfg->tau;
    a.eta_static = cfg->dpts == AS_PTS_STATIC ? cfg->eta_static : nullptr;
    a.g = g;
    a.rowsum = rowsum;
    a.mask_in = mask_in;
    a.y = y;
    a.out_bf16 = cfg->out_dtype == AS_BF16;
    a.mask_out = mask_out;
    a.eta_out = eta_out;
    a.colnorm_out = mask_in ? nullptr : colnorm_out;
    a.partial = partial;
    a.counters = counters;
    a.eta_in = eta_ws;
    return cuda_status(launch_decode(a, plan, stream));
}

}  // extern "C"

// Validation and GEMM arguments shared by the prefill entry points.
static as_status prefill_args(const as_select_out *sel, const void *W, int T, int K, int n_out, const float *rowsum,
                              const float *eta, const float *nu, const as_config *cfg, void *y, GemmArgs &a)
{
    if (!sel || !W || !y || T <= 0 || K <= 0 || n_out <= 0) return AS_ERR_INVALID_ARG;
    as_status st = check_cfg(cfg, K);
    if (st != AS_OK) return st;
    if (K % 8 != 0 || n_out % 8 != 0) return AS_ERR_SHAPE;
    const bool sparse = is24(cfg);
    if (sparse && (K % 16 != 0 || !sel->x_compact || !sel->meta24)) return AS_ERR_INVALID_ARG;
    if (!sparse && !sel->x_masked) return AS_ERR_INVALID_ARG;
    if (cfg->dpts && (!rowsum || !eta)) return AS_ERR_INVALID_ARG;
    if (cfg->var && !nu) return AS_ERR_INVALID_ARG;
    const void *ptrs[] = {W, rowsum, eta, nu, y, sel->x_compact, sel->meta24, sel->x_masked, sel->x_masked_lo,
                          sel->x_compact_lo};
    for (const void *p : ptrs)
        if (!aligned16(p)) return AS_ERR_ALIGN;
    a = GemmArgs{};
    a.A = sparse ? sel->x_compact : sel->x_masked;
    a.A_lo = sparse ? sel->x_compact_lo : sel->x_masked_lo;
    a.meta = sparse ? sel->meta24 : nullptr;
    a.W = W;
    a.T = T;
    a.K = K;
    a.n_out = n_out;
    a.sparse = sparse;
    a.rowsum = cfg->dpts ? rowsum : nullptr;
    a.eta = cfg->dpts ? eta : nullptr;
    a.nu = cfg->var ? nu : nullptr;
    a.y = y;
    a.out_bf16 = cfg->out_dtype == AS_BF16;
    return AS_OK;
}

extern "C" {

as_status as_linear_prefill(const as_select_out *sel, const void *W, int T, int K, int n_out, const float *rowsum,
                            const float *eta, const float *nu, const as_config *cfg, void *y, void *workspace,
                            size_t ws_bytes, cudaStream_t stream)
{
    (void)workspace;
    (void)ws_bytes;
    GemmArgs a;
    const as_status st = prefill_args(sel, W, T, K, n_out, rowsum, eta, nu, cfg, y, a);
    if (st != AS_OK) return st;
    return cuda_status(launch_gemm(a, stream));
}

size_t as_rsparse_prefill_workspace(int T, int K, int r)
{
    if (T <= 0 || K <= 0 || (r != 64 && r != 128)) return (size_t)-1;
    return rsp_layout(T, K, r).bytes;
}

as_status as_linear_prefill_rsparse(const as_select_out *sel, const void *x, const void *W, int T, int K, int n_out,
                                    const float *rowsum, const float *eta, const as_config *cfg, int r,
                                    const void *B, const void *A, void *y, void *workspace, size_t ws_bytes,
                                    cudaStream_t stream)
{
    if (!x || !B || !A || !sel || !sel->bitmask) return AS_ERR_INVALID_ARG;
    if (cfg && cfg->var) return AS_ERR_UNSUPPORTED;  // the pages define no VAR scale of the compensation
    GemmArgs a;
    as_status st = prefill_args(sel, W, T, K, n_out, rowsum, eta, nullptr, cfg, y, a);
    if (st != AS_OK) return st;
    if (r != 64 && r != 128) return AS_ERR_SHAPE;
    for (const void *p : {x, B, A, (const void *)sel->bitmask, (const void *)workspace})
        if (!aligned16(p)) return AS_ERR_ALIGN;
    const RspLayout L = rsp_layout(T, K, r);
    if (!workspace || ws_bytes < L.bytes) return AS_ERR_WORKSPACE;
    cudaError_t e = launch_rsp_u(x, sel->bitmask, cfg->dpts ? eta : nullptr, B, T, K, r, workspace, stream);
    if (e != cudaSuccess) return AS_ERR_CUDA;
    a.U2 = static_cast<const char *>(workspace) + L.u;
    a.Ar = A;
    a.r = r;
    return cuda_status(launch_gemm(a, stream));
}

int as_decode_launches(int T, int K, int n_out, as_dtype dt, const as_config *cfg)
{
    if (as_workspace_size(AS_OP_DECODE, T, K, n_out, cfg) == (size_t)-1) return -1;
    const int bf16 = dt == AS_BF16;
    DecodePlan plan = decode_plan(T, K, n_out, bf16);
    DecodeArgs a{};
    a.T = T;
    a.K = K;
    a.n_out = n_out;
    a.dpts = cfg->dpts;
    a.tau = cfg->tau;
    a.eta_static = cfg->dpts == AS_PTS_STATIC ? cfg->eta_static : nullptr;
    a.bf16 = bf16;
    a.sel = cfg->sel;
    a.out_bf16 = cfg->out_dtype == AS_BF16;
    int n = 0;
    if (decode_needs_select(T, K, n_out, bf16, a.out_bf16, cfg->sel))
        n += 1 + (cfg->score == AS_SCORE_CLACT ? 2 : 0);  // select kernel (+ column energy)
    return n + decode_launch_count(a, plan);
}

namespace {
// An mbarrier that nothing arrives on: the bounded wait runs out.
__global__ void k_probe_timeout(unsigned polls)
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(&bar, 0, polls);
}
}  // namespace

as_status as_probe_timeout(unsigned polls, cudaStream_t stream)
{
    if (polls < 1 || polls > (1u << 20)) return AS_ERR_INVALID_ARG;
    k_probe_timeout<<<1, 32, 0, stream>>>(polls);
    return cuda_status(cudaGetLastError());
}

int as_checked_line(void)
{
    int line = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&line, as::g_bounds_line, sizeof(int)) != cudaSuccess) return -1;
    if (line != 0 && cudaMemcpyToSymbol(as::g_bounds_line, &zero, sizeof(int)) != cudaSuccess) return -1;
    return line;
}

as_status as_stream_status(cudaStream_t stream)
{
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return AS_ERR_CUDA;
    int code = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&code, as::g_status, sizeof(int)) != cudaSuccess) return AS_ERR_CUDA;
    if (code != 0 && cudaMemcpyToSymbol(as::g_status, &zero, sizeof(int)) != cudaSuccess) return AS_ERR_CUDA;
    return code == 0 ? AS_OK : static_cast<as_status>(code);
}

}  // extern "C"
