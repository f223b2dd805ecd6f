/*
 * actsparse.h -- C ABI of the activation-sparsified linear layer
 *                y = prune(x) W^T  on NVIDIA B200 (sm_100a).
 *
 * The layer keeps, per token, a subset of the input channels of x and
 * contracts only those against W.  Sources (page title, section):
 *   [OVW] "激活稀疏化技术：提升LLM推理效率的动态剪枝方法" (activation-sparsity
 *         overview): 2.1 N:M patterns, 2.2.1 magnitude score, 2.2.3 CLACT
 *         score, 3.1 D-PTS mean shift, 3.2 VAR variance correction.
 *   [WIS] "大模型推理优化：WiSparse激活稀疏化技术解析": 2.1 eq. (4) weight-aware
 *         score, 2.2 per-layer keep fraction, 3.1 fused sparse operator.
 *   [SQR] "利用2:4稀疏性与Squared-ReLU加速Transformer训练与推理": 2.1 2:4 on
 *         tensor cores, 2.3 3-nonzero blocks, 3.3 compressed layout.
 *
 * Conventions for every entry point
 *   - Layouts are row-major.  x is [T, K] (T tokens, K input channels),
 *     W is [n_out, K] (PyTorch Linear layout), Wt is [K, n_out], y is
 *     [T, n_out].  All pointers are DEVICE pointers owned by the caller
 *     unless stated otherwise; the library never allocates and never frees.
 *   - Every call is asynchronous and ordered on `stream` (0 = legacy default
 *     stream).  Scratch memory is passed in as `workspace`, sized with
 *     as_workspace_size().  Workspace must be zero-filled once before its
 *     first use; every call leaves it zero-filled again.  The exceptions
 *     are as_weight_prep_amber, as_rsparse_decode, as_linear_prefill_hybrid
 *     and as_block_sparsity: they need no zero-fill and leave their
 *     workspace in an unspecified state (do not share it with the other
 *     calls).  Calls that share a workspace must not run concurrently.
 *   - Errors are returned, never raised: arguments are validated on the host
 *     and an invalid call launches nothing.  A kernel that gives up a bounded
 *     wait records AS_ERR_TIMEOUT in a device status word that
 *     as_stream_status() reports.  No entry point aborts, exits or traps.
 *   - A library built with -DAS_BOUNDS_CHECK (libactsparse_checked.so)
 *     checks the kernels' global and shared-memory indices against the
 *     buffers they address; a failed check skips that access and records
 *     AS_ERR_BOUNDS in the same status word.  Default builds have no checks.
 *   - Device pointers must be 16-byte aligned (AS_ERR_ALIGN otherwise).
 *   - Channel selection is deterministic: exactly N per M-block (or exactly
 *     k_keep per token), equal float32 scores broken towards the lower channel
 *     index; repeated calls give bitwise-identical results.
 */
#ifndef ACTSPARSE_H
#define ACTSPARSE_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define AS_ABI_VERSION 3
#define AS_MAX_DECODE_T 16

typedef enum as_status {
    AS_OK = 0,
    AS_ERR_INVALID_ARG = 1,  /* NULL where a buffer is required, bad enum */
    AS_ERR_SHAPE = 2,        /* K % M != 0, N > M, k_keep > K, T out of range */
    AS_ERR_DTYPE = 3,        /* dtype not supported by this operation */
    AS_ERR_ALIGN = 4,        /* pointer or row stride not 16-byte aligned */
    AS_ERR_UNSUPPORTED = 5,  /* valid but unsupported combination */
    AS_ERR_WORKSPACE = 6,    /* workspace NULL or smaller than required */
    AS_ERR_CUDA = 7,         /* a CUDA runtime/driver call failed */
    AS_ERR_TIMEOUT = 8,      /* a device-side bounded wait gave up */
    AS_ERR_BOUNDS = 9        /* a checked build found an index outside its buffer */
} as_status;

typedef enum as_dtype { AS_F32 = 0, AS_BF16 = 1 } as_dtype;

/* Channel score s_ti, taken in float32 ([OVW] 2.2.1, 2.2.3; [WIS] eq. 4):
 *   xhat = fl32(x - eta_t) with D-PTS, x otherwise;  s = fl32(|xhat| * f_i)
 *   AS_SCORE_MAG:    f_i = 1
 *   AS_SCORE_WEIGHT: f_i = g_i = ||W[:,i]||_2^alpha (from as_weight_prep)
 *   AS_SCORE_CLACT:  f_i = c_i = sqrt(sum over the T tokens of the call of
 *                    x_ti^2); the CLACT row factor 1/||x_t|| is the same for
 *                    every channel of a token and does not change the ranking. */
typedef enum as_score { AS_SCORE_MAG = 0, AS_SCORE_WEIGHT = 1, AS_SCORE_CLACT = 2 } as_score;

/* Selection ([OVW] 2.1; [WIS] 2.2):
 *   AS_SEL_NM:     in every block of m consecutive channels [jm, jm+m) keep the
 *                  n largest scores; m in {1,2,4,8,16,32}, 1 <= n <= m, K % m == 0.
 *   AS_SEL_TOPK:   keep the k_keep largest scores of each token, 0 <= k_keep <= K.
 *   AS_SEL_ALL:    keep every channel (dense layer, for baselines and checks).
 *   AS_SEL_THRESH: keep every channel whose score is > cfg->tau (a calibrated
 *                  per-layer threshold: [WIS] 3.1 builds on TEAL's sparse
 *                  operator, [WIS] 5 tunes its threshold tau); the number
 *                  kept varies per token. */
typedef enum as_sel { AS_SEL_NM = 0, AS_SEL_TOPK = 1, AS_SEL_ALL = 2, AS_SEL_THRESH = 3 } as_sel;

/* Token shift ([OVW] 3.1): */
enum {
    AS_PTS_OFF = 0,     /* no shift */
    AS_PTS_DYNAMIC = 1, /* D-PTS: eta_t = mean_i x_ti of the call's token */
    AS_PTS_STATIC = 2   /* S-PTS: eta_t = cfg->eta_static[t], a calibrated table
                           ([OVW] 3.1 static version, indexed per token; read here
                           as one float32 per token row of the call, [T]) */
};

typedef struct as_config {
    int32_t score;        /* as_score */
    int32_t sel;          /* as_sel */
    int32_t n, m;         /* N:M pattern (AS_SEL_NM) */
    int32_t k_keep;       /* kept channels per token (AS_SEL_TOPK) */
    int32_t dpts;         /* token shift, AS_PTS_*, [OVW] 3.1: score and keep
                             xhat = x - eta_t and add eta_t * rowsum_o back:
                             y = (xhat*m) W^T + eta * rowsum(W).  1: eta_t =
                             mean_i x_ti (D-PTS); 2: eta_t = eta_static[t] (S-PTS). */
    int32_t var;          /* 1: VAR, [OVW] 3.2 (prefill only; not with dpts):
                             running_t <- var_dense_t on the first batch, else
                             mom*running_t + (1-mom)*var_dense_t; then
                             nu_t = sqrt(running_t / (Var[x_t*m_t] + eps)),
                             y_t <- nu_t * y_t.  Variances are unbiased. */
    float var_momentum;   /* mom, 0.9 on the page */
    float var_eps;        /* eps, 1e-6 on the page */
    int32_t out_dtype;    /* as_dtype of y */
    float tau;            /* AS_SEL_THRESH: keep scores > tau */
    const float *eta_static; /* dpts == AS_PTS_STATIC: device [T] float32 eta table
                                (16-byte aligned); ignored otherwise */
} as_config;

/* Outputs of as_select.  Every pointer is optional (NULL = not written) unless
 * the operation needs it; all are device memory. */
typedef struct as_select_out {
    uint32_t *bitmask;   /* [T, ceil(K/32)]: bit (i % 32) of word i/32 = channel i kept */
    float *eta;          /* [T]  D-PTS mean (float32, the value the score used) */
    float *colnorm;      /* [K]  CLACT c_i (float32, the value the score used) */
    float *var_dense;    /* [T]  Var[x_t] (VAR) */
    float *var_kept;     /* [T]  Var[x_t * m_t] (VAR) */
    float *nu;           /* [T]  VAR scale */
    void *x_masked;      /* [T, K] in x's dtype: xhat*m, zeros where dropped */
    void *x_compact;     /* 2:4 only, bf16 [T, K/2]: the two kept values of every
                            4-block in ascending channel order ([SQR] 3.3) */
    uint32_t *meta24;    /* 2:4 only: positions of the kept values in the
                            tcgen05 sparse-MMA metadata layout; size in 32-bit
                            words is as_meta24_words(T, K).  Layout: tiles of
                            128 tokens x 128 channels, tile (r, c) at word offset
                            (r * ceil(K/128) + c) * 512; inside a tile, word
                            lane*4 + j holds MMA step j (channels 32j..32j+31 of
                            the tile) for TMEM lane
                                lane = 16*(p/16) + 8*(q/16) + p%8
                            (p = token within the tile, q = channel within the
                            32-channel step): bits [16*((p%16)/8) + 4*((q%16)/4),
                            +4) of that word hold the 4-block's two positions
                            i0 | i1 << 2, i0 < i1.  Padding blocks hold 0x4. */
    void *x_masked_lo;   /* bf16 x only, [T, K] bf16: bf16(xhat*m - x_masked), the
                            part of the kept values that rounding to bf16 lost.
                            With a token shift the kept values xhat = x - eta
                            are float32 numbers, not bf16 ones; for float32
                            output as_linear_prefill adds x_masked_lo W^T in a
                            second pass over K (hi + lo keeps xhat to about
                            2^-17 relative).  Needs x_masked. */
    void *x_compact_lo;  /* 2:4 only, bf16 [T, K/2]: the same residual of
                            x_compact (zeros when no shift).  Needs x_compact. */
    uint32_t *bitmask24; /* N:M with m a multiple of 4 and m >= 8 (optional,
                            with x_masked, x_compact and meta24): the 2:4-
                            compliant part of the selection ([SQR] 3.2 applied
                            to an N:M selection).  In every 4-block the two
                            channels ranked first by (kept, higher score,
                            lower index) form the part; x_compact/meta24 hold
                            their values xhat*m (zero for a dropped channel
                            that pads a block with fewer than two kept) and
                            positions, and bitmask24 [T, ceil(K/32)] the kept
                            channels inside the part.  See
                            as_linear_prefill_nm_split. */
} as_select_out;

/* --------------------------------------------------------------------------
 * Weight preparation, once per layer ([WIS] 2.1: norms precomputed; [OVW] 3.1).
 *   W      [n_out, K] in dtype `dt` (input).
 *   Wt     [K, n_out] in `dt` (output, optional): channel-major copy that the
 *          decode path streams, one contiguous row per kept channel.
 *   g      [K] float32 (optional): ||W[:,i]||_2^alpha, accumulated in float64.
 *   rowsum [n_out] float32 (optional): sum_i W[o,i], accumulated in float64.
 *   Workspace: as_workspace_size(AS_OP_WEIGHT_PREP, 0, K, n_out, NULL).
 * ------------------------------------------------------------------------ */
as_status as_weight_prep(const void *W, as_dtype dt, int n_out, int K, float alpha,
                         void *Wt, float *g, float *rowsum,
                         void *workspace, size_t ws_bytes, cudaStream_t stream);

/* --------------------------------------------------------------------------
 * Amber-Pruner channel importance, once per layer ([OVW] 2.2.2): the weights
 * outside the lo/hi percentiles are dropped, the rest standardised by their
 * own mean and standard deviation, and each input channel scored by the l2
 * norm of its standardised weights.  Feed g as the chan_factor of
 * AS_SCORE_WEIGHT (score s_ti = |x_ti| * g_i).
 *   W       [n_out, K] in `dt` (input); finite values.
 *   lo_pct, hi_pct: percentiles in [0, 100], lo_pct <= hi_pct (0.5 and 99.5
 *           on the page).  A percentile is the value of ascending rank
 *           floor(pct/100 * (N-1)) among all N = n_out*K weights (exact
 *           order statistic; -0 and +0 are equal); N < 2^32.
 *   kept:   v_lo <= W[o,i] <= v_hi (both ends inclusive).  mu and sigma are
 *           the mean and population standard deviation of the kept weights
 *           (float64); z[o,i] = (W[o,i] - mu) / sigma for kept weights, 0 for
 *           dropped ones, and 0 everywhere when sigma == 0.
 *   g       [K] float32 (output): (sqrt(sum_o z[o,i]^2))^alpha.
 *   bounds  [2] float32 (output, optional): v_lo, v_hi.
 *   Workspace: as_workspace_size(AS_OP_AMBER, 0, K, n_out, NULL); no
 *   zero-fill needed.  Deterministic (fixed reduction order).
 *   AS_ERR_INVALID_ARG for a NULL W or g, or percentiles out of range;
 *   AS_ERR_SHAPE when N >= 2^32.
 * ------------------------------------------------------------------------ */
as_status as_weight_prep_amber(const void *W, as_dtype dt, int n_out, int K, float alpha,
                               double lo_pct, double hi_pct, float *g, float *bounds,
                               void *workspace, size_t ws_bytes, cudaStream_t stream);

/* --------------------------------------------------------------------------
 * Score + selection + compensation statistics for T tokens (prefill side, or
 * to inspect a decode selection).  x [T, K] in `dt`.
 *   chan_factor: g [K] for AS_SCORE_WEIGHT (required); ignored otherwise
 *                (CLACT computes c over the T tokens and writes out->colnorm
 *                when given).
 *   running_var: [T] float32 in/out, required when cfg->var; when
 *                var_first_batch != 0 it is overwritten with var_dense.
 *   out:         see as_select_out.  2:4 outputs need dt == AS_BF16 and
 *                K % 16 == 0.  x_masked is written in x's dtype.
 *   Workspace: as_workspace_size(AS_OP_SELECT, T, K, 0, cfg).
 * ------------------------------------------------------------------------ */
as_status as_select(const void *x, as_dtype dt, int T, int K, const as_config *cfg,
                    const float *chan_factor, float *running_var, int var_first_batch,
                    const as_select_out *out, void *workspace, size_t ws_bytes,
                    cudaStream_t stream);

/* --------------------------------------------------------------------------
 * Per-token statistics of a selection ([SQR] 2.3: where a 4-block holds
 * three natural nonzeros, the 2:4 selection has to drop one of them; the
 * page puts that near 1 % of the values at 95 % sparsity).
 *   x        [T, K] in `dt` (AS_BF16 or AS_F32): the activations selected from.
 *   bitmask  [T, ceil(K/32)] keep words (bit c%32 of word c/32), as written
 *            by as_select or by the decode's mask_out.
 *   kept     [T] int32 (may be NULL): kept channels of each token.
 *   nz_dropped [T] int32 (may be NULL): channels with x != 0 that were not
 *            kept.
 * K % 8 == 0; pointers 16-byte aligned.  No workspace.  One kernel on
 * `stream`; exact integer counts.
 * ------------------------------------------------------------------------ */
as_status as_select_stats(const void *x, as_dtype dt, const uint32_t *bitmask, int T, int K, int32_t *kept,
                          int32_t *nz_dropped, cudaStream_t stream);

/* --------------------------------------------------------------------------
 * Decode: 1 <= T <= 16 tokens against the channel-major weight Wt [K, n_out].
 * For N:M selection the score, block top-N, D-PTS mean and the contraction
 * run in one kernel that streams only the union over the T tokens of the
 * kept rows of Wt ([WIS] 3.1: sparsify fused with the matmul, no
 * intermediate activation written); top-k runs a per-token selection kernel
 * first.  Accumulation is float32 in a fixed order (deterministic).
 *   x [T, K] and Wt in `dt`; g [K] float32 for AS_SCORE_WEIGHT; rowsum
 *   [n_out] float32 when cfg->dpts.  y [T, n_out] in cfg->out_dtype.
 *   mask_out [T, ceil(K/32)] (optional): the selection bitmask.
 *   eta_out [T] (optional): the float32 D-PTS mean the score used.
 *   colnorm_out [K] (optional): the float32 CLACT c the score used.
 *   Requires n_out % 8 == 0.  cfg->var is not supported (AS_ERR_UNSUPPORTED).
 *   Workspace: as_workspace_size(AS_OP_DECODE, T, K, n_out, cfg).
 * ------------------------------------------------------------------------ */
as_status as_linear_decode(const void *x, as_dtype dt, int T, int K, int n_out,
                           const void *Wt, const float *g, const float *rowsum,
                           const as_config *cfg, void *y, uint32_t *mask_out,
                           float *eta_out, float *colnorm_out,
                           void *workspace, size_t ws_bytes, cudaStream_t stream);

/* --------------------------------------------------------------------------
 * Prefill contraction on the tensor cores (bf16 in, float32 accumulate in
 * tensor memory, output in cfg->out_dtype) over a selection made by
 * as_select with the same cfg:
 *   cfg->sel == AS_SEL_NM with n=2, m=4: sel->x_compact + sel->meta24 are
 *     the sparse A operand of tcgen05.mma.sp ([SQR] 2.1: the tensor core
 *     skips the dropped half of the multiply-adds).
 *   any other selection: sel->x_masked is the A operand of a dense
 *     tcgen05.mma GEMM (tensor cores support 2:4 only).
 *   AS_SEL_ALL: x itself (sel->x_masked may point at x).
 *   W [n_out, K] bf16 (K-major, the PyTorch layout).  Epilogue:
 *   y = nu_t * acc (cfg->var, nu from as_select) or acc + eta_t * rowsum_o
 *   (cfg->dpts), then rounding to the output dtype.
 *   Residual operand: when sel->x_masked_lo (dense path) or
 *   sel->x_compact_lo (2:4 path) is given, a second pass over K adds its
 *   product with the same W blocks (and 2:4 positions) to the accumulator,
 *   so acc = (hi + lo) W^T.  Use it for float32 output with a token shift
 *   (twice the tensor-core work); with bf16 output the output's own
 *   rounding is as large as the kept values' and one pass suffices.
 *   Requires K % 8 == 0 (K % 16 == 0 for 2:4) and n_out % 8 == 0.
 *   Workspace: as_workspace_size(AS_OP_PREFILL, T, K, n_out, cfg) (zero).
 * ------------------------------------------------------------------------ */
as_status as_linear_prefill(const as_select_out *sel, const void *W, int T, int K,
                            int n_out, const float *rowsum, const float *eta,
                            const float *nu, const as_config *cfg, void *y,
                            void *workspace, size_t ws_bytes, cudaStream_t stream);

/* --------------------------------------------------------------------------
 * as_linear_decode_noalloc: as_linear_decode for callers that cannot
 * allocate device memory.  (The pages have no counterpart; this is a
 * deployment variant of the same decode.)
 *
 * Some callers cannot call cudaMalloc, for example code running inside a
 * host framework that owns all device memory through its own pool and
 * forbids allocations from outside it, or a process held to a device-memory
 * budget fixed at start-up.  This entry point takes no workspace: its scratch
 * (split-K partial sums, arrival counters, the top-k bitmask) lives in one
 * file-scope device array of AS_NOALLOC_SCRATCH_BYTES, which every GPU that
 * loads the library holds until the process exits.  The caller still passes
 * inputs and outputs, with the meaning, layouts and errors of
 * as_linear_decode.
 *   - It allocates nothing: no cudaMalloc, no cudaFree, no allocating library
 *     routine.  Calls whose scratch need (as_workspace_size(AS_OP_DECODE, ...))
 *     exceeds AS_NOALLOC_SCRATCH_BYTES return AS_ERR_WORKSPACE and launch nothing.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current) and caches it; make
 *     that first call before any stream capture.  The cached address is
 *     valid for the life of the device's context: after cudaDeviceReset the
 *     library's device code is loaded again and the array may move, so do
 *     not call this entry point again in that process.
 *   - Every argument is checked before the array is touched: a refused call
 *     (any error status) enqueues nothing on `stream`.
 *   - All calls share the array and it keeps the last call's contents.  The
 *     part that must start at zero is cleared on `stream` at every call.
 *     Calls whose executions overlap on the GPU (different streams without
 *     ordering, or several host threads) race on the array and give
 *     undefined results: order them on one stream.
 * ------------------------------------------------------------------------ */
#define AS_NOALLOC_SCRATCH_BYTES (8u << 20)
as_status as_linear_decode_noalloc(const void *x, as_dtype dt, int T, int K, int n_out,
                                   const void *Wt, const float *g, const float *rowsum,
                                   const as_config *cfg, void *y, uint32_t *mask_out,
                                   float *eta_out, float *colnorm_out, cudaStream_t stream);

/* Which operation a workspace size is asked for. */
enum { AS_OP_WEIGHT_PREP = 0, AS_OP_SELECT = 1, AS_OP_DECODE = 2, AS_OP_PREFILL = 3, AS_OP_AMBER = 4 };

/* Bytes of workspace the operation needs (0 if none); (size_t)-1 if the
 * arguments are invalid. */
size_t as_workspace_size(int op, int T, int K, int n_out, const as_config *cfg);

/* Number of kernels one as_linear_decode call with these arguments launches
 * (for sizing CUDA graphs and counting launches); -1 if the arguments are
 * invalid.  Host-only. */
int as_decode_launches(int T, int K, int n_out, as_dtype dt, const as_config *cfg);

/* --------------------------------------------------------------------------
 * Hybrid 2:4 prefill ([SQR] 3.2: the densest features are computed densely
 * and the rest with 2:4; [SQR] 3.3: the layer's sparsity picks the mode,
 * above 95 %: pure 2:4, 90-95 %: the split, below 90 %: dense).  Features
 * are 4-channel blocks.  The dense set D is the n_dense blocks with the most
 * nonzeros of x over the T tokens, ties to the lower block index; the result
 * is the masked product with D's blocks kept whole and 2:4 elsewhere:
 *   y = (x (.) m) W^T + (x (.) (1 - m))[:, D] W[:, D]^T,
 * m the 2:4 magnitude selection of x.  The second term runs inside the 2:4
 * GEMM: the gathered remainder of D's blocks and their W columns are extra
 * dense tcgen05 K blocks after the sparse ones, into the same accumulator.
 *   sel      the as_select outputs of x with sel = AS_SEL_NM, n = 2, m = 4,
 *            score AS_SCORE_MAG, no token shift or VAR: bitmask, x_compact
 *            and meta24 are required.
 *   x, W     bf16 [T, K] (the same x) and [n_out, K]; K % 64 == 0,
 *            K <= 32768, n_out % 8 == 0, T < 2^22.
 *   n_dense  0 <= n_dense <= K/4, a multiple of 16 (0: pure 2:4).
 *   y        [T, n_out] in out_dtype.
 *   dense_idx [n_dense] int32 (optional): D in ascending block order.
 *   sparsity [1] float32 (optional): 1 - nnz(x) / (T*K).
 * Workspace: as_hybrid_workspace(T, K, n_out, n_dense) bytes, no zero-fill
 * needed.  as_block_sparsity runs only the counting (and, with n_dense > 0,
 * the choice of D) for the mode decision; its workspace is
 * as_hybrid_workspace(T, K, 0, 0).
 * ------------------------------------------------------------------------ */
size_t as_hybrid_workspace(int T, int K, int n_out, int n_dense);
as_status as_linear_prefill_hybrid(const as_select_out *sel, const void *x, int T, int K, const void *W, int n_out,
                                   int n_dense, as_dtype out_dtype, void *y, int32_t *dense_idx, float *sparsity,
                                   void *workspace, size_t ws_bytes, cudaStream_t stream);
as_status as_block_sparsity(const void *x, int T, int K, int n_dense, int32_t *dense_idx, float *sparsity,
                            void *workspace, size_t ws_bytes, cudaStream_t stream);

/* --------------------------------------------------------------------------
 * Hybrid 2:4 decomposition of an N:M selection ([SQR] 3.2: the densest
 * features dense, the rest 2:4 on the sparse tensor cores; here applied to
 * an N:M selection that is not 2:4-compliant, 8:16 or 16:32):
 *   y = epilogue((xm (.) p) W^T + (xm (.) (1 - p))[:, D] W[:, D]^T),
 * xm = xhat (.) m the masked activation (sel->x_masked), p the 2:4 part
 * (sel->bitmask24, x_compact, meta24 from as_select), D the n_dense
 * 4-channel blocks with the most nonzeros of xm over the T tokens (ties to
 * the lower block index).  Kept channels outside p and outside D are
 * dropped, so the result is the N:M product exactly when D covers every
 * block with more than two kept channels for some token (n_dense = K/4
 * always does); fewer dense blocks trade that remainder for speed.  The
 * epilogue is as_linear_prefill's (x nu_t with VAR, + eta_t rowsum_o with a
 * token shift, rounding to cfg->out_dtype).
 *   cfg      the as_select configuration: AS_SEL_NM, m a multiple of 4 and
 *            m >= 8.
 *   n_dense  0 <= n_dense <= K/4, a multiple of 16.  K % 64 == 0,
 *            K <= 32768, n_out % 8 == 0, T < 2^22.
 *   dense_idx, sparsity: as as_linear_prefill_hybrid (sparsity: of xm).
 * Workspace: as_hybrid_workspace(T, K, n_out, n_dense), no zero-fill.
 * as_block_sparsity on xm gives the sparsity for as_prefill_mode.
 * ------------------------------------------------------------------------ */
as_status as_linear_prefill_nm_split(const as_select_out *sel, int T, int K, const void *W, int n_out, int n_dense,
                                     const as_config *cfg, const float *rowsum, const float *eta, const float *nu,
                                     void *y, int32_t *dense_idx, float *sparsity, void *workspace, size_t ws_bytes,
                                     cudaStream_t stream);

/* The inference mode switch ([SQR] 3.3), host-only.  The page keys the mode
 * on the layer's measured activation sparsity (as_block_sparsity's output):
 * above 95 %: pure 2:4; from 90 % to 95 % (both ends included): the split;
 * below 90 %: the dense product.  The page's snippet lost its comparison
 * signs, so the two thresholds themselves are read as "split".  Returns an
 * as_mode; a NaN sparsity returns AS_MODE_DENSE. */
typedef enum as_mode { AS_MODE_24 = 0, AS_MODE_SPLIT = 1, AS_MODE_DENSE = 2 } as_mode;
int as_prefill_mode(double sparsity);

/* Number of dense 4-channel blocks of the split ([SQR] 3.2 keeps about 5 %
 * of the features dense): dense_frac of the K/4 blocks rounded up to a
 * multiple of 16 (64 channels, the dense GEMM's K step), at least 16 and at
 * most the multiple-of-16 part of K/4 (as_linear_prefill_hybrid's bounds).
 * Host-only; -1 for K not a positive multiple of 64 or dense_frac outside
 * [0, 1]. */
int as_hybrid_dense_blocks(int K, double dense_frac);

/* --------------------------------------------------------------------------
 * R-Sparse low-rank compensation of a decode call ([OVW] 3.3).  The weight
 * is approximated as W ~ W_sparse + A_r B_r^T with A_r = U_r diag(S_r)
 * [n_out, r] and B_r = V_r [K, r] from a truncated SVD of W (computed
 * offline by the caller; the page uses r = 64).  The kept channels already
 * went through W in the call; this adds the dropped ones through the
 * factors:
 *   u[t, j]  = sum over channels i with mask bit (t, i) clear of xhat[t, i] B[i, j]
 *   y[t, o] += sum_j u[t, j] A[o, j]
 * with xhat = fl32(x - eta[t]) when eta is given (D-PTS or S-PTS: pass the
 * call's eta_out or table) and x otherwise.
 *   x      [T, K] in `dt`, the call's input, 1 <= T <= 16.
 *   mask   [T, ceil(K/32)] uint32, the call's mask_out (bit i%32 of word i/32 = kept).
 *   B, A   bf16 [K, r] and [n_out, r]; r in {32, 64, 128}; A 16-byte aligned.
 *   y      [T, n_out] float32, in/out (the call with out_dtype AS_F32).
 * Float32 accumulation in a fixed order (deterministic); two kernels.
 * Workspace: as_rsparse_workspace(T, K, r) bytes, no zero-fill needed.
 * ------------------------------------------------------------------------ */
size_t as_rsparse_workspace(int T, int K, int r);
as_status as_rsparse_decode(const void *x, as_dtype dt, int T, int K, int n_out, int r, const uint32_t *mask,
                            const float *eta, const void *B, const void *A, float *y, void *workspace,
                            size_t ws_bytes, cudaStream_t stream);

/* --------------------------------------------------------------------------
 * R-Sparse compensation of a prefill call ([OVW] 3.3): as_linear_prefill
 * plus the dropped channels through the rank-r factors of W (the same
 * factors as as_rsparse_decode):
 *   y = epilogue((xhat (.) m) W^T + U A^T),  U = (xhat (.) (1 - m)) B,
 * with xhat = fl32(x - eta_t) under a token shift (cfg->dpts, eta the
 * as_select output), x otherwise, and m the selection (sel->bitmask).  U is
 * computed first ([T, r], float32 accumulation in a fixed order, the dropped
 * values entering the tensor cores as bf16 hi + lo) and stored as bf16 hi
 * and lo; the prefill GEMM then runs 2 r/64 more K blocks whose A operand is
 * U and whose B operand is A, into the same accumulator.
 *   sel, W, T, K, n_out, rowsum, eta, cfg, y: as as_linear_prefill (sel
 *            must also hold the bitmask); cfg->var is not supported
 *            (AS_ERR_UNSUPPORTED: the pages define no VAR scale of the
 *            compensation).
 *   x        bf16 [T, K], the call's input.
 *   B, A     bf16 [K, r] and [n_out, r]; r in {64, 128}.
 * Workspace: as_rsparse_prefill_workspace(T, K, r) bytes, no zero-fill.
 * ------------------------------------------------------------------------ */
size_t as_rsparse_prefill_workspace(int T, int K, int r);
as_status as_linear_prefill_rsparse(const as_select_out *sel, const void *x, const void *W, int T, int K, int n_out,
                                    const float *rowsum, const float *eta, const as_config *cfg, int r,
                                    const void *B, const void *A, void *y, void *workspace, size_t ws_bytes,
                                    cudaStream_t stream);

/* Number of 32-bit metadata words of a 2:4 selection of T tokens x K channels. */
size_t as_meta24_words(int T, int K);

/* --------------------------------------------------------------------------
 * FP8 2:4 prefill ([SQR] 3.1: a fused Squared-ReLU + 2:4 + FP8 producer and
 * a 2:4 GEMM on FP8 operands with row scaling; [SQR] 5.3: sparsify before
 * quantising).  FP8 is E4M3 (largest finite 448, no infinities), converted
 * with round-to-nearest-even and saturation.  Every row carries one float32
 * scale: scale = fl32(amax / 448) over the row's (kept) values, 1 for an
 * all-zero row.  The codes use the reciprocal, one multiply per value:
 * code = E4M3(fl32(v * r)) with r = fl32(448 / amax) (r = 1 for an all-zero
 * row); the value a code stands for is E4M3value(code) * scale.
 * ------------------------------------------------------------------------ */

/* Number of 32-bit words of FP8 2:4 positions for T tokens x K channels:
 * ceil(T/256)*2 tiles of 128 tokens by ceil(K/256) tiles of 256 channels,
 * 1024 words each.  Tile (r, c) starts at word (r * ceil(K/256) + c) * 1024
 * and holds two 512-word halves (channels 0..127 and 128..255 of the tile);
 * in a half, word p*4 + j holds channels 32j..32j+31 of the half for token
 * p of the tile, with the 4-block at channel q in bits [4*((q%32)/4), +4):
 * i0 | i1 << 2, i0 < i1 the kept positions.  Channels past K and tokens past
 * T (up to the next multiple of 256) hold positions (0, 1). */
size_t as_meta8_words(int T, int K);

/* Weight side, once per layer: W [n_out, K] in `dt` -> Wq [n_out, K] E4M3
 * codes and w_scale [n_out] (amax over the output row).  K % 16 == 0;
 * pointers 16-byte aligned. */
as_status as_weight_quant_fp8(const void *W, as_dtype dt, int n_out, int K, uint8_t *Wq, float *w_scale,
                              cudaStream_t stream);

/* Activation side, the fused producer.  z [T, K] bf16 pre-activations:
 *   x = fl32(max(0, z))^2 (computed in registers, never written);
 *   in every block of 4 channels keep the 2 largest x (ties to the lower
 *   channel);
 *   x_scale[t] = amax of the kept x of token t / 448 (1 if all are zero);
 *   x8 [T, K/2] codes of the kept values, in channel order;
 *   meta8 [as_meta8_words(T, K)] their positions (layout above);
 *   bitmask [T, K/32] (optional): bit i%32 of word i/32 set if kept.
 * K % 64 == 0; pointers 16-byte aligned. */
as_status as_select_sqrelu24_fp8(const void *z, int T, int K, uint8_t *x8, uint32_t *meta8, float *x_scale,
                                 uint32_t *bitmask, cudaStream_t stream);

/* The FP8 2:4 GEMM on CTA pairs (tcgen05.mma.sp kind::f8f6f4, float32
 * accumulation in tensor memory):
 *   y[t, o] = fl32(fl32(acc[t, o] * x_scale[t]) * w_scale[o]),
 *   acc[t, o] = sum over the kept channels i of E4M3value(x8) * E4M3value(Wq[o, i]).
 * y [T, n_out] in out_dtype (AS_BF16 or AS_F32).  K % 64 == 0,
 * n_out % 8 == 0.  AS_ERR_UNSUPPORTED if the device cannot co-schedule the
 * CTA pairs. */
as_status as_linear_prefill_fp8(const uint8_t *x8, const uint32_t *meta8, const float *x_scale, int T, int K,
                                int n_out, const uint8_t *Wq, const float *w_scale, as_dtype out_dtype, void *y,
                                cudaStream_t stream);

/* Synchronises `stream`, then reports (and clears) a device-side error such
 * as AS_ERR_TIMEOUT recorded by a kernel of this library, or AS_ERR_CUDA if
 * the stream itself failed. */
as_status as_stream_status(cudaStream_t stream);

/* Checked builds (-DAS_BOUNDS_CHECK): the source line of the first index
 * check that failed since the last call (0 if none; always 0 in default
 * builds), then cleared.  -1 if the device could not be read. */
int as_checked_line(void);

/* Self-test of the failure path: launches on `stream` one small kernel
 * whose bounded wait (`polls` polls, 1 .. 1<<20) is on an mbarrier that
 * nothing signals.  The wait runs out and records AS_ERR_TIMEOUT, and the
 * kernel returns normally, so the context stays usable.  The next
 * as_stream_status() reports AS_ERR_TIMEOUT and clears it.  The probe is
 * the same bounded-wait code every library kernel uses.  Returns
 * AS_ERR_INVALID_ARG for `polls` out of range, AS_ERR_CUDA if the launch
 * fails, AS_OK otherwise. */
as_status as_probe_timeout(unsigned polls, cudaStream_t stream);

/* Static description of a status code. */
const char *as_status_string(as_status s);

/* AS_ABI_VERSION of the loaded library. */
int as_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* ACTSPARSE_H */
