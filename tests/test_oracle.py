"""Pins for the CPU oracle: each test checks it against something other than
itself (a value the pages print, a closed form, an invariant, a special case
that reduces to a plain library routine, or brute-force enumeration), chosen
so that a dropped term, a wrong sign or index, or a transposed operand in the
oracle fails at least one of them.  No GPU needed."""
import math
import os

import numpy as np
import pytest
import torch

import synth
from oracle import brute

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _bf16(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).float().numpy()


# --------------------------------------------------------------------------
# Page-printed values: the N:M pattern table (overview page, section 2.1).
# --------------------------------------------------------------------------
def _table():
    rows = []
    with open(os.path.join(GOLDEN, "nm_table.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            pat, cnt, bits = line.split()
            n, m = map(int, pat.split(":"))
            rows.append((n, m, float(cnt), float(bits)))
    return rows


def _count_dp(m, n):
    # Pascal's rule, a different route from enumeration.
    row = [1]
    for _ in range(m):
        row = [1] + [row[i] + row[i + 1] for i in range(len(row) - 1)] + [1]
    return row[n]


def test_nm_table_keep_pattern_counts():
    for n, m, cnt, _ in _table():
        if m <= 16:
            assert brute.count_subsets(m, n) == int(cnt)
        else:  # printed to one significant digit
            c = _count_dp(m, n)
            assert round(c / 1e8) == round(cnt / 1e8)


def test_nm_table_metadata_bits():
    for n, m, cnt, bits in _table():
        if (n, m) == (4, 8):
            continue  # printed 0.81, ceil(log2 70)/8 = 0.875: garbled row
        c = brute.count_subsets(m, n) if m <= 16 else _count_dp(m, n)
        assert round(math.ceil(math.log2(c)) / m, 2) == round(bits, 2)


# --------------------------------------------------------------------------
# Selection: brute-force enumeration of every C(M,N) subset.
# --------------------------------------------------------------------------
@pytest.mark.parametrize("n,m", [(2, 4), (1, 4), (3, 4), (4, 8), (2, 8)])
def test_select_nm_matches_enumeration(oracle_lib, n, m):
    r = _rng(10 + n * 100 + m)
    for quant in (None, 4):  # quantised scores force ties
        s = r.random((3, 8 * m)).astype(np.float32)
        if quant:
            s = (np.floor(s * quant) / quant).astype(np.float32)
        np.testing.assert_array_equal(oracle_lib.select_nm(s, n, m), brute.select_nm(s, n, m))


def test_select_8of16_matches_enumeration(oracle_lib):
    r = _rng(7)
    s = (np.floor(r.random((1, 32)) * 6) / 6).astype(np.float32)
    np.testing.assert_array_equal(oracle_lib.select_nm(s, 8, 16), brute.select_nm(s, 8, 16))


def test_tiny_layer_all_c42_subsets(oracle_lib):
    """Tiny layer (x f32 [4,256], 2:4 magnitude): every block checked against
    all C(4,2)=6 subsets."""
    x, _ = synth.tiny_layer()
    s = oracle_lib.score(x.numpy())
    np.testing.assert_array_equal(oracle_lib.select_nm(s, 2, 4), brute.select_nm(s, 2, 4))


@pytest.mark.parametrize("kk", [0, 1, 3, 5, 9, 10])
def test_select_topk_matches_enumeration(oracle_lib, kk):
    r = _rng(kk)
    s = (np.floor(r.random((4, 10)) * 5) / 5).astype(np.float32)
    np.testing.assert_array_equal(oracle_lib.select_topk(s, kk), brute.select_topk(s, kk))


def test_select_invariants(oracle_lib):
    """Exactly N per block; every kept score >= every dropped score in its
    block; equal scores kept from the lower index first."""
    r = _rng(3)
    x = _bf16(r.laplace(0, 0.3, size=(5, 1024)))
    s = oracle_lib.score(x)
    for n, m in [(2, 4), (8, 16), (16, 32)]:
        mask = oracle_lib.select_nm(s, n, m)
        blocks = mask.reshape(5, -1, m)
        assert (blocks.sum(-1) == n).all()
        sb = s.reshape(5, -1, m)
        kept_min = np.where(blocks == 1, sb, np.inf).min(-1)
        drop_max = np.where(blocks == 0, sb, -np.inf).max(-1)
        assert (kept_min >= drop_max).all()
    for kk in (0, 1, 400, 1024):
        mask = oracle_lib.select_topk(s, kk)
        assert (mask.sum(1) == kk).all()
    # all-equal scores: the lowest indices win
    s0 = np.ones((1, 16), np.float32)
    np.testing.assert_array_equal(oracle_lib.select_nm(s0, 2, 4)[0], [1, 1, 0, 0] * 4)
    np.testing.assert_array_equal(oracle_lib.select_topk(s0, 3)[0], [1] * 3 + [0] * 13)


def test_zero_block_keeps_lowest_indices(oracle_lib):
    """A block [0, 0, 0, v] under 2:4 keeps {0, 3} (zeros are eligible)."""
    s = oracle_lib.score(np.array([[0, 0, 0, 0.5, 0, -2, 0, 0]], np.float32))
    np.testing.assert_array_equal(oracle_lib.select_nm(s, 2, 4)[0], [1, 0, 0, 1, 1, 1, 0, 0])


def test_three_nonzero_block_drops_smallest(oracle_lib):
    """2:4 + Squared-ReLU page, section 2.3: a 4-block with 3 nonzeros drops the
    smallest-magnitude one."""
    x = np.array([[0.0, 3.0, 1.0, 2.0, 5.0, 0.0, 0.25, 4.0]], np.float32)
    mask = oracle_lib.select_nm(oracle_lib.score(x), 2, 4)
    np.testing.assert_array_equal(mask[0], [0, 1, 0, 1, 1, 0, 0, 1])


# --------------------------------------------------------------------------
# Scores
# --------------------------------------------------------------------------
def test_score_definition_special_cases(oracle_lib):
    x = np.array([[1.5, -2.0, 0.25, -0.75]], np.float32)
    np.testing.assert_array_equal(oracle_lib.score(x)[0], np.abs(x[0]))
    eta = np.array([0.5], np.float32)
    np.testing.assert_array_equal(oracle_lib.score(x, eta=eta)[0], [1.0, 2.5, 0.25, 1.25])
    f = np.array([2.0, 0.5, 4.0, 1.0], np.float32)
    np.testing.assert_array_equal(oracle_lib.score(x, f=f)[0], [3.0, 1.0, 1.0, 0.75])


def test_weight_aware_alpha0_is_magnitude(oracle_lib):
    r = _rng(5)
    x = _bf16(r.laplace(0, 0.3, size=(3, 512)))
    W = _bf16(r.normal(0, 0.02, size=(300, 512)))
    g, _ = oracle_lib.weight_prep(W, 0.0)
    np.testing.assert_array_equal(g, np.ones(512))
    s_w = oracle_lib.score(x, f=g.astype(np.float32))
    np.testing.assert_array_equal(oracle_lib.select_nm(s_w, 8, 16),
                                  oracle_lib.select_nm(oracle_lib.score(x), 8, 16))


def test_clact_single_token_is_magnitude(oracle_lib):
    """With T=1, c_j = |x_j|, so |x_j| c_j = x_j^2 (exact in fp32 for bf16
    inputs) ranks like |x_j|."""
    r = _rng(6)
    x = _bf16(r.standard_t(3, size=(1, 1024)) * 0.5)
    c = oracle_lib.channel_energy(x).astype(np.float32)
    np.testing.assert_array_equal(c, np.abs(x[0]))
    s = oracle_lib.score(x, f=c)
    for n, m in [(2, 4), (16, 32)]:
        np.testing.assert_array_equal(oracle_lib.select_nm(s, n, m),
                                      oracle_lib.select_nm(oracle_lib.score(x), n, m))


def test_clact_row_factor_is_constant_per_token(oracle_lib):
    """The full CLACT score divided by |x_ij| c_j equals 1/||x_t|| for every
    channel of token t (overview page §2.2.3), which is why ranking by
    |x_ij| c_j gives the same per-token order."""
    r = _rng(8)
    x = _bf16(r.standard_t(3, size=(6, 256)) * 0.5)
    S = oracle_lib.clact_full(x)
    c = np.sqrt((x.astype(np.float64) ** 2).sum(0))
    rn = np.sqrt((x.astype(np.float64) ** 2).sum(1))
    np.testing.assert_allclose(S, np.abs(x) * c[None, :] / rn[:, None], rtol=1e-13)
    np.testing.assert_allclose(oracle_lib.channel_energy(x), c, rtol=1e-14)


# --------------------------------------------------------------------------
# Statistics and weight preparation: closed forms
# --------------------------------------------------------------------------
def test_token_stats_closed_forms(oracle_lib):
    k = 1000
    x = np.stack([np.full(k, 0.75), np.arange(k) * 0.5 - 3.0]).astype(np.float32)
    eta = oracle_lib.token_mean(x)
    np.testing.assert_allclose(eta, [0.75, (k - 1) / 2 * 0.5 - 3.0], rtol=1e-15)
    var = oracle_lib.token_var(x)
    np.testing.assert_allclose(var, [0.0, 0.25 * k * (k + 1) / 12], rtol=1e-13)


def test_weight_prep_closed_form(oracle_lib):
    """W[o, i] = a_i * b_o with known column norms |a_i| ||b|| and row sums
    b_o * sum(a): a transposed norm axis or a dropped exponent fails."""
    a = np.array([0.5, -1.0, 2.0, 0.25, 4.0], np.float64)
    b = np.array([1.0, -0.5, 0.25, 2.0, 0.125, -1.0, 0.5], np.float64)
    W = np.outer(b, a).astype(np.float32)  # [n_out=7, k=5]
    for alpha in (0.0, 0.5, 1.0, 1.7):
        g, rs = oracle_lib.weight_prep(W, alpha)
        np.testing.assert_allclose(g, (np.abs(a) * np.linalg.norm(b)) ** alpha, rtol=1e-14)
        np.testing.assert_allclose(rs, b * a.sum(), rtol=1e-14)


# --------------------------------------------------------------------------
# Contraction
# --------------------------------------------------------------------------
def test_linear_keep_all_is_dense_matmul(oracle_lib):
    r = _rng(11)
    x = _bf16(r.laplace(0, 0.3, size=(5, 96)))
    W = _bf16(r.normal(0, 0.02, size=(40, 96)))
    y = oracle_lib.linear(x, np.ones_like(x, np.uint8), W)
    np.testing.assert_allclose(y, x.astype(np.float64) @ W.astype(np.float64).T, rtol=1e-12, atol=1e-15)


def test_linear_masked_and_rows(oracle_lib):
    r = _rng(12)
    x = _bf16(r.laplace(0, 0.3, size=(6, 64)))
    W = _bf16(r.normal(0, 0.02, size=(33, 64)))
    mask = oracle_lib.select_nm(oracle_lib.score(x), 2, 4)
    ref = (x.astype(np.float64) * mask) @ W.astype(np.float64).T
    np.testing.assert_allclose(oracle_lib.linear(x, mask, W), ref, rtol=1e-12, atol=1e-15)
    rows = [5, 0, 3]
    np.testing.assert_allclose(oracle_lib.linear(x, mask, W, rows=rows), ref[rows], rtol=1e-12, atol=1e-15)


def test_dpts_identity(oracle_lib):
    """(xhat*m + eta) W^T computed densely equals (xhat*m) W^T + eta*rowsum(W)
    (overview page §3.1)."""
    r = _rng(13)
    x = _bf16(r.laplace(0.2, 0.3, size=(4, 128)))
    W = _bf16(r.normal(0, 0.02, size=(50, 128)))
    eta = oracle_lib.token_mean(x)
    eta32 = eta.astype(np.float32)
    mask = oracle_lib.select_nm(oracle_lib.score(x, eta=eta32), 8, 16)
    _, rs = oracle_lib.weight_prep(W, 1.0)
    y = oracle_lib.linear(x, mask, W, eta=eta, rowsum=rs)
    xhat = x.astype(np.float64) - eta[:, None]
    dense = (xhat * mask + eta[:, None]) @ W.astype(np.float64).T
    np.testing.assert_allclose(y, dense, rtol=1e-11, atol=1e-14)
    # and the shift really matters: without eta the result differs
    assert not np.allclose(oracle_lib.linear(x, mask, W), dense, rtol=1e-6)


def test_var_closed_form(oracle_lib):
    """Blocks [a, -a, b, -b] with |a| > |b| under 2:4: dense and kept sums are
    zero, so nu = sqrt(sum x^2 / (sum_kept x^2 + eps (K-1))) on the first
    batch (overview page §3.2)."""
    r = _rng(14)
    k = 256
    a = r.uniform(1.0, 2.0, size=k // 4)
    b = r.uniform(0.0, 0.9, size=k // 4)
    x = np.stack([a, -a, b, -b], 1).reshape(1, k).astype(np.float32)
    mask = oracle_lib.select_nm(oracle_lib.score(x), 2, 4)
    np.testing.assert_array_equal(mask.reshape(-1, 4), np.tile([1, 1, 0, 0], (k // 4, 1)))
    eps = 1e-6
    out = oracle_lib.var_scale(x, mask, None, 0.9, eps)
    x64 = x.astype(np.float64)[0]
    nu = math.sqrt((x64 ** 2).sum() / ((x64[mask[0] == 1] ** 2).sum() + eps * (k - 1)))
    np.testing.assert_allclose(out["nu"], [nu], rtol=1e-12)
    np.testing.assert_allclose(out["var_dense"], [(x64 ** 2).sum() / (k - 1)], rtol=1e-12)
    # keep-all: nu = sqrt(v / (v + eps))
    out = oracle_lib.var_scale(x, np.ones_like(mask), None, 0.9, eps)
    v = out["var_dense"][0]
    np.testing.assert_allclose(out["nu"], [math.sqrt(v / (v + eps))], rtol=1e-12)


def test_var_running_average_over_batches(oracle_lib):
    """Eight batches chained through the oracle equal a scalar recomputation
    of running <- 0.9 running + 0.1 var_dense (first batch: var_dense)."""
    r = _rng(15)
    T, k = 3, 64
    run = None
    scal = [None] * T
    for b in range(8):
        x = _bf16(r.standard_t(3, size=(T, k)) * 0.5)
        mask = oracle_lib.select_nm(oracle_lib.score(x), 16, 32)
        out = oracle_lib.var_scale(x, mask, run, 0.9, 1e-6)
        for t in range(T):
            vd = np.var(x[t].astype(np.float64), ddof=1)
            vk = np.var(x[t].astype(np.float64) * mask[t], ddof=1)
            scal[t] = vd if scal[t] is None else 0.9 * scal[t] + 0.1 * vd
            np.testing.assert_allclose(out["running"][t], scal[t], rtol=1e-12)
            np.testing.assert_allclose(out["nu"][t], math.sqrt(scal[t] / (vk + 1e-6)), rtol=1e-12)
        run = out["running"]


def test_vr_scale_applies_to_whole_row(oracle_lib):
    r = _rng(16)
    x = _bf16(r.laplace(0, 0.3, size=(3, 64)))
    W = _bf16(r.normal(0, 0.02, size=(20, 64)))
    mask = oracle_lib.select_nm(oracle_lib.score(x), 16, 32)
    nu = np.array([1.5, 0.5, 2.0])
    np.testing.assert_allclose(oracle_lib.linear(x, mask, W, nu=nu),
                               oracle_lib.linear(x, mask, W) * nu[:, None], rtol=1e-13)


def test_compress_roundtrip(oracle_lib):
    r = _rng(17)
    x = _bf16(r.laplace(0, 0.3, size=(3, 64)))
    mask = oracle_lib.select_nm(oracle_lib.score(x), 2, 4)
    vals, pos = oracle_lib.compress_nm(x, mask, 2, 4)
    assert vals.shape == (3, 32)
    back = np.zeros_like(x)
    for t in range(3):
        for j in range(32):
            back[t, (j // 2) * 4 + pos[t, j]] = vals[t, j]
    np.testing.assert_array_equal(back, x * mask)
    assert (pos.reshape(3, -1, 2)[:, :, 0] < pos.reshape(3, -1, 2)[:, :, 1]).all()


# --------------------------------------------------------------------------
# Squared-ReLU workload: closed-form sparsity statistics
# --------------------------------------------------------------------------
def test_sqrelu_sparsity_closed_form(oracle_lib):
    """z ~ N(-1.2, 1): natural zeros Phi(1.2) = 0.88493; enforcing 2:4 by
    magnitude drops (4p^3(1-p) + 2p^4) / (4p) = 1.248% of the nonzeros,
    p = 1 - Phi(1.2) (2:4 + Squared-ReLU page §2.2-2.3 report ~1% at high
    natural sparsity)."""
    _, x, _ = synth.prefill_sqrelu(T=256, with_weight=False)
    xf = x.float().numpy()
    n = xf.size
    p = 0.5 * math.erfc(1.2 / math.sqrt(2))
    zero = (xf == 0).mean()
    assert abs(zero - (1 - p)) < 5 * math.sqrt(p * (1 - p) / n)
    mask = oracle_lib.select_nm(oracle_lib.score(xf), 2, 4)
    nz = xf != 0
    dropped = (nz & (mask == 0)).sum() / nz.sum()
    expect = (4 * p ** 3 * (1 - p) + 2 * p ** 4) / (4 * p)
    # per-block variance of the dropped count, delta method on the ratio
    blocks = nz.reshape(-1, 4).sum(1)
    d = np.maximum(blocks - 2, 0)
    sig = math.sqrt(np.var(d - expect * blocks) / len(blocks)) / (4 * p)
    assert abs(dropped - expect) < 5 * sig, (dropped, expect, sig)


# ---------------------------------------------------------------- threshold selection
def test_thresh_extremes_reduce_to_dense_and_empty(oracle_lib):
    """tau below every score keeps all (y = x W^T, the dense product); tau at
    or above the largest score keeps none (y = eta * rowsum with the shift)."""
    import synth
    x, W = synth.random_layer(3, 64, 16, seed=41)
    xf, Wf = x.float().numpy(), W.float().numpy()
    s = oracle_lib.score(xf)
    assert oracle_lib.select_thresh(s, -1.0).all()
    y = oracle_lib.linear(xf, oracle_lib.select_thresh(s, -1.0), Wf)
    np.testing.assert_allclose(y, xf.astype(np.float64) @ Wf.astype(np.float64).T, rtol=1e-12, atol=1e-12)
    eta = oracle_lib.token_mean(xf)
    s_sh = oracle_lib.score(xf, eta=eta.astype(np.float32))
    none = oracle_lib.select_thresh(s_sh, float(s_sh.max()))
    assert not none.any()
    _, rs = oracle_lib.weight_prep(Wf, 1.0)
    y0 = oracle_lib.linear(xf, none, Wf, eta=eta, rowsum=rs)
    np.testing.assert_allclose(y0, np.outer(eta, rs), rtol=1e-12, atol=1e-15)


def test_thresh_kept_share_matches_laplace_tail(oracle_lib):
    """|x| for x ~ Laplace(0, b) exceeds tau with probability exp(-tau/b):
    the kept share over 4 x 2^16 channels lies within 5 sigma of it."""
    rng = np.random.default_rng(5)
    b, tau = 0.3, 0.2
    x = rng.laplace(0.0, b, size=(4, 1 << 16)).astype(np.float32)
    kept = oracle_lib.select_thresh(oracle_lib.score(x), tau).mean()
    p = math.exp(-tau / b)
    assert abs(kept - p) < 5 * math.sqrt(p * (1 - p) / x.size)


def test_thresh_is_monotone(oracle_lib):
    rng = np.random.default_rng(6)
    s = oracle_lib.score(rng.standard_normal((8, 256)).astype(np.float32))
    lo, hi = oracle_lib.select_thresh(s, 0.3), oracle_lib.select_thresh(s, 0.9)
    assert ((hi == 1) <= (lo == 1)).all() and hi.sum() < lo.sum()


# ---------------------------------------------------------------- Amber-Pruner importance
def test_amber_2x2_closed_form(oracle_lib):
    """W = [[1, 2], [3, 4]], all kept: mean 2.5, population variance 1.25,
    each column's z = +-(1.5, 0.5)/sqrt(1.25), so sum z^2 = 2 per column."""
    W = np.array([[1, 2], [3, 4]], np.float32)
    for alpha, want in ((1.0, math.sqrt(2.0)), (2.0, 2.0), (0.5, 2.0 ** 0.25)):
        g, lo, hi = oracle_lib.amber(W, alpha, 0.0, 100.0)
        np.testing.assert_allclose(g, [want, want], rtol=1e-14)
        assert (lo, hi) == (1.0, 4.0)


def test_amber_keep_all_is_standardised_column_norm(oracle_lib):
    """0th..100th percentile keeps every weight; the importance is then the
    column norm of numpy's population z-score (np.std, ddof=0)."""
    import synth
    W = synth.outlier_weight(seed=7, n_out=96, k=40, dtype=torch.float32).numpy()
    W64 = W.astype(np.float64)
    Z = (W64 - W64.mean()) / W64.std()
    for alpha in (1.0, 0.5):
        g, _, _ = oracle_lib.amber(W, alpha, 0.0, 100.0)
        np.testing.assert_allclose(g, np.linalg.norm(Z, axis=0) ** alpha, rtol=1e-12)


def test_amber_percentiles_are_numpy_lower_order_statistics(oracle_lib):
    """The clip values equal numpy's percentile with method='lower' (the
    order statistic of rank floor(q (N-1))) for several q and sizes."""
    import synth
    for (n_out, k, seed) in ((100, 37, 8), (256, 512, 9), (1, 7, 10)):
        W = synth.outlier_weight(seed=seed, n_out=n_out, k=k, dtype=torch.float32).numpy()
        for lo_p, hi_p in ((0.5, 99.5), (0.0, 100.0), (10.0, 90.0), (37.3, 62.9)):
            _, lo, hi = oracle_lib.amber(W, 1.0, lo_p, hi_p)
            assert lo == float(np.percentile(W, lo_p, method="lower"))
            assert hi == float(np.percentile(W, hi_p, method="lower"))


def test_amber_sum_of_squared_importance_counts_kept_weights(oracle_lib):
    """With alpha = 1, sum_i g_i^2 = sum of z^2 over the kept weights = the
    number of kept weights (population variance); a sample variance, a
    missing mean subtraction or clipping in place of dropping breaks it."""
    import synth
    W = synth.outlier_weight(seed=11, n_out=200, k=64, dtype=torch.float32).numpy()
    g, lo, hi = oracle_lib.amber(W, 1.0, 0.5, 99.5)
    kept = int(((W >= lo) & (W <= hi)).sum())
    assert kept < W.size
    np.testing.assert_allclose((g ** 2).sum(), kept, rtol=1e-12)


def test_amber_drops_outliers(oracle_lib):
    """One far outlier beyond the 99.5th percentile leaves the importance as
    it was without it, except in its own column and the column of the weight
    at the new clip edge; kept in (0..100 window) it would swamp sigma."""
    rng = np.random.default_rng(12)
    W = rng.normal(0.0, 0.02, size=(400, 50)).astype(np.float32)
    g0, _, _ = oracle_lib.amber(W, 1.0, 0.0, 99.5)
    W2 = W.copy()
    W2[3, 7] = 100.0
    g2, _, hi2 = oracle_lib.amber(W2, 1.0, 0.0, 99.5)
    assert hi2 < 1.0
    rel = np.abs(g2 - g0) / g0
    assert (rel > 1e-3).sum() <= 2 and rel.max() < 2e-2
    g_all, _, _ = oracle_lib.amber(W2, 1.0, 0.0, 100.0)
    assert (g_all[np.arange(50) != 7] < 0.1 * g0[np.arange(50) != 7]).all()


def test_amber_affine_invariance(oracle_lib):
    """z-scores are unchanged by W -> a W + b with a > 0 (the percentiles
    move with W, the kept set is the same).  Weights on a 1/64 grid keep
    a = 4, b = 3 exact in float32."""
    rng = np.random.default_rng(13)
    W = (rng.integers(-64, 65, size=(60, 30)) / 64.0).astype(np.float32)
    g, lo, hi = oracle_lib.amber(W, 1.0, 0.5, 99.5)
    g2, lo2, hi2 = oracle_lib.amber((4.0 * W + 3.0).astype(np.float32), 1.0, 0.5, 99.5)
    assert (lo2, hi2) == (4 * lo + 3, 4 * hi + 3)
    np.testing.assert_allclose(g2, g, rtol=1e-12)
    # a < 0 mirrors the distribution: the kept set changes only at the ends.
    perm = rng.permutation(30)
    g3, _, _ = oracle_lib.amber(W[:, perm], 1.0, 0.5, 99.5)
    np.testing.assert_allclose(g3, g[perm], rtol=1e-12)


def test_amber_ties_at_the_clip_values_are_kept(oracle_lib):
    """Values equal to a clip value are kept (inclusive ends); a 50..50
    window keeps only the median value, so sigma = 0 and g = 0."""
    W = np.array([[0, 1, 1, 2], [2, 2, 1, 0], [1, 2, 2, 2]], np.float32)
    g, lo, hi = oracle_lib.amber(W, 1.0, 20.0, 80.0)
    # sorted: 0 0 1 1 1 1 2 2 2 2 2 2; ranks floor(.2*11)=2 -> 1, floor(.8*11)=8 -> 2
    assert (lo, hi) == (1.0, 2.0)
    kept = W[W >= 1].astype(np.float64)
    mu, sd = kept.mean(), kept.std()
    Z = np.where(W >= 1, (W - mu) / sd, 0.0)
    np.testing.assert_allclose(g, np.linalg.norm(Z, axis=0), rtol=1e-12)
    g0, lo0, hi0 = oracle_lib.amber(W, 1.0, 50.0, 50.0)
    assert lo0 == hi0 == 1.0 and not g0.any()


# ---------------------------------------------------------------- FP8 (E4M3) producer and GEMM
def _e4m3_positive_values():
    import oracle as o
    return o.e4m3_decode(np.arange(0x7F, dtype=np.uint8))  # 0 .. 448, ascending


def test_e4m3_code_table(oracle_lib):
    """Codes fixed by the format: bias 7, 3 mantissa bits, 448 the largest
    finite value, 2^-9 the smallest subnormal, 0x7F NaN."""
    cases = {448.0: 0x7E, 1.0: 0x38, 2.0 ** -9: 0x01, 2.0 ** -6: 0x08, 7 * 2.0 ** -9: 0x07,
             -2.0: 0xC0, 240.0: 0x77, 0.0: 0x00, 1.125: 0x39, 256.0: 0x78, 3.0: 0x44}
    for v, c in cases.items():
        assert int(oracle_lib.e4m3_encode([v])[0]) == c, v
        assert oracle_lib.e4m3_decode([c])[0] == v
    assert int(oracle_lib.e4m3_encode([-0.0])[0]) == 0x80
    assert np.isnan(oracle_lib.e4m3_decode([0x7F])[0]) and np.isnan(oracle_lib.e4m3_decode([0xFF])[0])
    # every finite code round-trips; saturation clamps at 448
    codes = np.array([c for c in range(256) if c & 0x7F != 0x7F], np.uint8)
    np.testing.assert_array_equal(oracle_lib.e4m3_encode(oracle_lib.e4m3_decode(codes)), codes)
    np.testing.assert_array_equal(oracle_lib.e4m3_encode([449.0, 464.0, 1e9, -500.0]), [0x7E, 0x7E, 0x7E, 0xFE])
    assert int(oracle_lib.e4m3_encode([float("nan")])[0]) == 0x7F


def test_e4m3_matches_torch_cast_on_ties_and_random(oracle_lib):
    """In range, nearest-even rounding equals torch's float8_e4m3fn cast on
    every midpoint between neighbours, one float32 step either side of it,
    and random values over the whole range."""
    pos = _e4m3_positive_values()
    mid = (pos[:-1] + pos[1:]) / 2
    m32 = mid.astype(np.float32)
    near = np.concatenate([m32, np.nextafter(m32, np.float32(0)), np.nextafter(m32, np.float32(1e9))])
    rnd = (np.random.default_rng(14).uniform(-448, 448, 100000)).astype(np.float32)
    small = (np.random.default_rng(15).uniform(-2.0 ** -5, 2.0 ** -5, 20000)).astype(np.float32)
    v = np.concatenate([near, -near, rnd, small, pos.astype(np.float32)])
    got = oracle_lib.e4m3_encode(v.astype(np.float64))
    want = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(got, want)


def test_quant_rows_fp8_bounds(oracle_lib):
    """Per-row scale amax/448: the largest magnitude of every nonzero row
    codes to +-448; relative error at most 2^-4 in the normal range and
    absolute error at most 2^-10 * scale below it; an all-zero row gets
    scale 1 and zero codes."""
    r = np.random.default_rng(16)
    W = r.normal(0, 0.02, size=(33, 200)).astype(np.float32)
    W[5] = 0.0
    codes, scale = oracle_lib.quant_rows_fp8(W)
    assert scale[5] == 1.0 and not codes[5].any()
    for o in range(33):
        if o == 5:
            continue
        assert (codes[o] & 0x7F).max() == 0x7E
        assert scale[o] == np.float32(np.abs(W[o]).max()) / np.float32(448.0)
    deq = oracle_lib.dequant_fp8(codes, scale)
    q = np.abs(W.astype(np.float64)) / scale.astype(np.float64)[:, None]
    err = np.abs(deq - W)
    normal = q >= 2.0 ** -6
    assert (err[normal] <= 2.0 ** -4 * np.abs(W[normal]) * (1 + 1e-6)).all()
    assert (err[~normal] <= 2.0 ** -10 * np.broadcast_to(scale[:, None], W.shape)[~normal] * (1 + 1e-6)).all()


def _bf16_bits(vals):
    return torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_sqrelu24_fp8_worked_row(oracle_lib):
    """z = [1 -2 3 .5 | 0 0 0 0 | 2 2 -1 2]: x = [1 0 9 .25 | 0 0 0 0 | 4 4 0 4];
    kept (0, 2), (0, 1) (all equal: the lower indices), (0, 1); amax 9,
    scale fl32(9/448); codes 9 -> 448 (0x7E), 1 -> 48 (0x64), 4 -> 192 (0x74)."""
    z = _bf16_bits([[1, -2, 3, 0.5, 0, 0, 0, 0, 2, 2, -1, 2]])
    out = oracle_lib.sqrelu24_fp8(z)
    np.testing.assert_array_equal(out["x"][0], [1, 0, 9, 0.25, 0, 0, 0, 0, 4, 4, 0, 4])
    np.testing.assert_array_equal(out["mask"][0], [1, 0, 1, 0, 1, 1, 0, 0, 1, 1, 0, 0])
    np.testing.assert_array_equal(out["pos"][0], [0, 2, 0, 1, 0, 1])
    assert out["scale"][0] == np.float32(9.0) / np.float32(448.0)
    np.testing.assert_array_equal(out["codes"][0], [0x64, 0x7E, 0, 0, 0x74, 0x74])
    zero = oracle_lib.sqrelu24_fp8(_bf16_bits([[-1.0] * 8]))
    assert zero["scale"][0] == 1.0 and not zero["codes"].any()


def test_sqrelu24_fp8_matches_generator_and_selection(oracle_lib):
    """x equals the Squared-ReLU input generator's x before its bf16 rounding;
    the mask is the plain 2:4 magnitude selection of x; every row's largest
    kept value codes to 448."""
    import synth
    z, xb, _ = synth.prefill_sqrelu(T=16, k=256, with_weight=False)
    out = oracle_lib.sqrelu24_fp8(z)
    np.testing.assert_array_equal(torch.from_numpy(out["x"]).to(torch.bfloat16).float().numpy(), xb.float().numpy())
    np.testing.assert_array_equal(out["mask"], oracle_lib.select_nm(oracle_lib.score(out["x"]), 2, 4))
    for t in range(16):
        if out["x"][t][out["mask"][t] == 1].max() > 0:
            assert out["codes"][t].max() == 0x7E


def test_linear_fp8_integer_case(oracle_lib):
    """Scales 1 and small integer codes: the FP8 GEMM is an exact integer
    matmul of the scattered kept values against the weight."""
    r = np.random.default_rng(17)
    T, k, n_out = 5, 32, 7
    xv = r.integers(0, 9, size=(T, k)).astype(np.float64)
    mask = oracle_lib.select_nm(oracle_lib.score(xv.astype(np.float32)), 2, 4)
    xk = np.where(mask == 1, xv, 0.0)
    codes = oracle_lib.e4m3_encode(xk[mask == 1].reshape(T, k // 2))
    pos = np.tile(np.arange(4), (T, k // 4))[mask == 1].reshape(T, k // 2).astype(np.uint8)
    w = r.integers(-8, 9, size=(n_out, k)).astype(np.float64)
    y = oracle_lib.linear_fp8(codes, pos, np.ones(T, np.float32), oracle_lib.e4m3_encode(w), np.ones(n_out, np.float32))
    np.testing.assert_array_equal(y, xk @ w.T)


# ---------------------------------------------------------------- R-Sparse low-rank compensation
def test_rsparse_full_rank_restores_dense(oracle_lib):
    """With every singular vector kept (r = min(n_out, k)), A B^T = W, so the
    pruned product plus the compensation is the dense product (with and
    without D-PTS, whose eta * rowsum term restores the shift)."""
    import synth
    x, W = synth.random_layer(3, 48, 40, seed=61, dtype=torch.float32)
    xf, Wf = x.numpy(), W.numpy()
    A, B = oracle_lib.rsparse_factors(Wf, 40)
    mask = oracle_lib.select_nm(oracle_lib.score(xf), 8, 16)
    dense = xf.astype(np.float64) @ Wf.astype(np.float64).T
    for use_eta in (False, True):
        eta = oracle_lib.token_mean(xf) if use_eta else None
        _, rs = oracle_lib.weight_prep(Wf, 1.0)
        y = oracle_lib.linear(xf, mask, Wf, eta=eta, rowsum=rs if use_eta else None)
        comp = oracle_lib.rsparse(xf, mask, B.astype(np.float32), A.astype(np.float32), eta=eta)
        # A, B rounded to float32: the identity holds to float32 precision of the factors
        np.testing.assert_allclose(y + comp, dense, rtol=0, atol=2e-6 * np.abs(dense).max())


def test_rsparse_exact_low_rank_weight(oracle_lib):
    """W = P Q^T of rank 4 with P, Q on a coarse grid (exact in float32):
    rank-4 compensation with A = P, B = Q is exact, and keep-all adds 0."""
    r = np.random.default_rng(62)
    P = (r.integers(-4, 5, size=(24, 4)) / 4).astype(np.float32)
    Q = (r.integers(-4, 5, size=(32, 4)) / 4).astype(np.float32)
    W = (P.astype(np.float64) @ Q.T.astype(np.float64)).astype(np.float32)
    x = (r.integers(-8, 9, size=(5, 32)) / 8).astype(np.float32)
    mask = oracle_lib.select_nm(oracle_lib.score(x), 2, 4)
    y = oracle_lib.linear(x, mask, W) + oracle_lib.rsparse(x, mask, Q, P)
    np.testing.assert_array_equal(y, x.astype(np.float64) @ W.astype(np.float64).T)
    assert not oracle_lib.rsparse(x, np.ones_like(mask), Q, P).any()
    # the factors of an exactly rank-4 W from the SVD reproduce it
    A, B = oracle_lib.rsparse_factors(W, 4)
    np.testing.assert_allclose(A @ B.T, W, atol=1e-12)


def test_rsparse_truncation_error_is_the_tail(oracle_lib):
    """The compensation's error against the dense product is the dropped
    part times the discarded singular directions: it shrinks as r grows and
    vanishes at full rank (Eckart-Young ordering of the SVD)."""
    import synth
    x, W = synth.random_layer(2, 64, 48, seed=63, dtype=torch.float32)
    xf, Wf = x.numpy(), W.numpy()
    mask = oracle_lib.select_nm(oracle_lib.score(xf), 2, 4)
    dense = xf.astype(np.float64) @ Wf.astype(np.float64).T
    base = oracle_lib.linear(xf, mask, Wf)
    errs = []
    for rank in (0, 8, 24, 48):
        if rank:
            A, B = oracle_lib.rsparse_factors(Wf, rank)
            y = base + oracle_lib.rsparse(xf, mask, B.astype(np.float32), A.astype(np.float32))
        else:
            y = base
        errs.append(np.linalg.norm(y - dense))
    assert errs[0] > errs[1] > errs[2] > errs[3] and errs[3] < 1e-5 * errs[0]


# ---------------------------------------------------------------- hybrid 2:4 (sparse/dense split)
def test_hybrid_mode_thresholds(oracle_lib):
    """The page's inference rule: > 95 % pure 2:4, 90-95 % split, < 90 % dense."""
    assert [oracle_lib.hybrid_mode(s) for s in (0.99, 0.951, 0.95, 0.92, 0.90, 0.899, 0.5)] == \
        ["2:4", "2:4", "split", "split", "split", "dense", "dense"]


def test_pick_dense_ranks_by_nonzeros_then_index(oracle_lib):
    """Hand case with ties, checked against a stable sort (numpy lexsort)."""
    nnz = np.array([3, 9, 9, 0, 5, 9, 5, 1], np.int32)
    np.testing.assert_array_equal(oracle_lib.pick_dense(nnz, 3), [1, 2, 5])
    np.testing.assert_array_equal(oracle_lib.pick_dense(nnz, 5), [1, 2, 4, 5, 6])
    r = np.random.default_rng(81)
    for _ in range(20):
        v = r.integers(0, 6, size=50).astype(np.int32)
        n = int(r.integers(0, 51))
        order = np.lexsort((np.arange(50), -v.astype(np.int64)))
        np.testing.assert_array_equal(oracle_lib.pick_dense(v, n), np.sort(order[:n]))


def test_block_nnz_counts(oracle_lib):
    x = np.array([[0, 1, 0, 2, 0, 0, 0, 0], [3, 0, 0, 0, 0, 0, -1, 0]], np.float32)
    nnz, total = oracle_lib.block_nnz(x)
    np.testing.assert_array_equal(nnz, [3, 1])
    assert total == 4


def test_hybrid_extremes_are_pure_24_and_dense(oracle_lib):
    """No dense blocks: the pure 2:4 product; every block dense: x W^T."""
    import synth
    x, W = synth.random_layer(6, 64, 24, seed=82, dtype=torch.float32, dist="sqrelu")
    xf, Wf = x.numpy(), W.numpy()
    m0, idx0, s = oracle_lib.hybrid_mask(xf, 0)
    assert len(idx0) == 0 and 0.0 <= s <= 1.0
    np.testing.assert_array_equal(m0, oracle_lib.select_nm(oracle_lib.score(xf), 2, 4))
    mall, idx, _ = oracle_lib.hybrid_mask(xf, 16)
    np.testing.assert_array_equal(idx, np.arange(16))
    y = oracle_lib.linear(xf, mall, Wf)
    np.testing.assert_allclose(y, xf.astype(np.float64) @ Wf.astype(np.float64).T, rtol=1e-12, atol=1e-14)


def test_hybrid_recovers_dropped_nonzeros_of_dense_blocks(oracle_lib):
    """Blocks with more than two nonzeros lose values under 2:4; making the
    busiest blocks dense keeps all of theirs: the dropped nonzeros never grow
    with the dense set, the dense blocks drop none, and with every block
    dense the product is exact."""
    import synth
    x, W = synth.random_layer(16, 128, 32, seed=83, dtype=torch.float32, dist="sqrelu")
    xf, Wf = x.numpy(), W.numpy()
    dense = xf.astype(np.float64) @ Wf.astype(np.float64).T
    dropped = []
    for nd in (0, 4, 8, 16, 32):
        mask, idx, _ = oracle_lib.hybrid_mask(xf, nd)
        lost = (xf != 0) & (mask == 0)
        dropped.append(int(lost.sum()))
        for b in idx:
            assert not lost[:, 4 * b:4 * b + 4].any()
    assert dropped[0] > 0 and all(a >= b for a, b in zip(dropped, dropped[1:])) and dropped[-1] == 0
    np.testing.assert_allclose(oracle_lib.linear(xf, mask, Wf), dense, rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- hybrid split of an N:M selection
def test_nm_split_worked_blocks(oracle_lib):
    """Hand-worked 4-blocks (2:4 + Squared-ReLU page §3.2 reading): the two
    kept channels with the highest scores form the 2:4 part, ties to the
    lower index; a block with one kept channel pads with the lowest dropped
    one."""
    s = np.array([[5, 3, 4, 9, 2, 2, 2, 2, 0, 0, 7, 0, 1, 8, 6, 3, 1, 0, 9, 5]], np.float32)
    m = np.array([[1, 1, 1, 0, 0, 1, 1, 1, 0, 0, 1, 0, 1, 1, 1, 1, 0, 0, 1, 0]], np.uint8)
    r = oracle_lib.nm_split(s, m, s * m, 0)
    assert r["part"].tolist() == [[1, 0, 1, 0, 0, 1, 1, 0, 0, 0, 1, 0, 0, 1, 1, 0, 0, 0, 1, 0]]
    # the last block pads with channel 0, the lowest-indexed dropped one,
    # although dropped channel 3 has the higher score
    assert r["pos"].tolist() == [[1, 0, 1, 0, 0, 1, 1, 0, 1, 0, 1, 0, 0, 1, 1, 0, 1, 0, 1, 0]]
    assert r["m_split"].tolist() == r["part"].tolist()  # no dense block


def test_nm_split_invariants_and_extremes(oracle_lib):
    """On random 8:16 and 16:32 selections: positions exactly 2 per block,
    part within the selection, top-2 property per block; every block dense
    gives back the N:M selection; a selection that already fits 2:4 is its
    own 2:4 part for any number of dense blocks."""
    rng = np.random.default_rng(7)
    for n, m in ((8, 16), (16, 32)):
        x = rng.laplace(0, 0.3, size=(6, 128)).astype(np.float32)
        s = oracle_lib.score(x)
        mask = oracle_lib.select_nm(s, n, m)
        r = oracle_lib.nm_split(s, mask, x * mask, 0)
        pos, part = r["pos"].reshape(6, 32, 4), r["part"].reshape(6, 32, 4)
        assert (pos.sum(-1) == 2).all()
        assert ((part == 1) <= (mask.reshape(6, 32, 4) == 1)).all()
        kb = mask.reshape(6, 32, 4).astype(bool)
        assert (part.sum(-1) == np.minimum(kb.sum(-1), 2)).all()
        sb = s.reshape(6, 32, 4)
        over = kb & ~part.astype(bool)
        lo = np.where(part.astype(bool), sb, np.inf).min(-1)
        hi = np.where(over, sb, -np.inf).max(-1)
        assert (lo >= hi).all()
        full = oracle_lib.nm_split(s, mask, x * mask, 32)
        np.testing.assert_array_equal(full["m_split"], mask)
    # a 2:4 selection viewed as 8:16: already 2:4-compliant
    x = rng.laplace(0, 0.3, size=(5, 64)).astype(np.float32)
    s = oracle_lib.score(x)
    m24 = oracle_lib.select_nm(s, 2, 4)
    for nd in (0, 4, 16):
        np.testing.assert_array_equal(oracle_lib.nm_split(s, m24, x * m24, nd)["m_split"], m24)


def test_nm_split_exact_when_dense_blocks_cover_the_overflow(oracle_lib):
    """The split product equals the N:M product when the dense blocks cover
    every block whose kept channels exceed 2 for some token; with fewer
    dense blocks the overflow outside them is what is dropped."""
    rng = np.random.default_rng(8)
    x = rng.laplace(0, 0.3, size=(8, 256)).astype(np.float32)
    W = rng.normal(0, 0.02, size=(40, 256)).astype(np.float32)
    s = oracle_lib.score(x)
    mask = oracle_lib.select_nm(s, 8, 16)
    y_nm = oracle_lib.linear(x, mask, W)
    over_blocks = np.unique(np.nonzero((mask.reshape(8, 64, 4).sum(-1) > 2))[1])
    r = oracle_lib.nm_split(s, mask, x * mask, 64)
    np.testing.assert_allclose(oracle_lib.linear(x, r["m_split"], W), y_nm, rtol=0, atol=1e-12)
    r0 = oracle_lib.nm_split(s, mask, x * mask, 0)
    dropped = mask.astype(bool) & ~r0["m_split"].astype(bool)
    np.testing.assert_allclose(oracle_lib.linear(x, r0["m_split"], W) + (x * dropped) @ W.T.astype(np.float64),
                               y_nm, rtol=0, atol=1e-12)
    assert len(over_blocks) > 0


def test_select_stats_worked_row(oracle_lib):
    """Two 4-blocks by magnitude (2:4): [0, 3, -1, 2] keeps 3 and 2 and drops
    the natural nonzero -1; [0, 0, 5, 0] keeps 5 and the lowest-indexed zero,
    dropping no nonzero."""
    x = np.array([[0.0, 3.0, -1.0, 2.0, 0.0, 0.0, 5.0, 0.0]])
    mask = oracle_lib.select_nm(oracle_lib.score(x), 2, 4)
    np.testing.assert_array_equal(mask, [[0, 1, 0, 1, 1, 0, 1, 0]])
    kept, dropped = oracle_lib.select_stats(x, mask)
    assert kept.tolist() == [4] and dropped.tolist() == [1]


def test_select_stats_force_dropped_closed_form(oracle_lib):
    """2:4 + Squared-ReLU page §2.3: a 4-block with k > 2 natural nonzeros
    loses k - 2 of them.  For z ~ N(-1.2, 1), max(0, z)^2 is nonzero with
    p = 1 - Phi(1.2), k ~ Binomial(4, p), so the expected number dropped per
    block is 4 p^3 (1 - p) + 2 p^4 (0.0057 here: 1.25 % of the nonzeros,
    the page's 'about 1 %' at this sparsity).  Checked within 5 sigma over
    2^20 blocks; every token keeps exactly K / 2."""
    rng = np.random.default_rng(2024)
    T, K = 1024, 4096
    x = np.maximum(rng.normal(-1.2, 1.0, size=(T, K)), 0.0) ** 2
    mask = oracle_lib.select_nm(oracle_lib.score(x), 2, 4)
    kept, dropped = oracle_lib.select_stats(x, mask)
    assert (kept == K // 2).all()
    p = 0.5 * math.erfc(1.2 / math.sqrt(2.0))
    mu = 4 * p**3 * (1 - p) + 2 * p**4
    var = 4 * p**3 * (1 - p) + 4 * p**4 - mu * mu
    n_blocks = T * K // 4
    assert abs(dropped.sum() / n_blocks - mu) <= 5.0 * math.sqrt(var / n_blocks)
    share = dropped.sum() / (x != 0).sum()
    assert 0.010 < share < 0.015
