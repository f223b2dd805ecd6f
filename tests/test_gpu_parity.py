"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Masks and indices must match bit-exactly (the oracle's selection is run on
the float32 statistics the GPU exported: eta, g, c); statistics within the
stated relative bounds of the oracle's float64 values; outputs within
relative L2 error 2e-3 (float32 output) or 1e-2 (bf16 output)."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import decode_meta8, decode_meta24, f32, rel_l2, unpack_bitmask

pytestmark = pytest.mark.gpu

TOL_F32, TOL_BF16 = 2e-3, 1e-2


@pytest.fixture(scope="module")
def sl():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import sparse_linear_b200 as m
    return m


def dev(t):
    return t.cuda().contiguous()


def layer(sl, W, cfg, alpha=0.0, importance="norm"):
    from sparse_linear_b200.layer import SparseLinear
    return SparseLinear(dev(W), cfg, alpha=alpha, importance=importance)


# ---------------------------------------------------------------- weight prep
@pytest.mark.parametrize("alpha", [0.0, 0.5, 1.0])
def test_weight_prep(sl, alpha):
    _, W = synth.random_layer(1, 520, 1000, seed=21)
    L = layer(sl, W, sl.config(), alpha)
    g_ref, rs_ref = oracle.weight_prep(W.float().numpy(), alpha)
    np.testing.assert_allclose(f32(L.g), g_ref, rtol=1e-6)
    scale = np.sqrt((W.double().numpy() ** 2).sum(1))
    assert (np.abs(f32(L.rowsum) - rs_ref) <= 1e-6 * scale + 1e-30).all()
    assert torch.equal(L.Wt.cpu(), W.t().contiguous())


# ---------------------------------------------------------------- Amber-Pruner importance
@pytest.mark.parametrize("n_out,K,lo,hi,alpha,dtype", [
    (1024, 4096, 0.5, 99.5, 1.0, torch.bfloat16),   # v-projection shape
    (4096, 11008, 0.5, 99.5, 0.5, torch.bfloat16),  # down-projection, full size
    (37, 250, 0.5, 99.5, 1.0, torch.float32),       # ragged
    (300, 1000, 10.0, 90.0, 0.5, torch.bfloat16),
    (1, 7, 0.0, 100.0, 1.0, torch.float32),         # one row, keep all
    (64, 64, 50.0, 50.0, 1.0, torch.bfloat16),      # one value kept: sigma 0, g 0
])
def test_amber_importance(sl, n_out, K, lo, hi, alpha, dtype):
    """Clip values are the exact order statistics; g within float32 rounding
    of the float64 oracle.  The workspace starts as 0xFF bytes: no zero-fill
    is needed."""
    W = synth.outlier_weight(seed=31, n_out=n_out, k=K, dtype=dtype)
    g = torch.empty(K, dtype=torch.float32, device="cuda")
    b = torch.empty(4, dtype=torch.float32, device="cuda")
    ws = torch.full((sl.as_workspace_size(sl.AS_OP_AMBER, 0, K, n_out, None),), 255, dtype=torch.uint8,
                    device="cuda")
    sl.as_weight_prep_amber(dev(W), g, alpha, lo, hi, bounds=b, workspace=ws)
    torch.cuda.synchronize()
    g_ref, v_lo, v_hi = oracle.amber(W.float().numpy(), alpha, lo, hi)
    bb = f32(b)
    assert (bb[0], bb[1]) == (v_lo, v_hi)
    np.testing.assert_allclose(f32(g), g_ref, rtol=1e-6, atol=0)


def test_amber_deterministic(sl):
    W = dev(synth.outlier_weight(seed=32))
    out = []
    for _ in range(2):
        g = torch.empty(W.shape[1], dtype=torch.float32, device="cuda")
        ws = torch.empty(sl.as_workspace_size(sl.AS_OP_AMBER, 0, W.shape[1], W.shape[0], None),
                         dtype=torch.uint8, device="cuda")
        sl.as_weight_prep_amber(W, g, workspace=ws)
        out.append(g)
    assert torch.equal(out[0], out[1])


def test_decode_amber_importance(sl):
    """Weight-aware 8:16 decode with D-PTS on the Amber-Pruner channel
    factors of a bimodal weight with outliers (the layer's g is checked
    against the oracle first, then used as the score factor)."""
    x, _, _ = synth.decode_downproj(T=4, k=4096, with_weight=False)
    W = synth.outlier_weight(seed=33, n_out=1024, k=4096)
    cfg = sl.config(score=sl.AS_SCORE_WEIGHT, sel=sl.AS_SEL_NM, n=8, m=16, dpts=True)
    L = layer(sl, W, cfg, 1.0, "amber")
    g_ref, _, _ = oracle.amber(W.float().numpy(), 1.0)
    np.testing.assert_allclose(f32(L.g), g_ref, rtol=1e-6)
    check_decode(sl, x, W, cfg, alpha=1.0, importance="amber")


# ---------------------------------------------------------------- decode
def ref_selection(sl, s, cfg):
    if cfg.sel == sl.AS_SEL_NM:
        return oracle.select_nm(s, cfg.n, cfg.m)
    if cfg.sel == sl.AS_SEL_TOPK:
        return oracle.select_topk(s, cfg.k_keep)
    if cfg.sel == sl.AS_SEL_THRESH:
        return oracle.select_thresh(s, cfg.tau)
    return np.ones_like(s, np.uint8)


def check_decode(sl, x, W, cfg, alpha=0.0, tol=None, f_override=None, eta_static=None, importance="norm"):
    """Runs as_linear_decode; checks eta, mask (bit-exact) and y."""
    T, K = x.shape
    L = layer(sl, W, cfg, alpha, importance)
    xd = dev(x)
    words = (K + 31) // 32
    mask_d = torch.zeros(T, words, dtype=torch.int32, device="cuda")
    eta_d = torch.zeros(T, dtype=torch.float32, device="cuda")
    c_d = torch.zeros(K, dtype=torch.float32, device="cuda")
    y = L.decode(xd, mask_out=mask_d, eta_out=eta_d, colnorm_out=c_d)
    torch.cuda.synchronize()
    assert sl.as_stream_status() == sl.AS_OK
    xf = x.float().numpy()
    eta32 = None
    eta64 = None
    if cfg.dpts == sl.AS_PTS_STATIC:  # S-PTS: the table itself, bit for bit
        eta32 = f32(eta_d)
        np.testing.assert_array_equal(eta32, f32(eta_static))
        eta64 = eta32.astype(np.float64)
    elif cfg.dpts:
        eta64 = oracle.token_mean(xf)
        eta32 = f32(eta_d)
        assert (np.abs(eta32 - eta64) <= 1e-6 * np.abs(xf).mean(1)).all()
    if cfg.score == sl.AS_SCORE_WEIGHT:
        f = f32(L.g)
    elif cfg.score == sl.AS_SCORE_CLACT:
        f = f32(c_d)
        np.testing.assert_allclose(f, oracle.channel_energy(xf), rtol=1e-6)
    else:
        f = None
    s = oracle.score(xf, eta=eta32, f=f)
    ref_mask = ref_selection(sl, s, cfg)
    got = unpack_bitmask(mask_d, K)
    np.testing.assert_array_equal(got, ref_mask)
    _, rs = oracle.weight_prep(W.float().numpy(), 1.0)
    ref = oracle.linear(xf, ref_mask, W.float().numpy(), eta=eta64, rowsum=rs if cfg.dpts else None)
    if tol is None:
        tol = TOL_BF16 if cfg.out_dtype == sl.AS_BF16 else TOL_F32
    err = rel_l2(f32(y), ref)
    assert err <= tol, err
    return y, got


def test_decode_tiny_layer(sl):
    """x f32 [4,256], W f32 [512,256], 2:4 magnitude, no compensation."""
    x, W = synth.tiny_layer()
    cfg = sl.config(sel=sl.AS_SEL_NM, n=2, m=4, out_dtype=sl.AS_F32)
    check_decode(sl, x, W, cfg)


@pytest.mark.parametrize("T", [1, 8, 16])
@pytest.mark.parametrize("out", ["bf16", "f32"])
def test_decode_downproj(sl, T, out):
    """Llama-7B down-projection: 8:16 weight-aware alpha=0.5 with D-PTS."""
    x, W, _ = synth.decode_downproj(T)
    cfg = sl.config(score=sl.AS_SCORE_WEIGHT, sel=sl.AS_SEL_NM, n=8, m=16, dpts=True,
                    out_dtype=sl.AS_BF16 if out == "bf16" else sl.AS_F32)
    check_decode(sl, x, W, cfg, alpha=0.5)


@pytest.mark.parametrize("T,K,n_out,n,m,score,dpts,ties", [
    (3, 1040, 264, 2, 4, 0, False, 0),
    (5, 1040, 264, 8, 16, 1, True, 0),
    (2, 2048, 520, 16, 32, 2, False, 0),
    (7, 1056, 72, 1, 4, 0, True, 3),
    (16, 512, 256, 4, 8, 1, False, 2),
    (4, 4096, 1024, 16, 32, 0, True, 2),
    (11, 8192, 136, 8, 16, 2, True, 0),
    (1, 96, 8, 2, 4, 0, False, 1),
])
def test_decode_ragged(sl, T, K, n_out, n, m, score, dpts, ties):
    x, W = synth.random_layer(T, K, n_out, seed=T * 1000 + K + m, ties=ties)
    cfg = sl.config(score=score, sel=sl.AS_SEL_NM, n=n, m=m, dpts=dpts, out_dtype=sl.AS_F32)
    check_decode(sl, x, W, cfg, alpha=0.5)


def test_decode_fp32_weights(sl):
    x, W = synth.random_layer(6, 1024, 264, seed=5, dtype=torch.float32)
    cfg = sl.config(score=sl.AS_SCORE_WEIGHT, sel=sl.AS_SEL_NM, n=8, m=16, dpts=True, out_dtype=sl.AS_F32)
    check_decode(sl, x, W, cfg, alpha=1.0)


def test_decode_block_topk(sl):
    """Llama3.1-8B block at one token: per-layer exact top-k keep fraction and
    weight-aware exponent."""
    blk = synth.decode_block()
    for ly in blk["layers"]:
        K = ly["k"]
        kk = int(math.floor(ly["keep_frac"] * K + 0.5))
        cfg = sl.config(score=sl.AS_SCORE_WEIGHT, sel=sl.AS_SEL_TOPK, k_keep=kk)
        check_decode(sl, blk["x"][ly["x_key"]], ly["W"], cfg, alpha=ly["alpha"])


@pytest.mark.parametrize("kk", [0, 1, 100, 1023, 1024])
def test_decode_topk_edges(sl, kk):
    x, W = synth.random_layer(3, 1024, 64, seed=kk, ties=2)
    cfg = sl.config(score=sl.AS_SCORE_MAG, sel=sl.AS_SEL_TOPK, k_keep=kk, dpts=True, out_dtype=sl.AS_F32)
    check_decode(sl, x, W, cfg)


def test_decode_keep_all_is_dense(sl):
    x, W = synth.random_layer(4, 1024, 136, seed=9)
    cfg = sl.config(sel=sl.AS_SEL_ALL, out_dtype=sl.AS_F32)
    y, mask = check_decode(sl, x, W, cfg)
    assert mask.all()


def test_decode_plan_stable_across_calls(sl):
    """Workspace sizes and launch counts asked for up front stay valid after
    calls of other token counts have run (the plan must not depend on which
    calls ran before it)."""
    x, W, _ = synth.decode_downproj(16)
    cfg = sl.config(score=sl.AS_SCORE_WEIGHT, sel=sl.AS_SEL_NM, n=8, m=16, dpts=True)
    from sparse_linear_b200.layer import SparseLinear, workspace
    L = SparseLinear(dev(W), cfg, alpha=0.5)
    Ts = (1, 8, 16, 2, 4)
    sizes = {T: sl.as_workspace_size(sl.AS_OP_DECODE, T, 11008, 4096, cfg) for T in Ts}
    launches = {T: sl.as_decode_launches(T, 11008, 4096, sl.AS_BF16, cfg) for T in Ts}
    wss = {T: workspace(sizes[T], "cuda") for T in Ts}
    xd = dev(x)
    for _ in range(2):
        for T in Ts:
            y = torch.empty(T, 4096, dtype=torch.bfloat16, device="cuda")
            sl.as_linear_decode(xd[:T], L.Wt, cfg, y, g=L.g, rowsum=L.rowsum, workspace=wss[T])
            assert sl.as_workspace_size(sl.AS_OP_DECODE, T, 11008, 4096, cfg) == sizes[T]
            assert sl.as_decode_launches(T, 11008, 4096, sl.AS_BF16, cfg) == launches[T]
    torch.cuda.synchronize()
    assert sl.as_stream_status() == sl.AS_OK


def test_decode_repeated_and_graph(sl):
    """Many calls in a row, eagerly and replayed from a CUDA graph, give the
    same result as the first (the workspace's counters return to zero after
    every call), with no timeout recorded."""
    x, W, _ = synth.decode_downproj(16)
    cfg = sl.config(score=sl.AS_SCORE_WEIGHT, sel=sl.AS_SEL_NM, n=8, m=16, dpts=True)
    L = layer(sl, W, cfg, 0.5)
    xd = dev(x)
    y0 = L.decode(xd).clone()
    for _ in range(20):
        assert torch.equal(L.decode(xd), y0)
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        L.decode(xd)
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s):
            yg = L.decode(xd)
    for _ in range(10):
        g.replay()
    torch.cuda.synchronize()
    assert torch.equal(yg, y0)
    assert sl.as_stream_status() == sl.AS_OK


def test_decode_deterministic(sl):
    x, W, _ = synth.decode_downproj(8)
    cfg = sl.config(score=sl.AS_SCORE_WEIGHT, sel=sl.AS_SEL_NM, n=8, m=16, dpts=True)
    L = layer(sl, W, cfg, 0.5)
    xd = dev(x)
    y1 = L.decode(xd).clone()
    y2 = L.decode(xd).clone()
    assert torch.equal(y1, y2)


# ---------------------------------------------------------------- prefill
def check_select_24(sl, x, bufs, rows):
    """2:4 select outputs on the given rows: bitmask, compact values, metadata."""
    T, K = x.shape
    xf = x.float().numpy()[rows]
    ref_mask = oracle.select_nm(oracle.score(xf), 2, 4)
    got = unpack_bitmask(bufs["bitmask"], K)[rows]
    np.testing.assert_array_equal(got, ref_mask)
    vals, pos = oracle.compress_nm(xf, ref_mask, 2, 4)
    np.testing.assert_array_equal(f32(bufs["x_compact"])[rows], vals)  # exact: x is bf16, no shift
    meta = decode_meta24(bufs["meta24"], T, K)[rows]
    np.testing.assert_array_equal(meta.reshape(len(rows), -1), pos.astype(np.int64))
    return ref_mask


# (300, 1024, 520), (128, ...), (5, ...): odd number of 128-row tiles, one SM
# per tile; the others run on CTA pairs, including a ragged weight tail that
# leaves the second CTA's weight box wholly outside W (512, 1024, 264).
@pytest.mark.parametrize("T,K,n_out", [(300, 1024, 520), (128, 14336, 256), (5, 256, 64), (1000, 2048, 1024),
                                       (256, 512, 200), (512, 1024, 264), (512, 4096, 768)])
def test_prefill_24(sl, T, K, n_out):
    x, W = synth.random_layer(T, K, n_out, seed=T + K, dist="sqrelu")
    for out in (sl.AS_BF16, sl.AS_F32):
        cfg = sl.config(sel=sl.AS_SEL_NM, n=2, m=4, out_dtype=out)
        L = layer(sl, W, cfg)
        y, bufs = L.prefill(dev(x))
        torch.cuda.synchronize()
        assert sl.as_stream_status() == sl.AS_OK
        rows = np.arange(T)
        mask = check_select_24(sl, x, bufs, rows)
        ref = oracle.linear(x.float().numpy(), mask, W.float().numpy())
        err = rel_l2(f32(y), ref)
        assert err <= (TOL_BF16 if out == sl.AS_BF16 else TOL_F32), err


def test_prefill_24_partial_wave(sl):
    """80 CTA-pair tiles on 74 pairs: a partial second wave (the tiles of
    output columns [2304, 2560) in row blocks 2..7); sampled rows in those
    blocks and in others, every column."""
    T, K, n_out = 2048, 512, 2560
    x, W = synth.random_layer(T, K, n_out, seed=77, dist="sqrelu")
    cfg = sl.config(sel=sl.AS_SEL_NM, n=2, m=4)
    L = layer(sl, W, cfg)
    y, bufs = L.prefill(dev(x))
    torch.cuda.synchronize()
    assert sl.as_stream_status() == sl.AS_OK
    rows = np.array([3, 255, 600, 1000, 1300, 1790, 2047])
    mask = check_select_24(sl, x, bufs, rows)
    ref = oracle.linear(x.float().numpy()[rows], mask, W.float().numpy())
    assert rel_l2(f32(y)[rows], ref) <= TOL_BF16
    assert rel_l2(f32(y)[rows][:, 2304:], ref[:, 2304:]) <= TOL_BF16


def test_prefill_24_full_size(sl):
    """FFN down-projection at prefill: squared-ReLU activations [4096, 14336],
    2:4 by magnitude on the sparse tensor-core path; sampled rows."""
    _, x, W = synth.prefill_sqrelu()
    cfg = sl.config(sel=sl.AS_SEL_NM, n=2, m=4)
    L = layer(sl, W, cfg)
    y, bufs = L.prefill(dev(x))
    torch.cuda.synchronize()
    assert sl.as_stream_status() == sl.AS_OK
    rows = np.array([0, 1, 127, 128, 1000, 2047, 2048, 3071, 4094, 4095])
    mask = check_select_24(sl, x, bufs, rows)
    ref = oracle.linear(x.float().numpy()[rows], mask, W.float().numpy())
    assert rel_l2(f32(y)[rows], ref) <= TOL_BF16
    # property over the whole output: the share of natural nonzeros that the
    # 2:4 enforcement drops matches its closed form (2:4 + Squared-ReLU page, 2.3)
    nzm = unpack_bitmask(bufs["bitmask"], x.shape[1])
    nz = x.float().numpy() != 0
    dropped = (nz & (nzm == 0)).sum() / nz.sum()
    p = 0.5 * math.erfc(1.2 / math.sqrt(2))
    assert abs(dropped - (4 * p ** 3 * (1 - p) + 2 * p ** 4) / (4 * p)) < 2e-4
    # the same counts per token from as_select_stats, exact against the oracle
    kept = torch.empty(x.shape[0], dtype=torch.int32, device="cuda")
    nzd = torch.empty_like(kept)
    sl.as_select_stats(dev(x), bufs["bitmask"], kept, nzd)
    torch.cuda.synchronize()
    ref_k, ref_d = oracle.select_stats(x.float().numpy(), nzm)
    np.testing.assert_array_equal(kept.cpu().numpy(), ref_k)
    np.testing.assert_array_equal(nzd.cpu().numpy(), ref_d)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_select_stats_ragged(sl, dtype):
    """Kept and natural-nonzero-dropped counts for an arbitrary keep mask
    (K = 1000: a partial last keep word), float32 and bf16 activations with
    exact zeros, against the oracle's counts."""
    T, K = 7, 1000
    rng = np.random.default_rng(11)
    x64 = rng.normal(size=(T, K)) * (rng.random((T, K)) < 0.3)
    mask = (rng.random((T, K)) < 0.4).astype(np.uint8)
    words = np.zeros((T, (K + 31) // 32), np.uint32)
    for t in range(T):
        for c in np.flatnonzero(mask[t]):
            words[t, c // 32] |= np.uint32(1) << np.uint32(c % 32)
    x = torch.from_numpy(x64).to(dtype)
    kept = torch.empty(T, dtype=torch.int32, device="cuda")
    nzd = torch.empty_like(kept)
    sl.as_select_stats(dev(x), torch.from_numpy(words.view(np.int32)).cuda(), kept, nzd)
    torch.cuda.synchronize()
    ref_k, ref_d = oracle.select_stats(x.float().numpy(), mask)
    np.testing.assert_array_equal(kept.cpu().numpy(), ref_k)
    np.testing.assert_array_equal(nzd.cpu().numpy(), ref_d)


def check_prefill_masked(sl, xs, W, cfg, alpha=0.0, rows=None, eta_static=None):
    """Runs select + prefill over a list of batches (VAR running state
    carried); checks statistics, masks and outputs on `rows`."""
    L = layer(sl, W, cfg, alpha)
    T, K = xs[0].shape
    running = torch.zeros(T, dtype=torch.float32, device="cuda")
    run_ref = None
    rows = np.arange(T) if rows is None else rows
    for b, x in enumerate(xs):
        y, bufs = L.prefill(dev(x), running_var=running, first_batch=(b == 0))
        torch.cuda.synchronize()
        assert sl.as_stream_status() == sl.AS_OK
        xf = x.float().numpy()
        if cfg.score == sl.AS_SCORE_CLACT:
            f = f32(bufs["colnorm"])
            np.testing.assert_allclose(f, oracle.channel_energy(xf), rtol=1e-6)
        elif cfg.score == sl.AS_SCORE_WEIGHT:
            f = f32(L.g)
        else:
            f = None
        eta32 = f32(bufs["eta"])[rows] if cfg.dpts else None
        if cfg.dpts == sl.AS_PTS_STATIC:
            np.testing.assert_array_equal(eta32, f32(eta_static)[rows])
            eta64 = eta32.astype(np.float64)
        else:
            eta64 = oracle.token_mean(xf[rows]) if cfg.dpts else None
            if cfg.dpts:
                assert (np.abs(eta32 - eta64) <= 1e-6 * np.abs(xf[rows]).mean(1)).all()
        s = oracle.score(xf[rows], eta=eta32, f=f)
        ref_mask = ref_selection(sl, s, cfg)
        np.testing.assert_array_equal(unpack_bitmask(bufs["bitmask"], K)[rows], ref_mask)
        nu = None
        if cfg.var:
            st = oracle.var_scale(xf[rows], ref_mask, None if run_ref is None else run_ref[rows],
                                  cfg.var_momentum, cfg.var_eps)
            if run_ref is None:
                run_ref = np.zeros(T)
            run_ref[rows] = st["running"]
            np.testing.assert_allclose(f32(bufs["var_dense"])[rows], st["var_dense"], rtol=1e-6)
            np.testing.assert_allclose(f32(bufs["var_kept"])[rows], st["var_kept"], rtol=1e-6)
            np.testing.assert_allclose(f32(running)[rows], st["running"], rtol=1e-5)
            np.testing.assert_allclose(f32(bufs["nu"])[rows], st["nu"], rtol=1e-5)
            nu = st["nu"]
        _, rs = oracle.weight_prep(W.float().numpy(), 1.0)
        ref = oracle.linear(xf[rows], ref_mask, W.float().numpy(), eta=eta64,
                            rowsum=rs if cfg.dpts else None, nu=nu)
        tol = TOL_BF16 if cfg.out_dtype == sl.AS_BF16 else TOL_F32
        err = rel_l2(f32(y)[rows], ref)
        assert err <= tol, (b, err)


def test_prefill_clact_var_small(sl):
    T, K, n_out = 264, 1024, 264
    xs = [synth.random_layer(T, K, n_out, seed=100 + b, dist="t3")[0] for b in range(3)]
    W = synth.random_layer(1, K, n_out, seed=99)[1]
    cfg = sl.config(score=sl.AS_SCORE_CLACT, sel=sl.AS_SEL_NM, n=16, m=32, var=True)
    check_prefill_masked(sl, xs, W, cfg)


@pytest.mark.parametrize("n,m,score,dpts", [(8, 16, 1, True), (4, 8, 0, False), (1, 4, 2, False)])
def test_prefill_dense_path(sl, n, m, score, dpts):
    T, K, n_out = 200, 2048, 392
    x, W = synth.random_layer(T, K, n_out, seed=n * m, dist="laplace")
    cfg = sl.config(score=score, sel=sl.AS_SEL_NM, n=n, m=m, dpts=dpts, out_dtype=sl.AS_F32)
    check_prefill_masked(sl, [x], W, cfg, alpha=0.5)


def test_prefill_topk_and_all(sl):
    T, K, n_out = 130, 1024, 256
    x, W = synth.random_layer(T, K, n_out, seed=3)
    check_prefill_masked(sl, [x], W, sl.config(sel=sl.AS_SEL_TOPK, k_keep=600))
    check_prefill_masked(sl, [x], W, sl.config(sel=sl.AS_SEL_ALL, out_dtype=sl.AS_F32))


def test_prefill_clact_var_eight_batches(sl):
    """The CLACT + VAR 16:32 chain over all eight seeded batches (momentum
    0.9) on a smaller problem of the same distributions, x [512, 2048] and W
    [1024, 2048]: every batch's masks, variances, running variance, nu and y
    against the oracle, whose running state is carried through its own
    chain (float64), not taken from the GPU."""
    W = synth.prefill_clact_weight(k=2048, n_out=1024)
    xs = [synth.prefill_clact_batch(b, T=512, k=2048) for b in range(8)]
    cfg = sl.config(score=sl.AS_SCORE_CLACT, sel=sl.AS_SEL_NM, n=16, m=32, var=True)
    check_prefill_masked(sl, xs, W, cfg)
    cfg32 = sl.config(score=sl.AS_SCORE_CLACT, sel=sl.AS_SEL_NM, n=16, m=32, var=True, out_dtype=sl.AS_F32)
    check_prefill_masked(sl, xs, W, cfg32)


# T = 256: an even number of 128-row tiles (CTA-pair kernels); T = 300: odd
# (one-SM kernels)
@pytest.mark.parametrize("T,case", [(256, "2:4 D-PTS"), (300, "2:4 D-PTS"), (256, "8:16 D-PTS"),
                                    (300, "8:16 D-PTS"), (256, "2:4 S-PTS"), (300, "top-k D-PTS")])
def test_prefill_shift_float32_residual_pass(sl, T, case):
    """Float32 output with a token shift: the shifted kept values are not
    bf16 numbers, so they enter the tensor cores as bf16 hi + lo (a second
    pass over K with the residual operand) and y holds the float32
    tolerance against the oracle."""
    K, n_out = 1024, 264
    x, W = synth.random_layer(T, K, n_out, seed=T + len(case), dist="sqrelu" if "2:4" in case else "laplace")
    eta_static = None
    if case == "2:4 D-PTS":
        cfg = sl.config(sel=sl.AS_SEL_NM, n=2, m=4, dpts=True, out_dtype=sl.AS_F32)
    elif case == "8:16 D-PTS":
        cfg = sl.config(score=sl.AS_SCORE_WEIGHT, sel=sl.AS_SEL_NM, n=8, m=16, dpts=True, out_dtype=sl.AS_F32)
    elif case == "2:4 S-PTS":
        eta_static = dev(torch.from_numpy((0.05 + 0.01 * np.cos(np.arange(T))).astype(np.float32)))
        cfg = sl.config(sel=sl.AS_SEL_NM, n=2, m=4, dpts=sl.AS_PTS_STATIC, eta_static=eta_static,
                        out_dtype=sl.AS_F32)
    else:
        cfg = sl.config(sel=sl.AS_SEL_TOPK, k_keep=400, dpts=True, out_dtype=sl.AS_F32)
    check_prefill_masked(sl, [x], W, cfg, alpha=0.5, eta_static=eta_static)


def test_prefill_residual_pass_is_used(sl):
    """The float32 D-PTS prefill with the residual operand is closer to the
    oracle than the same call without it (one bf16 pass), which shows the
    second pass adds the residual rather than leaving it out."""
    T, K, n_out = 256, 2048, 392
    x, W = synth.random_layer(T, K, n_out, seed=5, dist="laplace")
    cfg = sl.config(sel=sl.AS_SEL_NM, n=8, m=16, dpts=True, out_dtype=sl.AS_F32)
    L = layer(sl, W, cfg)
    xd = dev(x)
    bufs = L.select_buffers(T)
    assert "x_masked_lo" in bufs
    L.select(xd, bufs)
    y2 = L.prefill_from(bufs, T)
    one = {k: v for k, v in bufs.items() if k != "x_masked_lo"}
    y1 = L.prefill_from(one, T)
    torch.cuda.synchronize()
    xf = x.float().numpy()
    eta64 = oracle.token_mean(xf)
    s = oracle.score(xf, eta=f32(bufs["eta"]))
    mask = oracle.select_nm(s, 8, 16)
    _, rs = oracle.weight_prep(W.float().numpy(), 1.0)
    ref = oracle.linear(xf, mask, W.float().numpy(), eta=eta64, rowsum=rs)
    e2, e1 = rel_l2(f32(y2), ref), rel_l2(f32(y1), ref)
    assert e2 <= TOL_F32 and e2 < 0.25 * e1, (e2, e1)


def test_prefill_clact_var_full_size(sl):
    """CLACT + VAR at 16:32 on [8192, 8192] (masked dense tensor-core GEMM):
    two of the eight batches, sampled rows."""
    W = synth.prefill_clact_weight()
    xs = [synth.prefill_clact_batch(b) for b in range(2)]
    cfg = sl.config(score=sl.AS_SCORE_CLACT, sel=sl.AS_SEL_NM, n=16, m=32, var=True)
    rows = np.array([0, 127, 128, 4097, 8190, 8191])
    check_prefill_masked(sl, xs, W, cfg, rows=rows)


# ---------------------------------------------------------------- threshold and S-PTS
def _tau_for_share(sl, x, W, alpha, share, eta=None):
    """A threshold that keeps about `share` of the scores (a calibration
    stand-in: the quantile of the scores of this input)."""
    from sparse_linear_b200.layer import SparseLinear
    g = f32(SparseLinear(dev(W), sl.config(), alpha=alpha).g)
    s = oracle.score(x.float().numpy(), eta=eta, f=g)
    return float(np.quantile(s, 1.0 - share))


@pytest.mark.parametrize("T,dpts", [(1, 1), (2, 0), (8, 1), (13, 0)])
def test_decode_thresh(sl, T, dpts):
    x, W, _ = synth.decode_downproj(T)
    eta = oracle.token_mean(x.float().numpy()).astype(np.float32) if dpts else None
    tau = _tau_for_share(sl, x, W, 0.5, 0.5, eta)
    cfg = sl.config(score=sl.AS_SCORE_WEIGHT, sel=sl.AS_SEL_THRESH, tau=tau, dpts=dpts)
    y, got = check_decode(sl, x, W, cfg, alpha=0.5)
    assert 0.3 < got.mean() < 0.7


def test_decode_thresh_fp32_weights(sl):
    x, W = synth.random_layer(3, 1024, 264, seed=31, dtype=torch.float32)
    cfg = sl.config(sel=sl.AS_SEL_THRESH, tau=0.4, out_dtype=sl.AS_F32)
    check_decode(sl, x, W, cfg)


@pytest.mark.parametrize("T", [1, 2, 8, 16])
def test_decode_static_pts(sl, T):
    """S-PTS: eta from a calibrated table (here: the means of another batch
    of the same distribution), 8:16 weight-aware."""
    x, W, _ = synth.decode_downproj(T)
    calib = synth.decode_downproj(T, seed=91, with_weight=False)[0]
    eta_static = dev(torch.from_numpy(oracle.token_mean(calib.float().numpy()).astype(np.float32)))
    cfg = sl.config(score=sl.AS_SCORE_WEIGHT, sel=sl.AS_SEL_NM, n=8, m=16, dpts=sl.AS_PTS_STATIC,
                    eta_static=eta_static)
    check_decode(sl, x, W, cfg, alpha=0.5, eta_static=eta_static)


def test_prefill_thresh_and_static_pts(sl):
    T, K, n_out = 200, 2048, 392
    x, W = synth.random_layer(T, K, n_out, seed=57, dist="laplace")
    eta_static = dev(torch.from_numpy((0.01 * np.sin(np.arange(T))).astype(np.float32)))
    cfg = sl.config(sel=sl.AS_SEL_THRESH, tau=0.25, dpts=sl.AS_PTS_STATIC, eta_static=eta_static,
                    out_dtype=sl.AS_F32)
    check_prefill_masked(sl, [x], W, cfg, eta_static=eta_static)
    cfg2 = sl.config(sel=sl.AS_SEL_NM, n=8, m=16, dpts=sl.AS_PTS_STATIC, eta_static=eta_static,
                     out_dtype=sl.AS_F32)
    check_prefill_masked(sl, [x], W, cfg2, eta_static=eta_static)


# ---------------------------------------------------------------- FP8 2:4 prefill
def _fp8_weight(sl, W):
    n_out, K = W.shape
    Wq = torch.empty(n_out, K, dtype=torch.uint8, device="cuda")
    ws = torch.empty(n_out, dtype=torch.float32, device="cuda")
    sl.as_weight_quant_fp8(dev(W), Wq, ws)
    return Wq, ws


def _fp8_produce(sl, z):
    T, K = z.shape
    x8 = torch.empty(T, K // 2, dtype=torch.uint8, device="cuda")
    meta = torch.full((sl.as_meta8_words(T, K),), 0x7777, dtype=torch.int32, device="cuda")
    xs = torch.empty(T, dtype=torch.float32, device="cuda")
    bm = torch.empty(T, K // 32, dtype=torch.int32, device="cuda")
    sl.as_select_sqrelu24_fp8(dev(z), x8, meta, xs, bitmask=bm)
    return x8, meta, xs, bm


@pytest.mark.parametrize("n_out,K,dtype", [(264, 1024, torch.bfloat16), (64, 272, torch.float32),
                                           (4096, 14336, torch.bfloat16)])
def test_fp8_weight_quant(sl, n_out, K, dtype):
    """Codes and row scales bit-exact against the oracle (one IEEE division
    and one round-to-nearest-even conversion on both sides)."""
    _, W = synth.random_layer(1, K, n_out, seed=51, dtype=dtype)
    W[3] = 0  # an all-zero row: scale 1, zero codes
    Wq, ws = _fp8_weight(sl, W)
    torch.cuda.synchronize()
    codes, scale = oracle.quant_rows_fp8(W.float().numpy())
    np.testing.assert_array_equal(ws.cpu().numpy(), scale)
    np.testing.assert_array_equal(Wq.cpu().numpy(), codes)


@pytest.mark.parametrize("T,K", [(1, 64), (300, 1024), (129, 832)])
def test_fp8_producer(sl, T, K):
    """Fused Squared-ReLU + 2:4 + FP8: codes, scales, bitmask and positions
    bit-exact; padding blocks (channels past K, tokens past T up to the pair
    tile) hold positions (0, 1)."""
    z, _, _ = synth.prefill_sqrelu(T=T, k=K, with_weight=False)
    z[0, :8] = torch.tensor([1, -2, 3, 0.5, 2, 2, -1, 2], dtype=torch.bfloat16)
    if T > 2:
        z[2] = -1  # all-zero row
    x8, meta, xs, bm = _fp8_produce(sl, z)
    torch.cuda.synchronize()
    ref = oracle.sqrelu24_fp8(z)
    np.testing.assert_array_equal(xs.cpu().numpy(), ref["scale"])
    np.testing.assert_array_equal(x8.cpu().numpy(), ref["codes"])
    np.testing.assert_array_equal(unpack_bitmask(bm, K), ref["mask"])
    T_pad = (T + 255) // 256 * 256
    pos = decode_meta8(meta, T, K, T_pad)
    want = ref["pos"].reshape(T, K // 4, 2).astype(np.int64)
    np.testing.assert_array_equal(pos[:T, :K // 4], want)
    assert (pos[:, K // 4:] == [0, 1]).all() and (pos[T:] == [0, 1]).all()


def check_fp8_gemm(sl, T, K, n_out, out_dtype, seed=52, rows=None):
    z, _, W = synth.prefill_sqrelu(T=T, k=K, n_out=n_out, seed=seed)
    x8, meta, xs, _ = _fp8_produce(sl, z)
    Wq, ws = _fp8_weight(sl, W)
    y = torch.empty(T, n_out, dtype=out_dtype, device="cuda")
    sl.as_linear_prefill_fp8(x8, meta, xs, Wq, ws, y)
    torch.cuda.synchronize()
    assert sl.as_stream_status() == sl.AS_OK
    ref_x = oracle.sqrelu24_fp8(z if rows is None else z[rows])
    np.testing.assert_array_equal(x8.cpu().numpy()[rows] if rows is not None else x8.cpu().numpy(), ref_x["codes"])
    codes_w, scale_w = oracle.quant_rows_fp8(W.float().numpy())
    ref = oracle.linear_fp8(ref_x["codes"], ref_x["pos"], ref_x["scale"], codes_w, scale_w)
    got = f32(y) if rows is None else f32(y)[rows]
    tol = TOL_BF16 if out_dtype == torch.bfloat16 else TOL_F32
    err = rel_l2(got, ref)
    assert err <= tol, err
    return err


@pytest.mark.parametrize("T,K,n_out,out", [
    (256, 512, 256, torch.float32),     # one pair tile, two K blocks
    (300, 1024, 264, torch.bfloat16),   # ragged T and n_out
    (384, 832, 512, torch.float32),     # odd number of 128-row tiles, ragged last K block
    (512, 4096, 768, torch.bfloat16),   # several tiles per CTA pair
])
def test_fp8_gemm(sl, T, K, n_out, out):
    check_fp8_gemm(sl, T, K, n_out, out)


def test_fp8_gemm_full_size(sl):
    """The Squared-ReLU down-projection at full size (T 4096, K 14336,
    n_out 4096), checked on sampled rows spread over every row tile."""
    rows = np.arange(5, 4096, 61)
    check_fp8_gemm(sl, 4096, 14336, 4096, torch.bfloat16, seed=3, rows=rows)


# ---------------------------------------------------------------- R-Sparse compensation (decode)
def _bf16r(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16)


@pytest.mark.parametrize("T,K,n_out,r,dpts,svd", [
    (1, 1024, 512, 64, True, True),
    (5, 1008, 264, 32, False, True),
    (16, 2048, 1024, 128, True, True),
    (8, 11008, 4096, 64, True, False),   # the down-projection, random factors
])
def test_rsparse_decode(sl, T, K, n_out, r, dpts, svd):
    """The decode call (float32 out) followed by the compensation against the
    oracle's pruned product plus its float64 compensation, on the same
    bf16-rounded factors (from numpy's SVD of W, or random at full size)."""
    x, W = synth.random_layer(T, K, n_out, seed=71)
    cfg = sl.config(score=sl.AS_SCORE_WEIGHT, sel=sl.AS_SEL_NM, n=8, m=16, dpts=dpts, out_dtype=sl.AS_F32)
    L = layer(sl, W, cfg, 0.5)
    if svd:
        U, S, Vh = np.linalg.svd(W.double().numpy(), full_matrices=False)
        A, B = _bf16r(U[:, :r] * S[:r]), _bf16r(Vh[:r, :].T)
    else:
        rng = np.random.default_rng(72)
        A, B = _bf16r(rng.normal(0, 0.05, (n_out, r))), _bf16r(rng.normal(0, 0.02, (K, r)))
    xd = dev(x)
    mask_d = torch.zeros(T, (K + 31) // 32, dtype=torch.int32, device="cuda")
    eta_d = torch.zeros(T, dtype=torch.float32, device="cuda")
    y = L.decode(xd, mask_out=mask_d, eta_out=eta_d)
    ws = torch.empty(sl.as_rsparse_workspace(T, K, r), dtype=torch.uint8, device="cuda")
    sl.as_rsparse_decode(xd, mask_d, dev(B), dev(A), y, eta=eta_d if dpts else None, workspace=ws)
    torch.cuda.synchronize()
    assert sl.as_stream_status() == sl.AS_OK
    xf, Wf = x.float().numpy(), W.float().numpy()
    mask = unpack_bitmask(mask_d, K)
    eta32 = f32(eta_d) if dpts else None
    s = oracle.score(xf, eta=eta32, f=f32(L.g))
    np.testing.assert_array_equal(mask, oracle.select_nm(s, 8, 16))
    eta64 = oracle.token_mean(xf) if dpts else None
    _, rs = oracle.weight_prep(Wf, 1.0)
    ref = oracle.linear(xf, mask, Wf, eta=eta64, rowsum=rs if dpts else None)
    comp = oracle.rsparse(xf, mask, B.float().numpy(), A.float().numpy(), eta=eta64)
    assert rel_l2(f32(y), ref + comp) <= TOL_F32
    # the compensation itself, isolated from the pruned product
    y2 = L.decode(xd)
    y0 = y2.clone()
    sl.as_rsparse_decode(xd, mask_d, dev(B), dev(A), y2, eta=eta_d if dpts else None, workspace=ws)
    torch.cuda.synchronize()
    assert rel_l2(f32(y2) - f32(y0), comp) <= TOL_F32


# (T, K, n_out, r, selection, shift, out, factors): even tile counts run the
# CTA-pair kernels, T = 300 the one-SM kernels; 2:4 runs the sparse GEMM with
# dense R-Sparse K blocks, the others the masked dense GEMM
@pytest.mark.parametrize("T,K,n_out,r,sel,dpts,out,svd", [
    (256, 1024, 264, 64, "2:4", True, "f32", True),
    (300, 1024, 264, 128, "8:16", True, "f32", True),
    (300, 2048, 520, 64, "2:4", False, "bf16", False),
    (512, 1024, 1024, 64, "top-k", False, "f32", True),
    (256, 1024, 264, 128, "2:4", False, "f32", True),
])
def test_rsparse_prefill(sl, T, K, n_out, r, sel, dpts, out, svd):
    """Prefill with R-Sparse: the selection bit-exact, y against the oracle's
    pruned product plus its float64 compensation with the same bf16 factors
    (numpy SVD of W, or random)."""
    x, W = synth.random_layer(T, K, n_out, seed=81 + T, dist="sqrelu" if sel == "2:4" else "laplace")
    odt = sl.AS_F32 if out == "f32" else sl.AS_BF16
    if sel == "2:4":
        cfg = sl.config(sel=sl.AS_SEL_NM, n=2, m=4, dpts=dpts, out_dtype=odt)
    elif sel == "8:16":
        cfg = sl.config(score=sl.AS_SCORE_WEIGHT, sel=sl.AS_SEL_NM, n=8, m=16, dpts=dpts, out_dtype=odt)
    else:
        cfg = sl.config(sel=sl.AS_SEL_TOPK, k_keep=K // 3, dpts=dpts, out_dtype=odt)
    L = layer(sl, W, cfg, 0.5)
    if svd:
        A64, B64 = oracle.rsparse_factors(W, r)
        A, B = _bf16r(A64), _bf16r(B64)
    else:
        rng = np.random.default_rng(83)
        A, B = _bf16r(rng.normal(0, 0.05, (n_out, r))), _bf16r(rng.normal(0, 0.02, (K, r)))
    y, bufs = L.prefill_rsparse(dev(x), dev(B), dev(A))
    torch.cuda.synchronize()
    assert sl.as_stream_status() == sl.AS_OK
    xf, Wf = x.float().numpy(), W.float().numpy()
    eta32 = f32(bufs["eta"]) if dpts else None
    f = f32(L.g) if sel == "8:16" else None
    mask = ref_selection(sl, oracle.score(xf, eta=eta32, f=f), cfg)
    np.testing.assert_array_equal(unpack_bitmask(bufs["bitmask"], K), mask)
    eta64 = oracle.token_mean(xf) if dpts else None
    _, rs = oracle.weight_prep(Wf, 1.0)
    ref = oracle.linear(xf, mask, Wf, eta=eta64, rowsum=rs if dpts else None)
    comp = oracle.rsparse(xf, mask, B.float().numpy(), A.float().numpy(), eta=eta64)
    err = rel_l2(f32(y), ref + comp)
    assert err <= (TOL_F32 if out == "f32" else TOL_BF16), err
    if out == "f32":  # the compensation is really in y: without it the error is far larger
        assert rel_l2(ref, ref + comp) > 20 * err


def test_rsparse_prefill_full_rank_restores_dense(sl):
    """Full-rank factors (r = K = 128): W = A B^T up to the factors' bf16
    rounding, so the compensated prefill of a 2:4 selection gives the dense
    product of the unpruned input."""
    T, K, n_out, r = 256, 128, 256, 128
    x, W = synth.random_layer(T, K, n_out, seed=91, dist="laplace")
    cfg = sl.config(sel=sl.AS_SEL_NM, n=2, m=4, out_dtype=sl.AS_F32)
    L = layer(sl, W, cfg)
    A64, B64 = oracle.rsparse_factors(W, r)
    y, _ = L.prefill_rsparse(dev(x), dev(_bf16r(B64)), dev(_bf16r(A64)))
    torch.cuda.synchronize()
    dense = x.double().numpy() @ W.double().numpy().T
    assert rel_l2(f32(y), dense) <= 1e-2


def test_rsparse_keep_all_adds_nothing(sl):
    """A mask with every bit set (nothing dropped) leaves y unchanged, bit for bit."""
    T, K, n_out, r = 4, 512, 256, 32
    x, _ = synth.random_layer(T, K, n_out, seed=73)
    rng = np.random.default_rng(74)
    A, B = _bf16r(rng.normal(0, 0.05, (n_out, r))), _bf16r(rng.normal(0, 0.02, (K, r)))
    y = torch.randn(T, n_out, device="cuda")
    y0 = y.clone()
    full = torch.full((T, K // 32), -1, dtype=torch.int32, device="cuda")
    ws = torch.empty(sl.as_rsparse_workspace(T, K, r), dtype=torch.uint8, device="cuda")
    sl.as_rsparse_decode(dev(x), full, dev(B), dev(A), y, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(y, y0)


# ---------------------------------------------------------------- hybrid 2:4 (sparse/dense split)
def check_hybrid(sl, T, K, n_out, n_dense, out_dtype, rows=None, seed=91):
    _, x, W, _ = synth.prefill_sqrelu_hot(T=T, k=K, n_out=n_out, seed=seed)
    cfg = sl.config(sel=sl.AS_SEL_NM, n=2, m=4, out_dtype=sl.AS_BF16 if out_dtype == torch.bfloat16 else sl.AS_F32)
    L = layer(sl, W, cfg)
    xd = dev(x)
    bufs = L.select_buffers(T)
    L.select(xd, bufs)
    idx = torch.full((max(n_dense, 1),), -1, dtype=torch.int32, device="cuda")
    sp = torch.empty(1, dtype=torch.float32, device="cuda")
    y = L.prefill_hybrid_from(xd, bufs, n_dense, dense_idx=idx, sparsity=sp)
    torch.cuda.synchronize()
    assert sl.as_stream_status() == sl.AS_OK
    xf, Wf = x.float().numpy(), W.float().numpy()
    mask_h, idx_ref, s_ref = oracle.hybrid_mask(xf, n_dense)
    if n_dense:
        np.testing.assert_array_equal(idx.cpu().numpy(), idx_ref)
    assert sp.item() == np.float32(s_ref)
    ref = oracle.linear(xf, mask_h, Wf, rows=rows)
    got = f32(y) if rows is None else f32(y)[rows]
    tol = TOL_BF16 if out_dtype == torch.bfloat16 else TOL_F32
    assert rel_l2(got, ref) <= tol
    return L, xd, bufs, y


@pytest.mark.parametrize("T,K,n_out,n_dense,out", [
    (256, 1024, 256, 16, torch.bfloat16),     # pair kernels
    (384, 2048, 264, 32, torch.float32),      # odd number of 128-row tiles: one-SM kernels, ragged n_out
    (512, 4096, 512, 48, torch.bfloat16),
])
def test_hybrid_split(sl, T, K, n_out, n_dense, out):
    check_hybrid(sl, T, K, n_out, n_dense, out)


def test_hybrid_without_dense_blocks_is_the_24_prefill(sl):
    """n_dense = 0 runs the 2:4 GEMM alone: bitwise the plain 2:4 prefill."""
    L, xd, bufs, y = check_hybrid(sl, 256, 1024, 256, 0, torch.bfloat16)
    y0 = L.prefill_from(bufs, 256)
    torch.cuda.synchronize()
    assert torch.equal(y, y0)


def check_nm_split(sl, T, K, n_out, n, m, score, dpts, var, n_dense, out, seed=61):
    """The hybrid decomposition of an N:M selection through the C ABI: the
    selection, its 2:4 part (kept bits, positions, compact values) and the
    dense blocks bit-exact against the oracle; y against the oracle's split
    product with the same epilogue."""
    x, W = synth.random_layer(T, K, n_out, seed=seed, dist="t3" if score == sl.AS_SCORE_CLACT else "laplace")
    cfg = sl.config(score=score, sel=sl.AS_SEL_NM, n=n, m=m, dpts=dpts, var=var, out_dtype=out)
    L = layer(sl, W, cfg, 0.5)
    running = torch.zeros(T, dtype=torch.float32, device="cuda") if var else None
    idx = torch.full((max(n_dense, 1),), -1, dtype=torch.int32, device="cuda")
    sp = torch.empty(1, dtype=torch.float32, device="cuda")
    y, bufs = L.prefill_nm_split(dev(x), n_dense, running_var=running, first_batch=True, dense_idx=idx, sparsity=sp)
    torch.cuda.synchronize()
    assert sl.as_stream_status() == sl.AS_OK
    xf, Wf = x.float().numpy(), W.float().numpy()
    f = f32(bufs["colnorm"]) if score == sl.AS_SCORE_CLACT else (f32(L.g) if score == sl.AS_SCORE_WEIGHT else None)
    eta32 = f32(bufs["eta"]) if dpts else None
    sc = oracle.score(xf, eta=eta32, f=f)
    mask = oracle.select_nm(sc, n, m)
    np.testing.assert_array_equal(unpack_bitmask(bufs["bitmask"], K), mask)
    xm = f32(bufs["x_masked"])
    r = oracle.nm_split(sc, mask, xm, n_dense)
    np.testing.assert_array_equal(unpack_bitmask(bufs["bitmask24"], K), r["part"])
    pos = decode_meta24(bufs["meta24"], T, K)
    ref_pos = np.nonzero(r["pos"].reshape(T, K // 4, 4))[2].reshape(T, K // 4, 2)
    np.testing.assert_array_equal(pos, ref_pos)
    vals = np.take_along_axis(xm.reshape(T, K // 4, 4), ref_pos, axis=2).reshape(T, K // 2)
    np.testing.assert_array_equal(f32(bufs["x_compact"]), vals)
    if n_dense:
        np.testing.assert_array_equal(idx.cpu().numpy(), r["idx"])
    assert sp.item() == np.float32(r["sparsity"])
    nu = None
    if var:
        nu = oracle.var_scale(xf, mask, None, cfg.var_momentum, cfg.var_eps)["nu"]
    eta64 = oracle.token_mean(xf) if dpts else None
    _, rs = oracle.weight_prep(Wf, 1.0)
    ref = oracle.linear(xf, r["m_split"], Wf, eta=eta64, rowsum=rs if dpts else None, nu=nu)
    err = rel_l2(f32(y), ref)
    assert err <= (TOL_BF16 if out == sl.AS_BF16 else TOL_F32), err
    return y, mask, r


# (T, K, n_out, n, m, score, dpts, var, n_dense, out): T = 300 runs the
# one-SM kernels, the others the CTA pairs
@pytest.mark.parametrize("T,K,n_out,n,m,score,dpts,var,n_dense,out", [
    (256, 1024, 264, 8, 16, 1, True, False, 16, 1),     # weight-aware 8:16 with D-PTS
    (300, 2048, 264, 16, 32, 2, False, True, 64, 0),    # CLACT + VAR 16:32, float32 out
    (256, 1024, 256, 16, 32, 0, False, False, 0, 0),    # no dense block: the 2:4 part alone
    (512, 2048, 520, 8, 16, 0, False, False, 32, 1),
])
def test_nm_split(sl, T, K, n_out, n, m, score, dpts, var, n_dense, out):
    check_nm_split(sl, T, K, n_out, n, m, score, dpts, var, n_dense, out)


def test_nm_split_all_blocks_dense_is_the_nm_product(sl):
    """With every block dense the split is exactly the 16:32 selection's
    product: against the oracle and the masked dense prefill of the same
    selection."""
    T, K, n_out = 256, 1024, 256
    y, mask, r = check_nm_split(sl, T, K, n_out, 16, 32, 0, False, False, K // 4, 0)
    np.testing.assert_array_equal(r["m_split"], mask)
    x, W = synth.random_layer(T, K, n_out, seed=61, dist="laplace")
    cfg = sl.config(sel=sl.AS_SEL_NM, n=16, m=32, out_dtype=sl.AS_F32)
    y_nm, _ = layer(sl, W, cfg).prefill(dev(x))
    torch.cuda.synchronize()
    assert rel_l2(f32(y), f32(y_nm)) <= TOL_F32


def test_hybrid_full_size(sl):
    """The down-projection shape with hot channels (T 4096, K 14336, n_out
    4096, 192 dense blocks = 768 channels), sampled rows of every tile."""
    check_hybrid(sl, 4096, 14336, 4096, 192, torch.bfloat16, rows=np.arange(3, 4096, 67))


def test_prefill_auto_modes(sl):
    """The page's mode rule on three activation mixes: hot channels (~94 %
    zeros: split), all cold (~96 %: pure 2:4), plain N(-1.2, 1) (~88 %: dense);
    each result against the oracle for that mode."""
    from sparse_linear_b200.layer import SparseLinear
    T, K, n_out = 256, 2048, 256
    cases = [synth.prefill_sqrelu_hot(T=T, k=K, n_out=n_out, seed=92)[1:3],
             synth.prefill_sqrelu_hot(T=T, k=K, n_out=n_out, seed=93, hot_frac=0.0005, mu_hot=-1.8)[1:3],
             synth.prefill_sqrelu(T=T, k=K, n_out=n_out, seed=94)[1:3]]
    modes = []
    for x, W in cases:
        L = SparseLinear(dev(W), sl.config(sel=sl.AS_SEL_NM, n=2, m=4, out_dtype=sl.AS_F32), keep_wt=False)
        y, mode, s = L.prefill_auto(dev(x))
        torch.cuda.synchronize()
        xf, Wf = x.float().numpy(), W.float().numpy()
        _, total = oracle.block_nnz(xf)
        s_ref = 1.0 - total / float(T * K)
        assert s == np.float32(s_ref) and mode == oracle.hybrid_mode(s_ref)
        if mode == "dense":
            mask = np.ones_like(xf, np.uint8)
        elif mode == "2:4":
            mask = oracle.select_nm(oracle.score(xf), 2, 4)
        else:
            mask = oracle.hybrid_mask(xf, 32)[0]   # ceil(0.05 * 512 / 16) * 16 = 32 blocks
        assert rel_l2(f32(y), oracle.linear(xf, mask, Wf)) <= TOL_F32
        modes.append(mode)
    assert modes == ["split", "2:4", "dense"]
