"""Failure reporting, determinism and resumable VAR state, through the C ABI.

The failure path is exercised without faulting the GPU: the probe kernel's
bounded wait runs out on an mbarrier that nothing signals, records
AS_ERR_TIMEOUT and returns.
"""
import numpy as np
import pytest
import torch

import synth
from gpu_util import f32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sl():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import sparse_linear_b200 as m
    return m


def dev(t):
    return t.contiguous().cuda()


def test_timeout_is_reported_and_cleared(sl):
    sl.as_probe_timeout(1000)
    assert sl.as_stream_status() == sl.AS_ERR_TIMEOUT
    assert sl.as_stream_status() == sl.AS_OK  # cleared by the first report
    # the context is still usable: a decode afterwards runs and reports OK
    from sparse_linear_b200.layer import SparseLinear
    x, W = synth.random_layer(2, 1024, 256, seed=5)
    L = SparseLinear(dev(W), sl.config(sel=sl.AS_SEL_NM, n=8, m=16, dpts=True))
    y = L.decode(dev(x))
    torch.cuda.synchronize()
    assert sl.as_stream_status() == sl.AS_OK
    assert torch.isfinite(y.float()).all()


@pytest.mark.parametrize("n,m", [(2, 4), (8, 16)])
def test_prefill_is_deterministic(sl, n, m):
    from sparse_linear_b200.layer import SparseLinear
    x, W = synth.random_layer(512, 2048, 768, seed=21, dist="sqrelu")
    L = SparseLinear(dev(W), sl.config(sel=sl.AS_SEL_NM, n=n, m=m))
    xd = dev(x)
    y1, b1 = L.prefill(xd)
    y2, b2 = L.prefill(xd)
    torch.cuda.synchronize()
    assert sl.as_stream_status() == sl.AS_OK
    assert torch.equal(y1, y2)
    assert torch.equal(b1["bitmask"], b2["bitmask"])


def test_var_state_checkpoint_and_resume(sl):
    """Six batches straight through equal three batches, a checkpoint of the
    running variance (copied to the host), a fresh layer and buffer restored
    from it, and the last three batches: same state and outputs, bitwise."""
    from sparse_linear_b200.layer import SparseLinear
    T, K, n_out = 264, 1024, 264
    xs = [dev(synth.random_layer(T, K, n_out, seed=300 + b, dist="t3")[0]) for b in range(6)]
    W = dev(synth.random_layer(1, K, n_out, seed=299)[1])
    cfg = sl.config(score=sl.AS_SCORE_CLACT, sel=sl.AS_SEL_NM, n=16, m=32, var=True)

    L = SparseLinear(W, cfg)
    run = torch.zeros(T, dtype=torch.float32, device="cuda")
    ys = []
    for b, x in enumerate(xs):
        y, _ = L.prefill(x, running_var=run, first_batch=(b == 0))
        ys.append(y.clone())
    torch.cuda.synchronize()
    state_full = run.clone()

    L1 = SparseLinear(W, cfg)
    run1 = torch.zeros(T, dtype=torch.float32, device="cuda")
    for b in range(3):
        L1.prefill(xs[b], running_var=run1, first_batch=(b == 0))
    torch.cuda.synchronize()
    ckpt = run1.cpu().numpy().copy()  # the whole resumable state

    L2 = SparseLinear(W, cfg)
    run2 = torch.from_numpy(ckpt).cuda()
    ys2 = []
    for b in range(3, 6):
        y, _ = L2.prefill(xs[b], running_var=run2, first_batch=False)
        ys2.append(y.clone())
    torch.cuda.synchronize()
    assert sl.as_stream_status() == sl.AS_OK
    np.testing.assert_array_equal(f32(run2), f32(state_full))
    for a, b in zip(ys[3:], ys2):
        assert torch.equal(a, b)


def test_prepared_decode_call_matches(sl):
    """sl.DecodeCall (fixed arguments marshalled once) gives the bitwise
    result of as_linear_decode, across calls with different x."""
    from sparse_linear_b200.layer import SparseLinear, workspace
    x, W, _ = synth.decode_downproj(8)
    cfg = sl.config(score=sl.AS_SCORE_WEIGHT, sel=sl.AS_SEL_NM, n=8, m=16, dpts=True)
    L = SparseLinear(dev(W), cfg, alpha=0.5)
    ws = workspace(sl.as_workspace_size(sl.AS_OP_DECODE, 8, L.K, L.n_out, cfg), "cuda")
    call = sl.DecodeCall(L.Wt, cfg, g=L.g, rowsum=L.rowsum, workspace=ws)
    for T in (1, 8):
        xd = dev(x[:T])
        y1 = torch.empty(T, L.n_out, dtype=torch.bfloat16, device="cuda")
        y2 = torch.empty_like(y1)
        call(xd, y1)
        sl.as_linear_decode(xd, L.Wt, cfg, y2, g=L.g, rowsum=L.rowsum, workspace=ws)
        torch.cuda.synchronize()
        assert sl.as_stream_status() == sl.AS_OK
        assert torch.equal(y1, y2)
