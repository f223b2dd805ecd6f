"""The decode entry point that allocates nothing (as_linear_decode_noalloc).

It serves callers that cannot call cudaMalloc (code inside a framework that
owns every device allocation through its own pool, or a process held to a
fixed device-memory budget): its scratch is the library's own fixed device
array.  Through the C ABI, two calls in a row must give the same output as
the regular workspace entry point: the kernels are deterministic and the
two entry points run the same kernels, so the outputs must be bitwise
equal (which is within every tolerance the other GPU tests use).  A call
needing more scratch than the array holds is refused.  This file is
collected last on purpose."""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

TOL_BF16, TOL_F32 = 1e-2, 2e-3


def _rel_l2(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


@pytest.fixture(scope="module")
def sl():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import sparse_linear_b200 as m
    return m


@pytest.mark.parametrize("T,out", [(1, "bf16"), (16, "f32")])
def test_noalloc_decode_matches_workspace_entry_point(sl, T, out):
    from sparse_linear_b200.layer import SparseLinear
    x, W, _ = synth.decode_downproj(T)
    x2, _, _ = synth.decode_downproj(T, seed=77, with_weight=False)
    cfg = sl.config(score=sl.AS_SCORE_WEIGHT, sel=sl.AS_SEL_NM, n=8, m=16, dpts=True,
                    out_dtype=sl.AS_BF16 if out == "bf16" else sl.AS_F32)
    tol = TOL_BF16 if out == "bf16" else TOL_F32
    L = SparseLinear(W.cuda(), cfg, alpha=0.5)
    for xin in (x, x2):  # two calls in a row share the static scratch
        xd = xin.cuda()
        ref = L.decode(xd)
        y = torch.empty_like(ref)
        sl.as_linear_decode_noalloc(xd, L.Wt, cfg, y, g=L.g, rowsum=L.rowsum)
        torch.cuda.synchronize()
        assert sl.as_stream_status() == sl.AS_OK
        assert _rel_l2(y, ref) <= tol
        assert torch.equal(y, ref)


def test_noalloc_topk_two_calls(sl):
    from sparse_linear_b200.layer import SparseLinear
    blk = synth.decode_block()
    for ly in blk["layers"][:2]:
        kk = int(ly["keep_frac"] * ly["k"] + 0.5)
        cfg = sl.config(score=sl.AS_SCORE_WEIGHT, sel=sl.AS_SEL_TOPK, k_keep=kk)
        L = SparseLinear(ly["W"].cuda(), cfg, alpha=ly["alpha"])
        xd = blk["x"][ly["x_key"]].cuda()
        ref = L.decode(xd)
        y = torch.empty_like(ref)
        sl.as_linear_decode_noalloc(xd, L.Wt, cfg, y, g=L.g, rowsum=L.rowsum)
        torch.cuda.synchronize()
        assert sl.as_stream_status() == sl.AS_OK
        assert _rel_l2(y, ref) <= TOL_BF16
        assert torch.equal(y, ref)


def test_noalloc_refuses_oversized_scratch(sl):
    """A call whose scratch need exceeds the fixed array is refused with
    AS_ERR_WORKSPACE before anything is launched."""
    T, K, n_out = 16, 11008, 16384
    cfg = sl.config(score=sl.AS_SCORE_MAG, sel=sl.AS_SEL_NM, n=8, m=16)
    assert sl.as_workspace_size(sl.AS_OP_DECODE, T, K, n_out, cfg) > sl.AS_NOALLOC_SCRATCH_BYTES
    x = torch.zeros(T, K, dtype=torch.bfloat16, device="cuda")
    Wt = torch.zeros(K, n_out, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(T, n_out, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(sl.ASError) as e:
        sl.as_linear_decode_noalloc(x, Wt, cfg, y)
    assert e.value.code == sl.AS_ERR_WORKSPACE
