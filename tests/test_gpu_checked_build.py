"""The index-checked build of the library (-DAS_BOUNDS_CHECK) on small cases
of every kernel family.

With ``libactsparse_checked.so`` swapped in for the default library, a set of
the GPU parity tests runs unchanged: their oracle comparisons hold and every
call's device status stays AS_OK, so no checked global or shared-memory index
left its buffer (a failed check skips the access and records AS_ERR_BOUNDS;
nothing traps).  The checked library is built in-tree if it is stale."""
import ctypes

import pytest
import torch

import test_gpu_parity as P

pytestmark = pytest.mark.gpu

CASES = [
    # decode: fused (1 token), select kernel + union list, DENSE streaming,
    # top-k, keep-all, float32 weights, threshold, S-PTS, R-Sparse
    (P.test_decode_tiny_layer, {}),
    (P.test_decode_downproj, dict(T=1, out="bf16")),
    (P.test_decode_downproj, dict(T=8, out="f32")),
    (P.test_decode_downproj, dict(T=16, out="bf16")),
    (P.test_decode_ragged, dict(T=3, K=1040, n_out=264, n=2, m=4, score=0, dpts=False, ties=0)),
    (P.test_decode_ragged, dict(T=5, K=1040, n_out=264, n=8, m=16, score=1, dpts=True, ties=0)),
    (P.test_decode_ragged, dict(T=11, K=8192, n_out=136, n=8, m=16, score=2, dpts=True, ties=0)),
    (P.test_decode_topk_edges, dict(kk=100)),
    (P.test_decode_keep_all_is_dense, {}),
    (P.test_decode_fp32_weights, {}),
    (P.test_decode_thresh, dict(T=8, dpts=1)),
    (P.test_decode_static_pts, dict(T=2)),
    (P.test_rsparse_decode, dict(T=5, K=1008, n_out=264, r=32, dpts=False, svd=True)),
    # weight preparation and FP8 quantisation
    (P.test_weight_prep, dict(alpha=0.5)),
    (P.test_amber_deterministic, {}),
    (P.test_fp8_weight_quant, dict(n_out=264, K=1024, dtype=torch.bfloat16)),
    # prefill: selection kernels, 2:4 and masked dense GEMMs (pair and one-SM),
    # residual pass, FP8, R-Sparse, hybrid and N:M split, statistics
    (P.test_prefill_24, dict(T=300, K=1024, n_out=520)),
    (P.test_prefill_24, dict(T=5, K=256, n_out=64)),
    (P.test_prefill_dense_path, dict(n=8, m=16, score=1, dpts=True)),
    (P.test_prefill_topk_and_all, {}),
    (P.test_prefill_clact_var_small, {}),
    (P.test_prefill_shift_float32_residual_pass, dict(T=300, case="2:4 D-PTS")),
    (P.test_prefill_thresh_and_static_pts, {}),
    (P.test_fp8_producer, dict(T=129, K=832)),
    (P.test_fp8_gemm, dict(T=384, K=832, n_out=512, out=torch.float32)),
    (P.test_rsparse_prefill, dict(T=300, K=1024, n_out=264, r=128, sel="8:16", dpts=True, out="f32", svd=True)),
    (P.test_hybrid_split, dict(T=384, K=2048, n_out=264, n_dense=32, out=torch.float32)),
    (P.test_nm_split, dict(T=300, K=2048, n_out=264, n=16, m=32, score=2, dpts=False, var=True, n_dense=64,
                           out=0)),
    (P.test_select_stats_ragged, dict(dtype=torch.bfloat16)),
]


@pytest.fixture(scope="module")
def sl_checked():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import sparse_linear_b200 as m
    from sparse_linear_b200 import build
    lib = ctypes.CDLL(build.build_checked())
    for name, (args, res) in m._sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    default = m._lib
    m._lib = lib
    try:
        yield m
    finally:
        m._lib = default


@pytest.mark.parametrize("i", range(len(CASES)), ids=[f"{f.__name__}-{j}" for j, (f, _) in enumerate(CASES)])
def test_checked_build(sl_checked, i):
    fn, kw = CASES[i]
    try:
        fn(sl_checked, **kw)
        torch.cuda.synchronize()
        assert sl_checked.as_stream_status() == sl_checked.AS_OK
    finally:
        line = sl_checked.as_checked_line()
        assert line == 0, f"index check failed at source line {line}"
