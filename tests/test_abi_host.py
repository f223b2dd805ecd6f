"""Host-only checks of the C-ABI library: it loads without a GPU, exports
every entry point include/actsparse.h declares, and its argument validation
rejects invalid calls with the documented status before touching the GPU."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "actsparse.h")


@pytest.fixture(scope="module")
def lib():
    import importlib.util
    spec = importlib.util.spec_from_file_location("_as_build", os.path.join(ROOT, "sparse_linear_b200", "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    b.build()
    import sparse_linear_b200 as sl
    return sl


def declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(as_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared()
    for n in ("as_weight_prep", "as_select", "as_linear_decode", "as_linear_prefill",
              "as_workspace_size", "as_stream_status", "as_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    raw = ctypes.CDLL(lib.LIB_PATH)
    for n in declared():
        assert hasattr(raw, n), n
    assert set(lib.EXPORTS) == set(declared())
    assert lib.as_abi_version() == 3


def test_status_strings(lib):
    for code in range(9):
        assert lib.as_status_string(code).startswith("AS_")


def test_workspace_sizes(lib):
    cfg = lib.config(score=lib.AS_SCORE_WEIGHT, sel=lib.AS_SEL_NM, n=8, m=16, dpts=True)
    ws = lib.as_workspace_size(lib.AS_OP_DECODE, 1, 11008, 4096, cfg)
    assert ws > 0
    assert lib.as_workspace_size(lib.AS_OP_WEIGHT_PREP, 0, 4096, 1024, None) == 4 * 4096 * 8
    assert lib.as_workspace_size(lib.AS_OP_PREFILL, 4096, 14336, 4096, lib.config()) == 0
    bad = lib.config(sel=lib.AS_SEL_NM, n=2, m=4)
    with pytest.raises(lib.ASError):
        lib.as_workspace_size(lib.AS_OP_DECODE, 17, 1024, 64, bad)  # T > 16
    with pytest.raises(lib.ASError):
        lib.as_workspace_size(lib.AS_OP_SELECT, 4, 1022, 0, bad)  # K % M
    assert lib.as_meta24_words(4096, 14336) == 32 * 112 * 512
    assert lib.as_meta24_words(1, 16) == 512


def _call_decode(lib, x, K, n_out, cfg, T=1, dt=None, y=16, wt=16, ws=16, ws_bytes=1 << 20):
    f = lib._lib.as_linear_decode
    return f(x, lib.AS_BF16 if dt is None else dt, T, K, n_out, wt, None, None, ctypes.byref(cfg), y,
             None, None, None, ws, ws_bytes, None)


def test_decode_validation_launches_nothing(lib):
    """Invalid calls are rejected on the host (fake, never-dereferenced
    16-byte-aligned addresses: a launch would fault, so any call reaching
    the GPU would fail here without a GPU)."""
    fake = 1 << 20
    ok = lib.config(sel=lib.AS_SEL_NM, n=2, m=4)
    assert _call_decode(lib, fake, 1000, 64, ok, T=0) == lib.AS_ERR_SHAPE
    assert _call_decode(lib, fake, 1000, 64, ok, T=17) == lib.AS_ERR_SHAPE
    assert _call_decode(lib, fake, 1002, 64, ok) == lib.AS_ERR_SHAPE                # K % M
    assert _call_decode(lib, fake, 1024, 60, ok) == lib.AS_ERR_SHAPE                # n_out % 8
    assert _call_decode(lib, fake, 1024, 64, lib.config(n=5, m=4)) == lib.AS_ERR_SHAPE
    assert _call_decode(lib, fake, 1024, 64, lib.config(n=2, m=3)) == lib.AS_ERR_SHAPE
    assert _call_decode(lib, fake, 1024, 64, lib.config(sel=lib.AS_SEL_TOPK, k_keep=2000)) == lib.AS_ERR_SHAPE
    assert _call_decode(lib, fake, 1024, 64, ok, dt=7) == lib.AS_ERR_DTYPE
    assert _call_decode(lib, fake + 4, 1024, 64, ok) == lib.AS_ERR_ALIGN
    assert _call_decode(lib, None, 1024, 64, ok) == lib.AS_ERR_INVALID_ARG
    assert _call_decode(lib, fake, 1024, 64, lib.config(var=True)) == lib.AS_ERR_UNSUPPORTED
    assert _call_decode(lib, fake, 1024, 64, lib.config(dpts=True)) == lib.AS_ERR_INVALID_ARG  # no rowsum
    assert _call_decode(lib, fake, 1024, 64, lib.config(score=lib.AS_SCORE_WEIGHT)) == lib.AS_ERR_INVALID_ARG
    assert _call_decode(lib, fake, 1024, 64, ok, ws=None) == lib.AS_ERR_WORKSPACE
    assert _call_decode(lib, fake, 1024, 64, ok, ws_bytes=0) == lib.AS_ERR_WORKSPACE


def test_select_and_prefill_validation(lib):
    fake = 1 << 20
    sel = lib._lib.as_select
    cfg24 = lib.config(sel=lib.AS_SEL_NM, n=2, m=4)
    out = lib.as_select_out()
    out.x_compact = fake
    out.meta24 = fake
    # compact 2:4 operand needs bf16 and K % 16 == 0
    assert sel(fake, lib.AS_F32, 4, 64, ctypes.byref(cfg24), None, None, 0, ctypes.byref(out), None, 0,
               None) == lib.AS_ERR_UNSUPPORTED
    assert sel(fake, lib.AS_BF16, 4, 72, ctypes.byref(cfg24), None, None, 0, ctypes.byref(out), None, 0,
               None) == lib.AS_ERR_UNSUPPORTED
    cfg816 = lib.config(sel=lib.AS_SEL_NM, n=8, m=16)
    assert sel(fake, lib.AS_BF16, 4, 64, ctypes.byref(cfg816), None, None, 0, ctypes.byref(out), None, 0,
               None) == lib.AS_ERR_UNSUPPORTED
    both = lib.config(dpts=True, var=True)
    assert sel(fake, lib.AS_BF16, 4, 64, ctypes.byref(both), None, fake, 1, ctypes.byref(lib.as_select_out()),
               None, 0, None) == lib.AS_ERR_UNSUPPORTED
    var = lib.config(var=True)
    assert sel(fake, lib.AS_BF16, 4, 64, ctypes.byref(var), None, None, 1, ctypes.byref(lib.as_select_out()),
               None, 0, None) == lib.AS_ERR_INVALID_ARG  # no running_var
    clact = lib.config(score=lib.AS_SCORE_CLACT, n=16, m=32)
    assert sel(fake, lib.AS_BF16, 4, 64, ctypes.byref(clact), None, None, 0, ctypes.byref(lib.as_select_out()),
               None, 0, None) == lib.AS_ERR_WORKSPACE
    # residual operands need their main operand (and bf16 x for the masked one)
    lo = lib.as_select_out()
    lo.x_masked_lo = fake
    assert sel(fake, lib.AS_BF16, 4, 64, ctypes.byref(cfg816), None, None, 0, ctypes.byref(lo), None, 0,
               None) == lib.AS_ERR_INVALID_ARG
    lo.x_masked = fake
    assert sel(fake, lib.AS_F32, 4, 64, ctypes.byref(cfg816), None, None, 0, ctypes.byref(lo), None, 0,
               None) == lib.AS_ERR_INVALID_ARG
    lo2 = lib.as_select_out()
    lo2.x_compact_lo = fake
    assert sel(fake, lib.AS_BF16, 4, 64, ctypes.byref(cfg24), None, None, 0, ctypes.byref(lo2), None, 0,
               None) == lib.AS_ERR_INVALID_ARG
    lo.x_masked_lo = fake + 4
    assert sel(fake, lib.AS_BF16, 4, 64, ctypes.byref(cfg816), None, None, 0, ctypes.byref(lo), None, 0,
               None) == lib.AS_ERR_ALIGN
    pre = lib._lib.as_linear_prefill
    empty = lib.as_select_out()
    assert pre(ctypes.byref(empty), fake, 4, 64, 64, None, None, None, ctypes.byref(cfg816), fake, None, 0,
               None) == lib.AS_ERR_INVALID_ARG  # no x_masked
    assert pre(ctypes.byref(empty), fake, 4, 64, 64, None, None, None, ctypes.byref(cfg24), fake, None, 0,
               None) == lib.AS_ERR_INVALID_ARG  # no compact operand
    masked = lib.as_select_out()
    masked.x_masked = fake
    assert pre(ctypes.byref(masked), fake, 4, 60, 64, None, None, None, ctypes.byref(lib.config(n=2, m=2)),
               fake, None, 0, None) == lib.AS_ERR_SHAPE  # K % 8
    assert pre(ctypes.byref(masked), fake, 4, 64, 64, None, None, None, ctypes.byref(lib.config(dpts=True, n=8, m=16)),
               fake, None, 0, None) == lib.AS_ERR_INVALID_ARG  # dpts needs eta and rowsum


def test_binding_refuses_cpu_tensors(lib):
    import torch
    x = torch.zeros(1, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        lib.as_linear_decode(x, x, lib.config(), x)


def test_timeout_probe_validates_polls(lib):
    # out-of-range poll counts are refused on the host, before any launch
    for polls in (0, (1 << 20) + 1):
        assert lib._lib.as_probe_timeout(polls, None) == lib.AS_ERR_INVALID_ARG


def test_threshold_and_static_pts_validation(lib):
    # S-PTS without its table, an unknown shift mode, and a NaN threshold are
    # refused on the host (workspace sizing validates the config too)
    bad = [lib.config(dpts=lib.AS_PTS_STATIC), lib.config(dpts=3),
           lib.config(sel=lib.AS_SEL_THRESH, tau=float("nan"))]
    for cfg in bad:
        assert lib._lib.as_workspace_size(lib.AS_OP_DECODE, 1, 64, 64, ctypes.byref(cfg)) == ctypes.c_size_t(-1).value
    ok = lib.config(sel=lib.AS_SEL_THRESH, tau=0.5)
    assert lib._lib.as_workspace_size(lib.AS_OP_DECODE, 1, 64, 64, ctypes.byref(ok)) != ctypes.c_size_t(-1).value


def test_amber_validation_launches_nothing(lib):
    """Percentiles out of [0, 100] or reversed, NULL outputs, too many
    weights and a short workspace are refused on the host (fake addresses:
    any launch would fail here without a GPU)."""
    fake = 1 << 20
    f = lib._lib.as_weight_prep_amber
    ws = lib.as_workspace_size(lib.AS_OP_AMBER, 0, 4096, 1024, None)
    assert ws == 4096 + 296 * 16 + 4 * 4096 * 8

    def call(W=fake, n_out=1024, K=4096, lo=0.5, hi=99.5, g=fake, b=None, w=fake, wb=ws, dt=lib.AS_BF16):
        return f(W, dt, n_out, K, 1.0, lo, hi, g, b, w, wb, None)

    assert call(lo=-0.1) == lib.AS_ERR_INVALID_ARG
    assert call(hi=100.5) == lib.AS_ERR_INVALID_ARG
    assert call(lo=60.0, hi=40.0) == lib.AS_ERR_INVALID_ARG
    assert call(lo=float("nan")) == lib.AS_ERR_INVALID_ARG
    assert call(W=None) == lib.AS_ERR_INVALID_ARG
    assert call(g=None) == lib.AS_ERR_INVALID_ARG
    assert call(n_out=65536, K=65536) == lib.AS_ERR_SHAPE
    assert call(dt=5) == lib.AS_ERR_DTYPE
    assert call(b=fake + 8) == lib.AS_ERR_ALIGN
    assert call(w=None) == lib.AS_ERR_WORKSPACE
    assert call(wb=ws - 1) == lib.AS_ERR_WORKSPACE


def test_fp8_validation_launches_nothing(lib):
    """Shape, dtype, alignment and NULL checks of the FP8 entry points run on
    the host (fake addresses: a launch would fail without a GPU)."""
    fake = 1 << 20
    L = lib._lib
    assert lib.as_meta8_words(4096, 14336) == 16 * 2 * 56 * 1024
    assert lib.as_meta8_words(1, 64) == 2 * 1 * 1024
    assert L.as_weight_quant_fp8(fake, lib.AS_BF16, 64, 40, fake, fake, None) == lib.AS_ERR_SHAPE
    assert L.as_weight_quant_fp8(fake, 9, 64, 64, fake, fake, None) == lib.AS_ERR_DTYPE
    assert L.as_weight_quant_fp8(None, lib.AS_BF16, 64, 64, fake, fake, None) == lib.AS_ERR_INVALID_ARG
    assert L.as_weight_quant_fp8(fake, lib.AS_BF16, 64, 64, fake + 1, fake, None) == lib.AS_ERR_ALIGN
    assert L.as_select_sqrelu24_fp8(fake, 8, 96, fake, fake, fake, None, None) == lib.AS_ERR_SHAPE
    assert L.as_select_sqrelu24_fp8(fake, 0, 128, fake, fake, fake, None, None) == lib.AS_ERR_INVALID_ARG
    assert L.as_select_sqrelu24_fp8(fake, 8, 128, fake, None, fake, None, None) == lib.AS_ERR_INVALID_ARG
    assert L.as_select_sqrelu24_fp8(fake, 8, 128, fake, fake, fake, fake + 4, None) == lib.AS_ERR_ALIGN
    f = L.as_linear_prefill_fp8
    assert f(fake, fake, fake, 8, 96, 64, fake, fake, lib.AS_BF16, fake, None) == lib.AS_ERR_SHAPE
    assert f(fake, fake, fake, 8, 128, 60, fake, fake, lib.AS_BF16, fake, None) == lib.AS_ERR_SHAPE
    assert f(fake, fake, fake, 8, 128, 64, fake, fake, 5, fake, None) == lib.AS_ERR_DTYPE
    assert f(fake, None, fake, 8, 128, 64, fake, fake, lib.AS_BF16, fake, None) == lib.AS_ERR_INVALID_ARG
    assert f(fake, fake, fake, 8, 128, 64, fake, fake + 8, lib.AS_BF16, fake, None) == lib.AS_ERR_ALIGN


def test_rsparse_validation_launches_nothing(lib):
    fake = 1 << 20
    f = lib._lib.as_rsparse_decode
    ws = lib.as_rsparse_workspace(16, 11008, 64)
    assert ws == 86 * 16 * 64 * 4
    for r in (0, 8, 16, 48, 256):
        with pytest.raises(lib.ASError):
            lib.as_rsparse_workspace(1, 64, r)

    def call(T=1, K=64, n_out=64, r=64, x=fake, A=fake, wb=1 << 20, dt=lib.AS_BF16):
        return f(x, dt, T, K, n_out, r, fake, None, fake, A, fake, fake, wb, None)

    assert call(T=0) == lib.AS_ERR_SHAPE and call(T=17) == lib.AS_ERR_SHAPE
    assert call(r=48) == lib.AS_ERR_SHAPE
    assert call(x=None) == lib.AS_ERR_INVALID_ARG
    assert call(dt=3) == lib.AS_ERR_DTYPE
    assert call(A=fake + 2) == lib.AS_ERR_ALIGN
    assert call(wb=0) == lib.AS_ERR_WORKSPACE


def test_hybrid_validation_launches_nothing(lib):
    fake = 1 << 20
    # the gathered remainder [T, 4 n_dense] and W columns [n_out, 4 n_dense];
    # no float32 output-sized term (the dense blocks run inside the 2:4 GEMM)
    ws = lib.as_hybrid_workspace(4096, 14336, 4096, 192)
    assert 2 * 4096 * 768 * 2 < ws < 4096 * 4096 * 4
    for bad in ((4096, 14300, 4096, 16), (4096, 14336, 4096, 17), (4096, 14336, 4096, 14336 // 4 + 16),
                (16, 65536, 64, 16), (16, 1024, 60, 16), (1 << 22, 1024, 64, 16)):
        with pytest.raises(lib.ASError):
            lib.as_hybrid_workspace(*bad)
    # the gather rows are strided over the grid: no limit on T + n_out
    assert lib.as_hybrid_workspace(60000, 1024, 8192, 16) > 0
    assert lib.as_hybrid_workspace(8192, 1024, 57344, 16) > 0
    assert lib.as_hybrid_workspace(70000, 1024, 0, 0) > 0
    sel = lib.select_out(bitmask=None)
    f = lib._lib.as_linear_prefill_hybrid
    assert f(ctypes.byref(sel), fake, 16, 1024, fake, 64, 16, lib.AS_BF16, fake, None, None, fake, 1 << 30,
             None) == lib.AS_ERR_INVALID_ARG  # no 2:4 outputs
    assert lib._lib.as_block_sparsity(fake, 16, 1000, 0, None, fake, fake, 1 << 20, None) == lib.AS_ERR_SHAPE
    assert lib._lib.as_block_sparsity(fake, 16, 1024, 16, None, fake, fake, 1 << 20, None) == lib.AS_ERR_INVALID_ARG
    assert lib._lib.as_block_sparsity(fake, 16, 1024, 0, None, fake, fake, 0, None) == lib.AS_ERR_WORKSPACE
    # T = 70000 passes validation (without a GPU the accepted call then fails
    # at its first CUDA call, never with a shape error)
    ws = lib.as_hybrid_workspace(70000, 1024, 0, 0)
    assert lib._lib.as_block_sparsity(fake, 70000, 1024, 0, None, fake, fake, ws, None) not in (
        lib.AS_ERR_SHAPE, lib.AS_ERR_INVALID_ARG, lib.AS_ERR_WORKSPACE, lib.AS_OK)


def test_hybrid_mode_rule_and_dense_block_count(lib):
    """The library's mode switch (a C entry point) equals the oracle's
    reading of the page's thresholds; the dense-block count is 5 % of the
    blocks rounded up to 64 channels, within [16, K/4]."""
    import oracle
    from sparse_linear_b200.layer import dense_blocks_for, hybrid_mode
    names = {lib.AS_MODE_24: "2:4", lib.AS_MODE_SPLIT: "split", lib.AS_MODE_DENSE: "dense"}
    for s in np.linspace(0.0, 1.0, 2001):
        assert names[lib._lib.as_prefill_mode(float(s))] == oracle.hybrid_mode(float(s))
        assert hybrid_mode(float(s)) == oracle.hybrid_mode(float(s))
    for s in (0.95, 0.90, 0.9500001, 0.8999999, float(np.float32(0.95)), float(np.float32(0.9))):
        assert hybrid_mode(s) == oracle.hybrid_mode(s)
    assert lib._lib.as_prefill_mode(float("nan")) == lib.AS_MODE_DENSE
    for K, f in ((1000, 0.05), (0, 0.05), (1024, -0.1), (1024, 1.5), (1024, float("nan"))):
        assert lib._lib.as_hybrid_dense_blocks(K, f) == -1
    assert dense_blocks_for(14336, 0.05) == 192      # 179.2 blocks -> 12 x 16
    assert dense_blocks_for(2048, 0.05) == 32        # 25.6 -> 2 x 16
    assert dense_blocks_for(256, 0.05) == 16         # at least 16
    assert dense_blocks_for(1024, 1.0) == 256        # at most K/4
    for K in range(64, 32769, 64):
        n = dense_blocks_for(K, 0.05)
        assert n % 16 == 0 and 16 <= n <= max(16, K // 4 // 16 * 16)


def test_noalloc_refusals_enqueue_nothing(lib):
    """as_linear_decode_noalloc checks every argument before it touches its
    shared scratch: each invalid call returns its own status (fake,
    never-dereferenced addresses; any launch or memset would fail here
    without a GPU, with AS_ERR_CUDA)."""
    fake = 1 << 20
    f = lib._lib.as_linear_decode_noalloc
    ok = lib.config(sel=lib.AS_SEL_NM, n=2, m=4)

    def call(x=fake, dt=lib.AS_BF16, T=1, K=1024, n_out=64, wt=fake, g=None, rs=None, cfg=ok, y=fake, mask=None):
        return f(x, dt, T, K, n_out, wt, g, rs, ctypes.byref(cfg), y, mask, None, None, None)

    assert call(x=None) == lib.AS_ERR_INVALID_ARG
    assert call(y=None) == lib.AS_ERR_INVALID_ARG
    assert call(dt=7) == lib.AS_ERR_DTYPE
    assert call(T=0) == lib.AS_ERR_SHAPE and call(T=17) == lib.AS_ERR_SHAPE
    assert call(K=1002) == lib.AS_ERR_SHAPE
    assert call(n_out=60) == lib.AS_ERR_SHAPE
    assert call(cfg=lib.config(var=True)) == lib.AS_ERR_UNSUPPORTED
    assert call(cfg=lib.config(dpts=True)) == lib.AS_ERR_INVALID_ARG          # no rowsum
    assert call(cfg=lib.config(score=lib.AS_SCORE_WEIGHT)) == lib.AS_ERR_INVALID_ARG  # no g
    assert call(x=fake + 4) == lib.AS_ERR_ALIGN
    assert call(mask=fake + 8) == lib.AS_ERR_ALIGN
    assert call(T=16, K=11008, n_out=16384, cfg=lib.config(sel=lib.AS_SEL_NM, n=8, m=16)) == lib.AS_ERR_WORKSPACE


def test_rsparse_prefill_validation_launches_nothing(lib):
    fake = 1 << 20
    f = lib._lib.as_linear_prefill_rsparse
    assert lib.as_rsparse_prefill_workspace(4096, 14336, 64) > 4096 * 64 * 2 * 2
    for r in (0, 32, 96, 256):
        with pytest.raises(lib.ASError):
            lib.as_rsparse_prefill_workspace(16, 1024, r)
    sel = lib.as_select_out()
    sel.bitmask = fake
    sel.x_compact = fake
    sel.meta24 = fake
    cfg = lib.config(sel=lib.AS_SEL_NM, n=2, m=4)
    ws = lib.as_rsparse_prefill_workspace(16, 1024, 64)

    def call(s=sel, x=fake, r=64, c=cfg, B=fake, wb=ws, T=16):
        return f(ctypes.byref(s), x, fake, T, 1024, 64, None, None, ctypes.byref(c), r, B, fake, fake, fake, wb, None)

    assert call(r=32) == lib.AS_ERR_SHAPE
    assert call(x=None) == lib.AS_ERR_INVALID_ARG
    assert call(B=None) == lib.AS_ERR_INVALID_ARG
    assert call(c=lib.config(var=True, sel=lib.AS_SEL_NM, n=2, m=4)) == lib.AS_ERR_UNSUPPORTED
    assert call(B=fake + 4) == lib.AS_ERR_ALIGN
    assert call(wb=ws - 1) == lib.AS_ERR_WORKSPACE
    nomask = lib.as_select_out()
    nomask.x_compact = fake
    nomask.meta24 = fake
    assert call(s=nomask) == lib.AS_ERR_INVALID_ARG


def test_nm_split_validation_launches_nothing(lib):
    fake = 1 << 20
    cfg = lib.config(sel=lib.AS_SEL_NM, n=16, m=32)
    sel = lib.select_out(x_masked=fake, x_compact=fake, meta24=fake, bitmask24=fake)
    f = lib._lib.as_linear_prefill_nm_split
    ws = lib.as_hybrid_workspace(256, 1024, 256, 16)

    def call(s=sel, c=cfg, nd=16, wb=ws, K=1024):
        return f(ctypes.byref(s), 256, K, fake, 256, nd, ctypes.byref(c), None, None, None, fake, None, None, fake,
                 wb, None)

    assert call(c=lib.config(sel=lib.AS_SEL_NM, n=2, m=4)) == lib.AS_ERR_UNSUPPORTED   # already 2:4
    assert call(c=lib.config(sel=lib.AS_SEL_TOPK, k_keep=10)) == lib.AS_ERR_UNSUPPORTED
    assert call(nd=17) == lib.AS_ERR_SHAPE
    assert call(K=1000) == lib.AS_ERR_SHAPE
    assert call(s=lib.select_out(x_masked=fake, x_compact=fake, meta24=fake)) == lib.AS_ERR_INVALID_ARG
    assert call(c=lib.config(sel=lib.AS_SEL_NM, n=16, m=32, dpts=True)) == lib.AS_ERR_INVALID_ARG  # no eta/rowsum
    assert call(wb=ws - 1) == lib.AS_ERR_WORKSPACE
    # as_select: the 2:4 part needs an N:M selection with m a multiple of 4, m >= 8
    sel_f = lib._lib.as_select
    out = lib.select_out(x_masked=fake, x_compact=fake, meta24=fake, bitmask24=fake)
    for c in (lib.config(sel=lib.AS_SEL_NM, n=2, m=4), lib.config(sel=lib.AS_SEL_TOPK, k_keep=3)):
        assert sel_f(fake, lib.AS_BF16, 4, 64, ctypes.byref(c), None, None, 0, ctypes.byref(out), None, 0,
                     None) == lib.AS_ERR_UNSUPPORTED
    nomask = lib.select_out(x_compact=fake, meta24=fake, bitmask24=fake)
    assert sel_f(fake, lib.AS_BF16, 4, 64, ctypes.byref(cfg), None, None, 0, ctypes.byref(nomask), None, 0,
                 None) == lib.AS_ERR_INVALID_ARG


def test_select_stats_validation(lib):
    fake = 1 << 20
    f = lib._lib.as_select_stats
    assert f(None, lib.AS_BF16, fake, 4, 64, fake, fake, None) == lib.AS_ERR_INVALID_ARG
    assert f(fake, lib.AS_BF16, None, 4, 64, fake, fake, None) == lib.AS_ERR_INVALID_ARG
    assert f(fake, 7, fake, 4, 64, fake, fake, None) == lib.AS_ERR_DTYPE
    assert f(fake, lib.AS_BF16, fake, 0, 64, fake, fake, None) == lib.AS_ERR_SHAPE
    assert f(fake, lib.AS_BF16, fake, 4, 60, fake, fake, None) == lib.AS_ERR_SHAPE
    assert f(fake + 4, lib.AS_BF16, fake, 4, 64, fake, fake, None) == lib.AS_ERR_ALIGN
    assert f(fake, lib.AS_BF16, fake, 4, 64, None, None, None) == lib.AS_OK  # nothing asked, nothing launched
