"""Python binding of libactsparse, the B200 activation-sparsified linear layer.

Argument marshalling only: every step of the layer (weight preparation,
scores, selection, compensation statistics, the contraction) runs in the CUDA
kernels of ``libactsparse.so``; this module passes device pointers, sizes and
the current CUDA stream through the C ABI declared in ``include/actsparse.h``
and raises ``ASError`` for a non-zero status.  The functions keep the C names.

There is no CPU fallback: importing this package on a machine where the
library cannot be loaded raises immediately.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libactsparse.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python sparse_linear_b200/build.py` "
        "(nvcc, sm_100a) before using sparse_linear_b200")
_lib = ctypes.CDLL(LIB_PATH)

# ---------------------------------------------------------------- constants
AS_OK, AS_ERR_INVALID_ARG, AS_ERR_SHAPE, AS_ERR_DTYPE, AS_ERR_ALIGN = 0, 1, 2, 3, 4
AS_ERR_UNSUPPORTED, AS_ERR_WORKSPACE, AS_ERR_CUDA, AS_ERR_TIMEOUT = 5, 6, 7, 8
AS_ERR_BOUNDS = 9
AS_F32, AS_BF16 = 0, 1
AS_SCORE_MAG, AS_SCORE_WEIGHT, AS_SCORE_CLACT = 0, 1, 2
AS_SEL_NM, AS_SEL_TOPK, AS_SEL_ALL, AS_SEL_THRESH = 0, 1, 2, 3
AS_PTS_OFF, AS_PTS_DYNAMIC, AS_PTS_STATIC = 0, 1, 2
AS_OP_WEIGHT_PREP, AS_OP_SELECT, AS_OP_DECODE, AS_OP_PREFILL, AS_OP_AMBER = 0, 1, 2, 3, 4
AS_MAX_DECODE_T = 16
AS_MODE_24, AS_MODE_SPLIT, AS_MODE_DENSE = 0, 1, 2

EXPORTS = [
    "as_weight_prep", "as_select", "as_linear_decode", "as_linear_prefill",
    "as_workspace_size", "as_meta24_words", "as_stream_status", "as_status_string",
    "as_abi_version", "as_linear_decode_noalloc", "as_decode_launches", "as_probe_timeout",
    "as_weight_prep_amber", "as_meta8_words", "as_weight_quant_fp8", "as_select_sqrelu24_fp8",
    "as_linear_prefill_fp8", "as_rsparse_workspace", "as_rsparse_decode", "as_hybrid_workspace",
    "as_linear_prefill_hybrid", "as_block_sparsity", "as_prefill_mode", "as_hybrid_dense_blocks",
    "as_rsparse_prefill_workspace", "as_linear_prefill_rsparse", "as_linear_prefill_nm_split",
    "as_select_stats", "as_checked_line",
]
AS_NOALLOC_SCRATCH_BYTES = 8 << 20


class as_config(ctypes.Structure):
    _fields_ = [("score", ctypes.c_int32), ("sel", ctypes.c_int32), ("n", ctypes.c_int32),
                ("m", ctypes.c_int32), ("k_keep", ctypes.c_int32), ("dpts", ctypes.c_int32),
                ("var", ctypes.c_int32), ("var_momentum", ctypes.c_float),
                ("var_eps", ctypes.c_float), ("out_dtype", ctypes.c_int32),
                ("tau", ctypes.c_float), ("eta_static", ctypes.c_void_p)]


class as_select_out(ctypes.Structure):
    _fields_ = [(name, ctypes.c_void_p) for name in (
        "bitmask", "eta", "colnorm", "var_dense", "var_kept", "nu", "x_masked",
        "x_compact", "meta24", "x_masked_lo", "x_compact_lo", "bitmask24")]


_P, _I, _F, _S = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
_sig = {
    "as_weight_prep": ([_P, _I, _I, _I, _F, _P, _P, _P, _P, _S, _P], _I),
    "as_weight_prep_amber": ([_P, _I, _I, _I, _F, ctypes.c_double, ctypes.c_double, _P, _P, _P, _S, _P], _I),
    "as_meta8_words": ([_I, _I], _S),
    "as_rsparse_workspace": ([_I, _I, _I], _S),
    "as_hybrid_workspace": ([_I, _I, _I, _I], _S),
    "as_linear_prefill_hybrid": ([ctypes.POINTER(as_select_out), _P, _I, _I, _P, _I, _I, _I, _P, _P, _P, _P, _S,
                                  _P], _I),
    "as_block_sparsity": ([_P, _I, _I, _I, _P, _P, _P, _S, _P], _I),
    "as_select_stats": ([_P, _I, _P, _I, _I, _P, _P, _P], _I),
    "as_checked_line": ([], _I),
    "as_rsparse_decode": ([_P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _S, _P], _I),
    "as_weight_quant_fp8": ([_P, _I, _I, _I, _P, _P, _P], _I),
    "as_select_sqrelu24_fp8": ([_P, _I, _I, _P, _P, _P, _P, _P], _I),
    "as_linear_prefill_fp8": ([_P, _P, _P, _I, _I, _I, _P, _P, _I, _P, _P], _I),
    "as_select": ([_P, _I, _I, _I, ctypes.POINTER(as_config), _P, _P, _I,
                   ctypes.POINTER(as_select_out), _P, _S, _P], _I),
    "as_linear_decode": ([_P, _I, _I, _I, _I, _P, _P, _P, ctypes.POINTER(as_config), _P, _P, _P, _P,
                          _P, _S, _P], _I),
    "as_linear_prefill": ([ctypes.POINTER(as_select_out), _P, _I, _I, _I, _P, _P, _P,
                           ctypes.POINTER(as_config), _P, _P, _S, _P], _I),
    "as_linear_decode_noalloc": ([_P, _I, _I, _I, _I, _P, _P, _P, ctypes.POINTER(as_config), _P, _P, _P,
                                  _P, _P], _I),
    "as_workspace_size": ([_I, _I, _I, _I, ctypes.POINTER(as_config)], _S),
    "as_meta24_words": ([_I, _I], _S),
    "as_decode_launches": ([_I, _I, _I, _I, ctypes.POINTER(as_config)], _I),
    "as_stream_status": ([_P], _I),
    "as_probe_timeout": ([ctypes.c_uint, _P], _I),
    "as_status_string": ([_I], ctypes.c_char_p),
    "as_abi_version": ([], _I),
    "as_prefill_mode": ([ctypes.c_double], _I),
    "as_rsparse_prefill_workspace": ([_I, _I, _I], _S),
    "as_linear_prefill_nm_split": ([ctypes.POINTER(as_select_out), _I, _I, _P, _I, _I, ctypes.POINTER(as_config),
                                    _P, _P, _P, _P, _P, _P, _P, _S, _P], _I),
    "as_linear_prefill_rsparse": ([ctypes.POINTER(as_select_out), _P, _P, _I, _I, _I, _P, _P,
                                   ctypes.POINTER(as_config), _I, _P, _P, _P, _P, _S, _P], _I),
    "as_hybrid_dense_blocks": ([_I, ctypes.c_double], _I),
}
for _name, (_args, _res) in _sig.items():
    _fn = getattr(_lib, _name)
    _fn.argtypes = _args
    _fn.restype = _res


class ASError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {_lib.as_status_string(code).decode()}")


def _check(code: int, where: str) -> None:
    if code != AS_OK:
        raise ASError(code, where)


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("libactsparse takes device tensors; got a CPU tensor")
    if not t.is_contiguous():
        raise ValueError("libactsparse takes contiguous (row-major) tensors")
    return t.data_ptr()


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return AS_BF16
    if t.dtype == torch.float32:
        return AS_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def config(score: int = AS_SCORE_MAG, sel: int = AS_SEL_NM, n: int = 2, m: int = 4, k_keep: int = 0,
           dpts: int = AS_PTS_OFF, var: bool = False, var_momentum: float = 0.9, var_eps: float = 1e-6,
           out_dtype: int = AS_BF16, tau: float = 0.0, eta_static=None) -> as_config:
    """dpts: False/0 off, True/1 D-PTS, 2 S-PTS (eta_static: device [T] float32,
    kept alive by the caller for as long as the config is used)."""
    return as_config(score, sel, n, m, k_keep, int(dpts), int(var), var_momentum, var_eps, out_dtype,
                     float(tau), _ptr(eta_static))


def select_out(**bufs) -> as_select_out:
    o = as_select_out()
    for k, v in bufs.items():
        setattr(o, k, _ptr(v))
    return o


# ---------------------------------------------------------------- entry points
def as_abi_version() -> int:
    return _lib.as_abi_version()


def as_status_string(code: int) -> str:
    return _lib.as_status_string(code).decode()


def as_workspace_size(op: int, T: int, K: int, n_out: int, cfg: as_config | None) -> int:
    r = _lib.as_workspace_size(op, T, K, n_out, ctypes.byref(cfg) if cfg is not None else None)
    if r == ctypes.c_size_t(-1).value:
        raise ASError(AS_ERR_INVALID_ARG, "as_workspace_size")
    return r


def as_decode_launches(T: int, K: int, n_out: int, dtype: int, cfg: as_config) -> int:
    return _lib.as_decode_launches(T, K, n_out, dtype, ctypes.byref(cfg))


def as_meta24_words(T: int, K: int) -> int:
    return _lib.as_meta24_words(T, K)


def as_weight_prep(W, alpha: float, Wt=None, g=None, rowsum=None, workspace=None, stream=None) -> None:
    n_out, K = W.shape
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(_lib.as_weight_prep(_ptr(W), _dt(W), n_out, K, float(alpha), _ptr(Wt), _ptr(g), _ptr(rowsum),
                               _ptr(workspace), ws_bytes, _stream(stream)), "as_weight_prep")


def as_weight_prep_amber(W, g, alpha: float = 1.0, lo_pct: float = 0.5, hi_pct: float = 99.5,
                         bounds=None, workspace=None, stream=None) -> None:
    n_out, K = W.shape
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(_lib.as_weight_prep_amber(_ptr(W), _dt(W), n_out, K, float(alpha), float(lo_pct), float(hi_pct),
                                     _ptr(g), _ptr(bounds), _ptr(workspace), ws_bytes, _stream(stream)),
           "as_weight_prep_amber")


def as_hybrid_workspace(T: int, K: int, n_out: int, n_dense: int) -> int:
    n = _lib.as_hybrid_workspace(T, K, n_out, n_dense)
    if n == ctypes.c_size_t(-1).value:
        raise ASError(AS_ERR_SHAPE, "as_hybrid_workspace")
    return n


def as_linear_prefill_hybrid(out: as_select_out, x, W, y, n_dense: int, dense_idx=None, sparsity=None,
                             workspace=None, stream=None) -> None:
    T, K = x.shape
    n_out = W.shape[0]
    odt = AS_BF16 if y.dtype == torch.bfloat16 else AS_F32
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(_lib.as_linear_prefill_hybrid(ctypes.byref(out), _ptr(x), T, K, _ptr(W), n_out, int(n_dense), odt,
                                         _ptr(y), _ptr(dense_idx), _ptr(sparsity), _ptr(workspace), ws_bytes,
                                         _stream(stream)), "as_linear_prefill_hybrid")


def as_block_sparsity(x, sparsity, n_dense: int = 0, dense_idx=None, workspace=None, stream=None) -> None:
    T, K = x.shape
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(_lib.as_block_sparsity(_ptr(x), T, K, int(n_dense), _ptr(dense_idx), _ptr(sparsity), _ptr(workspace),
                                  ws_bytes, _stream(stream)), "as_block_sparsity")


def as_checked_line() -> int:
    """Checked builds: source line of the first failed index check (0: none)."""
    return _lib.as_checked_line()


def as_select_stats(x, bitmask, kept=None, nz_dropped=None, stream=None) -> None:
    """Per-token kept count and natural nonzeros dropped (int32 [T] each)."""
    T, K = x.shape
    dt = AS_BF16 if x.dtype == torch.bfloat16 else AS_F32
    _check(_lib.as_select_stats(_ptr(x), dt, _ptr(bitmask), T, K, _ptr(kept), _ptr(nz_dropped), _stream(stream)),
           "as_select_stats")


def as_prefill_mode(sparsity: float) -> int:
    """The mode switch of the 2:4 + Squared-ReLU page (section 3.3), run in
    the library: AS_MODE_24, AS_MODE_SPLIT or AS_MODE_DENSE."""
    return _lib.as_prefill_mode(float(sparsity))


def as_hybrid_dense_blocks(K: int, dense_frac: float) -> int:
    n = _lib.as_hybrid_dense_blocks(int(K), float(dense_frac))
    if n < 0:
        raise ASError(AS_ERR_SHAPE, "as_hybrid_dense_blocks")
    return n


def as_rsparse_workspace(T: int, K: int, r: int) -> int:
    n = _lib.as_rsparse_workspace(T, K, r)
    if n == ctypes.c_size_t(-1).value:
        raise ASError(AS_ERR_SHAPE, "as_rsparse_workspace")
    return n


def as_rsparse_decode(x, mask, B, A, y, eta=None, workspace=None, stream=None) -> None:
    """y (float32, in/out) += R-Sparse compensation of the dropped channels."""
    T, K = x.shape
    n_out, r = A.shape
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(_lib.as_rsparse_decode(_ptr(x), _dt(x), T, K, n_out, r, _ptr(mask), _ptr(eta), _ptr(B), _ptr(A),
                                  _ptr(y), _ptr(workspace), ws_bytes, _stream(stream)), "as_rsparse_decode")


def as_meta8_words(T: int, K: int) -> int:
    return _lib.as_meta8_words(T, K)


def as_weight_quant_fp8(W, Wq, w_scale, stream=None) -> None:
    n_out, K = W.shape
    _check(_lib.as_weight_quant_fp8(_ptr(W), _dt(W), n_out, K, _ptr(Wq), _ptr(w_scale), _stream(stream)),
           "as_weight_quant_fp8")


def as_select_sqrelu24_fp8(z, x8, meta8, x_scale, bitmask=None, stream=None) -> None:
    T, K = z.shape
    _check(_lib.as_select_sqrelu24_fp8(_ptr(z), T, K, _ptr(x8), _ptr(meta8), _ptr(x_scale), _ptr(bitmask),
                                       _stream(stream)), "as_select_sqrelu24_fp8")


def as_linear_prefill_fp8(x8, meta8, x_scale, Wq, w_scale, y, stream=None) -> None:
    T = x8.shape[0]
    n_out, K = Wq.shape
    out = AS_BF16 if y.dtype == torch.bfloat16 else AS_F32
    _check(_lib.as_linear_prefill_fp8(_ptr(x8), _ptr(meta8), _ptr(x_scale), T, K, n_out, _ptr(Wq), _ptr(w_scale),
                                      out, _ptr(y), _stream(stream)), "as_linear_prefill_fp8")


def as_select(x, cfg: as_config, out: as_select_out, chan_factor=None, running_var=None,
              var_first_batch: bool = False, workspace=None, stream=None) -> None:
    T, K = x.shape
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(_lib.as_select(_ptr(x), _dt(x), T, K, ctypes.byref(cfg), _ptr(chan_factor), _ptr(running_var),
                          int(var_first_batch), ctypes.byref(out), _ptr(workspace), ws_bytes,
                          _stream(stream)), "as_select")


def as_linear_decode(x, Wt, cfg: as_config, y, g=None, rowsum=None, mask_out=None, eta_out=None,
                     colnorm_out=None, workspace=None, stream=None) -> None:
    T, K = x.shape
    n_out = Wt.shape[1]
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(_lib.as_linear_decode(_ptr(x), _dt(x), T, K, n_out, _ptr(Wt), _ptr(g), _ptr(rowsum),
                                 ctypes.byref(cfg), _ptr(y), _ptr(mask_out), _ptr(eta_out),
                                 _ptr(colnorm_out), _ptr(workspace), ws_bytes, _stream(stream)),
           "as_linear_decode")


class DecodeCall:
    """as_linear_decode with a layer's fixed arguments (Wt, cfg, g, rowsum,
    workspace, stream) converted once; each call passes x and y.  For
    decode loops where the per-call marshalling would otherwise cost more
    host time than the GPU spends."""

    def __init__(self, Wt, cfg: as_config, g=None, rowsum=None, workspace=None, stream=None):
        self._K, self._n_out = Wt.shape
        self._dt = _dt(Wt)
        self._cfg = cfg  # keeps the structure alive
        self._args = (_ptr(Wt), _ptr(g), _ptr(rowsum), ctypes.byref(cfg))
        self._ws = _ptr(workspace)
        self._wsb = workspace.numel() * workspace.element_size() if workspace is not None else 0
        self._st = _stream(stream)
        self._fn = _lib.as_linear_decode

    def __call__(self, x, y, mask_out=None, eta_out=None, colnorm_out=None) -> None:
        if _dt(x) != self._dt:
            raise TypeError("x must have the weights' dtype")
        wt, g, rs, cfgp = self._args
        code = self._fn(_ptr(x), self._dt, x.shape[0], self._K, self._n_out, wt, g, rs, cfgp, _ptr(y),
                        _ptr(mask_out), _ptr(eta_out), _ptr(colnorm_out), self._ws, self._wsb, self._st)
        if code != AS_OK:
            raise ASError(code, "as_linear_decode")


def as_linear_decode_noalloc(x, Wt, cfg: as_config, y, g=None, rowsum=None, mask_out=None, eta_out=None,
                             colnorm_out=None, stream=None) -> None:
    """as_linear_decode without a workspace argument: the scratch is the
    library's own fixed device array (see include/actsparse.h)."""
    T, K = x.shape
    n_out = Wt.shape[1]
    _check(_lib.as_linear_decode_noalloc(_ptr(x), _dt(x), T, K, n_out, _ptr(Wt), _ptr(g), _ptr(rowsum),
                                         ctypes.byref(cfg), _ptr(y), _ptr(mask_out), _ptr(eta_out),
                                         _ptr(colnorm_out), _stream(stream)),
           "as_linear_decode_noalloc")


def as_linear_prefill(sel: as_select_out, W, T: int, cfg: as_config, y, rowsum=None, eta=None, nu=None,
                      workspace=None, stream=None) -> None:
    n_out, K = W.shape
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(_lib.as_linear_prefill(ctypes.byref(sel), _ptr(W), T, K, n_out, _ptr(rowsum), _ptr(eta), _ptr(nu),
                                  ctypes.byref(cfg), _ptr(y), _ptr(workspace), ws_bytes, _stream(stream)),
           "as_linear_prefill")


def as_rsparse_prefill_workspace(T: int, K: int, r: int) -> int:
    n = _lib.as_rsparse_prefill_workspace(T, K, r)
    if n == ctypes.c_size_t(-1).value:
        raise ASError(AS_ERR_SHAPE, "as_rsparse_prefill_workspace")
    return n


def as_linear_prefill_rsparse(sel: as_select_out, x, W, cfg: as_config, y, B, A, rowsum=None, eta=None,
                              workspace=None, stream=None) -> None:
    """as_linear_prefill plus the R-Sparse compensation of the dropped
    channels through the rank-r factors B [K, r] and A [n_out, r]."""
    T, K = x.shape
    n_out = W.shape[0]
    r = A.shape[1]
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(_lib.as_linear_prefill_rsparse(ctypes.byref(sel), _ptr(x), _ptr(W), T, K, n_out, _ptr(rowsum), _ptr(eta),
                                          ctypes.byref(cfg), r, _ptr(B), _ptr(A), _ptr(y), _ptr(workspace), ws_bytes,
                                          _stream(stream)), "as_linear_prefill_rsparse")


def as_linear_prefill_nm_split(sel: as_select_out, T: int, W, cfg: as_config, y, n_dense: int, rowsum=None,
                               eta=None, nu=None, dense_idx=None, sparsity=None, workspace=None, stream=None) -> None:
    """Hybrid 2:4 decomposition of an N:M selection (see include/actsparse.h)."""
    n_out, K = W.shape
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(_lib.as_linear_prefill_nm_split(ctypes.byref(sel), T, K, _ptr(W), n_out, int(n_dense), ctypes.byref(cfg),
                                           _ptr(rowsum), _ptr(eta), _ptr(nu), _ptr(y), _ptr(dense_idx),
                                           _ptr(sparsity), _ptr(workspace), ws_bytes, _stream(stream)),
           "as_linear_prefill_nm_split")


def as_stream_status(stream=None) -> int:
    return _lib.as_stream_status(_stream(stream))


def as_probe_timeout(polls: int = 1000, stream=None) -> None:
    """Runs the failure-path self-test kernel (a bounded wait that runs out)."""
    _check(_lib.as_probe_timeout(int(polls), _stream(stream)), "as_probe_timeout")
