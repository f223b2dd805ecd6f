"""CPU oracle for the activation-sparsified linear layer (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It shares no code with the CUDA
library ``sparse_linear_b200`` and never imports it.

``oracle.c`` holds the float64 definitions (plus the float32 score/selection
decision); this module compiles it with gcc on first use, loads it with
ctypes and wraps each function for numpy arrays.  ``brute.py`` holds an
independent pure-Python enumerator for tiny cases.

Functions and the passages they follow (page title, section):

* ``weight_prep``   WiSparse page §2.1 eq. (4) (g) and activation-sparsity
                    overview §3.1 (rowsum for the mean shift).
* ``amber``         overview §2.2.2 (Amber-Pruner channel importance).
* ``token_mean``    overview §3.1 (D-PTS eta).
* ``token_var``     overview §3.2 (VAR, unbiased variance).
* ``channel_energy``/``clact_full``  overview §2.2.3 (CLACT).
* ``score``         overview §2.2.1, §2.2.3, §3.1; WiSparse eq. (4).
* ``select_nm``     overview §2.1 / §2.2.1 (block top-N).
* ``select_topk``   WiSparse §2.2 (per-layer keep fraction).
* ``select_thresh`` WiSparse §3.1 / §5 (TEAL-style threshold tau).
  S-PTS (overview §3.1, static version) needs no function of its own:
  ``score`` and ``linear`` take the token shift eta as an input, dynamic
  (``token_mean``) or a calibrated table.
* ``var_scale``     overview §3.2.
* ``linear``        overview §3.1 / §3.2 and the layer definition y = prune(x) W^T.
* ``block_nnz``, ``pick_dense``, ``hybrid_mode``, ``hybrid_mask``, ``nm_split``
                    2:4 + Squared-ReLU page §3.2-3.3 (sparse/dense split of a
                    2:4 activation and of an N:M selection, mode switch).
* ``rsparse``, ``rsparse_factors``  overview §3.3 (R-Sparse low-rank compensation;
                    the factors from a truncated SVD, numpy's).
* ``compress_nm``   2:4 + Squared-ReLU page §3.3 (kept values stored contiguously).
* ``select_stats``  2:4 + Squared-ReLU page §2.3 (natural nonzeros a 2:4
                    selection must drop) and the kept count per token.
* ``e4m3_encode``/``e4m3_decode``, ``quant_rows_fp8``, ``sqrelu24_fp8``,
  ``linear_fp8``    2:4 + Squared-ReLU page §3.1 (fused Squared-ReLU + 2:4 +
                    FP8 producer, FP8 row-scaled GEMM) and §5.3 (sparsify
                    before quantising).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
          "-fno-fast-math", "-Wall"]


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` into ``liboracle.so`` (gcc, no CUDA)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            I = ctypes.c_int
            D = ctypes.c_double
            sig = {
                "or_weight_prep": [P, I, I, D, P, P],
                "or_amber": [P, I, I, D, D, D, P, P, P],
                "or_token_mean": [P, I, I, P],
                "or_token_var": [P, I, I, P],
                "or_channel_energy": [P, I, I, P],
                "or_clact_full": [P, I, I, P],
                "or_score": [P, I, I, P, P, P],
                "or_select_nm": [P, I, I, I, I, P],
                "or_select_topk": [P, I, I, I, P],
                "or_select_thresh": [P, I, I, ctypes.c_float, P],
                "or_var_scale": [P, P, I, I, P, D, D, P, P, P, P],
                "or_linear": [P, P, I, I, P, P, I, P, P, P, I, P],
                "or_compress_nm": [P, P, I, I, I, I, P, P],
                "or_quant_rows_fp8": [P, I, I, P, P],
                "or_rsparse": [P, P, I, I, P, P, P, I, I, P],
                "or_pick_dense": [P, I, I, P],
                "or_sqrelu24_fp8": [P, I, I, P, P, P, P, P],
            }
            for name, args in sig.items():
                fn = getattr(lib, name)
                fn.argtypes = args
                fn.restype = None
            lib.or_block_nnz.argtypes = [P, I, I, P]
            lib.or_block_nnz.restype = ctypes.c_longlong
            lib.or_e4m3_encode.argtypes = [D]
            lib.or_e4m3_encode.restype = ctypes.c_uint8
            lib.or_e4m3_decode.argtypes = [ctypes.c_uint8]
            lib.or_e4m3_decode.restype = D
            _lib = lib
    return _lib


def _f32(a):
    a = a.float().numpy() if hasattr(a, "numpy") and not isinstance(a, np.ndarray) else a
    return np.ascontiguousarray(a, dtype=np.float32)


def _ptr(a):
    return None if a is None else a.ctypes.data


def weight_prep(W, alpha: float):
    """g [k] = ||W[:,i]||_2^alpha and rowsum [n_out], float64."""
    W = _f32(W)
    n_out, k = W.shape
    g = np.empty(k, np.float64)
    rs = np.empty(n_out, np.float64)
    _load().or_weight_prep(_ptr(W), n_out, k, float(alpha), _ptr(g), _ptr(rs))
    return g, rs


def amber(W, alpha: float = 1.0, lo_pct: float = 0.5, hi_pct: float = 99.5):
    """Amber-Pruner importance g [k] (float64) and the two percentile values."""
    W = _f32(W)
    n_out, k = W.shape
    g = np.empty(k, np.float64)
    lo = ctypes.c_double()
    hi = ctypes.c_double()
    _load().or_amber(_ptr(W), n_out, k, float(alpha), float(lo_pct), float(hi_pct), _ptr(g),
                     ctypes.addressof(lo), ctypes.addressof(hi))
    return g, lo.value, hi.value


def token_mean(x):
    x = _f32(x)
    T, k = x.shape
    out = np.empty(T, np.float64)
    _load().or_token_mean(_ptr(x), T, k, _ptr(out))
    return out


def token_var(x):
    x = _f32(x)
    T, k = x.shape
    out = np.empty(T, np.float64)
    _load().or_token_var(_ptr(x), T, k, _ptr(out))
    return out


def channel_energy(x):
    x = _f32(x)
    T, k = x.shape
    out = np.empty(k, np.float64)
    _load().or_channel_energy(_ptr(x), T, k, _ptr(out))
    return out


def clact_full(x):
    x = _f32(x)
    T, k = x.shape
    out = np.empty((T, k), np.float64)
    _load().or_clact_full(_ptr(x), T, k, _ptr(out))
    return out


def score(x, eta=None, f=None):
    """float32 score: fl32(|fl32(x - eta)| * f) (eta, f optional, float32)."""
    x = _f32(x)
    T, k = x.shape
    e = None if eta is None else np.ascontiguousarray(eta, np.float32).reshape(T)
    ff = None if f is None else np.ascontiguousarray(f, np.float32).reshape(k)
    s = np.empty((T, k), np.float32)
    _load().or_score(_ptr(x), T, k, _ptr(e), _ptr(ff), _ptr(s))
    return s


def select_nm(s, n: int, m: int):
    s = np.ascontiguousarray(s, np.float32)
    T, k = s.shape
    if k % m:
        raise ValueError("k must be a multiple of m")
    mask = np.empty((T, k), np.uint8)
    _load().or_select_nm(_ptr(s), T, k, int(n), int(m), _ptr(mask))
    return mask


def select_topk(s, kk: int):
    s = np.ascontiguousarray(s, np.float32)
    T, k = s.shape
    mask = np.empty((T, k), np.uint8)
    _load().or_select_topk(_ptr(s), T, k, int(kk), _ptr(mask))
    return mask


def select_thresh(s, tau: float):
    s = np.ascontiguousarray(s, np.float32)
    T, k = s.shape
    mask = np.empty((T, k), np.uint8)
    _load().or_select_thresh(_ptr(s), T, k, ctypes.c_float(tau), _ptr(mask))
    return mask


def var_scale(x, mask, running_in=None, momentum: float = 0.9, eps: float = 1e-6):
    """Returns dict var_dense, var_kept, running, nu (float64 [T])."""
    x = _f32(x)
    T, k = x.shape
    mask = np.ascontiguousarray(mask, np.uint8)
    rin = None if running_in is None else np.ascontiguousarray(running_in, np.float64)
    out = {n: np.empty(T, np.float64) for n in ("var_dense", "var_kept", "running", "nu")}
    _load().or_var_scale(_ptr(x), _ptr(mask), T, k, _ptr(rin), float(momentum), float(eps),
                         _ptr(out["var_dense"]), _ptr(out["var_kept"]),
                         _ptr(out["running"]), _ptr(out["nu"]))
    return out


def linear(x, mask, W, eta=None, rowsum=None, nu=None, rows=None):
    """float64 y[r, o] over the kept channels (see oracle.c)."""
    x = _f32(x)
    W = _f32(W)
    T, k = x.shape
    n_out = W.shape[0]
    mask = np.ascontiguousarray(mask, np.uint8)
    e = None if eta is None else np.ascontiguousarray(eta, np.float64)
    rs = None if rowsum is None else np.ascontiguousarray(rowsum, np.float64)
    if e is not None and rs is None:
        raise ValueError("eta needs rowsum")
    nv = None if nu is None else np.ascontiguousarray(nu, np.float64)
    rr = None if rows is None else np.ascontiguousarray(rows, np.int32)
    n_rows = T if rr is None else len(rr)
    y = np.empty((n_rows, n_out), np.float64)
    _load().or_linear(_ptr(x), _ptr(mask), T, k, _ptr(e), _ptr(W), n_out, _ptr(rs),
                      _ptr(nv), _ptr(rr), n_rows, _ptr(y))
    return y


def compress_nm(v, mask, n: int, m: int):
    """Kept values of each block, contiguous in channel order, and positions."""
    v = _f32(v)
    T, k = v.shape
    mask = np.ascontiguousarray(mask, np.uint8)
    kc = k // m * n
    vals = np.empty((T, kc), np.float32)
    pos = np.empty((T, kc), np.uint8)
    _load().or_compress_nm(_ptr(v), _ptr(mask), T, k, int(n), int(m), _ptr(vals), _ptr(pos))
    return vals, pos


def e4m3_encode(v) -> np.ndarray:
    """E4M3 codes (uint8) of float64 values: nearest, ties to even, clamp at 448."""
    lib = _load()
    v = np.asarray(v, np.float64)
    return np.array([lib.or_e4m3_encode(float(a)) for a in v.reshape(-1)], np.uint8).reshape(v.shape)


def e4m3_decode(c) -> np.ndarray:
    """float64 values of E4M3 codes."""
    lib = _load()
    c = np.asarray(c, np.uint8)
    return np.array([lib.or_e4m3_decode(int(a)) for a in c.reshape(-1)], np.float64).reshape(c.shape)


def quant_rows_fp8(W):
    """W [n_out, k] -> (codes uint8 [n_out, k], scale float32 [n_out])."""
    W = _f32(W)
    n_out, k = W.shape
    codes = np.empty((n_out, k), np.uint8)
    scale = np.empty(n_out, np.float32)
    _load().or_quant_rows_fp8(_ptr(W), n_out, k, _ptr(codes), _ptr(scale))
    return codes, scale


def sqrelu24_fp8(z):
    """Fused producer from bf16 z [T, k] (torch tensor or uint16 bit array).

    Returns dict mask [T, k], codes [T, k/2], pos [T, k/2], scale [T], x [T, k].
    """
    if hasattr(z, "view") and not isinstance(z, np.ndarray):
        import torch
        z = z.contiguous().view(torch.int16).numpy().view(np.uint16)
    z = np.ascontiguousarray(z, np.uint16)
    T, k = z.shape
    if k % 4:
        raise ValueError("k must be a multiple of 4")
    out = dict(mask=np.empty((T, k), np.uint8), codes=np.empty((T, k // 2), np.uint8),
               pos=np.empty((T, k // 2), np.uint8), scale=np.empty(T, np.float32),
               x=np.empty((T, k), np.float32))
    _load().or_sqrelu24_fp8(_ptr(z), T, k, _ptr(out["mask"]), _ptr(out["codes"]), _ptr(out["pos"]),
                            _ptr(out["scale"]), _ptr(out["x"]))
    return out


_E4M3 = None


def _e4m3_table():
    global _E4M3
    if _E4M3 is None:
        _E4M3 = e4m3_decode(np.arange(256, dtype=np.uint8))
    return _E4M3


def dequant_fp8(codes, scale):
    """float64 codes * row scale."""
    return _e4m3_table()[np.asarray(codes, np.uint8)] * np.asarray(scale, np.float64).reshape(-1, 1)


def linear_fp8(x_codes, x_pos, x_scale, w_codes, w_scale, rows=None):
    """float64 y [T, n_out] of the FP8 2:4 GEMM: the kept values (codes at
    their block positions, times the token's scale) against the dequantised
    weight (codes times the output row's scale), summed in float64."""
    x_codes = np.asarray(x_codes, np.uint8)
    x_pos = np.asarray(x_pos, np.uint8)
    if rows is not None:
        x_codes, x_pos, x_scale = x_codes[rows], x_pos[rows], np.asarray(x_scale)[rows]
    T, kc = x_codes.shape
    k = 2 * kc
    xd = np.zeros((T, k), np.float64)
    col = (np.arange(kc) // 2) * 4 + x_pos.astype(np.int64)
    np.put_along_axis(xd, col, dequant_fp8(x_codes, x_scale), axis=1)
    return xd @ dequant_fp8(w_codes, w_scale).T


def rsparse_factors(W, r: int):
    """A_r = U_r diag(S_r) [n_out, r] and B_r = V_r [k, r] from numpy's SVD of
    W [n_out, k] in float64 (overview page §3.3)."""
    W64 = np.asarray(W.float().numpy() if hasattr(W, "numpy") and not isinstance(W, np.ndarray) else W,
                     np.float64)
    U, S, Vh = np.linalg.svd(W64, full_matrices=False)
    return U[:, :r] * S[:r], Vh[:r, :].T.copy()


def rsparse(x, mask, B, A, eta=None):
    """float64 compensation [T, n_out] = (xhat * (1 - mask)) B A^T."""
    x = _f32(x)
    T, k = x.shape
    B = _f32(B)
    A = _f32(A)
    r = B.shape[1]
    n_out = A.shape[0]
    mask = np.ascontiguousarray(mask, np.uint8)
    e = None if eta is None else np.ascontiguousarray(eta, np.float64)
    comp = np.empty((T, n_out), np.float64)
    _load().or_rsparse(_ptr(x), _ptr(mask), T, k, _ptr(e), _ptr(B), _ptr(A), n_out, r, _ptr(comp))
    return comp


def select_stats(x, mask):
    """Per token: the number of kept channels and the number of channels with
    x != 0 that the selection dropped (the 2:4 + Squared-ReLU page §2.3: a
    4-block with three natural nonzeros has to lose one of them).  Plain
    counting over the definition; int64 [T] each."""
    x = np.asarray(x, np.float64)
    mask = np.asarray(mask).astype(bool)
    kept = mask.sum(axis=1, dtype=np.int64)
    dropped = ((x != 0.0) & ~mask).sum(axis=1, dtype=np.int64)
    return kept, dropped


def block_nnz(x):
    """Nonzeros per 4-channel block over all tokens [k/4] and the total."""
    x = _f32(x)
    T, k = x.shape
    nnz = np.empty(k // 4, np.int32)
    total = _load().or_block_nnz(_ptr(x), T, k, _ptr(nnz))
    return nnz, int(total)


def pick_dense(nnz, n_dense: int):
    """Block indices (ascending) of the n_dense blocks with the most nonzeros."""
    nnz = np.ascontiguousarray(nnz, np.int32)
    idx = np.empty(n_dense, np.int32)
    _load().or_pick_dense(_ptr(nnz), len(nnz), int(n_dense), _ptr(idx))
    return idx


def hybrid_mode(sparsity: float) -> str:
    """The 2:4 + Squared-ReLU page §3.3: above 95 % pure 2:4, 90-95 % split,
    below 90 % dense."""
    if sparsity > 0.95:
        return "2:4"
    if sparsity >= 0.90:
        return "split"
    return "dense"


def nm_split(s, mask_nm, xm, n_dense: int):
    """The hybrid 2:4 decomposition of an N:M selection (2:4 + Squared-ReLU
    page §3.2, the sparse/dense feature split, applied to an N:M selection;
    §3.3 for the mode).  Readings:
    * the 2:4-compliant part takes, in every 4-channel block, the two
      channels ranked first by (kept by the N:M selection, then higher
      float32 score, then lower index); a block with fewer than two kept
      channels fills its positions with the lowest-indexed dropped ones,
      whose values are zero (``pos``, exactly 2 per block);
    * ``part`` = the kept channels inside the 2:4 part;
    * the dense blocks D are the n_dense blocks with the most nonzeros of
      the masked activation xm = xhat * mask over the tokens (ties to the
      lower block index), as in ``hybrid_mask``;
    * the split keeps ``part`` plus every kept channel of D:
      m_split = part | (mask_nm & D); with D covering every block whose
      kept channels do not fit 2:4, m_split equals mask_nm.
    s, mask_nm, xm: [T, k]; returns dict(pos, part, idx, m_split, sparsity)."""
    s = np.asarray(s, np.float32)
    kept = np.asarray(mask_nm, np.uint8).astype(bool)
    T, k = s.shape
    sb = s.reshape(T, k // 4, 4)
    kb = kept.reshape(T, k // 4, 4)
    rank = np.zeros((T, k // 4, 4), np.int64)
    for i in range(4):
        for j in range(4):
            if i == j:
                continue
            # kept before dropped; kept ones by score, then index; dropped
            # ones (zero-valued padding) by index alone
            both_kept = kb[..., j] & kb[..., i]
            both_dropped = ~kb[..., j] & ~kb[..., i]
            beats = (kb[..., j] & ~kb[..., i]) | (both_kept & ((sb[..., j] > sb[..., i]) |
                                                               ((sb[..., j] == sb[..., i]) & (j < i)))) | \
                    (both_dropped & (j < i))
            rank[..., i] += beats
    pos = (rank < 2).reshape(T, k)
    part = pos & kept
    nnz, total = block_nnz(np.asarray(xm, np.float32))
    idx = pick_dense(nnz, n_dense)
    dense = np.zeros(k, bool)
    for b in idx:
        dense[4 * b:4 * b + 4] = True
    m_split = part | (kept & dense[None, :])
    return dict(pos=pos.astype(np.uint8), part=part.astype(np.uint8), idx=idx,
                m_split=m_split.astype(np.uint8), sparsity=1.0 - total / float(T * k))


def hybrid_mask(x, n_dense: int):
    """Mask of the split: all channels of the dense blocks, 2:4 by magnitude
    elsewhere; returns (mask, dense block indices, sparsity)."""
    x = _f32(x)
    T, k = x.shape
    nnz, total = block_nnz(x)
    idx = pick_dense(nnz, n_dense)
    mask = select_nm(score(x), 2, 4)
    for b in idx:
        mask[:, 4 * b:4 * b + 4] = 1
    return mask, idx, 1.0 - total / float(T * k)
