"""Buffer management around the C ABI: a prepared sparse linear layer.

``SparseLinear`` owns the per-layer tensors (channel-major weight copy,
weight-aware channel factors, row sums) and a zero-filled workspace, all
allocated through torch on the current CUDA device, and calls the C entry
points.  It performs no arithmetic of its own.
"""
from __future__ import annotations

import torch

from . import (AS_BF16, AS_F32, AS_MODE_24, AS_MODE_DENSE, AS_MODE_SPLIT, AS_OP_AMBER, AS_OP_DECODE,
               AS_OP_PREFILL, AS_OP_SELECT, AS_OP_WEIGHT_PREP, AS_SCORE_CLACT, AS_SCORE_MAG, AS_SEL_ALL, AS_SEL_NM,
               as_block_sparsity, as_hybrid_dense_blocks, as_hybrid_workspace, as_linear_decode, as_linear_prefill,
               as_linear_prefill_hybrid, as_linear_prefill_nm_split, as_linear_prefill_rsparse, as_meta24_words,
               as_prefill_mode,
               as_rsparse_prefill_workspace, as_select, as_weight_prep, as_weight_prep_amber, as_workspace_size,
               config, select_out)


_MODE_NAMES = {AS_MODE_24: "2:4", AS_MODE_SPLIT: "split", AS_MODE_DENSE: "dense"}


def hybrid_mode(sparsity: float) -> str:
    """Name of the mode the library's switch (as_prefill_mode) picks for a
    layer's measured sparsity."""
    return _MODE_NAMES[as_prefill_mode(sparsity)]


def dense_blocks_for(K: int, dense_frac: float) -> int:
    """Dense 4-channel blocks of the split (as_hybrid_dense_blocks)."""
    return as_hybrid_dense_blocks(K, dense_frac)


def workspace(nbytes: int, device) -> torch.Tensor:
    """Zero-filled byte buffer (the ABI requires zeros before first use)."""
    return torch.zeros(max(int(nbytes), 16), dtype=torch.uint8, device=device)


class SparseLinear:
    """One activation-sparsified linear layer y = prune(x) W^T.

    W: [n_out, K] bf16 or f32 CUDA tensor (PyTorch Linear layout).
    cfg: ``as_config``; ``alpha`` is the weight-aware exponent.
    ``keep_wt`` builds the channel-major copy needed by the decode path.
    ``importance`` picks the channel factor g of the weight-aware score:
    ``"norm"`` (column norm of W) or ``"amber"`` (Amber-Pruner: column norm
    of the standardised weights inside the ``amber_pct`` percentiles).
    """

    def __init__(self, W: torch.Tensor, cfg, alpha: float = 0.0, keep_wt: bool = True,
                 importance: str = "norm", amber_pct: tuple[float, float] = (0.5, 99.5)):
        if importance not in ("norm", "amber"):
            raise ValueError(f"unknown importance {importance!r}")
        self.W = W.contiguous()
        self.cfg = cfg
        self.alpha = float(alpha)
        self.n_out, self.K = W.shape
        dev = W.device
        self.g = torch.empty(self.K, dtype=torch.float32, device=dev)
        self.rowsum = torch.empty(self.n_out, dtype=torch.float32, device=dev)
        self.Wt = torch.empty(self.K, self.n_out, dtype=W.dtype, device=dev) if keep_wt else None
        ws = workspace(as_workspace_size(AS_OP_WEIGHT_PREP, 0, self.K, self.n_out, None), dev)
        amber = importance == "amber"
        as_weight_prep(self.W, self.alpha, Wt=self.Wt, g=None if amber else self.g, rowsum=self.rowsum,
                       workspace=ws)
        self.amber_bounds = None
        if amber:
            self.amber_bounds = torch.empty(4, dtype=torch.float32, device=dev)
            ws = workspace(as_workspace_size(AS_OP_AMBER, 0, self.K, self.n_out, None), dev)
            as_weight_prep_amber(self.W, self.g, self.alpha, amber_pct[0], amber_pct[1],
                                 bounds=self.amber_bounds, workspace=ws)
        self._ws = {}

    def _workspace(self, op: int, T: int) -> torch.Tensor:
        key = (op, T)
        if key not in self._ws:
            self._ws[key] = workspace(as_workspace_size(op, T, self.K, self.n_out, self.cfg), self.W.device)
        return self._ws[key]

    def out_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.cfg.out_dtype == AS_BF16 else torch.float32

    # ---------------------------------------------------------------- decode
    def decode(self, x: torch.Tensor, y: torch.Tensor | None = None, mask_out=None, eta_out=None,
               colnorm_out=None, stream=None) -> torch.Tensor:
        T = x.shape[0]
        if y is None:
            y = torch.empty(T, self.n_out, dtype=self.out_dtype(), device=x.device)
        as_linear_decode(x, self.Wt, self.cfg, y, g=self.g, rowsum=self.rowsum, mask_out=mask_out,
                         eta_out=eta_out, colnorm_out=colnorm_out,
                         workspace=self._workspace(AS_OP_DECODE, T), stream=stream)
        return y

    # ---------------------------------------------------------------- prefill
    def select_buffers(self, T: int, device=None) -> dict:
        """Device buffers for every as_select output this layer's cfg uses."""
        dev = device or self.W.device
        K = self.K
        c = self.cfg
        b = dict(bitmask=torch.empty(T, (K + 31) // 32, dtype=torch.int32, device=dev),
                 eta=torch.empty(T, dtype=torch.float32, device=dev),
                 colnorm=torch.empty(K, dtype=torch.float32, device=dev))
        if c.var:
            for k in ("var_dense", "var_kept", "nu"):
                b[k] = torch.empty(T, dtype=torch.float32, device=dev)
        # float32 output with a token shift: the kept values also go in as
        # their bf16 residuals (a second pass of the GEMM over K)
        lo = c.out_dtype == AS_F32 and bool(c.dpts) and self.W.dtype == torch.bfloat16
        if c.sel == AS_SEL_NM and c.n == 2 and c.m == 4 and self.W.dtype == torch.bfloat16:
            b["x_compact"] = torch.empty(T, K // 2, dtype=torch.bfloat16, device=dev)
            b["meta24"] = torch.empty(as_meta24_words(T, K), dtype=torch.int32, device=dev)
            if lo:
                b["x_compact_lo"] = torch.empty(T, K // 2, dtype=torch.bfloat16, device=dev)
        else:
            b["x_masked"] = torch.empty(T, K, dtype=self.W.dtype, device=dev)
            if lo:
                b["x_masked_lo"] = torch.empty(T, K, dtype=torch.bfloat16, device=dev)
        return b

    def select(self, x: torch.Tensor, bufs: dict, running_var=None, first_batch: bool = False,
               stream=None) -> None:
        T = x.shape[0]
        chan = self.g if self.cfg.score != AS_SCORE_CLACT else None
        as_select(x, self.cfg, select_out(**bufs), chan_factor=chan, running_var=running_var,
                  var_first_batch=first_batch, workspace=self._workspace(AS_OP_SELECT, T), stream=stream)

    def prefill_from(self, bufs: dict, T: int, y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        if y is None:
            y = torch.empty(T, self.n_out, dtype=self.out_dtype(), device=self.W.device)
        as_linear_prefill(select_out(**{k: v for k, v in bufs.items()
                                        if k in ("x_masked", "x_compact", "meta24", "x_masked_lo",
                                                 "x_compact_lo")}),
                          self.W, T, self.cfg, y, rowsum=self.rowsum, eta=bufs.get("eta"),
                          nu=bufs.get("nu"), workspace=self._workspace(AS_OP_PREFILL, T), stream=stream)
        return y

    # ---------------------------------------------------------------- hybrid 2:4
    def prefill_hybrid_from(self, x: torch.Tensor, bufs: dict, n_dense: int, y: torch.Tensor | None = None,
                            dense_idx=None, sparsity=None, stream=None) -> torch.Tensor:
        """The split of the 2:4 + Squared-ReLU page (section 3.2): the n_dense
        busiest 4-channel blocks dense, 2:4 elsewhere.  `bufs` holds this
        layer's 2:4 selection of x (cfg: 2:4 by magnitude)."""
        T = x.shape[0]
        if y is None:
            y = torch.empty(T, self.n_out, dtype=self.out_dtype(), device=x.device)
        key = ("hybrid", T, n_dense)
        if key not in self._ws:
            self._ws[key] = workspace(as_hybrid_workspace(T, self.K, self.n_out, n_dense), x.device)
        sel = select_out(**{k: v for k, v in bufs.items() if k in ("bitmask", "x_compact", "meta24")})
        as_linear_prefill_hybrid(sel, x, self.W, y, n_dense, dense_idx=dense_idx, sparsity=sparsity,
                                 workspace=self._ws[key], stream=stream)
        return y

    def prefill_auto(self, x: torch.Tensor, dense_frac: float = 0.05, stream=None):
        """Mode chosen by the library's switch (as_prefill_mode) on the
        measured sparsity of x, with as_hybrid_dense_blocks(K, dense_frac)
        dense blocks for the split.  Reads the sparsity back to the host (one
        synchronisation).  Returns (y, mode, sparsity)."""
        if not (self.cfg.sel == AS_SEL_NM and self.cfg.n == 2 and self.cfg.m == 4
                and self.cfg.score == AS_SCORE_MAG and not self.cfg.dpts and not self.cfg.var):
            raise ValueError("prefill_auto needs a 2:4 magnitude configuration")
        T = x.shape[0]
        key = ("sparsity", T)
        if key not in self._ws:
            self._ws[key] = workspace(as_hybrid_workspace(T, self.K, 0, 0), x.device)
        sp = torch.empty(1, dtype=torch.float32, device=x.device)
        as_block_sparsity(x, sp, workspace=self._ws[key], stream=stream)
        s = float(sp.item())
        code = as_prefill_mode(s)
        mode = _MODE_NAMES[code]
        if code == AS_MODE_DENSE:
            cfg_all = config(sel=AS_SEL_ALL, out_dtype=self.cfg.out_dtype)
            y = torch.empty(T, self.n_out, dtype=self.out_dtype(), device=x.device)
            as_linear_prefill(select_out(x_masked=x), self.W, T, cfg_all, y,
                              workspace=self._workspace(AS_OP_PREFILL, T), stream=stream)
            return y, mode, s
        bufs = self.select_buffers(T, x.device)
        self.select(x, bufs, stream=stream)
        if code == AS_MODE_24:
            return self.prefill_from(bufs, T, stream=stream), mode, s
        return self.prefill_hybrid_from(x, bufs, as_hybrid_dense_blocks(self.K, dense_frac), stream=stream), mode, s

    def prefill_rsparse(self, x: torch.Tensor, B: torch.Tensor, A: torch.Tensor, stream=None):
        """Selection + prefill with the R-Sparse compensation of the dropped
        channels (overview page, section 3.3): B [K, r], A [n_out, r] bf16
        factors of W, r in {64, 128}.  Returns (y, bufs)."""
        T = x.shape[0]
        bufs = self.select_buffers(T, x.device)
        self.select(x, bufs, stream=stream)
        key = ("rsparse", T, A.shape[1])
        if key not in self._ws:
            self._ws[key] = workspace(as_rsparse_prefill_workspace(T, self.K, A.shape[1]), x.device)
        y = torch.empty(T, self.n_out, dtype=self.out_dtype(), device=x.device)
        sel = select_out(**{k: v for k, v in bufs.items()
                            if k in ("bitmask", "x_masked", "x_compact", "meta24", "x_masked_lo", "x_compact_lo")})
        as_linear_prefill_rsparse(sel, x, self.W, self.cfg, y, B, A, rowsum=self.rowsum, eta=bufs.get("eta"),
                                  workspace=self._ws[key], stream=stream)
        return y, bufs

    def prefill_nm_split(self, x: torch.Tensor, n_dense: int, running_var=None, first_batch: bool = False,
                         dense_idx=None, sparsity=None, stream=None):
        """Selection with the 2:4 part of this layer's N:M configuration, then
        the hybrid split: the 2:4 part on the sparse tensor cores, the kept
        channels of the n_dense busiest blocks dense (2:4 + Squared-ReLU page,
        section 3.2).  Returns (y, bufs)."""
        T, K = x.shape
        dev = x.device
        bufs = self.select_buffers(T, dev)
        bufs["x_compact"] = torch.empty(T, K // 2, dtype=torch.bfloat16, device=dev)
        bufs["meta24"] = torch.empty(as_meta24_words(T, K), dtype=torch.int32, device=dev)
        bufs["bitmask24"] = torch.empty(T, (K + 31) // 32, dtype=torch.int32, device=dev)
        self.select(x, bufs, running_var=running_var, first_batch=first_batch, stream=stream)
        key = ("hybrid", T, n_dense)
        if key not in self._ws:
            self._ws[key] = workspace(as_hybrid_workspace(T, K, self.n_out, n_dense), dev)
        y = torch.empty(T, self.n_out, dtype=self.out_dtype(), device=dev)
        sel = select_out(**{k: v for k, v in bufs.items() if k in ("x_masked", "x_compact", "meta24", "bitmask24")})
        as_linear_prefill_nm_split(sel, T, self.W, self.cfg, y, n_dense, rowsum=self.rowsum, eta=bufs.get("eta"),
                                   nu=bufs.get("nu"), dense_idx=dense_idx, sparsity=sparsity,
                                   workspace=self._ws[key], stream=stream)
        return y, bufs

    def prefill(self, x: torch.Tensor, running_var=None, first_batch: bool = False, stream=None):
        bufs = self.select_buffers(x.shape[0], x.device)
        self.select(x, bufs, running_var=running_var, first_batch=first_batch, stream=stream)
        return self.prefill_from(bufs, x.shape[0], stream=stream), bufs


__all__ = ["SparseLinear", "workspace", "hybrid_mode", "dense_blocks_for", "AS_F32", "AS_BF16"]
