"""Seeded synthetic workloads for the activation-sparsified linear layer.

This module only draws random numbers and rounds them to the storage dtype.
It holds none of the method's arithmetic (no scores, no selection, no
compensation, no contraction), so that both the CUDA path and the CPU oracle
can be fed from it without sharing any computation.

Recipe (all workloads): numpy ``default_rng`` streams spawned from
``SeedSequence(seed)``; values are drawn in float64, cast to float32, and,
for bf16 workloads, rounded to bfloat16 round-to-nearest-even by torch on the
CPU.  Every array is returned as a CPU torch tensor in its storage dtype.

Workloads (LLM-shaped stand-ins for the model layers the pages measure on;
no model weights or datasets are used):

* ``tiny_layer``      x f32 [4, 256] ~ 0.5 * Student-t(4),
                      W f32 [512, 256] ~ N(0, 0.02^2), seed 0.
* ``decode_downproj`` Llama-7B down-projection: x bf16 [T, 11008] ~
                      Laplace(0, 0.3) with a fixed seeded 1% of channels
                      scaled by 20 (outlier channels), W bf16 [4096, 11008]
                      ~ N(0, 0.02^2), seed 1.
* ``decode_block``    Llama3.1-8B decoder block at one token: q/o [4096,4096],
                      k/v [1024,4096], gate/up [14336,4096], down [4096,14336];
                      x ~ Laplace(0, 0.3); per-layer keep fraction
                      ~ U[0.4, 0.7] and weight exponent from {0, 0.5, 1}, seed 2.
* ``prefill_sqrelu``  z bf16 [T, 14336] ~ N(-1.2, 1), x = bf16(fp32(max(0,z))^2),
                      W bf16 [4096, 14336] ~ N(0, 0.02^2), seed 3.
* ``prefill_clact``   x bf16 [8192, 8192] ~ 0.5 * Student-t(3) per batch
                      (8 batches), W bf16 [8192, 8192] ~ N(0, 0.02^2), seed 4.
* ``prefill_sqrelu_hot`` Squared-ReLU input with feature-dependent sparsity:
                      a seeded 5% of channels ("hot") have z ~ N(0, 1), the
                      rest z ~ N(-1.8, 1); x = bf16(fp32(max(0,z))^2), about
                      94% zeros overall; W bf16 ~ N(0, 0.02^2), seed 6.
* ``outlier_weight``  W [n_out, k], a two-component mixture: each weight is
                      N(-0.02, 0.01^2) or N(+0.02, 0.01^2) with probability
                      1/2 (a bimodal layer), and a seeded 0.2% of the entries
                      replaced by +-U[0.5, 1.0] (outliers), seed 5.  Default
                      shape: the v-projection [1024, 4096].
"""
from __future__ import annotations

import numpy as np
import torch

__all__ = [
    "streams", "to_dtype", "tiny_layer", "decode_downproj", "decode_block",
    "prefill_sqrelu", "prefill_clact_weight", "prefill_clact_batch",
    "random_layer", "BLOCK_LAYERS", "outlier_weight", "prefill_sqrelu_hot",
]


def streams(seed: int, n: int) -> list[np.random.Generator]:
    """``n`` independent generators spawned from ``SeedSequence(seed)``."""
    return [np.random.default_rng(s) for s in np.random.SeedSequence(seed).spawn(n)]


def to_dtype(a64: np.ndarray, dtype: torch.dtype) -> torch.Tensor:
    """float64 -> float32 -> ``dtype`` (round to nearest even), CPU tensor."""
    t = torch.from_numpy(np.ascontiguousarray(a64, dtype=np.float32))
    return t if dtype == torch.float32 else t.to(dtype)


def _normal(rng, shape, std, dtype):
    return to_dtype(rng.normal(0.0, std, size=shape), dtype)


def tiny_layer(seed: int = 0):
    """x f32 [4,256] ~ 0.5*t(4); W f32 [512,256] ~ N(0, 0.02^2)."""
    rx, rw = streams(seed, 2)
    x = to_dtype(0.5 * rx.standard_t(4.0, size=(4, 256)), torch.float32)
    w = to_dtype(rw.normal(0.0, 0.02, size=(512, 256)), torch.float32)
    return x, w


def decode_downproj(T: int = 16, seed: int = 1, k: int = 11008, n_out: int = 4096,
                    with_weight: bool = True):
    """Decode down-projection activations and weight.

    Returns ``(x, W, outlier_channels)``; ``x`` is the first ``T`` of 16 drawn
    tokens, so the T=1/8/16 cases are nested.  ``W`` is None when
    ``with_weight`` is False.
    """
    if not 1 <= T <= 16:
        raise ValueError("T must be in [1, 16]")
    rx, rw, ro = streams(seed, 3)
    n_outl = max(1, round(0.01 * k))
    outl = np.sort(ro.choice(k, size=n_outl, replace=False))
    x64 = rx.laplace(0.0, 0.3, size=(16, k))
    x64[:, outl] *= 20.0
    x = to_dtype(x64[:T], torch.bfloat16)
    w = _normal(rw, (n_out, k), 0.02, torch.bfloat16) if with_weight else None
    return x, w, torch.from_numpy(outl)


# name, n_out, k, which activation vector feeds it
BLOCK_LAYERS = [
    ("q", 4096, 4096, "attn_in"),
    ("k", 1024, 4096, "attn_in"),
    ("v", 1024, 4096, "attn_in"),
    ("o", 4096, 4096, "attn_out"),
    ("gate", 14336, 4096, "ffn_in"),
    ("up", 14336, 4096, "ffn_in"),
    ("down", 4096, 14336, "ffn_mid"),
]


def decode_block(seed: int = 2, with_weights: bool = True):
    """Seven linear layers of one decoder block at T=1.

    Returns a dict with ``layers``: list of dicts {name, n_out, k, W, x_key,
    keep_frac, alpha} and ``x``: dict of activation vectors [1, k] bf16.
    """
    rx, rw, rf, ra = streams(seed, 4)
    xs = {
        "attn_in": to_dtype(rx.laplace(0.0, 0.3, size=(1, 4096)), torch.bfloat16),
        "attn_out": to_dtype(rx.laplace(0.0, 0.3, size=(1, 4096)), torch.bfloat16),
        "ffn_in": to_dtype(rx.laplace(0.0, 0.3, size=(1, 4096)), torch.bfloat16),
        "ffn_mid": to_dtype(rx.laplace(0.0, 0.3, size=(1, 14336)), torch.bfloat16),
    }
    fr = rf.uniform(0.4, 0.7, size=len(BLOCK_LAYERS))
    al = ra.choice(np.array([0.0, 0.5, 1.0]), size=len(BLOCK_LAYERS))
    layers = []
    for i, (name, n_out, k, xk) in enumerate(BLOCK_LAYERS):
        w = _normal(rw, (n_out, k), 0.02, torch.bfloat16) if with_weights else None
        layers.append(dict(name=name, n_out=n_out, k=k, W=w, x_key=xk,
                           keep_frac=float(fr[i]), alpha=float(al[i])))
    return dict(layers=layers, x=xs)


def prefill_sqrelu(T: int = 4096, seed: int = 3, k: int = 14336, n_out: int = 4096,
                   with_weight: bool = True):
    """Squared-ReLU activations of an FFN down-projection at prefill.

    Returns ``(z, x, W)`` with z ~ N(-1.2, 1) in bf16, and x the squared ReLU
    of z computed in float32 and rounded to bf16 (the layer input), W bf16.
    """
    rz, rw = streams(seed, 2)
    z = to_dtype(rz.normal(-1.2, 1.0, size=(T, k)), torch.bfloat16)
    zf = z.float()
    x = (torch.clamp_min(zf, 0.0) * torch.clamp_min(zf, 0.0)).to(torch.bfloat16)
    w = _normal(rw, (n_out, k), 0.02, torch.bfloat16) if with_weight else None
    return z, x, w


def prefill_clact_weight(seed: int = 4, k: int = 8192, n_out: int = 8192):
    """W bf16 [n_out, k] ~ N(0, 0.02^2) for the CLACT + VAR prefill layer."""
    rw = streams(seed, 2)[0]
    return _normal(rw, (n_out, k), 0.02, torch.bfloat16)


def prefill_clact_batch(b: int, seed: int = 4, T: int = 8192, k: int = 8192):
    """Batch ``b`` (0..7) of x bf16 [T, k] ~ 0.5 * Student-t(3)."""
    rb = streams(seed, 2)[1]
    rng = np.random.default_rng(np.random.SeedSequence(int(rb.integers(1 << 62)) + b))
    return to_dtype(0.5 * rng.standard_t(3.0, size=(T, k)), torch.bfloat16)


def random_layer(T: int, k: int, n_out: int, seed: int, dtype=torch.bfloat16,
                 dist: str = "laplace", ties: int = 0):
    """Generic seeded case for parity tests at ragged sizes.

    ``dist``: "laplace" (scale 0.3), "t3" (0.5 * Student-t(3)) or "sqrelu".
    ``ties`` > 0 quantises x to multiples of 2^-ties so that equal scores occur.
    """
    rx, rw = streams(seed, 2)
    if dist == "laplace":
        x64 = rx.laplace(0.0, 0.3, size=(T, k))
    elif dist == "t3":
        x64 = 0.5 * rx.standard_t(3.0, size=(T, k))
    elif dist == "sqrelu":
        z = np.maximum(rx.normal(-1.2, 1.0, size=(T, k)), 0.0)
        x64 = z * z
    else:
        raise ValueError(dist)
    if ties:
        x64 = np.round(x64 * (1 << ties)) / (1 << ties)
    x = to_dtype(x64, dtype)
    w = to_dtype(rw.normal(0.0, 0.02, size=(n_out, k)), dtype)
    return x, w


def outlier_weight(seed: int = 5, n_out: int = 1024, k: int = 4096, dtype=torch.bfloat16,
                   outlier_frac: float = 0.002):
    """Bimodal weight with a few large outliers (see the module recipe)."""
    rm, rn, ro, rs, rv = streams(seed, 5)
    mode = np.where(rm.random(size=(n_out, k)) < 0.5, -0.02, 0.02)
    w = mode + rn.normal(0.0, 0.01, size=(n_out, k))
    n_o = int(round(outlier_frac * n_out * k))
    if n_o:
        idx = ro.choice(n_out * k, size=n_o, replace=False)
        sign = np.where(rs.random(size=n_o) < 0.5, -1.0, 1.0)
        w.reshape(-1)[idx] = sign * rv.uniform(0.5, 1.0, size=n_o)
    return to_dtype(w, dtype)


def prefill_sqrelu_hot(T: int = 4096, seed: int = 6, k: int = 14336, n_out: int = 4096, hot_frac: float = 0.05,
                       mu_cold: float = -1.8, mu_hot: float = 0.0, with_weight: bool = True):
    """Squared-ReLU activations whose sparsity differs by channel (see the
    module recipe).  Returns ``(z, x, W, hot_channels)``."""
    rz, rw, rh = streams(seed, 3)
    hot = np.sort(rh.choice(k, size=max(1, round(hot_frac * k)), replace=False))
    mu = np.full(k, mu_cold)
    mu[hot] = mu_hot
    z = to_dtype(rz.normal(0.0, 1.0, size=(T, k)) + mu[None, :], torch.bfloat16)
    zf = z.float()
    x = (torch.clamp_min(zf, 0.0) * torch.clamp_min(zf, 0.0)).to(torch.bfloat16)
    w = _normal(rw, (n_out, k), 0.02, torch.bfloat16) if with_weight else None
    return z, x, w, torch.from_numpy(hot)
