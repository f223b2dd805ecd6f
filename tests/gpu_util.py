"""Test-side helpers for the GPU parity tests (no method arithmetic here:
decoding the documented 2:4 metadata layout, error norms, bit unpacking)."""
import numpy as np
import torch


def rel_l2(y, ref) -> float:
    y = np.asarray(y, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.linalg.norm(y - ref) / max(np.linalg.norm(ref), 1e-300))


def unpack_bitmask(words: torch.Tensor, K: int) -> np.ndarray:
    """[T, ceil(K/32)] int32 words -> [T, K] uint8 (bit i%32 of word i/32)."""
    w = words.cpu().numpy().view(np.uint32)
    T = w.shape[0]
    bits = ((w[:, :, None] >> np.arange(32, dtype=np.uint32)[None, None, :]) & 1).astype(np.uint8)
    return bits.reshape(T, -1)[:, :K]


def decode_meta24(meta: torch.Tensor, T: int, K: int):
    """Metadata words in the layout documented in include/actsparse.h ->
    ([T, K/4, 2] kept positions i0, i1 per 4-block)."""
    m = meta.cpu().numpy().view(np.uint32)
    kt = (K + 127) // 128
    out = np.zeros((T, K // 4, 2), np.int64)
    t = np.arange(T)[:, None]
    c = (np.arange(K // 4) * 4)[None, :]
    p = t % 128
    tile = (t // 128) * kt + c // 128
    j = (c % 128) // 32
    q = c % 32
    lane = 16 * (p // 16) + 8 * (q // 16) + p % 8
    word = m[tile * 512 + lane * 4 + j]
    shift = 16 * ((p % 16) // 8) + 4 * ((q % 16) // 4)
    nib = (word >> shift.astype(np.uint32)) & 0xF
    out[:, :, 0] = nib & 3
    out[:, :, 1] = nib >> 2
    return out


def f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def decode_meta8(meta: torch.Tensor, T: int, K: int, T_pad: int | None = None):
    """FP8 2:4 position words (layout documented in include/actsparse.h) ->
    [T_pad or T, ceil(K/256)*64, 2] positions i0, i1 per 4-block, padding
    blocks included."""
    m = meta.cpu().numpy().view(np.uint32)
    kt = (K + 255) // 256
    rows = T if T_pad is None else T_pad
    t = np.arange(rows)[:, None]
    c = (np.arange(kt * 64) * 4)[None, :]
    p = t % 128
    tile = (t // 128) * kt + c // 256
    q = c % 256
    j = q // 32
    word = m[tile * 1024 + (j // 4) * 512 + p * 4 + (j % 4)]
    shift = (4 * ((q % 32) // 4)).astype(np.uint32)
    nib = (word >> shift) & 0xF
    return np.stack([nib & 3, nib >> 2], axis=-1).astype(np.int64)
