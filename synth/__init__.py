"""Seeded synthetic inputs shared by the oracle side and the CUDA side.

This module draws random numbers and rounds them to the storage type. It holds
none of the attention arithmetic: no masks, no softmax, no merge, no planner.
Every generator takes an explicit seed so a test, the bench and the oracle see
the same values.

Recipe (one place, so every caller agrees):
  * streams: ``numpy.random.SeedSequence(seed).spawn(n)`` in a fixed order
    (q, k, v, dout, lengths, perm, ...), each feeding a PCG64 generator;
  * values: ``standard_normal`` in float32, then round-to-nearest-even to
    bfloat16; the oracle reads those bf16 values widened to float64;
  * document lengths, decode key counts and page permutations are integer
    draws from their own stream.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "streams",
    "bf16_round",
    "bf16_bits",
    "normal_bf16",
    "packed_doc_lengths",
    "decode_key_counts",
    "block_permutation",
    "cu_from_lengths",
    "to_torch_bf16",
]


def streams(seed: int, n: int) -> list[np.random.Generator]:
    """``n`` independent generators spawned from one base seed, in a fixed order."""
    return [np.random.Generator(np.random.PCG64(s)) for s in np.random.SeedSequence(seed).spawn(n)]


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); return the 16-bit patterns."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16) & 0xFFFF
    return r.astype(np.uint16)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """float32 values rounded to the nearest bfloat16 (ties to even), returned as float32."""
    b = bf16_bits(x).astype(np.uint32) << 16
    return b.view(np.float32)


def normal_bf16(rng: np.random.Generator, shape) -> np.ndarray:
    """Standard normal draws in float32, rounded to bfloat16, returned as float32."""
    return bf16_round(rng.standard_normal(size=shape, dtype=np.float32))


def cu_from_lengths(lengths) -> np.ndarray:
    """Prefix sums ``[0, L0, L0+L1, ...]`` as int32."""
    cu = np.zeros(len(lengths) + 1, dtype=np.int64)
    cu[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64))
    return cu.astype(np.int32)


def packed_doc_lengths(rng: np.random.Generator, total: int, lo: int, hi: int, multiple: int) -> np.ndarray:
    """Packed-document lengths summing to ``total``.

    Each length is drawn uniform on the integers ``[lo, hi]`` and floored to a
    multiple of ``multiple``; draws continue until the running sum reaches
    ``total``, and the last document is trimmed to fill exactly (dropped if the
    trim leaves nothing).  ``total`` must itself be a multiple of ``multiple``.
    """
    if total % multiple:
        raise ValueError("total must be a multiple of `multiple`")
    out = []
    acc = 0
    while acc < total:
        L = int(rng.integers(lo, hi + 1)) // multiple * multiple
        if acc + L >= total:
            L = total - acc
        if L > 0:
            out.append(L)
        acc += L
    return np.asarray(out, dtype=np.int64)


def decode_key_counts(rng: np.random.Generator, n: int, lo: int, hi: int) -> np.ndarray:
    """Per-sequence gathered key counts, uniform on the integers ``[lo, hi]``."""
    return rng.integers(lo, hi + 1, size=n).astype(np.int64)


def block_permutation(rng: np.random.Generator, nblocks: int) -> np.ndarray:
    """A seeded permutation of physical page ids ``0..nblocks-1`` (int32)."""
    return rng.permutation(nblocks).astype(np.int32)


def to_torch_bf16(x: np.ndarray, device="cpu"):
    """A torch bfloat16 tensor holding exactly the bf16 values of ``x``."""
    import torch

    bits = bf16_bits(np.asarray(x, dtype=np.float32))
    t = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16)
    return t.to(device)


def torch_normal_bf16(shape, seed: int, device="cuda"):
    """Standard normal float32 draws from torch's generator on ``device``, rounded to bfloat16.

    For full-size workloads that are too large to draw on the host; tests that
    check such inputs copy the rows they need back to the host.
    """
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    flat = out.view(-1)
    step = 1 << 28
    for i in range(0, flat.numel(), step):
        n = min(step, flat.numel() - i)
        flat[i:i + n] = torch.randn(n, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
    return out
