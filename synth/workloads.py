"""The synthetic workloads, by name and size, and their seeded integer structure.

Only shapes, sizes and the integer structure drawn from the seed live here
(document lengths, page permutations, decode key counts); the float tensors are
drawn by the callers through :mod:`synth`.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from . import cu_from_lengths, decode_key_counts, packed_doc_lengths, block_permutation, streams


@dataclass
class RingWorkload:
    name: str
    cu_seqlens: np.ndarray  # int32 [docs+1], global, natural packed order
    cp: int
    heads: int
    head_dim: int
    window: int = 0

    @property
    def total(self) -> int:
        return int(self.cu_seqlens[-1])


@dataclass
class PagedWorkload:
    name: str
    q_len: int
    hq: int
    hkv: int
    head_dim: int
    kv_len: int
    block_size: int
    shards: int
    seg_size: int
    global_q_offset: int
    window: int
    perm: np.ndarray = field(repr=False)  # int32 [kv_len // block_size], logical block -> physical page


@dataclass
class DecodeWorkload:
    name: str
    num_seqs: int
    hq: int
    hkv: int
    head_dim: int
    key_counts: np.ndarray = field(repr=False)

    @property
    def cu_seqlens_k(self) -> np.ndarray:
        return cu_from_lengths(self.key_counts)


def tiny_zigzag() -> RingWorkload:
    """One packed batch of 256 tokens in two documents (96 + 160), cp=2, H=2, D=64."""
    return RingWorkload("tiny_zigzag_S256_cp2_H2_D64", np.array([0, 96, 256], np.int32), 2, 2, 64)


def packed_zigzag(seed: int = 0, total: int = 16384, cp: int = 4, heads: int = 32, head_dim: int = 128) -> RingWorkload:
    """Packed documents, lengths uniform in [512, 4096] floored to multiples of 2*cp, last trimmed."""
    rng = streams(seed, 6)[4]
    lengths = packed_doc_lengths(rng, total, 512, 4096, 2 * cp)
    return RingWorkload(f"packed_zigzag_S{total}_cp{cp}_H{heads}_D{head_dim}", cu_from_lengths(lengths), cp, heads, head_dim)


def long_doc(total: int = 65536, cp: int = 8, heads: int = 16, head_dim: int = 128, window: int = 0) -> RingWorkload:
    """One document of ``total`` tokens, cp virtual ranks, optional sliding window."""
    w = f"_W{window}" if window > 0 else ""
    return RingWorkload(f"long_doc_S{total}_cp{cp}_H{heads}_D{head_dim}{w}", np.array([0, total], np.int32), cp, heads, head_dim, window)


def paged_prefill(seed: int = 0, window: int = 0, q_len: int = 4096, kv_len: int = 32768, hq: int = 32, hkv: int = 8,
                  head_dim: int = 128, block_size: int = 32, shards: int = 8, seg_size: int = 512,
                  global_q_offset: int | None = None) -> PagedWorkload:
    """Paged KV-parallel prefill: Q is the last ``q_len`` tokens of a ``kv_len`` context."""
    rng = streams(seed, 6)[5]
    perm = block_permutation(rng, kv_len // block_size)
    if global_q_offset is None:
        global_q_offset = kv_len - q_len
    w = f"_W{window}" if window > 0 else ""
    return PagedWorkload(f"paged_prefill_S{q_len}_KV{kv_len}_HQ{hq}_HKV{hkv}_D{head_dim}{w}", q_len, hq, hkv, head_dim,
                         kv_len, block_size, shards, seg_size, global_q_offset, window, perm)


def varlen_decode(seed: int = 0, num_seqs: int = 8192, lo: int = 1, hi: int = 2048, hq: int = 32, hkv: int = 4,
                  head_dim: int = 128) -> DecodeWorkload:
    """One query per sequence; per-sequence key counts uniform on [lo, hi]."""
    rng = streams(seed, 6)[4]
    counts = decode_key_counts(rng, num_seqs, lo, hi)
    return DecodeWorkload(f"varlen_decode_N{num_seqs}_HQ{hq}_HKV{hkv}_D{head_dim}", num_seqs, hq, hkv, head_dim, counts)
