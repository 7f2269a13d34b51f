"""KV-parallel segmented prefill over a paged KV cache, in float64.

Test infrastructure only (see the package docstring).

NKI library, ``attention_kv_parallel_segmented_cte`` (Background and API
Reference): every shard ("rank") holds part of a paged KV cache
``[num_blocks, num_kv_heads, block_size, D]`` addressed through its own block
table; it walks its local KV in segments of ``seg_size`` tokens with online
softmax, and the shards' partial results are merged by online softmax.  Q token
``i`` sits at global position ``global_q_offset + i``.  In the contiguous
distribution shard ``r`` holds global tokens ``[r*local_kv_len, (r+1)*local_kv_len)``;
in the round-robin (interleaved) one it holds global blocks ``r, r+R, r+2R, ...``.
``sliding_window = W > 0`` keeps keys with ``0 <= qpos - kpos < W``.

Layouts here: q ``[HQ, S, D]`` (the page's ``[BS, S, D]`` with BS = q heads),
out ``[HQ, S, D]``, lse ``[HQ, S]``; ``block_tables`` is ``[R, blocks_per_shard]``.
"""
from __future__ import annotations

import numpy as np

from .attention import NEG_INF, attention_fwd_masked, update_out_and_lse

CONTIGUOUS = "contiguous"
ROUND_ROBIN = "round_robin"


def shard_block_tables(perm, shards: int, mode: str) -> np.ndarray:
    """Per-shard block tables from a logical-block -> physical-page permutation."""
    perm = np.asarray(perm, np.int64)
    nb = len(perm)
    if nb % shards:
        raise ValueError("number of logical blocks must divide evenly over the shards")
    if mode == ROUND_ROBIN:
        return np.stack([perm[r::shards] for r in range(shards)]).astype(np.int32)
    per = nb // shards
    return np.stack([perm[r * per:(r + 1) * per] for r in range(shards)]).astype(np.int32)


def local_to_global_positions(r: int, n_local: int, block_size: int, shards: int, mode: str) -> np.ndarray:
    """Global token position of shard ``r``'s local tokens ``0..n_local-1``."""
    t = np.arange(n_local, dtype=np.int64)
    if mode == ROUND_ROBIN:
        return ((t // block_size) * shards + r) * block_size + t % block_size
    return r * n_local + t


def gather_shard_kv(cache, table, block_size: int) -> np.ndarray:
    """Shard-local KV sequence ``[n_local, HKV, D]`` read through a block table."""
    cache = np.asarray(cache)
    pages = cache[np.asarray(table, np.int64)]  # [nb, HKV, bs, D]
    nb, hkv, bs, d = pages.shape
    return pages.transpose(0, 2, 1, 3).reshape(nb * bs, hkv, d)


def global_kv(k_cache, v_cache, block_tables, block_size: int, mode: str):
    """The whole context ``(K, V)`` ``[kv_len, HKV, D]`` in global position order."""
    R, nbl = np.asarray(block_tables).shape
    n_local = nbl * block_size
    kv_len = R * n_local
    d = np.asarray(k_cache).shape[-1]
    hkv = np.asarray(k_cache).shape[1]
    K = np.zeros((kv_len, hkv, d), np.float64)
    V = np.zeros((kv_len, hkv, d), np.float64)
    for r in range(R):
        pos = local_to_global_positions(r, n_local, block_size, R, mode)
        K[pos] = gather_shard_kv(k_cache, block_tables[r], block_size)
        V[pos] = gather_shard_kv(v_cache, block_tables[r], block_size)
    return K, V


def _mask(qpos, kpos, window):
    qp = np.asarray(qpos, np.int64)[:, None]
    kp = np.asarray(kpos, np.int64)[None, :]
    m = kp <= qp
    if window > 0:
        m = m & (qp - kp < window)
    return m


def prefill_full(q, K, V, scale, global_q_offset, window=0, rows=None):
    """Causal (+ window) attention of q ``[HQ,S,D]`` over the whole context; ``(out [HQ,S,D], lse [HQ,S])``."""
    q = np.asarray(q, np.float64)
    hq, S, d = q.shape
    sel = np.arange(S) if rows is None else np.asarray(rows, np.int64)
    qpos = global_q_offset + sel
    mask = _mask(qpos, np.arange(K.shape[0]), window)
    o, l = attention_fwd_masked(q[:, sel].transpose(1, 0, 2), K, V, mask, scale)
    out = np.zeros((hq, S, V.shape[2]))
    lse = np.full((hq, S), NEG_INF)
    out[:, sel] = o.transpose(1, 0, 2)
    lse[:, sel] = l
    return out, lse


def prefill_segmented(q, k_cache, v_cache, block_tables, block_size, seg_size, scale, global_q_offset,
                      window=0, mode=ROUND_ROBIN, return_shards=False):
    """The page's decomposition: per shard, per segment, online-softmax merge; then merge the shards."""
    q = np.asarray(q, np.float64)
    hq, S, d = q.shape
    qpos = global_q_offset + np.arange(S)
    R, nbl = np.asarray(block_tables).shape
    n_local = nbl * block_size
    shard_parts = []
    for r in range(R):
        kloc = gather_shard_kv(k_cache, block_tables[r], block_size)
        vloc = gather_shard_kv(v_cache, block_tables[r], block_size)
        kpos_all = local_to_global_positions(r, n_local, block_size, R, mode)
        o_r = np.zeros((S, hq, d))
        l_r = np.full((hq, S), NEG_INF)
        for s0 in range(0, n_local, seg_size):
            seg = np.arange(s0, min(s0 + seg_size, n_local))
            mask = _mask(qpos, kpos_all[seg], window)
            bo, bl = attention_fwd_masked(q.transpose(1, 0, 2), kloc[seg], vloc[seg], mask, scale)
            o_r, l_r, _ = update_out_and_lse(o_r, l_r, bo, bl)
        shard_parts.append((o_r, l_r))
    out = np.zeros((S, hq, d))
    lse = np.full((hq, S), NEG_INF)
    for o_r, l_r in shard_parts:
        out, lse, _ = update_out_and_lse(out, lse, o_r, l_r)
    res = (out.transpose(1, 0, 2), lse)
    if return_shards:
        return res, [(o.transpose(1, 0, 2), l) for o, l in shard_parts]
    return res
