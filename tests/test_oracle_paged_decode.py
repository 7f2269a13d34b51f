"""Pins of the paged-prefill and decode oracles."""
import math

import numpy as np
import pytest

from oracle import attention as A
from oracle import decode as DEC
from oracle import paged as PG
from synth import block_permutation, cu_from_lengths, normal_bf16, streams


def _cache(seed, nblocks, hkv, bs, d):
    g = streams(seed, 3)
    return (normal_bf16(g[0], (nblocks, hkv, bs, d)).astype(np.float64),
            normal_bf16(g[1], (nblocks, hkv, bs, d)).astype(np.float64), g[2])


@pytest.mark.parametrize("mode", [PG.ROUND_ROBIN, PG.CONTIGUOUS])
def test_shard_positions_cover_context_once(mode):
    R, bs, nbl = 4, 8, 6
    pos = np.concatenate([PG.local_to_global_positions(r, nbl * bs, bs, R, mode) for r in range(R)])
    assert np.array_equal(np.sort(pos), np.arange(R * nbl * bs))
    if mode == PG.ROUND_ROBIN:
        # shard r holds global blocks r, r+R, r+2R, ...
        p1 = PG.local_to_global_positions(1, nbl * bs, bs, R, mode)
        assert np.array_equal(np.unique(p1 // bs), np.arange(1, R * nbl, R))


def test_global_kv_inverts_block_tables():
    R, bs, nbl, hkv, d = 4, 4, 3, 2, 8
    kc, vc, g = _cache(20, R * nbl, hkv, bs, d)
    perm = block_permutation(g, R * nbl)
    for mode in (PG.ROUND_ROBIN, PG.CONTIGUOUS):
        bt = PG.shard_block_tables(perm, R, mode)
        K, V = PG.global_kv(kc, vc, bt, bs, mode)
        for gb in range(R * nbl):  # logical block gb lives in physical page perm[gb]
            np.testing.assert_array_equal(K[gb * bs:(gb + 1) * bs], kc[perm[gb]].transpose(1, 0, 2))
            np.testing.assert_array_equal(V[gb * bs:(gb + 1) * bs], vc[perm[gb]].transpose(1, 0, 2))


@pytest.mark.parametrize("mode,window,seg", [(PG.ROUND_ROBIN, 0, 16), (PG.ROUND_ROBIN, 20, 8), (PG.CONTIGUOUS, 0, 24),
                                             (PG.CONTIGUOUS, 37, 96)])
def test_segmented_shards_equal_full_attention(mode, window, seg):
    R, bs, nbl, hq, hkv, d, S = 4, 8, 3, 4, 2, 8, 40
    kc, vc, g = _cache(21, R * nbl, hkv, bs, d)
    perm = block_permutation(g, R * nbl)
    bt = PG.shard_block_tables(perm, R, mode)
    q = normal_bf16(streams(22, 1)[0], (hq, S, d)).astype(np.float64)
    gqo = R * nbl * bs - S
    out, lse = PG.prefill_segmented(q, kc, vc, bt, bs, seg, 0.3, gqo, window=window, mode=mode)
    K, V = PG.global_kv(kc, vc, bt, bs, mode)
    fo, fl = PG.prefill_full(q, K, V, 0.3, gqo, window=window)
    np.testing.assert_allclose(out, fo, atol=1e-12)
    np.testing.assert_allclose(lse, fl, atol=1e-12)
    # the same as varlen causal attention with explicit positions
    qpos = gqo + np.arange(S)
    ao, al = A.attention_fwd(q.transpose(1, 0, 2), K, V, [0, S], [0, len(K)], 0.3, causal=True, window=window,
                             qpos=qpos, kpos=np.arange(len(K)))
    np.testing.assert_allclose(out, ao.transpose(1, 0, 2), atol=1e-12)
    np.testing.assert_allclose(lse, al, atol=1e-12)


def test_segment_size_does_not_change_the_result():
    R, bs, nbl, hq, hkv, d, S = 2, 8, 8, 2, 1, 8, 32
    kc, vc, g = _cache(23, R * nbl, hkv, bs, d)
    bt = PG.shard_block_tables(block_permutation(g, R * nbl), R, PG.ROUND_ROBIN)
    q = normal_bf16(streams(24, 1)[0], (hq, S, d)).astype(np.float64)
    a = PG.prefill_segmented(q, kc, vc, bt, bs, 8, 0.5, 100, window=50)
    b = PG.prefill_segmented(q, kc, vc, bt, bs, 64, 0.5, 100, window=50)
    np.testing.assert_allclose(a[0], b[0], atol=1e-12)
    np.testing.assert_allclose(a[1], b[1], atol=1e-12)


@pytest.mark.parametrize("mode", [PG.ROUND_ROBIN, PG.CONTIGUOUS])
def test_zero_query_closed_form_paged(mode):
    R, bs, nbl, hq, hkv, d, S, W = 4, 4, 4, 2, 1, 4, 20, 7
    kc, vc, g = _cache(25, R * nbl, hkv, bs, d)
    bt = PG.shard_block_tables(block_permutation(g, R * nbl), R, mode)
    gqo = 30
    out, lse = PG.prefill_segmented(np.zeros((hq, S, d)), kc, vc, bt, bs, 8, 1.0, gqo, window=W, mode=mode)
    K, V = PG.global_kv(kc, vc, bt, bs, mode)
    for i in range(S):
        p = gqo + i
        lo = max(0, p - W + 1)
        assert lse[0, i] == pytest.approx(math.log(p - lo + 1), abs=1e-13)
        np.testing.assert_allclose(out[1, i], V[lo:p + 1, 0].mean(axis=0), atol=1e-13)


def test_decode_closed_forms_and_full_attention():
    lengths = [1, 0, 5, 17, 3]
    cu_k = cu_from_lengths(lengths)
    n = len(lengths)
    g = streams(26, 3)
    hq, hkv, d = 4, 2, 8
    q = normal_bf16(g[0], (n, hq, d)).astype(np.float64)
    k = normal_bf16(g[1], (int(cu_k[-1]), hkv, d)).astype(np.float64)
    v = normal_bf16(g[2], (int(cu_k[-1]), hkv, d)).astype(np.float64)
    cu_q = np.arange(n + 1)
    out = DEC.varlen_decode(q, k, v, cu_q, cu_k, 0.3)
    # one key: out = v exactly; empty range: zeros
    np.testing.assert_allclose(out[0], np.repeat(v[0], 2, axis=0), atol=1e-15)
    assert np.all(out[1] == 0)
    # equals one-query varlen attention with no mask (kv head = h // (HQ/HKV))
    for s in range(n):
        if lengths[s] == 0:
            continue
        a, b = int(cu_k[s]), int(cu_k[s + 1])
        o, _ = A.attention_fwd(q[s:s + 1], k[a:b], v[a:b], [0, 1], [0, b - a], 0.3, causal=False)
        np.testing.assert_allclose(out[s], o[0], atol=1e-13)
    # q = 0: mean of the sequence's values
    out0 = DEC.varlen_decode(np.zeros_like(q), k, v, cu_q, cu_k, 0.3)
    np.testing.assert_allclose(out0[3, 3], v[6:23, 1].mean(axis=0), atol=1e-13)
