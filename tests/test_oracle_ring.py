"""Pins of the ring oracle and the planner: the blockwise ring equals full attention.

The zig-zag page states the invariants used here: merging the blocks of the
ring reproduces full causal attention, the backward fed the MERGED out/lse
reproduces the full gradients, the block-local-lse variant does not, and the
zig-zag layout gives every rank equal causal work while a contiguous shard
puts about twice the mean on the last rank.
"""
import os

import numpy as np
import pytest

from oracle import attention as A
from oracle import planner as P
from oracle import ring as R
from synth import cu_from_lengths, normal_bf16, streams

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "zigzag_cp2_S256.txt")


def _read_golden():
    d = {}
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, val = line.split(":", 1)
        d[key.strip()] = val.split()
    return d


def _ranges(tokens):
    out = []
    for t in tokens:
        a, b = t.strip("[)").split(",")
        out.append((int(a), int(b)))
    return out


def _expand(ranges):
    return np.concatenate([np.arange(a, b) for a, b in ranges])


def test_planner_worked_example():
    g = _read_golden()
    cu = np.array([int(x) for x in g["cu_seqlens_global"]])
    cp = int(g["cp"][0])
    assert list(np.diff(cu) // (2 * cp)) == [int(x) for x in g["chunk_sizes"]]
    assert P.local_cu_seqlens(cu, cp).tolist() == [int(x) for x in g["cu_seqlens_local"]]
    assert P.half_cu_seqlens(cu, cp).tolist() == [int(x) for x in g["cu_seqlens_half"]]
    cu_loc = P.local_cu_seqlens(cu, cp)
    assert np.array_equal(P.get_half_index(cu_loc, True), _expand(_ranges(g["front_index"])))
    assert np.array_equal(P.get_half_index(cu_loc, False), _expand(_ranges(g["back_index"])))
    assert np.array_equal(P.rank_tokens(cu, cp, 0), _expand(_ranges(g["rank0_tokens"])))
    assert np.array_equal(P.rank_tokens(cu, cp, 1), _expand(_ranges(g["rank1_tokens"])))
    assert P.rank_pair_counts(cu, cp, P.ZIGZAG).tolist() == [int(x) for x in g["rank_pairs_zigzag"]]
    assert P.rank_pair_counts(cu, cp, P.CONTIGUOUS).tolist() == [int(x) for x in g["rank_pairs_contiguous"]]


@pytest.mark.parametrize("lengths,cp", [([96, 160], 2), ([64], 4), ([24, 8, 40], 2), ([48, 96, 16], 4)])
def test_every_token_assigned_once_and_halves_tile(lengths, cp):
    cu = cu_from_lengths(lengths)
    S = int(cu[-1])
    for layout in (P.ZIGZAG, P.CONTIGUOUS):
        allt = np.concatenate([P.rank_tokens(cu, cp, r, layout) for r in range(cp)])
        assert np.array_equal(np.sort(allt), np.arange(S))
    cu_loc = P.local_cu_seqlens(cu, cp)
    f = P.get_half_index(cu_loc, True)
    b = P.get_half_index(cu_loc, False)
    assert np.array_equal(np.sort(np.concatenate([f, b])), np.arange(int(cu_loc[-1])))
    assert len(f) == len(b) == int(cu_loc[-1]) // 2
    # front positions map to each rank's early chunk, back positions to its late chunk
    for r in range(cp):
        tok = P.rank_tokens(cu, cp, r)
        c = np.diff(cu) // (2 * cp)
        doc = A.doc_ids(cu, S)
        chunk = (tok - cu[doc[tok]]) // c[doc[tok]]
        assert np.all(chunk[f] == r) and np.all(chunk[b] == 2 * cp - 1 - r)


@pytest.mark.parametrize("cp,c", [(2, 3), (4, 5), (8, 4096)])
def test_work_balance_closed_forms(cp, c):
    L = 2 * c * cp
    cu = np.array([0, L])
    zz = P.rank_pair_counts(cu, cp, P.ZIGZAG)
    ct = P.rank_pair_counts(cu, cp, P.CONTIGUOUS)
    assert np.all(zz == 2 * c * c * cp + c)
    assert ct.tolist() == [4 * c * c * r + c * (2 * c + 1) for r in range(cp)]
    assert zz.sum() == ct.sum() == L * (L + 1) // 2


def test_long_doc_imbalance_is_about_two():
    cu = np.array([0, 65536])
    zz = P.rank_pair_counts(cu, 8, P.ZIGZAG)
    ct = P.rank_pair_counts(cu, 8, P.CONTIGUOUS)
    assert np.all(zz == 268439552)
    assert ct[0] == 33558528 and ct[-1] == 503320576
    assert ct[-1] / ct.mean() == pytest.approx(1.875, abs=1e-3)


def _inputs(seed, S, H, D):
    g = streams(seed, 4)
    return tuple(normal_bf16(g[i], (S, H, D)).astype(np.float64) for i in range(4))


@pytest.mark.parametrize("lengths,cp,window,layout", [
    ([96, 160], 2, 0, P.ZIGZAG),
    ([32, 48, 16], 4, 0, P.ZIGZAG),
    ([64, 32], 2, 7, P.ZIGZAG),
    ([64], 4, 13, P.ZIGZAG),
    ([48, 24], 4, 0, P.CONTIGUOUS),
    ([64], 2, 9, P.CONTIGUOUS),
])
def test_ring_forward_equals_full_attention(lengths, cp, window, layout):
    cu = cu_from_lengths(lengths)
    S = int(cu[-1])
    q, k, v, _ = _inputs(11, S, 2, 8)
    out, lse = R.ring_fwd(q, k, v, cu, cp, 0.35, window=window, layout=layout)
    fo, fl = A.attention_fwd(q, k, v, cu, cu, 0.35, causal=True, window=window)
    np.testing.assert_allclose(out, fo, atol=1e-12)
    np.testing.assert_allclose(lse, fl, atol=1e-12)


@pytest.mark.parametrize("lengths,cp,window,layout", [
    ([48, 80], 2, 0, P.ZIGZAG),
    ([32, 16], 4, 5, P.ZIGZAG),
    ([48, 24], 4, 0, P.CONTIGUOUS),
])
def test_ring_backward_with_merged_lse_equals_full_gradients(lengths, cp, window, layout):
    cu = cu_from_lengths(lengths)
    S = int(cu[-1])
    q, k, v, dout = _inputs(12, S, 2, 8)
    out, lse = R.ring_fwd(q, k, v, cu, cp, 0.35, window=window, layout=layout)
    dq, dk, dv = R.ring_bwd(dout, q, k, v, out, lse, cu, cp, 0.35, window=window, layout=layout)
    fq, fk, fv = A.attention_bwd(dout, q, k, v, out, lse, cu, cu, 0.35, causal=True, window=window)
    np.testing.assert_allclose(dq, fq, atol=1e-11)
    np.testing.assert_allclose(dk, fk, atol=1e-11)
    np.testing.assert_allclose(dv, fv, atol=1e-11)


def test_block_local_lse_variant_is_wrong():
    # Feeding each block its own softmax statistics (the variant that drops the
    # lse path) must NOT reproduce the joint-softmax gradients.
    cu = cu_from_lengths([48, 80])
    q, k, v, dout = _inputs(13, 128, 2, 8)
    out, lse = R.ring_fwd(q, k, v, cu, 2, 0.35)
    fq, fk, fv = A.attention_bwd(dout, q, k, v, out, lse, cu, cu, 0.35, causal=True)
    bq, bk, bv = R.ring_bwd(dout, q, k, v, out, lse, cu, 2, 0.35, lse_mode="block_local")
    assert np.abs(bq - fq).max() > 1e-2 * np.abs(fq).max()
    assert np.abs(bk - fk).max() > 1e-2 * np.abs(fk).max()
    # and the sum rules of the joint softmax break too
    assert np.abs(bk[:48].sum(axis=0)).max() > 1e-6 or np.abs(bv[:48].sum(axis=0) - dout[:48].sum(axis=0)).max() > 1e-6


def test_zigzag_step_schedule_covers_each_visible_pair_once():
    cu = cu_from_lengths([32, 16])
    cp = 4
    S = 48
    cnt = np.zeros((S, S), np.int64)
    q = np.zeros((S, 1, 1)); k = np.zeros((S, 1, 1)); v = np.zeros((S, 1, 1))
    _, _, blocks = R.ring_fwd(q, k, v, cu, cp, 1.0, return_blocks=True)
    qpos, kpos = A.default_positions(cu, cu)
    doc = A.doc_ids(cu, S)
    for r, s, rows, kv, causal in blocks:
        m = A.visible(rows, kv, doc[rows], doc[kv], causal, 0)
        if not causal:
            same_doc = doc[rows][:, None] == doc[kv][None, :]
            assert np.array_equal(m, same_doc), "non-causal blocks must be fully visible within each document"
        cnt[np.ix_(rows, kv)] += m
    full = A.visible(np.arange(S), np.arange(S), doc, doc, True, 0)
    assert np.array_equal(cnt, full.astype(np.int64))
