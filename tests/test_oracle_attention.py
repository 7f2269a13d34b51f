"""Pins of the fp64 oracle's attention, gradients and merge against independent facts.

Each test checks the oracle against something other than itself: a scalar
brute-force loop, a closed form, finite differences, or an identity of the
mathematics.  A plausible slip (a dropped mask term, a sign, a transposed
operand, a wrong kv-head map) fails at least one of them.
"""
import math

import numpy as np
import pytest

from oracle import attention as A
from synth import cu_from_lengths, normal_bf16, streams


def _inputs(seed, S, H, HKV, D):
    g = streams(seed, 4)
    return (normal_bf16(g[0], (S, H, D)).astype(np.float64),
            normal_bf16(g[1], (S, HKV, D)).astype(np.float64),
            normal_bf16(g[2], (S, HKV, D)).astype(np.float64),
            normal_bf16(g[3], (S, H, D)).astype(np.float64))


CASES = [
    # lengths, H, HKV, D, causal, window
    ([7, 13, 1, 9], 2, 2, 8, True, 0),
    ([16, 24], 2, 1, 16, True, 5),
    ([30], 4, 2, 8, False, 0),
    ([11, 5], 2, 2, 4, True, 1),
    ([20, 12], 2, 2, 8, False, 3),
]


@pytest.mark.parametrize("lengths,H,HKV,D,causal,window", CASES)
def test_fwd_matches_brute_force(lengths, H, HKV, D, causal, window):
    cu = cu_from_lengths(lengths)
    S = int(cu[-1])
    q, k, v, _ = _inputs(1, S, H, HKV, D)
    scale = 0.37
    out, lse = A.attention_fwd(q, k, v, cu, cu, scale, causal=causal, window=window)
    qpos, kpos = A.default_positions(cu, cu)
    doc = A.doc_ids(cu, S)
    bo, bl = A.brute_force_attention(q.tolist(), k.tolist(), v.tolist(), qpos, kpos, doc, doc, scale, causal, window)
    np.testing.assert_allclose(out, bo, rtol=0, atol=1e-12)
    fin = np.isfinite(bl)
    assert np.array_equal(fin, np.isfinite(lse))
    np.testing.assert_allclose(lse[fin], bl[fin], rtol=0, atol=1e-12)


def test_bottom_right_alignment_brute_force():
    # len_q != len_k inside each document: queries align to the last keys.
    cu_q = cu_from_lengths([3, 5])
    cu_k = cu_from_lengths([7, 6])
    g = streams(3, 3)
    q = normal_bf16(g[0], (8, 2, 8)).astype(np.float64)
    k = normal_bf16(g[1], (13, 2, 8)).astype(np.float64)
    v = normal_bf16(g[2], (13, 2, 8)).astype(np.float64)
    out, lse = A.attention_fwd(q, k, v, cu_q, cu_k, 0.5, causal=True)
    qpos = [4, 5, 6, 1, 2, 3, 4, 5]
    kpos = list(range(7)) + list(range(6))
    bo, bl = A.brute_force_attention(q.tolist(), k.tolist(), v.tolist(), qpos, kpos, [0] * 3 + [1] * 5,
                                     [0] * 7 + [1] * 6, 0.5, True, 0)
    np.testing.assert_allclose(out, bo, atol=1e-12)
    np.testing.assert_allclose(lse, bl, atol=1e-12)


@pytest.mark.parametrize("window", [0, 1, 4, 100])
def test_zero_query_closed_form(window):
    # q = 0 makes every visible score 0: lse = log|V(i)|, out = mean of visible v.
    lengths = [9, 17, 6]
    cu = cu_from_lengths(lengths)
    S = int(cu[-1])
    _, k, v, _ = _inputs(2, S, 2, 1, 8)
    q = np.zeros((S, 2, 8))
    out, lse = A.attention_fwd(q, k, v, cu, cu, 1.0, causal=True, window=window)
    for d in range(len(lengths)):
        a = int(cu[d])
        for i in range(lengths[d]):
            lo = 0 if window <= 0 else max(0, i - window + 1)
            n = i - lo + 1
            for h in range(2):
                assert lse[h, a + i] == pytest.approx(math.log(n), abs=1e-13)
                np.testing.assert_allclose(out[a + i, h], v[a + lo:a + i + 1, 0].mean(axis=0), atol=1e-13)


def test_constant_value_closed_form():
    cu = cu_from_lengths([10, 7])
    q, k, _, _ = _inputs(4, 17, 2, 2, 8)
    v = np.full((17, 2, 8), 2.5)
    out, _ = A.attention_fwd(q, k, v, cu, cu, 0.7, causal=True, window=3)
    np.testing.assert_allclose(out, 2.5, atol=1e-13)


def test_fully_masked_rows_are_zero_with_neg_inf_lse():
    # every key of the second document lies after every query: nothing is visible.
    cu_q = cu_from_lengths([4, 3])
    cu_k = cu_from_lengths([4, 3])
    q, k, v, _ = _inputs(5, 7, 1, 1, 4)
    out, lse = A.attention_fwd(q, k, v, cu_q, cu_k, 1.0, causal=True, qpos=np.array([0, 1, 2, 3, 0, 1, 2]),
                               kpos=np.array([0, 1, 2, 3, 10, 11, 12]))
    assert np.all(np.isneginf(lse[:, 4:]))
    assert np.all(out[4:] == 0)
    assert np.all(np.isfinite(lse[:, :4]))


def _loss(q, k, v, dout, cu, scale, causal, window):
    out, _ = A.attention_fwd(q, k, v, cu, cu, scale, causal=causal, window=window)
    return float((out * dout).sum())


@pytest.mark.parametrize("causal,window,HKV", [(True, 0, 2), (True, 3, 1), (False, 0, 2)])
def test_bwd_matches_finite_differences(causal, window, HKV):
    cu = cu_from_lengths([5, 6])
    q, k, v, dout = _inputs(6, 11, 2, HKV, 4)
    scale = 0.6
    out, lse = A.attention_fwd(q, k, v, cu, cu, scale, causal=causal, window=window)
    dq, dk, dv = A.attention_bwd(dout, q, k, v, out, lse, cu, cu, scale, causal=causal, window=window)
    eps = 1e-6
    rng = np.random.default_rng(0)
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for _ in range(12):
            idx = tuple(rng.integers(0, n) for n in x.shape)
            xp = x.copy(); xp[idx] += eps
            xm = x.copy(); xm[idx] -= eps
            args = {"q": q, "k": k, "v": v}
            args[name] = xp
            lp = _loss(args["q"], args["k"], args["v"], dout, cu, scale, causal, window)
            args[name] = xm
            lm = _loss(args["q"], args["k"], args["v"], dout, cu, scale, causal, window)
            fd = (lp - lm) / (2 * eps)
            assert g[idx] == pytest.approx(fd, abs=2e-7, rel=1e-6), (name, idx)


def test_gradient_sum_rules():
    # rows of P sum to 1 -> sum_j dv_j = sum_i dO_i ; softmax shift invariance -> sum_j dk_j = 0
    cu = cu_from_lengths([12, 20])
    q, k, v, dout = _inputs(7, 32, 2, 2, 8)
    out, lse = A.attention_fwd(q, k, v, cu, cu, 0.4, causal=True, window=6)
    dq, dk, dv = A.attention_bwd(dout, q, k, v, out, lse, cu, cu, 0.4, causal=True, window=6)
    for d in range(2):
        a, b = int(cu[d]), int(cu[d + 1])
        np.testing.assert_allclose(dv[a:b].sum(axis=0), dout[a:b].sum(axis=0), atol=1e-11)
        np.testing.assert_allclose(dk[a:b].sum(axis=0), 0.0, atol=1e-11)


def test_merge_sigmoid_form_equals_logaddexp():
    g = streams(8, 4)
    out = g[0].standard_normal((6, 3, 4))
    bout = g[1].standard_normal((6, 3, 4))
    lse = g[2].standard_normal((3, 6)) * 5
    blse = g[3].standard_normal((3, 6)) * 5
    lse[0, 0] = -np.inf
    blse[1, 2] = -np.inf
    lse[2, 3] = blse[2, 3] = -np.inf
    no, nl, w = A.update_out_and_lse(out, lse, bout, blse)
    ref_l = np.logaddexp(lse, blse)
    fin = np.isfinite(ref_l)
    np.testing.assert_allclose(nl[fin], ref_l[fin], atol=1e-13)
    assert np.isneginf(nl[2, 3])
    with np.errstate(invalid="ignore"):
        wa = np.where(fin, np.exp(lse - np.where(fin, ref_l, 0)), 0.0).T[:, :, None]
        wb = np.where(fin, np.exp(blse - np.where(fin, ref_l, 0)), 0.0).T[:, :, None]
    ref_o = np.where(fin.T[:, :, None], wa * out + wb * bout, out)
    np.testing.assert_allclose(no, ref_o, atol=1e-13)
    # the returned weight is sigmoid(block_lse - lse) of the pre-merge lse
    assert w[0, 0] == 1.0 and w[1, 2] == 0.0 and w[2, 3] == 0.0
    assert w[0, 1] == pytest.approx(1 / (1 + math.exp(lse[0, 1] - blse[0, 1])), abs=1e-15)


def test_merge_of_any_partition_in_any_order_equals_full():
    lengths = [20, 28]
    cu = cu_from_lengths(lengths)
    S = int(cu[-1])
    q, k, v, _ = _inputs(9, S, 2, 1, 8)
    full_o, full_l = A.attention_fwd(q, k, v, cu, cu, 0.5, causal=True, window=9)
    qpos, kpos = A.default_positions(cu, cu)
    doc = A.doc_ids(cu, S)
    rng = np.random.default_rng(1)
    labels = rng.integers(0, 4, size=S)  # a random partition of the keys into 4 blocks
    for order in ([0, 1, 2, 3], [3, 1, 0, 2], [2, 3, 1, 0]):
        o = np.zeros_like(full_o)
        l = np.full_like(full_l, -np.inf)
        for b in order:
            mask = A.visible(qpos, kpos, doc, doc, True, 9) & (labels[None, :] == b)
            bo, bl = A.attention_fwd_masked(q, k, v, mask, 0.5)
            o, l, _ = A.update_out_and_lse(o, l, bo, bl)
        np.testing.assert_allclose(o, full_o, atol=1e-12)
        np.testing.assert_allclose(l, full_l, atol=1e-12)
    # association: merge (0,1) and (2,3) separately, then together
    parts = []
    for pair in ((0, 1), (2, 3)):
        o = np.zeros_like(full_o)
        l = np.full_like(full_l, -np.inf)
        for b in pair:
            mask = A.visible(qpos, kpos, doc, doc, True, 9) & (labels[None, :] == b)
            bo, bl = A.attention_fwd_masked(q, k, v, mask, 0.5)
            o, l, _ = A.update_out_and_lse(o, l, bo, bl)
        parts.append((o, l))
    o, l, _ = A.update_out_and_lse(parts[0][0], parts[0][1], parts[1][0], parts[1][1])
    np.testing.assert_allclose(o, full_o, atol=1e-12)
    np.testing.assert_allclose(l, full_l, atol=1e-12)


def test_rows_subset_matches_full():
    cu = cu_from_lengths([40, 24])
    q, k, v, _ = _inputs(10, 64, 2, 2, 8)
    fo, fl = A.attention_fwd(q, k, v, cu, cu, 0.3, causal=True)
    rows = np.array([0, 5, 39, 40, 63])
    so, sl = A.attention_fwd(q, k, v, cu, cu, 0.3, causal=True, rows=rows)
    np.testing.assert_allclose(so[rows], fo[rows], atol=1e-14)
    np.testing.assert_allclose(sl[:, rows], fl[:, rows], atol=1e-14)


def test_row_and_column_gradient_subsets_match_the_full_backward():
    cu = cu_from_lengths([40, 56])
    q, k, v, do = _inputs(14, 96, 4, 2, 8)
    out, lse = A.attention_fwd(q, k, v, cu, cu, 0.3, causal=True, window=17)
    dq, dk, dv = A.attention_bwd(do, q, k, v, out, lse, cu, cu, 0.3, causal=True, window=17)
    rows, heads = [0, 5, 39, 40, 95], [0, 3]
    gq = A.attention_grad_rows(do, q, k, v, out, lse, cu, cu, 0.3, rows, heads, causal=True, window=17)
    np.testing.assert_allclose(gq, dq[np.ix_(rows, heads)], atol=1e-12)
    cols = [0, 20, 39, 40, 90]
    gk, gv = A.attention_grad_cols(do, q, k, v, out, lse, cu, cu, 0.3, cols, [0, 1, 2, 3], causal=True, window=17)
    # kv head h gathers q heads 2h and 2h+1
    for kh in range(2):
        np.testing.assert_allclose(gk[:, 2 * kh] + gk[:, 2 * kh + 1], dk[cols, kh], atol=1e-12)
        np.testing.assert_allclose(gv[:, 2 * kh] + gv[:, 2 * kh + 1], dv[cols, kh], atol=1e-12)
