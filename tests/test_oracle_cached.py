"""Pins of the EAGLE-3 cached-attention oracle against what the pages and the mathematics fix."""
import numpy as np
import pytest

from oracle import attention as A
from oracle import cached as C
from oracle import planner as P
from synth import cu_from_lengths, normal_bf16, streams


def _case(seed, lengths, H, HKV, D, nb):
    cu = cu_from_lengths(lengths)
    T = int(cu[-1])
    g = streams(seed, 4)
    q = normal_bf16(g[0], (T, H, D)).astype(np.float64)
    ck = normal_bf16(g[1], (nb, T, HKV, D)).astype(np.float64)
    cv = normal_bf16(g[2], (nb, T, HKV, D)).astype(np.float64)
    do = normal_bf16(g[3], (T, H, D)).astype(np.float64)
    return cu, q, ck, cv, do


def test_one_block_is_plain_causal_attention():
    cu, q, ck, cv, do = _case(1, [24, 40], 2, 1, 8, 1)
    out, lse = C.cached_fwd(q, ck, cv, cu, 0.3)
    ro, rl = A.attention_fwd(q, ck[0], cv[0], cu, cu, 0.3)
    np.testing.assert_allclose(out, ro, atol=1e-12)
    np.testing.assert_allclose(lse, rl, atol=1e-12)
    g = C.cached_bwd(do, q, ck, cv, out, lse, cu, 0.3)
    rq, rk, rv = A.attention_bwd(do, q, ck[0], cv[0], ro, rl, cu, cu, 0.3)
    np.testing.assert_allclose(g[0], rq, atol=1e-12)
    np.testing.assert_allclose(g[1][0], rk, atol=1e-12)
    np.testing.assert_allclose(g[2][0], rv, atol=1e-12)


@pytest.mark.parametrize("window", [0, 5])
def test_zero_queries_give_uniform_weights(window):
    # every visible score is 0: lse = log(#visible sequence keys + NB - 1), out = their mean value
    cu, _, ck, cv, _ = _case(2, [12, 20], 2, 2, 4, 3)
    T = int(cu[-1])
    q = np.zeros((T, 2, 4))
    out, lse = C.cached_fwd(q, ck, cv, cu, 0.5, window=window)
    for d in range(2):
        for t in range(int(cu[d]), int(cu[d + 1])):
            lo = int(cu[d]) if window == 0 else max(int(cu[d]), t - window + 1)
            n = t - lo + 1
            for h in range(2):
                assert lse[h, t] == pytest.approx(np.log(n + 2), abs=1e-12)
                mean = (cv[0, lo:t + 1, h].sum(0) + cv[1, t, h] + cv[2, t, h]) / (n + 2)
                np.testing.assert_allclose(out[t, h], mean, atol=1e-12)


def test_brute_force_on_a_tiny_case():
    cu, q, ck, cv, _ = _case(3, [7, 5], 2, 1, 3, 3)
    out, lse = C.cached_fwd(q, ck, cv, cu, 0.7, window=4)
    for d in range(2):
        for t in range(int(cu[d]), int(cu[d + 1])):
            for h in range(2):
                keys, vals = [], []
                for j in range(int(cu[d]), t + 1):
                    if t - j < 4:
                        keys.append(ck[0, j, 0]); vals.append(cv[0, j, 0])
                for i in (1, 2):
                    keys.append(ck[i, t, 0]); vals.append(cv[i, t, 0])
                s = np.array([0.7 * float(np.dot(q[t, h], kk)) for kk in keys])
                w = np.exp(s - s.max())
                assert lse[h, t] == pytest.approx(s.max() + np.log(w.sum()), abs=1e-12)
                np.testing.assert_allclose(out[t, h], (w[:, None] * np.array(vals)).sum(0) / w.sum(), atol=1e-12)


@pytest.mark.parametrize("layout", [P.ZIGZAG, P.CONTIGUOUS])
def test_ring_then_diagonal_merges_in_any_order_equal_the_joint_softmax(layout):
    cu, q, ck, cv, _ = _case(4, [32, 48], 2, 1, 8, 4)
    out, lse = C.cached_fwd(q, ck, cv, cu, 0.25)
    for order in ([1, 2, 3], [3, 1, 2]):
        bo, bl = C.cached_fwd_blockwise(q, ck, cv, cu, 2, 0.25, layout=layout, order=order)
        np.testing.assert_allclose(bo, out, atol=1e-12)
        np.testing.assert_allclose(bl, lse, atol=1e-12)


def test_gradients_match_finite_differences():
    cu, q, ck, cv, do = _case(5, [6, 4], 2, 1, 3, 3)
    scale, eps = 0.6, 1e-6

    def loss(q_, ck_, cv_):
        o, _ = C.cached_fwd(q_, ck_, cv_, cu, scale)
        return float((o * do).sum())

    out, lse = C.cached_fwd(q, ck, cv, cu, scale)
    dq, dk, dv = C.cached_bwd(do, q, ck, cv, out, lse, cu, scale)
    rng = np.random.default_rng(0)
    for name, x, g in (("q", q, dq), ("k", ck, dk), ("v", cv, dv)):
        for _ in range(12):
            idx = tuple(int(rng.integers(0, s)) for s in x.shape)
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = [q, ck, cv]
            args_m = [q, ck, cv]
            k = {"q": 0, "k": 1, "v": 2}[name]
            args_p[k], args_m[k] = xp, xm
            fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            assert g[idx] == pytest.approx(fd, abs=1e-6), (name, idx)


def test_value_gradients_sum_to_the_output_gradient():
    # every row's weights sum to one, so the value gradients of all keys add up to sum_t dO_t
    cu, q, ck, cv, do = _case(6, [16, 24], 4, 2, 8, 3)
    out, lse = C.cached_fwd(q, ck, cv, cu, 0.35)
    _, _, dv = C.cached_bwd(do, q, ck, cv, out, lse, cu, 0.35)
    for kh in range(2):
        np.testing.assert_allclose(dv[:, :, kh].sum(axis=(0, 1)), do[:, 2 * kh:2 * kh + 2].sum(axis=(0, 1)), atol=1e-10)
