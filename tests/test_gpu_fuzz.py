"""Seeded random shapes against the fp64 oracle: ring forward and backward over random document
mixes, cp, layouts, GQA ratios, head dims and windows, the cached ring, and the deterministic flag.
The shapes are drawn so that chunk tails of every raggedness occur (single-tile forward tasks, key
tiles that share two ranges, empty documents)."""
import numpy as np
import pytest
import torch

import context_blockwise_causal_varlen_b200 as cbv
from oracle import attention as A
from oracle import cached as C
from synth import cu_from_lengths
from tests.gpu_util import check_lse, check_out, check_rel, dev, f64, gen, host, sync

pytestmark = pytest.mark.gpu


def _draw(seed):
    rng = np.random.default_rng(1000 + seed)
    cp = int(rng.choice([1, 2, 3, 4]))
    unit = 2 * cp
    ndocs = int(rng.integers(1, 5))
    lengths = [int(rng.integers(0, 1600 // unit // ndocs + 1)) * unit for _ in range(ndocs)]
    if sum(lengths) == 0:
        lengths[0] = unit * 17
    H, HKV = [(2, 1), (4, 2), (4, 4), (8, 2)][int(rng.integers(0, 4))]
    D = int(rng.choice([64, 128]))
    window = int(rng.choice([0, 0, 1 + int(rng.integers(0, 700))]))
    layout = "zigzag" if rng.random() < 0.7 else "contiguous"
    if layout == "contiguous":
        lengths = [L // unit * unit for L in lengths]
    return cp, lengths, H, HKV, D, window, layout, bool(rng.random() < 0.3)


@pytest.mark.parametrize("seed", range(12))
def test_random_ring_matches_oracle(seed):
    cp, lengths, H, HKV, D, window, layout, det = _draw(seed)
    cu = cu_from_lengths(lengths)
    S = int(cu[-1])
    scale = 0.11
    q, k, v, do = gen(50 + seed, (S, H, D), (S, HKV, D), (S, HKV, D), (S, H, D))
    out, lse = cbv.zigzag_ring_fwd(dev(q), dev(k), dev(v), cu, cp, scale=scale, window=window, layout=layout)
    sync()
    ro, rl = A.attention_fwd(f64(q), f64(k), f64(v), cu, cu, scale, causal=True, window=window)
    check_out(host(out), ro)
    check_lse(host(lse), rl)
    dq, dk, dv = cbv.zigzag_ring_bwd(dev(do), dev(q), dev(k), dev(v), out, lse, cu, cp, scale=scale, window=window,
                                     layout=layout, deterministic=det)
    sync()
    rq, rk, rv = A.attention_bwd(f64(do), f64(q), f64(k), f64(v), host(out), host(lse), cu, cu, scale, causal=True,
                                 window=window)
    check_rel(host(dq), rq, what="dq")
    check_rel(host(dk), rk, what="dk")
    check_rel(host(dv), rv, what="dv")


@pytest.mark.parametrize("seed", range(4))
def test_random_cached_ring_matches_oracle(seed):
    cp, lengths, H, HKV, D, window, layout, det = _draw(100 + seed)
    nb = 2 + seed
    cu = cu_from_lengths(lengths)
    S = int(cu[-1])
    q, ck, cv, do = gen(80 + seed, (S, H, D), (nb, S, HKV, D), (nb, S, HKV, D), (S, H, D))
    out, lse = cbv.cached_ring_fwd(dev(q), dev(ck), dev(cv), cu, cp, scale=0.1, window=window, layout=layout)
    sync()
    ro, rl = C.cached_fwd(f64(q), f64(ck), f64(cv), cu, 0.1, window=window)
    check_out(host(out), ro)
    check_lse(host(lse), rl)
    dq, dck, dcv = cbv.cached_ring_bwd(dev(do), dev(q), dev(ck), dev(cv), out, lse, cu, cp, scale=0.1, window=window,
                                       layout=layout, deterministic=det)
    sync()
    rq, rk, rv = C.cached_bwd(f64(do), f64(q), f64(ck), f64(cv), host(out), host(lse), cu, 0.1, window=window)
    check_rel(host(dq), rq, what="dq")
    for i in range(nb):
        check_rel(host(dck[i]), rk[i], what=f"dcache_k[{i}]")
        check_rel(host(dcv[i]), rv[i], what=f"dcache_v[{i}]")
