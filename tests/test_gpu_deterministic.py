"""Deterministic backward: dq summed in 64-bit fixed point is bit-identical from run to run and
matches the oracle like the fp32 path does."""
import numpy as np
import pytest
import torch

import context_blockwise_causal_varlen_b200 as cbv
from oracle import attention as A
from oracle import cached as C
from synth import cu_from_lengths
from tests.gpu_util import check_rel, dev, f64, gen, host, sync

pytestmark = pytest.mark.gpu


def _inputs(seed, lengths, H, HKV, D):
    cu = cu_from_lengths(lengths)
    S = int(cu[-1])
    q, k, v, do = gen(seed, (S, H, D), (S, HKV, D), (S, HKV, D), (S, H, D))
    return cu, q, k, v, do


@pytest.mark.parametrize("lengths,cp,H,HKV,D,window", [
    ([3072, 1024], 2, 4, 2, 128, 0),   # rows see up to 24 key tiles
    ([2048, 520, 8], 4, 2, 1, 64, 700),
])
def test_ring_backward_is_bit_reproducible_and_matches_oracle(lengths, cp, H, HKV, D, window):
    cu, q, k, v, do = _inputs(21, lengths, H, HKV, D)
    scale = 0.08
    tq, tk, tv, tdo = dev(q), dev(k), dev(v), dev(do)
    out, lse = cbv.zigzag_ring_fwd(tq, tk, tv, cu, cp, scale=scale, window=window)
    runs = [cbv.zigzag_ring_bwd(tdo, tq, tk, tv, out, lse, cu, cp, scale=scale, window=window, deterministic=True)
            for _ in range(3)]
    fast = cbv.zigzag_ring_bwd(tdo, tq, tk, tv, out, lse, cu, cp, scale=scale, window=window)
    sync()
    for other in runs[1:]:
        for a, b in zip(runs[0], other):
            assert torch.equal(a, b)
    rq, rk, rv = A.attention_bwd(f64(do), f64(q), f64(k), f64(v), host(out), host(lse), cu, cu, scale, causal=True,
                                 window=window)
    dq, dk, dv = runs[0]
    check_rel(host(dq), rq, what="dq")
    check_rel(host(dk), rk, what="dk")
    check_rel(host(dv), rv, what="dv")
    # dk / dv are written once per key tile in both modes; dq differs by summation rounding only
    assert torch.equal(dk, fast[1]) and torch.equal(dv, fast[2])
    check_rel(host(dq), host(fast[0]), rel=8e-3, what="dq fixed vs fp32")


def test_block_backward_deterministic_adds_into_the_accumulator():
    cu, q, k, v, do = _inputs(22, [1536, 512], 4, 4, 128)
    scale = 0.09
    tq, tk, tv, tdo = dev(q), dev(k), dev(v), dev(do)
    ro, rl = A.attention_fwd(f64(q), f64(k), f64(v), cu, cu, scale, causal=True)
    out = dev(ro.astype(np.float32))
    lse = torch.from_numpy(rl.astype(np.float32)).cuda()
    base = torch.randn((int(cu[-1]), 4, 128), device="cuda", generator=torch.Generator("cuda").manual_seed(3))
    results = []
    for _ in range(2):
        dq_acc = base.clone()
        dk_acc = torch.zeros((int(cu[-1]), 4, 128), device="cuda")
        dv_acc = torch.zeros_like(dk_acc)
        cbv.attn_block_bwd(tdo, tq, tk, tv, out, lse, cu, cu, scale=scale, dq_acc=dq_acc, dk_acc=dk_acc,
                           dv_acc=dv_acc, deterministic=True)
        results.append(dq_acc)
    sync()
    assert torch.equal(results[0], results[1])
    rq, _, _ = A.attention_bwd(f64(do), f64(q), f64(k), f64(v), host(out), rl, cu, cu, scale, causal=True)
    check_rel(host(results[0]) - host(base), rq, what="dq added")


def test_cached_backward_is_bit_reproducible():
    cu = cu_from_lengths([2048, 512])
    S = int(cu[-1])
    q, ck, cv, do = gen(23, (S, 4, 128), (4, S, 2, 128), (4, S, 2, 128), (S, 4, 128))
    tq, tdo, tck, tcv = dev(q), dev(do), dev(ck), dev(cv)
    out, lse = cbv.cached_ring_fwd(tq, tck, tcv, cu, 2)
    a = cbv.cached_ring_bwd(tdo, tq, tck, tcv, out, lse, cu, 2, deterministic=True)
    b = cbv.cached_ring_bwd(tdo, tq, tck, tcv, out, lse, cu, 2, deterministic=True)
    sync()
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    rq, rk, rv = C.cached_bwd(f64(do), f64(q), f64(ck), f64(cv), host(out), host(lse), cu, 128 ** -0.5)
    check_rel(host(a[0]), rq, what="dq")
    for i in range(4):
        check_rel(host(a[1])[i], rk[i], what=f"dcache_k[{i}]")
        check_rel(host(a[2])[i], rv[i], what=f"dcache_v[{i}]")
