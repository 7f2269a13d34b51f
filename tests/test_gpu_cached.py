"""EAGLE-3 cached ring (sequence block plus per-position cache diagonals) on the GPU against the
fp64 oracle: forward out/lse, backward dq and every cache block's gradients."""
import numpy as np
import pytest
import torch

import context_blockwise_causal_varlen_b200 as cbv
from oracle import cached as C
from synth import cu_from_lengths
from tests.gpu_util import check_lse, check_out, check_rel, dev, f64, gen, host, sync

pytestmark = pytest.mark.gpu

CASES = [
    # lengths, cp, H, HKV, D, window, num_blocks
    ([264, 520, 128], 2, 2, 2, 128, 0, 3),
    ([1000, 48], 4, 4, 1, 128, 0, 8),
    ([512], 4, 4, 2, 64, 0, 2),
    ([776, 136, 1024], 4, 2, 2, 128, 300, 4),
    ([40, 8, 360], 2, 2, 2, 64, 5, 5),
    ([256, 0, 128], 2, 8, 1, 64, 0, 7),
]


def _case(seed, lengths, H, HKV, D, nb, q_mul=1.0):
    cu = cu_from_lengths(lengths)
    S = int(cu[-1])
    q, ck, cv, do = gen(seed, (S, H, D), (nb, S, HKV, D), (nb, S, HKV, D), (S, H, D))
    return cu, q * np.float32(q_mul), ck, cv, do


@pytest.mark.parametrize("lengths,cp,H,HKV,D,window,nb", CASES)
@pytest.mark.parametrize("layout", ["zigzag", "contiguous"])
def test_cached_forward_matches_oracle(lengths, cp, H, HKV, D, window, nb, layout):
    cu, q, ck, cv, _ = _case(11, lengths, H, HKV, D, nb)
    out, lse = cbv.cached_ring_fwd(dev(q), dev(ck), dev(cv), cu, cp, scale=0.09, window=window, layout=layout)
    sync()
    ro, rl = C.cached_fwd(f64(q), f64(ck), f64(cv), cu, 0.09, window=window)
    check_out(host(out), ro)
    check_lse(host(lse), rl)


@pytest.mark.parametrize("lengths,cp,H,HKV,D,window,nb", CASES)
def test_cached_backward_matches_oracle(lengths, cp, H, HKV, D, window, nb):
    cu, q, ck, cv, do = _case(12, lengths, H, HKV, D, nb)
    scale = 0.09
    ro, rl = C.cached_fwd(f64(q), f64(ck), f64(cv), cu, scale, window=window)
    out_b = dev(ro.astype(np.float32))  # the backward is fed the merged out as the bf16 tensor the forward returns
    rq, rk, rv = C.cached_bwd(f64(do), f64(q), f64(ck), f64(cv), host(out_b), rl, cu, scale, window=window)
    lse_d = torch.from_numpy(rl.astype(np.float32)).cuda()
    dq, dck, dcv = cbv.cached_ring_bwd(dev(do), dev(q), dev(ck), dev(cv), out_b, lse_d, cu, cp, scale=scale,
                                       window=window)
    sync()
    check_rel(host(dq), rq, what="dq")
    dck, dcv = host(dck), host(dcv)
    for i in range(nb):  # each block on its own scale: the diagonals' gradients are much smaller than block 0's
        check_rel(dck[i], rk[i], what=f"dcache_k[{i}]")
        check_rel(dcv[i], rv[i], what=f"dcache_v[{i}]")


def test_dominant_diagonals():
    # large q: some rows are carried almost entirely by one diagonal key, others by the sequence.
    # Such rows copy one value vector, up to |4| here, and a bf16 output rounds it by up to
    # 2^-8 |out| on its own: the bound is 1e-2 plus that one rounding, element by element.
    cu, q, ck, cv, do = _case(13, [384, 640], 4, 2, 128, 4, q_mul=4.0)
    scale = 0.125
    out, lse = cbv.cached_ring_fwd(dev(q), dev(ck), dev(cv), cu, 2, scale=scale)
    sync()
    ro, rl = C.cached_fwd(f64(q), f64(ck), f64(cv), cu, scale)
    excess = np.abs(host(out) - ro) - (1e-2 + 2.0 ** -8 * np.abs(ro))
    assert excess.max() <= 0, f"out: worst element exceeds its bound by {excess.max():.3e}"
    check_lse(host(lse), rl)
    rq, rk, rv = C.cached_bwd(f64(do), f64(q), f64(ck), f64(cv), host(out), host(lse), cu, scale)
    dq, dck, dcv = cbv.cached_ring_bwd(dev(do), dev(q), dev(ck), dev(cv), out, lse, cu, 2, scale=scale)
    sync()
    check_rel(host(dq), rq, what="dq")
    for i in range(4):
        check_rel(host(dck)[i], rk[i], what=f"dcache_k[{i}]")
        check_rel(host(dcv)[i], rv[i], what=f"dcache_v[{i}]")


def test_one_block_is_the_plain_ring():
    cu, q, ck, cv, do = _case(14, [512, 256], 4, 2, 128, 1)
    out, lse = cbv.cached_ring_fwd(dev(q), dev(ck), dev(cv), cu, 2)
    ro, rl = cbv.zigzag_ring_fwd(dev(q), dev(ck[0]), dev(cv[0]), cu, 2)
    dq, dck, dcv = cbv.cached_ring_bwd(dev(do), dev(q), dev(ck), dev(cv), out, lse, cu, 2)
    rq, rk, rv = cbv.zigzag_ring_bwd(dev(do), dev(q), dev(ck[0]), dev(cv[0]), ro, rl, cu, 2)
    sync()
    assert torch.equal(out, ro) and torch.equal(lse, rl)
    assert torch.equal(dck[0], rk) and torch.equal(dcv[0], rv)
    # dq sums fp32 partials with reduce-adds whose order varies from run to run: equal up to one bf16 rounding
    check_rel(host(dq), host(rq), rel=8e-3, what="dq")


def test_window_of_one_sees_only_the_diagonals_and_itself():
    # window 1: every row's keys are its own sequence key and its own cache entries, no neighbour
    cu, q, ck, cv, _ = _case(15, [130, 70], 2, 2, 64, 3)
    out, lse = cbv.cached_ring_fwd(dev(q), dev(ck), dev(cv), cu, 1, scale=0.2, window=1)
    sync()
    ro, rl = C.cached_fwd(f64(q), f64(ck), f64(cv), cu, 0.2, window=1)
    check_out(host(out), ro)
    check_lse(host(lse), rl)


def test_separate_block_tensors_equal_the_stacked_cache():
    # the public form: the cache as a list of [S, Hkv, D] tensors at unrelated addresses
    cu, q, ck, cv, do = _case(16, [256, 128], 4, 2, 128, 3)
    tq, tdo = dev(q), dev(do)
    sk, sv = dev(ck), dev(cv)
    lk = [dev(ck[i]) for i in range(3)]
    lv = [dev(cv[i]) for i in range(3)]
    out_s, lse_s = cbv.cached_ring_fwd(tq, sk, sv, cu, 2)
    out_l, lse_l = cbv.cached_ring_fwd(tq, lk, lv, cu, 2)
    dq_s, dk_s, dv_s = cbv.cached_ring_bwd(tdo, tq, sk, sv, out_s, lse_s, cu, 2)
    dq_l, dk_l, dv_l = cbv.cached_ring_bwd(tdo, tq, lk, lv, out_l, lse_l, cu, 2)
    sync()
    assert torch.equal(out_s, out_l) and torch.equal(lse_s, lse_l)
    assert isinstance(dk_l, list) and len(dk_l) == 3 and dk_s.shape == (3, 384, 2, 128)
    for i in range(3):  # key-stationary block 0 and the closed-form diagonals are deterministic
        assert torch.equal(dk_s[i], dk_l[i]) and torch.equal(dv_s[i], dv_l[i])
    check_rel(host(dq_l), host(dq_s), rel=8e-3, what="dq")
