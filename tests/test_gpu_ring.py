"""Ring forward / backward on the GPU against the fp64 oracle (small and tiny workloads)."""
import numpy as np
import pytest
import torch

import context_blockwise_causal_varlen_b200 as cbv
from oracle import attention as A
from oracle import planner as P
from oracle import ring as R
from synth import cu_from_lengths
from synth.workloads import tiny_zigzag
from tests.gpu_util import (GuardedWorkspaces, check_guards, check_lse, check_out, check_rel, dev, f64, gen, guarded,
                            host, sync)

pytestmark = pytest.mark.gpu


def _case(seed, lengths, H, HKV, D):
    cu = cu_from_lengths(lengths)
    S = int(cu[-1])
    q, k, v, do = gen(seed, (S, H, D), (S, HKV, D), (S, HKV, D), (S, H, D))
    return cu, q, k, v, do


@pytest.mark.parametrize("schedule", [cbv.SCHEDULE_FUSED, cbv.SCHEDULE_STEPWISE])
@pytest.mark.parametrize("layout", ["zigzag", "contiguous"])
def test_tiny_zigzag_forward(schedule, layout):
    w = tiny_zigzag()
    S = w.total
    q, k, v = gen(0, (S, w.heads, w.head_dim), (S, w.heads, w.head_dim), (S, w.heads, w.head_dim))
    (out, ob), (lse, lb) = guarded((S, w.heads, w.head_dim), torch.bfloat16), guarded((w.heads, S), torch.float32)
    wss = GuardedWorkspaces()
    cbv.zigzag_ring_fwd(dev(q), dev(k), dev(v), w.cu_seqlens, w.cp, scale=1 / 8, layout=layout, schedule=schedule,
                        out=out, lse=lse, workspace=wss)
    sync()
    check_guards(out, ob, what="out")
    check_guards(lse, lb, what="lse")
    wss.check()
    ro, rl = R.ring_fwd(f64(q), f64(k), f64(v), w.cu_seqlens, w.cp, 1 / 8,
                        layout=P.ZIGZAG if layout == "zigzag" else P.CONTIGUOUS)
    assert out.shape == (256, 2, 64) and lse.shape == (2, 256)
    check_out(host(out), ro)
    check_lse(host(lse), rl)


RING_CASES = [
    # lengths, cp, H, HKV, D, window
    ([264, 520, 128], 2, 2, 2, 128, 0),
    ([1000, 48], 4, 2, 1, 128, 0),
    ([512], 4, 4, 2, 64, 0),
    ([776, 136, 2048], 4, 2, 2, 128, 300),
    ([1536], 8, 2, 2, 128, 129),
    ([40, 8, 360], 2, 2, 2, 64, 5),
]


@pytest.mark.parametrize("lengths,cp,H,HKV,D,window", RING_CASES)
@pytest.mark.parametrize("layout", ["zigzag", "contiguous"])
def test_ring_forward_matches_oracle(lengths, cp, H, HKV, D, window, layout):
    cu, q, k, v, _ = _case(1, lengths, H, HKV, D)
    ro, rl = A.attention_fwd(f64(q), f64(k), f64(v), cu, cu, 0.09, causal=True, window=window)
    S, H = q.shape[0], q.shape[1]
    for schedule in (cbv.SCHEDULE_FUSED, cbv.SCHEDULE_STEPWISE):
        (out, ob), (lse, lb) = guarded(q.shape, torch.bfloat16), guarded((H, S), torch.float32)
        wss = GuardedWorkspaces()
        cbv.zigzag_ring_fwd(dev(q), dev(k), dev(v), cu, cp, scale=0.09, window=window, layout=layout,
                            schedule=schedule, out=out, lse=lse, workspace=wss)
        sync()
        check_guards(out, ob, what="out")
        check_guards(lse, lb, what="lse")
        wss.check()
        check_out(host(out), ro)
        check_lse(host(lse), rl)


@pytest.mark.parametrize("lengths,cp,H,HKV,D,window", RING_CASES)
def test_ring_backward_matches_oracle(lengths, cp, H, HKV, D, window):
    cu, q, k, v, do = _case(2, lengths, H, HKV, D)
    scale = 0.09
    ro, rl = A.attention_fwd(f64(q), f64(k), f64(v), cu, cu, scale, causal=True, window=window)
    # the block backward fed the merged out/lse: out as the bf16 tensor the forward returns
    out_b = dev(ro.astype(np.float32))
    ro_b = host(out_b)
    rq, rk, rv = A.attention_bwd(f64(do), f64(q), f64(k), f64(v), ro_b, rl, cu, cu, scale, causal=True, window=window)
    lse_d = torch.from_numpy(rl.astype(np.float32)).cuda()
    (dq, gq), (dk, gk), (dv, gv) = (guarded(x.shape, torch.bfloat16) for x in (q, k, v))
    wss = GuardedWorkspaces()
    for det in (False, True):
        for t in (dq, dk, dv):
            t.fill_(float("nan"))
        cbv.zigzag_ring_bwd(dev(do), dev(q), dev(k), dev(v), out_b, lse_d, cu, cp, scale=scale, window=window, dq=dq,
                            dk=dk, dv=dv, workspace=wss, deterministic=det)
        sync()
        for t, b, n in ((dq, gq, "dq"), (dk, gk, "dk"), (dv, gv, "dv")):
            check_guards(t, b, what=n)
        wss.check()
        check_rel(host(dq), rq, what="dq")
        check_rel(host(dk), rk, what="dk")
        check_rel(host(dv), rv, what="dv")


def test_forward_then_backward_chain():
    cu, q, k, v, do = _case(3, [1032, 520], 2, 2, 128)
    out, lse = cbv.zigzag_ring_fwd(dev(q), dev(k), dev(v), cu, 4)
    dq, dk, dv = cbv.zigzag_ring_bwd(dev(do), dev(q), dev(k), dev(v), out, lse, cu, 4)
    sync()
    scale = 128 ** -0.5
    ro, rl = A.attention_fwd(f64(q), f64(k), f64(v), cu, cu, scale)
    rq, rk, rv = A.attention_bwd(f64(do), f64(q), f64(k), f64(v), ro, rl, cu, cu, scale)
    check_rel(host(dq), rq, what="dq")
    check_rel(host(dk), rk, what="dk")
    check_rel(host(dv), rv, what="dv")
    # sum rules of the joint softmax hold on the GPU result too
    for d in range(2):
        a, b = int(cu[d]), int(cu[d + 1])
        np.testing.assert_allclose(host(dv)[a:b].sum(0), f64(do)[a:b].sum(0), atol=0.05 * np.abs(rv).max() * (b - a) ** 0.5)


def test_zigzag_and_contiguous_give_the_same_result():
    cu, q, k, v, _ = _case(4, [1024], 2, 2, 128)
    a = cbv.zigzag_ring_fwd(dev(q), dev(k), dev(v), cu, 4, layout="zigzag")
    b = cbv.zigzag_ring_fwd(dev(q), dev(k), dev(v), cu, 4, layout="contiguous")
    sync()
    assert torch.allclose(a[0].float(), b[0].float(), atol=1e-2)
    assert torch.allclose(a[1], b[1], atol=1e-3)


def test_status_word_is_clear_after_a_run():
    cu, q, k, v, _ = _case(5, [256], 2, 2, 128)
    _, _, ws = cbv.zigzag_ring_fwd(dev(q), dev(k), dev(v), cu, 2, return_workspace=True)
    assert cbv.read_status(ws) == 0


def test_each_call_launches_its_schedule_upload_and_kernels():
    # forward: the schedule (image and task expansion in one launch while the image fits 30 KB) + the
    # forward kernel; backward: the schedule + Delta + the backward kernel + the dq conversion
    cu, q, k, v, do = _case(3, [264, 520, 128], 2, 2, 128)
    tq, tk, tv, tdo = dev(q), dev(k), dev(v), dev(do)
    n0 = cbv.launch_count()
    out, lse = cbv.zigzag_ring_fwd(tq, tk, tv, cu, 2)
    n1 = cbv.launch_count()
    cbv.zigzag_ring_bwd(tdo, tq, tk, tv, out, lse, cu, 2)
    n2 = cbv.launch_count()
    sync()
    assert n1 - n0 == 2 and n2 - n1 == 4


def test_kernel_events_bracket_the_attention_kernels_only():
    # the measurement hook records the caller's events around the attention kernel of each call:
    # they lie inside events taken around the whole call, and clearing the hook stops the records
    cu, q, k, v, do = _case(7, [2048, 1024], 4, 4, 128)
    args = (dev(q), dev(k), dev(v), cu, 2)
    out, lse = cbv.zigzag_ring_fwd(*args)
    sync()
    call = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    kern = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    for fn in (lambda: cbv.zigzag_ring_fwd(*args),
               lambda: cbv.zigzag_ring_bwd(dev(do), dev(q), dev(k), dev(v), out, lse, cu, 2)):
        cbv.set_kernel_events(*kern)
        call[0].record()
        fn()
        call[1].record()
        cbv.set_kernel_events()
        sync()
        whole, inner = call[0].elapsed_time(call[1]), kern[0].elapsed_time(kern[1])
        assert 0 < inner <= whole
        assert call[0].elapsed_time(kern[0]) >= 0 and kern[1].elapsed_time(call[1]) >= 0
    # cleared: a further call records nothing, so the stop event stays before it
    mark = torch.cuda.Event(enable_timing=True)
    mark.record()
    cbv.zigzag_ring_fwd(*args)
    sync()
    assert kern[1].elapsed_time(mark) >= 0
