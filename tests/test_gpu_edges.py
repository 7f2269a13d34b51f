"""Edge cases on the GPU against the fp64 oracle: empty documents and inputs, the smallest
window, wide GQA groups, keyless rows, every paged block size, and the merge's identities."""
import numpy as np
import pytest
import torch

import context_blockwise_causal_varlen_b200 as cbv
from oracle import attention as A
from oracle import paged as PG
from synth import block_permutation, cu_from_lengths, streams
from tests.gpu_util import check_lse, check_out, check_rel, dev, f64, gen, host, sync

pytestmark = pytest.mark.gpu


def _ring_case(seed, lengths, H, HKV, D):
    cu = cu_from_lengths(lengths)
    S = int(cu[-1])
    q, k, v, do = gen(seed, (S, H, D), (S, HKV, D), (S, HKV, D), (S, H, D))
    return cu, q, k, v, do


@pytest.mark.parametrize("layout", ["zigzag", "contiguous"])
@pytest.mark.parametrize("schedule", [cbv.SCHEDULE_FUSED, cbv.SCHEDULE_STEPWISE])
def test_empty_and_tiny_documents_in_the_batch(layout, schedule):
    # documents of length 0 and of one token per chunk sit between ordinary ones
    lengths, cp = [0, 264, 0, 4, 520, 0], 2
    cu, q, k, v, do = _ring_case(40, lengths, 2, 2, 128)
    scale = 0.1
    out, lse = cbv.zigzag_ring_fwd(dev(q), dev(k), dev(v), cu, cp, scale=scale, layout=layout, schedule=schedule)
    dq, dk, dv = cbv.zigzag_ring_bwd(dev(do), dev(q), dev(k), dev(v), out, lse, cu, cp, scale=scale, layout=layout)
    sync()
    ro, rl = A.attention_fwd(f64(q), f64(k), f64(v), cu, cu, scale)
    check_out(host(out), ro)
    check_lse(host(lse), rl)
    rq, rk, rv = A.attention_bwd(f64(do), f64(q), f64(k), f64(v), host(out), rl, cu, cu, scale)
    check_rel(host(dq), rq, what="dq")
    check_rel(host(dk), rk, what="dk")
    check_rel(host(dv), rv, what="dv")


def test_empty_input_and_all_empty_documents():
    for lengths in ([], [0], [0, 0, 0]):
        cu = cu_from_lengths(lengths)
        e = torch.empty((0, 2, 128), dtype=torch.bfloat16, device="cuda")
        out, lse = cbv.zigzag_ring_fwd(e, e, e, cu, 2)
        dq, dk, dv = cbv.zigzag_ring_bwd(e, e, e, e, out, lse, cu, 2)
        sync()
        assert out.shape == (0, 2, 128) and lse.shape == (2, 0) and dq.shape == (0, 2, 128)


def test_window_of_one_sees_only_the_query_itself():
    cu, q, k, v, do = _ring_case(41, [256, 512], 2, 2, 64)
    out, lse = cbv.zigzag_ring_fwd(dev(q), dev(k), dev(v), cu, 2, scale=0.125, window=1)
    dq, dk, dv = cbv.zigzag_ring_bwd(dev(do), dev(q), dev(k), dev(v), out, lse, cu, 2, scale=0.125, window=1)
    sync()
    # one visible key: out = v_i, lse = s_ii, dv = dO, and dq = dk = 0 (dP - Delta vanishes up to
    # the rounding of two fp32 dot products)
    np.testing.assert_array_equal(host(out), f64(v))
    check_lse(host(lse), (0.125 * (f64(q) * f64(k)).sum(-1)).T)
    assert np.abs(host(dq)).max() <= 1e-3 and np.abs(host(dk)).max() <= 1e-3
    np.testing.assert_array_equal(host(dv), f64(do))


def test_wide_gqa_group_with_head_dim_64():
    cu, q, k, v, do = _ring_case(42, [512, 128, 264], 8, 1, 64)
    scale = 0.125
    out, lse = cbv.zigzag_ring_fwd(dev(q), dev(k), dev(v), cu, 2, scale=scale)
    dq, dk, dv = cbv.zigzag_ring_bwd(dev(do), dev(q), dev(k), dev(v), out, lse, cu, 2, scale=scale)
    sync()
    ro, rl = A.attention_fwd(f64(q), f64(k), f64(v), cu, cu, scale)
    check_out(host(out), ro)
    check_lse(host(lse), rl)
    rq, rk, rv = A.attention_bwd(f64(do), f64(q), f64(k), f64(v), host(out), rl, cu, cu, scale)
    check_rel(host(dq), rq, what="dq")
    check_rel(host(dk), rk, what="dk")
    check_rel(host(dv), rv, what="dv")


def test_block_forward_rows_without_keys():
    # document 0 has queries but no keys; document 1 has keys but no queries; document 2 is ordinary
    cu_q, cu_k = np.array([0, 70, 70, 200], np.int32), np.array([0, 0, 90, 330], np.int32)
    q, k, v = gen(43, (200, 2, 128), (330, 2, 128), (330, 2, 128))
    out, lse = cbv.attn_block_fwd(dev(q), dev(k), dev(v), cu_q, cu_k, scale=0.1, causal=True)
    sync()
    ro, rl = A.attention_fwd(f64(q), f64(k), f64(v), cu_q, cu_k, 0.1, causal=True)
    assert np.all(host(out)[:70] == 0) and np.all(np.isneginf(host(lse)[:, :70]))
    check_out(host(out), ro)
    check_lse(host(lse), rl)


@pytest.mark.parametrize("bs,D,mode", [(8, 128, PG.ROUND_ROBIN), (16, 64, PG.CONTIGUOUS), (64, 128, PG.ROUND_ROBIN),
                                       (128, 64, PG.ROUND_ROBIN), (128, 128, PG.CONTIGUOUS)])
def test_kvp_prefill_every_block_size(bs, D, mode):
    R, n_local, hq, hkv, S = 2, 256, 4, 2, 200
    bps = n_local // bs
    nb = R * bps
    q, kc, vc = gen(44, (hq, S, D), (nb, hkv, bs, D), (nb, hkv, bs, D))
    perm = block_permutation(streams(144, 1)[0], nb)
    bt = PG.shard_block_tables(perm, R, mode)
    gqo = R * n_local - S - 5
    K, V = PG.global_kv(f64(kc), f64(vc), bt, bs, mode)
    for window in (0, 77):
        ro, rl = PG.prefill_full(f64(q), K, V, 0.1, gqo, window=window)
        kv_mode = cbv.KV_ROUND_ROBIN if mode == PG.ROUND_ROBIN else cbv.KV_CONTIGUOUS
        out, lse = cbv.kvp_segmented_prefill(dev(q), dev(kc), dev(vc), torch.from_numpy(bt), kv_mode=kv_mode,
                                             seg_size=128, scale=0.1, global_q_offset=gqo, sliding_window=window)
        sync()
        check_out(host(out), ro, what=f"out bs={bs} W={window}")
        check_lse(host(lse), rl, what=f"lse bs={bs} W={window}")


def test_merge_identities_of_minus_infinity():
    S, H, D = 64, 2, 128
    (a,) = gen(45, (S, H, D))
    (b,) = gen(46, (S, H, D))
    out = torch.from_numpy(a).cuda()
    lse = torch.full((H, S), 0.5, device="cuda")
    # a block with lse = -inf leaves the running pair unchanged
    o2, l2 = cbv.attn_merge(out.clone(), lse.clone(), dev(b), torch.full((H, S), -float("inf"), device="cuda"))
    sync()
    assert torch.equal(o2, out) and torch.equal(l2, lse)
    # a running pair with lse = -inf takes the block
    blk = dev(b)
    o3, l3 = cbv.attn_merge(torch.zeros_like(out), torch.full((H, S), -float("inf"), device="cuda"), blk,
                            torch.full((H, S), 0.25, device="cuda"))
    sync()
    assert torch.equal(o3, blk.float()) and torch.all(l3 == 0.25)
    # both -inf: stays -inf, out unchanged
    o4, l4 = cbv.attn_merge(out.clone(), torch.full((H, S), -float("inf"), device="cuda"), blk,
                            torch.full((H, S), -float("inf"), device="cuda"))
    sync()
    assert torch.equal(o4, out) and torch.all(torch.isneginf(l4))


def test_ring_step_replays_from_a_cuda_graph():
    # every upload of a ring call travels inside kernel launch parameters, so a fixed-shape forward +
    # backward step can be captured once and replayed on new input values
    cu = cu_from_lengths([264, 520, 128])
    S, H, D = int(cu[-1]), 4, 128
    ins = [torch.empty((S, H, D), dtype=torch.bfloat16, device="cuda") for _ in range(4)]
    out = torch.empty((S, H, D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((H, S), dtype=torch.float32, device="cuda")
    dq, dk, dv = (torch.empty((S, H, D), dtype=torch.bfloat16, device="cuda") for _ in range(3))

    def step():
        q, k, v, do = ins
        cbv.zigzag_ring_fwd(q, k, v, cu, 2, out=out, lse=lse)
        cbv.zigzag_ring_bwd(do, q, k, v, out, lse, cu, 2, dq=dq, dk=dk, dv=dv)

    for t, x in zip(ins, gen(61, *[(S, H, D)] * 4)):
        t.copy_(dev(x))
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()  # warm-up outside the graph (kernel attributes, workspace sizes)
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for seed in (62, 63):
        vals = gen(seed, *[(S, H, D)] * 4)
        for t, x in zip(ins, vals):
            t.copy_(dev(x))
        g.replay()
        sync()
        q, k, v, do = (f64(x) for x in vals)
        ro, rl = A.attention_fwd(q, k, v, cu, cu, D ** -0.5, causal=True)
        check_out(host(out), ro)
        check_lse(host(lse), rl)
        rq, rk, rv = A.attention_bwd(do, q, k, v, host(out), host(lse), cu, cu, D ** -0.5, causal=True)
        check_rel(host(dq), rq, what="dq")
        check_rel(host(dk), rk, what="dk")
        check_rel(host(dv), rv, what="dv")


def test_wrong_output_tensors_are_refused_before_any_launch():
    cu = cu_from_lengths([64, 64])
    q, k, v, do = (dev(x) for x in gen(64, *[(128, 2, 64)] * 4))
    n0 = cbv.launch_count()
    for kw in ({"out": torch.empty((128, 2, 32), dtype=torch.bfloat16, device="cuda")},
               {"lse": torch.empty((128, 2), dtype=torch.float32, device="cuda")},
               {"out": torch.empty((128, 2, 64), dtype=torch.float32, device="cuda")}):
        with pytest.raises(cbv.CbvError):
            cbv.zigzag_ring_fwd(q, k, v, cu, 2, **kw)
    out, lse = cbv.zigzag_ring_fwd(q, k, v, cu, 2)
    n1 = cbv.launch_count()
    with pytest.raises(cbv.CbvError):
        cbv.zigzag_ring_bwd(do, q, k, v, out, lse, cu, 2, dk=torch.empty((128, 1, 64), dtype=torch.bfloat16, device="cuda"))
    with pytest.raises(cbv.CbvError):
        # the right shape, but not contiguous
        cbv.attn_block_bwd(do, q, k, v, out, lse, cu, cu, dq_acc=torch.zeros((2, 128, 64), device="cuda").transpose(0, 1))
    assert n1 - n0 == 2 and cbv.launch_count() == n1  # only the good forward launched anything


def test_many_tiny_documents_take_the_large_schedule_path():
    # 600 documents of 16 tokens: thousands of tiles, a schedule image far over one launch's 30 KB of
    # parameters, so it is uploaded in pieces and expanded by a second kernel
    cu = cu_from_lengths([16] * 600)
    S, H, D = int(cu[-1]), 2, 64
    q, k, v, do = gen(65, (S, H, D), (S, H, D), (S, H, D), (S, H, D))
    n0 = cbv.launch_count()
    out, lse = cbv.zigzag_ring_fwd(dev(q), dev(k), dev(v), cu, 2)
    n1 = cbv.launch_count()
    dq, dk, dv = cbv.zigzag_ring_bwd(dev(do), dev(q), dev(k), dev(v), out, lse, cu, 2)
    sync()
    assert n1 - n0 > 2  # the schedule took more than the one-launch path
    ro, rl = A.attention_fwd(f64(q), f64(k), f64(v), cu, cu, D ** -0.5, causal=True)
    check_out(host(out), ro)
    check_lse(host(lse), rl)
    rq, rk, rv = A.attention_bwd(f64(do), f64(q), f64(k), f64(v), host(out), host(lse), cu, cu, D ** -0.5, causal=True)
    check_rel(host(dq), rq, what="dq")
    check_rel(host(dk), rk, what="dk")
    check_rel(host(dv), rv, what="dv")
