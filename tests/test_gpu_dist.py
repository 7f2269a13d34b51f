"""The ring over real ranks and Ulysses on the GPU, against the fp64 oracle.

(1) The per-step block calls (cbv_ring_step_fwd / _bwd) on local buffers, with the
ranks simulated in one process: every rank's k/v visits every other rank in ring
order, the running (out, lse) is merged on the GPU, and the backward adds into the
owner's dK/dV directly (the accumulators' travel is the driver's and is covered by the
multi-process tests).  (2) The package's drivers (ring, Ulysses, KV-parallel prefill)
with two processes that share this GPU, over gloo with the tensors staged through host
memory: no kernel of one process waits on the other.  (3) The Ulysses building blocks: the axis swap and the diagonal
merge / gradients on their own.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import context_blockwise_causal_varlen_b200 as cbv
from oracle import attention as A
from oracle import cached as C
from oracle import planner as P
from synth import cu_from_lengths
from tests.gpu_util import check_guards, check_lse, check_out, check_rel, dev, f64, gen, guarded, host, sync

pytestmark = pytest.mark.gpu

STEP_CASES = [
    # lengths, cp, H, HKV, D, window, layout
    ([264, 520, 128], 2, 2, 2, 128, 0, "zigzag"),
    ([1000, 48], 4, 4, 2, 128, 0, "zigzag"),
    ([776, 136, 2048], 4, 2, 2, 128, 300, "zigzag"),
    ([40, 8, 360], 2, 2, 1, 64, 5, "zigzag"),
    ([1000, 48], 4, 2, 2, 128, 0, "contiguous"),
]


@pytest.mark.parametrize("lengths,cp,H,HKV,D,window,layout", STEP_CASES)
def test_ring_steps_on_local_buffers_equal_full_attention(lengths, cp, H, HKV, D, window, layout):
    cu = cu_from_lengths(lengths)
    S = int(cu[-1])
    q, k, v, do = gen(81, (S, H, D), (S, HKV, D), (S, HKV, D), (S, H, D))
    scale = 0.09
    name = P.ZIGZAG if layout == "zigzag" else P.CONTIGUOUS
    loc = [cbv.rank_tokens(cu, cp, r, layout) for r in range(cp)]
    L = lambda x, r: dev(np.ascontiguousarray(x[loc[r]]))
    Q, K, V, DO = ([L(x, r) for r in range(cp)] for x in (q, k, v, do))
    n = S // cp
    outs, lses = [], []
    for r in range(cp):
        (oa, ob), (la, lb) = guarded((n, H, D), torch.float32), guarded((H, n), torch.float32)
        (o16, o16b) = guarded((n, H, D), torch.bfloat16)
        for s in range(cp):
            src = (r - s) % cp
            cbv.ring_step_fwd(r, s, Q[r], K[src], V[src], cu, cp, oa, la, out=o16 if s == cp - 1 else None,
                              scale=scale, window=window, layout=layout)
        sync()
        for t, b, what in ((oa, ob, "out_acc"), (la, lb, "lse_acc"), (o16, o16b, "out")):
            check_guards(t, b, what=what)
        outs.append(o16)
        lses.append(la)
    out, lse = np.zeros((S, H, D)), np.zeros((H, S))
    for r in range(cp):
        out[loc[r]], lse[:, loc[r]] = host(outs[r]), host(lses[r])
    ro, rl = A.attention_fwd(f64(q), f64(k), f64(v), cu, cu, scale, causal=True, window=window)
    check_out(out, ro)
    check_lse(lse, rl)
    # backward fed the merged out / lse of every rank's rows
    dq = [torch.zeros((n, H, D), dtype=torch.float32, device="cuda") for _ in range(cp)]
    dk = [torch.zeros((n, HKV, D), dtype=torch.float32, device="cuda") for _ in range(cp)]
    dvv = [torch.zeros((n, HKV, D), dtype=torch.float32, device="cuda") for _ in range(cp)]
    for r in range(cp):
        for s in range(cp):
            src = (r - s) % cp
            cbv.ring_step_bwd(r, s, DO[r], Q[r], K[src], V[src], outs[r], lses[r], cu, cp, dq[r], dk[src], dvv[src],
                              scale=scale, window=window, layout=layout)
    sync()
    gq, gk, gv = np.zeros((S, H, D)), np.zeros((S, HKV, D)), np.zeros((S, HKV, D))
    for r in range(cp):
        gq[loc[r]], gk[loc[r]], gv[loc[r]] = host(dq[r]), host(dk[r]), host(dvv[r])
    rq, rk, rv = A.attention_bwd(f64(do), f64(q), f64(k), f64(v), out, rl, cu, cu, scale, causal=True, window=window)
    check_rel(gq, rq, what="dq")
    check_rel(gk, rk, what="dk")
    check_rel(gv, rv, what="dv")
    assert name in (P.ZIGZAG, P.CONTIGUOUS)


def test_ring_step_argument_errors():
    cu = cu_from_lengths([96, 160])
    q, k, v = (dev(x) for x in gen(82, (128, 2, 64), (128, 2, 64), (128, 2, 64)))
    oa = torch.empty((128, 2, 64), dtype=torch.float32, device="cuda")
    la = torch.empty((2, 128), dtype=torch.float32, device="cuda")
    n0 = cbv.launch_count()
    for rank, step, status in ((2, 0, "BAD_ARG"), (0, 2, "BAD_ARG"), (-1, 0, "BAD_ARG")):
        with pytest.raises(cbv.CbvError) as e:
            cbv.ring_step_fwd(rank, step, q, k, v, cu, 2, oa, la)
        assert e.value.status == status
    with pytest.raises(cbv.CbvError) as e:
        cbv.ring_step_fwd(0, 0, q, k, v, cu_from_lengths([96, 100]), 2, oa, la)
    assert e.value.status in ("BAD_CU_SEQLENS", "NOT_DIVISIBLE_2CP")
    assert cbv.launch_count() == n0


# ----------------------------------------------------------------------------- two processes, one GPU
def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _kvp_case():
    from oracle import paged as PG
    from synth import block_permutation, streams

    R, bps, bs, hq, hkv, D, S = 4, 4, 32, 4, 2, 128, 160
    q, kc, vc = gen(85, (hq, S, D), (R * bps, hkv, bs, D), (R * bps, hkv, bs, D))
    perm = block_permutation(streams(185, 1)[0], R * bps)
    return q, kc, vc, PG.shard_block_tables(perm, R, PG.ROUND_ROBIN), R * bps * bs - S - 5


def _dist_worker(rank, world, port, res):
    from context_blockwise_causal_varlen_b200 import dist as cdist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        # ring: zig-zag, cp = world, GQA 2:1, D = 128
        cu = cu_from_lengths([264, 520, 128])
        S, H, HKV, D = int(cu[-1]), 4, 2, 128
        q, k, v, do = gen(83, (S, H, D), (S, HKV, D), (S, HKV, D), (S, H, D))
        loc = cbv.rank_tokens(cu, world, rank, "zigzag")
        L = lambda x: dev(np.ascontiguousarray(x[loc]))
        out, lse = cdist.zigzag_ring_fwd(L(q), L(k), L(v), cu, scale=0.1, via_host=True)
        dq, dk, dv = cdist.zigzag_ring_bwd(L(do), L(q), L(k), L(v), out, lse, cu, scale=0.1, via_host=True)
        ring = tuple(host(x) for x in (out, lse, dq, dk, dv))
        # Ulysses with two cache diagonals: contiguous sequence slices, heads split over the ranks
        cu2 = cu_from_lengths([100, 156])
        S2, NB = int(cu2[-1]), 3
        q2, ck, cv, do2 = gen(84, (S2, H, D), (NB, S2, HKV, D), (NB, S2, HKV, D), (S2, H, D))
        n = S2 // world
        sl = slice(rank * n, (rank + 1) * n)
        lck = [dev(np.ascontiguousarray(ck[i, sl])) for i in range(NB)]
        lcv = [dev(np.ascontiguousarray(cv[i, sl])) for i in range(NB)]
        o2, l2 = cdist.ulysses_fwd(dev(q2[sl]), lck, lcv, cu2, scale=0.1, via_host=True)
        g = cdist.ulysses_bwd(dev(do2[sl]), dev(q2[sl]), lck, lcv, o2, l2, cu2, scale=0.1, via_host=True)
        torch.cuda.synchronize()
        uly = (host(o2), host(l2), host(g[0]), [host(x) for x in g[1]], [host(x) for x in g[2]])
        # KV-parallel prefill: rank r holds the pages of shards 2r, 2r + 1 of 4 in a pool of its own
        q3, kc, vc, bt, gqo = _kvp_case()
        mine = bt[2 * rank:2 * rank + 2]
        pages = np.unique(mine)
        remap = {int(pg): i for i, pg in enumerate(pages)}
        local_bt = torch.tensor([[remap[int(pg)] for pg in row] for row in mine], dtype=torch.int32)
        o3, l3 = cdist.kvp_segmented_prefill(dev(q3), dev(kc[pages]), dev(vc[pages]), local_bt, seg_size=128, scale=0.1,
                                             global_q_offset=gqo, sliding_window=400, via_host=True)
        torch.cuda.synchronize()
        res[rank] = (ring, uly, (host(o3), host(l3)))
    finally:
        dist.destroy_process_group()


def test_ring_ulysses_and_prefill_drivers_with_two_processes_on_this_gpu():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        res = m.dict()
        mp.start_processes(_dist_worker, args=(world, port, res), nprocs=world, join=True, start_method="spawn")
        res = dict(res)
    # ring
    cu = cu_from_lengths([264, 520, 128])
    S, H, HKV, D = int(cu[-1]), 4, 2, 128
    q, k, v, do = gen(83, (S, H, D), (S, HKV, D), (S, HKV, D), (S, H, D))
    out, lse = np.zeros((S, H, D)), np.zeros((H, S))
    gq, gk, gv = np.zeros((S, H, D)), np.zeros((S, HKV, D)), np.zeros((S, HKV, D))
    for r in range(world):
        loc = cbv.rank_tokens(cu, world, r, "zigzag")
        o, l, a, b, c = res[r][0]
        out[loc], lse[:, loc], gq[loc], gk[loc], gv[loc] = o, l, a, b, c
    ro, rl = A.attention_fwd(f64(q), f64(k), f64(v), cu, cu, 0.1)
    check_out(out, ro, what="ring out")
    check_lse(lse, rl, what="ring lse")
    rq, rk, rv = A.attention_bwd(f64(do), f64(q), f64(k), f64(v), out, rl, cu, cu, 0.1)
    check_rel(gq, rq, what="ring dq")
    check_rel(gk, rk, what="ring dk")
    check_rel(gv, rv, what="ring dv")
    # Ulysses
    cu2 = cu_from_lengths([100, 156])
    S2, NB = int(cu2[-1]), 3
    q2, ck, cv, do2 = gen(84, (S2, H, D), (NB, S2, HKV, D), (NB, S2, HKV, D), (S2, H, D))
    o2 = np.concatenate([res[r][1][0] for r in range(world)])
    l2 = np.concatenate([res[r][1][1] for r in range(world)], axis=1)
    dq2 = np.concatenate([res[r][1][2] for r in range(world)])
    dck = np.stack([np.concatenate([res[r][1][3][i] for r in range(world)]) for i in range(NB)])
    dcv = np.stack([np.concatenate([res[r][1][4][i] for r in range(world)]) for i in range(NB)])
    ro, rl = C.cached_fwd(f64(q2), f64(ck), f64(cv), cu2, 0.1)
    check_out(o2, ro, what="ulysses out")
    check_lse(l2, rl, what="ulysses lse")
    rq, rk, rv = C.cached_bwd(f64(do2), f64(q2), f64(ck), f64(cv), o2, rl, cu2, 0.1)
    check_rel(dq2, rq, what="ulysses dq")
    check_rel(dck, rk, what="ulysses dcache_k")
    check_rel(dcv, rv, what="ulysses dcache_v")
    # KV-parallel prefill: every rank returns the whole result, the same on both
    from oracle import paged as PG

    q3, kc, vc, bt, gqo = _kvp_case()
    K, V = PG.global_kv(f64(kc), f64(vc), bt, 32, PG.ROUND_ROBIN)
    ro, rl = PG.prefill_full(f64(q3), K, V, 0.1, gqo, window=400)
    for r in range(world):
        check_out(res[r][2][0], ro, what=f"prefill out on rank {r}")
        check_lse(res[r][2][1], rl, what=f"prefill lse on rank {r}")
    assert np.array_equal(res[0][2][0], res[1][2][0]) and np.array_equal(res[0][2][1], res[1][2][1])


# ----------------------------------------------------------------------------- Ulysses building blocks
@pytest.mark.parametrize("shape,dtype", [((2, 96, 3, 64), torch.bfloat16), ((4, 2, 37), torch.float32),
                                         ((3, 5, 16, 128), torch.float32)])
def test_swap_leading_axes_is_the_transpose(shape, dtype):
    x = torch.randn(shape, device="cuda").to(dtype)
    got = cbv.swap_leading_axes(x)
    sync()
    assert torch.equal(got, x.transpose(0, 1).contiguous())


@pytest.mark.parametrize("nb", [1, 3])
def test_diagonals_alone_on_a_block0_result(nb):
    cu = cu_from_lengths([70, 58])
    S, H, HKV, D = int(cu[-1]), 4, 2, 128
    q, ck, cv, do = gen(85, (S, H, D), (nb, S, HKV, D), (nb, S, HKV, D), (S, H, D))
    ro0, rl0 = A.attention_fwd(f64(q), f64(ck[0]), f64(cv[0]), cu, cu, 0.1)  # block 0 alone
    o0 = torch.from_numpy(ro0.astype(np.float32)).cuda()
    lse = torch.from_numpy(rl0.astype(np.float32)).cuda()
    tck, tcv = [dev(ck[i]) for i in range(nb)], [dev(cv[i]) for i in range(nb)]
    out, lse = cbv.cached_diag_merge(dev(q), tck, tcv, o0, lse, scale=0.1)
    sync()
    ro, rl = C.cached_fwd(f64(q), f64(ck), f64(cv), cu, 0.1)
    check_out(host(out), ro)
    check_lse(host(lse), rl)
    # gradients: block 0's dq from the oracle fed the merged statistics, the diagonals on the GPU
    rq, rk, rv = C.cached_bwd(f64(do), f64(q), f64(ck), f64(cv), host(out), rl, cu, 0.1)
    q0, _, _ = A.attention_bwd(f64(do), f64(q), f64(ck[0]), f64(cv[0]), host(out), rl, cu, cu, 0.1)
    dq0 = torch.from_numpy(q0.astype(np.float32)).cuda()
    dq, dck, dcv = cbv.cached_diag_grad(dev(do), dev(q), tck, tcv, out, lse, dq0, scale=0.1)
    sync()
    check_rel(host(dq), rq, what="dq")
    for i in range(1, nb):
        check_rel(host(dck[i]), rk[i], what=f"dk {i}")
        check_rel(host(dcv[i]), rv[i], what=f"dv {i}")
