"""The multi-rank drivers (ring over real ranks, Ulysses, KV-parallel prefill) with two gloo ranks on CPU.

The exchange code under test is the package's own: ``RingComm`` (send to rank+1,
receive from rank-1, commit / wait), the ring forward and backward with the dK/dV
accumulators travelling back to their owners, and Ulysses' all-to-alls between
sequence shards and head shards.  On CPU the per-step compute cannot be the CUDA
kernels, so each test hands the driver fp64 oracle blocks for its compute steps
(the way the GPU runs hand it the libcbv.so calls) and checks the assembled result
against full attention from the oracle.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import attention as A
from oracle import cached as C
from oracle import planner as P
from oracle.ring import _block_rows
from synth import normal_bf16, streams


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, world, port):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))


def _np(t):
    return t.detach().to(torch.float64).numpy()


# ----------------------------------------------------------------------------- ring
def _oracle_step_fwd(r, s, q, k, v, cu, cp, out_acc, lse_acc, out=None, scale=None, window=0, layout="zigzag"):
    name = P.ZIGZAG if layout == "zigzag" else P.CONTIGUOUS
    b = _block_rows(cu, cp, r, s, name)
    if b is not None:
        qi, kj, causal, cu_q, cu_k, src = b
        qpos = P.rank_tokens(cu, cp, r, name)[qi]
        kpos = P.rank_tokens(cu, cp, src, name)[kj]
        bo, bl = A.attention_fwd(_np(q)[qi], _np(k)[kj], _np(v)[kj], cu_q, cu_k, scale, causal=causal,
                                 window=window, qpos=qpos, kpos=kpos)
        if s == 0:
            no, nl = bo, bl
        else:
            no, nl, _ = A.update_out_and_lse(_np(out_acc)[qi], _np(lse_acc)[:, qi], bo, bl)
        out_acc[qi] = torch.from_numpy(no).to(out_acc.dtype)
        lse_acc[:, qi] = torch.from_numpy(nl).to(lse_acc.dtype)
    if out is not None:
        out.copy_(out_acc)


def _oracle_step_bwd(r, s, dout, q, k, v, out, lse, cu, cp, dq_acc, dk_acc, dv_acc, scale=None, window=0,
                     layout="zigzag"):
    name = P.ZIGZAG if layout == "zigzag" else P.CONTIGUOUS
    b = _block_rows(cu, cp, r, s, name)
    if b is None:
        return
    qi, kj, causal, cu_q, cu_k, src = b
    qpos = P.rank_tokens(cu, cp, r, name)[qi]
    kpos = P.rank_tokens(cu, cp, src, name)[kj]
    gq, gk, gv = A.attention_bwd(_np(dout)[qi], _np(q)[qi], _np(k)[kj], _np(v)[kj], _np(out)[qi], _np(lse)[:, qi],
                                 cu_q, cu_k, scale, causal=causal, window=window, qpos=qpos, kpos=kpos)
    dq_acc[qi] += torch.from_numpy(gq).to(dq_acc.dtype)
    dk_acc[kj] += torch.from_numpy(gk).to(dk_acc.dtype)
    dv_acc[kj] += torch.from_numpy(gv).to(dv_acc.dtype)


def _ring_inputs(lengths, H, HKV, D, seed):
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    S = int(cu[-1])
    g = streams(seed, 4)
    q, k, v, do = (normal_bf16(g[i], (S, h, D)).astype(np.float64) for i, h in enumerate((H, HKV, HKV, H)))
    return cu, q, k, v, do


def _ring_worker(rank, world, port, case, res):
    from context_blockwise_causal_varlen_b200 import dist as cdist

    _init(rank, world, port)
    try:
        lengths, H, HKV, D, layout, window = case
        cu, q, k, v, do = _ring_inputs(lengths, H, HKV, D, 3)
        name = P.ZIGZAG if layout == "zigzag" else P.CONTIGUOUS
        loc = P.rank_tokens(cu, world, rank, name)
        t = lambda x: torch.from_numpy(np.ascontiguousarray(x[loc]))
        out, lse = cdist.zigzag_ring_fwd(t(q), t(k), t(v), cu, scale=0.2, window=window, layout=layout,
                                         step_fwd=_oracle_step_fwd)
        dq, dk, dv = cdist.zigzag_ring_bwd(t(do), t(q), t(k), t(v), out, lse, cu, scale=0.2, window=window,
                                           layout=layout, step_bwd=_oracle_step_bwd, finish=lambda x: x)
        res[rank] = tuple(_np(x) for x in (out, lse, dq, dk, dv))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("case", [([48, 80], 2, 1, 16, "zigzag", 0), ([40, 8, 72], 2, 2, 8, "zigzag", 21),
                                  ([48, 80], 2, 1, 16, "contiguous", 0)])
def test_ring_over_two_ranks_equals_full_attention(case):
    world, port = 2, _free_port()
    with mp.Manager() as m:
        res = m.dict()
        mp.spawn(_ring_worker, args=(world, port, case, res), nprocs=world, join=True)
        res = dict(res)
    lengths, H, HKV, D, layout, window = case
    cu, q, k, v, do = _ring_inputs(lengths, H, HKV, D, 3)
    name = P.ZIGZAG if layout == "zigzag" else P.CONTIGUOUS
    S = int(cu[-1])
    out, lse = np.zeros((S, H, D)), np.zeros((H, S))
    dq, dk, dv = np.zeros((S, H, D)), np.zeros((S, HKV, D)), np.zeros((S, HKV, D))
    for r in range(world):
        loc = P.rank_tokens(cu, world, r, name)
        o, l, gq, gk, gv = res[r]
        out[loc], lse[:, loc], dq[loc], dk[loc], dv[loc] = o, l, gq, gk, gv
    ro, rl = A.attention_fwd(q, k, v, cu, cu, 0.2, causal=True, window=window)
    rq, rk, rv = A.attention_bwd(do, q, k, v, ro, rl, cu, cu, 0.2, causal=True, window=window)
    np.testing.assert_allclose(out, ro, atol=1e-5)
    np.testing.assert_allclose(lse, rl, atol=1e-5)
    for got, ref in ((dq, rq), (dk, rk), (dv, rv)):
        np.testing.assert_allclose(got, ref, atol=1e-5 * max(1.0, np.abs(ref).max()))


# ----------------------------------------------------------------------------- Ulysses
class _OracleUlyssesOps:
    """Ulysses' compute steps as fp64 oracle blocks on CPU (the GPU path uses libcbv.so calls)."""

    scale = 0.25

    @staticmethod
    def swap(x):
        return x.transpose(0, 1).contiguous()

    @staticmethod
    def block0_fwd(q, k, v, cu, scale):
        o, l = A.attention_fwd(_np(q), _np(k), _np(v), cu, cu, scale, causal=True)
        return torch.from_numpy(o), torch.from_numpy(l)

    @staticmethod
    def block0_bwd(dout, q, k, v, out, lse, cu, scale):
        g = A.attention_bwd(_np(dout), _np(q), _np(k), _np(v), _np(out), _np(lse), cu, cu, scale, causal=True)
        return tuple(torch.from_numpy(x) for x in g)

    @staticmethod
    def _diag(q, ck, cv, scale):
        qn = _np(q)
        H, hkv = qn.shape[1], ck[0].shape[1]
        g = H // hkv
        ks = [np.repeat(_np(x), g, axis=1) for x in ck]
        vs = [np.repeat(_np(x), g, axis=1) for x in cv]
        s = [scale * (qn * ks[i]).sum(-1).T for i in range(len(ck))]  # [H, T]
        return qn, ks, vs, s, g

    @classmethod
    def diag_merge(cls, q, ck, cv, o32, lse, scale):
        _, ks, vs, s, _ = cls._diag(q, ck, cv, scale)
        out, l = _np(o32), _np(lse)
        for i in range(1, len(ck)):
            out, l, _ = A.update_out_and_lse(out, l, vs[i], s[i])
        return torch.from_numpy(out), torch.from_numpy(l)

    @classmethod
    def diag_grad(cls, dout, q, ck, cv, out, lse, dq0, scale):
        qn, ks, vs, s, g = cls._diag(q, ck, cv, scale)
        do, o, l = _np(dout), _np(out), _np(lse)
        delta = (do * o).sum(-1)  # [T, H]
        dq = _np(dq0)
        dck, dcv = [None], [None]
        for i in range(1, len(ck)):
            p = np.exp(s[i] - l).T  # [T, H]
            ds = p * ((do * vs[i]).sum(-1) - delta)
            dq = dq + scale * ds[..., None] * ks[i]
            T, H, D = qn.shape
            dck.append(torch.from_numpy((scale * ds[..., None] * qn).reshape(T, H // g, g, D).sum(2)))
            dcv.append(torch.from_numpy((p[..., None] * do).reshape(T, H // g, g, D).sum(2)))
        return torch.from_numpy(dq), dck, dcv

    @staticmethod
    def finish(x):
        return x


def _ulysses_inputs(lengths, H, HKV, D, NB, seed):
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    S = int(cu[-1])
    g = streams(seed, 4)
    q, do = normal_bf16(g[0], (S, H, D)).astype(np.float64), normal_bf16(g[3], (S, H, D)).astype(np.float64)
    ck = normal_bf16(g[1], (NB, S, HKV, D)).astype(np.float64)
    cv = normal_bf16(g[2], (NB, S, HKV, D)).astype(np.float64)
    return cu, q, ck, cv, do


def _ulysses_worker(rank, world, port, case, res):
    from context_blockwise_causal_varlen_b200 import dist as cdist

    _init(rank, world, port)
    try:
        lengths, H, HKV, D, NB = case
        cu, q, ck, cv, do = _ulysses_inputs(lengths, H, HKV, D, NB, 5)
        S = int(cu[-1])
        n = S // world
        sl = slice(rank * n, (rank + 1) * n)
        t = lambda x: torch.from_numpy(np.ascontiguousarray(x))
        lck, lcv = [t(ck[i, sl]) for i in range(NB)], [t(cv[i, sl]) for i in range(NB)]
        ops = _OracleUlyssesOps()
        out, lse = cdist.ulysses_fwd(t(q[sl]), lck, lcv, cu, scale=0.25, ops=ops)
        dq, dck, dcv = cdist.ulysses_bwd(t(do[sl]), t(q[sl]), lck, lcv, out, lse, cu, scale=0.25, ops=ops)
        res[rank] = (_np(out), _np(lse), _np(dq), [_np(x) for x in dck], [_np(x) for x in dcv])
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("case", [([24, 40], 4, 2, 16, 3), ([64], 2, 2, 8, 1)])
def test_ulysses_over_two_ranks_equals_the_joint_softmax(case):
    world, port = 2, _free_port()
    with mp.Manager() as m:
        res = m.dict()
        mp.spawn(_ulysses_worker, args=(world, port, case, res), nprocs=world, join=True)
        res = dict(res)
    lengths, H, HKV, D, NB = case
    cu, q, ck, cv, do = _ulysses_inputs(lengths, H, HKV, D, NB, 5)
    S = int(cu[-1])
    n = S // world
    out = np.concatenate([res[r][0] for r in range(world)])
    lse = np.concatenate([res[r][1] for r in range(world)], axis=1)
    dq = np.concatenate([res[r][2] for r in range(world)])
    dck = np.stack([np.concatenate([res[r][3][i] for r in range(world)]) for i in range(NB)])
    dcv = np.stack([np.concatenate([res[r][4][i] for r in range(world)]) for i in range(NB)])
    ro, rl = C.cached_fwd(q, ck, cv, cu, 0.25)
    rq, rk, rv = C.cached_bwd(do, q, ck, cv, ro, rl, cu, 0.25)
    np.testing.assert_allclose(out, ro, atol=1e-10)
    np.testing.assert_allclose(lse, rl, atol=1e-10)
    np.testing.assert_allclose(dq, rq, atol=1e-9)
    np.testing.assert_allclose(dck, rk, atol=1e-9)
    np.testing.assert_allclose(dcv, rv, atol=1e-9)
    assert out.shape == (S, H, D) and n * world == S


# ----------------------------------------------------------------------------- KV-parallel prefill
def _kvp_inputs():
    from oracle import paged as PG
    from synth import block_permutation

    R, bps, bs, hq, hkv, D, S = 4, 2, 8, 2, 1, 8, 24
    g = streams(7, 4)
    q = normal_bf16(g[0], (hq, S, D)).astype(np.float64)
    kc = normal_bf16(g[1], (R * bps, hkv, bs, D)).astype(np.float64)
    vc = normal_bf16(g[2], (R * bps, hkv, bs, D)).astype(np.float64)
    bt = PG.shard_block_tables(block_permutation(g[3], R * bps), R, PG.ROUND_ROBIN)
    return q, kc, vc, bt, R * bps * bs - S - 3


def _kvp_worker(rank, world, port, res):
    from context_blockwise_causal_varlen_b200 import dist as cdist
    from oracle import paged as PG
    from oracle.attention import attention_fwd_masked

    _init(rank, world, port)
    try:
        q, kc, vc, bt, gqo = _kvp_inputs()
        n, bs, R = 2, 8, bt.shape[0]
        mine = bt[rank * n:(rank + 1) * n]

        def partial(shard_base, total_shards):
            # the shards' partials from the oracle, at their GLOBAL positions (shard_base + i of total_shards)
            so, sl = [], []
            for i in range(n):
                kpos = PG.local_to_global_positions(shard_base + i, mine.shape[1] * bs, bs, total_shards,
                                                    PG.ROUND_ROBIN)
                mask = PG._mask(gqo + np.arange(q.shape[1]), kpos, 10)
                o, l = attention_fwd_masked(q.transpose(1, 0, 2), PG.gather_shard_kv(kc, mine[i], bs),
                                            PG.gather_shard_kv(vc, mine[i], bs), mask, 0.3)
                so.append(o.transpose(1, 0, 2))
                sl.append(l)
            return torch.from_numpy(np.stack(so)), torch.from_numpy(np.stack(sl))

        def merge(out, lse, bo, bl):
            no, nl, _ = A.update_out_and_lse(_np(out), _np(lse), _np(bo), _np(bl))
            out.copy_(torch.from_numpy(no))
            lse.copy_(torch.from_numpy(nl))

        out, lse = cdist.kvp_segmented_prefill(torch.from_numpy(q), None, None, torch.from_numpy(mine),
                                               partial=partial, merge=merge, finish=lambda x: x)
        res[rank] = (_np(out), _np(lse))
    finally:
        dist.destroy_process_group()


def test_kvp_prefill_over_two_ranks_equals_the_whole_context():
    from oracle import paged as PG

    world, port = 2, _free_port()
    with mp.Manager() as m:
        res = m.dict()
        mp.spawn(_kvp_worker, args=(world, port, res), nprocs=world, join=True)
        res = dict(res)
    q, kc, vc, bt, gqo = _kvp_inputs()
    K, V = PG.global_kv(kc, vc, bt, 8, PG.ROUND_ROBIN)
    ro, rl = PG.prefill_full(q, K, V, 0.3, gqo, window=10)
    for r in range(world):
        np.testing.assert_allclose(res[r][0], ro, atol=1e-12)
        np.testing.assert_allclose(res[r][1], rl, atol=1e-12)
