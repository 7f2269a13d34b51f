"""Paged KV-parallel prefill and varlen decode on the GPU against the fp64 oracle."""
import numpy as np
import pytest
import torch

import context_blockwise_causal_varlen_b200 as cbv
from oracle import decode as DEC
from oracle import paged as PG
from synth import block_permutation, cu_from_lengths, streams
from tests.gpu_util import GuardedWorkspaces, check_guards, check_lse, check_out, dev, f64, gen, guarded, host, sync

pytestmark = pytest.mark.gpu


def _paged(seed, R, bps, bs, hq, hkv, D, S):
    nb = R * bps
    q, kc, vc = gen(seed, (hq, S, D), (nb, hkv, bs, D), (nb, hkv, bs, D))
    perm = block_permutation(streams(seed + 100, 1)[0], nb)
    return q, kc, vc, perm


@pytest.mark.parametrize("mode", [PG.ROUND_ROBIN, PG.CONTIGUOUS])
@pytest.mark.parametrize("window,seg", [(0, 128), (300, 256), (700, 128)])
def test_kvp_prefill_matches_oracle(mode, window, seg):
    R, bps, bs, hq, hkv, D, S = 4, 8, 32, 8, 2, 128, 300
    q, kc, vc, perm = _paged(20, R, bps, bs, hq, hkv, D, S)
    bt = PG.shard_block_tables(perm, R, mode)
    gqo = R * bps * bs - S - 17
    K, V = PG.global_kv(f64(kc), f64(vc), bt, bs, mode)
    ro, rl = PG.prefill_full(f64(q), K, V, 0.1, gqo, window=window)
    kv_mode = cbv.KV_ROUND_ROBIN if mode == PG.ROUND_ROBIN else cbv.KV_CONTIGUOUS
    (out, ob), (lse, lb) = guarded((hq, S, D), torch.bfloat16), guarded((hq, S), torch.float32)
    wss = GuardedWorkspaces()
    cbv.kvp_segmented_prefill(dev(q), dev(kc), dev(vc), torch.from_numpy(bt), kv_mode=kv_mode, seg_size=seg,
                              scale=0.1, global_q_offset=gqo, sliding_window=window, out=out, lse=lse, workspace=wss)
    sync()
    check_guards(out, ob, what="out")
    check_guards(lse, lb, what="lse")
    wss.check()
    check_out(host(out), ro)
    check_lse(host(lse), rl)


def test_kvp_per_shard_partials_and_their_merge():
    R, bps, bs, hq, hkv, D, S = 4, 4, 32, 4, 1, 128, 200
    q, kc, vc, perm = _paged(21, R, bps, bs, hq, hkv, D, S)
    bt = PG.shard_block_tables(perm, R, PG.ROUND_ROBIN)
    gqo = 300
    (ro, rl), shards = PG.prefill_segmented(f64(q), f64(kc), f64(vc), bt, bs, 128, 0.1, gqo, window=0,
                                            mode=PG.ROUND_ROBIN, return_shards=True)
    (so_, sob), (sl_, slb) = guarded((R, hq, S, D), torch.float32), guarded((R, hq, S), torch.float32)
    (o_, obuf), (l_, lbuf) = guarded((hq, S, D), torch.bfloat16), guarded((hq, S), torch.float32)
    wss = GuardedWorkspaces()
    out, lse, so, sl = cbv.kvp_segmented_prefill(dev(q), dev(kc), dev(vc), torch.from_numpy(bt), seg_size=128,
                                                 scale=0.1, global_q_offset=gqo, per_shard=True, out=o_, lse=l_,
                                                 shard_out=so_, shard_lse=sl_, workspace=wss)
    sync()
    for t, b, n in ((so_, sob, "shard_out"), (sl_, slb, "shard_lse"), (o_, obuf, "out"), (l_, lbuf, "lse")):
        check_guards(t, b, what=n)
    wss.check()
    check_out(host(out), ro)
    check_lse(host(lse), rl)
    for r in range(R):
        check_out(host(so[r]), shards[r][0], what=f"shard {r} out")
        check_lse(host(sl[r]), shards[r][1], what=f"shard {r} lse")


@pytest.mark.parametrize("mode,window", [(PG.ROUND_ROBIN, 0), (PG.CONTIGUOUS, 0), (PG.ROUND_ROBIN, 500)])
def test_kvp_shards_split_over_calls_give_the_same_partials(mode, window):
    # a call that holds only some of the shards (shard_base / total_shards, as a process that holds only
    # its own pages would) computes exactly the partials the whole call computes for them, and the
    # partials of two calls merge to the full result
    R, bps, bs, hq, hkv, D, S = 4, 4, 32, 4, 2, 128, 200
    q, kc, vc, perm = _paged(23, R, bps, bs, hq, hkv, D, S)
    bt = PG.shard_block_tables(perm, R, mode)
    gqo = R * bps * bs - S - 9
    kv_mode = cbv.KV_ROUND_ROBIN if mode == PG.ROUND_ROBIN else cbv.KV_CONTIGUOUS
    kw = dict(kv_mode=kv_mode, seg_size=128, scale=0.1, global_q_offset=gqo, sliding_window=window,
              per_shard=True, return_lse=True)
    _, _, so_all, sl_all = cbv.kvp_segmented_prefill(dev(q), dev(kc), dev(vc), torch.from_numpy(bt), **kw)
    parts = []
    for base in (0, 2):
        (so_, sob), (sl_, slb) = guarded((2, hq, S, D), torch.float32), guarded((2, hq, S), torch.float32)
        out, lse, so, sl = cbv.kvp_segmented_prefill(dev(q), dev(kc), dev(vc), torch.from_numpy(bt[base:base + 2]),
                                                     shard_base=base, total_shards=R, shard_out=so_, shard_lse=sl_,
                                                     **kw)
        sync()
        check_guards(so_, sob, what="shard_out")
        check_guards(sl_, slb, what="shard_lse")
        assert torch.equal(so, so_all[base:base + 2]) and torch.equal(sl, sl_all[base:base + 2])
        parts.append((out, lse))
    K, V = PG.global_kv(f64(kc), f64(vc), bt, bs, mode)
    ro, rl = PG.prefill_full(f64(q), K, V, 0.1, gqo, window=window)
    # the two calls' merged halves (each over its own shards) merge to the whole result
    o32 = parts[0][0].float().reshape(hq * S, 1, D).contiguous()
    l32 = parts[0][1].reshape(1, hq * S).contiguous()
    cbv.attn_merge(o32, l32, parts[1][0].reshape(hq * S, 1, D), parts[1][1].reshape(1, hq * S))
    sync()
    check_lse(host(l32.reshape(hq, S)), rl)
    np.testing.assert_allclose(host(o32.reshape(hq, S, D)), ro, atol=2e-2)


def test_kvp_segment_size_does_not_change_the_result():
    R, bps, bs, hq, hkv, D, S = 2, 16, 16, 4, 2, 64, 256
    q, kc, vc, perm = _paged(22, R, bps, bs, hq, hkv, D, S)
    bt = torch.from_numpy(PG.shard_block_tables(perm, R, PG.ROUND_ROBIN))
    a = cbv.kvp_segmented_prefill(dev(q), dev(kc), dev(vc), bt, seg_size=128, global_q_offset=256)
    b = cbv.kvp_segmented_prefill(dev(q), dev(kc), dev(vc), bt, seg_size=256, global_q_offset=256)
    sync()
    assert torch.allclose(a[0].float(), b[0].float(), atol=1e-2)
    assert torch.allclose(a[1], b[1], atol=1e-4)


@pytest.mark.parametrize("hq,hkv,D", [(32, 4, 128), (8, 8, 128), (16, 2, 64), (12, 3, 128)])
def test_decode_matches_oracle(hq, hkv, D):
    lengths = np.concatenate([[0, 1, 2, 31, 32, 33, 64, 65], streams(30, 1)[0].integers(1, 700, 40)])
    n = len(lengths)
    cu_k = cu_from_lengths(lengths)
    q, k, v = gen(31, (n, hq, D), (int(cu_k[-1]), hkv, D), (int(cu_k[-1]), hkv, D))
    cu_q = np.arange(n + 1, dtype=np.int32)
    ref = DEC.varlen_decode(f64(q), f64(k), f64(v), cu_q, cu_k, 0.1)
    out, ob = guarded((n, hq, D), torch.bfloat16)
    cbv.varlen_decode(dev(q), dev(k), dev(v), torch.from_numpy(cu_q), torch.from_numpy(cu_k), scale=0.1, out=out)
    sync()
    check_guards(out, ob, what="decode out")
    check_out(host(out), ref)
    assert np.all(host(out)[0] == 0)  # empty key range -> zeros


def test_decode_reads_offsets_on_device():
    # change cu_seqlens_k contents in place (no host round trip) and run again
    hq, hkv, D = 8, 2, 128
    lengths = np.array([5, 100, 0, 77])
    cu_k = cu_from_lengths(lengths)
    q, k, v = gen(32, (4, hq, D), (400, hkv, D), (400, hkv, D))
    cu_q = torch.arange(5, dtype=torch.int32, device="cuda")
    ck = torch.from_numpy(cu_k).cuda()
    out = torch.empty((4, hq, D), dtype=torch.bfloat16, device="cuda")
    cbv.varlen_decode(dev(q), dev(k), dev(v), cu_q, ck, scale=0.1, validate=False, out=out)
    new = cu_from_lengths([50, 0, 200, 1])
    ck.copy_(torch.from_numpy(new))
    cbv.varlen_decode(dev(q), dev(k), dev(v), cu_q, ck, scale=0.1, validate=False, out=out)
    sync()
    ref = DEC.varlen_decode(f64(q), f64(k), f64(v), np.arange(5), new, 0.1)
    check_out(host(out), ref)


def test_decode_rejects_more_than_one_query_per_sequence():
    q, k, v = gen(33, (4, 8, 128), (10, 2, 128), (10, 2, 128))
    with pytest.raises(cbv.CbvError) as e:
        cbv.varlen_decode(dev(q), dev(k), dev(v), torch.tensor([0, 1, 3, 4]), torch.tensor([0, 3, 6, 10]))
    assert e.value.status == "Q_LEN_NOT_ONE"


@pytest.mark.parametrize("per_shard", [False, True])
@pytest.mark.parametrize("D,S", [(128, 300), (64, 1), (64, 97)])
def test_kvp_transposed_output_is_the_transpose(per_shard, D, S):
    # tp_out: out is [HQ, D, S], element for element the transpose of the [HQ, S, D] output
    R, bps, bs, hq, hkv = 4, 8, 32, 4, 2
    q, kc, vc, perm = _paged(23, R, bps, bs, hq, hkv, D, S)
    bt = torch.from_numpy(PG.shard_block_tables(perm, R, PG.ROUND_ROBIN))
    gqo = R * bps * bs - S
    kw = dict(seg_size=256, scale=0.1, global_q_offset=gqo, sliding_window=500, per_shard=per_shard)
    a = cbv.kvp_segmented_prefill(dev(q), dev(kc), dev(vc), bt, **kw)
    b = cbv.kvp_segmented_prefill(dev(q), dev(kc), dev(vc), bt, tp_out=True, **kw)
    sync()
    assert b[0].shape == (hq, D, S)
    assert torch.equal(b[0], a[0].transpose(1, 2))
    assert torch.equal(b[1], a[1])
    K, V = PG.global_kv(f64(kc), f64(vc), bt.numpy(), bs, PG.ROUND_ROBIN)
    ro, _ = PG.prefill_full(f64(q), K, V, 0.1, gqo, window=500)
    check_out(host(b[0]).transpose(0, 2, 1), ro)


@pytest.mark.parametrize("window,tp_out", [(0, False), (3000, True)])
def test_kvp_tail_tasks_split_in_halves(window, tp_out):
    # 11 q tile pairs x 16 heads = 176 tasks: 148 fill one wave and the other 28 run as two halves
    # each (cut along the segment list), merged afterwards; every pair and head is sampled
    R, bps, bs, hq, hkv, D, S = 4, 64, 32, 16, 4, 128, 11 * 256
    q, kc, vc, perm = _paged(60, R, bps, bs, hq, hkv, D, S)
    bt = PG.shard_block_tables(perm, R, PG.ROUND_ROBIN)
    gqo = R * bps * bs - S
    (out, ob), (lse, lb) = guarded((hq, D, S) if tp_out else (hq, S, D), torch.bfloat16), guarded((hq, S), torch.float32)
    wss = GuardedWorkspaces()
    n0 = cbv.launch_count()
    cbv.kvp_segmented_prefill(dev(q), dev(kc), dev(vc), torch.from_numpy(bt), seg_size=512, scale=0.1,
                              global_q_offset=gqo, sliding_window=window, tp_out=tp_out, out=out, lse=lse,
                              workspace=wss)
    sync()
    check_guards(out, ob, what="out")
    check_guards(lse, lb, what="lse")
    wss.check()
    assert cbv.launch_count() - n0 == 3  # schedule, the prefill (whole tasks and halves), the merge
    rows = np.unique(np.concatenate([[p, p + 1, p + 127, p + 128, p + 255] for p in range(0, S, 256)]))
    K, V = PG.global_kv(f64(kc), f64(vc), bt, bs, PG.ROUND_ROBIN)
    ro, rl = PG.prefill_full(f64(q), K, V, 0.1, gqo, window=window, rows=rows)
    got = host(out).transpose(0, 2, 1) if tp_out else host(out)
    check_out(got[:, rows], ro[:, rows])
    check_lse(host(lse)[:, rows], rl[:, rows])


def test_kvp_every_task_split_when_fewer_than_half_the_sms():
    # one q tile pair x 16 heads = 16 tasks, fewer than half the SMs: every task runs as two halves
    R, bps, bs, hq, hkv, D, S = 4, 32, 32, 16, 4, 128, 256
    q, kc, vc, perm = _paged(61, R, bps, bs, hq, hkv, D, S)
    bt = PG.shard_block_tables(perm, R, PG.CONTIGUOUS)
    gqo = R * bps * bs - S
    n0 = cbv.launch_count()
    out, lse = cbv.kvp_segmented_prefill(dev(q), dev(kc), dev(vc), torch.from_numpy(bt), kv_mode=cbv.KV_CONTIGUOUS,
                                         seg_size=256, scale=0.1, global_q_offset=gqo, sliding_window=3000)
    sync()
    assert cbv.launch_count() - n0 == 3
    K, V = PG.global_kv(f64(kc), f64(vc), bt, bs, PG.CONTIGUOUS)
    ro, rl = PG.prefill_full(f64(q), K, V, 0.1, gqo, window=3000)
    check_out(host(out), ro)
    check_lse(host(lse), rl)
