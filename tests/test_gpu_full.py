"""Parity at the benchmark's full sizes, in the launch configuration bench.py times.

The oracle cannot run these sizes whole, so each test checks outputs it can compute
one by one: whole documents (documents are independent), sampled query rows
(each row's softmax is independent), the last key tiles (whose gradients only the
last rows reach), sampled decode sequences; plus properties that hold at any size
(the sum rules of the joint softmax).
"""
import numpy as np
import pytest
import torch

import context_blockwise_causal_varlen_b200 as cbv
from oracle import attention as A
from oracle import decode as DEC
from oracle import paged as PG
from synth import torch_normal_bf16
from synth.workloads import long_doc, packed_zigzag, paged_prefill, varlen_decode
from tests.gpu_util import GuardedWorkspaces, check_guards, check_lse, check_out, check_rel, guarded, host

pytestmark = pytest.mark.gpu


def _ring_inputs(w, seed):
    return [torch_normal_bf16((w.total, w.heads, w.head_dim), seed * 10 + i) for i in range(4)]


def _f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("schedule", [cbv.SCHEDULE_FUSED, cbv.SCHEDULE_STEPWISE])
def test_packed_zigzag_full_size(schedule):
    # every document (documents are independent) for three heads, forward and backward, with
    # canaries around every output and workspace
    w = packed_zigzag(0)
    cu = w.cu_seqlens
    S, H, D = w.total, w.heads, w.head_dim
    q, k, v, do = _ring_inputs(w, 0)
    (out, ob), (lse, lb) = guarded((S, H, D), torch.bfloat16), guarded((H, S), torch.float32)
    (dq, gq), (dk, gk), (dv, gv) = (guarded((S, H, D), torch.bfloat16) for _ in range(3))
    wss = GuardedWorkspaces()
    cbv.zigzag_ring_fwd(q, k, v, cu, w.cp, schedule=schedule, out=out, lse=lse, workspace=wss)
    cbv.zigzag_ring_bwd(do, q, k, v, out, lse, cu, w.cp, dq=dq, dk=dk, dv=dv, workspace=wss)
    torch.cuda.synchronize()
    for t, b, n in ((out, ob, "out"), (lse, lb, "lse"), (dq, gq, "dq"), (dk, gk, "dk"), (dv, gv, "dv")):
        check_guards(t, b, what=n)
    wss.check()
    scale = D ** -0.5
    for d in range(len(cu) - 1):
        a, b = int(cu[d]), int(cu[d + 1])
        one = np.array([0, b - a])
        for h in (0, 17, 31):
            sl = (slice(a, b), slice(h, h + 1))
            qh, kh, vh, dh = (_f64(t[sl]) for t in (q, k, v, do))
            ro, rl = A.attention_fwd(qh, kh, vh, one, one, scale)
            check_out(_f64(out[sl]), ro, what=f"out doc {d} head {h}")
            check_lse(host(lse[h:h + 1, a:b]), rl, what=f"lse doc {d} head {h}")
            rq, rk, rv = A.attention_bwd(dh, qh, kh, vh, _f64(out[sl]), rl, one, one, scale)
            check_rel(_f64(dq[sl]), rq, what=f"dq doc {d} head {h}")
            check_rel(_f64(dk[sl]), rk, what=f"dk doc {d} head {h}")
            check_rel(_f64(dv[sl]), rv, what=f"dv doc {d} head {h}")


@pytest.mark.parametrize("window,layout", [(0, "zigzag"), (4096, "zigzag"), (0, "contiguous")])
def test_long_document_full_size(window, layout):
    w = long_doc(window=window)
    S, cu = w.total, w.cu_seqlens
    q, k, v, do = _ring_inputs(w, 7)
    out, lse = cbv.zigzag_ring_fwd(q, k, v, cu, w.cp, window=window, layout=layout)
    dq, dk, dv = cbv.zigzag_ring_bwd(do, q, k, v, out, lse, cu, w.cp, window=window, layout=layout)
    torch.cuda.synchronize()
    scale = w.head_dim ** -0.5
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([[0, 1, 4095, 4096, 8191, 32767, 32768, S - 1], rng.integers(0, S, 12)]))
    tail = np.arange(S - 64, S)
    for h in (0, 15):
        qh, kh, vh, dh = (_f64(t[:, h:h + 1]) for t in (q, k, v, do))
        ro, rl = A.attention_fwd(qh, kh, vh, cu, cu, scale, window=window, rows=np.concatenate([rows, tail]))
        check_out(_f64(out[rows, h:h + 1]), ro[rows], what=f"out head {h}")
        check_lse(host(lse[h:h + 1, rows]), rl[:, rows], what=f"lse head {h}")
        gq = A.attention_grad_rows(dh, qh, kh, vh, ro, rl, cu, cu, scale, rows, [0], window=window)
        check_rel(_f64(dq[rows, h:h + 1]), gq, what=f"dq head {h}")
        gk, gv = A.attention_grad_cols(dh, qh, kh, vh, ro, rl, cu, cu, scale, tail, [0], window=window)
        check_rel(_f64(dk[tail, h:h + 1]), gk, what=f"dk tail head {h}")
        check_rel(_f64(dv[tail, h:h + 1]), gv, what=f"dv tail head {h}")
        # sum rules over the whole sequence: sum_j dv_j = sum_i dO_i, sum_j dk_j = 0
        gdv, gdk = _f64(dv[:, h]), _f64(dk[:, h])
        assert np.abs(gdv.sum(0) - dh[:, 0].sum(0)).max() <= 0.05 * np.sqrt((dh[:, 0] ** 2).sum(0)).max()
        assert np.abs(gdk.sum(0)).max() <= 0.05 * np.sqrt((gdk ** 2).sum(0)).max()


@pytest.mark.parametrize("window,mode", [(0, PG.ROUND_ROBIN), (8192, PG.ROUND_ROBIN), (0, PG.CONTIGUOUS)])
def test_paged_prefill_full_size(window, mode):
    w = paged_prefill(window=window)
    q = torch_normal_bf16((w.hq, w.q_len, w.head_dim), 11)
    kc = torch_normal_bf16((w.kv_len // w.block_size, w.hkv, w.block_size, w.head_dim), 12)
    vc = torch_normal_bf16(kc.shape, 13)
    bt = PG.shard_block_tables(w.perm, w.shards, mode)
    kv_mode = cbv.KV_ROUND_ROBIN if mode == PG.ROUND_ROBIN else cbv.KV_CONTIGUOUS
    out, lse = cbv.kvp_segmented_prefill(q, kc, vc, torch.from_numpy(bt), kv_mode, w.seg_size, None,
                                         w.global_q_offset, window)
    torch.cuda.synchronize()
    rng = np.random.default_rng(6)
    rows = np.unique(np.concatenate([[0, 1, 2047, w.q_len - 1], rng.integers(0, w.q_len, 12)]))
    for h in (0, 5, 31):
        kv = h // (w.hq // w.hkv)
        K, V = PG.global_kv(_f64(kc[:, kv:kv + 1]), _f64(vc[:, kv:kv + 1]), bt, w.block_size, mode)
        ro, rl = PG.prefill_full(_f64(q[h:h + 1]), K, V, w.head_dim ** -0.5, w.global_q_offset, window, rows=rows)
        check_out(_f64(out[h:h + 1, rows]), ro[:, rows], what=f"prefill out head {h}")
        check_lse(host(lse[h:h + 1, rows]), rl[:, rows], what=f"prefill lse head {h}")


def test_varlen_decode_full_size():
    w = varlen_decode()
    cu_k = w.cu_seqlens_k
    tk = int(cu_k[-1])
    q = torch_normal_bf16((w.num_seqs, w.hq, w.head_dim), 21)
    k = torch_normal_bf16((tk, w.hkv, w.head_dim), 22)
    v = torch_normal_bf16((tk, w.hkv, w.head_dim), 23)
    cu_q = torch.arange(w.num_seqs + 1, dtype=torch.int32)
    out = cbv.varlen_decode(q, k, v, cu_q, torch.from_numpy(cu_k))
    torch.cuda.synchronize()
    counts = np.diff(cu_k)
    rng = np.random.default_rng(7)
    seqs = np.unique(np.concatenate([[0, w.num_seqs - 1, int(np.argmax(counts)), int(np.argmin(counts))],
                                     rng.integers(0, w.num_seqs, 60)]))
    for s in seqs:
        a, b = int(cu_k[s]), int(cu_k[s + 1])
        ref = DEC.varlen_decode(_f64(q[s:s + 1]), _f64(k[a:b]), _f64(v[a:b]), [0, 1], [0, b - a],
                                w.head_dim ** -0.5)
        check_out(_f64(out[s:s + 1]), ref, what=f"decode seq {s}")
