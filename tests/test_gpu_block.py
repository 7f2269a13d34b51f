"""Block forward / merge / block backward on the GPU against the fp64 oracle."""
import numpy as np
import pytest
import torch

import context_blockwise_causal_varlen_b200 as cbv
from oracle import attention as A
from synth import cu_from_lengths
from tests.gpu_util import check_lse, check_out, check_rel, dev, f64, gen, host, sync

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("lq,lk,causal,window,D", [
    ([200, 130], [300, 130], True, 0, 128),
    ([64, 257], [64, 400], True, 50, 64),
    ([128], [500], False, 0, 128),
    ([1, 300, 0], [5, 0, 7], True, 0, 128),
])
def test_block_forward_default_positions(lq, lk, causal, window, D):
    cq, ck = cu_from_lengths(lq), cu_from_lengths(lk)
    q, k, v = gen(10, (int(cq[-1]), 4, D), (int(ck[-1]), 2, D), (int(ck[-1]), 2, D))
    ro, rl = A.attention_fwd(f64(q), f64(k), f64(v), cq, ck, 0.1, causal=causal, window=window)
    for dt in (torch.bfloat16, torch.float32):
        out, lse = cbv.attn_block_fwd(dev(q), dev(k), dev(v), cq, ck, scale=0.1, causal=causal, window=window,
                                      out_dtype=dt)
        sync()
        assert out.dtype == dt
        check_out(host(out), ro)
        check_lse(host(lse), rl)


@pytest.mark.parametrize("offset", [0, 5])
@pytest.mark.parametrize("window", [31, 32, 33, 96, 128, 129])
def test_window_edges_on_and_beside_every_32_column_boundary(window, offset):
    # the forward masks 32 score columns at a time and skips the chunks that every row of a warp
    # sees whole: windows whose lower edge falls just before, on and just after a chunk boundary,
    # and queries shifted by a few positions against the keys, so the edges pass through every lane
    L, H, D = 384, 2, 128
    q, k, v = gen(30 + window + offset, (L, H, D), (L, H, D), (L, H, D))
    qpos, kpos = offset + np.arange(L), np.arange(L)
    ro, rl = A.attention_fwd(f64(q), f64(k), f64(v), [0, L], [0, L], 0.1, causal=True, window=window, qpos=qpos,
                             kpos=kpos)
    out, lse = cbv.attn_block_fwd(dev(q), dev(k), dev(v), [0, L], [0, L], scale=0.1, causal=True, window=window,
                                  q_pos_base=[offset], k_pos_base=[0])
    sync()
    check_out(host(out), ro)
    check_lse(host(lse), rl)


def test_blocks_merged_in_place_equal_full_attention():
    # one document split into three key blocks with explicit global positions,
    # merged into a running pair by the fused epilogue in a scrambled order
    L, H, D = 700, 2, 128
    q, k, v = gen(11, (L, H, D), (L, H, D), (L, H, D))
    ro, rl = A.attention_fwd(f64(q), f64(k), f64(v), [0, L], [0, L], 0.08, causal=True, window=333)
    cuts = [0, 250, 251, 700]
    out = torch.zeros((L, H, D), dtype=torch.float32, device="cuda")
    lse = torch.full((H, L), -float("inf"), dtype=torch.float32, device="cuda")
    for b in (2, 0, 1):
        a0, a1 = cuts[b], cuts[b + 1]
        cbv.attn_block_fwd(dev(q), dev(k[a0:a1]), dev(v[a0:a1]), [0, L], [0, a1 - a0], scale=0.08, causal=True,
                           window=333, q_pos_base=[0], k_pos_base=[a0], out=out, lse=lse, merge=True)
    sync()
    check_out(host(out), ro)
    check_lse(host(lse), rl)


def test_standalone_merge_matches_the_oracle():
    S, H, D = 300, 3, 128
    o1, o2 = gen(12, (S, H, D), (S, H, D))
    g = np.random.default_rng(0)
    l1 = g.standard_normal((H, S)) * 3
    l2 = g.standard_normal((H, S)) * 3
    l1[0, :7] = -np.inf
    l2[1, 3:9] = -np.inf
    l1[2, 5] = l2[2, 5] = -np.inf
    ro, rl, rw = A.update_out_and_lse(f64(o1), l1, f64(o2), l2)
    for bdt in (torch.bfloat16, torch.float32):
        out = torch.from_numpy(o1).cuda()
        lse = torch.from_numpy(l1.astype(np.float32)).cuda()
        bo = dev(o2) if bdt == torch.bfloat16 else torch.from_numpy(o2).cuda()
        _, _, w = cbv.attn_merge(out, lse, bo, torch.from_numpy(l2.astype(np.float32)).cuda(), return_weight=True)
        sync()
        check_out(host(out), ro, atol=1e-5)
        check_lse(host(lse), rl, atol=1e-5)
        np.testing.assert_allclose(host(w), rw, atol=1e-5)


@pytest.mark.parametrize("D,HKV", [(128, 2), (64, 1)])
def test_block_backward_accumulates_to_the_full_gradient(D, HKV):
    # two key blocks, each fed the MERGED out/lse, accumulate into the full gradients
    L, H = 520, 2
    q, k, v, do = gen(13, (L, H, D), (L, HKV, D), (L, HKV, D), (L, H, D))
    scale = 0.1
    ro, rl = A.attention_fwd(f64(q), f64(k), f64(v), [0, L], [0, L], scale, causal=True)
    out_b = dev(ro.astype(np.float32))
    rq, rk, rv = A.attention_bwd(f64(do), f64(q), f64(k), f64(v), host(out_b), rl, [0, L], [0, L], scale, causal=True)
    lse_d = torch.from_numpy(rl.astype(np.float32)).cuda()
    dq = torch.zeros((L, H, D), dtype=torch.float32, device="cuda")
    dk = torch.zeros((L, HKV, D), dtype=torch.float32, device="cuda")
    dv = torch.zeros((L, HKV, D), dtype=torch.float32, device="cuda")
    for a0, a1 in ((0, 300), (300, L)):
        kk, vv = dev(k[a0:a1]), dev(v[a0:a1])
        dk_b = torch.zeros((a1 - a0, HKV, D), dtype=torch.float32, device="cuda")
        dv_b = torch.zeros((a1 - a0, HKV, D), dtype=torch.float32, device="cuda")
        cbv.attn_block_bwd(dev(do), dev(q), kk, vv, out_b, lse_d, [0, L], [0, a1 - a0], scale=scale, causal=True,
                           q_pos_base=[0], k_pos_base=[a0], dq_acc=dq, dk_acc=dk_b, dv_acc=dv_b)
        sync()
        dk[a0:a1] += dk_b
        dv[a0:a1] += dv_b
    check_rel(host(dq), rq, what="dq")
    check_rel(host(dk), rk, what="dk")
    check_rel(host(dv), rv, what="dv")
