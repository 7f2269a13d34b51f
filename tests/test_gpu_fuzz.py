"""Seeded random shapes against the fp64 oracle: ring forward and backward over random document
mixes, cp, layouts, GQA ratios, head dims and windows, the cached ring, and the deterministic flag;
standalone blocks with unequal q/k lengths and explicit positions, causal or not; the paged prefill
over random shard counts, page sizes, layouts, segment sizes and windows; and the decode.
The shapes are drawn so that chunk tails of every raggedness occur (single-tile forward tasks, key
tiles that share two ranges, empty documents)."""
import numpy as np
import pytest
import torch

import context_blockwise_causal_varlen_b200 as cbv
from oracle import attention as A
from oracle import cached as C
from oracle import decode as DEC
from oracle import paged as PG
from synth import block_permutation, cu_from_lengths, streams
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


def _positions(cu, base):
    """Every row's position: the document's base plus the row's offset in the document."""
    cu = np.asarray(cu, np.int64)
    pos = np.zeros(int(cu[-1]), np.int64)
    for d in range(len(cu) - 1):
        pos[cu[d]:cu[d + 1]] = base[d] + np.arange(cu[d + 1] - cu[d])
    return pos


@pytest.mark.parametrize("seed", range(8))
def test_random_block_matches_oracle(seed):
    rng = np.random.default_rng(2000 + seed)
    ndocs = int(rng.integers(1, 5))
    lq = [int(rng.integers(0, 400)) for _ in range(ndocs)]
    lk = [int(rng.integers(0, 500)) for _ in range(ndocs)]
    H, HKV = [(2, 1), (4, 2), (4, 4), (8, 2)][int(rng.integers(0, 4))]
    D = int(rng.choice([64, 128]))
    causal = bool(rng.random() < 0.75)
    window = int(rng.choice([0, 0, 1 + int(rng.integers(0, 300))])) if causal else 0
    explicit = bool(rng.random() < 0.5)
    cq, ck = cu_from_lengths(lq), cu_from_lengths(lk)
    kb = [int(rng.integers(0, 300)) for _ in range(ndocs)]
    qb = [kb[d] + int(rng.integers(-100, 400)) for d in range(ndocs)]
    kw = dict(q_pos_base=qb, k_pos_base=kb) if explicit else {}
    okw = dict(qpos=_positions(cq, qb), kpos=_positions(ck, kb)) if explicit else {}
    q, k, v, do = gen(90 + seed, (int(cq[-1]), H, D), (int(ck[-1]), HKV, D), (int(ck[-1]), HKV, D), (int(cq[-1]), H, D))
    out, lse = cbv.attn_block_fwd(dev(q), dev(k), dev(v), cq, ck, scale=0.1, causal=causal, window=window, **kw)
    sync()
    ro, rl = A.attention_fwd(f64(q), f64(k), f64(v), cq, ck, 0.1, causal=causal, window=window, **okw)
    check_out(host(out), ro)
    check_lse(host(lse), rl)
    dq, dk, dv = cbv.attn_block_bwd(dev(do), dev(q), dev(k), dev(v), out, lse, cq, ck, scale=0.1, causal=causal,
                                    window=window, **kw)
    sync()
    rq, rk, rv = A.attention_bwd(f64(do), f64(q), f64(k), f64(v), host(out), host(lse), cq, ck, 0.1, causal=causal,
                                 window=window, **okw)
    check_rel(host(dq), rq, what="dq")
    check_rel(host(dk), rk, what="dk")
    check_rel(host(dv), rv, what="dv")


@pytest.mark.parametrize("seed", range(8))
def test_random_paged_prefill_matches_oracle(seed):
    rng = np.random.default_rng(3000 + seed)
    R = int(rng.choice([1, 2, 4, 8]))
    bs = int(rng.choice([8, 16, 32, 64, 128]))
    bps = int(rng.integers(1, 1 + 2048 // (R * bs)))
    hq, hkv = [(4, 1), (8, 2), (4, 4), (12, 3)][int(rng.integers(0, 4))]
    D = int(rng.choice([64, 128]))
    mode = PG.ROUND_ROBIN if rng.random() < 0.6 else PG.CONTIGUOUS
    seg = int(rng.choice([128, 256, 512, 100, 300, 1]))  # any positive length (rounded up to whole key tiles)
    window = int(rng.choice([0, 0, 1 + int(rng.integers(0, 600))]))
    kv_len = R * bps * bs
    S = int(rng.integers(1, min(kv_len, 400) + 1))
    gqo = int(rng.integers(0, kv_len - S + 1))
    nb = R * bps
    q, kc, vc = gen(110 + seed, (hq, S, D), (nb, hkv, bs, D), (nb, hkv, bs, D))
    perm = block_permutation(streams(120 + seed, 1)[0], nb)
    bt = PG.shard_block_tables(perm, R, mode)
    K, V = PG.global_kv(f64(kc), f64(vc), bt, bs, mode)
    ro, rl = PG.prefill_full(f64(q), K, V, 0.1, gqo, window=window)
    kv_mode = cbv.KV_ROUND_ROBIN if mode == PG.ROUND_ROBIN else cbv.KV_CONTIGUOUS
    out, lse = cbv.kvp_segmented_prefill(dev(q), dev(kc), dev(vc), torch.from_numpy(bt), kv_mode=kv_mode, seg_size=seg,
                                         scale=0.1, global_q_offset=gqo, sliding_window=window)
    sync()
    check_out(host(out), ro)
    check_lse(host(lse), rl)


@pytest.mark.parametrize("seed", range(4))
def test_random_decode_matches_oracle(seed):
    rng = np.random.default_rng(4000 + seed)
    hq, hkv = [(32, 4), (16, 16), (8, 1), (24, 6)][seed]
    D = int(rng.choice([64, 128]))
    n = int(rng.integers(1, 300))
    lengths = rng.integers(0, 1500, n)
    cu_k = cu_from_lengths(lengths)
    q, k, v = gen(130 + seed, (n, hq, D), (int(cu_k[-1]), hkv, D), (int(cu_k[-1]), hkv, D))
    cu_q = np.arange(n + 1, dtype=np.int32)
    out = cbv.varlen_decode(dev(q), dev(k), dev(v), torch.from_numpy(cu_q), torch.from_numpy(cu_k), scale=0.1)
    sync()
    check_out(host(out), DEC.varlen_decode(f64(q), f64(k), f64(v), cu_q, cu_k, 0.1))
