"""EAGLE-3 cached attention: the causal sequence block plus per-position cache diagonals, in float64.

Test infrastructure only (see the package docstring).

NeMo AutoModel, ring_attention, ``_CachedRingAttention`` and
``_CachedZigZagRingAttention``: the cache holds ``num_blocks`` blocks of keys and
values, ``cache_k[i]`` / ``cache_v[i]`` of shape ``[T, H_kv, D]`` (the pages'
``[B, num_blocks, T, H, D]`` with B = 1, block axis first).  A query at position t
sees one joint softmax over

  * block 0, the sequence: every key of its own document at a position <= t
    (causal; with a sliding window W also within W positions), score
    ``scale <q_t, k_0[j]>``, value ``v_0[j]``;
  * every later block i >= 1, one key each: the cache entry at the same position,
    score ``scale <q_t, k_i[t]>`` ("per-position diagonal"), value ``v_i[t]``.

:func:`cached_fwd` writes that joint softmax out as its plain definition.
:func:`cached_fwd_blockwise` takes the method's steps instead: block 0 through the
ring, then each diagonal merged in by :func:`oracle.attention.update_out_and_lse`.
:func:`cached_bwd` gives the analytic gradients of the joint softmax: for every key
``P = exp(s - lse)`` of the merged lse, ``dS = P (dP - Delta)`` with
``Delta_t = <dO_t, out_t>``; block 0's part is the ordinary block backward fed the
merged out and lse, and the diagonal parts are the same formulas on one key per row.

GQA: q head h reads kv head ``h // (H / H_kv)`` in every block; gradients of a kv head
sum over its q heads.
"""
from __future__ import annotations

import numpy as np

from . import planner
from .attention import NEG_INF, _kv_head, default_positions, doc_ids, update_out_and_lse, visible
from .ring import ring_fwd


def _f64(x):
    return np.asarray(x, np.float64)


def _diag_scores(q, ck, scale):
    """``[NB-1, H, T]`` scores ``scale <q_t, k_i[t]>`` of the diagonal blocks i >= 1."""
    T, H, _ = q.shape
    nb, _, hkv, _ = ck.shape
    s = np.zeros((nb - 1, H, T))
    for i in range(1, nb):
        for h in range(H):
            s[i - 1, h] = scale * (q[:, h] * ck[i, :, _kv_head(h, H, hkv)]).sum(axis=1)
    return s


def cached_fwd(q, cache_k, cache_v, cu, scale, window=0):
    """``(out [T,H,D], lse [H,T])`` of the joint softmax over block 0 and the diagonals."""
    q, ck, cv = _f64(q), _f64(cache_k), _f64(cache_v)
    T, H, D = q.shape
    nb, _, hkv, _ = ck.shape
    pos, _ = default_positions(cu, cu)
    doc = doc_ids(cu, T)
    sd = _diag_scores(q, ck, scale)
    out = np.zeros((T, H, cv.shape[3]))
    lse = np.full((H, T), NEG_INF)
    cu = np.asarray(cu, np.int64)
    for d in range(len(cu) - 1):
        rows = np.arange(cu[d], cu[d + 1])
        if len(rows) == 0:
            continue
        mask = visible(pos[rows], pos[rows], doc[rows], doc[rows], True, window)
        for h in range(H):
            kh = _kv_head(h, H, hkv)
            s0 = np.where(mask, scale * (q[rows, h] @ ck[0, rows, kh].T), NEG_INF)  # [n, n]
            s = np.concatenate([s0, sd[:, h, rows].T], axis=1)                       # [n, n + NB - 1]
            mx = s.max(axis=1)
            e = np.exp(s - mx[:, None])
            z = e.sum(axis=1)
            p = e / z[:, None]
            n = len(rows)
            vals = p[:, :n] @ cv[0, rows, kh] + sum(p[:, n + i - 1, None] * cv[i, rows, kh] for i in range(1, nb))
            out[rows, h] = vals
            lse[h, rows] = mx + np.log(z)
    return out, lse


def cached_fwd_blockwise(q, cache_k, cache_v, cu, cp, scale, window=0, layout=planner.ZIGZAG, order=None):
    """The method's steps: block 0 by the ring over ``cp`` virtual ranks, then each diagonal
    block merged into the running ``(out, lse)`` with the log-sum-exp identity (in ``order``)."""
    q, ck, cv = _f64(q), _f64(cache_k), _f64(cache_v)
    T, H, _ = q.shape
    nb, _, hkv, _ = ck.shape
    out, lse = ring_fwd(q, ck[0], cv[0], cu, cp, scale, window=window, layout=layout)
    sd = _diag_scores(q, ck, scale)
    for i in (range(1, nb) if order is None else order):
        bout = np.stack([cv[i, :, _kv_head(h, H, hkv)] for h in range(H)], axis=1)  # [T, H, D]
        out, lse, _ = update_out_and_lse(out, lse, bout, sd[i - 1])
    return out, lse


def cached_bwd(dout, q, cache_k, cache_v, out, lse, cu, scale, window=0):
    """``(dq [T,H,D], dcache_k [NB,T,H_kv,D], dcache_v [NB,T,H_kv,D])`` of the joint softmax."""
    dout, q, ck, cv, out, lse = (_f64(x) for x in (dout, q, cache_k, cache_v, out, lse))
    T, H, D = q.shape
    nb, _, hkv, _ = ck.shape
    pos, _ = default_positions(cu, cu)
    doc = doc_ids(cu, T)
    sd = _diag_scores(q, ck, scale)
    dq = np.zeros_like(q)
    dk = np.zeros_like(ck)
    dv = np.zeros_like(cv)
    cu = np.asarray(cu, np.int64)
    for d in range(len(cu) - 1):
        rows = np.arange(cu[d], cu[d + 1])
        if len(rows) == 0:
            continue
        mask = visible(pos[rows], pos[rows], doc[rows], doc[rows], True, window)
        for h in range(H):
            kh = _kv_head(h, H, hkv)
            qh, do, o, l = q[rows, h], dout[rows, h], out[rows, h], lse[h, rows]
            delta = (do * o).sum(axis=1)
            # block 0: the sequence keys
            k0, v0 = ck[0, rows, kh], cv[0, rows, kh]
            p0 = np.where(mask, np.exp(np.where(mask, scale * (qh @ k0.T), 0.0) - l[:, None]), 0.0)
            ds0 = p0 * (do @ v0.T - delta[:, None])
            dv[0, rows, kh] += p0.T @ do
            dq[rows, h] += scale * (ds0 @ k0)
            dk[0, rows, kh] += scale * (ds0.T @ qh)
            # blocks i >= 1: one key per row, at the row's own position
            for i in range(1, nb):
                ki, vi = ck[i, rows, kh], cv[i, rows, kh]
                pi = np.exp(sd[i - 1, h, rows] - l)
                dsi = pi * ((do * vi).sum(axis=1) - delta)
                dv[i, rows, kh] += pi[:, None] * do
                dq[rows, h] += scale * dsi[:, None] * ki
                dk[i, rows, kh] += scale * dsi[:, None] * qh
    return dq, dk, dv
