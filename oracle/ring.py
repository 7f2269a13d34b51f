"""Ring context-parallel attention over virtual ranks, block by block, in float64.

Test infrastructure only (see the package docstring).

Every virtual rank keeps its local q and a running ``(out, lse)``; at ring step
``s`` it holds the k/v of ``src = (r - s) mod cp`` and runs one attention block,
merging its ``(block_out, block_lse)`` into the running pair with
:func:`oracle.attention.update_out_and_lse` (NeMo AutoModel,
zigzag_ring_attention, ``zigzag_ring_flash_attn_varlen_forward``: rotate K/V,
per-block flash, online-softmax merge).  The backward runs the same blocks,
each fed the FINAL merged out and lse (``zigzag_ring_flash_attn_varlen_backward``,
the merged-lse identity), and adds every block's dq to the local rows and its
dk/dv to the rows of the rank that owns those k/v.

Masks use the tokens' global positions, so a sliding window means the same
thing in every block.
"""
from __future__ import annotations

import numpy as np

from . import planner
from .attention import NEG_INF, attention_bwd, attention_fwd, update_out_and_lse


def _block_rows(cu_global, cp, r, s, layout):
    """(local q rows, src-local k rows, causal, q cu, k cu, src) of rank r's block at step s, or None."""
    cu_loc = planner.local_cu_seqlens(cu_global, cp)
    n_loc = int(cu_loc[-1])
    if layout == planner.ZIGZAG:
        src, kind = planner.zigzag_step(r, s, cp)
        cu_half = planner.half_cu_seqlens(cu_global, cp)
        if kind == "diag":
            return np.arange(n_loc), np.arange(n_loc), True, cu_loc, cu_loc, src
        if kind == "front_k":
            return np.arange(n_loc), planner.get_half_index(cu_loc, True), False, cu_loc, cu_half, src
        return planner.get_half_index(cu_loc, False), np.arange(n_loc), False, cu_half, cu_loc, src
    src, kind = planner.contiguous_step(r, s, cp)
    if kind == "skip":
        return None
    return np.arange(n_loc), np.arange(n_loc), kind == "diag", cu_loc, cu_loc, src


def ring_fwd(q, k, v, cu_global, cp, scale, window=0, layout=planner.ZIGZAG, return_blocks=False):
    """``(out [S,H,D], lse [H,S])`` of the ring in natural order (inputs in natural order too)."""
    planner.check_divisible(cu_global, cp, layout)
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    S, H, D = q.shape
    out = np.zeros((S, H, v.shape[2]))
    lse = np.full((H, S), NEG_INF)
    blocks = []
    for r in range(cp):
        loc = planner.rank_tokens(cu_global, cp, r, layout)
        o_r = np.zeros((len(loc), H, v.shape[2]))
        l_r = np.full((H, len(loc)), NEG_INF)
        for s in range(cp):
            b = _block_rows(cu_global, cp, r, s, layout)
            if b is None:
                continue
            qi, kj, causal, cu_q, cu_k, src = b
            kv = planner.rank_tokens(cu_global, cp, src, layout)[kj]
            bo, bl = attention_fwd(q[loc[qi]], k[kv], v[kv], cu_q, cu_k, scale, causal=causal, window=window,
                                   qpos=loc[qi], kpos=kv)
            no, nl, _ = update_out_and_lse(o_r[qi], l_r[:, qi], bo, bl)
            o_r[qi] = no
            l_r[:, qi] = nl
            blocks.append((r, s, loc[qi], kv, causal))
        out[loc] = o_r
        lse[:, loc] = l_r
    if return_blocks:
        return out, lse, blocks
    return out, lse


def ring_bwd(dout, q, k, v, out, lse, cu_global, cp, scale, window=0, layout=planner.ZIGZAG, lse_mode="merged"):
    """``(dq, dk, dv)`` of the ring, natural order.

    ``lse_mode="merged"`` feeds every block the final merged out/lse (the pages'
    method).  ``lse_mode="block_local"`` instead feeds each block its OWN
    forward out/lse, the variant the zig-zag page says skews dq/dk; it exists
    only so a test can show that it is wrong.
    """
    dout = np.asarray(dout, np.float64)
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for r in range(cp):
        loc = planner.rank_tokens(cu_global, cp, r, layout)
        cu_loc = planner.local_cu_seqlens(cu_global, cp)
        for s in range(cp):
            b = _block_rows(cu_global, cp, r, s, layout)
            if b is None:
                continue
            qi, kj, causal, cu_q, cu_k, src = b
            kv = planner.rank_tokens(cu_global, cp, src, layout)[kj]
            rows = loc[qi]
            if lse_mode == "merged":
                # the merged lse of the selected rows: get_half_lse for back halves
                o_b = np.asarray(out)[rows]
                if len(qi) == len(loc):
                    l_b = np.asarray(lse)[:, rows]
                else:
                    l_b = planner.get_half_lse(np.asarray(lse)[:, loc], cu_loc, front=False)
            else:
                o_b, l_b = attention_fwd(q[rows], k[kv], v[kv], cu_q, cu_k, scale, causal=causal, window=window,
                                         qpos=rows, kpos=kv)
            gq, gk, gv = attention_bwd(dout[rows], q[rows], k[kv], v[kv], o_b, l_b, cu_q, cu_k, scale,
                                       causal=causal, window=window, qpos=rows, kpos=kv)
            dq[rows] += gq
            np.add.at(dk, kv, gk)
            np.add.at(dv, kv, gv)
    return dq, dk, dv
