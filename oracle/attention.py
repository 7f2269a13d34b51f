"""Exact softmax attention in float64: forward, log-sum-exp, analytic backward, merge.

Test infrastructure only (see the package docstring).

Conventions (readings of the pages where they are silent or disagree):
  * q, out, dq are ``[S_q, H, D]``; k, v, dk, dv are ``[S_k, H_kv, D]`` (the
    FlashAttention varlen layout of the NeMo AutoModel zig-zag ring page,
    ``zigzag_ring_flash_attn_varlen_func``).  GQA maps q head ``h`` to kv head
    ``h // (H / H_kv)`` (qsa_fa_fallback.py, ``_varlen_one_q_attn_kernel``).
  * lse is ``[H, S_q]`` float64, natural log (the ``[num_heads, seqlen]`` lse of
    ``get_half_lse`` on the zig-zag page).
  * A key j is visible from a query i when both lie in the same document and,
    with ``causal``, ``kpos_j <= qpos_i``; with ``window = W > 0`` also
    ``0 <= qpos_i - kpos_j < W`` (W keys including the query itself; the
    ``sliding_window`` integer of the NKI KV-parallel page, 0 = disabled).
  * A query with no visible key has out = 0 and lse = -inf (the
    ``acc / (l > 0 ? l : 1)`` rule of qsa_fa_fallback.py).
"""
from __future__ import annotations

import numpy as np

NEG_INF = -np.inf


# --------------------------------------------------------------------------- masks

def doc_ids(cu_seqlens, n: int) -> np.ndarray:
    """Document index of every packed row ``0..n-1`` given cu_seqlens."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    ids = np.searchsorted(cu, np.arange(n), side="right") - 1
    return ids


def default_positions(cu_q, cu_k):
    """Per-row positions for a varlen block without explicit positions.

    Keys count from 0 inside their document; queries are aligned to the bottom
    right, ``qpos = i - cu_q[d] + (L_k[d] - L_q[d])`` (the FlashAttention >= 2.1
    convention for ``len_q != len_k``; the pages do not state one).
    """
    cu_q = np.asarray(cu_q, np.int64)
    cu_k = np.asarray(cu_k, np.int64)
    nq, nk = int(cu_q[-1]), int(cu_k[-1])
    dq = doc_ids(cu_q, nq)
    dk = doc_ids(cu_k, nk)
    lq = np.diff(cu_q)
    lk = np.diff(cu_k)
    qpos = np.arange(nq) - cu_q[dq] + (lk[dq] - lq[dq])
    kpos = np.arange(nk) - cu_k[dk]
    return qpos, kpos


def visible(qpos, kpos, qdoc, kdoc, causal: bool, window: int) -> np.ndarray:
    """Boolean ``[nq, nk]``: which keys each query may attend to."""
    qp = np.asarray(qpos, np.int64)[:, None]
    kp = np.asarray(kpos, np.int64)[None, :]
    m = np.asarray(qdoc)[:, None] == np.asarray(kdoc)[None, :]
    if causal:
        m = m & (kp <= qp)
    if window > 0:
        d = qp - kp
        m = m & (d >= 0) & (d < window)
    return m


# --------------------------------------------------------------------------- one head

def _softmax_rows(q, k, v, mask, scale):
    """out, lse for one head: ``s = scale q k^T`` masked, ``lse = log sum exp s``, ``out = softmax(s) v``."""
    s = scale * (q @ k.T)
    s = np.where(mask, s, NEG_INF)
    any_vis = mask.any(axis=1)
    mx = np.where(any_vis, s.max(axis=1, initial=NEG_INF), 0.0)
    e = np.where(mask, np.exp(s - mx[:, None]), 0.0)
    tot = e.sum(axis=1)
    lse = np.where(any_vis, mx + np.log(np.where(any_vis, tot, 1.0)), NEG_INF)
    p = np.where(mask, np.exp(s - np.where(any_vis, lse, 0.0)[:, None]), 0.0)
    out = p @ v
    return out, lse


def _kv_head(h: int, hq: int, hkv: int) -> int:
    if hq % hkv:
        raise ValueError("number of q heads must be a multiple of kv heads")
    return h // (hq // hkv)


# --------------------------------------------------------------------------- forward

def attention_fwd(q, k, v, cu_q, cu_k, scale, causal=True, window=0, qpos=None, kpos=None, rows=None):
    """Varlen attention ``(out [S_q,H,D], lse [H,S_q])`` of one block, in float64.

    This is the operation one flash varlen block returns (NeMo AutoModel,
    zigzag_ring_attention, ``_block_forward``; ring_attention, ``_fa_forward``
    returning ``(out[B,S,H,D], lse[B,H,S])``), written as its plain definition.

    ``qpos``/``kpos`` give every row's position for the mask (default:
    :func:`default_positions`).  ``rows`` restricts the computation to a subset
    of query rows (the others come back as out=0, lse=-inf); each row's
    softmax is independent, so this is the same definition evaluated on fewer
    rows.
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    nq, hq, d = q.shape
    nk, hkv, _ = k.shape
    if qpos is None or kpos is None:
        dq_, dk_ = default_positions(cu_q, cu_k)
        qpos = dq_ if qpos is None else qpos
        kpos = dk_ if kpos is None else kpos
    qdoc = doc_ids(cu_q, nq)
    kdoc = doc_ids(cu_k, nk)
    out = np.zeros((nq, hq, v.shape[2]), np.float64)
    lse = np.full((hq, nq), NEG_INF, np.float64)
    sel = np.arange(nq) if rows is None else np.asarray(rows, np.int64)
    cu_k = np.asarray(cu_k, np.int64)
    for doc in np.unique(qdoc[sel]) if len(sel) else []:
        qi = sel[qdoc[sel] == doc]
        if doc >= len(cu_k) - 1:
            continue
        kj = np.arange(cu_k[doc], cu_k[doc + 1])
        for c0 in range(0, len(qi), 1024):
            qc = qi[c0:c0 + 1024]
            mask = visible(np.asarray(qpos)[qc], np.asarray(kpos)[kj], qdoc[qc], kdoc[kj], causal, window)
            for h in range(hq):
                kh = _kv_head(h, hq, hkv)
                o, l = _softmax_rows(q[qc, h], k[kj, kh], v[kj, kh], mask, scale)
                out[qc, h] = o
                lse[h, qc] = l
    return out, lse


def attention_fwd_masked(q, k, v, mask, scale):
    """``(out, lse)`` for an explicit boolean visibility matrix shared by all heads."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    nq, hq, _ = q.shape
    hkv = k.shape[1]
    out = np.zeros((nq, hq, v.shape[2]), np.float64)
    lse = np.full((hq, nq), NEG_INF, np.float64)
    for h in range(hq):
        kh = _kv_head(h, hq, hkv)
        o, l = _softmax_rows(q[:, h], k[:, kh], v[:, kh], mask, scale)
        out[:, h] = o
        lse[h] = l
    return out, lse


# --------------------------------------------------------------------------- backward

def attention_bwd(dout, q, k, v, out, lse, cu_q, cu_k, scale, causal=True, window=0, qpos=None, kpos=None):
    """Analytic gradients ``(dq, dk, dv)`` of one block given the softmax statistics to use.

    The block backward of the zig-zag ring page (``_block_backward``,
    ``zigzag_ring_flash_attn_varlen_backward``): each block is fed the FINAL
    merged ``out`` and ``lse``, so that ``P = exp(scale q k^T - lse)`` is the
    block's slice of the joint softmax and no separate merge backward is
    needed.  With ``dO`` the upstream gradient:

        dV = P^T dO,   dP = dO V^T,   Delta_i = <dO_i, out_i>,
        dS = P * (dP - Delta),   dQ = scale dS K,   dK = scale dS^T Q.

    GQA: dk/dv of a kv head sum the contributions of its q heads.
    """
    dout = np.asarray(dout, np.float64)
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    out = np.asarray(out, np.float64)
    lse = np.asarray(lse, np.float64)
    nq, hq, _ = q.shape
    nk, hkv, _ = k.shape
    if qpos is None or kpos is None:
        dq_, dk_ = default_positions(cu_q, cu_k)
        qpos = dq_ if qpos is None else qpos
        kpos = dk_ if kpos is None else kpos
    qdoc = doc_ids(cu_q, nq)
    kdoc = doc_ids(cu_k, nk)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    cu_q = np.asarray(cu_q, np.int64)
    cu_k = np.asarray(cu_k, np.int64)
    for doc in range(min(len(cu_q), len(cu_k)) - 1):
        qi = np.arange(cu_q[doc], cu_q[doc + 1])
        kj = np.arange(cu_k[doc], cu_k[doc + 1])
        if len(qi) == 0 or len(kj) == 0:
            continue
        mask = visible(np.asarray(qpos)[qi], np.asarray(kpos)[kj], qdoc[qi], kdoc[kj], causal, window)
        for h in range(hq):
            kh = _kv_head(h, hq, hkv)
            qh, kk, vv = q[qi, h], k[kj, kh], v[kj, kh]
            do, o, l = dout[qi, h], out[qi, h], lse[h, qi]
            s = scale * (qh @ kk.T)
            fin = np.isfinite(l)
            p = np.where(mask & fin[:, None], np.exp(np.where(mask, s, 0.0) - np.where(fin, l, 0.0)[:, None]), 0.0)
            dv[kj, kh] += p.T @ do
            dp = do @ vv.T
            delta = (do * o).sum(axis=1)
            ds = p * (dp - delta[:, None])
            dq[qi, h] += scale * (ds @ kk)
            dk[kj, kh] += scale * (ds.T @ qh)
    return dq, dk, dv


# --------------------------------------------------------------------------- merge

def _sigmoid(x):
    x = np.asarray(x, np.float64)
    out = np.empty_like(x)
    pos = x >= 0
    out[pos] = 1.0 / (1.0 + np.exp(-x[pos]))
    ex = np.exp(x[~pos])
    out[~pos] = ex / (1.0 + ex)
    return out


def _logsigmoid(x):
    x = np.asarray(x, np.float64)
    out = np.empty_like(x)
    pos = x >= 0
    out[pos] = -np.log1p(np.exp(-x[pos]))
    out[~pos] = x[~pos] - np.log1p(np.exp(x[~pos]))
    return out


def update_out_and_lse(out, lse, block_out, block_lse):
    """Online-softmax merge of one block's ``(block_out, block_lse)`` into ``(out, lse)``.

    NeMo AutoModel, zigzag_ring_attention, ``update_out_and_lse``, and
    ring_attention, ``_update_out_and_lse`` (the numerically stable sigmoid
    form): with ``w = sigmoid(block_lse - lse)``

        out' = out - w * (out - block_out),   lse' = lse - logsigmoid(lse - block_lse).

    Also returns ``w`` computed from the running lse before the merge (the
    zig-zag page's extra return).  ``out``/``block_out`` are ``[S,H,D]``,
    ``lse``/``block_lse`` are ``[H,S]``.  A side at ``-inf`` (no visible key yet)
    is the identity of the merge: the other side is taken as it is.
    """
    out = np.asarray(out, np.float64)
    lse = np.asarray(lse, np.float64)
    block_out = np.asarray(block_out, np.float64)
    block_lse = np.asarray(block_lse, np.float64)
    a_inf = np.isneginf(lse)
    b_inf = np.isneginf(block_lse)
    both = ~a_inf & ~b_inf
    with np.errstate(invalid="ignore"):
        diff = np.where(both, block_lse - lse, 0.0)
    w = np.where(both, _sigmoid(diff), np.where(a_inf & ~b_inf, 1.0, 0.0))
    new_lse = np.where(both, lse - _logsigmoid(-diff), np.where(a_inf, block_lse, lse))
    wt = w.T[:, :, None]  # [S,H,1]
    new_out = out - wt * (out - block_out)
    return new_out, new_lse, w


# --------------------------------------------------------------------------- brute force

def brute_force_attention(q, k, v, qpos, kpos, qdoc, kdoc, scale, causal, window):
    """Scalar triple loop, for tiny inputs only (pins :func:`attention_fwd`)."""
    nq, hq, d = len(q), len(q[0]), len(q[0][0])
    nk, hkv = len(k), len(k[0])
    dv = len(v[0][0])
    out = [[[0.0] * dv for _ in range(hq)] for _ in range(nq)]
    lse = [[float("-inf")] * nq for _ in range(hq)]
    import math

    for i in range(nq):
        for h in range(hq):
            kh = h // (hq // hkv)
            scores = []
            for j in range(nk):
                ok = qdoc[i] == kdoc[j]
                if causal and not kpos[j] <= qpos[i]:
                    ok = False
                if window > 0 and not (0 <= qpos[i] - kpos[j] < window):
                    ok = False
                if ok:
                    s = 0.0
                    for t in range(d):
                        s += float(q[i][h][t]) * float(k[j][kh][t])
                    scores.append((j, scale * s))
            if not scores:
                continue
            m = max(s for _, s in scores)
            tot = sum(math.exp(s - m) for _, s in scores)
            lse[h][i] = m + math.log(tot)
            for j, s in scores:
                p = math.exp(s - lse[h][i])
                for t in range(dv):
                    out[i][h][t] += p * float(v[j][kh][t])
    return np.asarray(out), np.asarray(lse)


# --------------------------------------------------------------------------- subsets (large inputs)

def _row_stats(q, k, v, qpos, kpos, qdoc, kdoc, i, h, kh, scale, causal, window, lse_i):
    """Visible key indices, P row and scores of one query row against all keys."""
    m = visible(qpos[i:i + 1], kpos, qdoc[i:i + 1], kdoc, causal, window)[0]
    j = np.nonzero(m)[0]
    s = scale * (k[j, kh] @ q[i, h])
    p = np.exp(s - lse_i) if np.isfinite(lse_i) else np.zeros_like(s)
    return j, p


def attention_grad_rows(dout, q, k, v, out, lse, cu_q, cu_k, scale, rows, heads, causal=True, window=0,
                        qpos=None, kpos=None):
    """``dq`` of the given query rows and heads (``[len(rows), len(heads), D]``).

    The same definition as :func:`attention_bwd`, evaluated row by row:
    ``dq_i = scale * sum_j P_ij (<dO_i, v_j> - Delta_i) k_j`` with
    ``P_ij = exp(scale <q_i, k_j> - lse_i)`` and ``Delta_i = <dO_i, out_i>``.
    ``out`` and ``lse`` are needed only at the given rows.
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    nq, hq, d = q.shape
    nk, hkv, _ = k.shape
    if qpos is None or kpos is None:
        dq_, dk_ = default_positions(cu_q, cu_k)
        qpos = dq_ if qpos is None else qpos
        kpos = dk_ if kpos is None else kpos
    qdoc, kdoc = doc_ids(cu_q, nq), doc_ids(cu_k, nk)
    res = np.zeros((len(rows), len(heads), d))
    for a, i in enumerate(rows):
        for b, h in enumerate(heads):
            kh = _kv_head(h, hq, hkv)
            do = np.asarray(dout[i, h], np.float64)
            j, p = _row_stats(q, k, v, np.asarray(qpos), np.asarray(kpos), qdoc, kdoc, i, h, kh, scale, causal,
                              window, float(lse[h, i]))
            delta = float(do @ np.asarray(out[i, h], np.float64))
            ds = p * (v[j, kh] @ do - delta)
            res[a, b] = scale * (ds @ k[j, kh])
    return res


def attention_grad_cols(dout, q, k, v, out, lse, cu_q, cu_k, scale, cols, heads, causal=True, window=0,
                        qpos=None, kpos=None):
    """``(dk, dv)`` of the given key rows for the given q heads' contributions.

    ``dv_j = sum_i P_ij dO_i`` and ``dk_j = scale * sum_i P_ij (<dO_i, v_j> - Delta_i) q_i``
    over every query row i that sees key j; ``out``/``lse`` must be exact at those rows.
    Returns arrays ``[len(cols), len(heads), D]`` (one entry per q head; a kv head's
    gradient is the sum over its q heads).
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    nq, hq, d = q.shape
    nk, hkv, _ = k.shape
    if qpos is None or kpos is None:
        dq_, dk_ = default_positions(cu_q, cu_k)
        qpos = dq_ if qpos is None else qpos
        kpos = dk_ if kpos is None else kpos
    qpos, kpos = np.asarray(qpos), np.asarray(kpos)
    qdoc, kdoc = doc_ids(cu_q, nq), doc_ids(cu_k, nk)
    dk = np.zeros((len(cols), len(heads), d))
    dv = np.zeros((len(cols), len(heads), d))
    for a, j in enumerate(cols):
        m = visible(qpos, kpos[j:j + 1], qdoc, kdoc[j:j + 1], causal, window)[:, 0]
        i = np.nonzero(m)[0]
        for b, h in enumerate(heads):
            kh = _kv_head(h, hq, hkv)
            l = np.asarray(lse[h, i], np.float64)
            fin = np.isfinite(l)
            s = scale * (q[i, h] @ k[j, kh])
            p = np.where(fin, np.exp(s - np.where(fin, l, 0.0)), 0.0)
            do = np.asarray(dout[i, h], np.float64)
            delta = (do * np.asarray(out[i, h], np.float64)).sum(axis=1)
            ds = p * (do @ v[j, kh] - delta)
            dv[a, b] = p @ do
            dk[a, b] = scale * (ds @ q[i, h])
    return dk, dv
