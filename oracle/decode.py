"""One-query-per-sequence GQA varlen decode, in float64.

Test infrastructure only (see the package docstring).

qsa_fa_fallback.py (SM121 recipe), ``_varlen_one_q_attn_kernel`` and
``triton_varlen_attn_func``: sequence ``s`` has one query row ``cu_seqlens_q[s]``
and keys ``[cu_seqlens_k[s], cu_seqlens_k[s+1])``; q head ``h`` reads kv head
``h // (HQ / HKV)``; no mask applies; an empty key range gives a zero output.
The result is written at row ``cu_seqlens_q[s]``.
"""
from __future__ import annotations

import numpy as np


def varlen_decode(q, k, v, cu_q, cu_k, scale, seqs=None):
    """``out [total_q, HQ, D]``; only the sequences in ``seqs`` (default: all) are computed."""
    q = np.asarray(q)
    k = np.asarray(k)
    v = np.asarray(v)
    nq, hq, d = q.shape
    hkv = k.shape[1]
    if hq % hkv:
        raise ValueError("GQA mismatch")
    g = hq // hkv
    out = np.zeros((nq, hq, v.shape[2]), np.float64)
    cu_q = np.asarray(cu_q, np.int64)
    cu_k = np.asarray(cu_k, np.int64)
    n = len(cu_k) - 1
    for s in (range(n) if seqs is None else seqs):
        row = int(cu_q[s])
        a, b = int(cu_k[s]), int(cu_k[s + 1])
        if b <= a:
            continue
        for kh in range(hkv):
            kk = np.asarray(k[a:b, kh], np.float64)
            vv = np.asarray(v[a:b, kh], np.float64)
            qq = np.asarray(q[row, kh * g:(kh + 1) * g], np.float64)  # [g, D]
            sc = scale * (qq @ kk.T)
            m = sc.max(axis=1, keepdims=True)
            e = np.exp(sc - m)
            out[row, kh * g:(kh + 1) * g] = (e @ vv) / e.sum(axis=1, keepdims=True)
    return out
