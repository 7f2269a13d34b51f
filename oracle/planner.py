"""Context-parallel layouts over virtual ranks: integer, exact.

Test infrastructure only (see the package docstring).

From the NeMo AutoModel zig-zag ring page (module docstring, ``get_half_index``,
``get_half_lse``, ``_block_forward``): every document of the packed batch is cut
into ``2*cp`` equal chunks and virtual rank ``r`` owns chunk ``r`` (early) and
chunk ``2*cp-1-r`` (late).  A rank's local sequence is its chunks in document
order, front chunk before back chunk, so its local ``cu_seqlens`` is the global
one divided by ``cp``, and the front or back halves of the local documents use
the global one divided by ``2*cp``.

From the ring_attention page (module docstring): a contiguous layout gives rank
``r`` one contiguous piece of every document (here: the ``r``-th of ``cp`` equal
pieces), so its local ``cu_seqlens`` is also the global one divided by ``cp``.
"""
from __future__ import annotations

import numpy as np

ZIGZAG = "zigzag"
CONTIGUOUS = "contiguous"


def _cu(cu):
    return np.asarray(cu, dtype=np.int64)


def check_divisible(cu_global, cp: int, layout: str = ZIGZAG) -> None:
    """Every document length must split into ``2*cp`` (zig-zag) or ``cp`` (contiguous) equal chunks."""
    lengths = np.diff(_cu(cu_global))
    n = 2 * cp if layout == ZIGZAG else cp
    if np.any(lengths % n):
        raise ValueError(f"every document length must be divisible by {n}")


def local_cu_seqlens(cu_global, cp: int) -> np.ndarray:
    """Local cu_seqlens of every virtual rank: ``G / cp`` (int32)."""
    return (_cu(cu_global) // cp).astype(np.int32)


def half_cu_seqlens(cu_global, cp: int) -> np.ndarray:
    """cu_seqlens of the front or back halves of the local documents: ``G / (2 cp)`` (int32)."""
    return (_cu(cu_global) // (2 * cp)).astype(np.int32)


def get_half_index(cu_local, front: bool) -> np.ndarray:
    """Ascending local positions of the front (early) or back (late) half of each local document (int32)."""
    cu = _cu(cu_local)
    parts = []
    for d in range(len(cu) - 1):
        a, b = int(cu[d]), int(cu[d + 1])
        mid = a + (b - a) // 2
        parts.append(np.arange(a, mid) if front else np.arange(mid, b))
    return (np.concatenate(parts) if parts else np.zeros(0)).astype(np.int32)


def get_half_lse(lse, cu_local, front: bool) -> np.ndarray:
    """Front or back half of a ``[num_heads, seqlen]`` lse, document by document."""
    return np.asarray(lse)[:, get_half_index(cu_local, front)]


def rank_tokens(cu_global, cp: int, r: int, layout: str = ZIGZAG) -> np.ndarray:
    """Global row of every local token of virtual rank ``r``, in local order (int64)."""
    cu = _cu(cu_global)
    parts = []
    for d in range(len(cu) - 1):
        g, L = int(cu[d]), int(cu[d + 1] - cu[d])
        if layout == ZIGZAG:
            c = L // (2 * cp)
            parts.append(np.arange(g + r * c, g + (r + 1) * c))
            parts.append(np.arange(g + (2 * cp - 1 - r) * c, g + (2 * cp - r) * c))
        else:
            c = L // cp
            parts.append(np.arange(g + r * c, g + (r + 1) * c))
    return np.concatenate(parts).astype(np.int64) if parts else np.zeros(0, np.int64)


def zigzag_step(r: int, s: int, cp: int) -> tuple[int, str]:
    """Source rank and block kind of virtual rank ``r`` at ring step ``s``.

    The K/V that reach rank ``r`` at step ``s`` come from ``src = (r - s) mod cp``.
    ``"diag"``: step 0, local q against local k, causal.  ``"front_k"``: src < r,
    all local q against src's front halves (all visible, non-causal).
    ``"back_q"``: src > r, the back halves of local q against all of src's
    k/v (all visible, non-causal).  This is the plainest reading of the
    zig-zag page's ``_block_forward`` ("front/back half uses the halved
    cu_seqlens") given which chunks precede which.
    """
    src = (r - s) % cp
    if s == 0:
        return src, "diag"
    return src, ("front_k" if src < r else "back_q")


def contiguous_step(r: int, s: int, cp: int) -> tuple[int, str]:
    """Source rank and block kind for the contiguous ring (ring_attention page).

    A rank attends only to blocks from itself and earlier ranks (``step <= rank``)
    and applies the causal mask only at ``step == 0``; later steps are ``"skip"``.
    """
    src = (r - s) % cp
    if s == 0:
        return src, "diag"
    return src, ("full" if s <= r else "skip")


def visible_count_per_query(cu_global, window: int = 0) -> np.ndarray:
    """Number of keys each global query row sees under causal (+ window) masking."""
    cu = _cu(cu_global)
    n = int(cu[-1])
    counts = np.zeros(n, np.int64)
    for d in range(len(cu) - 1):
        a, b = int(cu[d]), int(cu[d + 1])
        c = np.arange(1, b - a + 1)
        if window > 0:
            c = np.minimum(c, window)
        counts[a:b] = c
    return counts


def rank_pair_counts(cu_global, cp: int, layout: str = ZIGZAG, window: int = 0) -> np.ndarray:
    """Visible (q, k) pairs per virtual rank: the causal work each rank does (int64 [cp])."""
    per_q = visible_count_per_query(cu_global, window)
    return np.array([int(per_q[rank_tokens(cu_global, cp, r, layout)].sum()) for r in range(cp)], np.int64)
