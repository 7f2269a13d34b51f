"""Context parallelism over real ranks (one process per GPU): the ring and Ulysses.

Ring (NeMo AutoModel zigzag_ring_attention: ``RingComm``,
``zigzag_ring_flash_attn_varlen_forward`` / ``_backward``; ring_attention for the
contiguous layout).  Every rank holds its LOCAL tokens (``rank_tokens``: for every
document its front chunk, then its back chunk).  At step ``s`` rank ``r`` holds the
k/v of ``src = (r - s) mod cp``, runs that step's block on the GPU
(``cbv_ring_step_fwd`` / ``_bwd``) and passes the k/v on to ``r + 1`` while it
computes.  The forward merges every block into a running fp32 (out, lse) with the
online-softmax identity; the backward feeds every block the MERGED out/lse and sends
the fp32 dK/dV accumulators along with the k/v they belong to, so after ``cp`` hops
they arrive back at their owner.

Ulysses (ulysses_attention: ``_gather_seq_scatter_heads``, ``_block0_forward``,
``_block0_backward``, ``_scatter_seq_gather_heads``, ``_gather_lse``,
``_scatter_lse``, ``cached_ulysses_attention``).  Every rank holds a contiguous
``S / P`` slice of the tokens with all heads; an all-to-all turns it into the full
sequence for ``H / P`` heads, block 0 runs causally over it (documents from the
GLOBAL ``cu_seqlens``), the result goes back by the inverse all-to-all, and the
per-position cache diagonals merge into it shard-locally.  The backward gathers
dout, q, k, v and the MERGED out/lse the same way and runs block 0's backward
against the merged statistics; the diagonals' gradients are closed-form and local.

KV-parallel prefill (NKI attention_kv_parallel_segmented_cte: every shard attends its own
paged KV, the shards' partial (out, lse) merge by the log-sum-exp identity).  Every rank
holds the pages of its own shards and the whole q; it computes its shards' partials
(``cbv_kvp_segmented_prefill`` with ``shard_base`` / ``total_shards``, so that key
positions follow the global shard index), the partials are all-gathered, and every rank
merges all of them in shard order.

Every arithmetic step runs in libcbv.so; torch.distributed moves the data (NCCL on
GPUs; with ``via_host=True`` the tensors travel through host memory, which lets a
gloo group carry the exchange).  No kernel of one rank ever waits on another rank.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import (KV_ROUND_ROBIN, attn_block_bwd, attn_block_fwd, attn_merge, cached_diag_grad, cached_diag_merge,
               convert_f32_bf16, kvp_segmented_prefill as _kvp_prefill, ring_step_bwd, ring_step_fwd,
               swap_leading_axes)


class RingComm:
    """P2P ring over a process group: send to ``rank + 1``, receive from ``rank - 1`` (group order).

    ``send_recv`` / ``send_recv_kv`` queue one send and one receive each, ``commit`` starts the
    queued operations, ``wait`` completes them (the receive buffers are then valid)."""

    def __init__(self, group=None, via_host: bool = False):
        self.group = group
        self.rank = dist.get_rank(group)
        self.world_size = dist.get_world_size(group)
        ranks = dist.get_process_group_ranks(group) if group is not None else list(range(self.world_size))
        self.send_to = ranks[(self.rank + 1) % self.world_size]
        self.recv_from = ranks[(self.rank - 1) % self.world_size]
        self.via_host = via_host
        self._ops = []
        self._reqs = []
        self._copy_back = []

    def send_recv(self, to_send: torch.Tensor, recv_tensor: torch.Tensor | None = None) -> torch.Tensor:
        recv = torch.empty_like(to_send) if recv_tensor is None else recv_tensor
        if self.via_host:
            send_buf = to_send.detach().to("cpu")
            recv_buf = torch.empty(recv.shape, dtype=recv.dtype)
            self._copy_back.append((recv_buf, recv))
        else:
            send_buf, recv_buf = to_send, recv
        self._ops.append(dist.P2POp(dist.isend, send_buf, self.send_to, self.group))
        self._ops.append(dist.P2POp(dist.irecv, recv_buf, self.recv_from, self.group))
        return recv

    def send_recv_kv(self, k, v, k_buffer=None, v_buffer=None):
        return self.send_recv(k, k_buffer), self.send_recv(v, v_buffer)

    def commit(self):
        if self._ops:
            self._reqs = dist.batch_isend_irecv(self._ops)
        self._ops = []

    def wait(self):
        for r in self._reqs:
            r.wait()
        self._reqs = []
        for host, dev in self._copy_back:
            dev.copy_(host, non_blocking=False)
        self._copy_back = []


def zigzag_ring_fwd(q, k, v, cu_seqlens, group=None, scale=None, window: int = 0, layout="zigzag",
                    via_host: bool = False, step_fwd=ring_step_fwd):
    """Ring forward over the ranks of ``group``: ``q`` / ``k`` / ``v`` are this rank's LOCAL
    ``[n_local, H(kv), D]`` bf16 tensors; returns ``(out bf16 [n_local, H, D], lse f32 [H, n_local])``.
    ``step_fwd`` is the per-step block (``ring_step_fwd``: the CUDA kernel)."""
    comm = RingComm(group, via_host)
    cp, r = comm.world_size, comm.rank
    n, H, D = q.shape
    out_acc = torch.empty((n, H, D), dtype=torch.float32, device=q.device)
    lse_acc = torch.empty((H, n), dtype=torch.float32, device=q.device)
    out = torch.empty_like(q)
    bufs = [(torch.empty_like(k), torch.empty_like(v)) for _ in range(2)]
    kc, vc = k, v
    for s in range(cp):
        if s + 1 < cp:
            nk, nv = comm.send_recv_kv(kc, vc, *bufs[s % 2])  # the next k/v travel while this block runs
            comm.commit()
        step_fwd(r, s, q, kc, vc, cu_seqlens, cp, out_acc, lse_acc, out=out if s == cp - 1 else None, scale=scale,
                 window=window, layout=layout)
        if s + 1 < cp:
            comm.wait()
            kc, vc = nk, nv
    return out, lse_acc


def zigzag_ring_bwd(dout, q, k, v, out, lse, cu_seqlens, group=None, scale=None, window: int = 0, layout="zigzag",
                    via_host: bool = False, step_bwd=ring_step_bwd, finish=convert_f32_bf16):
    """Ring backward fed this rank's merged ``(out, lse)``: returns this rank's ``(dq, dk, dv)`` (bf16,
    local rows).  The fp32 dk/dv accumulators travel with the k/v they belong to and are home after
    ``cp`` hops."""
    kv_comm, acc_comm = RingComm(group, via_host), RingComm(group, via_host)
    cp, r = kv_comm.world_size, kv_comm.rank
    n, H, D = q.shape
    f32 = dict(dtype=torch.float32, device=q.device)
    dq_acc = torch.zeros((n, H, D), **f32)
    dk_acc = torch.zeros(k.shape, **f32)
    dv_acc = torch.zeros(v.shape, **f32)
    kv_bufs = [(torch.empty_like(k), torch.empty_like(v)) for _ in range(2)]
    acc_bufs = [(torch.empty_like(dk_acc), torch.empty_like(dv_acc)) for _ in range(2)]
    kc, vc = k, v
    for s in range(cp):
        if s + 1 < cp:
            nk, nv = kv_comm.send_recv_kv(kc, vc, *kv_bufs[s % 2])
            kv_comm.commit()
        step_bwd(r, s, dout, q, kc, vc, out, lse, cu_seqlens, cp, dq_acc, dk_acc, dv_acc, scale=scale, window=window,
                 layout=layout)
        # the accumulators of src's k/v follow them to the next rank (after the last step: home)
        ndk, ndv = acc_comm.send_recv_kv(dk_acc, dv_acc, *acc_bufs[s % 2])
        acc_comm.commit()
        acc_comm.wait()
        dk_acc, dv_acc = ndk, ndv
        if s + 1 < cp:
            kv_comm.wait()
            kc, vc = nk, nv
    return finish(dq_acc), finish(dk_acc), finish(dv_acc)


# ----------------------------------------------------------------------------- Ulysses
class _AllToAll:
    """Equal-split all_to_all_single along dim 0 (ulysses_attention._all_to_all_single)."""

    def __init__(self, group=None, via_host: bool = False):
        self.group = group
        self.world_size = dist.get_world_size(group)
        self.via_host = via_host

    def __call__(self, x: torch.Tensor) -> torch.Tensor:
        if self.via_host:
            src = x.detach().to("cpu").contiguous()
            dst = torch.empty_like(src)
            dist.all_to_all_single(dst, src, group=self.group)
            return dst.to(x.device)
        dst = torch.empty_like(x)
        dist.all_to_all_single(dst, x.contiguous(), group=self.group)
        return dst


def gather_seq_scatter_heads(x, a2a: _AllToAll, swap=swap_leading_axes):
    """``[S_local, H, D]`` (this rank's tokens, all heads) -> ``[S_full, H / P, D]`` (all tokens, its heads)."""
    P = a2a.world_size
    S, H, D = x.shape
    send = swap(x.reshape(S, P, (H // P) * D))  # [P, S_local, H/P * D]: chunk j goes to rank j
    return a2a(send).reshape(P * S, H // P, D)


def scatter_seq_gather_heads(x, a2a: _AllToAll, swap=swap_leading_axes):
    """Inverse of :func:`gather_seq_scatter_heads`: ``[S_full, H / P, D]`` -> ``[S_local, H, D]``."""
    P = a2a.world_size
    S_full, Hl, D = x.shape
    recv = a2a(x.reshape(P, S_full // P, Hl * D))  # chunk i came from rank i: heads [i Hl, (i + 1) Hl)
    return swap(recv).reshape(S_full // P, P * Hl, D)


def gather_lse(lse, a2a: _AllToAll, swap=swap_leading_axes):
    """``[H, S_local]`` -> ``[H / P, S_full]`` (contiguous)."""
    P = a2a.world_size
    H, S = lse.shape
    recv = a2a(lse.reshape(P, H // P, S))
    return swap(recv).reshape(H // P, P * S)


def scatter_lse(lse, a2a: _AllToAll, swap=swap_leading_axes):
    """``[H / P, S_full]`` -> ``[H, S_local]``."""
    P = a2a.world_size
    Hl, S_full = lse.shape
    send = swap(lse.reshape(Hl, P, S_full // P))  # [P, H/P, S_local]
    return a2a(send).reshape(P * Hl, S_full // P)


def _cache_list(cache):
    return list(cache.unbind(0)) if isinstance(cache, torch.Tensor) else list(cache)


def ulysses_fwd(q, cache_k, cache_v, cu_seqlens, group=None, scale=None, via_host: bool = False, ops=None):
    """Ulysses attention (with EAGLE-3 cache diagonals when ``len(cache_k) > 1``): ``q`` is this rank's
    contiguous ``[S_local, H, D]`` slice, ``cache_k`` / ``cache_v`` lists of ``[S_local, Hkv, D]`` (index 0:
    the sequence keys/values).  ``cu_seqlens`` are GLOBAL.  Returns ``(out bf16, lse f32 [H, S_local])``."""
    ops = ops or _Ops()
    a2a = _AllToAll(group, via_host)
    ck, cv = _cache_list(cache_k), _cache_list(cache_v)
    q_g, k_g, v_g = (gather_seq_scatter_heads(x, a2a, ops.swap) for x in (q, ck[0], cv[0]))
    o_g, l_g = ops.block0_fwd(q_g, k_g, v_g, cu_seqlens, scale)  # normalised fp32 out, lse [H/P, S_full]
    o32 = scatter_seq_gather_heads(o_g, a2a, ops.swap)
    lse = scatter_lse(l_g, a2a, ops.swap).contiguous()
    return ops.diag_merge(q, ck, cv, o32, lse, scale)


def ulysses_bwd(dout, q, cache_k, cache_v, out, lse, cu_seqlens, group=None, scale=None, via_host: bool = False,
                ops=None):
    """Backward of :func:`ulysses_fwd` fed the merged ``(out, lse)``: ``(dq, dcache_k, dcache_v)`` with the
    cache gradients as lists (bf16, this rank's rows)."""
    ops = ops or _Ops()
    a2a = _AllToAll(group, via_host)
    ck, cv = _cache_list(cache_k), _cache_list(cache_v)
    dout_g, q_g, k_g, v_g, out_g = (gather_seq_scatter_heads(x, a2a, ops.swap) for x in (dout, q, ck[0], cv[0], out))
    lse_g = gather_lse(lse, a2a, ops.swap)
    dq_g, dk_g, dv_g = ops.block0_bwd(dout_g, q_g, k_g, v_g, out_g, lse_g, cu_seqlens, scale)  # fp32
    dq0, dk0, dv0 = (scatter_seq_gather_heads(x, a2a, ops.swap) for x in (dq_g, dk_g, dv_g))
    dq, dck, dcv = ops.diag_grad(dout, q, ck, cv, out, lse, dq0, scale)
    dck[0], dcv[0] = ops.finish(dk0), ops.finish(dv0)
    return dq, dck, dcv


class _Ops:
    """The compute steps of Ulysses, each one libcbv.so call."""

    @staticmethod
    def swap(x):
        return swap_leading_axes(x)

    @staticmethod
    def block0_fwd(q, k, v, cu, scale):
        return attn_block_fwd(q, k, v, cu, cu, scale=scale, causal=True, out_dtype=torch.float32)

    @staticmethod
    def block0_bwd(dout, q, k, v, out, lse, cu, scale):
        return attn_block_bwd(dout, q, k, v, out, lse, cu, cu, scale=scale, causal=True)

    @staticmethod
    def diag_merge(q, ck, cv, o32, lse, scale):
        return cached_diag_merge(q, ck, cv, o32, lse, scale=scale)

    @staticmethod
    def diag_grad(dout, q, ck, cv, out, lse, dq0, scale):
        return cached_diag_grad(dout, q, ck, cv, out, lse, dq0, scale=scale)

    @staticmethod
    def finish(x):
        return convert_f32_bf16(x)


# ----------------------------------------------------------------------------- KV-parallel prefill
def _all_gather(x: torch.Tensor, group, via_host: bool) -> list[torch.Tensor]:
    world = dist.get_world_size(group)
    src = x.detach().to("cpu") if via_host else x.contiguous()
    parts = [torch.empty_like(src) for _ in range(world)]
    dist.all_gather(parts, src, group=group)
    return [t.to(x.device) for t in parts] if via_host else parts


def kvp_segmented_prefill(q, k_cache, v_cache, block_tables, kv_mode=KV_ROUND_ROBIN, seg_size: int = 512,
                          scale=None, global_q_offset: int = 0, sliding_window: int = 0, group=None,
                          via_host: bool = False, partial=None, merge=attn_merge, finish=convert_f32_bf16):
    """KV-parallel prefill with the shards on the ranks of ``group``.  Rank r holds the pages of shards
    ``r*n .. r*n + n - 1`` (``block_tables`` ``[n, blocks]`` into its own page pool ``k_cache`` /
    ``v_cache``; ``n`` the same on every rank) and the whole ``q [HQ, S, D]``.  Returns the same
    ``(out bf16 [HQ, S, D], lse f32 [HQ, S])`` on every rank.  ``partial(shard_base, total_shards)``
    computes this rank's ``(shard_out f32 [n, HQ, S, D], shard_lse f32 [n, HQ, S])`` (default: the
    paged prefill kernel); ``merge`` is the online-softmax merge (default: ``attn_merge``)."""
    world, r = dist.get_world_size(group), dist.get_rank(group)
    n = block_tables.shape[0]
    HQ, S, D = q.shape
    if partial is None:
        def partial(shard_base, total_shards):
            res = _kvp_prefill(q, k_cache, v_cache, block_tables, kv_mode, seg_size, scale, global_q_offset,
                               sliding_window, per_shard=True, return_lse=False, shard_base=shard_base,
                               total_shards=total_shards)
            return res[1], res[2]
    so, sl = partial(r * n, world * n)
    outs = torch.cat(_all_gather(so, group, via_host))  # [world * n, HQ, S, D], in global shard order
    lses = torch.cat(_all_gather(sl, group, via_host))
    out, lse = outs[0].clone(), lses[0].clone()
    # one (row, head) pair per merge row: [HQ * S, 1, D] outputs, [1, HQ * S] lse
    for i in range(1, outs.shape[0]):
        merge(out.view(HQ * S, 1, D), lse.view(1, HQ * S), outs[i].view(HQ * S, 1, D), lses[i].view(1, HQ * S))
    return finish(out), lse
