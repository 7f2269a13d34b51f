"""Blockwise causal varlen attention on B200: Python binding of libcbv.so.

Argument marshalling only: every step of the computation runs in the library's
CUDA kernels (see ``include/cbv.h``).  PyTorch provides device memory and the
current stream.  The binding fails loudly when ``libcbv.so`` is missing; there is
no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# CBV_LIBRARY=debug selects the bounds-checking build (libcbv_debug.so): its kernels check every row
# and page index against its tensor, and every call below then also reads the status word back.
LIB_PATH = os.path.join(_HERE, "libcbv_debug.so" if os.environ.get("CBV_LIBRARY") == "debug" else "libcbv.so")
ABI_VERSION = 1

ZIGZAG, CONTIGUOUS = 0, 1
KV_CONTIGUOUS, KV_ROUND_ROBIN = 0, 1
SCHEDULE_FUSED, SCHEDULE_STEPWISE = 0, 1
DTYPE_BF16, DTYPE_F32 = 0, 1

STATUS = {
    0: "OK", -1: "BAD_ARG", -2: "BAD_SHAPE", -3: "BAD_DTYPE", -4: "MISALIGNED", -5: "UNSUPPORTED_HEAD_DIM",
    -6: "NOT_DIVISIBLE_2CP", -7: "NOT_CAUSAL", -8: "GQA_MISMATCH", -9: "BAD_CU_SEQLENS", -10: "Q_LEN_NOT_ONE",
    -11: "WORKSPACE_TOO_SMALL", -12: "TIMEOUT", -13: "CUDA", -14: "VERSION",
}


class CbvError(RuntimeError):
    def __init__(self, code: int, message: str):
        super().__init__(f"cbv error {STATUS.get(code, code)} ({code}): {message}")
        self.code = code
        self.status = STATUS.get(code, str(code))


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libcbv.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m context_blockwise_causal_varlen_b200.build`")
        _lib = ctypes.CDLL(LIB_PATH)
        _declare(_lib)
        if _lib.cbv_abi_version() != ABI_VERSION:
            raise ImportError("libcbv.so ABI version mismatch")
    return _lib


# ----------------------------------------------------------------------------- C structs
c_i32p = ctypes.POINTER(ctypes.c_int32)
c_i64p = ctypes.POINTER(ctypes.c_int64)
c_f32p = ctypes.POINTER(ctypes.c_float)


class BlockFwdArgs(ctypes.Structure):
    _fields_ = [
        ("struct_size", ctypes.c_uint32), ("abi_version", ctypes.c_uint32),
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("total_q", ctypes.c_int64), ("total_k", ctypes.c_int64),
        ("num_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("num_docs", ctypes.c_int32),
        ("cu_seqlens_q", c_i32p), ("cu_seqlens_k", c_i32p), ("q_pos_base", c_i32p), ("k_pos_base", c_i32p),
        ("max_seqlen", ctypes.c_int32), ("scale", ctypes.c_float), ("causal", ctypes.c_int32),
        ("window", ctypes.c_int32), ("merge", ctypes.c_int32), ("out_dtype", ctypes.c_int32),
        ("out", ctypes.c_void_p), ("lse", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
    ]


class RingArgs(ctypes.Structure):
    _fields_ = [
        ("struct_size", ctypes.c_uint32), ("abi_version", ctypes.c_uint32),
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("total", ctypes.c_int64),
        ("num_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("num_docs", ctypes.c_int32), ("cu_seqlens", c_i32p), ("max_seqlen", ctypes.c_int32),
        ("cp", ctypes.c_int32), ("layout", ctypes.c_int32), ("scale", ctypes.c_float), ("causal", ctypes.c_int32),
        ("window", ctypes.c_int32), ("schedule", ctypes.c_int32), ("deterministic", ctypes.c_int32),
        ("out", ctypes.c_void_p), ("lse", ctypes.c_void_p), ("dout", ctypes.c_void_p),
        ("dq", ctypes.c_void_p), ("dk", ctypes.c_void_p), ("dv", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
    ]


class BlockBwdArgs(ctypes.Structure):
    _fields_ = [
        ("struct_size", ctypes.c_uint32), ("abi_version", ctypes.c_uint32),
        ("dout", ctypes.c_void_p), ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("out", ctypes.c_void_p), ("lse", ctypes.c_void_p),
        ("total_q", ctypes.c_int64), ("total_k", ctypes.c_int64),
        ("num_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("num_docs", ctypes.c_int32),
        ("cu_seqlens_q", c_i32p), ("cu_seqlens_k", c_i32p), ("q_pos_base", c_i32p), ("k_pos_base", c_i32p),
        ("scale", ctypes.c_float), ("causal", ctypes.c_int32), ("window", ctypes.c_int32),
        ("deterministic", ctypes.c_int32), ("dq_acc", ctypes.c_void_p), ("dk_acc", ctypes.c_void_p), ("dv_acc", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
    ]


class KvpArgs(ctypes.Structure):
    _fields_ = [
        ("struct_size", ctypes.c_uint32), ("abi_version", ctypes.c_uint32),
        ("q", ctypes.c_void_p), ("q_stride_head", ctypes.c_int64), ("q_stride_token", ctypes.c_int64),
        ("q_len", ctypes.c_int32), ("num_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("k_cache", ctypes.c_void_p), ("v_cache", ctypes.c_void_p),
        ("num_blocks", ctypes.c_int32), ("block_size", ctypes.c_int32),
        ("block_tables", ctypes.c_void_p), ("shards", ctypes.c_int32), ("blocks_per_shard", ctypes.c_int32),
        ("kv_mode", ctypes.c_int32), ("seg_size", ctypes.c_int32), ("scale", ctypes.c_float),
        ("global_q_offset", ctypes.c_int32), ("sliding_window", ctypes.c_int32), ("tp_out", ctypes.c_int32),
        ("out", ctypes.c_void_p), ("lse", ctypes.c_void_p), ("shard_out", ctypes.c_void_p),
        ("shard_lse", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("shard_base", ctypes.c_int32), ("total_shards", ctypes.c_int32),
    ]


class DecodeArgs(ctypes.Structure):
    _fields_ = [
        ("struct_size", ctypes.c_uint32), ("abi_version", ctypes.c_uint32),
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("out", ctypes.c_void_p),
        ("cu_seqlens_q", ctypes.c_void_p), ("cu_seqlens_k", ctypes.c_void_p),
        ("num_seqs", ctypes.c_int32), ("total_q", ctypes.c_int64), ("total_k", ctypes.c_int64),
        ("num_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("scale", ctypes.c_float), ("validate", ctypes.c_int32),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
    ]


class CachedRingArgs(ctypes.Structure):
    _fields_ = [
        ("struct_size", ctypes.c_uint32), ("abi_version", ctypes.c_uint32),
        ("q", ctypes.c_void_p), ("cache_k", ctypes.POINTER(ctypes.c_void_p)),
        ("cache_v", ctypes.POINTER(ctypes.c_void_p)), ("num_blocks", ctypes.c_int32), ("total", ctypes.c_int64),
        ("num_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("num_docs", ctypes.c_int32), ("cu_seqlens", c_i32p), ("max_seqlen", ctypes.c_int32),
        ("cp", ctypes.c_int32), ("layout", ctypes.c_int32), ("scale", ctypes.c_float), ("window", ctypes.c_int32),
        ("deterministic", ctypes.c_int32), ("out", ctypes.c_void_p), ("lse", ctypes.c_void_p), ("dout", ctypes.c_void_p),
        ("dq", ctypes.c_void_p), ("dcache_k", ctypes.POINTER(ctypes.c_void_p)),
        ("dcache_v", ctypes.POINTER(ctypes.c_void_p)),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
    ]


class RingStepArgs(ctypes.Structure):
    _fields_ = [
        ("struct_size", ctypes.c_uint32), ("abi_version", ctypes.c_uint32),
        ("rank", ctypes.c_int32), ("step", ctypes.c_int32),
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("n_local", ctypes.c_int64),
        ("num_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("num_docs", ctypes.c_int32), ("cu_seqlens", c_i32p), ("cp", ctypes.c_int32), ("layout", ctypes.c_int32),
        ("scale", ctypes.c_float), ("window", ctypes.c_int32),
        ("out_acc", ctypes.c_void_p), ("lse_acc", ctypes.c_void_p), ("out", ctypes.c_void_p),
        ("dout", ctypes.c_void_p), ("out_merged", ctypes.c_void_p), ("lse_merged", ctypes.c_void_p),
        ("dq_acc", ctypes.c_void_p), ("dk_acc", ctypes.c_void_p), ("dv_acc", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
    ]


class DiagArgs(ctypes.Structure):
    _fields_ = [
        ("struct_size", ctypes.c_uint32), ("abi_version", ctypes.c_uint32),
        ("q", ctypes.c_void_p), ("cache_k", ctypes.POINTER(ctypes.c_void_p)),
        ("cache_v", ctypes.POINTER(ctypes.c_void_p)), ("num_blocks", ctypes.c_int32), ("total", ctypes.c_int64),
        ("num_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("scale", ctypes.c_float), ("out0", ctypes.c_void_p), ("lse", ctypes.c_void_p), ("out", ctypes.c_void_p),
        ("dout", ctypes.c_void_p), ("out_merged", ctypes.c_void_p), ("lse_merged", ctypes.c_void_p),
        ("dq0", ctypes.c_void_p), ("dq", ctypes.c_void_p), ("dcache_k", ctypes.POINTER(ctypes.c_void_p)),
        ("dcache_v", ctypes.POINTER(ctypes.c_void_p)),
    ]


class RowRun(ctypes.Structure):
    _fields_ = [("doc", ctypes.c_int32), ("row0", ctypes.c_int32), ("rows", ctypes.c_int32), ("pos0", ctypes.c_int32),
                ("local0", ctypes.c_int32)]


class RingBlock(ctypes.Structure):
    _fields_ = [("rank", ctypes.c_int32), ("step", ctypes.c_int32), ("src", ctypes.c_int32), ("kind", ctypes.c_int32),
                ("causal", ctypes.c_int32), ("q_half", ctypes.c_int32), ("k_half", ctypes.c_int32),
                ("q_run0", ctypes.c_int32), ("q_nruns", ctypes.c_int32), ("k_run0", ctypes.c_int32),
                ("k_nruns", ctypes.c_int32)]


EXPORTS = [
    "cbv_last_error_message", "cbv_abi_version", "cbv_read_status", "cbv_launch_count", "cbv_build_flags",
    "cbv_set_kernel_events",
    "cbv_local_cu_seqlens", "cbv_half_cu_seqlens", "cbv_get_half_index", "cbv_get_half_lse", "cbv_rank_tokens",
    "cbv_rank_pair_counts", "cbv_ring_step", "cbv_plan_zigzag",
    "cbv_block_fwd_workspace_size", "cbv_attn_block_fwd", "cbv_attn_merge",
    "cbv_zigzag_ring_fwd_workspace_size", "cbv_zigzag_ring_fwd", "cbv_zigzag_ring_bwd_workspace_size",
    "cbv_zigzag_ring_bwd", "cbv_block_bwd_workspace_size", "cbv_attn_block_bwd",
    "cbv_kvp_workspace_size", "cbv_kvp_segmented_prefill", "cbv_decode_workspace_size", "cbv_varlen_decode",
    "cbv_noalloc_scratch_bytes", "cbv_zigzag_ring_fwd_noalloc", "cbv_noalloc_read_status",
    "cbv_debug_ring_fwd_stalled", "cbv_ring_step_fwd_workspace_size", "cbv_ring_step_fwd",
    "cbv_ring_step_bwd_workspace_size", "cbv_ring_step_bwd", "cbv_cached_diag_merge", "cbv_cached_diag_grad",
    "cbv_convert_f32_bf16", "cbv_swap_leading_axes",
    "cbv_cached_ring_fwd_workspace_size", "cbv_cached_ring_fwd", "cbv_cached_ring_bwd_workspace_size",
    "cbv_cached_ring_bwd",
]


def _declare(L):
    L.cbv_last_error_message.restype = ctypes.c_char_p
    L.cbv_abi_version.restype = ctypes.c_int
    L.cbv_launch_count.restype = ctypes.c_size_t
    L.cbv_build_flags.restype = ctypes.c_int
    L.cbv_set_kernel_events.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    L.cbv_read_status.argtypes = [ctypes.c_void_p, ctypes.POINTER(ctypes.c_int), ctypes.c_void_p]
    L.cbv_local_cu_seqlens.argtypes = [c_i32p, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, c_i32p]
    L.cbv_half_cu_seqlens.argtypes = [c_i32p, ctypes.c_int32, ctypes.c_int32, c_i32p]
    L.cbv_get_half_index.argtypes = [c_i32p, ctypes.c_int32, ctypes.c_int32, c_i32p, c_i64p]
    L.cbv_get_half_lse.argtypes = [c_f32p, ctypes.c_int32, c_i32p, ctypes.c_int32, ctypes.c_int32, c_f32p]
    L.cbv_rank_tokens.argtypes = [c_i32p, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, c_i32p]
    L.cbv_rank_pair_counts.argtypes = [c_i32p, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, c_i64p]
    L.cbv_ring_step.argtypes = [ctypes.c_int32] * 4 + [c_i32p, c_i32p]
    L.cbv_plan_zigzag.argtypes = [c_i32p, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.POINTER(RingBlock),
                                  ctypes.c_int32, c_i32p, ctypes.POINTER(RowRun), ctypes.c_int32, c_i32p]
    for name, st in (("block_fwd", BlockFwdArgs), ("zigzag_ring_fwd", RingArgs), ("zigzag_ring_bwd", RingArgs),
                     ("block_bwd", BlockBwdArgs), ("kvp", KvpArgs), ("decode", DecodeArgs),
                     ("cached_ring_fwd", CachedRingArgs), ("cached_ring_bwd", CachedRingArgs)):
        f = getattr(L, f"cbv_{name}_workspace_size")
        f.argtypes = [ctypes.POINTER(st)]
        f.restype = ctypes.c_size_t
    for name, st in (("cbv_attn_block_fwd", BlockFwdArgs), ("cbv_zigzag_ring_fwd", RingArgs),
                     ("cbv_zigzag_ring_bwd", RingArgs), ("cbv_attn_block_bwd", BlockBwdArgs),
                     ("cbv_kvp_segmented_prefill", KvpArgs), ("cbv_varlen_decode", DecodeArgs),
                     ("cbv_cached_ring_fwd", CachedRingArgs), ("cbv_cached_ring_bwd", CachedRingArgs)):
        getattr(L, name).argtypes = [ctypes.POINTER(st), ctypes.c_void_p]
    L.cbv_noalloc_scratch_bytes.restype = ctypes.c_size_t
    L.cbv_zigzag_ring_fwd_noalloc.argtypes = [ctypes.POINTER(RingArgs), ctypes.c_void_p]
    L.cbv_noalloc_read_status.argtypes = [ctypes.POINTER(ctypes.c_int), ctypes.c_void_p]
    L.cbv_debug_ring_fwd_stalled.argtypes = [ctypes.POINTER(RingArgs), ctypes.c_uint64, ctypes.c_void_p]
    for name in ("fwd", "bwd"):
        getattr(L, f"cbv_ring_step_{name}_workspace_size").argtypes = [ctypes.POINTER(RingStepArgs)]
        getattr(L, f"cbv_ring_step_{name}_workspace_size").restype = ctypes.c_size_t
        getattr(L, f"cbv_ring_step_{name}").argtypes = [ctypes.POINTER(RingStepArgs), ctypes.c_void_p]
    L.cbv_cached_diag_merge.argtypes = [ctypes.POINTER(DiagArgs), ctypes.c_void_p]
    L.cbv_cached_diag_grad.argtypes = [ctypes.POINTER(DiagArgs), ctypes.c_void_p]
    L.cbv_convert_f32_bf16.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_void_p]
    L.cbv_swap_leading_axes.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                        ctypes.c_int64, ctypes.c_void_p]
    L.cbv_attn_merge.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p,
                                 ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p]


# ----------------------------------------------------------------------------- helpers
def _check(rc: int):
    if rc != 0:
        raise CbvError(rc, lib().cbv_last_error_message().decode())


def debug_build() -> bool:
    """True when the loaded library is the bounds-checking build."""
    return bool(lib().cbv_build_flags() & 1)


def _run(fn, args, ws, device):
    """One library call; in the bounds-checking build, the call's status word is read back (the stream
    synchronises; not while a CUDA graph is being captured) and a kernel that reported a bad index or gave
    up a wait raises."""
    _check(fn(ctypes.byref(args), _stream(device)))
    if debug_build() and not torch.cuda.is_current_stream_capturing():  # no synchronising inside a capture
        code = read_status(ws)
        if code:
            raise CbvError(-12, f"a kernel reported status 0x{code:x}")


def _host_i32(x) -> np.ndarray:
    if isinstance(x, torch.Tensor):
        x = x.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def _p32(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(c_i32p)


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _bf16(t: torch.Tensor, name: str) -> torch.Tensor:
    if not t.is_cuda:
        raise CbvError(-1, f"{name} must be a CUDA tensor")
    if t.dtype != torch.bfloat16:
        raise CbvError(-3, f"{name} must be bfloat16, got {t.dtype}")
    return t.contiguous()


def _shape(t, shape, name, dtype=None):
    """An input the kernels read as exactly this shape (and dtype): check it before any launch."""
    if tuple(t.shape) != tuple(shape) or (dtype is not None and t.dtype != dtype):
        want = f"{tuple(shape)}" + (f" {dtype}" if dtype is not None else "")
        raise CbvError(-2, f"{name} has shape {tuple(t.shape)} {t.dtype}, expected {want}")
    return t


def _given(t, like_shape, dtype, device, name):
    """A caller-provided output: the kernels write exactly this shape, contiguous, so check it."""
    if t is None:
        return None
    if not (isinstance(t, torch.Tensor) and t.is_cuda and t.device == device and t.dtype == dtype
            and tuple(t.shape) == tuple(like_shape) and t.is_contiguous()):
        raise CbvError(-2, f"{name} must be a contiguous {dtype} CUDA tensor of shape {tuple(like_shape)} on {device}")
    return t


def _workspace(nbytes: int, device) -> torch.Tensor:
    # zeroed in the bounds-checking build, whose status check must not read what a call that launched
    # nothing (an empty problem) left unwritten
    alloc = torch.zeros if debug_build() else torch.empty
    return alloc(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def _header(st):
    return dict(struct_size=ctypes.sizeof(st), abi_version=ABI_VERSION)


def _scale(scale):
    return 0.0 if scale is None else float(scale)


def _layout(layout) -> int:
    if isinstance(layout, str):
        return {"zigzag": ZIGZAG, "contiguous": CONTIGUOUS}[layout]
    return int(layout)


def launch_count() -> int:
    """Kernels the library has launched from this thread so far (diagnostic)."""
    return int(lib().cbv_launch_count())


def set_kernel_events(start=None, stop=None) -> None:
    """Measurement hook for this thread: ``torch.cuda.Event`` ``start`` / ``stop`` are recorded
    right before and after every attention-kernel launch (forward, backward, decode) until
    cleared with ``set_kernel_events()``.  Events not yet recorded are recorded once on the
    current stream first, which creates them."""
    def handle(ev):
        if ev is None:
            return None
        if not ev.cuda_event:
            ev.record()
        return ctypes.c_void_p(ev.cuda_event)

    _check(lib().cbv_set_kernel_events(handle(start), handle(stop)))


def read_status(workspace: torch.Tensor) -> int:
    """Device status word of the last call that used ``workspace`` (synchronises)."""
    v = ctypes.c_int(0)
    lib().cbv_read_status(_ptr(workspace), ctypes.byref(v), _stream(workspace.device))
    return v.value


# ----------------------------------------------------------------------------- planner (host)
def local_cu_seqlens(cu_seqlens, cp: int, layout="zigzag") -> np.ndarray:
    cu = _host_i32(cu_seqlens)
    out = np.zeros_like(cu)
    _check(lib().cbv_local_cu_seqlens(_p32(cu), len(cu) - 1, cp, _layout(layout), _p32(out)))
    return out


def half_cu_seqlens(cu_seqlens, cp: int) -> np.ndarray:
    cu = _host_i32(cu_seqlens)
    out = np.zeros_like(cu)
    _check(lib().cbv_half_cu_seqlens(_p32(cu), len(cu) - 1, cp, _p32(out)))
    return out


def get_half_index(cu_local, front: bool) -> np.ndarray:
    cu = _host_i32(cu_local)
    n = ctypes.c_int64(0)
    out = np.zeros(max(int(cu[-1]) // 2, 1), np.int32)
    _check(lib().cbv_get_half_index(_p32(cu), len(cu) - 1, int(front), _p32(out), ctypes.byref(n)))
    return out[: n.value]


def get_half_lse(lse, cu_local, front: bool) -> np.ndarray:
    lse = np.ascontiguousarray(np.asarray(lse, dtype=np.float32))
    cu = _host_i32(cu_local)
    out = np.zeros((lse.shape[0], int(cu[-1]) // 2), np.float32)
    _check(lib().cbv_get_half_lse(lse.ctypes.data_as(c_f32p), lse.shape[0], _p32(cu), len(cu) - 1, int(front),
                                  out.ctypes.data_as(c_f32p)))
    return out


def rank_tokens(cu_seqlens, cp: int, rank: int, layout="zigzag") -> np.ndarray:
    cu = _host_i32(cu_seqlens)
    out = np.zeros(max(int(cu[-1]) // cp, 1), np.int32)
    _check(lib().cbv_rank_tokens(_p32(cu), len(cu) - 1, cp, rank, _layout(layout), _p32(out)))
    return out[: int(cu[-1]) // cp]


def rank_pair_counts(cu_seqlens, cp: int, layout="zigzag", window: int = 0) -> np.ndarray:
    cu = _host_i32(cu_seqlens)
    out = np.zeros(cp, np.int64)
    _check(lib().cbv_rank_pair_counts(_p32(cu), len(cu) - 1, cp, _layout(layout), int(window),
                                      out.ctypes.data_as(c_i64p)))
    return out


def ring_step(rank: int, step: int, cp: int, layout="zigzag") -> tuple[int, int]:
    src, kind = ctypes.c_int32(0), ctypes.c_int32(0)
    _check(lib().cbv_ring_step(rank, step, cp, _layout(layout), ctypes.byref(src), ctypes.byref(kind)))
    return src.value, kind.value


def plan_zigzag(cu_seqlens, cp: int, layout="zigzag") -> list[dict]:
    """Per-step block descriptors of the ring (see ``cbv_plan_zigzag``): one dict per (rank, step) with
    ``rank, step, src, kind, causal, q_half, k_half`` and ``q_runs`` / ``k_runs``, lists of
    ``(doc, row0, rows, pos0, local0)`` runs of global rows in local order."""
    cu = _host_i32(cu_seqlens)
    nb, nr = ctypes.c_int32(0), ctypes.c_int32(0)
    L = lib()
    _check(L.cbv_plan_zigzag(_p32(cu), len(cu) - 1, cp, _layout(layout), None, 0, ctypes.byref(nb), None, 0,
                             ctypes.byref(nr)))
    blocks = (RingBlock * max(nb.value, 1))()
    runs = (RowRun * max(nr.value, 1))()
    _check(L.cbv_plan_zigzag(_p32(cu), len(cu) - 1, cp, _layout(layout), blocks, nb.value, ctypes.byref(nb), runs,
                             nr.value, ctypes.byref(nr)))
    out = []
    for b in blocks[: nb.value]:
        d = {f: getattr(b, f) for f, _ in RingBlock._fields_}
        d["q_runs"] = [(x.doc, x.row0, x.rows, x.pos0, x.local0) for x in runs[b.q_run0: b.q_run0 + b.q_nruns]]
        d["k_runs"] = [(x.doc, x.row0, x.rows, x.pos0, x.local0) for x in runs[b.k_run0: b.k_run0 + b.k_nruns]]
        out.append(d)
    return out


# ----------------------------------------------------------------------------- attention calls
def _given_workspace(ws, nbytes: int, device):
    """A caller-given uint8 workspace of at least ``nbytes`` (else one is allocated).  ``ws`` may also be
    a callable that takes the byte count and returns such a tensor."""
    if ws is None:
        return _workspace(nbytes, device)
    if callable(ws):
        ws = ws(max(int(nbytes), 256))
    if not (isinstance(ws, torch.Tensor) and ws.is_cuda and ws.dtype == torch.uint8 and ws.is_contiguous()):
        raise CbvError(-1, "workspace must be a contiguous uint8 CUDA tensor")
    if ws.numel() < nbytes or ws.data_ptr() % 256:
        raise CbvError(-11, f"workspace needs {nbytes} bytes, 256-byte aligned")
    return ws


def zigzag_ring_fwd(q, k, v, cu_seqlens, cp: int, scale=None, window: int = 0, layout="zigzag",
                    schedule: int = SCHEDULE_FUSED, max_seqlen: int = 0, out=None, lse=None, return_workspace=False,
                    workspace=None):
    """Ring forward over ``cp`` virtual ranks: ``(out [S,H,D] bf16, lse [H,S] f32)``."""
    q, k, v = _bf16(q, "q"), _bf16(k, "k"), _bf16(v, "v")
    S, H, D = q.shape
    _shape(k, (S, k.shape[1], D), "k")
    _shape(v, k.shape, "v")
    cu = _host_i32(cu_seqlens)
    out = _given(out, q.shape, q.dtype, q.device, "out")
    lse = _given(lse, (H, S), torch.float32, q.device, "lse")
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((H, S), dtype=torch.float32, device=q.device) if lse is None else lse
    a = RingArgs(**_header(RingArgs), q=_ptr(q), k=_ptr(k), v=_ptr(v), total=S, num_heads=H, num_kv_heads=k.shape[1],
                 head_dim=D, num_docs=len(cu) - 1, cu_seqlens=_p32(cu), max_seqlen=max_seqlen, cp=cp,
                 layout=_layout(layout), scale=_scale(scale), causal=1, window=int(window), schedule=int(schedule),
                 out=_ptr(out), lse=_ptr(lse))
    ws = _given_workspace(workspace, lib().cbv_zigzag_ring_fwd_workspace_size(ctypes.byref(a)), q.device)
    a.workspace, a.workspace_bytes = _ptr(ws), ws.numel()
    _run(lib().cbv_zigzag_ring_fwd, a, ws, q.device)
    return (out, lse, ws) if return_workspace else (out, lse)


def zigzag_ring_bwd(dout, q, k, v, out, lse, cu_seqlens, cp: int, scale=None, window: int = 0, layout="zigzag",
                    max_seqlen: int = 0, dq=None, dk=None, dv=None, return_workspace=False, deterministic=False,
                    workspace=None):
    """Ring backward fed the merged out/lse: ``(dq, dk, dv)`` bf16.  ``deterministic``: dq summed in
    64-bit fixed point, bit-identical from run to run."""
    dout, q, k, v, out = (_bf16(t, n) for t, n in ((dout, "dout"), (q, "q"), (k, "k"), (v, "v"), (out, "out")))
    S, H, D = q.shape
    _shape(k, (S, k.shape[1], D), "k")
    _shape(v, k.shape, "v")
    _shape(dout, q.shape, "dout")
    _shape(out, q.shape, "out")
    _shape(lse, (H, S), "lse", torch.float32)
    cu = _host_i32(cu_seqlens)
    dq = _given(dq, q.shape, q.dtype, q.device, "dq")
    dk = _given(dk, k.shape, k.dtype, q.device, "dk")
    dv = _given(dv, v.shape, v.dtype, q.device, "dv")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    a = RingArgs(**_header(RingArgs), q=_ptr(q), k=_ptr(k), v=_ptr(v), total=S, num_heads=H, num_kv_heads=k.shape[1],
                 head_dim=D, num_docs=len(cu) - 1, cu_seqlens=_p32(cu), max_seqlen=max_seqlen, cp=cp,
                 layout=_layout(layout), scale=_scale(scale), causal=1, window=int(window), schedule=0,
                 deterministic=int(bool(deterministic)), out=_ptr(out), lse=_ptr(lse.contiguous()), dout=_ptr(dout),
                 dq=_ptr(dq), dk=_ptr(dk), dv=_ptr(dv))
    ws = _given_workspace(workspace, lib().cbv_zigzag_ring_bwd_workspace_size(ctypes.byref(a)), q.device)
    a.workspace, a.workspace_bytes = _ptr(ws), ws.numel()
    _run(lib().cbv_zigzag_ring_bwd, a, ws, q.device)
    return (dq, dk, dv, ws) if return_workspace else (dq, dk, dv)


def _blocks(cache, name: str) -> list[torch.Tensor]:
    """A stacked ``[NB, T, Hkv, D]`` tensor or a list of ``[T, Hkv, D]`` tensors, as bf16 blocks."""
    blocks = list(cache.unbind(0)) if isinstance(cache, torch.Tensor) else list(cache)
    return [_bf16(b, f"{name}[{i}]") for i, b in enumerate(blocks)]


def _ptr_array(blocks):
    return (ctypes.c_void_p * len(blocks))(*[b.data_ptr() for b in blocks])


def _cached_args(q, ck, cv, cu, cp, scale, window, layout, max_seqlen, dck=None, dcv=None, deterministic=False,
                 **tensors):
    S, H, D = q.shape
    keep = [_ptr_array(ck), _ptr_array(cv)] + ([_ptr_array(dck), _ptr_array(dcv)] if dck is not None else [])
    a = CachedRingArgs(**_header(CachedRingArgs), q=_ptr(q), num_blocks=len(ck), total=S, num_heads=H,
                       num_kv_heads=ck[0].shape[1], head_dim=D, num_docs=len(cu) - 1, cu_seqlens=_p32(cu),
                       max_seqlen=max_seqlen, cp=cp, layout=_layout(layout), scale=_scale(scale),
                       window=int(window), deterministic=int(bool(deterministic)),
                       **{k: _ptr(t) for k, t in tensors.items()})
    a.cache_k = ctypes.cast(keep[0], ctypes.POINTER(ctypes.c_void_p))
    a.cache_v = ctypes.cast(keep[1], ctypes.POINTER(ctypes.c_void_p))
    if dck is not None:
        a.dcache_k = ctypes.cast(keep[2], ctypes.POINTER(ctypes.c_void_p))
        a.dcache_v = ctypes.cast(keep[3], ctypes.POINTER(ctypes.c_void_p))
    return a, keep


def cached_ring_fwd(q, cache_k, cache_v, cu_seqlens, cp: int, scale=None, window: int = 0, layout="zigzag",
                    max_seqlen: int = 0, out=None, lse=None, return_workspace=False):
    """EAGLE-3 cached ring forward.  ``cache_k`` / ``cache_v``: a stacked ``[NB,S,Hkv,D]`` tensor or a
    list of ``[S,Hkv,D]`` tensors; block 0 is the sequence (ring over ``cp`` virtual ranks), blocks
    1.. are per-position diagonals; one softmax.  Returns ``(out [S,H,D] bf16, lse [H,S] f32)``."""
    q = _bf16(q, "q")
    ck, cv = _blocks(cache_k, "cache_k"), _blocks(cache_v, "cache_v")
    S, H, _ = q.shape
    for i, (bk, bv) in enumerate(zip(ck, cv)):
        _shape(bk, (S, ck[0].shape[1], q.shape[2]), f"cache_k[{i}]")
        _shape(bv, bk.shape, f"cache_v[{i}]")
    if len(ck) != len(cv):
        raise CbvError(-2, "cache_k and cache_v have different block counts")
    cu = _host_i32(cu_seqlens)
    out = _given(out, q.shape, q.dtype, q.device, "out")
    lse = _given(lse, (H, S), torch.float32, q.device, "lse")
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((H, S), dtype=torch.float32, device=q.device) if lse is None else lse
    a, keep = _cached_args(q, ck, cv, cu, cp, scale, window, layout, max_seqlen, out=out, lse=lse)
    ws = _workspace(lib().cbv_cached_ring_fwd_workspace_size(ctypes.byref(a)), q.device)
    a.workspace, a.workspace_bytes = _ptr(ws), ws.numel()
    _run(lib().cbv_cached_ring_fwd, a, ws, q.device)
    return (out, lse, ws) if return_workspace else (out, lse)


def cached_ring_bwd(dout, q, cache_k, cache_v, out, lse, cu_seqlens, cp: int, scale=None, window: int = 0,
                    layout="zigzag", max_seqlen: int = 0, dq=None, dcache_k=None, dcache_v=None,
                    return_workspace=False, deterministic=False):
    """EAGLE-3 cached ring backward fed the merged out/lse: ``(dq, dcache_k, dcache_v)`` bf16.  The cache
    gradients come back in the form of the cache (stacked tensor or list) unless given."""
    dout, q, out = _bf16(dout, "dout"), _bf16(q, "q"), _bf16(out, "out")
    ck, cv = _blocks(cache_k, "cache_k"), _blocks(cache_v, "cache_v")
    cu = _host_i32(cu_seqlens)
    S, H, D = q.shape
    for i, (bk, bv) in enumerate(zip(ck, cv)):
        _shape(bk, (S, ck[0].shape[1], D), f"cache_k[{i}]")
        _shape(bv, bk.shape, f"cache_v[{i}]")
    if len(ck) != len(cv):
        raise CbvError(-2, "cache_k and cache_v have different block counts")
    _shape(dout, q.shape, "dout")
    _shape(out, q.shape, "out")
    _shape(lse, (H, S), "lse", torch.float32)
    dq = _given(dq, q.shape, q.dtype, q.device, "dq")
    dq = torch.empty_like(q) if dq is None else dq
    stacked = isinstance(cache_k, torch.Tensor)
    if dcache_k is None:
        dcache_k = torch.empty((len(ck),) + tuple(ck[0].shape), dtype=q.dtype, device=q.device) if stacked \
            else [torch.empty_like(b) for b in ck]
    if dcache_v is None:
        dcache_v = torch.empty((len(cv),) + tuple(cv[0].shape), dtype=q.dtype, device=q.device) if stacked \
            else [torch.empty_like(b) for b in cv]
    dck, dcv = _blocks(dcache_k, "dcache_k"), _blocks(dcache_v, "dcache_v")
    for b, given in zip(dck + dcv, list(dcache_k.unbind(0) if isinstance(dcache_k, torch.Tensor) else dcache_k)
                        + list(dcache_v.unbind(0) if isinstance(dcache_v, torch.Tensor) else dcache_v)):
        if b.data_ptr() != given.data_ptr():
            raise CbvError(-2, "dcache blocks must be contiguous bf16 CUDA tensors")
    lse = lse.contiguous()
    a, keep = _cached_args(q, ck, cv, cu, cp, scale, window, layout, max_seqlen, dck=dck, dcv=dcv,
                           deterministic=deterministic, out=out, lse=lse, dout=dout, dq=dq)
    ws = _workspace(lib().cbv_cached_ring_bwd_workspace_size(ctypes.byref(a)), q.device)
    a.workspace, a.workspace_bytes = _ptr(ws), ws.numel()
    _run(lib().cbv_cached_ring_bwd, a, ws, q.device)
    return (dq, dcache_k, dcache_v, ws) if return_workspace else (dq, dcache_k, dcache_v)


def attn_block_fwd(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen: int = 0, scale=None, causal: bool = True,
                   window: int = 0, q_pos_base=None, k_pos_base=None, out=None, lse=None, merge: bool = False,
                   out_dtype=torch.bfloat16):
    """One varlen block: ``(out, lse)``; with ``merge=True`` merges into the running f32 ``(out, lse)`` in place."""
    q, k, v = _bf16(q, "q"), _bf16(k, "k"), _bf16(v, "v")
    Sq, H, D = q.shape
    _shape(k, (k.shape[0], k.shape[1], D), "k")
    _shape(v, k.shape, "v")
    cq, ck = _host_i32(cu_seqlens_q), _host_i32(cu_seqlens_k)
    qb = None if q_pos_base is None else _host_i32(q_pos_base)
    kb = None if k_pos_base is None else _host_i32(k_pos_base)
    if merge:
        out_dtype = torch.float32
        if out is None or lse is None:
            raise CbvError(-1, "merge=True needs the running out (f32) and lse")
    out = _given(out, (Sq, H, D), out_dtype, q.device, "out")
    lse = _given(lse, (H, Sq), torch.float32, q.device, "lse")
    if out is None:
        out = torch.empty((Sq, H, D), dtype=out_dtype, device=q.device)
    if lse is None:
        lse = torch.empty((H, Sq), dtype=torch.float32, device=q.device)
    a = BlockFwdArgs(**_header(BlockFwdArgs), q=_ptr(q), k=_ptr(k), v=_ptr(v), total_q=Sq, total_k=k.shape[0],
                     num_heads=H, num_kv_heads=k.shape[1], head_dim=D, num_docs=len(cq) - 1, cu_seqlens_q=_p32(cq),
                     cu_seqlens_k=_p32(ck), q_pos_base=_p32(qb), k_pos_base=_p32(kb), max_seqlen=int(max_seqlen),
                     scale=_scale(scale), causal=int(bool(causal)), window=int(window), merge=int(bool(merge)),
                     out_dtype=DTYPE_F32 if out.dtype == torch.float32 else DTYPE_BF16, out=_ptr(out), lse=_ptr(lse))
    ws = _workspace(lib().cbv_block_fwd_workspace_size(ctypes.byref(a)), q.device)
    a.workspace, a.workspace_bytes = _ptr(ws), ws.numel()
    _run(lib().cbv_attn_block_fwd, a, ws, q.device)
    return out, lse


def attn_merge(out, lse, block_out, block_lse, return_weight: bool = False):
    """In-place online-softmax merge of ``(block_out, block_lse)`` into the f32 running ``(out, lse)``."""
    S, H, D = out.shape
    _given(out, (S, H, D), torch.float32, out.device, "out")
    _given(lse, (H, S), torch.float32, out.device, "lse")
    _shape(block_out, (S, H, D), "block_out")
    _shape(block_lse, (H, S), "block_lse", torch.float32)
    w = torch.empty((H, S), dtype=torch.float32, device=out.device) if return_weight else None
    dt = DTYPE_F32 if block_out.dtype == torch.float32 else DTYPE_BF16
    _check(lib().cbv_attn_merge(_ptr(out), _ptr(lse), _ptr(block_out.contiguous()), dt, _ptr(block_lse.contiguous()),
                                _ptr(w), S, H, D, _stream(out.device)))
    return (out, lse, w) if return_weight else (out, lse)


def attn_block_bwd(dout, q, k, v, out, lse, cu_seqlens_q, cu_seqlens_k, scale=None, causal: bool = True,
                   window: int = 0, q_pos_base=None, k_pos_base=None, dq_acc=None, dk_acc=None, dv_acc=None,
                   deterministic=False):
    """One block's backward fed the merged ``(out, lse)``; adds into f32 ``(dq_acc, dk_acc, dv_acc)``."""
    dout, q, k, v, out = (_bf16(t, n) for t, n in ((dout, "dout"), (q, "q"), (k, "k"), (v, "v"), (out, "out")))
    Sq, H, D = q.shape
    Sk, Hkv, _ = k.shape
    _shape(v, k.shape, "v")
    _shape(k, (Sk, Hkv, D), "k")
    _shape(dout, q.shape, "dout")
    _shape(out, q.shape, "out")
    _shape(lse, (H, Sq), "lse", torch.float32)
    cq, ck = _host_i32(cu_seqlens_q), _host_i32(cu_seqlens_k)
    qb = None if q_pos_base is None else _host_i32(q_pos_base)
    kb = None if k_pos_base is None else _host_i32(k_pos_base)
    f32 = dict(dtype=torch.float32, device=q.device)
    dq_acc = _given(dq_acc, (Sq, H, D), torch.float32, q.device, "dq_acc")
    dk_acc = _given(dk_acc, (Sk, Hkv, D), torch.float32, q.device, "dk_acc")
    dv_acc = _given(dv_acc, (Sk, Hkv, D), torch.float32, q.device, "dv_acc")
    dq_acc = torch.zeros((Sq, H, D), **f32) if dq_acc is None else dq_acc
    dk_acc = torch.zeros((Sk, Hkv, D), **f32) if dk_acc is None else dk_acc
    dv_acc = torch.zeros((Sk, Hkv, D), **f32) if dv_acc is None else dv_acc
    a = BlockBwdArgs(**_header(BlockBwdArgs), dout=_ptr(dout), q=_ptr(q), k=_ptr(k), v=_ptr(v), out=_ptr(out),
                     lse=_ptr(lse.contiguous()), total_q=Sq, total_k=Sk, num_heads=H, num_kv_heads=Hkv, head_dim=D,
                     num_docs=len(cq) - 1, cu_seqlens_q=_p32(cq), cu_seqlens_k=_p32(ck), q_pos_base=_p32(qb),
                     k_pos_base=_p32(kb), scale=_scale(scale), causal=int(bool(causal)), window=int(window),
                     deterministic=int(bool(deterministic)), dq_acc=_ptr(dq_acc), dk_acc=_ptr(dk_acc),
                     dv_acc=_ptr(dv_acc))
    ws = _workspace(lib().cbv_block_bwd_workspace_size(ctypes.byref(a)), q.device)
    a.workspace, a.workspace_bytes = _ptr(ws), ws.numel()
    _run(lib().cbv_attn_block_bwd, a, ws, q.device)
    return dq_acc, dk_acc, dv_acc


def kvp_segmented_prefill(q, k_cache, v_cache, block_tables, kv_mode=KV_ROUND_ROBIN, seg_size: int = 512,
                          scale=None, global_q_offset: int = 0, sliding_window: int = 0, per_shard: bool = False,
                          return_lse: bool = True, tp_out: bool = False, out=None, lse=None, shard_out=None,
                          shard_lse=None, workspace=None, shard_base: int = 0, total_shards: int = 0):
    """Paged KV-parallel prefill; q ``[HQ, S, D]`` -> ``out [HQ, S, D]`` (``[HQ, D, S]`` with ``tp_out``)
    (+ lse, + per-shard partials).  ``block_tables`` are shards ``shard_base ..`` of ``total_shards``
    (0: all of them): key positions follow the global shard index."""
    if not q.is_cuda or q.dtype != torch.bfloat16:
        raise CbvError(-3, "q must be a CUDA bfloat16 tensor")
    k_cache, v_cache = _bf16(k_cache, "k_cache"), _bf16(v_cache, "v_cache")
    HQ, S, D = q.shape
    nb, HKV, bs, _ = k_cache.shape
    _shape(k_cache, (nb, HKV, bs, D), "k_cache")
    _shape(v_cache, k_cache.shape, "v_cache")
    bt = block_tables.to(device=q.device, dtype=torch.int32).contiguous()
    R, bps = bt.shape
    oshape = (HQ, D, S) if tp_out else (HQ, S, D)
    out = _given(out, oshape, torch.bfloat16, q.device, "out")
    out = torch.empty(oshape, dtype=torch.bfloat16, device=q.device) if out is None else out
    lse = _given(lse, (HQ, S), torch.float32, q.device, "lse") if return_lse else None
    if return_lse and lse is None:
        lse = torch.empty((HQ, S), dtype=torch.float32, device=q.device)
    so = sl = None
    if per_shard:
        so = _given(shard_out, (R, HQ, S, D), torch.float32, q.device, "shard_out")
        sl = _given(shard_lse, (R, HQ, S), torch.float32, q.device, "shard_lse")
        so = torch.empty((R, HQ, S, D), dtype=torch.float32, device=q.device) if so is None else so
        sl = torch.empty((R, HQ, S), dtype=torch.float32, device=q.device) if sl is None else sl
    a = KvpArgs(**_header(KvpArgs), q=_ptr(q), q_stride_head=q.stride(0), q_stride_token=q.stride(1), q_len=S,
                num_heads=HQ, num_kv_heads=HKV, head_dim=D, k_cache=_ptr(k_cache), v_cache=_ptr(v_cache),
                num_blocks=nb, block_size=bs, block_tables=_ptr(bt), shards=R, blocks_per_shard=bps,
                kv_mode=int(kv_mode), seg_size=int(seg_size), scale=_scale(scale),
                global_q_offset=int(global_q_offset), sliding_window=int(sliding_window), tp_out=int(bool(tp_out)),
                out=_ptr(out),
                lse=_ptr(lse), shard_out=_ptr(so), shard_lse=_ptr(sl), shard_base=int(shard_base),
                total_shards=int(total_shards))
    if q.stride(2) != 1:
        raise CbvError(-4, "q's last dimension must be contiguous")
    ws = _given_workspace(workspace, lib().cbv_kvp_workspace_size(ctypes.byref(a)), q.device)
    a.workspace, a.workspace_bytes = _ptr(ws), ws.numel()
    _run(lib().cbv_kvp_segmented_prefill, a, ws, q.device)
    res = [out]
    if return_lse:
        res.append(lse)
    if per_shard:
        res += [so, sl]
    return tuple(res) if len(res) > 1 else out


def varlen_decode(q, k, v, cu_seqlens_q, cu_seqlens_k, scale=None, validate=None, out=None, workspace=None):
    """One query per sequence, GQA, offsets read on the device: ``out [total_q, HQ, D]`` bf16."""
    q, k, v = _bf16(q, "q"), _bf16(k, "k"), _bf16(v, "v")
    _shape(k, (k.shape[0], k.shape[1], q.shape[2]), "k")
    _shape(v, k.shape, "v")
    if validate is None:
        validate = not torch.cuda.is_current_stream_capturing()
    cq = cu_seqlens_q.to(device=q.device, dtype=torch.int32).contiguous()
    ck = cu_seqlens_k.to(device=q.device, dtype=torch.int32).contiguous()
    out = _given(out, q.shape, q.dtype, q.device, "out")
    out = torch.empty_like(q) if out is None else out
    a = DecodeArgs(**_header(DecodeArgs), q=_ptr(q), k=_ptr(k), v=_ptr(v), out=_ptr(out), cu_seqlens_q=_ptr(cq),
                   cu_seqlens_k=_ptr(ck), num_seqs=ck.numel() - 1, total_q=q.shape[0], total_k=k.shape[0],
                   num_heads=q.shape[1], num_kv_heads=k.shape[1], head_dim=q.shape[2], scale=_scale(scale),
                   validate=int(bool(validate)))
    if cq.numel() != ck.numel():
        raise CbvError(-9, "cu_seqlens_q and cu_seqlens_k sizes differ")
    ws = _workspace(lib().cbv_decode_workspace_size(ctypes.byref(a)), q.device) if workspace is None else workspace
    a.workspace, a.workspace_bytes = _ptr(ws), ws.numel()
    _run(lib().cbv_varlen_decode, a, ws, q.device)
    return out


# ----------------------------------------------------------------------------- ring steps on real ranks
def _step_args(rank, step, q, k, v, cu, cp, scale, window, layout, **tensors):
    n, H, D = q.shape
    return RingStepArgs(**_header(RingStepArgs), rank=int(rank), step=int(step), q=_ptr(q), k=_ptr(k), v=_ptr(v),
                        n_local=n, num_heads=H, num_kv_heads=k.shape[1], head_dim=D, num_docs=len(cu) - 1,
                        cu_seqlens=_p32(cu), cp=int(cp), layout=_layout(layout), scale=_scale(scale),
                        window=int(window), **{name: _ptr(t) for name, t in tensors.items()})


def ring_step_fwd(rank: int, step: int, q, k, v, cu_seqlens, cp: int, out_acc, lse_acc, out=None, scale=None,
                  window: int = 0, layout="zigzag"):
    """One rank's block at one ring step on local buffers (see ``cbv_ring_step_fwd``): merges into the
    running f32 ``(out_acc [n,H,D], lse_acc [H,n])``; with ``out`` (bf16) also rounds the running out into it."""
    q, k, v = _bf16(q, "q"), _bf16(k, "k"), _bf16(v, "v")
    n, H, D = q.shape
    _shape(k, (n, k.shape[1], D), "k")
    _shape(v, k.shape, "v")
    _given(out_acc, (n, H, D), torch.float32, q.device, "out_acc")
    _given(lse_acc, (H, n), torch.float32, q.device, "lse_acc")
    if out is not None:
        _given(out, (n, H, D), torch.bfloat16, q.device, "out")
    cu = _host_i32(cu_seqlens)
    a = _step_args(rank, step, q, k, v, cu, cp, scale, window, layout, out_acc=out_acc, lse_acc=lse_acc, out=out)
    ws = _workspace(lib().cbv_ring_step_fwd_workspace_size(ctypes.byref(a)), q.device)
    a.workspace, a.workspace_bytes = _ptr(ws), ws.numel()
    _run(lib().cbv_ring_step_fwd, a, ws, q.device)
    return out_acc, lse_acc


def ring_step_bwd(rank: int, step: int, dout, q, k, v, out, lse, cu_seqlens, cp: int, dq_acc, dk_acc, dv_acc,
                  scale=None, window: int = 0, layout="zigzag"):
    """One rank's block backward at one ring step, fed this rank's merged ``(out, lse)``: adds into
    ``dq_acc`` (this rank's rows) and ``dk_acc`` / ``dv_acc`` (the rows of the k/v held at this step)."""
    dout, q, k, v, out = (_bf16(t, nm) for t, nm in ((dout, "dout"), (q, "q"), (k, "k"), (v, "v"), (out, "out")))
    n, H, D = q.shape
    _shape(k, (n, k.shape[1], D), "k")
    _shape(v, k.shape, "v")
    _shape(dout, q.shape, "dout")
    _shape(out, q.shape, "out")
    _shape(lse, (H, n), "lse", torch.float32)
    _given(dq_acc, (n, H, D), torch.float32, q.device, "dq_acc")
    _given(dk_acc, k.shape, torch.float32, q.device, "dk_acc")
    _given(dv_acc, k.shape, torch.float32, q.device, "dv_acc")
    cu = _host_i32(cu_seqlens)
    a = _step_args(rank, step, q, k, v, cu, cp, scale, window, layout, dout=dout, out_merged=out,
                   lse_merged=lse.contiguous(), dq_acc=dq_acc, dk_acc=dk_acc, dv_acc=dv_acc)
    ws = _workspace(lib().cbv_ring_step_bwd_workspace_size(ctypes.byref(a)), q.device)
    a.workspace, a.workspace_bytes = _ptr(ws), ws.numel()
    _run(lib().cbv_ring_step_bwd, a, ws, q.device)
    return dq_acc, dk_acc, dv_acc


def _diag_args(q, ck, cv, scale, **tensors):
    T, H, D = q.shape
    keep = [_ptr_array(ck), _ptr_array(cv)]
    a = DiagArgs(**_header(DiagArgs), q=_ptr(q), num_blocks=len(ck), total=T, num_heads=H,
                 num_kv_heads=ck[0].shape[1], head_dim=D, scale=_scale(scale),
                 **{name: _ptr(t) for name, t in tensors.items()})
    a.cache_k = ctypes.cast(keep[0], ctypes.POINTER(ctypes.c_void_p))
    a.cache_v = ctypes.cast(keep[1], ctypes.POINTER(ctypes.c_void_p))
    return a, keep


def cached_diag_merge(q, cache_k, cache_v, out0, lse, scale=None, out=None):
    """Merge the per-position cache diagonals (blocks 1..) into block 0's normalised f32 ``out0`` and
    ``lse`` (updated in place): returns ``(out bf16, lse)``."""
    q = _bf16(q, "q")
    ck, cv = _blocks(cache_k, "cache_k"), _blocks(cache_v, "cache_v")
    T, H, D = q.shape
    _shape(out0, q.shape, "out0", torch.float32)
    _given(lse, (H, T), torch.float32, q.device, "lse")
    out = torch.empty_like(q) if out is None else _given(out, q.shape, torch.bfloat16, q.device, "out")
    a, keep = _diag_args(q, ck, cv, scale, out0=out0.contiguous(), lse=lse, out=out)
    _check(lib().cbv_cached_diag_merge(ctypes.byref(a), _stream(q.device)))
    return out, lse


def cached_diag_grad(dout, q, cache_k, cache_v, out, lse, dq0, scale=None, dq=None, dcache_k=None, dcache_v=None):
    """Closed-form gradients of the cache diagonals fed the merged ``(out, lse)``: ``dq = dq0 + diagonal
    terms`` (bf16) and the gradients of blocks 1.. (lists; entry 0 is None)."""
    dout, q, out = _bf16(dout, "dout"), _bf16(q, "q"), _bf16(out, "out")
    ck, cv = _blocks(cache_k, "cache_k"), _blocks(cache_v, "cache_v")
    T, H, D = q.shape
    _shape(dq0, q.shape, "dq0", torch.float32)
    _shape(lse, (H, T), "lse", torch.float32)
    dq = torch.empty_like(q) if dq is None else _given(dq, q.shape, torch.bfloat16, q.device, "dq")
    dck = [None] + ([torch.empty_like(b) for b in ck[1:]] if dcache_k is None else list(dcache_k)[1:])
    dcv = [None] + ([torch.empty_like(b) for b in cv[1:]] if dcache_v is None else list(dcache_v)[1:])
    a, keep = _diag_args(q, ck, cv, scale, dout=dout, out_merged=out, lse_merged=lse.contiguous(), dq0=dq0.contiguous(),
                         dq=dq)
    pk = (ctypes.c_void_p * len(ck))(*[0] + [b.data_ptr() for b in dck[1:]])
    pv = (ctypes.c_void_p * len(cv))(*[0] + [b.data_ptr() for b in dcv[1:]])
    a.dcache_k = ctypes.cast(pk, ctypes.POINTER(ctypes.c_void_p))
    a.dcache_v = ctypes.cast(pv, ctypes.POINTER(ctypes.c_void_p))
    _check(lib().cbv_cached_diag_grad(ctypes.byref(a), _stream(q.device)))
    return dq, dck, dcv


def convert_f32_bf16(src, dst=None, mul: float = 1.0):
    """bf16 rounding of an f32 tensor (``cbv_convert_f32_bf16``)."""
    if not src.is_cuda or src.dtype != torch.float32:
        raise CbvError(-3, "src must be a CUDA float32 tensor")
    src = src.contiguous()
    dst = torch.empty(src.shape, dtype=torch.bfloat16, device=src.device) if dst is None else dst
    _given(dst, src.shape, torch.bfloat16, src.device, "dst")
    _check(lib().cbv_convert_f32_bf16(_ptr(src), _ptr(dst), src.numel(), float(mul), _stream(src.device)))
    return dst


def swap_leading_axes(src, dst=None):
    """``dst[b, a, ...] = src[a, b, ...]`` for a contiguous CUDA tensor of >= 2 dims (``cbv_swap_leading_axes``)."""
    if not src.is_cuda or src.dim() < 2:
        raise CbvError(-1, "src must be a CUDA tensor with at least two dimensions")
    src = src.contiguous()
    a, b = src.shape[0], src.shape[1]
    shape = (b, a) + tuple(src.shape[2:])
    dst = torch.empty(shape, dtype=src.dtype, device=src.device) if dst is None else dst
    _given(dst, shape, src.dtype, src.device, "dst")
    row = src[0, 0].numel() * src.element_size() if src.numel() else 0
    _check(lib().cbv_swap_leading_axes(_ptr(src), _ptr(dst), a, b, row, _stream(src.device)))
    return dst

