"""The allocation-free ring forward, through the C ABI.

cbv_zigzag_ring_fwd_noalloc serves callers that cannot call cudaMalloc where they
run attention (a serving loop whose memory budget is fixed at start-up, a runtime
that owns all device memory, a plain C host without a device allocator): its
scratch is a fixed array compiled into the library.  These tests check that it
returns what the workspace entry point returns, on two calls in a row that share
the array, and that a problem too large for the array is refused with a message.
The file is named to run last, so a stop at the first failure has already run
everything else.
"""
import ctypes

import numpy as np
import pytest
import torch

import context_blockwise_causal_varlen_b200 as cbv
from synth import cu_from_lengths
from tests.gpu_util import LSE_ATOL, OUT_ATOL, dev, gen, sync

pytestmark = pytest.mark.gpu


def _args(q, k, v, cu, cp, out, lse, schedule=cbv.SCHEDULE_FUSED):
    S, H, D = q.shape
    return cbv.RingArgs(struct_size=ctypes.sizeof(cbv.RingArgs), abi_version=cbv.ABI_VERSION, q=q.data_ptr(),
                        k=k.data_ptr(), v=v.data_ptr(), total=S, num_heads=H, num_kv_heads=k.shape[1], head_dim=D,
                        num_docs=len(cu) - 1, cu_seqlens=cu.ctypes.data_as(cbv.c_i32p), cp=cp, layout=cbv.ZIGZAG,
                        scale=0.0, causal=1, window=0, schedule=schedule, out=out.data_ptr(), lse=lse.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("lengths,cp,H,D", [([96, 160], 2, 2, 64), ([1000, 48, 2048], 4, 4, 128)])
def test_noalloc_matches_the_workspace_entry_point_twice(lengths, cp, H, D):
    L = cbv.lib()
    cu = cu_from_lengths(lengths)
    S = int(cu[-1])
    q, k, v = (dev(x) for x in gen(41, (S, H, D), (S, H, D), (S, H, D)))
    ref_out, ref_lse = cbv.zigzag_ring_fwd(q, k, v, cu, cp)
    for _ in range(2):  # the second call reuses the array the first one left behind
        out = torch.full_like(q, float("nan"))
        lse = torch.full((H, S), float("nan"), dtype=torch.float32, device="cuda")
        a = _args(q, k, v, cu, cp, out, lse)
        rc = L.cbv_zigzag_ring_fwd_noalloc(ctypes.byref(a), _stream())
        assert rc == 0, L.cbv_last_error_message().decode()
        sync()
        assert torch.isfinite(out.float()).all()
        assert (out.float() - ref_out.float()).abs().max().item() <= OUT_ATOL
        assert (lse - ref_lse).abs().max().item() <= LSE_ATOL


def test_noalloc_refuses_what_does_not_fit():
    L = cbv.lib()
    cu = np.array([0, 4096], np.int32)
    q = torch.empty((4096, 8, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    lse = torch.empty((8, 4096), dtype=torch.float32, device="cuda")
    a = _args(q, q, q, cu, 2, out, lse, schedule=cbv.SCHEDULE_STEPWISE)  # needs an fp32 running output
    assert L.cbv_zigzag_ring_fwd_workspace_size(ctypes.byref(a)) > L.cbv_noalloc_scratch_bytes()
    rc = L.cbv_zigzag_ring_fwd_noalloc(ctypes.byref(a), _stream())
    assert cbv.STATUS[rc] == "WORKSPACE_TOO_SMALL"
    assert b"static scratch" in L.cbv_last_error_message()
