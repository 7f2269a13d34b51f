"""The allocation-free ring forward, through the C ABI.

cbv_zigzag_ring_fwd_noalloc serves callers that cannot call cudaMalloc where they
run attention (a serving loop whose memory budget is fixed at start-up, a runtime
that owns all device memory, a plain C host without a device allocator): its
scratch is a fixed array compiled into the library.  These tests check that it
returns what the workspace entry point returns and what the oracle computes, on two
calls in a row that share the array, that its status word reads clear afterwards,
and that a problem too large for the array is refused with a message.  The file is
named to run last, so a stop at the first failure has already run everything else.
"""
import ctypes

import numpy as np
import pytest
import torch

import context_blockwise_causal_varlen_b200 as cbv
from oracle import attention as A
from synth import cu_from_lengths
from tests.gpu_util import LSE_ATOL, OUT_ATOL, check_guards, check_lse, check_out, dev, f64, gen, guarded, host, sync

pytestmark = pytest.mark.gpu


def _args(q, k, v, cu, cp, out, lse, schedule=cbv.SCHEDULE_FUSED, total=None, heads=None):
    S, H, D = q.shape
    return cbv.RingArgs(struct_size=ctypes.sizeof(cbv.RingArgs), abi_version=cbv.ABI_VERSION, q=q.data_ptr(),
                        k=k.data_ptr(), v=v.data_ptr(), total=S if total is None else total,
                        num_heads=H if heads is None else heads, num_kv_heads=k.shape[1] if heads is None else heads,
                        head_dim=D, num_docs=len(cu) - 1, cu_seqlens=cu.ctypes.data_as(cbv.c_i32p), cp=cp,
                        layout=cbv.ZIGZAG, scale=0.0, causal=1, window=0, schedule=schedule, out=out.data_ptr(),
                        lse=lse.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("lengths,cp,H,D", [([96, 160], 2, 2, 64), ([1000, 48, 2048], 4, 4, 128)])
def test_noalloc_matches_the_workspace_entry_point_twice(lengths, cp, H, D):
    L = cbv.lib()
    cu = cu_from_lengths(lengths)
    S = int(cu[-1])
    q, k, v = gen(41, (S, H, D), (S, H, D), (S, H, D))
    tq, tk, tv = dev(q), dev(k), dev(v)
    ref_out, ref_lse = cbv.zigzag_ring_fwd(tq, tk, tv, cu, cp)
    ro, rl = A.attention_fwd(f64(q), f64(k), f64(v), cu, cu, D ** -0.5)
    # the second call reuses the array the first one left behind; the second asks for the stepwise
    # schedule, which this entry point ignores (it always runs the fused one)
    for schedule in (cbv.SCHEDULE_FUSED, cbv.SCHEDULE_STEPWISE):
        (out, ob), (lse, lb) = guarded((S, H, D), torch.bfloat16), guarded((H, S), torch.float32)
        a = _args(tq, tk, tv, cu, cp, out, lse, schedule=schedule)
        rc = L.cbv_zigzag_ring_fwd_noalloc(ctypes.byref(a), _stream())
        assert rc == 0, L.cbv_last_error_message().decode()
        sync()
        check_guards(out, ob, what="out")
        check_guards(lse, lb, what="lse")
        assert (out.float() - ref_out.float()).abs().max().item() <= OUT_ATOL
        assert (lse - ref_lse).abs().max().item() <= LSE_ATOL
        check_out(host(out), ro)
        check_lse(host(lse), rl)
        st = ctypes.c_int(-1)
        assert L.cbv_noalloc_read_status(ctypes.byref(st), _stream()) == 0 and st.value == 0


def test_noalloc_refuses_what_does_not_fit():
    # 1000 documents of 16 tokens at cp = 2 and 8 heads: 32000 forward tasks, a schedule over 1 MiB.
    # The call is refused on the host before anything is launched, so the tensors need only exist.
    L = cbv.lib()
    cu = cu_from_lengths([16] * 1000)
    q = torch.zeros((16, 8, 64), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((8, 16), dtype=torch.float32, device="cuda")
    a = _args(q, q, q, cu, 2, q, lse, total=16000, heads=8)
    assert L.cbv_zigzag_ring_fwd_workspace_size(ctypes.byref(a)) > L.cbv_noalloc_scratch_bytes()
    n0 = cbv.launch_count()
    rc = L.cbv_zigzag_ring_fwd_noalloc(ctypes.byref(a), _stream())
    assert cbv.STATUS[rc] == "WORKSPACE_TOO_SMALL"
    assert b"static scratch" in L.cbv_last_error_message()
    assert cbv.launch_count() == n0
