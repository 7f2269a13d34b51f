"""The failure path, exercised without faulting or hanging anything.

Every wait in the kernels is bounded: a stalled pipeline records a code in the
workspace status word and the kernel returns, so the host reads CBV_ERR_TIMEOUT and
the context stays usable.  These tests (1) put a code into a status word from the
host and read it back through the C ABI, and (2) run a forward whose copy producer
issues no loads at all with a 1 ms wait limit, so every wait runs out before any
copy or tensor-core operation is in flight, then run a normal call on the same
stream and check it against the oracle.
"""
import ctypes
import time

import numpy as np
import pytest
import torch

import context_blockwise_causal_varlen_b200 as cbv
from oracle import attention as A
from synth import cu_from_lengths
from tests.gpu_util import check_lse, check_out, dev, f64, gen, host, sync

pytestmark = pytest.mark.gpu

TIMEOUT_CODES = {0x101, 0x102, 0x103, 0x104, 0x105}


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _read(ws):
    st = ctypes.c_int(0)
    rc = cbv.lib().cbv_read_status(ctypes.c_void_p(ws.data_ptr()), ctypes.byref(st), _stream())
    return rc, st.value


def test_a_status_word_set_on_the_host_reads_as_a_timeout():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    assert _read(ws) == (0, 0)
    ws.view(torch.int32)[0] = 0x104
    rc, code = _read(ws)
    assert cbv.STATUS[rc] == "TIMEOUT" and code == 0x104
    assert b"0x104" in cbv.lib().cbv_last_error_message()


@pytest.mark.parametrize("lengths,cp,H,D", [([264, 520, 128], 2, 2, 128), ([96, 160], 2, 2, 64)])
def test_a_stalled_forward_times_out_and_the_stream_stays_usable(lengths, cp, H, D):
    L = cbv.lib()
    cu = cu_from_lengths(lengths)
    S = int(cu[-1])
    q, k, v = gen(71, (S, H, D), (S, H, D), (S, H, D))
    tq, tk, tv = dev(q), dev(k), dev(v)
    out = torch.zeros_like(tq)
    lse = torch.zeros((H, S), dtype=torch.float32, device="cuda")
    a = cbv.RingArgs(struct_size=ctypes.sizeof(cbv.RingArgs), abi_version=cbv.ABI_VERSION, q=tq.data_ptr(),
                     k=tk.data_ptr(), v=tv.data_ptr(), total=S, num_heads=H, num_kv_heads=H, head_dim=D,
                     num_docs=len(cu) - 1, cu_seqlens=cu.ctypes.data_as(cbv.c_i32p), cp=cp, layout=cbv.ZIGZAG,
                     scale=0.0, causal=1, window=0, schedule=cbv.SCHEDULE_FUSED, out=out.data_ptr(),
                     lse=lse.data_ptr())
    ws = torch.zeros(max(L.cbv_zigzag_ring_fwd_workspace_size(ctypes.byref(a)), 256), dtype=torch.uint8,
                     device="cuda")
    a.workspace, a.workspace_bytes = ws.data_ptr(), ws.numel()
    t0 = time.perf_counter()
    rc = L.cbv_debug_ring_fwd_stalled(ctypes.byref(a), 1_000_000, _stream())
    assert rc == 0, L.cbv_last_error_message().decode()
    rc, code = _read(ws)  # synchronises the stream
    elapsed = time.perf_counter() - t0
    assert cbv.STATUS[rc] == "TIMEOUT" and code in TIMEOUT_CODES, (rc, hex(code))
    assert elapsed < 10.0
    assert bool((out == 0).all()) and bool((lse == 0).all())  # nothing was written
    # the same stream, a normal call: correct result and a clear status word
    o2, l2, ws2 = cbv.zigzag_ring_fwd(tq, tk, tv, cu, cp, return_workspace=True)
    sync()
    assert cbv.read_status(ws2) == 0
    ro, rl = A.attention_fwd(f64(q), f64(k), f64(v), cu, cu, D ** -0.5)
    check_out(host(o2), ro)
    check_lse(host(l2), rl)
