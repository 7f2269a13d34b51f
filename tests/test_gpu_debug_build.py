"""Out-of-bounds evidence without compute-sanitizer.

The bounds-checking build (libcbv_debug.so, compiled with CBV_DEBUG) checks every row and
page index a kernel copies from or stores to against its tensor; a violation is recorded in
the call's status word, and the binding reads that word back after every call of this build.
The parity suites are run again against it in a subprocess, so every call they make must both
match the oracle and report a clear status.  The varlen decode checks its device-side offsets
in every build: a sequence whose offsets leave the tensors is reported and skipped.
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import context_blockwise_causal_varlen_b200 as cbv
from context_blockwise_causal_varlen_b200.build import DEBUG_LIB, build
from oracle import decode as DEC
from synth import cu_from_lengths
from tests.gpu_util import check_out, dev, f64, gen, host, sync

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SUITES = ["tests/test_gpu_ring.py", "tests/test_gpu_block.py", "tests/test_gpu_kvp_decode.py", "tests/test_gpu_edges.py",
          "tests/test_gpu_fuzz.py", "tests/test_gpu_cached.py", "tests/test_gpu_deterministic.py",
          "tests/test_gpu_dist.py"]


def test_parity_suites_pass_on_the_bounds_checking_build():
    if not os.path.exists(DEBUG_LIB):
        build(debug=True)
    env = dict(os.environ, CBV_LIBRARY="debug")
    res = subprocess.run([sys.executable, "-m", "pytest", *SUITES, "-m", "gpu", "-q", "-x", "-p", "no:cacheprovider"],
                         cwd=ROOT, env=env, capture_output=True, text=True, timeout=1800)
    assert res.returncode == 0, res.stdout[-3000:] + res.stderr[-2000:]
    assert " passed" in res.stdout


def test_the_bounds_checking_build_is_the_one_loaded_there():
    if not os.path.exists(DEBUG_LIB):
        build(debug=True)
    code = "import context_blockwise_causal_varlen_b200 as c; print(c.LIB_PATH, c.debug_build())"
    out = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=dict(os.environ, CBV_LIBRARY="debug"),
                         capture_output=True, text=True, timeout=300).stdout
    assert out.strip().endswith("libcbv_debug.so True")


def test_decode_skips_and_reports_sequences_whose_offsets_leave_the_tensors():
    # offsets change on the device between graph replays, so the kernel checks them itself: sequences
    # 2 and 3 point past the 400 key rows; the kernel reports them (0x205) before reading anything
    hq, hkv, D = 8, 2, 128
    q, k, v = gen(91, (4, hq, D), (400, hkv, D), (400, hkv, D))
    cu_q = torch.arange(5, dtype=torch.int32, device="cuda")
    good = cu_from_lengths([5, 100])
    ck = torch.tensor([0, 5, 105, 5000, 6000], dtype=torch.int32, device="cuda")
    out = torch.zeros((4, hq, D), dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    if cbv.debug_build():
        with pytest.raises(cbv.CbvError):
            cbv.varlen_decode(dev(q), dev(k), dev(v), cu_q, ck, scale=0.1, validate=False, out=out, workspace=ws)
    else:
        cbv.varlen_decode(dev(q), dev(k), dev(v), cu_q, ck, scale=0.1, validate=False, out=out, workspace=ws)
    sync()
    assert cbv.read_status(ws) == 0x205
    ref = DEC.varlen_decode(f64(q[:2]), f64(k), f64(v), np.arange(3), good, 0.1)
    check_out(host(out[:2]), ref)
    assert bool((out[2:] == 0).all())  # skipped: left as they were
