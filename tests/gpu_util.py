"""Shared helpers for the GPU parity tests (inputs from synth, comparisons to the oracle)."""
import numpy as np
import torch

from synth import normal_bf16, streams, to_torch_bf16

OUT_ATOL = 1e-2      # out: max-abs error (bf16 in, fp32 accumulate)
LSE_ATOL = 1e-3      # lse: max-abs error
GRAD_REL = 2e-2      # dq/dk/dv: max-abs error relative to the tensor's max-abs


def gen(seed, *shapes):
    """bf16-valued float32 arrays, one stream per shape, in order."""
    g = streams(seed, len(shapes))
    return [normal_bf16(g[i], s) for i, s in enumerate(shapes)]


def dev(x):
    return to_torch_bf16(x, "cuda")


def f64(x):
    return np.asarray(x, dtype=np.float64)


def host(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def check_out(got, ref, atol=OUT_ATOL, what="out"):
    got = np.asarray(got, np.float64)
    err = np.abs(got - ref).max() if got.size else 0.0
    assert err <= atol, f"{what}: max abs err {err:.3e} > {atol}"
    return err


def check_lse(got, ref, atol=LSE_ATOL, what="lse"):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    gi, ri = np.isneginf(got), np.isneginf(ref)
    assert np.array_equal(gi, ri), f"{what}: -inf pattern differs ({gi.sum()} vs {ri.sum()})"
    fin = ~ri
    err = np.abs(got[fin] - ref[fin]).max() if fin.any() else 0.0
    assert err <= atol, f"{what}: max abs err {err:.3e} > {atol}"
    return err


def check_rel(got, ref, rel=GRAD_REL, what="grad"):
    got = np.asarray(got, np.float64)
    scale = max(np.abs(ref).max(), 1e-30)
    err = np.abs(got - ref).max() / scale
    assert err <= rel, f"{what}: max abs err / max|ref| = {err:.3e} > {rel}"
    return err


def sync():
    torch.cuda.synchronize()


# ----------------------------------------------------------------------------- guard regions
# Outputs and workspaces of the parity tests sit inside larger buffers whose extra elements
# before and after are filled with a NaN canary.  A kernel writing outside its output changes a
# canary; one leaving part of its output unwritten leaves a NaN inside.
GUARD = 4096  # elements of canary on each side (16-byte multiple for every dtype used)


def guarded(shape, dtype, device="cuda", guard=GUARD):
    """``(t, buf)``: an uninitialised-looking tensor ``t`` of ``shape`` (NaN-filled) inside ``buf``."""
    n = int(np.prod(shape)) if len(shape) else 1
    if dtype == torch.uint8:
        buf = torch.full((n + 2 * guard,), 0xFF, dtype=dtype, device=device)  # 0xFFFFFFFF is a NaN as f32
    else:
        buf = torch.full((n + 2 * guard,), float("nan"), dtype=dtype, device=device)
    return buf[guard:guard + n].view(shape), buf


def check_guards(t, buf, guard=GUARD, what="output", inside_nan_ok=False):
    """The canaries around ``t`` are intact and (unless allowed) no NaN is left inside ``t``."""
    torch.cuda.synchronize()
    if buf.dtype == torch.uint8:
        intact = bool((buf[:guard] == 0xFF).all()) and bool((buf[-guard:] == 0xFF).all())
    else:
        intact = bool(torch.isnan(buf[:guard]).all()) and bool(torch.isnan(buf[-guard:]).all())
    assert intact, f"{what}: a kernel wrote outside the tensor (guard region changed)"
    if not inside_nan_ok and t.dtype != torch.uint8:
        assert not bool(torch.isnan(t).any()), f"{what}: NaN canary left inside (element not written)"


def guarded_workspace(nbytes, device="cuda"):
    """A workspace of ``nbytes`` (256-byte aligned start) with canary bytes after it and before it."""
    t, buf = guarded((max(int(nbytes), 256),), torch.uint8, device, guard=GUARD * 4)
    return t, buf


class GuardedWorkspaces:
    """A workspace factory for the binding (``workspace=``) that keeps every buffer it hands out,
    so that a test can check their guard bytes after the calls."""

    def __init__(self):
        self.made = []

    def __call__(self, nbytes):
        t, buf = guarded_workspace(nbytes)
        self.made.append((t, buf))
        return t

    def check(self, what="workspace"):
        for t, buf in self.made:
            check_guards(t, buf, guard=GUARD * 4, what=what)
