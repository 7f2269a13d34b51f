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
