#!/usr/bin/env python
"""Benchmark of blockwise causal varlen attention on B200.

One step = the whole hot path on the packed zig-zag workload: zig-zag ring forward
(planner, block forward with the online-softmax merge, finalise) and the ring
backward fed the merged out/lse (Delta preprocess, block backward, dq conversion)
over S = 16384 packed tokens (document lengths uniform in [512, 4096], multiples of
2*cp), cp = 4 virtual ranks, 32 heads, head_dim 128, bf16 inputs.

Metric: attention TFLOP/s of forward + backward, counting visible (q, k) pairs
only: 4*D*H*pairs for the forward and 10*D*H*pairs for the backward.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl cbv|reference] [--no-extra]

With N > 1 (torchrun) every rank runs its own batch (different seed) on its own GPU:
weak scaling, no data-path collective; the step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import re
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "causal varlen attn TFLOP/s fwd & fwd+bwd; decode HBM GB/s; % of B200 roofline"
MEASURES = "fwd+bwd TFLOP/s of the zig-zag ring (fused schedule), visible pairs only; fwd, decode GB/s and the other workloads under extra"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# the nominal figures the targets are stated against: dense bf16 tensor peak and HBM3e bandwidth of one B200
STATED_PEAKS = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["cbv", "reference"], default="cbv")
    p.add_argument("--seed", type=int, default=0)
    p.add_argument("--no-extra", action="store_true", help="skip the other workloads' sub-benchmarks")
    p.add_argument("--no-cpu", action="store_true", help="skip the oracle CPU baseline")
    p.add_argument("--workload", choices=["packed", "long_doc", "long_doc_small"], default="packed",
                   help="ring workload of the timed step (the headline is `packed`; the others are for profiling)")
    p.add_argument("--only", choices=["long_doc", "rank_balance", "deterministic", "cached", "paged", "decode", "merge"],
                   default=None,
                   help="run one of the sub-benchmarks alone and print its result (for profiling); no headline line")
    p.add_argument("--decode-seqs", type=int, default=8192, help="sequences of the decode sub-benchmark")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


def profile_traffic(name: str):
    """dram bytes per launch recorded in profiles/<name>.md ("dram_bytes_per_launch: N"), else None."""
    path = os.path.join(ROOT, "profiles", name + ".md")
    if not os.path.exists(path):
        return None
    m = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", open(path).read())
    return float(m.group(1)) if m else None


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and clock-event reasons sampled every 5 ms while the timed region runs.

    Reads NVML (the library nvidia-smi reports from; read-only queries) in a thread, so that
    a timed region of a few tens of milliseconds still holds several samples; falls back to
    ``nvidia-smi -lms 100`` when NVML cannot be loaded."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown", 0x4: "sw_power_cap"}

    def __init__(self, index: int):
        self.index = index
        self.rows: list[tuple[float, float, list[str]]] = []
        self.lines: list[str] = []
        self.proc = None
        self.nvml = None
        self.stop_flag = threading.Event()
        self.first = threading.Event()

    def _handle(self, nv):
        try:
            import torch

            pr = torch.cuda.get_device_properties(self.index)
            bus = f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"
            return nv.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(self.index)

    def _poll(self, nv, h):
        max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
        while not self.stop_flag.is_set():
            mhz = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
            bits = int(nv.nvmlDeviceGetCurrentClocksEventReasons(h))
            self.rows.append((mhz, max_mhz, [n for b, n in self.REASONS.items() if bits & b], time.monotonic()))
            self.first.set()
            time.sleep(0.005)

    def start(self):
        try:
            import pynvml as nv

            nv.nvmlInit()
            h = self._handle(nv)
            self.nvml = nv
            self.thread = threading.Thread(target=self._poll, args=(nv, h), daemon=True)
            self.thread.start()
            self.first.wait(timeout=5)
            return
        except Exception:
            self.nvml = None
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "100", "-i", str(self.index)], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.strip().split(",")]
            if len(parts) != 8:
                continue
            try:
                names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
                self.rows.append((float(parts[0]), float(parts[1]),
                                  [names[i] for i, v in enumerate(parts[4:8]) if v.lower() == "active"],
                                  time.monotonic()))
            except ValueError:
                continue

    def begin(self):
        """Marks the start of the timed region: earlier samples are dropped."""
        self.t_begin = time.monotonic()

    def stop(self):
        t_end = time.monotonic()
        if self.nvml is not None:
            self.stop_flag.set()
            self.thread.join(timeout=5)
            try:
                self.nvml.nvmlShutdown()
            except Exception:
                pass
            source = "nvml 5 ms"
        elif self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            source = "nvidia-smi 100 ms"
        else:
            return None
        t0 = getattr(self, "t_begin", 0.0)
        rows = [r for r in self.rows if t0 <= r[3] <= t_end]
        if not rows:
            return None
        reasons = sorted({n for _, _, r, _ in rows for n in r})
        return {"sm_mhz": float(np.median([r[0] for r in rows])), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows), "source": source}


# ----------------------------------------------------------------------------- workload
def visible_pairs(cu, window=0):
    from context_blockwise_causal_varlen_b200 import rank_pair_counts

    return int(rank_pair_counts(cu, 1, "zigzag", window).sum())


def slice_pair_counts(cu, cp):
    """Visible causal pairs of each of cp contiguous S/cp slices of the packed batch (slices cross document
    boundaries): query row i of document d sees i - cu[d] + 1 keys."""
    cu = np.asarray(cu, np.int64)
    S = int(cu[-1])
    per_q = np.concatenate([np.arange(1, int(b - a) + 1) for a, b in zip(cu[:-1], cu[1:])]) if S else np.zeros(0)
    n = S // cp
    return [int(per_q[r * n:(r + 1) * n if r < cp - 1 else S].sum()) for r in range(cp)]


def make_ring_inputs(cu, H, D, seed, device):
    from synth import torch_normal_bf16

    S = int(cu[-1])
    return [torch_normal_bf16((S, H, D), seed * 10 + i, device) for i in range(4)]  # q, k, v, dout


def timed(fn, steps, warmup, stream_events=True):
    import torch

    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        fn()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / steps


def e2e_pipelined(cbv, torch, inputs, cu, cp, steps, warmup):
    """Forward + backward through the public API with every step's inputs uploaded from pinned host memory and
    its results (out, dq, dk, dv) downloaded into pinned host memory, all inside the timed region.

    Steps are pipelined the way a serving or training loop runs them: two device buffer sets, uploads on one copy
    stream, downloads on another, compute on the current stream, so step k+1's upload and step k-1's download run
    while step k computes (the two copy directions use separate copy engines).  Returns (ms per step, bytes
    uploaded per step, bytes downloaded per step)."""
    q, k, v, do = inputs
    H = q.shape[1]
    host_in = [t.cpu().pin_memory() for t in (q, k, v, do)]
    host_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in (q, q, k, v)]  # out, dq, dk, dv
    sets = []
    for _ in range(2):
        dev_in = [torch.empty_like(t) for t in (q, k, v, do)]
        dev_out = [torch.empty_like(t) for t in (q, q, k, v)]
        lse = torch.empty((H, q.shape[0]), dtype=torch.float32, device=q.device)
        sets.append((dev_in, dev_out, lse))
    comp = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    computed = [ev(), ev()]   # the compute of the last step on set b is done (its inputs may be overwritten)
    fetched = [ev(), ev()]    # the download of the last step on set b is done (its outputs may be overwritten)
    used = [False, False]

    def step(i):
        b = i % 2
        dev_in, dev_out, lse = sets[b]
        uploaded = ev()
        with torch.cuda.stream(up):
            if used[b]:
                up.wait_event(computed[b])
            for h, d in zip(host_in, dev_in):
                d.copy_(h, non_blocking=True)
            uploaded.record(up)
        comp.wait_event(uploaded)
        if used[b]:
            comp.wait_event(fetched[b])
        dq_, dk_, dv_ = dev_out[1:]
        out, l = cbv.zigzag_ring_fwd(dev_in[0], dev_in[1], dev_in[2], cu, cp, out=dev_out[0], lse=lse)
        cbv.zigzag_ring_bwd(dev_in[3], dev_in[0], dev_in[1], dev_in[2], out, l, cu, cp, dq=dq_, dk=dk_, dv=dv_)
        computed[b].record(comp)
        with torch.cuda.stream(down):
            down.wait_event(computed[b])
            for h, d in zip(host_out, dev_out):
                h.copy_(d, non_blocking=True)
            fetched[b].record(down)
        used[b] = True

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(comp)
    up.wait_event(t0)
    for i in range(warmup, warmup + steps):
        step(i)
    for b in range(2):
        comp.wait_event(fetched[b])
    t1.record(comp)
    torch.cuda.synchronize()
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = sum(t.numel() * t.element_size() for t in host_out)
    return t0.elapsed_time(t1) / steps, h2d, d2h


def extra_benchmarks(device, pk, pk_kind, only=None, decode_seqs=8192):
    """The other workloads, one line each (not the headline); `only` selects one of them."""
    run = lambda name: only is None or only == name
    import torch

    import context_blockwise_causal_varlen_b200 as cbv
    from synth import torch_normal_bf16
    from synth.workloads import long_doc, packed_zigzag, paged_prefill, varlen_decode

    res = {}
    tf_peak = pk["bf16_tflops"]
    if run("long_doc"):
        # long single document, zig-zag and contiguous, full causal and sliding window
        for layout, window in (("zigzag", 0), ("contiguous", 0), ("zigzag", 4096)):
            w = long_doc(window=window)
            q, k, v, do = make_ring_inputs(w.cu_seqlens, w.heads, w.head_dim, 7, device)
            pairs = visible_pairs(w.cu_seqlens, window)
            st = {}

            def fwd():
                st["o"], st["l"] = cbv.zigzag_ring_fwd(q, k, v, w.cu_seqlens, w.cp, window=window, layout=layout)

            def bwd():
                cbv.zigzag_ring_bwd(do, q, k, v, st["o"], st["l"], w.cu_seqlens, w.cp, window=window, layout=layout)

            fwd()
            t_f = timed(fwd, 5, 2)
            t_b = timed(bwd, 5, 2)
            f_fwd = 4 * w.head_dim * w.heads * pairs
            f_bwd = 10 * w.head_dim * w.heads * pairs
            key = f"long_doc_S65536_cp8_H16_{layout}" + (f"_W{window}" if window else "")
            res[key] = {"fwd_tflops": f_fwd / t_f / 1e9, "bwd_tflops": f_bwd / t_b / 1e9,
                        "fwd_bwd_tflops": (f_fwd + f_bwd) / (t_f + t_b) / 1e9,
                        "fwd_bwd_frac": (f_fwd + f_bwd) / (t_f + t_b) / 1e9 / tf_peak,
                        "fwd_bwd_frac_of_stated_peak": (f_fwd + f_bwd) / (t_f + t_b) / 1e9 / STATED_PEAKS["bf16_tflops"],
                        "ms": t_f + t_b}
            del q, k, v, do, st
            torch.cuda.empty_cache()
    if run("rank_balance"):
        # each virtual rank's forward work alone (its q rows against the keys they see, one block
        # call with explicit positions), long document: zig-zag ranks do equal work, contiguous
        # ranks a growing share (the last about 2x the mean)
        w = long_doc()
        S, H, D, cp = w.total, w.heads, w.head_dim, w.cp
        q, k, v, _ = make_ring_inputs(w.cu_seqlens, H, D, 9, device)
        bal = {}
        for layout in ("zigzag", "contiguous"):
            times = []
            for r in range(cp):
                if layout == "zigzag":
                    c = S // (2 * cp)
                    parts = [(r * c, c), ((2 * cp - 1 - r) * c, c)]
                else:
                    c = S // cp
                    parts = [(r * c, c)]
                qr = torch.cat([q[a:a + n] for a, n in parts]).contiguous()
                kr = torch.cat([k[:a + n] for a, n in parts]).contiguous()
                vr = torch.cat([v[:a + n] for a, n in parts]).contiguous()
                cu_q = np.cumsum([0] + [n for _, n in parts]).astype(np.int32)
                cu_k = np.cumsum([0] + [a + n for a, n in parts]).astype(np.int32)
                qb = np.array([a for a, _ in parts], np.int32)
                kb = np.zeros(len(parts), np.int32)
                fn = lambda: cbv.attn_block_fwd(qr, kr, vr, cu_q, cu_k, q_pos_base=qb, k_pos_base=kb)
                times.append(timed(fn, 4, 2))
                del qr, kr, vr
            bal[layout] = {"rank_ms": times, "max_over_mean": max(times) / (sum(times) / len(times))}
        res[f"rank_balance_{w.name}_fwd"] = bal
        del q, k, v
        torch.cuda.empty_cache()
    if run("deterministic"):
        # deterministic backward (dq summed in 64-bit fixed point) against the default, packed workload
        w = packed_zigzag()
        q, k, v, do = make_ring_inputs(w.cu_seqlens, w.heads, w.head_dim, 41, device)
        o, l = cbv.zigzag_ring_fwd(q, k, v, w.cu_seqlens, w.cp)
        t_fast = timed(lambda: cbv.zigzag_ring_bwd(do, q, k, v, o, l, w.cu_seqlens, w.cp), 8, 3)
        t_det = timed(lambda: cbv.zigzag_ring_bwd(do, q, k, v, o, l, w.cu_seqlens, w.cp, deterministic=True), 8, 3)
        f_bwd = 10 * w.head_dim * w.heads * visible_pairs(w.cu_seqlens)
        res[f"deterministic_bwd_{w.name}"] = {"bwd_tflops": f_bwd / t_det / 1e9, "ms": t_det, "default_ms": t_fast}
        del q, k, v, do, o, l
        torch.cuda.empty_cache()
    if run("cached"):
        # EAGLE-3 cached ring on the packed workload: the sequence block plus 3 cache diagonals.  The
        # diagonals' cost is the time above the plain ring on the same sequence block, set against the
        # bytes that the two diagonal kernels must move (and the fp32 block output they add).
        w = packed_zigzag()
        nb, S, H, D = 4, w.total, w.heads, w.head_dim
        q = torch_normal_bf16((S, H, D), 31, device)
        ck = torch_normal_bf16((nb, S, H, D), 32, device)
        cv = torch_normal_bf16((nb, S, H, D), 33, device)
        do = torch_normal_bf16((S, H, D), 34, device)
        st = {}

        def cfwd():
            st["o"], st["l"] = cbv.cached_ring_fwd(q, ck, cv, w.cu_seqlens, w.cp)

        def cbwd():
            cbv.cached_ring_bwd(do, q, ck, cv, st["o"], st["l"], w.cu_seqlens, w.cp)

        def pfwd():
            st["po"], st["pl"] = cbv.zigzag_ring_fwd(q, ck[0], cv[0], w.cu_seqlens, w.cp)

        def pbwd():
            cbv.zigzag_ring_bwd(do, q, ck[0], cv[0], st["po"], st["pl"], w.cu_seqlens, w.cp)

        cfwd()
        pfwd()
        t_cf, t_cb = timed(cfwd, 8, 3), timed(cbwd, 8, 3)
        t_pf, t_pb = timed(pfwd, 8, 3), timed(pbwd, 8, 3)
        e = S * H * D
        diag_kv = 2 * (nb - 1) * S * H * D * 2
        b_fwd = e * 2 + e * 4 + diag_kv + S * H * 8 + e * 2 + e * 2  # q, o32, k/v diagonals, lse r/w, out, o32's extra write
        b_bwd = 3 * e * 2 + 2 * diag_kv + S * H * 4  # q, dO, out; k/v diagonals read, their gradients written; lse
        pairs = visible_pairs(w.cu_seqlens)
        f_all = 14 * D * H * pairs
        res[f"cached_ring_{w.name}_NB{nb}"] = {
            "fwd_bwd_tflops": f_all / (t_cf + t_cb) / 1e9, "ms": t_cf + t_cb, "plain_ms": t_pf + t_pb,
            "diag_fwd_ms": t_cf - t_pf, "diag_bwd_ms": t_cb - t_pb,
            "diag_fwd_gbs": b_fwd / max(t_cf - t_pf, 1e-6) / 1e6, "diag_bwd_gbs": b_bwd / max(t_cb - t_pb, 1e-6) / 1e6}
        del q, ck, cv, do, st
        torch.cuda.empty_cache()
    if run("paged"):
        # paged KV-parallel prefill, round-robin shards
        for window in (0, 8192):
            w = paged_prefill(window=window)
            q = torch_normal_bf16((w.hq, w.q_len, w.head_dim), 11, device)
            kc = torch_normal_bf16((w.kv_len // w.block_size, w.hkv, w.block_size, w.head_dim), 12, device)
            vc = torch_normal_bf16(kc.shape, 13, device)
            perm = w.perm.astype(np.int64)
            bt = torch.from_numpy(np.stack([perm[r::w.shards] for r in range(w.shards)]).astype(np.int32)).to(device)
            fn = lambda: cbv.kvp_segmented_prefill(q, kc, vc, bt, cbv.KV_ROUND_ROBIN, w.seg_size, None,
                                                   w.global_q_offset, window, return_lse=False)
            t = timed(fn, 10, 3)
            qpos = w.global_q_offset + np.arange(w.q_len)
            vis = np.minimum(qpos + 1, window) if window else qpos + 1
            flops = 4 * w.head_dim * w.hq * int(vis.sum())
            res[f"paged_prefill_S4096_KV32768_rr" + (f"_W{window}" if window else "")] = {
                "tflops": flops / t / 1e9, "frac": flops / t / 1e9 / tf_peak,
                "frac_of_stated_peak": flops / t / 1e9 / STATED_PEAKS["bf16_tflops"], "ms": t}
            del q, kc, vc
            torch.cuda.empty_cache()
    if run("decode"):
        # one-query GQA varlen decode
        w = varlen_decode(num_seqs=decode_seqs)
        cu_k = torch.from_numpy(w.cu_seqlens_k).to(device)
        cu_q = torch.arange(w.num_seqs + 1, dtype=torch.int32, device=device)
        tk = int(w.cu_seqlens_k[-1])
        q = torch_normal_bf16((w.num_seqs, w.hq, w.head_dim), 21, device)
        k = torch_normal_bf16((tk, w.hkv, w.head_dim), 22, device)
        v = torch_normal_bf16((tk, w.hkv, w.head_dim), 23, device)
        out = torch.empty_like(q)
        ws = torch.empty(256, dtype=torch.uint8, device=device)
        fn = lambda: cbv.varlen_decode(q, k, v, cu_q, cu_k, validate=False, out=out, workspace=ws)
        t = timed(fn, 10, 3)
        nbytes = 2 * tk * w.hkv * w.head_dim * 2 + 2 * q.numel() * 2 + 2 * cu_k.numel() * 4
        res[f"varlen_decode_N{w.num_seqs}_HQ32_HKV4"] = {"gbs": nbytes / t / 1e6, "frac": nbytes / t / 1e6 / pk["hbm_gbs"],
                                                "frac_of_stated_peak": nbytes / t / 1e6 / STATED_PEAKS["hbm_gbs"],
                                                "ms": t, "bytes": nbytes}
        del q, k, v, out
        torch.cuda.empty_cache()
    if run("merge"):
        # standalone merge at the packed workload's shapes
        S, H, D = 16384, 32, 128
        o = torch.randn((S, H, D), device=device)
        l = torch.randn((H, S), device=device)
        bo = torch.randn((S, H, D), device=device).to(torch.bfloat16)
        bl = torch.randn((H, S), device=device)
        t = timed(lambda: cbv.attn_merge(o, l, bo, bl), 20, 3)
        nbytes = S * H * (D * 4 * 2 + D * 2 + 3 * 4)
        res["merge_S16384_H32_D128"] = {"gbs": nbytes / t / 1e6, "frac": nbytes / t / 1e6 / pk["hbm_gbs"],
                                        "frac_of_stated_peak": nbytes / t / 1e6 / STATED_PEAKS["hbm_gbs"], "ms": t}
    res["peak_kind"] = f"frac: of {pk_kind}; frac_of_stated_peak: of 2250 TFLOP/s bf16 and 8000 GB/s HBM"
    return res


def cpu_baseline(cu, H, D, cp, budget_s=12.0):
    """The oracle (ring forward + merged-lse backward, fp64) on a bounded sample of the workload."""
    from threadpoolctl import threadpool_info

    from oracle import ring as R
    from synth import normal_bf16, streams

    d = int(np.argmax(np.diff(cu)))
    L = int(cu[d + 1] - cu[d])
    cu1 = np.array([0, L])
    g = streams(99, 4)
    flops = 0
    heads = 0
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < budget_s and heads < H:
        q, k, v, do = (normal_bf16(g[i], (L, 1, D)).astype(np.float64) for i in range(4))
        o, l = R.ring_fwd(q, k, v, cu1, cp, D ** -0.5)
        R.ring_bwd(do, q, k, v, o, l, cu1, cp, D ** -0.5)
        flops += 14 * D * (L * (L + 1) // 2)
        heads += 1
    dt = time.perf_counter() - t0
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s (sampled)", "cores": os.cpu_count(), "blas_threads": int(threads),
            "kind": "oracle",
            "sample": f"sampled: fp64 NumPy ring fwd+bwd of the longest document (L={L}, cp={cp}) for {heads} of {H} "
                      f"heads, {dt:.1f} s"}


# ----------------------------------------------------------------------------- reference arm
def run_reference(args):
    """The oracle, as it stands, on bounded samples of the same workload (rank 0 only)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from threadpoolctl import threadpool_info

    from oracle import ring as R
    from synth import normal_bf16, streams
    from synth.workloads import packed_zigzag

    w = packed_zigzag(args.seed)
    cu = w.cu_seqlens
    d = 0
    L = int(cu[d + 1] - cu[d])
    cu1 = np.array([0, L])
    g = streams(99, 4)
    q, k, v, do = (normal_bf16(g[i], (L, 1, w.head_dim)).astype(np.float64) for i in range(4))

    def step():
        o, l = R.ring_fwd(q, k, v, cu1, w.cp, w.head_dim ** -0.5)
        R.ring_bwd(do, q, k, v, o, l, cu1, w.cp, w.head_dim ** -0.5)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps
    flops = 14 * w.head_dim * (L * (L + 1) // 2)
    val = flops / dt / 1e12
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    sample = f"fp64 NumPy ring fwd+bwd of document 0 (L={L}, cp={w.cp}), one head per step"
    line = {"metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": w.name, "measures": MEASURES, "cp": w.cp, "heads": w.heads, "head_dim": w.head_dim,
                       "l2": "inputs larger than L2 not applicable (CPU)"},
            "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": os.cpu_count(), "blas_threads": int(threads),
                             "kind": "oracle", "sample": "sampled: " + sample},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- ranks
def rank_workload(kind: str, seed: int, rank: int):
    """The batch one rank runs.  Replicas: every rank draws its own packed batch (seed + rank) of the
    same total size, so per-rank work is fixed as ranks are added (weak scaling); the long-document
    workloads are one fixed document."""
    from synth.workloads import long_doc, packed_zigzag

    if kind == "packed":
        return packed_zigzag(seed + rank)
    if kind == "long_doc":
        return long_doc()
    return long_doc(total=16384, cp=8, heads=16)


def reduce_over_ranks(dist, torch, device, ms: float, flops: float, world: int):
    """Whole-job timing of replicas: (the slowest rank's step time, the flops of all ranks).
    Every rank takes the same collective steps (two all-reduces) in the same order."""
    if world <= 1:
        return ms, flops
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    f = torch.tensor([flops], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(f, op=dist.ReduceOp.SUM)
    return float(t.item()), float(f.item())


# ----------------------------------------------------------------------------- main arm
def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
        return
    import torch
    import torch.distributed as dist

    import context_blockwise_causal_varlen_b200 as cbv

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    pk, pk_kind = peaks()
    if args.only:
        print(json.dumps(extra_benchmarks(device, pk, pk_kind, only=args.only, decode_seqs=args.decode_seqs)), flush=True)
        if world > 1:
            dist.destroy_process_group()
        return

    w = rank_workload(args.workload, args.seed, rank)
    cu = w.cu_seqlens
    S, H, D, cp = w.total, w.heads, w.head_dim, w.cp
    q, k, v, do = make_ring_inputs(cu, H, D, args.seed + rank, device)
    pairs = visible_pairs(cu)
    f_fwd, f_bwd = 4 * D * H * pairs, 10 * D * H * pairs
    state = {}
    ev = {"f0": [], "f1": [], "b1": [], "kf": [], "kb": []}

    def mark(key):
        e = torch.cuda.Event(enable_timing=True)
        e.record()
        ev[key].append(e)

    def kernel_events(key):
        # the library records this pair around its attention-kernel launch, on the call's stream
        pair = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
        ev[key].append(pair)
        cbv.set_kernel_events(*pair)

    def step(record=False):
        if record:
            mark("f0")
            kernel_events("kf")
        state["out"], state["lse"] = cbv.zigzag_ring_fwd(q, k, v, cu, cp)
        if record:
            mark("f1")
            kernel_events("kb")
        state["grads"] = cbv.zigzag_ring_bwd(do, q, k, v, state["out"], state["lse"], cu, cp)
        if record:
            cbv.set_kernel_events()
            mark("b1")

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = ClockSampler(local)
    clocks.start()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks.begin()
    n0 = cbv.launch_count()
    t0.record()
    for _ in range(args.steps):
        step()
    t1.record()
    launches = cbv.launch_count() - n0
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = t0.elapsed_time(t1) / args.steps
    # the per-call and per-kernel durations come from a second, instrumented pass of the same steps:
    # the event records between the kernels would otherwise sit inside the timed steps
    for _ in range(args.steps):
        step(record=True)
    torch.cuda.synchronize()
    # each replica's batch has its own documents, hence its own visible-pair count
    ms, total_flops = reduce_over_ranks(dist, torch, device, ms, f_fwd + f_bwd, world)
    if world > 1:
        dist.barrier()
    fwd_ms = float(np.mean([a.elapsed_time(b) for a, b in zip(ev["f0"], ev["f1"])]))
    bwd_ms = float(np.mean([a.elapsed_time(b) for a, b in zip(ev["f1"], ev["b1"])]))
    fwd_kernel_ms = float(np.mean([a.elapsed_time(b) for a, b in ev["kf"]]))
    bwd_kernel_ms = float(np.mean([a.elapsed_time(b) for a, b in ev["kb"]]))

    # end to end through the public API with host buffers (pinned), copies inside the timed region
    e2e_ms, h2d, d2h = e2e_pipelined(cbv, torch, (q, k, v, do), cu, cp, max(6, args.steps // 2), 2)
    e2e_ms, _ = reduce_over_ranks(dist, torch, device, e2e_ms, 0.0, world)

    value = total_flops / (ms * 1e-3) / 1e12
    if rank == 0:
        # the dominant kernel: the block backward (10 of the 14 flops per pair)
        dom_ms, dom_flops, dom_name = ((bwd_kernel_ms, f_bwd, "bwd_kernel") if bwd_kernel_ms >= fwd_kernel_ms
                                       else (fwd_kernel_ms, f_fwd, "fwd_pp_kernel"))
        achieved = dom_flops / (dom_ms * 1e-3) / 1e12
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "measures": MEASURES, "tokens": S, "docs": len(cu) - 1, "cp": cp,
                       "heads": H, "head_dim": D,
                       "layout": "zigzag", "schedule": "fused", "visible_pairs_per_head": pairs,
                       "l2": f"inputs larger than L2 (q, k, v, dout {4 * S * H * D * 2 / 1e6:.0f} MB)",
                       "parallelism": f"replicas x{world}"},
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": achieved / pk["bf16_tflops"], "traffic": profile_traffic(f"{dom_name}_packed_zigzag"),
                         "kernel": dom_name, "peak_kind": f"{pk_kind} bf16 burst",
                         "stated_peak": STATED_PEAKS["bf16_tflops"],
                         "frac_of_stated_peak": achieved / STATED_PEAKS["bf16_tflops"],
                         "step_frac": value / pk["bf16_tflops"],
                         "step_frac_of_stated_peak": value / STATED_PEAKS["bf16_tflops"],
                         "duration_ms": dom_ms,
                         "note": "duration = CUDA events the library records on the call's stream right before "
                                 "and after the kernel's launch (cbv_set_kernel_events), averaged over a second "
                                 "pass of the same number of steps (the headline steps carry no such events)"},
            "phases_ms": {"fwd": fwd_ms, "bwd": bwd_ms, "fwd_kernel": fwd_kernel_ms, "bwd_kernel": bwd_kernel_ms,
                          "bwd_helpers": bwd_ms - bwd_kernel_ms},
            "e2e": {"value": total_flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
            "gpu_launches": launches,
            "clocks": clk,
            "balance": {"zigzag_pairs_per_rank": cbv.rank_pair_counts(cu, cp, "zigzag").tolist(),
                        "contiguous_per_doc_pairs_per_rank": cbv.rank_pair_counts(cu, cp, "contiguous").tolist(),
                        "contiguous_S_over_cp_slice_pairs_per_rank": slice_pair_counts(cu, cp)},
        }
        if world == 1 and not args.no_cpu:
            line["cpu_baseline"] = cpu_baseline(cu, H, D, cp)
        if world == 1 and not args.no_extra and args.workload == "packed":
            line["extra"] = extra_benchmarks(device, pk, pk_kind)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
