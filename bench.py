#!/usr/bin/env python
"""Benchmark of the Sketch Attention forward (history tokens/s, fraction of bf16 peak).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    torchrun --nproc-per-node N bench.py --gpus N ...      (one process per GPU)

Workload: 40 users of 100,000 tokens each (config 5's forward: the shape on which the
60%-of-peak target is stated), d=128, k=1024, bf16 inputs / fp32 accumulate, synthetic
N(0,1) inputs from the seeded generator. One step = one sa_sketch_forward call over the
batch (schedule, fold, tcgen05 forward, finalize). Inputs stay resident in HBM during
the timed region, and X (1.02 GB) is larger than L2. With N GPUs each rank runs its own
batch (users are independent; no collective on the data path), so scaling is weak and
`value` is total tokens / max-over-ranks time.

The JSON line also carries:
  roofline      the tcgen05 forward kernels alone (the clustered grid and, on the SMs
                clusters of 8 leave free, the helper grid beside it): algorithmic FLOP
                per launch (4*k*d per token) / their CUDA-event duration vs the measured
                bf16 peak
  e2e           the same metric through the C ABI with host buffers
                (sa_sketch_forward_host): the per-step H2D of X and offsets and the D2H
                of sketch and mass inside the timed region
  cpu_baseline  the fp64 oracle on the host cores, on a bounded sample (rank 0, N=1)
  clocks        SM clock median and throttle reasons sampled during the timed region
  backward      sa_sketch_backward on the same batch and on config 3
  other_workloads  (one GPU) the forward on one 100K-token user, on config 3 (40 users
                of 10K-100K tokens) and on the 300-user serving batch at k = 256 ... 2048:
                step and kernel times, kernel fraction of the bf16 peak
`--impl reference` times the oracle (the reference arm here) on the same config.
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "history tokens/s of SA sketch (k=1024,d=128) and % of bf16 tensor-core peak"
UNIT = "tokens/s"
WORKLOAD = ("R=40 users x n=100,000 (config 5's forward: the shape the 60%-of-peak target is "
            "stated on), d=128, k=1024, bf16 in / fp32 accumulate, forward")
HEADLINE_USERS, HEADLINE_N = 40, 100000
FALLBACK_PEAK_TFLOPS = 1590.0
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "sa_fwd_sm100_40x100k.md")
KERNEL_SOURCES = [os.path.join(ROOT, "prototype_sketch_attention_b200", "csrc", f)
                  for f in ("sa_fwd_sm100.cu", "sa_common.cuh")]


def kernel_source_hash() -> str:
    """Hash of the hot kernel's code with comments and blank space removed, so that a
    committed profile summary stays matched across comment-only edits."""
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(f) as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        h.update("\n".join(ln.strip() for ln in text.splitlines() if ln.strip()).encode())
    return h.hexdigest()[:16]


def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            j = json.load(f)
        return float(j["bf16_tflops"]), "measured (MEASURED_PEAKS.json bf16_tflops, burst)"
    except Exception:
        return FALLBACK_PEAK_TFLOPS, "fallback (1.59 PFLOP/s, profiling recipe)"


DATASHEET_BF16_TFLOPS = 2250.0  # B200 dense bf16, for context beside the measured peak


def sustained_peak():
    """The measured bf16 GEMM rate held for seconds under the power cap (None if absent)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops_sustained"])
    except Exception:
        return None


def measured_hbm() -> float:
    """The measured copy bandwidth in GB/s (the profiling recipe's 6.65 TB/s if absent)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"])
    except Exception:
        return 6650.0


def profiled_traffic():
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the
    current kernel source (null otherwise)."""
    try:
        text = open(PROFILE_SUMMARY).read()
    except OSError:
        return None
    vals = {}
    for line in text.splitlines():
        if ":" in line and line.strip().startswith(("source_sha256", "dram_bytes_per_launch")):
            key, v = line.strip().split(":", 1)
            vals[key.strip()] = v.strip().strip("`")
    if vals.get("source_sha256") != kernel_source_hash():
        return None
    try:
        return int(float(vals["dram_bytes_per_launch"]))
    except (KeyError, ValueError):
        return None


def event_ms(a, b) -> float:
    """Milliseconds between two torch.cuda.Event objects that the library recorded
    itself (cudaEventRecord inside libsa_sketch.so), read through the CUDA runtime."""
    import ctypes
    lib = ctypes.CDLL("libcudart.so.12")
    ms = ctypes.c_float(0.0)
    rc = lib.cudaEventElapsedTime(ctypes.byref(ms), ctypes.c_void_p(a.cuda_event),
                                  ctypes.c_void_p(b.cuda_event))
    if rc != 0:
        raise RuntimeError(f"cudaEventElapsedTime failed: {rc}")
    return float(ms.value)


# ------------------------------------------------------------------ clocks
THROTTLE_BITS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
                 0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
                 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}


class ClockSampler:
    """Samples SM clock and clock-event reasons with NVML while the timed region runs."""

    def __init__(self, torch_device_index: int):
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._h = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(torch_device_index)
            bus = "%08x:%02x:%02x.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
            try:
                self._h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(torch_device_index)
            self._nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: clocks stay empty and are reported as such
            self.error = repr(e)
        self._t = threading.Thread(target=self._run, daemon=True)

    def _reasons(self):
        nv = self._nv
        for fn in ("nvmlDeviceGetCurrentClocksEventReasons", "nvmlDeviceGetCurrentClocksThrottleReasons"):
            if hasattr(nv, fn):
                return getattr(nv, fn)(self._h)
        return 0

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
                self.reasons |= int(self._reasons())
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self._h is not None:
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._t.is_alive():
            self._t.join()

    def summary(self) -> dict:
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        names = [n for b, n in THROTTLE_BITS.items() if self.reasons & b and n != "gpu_idle"]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


# ------------------------------------------------------------------ CPU oracle baseline
def oracle_sample(w, S: int):
    """The first S tokens of the batch (spanning users 0, 1, ... with their own offsets),
    as fp64 arrays for the oracle."""
    import numpy as np
    off = w.offsets.numpy()
    S = int(min(S, off[-1]))
    cut = np.minimum(off, S)
    last = int(np.searchsorted(cut, S, side="left"))  # users [0, last) hold the sample
    sub_off = cut[:last + 1].astype(np.int64) if last > 0 else np.array([0, S], dtype=np.int64)
    return (w.X[:S].double().numpy(), sub_off, w.P.double().numpy(), w.Wk.double().numpy(),
            w.Wv.double().numpy())


def oracle_sample_rate(w, target_s: float, max_tokens: int = 2_000_000, keep: dict | None = None):
    """Times the fp64 oracle on the first S tokens of the batch (S sized for ~target_s of
    wall time). Returns (tokens/s, tokens, seconds, threads, users); `keep`, if given,
    receives the timed run's outputs and sample offsets."""
    import oracle
    threads = os.cpu_count() or 1

    def run(S):
        X, off, P, Wk, Wv = oracle_sample(w, S)
        t0 = time.perf_counter()
        res = oracle.forward(X, off, P, Wk, Wv, nthreads=threads)
        return time.perf_counter() - t0, len(off) - 1, res, off

    probe = 8192
    tp = run(probe)[0]
    S = int(min(w.n_total, max_tokens, max(probe, probe * target_s / max(tp, 1e-6))))
    t, users, res, off = run(S)
    if keep is not None:
        keep.update(res=res, off=off)
    used = min(threads, math.ceil(S / 1024))  # the oracle parallelises over 1024-token chunks
    return S / t, S, t, used, users


def sampled_parity(w, gpu_out: dict, keep: dict) -> dict:
    """The GPU forward's sketch and mass against the oracle's, on the users that lie
    wholly inside the oracle's timed sample (relative L2 and max |error| per user)."""
    import numpy as np
    off = w.offsets.numpy()
    whole = [u for u in range(len(keep["off"]) - 1) if off[u + 1] <= keep["off"][-1]]
    if not whole:
        return {"users": []}
    sk = gpu_out["sketch"][whole].double().cpu().numpy()
    ms = gpu_out["mass"][whole].double().cpu().numpy()
    rs, rm = keep["res"]["sketch"][whole], keep["res"]["mass"][whole]
    rel = lambda a, b: float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))
    return {"users": whole,
            "sketch_rel_l2_max": max(rel(sk[i], rs[i]) for i in range(len(whole))),
            "sketch_max_abs": float(np.abs(sk - rs).max()),
            "mass_rel_l2_max": max(rel(ms[i], rm[i]) for i in range(len(whole))),
            "tolerance": {"rel_l2": 1e-2, "max_abs": 5e-2}}


# ------------------------------------------------------------------ other workloads
OTHER_WORKLOADS = (
    (2, None, "1 user, n=100,000, d=128, k=1024, bf16 in / fp32 accumulate, forward"),
    (3, None, "config3: R=40 users, n~U[10000,100000], d=128, k=1024, bf16 in / fp32 "
              "accumulate, forward"),
) + tuple(
    (4, kk, f"serving batch: R=300 users, n~logU[1000,100000], d=128, k={kk}, bf16 in / "
            "fp32 accumulate, forward") for kk in (256, 512, 1024, 2048))


def time_other_workloads(binding, inputs, dev, steps: int, peak: float) -> list:
    """The single user of 100K tokens, the 40 x 100K batch and the 300-user serving
    batch at each k, each timed like the main workload (kernel events from the library,
    step events around each call) with a 256 MB L2 flush between steps outside the timed
    events. Reported beside the headline; a failure here is reported, not raised."""
    import torch
    out = []
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for idx, kk, desc in OTHER_WORKLOADS:
        try:
            w = inputs.make_config(idx, k=kk, with_grad=False)
            X, off = w.X.to(dev), w.offsets.to(dev)
            P, Wk, Wv = w.P.to(dev), w.Wk.to(dev), w.Wv.to(dev)
            o = binding.forward(X, off, P, Wk, Wv, want_lse=False, want_xsketch=False)
            for _ in range(3):
                binding.forward(X, off, P, Wk, Wv, ws=o["_ws"], out=o)
            torch.cuda.synchronize()
            stream = torch.cuda.current_stream()
            ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
            for e4 in ev:  # materialise the CUDA events before the library records them
                for e in e4:
                    e.record(stream)
            torch.cuda.synchronize()
            for e4 in ev:
                flush.zero_()
                e4[0].record(stream)
                binding.sa_sketch_profile_events(e4[2].cuda_event, e4[3].cuda_event)
                binding.forward(X, off, P, Wk, Wv, ws=o["_ws"], out=o)
                e4[1].record(stream)
            torch.cuda.synchronize()
            binding.sa_sketch_profile_events(None, None)
            st = binding.device_status(o["_ws"])
            if st != 0:
                raise RuntimeError(binding.sa_status_string(st))
            step_ms = sum(e4[0].elapsed_time(e4[1]) for e4 in ev) / steps
            kern_ms = sum(event_ms(e4[2], e4[3]) for e4 in ev) / steps
            graph_ms = graph_replay_ms(lambda: binding.forward(X, off, P, Wk, Wv, ws=o["_ws"], out=o),
                                       steps, flush)
            n = w.n_total
            achieved = 4.0 * w.k * w.d * n / (kern_ms / 1e3) / 1e12
            out.append({"workload": desc, "n_total": n, "steps": steps,
                        "ms_per_step": step_ms, "tokens_per_s": n / (step_ms / 1e3),
                        "graph_ms_per_step": graph_ms,
                        "kernel_ms": kern_ms, "kernel_tflops": achieved,
                        "kernel_frac": achieved / peak, "l2": "256 MB flush between steps"})
            del X, off, P, Wk, Wv, o
        except Exception as e:  # reported beside the headline, never fatal to it
            binding.sa_sketch_profile_events(None, None)
            out.append({"workload": desc, "error": repr(e)[:300]})
    del flush
    torch.cuda.synchronize()
    return out


RECENT_L, RECENT_CANDIDATES = 10000, 300


def graph_replay_ms(fn, steps: int, flush=None) -> float:
    """fn captured once into a CUDA graph (after a warm-up call on a side stream), then the
    mean time of its replays from CUDA events (with the L2 flush between replays, outside
    the events, when given). The library's calls allocate nothing and never synchronise,
    so they capture as plain kernel and memset nodes."""
    import torch
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    for _ in range(3):
        g.replay()
    stream = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    torch.cuda.synchronize()
    for a, b in ev:
        if flush is not None:
            flush.zero_()
        a.record(stream)
        g.replay()
        b.record(stream)
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in ev) / steps


def time_recent_branch(binding, dev, X, off, peak: float, steps: int = 20) -> dict:
    """The recent branch of STCA on the headline batch: every user's 300 candidates attend
    over the user's last 10K history rows, read in place from the resident X. Forward
    (sa_stca_keys_forward: folds, the flash kernel, the W_V projection) and backward
    (sa_stca_keys_backward) per step, with a 256 MB L2 flush between forward steps outside
    the timed events (the 40 users' recent rows, 102 MB, would otherwise stay in L2).
    Reported beside the headline; a failure here is reported, not raised."""
    import torch
    try:
        gen = torch.Generator().manual_seed(77)
        R, d = off.numel() - 1, X.shape[1]
        n_cand = R * RECENT_CANDIDATES
        coff = torch.arange(0, n_cand + 1, RECENT_CANDIDATES, dtype=torch.int64).to(dev)
        Q = torch.randn(n_cand, d, generator=gen).to(torch.bfloat16).to(dev)
        Wq, WK, WV = ((torch.randn(d, d, generator=gen) / d ** 0.5).to(torch.bfloat16).to(dev)
                      for _ in range(3))
        G = torch.randn(n_cand, d, generator=gen).to(dev)
        kb, ke = binding.recent_ranges(off, RECENT_L)
        pairs = int((ke - kb).sum().item()) * RECENT_CANDIDATES
        o = binding.stca_keys_forward(Q, coff, X, kb, ke, Wq, WK, WV)
        g = binding.stca_keys_backward(Q, coff, X, kb, ke, Wq, WK, WV, G)
        for _ in range(3):
            binding.stca_keys_forward(Q, coff, X, kb, ke, Wq, WK, WV, ws=o["_ws"])
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        stream = torch.cuda.current_stream()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
        for e4 in ev:  # materialise the CUDA events before the library records them
            for e in e4:
                e.record(stream)
        torch.cuda.synchronize()
        for e4 in ev:
            flush.zero_()
            e4[0].record(stream)
            binding.sa_sketch_profile_events(e4[2].cuda_event, e4[3].cuda_event)
            binding.stca_keys_forward(Q, coff, X, kb, ke, Wq, WK, WV, ws=o["_ws"])
            e4[1].record(stream)
        torch.cuda.synchronize()
        binding.sa_sketch_profile_events(None, None)
        st = binding.device_status(o["_ws"])
        if st != 0:
            raise RuntimeError(binding.sa_status_string(st))
        fwd_ms = sum(e4[0].elapsed_time(e4[1]) for e4 in ev) / steps
        kern_ms = sum(event_ms(e4[2], e4[3]) for e4 in ev) / steps
        fwd_graph_ms = graph_replay_ms(
            lambda: binding.stca_keys_forward(Q, coff, X, kb, ke, Wq, WK, WV, ws=o["_ws"]), steps,
            flush)
        nb = 5
        bev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(nb)]
        for e4 in bev:
            for e in e4:
                e.record(stream)
        binding.stca_keys_backward(Q, coff, X, kb, ke, Wq, WK, WV, G, ws=g["_ws"])
        torch.cuda.synchronize()
        for e4 in bev:
            flush.zero_()
            e4[0].record(stream)
            binding.sa_sketch_profile_events(e4[2].cuda_event, e4[3].cuda_event)
            binding.stca_keys_backward(Q, coff, X, kb, ke, Wq, WK, WV, G, ws=g["_ws"])
            e4[1].record(stream)
        torch.cuda.synchronize()
        binding.sa_sketch_profile_events(None, None)
        st = binding.device_status(g["_ws"])
        if st != 0:
            raise RuntimeError(binding.sa_status_string(st))
        bwd_ms = sum(e4[0].elapsed_time(e4[1]) for e4 in bev) / nb
        bwd_kern_ms = sum(event_ms(e4[2], e4[3]) for e4 in bev) / nb
        # the same backward adding into an existing history gradient (no zeroing of X's rows)
        dX = torch.zeros(X.shape, dtype=torch.float32, device=dev)
        binding.stca_keys_backward(Q, coff, X, kb, ke, Wq, WK, WV, G, dKx=dX, ws=g["_ws"])
        aev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(nb)]
        torch.cuda.synchronize()
        for a0, a1 in aev:
            flush.zero_()
            a0.record(stream)
            binding.stca_keys_backward(Q, coff, X, kb, ke, Wq, WK, WV, G, dKx=dX, ws=g["_ws"])
            a1.record(stream)
        torch.cuda.synchronize()
        acc_ms = sum(a0.elapsed_time(a1) for a0, a1 in aev) / nb
        del dX
        flop = 4.0 * d * pairs  # scores and weighted sum, per (candidate, key) pair
        achieved = flop / (kern_ms / 1e3) / 1e12
        bflop = 10.0 * d * pairs  # scores, dP, G1 and dKx (two terms), per pair
        bachieved = bflop / (bwd_kern_ms / 1e3) / 1e12
        return {"workload": f"{R} users x {RECENT_CANDIDATES} candidates over the last "
                            f"{RECENT_L} of {X.shape[0] // R} history rows each, d={d}",
                "pairs": pairs, "forward_ms": fwd_ms, "forward_graph_ms": fwd_graph_ms,
                "pairs_per_s": pairs / (fwd_ms / 1e3),
                "kernel": "stca_keys_fwd_kernel<128>", "kernel_ms": kern_ms,
                "kernel_tflops": achieved, "kernel_frac": achieved / peak,
                "flop_per_pair": 4 * d,
                "tensor_flop_per_pair": 6 * d,  # the score MMA runs twice (Q' hi and lo)
                "backward_ms": bwd_ms, "backward_accumulate_ms": acc_ms,
                "backward_kernel": "stca_keys_bwd_kernel<128>",
                "backward_kernel_ms": bwd_kern_ms, "backward_kernel_tflops": bachieved,
                "backward_kernel_frac": bachieved / peak, "backward_flop_per_pair": 10 * d,
                "note": "forward: M and Q' folds, flash kernel, O' split, O' W_V GEMM; the "
                        "backward recomputes the forward, then dO' and dW_V GEMMs, the tcgen05 "
                        "kernel (G1, dKx), dQ and the weight gradients",
                "l2": "256 MB flush between steps"}
    except Exception as e:  # reported beside the headline, never fatal to it
        binding.sa_sketch_profile_events(None, None)
        return {"error": repr(e)[:300]}


def time_sketch_branch(binding, dev, sketch, peak: float, hbm_gbs: float, steps: int = 20) -> dict:
    """The sketch branch of STCA with MRLB on the headline batch's sketches (40 users,
    k = 1024, d = 128): every user's 300 candidates read that user's one sketch
    (sa_stca_forward, sa_stca_backward), and the sketch cache codec packing and unpacking
    those 40 sketches (FP8 E4M3 with row scales). A 256 MB L2 flush precedes every timed
    call, outside its events. Reported beside the headline; a failure here is reported,
    not raised."""
    import torch
    out = {}
    try:
        gen = torch.Generator().manual_seed(78)
        R, k, d = sketch.shape
        n_cand = R * RECENT_CANDIDATES
        coff_h = torch.arange(0, n_cand + 1, RECENT_CANDIDATES, dtype=torch.int64)
        coff = coff_h.to(dev)
        Q = torch.randn(n_cand, d, generator=gen).to(torch.bfloat16).to(dev)
        Wq, WK, WV = ((torch.randn(d, d, generator=gen) / d ** 0.5).to(torch.bfloat16).to(dev)
                      for _ in range(3))
        G = torch.randn(n_cand, d, generator=gen).to(dev)
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        stream = torch.cuda.current_stream()

        def timed(fn, n):
            for _ in range(3):
                fn()
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(n)]
            torch.cuda.synchronize()
            for a, b in ev:
                flush.zero_()
                a.record(stream)
                fn()
                b.record(stream)
            torch.cuda.synchronize()
            return sum(a.elapsed_time(b) for a, b in ev) / n

        o = binding.stca_forward(Q, coff, sketch, Wq, WK, WV)
        g = binding.stca_backward(Q, coff, sketch, Wq, WK, WV, G, cand_offsets_host=coff_h)
        fwd_ms = timed(lambda: binding.stca_forward(Q, coff, sketch, Wq, WK, WV, ws=o["_ws"]), steps)
        bwd_ms = timed(lambda: binding.stca_backward(Q, coff, sketch, Wq, WK, WV, G,
                                                     cand_offsets_host=coff_h, ws=g["_ws"]), 5)
        fwd_graph_ms = graph_replay_ms(
            lambda: binding.stca_forward(Q, coff, sketch, Wq, WK, WV, ws=o["_ws"]), steps, flush)
        bwd_graph_ms = graph_replay_ms(
            lambda: binding.stca_backward(Q, coff, sketch, Wq, WK, WV, G, cand_offsets_host=coff_h,
                                          ws=g["_ws"]), 5, flush)
        for ws in (o["_ws"], g["_ws"]):
            st = binding.device_status(ws)
            if st != 0:
                raise RuntimeError(binding.sa_status_string(st))
        flop = 4.0 * k * d * n_cand  # scores and weighted sum over the k rows, per candidate
        out["stca_sketch"] = {
            "workload": f"{R} users x {RECENT_CANDIDATES} candidates over each user's k={k} x "
                        f"d={d} sketch",
            "forward_ms": fwd_ms, "forward_tflops": flop / (fwd_ms / 1e3) / 1e12,
            "forward_frac": flop / (fwd_ms / 1e3) / 1e12 / peak,
            "backward_ms": bwd_ms,
            "forward_graph_ms": fwd_graph_ms, "backward_graph_ms": bwd_graph_ms,
            "note": "the recent branch's kernels with the bf16 sketch rows as the keys; "
                    "4kd FLOP per candidate; one sketch read per user",
            "l2": "256 MB flush before every timed call"}
    except Exception as e:
        out["stca_sketch"] = {"error": repr(e)[:300]}
    try:
        rows = sketch.numel() // sketch.shape[-1]
        pk = binding.sketch_pack(sketch)
        pack_ms = timed(lambda: binding.sketch_pack(sketch), steps)
        unpack_ms = timed(lambda: binding.sketch_unpack(pk), steps)
        d = sketch.shape[-1]
        pack_bytes = rows * d * 4 + rows * d + rows * 4      # fp32 in; codes and scales out
        out["codec"] = {
            "workload": f"FP8 E4M3 with row scales, {rows} rows x d={d} (the 40 sketches)",
            "pack_ms": pack_ms, "unpack_ms": unpack_ms,
            "pack_gbs": pack_bytes / (pack_ms / 1e3) / 1e9,
            "unpack_gbs": pack_bytes / (unpack_ms / 1e3) / 1e9,
            "pack_frac_of_hbm": pack_bytes / (pack_ms / 1e3) / 1e9 / hbm_gbs,
            "bytes_per_call": pack_bytes,
            "note": "one kernel each; 21 MB moved, so launch latency is a visible share",
            "l2": "256 MB flush before every timed call"}
    except Exception as e:
        out["codec"] = {"error": repr(e)[:300]}
    return out


# ------------------------------------------------------------------ reference arm
def run_reference(args) -> None:
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from prototype_sketch_attention_b200 import inputs
    w = inputs.make_config(5, with_grad=False)
    import numpy as np
    import oracle
    threads = os.cpu_count() or 1
    # each step: the oracle on a bounded sample of the batch (whole run within a few minutes)
    per_step_target = max(0.5, 150.0 / max(1, args.steps + args.warmup))
    rate, S, t, used, users = oracle_sample_rate(w, per_step_target)
    X, off, P, Wk, Wv = oracle_sample(w, S)
    for _ in range(args.warmup):
        oracle.forward(X, off, P, Wk, Wv, nthreads=threads)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.forward(X, off, P, Wk, Wv, nthreads=threads)
        times.append(time.perf_counter() - t0)
    step_s = sum(times) / len(times)
    value = S / step_s
    sample = (f"first {S} tokens of the 40 x 100K batch ({users} users) per step (k=1024, "
              "d=128), fp64 oracle")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "n_total_per_gpu": w.n_total, "R": w.R, "k": w.k, "d": w.d,
                   "sample_tokens": S, "parallelism": "host cores, rank 0 only"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": min(threads, math.ceil(S / 1024)),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ our arm
def run_ours(args) -> None:
    import torch
    import torch.distributed as dist
    from prototype_sketch_attention_b200 import binding, inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}: launch N>1 with torchrun")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    w = inputs.make_config(5, with_grad=False)
    if rank > 0:  # each rank its own batch of 40 users of 100K tokens (different draws)
        w = inputs.make_workload([HEADLINE_N] * HEADLINE_USERS, 128, 1024, "bf16",
                                 seed=1005 + 7919 * rank, name="config5")
    X = w.X.to(dev)
    off = w.offsets.to(dev)
    P, Wk, Wv = w.P.to(dev), w.Wk.to(dev), w.Wv.to(dev)
    n_total, d, k, R = w.n_total, w.d, w.k, w.R
    out = binding.forward(X, off, P, Wk, Wv)
    ws = out["_ws"]
    st = binding.device_status(ws)
    if st != 0:
        raise SystemExit(f"forward failed on device: {binding.sa_status_string(st)}")
    stream = torch.cuda.current_stream()

    def step():
        binding.forward(X, off, P, Wk, Wv, ws=ws, out=out)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()

    ev_k = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(args.steps)]
    for a, b in ev_k:  # torch creates the CUDA event on first record: materialise the handles
        a.record(stream)
        b.record(stream)
    torch.cuda.synchronize()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        t_start.record(stream)
        for i in range(args.steps):
            binding.sa_sketch_profile_events(ev_k[i][0].cuda_event, ev_k[i][1].cuda_event)
            step()
        t_end.record(stream)
        torch.cuda.synchronize()
    binding.sa_sketch_profile_events(None, None)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    elapsed_ms = t_start.elapsed_time(t_end)
    kern_ms = sum(event_ms(a, b) for a, b in ev_k) / args.steps
    st = binding.device_status(ws)
    if st != 0:
        raise SystemExit(f"forward failed on device: {binding.sa_status_string(st)}")

    # ---- e2e through the C ABI with HOST buffers: sa_sketch_forward_host takes pinned
    # host X and offsets and writes pinned host sketch and mass; it cuts the users into
    # parts, so each part's host-to-device copy overlaps the previous part's forward.
    Xh = w.X.pin_memory()
    offh = w.offsets.pin_memory()
    e2e_state = {}
    e2e_steps = max(3, min(args.steps, 20))

    def e2e_step():
        binding.forward_from_host(Xh, offh, P, Wk, Wv, chunks=4, state=e2e_state)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps

    # ---- the backward (bf16 tensor-core path, single-pass kernel), reported alongside: on
    # the headline batch and on config 3, the training batch with ragged lengths
    bwd = None
    if not args.no_backward and world == 1:
        def time_backward(Xb, offb, fwd_out, nb=5):
            gen = torch.Generator().manual_seed(4242)
            G = torch.randn(fwd_out["sketch"].shape, generator=gen).to(dev)
            bout = binding.backward(Xb, offb, P, Wk, Wv, fwd_out, G)
            bws = bout["_ws"]
            for _ in range(2):
                binding.backward(Xb, offb, P, Wk, Wv, fwd_out, G, ws=bws)
            torch.cuda.synchronize()
            b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            b0.record(stream)
            for _ in range(nb):
                binding.backward(Xb, offb, P, Wk, Wv, fwd_out, G, ws=bws)
            b1.record(stream)
            torch.cuda.synchronize()
            st = binding.device_status(bws)
            if st != 0:
                raise SystemExit(f"backward failed on device: {binding.sa_status_string(st)}")
            ms = b0.elapsed_time(b1) / nb
            n = Xb.shape[0]
            return {"ms": ms, "tokens_per_s": n / (ms / 1e3),
                    "tflops_algorithmic": 10.0 * k * d * n / (ms / 1e3) / 1e12,
                    "frac_of_measured_peak": 10.0 * k * d * n / (ms / 1e3) / 1e12 / measured_peak()[0]}
        bwd = time_backward(X, off, out)
        bwd["workload"] = "the headline batch (40 x 100K tokens)"
        w3 = inputs.make_config(3, with_grad=False)
        X3, off3 = w3.X.to(dev), w3.offsets.to(dev)
        out3 = binding.forward(X3, off3, P, Wk, Wv)
        bwd["config3"] = time_backward(X3, off3, out3)
        bwd["config3"]["workload"] = "config3: R=40, n~U[10000,100000], 1,768,341 tokens"
        bwd["note"] = ("sa_sketch_backward (prep, Gh GEMM, dW_v GEMM, dX zeroing, the single-"
                       "pass kernel, tail), dL/dsketch ~ N(0,1); 10kd FLOP per token")
        del X3, off3, out3

    # ---- max over ranks
    t = torch.tensor([elapsed_ms, e2e_ms, kern_ms, float(n_total)], dtype=torch.float64, device=dev)
    if world > 1:
        tmax = t[:3].clone()
        dist.all_reduce(tmax, op=dist.ReduceOp.MAX)
        tot = t[3:].clone()
        dist.all_reduce(tot, op=dist.ReduceOp.SUM)
        elapsed_ms, e2e_ms, kern_ms = tmax.tolist()
        total_tokens = tot.item()
    else:
        total_tokens = float(n_total)
    ms_per_step = elapsed_ms / args.steps
    value = total_tokens / (ms_per_step / 1e3)
    peak, peak_src = measured_peak()
    flop_per_launch = 4.0 * k * d * n_total
    achieved = flop_per_launch / (kern_ms / 1e3) / 1e12
    n_clusters, cluster_size, n_helpers, helper_share = binding.forward_grid(k, d)
    step_tflops = 4.0 * k * d * total_tokens / (ms_per_step / 1e3) / 1e12
    h2d = X.numel() * X.element_size() + off.numel() * 8
    d2h = R * k * d * 4 + R * k * 4  # sketch and mass back to the host

    others = None
    if world == 1 and not args.no_other_workloads:
        others = time_other_workloads(binding, inputs, dev, max(3, min(args.steps, 50)), peak)

    recent = sketch_branch = None
    if world == 1 and not args.no_other_workloads:
        recent = time_recent_branch(binding, dev, X, off, peak)
        sketch_branch = time_sketch_branch(binding, dev, out["sketch"], peak, measured_hbm())

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        keep = {}
        rate, S, secs, used, users = oracle_sample_rate(w, args.cpu_seconds, keep=keep)
        cpu = {"value": rate, "unit": UNIT, "cores": used, "kind": "oracle",
               "sample": f"first {S} tokens of the 40 x 100K batch ({users} users; k=1024, d=128), "
                         f"fp64 oracle, {secs:.1f} s wall"}
        try:  # the same oracle run checks the timed forward's output on those users
            cpu["parity_sampled"] = sampled_parity(w, out, keep)
        except Exception as e:
            cpu["parity_sampled"] = {"error": repr(e)[:300]}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD,
                   "n_total_per_gpu": n_total, "R": R, "k": k, "d": d,
                   "l2": "inputs larger than L2 (X is %.0f MB per GPU)" % (h2d / 1e6),
                   "parallelism": f"users sharded, {world} independent batch(es)"},
        "pct_of_peak": step_tflops / peak,
        "step_tflops": step_tflops,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": profiled_traffic(),
                     "kernel": "sa_fwd_sm100_kernel<128,4,1> (%d clusters of %d) + "
                               "sa_fwd_sm100_helper_kernel<128> (%d CTAs, %d/1024 of the tiles), "
                               "concurrent" % (n_clusters, cluster_size, n_helpers, helper_share),
                     "kernel_ms": kern_ms,
                     "peak_source": peak_src, "flop_per_launch": flop_per_launch,
                     "frac_of_sustained": (achieved / sustained_peak()
                                           if sustained_peak() else None),
                     "frac_of_datasheet": achieved / DATASHEET_BF16_TFLOPS},
        "e2e": {"value": total_tokens / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        # per forward: schedule, fold, the tcgen05 kernel (and the helper grid when the
        # clusters leave SMs free), then the finalize (segment sums and the U Wv GEMM on the
        # tensor cores when k is a multiple of 128, else one kernel)
        "gpu_launches": ((5 if k % 128 == 0 else 4) + (1 if n_helpers > 0 else 0)) * args.steps,
        "clocks": clk.summary(),
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if bwd is not None and world == 1:
        line["backward"] = bwd
    if others is not None:
        line["other_workloads"] = others
    if recent is not None:
        line["stca_recent"] = recent
    if sketch_branch is not None:
        line.update(sketch_branch)
    print(json.dumps(line), flush=True)


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-backward", action="store_true", help="skip the backward timing")
    ap.add_argument("--no-other-workloads", action="store_true",
                    help="skip the 1 x 100K, 40 x 100K and serving-batch forward timings")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    args = ap.parse_args(argv)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)
    return 0


if __name__ == "__main__":
    sys.exit(main())
