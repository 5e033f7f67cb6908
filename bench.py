#!/usr/bin/env python3
"""Throughput of the exact attention forward on B200, one JSON line on stdout.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one ``fa_fwd`` call over the whole workload (inputs resident in
HBM).  Between timed steps the L2 is flushed by writing a 256 MiB buffer
outside the timed events.  Each step is timed with CUDA events on the
launching stream; ``ms_per_step`` is the mean, the job time is the max over
ranks.  Under torchrun every rank runs its own replica of the workload
(independent problems, no collective on the data path): weak scaling.

``--impl reference`` times the fp64 CPU oracle instead, on a bounded row
sample of the same workload per step (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from io_aware_exact_24_b200.inputs import (DECODE_WORKLOADS, WINDOW_WORKLOADS,  # noqa: E402
                                           WORKLOADS, WORKLOAD_ORDER, make_inputs,
                                           make_inputs_fp8)

METRIC = "attention fwd TFLOP/s (bf16, 1×B200) and % of dense BF16 tensor peak"
UNIT = "TFLOP/s"
DEFAULT_WORKLOAD = "causal_8000_d128"
NOMINAL_BF16_TFLOPS = 2250.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20
KERNEL_SOURCES = ["io_aware_exact_24_b200/csrc/fa_fwd_kernel.cuh",
                  "io_aware_exact_24_b200/csrc/fa_fwd_persist.cuh",
                  "io_aware_exact_24_b200/csrc/fa_decode_kernel.cuh",
                  "io_aware_exact_24_b200/csrc/sm100_ptx.cuh",
                  "io_aware_exact_24_b200/csrc/exp2_poly.cuh",
                  "io_aware_exact_24_b200/csrc/fa_api.cu"]


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            d = json.load(fh)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def load_traffic(workload: str):
    """Per-launch DRAM bytes from a committed ncu summary, if it matches the current kernel."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as fh:
        d = json.load(fh)
    e = d.get(workload)
    if not e or e.get("kernel_source_hash") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi sampled every 200 ms while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"fa_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.3)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as fh:
            for line in fh:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx.append(float(parts[2]))
                except ValueError:
                    continue
                for n, val in zip(names, parts[5:9]):
                    if val.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


def upload(x, device):
    import torch
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device).view(torch.bfloat16)
    kl = None if x["key_lens"] is None else torch.from_numpy(x["key_lens"]).to(device)
    return dev(x["q"]), dev(x["k"]), dev(x["v"]), kl


def ms_stats(per):
    """Mean, median, 10th and 90th percentile of per-launch times (ms)."""
    a = np.asarray(per, dtype=np.float64)
    return {"mean": float(a.mean()), "median": float(np.median(a)),
            "p10": float(np.percentile(a, 10)), "p90": float(np.percentile(a, 90)), "n": int(a.size)}


def time_device(w, x, steps, warmup, device, rank, world, clocks=None, flush_l2=True):
    """Mean per-launch device time (ms) of fa_fwd on resident inputs, L2 flushed between
    launches (flush_l2=False: back-to-back launches on a warm L2)."""
    import torch
    from io_aware_exact_24_b200 import fa_fwd
    q, k, v, kl = upload(x, device)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32, device=device)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()

    def launch():
        fa_fwd(q, k, v, o, lse, w.B, w.H, w.Nq, w.Nk, w.d, w.scale, w.causal, kl, stream)

    for _ in range(warmup):
        if flush_l2:
            flush.zero_()
        launch()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    if clocks:
        clocks.start()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for s, e in ev:
        if flush_l2:
            flush.zero_()
        s.record(stream)
        launch()
        e.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop() if clocks else None
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    per = [s.elapsed_time(e) for s, e in ev]
    del q, k, v, o, lse, flush
    return float(np.mean(per)), per, clk


def time_window(w, x, steps, warmup, device):
    """Mean per-call device time (ms) of fa_fwd_window / fa_fwd_bias, L2 flushed between calls."""
    import torch
    from io_aware_exact_24_b200 import fa_fwd_bias, fa_fwd_bias_table, fa_fwd_window
    from io_aware_exact_24_b200.inputs import alibi_slopes, bias_table
    q, k, v, kl = upload(x, device)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32, device=device)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()
    slopes = torch.from_numpy(alibi_slopes(w.H)).to(device) if w.alibi else None
    R = w.bias_table_radius
    table = torch.from_numpy(bias_table(w.H, R, w.seed)).to(device) if R >= 0 else None

    def launch():
        if R >= 0:
            fa_fwd_bias_table(q, k, v, o, lse, w.B, w.H, w.Nq, w.Nk, w.d, w.scale, w.causal, kl,
                              table, R, w.window_left, stream)
        elif w.alibi:
            fa_fwd_bias(q, k, v, o, lse, w.B, w.H, w.Nq, w.Nk, w.d, w.scale, w.causal, kl,
                        slopes, w.window_left, stream)
        else:
            fa_fwd_window(q, k, v, o, lse, w.B, w.H, w.Nq, w.Nk, w.d, w.scale, w.causal, kl,
                          w.window_left, stream)

    for _ in range(warmup):
        flush.zero_()
        launch()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for st, en in ev:
        flush.zero_()
        st.record(stream)
        launch()
        en.record(stream)
    torch.cuda.synchronize()
    per = [st.elapsed_time(en) for st, en in ev]
    del q, k, v, o, lse, flush
    return float(np.mean(per))


def window_table(steps, warmup, device, peak_tflops):
    """Mask variants: TFLOP/s (a window counts the visible query-key pairs only)."""
    out = {}
    for name, w in WINDOW_WORKLOADS.items():
        x = make_inputs(w)
        ms = time_window(w, x, steps, warmup, device)
        tf = w.flop / (ms / 1000.0) / 1e12
        entry = ("fa_fwd_bias_table" if w.bias_table_radius >= 0 else
                 "fa_fwd_bias" if w.alibi else "fa_fwd_window")
        out[name] = {"entry": entry, "window_left": w.window_left, "alibi": w.alibi,
                     "bias_table_radius": w.bias_table_radius, "ms": ms,
                     "tflops": tf, "roofline": {"bound": "tensor", "achieved": tf,
                                                "peak": peak_tflops, "unit": "TFLOP/s",
                                                "frac": tf / peak_tflops},
                     "flop": ("4*B*H*d*(visible query-key pairs)" if w.window_left >= 0
                              else "4*B*H*Nq*Nk*d, causal halved"),
                     "config": config_of(w, "flushed between timed launches", "single GPU")}
        del x
    return out


def time_fp8(w, x, steps, warmup, device):
    """Mean per-launch device time (ms) of fa_fwd_fp8 on resident E4M3 inputs, L2 flushed."""
    import torch
    from io_aware_exact_24_b200 import fa_fwd_fp8
    q8, k8, v8 = (torch.from_numpy(np.ascontiguousarray(x[n])).to(device) for n in ("q8", "k8", "v8"))
    kl = None if x["key_lens"] is None else torch.from_numpy(x["key_lens"]).to(device)
    o = torch.empty((w.B, w.H, w.Nq, w.d), dtype=torch.bfloat16, device=device)
    lse = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32, device=device)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()

    def launch():
        fa_fwd_fp8(q8, k8, v8, o, lse, w.B, w.H, w.Nq, w.Nk, w.d, w.scale, x["q_descale"],
                   x["k_descale"], x["v_descale"], w.causal, kl, stream)

    for _ in range(warmup):
        flush.zero_()
        launch()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for st, en in ev:
        flush.zero_()
        st.record(stream)
        launch()
        en.record(stream)
    torch.cuda.synchronize()
    per = [st.elapsed_time(en) for st, en in ev]
    del q8, k8, v8, o, lse, flush
    return float(np.mean(per))


def fp8_table(steps, warmup, device, peak_bf16_tflops):
    """E4M3 inputs (fa_fwd_fp8) on the two long workloads.  The roofline peak is the
    measured bf16 peak times the nominal FP8 / BF16 dense ratio (4.5 / 2.25 = 2)."""
    out = {}
    for name in ("causal_8000_d128", "long_16k_d64"):
        w = WORKLOADS[name]
        x = make_inputs_fp8(w)
        ms = time_fp8(w, x, steps, warmup, device)
        tf = w.flop / (ms / 1000.0) / 1e12
        peak = 2.0 * peak_bf16_tflops
        out[name] = {"entry": "fa_fwd_fp8", "dtype": "e4m3 in, bf16 out", "ms": ms, "tflops": tf,
                     "roofline": {"bound": "tensor", "achieved": tf, "peak": peak, "unit": "TFLOP/s",
                                  "frac": tf / peak,
                                  "peak_basis": "measured bf16 x nominal fp8/bf16 ratio 2"},
                     "config": config_of(w, "flushed between timed launches", "single GPU")}
        del x
    return out


def time_bwd(w, x, steps, warmup, device):
    """Mean per-call device time (ms) of fa_bwd (its three kernels) on resident inputs,
    the forward's O and LSE computed once beforehand; L2 flushed between calls."""
    import torch
    from io_aware_exact_24_b200 import fa_bwd, fa_bwd_workspace_size, fa_fwd
    from io_aware_exact_24_b200.inputs import TENSOR_DO, normal_bf16
    q, k, v, kl = upload(x, device)
    do = torch.from_numpy(normal_bf16((w.B, w.H, w.Nq, w.d), w.seed, TENSOR_DO, w.sigma).view(np.int16)).to(
        device).view(torch.bfloat16)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream()
    fa_fwd(q, k, v, o, lse, w.B, w.H, w.Nq, w.Nk, w.d, w.scale, w.causal, kl, stream)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    nb = fa_bwd_workspace_size(w.B, w.H, w.Nq, w.d)
    ws = torch.empty(nb, dtype=torch.uint8, device=device)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)

    def launch():
        fa_bwd(q, k, v, o, lse, do, dq, dk, dv, w.B, w.H, w.Nq, w.Nk, w.d, w.scale, w.causal, kl, ws, nb,
               stream)

    for _ in range(warmup):
        flush.zero_()
        launch()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for st, en in ev:
        flush.zero_()
        st.record(stream)
        launch()
        en.record(stream)
    torch.cuda.synchronize()
    per = [st.elapsed_time(en) for st, en in ev]
    del q, k, v, o, lse, do, dq, dk, dv, ws, flush
    return float(np.mean(per))


def bwd_table(steps, warmup, device, peak_tflops):
    """Backward pass (fa_bwd): FLOPs = 2.5 x the forward's (five products of the
    forward's size instead of two), tensor roofline against the measured bf16 peak."""
    out = {}
    for name in ("causal_8000_d128", "long_16k_d64"):
        w = WORKLOADS[name]
        ms = time_bwd(w, make_inputs(w), steps, warmup, device)
        flop = 2.5 * w.flop
        tf = flop / (ms / 1000.0) / 1e12
        out[name] = {"entry": "fa_bwd", "ms": ms, "tflops": tf,
                     "roofline": {"bound": "tensor", "achieved": tf, "peak": peak_tflops,
                                  "unit": "TFLOP/s", "frac": tf / peak_tflops},
                     "flop": "2.5 x (4*B*H*Nq*Nk*d, causal halved)",
                     "config": config_of(w, "flushed between timed calls", "single GPU")}
    return out


def varlen_table(steps, warmup, device, peak_tflops):
    """Packed variable-length batch with the BERT-shaped lengths of bert_padded_512
    (each sequence's queries and keys = its key length), against the padded
    fa_fwd run of the same batch.  TFLOP/s on the real (unpadded) work."""
    import torch
    from io_aware_exact_24_b200 import fa_fwd_varlen
    w = WORKLOADS["bert_padded_512"]
    x = make_inputs(w)
    lens = x["key_lens"].astype(np.int64)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    pack = lambda a: np.ascontiguousarray(np.concatenate(
        [a[b, :, :lens[b]].transpose(1, 0, 2) for b in range(w.B)], axis=0))
    dev = lambda a: torch.from_numpy(a.view(np.int16)).to(device).view(torch.bfloat16)
    q, k, v = dev(pack(x["q"])), dev(pack(x["k"])), dev(pack(x["v"]))
    o = torch.empty_like(q)
    lse = torch.empty((T, w.H), dtype=torch.float32, device=device)
    tcu = torch.from_numpy(cu).to(device)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()
    maxq = int(lens.max())

    def launch():
        fa_fwd_varlen(q, k, v, o, lse, tcu, tcu, w.B, w.H, T, T, maxq, w.d, w.scale, False, stream)

    for _ in range(warmup):
        flush.zero_()
        launch()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for st, en in ev:
        flush.zero_()
        st.record(stream)
        launch()
        en.record(stream)
    torch.cuda.synchronize()
    ms = float(np.mean([st.elapsed_time(en) for st, en in ev]))
    ms_pad, _, _ = time_device(w, x, steps, warmup, device, 0, 1)
    flop = 4.0 * w.H * w.d * float((lens * lens).sum())
    tf = flop / (ms / 1000.0) / 1e12
    return {"varlen_bert_d64": {"entry": "fa_fwd_varlen", "B": w.B, "H": w.H, "d": w.d,
                                "total_tokens": T, "max_seqlen": maxq, "ms": ms, "tflops": tf,
                                "flop": "4*H*d*sum_b len_b^2 (no padding)",
                                "roofline": {"bound": "tensor", "achieved": tf, "peak": peak_tflops,
                                             "unit": "TFLOP/s", "frac": tf / peak_tflops},
                                "padded_fa_fwd_ms": ms_pad,
                                "config": "bert_padded_512 inputs, each sequence packed to its key length"}}


def time_splitkv(w, x, steps, warmup, device, num_splits=None, flush_l2=True):
    """Mean per-call device time (ms) of fa_fwd_splitkv (partials + merge); with flush_l2 a
    256 MB buffer is written between calls (whose dirty lines the next call writes back)."""
    import torch
    from io_aware_exact_24_b200 import (fa_fwd_splitkv, fa_fwd_splitkv_workspace_size,
                                        fa_splitkv_num_splits)
    q, k, v, kl = upload(x, device)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32, device=device)
    if num_splits is None:
        num_splits = fa_splitkv_num_splits(w.B, w.H, w.Nq, w.Nk)
    ws_bytes = fa_fwd_splitkv_workspace_size(w.B, w.H, w.Nq, w.d, num_splits)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=device)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()

    def launch():
        fa_fwd_splitkv(q, k, v, o, lse, w.B, w.H, w.Nq, w.Nk, w.d, w.scale, w.causal, kl,
                       num_splits, ws, ws_bytes, stream)

    for _ in range(warmup):
        if flush_l2:
            flush.zero_()
        launch()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for st, en in ev:
        if flush_l2:
            flush.zero_()
        st.record(stream)
        launch()
        en.record(stream)
    torch.cuda.synchronize()
    per = [st.elapsed_time(en) for st, en in ev]
    del q, k, v, o, lse, flush, ws
    return float(np.mean(per)), num_splits


def kv_exceeds_l2(w):
    """K and V of the problem together larger than the L2: back-to-back calls stream them
    from HBM without a flush."""
    return 2 * w.B * w.H * w.Nk * w.d * 2 > (126 << 20)


def decode_table(steps, warmup, device, hbm_gbs):
    """Split-KV forward on the decode-shaped workloads: HBM-bound, reported in GB/s."""
    out = {}
    for name, w in DECODE_WORKLOADS.items():
        x = make_inputs(w)
        big = kv_exceeds_l2(w)
        ms, ns = time_splitkv(w, x, steps, warmup, device, flush_l2=not big)
        ms_flushed, _ = time_splitkv(w, x, steps, warmup, device) if big else (ms, ns)
        ms1, _, _ = time_device(w, x, steps, warmup, device, 0, 1)
        gbs = w.algorithmic_bytes / (ms / 1000.0) / 1e9
        l2 = ("not flushed: K/V larger than the 126 MB L2" if big else "flushed between timed launches")
        out[name] = {"entry": "fa_fwd_splitkv", "num_splits": ns, "ms": ms,
                     "algorithmic_gbs": gbs, "roofline": {"bound": "hbm", "achieved": gbs,
                                                          "peak": hbm_gbs, "unit": "GB/s",
                                                          "frac": gbs / hbm_gbs},
                     "ms_after_l2_write_flush": ms_flushed,
                     "single_pass_fa_fwd_ms": ms1,
                     "config": config_of(w, l2, "single GPU")}
        del x
    return out


def time_e2e(w, x, steps, warmup, device):
    """The same forward through the host-buffer C entry point: H2D + kernel + D2H per step."""
    import torch
    from io_aware_exact_24_b200 import fa_fwd_host, fa_fwd_host_workspace_size
    pin = lambda a: torch.from_numpy(np.ascontiguousarray(a)).pin_memory()
    hq, hk, hv = pin(x["q"]), pin(x["k"]), pin(x["v"])
    hkl = None if x["key_lens"] is None else pin(x["key_lens"])
    ho = torch.empty((w.B, w.H, w.Nq, w.d), dtype=torch.int16).pin_memory()
    hl = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32).pin_memory()
    ws_bytes = fa_fwd_host_workspace_size(w.B, w.H, w.Nq, w.Nk, w.d, hkl is not None)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()

    def step():
        fa_fwd_host(hq, hk, hv, ho, hl, w.B, w.H, w.Nq, w.Nk, w.d, w.scale, w.causal, hkl, ws,
                    ws_bytes, stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for _ in range(steps):
        step()
    e.record(stream)
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / steps
    h2d = hq.numel() * 2 + hk.numel() * 2 + hv.numel() * 2 + (0 if hkl is None else hkl.numel() * 4)
    d2h = ho.numel() * 2 + hl.numel() * 4
    del ws
    return ms, h2d, d2h


def oracle_sample_rate(w, x, target_s, rng_seed=0):
    """Oracle TFLOP/s on a random row sample of the workload sized to ~target_s seconds."""
    import oracle
    total_rows = w.B * w.H * w.Nq
    flop_per_row = w.flop / total_rows
    rng = np.random.default_rng(rng_seed)
    n = min(64, total_rows)
    rows = rng.choice(total_rows, size=n, replace=False)
    t0 = time.perf_counter()
    oracle.attn_ref_rows(x["q"], x["k"], x["v"], w.scale, rows, w.causal, x["key_lens"])
    t = max(time.perf_counter() - t0, 1e-6)
    # the first, small call also pays thread start-up: re-scale until the sample
    # takes at least 60 % of the target (at most three more calls)
    for _ in range(3):
        n = int(min(total_rows, max(n, n * target_s / t)))
        rows = rng.choice(total_rows, size=n, replace=False)
        t0 = time.perf_counter()
        oracle.attn_ref_rows(x["q"], x["k"], x["v"], w.scale, rows, w.causal, x["key_lens"])
        t = max(time.perf_counter() - t0, 1e-6)
        if t >= 0.6 * target_s or n == total_rows:
            break
    return n * flop_per_row / t / 1e12, n, t, oracle.num_threads()


def oracle_single_thread_table(target_s=4.0):
    """The oracle on one host thread on the two small workloads (a bounded row
    sample of about target_s seconds each; the tiny one is evaluated whole)."""
    import oracle
    out = {}
    threads = oracle.num_threads()
    oracle.set_num_threads(1)
    try:
        for name in ("tiny", "gpt2_causal_1k"):
            w = WORKLOADS[name]
            x = make_inputs(w)
            rate, n, t, cores = oracle_sample_rate(w, x, target_s)
            out[name] = {"value": rate, "unit": UNIT, "cores": cores,
                         "sample": f"{n} of {w.B * w.H * w.Nq} query rows ({t:.2f} s)"}
    finally:
        oracle.set_num_threads(threads)
    return out


def job_time_ms(local_ms: float, world: int, device="cpu") -> float:
    """Job time = the slowest rank's timed region (max over ranks; no data moves)."""
    if world <= 1:
        return float(local_ms)
    import torch
    t = torch.tensor([float(local_ms)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput_tflops(flop_per_step: float, steps: int, world: int, job_ms: float) -> float:
    """Whole-job TFLOP/s: every rank runs its own replica of the workload."""
    return world * steps * flop_per_step / (job_ms / 1000.0) / 1e12


def config_of(w, l2_note, parallelism):
    mask = "causal" if w.causal else "none"
    if w.key_len_range:
        mask = f"key_len~U[{w.key_len_range[0]},{w.key_len_range[1]}]"
    return {"workload": w.name, "B": w.B, "H": w.H, "N_q": w.Nq, "N_k": w.Nk, "d": w.d,
            "mask": mask, "scale": w.scale, "value_dist": f"N(0,{w.sigma}^2) bf16",
            "seed": w.seed, "l2": l2_note, "parallelism": parallelism}


def run_reference(args):
    """The oracle as it stands, on the host cores, bounded row sample per step."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return 0
    w = WORKLOADS[args.workload]
    x = make_inputs(w)
    per_step_s = float(os.environ.get("FA_REFERENCE_STEP_SECONDS", "2.0"))
    for _ in range(args.warmup):
        oracle_sample_rate(w, x, per_step_s / 4, rng_seed=1)
    rates, times, rows_used, cores = [], [], 0, 1
    t_start = time.perf_counter()
    for i in range(args.steps):
        t0 = time.perf_counter()
        r, n, t, cores = oracle_sample_rate(w, x, per_step_s, rng_seed=100 + i)
        times.append(time.perf_counter() - t0)
        rates.append(r)
        rows_used += n
    wall_s = time.perf_counter() - t_start
    value = float(np.mean(rates))
    # ms_per_step is what each step really took (its bounded row sample, sizing
    # calls included); the time the oracle would need for one whole workload is
    # an extrapolation from the measured rate and is reported under its own name
    ms = 1000.0 * wall_s / args.steps
    sample = (f"{rows_used} random query rows of {w.B * w.H * w.Nq} over {args.steps} steps "
              f"(~{per_step_s:.1f} s of CPU each), fp64, all keys each row sees")
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms,
        "step_is": "one bounded row sample of the workload, not the whole workload",
        "full_workload_ms_extrapolated": 1000.0 * w.flop / (value * 1e12),
        "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, "n/a (CPU)", "host cores"), "impl": "reference",
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=WORKLOAD_ORDER)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the per-workload table, e2e and CPU baseline (profiling runs)")
    ap.add_argument("--decode", default=None, choices=sorted(DECODE_WORKLOADS),
                    help="time only the split-KV forward on this decode workload (profiling runs)")
    ap.add_argument("--fp8-only", action="store_true",
                    help="time only the E4M3 forward on causal_8000_d128 (profiling runs)")
    ap.add_argument("--bwd-only", default=None, choices=["causal_8000_d128", "long_16k_d64"],
                    help="time only the backward pass on this workload (profiling runs)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)

    import torch
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    from io_aware_exact_24_b200 import FA_OK, build, fa_get_device_status, load_library
    build.build()
    load_library()

    if args.decode:
        w = DECODE_WORKLOADS[args.decode]
        big = kv_exceeds_l2(w)
        ms, ns = time_splitkv(w, make_inputs(w), args.steps, args.warmup, device, flush_l2=not big)
        peaks, peaks_src = load_peaks()
        gbs = w.algorithmic_bytes / (ms / 1000.0) / 1e9
        print(json.dumps({"metric": "split-KV attention fwd, algorithmic GB/s", "value": gbs,
                          "unit": "GB/s", "ms_per_step": ms, "num_splits": ns,
                          "roofline": {"bound": "hbm", "achieved": gbs,
                                       "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
                                       "frac": gbs / float(peaks["hbm_gbs"])},
                          "config": config_of(w, "not flushed: K/V larger than the 126 MB L2" if big
                                              else "flushed between timed launches", "single GPU")}),
              flush=True)
        return 0
    if args.bwd_only:
        w = WORKLOADS[args.bwd_only]
        ms = time_bwd(w, make_inputs(w), args.steps, args.warmup, device)
        print(json.dumps({"backward": {args.bwd_only: {"ms": ms,
                                                       "tflops": 2.5 * w.flop / (ms / 1000.0) / 1e12}}}),
              flush=True)
        return 0
    if args.fp8_only:
        peaks, _ = load_peaks()
        print(json.dumps({"fp8": fp8_table(args.steps, args.warmup, device,
                                           float(peaks["bf16_tflops"]))}), flush=True)
        return 0
    w = WORKLOADS[args.workload]
    x = make_inputs(w)
    clocks = ClockSampler(local)
    ms, per, clk = time_device(w, x, args.steps, args.warmup, device, rank, world, clocks)
    status = fa_get_device_status()
    if status != FA_OK:
        raise SystemExit(f"device status {status} after the timed region")
    job_ms = job_time_ms(sum(per), world, device)
    value = job_throughput_tflops(w.flop, args.steps, world, job_ms)

    peaks, peaks_src = load_peaks()
    peak = float(peaks["bf16_tflops"])
    achieved = w.flop / (ms / 1000.0) / 1e12
    traffic = load_traffic(w.name)
    inputs_mb = 2 * w.B * w.H * (w.Nq + 2 * w.Nk) * w.d / 1e6
    l2_note = (f"flushed between timed launches (256 MiB write outside the events); "
               f"inputs {inputs_mb:.0f} MB")
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": job_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": config_of(w, l2_note, f"replicas x{world}" if world > 1 else "single GPU"),
        "pct_of_nominal_bf16_peak": 100.0 * achieved / NOMINAL_BF16_TFLOPS,
        "ms_stats": ms_stats(per),
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "frac_of_nominal_2250": achieved / NOMINAL_BF16_TFLOPS,
                     "peak_source": f"{peaks_src} bf16_tflops (burst: kernel timed alone)",
                     "kernel": f"fa_fwd_sm100_kernel<{w.d}>",
                     "algorithmic_flop_per_launch": w.flop,
                     "algorithmic_bytes_per_launch": w.algorithmic_bytes},
        "gpu_launches": args.steps,
        "clocks": clk,
        "kernel_source_hash": kernel_source_hash(),
    }
    if rank == 0 and world == 1 and not args.no_extras:
        e2e_ms, h2d, d2h = time_e2e(w, x, max(3, args.steps // 4), 3, device)
        line["e2e"] = {"value": w.flop / (e2e_ms / 1000.0) / 1e12, "unit": UNIT,
                       "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                       "ms_per_step": e2e_ms, "entry": "fa_fwd_host (pinned host buffers)"}
        per_wl = {}
        for name in WORKLOAD_ORDER:
            wn = WORKLOADS[name]
            xn = x if name == w.name else make_inputs(wn)
            ms_n, per_n, _ = time_device(wn, xn, args.steps, args.warmup, device, 0, 1)
            per_wl[name] = {"ms": ms_n, "ms_stats": ms_stats(per_n),
                            "tflops": wn.flop / (ms_n / 1000.0) / 1e12,
                            "frac_of_peak": wn.flop / (ms_n / 1000.0) / 1e12 / peak,
                            "frac_of_nominal_2250": wn.flop / (ms_n / 1000.0) / 1e12 / NOMINAL_BF16_TFLOPS,
                            "algorithmic_gbs": wn.algorithmic_bytes / (ms_n / 1000.0) / 1e9,
                            "l2": "flushed between launches"}
            if xn["key_lens"] is not None:
                # padded batches: also the FLOPs of the keys each sequence has
                # (4*H*d*N_q*sum_b key_len_b, causal halved), beside the formula's
                kl = np.clip(np.asarray(xn["key_lens"], np.int64), 0, wn.Nk)
                eff = 4.0 * wn.H * wn.d * wn.Nq * float(kl.sum()) * (0.5 if wn.causal else 1.0)
                per_wl[name]["effective"] = {"flop": eff, "tflops": eff / (ms_n / 1000.0) / 1e12,
                                             "flop_formula": "4*H*d*N_q*sum_b key_len_b"}
            if wn.algorithmic_bytes < (126 << 20):
                # inputs that fit in L2: also back-to-back launches on a warm L2
                ms_w, per_w, _ = time_device(wn, xn, args.steps, args.warmup, device, 0, 1,
                                             flush_l2=False)
                per_wl[name]["warm_l2"] = {"ms": ms_w, "ms_stats": ms_stats(per_w),
                                           "tflops": wn.flop / (ms_w / 1000.0) / 1e12}
        line["per_workload"] = per_wl
        line["splitkv_decode"] = decode_table(args.steps, args.warmup, device,
                                              float(peaks["hbm_gbs"]))
        line["sliding_window"] = window_table(args.steps, args.warmup, device, peak)
        line["varlen"] = varlen_table(args.steps, args.warmup, device, peak)
        line["fp8"] = fp8_table(args.steps, args.warmup, device, peak)
        line["backward"] = bwd_table(args.steps, args.warmup, device, peak)
        cpu_s = float(os.environ.get("FA_CPU_BASELINE_SECONDS", "15"))
        rate, n, t, cores = oracle_sample_rate(w, x, cpu_s)
        line["cpu_baseline"] = {"value": rate, "unit": UNIT, "cores": cores, "kind": "oracle",
                                "sample": f"{n} random query rows of {w.B * w.H * w.Nq} "
                                          f"({t:.1f} s), fp64, all keys each row sees",
                                "single_thread": oracle_single_thread_table()}
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
