#!/usr/bin/env python
"""Benchmark of the KLA filter scan on B200 (one JSON line on rank 0).

A step is one kla_scan_forward call (load, Moebius + affine chunk scan,
cross-chunk carry, emit lambda / eta / mu / var) over the long-sequence
workload (B=1, H=32, N=128, T=65536, fp32): 268.4 M token-channels per GPU,
8.59 GB of algorithmic HBM traffic.  The same line also reports the recurrent
decode step (B=256, H=32, N=128, fp32 resident state; 1024 tokens replayed
from a CUDA graph), the backward scan (kla_scan_backward) of the same
workload, and the fused KLA layer (kla_layer_forward) on its own workload.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs under torchrun, one process per GPU; every rank filters its own
independent channels (a different seed per rank), so work per GPU is fixed
("weak" scaling) and no collective touches the data path: the only
collectives are the barrier and the max-over-ranks of the timings.

``--impl reference`` times the fp64 CPU oracle (the method's plain sequential
definition) on the host cores, as the reference arm.
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from kalman_linear_attention_b200 import workloads as wl  # noqa: E402

METRIC = "scan throughput (token-channels/s) and achieved HBM GB/s vs B200 peak, 1 GPU"
UNIT = "token-channels/s"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e, nominal (context beside the measured peak)
CSRC = os.path.join(ROOT, "kalman_linear_attention_b200", "csrc")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic.json")


# --------------------------------------------------------------- host helpers
def algorithmic_bytes_per_tc(w: wl.Workload) -> int:
    """Bytes the method must move per token-channel: read a, p, phi, b once,
    write lambda, eta, mu, var (fp32) once."""
    return (2 if w.dtype == "bf16" else 4) * 4 + 4 * 4


def decode_bytes_per_channel(w: wl.Workload) -> int:
    """Per decode token and channel: inputs, state read, state write, mu and var."""
    return (2 if w.dtype == "bf16" else 4) * 4 + 8 + 8 + 8


def rank_workload(w: wl.Workload, rank: int) -> wl.Workload:
    """Each rank filters its own independent channels: same shape, own seed."""
    return w if rank == 0 else w.with_shape(seed=w.seed + 1000 * rank)


def max_over_ranks(x: float, dist_mod=None) -> float:
    """Max of a per-rank float over all ranks (identity without a process group)."""
    if dist_mod is None or not dist_mod.is_initialized() or dist_mod.get_world_size() == 1:
        return float(x)
    import torch
    backend = dist_mod.get_backend()
    dev = torch.device("cuda", torch.cuda.current_device()) if backend == "nccl" else torch.device("cpu")
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist_mod.all_reduce(t, op=dist_mod.ReduceOp.MAX)
    return float(t.item())


_COMMENT = re.compile(r"//[^\n]*|/\*.*?\*/", re.S)


def kernel_source_hash() -> str:
    """Hash of the CUDA sources with comments and blank space removed, so
    that recorded profiler figures stay attached to the code they measured
    and survive edits of the comments only."""
    h = hashlib.sha256()
    for f in sorted(os.listdir(CSRC)):
        if not f.endswith((".cu", ".cuh", ".h")) or f == "kla_host.cu":  # host-only pipeline, no kernel
            continue
        with open(os.path.join(CSRC, f), encoding="utf-8") as fh:
            code = " ".join(_COMMENT.sub(" ", fh.read()).split())
        h.update(f.encode() + b"\0" + code.encode())
    return h.hexdigest()[:16]


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def recorded_traffic(workload: str, kernel: int):
    """DRAM bytes per launch from a committed ncu summary, only if it was
    taken on this kernel with the kernel sources as they are now."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        d = json.load(f)
    e = d.get(workload)
    if not e or e.get("kernel_sha") != kernel_source_hash() or e.get("kernel") != kernel:
        return None
    return float(e["dram_bytes_per_launch"])


class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during a region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,clocks.mem,clocks.max.mem")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (FileNotFoundError, OSError):
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        power = [num(r[3]) for r in rows if num(r[3]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.strip().lower() == "active"})
        # under load: samples drawing more than the idle baseline
        loaded = [s for s, pw in zip(sm, power) if pw is not None and pw > 0.5 * max(power)] if power else sm
        mem = [num(r[9]) for r in rows if len(r) > 9 and num(r[9]) is not None]
        mem_max = [num(r[10]) for r in rows if len(r) > 10 and num(r[10]) is not None]
        return {"sm_mhz": statistics.median(loaded or sm), "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows), "power_w_max": max(power) if power else None,
                "mem_mhz": statistics.median(mem) if mem else None, "mem_max_mhz": max(mem_max) if mem_max else None}


# ----------------------------------------------------------------- our arm
def inputs_to_device(w: wl.Workload, device, keep_host: bool):
    """Generated inputs, streamed block by block into device tensors [B, T, H, N];
    optionally also kept as pinned host tensors (for the end-to-end leg)."""
    import torch
    B, T, H, N = w.B, w.T, w.H, w.N
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    dev = {k: torch.empty((B, T, H, N), dtype=dt, device=device) for k in wl.INPUT_NAMES}
    host = {k: torch.empty((B, T, H, N), dtype=dt, pin_memory=True) for k in wl.INPUT_NAMES} \
        if keep_host else None
    HN = H * N
    for r0, r1, blk in wl.iter_rows(w):
        for k in wl.INPUT_NAMES:
            x = torch.from_numpy(blk[k].reshape(r1 - r0, HN)).to(dt)
            dev[k].view(B * T, HN)[r0:r1].copy_(x)
            if host is not None:
                host[k].view(B * T, HN)[r0:r1].copy_(x)
    pri = wl.prior(w)
    dev["lam0"] = torch.from_numpy(pri["lam0"]).to(device)
    dev["eta0"] = torch.from_numpy(pri["eta0"]).to(device)
    if host is not None:
        host["lam0"] = torch.from_numpy(pri["lam0"]).pin_memory()
        host["eta0"] = torch.from_numpy(pri["eta0"]).pin_memory()
    return dev, host


def time_forward(kla, w, dev, steps: int, warmup: int, dist_mod):
    import torch
    B, T, H, N = w.B, w.T, w.H, w.N
    outs = [torch.empty((B, T, H, N), dtype=torch.float32, device=dev["a"].device) for _ in range(4)]
    ws = kla.new_workspace(B, T, H, N, dev["a"].dtype, dev["a"].device)
    stream = torch.cuda.current_stream()
    plan = kla.forward_plan(dev["a"], dev["p"], dev["phi"], dev["b"])
    args = (dev["a"], dev["p"], dev["phi"], dev["b"], dev["lam0"], dev["eta0"])
    for _ in range(warmup):
        kla.scan_forward(*args, out=outs, workspace=ws)
    torch.cuda.synchronize()
    if kla.get_error() != 0:
        raise RuntimeError("device-side error during warm-up")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist_mod is not None and dist_mod.is_initialized():
        dist_mod.barrier()
    torch.cuda.synchronize()
    t_start.record(stream)
    for i in range(steps):
        ev[i][0].record(stream)
        kla.scan_forward(*args, out=outs, workspace=ws)
        ev[i][1].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    if dist_mod is not None and dist_mod.is_initialized():
        dist_mod.barrier()
    if kla.get_error() != 0:
        raise RuntimeError("device-side error in the timed region")
    total_ms = t_start.elapsed_time(t_end)
    per_launch = [a.elapsed_time(b) for a, b in ev]
    return total_ms, per_launch, plan, outs


L2_FLUSH_BYTES = 256 << 20  # twice the B200's 126 MB L2
L2_BYTES = 126 << 20


def l2_flusher(device):
    """A function that overwrites a buffer twice the size of L2 (evicting
    whatever the previous launch left there), to be called between timed
    launches, outside the events."""
    import torch
    buf = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=device)

    def flush():
        buf.fill_(0)
    return flush


def time_launches(fn, steps: int, warmup: int, flush=None):
    """Per-launch CUDA-event times (ms) of `fn` on the current stream: `warmup`
    untimed calls, then `steps` calls each bracketed by its own events, the L2
    flushed before each one (outside the events) when `flush` is given."""
    import torch
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for e0, e1 in ev:
        if flush is not None:
            flush()
        e0.record(stream)
        fn()
        e1.record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ev]


FORWARD_KERNELS = {1: "kla_forward_kernel (chunked, cross-CTA carries; + its workspace clear kernel)",
                   2: "kla_forward_stream_kernel (channel-owning streaming)"}


def time_config(kla, w: wl.Workload, device, steps: int, warmup: int, peak: float, flush):
    """One forward workload timed on its own: the median of `steps` per-launch
    CUDA-event times of kla_scan_forward (every output written).  Workloads
    whose inputs are larger than L2 are timed back to back, as the headline
    is (each launch then also writes back what the previous one left dirty in
    L2: its own algorithmic bytes on average); smaller ones with the L2
    flushed by a 256 MB write between launches.  The flushed timing is
    reported beside the back-to-back one (``ms_l2_flushed``): there each
    launch also writes back the flush buffer's dirty lines.  Returns the
    entry of the bench line's ``configs`` object (without the CPU baseline)
    and the host arrays."""
    import torch
    x = wl.generate(w)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    d = {k: torch.from_numpy(x[k]).to(device=device, dtype=dt) for k in wl.INPUT_NAMES}
    for k in ("lam0", "eta0"):
        d[k] = torch.from_numpy(x[k]).to(device)
    outs = [torch.empty((w.B, w.T, w.H, w.N), dtype=torch.float32, device=device) for _ in range(4)]
    ws = kla.new_workspace(w.B, w.T, w.H, w.N, dt, device)
    plan = kla.forward_plan(d["a"], d["p"], d["phi"], d["b"])
    args = (d["a"], d["p"], d["phi"], d["b"], d["lam0"], d["eta0"])
    call = lambda: kla.scan_forward(*args, out=outs, workspace=ws)  # noqa: E731
    per_flushed = time_launches(call, steps, warmup, flush)
    tc = w.token_channels
    bpt = algorithmic_bytes_per_tc(w)
    in_bytes = (bpt - 16) * tc
    big = in_bytes > L2_BYTES
    per = time_launches(call, steps, warmup) if big else per_flushed
    if kla.get_error() != 0:
        raise RuntimeError(f"device-side error while timing {w.name}")
    ms = statistics.median(per)
    gbs = bpt * tc / (ms * 1e-3) / 1e9
    ms_fl = statistics.median(per_flushed)
    del d, outs, ws
    entry = {"workload": w.summary, "B": w.B, "H": w.H, "N": w.N, "T": w.T, "dtype": w.dtype,
             "ms": ms, "ms_min": min(per), "ms_max": max(per), "launches_timed": steps, "warmup": warmup,
             "value": tc / (ms * 1e-3), "unit": UNIT, "gb_per_s": gbs,
             "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                          "frac_of_nominal": gbs / NOMINAL_HBM_GBS,
                          "algorithmic_bytes_per_launch": bpt * tc, "bytes_per_token_channel": bpt,
                          "traffic": recorded_traffic(w.name, plan[0])},
             "kernel": FORWARD_KERNELS[plan[0]], "launches_per_call": plan[1],
             "timing": (f"median of per-launch CUDA events, back to back (inputs of {in_bytes / 1e6:.0f} MB, "
                        f"larger than the 126 MB L2)" if big else
                        "median of per-launch CUDA events, L2 flushed (256 MB write) between launches")}
    if big:
        gfl = bpt * tc / (ms_fl * 1e-3) / 1e9
        entry["ms_l2_flushed"] = ms_fl
        entry["frac_l2_flushed"] = gfl / peak
    return entry, x


def time_copy_bandwidth(device, steps: int = 20, nbytes: int = 4 << 30):
    """Device-to-device copy bandwidth of this GPU in this run: read + write
    bytes of a 4 GiB torch copy over the median CUDA-event time.  It is
    context for the roofline fractions (boxes differ), not their denominator."""
    import torch
    src = torch.empty(nbytes // 4, dtype=torch.float32, device=device)
    src.fill_(1.0)
    dst = torch.empty_like(src)
    per = time_launches(lambda: dst.copy_(src), steps, 3)
    ms = statistics.median(per)
    del src, dst
    dst2 = torch.empty(nbytes // 4, dtype=torch.float32, device=device)
    per_w = time_launches(lambda: dst2.fill_(0.5), steps, 3)
    ms_w = statistics.median(per_w)
    del dst2
    return {"gb_per_s": 2 * nbytes / (ms * 1e-3) / 1e9, "ms": ms,
            "write_only_gb_per_s": nbytes / (ms_w * 1e-3) / 1e9,
            "how": "torch copy_ of a 4 GiB fp32 buffer on the device, (read + write bytes) / median of "
                   f"{steps} CUDA-event times; write_only: torch fill_ of 4 GiB, bytes / median time"}


def time_lti(kla, device, steps: int, warmup: int, peak: float, tokens: int = 0):
    """The convolutional form (kla_scan_forward_lti) on the time-invariant
    workload, and the general scan on the same problem (a broadcast over
    time, p = 0) for comparison; each one's largest relative error of lambda
    against the oracle's filter on 8 sampled whole channels.  ``tokens``
    overrides T (smaller cases for profiler captures)."""
    import torch
    import oracle
    w = wl.LTI_WORKLOADS["lti"]
    if tokens:
        w = w.with_shape(T=tokens)
    x = wl.generate_lti(w)
    d = {k: torch.from_numpy(x[k]).to(device) for k in ("a", "phi", "b", "lam0", "eta0")}
    outs = [torch.empty((w.B, w.T, w.H, w.N), device=device) for _ in range(4)]
    ws = torch.empty(max(kla.lti_workspace_size(w.B, w.T, w.H, w.N), 1), dtype=torch.uint8, device=device)
    plan = kla.lti_plan(d["phi"], d["b"])
    args = (d["a"], d["phi"], d["b"], d["lam0"], d["eta0"])
    per = time_launches(lambda: kla.scan_forward_lti(*args, out=outs, workspace=ws), steps, warmup)
    if kla.get_error() != 0:
        raise RuntimeError("device-side error in the convolutional form")
    ms = statistics.median(per)
    tc = w.token_channels
    bpt = 2 * 4 + 4 * 4
    gbs = bpt * tc / (ms * 1e-3) / 1e9
    HN = w.H * w.N
    sample = wl.channel_sample(w, 8)
    sb, shn = np.divmod(sample, HN)
    K = len(sample)
    a_s = x["a"].reshape(w.B, HN)[sb, shn].reshape(1, 1, 1, K)
    phi_s = x["phi"].reshape(w.B, w.T, HN)[sb, :, shn].T.reshape(1, w.T, 1, K)
    b_s = x["b"].reshape(w.B, w.T, HN)[sb, :, shn].T.reshape(1, w.T, 1, K)
    ref = oracle.forward(np.broadcast_to(a_s, phi_s.shape), np.zeros(phi_s.shape), phi_s, b_s,
                         np.ones((1, 1, K)), np.zeros((1, 1, K)), threads=8)["lam"].reshape(w.T, K)

    def lam_err(lam):
        got = lam.view(w.B, w.T, HN)[torch.as_tensor(sb, device=device), :, torch.as_tensor(shn, device=device)]
        return float(np.max(np.abs(got.T.double().cpu().numpy() - ref) / ref))

    err_lti = lam_err(outs[0])
    # the general scan on the same problem
    a_full = d["a"][:, None].expand(w.B, w.T, w.H, w.N).contiguous()
    p_full = torch.zeros_like(a_full)
    gws = kla.new_workspace(w.B, w.T, w.H, w.N, torch.float32, device)
    gargs = (a_full, p_full, d["phi"], d["b"], d["lam0"], d["eta0"])
    gper = time_launches(lambda: kla.scan_forward(*gargs, out=outs, workspace=gws), steps, warmup)
    gms = statistics.median(gper)
    err_gen = lam_err(outs[0])
    del a_full, p_full, gws, d, outs, ws
    return {"workload": w.summary, "ms": ms, "value": tc / (ms * 1e-3), "unit": UNIT, "gb_per_s": gbs,
            "launches_timed": steps,
            "kernel": {1: "kla_lti_seq_kernel (one thread per channel)",
                       2: "kla_lti_stream_kernel (channel-owning streaming, blocked convolutions)"}[plan[0]],
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                         "algorithmic_bytes_per_launch": bpt * tc, "bytes_per_token_channel": bpt,
                         "traffic": recorded_traffic("lti" if not tokens else f"lti@T={tokens}", plan[0])},
            "max_rel_err_lambda_vs_oracle": err_lti,
            "general_scan_same_problem": {
                "ms": gms, "value": tc / (gms * 1e-3), "bytes_per_token_channel": 32,
                "gb_per_s": 32 * tc / (gms * 1e-3) / 1e9, "max_rel_err_lambda_vs_oracle": err_gen,
                "speedup_of_convolutional_form": gms / ms},
            "timing": "median of per-launch CUDA events (inputs of 2.1 GB, larger than L2)"}


def time_attention(kla, device, steps: int, warmup: int, peak: float, W: int = 64, rows: int = 0):
    """kla_attention_weights over every window of W tokens of the LM-layer
    workload (bf16 inputs), from the forward scan's lambda.  ``rows``
    overrides B (smaller cases for profiler captures)."""
    import torch
    w = wl.WORKLOADS["lm_layer"]
    if rows:
        w = w.with_shape(B=rows)
    x = wl.generate(w)
    d = {k: torch.from_numpy(x[k]).to(device=device, dtype=torch.bfloat16) for k in wl.INPUT_NAMES}
    lam0 = torch.from_numpy(x["lam0"]).to(device)
    eta0 = torch.from_numpy(x["eta0"]).to(device)
    del x
    lam = kla.scan_forward(d["a"], d["p"], d["phi"], d["b"], lam0, eta0, want_mu=False, want_var=False)[0]
    del d["phi"], d["b"]
    nwin = -(-w.T // W)
    F = torch.empty((w.B, nwin, W, W, w.H, w.N), device=device)
    per = time_launches(lambda: kla.attention_weights(d["a"], d["p"], lam, W=W, out=F), steps, warmup)
    if kla.get_error() != 0:
        raise RuntimeError("device-side error in the attention weights")
    ms = statistics.median(per)
    HN = w.H * w.N
    write_bytes = w.B * nwin * W * W * HN * 4
    read_bytes = w.token_channels * (2 + 2 + 4)
    gbs = (write_bytes + read_bytes) / (ms * 1e-3) / 1e9
    del F, lam, d
    return {"workload": f"Kalman attention weights, windows of {W} tokens over {w.summary}", "ms": ms,
            "value": w.token_channels / (ms * 1e-3), "unit": UNIT, "gb_per_s": gbs, "launches_timed": steps,
            "kernel": "kla_attention_kernel", "weights_per_s": write_bytes / 4 / (ms * 1e-3),
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                         "algorithmic_bytes_per_launch": write_bytes + read_bytes,
                         "bytes": f"{W}*{W}*4 written per channel and window + a, p (bf16) and lambda read",
                         "traffic": recorded_traffic("attention" if not rows and W == 64 else
                                                     f"attention@B={w.B},W={W}", 1)},
            "timing": "median of per-launch CUDA events (8.6 GB written per launch, larger than L2)"}


def backward_bytes_per_tc(w: wl.Workload) -> int:
    """Bytes the backward scan must move per token-channel with all four
    output gradients present: read a, p (input dtype), lambda, eta and the
    four output gradients (fp32); write the four input gradients (input
    dtype)."""
    e = 2 if w.dtype == "bf16" else 4
    return 2 * e + 2 * 4 + 4 * 4 + 4 * e


def time_backward(kla, w, dev, outs, steps: int, warmup: int, peak: float, traffic_key: str):
    """kla_scan_backward on the forward's lambda / eta with all four output
    gradients present (the general case), CUDA events per launch."""
    import torch
    B, T, H, N = w.B, w.T, w.H, w.N
    device = dev["a"].device
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed + 17)
    grads = [torch.randn((B, T, H, N), generator=gen, device=device) for _ in range(4)]
    res = [torch.empty((B, T, H, N), dtype=dev["a"].dtype, device=device) for _ in range(4)]
    res += [torch.empty((B, H, N), device=device) for _ in range(2)]
    ws = torch.empty(max(kla.backward_workspace_size(B, T, H, N, dev["a"].dtype), 1), dtype=torch.uint8,
                     device=device)
    plan = kla.backward_plan(dev["a"], dev["p"])
    args = (dev["a"], dev["p"], dev["lam0"], dev["eta0"], outs[0], outs[1], *grads)
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        kla.scan_backward(*args, out=res, workspace=ws)
    torch.cuda.synchronize()
    if kla.get_error() != 0:
        raise RuntimeError("device-side error during backward warm-up")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        ev[i][0].record(stream)
        kla.scan_backward(*args, out=res, workspace=ws)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    if kla.get_error() != 0:
        raise RuntimeError("device-side error in the timed backward region")
    ms = statistics.median(a.elapsed_time(b) for a, b in ev)
    bpt = backward_bytes_per_tc(w)
    tc = w.token_channels
    gbs = bpt * tc / (ms * 1e-3) / 1e9
    del grads, res
    return {"workload": f"{w.name}: {w.summary}, all four output gradients present",
            "ms_per_step": ms, "value": tc / (ms * 1e-3), "unit": UNIT, "steps": steps, "warmup": warmup,
            "kernel": {1: "kla_backward_seq_kernel (one thread per channel)",
                       2: "kla_backward_stream_kernel (channel-owning streaming, reverse time)"}[plan[0]],
            "gpu_launches": plan[1] * steps,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                         "algorithmic_bytes_per_launch": bpt * tc,
                         "traffic": recorded_traffic(traffic_key, plan[0])},
            "data": "forward outputs of the timed forward; output gradients from a seeded torch.randn on the device"}


def time_e2e(kla, w, host, steps: int):
    """Public API with pinned HOST tensors: H2D copies, scan, D2H copies, sync."""
    import torch
    B, T, H, N = w.B, w.T, w.H, w.N
    outs = [torch.empty((B, T, H, N), dtype=torch.float32, pin_memory=True) for _ in range(4)]
    args = (host["a"], host["p"], host["phi"], host["b"], host["lam0"], host["eta0"])
    kla.scan_forward(*args, out=outs)  # warm-up (allocator, first-touch of pinned pages)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for _ in range(steps):
        kla.scan_forward(*args, out=outs)
    torch.cuda.synchronize()
    dt = (time.perf_counter() - t0) / steps
    h2d = sum(host[k].numel() * host[k].element_size() for k in host)
    d2h = sum(o.numel() * o.element_size() for o in outs)
    return dt, h2d, d2h


def time_decode(kla, device, steps_tokens: int | None, replays: int, batch: int | None = None):
    """Decode workload: tokens replayed from a CUDA graph of kla_scan_step calls
    (``batch`` overrides B: with a single sequence the time per token is the
    fixed cost of one step, launch included)."""
    import torch
    w = wl.WORKLOADS["decode"]
    if steps_tokens is not None:
        w = w.with_shape(T=steps_tokens)
    if batch is not None:
        w = w.with_shape(B=batch)
    dev, _ = inputs_to_device(w, device, keep_host=False)
    steps = {k: dev.pop(k).transpose(0, 1).contiguous() for k in wl.INPUT_NAMES}  # [T, B, H, N]
    lam = dev["lam0"].clone()
    eta = dev["eta0"].clone()
    mu = torch.empty_like(lam)
    var = torch.empty_like(lam)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for t in range(3):  # warm-up, eager
            kla.scan_step(steps["a"][t], steps["p"][t], steps["phi"][t], steps["b"][t], lam, eta,
                          mu_out=mu, var_out=var, stream=s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for t in range(w.T):
            kla.scan_step(steps["a"][t], steps["p"][t], steps["phi"][t], steps["b"][t], lam, eta,
                          mu_out=mu, var_out=var, stream=s)
    g.replay()  # warm-up replay
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(replays):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / (replays * w.T)
    del g
    tc = w.channels
    bytes_step = decode_bytes_per_channel(w) * tc
    in_bytes = (2 if w.dtype == "bf16" else 4) * 4 * tc
    return {"workload": w.summary, "ms_per_token": ms, "value": tc / (ms * 1e-3), "unit": UNIT,
            "gb_per_s": bytes_step / (ms * 1e-3) / 1e9, "bytes_per_token": bytes_step,
            "input_bytes_per_token": in_bytes, "input_gb_per_s": in_bytes / (ms * 1e-3) / 1e9,
            "tokens_per_replay": w.T, "replays": replays,
            "note": "one kla_scan_step launch per token; the 8 MB fp32 state can stay L2-resident"}


def time_layer(kla, device, steps: int, warmup: int):
    """The fused KLA layer (kla_layer_forward) on the layer workload, and the
    same computation unfused for comparison: phi, b, a, p formed with torch,
    kla_scan_forward over the H x D x Ns channels, the readout with torch."""
    import torch
    w = wl.LAYER_WORKLOADS["layer"]
    x = wl.generate_layer(w)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    d = {k: torch.from_numpy(x[k]).to(device).to(dt) for k in wl.LAYER_TOKEN_NAMES}
    for k in ("a", "p", "lam0", "eta0"):
        d[k] = torch.from_numpy(x[k]).to(device)
    B, T, H, D, Ns = w.B, w.T, w.H, w.D, w.Ns
    outs = [torch.empty((B, T, H, D), device=device), torch.empty((B, T, H, D), device=device),
            torch.empty((B, H, D, Ns), device=device), torch.empty((B, H, D, Ns), device=device)]
    ws = torch.empty(max(kla.layer_workspace_size(B, T, H, D, Ns, dt), 1), dtype=torch.uint8, device=device)
    args = (d["k"], d["q"], d["v"], d["w"], d["a"], d["p"], d["lam0"], d["eta0"])

    def fused():
        kla.layer_forward(*args, out=outs, workspace=ws)

    def unfused():
        kk = d["k"].float()[:, :, :, None, :]
        ww = d["w"].float()[:, :, :, :, None]
        phi = (kk * kk * ww).reshape(B, T, H, D * Ns)
        info = (kk * ww * d["v"].float()[:, :, :, :, None]).reshape(B, T, H, D * Ns)
        aa = d["a"].expand(B, T, H, D, Ns).reshape(B, T, H, D * Ns).contiguous()
        pp = d["p"].expand(B, T, H, D, Ns).reshape(B, T, H, D * Ns).contiguous()
        lam, eta, mu, var = kla.scan_forward(aa, pp, phi, info, d["lam0"].reshape(B, H, D * Ns),
                                             d["eta0"].reshape(B, H, D * Ns))
        qq = d["q"].float()[:, :, :, None, :]
        (qq * mu.reshape(B, T, H, D, Ns)).sum(-1)
        (qq * qq * var.reshape(B, T, H, D, Ns)).sum(-1)

    def timed(fn, n):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        if kla.get_error() != 0:
            raise RuntimeError("device-side error in the layer warm-up")
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        for e0, e1 in ev:
            e0.record()
            fn()
            e1.record()
        torch.cuda.synchronize()
        if kla.get_error() != 0:
            raise RuntimeError("device-side error in the timed layer region")
        return statistics.median(a.elapsed_time(b) for a, b in ev)

    ms = timed(fused, steps)
    ms_unfused = timed(unfused, max(3, steps // 10))

    # decode: kla_layer_step tokens from a CUDA graph (B = 256 sequences)
    Bd, Td = 256, 256
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed + 29)
    dk = (torch.randn((Td, Bd, H, Ns), generator=gen, device=device) / Ns ** 0.5).to(dt)
    dq = (torch.randn((Td, Bd, H, Ns), generator=gen, device=device) / Ns ** 0.5).to(dt)
    dv = torch.randn((Td, Bd, H, D), generator=gen, device=device).to(dt)
    dw = torch.nn.functional.softplus(torch.randn((Td, Bd, H, D), generator=gen, device=device)).to(dt)
    lam = torch.ones((Bd, H, D, Ns), device=device)
    eta = torch.zeros((Bd, H, D, Ns), device=device)
    yd = torch.empty((Bd, H, D), device=device)
    sd = torch.empty((Bd, H, D), device=device)
    st = torch.cuda.Stream()
    st.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(st):
        for t in range(3):
            kla.layer_step(dk[t], dq[t], dv[t], dw[t], d["a"], d["p"], lam, eta, y=yd, s=sd, stream=st)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=st):
        for t in range(Td):
            kla.layer_step(dk[t], dq[t], dv[t], dw[t], d["a"], d["p"], lam, eta, y=yd, s=sd, stream=st)
    graph.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(4):
        graph.replay()
    e1.record()
    torch.cuda.synchronize()
    if kla.get_error() != 0:
        raise RuntimeError("device-side error in the layer decode")
    us_token = e0.elapsed_time(e1) * 1e3 / (4 * Td)
    del graph
    tc = w.token_channels
    esz = 2 if w.dtype == "bf16" else 4
    bytes_call = B * T * H * (2 * Ns * esz + 2 * D * esz + 2 * D * 4) + 4 * B * H * D * Ns * 4 + 2 * H * D * Ns * 4
    return {"workload": f"{w.name}: {w.summary}", "ms_per_step": ms, "value": tc / (ms * 1e-3), "unit": UNIT,
            "steps": steps, "kernel": "kla_layer_forward_kernel", "gpu_launches": steps,
            "algorithmic_bytes_per_call": bytes_call, "gb_per_s": bytes_call / (ms * 1e-3) / 1e9,
            "unfused_ms_per_step": ms_unfused, "speedup_vs_unfused": ms_unfused / ms,
            "decode": {"us_per_token": us_token, "batch": Bd,
                       "token_channels_per_s": Bd * H * D * Ns / (us_token * 1e-6),
                       "how": f"kla_layer_step, {Td} tokens captured in a CUDA graph, 4 replays"},
            "note": "ALU-bound: 0.9 B of HBM traffic per token-channel; the unfused path (torch forming phi, b, "
                    "a, p and reading out, kla_scan_forward in between) moves about 40 B per token-channel"}


def cpu_oracle_sample(w: wl.Workload, host_arrays, target_s: float = 10.0, threads: int | None = None):
    """Time the fp64 oracle on a bounded sample of whole channels of the
    workload, on `threads` host threads (default: every core)."""
    import oracle
    orc = oracle.default()
    threads = min(threads or os.cpu_count() or 1, orc.max_threads())
    HN = w.H * w.N

    def run(nch):
        idx = np.arange(nch)
        b_idx, c_idx = np.divmod(idx, HN)
        x = {k: np.ascontiguousarray(host_arrays[k].reshape(w.B, w.T, HN)[b_idx, :, c_idx].T)
             .reshape(1, w.T, 1, nch) for k in wl.INPUT_NAMES}
        t0 = time.perf_counter()
        orc.forward(x["a"], x["p"], x["phi"], x["b"], np.ones((1, 1, nch)), np.zeros((1, 1, nch)),
                    threads=threads)
        return time.perf_counter() - t0

    n = min(w.channels, max(threads, 8))
    dt = run(n)
    while dt < target_s / 4 and n < w.channels:
        n = min(w.channels, int(n * max(2.0, target_s / max(dt, 1e-3) / 2)))
        dt = run(n)
    reps = 1
    if dt < target_s / 4:  # the whole workload is a small sample: repeat it
        reps = max(1, min(1000, int(target_s / 4 / max(dt, 1e-6))))
        dt = min(sum(run(n) for _ in range(reps)) / reps for _ in range(2))
    return {"value": n * w.T / dt, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{n} of {w.channels} channels x all {w.T} tokens ({n * w.T:,} token-channels)"
                      + (f", best of 2 means of {reps} runs" if reps > 1 else "")
                      + f", fp64 sequential covariance-form filter, OpenMP over channels, {dt:.3g} s per run"}


def run_ours(args):
    import torch
    import torch.distributed as dist
    import kalman_linear_attention_b200 as kla

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)

    base = wl.WORKLOADS[args.workload]
    if args.tokens:
        base = base.with_shape(T=args.tokens)
    w = rank_workload(base, rank)
    keep_host = not args.no_e2e
    dev, host = inputs_to_device(w, device, keep_host=keep_host)

    sampler = ClockSampler(local)
    sampler.start()
    total_ms, per_launch, plan, fwd_outs = time_forward(kla, w, dev, args.steps, args.warmup,
                                                        dist if world > 1 else None)
    kernel_name = FORWARD_KERNELS[plan[0]]
    clocks = sampler.stop()

    max_ms = max_over_ranks(total_ms, dist if world > 1 else None)
    tc_rank = w.token_channels
    tc_all = tc_rank * world
    value = tc_all * args.steps / (max_ms * 1e-3)
    bpt = algorithmic_bytes_per_tc(w)
    launch_ms = statistics.median(per_launch)
    achieved = bpt * tc_rank / (launch_ms * 1e-3) / 1e9
    peak, peak_src = measured_peaks()
    traffic = recorded_traffic(args.workload if not args.tokens else f"{args.workload}@T={args.tokens}",
                               plan[0])

    backward = None
    if not args.no_backward:
        backward = time_backward(kla, w, dev, fwd_outs, args.backward_steps, args.warmup, peak,
                                 (args.workload if not args.tokens else f"{args.workload}@T={args.tokens}")
                                 + ":backward")
    del fwd_outs
    layer = None
    if not args.no_layer:
        layer = time_layer(kla, device, args.layer_steps, args.warmup)

    e2e = None
    if host is not None:
        del dev
        torch.cuda.empty_cache()
        e2e_s, h2d, d2h = time_e2e(kla, w, host, args.e2e_steps)
        e2e_s = max_over_ranks(e2e_s, dist if world > 1 else None)
        e2e = {"value": tc_all / e2e_s, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": e2e_s * 1e3,
               "how": "scan_forward on pinned host tensors (C ABI kla_scan_forward_host): the sequence in "
                      "64 blocks, H2D of a, p, phi, b (+ lam0, eta0), scan, D2H of lambda, eta, mu, var "
                      "pipelined on three streams, then a stream sync; wall clock"}
    decode = None
    if not args.no_decode:
        decode = time_decode(kla, device, None, args.decode_replays)
        probe = time_decode(kla, device, None, args.decode_replays, batch=1)
        decode["fixed_cost_probe"] = {
            "us_per_token": probe["ms_per_token"] * 1e3, "channels": 32 * 128,
            "note": "the same graph of 1024 kla_scan_step calls on one sequence (4096 channels, 16 KB of "
                    "inputs per step): the fixed cost of a step, launch included"}
        decode["input_roofline"] = {
            "bound": "hbm", "achieved": decode["input_gb_per_s"], "peak": peak, "unit": "GB/s",
            "frac": decode["input_gb_per_s"] / peak,
            "note": "the token inputs (a, p, phi, b) are the only bytes that must come from HBM each step; "
                    "the state and the mu / var buffers stay L2-resident between steps"}

    # every forward workload of the task timed on its own (one GPU only)
    configs = None
    copy_bw = None
    if world == 1 and not args.no_configs:
        flush = l2_flusher(device)
        configs = {}
        host_cfg = {}
        for name in ("tiny", "lm_layer", "stiff"):
            configs[name], host_cfg[name] = time_config(kla, wl.WORKLOADS[name], device, args.config_steps,
                                                        args.warmup, peak, flush)
        configs["long"] = {
            "workload": base.summary, "B": base.B, "H": base.H, "N": base.N, "T": base.T, "dtype": base.dtype,
            "ms": launch_ms, "ms_min": min(per_launch), "ms_max": max(per_launch),
            "launches_timed": len(per_launch), "warmup": args.warmup, "value": tc_rank / (launch_ms * 1e-3),
            "unit": UNIT, "gb_per_s": achieved,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "frac_of_nominal": achieved / NOMINAL_HBM_GBS,
                         "algorithmic_bytes_per_launch": bpt * tc_rank, "bytes_per_token_channel": bpt,
                         "traffic": traffic},
            "kernel": kernel_name, "launches_per_call": plan[1],
            "timing": "the headline's timed steps: median of per-launch CUDA events, back to back "
                      "(inputs of 4.3 GB, larger than L2)"}
        del flush
        torch.cuda.empty_cache()
        copy_bw = time_copy_bandwidth(device)
        for e in configs.values():
            e["roofline"]["frac_of_same_run_copy"] = e["gb_per_s"] / copy_bw["gb_per_s"]
        if rank == 0 and not args.no_cpu_baseline:
            for name in ("tiny", "lm_layer", "stiff"):
                w_c = wl.WORKLOADS[name]
                configs[name]["cpu_baseline"] = cpu_oracle_sample(w_c, host_cfg[name], args.cpu_target_s)
                configs[name]["cpu_baseline_1core"] = cpu_oracle_sample(w_c, host_cfg[name], args.cpu_target_s,
                                                                        threads=1)
        del host_cfg
        if not args.no_forms:
            torch.cuda.empty_cache()
            configs["lti"] = time_lti(kla, device, args.config_steps, args.warmup, peak, tokens=args.tokens)
            torch.cuda.empty_cache()
            configs["attention"] = time_attention(kla, device, args.config_steps, args.warmup, peak,
                                                  rows=args.attention_rows)
            torch.cuda.empty_cache()
            for name in ("lti", "attention"):
                configs[name]["roofline"]["frac_of_same_run_copy"] = (configs[name]["gb_per_s"]
                                                                      / copy_bw["gb_per_s"])

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and host is not None:
        arrays = {k: host[k].float().numpy() for k in wl.INPUT_NAMES}
        cpu = cpu_oracle_sample(w, arrays)
        if configs is not None:
            configs["long"]["cpu_baseline"] = cpu
            configs["long"]["cpu_baseline_1core"] = cpu_oracle_sample(w, arrays, args.cpu_target_s, threads=1)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": max_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32" if w.dtype == "f32" else "bf16",
        "data": "synthetic (seeded numpy draws of the workload's distributions; own seed per rank)",
        "config": {"workload": f"{base.name}: {base.summary}", "B": base.B, "H": base.H, "N": base.N,
                   "T": base.T, "token_channels_per_gpu": tc_rank, "parallelism": f"replicas x{world}",
                   "l2": f"inputs larger than L2 ({bpt // 2 * tc_rank / 1e9:.1f} GB of inputs vs 126 MB L2)"},
        "gb_per_s": bpt * tc_all * args.steps / (max_ms * 1e-3) / 1e9,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_source": f"{peak_src} copy bandwidth",
                     "frac_of_nominal": achieved / NOMINAL_HBM_GBS,
                     "traffic": traffic, "algorithmic_bytes_per_launch": bpt * tc_rank,
                     "kernel": kernel_name, "launch_ms": launch_ms},
        "gpu_launches": plan[1] * args.steps,
        "clocks": clocks,
        "e2e": e2e,
        "decode": decode,
        "backward": backward,
        "layer": layer,
        "configs": configs,
        "hbm_copy_same_run": copy_bw,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line))


# ----------------------------------------------------------- reference arm
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    w = wl.WORKLOADS[args.workload]
    threads = min(os.cpu_count() or 1, oracle.default().max_threads())
    # a bounded sample per step: whole channels, all tokens
    nch = max(1, min(w.channels, args.ref_channels))
    HN = w.H * w.N
    ws = w.with_shape(B=1, H=1, N=nch) if w.B * HN >= nch else w
    x = wl.generate(ws.with_shape(T=w.T))
    a = {k: x[k] for k in wl.INPUT_NAMES}
    orc = oracle.default()
    for _ in range(args.warmup):
        orc.forward(a["a"], a["p"], a["phi"], a["b"], x["lam0"], x["eta0"], threads=threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        orc.forward(a["a"], a["p"], a["phi"], a["b"], x["lam0"], x["eta0"], threads=threads)
    dt = (time.perf_counter() - t0) / args.steps
    tc = nch * w.T
    value = tc / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{w.name}: {w.summary}", "B": w.B, "H": w.H, "N": w.N, "T": w.T},
        "cpu_baseline": {"value": value, "unit": UNIT, "kind": "oracle", "cores": threads,
                         "sample": f"{nch} of {w.channels} channels x all {w.T} tokens per step "
                                   f"(same distributions, seed {w.seed}), fp64 sequential filter"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="long", choices=sorted(k for k, v in wl.WORKLOADS.items()
                                                                  if not v.decode))
    ap.add_argument("--tokens", type=int, default=0,
                    help="override T of the headline and time-invariant workloads (smaller cases for "
                         "profiler captures; not a bench line)")
    ap.add_argument("--attention-rows", type=int, default=0,
                    help="override B of the attention-weight leg (smaller cases for profiler captures)")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--decode-replays", type=int, default=5)
    ap.add_argument("--ref-channels", type=int, default=256)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--backward-steps", type=int, default=50)
    ap.add_argument("--no-layer", action="store_true")
    ap.add_argument("--layer-steps", type=int, default=50)
    ap.add_argument("--no-configs", action="store_true",
                    help="skip timing the tiny, LM-layer and stiff workloads on their own")
    ap.add_argument("--config-steps", type=int, default=30)
    ap.add_argument("--no-forms", action="store_true",
                    help="skip the convolutional-form and attention-weight legs")
    ap.add_argument("--cpu-target-s", type=float, default=4.0,
                    help="seconds of oracle work per CPU timing of the per-workload entries")
    return ap.parse_args(argv)


def main(argv=None):
    args = parse_args(argv)
    if args.warmup < 3:
        raise SystemExit("--warmup must be at least 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
