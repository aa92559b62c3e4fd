#!/usr/bin/env python
"""Benchmark of the selective scan (S6) hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one fused selective-scan forward over the Mamba-2.8B-shaped layer
(batch 4, dim 5120, N 16, L 4096, bf16 u/delta/z/B/C/y, fp32 state) through the
C ABI.  Its inputs (671 MB) exceed the 126 MB L2, so no flush is needed between
steps.  Timing: W untimed warm-up steps, then K steps between CUDA events on the
launching stream, bracketed by a barrier and a device synchronize; with N > 1
ranks (one process per GPU under torchrun) every rank scans its own independent
batch (weak scaling, no data-path collective) and the max time over ranks is
used.  The same run measures the decode workload (selective_state_update,
batch 256, dim 5120, N 16, 1000 fresh tokens, L2 flushed before each token),
the backward of the same layer's scan (recomputing states from chunk
checkpoints), the exact zero-order-hold variant of the scan and of decode, the
causal conv1d + SiLU that produces the scan's input (and its decode update), with
N > 1 the million-length layer split along L over the ranks, the end-to-end path from pinned host buffers, the SM clocks during
the timed region, and (rank 0, N = 1) the fp64 CPU oracle on bounded samples.

``--impl reference`` times the CPU oracle itself as the reference arm.
Rank 0 prints exactly one JSON line on stdout: the contract keys plus short objects
for decode (last), the backward, the exact-ZOH variant, the conv1d producer and the
other scan workloads.  The full record (samples, notes, probe results) goes to stderr
on a line starting with ``DETAIL``.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = ("selective-scan fwd (b·d·L) elems/s & % of roofline; "
          "decode state-updates/s")
WORKLOAD = "m2p8b"
SM_COUNT_B200 = 148
SFU_OPS_PER_CLK_PER_SM = 16  # ex2/lg2/rcp results per clock per SM
L2_BYTES = 126 * 1024 * 1024


# ----------------------------------------------------------------------------- ranks

def dist_setup():
    """Rank, world size and local rank from torchrun's environment (1 process per GPU)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120),
                                **({"device_id": torch.device("cuda", local)}
                                   if backend == "nccl" else {}))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(value: float, world: int) -> float:
    """Host-side reduction of one timing scalar (not a data-path collective)."""
    if world == 1:
        return value
    import torch.distributed as dist
    dev = torch.device("cuda", torch.cuda.current_device()) if torch.cuda.is_available() else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(base: int, rank: int) -> int:
    """Each rank scans an independent batch: same recipe, its own seed."""
    return base + 1000 * rank


def dist_teardown(world):
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="clk_", suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), smax=float(parts[2]), power=float(parts[3]),
                                 hw=parts[5], hwt=parts[6], swt=parts[7], pcap=parts[8]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        busy = [r for r in rows if r["power"] > 250.0] or rows
        reasons = set()
        for r in busy:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in busy),
                "sm_max_mhz": max(r["smax"] for r in rows), "reasons": sorted(reasons),
                "samples": len(busy), "power_w_median": statistics.median(r["power"] for r in busy)}


# ----------------------------------------------------------------------------- helpers

def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "sm_max_mhz": 1965.0}, "fallback"


def source_digest(path: str) -> str:
    """First 16 hex digits of the SHA-256 of a CUDA source with its comments and blank-space
    differences removed: it changes when the code changes, not when a comment does.
    Several sources joined by '+' are digested together, in that order."""
    import re
    codes = []
    for part in path.split("+"):
        text = open(part, encoding="utf-8").read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        codes.append("\n".join(" ".join(line.split()) for line in text.splitlines() if line.strip()))
    return hashlib.sha256("\n".join(codes).encode()).hexdigest()[:16]


def profile_traffic(name: str, source: str):
    """DRAM bytes per launch from a committed ncu summary, if the kernel code is unchanged."""
    path = os.path.join(ROOT, "profiles", name)
    if not os.path.exists(path):
        return None
    vals = {}
    for line in open(path):
        if ":" in line:
            k, v = line.split(":", 1)
            vals[k.strip()] = v.strip()
    digest = source_digest("+".join(os.path.join(ROOT, s) for s in source.split("+")))
    recorded = vals.get("source_sha256_16", "").split()
    if not recorded or recorded[0] != digest:  # the kernel changed since the capture
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def scan_bytes(b, d, n, L, in_size=2, out_size=2):
    """Algorithmic bytes of one scan: u, delta, z, B, C read once, y written once, plus
    A, D, bias and last_state (the expanded state is never materialised)."""
    return (3 * b * d * L * in_size + 2 * b * n * L * in_size + b * d * L * out_size +
            d * n * 4 + 2 * d * 4 + b * d * n * 4)


def decode_bytes(b, d, n, io_size=2):
    """Algorithmic bytes of one decode token: the state read and written, u/delta/z and
    y per lane, B/C per batch row, A/D/bias per channel."""
    return 2 * b * d * n * 4 + 4 * b * d * io_size + 2 * b * n * io_size + d * n * 4 + 2 * d * 4


def backward_bytes(b, d, n, L, in_size=2):
    """Algorithmic bytes of one scan backward: u, delta, z, dy, B, C read once; du, ddelta,
    dz (input dtype) and dB, dC (fp32) written once; A, D, bias and their fp32 gradients.
    Checkpoint traffic is a design choice and is not counted."""
    return (4 * b * d * L * in_size + 2 * b * n * L * in_size + 3 * b * d * L * in_size +
            2 * b * n * L * 4 + 2 * d * n * 4 + 4 * d * 4)


def flush_l2(buf, rbuf=None):
    """Evict L2: write a buffer of twice its size, then (when rbuf is given) read another
    such buffer, so the write-back of the lines the first pass left dirty happens here
    and not inside the timed launch that follows."""
    buf.add_(1)  # reads and writes 2x L2 worth of bytes
    if rbuf is not None:
        rbuf.amax()  # reads 2x L2 worth of bytes, writes one scalar


def med_ms(evs):
    """Median duration (ms) of (start, end) CUDA event pairs recorded on one stream."""
    return statistics.median(a.elapsed_time(b) for a, b in evs)


# ----------------------------------------------------------------------------- our arm

def run_ours(args, rank, world, local):
    from selective_state_space_56_b200 import inputs, ops
    import selective_state_space_56_b200.build as s6build

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (B200)")
    s6build.build()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = inputs.SCAN_WORKLOADS[WORKLOAD]
    b, d, n, L = w.batch, w.dim, w.dstate, w.seqlen
    host = inputs.scan_inputs(b, d, n, L, w.in_dtype, rank_seed(w.seed, rank))
    host = {k: (v.pin_memory() if v is not None else None) for k, v in host.items()}
    g = {k: v.to(dev) for k, v in host.items()}
    y = torch.empty((b, d, L), dtype=w.out_dtype, device=dev)
    last = torch.empty((b, d, n), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        ops.selective_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], D=g["D"], z=g["z"],
                               delta_bias=g["delta_bias"], y=y, last_state=last)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)

    # Per-launch durations for the roofline: events around each launch on the launching
    # stream, inside the same timed loop.
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier(world)
        torch.cuda.synchronize(dev)
        t0.record(stream)
        for i in range(args.steps):
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        t1.record(stream)
        torch.cuda.synchronize(dev)
        barrier(world)
    ms_total = t0.elapsed_time(t1)
    ms_kernel = med_ms(ev)
    ms_total = max_over_ranks(ms_total, world)
    ms_step = ms_total / args.steps
    elems = b * d * L
    value = world * elems * args.steps / (ms_total * 1e-3)
    clocks = clk.summary()

    peaks, peak_kind = measured_peaks()
    fmax_mhz = peaks.get("sm_max_mhz", 1965.0)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    sfu_peak = sms * SFU_OPS_PER_CLK_PER_SM * fmax_mhz * 1e6       # ops/s
    exps = elems * (n + 2)                                          # Abar x N, softplus, SiLU
    achieved = exps / (ms_kernel * 1e-3)
    byts = scan_bytes(b, d, n, L)
    roofline = {
        "bound": "alu", "unit": "Gexp/s",
        "achieved": achieved / 1e9, "peak": sfu_peak / 1e9, "frac": achieved / sfu_peak,
        "traffic": profile_traffic("scan_fwd_m2p8b.txt", "selective_state_space_56_b200/csrc/scan_fwd.cu+"
                                  "selective_state_space_56_b200/csrc/s6_device.cuh"),
        "algorithmic_bytes": byts,
        "hbm_GBps": byts / (ms_kernel * 1e-3) / 1e9,
        "hbm_frac": byts / (ms_kernel * 1e-3) / 1e9 / peaks["hbm_gbs"],
        "peak_note": "SFU: %d SMs x %d ops/clk x %.0f MHz (derived); HBM peak %s %.0f GB/s" % (
            sms, SFU_OPS_PER_CLK_PER_SM, fmax_mhz, peak_kind, peaks["hbm_gbs"]),
        "kernel_ms": ms_kernel,
    }

    # End to end through the C ABI from pinned host buffers: every step's inputs copied in
    # and its y copied out inside the timed region.  Copies run on their own streams with
    # two device buffer sets, so step i+1's host-to-device copy and step i's
    # device-to-host copy overlap step i's scan (PCIe is full duplex).
    e2e_steps = max(2, min(args.steps, 12))
    names = ("u", "delta", "z", "B", "C")
    h2d = sum(host[k].numel() * host[k].element_size() for k in names)
    d2h = y.numel() * y.element_size()
    dbuf = [{k: torch.empty_like(g[k]) for k in names} for _ in range(2)]
    ybuf = [torch.empty_like(y) for _ in range(2)]
    y_host = [torch.empty(y.shape, dtype=y.dtype).pin_memory() for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    computed = [torch.cuda.Event() for _ in range(2)]
    copied_out = [torch.cuda.Event() for _ in range(2)]
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier(world)
    e0.record(stream)
    s_in.wait_event(e0)
    for i in range(e2e_steps):
        sl = i % 2
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(computed[sl])  # the scan of step i-2 is done with this set
            for k in names:
                dbuf[sl][k].copy_(host[k], non_blocking=True)
            landed = torch.cuda.Event()
            landed.record(s_in)
        stream.wait_event(landed)
        if i >= 2:
            stream.wait_event(copied_out[sl])  # y of step i-2 has left this buffer
        x = dbuf[sl]
        ops.selective_scan_fwd(x["u"], x["delta"], g["A"], x["B"], x["C"], D=g["D"], z=x["z"],
                               delta_bias=g["delta_bias"], y=ybuf[sl])
        computed[sl].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(computed[sl])
            y_host[sl].copy_(ybuf[sl], non_blocking=True)
            copied_out[sl].record(s_out)
    stream.wait_stream(s_out)
    stream.wait_stream(s_in)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world) / e2e_steps
    e2e = {"value": world * elems / (e2e_ms * 1e-3), "unit": "elems/s", "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": e2e_steps,
           "pipeline": "two buffer sets; H2D, scan and D2H on three streams"}
    del dbuf, ybuf

    decode = run_decode(dev, stream, world, steps=args.decode_steps)
    del y, last
    torch.cuda.empty_cache()
    backward = run_backward(g, dev, stream, world, w, steps=args.backward_steps)
    zoh = run_zoh(g, dev, stream, world, w, steps=args.zoh_steps)
    del g
    torch.cuda.empty_cache()
    conv = run_conv(dev, stream, world, rank, steps=args.conv_steps)
    torch.cuda.empty_cache()
    lshard = None
    if world > 1:
        try:
            lshard = run_lshard(dev, stream, world, rank, steps=args.lshard_steps)
        except Exception as e:  # reported, not fatal: the headline line must still print
            lshard = {"error": "%s: %s" % (type(e).__name__, str(e)[:200])}
        torch.cuda.empty_cache()

    workloads = run_workloads(dev, stream, world)
    probes = run_probes(dev, stream, sms, fmax_mhz)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, budget_s=args.cpu_seconds)
        backward["cpu_baseline"] = cpu_baseline_backward(w, budget_s=args.cpu_seconds / 2)
        conv["cpu_baseline"] = cpu_baseline_conv(budget_s=args.cpu_seconds / 4)

    line = {
        "metric": METRIC, "value": value, "unit": "elems/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "io_dtype": "bf16", "data": "synthetic",
        "config": {"workload": "Mamba-2.8B-shaped layer scan (m2p8b): batch 4, dim 5120, N 16, "
                               "L 4096, bf16 I/O, fp32 state",
                   "batch": b, "dim": d, "dstate": n, "seqlen": L,
                   "l2": "no flush: each step reads %.0f MB of inputs (> %d MB L2)" % (
                       (h2d) / 1e6, L2_BYTES >> 20),
                   "parallelism": "replicas x%d (independent batches per GPU)" % world},
        "roofline": roofline, "e2e": e2e, "gpu_launches": args.steps,
        "clocks": clocks, "decode": decode, "backward": backward, "exact_zoh": zoh,
        "conv1d": conv, "lshard": lshard, "workloads": workloads, "pipe_probes": probes,
        "cpu_baseline": cpu,
        "impl": "ours",
    }
    return line


def _r(x, sig=5):
    """x rounded to `sig` significant digits (ints and non-numbers unchanged)."""
    if isinstance(x, float):
        return float("%.*g" % (sig, x))
    return x


def compact_line(line):
    """The one stdout line: every contract key, the other halves of the metric and the
    side measurements as short objects, floats to five significant digits, and the decode
    workload last (the consumer keeps the end of long output).  The full record, with
    samples, notes and probe details, goes to stderr."""
    rf, cb, e2e, ck = line["roofline"], line["cpu_baseline"], line["e2e"], line["clocks"]
    out = {k: _r(line[k]) for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup",
                                     "ms_per_step", "higher_is_better", "scaling",
                                     "vs_baseline", "dtype", "io_dtype", "data", "impl")}
    cfg = line["config"]
    out["config"] = {"workload": "m2p8b layer scan (4, 5120, 16, 4096), bf16 I/O, fp32 state",
                     "batch": cfg["batch"], "dim": cfg["dim"], "dstate": cfg["dstate"],
                     "seqlen": cfg["seqlen"], "l2": "no flush: 504 MB inputs per step > 126 MB L2",
                     "parallelism": cfg["parallelism"]}
    out["roofline"] = {k: _r(rf[k]) for k in ("bound", "achieved", "peak", "unit", "frac",
                                               "traffic", "kernel_ms", "hbm_frac")}
    out["cpu_baseline"] = None if cb is None else {
        "value": _r(cb["value"]), "unit": cb["unit"], "cores": cb["cores"], "kind": cb["kind"],
        "sample": cb["sample"].split(";")[0]}
    out["e2e"] = {k: _r(e2e[k]) for k in ("value", "unit", "h2d_bytes_per_step",
                                           "d2h_bytes_per_step", "ms_per_step")}
    out["gpu_launches"] = line["gpu_launches"]
    out["clocks"] = {k: _r(ck.get(k)) for k in ("sm_mhz", "sm_max_mhz", "reasons")}
    wl = line.get("workloads") or {}
    out["workloads"] = {k: {"ms": _r(v["ms"], 4), "frac": _r(v["frac"], 4)}
                        for k, v in wl.items() if isinstance(v, dict)}
    bw, z, cv = line["backward"], line["exact_zoh"], line["conv1d"]
    out["backward"] = {"ms": _r(bw["ms_per_call"], 4), "value": _r(bw["value"], 4),
                       "frac": _r(bw["roofline"]["frac"], 4),
                       "train_ms": _r(bw["train_step"]["ms_per_step"], 4),
                       "train_frac": _r(bw["train_step"]["roofline"]["frac"], 4)}
    out["exact_zoh"] = {"ms": _r(z["ms_per_call"], 4), "frac": _r(z["roofline"]["frac"], 4),
                        "bwd_ms": _r(z["backward"]["ms_per_call"], 4),
                        "bwd_frac": _r(z["backward"]["roofline"]["frac"], 4),
                        "decode_us": _r(z["decode"]["ms_per_token_l2_flushed"] * 1e3, 4),
                        "decode_hbm_frac": _r(z["decode"]["roofline"]["frac"], 4)}
    out["conv1d"] = {"ms": _r(cv["ms_per_call"], 4), "hbm_frac": _r(cv["roofline"]["frac"], 4),
                     "bwd_ms": _r(cv["backward"]["ms_per_call"], 4),
                     "bwd_hbm_frac": _r(cv["backward"]["roofline"]["frac"], 4),
                     "decode_us": _r(cv["decode"]["ms_per_token_l2_flushed"] * 1e3, 4),
                     "decode_hbm_frac": _r(cv["decode"]["roofline"]["frac"], 4)}
    if line.get("lshard") is not None:
        ls = line["lshard"]
        out["lshard"] = {k: _r(ls[k]) for k in ("value", "ms_per_step", "n_gpus")} \
            if "value" in ls else ls
    d = line["decode"]
    dr = d["roofline"]
    out["decode"] = {"metric": d["metric"], "value": _r(d["value"]), "unit": d["unit"],
                     "steps_per_s": _r(d["steps_per_s"]),
                     "us_per_token_l2_flushed": _r(d["ms_per_token_l2_flushed"] * 1e3, 4),
                     "us_per_token_back_to_back": _r(d["ms_per_token_back_to_back"] * 1e3, 4),
                     "l2": "252 MB written then read before each token",
                     "roofline": {k: _r(dr[k]) for k in ("bound", "achieved", "peak", "unit",
                                                          "frac", "traffic")}}
    return out


def run_probes(dev, stream, sms, fmax_mhz, reps=3):
    """Measured throughput of the pipes the rooflines are stated against (the library's
    probe: 8 independent chains per thread, 8 CTAs of 256 threads per SM): SFU ex2,
    fp32 FMA, packed fp32x2 FMA, each the best of `reps` launches of a few ms, beside the
    rate derived from unit counts and the maximum SM clock."""
    from selective_state_space_56_b200 import ops
    blocks = sms * 8
    sink = torch.empty(blocks * 256, dtype=torch.float32, device=dev)
    derived = {"sfu_ex2": sms * SFU_OPS_PER_CLK_PER_SM * fmax_mhz * 1e6,
               "ffma": sms * 128 * fmax_mhz * 1e6, "ffma2": sms * 128 * fmax_mhz * 1e6}
    iters = {"sfu_ex2": 8192, "ffma": 65536, "ffma2": 32768}
    out = {}
    with torch.cuda.stream(stream):
        for kind in ("sfu_ex2", "ffma", "ffma2"):
            ops.diag_throughput(kind, blocks, 64, sink)  # warm-up
            best = float("inf")
            for _ in range(reps):
                a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                n = ops.diag_throughput(kind, blocks, iters[kind], sink)
                e.record(stream)
                e.synchronize()
                best = min(best, a.elapsed_time(e))
            rate = n / (best * 1e-3)
            out[kind] = {"results_per_s": rate, "derived_per_s": derived[kind],
                         "frac_of_derived": rate / derived[kind], "ms": best}
    ops.check_device_error()
    out["note"] = ("derived: %d SMs x (SFU 16, FMA 128 fp32 results)/clk x %.0f MHz; ffma2 counts "
                   "two fp32 results per instruction" % (sms, fmax_mhz))
    return out


def run_zoh(g, dev, stream, world, w, steps=50):
    """The exact zero-order-hold variant (MAMBA_FLAG_EXACT_ZOH): the m2p8b scan per launch,
    its backward per call, and decode tokens after an L2 flush, each timed with events on the
    launching stream."""
    from selective_state_space_56_b200 import inputs, ops
    b, d, n, L = w.batch, w.dim, w.dstate, w.seqlen
    y = torch.empty((b, d, L), dtype=w.out_dtype, device=dev)

    def scan():
        ops.selective_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], D=g["D"], z=g["z"],
                               delta_bias=g["delta_bias"], y=y, exact_zoh=True)

    for _ in range(3):
        scan()
    torch.cuda.synchronize(dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for a, b_ in evs:
        a.record(stream)
        scan()
        b_.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(med_ms(evs), world)
    elems = b * d * L
    peaks, kind = measured_peaks()
    fmax_mhz = peaks.get("sm_max_mhz", 1965.0)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    sfu_peak = sms * SFU_OPS_PER_CLK_PER_SM * fmax_mhz * 1e6
    exps = elems * (n + 2)
    del y

    # its backward (checkpoint pass with the ZOH weight + sweep), for a fixed dy
    gen = torch.Generator(device=dev)
    gen.manual_seed(w.seed + 7)
    dy = torch.randn((b, d, L), generator=gen, device=dev).to(w.in_dtype)
    ws = torch.empty(ops.selective_scan_bwd_workspace_size(b, d, n, L), dtype=torch.uint8,
                     device=dev)

    def bwd():
        return ops.selective_scan_bwd(g["u"], g["delta"], g["A"], g["B"], g["C"], dy, D=g["D"],
                                      z=g["z"], delta_bias=g["delta_bias"], workspace=ws,
                                      exact_zoh=True)

    for _ in range(3):
        bwd()
    torch.cuda.synchronize(dev)
    bevs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(max(3, steps // 5))]
    for a, b_ in bevs:
        a.record(stream)
        bwd()
        b_.record(stream)
    torch.cuda.synchronize(dev)
    ms_bwd = max_over_ranks(med_ms(bevs), world)
    sfu_bwd = elems * (2 * n + 4)  # as the Delta*B backward: the weight needs no SFU result
    del dy, ws

    dw = inputs.DECODE_WORKLOAD
    prm = {k: v.to(dev) for k, v in inputs.decode_params(dw).items()}
    state = prm["state0"].clone()
    toks = inputs.decode_tokens_batched(steps, dw, device=dev)
    yd = torch.empty((dw.batch, dw.dim), dtype=dw.io_dtype, device=dev)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    rflush = torch.zeros(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)

    def tok(s):
        ops.selective_state_update(state, toks["u"][s], toks["delta"][s], prm["A"], toks["B"][s],
                                   toks["C"][s], D=prm["D"], z=toks["z"][s],
                                   delta_bias=prm["delta_bias"], y=yd, exact_zoh=True)

    for s in range(3):
        tok(s)
    torch.cuda.synchronize(dev)
    devs = []
    for s in range(steps):
        flush_l2(flush, rflush)
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        tok(s)
        b_.record(stream)
        devs.append((a, b_))
    torch.cuda.synchronize(dev)
    ms_tok = max_over_ranks(med_ms(devs), world)
    byts = decode_bytes(dw.batch, dw.dim, dw.dstate)
    del toks, flush, rflush, state
    return {
        "metric": "selective-scan fwd with exact ZOH Bbar, (b·d·L) elems/s", "unit": "elems/s",
        "value": world * elems / (ms * 1e-3), "ms_per_call": ms, "steps": steps,
        "workload": "m2p8b scan (batch 4, dim 5120, N 16, L 4096, bf16 I/O) with "
                    "Bbar = (exp(Delta A) - 1) / A * B",
        "roofline": {"bound": "alu", "unit": "Gexp/s", "achieved": exps / (ms * 1e-3) / 1e9,
                     "peak": sfu_peak / 1e9, "frac": exps / (ms * 1e-3) / sfu_peak,
                     "traffic": profile_traffic(
                         "scan_zoh_m2p8b.txt", "selective_state_space_56_b200/csrc/scan_fwd.cu+"
                         "selective_state_space_56_b200/csrc/s6_device.cuh"),
                     "note": "same N + 2 SFU exponentials per element as the Delta*B scan; the "
                             "exact weight adds FMA-pipe work (series + select), not SFU work"},
        "backward": {"ms_per_call": ms_bwd, "value": world * elems / (ms_bwd * 1e-3),
                     "unit": "elems/s",
                     "roofline": {"bound": "alu", "unit": "Gop/s (SFU)",
                                  "achieved": sfu_bwd / (ms_bwd * 1e-3) / 1e9,
                                  "peak": sfu_peak / 1e9,
                                  "frac": sfu_bwd / (ms_bwd * 1e-3) / sfu_peak,
                                  "sfu_ops_per_elem": 2 * n + 4}},
        "decode": {"ms_per_token_l2_flushed": ms_tok,
                   "value": world * dw.batch * dw.dim / (ms_tok * 1e-3),
                   "unit": "(b,d) lane updates/s",
                   "roofline": {"bound": "hbm", "unit": "GB/s",
                                "achieved": byts / (ms_tok * 1e-3) / 1e9, "peak": peaks["hbm_gbs"],
                                "frac": byts / (ms_tok * 1e-3) / 1e9 / peaks["hbm_gbs"],
                                "peak_kind": kind}},
        "gpu_launches": 2 * steps + 6 + 2 * (max(3, steps // 5) + 3),
    }


def run_conv(dev, stream, world, rank, steps=50):
    """The causal conv1d + SiLU producing the m2p8b layer's u (4, 5120, 4096, K = 4, bf16),
    per launch, its backward per call, and its decode update on (256, 5120) after an L2
    flush."""
    from selective_state_space_56_b200 import inputs, ops
    b, d, L, K = 4, 5120, 4096, inputs.CONV_WIDTH
    p = inputs.conv_inputs(b, d, L, K, torch.bfloat16, seed=rank_seed(inputs.CONV_SEED, rank),
                           device=dev)
    out = torch.empty_like(p["x"])
    fin = torch.empty((b, d, K - 1), dtype=torch.bfloat16, device=dev)

    def conv():
        ops.causal_conv1d_fwd(p["x"], p["weight"], p["bias"], out=out)

    for _ in range(3):
        conv()
    torch.cuda.synchronize(dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for a, b_ in evs:
        a.record(stream)
        conv()
        b_.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(med_ms(evs), world)
    elems = b * d * L
    byts = 2 * elems * 2 + d * K * 4 + d * 4  # x read, out written (bf16), weights, bias
    peaks, kind = measured_peaks()
    del out, fin

    # the backward: x and dout read, dx written (bf16); dweight, dbias summed in place
    gen = torch.Generator(device=dev)
    gen.manual_seed(inputs.CONV_SEED + 2)
    dout = torch.randn((b, d, L), generator=gen, device=dev).to(torch.bfloat16)

    def conv_bwd():
        return ops.causal_conv1d_bwd(p["x"], p["weight"], dout, p["bias"])

    for _ in range(3):
        conv_bwd()
    torch.cuda.synchronize(dev)
    bevs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(steps)]
    for a, b_ in bevs:
        a.record(stream)
        conv_bwd()
        b_.record(stream)
    torch.cuda.synchronize(dev)
    ms_bwd = max_over_ranks(med_ms(bevs), world)
    bbytes = 3 * elems * 2 + d * K * 4 * 2 + d * 4 * 2  # x, dout, dx; weights in, gradients out
    del dout

    db, dd = 256, 5120
    gen = torch.Generator(device=dev)
    gen.manual_seed(inputs.CONV_SEED + 1)
    state = torch.randn((db, dd, K - 1), generator=gen, device=dev).to(torch.bfloat16)
    xs = torch.randn((steps, db, dd), generator=gen, device=dev).to(torch.bfloat16)
    wd, bd = p["weight"][:dd].contiguous(), p["bias"][:dd].contiguous()
    yd = torch.empty((db, dd), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    rflush = torch.zeros(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    for s_ in range(3):
        ops.causal_conv1d_update(state, xs[s_], wd, bd, out=yd)
    torch.cuda.synchronize(dev)
    devs = []
    for s_ in range(steps):
        flush_l2(flush, rflush)
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        ops.causal_conv1d_update(state, xs[s_], wd, bd, out=yd)
        b_.record(stream)
        devs.append((a, b_))
    torch.cuda.synchronize(dev)
    ms_tok = max_over_ranks(med_ms(devs), world)
    rows = db * dd
    dbytes = rows * (2 * (K - 1) * 2 + 2 * 2) + dd * (K + 1) * 4
    del p, state, xs, flush, rflush
    return {
        "metric": "causal conv1d + SiLU (b·d·L) elems/s", "unit": "elems/s",
        "value": world * elems / (ms * 1e-3), "ms_per_call": ms, "steps": steps,
        "workload": "x (4, 5120, 4096) bf16, weight (5120, 4) and bias fp32, SiLU: the "
                    "producer of the m2p8b layer's u",
        "roofline": {"bound": "hbm", "unit": "GB/s", "achieved": byts / (ms * 1e-3) / 1e9,
                     "peak": peaks["hbm_gbs"], "frac": byts / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                     "algorithmic_bytes": byts, "peak_kind": kind,
                     "traffic": profile_traffic("conv1d_m2p8b.txt",
                                                "selective_state_space_56_b200/csrc/conv1d.cu")},
        "backward": {"ms_per_call": ms_bwd, "value": world * elems / (ms_bwd * 1e-3),
                     "unit": "elems/s",
                     "workload": "gradients of the same conv for a fixed dout (4, 5120, 4096) "
                                 "bf16: dx bf16, dweight and dbias fp32",
                     "roofline": {"bound": "hbm", "unit": "GB/s",
                                  "achieved": bbytes / (ms_bwd * 1e-3) / 1e9,
                                  "peak": peaks["hbm_gbs"],
                                  "frac": bbytes / (ms_bwd * 1e-3) / 1e9 / peaks["hbm_gbs"],
                                  "algorithmic_bytes": bbytes, "peak_kind": kind,
                                  "traffic": profile_traffic(
                                      "conv1d_bwd_m2p8b.txt",
                                      "selective_state_space_56_b200/csrc/conv1d.cu")}},
        "decode": {"ms_per_token_l2_flushed": ms_tok,
                   "workload": "conv state (256, 5120, 3) bf16 updated in place, x and out "
                               "(256, 5120) bf16",
                   "roofline": {"bound": "hbm", "unit": "GB/s",
                                "achieved": dbytes / (ms_tok * 1e-3) / 1e9,
                                "peak": peaks["hbm_gbs"],
                                "frac": dbytes / (ms_tok * 1e-3) / 1e9 / peaks["hbm_gbs"],
                                "algorithmic_bytes": dbytes}},
        "gpu_launches": 3 * steps + 9,
    }


def run_lshard(dev, stream, world, rank, steps=5):
    """The million-length layer (1, 2048, 16, 2^20, bf16) split along L over the ranks:
    each rank scans its consecutive shard after one all-gather of segment summaries
    (strong scaling: the whole sequence per step)."""
    from selective_state_space_56_b200 import inputs, sharded
    import torch.distributed as dist
    w = inputs.SCAN_WORKLOADS["million"]
    Ls = w.seqlen // world
    p = inputs.scan_inputs(w.batch, w.dim, w.dstate, Ls, w.in_dtype,
                           rank_seed(w.seed + 100, rank), device=dev)

    def step():
        return sharded.sharded_selective_scan_fwd(p["u"], p["delta"], p["A"], p["B"], p["C"],
                                                  D=p["D"], z=p["z"], delta_bias=p["delta_bias"])

    for _ in range(2):
        step()
    torch.cuda.synchronize(dev)
    dist.barrier()
    a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        step()
    b_.record(stream)
    torch.cuda.synchronize(dev)
    dist.barrier()
    ms = max_over_ranks(a.elapsed_time(b_) / steps, world)
    elems = w.batch * w.dim * w.seqlen
    del p
    return {"metric": "L-sharded selective-scan fwd (b·d·L) elems/s", "unit": "elems/s",
            "value": elems / (ms * 1e-3), "ms_per_step": ms, "steps": steps,
            "scaling": "strong", "n_gpus": world,
            "workload": "million-length layer (1, 2048, 16, 2^20) bf16, %d steps per rank, one "
                        "all-gather of b*d*(N+1) fp32 summaries per step" % Ls}


def run_backward(g, dev, stream, world, w, steps=50):
    """Backward of the m2p8b scan (gradients of every input for a fixed dy), each call
    timed with events on the launching stream; inputs exceed L2, so no flush."""
    from selective_state_space_56_b200 import ops
    b, d, n, L = w.batch, w.dim, w.dstate, w.seqlen
    gen = torch.Generator(device=dev)
    gen.manual_seed(w.seed + 7)
    dy = torch.randn((b, d, L), generator=gen, device=dev).to(w.in_dtype)
    ws = torch.empty(ops.selective_scan_bwd_workspace_size(b, d, n, L), dtype=torch.uint8,
                     device=dev)

    def call():
        return ops.selective_scan_bwd(g["u"], g["delta"], g["A"], g["B"], g["C"], dy, D=g["D"],
                                      z=g["z"], delta_bias=g["delta_bias"], workspace=ws)

    for _ in range(3):
        call()
    torch.cuda.synchronize(dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for a, b_ in evs:
        a.record(stream)
        call()
        b_.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(med_ms(evs), world)
    elems = b * d * L
    peaks, kind = measured_peaks()
    fmax_mhz = peaks.get("sm_max_mhz", 1965.0)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    sfu_peak = sms * SFU_OPS_PER_CLK_PER_SM * fmax_mhz * 1e6
    # SFU results the recomputing backward needs per element: Abar twice (states rebuilt,
    # then swept), softplus, sigmoid of the step (softplus'), sigmoid of the gate (ex2, rcp)
    sfu = elems * (2 * n + 4)
    byts = backward_bytes(b, d, n, L)

    # a training step: the forward recording the checkpoints, then the backward from them
    y = torch.empty((b, d, L), dtype=w.out_dtype, device=dev)

    def train_step():
        ops.selective_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], D=g["D"], z=g["z"],
                               delta_bias=g["delta_bias"], y=y, checkpoints=ws)
        return ops.selective_scan_bwd(g["u"], g["delta"], g["A"], g["B"], g["C"], dy, D=g["D"],
                                      z=g["z"], delta_bias=g["delta_bias"], checkpoints=ws)

    for _ in range(3):
        train_step()
    torch.cuda.synchronize(dev)
    tevs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(steps)]
    for a, b_ in tevs:
        a.record(stream)
        train_step()
        b_.record(stream)
    torch.cuda.synchronize(dev)
    ms_train = max_over_ranks(med_ms(tevs), world)
    sfu_train = elems * (3 * n + 6)  # forward N + 2, backward 2N + 4
    train = {"ms_per_step": ms_train, "value": world * elems / (ms_train * 1e-3),
             "unit": "elems/s",
             "what": "forward recording the backward's checkpoints, then the backward from "
                     "them (no checkpointing pass of its own)",
             "roofline": {"bound": "alu", "unit": "Gop/s (SFU)",
                          "achieved": sfu_train / (ms_train * 1e-3) / 1e9,
                          "peak": sfu_peak / 1e9, "frac": sfu_train / (ms_train * 1e-3) / sfu_peak,
                          "sfu_ops_per_elem": 3 * n + 6}}
    del dy, ws, y
    return {
        "metric": "selective-scan bwd (b·d·L) elems/s", "unit": "elems/s",
        "value": world * elems / (ms * 1e-3), "ms_per_call": ms, "steps": steps,
        "workload": "backward of the m2p8b scan: batch 4, dim 5120, N 16, L 4096, bf16 "
                    "inputs and du/ddelta/dz, fp32 dA/dB/dC/dD/dbias",
        "roofline": {"bound": "alu", "unit": "Gop/s (SFU)", "achieved": sfu / (ms * 1e-3) / 1e9,
                     "peak": sfu_peak / 1e9, "frac": sfu / (ms * 1e-3) / sfu_peak,
                     "sfu_ops_per_elem": 2 * n + 4,
                     "algorithmic_bytes": byts, "hbm_GBps": byts / (ms * 1e-3) / 1e9,
                     "hbm_frac": byts / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], "peak_kind": kind,
                     "traffic": profile_traffic("scan_bwd_m2p8b.txt",
                                                "selective_state_space_56_b200/csrc/scan_bwd.cu")},
        "train_step": train,
        "gpu_launches": 2 * steps + 6 + 2 * (steps + 3),
    }


def run_workloads(dev, stream, world, steps=20):
    """The forward scan on the other scan workloads of the metric: the Mamba-130M-shaped
    layer (8, 1536, 16, 2048) and the million-length layer (1, 2048, 16, 2^20, split along
    L inside the call), each call timed with events (median), against the same SFU
    roofline of N + 2 exponentials per element; and the million-length layer's backward
    (swept in segments inside the call) against its 2N + 4."""
    from selective_state_space_56_b200 import inputs, ops
    peaks, _ = measured_peaks()
    fmax_mhz = peaks.get("sm_max_mhz", 1965.0)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    sfu_peak = sms * SFU_OPS_PER_CLK_PER_SM * fmax_mhz * 1e6
    out = {}
    launches = 0
    for name, reps in (("m130m", steps), ("million", max(3, steps // 4))):
        w = inputs.SCAN_WORKLOADS[name]
        p = inputs.scan_inputs(w.batch, w.dim, w.dstate, w.seqlen, w.in_dtype, w.seed, device=dev)
        y = torch.empty((w.batch, w.dim, w.seqlen), dtype=w.out_dtype, device=dev)
        nws = ops.selective_scan_workspace_size(w.batch, w.dim, w.dstate, w.seqlen)
        ws = torch.empty(nws, dtype=torch.uint8, device=dev) if nws else None

        def call():
            ops.selective_scan_fwd(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"],
                                   z=p["z"], delta_bias=p["delta_bias"], y=y, workspace=ws)

        for _ in range(3):
            call()
        torch.cuda.synchronize(dev)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(reps)]
        for a, b_ in evs:
            a.record(stream)
            call()
            b_.record(stream)
        torch.cuda.synchronize(dev)
        ms = max_over_ranks(med_ms(evs), world)
        elems = w.batch * w.dim * w.seqlen
        out[name] = {"ms": ms, "value": world * elems / (ms * 1e-3),
                     "frac": elems * (w.dstate + 2) / (ms * 1e-3) / sfu_peak}
        launches += (reps + 3) * (3 if nws else 1)
        del y, ws
        if name == "million":
            gen = torch.Generator(device=dev)
            gen.manual_seed(w.seed + 7)
            dy = torch.randn((w.batch, w.dim, w.seqlen), generator=gen, device=dev).to(w.in_dtype)
            wsb = torch.empty(ops.selective_scan_bwd_workspace_size(w.batch, w.dim, w.dstate,
                                                                    w.seqlen),
                              dtype=torch.uint8, device=dev)

            def bwd():
                ops.selective_scan_bwd(p["u"], p["delta"], p["A"], p["B"], p["C"], dy, D=p["D"],
                                       z=p["z"], delta_bias=p["delta_bias"], workspace=wsb)

            bwd()
            torch.cuda.synchronize(dev)
            bevs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                    for _ in range(3)]
            for a, b_ in bevs:
                a.record(stream)
                bwd()
                b_.record(stream)
            torch.cuda.synchronize(dev)
            mb = max_over_ranks(med_ms(bevs), world)
            out["million_bwd"] = {"ms": mb, "value": world * elems / (mb * 1e-3),
                                  "frac": elems * (2 * w.dstate + 4) / (mb * 1e-3) / sfu_peak}
            launches += 4 * 6  # checkpoint split (2 + fold), summary, fold, sweep
            del dy, wsb
        del p
        torch.cuda.empty_cache()
    out["gpu_launches"] = launches
    return out


def run_decode(dev, stream, world, steps=1000):
    """Decode workload: 1000 tokens with fresh seeded inputs; each token timed alone with
    events after an L2 flush (the 84 MB state would otherwise stay in the 126 MB L2)."""
    from selective_state_space_56_b200 import inputs, ops
    w = inputs.DECODE_WORKLOAD
    prm = {k: v.to(dev) for k, v in inputs.decode_params(w).items()}
    state = prm["state0"].clone()
    allt = inputs.decode_tokens_batched(steps, w, device=dev)
    toks = [{k: v[s] for k, v in allt.items()} for s in range(steps)]
    y = torch.empty((w.batch, w.dim), dtype=w.io_dtype, device=dev)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    rflush = torch.zeros(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)

    def tok(x):
        ops.selective_state_update(state, x["u"], x["delta"], prm["A"], x["B"], x["C"],
                                   D=prm["D"], z=x["z"], delta_bias=prm["delta_bias"], y=y)

    for x in toks[:5]:
        tok(x)
    torch.cuda.synchronize(dev)
    evs = []
    for x in toks:
        flush_l2(flush, rflush)
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        tok(x)
        b_.record(stream)
        evs.append((a, b_))
    torch.cuda.synchronize(dev)
    ms_cold = med_ms(evs)
    # with the write-only flush, the flush's own dirty lines are written back during the
    # token: for context
    wevs = []
    for x in toks[: max(5, len(toks) // 5)]:
        flush_l2(flush)
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        tok(x)
        b_.record(stream)
        wevs.append((a, b_))
    torch.cuda.synchronize(dev)
    ms_wflush = med_ms(wevs)
    # back to back (state L2-resident between tokens), for context
    a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for x in toks:
        tok(x)
    b_.record(stream)
    torch.cuda.synchronize(dev)
    ms_warm = a.elapsed_time(b_) / steps
    ms_cold = max_over_ranks(ms_cold, world)
    peaks, kind = measured_peaks()
    byts = decode_bytes(w.batch, w.dim, w.dstate)
    lanes = w.batch * w.dim
    del toks, allt, flush, rflush
    return {
        "metric": "decode state-updates/s", "unit": "(b,d) lane updates/s",
        "value": world * lanes / (ms_cold * 1e-3), "steps_per_s": 1e3 / ms_cold,
        "ms_per_token_l2_flushed": ms_cold, "ms_per_token_back_to_back": ms_warm,
        "ms_per_token_write_flush_only": ms_wflush,
        "l2": "flushed before every token: 252 MB written, then 252 MB read",
        "workload": "decode: batch 256, dim 5120, N 16, bf16 I/O, fp32 state, %d fresh tokens" % steps,
        "roofline": {"bound": "hbm", "unit": "GB/s", "achieved": byts / (ms_cold * 1e-3) / 1e9,
                     "peak": peaks["hbm_gbs"], "frac": byts / (ms_cold * 1e-3) / 1e9 / peaks["hbm_gbs"],
                     "algorithmic_bytes": byts, "peak_kind": kind,
                     "traffic": profile_traffic("state_update_decode.txt",
                                                "selective_state_space_56_b200/csrc/state_update.cu")},
        "gpu_launches": 2 * steps + 5 + len(wevs),
    }


# ----------------------------------------------------------------------------- oracle arm

def _oracle_sample(p, w, nl, rng):
    """Seconds the oracle (as it stands) takes on nl random channels of the workload."""
    import oracle
    bi = rng.integers(0, w.batch, nl)
    di = rng.integers(0, w.dim, nl)
    t = time.perf_counter()
    oracle.scan_lanes(p["u"][bi, di], p["delta"][bi, di], p["A"][di], p["B"], p["C"], bi,
                      D=p["D"][di], z=p["z"][bi, di], delta_bias=p["delta_bias"][di])
    return time.perf_counter() - t


def _oracle_channels(p, w, budget_s, rng):
    """Channels the oracle scans in about budget_s seconds (calibrated on a small sample)."""
    import oracle
    probe = max(4 * oracle.num_threads(), 32)  # large enough that fixed costs do not dominate
    t = _oracle_sample(p, w, probe, rng)
    return int(min(w.batch * w.dim, max(probe, probe * budget_s / max(t, 1e-3))))


def _oracle_rate(p, w, budget_s, rng):
    """(elements/s, channels, seconds) of the oracle on a sample of about budget_s seconds."""
    nl = _oracle_channels(p, w, budget_s, rng)
    t = _oracle_sample(p, w, nl, rng)
    return nl * w.seqlen / t, nl, t


def cpu_baseline(w, budget_s=10.0, p=None):
    """The fp64 oracle as it stands, on a bounded channel sample of the same workload, on
    every core and (a quarter of the budget) on one thread."""
    import numpy as np
    import oracle
    from selective_state_space_56_b200 import inputs

    if p is None:
        p = inputs.workload_inputs(w)
    rng = np.random.default_rng(0)
    cores = oracle.num_threads()
    value, nl, t = _oracle_rate(p, w, budget_s, rng)
    prev = oracle.set_num_threads(1)
    try:
        v1, n1, t1 = _oracle_rate(p, w, budget_s / 4, rng)
    finally:
        oracle.set_num_threads(prev)
    return {"value": value, "unit": "elems/s", "cores": cores, "kind": "oracle",
            "cpu_model": cpu_model(), "single_thread_value": v1,
            "sample": "%d of %d channels x full L=%d (fp64, sequential per channel, %d OpenMP "
                      "threads), %.1f s; single thread: %d channels, %.1f s" % (
                          nl, w.batch * w.dim, w.seqlen, cores, t, n1, t1)}


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline_backward(w, budget_s=5.0):
    """The fp64 oracle's backward as it stands, on a bounded channel sample."""
    import numpy as np
    import oracle
    from selective_state_space_56_b200 import inputs

    p = inputs.workload_inputs(w)
    rng = np.random.default_rng(1)
    dy_all = None

    def run(nl):
        nonlocal dy_all
        bi = rng.integers(0, w.batch, nl)
        di = rng.integers(0, w.dim, nl)
        dy = rng.standard_normal((nl, w.seqlen))
        t = time.perf_counter()
        oracle.scan_backward_lanes(p["u"][bi, di], p["delta"][bi, di], p["A"][di], p["B"], p["C"],
                                   bi, dy, D=p["D"][di], z=p["z"][bi, di],
                                   delta_bias=p["delta_bias"][di])
        return time.perf_counter() - t

    t = run(8)
    nl = int(min(w.batch * w.dim, max(8, 8 * budget_s / max(t, 1e-3))))
    t = run(nl)
    return {"value": nl * w.seqlen / t, "unit": "elems/s", "cores": 1, "kind": "oracle",
            "sample": "%d of %d channels x full L=%d (fp64 backward, one thread), %.1f s" % (
                nl, w.batch * w.dim, w.seqlen, t)}


def cpu_baseline_conv(budget_s=2.5):
    """The fp64 oracle's causal conv1d as it stands, on a bounded channel sample of the
    m2p8b producer workload."""
    import oracle
    from selective_state_space_56_b200 import inputs
    p = inputs.conv_inputs(4, 5120, 4096, inputs.CONV_WIDTH, torch.bfloat16)

    def run(nch):
        t = time.perf_counter()
        oracle.causal_conv1d(p["x"][:, :nch], p["weight"][:nch], p["bias"][:nch])
        return time.perf_counter() - t

    t = run(16)
    nch = int(min(5120, max(16, 16 * budget_s / max(t, 1e-3))))
    t = run(nch)
    return {"value": 4 * nch * 4096 / t, "unit": "elems/s", "cores": 1, "kind": "oracle",
            "sample": "4 x %d of 5120 channels x L=4096 (fp64, one thread), %.1f s" % (nch, t)}


def run_reference(args, rank, world):
    """The reference arm: the CPU oracle as it stands, on the host cores, each step a
    bounded channel sample of the m2p8b workload; the whole run takes about two minutes
    whatever K and W are (the inputs are drawn once)."""
    import numpy as np
    from selective_state_space_56_b200 import inputs
    w = inputs.SCAN_WORKLOADS[WORKLOAD]
    if rank != 0:
        return None
    p = inputs.workload_inputs(w)
    rng = np.random.default_rng(1)
    # every step one fixed-size sample, sized once so that all steps take about two minutes
    per_step = max(0.02, min(20.0, 120.0 / max(1, args.steps + args.warmup)))
    nl = _oracle_channels(p, w, per_step, rng)
    for _ in range(args.warmup):
        _oracle_sample(p, w, nl, rng)
    rates = [nl * w.seqlen / _oracle_sample(p, w, nl, rng) for _ in range(args.steps)]
    v = statistics.fmean(rates)
    cpu = cpu_baseline(w, budget_s=4.0, p=p)
    cpu["value"] = v
    cpu["sample"] = ("each step %d random channels at full L=%d (about %.3f s; fp64, %d OpenMP "
                     "threads); " % (nl, w.seqlen, per_step, cpu["cores"])) + cpu["sample"]
    return {"metric": METRIC, "value": v, "unit": "elems/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": w.batch * w.dim * w.seqlen / v * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": "Mamba-2.8B-shaped layer scan (m2p8b): batch 4, dim 5120, "
                                   "N 16, L 4096; each step a bounded channel sample",
                       "batch": w.batch, "dim": w.dim, "dstate": w.dstate, "seqlen": w.seqlen},
            "cpu_baseline": cpu,
            "e2e": {"value": v, "unit": "elems/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}


def profile_target(which):
    """Three launches of the scan (m2p8b) or of its exact-ZOH variant, eight decode tokens
    (each after an L2 flush),
    two backward calls of the m2p8b scan, or three conv1d launches (forward or backward),
    for ncu captures."""
    from selective_state_space_56_b200 import inputs, ops
    import selective_state_space_56_b200.build as s6build
    s6build.build()
    dev = torch.device("cuda", 0)
    if which in ("scan", "zoh"):
        w = inputs.SCAN_WORKLOADS[WORKLOAD]
        p = inputs.scan_inputs(w.batch, w.dim, w.dstate, w.seqlen, w.in_dtype, w.seed, device=dev)
        y = torch.empty((w.batch, w.dim, w.seqlen), dtype=w.out_dtype, device=dev)
        for _ in range(3):
            ops.selective_scan_fwd(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"], z=p["z"],
                                   delta_bias=p["delta_bias"], y=y, exact_zoh=which == "zoh")
    elif which in ("conv", "conv_bwd"):
        p = inputs.conv_inputs(4, 5120, 4096, inputs.CONV_WIDTH, torch.bfloat16, device=dev)
        dout = torch.randn((4, 5120, 4096), device=dev).to(torch.bfloat16)
        for _ in range(3):
            if which == "conv":
                ops.causal_conv1d_fwd(p["x"], p["weight"], p["bias"])
            else:
                ops.causal_conv1d_bwd(p["x"], p["weight"], dout, p["bias"])
    elif which == "backward":
        w = inputs.SCAN_WORKLOADS[WORKLOAD]
        p = inputs.scan_inputs(w.batch, w.dim, w.dstate, w.seqlen, w.in_dtype, w.seed, device=dev)
        gen = torch.Generator(device=dev)
        gen.manual_seed(w.seed + 7)
        dy = torch.randn((w.batch, w.dim, w.seqlen), generator=gen, device=dev).to(w.in_dtype)
        for _ in range(2):
            ops.selective_scan_bwd(p["u"], p["delta"], p["A"], p["B"], p["C"], dy, D=p["D"],
                                   z=p["z"], delta_bias=p["delta_bias"])
    else:
        w = inputs.DECODE_WORKLOAD
        prm = {k: v.to(dev) for k, v in inputs.decode_params(w).items()}
        state = prm["state0"].clone()
        toks = inputs.decode_tokens_batched(8, w, device=dev)
        y = torch.empty((w.batch, w.dim), dtype=w.io_dtype, device=dev)
        flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
        rflush = torch.zeros(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
        for s in range(8):  # every token after an L2 flush, as the bench times them
            flush_l2(flush, rflush)
            ops.selective_state_update(state, toks["u"][s], toks["delta"][s], prm["A"], toks["B"][s],
                                       toks["C"][s], D=prm["D"], z=toks["z"][s],
                                       delta_bias=prm["delta_bias"], y=y)
    torch.cuda.synchronize(dev)
    ops.check_device_error()


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[1])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--decode-steps", type=int, default=1000)
    ap.add_argument("--backward-steps", type=int, default=50)
    ap.add_argument("--zoh-steps", type=int, default=50)
    ap.add_argument("--conv-steps", type=int, default=50)
    ap.add_argument("--lshard-steps", type=int, default=5)
    ap.add_argument("--profile", choices=["scan", "zoh", "decode", "backward", "conv", "conv_bwd"],
                    help="run a few untimed launches of one workload (an ncu capture target) "
                         "and exit")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.profile:
        profile_target(args.profile)
        return
    if args.impl == "reference":
        # The oracle arm runs on rank 0's host cores only; other ranks have no work and
        # take part in no collective.
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    rank, world, local = dist_setup()
    try:
        line = run_ours(args, rank, world, local)
        if rank == 0:
            print("DETAIL " + json.dumps(line), file=sys.stderr, flush=True)
            print(json.dumps(compact_line(line)), flush=True)
    finally:
        dist_teardown(world)


if __name__ == "__main__":
    main()
