#!/usr/bin/env python3
"""Benchmark of the FP4 microscaling hot path on B200.

Default workload (one GPU): activation quantize + rotate -- X bf16 4096 x 4096,
entries N(0,1) with 40 seeded channels x20; each step runs FWHT-128 + MXFP4
(group 32, truncation-free E8M0) once with round-to-nearest-even and once
with Philox stochastic rounding (seed 7).  value = algorithmic bytes moved
(one read of X plus codes and scales, 2.531 B/element per run) / step time.

Also reported: the roofline of the dominant kernel (live CUDA-event
durations, measured HBM peak), the block-scaled FP4 GEMM of the NVFP4
forward linear (8192 x 11008 x 4096) in TFLOP/s against the dense FP4 peak,
the largest configuration's calls (`largest_config`: the 2^30-element
quantize, FWHT + MXFP4 and NVFP4 under a given amax, and the fused rotate +
quantize + GEMM at 16384 x 14336 x 4096), the end-to-end figure through host
buffers, SM clocks sampled during the timed region, and the CPU oracle on
the host cores (single-threaded and row-partitioned over every core, plus
the binary64 oracle GEMM on a sub-problem, extrapolated by flops).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
Under torchrun (N > 1) every rank runs the same per-GPU workload (weak
scaling, no data-path collective); rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "FP4 quantize GB/s (% of HBM peak); block-scaled FP4 GEMM TFLOPS (% of peak)"
M2, K2 = 4096, 4096
BYTES_PER_ELEM_MXFP4 = 2 + 0.5 + 1 / 32           # bf16 read + E2M1 codes + E8M0 scales
EV_EVERY = 8                                       # steps bracketed by per-launch events
N_BUFS = 8                                         # rotating input/output sets: 8 x 40.5 MB > L2 (126 MB)
FP4_PER_BF16 = 4.0                                 # nominal dense FP4 : BF16 tensor throughput (9 : 2.25 PF)
GEMM_SHAPE = (8192, 11008, 4096)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="libqfp4", choices=["libqfp4", "reference"])
    ap.add_argument("--no-gemm", action="store_true", help="skip the GEMM sub-measurement")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--no-cfg5", action="store_true", help="skip the largest-configuration sub-measurements")
    ap.add_argument("--profile-case", choices=["quant", "gemm", "quant-nvfp4", "backward", "backward-sr", "dequant"],
                    default=None,
                    help="run a few untimed calls of one kernel family (for ncu captures) and exit")
    ap.add_argument("--rows", nargs="?", const="", default=None, metavar="FILTER",
                    help="time every entry point of the path on its own full-size workload (one JSON line each); "
                         "FILTER keeps only the rows whose label contains it")
    return ap.parse_args()


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained"), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


# the source files each profiled kernel is built from (its ncu figures stay
# valid while these are unchanged)
KERNEL_SOURCES = {
    "quant1d_mxfp4_rot_rne": ("qfp4_common.cuh", "quantize1d.cuh", "quantize1d.cu"),
    "quant1d_mxfp4_rot_sr": ("qfp4_common.cuh", "quantize1d.cuh", "quantize1d.cu"),
    "gemm_nvfp4_f32": ("qfp4_common.cuh", "gemm.cu"),
}


def _code_only(text):
    """Source text without comments and with whitespace runs collapsed, so
    that the hash follows code changes only."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return re.sub(r"\s+", " ", text).strip()


def csrc_hash(files=None):
    """Hash of the library sources' code (all files, or the named ones)."""
    h = hashlib.sha1()
    d = os.path.join(ROOT, "bit_fwht_hadamard_b200", "csrc")
    for n in sorted(files if files is not None else os.listdir(d)):
        with open(os.path.join(d, n), encoding="utf-8") as f:
            h.update(n.encode() + _code_only(f.read()).encode())
    return h.hexdigest()[:12]


def _ncu_figure(key, fname):
    """A per-launch figure from a committed ncu summary file (`key value
    source-hash ...` lines), if it was taken on the kernel's current sources
    (else None)."""
    p = os.path.join(ROOT, "profiles", fname)
    if not os.path.exists(p) or key not in KERNEL_SOURCES:
        return None
    cur = csrc_hash(KERNEL_SOURCES[key])
    with open(p) as f:
        for line in f:
            t = line.split()
            if len(t) >= 3 and not line.startswith("#") and t[0] == key and t[2] == cur:
                return float(t[1])
    return None


def ncu_traffic(key):
    """DRAM bytes (read + write) per launch of the kernel, from ncu."""
    return _ncu_figure(key, "ncu_traffic.txt")


def ncu_warp_insts(key):
    """Warp instructions executed per launch of the kernel, from ncu."""
    return _ncu_figure(key, "ncu_issue.txt")


def issue_roofline(key, ms, n_elem, sms, sm_mhz):
    """Instruction-issue roofline of a kernel: its warp instructions per
    launch (ncu) over its event-timed duration, against one warp
    instruction per cycle on each of the 4 schedulers of every SM at the
    SM clock seen during the run."""
    w = ncu_warp_insts(key)
    if w is None or not ms or not sm_mhz:
        return None
    peak = sms * 4 * sm_mhz * 1e6 / 1e9                   # G warp instructions / s
    achieved = w / (ms * 1e-3) / 1e9
    return {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "G warp-inst/s", "frac": achieved / peak,
            "warp_inst_per_launch": w, "thread_inst_per_element": 32.0 * w / n_elem,
            "issue_bound_ms": w / (peak * 1e9) * 1e3,
            "peak_source": f"{sms} SMs x 4 schedulers x 1 warp instruction/cycle x {sm_mhz:.0f} MHz (median SM clock)"}


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        rows = [r for r in csv.reader(io.StringIO(self.out or "")) if len(r) >= 9]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = [float(r[1]) for r in rows]
        mx = max(float(r[2]) for r in rows)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip() == "Active"})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": reasons, "samples": len(rows),
                "power_w_max": max(float(r[3]) for r in rows if r[3].strip() not in ("", "[N/A]"))}


# ------------------------------------------------------------------ reference arm (CPU oracle)
def run_reference(args, rank, world):
    """The oracle as it stands on the machine's host cores: each step is the
    default step (FWHT + MXFP4, RNE then SR seed 7) on a bounded sample of X,
    rows 0..1023, row-partitioned over every core."""
    if rank != 0:
        return
    import oracle
    import synth
    rows = 1024
    x = synth.cfg2_X()[:rows].copy()
    n = rows * K2
    cores = os.cpu_count() or 1
    for _ in range(args.warmup):
        _oracle_step_parallel(oracle, x, cores)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _oracle_step_parallel(oracle, x, cores)
    dt = (time.perf_counter() - t0) / max(args.steps, 1)
    gbs = 2 * n * BYTES_PER_ELEM_MXFP4 / dt / 1e9
    sample = (f"rows 0..{rows - 1} of X (4096 x 4096 bf16), RNE + SR per step, the C oracle row-partitioned over "
              f"{cores} threads")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": workload_config(),
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }))


def workload_config():
    return {"workload": "activation quantize + rotate: X bf16 4096x4096 N(0,1), 40 seeded channels x20; "
                        "FWHT-128 then MXFP4 g32 truncation-free E8M0; one RNE run + one Philox SR run (seed 7)",
            "global_batch": 1, "shape": [M2, K2], "parallelism": "replicas (weak scaling)",
            "l2": f"{N_BUFS} rotating input/output sets (> L2)"}


# ------------------------------------------------------------------ CPU baseline (oracle on the host)
def _oracle_step_parallel(oracle, x, threads):
    """The default step (FWHT + MXFP4, RNE then SR seed 7) by the oracle on
    row slices in `threads` threads (its ctypes calls release the GIL); each
    slice passes its first row so the random words stay keyed on the whole
    tensor's element index, which reassembles the single-threaded result."""
    from concurrent.futures import ThreadPoolExecutor
    M = x.shape[0]
    step = -(-M // (4 * threads))
    slices = [(a, min(M, a + step)) for a in range(0, M, step)]
    out = []
    with ThreadPoolExecutor(threads) as ex:
        for rounding, seed in ((oracle.RNE, 0), (oracle.SR, 7)):
            parts = list(ex.map(lambda s: oracle.quantize_ex(x[s[0]:s[1]], oracle.MXFP4, rounding, rotate=True,
                                                             seed=seed, row0=s[0]), slices))
            out.append({k: np.concatenate([p[k] for p in parts]) for k in ("codes", "scales")})
    return out


def cpu_baseline():
    """The oracle on the host cores: one full default step single-threaded,
    the same step row-partitioned over every core (checked identical), the
    single-threaded oracle on the full config-3 and config-4 quantize inputs,
    and the binary64 oracle GEMM on a 128 x 128 x 4096 sub-problem,
    extrapolated by flops to the 8192 x 11008 x 4096 GEMM."""
    import oracle
    import synth
    x = synth.cfg2_X()
    nproc = os.cpu_count() or 1
    step_bytes = 2 * x.size * BYTES_PER_ELEM_MXFP4
    t0 = time.perf_counter()
    single = [oracle.quantize(x, oracle.MXFP4, oracle.RNE, rotate=True),
              oracle.quantize(x, oracle.MXFP4, oracle.SR, rotate=True, seed=7)]
    dt1 = time.perf_counter() - t0
    t0 = time.perf_counter()
    par = _oracle_step_parallel(oracle, x, nproc)
    dtn = time.perf_counter() - t0
    identical = all(np.array_equal(a[k], b[k]) for a, b in zip(single, par) for k in ("codes", "scales"))
    # oracle GEMM: binary64 sum over dequantized NVFP4 operands, every output of a small sub-problem
    m = n = 128
    K = GEMM_SHAPE[2]
    A = oracle.quantize(synth.cfg3_X(m, K), oracle.NVFP4, four6=True)
    B = oracle.quantize(synth.cfg3_W(n, K), oracle.NVFP4, four6=True)
    r, c = np.meshgrid(np.arange(m), np.arange(n), indexing="ij")
    t0 = time.perf_counter()
    oracle.gemm_sampled(A, B, m, n, K, oracle.NVFP4, r.ravel(), c.ravel())
    dtg = time.perf_counter() - t0
    gflops = 2.0 * m * n * K / dtg / 1e9
    Mg, Ng, Kg = GEMM_SHAPE
    # single-threaded oracle on the full tensors of the other quantize configs
    configs = {}
    for name, fn, bpe in (
            ("cfg3 X 8192x4096 NVFP4 four-over-six RNE",
             lambda: oracle.quantize(synth.cfg3_X(), oracle.NVFP4, four6=True), 2.5625),
            ("cfg3 W 11008x4096 NVFP4 four-over-six RNE",
             lambda: oracle.quantize(synth.cfg3_W(), oracle.NVFP4, four6=True), 2.5625),
            ("cfg4 G 8192x4096 2D 16x16 NVFP4 SR (seed 1004), G and G^T",
             lambda: oracle.quantize(synth.cfg4_G(), oracle.NVFP4, oracle.SR, block2d=True, seed=1004,
                                     transposed=True), 3.125)):
        elems = {"cfg3 X": 8192 * 4096, "cfg3 W": 11008 * 4096, "cfg4 G": 8192 * 4096}[name[:6]]
        t0 = time.perf_counter()
        fn()
        dt = time.perf_counter() - t0
        configs[name] = {"seconds": dt, "elements_per_s": elems / dt, "GB/s": elems * bpe / dt / 1e9, "cores": 1}
    return {"value": step_bytes / dtn / 1e9, "unit": "GB/s", "cores": nproc, "kind": "oracle",
            "sample": f"one full step (X 4096x4096, FWHT-128 + MXFP4, RNE + SR) row-partitioned over {nproc} "
                      f"threads, output identical to the single-threaded run: {identical}",
            "seconds": dtn, "identical_to_single_thread": identical, "nproc": nproc,
            "single_thread": {"value": step_bytes / dt1 / 1e9, "unit": "GB/s", "cores": 1, "seconds": dt1},
            "single_thread_configs": configs,
            "gemm": {"value": gflops, "unit": "GFLOP/s", "cores": 1, "kind": "oracle",
                     "sample": f"binary64 oracle GEMM, every output of {m}x{n}x{K} (NVFP4 four-over-six operands)",
                     "seconds": dtg, "extrapolated_ms_for": f"{Mg}x{Ng}x{Kg}",
                     "extrapolated_ms": 2.0 * Mg * Ng * Kg / (gflops * 1e9) * 1e3, "label": "extrapolated"}}


def max_over_ranks(x, dist, device):
    """The largest x over all ranks, returned on every rank (x itself without a
    process group): timings are reported for the slowest rank."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ GPU arm
def run_gpu(args, rank, world):
    import torch

    import bit_fwht_hadamard_b200 as q
    import synth
    from bit_fwht_hadamard_b200 import build as _build

    local = int(os.environ.get("LOCAL_RANK", "0"))
    if int(os.environ.get("LOCAL_RANK", "0")) == 0:
        _build.build()                                   # no-op when libqfp4.so is newer than its sources
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if dist is not None:
            dist.barrier()

    hbm_peak, bf16_peak, bf16_sust, peak_src = measured_peaks()
    x_host = synth.cfg2_X()
    x0 = torch.from_numpy(x_host.view(np.int16)).view(torch.bfloat16)
    xs = [x0.to(dev)]
    for i in range(1, N_BUFS):
        xs.append(xs[0].clone())                          # distinct buffers (same values)
    outs = [[q.quantize(xs[0], q.MXFP4, q.RNE, rotate=True), q.quantize(xs[0], q.MXFP4, q.SR, rotate=True, seed=7)]
            for _ in range(N_BUFS)]
    stream = torch.cuda.current_stream()
    sh = stream.cuda_stream
    L = q.lib()
    # pre-marshalled C-ABI arguments: the timed loop is two ctypes calls per step
    args_rne = [(xs[b].data_ptr(), q.BF16, M2, K2, q.MXFP4, q.RNE, 1, 0, 0, 0, outs[b][0]["codes"].data_ptr(),
                 outs[b][0]["scales"].data_ptr(), None, None, None, None, 0, sh) for b in range(N_BUFS)]
    args_sr = [(xs[b].data_ptr(), q.BF16, M2, K2, q.MXFP4, q.SR, 1, 0, 0, 7, outs[b][1]["codes"].data_ptr(),
                outs[b][1]["scales"].data_ptr(), None, None, None, None, 0, sh) for b in range(N_BUFS)]
    status = []

    def step(i, ev=None):
        b = i % N_BUFS
        if ev is not None:
            ev[0].record(stream)
        status.append(L.qfp4_quantize(*args_rne[b]))
        if ev is not None:
            ev[1].record(stream)
        status.append(L.qfp4_quantize(*args_sr[b]))
        if ev is not None:
            ev[2].record(stream)

    for i in range(max(args.warmup, 3)):
        step(i)
    torch.cuda.synchronize()

    # ---- device-resident timed region (per-launch events inside it)
    # per-launch events bracket every EV_EVERY-th step only: an event between two
    # launches makes the second wait for the first, while without one the next
    # kernel's prologue overlaps the previous kernel's last CTAs
    sampled = [i for i in range(args.steps) if i % EV_EVERY == 0]
    evs = {i: [torch.cuda.Event(enable_timing=True) for _ in range(3)] for i in sampled}
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        soak_until = time.perf_counter() + 1.0           # load the GPU before the region so clocks are seen
        i = 0
        while time.perf_counter() < soak_until:
            step(i)
            i += 1
            if i % 64 == 0:
                torch.cuda.synchronize()
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        n_launch0 = q.qfp4_launch_count()
        # a spin kernel ahead of the start event lets the host enqueue the whole
        # region before the device reaches it, so host overhead leaves no gaps
        torch.cuda._sleep(int(2e9 * min(0.5, 40e-6 * args.steps + 2e-3)))
        start.record(stream)
        for i in range(args.steps):
            step(i, evs.get(i))
        stop.record(stream)
        torch.cuda.synchronize()
        n_launch = q.qfp4_launch_count() - n_launch0
        barrier()
    if any(st != q.OK for st in status):
        raise RuntimeError(f"qfp4_quantize failed: {set(status)}")
    elapsed_ms = max_over_ranks(start.elapsed_time(stop), dist, dev)
    ms_per_step = elapsed_ms / args.steps
    n = M2 * K2
    step_bytes = 2 * n * BYTES_PER_ELEM_MXFP4
    value = world * step_bytes / (ms_per_step * 1e-3) / 1e9

    rne_ms = statistics.mean(evs[i][0].elapsed_time(evs[i][1]) for i in sampled)
    sr_ms = statistics.mean(evs[i][1].elapsed_time(evs[i][2]) for i in sampled)
    dom_name, dom_ms = ("quant1d_mxfp4_rot_sr", sr_ms) if sr_ms >= rne_ms else ("quant1d_mxfp4_rot_rne", rne_ms)
    launch_bytes = n * BYTES_PER_ELEM_MXFP4
    achieved = launch_bytes / (dom_ms * 1e-3) / 1e9
    traffic = ncu_traffic(dom_name)
    roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s", "frac": achieved / hbm_peak,
                "traffic": traffic, "kernel": dom_name, "peak_source": f"{peak_src} hbm_gbs",
                "algorithmic_bytes_per_launch": launch_bytes,
                "launches": {"quant1d_mxfp4_rot_rne_ms": rne_ms, "quant1d_mxfp4_rot_sr_ms": sr_ms,
                             "rne_gbs": launch_bytes / (rne_ms * 1e-3) / 1e9,
                             "sr_gbs": launch_bytes / (sr_ms * 1e-3) / 1e9}}

    # ---- end to end through host buffers (pinned), same metric.  Every step
    # copies its input in from pinned host memory, runs both quantizes and
    # copies its codes and scales back; steps are pipelined over two buffer
    # slots (upload, compute and download on three streams), so step i+1's
    # upload overlaps step i's compute and download (PCIe is full duplex).
    x_pin = x0.pin_memory()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    xd = [torch.empty_like(xs[0]) for _ in range(2)]
    od = [[q.quantize(xs[0], q.MXFP4, q.RNE, rotate=True), q.quantize(xs[0], q.MXFP4, q.SR, rotate=True, seed=7)]
          for _ in range(2)]
    h_out = [[{k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for k, v in o.items()} for o in od[0]]
             for _ in range(2)]
    ev = lambda: torch.cuda.Event()                         # noqa: E731
    in_done, comp_done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    e_start, e_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_steps = max(3, min(args.steps, 50))
    torch.cuda.synchronize()
    barrier()
    e_start.record(stream)
    s_in.wait_event(e_start)
    s_out.wait_event(e_start)
    for i in range(e2e_steps):
        b = i % 2
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(comp_done[b])               # slot's device input no longer read
            xd[b].copy_(x_pin, non_blocking=True)
            in_done[b].record(s_in)
        stream.wait_event(in_done[b])
        if i >= 2:
            stream.wait_event(out_done[b])                  # slot's device outputs already copied out
        q.quantize(xd[b], q.MXFP4, q.RNE, rotate=True, out=od[b][0])
        q.quantize(xd[b], q.MXFP4, q.SR, rotate=True, seed=7, out=od[b][1])
        comp_done[b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[b])
            for j in range(2):
                for k in ("codes", "scales"):
                    h_out[b][j][k].copy_(od[b][j][k], non_blocking=True)
            out_done[b].record(s_out)
    stream.wait_event(out_done[(e2e_steps - 1) % 2])
    stream.wait_event(out_done[(e2e_steps - 2) % 2])
    e_stop.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e_start.elapsed_time(e_stop) / e2e_steps, dist, dev)
    h2d = x0.numel() * 2
    d2h = sum(v.numel() for o in od[0] for k, v in o.items() if k in ("codes", "scales"))
    e2e = {"value": world * step_bytes / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s", "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms}

    # ---- the same step with one input/output set, which stays in L2 (42.5 MB
    # of a 126 MB L2): the L2-warm figure beside the flushed one
    torch.cuda.synchronize()
    w0, w1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for i in range(3):
        step(0)
    torch.cuda.synchronize()
    barrier()
    torch.cuda._sleep(int(2e9 * min(0.5, 40e-6 * args.steps + 2e-3)))
    w0.record(stream)
    for i in range(args.steps):
        step(0)
    w1.record(stream)
    torch.cuda.synchronize()
    warm_ms = max_over_ranks(w0.elapsed_time(w1), dist, dev) / args.steps
    l2_warm = {"value": world * step_bytes / (warm_ms * 1e-3) / 1e9, "unit": "GB/s", "ms_per_step": warm_ms,
               "note": "one input/output set, L2-resident between steps"}

    # ---- GEMM of the NVFP4 forward linear (tensor-core roofline)
    gemm = None
    if not args.no_gemm:
        gemm = bench_gemm(q, synth, dev, stream, bf16_peak, peak_src, max(3, min(args.steps, 20)))
    cfg5 = None
    if not args.no_cfg5:
        cfg5 = bench_cfg5(q, synth, dev, stream, hbm_peak, bf16_peak, peak_src, max(3, min(args.steps, 10)))

    clocks = clk.summary()
    # the dominant kernel is issue-bound: its instruction roofline beside the HBM one
    roofline["issue"] = issue_roofline(dom_name, dom_ms, n, torch.cuda.get_device_properties(dev).multi_processor_count,
                                       clocks.get("sm_mhz") or clocks.get("sm_max_mhz"))
    result = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic", "config": workload_config(),
        "roofline": roofline, "e2e": e2e, "l2_warm": l2_warm, "gpu_launches": int(n_launch), "clocks": clocks,
        "frac_of_hbm_peak": value / world / hbm_peak,
    }
    if gemm is not None:
        result["gemm"] = gemm
    if cfg5 is not None:
        result["largest_config"] = cfg5
    if rank == 0 and world == 1 and not args.no_cpu:
        result["cpu_baseline"] = cpu_baseline()
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result))


def bench_gemm(q, synth, dev, stream, bf16_peak, peak_src, iters):
    import torch
    M, N, K = GEMM_SHAPE
    x = torch.from_numpy(synth.cfg3_X().view(np.int16)).view(torch.bfloat16).to(dev)
    w = torch.from_numpy(synth.cfg3_W().view(np.int16)).view(torch.bfloat16).to(dev)
    X = q.quantize(x, q.NVFP4, four6=True)
    W = q.quantize(w, q.NVFP4, four6=True)
    out = torch.empty((M, N), dtype=torch.float32, device=dev)
    ws = torch.empty(q.qfp4_gemm_workspace_bytes(M, N, K, q.NVFP4), dtype=torch.uint8, device=dev)
    for _ in range(3):
        q.gemm(X, W, M, N, K, q.NVFP4, out=out, workspace=ws)
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(iters)]
    for a, b in evs:
        a.record(stream)
        q.gemm(X, W, M, N, K, q.NVFP4, out=out, workspace=ws)
        b.record(stream)
    torch.cuda.synchronize()
    ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
    tflops = 2.0 * M * N * K / (ms * 1e-3) / 1e12
    peak = bf16_peak * FP4_PER_BF16
    return {"workload": "NVFP4 forward linear GEMM Y = X W^T, 8192 x 11008 x 4096, four-over-six operands, fp32 out",
            "value": tflops, "unit": "TFLOP/s", "ms_per_call": ms,
            "roofline": {"bound": "tensor", "achieved": tflops, "peak": peak, "unit": "TFLOP/s",
                         "frac": tflops / peak, "traffic": ncu_traffic("gemm_nvfp4_f32"),
                         "kernel": "gemm_nvfp4_f32 (scale-chunk prepass + 2-CTA tcgen05 main loop)",
                         "peak_source": f"{peak_src} bf16_tflops x {FP4_PER_BF16} (nominal FP4:BF16 dense ratio)"}}


def bench_cfg5(q, synth, dev, stream, hbm_peak, bf16_peak, peak_src, iters):
    """The largest configuration's two headline calls, each timed with CUDA
    events around every call on the launching stream: the standalone quantize
    of 2^30 bf16 elements (262144 x 4096; inputs far larger than L2) -- FWHT-128
    + MXFP4 RNE, and NVFP4 RNE under a caller-supplied tensor amax (one read) --
    and the fused rotate + quantize + GEMM at 16384 x 14336 x 4096."""
    import torch
    out = {}
    bf = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)   # noqa: E731
    base = bf(synth.cfg5_A(16384, 4096))
    x = base.repeat(16, 1)                                  # 2^30 elements, 2 GiB
    M, K = x.shape
    n = M * K

    def timed(call):
        for _ in range(3):
            call()
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(iters)]
        for a, b in evs:
            a.record(stream)
            call()
            b.record(stream)
        torch.cuda.synchronize()
        return statistics.mean(a.elapsed_time(b) for a, b in evs)

    o = q.quantize(x, q.MXFP4, q.RNE, rotate=True)
    ms = timed(lambda: q.quantize(x, q.MXFP4, q.RNE, rotate=True, out=o))
    nbytes = n * BYTES_PER_ELEM_MXFP4
    out["quantize_2^30_fwht_mxfp4_rne"] = {
        "workload": f"2^30 bf16 elements ({M}x{K}, N(0,1), 0.5% channels x30): FWHT-128 + MXFP4 RNE",
        "ms_per_call": ms, "roofline": {"bound": "hbm", "achieved": nbytes / (ms * 1e-3) / 1e9, "peak": hbm_peak,
                                        "unit": "GB/s", "frac": nbytes / (ms * 1e-3) / 1e9 / hbm_peak,
                                        "algorithmic_bytes_per_launch": nbytes, "traffic": None,
                                        "peak_source": f"{peak_src} hbm_gbs"}}
    amax = torch.tensor([float(x.abs().max())], dtype=torch.float32, device=dev)
    o = q.quantize(x, q.NVFP4, q.RNE, amax_in=amax)
    ms = timed(lambda: q.quantize(x, q.NVFP4, q.RNE, amax_in=amax, out=o))
    nbytes = n * (2 + 0.5 + 1 / 16)
    out["quantize_2^30_nvfp4_rne_given_amax"] = {
        "workload": f"2^30 bf16 elements ({M}x{K}): NVFP4 RNE with a caller-supplied tensor amax (one read of X)",
        "ms_per_call": ms, "roofline": {"bound": "hbm", "achieved": nbytes / (ms * 1e-3) / 1e9, "peak": hbm_peak,
                                        "unit": "GB/s", "frac": nbytes / (ms * 1e-3) / 1e9 / hbm_peak,
                                        "algorithmic_bytes_per_launch": nbytes, "traffic": None,
                                        "peak_source": f"{peak_src} hbm_gbs"}}
    del x, o
    M, N, K = 16384, 14336, 4096
    a5 = base
    B5 = q.quantize(bf(synth.cfg5_B(N, K)), q.NVFP4, q.RNE, rotate=True)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(q.qfp4_gemm_fused_rq_workspace_bytes(M, N, K, q.NVFP4), dtype=torch.uint8, device=dev)
    peak = bf16_peak * FP4_PER_BF16
    a_amax = torch.empty(1, dtype=torch.float32, device=dev)
    q.gemm_fused_rq(a5, B5, N, fmt=q.NVFP4, rotate=True, out=y, workspace=ws, A_amax_out=a_amax)
    for key, given, what in (("fused_rotate_quantize_gemm_16384x14336x4096", None, "A's own tensor amax (two reads of A)"),
                             ("fused_rotate_quantize_gemm_16384x14336x4096_given_amax", a_amax,
                              "a supplied tensor amax of A (one read of A)")):
        ms = timed(lambda: q.gemm_fused_rq(a5, B5, N, fmt=q.NVFP4, rotate=True, out=y, workspace=ws, A_amax_in=given))
        tf = 2.0 * M * N * K / (ms * 1e-3) / 1e12
        out[key] = {
            "workload": "A bf16 16384x4096 (0.5% channels x30) rotated + NVFP4-quantized inside the call under "
                        f"{what}, B 14336x4096 pre-rotated NVFP4, bf16 out",
            "ms_per_call": ms, "roofline": {"bound": "tensor", "achieved": tf, "peak": peak, "unit": "TFLOP/s",
                                            "frac": tf / peak, "flops_per_launch": 2.0 * M * N * K, "traffic": None,
                                            "peak_source": f"{peak_src} bf16_tflops x {FP4_PER_BF16}"}}
    return out


def run_profile_case(case):
    """Two warm-up and two measured calls of one kernel family, nothing timed:
    the small cases that ncu captures (inputs of the benchmark's own sizes)."""
    import torch

    import bit_fwht_hadamard_b200 as q
    import synth
    from bit_fwht_hadamard_b200 import build as _build
    _build.build()
    dev = torch.device("cuda:0")
    if case == "quant":
        x = torch.from_numpy(synth.cfg2_X().view(np.int16)).view(torch.bfloat16).to(dev)
        for _ in range(2):
            q.quantize(x, q.MXFP4, q.RNE, rotate=True)
            q.quantize(x, q.MXFP4, q.SR, rotate=True, seed=7)
    elif case == "backward":
        # gradient G 8192 x 4096: 2D NVFP4 with G^T, MXFP8 rows + columns,
        # 1D MXFP4 rows + independent columns (one launch of each tile kernel
        # per iteration, in that order)
        g = torch.from_numpy(synth.cfg4_G().view(np.int16)).view(torch.bfloat16).to(dev)
        for _ in range(2):
            q.quantize(g, q.NVFP4, q.RNE, block2d=True, transposed=True)
            q.quantize_mxfp8(g, q.RNE, transposed=True)
            q.quantize(g, q.MXFP4, q.RNE, transposed=True)
    elif case == "backward-sr":
        # gradient G 8192 x 4096 with stochastic rounding: 2D NVFP4 with G^T,
        # 1D NVFP4 rows + independent columns, MXFP8 rows + columns
        g = torch.from_numpy(synth.cfg4_G().view(np.int16)).view(torch.bfloat16).to(dev)
        for _ in range(2):
            q.quantize(g, q.NVFP4, q.SR, block2d=True, transposed=True, seed=11)
            q.quantize(g, q.NVFP4, q.SR, transposed=True, seed=11)
            q.quantize_mxfp8(g, q.SR, seed=11, transposed=True)
    elif case == "dequant":
        x = torch.from_numpy(synth.cfg3_X().view(np.int16)).view(torch.bfloat16).to(dev)
        X = q.quantize(x, q.NVFP4, q.RNE)
        for _ in range(2):
            q.dequantize(X, 8192, 4096, q.NVFP4, out_dtype=torch.bfloat16)
            q.dequantize(X, 8192, 4096, q.NVFP4, out_dtype=torch.float32)
    elif case == "quant-nvfp4":
        x = torch.from_numpy(synth.cfg3_X().view(np.int16)).view(torch.bfloat16).to(dev)
        for _ in range(2):
            q.quantize(x, q.NVFP4, q.RNE, four6=True)
    else:
        M, N, K = GEMM_SHAPE
        X = q.quantize(torch.from_numpy(synth.cfg3_X().view(np.int16)).view(torch.bfloat16).to(dev), q.NVFP4,
                       four6=True)
        W = q.quantize(torch.from_numpy(synth.cfg3_W().view(np.int16)).view(torch.bfloat16).to(dev), q.NVFP4,
                       four6=True)
        out = torch.empty((M, N), dtype=torch.float32, device=dev)
        for _ in range(2):
            q.gemm(X, W, M, N, K, q.NVFP4, out=out)
    torch.cuda.synchronize()
    print(f"profile case {case}: ok")


# ------------------------------------------------------------------ every entry point on its own workload
def time_calls(torch, stream, call, iters=20, warm=3):
    """Mean device time (ms) of call(i): CUDA events on the launching stream
    around each call, after a device-side head start so that host overhead
    leaves no gaps inside a bracket."""
    for i in range(warm):
        call(i)
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(iters)]
    torch.cuda._sleep(int(2e9 * 5e-3))
    for i, (a, b) in enumerate(evs):
        a.record(stream)
        call(warm + i)
        b.record(stream)
    torch.cuda.synchronize()
    return statistics.mean(a.elapsed_time(b) for a, b in evs)


def run_rows(only=""):
    """One JSON line per entry point of the path, each on the full-size
    synthetic workload it serves: quantize variants in GB/s of algorithmic
    bytes against the measured HBM peak, GEMMs in TFLOP/s against the dense
    FP4 peak.  Quantize inputs rotate over enough copies that consecutive
    calls never find their input in L2."""
    import torch

    import bit_fwht_hadamard_b200 as q
    import synth
    from bit_fwht_hadamard_b200 import build as _build
    _build.build()
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    sh = stream.cuda_stream
    hbm_peak, bf16_peak, _, peak_src = measured_peaks()
    fp4_peak = bf16_peak * FP4_PER_BF16
    L = q.lib()
    bad = []
    bf16 = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)   # noqa: E731

    def ok(st):
        if st != q.OK:
            bad.append(st)

    def emit(row, workload, ms, nbytes=None, flops=None, peak_ratio=FP4_PER_BF16, **extra):
        d = {"row": row, "workload": workload, "ms_per_call": ms}
        if nbytes is not None:
            a = nbytes / (ms * 1e-3) / 1e9
            d.update(bound="hbm", algorithmic_bytes=nbytes, achieved=a, unit="GB/s", peak=hbm_peak,
                     frac=a / hbm_peak, peak_source=f"{peak_src} hbm_gbs")
        else:
            a = flops / (ms * 1e-3) / 1e12
            pk = bf16_peak * peak_ratio
            d.update(bound="tensor", flops=flops, achieved=a, unit="TFLOP/s", peak=pk, frac=a / pk,
                     peak_source=f"{peak_src} bf16_tflops x {peak_ratio} (nominal dense ratio to bf16)")
        d.update(extra)
        print(json.dumps(d), flush=True)

    def n_sets(nbytes):
        return max(1, -(-(512 << 20) // nbytes))            # > 4x L2 between two calls on the same set

    def fp4_row(row, workload, x, fmt, rounding, bpe, rotate=False, block2d=False, four6=False, transposed=False,
                seed=0, rule=q.SCALE_DEFAULT, amax_in=False):
        M, K = x.shape
        ns = n_sets(x.numel() * 2)
        xs = [x] + [x.clone() for _ in range(ns - 1)]
        outs = [q.quantize(x, fmt, rounding, rotate=rotate, block2d=block2d, four6=four6, seed=seed,
                           transposed=transposed, rule=rule) for _ in range(ns)]
        wsb = q.qfp4_quantize_workspace_bytes(M, K, fmt, rotate, block2d)
        ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device=dev)
        amax = None
        if amax_in:                                     # the tensor's own amax, as a previous step would supply it
            amax = torch.empty(1, dtype=torch.float32, device=dev)
            q.quantize(x, fmt, rounding, rotate=rotate, amax_out=amax)
        av = [(xs[b].data_ptr(), q.BF16, M, K, fmt, rounding, int(rotate), int(block2d), int(four6), rule, seed,
               q._ptr(amax), None, o["codes"].data_ptr(), o["scales"].data_ptr(), q._ptr(o.get("codesT")),
               q._ptr(o.get("scalesT")), q._ptr(o.get("tscale")), ws.data_ptr(), wsb, sh) for b, o in enumerate(outs)]
        ms = time_calls(torch, stream, lambda i: ok(L.qfp4_quantize_ex(*av[i % ns])))
        emit(row, workload, ms, nbytes=bpe * M * K, bytes_per_element=bpe, input_sets=ns)

    def mxfp8_row(row, workload, x, rounding, transposed, seed=0):
        M, K = x.shape
        bpe = 2 + (1 + 1 / 32) * (2 if transposed else 1)
        ns = n_sets(x.numel() * 2)
        xs = [x] + [x.clone() for _ in range(ns - 1)]
        outs = [q.quantize_mxfp8(x, rounding, seed=seed, transposed=transposed) for _ in range(ns)]
        av = [(xs[b].data_ptr(), q.BF16, M, K, rounding, seed, o["codes"].data_ptr(), o["scales"].data_ptr(),
               q._ptr(o.get("codesT")), q._ptr(o.get("scalesT")), sh) for b, o in enumerate(outs)]
        ms = time_calls(torch, stream, lambda i: ok(L.qfp4_quantize_mxfp8(*av[i % ns])))
        emit(row, workload, ms, nbytes=bpe * M * K, bytes_per_element=bpe, input_sets=ns)

    def dequant_row(row, workload, x, fmt, out_dtype):
        M, K = x.shape
        g = 32 if fmt == q.MXFP4 else 16
        bpe = 0.5 + 1 / g + (4 if out_dtype == torch.float32 else 2)
        ns = n_sets(M * K // 2)
        src = [q.quantize(x, fmt) for _ in range(ns)]
        outs = [torch.empty((M, K), dtype=out_dtype, device=dev) for _ in range(ns)]
        odt = q.F32 if out_dtype == torch.float32 else q.BF16
        av = [(s["codes"].data_ptr(), s["scales"].data_ptr(), q._ptr(s.get("tscale")), M, K, fmt, odt,
               outs[b].data_ptr(), sh) for b, s in enumerate(src)]
        ms = time_calls(torch, stream, lambda i: ok(L.qfp4_dequantize(*av[i % ns])))
        emit(row, workload, ms, nbytes=bpe * M * K, bytes_per_element=bpe, input_sets=ns)

    def gemm_row(row, workload, A, B, M, N, K, fmt, out_dtype, peak_ratio=FP4_PER_BF16):
        out = torch.empty((M, N), dtype=out_dtype, device=dev)
        wsb = q.qfp4_gemm_workspace_bytes(M, N, K, fmt)
        ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device=dev)
        odt = q.F32 if out_dtype == torch.float32 else q.BF16
        av = (A["codes"].data_ptr(), A["scales"].data_ptr(), q._ptr(A.get("tscale")), B["codes"].data_ptr(),
              B["scales"].data_ptr(), q._ptr(B.get("tscale")), M, N, K, fmt, odt, out.data_ptr(), ws.data_ptr(), wsb,
              sh)
        ms = time_calls(torch, stream, lambda i: ok(L.qfp4_gemm_blockscaled(*av)))
        emit(row, workload, ms, flops=2.0 * M * N * K, peak_ratio=peak_ratio)

    def fused_row(row, workload, A_bf16, B, N, fmt, out_dtype):
        M, K = A_bf16.shape
        out = torch.empty((M, N), dtype=out_dtype, device=dev)
        wsb = q.qfp4_gemm_fused_rq_workspace_bytes(M, N, K, fmt)
        ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device=dev)
        odt = q.F32 if out_dtype == torch.float32 else q.BF16
        av = (A_bf16.data_ptr(), M, K, 1, 0, fmt, B["codes"].data_ptr(), B["scales"].data_ptr(),
              q._ptr(B.get("tscale")), N, ws.data_ptr(), wsb, odt, out.data_ptr(), sh)
        ms = time_calls(torch, stream, lambda i: ok(L.qfp4_gemm_fused_rq(*av)))
        emit(row, workload, ms, flops=2.0 * M * N * K)
        amax = torch.empty(1, dtype=torch.float32, device=dev)
        q.quantize(A_bf16, fmt, q.RNE, rotate=True, amax_out=amax)
        av2 = (A_bf16.data_ptr(), M, K, 1, 0, fmt, amax.data_ptr(), None, B["codes"].data_ptr(), B["scales"].data_ptr(),
               q._ptr(B.get("tscale")), N, ws.data_ptr(), wsb, odt, out.data_ptr(), sh)
        ms = time_calls(torch, stream, lambda i: ok(L.qfp4_gemm_fused_rq_ex(*av2)))
        emit(row, workload.replace("NVFP4 RNE of A", "NVFP4 RNE of A (supplied amax)"), ms, flops=2.0 * M * N * K)

    F32, BF = torch.float32, torch.bfloat16
    with ClockSampler(0) as clk:
        want = lambda *labels: any(only in lb for lb in labels)                   # noqa: E731
        # rotation + MXFP4 (the default bench step's two launches, one at a time)
        if want("rotate + mxfp4"):
            x2 = bf16(synth.cfg2_X())
            for r, name in ((q.RNE, "RNE"), (q.SR, "SR")):
                fp4_row("rotate + mxfp4", f"X bf16 4096x4096 (N(0,1), 40 channels x20): FWHT-128 + MXFP4 {name}", x2,
                        q.MXFP4, r, 2 + 0.5 + 1 / 32, rotate=True, seed=7)
            del x2
        # NVFP4 forward-linear operands: tensor amax, E4M3 scales, four-over-six
        nv = 2 + 0.5 + 1 / 16
        if want("nvfp4 four-over-six", "nvfp4", "dequantize", "scale rules"):
            x3, w3 = bf16(synth.cfg3_X()), bf16(synth.cfg3_W())
            if want("nvfp4 four-over-six"):
                fp4_row("nvfp4 four-over-six", "X bf16 8192x4096 Student-t(3)*0.5: NVFP4 four-over-six RNE", x3, q.NVFP4,
                        q.RNE, nv, four6=True)
                fp4_row("nvfp4 four-over-six", "W bf16 11008x4096 N(0,0.02^2): NVFP4 four-over-six RNE", w3, q.NVFP4,
                        q.RNE, nv, four6=True)
            if want("nvfp4"):
                fp4_row("nvfp4", "X bf16 8192x4096 Student-t(3)*0.5: NVFP4 RNE", x3, q.NVFP4, q.RNE, nv)
                fp4_row("nvfp4", "X bf16 8192x4096 Student-t(3)*0.5: NVFP4 Philox SR", x3, q.NVFP4, q.SR, nv, seed=7)
                fp4_row("nvfp4", "X bf16 8192x4096: NVFP4 RNE, supplied tensor amax (one read)", x3, q.NVFP4, q.RNE,
                        nv, amax_in=True)
                fp4_row("nvfp4", "X bf16 8192x4096: FWHT-128 + NVFP4 RNE", x3, q.NVFP4, q.RNE, nv, rotate=True)
                fp4_row("nvfp4", "X bf16 8192x4096: FWHT-128 + NVFP4 RNE, supplied tensor amax", x3, q.NVFP4, q.RNE,
                        nv, rotate=True, amax_in=True)
            if want("scale rules"):
                fp4_row("scale rules", "X bf16 8192x4096: NVFP4 RNE, E4M3 block scale rounded up", x3, q.NVFP4, q.RNE,
                        nv, rule=q.SCALE_E4M3_UP)
            if want("dequantize"):
                dequant_row("dequantize", "NVFP4 codes of X 8192x4096 -> bf16", x3, q.NVFP4, BF)
                dequant_row("dequantize", "NVFP4 codes of X 8192x4096 -> fp32", x3, q.NVFP4, F32)
            del x3, w3
        # Quartet-style backward: 2D blocks, MXFP8, column-wise 1D, backward GEMMs
        if want("2d blocks", "column-wise", "mxfp8", "gemm", "scale rules"):
            g4 = bf16(synth.cfg4_G())
            if want("scale rules"):
                fp4_row("scale rules", "G bf16 8192x4096: MXFP4 RNE, OCP floor E8M0 exponent", g4, q.MXFP4, q.RNE,
                        2 + 0.5 + 1 / 32, rule=q.SCALE_OCP_FLOOR)
                fp4_row("scale rules", "G bf16 8192x4096: MXFP4 four-over-six under the OCP floor rule", g4, q.MXFP4,
                        q.RNE, 2 + 0.5 + 1 / 32, four6=True, rule=q.SCALE_OCP_FLOOR)
                fp4_row("scale rules", "G bf16 8192x4096: 2D 32x32 MXFP4 RNE, G and G^T", g4, q.MXFP4, q.RNE,
                        2 + 2 * (0.5 + 1 / 32), block2d=True, transposed=True)
            if want("2d blocks"):
                fp4_row("2d blocks", "G bf16 8192x4096 (N(0,1e-6), 0.1% x100): 2D 16x16 NVFP4 Philox SR, G and G^T", g4,
                        q.NVFP4, q.SR, 2 + 2 * (0.5 + 1 / 16), block2d=True, transposed=True, seed=11)
                fp4_row("2d blocks", "G bf16 8192x4096: 2D 16x16 NVFP4 RNE, G and G^T", g4, q.NVFP4, q.RNE,
                        2 + 2 * (0.5 + 1 / 16), block2d=True, transposed=True)
            if want("column-wise"):
                fp4_row("column-wise", "G bf16 8192x4096: 1D MXFP4 RNE rows + independent column-wise groups", g4,
                        q.MXFP4, q.RNE, 2 + 2 * (0.5 + 1 / 32), transposed=True)
                fp4_row("column-wise", "G bf16 8192x4096: 1D NVFP4 Philox SR rows + independent column-wise groups", g4,
                        q.NVFP4, q.SR, 2 + 2 * (0.5 + 1 / 16), transposed=True, seed=11)
            if want("mxfp8"):
                for r, name in ((q.RNE, "RNE"), (q.SR, "SR")):
                    mxfp8_row("mxfp8", f"G bf16 8192x4096: MXFP8 E4M3 g32 {name}", g4, r, False, seed=11)
                mxfp8_row("mxfp8", "G bf16 8192x4096: MXFP8 E4M3 g32 RNE, rows + column-wise", g4, q.RNE, True)
                mxfp8_row("mxfp8", "G bf16 8192x4096: MXFP8 E4M3 g32 SR, rows + column-wise", g4, q.SR, True, seed=11)
            if want("gemm"):
                # backward GEMMs on 2D-quantized operands: dX = G W, dW = G^T X
                x4, w4 = bf16(synth.cfg4_X()), bf16(synth.cfg4_W())
                G2 = q.quantize(g4, q.NVFP4, q.SR, block2d=True, transposed=True, seed=11)
                W2 = q.quantize(w4, q.NVFP4, q.RNE, block2d=True, transposed=True)
                X2 = q.quantize(x4, q.NVFP4, q.RNE, block2d=True, transposed=True)
                T = lambda o: {"codes": o["codesT"], "scales": o["scalesT"], **({"tscale": o["tscale"]} if "tscale" in o else {})}   # noqa: E731,E501
                gemm_row("gemm", "dX = G W: NVFP4 8192x4096x4096, fp32 out", G2, T(W2), 8192, 4096, 4096, q.NVFP4, F32)
                gemm_row("gemm", "dW = G^T X: NVFP4 4096x4096x8192, fp32 out", T(G2), T(X2), 4096, 4096, 8192, q.NVFP4,
                         F32)
                # the FP8 backward: MXFP8 block-scaled GEMMs on kind::mxf8f6f4
                G8 = q.quantize_mxfp8(g4, q.SR, seed=11, transposed=True)
                W8 = q.quantize_mxfp8(w4, q.RNE, transposed=True)
                X8 = q.quantize_mxfp8(x4, q.RNE, transposed=True)
                gemm_row("gemm", "dX = G W: MXFP8 8192x4096x4096, fp32 out", G8, T(W8), 8192, 4096, 4096, q.MXFP8,
                         F32, peak_ratio=2.0)
                gemm_row("gemm", "dW = G^T X: MXFP8 4096x4096x8192, fp32 out", T(G8), T(X8), 4096, 4096, 8192, q.MXFP8,
                         F32, peak_ratio=2.0)
                del G2, W2, X2, G8, W8, X8, x4, w4
            del g4
        # 7B-class linear shapes: the GEMM alone and the fused rotate + quantize + GEMM
        if want("gemm", "fused rotate + quantize + gemm"):
            for (M, N, K) in ((16384, 4096, 4096), (16384, 14336, 4096), (16384, 4096, 14336)):
                a5 = bf16(synth.cfg5_A(M, K))
                B5 = q.quantize(bf16(synth.cfg5_B(N, K)), q.NVFP4, q.RNE, rotate=True)
                A5 = q.quantize(a5, q.NVFP4, q.RNE, rotate=True)
                if want("gemm"):
                    gemm_row("gemm", f"NVFP4 GEMM {M}x{N}x{K} (A pre-quantized), bf16 out", A5, B5, M, N, K, q.NVFP4,
                             BF)
                if want("fused rotate + quantize + gemm"):
                    fused_row("fused rotate + quantize + gemm",
                              f"fused FWHT-128 + NVFP4 RNE of A bf16 + GEMM {M}x{N}x{K}, bf16 out", a5, B5, N, q.NVFP4,
                              BF)
                del a5, B5, A5
        # the Quartet-style linear layer: forward on the forward-linear shapes, backward on the gradient shapes
        if want("linear"):
            x3, w3 = bf16(synth.cfg3_X()), bf16(synth.cfg3_W())
            M, K = x3.shape
            N = w3.shape[0]
            y = torch.empty((M, N), dtype=BF, device=dev)
            wsb = q.qfp4_linear_forward_workspace_bytes(M, N, K, q.NVFP4)
            ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
            av = (x3.data_ptr(), w3.data_ptr(), M, N, K, q.NVFP4, 0, q.BF16, y.data_ptr(), ws.data_ptr(), wsb, sh)
            ms = time_calls(torch, stream, lambda i: ok(L.qfp4_linear_forward(*av)))
            emit("linear", f"forward Y = Q(XH) Q(WH)^T: X {M}x{K}, W {N}x{K} bf16, NVFP4, bf16 out", ms,
                 flops=2.0 * M * N * K)
            del x3, w3, y, ws
            g4, x4, w4 = bf16(synth.cfg4_G()), bf16(synth.cfg4_X()), bf16(synth.cfg4_W())
            M, N = g4.shape
            K = x4.shape[1]
            dX = torch.empty((M, K), dtype=F32, device=dev)
            dW = torch.empty((N, K), dtype=F32, device=dev)
            for fmt, name, ratio in ((q.NVFP4, "2D NVFP4 (G stochastic)", FP4_PER_BF16),
                                     (q.MXFP8, "MXFP8 (G stochastic)", 2.0)):
                wsb = q.qfp4_linear_backward_workspace_bytes(M, N, K, fmt)
                ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
                av = (g4.data_ptr(), x4.data_ptr(), w4.data_ptr(), M, N, K, fmt, 11, q.F32, dX.data_ptr(),
                      dW.data_ptr(), ws.data_ptr(), wsb, sh)
                ms = time_calls(torch, stream, lambda i: ok(L.qfp4_linear_backward(*av)))
                emit("linear", f"backward dX = G W, dW = G^T X: G {M}x{N}, X {M}x{K}, W {N}x{K}, {name}, fp32 out",
                     ms, flops=2 * 2.0 * M * N * K, peak_ratio=ratio)
                del ws
            del g4, x4, w4, dX, dW
        if want("kl calibration"):
            xr = bf16(synth.relu_activation(8192, 4096))
            out = {"clip": torch.empty(1, dtype=F32, device=dev), "best": torch.empty(1, dtype=torch.int32, device=dev),
                   "kl": torch.empty(2048 - 8 + 1, dtype=torch.float64, device=dev),
                   "hist": torch.empty(2048, dtype=torch.int64, device=dev)}
            wsb = q.qfp4_kl_calibrate_workspace_bytes(2048, 8, 1)
            ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
            av = (xr.data_ptr(), q.BF16, xr.numel(), 2048, 8, 1, out["clip"].data_ptr(), out["best"].data_ptr(),
                  out["kl"].data_ptr(), out["hist"].data_ptr(), ws.data_ptr(), wsb, sh)
            ms = time_calls(torch, stream, lambda i: ok(L.qfp4_kl_calibrate(*av)))
            emit("kl calibration", "ReLU-like activation bf16 8192x4096: |x| histogram (2048 bins) + KL over every "
                 "candidate clip (E2M1 levels)", ms, nbytes=2 * 2.0 * xr.numel())
            del xr
        # standalone quantize bandwidth over 2^20 .. 2^30 bf16 elements (K = 4096):
        # rows of the 16384 x 4096 outlier-channel input, repeated past 2^26 elements
        if want("quantize sweep"):
            base = bf16(synth.cfg5_A(16384, 4096))
            for e in range(20, 31, 2):
                M = (1 << e) // 4096
                x = base[:M].clone() if M <= 16384 else base.repeat(M // 16384, 1)
                fp4_row("quantize sweep", f"2^{e} bf16 elements ({M}x4096): NVFP4 RNE", x, q.NVFP4, q.RNE, nv)
                fp4_row("quantize sweep", f"2^{e} bf16 elements ({M}x4096): NVFP4 RNE, supplied tensor amax", x,
                        q.NVFP4, q.RNE, nv, amax_in=True)
                fp4_row("quantize sweep", f"2^{e} bf16 elements ({M}x4096): FWHT-128 + MXFP4 RNE", x, q.MXFP4, q.RNE,
                        2 + 0.5 + 1 / 32, rotate=True)
                del x
    torch.cuda.synchronize()
    err = q.qfp4_last_device_error()
    print(json.dumps({"rows_done": True, "clocks": clk.summary(), "device_error": err, "bad_status": sorted(set(bad)),
                      "csrc": csrc_hash()}), flush=True)
    if bad or err:
        raise RuntimeError(f"status {sorted(set(bad))}, device error {err}")


def main():
    args = parse()
    if args.profile_case:
        run_profile_case(args.profile_case)
        return
    if args.rows is not None:
        run_rows(args.rows)
        return
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    run_gpu(args, rank, world)


if __name__ == "__main__":
    main()
