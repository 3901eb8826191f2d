#!/usr/bin/env python
"""FlashMask forward+backward benchmark on B200: effective TFLOP/s over unmasked pairs.

One step = one forward (``flashmask_fwd``) and one backward (``flashmask_bwd``)
over one batch of the workload, through the library's C ABI.  Effective FLOPs
count only unmasked (i, j) pairs: 4*d*pairs forward, 10*d*pairs backward
(pairs from the library's closed-form count).  The default (headline)
workload is the largest single-GPU one: the 131072-token causal-document mask
with 30% of its 128-key tiles dropped, 32 query / 8 KV heads, head_dim 128.
The 8K document and 32K share-question workloads are timed in the same run
and reported under "secondary".

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config NAME]

N > 1 runs as independent replicas (one process per GPU, no data-path
collective; the path has no exchange step): value = all ranks' FLOPs / max
over ranks of the device time.  Started without torchrun's environment,
``--gpus N`` re-launches itself under ``torch.distributed.run`` with N
processes.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import re
import platform
import socket
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from column_sparse_masked_b200 import workloads as wl  # noqa: E402

METRIC = "FlashMask fwd+bwd effective TFLOP/s (unmasked FLOPs only), % of B200 bf16 peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
CPU_SAMPLE_ROWS = 8192  # bounded oracle sample: first rows/keys of (batch 0, q-head 0)
DEFAULT_CONFIG = "docblocksparse128k"
SECONDARY = ("doc8k", "sharequestion32k", "prefixwindow64k")
SECONDARY_STEPS = 30


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default=DEFAULT_CONFIG, choices=wl.CONFIG_ORDER)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", action="store_true", help="time only the headline workload")
    ap.add_argument("--bwd-mode", choices=["fused", "split"], default="fused",
                    help="backward: one key-stationary pass (default) or the deterministic two-kernel split")
    return ap.parse_args(argv)


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def free_port() -> int:
    sk = socket.socket()
    sk.bind(("127.0.0.1", 0))
    port = sk.getsockname()[1]
    sk.close()
    return port


def relaunch_command(argv, gpus: int, port: int):
    """torch.distributed.run command that starts this script once per GPU (replicas)."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={gpus}",
            "--master-addr", "127.0.0.1", f"--master-port={port}", os.path.abspath(__file__), *argv]


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return platform.processor() or "unknown"


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f), "MEASURED_PEAKS.json"
    return FALLBACK_PEAKS, "fallback"


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def aggregate(local_ms: float, flops_per_step: float, steps: int, world: int, device) -> tuple:
    """Whole-job throughput of `world` replicas: all ranks' FLOPs / max-over-ranks device time.

    Returns (TFLOP/s, max ms).  Every rank calls it (it holds a collective).
    """
    total_ms = max_over_ranks(local_ms, world, device)
    return world * flops_per_step * steps / (total_ms / 1e3) / 1e12, total_ms


def barrier(world: int):
    if world > 1:
        torch.distributed.barrier()


class ClockSampler:
    """nvidia-smi clock/throttle samples every 50 ms while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-i", str(self.gpu), "-lms", "50"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        out = {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        if self.proc is None:
            return out
        time.sleep(0.06)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx.append(float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        if sm:
            out.update(sm_mhz=statistics.median(sm), sm_max_mhz=max(mx), reasons=sorted(reasons), samples=len(sm))
        return out


def effective_flops(pairs: int, d: int):
    return 4.0 * d * pairs, 10.0 * d * pairs


def kernel_source_hash(name: str) -> str:
    """sha256[:16] of a kernel source's code: the file with `//` comments, trailing blanks and
    empty lines removed, so that a comment edit keeps the recorded counters valid."""
    with open(os.path.join(ROOT, "column_sparse_masked_b200", "csrc", name), encoding="utf-8") as f:
        lines = [re.sub(r"//.*$", "", ln).rstrip() for ln in f]
    code = "\n".join(ln for ln in lines if ln)
    return hashlib.sha256(code.encode()).hexdigest()[:16]


def recorded_traffic(kernel_file: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it matches the current kernel source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    e = rec.get(kernel_file, {}).get(workload)
    if not e or e.get("source_sha256_16") != kernel_source_hash(kernel_file):
        return None
    return e.get("dram_bytes_per_launch")


# ----------------------------------------------------------------------------
# CPU oracle leg (bounded sample) -- the only place bench.py executes oracle/
# ----------------------------------------------------------------------------
def oracle_sample(w: wl.Workload, rows: int, inp=None, head: int = 0):
    """(b=0, q-head `head` with its KV head) restricted to its first `rows` queries and keys
    (mask localised onto [0, rows))."""
    import oracle

    full = wl.make_inputs(w, with_grad=True) if inp is None else inp
    n = min(rows, w.N)
    hk = head // (w.Hq // w.Hkv)
    hm = 0 if full["lts"].shape[1] == 1 else head
    q = full["q"][:1, :n, head:head + 1].contiguous()
    k = full["k"][:1, :n, hk:hk + 1].contiguous()
    v = full["v"][:1, :n, hk:hk + 1].contiguous()
    do = full["do"][:1, :n, head:head + 1].contiguous()
    vecs = [oracle.localize(full[m][:1, hm:hm + 1, :n].numpy(), 0, n) for m in ("lts", "lte", "uts", "ute")]
    pairs = oracle.count_unmasked(*vecs, n, n, 1)
    return q, k, v, do, vecs, pairs, n


def run_oracle_step(sample):
    import oracle

    q, k, v, do, vecs, pairs, n = sample
    t0 = time.perf_counter()
    oracle.attention_forward(q, k, v, *vecs)
    oracle.attention_backward(q, k, v, do, *vecs)
    return time.perf_counter() - t0


CPU_TARGET_SECONDS = 10.0  # the CPU leg runs whole heads until about this much oracle time


def cpu_baseline(w: wl.Workload, rows: int = CPU_SAMPLE_ROWS, inp=None):
    """The oracle as it stands on the host cores: fp64 fwd+bwd of (batch 0, q-head h) restricted to
    the first `rows` queries and keys, for h = 0, 1, ... until about CPU_TARGET_SECONDS of work."""
    import oracle

    full = wl.make_inputs(w, with_grad=True) if inp is None else inp
    dt, pairs, heads, n = 0.0, 0, 0, min(rows, w.N)
    while heads < w.Hq and dt < CPU_TARGET_SECONDS:
        sample = oracle_sample(w, rows, full, head=heads)
        dt += run_oracle_step(sample)
        pairs += sample[5]
        heads += 1
    ff, fb = effective_flops(pairs, w.d)
    return {"value": (ff + fb) / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
            "cpu_model": cpu_model(), "seconds": dt,
            "sample": f"{w.name}: batch 0, q-heads 0..{heads - 1} each with its KV head, first {n} queries x "
                      f"{n} keys (mask localised onto [0,{n})), fp64 fwd+bwd, {pairs} unmasked pairs"}


# ----------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------
MASK_NAMES = ("lts", "lte", "uts", "ute")
INPUT_NAMES = ("q", "k", "v", "do") + MASK_NAMES


def class_histogram(fm, masks, w) -> dict:
    """Skip / partial / full counts of the (batch, mask head, q-tile, k-tile) tiles."""
    cls = fm.classify(*masks, Nq=w.N)
    c = torch.bincount(cls.flatten().long(), minlength=3).tolist()
    return {"skip": c[0], "partial": c[1], "full": c[2], "tiles": sum(c),
            "unit": "128x128 (batch, mask head, q-tile, k-tile) tiles"}


def setup_problem(fm, w, dev) -> dict:
    """Pinned host inputs, their device copies, outputs and workspace of one workload."""
    inp = wl.make_inputs(w, with_grad=True)
    host = {n: inp[n].pin_memory() for n in INPUT_NAMES}
    d_in = {n: host[n].to(dev) for n in INPUT_NAMES}
    pb = {"w": w, "inp": inp, "host": host, "d_in": d_in,
          "o": torch.empty_like(d_in["q"]),
          "lse": torch.empty(w.B, w.Hq, w.N, dtype=torch.float32, device=dev),
          "dq": torch.empty_like(d_in["q"]), "dk": torch.empty_like(d_in["k"]), "dv": torch.empty_like(d_in["v"]),
          "ws": torch.empty(fm.workspace_size("bwd", w.B, w.Hq, w.Hkv, 1, w.N, w.N, w.d), dtype=torch.uint8,
                            device=dev)}
    pb["pairs"] = fm.count_unmasked(*[d_in[n] for n in MASK_NAMES], Nq=w.N, Hq=w.Hq)
    return pb


def run_step(fm, pb, src):
    """One step of the hot path: forward then backward, through the library's C ABI."""
    m = [src[n] for n in MASK_NAMES]
    fm.fwd(src["q"], src["k"], src["v"], *m, out=(pb["o"], pb["lse"]), workspace=pb["ws"])
    fm.bwd(src["q"], src["k"], src["v"], pb["o"], pb["lse"], src["do"], *m,
           out=(pb["dq"], pb["dk"], pb["dv"]), workspace=pb["ws"])


def time_device(fm, pb, steps, warmup, flush, world, clocks=None):
    """Device time of `steps` steps (CUDA events per step, L2 flushed before each step outside the
    events), with the library's per-kernel profiler on.  Returns (per-step ms, profiler, launches, clocks)."""
    for _ in range(warmup):
        flush.fill_(1)
        run_step(fm, pb, pb["d_in"])
    torch.cuda.synchronize()
    assert fm.get_status() == 0, "device status word set during warm-up"
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize()
    launches0 = fm.launch_count()
    fm.profiler_read()
    fm.profiler_enable(True)
    if clocks is not None:
        clocks.start()
    for i in range(steps):
        flush.fill_(i & 0xFF)
        evs[i][0].record()
        run_step(fm, pb, pb["d_in"])
        evs[i][1].record()
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop() if clocks is not None else None
    fm.profiler_enable(False)
    prof = fm.profiler_read()
    launches = fm.launch_count() - launches0
    assert fm.get_status() == 0, "device status word set during the timed steps"
    return [a.elapsed_time(b) for a, b in evs], prof, launches, clk


def unit_rates(prof, pairs, d, peak):
    """Effective TFLOP/s and fraction of peak of the forward unit and the backward pair."""
    out = {}
    for k, fl in (("fwd", 4.0 * d * pairs), ("bwd", 10.0 * d * pairs)):
        ms, nl = prof[f"{k}_ms"], prof[f"{k}_launches"]
        tf = fl / (ms / nl / 1e3) / 1e12 if nl else None
        out[k] = {"ms_per_launch": ms / nl if nl else None, "tflops": tf, "frac": tf / peak if tf else None}
    return out


def run_ours(args, rank, world, local_rank):
    import column_sparse_masked_b200 as fm

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    fm.set_bwd_mode(args.bwd_mode)
    peaks, peak_src = load_peaks()
    peak = float(peaks["bf16_tflops"])
    w = wl.CONFIGS[args.config]
    pb = setup_problem(fm, w, dev)
    pairs = pb["pairs"]
    f_fwd, f_bwd = effective_flops(pairs, w.d)
    hist = class_histogram(fm, [pb["d_in"][n] for n in MASK_NAMES], w)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(2 * l2, dtype=torch.uint8, device=dev)

    # ---- device-resident timing ----
    vis = [x for x in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if x.strip()]
    clocks = ClockSampler(vis[local_rank] if local_rank < len(vis) else str(local_rank))
    step_ms, prof, launches, clk = time_device(fm, pb, args.steps, args.warmup, flush, world, clocks)
    local_ms = sum(step_ms)
    value, total_ms = aggregate(local_ms, f_fwd + f_bwd, args.steps, world, dev)

    # ---- end to end: host buffers, copies inside the timed region ----
    # Every step copies its inputs from pinned host memory to the device, runs
    # the forward and backward through the library, and copies every output
    # back.  Measured two ways: serial (copy in, compute, copy out on one
    # stream) and pipelined the way a training loop prefetches: step i+1's
    # inputs go in on one copy stream and step i-1's outputs come out on
    # another while step i computes (device inputs and outputs
    # double-buffered).  `value` is the pipelined figure.
    host = pb["host"]
    out_names = ("o", "lse", "dq", "dk", "dv")
    d_out = [{n: pb[n] for n in out_names}, {n: torch.empty_like(pb[n]) for n in out_names}]
    h_out = [{n: torch.empty_like(t, device="cpu").pin_memory() for n, t in d_out[0].items()} for _ in range(2)]
    d_buf = [pb["d_in"], {n: torch.empty_like(pb["d_in"][n]) for n in INPUT_NAMES}]
    cmp_stream = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

    def compute(j):
        dst = dict(pb)
        dst.update(d_out[j])
        run_step(fm, dst, d_buf[j])

    def e2e_serial(steps):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for i in range(steps):
            flush.fill_(i & 0xFF)
            evs[i][0].record()
            for n in INPUT_NAMES:
                d_buf[1][n].copy_(host[n], non_blocking=True)
            compute(1)
            for n in out_names:
                h_out[1][n].copy_(d_out[1][n], non_blocking=True)
            evs[i][1].record()
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in evs)

    def e2e_pipelined(steps):
        ev = lambda: torch.cuda.Event(enable_timing=True)
        in_ready, in_free, out_ready, out_free = [ev(), ev()], [ev(), ev()], [ev(), ev()], [ev(), ev()]
        used_in, used_out = [False, False], [False, False]
        start, end = ev(), ev()
        start.record(cmp_stream)
        s_in.wait_event(start)
        s_out.wait_event(start)

        def copy_in(i):
            j = i % 2
            with torch.cuda.stream(s_in):
                if used_in[j]:
                    s_in.wait_event(in_free[j])  # step i-2 has finished reading this buffer
                for n in INPUT_NAMES:
                    d_buf[j][n].copy_(host[n], non_blocking=True)
                in_ready[j].record(s_in)

        copy_in(0)
        for i in range(steps):
            j = i % 2
            if i + 1 < steps:
                copy_in(i + 1)
            cmp_stream.wait_event(in_ready[j])
            if used_out[j]:
                cmp_stream.wait_event(out_free[j])  # step i-2's outputs are on the host
            flush.fill_(i & 0xFF)
            compute(j)
            in_free[j].record(cmp_stream)
            out_ready[j].record(cmp_stream)
            used_in[j] = used_out[j] = True
            with torch.cuda.stream(s_out):
                s_out.wait_event(out_ready[j])
                for n in out_names:
                    h_out[j][n].copy_(d_out[j][n], non_blocking=True)
                out_free[j].record(s_out)
        end.record(s_out)
        cmp_stream.wait_stream(s_out)
        cmp_stream.wait_stream(s_in)
        torch.cuda.synchronize()
        return start.elapsed_time(end)

    e2e_steps = min(args.steps, 20)
    e2e_serial(1)
    e2e_pipelined(2)
    barrier(world)
    torch.cuda.synchronize()
    serial_ms = e2e_serial(e2e_steps)
    barrier(world)
    torch.cuda.synchronize()
    pipe_ms = e2e_pipelined(e2e_steps)
    barrier(world)
    # the pipelined loop's two buffer sets computed the same step: O, LSE, dK, dV bit for bit (dQ
    # is summed in an order that varies), and the last copies out hold the device values
    e2e_check = all(torch.equal(d_out[0][n], d_out[1][n]) for n in ("o", "lse", "dk", "dv"))
    e2e_check = e2e_check and bool(torch.allclose(d_out[0]["dq"].float(), d_out[1]["dq"].float(), atol=2e-2, rtol=2 ** -6))
    jl = (e2e_steps - 1) % 2
    e2e_check = e2e_check and torch.equal(h_out[jl]["lse"], d_out[jl]["lse"].cpu())
    e2e_value, e2e_ms = aggregate(pipe_ms, f_fwd + f_bwd, e2e_steps, world, dev)
    e2e_serial_value, e2e_serial_ms = aggregate(serial_ms, f_fwd + f_bwd, e2e_steps, world, dev)
    h2d = sum(host[n].numel() * host[n].element_size() for n in INPUT_NAMES)
    d2h = sum(t.numel() * t.element_size() for t in h_out[0].values())
    del d_buf[1], d_out[1], h_out

    # ---- roofline of the dominant unit ----
    # Units: the forward kernel, and the backward's attention unit.  Fused
    # mode: the key-stationary kernel that computes all five matmuls of each
    # pair plus the dQ finalize (an HBM-bound conversion), timed together.
    # Split mode: the key-side and query-side kernels, which run concurrently
    # (key side on the caller's stream, query side on the library's second
    # stream), timed together from fork to join.
    # Algorithmic work = the matmuls the method needs over unmasked pairs:
    # forward 2 (QK^T, PV) = 4*d*pairs; backward 5 (S, dP, dV, dK, dQ) =
    # 10*d*pairs.  Executed work per kernel is reported beside it (split mode
    # adds the query side's recomputed S and dP: key side 8*d*pairs, query
    # side 6*d*pairs).
    d = w.d
    if args.bwd_mode == "fused":
        bwd_unit = (("bwd_fused_sm100.cu",), f"fm_bwd_fused_kernel<{d}> + fm_dq_finalize_kernel<{d}>",
                    10.0 * d * pairs)
        executed = {"fwd": (f"fm_fwd_kernel<{d}>", 4.0 * d * pairs),
                    "bwd_fused": (f"fm_bwd_fused_kernel<{d}>", 10.0 * d * pairs),
                    "dq_finalize": (f"fm_dq_finalize_kernel<{d}>", 0.0)}
    else:
        bwd_unit = (("bwd_dkdv_sm100.cu", "bwd_dq_sm100.cu"),
                    f"fm_bwd_dkdv_kernel<{d}> + fm_bwd_dq_kernel<{d}> (concurrent)", 10.0 * d * pairs)
        executed = {"fwd": (f"fm_fwd_kernel<{d}>", 4.0 * d * pairs),
                    "bwd_kv": (f"fm_bwd_dkdv_kernel<{d}>", 8.0 * d * pairs),
                    "bwd_q": (f"fm_bwd_dq_kernel<{d}>", 6.0 * d * pairs)}
    units = {"fwd": (("fwd_sm100.cu",), f"fm_fwd_kernel<{d}>", 4.0 * d * pairs), "bwd": bwd_unit}
    per_unit = {}
    for k, (srcs, kname, fl) in units.items():
        ms, nl = prof[f"{k}_ms"], prof[f"{k}_launches"]
        tr = [recorded_traffic(sf, w.name) for sf in srcs]
        per_unit[k] = {"kernel": kname, "ms_per_launch": ms / nl if nl else None, "launches": nl,
                       "tflops": fl / (ms / nl / 1e3) / 1e12 if nl else None, "flops": fl,
                       "frac": fl / (ms / nl / 1e3) / 1e12 / peak if nl else None,
                       "traffic": (sum(tr) if all(t is not None for t in tr) else None)}
    per_kernel = {}
    for k, (kname, fl) in executed.items():
        ms, nl = prof[f"{k}_ms"], prof[f"{k}_launches"]
        per_kernel[k] = {"kernel": kname, "ms_per_launch": ms / nl if nl else None, "launches": nl,
                         "executed_tflops": fl / (ms / nl / 1e3) / 1e12 if nl and fl else None,
                         "executed_flops": fl,
                         "note": "runs concurrently with the other backward kernel" if k in ("bwd_kv", "bwd_q") else ""}
    dom = max(per_unit, key=lambda k: prof[f"{k}_ms"])
    pk = per_unit[dom]
    roof = {"bound": "tensor", "achieved": pk["tflops"], "peak": peak, "unit": "TFLOP/s",
            "frac": (pk["tflops"] / peak) if pk["tflops"] else None,
            "traffic": pk["traffic"], "kernel": pk["kernel"],
            "kernel_ms_per_launch": pk["ms_per_launch"], "algorithmic_flops_per_launch": pk["flops"],
            "peak_source": f"{peak_src} bf16_tflops (burst, cuBLAS bf16)",
            "units": per_unit, "kernels": per_kernel,
            "kernel_share_of_step": sum(prof[f"{k}_ms"] for k in units) / local_ms if local_ms else None}

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "pct_of_bf16_peak": 100.0 * value / world / peak,
        "config": {"workload": w.name, "description": w.description, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv,
                   "seqlen": w.N, "head_dim": w.d, "unmasked_pairs": pairs,
                   "flops_per_step": {"fwd": f_fwd, "bwd": f_bwd}, "tile_classes": hist,
                   "bwd_mode": args.bwd_mode,
                   "l2": "flushed before every step (2x L2 bytes written, outside the step's events)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "steps": e2e_steps,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / e2e_steps,
                "mode": "pipelined: step i+1's inputs in and step i-1's outputs out overlap step i's compute "
                        "(two copy streams, device buffers doubled)",
                "serial": {"value": e2e_serial_value, "ms_per_step": e2e_serial_ms / e2e_steps},
                "outputs_checked": e2e_check},
        "roofline": roof,
        "gpu_launches": launches,
        "clocks": clk,
    }
    cpu_inp = pb["inp"]
    del pb

    # ---- the other workloads (document, share-question, prefix + window), same run (not the headline) ----
    if not args.no_secondary:
        sec = {}
        for name in SECONDARY:
            if name == w.name:
                continue
            ws_ = wl.CONFIGS[name]
            sp = setup_problem(fm, ws_, dev)
            sms, sprof, _, _ = time_device(fm, sp, SECONDARY_STEPS, args.warmup, flush, world)
            sff, sfb = effective_flops(sp["pairs"], ws_.d)
            sec[name] = {"value": (sff + sfb) / (sum(sms) / len(sms) / 1e3) / 1e12, "unit": "TFLOP/s",
                         "steps": SECONDARY_STEPS, "unmasked_pairs": sp["pairs"],
                         "tile_classes": class_histogram(fm, [sp["d_in"][n] for n in MASK_NAMES], ws_),
                         "units": unit_rates(sprof, sp["pairs"], ws_.d, peak)}
            del sp
            torch.cuda.empty_cache()
        line["secondary"] = sec
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, inp=cpu_inp)
    return line


def run_reference(args, rank, world):
    if rank != 0:
        return None
    import oracle

    w = wl.CONFIGS[args.config]
    rows = 4096
    sample = oracle_sample(w, rows)
    pairs, n = sample[5], sample[6]
    ff, fb = effective_flops(pairs, w.d)
    for _ in range(args.warmup):
        run_oracle_step(sample)
    times = [run_oracle_step(sample) for _ in range(args.steps)]
    total = sum(times)
    v = (ff + fb) * args.steps / total / 1e12
    desc = (f"{w.name}: batch 0, q-head 0 with its KV head, first {n} queries x {n} keys "
            f"(mask localised onto [0,{n})), fp64 fwd+bwd per step, {pairs} unmasked pairs")
    return {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "sample_rows": n, "unmasked_pairs_per_step": pairs},
        "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "cpu_model": cpu_model(), "sample": desc},
        "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse_args()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # one process per GPU: start the replicas under torch.distributed.run
        cmd = relaunch_command(sys.argv[1:], args.gpus, free_port())
        sys.stdout.flush()
        os.execv(cmd[0], cmd)
    rank, world, local_rank = dist_env()
    if world > 1 and args.impl == "ours":
        from datetime import timedelta

        torch.distributed.init_process_group("nccl", timeout=timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        line = run_ours(args, rank, world, local_rank) if args.impl == "ours" else run_reference(args, rank, world)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1 and torch.distributed.is_initialized():
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
