#!/usr/bin/env python
"""FlashMask forward+backward benchmark on B200: effective TFLOP/s over unmasked pairs.

One step = one forward (``flashmask_fwd``) and one backward (``flashmask_bwd``)
over one batch of the workload, through the library's C ABI.  Effective FLOPs
count only unmasked (i, j) pairs: 4*d*pairs forward, 10*d*pairs backward
(pairs from the library's closed-form count).  The default workload is the
8K causal-document mask with 32 query / 8 KV heads, head_dim 128.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config NAME]

N > 1 runs under torchrun as independent replicas (one per GPU, no data-path
collective; the path has no exchange step): value = all ranks' FLOPs / max
over ranks of the device time.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
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


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="doc8k", choices=wl.CONFIG_ORDER)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args()


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


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
    with open(os.path.join(ROOT, "column_sparse_masked_b200", "csrc", name), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


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
            "seconds": dt,
            "sample": f"{w.name}: batch 0, q-heads 0..{heads - 1} each with its KV head, first {n} queries x "
                      f"{n} keys (mask localised onto [0,{n})), fp64 fwd+bwd, {pairs} unmasked pairs"}


# ----------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------
def run_ours(args, rank, world, local_rank):
    import column_sparse_masked_b200 as fm

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = wl.CONFIGS[args.config]
    inp = wl.make_inputs(w, with_grad=True)
    names = ("q", "k", "v", "do", "lts", "lte", "uts", "ute")
    host = {n: inp[n].pin_memory() for n in names}
    d_in = {n: host[n].to(dev) for n in names}
    masks = [d_in[n] for n in ("lts", "lte", "uts", "ute")]
    pairs = fm.count_unmasked(*masks, Nq=w.N, Hq=w.Hq)
    f_fwd, f_bwd = effective_flops(pairs, w.d)
    o = torch.empty_like(d_in["q"])
    lse = torch.empty(w.B, w.Hq, w.N, dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(d_in["q"]), torch.empty_like(d_in["k"]), torch.empty_like(d_in["v"])
    ws = torch.empty(fm.workspace_size("bwd", w.B, w.Hq, w.Hkv, 1, w.N, w.N, w.d), dtype=torch.uint8, device=dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(2 * l2, dtype=torch.uint8, device=dev)

    def step(src):
        fm.fwd(src["q"], src["k"], src["v"], *[src[n] for n in ("lts", "lte", "uts", "ute")], out=(o, lse),
               workspace=ws)
        fm.bwd(src["q"], src["k"], src["v"], o, lse, src["do"], *[src[n] for n in ("lts", "lte", "uts", "ute")],
               out=(dq, dk, dv), workspace=ws)

    for _ in range(args.warmup):
        flush.fill_(1)
        step(d_in)
    torch.cuda.synchronize()
    assert fm.get_status() == 0, "device status word set during warm-up"

    # ---- device-resident timing ----
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    vis = [x for x in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if x.strip()]
    clocks = ClockSampler(vis[local_rank] if local_rank < len(vis) else str(local_rank))
    barrier(world)
    torch.cuda.synchronize()
    launches0 = fm.launch_count()
    fm.profiler_read()
    fm.profiler_enable(True)
    clocks.start()
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        evs[i][0].record()
        step(d_in)
        evs[i][1].record()
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    fm.profiler_enable(False)
    prof = fm.profiler_read()
    launches = fm.launch_count() - launches0
    step_ms = [a.elapsed_time(b) for a, b in evs]
    local_ms = sum(step_ms)
    value, total_ms = aggregate(local_ms, f_fwd + f_bwd, args.steps, world, dev)
    assert fm.get_status() == 0, "device status word set during the timed steps"

    # ---- end to end: host buffers, copies inside the timed region ----
    h_out = {"o": torch.empty_like(o, device="cpu").pin_memory(),
             "lse": torch.empty_like(lse, device="cpu").pin_memory(),
             "dq": torch.empty_like(dq, device="cpu").pin_memory(),
             "dk": torch.empty_like(dk, device="cpu").pin_memory(),
             "dv": torch.empty_like(dv, device="cpu").pin_memory()}
    d_e2e = {n: torch.empty_like(d_in[n]) for n in names}

    def e2e_step():
        for n in names:
            d_e2e[n].copy_(host[n], non_blocking=True)
        step(d_e2e)
        for n, t in (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv)):
            h_out[n].copy_(t, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    e_evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        e_evs[i][0].record()
        e2e_step()
        e_evs[i][1].record()
    torch.cuda.synchronize()
    barrier(world)
    e2e_value, e2e_ms = aggregate(sum(a.elapsed_time(b) for a, b in e_evs), f_fwd + f_bwd, args.steps, world, dev)
    h2d = sum(host[n].numel() * host[n].element_size() for n in names)
    d2h = sum(t.numel() * t.element_size() for t in h_out.values())

    # ---- roofline of the dominant unit ----
    # Units: the forward kernel, and the backward's two attention kernels,
    # which run concurrently (key side on the caller's stream, query side on
    # the library's second stream) and are timed together from fork to join.
    # Algorithmic work = the matmuls the method needs over unmasked pairs:
    # forward 2 (QK^T, PV) = 4*d*pairs; backward 5 (S, dP, dV, dK, dQ) =
    # 10*d*pairs.  Executed work per kernel (reported beside it) adds the
    # query side's recomputed S and dP: key side 8*d*pairs, query side
    # 6*d*pairs.
    peaks, peak_src = load_peaks()
    d = w.d
    units = {"fwd": (("fwd_sm100.cu",), f"fm_fwd_kernel<{d}>", 4.0 * d * pairs),
             "bwd_pair": (("bwd_dkdv_sm100.cu", "bwd_dq_sm100.cu"),
                          f"fm_bwd_dkdv_kernel<{d}> + fm_bwd_dq_kernel<{d}> (concurrent)", 10.0 * d * pairs)}
    executed = {"fwd": (f"fm_fwd_kernel<{d}>", 4.0 * d * pairs),
                "bwd_kv": (f"fm_bwd_dkdv_kernel<{d}>", 8.0 * d * pairs),
                "bwd_q": (f"fm_bwd_dq_kernel<{d}>", 6.0 * d * pairs)}
    per_unit = {}
    for k, (srcs, kname, fl) in units.items():
        ms, nl = prof[f"{k}_ms"], prof[f"{k}_launches"]
        tr = [recorded_traffic(sf, w.name) for sf in srcs]
        per_unit[k] = {"kernel": kname, "ms_per_launch": ms / nl if nl else None, "launches": nl,
                       "tflops": fl / (ms / nl / 1e3) / 1e12 if nl else None, "flops": fl,
                       "traffic": (sum(tr) if all(t is not None for t in tr) else None)}
    per_kernel = {}
    for k, (kname, fl) in executed.items():
        ms, nl = prof[f"{k}_ms"], prof[f"{k}_launches"]
        per_kernel[k] = {"kernel": kname, "ms_per_launch": ms / nl if nl else None, "launches": nl,
                         "executed_tflops": fl / (ms / nl / 1e3) / 1e12 if nl else None, "executed_flops": fl,
                         "note": "runs concurrently with the other backward kernel" if k != "fwd" else ""}
    dom = max(per_unit, key=lambda k: prof[f"{k}_ms"])
    pk = per_unit[dom]
    peak = float(peaks["bf16_tflops"])
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
                   "flops_per_step": {"fwd": f_fwd, "bwd": f_bwd},
                   "l2": "flushed before every step (2x L2 bytes written, outside the step's events)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "e2e": {"value": e2e_value, "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / args.steps},
        "roofline": roof,
        "gpu_launches": launches,
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, inp=inp)
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
                         "sample": desc},
        "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse_args()
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
