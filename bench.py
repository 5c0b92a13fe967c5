#!/usr/bin/env python
"""Benchmark: Muon optimizer steps/s on the GPT-124M matrix bank (B200).

Workload: 48 x 768x768, 12 x 768x3072, 12 x 3072x768 bf16 parameters (84.9 M),
bf16 gradients N(0, 1e-3^2) plus a rank-4 spike at 10x RMS, fp32 momentum,
mu = 0.95 Nesterov, five quintic Newton-Schulz steps (3.4445, -4.7750, 2.0315),
lr 0.05, no weight decay. A step is one muon_step over the whole bank:
momentum + norm -> the Newton-Schulz chain (one persistent launch: every
step, phase and matrix) -> scaled parameter write.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

The same run also times the 64 x 1024^2 bank (20 steps after 3 warm-up
steps) for its Newton-Schulz roofline line.
`--impl reference` times the CPU oracle (host cores) on the whole bank.

N > 1 (under torchrun, one process per GPU) is data-parallel training's
optimizer step: every rank holds the same bank and its own gradient; the
ranks average the gradients with a reduce-scatter, each steps the matrices
it owns, and an all-gather brings every rank the updated bank (the bank
storage is laid out in owner order, so nothing is packed or unpacked). The
total work is one bank step however many GPUs share it (strong scaling);
`--mode replica` instead gives every rank its own bank (weak scaling).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Muon steps/s on GPT-124M matrix bank; NS TFLOP/s as % bf16 tensor peak"
UNIT = "steps/s"
WORKLOAD_ID = 2
SQUARE_ID = 3
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one
# Newton-Schulz chain launch per workload, from an ncu capture of one chain
# launch, with a hash of the kernel sources it was taken from: once the
# sources change the figure no longer describes the kernel and is reported
# as null.
NS_CHAIN_TRAFFIC = {
    2: {"bytes": 5.411568e9, "source_sha16": "bb3e714f5d444709",
        "capture": "ncu --set full, one chain launch of the GPT-124M bank (second step)"},
    3: {"bytes": 4.918166e9, "source_sha16": "bb3e714f5d444709",
        "capture": "ncu --set full, one chain launch of the 64 x 1024^2 bank (second step)"},
    5: {"bytes": 9.765142e9, "source_sha16": "bb3e714f5d444709",
        "capture": "ncu --set full, one chain launch of the ANVIL bank with its 768 x 50304 readout (second step)"},
}
KERNEL_SOURCES = ("ns_gemm.cu", "plan.cuh", "ptx.cuh", "tiles.cuh")


def launches_per_step(w) -> int:
    """Kernel launches of one optimizer step: momentum+norm, norm finalize, the
    Newton-Schulz chain (one persistent launch) and the update pass."""
    return 4


def _args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    # the end-to-end leg: long enough that its first upload and last read-back,
    # which nothing overlaps, weigh little against the steady state
    ap.add_argument("--e2e-steps", type=int, default=100)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-square", action="store_true",
                    help="skip the 64 x 1024^2 roofline line")
    ap.add_argument("--mode", default="sharded", choices=["sharded", "replica"],
                    help="N > 1: data-parallel owner-sharded step (default) or one bank per rank")
    ap.add_argument("--workload", type=int, default=WORKLOAD_ID,
                    help="1..5 (default 2, the GPT-124M bank the metric names); the others "
                         "are measured for documentation only")
    return ap.parse_args()


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return dict(hbm=p["hbm_gbs"], burst=p["bf16_tflops"],
                    sustained=p.get("bf16_tflops_sustained", p["bf16_tflops"]), src="measured")
    except Exception:
        return dict(hbm=6650.0, burst=1590.0, sustained=1400.0, src="fallback")


def code_only(text: str) -> str:
    """C/CUDA source without comments, trailing blanks and empty lines, so
    that editing a comment does not change what a hash of it describes."""
    import re
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(ln.rstrip() for ln in text.splitlines() if ln.strip())


def kernel_source_sha16() -> str:
    """Hash of the Newton-Schulz kernel's sources, code only (what a traffic
    figure describes)."""
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "muon_newton_schulz_05_b200", "csrc", f)) as fh:
            h.update(code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def chain_traffic(wid: int):
    """(bytes per chain launch, where from) or (None, why not)."""
    t = NS_CHAIN_TRAFFIC.get(wid)
    if t is None:
        return None, "no ncu capture of this workload's chain launch"
    if t["source_sha16"] != kernel_source_sha16():
        return None, "the kernel sources changed since the ncu capture"
    return t["bytes"], t["capture"]


def _workload(wid: int = WORKLOAD_ID):
    import muon_inputs as mi
    return mi.workloads()[wid]


def _ns_flops(w) -> float:
    """Algorithmic Newton-Schulz flops of one step: per matrix and iteration
    r(r+1)c (symmetric Gram) + r^2(r+1) (symmetric square) + 2r^2c (B X),
    r = min(rows, cols), c = max(rows, cols)."""
    k = len(w.hp["coeffs"])
    tot = 0.0
    for b in w.banks:
        r, c = min(b.rows, b.cols), max(b.rows, b.cols)
        tot += b.count * k * (r * (r + 1) * c + r * r * (r + 1) + 2.0 * r * r * c)
    return tot


def _config(w, extra=None, parallelism="replica per GPU (independent banks)"):
    names = {1: "single_256x512_fp32", 2: "gpt124m_matrix_bank", 3: "square_1024x1024x64_bank",
             4: "transformer_2p5b_matrix_bank", 5: "anvil_gpt124m_bank_plus_readout"}
    if w.variant == "anvil":
        mom = (f"fp32 fast/slow, beta {w.hp['beta_fast']}/{w.hp['beta_slow']}, cautious decay, "
               f"EMA {w.hp['ema_beta']}")
    else:
        mom = f"fp32, mu={w.hp['mu']}" + (", nesterov" if w.hp.get("nesterov") else "")
    touched = w.n_params * (2 + 2 + 8 + 6) / 1e9
    c = {"workload": names.get(w.cid, w.name),
         "banks": [f"{b.count}x{b.rows}x{b.cols}" for b in w.banks],
         "params": w.n_params, "param_dtype": w.param_dtype, "grad_dtype": w.grad_dtype,
         "momentum": mom, "ns_steps": len(w.hp["coeffs"]),
         "coeffs": list(w.hp["coeffs"][0]), "lr": w.hp["lr"], "weight_decay": w.hp["weight_decay"],
         "grads": f"N(0,{w.grad_sigma:g}^2)" + (f" + rank-{w.spike_rank} spike at 10x RMS" if w.spike_rank else ""),
         "l2": (f"inputs larger than L2: ~{touched:.2f} GB touched per step (126 MB L2), no flush"
                if touched > 0.126 else f"~{touched*1e3:.0f} MB touched per step: fits in L2, no flush"),
         "parallelism": parallelism}
    if extra:
        c.update(extra)
    return c


# --------------------------------------------------------------- multi-rank
def max_over_ranks(x: float, dist=None, device="cpu") -> float:
    """The largest value of x over all ranks (x itself without a process group)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, steps: int, max_ms: float) -> float:
    """Whole-job steps/s: every rank stepped its own bank `steps` times and the
    slowest rank took max_ms."""
    return world * steps / (max_ms / 1e3)


# --------------------------------------------------------------- CPU oracle
def _cpu_threads():
    try:
        import numpy  # noqa: F401
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


_PARAM_CACHE = {}


def _oracle_bank_time(w, step: int = 0, max_layers=None):
    """Seconds of one oracle step over the whole bank (every matrix, one after
    another, float64), and a description. The gradients are generated and
    converted outside the timed calls. For a bank too large to time in full
    (max_layers set), the first max_layers matrices of each shape are timed
    and the time is scaled by the bank's counts, labelled as extrapolated."""
    import numpy as np
    import muon_inputs as mi
    import oracle
    total, n, scaled = 0.0, 0, False
    for b, spec in enumerate(w.banks):
        count = spec.count if max_layers is None else min(spec.count, max_layers)
        key = (w.cid, b, count)
        if key not in _PARAM_CACHE:  # the parameters are the same every step
            _PARAM_CACHE[key] = mi.make_params(w, b, list(range(count)))
        t_bank = 0.0
        for i in range(count):
            th = oracle.as_f64(_PARAM_CACHE[key][i])
            g = oracle.as_f64(mi.make_grads(w, b, step, [i])[0])
            m = np.zeros_like(g)
            t0 = time.perf_counter()
            if w.variant == "anvil":
                oracle.anvil_step(th, g, m, m, w.hp, w.param_dtype)
            else:
                oracle.muon_step(th, g, m, w.hp, w.param_dtype)
            t_bank += time.perf_counter() - t0
            n += 1
        if count < spec.count:
            scaled = True
            t_bank *= spec.count / count
        total += t_bank
    shapes = ", ".join(f"{s.count}x{s.rows}x{s.cols}" for s in w.banks)
    if scaled:
        desc = (f"oracle {w.variant}_step (float64, numpy) on the first {max_layers} matrices of "
                f"each shape of the bank {shapes} ({n} matrices), scaled by the bank's counts "
                f"(extrapolated)")
    else:
        desc = (f"oracle {w.variant}_step (float64, numpy) on every matrix of the bank "
                f"{shapes} ({n} matrices), one full step")
    return total, desc


def _oracle_layers(w):
    """Whole bank, except the 2.5B bank (about 161 dense TFLOP per step in
    float64): one matrix of each shape, extrapolated."""
    return 1 if w.n_params > 1_000_000_000 else None


REFERENCE_BUDGET_S = 180.0   # the reference arm's whole run, warm-up included


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = _workload(args.workload)
    layers = _oracle_layers(w)
    # One untimed step over the (capped) bank first: if the requested steps
    # would not fit the budget at that rate, every later step times the first
    # `layers` matrices of each shape instead and scales them by the bank's
    # counts (labelled as a sample in the line).
    t_probe, _ = _oracle_bank_time(w, 0, layers)
    remaining = args.steps + max(args.warmup - 1, 0)
    budget = max(REFERENCE_BUDGET_S - t_probe, 0.0)
    if remaining and t_probe * remaining > budget:
        # a matrix's oracle time goes with its Newton-Schulz work, R C min(R, C)
        def work(cap):
            return sum(min(sp.count, cap) * sp.rows * sp.cols * min(sp.rows, sp.cols) for sp in w.banks)
        most = max(sp.count for sp in w.banks) if layers is None else layers
        full = work(most)
        cap = most
        while cap > 1 and t_probe * work(cap) / full * remaining > budget:
            cap -= 1
        layers = cap
    for s in range(1, args.warmup):
        _oracle_bank_time(w, s, layers)
    times = []
    desc = ""
    for s in range(args.steps):
        t, desc = _oracle_bank_time(w, args.warmup + s, layers)
        times.append(t)
    spb = sum(times) / len(times)
    v = 1.0 / spb
    cores = _cpu_threads()
    line = {"metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": spb * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference", "config": _config(w),
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": f"each of the {args.steps} timed steps: " + desc},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------- GPU path
class Clocks:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        # raw samples go to a scratch file; their summary goes into the JSON line
        self.path = os.path.join(os.environ.get("MUON_BENCH_CLOCKS_DIR", tempfile.gettempdir()),
                                 f"muon_bench_clocks_rank{index}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in open(self.path):
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        top = max(sm)
        loaded = [x for x in sm if x >= 0.5 * top] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


def run_native(args):
    import torch
    import torch.distributed as dist
    import muon_inputs as mi
    import muon_newton_schulz_05_b200 as mb

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = _workload(args.workload)
    peaks = _peaks()
    anvil = w.variant == "anvil"

    # -------- inputs (host-generated, seeded, uploaded before timing)
    banks, host_grads = [], []
    for b, spec in enumerate(w.banks):
        th = mi.make_params(w, b).to(dev)
        g = mi.make_grads(w, b, 0)
        host_grads.append(g.pin_memory())
        z = torch.zeros(th.shape, dtype=torch.float32, device=dev)
        if anvil:
            banks.append(mb.Bank(th, g.to(dev), z, torch.zeros_like(z), th.float()))
        else:
            banks.append(mb.Bank(th, g.to(dev), z))
    ws = mb.alloc_workspace([bk.shape for bk in banks], device=dev)
    H = mb.Hparams.from_dict(w.hp)
    step_fn = mb.anvil_step if anvil else mb.muon_step
    stream = torch.cuda.current_stream(dev)
    flops_step = _ns_flops(w)
    n_launch = launches_per_step(w)

    for _ in range(args.warmup):
        step_fn(banks, H, ws)
    torch.cuda.synchronize()
    assert mb.device_status(ws) == 0

    # -------- timed region: K steps, device time, NS chain bracketed live
    K = args.steps
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4 * K)]
    for e in ev:  # materialise the event handles before timing
        e.record(stream)
    t_begin, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = Clocks(local)
    clocks.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_begin.record(stream)
    for s in range(K):
        e_step0, e_ns0, e_ns1, e_step1 = ev[4 * s:4 * s + 4]
        e_step0.record(stream)
        mb.set_ns_events(e_ns0, e_ns1)
        step_fn(banks, H, ws)
        e_step1.record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    total_ms = t_begin.elapsed_time(t_end)
    ns_ms = [ev[4 * s + 1].elapsed_time(ev[4 * s + 2]) for s in range(K)]
    pre_ms = [ev[4 * s].elapsed_time(ev[4 * s + 1]) for s in range(K)]
    post_ms = [ev[4 * s + 2].elapsed_time(ev[4 * s + 3]) for s in range(K)]
    assert mb.device_status(ws) == 0
    total_ms = max_over_ranks(total_ms, dist if world > 1 else None, dev)
    ms_per_step = total_ms / K
    value = job_throughput(world, K, total_ms)

    ns_avg_ms = statistics.mean(ns_ms)
    step_ms = [ev[4 * s].elapsed_time(ev[4 * s + 3]) for s in range(K)]
    achieved = flops_step / (ns_avg_ms * 1e-3) / 1e12
    elem_bytes = sum(b.count * b.rows * b.cols for b in w.banks)
    # algorithmic bytes of the two elementwise passes per element:
    # momentum+norm: G read, M read+write 8 (ANVIL: both momenta 16), iterate hi+lo write 4
    # update: O (bf16 hi) read 2, theta read+write (ANVIL: + slow momentum 4, EMA r+w 8)
    gsz = 2 if w.grad_dtype == "bf16" else 4
    psz = 2 if w.param_dtype == "bf16" else 4
    pre_b = gsz + (16 if anvil else 8) + 4
    post_b = 2 + 2 * psz + (12 if anvil else 0)
    pre_gbs = elem_bytes * pre_b / (statistics.mean(pre_ms) * 1e-3) / 1e9
    post_gbs = elem_bytes * post_b / (statistics.mean(post_ms) * 1e-3) / 1e9

    # -------- end to end through the public API with host buffers
    # Every step uploads its gradients from pinned host memory and reads the
    # updated parameters back, pipelined the way a training loop would: the
    # upload of step s+1 (its own device gradient buffer) and the read-back of
    # step s-1 (from an on-device snapshot of the parameters) run on two copy
    # streams while step s computes.
    e2e = None
    if rank == 0 or world > 1:
        E = args.e2e_steps
        up_s, down_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        gbufs = [[torch.empty_like(bk.grad) for bk in banks] for _ in range(2)]
        snaps = [[torch.empty_like(bk.param) for bk in banks] for _ in range(2)]
        host_params = [[torch.empty(bk.param.shape, dtype=bk.param.dtype).pin_memory()
                        for bk in banks] for _ in range(2)]
        bank_sets = [[mb.Bank(bk.param, g, bk.momentum, bk.momentum_slow, bk.ema)
                      for bk, g in zip(banks, gb)] for gb in gbufs]
        h2d = sum(g.numel() * g.element_size() for g in host_grads)
        d2h = sum(p_.numel() * p_.element_size() for p_ in host_params[0])
        up_done = [torch.cuda.Event() for _ in range(2)]
        grads_free = [torch.cuda.Event() for _ in range(2)]
        snap_done = [torch.cuda.Event() for _ in range(2)]
        down_done = [torch.cuda.Event() for _ in range(2)]
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for s_ in range(E):
            i = s_ % 2
            up_s.wait_event(e0 if s_ < 2 else grads_free[i])  # step s-2 has consumed buffer i
            with torch.cuda.stream(up_s):
                for gb, g in zip(gbufs[i], host_grads):
                    gb.copy_(g, non_blocking=True)
            up_done[i].record(up_s)
            stream.wait_event(up_done[i])
            step_fn(bank_sets[i], H, ws)
            grads_free[i].record(stream)
            if s_ >= 2:
                stream.wait_event(down_done[i])  # snapshot i has been read back
            for sn, bk in zip(snaps[i], banks):
                sn.copy_(bk.param, non_blocking=True)
            snap_done[i].record(stream)
            down_s.wait_event(snap_done[i])
            with torch.cuda.stream(down_s):
                for hp_, sn in zip(host_params[i], snaps[i]):
                    hp_.copy_(sn, non_blocking=True)
            down_done[i].record(down_s)
        for i in range(min(E, 2)):
            stream.wait_event(down_done[(E - 1 - i) % 2])
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), dist if world > 1 else None, dev)
        e2e = {"value": job_throughput(world, E, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h,
               "what": "per step: pinned host->device copy of the gradients, the optimizer step "
                       "through the public API, device->host copy of the updated parameters; "
                       "copies of neighbouring steps overlap the step on two copy streams"}

    square = None
    if args.workload == WORKLOAD_ID and not args.no_square:
        square = _square_roofline(args, dev, peaks)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        spb, desc = _oracle_bank_time(w, 0, _oracle_layers(w))
        cpu = {"value": 1.0 / spb, "unit": UNIT, "cores": _cpu_threads(), "kind": "oracle",
               "sample": desc}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    traffic, traffic_src = chain_traffic(args.workload)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": _config(w),
        "roofline": _roofline(achieved, peaks, flops_step, ns_avg_ms, traffic, traffic_src),
        "roofline_square_1024x1024x64": square,
        "breakdown_ms": {"momentum_norm": statistics.mean(pre_ms), "ns_chain": ns_avg_ms,
                         "update": statistics.mean(post_ms)},
        "step_ms_p10_p50_p90": _percentiles(step_ms), "ns_chain_ms_p10_p50_p90": _percentiles(ns_ms),
        "elementwise_gbs": {"momentum_norm": pre_gbs, "update": post_gbs, "peak": peaks["hbm"]},
        "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": n_launch * K,
        "clocks": clk,
    }
    print(json.dumps(line), flush=True)
    return 0


def _percentiles(xs):
    """p10, p50, p90 of a list of per-step times (nearest rank)."""
    ys = sorted(xs)
    pick = lambda q: ys[min(len(ys) - 1, max(0, int(round(q * (len(ys) - 1)))))]
    return [pick(0.1), pick(0.5), pick(0.9)]


def _roofline(achieved, peaks, flops, launch_ms, traffic, traffic_src):
    """The chain's roofline object. The timed region is well under a second,
    so the denominator is the measured burst bf16 peak; the fraction of the
    sustained (power-capped) peak is reported beside it."""
    return {
        "bound": "tensor", "achieved": achieved, "peak": peaks["burst"], "unit": "TFLOP/s",
        "frac": achieved / peaks["burst"], "traffic": traffic, "traffic_source": traffic_src,
        "kernel": "ns_gemm_kernel (one persistent launch: every Newton-Schulz step x "
                  "Gram/Poly/Apply over the bank)",
        "flops_per_launch": flops, "launch_ms": launch_ms,
        "peak_kind": f"bf16 dense burst, {peaks['src']} (timed region under a second)",
        "frac_of_sustained": achieved / peaks["sustained"],
    }


def _square_roofline(args, dev, peaks, steps=20, warmup=3):
    """Newton-Schulz roofline on the 64 x 1024^2 bank (inputs resident, 20
    timed steps after 3 warm-up steps; chain bracketed with CUDA events)."""
    import torch
    import muon_inputs as mi
    import muon_newton_schulz_05_b200 as mb
    w = _workload(SQUARE_ID)
    banks = []
    for b in range(len(w.banks)):
        th = mi.make_params(w, b).to(dev)
        banks.append(mb.Bank(th, mi.make_grads(w, b, 0).to(dev),
                             torch.zeros(th.shape, dtype=torch.float32, device=dev)))
    ws = mb.alloc_workspace([bk.shape for bk in banks], device=dev)
    H = mb.Hparams.from_dict(w.hp)
    stream = torch.cuda.current_stream(dev)
    for _ in range(warmup):
        mb.muon_step(banks, H, ws)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * steps)]
    for e in ev:  # torch creates the event handles lazily: make them exist
        e.record(stream)
    torch.cuda.synchronize()
    for s_ in range(steps):
        mb.set_ns_events(ev[2 * s_], ev[2 * s_ + 1])
        mb.muon_step(banks, H, ws)
    torch.cuda.synchronize()
    assert mb.device_status(ws) == 0
    ns_ms = statistics.mean(ev[2 * s_].elapsed_time(ev[2 * s_ + 1]) for s_ in range(steps))
    flops = _ns_flops(w)
    traffic, src = chain_traffic(SQUARE_ID)
    r = _roofline(flops / (ns_ms * 1e-3) / 1e12, peaks, flops, ns_ms, traffic, src)
    r["workload"] = "64 x 1024x1024 bf16, quintic x5, mu 0.95, wd 0.01 (inputs resident)"
    r["steps"], r["warmup"] = steps, warmup
    del banks, ws
    torch.cuda.empty_cache()
    return r


def run_sharded(args):
    """N ranks share one data-parallel optimizer step of the bank."""
    import datetime
    import torch
    import torch.distributed as dist
    import muon_inputs as mi
    import muon_newton_schulz_05_b200 as mb
    from muon_newton_schulz_05_b200.sharded import ShardedBankMuon

    world = int(os.environ["WORLD_SIZE"])
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    w = _workload(args.workload)
    peaks = _peaks()
    anvil = w.variant == "anvil"
    shapes = [(b.count, b.rows, b.cols) for b in w.banks]
    opt = ShardedBankMuon(shapes, mi.torch_dtype(w.param_dtype), mi.torch_dtype(w.grad_dtype),
                          variant=w.variant, device=dev, ema=anvil)
    host_grads = []
    for b in range(len(w.banks)):
        opt.params[b].copy_(mi.make_params(w, b).to(dev))   # the same bank on every rank
        g = mi.make_grads(w, b, rank)                         # this rank's own gradient
        host_grads.append(g.pin_memory())
        opt.grads[b].copy_(g.to(dev))
    H = mb.Hparams.from_dict(w.hp)
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        opt.step(H)
    torch.cuda.synchronize()
    assert opt.workspace is None or mb.device_status(opt.workspace) == 0

    K = args.steps
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * K)]
    for e in ev:  # torch creates the event handles lazily: make them exist
        e.record(stream)
    t_begin, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = Clocks(local)
    clocks.start()
    time.sleep(0.3)
    dist.barrier()
    torch.cuda.synchronize()
    t_begin.record(stream)
    for s_ in range(K):
        mb.set_ns_events(ev[2 * s_], ev[2 * s_ + 1])
        opt.step(H)
    t_end.record(stream)
    torch.cuda.synchronize()
    dist.barrier()
    clk = clocks.stop()
    mb.set_ns_events(None, None)
    step_ms = t_begin.elapsed_time(t_end)
    total_ms = max_over_ranks(step_ms, dist, dev)
    owned = opt.owned_shapes()
    ns_ms = statistics.mean(ev[2 * s_].elapsed_time(ev[2 * s_ + 1]) for s_ in range(K)) if owned else 0.0

    # the same owner step without the exchange (this rank's matrices only)
    local_ms = 0.0
    if owned:
        banks = [mb.Bank(opt.params[b][lo:hi], opt.grads[b][lo:hi], opt.momentum[b],
                         opt.momentum_slow[b], opt.ema[b])
                 for b, (lo, hi) in enumerate(opt.owned) if hi > lo]
        fn = mb.anvil_step if anvil else mb.muon_step
        l0, l1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        l0.record(stream)
        for _ in range(K):
            fn(banks, H, opt.workspace)
        l1.record(stream)
        torch.cuda.synchronize()
        local_ms = l0.elapsed_time(l1) / K
    local_max = max_over_ranks(local_ms, dist, dev)

    # end to end: every step this rank's gradients come in from pinned host
    # memory and the updated bank goes out, pipelined as a training loop would:
    # the next step's gradients upload into a staging buffer on one copy
    # stream while this step runs (a device copy moves them into the
    # optimizer's gradient storage at the step's start), and a device snapshot
    # of the parameters is read back on another copy stream during the next step
    host_params = [[torch.empty(p.shape, dtype=p.dtype).pin_memory() for p in opt.params]
                   for _ in range(2)]
    stage = [[torch.empty_like(g) for g in opt.grads] for _ in range(2)]
    snaps = [[torch.empty_like(p) for p in opt.params] for _ in range(2)]
    up_s, down_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    up_done = [torch.cuda.Event() for _ in range(2)]
    staged_free = [torch.cuda.Event() for _ in range(2)]
    snap_done = [torch.cuda.Event() for _ in range(2)]
    down_done = [torch.cuda.Event() for _ in range(2)]
    E = args.e2e_steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize()
    e0.record(stream)

    def upload(i):
        up_s.wait_event(staged_free[i])       # the step that read staging buffer i has started
        with torch.cuda.stream(up_s):
            for sg, hg in zip(stage[i], host_grads):
                sg.copy_(hg, non_blocking=True)
        up_done[i].record(up_s)

    for i in range(2):
        staged_free[i].record(stream)
    upload(0)
    for s_ in range(E):
        i = s_ % 2
        if s_ + 1 < E:
            upload(1 - i)                      # the next step's gradients, during this step
        stream.wait_event(up_done[i])
        for g, sg in zip(opt.grads, stage[i]):
            g.copy_(sg, non_blocking=True)
        staged_free[i].record(stream)
        opt.step(H)
        if s_ >= 2:
            stream.wait_event(down_done[i])    # snapshot i has been read back
        for sn, p in zip(snaps[i], opt.params):
            sn.copy_(p, non_blocking=True)
        snap_done[i].record(stream)
        down_s.wait_event(snap_done[i])
        with torch.cuda.stream(down_s):
            for hp_, sn in zip(host_params[i], snaps[i]):
                hp_.copy_(sn, non_blocking=True)
        down_done[i].record(down_s)
    for i in range(min(E, 2)):
        stream.wait_event(down_done[(E - 1 - i) % 2])
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dist, dev)
    host_params = host_params[0]
    h2d = sum(g.numel() * g.element_size() for g in host_grads)
    d2h = sum(p.numel() * p.element_size() for p in host_params)
    assert opt.workspace is None or mb.device_status(opt.workspace) == 0

    my_flops = 0.0
    k = len(w.hp["coeffs"])
    for c, r_, c_ in owned:
        rr, cc = min(r_, c_), max(r_, c_)
        my_flops += c * k * (rr * (rr + 1) * cc + rr * rr * (rr + 1) + 2.0 * rr * rr * cc)
    dist.barrier()
    dist.destroy_process_group()
    if rank != 0:
        return 0
    achieved = my_flops / (ns_ms * 1e-3) / 1e12 if ns_ms > 0 else 0.0
    roof = _roofline(achieved, peaks, my_flops, ns_ms, None,
                     "no ncu capture of a multi-rank run (ncu runs on one GPU only)")
    roof["kernel"] = "ns_gemm_kernel on rank 0's owned matrices"
    line = {
        "metric": METRIC, "value": K / (total_ms / 1e3), "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": total_ms / K, "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": _config(w, parallelism=f"dp{world}: owner-sharded data-parallel step "
                                         "(reduce-scatter, owner step, all-gather; NCCL)"),
        "roofline": roof,
        "sharded": {"owned_shapes_rank0": owned, "load_max_over_mean":
                    max(opt.layout.load) / (sum(opt.layout.load) / world),
                    "local_step_ms_max": local_max, "exchange_ms": total_ms / K - local_max},
        "cpu_baseline": None,
        "e2e": {"value": E / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "what": "per step and rank: pinned host->device copy of the rank's gradients, "
                        "the sharded step, device->host copy of the updated bank; copies of "
                        "neighbouring steps overlap the step on two copy streams"},
        "gpu_launches": launches_per_step(w) * K,
        "clocks": clk,
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = _args()
    if args.impl == "reference":
        return run_reference(args)
    # under torchrun (any N, one included) the data-parallel sharded step;
    # a plain `python bench.py` is the single-GPU bank step
    if "WORLD_SIZE" in os.environ and args.mode == "sharded":
        return run_sharded(args)
    return run_native(args)


if __name__ == "__main__":
    sys.exit(main())
