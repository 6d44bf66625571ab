#!/usr/bin/env python3
"""Benchmark of the B200 MicroAdam step: Gparams/s and achieved HBM GB/s.

Default workload: the LLaMA-2-7B-shaped parameter list (d = 6,738,415,616)
with bf16 Student-t(3) gradients scaled per tensor, B_d = 16384, k_b = 164,
m = 10, b = 4 (synthetic: random-init parameters, no dataset or weights).

One step = mua_step over the whole vector: one fused launch when every block
of the vector fits the GPU at once (small vectors), else select kernel + apply
kernel.
Timing: W warm-up steps, then K steps bracketed by a barrier and a device
synchronize, timed with CUDA events on the launching stream; with N > 1 ranks
the vector is sharded by blocks and the ranks combine their (delta, Delta)
partials with one 8-byte all-reduce MAX between the two kernels; the step time
is the max over ranks. Inputs (47 GB) are far larger than L2 (126 MB).

Other arms:
  --impl reference   the CPU oracle (oracle/), timed on the host cores on a
                     bounded sample of the same workload (rank 0 only).
The JSON line also carries `roofline` (the step's algorithmic bytes, 3d + 4K
+ 4mK + 8U, over its CUDA-event time, against the measured HBM copy peak, and
per kernel its own share of those bytes, the bytes it moves and its measured
DRAM traffic), `cpu_baseline` (the oracle on a bounded sample) and `e2e`
(host-resident gradients copied in every step, scalars read back).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MicroAdam step: Gparams/s and achieved HBM GB/s (% of peak) at 1 B200"
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="llama2_7b",
                    help="llama2_7b | llama2_7b_bf16 | llama2_7b_per_tensor | flat_134m | flat_1m | "
                         "bert_base | bert_base_<B_d>[_per_tensor] | flat_1g_m<m>")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--wd", type=float, default=None,
                    help="weight decay instead of the workload's (AdamW-style, every parameter)")
    ap.add_argument("--cpu-sample", type=int, default=1 << 23,
                    help="parameters in the oracle's bounded sample")
    return ap.parse_args()


def get_workload(name, wd=None):
    import dataclasses
    w = _named_workload(name)
    return w if wd is None else dataclasses.replace(w, wd=wd)


def _named_workload(name):
    from compressed_state_optimizer_b200 import workloads as W
    if name == "llama2_7b":
        return W.llama2_7b()
    if name == "llama2_7b_bf16":
        import dataclasses
        return dataclasses.replace(W.llama2_7b(), name="llama2_7b_bf16", params="bf16")
    if name == "llama2_7b_per_tensor":
        import dataclasses
        return dataclasses.replace(W.llama2_7b(), name="llama2_7b_per_tensor", per_tensor=True)
    if name == "flat_134m":
        return W.flat_134m()
    if name == "flat_1m":
        return W.flat_small()
    if name == "bert_base":
        return W.bert_base()
    m = re.fullmatch(r"bert_base_(\d+)(_per_tensor)?", name)
    if m:
        w = W.bert_base(int(m.group(1)))
        if m.group(2):
            import dataclasses
            w = dataclasses.replace(w, name=w.name + "_per_tensor", per_tensor=True)
        return w
    m = re.fullmatch(r"flat_1g_m(\d+)", name)
    if m:
        return W.flat_1g(int(m.group(1)))
    raise SystemExit(f"unknown workload {name}")


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# --------------------------------------------------------------------- clocks
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = max(mx, float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------- helpers
def gpu_id(dev) -> str:
    """nvidia-smi's id of a torch device (its UUID, robust to device remapping)."""
    import torch
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(dev.index or 0)


def kernel_source_sha(csrc: str | None = None) -> str:
    """Hash of the CUDA sources' code (// comments and blank lines dropped, so
    a comment edit keeps a profile taken on the same code valid)."""
    h = hashlib.sha256()
    csrc = csrc or os.path.join(ROOT, "compressed_state_optimizer_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        if f.endswith((".cu", ".cuh")):
            for line in open(os.path.join(csrc, f), encoding="utf-8"):
                code = re.sub(r"//.*", "", line).rstrip()
                if code:
                    h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", f"traffic_{kernel}_{workload}.txt")
    if not os.path.exists(path):
        return None
    kv = {}
    for line in open(path):
        if ":" in line:
            k, v = line.split(":", 1)
            kv[k.strip()] = v.strip()
    if kv.get("kernel_source_sha") != kernel_source_sha():
        return None
    try:
        return float(kv["dram_bytes_per_launch_full_size"])
    except (KeyError, ValueError):
        return None


def union_size(window_u32, nb, m, kp, Bd, d, torch):
    """|U|: distinct indices in the current window (all rows), counted on the GPU."""
    total = 0
    step = max(1, (1 << 28) // (m * kp))
    for b0 in range(0, nb, step):
        b1 = min(nb, b0 + step)
        w = window_u32[b0 * m * kp: b1 * m * kp].view(b1 - b0, m * kp)
        idx = (w & 0xFFFF).to(torch.int64)
        valid = idx != 0xFFFF
        base = (torch.arange(b0, b1, device=w.device, dtype=torch.int64) * Bd).unsqueeze(1)
        flat = (idx + base)[valid]
        mask = torch.zeros((b1 - b0) * Bd, dtype=torch.bool, device=w.device)
        mask[flat - b0 * Bd] = True
        total += int(mask.sum().item())
    return total


def host_info():
    """Host cores and RAM of this box (for the CPU legs' records)."""
    cores = os.cpu_count() or 1
    try:
        ram = int(re.search(r"MemTotal:\s+(\d+)", open("/proc/meminfo").read()).group(1)) * 1024
    except Exception:
        ram = None
    return cores, ram


def _time_oracle(w, n: int, openmp: bool, max_seconds: float, min_steps: int = 2):
    """Steps t = 1, 2, ... of the oracle on the first n parameters of the
    workload until max_seconds of oracle time (gradient generation excluded)."""
    import oracle
    from compressed_state_optimizer_b200 import workloads as W
    p = W.make_params(n, seed=7).numpy().copy()
    st = oracle.new_state(n, w.Bd, w.kb, w.m)
    steps, elapsed, t0 = 0, 0.0, time.perf_counter()
    while steps < min_steps or elapsed < max_seconds:
        g = W.bf16_bits(W.make_grads(w, steps + 1, start=0, length=n))
        s0 = time.perf_counter()
        oracle.step(st, p, g, lr=w.lr, beta1=w.beta1, beta2=w.beta2, eps=w.eps, wd=w.wd,
                    t=steps + 1, seed=w.seed, openmp=openmp)
        elapsed += time.perf_counter() - s0
        steps += 1
        if time.perf_counter() - t0 > 4 * max_seconds:
            break
    return n * steps / elapsed / 1e9, steps, elapsed


def cpu_baseline(w, sample: int, max_seconds: float = 12.0):
    """The oracle as it stands on the first `sample` parameters of the workload:
    its OpenMP build on every host core (the headline) and the plain
    single-threaded build (a sub-record)."""
    import oracle
    n = min(sample, w.d)
    cores, ram = host_info()
    oracle.set_threads(cores)
    v_omp, s_omp, e_omp = _time_oracle(w, n, True, max_seconds)
    v_one, s_one, e_one = _time_oracle(w, n, False, max_seconds / 2)
    return {"value": v_omp, "unit": "Gparams/s", "cores": cores, "kind": "oracle",
            "sample": f"first {n} parameters of {w.name}, {s_omp} steps (t=1..{s_omp}), "
                      f"C oracle built with OpenMP over blocks, {cores} threads, "
                      f"{e_omp:.1f} s",
            "host_ram_bytes": ram,
            "single_thread": {"value": v_one, "unit": "Gparams/s", "cores": 1,
                              "sample": f"first {n} parameters, {s_one} steps, plain build, "
                                        f"{e_one:.1f} s"}}


# --------------------------------------------------------------------- reference arm
def run_reference(args, rank, world):
    if rank != 0:
        return
    w = get_workload(args.workload, args.wd)
    n = min(args.cpu_sample, w.d)
    import oracle
    from compressed_state_optimizer_b200 import workloads as W
    cores, ram = host_info()
    oracle.set_threads(cores)
    p = W.make_params(n, seed=7).numpy().copy()
    st = oracle.new_state(n, w.Bd, w.kb, w.m)
    grads = [W.bf16_bits(W.make_grads(w, s, start=0, length=n)) for s in (1, 2)]
    hyper = dict(lr=w.lr, beta1=w.beta1, beta2=w.beta2, eps=w.eps, wd=w.wd, seed=w.seed,
                 openmp=True)
    t = 0
    for _ in range(args.warmup):
        t += 1
        oracle.step(st, p, grads[t % 2], t=t, **hyper)
    s0 = time.perf_counter()
    for _ in range(args.steps):
        t += 1
        oracle.step(st, p, grads[t % 2], t=t, **hyper)
    el = time.perf_counter() - s0
    value = n * args.steps / el / 1e9
    line = {"metric": METRIC, "value": value, "unit": "Gparams/s", "impl": "reference",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * el / args.steps, "higher_is_better": True, "scaling": "strong",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": w.name, "d": w.d, "B_d": w.Bd, "k_b": w.kb, "m": w.m, "b": 4, "wd": w.wd,
                       "sample_params": n, "l2": "host run"},
            "cpu_baseline": {"value": value, "unit": "Gparams/s", "cores": cores, "kind": "oracle",
                             "sample": f"first {n} parameters of {w.name} per step, C oracle "
                                       f"built with OpenMP over blocks, {cores} threads",
                             "host_ram_bytes": ram},
            "e2e": {"value": value, "unit": "Gparams/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------- our arm
def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from compressed_state_optimizer_b200 import MicroAdam, sharding, workloads as W

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = get_workload(args.workload, args.wd)
    segs = w.segments()
    if segs is not None and world > 1:
        raise SystemExit("the per-tensor cut runs on one GPU")
    mo = MicroAdam(w.d, block_size=w.Bd, k_per_block=w.kb, window=w.m, segments=segs,
                   shard=None if world == 1 else sharding.shard_blocks(w.d, w.Bd, rank, world))
    d_loc, off = mo.d, mo.offset
    params = W.make_params(d_loc, seed=7 + rank, device=dev)
    if w.params == "bf16":
        params = params.to(torch.bfloat16)
    grads = [W.make_grads(w, s, device=dev, start=off, length=d_loc) for s in (1, 2)]
    state = mo.new_state(dev)
    stream = torch.cuda.current_stream(dev)
    hyper = dict(lr=w.lr, beta1=w.beta1, beta2=w.beta2, eps=w.eps, wd=w.wd, seed=w.seed)

    def step(t, g):
        if world == 1:
            mo.step(params, g, state, t=t, **hyper)
            return
        mo.select(params, g, state, t=t, **hyper)
        sharding.combine_minmax_(state, mo.minmax_offset(t))
        mo.apply(params, g, state, t=t, **hyper)

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local_rank])
        torch.cuda.synchronize(dev)

    t = 0
    for _ in range(args.warmup):
        t += 1
        step(t, grads[t % 2])
    barrier()

    # ---- timed region: K full steps (mua_step at N = 1; select, the 8-byte
    # all-reduce and apply at N > 1), each bracketed by events on the launching
    # stream. A working set that fits in L2 is flushed from it before every step (a
    # write of twice L2's size, outside the events around the step); larger
    # ones are streamed from HBM anyway.
    work_bytes = params.element_size() * d_loc + 2 * 2 * d_loc + mo.state_bytes
    l2_bytes = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = None
    if work_bytes < 4 * l2_bytes:
        flush = torch.empty(2 * l2_bytes // 4, dtype=torch.int32, device=dev)
    clocks = ClockSampler(gpu_id(dev))
    clocks.start()
    time.sleep(0.3)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    start.record(stream)
    for i in range(args.steps):
        t += 1
        if flush is not None:
            flush.fill_(i)
        ev[i][0].record(stream)
        step(t, grads[t % 2])
        ev[i][1].record(stream)
    end.record(stream)
    barrier()
    clk = clocks.stop()
    if flush is None:
        total_ms = start.elapsed_time(end)
    else:  # the steps alone, without the flushes between them
        total_ms = sum(e[0].elapsed_time(e[1]) for e in ev)

    # ---- per-kernel breakdown (outside the timed region): the two-kernel
    # path's select and apply, each timed on the launching stream.
    launches = 2 if world > 1 else mo.step_launches(bf16_params=w.params == "bf16")
    nb_steps = max(3, min(10, args.steps))
    kev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(nb_steps)]
    barrier()
    for i in range(nb_steps):
        t += 1
        g = grads[t % 2]
        if flush is not None:
            flush.fill_(i)
        kev[i][0].record(stream)
        mo.select(params, g, state, t=t, **hyper)
        kev[i][1].record(stream)
        if world > 1:
            sharding.combine_minmax_(state, mo.minmax_offset(t))
        mo.apply(params, g, state, t=t, **hyper)
        kev[i][2].record(stream)
    barrier()
    sel_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in kev)
    app_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in kev)
    fused_ms = total_ms / args.steps if launches == 1 else None
    if world > 1:
        tm = torch.tensor([total_ms], device=dev)
        dist.all_reduce(tm, op=dist.ReduceOp.MAX)
        total_ms = float(tm.item())
    ms_per_step = total_ms / args.steps
    value = w.d / (ms_per_step * 1e-3) / 1e9

    # ---- algorithmic bytes per step (this rank's shard): the method's bytes,
    # each kernel billed for its own share of them (select: g, e read, new row
    # written; apply: e written, window read, parameter read-modify-write on
    # the window's index union), and what each kernel must move in this
    # two-kernel design (apply re-reads g and e to recompute a_t).
    lay = mo.layout
    nb = lay.blocks
    if segs is None:
        L_last = d_loc - (nb - 1) * w.Bd
        K = (nb - 1) * w.kb + -(-L_last * w.kb // w.Bd)
    else:  # every tensor's blocks, its ragged last one included
        K = sum((n // w.Bd) * w.kb + -(-(n % w.Bd) * w.kb // w.Bd) for n in segs)
    win = state[lay.window: lay.window + 4 * nb * w.m * lay.row_stride].view(torch.int32)
    U = union_size(win, nb, w.m, lay.row_stride, w.Bd, d_loc, torch)
    rows = min(t, w.m)
    # parameter read-modify-write: the union (and, with weight decay, every parameter)
    rmw = 2 * params.element_size() * (d_loc if w.wd else U)
    own = {"select": 2.5 * d_loc + 4 * K, "apply": 0.5 * d_loc + 4 * rows * K + rmw}
    moved = {"select": 2.5 * d_loc + 4 * K, "apply": 3.0 * d_loc + 4 * rows * K + rmw}
    bytes_step = own["select"] + own["apply"]  # 3 d + 4 K + 4 rows K + 8 U (fp32, wd = 0)
    peak, peak_kind = measured_peak()
    kms = {"select": sel_ms, "apply": app_ms}
    kernels = {}
    traffic_step = 0.0
    for kname in ("select", "apply"):
        tr = profiled_traffic(kname, w.name)
        kernels[kname] = {
            "ms": kms[kname], "bytes": own[kname],
            "frac": own[kname] / (kms[kname] * 1e-3) / 1e9 / peak,
            "bytes_moved": moved[kname],
            "frac_moved": moved[kname] / (kms[kname] * 1e-3) / 1e9 / peak,
            "traffic": tr,
            "dram_frac": None if tr is None else tr / (kms[kname] * 1e-3) / 1e9 / peak}
        traffic_step = None if (tr is None or traffic_step is None) else traffic_step + tr
    if fused_ms is not None:  # one launch moves the method's bytes only (no re-read)
        tr = profiled_traffic("fused", w.name)
        kernels["fused"] = {"ms": fused_ms, "bytes": bytes_step,
                            "frac": bytes_step / (fused_ms * 1e-3) / 1e9 / peak,
                            "bytes_moved": bytes_step, "traffic": tr,
                            "dram_frac": None if tr is None else tr / (fused_ms * 1e-3) / 1e9 / peak}
        traffic_step = tr
    achieved = bytes_step * world / (ms_per_step * 1e-3) / 1e9
    dominant = "fused" if fused_ms is not None else ("apply" if app_ms >= sel_ms else "select")

    # ---- end to end: gradients from pinned host memory every step, scalars back.
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, step, mo, state, grads, t, w, dev, world, local_rank)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "Gparams/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic",
            "config": {"workload": w.name, "d": w.d, "B_d": w.Bd, "k_b": w.kb, "m": w.m, "wd": w.wd,
                       "params": w.params,
                       "blocks": "per tensor" if segs is not None else "over the flat vector",
                       "b": 4, "grads": w.grad, "parallelism": f"blocks sharded over {world}"
                       if world > 1 else "single GPU",
                       "l2": (f"working set {work_bytes / 1e9:.2f} GB > L2; no flush"
                              if flush is None else
                              f"working set {work_bytes / 1e6:.1f} MB fits L2: flushed "
                              f"({2 * l2_bytes >> 20} MiB write) before every step, outside "
                              "the timed events")},
            "kernels_ms": dict({"select": sel_ms, "apply": app_ms},
                               **({"fused": fused_ms} if fused_ms is not None else {})),
            "step_path": "one fused launch" if launches == 1 else "select + apply",
            "union_fraction": U / d_loc,
            "roofline": {"bound": "hbm", "kernel": "step (select + apply)", "achieved": achieved,
                         "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                         "frac": achieved / peak, "step_frac": achieved / peak,
                         "traffic": traffic_step, "algorithmic_bytes": bytes_step,
                         "dominant_kernel": dominant, "kernels": kernels},
            "gpu_launches": launches * args.steps,
            "clocks": clk,
        }
        if e2e is not None:
            line["e2e"] = e2e
        if not args.no_cpu_baseline and world == 1:  # the oracle's timing: rank 0 at N = 1 only
            line["cpu_baseline"] = cpu_baseline(w, args.cpu_sample)
        print(json.dumps(line), flush=True)


def run_e2e(args, step, mo, state, grads, t, w, dev, world, local_rank):
    import torch
    import torch.distributed as dist
    need = grads[0].numel() * 2
    try:
        avail = int(re.search(r"MemAvailable:\s+(\d+)", open("/proc/meminfo").read()).group(1)) * 1024
    except Exception:
        avail = 0
    if avail < 3 * need:
        return {"value": None, "unit": "Gparams/s", "skipped": f"host RAM {avail} B < 3x {need} B",
                "h2d_bytes_per_step": need, "d2h_bytes_per_step": 12}
    host = torch.empty(grads[0].numel(), dtype=torch.bfloat16, pin_memory=True)
    host.copy_(grads[0])
    # Two device buffers: step i's gradients cross the host link on a copy
    # stream while step i - 1 computes (every copy inside the timed region).
    bufs = [torch.empty_like(grads[0]), torch.empty_like(grads[0])]
    back = torch.empty(12, dtype=torch.uint8, pin_memory=True)
    stream = torch.cuda.current_stream(dev)
    copy_stream = torch.cuda.Stream(dev)
    steps = max(3, min(args.steps, 10))
    for _ in range(2):
        t += 1
        bufs[0].copy_(host, non_blocking=True)
        step(t, bufs[0])
    if world > 1:
        dist.barrier(device_ids=[local_rank])
    torch.cuda.synchronize(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    copied = [torch.cuda.Event(), torch.cuda.Event()]
    used = [torch.cuda.Event(), torch.cuda.Event()]

    def issue_copy(i):
        k = i % 2
        if i >= 2:
            copy_stream.wait_event(used[k])  # step i - 2 is done with this buffer
        with torch.cuda.stream(copy_stream):
            bufs[k].copy_(host, non_blocking=True)
        copied[k].record(copy_stream)

    a.record(stream)
    copy_stream.wait_event(a)
    issue_copy(0)
    for i in range(steps):
        if i + 1 < steps:
            issue_copy(i + 1)
        t += 1
        stream.wait_event(copied[i % 2])
        step(t, bufs[i % 2])
        used[i % 2].record(stream)
        back.copy_(state[:12], non_blocking=True)
    b.record(stream)
    torch.cuda.synchronize(dev)
    ms = a.elapsed_time(b) / steps
    if world > 1:
        tm = torch.tensor([ms], device=dev)
        dist.all_reduce(tm, op=dist.ReduceOp.MAX)
        ms = float(tm.item())
    return {"value": w.d / (ms * 1e-3) / 1e9, "unit": "Gparams/s",
            "h2d_bytes_per_step": need, "d2h_bytes_per_step": 12, "ms_per_step": ms,
            "steps": steps}


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world and world != 1:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE {world}")
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
