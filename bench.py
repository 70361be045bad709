"""Benchmark of the compressed step of 1-bit Adam on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One STEP is one whole compressed step (worker compression of all W workers, the compressed
allreduce's server stage, the frozen-variance apply) over the workload's parameter bucket, with
its inputs resident in HBM. The default workload is the BERT-Large-shaped bucket (333,563,904
fp32 parameters, W = 16 simulated workers, C = d/W, bf16 gradients). The metric is
params x workers / s of the compressed step, with achieved HBM GB/s against the measured copy
bandwidth. With N > 1 (torchrun, one process per GPU) every rank runs its own replica of the
whole workload (the method's W workers are simulated inside each GPU; there is no data-path
collective) and the value is the sum over ranks, timed as the max over ranks. After that
headline, the same workload runs as N data-parallel ranks (one per GPU, W / N workers each,
the compressed allreduce between the GPUs fused into the kernels over peer memory), reported in
the line's "dp" object: its step time (max over ranks), its speed-up over the single-GPU step,
the bytes each rank stores into its peers per step and every rank's status word.

``--impl reference`` times the CPU oracle (plain single-threaded C) on a bounded sample of the
same workload; rank 0 alone runs it.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

TRAFFIC_JSON = os.path.join(ROOT, "profiles", "dram_traffic_bert_large_bucket.json")
KERNEL_SRC = os.path.join(ROOT, "communication_compressed_optimizer_momentum_b200", "csrc",
                          "kernels.cuh")
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0   # B200 HBM3e, the nominal figure the targets quote
METRIC = "compressed-step params×workers/sec and achieved HBM GB/s (% of B200 peak)"
UNIT = "params*workers/s"


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=100)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--workload", default="bert_large_bucket")
    p.add_argument("--impl", default="ours", choices=("ours", "reference"))
    p.add_argument("--e2e-steps", type=int, default=3)
    p.add_argument("--cpu-seconds", type=float, default=12.0,
                   help="CPU time budget of the oracle baseline sample")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--graph", action="store_true",
                   help="replay the timed steps from a captured CUDA graph")
    p.add_argument("--scale-d", type=int, default=0,
                   help="run the workload's distributions on a smaller vector (profiling)")
    p.add_argument("--dp", type=int, default=0,
                   help="data-parallel ranks: with one process, R ranks emulated on this GPU; "
                        "under torchrun, one rank per process (R = world size)")
    p.add_argument("--variant", default="onebit", choices=("onebit", "zero_one"),
                   help="zero_one: the 0/1 Adam variant's compression phase (local steps and a "
                        "synchronisation every --sync-every steps)")
    p.add_argument("--sync-every", type=int, default=4, help="0/1 Adam: H")
    p.add_argument("--refresh-every", type=int, default=2,
                   help="0/1 Adam: variance refresh every K-th synchronisation (0: never)")
    p.add_argument("--kernel-events", default="inline", choices=("inline", "separate"),
                   help="inline: the per-kernel CUDA events are recorded inside the timed "
                        "region; separate: the timed region runs without them and the "
                        "per-kernel times come from a second pass of the same length (for "
                        "launch-bound small workloads, where recording events costs host time)")
    p.add_argument("--no-dp-section", action="store_true",
                   help="under torchrun with N > 1, skip timing the data-parallel step after "
                        "the replica headline")
    p.add_argument("--write-traffic", metavar="CSV",
                   help="write the DRAM traffic summary from an ncu CSV captured with "
                        "--scale-d on the current kernels, then exit (no GPU needed)")
    p.add_argument("--traffic-command", default="",
                   help="with --write-traffic: the ncu command line that made the CSV")
    return p.parse_args()


def get_workload(name, scale_d=0):
    from communication_compressed_optimizer_momentum_b200 import workloads as wls
    if name in wls.WORKLOADS:
        wl = wls.WORKLOADS[name]
        return wls.scaled(wl, scale_d) if scale_d else wl
    if name.startswith("sweep_W"):
        # sweep_W<w>_C<c>, c = 0 for d/W
        w, c = name[len("sweep_W"):].split("_C")
        wl = wls.sweep_workload(int(w), int(c) or None)
        if scale_d:
            wl = wls.scaled(wl, scale_d, C=None if not int(c) else min(int(c), scale_d))
        return wl
    raise SystemExit("unknown workload %s" % name)


def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_sha():
    with open(KERNEL_SRC, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


def ncu_traffic(workload):
    """DRAM bytes per launch of the step's kernels at the workload's full size, from the
    committed ncu summary (profiles/dram_traffic_bert_large_bucket.json), when it was taken on
    the current kernel source for this workload: {kernel: bytes}; otherwise {}."""
    try:
        with open(TRAFFIC_JSON) as f:
            j = json.load(f)
    except (OSError, ValueError):
        return {}
    if j.get("kernel_source_sha256") != kernel_source_sha() or j.get("workload") != workload:
        return {}
    out = {}
    for name, k in j.get("kernels", {}).items():
        try:
            out[name] = float(k["dram_bytes_per_launch_full"])
        except (KeyError, TypeError, ValueError):
            continue
    return out


def write_traffic_json(csv_path, workload, captured_params, command, out=TRAFFIC_JSON):
    """Writes the DRAM traffic summary that ncu_traffic reads, from the CSV of an
    ``ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum,gpu__time_duration.sum --csv``
    capture of the step's kernels on a ``--scale-d captured_params`` copy of the workload. The
    last captured launch of each kernel (a steady-state step) is kept; every stream of the three
    kernels is per parameter, so its bytes scale to the full workload by d / captured_params."""
    import csv
    import re
    with open(csv_path) as f:
        lines = [ln for ln in f if ln.startswith('"')]
    rows = list(csv.DictReader(lines))
    launches = {}
    for r in rows:
        m = re.search(r"\bk_(worker|server|apply)\b", r["Kernel Name"])
        if not m:
            continue
        launches.setdefault(m.group(1), {}).setdefault(int(r["ID"]), {})[r["Metric Name"]] = \
            float(r["Metric Value"].replace(",", ""))
    wl = get_workload(workload)
    kb = wl.kernel_bytes_per_param()
    scale = wl.d / captured_params
    kernels = {}
    for name in ("worker", "server", "apply"):
        if name not in launches:
            raise SystemExit("no k_%s launch in %s" % (name, csv_path))
        met = launches[name][max(launches[name])]
        rd, wr = met["dram__bytes_read.sum"], met["dram__bytes_write.sum"]
        alg = kb[name] * captured_params
        kernels[name] = {"dram_bytes_read": int(rd), "dram_bytes_write": int(wr),
                         "duration_ns": int(met["gpu__time_duration.sum"]),
                         "algorithmic_bytes_per_param": kb[name], "algorithmic_bytes": alg,
                         "dram_over_algorithmic": round((rd + wr) / alg, 4),
                         "dram_bytes_per_launch_full": int(round((rd + wr) * scale))}
    j = {"workload": workload, "kernel_source_sha256": kernel_source_sha(),
         "capture": {"command": command, "captured_params": captured_params,
                     "full_params": wl.d, "scale": scale,
                     "note": "one launch of each kernel of a steady-state compressed step on a "
                             "smaller copy of the workload; every stream of the three kernels "
                             "is per parameter, so the bytes scale to the full workload by "
                             "full_params / captured_params. When the smaller copy's sign bytes "
                             "and server plane fit the 126 MB L2, the server and apply kernels "
                             "read part of their input from L2 and their DRAM/algorithmic ratio "
                             "is a lower bound for the full size. The server kernel's table "
                             "layout depends on the grid and can differ between the copy and "
                             "the full size; it changes no DRAM stream."},
         "kernels": kernels}
    with open(out, "w") as f:
        json.dump(j, f, indent=1)
    return j


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms in a background process."""
    QUERY = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.QUERY,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self, which):
        setattr(self, which, time.time())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for t, line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                rows.append((t, float(parts[2]), float(parts[3]), parts[5:]))
            except ValueError:
                continue
        if not rows:
            return None
        inside = [r for r in rows if self.t0 is not None and self.t0 - 0.2 <= r[0] <= self.t1 + 0.2]
        use = inside or rows
        sm = sorted(r[1] for r in use)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in use:
            for nm, flag in zip(names, r[3][1:5]):
                if flag.strip().lower() in ("active", "1"):
                    reasons.add(nm)
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": max(r[2] for r in use),
                "reasons": sorted(reasons), "samples": len(use),
                "in_timed_region": bool(inside)}


def max_over_ranks(value, device):
    """The max of a per-rank number over all ranks of the default process group (the number
    itself with one rank)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def warmup_phase(wl, warm_ms):
    """Device time of the full-precision Adam warm-up steps (one launch each): the mean over
    the steps after the first, and GB/s against their minimum traffic of W*G + 24 bytes per
    parameter (gradients read; m, v and x read and written)."""
    if len(warm_ms) < 2:
        return None
    ms = sum(warm_ms[1:]) / (len(warm_ms) - 1)
    nbytes = (wl.W * wl.grad_bytes + 24) * wl.d
    return {"steps": len(warm_ms), "ms_per_step": ms, "bytes_per_step": nbytes,
            "achieved_gbs": nbytes / (ms / 1e3) / 1e9}


def step_distribution(step_ms):
    """p10 / p50 / p90 of single steps' device times (ms), nearest-rank; None without any."""
    if not step_ms:
        return None
    v = sorted(step_ms)

    def q(p):
        return v[min(len(v) - 1, max(0, int(round(p * (len(v) - 1)))))]
    return {"p10": q(0.1), "p50": q(0.5), "p90": q(0.9), "steps": len(v)}


def whole_job_rate(units_per_rank, world, ms_max):
    """Units all ranks processed per second, timed by the slowest rank."""
    return units_per_rank * world / (ms_max / 1e3)


def _to_np(t):
    import numpy as np
    import torch
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16).copy()
    return t.numpy().copy()


def host_cpu():
    """Model string and logical CPU count of the host the CPU baseline runs on."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        affinity = len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        affinity = None
    return {"model": model, "nproc": os.cpu_count(), "affinity_cpus": affinity}


def oracle_sample_rate(wl, state, g, seconds):
    """Time oracle compressed steps on one chunk-sized problem until `seconds` have passed
    (at least one step). Returns (params*workers/s, steps, elements per step)."""
    import oracle
    x, m, v, e_w, e_s = (state[k].copy() for k in ("x", "m", "v", "e_w", "e_s"))
    n = x.size
    steps = 0
    t0 = time.perf_counter()
    while True:
        oracle.compressed_step(x, m, v, e_w, e_s, g, min(wl.C, n), wl.beta1, wl.eps, wl.lr)
        steps += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    return steps * n * wl.W / el, steps, n


FULL_STEP_MAX = 1 << 23   # params x workers up to which the oracle times the whole step


def cpu_baseline(wl, opt, x, g, seconds):
    """The oracle, single-threaded, on the GPU run's post-warm-up state: whole steps of a small
    workload, else steps of chunk 0, with the whole step's time extrapolated from that rate
    (chunks are independent, so the oracle's time grows in proportion to them)."""
    full = wl.d * wl.W <= FULL_STEP_MAX
    if full:
        st = {"x": _to_np(x), "m": _to_np(opt.get_state("m")), "v": _to_np(opt.get_state("v")),
              "e_w": _to_np(opt.get_state("e_w")), "e_s": _to_np(opt.get_state("e_s"))}
        gk = _to_np(g)
    else:
        lo, hi = 0, min(wl.d, wl.C)
        st = {"x": _to_np(x[lo:hi]), "m": _to_np(opt.get_chunk_state("m", 0)),
              "v": _to_np(opt.get_chunk_state("v", 0)),
              "e_w": _to_np(opt.get_chunk_state("e_w", 0)),
              "e_s": _to_np(opt.get_chunk_state("e_s", 0))}
        gk = _to_np(g[:, lo:hi])
    rate, n_steps, n = oracle_sample_rate(wl, st, gk, seconds)
    what = "the whole workload" if full else "chunk 0 of the workload"
    out = {"value": rate, "unit": UNIT, "cores": 1, "kind": "oracle",
           "sample": "%s (%d params x %d workers), %d oracle compressed step(s), "
                     "single-threaded C" % (what, n, wl.W, n_steps),
           "host": host_cpu()}
    if full:
        out["s_per_step"] = wl.d * wl.W / rate
    else:
        out["extrapolated_s_per_step"] = wl.d * wl.W / rate
    return out


def dp_ranks_supported(wl, world):
    """Whether the workload's W workers split evenly over `world` data-parallel ranks (at most
    eight, the library's limit)."""
    return 1 < world <= 8 and wl.W % world == 0


def dp_subobject(wl, R, ms_max, single_ms, flags_per_rank):
    """The data-parallel part of the multi-GPU JSON line: the step of R ranks (W / R workers
    each) timed as the max over ranks, its speed-up over the single-GPU step of the same
    workload, the bytes each rank stores into other ranks' memory per step, and every rank's
    status word (bit 4 = a barrier wait ran out)."""
    flags = [int(f) for f in flags_per_rank]
    return {"ranks": R, "workers_per_rank": wl.W // R, "ms_per_step": ms_max,
            "strong_scaling_vs_single": (single_ms / ms_max) if ms_max > 0 else None,
            "nvlink_bytes_per_rank_per_step": wl.dp_nvlink_bytes_per_rank(R),
            "status_flags_per_rank": flags,
            "timeout_seen": any(f & 4 for f in flags)}


def time_dp_process_ranks(wl, R, rank, dev, steps, warmup, warm_steps=None, sampler=None):
    """One data-parallel rank per process (this process is `rank` of R, connected to the others
    through CUDA IPC over the default process group): warm-up, freeze, `warmup` untimed and
    `steps` timed compressed steps. Returns (max-over-ranks ms for the timed steps, this rank's
    status word, the warm-up ms per step, rank 0's per-kernel ms per step). Every rank takes the
    same collective steps in the same order."""
    import torch
    import torch.distributed as dist

    from communication_compressed_optimizer_momentum_b200 import dp
    from communication_compressed_optimizer_momentum_b200 import workloads as wls
    Wl = wl.W // R
    dt = wls.torch_dtype(wl)
    x = wls.torch_params(wl, dev)
    g = torch.empty((wl.W, wl.d), dtype=dt, device=dev)
    opt = dp.OneBitAdamRank(wl.d, wl.W, wl.C, R, rank, wl.beta1, wl.beta2, wl.eps,
                            grad_dtype=dt, device=dev)
    dp.connect_process_group(opt)

    def mine(phase, t):
        wls.torch_fill_grads(wl, g, phase, t)
        v = g[rank * Wl:(rank + 1) * Wl]
        return v if v.data_ptr() % 16 == 0 else v.clone()
    warm_ms = []
    for t in range(wl.warmup_steps if warm_steps is None else warm_steps):
        gr = mine(0, t)
        w0 = torch.cuda.Event(enable_timing=True)
        w1 = torch.cuda.Event(enable_timing=True)
        w0.record()
        opt.warmup_step(x, gr, wl.lr)
        w1.record()
        w1.synchronize()
        warm_ms.append(w0.elapsed_time(w1))
    opt.freeze()
    gr = mine(1, 1)
    torch.cuda.synchronize()
    for _ in range(max(warmup, 0)):
        opt.step(x, gr, wl.lr)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    opt.timing(steps)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize()
    if sampler is not None:
        sampler.mark("t0")
    t0.record(stream)
    for _ in range(steps):
        opt.step(x, gr, wl.lr)
    t1.record(stream)
    torch.cuda.synchronize()
    if sampler is not None:
        sampler.mark("t1")
    dist.barrier()
    ms = t0.elapsed_time(t1)
    kms, nrec = opt.timing_read()
    opt.timing(0)
    ms_max = max_over_ranks(ms, dev)
    flags = opt.status()
    # every rank's exchange region stays mapped until all ranks are done with it
    torch.cuda.synchronize()
    dist.barrier()
    opt.close()
    del x, g, gr
    torch.cuda.empty_cache()
    return ms_max, flags, warm_ms, {k: v / max(nrec, 1) for k, v in kms.items()}


def gather_flags(flags, world):
    """Every rank's status word, in rank order (the flags themselves with one rank)."""
    import torch.distributed as dist
    if world == 1 or not (dist.is_available() and dist.is_initialized()):
        return [int(flags)]
    out = [0] * world
    dist.all_gather_object(out, int(flags))
    return out


def run_ours(args):
    import torch
    import torch.distributed as dist

    import communication_compressed_optimizer_momentum_b200 as ob
    from communication_compressed_optimizer_momentum_b200 import workloads as wls

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        # one replica per GPU; NCCL carries only the barriers and the max-over-ranks timing
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600), device_id=dev)
    wl = get_workload(args.workload, args.scale_d)
    dt = wls.torch_dtype(wl)

    x = wls.torch_params(wl, dev)
    g = torch.empty((wl.W, wl.d), dtype=dt, device=dev)
    zero_one = args.variant == "zero_one"
    if zero_one and args.graph:
        raise SystemExit("--graph: the 0/1 variant's steps differ from step to step")
    if zero_one:
        opt = ob.ZeroOneAdam(wl.d, wl.W, wl.C, args.sync_every, args.refresh_every, wl.beta1,
                             wl.beta2, wl.eps, grad_dtype=dt, device=dev)
    else:
        opt = ob.OneBitAdam(wl.d, wl.W, wl.C, wl.beta1, wl.beta2, wl.eps, grad_dtype=dt,
                            device=dev)
    warm_ms = []
    for t in range(wl.warmup_steps):             # full-precision Adam warm-up (setup)
        wls.torch_fill_grads(wl, g, 0, t)
        w0 = torch.cuda.Event(enable_timing=True)
        w1 = torch.cuda.Event(enable_timing=True)
        w0.record()
        opt.warmup_step(x, g, wl.lr)
        w1.record()
        w1.synchronize()
        warm_ms.append(w0.elapsed_time(w1))
    opt.freeze()
    wls.torch_fill_grads(wl, g, 1, 1)            # resident inputs for the timed steps
    torch.cuda.synchronize()
    for _ in range(max(args.warmup, 0)):
        opt.step(x, g, wl.lr)
    torch.cuda.synchronize()

    stream = torch.cuda.current_stream()
    graph = None
    if args.graph:
        # one step captured after the first (explicit-momentum) steps; each replay is one step
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            opt.step(x, g, wl.lr)
        torch.cuda.synchronize()
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.5)
    inline_events = graph is None and args.kernel_events == "inline"
    opt.timing(args.steps if inline_events else 0)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.mark("t0")
    t_start.record(stream)
    for _ in range(args.steps):
        if graph is not None:
            graph.replay()
        else:
            opt.step(x, g, wl.lr)
    t_end.record(stream)
    torch.cuda.synchronize()
    sampler.mark("t1")
    if world > 1:
        dist.barrier()
    ms = t_start.elapsed_time(t_end)
    if graph is None and not inline_events:
        # the same number of steps again, eager, with the per-kernel events
        opt.timing(args.steps)
        for _ in range(args.steps):
            opt.step(x, g, wl.lr)
        torch.cuda.synchronize()
    per_step = opt.timing_steps(args.steps) if graph is None else []
    kernel_ms, nrec = opt.timing_read()
    opt.timing(0)
    time.sleep(0.3)
    clocks = sampler.stop()
    ms_max = max_over_ranks(ms, dev)
    status = opt.status()

    value = whole_job_rate(wl.d * wl.W * args.steps, world, ms_max)
    step_bytes = (wl.zero_one_bytes_per_param(args.sync_every, args.refresh_every) if zero_one
                  else wl.algorithmic_bytes_per_param()) * wl.d
    achieved_step_gbs = step_bytes * args.steps / (ms_max / 1e3) / 1e9
    peak, peak_src = measured_hbm_peak()
    kb = wl.kernel_bytes_per_param()
    traffic = ncu_traffic(wl.name)
    worker_bytes = kb["worker"] * wl.d
    worker_ms = kernel_ms["worker"] / max(nrec, 1)
    worker_gbs = worker_bytes / (worker_ms / 1e3) / 1e9 if worker_ms > 0 else None
    if graph is not None:
        del graph

    # end to end through the host-buffer entry point: H2D grads, the step, D2H x
    e2e = None
    if not args.no_e2e and args.e2e_steps > 0 and not zero_one:
        g_host = torch.empty((wl.W, wl.d), dtype=dt, pin_memory=True)
        g_host.copy_(g)
        x_host = torch.empty(wl.d, dtype=torch.float32, pin_memory=True)
        opt.step_host(x, g, g_host, x_host, wl.lr)      # untimed first call
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            opt.step_host(x, g, g_host, x_host, wl.lr)
        opt.host_wait()                                 # the last read-back is inside the timing
        e1.record(stream)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
        e2e = {"value": whole_job_rate(wl.d * wl.W * args.e2e_steps, world, e_ms),
               "unit": UNIT, "steps": args.e2e_steps,
               "h2d_bytes_per_step": wl.W * wl.d * wl.grad_bytes,
               "d2h_bytes_per_step": wl.d * 4}
        del g_host, x_host

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not zero_one:
        cpu = cpu_baseline(wl, opt, x, g, args.cpu_seconds)

    line = None
    if rank == 0:
        from communication_compressed_optimizer_momentum_b200 import workloads as _w
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": dict(_w.describe(wl), parallelism="replicas" if world > 1 else "single",
                           l2="inputs larger than L2 (%.1f GB resident); no flush" % (
                               (opt.workspace_bytes + wl.W * wl.d * wl.grad_bytes
                                + wl.d * 4) / 1e9),
                           grads_resident="one seeded draw reused by every timed step",
                           cuda_graph=bool(args.graph),
                           kernel_events=("none (graph replay)" if args.graph else
                                          "inside the timed region" if inline_events else
                                          "separate pass after the timed region")),
            "achieved_hbm_gbs": achieved_step_gbs,
            "pct_of_hbm_peak": 100.0 * achieved_step_gbs / peak,
            "pct_of_nominal_hbm": 100.0 * achieved_step_gbs / NOMINAL_HBM_GBS,
            "algorithmic_bytes_per_step": step_bytes,
            "kernel_ms_per_step": {k2: v2 / max(nrec, 1) for k2, v2 in kernel_ms.items()},
            # the distribution of single steps' device time (first to last event of each step,
            # from the same per-kernel events)
            "step_ms_distribution": step_distribution(per_step),
            # one worker's message against its fp32 vector: d/8 sign bytes + one fp32 scale per
            # chunk, against 4d bytes
            "compression_ratio": 4.0 * wl.d / (wl.d / 8.0 + 4.0 * wl.nch),
            "roofline": {"bound": "hbm", "kernel": "worker", "achieved": worker_gbs,
                         "peak": peak, "peak_source": peak_src, "unit": "GB/s",
                         "frac": (worker_gbs / peak) if worker_gbs else None,
                         "traffic": traffic.get("worker"),
                         "algorithmic_bytes_per_launch": worker_bytes},
            # every streaming kernel's ncu DRAM bytes per launch against its algorithmic bytes
            "traffic_by_kernel": {k2: {"dram_bytes": traffic[k2],
                                       "algorithmic_bytes": kb[k2] * wl.d,
                                       "ratio": traffic[k2] / (kb[k2] * wl.d)}
                                  for k2 in ("worker", "server", "apply") if k2 in traffic},
            "warmup_phase": warmup_phase(wl, warm_ms),
            "gpu_launches": opt.info()["launches_per_step"] * args.steps,
            "clocks": clocks, "e2e": e2e, "cpu_baseline": cpu, "status_flags": status,
        }
    if line is not None and zero_one:
        # the variant's steps differ (local ones, a synchronising one every H): the roofline is
        # the whole step's average bytes against its average time
        line["config"].update(variant="0/1 Adam", sync_every=args.sync_every,
                              refresh_every=args.refresh_every)
        line["roofline"] = {"bound": "hbm", "kernel": "whole step (average over an interval)",
                            "achieved": achieved_step_gbs, "peak": peak,
                            "peak_source": peak_src, "unit": "GB/s",
                            "frac": achieved_step_gbs / peak, "traffic": None,
                            "algorithmic_bytes_per_launch": step_bytes}
        H, w0 = args.sync_every, max(args.warmup, 0)
        syncs = (w0 + args.steps) // H - w0 // H       # synchronising steps among the timed ones
        line["gpu_launches"] = args.steps + 4 * syncs
    opt.close()
    if world > 1:
        # after the replica headline, the same workload as data-parallel ranks: one rank per
        # GPU, W / N workers each, the compressed allreduce between the GPUs fused into the
        # kernels over peer memory (the same collective steps on every rank)
        del x, g
        torch.cuda.empty_cache()
        dp_obj = None
        if args.no_dp_section:
            dp_obj = {"skipped": "--no-dp-section"}
        elif zero_one:
            dp_obj = {"skipped": "the 0/1 Adam variant runs on one GPU only"}
        elif not dp_ranks_supported(wl, world):
            dp_obj = {"skipped": "the workload's %d workers do not split over %d ranks"
                                 % (wl.W, world)}
        else:
            dms, dflags, _, dkms = time_dp_process_ranks(wl, world, rank, dev, args.steps,
                                                         args.warmup, warm_steps=3)
            flags_all = gather_flags(dflags, world)
            dp_obj = dp_subobject(wl, world, dms / args.steps, ms_max / args.steps, flags_all)
            dp_obj["rank0_kernel_ms_per_step"] = dkms
        if line is not None:
            line["dp"] = dp_obj
    if line is not None:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_dp(args):
    """The data-parallel step: R ranks, W / R workers each, rank q serving a 1/R share of the
    chunks. One process: the R ranks are emulated as R handles on this GPU, stepped phase by
    phase (the exchange then moves through this GPU's own memory); the single-GPU step of the
    same workload is timed beside it. Under torchrun: one rank per process over CUDA IPC, the
    value the whole job's params x workers / s (the W workers are fixed: strong scaling)."""
    import torch
    import torch.distributed as dist

    import communication_compressed_optimizer_momentum_b200 as ob
    from communication_compressed_optimizer_momentum_b200 import dp
    from communication_compressed_optimizer_momentum_b200 import workloads as wls

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    # under torchrun (even with one process) each process is one rank over a process group;
    # a plain process emulates args.dp ranks on its GPU
    real = world > 1 or "LOCAL_RANK" in os.environ
    R = world if real else args.dp
    wl = get_workload(args.workload, args.scale_d)
    if wl.W % R:
        raise SystemExit("--dp %d: the workload's %d workers do not split over %d ranks"
                         % (R, wl.W, R))
    Wl = wl.W // R
    dt = wls.torch_dtype(wl)
    sampler = ClockSampler(local)
    single_ms = None
    if real:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600), device_id=dev)
        sampler.start()
        time.sleep(0.5)
        ms_max, flags, warm_ms, kernel_ms = time_dp_process_ranks(
            wl, R, rank, dev, args.steps, args.warmup, sampler=sampler)
        clocks = sampler.stop()
        status = 0
        for f in gather_flags(flags, world):
            status |= f
        launches = 7
    else:
        x0 = wls.torch_params(wl, dev)
        em = dp.EmulatedRanks(wl.d, wl.W, wl.C, R, wl.beta1, wl.beta2, wl.eps, grad_dtype=dt,
                              device=dev)
        xs = [x0.clone() for _ in range(R)]
        g = torch.empty((wl.W, wl.d), dtype=dt, device=dev)

        def fill(phase, t):
            wls.torch_fill_grads(wl, g, phase, t)
            out = []
            for r in range(R):
                v = g[r * Wl:(r + 1) * Wl]
                out.append(v if v.data_ptr() % 16 == 0 else v.clone())
            return out
        launches = 9 * R                  # phase by phase: a signal and a wait launch each
        warm_ms = []
        for t in range(wl.warmup_steps):
            gs = fill(0, t)
            w0 = torch.cuda.Event(enable_timing=True)
            w1 = torch.cuda.Event(enable_timing=True)
            w0.record()
            em.warmup_step(xs, gs, wl.lr)
            w1.record()
            w1.synchronize()
            warm_ms.append(w0.elapsed_time(w1))
        em.freeze()
        gs = fill(1, 1)
        torch.cuda.synchronize()
        for _ in range(max(args.warmup, 0)):
            em.step(xs, gs, wl.lr)
        torch.cuda.synchronize()
        stream = torch.cuda.current_stream()
        sampler.start()
        time.sleep(0.5)
        # per-kernel events of rank 0: only meaningful when its launches are not interleaved
        # with other emulated ranks' (a single rank)
        if R == 1:
            em.ranks[0].timing(args.steps)
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        sampler.mark("t0")
        t0.record(stream)
        for _ in range(args.steps):
            em.step(xs, gs, wl.lr)
        t1.record(stream)
        torch.cuda.synchronize()
        sampler.mark("t1")
        ms_max = t0.elapsed_time(t1)
        kernel_ms = None
        if R == 1:
            kms, nrec = em.ranks[0].timing_read()
            em.ranks[0].timing(0)
            kernel_ms = {k: v / max(nrec, 1) for k, v in kms.items()}
        time.sleep(0.3)
        clocks = sampler.stop()
        status = em.status()
        # the single-GPU step of the same workload, same process, for comparison
        em.close()
        del em, xs
        torch.cuda.empty_cache()
        one = ob.OneBitAdam(wl.d, wl.W, wl.C, wl.beta1, wl.beta2, wl.eps, grad_dtype=dt,
                            device=dev)
        x1 = x0.clone()
        one.warmup_step(x1, g, wl.lr)
        one.freeze()
        for _ in range(max(args.warmup, 0)):
            one.step(x1, g, wl.lr)
        torch.cuda.synchronize()
        s0 = torch.cuda.Event(enable_timing=True)
        s1 = torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        for _ in range(args.steps):
            one.step(x1, g, wl.lr)
        s1.record(stream)
        torch.cuda.synchronize()
        single_ms = s0.elapsed_time(s1) / args.steps
        one.close()
    peak, peak_src = measured_hbm_peak()
    n_gpu = max(world, 1)
    step_bytes = wl.dp_algorithmic_bytes_per_param(R) * wl.d
    achieved = step_bytes * args.steps / (ms_max / 1e3) / 1e9
    if rank == 0:
        line = {
            "metric": METRIC, "value": whole_job_rate(wl.d * wl.W * args.steps, 1, ms_max),
            "unit": UNIT, "n_gpus": n_gpu, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_max / args.steps, "higher_is_better": True,
            "scaling": "strong" if real else "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": dict(wls.describe(wl),
                           parallelism=("dp%d" % R) if real else
                           ("dp%d emulated on one GPU" % R),
                           workers_per_rank=Wl,
                           l2="inputs larger than L2; no flush"),
            "achieved_hbm_gbs": achieved,
            "pct_of_hbm_peak": 100.0 * achieved / (peak * n_gpu),
            "algorithmic_bytes_per_step": step_bytes,
            "roofline": {"bound": "hbm", "kernel": "whole data-parallel step",
                         "achieved": achieved / n_gpu, "peak": peak, "peak_source": peak_src,
                         "unit": "GB/s", "frac": achieved / n_gpu / peak, "traffic": None},
            "single_gpu_ms_per_step": single_ms,
            "rank0_kernel_ms_per_step": kernel_ms,
            # what crosses NVLink between real ranks (here it stays in this GPU's memory when
            # the ranks are emulated), against the measured 770 GB/s peer copy bandwidth
            "nvlink": {"bytes_per_rank_per_step": wl.dp_nvlink_bytes_per_rank(R),
                       "ms_at_770_gbs": wl.dp_nvlink_bytes_per_rank(R) / 770e9 * 1e3,
                       "hbm_ms_per_rank_at_peak": step_bytes / R / (peak * 1e9) * 1e3},
            "warmup_phase": ({"steps": len(warm_ms),
                              "ms_per_step": sum(warm_ms[1:]) / (len(warm_ms) - 1)}
                             if len(warm_ms) > 1 else None),
            "gpu_launches": launches * args.steps,
            "clocks": clocks, "e2e": None, "cpu_baseline": None, "status_flags": status,
        }
        print(json.dumps(line), flush=True)
    if real:
        dist.barrier()
        dist.destroy_process_group()


def run_reference(args):
    """The oracle as it stands on the host cores, on a bounded sample of the same workload."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    from communication_compressed_optimizer_momentum_b200 import workloads as wls
    wl = get_workload(args.workload)
    n = min(wl.d, 1 << 20)
    sw = wls.scaled(wl, n, C=min(wl.C, n))
    x = wls.np_params(sw)
    st = oracle.OracleState(x, sw.W, sw.C, sw.beta1, sw.beta2, sw.eps)
    st.warmup_step(wls.np_grads(sw, 0, 0), sw.lr)
    st.freeze()
    g = wls.np_grads(sw, 1, 1)
    for _ in range(max(args.warmup, 0)):
        st.compressed_step(g, sw.lr)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        st.compressed_step(g, sw.lr)
    el = time.perf_counter() - t0
    value = n * sw.W * args.steps / el
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * el / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic", "impl": "reference",
        "config": dict(wls.describe(wl), sample_d=n, sample_C=sw.C),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": "%d params x %d workers (one chunk) of %s per step, "
                                   "single-threaded C oracle" % (n, sw.W, wl.name),
                         "host": host_cpu()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    if args.write_traffic:
        if not args.scale_d:
            raise SystemExit("--write-traffic needs the --scale-d the capture ran with")
        j = write_traffic_json(args.write_traffic, args.workload, args.scale_d,
                               args.traffic_command)
        print(json.dumps({k: v["dram_over_algorithmic"] for k, v in j["kernels"].items()}))
    elif args.impl == "reference":
        run_reference(args)
    elif args.dp:
        run_dp(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
