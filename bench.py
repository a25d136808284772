"""Benchmark of the Key-only GLA hot path (gate projection + GLA forward).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 16k|640|640b8]
    python bench.py --impl reference ...       # the fp64 CPU oracle, same workload

One step = the whole hot path over one batch: gtr_gate_fwd (g from x) then
gtr_gla_fwd (summary, boundary scan, output with the fused RMSNorm x SiLU
epilogue), both through the C ABI.  Metric: token-heads per second,
B*T*H per step, whole job (all ranks).

Timing: inputs resident in HBM; four input sets rotate so that every step
reads data that is not in L2 (the four sets together exceed the 126 MB L2).
Each step is one CUDA graph replay (one graph per input set, captured once);
K steps are timed with CUDA events on the launch stream, bracketed by a
barrier and device synchronisation, max over ranks.  A second set of graphs
also holds CUDA events around every kernel (event nodes add a few us per
kernel boundary, so those graphs are timed separately, K more steps, and
give the per-kernel durations of the
roofline entry.  nvidia-smi samples clocks during the timed region.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from linear_vision_backbone_b200 import inputs as gin  # noqa: E402

N_SETS = 4
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.txt")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", default="ours", choices=("ours", "reference"))
    ap.add_argument("--workload", default="16k", choices=("16k", "640", "640b8"))
    ap.add_argument("--chunk", type=int, default=64)
    ap.add_argument("--e2e-steps", type=int, default=40)
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--fused", action="store_true",
                    help="time gtr_gla_fwd_gated (gate second half inside the summary kernel)")
    return ap.parse_args()


def workload_text(wl: gin.Workload) -> str:
    return (f"{wl.name}: B={wl.B}, {wl.gh}x{wl.gw} grid (T={wl.T}), H={wl.H}, dk=dv={wl.dk}, "
            f"{wl.dtype}, scans {'/'.join(wl.dirs)}, gate rank {wl.rank} tau {wl.tau:g}, seed {wl.seed}")


def step_dirs(wl):
    return list(wl.dirs)


def alg_bytes(wl, esz, fused=False):
    """Algorithmic bytes per launch of each kernel: the unique reads and writes
    of the operator's own tensors, without the workspace (boundary states).
    Per token-head at dk = dv = 64 with 16-bit tensors: output kernel q, k, v,
    z, out (2 x 64 bytes each) and g (4 x 64) = 896 bytes; summary kernel k, v,
    g = 512 bytes; the boundary scan touches only the workspace (0).  fused:
    the gate kernel writes the rank-16 rows x W_down (fp32) and the summary
    kernel reads them and writes g."""
    th = wl.token_heads
    dk, dv = wl.dk, wl.dv
    low = wl.B * wl.T * wl.rank * 4
    return {
        "gate": wl.B * wl.T * wl.d_model * esz + (low if fused else th * dk * 4),
        "summary": th * (dk * esz + dv * esz + dk * 4) + (low if fused else 0),
        "scan": 0,
        "output": th * (2 * dk * esz + 2 * dv * esz + dk * 4) + th * dv * esz,
    }


def workspace_bytes(wl, nstates):
    """Bytes of boundary-state traffic per launch (workspace, not algorithmic):
    the summary kernel writes each of the `nstates` states (dk x dv fp32 and a
    dk decay vector), the scan reads and rewrites them, the output kernel reads
    them."""
    st = wl.B * wl.H * nstates * (wl.dk * wl.dv + wl.dk) * 4
    return {"gate": 0, "summary": st, "scan": 2 * st, "output": st}


def host_cpu():
    """Core count and CPU model of the host the CPU baseline runs on."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    model = ln.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"host_cores": os.cpu_count(), "cpu_model": model}


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = []
        for ln in out.splitlines():
            p = [x.strip() for x in ln.split(",")]
            if len(p) < 9:
                continue
            try:
                rows.append({"sm": float(p[1]), "max": float(p[2]), "power": float(p[3]),
                             "hw": p[5], "hwt": p[6], "swt": p[7], "pcap": p[8]})
            except ValueError:
                continue
        if not rows:
            return None
        load = [r for r in rows if r["power"] > 200.0] or rows
        reasons = set()
        for r in load:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in load),
                "sm_max_mhz": max(r["max"] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows), "samples_under_load": len(load)}


# ---------------------------------------------------------------- helpers
def record_external(ev, stream):
    """Record a torch event as an external event node when the stream is being
    captured (a plain record inside capture is only a dependency, not a
    timestamp), else as an ordinary record."""
    from cuda.bindings import runtime as rt
    err, status = rt.cudaStreamIsCapturing(stream.cuda_stream)
    capturing = status == rt.cudaStreamCaptureStatus.cudaStreamCaptureStatusActive
    if capturing:
        (err,) = rt.cudaEventRecordWithFlags(ev.cuda_event, stream.cuda_stream,
                                             rt.cudaEventRecordExternal)
    else:
        (err,) = rt.cudaEventRecord(ev.cuda_event, stream.cuda_stream)
    assert err == rt.cudaError_t.cudaSuccess, err


def event_ms(a, b) -> float:
    """Elapsed ms between two recorded events, read through the CUDA runtime
    (the events may have been recorded by the library or by graph replays)."""
    from cuda.bindings import runtime as rt
    err, ms = rt.cudaEventElapsedTime(a.cuda_event, b.cuda_event)
    assert err == rt.cudaError_t.cudaSuccess, err
    return float(ms)


def read_peak():
    try:
        with open(PEAKS_FILE) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def read_traffic(kernel_name: str, src_hash: str):
    """DRAM bytes per launch of a kernel from the committed ncu summary, if the
    summary was taken on the current kernel source (matching hash)."""
    try:
        with open(TRAFFIC_FILE) as f:
            for ln in f:
                p = ln.split()
                if len(p) >= 4 and p[0] == kernel_name and p[1] == src_hash:
                    return float(p[2]), p[3]
    except OSError:
        pass
    return None, None


def kernel_source_hash():
    """Hash of the CUDA sources the gate + GLA step is compiled from (the
    translation unit gtr_gla.cu and the headers beside it, less the projection
    GEMM's own headers gemm_*.cuh and mixer_proj.cuh and the 128-dim head
    kernels tc128_kernels.cuh, which define no code the step runs; another .cu file is its own translation unit and cannot change
    these kernels), with comments and blank space removed, so that a figure
    measured on a kernel stays attached to it through comment edits."""
    import hashlib
    import re
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "linear_vision_backbone_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.endswith(".cu") and name != "gtr_gla.cu":
            continue
        if name.startswith("gemm_") or name in ("mixer_proj.cuh", "tc128_kernels.cuh"):
            continue
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        text = " ".join(text.split())
        h.update(name.encode())
        h.update(text.encode())
    return h.hexdigest()[:12]


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The largest value over all ranks (device timings: the slowest rank sets the time)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_value(units_per_rank: int, steps: int, ms_max: float, world: int) -> float:
    """Whole-job throughput: the units every rank processed over the slowest rank's time."""
    return world * units_per_rank * steps / (ms_max * 1e-3)


# ---------------------------------------------------------------- CPU oracle
def oracle_rate_config(wl, seconds=2.0):
    """Token-heads/s of the fp64 oracle on a bounded sample of any workload:
    the gate + GLA of the first grid rows for the projected workloads (as
    oracle_rate), the GLA on its drawn gates for the others (every head of
    batch entry 0 over the first rows holding about 4096 tokens)."""
    if wl.recipe == "proj":
        return oracle_rate(wl, seconds=seconds, rows=8)
    import oracle
    cores = os.cpu_count() or 1
    used = min(oracle.set_threads(cores), wl.H)
    d = gin.make_inputs(wl)
    rows = max(1, min(wl.gh, 4096 // wl.gw))
    T = rows * wl.gw
    q, k, v, g, z = (d[n][:1, :T] for n in ("q", "k", "v", "g", "z"))
    t0 = time.perf_counter()
    n = 0
    while True:
        oracle.gla_fwd(q, k, v, g, z, d["w"], gh=rows, gw=wl.gw, direction=wl.dirs[0])
        n += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    return {"value": n * T * wl.H / el, "unit": "token-heads/s", "cores": used, "kind": "oracle",
            "sample": f"GLA of all {wl.H} heads over the first {rows}x{wl.gw}={T} tokens of the "
                      f"{wl.name} workload (batch entry 0), {n} repetitions in {el:.2f} s, fp64"}


def oracle_rate(wl, seconds=10.0, rows=32):
    """Token-heads/s of the fp64 oracle (gate + GLA) on a bounded sample: every
    head of the first `rows` grid rows of batch entry 0, repeated for about
    `seconds`.  The oracle runs one (batch, head) sequence per OpenMP thread,
    so it uses min(H, host cores) threads."""
    import oracle
    cores = os.cpu_count() or 1
    used = min(oracle.set_threads(cores), wl.H)
    d = gin.make_inputs(wl)
    rows = max(1, min(wl.gh, rows))
    T = rows * wl.gw
    x = d["x"][:1, :T]
    q, k, v, z = (d[n][:1, :T] for n in ("q", "k", "v", "z"))
    t0 = time.perf_counter()
    n = 0
    while True:
        g = oracle.gate(x, d["w_down"], d["w_up"], None, tau=wl.tau).reshape(1, T, wl.H, wl.dk)
        oracle.gla_fwd(q, k, v, g, z, d["w"], gh=rows, gw=wl.gw, direction=wl.dirs[0])
        n += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    return {"value": n * T * wl.H / el, "unit": "token-heads/s", "cores": used, "kind": "oracle",
            **host_cpu(),
            "sample": f"gate + GLA of all {wl.H} heads over the first {rows}x{wl.gw}={T} tokens of "
                      f"the {wl.name} workload (batch entry 0), {n} repetitions in {el:.2f} s, fp64"}


def run_reference(args, world, rank):
    wl = gin.WORKLOADS[args.workload]
    if rank != 0:
        return
    import oracle
    oracle.set_threads(1)
    d = gin.make_inputs(wl)
    # bounded per-step sample: one head over 2 grid rows
    rows = 2
    T = rows * wl.gw
    x = d["x"][:1, :T]
    wu = d["w_up"][:, :wl.dk]
    q, k, v, z = (d[n][:1, :T, 0:1] for n in ("q", "k", "v", "z"))

    def step(i):
        g = oracle.gate(x, d["w_down"], wu, None, tau=wl.tau).reshape(1, T, 1, wl.dk)
        oracle.gla_fwd(q, k, v, g, z, d["w"], gh=rows, gw=wl.gw,
                       direction=wl.dirs[i % len(wl.dirs)])

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(i)
    el = time.perf_counter() - t0
    value = args.steps * T / el
    sample = (f"per step: gate + GLA of 1 head over {rows}x{wl.gw}={T} tokens of the {wl.name} "
              "workload (fp64 oracle, 1 thread)")
    line = {
        "impl": "reference", "metric": "GLA fwd token-heads/s (gate projection + Key-only GLA)",
        "value": value, "unit": "token-heads/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * el / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_text(wl), "sample": sample},
        "cpu_baseline": {"value": value, "unit": "token-heads/s", "cores": 1, "kind": "oracle",
                         "sample": sample, **host_cpu()},
        "e2e": {"value": value, "unit": "token-heads/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- GPU arm
def run_ours(args, world, rank, local):
    from linear_vision_backbone_b200 import binding, build
    if not os.path.exists(binding.LIB_PATH):
        build.build()
    binding.load()
    wl = gin.WORKLOADS[args.workload]
    dev = torch.device("cuda", torch.cuda.current_device())
    host = gin.make_inputs(wl)
    esz = host["q"].element_size()
    dirs = step_dirs(wl)
    # N_SETS device copies of the per-step tensors (activations + gate + output)
    sets = []
    for i in range(N_SETS):
        s = {n: host[n].to(dev) for n in ("x", "q", "k", "v", "z")}
        s["g"] = torch.empty(wl.B, wl.T, wl.H, wl.dk, device=dev, dtype=torch.float32)
        s["out"] = torch.empty(wl.B, wl.T, wl.H, wl.dv, device=dev, dtype=host["q"].dtype)
        sets.append(s)
    params = {n: host[n].to(dev) for n in ("w_down", "w_up", "bias", "w")}
    stream = torch.cuda.Stream(device=dev)
    path = binding.path_for(wl.B, wl.H, wl.gh, wl.gw, wl.dk, wl.dv, args.chunk, host["q"].dtype)

    step, fused = make_step(binding, wl, params, host["x"].dtype, args.chunk, stream, args.fused)
    torch.cuda.synchronize()

    # warm the library (workspace allocation happens outside capture)
    with torch.cuda.stream(stream):
        for i in range(N_SETS):
            step(sets[i], dirs[i % len(dirs)])
    stream.synchronize()

    # one plain graph per input set (the timed steps), and one per input set
    # holding kernel-boundary events (the per-kernel durations; torch creates
    # the CUDA event on its first record, so record each once first)
    graphs, igraphs, gevents = [], [], []
    for i in range(N_SETS):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            step(sets[i], dirs[i % len(dirs)])
        graphs.append(g)
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
        for e in evs:
            e.record(stream)
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            step(sets[i], dirs[i % len(dirs)], evs)
        igraphs.append(g)
        gevents.append(evs)
    stream.synchronize()

    for i in range(args.warmup):
        with torch.cuda.stream(stream):
            graphs[i % N_SETS].replay()
            igraphs[i % N_SETS].replay()
    stream.synchronize()

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    t_start = torch.cuda.Event(enable_timing=True)
    t_stop = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        t_start.record(stream)
        for i in range(args.steps):
            graphs[i % N_SETS].replay()
        t_stop.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms = t_start.elapsed_time(t_stop)
    ms_max = max_over_ranks(ms, world)

    # the same K steps with the instrumented graphs: per-kernel durations,
    # averaged over every replay (events are read after each round of the
    # N_SETS graphs, before a replay records them again)
    names = ("gate", "summary", "scan", "output")
    per = {n: 0.0 for n in names}
    barrier(world)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for i0 in range(0, args.steps, N_SETS):
            n_round = min(N_SETS, args.steps - i0)
            for j in range(n_round):
                igraphs[j].replay()
            stream.synchronize()
            for j in range(n_round):
                e = gevents[j]
                for jj, n in enumerate(names):
                    per[n] += event_ms(e[jj], e[jj + 1])
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop()
    per_ms = {n: v / args.steps for n, v in per.items()}

    # segment plan of this workload (for the state bytes)
    nc = (wl.T + args.chunk - 1) // args.chunk
    nseg = binding.segment_count(wl.B, wl.H, wl.gh, wl.gw, wl.dk, wl.dv, args.chunk, host["q"].dtype)
    ab = alg_bytes(wl, esz, fused)
    wsb = workspace_bytes(wl, nseg)
    dom = max(per_ms, key=lambda n: per_ms[n])
    peak, peak_kind = read_peak()
    achieved = ab[dom] / (per_ms[dom] * 1e-3) / 1e9
    kname = {"gate": "gate_low_tc" if fused else "gate_fwd_tc", "summary": "gla_sum_tc",
             "scan": "gla_state_scan", "output": "gla_out_tc"}[dom]
    traffic, _ = read_traffic(f"{kname}:{path}:{wl.name}", kernel_source_hash())

    # e2e: host buffers, copies inside the timed region, through the public API.
    # Two device buffer sets and a copy stream each way: step i's inputs go up
    # while step i-1 computes and step i-2's result comes down.  Each step
    # still waits for its own inputs, and a set is refilled only after the
    # step that read it has run and its result has been copied out.
    pinned = {n: host[n].pin_memory() for n in ("x", "q", "k", "v", "z")}
    out_host = [torch.empty(wl.B, wl.T, wl.H, wl.dv, dtype=host["q"].dtype).pin_memory()
                for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in pinned.values())
    d2h = out_host[0].numel() * out_host[0].element_size()
    s_up, s_down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_up = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_down = [torch.cuda.Event() for _ in range(2)]

    def e2e_step(i):
        j = i & 1
        s = sets[j]
        if i >= 2:
            s_up.wait_event(ev_done[j])       # step i - 2 has read this set's inputs
        with torch.cuda.stream(s_up):
            for n in pinned:
                s[n].copy_(pinned[n], non_blocking=True)
        ev_up[j].record(s_up)
        stream.wait_event(ev_up[j])
        if i >= 2:
            stream.wait_event(ev_down[j])     # step i - 2's result has left this set's output
        with torch.cuda.stream(stream):
            step(s, dirs[i % len(dirs)])
        ev_done[j].record(stream)
        s_down.wait_event(ev_done[j])
        with torch.cuda.stream(s_down):
            out_host[j].copy_(s["out"], non_blocking=True)
        ev_down[j].record(s_down)

    for i in range(3):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_up)
    for i in range(args.e2e_steps):
        e2e_step(i)
    e1.record(s_down)                         # after the last result's copy, which follows all the rest
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)

    units = wl.token_heads
    value = aggregate_value(units, args.steps, ms_max, world)
    e2e_value = aggregate_value(units, args.e2e_steps, e2e_ms, world)

    secondary = None
    others = None
    mixer = None
    ffn = None
    stack = None
    if not args.no_secondary and args.workload == "16k":
        secondary = secondary_line(binding, dev)
        others = configs_lines(binding, dev)
        mixer = mixer_line(binding, dev, wl, host)
        ffn = sswiglu_line(binding, dev, wl)
        stack = stack_line(binding, dev, wl)

    if rank == 0:
        cpu = oracle_rate(wl, seconds=10.0)
        if others is not None:
            for name, c in others.items():
                c["cpu_oracle"] = oracle_rate_config(config_workload(name), seconds=2.0)
        if secondary is not None:
            secondary["cpu_oracle"] = oracle_rate_config(gin.WORKLOADS["640"], seconds=2.0)
        line = {
            "metric": "GLA fwd token-heads/s (gate projection + Key-only GLA)",
            "value": value, "unit": "token-heads/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            # tensor-core path: two-term bf16 operands (hi + lo), fp32 accumulation
            "dtype": "f32" if path == "simt" else "bf16x2/f32",
            "data": "synthetic",
            "config": {"workload": workload_text(wl), "chunk": args.chunk, "kernel_path": path,
                       "step_call": ("gtr_gla_fwd_gated" if fused
                                     else "gtr_gate_fwd_packed + gtr_gla_fwd"),
                       "l2": f"{N_SETS} rotating input sets, inputs larger than L2",
                       "parallelism": f"replicas x{world} (independent (image, head) units)",
                       "timing": "value from plain graph replays; kernels_ms and the roofline "
                                 "from K more replays of graphs with events around each kernel"},
            "roofline": {"bound": "hbm", "kernel": kname, "achieved": achieved, "peak": peak,
                         "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                         "traffic": traffic, "alg_bytes": ab[dom],
                         "workspace_bytes": wsb[dom], "kernel_ms": per_ms[dom]},
            "kernels_ms": per_ms,
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "token-heads/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
                    "copies": "pinned host buffers; two device sets, uploads / compute / downloads "
                              "on three streams (step i's upload overlaps step i-1's compute)"},
            "gpu_launches": 4 * args.steps,
            "clocks": clocks,
        }
        if secondary is not None:
            line["secondary"] = secondary
        if others is not None:
            line["configs"] = others
        if mixer is not None:
            line["mixer"] = mixer
        if ffn is not None:
            line["sswiglu"] = ffn
        if stack is not None:
            line["stack"] = stack
        print(json.dumps(line), flush=True)

    graphs.clear()
    igraphs.clear()
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def make_step(binding, wl, params, x_dtype, chunk, stream, fused=False):
    """One step of the hot path: the gate projection then the GLA forward.
    The weights are static, so for the tensor-core gate shapes they are packed
    once here (outside any timed region) and every step runs
    gtr_gate_fwd_packed and gtr_gla_fwd, or with `fused` one
    gtr_gla_fwd_gated call (the gate's second half inside the summary
    kernel; measured slower on the 16k step); other shapes run gtr_gate_fwd
    and gtr_gla_fwd.  `evs` (5 events): before the gate, after each of the
    four kernels.  Returns (step, fused)."""
    rank = params["w_down"].shape[1]
    hd = wl.H * wl.dk
    packable = (x_dtype in (torch.float16, torch.bfloat16) and rank == 16 and wl.d_model % 64 == 0
                and wl.d_model <= 384 and hd % 64 == 0 and hd <= 448)
    if packable and not fused:
        packed = binding.gate_pack(params["w_down"], params["w_up"], x_dtype, wl.H, wl.dk)

        def step(s, direction, evs=None):
            if evs is not None:
                record_external(evs[0], stream)
            binding.gate_fwd_packed(s["x"], packed, params["bias"], rank, wl.H, wl.dk, wl.tau,
                                    out=s["g"], stream=stream)
            binding.gla_fwd(s["q"], s["k"], s["v"], s["g"], s["z"], params["w"], grid_h=wl.gh,
                            grid_w=wl.gw, direction=direction, chunk=chunk, out=s["out"],
                            stream=stream, events=None if evs is None else evs[1:])
        return step, False
    if packable:
        packed = binding.gate_pack(params["w_down"], params["w_up"], x_dtype, wl.H, wl.dk)

        def step(s, direction, evs=None):
            if evs is not None:
                record_external(evs[0], stream)
            binding.gla_fwd_gated(s["x"], packed, params["bias"], s["q"], s["k"], s["v"], s["z"],
                                  params["w"], tau=wl.tau, grid_h=wl.gh, grid_w=wl.gw,
                                  direction=direction, chunk=chunk, g_out=s["g"], out=s["out"],
                                  stream=stream, events=None if evs is None else [None] + evs[1:])
        return step, True

    def step(s, direction, evs=None):
        if evs is not None:
            record_external(evs[0], stream)
        binding.gate_fwd(s["x"], params["w_down"], params["w_up"], params["bias"], wl.H, wl.dk,
                         wl.tau, out=s["g"], stream=stream)
        binding.gla_fwd(s["q"], s["k"], s["v"], s["g"], s["z"], params["w"], grid_h=wl.gh,
                        grid_w=wl.gw, direction=direction, chunk=chunk, out=s["out"],
                        stream=stream, events=None if evs is None else evs[1:])
    return step, False


def mixer_line(binding, dev, wl, host, steps=200):
    """The token mixer around the timed step (the next row of the hot path):
    the input projection x -> q, k, v, z and the output projection y W_o on the
    library's tcgen05 GEMM (16-bit operands, fp32 accumulation in TMEM, random
    weights of the workload's shapes), each timed alone on graphs, and the whole mixer step (input
    projection, gate, GLA, output projection).  Tensor-bound: FLOP/s against
    the measured bf16 GEMM peak."""
    dt = host["q"].dtype
    H, dk, dm = wl.H, wl.dk, wl.d_model
    gen = torch.Generator().manual_seed(7)
    w_in = (torch.randn(dm, 4 * H * dk, generator=gen) / dm ** 0.5).to(dt).to(dev)
    w_o = (torch.randn(H * dk, dm, generator=gen) / (H * dk) ** 0.5).to(dt).to(dev)
    x = host["x"].to(dev)
    params = {n: host[n].to(dev) for n in ("w_down", "w_up", "bias", "w")}
    stream = torch.cuda.Stream(device=dev)
    step, _ = make_step(binding, wl, params, x.dtype, 64, stream)
    buf = {}

    def in_proj():
        buf["q"], buf["k"], buf["v"], buf["z"] = binding.mixer_in_proj(x, w_in, H, dk, stream=stream)

    def out_proj():
        buf["o"] = binding.mixer_out_proj(buf["y"], w_o, stream=stream)

    def whole():
        in_proj()
        s = {"x": x, "q": buf["q"], "k": buf["k"], "v": buf["v"], "z": buf["z"], "g": buf["g"],
             "out": buf["out"]}
        step(s, wl.dirs[0])
        buf["y"] = buf["out"].reshape(wl.B, wl.T, H * dk)
        out_proj()

    with torch.cuda.stream(stream):
        in_proj()
        buf["g"] = torch.empty(wl.B, wl.T, H, dk, device=dev)
        buf["out"] = torch.empty_like(buf["v"])
        buf["y"] = buf["out"].reshape(wl.B, wl.T, H * dk)
        out_proj()
        whole()
    stream.synchronize()

    def time_graph(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            fn()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            for _ in range(10):
                g.replay()
            a.record(stream)
            for _ in range(steps):
                g.replay()
            b.record(stream)
        stream.synchronize()
        return a.elapsed_time(b) / steps

    ms_in, ms_out, ms_all = time_graph(in_proj), time_graph(out_proj), time_graph(whole)
    n_tok = wl.B * wl.T
    fl_in, fl_out = 2.0 * n_tok * dm * 4 * H * dk, 2.0 * n_tok * H * dk * dm
    try:
        with open(PEAKS_FILE) as f:
            peak = float(json.load(f)["bf16_tflops"])
        kind = "measured"
    except (OSError, KeyError, ValueError):
        peak, kind = 1590.0, "fallback"
    return {"workload": workload_text(wl), "gemm": "gemm_tc_kernel (tcgen05, 128x128 tiles, fp32 accumulation)",
            "in_proj": {"ms": ms_in, "tflops": fl_in / (ms_in * 1e-3) / 1e12,
                        "frac": fl_in / (ms_in * 1e-3) / 1e12 / peak},
            "out_proj": {"ms": ms_out, "tflops": fl_out / (ms_out * 1e-3) / 1e12,
                         "frac": fl_out / (ms_out * 1e-3) / 1e12 / peak},
            "peak_tflops": peak, "peak_kind": kind,
            "mixer_step_ms": ms_all, "mixer_token_heads_per_s": wl.token_heads / (ms_all * 1e-3),
            "l2": "warm (one input set; weights and activations fit L2 at 16k only partly)"}


SSWIGLU_HIDDEN = 1024


def sswiglu_bytes(B, T, C):
    """Algorithmic bytes of one S-SwiGLU mixing launch (16-bit activations):
    u read once (2C channels), h written once (C channels), fp32 taps and bias."""
    return B * T * (2 * C + C) * 2 + (9 * C + C) * 4


def sswiglu_line(binding, dev, wl, steps=200):
    """The Spatial SwiGLU block on the workload's token grid (hidden width 1024,
    random weights): the mixing kernel alone (HBM-bound; two input sets
    alternate, 200 MB together, more than L2) with its achieved GB/s against
    the measured copy bandwidth, and the whole block (the two projections on the
    library's tcgen05 GEMM and the mixing kernel) on warm buffers."""
    B, gh, gw, dm, C = wl.B, wl.gh, wl.gw, wl.d_model, SSWIGLU_HIDDEN
    T = gh * gw
    gen = torch.Generator().manual_seed(23)
    x = torch.randn(B, T, dm, generator=gen).half().to(dev)
    w_in = (torch.randn(dm, 2 * C, generator=gen) / dm ** 0.5).half().to(dev)
    w_out = (torch.randn(C, dm, generator=gen) / C ** 0.5).half().to(dev)
    cw = (torch.randn(3, 3, C, generator=gen) / 3.0).float().to(dev)
    cb = (torch.randn(C, generator=gen) * 0.1).float().to(dev)
    sets = [(torch.randn(B, T, 2 * C, device=dev).half(), torch.empty(B, T, C, device=dev, dtype=torch.half))
            for _ in range(2)]
    stream = torch.cuda.Stream(device=dev)

    def mix():
        for u, h in sets:
            binding.sswiglu_mix(u, cw, cb, grid_h=gh, grid_w=gw, out=h, stream=stream)

    def block():
        binding.sswiglu_fwd(x, w_in, cw, cb, w_out, grid_h=gh, grid_w=gw, scratch=sets[0], stream=stream)

    with torch.cuda.stream(stream):
        mix()
        block()
    stream.synchronize()

    def time_graph(fn, reps):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            fn()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            for _ in range(10):
                g.replay()
            a.record(stream)
            for _ in range(reps):
                g.replay()
            b.record(stream)
        stream.synchronize()
        return a.elapsed_time(b) / reps

    ms_mix = time_graph(mix, steps) / len(sets)
    ms_block = time_graph(block, steps)
    peak, kind = read_peak()
    ab = sswiglu_bytes(B, T, C)
    gbs = ab / (ms_mix * 1e-3) / 1e9
    return {"workload": f"{B}x{gh}x{gw} tokens, d_model {dm}, hidden {C}, 3x3 depthwise, fp16",
            "mix_kernel": "sswiglu_mix_kernel", "mix_ms": ms_mix, "mix_alg_bytes": ab,
            "mix_gbs": gbs, "peak_gbs": peak, "peak_kind": kind, "mix_frac": gbs / peak,
            "block_ms": ms_block, "block_tokens_per_s": B * T / (ms_block * 1e-3),
            "l2": "mix: two alternating input sets (200 MB); block: warm"}


STACK_BLOCKS = 12


def stack_line(binding, dev, wl, reps=50):
    """The 12-block stack on the workload's token grid (random weights:
    d_model 384, six heads of 64, S-SwiGLU hidden width 1024, fp16
    activations, fp32 residual stream), block i scanning LR, RL, TB, BT for
    i mod 4, captured once into one CUDA graph (after an uncaptured call on
    the same stream) and replayed; each replay runs all 12 blocks on the
    residual stream the previous one left.  Reports ms per forward, tokens/s
    and the GEMM FLOP rate over the whole forward."""
    from linear_vision_backbone_b200 import inputs as gin2
    B, gh, gw, H, d, dm, C = wl.B, wl.gh, wl.gw, 6, 64, 384, SSWIGLU_HIDDEN
    x, blocks = gin2.make_stack(STACK_BLOCKS, B, gh, gw, d_model=dm, H=H, dk=d, dv=d, hidden=C,
                                dtype="f16", seed=11)
    stream = torch.cuda.Stream(device=dev)
    w = binding.stack_weights(blocks, torch.float16, H, d, dev, stream=stream)
    ws = torch.empty(binding.stack_workspace_bytes(B, gh, gw, dm, H, d, d, C), device=dev,
                     dtype=torch.uint8)
    xd = x.to(dev)
    kw = dict(grid_h=gh, grid_w=gw, H=H, dk=d, dv=d, dtype=torch.float16, workspace=ws, stream=stream)
    with torch.cuda.stream(stream):
        binding.stack_fwd(xd, w, **kw)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        binding.stack_fwd(xd, w, **kw)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        for _ in range(3):
            g.replay()
        a.record(stream)
        for _ in range(reps):
            g.replay()
        b.record(stream)
    stream.synchronize()
    ms = a.elapsed_time(b) / reps
    del g
    N = B * gh * gw
    flops = STACK_BLOCKS * 2.0 * N * (dm * 4 * H * d + H * d * dm + dm * 2 * C + C * dm)
    # per block: in-projection, gate, the GLA's three kernels, out-projection,
    # add + norm, expansion, mixing, projection, add + norm; one norm first
    per_block = 11
    return {"workload": f"{STACK_BLOCKS} GTR blocks, {B}x{gh}x{gw} tokens, d_model {dm}, H {H}, d {d}, "
                        f"S-SwiGLU hidden {C}, fp16 activations, fp32 residual",
            "ms": ms, "tokens_per_s": N / (ms * 1e-3), "gemm_tflops": flops / (ms * 1e-3) / 1e12,
            "kernels_per_forward": 1 + STACK_BLOCKS * per_block,
            "graph": "one CUDA graph per forward, replayed",
            "l2": "warm (16-bit weights 46 MB, activations of one block about 200 MB)"}


def step_alg_bytes(wl):
    """Algorithmic bytes of one whole step (gate projection when the workload
    has one, then the GLA): per token-head q, k, v, z, out in the storage
    dtype and g in fp32, plus, with the gate, x once (d_model values per token)
    and the g write."""
    esz = inputs_esz(wl)
    th = wl.token_heads
    gla = th * ((2 * wl.dk + 3 * wl.dv) * esz + wl.dk * 4)
    if wl.recipe != "proj":
        return gla
    return gla + wl.B * wl.T * wl.d_model * esz + th * wl.dk * 4


def inputs_esz(wl):
    return {"f32": 4, "f16": 2, "bf16": 2}[wl.dtype]


def config_line(binding, dev, wl, steps=200, nsets=8):
    """One workload timed as the headline step is: a CUDA graph per input set
    (gate projection + GLA for the projected workloads, GLA alone for the ones
    whose gates are drawn directly), a 256 MiB buffer written between steps
    (outside the timed events) so that every step starts with a cold L2, and
    the step's algorithmic bytes over its time against the measured copy
    bandwidth."""
    host = gin.make_inputs(wl)
    nsets = max(1, min(nsets, (1 << 30) // max(1, sum(t.numel() * t.element_size()
                                                       for t in host.values()))))
    sets = []
    for i in range(nsets):
        s = {n: host[n].to(dev) for n in host if n not in ("w_down", "w_up", "bias", "w")}
        if "g" not in s:
            s["g"] = torch.empty(wl.B, wl.T, wl.H, wl.dk, device=dev)
        s["out"] = torch.empty_like(s["v"])
        sets.append(s)
    stream = torch.cuda.Stream(device=dev)
    if wl.recipe == "proj":
        params = {n: host[n].to(dev) for n in ("w_down", "w_up", "bias", "w")}
        step, _ = make_step(binding, wl, params, host["x"].dtype, wl.chunk, stream)
    else:
        w = host["w"].to(dev)

        def step(s, direction, evs=None):
            binding.gla_fwd(s["q"], s["k"], s["v"], s["g"], s["z"], w, grid_h=wl.gh, grid_w=wl.gw,
                            direction=direction, chunk=wl.chunk, out=s["out"], stream=stream)
    torch.cuda.synchronize()
    dirs = list(wl.dirs)
    with torch.cuda.stream(stream):
        for i, s in enumerate(sets):
            step(s, dirs[i % len(dirs)])
    stream.synchronize()
    graphs = []
    for i, s in enumerate(sets):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            step(s, dirs[i % len(dirs)])
        graphs.append(g)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    with torch.cuda.stream(stream):
        for i in range(min(20, steps)):
            graphs[i % nsets].replay()
        for i in range(steps):
            flush.fill_(i & 255)
            ev[i][0].record(stream)
            graphs[i % nsets].replay()
            ev[i][1].record(stream)
    stream.synchronize()
    ms = sum(a.elapsed_time(b) for a, b in ev) / steps
    peak, kind = read_peak()
    ab = step_alg_bytes(wl)
    gbs = ab / (ms * 1e-3) / 1e9
    return {"workload": workload_text(wl), "value": wl.token_heads / (ms * 1e-3),
            "unit": "token-heads/s", "ms_per_step": ms, "steps": steps,
            "kernel_path": binding.path_for(wl.B, wl.H, wl.gh, wl.gw, wl.dk, wl.dv, wl.chunk,
                                            host["q"].dtype),
            "step_alg_bytes": ab, "achieved_gbs": gbs, "peak_gbs": peak, "peak_kind": kind,
            "frac": gbs / peak, "l2": "256 MiB buffer written between steps, outside the timed events"}


def secondary_line(binding, dev, steps=2000):
    """The same step on the 640x640 workload (T = 1600), timed the same way."""
    return config_line(binding, dev, gin.WORKLOADS["640"], steps=steps)


def config_workload(name):
    """The workload of a name in the configs entry: a workload's own name, or
    sweep-<grid> for the sweep at that square grid."""
    if name.startswith("sweep-"):
        return gin.WORKLOADS["sweep"].with_grid(int(name.split("-")[1]))
    return gin.WORKLOADS[name]


def configs_lines(binding, dev):
    """Every other workload: the batched 640x640 case and the d = 128 sweep."""
    out = {n: config_line(binding, dev, config_workload(n), steps=500) for n in ("640b8", "tiny")}
    for gsz in gin.SWEEP_GRIDS:
        name = f"sweep-{gsz}"
        out[name] = config_line(binding, dev, config_workload(name), steps=100 if gsz >= 128 else 300)
    return out


def main():
    args = parse()
    world, rank, local = dist_setup(args) if args.impl == "ours" else (
        int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
        int(os.environ.get("LOCAL_RANK", "0")))
    if args.impl == "reference":
        run_reference(args, world, rank)
        return
    run_ours(args, world, rank, local)


if __name__ == "__main__":
    main()
