"""Benchmark of the MoE expert-parallel load-balancing decision path on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config NAME]

A step is one pass of the whole decision path (lookahead gate + top-k,
per-rank counts, replica plan, normal gate + top-k, counts, Relief split,
destinations + stable permutation) over every layer of the workload's model,
all layers batched into one launch per kernel, replayed from a CUDA graph.
Inputs (hidden states, gate weights, biases) are resident in HBM before the
timed region; the per-step hidden-state stream (25.5 GB for the default
Qwen3-235B-shaped workload, 94 layers) is far larger than the 126 MB L2, so
no L2 flush is needed.

One JSON line is printed by rank 0.  `value` is whole-job routed
token-assignments per second (all ranks; each rank runs its own independent
copy of the workload: weak scaling, no collective on the data path).

`--impl reference` times the CPU oracle (the only reference implementation
this method has) on the host cores, on a bounded sample of the same workload.
"""
import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "routed token-assignments/s and per-layer T_solve (µs); % of HBM roofline"
UNIT = "token-assignments/s"
DEFAULT_WORKLOAD = "qwen3-235b"


def peaks():
    """(HBM GB/s, bf16 TFLOP/s burst, bf16 TFLOP/s sustained, kind): the
    pool's measured copy bandwidth and cuBLAS throughput, else the fallback
    figures measured earlier on this machine."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        burst = float(d["bf16_tflops"])
        return float(d["hbm_gbs"]), burst, float(d.get("bf16_tflops_sustained", burst)), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


GATE_SOURCES = ["moe_expert_load_bf16_b200/csrc/gate_topk.cuh", "moe_expert_load_bf16_b200/csrc/common.cuh"]


def source_sha(source_files):
    import hashlib
    h = hashlib.sha256()
    for f in source_files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profile_traffic(kernel_tag, source_files, units=None):
    """DRAM bytes of one launch from a committed ncu summary, if the
    kernel's source has not changed since the capture (else None).  A
    summary gives either `traffic_bytes_per_launch` (a capture of the same
    launch) or `traffic_bytes_per_unit` (a capture of a smaller launch of
    the same kernel, scaled here by the `units` this launch processes)."""
    path = os.path.join(ROOT, "profiles", f"{kernel_tag}.md")
    if not os.path.exists(path):
        return None
    got, per_launch, per_unit = None, None, None
    for line in open(path):
        if line.startswith("source_sha:"):
            got = line.split(":", 1)[1].strip()
        if line.startswith("traffic_bytes_per_launch:"):
            per_launch = float(line.split(":", 1)[1].strip())
        if line.startswith("traffic_bytes_per_unit:"):
            per_unit = float(line.split(":", 1)[1].strip())
    if got != source_sha(source_files):
        return None
    if per_unit is not None and units is not None:
        return per_unit * units
    return per_launch


class ClockSampler:
    """Samples SM clock and throttle reasons with NVML in a background thread."""

    def __init__(self, index, period=0.001):
        self.index, self.period = index, period
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._t = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nvml = None
            return self
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        return self

    def _run(self):
        nv = self._nvml
        names = {
            getattr(nv, "nvmlClocksEventReasonHwSlowdown", 0x8): "hw_slowdown",
            getattr(nv, "nvmlClocksEventReasonHwThermalSlowdown", 0x40): "hw_thermal_slowdown",
            getattr(nv, "nvmlClocksEventReasonSwThermalSlowdown", 0x20): "sw_thermal_slowdown",
            getattr(nv, "nvmlClocksEventReasonSwPowerCap", 0x4): "sw_power_cap",
            getattr(nv, "nvmlClocksEventReasonHwPowerBrakeSlowdown", 0x80): "hw_power_brake_slowdown",
        }
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in names.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __exit__(self, *exc):
        self._stop.set()
        if self._t is not None:
            self._t.join()
        return False

    def summary(self):
        return {"sm_mhz": int(statistics.median(self.samples)) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": len(self.samples)}


def dist_setup(backend=None):
    """One process per GPU (torchrun env); NCCL on GPUs, gloo on CPU-only hosts."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and not torch.distributed.is_initialized():
        import datetime
        backend = backend or ("nccl" if torch.cuda.is_available() else "gloo")
        if backend == "nccl":
            torch.cuda.set_device(local)
            torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                                 device_id=torch.device("cuda", local))
        else:
            torch.distributed.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def settle(seconds=0.5):
    """Let the GPU idle before a latency measurement: after the power-capped
    step loop the SM clock takes a while to climb back, and a kernel of a
    few microseconds timed at once would be timed at the low clock."""
    torch.cuda.synchronize()
    time.sleep(seconds)


def graph_us(fn, reps, world=1, rounds=2, inner=10):
    """Microseconds per call of fn: `inner` calls captured in one CUDA graph
    (so the host's launch rate never paces calls of a few microseconds),
    about reps calls per round between CUDA events on the launching stream;
    the faster of `rounds` rounds (a first round can run at a clock still
    recovering from the power-capped work before it), max over ranks."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(inner):
            fn()
    g.replay()
    torch.cuda.synchronize()
    replays = max(1, (reps + inner - 1) // inner)
    best = None
    for _ in range(rounds):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        a.record()
        for _ in range(replays):
            g.replay()
        b.record()
        torch.cuda.synchronize()
        t = a.elapsed_time(b) * 1e3 / (replays * inner)
        best = t if best is None else min(best, t)
    return max_over_ranks(best, world)


def max_over_ranks(x, world):
    """The slowest rank's time (whole-job timing is the max over ranks)."""
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def rank_workload(wl, rank):
    """Each rank decides its own independent problems (weak scaling): same
    shapes, seeds offset by rank."""
    return wl if rank == 0 else wl.with_(seed=wl.seed + 1000 * rank)


def whole_job_rate(units_per_step_per_rank, world, ms_per_step):
    return units_per_step_per_rank * world / (ms_per_step * 1e-3)


# ----------------------------------------------------------------------------- GPU arm
def run_ours(args, world, rank, local):
    from moe_expert_load_bf16_b200 import _lib, build, workloads
    from moe_expert_load_bf16_b200.pipeline import DecisionPath, StepPipeline

    build.build()
    wl = rank_workload(workloads.WORKLOADS[args.config], rank)
    Lyr, T, H, E, k, G, N, L = wl.layers, wl.T, wl.H, wl.E, wl.k, wl.G, wl.N, wl.L
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()

    # hidden slot 0 = h_0 again: the lookahead input of layer 0
    hid = torch.empty(Lyr + 1, T, H, dtype=torch.bfloat16, device=dev)
    workloads.hidden_chain(wl, Lyr, T=T, out=hid[1:])
    hid[0].copy_(hid[1])
    W = workloads.gate_weights(wl, Lyr, device=dev)
    bias = workloads.biases(wl, Lyr).to(dev)
    chain = args.gate == "chain"
    pipe = StepPipeline(Lyr, T, H, E, k, G, N, L, device=dev) if chain and args.in_flight == 2 else None
    path = pipe.paths[0] if pipe else DecisionPath(Lyr, T, H, E, k, G, N, L, device=dev)
    side = torch.cuda.Stream(device=dev)

    def step():
        if chain:
            path.run_chain(hid, W, bias)
        else:
            path.run(hid[:-1], hid[1:], W, bias, side_stream=side)
    launches = path.LAUNCHES_PER_CHAIN if chain else path.LAUNCHES_PER_RUN

    # warm-up (also loads the library, sets kernel attributes, builds maps)
    if pipe:
        pipe.run(args.warmup, hid, W, bias)
    else:
        for _ in range(args.warmup):
            step()
    torch.cuda.synchronize()
    if _lib.lb_get_status():
        raise RuntimeError("device status flagged during warm-up")

    # one step alone (its latency), and the K timed steps: one step per
    # graph replay, or with two steps in flight the K steps as one graph
    g_step = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step):
        step()
    g_step.replay()
    if pipe:
        g_steps = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_steps):
            pipe.run(args.steps, hid, W, bias)
        g_steps.replay()
    torch.cuda.synchronize()

    # ---------------- timed region: K steps
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier(world)
        torch.cuda.synchronize()
        ev0.record(stream)
        if pipe:
            g_steps.replay()
        else:
            for _ in range(args.steps):
                g_step.replay()
        ev1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
    ms_total = max_over_ranks(ev0.elapsed_time(ev1), world)
    ms_step = ms_total / args.steps
    if pipe:
        del g_steps
    assign_per_step = Lyr * T * k
    value = whole_job_rate(assign_per_step, world, ms_step)
    if args.lean:
        return {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_step, "lean": True,
                "gpu_launches": launches * args.steps, "clocks": clk.summary()}

    # ---------------- one step alone: its latency (graph replays, one at a time)
    barrier(world)
    ev0.record(stream)
    for _ in range(args.steps):
        g_step.replay()
    ev1.record(stream)
    torch.cuda.synchronize()
    step_latency_us = max_over_ranks(ev0.elapsed_time(ev1), world) / args.steps * 1e3

    # ---------------- dominant kernel: the gate (one chain launch per step,
    # or two launches in the two-pass form)
    g_gate = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_gate):
        if chain:
            _lib.lb_predict_topk_chain(hid, W, bias, k, ids_pred=path.ids_pred, ids_act=path.ids)
        else:
            _lib.lb_predict_topk(hid[:-1], W, bias, k, ids=path.ids_pred)
            _lib.lb_predict_topk(hid[1:], W, bias, k, ids=path.ids)
    g_gate.replay()
    torch.cuda.synchronize()
    barrier(world)
    ev0.record(stream)
    for _ in range(args.steps):
        g_gate.replay()
    ev1.record(stream)
    torch.cuda.synchronize()
    if chain:
        gate_ms = ev0.elapsed_time(ev1) / args.steps
        gate_bytes = (Lyr + 1) * 2 * T * H + Lyr * (2 * H * E + 4 * E + 2 * 4 * T * k)
        gate_flops = Lyr * 2 * 2.0 * T * H * E
        gate_units = Lyr + 1          # hidden states streamed by one launch
        tag = f"gate_chain_{wl.name}"
    else:
        gate_ms = ev0.elapsed_time(ev1) / (2 * args.steps)
        gate_bytes = Lyr * (2 * T * H + 2 * H * E + 4 * E + 4 * T * k)
        gate_flops = Lyr * 2.0 * T * H * E
        gate_units = Lyr
        tag = f"gate_topk_{wl.name}"
    gate_ms = max_over_ranks(gate_ms, world)
    hbm, tflops, tflops_sus, peak_kind = peaks()
    roofline = gate_roofline(gate_bytes, gate_flops, gate_ms, hbm, tflops, tflops_sus, peak_kind,
                             profile_traffic(tag, GATE_SOURCES, units=gate_units))
    roofline["kernel"] = "gate_topk_persistent (chain)" if chain else "gate_topk"

    # ---------------- per-layer latencies (single problem, graph replays),
    # this workload's and every other configuration's
    settle()
    lat = per_layer_latency(wl, hid, W, bias, dev, reps=max(50, args.steps))
    per_config = per_config_latency(dev, world, wl, lat, reps=max(50, args.steps),
                                    decode_steps=args.decode_steps)
    settle()
    gate_shapes = gate_fractions(dev, world)
    settle()

    # ---------------- count / split / assign as throughput kernels
    ints = integer_kernels_at_throughput(dev, world)
    swp = swap_planner(wl, path, world)

    # ---------------- end to end through the C ABI with host buffers
    e2e = end_to_end(args, wl, hid, W, bias, path, dev, world, chain)

    torch.cuda.synchronize()
    flags = _lib.lb_get_status()
    if flags:
        raise RuntimeError(f"device status flagged: {flags}")

    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{wl.name}: {Lyr} layers x T={T} tokens, H={H}, E={E}, top-{k}, "
                               f"G={G} ranks, N={N} replica slots (L={L})",
                   "layers": Lyr, "T": T, "H": H, "E": E, "k": k, "G": G, "N": N, "L": L, "passes": 12,
                   "batching": "all layers of a step in one launch per kernel, CUDA-graph replay",
                   "steps_in_flight": (2 if pipe else 1),
                   "overlap": ("two steps in flight: gate and count of each step on one stream, plan, split "
                               "and assign on a second, higher-priority stream, so the gate of step i+1 runs "
                               "beside the plan, split and assign of step i (two buffer sets); the K timed "
                               "steps are one CUDA graph"
                               if pipe else "none: one step after another"),
                   "gate": ("chain: one pass per hidden state evaluates the normal router of the layer before "
                            "it and the lookahead of the layer after it" if chain else
                            "two passes (lookahead, normal router); lookahead counts + plan on a second stream"),
                   "l2": "inputs larger than L2 (hidden states %.0f MB read per step)" % (
                       (Lyr + 1 if chain else 2 * Lyr) * T * H * 2 / 1e6),
                   "parallelism": f"{world} independent replicas"},
        "step_latency_us": step_latency_us,
        "t_solve_us": max_over_ranks(lat["solve"], world), "t_solve_fused_us": lat["solve_fused"],
        "t_split_us": max_over_ranks(lat["split"], world), "t_lookahead_us": lat["lookahead"],
        "per_kernel_us": lat["kernels"],
        "roofline": roofline,
        "per_config": per_config,
        "gate_shapes": gate_shapes,
        "integer_kernels": ints,
        "swap_planner": swp,
        "e2e": e2e,
        "gpu_launches": launches * args.steps,
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(wl, budget_s=args.cpu_budget)
    return out


def gate_roofline(nbytes, flops, ms, hbm, tflops, tflops_sus, peak_kind, traffic):
    """Roofline of one gate launch: its algorithmic bytes and flops against
    the measured HBM copy and bf16 tensor peaks.  The bound is the larger of
    the two minimum times (bytes / HBM peak, flops / tensor peak; burst
    figures, the launch being timed alone); both fractions are reported,
    and the tensor fraction against the sustained (power-capped) peak too."""
    s = ms * 1e-3
    t_hbm, t_tensor = nbytes / (hbm * 1e9), flops / (tflops * 1e12)
    out = {"bound": "tensor" if t_tensor > t_hbm else "hbm"}
    if t_tensor > t_hbm:
        out.update(achieved=flops / s / 1e12, peak=tflops, unit="TFLOP/s")
    else:
        out.update(achieved=nbytes / s / 1e9, peak=hbm, unit="GB/s")
    out.update(frac=max(t_hbm, t_tensor) / s, traffic=traffic, peak_kind=peak_kind,
               algorithmic_bytes_per_launch=nbytes, algorithmic_flops_per_launch=flops, launch_us=ms * 1e3,
               hbm_gbs=nbytes / s / 1e9, hbm_frac=t_hbm / s, tensor_tflops=flops / s / 1e12,
               tensor_frac=t_tensor / s, tensor_frac_of_sustained=flops / (tflops_sus * 1e12) / s,
               sustained_tflops=tflops_sus,
               traffic_over_algorithmic=(traffic / nbytes if traffic else None))
    return out


def gate_fractions(dev, world, reps=20):
    """The gate on every configuration's shape, against its roofline
    (max(bytes / HBM peak, flops / tensor peak) / time, burst peaks): the
    chain gate over 16 layers of each prefill configuration, and the
    per-layer gate of the decode shape (H=7168, E=256) at every T."""
    from moe_expert_load_bf16_b200 import _lib, workloads
    hbm, tflops, _, peak_kind = peaks()

    def timed(fn):
        return graph_us(fn, reps, world)

    def frac(nbytes, flops, us):
        return {"us": us, "hbm_frac": nbytes / us / 1e3 / hbm, "tensor_frac": flops / us / 1e6 / tflops,
                "roofline_frac": max(nbytes / (hbm * 1e3), flops / (tflops * 1e6)) / us}

    out = {"peak_kind": peak_kind}
    for name in ("olmoe", "qwen3-30b", "qwen3-235b"):
        wl = workloads.WORKLOADS[name]
        nl = min(16, wl.layers)
        hid = torch.empty(nl + 1, wl.T, wl.H, dtype=torch.bfloat16, device=dev)
        workloads.hidden_chain(wl, nl, out=hid[1:])
        hid[0].copy_(hid[1])
        W = workloads.gate_weights(wl, nl, device=dev)
        bias = workloads.biases(wl, nl).to(dev)
        ip = torch.empty(nl, wl.T, wl.k, dtype=torch.int32, device=dev)
        ia = torch.empty_like(ip)
        us = timed(lambda: _lib.lb_predict_topk_chain(hid, W, bias, wl.k, ids_pred=ip, ids_act=ia))
        nbytes = (nl + 1) * 2 * wl.T * wl.H + nl * (2 * wl.H * wl.E + 4 * wl.E + 8 * wl.T * wl.k)
        out[f"chain_{name}"] = dict(frac(nbytes, nl * 4.0 * wl.T * wl.H * wl.E, us), layers=nl)
        del hid, W, bias, ip, ia
    wl = workloads.WORKLOADS["decode"]
    W = workloads.gate_weights(wl, 1, device=dev)[0]
    bias = workloads.biases(wl, 1)[0].to(dev)
    settle()
    for T in wl.decode_T:
        h = workloads.hidden_chain(wl, 1, device=dev, T=T)[0]
        ids = torch.empty(T, wl.k, dtype=torch.int32, device=dev)
        us = timed(lambda: _lib.lb_predict_topk(h, W, bias, wl.k, ids=ids))
        nbytes = 2 * T * wl.H + 2 * wl.H * wl.E + 4 * wl.E + 4 * T * wl.k
        out[f"decode_T{T}"] = frac(nbytes, 2.0 * T * wl.H * wl.E, us)
        del h, ids
    torch.cuda.empty_cache()
    return out


def per_config_latency(dev, world, main_wl, main_lat, reps, decode_steps=1000):
    """T_solve, T_split and T_lookahead of one layer of every prefill
    configuration (the gate applied to that configuration's synthetic hidden
    states gives the ids), and the decode sweep per step."""
    from moe_expert_load_bf16_b200 import workloads
    out = {}
    for name in ("olmoe", "qwen3-30b", "qwen3-235b"):
        wl = workloads.WORKLOADS[name]
        if name == main_wl.name:
            lat = main_lat
        else:
            hid = workloads.hidden_chain(wl, 2, device=dev)
            W = workloads.gate_weights(wl, 1, device=dev)
            bias = workloads.biases(wl, 1).to(dev)
            settle()
            lat = per_layer_latency(wl, hid, W, bias, dev, reps)
            del hid, W, bias
        out[name] = {"shape": f"T={wl.T}, H={wl.H}, E={wl.E}, top-{wl.k}, G={wl.G}, N={wl.N} (L={wl.L})",
                     "t_solve_us": max_over_ranks(lat["solve"], world),
                     "t_solve_separate_us": lat["solve_separate"], "t_solve_fused_us": lat["solve_fused"],
                     "t_split_us": max_over_ranks(lat["split"], world),
                     "t_lookahead_us": max_over_ranks(lat["lookahead"], world),
                     "per_kernel_us": lat["kernels"]}
    torch.cuda.empty_cache()
    out["decode"] = decode_per_step(dev, world, decode_steps)
    return out


def decode_per_step(dev, world, nsteps=1000, chunk=100):
    """Decode-step sweep: E=256, top-8, G=64 ranks x 4 experts, N=2, T per
    step in {64, 256, 1024, 4096, 8192}.  `nsteps` consecutive steps with
    their own synthetic ids (per-step Zipf bias re-drawn with correlation
    0.5, so the counts shift every step); the plan is made once from step
    0's counts.  Every step's count + split + assign (lb_count + lb_decide)
    runs on its own ids, one step after another (graphs of `chunk` steps);
    T_solve and T_split are the mean per step.  The same steps as one
    batched launch give the throughput form."""
    from moe_expert_load_bf16_b200 import _lib, workloads
    from moe_expert_load_bf16_b200.pipeline import DecisionPath
    wl = workloads.WORKLOADS["decode"]
    G, E, N, L, k = wl.G, wl.E, wl.N, wl.L, wl.k
    res = {"shape": f"E={E}, top-{k}, G={G} ranks x {E // G} experts, N={N} (L={L}); plan from step 0",
           "steps": nsteps}

    def graphs_of(fns):
        gs = []
        for c0 in range(0, len(fns), chunk):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for f in fns[c0:c0 + chunk]:
                    f()
            gs.append(g)
        return gs

    def run_timed(gs, reps=1):
        for g in gs:
            g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        a.record()
        for _ in range(reps):
            for g in gs:
                g.replay()
        b.record()
        torch.cuda.synchronize()
        return max_over_ranks(a.elapsed_time(b) * 1e3 / reps, world)

    for T in wl.decode_T:
        path = DecisionPath(nsteps, T, wl.H, E, k, G, N, L, device=dev)
        for c0 in range(0, nsteps, 100):
            path.ids[c0:c0 + 100].copy_(workloads.decode_ids(wl.with_(T=T), T, range(c0, min(nsteps, c0 + 100)),
                                                             device=dev))
        _lib.lb_count(path.ids[0:1], G, E, cnt=path.cnt_pred[0:1])
        _lib.lb_plan_replicas(path.cnt_pred[0:1], N, L, plan=path.plan[0:1])
        path.plan[1:].copy_(path.plan[0:1].expand(nsteps - 1, -1))
        solve = graphs_of([(lambda b=b: path.solve_one(b)) for b in range(nsteps)])
        split = graphs_of([(lambda b=b: path.solve_one(b, split_only=True)) for b in range(nsteps)])
        t_solve = run_timed(solve) / nsteps
        t_split = run_timed(split) / nsteps
        gb = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gb):
            path.solve()
        t_batch = run_timed([gb], reps=5)
        if _lib.lb_get_status():
            raise RuntimeError("device status flagged in the decode sweep")
        res[str(T)] = {"t_solve_us": t_solve, "t_split_us": t_split,
                       "assignments_per_s_step_by_step": T * k / (t_solve * 1e-6),
                       "batched_us": t_batch, "assignments_per_s_batched": nsteps * T * k / (t_batch * 1e-6)}
        del solve, split, gb, path
        torch.cuda.empty_cache()
    return res


def per_layer_latency(wl, hid, W, bias, dev, reps):
    """Median-free mean latency per layer (one problem, CUDA-graph replays) of
    T_solve = count + split + assign on actual ids, T_split, T_lookahead =
    2 gate + count + plan, and each kernel group alone."""
    from moe_expert_load_bf16_b200 import _lib
    from moe_expert_load_bf16_b200.pipeline import DecisionPath
    T, H, E, k, G, N, L = wl.T, wl.H, wl.E, wl.k, wl.G, wl.N, wl.L
    p1 = DecisionPath(1, T, H, E, k, G, N, L, device=dev)
    p1.run(hid[0:1], hid[1:2], W[0:1], bias[0:1])
    torch.cuda.synchronize()

    def timed(fn):
        return graph_us(fn, reps)

    res = {
        "solve": timed(p1.solve),
        "solve_separate": timed(p1.solve_separate),
        "solve_fused": timed(p1.solve_fused),
        "split": timed(lambda: _lib.lb_split(p1.cnt, p1.plan, N, 12,
                                             out=(p1.tok, p1.mass, p1.loads, p1.passes_run))),
        "lookahead": timed(lambda: (p1.lookahead(hid[0:1], W[0:1], bias[0:1]), p1.route(hid[1:2], W[0:1],
                                                                                        bias[0:1]))),
    }
    res["kernels"] = {
        "gate": timed(lambda: _lib.lb_predict_topk(hid[1:2], W[0:1], bias[0:1], k, ids=p1.ids)),
        "count": timed(lambda: _lib.lb_count(p1.ids, G, E, cnt=p1.cnt)),
        "plan": timed(lambda: _lib.lb_plan_replicas(p1.cnt_pred, N, L, plan=p1.plan)),
        "split": res["split"],
        "assign": timed(lambda: _lib.lb_assign(p1.ids, p1.cnt, p1.plan, p1.tok, p1.mass, N,
                                               out=(p1.dest, p1.perm, p1.offs), workspace=p1.ws)),
    }
    return res


def swap_planner(wl, path, world, reps=50):
    """FreeBalance's budgeted pairwise-swap planner (lb_plan_swaps) as the
    alternative to replication, on the step's predicted counts of every
    layer: latency (one layer; all layers in one launch) and the max-to-mean
    rank load before and after the swaps, on the predicted counts and on the
    actual counts under the new placement.  Cost model (illustrative, stated):
    alpha = 10 us per swap, beta = 770 GB/s (this machine's measured peer copy),
    S = one expert's three bf16 matrices (3*H*I, I = 1024 for the OLMoE
    shape), budget 200 us per rank and per link; gamma = 1 / (T*k)."""
    from moe_expert_load_bf16_b200 import _lib
    G, E = wl.G, wl.E
    prm = dict(gamma=1.0 / (wl.T * wl.k), tau=0.0, alpha=10.0, beta=770e3, expert_bytes=3.0 * wl.H * 1024 * 2,
               budget=200.0)
    cp = path.cnt_pred.contiguous()
    out = _lib.lb_plan_swaps(cp, **prm)
    one = _lib.lb_plan_swaps(cp[0:1], **prm)
    torch.cuda.synchronize()

    def timed(fn):
        return graph_us(fn, reps, world)

    t_all = timed(lambda: _lib.lb_plan_swaps(cp, out=out, **prm))
    t_one = timed(lambda: _lib.lb_plan_swaps(cp[0:1], out=one, **prm))
    # quality (reporting only): rank loads under the even and the new placement
    even = (torch.arange(E, device=cp.device) // (E // G)).long()
    pi = out[0].long()

    def max_to_mean(n_e, placement):
        loads = torch.zeros(n_e.shape[0], G, dtype=torch.float64, device=n_e.device)
        loads.scatter_add_(1, placement.expand(n_e.shape[0], -1) if placement.dim() == 1 else placement,
                           n_e.double())
        return (loads.max(dim=1).values / loads.mean(dim=1)).mean().item()

    n_pred = path.cnt_pred.sum(dim=1)
    n_act = path.cnt.sum(dim=1)
    return {"t_one_layer_us": t_one, "t_all_layers_us": t_all, "layers": int(cp.shape[0]),
            "swaps_per_layer": out[2].double().mean().item(),
            "max_to_mean_predicted": {"even": max_to_mean(n_pred, even), "swapped": max_to_mean(n_pred, pi)},
            "max_to_mean_actual": {"even": max_to_mean(n_act, even), "swapped": max_to_mean(n_act, pi)},
            "params": prm}


def integer_kernels_at_throughput(dev, world, nbatch=128, reps=20):
    """Count, split and assign (prep + scatter) as throughput kernels: one
    launch over `nbatch` independent Qwen3-235B-shaped problems (T=32768,
    top-8, E=128, G=8, N=4), ids larger than L2 in total.  Each kernel group
    is graph-replayed alone; achieved = algorithmic bytes / mean time."""
    from moe_expert_load_bf16_b200 import _lib, workloads
    from moe_expert_load_bf16_b200.pipeline import DecisionPath
    wl = workloads.WORKLOADS["qwen3-235b"]
    T, E, k, G, N, L = wl.T, wl.E, wl.k, wl.G, wl.N, wl.L
    ids = torch.empty(nbatch, T, k, dtype=torch.int32, device=dev)
    for c0 in range(0, nbatch, 16):
        ids[c0:c0 + 16].copy_(workloads.decode_ids(wl, T, range(c0, min(nbatch, c0 + 16)), device=dev))
    path = DecisionPath(nbatch, T, 8, E, k, G, N, L, device=dev)
    path.ids.copy_(ids)
    del ids
    _lib.lb_count(path.ids, G, E, cnt=path.cnt)
    _lib.lb_plan_replicas(path.cnt, N, L, plan=path.plan)   # any valid plan serves the throughput run
    path.solve()
    torch.cuda.synchronize()

    def timed(fn):
        return graph_us(fn, reps, world)

    n_edges = sum(int(d["n_edges"]) for d in _lib.decode_plan(path.plan, G, E, N)) / nbatch
    t_count = timed(lambda: _lib.lb_count(path.ids, G, E, cnt=path.cnt))
    t_split = timed(lambda: _lib.lb_split(path.cnt, path.plan, N, 12,
                                          out=(path.tok, path.mass, path.loads, path.passes_run)))
    t_assign = timed(lambda: _lib.lb_assign(path.ids, path.cnt, path.plan, path.tok, path.mass, N,
                                            out=(path.dest, path.perm, path.offs), workspace=path.ws))
    if _lib.lb_get_status():
        raise RuntimeError("device status flagged in the integer-kernel run")
    hbm = peaks()[0]
    tk = T * k
    by = {"count": nbatch * (4 * tk + 4 * G * E),
          "split": int(nbatch * (4 * G * E + 12 * n_edges + 16 * G * N + 4 * G)),
          "assign": nbatch * (3 * 4 * tk + 4 * (G * E + 1) + 4 * G * E + 8 * G * N)}
    out = {"workload": f"{nbatch} problems x (T={T}, top-{k}, E={E}, G={G}, N={N}) per launch; ids "
                       f"{nbatch * tk * 4 / 1e6:.0f} MB",
           "peak_gbs": hbm}
    for name, t in (("count", t_count), ("split", t_split), ("assign", t_assign)):
        gbs = by[name] / (t * 1e-6) / 1e9
        out[name] = {"us": t, "algorithmic_bytes": by[name], "gbs": gbs, "frac": gbs / hbm,
                     "assignments_per_s": nbatch * tk / (t * 1e-6)}
    del path
    torch.cuda.empty_cache()
    return out


def end_to_end(args, wl, hid, W, bias, path, dev, world, chain=True):
    """Same metric through the public API with host buffers: every step
    copies its inputs from pinned host memory and reads its results back."""
    Lyr, T, k = wl.layers, wl.T, wl.k

    def pinned_copy(t):
        # allocated pinned directly (no pageable staging copy of a 25 GB input)
        hst = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
        hst.copy_(t)
        return hst
    h_host = pinned_copy(hid)
    w_host = pinned_copy(W)
    b_host = pinned_copy(bias)
    outs = (path.dest, path.perm, path.offs, path.loads)
    o_host = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs]
    h2d = h_host.numel() * 2 + w_host.numel() * 2 + b_host.numel() * 4
    d2h = sum(o.numel() * o.element_size() for o in o_host)

    def step():
        hid.copy_(h_host, non_blocking=True)
        W.copy_(w_host, non_blocking=True)
        bias.copy_(b_host, non_blocking=True)
        if chain:
            path.run_chain(hid, W, bias)
        else:
            path.run(hid[:-1], hid[1:], W, bias)
        for o, oh in zip(outs, o_host):
            oh.copy_(o, non_blocking=True)

    t0 = time.perf_counter()
    for _ in range(max(1, args.warmup)):
        step()
    torch.cuda.synchronize()
    per = (time.perf_counter() - t0) / max(1, args.warmup)
    # at least 3 steps, at most 20, about 6 s of copies in all
    n = max(3, min(args.steps, 20, int(6.0 / max(per, 1e-6))))
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    a.record()
    for _ in range(n):
        step()
    b.record()
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(a.elapsed_time(b), world) / n
    del h_host, w_host, b_host, o_host
    return {"value": Lyr * T * k * world / (ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "ms_per_step": ms, "steps": n}



# ----------------------------------------------------------------------------- decode sweep
def run_decode(args, world, rank, local):
    """Decode-step split sweep: E=256, top-8, G=64 ranks x 4 experts, N=2.
    The plan is made once from step 0's counts (placement changes minutes
    apart); each decode step then runs count + split + assign on its own ids,
    as separate launches and as the fused lb_solve.  Per T: T_solve of one
    step, T_split, the throughput of 64 steps per launch, and the gate at the
    decode shape (H=7168).  The line's value takes, per T, the faster of the
    two batched forms."""
    from moe_expert_load_bf16_b200 import _lib, build, workloads
    from moe_expert_load_bf16_b200.pipeline import DecisionPath
    build.build()
    wl = rank_workload(workloads.WORKLOADS["decode"], rank)
    dev = torch.device("cuda", local)
    B = 64

    def timed(fn, reps):
        return graph_us(fn, reps, world)

    per_T = {}
    total_assign, total_us = 0, 0.0
    for T in wl.decode_T:
        ids = workloads.decode_ids(wl.with_(T=T), T, range(B + 1), device=dev)
        path = DecisionPath(B, T, wl.H, wl.E, wl.k, wl.G, wl.N, wl.L, device=dev)
        path.ids.copy_(ids[1:])
        path.ids_pred.copy_(ids[0:1].expand(B, -1, -1))
        _lib.lb_count(path.ids_pred[0:1], wl.G, wl.E, cnt=path.cnt_pred[0:1])
        _lib.lb_plan_replicas(path.cnt_pred[0:1], wl.N, wl.L, plan=path.plan[0:1])
        path.plan[1:].copy_(path.plan[0:1].expand(B - 1, -1))
        one = DecisionPath(1, T, wl.H, wl.E, wl.k, wl.G, wl.N, wl.L, device=dev)
        one.ids.copy_(ids[1:2])
        one.plan.copy_(path.plan[0:1])
        for _ in range(args.warmup):
            path.solve()
            one.solve()
            path.solve_fused()
            one.solve_fused()
        torch.cuda.synchronize()
        reps = max(20, args.steps)
        t_solve = timed(one.solve, reps)
        t_fused = timed(one.solve_fused, reps)
        t_split = timed(lambda: _lib.lb_split(one.cnt, one.plan, wl.N, 12,
                                              out=(one.tok, one.mass, one.loads, one.passes_run)), reps)
        t_batch_sep = timed(path.solve, max(5, reps // 4))
        t_batch_fused = timed(path.solve_fused, max(5, reps // 4))
        t_batch = min(t_batch_sep, t_batch_fused)
        h = workloads.hidden_chain(wl, 1, device=dev, T=T)[0]
        W = workloads.gate_weights(wl, 1, device=dev)[0]
        bias = workloads.biases(wl, 1)[0].to(dev)
        gate_ids = torch.empty(T, wl.k, dtype=torch.int32, device=dev)
        t_gate = timed(lambda: _lib.lb_predict_topk(h, W, bias, wl.k, ids=gate_ids), reps)
        gate_bytes = 2 * T * wl.H + 2 * wl.H * wl.E + 4 * wl.E + 4 * T * wl.k
        per_T[str(T)] = {"t_solve_us": t_solve, "t_solve_fused_us": t_fused, "t_split_us": t_split,
                         "batch64_us": t_batch_sep, "batch64_fused_us": t_batch_fused,
                         "batch64_assignments_per_s": B * T * wl.k / (t_batch * 1e-6),
                         "gate_us": t_gate, "gate_gbs": gate_bytes / (t_gate * 1e-6) / 1e9}
        total_assign += B * T * wl.k
        total_us += t_batch
        del ids, path, one, h, W
        torch.cuda.empty_cache()
    if _lib.lb_get_status():
        raise RuntimeError("device status flagged")
    value = total_assign * world / (total_us * 1e-6)
    return {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_us / 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int32", "data": "synthetic",
            "config": {"workload": "decode-step split sweep: E=256, top-8, G=64 ranks x 4 experts, N=2 (L=1); "
                                   "64 steps per T per launch (separate or fused, the faster); plan from step 0",
                       "T": list(wl.decode_T), "steps_per_launch": B},
            "per_T": per_T}

# ----------------------------------------------------------------------------- one kernel
def run_kernel(args, local):
    """One kernel of the path alone, for timing and for ncu: `--launches`
    plain launches (a profiler picks one with -k/-s/-c), then the mean over
    20 calls replayed from a CUDA graph (graph_us).  gate: the chain gate over `--problems` layers of the
    workload (its default: all); gate1: one layer's gate (lb_predict_topk,
    its automatic kernel choice) on `--tokens` tokens; count, plan, split, assign: one launch over
    `--problems` independent problems of the workload's shape (T, k, E, G, N)
    with decode-style synthetic ids (`--problems` default 128)."""
    from moe_expert_load_bf16_b200 import _lib, build, workloads
    from moe_expert_load_bf16_b200.pipeline import DecisionPath
    build.build()
    wl = workloads.WORKLOADS[args.config]
    dev = torch.device("cuda", local)
    T, H, E, k, G, N, L = wl.T, wl.H, wl.E, wl.k, wl.G, wl.N, wl.L
    hbm, tflops, _, peak_kind = peaks()
    if args.kernel == "gate":
        nl = args.problems or wl.layers
        hid = torch.empty(nl + 1, T, H, dtype=torch.bfloat16, device=dev)
        workloads.hidden_chain(wl, nl, out=hid[1:])
        hid[0].copy_(hid[1])
        W = workloads.gate_weights(wl, nl, device=dev)
        bias = workloads.biases(wl, nl).to(dev)
        ip = torch.empty(nl, T, k, dtype=torch.int32, device=dev)
        ia = torch.empty_like(ip)

        def fn():
            _lib.lb_predict_topk_chain(hid, W, bias, k, ids_pred=ip, ids_act=ia)
        nbytes = (nl + 1) * 2 * T * H + nl * (2 * H * E + 4 * E + 8 * T * k)
        flops = nl * 4.0 * T * H * E
        work = f"chain gate, {nl} layers ({nl + 1} hidden states) of {wl.name}"
    elif args.kernel == "gate1":
        T1 = args.tokens or T
        h1 = workloads.hidden_chain(wl, 1, device=dev, T=T1)[0]
        W1 = workloads.gate_weights(wl, 1, device=dev)[0]
        b1 = workloads.biases(wl, 1)[0].to(dev)
        ids1 = torch.empty(T1, k, dtype=torch.int32, device=dev)

        def fn():
            _lib.lb_predict_topk(h1, W1, b1, k, ids=ids1)
        nbytes = 2 * T1 * H + 2 * H * E + 4 * E + 4 * T1 * k
        flops = 2.0 * T1 * H * E
        work = f"one layer's gate, T={T1} of {wl.name} (H={H}, E={E}, top-{k})"
    else:
        nb = args.problems or 128
        path = DecisionPath(nb, T, 8, E, k, G, N, L, device=dev)
        for c0 in range(0, nb, 16):
            path.ids[c0:c0 + 16].copy_(workloads.decode_ids(wl, T, range(c0, min(nb, c0 + 16)), device=dev))
        _lib.lb_count(path.ids, G, E, cnt=path.cnt)
        _lib.lb_plan_replicas(path.cnt, N, L, plan=path.plan)
        _lib.lb_split(path.cnt, path.plan, N, 12, out=(path.tok, path.mass, path.loads, path.passes_run))
        tk = T * k
        n_edges = sum(int(d["n_edges"]) for d in _lib.decode_plan(path.plan, G, E, N)) / nb
        fns = {
            "count": (lambda: _lib.lb_count(path.ids, G, E, cnt=path.cnt), nb * (4 * tk + 4 * G * E)),
            "plan": (lambda: _lib.lb_plan_replicas(path.cnt, N, L, plan=path.plan), nb * 4 * G * E),
            "split": (lambda: _lib.lb_split(path.cnt, path.plan, N, 12,
                                            out=(path.tok, path.mass, path.loads, path.passes_run)),
                      int(nb * (4 * G * E + 12 * n_edges + 16 * G * N + 4 * G))),
            "assign": (lambda: _lib.lb_assign(path.ids, path.cnt, path.plan, path.tok, path.mass, N,
                                              out=(path.dest, path.perm, path.offs), workspace=path.ws),
                       nb * (3 * 4 * tk + 4 * (G * E + 1) + 4 * G * E + 8 * G * N)),
        }
        fn, nbytes = fns[args.kernel]
        flops = 0.0
        work = f"{args.kernel}, {nb} problems of {wl.name} (T={T}, top-{k}, E={E}, G={G}, N={N}), decode-style ids"
    for _ in range(args.launches):
        fn()
    torch.cuda.synchronize()
    us = graph_us(fn, 20)
    if _lib.lb_get_status():
        raise RuntimeError("device status flagged")
    out = {"kernel": args.kernel, "work": work, "us": us, "algorithmic_bytes": nbytes,
           "gbs": nbytes / us / 1e3, "hbm_frac": nbytes / us / 1e3 / hbm, "peak_kind": peak_kind}
    if flops:
        out.update(tflops=flops / us / 1e6, tensor_frac=flops / us / 1e6 / tflops)
    return out


# ----------------------------------------------------------------------------- CPU oracle
_CPU_INPUTS = {}


def _cpu_inputs(wl):
    """One layer's host inputs (two hidden states, its gate and bias as bit
    patterns), made once per workload."""
    from moe_expert_load_bf16_b200 import workloads
    if wl.name not in _CPU_INPUTS:
        hid = workloads.hidden_chain(wl, 2)
        hb = [workloads.bf16_bits(hid[0]), workloads.bf16_bits(hid[1])]
        wb = workloads.bf16_bits(workloads.gate_weights(wl, 1)[0])
        _CPU_INPUTS[wl.name] = (hb, wb, workloads.biases(wl, 1)[0].numpy())
    return _CPU_INPUTS[wl.name]


def cpu_baseline(wl, budget_s=15.0):
    """The oracle, as it stands, on this host's cores, over whole layers of
    the workload (both gate calls, count, plan, count, split, assign),
    repeated on one layer's inputs until the time budget is spent.  If one layer's gate would not fit the budget,
    the gate runs on evenly spaced sampled rows and its time is scaled to the
    full layer (the integer stages always run on the whole layer)."""
    import oracle
    o = oracle.default()
    T, H, E, k, G, N, L = wl.T, wl.H, wl.E, wl.k, wl.G, wl.N, wl.L
    hb, wb, b = _cpu_inputs(wl)
    probe = np.arange(min(T, 64))
    t0 = time.perf_counter()
    o.gate(hb[1][probe], wb, b, k)
    per_row = (time.perf_counter() - t0) / len(probe)
    rows = T if 2 * per_row * T <= 0.5 * budget_s else max(64, int(0.5 * budget_s / (2 * per_row)))
    sel = np.linspace(0, T - 1, rows).astype(np.int64)
    # full ids for the integer stages (computed once, untimed, when the gate is sampled)
    ids_pred_full = ids_full = None
    if rows < T:
        ids_pred_full = o.gate(hb[0], wb, b, k)[1]
        ids_full = o.gate(hb[1], wb, b, k)[1]
    total, layers, t_start = 0.0, 0, time.perf_counter()
    while layers == 0 or time.perf_counter() - t_start < budget_s:
        t0 = time.perf_counter()
        _, ids_pred = o.gate(hb[0][sel], wb, b, k)
        t_gate = time.perf_counter() - t0
        if rows < T:
            ids_pred = ids_pred_full
        t1 = time.perf_counter()
        p = o.plan(o.count(ids_pred, G, E), N, L)
        t_int = time.perf_counter() - t1
        t0 = time.perf_counter()
        _, ids = o.gate(hb[1][sel], wb, b, k)
        t_gate += time.perf_counter() - t0
        if rows < T:
            ids = ids_full
        t1 = time.perf_counter()
        cnt = o.count(ids, G, E)
        s = o.split(cnt, p, 12)
        o.assign(ids, p, s, G, E)
        t_int += time.perf_counter() - t1
        total += t_gate * T / rows + t_int
        layers += 1
    sample = (f"{layers} full layer pass(es) of {wl.name} (T={T}, H={H}, E={E}, top-{k}) on one layer's "
              f"inputs: both gate calls, count, plan, count, split, assign")
    if rows < T:
        sample += f"; gate on {rows} of {T} rows per call, time scaled to the full layer"
    return {"value": layers * T * k / total, "unit": UNIT, "cores": o.threads(), "kind": "oracle",
            "sample": sample, "seconds": total}


def run_reference(args, world, rank):
    from moe_expert_load_bf16_b200 import workloads
    wl = workloads.WORKLOADS[args.config]
    if rank != 0:
        return None
    for _ in range(min(args.warmup, 1)):
        cpu_baseline(wl, budget_s=1.0)
    per = args.cpu_budget if args.cpu_budget_set else max(2.0, min(20.0, 120.0 / max(1, args.steps)))
    t0 = time.perf_counter()
    vals = [cpu_baseline(wl, budget_s=per) for _ in range(args.steps)]
    wall = time.perf_counter() - t0
    value = statistics.mean(v["value"] for v in vals)
    cb = dict(vals[-1])
    cb["value"] = value
    Lyr, T, k = wl.layers, wl.T, wl.k
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": Lyr * T * k / value * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": f"{wl.name}: {Lyr} layers x T={T} tokens, H={wl.H}, E={wl.E}, top-{k}, "
                                   f"G={wl.G} ranks, N={wl.N} replica slots (L={wl.L})"},
            "cpu_baseline": cb, "wall_s": wall,
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default=DEFAULT_WORKLOAD)
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--in-flight", type=int, choices=(1, 2), default=2,
                    help="steps in flight in the chain form (2: the gate of one step beside the integer "
                         "stages of the previous one, on two streams)")
    ap.add_argument("--gate", choices=("chain", "two-pass"), default="chain",
                    help="chain: one gate pass per hidden state for both gates that read it; two-pass: "
                         "lookahead and normal router as separate passes")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kernel", choices=("gate", "gate1", "count", "plan", "split", "assign"), default=None,
                    help="time one kernel alone (with --problems, --launches) instead of the step")
    ap.add_argument("--tokens", type=int, default=0,
                    help="--kernel gate1: tokens of the one layer (default: the workload's T)")
    ap.add_argument("--problems", type=int, default=0,
                    help="--kernel: layers of the chain gate, or problems per integer-kernel launch")
    ap.add_argument("--launches", type=int, default=3, help="--kernel: plain launches before the timed replays")
    ap.add_argument("--decode-steps", type=int, default=1000,
                    help="decode steps per T in the per-step decode sweep of the extra keys")
    ap.add_argument("--lean", action="store_true",
                    help="time the steps only (no gate-only loop, per-layer latencies, end-to-end or CPU "
                         "baseline): the command used for ncu launch lists")
    args = ap.parse_args()
    args.cpu_budget_set = "--cpu-budget" in sys.argv
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", str(args.gpus)))
        out = run_reference(args, world, rank)
        if out is not None:
            print(json.dumps(out), flush=True)
        return
    if args.kernel:
        local = int(os.environ.get("LOCAL_RANK", "0"))
        print(json.dumps(run_kernel(args, local)), flush=True)
        return
    world, rank, local = dist_setup()
    try:
        out = run_decode(args, world, rank, local) if args.config == "decode" else run_ours(args, world, rank, local)
        if rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1 and torch.distributed.is_initialized():
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
