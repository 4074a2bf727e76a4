"""Phase timing of the latency-bound kernels (plan, split, assign prep and
scatter) and of the per-layer gate as CTA pairs with H split over two pairs
on one problem, from a separate build of the library with
-DLB_TIMING: block 0 of each kernel stamps clock64() at its phase boundaries
into a device array, read back with lb_debug_ticks.  The product library is
untouched (the timing build goes to liblb_timing.so and is loaded in place of
liblb.so by this process only).

    python -m moe_expert_load_bf16_b200.phase_timing [--config decode] [--T 8192] [--reps 20]

Prints, per kernel, the cycles (and microseconds at the maximum SM clock)
between consecutive stamps, the median over --reps launches.
"""
import argparse
import ctypes
import json
import os
import statistics

import torch

from . import _lib, build, workloads

TIMING_LIB = os.path.join(os.path.dirname(os.path.abspath(__file__)), "liblb_timing.so")

PHASES = {
    "plan": (30, ["stage counts", "phase 1 (locality imports)", "load model", "phase 2 (greedy moves)",
                  "edges", "round colouring + order", "write blob"]),
    "split": (0, ["stage inputs", "per-expert setup and start loads", "round table", "passes + masses"]),
    "plan detail": (None, [(35, 38, "round colouring"), (38, 36, "order by round")]),
    "split detail": (None, [(1, 7, "per-expert setup (thread 0)"), (7, 2, "wait for the other experts"),
                            (2, 8, "round table (thread 0's edges)"), (8, 3, "round table (wait for the others)"),
                            (3, 6, "passes"), (6, 4, "masses")]),
    "assign prep": (20, ["stage inputs, segment scan, chunk sums, per expert", "bucket sizes + scan",
                         "block bases"]),
    "assign prep detail": (None, [(20, 60, "stage inputs"), (60, 61, "segment scan"), (61, 62, "chunk sums"),
                                  (62, 21, "per expert"), (21, 24, "bucket sizes"), (24, 25, "edge shares"), (25, 26, "scan in the CTA"),
                                  (26, 27, "cluster barrier + carries"), (27, 22, "offsets written"),
                                  (22, 28, "q0 of the own blocks"), (28, 29, "barrier"),
                                  (29, 55, "edge shares + replica bases"), (55, 56, "cluster barrier"),
                                  (56, 57, "other keys"), (57, 23, "segments")]),
    "assign scatter": (10, ["per-problem tables", "scatter"]),
    "assign scatter detail (token path)": (None, [(10, 63, "stage segments"), (63, 9, "segment experts"),
                                                  (9, 11, "per expert"), (11, 58, "block classes"), (58, 59, "mask clear + barrier"),
                                                  (59, 13, "first ids")]),
    "assign scatter, first chunk (warp 0)": (None, [(13, 14, "ids, lane masks, in-warp ranks"), (14, 15, "scan down the warps (2 barriers)"),
                                                    (15, 16, "local and home slots placed, replicated queued"),
                                                    (16, 17, "replicated queue resolved"), (17, 18, "dest rows written"),
                                                    (18, 19, "closing barrier")]),
    "gate (pairs, H split)": (None, [(40, 41, "prologue"), (41, 44, "loads + MMAs (MMA issuer)"),
                                     (44, 47, "accumulator complete (epilogue)"),
                                     (47, 54, "partial TMEM -> shared memory"), (54, 48, "cluster barrier"),
                                     (48, 52, "other pairs' slices arrive"), (52, 53, "rank own rows"),
                                     (53, 49, "merge lists"), (49, 50, "write ids"), (50, 51, "closing barrier")]),
}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--config", default="decode")
    ap.add_argument("--T", type=int, default=0, help="tokens per problem (default: the workload's)")
    ap.add_argument("--reps", type=int, default=20)
    args = ap.parse_args()
    build.build(extra=["-DLB_TIMING"], out=TIMING_LIB)
    _lib.LIB_PATH = TIMING_LIB
    lib = _lib._load()
    lib.lb_debug_ticks.argtypes = [ctypes.POINTER(ctypes.c_longlong), ctypes.c_int]
    lib.lb_debug_ticks.restype = ctypes.c_int
    wl = workloads.WORKLOADS[args.config]
    T = args.T or wl.T
    G, E, k, N, L = wl.G, wl.E, wl.k, wl.N, wl.L
    dev = torch.device("cuda", 0)
    ids = workloads.decode_ids(wl.with_(T=T), T, [0, 1], device=dev)
    cnt_pred = _lib.lb_count(ids[0:1], G, E)
    cnt = _lib.lb_count(ids[1:2], G, E)
    plan = _lib.lb_plan_replicas(cnt_pred, N, L)
    tok, mass, loads, pr = _lib.lb_split(cnt, plan, N, 12)
    ws = torch.empty(max(256, _lib.lb_assign_workspace_bytes(1, T, k, G, E, N)), dtype=torch.uint8, device=dev)
    launches = {
        "plan": lambda: _lib.lb_plan_replicas(cnt_pred, N, L, plan=plan),
        "split": lambda: _lib.lb_split(cnt, plan, N, 12, out=(tok, mass, loads, pr)),
        "assign": lambda: _lib.lb_assign(ids[1:2], cnt, plan, tok, mass, N, workspace=ws),
    }
    # the per-layer gate as CTA pairs with H split over two pairs, on the
    # workload's hidden size and experts
    hid = workloads.hidden_chain(wl, 1, device=dev, T=T)[0]
    Wg = workloads.gate_weights(wl, 1, device=dev)[0]
    bg = workloads.biases(wl, 1)[0].to(dev)
    ids_g = torch.empty(T, k, dtype=torch.int32, device=dev)

    def gate_pairs():
        _lib.lb_gate_tuning(0, 0, 5)
        try:
            _lib.lb_predict_topk(hid, Wg, bg, k, ids=ids_g)
        finally:
            _lib.lb_gate_tuning()

    launches["gate"] = gate_pairs
    try:   # clock64 counts SM cycles; microseconds below are at the maximum SM clock
        import pynvml
        pynvml.nvmlInit()
        khz = 1000 * pynvml.nvmlDeviceGetMaxClockInfo(pynvml.nvmlDeviceGetHandleByIndex(0), pynvml.NVML_CLOCK_SM)
    except Exception:
        khz = 1965000
    ticks = (ctypes.c_longlong * 64)()
    res = {"workload": f"{wl.name}: T={T}, E={E}, top-{k}, G={G}, N={N} (L={L}), one problem",
           "passes_run": int(pr.item()), "clock_khz": khz}
    samples = {}
    for name, fn in launches.items():
        for _ in range(args.reps):
            fn()
            if lib.lb_debug_ticks(ticks, 64) != 0:
                raise RuntimeError("lb_debug_ticks failed")
            kernels = [name] if name != "assign" else ["assign prep", "assign prep detail", "assign scatter",
                                                       "assign scatter detail (token path)",
                                                       "assign scatter, first chunk (warp 0)"]
            if name == "gate":
                kernels = ["gate (pairs, H split)"]
            if name == "split":
                kernels = kernels + ["split detail"]
            if name == "plan":
                kernels = kernels + ["plan detail"]
            for kn in kernels:
                first, labels = PHASES[kn]
                for i, lab in enumerate(labels):
                    if first is None:   # (from stamp, to stamp, label)
                        a, b, lab = lab
                        dt = ticks[b] - ticks[a]
                    else:
                        dt = ticks[first + i + 1] - ticks[first + i]
                    samples.setdefault(kn, {}).setdefault(lab, []).append(dt)
    for kn, d in samples.items():
        res[kn] = {lab: {"cycles": statistics.median(v), "us": statistics.median(v) / (khz * 1e-3)}
                   for lab, v in d.items()}
    print(json.dumps(res, indent=1))


if __name__ == "__main__":
    main()
