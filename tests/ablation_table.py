"""Relief's ablation on this library (Relief, Ablation Results, Table III;
Convergence and Pass Count; Pass Count Selection), on synthetic decode-step
routing: the placement is planned once from step 0's counts (placements
change minutes apart) and every later step is split with each variant.

    python tests/ablation_table.py [--steps S] [--out FILE]

Per group size (G=16: E=128 as the Qwen3-30B shape; G=64: E=256 as the
decode shape; top-8, T=4096 tokens per step) and replica slots per rank
(N=2, L=1 as the configs; N=8, L=4, the pages' Libra example, which gives
the split more to do):
  * attainment of the exact per-step optimum (the oracle's integer min-max,
    a max-flow computation) = optimum / max load, mean over steps, and the
    spatial balance sum L / (G max L), for every variant of lb_split_variant;
  * Relief's attainment after p passes, p = 0..32 (the s[p] curve);
  * T_split(p) of lb_split on one problem (CUDA events, graph replay) and
    I* = argmax_p s[p] / (1 + T_split(p) / T_moe) for several T_moe (the
    pages' pass-count selection with the measured solve time in place of
    the interface latency and cycle model).
Uses the GPU library for every split and the oracle only for the optimum.
"""
import argparse
import json
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from moe_expert_load_bf16_b200 import _lib, workloads  # noqa: E402


def timed(fn, reps=200):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        g.replay()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) * 1e3 / reps


def group(name, G, E, steps, T=4096, k=8, N=2, dev="cuda"):
    w = workloads.WORKLOADS["decode"].with_(E=E, G=G, T=T, k=k, N=N)
    L = w.L
    ids = workloads.decode_ids(w, T, range(steps + 1), device=dev)
    cnt = _lib.lb_count(ids, G, E)                       # [steps+1, G, E]
    plan0 = torch.empty(1, _lib.lb_plan_bytes(G, E, N), dtype=torch.uint8, device=dev)
    _lib.lb_plan_replicas(cnt[0:1], N, L, plan=plan0)
    plan = plan0.expand(steps, -1).contiguous()
    c = cnt[1:].contiguous()
    torch.cuda.synchronize()
    p_or = oracle.plan(cnt[0].cpu().numpy(), N, L)
    c_np = c.cpu().numpy()
    opt = np.array([oracle.split_optimum(c_np[s], p_or) for s in range(steps)], np.float64)
    total = c_np.reshape(steps, -1).sum(axis=1).astype(np.float64)

    def quality(loads):
        mx = loads.max(axis=1).astype(np.float64)
        return float(np.mean(opt / mx)), float(np.mean(total / (G * mx)))

    table = {}
    for v in _lib.SPLIT_VARIANTS:
        passes = 12 if v != "jacobi" else 48          # the pages: Jacobi needs about 4x the passes
        tok, mass, loads, pr = _lib.lb_split_variant(c, plan, N, passes, v)
        torch.cuda.synchronize()
        att, spatial = quality(loads.cpu().numpy())
        t = timed(lambda: _lib.lb_split_variant(c[0:1], plan[0:1], N, passes, v))
        table[v] = {"attainment": att, "spatial": spatial, "passes": passes,
                    "passes_run_mean": float(pr.double().mean()), "t_split_us_one_problem": t}
    curve, t_split = [], []
    for p in range(0, 33):
        _, _, loads, _ = _lib.lb_split_variant(c, plan, N, p, "relief")
        torch.cuda.synchronize()
        curve.append(quality(loads.cpu().numpy())[0])
        if p in (0, 1, 2, 4, 8, 12, 16, 24, 32):
            out = tuple(torch.empty_like(x) for x in _lib.lb_split(c[0:1], plan[0:1], N, p))
            t_split.append((p, timed(lambda: _lib.lb_split(c[0:1], plan[0:1], N, p, out=out))))
    ps = np.array([x[0] for x in t_split], np.float64)
    ts = np.array([x[1] for x in t_split], np.float64)
    a1, a0 = np.polyfit(ps, ts, 1)                          # T_split(p) ~ a0 + a1 p
    istar = {}
    for t_moe in (25.0, 50.0, 100.0, 200.0, 500.0, 1000.0, 5000.0):
        score = [curve[p] / (1.0 + (a0 + a1 * p) / t_moe) for p in range(len(curve))]
        istar[str(t_moe)] = int(np.argmax(score))
    return {"workload": f"{name}: G={G}, E={E}, top-{k}, N={N}, L={L}, T={T} per step, {steps} steps, plan from step 0",
            "variants": table, "relief_attainment_by_passes": curve,
            "t_split_fit_us": {"a0": a0, "a1_per_pass": a1, "points": t_split}, "i_star_by_t_moe_us": istar}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--steps", type=int, default=8)
    ap.add_argument("--out", default=None)
    args = ap.parse_args()
    res = {}
    for N in (2, 8):
        res[f"G16_N{N}"] = group("qwen3-30b-shaped", 16, 128, args.steps, N=N)
        res[f"G64_N{N}"] = group("decode-shaped", 64, 256, args.steps, N=N)
    txt = json.dumps(res, indent=1)
    if args.out:
        with open(args.out, "w") as f:
            f.write(txt)
    print(txt)


if __name__ == "__main__":
    main()
