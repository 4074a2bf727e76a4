"""Measurement studies over the library's kernels (no new kernel on the hot
path).

1. Lookahead quality (FreeBalance sec. 4, Table 2: early-router top-k hit
   and logit cosine): for every layer of a synthetic hidden-state chain, the
   lookahead gate (layer l's gate on the hidden state before layer l) against
   the normal router (the same gate on layer l's input), both from one
   lb_predict_topk_chain launch with logits.
     hit    = |predicted top-k  intersect  actual top-k| / k, mean over tokens
     cosine = cos(predicted logits, actual logits), mean over tokens
   and the max-to-mean rank load of the predicted and the actual counts.

2. Decision frequency (Relief, Failure of Existing Approaches: reusing a split
   for even one more step forfeits most of its gain): on synthetic decode
   steps with per-step routing, a split made at step s is reused at step
   s + r, each edge keeping the share of its tokens it kept at home
   (mass / tok, applied to the edge's tokens at s + r, rounded to nearest,
   ties to even).
     gain(split)  = max load without balancing - max load with the split
     forfeited(r) = 1 - gain(split of step s, used at s + r) / gain(fresh split at s + r)
   "Without balancing" keeps every remote token at its expert's home
   (lb_split with 0 passes).

3. Relief's ablation (Relief, Ablation Results, Table III; Convergence and
   Pass Count; Pass Count Selection): attainment of the exact per-step
   optimum for every split variant, the attainment-vs-passes curve s[p], and
   the pass count I* = argmax_p s[p] / (1 + T_split(p) / T_moe) with the
   measured split time.  The exact optimum is computed by a function the
   caller passes in (an exact integer min-max solver).

    python -m moe_expert_load_bf16_b200.studies [--out FILE]   (studies 1 and 2)
"""
import argparse
import json

import numpy as np
import torch

from . import _lib, workloads


def lookahead_quality(name, layers, T=None, dev="cuda"):
    """Study 1 on `layers` layers of a workload's synthetic chain.  Returns
    the summary and, under "ids"/"logits", the kernel's outputs (predicted
    and actual ids [layers, T, k], logits [layers, T, E]) and the inputs,
    so a caller can recompute the statistics independently."""
    w = workloads.WORKLOADS[name]
    T = T or w.T
    hid = torch.empty(layers + 1, T, w.H, dtype=torch.bfloat16, device=dev)
    workloads.hidden_chain(w, layers + 1, T=T, out=hid)
    W = workloads.gate_weights(w, layers, device=dev)
    bias = workloads.biases(w, layers).to(dev)
    ip, ia, lp, la = _lib.lb_predict_topk_chain(hid, W, bias, w.k, want_logits=True)
    cp, ca = _lib.lb_count(ip, w.G, w.E), _lib.lb_count(ia, w.G, w.E)
    torch.cuda.synchronize()
    hit, cos, mtm_p, mtm_a = [], [], [], []
    for l in range(layers):
        hit.append(topk_hit(ip[l], ia[l], w.E))
        cos.append(torch.nn.functional.cosine_similarity(lp[l].double(), la[l].double(), dim=1).mean().item())
        for c, out in ((cp[l], mtm_p), (ca[l], mtm_a)):
            out.append(rank_max_to_mean(c, w.G))
    return {"workload": f"{name}: {layers} layers x T={T}, H={w.H}, E={w.E}, top-{w.k}, drift {w.drift}",
            "hit_mean": float(np.mean(hit)), "hit_min": float(np.min(hit)), "cosine_mean": float(np.mean(cos)),
            "cosine_min": float(np.min(cos)), "rank_max_to_mean_predicted": float(np.mean(mtm_p)),
            "rank_max_to_mean_actual": float(np.mean(mtm_a)), "per_layer_hit": hit, "per_layer_cosine": cos,
            "tensors": {"hid": hid, "W": W, "bias": bias, "ids_pred": ip, "ids_act": ia, "logits_pred": lp,
                        "logits_act": la, "cnt_pred": cp, "cnt_act": ca}}


def topk_hit(a, b, E):
    """Mean over rows of |set(a[row]) & set(b[row])| / k (torch int tensors [T, k])."""
    T, k = a.shape
    pm = torch.zeros(T, E, dtype=torch.bool, device=a.device).scatter_(1, a.long(), True)
    am = torch.zeros(T, E, dtype=torch.bool, device=a.device).scatter_(1, b.long(), True)
    return ((pm & am).sum(dim=1).double() / k).mean().item()


def rank_max_to_mean(cnt, G):
    """Max-to-mean of the per-rank load of counts [G, E] under the even
    placement (expert e on rank e // (E / G))."""
    E = cnt.shape[1]
    rank = cnt.sum(dim=0).view(G, E // G).sum(dim=1).double()
    return (rank.max() / rank.mean()).item()


def stale_loads(fixed, eu, ev, tok_new, frac):
    """Loads at a later step when each edge keeps the home share `frac` of
    an earlier split: fixed loads plus round(frac * tok) at home and the rest
    at the replica."""
    loads = fixed.astype(np.int64).copy()
    mass = np.rint(frac * tok_new).astype(np.int64)
    mass = np.clip(mass, 0, tok_new)
    np.add.at(loads, eu, mass)
    np.add.at(loads, ev, tok_new - mass)
    return loads


def forfeited(loads0, loads, fixed, tok, mass, eu, ev, lags):
    """Study 2's arithmetic from per-step results: loads0 [S, G] without
    balancing, loads [S, G] with the fresh split, fixed [S, G] loads that no
    edge moves, tok/mass [S, n_edges] of the fresh split, edges (eu, ev).
    Returns {lag: [forfeited share per usable step pair]}."""
    out = {}
    steps = loads.shape[0]
    for r in lags:
        vals = []
        for s in range(steps - r):
            t = s + r
            gain_fresh = loads0[t].max() - loads[t].max()
            if gain_fresh <= 0:
                continue
            frac = np.where(tok[s] > 0, mass[s] / np.maximum(tok[s], 1), 1.0)
            stale = stale_loads(fixed[t], eu, ev, tok[t], frac)
            vals.append(1.0 - (loads0[t].max() - stale.max()) / gain_fresh)
        out[r] = vals
    return out


def decision_frequency(G, E, N, steps=24, T=4096, k=8, passes=12, lags=(1, 2, 4, 8), dev="cuda"):
    """Study 2 on `steps` synthetic decode steps after step 0 (which plans).
    Returns the summary and, under "raw", the ids, the plan and the per-lag
    values so a caller can recompute them independently."""
    w = workloads.WORKLOADS["decode"].with_(E=E, G=G, T=T, k=k, N=N)
    ids = workloads.decode_ids(w, T, range(steps + 1), device=dev)
    cnt = _lib.lb_count(ids, G, E)
    plan0 = torch.empty(1, _lib.lb_plan_bytes(G, E, N), dtype=torch.uint8, device=dev)
    _lib.lb_plan_replicas(cnt[0:1], N, w.L, plan=plan0)
    plan = plan0.expand(steps, -1).contiguous()
    c = cnt[1:].contiguous()
    tok, mass, loads, _ = _lib.lb_split(c, plan, N, passes)
    tok0, mass0, loads0, _ = _lib.lb_split(c, plan, N, 0)           # no balancing: all at home
    torch.cuda.synchronize()
    dec = _lib.decode_plan(plan0[0], G, E, N)[0]
    ne = int(dec["n_edges"])
    eu, ev = dec["edge_u"][:ne], dec["edge_v"][:ne]
    tok, mass, loads = tok.cpu().numpy()[:, :ne], mass.cpu().numpy()[:, :ne], loads.cpu().numpy()
    loads0 = loads0.cpu().numpy()
    fixed = loads0.astype(np.int64).copy()
    for s in range(steps):
        np.subtract.at(fixed[s], eu, tok[s])                           # remove the all-at-home masses
    vals = forfeited(loads0, loads, fixed, tok, mass, eu, ev, lags)
    out = {str(r): {"forfeited_mean": float(np.mean(v)) if v else None, "samples": len(v)} for r, v in vals.items()}
    return {"workload": f"decode steps: G={G}, E={E}, top-{k}, N={N}, T={T} per step, {steps} steps, plan from step 0",
            "forfeited_gain_by_reuse_lag": out,
            "raw": {"ids": ids, "L": w.L, "values": vals, "loads": loads, "loads0": loads0}}


def _timed(fn, reps=200):
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


def ablation(name, G, E, steps, optimum, T=4096, k=8, N=2, max_passes=32, timing=True, dev="cuda"):
    """Study 3 for one group size: `optimum(cnt, step)` gives the exact
    minimum max load of step `step` (counts [G, E] as numpy) over the plan
    made from step 0's counts.  Placement planned once from step 0's counts
    (placements change minutes apart); every later step split with each
    variant."""
    w = workloads.WORKLOADS["decode"].with_(E=E, G=G, T=T, k=k, N=N)
    L = w.L
    ids = workloads.decode_ids(w, T, range(steps + 1), device=dev)
    cnt = _lib.lb_count(ids, G, E)                       # [steps+1, G, E]
    plan0 = torch.empty(1, _lib.lb_plan_bytes(G, E, N), dtype=torch.uint8, device=dev)
    _lib.lb_plan_replicas(cnt[0:1], N, L, plan=plan0)
    plan = plan0.expand(steps, -1).contiguous()
    c = cnt[1:].contiguous()
    torch.cuda.synchronize()
    c_np = c.cpu().numpy()
    opt = np.array([optimum(cnt[0].cpu().numpy(), c_np[s]) for s in range(steps)], np.float64)
    total = c_np.reshape(steps, -1).sum(axis=1).astype(np.float64)

    def quality(loads):
        mx = loads.max(axis=1).astype(np.float64)
        return float(np.mean(opt / mx)), float(np.mean(total / (G * mx))), mx

    table = {}
    for v in _lib.SPLIT_VARIANTS:
        passes = 12 if v != "jacobi" else 48          # the pages: Jacobi needs about 4x the passes
        tok, mass, loads, pr = _lib.lb_split_variant(c, plan, N, passes, v)
        torch.cuda.synchronize()
        att, spatial, mx = quality(loads.cpu().numpy())
        row = {"attainment": att, "spatial": spatial, "passes": passes,
               "passes_run_mean": float(pr.double().mean()), "max_load": mx.tolist()}
        if timing:
            row["t_split_us_one_problem"] = _timed(lambda: _lib.lb_split_variant(c[0:1], plan[0:1], N, passes, v))
        table[v] = row
    curve, t_split = [], []
    for p in range(0, max_passes + 1):
        _, _, loads, _ = _lib.lb_split_variant(c, plan, N, p, "relief")
        torch.cuda.synchronize()
        curve.append(quality(loads.cpu().numpy())[0])
        if timing and p in (0, 1, 2, 4, 8, 12, 16, 24, 32):
            out = tuple(torch.empty_like(x) for x in _lib.lb_split(c[0:1], plan[0:1], N, p))
            t_split.append((p, _timed(lambda: _lib.lb_split(c[0:1], plan[0:1], N, p, out=out))))
    res = {"workload": f"{name}: G={G}, E={E}, top-{k}, N={N}, L={L}, T={T} per step, {steps} steps, plan from step 0",
           "variants": table, "relief_attainment_by_passes": curve, "optimum": opt.tolist()}
    if len(t_split) >= 2:
        ps = np.array([x[0] for x in t_split], np.float64)
        ts = np.array([x[1] for x in t_split], np.float64)
        a1, a0 = np.polyfit(ps, ts, 1)                          # T_split(p) ~ a0 + a1 p
        istar = {}
        for t_moe in (25.0, 50.0, 100.0, 200.0, 500.0, 1000.0, 5000.0):
            score = [curve[p] / (1.0 + (a0 + a1 * p) / t_moe) for p in range(len(curve))]
            istar[str(t_moe)] = int(np.argmax(score))
        res.update(t_split_fit_us={"a0": a0, "a1_per_pass": a1, "points": t_split}, i_star_by_t_moe_us=istar)
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--out", default=None)
    args = ap.parse_args()

    def public(d):
        return {k: v for k, v in d.items() if k not in ("tensors", "raw")}
    res = {"lookahead": [public(lookahead_quality("olmoe", 16)), public(lookahead_quality("qwen3-30b", 8, T=4096))],
           "decision_frequency": [public(decision_frequency(16, 128, 8)), public(decision_frequency(64, 256, 8)),
                                  public(decision_frequency(16, 128, 2))]}
    txt = json.dumps(res, indent=1)
    if args.out:
        with open(args.out, "w") as f:
            f.write(txt)
    print(txt)


if __name__ == "__main__":
    main()
