"""Two studies over the library's kernels (no new kernel on the hot path):

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
   (mass / tok, applied to the edge's tokens at s + r, rounded to nearest).
     gain(split)  = max load without balancing - max load with the split
     forfeited(r) = 1 - gain(split of step s, used at s + r) / gain(fresh split at s + r)
   "Without balancing" keeps every remote token at its expert's home
   (lb_split with 0 passes).

    python tests/lookahead_study.py [--out FILE]
"""
import argparse
import json
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from moe_expert_load_bf16_b200 import _lib, workloads  # noqa: E402


def lookahead_quality(name, layers, T=None, dev="cuda"):
    w = workloads.WORKLOADS[name]
    T = T or w.T
    hid = torch.empty(layers + 1, T, w.H, dtype=torch.bfloat16, device=dev)
    workloads.hidden_chain(w, layers + 1, T=T, out=hid)
    W = workloads.gate_weights(w, layers, device=dev)
    bias = workloads.biases(w, layers).to(dev)
    ip, ia, lp, la = _lib.lb_predict_topk_chain(hid, W, bias, w.k, want_logits=True)
    cp, ca = _lib.lb_count(ip, w.G, w.E), _lib.lb_count(ia, w.G, w.E)
    torch.cuda.synchronize()
    hit = []
    cos = []
    mtm_p, mtm_a = [], []
    for l in range(layers):
        a, b = ip[l].long(), ia[l].long()
        pm = torch.zeros(T, w.E, dtype=torch.bool, device=dev).scatter_(1, a, True)
        am = torch.zeros(T, w.E, dtype=torch.bool, device=dev).scatter_(1, b, True)
        hit.append(((pm & am).sum(dim=1).double() / w.k).mean().item())
        cos.append(torch.nn.functional.cosine_similarity(lp[l].double(), la[l].double(), dim=1).mean().item())
        Eg = w.E // w.G
        for c, out in ((cp[l], mtm_p), (ca[l], mtm_a)):
            rank = c.sum(dim=0).view(w.G, Eg).sum(dim=1).double()
            out.append((rank.max() / rank.mean()).item())
    return {"workload": f"{name}: {layers} layers x T={T}, H={w.H}, E={w.E}, top-{w.k}, drift {w.drift}",
            "hit_mean": float(np.mean(hit)), "hit_min": float(np.min(hit)), "cosine_mean": float(np.mean(cos)),
            "cosine_min": float(np.min(cos)), "rank_max_to_mean_predicted": float(np.mean(mtm_p)),
            "rank_max_to_mean_actual": float(np.mean(mtm_a)), "per_layer_hit": hit, "per_layer_cosine": cos}


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


def decision_frequency(G, E, N, steps=24, T=4096, k=8, passes=12, lags=(1, 2, 4, 8), dev="cuda"):
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
    out = {}
    for r in lags:
        forf = []
        for s in range(steps - r):
            t = s + r
            gain_fresh = loads0[t].max() - loads[t].max()
            if gain_fresh <= 0:
                continue
            frac = np.where(tok[s] > 0, mass[s] / np.maximum(tok[s], 1), 1.0)
            stale = stale_loads(fixed[t], eu, ev, tok[t], frac)
            forf.append(1.0 - (loads0[t].max() - stale.max()) / gain_fresh)
        out[str(r)] = {"forfeited_mean": float(np.mean(forf)) if forf else None, "samples": len(forf)}
    return {"workload": f"decode steps: G={G}, E={E}, top-{k}, N={N}, T={T} per step, {steps} steps, plan from step 0",
            "forfeited_gain_by_reuse_lag": out}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--out", default=None)
    args = ap.parse_args()
    res = {"lookahead": [lookahead_quality("olmoe", 16), lookahead_quality("qwen3-30b", 8, T=4096)],
           "decision_frequency": [decision_frequency(16, 128, 8), decision_frequency(64, 256, 8),
                                  decision_frequency(16, 128, 2)]}
    txt = json.dumps(res, indent=1)
    if args.out:
        with open(args.out, "w") as f:
            f.write(txt)
    print(txt)


if __name__ == "__main__":
    main()
