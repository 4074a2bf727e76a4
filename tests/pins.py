"""Pins for the CPU oracle: checks against what the pages and mathematics fix,
never against the oracle itself.  Each check takes an oracle instance so the
same checks can be run against deliberately broken builds of the oracle
(see test_oracle_mutants.py) to show that they catch plausible mistakes.

Kinds of pin used:
  * hand-worked examples derived from the pages' rules (tests/golden/*.json,
    each with its citation and derivation);
  * exact arithmetic (Python fractions) for the gate on tiny inputs;
  * an independent library computation of the same definition
    (numpy fp64 matmul for the logits, numpy stable argsort for top-k,
    numpy bincount for the histogram);
  * invariants and closed forms (conservation, bounds, monotonicity);
  * brute force over every integer split on tiny instances for the optimum.
"""
import itertools
import json
import os
from fractions import Fraction

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def f32_to_bf16_bits(x):
    """Round fp32 -> bf16 bit pattern, nearest even (inputs are finite)."""
    u = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    rounding = ((u >> 16) & 1) + 0x7FFF
    return ((u + rounding) >> 16).astype(np.uint16)


def bf16_bits_to_f64(b):
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def rand_gate(rng, T, H, E, bias=True):
    h = f32_to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
    w = f32_to_bf16_bits((rng.standard_normal((E, H)) / np.sqrt(H)).astype(np.float32))
    b = (2.0 * rng.permutation(np.arange(1, E + 1)) ** -1.2).astype(np.float32) if bias else None
    return h, w, b


def golden_plan(o, d):
    import oracle
    return oracle.plan_from_arrays(d["G"], d["E"], d.get("N", 0), d.get("L", 0), np.array(d["holds"]),
                                   [e[0] for e in d["edges"]], [e[1] for e in d["edges"]],
                                   [e[2] for e in d["edges"]], d["round_ptr"])


# ----------------------------------------------------------------------------- gate

def check_gate_exact_tiny(o):
    """Logits equal the exact rational sum, rounded to fp32 (within 1 ulp);
    ids are the k largest with ties to the lower id (brute-force sort)."""
    rng = np.random.default_rng(7)
    T, H, E, k = 6, 24, 7, 3
    h, w, b = rand_gate(rng, T, H, E)
    logits, ids = o.gate(h, w, b, k)
    hv = [[Fraction(float(x)) for x in row] for row in bf16_bits_to_f64(h)]
    wv = [[Fraction(float(x)) for x in row] for row in bf16_bits_to_f64(w)]
    for t in range(T):
        exact = [sum(hv[t][c] * wv[e][c] for c in range(H)) + Fraction(float(b[e])) for e in range(E)]
        want = np.array([float(x) for x in exact], np.float32)
        assert np.allclose(logits[t], want, rtol=2e-7, atol=1e-7), (t, logits[t], want)
        order = sorted(range(E), key=lambda e: (-want[e], e))
        assert list(ids[t]) == order[:k], (t, ids[t], order[:k])


def check_gate_matches_numpy(o):
    """Logits vs numpy fp64 h @ W^T + b; ids vs stable argsort of -logits."""
    rng = np.random.default_rng(11)
    T, H, E, k = 33, 256, 40, 5
    h, w, b = rand_gate(rng, T, H, E)
    logits, ids = o.gate(h, w, b, k)
    ref = (bf16_bits_to_f64(h) @ bf16_bits_to_f64(w).T + b.astype(np.float64)).astype(np.float32)
    assert np.allclose(logits, ref, rtol=1e-6, atol=1e-6)
    want = np.argsort(-logits, axis=1, kind="stable")[:, :k]
    assert np.array_equal(ids, want)
    # no bias: plain product
    logits0, _ = o.gate(h, w, None, k)
    ref0 = (bf16_bits_to_f64(h) @ bf16_bits_to_f64(w).T).astype(np.float32)
    assert np.allclose(logits0, ref0, rtol=1e-6, atol=1e-6)


def check_gate_ties(o):
    """Equal logits: the lower expert id ranks first."""
    H, E, k = 16, 6, 4
    w = np.zeros((E, H), np.uint16)
    one = f32_to_bf16_bits(np.float32(1.0))
    w[1, :] = one
    w[4, :] = one       # experts 1 and 4 tie
    w[3, 0] = f32_to_bf16_bits(np.float32(2.0))
    h = np.tile(one, (2, H))
    _, ids = o.gate(h, w, None, k)
    # logits: e1=16, e4=16, e3=2, others 0 -> [1,4,3,0]
    assert list(ids[0]) == [1, 4, 3, 0], ids[0]
    assert list(ids[1]) == [1, 4, 3, 0], ids[1]


def check_gate_cancellation(o):
    """A sum whose exact value is lost in fp32 accumulation: 2^24 + 1 - 2^24 = 1.
    The oracle's double accumulation must return the exact value."""
    H, E = 3, 2
    h = f32_to_bf16_bits(np.array([[2.0 ** 24, 1.0, -(2.0 ** 24)]], np.float32))
    w = f32_to_bf16_bits(np.array([[1.0, 1.0, 1.0], [0.0, 0.0, 0.0]], np.float32))
    logits, ids = o.gate(h, w, None, 1)
    assert logits[0, 0] == 1.0 and logits[0, 1] == 0.0
    assert ids[0, 0] == 0


# ----------------------------------------------------------------------------- count

def check_count(o):
    rng = np.random.default_rng(3)
    T, k, E, G = 96, 4, 12, 4
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    cnt = o.count(ids, G, E)
    assert cnt.sum() == T * k
    Tg = T // G
    for g in range(G):
        assert np.array_equal(cnt[g], np.bincount(ids[g * Tg:(g + 1) * Tg].ravel(), minlength=E))


def check_count_rejects(o):
    import oracle
    bad = np.array([[0, 1], [2, 2]], np.int32)            # duplicate in a row
    for arr, G, code in ((bad, 2, 3), (np.array([[0, 9]], np.int32), 1, 3),
                         (np.array([[0, 1]] * 3, np.int32), 2, 1)):
        try:
            o.count(arr, G, 4)
        except oracle.OracleError as e:
            assert e.code == code
        else:
            raise AssertionError("bad input accepted")


# ----------------------------------------------------------------------------- plan

def check_plan_golden(o):
    for name in ("plan_phase2_basic.json", "plan_phase1_phase2.json", "plan_stop_rule.json",
                 "plan_argmax_tie.json"):
        d = golden(name)
        p = o.plan(np.array(d["cnt"], np.int32), d["N"], d["L"])
        assert np.array_equal(p.holds, np.array(d["holds"])), name
        assert np.array_equal(p.used, d["used"]), name
        assert np.array_equal(p.slots, np.array(d["slots"])), name
        assert np.array_equal(p.slot_phase, np.array(d["slot_phase"])), name
        assert np.array_equal(p.plan_load, d["plan_load"]), name
        got = [[int(a), int(b), int(c)] for a, b, c in zip(p.edge_u, p.edge_v, p.edge_e)]
        assert got == d["edges"], (name, got)
        assert list(p.round_ptr) == d["round_ptr"], name


def check_plan_phase1_ties(o):
    """Phase 1 takes (count desc, id asc) and never imports an unrequested expert."""
    cnt = np.array([[5, 5, 4, 4], [0, 0, 0, 0]], np.int32)   # rank 0 ties between e2,e3
    p = o.plan(cnt, 2, 2)
    assert list(p.slots[0]) == [2, 3] and list(p.slot_phase[0]) == [1, 1]
    assert p.used[1] == 0 or all(p.slot_phase[1][:p.used[1]] == 2)
    cnt = np.array([[9, 9, 1, 3], [0, 0, 0, 0]], np.int32)
    p = o.plan(cnt, 2, 1)
    assert p.slots[0][0] == 3 and p.slot_phase[0][0] == 1   # e3 (3) before e2 (1)


def plan_invariants(cnt, p, N, L):
    G, E = cnt.shape
    Eg = E // G
    home = np.arange(E) // Eg
    assert all(p.holds[home[e], e] == 1 for e in range(E))
    rep = p.holds.copy()
    rep[home, np.arange(E)] = 0
    assert np.array_equal(rep.sum(1), p.used)
    assert (p.used <= N).all()
    assert ((p.slot_phase == 1).sum(1) <= L).all()
    for g in range(G):
        s = [x for x in p.slots[g] if x >= 0]
        assert len(s) == p.used[g] and len(set(s)) == len(s)
        assert all(rep[g, x] for x in s)
        ph = list(p.slot_phase[g][:p.used[g]])
        assert ph == sorted(ph)                    # phase-1 slots come first
        for x, f in zip(s, ph):
            if f == 1:
                assert cnt[g, x] > 0               # only requested experts are imported
    assert p.plan_load.sum() == cnt.sum()
    # one edge per replica, from home to the replica rank
    edges = sorted(zip(p.edge_e.tolist(), p.edge_v.tolist()))
    want = sorted((e, g) for g in range(G) for e in range(E) if rep[g, e])
    assert edges == want
    assert all(p.edge_u[i] == home[p.edge_e[i]] for i in range(p.n_edges))
    # rounds: rank-disjoint, contiguous, greedy bound 2*Delta-1
    for r in range(p.n_rounds):
        a, b = p.round_ptr[r], p.round_ptr[r + 1]
        ranks = list(p.edge_u[a:b]) + list(p.edge_v[a:b])
        assert len(ranks) == len(set(ranks)) and b > a
        assert (p.edge_round[a:b] == r).all()
    if p.n_edges:
        deg = np.bincount(np.concatenate([p.edge_u, p.edge_v]), minlength=G)
        assert p.n_rounds <= 2 * deg.max() - 1
    # inside a round edges keep edge order (e asc, then v asc)
    for r in range(p.n_rounds):
        a, b = p.round_ptr[r], p.round_ptr[r + 1]
        key = list(zip(p.edge_e[a:b].tolist(), p.edge_v[a:b].tolist()))
        assert key == sorted(key)
    # greedy colouring: each edge's round is the lowest one free at both ends
    # among the rounds given to earlier edges (edge order)
    order = sorted(range(p.n_edges), key=lambda i: (p.edge_e[i], p.edge_v[i]))
    busy = {}
    for i in order:
        u, v = int(p.edge_u[i]), int(p.edge_v[i])
        c = 0
        while (u, c) in busy or (v, c) in busy:
            c += 1
        assert c == p.edge_round[i]
        busy[(u, c)] = busy[(v, c)] = 1


def zipf_counts(rng, G, E, T, k, s=1.2):
    """Random per-rank counts with a Zipf-like skew and exactly T/G*k per rank."""
    pr = rng.permutation(np.arange(1, E + 1)) ** -s
    pr = pr / pr.sum()
    Tg = T // G
    ids = np.empty((T, k), np.int32)
    for t in range(T):
        ids[t] = rng.choice(E, size=k, replace=False, p=pr)
    return ids


def check_plan_invariants_random(o):
    rng = np.random.default_rng(5)
    for G, E, N, L, T, k in ((4, 16, 1, 0, 64, 2), (4, 16, 2, 1, 64, 2), (8, 64, 2, 1, 256, 8),
                             (3, 9, 3, 2, 60, 3), (1, 8, 0, 0, 8, 2), (4, 4, 2, 1, 32, 2)):
        ids = zipf_counts(rng, G, E, T, k)
        cnt = o.count(ids, G, E)
        p = o.plan(cnt, N, L)
        plan_invariants(cnt, p, N, L)


# ----------------------------------------------------------------------------- split

def check_split_golden(o):
    for name in ("split_halving.json", "split_reverse_move.json", "split_star_partition.json"):
        d = golden(name)
        p = golden_plan(o, d)
        cnt = np.array(d["cnt"], np.int32)
        s = o.split(cnt, p, d["passes"])
        assert list(s.tok) == d["tok"], (name, s.tok)
        assert list(s.mass) == d["mass"], (name, s.mass)
        assert list(s.loads) == d["loads"], (name, s.loads)
        assert s.passes_run == d["passes_run"], (name, s.passes_run)
        assert o.split_optimum(cnt, p) == d["optimum"], name


def split_invariants(o, cnt, p, passes=12):
    G, E = cnt.shape
    s = o.split(cnt, p, passes)
    total = int(cnt.sum())
    assert int(s.loads.sum()) == total
    assert ((s.mass >= 0) & (s.mass <= s.tok)).all()
    # tok of each replicated expert sums to its remote mass
    for e in set(p.edge_e.tolist()):
        R = sum(int(cnt[g, e]) for g in range(G) if not p.holds[g, e])
        assert int(s.tok[p.edge_e == e].sum()) == R
        toks = [int(s.tok[i]) for i in sorted(np.nonzero(p.edge_e == e)[0], key=lambda i: p.edge_v[i])]
        assert max(toks) - min(toks) <= 1 and toks == sorted(toks, reverse=True)
    assert s.loads.max() >= -(-total // G)
    opt = o.split_optimum(cnt, p)
    assert opt <= s.loads.max()
    assert opt >= -(-total // G)
    # more passes never raise the max load and never lower the squared sum's decrease
    prev_max, prev_sq = None, None
    for q in range(0, passes + 1):
        sq = o.split(cnt, p, q)
        m, ssq = int(sq.loads.max()), int((sq.loads.astype(np.int64) ** 2).sum())
        if prev_max is not None:
            assert m <= prev_max and ssq <= prev_sq
        prev_max, prev_sq = m, ssq
    return s


def check_split_invariants_random(o):
    rng = np.random.default_rng(9)
    for G, E, N, L, T, k in ((4, 16, 1, 0, 64, 2), (4, 16, 2, 1, 64, 2), (8, 64, 2, 1, 256, 8),
                             (3, 9, 3, 2, 60, 3), (16, 128, 2, 1, 1024, 8)):
        ids = zipf_counts(rng, G, E, T, k)
        cnt = o.count(ids, G, E)
        p = o.plan(cnt, N, L)
        split_invariants(o, cnt, p)


def brute_force_optimum(cnt, p):
    """min over every integer mass vector of max load (tiny instances)."""
    G, E = cnt.shape
    Eg = E // G
    home = np.arange(E) // Eg
    fixed = np.zeros(G, np.int64)
    for i in range(G):
        fixed[i] += sum(int(cnt[i, e]) for e in range(E) if p.holds[i, e])
    R = {e: sum(int(cnt[g, e]) for g in range(G) if not p.holds[g, e]) for e in range(E)}
    rep = {e: sorted(i for i in range(p.n_edges) if p.edge_e[i] == e) for e in range(E)}
    for e in range(E):
        if not rep[e]:
            fixed[home[e]] += R[e]
    tok = {}
    for e, lst in rep.items():
        lst = sorted(lst, key=lambda i: p.edge_v[i])
        for j, i in enumerate(lst):
            tok[i] = R[e] // len(lst) + (1 if j < R[e] % len(lst) else 0)
    best = None
    edges = list(range(p.n_edges))
    for masses in itertools.product(*[range(tok[i] + 1) for i in edges]):
        L = fixed.copy()
        for i, m in zip(edges, masses):
            L[p.edge_u[i]] += m
            L[p.edge_v[i]] += tok[i] - m
        v = int(L.max())
        best = v if best is None else min(best, v)
    return best


def check_optimum_brute_force(o):
    rng = np.random.default_rng(21)
    done = 0
    for trial in range(60):
        G = int(rng.integers(2, 5))
        Eg = int(rng.integers(1, 3))
        E = G * Eg
        k = int(rng.integers(1, min(E, 3) + 1))
        T = G * int(rng.integers(1, 4))
        N = int(rng.integers(1, min(3, E - Eg) + 1)) if E > Eg else 0
        L = int(rng.integers(0, N + 1))
        ids = zipf_counts(rng, G, E, T, k, s=1.5)
        cnt = o.count(ids, G, E)
        p = o.plan(cnt, N, L)
        space = 1
        for e in set(p.edge_e.tolist()):
            space *= (cnt.sum() + 1)
        if p.n_edges > 4:
            continue
        assert o.split_optimum(cnt, p) == brute_force_optimum(cnt, p)
        done += 1
    assert done >= 20


# ----------------------------------------------------------------------------- assign

def check_assign_golden(o):
    d = golden("assign_small.json")
    p = golden_plan(o, d)
    ids = np.array(d["ids"], np.int32)
    cnt = o.count(ids, d["G"], d["E"])
    s = o.split(cnt, p, d["passes"])
    assert list(s.tok) == d["tok"] and list(s.mass) == d["mass"]
    assert list(s.loads) == d["loads"] and s.passes_run == d["passes_run"]
    dest, perm, offs = o.assign(ids, p, s, d["G"], d["E"])
    assert list(dest.ravel()) == d["dest"], dest.ravel()
    assert list(perm) == d["perm"], perm
    assert list(offs) == d["offs"], offs


def assign_invariants(ids, cnt, p, s, dest, perm, offs):
    T, k = ids.shape
    G, E = cnt.shape
    Eg = E // G
    nf = T * k
    flat_e = ids.ravel().astype(np.int64)
    flat_d = dest.ravel().astype(np.int64)
    # every assignment exactly once
    assert np.array_equal(np.sort(perm), np.arange(nf))
    # destination holds the expert
    assert (p.holds[flat_d, flat_e] == 1).all()
    # local tokens stay local
    src = np.repeat(np.arange(T) // (T // G), k) if T else np.zeros(0, np.int64)
    local = p.holds[src, flat_e] == 1
    assert (flat_d[local] == src[local]).all()
    # sorted by key, stable in f
    key = flat_d * E + flat_e
    kp = key[perm]
    assert (np.diff(kp) >= 0).all()
    same = np.diff(kp) == 0
    assert (np.diff(perm)[same] > 0).all()
    # offs is the exclusive scan of bucket sizes
    sizes = np.bincount(key, minlength=G * E)
    assert offs[0] == 0 and offs[-1] == nf
    assert np.array_equal(np.diff(offs), sizes)
    # rank loads equal the split's loads
    assert np.array_equal(sizes.reshape(G, E).sum(1), s.loads)
    # per replica edge: tok - mass tokens of e go to v from non-holders
    for i in range(p.n_edges):
        e, v = int(p.edge_e[i]), int(p.edge_v[i])
        remote_to_v = int(((flat_d == v) & (flat_e == e) & ~local).sum())
        assert remote_to_v == int(s.tok[i] - s.mass[i])


def check_assign_invariants_random(o):
    rng = np.random.default_rng(13)
    for G, E, N, L, T, k in ((4, 16, 1, 0, 64, 2), (4, 16, 2, 1, 64, 2), (8, 64, 2, 1, 256, 8),
                             (3, 9, 3, 2, 60, 3), (16, 128, 2, 1, 1024, 8), (2, 2, 1, 1, 8, 1)):
        ids = zipf_counts(rng, G, E, T, k)
        cnt = o.count(ids, G, E)
        p = o.plan(cnt, N, L)
        s = o.split(cnt, p)
        dest, perm, offs = o.assign(ids, p, s, G, E)
        assign_invariants(ids, cnt, p, s, dest, perm, offs)


# ----------------------------------------------------------------------------- split variants (Relief Table III)

def check_split_variants_golden(o):
    d = golden("split_variants.json")
    for variant, rows in d["expect"].items():
        for fx, (mass, loads, passes_run) in zip(d["fixtures"], rows):
            f = golden(fx)
            s = o.split_variant(np.array(f["cnt"], np.int32), golden_plan(o, f), f["passes"], variant)
            assert s.mass.tolist() == mass, (variant, fx, s.mass.tolist())
            assert s.loads.tolist() == loads, (variant, fx, s.loads.tolist())
            assert s.passes_run == passes_run, (variant, fx, s.passes_run)
            assert s.tok.tolist() == f["tok"], (variant, fx)


def check_split_variants_invariants_random(o):
    """Every variant: the same starting partition as Relief, 0 <= mass <= tok,
    the loads equal the fixed loads plus the masses at home and the rest at
    the replicas, the total is T*k, and max L >= the exact optimum.
    Water-filling with one replicated expert reaches the exact optimum (the
    flow computation, a different method)."""
    rng = np.random.default_rng(17)
    for G, E, N, L, T, k in ((4, 16, 1, 0, 64, 2), (8, 64, 2, 1, 256, 8), (3, 9, 3, 2, 60, 3),
                             (16, 128, 2, 1, 1024, 8)):
        ids = zipf_counts(rng, G, E, T, k)
        cnt = o.count(ids, G, E)
        p = o.plan(cnt, N, L)
        ref = o.split(cnt, p)
        opt = o.split_optimum(cnt, p)
        for variant in o.SPLIT_VARIANTS:
            for passes in (0, 1, 12):
                s = o.split_variant(cnt, p, passes, variant)
                assert np.array_equal(s.tok, ref.tok)
                assert ((s.mass >= 0) & (s.mass <= s.tok)).all()
                loads = np.zeros(G, np.int64)
                for i in range(p.n_edges):
                    loads[p.edge_u[i]] += s.mass[i]
                    loads[p.edge_v[i]] += s.tok[i] - s.mass[i]
                fixed = ref.loads.copy()
                for i in range(p.n_edges):
                    fixed[p.edge_u[i]] -= ref.mass[i]
                    fixed[p.edge_v[i]] -= ref.tok[i] - ref.mass[i]
                assert np.array_equal(loads + fixed, s.loads), (variant, passes)
                assert s.loads.sum() == T * k
                assert s.loads.max() >= opt
    # single replicated expert: water-filling is optimal
    for trial in range(6):
        G, E = 6, 12
        cnt = rng.integers(0, 30, (G, E)).astype(np.int32)
        e0 = int(rng.integers(E))
        h = e0 // (E // G)
        reps = sorted(rng.choice([r for r in range(G) if r != h], size=int(rng.integers(1, 4)), replace=False))
        holds = np.zeros((G, E), np.uint8)
        for e in range(E):
            holds[e // (E // G), e] = 1
        for r in reps:
            holds[r, e0] = 1
        pl = __import__("oracle").plan_from_arrays(G, E, len(reps), 0, holds, [h] * len(reps), list(reps),
                                                   [e0] * len(reps), list(range(len(reps) + 1)))
        s = o.split_variant(cnt, pl, 4, "water")
        assert int(s.loads.max()) == o.split_optimum(cnt, pl), trial


# ----------------------------------------------------------------------------- swaps (FreeBalance sec. 3.3)

def check_swaps_golden(o):
    for name in ("swaps_gamma_budget_tau.json", "swaps_two_ranks.json"):
        d = golden(name)
        for c in d["cases"]:
            r = o.plan_swaps(np.array(d[c.get("cnt", "cnt")]), pi=c.get("pi_in"), gamma=c["gamma"], tau=c["tau"],
                             alpha=c["alpha"], beta=c["beta"], expert_bytes=c["expert_bytes"], budget=c["budget"],
                             link_budget=c.get("link_budget"))
            assert r.swaps.tolist() == c["swaps"], (name, c, r.swaps.tolist())
            assert r.pi.tolist() == c["pi"], (name, c)
            assert r.loads.tolist() == c["loads"], (name, c)


def phi_exact(L, gamma):
    """eq. 8 of FreeBalance sec. 3.3, in exact rational arithmetic, over every
    rank (the definition, not the two-rank update the planner uses)."""
    Lf = [Fraction(int(x)) for x in L]
    mean = sum(Lf) / len(Lf)
    return max(Lf) + Fraction(gamma) * sum((x - mean) ** 2 for x in Lf)


def swaps_invariants(cnt, pi_in, prm, r):
    """Replay a swap plan with exact arithmetic: each accepted swap is between
    the then most- and least-loaded ranks (lowest id on ties), while their
    gap exceeds tau; it lowers Phi; it is the best feasible candidate of that
    frontier by benefit / cost with ties by (a, b); no expert moves twice;
    budgets per rank and per pair hold; the plan stops only when the gap is
    within tau or the frontier has no feasible beneficial candidate; the
    final loads and placement are those the swaps produce."""
    G, E = cnt.shape
    nh = cnt.sum(axis=0).astype(np.int64)
    pi = list(pi_in) if pi_in is not None else [e // (E // G) for e in range(E)]
    gamma, tau = prm["gamma"], Fraction(prm["tau"])
    cost = Fraction(prm["alpha"]) + Fraction(2 * prm["expert_bytes"]) / Fraction(prm["beta"])
    budget = Fraction(prm["budget"])
    link_budget = Fraction(prm.get("link_budget", prm["budget"]))
    spent_rank = [Fraction(0)] * G
    spent_link = {}
    moved = set()

    def loads():
        L = [0] * G
        for e in range(E):
            L[pi[e]] += int(nh[e])
        return L

    def frontier():
        L = loads()
        u = min(range(G), key=lambda x: (-L[x], x))
        v = min(range(G), key=lambda x: (L[x], x))
        return L, u, v

    def candidates(L, u, v):
        out = []
        if not (spent_rank[u] + cost <= budget and spent_rank[v] + cost <= budget and
                spent_link.get((min(u, v), max(u, v)), Fraction(0)) + cost <= link_budget):
            return out
        for a in range(E):
            if pi[a] != u or a in moved:
                continue
            for b in range(E):
                if pi[b] != v or b in moved:
                    continue
                L2 = list(L)
                L2[u] += int(nh[b]) - int(nh[a])
                L2[v] += int(nh[a]) - int(nh[b])
                delta = phi_exact(L, gamma) - phi_exact(L2, gamma)
                if delta > 0:
                    out.append((delta / cost if cost > 0 else delta, a, b))
        return out

    for (u_, v_, a, b) in r.swaps.tolist():
        L, u, v = frontier()
        assert (u_, v_) == (u, v), "swap not on the most/least loaded pair"
        assert Fraction(L[u] - L[v]) > tau, "swap taken although the gap is within tau"
        cands = candidates(L, u, v)
        assert cands, "swap taken with no feasible beneficial candidate"
        best = max(x[0] for x in cands)
        first = min((x for x in cands if x[0] == best), key=lambda x: (x[1], x[2]))
        assert (a, b) == (first[1], first[2]), f"not the best candidate: {(a, b)} vs {first[1:]}"
        assert a not in moved and b not in moved
        pi[a], pi[b] = v, u
        moved.update((a, b))
        spent_rank[u] += cost
        spent_rank[v] += cost
        key = (min(u, v), max(u, v))
        spent_link[key] = spent_link.get(key, Fraction(0)) + cost
    assert all(x <= budget for x in spent_rank) and all(x <= link_budget for x in spent_link.values())
    L, u, v = frontier()
    assert Fraction(L[u] - L[v]) <= tau or not candidates(L, u, v), "planner stopped early"
    assert r.pi.tolist() == pi and r.loads.tolist() == L
    # swaps keep every rank's expert count
    assert np.array_equal(np.bincount(r.pi, minlength=G),
                          np.bincount(np.array(pi_in if pi_in is not None else [e // (E // G) for e in range(E)]),
                                      minlength=G))


def check_swaps_invariants_random(o):
    rng = np.random.default_rng(21)
    for G, E, T, k, prm in ((4, 16, 64, 2, dict(gamma=0.0, tau=0.0, alpha=0.0, beta=1.0, expert_bytes=0.0,
                                                 budget=1e300)),
                            (8, 64, 512, 8, dict(gamma=0.001, tau=0.0, alpha=5.0, beta=2.0, expert_bytes=9.0,
                                                 budget=200.0)),
                            (3, 12, 90, 3, dict(gamma=0.5, tau=4.0, alpha=1.0, beta=1.0, expert_bytes=1.0,
                                                budget=6.0)),
                            (2, 8, 40, 2, dict(gamma=0.25, tau=0.0, alpha=0.0, beta=1.0, expert_bytes=0.0,
                                               budget=1e300)),
                            (16, 128, 1024, 8, dict(gamma=1e-4, tau=2.0, alpha=2.0, beta=4.0, expert_bytes=8.0,
                                                    budget=40.0)),
                            (4, 32, 256, 4, dict(gamma=0.0, tau=0.0, alpha=1.0, beta=1.0, expert_bytes=0.0,
                                                 budget=6.0, link_budget=1.0))):
        for trial in range(3):
            cnt = o.count(zipf_counts(rng, G, E, T, k), G, E)
            pi_in = None if trial == 0 else rng.permutation(np.arange(E) // (E // G)).astype(np.int32)
            r = o.plan_swaps(cnt, pi=pi_in, **prm)
            swaps_invariants(cnt, pi_in, prm, r)


ALL_CHECKS = [
    check_gate_exact_tiny, check_gate_matches_numpy, check_gate_ties, check_gate_cancellation,
    check_count, check_count_rejects,
    check_plan_golden, check_plan_phase1_ties, check_plan_invariants_random,
    check_split_golden, check_split_invariants_random, check_optimum_brute_force,
    check_assign_golden, check_assign_invariants_random,
    check_swaps_golden, check_swaps_invariants_random,
    check_split_variants_golden, check_split_variants_invariants_random,
]
