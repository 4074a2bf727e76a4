"""CUDA path vs the CPU oracle, through the C ABI (needs a B200)."""
import numpy as np
import pytest
import torch

import oracle
import parity
from moe_expert_load_bf16_b200 import _lib, workloads
from moe_expert_load_bf16_b200.pipeline import DecisionPath, StepPipeline

pytestmark = pytest.mark.gpu

DEV = "cuda"
# lb_gate_tuning's persistent values for CTA pairs with H split over 2, 3, 4 pairs
PAIRS_SPLIT_H = {"pairs_split_h2": 5, "pairs_split_h3": 7, "pairs_split_h4": 6}


@pytest.fixture(autouse=True)
def _clean_status():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    _lib.lb_gate_tuning()
    _lib.lb_launch_options(1, 0)
    _lib.lb_get_status(clear=True)
    yield
    _lib.lb_gate_tuning()
    _lib.lb_launch_options(1, 0)


def run_model(w, layers, passes=12, T=None, sample_rows=None):
    hid, W, bias = parity.model_inputs(w, layers, DEV, T=T)
    T = hid.shape[1]
    path = DecisionPath(layers, T, w.H, w.E, w.k, w.G, w.N, w.L, passes=passes, device=DEV)
    path.run(hid[:-1], hid[1:], W, bias)
    torch.cuda.synchronize()
    assert _lib.lb_get_status() == 0
    return hid, W, bias, path


@pytest.mark.parametrize("name", ["tiny", "tiny-p1"])
def test_small_full_path(name):
    w = workloads.WORKLOADS[name]
    hid, W, bias, path = run_model(w, w.layers)
    # gate: every row, both calls, with logits
    for src, ids in ((hid[0], path.ids_pred[0]), (hid[1], path.ids[0])):
        ids2, logits = _lib.lb_predict_topk(src, W[0], bias[0], w.k, want_logits=True)
        assert torch.equal(ids2, ids)
        parity.gate_check(src, W[0], bias[0], w.k, ids, logits)
    parity.check_path(path, 0, 12)


def test_olmoe_all_layers_as_benchmarked():
    """The benchmark's launch configuration: all 16 OLMoE-shaped layers in one
    batched pass, lookahead counts and plan on a side stream, captured in a
    CUDA graph and replayed; gate on sampled rows of every layer, integer
    stages exact."""
    w = workloads.WORKLOADS["olmoe"]
    hid, W, bias = parity.model_inputs(w, w.layers, DEV)
    path = DecisionPath(w.layers, w.T, w.H, w.E, w.k, w.G, w.N, w.L, device=DEV)
    side = torch.cuda.Stream()
    path.run(hid[:-1], hid[1:], W, bias, side_stream=side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        path.run(hid[:-1], hid[1:], W, bias, side_stream=side)
    path.dest.fill_(-1)
    path.perm.fill_(-1)
    g.replay()
    torch.cuda.synchronize()
    assert _lib.lb_get_status() == 0
    rng = np.random.default_rng(0)
    for l in range(w.layers):
        rows = np.concatenate([rng.choice(w.T, 48, replace=False), [0, w.T - 1]])
        parity.gate_check(hid[l + 1], W[l], bias[l], w.k, path.ids[l], rows=rows)
        parity.gate_check(hid[l], W[l], bias[l], w.k, path.ids_pred[l], rows=rows)
        parity.check_path(path, l, 12)


def test_olmoe_one_layer_all_rows_with_logits():
    w = workloads.WORKLOADS["olmoe"]
    hid, W, bias = parity.model_inputs(w, 1, DEV)
    ids, logits = _lib.lb_predict_topk(hid[1], W[0], bias[0], w.k, want_logits=True)
    err, mism = parity.gate_check(hid[1], W[0], bias[0], w.k, ids, logits)
    assert mism <= 8


@pytest.mark.parametrize("name,layers", [("qwen3-30b", 2), ("qwen3-235b", 1)])
def test_large_configs(name, layers):
    w = workloads.WORKLOADS[name]
    hid, W, bias, path = run_model(w, layers)
    rng = np.random.default_rng(1)
    rows = np.concatenate([rng.choice(w.T, 96, replace=False), [0, w.T - 1]])
    for l in range(layers):
        # one problem alone may take the cluster split of H (another fp32
        # summation order than the batched call), so each is held to the oracle
        ids, logits = _lib.lb_predict_topk(hid[l + 1], W[l], bias[l], w.k, want_logits=True)
        parity.gate_check(hid[l + 1], W[l], bias[l], w.k, ids, logits, rows=rows)
        parity.gate_check(hid[l + 1], W[l], bias[l], w.k, path.ids[l], rows=rows)
        assert (ids == path.ids[l]).float().mean().item() > 0.999
        parity.check_path(path, l, 12)


@pytest.mark.parametrize("T", [64, 256, 1024, 4096, 8192])
def test_decode_steps(T):
    """Decode sweep shape: plan from step 0, split + assign for several steps."""
    w = workloads.WORKLOADS["decode"]
    steps = [0, 1, 2, 3]
    ids = workloads.decode_ids(w, T, steps).to(DEV)
    path = DecisionPath(len(steps), T, w.H, w.E, w.k, w.G, w.N, w.L, device=DEV)
    cnt0 = _lib.lb_count(ids[0], w.G, w.E)
    _lib.lb_plan_replicas(cnt0, w.N, w.L, plan=path.plan[0:1])
    path.plan[1:].copy_(path.plan[0:1].expand(len(steps) - 1, -1))
    path.ids.copy_(ids)
    path.ids_pred.copy_(ids[0:1].expand(len(steps), -1, -1))
    path.cnt_pred.copy_(cnt0.unsqueeze(0).expand(len(steps), -1, -1))
    path.solve()
    torch.cuda.synchronize()
    assert _lib.lb_get_status() == 0
    for b in range(len(steps)):
        parity.check_path(path, b, 12)


@pytest.mark.parametrize("B", [2, 3])
def test_decode_few_problems_per_launch(B):
    """A few decode-shaped problems in one launch: the assign's prep runs one
    cluster of 8 CTAs per problem, and the scatter one CTA per source block
    of every problem while they fit one wave (B = 2: 128 CTAs) or one warp
    per block once they do not (B = 3: 192 blocks); separate and fused forms
    agree, and every problem passes the oracle check."""
    w = workloads.WORKLOADS["decode"]
    T = 1024
    ids = workloads.decode_ids(w.with_(T=T), T, range(B + 1)).to(DEV)
    path = DecisionPath(B, T, w.H, w.E, w.k, w.G, w.N, w.L, device=DEV)
    cnt0 = _lib.lb_count(ids[0], w.G, w.E)
    _lib.lb_plan_replicas(cnt0, w.N, w.L, plan=path.plan[0:1])
    path.plan[1:].copy_(path.plan[0:1].expand(B - 1, -1))
    path.ids.copy_(ids[1:])
    path.ids_pred.copy_(ids[0:1].expand(B, -1, -1))
    path.cnt_pred.copy_(cnt0.unsqueeze(0).expand(B, -1, -1))
    path.solve()
    torch.cuda.synchronize()
    assert _lib.lb_get_status() == 0
    for b in range(B):
        parity.check_path(path, b, 12)
    sep = [t.clone() for t in (path.dest, path.perm, path.offs)]
    path.solve_separate()
    torch.cuda.synchronize()
    assert _lib.lb_get_status() == 0
    for a, c in zip(sep, (path.dest, path.perm, path.offs)):
        assert torch.equal(a, c)


@pytest.mark.parametrize("mode", ["auto", "pairs_split_h2", "pairs_split_h3", "pairs_split_h4"])
@pytest.mark.parametrize("T", [64, 1024, 4096, 8192])
def test_decode_gate(T, mode):
    """Gate at the decode shape (H=7168, E=256): the automatic choice, and
    CTA pairs with H split over two, three or four pairs (partials summed by
    a reduce-scatter over distributed shared memory)."""
    if mode != "auto":
        _lib.lb_gate_tuning(0, 0, PAIRS_SPLIT_H[mode])
    w = workloads.WORKLOADS["decode"]
    h = workloads.hidden_chain(w, 1, device=DEV, T=T)[0]
    W = workloads.gate_weights(w, 1, device=DEV)[0]
    bias = workloads.biases(w, 1)[0].to(DEV)
    ids, logits = _lib.lb_predict_topk(h, W, bias, w.k, want_logits=True)
    rows = np.arange(T) if T <= 256 else np.random.default_rng(2).choice(T, 128, replace=False)
    parity.gate_check(h, W, bias, w.k, ids, logits, rows=rows)


@pytest.mark.parametrize("mode", ["auto", "pairs_split_h2", "pairs_split_h3", "pairs_split_h4"])
@pytest.mark.parametrize("T", [200, 1024, 4100])
def test_gate_pairs_batched(T, mode):
    """CTA pairs with a split of H on a batch of three independent problems
    (the grid's second dimension; the automatic choice counts the units of
    the whole batch), E=256, H=2048, a ragged last unit at T=200 and 4100,
    every row against the oracle with logits."""
    if mode != "auto":
        _lib.lb_gate_tuning(0, 0, PAIRS_SPLIT_H[mode])
    B, H, E, k = 3, 2048, 256, 8
    g = torch.Generator(device=DEV).manual_seed(T + 17 * len(mode))
    h = torch.randn(B, T, H, generator=g, device=DEV).to(torch.bfloat16)
    W = (torch.randn(B, E, H, generator=g, device=DEV) / H ** 0.5).to(torch.bfloat16)
    bias = 0.1 * torch.randn(B, E, generator=g, device=DEV)
    ids, logits = _lib.lb_predict_topk(h, W, bias, k, want_logits=True)
    assert _lib.lb_get_status() == 0
    rows = np.arange(T) if T <= 1024 else np.random.default_rng(3).choice(T, 256, replace=False)
    for b in range(B):
        parity.gate_check(h[b], W[b], bias[b], k, ids[b], logits[b], rows=rows)


@pytest.mark.parametrize("T,H,E,k", [(200, 72, 60, 5), (1, 8, 16, 1), (333, 128, 256, 16), (130, 64, 17, 3),
                                     (4096, 256, 128, 8), (96, 2048, 32, 2), (300, 320, 80, 4)])
@pytest.mark.parametrize("split", [0, 1, 2, 4, -2, -4, -8, "persistent", "pairs_split_h2", "pairs_split_h3",
                                   "pairs_split_h4"])
def test_gate_shapes(T, H, E, k, split):
    """Ragged token tails, E not a multiple of 16, H not a multiple of 64,
    tiny and maximum k, every split of H, every split of N across a cluster
    (negative values), and the persistent kernel."""
    nkb = (H + 63) // 64
    Epad = (E + 15) // 16 * 16
    if split == "persistent":
        _lib.lb_gate_tuning(0, 0, 1)
    elif split in PAIRS_SPLIT_H:
        ks = int(split[-1])
        if k > 8 or (ks - 1) * ((nkb + ks - 1) // ks) >= nkb:
            pytest.skip("CTA pairs with a split of H take k <= 8 and a k-block of H for every pair")
        _lib.lb_gate_tuning(0, 0, PAIRS_SPLIT_H[split])
    else:
        if split > nkb or (split > 0 and Epad % (4 * split) != 0):
            pytest.skip("split of H not valid for this shape")
        if split < 0 and (Epad % (16 * -split) != 0 or Epad // -split < 16):
            pytest.skip("split of N not valid for this shape")
        _lib.lb_gate_tuning(0, split, -1)
    g = torch.Generator(device=DEV).manual_seed(T * 7 + H + E + k)
    h = torch.randn(T, H, generator=g, device=DEV).to(torch.bfloat16)
    W = (torch.randn(E, H, generator=g, device=DEV) / H ** 0.5).to(torch.bfloat16)
    bias = torch.randn(E, generator=g, device=DEV)
    ids, logits = _lib.lb_predict_topk(h, W, bias, k, want_logits=True)
    parity.gate_check(h, W, bias, k, ids, logits)
    ids0 = _lib.lb_predict_topk(h, W, None, k)
    parity.gate_check(h, W, None, k, ids0)


@pytest.mark.parametrize("split", [2, 4, 8, 16])
def test_gate_split_cluster(split):
    """Forced split of H across clusters of 2..16 CTAs."""
    _lib.lb_gate_tuning(0, split, -1)
    T, H, E, k = 300, 4096, 256, 8
    g = torch.Generator(device=DEV).manual_seed(split)
    h = torch.randn(T, H, generator=g, device=DEV).to(torch.bfloat16)
    W = (torch.randn(E, H, generator=g, device=DEV) / H ** 0.5).to(torch.bfloat16)
    ids, logits = _lib.lb_predict_topk(h, W, None, k, want_logits=True)
    parity.gate_check(h, W, None, k, ids, logits)


@pytest.mark.parametrize("persistent", [-1, 1])
@pytest.mark.parametrize("stages", [2, 3, 5, 8])
def test_gate_stages(stages, persistent):
    _lib.lb_gate_tuning(stages, 1 if persistent < 0 else 0, persistent, 1)
    T, H, E, k = 512, 1024, 64, 8
    g = torch.Generator(device=DEV).manual_seed(stages)
    h = torch.randn(T, H, generator=g, device=DEV).to(torch.bfloat16)
    W = (torch.randn(E, H, generator=g, device=DEV) / H ** 0.5).to(torch.bfloat16)
    ids, logits = _lib.lb_predict_topk(h, W, None, k, want_logits=True)
    parity.gate_check(h, W, None, k, ids, logits)


def test_gate_ties_lower_id():
    """Exactly equal logits: lower expert id first (identical weight rows)."""
    T, H, E, k = 256, 128, 32, 6
    g = torch.Generator(device=DEV).manual_seed(5)
    h = torch.randn(T, H, generator=g, device=DEV).to(torch.bfloat16)
    W = (torch.randn(E, H, generator=g, device=DEV) / H ** 0.5).to(torch.bfloat16)
    W[7] = W[3]
    W[20] = W[3]
    W[9] = W[1]
    ids, logits = _lib.lb_predict_topk(h, W, None, k, want_logits=True)
    # every row within the logit tolerance (ids differ only between near-ties)
    parity.gate_check(h, W, None, k, ids, logits)
    _, o_ids = oracle.gate(workloads.bf16_bits(h), workloads.bf16_bits(W), None, k)
    got = ids.cpu().numpy()
    lg = logits.cpu().numpy()
    for r in range(T):
        row = list(got[r])
        # duplicated rows give bit-identical logits: the lower id ranks first
        for lo, hi in ((3, 7), (3, 20), (7, 20), (1, 9)):
            assert lg[r, lo] == lg[r, hi]
            if lo in row and hi in row:
                assert row.index(lo) < row.index(hi)
            if hi in row:
                assert lo in row
        # rows without a near-tie among the kept ids equal the oracle's exactly
        kth = np.sort(lg[r])[::-1]
        gaps = np.abs(np.diff(kth[:k + 1]))
        if (gaps[gaps > 0] > 1e-3 * max(abs(kth[k - 1]), 1.0)).all():
            assert np.array_equal(got[r], o_ids[r]), r


def test_integer_stages_random_shapes():
    rng = np.random.default_rng(3)
    for trial in range(12):
        G = int(rng.choice([1, 2, 3, 4, 8, 16, 64]))
        Eg = int(rng.choice([1, 2, 4, 8]))
        E = G * Eg
        if E > 512:
            continue
        k = int(rng.integers(1, min(E, 8) + 1))
        T = G * int(rng.integers(0, 40))
        N = int(rng.integers(0, min(4, E - Eg) + 1))
        L = int(rng.integers(0, N + 1))
        pr = rng.permutation(np.arange(1, E + 1)) ** -1.3
        pr /= pr.sum()
        ids_np = np.stack([rng.choice(E, k, replace=False, p=pr) for _ in range(T)]).astype(np.int32) \
            if T else np.zeros((0, k), np.int32)
        ids = torch.from_numpy(ids_np).to(DEV)
        B = 2
        path = DecisionPath(B, T, 8, E, k, G, N, L, device=DEV)
        path.ids.copy_(ids.unsqueeze(0).expand(B, -1, -1))
        # problem 1 plans on counts of a shuffled copy: different prediction
        shuffled = ids_np[rng.permutation(T)] if T else ids_np
        path.ids_pred[0].copy_(ids)
        path.ids_pred[1].copy_(torch.from_numpy(np.ascontiguousarray(shuffled)).to(DEV))
        _lib.lb_count(path.ids_pred, G, E, cnt=path.cnt_pred)
        _lib.lb_plan_replicas(path.cnt_pred, N, L, plan=path.plan)
        path.solve()
        torch.cuda.synchronize()
        assert _lib.lb_get_status() == 0
        for b in range(B):
            parity.check_path(path, b, 12)


@pytest.mark.parametrize("passes", [0, 1, 2, 64])
def test_split_pass_counts(passes):
    w = workloads.WORKLOADS["qwen3-30b"]
    ids = workloads.decode_ids(w.with_(T=2048), 2048, [0]).to(DEV)[0]
    path = DecisionPath(1, 2048, 8, w.E, w.k, w.G, w.N, w.L, passes=passes, device=DEV)
    path.ids_pred.copy_(ids)
    path.ids.copy_(ids)
    _lib.lb_count(path.ids_pred, w.G, w.E, cnt=path.cnt_pred)
    _lib.lb_plan_replicas(path.cnt_pred, w.N, w.L, plan=path.plan)
    path.solve()
    torch.cuda.synchronize()
    parity.check_path(path, 0, passes)


def test_all_tokens_one_expert():
    G, E, k, T, N, L = 8, 64, 1, 1024, 4, 2
    ids = torch.zeros(T, k, dtype=torch.int32, device=DEV)
    path = DecisionPath(1, T, 8, E, k, G, N, L, device=DEV)
    path.ids_pred.copy_(ids)
    path.ids.copy_(ids)
    _lib.lb_count(path.ids_pred, G, E, cnt=path.cnt_pred)
    _lib.lb_plan_replicas(path.cnt_pred, N, L, plan=path.plan)
    path.solve()
    torch.cuda.synchronize()
    p, s = parity.check_path(path, 0, 12)
    assert int(s.loads.max()) == oracle.split_optimum(path.cnt[0].cpu().numpy(), p)


def test_empty_batch():
    G, E, k, N, L = 4, 16, 2, 1, 0
    path = DecisionPath(1, 0, 8, E, k, G, N, L, device=DEV)
    _lib.lb_count(path.ids_pred, G, E, cnt=path.cnt_pred)
    _lib.lb_plan_replicas(path.cnt_pred, N, L, plan=path.plan)
    path.solve()
    torch.cuda.synchronize()
    assert (path.cnt == 0).all() and (path.offs == 0).all()
    parity.check_path(path, 0, 12)


def test_bad_ids_are_flagged_not_fatal():
    G, E, k, T = 4, 16, 2, 64
    ids = torch.randint(0, E, (T, k), dtype=torch.int32, device=DEV)
    ids[:, 1] = (ids[:, 0] + 1) % E
    ids[5, 0] = E + 3           # out of range
    ids[9, 1] = ids[9, 0]       # repeated in a row
    _lib.lb_count(ids, G, E)
    flags = _lib.lb_get_status(clear=True)
    assert flags & _lib.LB_DEV_BAD_IDS
    # the context is still usable
    ok = torch.ones(4, device=DEV).sum().item()
    assert ok == 4.0


def test_invalid_arguments_rejected():
    h = torch.zeros(128, 64, dtype=torch.bfloat16, device=DEV)
    W = torch.zeros(300, 64, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(_lib.LBError) as e:
        _lib.lb_predict_topk(h, W, None, 8)       # E > 256
    assert e.value.code == _lib.LB_EINVAL
    ids = torch.zeros(10, 2, dtype=torch.int32, device=DEV)
    with pytest.raises(_lib.LBError):
        _lib.lb_count(ids, 4, 16)                 # T % G != 0
    cnt = torch.zeros(3, 16, dtype=torch.int32, device=DEV)
    with pytest.raises(_lib.LBError):
        _lib.lb_plan_replicas(cnt, 1, 0)          # E % G != 0
    assert _lib.lb_get_status() == 0


def test_batched_equals_unbatched():
    w = workloads.WORKLOADS["tiny-p1"].with_(layers=3)
    hid, W, bias = parity.model_inputs(w, 3, DEV)
    ids_b = _lib.lb_predict_topk(hid[1:], W, bias, w.k)
    for l in range(3):
        assert torch.equal(ids_b[l], _lib.lb_predict_topk(hid[l + 1], W[l], bias[l], w.k))
    cnt_b = _lib.lb_count(ids_b, w.G, w.E)
    plan_b = _lib.lb_plan_replicas(cnt_b, w.N, w.L)
    for l in range(3):
        assert torch.equal(cnt_b[l], _lib.lb_count(ids_b[l], w.G, w.E))
        assert torch.equal(plan_b[l], _lib.lb_plan_replicas(cnt_b[l], w.N, w.L)[0])


def test_split_long_schedule_falls_back():
    """A schedule longer than the per-(round, rank) table (every token asks
    for rank 0's experts, so rank 0 gets hundreds of replica edges): the
    shared-memory pass loop runs instead, with the same results."""
    G, E, k, N, L = 64, 320, 5, 16, 8
    T = G * 16
    ids = torch.arange(k, dtype=torch.int32, device=DEV).repeat(T, 1)
    path = DecisionPath(1, T, 8, E, k, G, N, L, device=DEV)
    path.ids_pred.copy_(ids)
    path.ids.copy_(ids)
    _lib.lb_count(path.ids_pred, G, E, cnt=path.cnt_pred)
    _lib.lb_plan_replicas(path.cnt_pred, N, L, plan=path.plan)
    path.solve()
    torch.cuda.synchronize()
    assert _lib.lb_get_status() == 0
    dec = _lib.decode_plan(path.plan[0], G, E, N)[0]
    assert dec["n_rounds"] > 256
    parity.check_path(path, 0, 12)


@pytest.mark.parametrize("persistent,kbox", [(-1, 0), (1, 1), (2, 1), (2, 2), (4, 1), (2, 4)])
def test_gate_persistent_many_tiles_batched(persistent, kbox):
    """Many tiles over several problems (more tiles than SMs, ragged last
    tile per problem): persistent and one-CTA-per-tile kernels both match
    the oracle on sampled rows of every problem."""
    _lib.lb_gate_tuning(0, 0, persistent, kbox)
    B, T, H, E, k = 5, 4000, 576, 64, 8   # H: 9 boxes, so a stage of 2 or 4 boxes runs past H
    g = torch.Generator(device=DEV).manual_seed(11)
    h = torch.randn(B, T, H, generator=g, device=DEV).to(torch.bfloat16)
    W = (torch.randn(B, E, H, generator=g, device=DEV) / H ** 0.5).to(torch.bfloat16)
    bias = torch.randn(B, E, generator=g, device=DEV)
    ids, logits = _lib.lb_predict_topk(h, W, bias, k, want_logits=True)
    rng = np.random.default_rng(4)
    for b in range(B):
        rows = np.concatenate([rng.choice(T, 64, replace=False), [0, 127, 128, T - 1]])
        parity.gate_check(h[b], W[b], bias[b], k, ids[b], logits[b], rows=rows)


@pytest.mark.parametrize("name,T,B", [("olmoe", 4096, 2), ("qwen3-235b", 32768, 1), ("qwen3-30b", 16384, 1),
                                      ("decode", 8192, 2), ("decode", 1024, 2), ("decode", 64, 3),
                                      ("tiny-p1", 256, 2), ("tiny", 0, 1)])
def test_solve_fused_equals_separate_calls(name, T, B):
    """lb_solve (one cluster launch: counts, split, permutation) gives the
    same bytes as lb_count + lb_split + lb_assign, whatever the cluster layout
    (several source blocks per CTA, parts of one block per CTA, one CTA)."""
    w = workloads.WORKLOADS[name]
    steps = list(range(B + 1))
    ids = workloads.decode_ids(w.with_(T=max(T, 1)), max(T, 1), steps).to(DEV)[:, :T]
    path = DecisionPath(B, T, 8, w.E, w.k, w.G, w.N, w.L, device=DEV)
    path.ids_pred.copy_(ids[0:1].expand(B, -1, -1))
    path.ids.copy_(ids[1:])
    _lib.lb_count(path.ids_pred, w.G, w.E, cnt=path.cnt_pred)
    _lib.lb_plan_replicas(path.cnt_pred, w.N, w.L, plan=path.plan)
    path.solve_fused()
    fused = [t.clone() for t in (path.cnt, path.tok, path.mass, path.loads, path.passes_run, path.dest, path.perm,
                                 path.offs)]
    path.solve()
    torch.cuda.synchronize()
    assert _lib.lb_get_status() == 0
    for f, s in zip(fused, (path.cnt, path.tok, path.mass, path.loads, path.passes_run, path.dest, path.perm,
                            path.offs)):
        assert torch.equal(f, s)
    for b in range(B):
        parity.check_path(path, b, 12)


@pytest.mark.parametrize("name,T,B", [("tiny", 256, 3), ("olmoe", 4096, 4), ("qwen3-235b", 8192, 3),
                                      ("decode", 1024, 5), ("decode", 64, 2), ("olmoe", 0, 2), ("decode", 0, 1)])
def test_decide_equals_separate_calls(name, T, B):
    """lb_decide (plan, split and the assign's tables in one launch per
    problem, then the scatter) gives the bytes of lb_plan_replicas + lb_split
    + lb_assign, with the plan computed from predicted counts and with the
    plan given; the result passes the oracle check.  Distinct predicted
    counts per problem, so a plan read from the wrong problem fails."""
    w = workloads.WORKLOADS[name]
    Tg = max(T, w.G)
    ids = workloads.decode_ids(w.with_(T=Tg), Tg, range(2 * B)).to(DEV)[:, :T]
    a = DecisionPath(B, T, 8, w.E, w.k, w.G, w.N, w.L, device=DEV)
    b = DecisionPath(B, T, 8, w.E, w.k, w.G, w.N, w.L, device=DEV)
    for p in (a, b):
        p.ids_pred.copy_(ids[:B])
        p.ids.copy_(ids[B:])
        p.count_chain()
    # separate calls
    _lib.lb_plan_replicas(a.cnt_pred, w.N, w.L, plan=a.plan)
    a.solve_separate(counted=True)
    # plan + split + tables in one launch
    b.plan.fill_(0x5a)
    b.decide(with_plan=True)
    torch.cuda.synchronize()
    assert _lib.lb_get_status() == 0
    for f in ("plan", "tok", "mass", "loads", "passes_run", "dest", "perm", "offs"):
        assert torch.equal(getattr(a, f), getattr(b, f)), f
    # plan given
    for t in (b.tok, b.mass, b.loads, b.passes_run, b.dest, b.perm, b.offs):
        t.fill_(-7)
    b.solve(counted=True)
    torch.cuda.synchronize()
    assert _lib.lb_get_status() == 0
    for f in ("plan", "tok", "mass", "loads", "passes_run", "dest", "perm", "offs"):
        assert torch.equal(getattr(a, f), getattr(b, f)), f
    for i in range(B):
        parity.check_path(b, i, 12)


@pytest.mark.parametrize("L,T,H,E,k,bias_on", [(3, 200, 128, 16, 2, True), (1, 256, 64, 16, 4, True),
                                               (4, 4096, 2048, 64, 8, True), (2, 1100, 2048, 128, 8, True),
                                               (5, 3000, 576, 64, 8, False), (2, 130, 8, 32, 16, True)])
def test_gate_chain(L, T, H, E, k, bias_on):
    """lb_predict_topk_chain: for every layer l, the lookahead ids from
    hid[l] and the normal-router ids from hid[l+1] (with gate W_l) pass the
    oracle check and agree with lb_predict_topk on the same rows.  Distinct
    hidden states, so reading the wrong one (or the wrong layer's gate) fails.
    Shapes: ragged last tile, one layer (both boundary states), E = 128 (one
    CTA per SM), a stage of boxes past H, no bias, H = 8."""
    g = torch.Generator(device=DEV).manual_seed(100 + L * 7 + E)
    hid = torch.randn(L + 1, T, H, generator=g, device=DEV).to(torch.bfloat16)
    W = (torch.randn(L, E, H, generator=g, device=DEV) / H ** 0.5).to(torch.bfloat16)
    bias = torch.randn(L, E, generator=g, device=DEV) if bias_on else None
    ip, ia, lp, la = _lib.lb_predict_topk_chain(hid, W, bias, k, want_logits=True)
    torch.cuda.synchronize()
    assert _lib.lb_get_status() == 0
    rng = np.random.default_rng(L + T)
    rows = None if T <= 256 else np.unique(np.concatenate([rng.choice(T, 96, replace=False),
                                                           [0, 127, 128, T - 1]]))
    for l in range(L):
        bl = None if bias is None else bias[l]
        for src, ids, lg in ((hid[l], ip[l], lp[l]), (hid[l + 1], ia[l], la[l])):
            parity.gate_check(src, W[l], bl, k, ids, lg, rows=rows)
            ids1, lg1 = _lib.lb_predict_topk(src, W[l], bl, k, want_logits=True)
            assert torch.allclose(lg, lg1, rtol=1e-5, atol=1e-5)
            assert (ids == ids1).all(dim=1).float().mean().item() > 0.999


def test_gate_chain_drives_the_path():
    """DecisionPath.run_chain (one gate pass per hidden state, both id sets
    counted in one launch) gives the same bytes downstream as run() on the
    same hidden chain, when the gates agree."""
    w = workloads.WORKLOADS["olmoe"]
    hid, W, bias = parity.model_inputs(w, 4, DEV)
    hid[0].copy_((hid[0].float() * 0.9).to(torch.bfloat16))   # a distinct h_0
    a = DecisionPath(4, w.T, w.H, w.E, w.k, w.G, w.N, w.L, device=DEV)
    b = DecisionPath(4, w.T, w.H, w.E, w.k, w.G, w.N, w.L, device=DEV)
    a.run_chain(hid, W, bias)
    b.run(hid[:-1], hid[1:], W, bias)
    torch.cuda.synchronize()
    assert _lib.lb_get_status() == 0
    if torch.equal(a.ids_both, b.ids_both):
        for f in ("cnt_both", "plan", "tok", "mass", "loads", "passes_run", "dest", "perm", "offs"):
            assert torch.equal(getattr(a, f), getattr(b, f)), f
    for l in range(4):
        parity.check_path(a, l, 12)


@pytest.mark.parametrize("graph", [False, True])
def test_programmatic_launch_is_invisible(graph):
    """The chained path launched with programmatic dependent launch (each
    kernel may be scheduled while its predecessor runs, and waits for it
    before touching memory) gives the same bytes as plain stream order, run
    back to back several times on one stream (each run's kernels overwrite
    buffers the previous run's later kernels read), eagerly and replayed from
    a CUDA graph; and the result passes the oracle check."""
    w = workloads.WORKLOADS["olmoe"]
    hid, W, bias = parity.model_inputs(w, 4, DEV)
    hid2 = hid.flip(0).contiguous()
    outs = []
    for pdl in (0, 1):
        _lib.lb_launch_options(pdl, 0)
        p = DecisionPath(4, w.T, w.H, w.E, w.k, w.G, w.N, w.L, device=DEV)
        if graph:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                p.run_chain(hid2, W, bias)
                p.run_chain(hid, W, bias)
            for _ in range(3):
                g.replay()
        else:
            for _ in range(3):
                p.run_chain(hid2, W, bias)
                p.run_chain(hid, W, bias)
        torch.cuda.synchronize()
        assert _lib.lb_get_status() == 0
        outs.append(p)
    a, b = outs
    for f in ("ids_both", "cnt_both", "plan", "tok", "mass", "loads", "passes_run", "dest", "perm", "offs"):
        assert torch.equal(getattr(a, f), getattr(b, f)), f
    for l in range(4):
        parity.check_path(b, l, 12)


@pytest.mark.parametrize("graph", [False, True])
@pytest.mark.parametrize("separate", [False, True])
def test_programmatic_launch_prep_to_scatter(graph, separate):
    """The decode-shaped path runs the split, the prep (a cluster of 8 CTAs)
    and the scatter as separate launches, through lb_decide or through
    lb_split + lb_assign.  With programmatic dependent launch the prep lets
    the scatter start while it runs, and the scatter builds its tables from
    the counts, plan and split before waiting on the prep.  Two steps run
    back to back on one set of buffers, each step's count, split and prep
    overwriting what the previous step's scatter read, eagerly and replayed
    from a CUDA graph.  The bytes are the same with and without programmatic
    launch, and they pass the oracle check."""
    w = workloads.WORKLOADS["decode"]
    T = 1024
    ids = workloads.decode_ids(w.with_(T=T), T, [0, 1, 2]).to(DEV)
    outs = []
    try:
        for pdl in (0, 1):
            _lib.lb_launch_options(pdl, 0)
            p = DecisionPath(1, T, w.H, w.E, w.k, w.G, w.N, w.L, device=DEV)
            p.ids_pred.copy_(ids[0:1])
            _lib.lb_count(p.ids_pred, w.G, w.E, cnt=p.cnt_pred)
            _lib.lb_plan_replicas(p.cnt_pred, w.N, w.L, plan=p.plan)
            step = p.solve_separate if separate else p.solve

            def two_steps():
                p.ids.copy_(ids[1:2])
                step()
                p.ids.copy_(ids[2:3])
                step()
            if graph:
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    two_steps()
                for _ in range(3):
                    g.replay()
            else:
                for _ in range(3):
                    two_steps()
            torch.cuda.synchronize()
            assert _lib.lb_get_status() == 0
            outs.append(p)
    finally:
        _lib.lb_launch_options(1, 0)
    a, b = outs
    for f in ("cnt", "tok", "mass", "loads", "passes_run", "dest", "perm", "offs"):
        assert torch.equal(getattr(a, f), getattr(b, f)), f
    parity.check_path(b, 0, 12)


@pytest.mark.parametrize("graph,narrow", [(False, False), (True, False), (True, True)])
def test_step_pipeline_equals_serial(graph, narrow):
    """Two steps in flight (the gate of step i+1 on one stream beside the
    integer stages of step i on another, buffers alternating): after five
    steps on alternating inputs both buffer sets hold exactly what a serial
    pass over their last inputs gives (a buffer reused before its previous
    step's integer stages finished would differ), eagerly and as one CUDA
    graph, also with 512-thread integer blocks and a capped gate grid."""
    w = workloads.WORKLOADS["olmoe"]
    hid, W, bias = parity.model_inputs(w, 4, DEV)
    hid2 = hid.flip(0).contiguous()
    if narrow:
        _lib.lb_launch_options(1, 512)
        _lib.lb_gate_tuning(0, 0, 0, 0, 0, 272)
    pipe = StepPipeline(4, w.T, w.H, w.E, w.k, w.G, w.N, w.L, device=DEV)

    def five():
        for i in range(5):
            pipe.run(1, hid if i % 2 == 0 else hid2, W, bias)   # one step per call: buffer 0 each time
        pipe.run(2, hid2, W, bias)                              # buffers 0 and 1
        pipe.run(3, hid, W, bias)                               # buffers 0, 1, 0

    if graph:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            five()
        g.replay()
        g.replay()
    else:
        five()
    torch.cuda.synchronize()
    assert _lib.lb_get_status() == 0
    ref = DecisionPath(4, w.T, w.H, w.E, w.k, w.G, w.N, w.L, device=DEV)
    ref.run_chain(hid, W, bias)
    torch.cuda.synchronize()
    for p in pipe.paths:
        for f in ("ids_both", "cnt_both", "plan", "tok", "mass", "loads", "passes_run", "dest", "perm", "offs"):
            assert torch.equal(getattr(p, f), getattr(ref, f)), f
    for l in range(4):
        parity.check_path(pipe.paths[0], l, 12)


@pytest.mark.parametrize("E,L", [(256, 2), (24, 2), (64, 0)])
def test_gate_chain_rejects_unsupported_shapes(E, L):
    hid = torch.zeros(L + 1, 128, 64, dtype=torch.bfloat16, device=DEV)
    W = torch.zeros(max(L, 1), E, 64, dtype=torch.bfloat16, device=DEV)[:L]
    with pytest.raises((_lib.LBError, ValueError)):
        _lib.lb_predict_topk_chain(hid, W, None, 2)


@pytest.mark.parametrize("name,T,B", [("qwen3-235b", 8192, 40), ("decode", 1024, 80)])
def test_assign_throughput_launch_equals_single(name, T, B):
    """Enough problems to fill the GPU twice over switch the scatter to
    512-thread CTAs (two per SM), in CTA mode (large source blocks) and in
    warp mode (small blocks); the bytes equal one-problem calls (1024-thread
    CTAs for large blocks, one CTA per small block) and pass the oracle
    check."""
    w = workloads.WORKLOADS[name]
    ids = workloads.decode_ids(w.with_(T=T), T, range(B + 1)).to(DEV)
    path = DecisionPath(B, T, 8, w.E, w.k, w.G, w.N, w.L, device=DEV)
    path.ids_pred.copy_(ids[0:1].expand(B, -1, -1))
    path.ids.copy_(ids[1:])
    _lib.lb_count(path.ids_pred, w.G, w.E, cnt=path.cnt_pred)
    _lib.lb_plan_replicas(path.cnt_pred, w.N, w.L, plan=path.plan)
    path.solve()
    torch.cuda.synchronize()
    assert _lib.lb_get_status() == 0
    for b in (0, B // 2, B - 1):
        one = DecisionPath(1, T, 8, w.E, w.k, w.G, w.N, w.L, device=DEV)
        one.ids.copy_(path.ids[b:b + 1])
        one.plan.copy_(path.plan[b:b + 1])
        one.solve()
        torch.cuda.synchronize()
        for f in ("cnt", "tok", "mass", "loads", "dest", "perm", "offs"):
            assert torch.equal(getattr(one, f)[0], getattr(path, f)[b]), (f, b)
    for b in (0, B - 1):
        parity.check_path(path, b, 12)


@pytest.mark.parametrize("k", [1, 2, 3, 4, 5, 8, 9])
def test_scatter_large_blocks_every_k(k):
    """Source blocks larger than one warp's share (the whole-CTA scatter):
    every top-k width through its path (token-wise for k <= 8, with and
    without 16-byte rows; assignment-wise above), fused and separate, against
    the oracle."""
    rng = np.random.default_rng(40 + k)
    G, E, N, L = 4, 32, 3, 1
    T = G * (2600 // k + 37)             # > 2048 assignments per block, ragged against the chunks
    pr = rng.permutation(np.arange(1, E + 1)) ** -1.2
    pr /= pr.sum()
    rows = [rng.choice(E, k, replace=False, p=pr) for _ in range(2 * T)]
    ids_np = np.stack(rows).astype(np.int32).reshape(2, T, k)
    path = DecisionPath(1, T, 8, E, k, G, N, L, device=DEV)
    path.ids_pred.copy_(torch.from_numpy(ids_np[0:1]).to(DEV))
    path.ids.copy_(torch.from_numpy(ids_np[1:2]).to(DEV))
    _lib.lb_count(path.ids_pred, G, E, cnt=path.cnt_pred)
    _lib.lb_plan_replicas(path.cnt_pred, N, L, plan=path.plan)
    path.solve()
    torch.cuda.synchronize()
    assert _lib.lb_get_status() == 0
    parity.check_path(path, 0, 12)
    sep = [t.clone() for t in (path.dest, path.perm, path.offs)]
    path.solve_fused()
    torch.cuda.synchronize()
    assert _lib.lb_get_status() == 0
    for a, b in zip(sep, (path.dest, path.perm, path.offs)):
        assert torch.equal(a, b)


@pytest.mark.parametrize("k", [1, 2, 3, 4, 5, 8, 9])
def test_scatter_small_blocks_every_k(k):
    """Small source blocks (at most one warp's share) take one warp each when
    many problems fill the GPU, and one CTA each when one problem's blocks fit
    one wave: every top-k width through both, with ragged blocks; the bytes of
    the two launches agree and pass the oracle check."""
    rng = np.random.default_rng(70 + k)
    G, E, N, L, B = 8, 32, 3, 1, 20      # G * B > the SM count: the batched launch is warp mode
    T = G * (1500 // k + 3)
    pr = rng.permutation(np.arange(1, E + 1)) ** -1.2
    pr /= pr.sum()
    rows = [rng.choice(E, k, replace=False, p=pr) for _ in range((B + 1) * T)]
    ids_np = np.stack(rows).astype(np.int32).reshape(B + 1, T, k)
    path = DecisionPath(B, T, 8, E, k, G, N, L, device=DEV)
    path.ids_pred.copy_(torch.from_numpy(ids_np[0:1]).to(DEV).expand(B, -1, -1))
    path.ids.copy_(torch.from_numpy(ids_np[1:]).to(DEV))
    _lib.lb_count(path.ids_pred, G, E, cnt=path.cnt_pred)
    _lib.lb_plan_replicas(path.cnt_pred, N, L, plan=path.plan)
    path.solve()
    torch.cuda.synchronize()
    assert _lib.lb_get_status() == 0
    for b in (0, B - 1):
        parity.check_path(path, b, 12)
        one = DecisionPath(1, T, 8, E, k, G, N, L, device=DEV)
        one.ids.copy_(path.ids[b:b + 1])
        one.plan.copy_(path.plan[b:b + 1])
        one.solve()
        torch.cuda.synchronize()
        assert _lib.lb_get_status() == 0
        for f in ("dest", "perm", "offs"):
            assert torch.equal(getattr(one, f)[0], getattr(path, f)[b]), (f, b)


def test_scatter_repeated_id_in_row_is_flagged_and_contained():
    """A repeated id in a row is bad data: lb_count flags it, and what
    lb_assign then writes for that row is unspecified, but every write stays
    inside dest and perm, the other rows are placed as the oracle places them
    on the same counts, and the context stays usable."""
    G, E, k = 4, 16, 4
    T = G * 700
    rng = np.random.default_rng(5)
    ids_np = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    ids_np[101, 3] = ids_np[101, 1]
    path = DecisionPath(1, T, 8, E, k, G, 2, 1, device=DEV)
    guard = torch.full((2, T * k + 64), -7, dtype=torch.int32, device=DEV)
    path.dest = guard[0, 32:32 + T * k].view(1, T, k)   # 32 guard words on either side
    path.perm = guard[1, 32:32 + T * k].view(1, T * k)
    path.ids_pred.copy_(torch.from_numpy(ids_np).to(DEV).unsqueeze(0))
    path.ids.copy_(path.ids_pred)
    _lib.lb_count(path.ids_pred, G, E, cnt=path.cnt_pred)
    flags = _lib.lb_get_status(clear=True)
    assert flags & _lib.LB_DEV_BAD_IDS
    _lib.lb_plan_replicas(path.cnt_pred, 2, 1, plan=path.plan)
    path.solve()
    torch.cuda.synchronize()
    _lib.lb_get_status(clear=True)
    g = guard.cpu().numpy()
    assert (g[:, :32] == -7).all() and (g[:, 32 + T * k:] == -7).all()
    dest = path.dest[0].cpu().numpy()
    assert ((dest >= -1) & (dest < G)).all()
    perm = path.perm[0].cpu().numpy()
    assert ((perm == -7) | ((perm >= 0) & (perm < T * k))).all()
    assert torch.ones(4, device=DEV).sum().item() == 4.0


# ----------------------------------------------------------------------------- swap planner (FreeBalance sec. 3.3)
def _swaps_check(cnt_np, pi_np, prm, gpu):
    r = oracle.plan_swaps(cnt_np, pi=pi_np, **prm)
    pi_out, sw, ns, lo = (t.cpu().numpy() for t in gpu)
    n = int(ns)
    assert n == r.n_swaps, (n, r.n_swaps)
    assert np.array_equal(sw[:n], r.swaps), (sw[:n], r.swaps)
    assert np.array_equal(pi_out, r.pi)
    assert np.array_equal(lo.astype(np.int64), r.loads)


def test_swaps_golden_cases():
    import pins
    for name in ("swaps_gamma_budget_tau.json", "swaps_two_ranks.json"):
        d = pins.golden(name)
        for c in d["cases"]:
            cnt = np.array(d[c.get("cnt", "cnt")], np.int32)
            prm = dict(gamma=c["gamma"], tau=c["tau"], alpha=c["alpha"], beta=c["beta"],
                       expert_bytes=c["expert_bytes"], budget=c["budget"], link_budget=c.get("link_budget"))
            pl = None if c.get("pi_in") is None else torch.tensor(c["pi_in"], dtype=torch.int32, device=DEV)
            out = _lib.lb_plan_swaps(torch.from_numpy(cnt).to(DEV), pl, **prm)
            torch.cuda.synchronize()
            assert out[1][:int(out[2])].cpu().tolist() == c["swaps"]
            assert out[0].cpu().tolist() == c["pi"] and out[3].cpu().tolist() == c["loads"]


@pytest.mark.parametrize("G,E,B,prm", [
    (8, 64, 16, dict(gamma=0.0)),
    (8, 64, 16, dict(gamma=1e-3, alpha=5.0, beta=2.0, expert_bytes=9.0, budget=200.0)),
    (16, 128, 8, dict(gamma=1e-4, tau=2.0, alpha=2.0, beta=4.0, expert_bytes=8.0, budget=40.0, link_budget=12.0)),
    (64, 256, 4, dict(gamma=1e-5, alpha=1.0, beta=1.0, expert_bytes=1.0, budget=9.0)),
    (2, 8, 6, dict(gamma=0.25)),
    (3, 12, 6, dict(gamma=0.5, tau=4.0, alpha=1.0, beta=1.0, expert_bytes=1.0, budget=6.0)),
    (40, 1000, 2, dict(gamma=0.0, alpha=1.0, beta=1.0, expert_bytes=0.0, budget=7.0)),
    (1, 4, 2, dict(gamma=1.0)),
])
def test_swaps_match_oracle(G, E, B, prm):
    """Batched problems with skewed predicted counts, even and shuffled
    placements: swaps, placement and loads bit-exact with the oracle."""
    rng = np.random.default_rng(G * 1000 + E)
    cnts, pis = [], []
    for b in range(B):
        pr = rng.permutation(np.arange(1, E + 1)) ** -1.2
        pr /= pr.sum()
        cnts.append(rng.multinomial(G * 400, pr, size=G).astype(np.int32))
        pis.append(rng.permutation(np.arange(E) // (E // G)).astype(np.int32))
    cnt = np.stack(cnts)
    for use_pi in (False, True):
        pl = torch.from_numpy(np.stack(pis)).to(DEV) if use_pi else None
        out = _lib.lb_plan_swaps(torch.from_numpy(cnt).to(DEV), pl, **prm)
        torch.cuda.synchronize()
        assert _lib.lb_get_status() == 0
        for b in range(B):
            _swaps_check(cnt[b], pis[b] if use_pi else None, prm, tuple(t[b] for t in out))


def test_swaps_bad_placement_flagged():
    cnt = torch.ones(2, 4, 16, dtype=torch.int32, device=DEV)
    pl = (torch.arange(16, dtype=torch.int32, device=DEV) // 4).repeat(2, 1)
    pl[1, 3] = 9
    out = _lib.lb_plan_swaps(cnt, pl)
    torch.cuda.synchronize()
    assert _lib.lb_get_status(clear=True) & _lib.LB_DEV_BAD_PLAN
    assert int(out[2][1]) == 0


# ----------------------------------------------------------------------------- split variants (Relief Table III)
@pytest.mark.parametrize("variant", _lib.SPLIT_VARIANTS)
@pytest.mark.parametrize("G,E,N,L,T,k,passes", [(8, 64, 2, 1, 4096, 8, 12), (16, 128, 2, 1, 2048, 8, 12),
                                                (64, 256, 2, 1, 1024, 8, 12), (4, 16, 3, 2, 400, 2, 3),
                                                (3, 9, 2, 1, 90, 3, 0), (64, 256, 2, 1, 8192, 8, 40)])
def test_split_variants_match_oracle(variant, G, E, N, L, T, k, passes):
    """Each ablation variant on batched problems (plans from the predicted
    counts, split of the actual counts): tok, mass, loads and passes_run
    bit-exact with the oracle."""
    B = 3
    rng = np.random.default_rng(G + E + T + passes)
    pr = rng.permutation(np.arange(1, E + 1)) ** -1.2
    pr /= pr.sum()
    ids_np = np.stack([np.stack([rng.choice(E, k, replace=False, p=pr) for _ in range(T)]) for _ in range(2 * B)])
    ids = torch.from_numpy(ids_np.astype(np.int32)).to(DEV)
    cnt_pred = _lib.lb_count(ids[:B], G, E)
    cnt = _lib.lb_count(ids[B:], G, E)
    plan = torch.empty(B, _lib.lb_plan_bytes(G, E, N), dtype=torch.uint8, device=DEV)
    _lib.lb_plan_replicas(cnt_pred, N, L, plan=plan)
    tok, mass, loads, prun = _lib.lb_split_variant(cnt, plan, N, passes, variant)
    torch.cuda.synchronize()
    assert _lib.lb_get_status() == 0
    for b in range(B):
        p = oracle.plan(cnt_pred[b].cpu().numpy(), N, L)
        s = oracle.split_variant(cnt[b].cpu().numpy(), p, passes, variant)
        ne = p.n_edges
        assert np.array_equal(tok[b].cpu().numpy()[:ne], s.tok), (variant, b)
        assert np.array_equal(mass[b].cpu().numpy()[:ne], s.mass), (variant, b)
        assert np.array_equal(loads[b].cpu().numpy().astype(np.int64), s.loads), (variant, b)
        assert int(prun[b]) == s.passes_run, (variant, b)


def test_split_variant_relief_equals_lb_split():
    w = workloads.WORKLOADS["qwen3-30b"]
    hid, W, bias, path = run_model(w, 1, T=4096)
    out = _lib.lb_split_variant(path.cnt, path.plan, w.N, 12, "relief")
    torch.cuda.synchronize()
    for a, b in zip(out, (path.tok, path.mass, path.loads, path.passes_run)):
        assert torch.equal(a, b)


@pytest.mark.parametrize("chain", [False, True])
@pytest.mark.parametrize("tpu,persistent,E", [(2, 0, 64), (2, 1, 64), (2, 2, 32), (1, 1, 64), (2, 0, 128), (2, 1, 16)])
def test_gate_two_tiles_per_unit(chain, tpu, persistent, E):
    """Work units of two token tiles sharing every W box (and one tile per
    unit for contrast), with an odd tile count per problem (the last unit's
    second tile lies past T): ids and logits pass the oracle check on sampled
    rows of every problem, and equal the per-tile kernel's ids."""
    if chain and E > 128:
        pytest.skip("chain needs 2E <= 256")
    _lib.lb_gate_tuning(0, 0, persistent, 0, tpu)
    B, T, H, k = 3, 2900, 576, 8   # 23 tiles per problem
    g = torch.Generator(device=DEV).manual_seed(7 + E + tpu)
    h = torch.randn(B + (1 if chain else 0), T, H, generator=g, device=DEV).to(torch.bfloat16)
    W = (torch.randn(B, E, H, generator=g, device=DEV) / H ** 0.5).to(torch.bfloat16)
    bias = torch.randn(B, E, generator=g, device=DEV)
    rng = np.random.default_rng(E)
    rows = np.unique(np.concatenate([rng.choice(T, 48, replace=False), [0, 127, 128, 255, 256, T - 1]]))
    if chain:
        ip, ia, lp, la = _lib.lb_predict_topk_chain(h, W, bias, k, want_logits=True)
        pairs = [(h[l], W[l], bias[l], ip[l], lp[l]) for l in range(B)] + \
                [(h[l + 1], W[l], bias[l], ia[l], la[l]) for l in range(B)]
    else:
        ids, lg = _lib.lb_predict_topk(h, W, bias, k, want_logits=True)
        pairs = [(h[b], W[b], bias[b], ids[b], lg[b]) for b in range(B)]
    torch.cuda.synchronize()
    assert _lib.lb_get_status() == 0
    _lib.lb_gate_tuning(0, 0, -1)
    for src, w_, b_, ids_, lg_ in pairs:
        parity.gate_check(src, w_, b_, k, ids_, lg_, rows=rows)
        ref = _lib.lb_predict_topk(src, w_, b_, k)
        assert (ref == ids_).all(dim=1).float().mean().item() > 0.999


@pytest.mark.parametrize("tpu", [1, 2])
@pytest.mark.parametrize("chain", [True, False])
@pytest.mark.parametrize("T,H,E,k,B,bias_on", [(4096, 2048, 128, 8, 3, True), (1100, 576, 64, 8, 2, True),
                                               (300, 128, 16, 2, 2, False), (2900, 4096, 128, 4, 1, True),
                                               (130, 64, 48, 8, 3, True)])
def test_gate_cta_pairs(chain, T, H, E, k, B, bias_on, tpu):
    """CTA pairs (clusters of two CTAs sharing one MMA of M = 256, each CTA
    loading its 128 tokens and half of the weight rows): ids and logits of
    every problem pass the oracle check on sampled rows (all rows of short
    problems), and agree with the one-CTA persistent kernel.  Shapes: an odd
    number of 128-token tiles (the last unit's second tile lies past T), a
    ragged tail, H past the last full stage of boxes, E = 16 (N = 32 chain),
    E = 48 (N = 48 per gate), no bias; one or two pair tiles per work unit
    (the second sharing every weight box)."""
    if not chain and E % 16:
        pytest.skip("pairs need E % 16 == 0 in the per-layer gate")
    g = torch.Generator(device=DEV).manual_seed(T + H + E + k + B)
    nh = B + 1 if chain else B
    h = torch.randn(nh, T, H, generator=g, device=DEV).to(torch.bfloat16)
    W = (torch.randn(B, E, H, generator=g, device=DEV) / H ** 0.5).to(torch.bfloat16)
    bias = torch.randn(B, E, generator=g, device=DEV) if bias_on else None
    _lib.lb_gate_tuning(0, 0, 3, 0, tpu)
    if chain:
        out = _lib.lb_predict_topk_chain(h, W, bias, k, want_logits=True)
    else:
        out = _lib.lb_predict_topk(h, W, bias, k, want_logits=True)
    torch.cuda.synchronize()
    assert _lib.lb_get_status() == 0
    _lib.lb_gate_tuning(0, 0, 1)
    ref = (_lib.lb_predict_topk_chain(h, W, bias, k, want_logits=True) if chain else
           _lib.lb_predict_topk(h, W, bias, k, want_logits=True))
    torch.cuda.synchronize()
    _lib.lb_gate_tuning()
    rng = np.random.default_rng(T + E)
    rows = None if T <= 512 else np.unique(np.concatenate([rng.choice(T, 64, replace=False),
                                                           [0, 127, 128, 255, 256, T - 1]]))
    if chain:
        ip, ia, lp, la = out
        pairs = [(h[l], W[l], None if bias is None else bias[l], ip[l], lp[l]) for l in range(B)] + \
                [(h[l + 1], W[l], None if bias is None else bias[l], ia[l], la[l]) for l in range(B)]
        for a_, r_ in zip(out, ref):
            if a_.dtype == torch.int32:
                assert (a_ == r_).all(dim=-1).float().mean().item() > 0.999
            else:
                assert torch.allclose(a_, r_, rtol=1e-5, atol=1e-5)
    else:
        ids, lg = out
        pairs = [(h[b], W[b], None if bias is None else bias[b], ids[b], lg[b]) for b in range(B)]
        assert (ids == ref[0]).all(dim=-1).float().mean().item() > 0.999
        assert torch.allclose(lg, ref[1], rtol=1e-5, atol=1e-5)
    for src, w_, b_, ids_, lg_ in pairs:
        parity.gate_check(src, w_, b_, k, ids_, lg_, rows=rows)
