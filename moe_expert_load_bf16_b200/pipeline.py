"""One pass of the decision path over a batch of independent problems (layers,
steps or micro-batches of identical shape), with every buffer preallocated so
the pass can be captured in a CUDA graph.

Per problem (Libra README, Key Ideas; FreeBalance sec. 3.2, Algorithm 1;
Relief, Algorithm 1); over a chain of consecutive layers, `run_chain` runs
both gates that read one hidden state in a single pass over it:
  ids_pred = top-k(gate(h_prev))           lookahead        lb_predict_topk
  cnt_pred = counts(ids_pred)                               lb_count
  plan     = replica plan(cnt_pred)                         lb_plan_replicas
  ids      = top-k(gate(h_cur))            normal router    lb_predict_topk
  cnt      = counts(ids)                                    lb_count
  tok, mass, loads = split(cnt, plan)                       lb_split
  dest, perm, offs = assign(ids, cnt, plan, split)          lb_assign
(`solve` runs count, split and assign as lb_count + lb_decide: split and the
assign's tables in one launch per problem, the scatter in a second;
`solve_fused` as one lb_solve launch, which gives the same outputs.)
"""
import torch

from . import _lib


class DecisionPath:
    def __init__(self, B, T, H, E, k, G, N, L, passes=12, device="cuda"):
        self.B, self.T, self.H, self.E, self.k, self.G, self.N, self.L = B, T, H, E, k, G, N, L
        self.passes = passes
        dev = torch.device(device)
        i32 = dict(dtype=torch.int32, device=dev)
        # predicted and actual ids (and counts) side by side, so one launch
        # can fill or count both
        self.ids_both = torch.empty(2, B, T, k, **i32)
        self.cnt_both = torch.empty(2, B, G, E, **i32)
        self.ids_pred, self.ids = self.ids_both[0], self.ids_both[1]
        self.cnt_pred, self.cnt = self.cnt_both[0], self.cnt_both[1]
        self.plan = torch.empty(B, _lib.lb_plan_bytes(G, E, N), dtype=torch.uint8, device=dev)
        self.tok = torch.empty(B, G * N, **i32)
        self.mass = torch.empty(B, G * N, **i32)
        self.loads = torch.empty(B, G, **i32)
        self.passes_run = torch.empty(B, **i32)
        self.dest = torch.empty(B, T, k, **i32)
        self.perm = torch.empty(B, T * k, **i32)
        self.offs = torch.empty(B, G * E + 1, **i32)
        self.ws = torch.empty(max(256, _lib.lb_assign_workspace_bytes(B, T, k, G, E, N)), dtype=torch.uint8,
                              device=dev)

    # lookahead half: prediction and placement (off the per-step critical path)
    def lookahead(self, h_prev, w, bias):
        _lib.lb_predict_topk(h_prev, w, bias, self.k, ids=self.ids_pred)
        _lib.lb_count(self.ids_pred, self.G, self.E, cnt=self.cnt_pred)
        _lib.lb_plan_replicas(self.cnt_pred, self.N, self.L, plan=self.plan)

    def route(self, h_cur, w, bias):
        _lib.lb_predict_topk(h_cur, w, bias, self.k, ids=self.ids)

    # the per-step decision on actual ids (T_solve): lb_count, then split and
    # assign by lb_decide (split and the assign's tables in one launch per
    # problem, the scatter in a second); solve_separate makes the same bytes
    # with lb_split and lb_assign
    # lb_count + lb_decide: since the scatter spreads one problem's large
    # source blocks over slices, this is the faster form on every measured
    # shape (per layer, one problem: Qwen3-235B-shaped 38.6 against 51.6 us
    # for the fused lb_solve, Qwen3-30B-shaped 36.1 against 43.7 us).  The
    # outputs are identical either way.
    def solve(self, ids=None, counted=False):
        ids = self.ids if ids is None else ids
        if not counted:
            _lib.lb_count(ids, self.G, self.E, cnt=self.cnt)
        self.decide(ids)

    def solve_separate(self, ids=None, counted=False):
        ids = self.ids if ids is None else ids
        if not counted:
            _lib.lb_count(ids, self.G, self.E, cnt=self.cnt)
        _lib.lb_split(self.cnt, self.plan, self.N, self.passes,
                      out=(self.tok, self.mass, self.loads, self.passes_run))
        _lib.lb_assign(ids, self.cnt, self.plan, self.tok, self.mass, self.N,
                       out=(self.dest, self.perm, self.offs), workspace=self.ws)

    def decide(self, ids=None, with_plan=False):
        """lb_decide on this path's buffers: the plan from cnt_pred first when
        with_plan, then split and assign of cnt."""
        ids = self.ids if ids is None else ids
        cnt_pred = self.cnt_pred if with_plan else None
        _lib.lb_decide(self.cnt, ids, self.plan, self.N, self.passes, cnt_pred=cnt_pred, L=self.L,
                       out=(self.tok, self.mass, self.loads, self.passes_run, self.dest, self.perm, self.offs),
                       workspace=self.ws)

    def solve_one(self, b, split_only=False):
        """The per-step decision of problem b alone, on views of this path's
        buffers (its plan must be in place): count + split + assign as
        lb_count and lb_decide, or the split alone (lb_split, on counts
        already made)."""
        s = slice(b, b + 1)
        if split_only:
            _lib.lb_split(self.cnt[s], self.plan[s], self.N, self.passes,
                          out=(self.tok[s], self.mass[s], self.loads[s], self.passes_run[s]))
            return
        _lib.lb_count(self.ids[s], self.G, self.E, cnt=self.cnt[s])
        wsb = _lib.lb_assign_workspace_bytes(1, self.T, self.k, self.G, self.E, self.N)
        _lib.lb_decide(self.cnt[s], self.ids[s], self.plan[s], self.N, self.passes,
                       out=(self.tok[s], self.mass[s], self.loads[s], self.passes_run[s], self.dest[s],
                            self.perm[s], self.offs[s]),
                       workspace=self.ws[b * wsb:(b + 1) * wsb])

    # the same decision as one fused launch (lb_solve)
    def solve_fused(self, ids=None):
        ids = self.ids if ids is None else ids
        _lib.lb_solve(ids, self.plan, self.G, self.E, self.N, self.passes,
                      out=(self.cnt, self.tok, self.mass, self.loads, self.passes_run, self.dest, self.perm,
                           self.offs), workspace=self.ws)

    def run(self, h_prev, h_cur, w, bias, side_stream=None):
        """One pass.  With `side_stream`, the lookahead's counts and plan run
        on it concurrently with the normal-router gate (they only meet at the
        solve); both streams join before the solve."""
        if side_stream is None:
            self.lookahead(h_prev, w, bias)
            self.route(h_cur, w, bias)
            self.solve()
            return
        main = torch.cuda.current_stream()
        _lib.lb_predict_topk(h_prev, w, bias, self.k, ids=self.ids_pred)
        side_stream.wait_stream(main)
        with torch.cuda.stream(side_stream):
            _lib.lb_count(self.ids_pred, self.G, self.E, cnt=self.cnt_pred)
            _lib.lb_plan_replicas(self.cnt_pred, self.N, self.L, plan=self.plan)
        self.route(h_cur, w, bias)
        main.wait_stream(side_stream)
        self.solve()

    LAUNCHES_PER_RUN = 7   # 2 gate, 2 count, plan, split + tables, scatter

    def run_chain(self, hid, w, bias):
        """One pass over a chain of B consecutive layers whose hidden states
        are hid [B+1, T, H]: layer l predicts from hid[l] and routes hid[l+1]
        (the same problems as run(hid[:-1], hid[1:], w, bias)).  Both gates
        that read one hidden state run in one pass over it
        (lb_predict_topk_chain); predicted and actual ids are counted in one
        launch."""
        self.gate_chain(hid, w, bias)
        self.decide_chain()

    def gate_chain(self, hid, w, bias):
        """The gate half of run_chain: predicted and actual ids."""
        _lib.lb_predict_topk_chain(hid, w, bias, self.k, ids_pred=self.ids_pred, ids_act=self.ids)

    def decide_chain(self):
        """The integer half of run_chain, from the ids in this path's
        buffers: both counts in one launch, plan, split, assign."""
        self.count_chain()
        self.finish_chain()

    def count_chain(self):
        """Predicted and actual ids counted in one launch."""
        B = self.B
        _lib.lb_count(self.ids_both.view(2 * B, self.T, self.k), self.G, self.E,
                      cnt=self.cnt_both.view(2 * B, self.G, self.E))

    def finish_chain(self):
        """Plan, split and assign from this path's counts, as separate
        launches (measured: beside the next step's gate in StepPipeline,
        lb_decide's single plan + split + tables launch per problem made
        the pipelined step slower, 76.6 against 63.4 us)."""
        _lib.lb_plan_replicas(self.cnt_pred, self.N, self.L, plan=self.plan)
        self.solve_separate(counted=True)

    LAUNCHES_PER_CHAIN = 6   # chain gate, count (both), plan, split, assign prep + scatter


class StepPipeline:
    """Consecutive steps of the chained path with two batches in flight.

    The gate of a step streams the hidden states at full HBM bandwidth on
    every SM; of the integer stages that follow it, count spreads over many
    blocks, while plan, split and assign are latency-bound chains with one
    block (or a few) per problem.  Here gate and count of each step run on
    one stream, and plan, split and assign on a second stream of higher
    priority: the gate of step i+1 follows step i's count and runs beside
    step i's plan, split and assign, which take the SM slots the gate's
    grid leaves free.  (Starting the next gate before the count was slower:
    its blocks, launched early, took the SMs before the count's.)  Two
    DecisionPath buffers alternate between steps; an event per buffer keeps
    a step's gate from overwriting ids that the integer stages of the step
    two before it still read.  Every step computes the whole path over its
    batch: step i's results are in paths[i % 2] once run() returns (in
    stream order).  run() forks from and joins back to the current stream,
    so a sequence of steps can be captured in a CUDA graph."""

    def __init__(self, B, T, H, E, k, G, N, L, passes=12, device="cuda"):
        dev = torch.device(device)
        self.paths = [DecisionPath(B, T, H, E, k, G, N, L, passes=passes, device=dev) for _ in range(2)]
        self.gate_stream = torch.cuda.Stream(device=dev)
        self.int_stream = torch.cuda.Stream(device=dev, priority=-1)
        self.counted = [torch.cuda.Event() for _ in range(2)]
        self.int_done = [torch.cuda.Event() for _ in range(2)]

    def run(self, steps, hid, w, bias):
        cur = torch.cuda.current_stream()
        self.gate_stream.wait_stream(cur)
        self.int_stream.wait_stream(cur)
        for i in range(steps):
            b = i % 2
            p = self.paths[b]
            with torch.cuda.stream(self.gate_stream):
                if i >= 2:
                    self.gate_stream.wait_event(self.int_done[b])
                p.gate_chain(hid, w, bias)
                p.count_chain()
                self.counted[b].record(self.gate_stream)
            with torch.cuda.stream(self.int_stream):
                self.int_stream.wait_event(self.counted[b])
                p.finish_chain()
                self.int_done[b].record(self.int_stream)
        cur.wait_stream(self.gate_stream)
        cur.wait_stream(self.int_stream)

    LAUNCHES_PER_STEP = DecisionPath.LAUNCHES_PER_CHAIN
