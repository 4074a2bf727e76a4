"""StepPipeline's schedule on the host, without a GPU: the streams, events and
kernel calls are replaced by fakes that record what is enqueued where, and
the recorded program is checked for the orderings the two-in-flight step
relies on (stream order plus event waits give happens-before):
  - a step's count follows its gate, and its plan/split/assign follow its
    count;
  - the gate of step i+1 follows the count of step i;
  - the gate of step i+2 (same buffers as step i) follows the plan, split
    and assign of step i, which still read that buffer's ids and counts;
  - work enqueued on the caller's stream after run() follows every step.
"""
import contextlib

import pytest
import torch

from moe_expert_load_bf16_b200 import pipeline


class Recorder:
    def __init__(self):
        self.ops = []          # (stream, kind, payload)
        self.current = None

    def emit(self, stream, kind, payload=None):
        self.ops.append((stream, kind, payload))
        return len(self.ops) - 1


class FakeStream:
    def __init__(self, rec, name):
        self.rec, self.name = rec, name

    def wait_stream(self, other):
        self.rec.emit(self, "wait_stream", other)

    def wait_event(self, ev):
        self.rec.emit(self, "wait_event", ev)


class FakeEvent:
    def __init__(self, rec):
        self.rec = rec

    def record(self, stream=None):
        self.rec.emit(stream if stream is not None else self.rec.current, "record", self)


class FakePath:
    def __init__(self, rec, b):
        self.rec, self.b = rec, b

    def gate_chain(self, hid, w, bias):
        self.rec.emit(self.rec.current, "gate", (hid, self.b))

    def count_chain(self):
        self.rec.emit(self.rec.current, "count", self.b)

    def finish_chain(self):
        self.rec.emit(self.rec.current, "finish", self.b)


def happens_before(ops):
    """Transitive predecessors of every op: the previous op on its stream,
    the last op before a wait_stream on the waited stream, the last record
    of a waited event before the wait."""
    pred = [set() for _ in ops]
    last_on = {}
    last_record = {}
    for i, (s, kind, payload) in enumerate(ops):
        if s in last_on:
            j = last_on[s]
            pred[i] |= pred[j] | {j}
        if kind == "wait_stream" and payload in last_on:
            j = last_on[payload]
            pred[i] |= pred[j] | {j}
        if kind == "wait_event" and id(payload) in last_record:
            j = last_record[id(payload)]
            pred[i] |= pred[j] | {j}
        if kind == "record":
            last_record[id(payload)] = i
        last_on[s] = i
    return pred


def run_recorded(steps_per_call):
    rec = Recorder()
    caller = FakeStream(rec, "caller")
    rec.current = caller
    sp = object.__new__(pipeline.StepPipeline)
    sp.paths = [FakePath(rec, 0), FakePath(rec, 1)]
    sp.gate_stream = FakeStream(rec, "gate")
    sp.int_stream = FakeStream(rec, "int")
    sp.counted = [FakeEvent(rec) for _ in range(2)]
    sp.int_done = [FakeEvent(rec) for _ in range(2)]

    @contextlib.contextmanager
    def use(stream):
        prev, rec.current = rec.current, stream
        try:
            yield
        finally:
            rec.current = prev

    mp = pytest.MonkeyPatch()
    mp.setattr(torch.cuda, "current_stream", lambda *a, **k: rec.current)
    mp.setattr(torch.cuda, "stream", use)
    try:
        step = 0
        for n in steps_per_call:
            sp.run(n, f"hid{step}", "w", "bias")
            step += n
            rec.emit(caller, "after", step)
    finally:
        mp.undo()
    return rec.ops


@pytest.mark.parametrize("calls", [[6], [1, 1, 1, 1], [2, 3], [5, 1, 2]])
def test_step_pipeline_orderings(calls):
    ops = run_recorded(calls)
    pred = happens_before(ops)
    # the k-th gate / count / finish in program order is step k (buffer k % 2)
    gates = [i for i, o in enumerate(ops) if o[1] == "gate"]
    counts = [i for i, o in enumerate(ops) if o[1] == "count"]
    finishes = [i for i, o in enumerate(ops) if o[1] == "finish"]
    n = sum(calls)
    assert len(gates) == len(counts) == len(finishes) == n
    for i in range(n):
        assert ops[gates[i]][0].name == "gate" and ops[counts[i]][0].name == "gate"
        assert ops[finishes[i]][0].name == "int"
        assert gates[i] in pred[counts[i]]
        assert counts[i] in pred[finishes[i]]
        if i + 1 < n:
            assert counts[i] in pred[gates[i + 1]]
        if i + 2 < n:
            # step i+2 reuses step i's buffers only after step i's integer stages
            assert finishes[i] in pred[gates[i + 2]]
    # a call's steps alternate buffers from 0, so buffers may be reused
    # across calls: every gate must follow the last finish on its buffer
    last_finish = {}
    k = 0
    for c in calls:
        for j in range(c):
            b = ops[gates[k]][2][1]
            assert b == j % 2
            if b in last_finish:
                assert last_finish[b] in pred[gates[k]]
            last_finish[b] = finishes[k]
            k += 1
    # the caller's stream sees every step complete after each run()
    afters = [i for i, o in enumerate(ops) if o[1] == "after"]
    done = 0
    for a, c in zip(afters, calls):
        done += c
        for i in range(done):
            assert finishes[i] in pred[a] and counts[i] in pred[a]


def test_schedule_check_catches_a_missing_wait():
    """The check itself fails when the gate of step i+2 does not wait for
    step i's integer stages (the wait on int_done removed)."""
    ops = run_recorded([6])
    int_done_waits = [i for i, o in enumerate(ops) if o[0].name == "gate" and o[1] == "wait_event"]
    assert int_done_waits
    broken = [o for i, o in enumerate(ops) if i not in int_done_waits]
    pred = happens_before(broken)
    gates = [i for i, o in enumerate(broken) if o[1] == "gate"]
    finishes = [i for i, o in enumerate(broken) if o[1] == "finish"]
    assert any(finishes[i] not in pred[gates[i + 2]] for i in range(4))
