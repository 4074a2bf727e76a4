"""CPU oracle for the MoE expert-parallel load-balancing decision path.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
benchmark's CPU-baseline leg may import this package.  It shares no code with
the CUDA library and never imports it.  The arithmetic lives in lb_oracle.c
(plain C, fp64 accumulation for the gate); this module only marshals numpy
arrays into it.

Functions (see lb_oracle.c for the definitions and the pages they follow):
  gate(h_bits, w_bits, bias, k)          -> logits fp32 [T,E], ids int32 [T,k]
  count(ids, G, E)                       -> cnt int32 [G,E]
  plan(cnt, N, L)                        -> Plan
  split(cnt, plan, passes)               -> Split
  assign(ids, plan, split, G, E)         -> dest, perm, offs
  split_optimum(cnt, plan)               -> exact integer min-max load
  plan_swaps(cnt, pi, gamma, tau, alpha, beta, expert_bytes, budget)
                                         -> Swaps (budgeted pairwise swaps)
  split_variant(cnt, plan, passes, variant)
                                         -> Split (Relief's ablation variants)

`Oracle(path)` binds the same functions to another build of lb_oracle.c
(the tests use it to check that the pins reject planted mistakes).
"""
import ctypes
import os
from dataclasses import dataclass

import numpy as np

from . import build as _build


class OracleError(RuntimeError):
    def __init__(self, fn, code):
        what = {1: "invalid argument", 3: "bad data"}.get(code, "error")
        super().__init__(f"{fn} returned {code} ({what})")
        self.code = code


@dataclass
class Plan:
    G: int
    E: int
    N: int
    L: int
    holds: np.ndarray       # [G,E] uint8
    used: np.ndarray        # [G] int32
    slots: np.ndarray       # [G,N] int32, expert id or -1
    slot_phase: np.ndarray  # [G,N] int32, 1 or 2 (0 = empty)
    plan_load: np.ndarray   # [G] int64, load model after phase 2
    edge_u: np.ndarray      # [n_edges] int32, schedule order
    edge_v: np.ndarray
    edge_e: np.ndarray
    edge_round: np.ndarray
    round_ptr: np.ndarray   # [n_rounds+1]

    @property
    def n_edges(self):
        return int(self.edge_u.shape[0])

    @property
    def n_rounds(self):
        return int(self.round_ptr.shape[0] - 1)


@dataclass
class Split:
    tok: np.ndarray         # [n_edges] int32, schedule order
    mass: np.ndarray        # [n_edges] int32, tokens kept at home
    loads: np.ndarray       # [G] int64
    passes_run: int


@dataclass
class Swaps:
    pi: np.ndarray          # [E] int32, rank of each expert after the swaps
    swaps: np.ndarray       # [n,4] int32 (u, v, a, b) in acceptance order
    loads: np.ndarray       # [G] int64, rank loads under pi

    @property
    def n_swaps(self):
        return int(self.swaps.shape[0])


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def plan_from_arrays(G, E, N, L, holds, edge_u, edge_v, edge_e, round_ptr):
    """A Plan made of given arrays (to run the oracle's split and assign on a
    plan that came from elsewhere, or on a hand-written one)."""
    z = np.zeros(0, np.int32)
    return Plan(G, E, N, L, _c(holds, np.uint8), z, z, z, np.zeros(G, np.int64),
                _c(edge_u, np.int32), _c(edge_v, np.int32), _c(edge_e, np.int32),
                np.full(len(edge_u), -1, np.int32), _c(round_ptr, np.int32))


class Oracle:
    def __init__(self, path):
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i64, i32 = ctypes.c_int64, ctypes.c_int
        lib.orc_gate.argtypes = [P, P, P, i64, i32, i32, i32, P, P]
        lib.orc_count.argtypes = [P, i64, i32, i32, i32, P]
        lib.orc_plan.argtypes = [P, i32, i32, i32, i32, P, P, P, P, P, P, P, P, P, P, P, P]
        lib.orc_split.argtypes = [P, i32, i32, P, i32, P, P, P, i32, P, i32, P, P, P, P]
        lib.orc_assign.argtypes = [P, i64, i32, i32, i32, P, i32, P, P, P, P, P, P, P, P]
        lib.orc_split_optimum.argtypes = [P, i32, i32, P, i32, P, P, P]
        lib.orc_split_optimum.restype = ctypes.c_int64
        d = ctypes.c_double
        lib.orc_plan_swaps.argtypes = [P, P, i32, i32, d, d, d, d, d, d, d, P, P, P, P]
        lib.orc_plan_swaps.restype = ctypes.c_int
        lib.orc_split_variant.argtypes = [P, i32, i32, P, i32, P, P, P, i32, P, i32, i32, P, P, P, P]
        lib.orc_split_variant.restype = ctypes.c_int
        for f in (lib.orc_gate, lib.orc_count, lib.orc_plan, lib.orc_split, lib.orc_assign):
            f.restype = ctypes.c_int
        lib.orc_threads.restype = ctypes.c_int
        self.lib = lib
        self.path = path

    @staticmethod
    def _check(fn, rc):
        if rc != 0:
            raise OracleError(fn, rc)

    def gate(self, h_bits, w_bits, bias, k):
        """h_bits [T,H] uint16 (bf16 bit patterns), w_bits [E,H] uint16, bias [E] f32 or None."""
        h = _c(h_bits, np.uint16)
        w = _c(w_bits, np.uint16)
        b = None if bias is None else _c(bias, np.float32)
        T, H = h.shape
        E = w.shape[0]
        assert w.shape[1] == H
        logits = np.empty((T, E), np.float32)
        ids = np.empty((T, k), np.int32)
        self._check("orc_gate", self.lib.orc_gate(_ptr(h), _ptr(w), _ptr(b), T, H, E, k,
                                                  _ptr(logits), _ptr(ids)))
        return logits, ids

    def count(self, ids, G, E):
        ids = _c(ids, np.int32)
        T, k = ids.shape
        cnt = np.empty((G, E), np.int32)
        self._check("orc_count", self.lib.orc_count(_ptr(ids), T, k, E, G, _ptr(cnt)))
        return cnt

    def plan(self, cnt, N, L):
        cnt = _c(cnt, np.int32)
        G, E = cnt.shape
        me = G * N
        holds = np.empty((G, E), np.uint8)
        used = np.empty(G, np.int32)
        slots = np.empty((G, N), np.int32)
        slot_phase = np.empty((G, N), np.int32)
        plan_load = np.empty(G, np.int64)
        eu, ev, ee, er = (np.empty(me + 1, np.int32) for _ in range(4))
        rp = np.empty(me + 2, np.int32)
        ne, nr = ctypes.c_int(0), ctypes.c_int(0)
        self._check("orc_plan", self.lib.orc_plan(
            _ptr(cnt), G, E, N, L, _ptr(holds), _ptr(used), _ptr(slots), _ptr(slot_phase),
            _ptr(plan_load), _ptr(eu), _ptr(ev), _ptr(ee), _ptr(er), _ptr(rp),
            ctypes.byref(ne), ctypes.byref(nr)))
        n, r = ne.value, nr.value
        return Plan(G, E, N, L, holds, used, slots, slot_phase, plan_load,
                    eu[:n].copy(), ev[:n].copy(), ee[:n].copy(), er[:n].copy(), rp[:r + 1].copy())

    @staticmethod
    def _plan_arrays(p):
        return (_c(p.holds, np.uint8), _c(p.edge_u, np.int32), _c(p.edge_v, np.int32),
                _c(p.edge_e, np.int32), _c(p.round_ptr, np.int32))

    def split(self, cnt, p, passes=12):
        cnt = _c(cnt, np.int32)
        G, E = cnt.shape
        holds, eu, ev, ee, rp = self._plan_arrays(p)
        ne = eu.shape[0]
        tok = np.empty(ne + 1, np.int32)
        mass = np.empty(ne + 1, np.int32)
        loads = np.empty(G, np.int64)
        pr = ctypes.c_int(0)
        self._check("orc_split", self.lib.orc_split(
            _ptr(cnt), G, E, _ptr(holds), ne, _ptr(eu), _ptr(ev), _ptr(ee), rp.shape[0] - 1,
            _ptr(rp), passes, _ptr(tok), _ptr(mass), _ptr(loads), ctypes.byref(pr)))
        return Split(tok[:ne].copy(), mass[:ne].copy(), loads, pr.value)

    def assign(self, ids, p, s, G, E):
        ids = _c(ids, np.int32)
        T, k = ids.shape
        holds, eu, ev, ee, _ = self._plan_arrays(p)
        tok = _c(s.tok, np.int32)
        mass = _c(s.mass, np.int32)
        dest = np.empty((T, k), np.int32)
        perm = np.empty(T * k, np.int32)
        offs = np.empty(G * E + 1, np.int32)
        self._check("orc_assign", self.lib.orc_assign(
            _ptr(ids), T, k, G, E, _ptr(holds), eu.shape[0], _ptr(eu), _ptr(ev), _ptr(ee),
            _ptr(tok), _ptr(mass), _ptr(dest), _ptr(perm), _ptr(offs)))
        return dest, perm, offs

    # variants of Relief's ablation (see orc_split_variant for the readings)
    SPLIT_VARIANTS = ("relief", "no_reverse", "jacobi", "hash", "water", "proportional", "fp32", "q1120")

    def split_variant(self, cnt, p, passes=12, variant="relief"):
        v = self.SPLIT_VARIANTS.index(variant) if isinstance(variant, str) else int(variant)
        cnt = _c(cnt, np.int32)
        G, E = cnt.shape
        holds, eu, ev, ee, rp = self._plan_arrays(p)
        ne = eu.shape[0]
        tok = np.zeros(max(ne, 1), np.int32)
        mass = np.zeros(max(ne, 1), np.int32)
        loads = np.zeros(G, np.int64)
        pr = ctypes.c_int32(0)
        self._check("orc_split_variant", self.lib.orc_split_variant(
            _ptr(cnt), G, E, _ptr(holds), ne, _ptr(eu), _ptr(ev), _ptr(ee), rp.shape[0] - 1, _ptr(rp), passes, v,
            _ptr(tok), _ptr(mass), _ptr(loads), ctypes.byref(pr)))
        return Split(tok[:ne].copy(), mass[:ne].copy(), loads, int(pr.value))

    def threads(self):
        return int(self.lib.orc_threads())

    def split_optimum(self, cnt, p):
        cnt = _c(cnt, np.int32)
        G, E = cnt.shape
        holds, eu, ev, ee, _ = self._plan_arrays(p)
        r = self.lib.orc_split_optimum(_ptr(cnt), G, E, _ptr(holds), eu.shape[0],
                                       _ptr(eu), _ptr(ev), _ptr(ee))
        if r < 0:
            raise OracleError("orc_split_optimum", -r)
        return int(r)


    def plan_swaps(self, cnt, pi=None, gamma=0.0, tau=0.0, alpha=0.0, beta=1.0, expert_bytes=0.0,
                   budget=float("inf"), link_budget=None):
        link_budget = budget if link_budget is None else link_budget
        cnt = _c(cnt, np.int32)
        G, E = cnt.shape
        pi_in = None if pi is None else _c(pi, np.int32)
        pi_out = np.zeros(E, np.int32)
        sw = np.zeros((max(1, E // 2 + 1), 4), np.int32)
        n = ctypes.c_int32(0)
        loads = np.zeros(G, np.int64)
        self._check("orc_plan_swaps", self.lib.orc_plan_swaps(
            _ptr(cnt), _ptr(pi_in), G, E, gamma, tau, alpha, beta, expert_bytes, budget, link_budget, _ptr(pi_out),
            _ptr(sw),
            ctypes.byref(n), _ptr(loads)))
        return Swaps(pi_out, sw[:n.value].copy(), loads)


_default = None


def default():
    global _default
    if _default is None:
        _default = Oracle(_build.build())
    return _default


def gate(*a, **kw):
    return default().gate(*a, **kw)


def count(*a, **kw):
    return default().count(*a, **kw)


def plan(*a, **kw):
    return default().plan(*a, **kw)


def split(*a, **kw):
    return default().split(*a, **kw)


def assign(*a, **kw):
    return default().assign(*a, **kw)


def split_optimum(*a, **kw):
    return default().split_optimum(*a, **kw)


def plan_swaps(*a, **kw):
    return default().plan_swaps(*a, **kw)


def split_variant(*a, **kw):
    return default().split_variant(*a, **kw)


def lib_path():
    return os.path.abspath(_build.LIB)
