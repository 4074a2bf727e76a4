"""The C-ABI library loads and exports every symbol include/lb.h declares
(CPU only: no compute call, only host-side functions and argument checks)."""
import ctypes
import os
import re

import pytest

from moe_expert_load_bf16_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lb.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib._load()


def declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:int|size_t|const char \*)\s*(lb_\w+)\s*\(", src, re.M)))


def test_header_declares_the_five_steps():
    names = declared()
    for n in ("lb_predict_topk", "lb_count", "lb_plan_replicas", "lb_split", "lb_assign"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for n in declared():
        assert hasattr(lib, n), n
        assert n in _lib.EXPORTS, n


def test_host_only_functions(lib):
    assert lib.lb_version() == 100
    assert lib.lb_strerror(_lib.LB_EINVAL) == b"invalid argument"
    nb = _lib.lb_plan_bytes(64, 256, 2)
    assert nb % 256 == 0
    lay = _lib.plan_layout(64, 256, 2)
    offs = [lay[k] for k in ("hdr", "used", "slots", "slot_phase", "plan_load", "edge_u", "edge_v", "edge_e",
                             "edge_round", "round_ptr", "rep_ptr", "rep_edge", "holds")]
    assert offs == sorted(offs) and all(o % 4 == 0 for o in offs)
    assert lay["holds"] + 64 * 256 <= lay["total"] == nb
    assert _lib.lb_assign_workspace_bytes(3, 100, 8, 8, 64, 2) % 256 == 0


def test_arguments_rejected_before_any_launch(lib):
    P = ctypes.c_void_p
    s = P(0)
    # nbatch = 0, E too large, k > E: rejected without touching the GPU
    assert lib.lb_predict_topk(P(16), P(16), None, 0, 128, 64, 16, 2, P(16), None, s) == _lib.LB_EINVAL
    assert lib.lb_predict_topk(P(16), P(16), None, 1, 128, 64, 300, 2, P(16), None, s) == _lib.LB_EINVAL
    assert lib.lb_predict_topk(P(16), P(16), None, 1, 128, 64, 4, 5, P(16), None, s) == _lib.LB_EINVAL
    assert lib.lb_predict_topk(P(16), P(16), None, 1, 128, 60, 16, 2, P(16), None, s) == _lib.LB_EINVAL
    # chain gate: E = 256 (N = 2E > 256), E % 16, L = 0, k > E
    for L, E, k in ((2, 256, 2), (2, 24, 2), (0, 64, 2), (2, 16, 17)):
        assert lib.lb_predict_topk_chain(P(16), P(16), None, L, 128, 64, E, k, P(16), P(16), None, None,
                                         s) == _lib.LB_EINVAL
    # swap planner: beta = 0, NaN gamma, E % G, G > 64, negative budget
    D = ctypes.c_double
    for G, E, gamma, beta, budget in ((4, 16, 0.0, 0.0, 1.0), (4, 16, float("nan"), 1.0, 1.0), (3, 16, 0.0, 1.0, 1.0),
                                      (128, 128, 0.0, 1.0, 1.0), (4, 16, 0.0, 1.0, -1.0)):
        assert lib.lb_plan_swaps(P(16), None, 1, G, E, D(gamma), D(0), D(0), D(beta), D(0), D(budget), D(budget),
                                 P(16), P(16), P(16), P(16), s) == _lib.LB_EINVAL
    assert lib.lb_swaps_capacity(16) == 8 and lib.lb_swaps_capacity(1) == 1
    # split variants: unknown variant, negative passes
    assert lib.lb_split_variant(P(256), P(256), 1, 4, 16, 1, 12, 8, P(16), P(16), P(16), P(16), s) == _lib.LB_EINVAL
    assert lib.lb_split_variant(P(256), P(256), 1, 4, 16, 1, -1, 0, P(16), P(16), P(16), P(16), s) == _lib.LB_EINVAL
    assert lib.lb_count(P(16), 1, 10, 2, 16, 4, P(16), s) == _lib.LB_EINVAL          # T % G
    assert lib.lb_plan_replicas(P(256), 1, 3, 16, 1, 0, P(256), s) == _lib.LB_EINVAL  # E % G
    assert lib.lb_plan_replicas(P(256), 1, 4, 16, 20, 0, P(256), s) == _lib.LB_EINVAL  # N > E - E/G
    assert lib.lb_plan_replicas(P(256), 1, 4, 16, 1, 2, P(256), s) == _lib.LB_EINVAL  # L > N
    assert lib.lb_plan_replicas(P(256), 1, 128, 128, 1, 0, P(256), s) == _lib.LB_EINVAL  # G > 64
    assert lib.lb_split(P(256), P(256), 1, 4, 16, 1, -1, P(16), P(16), P(16), P(16), s) == _lib.LB_EINVAL
    assert lib.lb_assign(P(16), P(16), P(256), P(16), P(16), 1, 8, 2, 4, 16, 1, P(16), P(16), P(16), P(256),
                         1, s) == _lib.LB_ENOSPACE
    # lb_decide: L > N with predicted counts, negative passes, T % G, unaligned plan
    #   (cnt_pred, cnt, ids, plan, nbatch, T, k, G, E, N, L, passes, tok, mass, loads, passes_run,
    #    dest, perm, offs, workspace, workspace_bytes, stream)
    for cp, T, L, passes, plan in ((P(256), 16, 3, 12, P(256)), (None, 16, 0, -1, P(256)),
                                   (None, 10, 0, 12, P(256)), (None, 16, 0, 12, P(16))):
        assert lib.lb_decide(cp, P(256), P(256), plan, 1, T, 2, 4, 16, 2, L, passes, P(16), P(16), P(16), P(16),
                             P(16), P(16), P(16), P(256), 1 << 20, s) == _lib.LB_EINVAL
    assert lib.lb_decide(None, P(256), P(256), P(256), 1, 16, 2, 4, 16, 2, 0, 12, P(16), P(16), P(16), P(16),
                         P(16), P(16), P(16), P(256), 1, s) == _lib.LB_ENOSPACE
    assert lib.lb_gate_tuning(3, 5, 0, 0, 0, 0) == _lib.LB_EINVAL
    assert lib.lb_gate_tuning(3, 2, 8, 0, 0, 0) == _lib.LB_EINVAL
    assert lib.lb_gate_tuning(3, 2, 1, 3, 0, 0) == _lib.LB_EINVAL
    assert lib.lb_gate_tuning(0, 0, 0, 0, 3, 0) == _lib.LB_EINVAL
    assert lib.lb_gate_tuning(0, 0, 0, 0, 0, -1) == _lib.LB_EINVAL
    assert lib.lb_gate_tuning(0, 0, 0, 0, 0, 0) == _lib.LB_OK
    assert lib.lb_launch_options(2, 0) == _lib.LB_EINVAL
    assert lib.lb_launch_options(-1, 0) == _lib.LB_EINVAL
    assert lib.lb_launch_options(1, 384) == _lib.LB_EINVAL
    assert lib.lb_launch_options(1, 2048) == _lib.LB_EINVAL
    assert lib.lb_launch_options(1, 512) == _lib.LB_OK
    assert lib.lb_launch_options(1, 0) == _lib.LB_OK


BAD_SHAPES = [(0, 16, 2), (-1, 16, 2), (65, 130, 2), (4, 0, 2), (4, 16, 0)]   # (G, E, k)


@pytest.mark.parametrize("G,E,k", BAD_SHAPES)
def test_bad_rank_expert_or_k_counts_return_einval(lib, G, E, k):
    """Every compute entry point that takes G, E or k rejects G <= 0, G beyond
    the maximum, E = 0 and k = 0 with LB_EINVAL before it divides by any of them
    or launches anything (a divide by G = 0 in the caller's process would end it
    with SIGFPE).  Each call is made only with a tuple that is invalid for that
    entry point, so no call can reach a launch."""
    P, D = ctypes.c_void_p, ctypes.c_double
    s, T, N, L, a = P(0), 16, 1, 0, P(256)
    EINVAL = _lib.LB_EINVAL
    # entry points that take G, E and k
    assert lib.lb_count(a, 1, T, k, E, G, a, s) == EINVAL
    assert lib.lb_assign(a, a, a, a, a, 1, T, k, G, E, N, a, a, a, a, 1 << 20, s) == EINVAL
    assert lib.lb_assign_noalloc(a, a, a, a, a, 1, T, k, G, E, N, a, a, a, s) == EINVAL
    assert lib.lb_decide(None, a, a, a, 1, T, k, G, E, N, L, 12, a, a, a, a, a, a, a, a, 1 << 20, s) == EINVAL
    assert lib.lb_decide(a, a, a, a, 1, T, k, G, E, N, L, 12, a, a, a, a, a, a, a, a, 1 << 20, s) == EINVAL
    assert lib.lb_solve(a, a, 1, T, k, G, E, N, 12, a, a, a, a, a, a, a, a, a, 1 << 20, s) == EINVAL
    if k > 0:   # entry points that take G and E but no k: the tuple is bad in G or E
        assert lib.lb_plan_replicas(a, 1, G, E, N, L, a, s) == EINVAL
        assert lib.lb_split(a, a, 1, G, E, N, 12, a, a, a, a, s) == EINVAL
        assert lib.lb_plan_swaps(a, None, 1, G, E, D(0), D(0), D(0), D(1), D(0), D(1), D(1), a, a, a, a,
                                 s) == EINVAL
        assert lib.lb_split_variant(a, a, 1, G, E, N, 12, 0, a, a, a, a, s) == EINVAL
    if E == 0 or k == 0:   # the gates take E and k but no G
        assert lib.lb_predict_topk(a, a, None, 1, T, 64, E, k, a, None, s) == EINVAL
        assert lib.lb_predict_topk_chain(a, a, None, 2, T, 64, E, k, a, a, None, None, s) == EINVAL
    if G <= 0 or E <= 0:   # sizes of shapes that cannot exist are zero
        assert lib.lb_plan_bytes(G, E, N) == 0
        assert lib.lb_assign_workspace_bytes(1, T, k, G, E, N) == 0


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        _lib._load()
