"""The oracle against its pins (CPU only)."""
import numpy as np
import pytest

import oracle
import pins


@pytest.fixture(scope="module")
def o():
    return oracle.default()


@pytest.mark.parametrize("check", pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_pin(o, check):
    check(o)


def test_empty_inputs(o):
    ids = np.zeros((0, 2), np.int32)
    cnt = o.count(ids, 4, 16)
    assert cnt.sum() == 0
    p = o.plan(cnt, 1, 0)
    assert p.n_edges == 0 and (p.used == 0).all()
    s = o.split(cnt, p)
    assert s.loads.sum() == 0 and s.passes_run == 1
    dest, perm, offs = o.assign(ids, p, s, 4, 16)
    assert dest.size == 0 and perm.size == 0 and (offs == 0).all()


def test_single_rank(o):
    """G=1: every expert is home, nothing to plan or split."""
    rng = np.random.default_rng(1)
    ids = np.stack([rng.permutation(8)[:3] for _ in range(10)]).astype(np.int32)
    cnt = o.count(ids, 1, 8)
    p = o.plan(cnt, 0, 0)
    s = o.split(cnt, p)
    dest, perm, offs = o.assign(ids, p, s, 1, 8)
    assert (dest == 0).all()
    assert np.array_equal(perm, np.argsort(ids.ravel(), kind="stable"))


def test_all_tokens_one_expert(o):
    """Every token asks for expert 0 (k=1): the split spreads its remote mass."""
    G, E, T = 4, 8, 64
    ids = np.zeros((T, 1), np.int32)
    cnt = o.count(ids, G, E)
    p = o.plan(cnt, 2, 1)
    pins.plan_invariants(cnt, p, 2, 1)
    s = pins.split_invariants(o, cnt, p)
    dest, perm, offs = o.assign(ids, p, s, G, E)
    pins.assign_invariants(ids, cnt, p, s, dest, perm, offs)
    assert s.loads.max() == o.split_optimum(cnt, p)


def test_invalid_arguments(o):
    cnt = np.zeros((4, 16), np.int32)
    with pytest.raises(oracle.OracleError):
        o.plan(cnt, 20, 0)         # N > E - E/G
    with pytest.raises(oracle.OracleError):
        o.plan(cnt, 1, 2)          # L > N
    with pytest.raises(oracle.OracleError):
        o.plan(np.zeros((3, 16), np.int32), 1, 0)   # E % G != 0
