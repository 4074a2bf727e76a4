"""lb_assign_noalloc: lb_assign for callers that cannot give the library device
scratch memory (a runtime whose device memory all belongs to its own arena,
or a plain-C caller without a device allocator).  It must give exactly what
lb_assign gives, call after call, although every call reuses one fixed
device array inside the library.

Collected last on purpose (file name), so a run that stops at the first
failure has already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

from moe_expert_load_bf16_b200 import _lib, workloads
from moe_expert_load_bf16_b200.pipeline import DecisionPath

pytestmark = pytest.mark.gpu


def _problem(name, T, steps):
    """Plan, counts and split for `steps` decode-like problems (on the GPU)."""
    w = workloads.WORKLOADS[name]
    ids = workloads.decode_ids(w.with_(T=T), T, steps).to("cuda")
    B = len(steps)
    path = DecisionPath(B, T, 8, w.E, w.k, w.G, w.N, w.L, device="cuda")
    path.ids_pred.copy_(ids[0:1].expand(B, -1, -1))
    path.ids.copy_(ids)
    _lib.lb_count(path.ids_pred, w.G, w.E, cnt=path.cnt_pred)
    _lib.lb_plan_replicas(path.cnt_pred, w.N, w.L, plan=path.plan)
    _lib.lb_count(path.ids, w.G, w.E, cnt=path.cnt)
    _lib.lb_split(path.cnt, path.plan, w.N, 12, out=(path.tok, path.mass, path.loads, path.passes_run))
    return w, path


def _call_noalloc_cabi(path, w):
    """Through the C ABI directly: device pointers, sizes and the stream."""
    lib = _lib._load()
    B, T, k = path.ids.shape
    dest = torch.full_like(path.dest, -7)
    perm = torch.full_like(path.perm, -7)
    offs = torch.full_like(path.offs, -7)
    P = ctypes.c_void_p
    rc = lib.lb_assign_noalloc(P(path.ids.data_ptr()), P(path.cnt.data_ptr()), P(path.plan.data_ptr()),
                               P(path.tok.data_ptr()), P(path.mass.data_ptr()), B, T, k, w.G, w.E, w.N,
                               P(dest.data_ptr()), P(perm.data_ptr()), P(offs.data_ptr()),
                               P(torch.cuda.current_stream().cuda_stream))
    assert rc == _lib.LB_OK, _lib._load().lb_last_error()
    return dest, perm, offs


def test_noalloc_matches_lb_assign_on_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    _lib.lb_get_status(clear=True)
    cases = [_problem("decode", 1024, [3, 4]), _problem("qwen3-30b", 2048, [0])]
    for w, path in cases:   # two calls in a row, different shapes and data
        ref = _lib.lb_assign(path.ids, path.cnt, path.plan, path.tok, path.mass, w.N)
        got = _call_noalloc_cabi(path, w)
        torch.cuda.synchronize()
        for r, g in zip(ref, got):
            assert torch.equal(r, g)     # integer outputs: bit-exact
    assert _lib.lb_get_status() == 0


def test_noalloc_rejects_work_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    lib = _lib._load()
    G, E, N, k, T = 64, 256, 2, 8, 64
    per = _lib.lb_assign_workspace_bytes(1, T, k, G, E, N)
    B = (1 << 20) // per + 1                    # one problem more than fits
    assert _lib.lb_assign_workspace_bytes(B, T, k, G, E, N) > (1 << 20)
    P = ctypes.c_void_p
    rc = lib.lb_assign_noalloc(P(256), P(256), P(256), P(256), P(256), B, T, k, G, E, N, P(256), P(256),
                               P(256), P(0))
    assert rc == _lib.LB_ENOSPACE
    assert b"scratch" in lib.lb_last_error()
