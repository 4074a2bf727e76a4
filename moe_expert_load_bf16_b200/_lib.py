"""Thin ctypes binding of liblb.so (include/lb.h).

Argument marshalling only: every function checks shapes, dtypes and devices
of torch CUDA tensors, passes their device pointers and the current CUDA
stream to the C entry point of the same name, and raises LBError on a
non-zero return code.  No step of the decision path runs here, and there is
no fallback: if liblb.so is missing or cannot be loaded, every call raises.
"""
import ctypes
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblb.so")

LB_OK, LB_EINVAL, LB_ECUDA, LB_EDATA, LB_ENOSPACE = 0, 1, 2, 3, 4
LB_DEV_BAD_IDS, LB_DEV_TIMEOUT, LB_DEV_BAD_PLAN, LB_DEV_BAD_SPLIT = 1, 2, 4, 8

_lib = None


class LBError(RuntimeError):
    def __init__(self, fn, code):
        msg = _load().lb_strerror(code).decode() if _lib is not None else str(code)
        if code == LB_ECUDA and _lib is not None:
            msg += ": " + _lib.lb_last_error().decode(errors="replace")
        super().__init__(f"{fn} failed: {msg} ({code})")
        self.code = code


class _Layout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in (
        "hdr", "used", "slots", "slot_phase", "plan_load", "edge_u", "edge_v", "edge_e",
        "edge_round", "round_ptr", "rep_ptr", "rep_edge", "holds", "total")]


def _load():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m moe_expert_load_bf16_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.lb_predict_topk.argtypes = [P, P, P, I, I, I, I, I, P, P, P]
    lib.lb_predict_topk_chain.argtypes = [P, P, P, I, I, I, I, I, P, P, P, P, P]
    lib.lb_gate_tuning.argtypes = [I, I, I, I, I, I]
    lib.lb_launch_options.argtypes = [I, I]
    D = ctypes.c_double
    lib.lb_swaps_capacity.argtypes = [I]
    lib.lb_plan_swaps.argtypes = [P, P, I, I, I, D, D, D, D, D, D, D, P, P, P, P, P]
    lib.lb_split_variant.argtypes = [P, P, I, I, I, I, I, I, P, P, P, P, P]
    lib.lb_count.argtypes = [P, I, I, I, I, I, P, P]
    lib.lb_plan_bytes.argtypes = [I, I, I]
    lib.lb_plan_bytes.restype = SZ
    lib.lb_plan_layout_of.argtypes = [I, I, I, ctypes.POINTER(_Layout)]
    lib.lb_plan_replicas.argtypes = [P, I, I, I, I, I, P, P]
    lib.lb_split.argtypes = [P, P, I, I, I, I, I, P, P, P, P, P]
    lib.lb_assign_workspace_bytes.argtypes = [I, I, I, I, I, I]
    lib.lb_assign_workspace_bytes.restype = SZ
    lib.lb_assign.argtypes = [P, P, P, P, P, I, I, I, I, I, I, P, P, P, P, SZ, P]
    lib.lb_decide.argtypes = [P, P, P, P, I, I, I, I, I, I, I, I, P, P, P, P, P, P, P, P, SZ, P]
    lib.lb_assign_noalloc.argtypes = [P, P, P, P, P, I, I, I, I, I, I, P, P, P, P]
    lib.lb_solve.argtypes = [P, P, I, I, I, I, I, I, I, P, P, P, P, P, P, P, P, P, SZ, P]
    lib.lb_get_status.argtypes = [ctypes.POINTER(ctypes.c_int32), I]
    lib.lb_strerror.argtypes = [I]
    lib.lb_strerror.restype = ctypes.c_char_p
    lib.lb_last_error.argtypes = []
    lib.lb_last_error.restype = ctypes.c_char_p
    for f in ("lb_predict_topk", "lb_predict_topk_chain", "lb_plan_swaps", "lb_swaps_capacity", "lb_split_variant",
              "lb_gate_tuning", "lb_launch_options",
              "lb_count", "lb_plan_layout_of", "lb_plan_replicas",
              "lb_split", "lb_assign", "lb_assign_noalloc", "lb_decide", "lb_solve", "lb_get_status", "lb_version"):
        getattr(lib, f).restype = ctypes.c_int
    _lib = lib
    return lib


def _check(fn, rc):
    if rc != LB_OK:
        raise LBError(fn, rc)


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _p(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _need(t, dtype, name):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _batched(t, nd):
    """Add a leading batch dimension to an unbatched tensor."""
    return t.unsqueeze(0) if t.dim() == nd - 1 else t


# ------------------------------------------------------------------ step 1
def lb_predict_topk(h, w, bias, k, want_logits=False, ids=None, logits=None):
    """h bf16 [B,T,H] (or [T,H]), w bf16 [B,E,H] (or [E,H]), bias f32 [B,E] or None.
    Returns ids int32 [B,T,k] (and logits f32 [B,T,E] when want_logits)."""
    lib = _load()
    squeeze = h.dim() == 2
    h, w = _batched(h, 3), _batched(w, 3)
    _need(h, torch.bfloat16, "h")
    _need(w, torch.bfloat16, "w")
    B, T, H = h.shape
    E = w.shape[1]
    if w.shape != (B, E, H):
        raise ValueError("w must be [B,E,H] matching h")
    if bias is not None:
        bias = _batched(bias, 2)
        _need(bias, torch.float32, "bias")
        if bias.shape != (B, E):
            raise ValueError("bias must be [B,E]")
    if ids is None:
        ids = torch.empty(B, T, k, dtype=torch.int32, device=h.device)
    if want_logits and logits is None:
        logits = torch.empty(B, T, E, dtype=torch.float32, device=h.device)
    _check("lb_predict_topk", lib.lb_predict_topk(_p(h), _p(w), _p(bias), B, T, H, E, k, _p(ids),
                                                  _p(logits if want_logits else None), _stream()))
    if squeeze:
        ids = ids[0]
        logits = logits[0] if want_logits else None
    return (ids, logits) if want_logits else ids


def lb_predict_topk_chain(h, w, bias, k, want_logits=False, ids_pred=None, ids_act=None, logits_pred=None,
                          logits_act=None):
    """Both gates that read each hidden state of a chain, in one pass.
    h bf16 [L+1,T,H], w bf16 [L,E,H], bias f32 [L,E] or None.
    ids_pred[l] = top-k(h[l] w[l]^T + b[l]) (lookahead of layer l),
    ids_act[l] = top-k(h[l+1] w[l]^T + b[l]) (normal router of layer l).
    Returns (ids_pred, ids_act) int32 [L,T,k], plus (logits_pred, logits_act)
    f32 [L,T,E] when want_logits."""
    lib = _load()
    _need(h, torch.bfloat16, "h")
    _need(w, torch.bfloat16, "w")
    if h.dim() != 3 or w.dim() != 3:
        raise ValueError("h must be [L+1,T,H] and w [L,E,H]")
    L1, T, H = h.shape
    L, E = w.shape[0], w.shape[1]
    if L1 != L + 1 or w.shape[2] != H:
        raise ValueError("h must be [L+1,T,H] for w [L,E,H]")
    if bias is not None:
        _need(bias, torch.float32, "bias")
        if bias.shape != (L, E):
            raise ValueError("bias must be [L,E]")
    outs = []
    for t in (ids_pred, ids_act):
        t = torch.empty(L, T, k, dtype=torch.int32, device=h.device) if t is None else t
        _need(t, torch.int32, "ids")
        if t.shape != (L, T, k):
            raise ValueError("ids outputs must be [L,T,k]")
        outs.append(t)
    lg = [None, None]
    if want_logits:
        lg = [torch.empty(L, T, E, dtype=torch.float32, device=h.device) if t is None else t
              for t in (logits_pred, logits_act)]
    _check("lb_predict_topk_chain", lib.lb_predict_topk_chain(_p(h), _p(w), _p(bias), L, T, H, E, k, _p(outs[0]),
                                                              _p(outs[1]), _p(lg[0]), _p(lg[1]), _stream()))
    return (outs[0], outs[1], lg[0], lg[1]) if want_logits else (outs[0], outs[1])


def lb_plan_swaps(cnt, placement=None, gamma=0.0, tau=0.0, alpha=0.0, beta=1.0, expert_bytes=0.0,
                  budget=float("inf"), link_budget=None, out=None):
    """Budgeted pairwise expert swaps (FreeBalance sec. 3.3).  cnt int32
    [B,G,E] (or [G,E]); placement int32 [B,E] or None (even).  Returns
    (placement_out [B,E], swaps [B,E//2,4], n_swaps [B], loads [B,G])."""
    lib = _load()
    squeeze = cnt.dim() == 2
    cnt = _batched(cnt, 3)
    _need(cnt, torch.int32, "cnt")
    B, G, E = cnt.shape
    if placement is not None:
        placement = _batched(placement, 2)
        _need(placement, torch.int32, "placement")
        if placement.shape != (B, E):
            raise ValueError("placement must be [B,E]")
    cap = int(lib.lb_swaps_capacity(E))
    if out is None:
        dev = cnt.device
        out = (torch.empty(B, E, dtype=torch.int32, device=dev), torch.empty(B, cap, 4, dtype=torch.int32, device=dev),
               torch.empty(B, dtype=torch.int32, device=dev), torch.empty(B, G, dtype=torch.int32, device=dev))
    pi_out, sw, ns, lo = out
    link_budget = budget if link_budget is None else link_budget
    _check("lb_plan_swaps", lib.lb_plan_swaps(_p(cnt), _p(placement), B, G, E, gamma, tau, alpha, beta, expert_bytes,
                                              budget, link_budget, _p(pi_out), _p(sw), _p(ns), _p(lo), _stream()))
    if squeeze:
        return pi_out[0], sw[0], ns[0], lo[0]
    return pi_out, sw, ns, lo


SPLIT_VARIANTS = ("relief", "no_reverse", "jacobi", "hash", "water", "proportional", "fp32", "q1120")


def lb_split_variant(cnt, plan, N, passes=12, variant="relief", out=None):
    """Relief's ablation variants (see include/lb.h); same shapes as lb_split."""
    lib = _load()
    v = SPLIT_VARIANTS.index(variant) if isinstance(variant, str) else int(variant)
    squeeze = cnt.dim() == 2
    cnt = _batched(cnt, 3)
    plan = _batched(plan, 2)
    _need(cnt, torch.int32, "cnt")
    B, G, E = cnt.shape
    if out is None:
        dev = cnt.device
        out = tuple(torch.zeros(*sh, dtype=torch.int32, device=dev) for sh in ((B, G * N), (B, G * N), (B, G), (B,)))
    tok, mass, loads, pr = out
    _check("lb_split_variant", lib.lb_split_variant(_p(cnt), _p(plan), B, G, E, N, passes, v, _p(tok), _p(mass),
                                                    _p(loads), _p(pr), _stream()))
    if squeeze:
        return tok[0], mass[0], loads[0], pr[0]
    return tok, mass, loads, pr


def lb_gate_tuning(stages=0, split=0, persistent=0, kbox=0, tiles_per_unit=0, max_ctas=0):
    _check("lb_gate_tuning", _load().lb_gate_tuning(stages, split, persistent, kbox, tiles_per_unit, max_ctas))


def lb_launch_options(programmatic_dependent_launch=1, max_block_threads=0):
    _check("lb_launch_options", _load().lb_launch_options(int(programmatic_dependent_launch), int(max_block_threads)))


# ------------------------------------------------------------------ step 2
def lb_count(ids, G, E, cnt=None):
    """ids int32 [B,T,k] (or [T,k]) -> cnt int32 [B,G,E] (or [G,E])."""
    lib = _load()
    squeeze = ids.dim() == 2
    ids = _batched(ids, 3)
    _need(ids, torch.int32, "ids")
    B, T, k = ids.shape
    if cnt is None:
        cnt = torch.empty(B, G, E, dtype=torch.int32, device=ids.device)
    _check("lb_count", lib.lb_count(_p(ids), B, T, k, E, G, _p(cnt), _stream()))
    return cnt[0] if squeeze else cnt


# ------------------------------------------------------------------ step 3
def lb_plan_bytes(G, E, N):
    return int(_load().lb_plan_bytes(G, E, N))


def plan_layout(G, E, N):
    lay = _Layout()
    _check("lb_plan_layout_of", _load().lb_plan_layout_of(G, E, N, ctypes.byref(lay)))
    return {n: int(getattr(lay, n)) for n, _ in _Layout._fields_}


def lb_plan_replicas(cnt, N, L, plan=None):
    """cnt int32 [B,G,E] (or [G,E]) -> plan blobs uint8 [B, lb_plan_bytes]."""
    lib = _load()
    cnt = _batched(cnt, 3)
    _need(cnt, torch.int32, "cnt")
    B, G, E = cnt.shape
    nb = lb_plan_bytes(G, E, N)
    if plan is None:
        plan = torch.empty(B, nb, dtype=torch.uint8, device=cnt.device)
    if plan.shape != (B, nb) or plan.data_ptr() % 256:
        raise ValueError("plan must be uint8 [B, lb_plan_bytes(G,E,N)], 256-byte aligned")
    _check("lb_plan_replicas", lib.lb_plan_replicas(_p(cnt), B, G, E, N, L, _p(plan), _stream()))
    return plan


def decode_plan(plan, G, E, N):
    """Host view of plan blobs: list (one per problem) of dicts of numpy arrays."""
    lay = plan_layout(G, E, N)
    raw = plan.detach().cpu().numpy()
    if raw.ndim == 1:
        raw = raw[None]
    GN = G * N
    out = []
    for row in raw:
        def i32(off, n):
            return row[off:off + 4 * n].view(np.int32).copy()
        hdr = i32(lay["hdr"], 16)
        ne, nr = int(hdr[0]), int(hdr[1])
        out.append(dict(
            n_edges=ne, n_rounds=nr, n_phase1=int(hdr[2]), n_phase2=int(hdr[3]),
            used=i32(lay["used"], G), slots=i32(lay["slots"], GN).reshape(G, N),
            slot_phase=i32(lay["slot_phase"], GN).reshape(G, N), plan_load=i32(lay["plan_load"], G),
            edge_u=i32(lay["edge_u"], GN)[:ne], edge_v=i32(lay["edge_v"], GN)[:ne],
            edge_e=i32(lay["edge_e"], GN)[:ne], edge_round=i32(lay["edge_round"], GN)[:ne],
            round_ptr=i32(lay["round_ptr"], GN + 1)[:nr + 1], rep_ptr=i32(lay["rep_ptr"], E + 1),
            rep_edge=i32(lay["rep_edge"], GN)[:ne],
            holds=row[lay["holds"]:lay["holds"] + G * E].copy().reshape(G, E)))
    return out


# ------------------------------------------------------------------ step 4
def lb_split(cnt, plan, N, passes=12, out=None):
    """Returns tok, mass int32 [B,G*N], loads int32 [B,G], passes_run int32 [B]."""
    lib = _load()
    cnt = _batched(cnt, 3)
    _need(cnt, torch.int32, "cnt")
    B, G, E = cnt.shape
    _need(plan, torch.uint8, "plan")
    if out is None:
        dev = cnt.device
        out = (torch.empty(B, G * N, dtype=torch.int32, device=dev), torch.empty(B, G * N, dtype=torch.int32, device=dev),
               torch.empty(B, G, dtype=torch.int32, device=dev), torch.empty(B, dtype=torch.int32, device=dev))
    tok, mass, loads, pr = out
    _check("lb_split", lib.lb_split(_p(cnt), _p(plan), B, G, E, N, passes, _p(tok), _p(mass), _p(loads),
                                    _p(pr), _stream()))
    return tok, mass, loads, pr


# ------------------------------------------------------------------ step 5
def lb_assign_workspace_bytes(B, T, k, G, E, N):
    return int(_load().lb_assign_workspace_bytes(B, T, k, G, E, N))


def lb_assign(ids, cnt, plan, tok, mass, N, out=None, workspace=None):
    """Returns dest int32 [B,T,k], perm int32 [B,T*k], offs int32 [B,G*E+1]."""
    lib = _load()
    ids, cnt = _batched(ids, 3), _batched(cnt, 3)
    _need(ids, torch.int32, "ids")
    _need(cnt, torch.int32, "cnt")
    B, T, k = ids.shape
    _, G, E = cnt.shape
    dev = ids.device
    if out is None:
        out = (torch.empty(B, T, k, dtype=torch.int32, device=dev), torch.empty(B, T * k, dtype=torch.int32, device=dev),
               torch.empty(B, G * E + 1, dtype=torch.int32, device=dev))
    dest, perm, offs = out
    nbytes = lb_assign_workspace_bytes(B, T, k, G, E, N)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=dev)
    _check("lb_assign", lib.lb_assign(_p(ids), _p(cnt), _p(plan), _p(tok), _p(mass), B, T, k, G, E, N,
                                      _p(dest), _p(perm), _p(offs), _p(workspace), workspace.numel(), _stream()))
    return dest, perm, offs


def lb_decide(cnt, ids, plan, N, passes=12, cnt_pred=None, L=0, out=None, workspace=None):
    """Plan (from cnt_pred, when given; else plan is an input), split and
    assign in two launches.  Returns (tok, mass, loads, passes_run, dest,
    perm, offs); out preallocates them."""
    lib = _load()
    ids, cnt = _batched(ids, 3), _batched(cnt, 3)
    _need(ids, torch.int32, "ids")
    _need(cnt, torch.int32, "cnt")
    if cnt_pred is not None:
        cnt_pred = _batched(cnt_pred, 3)
        _need(cnt_pred, torch.int32, "cnt_pred")
    B, T, k = ids.shape
    _, G, E = cnt.shape
    dev = ids.device
    if out is None:
        i32 = dict(dtype=torch.int32, device=dev)
        out = (torch.empty(B, G * N, **i32), torch.empty(B, G * N, **i32), torch.empty(B, G, **i32),
               torch.empty(B, **i32), torch.empty(B, T, k, **i32), torch.empty(B, T * k, **i32),
               torch.empty(B, G * E + 1, **i32))
    tok, mass, loads, passes_run, dest, perm, offs = out
    nbytes = lb_assign_workspace_bytes(B, T, k, G, E, N)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=dev)
    _check("lb_decide", lib.lb_decide(_p(cnt_pred), _p(cnt), _p(ids), _p(plan), B, T, k, G, E, N, L, passes,
                                      _p(tok), _p(mass), _p(loads), _p(passes_run), _p(dest), _p(perm), _p(offs),
                                      _p(workspace), workspace.numel(), _stream()))
    return out


def lb_solve(ids, plan, G, E, N, passes=12, out=None, workspace=None):
    """Count + split + assign in one launch.  out = (cnt, tok, mass, loads,
    passes_run, dest, perm, offs) preallocated, or None."""
    lib = _load()
    ids = _batched(ids, 3)
    _need(ids, torch.int32, "ids")
    B, T, k = ids.shape
    dev = ids.device
    if out is None:
        i32 = dict(dtype=torch.int32, device=dev)
        out = (torch.empty(B, G, E, **i32), torch.empty(B, G * N, **i32), torch.empty(B, G * N, **i32),
               torch.empty(B, G, **i32), torch.empty(B, **i32), torch.empty(B, T, k, **i32),
               torch.empty(B, T * k, **i32), torch.empty(B, G * E + 1, **i32))
    cnt, tok, mass, loads, pr, dest, perm, offs = out
    nbytes = lb_assign_workspace_bytes(B, T, k, G, E, N)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=dev)
    _check("lb_solve", lib.lb_solve(_p(ids), _p(plan), B, T, k, G, E, N, passes, _p(cnt), _p(tok), _p(mass),
                                    _p(loads), _p(pr), _p(dest), _p(perm), _p(offs), _p(workspace),
                                    workspace.numel(), _stream()))
    return out


def lb_assign_noalloc(ids, cnt, plan, tok, mass, N, out=None):
    """lb_assign for callers that cannot provide device scratch memory: the
    library uses its own fixed device array instead (see include/lb.h).
    Output buffers are still the caller's; pass `out` to avoid allocating
    them here.  Calls that overlap on the GPU race on the shared array."""
    lib = _load()
    ids, cnt = _batched(ids, 3), _batched(cnt, 3)
    _need(ids, torch.int32, "ids")
    _need(cnt, torch.int32, "cnt")
    B, T, k = ids.shape
    _, G, E = cnt.shape
    dev = ids.device
    if out is None:
        out = (torch.empty(B, T, k, dtype=torch.int32, device=dev), torch.empty(B, T * k, dtype=torch.int32, device=dev),
               torch.empty(B, G * E + 1, dtype=torch.int32, device=dev))
    dest, perm, offs = out
    _check("lb_assign_noalloc", lib.lb_assign_noalloc(_p(ids), _p(cnt), _p(plan), _p(tok), _p(mass), B, T, k, G, E,
                                                      N, _p(dest), _p(perm), _p(offs), _stream()))
    return dest, perm, offs


# ------------------------------------------------------------------ status
def lb_get_status(clear=True):
    """Synchronizes the device; returns the LB_DEV_* bits seen since the last clear."""
    flags = ctypes.c_int32(0)
    rc = _load().lb_get_status(ctypes.byref(flags), 1 if clear else 0)
    if rc not in (LB_OK, LB_EDATA):
        raise LBError("lb_get_status", rc)
    return int(flags.value)


def lb_version():
    return int(_load().lb_version())


EXPORTS = ("lb_predict_topk", "lb_predict_topk_chain", "lb_gate_tuning", "lb_launch_options", "lb_plan_swaps", "lb_swaps_capacity",
           "lb_split_variant", "lb_count", "lb_plan_bytes", "lb_plan_layout_of",
           "lb_plan_replicas", "lb_split", "lb_assign_workspace_bytes", "lb_assign", "lb_assign_noalloc", "lb_decide",
           "lb_solve",
           "lb_get_status",
           "lb_strerror", "lb_last_error", "lb_version")
