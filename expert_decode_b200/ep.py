"""The expert-parallel form across ranks, over the C ABI.

fak note "GLM-5.2 multi-GPU", "What landed": the experts are split into
contiguous bands (ep_plan), every rank holds the weights of its band and
computes the partial FFN output of the picks in it, and the partials are
summed in rank order (TensorFold #310: one fixed order of that sum).

  moe_ffn_partial  one rank's band partial (band-resident expert weights)
  moe_ep_combine   y = the partials left-folded in rank order, then + the
                   shared expert's output
  shared_expert    the shared expert's output alone (moe_ffn_forward with
                   every pick slot empty)
  ep_forward       one rank's share of the layer: its partial, then one of
                   two exchanges over a torch.distributed process group (NCCL
                   between GPUs), after which every rank holds the same y:
                   "reduce_scatter" (default): rank j receives row slice j of
                     every rank's partial (one all-to-all), folds them in rank
                     order with the shared expert of its rows only, and the
                     folded slices are all-gathered: 2 (R - 1) / R of a
                     partial's bytes in and out per rank (TensorFold #310,
                     maintainer's reply: the exact reduce-scatter in rank
                     order);
                   "all_gather": every rank gathers every partial and folds
                     all rows itself: (R - 1) partials in per rank

Argument marshalling only: every step runs in the library's kernels.
"""
import ctypes

import torch

from .api import (EP_OK, EPError, Plan, _check, _dense, _dtype, _ptr, _stream, library,
                  moe_ffn_forward)

EP_ID_NONE = -(1 << 31)

_declared = False


def _lib():
    global _declared
    lib = library()
    if not _declared:
        P, I64, I32, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
        lib.moe_ffn_partial_workspace_size.argtypes = [I64, I64, I64, I32, I64]
        lib.moe_ffn_partial_workspace_size.restype = SZ
        lib.moe_ffn_partial.argtypes = [P, ctypes.c_int, I64, I64, P, P, I32, P, P, P, I64,
                                        ctypes.POINTER(Plan), I32, P, P, SZ, P]
        lib.moe_ffn_partial.restype = ctypes.c_int
        lib.moe_ep_combine.argtypes = [P, I64, I64, P, I32, ctypes.POINTER(Plan), P, P, P]
        lib.moe_ep_combine.restype = ctypes.c_int
        _declared = True
    return lib


def moe_ffn_partial_workspace_size(T, H, E_band, top_k, I):
    return int(_lib().moe_ffn_partial_workspace_size(int(T), int(H), int(E_band), int(top_k),
                                                     int(I)))


def moe_ffn_partial(x, ids, weights, w_gate, w_up, w_down, plan, rank, partial=None,
                    workspace=None, stream=None):
    """partial [T, H] fp32 of band `rank`; w_* hold that band's experts only."""
    _dense(x, "x", ndim=2)
    _dense(ids, "ids", torch.int32, 2)
    _dense(weights, "weights", torch.float32, 2)
    for name, t in (("w_gate", w_gate), ("w_up", w_up), ("w_down", w_down)):
        _dense(t, name, torch.bfloat16, 3)
    T, H = x.shape
    top_k = ids.shape[1]
    E_band, I = w_gate.shape[0], w_gate.shape[1]
    if partial is None:
        partial = torch.empty((T, H), dtype=torch.float32, device=x.device)
    _dense(partial, "partial", torch.float32, 2)
    need = moe_ffn_partial_workspace_size(T, H, E_band, top_k, I)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=x.device)
    _check(_lib().moe_ffn_partial(
        _ptr(x), _dtype(x), T, H, _ptr(ids), _ptr(weights), top_k, _ptr(w_gate), _ptr(w_up),
        _ptr(w_down), I, ctypes.byref(plan), int(rank), _ptr(partial), _ptr(workspace),
        workspace.numel(), _stream(stream)))
    return partial


def moe_ep_combine(partials, ids, plan, shared=None, y=None, stream=None):
    """y [T, H] fp32 from partials [bands, T, H] (rank r's at r)."""
    _dense(partials, "partials", torch.float32, 3)
    _dense(ids, "ids", torch.int32, 2)
    _dense(shared, "shared", torch.float32, 2)
    R, T, H = partials.shape
    if R != plan.bands:
        raise ValueError(f"{R} partials for a plan of {plan.bands} bands")
    if y is None:
        y = torch.empty((T, H), dtype=torch.float32, device=partials.device)
    _dense(y, "y", torch.float32, 2)
    _check(_lib().moe_ep_combine(_ptr(partials), T, H, _ptr(ids), ids.shape[1],
                                 ctypes.byref(plan), _ptr(shared), _ptr(y), _stream(stream)))
    return y


def shared_expert(x, ws_gate, ws_up, ws_down, stream=None):
    """The shared expert's output [T, H] fp32: the forward with every pick slot empty."""
    T, H = x.shape
    ids = torch.full((T, 1), EP_ID_NONE, dtype=torch.int32, device=x.device)
    w = torch.zeros((T, 1), dtype=torch.float32, device=x.device)
    # the routed weights are never read without a pick: the shared ones stand in
    wg, wu, wd = ws_gate.unsqueeze(0), ws_up.unsqueeze(0), ws_down.unsqueeze(0)
    one = Plan()
    _check(library().ep_plan(1, 1, ctypes.byref(one)))
    return moe_ffn_forward(x, ids, w, wg, wu, wd, (ws_gate, ws_up, ws_down), one, stream=stream)


class _Ops:
    """The compute steps of ep_forward (the library's kernels by default)."""
    partial = staticmethod(moe_ffn_partial)
    combine = staticmethod(moe_ep_combine)
    shared = staticmethod(shared_expert)


def row_slices(T, ranks):
    """Row offsets [ranks + 1] of the row slices of the reduce-scatter: whole
    rows, as even as they go, the first T % ranks slices one row longer (the
    share rule of ep_plan, applied to rows; a slice may be empty)."""
    base, extra = divmod(int(T), int(ranks))
    out = [0]
    for j in range(ranks):
        out.append(out[-1] + base + (1 if j < extra else 0))
    return out


def ep_forward(x, ids, weights, band_experts, shared, plan, rank, group=None, ops=_Ops,
               exchange="reduce_scatter"):
    """One rank's share of the expert-parallel layer.

    band_experts = (w_gate, w_up, w_down) of this rank's band; shared =
    (ws_gate, ws_up, ws_down) replicated on every rank, or None.  The partials
    are exchanged over `group` (torch.distributed) and folded in rank order,
    so every rank returns the same y [T, H], bit for bit the same whichever
    exchange runs (each row's fold is the same additions in the same order).
    """
    import torch.distributed as dist
    w_gate, w_up, w_down = band_experts
    part = ops.partial(x, ids, weights, w_gate, w_up, w_down, plan, rank).contiguous()
    world = dist.get_world_size(group)
    if world != plan.bands:
        raise ValueError(f"{world} ranks for a plan of {plan.bands} bands")
    T, H = part.shape
    if exchange == "all_gather":
        slots = [torch.empty_like(part) for _ in range(world)]
        dist.all_gather(slots, part, group=group)
        gathered = torch.stack(slots)  # rank r's partial at r
        s = None if shared is None else ops.shared(x, *shared)
        return ops.combine(gathered, ids, plan, s)
    if exchange != "reduce_scatter":
        raise ValueError(f"unknown exchange {exchange!r}")
    # row slice j of every rank's partial to rank j, in rank order
    rs = row_slices(T, world)
    sizes = [rs[j + 1] - rs[j] for j in range(world)]
    lo, hi = rs[rank], rs[rank + 1]
    mine = torch.empty((world * sizes[rank], H), dtype=part.dtype, device=part.device)
    dist.all_to_all_single(mine, part, output_split_sizes=[sizes[rank]] * world,
                           input_split_sizes=sizes, group=group)
    s = None if shared is None else ops.shared(x[lo:hi], *shared)
    y_mine = ops.combine(mine.view(world, sizes[rank], H), ids[lo:hi].contiguous(), plan, s)
    # the folded slices to every rank (padded to the longest slice)
    pad = max(sizes)
    send = torch.zeros((pad, H), dtype=part.dtype, device=part.device)
    send[:sizes[rank]] = y_mine
    every = torch.empty((world * pad, H), dtype=part.dtype, device=part.device)
    dist.all_gather_into_tensor(every, send, group=group)
    every = every.view(world, pad, H)
    return torch.cat([every[j, :sizes[j]] for j in range(world)], dim=0)


__all__ = ["EP_ID_NONE", "moe_ffn_partial_workspace_size", "moe_ffn_partial", "moe_ep_combine",
           "shared_expert", "ep_forward", "row_slices", "EPError", "EP_OK"]
