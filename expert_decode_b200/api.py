"""ctypes binding of the C ABI in include/expert_decode.h.

Argument marshalling only: each wrapper checks that the torch tensors have the
layout the ABI documents, passes their device pointers and sizes, and raises
EPError when the library returns a status other than EP_OK.  Outputs that the
caller does not pass are allocated with torch (device memory is plumbing).
The library must be present: there is no fallback of any kind.
"""
import ctypes
import os
import threading

import torch

EP_OK, EP_EINVAL, EP_EDIM, EP_EBADID, EP_ENOMEM, EP_ECUDA, EP_ETIMEOUT = range(7)
EP_BF16, EP_F32 = 0, 1
EP_MAX_BANDS = 64
_DISPATCH = {"auto": 0, "streaming": 1, "tensor": 2, "streaming_tc": 3, "streaming_simt": 4}
_NAMES = {0: "EP_OK", 1: "EP_EINVAL", 2: "EP_EDIM", 3: "EP_EBADID", 4: "EP_ENOMEM",
          5: "EP_ECUDA", 6: "EP_ETIMEOUT"}

library_path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib",
                            "libexpert_decode.so")


class EPError(RuntimeError):
    def __init__(self, code, message):
        super().__init__(f"{_NAMES.get(code, code)}: {message}")
        self.code = code


class WorkspaceLayout(ctypes.Structure):
    _fields_ = [("bytes", ctypes.c_size_t), ("contrib_offset", ctypes.c_size_t),
                ("shared_offset", ctypes.c_size_t), ("group_offset_offset", ctypes.c_size_t),
                ("perm_offset", ctypes.c_size_t)]


class NvFp4(ctypes.Structure):
    """ep_nvfp4_t: codes and block scales on the device, one fp32 tensor scale."""
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("tensor_scale", ctypes.c_float)]


class Plan(ctypes.Structure):
    _fields_ = [("num_experts", ctypes.c_int32), ("bands", ctypes.c_int32),
                ("band_start", ctypes.c_int32 * (EP_MAX_BANDS + 1))]

    def starts(self):
        return [self.band_start[r] for r in range(self.bands + 1)]


_lock = threading.Lock()
_lib = None


def library():
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(library_path):
                raise RuntimeError(f"CUDA library {library_path} is missing: build it with "
                                   "`python -c 'import __graft_entry__ as g; g.build()'`")
            lib = ctypes.CDLL(library_path)
            P, I64, I32, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
            lib.ep_plan.argtypes = [I32, I32, ctypes.POINTER(Plan)]
            lib.moe_route.argtypes = [P, ctypes.c_int, I64, I64, P, P, I64, I32, P, P, P]
            lib.moe_route_logits.argtypes = [P, ctypes.c_int, I64, I64, P, P, I64, P, P, P]
            lib.moe_route_sigmoid.argtypes = [P, ctypes.c_int, I64, I64, P, P, I64, I32, I32,
                                              ctypes.c_float, P, P, P]
            lib.moe_ffn_workspace_size.argtypes = [I64, I64, I64, I32, I64, I64]
            lib.moe_ffn_workspace_size.restype = SZ
            lib.moe_ffn_workspace_layout.argtypes = [I64, I64, I64, I32, I64, I64,
                                                     ctypes.POINTER(WorkspaceLayout)]
            lib.moe_ffn_forward.argtypes = [P, ctypes.c_int, I64, I64, P, P, I32, P, P, P, I64,
                                            I64, P, P, P, I64, ctypes.POINTER(Plan), P, P, SZ, P]
            lib.moe_ffn_forward_noalloc.argtypes = [P, ctypes.c_int, I64, I64, P, P, I32, P, P,
                                                    P, I64, I64, P, P, P, I64,
                                                    ctypes.POINTER(Plan), P, P]
            F4 = ctypes.POINTER(NvFp4)
            lib.moe_ffn_nvfp4_workspace_size.argtypes = [I64, I64, I64, I32, I64, I64]
            lib.moe_ffn_nvfp4_workspace_size.restype = SZ
            lib.moe_ffn_forward_nvfp4.argtypes = [P, I64, I64, P, P, I32, F4, F4, F4, I64, I64,
                                                  F4, F4, F4, I64, ctypes.POINTER(Plan), P, P,
                                                  SZ, P]
            lib.ep_set_dispatch.argtypes = [ctypes.c_int]
            lib.ep_set_router.argtypes = [ctypes.c_int]
            lib.ep_check_status.argtypes = [P]
            lib.ep_last_error.restype = ctypes.c_char_p
            lib.ep_last_launch_count.restype = I32
            lib.ep_profile_events.argtypes = [P, I32]
            lib.ep_profile_events.restype = ctypes.c_int
            for fn in ("ep_plan", "moe_route", "moe_route_logits", "moe_route_sigmoid",
                       "moe_ffn_forward",
                       "moe_ffn_workspace_layout",
                       "moe_ffn_forward_noalloc", "moe_ffn_forward_nvfp4",
                       "ep_set_dispatch", "ep_set_router", "ep_check_status"):
                getattr(lib, fn).restype = ctypes.c_int
            _lib = lib
        return _lib


def _check(rc):
    if rc != EP_OK:
        raise EPError(rc, library().ep_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype(x):
    if x.dtype == torch.bfloat16:
        return EP_BF16
    if x.dtype == torch.float32:
        return EP_F32
    raise TypeError(f"activations must be bf16 or fp32, got {x.dtype}")


def _dense(t, name, dtype=None, ndim=None):
    if t is None:
        return
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous (row-major)")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions")


def ep_plan(num_experts, bands):
    plan = Plan()
    _check(library().ep_plan(int(num_experts), int(bands), ctypes.byref(plan)))
    return plan


def moe_route(x, w_router, bias, top_k, ids=None, weights=None, stream=None):
    """ids [T, top_k] int32 and weights [T, top_k] fp32 of the replicated router."""
    _dense(x, "x", ndim=2)
    _dense(w_router, "w_router", torch.bfloat16, 2)
    _dense(bias, "bias", torch.float32, 1)
    T, H = x.shape
    E = w_router.shape[0]
    if ids is None:
        ids = torch.empty((T, top_k), dtype=torch.int32, device=x.device)
    if weights is None:
        weights = torch.empty((T, top_k), dtype=torch.float32, device=x.device)
    _dense(ids, "ids", torch.int32)
    _dense(weights, "weights", torch.float32)
    _check(library().moe_route(_ptr(x), _dtype(x), T, H, _ptr(w_router), _ptr(bias), E,
                               int(top_k), _ptr(ids), _ptr(weights), _stream(stream)))
    return ids, weights


def moe_route_logits(x, w_router, bias, stream=None):
    """(logits, bounds) [T, E] fp32: the router's fp32 logits above 32 tokens
    and the bound of each one's error (inspection)."""
    _dense(x, "x", ndim=2)
    _dense(w_router, "w_router", torch.bfloat16, 2)
    _dense(bias, "bias", torch.float32, 1)
    T, H = x.shape
    E = w_router.shape[0]
    logits = torch.empty((T, E), dtype=torch.float32, device=x.device)
    bounds = torch.empty((T, E), dtype=torch.float32, device=x.device)
    _check(library().moe_route_logits(_ptr(x), _dtype(x), T, H, _ptr(w_router), _ptr(bias), E,
                                      _ptr(logits), _ptr(bounds), _stream(stream)))
    return logits, bounds


def moe_route_sigmoid(x, w_router, bias, top_k, normalize=False, scale=1.0, ids=None,
                      weights=None, stream=None):
    """ids and weights of the sigmoid router variant (bias selects only)."""
    _dense(x, "x", ndim=2)
    _dense(w_router, "w_router", torch.bfloat16, 2)
    _dense(bias, "bias", torch.float32, 1)
    T, H = x.shape
    E = w_router.shape[0]
    if ids is None:
        ids = torch.empty((T, top_k), dtype=torch.int32, device=x.device)
    if weights is None:
        weights = torch.empty((T, top_k), dtype=torch.float32, device=x.device)
    _dense(ids, "ids", torch.int32)
    _dense(weights, "weights", torch.float32)
    _check(library().moe_route_sigmoid(_ptr(x), _dtype(x), T, H, _ptr(w_router), _ptr(bias), E,
                                       int(top_k), 1 if normalize else 0, float(scale),
                                       _ptr(ids), _ptr(weights), _stream(stream)))
    return ids, weights


def moe_ffn_workspace_size(T, H, E, top_k, I, I_s):
    return int(library().moe_ffn_workspace_size(int(T), int(H), int(E), int(top_k), int(I),
                                                int(I_s)))


def moe_ffn_workspace_layout(T, H, E, top_k, I, I_s):
    """Byte offsets, inside moe_ffn_forward's workspace, of the per-pick
    contributions [T * top_k, H] fp32 and the shared expert's output [T, H]
    fp32 that the tensor-core paths fold into y; returns a WorkspaceLayout."""
    out = WorkspaceLayout()
    _check(library().moe_ffn_workspace_layout(int(T), int(H), int(E), int(top_k), int(I),
                                              int(I_s), ctypes.byref(out)))
    return out


def moe_ffn_forward(x, ids, weights, w_gate, w_up, w_down, shared, plan, y=None,
                    workspace=None, stream=None):
    """y [T, H] fp32 of the routed MoE FFN; shared = (ws_gate, ws_up, ws_down) or None."""
    _dense(x, "x", ndim=2)
    _dense(ids, "ids", torch.int32, 2)
    _dense(weights, "weights", torch.float32, 2)
    for name, t in (("w_gate", w_gate), ("w_up", w_up), ("w_down", w_down)):
        _dense(t, name, torch.bfloat16, 3)
    T, H = x.shape
    top_k = ids.shape[1]
    E, I = w_gate.shape[0], w_gate.shape[1]
    if shared is not None:
        ws_gate, ws_up, ws_down = shared
        for name, t in (("ws_gate", ws_gate), ("ws_up", ws_up), ("ws_down", ws_down)):
            _dense(t, name, torch.bfloat16, 2)
        I_s = ws_gate.shape[0]
    else:
        ws_gate = ws_up = ws_down = None
        I_s = 0
    if y is None:
        y = torch.empty((T, H), dtype=torch.float32, device=x.device)
    _dense(y, "y", torch.float32, 2)
    need = moe_ffn_workspace_size(T, H, E, top_k, I, I_s)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=x.device)
    _check(library().moe_ffn_forward(
        _ptr(x), _dtype(x), T, H, _ptr(ids), _ptr(weights), top_k, _ptr(w_gate), _ptr(w_up),
        _ptr(w_down), E, I, _ptr(ws_gate), _ptr(ws_up), _ptr(ws_down), I_s, ctypes.byref(plan),
        _ptr(y), _ptr(workspace), workspace.numel(), _stream(stream)))
    return y


def moe_ffn_forward_noalloc(x, ids, weights, w_gate, w_up, w_down, shared, plan, y,
                            stream=None):
    """moe_ffn_forward into the caller's y [T, H] fp32, with the library's static
    scratch in place of a workspace: neither this wrapper nor the library
    allocates anything."""
    _dense(x, "x", ndim=2)
    _dense(ids, "ids", torch.int32, 2)
    _dense(weights, "weights", torch.float32, 2)
    for name, t in (("w_gate", w_gate), ("w_up", w_up), ("w_down", w_down)):
        _dense(t, name, torch.bfloat16, 3)
    _dense(y, "y", torch.float32, 2)
    T, H = x.shape
    E, I = w_gate.shape[0], w_gate.shape[1]
    if shared is not None:
        ws_gate, ws_up, ws_down = shared
        for name, t in (("ws_gate", ws_gate), ("ws_up", ws_up), ("ws_down", ws_down)):
            _dense(t, name, torch.bfloat16, 2)
        I_s = ws_gate.shape[0]
    else:
        ws_gate = ws_up = ws_down = None
        I_s = 0
    _check(library().moe_ffn_forward_noalloc(
        _ptr(x), _dtype(x), T, H, _ptr(ids), _ptr(weights), ids.shape[1], _ptr(w_gate),
        _ptr(w_up), _ptr(w_down), E, I, _ptr(ws_gate), _ptr(ws_up), _ptr(ws_down), I_s,
        ctypes.byref(plan), _ptr(y), _stream(stream)))
    return y


def _nvfp4(m, name, mats, rows, cols):
    """m = {"packed": uint8 [mats,] rows, cols / 2; "scales": uint8 [mats,]
    rows, cols / 16; "tensor_scale": float} -> NvFp4 (keeps no reference)."""
    packed, scales = m["packed"], m["scales"]
    lead = (mats,) if mats is not None else ()
    for what, t, shape in (("packed", packed, lead + (rows, cols // 2)),
                           ("scales", scales, lead + (rows, cols // 16))):
        _dense(t, f"{name}.{what}", torch.uint8)
        if tuple(t.shape) != shape:
            raise ValueError(f"{name}.{what} must be {shape}, got {tuple(t.shape)}")
    return NvFp4(packed.data_ptr(), scales.data_ptr(), float(m["tensor_scale"]))


def moe_ffn_nvfp4_workspace_size(T, H, E, top_k, I, I_s):
    return int(library().moe_ffn_nvfp4_workspace_size(int(T), int(H), int(E), int(top_k),
                                                      int(I), int(I_s)))


def moe_ffn_forward_nvfp4(x, ids, weights, w_gate, w_up, w_down, shared, plan, y=None,
                          workspace=None, stream=None):
    """y [T, H] fp32 of the routed MoE FFN for a decode batch (T <= 8) with
    NVFP4 experts.  w_gate, w_up: {"packed" [E, I, H/2], "scales" [E, I, H/16],
    "tensor_scale"}; w_down: [E, H, I/2], [E, H, I/16]; shared = (ws_gate,
    ws_up, ws_down) of the same form without the expert dimension, or None."""
    _dense(x, "x", torch.bfloat16, 2)
    _dense(ids, "ids", torch.int32, 2)
    _dense(weights, "weights", torch.float32, 2)
    T, H = x.shape
    top_k = ids.shape[1]
    E, I = w_gate["packed"].shape[0], w_gate["packed"].shape[1]
    g, u, d = (_nvfp4(w_gate, "w_gate", E, I, H), _nvfp4(w_up, "w_up", E, I, H),
               _nvfp4(w_down, "w_down", E, H, I))
    if shared is not None:
        I_s = shared[0]["packed"].shape[0]
        sg, su, sd = (_nvfp4(shared[0], "ws_gate", None, I_s, H),
                      _nvfp4(shared[1], "ws_up", None, I_s, H),
                      _nvfp4(shared[2], "ws_down", None, H, I_s))
        sp = [ctypes.byref(sg), ctypes.byref(su), ctypes.byref(sd)]
    else:
        I_s = 0
        sp = [None, None, None]
    if y is None:
        y = torch.empty((T, H), dtype=torch.float32, device=x.device)
    _dense(y, "y", torch.float32, 2)
    need = moe_ffn_nvfp4_workspace_size(T, H, E, top_k, I, I_s)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=x.device)
    _check(library().moe_ffn_forward_nvfp4(
        _ptr(x), T, H, _ptr(ids), _ptr(weights), top_k, ctypes.byref(g), ctypes.byref(u),
        ctypes.byref(d), E, I, *sp, I_s, ctypes.byref(plan), _ptr(y), _ptr(workspace),
        workspace.numel(), _stream(stream)))
    return y


def ep_check_status(stream=None):
    _check(library().ep_check_status(_stream(stream)))


def ep_set_dispatch(mode):
    """Process-wide path choice: "auto", "tensor", "streaming" (kernels as in
    auto), "streaming_tc" (gate/up and down on the tensor cores, then the
    fold) or "streaming_simt" (gate/up, then down with the fold, on the CUDA
    cores)."""
    _check(library().ep_set_dispatch(_DISPATCH[mode]))


_ROUTER = {"auto": 0, "tiled": 1, "tensor": 2}


def ep_set_router(mode):
    """Process-wide router choice above 32 tokens: "auto", "tiled" (CUDA-core
    fp32 logits) or "tensor" (tcgen05 logits)."""
    _check(library().ep_set_router(_ROUTER[mode]))


def ep_last_launch_count():
    return int(library().ep_last_launch_count())


_profile_keep = threading.local()


def ep_profile_events(events):
    """Bracket each kernel of later calls (this thread) with these torch.cuda.Events:
    kernel j between events[2j] and events[2j+1].  None stops.  Each event must
    have been recorded once so that its CUDA handle exists."""
    if events is None:
        _profile_keep.arr = None
        _check(library().ep_profile_events(None, 0))
        return
    arr = (ctypes.c_void_p * len(events))(*[ctypes.c_void_p(e.cuda_event) for e in events])
    _profile_keep.arr = arr
    _check(library().ep_profile_events(ctypes.cast(arr, ctypes.c_void_p), len(events)))
