"""numpy/ctypes front end of the fp64 CPU oracle (test infrastructure only).

Only tests/, __graft_entry__.smoke() and the cpu_baseline / reference legs of
bench.py may import this module.  It imports nothing from the CUDA package.

Array conventions: bf16 tensors are passed as numpy uint16 arrays holding the
bf16 bit patterns; fp32 activations as float32.  Expert weights are either a
contiguous [E, rows, cols] uint16 array or a mapping {expert id: 2-D array}
that holds only the experts a call touches (the rest stay absent, and a pick
of an absent expert is an error).
"""
import ctypes
import os

import numpy as np

from . import build as _build

OK, EINVAL, EPLAN, EBADID = 0, -1, -2, -3


class OracleError(RuntimeError):
    def __init__(self, code, what):
        names = {EINVAL: "invalid argument", EPLAN: "plan refused", EBADID: "expert id out of range"}
        super().__init__(f"oracle {what}: {names.get(code, code)}")
        self.code = code


_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I32 = ctypes.c_int32
_INT = ctypes.c_int


def _ptr(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


class Oracle:
    def __init__(self, path=None):
        path = path or _build.build()
        self.path = path
        lib = ctypes.CDLL(path)
        lib.oracle_expert_parallel_plan.argtypes = [_I64, _I64, _I32, _P]
        lib.oracle_route.argtypes = [_P, _INT, _I64, _I64, _P, _P, _I64, _I32, _P, _P, _P, _INT]
        lib.oracle_route_sigmoid.argtypes = [_P, _INT, _I64, _I64, _P, _P, _I64, _I32, _INT,
                                             ctypes.c_double, _P, _P, _P, _P, _INT]
        lib.oracle_expert_swiglu.argtypes = [_P, _P, _P, _P, _I64, _I64, _P]
        common = [_P, _INT, _I64, _I64, _P, _P, _I32, _P, _P, _P, _I64, _I64, _P, _P, _P, _I64]
        lib.oracle_moe_ffn_monolith.argtypes = common + [_P, _INT]
        lib.oracle_moe_ffn_expert_parallel.argtypes = common + [_P, _I32, _P, _INT]
        lib.oracle_max_threads.argtypes = []
        for fn in ("oracle_expert_parallel_plan", "oracle_route", "oracle_route_sigmoid",
                   "oracle_expert_swiglu",
                   "oracle_moe_ffn_monolith", "oracle_moe_ffn_expert_parallel",
                   "oracle_max_threads"):
            getattr(lib, fn).restype = ctypes.c_int
        self.lib = lib

    # -- plan ---------------------------------------------------------------
    def expert_parallel_plan(self, extent, ranks, unit=1):
        start = np.zeros(max(int(ranks), 0) + 1, dtype=np.int64)
        rc = self.lib.oracle_expert_parallel_plan(int(extent), int(unit), int(ranks), _ptr(start))
        if rc != OK:
            raise OracleError(rc, "plan")
        return start

    # -- router -------------------------------------------------------------
    @staticmethod
    def _activations(x):
        x = np.ascontiguousarray(x)
        if x.dtype == np.float32:
            return x, 1
        if x.dtype == np.uint16:
            return x, 0
        raise TypeError("activations must be float32 or bf16 bits (uint16)")

    def route(self, x, w_router, bias, top_k, threads=None):
        x, is_f32 = self._activations(x)
        T, H = x.shape
        w_router = np.ascontiguousarray(w_router, dtype=np.uint16)
        E = w_router.shape[0]
        assert w_router.shape == (E, H)
        b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float64)
        ids = np.zeros((T, top_k), dtype=np.int32)
        weights = np.zeros((T, top_k), dtype=np.float64)
        logits = np.zeros((T, E), dtype=np.float64)
        rc = self.lib.oracle_route(_ptr(x), is_f32, T, H, _ptr(w_router), _ptr(b), E, int(top_k),
                                   _ptr(ids), _ptr(weights), _ptr(logits), self._threads(threads))
        if rc != OK:
            raise OracleError(rc, "route")
        return ids, weights, logits

    def route_sigmoid(self, x, w_router, bias, top_k, normalize=False, scale=1.0, threads=None):
        """The sigmoid router variant: ids, weights, keys (s + b), scores (s)."""
        x, is_f32 = self._activations(x)
        T, H = x.shape
        w_router = np.ascontiguousarray(w_router, dtype=np.uint16)
        E = w_router.shape[0]
        assert w_router.shape == (E, H)
        b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float64)
        ids = np.zeros((T, top_k), dtype=np.int32)
        weights = np.zeros((T, top_k), dtype=np.float64)
        keys = np.zeros((T, E), dtype=np.float64)
        scores = np.zeros((T, E), dtype=np.float64)
        rc = self.lib.oracle_route_sigmoid(_ptr(x), is_f32, T, H, _ptr(w_router), _ptr(b), E,
                                           int(top_k), 1 if normalize else 0, float(scale),
                                           _ptr(ids), _ptr(weights), _ptr(keys), _ptr(scores),
                                           self._threads(threads))
        if rc != OK:
            raise OracleError(rc, "route_sigmoid")
        return ids, weights, keys, scores

    # -- experts ------------------------------------------------------------
    def expert_swiglu(self, xt, w_gate, w_up, w_down):
        xt = np.ascontiguousarray(xt, dtype=np.float64)
        w_gate = np.ascontiguousarray(w_gate, dtype=np.uint16)
        w_up = np.ascontiguousarray(w_up, dtype=np.uint16)
        w_down = np.ascontiguousarray(w_down, dtype=np.uint16)
        I, H = w_gate.shape
        out = np.zeros(H, dtype=np.float64)
        rc = self.lib.oracle_expert_swiglu(_ptr(xt), _ptr(w_gate), _ptr(w_up), _ptr(w_down), H, I, _ptr(out))
        if rc != OK:
            raise OracleError(rc, "expert_swiglu")
        return out

    @staticmethod
    def _expert_table(w, E):
        """Pointer table over the experts; keeps the arrays alive in `keep`."""
        table = (ctypes.c_void_p * E)()
        keep = []
        if isinstance(w, dict):
            for e, a in w.items():
                a = np.ascontiguousarray(a, dtype=np.uint16)
                keep.append(a)
                table[int(e)] = a.ctypes.data
            shape = keep[0].shape if keep else None
        else:
            a = np.ascontiguousarray(w, dtype=np.uint16)
            assert a.shape[0] == E
            keep.append(a)
            stride = a.strides[0]
            for e in range(E):
                table[e] = a.ctypes.data + e * stride
            shape = a.shape[1:]
        return table, keep, shape

    def _moe(self, fn, x, ids, weights, w_gate, w_up, w_down, E, shared, extra, threads):
        x, is_f32 = self._activations(x)
        T, H = x.shape
        ids = np.ascontiguousarray(ids, dtype=np.int32)
        top_k = ids.shape[1]
        weights = np.ascontiguousarray(weights, dtype=np.float64)
        assert weights.shape == ids.shape
        tg, kg, sg = self._expert_table(w_gate, E)
        tu, ku, _ = self._expert_table(w_up, E)
        td, kd, _ = self._expert_table(w_down, E)
        I = sg[0] if sg is not None else 1
        if shared is not None:
            sgate, sup, sdown = (np.ascontiguousarray(a, dtype=np.uint16) for a in shared)
            I_s = sgate.shape[0]
        else:
            sgate = sup = sdown = None
            I_s = 0
        y = np.zeros((T, H), dtype=np.float64)
        args = [_ptr(x), is_f32, T, H, _ptr(ids), _ptr(weights), top_k, tg, tu, td, E, I,
                _ptr(sgate), _ptr(sup), _ptr(sdown), I_s]
        rc = fn(*args, *extra, _ptr(y), self._threads(threads))
        del kg, ku, kd
        if rc != OK:
            raise OracleError(rc, "moe_ffn")
        return y

    def moe_ffn_monolith(self, x, ids, weights, w_gate, w_up, w_down, num_experts,
                         shared=None, threads=None):
        """Routed monolith (moeFFN) plus the shared expert; y is float64 [T, H]."""
        return self._moe(self.lib.oracle_moe_ffn_monolith, x, ids, weights, w_gate, w_up,
                         w_down, num_experts, shared, (), threads)

    def moe_ffn_expert_parallel(self, x, ids, weights, w_gate, w_up, w_down, num_experts,
                                band_start, shared=None, threads=None):
        """Per-band partials summed in rank order, plus the shared expert."""
        band_start = np.ascontiguousarray(band_start, dtype=np.int64)
        bands = band_start.shape[0] - 1
        return self._moe(self.lib.oracle_moe_ffn_expert_parallel, x, ids, weights, w_gate,
                         w_up, w_down, num_experts, shared, (_ptr(band_start), bands), threads)

    def max_threads(self):
        return self.lib.oracle_max_threads()

    def _threads(self, threads):
        return int(threads) if threads else int(os.environ.get("ORACLE_THREADS", "1"))


_default = None


def load():
    global _default
    if _default is None:
        _default = Oracle()
    return _default
