"""The C-ABI library on the CPU: it loads, exports what include/expert_decode.h
declares, builds plans with the share rule, and fails closed on bad arguments
before touching a GPU (no compute call runs here)."""
import ctypes
import os
import re

import pytest

import expert_decode_b200 as ed
from expert_decode_b200 import api

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "expert_decode.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*"
                                 r"([a-z][a-z0-9_]*)\s*\(", text, flags=re.M)))


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    assert {"ep_plan", "moe_route", "moe_ffn_workspace_size", "moe_ffn_forward",
            "ep_check_status", "ep_last_error"} <= set(names)
    lib = ctypes.CDLL(api.library_path)
    for name in names:
        assert hasattr(lib, name), name


def test_plan_matches_oracle_share_rule(oracle_lib):
    for E in (1, 4, 16, 64, 128, 256, 1000):
        for R in (1, 2, 3, 4, 7, 8, 64):
            if R > E:
                with pytest.raises(ed.EPError) as ei:
                    ed.ep_plan(E, R)
                assert ei.value.code == ed.EP_EINVAL
                continue
            p = ed.ep_plan(E, R)
            assert p.num_experts == E and p.bands == R
            assert p.starts() == oracle_lib.expert_parallel_plan(E, R).tolist()


def test_plan_refusals():
    for E, R in ((0, 1), (16, 0), (16, -1), (4, 5), (200, 65)):
        with pytest.raises(ed.EPError):
            ed.ep_plan(E, R)


def _fake(addr=0x10000):
    return ctypes.c_void_p(addr)


def _ffn(lib, plan, **kw):
    a = dict(x=_fake(), xdt=0, T=4, H=256, ids=_fake(), w=_fake(), k=4, wg=_fake(), wu=_fake(),
             wd=_fake(), E=16, I=128, sg=_fake(), su=_fake(), sd=_fake(), I_s=128, y=_fake(),
             ws=_fake(), wsb=1 << 30)
    a.update(kw)
    return lib.moe_ffn_forward(a["x"], a["xdt"], a["T"], a["H"], a["ids"], a["w"], a["k"],
                               a["wg"], a["wu"], a["wd"], a["E"], a["I"], a["sg"], a["su"],
                               a["sd"], a["I_s"], ctypes.byref(plan), a["y"], a["ws"], a["wsb"],
                               None)


def test_ffn_fails_closed_before_any_launch():
    lib = api.library()
    plan16 = ed.ep_plan(16, 4)
    plan8 = ed.ep_plan(8, 2)
    assert _ffn(lib, plan8) == ed.EP_EDIM                      # plan.Dim != NumExperts
    bad = ed.ep_plan(16, 4)
    bad.band_start[2] = bad.band_start[1]                      # an empty band
    assert _ffn(lib, bad) == ed.EP_EINVAL
    assert _ffn(lib, plan16, H=250) == ed.EP_EINVAL            # H % 8 != 0
    assert _ffn(lib, plan16, I=100) == ed.EP_EINVAL
    assert _ffn(lib, plan16, k=17) == ed.EP_EINVAL
    assert _ffn(lib, plan16, k=0) == ed.EP_EINVAL
    assert _ffn(lib, plan16, sd=None) == ed.EP_EINVAL          # shared pointers inconsistent
    assert _ffn(lib, plan16, x=_fake(0x10008)) == ed.EP_EINVAL  # misaligned
    assert _ffn(lib, plan16, ws=_fake(0x10080)) == ed.EP_EINVAL
    assert _ffn(lib, plan16, wsb=16) == ed.EP_ENOMEM
    assert _ffn(lib, plan16, ids=None) == ed.EP_EINVAL
    assert _ffn(lib, plan16, T=0) == ed.EP_OK                 # empty input: a no-op
    assert b"plan" in lib.ep_last_error() or lib.ep_last_error() == b""


def test_route_fails_closed_before_any_launch():
    lib = api.library()
    f = _fake()
    def route(**kw):
        a = dict(x=f, xdt=0, T=4, H=256, w=f, b=None, E=16, k=4, ids=f, wts=f)
        a.update(kw)
        return lib.moe_route(a["x"], a["xdt"], a["T"], a["H"], a["w"], a["b"], a["E"], a["k"],
                             a["ids"], a["wts"], None)
    assert route(k=17) == ed.EP_EINVAL
    assert route(k=0) == ed.EP_EINVAL
    assert route(E=4, k=5) == ed.EP_EINVAL
    assert route(H=12) == ed.EP_EINVAL
    assert route(xdt=7) == ed.EP_EINVAL
    assert route(x=_fake(0x10004)) == ed.EP_EINVAL
    assert route(T=0) == ed.EP_OK


def test_workspace_size_grows_with_work():
    small = ed.moe_ffn_workspace_size(1, 4096, 128, 8, 1536, 1536)
    big = ed.moe_ffn_workspace_size(512, 4096, 128, 8, 2048, 2048)
    assert 0 < small < big
    assert ed.moe_ffn_workspace_size(0, 4096, 128, 8, 1536, 1536) == 0


def test_sigmoid_route_fails_closed_before_any_launch():
    lib = api.library()
    f = _fake()
    def route(**kw):
        a = dict(x=f, xdt=0, T=4, H=256, w=f, b=None, E=16, k=4, norm=0, scale=1.0, ids=f, wts=f)
        a.update(kw)
        return lib.moe_route_sigmoid(a["x"], a["xdt"], a["T"], a["H"], a["w"], a["b"], a["E"],
                                     a["k"], a["norm"], a["scale"], a["ids"], a["wts"], None)
    assert route(norm=2) == ed.EP_EINVAL
    assert route(scale=0.0) == ed.EP_EINVAL
    assert route(scale=-1.0) == ed.EP_EINVAL
    assert route(scale=float("nan")) == ed.EP_EINVAL
    assert route(scale=float("inf")) == ed.EP_EINVAL
    assert route(k=17) == ed.EP_EINVAL
    assert route(T=65537) == ed.EP_EINVAL
    assert route(x=None) == ed.EP_EINVAL
    assert route(T=0) == ed.EP_OK
    assert b"moe_route_sigmoid" in lib.ep_last_error() or lib.ep_last_error() == b""


def test_noalloc_refuses_sizes_beyond_its_static_scratch():
    lib = api.library()
    f = _fake()
    plan = ed.ep_plan(128, 8)
    # T = 64 at H = 4096, E = 128, top_k = 8, I = I_s = 1536 needs about 16 MB
    need = ed.moe_ffn_workspace_size(64, 4096, 128, 8, 1536, 1536)
    assert need > (4 << 20)
    rc = lib.moe_ffn_forward_noalloc(f, 0, 64, 4096, f, f, 8, f, f, f, 128, 1536, f, f, f, 1536,
                                     ctypes.byref(plan), f, None)
    assert rc == ed.EP_ENOMEM
    assert b"static scratch" in lib.ep_last_error()
