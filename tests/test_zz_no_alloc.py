"""moe_ffn_forward_noalloc (the library's static scratch in place of a
workspace) against moe_ffn_forward with a caller's workspace, on the same
inputs.  Collected last so that it also runs after every other GPU test."""
import pytest
import torch

import workloads
import expert_decode_b200 as ed
from gpu_parity import check_y, device_inputs, gpu_ffn, shared_of

pytestmark = pytest.mark.gpu
WL = workloads.WORKLOADS
STATIC_SCRATCH_BYTES = 4 << 20


@pytest.fixture(autouse=True)
def auto_dispatch():
    ed.ep_set_dispatch("auto")
    yield
    ed.ep_set_dispatch("auto")


def _noalloc(x, ids, w, W, plan, y):
    ed.moe_ffn_forward_noalloc(x, ids, w, W["w_gate"], W["w_up"], W["w_down"], shared_of(W),
                               plan, y)
    torch.cuda.synchronize()
    ed.ep_check_status()
    return y


# T = 1, 8: the weight-streaming path; T = 16: the tensor-core path, whose
# workspace still fits the static scratch at these sizes.
@pytest.mark.parametrize("T", [1, 8, 16])
def test_noalloc_matches_workspace_entry_point(T):
    wl = WL["decode"]
    assert ed.moe_ffn_workspace_size(T, wl.H, wl.E, wl.top_k, wl.I, wl.I_s) <= \
        STATIC_SCRATCH_BYTES
    W, x = device_inputs(wl, T, batch=5)
    ids, w = ed.moe_route(x, W["w_router"], W["bias"], wl.top_k)
    plan = ed.ep_plan(wl.E, 8)
    y_ref = gpu_ffn(x, ids, w, W, plan)
    ed.ep_check_status()
    ref = y_ref.cpu().double().numpy()
    # two calls in a row into separate outputs; the second reuses the scratch
    # the first left behind
    y1 = torch.full((T, wl.H), float("nan"), dtype=torch.float32, device="cuda")
    y2 = torch.full((T, wl.H), float("nan"), dtype=torch.float32, device="cuda")
    _noalloc(x, ids, w, W, plan, y1)
    _noalloc(x, ids, w, W, plan, y2)
    # the same kernels in the same order as the workspace entry point, so the
    # same bits; a scratch area shared wrongly between steps or calls would
    # show here first
    assert torch.equal(y1, y_ref), f"noalloc T={T}: first call differs from moe_ffn_forward"
    assert torch.equal(y2, y_ref), f"noalloc T={T}: second call differs from moe_ffn_forward"
    check_y(y1, ref, what=f"noalloc T={T} first call")
    check_y(y2, ref, what=f"noalloc T={T} second call")


def test_noalloc_refuses_sizes_beyond_its_scratch():
    wl = WL["decode"]
    T = 64
    assert ed.moe_ffn_workspace_size(T, wl.H, wl.E, wl.top_k, wl.I, wl.I_s) > \
        STATIC_SCRATCH_BYTES
    W, x = device_inputs(wl, T)
    ids = torch.zeros((T, wl.top_k), dtype=torch.int32, device="cuda")
    w = torch.zeros((T, wl.top_k), dtype=torch.float32, device="cuda")
    y = torch.zeros((T, wl.H), dtype=torch.float32, device="cuda")
    with pytest.raises(ed.EPError) as err:
        ed.moe_ffn_forward_noalloc(x, ids, w, W["w_gate"], W["w_up"], W["w_down"],
                                   shared_of(W), ed.ep_plan(wl.E, 8), y)
    assert err.value.code == ed.EP_ENOMEM
    assert "static scratch" in str(err.value)
    torch.cuda.synchronize()
    assert torch.count_nonzero(y).item() == 0, "a refused call wrote its output"
