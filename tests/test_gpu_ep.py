"""The expert-parallel form on one GPU: every band's partial (band-resident
weights) computed in turn, then the rank-order combine, against the fp64
oracle's band form; one band against moe_ffn_forward bit for bit; empty pick
slots (EP_ID_NONE) skipped without a report."""
import numpy as np
import pytest
import torch

import workloads
import expert_decode_b200 as ed
from expert_decode_b200 import ep
from gpu_parity import check_y, device_inputs, gpu_ffn, oracle_ffn, oracle_route

pytestmark = pytest.mark.gpu
WL = workloads.WORKLOADS


def _routed(o, wl, T, seed=workloads.SEED_BASE):
    W, x = device_inputs(wl, T, seed=seed)
    ids_ref, w_ref, _ = oracle_route(o, x, W, wl.top_k)
    return W, x, torch.from_numpy(ids_ref).cuda(), torch.from_numpy(w_ref.astype(np.float32)).cuda()


def _ep(W, x, ids, w, plan):
    """Every band's partial on this GPU in rank order, then the combine."""
    parts = []
    for r in range(plan.bands):
        lo, hi = plan.band_start[r], plan.band_start[r + 1]
        parts.append(ep.moe_ffn_partial(x, ids, w, W["w_gate"][lo:hi], W["w_up"][lo:hi],
                                        W["w_down"][lo:hi], plan, r))
    s = None if W["ws_gate"] is None else ep.shared_expert(x, W["ws_gate"], W["ws_up"], W["ws_down"])
    y = ep.moe_ep_combine(torch.stack(parts), ids, plan, s)
    torch.cuda.synchronize()
    return y


@pytest.mark.parametrize("wl_name,T", [("tiny", 4), ("decode", 1), ("decode", 8), ("decode", 24)])
@pytest.mark.parametrize("bands", [1, 2, 5, 8])
def test_band_partials_and_rank_order_combine(oracle_lib, wl_name, T, bands):
    wl = WL[wl_name]
    W, x, ids, w = _routed(oracle_lib, wl, T)
    plan = ed.ep_plan(wl.E, bands)
    y = _ep(W, x, ids, w, plan)
    ed.ep_check_status()
    ref = oracle_ffn(oracle_lib, x, ids, w, W, bands=plan.starts())
    tol = 1e-4 if T <= 8 else 1e-2  # T > 8 takes the tensor-core path (bf16 h)
    check_y(y, ref, rel_tol=tol, what=f"{wl_name} T={T} EP({bands})")
    if bands == 1:
        assert torch.equal(y, gpu_ffn(x, ids, w, W, plan)), "one band differs from the forward"


def test_empty_pick_slots_are_skipped_silently(oracle_lib):
    wl = WL["decode"]
    W, x, ids, w = _routed(oracle_lib, wl, 4, seed=17)
    ed.ep_check_status()
    none_ids = ids.clone()
    none_ids[:, -2:] = ep.EP_ID_NONE          # the last two slots of every token are empty
    y = gpu_ffn(x, none_ids, w, W, ed.ep_plan(wl.E, 4))
    ed.ep_check_status()                        # no bad-id report
    ref_w = w.clone()
    ref_w[:, -2:] = 0.0
    check_y(y, oracle_ffn(oracle_lib, x, ids, ref_w, W), rel_tol=1e-4, what="empty slots")
    bad = ids.clone()
    bad[0, 0] = -5
    gpu_ffn(x, bad, w, W, ed.ep_plan(wl.E, 4))
    with pytest.raises(ed.EPError) as ei:
        ed.ep_check_status()
    assert ei.value.code == ed.EP_EBADID


def test_partial_refuses_a_rank_outside_the_plan():
    wl = WL["tiny"]
    W, x = device_inputs(wl, 2)
    ids = torch.zeros((2, wl.top_k), dtype=torch.int32, device="cuda")
    w = torch.zeros((2, wl.top_k), dtype=torch.float32, device="cuda")
    plan = ed.ep_plan(wl.E, 2)
    with pytest.raises(ed.EPError) as ei:
        ep.moe_ffn_partial(x, ids, w, W["w_gate"][:8], W["w_up"][:8], W["w_down"][:8], plan, 2)
    assert ei.value.code == ed.EP_EINVAL
