"""The order of the fold, pinned on the GPU bit for bit.

The method's defining property is the order in which the picks' outputs are
summed: band by band in rank order (fak note "GLM-5.2 multi-GPU", "What
landed" and its gate table; TensorFold #214 "Per MoE layer"; TensorFold
#310, maintainer's reply).  Tolerance checks against the oracle cannot see
that order, and neither can the bit identity across band counts (the
single-GPU fold passes its running sum from band to band, so it never depends
on the plan).  These tests use fp32 values where the order shows in the
result (tests/golden/fold_order_f32.json):

  * moe_ffn_forward on every path (CUDA-core streaming kernels, tensor-core
    streaming kernels, grouped tensor-core path) equals the host fp32 left
    fold in ascending (expert id, slot), then + the shared expert, exactly,
    for every plan;
  * the band form (moe_ffn_partial per band, then moe_ep_combine) equals the
    host fp32 fold of the bands' partials in rank order, exactly, for plans
    where that order changes the bits; moe_ep_combine alone, on given
    partials, likewise;
  * on real inputs, y equals the host fp32 fold of the per-pick contributions
    that the tensor-core paths leave in their workspace (contrib + shared).
"""
import numpy as np
import pytest
import torch

import workloads
import expert_decode_b200 as ed
from expert_decode_b200 import ep
from expert_decode_b200.api import Plan
import fold_fixture as ff
from gpu_parity import device_inputs, oracle_route, shared_of

pytestmark = pytest.mark.gpu

PATHS = ["streaming_simt", "streaming_tc", "tensor"]


@pytest.fixture(autouse=True)
def restore_dispatch():
    yield
    ed.ep_set_dispatch("auto")


def _plan(band_start):
    p = Plan()
    p.num_experts = band_start[-1]
    p.bands = len(band_start) - 1
    for r, s in enumerate(band_start):
        p.band_start[r] = s
    return p


def _fixture_on_device(fx, width):
    """The fixture's tensors zero-padded to H = I = I_s = width (>= 8)."""
    x, wg, wu, wd, (sg, su, sd) = ff.tensors(fx)
    E, h0 = wd.shape[0], wd.shape[1]

    def pad(a, shape):
        out = np.zeros(shape, dtype=np.float32)
        out[tuple(slice(0, s) for s in a.shape)] = a
        return torch.from_numpy(out).to(torch.bfloat16).cuda()

    T = x.shape[0]
    dev = {
        "x": pad(x, (T, width)),
        "w_gate": pad(wg, (E, width, width)),
        "w_up": pad(wu, (E, width, width)),
        "w_down": pad(wd, (E, width, width)),
        "shared": (pad(sg, (width, width)), pad(su, (width, width)), pad(sd, (width, width))),
        "ids": torch.tensor(fx["ids"], dtype=torch.int32, device="cuda"),
        "weights": torch.tensor(fx["weights"], dtype=torch.float32, device="cuda"),
    }
    assert h0 == 8
    return dev


def _expected(fx, width):
    c = ff.contributions(fx)
    T, k, h0 = c.shape
    cp = np.zeros((T, k, width), dtype=np.float32)
    cp[:, :, :h0] = c
    S = np.zeros(width, dtype=np.float32)
    S[:h0] = fx["S"]
    return cp, np.broadcast_to(S, (T, width))


@pytest.mark.parametrize("width", [8, 64])
@pytest.mark.parametrize("path", PATHS)
def test_forward_folds_in_ascending_expert_id_on_every_path(path, width):
    fx = ff.load()
    d = _fixture_on_device(fx, width)
    c, S = _expected(fx, width)
    want = ff.host_fold_f32(c, fx["ids"], 4, S)
    ed.ep_set_dispatch(path)
    for band_start in ([0, 4], [0, 2, 4], [0, 2, 3, 4], [0, 1, 2, 3, 4], [0, 1, 4]):
        y = ed.moe_ffn_forward(d["x"], d["ids"], d["weights"], d["w_gate"], d["w_up"],
                               d["w_down"], d["shared"], _plan(band_start))
        torch.cuda.synchronize()
        ed.ep_check_status()
        got = y.cpu().numpy()
        assert np.array_equal(got.view(np.uint32), want.view(np.uint32)), (
            path, width, band_start, got[:, :2], want[:, :2])
    assert got[:, 0].tolist() == fx["expected_column0"]


@pytest.mark.parametrize("path", PATHS)
def test_band_form_folds_the_partials_in_rank_order(path):
    fx = ff.load()
    width = 64
    d = _fixture_on_device(fx, width)
    c, S = _expected(fx, width)
    ed.ep_set_dispatch(path)
    s = ep.shared_expert(d["x"], *d["shared"])
    torch.cuda.synchronize()
    assert np.array_equal(s.cpu().numpy(), np.ascontiguousarray(S))
    for case in fx["band_form"]["cases"]:
        bs = case["band_start"]
        plan = _plan(bs)
        parts = [ep.moe_ffn_partial(d["x"], d["ids"], d["weights"], d["w_gate"][bs[r]:bs[r + 1]],
                                    d["w_up"][bs[r]:bs[r + 1]], d["w_down"][bs[r]:bs[r + 1]],
                                    plan, r) for r in range(plan.bands)]
        y = ep.moe_ep_combine(torch.stack(parts), d["ids"], plan, s)
        torch.cuda.synchronize()
        ed.ep_check_status()
        want = ff.host_band_form_f32(c, fx["ids"], bs, S)
        got = y.cpu().numpy()
        assert np.array_equal(got.view(np.uint32), want.view(np.uint32)), (path, bs)
        assert float(got[0, 0]) == case["y"], (path, bs, case["why"])


def test_combine_alone_folds_given_partials_in_rank_order():
    """moe_ep_combine on partials written by the host: the bands holding a
    pick of the token, left-folded in rank order, then + shared; a band
    without a pick is left out even when its partial is not zero."""
    T, H = 3, 8
    big = np.float32(2.0 ** 24)
    parts = np.zeros((4, T, H), dtype=np.float32)
    parts[:, :, 0] = np.array([big, 1.0, 1.0, -big], dtype=np.float32)[:, None]
    parts[:, :, 1] = np.array([1.0, big, -big, 1.0], dtype=np.float32)[:, None]
    parts[:, :, 2:] = 0.25
    ids = np.array([[3, 1, 0, 2],      # every band: ((2^24 + 1) + 1) - 2^24 = 0
                    [0, 0, 2, 3],      # band 1 absent: (2^24 + 1) - 2^24 = 0
                    [3, 1, 1, 2]],     # band 0 absent: (1 + 1) - 2^24 exactly
                   dtype=np.int32)
    shared = np.full((T, H), 0.5, dtype=np.float32)
    plan = ed.ep_plan(4, 4)
    y = ep.moe_ep_combine(torch.from_numpy(parts).cuda(), torch.from_numpy(ids).cuda(), plan,
                          torch.from_numpy(shared).cuda())
    torch.cuda.synchronize()
    got = y.cpu().numpy()
    want = np.zeros((T, H), dtype=np.float32)
    for t in range(T):
        acc = None
        for r in range(4):
            if r in set(ids[t].tolist()):
                acc = parts[r, t].copy() if acc is None else acc + parts[r, t]
        want[t] = acc + shared[t]
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
    assert got[:, 0].tolist() == [0.5, 0.5, float(np.float32(2.0 - big) + np.float32(0.5))]


def _workspace_fold(x, ids, w, W, plan, path):
    """Run the forward with a workspace of our own; return y and the host fp32
    fold of the contributions the call left in that workspace."""
    T, H = x.shape
    k = ids.shape[1]
    E, I = W["w_gate"].shape[0], W["w_gate"].shape[1]
    I_s = 0 if W["ws_gate"] is None else W["ws_gate"].shape[0]
    lay = ed.moe_ffn_workspace_layout(T, H, E, k, I, I_s)
    assert lay.bytes == ed.moe_ffn_workspace_size(T, H, E, k, I, I_s)
    ws = torch.empty(lay.bytes, dtype=torch.uint8, device="cuda")
    ed.ep_set_dispatch(path)
    y = ed.moe_ffn_forward(x, ids, w, W["w_gate"], W["w_up"], W["w_down"], shared_of(W), plan,
                           workspace=ws)
    torch.cuda.synchronize()
    ed.ep_check_status()
    wsh = ws.cpu().numpy()
    c = wsh[lay.contrib_offset:lay.contrib_offset + T * k * H * 4].view(np.float32)
    c = c.reshape(T, k, H)
    s = None
    if I_s:
        s = wsh[lay.shared_offset:lay.shared_offset + T * H * 4].view(np.float32).reshape(T, H)
    return y.cpu().numpy(), ff.host_fold_f32(c, ids.cpu().numpy(), E, s)


@pytest.mark.parametrize("name,T,path", [("decode", 4, "streaming_tc"),
                                         ("decode", 8, "streaming_tc"),
                                         ("decode", 8, "tensor"),
                                         ("prefill", 512, "tensor"),
                                         ("imbalanced", 2048, "tensor")])
def test_y_is_the_host_fold_of_the_dumped_contributions(oracle_lib, name, T, path):
    wl = workloads.WORKLOADS[name]
    W, x = device_inputs(wl, T, batch=4)
    ids, w = ed.moe_route(x, W["w_router"], W["bias"], wl.top_k)
    torch.cuda.synchronize()
    if T <= 8:
        ids_ref, _, _ = oracle_route(oracle_lib, x, W, wl.top_k)
        assert np.array_equal(ids.cpu().numpy(), ids_ref)
    y, want = _workspace_fold(x, ids, w, W, ed.ep_plan(wl.E, wl.bands[0]), path)
    assert np.array_equal(y.view(np.uint32), want.view(np.uint32)), (name, T, path)


@pytest.mark.parametrize("name,T,seed", [("prefill", 512, 1000), ("large", 4096, 1000),
                                         ("tiny", 300, 7), ("many_experts", 333, 5)])
def test_grouping_is_a_stable_sort_by_expert(name, T, seed):
    """The grouped path's plan (group_count_kernel, group_plan_kernel: chunk counts,
    stable scatter) against a host stable sort of the picks by expert id, bit
    for bit, with some empty, repeated and out-of-range ids mixed in."""
    # many_experts: 1000 experts, top_k 7, so that T k = 2331 picks fall in
    # three chunks of the plan (the last one ragged) over an expert count that
    # is no power of two
    wl = (workloads.Workload("many_experts", (T,), 128, 1000, 7, 64, 64, "bf16", "none", (1,))
          if name == "many_experts" else workloads.WORKLOADS[name])
    W, x = device_inputs(wl, T, seed=seed)
    ids, w = ed.moe_route(x, W["w_router"], W["bias"], wl.top_k)
    ids = ids.clone()
    ids[3, 0] = ep.EP_ID_NONE
    ids[5, 1] = ids[5, 0]
    ids[T - 1, wl.top_k - 1] = wl.E + 4
    E, k = wl.E, wl.top_k
    I, I_s = wl.I, wl.I_s
    lay = ed.moe_ffn_workspace_layout(T, wl.H, E, k, I, I_s)
    ws = torch.empty(lay.bytes, dtype=torch.uint8, device="cuda")
    ed.ep_set_dispatch("tensor")
    ed.moe_ffn_forward(x, ids, w, W["w_gate"], W["w_up"], W["w_down"], shared_of(W),
                       ed.ep_plan(E, 1), workspace=ws)
    torch.cuda.synchronize()
    with pytest.raises(ed.EPError):   # the out-of-range id is reported
        ed.ep_check_status()
    wsh = ws.cpu().numpy()
    go = wsh[lay.group_offset_offset:lay.group_offset_offset + (E + 2) * 4].view(np.int32)
    P = T * k
    perm = wsh[lay.perm_offset:lay.perm_offset + P * 4].view(np.int32)
    flat = ids.cpu().numpy().reshape(-1)
    valid = [p for p in range(P) if 0 <= flat[p] < E]
    want = sorted(valid, key=lambda p: (int(flat[p]), p))   # stable by expert id
    counts = np.bincount(flat[valid], minlength=E)
    want_go = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    assert np.array_equal(go[:E + 1], want_go)
    assert go[E + 1] == P
    assert np.array_equal(perm[:len(valid)], np.array(want, dtype=np.int32))
