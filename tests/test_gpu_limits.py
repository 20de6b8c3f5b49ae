"""The documented size limits, at their maxima, against the fp64 oracle on
sampled rows: H = I = I_s = 16384 (the largest hidden and intermediate
sizes), T = 65536 tokens (the largest batch) and T * top_k = 2^20 picks (the
largest pick count), plus the refusal just past each limit."""
import numpy as np
import pytest
import torch

import workloads
import expert_decode_b200 as ed
from gpu_parity import check_route, check_y, device_inputs, gpu_ffn, oracle_ffn, oracle_route

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T", [1, 4, 9])
def test_ffn_at_the_largest_hidden_and_intermediate_sizes(oracle_lib, T):
    """H = I = I_s = 16384 with two experts: T = 1 and 4 take the streaming
    kernels where their buffers fit, T = 9 the tensor-core path."""
    wl = workloads.Workload("widest", (T,), 16384, 2, 2, 16384, 16384, "bf16", "none", (1,))
    W, x = device_inputs(wl, T, seed=91)
    ids, w = ed.moe_route(x, W["w_router"], W["bias"], wl.top_k)
    y = gpu_ffn(x, ids, w, W, ed.ep_plan(wl.E, 2))
    ed.ep_check_status()
    rows = [0] if T == 1 else [0, T - 1]
    ref = oracle_ffn(oracle_lib, x, ids, w, W, rows=rows)
    check_y(y[rows], ref, what=f"H = I = I_s = 16384, T = {T}")


def test_route_at_the_largest_batch(oracle_lib):
    wl = workloads.Workload("most_tokens", (65536,), 64, 16, 16, 64, 0, "bf16", "zipf1.1", (1,))
    T = 65536
    W, x = device_inputs(wl, T, seed=92)
    ids, w = ed.moe_route(x, W["w_router"], W["bias"], wl.top_k)
    torch.cuda.synchronize()
    ed.ep_check_status()
    rows = np.r_[0:8, 8:T - 8:4093, T - 8:T]
    ids_ref, w_ref, logits = oracle_route(oracle_lib, x, W, wl.top_k, rows=rows)
    check_route(ids[rows], w[rows], ids_ref, w_ref, logits)


def test_ffn_at_the_largest_pick_count(oracle_lib):
    """T = 65536 tokens x top_k = 16 = 2^20 picks, small experts."""
    wl = workloads.Workload("most_picks", (65536,), 64, 16, 16, 64, 64, "bf16", "none", (4,))
    T = 65536
    W, x = device_inputs(wl, T, seed=93)
    ids, w = ed.moe_route(x, W["w_router"], W["bias"], wl.top_k)
    y = gpu_ffn(x, ids, w, W, ed.ep_plan(wl.E, 4))
    ed.ep_check_status()
    rows = np.r_[0:8, 8:T - 8:4093, T - 8:T]
    ref = oracle_ffn(oracle_lib, x, ids, w, W, rows=rows)
    check_y(y[rows], ref, what="2^20 picks")


def test_one_past_each_limit_is_refused():
    wl = workloads.Workload("limits", (1,), 64, 16, 16, 64, 64, "bf16", "none", (1,))
    W, _ = device_inputs(wl, 1, seed=94)
    plan = ed.ep_plan(wl.E, 1)
    # T * top_k = 2^20 + 16
    x = torch.zeros((65537, 64), device="cuda", dtype=torch.bfloat16)
    ids = torch.zeros((65537, 16), device="cuda", dtype=torch.int32)
    w = torch.zeros((65537, 16), device="cuda", dtype=torch.float32)
    with pytest.raises(ed.EPError) as ei:
        gpu_ffn(x, ids, w, W, plan)
    assert ei.value.code == ed.EP_EINVAL
    with pytest.raises(ed.EPError) as ei:
        ed.moe_route(x, W["w_router"], None, 16)
    assert ei.value.code == ed.EP_EINVAL
