"""moe_route on the GPU against the fp64 oracle: ids exact (barring ties within
1e-6 of the oracle's own logits), weights within 1e-6, run-to-run identical."""
import numpy as np
import pytest
import torch

import workloads
import expert_decode_b200 as ed
from gpu_parity import check_route, device_inputs, oracle_route

pytestmark = pytest.mark.gpu
WL = workloads.WORKLOADS


# Above 32 tokens two routers form the fp32 logits: on the CUDA cores
# (register tiles) or on the tensor cores (tcgen05; bf16 x, E <= 256).  Both
# refine every expert that could reach the top_k by Dot2, so every test of
# that range runs on both and must give the oracle's ids and weights.
@pytest.fixture(params=["tiled", "tensor"])
def router(request):
    ed.ep_set_router(request.param)
    yield request.param
    ed.ep_set_router("auto")


def _tensor_takes(router, E, x_dtype="bf16", H=4096):
    if router == "tensor" and (E > 256 or x_dtype != "bf16" or H < 128):
        pytest.skip("the tensor-core router takes bf16 x, E <= 256, H >= 128")


def _route_and_check(o, wl, T, rows=None, seed=workloads.SEED_BASE, **sizes):
    W, x = device_inputs(wl, T, seed=seed, **sizes)
    ids, w = ed.moe_route(x, W["w_router"], W["bias"], wl.top_k)
    ids2, w2 = ed.moe_route(x, W["w_router"], W["bias"], wl.top_k)
    torch.cuda.synchronize()
    assert torch.equal(ids, ids2) and torch.equal(w, w2), "router not run-to-run identical"
    ed.ep_check_status()
    ids_ref, w_ref, logits = oracle_route(o, x, W, wl.top_k, rows=rows)
    if rows is not None:
        ids, w = ids[rows], w[rows]
    return check_route(ids, w, ids_ref, w_ref, logits)


@pytest.mark.parametrize("T", [1, 4, 8])
def test_router_decode(oracle_lib, T):
    _route_and_check(oracle_lib, WL["decode"], T)


def test_router_tiny_fp32_x(oracle_lib):
    _route_and_check(oracle_lib, WL["tiny"], 4)


def test_router_prefill_full(oracle_lib, router):
    _route_and_check(oracle_lib, WL["prefill"], 512)


def test_router_imbalanced_full(oracle_lib, router):
    excused = _route_and_check(oracle_lib, WL["imbalanced"], 2048)
    assert excused == 0


def test_router_large_sampled(oracle_lib, router):
    T = 4096
    rows = np.r_[0:16, 16:T - 16:61, T - 16:T]
    _route_and_check(oracle_lib, WL["large"], T, rows=rows)


def test_routers_agree_bit_for_bit(router):
    """Both routers end in the same Dot2 refinement, so the same ids and the
    same weights, bit for bit, on the large workload's 4096 tokens."""
    wl = WL["large"]
    W, x = device_inputs(wl, 4096, seed=123)
    ed.ep_set_router("tiled")
    ids_t, w_t = ed.moe_route(x, W["w_router"], W["bias"], wl.top_k)
    ed.ep_set_router(router)
    ids, w = ed.moe_route(x, W["w_router"], W["bias"], wl.top_k)
    torch.cuda.synchronize()
    ed.ep_check_status()
    assert torch.equal(ids, ids_t) and torch.equal(w, w_t)


@pytest.mark.parametrize("T", [3, 13, 17])
def test_router_ragged_token_blocks(oracle_lib, T):
    _route_and_check(oracle_lib, WL["decode"], T, seed=77)


# Up to 32 tokens every logit is a compensated (Dot2) fp32 dot product: one
# token per cluster of 8 CTAs while the clusters fit on the SMs at once
# (T <= 18 on 148 SMs), else two.  fp32 activations add the exact product
# errors (TwoProd) to the compensation term.
@pytest.mark.parametrize("T,x_dtype", [(1, "f32"), (8, "f32"), (19, "bf16"), (32, "bf16"),
                                       (27, "f32")])
def test_router_dot2_small_batches(oracle_lib, T, x_dtype):
    wl = workloads.Workload("dot2", (T,), 4096, 128, 8, 16, 0, x_dtype, "zipf1.1", (1,))
    excused = _route_and_check(oracle_lib, wl, T, seed=40 + T)
    assert excused == 0


def test_router_odd_sizes(oracle_lib):
    wl = workloads.Workload("odd", (5,), 200, 37, 5, 16, 0, "bf16", "zipf1.1", (1,))
    _route_and_check(oracle_lib, wl, 11, seed=5)


def test_router_max_experts_and_top_k(oracle_lib):
    wl = workloads.Workload("wide", (3,), 512, 1024, 16, 16, 0, "bf16", "none", (1,))
    _route_and_check(oracle_lib, wl, 3, seed=9)


def test_router_all_equal_logits():
    """Zero router weights: every logit ties; ids 0..k-1, weights 1/k (the
    candidate set exceeds the parallel budget, so the streaming fallback runs)."""
    E, H, k, T = 128, 256, 8, 3
    x = torch.randn(T, H, device="cuda").to(torch.bfloat16)
    w = torch.zeros(E, H, device="cuda", dtype=torch.bfloat16)
    ids, wts = ed.moe_route(x, w, None, k)
    torch.cuda.synchronize()
    assert ids.cpu().tolist() == [list(range(k))] * T
    assert torch.all(wts.cpu() == 1.0 / k)


def test_router_empty_is_a_no_op():
    x = torch.empty((0, 256), device="cuda", dtype=torch.bfloat16)
    w = torch.randn(16, 256, device="cuda").to(torch.bfloat16)
    ids = torch.full((0, 4), -7, dtype=torch.int32, device="cuda")
    ed.moe_route(x, w, None, 4, ids=ids)
    assert ed.ep_last_launch_count() == 0


# ---------------------------------------------------- tiled path (T > 32 tokens)
@pytest.mark.parametrize("E,T,k", [(37, 45, 5), (300, 70, 8), (1024, 41, 16), (64, 33, 4)])
def test_router_tiled_odd_shapes(oracle_lib, router, E, T, k):
    """Tiled: clusters of 1, 3 and 8 CTAs, ragged token blocks of 32 / 16 / 8.
    Tensor cores: one or two M tiles of experts, ragged 64-token tiles, H not
    a multiple of 64 (the last block of every slice zero-filled)."""
    _tensor_takes(router, E)
    wl = workloads.Workload("tiled", (T,), 328, E, k, 16, 0, "bf16", "zipf1.1", (1,))
    _route_and_check(oracle_lib, wl, T, seed=E + T)


@pytest.mark.parametrize("E,T,H,k", [(256, 200, 6144, 8), (192, 97, 1032, 6), (16, 300, 128, 2)])
def test_router_tensor_core_shapes(oracle_lib, E, T, H, k):
    """The tensor-core router at two M tiles (E = 192, 256), the smallest H it
    takes (two 64-wide blocks), clusters of 2..8 CTAs and ragged token tiles."""
    ed.ep_set_router("tensor")
    try:
        wl = workloads.Workload("tc", (T,), H, E, k, 16, 0, "bf16", "zipf1.1", (1,))
        excused = _route_and_check(oracle_lib, wl, T, seed=E + T + H)
        assert excused == 0
    finally:
        ed.ep_set_router("auto")


def test_router_tiled_fp32_activations(oracle_lib):
    wl = workloads.Workload("tiled32", (40,), 256, 16, 4, 16, 0, "f32", "none", (1,))
    _route_and_check(oracle_lib, wl, 40, seed=2)


def test_router_tiled_all_equal_logits(router):
    """Every logit ties: more candidates than the parallel budget (fallback list)."""
    E, H, k, T = 128, 256, 8, 40
    x = torch.randn(T, H, device="cuda").to(torch.bfloat16)
    w = torch.zeros(E, H, device="cuda", dtype=torch.bfloat16)
    ids, wts = ed.moe_route(x, w, None, k)
    torch.cuda.synchronize()
    assert ids.cpu().tolist() == [list(range(k))] * T
    assert torch.all(wts.cpu() == 1.0 / k)
