"""moe_route_sigmoid (the GLM router variant: sigmoid scores, the bias moves
the selection only, weights from the unbiased scores) on the GPU against the fp64 oracle:
ids exact except where the oracle's own keys tie within 1e-6, weights within
1e-6 of the oracle's (relative to the scale), run-to-run identical."""
import ctypes

import numpy as np
import pytest
import torch

import workloads
import expert_decode_b200 as ed
from gpu_parity import check_route, device_inputs

pytestmark = pytest.mark.gpu
WL = workloads.WORKLOADS


# above 32 tokens: the CUDA-core (tiled) and the tensor-core logits
@pytest.fixture(params=["tiled", "tensor"])
def router(request):
    ed.ep_set_router(request.param)
    yield request.param
    ed.ep_set_router("auto")


def _route_and_check(o, wl, T, normalize=False, scale=1.0, rows=None, seed=workloads.SEED_BASE,
                     **sizes):
    W, x = device_inputs(wl, T, seed=seed, **sizes)
    ids, w = ed.moe_route_sigmoid(x, W["w_router"], W["bias"], wl.top_k, normalize, scale)
    ids2, w2 = ed.moe_route_sigmoid(x, W["w_router"], W["bias"], wl.top_k, normalize, scale)
    torch.cuda.synchronize()
    assert torch.equal(ids, ids2) and torch.equal(w, w2), "router not run-to-run identical"
    ed.ep_check_status()
    xh = workloads.bits(x if rows is None else x[rows])
    b = None if W["bias"] is None else W["bias"].cpu().numpy()
    ids_ref, w_ref, keys, _ = o.route_sigmoid(xh, workloads.bits(W["w_router"]), b, wl.top_k,
                                              normalize=normalize, scale=scale, threads=8)
    if rows is not None:
        ids, w = ids[rows], w[rows]
    return check_route(ids, w / scale, ids_ref, w_ref / scale, keys)


@pytest.mark.parametrize("T", [1, 4, 8])
@pytest.mark.parametrize("normalize,scale", [(False, 1.0), (True, 2.5)])
def test_sigmoid_decode(oracle_lib, T, normalize, scale):
    _route_and_check(oracle_lib, WL["decode"], T, normalize, scale)


@pytest.mark.parametrize("T,x_dtype", [(8, "f32"), (19, "bf16"), (32, "bf16")])
def test_sigmoid_small_batches_with_bias(oracle_lib, T, x_dtype):
    wl = workloads.Workload("sig", (T,), 4096, 128, 8, 16, 0, x_dtype, "zipf1.1", (1,))
    assert _route_and_check(oracle_lib, wl, T, seed=60 + T) == 0


@pytest.mark.parametrize("T", [40, 200])
def test_sigmoid_tiled_odd_sizes(oracle_lib, router, T):
    wl = workloads.Workload("sig_tiled", (T,), 200, 37, 5, 16, 0, "bf16", "zipf1.1", (1,))
    _route_and_check(oracle_lib, wl, T, normalize=True, seed=7)


def test_sigmoid_prefill_full(oracle_lib, router):
    _route_and_check(oracle_lib, WL["prefill"], 512)


def test_sigmoid_imbalanced_bias_selects_only(oracle_lib, router):
    """+8 on experts 0..15 puts every pick there, but the weights stay the raw
    sigmoid scores (no 8 in them)."""
    wl = WL["imbalanced"]
    W, x = device_inputs(wl, 2048)
    ids, w = ed.moe_route_sigmoid(x, W["w_router"], W["bias"], wl.top_k)
    torch.cuda.synchronize()
    assert int(ids.max()) < 16
    assert float(w.max()) < 1.0
    _route_and_check(oracle_lib, wl, 2048)


def test_sigmoid_large_sampled(oracle_lib, router):
    T = 4096
    rows = np.r_[0:16, 16:T - 16:61, T - 16:T]
    _route_and_check(oracle_lib, WL["large"], T, rows=rows)


@pytest.mark.parametrize("T", [3, 40])
def test_sigmoid_all_equal_scores(T):
    """Zero router weights: every score is 1/2 and every key ties; ids 0..k-1,
    raw weights 1/2 (or 1/k normalised)."""
    E, H, k = 128, 256, 8
    x = torch.randn(T, H, device="cuda").to(torch.bfloat16)
    wr = torch.zeros(E, H, device="cuda", dtype=torch.bfloat16)
    ids, w = ed.moe_route_sigmoid(x, wr, None, k)
    ids_n, w_n = ed.moe_route_sigmoid(x, wr, None, k, normalize=True)
    torch.cuda.synchronize()
    assert ids.cpu().tolist() == [list(range(k))] * T
    assert ids_n.cpu().tolist() == [list(range(k))] * T
    assert torch.all(w.cpu() == 0.5)
    assert torch.all(w_n.cpu() == 1.0 / k)


def test_sigmoid_refuses_bad_arguments():
    x = torch.zeros((2, 64), device="cuda", dtype=torch.bfloat16)
    wr = torch.zeros((8, 64), device="cuda", dtype=torch.bfloat16)
    lib = ed.library()
    ids = torch.zeros((2, 2), device="cuda", dtype=torch.int32)
    w = torch.zeros((2, 2), device="cuda", dtype=torch.float32)
    for normalize, scale in ((2, 1.0), (0, 0.0), (0, float("nan")), (1, -1.0)):
        rc = lib.moe_route_sigmoid(ctypes.c_void_p(x.data_ptr()), 0, 2, 64,
                                   ctypes.c_void_p(wr.data_ptr()), None, 8, 2, normalize, scale,
                                   ctypes.c_void_p(ids.data_ptr()), ctypes.c_void_p(w.data_ptr()),
                                   None)
        assert rc == ed.EP_EINVAL, (normalize, scale, rc)
