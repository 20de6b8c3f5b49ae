"""The error bounds the routers' candidate selection relies on, checked on the
GPU against the fp64 oracle's logits element by element.

Above 32 tokens the router forms fp32 logits (on the CUDA cores, or on the
tensor cores, whose accumulation order and rounding are not documented) and
refines by Dot2 only the experts that could reach the top_k under a bound of
each logit's error.  If a bound were too small, an expert could be left out
of the refinement and the pick could differ from the exact one on some other
input.  moe_route_logits returns those fp32 logits and bounds; here every
|logit - oracle logit| must be within its bound, and the worst ratio is
printed (how much room the bound leaves)."""
import numpy as np
import pytest
import torch

import workloads
import expert_decode_b200 as ed
from gpu_parity import device_inputs, oracle_route

pytestmark = pytest.mark.gpu
WL = workloads.WORKLOADS


@pytest.fixture(params=["tiled", "tensor"])
def router(request):
    ed.ep_set_router(request.param)
    yield request.param
    ed.ep_set_router("auto")


def _check_bound(o, wl, T, router, seed=workloads.SEED_BASE, rows=None):
    W, x = device_inputs(wl, T, seed=seed)
    logits, bounds = ed.moe_route_logits(x, W["w_router"], W["bias"])
    torch.cuda.synchronize()
    ed.ep_check_status()
    _, _, ref = oracle_route(o, x, W, wl.top_k, rows=rows)
    got = logits.cpu().double().numpy()
    bnd = bounds.cpu().double().numpy()
    if rows is not None:
        got, bnd = got[rows], bnd[rows]
    assert np.all(np.isfinite(got)) and np.all(bnd > 0)
    err = np.abs(got - ref)
    ratio = err / bnd
    worst = np.unravel_index(np.argmax(ratio), ratio.shape)
    print(f"{router} {wl.name} T={T}: max |l - exact| = {err.max():.3e}, max bound "
          f"{bnd.max():.3e}, worst error / bound = {ratio.max():.3e} at {worst}")
    assert ratio.max() <= 1.0, (worst, err[worst], bnd[worst])
    return ratio.max()


@pytest.mark.parametrize("name", ["prefill", "imbalanced"])
def test_bounds_hold_on_the_workloads(oracle_lib, router, name):
    wl = WL[name]
    _check_bound(oracle_lib, wl, wl.T[0], router)


def test_bounds_hold_on_the_large_workload(oracle_lib, router):
    rows = np.r_[0:64, 64:4096 - 64:37, 4096 - 64:4096]
    _check_bound(oracle_lib, WL["large"], 4096, router, rows=rows)


@pytest.mark.parametrize("E,T,H", [(37, 45, 328), (256, 70, 6144), (64, 33, 128), (192, 300, 1032)])
def test_bounds_hold_on_odd_shapes(oracle_lib, router, E, T, H):
    if router == "tensor" and H < 128:
        pytest.skip("the tensor-core router takes H >= 128")
    wl = workloads.Workload("bound", (T,), H, E, 4, 16, 0, "bf16", "zipf1.1", (1,))
    _check_bound(oracle_lib, wl, T, router, seed=E * 7 + T)


def test_bounds_hold_for_large_activations(oracle_lib, router):
    """x scaled by 64 and heavy-tailed weights: larger logits and sums."""
    wl = workloads.Workload("big", (128,), 2048, 128, 8, 16, 0, "bf16", "none", (1,))
    W, x = device_inputs(wl, 128, seed=321)
    x = (x.float() * 64).to(torch.bfloat16)
    W["w_router"] = (W["w_router"].float() ** 3 * 2500).to(torch.bfloat16)
    logits, bounds = ed.moe_route_logits(x, W["w_router"], None)
    torch.cuda.synchronize()
    _, _, ref = oracle_route(oracle_lib, x, W, wl.top_k)
    err = np.abs(logits.cpu().double().numpy() - ref)
    ratio = err / bounds.cpu().double().numpy()
    print(f"{router} large activations: worst error / bound = {ratio.max():.3e}")
    assert ratio.max() <= 1.0
