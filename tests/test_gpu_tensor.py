"""The tensor-core path (tcgen05 grouped GEMMs) of moe_ffn_forward against the fp64
oracle: small cases that span several tiles with ragged tails, element by
element; the full-size workloads on rows the oracle computes one by one; and
the bit-identity across runs and band counts at every size."""
import numpy as np
import pytest
import torch

import workloads
import expert_decode_b200 as ed
from gpu_parity import (check_route, check_y, device_inputs, gpu_ffn, oracle_ffn,
                        oracle_ffn_rows, oracle_route, spread_rows)

pytestmark = pytest.mark.gpu
WL = workloads.WORKLOADS


@pytest.fixture(autouse=True)
def tensor_dispatch():
    ed.ep_set_dispatch("tensor")
    yield "tensor"
    ed.ep_set_dispatch("auto")


def _routed(o, wl, T, seed=workloads.SEED_BASE, batch=0, **sizes):
    """GPU-routed inputs whose ids equal the oracle's; returns the GPU's ids and
    weights (the forward's inputs) and the oracle's weights (the reference's)."""
    W, x = device_inputs(wl, T, seed=seed, batch=batch, **sizes)
    ids, w = ed.moe_route(x, W["w_router"], W["bias"], wl.top_k)
    torch.cuda.synchronize()
    ids_ref, w_ref, logits = oracle_route(o, x, W, wl.top_k)
    assert check_route(ids, w, ids_ref, w_ref, logits) == 0
    return W, x, ids, w, w_ref


def test_tiny_tensor_path_all_bands(oracle_lib):
    wl = WL["tiny"]
    W, x, ids, w, w_ref = _routed(oracle_lib, wl, 24)
    ys = [gpu_ffn(x, ids, w, W, ed.ep_plan(wl.E, R)) for R in (1, 2, 4, 8)]
    ed.ep_check_status()
    assert ed.ep_last_launch_count() == 6
    for y in ys[1:]:
        assert torch.equal(y, ys[0])
    check_y(ys[0], oracle_ffn(oracle_lib, x, ids, w_ref, W), what="tiny T=24 tensor")
    check_y(ys[0], oracle_ffn(oracle_lib, x, ids, w_ref, W,
                             bands=oracle_lib.expert_parallel_plan(16, 4)),
            what="tiny T=24 tensor vs EP(4)")


@pytest.mark.parametrize("T", [1, 8, 33, 300])
def test_ragged_multi_tile(oracle_lib, T):
    """H, I, I_s not multiples of the tile; groups of every size incl. > 256 rows."""
    wl = workloads.Workload("ragged", (T,), 200, 12, 6, 136, 72, "bf16", "none", (3,))
    W, x, ids, w, w_ref = _routed(oracle_lib, wl, T, seed=31)
    y = gpu_ffn(x, ids, w, W, ed.ep_plan(wl.E, 3))
    ed.ep_check_status()
    check_y(y, oracle_ffn(oracle_lib, x, ids, w_ref, W), what=f"ragged T={T}")


def test_fp32_activations(oracle_lib):
    wl = workloads.Workload("f32", (40,), 256, 16, 4, 128, 128, "f32", "none", (2,))
    W, x, ids, w, w_ref = _routed(oracle_lib, wl, 40, seed=3)
    y = gpu_ffn(x, ids, w, W, ed.ep_plan(wl.E, 2))
    check_y(y, oracle_ffn(oracle_lib, x, ids, w_ref, W), what="fp32 x tensor")


def test_hot_expert_many_tiles(oracle_lib):
    """One expert takes every token's first pick: > 256 rows, several N tiles."""
    wl = workloads.Workload("hot", (600,), 256, 8, 2, 192, 0, "bf16", "none", (2,))
    W, x = device_inputs(wl, 600, seed=6)
    ids = torch.stack([torch.zeros(600, dtype=torch.int32),
                       torch.arange(600, dtype=torch.int32) % 7 + 1], 1).cuda()
    w = torch.full((600, 2), 0.5, device="cuda")
    y = gpu_ffn(x, ids, w, W, ed.ep_plan(wl.E, 2))
    rows = np.r_[0:8, 250:262, 590:600]
    ref = oracle_ffn(oracle_lib, x, ids, w, W, rows=rows)
    check_y(y[rows], ref, what="hot expert")


def test_tensor_matches_streaming_within_tolerance(oracle_lib, tensor_dispatch):
    wl = WL["decode"]
    W, x, ids, w, w_ref = _routed(oracle_lib, wl, 8, batch=2)
    plan = ed.ep_plan(wl.E, 8)
    y_t = gpu_ffn(x, ids, w, W, plan)
    mode = tensor_dispatch
    ed.ep_set_dispatch("streaming")
    y_s = gpu_ffn(x, ids, w, W, plan)
    ed.ep_set_dispatch(mode)
    ref = oracle_ffn(oracle_lib, x, ids, w_ref, W)
    check_y(y_t, ref, what="decode T=8 tensor")
    check_y(y_s, ref, rel_tol=1e-4, what="decode T=8 streaming")


def test_repeated_and_bad_ids(oracle_lib):
    wl = WL["tiny"]
    W, x, ids, w, w_ref = _routed(oracle_lib, wl, 20, seed=14)
    ed.ep_check_status()
    ids = ids.clone()
    ids[2, 1] = ids[2, 0]
    ids[5, 3] = -3
    y = gpu_ffn(x, ids, w, W, ed.ep_plan(wl.E, 4))
    with pytest.raises(ed.EPError):
        ed.ep_check_status()
    ref_ids, ref_w = ids.clone(), w_ref.copy()
    ref_ids[5, 3] = 0
    ref_w[5, 3] = 0.0
    check_y(y, oracle_ffn(oracle_lib, x, ref_ids, ref_w, W), what="repeated / bad ids")


# ------------------------------------------------------------ full-size workloads
# At full size the oracle computes sampled rows only: at least 64, spread over
# every N tile of the hottest experts, one expert of every activation-box
# class and the least-picked expert (spread_rows).  The oracle routes those
# rows itself; the GPU's ids must equal its ids there, and the FFN reference
# takes the oracle's own ids and weights.
def _full(o, name, bands):
    wl = WL[name]
    T = wl.T[0]
    W, x = device_inputs(wl, T)
    ids, w = ed.moe_route(x, W["w_router"], W["bias"], wl.top_k)
    ys = [gpu_ffn(x, ids, w, W, ed.ep_plan(wl.E, R)) for R in bands]
    ed.ep_check_status()
    for y in ys[1:]:
        assert torch.equal(y, ys[0]), "band counts differ"
    assert torch.equal(gpu_ffn(x, ids, w, W, ed.ep_plan(wl.E, bands[0])), ys[0]), "runs differ"
    rows = spread_rows(ids.cpu().numpy(), wl.E)
    assert len(rows) >= 64
    ids_ref, w_ref, logits = oracle_route(o, x, W, wl.top_k, rows=rows)
    assert check_route(ids[rows], w[rows], ids_ref, w_ref, logits) == 0
    ref = oracle_ffn_rows(o, x[rows], ids_ref, w_ref, W, np.arange(len(rows)))
    check_y(ys[0][rows], ref, what=f"{name}: {len(rows)} sampled rows")
    return W, x, ids, w, ys[0]


def test_prefill_full_size(oracle_lib):
    _full(oracle_lib, "prefill", (4, 1, 2, 8))


def test_imbalanced_full_size(oracle_lib):
    W, x, ids, w, y = _full(oracle_lib, "imbalanced", (4, 1))
    assert int(ids.max()) < 16, "bias +8 on experts 0..15 must put every pick in band 0"


def test_large_full_size(oracle_lib):
    _full(oracle_lib, "large", (8, 1))
