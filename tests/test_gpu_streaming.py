"""The weight-streaming path (T <= 8) of moe_ffn_forward against the fp64 oracle,
with the bit-identity the method promises: across runs and across band counts.
Every test runs with the projections on the CUDA cores, on the tensor cores
(bf16 activations only), and with the default choice of kernels."""
import numpy as np
import pytest
import torch

import workloads
import expert_decode_b200 as ed
from gpu_parity import check_y, device_inputs, gpu_ffn, oracle_ffn, oracle_route

pytestmark = pytest.mark.gpu
WL = workloads.WORKLOADS


# the tiny workload with bf16 activations, for the tensor-core gate/up
TINY_BF16 = workloads.Workload("tiny_bf16", (4,), 256, 16, 4, 128, 128, "bf16", "none", (1, 2, 4))


# streaming_simt: gate/up, then down with the fold, on the CUDA cores;
# streaming_tc: gate/up and down on the tensor cores (bf16 activations only),
# then the fold of the picks' contributions; streaming: the default choice
# (tensor cores from 2 tokens with bf16 activations).
@pytest.fixture(autouse=True, params=["streaming_simt", "streaming_tc", "streaming"])
def gate_up(request):
    ed.ep_set_dispatch(request.param)
    yield request.param
    ed.ep_set_dispatch("auto")


def _activations_supported(gate_up, x_dtype):
    if gate_up == "streaming_tc" and x_dtype != "bf16":
        pytest.skip("the tensor-core gate/up takes bf16 activations")


def _routed(o, wl, T, seed=workloads.SEED_BASE, batch=0, **sizes):
    W, x = device_inputs(wl, T, seed=seed, batch=batch, **sizes)
    ids_ref, w_ref, _ = oracle_route(o, x, W, wl.top_k)
    ids = torch.from_numpy(ids_ref).cuda()
    w = torch.from_numpy(w_ref.astype(np.float32)).cuda()
    return W, x, ids, w


@pytest.mark.parametrize("wl", [WL["tiny"], TINY_BF16], ids=["fp32_x", "bf16_x"])
def test_tiny_all_band_counts(oracle_lib, gate_up, wl):
    _activations_supported(gate_up, wl.x_dtype)
    W, x, ids, w = _routed(oracle_lib, wl, 4)
    ys = {}
    for R in wl.bands + (8, 16):
        ys[R] = gpu_ffn(x, ids, w, W, ed.ep_plan(wl.E, R))
        ed.ep_check_status()
        ref = oracle_ffn(oracle_lib, x, ids, w, W, bands=oracle_lib.expert_parallel_plan(wl.E, R))
        check_y(ys[R], ref, what=f"tiny bands={R}")
    mono = oracle_ffn(oracle_lib, x, ids, w, W)
    check_y(ys[1], mono, rel_tol=1e-4, what="tiny vs monolith")
    for R, y in ys.items():
        assert torch.equal(y, ys[1]), f"bands={R} differs from bands=1"


@pytest.mark.parametrize("T", [1, 4, 8])
def test_decode_full_size(oracle_lib, T):
    wl = WL["decode"]
    W, x, ids, w = _routed(oracle_lib, wl, T)
    plan = ed.ep_plan(wl.E, 8)
    y = gpu_ffn(x, ids, w, W, plan)
    ed.ep_check_status()
    check_y(y, oracle_ffn(oracle_lib, x, ids, w, W), rel_tol=1e-4, what=f"decode T={T}")
    check_y(y, oracle_ffn(oracle_lib, x, ids, w, W, bands=plan.starts()),
            what=f"decode T={T} vs EP(8)")
    for R in (1, 2, 4):
        assert torch.equal(gpu_ffn(x, ids, w, W, ed.ep_plan(wl.E, R)), y)
    assert torch.equal(gpu_ffn(x, ids, w, W, plan), y), "not run-to-run identical"


@pytest.mark.parametrize("T", [1, 8])
def test_decode_at_the_large_sizes(oracle_lib, gate_up, T):
    """H = 6144, E = 256, top_k = 8, I = I_s = 2048 with the Zipf bias: 96 k blocks
    per tensor-core tile, 8-chunk rows in the down kernel's register path."""
    wl = WL["large"]
    W, x, ids, w = _routed(oracle_lib, wl, T, seed=51)
    y = gpu_ffn(x, ids, w, W, ed.ep_plan(wl.E, 8))
    ed.ep_check_status()
    check_y(y, oracle_ffn(oracle_lib, x, ids, w, W), rel_tol=1e-4, what=f"large sizes T={T}")


def test_decode_end_to_end_with_gpu_router(oracle_lib):
    wl = WL["decode"]
    W, x = device_inputs(wl, 8, batch=3)
    ids, w = ed.moe_route(x, W["w_router"], W["bias"], wl.top_k)
    y = gpu_ffn(x, ids, w, W, ed.ep_plan(wl.E, 8))
    ids_ref, w_ref, _ = oracle_route(oracle_lib, x, W, wl.top_k)
    assert np.array_equal(ids.cpu().numpy(), ids_ref)
    check_y(y, oracle_ffn(oracle_lib, x, ids_ref, w_ref, W), rel_tol=1e-4, what="decode e2e")


def test_odd_sizes_and_max_pairs(oracle_lib):
    wl = workloads.Workload("odd", (8,), 200, 23, 16, 72, 40, "bf16", "none", (1,))
    W, x, ids, w = _routed(oracle_lib, wl, 8, seed=21)
    y = gpu_ffn(x, ids, w, W, ed.ep_plan(wl.E, 5))
    check_y(y, oracle_ffn(oracle_lib, x, ids, w, W), rel_tol=1e-4, what="odd sizes, 128 picks")


# Wide rows shrink the gate/up weight ring: at H = 8192 one slot (a W_gate and
# a W_up row) takes 32 KB, so 2 (T = 8, bf16 x) or 4 (T = 2, x widened to
# fp32) slots fit beside x, and fewer consumer warps than usual take tasks.
# H = 6144 with fp32 x at T = 4 leaves 4 slots of 24 KB.
@pytest.mark.parametrize("T,H,x_dtype", [(8, 8192, "bf16"), (2, 8192, "bf16"),
                                         (4, 6144, "f32")])
def test_wide_rows_few_gate_up_slots(oracle_lib, gate_up, T, H, x_dtype):
    _activations_supported(gate_up, x_dtype)
    wl = workloads.Workload("wide", (T,), H, 16, 4, 256, 128, x_dtype, "none", (1,))
    W, x, ids, w = _routed(oracle_lib, wl, T, seed=31 + T)
    y = gpu_ffn(x, ids, w, W, ed.ep_plan(wl.E, 4))
    ed.ep_check_status()
    check_y(y, oracle_ffn(oracle_lib, x, ids, w, W), rel_tol=1e-4,
            what=f"wide rows T={T} H={H} {x_dtype}")
    assert torch.equal(gpu_ffn(x, ids, w, W, ed.ep_plan(wl.E, 4)), y), "not run-to-run identical"


def test_no_shared_expert(oracle_lib):
    wl = WL["imbalanced"]
    W, x, ids, w = _routed(oracle_lib, wl, 5, H=512, I=64, seed=4)
    assert W["ws_gate"] is None
    y = gpu_ffn(x, ids, w, W, ed.ep_plan(wl.E, 4))
    y1 = gpu_ffn(x, ids, w, W, ed.ep_plan(wl.E, 1))
    assert torch.equal(y, y1)
    assert int(ids.max()) < 16
    check_y(y, oracle_ffn(oracle_lib, x, ids, w, W), rel_tol=1e-4, what="imbalanced, small")


@pytest.mark.parametrize("wl", [WL["tiny"], TINY_BF16], ids=["fp32_x", "bf16_x"])
def test_repeated_expert_in_one_token(oracle_lib, gate_up, wl):
    _activations_supported(gate_up, wl.x_dtype)
    W, x, ids, w = _routed(oracle_lib, wl, 4, seed=8)
    ids[1, 2] = ids[1, 0]          # token 1 picks one expert twice
    ids[3, :] = ids[3, 1]          # token 3 picks one expert four times
    y = gpu_ffn(x, ids, w, W, ed.ep_plan(wl.E, 2))
    check_y(y, oracle_ffn(oracle_lib, x, ids, w, W), rel_tol=1e-4, what="repeated picks")


# More than 8 picks of one expert (repeats within tokens): the tensor-core down
# projection takes a group in slices of up to 8 picks (T = 3: 15 picks of
# expert 3, two slices; T = 8: 40 picks, five slices).
@pytest.mark.parametrize("T", [3, 8])
def test_more_than_eight_picks_of_one_expert(oracle_lib, gate_up, T):
    wl = workloads.Workload("many_picks", (T,), 256, 16, 8, 128, 128, "bf16", "none", (1,))
    W, x, ids, w = _routed(oracle_lib, wl, T, seed=40 + T)
    ids[:, :5] = 3
    ids[0, 5:] = 7
    y = gpu_ffn(x, ids, w, W, ed.ep_plan(wl.E, 4))
    ed.ep_check_status()
    check_y(y, oracle_ffn(oracle_lib, x, ids, w, W), rel_tol=1e-4,
            what=f"{5 * T} picks of one expert")
    assert torch.equal(gpu_ffn(x, ids, w, W, ed.ep_plan(wl.E, 1)), y), "bands=1 differs"


@pytest.mark.parametrize("wl", [WL["tiny"], TINY_BF16], ids=["fp32_x", "bf16_x"])
def test_bad_ids_are_skipped_and_reported(oracle_lib, gate_up, wl):
    _activations_supported(gate_up, wl.x_dtype)
    W, x, ids, w = _routed(oracle_lib, wl, 4, seed=12)
    ed.ep_check_status()
    bad = ids.clone()
    bad[0, 1] = -1
    bad[2, 3] = wl.E
    y = gpu_ffn(x, bad, w, W, ed.ep_plan(wl.E, 1))
    with pytest.raises(ed.EPError) as ei:
        ed.ep_check_status()
    assert ei.value.code == ed.EP_EBADID
    ed.ep_check_status()  # cleared
    # the skipped picks contribute nothing: same as a valid pick with weight 0
    ref_ids, ref_w = ids.clone(), w.clone()
    ref_w[0, 1] = 0.0
    ref_w[2, 3] = 0.0
    check_y(y, oracle_ffn(oracle_lib, x, ref_ids, ref_w, W), rel_tol=1e-4, what="bad ids")


def test_all_ids_bad_without_shared_expert_gives_zero(oracle_lib, gate_up):
    """No valid pick and no shared expert: y = 0 (nothing folds a row)."""
    wl = workloads.Workload("noshared", (4,), 256, 16, 4, 128, 0, "bf16", "none", (1,))
    W, x = device_inputs(wl, 4, seed=3)
    ids = torch.full((4, wl.top_k), wl.E + 3, dtype=torch.int32, device="cuda")
    w = torch.full((4, wl.top_k), 0.25, dtype=torch.float32, device="cuda")
    y = torch.full((4, wl.H), float("nan"), dtype=torch.float32, device="cuda")
    ed.moe_ffn_forward(x, ids, w, W["w_gate"], W["w_up"], W["w_down"], None,
                       ed.ep_plan(wl.E, 1), y=y)
    torch.cuda.synchronize()
    with pytest.raises(ed.EPError) as ei:
        ed.ep_check_status()
    assert ei.value.code == ed.EP_EBADID
    assert torch.count_nonzero(y).item() == 0


def test_empty_batch_is_a_no_op():
    wl = WL["tiny"]
    W, _ = device_inputs(wl, 1)
    x = torch.empty((0, wl.H), device="cuda", dtype=torch.float32)
    ids = torch.empty((0, wl.top_k), device="cuda", dtype=torch.int32)
    w = torch.empty((0, wl.top_k), device="cuda", dtype=torch.float32)
    y = gpu_ffn(x, ids, w, W, ed.ep_plan(wl.E, 1))
    assert y.shape == (0, wl.H)
    assert ed.ep_last_launch_count() == 0
