"""moe_ffn_forward_nvfp4 (decode batches, every expert matrix in NVFP4) against
the fp64 oracle, and its bit-identity across runs and band counts.

The oracle takes the experts' dequantised weights (oracle/nvfp4.py: tensor
scale x E4M3 block scale x E2M1 element, exact in bf16 for the power-of-two
tensor scales used here) and computes the same FFN in fp64.  The GPU
dequantises on chip to fp16 (exact), rounds x to fp16 (exact for these
activations) and passes h between the projections as an fp16 hi/lo pair
(about 22 significant bits), all with fp32 accumulation.  Tolerance:
max |y_gpu - y_oracle| <= 1e-4 max |y_oracle|, about a hundred times the
expected fp32 error (sqrt(K) 2^-24 relative for K = 4096 products, plus
2^-22 relative for h)."""
import numpy as np
import pytest
import torch

import workloads
import expert_decode_b200 as ed
from gpu_parity import check_y, oracle_ffn, oracle_route
from oracle import nvfp4 as onv

pytestmark = pytest.mark.gpu
WL = workloads.WORKLOADS
REL_TOL = 1e-4


class _Dequantised:
    """W[k][e] for the oracle: expert e's dequantised weights as a host bf16
    tensor, computed on demand from the stored bytes."""

    def __init__(self, m):
        self.packed = m["packed"].cpu().numpy()
        self.scales = m["scales"].cpu().numpy()
        self.ts = m["tensor_scale"]
        self.shape = self.packed.shape[:1] + (self.packed.shape[1], 2 * self.packed.shape[2])

    def __getitem__(self, e):
        return workloads.from_bits(onv.nvfp4_to_bf16_bits(self.packed[e], self.scales[e],
                                                          self.ts))


def _shared_host(m):
    return workloads.from_bits(onv.nvfp4_to_bf16_bits(m["packed"].cpu().numpy(),
                                                      m["scales"].cpu().numpy(),
                                                      m["tensor_scale"]))


def _nvfp4_weights(H, E, I, I_s, seed, scales=None):
    """The NVFP4 experts on the device; `scales` overrides the tensor scales
    of (gate, up, down) for routed and shared alike."""
    g = workloads.make_nvfp4_experts(E, I, H, seed + 11, device="cuda")
    u = workloads.make_nvfp4_experts(E, I, H, seed + 12, device="cuda")
    d = workloads.make_nvfp4_experts(E, H, I, seed + 13, device="cuda")
    shared = None
    if I_s:
        shared = tuple({"packed": m["packed"][0], "scales": m["scales"][0],
                        "tensor_scale": m["tensor_scale"]}
                       for m in (workloads.make_nvfp4_experts(1, I_s, H, seed + 14, "cuda"),
                                 workloads.make_nvfp4_experts(1, I_s, H, seed + 15, "cuda"),
                                 workloads.make_nvfp4_experts(1, H, I_s, seed + 16, "cuda")))
    if scales is not None:
        for m, s in zip((g, u, d), scales):
            m["tensor_scale"] = s
        if shared is not None:
            for m, s in zip(shared, scales):
                m["tensor_scale"] = s
    return g, u, d, shared


def _oracle_weights(g, u, d, shared):
    W = {"w_gate": _Dequantised(g), "w_up": _Dequantised(u), "w_down": _Dequantised(d)}
    if shared is None:
        W["ws_gate"] = W["ws_up"] = W["ws_down"] = None
    else:
        W["ws_gate"], W["ws_up"], W["ws_down"] = (_shared_host(m) for m in shared)
    return W


def _case(o, T, H, E, top_k, I, I_s, seed, scales=None):
    wl = workloads.Workload("nvfp4", (T,), H, E, top_k, I, I_s, "bf16", "none", (1,))
    w_router, bias = workloads.make_router(wl, device="cuda", seed=seed)
    x = workloads.make_x(wl, T, device="cuda", seed=seed)
    ids_ref, w_ref, _ = oracle_route(o, x, {"w_router": w_router, "bias": bias}, top_k)
    ids = torch.from_numpy(ids_ref).cuda()
    w = torch.from_numpy(w_ref.astype(np.float32)).cuda()
    g, u, d, shared = _nvfp4_weights(H, E, I, I_s, seed, scales)
    return x, ids, w, (g, u, d, shared)


def _run(x, ids, w, mats, plan):
    g, u, d, shared = mats
    y = ed.moe_ffn_forward_nvfp4(x, ids, w, g, u, d, shared, plan)
    torch.cuda.synchronize()
    ed.ep_check_status()
    return y


def _reference(o, x, ids, w, mats):
    return oracle_ffn(o, x, ids, w, _oracle_weights(*mats))


def test_tiny_all_band_counts(oracle_lib):
    T, H, E, k, I, I_s = 4, 256, 16, 4, 128, 128
    x, ids, w, mats = _case(oracle_lib, T, H, E, k, I, I_s, seed=3)
    ref = _reference(oracle_lib, x, ids, w, mats)
    ys = {R: _run(x, ids, w, mats, ed.ep_plan(E, R)) for R in (1, 2, 4, 8, 16)}
    check_y(ys[1], ref, rel_tol=REL_TOL, what="nvfp4 tiny")
    for R, y in ys.items():
        assert torch.equal(y, ys[1]), f"bands={R} differs from bands=1"
    assert ed.ep_last_launch_count() == 4


@pytest.mark.parametrize("T", [1, 2, 4, 8])
def test_decode_workload(oracle_lib, T):
    wl = WL["decode"]
    x, ids, w, mats = _case(oracle_lib, T, wl.H, wl.E, wl.top_k, wl.I, wl.I_s, seed=40 + T)
    y = _run(x, ids, w, mats, ed.ep_plan(wl.E, 8))
    check_y(y, _reference(oracle_lib, x, ids, w, mats), rel_tol=REL_TOL,
            what=f"nvfp4 decode T={T}")
    y2 = _run(x, ids, w, mats, ed.ep_plan(wl.E, 1))
    assert torch.equal(y, y2), "run to run / band count"


@pytest.mark.parametrize("H,E,k,I,I_s,T", [(320, 37, 5, 192, 64, 7), (192, 9, 3, 64, 0, 3),
                                           (1088, 24, 8, 448, 192, 8)])
def test_ragged_shapes(oracle_lib, H, E, k, I, I_s, T):
    """H not a multiple of the 128-row down tile, I of several k blocks, with
    and without the shared expert."""
    x, ids, w, mats = _case(oracle_lib, T, H, E, k, I, I_s, seed=H + E)
    y = _run(x, ids, w, mats, ed.ep_plan(E, min(E, 4)))
    check_y(y, _reference(oracle_lib, x, ids, w, mats), rel_tol=REL_TOL,
            what=f"nvfp4 H={H} E={E} I={I} I_s={I_s} T={T}")


def test_distinct_tensor_scales(oracle_lib):
    """Different tensor scales for gate, up and down: each must scale its own
    projection (a mix-up changes y by far more than the tolerance)."""
    x, ids, w, mats = _case(oracle_lib, 8, 512, 32, 6, 256, 128, seed=77,
                            scales=(2.0 ** -5, 2.0 ** -9, 2.0 ** -6))
    y = _run(x, ids, w, mats, ed.ep_plan(32, 2))
    check_y(y, _reference(oracle_lib, x, ids, w, mats), rel_tol=REL_TOL,
            what="nvfp4 distinct tensor scales")


def test_one_expert_for_every_token(oracle_lib):
    """Every token picks the same experts: the groups hold T picks each."""
    T, H, E, k, I, I_s = 8, 512, 16, 4, 256, 0
    x, ids, w, mats = _case(oracle_lib, T, H, E, k, I, I_s, seed=5)
    ids = ids[:1].repeat(T, 1).contiguous()
    y = _run(x, ids, w, mats, ed.ep_plan(E, 1))
    check_y(y, _reference(oracle_lib, x, ids, w, mats), rel_tol=REL_TOL,
            what="nvfp4 shared picks")


def test_bad_ids_are_reported_and_skipped(oracle_lib):
    T, H, E, k, I, I_s = 6, 256, 16, 4, 128, 128
    x, ids, w, mats = _case(oracle_lib, T, H, E, k, I, I_s, seed=9)
    ids = ids.clone()
    ids[2, 1] = ids[2, 0]
    ids[4, 3] = -3
    g, u, d, shared = mats
    y = ed.moe_ffn_forward_nvfp4(x, ids, w, g, u, d, shared, ed.ep_plan(E, 2))
    torch.cuda.synchronize()
    with pytest.raises(ed.EPError):
        ed.ep_check_status()
    ref_ids, ref_w = ids.cpu().numpy().copy(), w.cpu().double().numpy().copy()
    ref_ids[4, 3] = 0
    ref_w[4, 3] = 0.0
    check_y(y, oracle_ffn(oracle_lib, x, ref_ids, ref_w, _oracle_weights(*mats)),
            rel_tol=REL_TOL, what="nvfp4 repeated / bad ids")


def test_limits():
    T, H, E, k, I, I_s = 4, 256, 16, 4, 128, 128
    g, u, d, shared = _nvfp4_weights(H, E, I, I_s, seed=1)
    ids = torch.zeros((T, k), dtype=torch.int32, device="cuda")
    ids[:, :] = torch.arange(k, dtype=torch.int32, device="cuda")
    w = torch.full((T, k), 0.25, dtype=torch.float32, device="cuda")
    x = torch.zeros((T, H), dtype=torch.bfloat16, device="cuda")
    plan = ed.ep_plan(E, 1)
    # T = 0: a no-op
    y0 = ed.moe_ffn_forward_nvfp4(x[:0], ids[:0], w[:0], g, u, d, shared, plan)
    assert y0.shape == (0, H) and ed.ep_last_launch_count() == 0
    # zero activations give zero output
    y = ed.moe_ffn_forward_nvfp4(x, ids, w, g, u, d, shared, plan)
    torch.cuda.synchronize()
    assert torch.count_nonzero(y) == 0
    # T = 9 is past the decode kernels
    x9 = torch.zeros((9, H), dtype=torch.bfloat16, device="cuda")
    ids9 = torch.zeros((9, k), dtype=torch.int32, device="cuda")
    w9 = torch.zeros((9, k), dtype=torch.float32, device="cuda")
    with pytest.raises(ed.EPError) as err:
        ed.moe_ffn_forward_nvfp4(x9, ids9, w9, g, u, d, shared, plan)
    assert err.value.code == ed.EP_EINVAL
    # a plan for another expert count
    with pytest.raises(ed.EPError) as err:
        ed.moe_ffn_forward_nvfp4(x, ids, w, g, u, d, shared, ed.ep_plan(E - 1, 1))
    assert err.value.code == ed.EP_EDIM
    # fp32 activations are refused by the binding
    with pytest.raises(TypeError):
        ed.moe_ffn_forward_nvfp4(x.float(), ids, w, g, u, d, shared, plan)
    # a workspace one byte short
    need = ed.moe_ffn_nvfp4_workspace_size(T, H, E, k, I, I_s)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    with pytest.raises(ed.EPError) as err:
        ed.moe_ffn_forward_nvfp4(x, ids, w, g, u, d, shared, plan, workspace=ws[:need - 1])
    assert err.value.code == ed.EP_ENOMEM
    ed.ep_check_status()


def test_longest_rows_and_empty_slots(oracle_lib):
    """H = 16384, the longest rows (256 block-scale words per row, 64 stages per
    tile), against I = 64 (one k block, a quarter stage), and EP_ID_NONE slots,
    which contribute nothing and are not reported."""
    T, H, E, k, I, I_s = 3, 16384, 4, 2, 64, 64
    x, ids, w, mats = _case(oracle_lib, T, H, E, k, I, I_s, seed=16)
    ids = ids.clone()
    ids[1, 1] = -(2 ** 31)  # EP_ID_NONE
    g, u, d, shared = mats
    y = ed.moe_ffn_forward_nvfp4(x, ids, w, g, u, d, shared, ed.ep_plan(E, 2))
    torch.cuda.synchronize()
    ed.ep_check_status()
    ref_ids, ref_w = ids.cpu().numpy().copy(), w.cpu().double().numpy().copy()
    ref_ids[1, 1] = 0
    ref_w[1, 1] = 0.0
    check_y(y, oracle_ffn(oracle_lib, x, ref_ids, ref_w, _oracle_weights(*mats)),
            rel_tol=REL_TOL, what="nvfp4 H=16384 I=64")
