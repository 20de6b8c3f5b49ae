"""Pins of the fp64 oracle: checks against values the pages and mathematics fix.

Each pin takes an Oracle instance and raises AssertionError when the oracle
disagrees.  The pins are kept as plain functions so that the same set runs
against the oracle itself (test_oracle_pins.py) and against copies of it with
a planted mistake (test_oracle_mutations.py), which every pin set must catch.

What pins what:
  plan            worked shares printed in TensorFold #310 (golden/plan_shares.json)
  router          exact rational brute force on tiny inputs; closed forms
                  (large logits, top_k = 1, ties, all-equal, Zipf skew);
                  top_k = E against torch.softmax in float64
  sigmoid router  closed forms (golden/router_sigmoid_closed_forms.json);
                  without a bias its picks are the softmax router's (the
                  sigmoid is increasing); its scores against torch.sigmoid of
                  the pinned fp64 logits
  expert          a hand-derived 2x2 SwiGLU (golden/swiglu_hand.json); E = 1,
                  top_k = 1 against a dense SwiGLU from torch.nn.functional
  fold / bands    exact IEEE folds where the order shows (golden/fold_order.json);
                  the gate-table invariants of the fak expert-parallel note
  shared expert   y(with) - y(without) equals the dense SwiGLU of the shared weights
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import torch
import torch.nn.functional as F

import workloads
from oracle import OracleError

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def exact_bf16_bits(values):
    """bf16 bit patterns of values that bf16 represents exactly."""
    t = torch.tensor(values, dtype=torch.float64)
    b = t.to(torch.bfloat16)
    assert torch.equal(b.to(torch.float64), t), "fixture value not exact in bf16"
    return workloads.bits(b)


def _bf16_to_f64(bits_arr):
    return workloads.from_bits(bits_arr).to(torch.float64)


# ----------------------------------------------------------------------------- plan
def pin_plan_shares(o):
    g = golden("plan_shares.json")
    for case in g["cases"]:
        start = o.expert_parallel_plan(case["extent"], case["ranks"], case["unit"])
        shares = np.diff(start).tolist()
        assert shares == case["shares"], (case["what"], shares)
        assert start[0] == 0 and start[-1] == case["extent"]


def pin_plan_refused(o):
    g = golden("plan_shares.json")
    for case in g["refused"]:
        try:
            o.expert_parallel_plan(case["extent"], case["ranks"], case["unit"])
        except OracleError:
            continue
        raise AssertionError("plan not refused: " + case["what"])


# --------------------------------------------------------------------------- router
def _tiny_router_case(seed, T=6, H=16, E=8, with_bias=True):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(T, H, generator=g).to(torch.bfloat16)
    w = (torch.randn(E, H, generator=g) * 0.3).to(torch.bfloat16)
    b = (torch.randn(E, generator=g) * 0.1) if with_bias else None
    return x, w, b


def pin_router_brute_force(o):
    """Exact rational logits, full sort by (-l, id), weights by torch.softmax."""
    for seed in range(6):
        x, w, b = _tiny_router_case(seed)
        # make experts 5 and 6 share a row, an exact tie at every token
        w[6] = w[5]
        if b is not None:
            b[6] = b[5]
        k = 3
        ids, wts, logits = o.route(workloads.bits(x), workloads.bits(w),
                                   None if b is None else b.numpy(), k)
        xf, wf = x.to(torch.float64).numpy(), w.to(torch.float64).numpy()
        bf = None if b is None else b.to(torch.float64).numpy()
        for t in range(x.shape[0]):
            exact = []
            for e in range(w.shape[0]):
                acc = sum(Fraction(float(xf[t, h])) * Fraction(float(wf[e, h]))
                          for h in range(x.shape[1]))
                if bf is not None:
                    acc += Fraction(float(bf[e]))
                exact.append(acc)
            order = sorted(range(w.shape[0]), key=lambda e: (-exact[e], e))
            assert ids[t].tolist() == order[:k], (seed, t, ids[t], order[:k])
            for e in range(w.shape[0]):
                assert abs(logits[t, e] - float(exact[e])) <= 1e-12 * (1 + abs(float(exact[e])))
            ref = torch.softmax(torch.tensor([float(exact[e]) for e in order[:k]],
                                             dtype=torch.float64), 0).numpy()
            assert np.allclose(wts[t], ref, rtol=0, atol=1e-14), (wts[t], ref)


def pin_router_closed_forms(o):
    g = golden("router_closed_forms.json")
    for case in g["cases"]:
        E = len(case["bias"])
        x = np.ones((1, 1), dtype=np.float32)
        w = exact_bf16_bits([[0.0]] * E)
        ids, wts, _ = o.route(x, w, np.array(case["bias"], dtype=np.float64), case["top_k"])
        assert ids[0].tolist() == case["ids"], (case["what"], ids[0])
        ref = np.array([float(v) for v in case["weights"]])
        assert np.all(np.isfinite(wts)), case["what"]
        assert np.allclose(wts[0], ref, rtol=0, atol=1e-15), (case["what"], wts[0], ref)


def pin_router_full_softmax(o):
    """top_k = E: the renormalised weights are the full softmax."""
    x, w, b = _tiny_router_case(11, T=4, H=32, E=12)
    ids, wts, logits = o.route(workloads.bits(x), workloads.bits(w), b.numpy(), 12)
    for t in range(4):
        sm = torch.softmax(torch.tensor(logits[t]), 0).numpy()
        assert np.allclose(wts[t], sm[ids[t]], rtol=0, atol=1e-15)
        assert sorted(ids[t].tolist()) == list(range(12))


def pin_router_zipf(o):
    """Zero router weights and the Zipf(1.1) bias: w_e / w_0 = (e + 1)^-1.1."""
    E = 32
    b = workloads.router_bias("zipf1.1", E).numpy()
    x = np.ones((1, 4), dtype=np.float32)
    w = exact_bf16_bits([[0.0] * 4] * E)
    ids, wts, _ = o.route(x, w, b, E)
    assert ids[0].tolist() == list(range(E))
    ratio = wts[0] / wts[0][0]
    ref = np.array([(e + 1.0) ** -1.1 for e in range(E)])
    assert np.allclose(ratio, ref, rtol=2e-6, atol=0)


def pin_router_bias_pull(o):
    """+8 on experts 0..15 moves every pick there (the load-imbalanced input)."""
    wl = workloads.WORKLOADS["imbalanced"]
    wts = workloads.make_weights(wl, H=128, I=8, seed=7)
    x = workloads.make_x(wl, 64, H=128, seed=7)
    ids, _, _ = o.route(workloads.bits(x), workloads.bits(wts["w_router"]),
                        wts["bias"].numpy(), wl.top_k)
    assert ids.max() < 16 and ids.min() >= 0


# --------------------------------------------------------------------------- expert
def _hand_expert():
    g = golden("swiglu_hand.json")
    return (g, np.array(g["x"]), exact_bf16_bits(g["w_gate"]), exact_bf16_bits(g["w_up"]),
            exact_bf16_bits(g["w_down"]))


def pin_router_sigmoid_closed_forms(o):
    g = golden("router_sigmoid_closed_forms.json")
    for case in g["cases"]:
        E = len(case["logits"])
        x = np.ones((1, 1), dtype=np.float32)
        w = exact_bf16_bits([[float(v)] for v in case["logits"]])
        b = None if case["bias"] is None else np.array(case["bias"], dtype=np.float64)
        ids, wts, keys, scores = o.route_sigmoid(x, w, b, case["top_k"],
                                                 normalize=case["normalize"], scale=case["scale"])
        assert ids[0].tolist() == case["ids"], (case["what"], ids[0])
        ref = np.array([float(v) for v in case["weights"]])
        assert np.allclose(wts[0], ref, rtol=1e-15, atol=1e-27), (case["what"], wts[0], ref)


def pin_router_sigmoid_vs_softmax_and_library(o):
    """No bias: the sigmoid router picks what the softmax router picks (the
    sigmoid is strictly increasing), and its scores are torch.sigmoid of the
    same fp64 logits; the raw weights are those scores, the normalised ones
    sum to the scale."""
    for seed in range(4):
        x, w, _ = _tiny_router_case(20 + seed, T=5, H=24, E=10, with_bias=False)
        k = 4
        ids_sm, _, logits = o.route(workloads.bits(x), workloads.bits(w), None, k)
        ids, wts, keys, scores = o.route_sigmoid(workloads.bits(x), workloads.bits(w), None, k)
        assert np.array_equal(ids, ids_sm), (seed, ids, ids_sm)
        ref = torch.sigmoid(torch.tensor(logits, dtype=torch.float64)).numpy()
        assert np.allclose(scores, ref, rtol=1e-15, atol=0), seed
        assert np.array_equal(keys, scores)
        for t in range(x.shape[0]):
            assert np.allclose(wts[t], ref[t][ids[t]], rtol=1e-15, atol=0)
        ids_n, wts_n, _, _ = o.route_sigmoid(workloads.bits(x), workloads.bits(w), None, k,
                                             normalize=True, scale=2.0)
        assert np.array_equal(ids_n, ids)
        assert np.allclose(wts_n.sum(axis=1), 2.0, rtol=1e-15, atol=0)
        assert np.allclose(wts_n, 2.0 * wts / wts.sum(axis=1, keepdims=True), rtol=1e-15, atol=0)


def pin_swiglu_hand(o):
    g, x, wg, wu, wd = _hand_expert()
    f = o.expert_swiglu(x, wg, wu, wd)
    ref = np.array([float(v) for v in g["f"]])
    assert np.allclose(f, ref, rtol=1e-15, atol=0), (f, ref)


def pin_swiglu_routed_hand(o):
    g, x, wg, wu, wd = _hand_expert()
    zeros = exact_bf16_bits([[0.0, 0.0], [0.0, 0.0]])
    w_gate = {0: zeros, 1: wg}
    w_up = {0: zeros, 1: wu}
    w_down = {0: zeros, 1: wd}
    xf = np.array([g["x"]], dtype=np.float32)
    ids = np.array([[1]], dtype=np.int32)
    wts = np.array([[0.75]])
    y = o.moe_ffn_monolith(xf, ids, wts, w_gate, w_up, w_down, 2)
    ref = np.array([float(v) for v in g["routed"]["y_routed_only"]])
    assert np.allclose(y[0], ref, rtol=1e-15, atol=0), (y, ref)
    y = o.moe_ffn_monolith(xf, ids, wts, w_gate, w_up, w_down, 2, shared=(wg, wu, wd))
    ref = np.array([float(v) for v in g["routed"]["y_with_shared"]])
    assert np.allclose(y[0], ref, rtol=1e-15, atol=0), (y, ref)


def _dense_swiglu_torch(x64, wg, wu, wd):
    g = x64 @ _bf16_to_f64(wg).T
    u = x64 @ _bf16_to_f64(wu).T
    return (F.silu(g) * u) @ _bf16_to_f64(wd).T


def pin_dense_swiglu_library(o):
    """E = 1, top_k = 1: the routed FFN is a dense SwiGLU FFN (torch, float64)."""
    wl = workloads.WORKLOADS["tiny"]
    wts = workloads.make_weights(wl, H=64, E=1, I=48, I_s=0, seed=3)
    x = workloads.make_x(wl, 5, H=64, seed=3)
    ids = np.zeros((5, 1), dtype=np.int32)
    w1 = np.ones((5, 1))
    wg, wu, wd = (workloads.bits(wts[k]) for k in ("w_gate", "w_up", "w_down"))
    y = o.moe_ffn_monolith(workloads.bits(x), ids, w1, wg, wu, wd, 1)
    ref = _dense_swiglu_torch(x.to(torch.float64), wg[0], wu[0], wd[0]).numpy()
    assert np.allclose(y, ref, rtol=0, atol=1e-12 * np.abs(ref).max())


def pin_shared_additive(o):
    """The shared expert enters after the routed sum: y(with) - y(without) = f_s."""
    wl = workloads.WORKLOADS["tiny"]
    wts = workloads.make_weights(wl, H=64, E=8, I=32, I_s=40, seed=5)
    x = workloads.make_x(wl, 6, H=64, seed=5)
    xb = workloads.bits(x)
    ids, w, _ = o.route(xb, workloads.bits(wts["w_router"]), None, 3)
    wg, wu, wd = (workloads.bits(wts[k]) for k in ("w_gate", "w_up", "w_down"))
    sh = tuple(workloads.bits(wts[k]) for k in ("ws_gate", "ws_up", "ws_down"))
    y0 = o.moe_ffn_monolith(xb, ids, w, wg, wu, wd, 8)
    y1 = o.moe_ffn_monolith(xb, ids, w, wg, wu, wd, 8, shared=sh)
    fs = _dense_swiglu_torch(x.to(torch.float64), *sh).numpy()
    assert np.allclose(y1 - y0, fs, rtol=0, atol=1e-12 * np.abs(fs).max())


# ------------------------------------------------------------------ fold and bands
def _fold_case(o, band_start, with_shared):
    g = golden("fold_order.json")
    one_gate = exact_bf16_bits([[8192.0]])
    one_up = exact_bf16_bits([[2.0 ** -13]])
    w_gate = np.stack([one_gate] * 4)
    w_up = np.stack([one_up] * 4)
    w_down = np.stack([exact_bf16_bits([[v]]) for v in g["w_down"]])
    x = np.ones((1, 1), dtype=np.float32)
    ids = np.array([g["ids"]], dtype=np.int32)
    wts = np.ones((1, 4))
    shared = (one_gate, one_up, exact_bf16_bits([[0.5]])) if with_shared else None
    if band_start is None:
        return o.moe_ffn_monolith(x, ids, wts, w_gate, w_up, w_down, 4, shared=shared)
    return o.moe_ffn_expert_parallel(x, ids, wts, w_gate, w_up, w_down, 4,
                                     np.array(band_start), shared=shared)


def pin_fold_order(o):
    g = golden("fold_order.json")
    for case in g["expected"]:
        for with_shared, key in ((False, "y"), (True, "y_with_shared")):
            y = _fold_case(o, case["band_start"], with_shared)
            assert y[0, 0] == case[key], (case["band_start"], with_shared, y[0, 0], case[key])


def _tiny_forward(o, seed=0):
    wl = workloads.WORKLOADS["tiny"]
    wts = workloads.make_weights(wl, seed=seed)
    x = workloads.make_x(wl, 4, seed=seed)
    xb = workloads.bits(x)
    ids, w, _ = o.route(xb, workloads.bits(wts["w_router"]), None, wl.top_k)
    mats = tuple(workloads.bits(wts[k]) for k in ("w_gate", "w_up", "w_down"))
    sh = tuple(workloads.bits(wts[k]) for k in ("ws_gate", "ws_up", "ws_down"))
    return wl, xb, ids, w, mats, sh


def pin_ep_invariants(o):
    """Gate table of the fak expert-parallel note, on the tiny workload."""
    wl, xb, ids, w, mats, sh = _tiny_forward(o)
    mono = o.moe_ffn_monolith(xb, ids, w, *mats, wl.E, shared=sh)
    one = o.moe_ffn_expert_parallel(xb, ids, w, *mats, wl.E, o.expert_parallel_plan(wl.E, 1),
                                    shared=sh)
    assert np.array_equal(one, mono), "EP(ranks=1) must equal the monolith bit for bit"
    scale = np.abs(mono).max()
    for R in (2, 4, 8, 16):
        yr = o.moe_ffn_expert_parallel(xb, ids, w, *mats, wl.E, o.expert_parallel_plan(wl.E, R),
                                       shared=sh)
        assert np.abs(yr - mono).max() <= 1e-12 * scale, R
        cos = float((yr * mono).sum() / np.sqrt((yr * yr).sum() * (mono * mono).sum()))
        assert abs(cos - 1.0) < 1e-14


def pin_imbalanced(o):
    """All picks on band 0 of 4: ranks=4 equals ranks=1 bit for bit."""
    wl = workloads.WORKLOADS["imbalanced"]
    wts = workloads.make_weights(wl, H=64, I=16, seed=9)
    x = workloads.make_x(wl, 24, H=64, seed=9)
    xb = workloads.bits(x)
    ids, w, _ = o.route(xb, workloads.bits(wts["w_router"]), wts["bias"].numpy(), wl.top_k)
    plan4 = o.expert_parallel_plan(wl.E, 4)
    assert ids.max() < plan4[1], "every pick must land in band 0"
    mats = tuple(workloads.bits(wts[k]) for k in ("w_gate", "w_up", "w_down"))
    y4 = o.moe_ffn_expert_parallel(xb, ids, w, *mats, wl.E, plan4)
    y1 = o.moe_ffn_expert_parallel(xb, ids, w, *mats, wl.E, o.expert_parallel_plan(wl.E, 1))
    y2 = o.moe_ffn_expert_parallel(xb, ids, w, *mats, wl.E, o.expert_parallel_plan(wl.E, 2))
    assert np.array_equal(y4, y1) and np.array_equal(y2, y1)


def pin_fail_closed(o):
    wl, xb, ids, w, mats, sh = _tiny_forward(o)
    bad_plans = [np.array([0, 8]),            # plan over 8 experts, E = 16
                 np.array([0, 8, 4, 16]),     # not monotone
                 np.array([0, 16, 17])]       # runs past E
    for plan in bad_plans:
        try:
            o.moe_ffn_expert_parallel(xb, ids, w, *mats, wl.E, plan, shared=sh)
        except OracleError:
            continue
        raise AssertionError(f"plan {plan} not refused")
    bad = ids.copy()
    bad[0, 0] = wl.E
    try:
        o.moe_ffn_monolith(xb, bad, w, *mats, wl.E, shared=sh)
    except OracleError:
        return
    raise AssertionError("id out of range not refused")


ALL_PINS = [pin_plan_shares, pin_plan_refused, pin_router_brute_force, pin_router_closed_forms,
            pin_router_full_softmax, pin_router_zipf, pin_router_bias_pull,
            pin_router_sigmoid_closed_forms, pin_router_sigmoid_vs_softmax_and_library,
            pin_swiglu_hand,
            pin_swiglu_routed_hand, pin_dense_swiglu_library, pin_shared_additive,
            pin_fold_order, pin_ep_invariants, pin_imbalanced, pin_fail_closed]
