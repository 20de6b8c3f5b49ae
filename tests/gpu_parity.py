"""Helpers of the GPU parity tests: seeded inputs on the device, host copies for
the oracle, and the comparisons with the tolerances the tests state.

Tolerances.
  ids      equal to the oracle's, except where the oracle's own fp64 logits of
           the two experts involved lie within TIE_EPS of each other (a tie
           within 1e-6: either order is correct, and the rest must still be a
           valid top-k).
  weights  |w_gpu - w_oracle| <= WEIGHT_TOL.  Both sides decide on fp64
           logits; the GPU rounds the fp64 weight to fp32 once (<= 2^-24
           relative), so 1e-6 absolute is generous.
  y        max |y_gpu - y_oracle| <= Y_REL_TOL * max |y_oracle| (bf16 weights,
           fp32 accumulation), reported per output column (worst columns).
"""
import numpy as np
import torch

import workloads
import expert_decode_b200 as ed

TIE_EPS = 1e-6
WEIGHT_TOL = 1e-6
Y_REL_TOL = 1e-2


def device_inputs(wl, T, seed=workloads.SEED_BASE, batch=0, **sizes):
    W = workloads.make_weights(wl, device="cuda", seed=seed, **sizes)
    x = workloads.make_x(wl, T, device="cuda", seed=seed, batch=batch,
                         H=sizes.get("H"), x_dtype=sizes.get("x_dtype"))
    return W, x


def shared_of(W):
    return None if W["ws_gate"] is None else (W["ws_gate"], W["ws_up"], W["ws_down"])


def host_shared(W):
    s = shared_of(W)
    return None if s is None else tuple(workloads.bits(t) for t in s)


def oracle_route(o, x, W, top_k, rows=None, threads=8):
    xh = workloads.bits(x if rows is None else x[rows])
    b = None if W["bias"] is None else W["bias"].cpu().numpy()
    return o.route(xh, workloads.bits(W["w_router"]), b, top_k, threads=threads)


def check_route(ids_gpu, w_gpu, ids_ref, w_ref, logits_ref):
    """Returns the number of tokens excused by a tie within TIE_EPS."""
    ids_gpu = ids_gpu.cpu().numpy()
    w_gpu = w_gpu.cpu().numpy().astype(np.float64)
    excused = 0
    for t in range(ids_ref.shape[0]):
        if np.array_equal(ids_gpu[t], ids_ref[t]):
            err = np.abs(w_gpu[t] - w_ref[t]).max()
            assert err <= WEIGHT_TOL, (t, err, w_gpu[t], w_ref[t])
            continue
        lt = logits_ref[t]
        # a tie: each differing position swaps experts whose logits agree within TIE_EPS
        for j in range(ids_ref.shape[1]):
            a, b = ids_gpu[t, j], ids_ref[t, j]
            assert 0 <= a < lt.shape[0], (t, j, a)
            assert abs(lt[a] - lt[b]) <= TIE_EPS, (t, j, a, b, lt[a], lt[b])
        assert len(set(ids_gpu[t].tolist())) == ids_gpu.shape[1]
        excused += 1
    return excused


def check_y(y_gpu, y_ref, rel_tol=Y_REL_TOL, what=""):
    y = y_gpu.detach().cpu().double().numpy()
    assert np.all(np.isfinite(y)), f"{what}: non-finite output"
    scale = np.abs(y_ref).max()
    col_err = np.abs(y - y_ref).max(axis=0)
    worst = np.argsort(col_err)[::-1][:4]
    msg = (f"{what}: max|dy| = {col_err.max():.3e} vs max|y| = {scale:.3e} "
           f"(rel {col_err.max() / scale:.3e}); worst columns "
           + ", ".join(f"{c}:{col_err[c]:.2e}" for c in worst))
    print(msg)
    assert col_err.max() <= rel_tol * scale, msg
    return col_err.max() / scale


def oracle_ffn(o, x, ids, weights, W, bands=None, rows=None, threads=8):
    """fp64 oracle on host copies.  ids / weights are the arrays both sides got."""
    xh = workloads.bits(x if rows is None else x[rows])
    ids_h = ids if isinstance(ids, np.ndarray) else ids.cpu().numpy()
    w_h = weights if isinstance(weights, np.ndarray) else weights.cpu().double().numpy()
    if rows is not None:
        ids_h, w_h = ids_h[rows], w_h[rows]
    E = W["w_gate"].shape[0]
    used = sorted(set(int(e) for e in ids_h.ravel() if 0 <= e < E))
    mats = tuple({e: workloads.bits(W[k][e]) for e in used} for k in ("w_gate", "w_up", "w_down"))
    sh = host_shared(W)
    if bands is None:
        return o.moe_ffn_monolith(xh, ids_h, w_h, *mats, E, shared=sh, threads=threads)
    return o.moe_ffn_expert_parallel(xh, ids_h, w_h, *mats, E, np.asarray(bands), shared=sh,
                                     threads=threads)


def oracle_ffn_rows(o, x, ids, weights, W, rows, chunk=8, threads=8):
    """oracle_ffn on the given rows, `chunk` rows per oracle call so that the
    host copies of the experts they pick stay bounded (a few GB)."""
    rows = np.asarray(rows)
    parts = [oracle_ffn(o, x, ids, weights, W, rows=rows[i:i + chunk], threads=threads)
             for i in range(0, len(rows), chunk)]
    return np.concatenate(parts, axis=0)


def spread_rows(ids, E, n_min=64, n_tile=256):
    """Rows (tokens) that cover the grouped GEMMs' tiling of this batch:
      * for the three most-picked experts, the first and last token of every
        n_tile-row N tile of the expert's group (rows in (token, slot) order);
      * for every group-size class of the activation boxes (1-32, 33-64,
        65-128, 129-256, more), the first and last token of one expert of
        that class, and of the least-picked expert present;
      * the first and last tokens, and an even spread up to n_min rows."""
    ids = np.asarray(ids)
    T, k = ids.shape
    flat = ids.reshape(-1)
    groups = {}
    for p, e in enumerate(flat.tolist()):
        if 0 <= e < E:
            groups.setdefault(e, []).append(p // k)
    picked = {0, T - 1}
    by_size = sorted(groups, key=lambda e: (-len(groups[e]), e))
    for e in by_size[:3]:
        toks = groups[e]
        for n0 in range(0, len(toks), n_tile):
            picked.add(toks[n0])
            picked.add(toks[min(n0 + n_tile, len(toks)) - 1])
    classes = [(1, 32), (33, 64), (65, 128), (129, 256), (257, 1 << 30)]
    for lo, hi in classes:
        for e in sorted(groups):
            if lo <= len(groups[e]) <= hi:
                picked.update((groups[e][0], groups[e][-1]))
                break
    if by_size:
        last = by_size[-1]
        picked.update((groups[last][0], groups[last][-1]))
    step = max(1, T // n_min)
    t = 0
    while len(picked) < min(n_min, T):
        picked.add(t % T)
        t += step
        if t >= T:
            t = t % T + 1
    return np.array(sorted(picked))


def gpu_ffn(x, ids, weights, W, plan, **kw):
    y = ed.moe_ffn_forward(x, ids, weights, W["w_gate"], W["w_up"], W["w_down"], shared_of(W),
                           plan, **kw)
    torch.cuda.synchronize()
    return y
