"""The fp32 fold-order fixture (tests/golden/fold_order_f32.json): its tensors
and the plain host fp32 folds its expected values follow.

host_fold_f32 restates the summation order the library promises (one left
fold of every valid pick in ascending (expert id, slot), starting from the
first term, then + the shared expert), element by element in numpy float32,
where each addition is one IEEE round-to-nearest-even operation.  It holds no
other arithmetic of the method: the contributions are given to it.
"""
import json
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
FIXTURE = os.path.join(HERE, "golden", "fold_order_f32.json")


def load():
    with open(FIXTURE) as f:
        return json.load(f)


def fold_order(ids_row, E):
    """Slots of one token's valid picks in ascending (expert id, slot)."""
    valid = [j for j, e in enumerate(ids_row) if 0 <= e < E]
    return sorted(valid, key=lambda j: (ids_row[j], j))


def host_fold_f32(contrib, ids, E, shared=None):
    """y[t] = left fold of contrib[t, j] over t's valid picks in ascending
    (id, slot), then + shared[t].  contrib [T, top_k, H] float32."""
    contrib = np.asarray(contrib, dtype=np.float32)
    T, _, H = contrib.shape
    y = np.zeros((T, H), dtype=np.float32)
    for t in range(T):
        order = fold_order([int(e) for e in ids[t]], E)
        if order:
            acc = contrib[t, order[0]].copy()
            for j in order[1:]:
                acc = acc + contrib[t, j]
            y[t] = acc
        if shared is not None:
            y[t] = y[t] + np.asarray(shared[t], dtype=np.float32)
    return y


def host_band_form_f32(contrib, ids, band_start, shared=None):
    """The band form: each band's partial folds its own picks as above, the
    partials of the bands holding a valid pick are left-folded in rank order,
    then + shared."""
    contrib = np.asarray(contrib, dtype=np.float32)
    T, _, H = contrib.shape
    E = band_start[-1]
    y = np.zeros((T, H), dtype=np.float32)
    for t in range(T):
        total = None
        for r in range(len(band_start) - 1):
            lo, hi = band_start[r], band_start[r + 1]
            order = [j for j in fold_order([int(e) for e in ids[t]], E) if lo <= ids[t][j] < hi]
            if not order:
                continue
            part = contrib[t, order[0]].copy()
            for j in order[1:]:
                part = part + contrib[t, j]
            total = part if total is None else total + part
        if total is not None:
            y[t] = total
        if shared is not None:
            y[t] = y[t] + np.asarray(shared[t], dtype=np.float32)
    return y


def contributions(fx):
    """contrib[t, j, r] = weights[t][j] * D[ids[t][j]][r] (exact in fp32 here)."""
    D = np.asarray(fx["D"], dtype=np.float32)
    ids = fx["ids"]
    w = np.asarray(fx["weights"], dtype=np.float32)
    T, k = len(ids), len(ids[0])
    c = np.zeros((T, k, D.shape[1]), dtype=np.float32)
    for t in range(T):
        for j in range(k):
            c[t, j] = w[t, j] * D[ids[t][j]]
    return c


def tensors(fx):
    """The fixture's weights as float32 arrays: x [T, H], w_gate / w_up [E, I, H],
    w_down [E, H, I], shared (gate, up, down)."""
    D = np.asarray(fx["D"], dtype=np.float32)
    S = np.asarray(fx["S"], dtype=np.float32)
    E, H = D.shape
    I = H
    T = len(fx["ids"])
    x = np.zeros((T, H), dtype=np.float32)
    x[:, 0] = 1.0
    wg = np.zeros((E, I, H), dtype=np.float32)
    wu = np.zeros((E, I, H), dtype=np.float32)
    wd = np.zeros((E, H, I), dtype=np.float32)
    wg[:, 0, 0] = 128.0
    wu[:, 0, 0] = 2.0 ** -7
    wd[:, :, 0] = D
    sg = np.zeros((I, H), dtype=np.float32)
    su = np.zeros((I, H), dtype=np.float32)
    sd = np.zeros((H, I), dtype=np.float32)
    sg[0, 0] = 128.0
    su[0, 0] = 2.0 ** -7
    sd[:, 0] = S
    return x, wg, wu, wd, (sg, su, sd)
