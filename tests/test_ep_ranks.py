"""ep_forward's exchanges on the CPU, as two and three gloo ranks.

The compute steps are stand-ins (the CUDA kernels need a GPU) that keep the
arithmetic the exchanges must preserve: a rank's partial is the host fp32
fold of its band's picks in ascending (expert id, slot), and the combine is
the rank-order left fold of the bands that hold a valid pick of the token,
then + the shared expert's output (moe_ep_combine's definition).  The
contributions use fp32 values where the order of the sum shows (2^24 + 1 is
a rounding tie), so a slice folded out of rank order, a row slice sent to the
wrong rank or a shared-expert row taken from the wrong slice changes the bits.
Both exchanges ("reduce_scatter": all-to-all of row slices, fold, all-gather;
"all_gather": every partial to every rank) must give every rank the same y,
equal bit for bit to the single-process band form.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HERE = os.path.dirname(os.path.abspath(__file__))

E, H = 8, 5
BIG = 2.0 ** 24
# D[e]: the output of expert e for every token (before its routing weight)
D = np.array([[BIG, 1.0, 0.5, 1.0, 2.0],
              [1.0, BIG, 0.25, -1.0, 2.0],
              [1.0, -BIG, 2.0, 1.0, -2.0],
              [-BIG, 1.0, 4.0, 3.0, 1.0],
              [BIG, 1.0, 1.0, -BIG, 0.5],
              [1.0, 1.0, -BIG, 1.0, 0.25],
              [1.0, -BIG, BIG, 1.0, 8.0],
              [-BIG, 1.0, 1.0, BIG, 1.0]], dtype=np.float32)
NONE = -(1 << 31)
IDS = np.array([[3, 1, 0, 2],
                [7, 4, 0, 5],
                [1, 3, 1, 0],
                [6, -1, 2, 5],
                [4, 4, 4, 4],
                [NONE, 0, 7, 3],
                [2, 6, 1, NONE],
                [7, 5, 1, 0]], dtype=np.int32)
W = np.array([[1, 1, 1, 1], [1, 2, 1, 1], [1, 1, 2, 1], [1, 1, 1, 4], [1, 2, 1, 1],
              [1, 1, 1, 1], [2, 1, 1, 1], [1, 1, 1, 1]], dtype=np.float32)
T = IDS.shape[0]


def _plan(bands):
    from expert_decode_b200.api import Plan
    p = Plan()
    p.num_experts = E
    p.bands = len(bands) - 1
    for r, s in enumerate(bands):
        p.band_start[r] = s
    return p


def _band_partial(ids, w, lo, hi):
    out = np.zeros((ids.shape[0], H), dtype=np.float32)
    for t in range(ids.shape[0]):
        js = sorted((j for j in range(ids.shape[1]) if lo <= ids[t, j] < hi),
                    key=lambda j: (ids[t, j], j))
        if js:
            acc = w[t, js[0]] * D[ids[t, js[0]]]
            for j in js[1:]:
                acc = acc + w[t, j] * D[ids[t, j]]
            out[t] = acc
    return out


class _StandIns:
    @staticmethod
    def partial(x, ids, weights, w_gate, w_up, w_down, plan, rank):
        lo, hi = plan.band_start[rank], plan.band_start[rank + 1]
        return torch.from_numpy(_band_partial(ids.numpy(), weights.numpy(), lo, hi))

    @staticmethod
    def shared(x, ws_gate, ws_up, ws_down):
        return x * 0.5

    @staticmethod
    def combine(partials, ids, plan, shared):
        parts = partials.numpy()
        ids = ids.numpy()
        y = np.zeros((ids.shape[0], H), dtype=np.float32)
        starts = [plan.band_start[r] for r in range(plan.bands + 1)]
        for t in range(ids.shape[0]):
            acc = None
            for r in range(plan.bands):
                if any(starts[r] <= e < starts[r + 1] for e in ids[t]):
                    acc = parts[r, t].copy() if acc is None else acc + parts[r, t]
            if acc is not None:
                y[t] = acc
        y = torch.from_numpy(y)
        return y if shared is None else y + shared


def _x():
    return torch.arange(T * H, dtype=torch.float32).view(T, H) * 0.25


def _reference(bands):
    """Single-process band form: every band's partial, the rank-order fold."""
    plan = _plan(bands)
    parts = torch.stack([_StandIns.partial(None, torch.from_numpy(IDS), torch.from_numpy(W),
                                           None, None, None, plan, r) for r in range(plan.bands)])
    return _StandIns.combine(parts, torch.from_numpy(IDS), plan, _StandIns.shared(_x(), 0, 0, 0))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, bands, out_path):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from expert_decode_b200 import ep
        plan = _plan(bands)
        for exchange in ("reduce_scatter", "all_gather"):
            y = ep.ep_forward(_x(), torch.from_numpy(IDS), torch.from_numpy(W),
                              ("g", "u", "d"), ("sg", "su", "sd"), plan, rank, ops=_StandIns,
                              exchange=exchange)
            np.save(f"{out_path}.{exchange}.{rank}.npy", y.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("bands", [[0, 4, 8], [0, 3, 6, 8]], ids=["2 ranks", "3 ranks"])
def test_ep_forward_exchanges_fold_in_rank_order_on_gloo_ranks(tmp_path, bands):
    world = len(bands) - 1
    out = str(tmp_path / "y")
    mp.spawn(_rank_main, args=(world, _free_port(), bands, out), nprocs=world, join=True)
    want = _reference(bands).numpy()
    for exchange in ("reduce_scatter", "all_gather"):
        for r in range(world):
            got = np.load(f"{out}.{exchange}.{r}.npy")
            assert got.shape == (T, H)
            assert np.array_equal(got.view(np.uint32), want.view(np.uint32)), (exchange, r)


def test_the_fixture_shows_the_order():
    """On the last token (picks 0, 1, 5, 7: 2^24, 1, 1, -2^24 in column 0) the
    band form differs from the monolith's single fold (2 bands: 1 against 0),
    and with 3 bands the rank order differs from the reverse (0 against 1),
    so the test above can fail."""
    shared = _x().numpy()[-1, 0] * 0.5
    mono = _band_partial(IDS, W, 0, E)[-1, 0] + shared
    assert _reference([0, 4, 8]).numpy()[-1, 0] == 1.0 + shared
    assert mono == 0.0 + shared
    parts = [_band_partial(IDS, W, lo, hi)[-1, 0] for lo, hi in ((0, 3), (3, 6), (6, 8))]
    assert _reference([0, 3, 6, 8]).numpy()[-1, 0] == 0.0 + shared
    rev = np.float32(np.float32(parts[2] + parts[1]) + parts[0]) + shared
    assert rev == 1.0 + shared


def test_row_slices_follow_the_share_rule():
    sys.path.insert(0, ROOT)
    from expert_decode_b200.ep import row_slices
    assert row_slices(7, 3) == [0, 3, 5, 7]
    assert row_slices(2, 3) == [0, 1, 2, 2]
    assert row_slices(8, 8) == list(range(9))
    assert row_slices(0, 2) == [0, 0, 0]
