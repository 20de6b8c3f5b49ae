"""ep_forward's exchange on the CPU, as two gloo ranks: each rank's partial is
gathered in rank order and every rank folds the same list.  The compute steps
are stand-ins here (the CUDA kernels need a GPU); the gather, its order and
the hand-off to the combine are the code under test."""
import os
import socket
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class _StandIns:
    """Partial of rank r: every value r + 1; combine: rank-order left fold of
    the partials, then + shared; shared: every value 0.5."""
    @staticmethod
    def partial(x, ids, weights, w_gate, w_up, w_down, plan, rank):
        return torch.full((x.shape[0], x.shape[1]), float(rank + 1))

    @staticmethod
    def shared(x, ws_gate, ws_up, ws_down):
        return torch.full((x.shape[0], x.shape[1]), 0.5)

    @staticmethod
    def combine(partials, ids, plan, shared):
        order = [int(p[0, 0].item()) for p in partials]
        y = partials[0].clone()
        for p in partials[1:]:
            y = y + p
        return (y + shared, order)


def _rank_main(rank, world, port, out_path):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from expert_decode_b200 import ep
        from expert_decode_b200.api import Plan
        plan = Plan()
        plan.num_experts, plan.bands = 8, world
        plan.band_start[0], plan.band_start[1], plan.band_start[2] = 0, 4, 8
        x = torch.zeros((3, 5))
        y, order = ep.ep_forward(x, None, None, (None, None, None), ("g", "u", "d"), plan, rank,
                                 ops=_StandIns)
        with open(f"{out_path}.{rank}", "w") as f:
            f.write(f"{order} {y[0, 0].item()} {tuple(y.shape)}\n")
    finally:
        dist.destroy_process_group()


def test_ep_forward_gathers_in_rank_order_on_two_gloo_ranks(tmp_path):
    out = str(tmp_path / "rank")
    mp.spawn(_rank_main, args=(2, _free_port(), out), nprocs=2, join=True)
    lines = [open(f"{out}.{r}").read().strip() for r in range(2)]
    assert lines[0] == lines[1]
    assert lines[0] == "[1, 2] 3.5 (3, 5)"
