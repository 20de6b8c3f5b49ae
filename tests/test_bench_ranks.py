"""The N > 1 host logic of bench.py on the CPU, as two gloo ranks: the
whole-job throughput is every rank's tokens over the slowest rank's time, and
the reference arm does no work on ranks other than 0."""
import importlib.util
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_path):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        b = _bench()
        # rank r ran 13 * 10 tokens in (1 + r) seconds
        value, slowest = b.whole_job_throughput(130, 1.0 + rank, dist, "cpu")
        # the reference arm returns at once on ranks other than 0
        returned = None
        if rank != 0:
            returned = b.run_reference(None, None)
        dist.barrier()
        with open(f"{out_path}.{rank}", "w") as f:
            f.write(f"{value} {slowest} {returned}\n")
    finally:
        dist.destroy_process_group()


def test_whole_job_throughput_over_two_gloo_ranks(tmp_path):
    port = _free_port()
    out = str(tmp_path / "rank")
    mp.spawn(_rank_main, args=(2, port, out), nprocs=2, join=True)
    for rank in range(2):
        value, slowest, returned = open(f"{out}.{rank}").read().split()
        assert float(slowest) == 2.0
        assert float(value) == pytest.approx(2 * 130 / 2.0, rel=0, abs=1e-12)
        assert returned == "None"


def test_whole_job_throughput_single_rank():
    b = _bench()
    assert b.whole_job_throughput(130, 2.0) == (65.0, 2.0)


def test_source_digest_ignores_comments_only():
    """The digest that ties profiles/traffic.json to the kernels changes with the
    code and not with comments or white space; literals are kept whole."""
    b = _bench()
    code = 'int f(int a) { return a + 1; } const char *s = "a // b /* c */";'
    commented = ('// leading note\nint f(int a) {  /* inline */ return a + 1; }\n'
                 'const char *s = "a // b /* c */";  // trailing\n')
    assert b._code_only(code) == b._code_only(commented)
    assert b._code_only(code) != b._code_only(code.replace("a + 1", "a + 2"))
    assert '"a // b /* c */"' in b._code_only(commented)
    assert b.source_digest() == b.source_digest()
