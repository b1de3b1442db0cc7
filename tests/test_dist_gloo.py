"""The multi-rank bench plumbing on CPU: two gloo ranks, as torchrun would
launch them (RANK / WORLD_SIZE / MASTER_* from the environment)."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench

    d = bench.Dist(world)
    try:
        assert d.rank == rank and d.world == world and d.pg is not None
        d.barrier()
        # each rank reports its own time; every rank must see the slowest one
        m = d.max(10.0 + 5.0 * rank)
        v, step_s = bench.weak_scaling_throughput(d.world, 100, 4, m)

        class A:  # the reference arm runs on rank 0 only; other ranks return at once
            config, tokens, steps, warmup = "tiny", None, 1, 0

        if rank != 0:
            bench.run_reference(A, d)
        d.barrier()
        out.put((rank, m, v, step_s))
    finally:
        d.close()


def test_two_gloo_ranks_max_and_weak_scaling():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(timeout=120)
    codes = [p.exitcode for p in ps]
    for p in ps:
        if p.is_alive():
            p.kill()
    assert codes == [0, 0]
    res = sorted(q.get(timeout=5) for _ in range(2))
    for rank, m, v, step_s in res:
        assert m == 15.0  # max over ranks
        assert v == pytest.approx(2 * 100 * 4 / 0.015)  # all ranks' tokens / the slowest rank's time
        assert step_s == pytest.approx(0.015 / 100)


def test_single_rank_has_no_process_group(monkeypatch):
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    sys.path.insert(0, ROOT)
    import bench

    d = bench.Dist(1)
    assert d.world == 1 and d.pg is None and d.max(3.0) == 3.0
    d.barrier()
    d.close()
