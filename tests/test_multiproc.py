"""The N > 1 launch of bench.py on CPU: two ranks under gloo, as
torch.distributed.run would start them (RANK / WORLD_SIZE / MASTER_* in the
environment). The forward pass shards by (batch, head) with no exchange, so the
only multi-rank logic is the barrier around the timed region and the max over
ranks of the step time; both are exercised here."""
import os
import socket
import sys
from pathlib import Path

import pytest
import torch.multiprocessing as mp

ROOT = Path(__file__).resolve().parents[1]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    sys.path.insert(0, str(ROOT))
    import bench

    w, r, _ = bench.dist_setup()
    bench.dist_barrier(w)
    got = bench.dist_max(float(10 * (r + 1)), w)  # rank 0 -> 10, rank 1 -> 20
    bench.dist_barrier(w)
    bench.dist_done(w)
    q.put((r, w, got))


def test_two_gloo_ranks_take_the_max_step_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
            pytest.fail("a rank did not finish")
        assert p.exitcode == 0
    results = sorted(q.get(timeout=10) for _ in range(2))
    assert results == [(0, 2, 20.0), (1, 2, 20.0)]


def test_single_rank_is_identity():
    sys.path.insert(0, str(ROOT))
    import bench

    assert bench.dist_max(3.5, 1) == 3.5
